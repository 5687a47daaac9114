// Shared-prefix decode (sm_100a): sequences forked from one prompt (parallel sampling, a
// common system prompt) share the physical blocks of that prompt ("深入解析
// PagedAttention", 多序列共享; "什么是 LLM 中的分页注意力", 跨请求的内存共享: the requests
// point at the same blocks instead of storing two copies).  Plain paged decode still reads
// those shared blocks once per sequence.  This kernel reads them once per group.
//
// The result is exactly plain attention per (sequence, query head).
//
// Units (laid end to end, balanced over warp streams as in decode_stream.cu):
//   * group row r < ngroups, KV head h: the Q rows are the members' query heads of KV head
//     h stacked (members x G <= 16 MMA rows).  Its tiles are first the shared tokens
//     [0, prefix_r), read once through the first member's table for all rows, then each
//     member's own tokens [prefix_r, L_m) through that member's table, with every other
//     member's rows masked out of the online softmax.  The unit ends with each member's
//     complete softmax, so it writes the members' outputs itself;
//   * sequence row ngroups + b, KV head h, for an ungrouped sequence b: [0, L_b).
// Units cut by a stream boundary leave partials that the cut-unit reduce merges by
// log-sum-exp (a piece may hold no tile of some member's rows: its max is -inf and it is
// skipped).

#include <cudaTypedefs.h>

#include "pa_device.cuh"
#include "pa_internal.h"
#include "tc_tile.cuh"

namespace pa {

namespace {

constexpr unsigned kFull = 0xffffffffu;
// As in decode_stream.cu: 16-token stages (half of a 32-token block each), 4 warps per
// CTA and 2 CTAs per SM, so every SM sub-partition runs two streams.  Shared prefixes
// are multiples of PA_SHARED_PREFIX_ALIGN tokens, so no stage straddles a prefix end.
constexpr int kNCW = 4;                 // warps (= streams) per CTA
constexpr int kThreads = kNCW * 32;
constexpr int kMinCtas = 2;             // CTAs per SM the register allocation allows
constexpr int kSPW = 2;                 // ring stages per stream
constexpr int kRows = 16;               // MMA rows of a unit (members x G of a group)
constexpr int kTT = 16;                 // tokens per stage
static_assert(PA_SHARED_PREFIX_ALIGN % kTT == 0, "a prefix ends on a stage boundary");

template <int D_, int BS_>
struct PrefCfg : TileCfg<D_, BS_, true, kTT, true> {
  static constexpr int SPW = kSPW;
  static constexpr int NST = kNCW * SPW;
  static constexpr int RING_BYTES = NST * PrefCfg::STAGE_BYTES;
  static constexpr int Q_BYTES = WarpAcc<PrefCfg, true>::Q_BYTES;
  // two Q tiles per warp: the next unit's rows are copied in while the current streams
  static constexpr int FIXED_BYTES = RING_BYTES + kNCW * 2 * Q_BYTES;
};

template <class C>
size_t pref_smem_bytes(int R) {
  return C::FIXED_BYTES + 1024 + static_cast<size_t>(R + 1) * 4;
}

__device__ __forceinline__ int clamp_len(const DecodeParams& p, int b, bool flag) {
  int L = __ldg(p.seq_lens + b);
  const int Lmax = p.max_blocks * p.block_size;
  if (L < 0 || L > Lmax) {
    if (flag) flag_error(p.err, PA_DEVERR_BAD_SEQ_LEN);
    L = L < 0 ? 0 : Lmax;
  }
  return L;
}

__device__ __forceinline__ int upper_bound(const int* P, int n, int v) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (P[mid] > v) hi = mid; else lo = mid + 1;
  }
  return lo;
}

// Group of batch row b (-1 if none or out of range: flagged, then treated as ungrouped).
__device__ __forceinline__ int group_of(const PrefixParams& pp, int b, bool flag) {
  const int g = __ldg(pp.group_of + b);
  if (g >= pp.ngroups || g < -1) {
    if (flag) flag_error(pp.d.err, PA_DEVERR_BAD_SEQ_LEN);
    return -1;
  }
  return g;
}

__device__ __forceinline__ int member_of(const PrefixParams& pp, int r, int m) {
  return __ldg(pp.group_members + static_cast<size_t>(r) * pp.max_members + m);
}

// Members of group r (up to max_members batch rows, -1 padded at the end).
__device__ __forceinline__ int group_size(const PrefixParams& pp, int r) {
  int n = 0;
  while (n < pp.max_members && member_of(pp, r, n) >= 0) ++n;
  return n;
}

// Shared tokens of group r; -1 for a malformed group (flagged), whose rows then get no
// tile.  A prefix of 0 is valid: the unit streams only the members' own tokens.
__device__ __forceinline__ int group_prefix_tokens(const PrefixParams& pp, int r, bool flag) {
  const int b0 = member_of(pp, r, 0);
  const int pre = __ldg(pp.group_prefix + r);
  if (b0 < 0 || b0 >= pp.d.B || pre < 0 || pre % PA_SHARED_PREFIX_ALIGN != 0) {
    if (flag) flag_error(pp.d.err, PA_DEVERR_BAD_SEQ_LEN);
    return -1;
  }
  return pre;
}

// Own tiles of member m of group r (tokens [pre, L_m)); a member shorter than the prefix is
// flagged and contributes none.
template <int TT>
__device__ __forceinline__ int member_tiles(const PrefixParams& pp, int r, int m, int pre,
                                            bool flag) {
  const int b = member_of(pp, r, m);
  if (b < 0 || b >= pp.d.B) return 0;
  const int L = clamp_len(pp.d, b, flag);
  if (L < pre) {
    if (flag) flag_error(pp.d.err, PA_DEVERR_BAD_SEQ_LEN);
    return 0;
  }
  return (L - pre + TT - 1) / TT;
}

template <int TT>
__device__ __forceinline__ int row_tiles(const PrefixParams& pp, int r, bool flag) {
  if (r < pp.ngroups) {
    const int pre = group_prefix_tokens(pp, r, flag);
    if (pre < 0) return 0;
    // member ids first (independent loads), then their lengths (independent loads)
    int ids[kRows];
#pragma unroll
    for (int m = 0; m < kRows; ++m) ids[m] = m < pp.max_members ? member_of(pp, r, m) : -1;
    int n = pre / TT;
    bool live = true;
#pragma unroll
    for (int m = 0; m < kRows; ++m) {
      live = live && ids[m] >= 0;
      if (live && ids[m] < pp.d.B) {
        const int L = clamp_len(pp.d, ids[m], flag);
        if (L < pre) {
          if (flag) flag_error(pp.d.err, PA_DEVERR_BAD_SEQ_LEN);
        } else {
          n += (L - pre + TT - 1) / TT;
        }
      }
    }
    return n;
  }
  const int b = r - pp.ngroups;
  if (group_of(pp, b, flag) >= 0) return 0;  // covered by its group's unit
  return (clamp_len(pp.d, b, flag) + TT - 1) / TT;
}

// Where tile j of unit row r comes from.
struct TileSrc {
  int table_b;         // batch row whose block table holds the tokens
  int tok0, tok1;      // tile starts at tok0; the run of tokens ends at tok1
  int row_lo, row_hi;  // MMA rows that take part
};

template <int TT>
__device__ __forceinline__ TileSrc tile_src(const PrefixParams& pp, int r, int j) {
  TileSrc t;
  if (r >= pp.ngroups) {
    const int b = r - pp.ngroups;
    t.table_b = b;
    t.tok0 = j * TT;
    t.tok1 = clamp_len(pp.d, b, false);
    t.row_lo = 0;
    t.row_hi = 16;
    return t;
  }
  const int pre = max(group_prefix_tokens(pp, r, false), 0);
  const int np = pre / TT;
  if (j < np) {
    t.table_b = member_of(pp, r, 0);
    t.tok0 = j * TT;
    t.tok1 = pre;
    t.row_lo = 0;
    t.row_hi = 16;
    return t;
  }
  int k = j - np;
  const int gs = group_size(pp, r);
  for (int m = 0; m < gs; ++m) {
    const int n = member_tiles<TT>(pp, r, m, pre, false);
    if (k < n) {
      const int b = member_of(pp, r, m);
      t.table_b = b;
      t.tok0 = pre + k * TT;
      t.tok1 = clamp_len(pp.d, b, false);
      t.row_lo = m * pp.d.G;
      t.row_hi = (m + 1) * pp.d.G;
      return t;
    }
    k -= n;
  }
  t.table_b = member_of(pp, r, 0);  // not reached for j < row_tiles
  t.tok0 = t.tok1 = 0;
  t.row_lo = t.row_hi = 0;
  return t;
}

struct TilePos {
  int r, kvh, j, nt;
};

__device__ __forceinline__ TilePos locate(const int* P, int R, int Hkv, int g) {
  TilePos t;
  t.r = upper_bound(P, R + 1, g / Hkv) - 1;
  t.nt = P[t.r + 1] - P[t.r];
  const int off = g - Hkv * P[t.r];
  t.kvh = off / t.nt;
  t.j = off - t.kvh * t.nt;
  return t;
}

struct TileIds {
  int kvh, nb, row0;
  int id[4];
};

template <class C>
__device__ __forceinline__ TileIds resolve_tile(const PrefixParams& pp, const int* P, int R, int g,
                                                int end) {
  TileIds out{0, 0, 0, {0, 0, 0, 0}};
  if (g >= end) return out;
  const DecodeParams& p = pp.d;
  const TilePos t = locate(P, R, p.Hkv, g);
  out.kvh = t.kvh;
  const TileSrc s = tile_src<C::TILE_T>(pp, t.r, t.j);
  const int blk = s.tok0 / C::BS;
  out.row0 = s.tok0 % C::BS;  // non-zero only when a stage holds part of a block
  const int nblk = (s.tok1 + C::BS - 1) / C::BS;
  out.nb = min(C::BPS, nblk - blk);
  const int32_t* tab = p.block_tables + static_cast<size_t>(s.table_b) * p.max_blocks + blk;
#pragma unroll
  for (int k = 0; k < C::BPS; ++k)
    if (k < out.nb) out.id[k] = __ldg(tab + k);
  return out;
}

// Batch row and query head of MMA row rr of unit row r (rows < nrows).
__device__ __forceinline__ void row_target(const PrefixParams& pp, int r, int kvh, int rr, int& b,
                                           int& h) {
  const int G = pp.d.G;
  if (r < pp.ngroups) {
    b = member_of(pp, r, rr / G);
    h = kvh * G + rr % G;
  } else {
    b = r - pp.ngroups;
    h = kvh * G + rr;
  }
}

template <class C>
__global__ void __launch_bounds__(kThreads, kMinCtas)
    decode_prefix_kernel(const __grid_constant__ CUtensorMap tmk,
                         const __grid_constant__ CUtensorMap tmv, const PrefixParams pp) {
  constexpr int D = C::D, TILE_T = C::TILE_T, SPW = C::SPW, NST = C::NST;
  const DecodeParams& p = pp.d;
  const int B = p.B, Hkv = p.Hkv, G = p.G, NG = pp.ngroups;
  const int R = NG + B;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* qtiles = smem + C::RING_BYTES;
  int* P = reinterpret_cast<int*>(smem + C::FIXED_BYTES);  // [R + 1] tiles before row r
  __shared__ __align__(8) uint64_t full_bar[NST];

  __shared__ int warp_sum[kNCW];
  if (threadIdx.x == 0) {
    for (int st = 0; st < NST; ++st) mbar_init(smem_addr(&full_bar[st]), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    fence_proxy_async_smem();
  }
  // Launched as a programmatic dependent of the previous kernel on the stream: nothing
  // above reads global memory; wait for that kernel before anything below does.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // ---- tile counts of every unit row, scanned (every CTA, identical): P[r] = tiles of
  // the rows before r, P[R] = total.  Rows first, with their dependent loads (group ->
  // members -> lengths) overlapping across threads, then an in-place scan.
  for (int r = threadIdx.x; r < R; r += kThreads) P[r] = row_tiles<TILE_T>(pp, r, blockIdx.x == 0);
  __syncthreads();
  {
    const int chunk = (R + kThreads - 1) / kThreads;
    const int lo = min(R, static_cast<int>(threadIdx.x) * chunk);
    const int hi = min(R, lo + chunk);
    int sum = 0;
    for (int r = lo; r < hi; ++r) sum += P[r];
    int incl = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(kFull, incl, off);
      if (lane >= off) incl += v;
    }
    if (lane == 31) warp_sum[warp] = incl;
    __syncthreads();
    int run = incl - sum;
    for (int w = 0; w < warp; ++w) run += warp_sum[w];
    for (int r = lo; r < hi; ++r) {
      const int n = P[r];
      P[r] = run;
      run += n;
    }
    if (threadIdx.x == 0) {
      int total = 0;
      for (int w = 0; w < kNCW; ++w) total += warp_sum[w];
      P[R] = total;
    }
  }
  __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out);
  for (int b = blockIdx.x; b < B; b += gridDim.x) {
    if (clamp_len(p, b, false) == 0) {
      uint32_t* row = reinterpret_cast<uint32_t*>(out + static_cast<size_t>(b) * p.Hq * D);
      for (int i = threadIdx.x; i < p.Hq * D / 2; i += kThreads) row[i] = 0u;
    }
  }
  if (threadIdx.x == 0) {
    prefetch_tensormap(&tmk);
    prefetch_tensormap(&tmv);
  }
  __syncthreads();

  const int T = Hkv * P[R];
  const int S = static_cast<int>(gridDim.x) * kNCW;
  const int per = (T + S - 1) / S;
  // Let the cut reduce be launched now; it waits for this grid to complete.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int s = static_cast<int>(blockIdx.x) * kNCW + warp;
  const int beg = min(T, s * per);
  const int end = min(T, beg + per);
  const int cnt = end - beg;
  const uint64_t policy = l2_policy_evict_first();

  TileIds cur = resolve_tile<C>(pp, P, R, beg + lane, end);
  TileIds nxt = resolve_tile<C>(pp, P, R, beg + 32 + lane, end);
  int batch = 0;
  auto issue = [&](int k) {
    if ((k >> 5) != batch) {
      cur = nxt;
      ++batch;
      nxt = resolve_tile<C>(pp, P, R, beg + 32 * (batch + 1) + lane, end);
    }
    const int src = k & 31;
    const int kv = __shfl_sync(kFull, cur.kvh, src);
    const int n = __shfl_sync(kFull, cur.nb, src);
    const int row0 = __shfl_sync(kFull, cur.row0, src);
    int ids[C::BPS];
#pragma unroll
    for (int q = 0; q < C::BPS; ++q) ids[q] = __shfl_sync(kFull, cur.id[q], src);
    if (lane == 0) {
      const int stage = warp * SPW + k % SPW;
      const uint32_t fb = smem_addr(&full_bar[stage]);
      const uint32_t kt = smem_addr(smem + stage * C::STAGE_BYTES);
      const uint32_t vt = kt + C::TILE_BYTES;
      fence_proxy_async_smem();
      mbar_arrive_expect_tx(fb, static_cast<uint32_t>(n * C::BOXR * D * 2 * 2));
#pragma unroll
      for (int sub = 0; sub < C::BPS; ++sub) {
        if (sub >= n) break;
        int phys = ids[sub];
        if (phys < 0 || phys >= p.num_blocks) {
          flag_error(p.err, PA_DEVERR_BAD_BLOCK_ID);
          phys = 0;
        }
#pragma unroll
        for (int c = 0; c < C::DCH; ++c) {
          tma_load_4d(kt + c * C::CHUNK_BYTES + sub * C::BOXR * 128, &tmk, c * 64, kv, row0,
                      phys, fb, policy);
          tma_load_4d(vt + c * C::CHUNK_BYTES + sub * C::BOXR * 128, &tmv, c * 64, kv, row0,
                      phys, fb, policy);
        }
      }
    }
    __syncwarp();
  };
  for (int k = 0; k < SPW && k < cnt; ++k) issue(k);

  const int g = lane >> 2, tig = lane & 3;
  const float sl2 = p.scale_log2;
  // The cut unit this stream owns (it starts in this stream's range and continues past
  // it): unit id, slot of this stream's piece, number of pieces.
  int own_u = -1, own_slot = 0, own_n = 0, own_rows = 0;
  int i = 0;
  bool ok = true;
  WarpAcc<C, true> acc;
  uint8_t* my_q = qtiles + warp * 2 * C::Q_BYTES;
  const __nv_bfloat16* qbase = static_cast<const __nv_bfloat16*>(p.q);
  // A unit's inputs, lane-distributed: a group's member ids (lane m) and shared tokens, or
  // an ungrouped sequence's row; then their lengths.  The next unit's are loaded while
  // the current one streams: ids at its start, lengths after its first tile.
  auto load_ids = [&](const TilePos& u, int& id, int& pre) {
    if (u.r < NG) {
      id = lane < pp.max_members ? member_of(pp, u.r, lane) : -1;
      pre = max(group_prefix_tokens(pp, u.r, false), 0);
    } else {
      id = u.r - NG;
      pre = 0;
    }
  };
  auto load_len = [&](const TilePos& u, int id) {
    if (u.r < NG) return (id >= 0 && id < B) ? clamp_len(p, id, false) : 0;
    return clamp_len(p, id, false);
  };
  // Copy unit u's Q rows into a Q tile with cp.async (rows past the unit's, or of a
  // member id outside [0, B), zero-filled): a group's members' heads of its KV head,
  // or the sequence's.
  auto prefetch_q = [&](const TilePos& u, int id, uint8_t* tile) {
    constexpr int CPR = D * 2 / 16;
    const bool grp = u.r < NG;
    const int gs = grp ? __ffs(~__ballot_sync(kFull, id >= 0)) - 1 : 1;
    const int nrows = grp ? gs * G : G;
    for (int idx0 = 0; idx0 < kRows * CPR; idx0 += 32) {
      const int idx = idx0 + lane;
      const int rr = idx / CPR, c = idx - rr * CPR;
      const int b = __shfl_sync(kFull, id, grp ? (rr < kRows ? rr : 0) / G : 0);
      const bool live = rr < nrows && b >= 0 && b < B;
      const int h = u.kvh * G + (grp ? rr % G : rr);
      const __nv_bfloat16* src = qbase + (live ? (static_cast<size_t>(b) * p.Hq + h) * D : 0);
      if (idx < kRows * CPR)
        cp_async_16_zfill(smem_addr(tile + WarpAcc<C, true>::q_off(rr, c)),
                          reinterpret_cast<const uint4*>(src) + (live ? c : 0), live ? 16 : 0);
    }
    cp_async_commit();
  };

  int gpos = beg;
  int qb = 0;                  // Q tile of the current unit
  TilePos t{};
  int cid = -1, cpre = 0, cL = 0;  // the current unit's inputs
  if (gpos < end) {
    t = locate(P, R, Hkv, gpos);
    load_ids(t, cid, cpre);
    cL = load_len(t, cid);
    prefetch_q(t, cid, my_q);
  }
  while (gpos < end && ok) {
    const int ubeg = Hkv * P[t.r] + t.kvh * t.nt;
    const int uend = ubeg + t.nt;
    const int pend = min(end, uend);
    const int u = t.r * Hkv + t.kvh;
    const bool is_group = t.r < NG;
    // The unit's sources (the same rules as row_tiles / tile_src): for a group, lane
    // m < gs holds member m's batch row mb, length mL and the unit tile mst where its own
    // tokens start (after the np shared tiles); a tile's member is then a ballot, with no
    // global load per tile.  An ungrouped sequence: its row and length.
    int gs = 1, mb = cid, mL = cL, mst = 0x7fffffff;
    const int pre = cpre, np = cpre / TILE_T;
    if (is_group) {
      gs = __ffs(~__ballot_sync(kFull, cid >= 0)) - 1;  // members before the first -1
      const int own = (lane < gs && cid < B && cL >= pre) ? (cL - pre + TILE_T - 1) / TILE_T : 0;
      int incl = own;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(kFull, incl, off);
        if (lane >= off) incl += v;
      }
      if (lane < gs) mst = np + incl - own;
      else mb = -1;
    }
    const int nrows = is_group ? gs * G : G;
    // batch row of MMA row rr (member rr / G of a group, or the sequence)
    auto row_b = [&](int rr) { return __shfl_sync(kFull, mb, is_group ? rr / G : 0); };
    // whether MMA row rr has an output here: a row of length 0 (a member of a group with
    // no shared tokens, or one flagged for being shorter than the prefix) is left to the
    // zero fill of the prologue, which writes every such row and nothing else
    auto row_live = [&](int rr) { return __shfl_sync(kFull, mL, is_group ? rr / G : 0) > 0; };
    // the next unit of this stream (if any) starts at tile pend
    const bool has_next = pend < end;
    TilePos tn{};
    int nid = -1, npre = 0, nL = 0;
    if (has_next) {
      tn = locate(P, R, Hkv, pend);
      load_ids(tn, nid, npre);
    }
    acc.use_q(my_q + qb * C::Q_BYTES);
    acc.reset();
    const int jend = t.j + (pend - gpos);
    for (int j = t.j; j < jend; ++j, ++i) {
      const int stage = warp * SPW + i % SPW;
      if (!mbar_wait_warp(smem_addr(&full_bar[stage]), (i / SPW) & 1, p.err)) {
        ok = false;  // the same in every lane: the warp leaves the loop together
        break;
      }
      int valid, row_lo = 0, row_hi = kRows;
      if (!is_group) {
        valid = min(TILE_T, mL - j * TILE_T);
      } else if (j < np) {
        valid = TILE_T;  // shared tokens: the prefix is a whole number of stages
      } else {
        const unsigned mk = __ballot_sync(kFull, lane < gs && mst <= j);
        const int m = 31 - __clz(mk);
        const int Lm = __shfl_sync(kFull, mL, m), sm = __shfl_sync(kFull, mst, m);
        valid = min(TILE_T, Lm - (pre + (j - sm) * TILE_T));
        row_lo = m * G;
        row_hi = row_lo + G;
      }
      uint8_t* st_ptr = smem + stage * C::STAGE_BYTES;
      if (valid < TILE_T) zero_tail_rows<C>(st_ptr, valid, lane);
      if (is_group)
        acc.template tile<true>(smem_addr(st_ptr), valid, sl2, lane, row_lo, row_hi);
      else
        acc.tile(smem_addr(st_ptr), valid, sl2, lane);
      __syncwarp();
      if (i + SPW < cnt) issue(i + SPW);
      if (j == t.j && has_next) {  // the next unit's ids have landed by now
        nL = load_len(tn, nid);
        prefetch_q(tn, nid, my_q + (qb ^ 1) * C::Q_BYTES);
      }
    }
    if (!ok) break;
    acc.reduce_l();
    const bool complete = (gpos == ubeg) && (pend == uend);
    if (complete) {
      const float inv_lo = 1.f / acc.l_lo, inv_hi = 1.f / acc.l_hi;
      // shuffles first, by every lane; then the per-lane choice
      const int rb0 = row_b(g), rb1 = row_b(g + 8);
      const bool live0 = row_live(g), live1 = row_live(g + 8);
      const int b0 = live0 ? rb0 : -1, b1 = live1 ? rb1 : -1;
      const int h0 = t.kvh * G + (is_group ? g % G : g);
      const int h1 = t.kvh * G + (is_group ? (g + 8) % G : g + 8);
#pragma unroll
      for (int jn = 0; jn < C::NT; ++jn) {
        const size_t col = 8 * jn + 2 * tig;
        if (g < nrows && b0 >= 0 && b0 < B)  // a member id outside [0, B) has no output row
          *reinterpret_cast<uint32_t*>(out + (static_cast<size_t>(b0) * p.Hq + h0) * D + col) =
              pack_bf16x2(acc.o_lo[jn][0] * inv_lo, acc.o_lo[jn][1] * inv_lo);
        if (g + 8 < nrows && b1 >= 0 && b1 < B)
          *reinterpret_cast<uint32_t*>(out + (static_cast<size_t>(b1) * p.Hq + h1) * D + col) =
              pack_bf16x2(acc.o_hi[jn][0] * inv_hi, acc.o_hi[jn][1] * inv_hi);
      }
    } else {
      const int slot = gpos == beg ? 0 : 1;  // a cut piece is the stream's first or last
      const size_t row0 = (static_cast<size_t>(s) * 2 + slot) * kRows;
      if (ubeg >= beg) {  // the unit starts here: its pieces are streams s .. (uend-1)/per
        own_u = u;
        own_slot = slot;
        own_n = (uend - 1) / per - s + 1;
        own_rows = nrows;
      }
      // a row without output gets sum 0 in every piece, so the reduce skips it
      const bool live0 = row_live(g), live1 = row_live(g + 8);
      if (tig == 0) {
        if (g < nrows)
          *reinterpret_cast<float2*>(pp.pml + (row0 + g) * 2) =
              make_float2(acc.m_lo, live0 ? acc.l_lo : 0.f);
        if (g + 8 < nrows)
          *reinterpret_cast<float2*>(pp.pml + (row0 + g + 8) * 2) =
              make_float2(acc.m_hi, live1 ? acc.l_hi : 0.f);
      }
#pragma unroll
      for (int jn = 0; jn < C::NT; ++jn) {
        if (g < nrows)
          *reinterpret_cast<float2*>(pp.pacc + (row0 + g) * D + 8 * jn + 2 * tig) =
              make_float2(acc.o_lo[jn][0], acc.o_lo[jn][1]);
        if (g + 8 < nrows)
          *reinterpret_cast<float2*>(pp.pacc + (row0 + g + 8) * D + 8 * jn + 2 * tig) =
              make_float2(acc.o_hi[jn][0], acc.o_hi[jn][1]);
      }
    }
    gpos = pend;
    t = tn;
    cid = nid;
    cpre = npre;
    cL = nL;
    qb ^= 1;
  }
  cp_async_wait_all();  // a Q copy still in flight after an early exit
  if (!ok) {
    for (int k = i; k < cnt && k < i + SPW; ++k) {
      const int stage = warp * SPW + k % SPW;
      mbar_wait(smem_addr(&full_bar[stage]), (k / SPW) & 1, p.err);
    }
  }
  if (lane == 0) {
    int4 m = make_int4(ok ? own_u : -1, own_slot, own_n, own_rows);
    *reinterpret_cast<int4*>(pp.meta + s * 4) = m;
  }
}

// Merge the pieces of units cut by a stream boundary (as in decode_stream.cu) and write
// the outputs of their rows.  A piece that holds no tile of a row has max -inf and is
// skipped for that row.
template <int D>
__global__ void __launch_bounds__(512) prefix_cut_reduce_kernel(const PrefixParams pp) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const DecodeParams& p = pp.d;
  const int s = blockIdx.x;
  // the unit stream s owns, recorded with the slot of its first piece, the piece count and
  // the unit's rows (no dependent loads of group members here)
  const int4 m = *reinterpret_cast<const int4*>(pp.meta + static_cast<size_t>(s) * 4);
  if (m.x < 0) return;
  const int u = m.x, slot = m.y, n = m.z, nrows = m.w;
  const int r = u / p.Hkv, kvh = u - r * p.Hkv;
  const int row = threadIdx.x / (D / 4);
  const int c = (threadIdx.x % (D / 4)) * 4;
  if (row >= nrows) return;
  int b, h;
  row_target(pp, r, kvh, row, b, h);  // its load overlaps the pieces' loads
  float M = -INFINITY, l = 0.f, a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll 4
  for (int i = 0; i < n; ++i) {
    const size_t pr = (static_cast<size_t>(s + i) * 2 + (i == 0 ? slot : 0)) * kRows + row;
    const float2 ml = *reinterpret_cast<const float2*>(pp.pml + pr * 2);
    const float4 a = *reinterpret_cast<const float4*>(pp.pacc + pr * D + c);
    // no branch (a piece with no tile of this row has max -inf and weight 0), so that the
    // unrolled pieces' loads are all issued up front
    const float Mn = fmaxf(M, ml.x);
    const float so = M == -INFINITY ? 0.f : exp2f(M - Mn);
    const float sn = ml.x == -INFINITY ? 0.f : exp2f(ml.x - Mn);
    l = l * so + ml.y * sn;
    a0 = a0 * so + a.x * sn;
    a1 = a1 * so + a.y * sn;
    a2 = a2 * so + a.z * sn;
    a3 = a3 * so + a.w * sn;
    M = Mn;
  }
  if (b < 0 || b >= p.B || !(l > 0.f)) return;  // no output row, or one left to the zero fill
  __nv_bfloat16* o =
      static_cast<__nv_bfloat16*>(p.out) + (static_cast<size_t>(b) * p.Hq + h) * D + c;
  const float inv = 1.f / l;
  *reinterpret_cast<uint2*>(o) = make_uint2(pack_bf16x2(a0 * inv, a1 * inv),
                                            pack_bf16x2(a2 * inv, a3 * inv));
}

template <class C>
int pref_grid_for(int R, int sms) {
  int occ = 0;
  const size_t smem = pref_smem_bytes<C>(R);
  if (cudaFuncSetAttribute(decode_prefix_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, decode_prefix_kernel<C>, kThreads,
                                                    smem) != cudaSuccess)
    return 0;
  return occ * sms;
}

template <class C>
cudaError_t launch_pref_cfg(PrefixParams pp, int grid, cudaStream_t stream) {
  CUtensorMap tmk, tmv;
  const DecodeParams& p = pp.d;
  if (!make_pool_map(&tmk, p.k_pool, p.num_blocks, C::BS, p.Hkv, C::D, C::BOXR) ||
      !make_pool_map(&tmv, p.v_pool, p.num_blocks, C::BS, p.Hkv, C::D, C::BOXR))
    return cudaErrorInvalidValue;
  const size_t smem = pref_smem_bytes<C>(pp.ngroups + p.B);
  cudaError_t e = cudaFuncSetAttribute(decode_prefix_kernel<C>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  // the main kernel as a programmatic dependent of the previous kernel on the stream,
  // the cut reduce as one of the main kernel
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  if ((e = cudaLaunchKernelEx(&cfg, decode_prefix_kernel<C>, tmk, tmv, pp)) != cudaSuccess) return e;
  cfg.gridDim = dim3(static_cast<unsigned>(pp.streams));
  cfg.blockDim = dim3(kRows * C::D / 4);
  cfg.dynamicSmemBytes = 0;
  return cudaLaunchKernelEx(&cfg, prefix_cut_reduce_kernel<C::D>, pp);
}

}  // namespace

int prefix_grid(int D, int block_size, int R) {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 0;
  switch (D * 100 + block_size) {
    case 6408: return pref_grid_for<PrefCfg<64, 8>>(R, sms);
    case 6416: return pref_grid_for<PrefCfg<64, 16>>(R, sms);
    case 6432: return pref_grid_for<PrefCfg<64, 32>>(R, sms);
    case 12808: return pref_grid_for<PrefCfg<128, 8>>(R, sms);
    case 12816: return pref_grid_for<PrefCfg<128, 16>>(R, sms);
    case 12832: return pref_grid_for<PrefCfg<128, 32>>(R, sms);
    default: return 0;
  }
}

int prefix_warps_per_cta() { return kNCW; }

size_t prefix_workspace_bytes(int streams, int rows, int D) {
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  (void)rows;
  return up(static_cast<size_t>(streams) * 16) + up(static_cast<size_t>(streams) * 2 * kRows * 8) +
         static_cast<size_t>(streams) * 2 * kRows * D * 4;
}

void prefix_carve(PrefixParams* pp, void* workspace, int rows) {
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  char* w = static_cast<char*>(workspace);
  pp->meta = reinterpret_cast<int32_t*>(w);
  w += up(static_cast<size_t>(pp->streams) * 16);
  pp->pml = reinterpret_cast<float*>(w);
  w += up(static_cast<size_t>(pp->streams) * 2 * kRows * 8);
  pp->pacc = reinterpret_cast<float*>(w);
  (void)rows;
}

cudaError_t launch_decode_prefix(const PrefixParams& pp, int grid, cudaStream_t stream) {
  switch (pp.d.D * 100 + pp.d.block_size) {
    case 6408: return launch_pref_cfg<PrefCfg<64, 8>>(pp, grid, stream);
    case 6416: return launch_pref_cfg<PrefCfg<64, 16>>(pp, grid, stream);
    case 6432: return launch_pref_cfg<PrefCfg<64, 32>>(pp, grid, stream);
    case 12808: return launch_pref_cfg<PrefCfg<128, 8>>(pp, grid, stream);
    case 12816: return launch_pref_cfg<PrefCfg<128, 16>>(pp, grid, stream);
    case 12832: return launch_pref_cfg<PrefCfg<128, 32>>(pp, grid, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace pa
