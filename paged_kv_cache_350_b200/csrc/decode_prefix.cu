// Shared-prefix decode (sm_100a): sequences forked from one prompt (parallel sampling, a
// common system prompt) share the physical blocks of that prompt ("深入解析
// PagedAttention", 多序列共享; "什么是 LLM 中的分页注意力", 跨请求的内存共享: the requests
// point at the same blocks instead of storing two copies).  Plain paged decode still reads
// those shared blocks once per sequence.  This kernel reads them once per group.
//
// The result is exactly plain attention per (sequence, query head): softmax over the
// shared tokens and over the sequence's own tokens is merged by log-sum-exp.
//
// Units (laid end to end, balanced over warp streams as in decode_stream.cu):
//   * group row r < ngroups, KV head h: the group's shared tokens [0, prefix_r), read
//     through the first member's table; the Q rows are the members' query heads of KV
//     head h stacked (members x G <= 16 rows of the MMA);
//   * sequence row ngroups + b, KV head h: tokens [prefix of b's group (0 if none), L_b).
// A finished unit of an ungrouped sequence writes its output in place; group units and
// grouped sequences' units leave a partial (max, sum, unnormalised O) in a per-unit
// buffer; units cut by a stream boundary are first merged by the cut-unit reduce; a last
// kernel merges, for every grouped sequence, its group partial and its own partial.

#include <cudaTypedefs.h>

#include "pa_device.cuh"
#include "pa_internal.h"
#include "tc_tile.cuh"

namespace pa {

namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kNCW = 2;                 // warps (= streams) per CTA
constexpr int kThreads = kNCW * 32;
constexpr int kSPW = 2;                 // ring stages per stream
constexpr int kRows = 16;               // MMA rows of a unit (members x G of a group)

template <int D_, int BS_>
struct PrefCfg : TileCfg<D_, BS_, true, PA_SHARED_PREFIX_ALIGN> {
  static constexpr int SPW = kSPW;
  static constexpr int NST = kNCW * SPW;
  static constexpr int RING_BYTES = NST * PrefCfg::STAGE_BYTES;
  static constexpr int Q_BYTES = WarpAcc<PrefCfg, true>::Q_BYTES;
  static constexpr int FIXED_BYTES = RING_BYTES + kNCW * Q_BYTES;
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

// Token range and table of unit row r.
struct RowSpan {
  int table_b;  // batch row whose block table covers the tokens
  int tok0;     // first token (multiple of the stage size)
  int tok1;     // one past the last token
};

__device__ __forceinline__ RowSpan row_span(const PrefixParams& pp, int r, bool flag) {
  const DecodeParams& p = pp.d;
  RowSpan s;
  if (r < pp.ngroups) {
    s.table_b = __ldg(pp.group_members + static_cast<size_t>(r) * pp.max_members);
    s.tok0 = 0;
    s.tok1 = __ldg(pp.group_prefix + r);
    if (s.table_b < 0 || s.table_b >= p.B) {  // malformed group: no tokens
      if (flag) flag_error(p.err, PA_DEVERR_BAD_SEQ_LEN);
      s.table_b = 0;
      s.tok1 = 0;
    }
  } else {
    const int b = r - pp.ngroups;
    const int L = clamp_len(p, b, flag);
    const int g = group_of(pp, b, flag);
    const int pre = g >= 0 ? __ldg(pp.group_prefix + g) : 0;
    s.table_b = b;
    s.tok0 = pre < L ? pre : L;
    s.tok1 = L;
  }
  return s;
}

template <class C>
__device__ __forceinline__ int row_tiles(const PrefixParams& pp, int r, bool flag) {
  const RowSpan s = row_span(pp, r, flag);
  return (s.tok1 - s.tok0 + C::TILE_T - 1) / C::TILE_T;
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
  int kvh, nb;
  int id[4];
};

template <class C>
__device__ __forceinline__ TileIds resolve_tile(const PrefixParams& pp, const int* P, int R, int g,
                                                int end) {
  TileIds out{0, 0, {0, 0, 0, 0}};
  if (g >= end) return out;
  const DecodeParams& p = pp.d;
  const TilePos t = locate(P, R, p.Hkv, g);
  out.kvh = t.kvh;
  const RowSpan s = row_span(pp, t.r, false);
  const int blk = s.tok0 / C::BS + t.j * C::BPS;
  const int nblk = (s.tok1 + C::BS - 1) / C::BS;
  out.nb = min(C::BPS, nblk - blk);
  const int32_t* tab = p.block_tables + static_cast<size_t>(s.table_b) * p.max_blocks + blk;
#pragma unroll
  for (int k = 0; k < C::BPS; ++k)
    if (k < out.nb) out.id[k] = __ldg(tab + k);
  return out;
}

// Members of group r (up to max_members batch rows, -1 padded).
__device__ __forceinline__ int group_size(const PrefixParams& pp, int r) {
  int n = 0;
  while (n < pp.max_members &&
         __ldg(pp.group_members + static_cast<size_t>(r) * pp.max_members + n) >= 0)
    ++n;
  return n;
}

template <class C>
__global__ void __launch_bounds__(kThreads)
    decode_prefix_kernel(const __grid_constant__ CUtensorMap tmk,
                         const __grid_constant__ CUtensorMap tmv, const PrefixParams pp) {
  constexpr int D = C::D, BS = C::BS, TILE_T = C::TILE_T, SPW = C::SPW, NST = C::NST;
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
  __shared__ int warp_sum[kThreads / 32];

  {
    const int chunk = (R + kThreads - 1) / kThreads;
    const int lo = min(R, static_cast<int>(threadIdx.x) * chunk);
    const int hi = min(R, lo + chunk);
    int sum = 0;
    for (int r = lo; r < hi; ++r) sum += row_tiles<C>(pp, r, blockIdx.x == 0);
    int incl = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(kFull, incl, off);
      if (lane >= off) incl += v;
    }
    if (lane == 31) warp_sum[warp] = incl;
    __syncthreads();
    int base = 0;
    for (int w = 0; w < warp; ++w) base += warp_sum[w];
    int run = base + incl - sum;
    for (int r = lo; r < hi; ++r) {
      P[r] = run;
      run += row_tiles<C>(pp, r, false);
    }
    if (threadIdx.x == 0) {
      int total = 0;
      for (int w = 0; w < kThreads / 32; ++w) total += warp_sum[w];
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
    for (int st = 0; st < NST; ++st) mbar_init(smem_addr(&full_bar[st]), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    fence_proxy_async_smem();
  }
  __syncthreads();

  const int T = Hkv * P[R];
  const int S = static_cast<int>(gridDim.x) * kNCW;
  const int per = (T + S - 1) / S;
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
    int ids[C::BPS];
#pragma unroll
    for (int q = 0; q < C::BPS; ++q) ids[q] = __shfl_sync(kFull, cur.id[q], src);
    if (lane == 0) {
      const int stage = warp * SPW + k % SPW;
      const uint32_t fb = smem_addr(&full_bar[stage]);
      const uint32_t kt = smem_addr(smem + stage * C::STAGE_BYTES);
      const uint32_t vt = kt + C::TILE_BYTES;
      fence_proxy_async_smem();
      mbar_arrive_expect_tx(fb, static_cast<uint32_t>(n * BS * D * 2 * 2));
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
          tma_load_4d(kt + c * C::CHUNK_BYTES + sub * BS * 128, &tmk, c * 64, kv, 0, phys, fb,
                      policy);
          tma_load_4d(vt + c * C::CHUNK_BYTES + sub * BS * 128, &tmv, c * 64, kv, 0, phys, fb,
                      policy);
        }
      }
    }
    __syncwarp();
  };
  for (int k = 0; k < SPW && k < cnt; ++k) issue(k);

  const int g = lane >> 2, tig = lane & 3;
  const float sl2 = p.scale_log2;
  int unit_a = -1, a_starts = 0, unit_b = -1;
  int i = 0;
  bool ok = true;
  WarpAcc<C, true> acc;
  uint8_t* my_q = qtiles + warp * C::Q_BYTES;
  const __nv_bfloat16* qbase = static_cast<const __nv_bfloat16*>(p.q);

  int gpos = beg;
  while (gpos < end && ok) {
    const TilePos t = locate(P, R, Hkv, gpos);
    const RowSpan span = row_span(pp, t.r, false);
    const int ubeg = Hkv * P[t.r] + t.kvh * t.nt;
    const int uend = ubeg + t.nt;
    const int pend = min(end, uend);
    const int u = t.r * Hkv + t.kvh;
    const bool is_group = t.r < NG;
    int nrows = G;
    // Stage the unit's Q rows: a group's members' heads of this KV head, or the sequence's.
    {
      constexpr int CPR = D * 2 / 16;
      if (is_group) nrows = group_size(pp, t.r) * G;
      __syncwarp();
      for (int idx = lane; idx < kRows * CPR; idx += 32) {
        const int rr = idx / CPR, c = idx - rr * CPR;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (rr < nrows) {
          const int b = is_group
              ? __ldg(pp.group_members + static_cast<size_t>(t.r) * pp.max_members + rr / G)
              : t.r - NG;
          const int h = t.kvh * G + (rr % G);
          if (b >= 0 && b < B)
            v = __ldg(reinterpret_cast<const uint4*>(qbase + (static_cast<size_t>(b) * p.Hq + h) * D) + c);
        }
        *reinterpret_cast<uint4*>(my_q + WarpAcc<C, true>::q_off(rr, c)) = v;
      }
      acc.qs = smem_addr(my_q);
      __syncwarp();
    }
    acc.reset();
    const int jend = t.j + (pend - gpos);
    for (int j = t.j; j < jend; ++j, ++i) {
      const int stage = warp * SPW + i % SPW;
      if (!mbar_wait(smem_addr(&full_bar[stage]), (i / SPW) & 1, p.err)) {
        ok = false;
        break;
      }
      uint8_t* st_ptr = smem + stage * C::STAGE_BYTES;
      const int valid = min(TILE_T, span.tok1 - (span.tok0 + j * TILE_T));
      if (valid < TILE_T) zero_tail_rows<C>(st_ptr, valid, lane);
      acc.tile(smem_addr(st_ptr), valid, sl2, lane);
      __syncwarp();
      if (i + SPW < cnt) issue(i + SPW);
    }
    if (!ok) break;
    acc.reduce_l();
    const bool complete = (gpos == ubeg) && (pend == uend);
    const bool plain = !is_group && group_of(pp, t.r - NG, false) < 0;
    if (complete && plain) {
      const size_t head0 = static_cast<size_t>(t.r - NG) * p.Hq + static_cast<size_t>(t.kvh) * G;
      const float inv_lo = 1.f / acc.l_lo, inv_hi = 1.f / acc.l_hi;
#pragma unroll
      for (int jn = 0; jn < C::NT; ++jn) {
        if (g < G)
          *reinterpret_cast<uint32_t*>(out + (head0 + g) * D + 8 * jn + 2 * tig) =
              pack_bf16x2(acc.o_lo[jn][0] * inv_lo, acc.o_lo[jn][1] * inv_lo);
        if (g + 8 < G)
          *reinterpret_cast<uint32_t*>(out + (head0 + g + 8) * D + 8 * jn + 2 * tig) =
              pack_bf16x2(acc.o_hi[jn][0] * inv_hi, acc.o_hi[jn][1] * inv_hi);
      }
    } else {
      // partial: the unit's own buffer when complete, else a stream slot
      size_t row0;
      float* ml;
      float* oacc;
      if (complete) {
        row0 = static_cast<size_t>(u) * kRows;
        ml = pp.fml;
        oacc = pp.facc;
      } else {
        const int slot = gpos == beg ? 0 : 1;
        row0 = (static_cast<size_t>(s) * 2 + slot) * kRows;
        ml = pp.pml;
        oacc = pp.pacc;
        if (slot == 0) {
          unit_a = u;
          a_starts = gpos == ubeg ? 1 : 0;
        } else {
          unit_b = u;
        }
      }
      if (tig == 0) {
        if (g < nrows)
          *reinterpret_cast<float2*>(ml + (row0 + g) * 2) = make_float2(acc.m_lo, acc.l_lo);
        if (g + 8 < nrows)
          *reinterpret_cast<float2*>(ml + (row0 + g + 8) * 2) = make_float2(acc.m_hi, acc.l_hi);
      }
#pragma unroll
      for (int jn = 0; jn < C::NT; ++jn) {
        if (g < nrows)
          *reinterpret_cast<float2*>(oacc + (row0 + g) * D + 8 * jn + 2 * tig) =
              make_float2(acc.o_lo[jn][0], acc.o_lo[jn][1]);
        if (g + 8 < nrows)
          *reinterpret_cast<float2*>(oacc + (row0 + g + 8) * D + 8 * jn + 2 * tig) =
              make_float2(acc.o_hi[jn][0], acc.o_hi[jn][1]);
      }
    }
    gpos = pend;
  }
  if (!ok) {
    for (int k = i; k < cnt && k < i + SPW; ++k) {
      const int stage = warp * SPW + k % SPW;
      mbar_wait(smem_addr(&full_bar[stage]), (k / SPW) & 1, p.err);
    }
  }
  if (lane == 0) {
    int4 m = make_int4(ok ? unit_a : -1, ok ? a_starts : 0, ok ? unit_b : -1, 0);
    *reinterpret_cast<int4*>(pp.meta + s * 4) = m;
  }
}

// Merge the pieces of units cut by a stream boundary (as in decode_stream.cu).  An
// ungrouped sequence's unit goes straight to the output; a group unit or a grouped
// sequence's unit becomes that unit's partial in the per-unit buffer.
template <int D>
__global__ void __launch_bounds__(512) prefix_cut_reduce_kernel(const PrefixParams pp) {
  const DecodeParams& p = pp.d;
  const int s = blockIdx.x;
  const int4 m = *reinterpret_cast<const int4*>(pp.meta + static_cast<size_t>(s) * 4);
  int u, slot;
  if (m.z >= 0) {
    u = m.z;
    slot = 1;
  } else if (m.x >= 0 && m.y) {
    u = m.x;
    slot = 0;
  } else {
    return;
  }
  const int lane = threadIdx.x & 31;
  int n = 1;
  for (int base = s + 1;; base += 32) {
    const int q = base + lane;
    const bool same = q < pp.streams && pp.meta[static_cast<size_t>(q) * 4] == u;
    const unsigned stop = __ballot_sync(kFull, !same);
    if (stop) {
      n += __ffs(stop) - 1;
      break;
    }
    n += 32;
  }
  const int G = p.G;
  const int r = u / p.Hkv, kvh = u - r * p.Hkv;
  const bool is_group = r < pp.ngroups;
  const int nrows = is_group ? group_size(pp, r) * G : G;
  const bool plain = !is_group && group_of(pp, r - pp.ngroups, false) < 0;
  const int row = threadIdx.x / (D / 4);
  const int c = (threadIdx.x % (D / 4)) * 4;
  if (row >= nrows) return;
  float M = -INFINITY, l = 0.f, a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll 4
  for (int i = 0; i < n; ++i) {
    const size_t pr = (static_cast<size_t>(s + i) * 2 + (i == 0 ? slot : 0)) * kRows + row;
    const float2 ml = *reinterpret_cast<const float2*>(pp.pml + pr * 2);
    const float4 a = *reinterpret_cast<const float4*>(pp.pacc + pr * D + c);
    const float Mn = fmaxf(M, ml.x);
    const float so = exp2f(M - Mn), sn = exp2f(ml.x - Mn);
    l = l * so + ml.y * sn;
    a0 = a0 * so + a.x * sn;
    a1 = a1 * so + a.y * sn;
    a2 = a2 * so + a.z * sn;
    a3 = a3 * so + a.w * sn;
    M = Mn;
  }
  if (plain) {
    const int b = r - pp.ngroups;
    __nv_bfloat16* o = static_cast<__nv_bfloat16*>(p.out) +
                       (static_cast<size_t>(b) * p.Hq + static_cast<size_t>(kvh) * G + row) * D + c;
    const float inv = 1.f / l;
    *reinterpret_cast<uint2*>(o) = make_uint2(pack_bf16x2(a0 * inv, a1 * inv),
                                              pack_bf16x2(a2 * inv, a3 * inv));
  } else {
    const size_t fr = static_cast<size_t>(u) * kRows + row;
    if (c == 0) *reinterpret_cast<float2*>(pp.fml + fr * 2) = make_float2(M, l);
    *reinterpret_cast<float4*>(pp.facc + fr * D + c) = make_float4(a0, a1, a2, a3);
  }
}

// out[b][h] for every grouped sequence b = merge(group partial, own partial).
template <int D>
__global__ void __launch_bounds__(256) prefix_merge_kernel(const PrefixParams pp) {
  const DecodeParams& p = pp.d;
  const int b = blockIdx.x;
  const int grp = group_of(pp, b, false);
  if (grp < 0) return;
  const int L = clamp_len(p, b, false);
  if (L == 0) return;
  int mpos = 0;
  for (int m = 0; m < pp.max_members; ++m)
    if (__ldg(pp.group_members + static_cast<size_t>(grp) * pp.max_members + m) == b) mpos = m;
  const int pre = __ldg(pp.group_prefix + grp);
  const bool has_own = L > pre;
  const int G = p.G;
  __nv_bfloat16* o = static_cast<__nv_bfloat16*>(p.out) + static_cast<size_t>(b) * p.Hq * D;
  for (int idx = threadIdx.x; idx < p.Hq * (D / 4); idx += blockDim.x) {
    const int h = idx / (D / 4), c = (idx % (D / 4)) * 4;
    const int kvh = h / G, gh = h - kvh * G;
    const size_t gr = (static_cast<size_t>(grp) * p.Hkv + kvh) * kRows + mpos * G + gh;
    const float2 ga = *reinterpret_cast<const float2*>(pp.fml + gr * 2);
    const float4 gacc = *reinterpret_cast<const float4*>(pp.facc + gr * D + c);
    float M = ga.x, l = ga.y;
    float a0 = gacc.x, a1 = gacc.y, a2 = gacc.z, a3 = gacc.w;
    if (has_own) {
      const size_t sr = (static_cast<size_t>(pp.ngroups + b) * p.Hkv + kvh) * kRows + gh;
      const float2 sa = *reinterpret_cast<const float2*>(pp.fml + sr * 2);
      const float4 sacc = *reinterpret_cast<const float4*>(pp.facc + sr * D + c);
      const float Mn = fmaxf(M, sa.x);
      const float so = exp2f(M - Mn), sn = exp2f(sa.x - Mn);
      l = l * so + sa.y * sn;
      a0 = a0 * so + sacc.x * sn;
      a1 = a1 * so + sacc.y * sn;
      a2 = a2 * so + sacc.z * sn;
      a3 = a3 * so + sacc.w * sn;
    }
    const float inv = 1.f / l;
    *reinterpret_cast<uint2*>(o + static_cast<size_t>(h) * D + c) =
        make_uint2(pack_bf16x2(a0 * inv, a1 * inv), pack_bf16x2(a2 * inv, a3 * inv));
  }
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
  if (!make_pool_map(&tmk, p.k_pool, p.num_blocks, C::BS, p.Hkv, C::D) ||
      !make_pool_map(&tmv, p.v_pool, p.num_blocks, C::BS, p.Hkv, C::D))
    return cudaErrorInvalidValue;
  const size_t smem = pref_smem_bytes<C>(pp.ngroups + p.B);
  cudaError_t e = cudaFuncSetAttribute(decode_prefix_kernel<C>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  decode_prefix_kernel<C><<<grid, kThreads, smem, stream>>>(tmk, tmv, pp);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  prefix_cut_reduce_kernel<C::D><<<pp.streams, kRows * C::D / 4, 0, stream>>>(pp);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  prefix_merge_kernel<C::D><<<p.B, 256, 0, stream>>>(pp);
  return cudaGetLastError();
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

size_t prefix_workspace_bytes(int streams, int units, int D) {
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  return up(static_cast<size_t>(streams) * 16) + up(static_cast<size_t>(streams) * 2 * kRows * 8) +
         up(static_cast<size_t>(streams) * 2 * kRows * D * 4) +
         up(static_cast<size_t>(units) * kRows * 8) + static_cast<size_t>(units) * kRows * D * 4;
}

void prefix_carve(PrefixParams* pp, void* workspace, int units) {
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  char* w = static_cast<char*>(workspace);
  const int D = pp->d.D;
  pp->meta = reinterpret_cast<int32_t*>(w);
  w += up(static_cast<size_t>(pp->streams) * 16);
  pp->pml = reinterpret_cast<float*>(w);
  w += up(static_cast<size_t>(pp->streams) * 2 * kRows * 8);
  pp->pacc = reinterpret_cast<float*>(w);
  w += up(static_cast<size_t>(pp->streams) * 2 * kRows * D * 4);
  pp->fml = reinterpret_cast<float*>(w);
  w += up(static_cast<size_t>(units) * kRows * 8);
  pp->facc = reinterpret_cast<float*>(w);
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
