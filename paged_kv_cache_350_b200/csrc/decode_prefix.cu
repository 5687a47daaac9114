// Shared-prefix decode on the 5th-generation tensor cores (sm_100a).
//
// Sequences forked from one prompt (parallel sampling, a common system prompt) share the
// physical blocks of that prompt ("深入解析 PagedAttention", 多序列共享; "什么是 LLM 中的分页
// 注意力", 跨请求的内存共享: the requests point at the same blocks instead of storing two
// copies).  Plain paged decode still reads those shared blocks once per sequence; this
// kernel reads them once per group.  The result is exactly plain attention per (sequence,
// query head).
//
// Units.  One unit per (group row, KV head): the query heads of that KV head of all the
// group's members are stacked as the rows of one tile (members x G <= 64 rows).  A unit's
// tokens are a list of 32-token chunks: first the shared tokens [0, prefix) through the
// first member's table, which every row attends to, then each member's own tokens
// [prefix, L_m) through that member's table, which only that member's rows attend to.  An
// ungrouped sequence is a unit of its own G rows and tokens [0, L).
//
// Schedule.  One persistent CTA per SM; the chunks of all units laid end to end are split
// into equal contiguous ranges, one per CTA, so the work is balanced to one chunk.  A CTA
// walks its range in tiles of up to four chunks (128 tokens) of one unit; a tile may hold
// several members' own chunks (each row masks the chunks that are not its own).  A unit
// cut by a range boundary leaves a partial (max, sum, unnormalised output) per row, which
// the cut reduce merges by log-sum-exp.
//
// Per CTA, warp-specialised:
//   warp 0     producer: resolves block ids through the tables, loads each tile's K and V
//              blocks with TMA (one box per block and 64-column chunk) into a ring of
//              stages, and writes each unit's Q rows into one of two Q buffers;
//   warp 1     MMA: one thread issues, per tile, S = Q.K^T (M = 64 rows, N = tile tokens,
//              K = head dim; A = Q, B = K, both K-major in shared memory) into one of two
//              S accumulators in tensor memory, and O += P.V (A = P from tensor memory,
//              B = V, MN-major in shared memory) into the O accumulator in tensor memory;
//              S of the next tile is issued before P.V of this one;
//   warps 2-5  softmax: two threads per query row (rows spread over the four tensor-memory
//              sub-partitions, each row's columns split in halves) read its S row, mask,
//              and run the online softmax in fp32
//              base 2 with a lazy rescale (the reference max moves only when a tile's max
//              passes it by more than 2^8, and only then is O rescaled in tensor memory);
//              P enters the P.V product as two bf16 parts, hi = rn(p) and lo = rn(p - hi),
//              so it keeps ~16 significant bits; at a unit's end the row's output (or
//              partial) is read from tensor memory and written out.
// Tensor memory: S buffers at columns 0 and 128, each overwritten by its P (hi parts in
// its columns 0-63, lo parts in 64-127) once the softmax has read it, so P is double
// buffered with S; O at 256.
//
// Every wait is bounded in time; on expiry the kernel records PA_DEVERR_TIMEOUT, every
// role stops, the loads and tensor-core operations in flight are drained (bounded), and
// the tensor memory is freed before the CTA exits.

#include <cudaTypedefs.h>

#include <climits>

#include "pa_device.cuh"
#include "pa_internal.h"
#include "tc05.cuh"

namespace pa {

namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kCT = 32;                  // tokens per chunk
constexpr int kCPT = 4;                  // chunks per tile
constexpr int kTT = kCT * kCPT;          // tokens per tile (S columns)
constexpr int kRows = 64;                // MMA rows (M)
constexpr int kWarps = 6;                // producer, MMA, 4 softmax
constexpr int kThreads = kWarps * 32;
constexpr int kSoftThreads = 128;
constexpr int kMaxStages = 4;
constexpr int kMaxMembers = 32;          // members of a group (one per producer lane)
constexpr float kRescaleLog2 = 8.f;      // lazy rescale threshold (log2 units)
static_assert(PA_SHARED_PREFIX_ALIGN % kCT == 0, "a shared prefix ends on a chunk boundary");

// Tensor-memory columns: two S buffers, each overwritten in place by its P (bf16 hi parts
// packed in columns 0-63, lo parts in 64-127), and O.
constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO = 256;
constexpr uint32_t kColPlo = 64;  // P lo, relative to its S buffer (P hi at +0)
constexpr uint32_t kTmemCols = 512;

// Tile flags.
constexpr int kFirstOfPiece = 1, kLastOfPiece = 2, kLastOfCta = 4, kCompleteUnit = 8;

struct TileInfo {
  int unit;       // r * Hkv + kvh
  int rows;       // query rows of the unit (members x G)
  int nch;        // chunks in this tile (1..4)
  int flags;
  int piece;      // index of the piece (unit part) within this CTA
  int slot;       // partial slot of a cut piece (0: the CTA's first piece, 1: last)
  int mem[kCPT];  // per chunk: member (-1: shared tokens, every row)
  int nv[kCPT];   // per chunk: valid tokens (1..32)
};

template <int D_, int BS_>
struct GroupCfg {
  static constexpr int D = D_;
  static constexpr int BS = BS_;
  static constexpr int DCH = D / 64;                 // 64-column chunks of a head row
  static constexpr int KV_CHUNK_BYTES = kTT * 128;   // one 64-column chunk of a tile
  static constexpr int K_BYTES = DCH * KV_CHUNK_BYTES;
  static constexpr int STAGE_BYTES = 2 * K_BYTES;    // K then V
  static constexpr int Q_CHUNK_BYTES = kRows * 128;
  static constexpr int Q_BYTES = DCH * Q_CHUNK_BYTES;
  static constexpr int BPC = kCT / BS;               // blocks per chunk
  static_assert(D == 64 || D == 128, "head dim");
  static_assert(BS == 8 || BS == 16 || BS == 32, "block size");
};

// Static shared memory of the kernel is below this (barriers, tile records, scan: ~400 B).
constexpr size_t kStaticSmemBound = 512;

template <class C>
size_t group_smem_bytes(int nst, int R) {
  return 1024 + static_cast<size_t>(nst) * C::STAGE_BYTES + 2 * C::Q_BYTES +
         static_cast<size_t>(R + 1) * 4;
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

__device__ __forceinline__ int member_of(const PrefixParams& pp, int r, int m) {
  return __ldg(pp.group_members + static_cast<size_t>(r) * pp.max_members + m);
}

// Group of batch row b (-1 if none, or out of range: flagged, then treated as ungrouped).
__device__ __forceinline__ int group_of(const PrefixParams& pp, int b, bool flag) {
  const int g = __ldg(pp.group_of + b);
  if (g >= pp.ngroups || g < -1) {
    if (flag) flag_error(pp.d.err, PA_DEVERR_BAD_SEQ_LEN);
    return -1;
  }
  return g;
}

// Shared tokens of group r; -1 for a malformed group (flagged): its unit has no chunk.
__device__ __forceinline__ int group_prefix_tokens(const PrefixParams& pp, int r, bool flag) {
  const int b0 = member_of(pp, r, 0);
  const int pre = __ldg(pp.group_prefix + r);
  if (b0 < 0 || b0 >= pp.d.B || pre < 0 || pre % PA_SHARED_PREFIX_ALIGN != 0) {
    if (flag) flag_error(pp.d.err, PA_DEVERR_BAD_SEQ_LEN);
    return -1;
  }
  return pre;
}

// Chunks of unit row r (the same for each of its KV heads).  A group's member ids are
// loaded first and their lengths second, each round as independent loads, so that the
// prologue waits for two memory round trips per row, not two per member.
__device__ int row_chunks(const PrefixParams& pp, int r, bool flag) {
  const int NG = pp.ngroups;
  if (r < NG) {
    const int pre = group_prefix_tokens(pp, r, flag);
    if (pre < 0) return 0;
    int ids[kMaxMembers];
#pragma unroll
    for (int m = 0; m < kMaxMembers; ++m) ids[m] = m < pp.max_members ? member_of(pp, r, m) : -1;
    int lens[kMaxMembers];
    bool live = true;  // members before the first -1
#pragma unroll
    for (int m = 0; m < kMaxMembers; ++m) {
      live = live && ids[m] >= 0;
      lens[m] = (live && ids[m] < pp.d.B) ? clamp_len(pp.d, ids[m], flag) : -1;
    }
    int n = pre / kCT;
#pragma unroll
    for (int m = 0; m < kMaxMembers; ++m) {
      if (lens[m] < 0) continue;
      if (lens[m] < pre) {
        if (flag) flag_error(pp.d.err, PA_DEVERR_BAD_SEQ_LEN);
      } else {
        n += (lens[m] - pre + kCT - 1) / kCT;
      }
    }
    return n;
  }
  const int b = r - NG;
  if (group_of(pp, b, flag) >= 0) return 0;  // covered by its group's unit
  return (clamp_len(pp.d, b, flag) + kCT - 1) / kCT;
}

struct UnitPos {
  int r, kvh, j, nt;  // unit row, KV head, chunk within the unit, chunks of the unit
};

__device__ __forceinline__ UnitPos locate(const int* P, int R, int Hkv, int g) {
  UnitPos u;
  u.r = upper_bound(P, R + 1, g / Hkv) - 1;
  u.nt = P[u.r + 1] - P[u.r];
  const int off = g - Hkv * P[u.r];
  u.kvh = off / u.nt;
  u.j = off - u.kvh * u.nt;
  return u;
}

// Bounded wait that also gives up when another role has given up (the CTA-wide abort
// word); on its own expiry it records the timeout and raises the abort word.
__device__ __forceinline__ bool wait_or_abort(uint32_t bar, uint32_t parity, int32_t* err,
                                              volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (global_timer_ns() - t0 > kWaitLimitNs) {
      flag_error(err, PA_DEVERR_TIMEOUT);
      *abort_flag = 1;
      return false;
    }
  }
}

// The same, decided by lane 0 and shared with the warp.
__device__ __forceinline__ bool wait_lane0(uint32_t bar, uint32_t parity, int32_t* err,
                                           volatile int* abort_flag) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0) ok = wait_or_abort(bar, parity, err, abort_flag) ? 1 : 0;
  return __shfl_sync(kFull, ok, 0) != 0;
}

// The same for a whole warp: every lane waits, and the warp agrees.
__device__ __forceinline__ bool wait_warp(uint32_t bar, uint32_t parity, int32_t* err,
                                          volatile int* abort_flag) {
  const bool ok = wait_or_abort(bar, parity, err, abort_flag);
  return __all_sync(kFull, ok) != 0;
}

// Byte offset of the 16-byte piece c16 of row r of 64-column chunk `chunk` in a K-major
// 128-byte-swizzled operand whose chunks hold `rows` rows.
__device__ __forceinline__ uint32_t sw_piece(int r, int c16, int chunk, int rows) {
  return static_cast<uint32_t>(chunk * rows * 128 + r * 128 + ((c16 ^ (r & 7)) << 4));
}

template <class C>
__global__ void __launch_bounds__(kThreads, 1)
    decode_group_kernel(const __grid_constant__ CUtensorMap tmk,
                        const __grid_constant__ CUtensorMap tmv, const PrefixParams pp,
                        int nst) {
  constexpr int D = C::D, BS = C::BS, DCH = C::DCH;
  const DecodeParams& p = pp.d;
  const int B = p.B, Hkv = p.Hkv, G = p.G, NG = pp.ngroups;
  const int R = NG + B;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* qbuf = smem + static_cast<size_t>(nst) * C::STAGE_BYTES;  // [2][Q_BYTES]
  int* P = reinterpret_cast<int*>(qbuf + 2 * C::Q_BYTES);            // [R + 1]

  __shared__ __align__(8) uint64_t full_bar[kMaxStages], empty_bar[kMaxStages];
  __shared__ __align__(8) uint64_t qfull_bar[2], qempty_bar[2], sfull_bar[2];
  // pvdone_bar[b]: P.V of the tiles using S buffer b (tiles b, b + 2, ...), one phase each
  __shared__ __align__(8) uint64_t pfull_bar, pvdone_bar[2], drain_bar;
  __shared__ TileInfo info[kMaxStages];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int warp_sum[kWarps];
  __shared__ volatile int abort_flag;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kMaxStages; ++s) {
      mbar_init(smem_addr(&full_bar[s]), 1);
      mbar_init(smem_addr(&empty_bar[s]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_addr(&qfull_bar[i]), 32);
      mbar_init(smem_addr(&qempty_bar[i]), 1);
      mbar_init(smem_addr(&sfull_bar[i]), 1);
    }
    mbar_init(smem_addr(&pfull_bar), kSoftThreads);
    mbar_init(smem_addr(&pvdone_bar[0]), 1);
    mbar_init(smem_addr(&pvdone_bar[1]), 1);
    mbar_init(smem_addr(&drain_bar), 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    fence_proxy_async_smem();
  }
  if (warp == 1) tc05::alloc(smem_addr(&tmem_base_sh), kTmemCols);
  // Launched as a programmatic dependent of the previous kernel on the stream: nothing
  // above reads global memory; wait for that kernel before anything below does.
  asm volatile("griddepcontrol.wait;" ::: "memory");

  // ---- chunk counts of every unit row, scanned (every CTA, identical) ----------------
  for (int r = threadIdx.x; r < R; r += kThreads) P[r] = row_chunks(pp, r, blockIdx.x == 0);
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
      for (int w = 0; w < kWarps; ++w) total += warp_sum[w];
      P[R] = total;
    }
  }
  // Empty sequences have no chunk: their output rows are zero (written by one CTA each).
  __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out);
  for (int b = blockIdx.x; b < B; b += gridDim.x) {
    if (clamp_len(p, b, false) == 0) {
      uint32_t* row = reinterpret_cast<uint32_t*>(out + static_cast<size_t>(b) * p.Hq * D);
      for (int i = threadIdx.x; i < p.Hq * D / 2; i += kThreads) row[i] = 0u;
    }
  }
  tc05::fence_before_sync();
  __syncthreads();
  tc05::fence_after_sync();
  const uint32_t tmem = tmem_base_sh;

  const int T = Hkv * P[R];
  const int S = static_cast<int>(gridDim.x);
  const int per = (T + S - 1) / S;
  const int cta = static_cast<int>(blockIdx.x);
  const int beg = min(T, cta * per);
  const int end = min(T, beg + per);
  // Let the cut reduce be launched now; it waits for this grid to complete.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const float sl2 = p.scale_log2;
  const uint8_t* qg = static_cast<const uint8_t*>(p.q);

  if (warp == 0) {
    // ============================ producer ============================
    // The producer's global loads (block ids, members, Q rows) are the step's latency
    // chain, each a round trip of about a microsecond, so none is issued where it is used:
    //   * block ids are loaded 64 at a time (two per lane), one batch ahead: a batch holds
    //     the ids of 64 / BPC chunks (2 to 16 tiles);
    //   * the next piece (members, Q rows, first two batches) is prepared while this one
    //     streams, once its first three tiles are out (so the stages are full);
    //   * Q rows are asynchronous copies, published to the MMA thread at the piece's first
    //     tile.
    const uint64_t policy = l2_policy_evict_first();
    if (lane == 0) {
      prefetch_tensormap(&tmk);
      prefetch_tensormap(&tmv);
    }
    // One unit piece (the part of a unit inside this CTA's range); lane m holds member m.
    struct Piece {
      int g, pend, ubeg, uend, r, kvh, j;  // first chunk, end; unit bounds, row, head, chunk
      int mb, mL, mst;                     // member's batch row, length, first own chunk
      int pre, n0, gs, rows;               // shared tokens and chunks, members, query rows
    };
    auto load_piece = [&](int g) {
      Piece pc;
      const UnitPos u = locate(P, R, Hkv, g);
      pc.g = g;
      pc.ubeg = g - u.j;
      pc.uend = pc.ubeg + u.nt;
      pc.pend = min(end, pc.uend);
      pc.r = u.r;
      pc.kvh = u.kvh;
      pc.j = u.j;
      const bool grp = u.r < NG;
      int mb = -1, pre = 0;
      if (grp) {
        mb = lane < pp.max_members ? member_of(pp, u.r, lane) : -1;
        pre = max(group_prefix_tokens(pp, u.r, false), 0);
      } else if (lane == 0) {
        mb = u.r - NG;
      }
      const unsigned live_mask = __ballot_sync(kFull, mb >= 0);
      const int gs = grp ? (~live_mask ? __ffs(~live_mask) - 1 : 32) : 1;  // before the first -1
      if (lane >= gs) mb = -1;
      pc.mb = mb;
      pc.pre = pre;
      pc.gs = gs;
      pc.n0 = pre / kCT;
      pc.rows = gs * G;
      pc.mL = (mb >= 0 && mb < B) ? clamp_len(p, mb, false) : 0;
      const int own = (mb >= 0 && mb < B && pc.mL >= pre) ? (pc.mL - pre + kCT - 1) / kCT : 0;
      int incl = own;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(kFull, incl, off);
        if (lane >= off) incl += v;
      }
      pc.mst = pc.n0 + incl - own;
      return pc;
    };
    // Where unit chunk jj comes from (lanes may ask for different chunks): the table row,
    // first token and valid tokens; the member is the last one whose own chunks start at
    // or before jj (a binary search over the lanes' starts).
    auto chunk_src = [&](const Piece& pc, int jj, int& tb, int& t0, int& nv, int& mem) {
      int m = 0;
#pragma unroll
      for (int step = 16; step >= 1; step >>= 1) {
        const int cand = m + step;
        const int v = __shfl_sync(kFull, pc.mst, cand < 32 ? cand : 31);
        if (cand < pc.gs && v <= jj) m = cand;
      }
      const bool shared = jj < pc.n0;
      const int mm = shared ? 0 : m;
      tb = __shfl_sync(kFull, pc.mb, mm);
      const int Lm = __shfl_sync(kFull, pc.mL, mm);
      const int sm = __shfl_sync(kFull, pc.mst, m);
      t0 = shared ? jj * kCT : pc.pre + (jj - sm) * kCT;
      nv = shared ? kCT : min(kCT, Lm - t0);
      mem = shared ? -1 : m;
    };
    // Block-id batch n of a piece: slot k (lane k % 32, entry k / 32) is block k % BPC of
    // the piece's chunk n * CPB + k / BPC; kNoBlock where there is none.
    constexpr int CPB = 64 / C::BPC;
    constexpr int kNoBlock = INT_MIN;
    auto load_batch = [&](const Piece& pc, int n, int (&ids)[2]) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int k = lane + 32 * e;
        const int jrel = n * CPB + k / C::BPC;
        const int i = k % C::BPC;
        int tb, t0, nv, mem;
        chunk_src(pc, pc.j + jrel, tb, t0, nv, mem);
        const bool live = pc.g + jrel < pc.pend && i * BS < nv && tb >= 0 && tb < B;
        ids[e] = live ? __ldg(p.block_tables + static_cast<size_t>(tb) * p.max_blocks + t0 / BS + i)
                      : kNoBlock;
      }
    };
    // Q rows of a piece into Q buffer qb (row r at MMA row 16*(r%4) + r/4), asynchronous
    // copies (rows past the unit zero-filled); published at the piece's first tile.
    auto copy_q = [&](const Piece& pc, int qb) {
      uint8_t* qt = qbuf + qb * C::Q_BYTES;
      constexpr int CPR = D * 2 / 16;  // 16-byte pieces per row
      for (int idx = lane; idx < kRows * CPR; idx += 32) {
        const int r = idx / CPR, c = idx - r * CPR;
        const int m = 16 * (r & 3) + (r >> 2);
        const int k = r / G;  // member
        const int b = __shfl_sync(kFull, pc.mb, k < 32 ? k : 0);
        const bool live = r < pc.rows && b >= 0 && b < B;
        const uint8_t* src = qg + (live ? (static_cast<size_t>(b) * p.Hq + pc.kvh * G + r % G) * D * 2 : 0);
        cp_async_16_zfill(smem_addr(qt + sw_piece(m, c & 7, c >> 3, kRows)),
                          reinterpret_cast<const uint4*>(src) + (live ? c : 0), live ? 16 : 0);
      }
      cp_async_commit();
    };

    int own_u = -1, own_slot = 0, own_n = 0, own_rows = 0;
    int t = 0, piece = 0;
    bool ok = beg < end;
    Piece pc, nx;
    int cur[2], nxt[2], nb0[2], nb1[2];
    if (ok) {
      pc = load_piece(beg);
      copy_q(pc, 0);
      load_batch(pc, 0, cur);
      load_batch(pc, 1, nxt);
    }
    while (ok) {
      const int slot = pc.g == beg ? 0 : 1;
      const bool complete = pc.g == pc.ubeg && pc.pend == pc.uend;
      if (!complete && pc.ubeg >= beg) {  // the unit starts here: it is this CTA's to merge
        own_u = pc.r * Hkv + pc.kvh;
        own_slot = slot;
        own_n = (pc.uend - 1) / per - cta + 1;
        own_rows = pc.rows;
      }
      const int qb = piece & 1;
      const bool has_next = pc.pend < end;
      bool prepared = false;
      int batch = 0;        // batch held in cur
      int tiles_out = 0;    // tiles of this piece issued
      for (int c0 = pc.g; ok;) {
        const int nch = min(kCPT, pc.pend - c0);
        const int jrel = c0 - pc.g;
        if (jrel / CPB != batch) {  // move to the next batch; load the one after it
          cur[0] = nxt[0];
          cur[1] = nxt[1];
          ++batch;
          load_batch(pc, batch + 1, nxt);
        }
        const int s = t % nst;
        if (t >= nst) {
          ok = wait_lane0(smem_addr(&empty_bar[s]), ((t / nst) - 1) & 1, p.err, &abort_flag);
          if (!ok) break;
        }
        if (c0 == pc.g) {  // the piece's Q rows have landed: publish them to the MMA thread
          cp_async_wait_all();
          fence_proxy_async_smem();
          mbar_arrive(smem_addr(&qfull_bar[qb]));
        }
        // chunk q of the tile (lane q < nch): member and valid tokens, for the record
        int cm = -1, cnv = 0;
        {
          int tb, t0, nv, mem;
          chunk_src(pc, pc.j + jrel + (lane < kCPT ? lane : 0), tb, t0, nv, mem);
          if (lane < nch) {
            cm = mem;
            cnv = nv;
          }
        }
        int qm[kCPT], qv[kCPT];
#pragma unroll
        for (int q = 0; q < kCPT; ++q) {
          qm[q] = __shfl_sync(kFull, cm, q);
          qv[q] = __shfl_sync(kFull, cnv, q);
        }
        const bool last_of_piece = c0 + nch >= pc.pend;
        if (lane == 0) {
          TileInfo* ti = &info[s];
          ti->unit = pc.r * Hkv + pc.kvh;
          ti->rows = pc.rows;
          ti->nch = nch;
          ti->piece = piece;
          ti->slot = slot;
          ti->flags = (c0 == pc.g ? kFirstOfPiece : 0) | (last_of_piece ? kLastOfPiece : 0) |
                      (last_of_piece && !has_next ? kLastOfCta : 0) |
                      (complete ? kCompleteUnit : 0);
#pragma unroll
          for (int q = 0; q < kCPT; ++q) {
            ti->mem[q] = qm[q];
            ti->nv[q] = qv[q];
          }
        }
        // this tile's block ids from the batch: lane l < nch * BPC takes slot
        // (jrel % CPB) * BPC + l
        const int k = (jrel % CPB) * C::BPC + (lane < kCPT * C::BPC ? lane : 0);
        const int a0 = __shfl_sync(kFull, cur[0], k & 31);
        const int a1 = __shfl_sync(kFull, cur[1], k & 31);
        int phys = (k >> 5) ? a1 : a0;
        const bool live = lane < nch * C::BPC && phys != kNoBlock;
        if (live && (phys < 0 || phys >= p.num_blocks)) {
          flag_error(p.err, PA_DEVERR_BAD_BLOCK_ID);
          phys = 0;
        }
        const int nboxes = __popc(__ballot_sync(kFull, live));
        const uint32_t fb = smem_addr(&full_bar[s]);
        if (lane == 0) {
          fence_proxy_async_smem();  // this stage's earlier generic writes come first
          mbar_arrive_expect_tx(fb, static_cast<uint32_t>(nboxes * BS * D * 2 * 2));
        }
        __syncwarp();
        if (live) {
          const int q = lane / C::BPC, i = lane % C::BPC;
          const uint32_t kt = smem_addr(smem + static_cast<size_t>(s) * C::STAGE_BYTES) +
                              (q * kCT + i * BS) * 128;
          const uint32_t vt = kt + C::K_BYTES;
#pragma unroll
          for (int c = 0; c < DCH; ++c) {
            tma_load_4d(kt + c * C::KV_CHUNK_BYTES, &tmk, c * 64, pc.kvh, 0, phys, fb, policy);
            tma_load_4d(vt + c * C::KV_CHUNK_BYTES, &tmv, c * 64, pc.kvh, 0, phys, fb, policy);
          }
        }
        __syncwarp();
        ++t;
        ++tiles_out;
        // the next piece, prepared once this one's stages are full (its Q buffer was last
        // read by the piece before this one, whose last tile has been consumed by then)
        if (has_next && !prepared && (tiles_out >= nst || last_of_piece)) {
          nx = load_piece(pc.pend);
          const int qn = piece + 1;
          if (qn >= 2) {
            ok = wait_lane0(smem_addr(&qempty_bar[qn & 1]), ((qn >> 1) - 1) & 1, p.err, &abort_flag);
            if (!ok) break;
          }
          copy_q(nx, qn & 1);
          load_batch(nx, 0, nb0);
          load_batch(nx, 1, nb1);
          prepared = true;
        }
        if (last_of_piece) break;
        c0 += nch;
      }
      if (!ok || !has_next) break;
      pc = nx;
      cur[0] = nb0[0];
      cur[1] = nb0[1];
      nxt[0] = nb1[0];
      nxt[1] = nb1[1];
      ++piece;
    }
    cp_async_wait_all();  // a Q copy still in flight after an early exit
    if (!ok) {
      // wait (bounded) for the loads issued but never consumed, so none lands after exit
      for (int k = max(0, t - nst); k < t; ++k)
        mbar_wait(smem_addr(&full_bar[k % nst]), (k / nst) & 1, nullptr, kWaitLimitNs);
    }
    if (lane == 0) {
      const int4 m = make_int4(abort_flag ? -1 : own_u, own_slot, own_n, own_rows);
      *reinterpret_cast<int4*>(pp.meta + cta * 4) = m;
    }
  } else if (warp == 1) {
    // ============================ MMA issuer ============================
    if (lane == 0 && beg < end) {
      const uint32_t id_s_base = tc05::instr_desc_bf16(kRows, 8, 0) & ~(0x3Fu << 17);
      const uint32_t id_pv = tc05::instr_desc_bf16(kRows, D, 1);
      bool ok = true;
      // S of tile t (its stage has landed and its record is read here)
      auto issue_s = [&](int t, const TileInfo& ti) -> bool {
        const int s = t % nst;
        const int qb = ti.piece & 1;
        if ((ti.flags & kFirstOfPiece) &&
            !wait_or_abort(smem_addr(&qfull_bar[qb]), (ti.piece >> 1) & 1, p.err, &abort_flag))
          return false;
        tc05::fence_after_sync();
        const uint32_t qa = smem_addr(qbuf + qb * C::Q_BYTES);
        const uint32_t ka = smem_addr(smem + static_cast<size_t>(s) * C::STAGE_BYTES);
        const uint32_t idesc = id_s_base | (static_cast<uint32_t>((ti.nch * kCT) >> 3) << 17);
        const uint32_t ts = tmem + ((t & 1) ? kColS1 : kColS0);
        // this S buffer's P was last read by P.V of tile t - 2: it must have completed (the
        // buffer's barrier has one phase per use, and the use before that was waited for
        // when S of tile t - 2 was issued)
        if (t >= 2 && !wait_or_abort(smem_addr(&pvdone_bar[t & 1]), ((t - 2) >> 1) & 1, p.err,
                                     &abort_flag))
          return false;
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off_q = (k >> 2) * C::Q_CHUNK_BYTES + (k & 3) * 32;
          const uint32_t off_k = (k >> 2) * C::KV_CHUNK_BYTES + (k & 3) * 32;
          tc05::mma_ss(ts, tc05::smem_desc(qa + off_q, 16, 1024),
                       tc05::smem_desc(ka + off_k, 16, 1024), idesc, k > 0);
        }
        tc05::commit(smem_addr(&sfull_bar[t & 1]));
        if (ti.flags & kLastOfPiece) tc05::commit(smem_addr(&qempty_bar[qb]));
        return true;
      };
      TileInfo cur;
      ok = wait_or_abort(smem_addr(&full_bar[0]), 0, p.err, &abort_flag);
      if (ok) {
        cur = info[0];
        ok = issue_s(0, cur);
      }
      for (int t = 0; ok; ++t) {
        TileInfo nxt;
        const bool more = !(cur.flags & kLastOfCta);
        const int s1 = (t + 1) % nst;
        const uint32_t par1 = ((t + 1) / nst) & 1;
        // S of the next tile goes first when its K has landed, so that it overlaps this
        // tile's softmax; P.V of this tile never waits for the next tile's loads
        bool s_next = false;
        if (more && mbar_try_wait(smem_addr(&full_bar[s1]), par1)) {
          nxt = info[s1];
          ok = issue_s(t + 1, nxt);
          if (!ok) break;
          s_next = true;
        }
        // P of tile t written (and the softmax is done with S of tile t)
        ok = wait_or_abort(smem_addr(&pfull_bar), t & 1, p.err, &abort_flag);
        if (!ok) break;
        tc05::fence_after_sync();
        const int s = t % nst;
        const uint32_t va = smem_addr(smem + static_cast<size_t>(s) * C::STAGE_BYTES) + C::K_BYTES;
        const uint32_t tp = tmem + ((t & 1) ? kColS1 : kColS0);  // P of tile t
        bool first = (cur.flags & kFirstOfPiece) != 0;
        for (int q = 0; q < cur.nch; ++q) {
          const int ksteps = cur.nv[q] > 16 ? 2 : 1;
          for (int kk = 0; kk < ksteps; ++kk) {
            const int k = 2 * q + kk;
            const uint64_t vdesc = tc05::smem_desc(va + k * 2048, C::KV_CHUNK_BYTES, 1024);
            tc05::mma_ts(tmem + kColO, tp + 8 * k, vdesc, id_pv, !first);
            tc05::mma_ts(tmem + kColO, tp + kColPlo + 8 * k, vdesc, id_pv, true);
            first = false;
          }
        }
        tc05::commit(smem_addr(&pvdone_bar[t & 1]));
        tc05::commit(smem_addr(&empty_bar[s]));
        if (!more) break;
        if (!s_next) {
          ok = wait_or_abort(smem_addr(&full_bar[s1]), par1, p.err, &abort_flag);
          if (!ok) break;
          nxt = info[s1];
          ok = issue_s(t + 1, nxt);
          if (!ok) break;
        }
        cur = nxt;
      }
      if (!ok) abort_flag = 1;
      // every tensor-core operation issued has completed before the memory is freed
      tc05::commit(smem_addr(&drain_bar));
      mbar_wait(smem_addr(&drain_bar), 0, p.err);
    }
    __syncwarp();
  } else {
    // ============================ softmax ============================
    // Warp w serves tensor-memory sub-partition sp = w % 4, whose lanes 0-15 hold MMA rows
    // 16*sp .. 16*sp + 15 (the M = 64 accumulator layout).  Threads t and t + 16 share the
    // row of lane t % 16 (the 16x32bx2 shape): half h = t / 16 takes chunks h and h + 2 of
    // the tile (S columns 32h.. and 64 + 32h..) and the same columns of O, so every row's
    // work is split over two threads and a row's max and sum combine by one shuffle.
    const int sp = warp & 3;                    // tensor-memory sub-partition
    const int h = lane >> 4;                    // column half
    const int r = 4 * (lane & 15) + sp;         // this thread's query row
    const uint32_t lane_addr = static_cast<uint32_t>(32 * sp) << 16;
    const int tid_s = threadIdx.x - 64;         // 0..127
    float m_ref = -INFINITY, lsum = 0.f;        // lsum: this half's part of the row sum
    bool ok = beg < end;
    for (int t = 0; ok; ++t) {
      const int s = t % nst;
      if (!wait_warp(smem_addr(&full_bar[s]), (t / nst) & 1, p.err, &abort_flag)) break;
      const TileInfo ti = info[s];
      const bool first = (ti.flags & kFirstOfPiece) != 0;
      const bool last = (ti.flags & kLastOfPiece) != 0;
      const bool active = r < ti.rows;
      const int my_member = r / G;
      if (first) {
        m_ref = -INFINITY;
        lsum = 0.f;
      }
      // zero the V rows of a chunk past its valid tokens, up to the 16-token step the
      // P.V product reads (pool slots there may hold anything, and 0 * Inf is NaN)
      {
        uint8_t* vt = smem + static_cast<size_t>(s) * C::STAGE_BYTES + C::K_BYTES;
        for (int q = 0; q < ti.nch; ++q) {
          const int nv = ti.nv[q];
          const int nz = ((nv + 15) & ~15) - nv;  // rows to clear
          for (int idx = tid_s; idx < nz * DCH * 8; idx += kSoftThreads) {
            const int rr = q * kCT + nv + idx / (DCH * 8);
            const int rem = idx % (DCH * 8);
            *reinterpret_cast<uint4*>(vt + (rem >> 3) * C::KV_CHUNK_BYTES + rr * 128 +
                                      (rem & 7) * 16) = make_uint4(0u, 0u, 0u, 0u);
          }
        }
        fence_proxy_async_smem();
      }
      if (!wait_warp(smem_addr(&sfull_bar[t & 1]), (t >> 1) & 1, p.err, &abort_flag)) break;
      tc05::fence_after_sync();
      // this half's scores of chunks h and h + 2, masked: a column past its chunk's valid
      // tokens, an own chunk of another member, or a chunk the tile does not have is -inf
      const bool two = ti.nch > 2;  // the tile reaches chunks 2 and 3
      float x[2][32];
      {
        const uint32_t sa = tmem + ((t & 1) ? kColS1 : kColS0) + lane_addr;
        uint32_t v0[32], v1[32];
        tc05::ld_pair32(sa, v0);
        if (two) tc05::ld_pair32(sa + 64, v1);
        tc05::wait_ld();
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const int q = h + 2 * k;
          const bool mine = q < ti.nch && (ti.mem[q] < 0 || ti.mem[q] == my_member);
          const int nv = mine ? ti.nv[q] : 0;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const uint32_t raw = k == 0 ? v0[j] : v1[j];
            x[k][j] = j < nv ? __uint_as_float(raw) * sl2 : -INFINITY;
          }
        }
      }
      float mt0 = -INFINITY, mt1 = -INFINITY;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        mt0 = fmaxf(mt0, x[0][j]);
        mt1 = fmaxf(mt1, x[1][j]);
      }
      float mt = fmaxf(mt0, mt1);
      mt = fmaxf(mt, __shfl_xor_sync(kFull, mt, 16));
      if (!active) mt = -INFINITY;
      // lazy rescale: move the reference max only when this tile passes it by > 2^8
      const bool raise = mt > m_ref + kRescaleLog2;
      const float new_ref = raise ? mt : m_ref;
      const float alpha = (raise && m_ref > -INFINITY) ? exp2f(m_ref - new_ref) : 1.f;
      // a rescale of O waits for the previous tile's P.V (it accumulates at the old scale)
      if (!first && __any_sync(kFull, alpha != 1.f)) {
        if (!wait_warp(smem_addr(&pvdone_bar[(t - 1) & 1]), ((t - 1) >> 1) & 1, p.err,
                       &abort_flag))
          break;
        tc05::fence_after_sync();
        const uint32_t oa = tmem + kColO + lane_addr;
#pragma unroll
        for (int c = 0; c < D; c += 64) {
          uint32_t v[32];
          tc05::ld_pair32(oa + c, v);
          tc05::wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) * alpha);
          tc05::st_pair32(oa + c, v);
        }
      }
      lsum *= alpha;
      m_ref = new_ref;
      const float mref = m_ref == -INFINITY ? 0.f : m_ref;  // a row with no token yet: p = 0
      {
        float ls0 = 0.f, ls1 = 0.f;
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          if (k == 1 && !two) break;
          uint32_t hi[16], lo[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float p0 = exp2f(x[k][2 * j] - mref), p1 = exp2f(x[k][2 * j + 1] - mref);
            ls0 += p0;
            ls1 += p1;
            split_bf16x2(p0, p1, hi[j], lo[j]);
          }
          // packed P columns of this tile's S buffer: chunks 0|1 at 0..31, 2|3 at 32..63
          const uint32_t pa_ = tmem + ((t & 1) ? kColS1 : kColS0) + lane_addr;
          tc05::st_pair16(pa_ + 32 * k, hi);
          tc05::st_pair16(pa_ + kColPlo + 32 * k, lo);
        }
        lsum += ls0 + ls1;
      }
      tc05::wait_st();
      tc05::fence_before_sync();
      mbar_arrive(smem_addr(&pfull_bar));
      if (last) {
        // the piece's output: wait for its last P.V, read this half of the row of O
        if (!wait_warp(smem_addr(&pvdone_bar[t & 1]), (t >> 1) & 1, p.err, &abort_flag)) break;
        tc05::fence_after_sync();
        const float ltot = lsum + __shfl_xor_sync(kFull, lsum, 16);
        const int kvh = ti.unit % Hkv, ur = ti.unit / Hkv;
        int b = -1;
        if (active) b = ur < NG ? member_of(pp, ur, my_member) : ur - NG;
        const bool complete = (ti.flags & kCompleteUnit) != 0;
        const float inv = ltot > 0.f ? 1.f / ltot : 0.f;
        const size_t prow = (static_cast<size_t>(cta) * 2 + ti.slot) * kRows + r;
        const uint32_t oa = tmem + kColO + lane_addr;
#pragma unroll
        for (int c = 0; c < D; c += 64) {
          uint32_t v[32];
          tc05::ld_pair32(oa + c, v);
          tc05::wait_ld();
          if (!active) continue;
          const int col = c + 32 * h;  // this half's 32 output columns
          if (complete) {
            // a row without output (length 0) is left to the prologue's zero fill
            if (b >= 0 && b < B && ltot > 0.f) {
              uint4* o = reinterpret_cast<uint4*>(
                  out + (static_cast<size_t>(b) * p.Hq + kvh * G + r % G) * D + col);
#pragma unroll
              for (int j = 0; j < 4; ++j)
                o[j] = make_uint4(
                    pack_bf16x2(__uint_as_float(v[8 * j]) * inv, __uint_as_float(v[8 * j + 1]) * inv),
                    pack_bf16x2(__uint_as_float(v[8 * j + 2]) * inv, __uint_as_float(v[8 * j + 3]) * inv),
                    pack_bf16x2(__uint_as_float(v[8 * j + 4]) * inv, __uint_as_float(v[8 * j + 5]) * inv),
                    pack_bf16x2(__uint_as_float(v[8 * j + 6]) * inv, __uint_as_float(v[8 * j + 7]) * inv));
            }
          } else {
            float4* o = reinterpret_cast<float4*>(pp.pacc + prow * D + col);
#pragma unroll
            for (int j = 0; j < 8; ++j)
              o[j] = make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                 __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
          }
        }
        if (active && !complete && h == 0)  // a row with no token here has max -inf, sum 0
          *reinterpret_cast<float2*>(pp.pml + prow * 2) = make_float2(m_ref, ltot);
      }
      if (ti.flags & kLastOfCta) break;
    }
  }

  // ---- exit: every role is done; free the tensor memory --------------------------
  tc05::fence_before_sync();
  __syncthreads();
  tc05::fence_after_sync();
  if (warp == 1) tc05::dealloc(tmem, kTmemCols);
}

// Merge the pieces of units cut by a CTA boundary and write the outputs of their rows.
// Piece i of the unit CTA s owns is slot 0 of CTA s + i, except the first, which is in the
// slot CTA s recorded.  A piece that holds no token of a row has max -inf and is skipped
// for that row.
template <int D>
__global__ void __launch_bounds__(256) group_cut_reduce_kernel(const PrefixParams pp) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const DecodeParams& p = pp.d;
  const int s = blockIdx.x;
  const int4 m = *reinterpret_cast<const int4*>(pp.meta + static_cast<size_t>(s) * 4);
  if (m.x < 0) return;
  const int u = m.x, slot0 = m.y, n = m.z, nrows = m.w;
  const int ur = u / p.Hkv, kvh = u - ur * p.Hkv;
  const int G = p.G;
  constexpr int TPR = D / 4;  // threads per row
  for (int idx = threadIdx.x; idx < nrows * TPR; idx += blockDim.x) {
    const int row = idx / TPR;
    const int c = (idx % TPR) * 4;
    const int b = ur < pp.ngroups ? member_of(pp, ur, row / G) : ur - pp.ngroups;
    float M = -INFINITY, l = 0.f, a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll 4
    for (int i = 0; i < n; ++i) {
      const size_t pr = (static_cast<size_t>(s + i) * 2 + (i == 0 ? slot0 : 0)) * kRows + row;
      const float2 ml = *reinterpret_cast<const float2*>(pp.pml + pr * 2);
      const float4 a = *reinterpret_cast<const float4*>(pp.pacc + pr * D + c);
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
    if (b < 0 || b >= p.B || !(l > 0.f)) continue;  // no output row, or one left to the zero fill
    __nv_bfloat16* o = static_cast<__nv_bfloat16*>(p.out) +
                       (static_cast<size_t>(b) * p.Hq + kvh * G + row % G) * D + c;
    const float inv = 1.f / l;
    *reinterpret_cast<uint2*>(o) = make_uint2(pack_bf16x2(a0 * inv, a1 * inv),
                                              pack_bf16x2(a2 * inv, a3 * inv));
  }
}

// Ring stages that fit the shared memory next to the Q buffers and the unit-row table.
template <class C>
int group_stages(int R) {
  int dev = 0, optin = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
    return 0;
  for (int nst = kMaxStages; nst >= 2; --nst)
    if (group_smem_bytes<C>(nst, R) + kStaticSmemBound <= static_cast<size_t>(optin)) return nst;
  return 0;
}

template <class C>
int group_grid_for(int R, int sms) {
  const int nst = group_stages<C>(R);
  if (nst == 0) return 0;
  int occ = 0;
  const size_t smem = group_smem_bytes<C>(nst, R);
  if (cudaFuncSetAttribute(decode_group_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, decode_group_kernel<C>, kThreads,
                                                    smem) != cudaSuccess || occ < 1)
    return 0;
  return sms;  // one CTA per SM: each holds all of its SM's tensor memory
}

template <class C>
cudaError_t launch_group_cfg(PrefixParams pp, int grid, cudaStream_t stream) {
  CUtensorMap tmk, tmv;
  const DecodeParams& p = pp.d;
  if (!make_pool_map(&tmk, p.k_pool, p.num_blocks, C::BS, p.Hkv, C::D, C::BS) ||
      !make_pool_map(&tmv, p.v_pool, p.num_blocks, C::BS, p.Hkv, C::D, C::BS))
    return cudaErrorInvalidValue;
  const int R = pp.ngroups + p.B;
  const int nst = group_stages<C>(R);
  if (nst == 0) return cudaErrorInvalidValue;
  const size_t smem = group_smem_bytes<C>(nst, R);
  cudaError_t e = cudaFuncSetAttribute(decode_group_kernel<C>,
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
  if ((e = cudaLaunchKernelEx(&cfg, decode_group_kernel<C>, tmk, tmv, pp, nst)) != cudaSuccess)
    return e;
  cfg.gridDim = dim3(static_cast<unsigned>(pp.streams));
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  return cudaLaunchKernelEx(&cfg, group_cut_reduce_kernel<C::D>, pp);
}

}  // namespace

int prefix_grid(int D, int block_size, int R) {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 0;
  switch (D * 100 + block_size) {
    case 6408: return group_grid_for<GroupCfg<64, 8>>(R, sms);
    case 6416: return group_grid_for<GroupCfg<64, 16>>(R, sms);
    case 6432: return group_grid_for<GroupCfg<64, 32>>(R, sms);
    case 12808: return group_grid_for<GroupCfg<128, 8>>(R, sms);
    case 12816: return group_grid_for<GroupCfg<128, 16>>(R, sms);
    case 12832: return group_grid_for<GroupCfg<128, 32>>(R, sms);
    default: return 0;
  }
}

int prefix_warps_per_cta() { return 1; }  // one partial-slot owner per CTA

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
    case 6408: return launch_group_cfg<GroupCfg<64, 8>>(pp, grid, stream);
    case 6416: return launch_group_cfg<GroupCfg<64, 16>>(pp, grid, stream);
    case 6432: return launch_group_cfg<GroupCfg<64, 32>>(pp, grid, stream);
    case 12808: return launch_group_cfg<GroupCfg<128, 8>>(pp, grid, stream);
    case 12816: return launch_group_cfg<GroupCfg<128, 16>>(pp, grid, stream);
    case 12832: return launch_group_cfg<GroupCfg<128, 32>>(pp, grid, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace pa
