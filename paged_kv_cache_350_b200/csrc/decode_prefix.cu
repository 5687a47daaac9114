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
// group's members are stacked as the rows of one tile (members x G <= 64 rows; member m's
// G heads are rows m*G .. m*G + G - 1, the order of q).  A unit's
// tokens are a list of 32-token chunks: first the shared tokens [0, prefix) through the
// first member's table, which every row attends to, then each member's own tokens
// [prefix, L_m) through that member's table, which only that member's rows attend to.  An
// ungrouped sequence is a unit of its own G rows and tokens [0, L).
//
// Schedule.  One persistent CTA per SM; the chunks of all units laid end to end are split
// into equal contiguous ranges, one per CTA, so the work is balanced to one chunk.  A CTA
// walks its range in tiles of up to four chunks (128 tokens) of one unit; a tile may hold
// several members' own chunks (each row masks the chunks that are not its own).  The
// pieces of a unit cut by range boundaries are merged by log-sum-exp in the same launch:
// the later CTAs publish per-row partials (max, sum, unnormalised output), which the CTA
// holding the unit's first chunk folds into its own rows' output.
//
// Per CTA, warp-specialised:
//   warps 0, 1  producers, taking turns tile by tile: resolve block ids through the
//               tables and load each tile's K and V blocks with TMA (one box per block
//               and 64-column chunk) into a ring of stages; warp 0 also loads each unit's
//               Q rows (one box per member) into one of two Q buffers;
//   warp 3      MMA: one thread issues, per tile, S = Q.K^T (M = 64 rows, N = tile
//               tokens, K = head dim; A = Q, B = K, both K-major in shared memory) into
//               one of two S accumulators in tensor memory, and O += P.V (M = 64, once
//               for the P hi parts and once for the P lo parts; A = P from tensor memory,
//               B = V, MN-major in shared memory); S of the next tile is issued as soon as
//               its K has landed, so that it overlaps this tile's softmax;
//   warps 4-11  softmax, two column groups of four warps: group g takes chunks 2g and
//               2g + 1 of every tile, with its own online softmax (fp32, base 2, a lazy
//               rescale: the reference max moves only when a tile's max passes it by more
//               than 2^8, and only then is the group's O rescaled in tensor memory) and
//               its own O accumulator; the groups merge their (max, sum, O) once per
//               piece, when the rows' output (or partial) is read from tensor memory and
//               written out.  P enters the P.V product as two bf16 parts, hi = rn(p) and
//               lo = rn(p - hi), so it keeps ~16 significant bits;
//   warp 2      spare.
// Tensor memory: S buffers at columns 0 and 128 (lanes 0-15 of each sub-partition, the
// M = 64 layout), each overwritten by its P once the softmax has read it (in the row's
// lane, group g's hi parts at columns 64g .. 64g + 31 and its lo parts at 64g + 32 ..
// 64g + 63, packed pairs), so P is double buffered with S; the groups' O accumulators at
// 256 and 384 (the M = 64 layout as well: P hi.V and P lo.V accumulate in the same rows).
// Softmax warps whose rows are all past a unit's rows skip their score reads and P.
//
// Every wait is bounded in time; on expiry the kernel records PA_DEVERR_TIMEOUT, every
// role stops, the loads and tensor-core operations in flight are drained (bounded), and
// the tensor memory is freed before the CTA exits.

#include <cudaTypedefs.h>

#include <atomic>
#include <climits>
#include <random>

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
// Warp roles: producers 0 and 1, a spare, the MMA issuer (warp 3, the one sub-partition
// without a producer), and softmax warps 4-11 (two per sub-partition).
constexpr int kWarps = 12;
constexpr int kMmaWarp = 3;
constexpr int kThreads = kWarps * 32;
constexpr int kSoftThreads = 256;
constexpr int kMaxStages = 4;
constexpr int kMaxMembers = 32;          // members of a group (one per producer lane)
static_assert(kMaxMembers == 32, "a piece keeps member m in producer lane m");
constexpr float kRescaleLog2 = 8.f;      // lazy rescale threshold (log2 units)
static_assert(PA_SHARED_PREFIX_ALIGN % kCT == 0, "a shared prefix ends on a chunk boundary");

// Tensor-memory columns: two S buffers, each overwritten in place by its P, and the two
// column groups' O accumulators (group 0: the tile's chunks 0 and 1, group 1: 2 and 3).
constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO0 = 256, kColO1 = 384;
constexpr uint32_t kTmemCols = 512;

// Tile flags.
constexpr int kFirstOfPiece = 1, kLastOfPiece = 2, kLastOfCta = 4, kCompleteUnit = 8;

struct TileInfo {
  int unit;       // r * Hkv + kvh
  int rows;       // query rows of the unit (members x G)
  int nch;        // chunks in this tile (1..4)
  int flags;
  int piece;      // index of the piece (unit part) within this CTA
  int ubeg, uend; // the unit's chunk range (for the merge of a cut unit)
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

// Static shared memory of the kernel is below this (barriers, tile records: ~560 B).
constexpr size_t kStaticSmemBound = 640;

template <class C>
size_t group_smem_bytes(int nst, int R) {
  return 1024 + static_cast<size_t>(nst) * C::STAGE_BYTES + 2 * C::Q_BYTES +
         static_cast<size_t>(R + 1) * 4;
}

// The step's sequence and group arrays, read through generic pointers: in global memory,
// or in a shared-memory copy the prologue makes (one round trip for all of them).
struct MetaView {
  const int32_t* lens;  // [B] seq_lens
  const int32_t* gof;   // [B] group_of
  const int32_t* pre;   // [ngroups] group_prefix
  const int32_t* mem;   // [ngroups][max_members] group_members
};

// Length of batch row b, clamped to the table's capacity (flagged when out of range).
__device__ __forceinline__ int clamp_len(const DecodeParams& p, const MetaView& mv, int b,
                                         bool flag) {
  int L = mv.lens[b];
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
__device__ __forceinline__ int group_of(const PrefixParams& pp, const MetaView& mv, int b,
                                        bool flag) {
  const int g = mv.gof[b];
  if (g >= pp.ngroups || g < -1) {
    if (flag) flag_error(pp.d.err, PA_DEVERR_BAD_SEQ_LEN);
    return -1;
  }
  return g;
}

// Shared tokens of group r; -1 for a malformed group (flagged): its unit has no chunk.
__device__ __forceinline__ int group_prefix_tokens(const PrefixParams& pp, const MetaView& mv,
                                                   int r, bool flag) {
  const int b0 = mv.mem[static_cast<size_t>(r) * pp.max_members];
  const int pre = mv.pre[r];
  if (b0 < 0 || b0 >= pp.d.B || pre < 0 || pre % PA_SHARED_PREFIX_ALIGN != 0) {
    if (flag) flag_error(pp.d.err, PA_DEVERR_BAD_SEQ_LEN);
    return -1;
  }
  return pre;
}

// Chunks of unit row r (the same for each of its KV heads): a group's shared chunks and
// its members' own chunks (members before the first -1), or an ungrouped row's chunks.
__device__ int row_chunks(const PrefixParams& pp, const MetaView& mv, int r, bool flag) {
  const int NG = pp.ngroups;
  if (r < NG) {
    const int pre = group_prefix_tokens(pp, mv, r, flag);
    if (pre < 0) return 0;
    int n = pre / kCT;
    for (int m = 0; m < pp.max_members; ++m) {
      const int b = mv.mem[static_cast<size_t>(r) * pp.max_members + m];
      if (b < 0) break;
      if (b >= pp.d.B) continue;
      const int L = clamp_len(pp.d, mv, b, flag);
      if (L < pre) {
        if (flag) flag_error(pp.d.err, PA_DEVERR_BAD_SEQ_LEN);
      } else {
        n += (L - pre + kCT - 1) / kCT;
      }
    }
    return n;
  }
  const int b = r - NG;
  if (group_of(pp, mv, b, flag) >= 0) return 0;  // covered by its group's unit
  return (clamp_len(pp.d, mv, b, flag) + kCT - 1) / kCT;
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

template <class C>
__global__ void __launch_bounds__(kThreads, 1)
    decode_group_kernel(const __grid_constant__ CUtensorMap tmk,
                        const __grid_constant__ CUtensorMap tmv,
                        const __grid_constant__ CUtensorMap tmq, const PrefixParams pp,
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

  // kfull / vfull: a stage's K / V have landed (S needs only K); empty: its P.V is done
  __shared__ __align__(8) uint64_t kfull_bar[kMaxStages], vfull_bar[kMaxStages];
  __shared__ __align__(8) uint64_t empty_bar[kMaxStages];
  __shared__ __align__(8) uint64_t qfull_bar[2], qempty_bar[2], sfull_bar[2];
  // pvdone_bar[b]: P.V of the tiles using S buffer b (tiles b, b + 2, ...), one phase each
  __shared__ __align__(8) uint64_t pfull_bar[2], pvdone_bar[2], drain_bar;
  // xch_bar[i][sp]: the two softmax warps of sub-partition sp have posted a piece's
  // (max, sum) in the CTA's exchange slots i (i = piece parity, so a post never meets an
  // unread one); the slots are in global memory, as shared memory is full
  __shared__ __align__(8) uint64_t xch_bar[2][4];
  // cut_bar[0]: the softmax threads have written a cut piece's partial; cut_bar[1]: the
  // partials the owner of a cut unit merges have been published
  __shared__ __align__(8) uint64_t cut_bar[2];
  __shared__ TileInfo info[kMaxStages];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int warp_sum[kWarps];
  __shared__ volatile int abort_flag;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kMaxStages; ++s) {
      mbar_init(smem_addr(&kfull_bar[s]), 1);
      mbar_init(smem_addr(&vfull_bar[s]), 1);
      mbar_init(smem_addr(&empty_bar[s]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_addr(&qfull_bar[i]), 1);
      mbar_init(smem_addr(&qempty_bar[i]), 1);
      mbar_init(smem_addr(&sfull_bar[i]), 1);
    }
    mbar_init(smem_addr(&pfull_bar[0]), kSoftThreads);
    mbar_init(smem_addr(&pfull_bar[1]), kSoftThreads);
    for (int i = 0; i < 8; ++i) mbar_init(smem_addr(&xch_bar[i >> 2][i & 3]), 64);
    mbar_init(smem_addr(&cut_bar[0]), kSoftThreads);
    mbar_init(smem_addr(&cut_bar[1]), 1);
    mbar_init(smem_addr(&pvdone_bar[0]), 1);
    mbar_init(smem_addr(&pvdone_bar[1]), 1);
    mbar_init(smem_addr(&drain_bar), 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    fence_proxy_async_smem();
  }
  if (warp == kMmaWarp) tc05::alloc(smem_addr(&tmem_base_sh), kTmemCols);
  // Launched as a programmatic dependent of the previous kernel on the stream: nothing
  // above reads global memory; wait for that kernel before anything below does.
  asm volatile("griddepcontrol.wait;" ::: "memory");

  // ---- the step's arrays in shared memory (the last stage, unused until the producers
  // have prepared their first piece), in one round trip of independent loads; in global
  // memory when they do not fit -----------------------------------------------------------
  const MetaView gv{p.seq_lens, pp.group_of, pp.group_prefix, pp.group_members};
  MetaView mv = gv;
  {
    const int n_mem = NG * pp.max_members;
    const int n_scr = 2 * B + NG + n_mem;
    if (static_cast<size_t>(n_scr) * 4 <= static_cast<size_t>(C::STAGE_BYTES)) {
      int32_t* scr = reinterpret_cast<int32_t*>(smem + static_cast<size_t>(nst - 1) * C::STAGE_BYTES);
      for (int i = threadIdx.x; i < n_scr; i += kThreads) {
        int32_t v;
        if (i < B) v = __ldg(p.seq_lens + i);
        else if (i < 2 * B) v = __ldg(pp.group_of + (i - B));
        else if (i < 2 * B + NG) v = __ldg(pp.group_prefix + (i - 2 * B));
        else v = __ldg(pp.group_members + (i - 2 * B - NG));
        scr[i] = v;
      }
      mv = MetaView{scr, scr + B, scr + 2 * B, scr + 2 * B + NG};
      __syncthreads();
    }
  }

  // ---- chunk counts of every unit row, scanned (every CTA, identical) ----------------
  for (int r = threadIdx.x; r < R; r += kThreads) P[r] = row_chunks(pp, mv, r, blockIdx.x == 0);
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
    if (clamp_len(p, mv, b, false) == 0) {
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
  // Let the next kernel on the stream be launched now; it waits for this grid to complete
  // before it touches memory.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const float sl2 = p.scale_log2;

  if (warp <= 1) {
    // ============================ producers ============================
    // Two producer warps walk the same tiles and take turns: producer pw loads the tiles t
    // with t % 2 == pw, so that one's tile set-up overlaps the other's loads and the TMA
    // unit stays busy.  Producer 0 alone loads each piece's Q rows and records the CTA's
    // cut-unit slot.
    const int pw = warp;
    // The producers' global loads (block ids, members, lengths) are the step's latency
    // chain, each a round trip of about a microsecond, so none is issued where it is used:
    //   * block ids are loaded 64 at a time (two per lane), one batch ahead: a batch holds
    //     the ids of 64 / BPC chunks (2 to 16 tiles);
    //   * the next piece (members, lengths, first two batches, then its Q rows by TMA) is
    //     prepared while this one streams, one dependent step after each of its tiles.
    const uint64_t policy = l2_policy_evict_first();
    if (lane == 0) {
      prefetch_tensormap(&tmk);
      prefetch_tensormap(&tmv);
      prefetch_tensormap(&tmq);
    }
    // One unit piece (the part of a unit inside this CTA's range); lane m holds member m.
    struct Piece {
      int g, pend, ubeg, uend, r, kvh, j;  // first chunk, end; unit bounds, row, head, chunk
      int mb, mL, mst;                     // member's batch row, length, first own chunk
      int pre, n0, gs, rows;               // shared tokens and chunks, members, query rows
    };
    // A piece is prepared in three steps, each consuming the loads the one before issued,
    // so that the producer can spread them over the tiles it issues meanwhile:
    //   (a) locate the unit; load the member ids and the shared-token count;
    //   (b) the members before the first -1; load their lengths;
    //   (c) each member's own chunks and where they start (a scan over the lanes).
    auto prep_a = [&](const MetaView& v, int g, Piece& pc, int& pre_raw) {
      const UnitPos u = locate(P, R, Hkv, g);
      pc.g = g;
      pc.ubeg = g - u.j;
      pc.uend = pc.ubeg + u.nt;
      pc.pend = min(end, pc.uend);
      pc.r = u.r;
      pc.kvh = u.kvh;
      pc.j = u.j;
      pre_raw = 0;
      if (u.r < NG) {
        pc.mb = lane < pp.max_members ? v.mem[static_cast<size_t>(u.r) * pp.max_members + lane] : -1;
        if (lane == 0) pre_raw = v.pre[u.r];
      } else {
        pc.mb = lane == 0 ? u.r - NG : -1;
      }
    };
    auto prep_b = [&](const MetaView& v, Piece& pc, int pre_raw, int& len_raw) {
      const bool grp = pc.r < NG;
      const unsigned live_mask = __ballot_sync(kFull, pc.mb >= 0);
      const int gs = grp ? (~live_mask ? __ffs(~live_mask) - 1 : 32) : 1;  // before the first -1
      if (lane >= gs) pc.mb = -1;
      int pre = 0;
      if (grp) {  // a malformed group (flagged in the prologue) has no shared tokens here
        const int b0 = __shfl_sync(kFull, pc.mb, 0);
        const int pr = __shfl_sync(kFull, pre_raw, 0);
        pre = (b0 < 0 || b0 >= B || pr < 0 || pr % PA_SHARED_PREFIX_ALIGN != 0) ? 0 : pr;
      }
      pc.pre = pre;
      pc.gs = gs;
      pc.n0 = pre / kCT;
      pc.rows = gs * G;
      len_raw = (pc.mb >= 0 && pc.mb < B) ? v.lens[pc.mb] : 0;
    };
    auto prep_c = [&](Piece& pc, int len_raw) {
      const int Lmax = p.max_blocks * p.block_size;  // lengths clamped as the prologue does
      pc.mL = (pc.mb >= 0 && pc.mb < B) ? min(max(len_raw, 0), Lmax) : 0;
      const int own = (pc.mb >= 0 && pc.mb < B && pc.mL >= pc.pre)
                          ? (pc.mL - pc.pre + kCT - 1) / kCT : 0;
      int incl = own;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(kFull, incl, off);
        if (lane >= off) incl += v;
      }
      pc.mst = pc.n0 + incl - own;
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
    // the piece's chunk n * CPB + k / BPC (kNoBlock where there is none), with that chunk's
    // record (valid tokens | (member + 1) << 8; 0 past the piece), so that a tile's records
    // and block ids are shuffles.  A tile never straddles two batches (CPB is a multiple
    // of the 4 chunks of a tile, and tiles start every 4 chunks of a piece).
    constexpr int CPB = 64 / C::BPC;
    constexpr int kNoBlock = INT_MIN;
    struct Batch {
      int id[2], rec[2];
    };
    auto load_batch = [&](const Piece& pc, int n, Batch& bt) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int k = lane + 32 * e;
        const int jrel = n * CPB + k / C::BPC;
        const int i = k % C::BPC;
        int tb, t0, nv, mem;
        chunk_src(pc, pc.j + jrel, tb, t0, nv, mem);
        const bool in = pc.g + jrel < pc.pend;
        const bool live = in && i * BS < nv && tb >= 0 && tb < B;
        bt.id[e] = live ? __ldg(p.block_tables + static_cast<size_t>(tb) * p.max_blocks + t0 / BS + i)
                        : kNoBlock;
        bt.rec[e] = in ? (nv | ((mem + 1) << 8)) : 0;
      }
    };
    // A piece's Q rows into Q buffer qb with TMA: member m's G query heads of this KV head
    // are G consecutive rows of q and land at rows m*G.. of the buffer (one box per member
    // and 64-column chunk, written 128-byte swizzled as the MMA reads it); a member outside
    // the batch reads zeros.  Rows past the unit are left as they are: their scores are
    // masked and their P is 0.  The buffer's barrier completes when the bytes have landed.
    auto load_q = [&](const Piece& pc, int qb) {
      const uint32_t bar = smem_addr(&qfull_bar[qb]);
      if (lane == 0) mbar_arrive_expect_tx(bar, static_cast<uint32_t>(pc.gs * G * D * 2));
      __syncwarp();
      if (lane < pc.gs) {
        const uint32_t qt = smem_addr(qbuf + qb * C::Q_BYTES) + lane * G * 128;
#pragma unroll
        for (int c = 0; c < DCH; ++c)
          tma_load_3d(qt + c * C::Q_CHUNK_BYTES, &tmq, c * 64, pc.kvh * G, pc.mb, bar, policy);
      }
      __syncwarp();
    };

    int q_loads = 0;  // Q loads issued (pieces 0 .. q_loads - 1)
    int t = 0, piece = 0;
    bool ok = beg < end;
    Piece pc, nx;
    Batch cur, nxt, nb0, nb1;
    int nx_pre = 0, nx_len = 0;
    if (ok) {
      int pre_raw, len_raw;
      prep_a(mv, beg, pc, pre_raw);
      prep_b(mv, pc, pre_raw, len_raw);
      prep_c(pc, len_raw);
      if (pw == 0) {
        load_q(pc, 0);
        q_loads = 1;
      }
      load_batch(pc, 0, cur);
      load_batch(pc, 1, nxt);
    }
    // both producers have read the prologue's copy of the step's arrays (in the last
    // stage) before either loads a tile
    asm volatile("bar.sync 1, 64;" ::: "memory");
    while (ok) {
      const bool complete = pc.g == pc.ubeg && pc.pend == pc.uend;
      const bool has_next = pc.pend < end;
      // steps of the next piece's preparation done (4: all; producer 1 has no Q step)
      int prep = has_next ? 0 : 4;
      int batch = 0;        // batch held in cur
      for (int c0 = pc.g; ok;) {
        const int nch = min(kCPT, pc.pend - c0);
        const int jrel = c0 - pc.g;
        if (jrel / CPB != batch) {  // move to the next batch; load the one after it
          cur = nxt;
          ++batch;
          load_batch(pc, batch + 1, nxt);
        }
        const int s = t % nst;
        const bool mine = (t & 1) == pw;
        if (mine && t >= nst) {
          ok = wait_lane0(smem_addr(&empty_bar[s]), ((t / nst) - 1) & 1, p.err, &abort_flag);
          if (!ok) break;
        }
        const bool last_of_piece = c0 + nch >= pc.pend;
        if (mine) {
          // chunk q of the tile: member and valid tokens, for the record (from the batch)
          int qm[kCPT], qv[kCPT];
#pragma unroll
          for (int q = 0; q < kCPT; ++q) {
            const int kq = (jrel % CPB + q) * C::BPC;
            const int r0 = __shfl_sync(kFull, cur.rec[0], kq & 31);
            const int r1 = __shfl_sync(kFull, cur.rec[1], kq & 31);
            const int rec = q < nch ? ((kq >> 5) ? r1 : r0) : 0;
            qm[q] = q < nch ? (rec >> 8) - 1 : -1;
            qv[q] = rec & 0xFF;
          }
          if (lane == 0) {
            TileInfo* ti = &info[s];
            ti->unit = pc.r * Hkv + pc.kvh;
            ti->rows = pc.rows;
            ti->nch = nch;
            ti->piece = piece;
            ti->ubeg = pc.ubeg;
            ti->uend = pc.uend;
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
          const int a0 = __shfl_sync(kFull, cur.id[0], k & 31);
          const int a1 = __shfl_sync(kFull, cur.id[1], k & 31);
          int phys = (k >> 5) ? a1 : a0;
          const bool live = lane < nch * C::BPC && phys != kNoBlock;
          if (live && (phys < 0 || phys >= p.num_blocks)) {
            flag_error(p.err, PA_DEVERR_BAD_BLOCK_ID);
            phys = 0;
          }
          const int nboxes = __popc(__ballot_sync(kFull, live));
          const uint32_t kb = smem_addr(&kfull_bar[s]), vb = smem_addr(&vfull_bar[s]);
          if (lane == 0) {
            fence_proxy_async_smem();  // this stage's earlier generic writes come first
            mbar_arrive_expect_tx(kb, static_cast<uint32_t>(nboxes * BS * D * 2));
            mbar_arrive_expect_tx(vb, static_cast<uint32_t>(nboxes * BS * D * 2));
          }
          __syncwarp();
          if (live) {  // every K box first (S needs only K), then the V boxes
            const int q = lane / C::BPC, i = lane % C::BPC;
            const uint32_t kt = smem_addr(smem + static_cast<size_t>(s) * C::STAGE_BYTES) +
                                (q * kCT + i * BS) * 128;
            const uint32_t vt = kt + C::K_BYTES;
#pragma unroll
            for (int c = 0; c < DCH; ++c)
              tma_load_4d(kt + c * C::KV_CHUNK_BYTES, &tmk, c * 64, pc.kvh, 0, phys, kb, policy);
#pragma unroll
            for (int c = 0; c < DCH; ++c)
              tma_load_4d(vt + c * C::KV_CHUNK_BYTES, &tmv, c * 64, pc.kvh, 0, phys, vb, policy);
          }
          __syncwarp();
        }
        ++t;
        // the next piece: one preparation step after each tile of this one (all that are
        // left after its last tile), so its loads land while this piece streams
        while (prep < 4) {
          if (prep == 0) {
            prep_a(gv, pc.pend, nx, nx_pre);
          } else if (prep == 1) {
            prep_b(gv, nx, nx_pre, nx_len);
          } else if (prep == 2) {
            prep_c(nx, nx_len);
            load_batch(nx, 0, nb0);
            load_batch(nx, 1, nb1);
          } else if (pw == 0) {
            // its Q buffer was last read by the piece before this one (the wait is for the
            // S of that piece's last tile)
            const int qn = piece + 1;
            if (qn >= 2) {
              ok = wait_lane0(smem_addr(&qempty_bar[qn & 1]), ((qn >> 1) - 1) & 1, p.err,
                              &abort_flag);
              if (!ok) break;
            }
            load_q(nx, qn & 1);
            q_loads = qn + 1;
          }
          ++prep;
          if (!last_of_piece) break;
        }
        if (!ok) break;
        if (last_of_piece) break;
        c0 += nch;
      }
      if (!ok || !has_next) break;
      pc = nx;
      cur = nb0;
      nxt = nb1;
      ++piece;
    }
    if (!ok) {
      // wait (bounded) for this producer's loads issued but never consumed, so none lands
      // after exit: the last two Q loads and the last tiles
      if (pw == 0)
        for (int n = max(0, q_loads - 2); n < q_loads; ++n)
          mbar_wait(smem_addr(&qfull_bar[n & 1]), (n >> 1) & 1, nullptr, kWaitLimitNs);
      for (int k = max(0, t - nst - 1); k < t; ++k) {
        if ((k & 1) != pw) continue;
        mbar_wait(smem_addr(&kfull_bar[k % nst]), (k / nst) & 1, nullptr, kWaitLimitNs);
        mbar_wait(smem_addr(&vfull_bar[k % nst]), (k / nst) & 1, nullptr, kWaitLimitNs);
      }
    }
  } else if (warp == 2) {
    // spare: no work after the prologue
  } else if (warp == kMmaWarp) {
    // ============================ MMA issuer ============================
    if (lane == 0 && beg < end) {
      const uint32_t id_s_base = tc05::instr_desc_bf16(kRows, 8, 0) & ~(0x3Fu << 17);
      const uint32_t id_pv = tc05::instr_desc_bf16(kRows, D, 1);
      bool ok = true;
      // The tile records are read from shared memory where they are used (a record stays
      // until its stage is released after the tile's P.V), and every loop below is
      // unrolled, so the issuing thread keeps its state in registers.
      // S of tile t (its stage's K has landed)
      auto issue_s = [&](int t) -> bool {
        const int s = t % nst;
        const int flags = info[s].flags, piece = info[s].piece, nch = info[s].nch;
        const int qb = piece & 1;
        if ((flags & kFirstOfPiece) &&
            !wait_or_abort(smem_addr(&qfull_bar[qb]), (piece >> 1) & 1, p.err, &abort_flag))
          return false;
        tc05::fence_after_sync();
        const uint32_t qa = smem_addr(qbuf + qb * C::Q_BYTES);
        const uint32_t ka = smem_addr(smem + static_cast<size_t>(s) * C::STAGE_BYTES);
        const uint32_t idesc = id_s_base | (static_cast<uint32_t>((nch * kCT) >> 3) << 17);
        const uint32_t ts = tmem + ((t & 1) ? kColS1 : kColS0);
        // this S buffer's P was last read by P.V of tile t - 2: it must have completed (the
        // buffer's barrier has one phase per use, and the use before that was waited for
        // when S of tile t - 2 was issued)
        if (t >= 2 && !wait_or_abort(smem_addr(&pvdone_bar[t & 1]), ((t - 2) >> 1) & 1, p.err,
                                     &abort_flag))
          return false;
        // descriptors of the operands' starts; a k-step moves the start address field
        // (16-byte units) by its byte offset
        const uint64_t dq = tc05::smem_desc(qa, 16, 1024), dk = tc05::smem_desc(ka, 16, 1024);
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off_q = (k >> 2) * C::Q_CHUNK_BYTES + (k & 3) * 32;
          const uint32_t off_k = (k >> 2) * C::KV_CHUNK_BYTES + (k & 3) * 32;
          tc05::mma_ss(ts, dq + (off_q >> 4), dk + (off_k >> 4), idesc, k > 0);
        }
        tc05::commit(smem_addr(&sfull_bar[t & 1]));
        if (flags & kLastOfPiece) tc05::commit(smem_addr(&qempty_bar[qb]));
        return true;
      };
      bool fresh0 = true, fresh1 = true;  // accumulator not yet written in this piece
      // One event loop, so that S and P.V each have a single issue site: in step t, P.V of
      // tile t is issued once its P is written, and S of tile t + 1 as soon as its K has
      // landed and the P.V that last read its S buffer (tile t - 1) is done, whichever
      // comes first, so that S of the next tile overlaps this tile's softmax and P.V never
      // waits for the next tile's loads.  Step -1 only issues S of tile 0.  P of tile t
      // has one barrier per S buffer, since the softmax may finish tile t + 1 first.
      uint64_t idle_since = 0;
      for (int t = -1; ok; ++t) {
        const int s = t >= 0 ? t % nst : 0;
        const int flags = t >= 0 ? info[s].flags : 0;
        const bool more = !(flags & kLastOfCta);
        const int s1 = (t + 1) % nst;
        const uint32_t kb1 = smem_addr(&kfull_bar[s1]), par1 = ((t + 1) / nst) & 1;
        const uint32_t db = smem_addr(&pvdone_bar[(t + 1) & 1]), dpar = ((t - 1) >> 1) & 1;
        const uint32_t pb = smem_addr(&pfull_bar[t & 1]), ppar = (t >> 1) & 1;
        bool s_next = !more, pv_done = t < 0;
        while (!(s_next && pv_done)) {
          bool progress = false;
          if (!s_next && mbar_test_wait(kb1, par1) && (t < 1 || mbar_test_wait(db, dpar))) {
            ok = issue_s(t + 1);
            if (!ok) break;
            s_next = progress = true;
          }
          if (!pv_done && mbar_test_wait(pb, ppar)) {
            // (the softmax waited for this stage's V before it zeroed V's tail rows)
            tc05::fence_after_sync();
            const int nch = info[s].nch;
            const uint64_t dv = tc05::smem_desc(
                smem_addr(smem + static_cast<size_t>(s) * C::STAGE_BYTES) + C::K_BYTES,
                C::KV_CHUNK_BYTES, 1024);
            const uint32_t tp = tmem + ((t & 1) ? kColS1 : kColS0);  // P of tile t
            if (flags & kFirstOfPiece) fresh0 = fresh1 = true;
            // chunk q's P hi parts at S columns 64 * (q / 2) + 16 * (q % 2), its lo parts 32
            // columns on; chunks 0-1 go into O0, 2-3 into O1 (hi, then lo, accumulated); a
            // chunk's second 16-token step only where it has valid tokens
#pragma unroll
            for (int q = 0; q < kCPT; ++q) {
              if (q < nch) {
                const int nvq = info[s].nv[q];
#pragma unroll
                for (int kk = 0; kk < 2; ++kk) {
                  if (kk == 0 || nvq > 16) {
                    const int k = 2 * q + kk;
                    const uint64_t vdesc = dv + (k * 2048 >> 4);
                    const uint32_t pa = tp + 64 * (q >> 1) + 16 * (q & 1) + 8 * kk;
                    if (q < 2) {
                      tc05::mma_ts(tmem + kColO0, pa, vdesc, id_pv, !fresh0);
                      tc05::mma_ts(tmem + kColO0, pa + 32, vdesc, id_pv, true);
                      fresh0 = false;
                    } else {
                      tc05::mma_ts(tmem + kColO1, pa, vdesc, id_pv, !fresh1);
                      tc05::mma_ts(tmem + kColO1, pa + 32, vdesc, id_pv, true);
                      fresh1 = false;
                    }
                  }
                }
              }
            }
            tc05::commit(smem_addr(&pvdone_bar[t & 1]));
            tc05::commit(smem_addr(&empty_bar[s]));
            pv_done = progress = true;
          }
          if (progress) {
            idle_since = 0;
            continue;
          }
          if (abort_flag) {
            ok = false;
            break;
          }
          const uint64_t now = global_timer_ns();
          if (idle_since == 0) {
            idle_since = now;
          } else if (now - idle_since > kWaitLimitNs) {
            flag_error(p.err, PA_DEVERR_TIMEOUT);
            ok = false;
            break;
          }
          // nothing ready: a short pause, then look at both events again (a wait on one of
          // them would hold up the other: S of the next tile is due as soon as its K has
          // landed, P.V of this one as soon as its P is written)
          __nanosleep(32);
        }
        if (!more) break;
      }
      if (!ok) abort_flag = 1;
      // every tensor-core operation issued has completed before the memory is freed
      tc05::commit(smem_addr(&drain_bar));
      mbar_wait(smem_addr(&drain_bar), 0, p.err);
    }
    __syncwarp();
  } else {
    // ============================ softmax ============================
    // Two column groups of four warps: group g takes chunks 2g and 2g + 1 of every tile,
    // with its own online-softmax state and its own O accumulator, and the two merge once
    // per piece.  Warp w serves tensor-memory sub-partition sp = w % 4, whose lanes 0-15
    // hold S rows 16*sp .. 16*sp + 15 (the M = 64 accumulator layout); one warp of each
    // group serves each sub-partition.  Threads t and t + 16 share the row of lane t % 16
    // when reading S (the 16x32bx2 shape): half h = t / 16 takes chunk 2g + h, so a row's
    // max and sum within the group combine by one shuffle.  P goes back over the group's
    // S columns in the same shape, each half writing its own chunk's hi parts and lo
    // parts in separate column blocks, so P.V is two M = 64 products per 16 tokens (hi,
    // then lo) into the same accumulator rows, and no lane exchange is needed.
    const int sp = warp & 3;                    // tensor-memory sub-partition
    const int grp = (warp - 4) >> 2;            // column group
    const int h = lane >> 4;                    // chunk within the group's pair
    const int q_mine = 2 * grp + h;             // this thread's chunk of a tile
    const int r = 16 * sp + (lane & 15);        // this thread's query row (= MMA row)
    const uint32_t lane_addr = static_cast<uint32_t>(32 * sp) << 16;
    const uint32_t col_o = grp ? kColO1 : kColO0;
    const int tid_g = (warp & 3) * 32 + lane;   // 0..127 within the group
    float m_ref = -INFINITY, lsum = 0.f;        // lsum: this thread's part of the row sum
    int b_row = -1;  // the row's batch row, loaded at the piece's first tile, used at its end
    int pub_uses = 0, own_uses = 0;  // phases of cut_bar[0] and cut_bar[1]
    // A unit cut by CTA range boundaries: its first piece is the last piece of the CTA c0
    // holding its first chunk (the owner), each other piece the first piece of a later
    // CTA.  A later CTA writes its piece's partial (max, sum, unnormalised output per row)
    // and publishes it with an epoch-tagged flag; the owner, at its piece's end, takes
    // those partials and merges them with its own piece by log-sum-exp as it writes the
    // rows' output.  The other pieces are at the start of their CTAs' ranges, so the
    // owner's wait (bounded) has normally ended before it begins; every CTA of the grid is
    // resident before any later kernel can be (a dependent grid launches only once each
    // CTA has passed the prologue's trigger), so the CTAs it waits for do run.
    auto publish_partial = [&](int use) -> bool {
      mbar_arrive(smem_addr(&cut_bar[0]));  // release: this thread's partial first
      if (threadIdx.x == 4 * 32) {
        if (!wait_or_abort(smem_addr(&cut_bar[0]), use & 1, p.err, &abort_flag)) return false;
        st_release_gpu(pp.cut_flag + cta, pp.epoch);
      }
      return true;
    };
    // The owner: wait for the flags of CTAs c0 + 1 .. c0 + n - 1 (one thread), then let
    // every softmax thread read the partials.
    auto await_partials = [&](int n, int use) -> bool {
      if (threadIdx.x == 4 * 32) {
        const uint64_t t0 = global_timer_ns();
        for (int i = 1; i < n && !abort_flag; ++i) {
          while (ld_acquire_gpu(pp.cut_flag + cta + i) != pp.epoch) {
            if (abort_flag) break;
            if (global_timer_ns() - t0 > kWaitLimitNs) {
              flag_error(p.err, PA_DEVERR_TIMEOUT);
              abort_flag = 1;
              break;
            }
          }
        }
        mbar_arrive(smem_addr(&cut_bar[1]));  // release: the acquired flags come first
      }
      return wait_warp(smem_addr(&cut_bar[1]), use & 1, p.err, &abort_flag) && !abort_flag;
    };
    bool ok = beg < end;
    for (int t = 0; ok; ++t) {
      const int s = t % nst;
      if (!wait_warp(smem_addr(&kfull_bar[s]), (t / nst) & 1, p.err, &abort_flag)) break;
      const TileInfo ti = info[s];
      const bool first = (ti.flags & kFirstOfPiece) != 0;
      const bool last = (ti.flags & kLastOfPiece) != 0;
      const bool active = r < ti.rows;
      const int my_member = r / G;
      const bool has = ti.nch > 2 * grp;        // the tile reaches this group's chunks
      // a warp whose 16 rows are all past the unit's rows (a unit of up to 32 rows leaves
      // sub-partitions 2 and 3 idle) keeps only the barrier protocol and its share of the V
      // zeroing: the P rows it leaves unwritten only reach accumulator rows never output
      const bool live = has && 16 * sp < ti.rows;
      if (first) {
        m_ref = -INFINITY;
        lsum = 0.f;
        const int ur = ti.unit / Hkv;
        b_row = !active ? -1 : ur < NG ? member_of(pp, ur, my_member) : ur - NG;
      }
      if (!wait_warp(smem_addr(&sfull_bar[t & 1]), (t >> 1) & 1, p.err, &abort_flag)) break;
      tc05::fence_after_sync();
      const uint32_t sbuf = tmem + ((t & 1) ? kColS1 : kColS0) + lane_addr;
      float x[32];  // this thread's chunk of raw scores; -inf where masked
      float mt = -INFINITY;
      if (live) {
        uint32_t v[32];
        tc05::ld_pair32(sbuf + 64 * grp, v);
        tc05::wait_ld();
        // a column past its chunk's valid tokens, an own chunk of another member, or a
        // chunk the tile does not have is masked (the per-chunk fields are read from the
        // stage's record, which stays until the stage is released after this tile's P.V);
        // most tiles need no mask at all
        const int mq = info[s].mem[q_mine];
        const bool mine = q_mine < ti.nch && (mq < 0 || mq == my_member);
        const int nv = mine && active ? info[s].nv[q_mine] : 0;
        float mr = -INFINITY;
        if (__all_sync(kFull, nv == kCT)) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            x[j] = __uint_as_float(v[j]);
            mr = fmaxf(mr, x[j]);
          }
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            x[j] = j < nv ? __uint_as_float(v[j]) : -INFINITY;
            mr = fmaxf(mr, x[j]);
          }
        }
        mr = fmaxf(mr, __shfl_xor_sync(kFull, mr, 16));
        mt = mr * sl2;  // the scale is positive: the max commutes with it
      }
      // lazy rescale: move the reference max only when this tile passes it by > 2^8
      const bool raise = mt > m_ref + kRescaleLog2;
      const float new_ref = raise ? mt : m_ref;
      const float alpha = (raise && m_ref > -INFINITY) ? ex2_approx(m_ref - new_ref) : 1.f;
      // a rescale of O waits for the previous tile's P.V (it accumulates at the old scale)
      if (!first && __any_sync(kFull, alpha != 1.f)) {
        if (!wait_warp(smem_addr(&pvdone_bar[(t - 1) & 1]), ((t - 1) >> 1) & 1, p.err,
                       &abort_flag))
          break;
        tc05::fence_after_sync();
        const uint32_t oa = tmem + col_o + lane_addr;  // the row's O (lanes 0-15)
#pragma unroll
        for (int c = 0; c < D; c += 64) {
          uint32_t v[32];
          tc05::ld_pair32(oa + c, v);  // this half's 32 of the 64 columns
          tc05::wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) * alpha);
          tc05::st_pair32(oa + c, v);
        }
      }
      lsum *= alpha;
      m_ref = new_ref;
      const float mref = m_ref == -INFINITY ? 0.f : m_ref;  // a row with no token yet: p = 0
      // zero the V rows of this group's chunks past their valid tokens, up to the
      // 16-token step the P.V product reads (pool slots there may hold anything, and
      // 0 * Inf is NaN)
      if (!wait_warp(smem_addr(&vfull_bar[s]), (t / nst) & 1, p.err, &abort_flag)) break;
      if (has) {
        uint8_t* vt = smem + static_cast<size_t>(s) * C::STAGE_BYTES + C::K_BYTES;
        for (int q = 2 * grp; q < min(ti.nch, 2 * grp + 2); ++q) {
          const int nv = info[s].nv[q];
          const int nz = ((nv + 15) & ~15) - nv;  // rows to clear
          for (int idx = tid_g; idx < nz * DCH * 8; idx += 128) {
            const int rr = q * kCT + nv + idx / (DCH * 8);
            const int rem = idx % (DCH * 8);
            *reinterpret_cast<uint4*>(vt + (rem >> 3) * C::KV_CHUNK_BYTES + rr * 128 +
                                      (rem & 7) * 16) = make_uint4(0u, 0u, 0u, 0u);
          }
        }
        fence_proxy_async_smem();
      }
      if (live) {
        // P over this group's S columns, in the row's lane: the hi parts of chunks 2g and
        // 2g + 1 (packed pairs) at columns 64g .. 64g + 31, their lo parts at 64g + 32 ..
        // 64g + 63; each half of the lane pair writes its own chunk (the 16x32bx2 shape)
        uint32_t whi[16], wlo[16];
        float ls = 0.f;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          // p = 2^(s * scale * log2(e) - m); a masked score (-inf) gives 0
          const float p0 = ex2_approx(fmaf(x[2 * j], sl2, -mref));
          const float p1 = ex2_approx(fmaf(x[2 * j + 1], sl2, -mref));
          ls += p0 + p1;
          split_bf16x2(p0, p1, whi[j], wlo[j]);
        }
        tc05::st_pair16(sbuf + 64 * grp, whi);
        tc05::st_pair16(sbuf + 64 * grp + 32, wlo);
        lsum += ls;
        tc05::wait_st();
      }
      tc05::fence_before_sync();
      mbar_arrive(smem_addr(&pfull_bar[t & 1]));
      if (last) {
        // the piece's output: post this group's (max, sum) of the row, take the other
        // group's, and wait for the piece's last P.V
        const float lgrp = lsum + __shfl_xor_sync(kFull, lsum, 16);
        const int xi = ti.piece & 1;
        float2* xch = reinterpret_cast<float2*>(pp.pxch) + (static_cast<size_t>(cta) * 2 + xi) * 2 * kRows;
        if (h == 0) xch[grp * kRows + r] = make_float2(m_ref, lgrp);
        mbar_arrive(smem_addr(&xch_bar[xi][sp]));  // release: the post comes first
        if (!wait_warp(smem_addr(&xch_bar[xi][sp]), (ti.piece >> 1) & 1, p.err, &abort_flag))
          break;
        const float2 ml0 = xch[r], ml1 = xch[kRows + r];
        const float mx = fmaxf(ml0.x, ml1.x);
        const float w0 = ml0.x == -INFINITY ? 0.f : ex2_approx(ml0.x - mx);
        const float w1 = ml1.x == -INFINITY ? 0.f : ex2_approx(ml1.x - mx);
        const float ltot = w0 * ml0.y + w1 * ml1.y;
        if (!wait_warp(smem_addr(&pvdone_bar[t & 1]), (t >> 1) & 1, p.err, &abort_flag)) break;
        tc05::fence_after_sync();
        const int kvh = ti.unit % Hkv;
        const int b = b_row;
        const bool complete = (ti.flags & kCompleteUnit) != 0;
        const bool owner = !complete && ti.ubeg >= beg;  // the unit's first chunk is here
        const int n = owner ? (ti.uend - 1) / per - cta + 1 : 1;  // pieces of the unit
        // the owner merges the partials of the unit's other pieces (those of CTAs
        // cta + 1 .. cta + n - 1) with its own: the row's max, its own weight, the sum
        float M = mx, e_own = 1.f, L = ltot;
        if (n > 1) {
          if (!await_partials(n, own_uses++)) break;
          for (int i = 1; i < n; ++i)
            M = fmaxf(M, __ldcg(reinterpret_cast<const float2*>(pp.pml) +
                                static_cast<size_t>(cta + i) * kRows + r).x);
          e_own = mx == -INFINITY ? 0.f : ex2_approx(mx - M);
          L = e_own * ltot;
          for (int i = 1; i < n; ++i) {
            const float2 ml = __ldcg(reinterpret_cast<const float2*>(pp.pml) +
                                     static_cast<size_t>(cta + i) * kRows + r);
            L += ml.x == -INFINITY ? 0.f : ex2_approx(ml.x - M) * ml.y;
          }
        }
        const float inv = L > 0.f ? 1.f / L : 0.f;
        const size_t prow = static_cast<size_t>(cta) * kRows + r;  // this CTA's partial row
        // group g writes output columns [g * D / 2, (g + 1) * D / 2): each half of the lane
        // pair reads W = D / 4 of them from both accumulators (the row's lane)
        {
          constexpr int W = D / 4;
          const int c = grp * D / 2;
          uint32_t a0[W], a1[W];
          if constexpr (W == 32) {
            tc05::ld_pair32(tmem + kColO0 + lane_addr + c, a0);
            tc05::ld_pair32(tmem + kColO1 + lane_addr + c, a1);
          } else {
            tc05::ld_pair16(tmem + kColO0 + lane_addr + c, a0);
            tc05::ld_pair16(tmem + kColO1 + lane_addr + c, a1);
          }
          tc05::wait_ld();
          const int col = c + W * h;  // this thread's W columns
          float vv[W];
#pragma unroll
          for (int j = 0; j < W; ++j)
            // an accumulator with weight 0 may never have been written in this piece
            vv[j] = ((w0 > 0.f ? w0 * __uint_as_float(a0[j]) : 0.f) +
                     (w1 > 0.f ? w1 * __uint_as_float(a1[j]) : 0.f)) * e_own;
          if (active) {
            // the other pieces' partials (the owner of a cut unit)
            for (int i = 1; i < n; ++i) {
              const size_t pr = static_cast<size_t>(cta + i) * kRows + r;
              const float2 ml = __ldcg(reinterpret_cast<const float2*>(pp.pml) + pr);
              if (ml.x == -INFINITY) continue;
              const float wi = ex2_approx(ml.x - M);
              const float4* src = reinterpret_cast<const float4*>(pp.pacc + pr * D + col);
#pragma unroll
              for (int j = 0; j < W / 4; ++j) {
                const float4 a = __ldcg(src + j);
                vv[4 * j] += wi * a.x;
                vv[4 * j + 1] += wi * a.y;
                vv[4 * j + 2] += wi * a.z;
                vv[4 * j + 3] += wi * a.w;
              }
            }
            if (complete || owner) {
              // a row without output (length 0) is left to the prologue's zero fill
              if (b >= 0 && b < B && L > 0.f) {
                uint4* o = reinterpret_cast<uint4*>(
                    out + (static_cast<size_t>(b) * p.Hq + kvh * G + r % G) * D + col);
#pragma unroll
                for (int j = 0; j < W / 8; ++j)
                  o[j] = make_uint4(pack_bf16x2(vv[8 * j] * inv, vv[8 * j + 1] * inv),
                                    pack_bf16x2(vv[8 * j + 2] * inv, vv[8 * j + 3] * inv),
                                    pack_bf16x2(vv[8 * j + 4] * inv, vv[8 * j + 5] * inv),
                                    pack_bf16x2(vv[8 * j + 6] * inv, vv[8 * j + 7] * inv));
              }
            } else {  // a later piece of a cut unit: its partial, for the owner
              float4* o = reinterpret_cast<float4*>(pp.pacc + prow * D + col);
#pragma unroll
              for (int j = 0; j < W / 4; ++j)
                o[j] = make_float4(vv[4 * j], vv[4 * j + 1], vv[4 * j + 2], vv[4 * j + 3]);
            }
          }
        }
        if (n > 1 && threadIdx.x == 4 * 32) {
          // consumed: clear the flags, so that a replay of this same launch (a CUDA graph
          // keeps its tag) waits for fresh partials
          for (int i = 1; i < n; ++i) pp.cut_flag[cta + i] = 0ull;
        }
        if (!complete && !owner) {
          // a row with no token here has max -inf, sum 0
          if (active && grp == 0 && h == 0)
            *reinterpret_cast<float2*>(pp.pml + prow * 2) = make_float2(mx, ltot);
          if (!publish_partial(pub_uses++)) break;
        }
      }
      if (ti.flags & kLastOfCta) break;
    }
  }

  // ---- exit: every role is done; free the tensor memory --------------------------
  tc05::fence_before_sync();
  __syncthreads();
  tc05::fence_after_sync();
  if (warp == kMmaWarp) tc05::dealloc(tmem, kTmemCols);
}

// Per device: the opt-in shared memory per block and the SM count, read once; per kernel
// configuration and device: the largest dynamic shared memory already granted, so that a
// launch calls cudaFuncSetAttribute only when it needs more (the launch path stays cheap
// on the host, which enqueues a step in tens of microseconds).
constexpr int kMaxDevices = 64;

struct DeviceLimits {
  std::atomic<int> optin{0}, sms{0};
};

bool device_limits(int* dev, int* optin, int* sms) {
  static DeviceLimits lim[kMaxDevices];
  if (cudaGetDevice(dev) != cudaSuccess || *dev < 0 || *dev >= kMaxDevices) return false;
  DeviceLimits& l = lim[*dev];
  int o = l.optin.load(std::memory_order_relaxed), n = l.sms.load(std::memory_order_relaxed);
  if (o == 0 || n == 0) {
    if (cudaDeviceGetAttribute(&o, cudaDevAttrMaxSharedMemoryPerBlockOptin, *dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, *dev) != cudaSuccess)
      return false;
    l.optin.store(o, std::memory_order_relaxed);
    l.sms.store(n, std::memory_order_relaxed);
  }
  *optin = o;
  *sms = n;
  return true;
}

// Ring stages that fit the shared memory next to the Q buffers and the unit-row table.
template <class C>
int group_stages(int R, int optin) {
  for (int nst = kMaxStages; nst >= 2; --nst)
    if (group_smem_bytes<C>(nst, R) + kStaticSmemBound <= static_cast<size_t>(optin)) return nst;
  return 0;
}

// Grant the kernel `smem` bytes of dynamic shared memory on device dev (once per size).
template <class C>
bool grant_smem(int dev, size_t smem) {
  static std::atomic<int> granted[kMaxDevices];
  if (static_cast<int>(smem) <= granted[dev].load(std::memory_order_relaxed)) return true;
  if (cudaFuncSetAttribute(decode_group_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return false;
  int cur = granted[dev].load(std::memory_order_relaxed);
  while (cur < static_cast<int>(smem) &&
         !granted[dev].compare_exchange_weak(cur, static_cast<int>(smem))) {
  }
  return true;
}

template <class C>
int group_grid_for(int R) {
  int dev = 0, optin = 0, sms = 0;
  if (!device_limits(&dev, &optin, &sms)) return 0;
  const int nst = group_stages<C>(R, optin);
  if (nst == 0 || !grant_smem<C>(dev, group_smem_bytes<C>(nst, R))) return 0;
  return sms;  // one CTA per SM: each holds all of its SM's tensor memory
}

template <class C>
cudaError_t launch_group_cfg(PrefixParams pp, int grid, cudaStream_t stream) {
  CUtensorMap tmk, tmv, tmq;
  const DecodeParams& p = pp.d;
  if (!make_pool_map(&tmk, p.k_pool, p.num_blocks, C::BS, p.Hkv, C::D, C::BS) ||
      !make_pool_map(&tmv, p.v_pool, p.num_blocks, C::BS, p.Hkv, C::D, C::BS) ||
      !make_q_map(&tmq, p.q, p.B, p.Hq, C::D, p.G))
    return cudaErrorInvalidValue;
  const int R = pp.ngroups + p.B;
  int dev = 0, optin = 0, sms = 0;
  if (!device_limits(&dev, &optin, &sms)) return cudaErrorInvalidValue;
  const int nst = group_stages<C>(R, optin);
  if (nst == 0) return cudaErrorInvalidValue;
  const size_t smem = group_smem_bytes<C>(nst, R);
  if (!grant_smem<C>(dev, smem)) return cudaErrorInvalidValue;
  // a programmatic dependent of the previous kernel on the stream
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
  return cudaLaunchKernelEx(&cfg, decode_group_kernel<C>, tmk, tmv, tmq, pp, nst);
}

}  // namespace

int prefix_grid(int D, int block_size, int R) {
  switch (D * 100 + block_size) {
    case 6408: return group_grid_for<GroupCfg<64, 8>>(R);
    case 6416: return group_grid_for<GroupCfg<64, 16>>(R);
    case 6432: return group_grid_for<GroupCfg<64, 32>>(R);
    case 12808: return group_grid_for<GroupCfg<128, 8>>(R);
    case 12816: return group_grid_for<GroupCfg<128, 16>>(R);
    case 12832: return group_grid_for<GroupCfg<128, 32>>(R);
    default: return 0;
  }
}

int prefix_warps_per_cta() { return 1; }  // one partial-slot owner per CTA

size_t prefix_workspace_bytes(int streams, int rows, int D) {
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  (void)rows;
  return up(static_cast<size_t>(streams) * 8) + up(static_cast<size_t>(streams) * kRows * 8) +
         up(static_cast<size_t>(streams) * kRows * D * 4) +
         static_cast<size_t>(streams) * 2 * 2 * kRows * 8;
}

void prefix_carve(PrefixParams* pp, void* workspace, int rows) {
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  char* w = static_cast<char*>(workspace);
  pp->cut_flag = reinterpret_cast<unsigned long long*>(w);
  w += up(static_cast<size_t>(pp->streams) * 8);
  pp->pml = reinterpret_cast<float*>(w);
  w += up(static_cast<size_t>(pp->streams) * kRows * 8);
  pp->pacc = reinterpret_cast<float*>(w);
  w += up(static_cast<size_t>(pp->streams) * kRows * pp->d.D * 4);
  pp->pxch = reinterpret_cast<float*>(w);
  (void)rows;
}

uint64_t prefix_epoch() {
  // a 64-bit tag per call for the cut-unit flags: a flag left by another call, or never
  // written, holds another value (the owner clears the flags it consumed, for replays of
  // a captured launch, which keep their tag)
  static std::atomic<uint64_t> next{[] {
    std::random_device rd;
    return (static_cast<uint64_t>(rd()) << 32) ^ rd();
  }()};
  return next.fetch_add(1, std::memory_order_relaxed);
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
