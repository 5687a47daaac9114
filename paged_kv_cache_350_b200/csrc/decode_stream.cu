// Paged decode attention, bf16 tensor-core path with a balanced persistent schedule
// (sm_100a).  Same result as decode_tc.cu — softmax(scale * q.K^T) V per (sequence,
// query head), K/V read through the block table ("PagedAttention" concept card,
// 实现要点) — scheduled for a whole batch of ragged lengths.
//
// Schedule ("streams"):
//   * Every (sequence b, KV head) is a unit of nt(b) = ceil(L_b / TILE_T) tiles of
//     TILE_T = 16 tokens (one block of 16, two of 8, or half of a block of 32); units
//     are laid end to end in (b, KV head) order, T = Hkv * sum_b nt(b) tiles in all.
//   * The grid is one wave of persistent CTAs (SM count x occupancy: 2 CTAs of 4 warps
//     per SM).  Every warp is one stream: stream s owns the global tiles
//     [s*per, (s+1)*per), per = ceil(T / streams).  Work is balanced to one tile.
//   * Each CTA first computes the prefix sums of nt(b) in shared memory; a global tile
//     index maps to (b, KV head, tile) by binary search.
//   * Each warp feeds itself: it resolves the block ids of its next 32 tiles with one
//     table read per lane (the following 32 are read one batch ahead), keeps SPW 4-D
//     TMA loads in flight in its own ring of stages (mbarrier expect-tx), and refills a
//     stage as soon as it has consumed it, across unit boundaries, so its HBM stream
//     never drains between units and no warp waits for another.
//   * The warp runs the tile math of tc_tile.cuh over its range.  A unit that
//     lies wholly inside the range is finished in place: normalised bf16 output.  A unit
//     cut by a range boundary leaves a partial (max, sum, unnormalised O) in one of the
//     stream's two slots; the reduce kernel merges the pieces of each cut unit by
//     log-sum-exp.  The stream in which a cut unit starts records it, with its piece
//     count, every launch.
//   * pa_decode_append fuses the step's cache write: the stream that consumes a unit's
//     last tile writes the new token's K/V to its slot and into the staged tile.

#include <cudaTypedefs.h>

#include "pa_device.cuh"
#include "pa_internal.h"
#include "tc_tile.cuh"

namespace pa {

namespace {

// Build-time tunable: ring stages per stream.
#ifndef PA_STREAM_SPW
#define PA_STREAM_SPW 2
#endif
// Launch the reduce as a programmatic dependent of the main kernel (its launch overlaps
// the main kernel's tail; it waits for the main grid's completion before reading).
#ifndef PA_STREAM_PDL
#define PA_STREAM_PDL 1
#endif

constexpr unsigned kFull = 0xffffffffu;

// Stage and CTA shape: 16-token stages (8 KB with D = 128; a 32-token block is staged
// in two halves), 4 warps per CTA and 2 CTAs per SM, so every SM runs 8 streams, two on
// each of its four sub-partitions (the tile math's issue and tensor rate per
// sub-partition is part of the pace: 6 streams per SM left two sub-partitions with
// double load).  PA_STREAM_TILE / PA_STREAM_NCW / PA_STREAM_MIN_CTAS override them
// (sweeps).
template <int BS>
struct StreamShape {
#ifdef PA_STREAM_TILE
  static constexpr int TILE = PA_STREAM_TILE;
#else
  static constexpr int TILE = 16;
#endif
#ifdef PA_STREAM_NCW
  static constexpr int NCW = PA_STREAM_NCW;
#else
  static constexpr int NCW = 4;
#endif
#ifdef PA_STREAM_MIN_CTAS
  static constexpr int MIN_CTAS = PA_STREAM_MIN_CTAS;
#else
  static constexpr int MIN_CTAS = 2;
#endif
};

template <int D_, int BS_, bool ROWS16_, int SPW_>
struct StreamCfg : TileCfg<D_, BS_, ROWS16_, StreamShape<BS_>::TILE, true> {
  static constexpr int NCW = StreamShape<BS_>::NCW;  // warps (= streams) per CTA
  static constexpr int THREADS = NCW * 32;
  static constexpr int MIN_CTAS = StreamShape<BS_>::MIN_CTAS;  // register bound
  static constexpr int SPW = SPW_;                 // ring stages per stream
  static constexpr int NST = NCW * SPW;
  static constexpr int RING_BYTES = NST * StreamCfg::STAGE_BYTES;
  static constexpr int Q_BYTES = WarpAcc<StreamCfg, true>::Q_BYTES;  // per consumer warp
  // Q tiles per warp: two, so that the next unit's Q is copied in while the current unit
  // streams; one for 16 query rows with 32-token stages (a sweep shape), where a second
  // would cost a CTA per SM (the next unit's Q is then only prefetched into L2).
  static constexpr int QBUF = (StreamCfg::ROWS16 && StreamCfg::TILE_T == 32) ? 1 : 2;
  static constexpr int FIXED_BYTES = RING_BYTES + NCW * QBUF * Q_BYTES;
};

template <class C>
size_t stream_smem_bytes(int B) {
  return C::FIXED_BYTES + 1024 + static_cast<size_t>(B + 1) * 4;
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

// First index in P[0..n) with P[idx] > v.
__device__ __forceinline__ int upper_bound(const int* P, int n, int v) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (P[mid] > v) hi = mid; else lo = mid + 1;
  }
  return lo;
}

struct TilePos {
  int b, kvh, j, nt;
};

// Global tile index -> (sequence, KV head, tile within the unit).  The host keeps the
// total tile count below 2^31.
__device__ __forceinline__ TilePos locate(const int* P, int B, int Hkv, int g) {
  TilePos t;
  const int v = g / Hkv;
  t.b = upper_bound(P, B + 1, v) - 1;
  t.nt = P[t.b + 1] - P[t.b];
  const int off = g - Hkv * P[t.b];
  t.kvh = off / t.nt;
  t.j = off - t.kvh * t.nt;
  return t;
}

// Block ids, KV head, block count and first row inside the (first) block of one tile,
// resolved by one lane.
struct TileIds {
  int kvh, nb, row0;
  int id[4];
};

template <class C>
__device__ __forceinline__ TileIds resolve_tile(const DecodeParams& p, const int* P, int g,
                                                int end) {
  TileIds r{0, 0, 0, {0, 0, 0, 0}};
  if (g >= end) return r;
  const TilePos t = locate(P, p.B, p.Hkv, g);
  r.kvh = t.kvh;
  const int L = clamp_len(p, t.b, false);
  const int nblk = (L + C::BS - 1) / C::BS;
  const int tok0 = t.j * C::TILE_T;
  const int blk = tok0 / C::BS;
  r.row0 = tok0 % C::BS;  // non-zero only when a stage holds part of a block
  r.nb = min(C::BPS, nblk - blk);
  const int32_t* tab = p.block_tables + static_cast<size_t>(t.b) * p.max_blocks + blk;
#pragma unroll
  for (int k = 0; k < C::BPS; ++k)
    if (k < r.nb) r.id[k] = __ldg(tab + k);
  return r;
}

// Fused cache write of pa_decode_append: put the step's token (K and V, one 16-byte chunk
// per lane in `v`: lanes [0, D/8) K, [D/8, D/4) V) into row r of the staged tile, and into
// its slot (block `phys`, offset `off`, KV head `kvh`) of the pools.  The tile was loaded
// from the pool before the write, so the staged row is replaced here; the proxy fence
// orders these shared writes before the next TMA write to the stage.
template <class C>
__device__ __forceinline__ void put_token(uint8_t* stage_ptr, int r, const uint4& v, int phys,
                                          int off, int kvh, const StreamParams& sp, int lane) {
  constexpr int VPR = C::D / 8;  // 16-byte chunks per head row
  if (lane < 2 * VPR) {
    const int which = lane / VPR, ch = lane % VPR;
    *reinterpret_cast<uint4*>(stage_ptr + which * C::TILE_BYTES + (ch >> 3) * C::CHUNK_BYTES +
                              sw128(r, ch & 7)) = v;
    fence_proxy_async_smem();
    if (phys >= 0 && phys < sp.d.num_blocks) {  // a bad id was flagged when the tile was loaded
      uint4* pool = static_cast<uint4*>(which ? sp.v_pool_w : sp.k_pool_w);
      pool[((static_cast<size_t>(phys) * C::BS + off) * sp.d.Hkv + kvh) * VPR + ch] = v;
    }
  }
  __syncwarp();
}

template <class C>
__global__ void __launch_bounds__(C::THREADS, C::MIN_CTAS)
    decode_stream_kernel(const __grid_constant__ CUtensorMap tmk,
                         const __grid_constant__ CUtensorMap tmv, const StreamParams sp) {
  constexpr int D = C::D, BS = C::BS, TILE_T = C::TILE_T, SPW = C::SPW, NST = C::NST;
  constexpr int kNCW = C::NCW, kThreads = C::THREADS;
  const DecodeParams& p = sp.d;
  const int B = p.B, Hkv = p.Hkv, G = p.G;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* qtiles = smem + C::RING_BYTES;                  // [kNCW][QBUF][Q_BYTES]
  int* P = reinterpret_cast<int*>(smem + C::FIXED_BYTES);  // [B + 1] tiles before sequence b
  __shared__ __align__(8) uint64_t full_bar[NST];
  __shared__ int warp_sum[kThreads / 32];

  // Set-up that reads no global data, then wait for the kernel before this one on the
  // stream (launched as its programmatic dependent, this CTA may start while it drains;
  // everything it wrote is visible after the wait, and this kernel reads or writes global
  // memory only after it).
  if (threadIdx.x == 0) {
    prefetch_tensormap(&tmk);
    prefetch_tensormap(&tmv);
    for (int st = 0; st < NST; ++st) mbar_init(smem_addr(&full_bar[st]), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    fence_proxy_async_smem();
  }
#if PA_STREAM_PDL
  asm volatile("griddepcontrol.wait;" ::: "memory");
#endif
  // ---- prefix sums of per-sequence tile counts (every CTA, identical) --------------
  {
    // tile counts first, read with independent coalesced loads, then scanned in place
#pragma unroll 4
    for (int b = threadIdx.x; b < B; b += kThreads)
      P[b] = (clamp_len(p, b, blockIdx.x == 0) + TILE_T - 1) / TILE_T;
    __syncthreads();
    const int chunk = (B + kThreads - 1) / kThreads;
    const int lo = min(B, static_cast<int>(threadIdx.x) * chunk);
    const int hi = min(B, lo + chunk);
    int sum = 0;
    for (int b = lo; b < hi; ++b) sum += P[b];
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
    for (int b = lo; b < hi; ++b) {
      const int n = P[b];
      P[b] = run;
      run += n;
    }
    if (threadIdx.x == 0) {
      int total = 0;
      for (int w = 0; w < kThreads / 32; ++w) total += warp_sum[w];
      P[B] = total;
    }
  }
  // Empty sequences have no tiles: their output rows are zero (written by one CTA each).
  __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out);
  for (int b = blockIdx.x; b < B; b += gridDim.x) {
    if (clamp_len(p, b, false) == 0) {
      uint32_t* row = reinterpret_cast<uint32_t*>(out + static_cast<size_t>(b) * p.Hq * D);
      for (int i = threadIdx.x; i < p.Hq * D / 2; i += kThreads) row[i] = 0u;
    }
  }
  __syncthreads();

  const int T = Hkv * P[B];
  const int S = static_cast<int>(gridDim.x) * kNCW;
  const int per = (T + S - 1) / S;
#if PA_STREAM_PDL
  // Let the reduce grid be launched now; it waits for this grid to complete.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
#endif

  // ---------------- every warp is one stream and feeds itself ----------------
  const int s = static_cast<int>(blockIdx.x) * kNCW + warp;
  const int beg = min(T, s * per);
  const int end = min(T, beg + per);
  const int cnt = end - beg;
  const uint64_t policy = l2_policy_evict_first();

  // Block ids of this stream's tiles, 32 at a time (lane j holds tile 32*batch + j);
  // the next batch's table reads are issued one batch ahead.
  TileIds cur = resolve_tile<C>(p, P, beg + lane, end);
  TileIds nxt = resolve_tile<C>(p, P, beg + 32 + lane, end);
  int batch = 0;
  // Issue the TMA loads of this stream's tile k into its stage (warp-collective).
  auto issue = [&](int k) {
    if ((k >> 5) != batch) {
      cur = nxt;
      ++batch;
      nxt = resolve_tile<C>(p, P, beg + 32 * (batch + 1) + lane, end);
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
      fence_proxy_async_smem();  // this stage's earlier generic reads/writes come first
      mbar_arrive_expect_tx(fb, static_cast<uint32_t>(n * C::BOXR * D * 2 * 2));
#pragma unroll
      for (int sub = 0; sub < C::BPS; ++sub) {
        if (sub >= n) break;
        int phys = ids[sub];
        if (phys < 0 || phys >= p.num_blocks) {
          flag_error(p.err, PA_DEVERR_BAD_BLOCK_ID);
          phys = 0;
        }
        if constexpr (C::BPS == 1) {
          // chunk c lands at c * CHUNK_BYTES (CHUNK_BYTES = BOXR rows of 128 bytes)
          static_assert(C::BOXR == C::TILE_T, "one box spans the stage's rows");
          tma_load_5d(kt, &tmk, 0, row0, 0, kv, phys, fb, policy);
          tma_load_5d(vt, &tmv, 0, row0, 0, kv, phys, fb, policy);
        } else {
#pragma unroll
          for (int c = 0; c < C::DCH; ++c) {
            tma_load_4d(kt + c * C::CHUNK_BYTES + sub * C::BOXR * 128, &tmk, c * 64, kv, row0,
                        phys, fb, policy);
            tma_load_4d(vt + c * C::CHUNK_BYTES + sub * C::BOXR * 128, &tmv, c * 64, kv, row0,
                        phys, fb, policy);
          }
        }
      }
    }
    __syncwarp();
  };
  for (int k = 0; k < SPW && k < cnt; ++k) issue(k);

  const int g = lane >> 2, tig = lane & 3;
  const float sl2 = p.scale_log2;
  const bool append = sp.k_new != nullptr;
  constexpr int VPR = D / 8;
  // The cut unit this stream owns (it starts in this stream's range and continues past
  // it): unit id, slot of this stream's piece, number of pieces.
  int own_u = -1, own_slot = 0, own_n = 0;
  int i = 0;  // tiles consumed by this stream (ring position)
  bool ok = true;
  WarpAcc<C, true> acc;
  uint8_t* my_q = qtiles + warp * C::QBUF * C::Q_BYTES;
  const __nv_bfloat16* qg = static_cast<const __nv_bfloat16*>(p.q);
  auto q_rows = [&](const TilePos& u) {  // the group's query rows of unit u
    return qg + (static_cast<size_t>(u.b) * p.Hq + static_cast<size_t>(u.kvh) * G) * D;
  };

  int gpos = beg;
  int qb = 0;  // Q tile of the current unit (QBUF == 2)
  TilePos t{};
  if (gpos < end) {
    t = locate(P, B, Hkv, gpos);
    if constexpr (C::QBUF == 2) acc.prefetch_q(q_rows(t), G, my_q, lane);
  }
  while (gpos < end && ok) {
    const int L = clamp_len(p, t.b, false);
    const int ubeg = Hkv * P[t.b] + t.kvh * t.nt;
    const int uend = ubeg + t.nt;
    const int pend = min(end, uend);
    const size_t head0 = static_cast<size_t>(t.b) * p.Hq + static_cast<size_t>(t.kvh) * G;
    // pa_decode_append: the step's token is position L-1, in the unit's last tile.  The
    // stream that owns that tile fetches the token's K/V now and writes them when the
    // tile has landed (not for a length that was clamped as out of range).
    bool put = false;
    uint4 put_kv = make_uint4(0u, 0u, 0u, 0u);
    int put_phys = -1;
    if (append && pend == uend && __ldg(p.seq_lens + t.b) == L) {
      put = true;
      if (lane < 2 * VPR)
        put_kv = __ldg(static_cast<const uint4*>(lane < VPR ? sp.k_new : sp.v_new) +
                       (static_cast<size_t>(t.b) * Hkv + t.kvh) * VPR + lane % VPR);
      put_phys = __ldg(p.block_tables + static_cast<size_t>(t.b) * p.max_blocks + (L - 1) / BS);
    }
    // The next unit of this stream (if any) starts at tile pend: its Q rows are copied
    // while this unit streams.
    TilePos tn{};
    if (pend < end) tn = locate(P, B, Hkv, pend);
    if constexpr (C::QBUF == 2) {
      acc.use_q(my_q + qb * C::Q_BYTES);
      if (pend < end) acc.prefetch_q(q_rows(tn), G, my_q + (qb ^ 1) * C::Q_BYTES, lane);
      qb ^= 1;
    } else {
      if (pend < end && lane < G * D * 2 / 128)
        prefetch_l2(reinterpret_cast<const uint8_t*>(q_rows(tn)) + lane * 128);
      acc.stage_q(qg + head0 * D, G, my_q, lane);
    }
    acc.reset();
    const int jend = t.j + (pend - gpos);
    for (int j = t.j; j < jend; ++j, ++i) {
      const int stage = warp * SPW + i % SPW;
      if (!mbar_wait_warp(smem_addr(&full_bar[stage]), (i / SPW) & 1, p.err)) {
        ok = false;  // the same in every lane: the warp leaves the loop together
        break;
      }
      uint8_t* st_ptr = smem + stage * C::STAGE_BYTES;
      const int valid = min(TILE_T, L - j * TILE_T);
      if (valid < TILE_T) zero_tail_rows<C>(st_ptr, valid, lane);
      if (put && j == t.nt - 1)
        put_token<C>(st_ptr, valid - 1, put_kv, put_phys, (L - 1) % BS, t.kvh, sp, lane);
      acc.tile(smem_addr(st_ptr), valid, sl2, lane);
      __syncwarp();
      if (i + SPW < cnt) issue(i + SPW);  // refill the stage just consumed
    }
    if (!ok) break;
    acc.reduce_l();
    const bool complete = (gpos == ubeg) && (pend == uend);
    if (complete) {
      const float inv_lo = 1.f / acc.l_lo;
      const float inv_hi = C::ROWS16 ? 1.f / acc.l_hi : 0.f;
#pragma unroll
      for (int jn = 0; jn < C::NT; ++jn) {
        if (g < G)
          *reinterpret_cast<uint32_t*>(out + (head0 + g) * D + 8 * jn + 2 * tig) =
              pack_bf16x2(acc.o_lo[jn][0] * inv_lo, acc.o_lo[jn][1] * inv_lo);
        if (C::ROWS16 && g + 8 < G)
          *reinterpret_cast<uint32_t*>(out + (head0 + g + 8) * D + 8 * jn + 2 * tig) =
              pack_bf16x2(acc.o_hi[jn][0] * inv_hi, acc.o_hi[jn][1] * inv_hi);
      }
    } else {
      const int slot = gpos == beg ? 0 : 1;  // a cut piece is the stream's first or last
      const size_t row0 = (static_cast<size_t>(s) * 2 + slot) * G;
      if (tig == 0) {
        if (g < G)
          *reinterpret_cast<float2*>(sp.pml + (row0 + g) * 2) = make_float2(acc.m_lo, acc.l_lo);
        if (C::ROWS16 && g + 8 < G)
          *reinterpret_cast<float2*>(sp.pml + (row0 + g + 8) * 2) = make_float2(acc.m_hi, acc.l_hi);
      }
#pragma unroll
      for (int jn = 0; jn < C::NT; ++jn) {
        if (g < G)
          *reinterpret_cast<float2*>(sp.pacc + (row0 + g) * D + 8 * jn + 2 * tig) =
              make_float2(acc.o_lo[jn][0], acc.o_lo[jn][1]);
        if (C::ROWS16 && g + 8 < G)
          *reinterpret_cast<float2*>(sp.pacc + (row0 + g + 8) * D + 8 * jn + 2 * tig) =
              make_float2(acc.o_hi[jn][0], acc.o_hi[jn][1]);
      }
      if (ubeg >= beg) {  // the unit starts here: its pieces are streams s .. (uend-1)/per
        own_u = t.b * Hkv + t.kvh;
        own_slot = slot;
        own_n = (uend - 1) / per - s + 1;
      }
    }
    gpos = pend;
    t = tn;
  }
  cp_async_wait_all();  // a Q copy still in flight after an early exit
  if (!ok) {
    // A load never arrived: wait (bounded) for this stream's loads still in flight so no
    // TMA write lands after the CTA has left, then report nothing for this stream.
    for (int k = i; k < cnt && k < i + SPW; ++k) {
      const int stage = warp * SPW + k % SPW;
      mbar_wait(smem_addr(&full_bar[stage]), (k / SPW) & 1, p.err);
    }
  }
  if (lane == 0) {
    int4 m = make_int4(ok ? own_u : -1, own_slot, own_n, 0);
    *reinterpret_cast<int4*>(sp.meta + s * 4) = m;
  }
}

// Merge the pieces of every unit cut by a stream boundary.  Block s merges the unit that
// starts in stream s and continues into the following streams, recorded by stream s with
// its piece count n: piece i is slot 0 of stream s + i, except the first, which is in
// the slot stream s recorded.
//
// Threads: PS groups of BT = G * D/4 threads (rounded up to whole warps); in a group, one
// thread per (query-head row, 4 output columns).  Group k merges pieces k, k + PS, ...
// online (running max, sum, output; base 2), with the piece loop unrolled so that the
// loads overlap; with PS > 1 the groups' results are then combined through shared
// memory.  PS > 1 only when units are fewer than streams: then every unit spans several
// streams (a long sequence's unit can have tens of pieces), while with many short units
// a bigger block would only slow the launch of the many blocks that find no unit.
template <int D>
__global__ void __launch_bounds__(1024) stream_reduce_kernel(const StreamParams sp, int BT,
                                                             int PS) {
#if PA_STREAM_PDL
  // Wait until the main kernel has completed and its writes are visible; the next kernel
  // on the stream may launch now (it waits for this grid before reading).
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
#endif
  const DecodeParams& p = sp.d;
  const int s = blockIdx.x;
  const int4 m = *reinterpret_cast<const int4*>(sp.meta + static_cast<size_t>(s) * 4);
  if (m.x < 0) return;
  const int u = m.x, slot0 = m.y, n = m.z;
  const int G = p.G;
  const int grp = threadIdx.x / BT, idx = threadIdx.x - grp * BT;
  const int r = idx / (D / 4);
  const int c = (idx % (D / 4)) * 4;
  const bool live = r < G;
  float M = -INFINITY, l = 0.f, a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
  if (live) {
#pragma unroll 4
    for (int i = grp; i < n; i += PS) {
      const size_t row = (static_cast<size_t>(s + i) * 2 + (i == 0 ? slot0 : 0)) * G + r;
      const float2 ml = *reinterpret_cast<const float2*>(sp.pml + row * 2);
      const float4 a = *reinterpret_cast<const float4*>(sp.pacc + row * D + c);
      const float Mn = fmaxf(M, ml.x);
      const float so = exp2f(M - Mn), sn = exp2f(ml.x - Mn);
      l = l * so + ml.y * sn;
      a0 = a0 * so + a.x * sn;
      a1 = a1 * so + a.y * sn;
      a2 = a2 * so + a.z * sn;
      a3 = a3 * so + a.w * sn;
      M = Mn;
    }
  }
  if (PS > 1) {
    extern __shared__ float red[];  // [PS][BT][6]
    float* mine = red + (static_cast<size_t>(grp) * BT + idx) * 6;
    mine[0] = M;
    mine[1] = l;
    mine[2] = a0;
    mine[3] = a1;
    mine[4] = a2;
    mine[5] = a3;
    __syncthreads();
    if (grp != 0) return;
    for (int k = 1; k < PS; ++k) {
      const float* o = red + (static_cast<size_t>(k) * BT + idx) * 6;
      const float Mn = fmaxf(M, o[0]);
      // a group with no piece (n < PS) holds max -inf and adds nothing
      const float so = M == -INFINITY ? 0.f : exp2f(M - Mn);
      const float sn = o[0] == -INFINITY ? 0.f : exp2f(o[0] - Mn);
      l = l * so + o[1] * sn;
      a0 = a0 * so + o[2] * sn;
      a1 = a1 * so + o[3] * sn;
      a2 = a2 * so + o[4] * sn;
      a3 = a3 * so + o[5] * sn;
      M = Mn;
    }
  }
  if (!live) return;
  const int b = u / p.Hkv, kvh = u - b * p.Hkv;
  __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out) +
                       (static_cast<size_t>(b) * p.Hq + static_cast<size_t>(kvh) * G + r) * D + c;
  const float inv = 1.f / l;
  *reinterpret_cast<uint2*>(out) = make_uint2(pack_bf16x2(a0 * inv, a1 * inv),
                                              pack_bf16x2(a2 * inv, a3 * inv));
}

// Reduce block shape: BT = G * D/4 threads rounded up to whole warps, and PS piece groups
// (4 when the units, B * Hkv, are fewer than the streams; at most 1024 threads).
struct ReduceShape {
  int BT, PS;
};

template <int D>
ReduceShape reduce_shape(const StreamParams& sp) {
  ReduceShape r;
  r.BT = ((sp.d.G * D / 4 + 31) / 32) * 32;
  const long long units = static_cast<long long>(sp.d.B) * sp.d.Hkv;
  r.PS = units < sp.streams ? (1024 / r.BT < 4 ? 1024 / r.BT : 4) : 1;
  if (r.PS < 1) r.PS = 1;
  return r;
}

template <class C>
int stream_grid_for(int B, int device_sms) {
  int occ = 0;
  const size_t smem = stream_smem_bytes<C>(B);
  if (cudaFuncSetAttribute(decode_stream_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, decode_stream_kernel<C>, C::THREADS,
                                                    smem) != cudaSuccess)
    return 0;
  return occ * device_sms;
}

template <class C>
cudaError_t launch_stream_cfg(const StreamParams& sp, int grid, cudaStream_t stream) {
  CUtensorMap tmk, tmv;
  const DecodeParams& p = sp.d;
  // a stage of one block (or of part of one): one box of all D columns per stage and pool
  // (the 5-D view lands in the stage's chunk-major layout); several blocks a stage: one
  // box per block and 64-column chunk
  const bool ok = C::BPS == 1
      ? make_pool_map_rows(&tmk, p.k_pool, p.num_blocks, C::BS, p.Hkv, C::D, C::BOXR) &&
        make_pool_map_rows(&tmv, p.v_pool, p.num_blocks, C::BS, p.Hkv, C::D, C::BOXR)
      : make_pool_map(&tmk, p.k_pool, p.num_blocks, C::BS, p.Hkv, C::D, C::BOXR) &&
        make_pool_map(&tmv, p.v_pool, p.num_blocks, C::BS, p.Hkv, C::D, C::BOXR);
  if (!ok) return cudaErrorInvalidValue;
  const size_t smem = stream_smem_bytes<C>(p.B);
  cudaError_t e = cudaFuncSetAttribute(decode_stream_kernel<C>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
#if PA_STREAM_PDL
  {
    // a programmatic dependent of the previous kernel on the stream (see the kernel's
    // griddepcontrol.wait)
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(C::THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, decode_stream_kernel<C>, tmk, tmv, sp);
  }
#else
  decode_stream_kernel<C><<<grid, C::THREADS, smem, stream>>>(tmk, tmv, sp);
  e = cudaGetLastError();
#endif
  if (e != cudaSuccess) return e;
  const ReduceShape rs = reduce_shape<C::D>(sp);
  const size_t red_smem = rs.PS > 1 ? static_cast<size_t>(rs.PS) * rs.BT * 6 * sizeof(float) : 0;
#if PA_STREAM_PDL
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(sp.streams));
  cfg.blockDim = dim3(static_cast<unsigned>(rs.BT * rs.PS));
  cfg.dynamicSmemBytes = red_smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, stream_reduce_kernel<C::D>, sp, rs.BT, rs.PS);
#else
  stream_reduce_kernel<C::D><<<sp.streams, rs.BT * rs.PS, red_smem, stream>>>(sp, rs.BT, rs.PS);
  return cudaGetLastError();
#endif
}

constexpr int kSPW = PA_STREAM_SPW;

template <int D, int BS>
int grid_d_bs(bool rows16, int B, int sms) {
  return rows16 ? stream_grid_for<StreamCfg<D, BS, true, kSPW>>(B, sms)
                : stream_grid_for<StreamCfg<D, BS, false, kSPW>>(B, sms);
}

template <int D, int BS>
cudaError_t launch_d_bs(const StreamParams& sp, int grid, cudaStream_t stream) {
  if (sp.d.G > 8) return launch_stream_cfg<StreamCfg<D, BS, true, kSPW>>(sp, grid, stream);
  return launch_stream_cfg<StreamCfg<D, BS, false, kSPW>>(sp, grid, stream);
}

}  // namespace

int stream_warps_per_cta(int block_size) {
  switch (block_size) {
    case 8: return StreamShape<8>::NCW;
    case 16: return StreamShape<16>::NCW;
    case 32: return StreamShape<32>::NCW;
    default: return 0;
  }
}

int stream_grid(int D, int block_size, int G, int B) {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 0;
  const bool r16 = G > 8;
  switch (D * 100 + block_size) {
    case 6408: return grid_d_bs<64, 8>(r16, B, sms);
    case 6416: return grid_d_bs<64, 16>(r16, B, sms);
    case 6432: return grid_d_bs<64, 32>(r16, B, sms);
    case 12808: return grid_d_bs<128, 8>(r16, B, sms);
    case 12816: return grid_d_bs<128, 16>(r16, B, sms);
    case 12832: return grid_d_bs<128, 32>(r16, B, sms);
    default: return 0;
  }
}

size_t stream_workspace_bytes(int streams, int G, int D) {
  const size_t meta = static_cast<size_t>(streams) * 4 * 4;
  const size_t pml = static_cast<size_t>(streams) * 2 * G * 2 * 4;
  const size_t pacc = static_cast<size_t>(streams) * 2 * G * D * 4;
  return ((meta + 255) / 256) * 256 + ((pml + 255) / 256) * 256 + pacc;
}

void stream_carve(StreamParams* sp, void* workspace) {
  char* ws = static_cast<char*>(workspace);
  const size_t meta = static_cast<size_t>(sp->streams) * 4 * 4;
  const size_t pml = static_cast<size_t>(sp->streams) * 2 * sp->d.G * 2 * 4;
  sp->meta = reinterpret_cast<int32_t*>(ws);
  sp->pml = reinterpret_cast<float*>(ws + ((meta + 255) / 256) * 256);
  sp->pacc = reinterpret_cast<float*>(ws + ((meta + 255) / 256) * 256 + ((pml + 255) / 256) * 256);
}

cudaError_t launch_decode_stream(const StreamParams& sp, int grid, cudaStream_t stream) {
  switch (sp.d.D * 100 + sp.d.block_size) {
    case 6408: return launch_d_bs<64, 8>(sp, grid, stream);
    case 6416: return launch_d_bs<64, 16>(sp, grid, stream);
    case 6432: return launch_d_bs<64, 32>(sp, grid, stream);
    case 12808: return launch_d_bs<128, 8>(sp, grid, stream);
    case 12816: return launch_d_bs<128, 16>(sp, grid, stream);
    case 12832: return launch_d_bs<128, 32>(sp, grid, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace pa
