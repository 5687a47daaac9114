// Paged decode attention, bf16 tensor-core path (sm_100a).
//
// What it computes: for each sequence b and query head h, softmax(scale * q.K^T) V over
// the sequence's tokens, with K/V read from the block pool through the block table
// ("PagedAttention" concept card, 实现要点: the kernel takes the block table and reads
// K/V scatter-gather; the extra lookup happens once per block and the access inside a
// block stays contiguous).  The math is plain attention ("什么是分页注意力", 边界与常见误解).
//
// Design (B200):
//   * One CTA per (sequence, KV head, context partition); the whole GQA group of
//     G = Hq/Hkv query heads rides along, so every K/V byte is read from HBM once.
//   * Warp 4 is the producer: it reads the partition's block ids (32 per coalesced warp
//     load), and lane 0 issues one 4-D TMA load per (block, K|V, 64-column chunk) into a
//     ring of NSTAGE shared-memory stages, completion tracked by an mbarrier with an
//     expected byte count.  The tensor map views a pool as [NB][BS][Hkv][D] and each box
//     is one block's BS rows x 64 columns of one KV head, written 128-byte swizzled.
//   * Warps 0-3 are consumers; warp w takes stages w, w+4, ...  Per 16-token sub-tile:
//     S = Q(16 x D, heads padded to 16 rows) . K^T with m16n8k16 bf16 MMAs (K fragments
//     by ldmatrix from the swizzled tile), an fp32 online softmax in base 2 (the scale
//     folded with log2 e), and P fed straight back from registers as the A operand of
//     O += P.V (V fragments by ldmatrix.trans).  P goes in as two bf16 MMAs, hi and lo
//     parts, so the only rounding that reaches the output is the final one to bf16.
//   * Tokens past the sequence end in the last block are masked out of the softmax and
//     their V rows zeroed in shared memory, so stale or poisoned slots never reach the
//     output.  Block ids outside [0, num_blocks) raise PA_DEVERR_BAD_BLOCK_ID and read
//     block 0 instead.
//   * The four warps' (max, sum, O) merge in shared memory.  A single-partition sequence
//     writes the normalised bf16 output; otherwise the partition writes its partial
//     (max, sum, unnormalised O) and the reduce kernel merges partitions.

#include <cudaTypedefs.h>

#include <mutex>

#include "pa_device.cuh"
#include "pa_internal.h"
#include "tc_tile.cuh"

namespace pa {

namespace {

constexpr unsigned kFull = 0xffffffffu;

template <int D_, int BS_, bool ROWS16_, int NSTAGE_>
struct TcCfg : TileCfg<D_, BS_, ROWS16_> {
  static constexpr int NSTAGE = NSTAGE_;
  static constexpr int NCW = 4;  // consumer warps
  static constexpr int THREADS = (NCW + 1) * 32;
  static constexpr int MERGE_BYTES = NCW * TcCfg::ROWS * TcCfg::D * 4;
  static constexpr int RING_BYTES = NSTAGE * TcCfg::STAGE_BYTES;
  static constexpr int BUF_BYTES = RING_BYTES > MERGE_BYTES ? RING_BYTES : MERGE_BYTES;
  static constexpr int SMEM_BYTES = BUF_BYTES + 1024;  // + alignment slack
};

template <class C>
__global__ void __launch_bounds__(C::THREADS)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tmk,
                     const __grid_constant__ CUtensorMap tmv, const DecodeParams p) {
  constexpr int D = C::D, BS = C::BS, TILE_T = C::TILE_T, NSTAGE = C::NSTAGE;
  constexpr int NCW = C::NCW, ROWS = C::ROWS;

  const int part = blockIdx.x % p.max_parts;
  const int unit = blockIdx.x / p.max_parts;
  const int b = unit / p.Hkv;
  const int kvh = unit - b * p.Hkv;
  const int G = p.G;
  const int P = p.partition_tokens;

  int L = __ldg(p.seq_lens + b);
  const int Lmax = p.max_blocks * BS;
  if (L < 0 || L > Lmax) {
    if (threadIdx.x == 0 && part == 0) flag_error(p.err, PA_DEVERR_BAD_SEQ_LEN);
    L = L < 0 ? 0 : Lmax;
  }
  const int nparts = L > 0 ? (L + P - 1) / P : 1;
  if (part >= nparts) return;

  __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out);
  const size_t head0 = static_cast<size_t>(b) * p.Hq + static_cast<size_t>(kvh) * G;
  if (L == 0) {  // empty sequence: the output rows are an empty sum
    for (int i = threadIdx.x; i < G * (D / 2); i += blockDim.x) {
      const int r = i / (D / 2), d = (i % (D / 2)) * 2;
      *reinterpret_cast<uint32_t*>(out + (head0 + r) * D + d) = 0u;
    }
    return;
  }

  const int tok0 = part * P;
  const int tok1 = min(L, tok0 + P);
  const int ntiles = (tok1 - tok0 + TILE_T - 1) / TILE_T;
  const int blk0 = tok0 / BS;
  const int nblk = (tok1 - tok0 + BS - 1) / BS;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  __shared__ __align__(8) uint64_t full_bar[NSTAGE];
  __shared__ __align__(8) uint64_t empty_bar[NSTAGE];
  __shared__ float sm_m[NCW][ROWS];
  __shared__ float sm_l[NCW][ROWS];

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(smem_addr(&full_bar[s]), 1);
      mbar_init(smem_addr(&empty_bar[s]), 1);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    fence_proxy_async_smem();
  }
  __syncthreads();

  if (warp == NCW) {
    // ---------------- producer warp ----------------
    if (lane == 0) {
      prefetch_tensormap(&tmk);
      prefetch_tensormap(&tmv);
    }
    const uint64_t policy = l2_policy_evict_first();
    const int32_t* tab = p.block_tables + static_cast<size_t>(b) * p.max_blocks + blk0;
    bool ok = true;
    for (int j0 = 0; j0 < nblk && ok; j0 += 32) {
      int id = 0;
      if (j0 + lane < nblk) {
        id = __ldg(tab + j0 + lane);
        if (id < 0 || id >= p.num_blocks) {
          flag_error(p.err, PA_DEVERR_BAD_BLOCK_ID);
          id = 0;
        }
      }
      const int n = min(32, nblk - j0);
      for (int jj = 0; jj < n; ++jj) {
        const int phys = __shfl_sync(kFull, id, jj);
        if (lane == 0 && ok) {
          const int j = j0 + jj;
          const int tile = j / C::BPS;
          const int sub = j - tile * C::BPS;
          const int stage = tile % NSTAGE;
          const uint32_t fb = smem_addr(&full_bar[stage]);
          if (sub == 0) {
            if (tile >= NSTAGE)
              ok = mbar_wait(smem_addr(&empty_bar[stage]), ((tile / NSTAGE) - 1) & 1, p.err);
            if (ok) {
              const int blocks_here = min(C::BPS, nblk - tile * C::BPS);
              mbar_arrive_expect_tx(fb, static_cast<uint32_t>(blocks_here * BS * D * 2 * 2));
            }
          }
          if (ok) {
            const uint32_t kt = smem_addr(smem + stage * C::STAGE_BYTES) + sub * BS * 128;
            const uint32_t vt = kt + C::TILE_BYTES;
            if constexpr (C::BPS == 1) {
              // a stage is one block: one box of all D columns per pool, chunk c landing
              // at c * CHUNK_BYTES (CHUNK_BYTES = BS rows of 128 bytes)
              static_assert(C::TILE_T == BS, "one block a stage");
              tma_load_5d(kt, &tmk, 0, 0, 0, kvh, phys, fb, policy);
              tma_load_5d(vt, &tmv, 0, 0, 0, kvh, phys, fb, policy);
            } else {
#pragma unroll
              for (int c = 0; c < C::DCH; ++c) {
                tma_load_4d(kt + c * C::CHUNK_BYTES, &tmk, c * 64, kvh, 0, phys, fb, policy);
                tma_load_4d(vt + c * C::CHUNK_BYTES, &tmv, c * 64, kvh, 0, phys, fb, policy);
              }
            }
          }
        }
      }
      ok = __shfl_sync(kFull, ok ? 1 : 0, 0) != 0;
    }
    return;
  }

  // ---------------- consumer warps ----------------
  const int g = lane >> 2;
  const int tig = lane & 3;
  WarpAcc<C> acc;
  acc.load_q(static_cast<const __nv_bfloat16*>(p.q) + head0 * D, G, lane);
  acc.reset();
  const float sl2 = p.scale_log2;

  for (int tile = warp; tile < ntiles; tile += NCW) {
    const int stage = tile % NSTAGE;
    // one verdict per warp: no lane goes on alone into the tile's ldmatrix / mma.sync
    if (!mbar_wait_warp(smem_addr(&full_bar[stage]), (tile / NSTAGE) & 1, p.err)) break;
    uint8_t* st_ptr = smem + stage * C::STAGE_BYTES;
    const int valid = min(TILE_T, tok1 - (tok0 + tile * TILE_T));
    if (valid < TILE_T) zero_tail_rows<C>(st_ptr, valid, lane);
    acc.tile(smem_addr(st_ptr), valid, sl2, lane);
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_addr(&empty_bar[stage]));
  }

  // ---- merge the consumer warps: (m, l, O) per warp -> shared memory -> combine
  acc.reduce_l();
  named_barrier_sync(1, NCW * 32);  // every consumer is done with the stage ring
  float* mo = reinterpret_cast<float*>(smem);  // [NCW][ROWS][D]
  if (tig == 0) {
    sm_m[warp][g] = acc.m_lo;
    sm_l[warp][g] = acc.l_lo;
    if constexpr (C::ROWS16) {
      sm_m[warp][g + 8] = acc.m_hi;
      sm_l[warp][g + 8] = acc.l_hi;
    }
  }
#pragma unroll
  for (int j = 0; j < C::NT; ++j) {
    *reinterpret_cast<float2*>(mo + (warp * ROWS + g) * D + 8 * j + 2 * tig) =
        make_float2(acc.o_lo[j][0], acc.o_lo[j][1]);
    if constexpr (C::ROWS16)
      *reinterpret_cast<float2*>(mo + (warp * ROWS + g + 8) * D + 8 * j + 2 * tig) =
          make_float2(acc.o_hi[j][0], acc.o_hi[j][1]);
  }
  named_barrier_sync(1, NCW * 32);

  const int nrow = min(G, ROWS);
  for (int i = threadIdx.x; i < nrow * (D / 2); i += NCW * 32) {
    const int r = i / (D / 2);
    const int d = (i - r * (D / 2)) * 2;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NCW; ++w) M = fmaxf(M, sm_m[w][r]);
    float lsum = 0.f, a0 = 0.f, a1 = 0.f;
#pragma unroll
    for (int w = 0; w < NCW; ++w) {
      const float sc = exp2f(sm_m[w][r] - M);
      lsum += sc * sm_l[w][r];
      const float2 v = *reinterpret_cast<const float2*>(mo + (w * ROWS + r) * D + d);
      a0 += sc * v.x;
      a1 += sc * v.y;
    }
    const size_t h = head0 + r;
    if (nparts == 1) {
      const float inv = 1.f / lsum;
      *reinterpret_cast<uint32_t*>(out + h * D + d) = pack_bf16x2(a0 * inv, a1 * inv);
    } else {
      const size_t slot = h * p.max_parts + part;
      *reinterpret_cast<float2*>(p.ws_acc + slot * D + d) = make_float2(a0, a1);
      if (d == 0) *reinterpret_cast<float2*>(p.ws_ml + slot * 2) = make_float2(M, lsum);
    }
  }
}

}  // namespace

// ---- tensor maps --------------------------------------------------------------

namespace {

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// View a pool [NB][BS][Hkv][D] (bf16) as a 4-D tensor; box = one block's BS rows x 64
// columns of one KV head, 128-byte swizzled in shared memory.
}  // namespace

bool make_pool_map(CUtensorMap* map, const void* pool, int NB, int BS, int Hkv, int D,
                   int box_rows) {
  auto encode = get_encode_fn();
  if (!encode) return false;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(Hkv),
                        static_cast<cuuint64_t>(BS), static_cast<cuuint64_t>(NB)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(D) * 2,
                           static_cast<cuuint64_t>(Hkv) * D * 2,
                           static_cast<cuuint64_t>(BS) * Hkv * D * 2};
  cuuint32_t box[4] = {64, 1, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(pool), dims,
                      strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                      CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// The same pool as a 5-D tensor (64 columns, rows, D / 64 column chunks, heads, blocks)
// whose box is box_rows rows of one head and all D columns, landing as
// [D / 64][box_rows][64] (128-byte swizzled): one box where the 4-D view needs D / 64.
bool make_pool_map_rows(CUtensorMap* map, const void* pool, int NB, int BS, int Hkv, int D,
                        int box_rows) {
  auto encode = get_encode_fn();
  if (!encode || D % 64 != 0) return false;
  cuuint64_t dims[5] = {64, static_cast<cuuint64_t>(BS), static_cast<cuuint64_t>(D / 64),
                        static_cast<cuuint64_t>(Hkv), static_cast<cuuint64_t>(NB)};
  cuuint64_t strides[4] = {static_cast<cuuint64_t>(Hkv) * D * 2, 128,
                           static_cast<cuuint64_t>(D) * 2,
                           static_cast<cuuint64_t>(BS) * Hkv * D * 2};
  cuuint32_t box[5] = {64, static_cast<cuuint32_t>(box_rows), static_cast<cuuint32_t>(D / 64),
                       1, 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(pool), dims,
                      strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                      CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_q_map(CUtensorMap* map, const void* q, int B, int Hq, int D, int G) {
  auto encode = get_encode_fn();
  if (!encode || G < 1 || G > 256) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(Hq),
                        static_cast<cuuint64_t>(B)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(Hq) * D * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(G), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), dims,
                      strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                      CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

namespace {

template <class C>
cudaError_t launch_cfg(const DecodeParams& p, cudaStream_t stream) {
  CUtensorMap tmk, tmv;
  // a stage of one block: the 5-D view (one box per pool); several: one box per chunk
  const bool maps = C::BPS == 1
      ? make_pool_map_rows(&tmk, p.k_pool, p.num_blocks, C::BS, p.Hkv, C::D, C::BS) &&
        make_pool_map_rows(&tmv, p.v_pool, p.num_blocks, C::BS, p.Hkv, C::D, C::BS)
      : make_pool_map(&tmk, p.k_pool, p.num_blocks, C::BS, p.Hkv, C::D, C::BS) &&
        make_pool_map(&tmv, p.v_pool, p.num_blocks, C::BS, p.Hkv, C::D, C::BS);
  if (!maps)
    return cudaErrorInvalidValue;
  auto kern = decode_tc_kernel<C>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const long long grid = static_cast<long long>(p.B) * p.Hkv * p.max_parts;
  if (grid <= 0) return cudaSuccess;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  kern<<<static_cast<unsigned>(grid), C::THREADS, C::SMEM_BYTES, stream>>>(tmk, tmv, p);
  return cudaGetLastError();
}

template <int D, int BS>
cudaError_t launch_d_bs(const DecodeParams& p, cudaStream_t stream) {
  constexpr int NSTAGE = 8;
  if (p.G <= 8) return launch_cfg<TcCfg<D, BS, false, NSTAGE>>(p, stream);
  return launch_cfg<TcCfg<D, BS, true, NSTAGE>>(p, stream);
}

}  // namespace

bool tc_eligible(int G, int D, int block_size, pa_dtype dtype) {
  return dtype == PA_BF16 && G >= 1 && G <= 16 && (D == 64 || D == 128) &&
         (block_size == 8 || block_size == 16 || block_size == 32);
}

cudaError_t launch_decode_tc(const DecodeParams& p, cudaStream_t stream) {
  cudaError_t e;
  switch (p.D * 100 + p.block_size) {
    case 6408: e = launch_d_bs<64, 8>(p, stream); break;
    case 6416: e = launch_d_bs<64, 16>(p, stream); break;
    case 6432: e = launch_d_bs<64, 32>(p, stream); break;
    case 12808: e = launch_d_bs<128, 8>(p, stream); break;
    case 12816: e = launch_d_bs<128, 16>(p, stream); break;
    case 12832: e = launch_d_bs<128, 32>(p, stream); break;
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess || p.max_parts <= 1) return e;
  return launch_decode_reduce(p, PA_BF16, stream);
}

}  // namespace pa
