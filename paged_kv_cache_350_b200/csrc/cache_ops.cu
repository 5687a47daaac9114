// The kernels that keep the paged KV pool consistent (sm_100a).
//
// reshape_and_cache: every decode step computes a key and a value for each new token
// and caches them for later steps ("什么是 LLM 中的分页注意力", 快速回顾:KV 缓存).  In the
// paged layout token t goes to slot s = slot_mapping[t]: block s / block_size, offset
// s % block_size.  Because the pool is [NB][BS][Hkv][D], slot s is simply row s of the
// pool viewed as [NB*BS][Hkv][D], so the copy is one contiguous Hkv*D row per token.
//
// append_kv: the same write for a decode step whose slots are implied by the tables: row
// b's token is position seq_lens[b]-1 (pa_decode_append on the paths whose decode kernel
// does not write it itself).
//
// copy_blocks: copy on write of shared blocks before a forked sequence writes into one
// ("PagedAttention" concept card, 实现要点; "深入解析 PagedAttention", 多序列共享): whole
// physical blocks, K and V, src -> dst.
//
// Both move 16-byte vectors (rows are multiples of 16 bytes for D in {64, 128}), one per
// thread per iteration, with bounds checks on every id that raise a device error flag
// and skip instead of faulting.

#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {

namespace {

// grid.y = token; x covers the token's row (Hkv*D elements) in 16-byte vectors, K and V.
__global__ void reshape_and_cache_kernel(const uint4* __restrict__ key,
                                         const uint4* __restrict__ value,
                                         uint4* __restrict__ k_pool, uint4* __restrict__ v_pool,
                                         const int64_t* __restrict__ slot_mapping,
                                         int vec_per_row, int64_t num_slots, int32_t* err) {
  // a decode launched as this kernel's programmatic dependent may start its set-up now;
  // this kernel, launched as one of the previous kernel, waits for it before any access
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int t = blockIdx.y;
  const int64_t s = __ldg(slot_mapping + t);
  if (s < 0) return;
  if (s >= num_slots) {
    if (threadIdx.x == 0 && blockIdx.x == 0) flag_error(err, PA_DEVERR_BAD_SLOT);
    return;
  }
  const int64_t src = static_cast<int64_t>(t) * vec_per_row;
  const int64_t dst = s * vec_per_row;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < vec_per_row;
       i += gridDim.x * blockDim.x) {
    k_pool[dst + i] = __ldg(key + src + i);
    v_pool[dst + i] = __ldg(value + src + i);
  }
}

// One block per batch row: the step's token is position L-1 of the row (L = seq_lens[b]),
// so its slot is the table entry of block (L-1) / block_size at offset (L-1) % block_size
// ("什么是 LLM 中的分页注意力", 使用分页注意力: a new token fills the next free slot of the
// sequence's current block).  Rows with L = 0 have no token this step.
__global__ void append_kv_kernel(const uint4* __restrict__ k_new, const uint4* __restrict__ v_new,
                                 uint4* __restrict__ k_pool, uint4* __restrict__ v_pool,
                                 const int32_t* __restrict__ block_tables,
                                 const int32_t* __restrict__ seq_lens, int max_blocks,
                                 int block_size, int num_blocks, int vec_per_row, int32_t* err) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int b = blockIdx.x;
  const int L = __ldg(seq_lens + b);
  if (L == 0) return;
  if (L < 0 || static_cast<int64_t>(L) > static_cast<int64_t>(max_blocks) * block_size) {
    if (threadIdx.x == 0) flag_error(err, PA_DEVERR_BAD_SEQ_LEN);
    return;
  }
  const int phys = __ldg(block_tables + static_cast<int64_t>(b) * max_blocks + (L - 1) / block_size);
  if (phys < 0 || phys >= num_blocks) {
    if (threadIdx.x == 0) flag_error(err, PA_DEVERR_BAD_BLOCK_ID);
    return;
  }
  const int64_t src = static_cast<int64_t>(b) * vec_per_row;
  const int64_t dst = (static_cast<int64_t>(phys) * block_size + (L - 1) % block_size) * vec_per_row;
  for (int i = threadIdx.x; i < vec_per_row; i += blockDim.x) {
    k_pool[dst + i] = __ldg(k_new + src + i);
    v_pool[dst + i] = __ldg(v_new + src + i);
  }
}

// grid.y = pair; x strides over the block's 16-byte vectors, K and V.
__global__ void copy_blocks_kernel(uint4* __restrict__ k_pool, uint4* __restrict__ v_pool,
                                   const int32_t* __restrict__ pairs, int64_t vec_per_block,
                                   int num_blocks, int32_t* err) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int i = blockIdx.y;
  const int src = __ldg(pairs + 2 * i);
  const int dst = __ldg(pairs + 2 * i + 1);
  if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
    if (threadIdx.x == 0 && blockIdx.x == 0) flag_error(err, PA_DEVERR_BAD_BLOCK_ID);
    return;
  }
  const int64_t so = static_cast<int64_t>(src) * vec_per_block;
  const int64_t d_o = static_cast<int64_t>(dst) * vec_per_block;
  for (int64_t v = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
       v < vec_per_block; v += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    k_pool[d_o + v] = k_pool[so + v];
    v_pool[d_o + v] = v_pool[so + v];
  }
}

// Launch as a programmatic dependent of the previous kernel on the stream: the grid may
// be scheduled while that kernel drains, and waits for it (griddepcontrol.wait) before
// touching memory, so a step of cache kernels and a decode pays no launch gap between
// them.  Without a previous kernel this is an ordinary launch.
template <class... KArgs, class... Args>
cudaError_t launch_dependent(void (*kernel)(KArgs...), dim3 grid, int threads,
                             cudaStream_t stream, Args... args) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(static_cast<unsigned>(threads));
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

}  // namespace

cudaError_t launch_reshape_and_cache(const void* key, const void* value, void* k_pool,
                                     void* v_pool, const int64_t* slot_mapping, int T, int Hkv,
                                     int row_bytes, int64_t num_slots, int32_t* err,
                                     cudaStream_t stream) {
  (void)Hkv;
  if (T <= 0) return cudaSuccess;
  const int vec = row_bytes / 16;
  const int threads = vec < 256 ? ((vec + 31) / 32) * 32 : 256;
  const int gx = (vec + threads - 1) / threads;
  if (T > 65535) {
    // one launch per 65535 tokens (grid.y limit)
    for (int t0 = 0; t0 < T; t0 += 65535) {
      const int n = T - t0 < 65535 ? T - t0 : 65535;
      cudaError_t e = launch_dependent(
          reshape_and_cache_kernel, dim3(gx, n), threads, stream,
          static_cast<const uint4*>(key) + static_cast<int64_t>(t0) * vec,
          static_cast<const uint4*>(value) + static_cast<int64_t>(t0) * vec,
          static_cast<uint4*>(k_pool), static_cast<uint4*>(v_pool), slot_mapping + t0, vec,
          num_slots, err);
      if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
  }
  return launch_dependent(reshape_and_cache_kernel, dim3(gx, T), threads, stream,
                          static_cast<const uint4*>(key), static_cast<const uint4*>(value),
                          static_cast<uint4*>(k_pool), static_cast<uint4*>(v_pool), slot_mapping,
                          vec, num_slots, err);
}

cudaError_t launch_append_kv(const void* k_new, const void* v_new, void* k_pool, void* v_pool,
                             const int32_t* block_tables, const int32_t* seq_lens, int B,
                             int max_blocks, int block_size, int num_blocks, int row_bytes,
                             int32_t* err, cudaStream_t stream) {
  if (B <= 0) return cudaSuccess;
  const int vec = row_bytes / 16;
  const int threads = vec < 256 ? ((vec + 31) / 32) * 32 : 256;
  return launch_dependent(append_kv_kernel, dim3(static_cast<unsigned>(B)), threads, stream,
                          static_cast<const uint4*>(k_new), static_cast<const uint4*>(v_new),
                          static_cast<uint4*>(k_pool), static_cast<uint4*>(v_pool), block_tables,
                          seq_lens, max_blocks, block_size, num_blocks, vec, err);
}

cudaError_t launch_copy_blocks(void* k_pool, void* v_pool, const int32_t* pairs, int n,
                               int64_t block_bytes, int num_blocks, int32_t* err,
                               cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  const int64_t vec = block_bytes / 16;
  const int threads = 256;
  int64_t gx = (vec + threads - 1) / threads;
  if (gx > 64) gx = 64;
  for (int i0 = 0; i0 < n; i0 += 65535) {
    const int m = n - i0 < 65535 ? n - i0 : 65535;
    cudaError_t e = launch_dependent(copy_blocks_kernel, dim3(static_cast<unsigned>(gx), m),
                                     threads, stream, static_cast<uint4*>(k_pool),
                                     static_cast<uint4*>(v_pool), pairs + 2 * i0, vec, num_blocks,
                                     err);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace pa
