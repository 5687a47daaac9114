// Internal host/device interface of libpagedattn: kernel parameter blocks and the
// launchers the C ABI (api.cu) dispatches to.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "pa.h"

namespace pa {

// Parameters of one pa_decode call, as the kernels see them.
struct DecodeParams {
  void* out;                   // [B][Hq][D], dtype of q
  const void* q;               // [B][Hq][D]
  const void* k_pool;          // [NB][BS][Hkv][D]
  const void* v_pool;
  const int32_t* block_tables; // [B][max_blocks]
  const int32_t* seq_lens;     // [B]
  int B, Hq, Hkv, G, D, block_size, max_blocks, num_blocks;
  float scale_log2;            // scale * log2(e): softmax runs in base 2
  int partition_tokens;        // P: tokens per context partition
  int max_parts;               // ceil(max_blocks*block_size / P); 1 = no split
  float* ws_ml;                // [B][Hq][max_parts][2]: (running max, sum), base-2
  float* ws_acc;               // [B][Hq][max_parts][D]: unnormalised output
  int32_t* err;                // nullable device error flag
};

// Launch the bf16 tensor-core decode kernel (+ reduce when max_parts > 1).
cudaError_t launch_decode_tc(const DecodeParams& p, cudaStream_t stream);
// Launch the CUDA-core decode kernel (+ reduce when max_parts > 1).
cudaError_t launch_decode_generic(const DecodeParams& p, pa_dtype dtype, cudaStream_t stream);
// Launch the split-context reduce kernel.
cudaError_t launch_decode_reduce(const DecodeParams& p, pa_dtype dtype, cudaStream_t stream);

cudaError_t launch_reshape_and_cache(const void* key, const void* value, void* k_pool,
                                     void* v_pool, const int64_t* slot_mapping, int T, int Hkv,
                                     int row_bytes, int64_t num_slots, int32_t* err,
                                     cudaStream_t stream);
cudaError_t launch_copy_blocks(void* k_pool, void* v_pool, const int32_t* pairs, int n,
                               int64_t block_bytes, int num_blocks, int32_t* err,
                               cudaStream_t stream);

// Tensor-core path eligibility (shape/dtype only; alignment is checked by the caller).
bool tc_eligible(int G, int D, int block_size, pa_dtype dtype);

}  // namespace pa
