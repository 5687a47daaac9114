// Internal host/device interface of libpagedattn: kernel parameter blocks and the
// launchers the C ABI (api.cu) dispatches to.
#pragma once

#include <cuda.h>
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

// Parameters of the balanced persistent ("stream") tensor-core kernel.
struct StreamParams {
  DecodeParams d;
  int streams;     // consumer warps in the grid = tile ranges
  int32_t* meta;   // [streams][4]: unit in slot 0, it starts in this stream, unit in slot 1
  float* pml;      // [streams][2][G][2]: (max, sum) of cut-unit pieces, base 2
  float* pacc;     // [streams][2][G][D]: unnormalised outputs of those pieces
  // Fused cache write (pa_decode_append); all null for a plain decode.
  const void* k_new;  // [B][Hkv][D] the step's keys: position seq_lens[b]-1 of row b
  const void* v_new;
  void* k_pool_w;     // the pools of `d`, written at that position
  void* v_pool_w;
};

// One wave of the stream kernel for this shape on the current device (0 if unknown).
int stream_grid(int D, int block_size, int G, int B);
// Streams (warps) per CTA of the stream kernel for this block size:
// streams = grid * stream_warps_per_cta(block_size).
int stream_warps_per_cta(int block_size);
size_t stream_workspace_bytes(int streams, int G, int D);
void stream_carve(StreamParams* sp, void* workspace);
cudaError_t launch_decode_stream(const StreamParams& sp, int grid, cudaStream_t stream);

// Parameters of the shared-prefix decode (decode_prefix.cu).
struct PrefixParams {
  DecodeParams d;
  const int32_t* group_of;       // [B] group of batch row b, or -1
  const int32_t* group_prefix;   // [ngroups] shared tokens (multiple of PA_SHARED_PREFIX_ALIGN)
  const int32_t* group_members;  // [ngroups][max_members] batch rows, -1 padded
  int ngroups, max_members;
  int streams;
  uint64_t epoch;  // this call's tag for the cut-unit flags
  unsigned long long* cut_flag;  // [streams]: = epoch once CTA s has published the partial
                                 // of its first piece (a later piece of a cut unit)
  float* pml;      // [streams][64][2]: (max, sum) of that piece per row, base 2
  float* pacc;     // [streams][64][D]: its unnormalised output per row
  float* pxch;     // [streams][2][2][64][2]: per piece parity and column group, the
                   // (max, sum) the two softmax column groups exchange
};
int prefix_grid(int D, int block_size, int R);
int prefix_warps_per_cta();
size_t prefix_workspace_bytes(int streams, int rows, int D);
void prefix_carve(PrefixParams* pp, void* workspace, int rows);
// A fresh tag for one shared-prefix call (its cut-unit flags).
uint64_t prefix_epoch();
cudaError_t launch_decode_prefix(const PrefixParams& pp, int grid, cudaStream_t stream);

// 4-D TMA view of a bf16 pool [NB][BS][Hkv][D]: box = box_rows rows (BS, or a part of a
// block starting at a row coordinate) x 64 columns of one head.
bool make_pool_map(CUtensorMap* map, const void* pool, int NB, int BS, int Hkv, int D,
                   int box_rows);
// 5-D TMA view of the same pool: box = box_rows rows of one head with all D columns,
// landing as [D / 64][box_rows][64], 128-byte swizzled.
bool make_pool_map_rows(CUtensorMap* map, const void* pool, int NB, int BS, int Hkv, int D,
                        int box_rows);
// Tensor map over q viewed as [B][Hq][D] (bf16): boxes of 64 columns x G heads of one
// batch row, 128-byte swizzled.
bool make_q_map(CUtensorMap* map, const void* q, int B, int Hq, int D, int G);

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
// Write k_new/v_new[b] ([B][Hkv][D]) at position seq_lens[b]-1 of row b's block table.
cudaError_t launch_append_kv(const void* k_new, const void* v_new, void* k_pool, void* v_pool,
                             const int32_t* block_tables, const int32_t* seq_lens, int B,
                             int max_blocks, int block_size, int num_blocks, int row_bytes,
                             int32_t* err, cudaStream_t stream);
cudaError_t launch_copy_blocks(void* k_pool, void* v_pool, const int32_t* pairs, int n,
                               int64_t block_bytes, int num_blocks, int32_t* err,
                               cudaStream_t stream);

// Tensor-core path eligibility (shape/dtype only; alignment is checked by the caller).
bool tc_eligible(int G, int D, int block_size, pa_dtype dtype);

}  // namespace pa
