// C ABI of libpagedattn: argument validation, path selection, workspace carving.
// Every check happens on the host before anything is queued; a failing call queues
// nothing.  See include/pa.h for the contract of each entry point.

#include <algorithm>
#include <cmath>
#include <cstdint>

#include "pa.h"
#include "pa_internal.h"

namespace {

// Smallest context partition the automatic policy ever picks; pa_decode_workspace_size
// with partition_tokens == 0 sizes the workspace for it, which bounds every automatic
// choice.
constexpr int kAutoMinPartition = 512;
// Largest batch the balanced stream kernel takes (its prefix sums live in shared memory).
constexpr int kStreamMaxB = 8192;
// Stream-kernel CTAs assumed when no device can be asked.
constexpr int kStreamGridBound = 1024;

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool block_size_ok(int bs) { return bs == 4 || bs == 8 || bs == 16 || bs == 32; }

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

int64_t round_up(int64_t a, int64_t b) { return ceil_div(a, b) * b; }

// Automatic partition size: 512 tokens, grown for very long contexts so that a
// sequence splits into at most ~64 partitions (bounding the reduce traffic).
int auto_partition(int64_t max_seq, int tile) {
  if (max_seq <= kAutoMinPartition) return static_cast<int>(round_up(max_seq > 0 ? max_seq : 1, tile));
  int64_t p = round_up(ceil_div(max_seq, 64), kAutoMinPartition);
  if (p < kAutoMinPartition) p = kAutoMinPartition;
  return static_cast<int>(round_up(p, tile));
}

size_t workspace_bytes_for(int64_t B, int64_t Hq, int64_t D, int64_t parts) {
  if (parts <= 1) return 0;
  const int64_t ml = round_up(B * Hq * parts * 2 * 4, 256);
  const int64_t acc = B * Hq * parts * D * 4;
  return static_cast<size_t>(ml + acc);
}

}  // namespace

extern "C" {

const char* pa_status_string(pa_status s) {
  switch (s) {
    case PA_OK: return "ok";
    case PA_ERR_INVALID_ARG: return "invalid argument";
    case PA_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case PA_ERR_OUT_OF_BLOCKS: return "no free block left in the pool";
    case PA_ERR_BAD_BLOCK_ID: return "block id outside [0, num_blocks)";
    case PA_ERR_CUDA: return "CUDA runtime error";
    case PA_ERR_NOT_FOUND: return "unknown sequence id";
    case PA_ERR_EXISTS: return "sequence id already exists";
    case PA_ERR_BAD_SEQ_LEN: return "sequence length outside [0, max_blocks*block_size]";
    case PA_ERR_BAD_SLOT: return "slot outside the pool";
    case PA_ERR_TIMEOUT: return "a bounded device wait expired";
    case PA_ERR_SCRATCH_LIMIT: return "shape needs more scratch than the static no-alloc buffer";
    case PA_ERR_HOST_MEMORY: return "out of host memory";
  }
  return "unknown status";
}

pa_status pa_status_from_device_flag(int32_t flag) {
  if (flag == 0) return PA_OK;
  if (flag & PA_DEVERR_BAD_BLOCK_ID) return PA_ERR_BAD_BLOCK_ID;
  if (flag & PA_DEVERR_BAD_SEQ_LEN) return PA_ERR_BAD_SEQ_LEN;
  if (flag & PA_DEVERR_BAD_SLOT) return PA_ERR_BAD_SLOT;
  if (flag & PA_DEVERR_TIMEOUT) return PA_ERR_TIMEOUT;
  return PA_ERR_INVALID_ARG;
}

const char* pa_version(void) { return "0.1.0"; }

size_t pa_decode_workspace_size(int B, int Hq, int Hkv, int D, int max_seq_len,
                                int block_size, int partition_tokens) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || D <= 0 || max_seq_len < 0 ||
      !block_size_ok(block_size) || partition_tokens < 0 ||
      (partition_tokens > 0 && partition_tokens % block_size != 0))
    return static_cast<size_t>(-1);
  const int64_t P = partition_tokens > 0 ? partition_tokens : kAutoMinPartition;
  size_t need = workspace_bytes_for(B, Hq, D, ceil_div(max_seq_len, P));
  const int G = Hq / Hkv;
  if (partition_tokens == 0 && B > 0 && B <= kStreamMaxB &&
      pa::tc_eligible(G, D, block_size, PA_BF16)) {
    int grid = pa::stream_grid(D, block_size, G, B);
    if (grid <= 0) grid = kStreamGridBound;  // no device to ask: an upper bound
    const size_t s = pa::stream_workspace_bytes(grid * pa::stream_warps_per_cta(block_size), G, D);
    if (s > need) need = s;
  }
  return need;
}

// Shape/dtype checks and the launch plan shared by pa_decode_plan and pa_decode_ex.
static pa_status plan_decode(int B, int Hq, int Hkv, int D, int block_size, int max_blocks,
                             int num_blocks, float scale, pa_dtype dtype, bool have_ws,
                             size_t workspace_bytes, const pa_decode_opts* opts,
                             pa_decode_plan_info* info) {
  const int partition = opts ? opts->partition_tokens : 0;
  const int path = opts ? opts->path : PA_PATH_AUTO;
  const int max_ctas = opts ? opts->max_ctas : 0;
  if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || max_blocks <= 0 || num_blocks <= 0 ||
      block_size <= 0 || !std::isfinite(scale) || partition < 0 || max_ctas < 0 ||
      (path != PA_PATH_AUTO && path != PA_PATH_GENERIC && path != PA_PATH_TENSOR) ||
      (dtype != PA_F32 && dtype != PA_BF16))
    return PA_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return PA_ERR_UNSUPPORTED;
  if (!block_size_ok(block_size)) return PA_ERR_UNSUPPORTED;
  if (partition > 0 && partition % block_size != 0) return PA_ERR_INVALID_ARG;
  const int64_t max_seq = static_cast<int64_t>(max_blocks) * block_size;
  if (max_seq > 0x7fffffffLL) return PA_ERR_INVALID_ARG;

  const int G = Hq / Hkv;
  const bool tc_ok = path != PA_PATH_GENERIC && pa::tc_eligible(G, D, block_size, dtype);
  const int tc_tile = block_size > 16 ? block_size : 16;
  if (path == PA_PATH_TENSOR && !tc_ok) return PA_ERR_UNSUPPORTED;
  if (path == PA_PATH_TENSOR && partition > 0 && partition % tc_tile != 0)
    return PA_ERR_INVALID_ARG;  // partition not a multiple of the 16-token tile
  info->kernel = PA_KERNEL_NONE;
  info->partition_tokens = 0;
  info->max_parts = 0;
  info->grid = 0;
  info->launches = 0;
  if (B == 0) return PA_OK;

  // Balanced persistent tensor-core kernel: the default for bf16 batches whose total
  // tile count (16-token tiles x KV heads) stays below 2^31.
  const int64_t tile_bound = static_cast<int64_t>(B) * Hkv * ceil_div(max_seq, 16);
  if (tc_ok && partition == 0 && B <= kStreamMaxB && tile_bound < (int64_t(1) << 31)) {
    int grid = pa::stream_grid(D, block_size, G, B);
    if (max_ctas > 0 && grid > max_ctas) grid = max_ctas;
    const size_t need = grid > 0 ? pa::stream_workspace_bytes(
                                       grid * pa::stream_warps_per_cta(block_size), G, D)
                                 : 0;
    if (grid > 0 && have_ws && workspace_bytes >= need) {
      info->kernel = PA_KERNEL_TC_STREAM;
      info->grid = grid;
      info->max_parts = 1;
      info->launches = 2;
      return PA_OK;
    }
  }

  const bool use_tc = tc_ok && (partition == 0 || partition % tc_tile == 0);
  const int tile = use_tc ? tc_tile : block_size;
  int P = partition > 0 ? partition : auto_partition(max_seq, tile);
  int64_t parts = ceil_div(max_seq, P);
  if (parts > 1) {
    const size_t need = workspace_bytes_for(B, Hq, D, parts);
    if (!have_ws || workspace_bytes < need) {
      if (partition > 0) return PA_ERR_INVALID_ARG;
      P = static_cast<int>(round_up(max_seq, tile));  // single pass, no workspace
      parts = 1;
    }
  }
  info->kernel = use_tc ? PA_KERNEL_TC_PARTITION : PA_KERNEL_GENERIC;
  info->partition_tokens = P;
  info->max_parts = static_cast<int>(parts);
  const int64_t units = static_cast<int64_t>(B) * Hkv * (use_tc ? 1 : (G + 3) / 4);
  info->grid = static_cast<int>(std::min<int64_t>(units * parts, 0x7fffffff));
  info->launches = parts > 1 ? 2 : 1;
  return PA_OK;
}

pa_status pa_decode_plan(int B, int Hq, int Hkv, int D, int block_size, int max_blocks,
                         pa_dtype dtype, size_t workspace_bytes, const pa_decode_opts* opts,
                         pa_decode_plan_info* info) {
  if (!info) return PA_ERR_INVALID_ARG;
  return plan_decode(B, Hq, Hkv, D, block_size, max_blocks, 1, 1.0f, dtype, true,
                     workspace_bytes, opts, info);
}

// pa_decode_ex and pa_decode_append: k_new/v_new null = plain decode.
static pa_status decode_call(void* out, const void* q, const void* k_new, const void* v_new,
                             const void* k_pool, const void* v_pool, const int32_t* block_tables,
                             const int32_t* seq_lens, int B, int Hq, int Hkv, int D,
                             int block_size, int max_blocks, int num_blocks, float scale,
                             pa_dtype dtype, void* workspace, size_t workspace_bytes,
                             int32_t* dev_err_flag, pa_stream_t stream,
                             const pa_decode_opts* opts) {
  pa_decode_plan_info plan;
  const bool have_ws = workspace != nullptr && aligned(workspace, 256);
  pa_status st = plan_decode(B, Hq, Hkv, D, block_size, max_blocks, num_blocks, scale, dtype,
                             have_ws, workspace_bytes, opts, &plan);
  if (st != PA_OK) return st;
  if (B == 0) return PA_OK;
  if (!out || !q || !k_pool || !v_pool || !block_tables || !seq_lens) return PA_ERR_INVALID_ARG;
  if (!aligned(out, 16) || !aligned(q, 16) || !aligned(k_pool, 16) || !aligned(v_pool, 16) ||
      !aligned(block_tables, 4) || !aligned(seq_lens, 4) ||
      (dev_err_flag && !aligned(dev_err_flag, 4)))
    return PA_ERR_INVALID_ARG;
  const bool append = k_new != nullptr;
  if (append && (!v_new || !aligned(k_new, 16) || !aligned(v_new, 16))) return PA_ERR_INVALID_ARG;

  pa::DecodeParams p{};
  p.out = out;
  p.q = q;
  p.k_pool = k_pool;
  p.v_pool = v_pool;
  p.block_tables = block_tables;
  p.seq_lens = seq_lens;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.D = D;
  p.block_size = block_size;
  p.max_blocks = max_blocks;
  p.num_blocks = num_blocks;
  p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  p.partition_tokens = plan.partition_tokens;
  p.max_parts = plan.max_parts;
  p.err = dev_err_flag;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (plan.kernel == PA_KERNEL_TC_STREAM) {
    pa::StreamParams sp{};
    sp.d = p;
    sp.streams = plan.grid * pa::stream_warps_per_cta(block_size);
    pa::stream_carve(&sp, workspace);
    if (append) {  // the decode kernel writes the step's token itself
      sp.k_new = k_new;
      sp.v_new = v_new;
      sp.k_pool_w = const_cast<void*>(k_pool);
      sp.v_pool_w = const_cast<void*>(v_pool);
    }
    e = pa::launch_decode_stream(sp, plan.grid, s);
  } else {
    if (append) {
      const int esize = dtype == PA_BF16 ? 2 : 4;
      e = pa::launch_append_kv(k_new, v_new, const_cast<void*>(k_pool), const_cast<void*>(v_pool),
                               block_tables, seq_lens, B, max_blocks, block_size, num_blocks,
                               Hkv * D * esize, dev_err_flag, s);
      if (e != cudaSuccess) return PA_ERR_CUDA;
    }
    const int parts = plan.max_parts;
    if (parts > 1) {
      char* ws = static_cast<char*>(workspace);
      p.ws_ml = reinterpret_cast<float*>(ws);
      p.ws_acc = reinterpret_cast<float*>(
          ws + round_up(static_cast<int64_t>(B) * Hq * parts * 2 * 4, 256));
    }
    e = plan.kernel == PA_KERNEL_TC_PARTITION ? pa::launch_decode_tc(p, s)
                                               : pa::launch_decode_generic(p, dtype, s);
  }
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

pa_status pa_decode_ex(void* out, const void* q, const void* k_pool, const void* v_pool,
                       const int32_t* block_tables, const int32_t* seq_lens, int B, int Hq,
                       int Hkv, int D, int block_size, int max_blocks, int num_blocks,
                       float scale, pa_dtype dtype, void* workspace, size_t workspace_bytes,
                       int32_t* dev_err_flag, pa_stream_t stream, const pa_decode_opts* opts) {
  return decode_call(out, q, nullptr, nullptr, k_pool, v_pool, block_tables, seq_lens, B, Hq,
                     Hkv, D, block_size, max_blocks, num_blocks, scale, dtype, workspace,
                     workspace_bytes, dev_err_flag, stream, opts);
}

pa_status pa_decode_append(void* out, const void* q, const void* k_new, const void* v_new,
                           void* k_pool, void* v_pool, const int32_t* block_tables,
                           const int32_t* seq_lens, int B, int Hq, int Hkv, int D,
                           int block_size, int max_blocks, int num_blocks, float scale,
                           pa_dtype dtype, void* workspace, size_t workspace_bytes,
                           int32_t* dev_err_flag, pa_stream_t stream,
                           const pa_decode_opts* opts) {
  if (B > 0 && (!k_new || !v_new)) return PA_ERR_INVALID_ARG;
  return decode_call(out, q, k_new, v_new, k_pool, v_pool, block_tables, seq_lens, B, Hq, Hkv,
                     D, block_size, max_blocks, num_blocks, scale, dtype, workspace,
                     workspace_bytes, dev_err_flag, stream, opts);
}

pa_status pa_decode(void* out, const void* q, const void* k_pool, const void* v_pool,
                    const int32_t* block_tables, const int32_t* seq_lens, int B, int Hq,
                    int Hkv, int D, int block_size, int max_blocks, int num_blocks,
                    float scale, pa_dtype dtype, void* workspace, size_t workspace_bytes,
                    int32_t* dev_err_flag, pa_stream_t stream) {
  return pa_decode_ex(out, q, k_pool, v_pool, block_tables, seq_lens, B, Hq, Hkv, D, block_size,
                      max_blocks, num_blocks, scale, dtype, workspace, workspace_bytes,
                      dev_err_flag, stream, nullptr);
}

size_t pa_decode_shared_prefix_workspace_size(int B, int Hq, int Hkv, int D, int block_size,
                                              int ngroups) {
  if (B < 0 || ngroups < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || (D != 64 && D != 128) ||
      !block_size_ok(block_size))
    return static_cast<size_t>(-1);
  int grid = pa::prefix_grid(D, block_size, B + ngroups);
  if (grid <= 0) grid = kStreamGridBound;  // no device to ask: an upper bound
  return pa::prefix_workspace_bytes(grid * pa::prefix_warps_per_cta(), B + ngroups, D);
}

pa_status pa_decode_shared_prefix(void* out, const void* q, const void* k_pool,
                                  const void* v_pool, const int32_t* block_tables,
                                  const int32_t* seq_lens, int B, int Hq, int Hkv, int D,
                                  int block_size, int max_blocks, int num_blocks, float scale,
                                  pa_dtype dtype, const int32_t* group_of,
                                  const int32_t* group_prefix, const int32_t* group_members,
                                  int ngroups, int max_members, void* workspace,
                                  size_t workspace_bytes, int32_t* dev_err_flag,
                                  pa_stream_t stream) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || max_blocks <= 0 || num_blocks <= 0 ||
      block_size <= 0 || !std::isfinite(scale) || ngroups < 0 || max_members < 1 ||
      (dtype != PA_F32 && dtype != PA_BF16))
    return PA_ERR_INVALID_ARG;
  const int G = Hq / Hkv;
  if (!pa::tc_eligible(G, D, block_size, dtype)) return PA_ERR_UNSUPPORTED;
  if (max_members > 32 || G * max_members > 64 || B + ngroups > kStreamMaxB)
    return PA_ERR_UNSUPPORTED;
  const int64_t max_seq = static_cast<int64_t>(max_blocks) * block_size;
  if (max_seq > 0x7fffffffLL) return PA_ERR_INVALID_ARG;
  if (static_cast<int64_t>(B + ngroups) * Hkv * ceil_div(max_seq, PA_SHARED_PREFIX_ALIGN) >=
      (int64_t(1) << 31))
    return PA_ERR_UNSUPPORTED;
  if (B == 0) return PA_OK;
  if (!out || !q || !k_pool || !v_pool || !block_tables || !seq_lens || !group_of ||
      (ngroups > 0 && (!group_prefix || !group_members)))
    return PA_ERR_INVALID_ARG;
  if (!aligned(out, 16) || !aligned(q, 16) || !aligned(k_pool, 16) || !aligned(v_pool, 16) ||
      !aligned(block_tables, 4) || !aligned(seq_lens, 4) || !aligned(group_of, 4) ||
      (ngroups > 0 && (!aligned(group_prefix, 4) || !aligned(group_members, 4))) ||
      (dev_err_flag && !aligned(dev_err_flag, 4)) || !workspace || !aligned(workspace, 256))
    return PA_ERR_INVALID_ARG;
  const int grid = pa::prefix_grid(D, block_size, B + ngroups);
  if (grid <= 0) return PA_ERR_CUDA;
  pa::PrefixParams pp{};
  pp.streams = grid * pa::prefix_warps_per_cta();
  const int rows = B + ngroups;
  if (workspace_bytes < pa::prefix_workspace_bytes(pp.streams, rows, D)) return PA_ERR_INVALID_ARG;
  pa::DecodeParams& p = pp.d;
  p.out = out;
  p.q = q;
  p.k_pool = k_pool;
  p.v_pool = v_pool;
  p.block_tables = block_tables;
  p.seq_lens = seq_lens;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = G;
  p.D = D;
  p.block_size = block_size;
  p.max_blocks = max_blocks;
  p.num_blocks = num_blocks;
  p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  p.max_parts = 1;
  p.err = dev_err_flag;
  pp.group_of = group_of;
  pp.group_prefix = group_prefix;
  pp.group_members = group_members;
  pp.ngroups = ngroups;
  pp.max_members = max_members;
  pa::prefix_carve(&pp, workspace, rows);
  pp.epoch = pa::prefix_epoch();
  const cudaError_t e = pa::launch_decode_prefix(pp, grid, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

pa_status pa_reshape_and_cache(const void* key, const void* value, void* k_pool, void* v_pool,
                               const int64_t* slot_mapping, int T, int Hkv, int D,
                               int block_size, int num_blocks, pa_dtype dtype,
                               int32_t* dev_err_flag, pa_stream_t stream) {
  if (T < 0 || Hkv <= 0 || num_blocks <= 0 || block_size <= 0 ||
      (dtype != PA_F32 && dtype != PA_BF16))
    return PA_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return PA_ERR_UNSUPPORTED;
  if (!block_size_ok(block_size)) return PA_ERR_UNSUPPORTED;
  if (T == 0) return PA_OK;
  if (!key || !value || !k_pool || !v_pool || !slot_mapping) return PA_ERR_INVALID_ARG;
  if (!aligned(key, 16) || !aligned(value, 16) || !aligned(k_pool, 16) || !aligned(v_pool, 16) ||
      !aligned(slot_mapping, 8) || (dev_err_flag && !aligned(dev_err_flag, 4)))
    return PA_ERR_INVALID_ARG;
  const int esize = dtype == PA_BF16 ? 2 : 4;
  const int64_t row_bytes = static_cast<int64_t>(Hkv) * D * esize;
  if (row_bytes > 0x7fffffffLL) return PA_ERR_INVALID_ARG;
  const int64_t num_slots = static_cast<int64_t>(num_blocks) * block_size;
  cudaError_t e = pa::launch_reshape_and_cache(
      key, value, k_pool, v_pool, slot_mapping, T, Hkv, static_cast<int>(row_bytes), num_slots,
      dev_err_flag, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

pa_status pa_copy_blocks(void* k_pool, void* v_pool, const int32_t* pairs, int n,
                         int block_size, int Hkv, int D, int num_blocks, pa_dtype dtype,
                         int32_t* dev_err_flag, pa_stream_t stream) {
  if (n < 0 || Hkv <= 0 || num_blocks <= 0 || block_size <= 0 ||
      (dtype != PA_F32 && dtype != PA_BF16))
    return PA_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return PA_ERR_UNSUPPORTED;
  if (!block_size_ok(block_size)) return PA_ERR_UNSUPPORTED;
  if (n == 0) return PA_OK;
  if (!k_pool || !v_pool || !pairs) return PA_ERR_INVALID_ARG;
  if (!aligned(k_pool, 16) || !aligned(v_pool, 16) || !aligned(pairs, 4) ||
      (dev_err_flag && !aligned(dev_err_flag, 4)))
    return PA_ERR_INVALID_ARG;
  const int esize = dtype == PA_BF16 ? 2 : 4;
  const int64_t block_bytes = static_cast<int64_t>(block_size) * Hkv * D * esize;
  cudaError_t e = pa::launch_copy_blocks(k_pool, v_pool, pairs, n, block_bytes, num_blocks,
                                         dev_err_flag, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

}  // extern "C"
