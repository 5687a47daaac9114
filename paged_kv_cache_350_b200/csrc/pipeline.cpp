// pa_pipeline_*: decode steps of a fixed batch queued back to back, one C call per step.
//
// A serving loop's step is host work (the allocator reserves each sequence's next slot and
// reports copy-on-write pairs; the tables and lengths are written out), a host->device copy
// of the step input, the kernels (pa_copy_blocks when a shared partial block is appended
// to, then pa_decode_append) and a device->host copy of the output.  Done one call at a
// time from an interpreter, the host work and the queueing cost more than the kernels of a
// batch of a few hundred sequences.  Here one call does the whole step's host work in C and
// queues it, so the host prepares step t+1 while the GPU decodes step t.
//
// With shared_prefix_members > 0 the step is the parallel-sampling one: the allocator also
// groups the sequences that share a prompt's blocks (pa_alloc_prefix_groups) and writes the
// slot mapping, and the kernels are pa_copy_blocks, pa_reshape_and_cache and
// pa_decode_shared_prefix, which reads each group's shared blocks once.
//
// Staging: `depth` slots, each a pinned host input buffer, a device input buffer, a device
// output and a pinned host output, all caller-owned.  The input copy runs on `copy_in`,
// the kernels on `compute`, the output copy on `copy_out`; events order every reuse of a
// slot (a host input is rewritten only after its copy has finished, a device input only
// after the kernels that read it, a device output only after its copy to the host).

#include <cuda_runtime.h>

#include <cstdint>
#include <new>
#include <vector>

#include "pa.h"

namespace {

constexpr size_t kAlign = 256;

size_t up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

}  // namespace

struct pa_pipeline {
  pa_allocator* alloc = nullptr;
  pa_pipeline_desc d{};
  // q, k_new, v_new, block_tables, seq_lens, pairs; with shared_prefix_members > 0 also
  // slot_mapping, group_of, group_prefix, group_members
  size_t off[10] = {};
  size_t in_bytes = 0, out_bytes = 0;
  std::vector<void*> h_in, d_in, h_out, d_out;
  std::vector<cudaEvent_t> h2d_done, kern_done, d2h_done;
  std::vector<char> used;
  std::vector<int64_t> slots;  // the allocator's slot mapping (the kernels derive it)
  int64_t next = 0;
};

namespace {

bool valid_desc(const pa_pipeline_desc* d) {
  return d && d->B > 0 && d->Hq > 0 && d->Hkv > 0 && d->Hq % d->Hkv == 0 && d->D > 0 &&
         d->block_size > 0 && d->max_blocks > 0 && d->num_blocks > 0 && d->depth >= 1 &&
         d->shared_prefix_members >= 0 && d->shared_prefix_members <= 32 &&
         d->depth <= 64 && (d->dtype == PA_F32 || d->dtype == PA_BF16) && d->k_pool &&
         d->v_pool && d->host_in && d->dev_in && d->host_out && d->dev_out;
}

// The shared-prefix step's shape and workspace, checked when the pipeline is made, so that
// no submit can fail in the decode after the cache write was queued.
bool prefix_desc_ok(const pa_pipeline_desc* d) {
  const int m = d->shared_prefix_members, G = d->Hq / d->Hkv;
  if (m == 0) return true;
  if (d->dtype != PA_BF16 || (d->D != 64 && d->D != 128) || G > 16 || m * G > 64 ||
      (d->block_size != 8 && d->block_size != 16 && d->block_size != 32) || !d->workspace ||
      reinterpret_cast<uintptr_t>(d->workspace) % 256 != 0)
    return false;
  // a group has two members or more, so a step has at most B / 2 of them; the decode
  // takes B + ngroups <= 8192 rows and fewer than 2^31 row chunks (32 tokens each)
  const int64_t rows = static_cast<int64_t>(d->B) + d->B / 2;
  const int64_t chunks_per_row =
      (static_cast<int64_t>(d->max_blocks) * d->block_size + PA_SHARED_PREFIX_ALIGN - 1) /
      PA_SHARED_PREFIX_ALIGN;
  if (rows > 8192 || rows * d->Hkv * chunks_per_row >= (int64_t(1) << 31)) return false;
  const size_t need = pa_decode_shared_prefix_workspace_size(d->B, d->Hq, d->Hkv, d->D,
                                                             d->block_size, d->B / 2);
  return need != static_cast<size_t>(-1) && d->workspace_bytes >= need;
}

void destroy_events(pa_pipeline* p) {
  for (auto* v : {&p->h2d_done, &p->kern_done, &p->d2h_done})
    for (cudaEvent_t e : *v)
      if (e) cudaEventDestroy(e);
}

}  // namespace

extern "C" {

size_t pa_pipeline_input_bytes_prefix(int B, int Hq, int Hkv, int D, int max_blocks,
                                      pa_dtype dtype, int shared_prefix_members,
                                      size_t* offsets) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || max_blocks <= 0 ||
      (dtype != PA_F32 && dtype != PA_BF16) || shared_prefix_members < 0 ||
      shared_prefix_members > 32)
    return 0;
  const size_t e = dtype == PA_BF16 ? 2 : 4;
  const size_t b = static_cast<size_t>(B);
  const bool sp = shared_prefix_members > 0;
  const size_t sizes[10] = {b * Hq * D * e, b * Hkv * D * e, b * Hkv * D * e,
                            b * max_blocks * 4, b * 4, b * 8,
                            sp ? b * 8 : 0, sp ? b * 4 : 0, sp ? b * 4 : 0,
                            b * static_cast<size_t>(shared_prefix_members) * 4};
  size_t off = 0;
  for (int i = 0; i < 10; ++i) {
    if (offsets) offsets[i] = off;
    off += up(sizes[i]);
  }
  return off;
}

size_t pa_pipeline_input_bytes(int B, int Hq, int Hkv, int D, int max_blocks, pa_dtype dtype,
                               size_t* offsets) {
  size_t all[10];
  const size_t n = pa_pipeline_input_bytes_prefix(B, Hq, Hkv, D, max_blocks, dtype, 0, all);
  if (n && offsets)
    for (int i = 0; i < 6; ++i) offsets[i] = all[i];
  return n;
}

pa_status pa_pipeline_create(pa_allocator* alloc, const pa_pipeline_desc* desc,
                             pa_pipeline** out) {
  if (!out) return PA_ERR_INVALID_ARG;
  *out = nullptr;
  if (!alloc || !valid_desc(desc) || !prefix_desc_ok(desc)) return PA_ERR_INVALID_ARG;
  const int depth = desc->depth;
  for (int k = 0; k < depth; ++k)
    if (!desc->host_in[k] || !desc->dev_in[k] || !desc->host_out[k] || !desc->dev_out[k] ||
        reinterpret_cast<uintptr_t>(desc->dev_in[k]) % kAlign != 0 ||
        reinterpret_cast<uintptr_t>(desc->dev_out[k]) % 16 != 0)
      return PA_ERR_INVALID_ARG;
  pa_pipeline* p = new (std::nothrow) pa_pipeline;
  if (!p) return PA_ERR_HOST_MEMORY;
  try {
    p->alloc = alloc;
    p->d = *desc;
    p->in_bytes = pa_pipeline_input_bytes_prefix(desc->B, desc->Hq, desc->Hkv, desc->D,
                                                 desc->max_blocks, desc->dtype,
                                                 desc->shared_prefix_members, p->off);
    p->out_bytes = static_cast<size_t>(desc->B) * desc->Hq * desc->D *
                   (desc->dtype == PA_BF16 ? 2 : 4);
    p->h_in.assign(desc->host_in, desc->host_in + depth);
    p->d_in.assign(desc->dev_in, desc->dev_in + depth);
    p->h_out.assign(desc->host_out, desc->host_out + depth);
    p->d_out.assign(desc->dev_out, desc->dev_out + depth);
    p->h2d_done.assign(depth, nullptr);
    p->kern_done.assign(depth, nullptr);
    p->d2h_done.assign(depth, nullptr);
    p->used.assign(depth, 0);
    p->slots.assign(desc->B, 0);
  } catch (const std::bad_alloc&) {
    delete p;
    return PA_ERR_HOST_MEMORY;
  }
  p->d.host_in = p->d.dev_in = p->d.host_out = p->d.dev_out = nullptr;  // copied above
  for (int k = 0; k < depth; ++k)
    for (auto* v : {&p->h2d_done, &p->kern_done, &p->d2h_done})
      if (cudaEventCreateWithFlags(&(*v)[k], cudaEventDisableTiming) != cudaSuccess) {
        destroy_events(p);
        delete p;
        return PA_ERR_CUDA;
      }
  *out = p;
  return PA_OK;
}

void pa_pipeline_destroy(pa_pipeline* p) {
  if (!p) return;
  pa_pipeline_sync(p);
  destroy_events(p);
  delete p;
}

pa_status pa_pipeline_next_slot(pa_pipeline* p, int* slot) {
  if (!p || !slot) return PA_ERR_INVALID_ARG;
  const int k = static_cast<int>(p->next % p->d.depth);
  if (p->used[k] && cudaEventSynchronize(p->h2d_done[k]) != cudaSuccess) return PA_ERR_CUDA;
  *slot = k;
  return PA_OK;
}

pa_status pa_pipeline_submit(pa_pipeline* p, const int64_t* seq_ids, float scale,
                             int64_t* step, size_t* h2d_bytes) {
  if (!p || !seq_ids) return PA_ERR_INVALID_ARG;
  const pa_pipeline_desc& d = p->d;
  const int k = static_cast<int>(p->next % d.depth);
  char* h = static_cast<char*>(p->h_in[k]);
  char* dv = static_cast<char*>(p->d_in[k]);
  // the host slot was last copied for step next - depth: normally long done
  if (p->used[k] && cudaEventSynchronize(p->h2d_done[k]) != cudaSuccess) return PA_ERR_CUDA;
  // every row's table must still fit the slot's max_blocks after this token: checked first,
  // so that a step that cannot be described changes no allocator state
  pa_status st = pa_alloc_check_append_fits(p->alloc, seq_ids, d.B, d.max_blocks);
  if (st != PA_OK) return st;
  const int m = d.shared_prefix_members;
  int npairs = 0;
  int32_t* pairs_h = reinterpret_cast<int32_t*>(h + p->off[5]);
  int64_t* slots_h = m ? reinterpret_cast<int64_t*>(h + p->off[6]) : p->slots.data();
  st = pa_alloc_append_slots(p->alloc, seq_ids, d.B, slots_h, pairs_h, &npairs);
  if (st != PA_OK) return st;
  st = pa_alloc_block_tables(p->alloc, seq_ids, d.B, reinterpret_cast<int32_t*>(h + p->off[3]),
                             d.max_blocks, reinterpret_cast<int32_t*>(h + p->off[4]));
  if (st != PA_OK) return st;
  int ngroups = 0;
  if (m) {
    // after this step's appends, so that a block copied on write is a member's own
    st = pa_alloc_prefix_groups(p->alloc, seq_ids, d.B, m, PA_SHARED_PREFIX_ALIGN,
                                reinterpret_cast<int32_t*>(h + p->off[7]),
                                reinterpret_cast<int32_t*>(h + p->off[8]),
                                reinterpret_cast<int32_t*>(h + p->off[9]), &ngroups);
    if (st != PA_OK) return st;
  }
  const size_t used = m ? p->off[9] + static_cast<size_t>(ngroups) * m * 4
                      : npairs ? p->off[5] + static_cast<size_t>(npairs) * 8
                               : p->off[4] + static_cast<size_t>(d.B) * 4;
  cudaStream_t cin = reinterpret_cast<cudaStream_t>(d.copy_in);
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(d.compute);
  cudaStream_t cout = reinterpret_cast<cudaStream_t>(d.copy_out);
  // step next - depth has finished reading the device input slot
  if (p->used[k] && cudaStreamWaitEvent(cin, p->kern_done[k], 0) != cudaSuccess)
    return PA_ERR_CUDA;
  if (cudaMemcpyAsync(dv, h, used, cudaMemcpyHostToDevice, cin) != cudaSuccess ||
      cudaEventRecord(p->h2d_done[k], cin) != cudaSuccess ||
      cudaStreamWaitEvent(cs, p->h2d_done[k], 0) != cudaSuccess)
    return PA_ERR_CUDA;
  // the device output slot has been copied out for step next - depth
  if (p->used[k] && cudaStreamWaitEvent(cs, p->d2h_done[k], 0) != cudaSuccess) return PA_ERR_CUDA;
  if (npairs) {
    st = pa_copy_blocks(d.k_pool, d.v_pool, reinterpret_cast<const int32_t*>(dv + p->off[5]),
                        npairs, d.block_size, d.Hkv, d.D, d.num_blocks, d.dtype, d.dev_err_flag,
                        d.compute);
    if (st != PA_OK) return st;
  }
  if (m) {
    st = pa_reshape_and_cache(dv + p->off[1], dv + p->off[2], d.k_pool, d.v_pool,
                              reinterpret_cast<const int64_t*>(dv + p->off[6]), d.B, d.Hkv, d.D,
                              d.block_size, d.num_blocks, d.dtype, d.dev_err_flag, d.compute);
    if (st != PA_OK) return st;
    st = pa_decode_shared_prefix(
        p->d_out[k], dv + p->off[0], d.k_pool, d.v_pool,
        reinterpret_cast<const int32_t*>(dv + p->off[3]),
        reinterpret_cast<const int32_t*>(dv + p->off[4]), d.B, d.Hq, d.Hkv, d.D, d.block_size,
        d.max_blocks, d.num_blocks, scale, d.dtype,
        reinterpret_cast<const int32_t*>(dv + p->off[7]),
        reinterpret_cast<const int32_t*>(dv + p->off[8]),
        reinterpret_cast<const int32_t*>(dv + p->off[9]), ngroups, m, d.workspace,
        d.workspace_bytes, d.dev_err_flag, d.compute);
  } else {
    st = pa_decode_append(p->d_out[k], dv + p->off[0], dv + p->off[1], dv + p->off[2], d.k_pool,
                          d.v_pool, reinterpret_cast<const int32_t*>(dv + p->off[3]),
                          reinterpret_cast<const int32_t*>(dv + p->off[4]), d.B, d.Hq, d.Hkv,
                          d.D, d.block_size, d.max_blocks, d.num_blocks, scale, d.dtype,
                          d.workspace, d.workspace_bytes, d.dev_err_flag, d.compute, nullptr);
  }
  if (st != PA_OK) return st;
  if (cudaEventRecord(p->kern_done[k], cs) != cudaSuccess ||
      cudaStreamWaitEvent(cout, p->kern_done[k], 0) != cudaSuccess ||
      cudaMemcpyAsync(p->h_out[k], p->d_out[k], p->out_bytes, cudaMemcpyDeviceToHost, cout) !=
          cudaSuccess ||
      cudaEventRecord(p->d2h_done[k], cout) != cudaSuccess)
    return PA_ERR_CUDA;
  p->used[k] = 1;
  if (step) *step = p->next;
  if (h2d_bytes) *h2d_bytes = used;
  ++p->next;
  return PA_OK;
}

pa_status pa_pipeline_result(pa_pipeline* p, int64_t step, int* slot) {
  if (!p || !slot || step < 0 || step >= p->next || step < p->next - p->d.depth)
    return PA_ERR_INVALID_ARG;
  const int k = static_cast<int>(step % p->d.depth);
  if (cudaEventSynchronize(p->d2h_done[k]) != cudaSuccess) return PA_ERR_CUDA;
  *slot = k;
  return PA_OK;
}

pa_status pa_pipeline_sync(pa_pipeline* p) {
  if (!p) return PA_ERR_INVALID_ARG;
  for (int k = 0; k < p->d.depth; ++k)
    if (p->used[k] && cudaEventSynchronize(p->d2h_done[k]) != cudaSuccess) return PA_ERR_CUDA;
  return PA_OK;
}

}  // extern "C"
