// Paged decode attention, CUDA-core path (fp32 or bf16 storage, fp32 arithmetic).
//
// Same result as the tensor-core path — softmax(scale * q.K^T) V over each sequence's
// tokens, K/V read through the block table ("PagedAttention" concept card, 实现要点) —
// for every supported shape: fp32 inputs (which must not go through TF32), block size
// 4, or GQA groups wider than 16.
//
// One CTA per (sequence, KV head, chunk of up to 4 query heads of its group, context
// partition).  The 4 warps take the partition's blocks round-robin; in a warp each lane
// holds D/32 consecutive columns of q, of each key/value row it reads, and of the
// output accumulator.  Per token: a partial dot product per lane, a butterfly
// all-reduce over the warp, and an fp32 online-softmax update in base 2.  The warps'
// (max, sum, O) merge in shared memory; a single-partition sequence writes the
// normalised output, otherwise a partial for the reduce kernel.

#include <cuda_bf16.h>

#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {

namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kHC = 4;      // query heads per CTA
constexpr int kWarps = 4;

template <typename T>
__device__ __forceinline__ float to_f(T v);
template <>
__device__ __forceinline__ float to_f<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) {
  return __bfloat162float(v);
}

template <typename T>
__device__ __forceinline__ T from_f(float v);
template <>
__device__ __forceinline__ float from_f<float>(float v) { return v; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

template <typename T, int VPT>
__device__ __forceinline__ void load_row(const T* src, float (&dst)[VPT]) {
#pragma unroll
  for (int i = 0; i < VPT; ++i) dst[i] = to_f(src[i]);
}

template <typename T, int D>
__global__ void __launch_bounds__(kWarps * 32) decode_generic_kernel(const DecodeParams p) {
  constexpr int VPT = D / 32;  // columns per lane
  const int nhc = (p.G + kHC - 1) / kHC;
  const int part = blockIdx.x % p.max_parts;
  int rest = blockIdx.x / p.max_parts;
  const int hc = rest % nhc;
  rest /= nhc;
  const int kvh = rest % p.Hkv;
  const int b = rest / p.Hkv;
  const int BS = p.block_size;
  const int P = p.partition_tokens;
  const int h_begin = kvh * p.G + hc * kHC;
  const int nh = min(kHC, p.G - hc * kHC);

  int L = __ldg(p.seq_lens + b);
  const int Lmax = p.max_blocks * BS;
  if (L < 0 || L > Lmax) {
    if (threadIdx.x == 0 && part == 0) flag_error(p.err, PA_DEVERR_BAD_SEQ_LEN);
    L = L < 0 ? 0 : Lmax;
  }
  const int nparts = L > 0 ? (L + P - 1) / P : 1;
  if (part >= nparts) return;

  T* out = static_cast<T*>(p.out);
  const size_t row0 = static_cast<size_t>(b) * p.Hq + h_begin;
  if (L == 0) {
    for (int i = threadIdx.x; i < nh * D; i += blockDim.x) out[row0 * D + i] = from_f<T>(0.f);
    return;
  }

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int tok0 = part * P;
  const int tok1 = min(L, tok0 + P);
  const int blk0 = tok0 / BS;
  const int nblk = (tok1 - tok0 + BS - 1) / BS;

  const T* qp = static_cast<const T*>(p.q);
  const T* kp = static_cast<const T*>(p.k_pool);
  const T* vp = static_cast<const T*>(p.v_pool);
  const float sl2 = p.scale_log2;

  float q[kHC][VPT], acc[kHC][VPT], m[kHC], l[kHC];
#pragma unroll
  for (int h = 0; h < kHC; ++h) {
    if (h < nh) load_row<T, VPT>(qp + (row0 + h) * D + lane * VPT, q[h]);
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      if (h >= nh) q[h][i] = 0.f;
      acc[h][i] = 0.f;
    }
    m[h] = -INFINITY;
    l[h] = 0.f;
  }

  const int32_t* tab = p.block_tables + static_cast<size_t>(b) * p.max_blocks + blk0;
  const size_t row_stride = static_cast<size_t>(p.Hkv) * D;  // elements between tokens
  for (int j = warp; j < nblk; j += kWarps) {
    int phys = __ldg(tab + j);
    if (phys < 0 || phys >= p.num_blocks) {
      if (lane == 0) flag_error(p.err, PA_DEVERR_BAD_BLOCK_ID);
      phys = 0;
    }
    const int t_begin = tok0 + j * BS;
    const int nt = min(BS, tok1 - t_begin);
    const size_t base = (static_cast<size_t>(phys) * BS * p.Hkv + kvh) * D + lane * VPT;
    for (int t = 0; t < nt; ++t) {
      float kr[VPT], vr[VPT];
      load_row<T, VPT>(kp + base + t * row_stride, kr);
      load_row<T, VPT>(vp + base + t * row_stride, vr);
#pragma unroll
      for (int h = 0; h < kHC; ++h) {
        if (h >= nh) continue;
        float s = 0.f;
#pragma unroll
        for (int i = 0; i < VPT; ++i) s = fmaf(q[h][i], kr[i], s);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(kFull, s, off);
        const float x = s * sl2;
        const float m_new = fmaxf(m[h], x);
        const float alpha = exp2f(m[h] - m_new);
        const float w = exp2f(x - m_new);
        m[h] = m_new;
        l[h] = l[h] * alpha + w;
#pragma unroll
        for (int i = 0; i < VPT; ++i) acc[h][i] = fmaf(acc[h][i], alpha, w * vr[i]);
      }
    }
  }

  // merge the warps
  __shared__ float sm_m[kWarps][kHC], sm_l[kWarps][kHC];
  __shared__ float sm_o[kWarps][kHC][D];
  if (lane == 0) {
#pragma unroll
    for (int h = 0; h < kHC; ++h) {
      sm_m[warp][h] = m[h];
      sm_l[warp][h] = l[h];
    }
  }
#pragma unroll
  for (int h = 0; h < kHC; ++h)
#pragma unroll
    for (int i = 0; i < VPT; ++i) sm_o[warp][h][lane * VPT + i] = acc[h][i];
  __syncthreads();

  for (int i = threadIdx.x; i < nh * D; i += blockDim.x) {
    const int h = i / D, d = i - h * D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, sm_m[w][h]);
    float lsum = 0.f, a = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float sc = exp2f(sm_m[w][h] - M);
      lsum += sc * sm_l[w][h];
      a += sc * sm_o[w][h][d];
    }
    const size_t hrow = row0 + h;
    if (nparts == 1) {
      out[hrow * D + d] = from_f<T>(a / lsum);
    } else {
      const size_t slot = hrow * p.max_parts + part;
      p.ws_acc[slot * D + d] = a;
      if (d == 0) {
        p.ws_ml[slot * 2] = M;
        p.ws_ml[slot * 2 + 1] = lsum;
      }
    }
  }
}

// Merge the partitions of every split sequence by log-sum-exp (base 2):
// M = max_p m_p, out = sum_p 2^(m_p - M) acc_p / sum_p 2^(m_p - M) l_p.
template <typename T, int D>
__global__ void __launch_bounds__(D) decode_reduce_kernel(const DecodeParams p) {
  const int bh = blockIdx.x;
  const int b = bh / p.Hq;
  int L = __ldg(p.seq_lens + b);
  const int Lmax = p.max_blocks * p.block_size;
  L = L < 0 ? 0 : (L > Lmax ? Lmax : L);
  const int nparts = L > 0 ? (L + p.partition_tokens - 1) / p.partition_tokens : 1;
  if (nparts <= 1) return;

  extern __shared__ float wts[];  // [max_parts]
  __shared__ float red[D / 32];
  __shared__ float s_M, s_inv;
  const float* ml = p.ws_ml + static_cast<size_t>(bh) * p.max_parts * 2;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  float mx = -INFINITY;
  for (int i = tid; i < nparts; i += D) mx = fmaxf(mx, ml[2 * i]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, off));
  if (lane == 0) red[warp] = mx;
  __syncthreads();
  if (tid == 0) {
    float M = red[0];
    for (int w = 1; w < D / 32; ++w) M = fmaxf(M, red[w]);
    s_M = M;
  }
  __syncthreads();
  const float M = s_M;
  float ls = 0.f;
  for (int i = tid; i < nparts; i += D) {
    const float w = exp2f(ml[2 * i] - M);
    wts[i] = w;
    ls += w * ml[2 * i + 1];
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) ls += __shfl_xor_sync(kFull, ls, off);
  __syncthreads();  // red[] reuse, wts[] complete
  if (lane == 0) red[warp] = ls;
  __syncthreads();
  if (tid == 0) {
    float s = 0.f;
    for (int w = 0; w < D / 32; ++w) s += red[w];
    s_inv = 1.f / s;
  }
  __syncthreads();
  const float* acc = p.ws_acc + static_cast<size_t>(bh) * p.max_parts * D;
  float a = 0.f;
  for (int i = 0; i < nparts; ++i) a = fmaf(wts[i], acc[static_cast<size_t>(i) * D + tid], a);
  static_cast<T*>(p.out)[static_cast<size_t>(bh) * D + tid] = from_f<T>(a * s_inv);
}

template <typename T, int D>
cudaError_t launch_generic_t(const DecodeParams& p, cudaStream_t stream) {
  const int nhc = (p.G + kHC - 1) / kHC;
  const long long grid = static_cast<long long>(p.B) * p.Hkv * nhc * p.max_parts;
  if (grid <= 0) return cudaSuccess;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  decode_generic_kernel<T, D><<<static_cast<unsigned>(grid), kWarps * 32, 0, stream>>>(p);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_reduce_t(const DecodeParams& p, cudaStream_t stream) {
  const long long grid = static_cast<long long>(p.B) * p.Hq;
  if (grid <= 0) return cudaSuccess;
  const size_t smem = sizeof(float) * static_cast<size_t>(p.max_parts);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(decode_reduce_kernel<T, D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  decode_reduce_kernel<T, D><<<static_cast<unsigned>(grid), D, smem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_reduce(const DecodeParams& p, pa_dtype dtype, cudaStream_t stream) {
  if (dtype == PA_BF16)
    return p.D == 64 ? launch_reduce_t<__nv_bfloat16, 64>(p, stream)
                     : launch_reduce_t<__nv_bfloat16, 128>(p, stream);
  return p.D == 64 ? launch_reduce_t<float, 64>(p, stream) : launch_reduce_t<float, 128>(p, stream);
}

cudaError_t launch_decode_generic(const DecodeParams& p, pa_dtype dtype, cudaStream_t stream) {
  cudaError_t e;
  if (dtype == PA_BF16)
    e = p.D == 64 ? launch_generic_t<__nv_bfloat16, 64>(p, stream)
                  : launch_generic_t<__nv_bfloat16, 128>(p, stream);
  else
    e = p.D == 64 ? launch_generic_t<float, 64>(p, stream)
                  : launch_generic_t<float, 128>(p, stream);
  if (e != cudaSuccess || p.max_parts <= 1) return e;
  return launch_decode_reduce(p, dtype, stream);
}

}  // namespace pa
