// pa_decode_no_alloc: the balanced tensor-core decode (decode_stream.cu) with its scratch
// in a static device buffer of this library, for callers that cannot allocate device
// memory.
//
// Who needs it: a caller whose device memory is entirely owned by its own runtime or
// pool (a serving engine that reserves the KV pool and every buffer up front and then
// forbids any further device allocation), or a latency-critical caller for whom a
// cudaMalloc is not acceptable (it may synchronise the device).  Such a caller cannot
// allocate the workspace pa_decode takes.  This entry point takes the same inputs and
// output and uses kScratchBytes of file-scope device memory instead.
//
// Properties:
//   * Allocates nothing: no cudaMalloc, cudaFree or allocating library routine.  The
//     scratch array exists once per device that loads the library, until exit.
//   * The array is device memory of the library's module: it is reserved when the module
//     loads, at context creation under CUDA_MODULE_LOADING=EAGER, or in the first call
//     on the device under lazy loading (the default).
//   * The first call on each device looks up the array's device address with
//     cudaGetSymbolAddress (with that device current) and caches it for the current
//     context (looked up again if the context changes, e.g. after cudaDeviceReset); make
//     that first call before any stream capture, so that neither the module load nor
//     the lookup happens inside one.
//   * Every call on a device uses the same array and leaves its contents behind.  The
//     stream kernel writes every metadata slot and partial it later reads within the
//     same call, so nothing has to start at zero.  Two calls whose kernels overlap on
//     the GPU (different streams, no ordering between them) race on the array: order
//     them, e.g. issue them on one stream.
//   * A shape whose one-wave schedule needs more than kScratchBytes is rejected with
//     PA_ERR_SCRATCH_LIMIT before anything is queued; shapes the stream kernel does not
//     take (fp32, block size 4, G > 16, B > 8192) get PA_ERR_UNSUPPORTED.

#include <cuda.h>

#include <cmath>
#include <mutex>

#include "pa.h"
#include "pa_internal.h"

namespace {

constexpr size_t kScratchBytes = PA_NO_ALLOC_SCRATCH_BYTES;  // 32 MiB per device
constexpr int kMaxDevices = 64;
constexpr int kStreamMaxB = 8192;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

std::mutex g_mu;
// Per device: the context the address was looked up in, and the address.  A device reset
// (cudaDeviceReset) destroys the device's primary context, and the array of the next
// context on that device has another address, so a cached address holds only while the
// current context is the one it came from.
CUcontext g_ctx[kMaxDevices] = {};
void* g_addr[kMaxDevices] = {};

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

// cuCtxGetCurrent through the runtime's driver entry point (the library links only the
// runtime); null if unavailable.
CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(ptr);
  });
  return fn;
}

CUcontext current_context() {
  CUcontext c = nullptr;
  const CtxGetCurrentFn fn = ctx_get_current();
  if (!fn || fn(&c) != CUDA_SUCCESS) return nullptr;
  return c;
}

// Device address of the scratch array in the current context.  The first call on a
// device (and the first after its context changed) looks it up with cudaGetSymbolAddress,
// with that device current; later calls reuse it.  The lookup allocates nothing: the
// array is part of the library's module, reserved when the module loads.
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  CUcontext ctx = current_context();
  if (!g_addr[dev] || !ctx || ctx != g_ctx[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    if (!p) return cudaErrorInvalidSymbol;
    // the lookup made the device's context current if none was
    g_ctx[dev] = ctx ? ctx : current_context();
    g_addr[dev] = p;
  }
  *out = g_addr[dev];
  return cudaSuccess;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace

extern "C" pa_status pa_decode_no_alloc(void* out, const void* q, const void* k_pool,
                                        const void* v_pool, const int32_t* block_tables,
                                        const int32_t* seq_lens, int B, int Hq, int Hkv, int D,
                                        int block_size, int max_blocks, int num_blocks,
                                        float scale, pa_dtype dtype, int32_t* dev_err_flag,
                                        pa_stream_t stream) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || max_blocks <= 0 || num_blocks <= 0 ||
      block_size <= 0 || !std::isfinite(scale) ||
      (dtype != PA_F32 && dtype != PA_BF16))
    return PA_ERR_INVALID_ARG;
  const int G = Hq / Hkv;
  if (!pa::tc_eligible(G, D, block_size, dtype) || B > kStreamMaxB) return PA_ERR_UNSUPPORTED;
  const int tile = 16;  // the stream kernel's tokens per tile
  const int64_t max_seq = static_cast<int64_t>(max_blocks) * block_size;
  if (max_seq > 0x7fffffffLL) return PA_ERR_INVALID_ARG;
  if (static_cast<int64_t>(B) * Hkv * ((max_seq + tile - 1) / tile) >= (int64_t(1) << 31))
    return PA_ERR_UNSUPPORTED;
  if (B == 0) return PA_OK;
  if (!out || !q || !k_pool || !v_pool || !block_tables || !seq_lens) return PA_ERR_INVALID_ARG;
  if (!aligned(out, 16) || !aligned(q, 16) || !aligned(k_pool, 16) || !aligned(v_pool, 16) ||
      !aligned(block_tables, 4) || !aligned(seq_lens, 4) ||
      (dev_err_flag && !aligned(dev_err_flag, 4)))
    return PA_ERR_INVALID_ARG;

  const int grid = pa::stream_grid(D, block_size, G, B);
  if (grid <= 0) return PA_ERR_CUDA;
  if (pa::stream_workspace_bytes(grid * pa::stream_warps_per_cta(block_size), G, D) >
      kScratchBytes)
    return PA_ERR_SCRATCH_LIMIT;
  void* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return PA_ERR_CUDA;

  pa::StreamParams sp{};
  pa::DecodeParams& p = sp.d;
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
  sp.streams = grid * pa::stream_warps_per_cta(block_size);
  pa::stream_carve(&sp, scratch);
  const cudaError_t e =
      pa::launch_decode_stream(sp, grid, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}
