// velox_block_importance_noalloc: block importance without a caller workspace.
//
// Some callers cannot allocate device memory at all: a host framework that
// budgets every byte of the GPU up front and gives its plugins no allocator,
// or a latency-critical loop that cannot afford the device-wide
// synchronisation that cudaMalloc / cudaFree imply.  This entry point serves
// them: the block means that velox_block_importance keeps in the caller's
// workspace live here in one fixed array in the library's own device memory.
//
// The array is a file-scope __device__ variable, so every GPU that loads the
// library holds it (kNoAllocScratchBytes) until the process exits.  In host
// code its name is only a host-side stand-in; its device address is looked up
// with cudaGetSymbolAddress on the first call made while that device is
// current, cached, and passed to the kernels.  The cache is keyed on the
// device's current context (its driver-assigned context id, never reused in a
// process): after cudaDeviceReset, or anything else that replaces the
// device's primary context, the module is loaded again and the array may sit
// at another address, so the next call looks it up again instead of handing
// the kernels a stale pointer.  A failed lookup is not cached.  Nothing in the
// array must start at zero (the pooling kernel writes every mean before the
// logit kernel reads it), so no call clears it.  All calls on a device share
// the one array: calls that overlap on the GPU (other streams, unordered host
// threads) race on it.
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"

namespace velox {
size_t importance_workspace_bytes(int H, int N, int M);
cudaError_t launch_importance(const uint16_t *Q, const uint16_t *K, int H, int N, int M,
                              float scale, float *p, void *ws, cudaStream_t stream);
}  // namespace velox

namespace {

constexpr size_t kNoAllocScratchBytes = VELOX_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char velox_noalloc_scratch[kNoAllocScratchBytes];

struct DeviceScratch {
  std::mutex mu;
  bool valid = false;
  unsigned long long ctx_id = 0;  // context the cached address belongs to
  void *ptr = nullptr;
};
DeviceScratch g_scratch[kMaxDevices];

// Driver entry points for the current context and its id (CUDA 12.0+).
struct CtxFns {
  PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  PFN_cuCtxGetId_v12000 get_id = nullptr;
};
const CtxFns &ctx_fns() {
  static CtxFns f;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      f.get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      f.get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
    cudaGetLastError();
  });
  return f;
}

// Id of the calling thread's current context; false when there is none yet.
bool current_ctx_id(unsigned long long *id) {
  const CtxFns &f = ctx_fns();
  if (!f.get_current || !f.get_id) return false;
  CUcontext ctx = nullptr;
  if (f.get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  return f.get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of the scratch array on the current device, looked up on
// the first call in the device's current context; null with *err set when
// the lookup failed.
void *scratch_on_current_device(cudaError_t *err) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    *err = e != cudaSuccess ? e : cudaErrorInvalidDevice;
    return nullptr;
  }
  DeviceScratch &s = g_scratch[dev];
  std::lock_guard<std::mutex> lock(s.mu);
  unsigned long long id = 0;
  if (s.valid && current_ctx_id(&id) && id == s.ctx_id) {
    *err = cudaSuccess;
    return s.ptr;
  }
  void *p = nullptr;
  e = cudaGetSymbolAddress(&p, velox_noalloc_scratch);  // creates the context if needed
  if (e != cudaSuccess) {
    cudaGetLastError();
    s.valid = false;
    *err = e;
    return nullptr;
  }
  // cache only when the context can be named, so a later context is noticed
  s.valid = current_ctx_id(&id);
  s.ctx_id = id;
  s.ptr = p;
  *err = cudaSuccess;
  return p;
}

}  // namespace

extern "C" velox_status velox_block_importance_noalloc(const velox_bf16 *Q, const velox_bf16 *K,
                                                       int H, int N, int M, int d, int b_tok,
                                                       float scale, float *p,
                                                       velox_stream_t stream) {
  if (!Q || !K || !p || H <= 0 || N <= 0 || M <= 0) return VELOX_ERR_INVALID_ARG;
  if (d != VELOX_HEAD_DIM || b_tok != VELOX_BLOCK_TOK) return VELOX_ERR_UNSUPPORTED;
  if (M > VELOX_MAX_BLOCKS || velox::product_exceeds({H, M, b_tok}, 2147483647LL) ||
      velox::product_exceeds({H, N, b_tok}, 2147483647LL))
    return VELOX_ERR_UNSUPPORTED;
  if (!(scale == scale) || scale - scale != 0.0f) return VELOX_ERR_INVALID_ARG;  // NaN / inf
  if ((reinterpret_cast<uintptr_t>(Q) | reinterpret_cast<uintptr_t>(K) |
       reinterpret_cast<uintptr_t>(p)) & 15u)
    return VELOX_ERR_INVALID_ARG;
  // The fixed array must hold the fp32 means of every query and key block.
  if (velox::importance_workspace_bytes(H, N, M) > kNoAllocScratchBytes)
    return VELOX_ERR_WORKSPACE;
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
    cudaGetLastError();
    return VELOX_ERR_DEVICE;
  }
  if (major != 10) return VELOX_ERR_DEVICE;
  cudaError_t e;
  void *ws = scratch_on_current_device(&e);
  if (ws == nullptr) return VELOX_ERR_CUDA;
  e = velox::launch_importance(Q, K, H, N, M, scale, p, ws, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) {
    cudaGetLastError();
    return VELOX_ERR_CUDA;
  }
  return VELOX_OK;
}
