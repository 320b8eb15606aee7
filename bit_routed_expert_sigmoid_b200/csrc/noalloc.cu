// Routing entry point that needs no device memory from its caller beyond inputs and outputs.
//
// Some callers cannot allocate device memory at the moment they need routing: plug-ins whose host
// framework owns the device allocator and hands out no workspace, and latency-critical loops that
// cannot afford the implicit device synchronisation a cudaMalloc/cudaFree may perform. flint_moe_route_noalloc serves them: it runs the same router
// logits and top-k kernels as flint_moe_forward, but the fp32 logits it produces between the two
// kernels live in a fixed, file-scope device array instead of a caller-provided workspace.
//
// The array is part of the library image: every GPU on which the library is used holds it (64 KiB
// plus a small tail) until the process exits. It bounds the sizes this entry point accepts.
#include <cudaTypedefs.h>

#include <mutex>

#include "../../include/flint_moe.h"
#include "kernels.cuh"

namespace {

constexpr int kNoAllocMaxTokens = 64;
constexpr int kNoAllocMaxExperts = 256;
constexpr int kScratchFloats = kNoAllocMaxTokens * kNoAllocMaxExperts + 64;   // logits + status words

// Logits scratch shared by every call on a device. Its contents persist between calls; each call
// writes the logits of its tokens before reading them, so nothing in it has to start at zero.
static __device__ __align__(256) float g_route_scratch[kScratchFloats];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
float* g_scratch_addr[kMaxDevices] = {};
CUcontext g_scratch_ctx[kMaxDevices] = {};

// The driver's cuCtxGetCurrent, through the runtime (no link-time driver dependency).
PFN_cuCtxGetCurrent_v4000 ctx_getter() {
  static PFN_cuCtxGetCurrent_v4000 fn = nullptr;
  if (!fn) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(f);
  }
  return fn;
}

// Device address of the scratch array for the current device. In host code the symbol itself is
// only a host-side stand-in, so the address must come from cudaGetSymbolAddress, with that device
// current. It is looked up once per device and context: the cached address is kept with the
// context it belongs to, and a different current context (after cudaDeviceReset, say) looks it up
// again.
cudaError_t scratch_for_current_device(float** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  CUcontext ctx = nullptr;
  PFN_cuCtxGetCurrent_v4000 get = ctx_getter();
  if (!get || get(&ctx) != CUDA_SUCCESS) return cudaErrorUnknown;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_addr[dev] || !ctx || g_scratch_ctx[dev] != ctx) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_route_scratch);     // also makes the device's context current
    if (e != cudaSuccess) return e;
    if (get(&ctx) != CUDA_SUCCESS) return cudaErrorUnknown;
    g_scratch_addr[dev] = static_cast<float*>(p);
    g_scratch_ctx[dev] = ctx;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

bool aligned(const void* p, uintptr_t a) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace

extern "C" flint_status flint_moe_route_noalloc(const void* x, const void* router_w, int T, int n_experts, int top_k,
                                                float norm_floor, int* ids, float* w, void* stream) {
  if (T < 0 || T > kNoAllocMaxTokens) return FLINT_ERR_INVALID_ARG;
  if (n_experts < 32 || n_experts > kNoAllocMaxExperts || n_experts % 32 != 0) return FLINT_ERR_INVALID_ARG;
  if (top_k < 1 || top_k > flint::kMaxTopK || top_k > n_experts) return FLINT_ERR_INVALID_ARG;
  if (!(norm_floor > 0.f)) return FLINT_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(router_w, 16) || !aligned(ids, 4) || !aligned(w, 4)) return FLINT_ERR_INVALID_ARG;
  float* scratch = nullptr;
  if (scratch_for_current_device(&scratch) != cudaSuccess) return FLINT_ERR_CUDA;
  if (T == 0) return FLINT_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  float* logits = scratch;
  unsigned* status_word = reinterpret_cast<unsigned*>(scratch + kNoAllocMaxTokens * kNoAllocMaxExperts);
  if (flint::launch_router_logits(static_cast<const uint16_t*>(x), static_cast<const uint16_t*>(router_w), T,
                                  n_experts, logits, s) != cudaSuccess)
    return FLINT_ERR_CUDA;
  // flags = 0: the debug checks (which would write status_word) stay off
  if (flint::launch_topk(logits, 1, nullptr, T, n_experts, top_k, norm_floor, ids, w, 0u, status_word, s) != cudaSuccess)
    return FLINT_ERR_CUDA;
  return FLINT_OK;
}
