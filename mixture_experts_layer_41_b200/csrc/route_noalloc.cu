// moe_route_noalloc: the router for callers that cannot allocate device memory.
//
// Some callers have no way to hand the library a workspace: code embedded in
// a host framework that owns every device allocation and exposes none to
// plugins, or latency-critical paths where a cudaMalloc (and the device-wide
// synchronisation it may imply) is not acceptable.  For them the router keeps
// its only scratch -- one float64 partial probability sum per (32-token block,
// expert) -- in a fixed array compiled into the library instead of in `ws`.
//
// The array lives in device global memory on every GPU that loads the library
// and stays allocated until the process exits.  Its size caps the problem:
// ceil(T / 32) * E <= kNoAllocPartials (1 MiB of float64).  Every call shares
// it, so calls that overlap on the GPU (two streams, two threads) race and
// must be serialised by the caller.  Each call writes every entry it later
// reads, so nothing needs clearing between calls.
//
// It always runs the CUDA-core router with whole-row blocks: the split and
// tensor-core passes of moe_route keep their logits in the workspace, which
// this call does not have.  Its ids, weights and probability sums therefore
// agree with moe_route's within the router tolerances (ids on tokens whose
// selection margin is clear, weights 1e-6 and sums 1e-5 relative), not bit
// for bit, and large bf16 batches route more slowly than through moe_route.
#include "common.cuh"

#include <cuda.h>
#include <mutex>
#include <stdio.h>

namespace {

constexpr int kNoAllocPartials = 131072;   // float64 entries = 1 MiB
constexpr int kMaxDevices = 64;

// Device-side scratch.  In host code this name is only a handle for the CUDA
// runtime, never a device address: the address comes from
// cudaGetSymbolAddress below, once per device and CUDA context.
static __device__ __align__(256) double g_route_partials[kNoAllocPartials];

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);

struct CachedAddress {
  unsigned long long ctx_id;   // the context the address belongs to (0: none yet)
  void *addr;
};

std::mutex g_mu;
CachedAddress g_cache[kMaxDevices] = {};

template <class Fn>
Fn driver_fn(const char *name) {
  void *p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess || q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<Fn>(p);
}

// Unique id of the context current on this thread (0 if there is none yet).
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
  static CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx) return 0;
  return get_id(ctx, &id) == CUDA_SUCCESS ? id : 0;
}

// Address of the scratch array in the current device's context.  Looked up
// with cudaGetSymbolAddress on the first call in each context and cached per
// device under the context's unique id, so a context created later (after a
// cudaDeviceReset, or a different context made current by the caller) gets
// its own lookup instead of a stale address.
cudaError_t scratch_address(double **out) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  unsigned long long id = current_context_id();
  if (id == 0 || g_cache[dev].ctx_id != id) {
    void *p = nullptr;
    err = cudaGetSymbolAddress(&p, g_route_partials);   // binds the device's context if none was current
    if (err != cudaSuccess) return err;
    if (id == 0) id = current_context_id();
    g_cache[dev].ctx_id = id;   // 0 (no id available): looked up again on the next call
    g_cache[dev].addr = p;
    *out = static_cast<double *>(p);
    return cudaSuccess;
  }
  *out = static_cast<double *>(g_cache[dev].addr);
  return cudaSuccess;
}

bool aligned16(const void *p) { return p != nullptr && ((uintptr_t)p & 15u) == 0; }

}  // namespace

extern "C" moe_status moe_route_noalloc(const moe_config *cfg, const void *x, const float *w_router,
                                        const float *router_bias, int32_t *topk_ids, float *topk_w,
                                        float *prob_sum, moe_stream_t stream) {
  moe_status st = moe_validate(cfg);
  if (st != MOE_OK) return st;
  const moe_config &c = *cfg;
  if (!aligned16(x) || !aligned16(w_router) || ((uintptr_t)router_bias & 15u) != 0 || !aligned16(topk_ids) ||
      !aligned16(topk_w) || !aligned16(prob_sum))
    return MOE_ERR_INVALID_ARG;
  const long long need = (long long)moe::route_blocks(c) * c.num_experts;
  if (need > kNoAllocPartials) {
    char msg[256];
    snprintf(msg, sizeof(msg),
             "moe_route_noalloc: ceil(T/32)*E = %lld partial sums exceed the fixed scratch of %d "
             "(T=%d, E=%d); use moe_route with a workspace",
             need, kNoAllocPartials, c.num_tokens, c.num_experts);
    moe::set_last_error_text(msg);
    return MOE_ERR_UNSUPPORTED;
  }
  double *partials = nullptr;
  cudaError_t err = scratch_address(&partials);
  if (err == cudaSuccess)
    err = moe::launch_route(c, x, w_router, router_bias, topk_ids, topk_w, partials, prob_sum,
                            reinterpret_cast<cudaStream_t>(stream));
  if (err != cudaSuccess) {
    char msg[256];
    snprintf(msg, sizeof(msg), "moe_route_noalloc: %s", cudaGetErrorString(err));
    moe::set_last_error_text(msg);
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}
