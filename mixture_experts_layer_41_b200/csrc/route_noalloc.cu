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
#include "common.cuh"

#include <mutex>
#include <stdio.h>

namespace {

constexpr int kNoAllocPartials = 131072;   // float64 entries = 1 MiB
constexpr int kMaxDevices = 64;

// Device-side scratch.  In host code this name is only a handle for the CUDA
// runtime, never a device address: the address comes from
// cudaGetSymbolAddress below, once per device.
static __device__ __align__(256) double g_route_partials[kNoAllocPartials];

std::mutex g_mu;
void *g_addr[kMaxDevices] = {};

// Address of this device's copy of the scratch array (looked up on the first
// call made on each device, with that device current).
cudaError_t scratch_address(double **out) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_addr[dev]) {
    void *p = nullptr;
    err = cudaGetSymbolAddress(&p, g_route_partials);
    if (err != cudaSuccess) return err;
    g_addr[dev] = p;
  }
  *out = static_cast<double *>(g_addr[dev]);
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
