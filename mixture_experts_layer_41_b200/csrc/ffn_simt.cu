// Grouped expert FFN in exact fp32 on the CUDA cores.
//
// The fp32 path exists for fp32 layers, whose 1e-5 parity bound a TF32 or
// bf16 tensor-core product cannot meet.  Expert math as in the "Mixture of
// Experts" blog (expert_forward: W_out relu(W_in x)) and the SwiGLU form of
// the "moe-architecture" skill page / Edge0 _swiglu (silu(gate) * up).  One
// thread per output element; each block stages the group offsets in shared
// memory and finds a row's expert by binary search.
#include "common.cuh"

namespace moe {
namespace {

__device__ __forceinline__ int group_of(const int32_t *off, int E, int r) {
  int lo = 0, hi = E;   // largest e with off[e] <= r (off[E] > r)
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (off[mid] <= r) lo = mid; else hi = mid;
  }
  return lo;
}

struct SimtArgs {
  const int32_t *offsets;
  int E, rows, rows_cap, d, F, act;
  int w_stride;   // rows between experts in w1 / w2
  const float *x, *w1, *w2, *w3;
  float *h, *y;
  int *status;
};

// The group offsets in shared memory, clamped to [0, rows_cap] and made
// non-decreasing by the first warp (a repair records kDevBadOffsets).
__device__ __forceinline__ void load_offsets(const SimtArgs &a, int nE, int32_t *off) {
  __shared__ int32_t unused[kMaxExperts + 1];
  if (threadIdx.y == 0) {
    const bool bad = warp_group_offsets(a.offsets, nE, a.rows, a.rows_cap, off, unused, [](int) { return 0; });
    if (bad && threadIdx.x == 0 && a.status) record_status(a.status, kDevBadOffsets);
  }
  __syncthreads();
}

__global__ void simt_phase1(SimtArgs a) {
  pdl_enter();
  __shared__ int32_t off[kMaxExperts + 1];
  const int nE = a.offsets ? a.E : 1;
  load_offsets(a, nE, off);
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  const int r = blockIdx.y * blockDim.y + threadIdx.y;
  if (c >= a.F || r >= off[nE]) return;
  const int e = group_of(off, nE, r);
  const float *xr = a.x + (size_t)r * a.d;
  const float *g = a.w1 + ((size_t)e * a.w_stride + c) * a.d;
  float acc = 0.f;
  for (int k = 0; k < a.d; ++k) acc = fmaf(xr[k], g[k], acc);
  float hv;
  if (a.act == MOE_ACT_RELU) {
    hv = acc > 0.f ? acc : 0.f;
  } else {
    const float *u = a.w2 + ((size_t)e * a.w_stride + c) * a.d;
    float up = 0.f;
    for (int k = 0; k < a.d; ++k) up = fmaf(xr[k], u[k], up);
    hv = acc / (1.f + expf(-acc)) * up;
  }
  a.h[(size_t)r * a.F + c] = hv;
}

__global__ void simt_phase2(SimtArgs a) {
  pdl_enter();
  __shared__ int32_t off[kMaxExperts + 1];
  const int nE = a.offsets ? a.E : 1;
  load_offsets(a, nE, off);
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  const int r = blockIdx.y * blockDim.y + threadIdx.y;
  if (c >= a.d || r >= off[nE]) return;
  const int e = group_of(off, nE, r);
  const float *hr = a.h + (size_t)r * a.F;
  const float *w = a.w3 + ((size_t)e * a.d + c) * a.F;
  float acc = 0.f;
  for (int f = 0; f < a.F; ++f) acc = fmaf(hr[f], w[f], acc);
  a.y[(size_t)r * a.d + c] = acc;
}

}  // namespace

cudaError_t launch_ffn_simt_f32(const FfnArgs &f, cudaStream_t s) {
  SimtArgs a;
  a.offsets = f.offsets;
  a.E = f.E;
  a.rows = f.rows;
  a.rows_cap = f.rows_cap;
  a.status = f.status;
  a.d = f.d;
  a.F = f.F;
  a.act = f.act;
  a.w_stride = f.w_stride;
  a.x = static_cast<const float *>(f.x);
  a.w1 = static_cast<const float *>(f.w1);
  a.w2 = static_cast<const float *>(f.w2);
  a.w3 = static_cast<const float *>(f.w3);
  a.h = static_cast<float *>(f.h);
  a.y = static_cast<float *>(f.y);
  const dim3 blk(32, 8);
  const dim3 g1((f.F + 31) / 32, (f.rows_cap + 7) / 8);
  launch_pdl(simt_phase1, g1, blk, 0, s, a);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  if (f.mid_event && (err = cudaEventRecord(f.mid_event, s)) != cudaSuccess) return err;
  const dim3 g2((f.d + 31) / 32, (f.rows_cap + 7) / 8);
  launch_pdl(simt_phase2, g2, blk, 0, s, a);
  return cudaGetLastError();
}

}  // namespace moe
