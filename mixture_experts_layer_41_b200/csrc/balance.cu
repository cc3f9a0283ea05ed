// Aux-loss-free load balancing ("Mixture-of-Experts" design doc, Aux-loss-free
// load balancing; the bias scheme it names): after a step, every expert's
// routing bias moves one fixed step toward balanced use, up when the expert
// took fewer assignments than the mean and down when it took more.
//
// One block.  The mean is sum/E; the comparison counts[e] < sum/E is taken as
// E * counts[e] < sum in 64-bit integers, so it is exact and order-free.  The
// update itself is one fp32 add (bias +/- coeff).
#include "common.cuh"

namespace moe {
namespace {

__global__ void __launch_bounds__(kMaxExperts)
bias_update_kernel(int E, const int32_t *counts, float *bias, float coeff) {
  pdl_enter();
  __shared__ long long part[kMaxExperts / 32];
  const int e = threadIdx.x, lane = e & 31, warp = e >> 5;
  const long long c = e < E ? (long long)counts[e] : 0;
  long long v = c;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if (lane == 0) part[warp] = v;
  __syncthreads();
  long long total = 0;
  for (int w = 0; w < kMaxExperts / 32; ++w) total += part[w];
  if (e >= E || coeff == 0.0f) return;
  const long long scaled = (long long)E * c;
  if (scaled < total) bias[e] = bias[e] + coeff;
  else if (scaled > total) bias[e] = bias[e] - coeff;
}

}  // namespace

cudaError_t launch_bias_update(int E, const int32_t *counts, float *expert_bias, float coeff, cudaStream_t s) {
  launch_pdl(bias_update_kernel, 1, kMaxExperts, 0, s, E, counts, expert_bias, coeff);
  return cudaGetLastError();
}

}  // namespace moe
