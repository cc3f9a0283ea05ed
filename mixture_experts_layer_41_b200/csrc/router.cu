// Router: fused gate GEMV + softmax top-k / sigmoid group-limited top-k.
//
// Follows the "Mixture of Experts" blog (route; Router.route: max-shifted
// softmax, the k best experts, renormalisation over the kept mass) and Edge0
// "MoE Spec and Routing" (select_from_logits, group_select_from_logits:
// sigmoid scores, selection = score + bias, groups ranked by the sum of their
// two best selection scores, routed scaling).
//
// One block = 32 tokens x all E experts, 8 warps.  Warp w owns tokens
// 4w..4w+3; lane l owns experts l, l+32, ... (EPL = ceil(E/32) of them), so
// after the dot products each warp holds every logit of its tokens in
// registers and the selection runs on warp shuffles with no shared-memory
// round trip.  Logits: fp32 products summed over runs of 8 elements, the runs
// added in float64 (keeps the logit error near 1e-7 at d = 7168 where a
// straight fp32 sum would reach ~1e-6).  Scores, selection and weights are
// computed in float64 and rounded to float32 on the store.
#include "common.cuh"

#include <math.h>

namespace moe {
namespace {

constexpr int KC = 32;      // reduction chunk staged in shared memory
constexpr int RUN = 8;      // fp32 run length before the float64 add
constexpr int TPW = 4;      // tokens per warp

struct RouteParams {
  const void *x;
  const float *w;
  const float *bias;
  int T, d, E, k;
  int router, norm;
  double scaling;
  int n_group, topk_group;
  int32_t *ids;
  float *wts;
  double *part;
};

__device__ __forceinline__ void argmax_merge(double &v, int &i, double ov, int oi) {
  if (ov > v || (ov == v && oi < i)) { v = ov; i = oi; }
}

__device__ __forceinline__ void warp_argmax(double &v, int &i) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    double ov = __shfl_xor_sync(0xffffffffu, v, o);
    int oi = __shfl_xor_sync(0xffffffffu, i, o);
    argmax_merge(v, i, ov, oi);
  }
}

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ double warp_max(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmax(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

template <int EPL, bool BF16>
__global__ void __launch_bounds__(kRouteThreads)
route_kernel(RouteParams p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  float *xs = reinterpret_cast<float *>(smem_raw);                  // [32][KC+1]
  float *wsm = xs + kRouteTokens * (KC + 1);                         // [E][KC+1]
  double *gscr = reinterpret_cast<double *>(smem_raw);               // reused after the dot loop
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int t0 = blockIdx.x * kRouteTokens;
  const int E = p.E, d = p.d;

  double acc[TPW][EPL];
#pragma unroll
  for (int i = 0; i < TPW; ++i)
#pragma unroll
    for (int j = 0; j < EPL; ++j) acc[i][j] = 0.0;

  for (int k0 = 0; k0 < d; k0 += KC) {
    // stage x[t0:t0+32, k0:k0+KC] and W_r[:, k0:k0+KC] as fp32
    for (int i = tid; i < kRouteTokens * KC; i += kRouteThreads) {
      const int tok = i / KC, kk = i % KC, t = t0 + tok, kg = k0 + kk;
      float v = 0.f;
      if (t < p.T && kg < d) {
        if (BF16) v = bf16_to_f32(reinterpret_cast<const uint16_t *>(p.x)[(size_t)t * d + kg]);
        else v = reinterpret_cast<const float *>(p.x)[(size_t)t * d + kg];
      }
      xs[tok * (KC + 1) + kk] = v;
    }
    for (int i = tid; i < E * KC; i += kRouteThreads) {
      const int e = i / KC, kk = i % KC, kg = k0 + kk;
      wsm[e * (KC + 1) + kk] = kg < d ? __ldg(p.w + (size_t)e * d + kg) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int r0 = 0; r0 < KC; r0 += RUN) {
      float run[TPW][EPL];
#pragma unroll
      for (int i = 0; i < TPW; ++i)
#pragma unroll
        for (int j = 0; j < EPL; ++j) run[i][j] = 0.f;
#pragma unroll
      for (int kk = r0; kk < r0 + RUN; ++kk) {
        float xv[TPW], wv[EPL];
#pragma unroll
        for (int i = 0; i < TPW; ++i) xv[i] = xs[(warp * TPW + i) * (KC + 1) + kk];
#pragma unroll
        for (int j = 0; j < EPL; ++j) {
          const int e = lane + 32 * j;
          wv[j] = e < E ? wsm[e * (KC + 1) + kk] : 0.f;
        }
#pragma unroll
        for (int i = 0; i < TPW; ++i)
#pragma unroll
          for (int j = 0; j < EPL; ++j) run[i][j] = fmaf(xv[i], wv[j], run[i][j]);
      }
#pragma unroll
      for (int i = 0; i < TPW; ++i)
#pragma unroll
        for (int j = 0; j < EPL; ++j) acc[i][j] += (double)run[i][j];
    }
    __syncthreads();
  }

  // ------------------------------------------------------------ selection
  double psum[EPL];
#pragma unroll
  for (int j = 0; j < EPL; ++j) psum[j] = 0.0;
  double *wscr = gscr + warp * kMaxExperts;   // per-warp scratch row (sigmoid groups)

#pragma unroll 1
  for (int i = 0; i < TPW; ++i) {
    const int t = t0 + warp * TPW + i;
    if (t >= p.T) break;                       // warp-uniform
    double prob[EPL], score[EPL];
    if (p.router == MOE_ROUTER_SOFTMAX_TOPK) {
      double l[EPL];
      double m = -INFINITY;
#pragma unroll
      for (int j = 0; j < EPL; ++j) {
        const int e = lane + 32 * j;
        l[j] = e < E ? acc[i][j] + (p.bias ? (double)p.bias[e] : 0.0) : -INFINITY;
        m = fmax(m, l[j]);
      }
      m = warp_max(m);
      double s = 0.0;
#pragma unroll
      for (int j = 0; j < EPL; ++j) {
        prob[j] = (lane + 32 * j) < E ? exp(l[j] - m) : 0.0;
        s += prob[j];
      }
      s = warp_sum(s);
#pragma unroll
      for (int j = 0; j < EPL; ++j) {
        prob[j] = prob[j] / s;
        score[j] = (lane + 32 * j) < E ? prob[j] : -INFINITY;
      }
    } else {
#pragma unroll
      for (int j = 0; j < EPL; ++j) {
        const int e = lane + 32 * j;
        if (e < E) {
          prob[j] = 1.0 / (1.0 + exp(-acc[i][j]));
          score[j] = prob[j] + (p.bias ? (double)p.bias[e] : 0.0);
          wscr[e] = score[j];
        } else {
          prob[j] = 0.0;
          score[j] = -INFINITY;
        }
      }
      __syncwarp();
      // group score = sum of the two largest selection scores in the group
      const int G = E / p.n_group;
      double gs = -INFINITY;
      if (lane < p.n_group) {
        double b1 = -INFINITY, b2 = -INFINITY;
        for (int q = 0; q < G; ++q) {
          const double v = wscr[lane * G + q];
          if (v > b1) { b2 = b1; b1 = v; } else if (v > b2) { b2 = v; }
        }
        gs = b1 + b2;
      }
      __syncwarp();
      uint32_t keep = 0;
      for (int r = 0; r < p.topk_group; ++r) {
        double v = (keep >> lane) & 1u ? -INFINITY : gs;
        int gi = lane < p.n_group && !((keep >> lane) & 1u) ? lane : 0x7fffffff;
        if (lane >= p.n_group) v = -INFINITY;
        warp_argmax(v, gi);
        keep |= 1u << gi;
      }
#pragma unroll
      for (int j = 0; j < EPL; ++j) {
        const int e = lane + 32 * j;
        if (e < E && !((keep >> (e / G)) & 1u)) score[j] = -INFINITY;
      }
    }
    // psum over all tokens (softmax probability / raw sigmoid)
#pragma unroll
    for (int j = 0; j < EPL; ++j) psum[j] += prob[j];

    // top-k by score, ties to the lower expert index
    uint32_t taken = 0;
    int my_e = -1;
    double my_w = 0.0;
    for (int r = 0; r < p.k; ++r) {
      double bv = -INFINITY;
      int bi = 0x7fffffff;
#pragma unroll
      for (int j = 0; j < EPL; ++j) {
        const int e = lane + 32 * j;
        if (e < E && !((taken >> j) & 1u)) argmax_merge(bv, bi, score[j], e);
      }
      warp_argmax(bv, bi);
      double wv = 0.0;
#pragma unroll
      for (int j = 0; j < EPL; ++j)
        if (lane + 32 * j == bi) { wv = prob[j]; taken |= 1u << j; }
      wv = __shfl_sync(0xffffffffu, wv, bi & 31);
      if (lane == r) { my_e = bi; my_w = wv; }
    }
    const double tot = warp_sum(lane < p.k ? my_w : 0.0);
    double wout;
    if (p.router == MOE_ROUTER_SOFTMAX_TOPK) {
      wout = p.norm ? my_w / fmax(tot, 1e-12) : my_w;
    } else {
      wout = (p.norm ? my_w / (tot + 1e-20) : my_w) * p.scaling;
    }
    if (lane < p.k) {
      p.ids[(size_t)t * p.k + lane] = my_e;
      p.wts[(size_t)t * p.k + lane] = (float)wout;
    }
  }

  // per-block probability sums in a fixed order
  __syncthreads();
  double *part = gscr;  // [8][E]
#pragma unroll
  for (int j = 0; j < EPL; ++j) {
    const int e = lane + 32 * j;
    if (e < E) part[warp * E + e] = psum[j];
  }
  __syncthreads();
  for (int e = tid; e < E; e += kRouteThreads) {
    double s = 0.0;
    for (int w = 0; w < kRouteThreads / 32; ++w) s += part[w * E + e];
    p.part[(size_t)blockIdx.x * E + e] = s;
  }
}

__global__ void route_finalize(const double *part, int nb, int E, float *prob_sum) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= E) return;
  double s = 0.0;
  for (int b = 0; b < nb; ++b) s += part[(size_t)b * E + e];
  prob_sum[e] = (float)s;
}

template <int EPL, bool BF16>
cudaError_t launch_variant(const RouteParams &p, int nb, cudaStream_t s) {
  const size_t stage = sizeof(float) * (size_t)(kRouteTokens + p.E) * (KC + 1);
  const size_t scratch = sizeof(double) * (size_t)(kRouteThreads / 32) * kMaxExperts;
  const size_t smem = stage > scratch ? stage : scratch;
  auto kern = route_kernel<EPL, BF16>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  kern<<<nb, kRouteThreads, smem, s>>>(p);
  return cudaGetLastError();
}

template <bool BF16>
cudaError_t launch_epl(const RouteParams &p, int nb, cudaStream_t s) {
  const int epl = (p.E + 31) / 32;
  if (epl <= 1) return launch_variant<1, BF16>(p, nb, s);
  if (epl <= 2) return launch_variant<2, BF16>(p, nb, s);
  if (epl <= 4) return launch_variant<4, BF16>(p, nb, s);
  return launch_variant<8, BF16>(p, nb, s);
}

}  // namespace

cudaError_t launch_route(const moe_config &c, const void *x, const float *w_router,
                         const float *router_bias, int32_t *topk_ids, float *topk_w,
                         double *route_part, float *prob_sum, cudaStream_t s) {
  RouteParams p;
  p.x = x;
  p.w = w_router;
  p.bias = router_bias;
  p.T = c.num_tokens;
  p.d = c.hidden;
  p.E = c.num_experts;
  p.k = c.top_k;
  p.router = c.router;
  p.norm = c.norm_topk_prob;
  p.scaling = (double)c.routed_scaling;
  p.n_group = c.router == MOE_ROUTER_SIGMOID_GROUP ? c.n_group : 1;
  p.topk_group = c.router == MOE_ROUTER_SIGMOID_GROUP ? c.topk_group : 1;
  p.ids = topk_ids;
  p.wts = topk_w;
  p.part = route_part;
  const int nb = route_blocks(c);
  cudaError_t err = c.act_dtype == MOE_BF16 ? launch_epl<true>(p, nb, s) : launch_epl<false>(p, nb, s);
  if (err != cudaSuccess) return err;
  route_finalize<<<(c.num_experts + 127) / 128, 128, 0, s>>>(route_part, nb, c.num_experts, prob_sum);
  return cudaGetLastError();
}

}  // namespace moe
