// Router: fused gate GEMV + softmax top-k / sigmoid group-limited top-k.
//
// Follows the "Mixture of Experts" blog (route; Router.route: max-shifted
// softmax, the k best experts, renormalisation over the kept mass) and Edge0
// "MoE Spec and Routing" (select_from_logits, group_select_from_logits:
// sigmoid scores, selection = score + bias, groups ranked by the sum of their
// two best selection scores, routed scaling).
//
// Two ways to the logits.  bf16 batches of 512 tokens or more whose weights
// depend on the chosen experts alone (renormalised softmax, sigmoid) take
// the integer tensor-core GEMM of router_i8.cu (float64 partials per hidden
// slice, each logit within a computed bound of exact; or, with
// MOE_ROUTER_TC=bf16, the selection-grade bf16 GEMMs of router_tc.cu);
// route_select_refine (or route_select_group8, a lane per eight experts, for
// sigmoid groups of 8, 16, 32, ... experts over bounded logits) then selects
// from those logits in fp32 and weights the k chosen experts from their
// float64 logits: with bounded logits after adding the x-rounding term
// exactly, listing for route_finish_listed the tokens whose bound could
// matter; with selection-grade ones after an exact recomputation.  All other cases stay on the CUDA cores: fp32 products summed over runs of 8 elements,
// the runs added in float64 (a straight fp32 sum over d = 7168 misses the
// 1e-6 weight bound); scores, selection and weights are float64 and rounded
// to float32 on the store.  CUDA-core shapes:
//   route_rows    E <= 16: one warp per 2-4 tokens, lanes split the hidden
//                 dimension with 16-byte loads, W_r read through L1; the
//                 E logits of a token are warp all-reduced, lane e owns e.
//   route_tiled   E > 16: a block owns 8*TPW tokens x all E experts; x and W_r
//                 chunks of 32 elements are copied k-major into shared memory
//                 with cp.async, double-buffered one chunk ahead; lane l owns
//                 experts l, l+32, ...  With SPLIT the block covers one slice
//                 of the hidden dimension and writes float64 partial logits.
//   route_select  after a SPLIT pass (8-token x 32-expert x hidden-slice
//                 blocks, used when T is too small to fill the GPU with
//                 whole-row blocks, e.g. decode): sums the partial logits of
//                 its tokens (32, or 8 for small T) in slice order into shared
//                 memory, then selects with one warp per token.
// Every selecting block writes one float64 probability sum per (block,
// expert); route_finalize adds the rows in order, so prob_sum is
// deterministic (on the bounded-logit plan route_finish_listed does it, in
// the same launch as the listed tokens' exact re-weighting).
#include "common.cuh"

#include <math.h>
#include <stdlib.h>
#include <string.h>

namespace moe {
namespace {

constexpr int KC = 32;      // hidden-dimension chunk staged in shared memory
constexpr int kMaxSplitSlices = 16;   // hidden slices of the split pass (their sums are read at once)
constexpr int RUN = 8;      // fp32 run length before the float64 add
constexpr int WARPS = kRouteThreads / 32;

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
  double *part;      // [ceil(T/32)][E] probability sums per 32-token group
  double *logits;    // [ks][T][E] partial logits (split path)
  int ks, kchunk;    // split path: number of hidden slices and their length
  const int32_t *forced;   // [T][k] replayed expert ids, or null to select
  int *status;             // device status word (bad / repeated forced ids)
  int refine;              // logits are selection-grade only: weight from exact chosen logits
  // approx: the logits carry a bound per (token, expert),
  //   xst[t] . wst[e] = |dx_t|_1 |w_e|_inf + |xhat_t|_2 |dw_e|_2 + |x2_t|_2 |w3_e|_2
  // (router_i8.cu); a token's chosen logits are recomputed exactly when a
  // chosen bound exceeds tau or two chosen experts' keys lie within their
  // bounds of each other.
  int approx;
  const double *xst, *wst;
  double tau;
  // the x-rounding term is corrected exactly (sum of dx * w over the listed
  // rounded elements) when a token lists all of them (xcnt <= round_list)
  const int *xcnt, *xidx;
  const double *xdx;
  int round_list;
  // tokens whose chosen logits need the exact recomputation are appended
  // here (the count zeroed by the preparation pass) for route_finish_listed
  int *flag_count, *flag_list;
};

__device__ __forceinline__ void argmax_merge(double &v, int &i, double ov, int oi) {
  if (ov > v || (ov == v && oi < i)) { v = ov; i = oi; }
}

// Warp arg-max of (v, i), ties to the lower index (i >= 0): three warp
// reductions on the order-preserving 64-bit image of v.
__device__ __forceinline__ void warp_argmax(double &v, int &i) {
  const unsigned full = 0xffffffffu;
  const unsigned long long u = (unsigned long long)__double_as_longlong(v);
  const unsigned long long key = (u >> 63) ? ~u : (u | 0x8000000000000000ull);
  const uint32_t hi = (uint32_t)(key >> 32), lo = (uint32_t)key;
  const uint32_t mhi = __reduce_max_sync(full, hi);
  const uint32_t mlo = __reduce_max_sync(full, hi == mhi ? lo : 0u);
  i = (int)__reduce_min_sync(full, hi == mhi && lo == mlo ? (uint32_t)i : 0xFFFFFFFFu);
  const unsigned long long mk = ((unsigned long long)mhi << 32) | mlo;
  v = __longlong_as_double((long long)((mk >> 63) ? (mk & 0x7FFFFFFFFFFFFFFFull) : ~mk));
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

// A float32 w as the float64 w * 2^-896, built with integer operations
// (shifts and one multiply-add) instead of a float conversion: the fp32
// exponent and significand bits are placed in the float64 fields unchanged,
// without the exponent re-bias, and the sign moved to bit 63.  Exact for every
// finite w, subnormals and zeros included (the 2^-896 scale maps the fp32
// range onto the float64 normal range); a sum of products with these values
// is multiplied by 2^896 at the end.  Half of the chosen logits' weights are
// converted this way and half with the conversion instruction, so the
// integer and the conversion pipes share the work.
__device__ __forceinline__ double f32_as_f64_scaled(float w) {
  const uint32_t u = __float_as_uint(w);
  const uint32_t t = u >> 3;                       // sign lands in bit 28
  const uint32_t hi = t + (u >> 31) * 0x70000000u; // ... moved to bit 31
  return __hiloint2double((int)hi, (int)(u << 29));
}
constexpr double kTwoTo896 = 0x1p896;

// Exact logits of up to 8 chosen experts (ids[j], valid[j]) of bf16 token t.
// Returns, on every lane, the sum for slot ((lane >> 4) & 1) * 4 +
// ((lane >> 3) & 1) * 2 + ((lane >> 2) & 1).
__device__ __noinline__ double exact_logits8(const RouteParams &p, int t, const int (&ids)[8],
                                                const bool (&valid)[8], int lane) {
  const uint4 *xr = reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(p.x) + (size_t)t * p.d);
  const float4 *wr[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) wr[j] = reinterpret_cast<const float4 *>(p.w + (size_t)(valid[j] ? ids[j] : 0) * p.d);
  double acc[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) acc[j] = 0.0;
  const int nchunk = p.d / 8;
#pragma unroll 1
  for (int i = lane; i < nchunk; i += 32) {
    const uint4 xv = __ldg(xr + i);
    const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
    // the token's 8 elements, widened once for all chosen experts
    double xd[8];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      xd[2 * u] = (double)__uint_as_float(xw[u] << 16);
      xd[2 * u + 1] = (double)__uint_as_float(xw[u] & 0xFFFF0000u);
    }
#pragma unroll
    for (int h = 0; h < 8; h += 4) {               // four chosen experts' loads in flight at a time
    float4 wv[4][2];
#pragma unroll
    for (int jj = 0; jj < 4; ++jj)
      if (valid[h + jj]) {
        wv[jj][0] = __ldg(wr[h + jj] + 2 * i);
        wv[jj][1] = __ldg(wr[h + jj] + 2 * i + 1);
      }
#pragma unroll
    for (int jj = 0; jj < 4; ++jj)
      if (valid[h + jj]) {
        const int j = h + jj;
        // elements 0-3 against the integer-built w * 2^-896 (their sum is
        // scaled back by 2^896, exactly), elements 4-7 against the converted w;
        // every product is exact in float64
        double lo = 0.0;
        lo = fma(xd[0], f32_as_f64_scaled(wv[jj][0].x), lo);
        lo = fma(xd[1], f32_as_f64_scaled(wv[jj][0].y), lo);
        lo = fma(xd[2], f32_as_f64_scaled(wv[jj][0].z), lo);
        lo = fma(xd[3], f32_as_f64_scaled(wv[jj][0].w), lo);
        acc[j] = fma(lo, kTwoTo896, acc[j]);
        acc[j] = fma(xd[4], (double)wv[jj][1].x, acc[j]);
        acc[j] = fma(xd[5], (double)wv[jj][1].y, acc[j]);
        acc[j] = fma(xd[6], (double)wv[jj][1].z, acc[j]);
        acc[j] = fma(xd[7], (double)wv[jj][1].w, acc[j]);
      }
    }
  }
  // halving exchanges: lanes split by bit 4, then 3, then 2 keep half of the slots
  const unsigned full = 0xffffffffu;
  const int b4 = (lane >> 4) & 1, b3 = (lane >> 3) & 1, b2 = (lane >> 2) & 1;
  double h4[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const double keep = b4 ? acc[i + 4] : acc[i];
    const double send = b4 ? acc[i] : acc[i + 4];
    h4[i] = keep + __shfl_xor_sync(full, send, 16);
  }
  double h3[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const double keep = b3 ? h4[i + 2] : h4[i];
    const double send = b3 ? h4[i] : h4[i + 2];
    h3[i] = keep + __shfl_xor_sync(full, send, 8);
  }
  double h2 = (b2 ? h3[1] : h3[0]) + __shfl_xor_sync(full, b2 ? h3[0] : h3[1], 4);
  h2 += __shfl_xor_sync(full, h2, 2);
  h2 += __shfl_xor_sync(full, h2, 1);
  return h2;
}

// Scores, selection and weights of token t, whose logits (without bias) sit
// in l[j] for expert lane + 32 j.  Adds the token's probabilities to psum.
// wscr: this warp's shared scratch row of kMaxExperts doubles.  (The
// tensor-core plans select in route_select_refine instead.)
template <int EPL>
__device__ __forceinline__ void select_token(const RouteParams &p, int t, const double (&lg)[EPL],
                                             double (&psum)[EPL], double *wscr, int lane) {
  const int E = p.E;
  double prob[EPL], score[EPL];
  if (p.router == MOE_ROUTER_SOFTMAX_TOPK) {
    double l[EPL];
    double m = -INFINITY;
#pragma unroll
    for (int j = 0; j < EPL; ++j) {
      const int e = lane + 32 * j;
      l[j] = e < E ? lg[j] + (p.bias ? (double)p.bias[e] : 0.0) : -INFINITY;
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
        prob[j] = 1.0 / (1.0 + exp(-lg[j]));
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
      const bool live = lane < p.n_group && !((keep >> lane) & 1u);
      double v = live ? gs : -INFINITY;
      int gi = live ? lane : 0x7fffffff;
      warp_argmax(v, gi);
      keep |= 1u << (gi & 31);
    }
#pragma unroll
    for (int j = 0; j < EPL; ++j) {
      const int e = lane + 32 * j;
      if (e < E && !((keep >> (e / G)) & 1u)) score[j] = -INFINITY;
    }
  }
#pragma unroll
  for (int j = 0; j < EPL; ++j) psum[j] += prob[j];

  // top-k by score, ties to the lower expert index; or, when replaying, the
  // recorded ids in their recorded order (an id outside [0, E) or one already
  // taken gets weight 0 and flags the status word)
  uint32_t taken = 0;
  int my_e = -1;
  double my_w = 0.0;
  for (int r = 0; r < p.k; ++r) {
    int bi = 0x7fffffff;
    if (p.forced) {
      bi = p.forced[(size_t)t * p.k + r];
    } else {
      double bv = -INFINITY;
#pragma unroll
      for (int j = 0; j < EPL; ++j) {
        const int e = lane + 32 * j;
        if (e < E && !((taken >> j) & 1u)) argmax_merge(bv, bi, score[j], e);
      }
      warp_argmax(bv, bi);
    }
    double wv = 0.0;
    bool again = false;
#pragma unroll
    for (int j = 0; j < EPL; ++j)
      if (lane + 32 * j == bi && bi < E) {
        again = (taken >> j) & 1u;
        wv = again ? 0.0 : prob[j];
        taken |= 1u << j;
      }
    if (p.forced) {
      again = __any_sync(0xffffffffu, again);
      if (lane == 0 && (bi < 0 || bi >= E)) record_status(p.status, kDevBadExpertId);
      else if (lane == 0 && again) record_status(p.status, kDevDuplicateId);
    }
    wv = __shfl_sync(0xffffffffu, wv, bi & 31);
    if (lane == r) { my_e = bi; my_w = wv; }
  }
  const double tot = warp_sum(lane < p.k ? my_w : 0.0);
  double wout;
  if (p.router == MOE_ROUTER_SOFTMAX_TOPK) wout = p.norm ? my_w / fmax(tot, 1e-12) : my_w;
  else wout = (p.norm ? my_w / (tot + 1e-20) : my_w) * p.scaling;
  if (lane < p.k) {
    p.ids[(size_t)t * p.k + lane] = my_e;
    p.wts[(size_t)t * p.k + lane] = (float)wout;
  }
}

// Per-warp probability sums -> one row per 32-token group, warps added in
// order.  tok0_of_warp(w) gives the first token of warp w; every warp's
// tokens lie inside one group.
template <int EPL, int NW = WARPS>
__device__ __forceinline__ void write_prob_partials(const RouteParams &p, double *scratch, const double (&psum)[EPL],
                                                    int block_tok0, int tokens_per_warp, int lane, int warp) {
  __syncthreads();
  const int E = p.E;
#pragma unroll
  for (int j = 0; j < EPL; ++j) {
    const int e = lane + 32 * j;
    if (e < E) scratch[warp * E + e] = psum[j];
  }
  __syncthreads();
  const int warps_per_group = 32 / tokens_per_warp;
  const int groups = (NW + warps_per_group - 1) / warps_per_group;
  for (int i = threadIdx.x; i < groups * E; i += 32 * NW) {
    const int g = i / E, e = i % E;
    const int grow = block_tok0 / 32 + g;
    if (grow * 32 >= p.T) continue;
    double s = 0.0;
    for (int w = g * warps_per_group; w < (g + 1) * warps_per_group && w < NW; ++w) s += scratch[w * E + e];
    p.part[(size_t)grow * E + e] = s;
  }
}

// ---------------------------------------------------------------- E <= 16
template <int EP, bool BF16, int TPW = 2>
__global__ void __launch_bounds__(32 * (32 / TPW))
route_rows(RouteParams p) {
  pdl_enter();
  constexpr int NW = 32 / TPW;                 // warps per 32-token block
  __shared__ double scratch[NW * 16];          // per-warp probability sums
  __shared__ double wscr_all[NW * 32];         // per-warp selection scores (sigmoid groups)
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int E = p.E, d = p.d;
  const int t0 = blockIdx.x * kRouteTokens + warp * TPW;
  double acc[TPW][EP];
#pragma unroll
  for (int i = 0; i < TPW; ++i)
#pragma unroll
    for (int e = 0; e < EP; ++e) acc[i][e] = 0.0;

  constexpr int V = BF16 ? 8 : 4;   // elements per step and lane
  const bool vec = (d % V) == 0;
  if (vec) {
#pragma unroll 2
    for (int k = lane * V; k < d; k += 32 * V) {
      float xv[TPW][V];
#pragma unroll
      for (int i = 0; i < TPW; ++i) {
        const int t = t0 + i;
        if (t < p.T) {
          if (BF16) {
            const uint4 u = __ldg(reinterpret_cast<const uint4 *>(
                static_cast<const uint16_t *>(p.x) + (size_t)t * d + k));
            const uint32_t q[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              xv[i][2 * c] = __uint_as_float(q[c] << 16);
              xv[i][2 * c + 1] = __uint_as_float(q[c] & 0xffff0000u);
            }
          } else {
            const float4 f = __ldg(reinterpret_cast<const float4 *>(
                static_cast<const float *>(p.x) + (size_t)t * d + k));
            xv[i][0] = f.x; xv[i][1] = f.y; xv[i][2] = f.z; xv[i][3] = f.w;
          }
        } else {
#pragma unroll
          for (int c = 0; c < V; ++c) xv[i][c] = 0.f;
        }
      }
#pragma unroll
      for (int e = 0; e < EP; ++e) {
        if (e < E) {
          float wv[V];
          const float4 a = __ldg(reinterpret_cast<const float4 *>(p.w + (size_t)e * d + k));
          wv[0] = a.x; wv[1] = a.y; wv[2] = a.z; wv[3] = a.w;
          if constexpr (V == 8) {
            const float4 b = __ldg(reinterpret_cast<const float4 *>(p.w + (size_t)e * d + k + 4));
            wv[4] = b.x; wv[5] = b.y; wv[6] = b.z; wv[7] = b.w;
          }
#pragma unroll
          for (int i = 0; i < TPW; ++i) {
            float run = 0.f;
#pragma unroll
            for (int c = 0; c < V; ++c) run = fmaf(xv[i][c], wv[c], run);
            acc[i][e] += (double)run;
          }
        }
      }
    }
  } else {
    // fp32 rows whose length is not a multiple of 4: one element per step
    for (int k = lane; k < d; k += 32) {
#pragma unroll
      for (int i = 0; i < TPW; ++i) {
        const int t = t0 + i;
        const float xv = t < p.T ? static_cast<const float *>(p.x)[(size_t)t * d + k] : 0.f;
#pragma unroll
        for (int e = 0; e < EP; ++e)
          if (e < E) acc[i][e] += (double)(xv * __ldg(p.w + (size_t)e * d + k));
      }
    }
  }
#pragma unroll
  for (int i = 0; i < TPW; ++i)
#pragma unroll
    for (int e = 0; e < EP; ++e) acc[i][e] = warp_sum(acc[i][e]);

  double psum[1] = {0.0};
  double *wscr = wscr_all + warp * 32;
#pragma unroll
  for (int i = 0; i < TPW; ++i) {
    const int t = t0 + i;
    if (t < p.T) {
      double lg[1];
      lg[0] = 0.0;
#pragma unroll
      for (int e = 0; e < EP; ++e)
        if (e == lane) lg[0] = acc[i][e];
      select_token<1>(p, t, lg, psum, wscr, lane);
    }
  }
  write_prob_partials<1, NW>(p, scratch, psum, blockIdx.x * kRouteTokens, TPW, lane, warp);
}

// ---------------------------------------------------------------- E > 16
template <int EPL, int TPW, bool BF16>
struct TiledShape {
  static constexpr int TM = WARPS * TPW;             // tokens per block
  static constexpr int XS = TM + 4;                  // x row stride (words), keeps 16-byte rows
  static constexpr int XW = (BF16 ? KC / 2 : KC) * XS;   // x words per stage (bf16 kept as pairs)
  __host__ __device__ static int stage_words(int E) { return (XW + KC * (E + 1) + 3) / 4 * 4; }
};

__device__ __forceinline__ void cp_async4(void *smem, const void *gmem, bool valid) {
  const uint32_t s = (uint32_t)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(s), "l"(gmem), "r"(valid ? 4 : 0) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

template <int EPL, int TPW, bool BF16, bool SPLIT>
__global__ void __launch_bounds__(kRouteThreads, 1)
route_tiled(RouteParams p) {
  pdl_enter();
  using S = TiledShape<EPL, TPW, BF16>;
  constexpr int TM = S::TM, XS = S::XS, XW = S::XW;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  uint32_t *stage_base = reinterpret_cast<uint32_t *>(smem_raw);
  double *dscr = reinterpret_cast<double *>(smem_raw);   // reused after the dot loop
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int E = p.E, d = p.d;
  // experts of this block: all of them, or (SPLIT) a slice of 32*EPL
  const int e0 = SPLIT ? blockIdx.z * 32 * EPL : 0;
  const int EB = SPLIT ? min(32 * EPL, E - e0) : E;
  const int WSTR = EB + 1;
  const int SW = S::stage_words(EB);
  const int t0 = blockIdx.x * TM;
  int kbeg = 0, kend = d;
  if (SPLIT) {
    kbeg = blockIdx.y * p.kchunk;
    kend = min(d, kbeg + p.kchunk);
  }

  // chunk k0 -> stage st: x as bf16 pairs (or fp32) k-major, W_r fp32 k-major;
  // 4-byte cp.async, zero fill outside the tile
  auto issue = [&](int k0, int st) {
    uint32_t *xs = stage_base + st * SW;
    float *ws = reinterpret_cast<float *>(xs + XW);
    if (BF16) {
      const uint32_t *xg = static_cast<const uint32_t *>(p.x);
      for (int i = tid; i < TM * (KC / 2); i += kRouteThreads) {
        const int tok = i / (KC / 2), j = i % (KC / 2);
        const int t = t0 + tok, kg = k0 + 2 * j;
        const bool ok = t < p.T && kg < kend;
        cp_async4(xs + j * XS + tok, ok ? xg + ((size_t)t * d + kg) / 2 : xg, ok);
      }
    } else {
      const float *xg = static_cast<const float *>(p.x);
      for (int i = tid; i < TM * KC; i += kRouteThreads) {
        const int tok = i / KC, kk = i % KC;
        const int t = t0 + tok, kg = k0 + kk;
        const bool ok = t < p.T && kg < kend;
        cp_async4(xs + kk * XS + tok, ok ? xg + (size_t)t * d + kg : xg, ok);
      }
    }
    for (int i = tid; i < EB * KC; i += kRouteThreads) {
      const int e = i / KC, kk = i % KC, kg = k0 + kk;
      const bool ok = kg < kend;
      cp_async4(ws + kk * WSTR + e, ok ? p.w + (size_t)(e0 + e) * d + kg : p.w, ok);
    }
    cp_async_commit();
  };

  double acc[TPW][EPL];
#pragma unroll
  for (int i = 0; i < TPW; ++i)
#pragma unroll
    for (int j = 0; j < EPL; ++j) acc[i][j] = 0.0;

  int st = 0;
  if (kbeg < kend) issue(kbeg, 0);
  for (int k0 = kbeg; k0 < kend; k0 += KC, st ^= 1) {
    if (k0 + KC < kend) {
      issue(k0 + KC, st ^ 1);               // next chunk lands while this one is used
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const uint32_t *xs = stage_base + st * SW;
    const float *ws = reinterpret_cast<const float *>(xs + XW);
#pragma unroll
    for (int r0 = 0; r0 < KC; r0 += RUN) {
      float run[TPW][EPL];
#pragma unroll
      for (int i = 0; i < TPW; ++i)
#pragma unroll
        for (int j = 0; j < EPL; ++j) run[i][j] = 0.f;
      if (BF16) {
#pragma unroll
        for (int kk = r0; kk < r0 + RUN; kk += 2) {
          uint32_t xp[TPW];
          if (TPW % 4 == 0) {
#pragma unroll
            for (int m = 0; m < TPW / 4; ++m) {
              const uint4 q = *reinterpret_cast<const uint4 *>(xs + (kk / 2) * XS + warp * TPW + 4 * m);
              xp[4 * m] = q.x; xp[4 * m + 1] = q.y; xp[4 * m + 2] = q.z; xp[4 * m + 3] = q.w;
            }
          } else {
#pragma unroll
            for (int i = 0; i < TPW; ++i) xp[i] = xs[(kk / 2) * XS + warp * TPW + i];
          }
          float w0[EPL], w1[EPL];
#pragma unroll
          for (int j = 0; j < EPL; ++j) {
            const int e = lane + 32 * j;
            w0[j] = e < EB ? ws[kk * WSTR + e] : 0.f;
            w1[j] = e < EB ? ws[(kk + 1) * WSTR + e] : 0.f;
          }
#pragma unroll
          for (int i = 0; i < TPW; ++i) {
            const float x0 = __uint_as_float(xp[i] << 16), x1 = __uint_as_float(xp[i] & 0xffff0000u);
#pragma unroll
            for (int j = 0; j < EPL; ++j) {
              run[i][j] = fmaf(x0, w0[j], run[i][j]);
              run[i][j] = fmaf(x1, w1[j], run[i][j]);
            }
          }
        }
      } else {
        const float *xf = reinterpret_cast<const float *>(xs);
#pragma unroll
        for (int kk = r0; kk < r0 + RUN; ++kk) {
          float xv[TPW], wv[EPL];
          if (TPW % 4 == 0) {
#pragma unroll
            for (int m = 0; m < TPW / 4; ++m) {
              const float4 f = *reinterpret_cast<const float4 *>(xf + kk * XS + warp * TPW + 4 * m);
              xv[4 * m] = f.x; xv[4 * m + 1] = f.y; xv[4 * m + 2] = f.z; xv[4 * m + 3] = f.w;
            }
          } else {
#pragma unroll
            for (int i = 0; i < TPW; ++i) xv[i] = xf[kk * XS + warp * TPW + i];
          }
#pragma unroll
          for (int j = 0; j < EPL; ++j) {
            const int e = lane + 32 * j;
            wv[j] = e < EB ? ws[kk * WSTR + e] : 0.f;
          }
#pragma unroll
          for (int i = 0; i < TPW; ++i)
#pragma unroll
            for (int j = 0; j < EPL; ++j) run[i][j] = fmaf(xv[i], wv[j], run[i][j]);
        }
      }
#pragma unroll
      for (int i = 0; i < TPW; ++i)
#pragma unroll
        for (int j = 0; j < EPL; ++j) acc[i][j] += (double)run[i][j];
    }
    __syncthreads();
  }

  if constexpr (SPLIT) {
#pragma unroll
    for (int i = 0; i < TPW; ++i) {
      const int t = t0 + warp * TPW + i;
      if (t < p.T) {
#pragma unroll
        for (int j = 0; j < EPL; ++j) {
          const int e = lane + 32 * j;
          if (e < EB) p.logits[((size_t)blockIdx.y * p.T + t) * E + e0 + e] = acc[i][j];
        }
      }
    }
  } else {
    double psum[EPL];
#pragma unroll
    for (int j = 0; j < EPL; ++j) psum[j] = 0.0;
    double *wscr = dscr + warp * kMaxExperts;
#pragma unroll
    for (int i = 0; i < TPW; ++i) {
      const int t = t0 + warp * TPW + i;
      if (t < p.T) select_token<EPL>(p, t, acc[i], psum, wscr, lane);
    }
    write_prob_partials<EPL>(p, dscr, psum, t0, TPW, lane, warp);
  }
}

// route_select: one warp per token, TPB tokens per block (32, or 8 when a
// 32-token grid would leave more than half of the SMs idle); block b writes
// probability-sum row b of p.part.
// The selection of block-tile `tile` (tokens tile*TPB ..): sums the float64
// partial logits of its tokens in slice order, selects with one warp per
// token and writes probability-sum row `tile`.
// TPB tokens per block, WPB warps (tokens warp, warp + WPB, ... in order).
template <int EPL, int TPB, int WPB>
__device__ __forceinline__ void select_tile(const RouteParams &p, int tile, unsigned char *smem_raw) {
  double *lgs = reinterpret_cast<double *>(smem_raw);                 // [TPB][E] summed logits
  double *dscr = lgs + TPB * p.E;                                    // [TPB][kMaxExperts]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int E = p.E;
  const int tb = tile * TPB;
  constexpr int NT = 32 * WPB;
  // every thread sums the slices of its (token, expert) logits in slice
  // order, the loads of all slices of one logit in flight together
  const int n = TPB * E;
  for (int o = threadIdx.x; o < n; o += NT) {
    // all of the entry's slices (at most 16) in flight at once, then added in order
    const int t = tb + o / E;
    const bool live = t < p.T;
    const double *src = p.logits + (size_t)(live ? t : 0) * E + o % E;
    double v[kMaxSplitSlices];
#pragma unroll
    for (int q = 0; q < kMaxSplitSlices; ++q) v[q] = live && q < p.ks ? src[(size_t)q * p.T * E] : 0.0;
    double acc = 0.0;
#pragma unroll
    for (int q = 0; q < kMaxSplitSlices; ++q)
      if (q < p.ks) acc += v[q];
    lgs[o] = acc;
  }
  __syncthreads();
  double psum[EPL];
#pragma unroll
  for (int j = 0; j < EPL; ++j) psum[j] = 0.0;
  double *wscr = dscr + warp * kMaxExperts;
  for (int i = warp; i < TPB; i += WPB) {
    const int t = tb + i;
    if (t >= p.T) break;
    double lg[EPL];
#pragma unroll
    for (int j = 0; j < EPL; ++j) {
      const int e = lane + 32 * j;
      lg[j] = e < E ? lgs[i * E + e] : 0.0;
    }
    select_token<EPL>(p, t, lg, psum, wscr, lane);
    __syncwarp();
  }
  // the block's probability sums, warps added in order
  __syncthreads();
#pragma unroll
  for (int j = 0; j < EPL; ++j) {
    const int e = lane + 32 * j;
    if (e < E) dscr[warp * E + e] = psum[j];
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += NT) {
    double sum = 0.0;
    for (int w = 0; w < WPB; ++w) sum += dscr[w * E + e];
    p.part[(size_t)tile * E + e] = sum;
  }
}

template <int EPL, int TPB, int WPB>
__global__ void __launch_bounds__(32 * WPB, 1)
route_select(RouteParams p) {
  pdl_enter();
  extern __shared__ __align__(16) unsigned char smem_raw[];
  select_tile<EPL, TPB, WPB>(p, blockIdx.x, smem_raw);
}

// ---------------------------------------------------------------- tensor-core plan: selection + exact weights
// After the tensor-core logits (selection grade, within about 1e-5 of the
// exact value) every token is handled by one warp in two parts:
//  * selection in fp32 on those logits: softmax top-k (ranked by logit plus
//    logit bias), or sigmoid scores, selection = score + bias, group top-two
//    sums, the best topk_group groups and the top-k inside them; the token's
//    probabilities (softmax p, or raw sigmoid s) feed the block's prob sums;
//  * the chosen experts' logits recomputed exactly in ONE pass over the
//    token's row: each 8-element chunk of x is widened to float64 once and
//    used for up to 8 chosen experts (float64 products of bf16 x fp32 are
//    exact, summed in float64 per lane in index order), then the eight lane
//    sums are reduced across the warp by halving exchanges (18 shuffles
//    instead of 8 full reductions).  Weights and the slot order come from
//    these exact logits, as in the CUDA-core router.
// Router replay (forced ids) takes the recorded ids instead of the top-k.

// Warp arg-max of (v, i), ties to the lower index: two warp reductions on
// an order-preserving integer image of v.
__device__ __forceinline__ void warp_argmax_f(float &v, int &i) {
  const uint32_t u = __float_as_uint(v);
  const uint32_t key = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  const uint32_t kmax = __reduce_max_sync(0xffffffffu, key);
  i = __reduce_min_sync(0xffffffffu, key == kmax ? i : 0x7fffffff);
  v = __uint_as_float((kmax & 0x80000000u) ? (kmax & 0x7fffffffu) : ~kmax);
}

// TPB tokens per block, WPB warps (TPB / WPB tokens per warp, in order).
// Shared memory: the block's per-token probabilities [TPB][E] (fp32) and a
// selection-score row per warp [WPB][E].
template <int EPL, int TPB, int WPB>
__global__ void __launch_bounds__(32 * WPB, WPB <= 8 ? 2 : 1)
route_select_refine(RouteParams p) {
  pdl_enter();
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int E = p.E;
  float *pr = reinterpret_cast<float *>(smem_raw);        // [TPB][E]
  float *scr_all = pr + (size_t)TPB * E;                   // [WPB][E]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const unsigned full = 0xffffffffu;
  float *scr = scr_all + (size_t)warp * E;
  const bool softmax = p.router == MOE_ROUTER_SOFTMAX_TOPK;
  const int G = E / p.n_group;

  for (int i = 0; i < TPB / WPB; ++i) {
    const int tl = warp * (TPB / WPB) + i;                 // token within the block
    const int t = blockIdx.x * TPB + tl;
    if (t >= p.T) {
#pragma unroll
      for (int j = 0; j < EPL; ++j)
        if (lane + 32 * j < E) pr[tl * E + lane + 32 * j] = 0.f;
      continue;
    }
    // the logits: the hidden slices added in order, the loads of four
    // slices (all of the token's experts) in flight together; the float64
    // sums stay for the chosen experts
    float lg[EPL];
    double lgd[EPL];
#pragma unroll
    for (int j = 0; j < EPL; ++j) lgd[j] = 0.0;
#pragma unroll 4
    for (int q = 0; q < p.ks; ++q) {
      const double *row = p.logits + ((size_t)q * p.T + t) * E;
#pragma unroll
      for (int j = 0; j < EPL; ++j)
        if (lane + 32 * j < E) lgd[j] += row[lane + 32 * j];
    }
    // the token's bound factors, loaded while the selection runs
    int xcnt = 0;
    double xs0 = 0.0, xs1 = 0.0, xs2 = 0.0;
    if (p.approx) {
      xcnt = p.xcnt[t];
      xs0 = p.xst[(size_t)t * 4];
      xs1 = p.xst[(size_t)t * 4 + 1];
      xs2 = p.xst[(size_t)t * 4 + 2];
    }
#pragma unroll
    for (int j = 0; j < EPL; ++j) lg[j] = (float)lgd[j];
    float score[EPL], prob[EPL];
    if (softmax) {
      float m = -INFINITY;
#pragma unroll
      for (int j = 0; j < EPL; ++j) {
        const int e = lane + 32 * j;
        score[j] = e < E ? lg[j] + (p.bias ? p.bias[e] : 0.f) : -INFINITY;
        m = fmaxf(m, score[j]);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(full, m, o));
      float sum = 0.f;
#pragma unroll
      for (int j = 0; j < EPL; ++j) {
        prob[j] = (lane + 32 * j) < E ? __expf(score[j] - m) : 0.f;
        sum += prob[j];
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(full, sum, o);
#pragma unroll
      for (int j = 0; j < EPL; ++j) prob[j] = __fdividef(prob[j], sum);
    } else {
#pragma unroll
      for (int j = 0; j < EPL; ++j) {
        const int e = lane + 32 * j;
        if (e < E) {
          prob[j] = __fdividef(1.f, 1.f + __expf(-lg[j]));
          score[j] = prob[j] + (p.bias ? p.bias[e] : 0.f);
          if (G != 32) scr[e] = score[j];
        } else {
          prob[j] = 0.f;
          score[j] = -INFINITY;
        }
      }
      // group score: the sum of the group's two largest selection scores
      float gs = -INFINITY;
      if (G == 32) {
        // group g is column g of the lanes' scores: two warp arg-max reductions
#pragma unroll
        for (int g = 0; g < EPL; ++g)
          if (g < p.n_group) {
            float v1 = score[g];
            int i1 = lane;
            warp_argmax_f(v1, i1);
            float v2 = lane == i1 ? -INFINITY : score[g];
            int i2 = lane;
            warp_argmax_f(v2, i2);
            if (lane == g) gs = v1 + v2;
          }
      } else {
        __syncwarp();
        if (lane < p.n_group) {
          float b1 = -INFINITY, b2 = -INFINITY;
          for (int q = 0; q < G; ++q) {
            const float v = scr[lane * G + q];
            if (v > b1) { b2 = b1; b1 = v; } else if (v > b2) { b2 = v; }
          }
          gs = b1 + b2;
        }
      }
      __syncwarp();
      uint32_t keep = 0;
      for (int r = 0; r < p.topk_group; ++r) {
        const bool live = lane < p.n_group && !((keep >> lane) & 1u);
        float v = live ? gs : -INFINITY;
        int gi = live ? lane : 0x7fffffff;
        warp_argmax_f(v, gi);
        keep |= 1u << (gi & 31);
      }
#pragma unroll
      for (int j = 0; j < EPL; ++j) {
        const int e = lane + 32 * j;
        if (e < E && !((keep >> (e / G)) & 1u)) score[j] = -INFINITY;
      }
    }
#pragma unroll
    for (int j = 0; j < EPL; ++j)
      if (lane + 32 * j < E) pr[tl * E + lane + 32 * j] = prob[j];

    // the k choices (lane r keeps choice r): top-k by score, ties to the lower
    // index, or the recorded ids (an id outside [0, E) or already taken is a
    // bad route: weight 0, status flagged)
    uint32_t taken = 0;
    int my_e = -1;
    bool my_ok = false;
    double my_l = 0.0;
    for (int r = 0; r < p.k; ++r) {
      int bi;
      if (p.forced) {
        bi = p.forced[(size_t)t * p.k + r];
      } else {
        float bv = -INFINITY;
        bi = 0x7fffffff;
#pragma unroll
        for (int j = 0; j < EPL; ++j) {
          const int e = lane + 32 * j;
          if (e < E && !((taken >> j) & 1u) && (score[j] > bv || (score[j] == bv && e < bi))) {
            bv = score[j];
            bi = e;
          }
        }
        warp_argmax_f(bv, bi);
      }
      bool again = false;
      double lv = 0.0;
#pragma unroll
      for (int j = 0; j < EPL; ++j)
        if (lane + 32 * j == bi && bi >= 0 && bi < E) {
          again = (taken >> j) & 1u;
          taken |= 1u << j;
          lv = lgd[j];
        }
      again = __any_sync(full, again);
      lv = __shfl_sync(full, lv, bi & 31);
      if (lane == r) my_l = lv;
      if (p.forced && lane == 0) {
        if (bi < 0 || bi >= E) record_status(p.status, kDevBadExpertId);
        else if (again) record_status(p.status, kDevDuplicateId);
      }
      if (lane == r) {
        my_e = bi;
        my_ok = bi >= 0 && bi < E && !again;
      }
    }

    // the chosen experts' logits: with bounded logits (approx) the float64
    // sums, the x-rounding term added exactly where listed, and an exact
    // recomputation only where a bound exceeds tau or two chosen keys lie
    // within their bounds; selection-grade logits are always recomputed
    bool exact = true;
    if (p.approx) {
      double bnd = 0.0, key = 0.0;
      const bool mine = lane < p.k && my_ok;
      if (mine) {
        const double *ws = p.wst + (size_t)my_e * 4;
        if (xcnt <= p.round_list) {
          const size_t o = (size_t)t * p.round_list;
          const float *wr = p.w + (size_t)my_e * p.d;
          double corr = 0.0;
          for (int q = 0; q < xcnt; ++q) {
            // (an index outside the row, left by a preparation pass that gave up, adds nothing)
            const int ix = p.xidx[o + q];
            if ((unsigned)ix < (unsigned)p.d) corr = fma(p.xdx[o + q], (double)__ldg(wr + ix), corr);
          }
          my_l += corr;
        } else {
          bnd = xs0 * ws[0];
        }
        bnd += xs1 * ws[1] + xs2 * ws[2];
        const double b = p.bias ? (double)p.bias[my_e] : 0.0;
        key = softmax ? my_l + b : 1.0 / (1.0 + exp(-my_l)) + b;
      }
      bool need = mine && bnd > p.tau;
      if (!p.forced)
        for (int j = 0; j < p.k; ++j) {
          const double kj = __shfl_sync(full, key, j), bj = __shfl_sync(full, bnd, j);
          const bool okj = __shfl_sync(full, my_ok, j) && j < p.k;
          // |key error| <= bound (softmax: key = logit + bias; sigmoid: a quarter of it)
          if (mine && okj && j != lane && fabs(kj - key) <= bj + bnd) need = true;
        }
      exact = __any_sync(full, need);
      if (exact) {
        // the provisional weights below are replaced by route_finish_listed
        if (lane == 0) p.flag_list[atomicAdd(p.flag_count, 1)] = t;
        exact = false;
      }
    }
    if (!p.approx) my_l = 0.0;
    for (int j0 = 0; exact && j0 < p.k; j0 += 8) {
      int ids[8];
      bool valid[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        ids[j] = __shfl_sync(full, my_e, (j0 + j) & 31);
        valid[j] = __shfl_sync(full, my_ok ? 1 : 0, (j0 + j) & 31) != 0 && j0 + j < p.k;
      }
      const double part = exact_logits8(p, t, ids, valid, lane);
      // slot j of this pass sits on lane ((j >> 2) & 1) * 16 + ((j >> 1) & 1) * 8 + (j & 1) * 4
      const int j = lane - j0;
      const int src = j >= 0 && j < 8 ? (((j >> 2) & 1) << 4) | (((j >> 1) & 1) << 3) | ((j & 1) << 2) : 0;
      const double got = __shfl_sync(full, part, src);
      if (j >= 0 && j < 8) my_l = got;
    }
    // weights from the exact logits; key = the exact selection score (slot order)
    double wv = 0.0, key = -INFINITY;
    if (lane < p.k && my_ok) {
      const double b = p.bias ? (double)p.bias[my_e] : 0.0;
      if (softmax) {
        wv = my_l + b;
        key = wv;
      } else {
        wv = 1.0 / (1.0 + exp(-my_l));
        key = wv + b;
      }
    }
    if (softmax) {
      double m = lane < p.k && my_ok ? wv : -INFINITY;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmax(m, __shfl_xor_sync(full, m, o));
      wv = lane < p.k && my_ok ? exp(wv - m) : 0.0;
    }
    double tot = lane < p.k ? wv : 0.0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(full, tot, o);
    double wout;
    if (softmax) wout = p.norm ? wv / fmax(tot, 1e-12) : wv;
    else wout = (p.norm ? wv / (tot + 1e-20) : wv) * p.scaling;
    int slot = lane;
    if (!p.forced) {
      slot = 0;
      for (int j = 0; j < p.k; ++j) {
        const double kj = __shfl_sync(full, key, j);
        const int ej = __shfl_sync(full, my_e, j);
        if (kj > key || (kj == key && ej < my_e)) ++slot;
      }
    }
    if (lane < p.k) {
      p.ids[(size_t)t * p.k + slot] = my_e;
      p.wts[(size_t)t * p.k + slot] = (float)wout;
    }
  }
  // the block's probability sums, tokens added in order
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += 32 * WPB) {
    double sum = 0.0;
    for (int tl = 0; tl < TPB; ++tl) sum += (double)pr[tl * E + e];
    p.part[(size_t)blockIdx.x * E + e] = sum;
  }
}

// Sigmoid group-limited selection over bounded logits (the integer plan),
// for E <= 256 experts (E a multiple of 8) in groups of G = 8 LG experts, LG a
// power of two: lane l holds experts 8 l .. 8 l + 7, so a group is LG
// adjacent lanes.  A group's two largest selection scores come from each
// lane's own top two and log2(LG) butterfly merges; the kept groups from one
// rank count over the n_group group scores; the top k from each lane's
// scores sorted once (keys: score, then the lower expert), k rounds taking
// the largest head over the warp.  Same choices, weights, bound checks and
// listing as route_select_refine (ties to the lower index throughout).
__device__ __forceinline__ uint32_t score_key(float v) {
  const uint32_t u = __float_as_uint(v);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ void cas_desc(unsigned long long &a, unsigned long long &b) {
  const unsigned long long hi = a > b ? a : b, lo = a > b ? b : a;
  a = hi;
  b = lo;
}

template <int TPB>
__global__ void __launch_bounds__(256, 2) route_select_group8(RouteParams p) {
  pdl_enter();
  constexpr int WPB = 8;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int E = p.E;
  float *pr = reinterpret_cast<float *>(smem_raw);        // [TPB][E] per-token probabilities
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const unsigned full = 0xffffffffu;
  const int LG = E / p.n_group / 8;                        // lanes per group
  const int e0 = 8 * lane;
  const bool live = e0 < E;
  float bias[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) bias[j] = live && p.bias ? p.bias[e0 + j] : 0.f;

  for (int i = 0; i < TPB / WPB; ++i) {
    const int tl = warp * (TPB / WPB) + i;
    const int t = blockIdx.x * TPB + tl;
    float4 *prow = reinterpret_cast<float4 *>(pr + (size_t)tl * E + e0);
    if (t >= p.T) {
      if (live) prow[0] = prow[1] = make_float4(0.f, 0.f, 0.f, 0.f);
      continue;
    }
    // the logits: the hidden slices added in order; the token's bound factors
    // loaded while the selection runs
    double lgd[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) lgd[j] = 0.0;
    if (live) {
#pragma unroll 2
      for (int q = 0; q < p.ks; ++q) {
        const double2 *row = reinterpret_cast<const double2 *>(p.logits + ((size_t)q * p.T + t) * E + e0);
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const double2 v = row[h];
          lgd[2 * h] += v.x;
          lgd[2 * h + 1] += v.y;
        }
      }
    }
    const int xcnt = p.xcnt[t];
    const double xs0 = p.xst[(size_t)t * 4], xs1 = p.xst[(size_t)t * 4 + 1], xs2 = p.xst[(size_t)t * 4 + 2];
    float prob[8], score[8];
    float a1 = -INFINITY, a2 = -INFINITY;                  // this lane's two largest scores
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (live) {
        prob[j] = __fdividef(1.f, 1.f + __expf(-(float)lgd[j]));
        score[j] = prob[j] + bias[j];
      } else {
        prob[j] = 0.f;
        score[j] = -INFINITY;
      }
      a2 = fmaxf(a2, fminf(a1, score[j]));
      a1 = fmaxf(a1, score[j]);
    }
    if (live) {
      prow[0] = make_float4(prob[0], prob[1], prob[2], prob[3]);
      prow[1] = make_float4(prob[4], prob[5], prob[6], prob[7]);
    }
    // the group's two largest: merge the lanes' pairs
    for (int o = 1; o < LG; o <<= 1) {
      const float b1 = __shfl_xor_sync(full, a1, o), b2 = __shfl_xor_sync(full, a2, o);
      a2 = fmaxf(fminf(a1, b1), fmaxf(a2, b2));
      a1 = fmaxf(a1, b1);
    }
    const float gs = a1 + a2;
    // kept groups: rank of this lane's group among the group scores
    const int g = lane / LG;
    int rank = 0;
    for (int h = 0; h < p.n_group; ++h) {
      const float gh = __shfl_sync(full, gs, (h * LG) & 31);
      rank += (gh > gs || (gh == gs && h < g)) ? 1 : 0;
    }
    const bool keep = live && g < p.n_group && rank < p.topk_group;
    // this lane's candidates, sorted: key (score, then the lower expert) in
    // the high word, 7 - j in the low one; absent experts sort last (0)
    unsigned long long c[8];
#pragma unroll
    for (int j = 0; j < 8; ++j)
      c[j] = live ? ((unsigned long long)score_key(keep ? score[j] : -INFINITY) << 32) | (unsigned)(7 - j) : 0ull;
    // Batcher's odd-even merge sort on 8 keys, largest first
    cas_desc(c[0], c[1]); cas_desc(c[2], c[3]); cas_desc(c[4], c[5]); cas_desc(c[6], c[7]);
    cas_desc(c[0], c[2]); cas_desc(c[1], c[3]); cas_desc(c[4], c[6]); cas_desc(c[5], c[7]);
    cas_desc(c[1], c[2]); cas_desc(c[5], c[6]);
    cas_desc(c[0], c[4]); cas_desc(c[1], c[5]); cas_desc(c[2], c[6]); cas_desc(c[3], c[7]);
    cas_desc(c[2], c[4]); cas_desc(c[3], c[5]);
    cas_desc(c[1], c[2]); cas_desc(c[3], c[4]); cas_desc(c[5], c[6]);
    // the k choices (lane r keeps choice r): the largest head, ties to the
    // lower lane (the lower experts); that lane pops it
    int my_e = -1;
    double my_l = 0.0;
    for (int r = 0; r < p.k; ++r) {
      const uint32_t hk = (uint32_t)(c[0] >> 32);
      const uint32_t best = __reduce_max_sync(full, hk);
      const int wl = (int)__reduce_min_sync(full, hk == best ? (uint32_t)lane : 32u);
      const int jw = 7 - (int)__shfl_sync(full, (uint32_t)c[0] & 7u, wl);
      double lv = lgd[0];
#pragma unroll
      for (int j = 1; j < 8; ++j)
        if (jw == j) lv = lgd[j];
      lv = __shfl_sync(full, lv, wl);
      if (lane == r) {
        my_e = 8 * wl + jw;
        my_l = lv;
      }
      if (lane == wl) {
#pragma unroll
        for (int j = 0; j < 7; ++j) c[j] = c[j + 1];
        c[7] = 0ull;
      }
    }
    // the chosen logits with the x-rounding term added where listed; the
    // token is listed for the exact pass when a chosen bound exceeds tau or
    // two chosen keys lie within their bounds of each other
    double bnd = 0.0, key = 0.0, sig = 0.0;
    const bool mine = lane < p.k;
    if (mine) {
      const double *ws = p.wst + (size_t)my_e * 4;
      if (xcnt <= p.round_list) {
        const size_t o = (size_t)t * p.round_list;
        const float *wr = p.w + (size_t)my_e * p.d;
        double corr = 0.0;
        for (int q = 0; q < xcnt; ++q) {
          // (an index outside the row, left by a preparation pass that gave up, adds nothing)
          const int ix = p.xidx[o + q];
          if ((unsigned)ix < (unsigned)p.d) corr = fma(p.xdx[o + q], (double)__ldg(wr + ix), corr);
        }
        my_l += corr;
      } else {
        bnd = xs0 * ws[0];
      }
      bnd += xs1 * ws[1] + xs2 * ws[2];
      sig = 1.0 / (1.0 + exp(-my_l));
      key = sig + (p.bias ? (double)p.bias[my_e] : 0.0);
    }
    bool need = mine && bnd > p.tau;
    for (int j = 0; j < p.k; ++j) {
      const double kj = __shfl_sync(full, key, j), bj = __shfl_sync(full, bnd, j);
      // |key error| <= a quarter of the logit bound
      if (mine && j != lane && fabs(kj - key) <= bj + bnd) need = true;
    }
    if (__any_sync(full, need) && lane == 0) p.flag_list[atomicAdd(p.flag_count, 1)] = t;
    // weights from these logits (replaced by route_finish_listed for a listed
    // token); key = the selection score that orders the slots
    double tot = mine ? sig : 0.0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(full, tot, o);
    const double wout = (p.norm ? sig / (tot + 1e-20) : sig) * p.scaling;
    if (!mine) key = -INFINITY;
    int slot = 0;
    for (int j = 0; j < p.k; ++j) {
      const double kj = __shfl_sync(full, key, j);
      const int ej = __shfl_sync(full, my_e, j);
      if (kj > key || (kj == key && ej < my_e)) ++slot;
    }
    if (mine) {
      p.ids[(size_t)t * p.k + slot] = my_e;
      p.wts[(size_t)t * p.k + slot] = (float)wout;
    }
  }
  // the block's probability sums, tokens added in order
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += 32 * WPB) {
    double sum = 0.0;
    for (int tl = 0; tl < TPB; ++tl) sum += (double)pr[tl * E + e];
    p.part[(size_t)blockIdx.x * E + e] = sum;
  }
}

// Exact re-weighting of the listed tokens (bounded-logit plan): a block per
// token (grid-stride over the list), every thread a share of the hidden
// dimension for eight chosen experts at a time (bf16 x fp32 products exact in
// float64, float64 sums reduced in a fixed order), then warp 0 weights and
// orders the slots from the exact logits as the selection pass would.
constexpr int RL_THREADS = 1024;
__device__ __forceinline__ void refine_listed(const RouteParams &p, int bx, int nbx) {
  __shared__ double red[RL_THREADS / 32][8];
  __shared__ double lsh[32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const unsigned full = 0xffffffffu;
  const int n = *p.flag_count;
  const bool softmax = p.router == MOE_ROUTER_SOFTMAX_TOPK;
  for (int j = bx; j < n; j += nbx) {
    const int t = p.flag_list[j];
    const uint4 *xr = reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(p.x) + (size_t)t * p.d);
    for (int r0 = 0; r0 < p.k; r0 += 8) {
      int ids[8];
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        const int e = r0 + s < p.k ? p.ids[(size_t)t * p.k + r0 + s] : -1;
        ids[s] = e >= 0 && e < p.E ? e : -1;
      }
      double acc[8];
#pragma unroll
      for (int s = 0; s < 8; ++s) acc[s] = 0.0;
      for (int i = threadIdx.x; i < p.d / 8; i += RL_THREADS) {
        const uint4 xv = __ldg(xr + i);
        const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
        double xd[8];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          xd[2 * u] = (double)__uint_as_float(xw[u] << 16);
          xd[2 * u + 1] = (double)__uint_as_float(xw[u] & 0xFFFF0000u);
        }
#pragma unroll
        for (int s = 0; s < 8; ++s)
          if (ids[s] >= 0) {
            const float4 *wr = reinterpret_cast<const float4 *>(p.w + (size_t)ids[s] * p.d) + 2 * i;
            const float4 a = __ldg(wr), b = __ldg(wr + 1);
            acc[s] = fma(xd[0], (double)a.x, acc[s]);
            acc[s] = fma(xd[1], (double)a.y, acc[s]);
            acc[s] = fma(xd[2], (double)a.z, acc[s]);
            acc[s] = fma(xd[3], (double)a.w, acc[s]);
            acc[s] = fma(xd[4], (double)b.x, acc[s]);
            acc[s] = fma(xd[5], (double)b.y, acc[s]);
            acc[s] = fma(xd[6], (double)b.z, acc[s]);
            acc[s] = fma(xd[7], (double)b.w, acc[s]);
          }
      }
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        double v = acc[s];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(full, v, o);
        if (lane == 0) red[warp][s] = v;
      }
      __syncthreads();
      if (threadIdx.x < 8 && r0 + (int)threadIdx.x < p.k) {
        double v = 0.0;
        for (int w = 0; w < RL_THREADS / 32; ++w) v += red[w][threadIdx.x];
        lsh[r0 + threadIdx.x] = v;
      }
      __syncthreads();
    }
    if (warp == 0) {
      int my_e = lane < p.k ? p.ids[(size_t)t * p.k + lane] : -1;
      // a slot is live when its id is in range and not taken by an earlier slot
      bool ok = lane < p.k && my_e >= 0 && my_e < p.E;
      for (int s = 0; s < p.k; ++s) {
        const int es = __shfl_sync(full, my_e, s);
        if (s < lane && es == my_e) ok = false;
      }
      double wv = 0.0, key = -INFINITY;
      if (ok) {
        const double l = lsh[lane];
        const double b = p.bias ? (double)p.bias[my_e] : 0.0;
        if (softmax) {
          wv = l + b;
          key = wv;
        } else {
          wv = 1.0 / (1.0 + exp(-l));
          key = wv + b;
        }
      }
      if (softmax) {
        double m = ok ? wv : -INFINITY;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmax(m, __shfl_xor_sync(full, m, o));
        wv = ok ? exp(wv - m) : 0.0;
      }
      double tot = lane < p.k ? wv : 0.0;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(full, tot, o);
      double wout;
      if (softmax) wout = p.norm ? wv / fmax(tot, 1e-12) : wv;
      else wout = (p.norm ? wv / (tot + 1e-20) : wv) * p.scaling;
      int slot = lane;
      if (!p.forced) {
        slot = 0;
        for (int s = 0; s < p.k; ++s) {
          const double ks = __shfl_sync(full, key, s);
          const int es = __shfl_sync(full, my_e, s);
          if (ks > key || (ks == key && es < my_e)) ++slot;
        }
      }
      __syncwarp();
      if (lane < p.k) {
        p.ids[(size_t)t * p.k + slot] = my_e;
        p.wts[(size_t)t * p.k + slot] = (float)wout;
      }
    }
    __syncthreads();
  }
}

// prob_sum[e] = sum over 32-token groups in a fixed order: a block per 32
// experts; warp w adds groups w, w + 32, w + 64, ... with eight loads in
// flight, then the 32 warp sums are added in warp order.  Deterministic for a
// given T and E.
constexpr int FIN_WARPS = 32;
constexpr int FIN_UNROLL = 16;
__device__ __forceinline__ void finalize_block(const double *part, int nb, int E, float *prob_sum, int bx) {
  __shared__ double ws[FIN_WARPS][32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int e = bx * 32 + lane;
  double s = 0.0;
  if (e < E) {
    for (int b0 = warp; b0 < nb; b0 += FIN_WARPS * FIN_UNROLL) {
      double v[FIN_UNROLL];
#pragma unroll
      for (int u = 0; u < FIN_UNROLL; ++u) {
        const int b = b0 + u * FIN_WARPS;
        v[u] = b < nb ? part[(size_t)b * E + e] : 0.0;
      }
#pragma unroll
      for (int u = 0; u < FIN_UNROLL; ++u) s += v[u];
    }
  }
  ws[warp][lane] = s;
  __syncthreads();
  if (warp == 0 && e < E) {
    double t = 0.0;
#pragma unroll
    for (int w = 0; w < FIN_WARPS; ++w) t += ws[w][lane];
    prob_sum[e] = (float)t;
  }
}

__global__ void __launch_bounds__(32 * FIN_WARPS) route_finalize(const double *part, int nb, int E, float *prob_sum) {
  pdl_enter();
  finalize_block(part, nb, E, prob_sum, blockIdx.x);
}

// The bounded-logit plan's last launch: blocks [0, fin_blocks) add the
// probability-sum rows (route_finalize), the rest re-weight the listed tokens
// exactly (both only read what the selection wrote).
static_assert(RL_THREADS == 32 * FIN_WARPS, "one block shape for both halves");
__global__ void __launch_bounds__(RL_THREADS) route_finish_listed(RouteParams p, const double *part, int nb,
                                                                  float *prob_sum, int fin_blocks) {
  pdl_enter();
  if ((int)blockIdx.x < fin_blocks) finalize_block(part, nb, p.E, prob_sum, blockIdx.x);
  else refine_listed(p, blockIdx.x - fin_blocks, gridDim.x - fin_blocks);
}

template <int EPL, int TPW, bool BF16, bool SPLIT>
cudaError_t launch_tiled(const RouteParams &p, dim3 grid, cudaStream_t s) {
  const size_t stage = sizeof(uint32_t) * 2 * (size_t)TiledShape<EPL, TPW, BF16>::stage_words(p.E);
  const size_t scratch = sizeof(double) * (size_t)WARPS * kMaxExperts;
  const size_t smem = stage > scratch ? stage : scratch;
  auto kern = route_tiled<EPL, TPW, BF16, SPLIT>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  launch_pdl(kern, grid, kRouteThreads, smem, s, p);
  return cudaGetLastError();
}

// The selection pass over float64 logits partials [ks][T][E].
template <int EPL, int TPB, int WPB>
cudaError_t launch_select_tpb(const RouteParams &p, cudaStream_t s) {
  const size_t smem = sizeof(double) * ((size_t)TPB * p.E + (size_t)TPB * kMaxExperts);
  auto sel = route_select<EPL, TPB, WPB>;
  cudaError_t err = cudaFuncSetAttribute(sel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  launch_pdl(sel, (p.T + TPB - 1) / TPB, 32 * WPB, smem, s, p);
  return cudaGetLastError();
}

// 32-token blocks run 16 warps (two tokens each) so that a selecting thread
// keeps up to 128 registers
template <int EPL>
cudaError_t launch_select_epl(const RouteParams &p, cudaStream_t s) {
  return select_tokens_per_block(p.T) == 8 ? launch_select_tpb<EPL, 8, 8>(p, s)
                                           : launch_select_tpb<EPL, 32, 16>(p, s);
}

template <int EPL, bool BF16>
cudaError_t launch_wide(const RouteParams &p, const RoutePlan &plan, cudaStream_t s) {
  if (plan.split) {
    // 8-token tiles x 32-expert slices x hidden-dimension slices
    const dim3 grid((p.T + 7) / 8, plan.ks, (p.E + 31) / 32);
    cudaError_t err = launch_tiled<1, 1, BF16, true>(p, grid, s);
    if (err != cudaSuccess) return err;
    return launch_select_epl<EPL>(p, s);
  }
  if (plan.tpw == 8) return launch_tiled<EPL, 8, BF16, false>(p, dim3((p.T + 63) / 64), s);
  return launch_tiled<EPL, 4, BF16, false>(p, dim3((p.T + 31) / 32), s);
}


template <int EPL, int TPB, int WPB>
cudaError_t launch_refine_tpb(const RouteParams &p, cudaStream_t s) {
  const size_t smem = sizeof(float) * ((size_t)TPB * p.E + (size_t)WPB * p.E);
  auto kern = route_select_refine<EPL, TPB, WPB>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  launch_pdl(kern, (p.T + TPB - 1) / TPB, 32 * WPB, smem, s, p);
  return cudaGetLastError();
}

// tokens per block as the probability-sum rows were sized (select_tokens_per_block)
template <int EPL>
cudaError_t launch_refine_epl(const RouteParams &p, cudaStream_t s) {
  return select_tokens_per_block(p.T) == 8 ? launch_refine_tpb<EPL, 8, 8>(p, s) : launch_refine_tpb<EPL, 32, 8>(p, s);
}

// The lane-per-8-experts selection for sigmoid group routing over bounded logits
bool group8_select(const RouteParams &p) {
  if (!p.approx || p.forced || p.router != MOE_ROUTER_SIGMOID_GROUP || p.E > 256 || p.E % 8 != 0) return false;
  if (p.n_group < 1 || p.E % p.n_group != 0 || (p.E / p.n_group) % 8 != 0) return false;
  const int lg = p.E / p.n_group / 8;
  return (lg & (lg - 1)) == 0 && p.k <= 32;
}

template <int TPB>
cudaError_t launch_group8_tpb(const RouteParams &p, cudaStream_t s) {
  const size_t smem = sizeof(float) * (size_t)TPB * p.E;
  auto kern = route_select_group8<TPB>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  launch_pdl(kern, (p.T + TPB - 1) / TPB, 256, smem, s, p);
  return cudaGetLastError();
}

cudaError_t launch_select(const RouteParams &p, cudaStream_t s) {
  if (group8_select(p))
    return select_tokens_per_block(p.T) == 8 ? launch_group8_tpb<8>(p, s) : launch_group8_tpb<32>(p, s);
  if (p.refine || p.approx) {
    if (p.E <= 32) return launch_refine_epl<1>(p, s);
    if (p.E <= 64) return launch_refine_epl<2>(p, s);
    if (p.E <= 128) return launch_refine_epl<4>(p, s);
    return launch_refine_epl<8>(p, s);
  }
  if (p.E <= 32) return launch_select_epl<1>(p, s);
  if (p.E <= 64) return launch_select_epl<2>(p, s);
  if (p.E <= 128) return launch_select_epl<4>(p, s);
  return launch_select_epl<8>(p, s);
}

template <bool BF16>
cudaError_t launch_any(const RouteParams &p, const RoutePlan &plan, cudaStream_t s) {
  const int nb32 = (p.T + kRouteTokens - 1) / kRouteTokens;
  if (p.E <= 8) {
    launch_pdl(route_rows<8, BF16, 2>, nb32, 32 * 16, 0, s, p);
    return cudaGetLastError();
  }
  if (p.E <= 16) {
    launch_pdl(route_rows<16, BF16, 4>, nb32, 32 * 8, 0, s, p);    // 16 experts x 4 tokens of accumulators
    return cudaGetLastError();
  }
  if (p.E <= 64) return launch_wide<2, BF16>(p, plan, s);
  if (p.E <= 128) return launch_wide<4, BF16>(p, plan, s);
  return launch_wide<8, BF16>(p, plan, s);
}

}  // namespace

// MOE_ROUTER_TC=bf16 keeps the bf16 tensor-core logits with the exact
// re-weighting of every token (read once per process)
static bool bf16_tc_router_requested() {
  static const bool on = [] {
    const char *v = getenv("MOE_ROUTER_TC");
    return v != nullptr && strcmp(v, "bf16") == 0;
  }();
  return on;
}

RoutePlan route_plan(const moe_config &c, bool allow_split) {
  RoutePlan plan{};
  plan.split = false;
  plan.tc = false;
  plan.i8 = false;
  plan.ks = 1;
  plan.kchunk = c.hidden;
  plan.tpw = 4;
  // the weights then depend on the chosen experts' logits alone (renormalised
  // softmax, or sigmoid scores), which the selection pass recomputes exactly
  const bool chosen_only = c.router == MOE_ROUTER_SIGMOID_GROUP || c.norm_topk_prob;
  // (a decode-sized batch is served faster by the split CUDA-core pass)
  if (allow_split && c.act_dtype == MOE_BF16 && chosen_only && c.num_tokens >= 512) {
    if (i8_route_supported(c) && !bf16_tc_router_requested()) {
      plan.i8 = true;
      plan.ks = i8_route_plan(c).ks;
      return plan;
    }
    const TcRoutePlan t = tc_route_plan(c);
    plan.tc = true;
    plan.ks = t.ks;
    return plan;
  }
  if (c.num_experts <= 16) return plan;
  const int sms = 148;
  const int whole_row_blocks = (c.num_tokens + kRouteTokens - 1) / kRouteTokens;
  const bool vec_ok = c.act_dtype == MOE_BF16 ? (c.hidden % 8 == 0) : (c.hidden % 4 == 0);
  if (allow_split && vec_ok && whole_row_blocks < sms) {
    // 8-token tiles x 32-expert slices, then as many hidden-dimension slices
    // (each a multiple of 32 elements, at most 16) as it takes to give every
    // SM four blocks: a block's chain of staged 32-element chunks is what
    // takes the time at these sizes, so shorter slices finish sooner
    const int base = ((c.num_tokens + 7) / 8) * ((c.num_experts + 31) / 32);
    int ks = (4 * sms + base - 1) / base;
    const int max_ks = c.hidden / KC < kMaxSplitSlices ? c.hidden / KC : kMaxSplitSlices;
    ks = ks < max_ks ? ks : max_ks;
    ks = ks < 1 ? 1 : ks;
    int kchunk = (c.hidden + ks - 1) / ks;
    kchunk = (kchunk + KC - 1) / KC * KC;
    plan.ks = (c.hidden + kchunk - 1) / kchunk;
    plan.kchunk = kchunk;
    plan.split = true;
    return plan;
  }
  // 8 tokens per warp halves the shared-memory reads per FMA once the batch
  // still fills every SM with 64-token blocks.
  if (c.num_experts > 64 && (c.num_tokens + 63) / 64 >= sms) plan.tpw = 8;
  return plan;
}

// logits partials, then (tensor-core plan) the split router weight
static size_t tc_logits_part(const moe_config &c, int ks) {
  return align_up(sizeof(double) * (size_t)ks * c.num_tokens * c.num_experts, 256);
}

size_t route_logits_bytes(const moe_config &c) {
  const RoutePlan plan = route_plan(c, true);
  if (plan.i8) return i8_route_bytes(c, i8_route_plan(c));
  if (plan.tc) return tc_logits_part(c, plan.ks) + tc_route_plan(c).wsplit_bytes;
  return plan.split ? sizeof(double) * (size_t)plan.ks * c.num_tokens * c.num_experts : 0;
}

size_t route_logits_f64_bytes(const moe_config &c) {
  const RoutePlan plan = route_plan(c, true);
  return plan.tc || plan.i8 || plan.split ? sizeof(double) * (size_t)plan.ks * c.num_tokens * c.num_experts : 0;
}

cudaError_t launch_route(const moe_config &c, const void *x, const float *w_router,
                         const float *router_bias, int32_t *topk_ids, float *topk_w,
                         double *route_part, float *prob_sum, cudaStream_t s, double *logits,
                         const int32_t *forced_ids, int *status) {
  RouteParams p;
  p.forced = forced_ids;
  p.status = status;
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
  const RoutePlan plan = route_plan(c, logits != nullptr);
  p.refine = plan.tc ? 1 : 0;
  p.approx = 0;
  p.xst = nullptr;
  p.wst = nullptr;
  p.tau = 0.0;
  p.xcnt = nullptr;
  p.xidx = nullptr;
  p.xdx = nullptr;
  p.round_list = 0;
  p.flag_count = nullptr;
  p.flag_list = nullptr;
  p.logits = logits;
  p.ks = plan.ks;
  p.kchunk = plan.kchunk;

  cudaError_t err;
  if (plan.i8) {
    const I8RoutePlan t = i8_route_plan(c);
    const I8RouteBuffers b = i8_route_buffers(c, t, logits);
    p.logits = b.logits;
    p.approx = 1;
    p.xst = b.xst;
    p.wst = b.wst;
    p.xcnt = b.xcnt;
    p.xidx = b.xidx;
    p.xdx = b.xdx;
    p.round_list = b.round_list;
    // a chosen logit within 2.5e-7 moves a renormalised weight by at most
    // about 5e-7 of itself (twice the logit error), inside the 1e-6 bound
    p.tau = 2.5e-7;
    p.flag_count = b.flag_count;
    p.flag_list = b.flag_list;
    err = launch_route_i8_logits(c, x, w_router, t, b, status, s);
    if (err == cudaSuccess) err = launch_select(p, s);
  } else if (plan.tc) {
    __nv_bfloat16 *wsplit =
        reinterpret_cast<__nv_bfloat16 *>(reinterpret_cast<char *>(logits) + tc_logits_part(c, plan.ks));
    err = launch_route_tc_logits(c, x, w_router, wsplit, logits, status, s);
    if (err == cudaSuccess) err = launch_select(p, s);
  } else {
    err = c.act_dtype == MOE_BF16 ? launch_any<true>(p, plan, s) : launch_any<false>(p, plan, s);
  }
  if (err != cudaSuccess) return err;
  // probability-sum rows: one per selection block when route_select ran,
  // else one per 32-token block of the fused router kernels
  const int nb = plan.tc || plan.i8 || plan.split ? (c.num_tokens + select_tokens_per_block(c.num_tokens) - 1) /
                                             select_tokens_per_block(c.num_tokens)
                                       : route_blocks(c);
  const int fin_blocks = (c.num_experts + 31) / 32;
  if (plan.i8) {
    // the listed tokens' exact re-weighting shares the launch
    const int listed_blocks = c.num_tokens < 148 ? c.num_tokens : 148;
    launch_pdl(route_finish_listed, fin_blocks + listed_blocks, RL_THREADS, 0, s, p, (const double *)route_part, nb,
               prob_sum, fin_blocks);
  } else {
    launch_pdl(route_finalize, fin_blocks, 32 * FIN_WARPS, 0, s, route_part, nb, c.num_experts, prob_sum);
  }
  return cudaGetLastError();
}

}  // namespace moe
