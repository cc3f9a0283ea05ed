// Combine: out[t] = sum_j w[t,j] * y_perm[slot_row[t,j]] (+ shared[t]).
//
// The "Mixture of Experts" blog scales each expert output by its router
// weight and scatter-adds it into the token's row (moe_layer; moe_forward's
// np.add.at, a token appearing once per kept slot).  Here the same sum is a
// gather: a block per token (and per slice of the row when there are too
// few tokens to fill the GPU) reads its k rows in slot order, accumulates in
// fp32 and rounds once, so the result is deterministic and needs no atomics.
// Each thread moves 16 bytes per row per step (8 bf16 or 4 fp32 elements),
// with the loads of four slots in flight together.
#include "common.cuh"

namespace moe {
namespace {

constexpr int kThreads = 128;

template <bool BF16>
__global__ void __launch_bounds__(kThreads)
combine_kernel(const void *y_perm, const int32_t *slot_row, const float *topk_w,
               const void *shared_out, void *out, int k, int d) {
  pdl_enter();
  const int t = blockIdx.x;
  __shared__ int rows[kMaxTopK];
  __shared__ float wts[kMaxTopK];
  if (threadIdx.x < k) {
    rows[threadIdx.x] = slot_row[(size_t)t * k + threadIdx.x];
    wts[threadIdx.x] = topk_w[(size_t)t * k + threadIdx.x];
  }
  __syncthreads();
  constexpr int V = BF16 ? 8 : 4;     // elements per 16-byte vector
  const bool vec = (d % V) == 0;
  if (vec) {
    const int nv = d / V;
    for (int c = blockIdx.y * kThreads + threadIdx.x; c < nv; c += gridDim.y * kThreads) {
      float acc[V];
#pragma unroll
      for (int q = 0; q < V; ++q) acc[q] = 0.f;
      for (int j0 = 0; j0 < k; j0 += 4) {
        uint4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int j = j0 + u;
          if (j < k && rows[j] >= 0) v[u] = __ldg(reinterpret_cast<const uint4 *>(y_perm) + (size_t)rows[j] * nv + c);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int j = j0 + u;
          if (j >= k || rows[j] < 0) continue;
          const float w = wts[j];
          if (BF16) {
            const uint32_t h[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              acc[2 * q] = fmaf(w, __uint_as_float(h[q] << 16), acc[2 * q]);
              acc[2 * q + 1] = fmaf(w, __uint_as_float(h[q] & 0xffff0000u), acc[2 * q + 1]);
            }
          } else {
            acc[0] = fmaf(w, __uint_as_float(v[u].x), acc[0]);
            acc[1] = fmaf(w, __uint_as_float(v[u].y), acc[1]);
            acc[2] = fmaf(w, __uint_as_float(v[u].z), acc[2]);
            acc[3] = fmaf(w, __uint_as_float(v[u].w), acc[3]);
          }
        }
      }
      if (shared_out) {
        const uint4 v = __ldg(reinterpret_cast<const uint4 *>(shared_out) + (size_t)t * nv + c);
        if (BF16) {
          const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            acc[2 * q] += __uint_as_float(u[q] << 16);
            acc[2 * q + 1] += __uint_as_float(u[q] & 0xffff0000u);
          }
        } else {
          acc[0] += __uint_as_float(v.x);
          acc[1] += __uint_as_float(v.y);
          acc[2] += __uint_as_float(v.z);
          acc[3] += __uint_as_float(v.w);
        }
      }
      uint4 o;
      if (BF16) {
        o.x = pack_bf16x2(acc[0], acc[1]);
        o.y = pack_bf16x2(acc[2], acc[3]);
        o.z = pack_bf16x2(acc[4], acc[5]);
        o.w = pack_bf16x2(acc[6], acc[7]);
      } else {
        o.x = __float_as_uint(acc[0]);
        o.y = __float_as_uint(acc[1]);
        o.z = __float_as_uint(acc[2]);
        o.w = __float_as_uint(acc[3]);
      }
      reinterpret_cast<uint4 *>(out)[(size_t)t * nv + c] = o;
    }
  } else {
    for (int c = blockIdx.y * kThreads + threadIdx.x; c < d; c += gridDim.y * kThreads) {
      float acc = 0.f;
      for (int j = 0; j < k; ++j) {
        const int r = rows[j];
        if (r < 0) continue;
        const float yv = BF16 ? bf16_to_f32(reinterpret_cast<const uint16_t *>(y_perm)[(size_t)r * d + c])
                              : reinterpret_cast<const float *>(y_perm)[(size_t)r * d + c];
        acc = fmaf(wts[j], yv, acc);
      }
      if (shared_out)
        acc += BF16 ? bf16_to_f32(reinterpret_cast<const uint16_t *>(shared_out)[(size_t)t * d + c])
                    : reinterpret_cast<const float *>(shared_out)[(size_t)t * d + c];
      if (BF16)
        reinterpret_cast<__nv_bfloat16 *>(out)[(size_t)t * d + c] = __float2bfloat16_rn(acc);
      else
        reinterpret_cast<float *>(out)[(size_t)t * d + c] = acc;
    }
  }
}

}  // namespace

cudaError_t launch_combine(const moe_config &c, const void *y_perm, const int32_t *slot_row,
                           const float *topk_w, const void *shared_out, void *out,
                           cudaStream_t s) {
  // slices of a row per token: enough blocks for two per SM, at most one
  // slice per kThreads vectors of the row
  const int V = c.act_dtype == MOE_BF16 ? 8 : 4;
  const int per_row = (c.hidden % V == 0 ? c.hidden / V : c.hidden);
  const int max_split = (per_row + kThreads - 1) / kThreads;
  int split = (2 * 148 + c.num_tokens - 1) / c.num_tokens;
  split = split < max_split ? split : max_split;
  split = split < 1 ? 1 : split;
  const dim3 grid(c.num_tokens, split);
  if (c.act_dtype == MOE_BF16)
    launch_pdl(combine_kernel<true>, grid, kThreads, 0, s, y_perm, slot_row, topk_w, shared_out, out, c.top_k,
               c.hidden);
  else
    launch_pdl(combine_kernel<false>, grid, kThreads, 0, s, y_perm, slot_row, topk_w, shared_out, out, c.top_k,
               c.hidden);
  return cudaGetLastError();
}

}  // namespace moe
