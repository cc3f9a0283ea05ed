// Grouped SwiGLU expert FFN with 4-bit affine group-64 weights (decode).
//
// Weight format (Edge0 QuantSpec: bits=4, group_size=64, mode="affine"):
// codes packed 8 per 32-bit word, element j of a row at bits 4*(j%8) of word
// j/8; one bf16 scale s and bias b per 64 consecutive elements of the
// reduction axis; w = s*q + b.  Dequantisation is fused into the dot
// products: codes are read once from HBM, widened in registers and used for
// every token row of the expert.
//
// Decode has few rows per expert (T*k/E ~ 4), so the weight stream is the
// whole cost: one block owns 64 output features of one expert, stages the
// expert's token rows (bf16) in shared memory, and each warp walks its
// features' code rows with 16-byte loads (32 codes per lane per load).
// Phase 1 writes h = silu(x W_gate^T) * (x W_up^T) in bf16, phase 2
// y = h W_down^T.
#include "common.cuh"

namespace moe {
namespace {

constexpr int FEAT = 64;           // output features per block
constexpr int WARPS = 8;
constexpr int MAXR = 8;            // token rows per pass
constexpr int SMEM_ROW_LIMIT = 96 * 1024;

struct Q4Args {
  const int32_t *offsets;
  int E, K, N, rows_cap;
  int w_stride;                    // weight rows from one expert to the next (N, or 2N for stacked gate/up)
  const uint16_t *a;               // activations [rows_cap, K] bf16
  const uint32_t *q0, *q1;         // codes [E, N, K/8] (q1 only for the SwiGLU pair)
  const uint16_t *s0, *s1, *b0, *b1;   // [E, N, K/64] bf16
  uint16_t *out;                   // [rows_cap, N] bf16
  int swiglu;
  int rows_per_pass;
};

__device__ __forceinline__ void dot_row(const uint32_t *codes, const uint16_t *sc, const uint16_t *bi,
                                        const uint16_t *xs, int K, int nr, int lane, float (&acc)[MAXR]) {
  const int nw4 = K / 32;            // uint4 loads per code row (32 codes each)
  for (int w4 = lane; w4 < nw4; w4 += 32) {
    const uint4 c4 = __ldg(reinterpret_cast<const uint4 *>(codes) + w4);
    const int grp = w4 >> 1;         // 64 codes per group = 2 uint4
    const float s = bf16_to_f32(__ldg(sc + grp));
    const float b = bf16_to_f32(__ldg(bi + grp));
    const uint32_t words[4] = {c4.x, c4.y, c4.z, c4.w};
#pragma unroll
    for (int wi = 0; wi < 4; ++wi) {
      float wv[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) wv[j] = fmaf(s, (float)((words[wi] >> (4 * j)) & 0xFu), b);
      const int k0 = w4 * 32 + wi * 8;
#pragma unroll
      for (int r = 0; r < MAXR; ++r) {
        if (r < nr) {
          const uint4 xv = *reinterpret_cast<const uint4 *>(xs + (size_t)r * K + k0);
          const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
          float a = acc[r];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            a = fmaf(wv[2 * j], __uint_as_float(xw[j] << 16), a);
            a = fmaf(wv[2 * j + 1], __uint_as_float(xw[j] & 0xffff0000u), a);
          }
          acc[r] = a;
        }
      }
    }
  }
}

__device__ __forceinline__ float warp_sum_f(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__global__ void __launch_bounds__(WARPS * 32)
q4_gemm(Q4Args a) {
  pdl_enter();
  extern __shared__ __align__(16) unsigned char smem_raw[];
  uint16_t *xs = reinterpret_cast<uint16_t *>(smem_raw);   // [rows_per_pass][K]
  const int e = blockIdx.x;
  const int f0 = blockIdx.y * FEAT;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int r_begin = a.offsets[e], r_end = a.offsets[e + 1];
  r_begin = max(0, min(r_begin, a.rows_cap));
  r_end = max(r_begin, min(r_end, a.rows_cap));
  if (r_end <= r_begin) return;
  const int rpp = a.rows_per_pass;
  for (int rc = r_begin; rc < r_end; rc += rpp) {
    const int nr = min(rpp, r_end - rc);
    // stage the rows (16-byte copies)
    const int v_per_row = a.K / 8;
    for (int i = threadIdx.x; i < nr * v_per_row; i += blockDim.x) {
      const int r = i / v_per_row, c = i % v_per_row;
      reinterpret_cast<uint4 *>(xs)[(size_t)r * v_per_row + c] =
          __ldg(reinterpret_cast<const uint4 *>(a.a + (size_t)(rc + r) * a.K) + c);
    }
    __syncthreads();
    for (int fi = warp; fi < FEAT; fi += WARPS) {
      const int f = f0 + fi;
      if (f >= a.N) break;
      const size_t row = (size_t)e * a.w_stride + f;
      float acc0[MAXR], acc1[MAXR];
#pragma unroll
      for (int r = 0; r < MAXR; ++r) { acc0[r] = 0.f; acc1[r] = 0.f; }
      dot_row(a.q0 + row * (a.K / 8), a.s0 + row * (a.K / 64), a.b0 + row * (a.K / 64), xs, a.K, nr, lane,
              acc0);
      if (a.swiglu)
        dot_row(a.q1 + row * (a.K / 8), a.s1 + row * (a.K / 64), a.b1 + row * (a.K / 64), xs, a.K, nr, lane,
                acc1);
#pragma unroll
      for (int r = 0; r < MAXR; ++r) {
        if (r < nr) {
          const float g = warp_sum_f(acc0[r]);
          float v = g;
          if (a.swiglu) {
            const float u = warp_sum_f(acc1[r]);
            v = g / (1.f + __expf(-g)) * u;
          }
          if (lane == 0) {
            const __nv_bfloat16 hb = __float2bfloat16_rn(v);
            a.out[(size_t)(rc + r) * a.N + f] = *reinterpret_cast<const uint16_t *>(&hb);
          }
        }
      }
    }
    __syncthreads();
  }
}

cudaError_t run_q4(const Q4Args &base, int N, int K, cudaStream_t s) {
  Q4Args a = base;
  a.N = N;
  a.K = K;
  int rpp = SMEM_ROW_LIMIT / (K * 2);
  rpp = rpp < 1 ? 1 : (rpp > MAXR ? MAXR : rpp);
  a.rows_per_pass = rpp;
  const size_t smem = (size_t)rpp * K * 2;
  cudaError_t err = cudaFuncSetAttribute(q4_gemm, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  dim3 grid(a.E, (N + FEAT - 1) / FEAT);
  launch_pdl(q4_gemm, grid, WARPS * 32, smem, s, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_ffn_q4(const FfnArgs &f, cudaStream_t s) {
  Q4Args a{};
  a.offsets = f.offsets;
  a.E = f.E;
  a.rows_cap = f.rows_cap;
  // phase 1: h = silu(x W1^T) * (x W2^T)
  a.a = static_cast<const uint16_t *>(f.x);
  a.q0 = static_cast<const uint32_t *>(f.w1);
  a.q1 = static_cast<const uint32_t *>(f.w2);
  a.s0 = static_cast<const uint16_t *>(f.s1);
  a.s1 = static_cast<const uint16_t *>(f.s2);
  a.b0 = static_cast<const uint16_t *>(f.b1);
  a.b1 = static_cast<const uint16_t *>(f.b2);
  a.out = static_cast<uint16_t *>(f.h);
  a.swiglu = 1;
  a.w_stride = f.w_stride;
  cudaError_t err = run_q4(a, f.F, f.d, s);
  if (err != cudaSuccess) return err;
  if (f.mid_event && (err = cudaEventRecord(f.mid_event, s)) != cudaSuccess) return err;
  // phase 2: y = h W3^T
  a.a = static_cast<const uint16_t *>(f.h);
  a.q0 = static_cast<const uint32_t *>(f.w3);
  a.s0 = static_cast<const uint16_t *>(f.s3);
  a.b0 = static_cast<const uint16_t *>(f.b3);
  a.q1 = nullptr;
  a.s1 = a.b1 = nullptr;
  a.out = static_cast<uint16_t *>(f.y);
  a.swiglu = 0;
  a.w_stride = f.d;
  return run_q4(a, f.d, f.F, s);
}

}  // namespace moe
