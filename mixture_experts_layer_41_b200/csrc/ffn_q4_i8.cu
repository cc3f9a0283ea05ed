// Grouped SwiGLU expert FFN with 4-bit affine group-64 weights for decode
// batches, on 8-bit integer warp-level MMAs.
//
// Weight format (Edge0 QuantSpec: bits=4, group_size=64, mode="affine"):
// element j of a weight row is the nibble at bits 4*(j%8) of 32-bit word j/8;
// w = s*q + b with one bf16 scale s and bias b per 64 consecutive elements of
// the reduction axis.  For a token x the sum over one group g is therefore
//     sum_{k in g} w_k x_k = s_g * sum_{k in g} q_k x_k + b_g * sum_{k in g} x_k,
// so the codes q never need to be turned into floating-point weights: they
// go into the tensor core as unsigned 8-bit integers (one AND, or a shift and
// an AND, per four codes), and s_g and b_g are applied once per group to the
// exact integer sum.
//
// The tokens are turned into integers beforehand (quant_tokens): each
// 128-element block of a token row gets a power-of-two scale that puts its
// largest magnitude just under 2^14, and every element becomes the nearest
// integer v in [-2^14, 2^14), split as v = 128*hi + lo with hi a signed and lo
// an unsigned 7-bit byte.  hi and lo ride in two columns of the MMA's token
// operand, so one mma.sync m16n8k32 (u8 x s8 -> s32, exact) covers 16 weight
// rows x 32 K x 4 tokens, and 128*D[hi] + D[lo] is the exact integer sum.  The
// only rounding besides fp32 accumulation across groups is that of v: at most
// 2^-15 of the block's largest magnitude per element.  The per-group sums of
// v (for the bias term) are kept beside the integers.
//
// MMA operand order.  A thread (group row g = lane/4, c = lane%4) owns weight
// rows g and g+8 of its warp's 16 and, per 128-element K-block, code words
// 2c, 2c+1 of the block's first 64-element group and 8+2c, 9+2c of the
// second, so each MMA (group, j) sums one group only: thread c's word 8*group
// + 2c + j gives A bytes (q0, q2, q4, q6) (the word masked with 0x0F0F0F0F)
// and (q1, q3, q5, q7) (the word shifted right by 4 and masked).  The token
// operand is stored in the same K order: for each row and K-block, 256 bytes
// laid out [group][j][c][hi|lo][4 even elements, 4 odd elements] of word
// 8*group + 2c + j, so a thread's two B registers are one 8-byte load.
//
// Per CTA (8 warps, persistent over (expert, token pass, 128-feature block)
// tasks, two CTAs per SM): the pass's token rows (<= 4*NB_MAX) are copied into
// shared memory, each warp owns 16 features (x2 for the gate/up pair) and
// walks K in 128-element blocks with the codes, scales and biases of the next
// PF blocks in flight in a register ring.  Phase 1 writes
// h = silu(x W_gate^T) * (x W_up^T) in bf16 (row order); phase 2 y = h W_down^T.
#include "common.cuh"

namespace moe {
namespace {

constexpr int WARPS = 8;
constexpr int THREADS = 32 * WARPS;
constexpr int FW = 16;                  // features per warp (MMA M)
constexpr int FB = FW * WARPS;          // features per CTA task
constexpr int KB = 128;                 // K per block: two quantisation groups
constexpr int MIN_CTAS = 2;             // resident CTAs per SM the register budget is set for
constexpr int QMAX = 1 << 14;           // |token integer| < 2^14 (hi fits a signed byte)

struct I8Params {
  const int32_t *offsets;   // [E+1]
  int E;
  int rows_cap;
  int N;                    // output features per expert
  int w_stride;             // weight rows from one expert to the next
  int K;                    // reduction length (multiple of 128)
  int ntok;                 // token rows per pass (4 * NB_MAX)
  const uint8_t *tq;        // quantised tokens [rows_cap][K/128][256]
  const float *tscale;      // [rows_cap][K/128]: the block's value of one integer step
  const float *tsum;        // [rows_cap][K/64]: per-group sums of the integers
  const uint32_t *q[2];     // codes [.., K/8] (gate / up, or down)
  const uint16_t *sc[2];    // scales [.., K/64] bf16
  const uint16_t *bi[2];    // biases, same layout
  uint16_t *out;            // [rows_cap, N] bf16
  int *status;
};

__device__ __forceinline__ void mma_u8s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint2 ldg_stream8(const void *p) {
  uint2 v;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
  return v;
}
__device__ __forceinline__ float silu_f(float g) { return g / (1.f + __expf(-g)); }
// asynchronous global -> shared copies; valid == false writes zeros
__device__ __forceinline__ void cp_async16(void *smem, const void *gmem, bool valid) {
  const uint32_t s = (uint32_t)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(s), "l"(gmem), "r"(valid ? 16 : 0) : "memory");
}
__device__ __forceinline__ void cp_async4(void *smem, const void *gmem, bool valid) {
  const uint32_t s = (uint32_t)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(s), "l"(gmem), "r"(valid ? 4 : 0) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// ---------------------------------------------------------------- token quantisation
// One warp per (row, 128-element block); lane l holds elements 4l..4l+3.
__global__ void __launch_bounds__(256)
quant_tokens(const uint16_t *a, int rows, int K, uint8_t *tq, float *tscale, float *tsum) {
  pdl_enter();
  const int lane = threadIdx.x & 31;
  const int nkb = K / KB;
  const long long item = (long long)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  if (item >= (long long)rows * nkb) return;
  const int r = (int)(item / nkb), b = (int)(item % nkb);
  const uint2 raw = *reinterpret_cast<const uint2 *>(a + (size_t)r * K + (size_t)b * KB + 4 * lane);
  const float x[4] = {bf16_lo(raw.x), bf16_hi(raw.x), bf16_lo(raw.y), bf16_hi(raw.y)};
  float m = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  // m < 2^e: one integer step is 2^(e - 14), so |v| <= 2^14 before the clamp
  int e = 0;
  if (m > 0.f) frexpf(m, &e);
  const float up = m > 0.f ? ldexpf(1.f, 14 - e) : 0.f;
  int v[4], s = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[i] = __float2int_rn(x[i] * up);
    v[i] = max(-QMAX, min(QMAX - 1, v[i]));
    s += v[i];
  }
  // group sums: lanes 0-15 hold the block's first group, 16-31 the second
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  // lanes l and l^1 hold the two halves of code word l/2: the even lane
  // writes its 16 bytes [hi even, hi odd, lo even, lo odd]
  int w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) w[i] = __shfl_xor_sync(0xffffffffu, v[i], 1);
  if ((lane & 1) == 0) {
    int el[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      el[i] = v[i];
      el[4 + i] = w[i];
    }
    uint32_t hi_e = 0, hi_o = 0, lo_e = 0, lo_o = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int ve = el[2 * i], vo = el[2 * i + 1];
      hi_e |= (uint32_t)((ve >> 7) & 0xFF) << (8 * i);
      hi_o |= (uint32_t)((vo >> 7) & 0xFF) << (8 * i);
      lo_e |= (uint32_t)(ve & 0x7F) << (8 * i);
      lo_o |= (uint32_t)(vo & 0x7F) << (8 * i);
    }
    const int word = lane >> 1;                 // 0..15 within the block
    const int grp = word >> 3, t = word & 7, c = t >> 1, j = t & 1;
    uint8_t *dst = tq + ((size_t)r * nkb + b) * 256 + ((grp * 2 + j) * 4 + c) * 16;
    *reinterpret_cast<uint4 *>(dst) = make_uint4(hi_e, hi_o, lo_e, lo_o);
  }
  if (lane == 0) {
    tscale[(size_t)r * nkb + b] = m > 0.f ? ldexpf(1.f, e - 14) : 0.f;
    tsum[(size_t)r * 2 * nkb + 2 * b] = (float)s;
  }
  if (lane == 16) tsum[(size_t)r * 2 * nkb + 2 * b + 1] = (float)s;
}

// ---------------------------------------------------------------- grouped GEMM
// One K-block of one matrix for this thread: rows g and g + 8, code words
// 2c, 2c+1 (first group) and 8+2c, 9+2c (second group), and the scale and
// bias words that hold the block's two groups.
struct Frag {
  uint2 g0_lo, g1_lo, g0_hi, g1_hi;   // [group][row g | g+8]
  uint32_t s_lo, s_hi, b_lo, b_hi;
};

__device__ __forceinline__ void load_frag(Frag &f, const uint32_t *q_lo, size_t qrow, const uint16_t *s_lo,
                                          const uint16_t *b_lo, size_t srow, int blk, int c) {
  const uint32_t *p0 = q_lo + blk * (KB / 8) + 2 * c;
  f.g0_lo = ldg_stream8(p0);
  f.g1_lo = ldg_stream8(p0 + 8);
  f.g0_hi = ldg_stream8(p0 + 8 * qrow);
  f.g1_hi = ldg_stream8(p0 + 8 * qrow + 8);
  f.s_lo = __ldg(reinterpret_cast<const uint32_t *>(s_lo + 2 * blk));
  f.s_hi = __ldg(reinterpret_cast<const uint32_t *>(s_lo + 8 * srow + 2 * blk));
  f.b_lo = __ldg(reinterpret_cast<const uint32_t *>(b_lo + 2 * blk));
  f.b_hi = __ldg(reinterpret_cast<const uint32_t *>(b_lo + 8 * srow + 2 * blk));
}

struct TaskPos {
  int e, fb, row0, nrows;
};

__device__ __forceinline__ TaskPos decode_task(const int32_t *off, const int32_t *task_start, int E, int fblocks,
                                               int ntok, int task) {
  int lo = 0, hi = E;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (task_start[mid] <= task) lo = mid; else hi = mid;
  }
  TaskPos t;
  t.e = lo;
  const int local = task - task_start[lo];
  t.fb = local % fblocks;
  t.row0 = off[lo] + (local / fblocks) * ntok;
  t.nrows = min(ntok, off[lo + 1] - t.row0);
  return t;
}

template <int MATS, int NB_MAX, int PF>
__global__ void __launch_bounds__(THREADS, MIN_CTAS)
q4_i8_gemm(const I8Params p) {
  pdl_wait();
  extern __shared__ __align__(16) uint8_t smem_raw[];
  constexpr int NT = 4 * NB_MAX;
  int32_t *off = reinterpret_cast<int32_t *>(smem_raw);              // [E+1]
  int32_t *task_start = off + (p.E + 1);                              // [E+1]
  const int hdr = ((2 * (p.E + 1) * 4 + 127) / 128) * 128;
  const int nkb = p.K / KB;
  float *ts_s = reinterpret_cast<float *>(smem_raw + hdr);            // [NT][nkb]
  float *sum_s = ts_s + NT * nkb;                                     // [NT][2 nkb]
  const int row_bytes = p.K * 2 + 64;                                 // == 64 mod 128: conflict-free B loads
  uint8_t *xs = smem_raw + hdr + ((NT * nkb * 3 * 4 + 127) / 128) * 128;   // [NT][row_bytes]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, c = lane & 3;
  const int fblocks = p.N / FB;
  const size_t qrow = (size_t)p.K / 8, srow = (size_t)p.K / 64;

  if (warp == 0) {
    const int ntok = p.ntok;
    const bool bad = warp_group_offsets(p.offsets, p.E, 0, p.rows_cap, off, task_start,
                                        [ntok, fblocks](int cnt) { return ((cnt + ntok - 1) / ntok) * fblocks; });
    if (bad && lane == 0 && blockIdx.x == 0) record_status(p.status, kDevBadOffsets);
  }
  __syncthreads();
  const int total = task_start[p.E];

  for (int task = blockIdx.x; task < total; task += gridDim.x) {
    const TaskPos t = decode_task(off, task_start, p.E, fblocks, p.ntok, task);
    const int nb = (t.nrows + 3) >> 2;
    const int f0 = t.fb * FB + warp * FW;
    const size_t wrow = (size_t)t.e * p.w_stride + f0 + g;           // this thread's first weight row

    // the first K-blocks of this warp's rows are on their way while the tokens are staged
    Frag buf[PF + 1][MATS];
#pragma unroll
    for (int r = 0; r < PF; ++r)
      if (r < nkb) {
#pragma unroll
        for (int m = 0; m < MATS; ++m)
          load_frag(buf[r][m], p.q[m] + wrow * qrow, qrow, p.sc[m] + wrow * srow, p.bi[m] + wrow * srow, srow, r,
                    c);
      }

    // stage the pass's quantised token rows, their block scales and group
    // sums with asynchronous copies, all in flight together (zeros past the
    // last row: a copy of 0 source bytes fills its destination with zeros)
    __syncthreads();                                    // the previous task's readers are done
    {
      const int chunks = p.K * 2 / 16;                  // 16-byte chunks per row
      const int n = nb * 4 * chunks;
      for (int i = tid; i < n; i += THREADS) {
        const int r = i / chunks, q16 = i - r * chunks;
        const bool live = r < t.nrows;
        const uint8_t *src = p.tq + (size_t)(live ? t.row0 + r : 0) * p.K * 2 + q16 * 16;
        cp_async16(xs + (size_t)r * row_bytes + q16 * 16, src, live);
      }
      // the rows' block scales (nkb per row) and group sums (2 nkb per row):
      // 4-byte copies, scales first, then sums
      const int m = nb * 4 * nkb;
      for (int i = tid; i < 3 * m; i += THREADS) {
        if (i < m) {
          const int r = i / nkb;
          const bool live = r < t.nrows;
          cp_async4(ts_s + i, p.tscale + (size_t)(live ? t.row0 + r : 0) * nkb + (i - r * nkb), live);
        } else {
          const int j = i - m, r = j / (2 * nkb);
          const bool live = r < t.nrows;
          cp_async4(sum_s + j, p.tsum + (size_t)(live ? t.row0 + r : 0) * 2 * nkb + (j - r * 2 * nkb), live);
        }
      }
      cp_async_wait_all();
    }
    __syncthreads();

    // y[m][n][0 | 1] = this thread's (feature g | g + 8, token 4n + c), in units of the tokens' steps
    float acc[MATS][NB_MAX][2];
#pragma unroll
    for (int m = 0; m < MATS; ++m)
#pragma unroll
      for (int n = 0; n < NB_MAX; ++n) acc[m][n][0] = acc[m][n][1] = 0.f;
    // B operand: token 4n + (lane/4)/2, hi/lo column (lane/4)%2, word slot c
    const uint8_t *xb = xs + (size_t)(g >> 1) * row_bytes + (g & 1) * 8 + c * 16;

#pragma unroll 1
    for (int blk0 = 0; blk0 < nkb; blk0 += PF + 1) {
#pragma unroll
      for (int r = 0; r <= PF; ++r) {                   // slot r holds block blk0 + r
        const int blk = blk0 + r;
        if (blk >= nkb) break;
        if (blk + PF < nkb) {
#pragma unroll
          for (int m = 0; m < MATS; ++m)
            load_frag(buf[(r + PF) % (PF + 1)][m], p.q[m] + wrow * qrow, qrow, p.sc[m] + wrow * srow,
                      p.bi[m] + wrow * srow, srow, blk + PF, c);
        }
        const Frag *cur = buf[r];
#pragma unroll
        for (int grp = 0; grp < 2; ++grp) {
          // this group's token operand for every 4-token block, both MMAs (j = 0, 1)
          uint2 bv[NB_MAX][2];
          float gs[NB_MAX], st[NB_MAX];
#pragma unroll
          for (int n = 0; n < NB_MAX; ++n)
            if (n < nb) {
              const uint8_t *base = xb + (size_t)n * 4 * row_bytes + blk * 256 + grp * 128;
              bv[n][0] = *reinterpret_cast<const uint2 *>(base);
              bv[n][1] = *reinterpret_cast<const uint2 *>(base + 64);
              const int tok = 4 * n + c;
              st[n] = ts_s[tok * nkb + blk];
              gs[n] = sum_s[(tok * nkb + blk) * 2 + grp];
            }
#pragma unroll
          for (int m = 0; m < MATS; ++m) {
            const uint2 wl = grp == 0 ? cur[m].g0_lo : cur[m].g1_lo;
            const uint2 wh = grp == 0 ? cur[m].g0_hi : cur[m].g1_hi;
            const float s_lo = grp == 0 ? bf16_lo(cur[m].s_lo) : bf16_hi(cur[m].s_lo);
            const float s_hi = grp == 0 ? bf16_lo(cur[m].s_hi) : bf16_hi(cur[m].s_hi);
            const float b_lo = grp == 0 ? bf16_lo(cur[m].b_lo) : bf16_hi(cur[m].b_lo);
            const float b_hi = grp == 0 ? bf16_lo(cur[m].b_hi) : bf16_hi(cur[m].b_hi);
            // A for j = 0 (word 2c) and j = 1 (word 2c + 1): even and odd codes
            const uint32_t a0j0 = wl.x & 0x0F0F0F0Fu, a2j0 = (wl.x >> 4) & 0x0F0F0F0Fu;
            const uint32_t a1j0 = wh.x & 0x0F0F0F0Fu, a3j0 = (wh.x >> 4) & 0x0F0F0F0Fu;
            const uint32_t a0j1 = wl.y & 0x0F0F0F0Fu, a2j1 = (wl.y >> 4) & 0x0F0F0F0Fu;
            const uint32_t a1j1 = wh.y & 0x0F0F0F0Fu, a3j1 = (wh.y >> 4) & 0x0F0F0F0Fu;
#pragma unroll
            for (int n = 0; n < NB_MAX; ++n)
              if (n < nb) {
                int d[4] = {0, 0, 0, 0};
                mma_u8s8(d, a0j0, a1j0, a2j0, a3j0, bv[n][0].x, bv[n][0].y);
                mma_u8s8(d, a0j1, a1j1, a2j1, a3j1, bv[n][1].x, bv[n][1].y);
                // d = D[feature g | g + 8][token c hi | lo]: the exact integer sums
                const float v_lo = (float)(d[0] * 128 + d[1]);
                const float v_hi = (float)(d[2] * 128 + d[3]);
                acc[m][n][0] = fmaf(st[n], fmaf(s_lo, v_lo, b_lo * gs[n]), acc[m][n][0]);
                acc[m][n][1] = fmaf(st[n], fmaf(s_hi, v_hi, b_hi * gs[n]), acc[m][n][1]);
              }
          }
        }
      }
    }

    // epilogue: acc[.][n][i] = (feature f0 + g + 8i, token 4n + c)
#pragma unroll
    for (int n = 0; n < NB_MAX; ++n) {
      if (n >= nb) break;
      const int tok = 4 * n + c;
      if (tok < t.nrows) {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          float v = acc[0][n][i];
          if (MATS == 2) v = silu_f(v) * acc[MATS - 1][n][i];
          const __nv_bfloat16 hb = __float2bfloat16_rn(v);
          p.out[(size_t)(t.row0 + tok) * p.N + f0 + g + 8 * i] = *reinterpret_cast<const uint16_t *>(&hb);
        }
      }
    }
  }
  pdl_trigger();                         // tasks done: the next kernel may be scheduled
}

int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

// shared memory of one CTA: offsets header, token scales and sums, token tile
size_t smem_bytes(int E, int ntok, int K) {
  const size_t hdr = ((2 * (size_t)(E + 1) * 4 + 127) / 128) * 128;
  const size_t meta = (((size_t)ntok * (K / KB) * 3 * 4 + 127) / 128) * 128;
  return hdr + meta + (size_t)ntok * ((size_t)K * 2 + 64);
}

cudaError_t quantise(const void *tokens, int rows, int K, uint8_t *tq, float *tscale, float *tsum, cudaStream_t s) {
  const long long items = (long long)rows * (K / KB);
  if (items == 0) return cudaSuccess;
  const int blocks = (int)((items + 7) / 8);
  launch_pdl(quant_tokens, blocks, 256, 0, s, static_cast<const uint16_t *>(tokens), rows, K, tq, tscale, tsum);
  return cudaGetLastError();
}

template <int MATS, int NB_MAX, int PF>
cudaError_t run(const FfnArgs &a, int K, int N, int w_stride, const void *q0, const void *q1, const void *s0,
                const void *s1, const void *b0, const void *b1, void *out, cudaStream_t s) {
  I8Params p;
  p.offsets = a.offsets;
  p.E = a.E;
  p.rows_cap = a.rows_cap;
  p.N = N;
  p.w_stride = w_stride;
  p.K = K;
  p.ntok = 4 * NB_MAX;
  p.tq = static_cast<const uint8_t *>(a.q4_tokens);
  p.tscale = a.q4_tscale;
  p.tsum = a.q4_tsum;
  p.q[0] = static_cast<const uint32_t *>(q0);
  p.q[1] = static_cast<const uint32_t *>(MATS == 2 ? q1 : q0);
  p.sc[0] = static_cast<const uint16_t *>(s0);
  p.sc[1] = static_cast<const uint16_t *>(MATS == 2 ? s1 : s0);
  p.bi[0] = static_cast<const uint16_t *>(b0);
  p.bi[1] = static_cast<const uint16_t *>(MATS == 2 ? b1 : b0);
  p.out = static_cast<uint16_t *>(out);
  p.status = a.status;
  const size_t smem = smem_bytes(a.E, p.ntok, K);
  auto kern = q4_i8_gemm<MATS, NB_MAX, PF>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, THREADS, smem) != cudaSuccess || per_sm < 1) {
    cudaGetLastError();
    per_sm = 1;
  }
  const long long upper = ((long long)(a.rows_cap + p.ntok - 1) / p.ntok + a.E) * (N / FB);
  const int slots = per_sm * sm_count();
  const int grid = (int)(upper < slots ? upper : slots);
  launch_plain(kern, grid, THREADS, smem, s, p);
  return cudaGetLastError();
}

}  // namespace

bool q4_i8_supported(int d, int F) {
  if (d % FB != 0 || F % FB != 0 || d % KB != 0 || F % KB != 0) return false;
  // the token tile of a pass (8 rows of d in phase 1, 16 rows of F in phase 2) in shared memory
  return smem_bytes(kMaxExperts, 8, d) <= 227 * 1024 && smem_bytes(kMaxExperts, 16, F) <= 227 * 1024;
}

size_t q4_i8_token_bytes(int rows, int d, int F) {
  const size_t K = (size_t)(d > F ? d : F);
  return (size_t)rows * (K * 2 + (K / KB) * 4 + (K / 64) * 4) + 512;
}

cudaError_t launch_ffn_q4_i8(const FfnArgs &a, cudaStream_t s) {
  // the token buffer is reused: phase 1's tokens are read before h is quantised into it
  FfnArgs b = a;
  const int K1 = a.d, K2 = a.F;
  const int Kmax = K1 > K2 ? K1 : K2;
  uint8_t *tq = static_cast<uint8_t *>(a.q4_scratch);
  float *tscale = reinterpret_cast<float *>(tq + (((size_t)a.rows_cap * Kmax * 2 + 255) / 256) * 256);
  float *tsum = tscale + (size_t)a.rows_cap * (Kmax / KB);
  b.q4_tokens = tq;
  b.q4_tscale = tscale;
  b.q4_tsum = tsum;
  const int rows = a.rows_cap;
  cudaError_t err = quantise(a.x, rows, K1, tq, tscale, tsum, s);
  if (err == cudaSuccess)
    err = run<2, 2, 2>(b, K1, a.F, a.w_stride, a.w1, a.w2, a.s1, a.s2, a.b1, a.b2, a.h, s);
  if (err != cudaSuccess) return err;
  if (a.mid_event && (err = cudaEventRecord(a.mid_event, s)) != cudaSuccess) return err;
  err = quantise(a.h, rows, K2, tq, tscale, tsum, s);
  if (err != cudaSuccess) return err;
  return run<1, 4, 3>(b, K2, a.d, a.d, a.w3, nullptr, a.s3, nullptr, a.b3, nullptr, a.y, s);
}

}  // namespace moe
