// Grouped SwiGLU expert FFN with 4-bit affine group-64 weights for decode
// batches: dequantisation straight into warp-level tensor-core fragments.
//
// Weight format (Edge0 QuantSpec: bits=4, group_size=64, mode="affine"):
// element j of a weight row is the nibble at bits 4*(j%8) of 32-bit word j/8;
// w = s*q + b with one bf16 scale s and bias b per 64 consecutive elements of
// the reduction axis.
//
// Decode gives each expert a handful of token rows (T*k/E ~ 4), so the layer
// is a stream of 4-bit weights with a few dot products per weight.  The
// product is run swapped, D[feature, token] = sum_k W[feature, k] x[token, k],
// as mma.sync m16n8k16 (bf16 in, fp32 accumulate): 16 weight rows are the A
// operand and 8 tokens the B operand.  Each thread loads its own codes from
// global memory and dequantises them in registers directly into the A
// fragment layout (the 0x4300 magic makes 128 + q an exact bf16, one
// subtraction and one bf16x2 FMA give s*q + b with a single rounding), so
// no weight byte passes through shared or tensor memory and nothing waits
// on a commit.  N = 8 wastes little when an expert holds ~4 tokens, where the
// 128 x N tcgen05 tiles of the other 4-bit kernel spend a 32-wide token
// operand on them.
//
// Operand K order.  A thread of a quad (c = lane % 4) loads 16 bytes of a
// weight row per 128-element block: code words 4c..4c+3.  Nibble pair i of
// word u, (q_{8w+i}, q_{8w+i+4}) with w = 4c + u, feeds A register slot
// t = i % 2 of MMA step 2u + i / 2.  Sums over K do not depend on the order,
// so the token tile is stored in shared memory in the same order: for token
// n, block b, the pairs (x_{8w+i}, x_{8w+i+4}) of word w sit at 32-bit word
// 16u + 4c + i of the block, and one 16-byte load hands a thread its B
// registers for two MMA steps.
//
// Per CTA (8 warps, persistent over (expert, token pass, 128-feature block)
// tasks): the pass's token rows (<= NB_MAX * 8) are staged once in shared
// memory, each warp owns 16 features (x2 for the gate/up pair) and walks K
// in 128-element blocks with the codes and scales of the next PF blocks in
// flight into a register ring (PF = 2 for gate + up, 3 for down, two CTAs
// per SM; L2 bulk prefetches and a per-thread cp.async ring in shared memory
// were measured slower).  A pass covers 8 tokens in phase 1 and 16 in phase
// 2 (decode experts hold ~4); an expert with more takes further passes.
// Phase 1 writes h = silu(x W_gate^T) * (x W_up^T) in bf16 (row order),
// phase 2 y = h W_down^T.
#include "common.cuh"

namespace moe {
namespace {

constexpr int WARPS = 8;
constexpr int THREADS = 32 * WARPS;
constexpr int FW = 16;                  // features per warp (MMA M)
constexpr int FB = FW * WARPS;          // features per CTA task
constexpr int KB = 128;                 // K per block: 16 bytes of codes per quad thread
constexpr int MIN_CTAS = 2;             // resident CTAs per SM the register budget is set for

struct MmaQ4Params {
  const int32_t *offsets;   // [E+1]
  int E;
  int rows_cap;
  int N;                    // output features per expert
  int w_stride;             // weight rows from one expert to the next
  int K;                    // reduction length (multiple of 128)
  int ntok;                 // token rows per pass (8 * NB_MAX)
  const uint16_t *a;        // tokens [rows_cap, K] bf16
  const uint32_t *q[2];     // codes [.., K/8] (gate / up, or down)
  const uint16_t *sc[2];    // scales [.., K/64] bf16
  const uint16_t *bi[2];    // biases, same layout
  uint16_t *out;            // [rows_cap, N] bf16
  int *status;
};

__device__ __forceinline__ uint32_t bf2_sub(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t bf2_fma(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}
// nibble pair i of a code word -> bf16x2 (s*q_i + b, s*q_{i+4} + b)
__device__ __forceinline__ uint32_t deq_pair(uint32_t w, int i, uint32_t s2, uint32_t b2) {
  const uint32_t magic = 0x43004300u;   // bf16 128.0 in both halves
  const uint32_t v = ((w >> (4 * i)) & 0x000F000Fu) | magic;
  return bf2_fma(bf2_sub(v, magic), s2, b2);
}
__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint4 ldg_stream(const void *p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}
__device__ __forceinline__ float silu_f(float g) { return g / (1.f + __expf(-g)); }

// one K-block of one matrix for this thread: rows g and g + 8 of the warp's
// 16, code words 4c..4c+3 of the block, and the scale / bias words that hold
// the block's two groups
struct Frag {
  uint4 lo, hi;
  uint32_t s_lo, s_hi, b_lo, b_hi;
};

__device__ __forceinline__ void load_frag(Frag &f, const uint32_t *q_lo, size_t qrow, const uint16_t *s_lo,
                                          const uint16_t *b_lo, size_t srow, int blk, int c) {
  f.lo = ldg_stream(q_lo + blk * (KB / 8) + 4 * c);
  f.hi = ldg_stream(q_lo + 8 * qrow + blk * (KB / 8) + 4 * c);
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
q4_mma_gemm(const MmaQ4Params p) {
  pdl_wait();
  extern __shared__ __align__(16) uint8_t smem_raw[];
  int32_t *off = reinterpret_cast<int32_t *>(smem_raw);              // [E+1]
  int32_t *task_start = off + (p.E + 1);                              // [E+1]
  const int hdr = ((2 * (p.E + 1) * 4 + 127) / 128) * 128;
  uint8_t *xs = smem_raw + hdr;                                       // [ntok][row_bytes]
  const int row_bytes = p.K * 2 + 64;                                 // == 64 mod 128: conflict-free B loads
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, c = lane & 3;
  const int fblocks = p.N / FB;
  const int nblk = p.K / KB;
  const size_t qrow = (size_t)p.K / 8, srow = (size_t)p.K / 64;

  if (warp == 0) {
    const int ntok = p.ntok;
    const bool bad = warp_group_offsets(p.offsets, p.E, 0, p.rows_cap, off, task_start,
                                        [ntok, fblocks](int cnt) { return ((cnt + ntok - 1) / ntok) * fblocks; });
    if (bad && lane == 0 && blockIdx.x == 0) record_status(p.status, kDevBadOffsets);
  }
  __syncthreads();
  const int total = task_start[p.E];
  const uint32_t sel = (c >> 1) ? 0x3232u : 0x1010u;   // this thread's group of a block's two

  for (int task = blockIdx.x; task < total; task += gridDim.x) {
    const TaskPos t = decode_task(off, task_start, p.E, fblocks, p.ntok, task);
    const int nb = (t.nrows + 7) >> 3;
    const int f0 = t.fb * FB + warp * FW;
    const size_t wrow = (size_t)t.e * p.w_stride + f0 + g;           // this thread's first weight row

    // the first K-block of this warp's rows is on its way while the tokens are staged
    // register ring of PF + 1 K-blocks: PF blocks in flight ahead of the one in use
    Frag buf[PF + 1][MATS];
#pragma unroll
    for (int r = 0; r < PF; ++r)
      if (r < nblk) {
#pragma unroll
        for (int m = 0; m < MATS; ++m)
          load_frag(buf[r][m], p.q[m] + wrow * qrow, qrow, p.sc[m] + wrow * srow, p.bi[m] + wrow * srow, srow, r,
                    c);
      }

    // stage the pass's tokens in the operand K order (zero rows past the end)
    __syncthreads();                                    // the previous task's readers are done
    {
      const int chunks = p.K / 8;                       // 16-byte chunks per row
      const int n = nb * 8 * chunks;
      constexpr int BATCH = 4;                          // loads in flight per thread
      for (int base = tid; base < n; base += BATCH * THREADS) {
        uint4 v[BATCH];
#pragma unroll
        for (int k = 0; k < BATCH; ++k) {
          const int i = base + k * THREADS;
          const int r = i / chunks, w_all = i - r * chunks;
          v[k] = make_uint4(0u, 0u, 0u, 0u);
          if (i < n && r < t.nrows)
            v[k] = __ldg(reinterpret_cast<const uint4 *>(p.a + (size_t)(t.row0 + r) * p.K) + w_all);
        }
#pragma unroll
        for (int k = 0; k < BATCH; ++k) {
          const int i = base + k * THREADS;
          if (i < n) {
            const int r = i / chunks, w_all = i - r * chunks;
            const int blk = w_all >> 4, w = w_all & 15;   // code word w = 4c' + u of the block
            const uint4 o = make_uint4(prmt(v[k].x, v[k].z, 0x5410), prmt(v[k].x, v[k].z, 0x7632),
                                       prmt(v[k].y, v[k].w, 0x5410), prmt(v[k].y, v[k].w, 0x7632));
            *reinterpret_cast<uint4 *>(xs + (size_t)r * row_bytes + blk * 256 + (w & 3) * 64 + (w >> 2) * 16) = o;
          }
        }
      }
    }
    __syncthreads();

    float acc[MATS][NB_MAX][4];
#pragma unroll
    for (int m = 0; m < MATS; ++m)
#pragma unroll
      for (int n = 0; n < NB_MAX; ++n)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[m][n][j] = 0.f;
    const uint8_t *xb = xs + (size_t)g * row_bytes + c * 16;

#pragma unroll 1
    for (int blk0 = 0; blk0 < nblk; blk0 += PF + 1) {
#pragma unroll
      for (int r = 0; r <= PF; ++r) {                   // slot r holds block blk0 + r
        const int blk = blk0 + r;
        if (blk >= nblk) break;
        if (blk + PF < nblk) {
#pragma unroll
          for (int m = 0; m < MATS; ++m)
            load_frag(buf[(r + PF) % (PF + 1)][m], p.q[m] + wrow * qrow, qrow, p.sc[m] + wrow * srow,
                      p.bi[m] + wrow * srow, srow, blk + PF, c);
        }
        const Frag *cur = buf[r];
        uint32_t s2lo[MATS], s2hi[MATS], b2lo[MATS], b2hi[MATS];
#pragma unroll
        for (int m = 0; m < MATS; ++m) {
          s2lo[m] = prmt(cur[m].s_lo, 0u, sel);
          s2hi[m] = prmt(cur[m].s_hi, 0u, sel);
          b2lo[m] = prmt(cur[m].b_lo, 0u, sel);
          b2hi[m] = prmt(cur[m].b_hi, 0u, sel);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          // B registers of steps 2u and 2u+1 for every 8-token block
          uint4 bv[NB_MAX];
#pragma unroll
          for (int n = 0; n < NB_MAX; ++n)
            if (n < nb)
              bv[n] = *reinterpret_cast<const uint4 *>(xb + (size_t)n * 8 * row_bytes + blk * 256 + u * 64);
#pragma unroll
          for (int hs = 0; hs < 2; ++hs) {
#pragma unroll
            for (int m = 0; m < MATS; ++m) {
              const uint32_t wl = u == 0 ? cur[m].lo.x : u == 1 ? cur[m].lo.y : u == 2 ? cur[m].lo.z : cur[m].lo.w;
              const uint32_t wh = u == 0 ? cur[m].hi.x : u == 1 ? cur[m].hi.y : u == 2 ? cur[m].hi.z : cur[m].hi.w;
              const uint32_t a0 = deq_pair(wl, 2 * hs, s2lo[m], b2lo[m]);
              const uint32_t a1 = deq_pair(wh, 2 * hs, s2hi[m], b2hi[m]);
              const uint32_t a2 = deq_pair(wl, 2 * hs + 1, s2lo[m], b2lo[m]);
              const uint32_t a3 = deq_pair(wh, 2 * hs + 1, s2hi[m], b2hi[m]);
#pragma unroll
              for (int n = 0; n < NB_MAX; ++n)
                if (n < nb) {
                  const uint32_t b0 = hs == 0 ? bv[n].x : bv[n].z;
                  const uint32_t b1 = hs == 0 ? bv[n].y : bv[n].w;
                  mma_bf16(acc[m][n], a0, a1, a2, a3, b0, b1);
                }
            }
          }
        }
      }
    }

    // epilogue: acc[.][n] = D[feature g | g + 8][token 8n + 2c | 8n + 2c + 1]
#pragma unroll
    for (int n = 0; n < NB_MAX; ++n) {
      if (n >= nb) break;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int tok = 8 * n + 2 * c + (j & 1);
        const int feat = f0 + g + (j >> 1) * 8;
        if (tok < t.nrows) {
          float v = acc[0][n][j];
          if (MATS == 2) v = silu_f(v) * acc[MATS - 1][n][j];
          const __nv_bfloat16 hb = __float2bfloat16_rn(v);
          p.out[(size_t)(t.row0 + tok) * p.N + feat] = *reinterpret_cast<const uint16_t *>(&hb);
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

// shared memory of one CTA: offsets header and token tile
size_t smem_bytes(int E, int ntok, int K) {
  const size_t hdr = ((2 * (size_t)(E + 1) * 4 + 127) / 128) * 128;
  return hdr + (size_t)ntok * ((size_t)K * 2 + 64);
}

template <int MATS, int NB_MAX, int PF>
cudaError_t run(const FfnArgs &a, const void *tokens, int K, int N, int w_stride, const void *q0, const void *q1,
                const void *s0, const void *s1, const void *b0, const void *b1, void *out, cudaStream_t s) {
  MmaQ4Params p;
  p.offsets = a.offsets;
  p.E = a.E;
  p.rows_cap = a.rows_cap;
  p.N = N;
  p.w_stride = w_stride;
  p.K = K;
  p.ntok = 8 * NB_MAX;
  p.a = static_cast<const uint16_t *>(tokens);
  p.q[0] = static_cast<const uint32_t *>(q0);
  p.q[1] = static_cast<const uint32_t *>(MATS == 2 ? q1 : q0);
  p.sc[0] = static_cast<const uint16_t *>(s0);
  p.sc[1] = static_cast<const uint16_t *>(MATS == 2 ? s1 : s0);
  p.bi[0] = static_cast<const uint16_t *>(b0);
  p.bi[1] = static_cast<const uint16_t *>(MATS == 2 ? b1 : b0);
  p.out = static_cast<uint16_t *>(out);
  p.status = a.status;
  const size_t smem = smem_bytes(a.E, p.ntok, K);
  auto kern = q4_mma_gemm<MATS, NB_MAX, PF>;
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

bool q4_mma_supported(int d, int F) {
  if (d % FB != 0 || F % FB != 0 || d % KB != 0 || F % KB != 0) return false;
  // the token tile of a pass (8 rows of d in phase 1, 16 rows of F in phase 2) in shared memory
  return smem_bytes(kMaxExperts, 8, d) <= 227 * 1024 && smem_bytes(kMaxExperts, 16, F) <= 227 * 1024;
}

cudaError_t launch_ffn_q4_mma(const FfnArgs &a, cudaStream_t s) {
  cudaError_t err = run<2, 1, 2>(a, a.x, a.d, a.F, a.w_stride, a.w1, a.w2, a.s1, a.s2, a.b1, a.b2, a.h, s);
  if (err != cudaSuccess) return err;
  if (a.mid_event && (err = cudaEventRecord(a.mid_event, s)) != cudaSuccess) return err;
  return run<1, 2, 3>(a, a.h, a.F, a.d, a.d, a.w3, nullptr, a.s3, nullptr, a.b3, nullptr, a.y, s);
}

}  // namespace moe
