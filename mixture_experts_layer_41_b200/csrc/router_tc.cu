// Router logits for expert SELECTION on the tensor cores.
//
// The gate of the "Mixture of Experts" blog (route / Router.route) and of
// Edge0 "MoE Spec and Routing" is an fp32 linear map x W_r^T.  For bf16 tokens
// it runs here as two bf16 tcgen05 GEMMs: every fp32 weight w is split into
// w = hi + lo + r, hi = bf16(w) and lo = bf16(w - hi) carrying the top 16 bits
// of its significand, and a bf16 token times a bf16 slice is exact.  The
// dropped residual |r| <= 2^-17 |w| moves a logit at d = 7168 by about 1e-5
// (rms 8e-6 for the workloads' N(0, 0.02) weights), and the tensor core's own
// sums, flushed into float64 registers every FLUSH K-blocks (an fp32
// accumulator left running over thousands of products drifts much further),
// add about 1e-6: selection-grade logits, far inside the 1e-4 selection margin
// and the 1e-5 prob-sum bound.  The routing weights need 1e-6 relative, so the
// selection pass recomputes the k chosen logits of every token exactly
// (float64 products and sums) before weighting.
//
// Grid: (128-token tile, NTE-expert tile, hidden slice).  Per CTA:
//   warp 0      TMA producer: per K-block the token tile (128 x 64 bf16) and
//               the two weight-slice tiles (NTE x 64 bf16), 128-byte swizzle;
//   warp 1      TMEM owner and single-thread MMA issuer (kind::f16, M = 128,
//               N = NTE, K = 16), fp32 accumulators double-buffered per flush;
//   warps 2-9   epilogue: two warps per TMEM lane quarter, each half the expert
//               columns in float64 registers; the slice's sums go to
//               logits[slice][token][expert].
// The selection pass then adds the slices in order (route_select).  Every
// mbarrier wait is bounded by %globaltimer (2 s unless moe_set_wait_timeout_ns says otherwise); on expiry the CTA records a
// status, drains its own copies and MMAs, frees TMEM and exits.
#include "common.cuh"

#include <cuda.h>
#include <cudaTypedefs.h>

namespace moe {
namespace {

constexpr int TM = 128;                 // tokens per tile (MMA M)
constexpr int BK = 64;                  // K per block
constexpr int STAGES = 4;
constexpr int NSPLIT = 2;               // bf16 slices of the fp32 router weight
constexpr int FLUSH = 2;                // K-blocks per fp32 accumulation before the float64 add
constexpr int EPI_WARPS = 8;
constexpr int THREADS = 32 * (2 + EPI_WARPS);
constexpr uint64_t DRAIN_NS = 200000000ull;

template <int NTE>
struct TcShape {
  static constexpr int A_BYTES = TM * BK * 2;            // 16 KiB token tile
  static constexpr int B_BYTES = NTE * BK * 2;           // one weight slice tile
  static constexpr int STAGE_BYTES = A_BYTES + NSPLIT * B_BYTES;
  static constexpr int CPW = NTE / 2;                    // expert columns per epilogue warp
  static constexpr uint32_t TMEM_COLS = 2 * NTE < 32 ? 32 : 2 * NTE;   // two accumulators
  // kind::f16: D fp32, A/B bf16, both K-major, N = NTE, M = 128
  static constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(NTE >> 3) << 17) |
                                    ((uint32_t)(TM >> 4) << 24);
};

struct TcRouteParams {
  uint64_t timeout_ns;        // bound on every barrier wait (moe_set_wait_timeout_ns)
  int T, E, d;
  int e_pad;            // weight-slice rows per slice (E rounded up to the expert tile)
  int kb_total;         // K-blocks of the hidden dimension
  int kb_per_slice;
  double *logits;       // [ks][T][E]
  int *status;
};

struct TcShared {
  uint64_t full[STAGES], empty[STAGES];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

// ---------------------------------------------------------------- PTX wrappers
__device__ __forceinline__ uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ bool wait_bounded(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                             int *status, int code, uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  uint32_t spins = 0;
  while (!mbar_try_wait(bar, parity)) {
    if (*abort_flag) return false;
    // the clock is read every 32 polls, or every poll under a limit below 1 us
    if (((++spins & 31u) == 0 || limit_ns < 1000u) && global_ns() - t0 > limit_ns) {
      *abort_flag = 1;
      record_status(status, code);
      return false;
    }
  }
  return true;
}
__device__ __forceinline__ bool wait_drain(uint64_t *bar, uint32_t parity) {
  const uint64_t t0 = global_ns();
  while (!mbar_try_wait(bar, parity))
    if (global_ns() - t0 > DRAIN_NS) return false;
  return true;
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, uint32_t bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
          dst),
      "l"((uint64_t)map), "r"(bar), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_commit(uint64_t *bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accum));
}
// K-major tile written by TMA with the 128-byte swizzle (8-row groups 1024
// bytes apart); +2 in the address field moves K by 16 bf16.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// 32 lanes x N consecutive 32-bit TMEM columns
template <int N>
__device__ __forceinline__ void tmem_ld(uint32_t taddr, uint32_t (&v)[N]);
template <>
__device__ __forceinline__ void tmem_ld<8>(uint32_t taddr, uint32_t (&v)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7])
               : "r"(taddr));
}
template <>
__device__ __forceinline__ void tmem_ld<16>(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr));
}
template <>
__device__ __forceinline__ void tmem_ld<32>(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]),
        "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]),
        "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]),
        "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// ---------------------------------------------------------------- weight split
// w (fp32) -> hi, mid, lo (bf16, round to nearest even each) with
// hi = bf16(w), lo = bf16(w - hi) (the residual is exact in fp32).  Rows
// E..e_pad-1 are 0.  Layout [NSPLIT][e_pad][d].
__global__ void split_router_weights(const float *__restrict__ w, int E, int e_pad, int d,
                                     __nv_bfloat16 *__restrict__ out) {
  pdl_enter();
  const size_t n = (size_t)e_pad * d;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    const int e = (int)(i / d);
    const float v = e < E ? w[i] : 0.f;
    const __nv_bfloat16 hi = __float2bfloat16_rn(v);
    out[i] = hi;
    out[n + i] = __float2bfloat16_rn(v - __bfloat162float(hi));
  }
}

// ---------------------------------------------------------------- the GEMM
template <int NTE>
__global__ void __launch_bounds__(THREADS, 1)
route_tc_gemm(const __grid_constant__ CUtensorMap mapX, const __grid_constant__ CUtensorMap mapW,
              const TcRouteParams p) {
  pdl_enter();
  using S = TcShape<NTE>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t *tiles = smem_raw + pad;
  TcShared *st = reinterpret_cast<TcShared *>(tiles + (size_t)STAGES * S::STAGE_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = blockIdx.x * TM, e0 = blockIdx.y * NTE, slice = blockIdx.z;
  const int kb0 = slice * p.kb_per_slice;
  const int kb_n = max(0, min(p.kb_per_slice, p.kb_total - kb0));

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&st->full[s], 1);
      mbar_init(&st->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&st->acc_full[b], 1);
      mbar_init(&st->acc_empty[b], EPI_WARPS);
    }
    mbar_init(&st->drain, 1);
    st->abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&st->tmem_base)),
                 "r"(S::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = st->tmem_base;
  volatile int *abort_flag = &st->abort_flag;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (; it < kb_n; ++it) {
        const int s = it % STAGES;
        if (!wait_bounded(&st->empty[s], ((it / STAGES) & 1) ^ 1, abort_flag, p.status, kDevTimeoutProducer, p.timeout_ns)) {
          ok = false;
          break;
        }
        uint8_t *sp = tiles + (size_t)s * S::STAGE_BYTES;
        const uint32_t fb = smem_u32(&st->full[s]);
        const int kx = (kb0 + it) * BK;
        mbar_expect_tx(&st->full[s], S::STAGE_BYTES);
        tma_load_2d(smem_u32(sp), &mapX, fb, kx, t0);
#pragma unroll
        for (int part = 0; part < NSPLIT; ++part)
          tma_load_2d(smem_u32(sp + S::A_BYTES + part * S::B_BYTES), &mapW, fb, kx, part * p.e_pad + e0);
      }
      if (!ok) {
        const int first = it > STAGES ? it - STAGES : 0;
        for (int i = first; i < it; ++i)
          if (!wait_drain(&st->full[i % STAGES], (i / STAGES) & 1)) record_status(p.status, kDevTimeoutDrain);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = true;
      for (int it = 0; it < kb_n && ok; ++it) {
        const int chunk = it / FLUSH, first = it % FLUSH == 0;
        const uint32_t buf = chunk & 1, use = chunk >> 1;
        if (first && !wait_bounded(&st->acc_empty[buf], (use & 1) ^ 1, abort_flag, p.status, kDevTimeoutMma, p.timeout_ns)) {
          ok = false;
          break;
        }
        const int s = it % STAGES;
        if (!wait_bounded(&st->full[s], (it / STAGES) & 1, abort_flag, p.status, kDevTimeoutMma, p.timeout_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sa = smem_u32(tiles + (size_t)s * S::STAGE_BYTES);
        const uint64_t da = sw128_desc(sa);
        const uint32_t dt = tmem_base + buf * NTE;
#pragma unroll
        for (int part = 0; part < NSPLIT; ++part) {
          const uint64_t db = sw128_desc(sa + S::A_BYTES + part * S::B_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            tc_mma(dt, da + (uint64_t)(kk * 2), db + (uint64_t)(kk * 2), S::IDESC,
                   (!first || part || kk) ? 1u : 0u);
        }
        tc_commit(&st->empty[s]);
        if (it % FLUSH == FLUSH - 1 || it == kb_n - 1) tc_commit(&st->acc_full[buf]);
      }
      tc_commit(&st->drain);
      if (!wait_drain(&st->drain, 0u)) record_status(p.status, kDevTimeoutDrain);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                        // TMEM lane quarter
    const int half = (warp - 2) >> 2;              // which half of the expert columns
    const int col0 = half * S::CPW;
    constexpr int PIECE = S::CPW < 32 ? S::CPW : 32;
    double acc[S::CPW];
#pragma unroll
    for (int c = 0; c < S::CPW; ++c) acc[c] = 0.0;
    bool ok = true;
    const int n_chunks = (kb_n + FLUSH - 1) / FLUSH;
    for (int chunk = 0; chunk < n_chunks; ++chunk) {
      const uint32_t buf = chunk & 1, use = chunk >> 1;
      if (!wait_bounded(&st->acc_full[buf], use & 1, abort_flag, p.status, kDevTimeoutEpilogue, p.timeout_ns)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t v[S::CPW];
#pragma unroll
      for (int c0 = 0; c0 < S::CPW; c0 += PIECE)
        tmem_ld<PIECE>(tmem_base + ((uint32_t)(q * 32) << 16) + buf * NTE + col0 + c0,
                       *reinterpret_cast<uint32_t(*)[PIECE]>(&v[c0]));
      tmem_wait_ld();
      // the accumulator is in registers: hand it back before the float64 adds
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&st->acc_empty[buf]);
#pragma unroll
      for (int c = 0; c < S::CPW; ++c) acc[c] += (double)__uint_as_float(v[c]);
    }
    const int t = t0 + q * 32 + lane;
    if (ok && t < p.T) {
      double *row = p.logits + ((size_t)slice * p.T + t) * p.E;
#pragma unroll
      for (int c = 0; c < S::CPW; ++c) {
        const int e = e0 + col0 + c;
        if (e < p.E) row[e] = acc[c];
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(S::TMEM_COLS)
                 : "memory");
  }
}

// ---------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// Row-major bf16 [rows, k], box 64 x box_rows, 128-byte swizzle, zero fill.
cudaError_t make_map(CUtensorMap *m, const void *ptr, uint64_t k, uint64_t rows, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  cuuint64_t dims[2] = {k, rows};
  cuuint64_t strides[1] = {k * 2};
  cuuint32_t box[2] = {(cuuint32_t)BK, box_rows};
  cuuint32_t es[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int NTE>
cudaError_t run_tc(const moe_config &c, const void *x, const __nv_bfloat16 *wsplit, int e_pad, int ks,
                   int kb_per_slice, double *logits, int *status, cudaStream_t s) {
  using S = TcShape<NTE>;
  CUtensorMap mx, mw;
  cudaError_t err = make_map(&mx, x, (uint64_t)c.hidden, (uint64_t)c.num_tokens, TM);
  if (err == cudaSuccess) err = make_map(&mw, wsplit, (uint64_t)c.hidden, (uint64_t)NSPLIT * e_pad, NTE);
  if (err != cudaSuccess) return err;
  TcRouteParams p;
  p.T = c.num_tokens;
  p.E = c.num_experts;
  p.d = c.hidden;
  p.e_pad = e_pad;
  p.kb_total = (c.hidden + BK - 1) / BK;
  p.kb_per_slice = kb_per_slice;
  p.logits = logits;
  p.status = status;
  p.timeout_ns = wait_timeout_ns();
  const size_t smem = 1024 + (size_t)STAGES * S::STAGE_BYTES + sizeof(TcShared);
  auto kern = route_tc_gemm<NTE>;
  err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  const dim3 grid((c.num_tokens + TM - 1) / TM, e_pad / NTE, ks);
  launch_pdl(kern, grid, THREADS, smem, s, mx, mw, p);
  return cudaGetLastError();
}

}  // namespace

TcRoutePlan tc_route_plan(const moe_config &c) {
  TcRoutePlan t{};
  // wide expert tiles keep the MMAs at the full bf16 rate (N >= 128)
  t.nte = c.num_experts > 64 ? 128 : (c.num_experts > 32 ? 64 : (c.num_experts > 16 ? 32 : 16));
  t.e_pad = (c.num_experts + t.nte - 1) / t.nte * t.nte;
  const int kb_total = (c.hidden + BK - 1) / BK;
  const long long tiles = (long long)((c.num_tokens + TM - 1) / TM) * (t.e_pad / t.nte);
  // hidden slices until the grid covers about two waves of the 148 SMs, each
  // slice at least 4 K-blocks
  int ks = (int)((2 * 148 + tiles - 1) / tiles);
  const int max_ks = kb_total / 4 > 1 ? kb_total / 4 : 1;
  ks = ks < 1 ? 1 : (ks > max_ks ? max_ks : ks);
  t.kb_per_slice = (kb_total + ks - 1) / ks;
  t.ks = (kb_total + t.kb_per_slice - 1) / t.kb_per_slice;   // no empty slice
  t.wsplit_bytes = sizeof(__nv_bfloat16) * NSPLIT * (size_t)t.e_pad * c.hidden;
  return t;
}

cudaError_t launch_route_tc_logits(const moe_config &c, const void *x, const float *w_router,
                                   __nv_bfloat16 *wsplit, double *logits, int *status, cudaStream_t s) {
  const TcRoutePlan t = tc_route_plan(c);
  const size_t n = (size_t)t.e_pad * c.hidden;
  const int blocks = (int)((n + 255) / 256 < 1184 ? (n + 255) / 256 : 1184);
  launch_pdl(split_router_weights, blocks, 256, 0, s, w_router, c.num_experts, t.e_pad, c.hidden, wsplit);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  switch (t.nte) {
    case 16: return run_tc<16>(c, x, wsplit, t.e_pad, t.ks, t.kb_per_slice, logits, status, s);
    case 32: return run_tc<32>(c, x, wsplit, t.e_pad, t.ks, t.kb_per_slice, logits, status, s);
    case 64: return run_tc<64>(c, x, wsplit, t.e_pad, t.ks, t.kb_per_slice, logits, status, s);
    default: return run_tc<128>(c, x, wsplit, t.e_pad, t.ks, t.kb_per_slice, logits, status, s);
  }
}

}  // namespace moe
