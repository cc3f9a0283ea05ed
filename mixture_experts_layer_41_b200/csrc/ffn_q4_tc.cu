// Grouped SwiGLU expert FFN with 4-bit affine group-64 weights on the
// tensor cores (decode shapes).
//
// Weight format (Edge0 QuantSpec: bits=4, group_size=64, mode="affine"):
// element j of a weight row is the nibble at bits 4*(j%8) of 32-bit word j/8;
// w = s*q + b with one bf16 scale s and bias b per 64 consecutive elements of
// the reduction axis.  A K-block of 64 is exactly one quantisation group.
//
// Decode gives each expert a handful of token rows, so the product is run
// "swapped": D[feature, token] = sum_k W[feature, k] x[token, k] with the
// weights as the M = 128 operand and up to 32 tokens as N.  Per CTA
// (persistent over (expert, 32-token pass, 128-feature tile) tiles):
//   warp 0      TMA producer: per K-block the raw code tiles (128 rows x 32
//               bytes, one per matrix) and the token tile (32 rows x 64 bf16,
//               128-byte swizzle) into a stage; per tile the tile's scale and
//               bias rows (contiguous in [E, N, K/64]) by bulk copy.
//   warp 1      TMEM owner and single-thread tcgen05.mma issuer
//               (kind::f16, M=128, N=32, K=16) with the weight operand read
//               from TMEM and the token operand from shared memory; its
//               commits hand the operand slots back.
//   warps 2-17  dequantisers, in groups of 4 x (matrices) warps taking K-blocks
//               round robin: read a stage's codes and token chunks into
//               registers and release the stage at once, dequantise (nibble
//               -> exact bf16 through the 0x4300 magic, one bf16x2 FMA with
//               the group's scale and bias: a single rounding of s*q + b) and
//               write the weight operand straight into a TMEM slot
//               (tcgen05.st; thread = weight row = TMEM lane) and the token
//               tile into that slot's shared buffer.
//   warps 18-21 epilogue, one per TMEM lane quarter: SwiGLU of the gate and
//               up accumulators into h, or a plain store of y.
// Accumulators are double-buffered, so MMA and dequantisation stream across
// tile boundaries while the epilogue drains the previous tile.  The operand
// slots (6 with gate+up, 14 with one matrix) fill the rest of TMEM, so the
// dequantisers run many K-blocks ahead of the MMA and the per-K-block
// commit-to-reuse round trip stays hidden.
// Inside every 8-element chunk both operands use the K order 0,4,1,5,2,6,3,7
// (what the nibble extraction yields without byte permutes): phase 1
// reorders its token tile in shared memory, and writes h already in that
// order for phase 2.  Sums over K do not depend on the order.
// Every mbarrier wait is bounded by %globaltimer (2 s unless moe_set_wait_timeout_ns says otherwise) as in the bf16
// grouped GEMM: on expiry the CTA records a status, drains its own TMA/MMA
// work, frees TMEM and exits.
#include "common.cuh"

#include <cuda.h>
#include <cudaTypedefs.h>

namespace moe {
namespace {

constexpr int BM = 128;                 // weight rows (features) per tile
constexpr int BK = 64;                  // K per block = one quantisation group
constexpr int NT = 32;                  // tokens per pass (MMA N)
constexpr int DQ_WARPS = 16;
constexpr int EPI_WARPS = 4;            // one per TMEM lane quarter
constexpr int THREADS = 32 * (2 + DQ_WARPS + EPI_WARPS);
constexpr int CODE_BYTES = BM * BK / 2; // 4 KiB of codes per matrix per K-block
constexpr int B_BYTES = NT * BK * 2;    // 4 KiB token tile per K-block
constexpr uint64_t DRAIN_NS = 200000000ull;

// kind::f16: D fp32, A/B bf16, K-major, N = 32, M = 128
constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(NT >> 3) << 17) |
                           ((uint32_t)(BM >> 4) << 24);

template <bool PAIR>
struct Q4Shape {
  static constexpr int MATS = PAIR ? 2 : 1;
  static constexpr int STAGES = PAIR ? 8 : 12;
  static constexpr int STAGE_BYTES = MATS * CODE_BYTES + B_BYTES;   // multiple of 1024
  static constexpr int ACC_COLS = MATS * NT;                        // fp32 accumulators of one tile
  static constexpr int A_COLS = MATS * BK / 2;                      // one K-block of bf16 pairs per matrix
  static constexpr int SLOTS = (512 - 2 * ACC_COLS) / A_COLS;       // operand slots in TMEM
  static constexpr int WARPS_PER_KB = 4 * MATS;                     // one warp per (matrix, lane quarter)
  static constexpr int GROUPS = DQ_WARPS / WARPS_PER_KB;            // K-blocks in flight in dequant
};

struct Q4Params {
  uint64_t timeout_ns;        // bound on every barrier wait (moe_set_wait_timeout_ns)
  const int32_t *offsets;   // [E+1]
  int E;
  int rows_cap;
  int N;                    // weight rows per expert (output features)
  int w_stride;             // rows from one expert's block to the next (N, or 2N for stacked gate/up)
  int K;                    // reduction length
  int kgroups;              // K / 64
  const uint16_t *sc[2];    // [E, N, K/64] bf16 scales (gate / up, or down)
  const uint16_t *bi[2];    // biases, same layout
  uint16_t *out;            // [rows_cap, N] bf16
  int *status;
};

struct Q4Shared {
  uint64_t full[12], empty[12];
  uint64_t a_full[16], a_empty[16];
  uint64_t sc_full[2], sc_empty[2];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  int32_t off[kMaxExperts + 1];
  int32_t tile_start[kMaxExperts + 1];
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
__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"((uint64_t)src), "r"(bytes), "r"(bar)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_commit(uint64_t *bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// shared-memory accesses by 32-bit shared addresses
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}
__device__ __forceinline__ void sts128(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}
__device__ __forceinline__ uint32_t lds16(uint32_t addr) {
  unsigned short v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
      "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]),
      "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]),
      "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
// D (TMEM) += A (TMEM, M x 16, rows in lanes) * B (shared memory descriptor)
__device__ __forceinline__ void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %3, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %4, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(accum), "r"(IDESC));
}

// bf16x2 arithmetic (one rounding per lane)
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

// Eight 4-bit codes (element j at bits 4j) -> eight bf16 s*q + b.
// (w >> 4i) & 0x000F000F | 0x43004300 is the bf16 pair (128 + q_i, 128 + q_{i+4});
// subtracting 128 is exact, so each element is rounded once, in the FMA.
// The chunk keeps that pairing: its 16 bytes hold elements in the order
// 0,4,1,5,2,6,3,7 (the operand K order used throughout this kernel; the
// token operand is stored in the same order, see permute_chunk).
__device__ __forceinline__ uint4 dequant8(uint32_t w, uint32_t s2, uint32_t b2) {
  const uint32_t magic = 0x43004300u;   // bf16 128.0 in both halves
  uint32_t p[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t v = ((w >> (4 * i)) & 0x000F000Fu) | magic;
    p[i] = bf2_fma(bf2_sub(v, magic), s2, b2);      // (q_i, q_{i+4})
  }
  return make_uint4(p[0], p[1], p[2], p[3]);
}

// Eight consecutive bf16 (e0..e7) -> the order e0,e4,e1,e5,e2,e6,e3,e7.
__device__ __forceinline__ uint4 permute_chunk(uint4 c) {
  return make_uint4(prmt(c.x, c.z, 0x5410), prmt(c.x, c.z, 0x7632), prmt(c.y, c.w, 0x5410),
                    prmt(c.y, c.w, 0x7632));
}

// Position of logical element L (0..7) of an 8-element chunk in that order.
__device__ __forceinline__ int chunk_pos(int L) { return L < 4 ? 2 * L : 2 * L - 7; }

struct Tile {
  int e, row0, rows, m;
};

__device__ __forceinline__ Tile decode_tile(const Q4Shared *st, int nE, int m_tiles, int tile) {
  int lo = 0, hi = nE;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (st->tile_start[mid] <= tile) lo = mid; else hi = mid;
  }
  Tile t;
  t.e = lo;
  const int local = tile - st->tile_start[lo];
  t.m = local % m_tiles;
  const int pass = local / m_tiles;
  t.row0 = st->off[lo] + pass * NT;
  t.rows = min(NT, st->off[lo + 1] - t.row0);
  return t;
}

template <bool PAIR>
__global__ void __launch_bounds__(THREADS, 1)
q4_tc_gemm(const __grid_constant__ CUtensorMap mapC0, const __grid_constant__ CUtensorMap mapC1,
           const __grid_constant__ CUtensorMap mapB, const Q4Params p) {
  pdl_wait();
  using S = Q4Shape<PAIR>;
  constexpr int MATS = S::MATS, STAGES = S::STAGES, SLOTS = S::SLOTS, GROUPS = S::GROUPS;
  constexpr int WPK = S::WARPS_PER_KB;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t *base = smem_raw + pad;
  uint8_t *stages = base;                                            // STAGES x [codes(MATS) | tokens]
  uint8_t *bslots = stages + (size_t)STAGES * S::STAGE_BYTES;       // SLOTS x token tile (operand K order)
  uint16_t *sbuf = reinterpret_cast<uint16_t *>(bslots + (size_t)SLOTS * B_BYTES);   // 2 x MATS x {scale, bias}
  const int sc_elems = BM * p.kgroups;                               // per matrix per kind
  Q4Shared *st = reinterpret_cast<Q4Shared *>(sbuf + 2 * MATS * 2 * sc_elems + 64);   // +128 bytes
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nE = p.E;
  const int m_tiles = p.N / BM;
  const int kb_n = p.kgroups;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&st->full[s], 1);
      mbar_init(&st->empty[s], WPK);         // the warps that dequantise that K-block
    }
    for (int j = 0; j < SLOTS; ++j) {
      mbar_init(&st->a_full[j], WPK);
      mbar_init(&st->a_empty[j], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&st->sc_full[b], 1);
      mbar_init(&st->sc_empty[b], DQ_WARPS);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&st->acc_full[b], 1);
      mbar_init(&st->acc_empty[b], EPI_WARPS);   // the epilogue warps done reading the accumulators
    }
    mbar_init(&st->drain, 1);
    st->abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&st->tmem_base)),
                 "r"(512u)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (warp == 2) {
    const bool bad = warp_group_offsets(p.offsets, nE, 0, p.rows_cap, st->off, st->tile_start,
                                        [m_tiles](int cnt) { return ((cnt + NT - 1) / NT) * m_tiles; });
    if (bad && lane == 0) record_status(p.status, kDevBadOffsets);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = st->tmem_base;
  const int total = st->tile_start[nE];
  volatile int *abort_flag = &st->abort_flag;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t it = 0, tc = 0, sc_issued = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x, ++tc) {
        const Tile ti = decode_tile(st, nE, m_tiles, tile);
        const int wrow = ti.e * p.w_stride + ti.m * BM;           // first weight row of the tile
        // scale / bias rows of the tile: contiguous BM * kgroups bf16 per tensor
        const uint32_t sb = tc & 1u;
        if (!wait_bounded(&st->sc_empty[sb], ((tc >> 1) & 1u) ^ 1u, abort_flag, p.status, kDevTimeoutProducer, p.timeout_ns)) {
          ok = false;
          break;
        }
        const uint32_t sbytes = (uint32_t)(sc_elems * 2);
        mbar_expect_tx(&st->sc_full[sb], 2 * MATS * sbytes);
        for (int m = 0; m < MATS; ++m) {
          uint16_t *dst = sbuf + ((size_t)sb * MATS + m) * 2 * sc_elems;
          bulk_load(smem_u32(dst), p.sc[m] + (size_t)wrow * p.kgroups, sbytes, smem_u32(&st->sc_full[sb]));
          bulk_load(smem_u32(dst + sc_elems), p.bi[m] + (size_t)wrow * p.kgroups, sbytes,
                    smem_u32(&st->sc_full[sb]));
        }
        sc_issued = tc + 1;
        for (int kb = 0; kb < kb_n; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!wait_bounded(&st->empty[s], ph ^ 1u, abort_flag, p.status, kDevTimeoutProducer, p.timeout_ns)) {
            ok = false;
            break;
          }
          uint8_t *sp = stages + (size_t)s * S::STAGE_BYTES;
          const uint32_t fb = smem_u32(&st->full[s]);
          mbar_expect_tx(&st->full[s], S::STAGE_BYTES);
          tma_load_2d(smem_u32(sp), &mapC0, fb, kb * (BK / 2), wrow);
          if (PAIR) tma_load_2d(smem_u32(sp + CODE_BYTES), &mapC1, fb, kb * (BK / 2), wrow);
          tma_load_2d(smem_u32(sp + MATS * CODE_BYTES), &mapB, fb, kb * BK, ti.row0);
        }
      }
      if (!ok) {
        const uint32_t first = it > (uint32_t)STAGES ? it - STAGES : 0u;
        for (uint32_t i = first; i < it; ++i)
          if (!wait_drain(&st->full[i % STAGES], (i / STAGES) & 1u)) record_status(p.status, kDevTimeoutDrain);
        for (uint32_t b = 0; b < 2 && b < sc_issued; ++b) {
          const uint32_t last = sc_issued - 1 - b;
          if (!wait_drain(&st->sc_full[last & 1u], (last >> 1) & 1u)) record_status(p.status, kDevTimeoutDrain);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t it = 0, tcount = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x, ++tcount) {
        // accumulator buffer tcount % 2: the epilogue of two tiles ago must be done with it
        const uint32_t abuf = tcount & 1u;
        if (!wait_bounded(&st->acc_empty[abuf], ((tcount >> 1) & 1u) ^ 1u, abort_flag, p.status, kDevTimeoutMma, p.timeout_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t dcol = tmem_base + abuf * S::ACC_COLS;
        for (int kb = 0; kb < kb_n; ++kb, ++it) {
          const uint32_t j = it % SLOTS, use = it / SLOTS;
          if (!wait_bounded(&st->a_full[j], use & 1u, abort_flag, p.status, kDevTimeoutMma, p.timeout_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t db = sw128_desc(smem_u32(bslots + (size_t)j * B_BYTES));
          const uint32_t acol = tmem_base + 2 * S::ACC_COLS + j * S::A_COLS;
#pragma unroll
          for (int m = 0; m < MATS; ++m) {
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk)
              tc_mma_ts(dcol + m * NT, acol + m * (BK / 2) + kk * 8, db + (uint64_t)(kk * 2),
                        (kb | kk) != 0 ? 1u : 0u);
          }
          tc_commit(&st->a_empty[j]);
        }
        if (!ok) break;
        tc_commit(&st->acc_full[abuf]);
      }
      tc_commit(&st->drain);
      if (!wait_drain(&st->drain, 0u)) record_status(p.status, kDevTimeoutDrain);
    }
    __syncwarp();
  } else if (warp < 2 + DQ_WARPS) {
    // ------------------------------------------------------------ dequant
    // GROUPS groups of WPK warps take K-blocks round robin.  Inside a group a
    // warp owns one matrix and one TMEM lane quarter: thread = weight row
    // (= TMEM lane), 64 codes per K-block, stored as 32 columns of bf16 pairs.
    const int dw = warp - 2;
    const int grp = dw / WPK;
    const int gt = (dw % WPK) * 32 + lane;              // thread within the group
    const int mat = (dw % WPK) / 4;
    const int q = warp & 3;                             // TMEM lane quarter this warp may access
    const int row = q * 32 + lane;
    constexpr int BCH = (B_BYTES / 16) / (32 * WPK);    // token-tile chunks per thread
    const uint32_t stages_sa = smem_u32(stages), bslots_sa = smem_u32(bslots);
    uint32_t tc = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x, ++tc) {
      const Tile ti = decode_tile(st, nE, m_tiles, tile);
      const uint32_t sb = tc & 1u;
      if (!wait_bounded(&st->sc_full[sb], (tc >> 1) & 1u, abort_flag, p.status, kDevTimeoutEpilogue, p.timeout_ns)) {
        ok = false;
        break;
      }
      const uint32_t scl = smem_u32(sbuf + ((size_t)sb * MATS + mat) * 2 * sc_elems + (size_t)row * p.kgroups);
      const uint32_t bis = scl + 2u * (uint32_t)sc_elems;
      const uint32_t it0 = tc * (uint32_t)kb_n;
      const int kb_first = (int)((grp - (int)(it0 % GROUPS) + GROUPS) % GROUPS);
      for (int kb = kb_first; kb < kb_n; kb += GROUPS) {
        const uint32_t it = it0 + kb;                    // it % GROUPS == grp
        const int s = (int)(it % STAGES);
        const uint32_t ph = (it / STAGES) & 1u;
        const uint32_t j = it % SLOTS, use = it / SLOTS;
        if (!wait_bounded(&st->full[s], ph, abort_flag, p.status, kDevTimeoutEpilogue, p.timeout_ns)) {
          ok = false;
          break;
        }
        const uint32_t stage_sa = stages_sa + (uint32_t)(s * S::STAGE_BYTES);
        const uint32_t cp = stage_sa + (uint32_t)(mat * CODE_BYTES + row * (BK / 2));
        const uint4 c0 = lds128(cp), c1 = lds128(cp + 16);
        const uint32_t wv[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
        // token tile chunks (phase 1 reorders them into the operand K order;
        // phase 2's token tile, h, already is in it)
        uint4 bch[BCH];
#pragma unroll
        for (int i = 0; i < BCH; ++i) {
          bch[i] = lds128(stage_sa + (uint32_t)(MATS * CODE_BYTES) + (uint32_t)(gt + i * 32 * WPK) * 16u);
          if (PAIR) bch[i] = permute_chunk(bch[i]);
        }
        // the stage's bytes are all in registers: hand it back to the producer
        __syncwarp();
        if (lane == 0) mbar_arrive(&st->empty[s]);
        const uint32_t s1 = lds16(scl + 2u * kb), b1 = lds16(bis + 2u * kb);
        const uint32_t s2 = s1 | (s1 << 16), b2 = b1 | (b1 << 16);
        uint32_t av[32];
#pragma unroll
        for (int w = 0; w < 8; ++w) {
          const uint4 d = dequant8(wv[w], s2, b2);
          av[4 * w] = d.x; av[4 * w + 1] = d.y; av[4 * w + 2] = d.z; av[4 * w + 3] = d.w;
        }
        if (!wait_bounded(&st->a_empty[j], (use & 1u) ^ 1u, abort_flag, p.status, kDevTimeoutEpilogue, p.timeout_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        tmem_st32(tmem_base + ((uint32_t)(q * 32) << 16) + 2 * S::ACC_COLS + j * S::A_COLS + mat * (BK / 2), av);
#pragma unroll
        for (int i = 0; i < BCH; ++i)
          sts128(bslots_sa + j * (uint32_t)B_BYTES + (uint32_t)(gt + i * 32 * WPK) * 16u, bch[i]);
        tmem_wait_st();
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&st->a_full[j]);
      }
      if (!ok) break;
      // scale rows of this tile no longer needed
      __syncwarp();
      if (lane == 0) mbar_arrive(&st->sc_empty[sb]);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // warp quarter q reads TMEM lanes 32q..32q+31 (weight rows), 32 token columns
    const int q = warp & 3;
    const int row = q * 32 + lane;
    uint32_t tc = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++tc) {
      const Tile ti = decode_tile(st, nE, m_tiles, tile);
      const uint32_t abuf = tc & 1u;
      if (!wait_bounded(&st->acc_full[abuf], (tc >> 1) & 1u, abort_flag, p.status, kDevTimeoutEpilogue, p.timeout_ns)) break;
      tc_fence_after();
      const uint32_t ta = tmem_base + ((uint32_t)(q * 32) << 16) + abuf * S::ACC_COLS;
      const int f = ti.m * BM + row;
      if (PAIR) {
        uint32_t gv[16], uv[16];
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          tmem_ld16(ta + half * 16, gv);
          tmem_ld16(ta + NT + half * 16, uv);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const int tok = half * 16 + c;
            if (tok < ti.rows) {
              const float g = __uint_as_float(gv[c]);
              const float hv = g / (1.f + __expf(-g)) * __uint_as_float(uv[c]);
              const __nv_bfloat16 hb = __float2bfloat16_rn(hv);
              // h is the next phase's token operand: stored in its K order
              p.out[(size_t)(ti.row0 + tok) * p.N + ((f & ~7) | chunk_pos(f & 7))] =
                  *reinterpret_cast<const uint16_t *>(&hb);
            }
          }
        }
      } else {
        uint32_t y[16];
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          tmem_ld16(ta + half * 16, y);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const int tok = half * 16 + c;
            if (tok < ti.rows) {
              const __nv_bfloat16 yb = __float2bfloat16_rn(__uint_as_float(y[c]));
              p.out[(size_t)(ti.row0 + tok) * p.N + f] = *reinterpret_cast<const uint16_t *>(&yb);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&st->acc_empty[abuf]);
    }
  }

  tc_fence_before();
  __syncthreads();
  pdl_trigger();                         // tiles done: the next kernel may be scheduled
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(512u) : "memory");
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

// Codes as bytes: [rows, K/2] uint8, box 32 bytes x 128 rows, no swizzle.
cudaError_t map_codes(CUtensorMap *m, const void *ptr, uint64_t kbytes, uint64_t rows) {
  auto fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  cuuint64_t dims[2] = {kbytes, rows};
  cuuint64_t strides[1] = {kbytes};
  cuuint32_t box[2] = {(cuuint32_t)(BK / 2), (cuuint32_t)BM};
  cuuint32_t es[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(ptr), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// Token rows: [rows, K] bf16, box 64 x 32 rows, 128-byte swizzle.
cudaError_t map_tokens(CUtensorMap *m, const void *ptr, uint64_t k, uint64_t rows) {
  auto fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  cuuint64_t dims[2] = {k, rows};
  cuuint64_t strides[1] = {k * 2};
  cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)NT};
  cuuint32_t es[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

template <bool PAIR>
size_t smem_bytes(int kgroups) {
  using S = Q4Shape<PAIR>;
  return 1024 + (size_t)S::STAGES * S::STAGE_BYTES + (size_t)S::SLOTS * B_BYTES +
         2 * S::MATS * 2 * (size_t)BM * kgroups * 2 + 128 + sizeof(Q4Shared);
}

template <bool PAIR>
cudaError_t run(const FfnArgs &a, const void *tokens, int K, int N, int w_stride, const void *c0, const void *c1,
                const void *s0, const void *s1, const void *b0, const void *b1, void *out, cudaStream_t s) {
  CUtensorMap mc0, mc1, mb;
  // rows a map may address: the last expert's block ends N rows past its start
  const uint64_t wrows = (uint64_t)(a.E - 1) * w_stride + N;
  cudaError_t err = map_codes(&mc0, c0, (uint64_t)K / 2, wrows);
  if (err == cudaSuccess) err = map_codes(&mc1, PAIR ? c1 : c0, (uint64_t)K / 2, wrows);
  if (err == cudaSuccess) err = map_tokens(&mb, tokens, (uint64_t)K, (uint64_t)a.rows_cap);
  if (err != cudaSuccess) return err;
  Q4Params p;
  p.offsets = a.offsets;
  p.E = a.E;
  p.rows_cap = a.rows_cap;
  p.N = N;
  p.w_stride = w_stride;
  p.K = K;
  p.kgroups = K / BK;
  p.sc[0] = static_cast<const uint16_t *>(s0);
  p.sc[1] = static_cast<const uint16_t *>(PAIR ? s1 : s0);
  p.bi[0] = static_cast<const uint16_t *>(b0);
  p.bi[1] = static_cast<const uint16_t *>(PAIR ? b1 : b0);
  p.out = static_cast<uint16_t *>(out);
  p.status = a.status;
  p.timeout_ns = wait_timeout_ns();
  const size_t smem = smem_bytes<PAIR>(p.kgroups);
  auto kern = q4_tc_gemm<PAIR>;
  err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  const long long upper = ((long long)(a.rows_cap + NT - 1) / NT + a.E) * (N / BM);
  const int sms = sm_count();
  const int grid = (int)(upper < sms ? upper : sms);
  launch_plain(kern, grid, THREADS, smem, s, mc0, mc1, mb, p);
  return cudaGetLastError();
}

}  // namespace

bool q4_tc_supported(int d, int F) {
  // 128-row feature tiles, whole quantisation groups, scale rows of a tile
  // 16-byte aligned for the bulk copy, and the shared-memory budget
  if (d % BM != 0 || F % BM != 0 || d % BK != 0 || F % BK != 0) return false;
  if ((BM * (d / BK) * 2) % 16 != 0 || (BM * (F / BK) * 2) % 16 != 0) return false;
  return smem_bytes<true>(d / BK) <= 227 * 1024 && smem_bytes<false>(F / BK) <= 227 * 1024;
}

cudaError_t launch_ffn_q4_tc(const FfnArgs &a, cudaStream_t s) {
  cudaError_t err = run<true>(a, a.x, a.d, a.F, a.w_stride, a.w1, a.w2, a.s1, a.s2, a.b1, a.b2, a.h, s);
  if (err != cudaSuccess) return err;
  if (a.mid_event && (err = cudaEventRecord(a.mid_event, s)) != cudaSuccess) return err;
  return run<false>(a, a.h, a.F, a.d, a.d, a.w3, nullptr, a.s3, nullptr, a.b3, nullptr, a.y, s);
}

}  // namespace moe
