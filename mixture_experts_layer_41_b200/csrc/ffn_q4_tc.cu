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
//               (kind::f16, M=128, N=32, K=16), commits free the stages.
//   warps 2-17  dequantise codes into the K-major 128-byte-swizzled bf16
//               operand (nibble -> exact bf16 through the 0x4300 magic, one
//               bf16x2 FMA with the group's scale and bias: a single
//               rounding of s*q + b), then run the tile epilogue:
//               SwiGLU (gate, up accumulators) or a plain store of y.
// Every mbarrier wait is bounded (2 s of %globaltimer) as in the bf16
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
constexpr int THREADS = 32 * (2 + DQ_WARPS);
constexpr int CODE_BYTES = BM * BK / 2; // 4 KiB of codes per matrix per K-block
constexpr int B_BYTES = NT * BK * 2;    // 4 KiB token tile per K-block
constexpr int A_BYTES = BM * BK * 2;    // 16 KiB dequantised operand per matrix
constexpr uint64_t TIMEOUT_NS = 2000000000ull;
constexpr uint64_t DRAIN_NS = 200000000ull;

// kind::f16: D fp32, A/B bf16, K-major, N = 32, M = 128
constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(NT >> 3) << 17) |
                           ((uint32_t)(BM >> 4) << 24);

template <bool PAIR>
struct Q4Shape {
  static constexpr int MATS = PAIR ? 2 : 1;
  static constexpr int STAGES = PAIR ? 6 : 8;
  static constexpr int STAGE_BYTES = MATS * CODE_BYTES + B_BYTES;   // multiple of 1024
  static constexpr int TMEM_COLS = PAIR ? 64 : 32;
};

struct Q4Params {
  const int32_t *offsets;   // [E+1]
  int E;
  int rows_cap;
  int N;                    // weight rows per expert (output features)
  int K;                    // reduction length
  int kgroups;              // K / 64
  const uint16_t *sc[2];    // [E, N, K/64] bf16 scales (gate / up, or down)
  const uint16_t *bi[2];    // biases, same layout
  uint16_t *out;            // [rows_cap, N] bf16
  int *status;
};

struct Q4Shared {
  uint64_t full[8], empty[8];
  uint64_t a_full[2], a_empty[2];
  uint64_t sc_full[2], sc_empty[2];
  uint64_t acc_full;
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
__device__ __forceinline__ bool wait_bounded(uint64_t *bar, uint32_t parity, volatile int *abort_flag, int *status,
                                             int code) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  uint32_t spins = 0;
  while (!mbar_try_wait(bar, parity)) {
    if (*abort_flag) return false;
    if ((++spins & 31u) == 0 && global_ns() - t0 > TIMEOUT_NS) {
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
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(IDESC), "r"(accum));
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
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&v)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7])
               : "r"(taddr));
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

// Eight 4-bit codes (element j at bits 4j) -> eight bf16 s*q + b, in order.
// (w >> 4i) & 0x000F000F | 0x43004300 is the bf16 pair (128 + q_i, 128 + q_{i+4});
// subtracting 128 is exact, so each element is rounded once, in the FMA.
__device__ __forceinline__ uint4 dequant8(uint32_t w, uint32_t s2, uint32_t b2) {
  const uint32_t magic = 0x43004300u;   // bf16 128.0 in both halves
  uint32_t p[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t v = ((w >> (4 * i)) & 0x000F000Fu) | magic;
    p[i] = bf2_fma(bf2_sub(v, magic), s2, b2);      // (q_i, q_{i+4})
  }
  uint4 o;
  o.x = prmt(p[0], p[1], 0x5410);   // (q0, q1)
  o.y = prmt(p[2], p[3], 0x5410);   // (q2, q3)
  o.z = prmt(p[0], p[1], 0x7632);   // (q4, q5)
  o.w = prmt(p[2], p[3], 0x7632);   // (q6, q7)
  return o;
}

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
  using S = Q4Shape<PAIR>;
  constexpr int MATS = S::MATS, STAGES = S::STAGES;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t *base = smem_raw + pad;
  uint8_t *stages = base;                                            // STAGES x [codes(MATS) | B]
  uint8_t *abuf = stages + (size_t)STAGES * S::STAGE_BYTES;         // 2 x MATS x A_BYTES
  uint16_t *sbuf = reinterpret_cast<uint16_t *>(abuf + 2 * MATS * A_BYTES);   // 2 x MATS x {scale, bias}
  const int sc_elems = BM * p.kgroups;                               // per matrix per kind
  Q4Shared *st = reinterpret_cast<Q4Shared *>(sbuf + 2 * MATS * 2 * sc_elems + 64);   // +128 bytes
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nE = p.E;
  const int m_tiles = p.N / BM;
  const int kb_n = p.kgroups;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&st->full[s], 1);
      mbar_init(&st->empty[s], DQ_WARPS + 1);   // dequant warps read codes, MMA reads B
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&st->a_full[b], DQ_WARPS);
      mbar_init(&st->a_empty[b], 1);
      mbar_init(&st->sc_full[b], 1);
      mbar_init(&st->sc_empty[b], DQ_WARPS);
    }
    mbar_init(&st->acc_full, 1);
    mbar_init(&st->drain, 1);
    st->abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&st->tmem_base)),
                 "r"((uint32_t)S::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (threadIdx.x == 64) {
    int prev = 0;
    bool bad = false;
    for (int i = 0; i <= nE; ++i) {
      int v = p.offsets[i];
      if (i == 0 && v != 0) bad = true;
      if (v < prev) { v = prev; bad = true; }
      if (v > p.rows_cap) { v = p.rows_cap; bad = true; }
      st->off[i] = v;
      prev = v;
    }
    st->off[0] = 0;
    if (bad) record_status(p.status, kDevBadOffsets);
    int acc = 0;
    for (int e = 0; e < nE; ++e) {
      st->tile_start[e] = acc;
      acc += ((st->off[e + 1] - st->off[e] + NT - 1) / NT) * m_tiles;
    }
    st->tile_start[nE] = acc;
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
        const int wrow = ti.e * p.N + ti.m * BM;           // first weight row of the tile
        // scale / bias rows of the tile: contiguous BM * kgroups bf16 per tensor
        const uint32_t sb = tc & 1u;
        if (!wait_bounded(&st->sc_empty[sb], ((tc >> 1) & 1u) ^ 1u, abort_flag, p.status, kDevTimeoutProducer)) {
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
          if (!wait_bounded(&st->empty[s], ph ^ 1u, abort_flag, p.status, kDevTimeoutProducer)) {
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
      uint32_t it = 0, ab = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        for (int kb = 0; kb < kb_n; ++kb, ++it, ++ab) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          const uint32_t b = ab & 1u;
          if (!wait_bounded(&st->full[s], ph, abort_flag, p.status, kDevTimeoutMma) ||
              !wait_bounded(&st->a_full[b], (ab >> 1) & 1u, abort_flag, p.status, kDevTimeoutMma)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t bsm = smem_u32(stages + (size_t)s * S::STAGE_BYTES + MATS * CODE_BYTES);
          const uint64_t db = sw128_desc(bsm);
#pragma unroll
          for (int m = 0; m < MATS; ++m) {
            const uint64_t da = sw128_desc(smem_u32(abuf + ((size_t)b * MATS + m) * A_BYTES));
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk)
              tc_mma(tmem_base + m * NT, da + (uint64_t)(kk * 2), db + (uint64_t)(kk * 2), (kb | kk) != 0 ? 1u : 0u);
          }
          tc_commit(&st->a_empty[b]);
          tc_commit(&st->empty[s]);
        }
        if (!ok) break;
        tc_commit(&st->acc_full);
      }
      tc_commit(&st->drain);
      if (!wait_drain(&st->drain, 0u)) record_status(p.status, kDevTimeoutDrain);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ dequant + epilogue
    const int dt = threadIdx.x - 64;                    // 0 .. 32*DQ_WARPS-1
    constexpr int PER_MAT = 32 * DQ_WARPS / MATS;       // threads per matrix
    constexpr int PARTS = PER_MAT / BM;                  // threads per weight row
    constexpr int WORDS = 8 / PARTS;                     // 32-bit code words per thread per K-block
    const int mat = dt / PER_MAT;
    const int row = (dt % PER_MAT) / PARTS;
    const int part = dt % PARTS;
    const uint32_t stages_sa = smem_u32(stages), abuf_sa = smem_u32(abuf);
    uint32_t it = 0, ab = 0, tc = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x, ++tc) {
      const Tile ti = decode_tile(st, nE, m_tiles, tile);
      const uint32_t sb = tc & 1u;
      if (!wait_bounded(&st->sc_full[sb], (tc >> 1) & 1u, abort_flag, p.status, kDevTimeoutEpilogue)) {
        ok = false;
        break;
      }
      const uint32_t scl = smem_u32(sbuf + ((size_t)sb * MATS + mat) * 2 * sc_elems + (size_t)row * p.kgroups);
      const uint32_t bis = scl + 2u * (uint32_t)sc_elems;
      for (int kb = 0; kb < kb_n; ++kb, ++it, ++ab) {
        const int s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1u;
        const uint32_t b = ab & 1u;
        if (!wait_bounded(&st->full[s], ph, abort_flag, p.status, kDevTimeoutEpilogue)) {
          ok = false;
          break;
        }
        const uint32_t cp = stages_sa + (uint32_t)(s * S::STAGE_BYTES + mat * CODE_BYTES + row * (BK / 2) +
                                                   part * (WORDS * 4));
        uint32_t wv[WORDS];
#pragma unroll
        for (int q = 0; q < (WORDS + 3) / 4; ++q) {
          if constexpr (WORDS >= 4) {
            const uint4 u = lds128(cp + 16 * q);
            wv[4 * q] = u.x; wv[4 * q + 1] = u.y; wv[4 * q + 2] = u.z; wv[4 * q + 3] = u.w;
          } else {
            uint32_t a0, a1;
            asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(a0), "=r"(a1) : "r"(cp));
            wv[0] = a0;
            wv[WORDS - 1] = a1;
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&st->empty[s]);
        const uint32_t s1 = lds16(scl + 2u * kb), b1 = lds16(bis + 2u * kb);
        const uint32_t s2 = s1 | (s1 << 16), b2 = b1 | (b1 << 16);
        if (!wait_bounded(&st->a_empty[b], ((ab >> 1) & 1u) ^ 1u, abort_flag, p.status, kDevTimeoutEpilogue)) {
          ok = false;
          break;
        }
        const uint32_t arow = abuf_sa + (uint32_t)((b * MATS + mat) * A_BYTES + row * 128);
#pragma unroll
        for (int w = 0; w < WORDS; ++w) {
          const int chunk = part * WORDS + w;   // 16-byte chunk = 8 elements of the 64
          sts128(arow + ((chunk ^ (row & 7)) << 4), dequant8(wv[w], s2, b2));
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) mbar_arrive(&st->a_full[b]);
      }
      if (!ok) break;
      // scale rows of this tile no longer needed
      __syncwarp();
      if (lane == 0) mbar_arrive(&st->sc_empty[sb]);
      // epilogue: warp quarter q reads TMEM lanes 32q..32q+31, group g the tokens 8g..8g+7
      if (!wait_bounded(&st->acc_full, tc & 1u, abort_flag, p.status, kDevTimeoutEpilogue)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int q = warp & 3;
      const int g = (warp - 2) >> 2;
      const uint32_t ta = tmem_base + ((uint32_t)(q * 32) << 16) + g * 8;
      const int f = ti.m * BM + q * 32 + lane;
      if (PAIR) {
        uint32_t gv8[8], uv8[8];
        tmem_ld8(ta, gv8);
        tmem_ld8(ta + NT, uv8);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const int tok = g * 8 + c;
          if (tok < ti.rows) {
            const float gv = __uint_as_float(gv8[c]);
            const float hv = gv / (1.f + __expf(-gv)) * __uint_as_float(uv8[c]);
            const __nv_bfloat16 hb = __float2bfloat16_rn(hv);
            p.out[(size_t)(ti.row0 + tok) * p.N + f] = *reinterpret_cast<const uint16_t *>(&hb);
          }
        }
      } else {
        uint32_t y[8];
        tmem_ld8(ta, y);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const int tok = g * 8 + c;
          if (tok < ti.rows) {
            const __nv_bfloat16 yb = __float2bfloat16_rn(__uint_as_float(y[c]));
            p.out[(size_t)(ti.row0 + tok) * p.N + f] = *reinterpret_cast<const uint16_t *>(&yb);
          }
        }
      }
      tc_fence_before();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"((uint32_t)S::TMEM_COLS)
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
  return 1024 + (size_t)S::STAGES * S::STAGE_BYTES + 2 * S::MATS * A_BYTES +
         2 * S::MATS * 2 * (size_t)BM * kgroups * 2 + 128 + sizeof(Q4Shared);
}

template <bool PAIR>
cudaError_t run(const FfnArgs &a, const void *tokens, int K, int N, const void *c0, const void *c1, const void *s0,
                const void *s1, const void *b0, const void *b1, void *out, cudaStream_t s) {
  CUtensorMap mc0, mc1, mb;
  const uint64_t wrows = (uint64_t)a.E * N;
  cudaError_t err = map_codes(&mc0, c0, (uint64_t)K / 2, wrows);
  if (err == cudaSuccess) err = map_codes(&mc1, PAIR ? c1 : c0, (uint64_t)K / 2, wrows);
  if (err == cudaSuccess) err = map_tokens(&mb, tokens, (uint64_t)K, (uint64_t)a.rows_cap);
  if (err != cudaSuccess) return err;
  Q4Params p;
  p.offsets = a.offsets;
  p.E = a.E;
  p.rows_cap = a.rows_cap;
  p.N = N;
  p.K = K;
  p.kgroups = K / BK;
  p.sc[0] = static_cast<const uint16_t *>(s0);
  p.sc[1] = static_cast<const uint16_t *>(PAIR ? s1 : s0);
  p.bi[0] = static_cast<const uint16_t *>(b0);
  p.bi[1] = static_cast<const uint16_t *>(PAIR ? b1 : b0);
  p.out = static_cast<uint16_t *>(out);
  p.status = a.status;
  const size_t smem = smem_bytes<PAIR>(p.kgroups);
  auto kern = q4_tc_gemm<PAIR>;
  err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  const long long upper = ((long long)(a.rows_cap + NT - 1) / NT + a.E) * (N / BM);
  const int sms = sm_count();
  const int grid = (int)(upper < sms ? upper : sms);
  kern<<<grid, THREADS, smem, s>>>(mc0, mc1, mb, p);
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
  cudaError_t err = run<true>(a, a.x, a.d, a.F, a.w1, a.w2, a.s1, a.s2, a.b1, a.b2, a.h, s);
  if (err != cudaSuccess) return err;
  if (a.mid_event && (err = cudaEventRecord(a.mid_event, s)) != cudaSuccess) return err;
  return run<false>(a, a.h, a.F, a.d, a.w3, nullptr, a.s3, nullptr, a.b3, nullptr, a.y, s);
}

}  // namespace moe
