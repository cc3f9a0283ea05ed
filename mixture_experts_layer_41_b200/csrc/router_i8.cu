// Router logits x W_r^T on the 8-bit integer tensor cores, with a computed
// error bound per (token, expert).
//
// The gate of the "Mixture of Experts" blog (route / Router.route) and of
// Edge0 "MoE Spec and Routing" is a linear map whose weights must come out
// within 1e-6 of an fp64 evaluation.  Here both operands are written as sums
// of signed 8-bit digit planes over a power-of-two scale per row (the
// splitting idea of Ozaki, Ogita, Oishi and Rump, "Error-free transformations
// of matrix multiplication", Numer. Algorithms 59, 2012, in the integer form
// of Mukunoki, Ozaki, Ogita and Imamura, "DGEMM using Tensor Cores, and Its
// Accurate and Reproducible Versions", ISC 2020):
//
//   token t:  v = rne(x * 2^sx) with sx = min(22 - e_t, 127), |x| < 2^e_t over
//             the row, so |v| <= 2^22; u = v + 0x8080 gives the balanced digits
//             a0 = u >> 16 (in [-64, 64]), a1 = byte1(u) - 128, a2 = byte0(u) - 128,
//             v = a0 2^16 + a1 2^8 + a2.
//   expert e: v = rne(w * 2^sw) with sw = 30 - e_w, |v| <= 2^30; four balanced
//             digits b0..b3 the same way (u = v + 0x808080).
//
// Every digit product is exact and so is every int32 sum (|class sum| <
// 2^31 for d <= 52416), so the pairs (i, j) with i + j = c accumulate in one
// int32 TMEM accumulator per class c = 0..4; the pair (2, 3) is the one left
// out.  The epilogue forms S = sum_c C_c 2^(8 (4 - c)) in int64 and the logit
// S 2^(8 - sx - sw) in float64.  What differs from the exact logit is
//   dx . w  +  xhat . dw  +  x2 . w3
// (dx, dw: the rounding of x and w to their digits; x2, w3: the parts of
// xhat and what carried by the digits a2 and b3), bounded by
//   |dx|_1 |w|_inf + |xhat|_2 |dw|_2 + |x2|_2 |w3|_2,
// whose factors route_i8_prep writes per token and per expert (float64,
// rounded up; |xhat|_2 and |x2|_2 by upper bounds).  The preparation pass also
// lists the (few) elements of each token row that the digits round, so the
// selection pass adds dx . w exactly for the chosen experts; the rest of the
// bound is then about 1e-7 on the workloads' recipes.  Tokens whose bound
// could still move a weight past the routing tolerance, or swap two chosen
// experts, are recomputed exactly (route_finish_listed in router.cu).
//
// route_i8_prep   one block per SM: sixteen warps stream the token rows
//                 (scale, |x|_2, the list of rounded elements) through ring
//                 slots of their own filled by bulk copies; four warps split
//                 the expert rows (scale, four digit planes [4][e_pad][d_pad],
//                 norms) in integer arithmetic.
// route_i8_gemm   grid (N-expert tile, 128-token tile, hidden slice), one CTA
//                 per SM:
//   warp 0        TMA producer: the bf16 token tile (128 x 64, 128-byte
//                 swizzle) and the four weight digit tiles (N x 64 bytes,
//                 64-byte swizzle), stored one after another so that they
//                 read as one 4N-row operand;
//   warp 1        TMEM owner and single-thread MMA issuer: per 32-element K
//                 step three kind::i8 MMAs (M = 128), token digit i (from
//                 TMEM) against the weight digits side by side (N' = 4N, 4N,
//                 3N) into the class columns i N ..., which adds every kept
//                 pair (i, j) to class i + j;
//   warps 2-9     digit converters: each K-block's token tile into the three
//                 digit planes, stored into TMEM (lane = token row, four int8
//                 of K per column; three stages); after the last K-block, the
//                 epilogue (int64 combination, float64 scale, rows staged in
//                 shared memory for coalesced stores).
// Every mbarrier wait is bounded by %globaltimer (moe_set_wait_timeout_ns); on
// expiry the CTA records a status, drains its own copies and MMAs, frees TMEM
// and exits.
#include "common.cuh"

#include <cuda.h>
#include <cudaTypedefs.h>
#include <stdlib.h>

#include <algorithm>

namespace moe {
namespace {

constexpr int TM = 128;                 // tokens per tile (MMA M)
constexpr int BK = 64;                  // hidden elements per K-block
constexpr int XS = 3, AS = 3, WS = 3;   // ring depths: token tiles, token digit planes (TMEM), weight digit planes
static_assert(AS == WS, "one barrier releases a stage of both digit rings");
constexpr int XD = 3, WD = 4;           // digit planes of a token row and of a weight row
constexpr int NCLS = 5;                 // accumulator classes i + j = 0..4
constexpr int CONV_WARPS = 8;
constexpr int THREADS = 32 * (2 + CONV_WARPS);
constexpr uint64_t DRAIN_NS = 200000000ull;
constexpr float kMagic = 12582912.0f;   // 1.5 * 2^23: x + kMagic rounds x to an integer when |x| <= 2^22
constexpr int kMagicBits = 0x4B400000;
constexpr int kRoundList = 8;           // rounded elements listed per token row (exact correction)

template <int N>
struct I8Shape {
  static constexpr int X_BYTES = TM * BK * 2;   // bf16 token tile
  static constexpr int W_PLANE = N * BK;        // one weight digit plane
  static constexpr int W_BYTES = WD * W_PLANE;
  static constexpr int TILE_BYTES = XS * X_BYTES + WS * W_BYTES;
  // TMEM columns: the class accumulators [NCLS][N] (int32), then AS stages of
  // the token digit planes, row m in lane m, four int8 of K per column
  static constexpr int A_COLS = XD * (BK / 4);
  static constexpr int A_OFF = NCLS * N;
  static constexpr int COLS_USED = A_OFF + AS * A_COLS;
  static constexpr uint32_t TMEM_COLS =
      COLS_USED <= 32 ? 32 : (COLS_USED <= 64 ? 64 : (COLS_USED <= 128 ? 128 : (COLS_USED <= 256 ? 256 : 512)));
  static constexpr int CPW = N / 2;             // expert columns per epilogue warp
  // kind::i8: D s32, A s8, B s8, both K-major, M = 128.  The weight digit
  // planes lie one after another in the stage (rows j N .. j N + N - 1 hold
  // digit j), so one MMA of token digit i against the planes side by side
  // (N' = 4 N, or 3 N for i = 2) adds every pair (i, j) into the class
  // columns (i + j) N ... at once
  static constexpr uint32_t idesc(int n) {
    return (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(TM >> 4) << 24);
  }
  static constexpr uint32_t IDESC4 = idesc(WD * N), IDESC3 = idesc((WD - 1) * N);
  static_assert(WD * N <= 256, "an MMA spans at most 256 columns");
  static_assert(CONV_WARPS * 32 * (CPW + 1) * 8 <= XS * X_BYTES + WS * W_BYTES,
                "epilogue staging exceeds the rings");
  static_assert(COLS_USED <= 512, "accumulators and token digits exceed TMEM");
};

struct I8Params {
  uint64_t timeout_ns;
  int T, E;
  int kb_total, kb_per_slice;
  const int *sx;        // [T] token scale exponents
  const int *sw;        // [e_pad] expert scale exponents
  double *logits;       // [ks][T][E]
  int *status;
};

struct I8Shared {
  uint64_t x_full[XS], x_empty[XS];
  uint64_t a_full[AS], w_full[WS];
  uint64_t k_empty[AS];   // stage it % AS of both the token digits and the weight digits is free again
  uint64_t acc_full, drain;
  uint64_t tmem_full;   // the accumulators are allocated (warp 1)
  uint64_t acc_read;    // every converter warp has read them (warp 1 frees TMEM)
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
// Non-blocking test of the phase with the given parity.
__device__ __forceinline__ bool mbar_test_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
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
// A from tensor memory (a_tmem: lane = row, four int8 of K per column), B
// from shared memory: the shared-memory operand traffic is B's alone
__device__ __forceinline__ void tc_mma_i8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accum));
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&v)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
               "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
// K-major tile of 64-byte rows with the 64-byte swizzle (8-row groups 512
// bytes apart); +2 in the address field moves K by 32 int8.
__device__ __forceinline__ uint64_t sw64_desc(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(512 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)4 << 61);
}
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&v)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7])
               : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// 2^k as a double for -1022 <= k <= 1023
__device__ __forceinline__ double pow2d(int k) { return __longlong_as_double((long long)(1023 + k) << 52); }
// 2^k as a float for -126 <= k <= 127
__device__ __forceinline__ float pow2f(int k) { return __int_as_float((127 + k) << 23); }

// The digit value v of a bf16 element f (exactly as a float) at scale 2^sx,
// offset by 0x8080: one fused multiply-add rounds f 2^sx to the nearest
// integer (ties to even) in the low bits of kMagic.
__device__ __forceinline__ int token_u(float f, float scale) {
  return __float_as_int(__fmaf_rn(f, scale, kMagic)) - (kMagicBits - 0x8080);
}

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ uint32_t warp_max_u(uint32_t v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Norms are summed in float64 from exact terms; this factor covers their
// rounding (n * 2^-53 relative for n < 2^20 terms, and the square root).
constexpr double kRoundUp = 1.0 + 0x1p-30;

// ---------------------------------------------------------------- per-call preparation
struct PrepParams {
  const __nv_bfloat16 *x;
  const float *w;
  int T, d, E, e_pad, d_pad;
  int cw;                // token-row warps per block (PREP_EW expert-row warps follow)
  int nseg;              // ring segments of one token row (PREP_SEG bytes each, the last one shorter)
  uint64_t timeout_ns;
  int *status;
  int8_t *wdig;          // [WD][e_pad][d_pad]
  int *sx;               // [T]
  int *sw;               // [e_pad]
  double *xst;           // [T][4]:  |dx|_1, |xhat|_2, |x2|_2, 0
  double *wst;           // [e_pad][4]: |w|_inf, |dw|_2, |w3|_2, 0
  int *flag_count;       // zeroed here for the selection pass's exact-recompute list
  int *xcnt;             // [T] elements of the row that the digits round (dx != 0)
  int *xidx;             // [T][kRoundList] their indices, in order (the first kRoundList)
  double *xdx;           // [T][kRoundList] their dx
};

constexpr int PREP_CW_MAX = 16;   // token-row warps per block
constexpr int PREP_EW = 4;        // expert-row warps per block
constexpr int PREP_SPW = 3;       // ring slots per warp: one segment read while the next two land
constexpr int PREP_SEG = 4096;    // bytes of a token row per slot: 8 chunks of 16 bytes per lane
// fp32 sums of n < 2^16 non-negative terms (each rounded once) are within a
// factor (1 + 2^-7) of exact; the bound norms are rounded up by it
constexpr double kRoundUp32 = 1.0 + 0x1p-7;

struct PrepShared {
  uint64_t full[PREP_CW_MAX * PREP_SPW];
  double red[3][PREP_EW];
  uint32_t redm[PREP_EW];
  int abort_flag;
};

// Barrier 1 joins the expert-row warps (their reductions).
__device__ __forceinline__ void prep_bar(int nt) { asm volatile("bar.sync 1, %0;" ::"r"(nt) : "memory"); }

// One contiguous copy global -> shared memory completing on an mbarrier
// (16-byte aligned addresses, size a multiple of 16).
__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"((uint64_t)src), "r"(bytes), "r"(bar)
               : "memory");
}

// Whether an 8-element chunk of a token row holds an element the digits can
// round: only exponent fields below ethr can, unless the scale was clamped
// (all).
__device__ __forceinline__ bool chunk_may_round(uint4 v, bool all, int ethr) {
  const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
  bool any = all;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int elo = max((int)((w4[q] >> 7) & 0xFFu), 1), ehi = max((int)((w4[q] >> 23) & 0xFFu), 1);
    any |= min(elo, ehi) < ethr;
  }
  return any;
}

// Pass 2 on one 8-element chunk (index 8 i ..) of a token row, taken by the
// whole warp when any lane's chunk may round: the rounded elements listed in
// index order (cnt so far, warp-uniform), their |dx| added to l1.
__device__ __noinline__ void token_chunk_rounding(const PrepParams &p, int t, int i, uint4 v, double scale_d,
                                                  double inv, int lane, double &l1, int &cnt) {
  const unsigned full = 0xffffffffu;
  const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
  double dxs[8];
  int mine = 0;
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const uint32_t b = q & 1 ? (w4[q >> 1] & 0xFFFF0000u) : (w4[q >> 1] << 16);
    const double xd = (double)__uint_as_float(b);
    // the digits' value: x 2^sx rounded to the nearest integer, ties to even
    dxs[q] = xd - rint(xd * scale_d) * inv;
    l1 += fabs(dxs[q]);
    mine += dxs[q] != 0.0;
  }
  int before = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(full, before, o);
    if (lane >= o) before += y;
  }
  const int total = __shfl_sync(full, before, 31);
  before -= mine;
  if (mine) {
    int slot = cnt + before;
#pragma unroll
    for (int q = 0; q < 8; ++q)
      if (dxs[q] != 0.0) {
        if (slot < kRoundList) {
          p.xidx[(size_t)t * kRoundList + slot] = 8 * i + q;
          p.xdx[(size_t)t * kRoundList + slot] = dxs[q];
        }
        ++slot;
      }
  }
  cnt += total;
}

// The squares of the two bf16 values of w added into the two fp32 lanes of
// acc (one packed fused multiply-add: each lane rounded once).
__device__ __forceinline__ void sq_acc2(uint32_t w, unsigned long long &acc) {
  asm("{\n\t.reg .b64 t;\n\t"
      "mov.b64 t, {%1, %2};\n\t"
      "fma.rn.f32x2 %0, t, t, %0;\n\t}\n"
      : "+l"(acc)
      : "r"(w << 16), "r"(w & 0xFFFF0000u));
}
__device__ __forceinline__ uint32_t bf16x2_bits(__nv_bfloat162 v) { return *reinterpret_cast<uint32_t *>(&v); }

// Pass 1 on one 8-element chunk: the largest and smallest magnitude (as
// bf16 pairs: non-negative bf16 values order as their bits), |x|^2 in fp32,
// and the exponent field of the chunk's smallest magnitude (returned).
__device__ __forceinline__ uint32_t chunk_scan(uint4 v, __nv_bfloat162 &mx, __nv_bfloat162 &mn,
                                               unsigned long long &acc) {
  const uint32_t w4[4] = {v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu, v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu};
  const __nv_bfloat162 *b = reinterpret_cast<const __nv_bfloat162 *>(w4);
  const __nv_bfloat162 lo = __hmin2(__hmin2(b[0], b[1]), __hmin2(b[2], b[3]));
  mx = __hmax2(mx, __hmax2(__hmax2(b[0], b[1]), __hmax2(b[2], b[3])));
  mn = __hmin2(mn, lo);
  sq_acc2(v.x, acc);
  sq_acc2(v.y, acc);
  sq_acc2(v.z, acc);
  sq_acc2(v.w, acc);
  const uint32_t lb = bf16x2_bits(lo);
  return min(lb & 0xFFFFu, lb >> 16) >> 7;
}

// The row statistics from its largest / smallest magnitude bits and sums.
__device__ __forceinline__ void row_scale(uint32_t mb, int &sx, int &emax, bool &all, int &ethr) {
  // |x| < 2^e over the row (e = 0 for an all-zero row)
  int e = 0;
  if (mb >= 0x80u) e = (int)(mb >> 7) - 126;
  else if (mb != 0) e = (31 - __clz((int)mb)) - 132;
  sx = min(22 - e, 127);
  // x 2^sx = M 2^(E - Emax + 14) for a bf16 significand M, so only exponent
  // fields below Emax - 14 can round -- unless the scale was clamped
  // (Emax < 21), when any can
  emax = max((int)(mb >> 7), 1);
  all = emax < 21;
  ethr = emax - 14;
}

__device__ __forceinline__ void write_row_stats(const PrepParams &p, int t, int sx, int cnt, double l1, double l2) {
  const double inv = pow2d(-sx);
  p.sx[t] = sx;
  p.xcnt[t] = cnt;
  double *o = p.xst + (size_t)t * 4;
  o[0] = l1 * kRoundUp;
  o[1] = sqrt(l2) * kRoundUp32 + l1 * kRoundUp;        // |xhat|_2 <= |x|_2 + |dx|_1
  o[2] = 128.0 * sqrt((double)p.d) * inv * kRoundUp;   // |x2|_2 <= 128 sqrt(d) 2^-sx
  o[3] = 0.0;
}

// A warp's ring: PREP_SPW slots of its own; segment q of the warp's work
// (row j = w + (q / nseg) cw of the block, segment q mod nseg of it) lands in
// slot q mod PREP_SPW.  The warp copies its own segments in, PREP_SPW - 1
// ahead of the one it reads.
struct PrepRing {
  uint8_t *slots;               // this warp's [PREP_SPW][PREP_SEG]
  uint64_t *full;               // this warp's [PREP_SPW] barriers
  volatile int *abort_flag;
  int w, cw;                    // this warp, warps per block
  uint32_t nq;                  // segments of this warp's rows
};

__device__ __forceinline__ void seg_issue(const PrepParams &p, const PrepRing &r, uint32_t q, int lane) {
  if (lane != 0 || q >= r.nq) return;
  const int j = r.w + (int)(q / (uint32_t)p.nseg) * r.cw;
  const uint32_t off = (q % (uint32_t)p.nseg) * PREP_SEG;
  const uint32_t bytes = min((uint32_t)PREP_SEG, (uint32_t)p.d * 2u - off);
  const char *src = reinterpret_cast<const char *>(p.x + (size_t)(blockIdx.x + (size_t)j * gridDim.x) * p.d) + off;
  uint64_t *bar = r.full + q % PREP_SPW;
  mbar_expect_tx(bar, bytes);
  bulk_load(smem_u32(r.slots + (size_t)(q % PREP_SPW) * PREP_SEG), src, bytes, smem_u32(bar));
}

// The warp's q-th segment once it has landed (nullptr: the block gave up).
__device__ __forceinline__ const uint4 *seg_acquire(const PrepParams &p, const PrepRing &r, uint32_t q, int lane) {
  uint64_t *bar = r.full + q % PREP_SPW;
  const uint32_t par = (q / PREP_SPW) & 1u;
  int good = 1;
  if (lane == 0) good = wait_bounded(bar, par, r.abort_flag, p.status, kDevTimeoutEpilogue, p.timeout_ns);
  if (!__shfl_sync(0xffffffffu, good, 0)) return nullptr;
  // every lane observes the completed phase itself (it stays complete until
  // the slot is refilled by this warp, so this returns at once)
  wait_drain(bar, par);
  return reinterpret_cast<const uint4 *>(r.slots + (size_t)(q % PREP_SPW) * PREP_SEG);
}
// Done with segment q: its slot takes segment q + PREP_SPW.
__device__ __forceinline__ void seg_release(const PrepParams &p, const PrepRing &r, uint32_t q, int lane) {
  __syncwarp();
  seg_issue(p, r, q + PREP_SPW, lane);
}

// The row scale and statistics from the warp's pass-1 partials; then pass 2
// lists the rounded elements, reading again (from global memory) only the
// chunks that can round: those whose smallest exponent field (eb: a byte per
// chunk lane + 32 k) selects them when use_eb, else every chunk.
__device__ __forceinline__ void finish_row(const PrepParams &p, int t, int lane, __nv_bfloat162 mx,
                                           __nv_bfloat162 mn, double dl2, bool use_eb, const uint32_t (&eb)[8],
                                           uint32_t valid) {
  const unsigned full = 0xffffffffu;
  const int nv = p.d / 8;
  uint32_t mb = bf16x2_bits(mx), ml = bf16x2_bits(mn);
  mb = warp_max_u(max(mb & 0xFFFFu, mb >> 16));
  ml = min(ml & 0xFFFFu, ml >> 16);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ml = min(ml, __shfl_xor_sync(full, ml, o));
  int sx, emax, ethr;
  bool all;
  row_scale(mb, sx, emax, all, ethr);
  const double scale_d = pow2d(sx), inv = pow2d(-sx);
  const uint4 *xg = reinterpret_cast<const uint4 *>(p.x + (size_t)t * p.d);
  double l1 = 0.0;
  int cnt = 0;
  // (the smallest magnitude tells whether any element can round at all)
  if (all || max((int)(ml >> 7), 1) < ethr) {
    if (use_eb) {
      // chunk k can round when max(its smallest exponent field, 1) < ethr
      const uint32_t th = ethr > 0 ? (uint32_t)ethr * 0x01010101u : 0u;
      uint32_t sel = 0;
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const uint32_t f = __vcmpltu4(__vmaxu4(eb[r], 0x01010101u), th);   // 0xFF per selected byte
        sel |= ((f & 1u) | ((f >> 7) & 2u) | ((f >> 14) & 4u) | ((f >> 21) & 8u)) << (4 * r);
      }
      sel = (all ? 0xFFFFFFFFu : sel) & valid;
      uint32_t any = __reduce_or_sync(full, sel);
      while (any) {
        const int k = __ffs(any) - 1;
        any &= any - 1;
        const int i = lane + 32 * k;
        const uint4 v = (sel >> k) & 1u ? __ldg(xg + i) : make_uint4(0u, 0u, 0u, 0u);
        token_chunk_rounding(p, t, i, v, scale_d, inv, lane, l1, cnt);
      }
    } else {
      for (int base = 0; base < nv; base += 32) {
        const int i = base + lane;
        const uint4 v = i < nv ? __ldg(xg + i) : make_uint4(0u, 0u, 0u, 0u);
        if (__any_sync(full, chunk_may_round(v, all, ethr)))
          token_chunk_rounding(p, t, i, v, scale_d, inv, lane, l1, cnt);
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    l1 += __shfl_xor_sync(full, l1, o);
    dl2 += __shfl_xor_sync(full, dl2, o);
  }
  if (lane == 0) write_row_stats(p, t, sx, cnt, l1, dl2);
}

// One token row by one warp, its segments taken from the ring in order
// (lane: chunks lane + 32 k).  For rows of at most 4 segments each chunk's
// smallest exponent field is kept (a byte per chunk in eight registers), so
// pass 2 reads only the chunks that can round; longer rows check every chunk
// in pass 2.  Returns false when the block gave up.
__device__ __forceinline__ bool token_row(const PrepParams &p, const PrepRing &r, uint32_t &seq, int t, int lane) {
  const int nv = p.d / 8;
  const bool short_row = p.nseg <= 4;
  const uint32_t lo0 = 0u, hi0 = 0x7F7F7F7Fu;
  __nv_bfloat162 mx[2], mn[2];
  unsigned long long acc[2] = {0ull, 0ull};
#pragma unroll
  for (int a = 0; a < 2; ++a) {
    mx[a] = *reinterpret_cast<const __nv_bfloat162 *>(&lo0);
    mn[a] = *reinterpret_cast<const __nv_bfloat162 *>(&hi0);
  }
  uint32_t eb[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) eb[q] = 0xFFFFFFFFu;           // absent chunks: never selected
  uint32_t valid = 0;
#pragma unroll 1
  for (int s = 0; s < p.nseg; ++s) {
    const uint4 *seg = seg_acquire(p, r, seq, lane);
    if (!seg) return false;
    uint32_t w2[2] = {0xFFFFFFFFu, 0xFFFFFFFFu}, vb = 0;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      if (lane + 32 * kk + 256 * s < nv) {
        const uint32_t e = chunk_scan(seg[lane + 32 * kk], mx[kk & 1], mn[kk & 1], acc[(kk >> 1) & 1]);
        const int sh = 8 * (kk & 3);
        w2[kk >> 2] = (w2[kk >> 2] & ~(0xFFu << sh)) | (e << sh);
        vb |= 1u << kk;
      }
    }
    seg_release(p, r, seq, lane);
    ++seq;
#pragma unroll
    for (int q = 0; q < 4; ++q)
      if (s == q) {
        eb[2 * q] = w2[0];
        eb[2 * q + 1] = w2[1];
      }
    if (s < 4) valid |= vb << (8 * s);
  }
  const float2 a0 = *reinterpret_cast<const float2 *>(&acc[0]), a1 = *reinterpret_cast<const float2 *>(&acc[1]);
  const double dl2 = ((double)a0.x + (double)a0.y) + ((double)a1.x + (double)a1.y);
  finish_row(p, t, lane, __hmax2(mx[0], mx[1]), __hmin2(mn[0], mn[1]), dl2, short_row, eb, valid);
  return true;
}

// One expert row (scale, four digit planes, norms) by the block's
// expert-row warps (tid in [0, nt)).
__device__ __noinline__ void expert_row(const PrepParams &p, int e, int tid, int nt, PrepShared *sh) {
  const int lane = tid & 31, warp = tid >> 5, nw = nt >> 5;
  const size_t plane = (size_t)p.e_pad * p.d_pad;
  uint32_t *dst = reinterpret_cast<uint32_t *>(p.wdig + (size_t)e * p.d_pad);
  const int n4 = p.d / 4, nq = p.d_pad / 4;
  if (e >= p.E) {
    for (int i = tid; i < nq; i += nt)
#pragma unroll
      for (int j = 0; j < WD; ++j) dst[j * plane / 4 + i] = 0u;
    if (tid == 0) {
      p.sw[e] = 0;
      for (int j = 0; j < 4; ++j) p.wst[(size_t)e * 4 + j] = 0.0;
    }
    return;
  }
  const float4 *wr = reinterpret_cast<const float4 *>(p.w + (size_t)e * p.d);
  uint32_t mb = 0;
#pragma unroll 4
  for (int i = tid; i < n4; i += nt) {
    const float4 v = __ldg(wr + i);
    mb = max(max(mb, __float_as_uint(v.x) & 0x7FFFFFFFu), __float_as_uint(v.y) & 0x7FFFFFFFu);
    mb = max(max(mb, __float_as_uint(v.z) & 0x7FFFFFFFu), __float_as_uint(v.w) & 0x7FFFFFFFu);
  }
  mb = warp_max_u(mb);
  if (lane == 0) sh->redm[warp] = mb;
  prep_bar(nt);
  mb = 0;
  for (int w = 0; w < nw; ++w) mb = max(mb, sh->redm[w]);
  int ew = 0;
  if (mb >= 0x800000u) ew = (int)(mb >> 23) - 126;
  else if (mb != 0) ew = (31 - __clz((int)mb)) - 148;
  const int sw = 30 - ew;
  // v = rne(w 2^sw) from the fp32 fields in integer arithmetic: w 2^sw =
  // m 2^sh (m the 24-bit significand); the part rounded off, r = m - v 2^k
  // (k = -sh), gives dw 2^sw = r 2^-k exactly
  float dw2f = 0.f;                  // sum of (dw 2^sw)^2, each term and sum rounded once in fp32
  int w3s = 0;                       // sum of b3^2 (exact)
#pragma unroll 2
  for (int i = tid; i < nq; i += nt) {
    const float4 v4 = i < n4 ? __ldg(wr + i) : make_float4(0.f, 0.f, 0.f, 0.f);
    const uint32_t wb[4] = {__float_as_uint(v4.x), __float_as_uint(v4.y), __float_as_uint(v4.z),
                            __float_as_uint(v4.w)};
    uint32_t packed[WD] = {0, 0, 0, 0};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t fe = (wb[q] >> 23) & 0xFFu, mant = wb[q] & 0x7FFFFFu;
      const uint32_t m = fe ? (mant | 0x800000u) : mant;
      const int sh = (int)max(fe, 1u) - 150 + sw;     // <= 6: |v| <= 2^30
      uint32_t v = 0;
      float dws = 0.f;
      if (sh >= 0) {
        v = m << sh;
      } else if (sh >= -25) {
        const int k = -sh;
        const uint32_t rem = m & ((1u << k) - 1u), half = 1u << (k - 1);
        v = m >> k;
        v += (rem > half || (rem == half && (v & 1u))) ? 1u : 0u;   // ties to even
        dws = (float)((int)m - (int)(v << k)) * pow2f(-k);           // exact: |m - v 2^k| <= 2^24
      } else if (m != 0) {
        dws = 0.5f;                                                  // v = 0 and |w 2^sw| < 1/2
      }
      const int vs = (wb[q] >> 31) ? -(int)v : (int)v;
      const uint32_t u = (uint32_t)(vs + 0x808080);
      packed[0] |= ((u >> 24) & 0xFFu) << (8 * q);
      packed[1] |= (((u >> 16) & 0xFFu) ^ 0x80u) << (8 * q);
      packed[2] |= (((u >> 8) & 0xFFu) ^ 0x80u) << (8 * q);
      packed[3] |= ((u & 0xFFu) ^ 0x80u) << (8 * q);
      const int b3 = (int)(u & 0xFFu) - 128;
      w3s += b3 * b3;
      dw2f = fmaf(dws, dws, dw2f);
    }
#pragma unroll
    for (int j = 0; j < WD; ++j) dst[j * plane / 4 + i] = packed[j];
  }
  double dw2 = warp_sum_d((double)dw2f);
  double w3n = warp_sum_d((double)w3s);
  if (lane == 0) {
    sh->red[1][warp] = dw2;
    sh->red[2][warp] = w3n;
  }
  prep_bar(nt);
  if (tid == 0) {
    for (int w = 1; w < nw; ++w) {
      dw2 += sh->red[1][w];
      w3n += sh->red[2][w];
    }
    p.sw[e] = sw;
    double *o = p.wst + (size_t)e * 4;
    o[0] = (double)__uint_as_float(mb);                             // |w|_inf
    o[1] = sqrt(dw2) * pow2d(-sw) * (kRoundUp32 * kRoundUp);        // |dw|_2 (fp32 partial sums)
    o[2] = sqrt(w3n) * pow2d(-sw) * kRoundUp;                       // |w3|_2 (exact sum)
    o[3] = 0.0;
  }
}

// One block per SM: warps 0 .. cw - 1 take the block's token rows (block b:
// rows b, b + G, ...; warp w the block's rows j = w, w + cw, ...), segment by
// segment through their own rings, while warps cw .. cw + PREP_EW - 1 take
// the expert rows b, b + G, ... together.
__global__ void __launch_bounds__(32 * (PREP_CW_MAX + PREP_EW), 1) route_i8_prep(PrepParams p) {
  pdl_enter();
  extern __shared__ __align__(128) uint8_t prep_smem[];
  const int cw = p.cw, nslots = cw * PREP_SPW;
  PrepShared *sh = reinterpret_cast<PrepShared *>(prep_smem + (size_t)nslots * PREP_SEG);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < nslots; ++i) mbar_init(&sh->full[i], 1);
    sh->abort_flag = 0;
    if (blockIdx.x == 0) *p.flag_count = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  __syncthreads();
  const int G = gridDim.x;
  if (warp >= cw) {
    // ------------------------------------------------------------ expert rows
    for (int e = blockIdx.x; e < p.e_pad; e += G) expert_row(p, e, threadIdx.x - 32 * cw, 32 * PREP_EW, sh);
    return;
  }
  // -------------------------------------------------------------- token rows
  const int n_rows = p.T > (int)blockIdx.x ? (p.T - 1 - (int)blockIdx.x) / G + 1 : 0;
  const int my_rows = n_rows > warp ? (n_rows - 1 - warp) / cw + 1 : 0;
  const PrepRing ring{prep_smem + (size_t)warp * PREP_SPW * PREP_SEG, sh->full + warp * PREP_SPW, &sh->abort_flag,
                      warp, cw, (uint32_t)my_rows * (uint32_t)p.nseg};
  for (uint32_t q = 0; q < PREP_SPW; ++q) seg_issue(p, ring, q, lane);
  uint32_t seq = 0;
  bool ok = true;
  for (int j = warp; j < n_rows && ok; j += cw) {
    const int t = blockIdx.x + j * G;
    ok = token_row(p, ring, seq, t, lane);
  }
  if (!ok && lane == 0) {
    // let this warp's copies in flight land before the block goes away
    for (uint32_t q = seq; q < seq + PREP_SPW && q < ring.nq; ++q)
      if (!wait_drain(ring.full + q % PREP_SPW, (q / PREP_SPW) & 1u)) record_status(p.status, kDevTimeoutDrain);
  }
}

// ---------------------------------------------------------------- the GEMM
template <int N>
__global__ void __launch_bounds__(THREADS, 2)
route_i8_gemm(const __grid_constant__ CUtensorMap mapX, const __grid_constant__ CUtensorMap mapW,
              const I8Params p) {
  pdl_enter();
  using S = I8Shape<N>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t *xt = smem_raw + pad;
  uint8_t *wt = xt + XS * S::X_BYTES;
  I8Shared *st = reinterpret_cast<I8Shared *>(wt + WS * S::W_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int e0 = blockIdx.x * N, t0 = blockIdx.y * TM, slice = blockIdx.z;
  const int kb0 = slice * p.kb_per_slice;
  const int kb_n = max(0, min(p.kb_per_slice, p.kb_total - kb0));
  const int e_pad = gridDim.x * N;

  if (threadIdx.x == 0) {
    for (int s = 0; s < XS; ++s) {
      mbar_init(&st->x_full[s], 1);
      mbar_init(&st->x_empty[s], CONV_WARPS);
    }
    for (int s = 0; s < AS; ++s) {
      mbar_init(&st->a_full[s], CONV_WARPS);
      mbar_init(&st->k_empty[s], 1);
    }
    for (int s = 0; s < WS; ++s) {
      mbar_init(&st->w_full[s], 1);
    }
    mbar_init(&st->acc_full, 1);
    mbar_init(&st->drain, 1);
    mbar_init(&st->tmem_full, 1);
    mbar_init(&st->acc_read, CONV_WARPS);
    st->abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  __syncthreads();
  volatile int *abort_flag = &st->abort_flag;
  // Two CTAs share an SM: the copies start at once, while the tensor memory
  // may still belong to the other CTA (its allocation waits until that one
  // has read its accumulators and freed it).

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      // The two rings are filled independently, each as soon as its next
      // stage is free, so the token tiles run up to XS K-blocks ahead of the
      // MMAs whatever the weight ring waits for.
      int ix = 0, iw = 0;   // K-blocks issued on each ring
      bool ok = true;
      uint64_t t_idle = 0;  // start of the current wait without progress (0: none)
      uint32_t spins = 0;
      while (ok && (ix < kb_n || iw < kb_n)) {
        bool progressed = false;
        if (ix < kb_n && mbar_test_wait(&st->x_empty[ix % XS], ((ix / XS) & 1) ^ 1)) {
          mbar_expect_tx(&st->x_full[ix % XS], S::X_BYTES);
          tma_load_2d(smem_u32(xt + (ix % XS) * S::X_BYTES), &mapX, smem_u32(&st->x_full[ix % XS]),
                      (kb0 + ix) * BK, t0);
          ++ix;
          progressed = true;
        }
        if (iw < kb_n && mbar_test_wait(&st->k_empty[iw % WS], ((iw / WS) & 1) ^ 1)) {
          const int ws = iw % WS;
          mbar_expect_tx(&st->w_full[ws], S::W_BYTES);
#pragma unroll
          for (int j = 0; j < WD; ++j)
            tma_load_2d(smem_u32(wt + ws * S::W_BYTES + j * S::W_PLANE), &mapW, smem_u32(&st->w_full[ws]),
                        (kb0 + iw) * BK, j * e_pad + e0);
          ++iw;
          progressed = true;
        }
        if (progressed) {
          t_idle = 0;
          continue;
        }
        if (*abort_flag) {
          ok = false;
        } else if (t_idle == 0) {
          t_idle = global_ns();
        } else if ((++spins & 31u) == 0 && global_ns() - t_idle > p.timeout_ns) {
          *abort_flag = 1;
          record_status(p.status, kDevTimeoutProducer);
          ok = false;
        }
      }
      if (!ok) {
        for (int i = ix > XS ? ix - XS : 0; i < ix; ++i)
          if (!wait_drain(&st->x_full[i % XS], (i / XS) & 1)) record_status(p.status, kDevTimeoutDrain);
        for (int i = iw > WS ? iw - WS : 0; i < iw; ++i)
          if (!wait_drain(&st->w_full[i % WS], (i / WS) & 1)) record_status(p.status, kDevTimeoutDrain);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ TMEM owner and MMA issuer
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&st->tmem_base)),
                 "r"(S::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&st->tmem_full);
    const uint32_t tmem_base = st->tmem_base;
    if (lane == 0) {
      bool ok = true;
      for (int it = 0; it < kb_n && ok; ++it) {
        const int as = it % AS, ws = it % WS;
        if (!wait_bounded(&st->a_full[as], (it / AS) & 1, abort_flag, p.status, kDevTimeoutMma, p.timeout_ns) ||
            !wait_bounded(&st->w_full[ws], (it / WS) & 1, abort_flag, p.status, kDevTimeoutMma, p.timeout_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t ta = tmem_base + (uint32_t)(S::A_OFF + as * S::A_COLS);
        const uint64_t db = sw64_desc(smem_u32(wt + ws * S::W_BYTES));
        // the class columns were zeroed before the first K-block: every MMA adds
#pragma unroll
        for (int kk = 0; kk < BK / 32; ++kk)
#pragma unroll
          for (int i = 0; i < XD; ++i)
            tc_mma_i8_ts(tmem_base + (uint32_t)(i * N), ta + (uint32_t)(i * (BK / 4) + kk * 8), db + (uint64_t)(kk * 2),
                         i < XD - 1 ? S::IDESC4 : S::IDESC3, 1u);
        tc_commit(&st->k_empty[as]);   // one commit frees both operands' stage
      }
      if (ok) tc_commit(&st->acc_full);
      tc_commit(&st->drain);
      if (!wait_drain(&st->drain, 0u)) record_status(p.status, kDevTimeoutDrain);
      // the converters read the accumulators (or gave up): then TMEM is free
      // for the other CTA on this SM while this one stores the logits
      if (!wait_bounded(&st->acc_read, 0u, abort_flag, p.status, kDevTimeoutMma, p.timeout_ns))
        wait_drain(&st->acc_read, 0u);
    }
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(S::TMEM_COLS)
                 : "memory");
  } else {
    // ------------------------------------------------------------ digit converters, then the epilogue
    // warp (quarter q, half h): lane = token row 32 q + lane of the tile, the
    // K-block's elements [32 h, 32 h + 32) of it, i.e. one 32-element K step
    // of each digit plane (8 TMEM columns)
    const int cw = warp - 2;
    const int q = warp & 3, h = cw >> 2;
    const int r = q * 32 + lane;
    const bool have_tmem =
        wait_bounded(&st->tmem_full, 0u, abort_flag, p.status, kDevTimeoutEpilogue, p.timeout_ns);
    tc_fence_after();
    const uint32_t tmem_base = st->tmem_base;
    // (the row's scale is read here, so the copies start without waiting for it)
    const float sc = t0 + r < p.T ? pow2f(p.sx[t0 + r]) : 1.0f;
    const uint32_t lane_base = tmem_base + ((uint32_t)(q * 32) << 16);
    if (have_tmem) {
      // zero this quarter's half of the class accumulators (made visible to
      // the MMAs by the first K-block's wait and fence below)
      const uint32_t z[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
      constexpr int HALF = NCLS * N / 2;
#pragma unroll 1
      for (int c0 = 0; c0 < HALF; c0 += 8) tmem_st8(lane_base + (uint32_t)(h * HALF + c0), z);
    }
    bool ok = have_tmem;
    for (int it = 0; ok && it < kb_n; ++it) {
      const int xs = it % XS, as = it % AS;
      if (!wait_bounded(&st->x_full[xs], (it / XS) & 1, abort_flag, p.status, kDevTimeoutEpilogue, p.timeout_ns) ||
          !wait_bounded(&st->k_empty[as], ((it / AS) & 1) ^ 1, abort_flag, p.status, kDevTimeoutEpilogue,
                        p.timeout_ns)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint8_t *xrow = xt + xs * S::X_BYTES + r * 128;
      uint32_t pl[XD][8];   // [digit plane][4-element word]
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        const int c = 4 * h + cc;
        const uint4 v = *reinterpret_cast<const uint4 *>(xrow + ((c ^ (r & 7)) << 4));
        const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
        int u[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          u[2 * e] = token_u(__uint_as_float(w4[e] << 16), sc);
          u[2 * e + 1] = token_u(__uint_as_float(w4[e] & 0xFFFF0000u), sc);
        }
#pragma unroll
        for (int g = 0; g < 2; ++g) {
          const uint32_t u0 = u[4 * g], u1 = u[4 * g + 1], u2 = u[4 * g + 2], u3 = u[4 * g + 3];
          const uint32_t pa = __byte_perm(u0, u1, 0x5140), pb = __byte_perm(u2, u3, 0x5140);
          const uint32_t pc = __byte_perm(u0, u1, 0x0062), pd = __byte_perm(u2, u3, 0x0062);
          pl[2][2 * cc + g] = __byte_perm(pa, pb, 0x5410) ^ 0x80808080u;   // a2 = byte 0 - 128
          pl[1][2 * cc + g] = __byte_perm(pa, pb, 0x7632) ^ 0x80808080u;   // a1 = byte 1 - 128
          pl[0][2 * cc + g] = __byte_perm(pc, pd, 0x5410);                 // a0 = byte 2 (signed)
        }
      }
      const uint32_t col = (uint32_t)(S::A_OFF + as * S::A_COLS + h * 8);
#pragma unroll
      for (int i = 0; i < XD; ++i) tmem_st8(lane_base + col + (uint32_t)(i * (BK / 4)), pl[i]);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&st->x_empty[xs]);
        mbar_arrive(&st->a_full[as]);
      }
    }
    // ---------------------------------------------------------- epilogue
    const bool acc_ok = ok && kb_n > 0 &&
                        wait_bounded(&st->acc_full, 0u, abort_flag, p.status, kDevTimeoutEpilogue, p.timeout_ns);
    if (!acc_ok) {
      if (have_tmem) {
        tmem_wait_st();
        tc_fence_before();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&st->acc_read);   // nothing to read: TMEM may go
    } else {
      tc_fence_after();
      // each warp's 32 rows x CPW logits go through its own slice of the
      // (now idle) token-tile ring, so the global stores run along rows
      const int col0 = h * S::CPW;
      const int t = t0 + r;
      const int sxt = t < p.T ? p.sx[t] : 0;
      double *stage = reinterpret_cast<double *>(xt) + (size_t)cw * 32 * (S::CPW + 1);
#pragma unroll 1
      for (int cc = 0; cc < S::CPW; cc += 8) {
        uint32_t v[NCLS][8];
#pragma unroll
        for (int k = 0; k < NCLS; ++k) tmem_ld8(lane_base + (uint32_t)(k * N + col0 + cc), v[k]);
        tmem_wait_ld();
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          const long long s = ((long long)(int)v[0][m] << 32) + ((long long)(int)v[1][m] << 24) +
                              ((long long)(int)v[2][m] << 16) + ((long long)(int)v[3][m] << 8) +
                              (long long)(int)v[4][m];
          stage[lane * (S::CPW + 1) + cc + m] = (double)s * pow2d(8 - sxt - __ldg(p.sw + e0 + col0 + cc + m));
        }
      }
      // the accumulators are read: TMEM goes to the other CTA on this SM
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&st->acc_read);
      // row i of the warp: lanes take consecutive experts
      const int ne = min(S::CPW, p.E - (e0 + col0));
      for (int i = 0; i < 32; ++i) {
        const int tr = t0 + q * 32 + i;
        if (tr >= p.T) break;
        double *out = p.logits + ((size_t)slice * p.T + tr) * p.E + e0 + col0;
        for (int c = lane; c < ne; c += 32) out[c] = stage[i * (S::CPW + 1) + c];
      }
    }
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

cudaError_t make_map(CUtensorMap *m, CUtensorMapDataType dt, const void *ptr, uint64_t k, uint64_t rows,
                     uint64_t row_bytes, uint32_t box_k, uint32_t box_rows, CUtensorMapSwizzle sw) {
  auto fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  cuuint64_t dims[2] = {k, rows};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_k, box_rows};
  cuuint32_t es[2] = {1, 1};
  CUresult r = fn(m, dt, 2, const_cast<void *>(ptr), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

int prep_sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

template <int N>
cudaError_t run_gemm(const moe_config &c, const void *x, const I8RoutePlan &t, const I8RouteBuffers &b,
                     int *status, cudaStream_t s) {
  using S = I8Shape<N>;
  CUtensorMap mx, mw;
  cudaError_t err = make_map(&mx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, (uint64_t)c.hidden, (uint64_t)c.num_tokens,
                             (uint64_t)c.hidden * 2, BK, TM, CU_TENSOR_MAP_SWIZZLE_128B);
  if (err == cudaSuccess)
    err = make_map(&mw, CU_TENSOR_MAP_DATA_TYPE_UINT8, b.wdig, (uint64_t)t.d_pad, (uint64_t)WD * t.e_pad,
                   (uint64_t)t.d_pad, BK, N, CU_TENSOR_MAP_SWIZZLE_64B);
  if (err != cudaSuccess) return err;
  I8Params p;
  p.timeout_ns = wait_timeout_ns();
  p.T = c.num_tokens;
  p.E = c.num_experts;
  p.kb_total = t.d_pad / BK;
  p.kb_per_slice = t.kb_per_slice;
  p.sx = b.sx;
  p.sw = b.sw;
  p.logits = b.logits;
  p.status = status;
  const size_t smem = 1024 + (size_t)S::TILE_BYTES + sizeof(I8Shared);
  auto kern = route_i8_gemm<N>;
  err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  const dim3 grid(t.e_pad / N, (c.num_tokens + TM - 1) / TM, t.ks);
  launch_pdl(kern, grid, THREADS, smem, s, mx, mw, p);
  return cudaGetLastError();
}

}  // namespace

bool i8_route_supported(const moe_config &c) {
  // |class sum| < 2^31 needs d <= 52416; token rows are read as 16-byte vectors
  return c.act_dtype == MOE_BF16 && c.hidden % 8 == 0 && c.hidden <= 49152 && c.num_experts <= 256;
}

I8RoutePlan i8_route_plan(const moe_config &c) {
  I8RoutePlan t{};
  t.n = c.num_experts > 32 ? 64 : (c.num_experts > 16 ? 32 : 16);
  t.e_pad = (c.num_experts + t.n - 1) / t.n * t.n;
  t.d_pad = (c.hidden + BK - 1) / BK * BK;
  const int kb_total = t.d_pad / BK;
  const long long tiles = (long long)((c.num_tokens + TM - 1) / TM) * (t.e_pad / t.n);
  // hidden slices: the fewest rounds of 148 CTAs times K-blocks per CTA,
  // with about four K-blocks' worth of fixed cost per CTA
  int best_ks = 1;
  long long best = -1;
  const int max_ks = kb_total / 2 > 1 ? (kb_total / 2 < 16 ? kb_total / 2 : 16) : 1;
  for (int ks = 1; ks <= max_ks; ++ks) {
    const int per = (kb_total + ks - 1) / ks;
    const int used = (kb_total + per - 1) / per;
    const long long rounds = (tiles * used + 147) / 148;
    const long long cost = rounds * (per + 4);
    if (best < 0 || cost < best) {
      best = cost;
      best_ks = used;
    }
  }
  t.kb_per_slice = (kb_total + best_ks - 1) / best_ks;
  t.ks = (kb_total + t.kb_per_slice - 1) / t.kb_per_slice;
  return t;
}

size_t i8_route_bytes(const moe_config &c, const I8RoutePlan &t) {
  size_t n = 0;
  n += align_up(sizeof(double) * (size_t)t.ks * c.num_tokens * c.num_experts, 256);   // logits partials
  n += align_up((size_t)WD * t.e_pad * t.d_pad, 256);                                // weight digits
  n += align_up(sizeof(int) * (size_t)c.num_tokens, 256);                            // sx
  n += align_up(sizeof(int) * (size_t)t.e_pad, 256);                                 // sw
  n += align_up(sizeof(double) * 4 * (size_t)c.num_tokens, 256);                     // token norms
  n += align_up(sizeof(double) * 4 * (size_t)t.e_pad, 256);                          // expert norms
  n += align_up(sizeof(int) * (size_t)c.num_tokens, 256);                            // rounded counts
  n += align_up(sizeof(int) * kRoundList * (size_t)c.num_tokens, 256);               // their indices
  n += align_up(sizeof(double) * kRoundList * (size_t)c.num_tokens, 256);            // their dx
  n += align_up(sizeof(int) * (1 + (size_t)c.num_tokens), 256);                      // the exact-recompute list
  return n;
}

I8RouteBuffers i8_route_buffers(const moe_config &c, const I8RoutePlan &t, void *base) {
  I8RouteBuffers b{};
  char *p = static_cast<char *>(base);
  b.logits = reinterpret_cast<double *>(p);
  p += align_up(sizeof(double) * (size_t)t.ks * c.num_tokens * c.num_experts, 256);
  b.wdig = reinterpret_cast<int8_t *>(p);
  p += align_up((size_t)WD * t.e_pad * t.d_pad, 256);
  b.sx = reinterpret_cast<int *>(p);
  p += align_up(sizeof(int) * (size_t)c.num_tokens, 256);
  b.sw = reinterpret_cast<int *>(p);
  p += align_up(sizeof(int) * (size_t)t.e_pad, 256);
  b.xst = reinterpret_cast<double *>(p);
  p += align_up(sizeof(double) * 4 * (size_t)c.num_tokens, 256);
  b.wst = reinterpret_cast<double *>(p);
  p += align_up(sizeof(double) * 4 * (size_t)t.e_pad, 256);
  b.xcnt = reinterpret_cast<int *>(p);
  p += align_up(sizeof(int) * (size_t)c.num_tokens, 256);
  b.xidx = reinterpret_cast<int *>(p);
  p += align_up(sizeof(int) * kRoundList * (size_t)c.num_tokens, 256);
  b.xdx = reinterpret_cast<double *>(p);
  p += align_up(sizeof(double) * kRoundList * (size_t)c.num_tokens, 256);
  b.flag_count = reinterpret_cast<int *>(p);
  b.flag_list = b.flag_count + 1;
  b.round_list = kRoundList;
  return b;
}

cudaError_t launch_route_i8_logits(const moe_config &c, const void *x, const float *w_router,
                                   const I8RoutePlan &t, const I8RouteBuffers &b, int *status, cudaStream_t s) {
  PrepParams pp;
  pp.x = static_cast<const __nv_bfloat16 *>(x);
  pp.w = w_router;
  pp.T = c.num_tokens;
  pp.d = c.hidden;
  pp.E = c.num_experts;
  pp.e_pad = t.e_pad;
  pp.d_pad = t.d_pad;
  // one block per SM: 16 token-row warps with three ring segments each, and
  // the expert-row warps
  pp.cw = PREP_CW_MAX;
  pp.nseg = (int)((2 * (size_t)c.hidden + PREP_SEG - 1) / PREP_SEG);
  pp.timeout_ns = wait_timeout_ns();
  pp.status = status;
  pp.wdig = b.wdig;
  pp.sx = b.sx;
  pp.sw = b.sw;
  pp.xst = b.xst;
  pp.wst = b.wst;
  pp.xcnt = b.xcnt;
  pp.flag_count = b.flag_count;
  pp.xidx = b.xidx;
  pp.xdx = b.xdx;
  const size_t smem = (size_t)pp.cw * PREP_SPW * PREP_SEG + sizeof(PrepShared);
  cudaError_t err = cudaFuncSetAttribute(route_i8_prep, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  launch_pdl(route_i8_prep, prep_sm_count(), 32 * (pp.cw + PREP_EW), smem, s, pp);
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  switch (t.n) {
    case 16: return run_gemm<16>(c, x, t, b, status, s);
    case 32: return run_gemm<32>(c, x, t, b, status, s);
    default: return run_gemm<64>(c, x, t, b, status, s);
  }
}

}  // namespace moe
