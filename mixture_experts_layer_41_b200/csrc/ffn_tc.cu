// Grouped expert FFN in bf16 on the 5th-generation tensor cores (sm_100a).
//
// The grouped matmul of the "Mixture-of-Experts" design doc (The pipeline,
// step 3: the routed experts as one grouped matmul over the ragged
// per-expert token groups) with the expert MLPs of the "Mixture of Experts"
// blog (ReLU) and the "moe-architecture" skill page / Edge0 _swiglu
// (silu(gate) * up).  Two launches of one persistent kernel:
//   phase 1: h = act(x_perm W1^T [, x_perm W2^T])   A = x_perm [R, d]
//   phase 2: y = h W3^T                              A = h      [R, F]
// Both are "TN" products with K-major operands: D[r, n] = sum_k A[r, k] B[n, k].
//
// Per CTA (one per SM, persistent over a static tile schedule):
//   warp 0      TMA producer: A tile 128 x 64 and two 128 x 64 B halves per
//               stage into 128-byte-swizzled shared memory, 4 stages, one
//               mbarrier with a transaction count per stage;
//   warp 1      owns 512 TMEM columns (two 128 x 256 fp32 accumulators) and
//               issues tcgen05.mma (M=128, N=256, K=16) from one thread; a
//               tcgen05.commit frees each smem stage and publishes each tile;
//   warps 2-5   epilogue: tcgen05.ld of their 32-lane quarter, activation
//               (SwiGLU pairs accumulator column j with j+128: the gate and up
//               halves of the B tile), bf16 pack, row-masked 16-byte stores.
// Tiles run expert by expert, n-tile-major with the m-tiles of an expert
// innermost, so the CTAs in flight share B (weight) tiles through L2.
// Optionally one more group follows the experts: the shared expert ("Shared
// expert" of the MoE documentation: applied to every token with weight 1),
// whose A rows are the token matrix itself (phase 1) or its own intermediate
// (phase 2), with its own weights and output; its tiles run m-tile-major with
// the n-tiles innermost, so each 128-token tile of A is read once from HBM
// while its weights stay in L2.  The shared expert then costs no launch and
// no tail of its own.
// A tile's rows past its expert's end belong to the next expert (or are
// zero-filled by TMA past the buffer); their results are never stored.
//
// Every mbarrier wait is bounded by %globaltimer (2 s unless moe_set_wait_timeout_ns says otherwise): on expiry the thread
// records a status code in the workspace, raises a CTA-wide abort flag, waits
// (bounded) for its own in-flight copies or MMAs and the CTA frees its TMEM
// and exits.
#include "common.cuh"

#include <cuda.h>
#include <cudaTypedefs.h>

namespace moe {
namespace {

constexpr int BM = 128;
constexpr int BK = 64;                        // 64 bf16 = 128 bytes: one swizzle row
constexpr int BN = 256;                       // MMA N: two 128-row B halves
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;          // 16 KiB
constexpr int BH_BYTES = 128 * BK * 2;        // 16 KiB per B half
constexpr int STAGE_BYTES = A_BYTES + 2 * BH_BYTES;
constexpr int THREADS = 192;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint64_t DRAIN_NS = 200000000ull;

// kind::f16 instruction descriptor: D fp32, A and B bf16, both K-major,
// N = 256 (bits 17-22 hold N/8), M = 128 (bits 24-28 hold M/16).
constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) |
                           ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);

enum Mode { MODE_PLAIN = 0, MODE_RELU = 1, MODE_SWIGLU = 2 };

struct TcParams {
  uint64_t timeout_ns;        // bound on every barrier wait (moe_set_wait_timeout_ns)
  const int32_t *offsets;   // [E+1] or nullptr (one group of `rows`)
  int E;
  int rows;
  int rows_cap;             // rows of A and out
  int N;                    // output columns
  int b_stride;             // B rows from one expert to the next (N, or 2N for stacked gate/up)
  int K;
  int mode;
  int n_tiles;              // output tiles per group along N
  __nv_bfloat16 *out;       // [rows_cap, N]
  int *status;
  const int32_t *gather;    // A row r is token gather[r] of the token matrix (mapA over [T, K], one-row box),
                            // or nullptr: A row r is row r of mapA
  int shared_rows;          // rows of the shared-expert group (0: none); A from mapA2, B from mapS0 / mapS1
  __nv_bfloat16 *out2;      // its output [shared_rows, N]
};

struct SharedState {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  int32_t off[kMaxExperts + 1];
  int32_t tile_start[kMaxExperts + 2];   // [nE + 1]: start of the shared-expert group's tiles
};

constexpr size_t SMEM_BYTES = (size_t)STAGES * STAGE_BYTES + sizeof(SharedState) + 1024;

// ---------------------------------------------------------------- PTX wrappers
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
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

// Wait for the phase of `bar` with the given parity.  Returns false when the
// CTA is aborting or after limit_ns (then the abort flag and `code` are set).
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

// Wait used only while draining after an abort: ignores the abort flag.
__device__ __forceinline__ bool wait_drain(uint64_t *bar, uint32_t parity) {
  const uint64_t t0 = global_ns();
  while (!mbar_try_wait(bar, parity))
    if (global_ns() - t0 > DRAIN_NS) return false;
  return true;
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, uint32_t bar, int x,
                                            int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
          dst),
      "l"((uint64_t)map), "r"(bar), "r"(x), "r"(y)
      : "memory");
}

// Four rows (r0..r3) of a one-row-box map into four consecutive 128-byte rows
// at dst; the 128-byte swizzle follows the destination address as for a tile.
__device__ __forceinline__ void tma_gather4(uint32_t dst, const CUtensorMap *map, uint32_t bar, int x, int r0,
                                            int r1, int r2, int r3) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(dst),
      "l"((uint64_t)map), "r"(bar), "r"(x), "r"(r0), "r"(r1), "r"(r2), "r"(r3)
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_commit(uint64_t *bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(IDESC), "r"(accum));
}

// Shared-memory matrix descriptor for a K-major tile written by TMA with the
// 128-byte swizzle: 8-row core groups 1024 bytes apart (stride byte offset),
// descriptor version 1, layout SWIZZLE_128B.  Advancing K by 16 bf16 inside
// the 128-byte row moves the start address by 32 bytes.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
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

// ---------------------------------------------------------------- scheduling
struct TileInfo {
  int e, row0, rows, n;
  bool shared;   // a tile of the shared-expert group (e == nE)
};

__device__ __forceinline__ TileInfo decode_tile(const SharedState *st, int nE, int n_tiles, int shared_rows,
                                                int tile) {
  TileInfo ti;
  if (tile >= st->tile_start[nE]) {
    // shared-expert group: m-tile-major, n-tiles innermost
    const int local = tile - st->tile_start[nE];
    ti.e = nE;
    ti.shared = true;
    ti.n = local % n_tiles;
    ti.row0 = (local / n_tiles) * BM;
    ti.rows = min(BM, shared_rows - ti.row0);
    return ti;
  }
  int lo = 0, hi = nE;   // largest e with tile_start[e] <= tile; tile_start[nE] > tile
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (st->tile_start[mid] <= tile) lo = mid; else hi = mid;
  }
  ti.e = lo;
  ti.shared = false;
  const int local = tile - st->tile_start[lo];
  const int cnt = st->off[lo + 1] - st->off[lo];
  const int mt = (cnt + BM - 1) / BM;
  ti.n = local / mt;
  ti.row0 = st->off[lo] + (local % mt) * BM;
  ti.rows = min(BM, st->off[lo + 1] - ti.row0);
  return ti;
}

// B rows of a tile's two 128-row halves: SwiGLU takes the same 128 features
// of the gate (map 0) and up (map 1) weights; otherwise 256 consecutive rows
// of one weight.  The shared expert's weights start at row 0 of their maps.
__device__ __forceinline__ void b_rows(const TcParams &p, const TileInfo &ti, int &b0, int &b1) {
  const int base = ti.shared ? 0 : ti.e * p.b_stride;
  if (p.mode == MODE_SWIGLU) {
    b0 = base + ti.n * 128;
    b1 = b0;
  } else {
    b0 = base + ti.n * BN;
    b1 = b0 + 128;
  }
}

__device__ __forceinline__ float silu_f(float g) { return g / (1.f + __expf(-g)); }

__global__ void __launch_bounds__(THREADS, 1)
tc_grouped_gemm(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB0,
                const __grid_constant__ CUtensorMap mapB1, const __grid_constant__ CUtensorMap mapA2,
                const __grid_constant__ CUtensorMap mapS0, const __grid_constant__ CUtensorMap mapS1,
                const TcParams p) {
  pdl_wait();
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t *tiles = smem_raw + pad;
  SharedState *st = reinterpret_cast<SharedState *>(tiles + (size_t)STAGES * STAGE_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nE = p.offsets ? p.E : 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&st->full[s], 1);
      mbar_init(&st->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&st->acc_full[b], 1);
      mbar_init(&st->acc_empty[b], 4);
    }
    mbar_init(&st->drain, 1);
    st->abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 0 && lane == 0) {
    asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&mapA) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&mapB0) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&mapB1) : "memory");
    if (p.shared_rows > 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&mapA2) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&mapS0) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&mapS1) : "memory");
    }
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&st->tmem_base)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  // group offsets, clamped to [0, rows_cap] and made non-decreasing
  if (warp == 2) {
    const int n_tiles = p.n_tiles;
    const bool bad = warp_group_offsets(p.offsets, nE, p.rows, p.rows_cap, st->off, st->tile_start,
                                        [n_tiles](int cnt) { return ((cnt + BM - 1) / BM) * n_tiles; });
    if (bad && lane == 0) record_status(p.status, kDevBadOffsets);
    if (lane == 0) st->tile_start[nE + 1] = st->tile_start[nE] + ((p.shared_rows + BM - 1) / BM) * n_tiles;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = st->tmem_base;
  const int total = st->tile_start[nE + 1];
  const int kb_n = (p.K + BK - 1) / BK;
  volatile int *abort_flag = &st->abort_flag;

  if (warp == 0 && p.gather) {
    // ------------------------------------------------------------ TMA producer, gathered A
    // Fused dispatch: the A tile's 128 rows are fetched straight from the
    // token matrix, four per lane with tile::gather4 (one-row boxes); lane 0
    // waits for the stage, posts the byte count and loads the B halves.
    uint32_t it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
      const TileInfo ti = decode_tile(st, nE, p.n_tiles, p.shared_rows, tile);
      // rows past the expert's end repeat its first row (their results are masked)
      int g[4] = {0, 0, 0, 0};
      if (!ti.shared) {
        const int row_end = st->off[ti.e + 1];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int r = ti.row0 + lane * 4 + i;
          g[i] = p.gather[r < row_end ? r : ti.row0];
        }
      }
      int b0, b1;
      b_rows(p, ti, b0, b1);
      for (int kb = 0; kb < kb_n; ++kb, ++it) {
        const int s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1u;
        int good = 1;
        if (lane == 0) good = wait_bounded(&st->empty[s], ph ^ 1u, abort_flag, p.status, kDevTimeoutProducer, p.timeout_ns);
        good = __shfl_sync(0xffffffffu, good, 0);
        if (!good) {
          ok = false;
          break;
        }
        uint8_t *sa = tiles + (size_t)s * STAGE_BYTES;
        const uint32_t fb = smem_u32(&st->full[s]);
        if (lane == 0) mbar_expect_tx(&st->full[s], STAGE_BYTES);
        __syncwarp();
        if (!ti.shared) {
          tma_gather4(smem_u32(sa) + (uint32_t)lane * 512u, &mapA, fb, kb * BK, g[0], g[1], g[2], g[3]);
          if (lane == 0) {
            tma_load_2d(smem_u32(sa + A_BYTES), &mapB0, fb, kb * BK, b0);
            tma_load_2d(smem_u32(sa + A_BYTES + BH_BYTES), &mapB1, fb, kb * BK, b1);
          }
        } else if (lane == 0) {
          tma_load_2d(smem_u32(sa), &mapA2, fb, kb * BK, ti.row0);
          tma_load_2d(smem_u32(sa + A_BYTES), &mapS0, fb, kb * BK, b0);
          tma_load_2d(smem_u32(sa + A_BYTES + BH_BYTES), &mapS1, fb, kb * BK, b1);
        }
      }
    }
    if (!ok && lane == 0) {
      const uint32_t first = it > (uint32_t)STAGES ? it - STAGES : 0u;
      for (uint32_t i = first; i < it; ++i)
        if (!wait_drain(&st->full[i % STAGES], (i / STAGES) & 1u)) record_status(p.status, kDevTimeoutDrain);
    }
    __syncwarp();
  } else if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        const TileInfo ti = decode_tile(st, nE, p.n_tiles, p.shared_rows, tile);
        int b0, b1;
        b_rows(p, ti, b0, b1);
        const CUtensorMap *ma = ti.shared ? &mapA2 : &mapA;
        const CUtensorMap *mb0 = ti.shared ? &mapS0 : &mapB0;
        const CUtensorMap *mb1 = ti.shared ? &mapS1 : &mapB1;
        for (int kb = 0; kb < kb_n; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!wait_bounded(&st->empty[s], ph ^ 1u, abort_flag, p.status, kDevTimeoutProducer, p.timeout_ns)) {
            ok = false;
            break;
          }
          uint8_t *sa = tiles + (size_t)s * STAGE_BYTES;
          const uint32_t fb = smem_u32(&st->full[s]);
          mbar_expect_tx(&st->full[s], STAGE_BYTES);
          tma_load_2d(smem_u32(sa), ma, fb, kb * BK, ti.row0);
          tma_load_2d(smem_u32(sa + A_BYTES), mb0, fb, kb * BK, b0);
          tma_load_2d(smem_u32(sa + A_BYTES + BH_BYTES), mb1, fb, kb * BK, b1);
        }
      }
      if (!ok) {
        // let the copies already issued land before the CTA goes away
        const uint32_t first = it > (uint32_t)STAGES ? it - STAGES : 0u;
        for (uint32_t i = first; i < it; ++i)
          if (!wait_drain(&st->full[i % STAGES], (i / STAGES) & 1u)) record_status(p.status, kDevTimeoutDrain);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t it = 0, tcount = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        const uint32_t buf = tcount & 1u, use = tcount >> 1;
        if (!wait_bounded(&st->acc_empty[buf], (use & 1u) ^ 1u, abort_flag, p.status, kDevTimeoutMma, p.timeout_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t dt = tmem_base + buf * BN;
        for (int kb = 0; kb < kb_n; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!wait_bounded(&st->full[s], ph, abort_flag, p.status, kDevTimeoutMma, p.timeout_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(tiles + (size_t)s * STAGE_BYTES);
          const uint64_t da = sw128_desc(sa);
          const uint64_t db = sw128_desc(sa + A_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            tc_mma(dt, da + (uint64_t)(kk * 2), db + (uint64_t)(kk * 2), (kb | kk) != 0 ? 1u : 0u);
          tc_commit(&st->empty[s]);
        }
        if (!ok) break;
        tc_commit(&st->acc_full[buf]);
        ++tcount;
      }
      // every MMA this thread issued has completed once `drain` flips
      tc_commit(&st->drain);
      if (!wait_drain(&st->drain, 0u)) record_status(p.status, kDevTimeoutDrain);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                 // TMEM lane quarter of this warp
    const int rloc = q * 32 + lane;         // row of the tile this thread stores
    uint32_t tcount = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
      const TileInfo ti = decode_tile(st, nE, p.n_tiles, p.shared_rows, tile);
      const uint32_t buf = tcount & 1u, use = tcount >> 1;
      if (!wait_bounded(&st->acc_full[buf], use & 1u, abort_flag, p.status, kDevTimeoutEpilogue, p.timeout_ns)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + buf * BN + ((uint32_t)(q * 32) << 16);
      const bool valid = rloc < ti.rows;
      __nv_bfloat16 *orow = (ti.shared ? p.out2 : p.out) + (size_t)(ti.row0 + (valid ? rloc : 0)) * p.N;
      if (p.mode == MODE_SWIGLU) {
        const int col0 = ti.n * 128;
#pragma unroll 1
        for (int c = 0; c < 128; c += 32) {
          uint32_t g[32], u[32];
          tmem_ld32(tb + c, g);
          tmem_ld32(tb + 128 + c, u);
          tmem_wait_ld();
          if (valid) {
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              const int col = col0 + c + v * 8;
              if (col < p.N) {
                uint4 o;
                uint32_t *op = reinterpret_cast<uint32_t *>(&o);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                  const int a = v * 8 + 2 * i;
                  const float h0 = silu_f(__uint_as_float(g[a])) * __uint_as_float(u[a]);
                  const float h1 = silu_f(__uint_as_float(g[a + 1])) * __uint_as_float(u[a + 1]);
                  op[i] = pack_bf16x2(h0, h1);
                }
                *reinterpret_cast<uint4 *>(orow + col) = o;
              }
            }
          }
        }
      } else {
        const int col0 = ti.n * BN;
        const bool relu = p.mode == MODE_RELU;
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          uint32_t a[32];
          tmem_ld32(tb + c, a);
          tmem_wait_ld();
          if (valid) {
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              const int col = col0 + c + v * 8;
              if (col < p.N) {
                uint4 o;
                uint32_t *op = reinterpret_cast<uint32_t *>(&o);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                  float x0 = __uint_as_float(a[v * 8 + 2 * i]);
                  float x1 = __uint_as_float(a[v * 8 + 2 * i + 1]);
                  if (relu) {
                    x0 = fmaxf(x0, 0.f);
                    x1 = fmaxf(x1, 0.f);
                  }
                  op[i] = pack_bf16x2(x0, x1);
                }
                *reinterpret_cast<uint4 *>(orow + col) = o;
              }
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&st->acc_empty[buf]);
      ++tcount;
    }
  }

  tc_fence_before();
  __syncthreads();
  pdl_trigger();                         // tiles done: the next kernel may be scheduled
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TMEM_COLS)
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

// 2-D bf16 map over a row-major [outer, inner] matrix, box 64 x box_outer,
// 128-byte swizzle, zero fill out of bounds.
cudaError_t make_map(CUtensorMap *m, const void *ptr, uint64_t inner, uint64_t outer, uint32_t box_outer) {
  auto fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {(cuuint32_t)BK, box_outer};
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

// B0 / B1: expert e's rows start at e * b_stride; a map covers the rows up to
// the end of the last expert's N.
// gather (nullable): A row r is token gather[r] of A = [a_rows, K] (the
// fused dispatch); otherwise A is [rows_cap, K] in row order.
// shared (nullable): the shared-expert group, one more group after the
// experts with its own A ([shared->rows, K]), weights ([N, K] each) and output.
struct SharedGroup {
  const void *a, *b0, *b1;
  int rows;
  void *out;
};

cudaError_t run_gemm(const void *A, int rows_cap, int K, const void *B0, const void *B1, int b_stride, int N,
                     int mode, const int32_t *offsets, int E, int rows, void *out, int *status,
                     cudaStream_t s, const int32_t *gather = nullptr, int a_rows = 0,
                     const SharedGroup *shared = nullptr) {
  CUtensorMap ma, mb0, mb1, ma2, ms0, ms1;
  const int b_rows_total = ((offsets ? E : 1) - 1) * b_stride + N;
  cudaError_t err = gather ? make_map(&ma, A, (uint64_t)K, (uint64_t)a_rows, 1)
                           : make_map(&ma, A, (uint64_t)K, (uint64_t)rows_cap, BM);
  if (err == cudaSuccess) err = make_map(&mb0, B0, (uint64_t)K, (uint64_t)b_rows_total, 128);
  if (err == cudaSuccess) err = make_map(&mb1, B1, (uint64_t)K, (uint64_t)b_rows_total, 128);
  if (err == cudaSuccess && shared) {
    err = make_map(&ma2, shared->a, (uint64_t)K, (uint64_t)shared->rows, BM);
    if (err == cudaSuccess) err = make_map(&ms0, shared->b0, (uint64_t)K, (uint64_t)N, 128);
    if (err == cudaSuccess) err = make_map(&ms1, shared->b1, (uint64_t)K, (uint64_t)N, 128);
  } else {
    ma2 = ma;
    ms0 = mb0;
    ms1 = mb1;
  }
  if (err != cudaSuccess) return err;
  TcParams p;
  p.offsets = offsets;
  p.E = E;
  p.rows = rows;
  p.rows_cap = rows_cap;
  p.N = N;
  p.b_stride = b_stride;
  p.K = K;
  p.mode = mode;
  p.n_tiles = mode == MODE_SWIGLU ? (N + 127) / 128 : (N + BN - 1) / BN;
  p.out = static_cast<__nv_bfloat16 *>(out);
  p.status = status;
  p.timeout_ns = wait_timeout_ns();
  p.gather = gather;
  p.shared_rows = shared ? shared->rows : 0;
  p.out2 = shared ? static_cast<__nv_bfloat16 *>(shared->out) : nullptr;
  const int nE = offsets ? E : 1;
  const long long upper = ((long long)(rows_cap + BM - 1) / BM + nE + (p.shared_rows + BM - 1) / BM) * p.n_tiles;
  const int sms = sm_count();
  const int grid = (int)(upper < sms ? upper : sms);
  err = cudaFuncSetAttribute(tc_grouped_gemm, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
  if (err != cudaSuccess) return err;
  launch_plain(tc_grouped_gemm, grid, THREADS, SMEM_BYTES, s, ma, mb0, mb1, ma2, ms0, ms1, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_ffn_tc_bf16(const FfnArgs &a, cudaStream_t s) {
  cudaError_t err;
  SharedGroup sh1{}, sh2{};
  const bool sh = a.shared_rows > 0;
  if (sh) {
    sh1 = SharedGroup{a.shared_x, a.shared_w1, a.shared_w2, a.shared_rows, a.shared_h};
    sh2 = SharedGroup{a.shared_h, a.shared_w3, a.shared_w3, a.shared_rows, a.shared_y};
  }
  if (a.act == MOE_ACT_SWIGLU)
    err = run_gemm(a.x, a.rows_cap, a.d, a.w1, a.w2, a.w_stride, a.F, MODE_SWIGLU, a.offsets, a.E, a.rows, a.h,
                   a.status, s, a.gather, a.x_rows, sh ? &sh1 : nullptr);
  else
    err = run_gemm(a.x, a.rows_cap, a.d, a.w1, a.w1, a.w_stride, a.F, MODE_RELU, a.offsets, a.E, a.rows, a.h,
                   a.status, s, a.gather, a.x_rows, sh ? &sh1 : nullptr);
  if (err != cudaSuccess) return err;
  if (a.mid_event && (err = cudaEventRecord(a.mid_event, s)) != cudaSuccess) return err;
  return run_gemm(a.h, a.rows_cap, a.F, a.w3, a.w3, a.d, a.d, MODE_PLAIN, a.offsets, a.E, a.rows, a.y,
                  a.status, s, nullptr, 0, sh ? &sh2 : nullptr);
}

}  // namespace moe
