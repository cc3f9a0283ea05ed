// Grouped expert FFN in bf16 on pairs of SMs (tcgen05 cta_group::2).
//
// The same grouped matmul as ffn_tc.cu (the "Mixture-of-Experts" design doc,
// The pipeline step 3; SwiGLU per Edge0 _swiglu, ReLU per the "Mixture of
// Experts" blog), with each tile computed by a cluster of two CTAs on two SMs:
// a 256 x 256 output tile is one M = 256 MMA issued by the even CTA; each CTA
// stages its own 128 rows of A and one 128-row half of B (the gate half on
// one SM and the up half on the other for SwiGLU), so every B byte crosses
// into shared memory once per pair instead of once per SM.
//
// Per CTA pair (persistent over a static schedule of (expert, n-tile,
// m-tile pair) tiles):
//   warp 0      TMA producer in both CTAs: A (128 x 64) and the CTA's B half
//               (128 x 64) per stage, 128-byte swizzle; the copies of both
//               CTAs complete on the even CTA's stage barrier (the pair form
//               of the bulk tensor copy), which the even CTA's producer arms
//               with the bytes of both;
//   warp 1      both CTAs allocate 512 TMEM columns as a pair; the even CTA's
//               lane 0 issues tcgen05.mma.cta_group::2 (M = 256, N = 256,
//               K = 16) and commits to both CTAs' barriers at once;
//   warps 2-5   epilogue in both CTAs on their own 128 accumulator rows
//               (SwiGLU: column j with j + 128), releasing the accumulator on
//               the even CTA's barrier.
// No copy multicasts: each CTA loads only its own tiles.
//
// Every mbarrier wait is bounded by %globaltimer (2 s unless moe_set_wait_timeout_ns says otherwise); on expiry the thread
// records a status code, raises its CTA's abort flag and drains what it
// issued; both CTAs meet at the final cluster barrier and free TMEM.
#include "common.cuh"

#include <cuda.h>
#include <cudaTypedefs.h>

namespace moe {
namespace {

constexpr int BM = 128;                       // rows per CTA (256 per pair)
constexpr int BK = 64;
constexpr int BN = 256;
constexpr int STAGES = 6;
constexpr int A_BYTES = BM * BK * 2;          // 16 KiB
constexpr int B_BYTES = 128 * BK * 2;         // 16 KiB: this CTA's B half
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int THREADS = 192;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint64_t DRAIN_NS = 200000000ull;

// kind::f16, D fp32, A/B bf16 K-major, N = 256, M = 256 (pair)
constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                           ((uint32_t)(256 >> 4) << 24);

enum Mode { MODE_PLAIN = 0, MODE_RELU = 1, MODE_SWIGLU = 2 };

struct Tc2Params {
  uint64_t timeout_ns;        // bound on every barrier wait (moe_set_wait_timeout_ns)
  const int32_t *offsets;
  int E, rows, rows_cap, N, b_stride, b_rows, K, mode, n_tiles;
  __nv_bfloat16 *out;
  int *status;
};

struct Shared2 {
  uint64_t full[STAGES];     // even CTA: both CTAs' copies of a stage
  uint64_t empty[STAGES];    // every CTA: its stage is free again (pair commit)
  uint64_t acc_full[2];      // every CTA: an accumulator holds a finished tile
  uint64_t acc_empty[2];     // even CTA: both CTAs' epilogues have read it
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  int32_t off[kMaxExperts + 1];
  int32_t tile_start[kMaxExperts + 1];
};

constexpr size_t SMEM_BYTES = (size_t)STAGES * STAGE_BYTES + sizeof(Shared2) + 1024;

__device__ __forceinline__ uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// the shared::cluster address of the same variable in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t map_to_rank(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}
// arrive on a barrier given by its shared::cluster address (possibly the peer's)
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t caddr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(caddr) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
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
// pair form of the tiled copy: completes on the barrier at shared::cluster
// address `bar` (the even CTA's), data into this CTA's shared memory
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap *map, uint32_t bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], "
      "[%2];" ::"r"(dst),
      "l"((uint64_t)map), "r"(bar), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// arrive on the barrier at the same offset in both CTAs once the pair's MMAs issued so far are done
__device__ __forceinline__ void tc_commit_pair(uint64_t *bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"((uint16_t)3)
      : "memory");
}
__device__ __forceinline__ void tc_mma_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, {%5, %5, %5, %5, %5, %5, %5, %5}, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(IDESC), "r"(accum), "r"(0u));
}
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
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t *>(&v);
}
__device__ __forceinline__ float silu_f(float g) { return g / (1.f + __expf(-g)); }

struct Tile2 {
  int e, row0, n;     // row0: first row of the pair (the even CTA's m-tile)
};

// tiles: per expert, n-tiles x m-tile pairs, pairs innermost
__device__ __forceinline__ Tile2 decode_tile2(const Shared2 *st, int nE, int tile) {
  int lo = 0, hi = nE;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (st->tile_start[mid] <= tile) lo = mid; else hi = mid;
  }
  Tile2 t;
  t.e = lo;
  const int local = tile - st->tile_start[lo];
  const int cnt = st->off[lo + 1] - st->off[lo];
  const int pairs = (cnt + 2 * BM - 1) / (2 * BM);
  t.n = local / pairs;
  t.row0 = st->off[lo] + (local % pairs) * 2 * BM;
  return t;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
tc2_grouped_gemm(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB0,
                 const __grid_constant__ CUtensorMap mapB1, const Tc2Params p) {
  pdl_wait();
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t *tiles = smem_raw + pad;
  Shared2 *st = reinterpret_cast<Shared2 *>(tiles + (size_t)STAGES * STAGE_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int nE = p.offsets ? p.E : 1;
  const int cluster = blockIdx.x >> 1, n_clusters = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&st->full[s], 1);
      mbar_init(&st->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&st->acc_full[b], 1);
      mbar_init(&st->acc_empty[b], 8);          // 4 epilogue warps in each CTA
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
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&st->tmem_base)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  if (warp == 2) {
    const int n_tiles = p.n_tiles;
    const bool bad = warp_group_offsets(p.offsets, nE, p.rows, p.rows_cap, st->off, st->tile_start,
                                        [n_tiles](int cnt) { return ((cnt + 2 * BM - 1) / (2 * BM)) * n_tiles; });
    if (bad && leader && lane == 0) record_status(p.status, kDevBadOffsets);
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();                        // both CTAs' barriers and TMEM exist before any use
  tc_fence_after();
  const uint32_t tmem_base = st->tmem_base;
  const int total = st->tile_start[nE];
  const int kb_n = (p.K + BK - 1) / BK;
  volatile int *abort_flag = &st->abort_flag;
  const uint32_t full0 = map_to_rank(smem_u32(&st->full[0]), 0);        // the even CTA's stage barriers
  const uint32_t acc_empty0 = map_to_rank(smem_u32(&st->acc_empty[0]), 0);

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int tile = cluster; tile < total && ok; tile += n_clusters) {
        const Tile2 ti = decode_tile2(st, nE, tile);
        // the odd CTA's half of a pair can start past the last row of A: its
        // rows are never stored, so it loads the last in-range tile instead
        int arow = ti.row0 + (int)rank * BM;
        if (arow >= p.rows_cap) arow = p.rows_cap > BM ? p.rows_cap - BM : 0;
        int brow;
        const CUtensorMap *mb;
        if (p.mode == MODE_SWIGLU) {
          brow = ti.e * p.b_stride + ti.n * 128;      // gate rows on the even CTA, up rows on the odd one
          mb = leader ? &mapB0 : &mapB1;
        } else {
          brow = ti.e * p.b_stride + ti.n * BN + (int)rank * 128;
          mb = &mapB0;
        }
        if (brow >= p.b_rows) brow = p.b_rows > 128 ? p.b_rows - 128 : 0;   // columns past N: never stored
        for (int kb = 0; kb < kb_n; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!wait_bounded(&st->empty[s], ph ^ 1u, abort_flag, p.status, kDevTimeoutProducer, p.timeout_ns)) {
            ok = false;
            break;
          }
          uint8_t *sa = tiles + (size_t)s * STAGE_BYTES;
          const uint32_t fb = full0 + (uint32_t)(s * sizeof(uint64_t));
          if (leader) mbar_expect_tx(&st->full[s], 2 * STAGE_BYTES);
          tma_load_2d_pair(smem_u32(sa), &mapA, fb, kb * BK, arow);
          tma_load_2d_pair(smem_u32(sa + A_BYTES), mb, fb, kb * BK, brow);
        }
      }
      if (!ok) {
        if (leader) {
          const uint32_t first = it > (uint32_t)STAGES ? it - STAGES : 0u;
          for (uint32_t i = first; i < it; ++i)
            if (!wait_drain(&st->full[i % STAGES], (i / STAGES) & 1u)) record_status(p.status, kDevTimeoutDrain);
        } else {
          // the odd CTA's copies complete on the even CTA's barriers: give
          // the ones in flight time to land before this CTA can leave
          const uint64_t t0 = global_ns();
          while (global_ns() - t0 < 1000000ull) {
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    if (lane == 0 && leader) {
      uint32_t it = 0, tcount = 0;
      bool ok = true;
      for (int tile = cluster; tile < total && ok; tile += n_clusters) {
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
            tc_mma_pair(dt, da + (uint64_t)(kk * 2), db + (uint64_t)(kk * 2), (kb | kk) != 0 ? 1u : 0u);
          tc_commit_pair(&st->empty[s]);
        }
        if (!ok) break;
        tc_commit_pair(&st->acc_full[buf]);
        ++tcount;
      }
      tc_commit_pair(&st->drain);
      if (!wait_drain(&st->drain, 0u)) record_status(p.status, kDevTimeoutDrain);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int q = warp & 3;
    const int rloc = q * 32 + lane;
    uint32_t tcount = 0;
    for (int tile = cluster; tile < total; tile += n_clusters) {
      const Tile2 ti = decode_tile2(st, nE, tile);
      const uint32_t buf = tcount & 1u, use = tcount >> 1;
      if (!wait_bounded(&st->acc_full[buf], use & 1u, abort_flag, p.status, kDevTimeoutEpilogue, p.timeout_ns)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + buf * BN + ((uint32_t)(q * 32) << 16);
      const int row = ti.row0 + (int)rank * BM + rloc;
      const bool valid = row < st->off[ti.e + 1];
      __nv_bfloat16 *orow = p.out + (size_t)(valid ? row : 0) * p.N;
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
                  op[i] = pack_bf16x2(silu_f(__uint_as_float(g[a])) * __uint_as_float(u[a]),
                                      silu_f(__uint_as_float(g[a + 1])) * __uint_as_float(u[a + 1]));
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
                  float x0 = __uint_as_float(a[v * 8 + 2 * i]), x1 = __uint_as_float(a[v * 8 + 2 * i + 1]);
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
      if (lane == 0) mbar_arrive_cluster(acc_empty0 + buf * (uint32_t)sizeof(uint64_t));
      ++tcount;
    }
  }

  tc_fence_before();
  __syncthreads();
  pdl_trigger();                         // tiles done: the next kernel may be scheduled
  cluster_sync();                        // the pair's MMAs and remote arrivals are over
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TMEM_COLS)
                 : "memory");
  }
}

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

// CTA pairs that fit on the device at once (one CTA per SM; an SM left
// without a partner in its GPC takes no pair).  The static tile schedule
// assumes every launched pair is resident.
int resident_pairs() {
  static int cached = 0;
  if (cached > 0) return cached;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * (sm_count() / 2), 1, 1);
  cfg.blockDim = dim3(THREADS, 1, 1);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, tc2_grouped_gemm, &cfg) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    n = sm_count() / 2;
  }
  cached = n;
  return n;
}

cudaError_t run_gemm2(const void *A, int rows_cap, int K, const void *B0, const void *B1, int b_stride, int N,
                      int mode, const int32_t *offsets, int E, int rows, void *out, int *status, cudaStream_t s) {
  CUtensorMap ma, mb0, mb1;
  const int b_rows = ((offsets ? E : 1) - 1) * b_stride + N;
  cudaError_t err = make_map(&ma, A, (uint64_t)K, (uint64_t)rows_cap, BM);
  if (err == cudaSuccess) err = make_map(&mb0, B0, (uint64_t)K, (uint64_t)b_rows, 128);
  if (err == cudaSuccess) err = make_map(&mb1, B1, (uint64_t)K, (uint64_t)b_rows, 128);
  if (err != cudaSuccess) return err;
  Tc2Params p;
  p.offsets = offsets;
  p.E = E;
  p.rows = rows;
  p.rows_cap = rows_cap;
  p.N = N;
  p.b_stride = b_stride;
  p.b_rows = b_rows;
  p.K = K;
  p.mode = mode;
  p.n_tiles = mode == MODE_SWIGLU ? (N + 127) / 128 : (N + BN - 1) / BN;
  p.out = static_cast<__nv_bfloat16 *>(out);
  p.status = status;
  p.timeout_ns = wait_timeout_ns();
  const int nE = offsets ? E : 1;
  const long long upper = ((long long)(rows_cap + 2 * BM - 1) / (2 * BM) + nE) * p.n_tiles;
  err = cudaFuncSetAttribute(tc2_grouped_gemm, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
  if (err != cudaSuccess) return err;
  const int pairs = resident_pairs();
  const int clusters = (int)(upper < pairs ? upper : pairs);
  launch_plain(tc2_grouped_gemm, 2 * clusters, THREADS, SMEM_BYTES, s, ma, mb0, mb1, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_ffn_tc2_bf16(const FfnArgs &a, cudaStream_t s) {
  cudaError_t err;
  if (a.act == MOE_ACT_SWIGLU)
    err = run_gemm2(a.x, a.rows_cap, a.d, a.w1, a.w2, a.w_stride, a.F, MODE_SWIGLU, a.offsets, a.E, a.rows, a.h,
                    a.status, s);
  else
    err = run_gemm2(a.x, a.rows_cap, a.d, a.w1, a.w1, a.w_stride, a.F, MODE_RELU, a.offsets, a.E, a.rows, a.h,
                    a.status, s);
  if (err != cudaSuccess) return err;
  if (a.mid_event && (err = cudaEventRecord(a.mid_event, s)) != cudaSuccess) return err;
  return run_gemm2(a.h, a.rows_cap, a.F, a.w3, a.w3, a.d, a.d, MODE_PLAIN, a.offsets, a.E, a.rows, a.y, a.status, s);
}

}  // namespace moe
