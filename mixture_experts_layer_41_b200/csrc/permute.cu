// Dispatch: per-expert histogram, exclusive scan, in-order capacity cut,
// permutation and the gather of token rows into the expert-sorted buffer.
//
// Semantics from the "Mixture of Experts" blog: moe_layer (a slot joins its
// expert while fewer than `capacity` earlier slots hold it, else it is
// dropped) and route_and_sort / SortedRouting (rows grouped by expert,
// arrival order kept inside an expert, expert_offsets[E+1]).
//
// Three kernels, no atomics on anything order-dependent:
//  1. count: one block per 256 tokens.  Each expert gets a 256-bit mask of
//     the block's tokens that chose it (atomicOr is order-free), so a slot's
//     rank among the block's users of its expert is a prefix popcount.
//  2. scan: one block; per expert, an exclusive prefix over blocks (the
//     slot's rank base), the raw count, the capacity cut, the exclusive scan
//     over experts (offsets) and the dropped count.
//  3. scatter: one warp per slot; kept slots write perm_token / perm_w /
//     slot_row and copy the token row with 16-byte loads and stores.
#include "common.cuh"

namespace moe {
namespace {

constexpr int kWords = kPermTokens / 32;   // mask words per expert

__global__ void __launch_bounds__(kPermTokens)
count_kernel(const int32_t *ids, int T, int k, int E, int32_t *blk_counts, int32_t *local_rank,
             int *status) {
  pdl_enter();
  __shared__ uint32_t mask[kMaxExperts * kWords];
  const int tid = threadIdx.x, lane = tid & 31, word = tid >> 5;
  const int t = blockIdx.x * kPermTokens + tid;
  for (int i = tid; i < E * kWords; i += kPermTokens) mask[i] = 0u;
  __syncthreads();
  if (t < T) {
    for (int j = 0; j < k; ++j) {
      const int e = ids[(size_t)t * k + j];
      if (e < 0 || e >= E) { record_status(status, kDevBadExpertId); continue; }
      const uint32_t old = atomicOr(&mask[e * kWords + word], 1u << lane);
      if (old & (1u << lane)) record_status(status, kDevDuplicateId);
    }
  }
  __syncthreads();
  for (int e = tid; e < E; e += kPermTokens) {
    int c = 0;
#pragma unroll
    for (int w = 0; w < kWords; ++w) c += __popc(mask[e * kWords + w]);
    blk_counts[(size_t)blockIdx.x * E + e] = c;
  }
  if (t < T) {
    for (int j = 0; j < k; ++j) {
      const int e = ids[(size_t)t * k + j];
      int r = -1;
      if (e >= 0 && e < E) {
        r = __popc(mask[e * kWords + word] & ((1u << lane) - 1u));
        for (int w = 0; w < word; ++w) r += __popc(mask[e * kWords + w]);
      }
      local_rank[(size_t)t * k + j] = r;
    }
  }
}

// One block of up to 1024 threads, one thread per expert.
// counts_by_rank (nullable): [world, E] raw slot counts of every token shard
// of the same batch, in token order; the slots of expert e held by the
// shards before `rank` are the sum of rows 0..rank-1, and the capacity left
// for this shard is cap minus that.
__global__ void scan_kernel(const int32_t *blk_counts, int nb, int E, long long cap, const int32_t *counts_by_rank,
                            int rank, int32_t *blk_base, int32_t *raw_counts, int32_t *kept_counts,
                            int32_t *offsets, int32_t *dropped) {
  pdl_enter();
  __shared__ int32_t kept_s[kMaxExperts];
  __shared__ int32_t drop_s[kMaxExperts];
  const int e = threadIdx.x;
  if (e < E) {
    // exclusive prefix over the count blocks, 16 loads in flight at a time
    int run = 0;
    for (int b0 = 0; b0 < nb; b0 += 16) {
      int v[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) v[u] = b0 + u < nb ? __ldg(blk_counts + (size_t)(b0 + u) * E + e) : 0;
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        if (b0 + u < nb) blk_base[(size_t)(b0 + u) * E + e] = run;
        run += v[u];
      }
    }
    long long room = cap;
    if (cap >= 0 && counts_by_rank) {
      long long before = 0;
      for (int r = 0; r < rank; ++r) before += counts_by_rank[(size_t)r * E + e];
      room = cap - before > 0 ? cap - before : 0;
    }
    const int kept = (room >= 0 && (long long)run > room) ? (int)room : run;
    raw_counts[e] = run;
    kept_counts[e] = kept;
    kept_s[e] = kept;
    drop_s[e] = run - kept;
  }
  __syncthreads();
  if (e == 0) {
    int acc = 0, dsum = 0;
    for (int q = 0; q < E; ++q) {
      offsets[q] = acc;
      acc += kept_s[q];
      dsum += drop_s[q];
    }
    offsets[E] = acc;
    *dropped = dsum;
  }
}

template <int VEC_BYTES>
__global__ void __launch_bounds__(256)
scatter_kernel(const int32_t *ids, const float *wts, const int32_t *local_rank,
               const int32_t *blk_base, const int32_t *offsets, const int32_t *kept, int T, int k, int E,
               const char *x, size_t row_bytes, int32_t *perm_token, float *perm_w, int32_t *slot_row,
               char *x_perm) {
  pdl_enter();
  const int warp_global = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp_global >= T * k) return;
  const int t = warp_global / k;
  const int e = ids[warp_global];
  const int lr = local_rank[warp_global];
  int row = -1;
  if (e >= 0 && e < E && lr >= 0) {
    // the slot's rank among its expert's slots in token order; the capacity
    // cut kept the first kept[e] of them
    const int rank = blk_base[(size_t)(t / kPermTokens) * E + e] + lr;
    if (rank < kept[e]) row = offsets[e] + rank;
  }
  if (lane == 0) {
    slot_row[warp_global] = row;
    if (row >= 0) {
      perm_token[row] = t;
      perm_w[row] = wts ? wts[warp_global] : 0.f;
    }
  }
  if (row < 0 || x_perm == nullptr) return;
  const char *src = x + (size_t)t * row_bytes;
  char *dst = x_perm + (size_t)row * row_bytes;
  // four loads per lane in flight before their stores
  if (VEC_BYTES == 16) {
    const uint4 *s4 = reinterpret_cast<const uint4 *>(src);
    uint4 *d4 = reinterpret_cast<uint4 *>(dst);
    const size_t n = row_bytes / 16;
    for (size_t i0 = lane; i0 < n; i0 += 4 * 32) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (i0 + 32 * u < n) v[u] = __ldg(s4 + i0 + 32 * u);
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (i0 + 32 * u < n) d4[i0 + 32 * u] = v[u];
    }
  } else {
    const uint32_t *s1 = reinterpret_cast<const uint32_t *>(src);
    uint32_t *d1 = reinterpret_cast<uint32_t *>(dst);
    const size_t n = row_bytes / 4;
    for (size_t i0 = lane; i0 < n; i0 += 4 * 32) {
      uint32_t v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (i0 + 32 * u < n) v[u] = __ldg(s1 + i0 + 32 * u);
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (i0 + 32 * u < n) d1[i0 + 32 * u] = v[u];
    }
  }
}

// Expert parallelism: local expert of every received row.  The rows arrive
// grouped by source rank, and inside a source by local expert, with
// recv_counts[s][e] rows of (s, e); row i belongs to the segment whose
// prefix range holds i.  Rows past the last segment get -1.
__global__ void __launch_bounds__(256)
ep_local_ids_kernel(const int32_t *recv_counts, int nseg, int e_local, int rows, int32_t *ids) {
  pdl_enter();
  __shared__ int32_t end[kMaxExperts];      // inclusive prefix: segment q holds rows [end[q-1], end[q])
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int q = 0; q < nseg; ++q) {
      const int c = recv_counts[q];
      acc += c > 0 ? c : 0;
      end[q] = acc;
    }
  }
  __syncthreads();
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < rows; i += gridDim.x * blockDim.x) {
    int lo = 0, hi = nseg;                  // first segment with end > i
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (end[mid] > i) hi = mid; else lo = mid + 1;
    }
    ids[i] = lo < nseg ? lo % e_local : -1;
  }
}

}  // namespace

cudaError_t launch_ep_local_ids(const int32_t *recv_counts, int world, int e_local, int rows, int32_t *ids,
                                cudaStream_t s) {
  if (rows == 0) return cudaSuccess;
  const int blocks = (rows + 255) / 256 < 1024 ? (rows + 255) / 256 : 1024;
  launch_pdl(ep_local_ids_kernel, blocks, 256, 0, s, recv_counts, world * e_local, e_local, rows, ids);
  return cudaGetLastError();
}

cudaError_t launch_permute(const moe_config &c, const void *x, const int32_t *topk_ids,
                           const float *topk_w, int64_t capacity, int32_t *expert_offsets,
                           int32_t *perm_token, float *perm_w, int32_t *slot_row, void *x_perm,
                           int32_t *raw_counts, int32_t *kept_counts, int32_t *dropped,
                           int32_t *blk_counts, int32_t *blk_base, int32_t *local_rank,
                           int *status, cudaStream_t s, const int32_t *counts_by_rank, int rank) {
  const int T = c.num_tokens, k = c.top_k, E = c.num_experts;
  const int nb = perm_blocks(c);
  launch_pdl(count_kernel, nb, kPermTokens, 0, s, topk_ids, T, k, E, blk_counts, local_rank, status);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  launch_pdl(scan_kernel, 1, kMaxExperts, 0, s, blk_counts, nb, E, (long long)capacity, counts_by_rank, rank,
             blk_base, raw_counts, kept_counts, expert_offsets, dropped);
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  const size_t row_bytes = act_size(c) * (size_t)c.hidden;
  const long long warps = (long long)T * k;
  const int blocks = (int)((warps * 32 + 255) / 256);
  const bool vec16 = (row_bytes % 16) == 0;
  if (vec16)
    launch_pdl(scatter_kernel<16>, blocks, 256, 0, s, topk_ids, topk_w, local_rank, blk_base, expert_offsets,
               kept_counts, T, k, E, static_cast<const char *>(x), row_bytes, perm_token, perm_w, slot_row,
               static_cast<char *>(x_perm));
  else
    launch_pdl(scatter_kernel<4>, blocks, 256, 0, s, topk_ids, topk_w, local_rank, blk_base, expert_offsets,
               kept_counts, T, k, E, static_cast<const char *>(x), row_bytes, perm_token, perm_w, slot_row,
               static_cast<char *>(x_perm));
  return cudaGetLastError();
}

}  // namespace moe
