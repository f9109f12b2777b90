// permute.cu -- grouping of the flat (token, slot) indices i = t*k + j by
// expert: histogram -> exclusive scan -> stable scatter.  Integer only; the
// result is unique (ascending i inside each expert), which is the (token, k)
// order in which the TPU kernel of "tpu_inference/kernels/fused_moe/v1/
// kernel.py" hands rows to each expert and the ascending token order of
// nonzero() in atrex-bench #009 Model.forward.
//
// The flat index range is cut into chunks of kChunk entries; each chunk is
// split between kPermWarps warps, kChunk / kPermWarps consecutive entries
// each.  Stability comes from (chunk, warp, lane) order: a chunk's base for
// expert e counts the entries of e in all earlier chunks, a warp's base adds
// the earlier warps of its chunk, and inside a warp step lanes are ranked
// with __match_any_sync.
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kPermWarps = 8;
constexpr int kPermThreads = kPermWarps * 32;
constexpr int kChunk = 2048;
constexpr int kPerWarp = kChunk / kPermWarps;

// counts[c * E + e] = number of entries of expert e in chunk c.
__global__ void __launch_bounds__(kPermThreads)
    permute_count_kernel(const int32_t *__restrict__ ids, int64_t n, int E,
                         int32_t *__restrict__ chunk_counts) {
  extern __shared__ int32_t hist[];
  grid_dep_wait();
  grid_dep_launch();
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * kChunk;
  for (int r = threadIdx.x; r < kChunk; r += blockDim.x) {
    const int64_t i = c0 + r;
    if (i < n) {
      const int e = __ldg(ids + i);
      if (e >= 0 && e < E) atomicAdd(&hist[e], 1);
    }
  }
  __syncthreads();
  int32_t *dst = chunk_counts + static_cast<int64_t>(blockIdx.x) * E;
  for (int e = threadIdx.x; e < E; e += blockDim.x) dst[e] = hist[e];
}

// One CTA of 1024 threads.  Turns chunk_counts into per-chunk exclusive
// bases (in place) and writes expert_offsets[E+1] (exclusive scan of the
// per-expert totals).
__global__ void __launch_bounds__(1024)
    permute_scan_kernel(int32_t *__restrict__ chunk_counts, int n_chunks, int E,
                        int32_t *__restrict__ expert_offsets) {
  __shared__ int32_t s_warp_cnt[32];
  grid_dep_wait();
  grid_dep_launch();
  const int e = threadIdx.x;
  int32_t total = 0;
  if (e < E) {
    for (int c = 0; c < n_chunks; ++c) {
      int32_t *p = chunk_counts + static_cast<int64_t>(c) * E + e;
      const int32_t x = *p;
      *p = total;
      total += x;
    }
  }
  // block-wide inclusive scan of the totals
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int32_t a = total;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t xa = __shfl_up_sync(0xffffffffu, a, o);
    if (lane >= o) a += xa;
  }
  if (lane == 31) s_warp_cnt[warp] = a;
  __syncthreads();
  if (warp == 0) {
    int32_t wa = s_warp_cnt[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t xa = __shfl_up_sync(0xffffffffu, wa, o);
      if (lane >= o) wa += xa;
    }
    s_warp_cnt[lane] = wa;
  }
  __syncthreads();
  const int32_t incl_a = a + (warp > 0 ? s_warp_cnt[warp - 1] : 0);
  if (e < E) expert_offsets[e] = incl_a - total;
  if (e == E - 1) expert_offsets[E] = incl_a;
}

// Writes sorted_rows[pos] = i for every valid entry and, when inv is given,
// its inverse inv[i] = pos (-1 for an id outside [0, E)).  Shared memory
// holds one running base per (warp, expert).  An id outside [0, E) raises
// the bad-id bit of *status when status is given.
__global__ void __launch_bounds__(kPermThreads)
    permute_scatter_kernel(const int32_t *__restrict__ ids, int64_t n, int E,
                           const int32_t *__restrict__ chunk_bases,
                           const int32_t *__restrict__ expert_offsets,
                           int32_t *__restrict__ sorted_rows, int32_t *__restrict__ inv,
                           uint32_t *status) {
  extern __shared__ int32_t wbase[];  // [kPermWarps][E]
  grid_dep_wait();
  grid_dep_launch();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int x = threadIdx.x; x < kPermWarps * E; x += blockDim.x) wbase[x] = 0;
  __syncthreads();
  const int64_t w0 = static_cast<int64_t>(blockIdx.x) * kChunk + warp * kPerWarp;
  int32_t *mine = wbase + warp * E;
  for (int r = lane; r < kPerWarp; r += 32) {
    const int64_t i = w0 + r;
    if (i < n) {
      const int e = __ldg(ids + i);
      if (e >= 0 && e < E) atomicAdd(&mine[e], 1);
    }
  }
  __syncthreads();
  const int32_t *cb = chunk_bases + static_cast<int64_t>(blockIdx.x) * E;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int32_t run = expert_offsets[e] + cb[e];
    for (int w = 0; w < kPermWarps; ++w) {
      const int32_t x = wbase[w * E + e];
      wbase[w * E + e] = run;
      run += x;
    }
  }
  __syncthreads();
  const uint32_t lt_mask = (1u << lane) - 1u;
  for (int r0 = 0; r0 < kPerWarp; r0 += 32) {
    const int64_t i = w0 + r0 + lane;
    int e = -1;
    if (i < n) {
      e = __ldg(ids + i);
      if (e < 0 || e >= E) e = -1;
    }
    const uint32_t peers = __match_any_sync(0xffffffffu, e);
    if (status != nullptr && __any_sync(0xffffffffu, i < n && e < 0) && lane == 0)
      atomicOr(status, kStatusBadId);
    int32_t pos = -1;
    if (e >= 0) {
      pos = mine[e] + __popc(peers & lt_mask);
      sorted_rows[pos] = static_cast<int32_t>(i);
    }
    if (inv != nullptr && i < n) inv[i] = pos;
    __syncwarp();
    if (e >= 0 && (peers & lt_mask) == 0) mine[e] += __popc(peers);
    __syncwarp();
  }
}

// One CTA groups the whole (token, slot) index range by expert: per-expert
// counts (warp-aggregated shared-memory atomics), an exclusive scan into
// expert_offsets, then placement with a shared-memory cursor per expert.
// Positions inside an expert follow atomic order, so the grouping is not
// stable; the fused forward does not need it to be (each row's products and
// the fixed-order combine do not depend on where a row sits), and the
// exported stable grouping uses the three kernels above.
constexpr int kFusedThreads = 1024;
constexpr int64_t kFusedMaxN = 8192;  // above this the multi-CTA kernels are faster

__global__ void __launch_bounds__(kFusedThreads)
    permute_fused_kernel(const int32_t *__restrict__ ids, int n, int E,
                         int32_t *__restrict__ expert_offsets, int32_t *__restrict__ sorted_rows,
                         int32_t *__restrict__ inv, uint32_t *status) {
  __shared__ int32_t cnt[1024];
  __shared__ int32_t warp_tot[32];
  grid_dep_wait();
  grid_dep_launch();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int e = tid; e < E; e += kFusedThreads) cnt[e] = 0;
  __syncthreads();
  const uint32_t lt = (1u << lane) - 1u;
  for (int base = 0; base < n; base += kFusedThreads) {
    const int i = base + tid;
    int e = i < n ? __ldg(ids + i) : -1;
    if (e >= E) e = -1;
    const uint32_t peers = __match_any_sync(0xffffffffu, e);
    if (e >= 0 && (peers & lt) == 0) atomicAdd(&cnt[e], __popc(peers));
  }
  __syncthreads();
  // exclusive scan of cnt[0..E) (E <= 1024 = one entry per thread)
  const int c = tid < E ? cnt[tid] : 0;
  int incl = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int x = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += x;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = warp_tot[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int x = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += x;
    }
    warp_tot[lane] = w;
  }
  __syncthreads();
  const int excl = incl - c + (warp > 0 ? warp_tot[warp - 1] : 0);
  __syncthreads();
  if (tid < E) {
    cnt[tid] = excl;  // becomes the placement cursor
    expert_offsets[tid] = excl;
  }
  if (tid == E - 1) expert_offsets[E] = excl + c;
  __syncthreads();
  for (int base = 0; base < n; base += kFusedThreads) {
    const int i = base + tid;
    int e = i < n ? __ldg(ids + i) : -1;
    if (e >= E) e = -1;
    const uint32_t peers = __match_any_sync(0xffffffffu, e);
    if (status != nullptr && __any_sync(0xffffffffu, i < n && e < 0) && lane == 0)
      atomicOr(status, kStatusBadId);
    const int leader = __ffs(static_cast<int>(peers)) - 1;
    int pos0 = 0;
    if (e >= 0 && lane == leader) pos0 = atomicAdd(&cnt[e], __popc(peers));
    pos0 = __shfl_sync(0xffffffffu, pos0, leader);
    if (i < n) {
      const int pos = e >= 0 ? pos0 + __popc(peers & lt) : -1;
      if (e >= 0) sorted_rows[pos] = i;
      inv[i] = pos;
    }
  }
}

// Copies the hidden row of every grouped (token, slot) entry into expert-
// sorted order, xs[r] = hidden[sorted_rows[r] / k], so that GEMM1 can load
// its A tiles with TMA.  One warp per row, 16-byte chunks; rows past
// expert_offsets[E] (entries with invalid ids) are not written.  Block 0
// also zeroes the fused GEMM's counters.
__global__ void __launch_bounds__(256)
    gather_rows_kernel(const uint4 *__restrict__ hidden, int H8, int k,
                       const int32_t *__restrict__ sorted_rows,
                       const int32_t *__restrict__ expert_offsets, int E,
                       uint4 *__restrict__ xs, int *ready, int n_ready, int *zero_done) {
  grid_dep_wait();
  grid_dep_launch();
  if (blockIdx.x == 0) {
    for (int i = threadIdx.x; i < n_ready; i += blockDim.x) ready[i] = 0;
    if (threadIdx.x == 0) *zero_done = 0;
  }
  const int64_t n_valid = expert_offsets[E];
  const int lane = threadIdx.x & 31;
  const int64_t nw = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t r = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
       r < n_valid; r += nw) {
    const int64_t tok = sorted_rows[r] / k;
    const uint4 *src = hidden + tok * H8;
    uint4 *dst = xs + r * H8;
#pragma unroll 8
    for (int c = lane; c < H8; c += 32) dst[c] = __ldg(src + c);
  }
}

}  // namespace

cudaError_t launch_gather_rows(const uint16_t *hidden, int H, int k, const int32_t *sorted_rows,
                               const int32_t *expert_offsets, int E, int64_t n, int num_sms,
                               uint16_t *xs, int *ready, int n_ready, int *zero_done,
                               cudaStream_t s, const StageHook &hook) {
  const int64_t want = (n + 7) / 8;  // 8 warps per CTA, one row each per pass
  const int64_t cap = static_cast<int64_t>(num_sms) * 8;
  const int blocks = static_cast<int>(want < cap ? want : cap);
  hook.begin("gather_rows");
  cudaError_t e = launch_pdl(gather_rows_kernel, dim3(blocks > 0 ? blocks : 1), dim3(256), 0, s,
                             hook.pdl, reinterpret_cast<const uint4 *>(hidden), H / 8, k,
                             sorted_rows, expert_offsets, E, reinterpret_cast<uint4 *>(xs), ready,
                             n_ready, zero_done);
  return hook.end(e);
}

int permute_num_chunks(int64_t n) { return static_cast<int>((n + kChunk - 1) / kChunk); }

bool permute_fused_supported(int64_t n) { return n <= kFusedMaxN; }

cudaError_t launch_permute_fused(const int32_t *ids, int64_t n, int E, int32_t *expert_offsets,
                                 int32_t *sorted_rows, int32_t *inv, uint32_t *status,
                                 cudaStream_t s, const StageHook &hook) {
  hook.begin("permute");
  // first kernel of the call: ordinary stream order after earlier work
  cudaError_t err = launch_pdl(permute_fused_kernel, dim3(1), dim3(kFusedThreads), 0, s, false,
                               ids, static_cast<int>(n), E, expert_offsets, sorted_rows, inv,
                               status);
  return hook.end(err);
}

cudaError_t launch_permute(const int32_t *ids, int64_t n, int E, int32_t *chunk_counts,
                           int32_t *expert_offsets, int32_t *sorted_rows, int32_t *inv,
                           uint32_t *status, cudaStream_t s, const StageHook &hook) {
  const int n_chunks = permute_num_chunks(n);
  cudaError_t err;
  if (n_chunks > 0) {
    hook.begin("permute_count");
    // first kernel of the call: ordinary stream order after earlier work
    err = launch_pdl(permute_count_kernel, dim3(n_chunks), dim3(kPermThreads),
                     static_cast<size_t>(E) * sizeof(int32_t), s, false, ids, n, E,
                     chunk_counts);
    if ((err = hook.end(err)) != cudaSuccess) return err;
  }
  hook.begin("permute_scan");
  err = launch_pdl(permute_scan_kernel, dim3(1), dim3(1024), 0, s, hook.pdl, chunk_counts,
                   n_chunks, E, expert_offsets);
  if ((err = hook.end(err)) != cudaSuccess) return err;
  if (n_chunks > 0) {
    hook.begin("permute_scatter");
    err = launch_pdl(permute_scatter_kernel, dim3(n_chunks), dim3(kPermThreads),
                     static_cast<size_t>(kPermWarps) * E * sizeof(int32_t), s, hook.pdl, ids, n,
                     E, static_cast<const int32_t *>(chunk_counts),
                     static_cast<const int32_t *>(expert_offsets), sorted_rows, inv, status);
    if ((err = hook.end(err)) != cudaSuccess) return err;
  }
  return cudaSuccess;
}

}  // namespace moe
