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
// per-expert totals).  Also zeroes the GEMMs' counters zero[0..zero_n).
__global__ void __launch_bounds__(1024)
    permute_scan_kernel(int32_t *__restrict__ chunk_counts, int n_chunks, int E,
                        int32_t *__restrict__ expert_offsets, int *zero, int zero_n) {
  __shared__ int32_t s_warp_cnt[32];
  grid_dep_wait();
  grid_dep_launch();
  for (int x = threadIdx.x; x < zero_n; x += blockDim.x) zero[x] = 0;
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

// Grouping of up to kGroupMaxN entries inside one kernel, optionally with
// the copy of each grouped row's hidden vector into expert-sorted order
// (xs[r] = hidden[sorted_rows[r] / k]).  Every CTA computes the same stable
// counting sort in shared memory -- warp w owns a contiguous chunk of the
// entries and counts it into its own 16-bit histogram row, a scan over
// (expert, warp) turns the counts into bases, and a second pass ranks each
// warp step with __match_any_sync -- so the result equals the three-kernel
// grouping above.  CTA 0 publishes it (expert_offsets, sorted_rows, inv)
// and zeroes the GEMMs' counters zero[0..zero_n); all CTAs then copy their
// share of rows from their own copy of the permutation, with no grid-wide
// synchronisation.  Only CTA 0 runs when nothing is copied.
constexpr int kGroupThreads = 1024;
constexpr int kGroupWarps = kGroupThreads / 32;
constexpr int64_t kGroupMaxN = 8192;  // above this the multi-CTA kernels are faster
constexpr int kGroupSteps = kGroupMaxN / kGroupThreads;  // 32-entry steps per warp, at most

size_t group_smem_bytes(int n, int E) {
  return static_cast<size_t>((n + 3) & ~3) * sizeof(int32_t) +
         static_cast<size_t>(E) * sizeof(int32_t) +
         static_cast<size_t>(kGroupWarps) * E * sizeof(uint16_t);
}

__global__ void __launch_bounds__(kGroupThreads)
    group_kernel(const int32_t *__restrict__ ids, int n, int E, int k,
                 int32_t *__restrict__ expert_offsets, int32_t *__restrict__ sorted_rows,
                 int32_t *__restrict__ inv, uint32_t *status, const uint4 *__restrict__ hidden,
                 int H8, uint4 *__restrict__ xs, int *zero, int zero_n) {
  extern __shared__ __align__(16) unsigned char group_smem[];
  int32_t *s_sorted = reinterpret_cast<int32_t *>(group_smem);      // [n]
  int32_t *s_tot = s_sorted + ((n + 3) & ~3);                         // [E]
  uint16_t *s_hist = reinterpret_cast<uint16_t *>(s_tot + E);         // [warps][E]
  __shared__ int32_t s_warp_tot[kGroupWarps];
  __shared__ int32_t s_nvalid;
  grid_dep_wait();
  grid_dep_launch();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool publish = blockIdx.x == 0;
  // entries of warp w: [w * per_warp, (w + 1) * per_warp), a multiple of 32
  const int per_warp = (n + kGroupThreads - 1) / kGroupThreads * 32;
  const int i0 = warp * per_warp;
  const uint32_t lt = (1u << lane) - 1u;
  for (int x = tid; x < kGroupWarps * E; x += kGroupThreads) s_hist[x] = 0;
  __syncthreads();
  uint16_t *my_hist = s_hist + warp * E;
  // the warp's ids, loaded once (per_warp <= 32 * kGroupSteps), and the
  // __match_any_sync masks of the counting pass, reused by the ranking pass
  int ev[kGroupSteps];
  uint32_t pm[kGroupSteps];
#pragma unroll
  for (int q = 0; q < kGroupSteps; ++q) {
    const int i = i0 + 32 * q + lane;
    int e = -1;
    if (32 * q < per_warp && i < n) {
      e = __ldg(ids + i);
      if (e < 0 || e >= E) e = -1;
    }
    ev[q] = e;
  }
#pragma unroll
  for (int q = 0; q < kGroupSteps; ++q) {
    if (32 * q >= per_warp) break;
    const int i = i0 + 32 * q + lane;
    const int e = ev[q];
    const uint32_t peers = __match_any_sync(0xffffffffu, e);
    pm[q] = peers;
    if (e >= 0 && (peers & lt) == 0) my_hist[e] += static_cast<uint16_t>(__popc(peers));
    if (publish && status != nullptr && __any_sync(0xffffffffu, i < n && e < 0) && lane == 0)
      atomicOr(status, kStatusBadId);
    __syncwarp();
  }
  __syncthreads();
  // per expert: a warp scans the 32 warps' counts (lane w holds warp w's),
  // leaving each warp's exclusive prefix in place and the total in s_tot
  for (int e = warp; e < E; e += kGroupWarps) {
    const int c = s_hist[lane * E + e];
    int wi = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int x = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += x;
    }
    s_hist[lane * E + e] = static_cast<uint16_t>(wi - c);
    if (lane == 31) s_tot[e] = wi;
  }
  __syncthreads();
  // exclusive scan over experts (E <= 1024: one per thread)
  const int tot = tid < E ? s_tot[tid] : 0;
  int incl = tot;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int x = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += x;
  }
  if (lane == 31) s_warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = s_warp_tot[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int x = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += x;
    }
    s_warp_tot[lane] = w;
  }
  __syncthreads();
  const int excl = incl - tot + (warp > 0 ? s_warp_tot[warp - 1] : 0);
  if (tid < E) {
    s_tot[tid] = excl;  // becomes the expert's offset
    if (publish) expert_offsets[tid] = excl;
    if (tid == E - 1) {
      s_nvalid = excl + tot;
      if (publish) expert_offsets[E] = excl + tot;
    }
  }
  __syncthreads();
  // warp prefixes -> running bases (positions < n fit 16 bits)
  for (int x = tid; x < kGroupWarps * E; x += kGroupThreads) {
    const int e = x - (x / E) * E;
    s_hist[x] = static_cast<uint16_t>(s_hist[x] + s_tot[e]);
  }
  __syncthreads();
#pragma unroll
  for (int q = 0; q < kGroupSteps; ++q) {
    if (32 * q >= per_warp) break;
    const int i = i0 + 32 * q + lane;
    const int e = ev[q];
    const uint32_t peers = pm[q];
    const int pos = e >= 0 ? my_hist[e] + __popc(peers & lt) : -1;
    __syncwarp();
    if (e >= 0 && (peers & lt) == 0) my_hist[e] += static_cast<uint16_t>(__popc(peers));
    if (pos >= 0) s_sorted[pos] = i;
    if (publish && i < n) {
      if (inv != nullptr) inv[i] = pos;
      if (pos >= 0) sorted_rows[pos] = i;
    }
    __syncwarp();
  }
  if (publish)
    for (int x = tid; x < zero_n; x += kGroupThreads) zero[x] = 0;
  if (xs == nullptr) return;
  __syncthreads();
  const int nv = s_nvalid;
  for (int r = blockIdx.x * kGroupWarps + warp; r < nv; r += gridDim.x * kGroupWarps) {
    const int64_t tok = s_sorted[r] / k;
    const uint4 *src = hidden + tok * H8;
    uint4 *dst = xs + static_cast<int64_t>(r) * H8;
#pragma unroll 8
    for (int c = lane; c < H8; c += 32) dst[c] = __ldg(src + c);
  }
}

// Copies the hidden row of every grouped (token, slot) entry into expert-
// sorted order, xs[r] = hidden[sorted_rows[r] / k], so that GEMM1 can load
// its A tiles with TMA.  One warp per row, 16-byte chunks; rows past
// expert_offsets[E] (entries with invalid ids) are not written.  Block 0
// also zeroes the GEMMs' counters zero[0..zero_n).
__global__ void __launch_bounds__(256)
    gather_rows_kernel(const uint4 *__restrict__ hidden, int H8, int k,
                       const int32_t *__restrict__ sorted_rows,
                       const int32_t *__restrict__ expert_offsets, int E,
                       uint4 *__restrict__ xs, int *zero, int zero_n) {
  grid_dep_wait();
  grid_dep_launch();
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i < zero_n; i += blockDim.x) zero[i] = 0;
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
                               uint16_t *xs, int *zero, int zero_n, cudaStream_t s,
                               const StageHook &hook) {
  const int64_t want = (n + 7) / 8;  // 8 warps per CTA, one row each per pass
  const int64_t cap = static_cast<int64_t>(num_sms) * 8;
  const int blocks = static_cast<int>(want < cap ? want : cap);
  hook.begin("gather_rows");
  cudaError_t e = launch_pdl(gather_rows_kernel, dim3(blocks > 0 ? blocks : 1), dim3(256), 0, s,
                             hook.pdl, reinterpret_cast<const uint4 *>(hidden), H / 8, k,
                             sorted_rows, expert_offsets, E, reinterpret_cast<uint4 *>(xs), zero,
                             zero_n);
  return hook.end(e);
}

int permute_num_chunks(int64_t n) { return static_cast<int>((n + kChunk - 1) / kChunk); }

bool group_supported(int64_t n) { return n <= kGroupMaxN; }

cudaError_t group_setup() {
  return cudaFuncSetAttribute(group_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(group_smem_bytes(kGroupMaxN, 1024)));
}

cudaError_t launch_group(const int32_t *ids, int64_t n, int E, int k, int32_t *expert_offsets,
                         int32_t *sorted_rows, int32_t *inv, uint32_t *status,
                         const uint16_t *hidden, int H, uint16_t *xs, int *zero, int zero_n,
                         int num_sms, cudaStream_t s, const StageHook &hook) {
  int grid = 1;
  if (xs != nullptr) {
    const int64_t want = (n + kGroupWarps - 1) / kGroupWarps;  // one row per warp
    grid = static_cast<int>(want < num_sms ? want : num_sms);
    if (grid < 1) grid = 1;
  }
  hook.begin(xs != nullptr ? "group_gather" : "permute");
  // may start under the previous kernel (it waits for it before reading ids)
  cudaError_t err = launch_pdl(group_kernel, dim3(grid), dim3(kGroupThreads),
                               group_smem_bytes(static_cast<int>(n), E), s, hook.pdl, ids,
                               static_cast<int>(n), E, k, expert_offsets, sorted_rows, inv, status,
                               reinterpret_cast<const uint4 *>(hidden), H / 8,
                               reinterpret_cast<uint4 *>(xs), zero, zero_n);
  return hook.end(err);
}

cudaError_t launch_permute(const int32_t *ids, int64_t n, int E, int32_t *chunk_counts,
                           int32_t *expert_offsets, int32_t *sorted_rows, int32_t *inv,
                           uint32_t *status, int *zero, int zero_n, cudaStream_t s,
                           const StageHook &hook) {
  const int n_chunks = permute_num_chunks(n);
  cudaError_t err;
  if (n_chunks > 0) {
    hook.begin("permute_count");
    // may start under the previous kernel (it waits for it before reading ids)
    err = launch_pdl(permute_count_kernel, dim3(n_chunks), dim3(kPermThreads),
                     static_cast<size_t>(E) * sizeof(int32_t), s, hook.pdl, ids, n, E,
                     chunk_counts);
    if ((err = hook.end(err)) != cudaSuccess) return err;
  }
  hook.begin("permute_scan");
  err = launch_pdl(permute_scan_kernel, dim3(1), dim3(1024), 0, s, hook.pdl, chunk_counts,
                   n_chunks, E, expert_offsets, zero, zero_n);
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
