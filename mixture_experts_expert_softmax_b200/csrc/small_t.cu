// small_t.cu -- the fused MoE forward for a handful of tokens (decode).
// With T <= 16 the work is a stream over the chosen experts' weights, so it
// runs as one persistent, HBM-bound streaming kernel instead of tensor-core
// tiles: one CTA per SM (a cooperative launch, so all CTAs are resident),
// one producer thread that moves weights with bulk async copies (the TMA
// engine) through a ring of shared-memory stages, and eight consumer warps.
//
//   phase 1 (gate/up + SwiGLU): the work is (distinct chosen expert, row
//     pair), row pair i = (w1[e, i, :] gate, w1[e, I+i, :] up); chunks of
//     consecutive row pairs of one expert are dealt round-robin to the CTAs.
//     Consumers dot each row with every token routed to e and store
//     act[t*k + j, i] = silu(g) * u in fp32 (global memory).
//   grid barrier: every CTA has written its act values (bounded wait).
//   phase 2 (down + weighted combine): each CTA owns a slice of output rows
//     h and dots w2[e][h, :] with act[t*k + j, :] for every pair of every
//     chosen expert, then forms out[t, h] = sum_{j=0..k-1} w[t, j] * dot_j in
//     fixed j order -- deterministic, no extra buffer.
// The producer does not wait for the barrier: it keeps issuing the phase-2
// w2 rows (which depend on nothing from phase 1) as ring stages free up, so
// HBM keeps streaming while the consumers finish phase 1 and cross the
// barrier.
//
// Same function as ref_moe on the page "tpu_inference/kernels/fused_moe/v1/
// kernel.py" (per token: x.[W_gate|W_up] -> silu(gate)*up -> .W2, weighted
// sum) in the atrex-bench #009 layout (w1 [E,2I,H], w2 [E,H,I]); it follows
// the decode dispatch of "metrale_model_layers/layers/moe/forward_k2.rs"
// (gate-up, silu-down, weighted blend) with the activation fused into the
// first phase and the blend into the second.
#include <mutex>

#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kThreads = 288;  // warp 0: producer; warps 1..8: compute
constexpr int kComputeWarps = 8;
constexpr int kMaxPairs = 256;  // T*k <= 16*16
constexpr int kMaxStages = 8;
constexpr int kMaxRp = 4;     // phase 1: row pairs per chunk at most
constexpr int kRowSlots = 4;  // phase 2: rows per warp (rows per CTA <= 32)
constexpr int kMaxT = 16;     // tokens of the small-T path
constexpr int kU1 = 8;        // phase 1: 16-byte column chunks per lane per block
constexpr int kU2 = 4;        // phase 2: 16-byte column chunks per lane per block
constexpr uint32_t kStageBytes = 24576;
constexpr size_t kActCacheMax = 32768;
constexpr size_t kSmemBudgetMax = 216 * 1024;  // dynamic shared memory of the kernel, at most

struct Lists {
  uint32_t bitmap[32];
  int wpre[32];
  int ids[kMaxPairs];
  int pd[kMaxPairs];      // distinct-expert index of each pair, -1 if invalid
  int dexp[kMaxPairs];    // distinct experts, ascending
  int dstart[kMaxPairs + 1];
  int dcur[kMaxPairs];
  int plist[kMaxPairs];   // pairs grouped by distinct expert, ascending
  int n_distinct;
};

struct Pipe {
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
  int abort_flag;
};

// Warp 0 builds the distinct-expert list and the pairs of each expert.
__device__ void build_lists(Lists &L, const int32_t *ids, int TK, int E) {
  const int lane = threadIdx.x & 31;
  L.bitmap[lane] = 0;
  __syncwarp();
  for (int i = lane; i < TK; i += 32) {
    const int e = __ldg(ids + i);
    L.ids[i] = e;
    if (e >= 0 && e < E) atomicOr(&L.bitmap[e >> 5], 1u << (e & 31));
  }
  __syncwarp();
  const uint32_t word = L.bitmap[lane];
  const int cnt = __popc(word);
  int incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int x = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += x;
  }
  const int excl = incl - cnt;
  L.wpre[lane] = excl;
  uint32_t w = word;
  for (int r = excl; w != 0; ++r) {
    L.dexp[r] = lane * 32 + (__ffs(static_cast<int>(w)) - 1);
    w &= w - 1;
  }
  const int nd = __shfl_sync(0xffffffffu, incl, 31);
  if (lane == 0) L.n_distinct = nd;
  for (int d = lane; d < nd; d += 32) L.dcur[d] = 0;
  __syncwarp();
  for (int i = lane; i < TK; i += 32) {
    const int e = L.ids[i];
    int d = -1;
    if (e >= 0 && e < E)
      d = L.wpre[e >> 5] + __popc(L.bitmap[e >> 5] & ((1u << (e & 31)) - 1u));
    L.pd[i] = d;
    if (d >= 0) atomicAdd(&L.dcur[d], 1);
  }
  __syncwarp();
  if (lane == 0) {
    int run = 0;
    for (int d = 0; d < nd; ++d) {
      L.dstart[d] = run;
      run += L.dcur[d];
      L.dcur[d] = L.dstart[d];
    }
    L.dstart[nd] = run;
  }
  __syncwarp();
  const uint32_t lt = (1u << lane) - 1u;
  for (int base = 0; base < TK; base += 32) {
    const int i = base + lane;
    const int d = i < TK ? L.pd[i] : -1;
    const uint32_t peers = __match_any_sync(0xffffffffu, d);
    if (d >= 0) L.plist[L.dcur[d] + __popc(peers & lt)] = i;
    __syncwarp();
    if (d >= 0 && (peers & lt) == 0) L.dcur[d] += __popc(peers);
    __syncwarp();
  }
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4 &v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ unsigned long long ld_acquire_gpu(const unsigned long long *p) {
  unsigned long long v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

// Barrier among the 256 consumer threads (warps 1..8).
__device__ __forceinline__ void consumer_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kComputeWarps * 32) : "memory");
}

__device__ __forceinline__ void fail(uint32_t *status, int *abort_flag) {
  *reinterpret_cast<volatile int *>(abort_flag) = 1;
  atomicOr(status, kStatusTimeout);
}

// kTokens: the number of tokens, when it is 1 (decode), else kMaxT.
template <int kTokens>
__global__ void __launch_bounds__(kThreads, 1)
    small_t_kernel(const uint4 *__restrict__ hidden, const char *__restrict__ w1,
                   const char *__restrict__ w2, const float *__restrict__ topk_w,
                   const int32_t *__restrict__ ids, float *__restrict__ act,
                   float *__restrict__ out, int T, int k, int H, int I, int E, int stages, int rp,
                   int rows_per_cta, int hr, int cache_act, uint32_t *status,
                   unsigned long long *grid_sync, unsigned long long sync_target, uint64_t limit) {
  extern __shared__ __align__(128) uint8_t ring[];
  __shared__ Lists L;
  __shared__ Pipe pipe;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int TK = T * k;
  if (warp == 0) build_lists(L, ids, TK, E);
  if (threadIdx.x == 32) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&pipe.full[s], 1);
      mbar_init(&pipe.empty[s], kComputeWarps);
    }
    pipe.abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const int nd = L.n_distinct;
  const size_t row1 = static_cast<size_t>(H) * 2;  // bytes of a w1 row
  const size_t row2 = static_cast<size_t>(I) * 2;  // bytes of a w2 row
  // phase 1: chunks of rp row pairs, dealt round-robin over the grid
  const int cpe1 = (I + rp - 1) / rp;
  const int NC1 = nd * cpe1;
  const int n1 = blockIdx.x < NC1 ? (NC1 - 1 - static_cast<int>(blockIdx.x)) / gridDim.x + 1 : 0;
  // phase 2: this CTA's output rows, hr rows per chunk, for every expert
  const int h0 = blockIdx.x * rows_per_cta;
  const int nrows = max(0, min(H, h0 + rows_per_cta) - h0);
  const int cpe2 = (nrows + hr - 1) / hr;
  const int n2 = nd * cpe2;
  // act of every pair, when it is small enough to keep in shared memory
  float4 *sact = reinterpret_cast<float4 *>(ring + static_cast<size_t>(stages) * kStageBytes);

  if (warp == 0) {
    if (lane == 0) {
      for (int it = 0; it < n1 + n2; ++it) {
        const int s = it % stages;
        const uint32_t ph = (it / stages) & 1;
        if (!mbar_wait(&pipe.empty[s], ph ^ 1, limit, &pipe.abort_flag)) {
          fail(status, &pipe.abort_flag);
          break;
        }
        uint8_t *stage = ring + static_cast<size_t>(s) * kStageBytes;
        if (it < n1) {
          const int c = blockIdx.x + it * gridDim.x;
          const int d = c / cpe1, i0 = (c - d * cpe1) * rp;
          const int nr = min(rp, I - i0);
          const int e = L.dexp[d];
          const uint32_t bytes = static_cast<uint32_t>(nr * row1);
          mbar_arrive_expect_tx(&pipe.full[s], 2 * bytes);
          bulk_load(stage, w1 + (static_cast<size_t>(e) * 2 * I + i0) * row1, bytes,
                    &pipe.full[s]);
          bulk_load(stage + rp * row1, w1 + (static_cast<size_t>(e) * 2 * I + I + i0) * row1,
                    bytes, &pipe.full[s]);
        } else {
          const int c = it - n1;
          const int d = c / cpe2, hs = h0 + (c - d * cpe2) * hr;
          const int nr = min(hr, h0 + nrows - hs);
          const uint32_t bytes = static_cast<uint32_t>(nr * row2);
          mbar_arrive_expect_tx(&pipe.full[s], bytes);
          bulk_load(stage, w2 + (static_cast<size_t>(L.dexp[d]) * H + hs) * row2, bytes,
                    &pipe.full[s]);
        }
      }
    }
    __syncthreads();  // pairs with the consumers' final barrier
    return;
  }

  // ---------------------------------------------------------------- consumers
  // Phase 1: one warp per (row pair, token) task; the tasks of successive
  // chunks are dealt to the warps round-robin so that every warp stays busy
  // while chunks stream in.
  const int cw = warp - 1;
  const int H8 = H / 8, I8 = I / 8;
  int task_base = 0;
  int it = 0;
  bool stop = false;
  for (; it < n1 && !stop; ++it) {
    const int s = it % stages;
    const uint32_t ph = (it / stages) & 1;
    if (!mbar_wait(&pipe.full[s], ph, limit, &pipe.abort_flag)) {
      if (lane == 0) fail(status, &pipe.abort_flag);
      stop = true;
      break;
    }
    const int c = blockIdx.x + it * gridDim.x;
    const int d = c / cpe1, i0 = (c - d * cpe1) * rp;
    const int nr = min(rp, I - i0);
    const int p0 = L.dstart[d], np = L.dstart[d + 1] - p0;
    const uint8_t *stage = ring + static_cast<size_t>(s) * kStageBytes;
    const int ntask = nr * np;
    for (int task = (cw - task_base % kComputeWarps + kComputeWarps) % kComputeWarps;
         task < ntask; task += kComputeWarps) {
      const int r = task / np;
      const int pair = L.plist[p0 + task - r * np];
      const uint4 *g = reinterpret_cast<const uint4 *>(stage + r * row1);
      const uint4 *u = reinterpret_cast<const uint4 *>(stage + (rp + r) * row1);
      const uint4 *x = hidden + static_cast<size_t>(pair / k) * H8;
      // blocks of kU column chunks per lane: all loads of a block are in
      // flight together, each chunk has its own accumulators
      float ag = 0.f, au = 0.f;
      for (int base = 0; base < H8; base += 32 * kU1) {
        uint4 xv[kU1], gv[kU1], uv[kU1];
#pragma unroll
        for (int j = 0; j < kU1; ++j) {
          const int c8 = base + lane + 32 * j;
          if (c8 < H8) {
            xv[j] = __ldg(x + c8);
            gv[j] = g[c8];
            uv[j] = u[c8];
          }
        }
#pragma unroll
        for (int j = 0; j < kU1; ++j) {
          if (base + lane + 32 * j < H8) {
            float xf[8], gf[8], uf[8];
            bf16x8_to_f32(xv[j], xf);
            bf16x8_to_f32(gv[j], gf);
            bf16x8_to_f32(uv[j], uf);
            float pg = 0.f, pu = 0.f;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              pg = fmaf(gf[q], xf[q], pg);
              pu = fmaf(uf[q], xf[q], pu);
            }
            ag += pg;
            au += pu;
          }
        }
      }
      ag = warp_sum(ag);
      au = warp_sum(au);
      if (lane == 0) act[static_cast<size_t>(pair) * I + i0 + r] = silu_f(ag) * au;
    }
    task_base += ntask;
    __syncwarp();
    if (lane == 0) mbar_arrive(&pipe.empty[s]);
  }

  // ------------------------------------------------------------ grid barrier
  // Every CTA arrives exactly once per launch, so the counter reaches
  // sync_target = (launches so far) * gridDim when all act values are written.
  __threadfence();
  asm volatile("bar.sync 1, %0;" ::"n"(kComputeWarps * 32) : "memory");
  if (threadIdx.x == 32) {
    __threadfence();
    atomicAdd(grid_sync, 1ull);
    const uint64_t t0 = global_timer_ns();
    while (ld_acquire_gpu(grid_sync) < sync_target) {
      if (global_timer_ns() - t0 > limit) {
        fail(status, &pipe.abort_flag);
        break;
      }
    }
    __threadfence();
  }
  asm volatile("bar.sync 1, %0;" ::"n"(kComputeWarps * 32) : "memory");
  stop = stop || *reinterpret_cast<volatile int *>(&pipe.abort_flag) != 0;

  const float4 *act4 = reinterpret_cast<const float4 *>(act);
  if (cache_act && !stop) {
    // act was written by other CTAs in this launch: read it from L2
    const int n4 = TK * I / 4;
    constexpr int kU = 8;  // loads in flight per thread
    for (int x0 = threadIdx.x - 32; x0 < n4; x0 += kU * kComputeWarps * 32) {
      float4 v[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int x = x0 + u * kComputeWarps * 32;
        if (x < n4) v[u] = __ldcg(act4 + x);
      }
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int x = x0 + u * kComputeWarps * 32;
        if (x < n4) sact[x] = v[u];
      }
    }
    asm volatile("bar.sync 1, %0;" ::"n"(kComputeWarps * 32) : "memory");
    act4 = sact;
  }
  // Phase 2: warp cw owns local output rows cw + 8*rs.  For every pair of
  // each chunk's expert, each lane adds w_pair * (its slice of the dot) to a
  // per-(row, token) accumulator; one warp reduction per (row, token) at the
  // end gives out[t, h].  Terms are added in a fixed order (chunks by
  // ascending expert, then lanes by a fixed tree), so the result is
  // bit-reproducible.
  float acc[kRowSlots][kTokens];
#pragma unroll
  for (int rs = 0; rs < kRowSlots; ++rs)
#pragma unroll
    for (int tt = 0; tt < kTokens; ++tt) acc[rs][tt] = 0.f;
  for (int c = 0; c < n2 && !stop; ++c, ++it) {
    const int s = it % stages;
    const uint32_t ph = (it / stages) & 1;
    if (!mbar_wait(&pipe.full[s], ph, limit, &pipe.abort_flag)) {
      if (lane == 0) fail(status, &pipe.abort_flag);
      stop = true;
      break;
    }
    const int d = c / cpe2, hs = h0 + (c - d * cpe2) * hr;
    const int nr = min(hr, h0 + nrows - hs);
    const int p0 = L.dstart[d], np = L.dstart[d + 1] - p0;
    const uint8_t *stage = ring + static_cast<size_t>(s) * kStageBytes;
#pragma unroll
    for (int rs = 0; rs < kRowSlots; ++rs) {
      // this warp's row of the chunk, in CTA-local row numbering
      const int r = (cw + rs * kComputeWarps) - (hs - h0);
      if (r < 0 || r >= nr) continue;
      const uint4 *wrow = reinterpret_cast<const uint4 *>(stage + r * row2);
      for (int base = 0; base < I8; base += 32 * kU2) {
        uint4 wv[kU2];
#pragma unroll
        for (int j = 0; j < kU2; ++j)
          if (base + lane + 32 * j < I8) wv[j] = wrow[base + lane + 32 * j];
        for (int q = 0; q < np; ++q) {
          const int pair = L.plist[p0 + q];
          const float4 *a = act4 + static_cast<size_t>(pair) * (I / 4);
          float v = 0.f;
#pragma unroll
          for (int j = 0; j < kU2; ++j) {
            const int c8 = base + lane + 32 * j;
            if (c8 < I8) {
              const float4 a0 = cache_act ? a[2 * c8] : __ldcg(a + 2 * c8);
              const float4 a1 = cache_act ? a[2 * c8 + 1] : __ldcg(a + 2 * c8 + 1);
              float wf[8];
              bf16x8_to_f32(wv[j], wf);
              float pv = 0.f;
              pv = fmaf(wf[0], a0.x, pv);
              pv = fmaf(wf[1], a0.y, pv);
              pv = fmaf(wf[2], a0.z, pv);
              pv = fmaf(wf[3], a0.w, pv);
              pv = fmaf(wf[4], a1.x, pv);
              pv = fmaf(wf[5], a1.y, pv);
              pv = fmaf(wf[6], a1.z, pv);
              pv = fmaf(wf[7], a1.w, pv);
              v += pv;
            }
          }
          const float wp = __ldg(topk_w + pair);
          if (kTokens == 1) {
            acc[rs][0] = fmaf(wp, v, acc[rs][0]);
          } else {
            const int t = pair / k;
#pragma unroll
            for (int tt = 0; tt < kTokens; ++tt)
              if (tt == t) acc[rs][tt] = fmaf(wp, v, acc[rs][tt]);
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&pipe.empty[s]);
  }
  // out[t, h]: one warp reduction per (row, token); rows of this CTA only
  if (!stop) {
#pragma unroll
    for (int rs = 0; rs < kRowSlots; ++rs) {
      const int r = cw + rs * kComputeWarps;
#pragma unroll
      for (int tt = 0; tt < kTokens; ++tt) {
        if (tt < T && r < nrows) {
          const float v = warp_sum(acc[rs][tt]);
          if (lane == 0) out[static_cast<size_t>(tt) * H + h0 + r] = v;
        }
      }
    }
  }
  bool bad = false;
  if (threadIdx.x == 32)
    for (int i = 0; i < TK; ++i) bad = bad || L.pd[i] < 0;
  if (bad && blockIdx.x == 0) atomicOr(status, kStatusBadId);
  __syncthreads();
}

struct SmallTConfig {
  int stages, rp, hr, rows_per_cta, grid, cache_act;
  size_t smem;
};

SmallTConfig small_t_config(int TK, int H, int I, int num_sms, size_t kSmemBudget) {
  SmallTConfig c;
  c.rp = static_cast<int>(kStageBytes / (4u * H));
  if (c.rp > kMaxRp) c.rp = kMaxRp;
  c.hr = static_cast<int>(kStageBytes / (2u * I));
  if (c.hr > kRowSlots * kComputeWarps) c.hr = kRowSlots * kComputeWarps;
  c.grid = num_sms;
  c.rows_per_cta = (H + num_sms - 1) / num_sms;
  const size_t act_bytes = static_cast<size_t>(TK) * I * sizeof(float);
  c.cache_act = act_bytes + 2 * kStageBytes <= kSmemBudget && act_bytes <= kActCacheMax;
  const size_t extra = c.cache_act ? act_bytes : 0;
  const size_t fit = extra < kSmemBudget ? (kSmemBudget - extra) / kStageBytes : 0;
  c.stages = static_cast<int>(fit < static_cast<size_t>(kMaxStages) ? fit : kMaxStages);
  c.smem = static_cast<size_t>(c.stages) * kStageBytes + extra;
  return c;
}

}  // namespace

bool small_t_supported(int H, int I) {
  // a stage holds a w1 row pair and a w2 row; a CTA owns <= 32 output rows
  return H <= 4096 && 4u * static_cast<uint32_t>(H) <= kStageBytes &&
         2u * static_cast<uint32_t>(I) <= kStageBytes;
}

cudaError_t launch_small_t(const uint16_t *hidden, const uint16_t *w1, const uint16_t *w2,
                           const float *topk_weights, const int32_t *topk_ids, float *act,
                           float *out, int64_t T, int H, int I, int E, int k, uint32_t *status,
                           unsigned long long *grid_sync, unsigned long long *launches,
                           uint64_t wait_limit_ns, cudaStream_t s, const StageHook &hook) {
  static std::mutex mu;
  static uint64_t ready_mask = 0;
  static size_t budget[64] = {};
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  if (!small_t_supported(H, I) || dev >= 64) return cudaErrorInvalidValue;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!((ready_mask >> dev) & 1)) {
      // dynamic shared memory left next to the kernel's static shared memory
      int optin = 0;
      cudaFuncAttributes fa;
      e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
      if (e != cudaSuccess) return e;
      size_t b = kSmemBudgetMax;
      for (auto kern : {small_t_kernel<1>, small_t_kernel<kMaxT>}) {
        e = cudaFuncGetAttributes(&fa, kern);
        if (e != cudaSuccess) return e;
        const size_t left = static_cast<size_t>(optin) - fa.sharedSizeBytes;
        if (left < b) b = left;
      }
      for (auto kern : {small_t_kernel<1>, small_t_kernel<kMaxT>}) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(b));
        if (e != cudaSuccess) return e;
        int per_sm = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, b);
        if (e != cudaSuccess) return e;
        if (per_sm < 1) return cudaErrorCooperativeLaunchTooLarge;
      }
      budget[dev] = b;
      ready_mask |= 1ull << dev;
    }
  }
  const SmallTConfig cfg = small_t_config(static_cast<int>(T) * k, H, I, sms, budget[dev]);
  // each consumer warp owns at most kRowSlots of the CTA's output rows
  if (cfg.stages < 2 || cfg.rows_per_cta > kRowSlots * kComputeWarps || T > kMaxT)
    return cudaErrorInvalidValue;
  // every CTA adds one to the grid-sync counter per launch
  const unsigned long long target = (*launches + 1) * static_cast<unsigned long long>(cfg.grid);
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(cfg.grid);
  lc.blockDim = dim3(kThreads);
  lc.dynamicSmemBytes = cfg.smem;
  lc.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  lc.attrs = attr;
  lc.numAttrs = 1;
  hook.begin("small_t");
  e = cudaLaunchKernelEx(&lc, T == 1 ? small_t_kernel<1> : small_t_kernel<kMaxT>,
                         reinterpret_cast<const uint4 *>(hidden),
                         reinterpret_cast<const char *>(w1), reinterpret_cast<const char *>(w2),
                         topk_weights, topk_ids, act, out, static_cast<int>(T), k, H, I, E,
                         cfg.stages, cfg.rp, cfg.rows_per_cta, cfg.hr, cfg.cache_act, status,
                         grid_sync, target, wait_limit_ns);
  if (e == cudaSuccess) *launches += 1;
  return hook.end(e);
}

}  // namespace moe
