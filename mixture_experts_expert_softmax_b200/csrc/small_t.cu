// small_t.cu -- the fused MoE forward for a handful of tokens (decode).
// With T <= 16 the work is a stream over the chosen experts' weights, so it
// runs as two HBM-bound streaming GEMV kernels instead of tensor-core tiles.
// Both are persistent (one CTA per SM) and move weights with bulk async
// copies (the TMA engine) through a ring of shared-memory stages, so that
// every SM keeps tens of KB in flight without spending registers on it:
//
//   gemv1_stream: the work is (distinct chosen expert, row pair) with row
//     pair i = (w1[e, i, :] gate, w1[e, I+i, :] up); chunks of consecutive
//     row pairs of one expert are dealt round-robin to the CTAs.  A producer
//     thread streams each chunk's gate rows and up rows into a stage; eight
//     warps dot them with every token routed to e and store
//     act[t*k + j, i] = silu(g) * u in fp32.
//   gemv2_stream: each CTA owns a slice of output rows h; it prefetches its
//     w2 rows of every chosen expert into L2 and starts streaming them into
//     its stages while gemv1 still runs (programmatic dependent launch; w2
//     and the routing are inputs, only act comes from gemv1), then dots
//     each row with act[t*k + j, :] and finally forms
//     out[t, h] = sum_{j=0..k-1} w[t, j] * dot_j in fixed j order, so the
//     combine needs no buffer and is deterministic.
// The two kernels' shared-memory footprints are sized to fit on one SM
// together.  Every barrier wait is bounded.
//
// Same function as ref_moe on the page "tpu_inference/kernels/fused_moe/v1/
// kernel.py" (per token: x.[W_gate|W_up] -> silu(gate)*up -> .W2, weighted
// sum) in the atrex-bench #009 layout (w1 [E,2I,H], w2 [E,H,I]); the split
// follows the decode dispatch of "metrale_model_layers/layers/moe/
// forward_k2.rs" (gate-up, silu-down, weighted blend), with the activation
// fused into the first kernel and the blend into the second.
#include <mutex>

#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kThreads = 288;  // warp 0: producer; warps 1..8: compute
constexpr int kComputeWarps = 8;
constexpr int kMaxPairs = 256;  // T*k <= 16*16
constexpr int kStages1 = 4;
constexpr int kStages2 = 3;
constexpr uint32_t kStageBytes = 24576;

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
  uint64_t full[kStages1];
  uint64_t empty[kStages1];
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

__device__ __forceinline__ void fail(uint32_t *status, int *abort_flag) {
  *reinterpret_cast<volatile int *>(abort_flag) = 1;
  atomicOr(status, kStatusTimeout);
}

__global__ void __launch_bounds__(kThreads, 1)
    gemv1_stream_kernel(const uint4 *__restrict__ hidden, const char *__restrict__ w1,
                        const int32_t *__restrict__ ids, float *__restrict__ act, int TK, int k,
                        int H, int I, int E, int rp, uint32_t *status, uint64_t limit) {
  extern __shared__ __align__(128) uint8_t ring[];
  __shared__ Lists L;
  __shared__ Pipe pipe;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // gemv2 may start its prologue (w2 prefetch) right away
  grid_dep_launch();
  if (warp == 0) build_lists(L, ids, TK, E);
  if (threadIdx.x == 32) {
    for (int s = 0; s < kStages1; ++s) {
      mbar_init(&pipe.full[s], 1);
      mbar_init(&pipe.empty[s], kComputeWarps);
    }
    pipe.abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const int nd = L.n_distinct;
  const int cpe = (I + rp - 1) / rp;  // chunks per expert
  const int NC = nd * cpe;
  const size_t row_bytes = static_cast<size_t>(H) * 2;
  const uint32_t stage_bytes = static_cast<uint32_t>(2 * rp * row_bytes);

  if (warp == 0) {
    if (lane == 0) {
      int it = 0;
      for (int c = blockIdx.x; c < NC; c += gridDim.x, ++it) {
        const int s = it % kStages1;
        const uint32_t ph = (it / kStages1) & 1;
        if (!mbar_wait(&pipe.empty[s], ph ^ 1, limit, &pipe.abort_flag)) {
          fail(status, &pipe.abort_flag);
          break;
        }
        const int d = c / cpe, i0 = (c - d * cpe) * rp;
        const int nr = min(rp, I - i0);
        const int e = L.dexp[d];
        const uint32_t bytes = static_cast<uint32_t>(nr * row_bytes);
        uint8_t *stage = ring + static_cast<size_t>(s) * stage_bytes;
        const char *g = w1 + (static_cast<size_t>(e) * 2 * I + i0) * row_bytes;
        const char *u = w1 + (static_cast<size_t>(e) * 2 * I + I + i0) * row_bytes;
        mbar_arrive_expect_tx(&pipe.full[s], 2 * bytes);
        bulk_load(stage, g, bytes, &pipe.full[s]);
        bulk_load(stage + rp * row_bytes, u, bytes, &pipe.full[s]);
      }
    }
  } else {
    const int cw = warp - 1;
    const int H8 = H / 8;
    int it = 0;
    int task_base = 0;  // tasks of earlier chunks: spreads each chunk's tasks over all warps
    for (int c = blockIdx.x; c < NC; c += gridDim.x, ++it) {
      const int s = it % kStages1;
      const uint32_t ph = (it / kStages1) & 1;
      if (!mbar_wait(&pipe.full[s], ph, limit, &pipe.abort_flag)) {
        if (lane == 0) fail(status, &pipe.abort_flag);
        break;
      }
      const int d = c / cpe, i0 = (c - d * cpe) * rp;
      const int nr = min(rp, I - i0);
      const int p0 = L.dstart[d], np = L.dstart[d + 1] - p0;
      const uint8_t *stage = ring + static_cast<size_t>(s) * stage_bytes;
      const int ntask = nr * np;
      for (int task = (cw - task_base % kComputeWarps + kComputeWarps) % kComputeWarps;
           task < ntask; task += kComputeWarps) {
        const int r = task / np;
        const int pair = L.plist[p0 + task - r * np];
        const uint4 *g = reinterpret_cast<const uint4 *>(stage + r * row_bytes);
        const uint4 *u = reinterpret_cast<const uint4 *>(stage + (rp + r) * row_bytes);
        const uint4 *x = hidden + static_cast<size_t>(pair / k) * H8;
        float ag = 0.f, au = 0.f;
#pragma unroll 4
        for (int c8 = lane; c8 < H8; c8 += 32) {
          float xf[8], gf[8], uf[8];
          bf16x8_to_f32(__ldg(x + c8), xf);
          bf16x8_to_f32(g[c8], gf);
          bf16x8_to_f32(u[c8], uf);
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            ag = fmaf(gf[q], xf[q], ag);
            au = fmaf(uf[q], xf[q], au);
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
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kThreads, 1)
    gemv2_stream_kernel(const char *__restrict__ w2, const float4 *__restrict__ act,
                        const float *__restrict__ topk_w, const int32_t *__restrict__ ids,
                        float *__restrict__ out, int T, int k, int H, int I, int E,
                        int rows_per_cta, int hr, uint32_t *status, uint64_t limit) {
  extern __shared__ __align__(128) uint8_t ring[];
  __shared__ Lists L;
  __shared__ Pipe pipe;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int TK = T * k;
  const int h0 = blockIdx.x * rows_per_cta;
  const int h1 = min(H, h0 + rows_per_cta);
  const int nrows = max(0, h1 - h0);
  const size_t row_bytes = static_cast<size_t>(I) * 2;
  const uint32_t stage_bytes = static_cast<uint32_t>(hr * row_bytes);
  float *part = reinterpret_cast<float *>(ring + static_cast<size_t>(kStages2) * stage_bytes);

  if (warp == 0) build_lists(L, ids, TK, E);
  if (threadIdx.x == 32) {
    for (int s = 0; s < kStages2; ++s) {
      mbar_init(&pipe.full[s], 1);
      mbar_init(&pipe.empty[s], kComputeWarps);
    }
    pipe.abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const int nd = L.n_distinct;
  const int cpe = nrows > 0 ? (nrows + hr - 1) / hr : 0;
  const int NC = nd * cpe;

  if (warp == 0) {
    if (lane == 0 && nrows > 0) {
      // w2 does not depend on gemv1: warm L2 with this CTA's rows now
      for (int d = 0; d < nd; ++d)
        bulk_prefetch_l2(w2 + (static_cast<size_t>(L.dexp[d]) * H + h0) * row_bytes,
                         static_cast<uint32_t>(nrows * row_bytes));
      for (int c = 0, it = 0; c < NC; ++c, ++it) {
        const int s = it % kStages2;
        const uint32_t ph = (it / kStages2) & 1;
        if (!mbar_wait(&pipe.empty[s], ph ^ 1, limit, &pipe.abort_flag)) {
          fail(status, &pipe.abort_flag);
          break;
        }
        const int d = c / cpe, hs = h0 + (c - d * cpe) * hr;
        const int nr = min(hr, h1 - hs);
        const uint32_t bytes = static_cast<uint32_t>(nr * row_bytes);
        mbar_arrive_expect_tx(&pipe.full[s], bytes);
        bulk_load(ring + static_cast<size_t>(s) * stage_bytes,
                  w2 + (static_cast<size_t>(L.dexp[d]) * H + hs) * row_bytes, bytes,
                  &pipe.full[s]);
      }
    }
  } else {
    // act is written by gemv1
    grid_dep_wait();
    const int cw = warp - 1;
    const int I8 = I / 8;
    int task_base = 0;
    for (int c = 0, it = 0; c < NC; ++c, ++it) {
      const int s = it % kStages2;
      const uint32_t ph = (it / kStages2) & 1;
      if (!mbar_wait(&pipe.full[s], ph, limit, &pipe.abort_flag)) {
        if (lane == 0) fail(status, &pipe.abort_flag);
        break;
      }
      const int d = c / cpe, hs = h0 + (c - d * cpe) * hr;
      const int nr = min(hr, h1 - hs);
      const int p0 = L.dstart[d], np = L.dstart[d + 1] - p0;
      const uint8_t *stage = ring + static_cast<size_t>(s) * stage_bytes;
      const int ntask = nr * np;
      for (int task = (cw - task_base % kComputeWarps + kComputeWarps) % kComputeWarps;
           task < ntask; task += kComputeWarps) {
        const int r = task / np;
        const int pair = L.plist[p0 + task - r * np];
        const uint4 *wrow = reinterpret_cast<const uint4 *>(stage + r * row_bytes);
        const float4 *a = act + static_cast<size_t>(pair) * (I / 4);
        float acc = 0.f;
#pragma unroll 4
        for (int c8 = lane; c8 < I8; c8 += 32) {
          float wf[8];
          bf16x8_to_f32(wrow[c8], wf);
          const float4 a0 = a[2 * c8], a1 = a[2 * c8 + 1];
          acc = fmaf(wf[0], a0.x, acc);
          acc = fmaf(wf[1], a0.y, acc);
          acc = fmaf(wf[2], a0.z, acc);
          acc = fmaf(wf[3], a0.w, acc);
          acc = fmaf(wf[4], a1.x, acc);
          acc = fmaf(wf[5], a1.y, acc);
          acc = fmaf(wf[6], a1.z, acc);
          acc = fmaf(wf[7], a1.w, acc);
        }
        acc = warp_sum(acc);
        if (lane == 0) part[pair * rows_per_cta + (hs - h0) + r] = acc;
      }
      task_base += ntask;
      __syncwarp();
      if (lane == 0) mbar_arrive(&pipe.empty[s]);
    }
  }
  __syncthreads();
  // out[t, h] = sum over j in order of w[t, j] * dot_j (invalid ids skipped)
  bool bad = false;
  for (int idx = threadIdx.x; idx < T * nrows; idx += blockDim.x) {
    const int t = idx / nrows, hh = idx - t * nrows;
    float acc = 0.f;
    for (int j = 0; j < k; ++j) {
      const int pair = t * k + j;
      if (L.pd[pair] < 0) {
        bad = true;
        continue;
      }
      acc = fmaf(__ldg(topk_w + pair), part[pair * rows_per_cta + hh], acc);
    }
    out[static_cast<size_t>(t) * H + h0 + hh] = acc;
  }
  if (bad && blockIdx.x == 0) atomicOr(status, kStatusBadId);
}

struct SmallTConfig {
  int rp, hr, rows_per_cta, grid;
  size_t smem1, smem2;
};

SmallTConfig small_t_config(int H, int I, int num_sms) {
  SmallTConfig c;
  c.rp = static_cast<int>(kStageBytes / (4u * H));
  c.hr = static_cast<int>(kStageBytes / (2u * I));
  c.grid = num_sms;
  c.rows_per_cta = (H + num_sms - 1) / num_sms;
  c.smem1 = static_cast<size_t>(kStages1) * kStageBytes;
  c.smem2 = static_cast<size_t>(kStages2) * kStageBytes +
            static_cast<size_t>(kMaxPairs) * c.rows_per_cta * sizeof(float);
  return c;
}

}  // namespace

bool small_t_supported(int H, int I) {
  return 4u * static_cast<uint32_t>(H) <= kStageBytes && 2u * static_cast<uint32_t>(I) <= kStageBytes;
}

cudaError_t launch_small_t(const uint16_t *hidden, const uint16_t *w1, const uint16_t *w2,
                           const float *topk_weights, const int32_t *topk_ids, float *act,
                           float *out, int64_t T, int H, int I, int E, int k, uint32_t *status,
                           uint64_t wait_limit_ns, cudaStream_t s, const StageHook &hook) {
  static std::mutex mu;
  static uint64_t ready_mask = 0;
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  if (!small_t_supported(H, I)) return cudaErrorInvalidValue;
  const SmallTConfig cfg = small_t_config(H, I, sms);
  {
    std::lock_guard<std::mutex> lock(mu);
    if (dev >= 64 || !((ready_mask >> dev) & 1)) {
      // the largest dynamic footprint either kernel can ask for
      const int max_smem = 200 * 1024;
      e = cudaFuncSetAttribute(gemv1_stream_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               max_smem);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(gemv2_stream_kernel,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem);
      if (e != cudaSuccess) return e;
      if (dev < 64) ready_mask |= 1ull << dev;
    }
  }
  const int TK = static_cast<int>(T) * k;
  hook.begin("gemv1_swiglu");
  // first kernel of the call: ordinary stream order after earlier work
  e = launch_pdl(gemv1_stream_kernel, dim3(cfg.grid), dim3(kThreads), cfg.smem1, s, false,
                 reinterpret_cast<const uint4 *>(hidden), reinterpret_cast<const char *>(w1),
                 topk_ids, act, TK, k, H, I, E, cfg.rp, status, wait_limit_ns);
  if ((e = hook.end(e)) != cudaSuccess) return e;
  hook.begin("gemv2_combine");
  e = launch_pdl(gemv2_stream_kernel, dim3(cfg.grid), dim3(kThreads), cfg.smem2, s, hook.pdl,
                 reinterpret_cast<const char *>(w2), reinterpret_cast<const float4 *>(act),
                 topk_weights, topk_ids, out, static_cast<int>(T), k, H, I, E, cfg.rows_per_cta,
                 cfg.hr, status, wait_limit_ns);
  return hook.end(e);
}

}  // namespace moe
