// small_t.cu -- the fused MoE forward for a handful of tokens (decode).
// With T <= 16 the work is a stream over the chosen experts' weights, so it
// is written as two HBM-bound GEMV kernels with 16-byte loads instead of
// tiles for the tensor cores:
//
//   gemv1_swiglu: one CTA column per DISTINCT chosen expert e (ascending e)
//     and a slice of I; each warp streams row pairs (w1[e, i, :] gate,
//     w1[e, I+i, :] up) once and dots them with every token routed to e:
//     act[t*k + j, i] = silu(g) * u, kept in fp32.
//   gemv2_combine: each warp owns output rows h; for every token it walks
//     j = 0..k-1 in order, dots w2[id_j][h, :] with act[t*k + j, :] and
//     accumulates w_j * dot in fp32 -- the combine needs no buffer and is
//     deterministic.  Launched with programmatic dependent launch: it
//     prefetches its w2 rows into L2 while gemv1 still runs, then waits.
//
// Same function as ref_moe on the page "tpu_inference/kernels/fused_moe/v1/
// kernel.py" (per token: x.[W_gate|W_up] -> silu(gate)*up -> .W2, weighted
// sum) in the atrex-bench #009 layout (w1 [E,2I,H], w2 [E,H,I]).
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kRowsPerBlock = 16;  // gemv1: row pairs per CTA
constexpr int kMaxPairs = 256;     // T*k <= 16*16
constexpr int kTokGroup = 4;       // (token, slot) pairs dotted per pass over a weight row
constexpr int kMaxK = 16;

__device__ __forceinline__ void bf16x8_to_f32(const uint4 &v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

__device__ __forceinline__ float dot8(const uint4 &wv, const uint4 &xv, float acc) {
  float a[8], b[8];
  bf16x8_to_f32(wv, a);
  bf16x8_to_f32(xv, b);
#pragma unroll
  for (int i = 0; i < 8; ++i) acc = fmaf(a[i], b[i], acc);
  return acc;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__global__ void __launch_bounds__(kThreads)
    gemv1_swiglu_kernel(const uint4 *__restrict__ hidden, const uint4 *__restrict__ w1,
                        const int32_t *__restrict__ ids, float *__restrict__ act, int TK, int k,
                        int H, int I, int E) {
  __shared__ uint32_t bitmap[32];
  __shared__ int s_ids[kMaxPairs];
  __shared__ int s_pairs[kMaxPairs];
  __shared__ int s_expert, s_npairs;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  grid_dep_launch();
  if (threadIdx.x < 32) bitmap[threadIdx.x] = 0;
  __syncthreads();
  for (int i = threadIdx.x; i < TK; i += kThreads) {
    const int e = __ldg(ids + i);
    s_ids[i] = e;
    if (e >= 0 && e < E) atomicOr(&bitmap[e >> 5], 1u << (e & 31));
  }
  __syncthreads();
  if (warp == 0) {
    // this CTA's expert = the blockIdx.y-th set bit of the bitmap
    const uint32_t word = bitmap[lane];
    const int cnt = __popc(word);
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int x = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += x;
    }
    const int want = static_cast<int>(blockIdx.y);
    const int excl = incl - cnt;
    if (lane == 0) s_expert = -1;
    __syncwarp();
    if (want >= excl && want < incl) {
      uint32_t wbits = word;
      for (int r = want - excl; r > 0; --r) wbits &= wbits - 1;  // drop the lower set bits
      s_expert = lane * 32 + (__ffs(static_cast<int>(wbits)) - 1);
    }
    __syncwarp();
    // the flat indices routed to that expert, ascending
    const int e = s_expert;
    int n = 0;
    for (int base = 0; base < TK; base += 32) {
      const int i = base + lane;
      const bool hit = e >= 0 && i < TK && s_ids[i] == e;
      const uint32_t m = __ballot_sync(0xffffffffu, hit);
      if (hit) s_pairs[n + __popc(m & ((1u << lane) - 1u))] = i;
      n += __popc(m);
    }
    if (lane == 0) s_npairs = n;
  }
  __syncthreads();
  const int e = s_expert;
  if (e < 0) return;
  const int npairs = s_npairs;
  const int H8 = H / 8;
  const uint4 *W = w1 + static_cast<size_t>(e) * 2 * I * H8;
  for (int r = warp; r < kRowsPerBlock; r += kWarps) {
    const int i = blockIdx.x * kRowsPerBlock + r;
    if (i >= I) break;
    const uint4 *g_row = W + static_cast<size_t>(i) * H8;
    const uint4 *u_row = W + static_cast<size_t>(I + i) * H8;
    for (int p0 = 0; p0 < npairs; p0 += kTokGroup) {
      float ag[kTokGroup], au[kTokGroup];
      const uint4 *xr[kTokGroup];
#pragma unroll
      for (int q = 0; q < kTokGroup; ++q) {
        ag[q] = 0.f;
        au[q] = 0.f;
        const int pi = s_pairs[p0 + q < npairs ? p0 + q : p0];
        xr[q] = hidden + static_cast<size_t>(pi / k) * H8;
      }
#pragma unroll 4
      for (int c = lane; c < H8; c += 32) {
        const uint4 gv = __ldcs(g_row + c);
        const uint4 uv = __ldcs(u_row + c);
#pragma unroll
        for (int q = 0; q < kTokGroup; ++q) {
          const uint4 xv = __ldg(xr[q] + c);
          ag[q] = dot8(gv, xv, ag[q]);
          au[q] = dot8(uv, xv, au[q]);
        }
      }
#pragma unroll
      for (int q = 0; q < kTokGroup; ++q) {
        const float g = warp_sum(ag[q]);
        const float u = warp_sum(au[q]);
        if (lane == 0 && p0 + q < npairs)
          act[static_cast<size_t>(s_pairs[p0 + q]) * I + i] = silu_f(g) * u;
      }
    }
  }
}

// Each warp owns output row h; lanes split I in 8-element chunks.
__global__ void __launch_bounds__(kThreads)
    gemv2_combine_kernel(const uint4 *__restrict__ w2, const float4 *__restrict__ act,
                         const float *__restrict__ topk_w, const int32_t *__restrict__ ids,
                         float *__restrict__ out, int T, int k, int H, int I, int E,
                         uint32_t *status) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int h = blockIdx.x * kWarps + warp;
  const int I8 = I / 8;
  // w2 and the routing are inputs of the call, not outputs of gemv1: warm L2
  // with this warp's w2 rows before waiting for gemv1.
  if (h < H) {
    for (int t = 0; t < T; ++t)
      for (int j = 0; j < k; ++j) {
        const int e = __ldg(ids + t * k + j);
        if (e < 0 || e >= E) continue;
        const char *row = reinterpret_cast<const char *>(w2 + (static_cast<size_t>(e) * H + h) * I8);
        for (int off = lane * 128; off < I * 2; off += 32 * 128)
          asm volatile("prefetch.global.L2 [%0];" ::"l"(row + off));
      }
  }
  grid_dep_wait();
  if (h >= H) return;
  for (int t = 0; t < T; ++t) {
    float part[kMaxK];
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
      part[j] = 0.f;
      if (j < k) {
        const int e = __ldg(ids + t * k + j);
        if (e >= 0 && e < E) {
          const uint4 *wrow = w2 + (static_cast<size_t>(e) * H + h) * I8;
          const float4 *arow = act + static_cast<size_t>(t * k + j) * (I / 4);
          float acc = 0.f;
          for (int c = lane; c < I8; c += 32) {
            const uint4 wv = __ldg(wrow + c);
            const float4 a0 = __ldg(arow + 2 * c);
            const float4 a1 = __ldg(arow + 2 * c + 1);
            float wf[8];
            bf16x8_to_f32(wv, wf);
            acc = fmaf(wf[0], a0.x, acc);
            acc = fmaf(wf[1], a0.y, acc);
            acc = fmaf(wf[2], a0.z, acc);
            acc = fmaf(wf[3], a0.w, acc);
            acc = fmaf(wf[4], a1.x, acc);
            acc = fmaf(wf[5], a1.y, acc);
            acc = fmaf(wf[6], a1.z, acc);
            acc = fmaf(wf[7], a1.w, acc);
          }
          part[j] = acc;
        }
      }
    }
    float res = 0.f;
    bool bad = false;
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
      if (j < k) {
        const int e = __ldg(ids + t * k + j);
        const float d = warp_sum(part[j]);
        if (e >= 0 && e < E)
          res = fmaf(__ldg(topk_w + t * k + j), d, res);
        else
          bad = true;
      }
    }
    if (lane == 0) {
      out[static_cast<size_t>(t) * H + h] = res;
      if (bad && h == 0) atomicOr(status, kStatusBadId);
    }
  }
}

}  // namespace

cudaError_t launch_small_t(const uint16_t *hidden, const uint16_t *w1, const uint16_t *w2,
                           const float *topk_weights, const int32_t *topk_ids, float *act,
                           float *out, int64_t T, int H, int I, int E, int k, uint32_t *status,
                           cudaStream_t s, const StageHook &hook) {
  const int TK = static_cast<int>(T) * k;
  const int distinct_max = TK < E ? TK : E;
  hook.begin("gemv1_swiglu");
  // first kernel of the call: ordinary stream order after earlier work
  cudaError_t e = launch_pdl(gemv1_swiglu_kernel,
                             dim3((I + kRowsPerBlock - 1) / kRowsPerBlock, distinct_max),
                             dim3(kThreads), 0, s, false, reinterpret_cast<const uint4 *>(hidden),
                             reinterpret_cast<const uint4 *>(w1), topk_ids, act, TK, k, H, I, E);
  if ((e = hook.end(e)) != cudaSuccess) return e;
  hook.begin("gemv2_combine");
  e = launch_pdl(gemv2_combine_kernel, dim3((H + kWarps - 1) / kWarps), dim3(kThreads), 0, s,
                 hook.pdl, reinterpret_cast<const uint4 *>(w2),
                 reinterpret_cast<const float4 *>(act), topk_weights, topk_ids, out,
                 static_cast<int>(T), k, H, I, E, status);
  return hook.end(e);
}

}  // namespace moe
