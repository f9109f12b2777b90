// route.cu -- router softmax + top-k + optional renormalisation, one warp
// per token.
//
// Follows ref_moe on the page "tpu_inference/kernels/fused_moe/v1/kernel.py"
// (softmax over the experts, then top-k) and its 0.13.2 version (the k
// weights divided by their sum).  Experts are ranked by logit, which ranks
// the softmax exactly (exp is monotone); equal logits go to the lower expert
// index, as the in-kernel argmax of that page does.
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kRouteWarps = 8;

// Lane L holds experts L, L+32, L+64, ... (VPT of them) so that the row is
// read with coalesced loads.
template <int VPT>
__global__ void __launch_bounds__(kRouteWarps * 32)
    route_kernel(const float *__restrict__ logits, int64_t T, int E, int k, int renorm,
                 int32_t *__restrict__ ids, float *__restrict__ weights) {
  const int lane = threadIdx.x & 31;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * kRouteWarps + (threadIdx.x >> 5);
  // may start under the previous kernel: wait for it before reading logits
  grid_dep_wait();
  grid_dep_launch();
  if (t >= T) return;
  const float *row = logits + t * E;

  float v[VPT];
  int idx[VPT];
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int e = lane + 32 * i;
    const bool ok = e < E;
    v[i] = ok ? __ldg(row + e) : -INFINITY;
    idx[i] = ok ? e : INT_MAX;  // INT_MAX marks "not an expert" / "already taken"
  }

  // m = max over the experts
  float m = -INFINITY;
#pragma unroll
  for (int i = 0; i < VPT; ++i)
    if (idx[i] != INT_MAX) m = fmaxf(m, v[i]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));

  // s = sum over the experts of exp(l - m)
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < VPT; ++i)
    if (idx[i] != INT_MAX) s += expf(v[i] - m);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);

  // k rounds of (largest logit, lowest index) among the untaken experts;
  // slot j is written by lane j % 32, which also renormalises it
  float psum = 0.f;
  int32_t *ids_t = ids + t * k;
  float *w_t = weights + t * k;
  for (int j = 0; j < k; ++j) {
    float bv = -INFINITY;
    int bi = INT_MAX;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      if (idx[i] == INT_MAX) continue;
      if (bi == INT_MAX || v[i] > bv || (v[i] == bv && idx[i] < bi)) {
        bv = v[i];
        bi = idx[i];
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (oi != INT_MAX && (bi == INT_MAX || ov > bv || (ov == bv && oi < bi))) {
        bv = ov;
        bi = oi;
      }
    }
    // the owner of the winner marks it taken
#pragma unroll
    for (int i = 0; i < VPT; ++i)
      if (idx[i] == bi) idx[i] = INT_MAX;
    const float p = expf(bv - m) / s;
    psum += p;
    if (lane == (j & 31)) {
      ids_t[j] = bi;
      w_t[j] = p;
    }
  }
  if (renorm)
    for (int j = lane; j < k; j += 32) w_t[j] = w_t[j] / psum;
}

template <int VPT>
cudaError_t launch_route_vpt(const float *logits, int64_t T, int E, int k, int renorm,
                             int32_t *ids, float *weights, cudaStream_t s) {
  const int64_t blocks = (T + kRouteWarps - 1) / kRouteWarps;
  return launch_pdl(route_kernel<VPT>, dim3(static_cast<unsigned>(blocks)), dim3(kRouteWarps * 32),
                    0, s, true, logits, T, E, k, renorm, ids, weights);
}

}  // namespace

cudaError_t launch_route(const float *logits, int64_t T, int E, int k, int renorm, int32_t *ids,
                         float *weights, cudaStream_t s) {
  if (E <= 32) return launch_route_vpt<1>(logits, T, E, k, renorm, ids, weights, s);
  if (E <= 64) return launch_route_vpt<2>(logits, T, E, k, renorm, ids, weights, s);
  if (E <= 128) return launch_route_vpt<4>(logits, T, E, k, renorm, ids, weights, s);
  if (E <= 256) return launch_route_vpt<8>(logits, T, E, k, renorm, ids, weights, s);
  if (E <= 512) return launch_route_vpt<16>(logits, T, E, k, renorm, ids, weights, s);
  return launch_route_vpt<32>(logits, T, E, k, renorm, ids, weights, s);
}

}  // namespace moe
