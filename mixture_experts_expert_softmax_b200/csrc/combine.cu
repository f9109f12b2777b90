// combine.cu -- the top-k weighted sum of ref_moe ("tpu_inference/kernels/
// fused_moe/v1/kernel.py": sum over the chosen experts of w_j * y_j) from
// the expert outputs that GEMM2 stores in expert-sorted row order:
// out[t, h] = sum_{j=0..k-1} w[t, j] * P[inv[t*k + j], h], accumulated in
// fp32 with one FMA per term in ascending j, so the result does not depend
// on scheduling.  Slots whose id is outside [0, E) have inv = -1: they are
// skipped and raise the bad-id status bit; a token with no valid slot gets a
// zero row.  HBM-bound: reads T*k*H*4 bytes of P (whole rows), writes T*H*4.
#include "moe_internal.h"

namespace moe {
namespace {

__global__ void __launch_bounds__(256)
    combine_kernel(const float4 *__restrict__ P, const int32_t *__restrict__ inv,
                   const float *__restrict__ w, float4 *__restrict__ out, int64_t T, int H4, int k,
                   uint32_t *status) {
  grid_dep_wait();
  grid_dep_launch();
  const int64_t n = T * H4;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < n;
       idx += stride) {
    const int64_t t = idx / H4;
    const int64_t h4 = idx - t * H4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    bool bad = false;
    for (int j = 0; j < k; ++j) {
      const int r = __ldg(inv + t * k + j);
      if (r < 0) {
        bad = true;
        continue;
      }
      const float wj = __ldg(w + t * k + j);
      const float4 y = __ldcs(P + static_cast<int64_t>(r) * H4 + h4);
      acc.x = fmaf(wj, y.x, acc.x);
      acc.y = fmaf(wj, y.y, acc.y);
      acc.z = fmaf(wj, y.z, acc.z);
      acc.w = fmaf(wj, y.w, acc.w);
    }
    if (bad && h4 == 0) atomicOr(status, kStatusBadId);
    out[idx] = acc;
  }
}

}  // namespace

cudaError_t launch_combine(const float *P, const int32_t *inv, const float *topk_weights,
                           float *out, int64_t T, int H, int k, uint32_t *status, cudaStream_t s,
                           const StageHook &hook) {
  const int H4 = H / 4;
  const int64_t n = T * H4;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t want = (n + 255) / 256;
  const int64_t cap = static_cast<int64_t>(sms) * 8;
  const int blocks = static_cast<int>(want < cap ? want : cap);
  hook.begin("combine");
  cudaError_t e = launch_pdl(combine_kernel, dim3(blocks > 0 ? blocks : 1), dim3(256), 0, s,
                             hook.pdl, reinterpret_cast<const float4 *>(P), inv, topk_weights,
                             reinterpret_cast<float4 *>(out), T, H4, k, status);
  return hook.end(e);
}

}  // namespace moe
