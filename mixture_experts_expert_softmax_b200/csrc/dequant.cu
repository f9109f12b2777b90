// dequant.cu -- FP8 E4M3 expert weights with per-block fp32 scales (the
// sub-channel quantisation of the 0.13.2 version of the page
// "tpu_inference/kernels/fused_moe/v1/kernel.py": ref_moe multiplies every
// weight, widened to f32, by the scale of its block of subc_quant_wsz
// contraction elements) expanded to bf16 for the grouped-GEMM path:
//   out[r, c] = bf16_rn(e4m3(q[r, c]) * scale[r, c / block]).
// An HBM-bound stream: 1 byte read and 2 bytes written per weight, 16 codes
// per thread and step, 16-byte loads and stores.
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "moe_internal.h"

namespace moe {
namespace {

__device__ __forceinline__ uint32_t e4m3x2_scaled_bf16x2(uint32_t two, float sc) {
  const __half2_raw r =
      __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(two & 0xffffu), __NV_E4M3);
  __half2 h;
  memcpy(&h, &r, sizeof h);
  const float2 f = __half22float2(h);
  return pack_bf16x2(f.x * sc, f.y * sc);
}

// With expert_offsets (the grouping's [E+1] row offsets), the rows of an
// expert that no token chose (rows_per_expert rows each) are skipped.
__global__ void __launch_bounds__(256)
    dequant_e4m3_kernel(const uint4 *__restrict__ q, const float *__restrict__ scale,
                        int64_t rows, int K, int block, uint4 *__restrict__ out,
                        const int32_t *__restrict__ expert_offsets, int64_t rows_per_expert) {
  grid_dep_wait();
  grid_dep_launch();
  const int kc = K / 16;  // 16-code chunks per row
  const int nb = K / block;
  const int64_t n = rows * kc;
  for (int64_t x = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; x < n;
       x += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = x / kc;
    if (expert_offsets != nullptr) {
      const int64_t e = r / rows_per_expert;
      if (__ldg(expert_offsets + e + 1) == __ldg(expert_offsets + e)) continue;
    }
    const int c = static_cast<int>(x - r * kc);
    const float sc = __ldg(scale + r * nb + (c * 16) / block);
    const uint4 v = __ldcs(q + x);
    uint4 lo, hi;
    lo.x = e4m3x2_scaled_bf16x2(v.x, sc);
    lo.y = e4m3x2_scaled_bf16x2(v.x >> 16, sc);
    lo.z = e4m3x2_scaled_bf16x2(v.y, sc);
    lo.w = e4m3x2_scaled_bf16x2(v.y >> 16, sc);
    hi.x = e4m3x2_scaled_bf16x2(v.z, sc);
    hi.y = e4m3x2_scaled_bf16x2(v.z >> 16, sc);
    hi.z = e4m3x2_scaled_bf16x2(v.w, sc);
    hi.w = e4m3x2_scaled_bf16x2(v.w >> 16, sc);
    out[2 * x] = lo;
    out[2 * x + 1] = hi;
  }
}

}  // namespace

cudaError_t launch_dequant_e4m3(const uint8_t *q, const float *scale, int64_t rows, int K,
                                int block, uint16_t *out, int num_sms, cudaStream_t s,
                                const StageHook &hook, const int32_t *expert_offsets,
                                int64_t rows_per_expert) {
  if (expert_offsets != nullptr && (rows_per_expert < 1 || rows % rows_per_expert != 0))
    return cudaErrorInvalidValue;
  if (K % 16 != 0 || block % 16 != 0 || K % block != 0 || rows < 1) return cudaErrorInvalidValue;
  const int64_t n = rows * (K / 16);
  const int64_t want = (n + 255) / 256;
  const int64_t cap = static_cast<int64_t>(num_sms) * 8;
  const int blocks = static_cast<int>(want < cap ? want : cap);
  hook.begin("dequant_fp8");
  cudaError_t e = launch_pdl(dequant_e4m3_kernel, dim3(blocks), dim3(256), 0, s, hook.pdl,
                             reinterpret_cast<const uint4 *>(q), scale, rows, K, block,
                             reinterpret_cast<uint4 *>(out), expert_offsets, rows_per_expert);
  return hook.end(e);
}

}  // namespace moe
