// ep.cu -- the expert-parallel pieces of the fused MoE forward: the experts
// are split over `world` ranks in contiguous blocks (rank r owns experts
// [r * E / world, (r + 1) * E / world)), every rank routes its own tokens,
// sends each (token, slot) row to the owner of its expert, runs the expert
// FFNs of what it received, and gets the results back for the weighted sum.
// This is the structure of the TPU kernel on the page "tpu_inference/
// kernels/fused_moe/v1/kernel.py": per-device expert counts exchanged
// first (all_reduce_metadata), a scatter of token rows to the expert owners
// (start_a2a_scatter), the expert FFNs, a gather back to the token owner
// (start_a2a_gather) and the fixed-order sum of the k results (bt_acc).
//
// Kernels here: the owner of each expert id (for the grouping that builds
// the send order), the pack of the hidden rows into the receivers' buffers
// and the return of the expert outputs into the senders' buffers.  Both
// copies store straight into the destination buffers, which may be another
// GPU's memory mapped into this one (peer stores over NVLink); nothing here
// loads from another GPU's memory.
#include <algorithm>

#include "moe_internal.h"

namespace moe {
namespace {

// owner[i] = rank owning expert ids[i] (experts in blocks of E / world), or
// -1 when ids[i] is outside [0, E).
__global__ void __launch_bounds__(256)
    ep_owner_kernel(const int32_t *__restrict__ ids, int64_t n, int E, int world,
                    int32_t *__restrict__ owner) {
  grid_dep_wait();
  grid_dep_launch();
  const int per = E / world;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int e = __ldg(ids + i);
    owner[i] = (e >= 0 && e < E) ? e / per : -1;
  }
}

// Row r of the send order (r in [0, n_valid)): its destination d is the
// segment r falls in; it goes to row dst_row0[d] + (r - send_off[d]) of
// destination d's buffers: the hidden row of its token (bf16, H8 16-byte
// chunks) and the expert's index within d's block.  One warp per row.
__global__ void __launch_bounds__(256)
    ep_pack_kernel(const uint4 *__restrict__ hidden, int H8, const int32_t *__restrict__ ids,
                   int k, int E, int world, const int32_t *__restrict__ send_rows,
                   const __grid_constant__ EpRoutes routes) {
  grid_dep_wait();
  grid_dep_launch();
  const int lane = threadIdx.x & 31;
  const int64_t nw = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const int64_t n_valid = routes.off[world];
  const int per = E / world;
  for (int64_t r = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
       r < n_valid; r += nw) {
    int d = 0;
    while (d + 1 < world && routes.off[d + 1] <= r) ++d;
    const int64_t flat = send_rows[r];
    const int64_t q = routes.row0[d] + (r - routes.off[d]);
    const uint4 *src = hidden + (flat / k) * H8;
    uint4 *dst = reinterpret_cast<uint4 *>(routes.x[d]) + q * H8;
#pragma unroll 4
    for (int c = lane; c < H8; c += 32) dst[c] = __ldg(src + c);
    if (lane == 0) routes.eid[d][q] = __ldg(ids + flat) - d * per;
  }
}

// Received row q (in [0, n_recv)) came from source s (the segment q falls
// in); its expert output y[q] (fp32, H4 16-byte chunks) goes back to row
// dst_row0[s] + (q - recv_off[s]) of source s's buffer.  One warp per row.
__global__ void __launch_bounds__(256)
    ep_return_kernel(const float4 *__restrict__ y, int H4, int world,
                     const __grid_constant__ EpRoutes routes) {
  grid_dep_wait();
  grid_dep_launch();
  const int lane = threadIdx.x & 31;
  const int64_t nw = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const int64_t n_recv = routes.off[world];
  for (int64_t q = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
       q < n_recv; q += nw) {
    int s = 0;
    while (s + 1 < world && routes.off[s + 1] <= q) ++s;
    const int64_t row = routes.row0[s] + (q - routes.off[s]);
    const float4 *src = y + q * H4;
    float4 *dst = reinterpret_cast<float4 *>(routes.y[s]) + row * H4;
#pragma unroll 4
    for (int c = lane; c < H4; c += 32) dst[c] = __ldcs(src + c);
  }
}

int grid_for_rows(int64_t rows, int num_sms) {
  const int64_t want = (rows + 7) / 8;  // 8 warps per CTA, one row each per pass
  const int64_t cap = static_cast<int64_t>(num_sms) * 8;
  return static_cast<int>(std::max<int64_t>(1, std::min(want, cap)));
}

}  // namespace

cudaError_t launch_ep_owner(const int32_t *ids, int64_t n, int E, int world, int32_t *owner,
                            cudaStream_t s, const StageHook &hook) {
  const int64_t want = (n + 255) / 256;
  const int blocks = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(want, 4096)));
  hook.begin("ep_owner");
  cudaError_t e = launch_pdl(ep_owner_kernel, dim3(blocks), dim3(256), 0, s, hook.pdl, ids, n, E,
                             world, owner);
  return hook.end(e);
}

cudaError_t launch_ep_pack(const uint16_t *hidden, int H, const int32_t *ids, int k, int E,
                           int world, const int32_t *send_rows, const EpRoutes &routes,
                           int num_sms, cudaStream_t s, const StageHook &hook) {
  hook.begin("ep_pack");
  cudaError_t e = launch_pdl(ep_pack_kernel, dim3(grid_for_rows(routes.off[world], num_sms)),
                             dim3(256), 0, s, hook.pdl, reinterpret_cast<const uint4 *>(hidden),
                             H / 8, ids, k, E, world, send_rows, routes);
  return hook.end(e);
}

cudaError_t launch_ep_return(const float *y, int H, int world, const EpRoutes &routes,
                             int num_sms, cudaStream_t s, const StageHook &hook) {
  hook.begin("ep_return");
  cudaError_t e = launch_pdl(ep_return_kernel, dim3(grid_for_rows(routes.off[world], num_sms)),
                             dim3(256), 0, s, hook.pdl, reinterpret_cast<const float4 *>(y), H / 4,
                             world, routes);
  return hook.end(e);
}

}  // namespace moe
