// moe_internal.h -- launchers of the kernels of libmoe.so (host side), used
// by moe_api.cu.  Not part of the public ABI.
#pragma once

#include <utility>

#include "common.cuh"

namespace moe {

// Hooks called around every kernel launch: profiling events, the
// synchronise-after-each-stage debug mode, and whether launches may use
// programmatic dependent launch (PDL).
struct StageHook {
  bool pdl = false;
  void *ctx = nullptr;
  void (*on_begin)(void *, const char *) = nullptr;
  cudaError_t (*on_end)(void *, cudaError_t) = nullptr;
  void begin(const char *name) const {
    if (on_begin) on_begin(ctx, name);
  }
  cudaError_t end(cudaError_t e) const { return on_end ? on_end(ctx, e) : e; }
};

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t s, bool pdl, Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// route.cu
cudaError_t launch_route(const float *logits, int64_t T, int E, int k, int renorm, int32_t *ids,
                         float *weights, cudaStream_t s);

// permute.cu
// Every grouping launcher also zeroes zero[0..zero_n), the counters of the
// GEMM launches that follow (their tile schedulers, the act readiness
// counters of the one-launch GEMM); zero may be null when zero_n is 0.
int permute_num_chunks(int64_t n);
cudaError_t launch_permute(const int32_t *ids, int64_t n, int E, int32_t *chunk_counts,
                           int32_t *expert_offsets, int32_t *sorted_rows, int32_t *inv,
                           uint32_t *status, int *zero, int zero_n, cudaStream_t s,
                           const StageHook &hook);

// Stable grouping of n <= 8192 entries in one kernel (the same result as
// launch_permute), with the expert-sorted copy of the hidden rows when xs
// is given.  group_setup raises the kernel's shared-memory limit once per
// device.
bool group_supported(int64_t n);
cudaError_t group_setup();
cudaError_t launch_group(const int32_t *ids, int64_t n, int E, int k, int32_t *expert_offsets,
                         int32_t *sorted_rows, int32_t *inv, uint32_t *status,
                         const uint16_t *hidden, int H, uint16_t *xs, int *zero, int zero_n,
                         int num_sms, cudaStream_t s, const StageHook &hook);

// Expert-sorted copy of the hidden rows, xs[r] = hidden[sorted_rows[r] / k]
// for r < expert_offsets[E] (device value); n = T*k bounds the grid.
cudaError_t launch_gather_rows(const uint16_t *hidden, int H, int k, const int32_t *sorted_rows,
                               const int32_t *expert_offsets, int E, int64_t n, int num_sms,
                               uint16_t *xs, int *zero, int zero_n, cudaStream_t s,
                               const StageHook &hook);

// grouped_gemm.cu
// Counters of the GEMM launches of one forward, in one int block that the
// grouping stage zeroes: the number of epilogue warps of the one-launch GEMM
// that have zeroed their part of out, then one act readiness counter per
// 256-row m-tile.
constexpr int kCounterZeroDone = 0;
constexpr int kCounterReady = 32;
inline int64_t fused_gemm_ready_count(int64_t n, int E) { return (n + 255) / 256 + E; }
inline int64_t gemm_counter_count(int64_t n, int E) {
  return kCounterReady + fused_gemm_ready_count(n, E);
}

struct GroupedGemmArgs {
  const uint16_t *hidden;  // [T, H] bf16
  const uint16_t *w1;      // [E, 2I, H] bf16
  const uint16_t *w2;      // [E, H, I] bf16
  const int32_t *sorted_rows;
  const int32_t *expert_offsets;
  // [T*k, H] bf16 hidden rows in expert-sorted order (launch_gather_rows),
  // or null: GEMM1 then runs on single CTAs and gathers its A rows itself
  const uint16_t *xs;
  uint16_t *act;  // [T*k, I] bf16, expert-sorted rows
  float *out;                 // [T, H] fp32
  const float *topk_weights;  // [T, k] fp32
  // null (top-k <= 2): GEMM1 zeroes out and GEMM2 adds w * y of each row
  // into it in any order; else GEMM2 writes [T*k, H] fp32 expert-sorted
  // rows here for the fixed-order combine
  float *P;
  int *counters;  // gemm_counter_count(T*k, E) ints, zero at the first GEMM launch
  // epilogue variant: activation (kAct* of common.cuh) and optional fp32
  // biases b1 [E, 2I] (gate, then up) and b2 [E, H], 16-byte aligned
  const float *b1;
  const float *b2;
  int act_kind;
  int64_t T;
  int H, I, E, k;
  int num_sms;
  uint32_t *status;
  uint64_t wait_limit_ns;
  uint64_t *timeline;  // debug timeline buffer (timeline_rec), or null
  int64_t timeline_cap;
};
cudaError_t grouped_gemm_setup(int device);
cudaError_t launch_gemm1_swiglu(const GroupedGemmArgs &a, cudaStream_t s, const StageHook &hook);
cudaError_t launch_gemm2(const GroupedGemmArgs &a, cudaStream_t s, const StageHook &hook);
// GEMM1 + SwiGLU on CTA pairs from the expert-sorted rows xs, and (with_gemm2)
// GEMM2 in the same launch.  Without it, launch_gemm2 follows.
cudaError_t launch_fused_gemm(const GroupedGemmArgs &a, bool with_gemm2, cudaStream_t s,
                              const StageHook &hook);
cudaError_t launch_wait_probe(uint32_t *status, uint64_t limit_ns, cudaStream_t s);

// combine.cu
cudaError_t launch_combine(const float *P, const int32_t *inv, const float *topk_weights,
                           float *out, int64_t T, int H, int k, uint32_t *status, cudaStream_t s,
                           const StageHook &hook);

// dequant.cu: out[r, c] = bf16(e4m3(q[r, c]) * scale[r, c / block]) for a
// [rows, K] matrix of FP8 E4M3 codes (K and block multiples of 16, block
// divides K; q and out 16-byte aligned).  With expert_offsets (device,
// [E+1]), the rows_per_expert rows of every expert without rows are skipped.
cudaError_t launch_dequant_e4m3(const uint8_t *q, const float *scale, int64_t rows, int K,
                                int block, uint16_t *out, int num_sms, cudaStream_t s,
                                const StageHook &hook, const int32_t *expert_offsets = nullptr,
                                int64_t rows_per_expert = 0);

// ep.cu: expert parallelism over `world` ranks (experts in contiguous blocks
// of E / world).  EpRoutes holds, for every peer rank, the segment offsets
// of this rank's order (off, host values copied into the kernel's
// parameters), the first row in the peer's buffer and the peer's buffers
// (device pointers, possibly another GPU's memory mapped here).
constexpr int kEpMaxWorld = 64;
struct EpRoutes {
  int64_t off[kEpMaxWorld + 1];
  int64_t row0[kEpMaxWorld];
  void *x[kEpMaxWorld];       // pack: bf16 hidden rows [rows, H]
  int32_t *eid[kEpMaxWorld];  // pack: expert index within the peer's block
  void *y[kEpMaxWorld];       // return: fp32 expert outputs [rows, H]
};
cudaError_t launch_ep_owner(const int32_t *ids, int64_t n, int E, int world, int32_t *owner,
                            cudaStream_t s, const StageHook &hook);
cudaError_t launch_ep_pack(const uint16_t *hidden, int H, const int32_t *ids, int k, int E,
                           int world, const int32_t *send_rows, const EpRoutes &routes,
                           int num_sms, cudaStream_t s, const StageHook &hook);
cudaError_t launch_ep_return(const float *y, int H, int world, const EpRoutes &routes,
                             int num_sms, cudaStream_t s, const StageHook &hook);

// small_t.cu
bool small_t_supported(int H, int I);
// *fits: whether launch_small_t can run this shape in the shared memory of
// the current device (sets the kernels up for the device on first use).
cudaError_t small_t_fits(int64_t T, int H, int I, int E, int k, bool fp8, bool *fits);
// grid_sync: a 64-bit device counter that only this launcher's kernels
// touch, 0 before the first launch (each launch advances it by its grid
// size; launches on one counter must not overlap).  act: T*k*I fp32
// scratch.
// b1, b2, act_kind: the epilogue variant, as in GroupedGemmArgs.  block == 0:
// w1 [E, 2I, H] and w2 [E, H, I] are bf16; block > 0 (a multiple of 16 that
// divides H and I): they are FP8 E4M3 codes with fp32 scales w1_scale
// [E, 2I, H / block] and w2_scale [E, H, I / block].
cudaError_t launch_small_t(const uint16_t *hidden, const void *w1, const void *w2,
                           const float *w1_scale, const float *w2_scale, int block,
                           const float *b1, const float *b2, int act_kind,
                           const float *topk_weights, const int32_t *topk_ids, float *act,
                           float *out, int64_t T, int H, int I, int E, int k, uint32_t *status,
                           unsigned long long *grid_sync, uint64_t wait_limit_ns,
                           cudaStream_t s, const StageHook &hook,
                           uint64_t *timeline = nullptr, int64_t timeline_cap = 0);

}  // namespace moe
