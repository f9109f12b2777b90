// grouped_gemm.cu -- the two expert GEMMs of the fused MoE forward as
// persistent, warp-specialised tcgen05 kernels (sm_100a).
//
//   GEMM1 (+SwiGLU): for the rows of expert e in expert-sorted order,
//     g = x . w1[e, 0:I, :]^T, u = x . w1[e, I:2I, :]^T  (fp32 in TMEM),
//     act = silu(g) * u, stored as bf16 [rows, I].
//   GEMM2: y = act . w2[e]^T (fp32 in TMEM), stored to the per-(token, slot)
//     buffer P at row t*k + j; combine.cu then forms sum_j w_j * y_j.
// This is the expert FFN of ref_moe on the page "tpu_inference/kernels/
// fused_moe/v1/kernel.py" (gate = w1, up = w3, then act . w2) in the weight
// layout of atrex-bench #009 (w1 [E, 2I, H], w2 [E, H, I], both applied as
// F.linear, i.e. K-major).
//
// Work unit: a 128-row m-tile of one expert's rows times one n-tile (GEMM1:
// 128 act columns = 256 accumulator columns, gate and up side by side;
// GEMM2: 256 output columns).  Tiles are ordered expert-major, then n-tile,
// then m-tile, so CTAs that run together share an expert's weight tile in
// L2.  Each CTA loops over tiles with a stride of the grid size.
//
// Warp roles (288 threads):
//   warps 0-3  producers.  GEMM1: the 128 threads gather the A rows (hidden
//              rows of the tile's tokens) with 16-byte cp.async into the
//              128-byte-swizzled K-major layout, and thread 0 issues the two
//              TMA boxes of w1 (gate rows, up rows).  GEMM2: thread 0 issues
//              TMA for the act tile and the w2 tile.
//   warp 4     allocates 512 TMEM columns (two 128x256 fp32 accumulators)
//              and one thread issues tcgen05.mma (M=128, N=256, K=16).
//   warps 5-8  epilogue: tcgen05.ld of their 32-lane quarter, SwiGLU or
//              plain store, then release the accumulator.
// Pipelines: kStages smem stages (full/empty mbarriers) between producers
// and MMA; two accumulators (acc_full/acc_empty) between MMA and epilogue.
// Every wait is bounded; a wait that gives up raises the timeout bit of the
// status word and makes every role leave its loop.
#include <mutex>

#include "moe_internal.h"

namespace moe {
namespace {

constexpr int BM = kGemmTileM;  // 128 rows per tile (UMMA M)
constexpr int BK = 64;          // K per stage: one 128-byte swizzle row of bf16
constexpr int kStages = 4;
constexpr int kLag = kStages - 1;  // cp.async groups in flight before a stage is signalled
constexpr int kProducerThreads = 128;
constexpr int kMmaWarp = 4;
constexpr int kThreads = 9 * 32;
constexpr int kAccN = 256;               // UMMA N = accumulator columns per tile
constexpr int kTmemCols = 2 * kAccN;     // double-buffered accumulator
constexpr int kABytes = BM * BK * 2;     // 16 KB
constexpr int kBBytes = kAccN * BK * 2;  // 32 KB
constexpr int kMaxE = 1024;

enum { kModeGemm1 = 0, kModeGemm2 = 1 };

struct __align__(8) Bars {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

constexpr size_t kSmemBytes = 1024 + static_cast<size_t>(kStages) * (kABytes + kBBytes) +
                              sizeof(Bars) + 2 * (kMaxE + 1) * sizeof(int32_t);
static_assert(kSmemBytes <= 232448, "shared memory budget");

struct Params {
  const __nv_bfloat16 *hidden;
  const int32_t *sorted_rows;
  const int32_t *expert_offsets;
  const int32_t *tile_offsets;
  __nv_bfloat16 *act;
  float *P;
  int H, I, E, k;
  int K;                  // contraction length (H for GEMM1, I for GEMM2)
  int n_tiles_n;          // n-tiles per m-tile
  int b_rows_per_expert;  // 2I for w1, H for w2
  uint32_t *status;
  uint64_t wait_limit_ns;
};

struct Tile {
  int e, mt, nt, row0, rows;
};

// Tile t -> (expert, m-tile, n-tile).  tile_off[e] counts the m-tiles of
// experts < e, so expert e owns tiles [tile_off[e] * NT, tile_off[e+1] * NT).
__device__ __forceinline__ Tile decode_tile(int t, int NT, int E, const int32_t *tile_off,
                                            const int32_t *exp_off) {
  const int q = t / NT;
  int lo = 0, hi = E;  // tile_off[lo] <= q < tile_off[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (tile_off[mid] <= q)
      lo = mid;
    else
      hi = mid;
  }
  Tile tl;
  tl.e = lo;
  const int mt_cnt = tile_off[lo + 1] - tile_off[lo];
  const int local = t - tile_off[lo] * NT;
  tl.nt = local / mt_cnt;
  tl.mt = local - tl.nt * mt_cnt;
  tl.row0 = exp_off[lo] + tl.mt * BM;
  tl.rows = min(BM, exp_off[lo + 1] - tl.row0);
  return tl;
}

__device__ __forceinline__ void give_up(const Params &p, volatile int *abort_flag) {
  *abort_flag = 1;
  atomicOr(p.status, kStatusTimeout);
}

__device__ __forceinline__ float as_f32(uint32_t u) { return __uint_as_float(u); }

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tm_a,
                        const __grid_constant__ CUtensorMap tm_b, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *sA = smem;
  uint8_t *sB = smem + kStages * kABytes;
  Bars *bars = reinterpret_cast<Bars *>(sB + kStages * kBBytes);
  int32_t *s_tile_off = reinterpret_cast<int32_t *>(bars + 1);
  int32_t *s_exp_off = s_tile_off + (kMaxE + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->full[s], MODE == kModeGemm1 ? kProducerThreads + 1 : 1);
      mbar_init(&bars->empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&bars->acc_full[a], 1);
      mbar_init(&bars->acc_empty[a], 4);
    }
    mbar_init(&bars->drain, 1);
    bars->abort_flag = 0;
    fence_mbar_init();
    if (MODE == kModeGemm2) prefetch_tmap(&tm_a);
    prefetch_tmap(&tm_b);
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&bars->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  // Everything above overlaps the previous kernel under PDL; the routing
  // permutation (and, for GEMM2, act) is read only after this point.
  grid_dep_wait();
  grid_dep_launch();
  for (int i = threadIdx.x; i <= p.E; i += blockDim.x) {
    s_tile_off[i] = p.tile_offsets[i];
    s_exp_off[i] = p.expert_offsets[i];
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();

  const uint32_t tmem_base = bars->tmem_base;
  const int NT = p.n_tiles_n;
  const int total = s_tile_off[p.E] * NT;
  const int KB = p.K / BK;
  volatile int *abort_flag = &bars->abort_flag;
  const uint64_t limit = p.wait_limit_ns;

  if (warp < 4) {
    // ------------------------------------------------------------ producers
    if (MODE == kModeGemm1) {
      const int c = threadIdx.x & 7;      // 16-byte chunk of the 128-byte row
      const int rsub = threadIdx.x >> 3;  // rows rsub, rsub+16, ..., rsub+112
      int it = 0;
      bool stop = false;
      for (int t = blockIdx.x; t < total && !stop; t += gridDim.x) {
        const Tile tl = decode_tile(t, NT, p.E, s_tile_off, s_exp_off);
        const __nv_bfloat16 *src[8];
        uint32_t nbytes[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int r = rsub + 16 * i;
          if (r < tl.rows) {
            const int tok = p.sorted_rows[tl.row0 + r] / p.k;
            src[i] = p.hidden + static_cast<size_t>(tok) * p.H + c * 8;
            nbytes[i] = 16;
          } else {
            src[i] = p.hidden;  // zero-filled row
            nbytes[i] = 0;
          }
        }
        const int b_row = tl.e * p.b_rows_per_expert + tl.nt * (kAccN / 2);
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % kStages;
          const uint32_t ph = (it / kStages) & 1;
          if (!mbar_wait(&bars->empty[s], ph ^ 1, limit, abort_flag)) {
            give_up(p, abort_flag);
            stop = true;
            break;
          }
          if (threadIdx.x == 0) {
            mbar_arrive_expect_tx(&bars->full[s], kBBytes);
            uint8_t *b = sB + s * kBBytes;
            tma_load_2d(b, &tm_b, &bars->full[s], kb * BK, b_row);                   // gate
            tma_load_2d(b + kBBytes / 2, &tm_b, &bars->full[s], kb * BK, b_row + p.I);  // up
          }
          const uint32_t a_base = smem_addr(sA + s * kABytes);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int r = rsub + 16 * i;
            cp_async_16(a_base + r * 128 + ((c ^ (r & 7)) << 4), src[i] + kb * BK, nbytes[i]);
          }
          cp_async_commit();
          if (it >= kLag) {
            cp_async_wait_group<kLag>();
            fence_proxy_async_smem();
            mbar_arrive(&bars->full[(it - kLag) % kStages]);
          }
        }
      }
      cp_async_wait_all();
      fence_proxy_async_smem();
      for (int j = it - kLag > 0 ? it - kLag : 0; j < it; ++j) mbar_arrive(&bars->full[j % kStages]);
      if (stop && threadIdx.x == 0) {
        // let TMA copies already issued land before the CTA can exit
        const uint64_t t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 200000) {
        }
      }
    } else if (threadIdx.x == 0) {
      int it = 0;
      bool stop = false;
      for (int t = blockIdx.x; t < total && !stop; t += gridDim.x) {
        const Tile tl = decode_tile(t, NT, p.E, s_tile_off, s_exp_off);
        const int b_row = tl.e * p.b_rows_per_expert + tl.nt * kAccN;
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % kStages;
          const uint32_t ph = (it / kStages) & 1;
          if (!mbar_wait(&bars->empty[s], ph ^ 1, limit, abort_flag)) {
            give_up(p, abort_flag);
            stop = true;
            break;
          }
          mbar_arrive_expect_tx(&bars->full[s], kABytes + kBBytes);
          tma_load_2d(sA + s * kABytes, &tm_a, &bars->full[s], kb * BK, tl.row0);
          tma_load_2d(sB + s * kBBytes, &tm_b, &bars->full[s], kb * BK, b_row);
        }
      }
      if (stop) {
        const uint64_t t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 200000) {
        }
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(BM, kAccN);
      int it = 0, acc_it = 0;
      bool stop = false;
      for (int t = blockIdx.x; t < total && !stop; t += gridDim.x, ++acc_it) {
        const int a = acc_it & 1;
        const uint32_t aph = (acc_it >> 1) & 1;
        if (!mbar_wait(&bars->acc_empty[a], aph ^ 1, limit, abort_flag)) {
          give_up(p, abort_flag);
          break;
        }
        tc_fence_after_sync();
        const uint32_t d_tmem = tmem_base + a * kAccN;
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % kStages;
          const uint32_t ph = (it / kStages) & 1;
          if (!mbar_wait(&bars->full[s], ph, limit, abort_flag)) {
            give_up(p, abort_flag);
            stop = true;
            break;
          }
          tc_fence_after_sync();
          const uint64_t a_desc = smem_desc_sw128(smem_addr(sA + s * kABytes));
          const uint64_t b_desc = smem_desc_sw128(smem_addr(sB + s * kBBytes));
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            // +32 bytes of K per step, in 16-byte units of the start address
            umma_f16(d_tmem, a_desc + 2 * kk, b_desc + 2 * kk, idesc, (kb | kk) != 0);
          }
          umma_commit(&bars->empty[s]);
        }
        if (!stop) umma_commit(&bars->acc_full[a]);
      }
      // every MMA must be complete before TMEM is released
      umma_commit(&bars->drain);
      if (!mbar_wait(&bars->drain, 0, limit)) give_up(p, abort_flag);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lane quarter accessible to this warp
    const int row = q * 32 + lane;
    int acc_it = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++acc_it) {
      const int a = acc_it & 1;
      const uint32_t aph = (acc_it >> 1) & 1;
      if (!mbar_wait(&bars->acc_full[a], aph, limit, abort_flag)) {
        give_up(p, abort_flag);
        break;
      }
      tc_fence_after_sync();
      const Tile tl = decode_tile(t, NT, p.E, s_tile_off, s_exp_off);
      const bool valid = row < tl.rows;
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + a * kAccN;
      if (MODE == kModeGemm1) {
        __nv_bfloat16 *dst =
            p.act + static_cast<size_t>(tl.row0 + (valid ? row : 0)) * p.I + tl.nt * (kAccN / 2);
#pragma unroll 1
        for (int c0 = 0; c0 < kAccN / 2; c0 += 32) {
          uint32_t g[32], u[32];
          tmem_ld_32cols(tbase + c0, g);
          tmem_ld_32cols(tbase + kAccN / 2 + c0, u);
          tmem_ld_wait();
          if (valid) {
            uint32_t pk[16];
#pragma unroll
            for (int v = 0; v < 16; ++v) {
              const float a0 = silu_f(as_f32(g[2 * v])) * as_f32(u[2 * v]);
              const float a1 = silu_f(as_f32(g[2 * v + 1])) * as_f32(u[2 * v + 1]);
              pk[v] = pack_bf16x2(a0, a1);
            }
            uint4 *d4 = reinterpret_cast<uint4 *>(dst + c0);
#pragma unroll
            for (int v = 0; v < 4; ++v)
              d4[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
          }
        }
      } else {
        const int32_t flat = valid ? p.sorted_rows[tl.row0 + row] : 0;
        float *dst = p.P + static_cast<size_t>(flat) * p.H + tl.nt * kAccN;
#pragma unroll 1
        for (int c0 = 0; c0 < kAccN; c0 += 32) {
          uint32_t v[32];
          tmem_ld_32cols(tbase + c0, v);
          tmem_ld_wait();
          if (valid && tl.nt * kAccN + c0 < p.H) {
            float4 *d4 = reinterpret_cast<float4 *>(dst + c0);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              d4[i] = make_float4(as_f32(v[4 * i]), as_f32(v[4 * i + 1]), as_f32(v[4 * i + 2]),
                                  as_f32(v[4 * i + 3]));
          }
        }
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->acc_empty[a]);
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// A CTA that waits on a barrier nobody signals; exercises the bounded-wait
// failure path (see moe_debug_wait_timeout).
__global__ void wait_probe_kernel(uint32_t *status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !mbar_wait(&bar, 0, limit_ns)) atomicOr(status, kStatusTimeout);
  __syncthreads();
}

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// Row-major bf16 matrix [outer, inner] as a 2-D tensor map with a
// (64 x box_rows) box and the 128-byte swizzle.
bool make_map(CUtensorMap *m, const void *base, uint64_t inner, uint64_t outer,
              uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {inner * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(BK), box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int grid_for(const GroupedGemmArgs &a, int n_tiles_n) {
  const int64_t rows = a.T * a.k;
  const int64_t max_tiles = ((rows + BM - 1) / BM + a.E) * n_tiles_n;
  return static_cast<int>(max_tiles < a.num_sms ? max_tiles : a.num_sms);
}

Params base_params(const GroupedGemmArgs &a) {
  Params p = {};
  p.hidden = reinterpret_cast<const __nv_bfloat16 *>(a.hidden);
  p.sorted_rows = a.sorted_rows;
  p.expert_offsets = a.expert_offsets;
  p.tile_offsets = a.tile_offsets;
  p.act = reinterpret_cast<__nv_bfloat16 *>(a.act);
  p.P = a.P;
  p.H = a.H;
  p.I = a.I;
  p.E = a.E;
  p.k = a.k;
  p.status = a.status;
  p.wait_limit_ns = a.wait_limit_ns;
  return p;
}

}  // namespace

cudaError_t grouped_gemm_setup(int device) {
  static std::mutex mu;
  static uint64_t done_mask = 0;
  std::lock_guard<std::mutex> lock(mu);
  if (device >= 0 && device < 64 && (done_mask >> device) & 1) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(grouped_gemm_kernel<kModeGemm1>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kSmemBytes));
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(grouped_gemm_kernel<kModeGemm2>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(kSmemBytes));
  if (e != cudaSuccess) return e;
  if (encode_fn() == nullptr) return cudaErrorNotSupported;
  if (device >= 0 && device < 64) done_mask |= 1ull << device;
  return cudaSuccess;
}

cudaError_t launch_gemm1_swiglu(const GroupedGemmArgs &a, cudaStream_t s, const StageHook &hook) {
  CUtensorMap tm_w1;
  if (!make_map(&tm_w1, a.w1, static_cast<uint64_t>(a.H), static_cast<uint64_t>(a.E) * 2 * a.I,
                kAccN / 2))
    return cudaErrorInvalidValue;
  Params p = base_params(a);
  p.K = a.H;
  p.n_tiles_n = a.I / (kAccN / 2);
  p.b_rows_per_expert = 2 * a.I;
  hook.begin("gemm1_swiglu");
  cudaError_t e = launch_pdl(grouped_gemm_kernel<kModeGemm1>, dim3(grid_for(a, p.n_tiles_n)),
                             dim3(kThreads), kSmemBytes, s, hook.pdl, tm_w1, tm_w1, p);
  return hook.end(e);
}

cudaError_t launch_gemm2(const GroupedGemmArgs &a, cudaStream_t s, const StageHook &hook) {
  CUtensorMap tm_act, tm_w2;
  if (!make_map(&tm_act, a.act, static_cast<uint64_t>(a.I), static_cast<uint64_t>(a.T) * a.k, BM))
    return cudaErrorInvalidValue;
  if (!make_map(&tm_w2, a.w2, static_cast<uint64_t>(a.I), static_cast<uint64_t>(a.E) * a.H, kAccN))
    return cudaErrorInvalidValue;
  Params p = base_params(a);
  p.K = a.I;
  p.n_tiles_n = (a.H + kAccN - 1) / kAccN;  // H % 128 == 0: a last half tile is masked
  p.b_rows_per_expert = a.H;
  hook.begin("gemm2");
  cudaError_t e = launch_pdl(grouped_gemm_kernel<kModeGemm2>, dim3(grid_for(a, p.n_tiles_n)),
                             dim3(kThreads), kSmemBytes, s, hook.pdl, tm_act, tm_w2, p);
  return hook.end(e);
}

cudaError_t launch_wait_probe(uint32_t *status, uint64_t limit_ns, cudaStream_t s) {
  wait_probe_kernel<<<1, 32, 0, s>>>(status, limit_ns);
  return cudaGetLastError();
}

}  // namespace moe
