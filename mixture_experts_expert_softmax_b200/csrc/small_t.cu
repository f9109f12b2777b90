// small_t.cu -- the fused MoE forward for a handful of tokens (decode).
// With T <= 16 the work is a stream over the chosen experts' weights (tens
// of MB; the arithmetic is negligible), so it runs as one HBM-bound GEMV
// kernel on the CUDA cores: every warp streams whole weight rows with
// 128-bit loads, many rows in flight per SM, so that the loads alone keep
// HBM busy.  One cooperative launch (all CTAs resident, one per SM, 15
// compute warps and one copy warp):
//
//   phase 1 (gate/up + SwiGLU): the work items are (distinct chosen expert,
//     row i) row pairs -- gate row w1[e, i, :] and up row w1[e, I+i, :] --
//     dealt round-robin to every warp of the grid.  A warp dots both rows
//     with the vectors (staged in shared memory) of the tokens routed to e,
//     in groups of up to four, and stores act[t*k + j, i] = silu(g) * u
//     rounded to bf16 (global memory; the grouped-GEMM path keeps the same
//     intermediate in bf16) -- or the variant's activation of g + b1[e, i]
//     and u + b1[e, I + i].  Meanwhile the copy warp moves the w2 rows this
//     CTA needs in phase 2 into a ring of shared-memory slots (one chosen
//     expert per slot) with bulk copies, so w2 streams from HBM alongside
//     w1; when one expert's rows do not fit, it asks L2 to prefetch them.
//     Bulk copies can stall the issuing warp for microseconds while the copy
//     engine is busy, which is why a warp of its own issues them.
//   grid barrier: every CTA has written its act values (bounded wait).
//   phase 2 (down + weighted combine): each CTA owns a slice of output rows
//     h; a warp dots w2[e][h, :] (on chip) with act of every pair of e, one
//     pair and four rows h at a time (four independent sums); with more
//     chosen experts than slots, the copy warp refills a slot as soon as
//     every compute warp has released it.  out[t, h] = sum_{j=0..k-1}
//     w[t, j] * (dot_j + b2[e_j, h]) is summed in fixed j order (b2 only
//     when given) -- deterministic, no extra buffer.
//
// FP8 weights (the sub-channel quantisation of the 0.13.2 page): w1 and w2
// hold E4M3 codes, 16 per 16-byte chunk, converted by the hardware; each
// chunk's fp32 partial dot product is multiplied by the scale of its row
// and block before it is added, and the slots hold codes (half the bytes).
//
// Same function as ref_moe on the page "tpu_inference/kernels/fused_moe/v1/
// kernel.py" (per token: x.[W_gate|W_up] -> silu(gate)*up -> .W2, weighted
// sum) in the atrex-bench #009 layout (w1 [E,2I,H], w2 [E,H,I]); it follows
// the decode dispatch of "metrale_model_layers/layers/moe/forward_k2.rs"
// (gate-up, silu-down, weighted blend) with the activation fused into the
// first phase and the blend into the second.
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include <algorithm>
#include <mutex>

#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kWarps = 15;  // compute warps (with the copy warp, 4 warps per SM sub-partition)
constexpr int kCopyWarp = kWarps;         // issues the w2 bulk copies
constexpr int kThreads = (kWarps + 1) * 32;
constexpr int kBlocksPerSm = 1;
constexpr int kMaxPairs = 256;  // T*k <= 16*16
constexpr int kMaxT = 16;       // tokens of the small-T path
constexpr int kU2 = 4;          // phase 2: 16-byte chunks per lane per block of loads
constexpr int kR2 = 4;          // phase 2: output rows per item (independent dot products)
constexpr size_t kActCacheMax = 48 * 1024;
constexpr uint64_t kW2WaitNs = 2000000000ull;
constexpr int kMaxH = 4096;
constexpr int kMaxI = 12288;
constexpr int kMaxSlots = 16;   // w2 ring slots (one chosen expert's rows each)

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

// acc + sum over q = 0..7 of w[q] * x[q] for 8 bf16 weights and 8 bf16
// values, one fp32 FMA per term with bf16 operands (fma.rn.f32.bf16: the
// products are exact, the sum rounds once per term, as fmaf on the
// widened values would) -- no separate conversions.
__device__ __forceinline__ float fma8_bf16(const uint4 &w, const uint4 &x, float acc) {
  asm("{\n\t"
      ".reg .b16 w0, w1, w2, w3, w4, w5, w6, w7, x0, x1, x2, x3, x4, x5, x6, x7;\n\t"
      "mov.b32 {w0, w1}, %1;\n\t"
      "mov.b32 {w2, w3}, %2;\n\t"
      "mov.b32 {w4, w5}, %3;\n\t"
      "mov.b32 {w6, w7}, %4;\n\t"
      "mov.b32 {x0, x1}, %5;\n\t"
      "mov.b32 {x2, x3}, %6;\n\t"
      "mov.b32 {x4, x5}, %7;\n\t"
      "mov.b32 {x6, x7}, %8;\n\t"
      "fma.rn.f32.bf16 %0, w0, x0, %0;\n\t"
      "fma.rn.f32.bf16 %0, w1, x1, %0;\n\t"
      "fma.rn.f32.bf16 %0, w2, x2, %0;\n\t"
      "fma.rn.f32.bf16 %0, w3, x3, %0;\n\t"
      "fma.rn.f32.bf16 %0, w4, x4, %0;\n\t"
      "fma.rn.f32.bf16 %0, w5, x5, %0;\n\t"
      "fma.rn.f32.bf16 %0, w6, x6, %0;\n\t"
      "fma.rn.f32.bf16 %0, w7, x7, %0;\n\t"
      "}"
      : "+f"(acc)
      : "r"(w.x), "r"(w.y), "r"(w.z), "r"(w.w), "r"(x.x), "r"(x.y), "r"(x.z), "r"(x.w));
  return acc;
}

// Two E4M3 codes (low byte first) as floats, by the hardware conversion.
__device__ __forceinline__ float2 e4m3x2_to_float2(uint32_t two) {
  const __half2_raw r =
      __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(two & 0xffffu), __NV_E4M3);
  __half2 h;
  memcpy(&h, &r, sizeof h);
  return __half22float2(h);
}

// sum over q = 0..15 of e4m3(w[q]) * x[q] for 16 codes and 16 bf16 values
// (x0: values 0..7, x1: 8..15): fp32 FMAs into two interleaved partial
// sums (halving the dependent chain), added at the end.
__device__ __forceinline__ float dot16_e4m3_bf16(const uint4 &w, const uint4 &x0,
                                                 const uint4 &x1) {
  const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
  const uint32_t xv[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
  float s0 = 0.f, s1 = 0.f;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float2 lo = e4m3x2_to_float2(wv[q]);
    const float2 hi = e4m3x2_to_float2(wv[q] >> 16);
    s0 = fmaf(lo.x, __uint_as_float(xv[2 * q] << 16), s0);
    s1 = fmaf(lo.y, __uint_as_float(xv[2 * q] & 0xffff0000u), s1);
    s0 = fmaf(hi.x, __uint_as_float(xv[2 * q + 1] << 16), s0);
    s1 = fmaf(hi.y, __uint_as_float(xv[2 * q + 1] & 0xffff0000u), s1);
  }
  return s0 + s1;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ uint16_t bf16_bits(float v) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(v));
}

__device__ __forceinline__ unsigned long long ld_acquire_gpu(const unsigned long long *p) {
  unsigned long long v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

// Phase 1 for a group of NQ tokens (at most NQ live: nq) routed to one
// expert: the warp streams the (gate row g, up row u) pair once, dots both
// with the NQ token vectors (staged in shared memory, sx), and lane 0
// stores the activations of the group's pairs.  NQ is a template constant so that the accumulators stay
// in registers and no instruction is spent on token slots that do not
// exist; nq < NQ only wastes the predicated slots of the last group.
template <int NQ, int kU, bool kFp8>
__device__ __forceinline__ void phase1_group(const uint4 *__restrict__ g,
                                             const uint4 *__restrict__ u, const uint4 *sx,
                                             const int *plist,
                                             int nq, int k, int H8, int I, int i, float bg,
                                             float bu, bool bias, int act_kind,
                                             uint16_t *__restrict__ act, const float *sg,
                                             const float *su, int cpb) {
  const int lane = threadIdx.x & 31;
  const int HC = kFp8 ? H8 / 2 : H8;  // 16-byte weight chunks per row
  int xo[NQ];  // offsets of the token vectors (T <= 16 tokens, H8 <= 512 chunks)
#pragma unroll
  for (int q = 0; q < NQ; ++q) xo[q] = plist[q < nq ? q : 0] / k * H8;
  float ag[NQ], au[NQ];
#pragma unroll
  for (int q = 0; q < NQ; ++q) ag[q] = au[q] = 0.f;
  for (int base = 0; base < HC; base += 32 * kU) {
    uint4 gv[kU], uv[kU];
    float sgv[kU], suv[kU];  // FP8: the chunks' scales, loaded with the codes
#pragma unroll
    for (int j = 0; j < kU; ++j) {
      const int c = base + lane + 32 * j;
      if (c < HC) {
        gv[j] = __ldcs(g + c);
        uv[j] = __ldcs(u + c);
        if (kFp8) {
          sgv[j] = __ldg(sg + c / cpb);
          suv[j] = __ldg(su + c / cpb);
        }
      }
    }
#pragma unroll
    for (int j = 0; j < kU; ++j) {
      const int c = base + lane + 32 * j;
      if (c < HC) {
        if (kFp8) {
          // 16 codes per chunk, all in one scale block
#pragma unroll
          for (int q = 0; q < NQ; ++q) {
            if (q < nq) {
              const uint4 x0 = sx[xo[q] + 2 * c], x1 = sx[xo[q] + 2 * c + 1];
              ag[q] = fmaf(dot16_e4m3_bf16(gv[j], x0, x1), sgv[j], ag[q]);
              au[q] = fmaf(dot16_e4m3_bf16(uv[j], x0, x1), suv[j], au[q]);
            }
          }
        } else {
#pragma unroll
          for (int q = 0; q < NQ; ++q) {
            if (q < nq) {
              const uint4 xv = sx[xo[q] + c];
              ag[q] = fma8_bf16(gv[j], xv, ag[q]);
              au[q] = fma8_bf16(uv[j], xv, au[q]);
            }
          }
        }
      }
    }
  }
#pragma unroll
  for (int q = 0; q < NQ; ++q) {
    if (q < nq) {
      const float gs = warp_sum(ag[q]);
      const float us = warp_sum(au[q]);
      if (lane == 0)
        act[static_cast<size_t>(plist[q]) * I + i] =
            bf16_bits(bias ? gated_rt(act_kind, gs + bg, us + bu) : gated_rt(act_kind, gs, us));
    }
  }
}

// Phase 2 item: the kR2 dot products of w2 rows r0.. r0+kR2-1 of this CTA
// (ws: in shared memory, else wg: through L2) with act of one pair (bf16,
// a8: 8 values per 16-byte chunk, on chip when cache_act); the act chunks
// are loaded once for the kR2 independent sums.  Lane 0 writes
// sdots[r][pair].
// FP8 weights: 16 codes per chunk, each chunk's partial sum times the scale
// of its row and block (s2r: the scales of row r0, ipb per row).
template <bool kFp8>
__device__ __forceinline__ void phase2_item(const uint4 *ws, const uint4 *__restrict__ wg,
                                            const uint4 *a8, int cache_act, int pair, int r0,
                                            int nrows, int I, int TK, float *sdots,
                                            const float *s2r, int ipb, int cpb) {
  const int lane = threadIdx.x & 31;
  const uint4 *a = a8 + static_cast<size_t>(pair) * (I / 8);
  const int IC = kFp8 ? I / 16 : I / 8;  // 16-byte weight chunks per row
  float v[kR2];
#pragma unroll
  for (int rr = 0; rr < kR2; ++rr) v[rr] = 0.f;
  for (int base = 0; base < IC; base += 32 * kU2) {
    // FP8: the scales of this lane's chunks, loaded ahead of the dot products
    float sc[kU2][kR2];
    if (kFp8) {
#pragma unroll
      for (int j = 0; j < kU2; ++j) {
        const int c = base + lane + 32 * j;
#pragma unroll
        for (int rr = 0; rr < kR2; ++rr)
          // s2r may point into shared memory: a generic load
          sc[j][rr] = c < IC && r0 + rr < nrows ? s2r[rr * ipb + c / cpb] : 0.f;
      }
    }
#pragma unroll
    for (int j = 0; j < kU2; ++j) {
      const int c = base + lane + 32 * j;
      if (c < IC) {
        // the act values of this chunk: 16 (FP8) or 8 (bf16 weights)
        const uint4 x0 = cache_act ? a[(kFp8 ? 2 : 1) * c] : __ldcg(a + (kFp8 ? 2 : 1) * c);
        uint4 x1 = x0;
        if (kFp8) x1 = cache_act ? a[2 * c + 1] : __ldcg(a + 2 * c + 1);
#pragma unroll
        for (int rr = 0; rr < kR2; ++rr) {
          if (r0 + rr < nrows) {
            const uint4 wv =
                ws != nullptr ? ws[(r0 + rr) * IC + c] : __ldg(wg + (r0 + rr) * IC + c);
            if (kFp8)
              v[rr] = fmaf(dot16_e4m3_bf16(wv, x0, x1), sc[j][rr], v[rr]);
            else
              v[rr] = fma8_bf16(wv, x0, v[rr]);
          }
        }
      }
    }
  }
#pragma unroll
  for (int rr = 0; rr < kR2; ++rr) {
    const float sv = warp_sum(v[rr]);
    if (lane == 0 && r0 + rr < nrows) sdots[(r0 + rr) * TK + pair] = sv;
  }
}

// Phase 2 item with both operands on chip (w2 rows in a ring slot, act
// staged in shared memory): the same kR2 dot products as phase2_item, in
// the same order per lane (so the same sums), but every load of a block of
// chunks is issued before the first FMA, so a warp waits for shared memory
// once per block rather than once per load (with the loads behind the
// operand-location branches, each one was its own round trip: ~1.4 us per
// item).  Rows past nrows read the last row and are not stored.  FP8: sc0
// holds the scales of the CTA's local row 0 (ipb per row; on chip when the
// copy warp staged them, else in global memory).
constexpr int kU2c = 3;  // bf16: chunks per lane per block (I = 768: one block)
constexpr int kU2f = 1;  // FP8: chunks of 16 codes per lane per block
template <bool kFp8>
__device__ __forceinline__ void phase2_item_onchip(const uint4 *ws, const uint4 *sa,
                                                   const float *sc0, int pair, int r0,
                                                   int nrows, int I, int TK, float *sdots,
                                                   int ipb, int cpb) {
  const int lane = threadIdx.x & 31;
  constexpr int kU = kFp8 ? kU2f : kU2c;
  const int IC = kFp8 ? I / 16 : I / 8;
  int rows[kR2];
#pragma unroll
  for (int rr = 0; rr < kR2; ++rr) rows[rr] = min(r0 + rr, nrows - 1);
  float v[kR2];
#pragma unroll
  for (int rr = 0; rr < kR2; ++rr) v[rr] = 0.f;
  for (int base = 0; base < IC; base += 32 * kU) {
    uint4 x0[kU], x1[kU];
    uint4 wv[kU][kR2];
    float sc[kU][kR2];
#pragma unroll
    for (int j = 0; j < kU; ++j) {
      const int c = min(base + lane + 32 * j, IC - 1);
      if (kFp8) {
        x0[j] = sa[2 * c];
        x1[j] = sa[2 * c + 1];
      } else {
        x0[j] = sa[c];
      }
#pragma unroll
      for (int rr = 0; rr < kR2; ++rr) {
        wv[j][rr] = ws[rows[rr] * IC + c];
        if (kFp8) sc[j][rr] = sc0[rows[rr] * ipb + c / cpb];  // generic: shared or global
      }
    }
#pragma unroll
    for (int j = 0; j < kU; ++j) {
      if (base + lane + 32 * j < IC) {
#pragma unroll
        for (int rr = 0; rr < kR2; ++rr) {
          if (kFp8)
            v[rr] = fmaf(dot16_e4m3_bf16(wv[j][rr], x0[j], x1[j]), sc[j][rr], v[rr]);
          else
            v[rr] = fma8_bf16(wv[j][rr], x0[j], v[rr]);
        }
      }
    }
  }
#pragma unroll
  for (int rr = 0; rr < kR2; ++rr) {
    const float sv = warp_sum(v[rr]);
    if (lane == 0 && r0 + rr < nrows) sdots[(r0 + rr) * TK + pair] = sv;
  }
}

// Dynamic shared memory of a CTA: the token vectors in bf16 [T][H]; a ring of `slots` buffers, each holding this
// CTA's w2 rows of one chosen expert in bf16 [rows_per_cta][I] (no ring when
// one expert's rows do not fit: phase 2 then reads w2 through L2); act in
// bf16 [T*k][I] when it fits; the dot products [rows_per_cta][T*k].
struct SmemLayout {
  size_t w2_off, act_off, dots_off, scl_off, total;
};

// elem: bytes per weight (2: bf16, 1: FP8)
__host__ __device__ inline size_t w2_slot_bytes(int rows_per_cta, int I, int elem) {
  return (static_cast<size_t>(rows_per_cta) * I * elem + 127) & ~static_cast<size_t>(127);
}

// scl: fp32 w2 scales per row staged on chip (FP8: I / block, else 0), for
// the first `slots` chosen experts
__host__ __device__ inline SmemLayout smem_layout(int T, int TK, int H, int I,
                                                  int rows_per_cta, int slots, int cache_act,
                                                  int elem, int scl = 0) {
  SmemLayout s;
  s.w2_off = static_cast<size_t>(T) * H * 2;
  s.act_off = s.w2_off + static_cast<size_t>(slots) * w2_slot_bytes(rows_per_cta, I, elem);
  s.dots_off = s.act_off + (cache_act ? static_cast<size_t>(TK) * I * 2 : 0);  // bf16
  s.scl_off = s.dots_off + static_cast<size_t>(rows_per_cta) * TK * sizeof(float);
  s.total = s.scl_off + static_cast<size_t>(slots) * rows_per_cta * scl * sizeof(float);
  return s;
}

// kTokens: 1 (decode: 8 chunks per lane and row in flight) or kMaxT (up to
// 16 tokens, taken per expert in groups).  kFp8: the weights are FP8 E4M3
// codes (16 per 16-byte chunk) with fp32 scales s1 [E, 2I, H / block] and
// s2 [E, H, I / block]; every chunk's partial dot product is multiplied by
// the scale of its row and block before it is added.
template <int kTokens, bool kFp8>
__global__ void __launch_bounds__(kThreads, kBlocksPerSm)
    small_t_kernel(const uint4 *__restrict__ hidden, const uint4 *__restrict__ w1,
                   const uint4 *__restrict__ w2, const float *__restrict__ s1,
                   const float *__restrict__ s2, int block, const float *__restrict__ b1,
                   const float *__restrict__ b2, int act_kind, const float *__restrict__ topk_w,
                   const int32_t *__restrict__ ids, float *__restrict__ act,
                   float *__restrict__ out, int T, int k, int H, int I, int E, int rows_per_cta,
                   int slots, int cache_act, int stage_scl, uint32_t *status,
                   unsigned long long *grid_sync, uint64_t limit, uint64_t *tl_buf,
                   int64_t tl_cap) {
  // phase 1: chunks per lane and row in flight (an FP8 chunk holds 16 codes)
  constexpr int kU1 = kFp8 ? 4 : (kTokens == 1 ? 8 : 4);
  extern __shared__ __align__(16) uint8_t smem[];
  __shared__ Lists L;
  __shared__ volatile int s_abort;
  __shared__ uint64_t w2_full[kMaxSlots];   // a slot's rows have landed
  __shared__ uint64_t w2_empty[kMaxSlots];  // every compute warp is done with a slot
  __shared__ float s_topw[kMaxPairs];       // the top-k weights, for the final sum
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int TK = T * k;
  const int H8 = H / 8;
  constexpr int kElem = kFp8 ? 1 : 2;
  const int HC = H * kElem / 16, IC = I * kElem / 16;  // 16-byte weight chunks per row
  const int cpb = kFp8 ? block / 16 : 1;                // chunks per scale block
  const int hpb = kFp8 ? H / block : 0, ipb = kFp8 ? I / block : 0;  // blocks per row
  const SmemLayout lay =
      smem_layout(T, TK, H, I, rows_per_cta, slots, cache_act, kElem, stage_scl ? ipb : 0);
  const size_t slot_stride = w2_slot_bytes(rows_per_cta, I, kElem);
  uint8_t *sx = smem;  // the token's vector (one-token kernel)
  // act scratch (T*k*I values): bf16 bits in the caller's fp32-sized buffer
  uint16_t *act_h = reinterpret_cast<uint16_t *>(act);
  uint8_t *sw2 = smem + lay.w2_off;
  uint4 *sact = reinterpret_cast<uint4 *>(smem + lay.act_off);  // act in bf16 [T*k][I]
  float *sdots = reinterpret_cast<float *>(smem + lay.dots_off);
  float *sscl = reinterpret_cast<float *>(smem + lay.scl_off);  // [slots][rows_per_cta][ipb]
  const int h0 = blockIdx.x * rows_per_cta;
  const int nrows = max(0, min(H, h0 + rows_per_cta) - h0);

  const uint64_t tl_start = tl_buf ? global_timer_ns() : 0;
  if (warp == 0) build_lists(L, ids, TK, E);
  if (threadIdx.x == 32) {
    s_abort = 0;
    for (int q = 0; q < slots; ++q) {
      mbar_init(&w2_full[q], 1);
      mbar_init(&w2_empty[q], kWarps);
    }
    fence_mbar_init();
  }
  for (int c = threadIdx.x; c < T * H8; c += kThreads)
    reinterpret_cast<uint4 *>(sx)[c] = __ldg(hidden + c);
  // loaded now, while the weights stream, rather than at the end where the
  // final sum would wait for them
  for (int i = threadIdx.x; i < TK; i += kThreads) s_topw[i] = __ldg(topk_w + i);
  const uint4 *sx4 = reinterpret_cast<const uint4 *>(sx);
  __syncthreads();
  const int nd = L.n_distinct;
  const int nw = gridDim.x * kWarps;
  const int n1 = nd * I;
  // bytes of one expert's rows of this CTA (nrows may be 0 for the last CTAs)
  const uint32_t w2_bytes = static_cast<uint32_t>(nrows) * I * kElem;
  const bool ring = slots > 0 && nrows > 0;
  if (warp == kCopyWarp && lane == 0 && nrows > 0) {
    // the first experts' w2 rows, for phase 2, stream in alongside w1; the
    // rest follow in phase 2 as slots free up.  Without a ring, ask L2 to
    // prefetch them.
    if (ring) {
      for (int d = 0; d < nd && d < slots; ++d) {
        mbar_arrive_expect_tx(&w2_full[d], w2_bytes);
        bulk_load(sw2 + d * slot_stride, w2 + (static_cast<size_t>(L.dexp[d]) * H + h0) * IC,
                  w2_bytes, &w2_full[d]);
      }
    } else {
      for (int d = 0; d < nd; ++d)
        bulk_prefetch_l2(w2 + (static_cast<size_t>(L.dexp[d]) * H + h0) * IC, w2_bytes);
    }
  }
  if (kFp8 && stage_scl && warp == kCopyWarp && nrows > 0) {
    // the w2 scales of this CTA's rows, for the experts that get a slot:
    // read now, while the weights stream, so that no phase-2 item waits on
    // a global load for them (they are read once, but each costs a round
    // trip to memory where the phase-2 item needs it)
    __syncwarp();
    const int per = nrows * ipb;
    for (int d = 0; d < nd && d < slots; ++d) {
      const float *src = s2 + (static_cast<size_t>(L.dexp[d]) * H + h0) * ipb;
      for (int x = lane; x < per; x += 32)
        sscl[static_cast<size_t>(d) * rows_per_cta * ipb + x] = __ldg(src + x);
    }
  }

  // ------------------------------------------------------------ phase 1
  for (int task = blockIdx.x * kWarps + warp; task < n1 && warp < kWarps; task += nw) {
    const int d = task / I, i = task - d * I;
    const int p0 = L.dstart[d], np = L.dstart[d + 1] - p0;
    const uint4 *g = w1 + (static_cast<size_t>(L.dexp[d]) * 2 * I + i) * HC;
    const uint4 *u = g + static_cast<size_t>(I) * HC;
    // FP8: the scale rows of the gate and up rows
    const float *sg = kFp8 ? s1 + (static_cast<size_t>(L.dexp[d]) * 2 * I + i) * hpb : nullptr;
    const float *su = kFp8 ? sg + static_cast<size_t>(I) * hpb : nullptr;
    // the variant's bias of this row pair (0 without b1)
    float bg = 0.f, bu = 0.f;
    if (b1 != nullptr) {
      bg = __ldg(b1 + static_cast<size_t>(L.dexp[d]) * 2 * I + i);
      bu = __ldg(b1 + static_cast<size_t>(L.dexp[d]) * 2 * I + I + i);
    }
    if (kTokens == 1) {
      // one token: its pairs on e (more than one only for repeated ids) share
      // the same dot products
      float ag = 0.f, au = 0.f;
      for (int base = 0; base < HC; base += 32 * kU1) {
        uint4 gv[kU1], uv[kU1];
        float sgv[kU1], suv[kU1];  // FP8: the chunks' scales, loaded with the codes
#pragma unroll
        for (int j = 0; j < kU1; ++j) {
          const int c = base + lane + 32 * j;
          if (c < HC) {
            gv[j] = __ldcs(g + c);
            uv[j] = __ldcs(u + c);
            if (kFp8) {
              sgv[j] = __ldg(sg + c / cpb);
              suv[j] = __ldg(su + c / cpb);
            }
          }
        }
#pragma unroll
        for (int j = 0; j < kU1; ++j) {
          const int c = base + lane + 32 * j;
          if (c < HC) {
            if (kFp8) {
              const uint4 x0 = sx4[2 * c], x1 = sx4[2 * c + 1];
              ag = fmaf(dot16_e4m3_bf16(gv[j], x0, x1), sgv[j], ag);
              au = fmaf(dot16_e4m3_bf16(uv[j], x0, x1), suv[j], au);
            } else {
              const uint4 xv = sx4[c];
              ag = fma8_bf16(gv[j], xv, ag);
              au = fma8_bf16(uv[j], xv, au);
            }
          }
        }
      }
      ag = warp_sum(ag);
      au = warp_sum(au);
      if (lane == 0) {
        const float a = b1 != nullptr ? gated_rt(act_kind, ag + bg, au + bu)
                                      : gated_rt(act_kind, ag, au);
        const uint16_t ab = bf16_bits(a);
        for (int q = 0; q < np; ++q) act_h[static_cast<size_t>(L.plist[p0 + q]) * I + i] = ab;
      }
    } else {
      // the tokens routed to e, in groups of at most 4 (the row pair is
      // re-read from L2 for each further group)
      for (int q0 = 0; q0 < np; q0 += 4) {
        const int nq = min(4, np - q0);
        const int *pl = L.plist + p0 + q0;
        const bool bias = b1 != nullptr;
        if (nq == 1)
          phase1_group<1, kFp8 ? 4 : 8, kFp8>(g, u, sx4, pl, nq, k, H8, I, i, bg, bu, bias,
                                              act_kind, act_h, sg, su, cpb);
        else
          phase1_group<4, 4, kFp8>(g, u, sx4, pl, nq, k, H8, I, i, bg, bu, bias, act_kind, act_h,
                                   sg, su, cpb);
      }
    }
  }

  // ------------------------------------------------------------ grid barrier
  // Every CTA adds one per launch and every launch on this counter has the
  // same grid, so between launches the counter is a multiple of gridDim.x:
  // the value a CTA read decides which launch it belongs to, and the
  // barrier opens when the counter reaches the end of that launch's block
  // of arrivals.  (Derived here, not passed in, so that the target is right
  // whatever was launched before on the counter.)
  __threadfence();
  __syncthreads();
  const uint64_t tl_p1 = tl_buf ? global_timer_ns() : 0;
  if (threadIdx.x == 0) {
    const unsigned long long old = atomicAdd(grid_sync, 1ull);
    const unsigned long long target = (old / gridDim.x + 1) * gridDim.x;
    const uint64_t t0 = global_timer_ns();
    while (ld_acquire_gpu(grid_sync) < target) {
      if (global_timer_ns() - t0 > limit) {
        s_abort = 1;
        atomicOr(status, kStatusTimeout);
        break;
      }
      __nanosleep(32);
    }
    __threadfence();
  }
  __syncthreads();
  const uint64_t tl_bar = tl_buf ? global_timer_ns() : 0;
  const int64_t tl_slot = static_cast<int64_t>(blockIdx.x) * kTlPerCta;
  if (threadIdx.x == 0) {
    timeline_rec(tl_buf, tl_cap, tl_slot, kTlSmallT, kTlPhase1, 0, blockIdx.x, tl_start, tl_p1);
    timeline_rec(tl_buf, tl_cap, tl_slot + 1, kTlSmallT, kTlBarrier, 0, blockIdx.x, tl_p1, tl_bar);
  }
  if (s_abort) {
    // let the bulk copies already issued land before the CTA exits
    if (warp == kCopyWarp && lane == 0 && ring)
      for (int d = 0; d < nd && d < slots; ++d) mbar_wait(&w2_full[d], 0, kW2WaitNs);
    return;
  }

  // ------------------------------------------------------------ phase 2
  const uint4 *act8 = reinterpret_cast<const uint4 *>(act_h);
  // every operand on chip (w2 rows in the ring, act staged below):
  // phase2_item_onchip
  const bool onchip = ring && cache_act;
  if (cache_act) {
    // act was written by other CTAs in this launch: read it from L2
    const int n8 = TK * I / 8;
    for (int x = threadIdx.x; x < n8; x += kThreads) sact[x] = __ldcg(act8 + x);
    __syncthreads();
    act8 = sact;
  }
  const uint64_t tl_act = tl_buf ? global_timer_ns() : 0;
  if (threadIdx.x == 0)
    timeline_rec(tl_buf, tl_cap, tl_slot + 2, kTlSmallT, kTlActLoad, 0, blockIdx.x, tl_bar, tl_act);
  const int rgroups = (nrows + kR2 - 1) / kR2;
  if (warp == kCopyWarp) {
    // refill the ring: expert d goes into slot d % slots once every compute
    // warp has finished with expert d - slots
    if (lane == 0 && ring) {
      int issued = min(nd, slots);
      for (int d = slots; d < nd; ++d) {
        const int q = d % slots;
        if (!mbar_wait(&w2_empty[q], ((d / slots) - 1) & 1, kW2WaitNs, &s_abort)) {
          s_abort = 1;
          atomicOr(status, kStatusTimeout);
          break;
        }
        mbar_arrive_expect_tx(&w2_full[q], w2_bytes);
        bulk_load(sw2 + q * slot_stride, w2 + (static_cast<size_t>(L.dexp[d]) * H + h0) * IC,
                  w2_bytes, &w2_full[q]);
        issued = d + 1;
      }
      if (s_abort) {
        // the last load of each slot must land before the CTA exits
        for (int d = max(0, issued - slots); d < issued; ++d)
          mbar_wait(&w2_full[d % slots], (d / slots) & 1, kW2WaitNs);
      }
    }
  } else if (rgroups > 0 && (!ring || nd <= slots)) {
    // every chosen expert's rows are on chip (or read through L2): wait for
    // the copies once, then deal all items (pair, group of kR2 local rows)
    // round-robin over the compute warps
    for (int d = 0; ring && d < nd; ++d) {
      if (!mbar_wait(&w2_full[d], 0, kW2WaitNs, &s_abort)) {
        s_abort = 1;
        atomicOr(status, kStatusTimeout);
        break;
      }
    }
    if (warp == 0 && lane == 0)
      timeline_rec(tl_buf, tl_cap, tl_slot + 3, kTlSmallT, kTlW2Wait, 0, blockIdx.x, tl_act,
                   global_timer_ns());
    const int n_items = L.dstart[nd] * rgroups;
    for (int it = warp; it < n_items && !s_abort; it += kWarps) {
      const int pq = it / rgroups, rg = it - pq * rgroups;  // pq: position in plist
      const int pair = L.plist[pq];
      const int d = L.pd[pair];
      const size_t row0 = static_cast<size_t>(L.dexp[d]) * H + h0;  // w2 row of local row 0
      const float *s2r = kFp8 ? s2 + (row0 + rg * kR2) * ipb : nullptr;  // FP8 scales
      if (onchip)
        phase2_item_onchip<kFp8>(
            reinterpret_cast<const uint4 *>(sw2 + d * slot_stride),
            act8 + static_cast<size_t>(pair) * (I / 8),
            !kFp8 ? nullptr
                  : stage_scl ? sscl + static_cast<size_t>(d) * rows_per_cta * ipb : s2 + row0 * ipb,
            pair, rg * kR2, nrows, I, TK, sdots, ipb, cpb);
      else
        phase2_item<kFp8>(ring ? reinterpret_cast<const uint4 *>(sw2 + d * slot_stride) : nullptr,
                          w2 + row0 * IC, act8, cache_act, pair, rg * kR2, nrows, I, TK, sdots,
                          s2r, ipb, cpb);
    }
  } else if (rgroups > 0) {
    // more experts than slots: take the experts in order, waiting for each
    // one's slot and releasing it after this warp's share of its items (the
    // round-robin continues from one expert to the next)
    int before = 0;  // items of the experts before d
    for (int d = 0; d < nd; ++d) {
      const int q = d % slots;
      if (!mbar_wait(&w2_full[q], (d / slots) & 1, kW2WaitNs, &s_abort)) {
        s_abort = 1;
        atomicOr(status, kStatusTimeout);
        break;
      }
      const int p0 = L.dstart[d];
      const int n_items = (L.dstart[d + 1] - p0) * rgroups;
      int it = warp - before % kWarps;
      if (it < 0) it += kWarps;
      for (; it < n_items; it += kWarps) {
        const int pq = p0 + it / rgroups, rg = it % rgroups;
        const size_t row0 = static_cast<size_t>(L.dexp[d]) * H + h0;
        if (onchip)
          phase2_item_onchip<kFp8>(
              reinterpret_cast<const uint4 *>(sw2 + q * slot_stride),
              act8 + static_cast<size_t>(L.plist[pq]) * (I / 8),
              !kFp8                     ? nullptr
              : stage_scl && d < slots ? sscl + static_cast<size_t>(d) * rows_per_cta * ipb
                                       : s2 + row0 * ipb,
              L.plist[pq], rg * kR2, nrows, I, TK, sdots, ipb, cpb);
        else
          phase2_item<kFp8>(reinterpret_cast<const uint4 *>(sw2 + q * slot_stride), nullptr,
                            act8, cache_act, L.plist[pq], rg * kR2, nrows, I, TK, sdots,
                            kFp8 ? s2 + (row0 + rg * kR2) * ipb : nullptr, ipb, cpb);
      }
      before += n_items;
      __syncwarp();
      if (lane == 0) mbar_arrive(&w2_empty[q]);
    }
  }
  __syncthreads();
  if (threadIdx.x == 0)
    timeline_rec(tl_buf, tl_cap, tl_slot + 5, kTlSmallT, kTlItems, 0, blockIdx.x, tl_bar,
                 global_timer_ns());
  if (s_abort) return;
  // out[t, h] = sum over j in ascending order of w[t, j] * dot(t*k + j)
  for (int x = threadIdx.x; x < T * nrows; x += kThreads) {
    const int t = x / nrows, r = x - t * nrows;
    float acc = 0.f;
    for (int j = 0; j < k; ++j) {
      const int pair = t * k + j;
      if (L.pd[pair] >= 0) {
        float y = sdots[r * TK + pair];
        if (b2 != nullptr) y += __ldg(b2 + static_cast<size_t>(L.ids[pair]) * H + h0 + r);
        acc = fmaf(s_topw[pair], y, acc);
      }
    }
    out[static_cast<size_t>(t) * H + h0 + r] = acc;
  }
  if (tl_buf != nullptr) {
    __syncthreads();
    if (threadIdx.x == 0)
      timeline_rec(tl_buf, tl_cap, tl_slot + 4, kTlSmallT, kTlPhase2, 0, blockIdx.x, tl_bar,
                   global_timer_ns());
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    bool bad = false;
    for (int i = 0; i < TK; ++i) bad = bad || L.pd[i] < 0;
    if (bad) atomicOr(status, kStatusBadId);
  }
}

struct SmallTConfig {
  int rows_per_cta, slots, cache_act, stage_scl;
  size_t smem;
};

// What goes into `budget` bytes of dynamic shared memory: as many w2 ring
// slots as there can be distinct experts (at most kMaxSlots), and the act
// cache when it fits beside them -- unless it would leave fewer than two
// slots (no overlap of copies and dot products) where dropping it gives more.
// scl: FP8 w2 scales per row (I / block; 0 for bf16), staged on chip when
// they fit beside the rest (at most kSclStageMax bytes).
constexpr size_t kSclStageMax = 16 * 1024;
SmallTConfig small_t_config(int T, int TK, int H, int I, int E, int grid, size_t budget,
                            int elem, int scl) {
  SmallTConfig c;
  c.rows_per_cta = (H + grid - 1) / grid;
  const int want = std::min(std::min(TK, E), kMaxSlots);
  auto size = [&](int slots, int cache) {
    return smem_layout(T, TK, H, I, c.rows_per_cta, slots, cache, elem).total;
  };
  auto fit = [&](int cache) {
    int n = want;
    while (n > 0 && size(n, cache) > budget) --n;
    return n;
  };
  c.cache_act = static_cast<size_t>(TK) * I * 2 <= kActCacheMax ? 1 : 0;
  c.slots = fit(c.cache_act);
  if (c.cache_act && c.slots < std::min(want, 2) && fit(0) > c.slots) {
    c.cache_act = 0;
    c.slots = fit(0);
  }
  if (c.cache_act && size(c.slots, 1) > budget) c.cache_act = 0;
  c.smem = size(c.slots, c.cache_act);
  const size_t with_scl =
      smem_layout(T, TK, H, I, c.rows_per_cta, c.slots, c.cache_act, elem, scl).total;
  c.stage_scl = scl > 0 && c.slots > 0 && with_scl - c.smem <= kSclStageMax && with_scl <= budget;
  if (c.stage_scl) c.smem = with_scl;
  return c;
}

// The dynamic shared memory the kernel may use next to its static shared
// memory, with kBlocksPerSm CTAs on an SM.
size_t smem_budget(int dev, const void *kern) {
  int per_sm = 0, reserved = 0;
  cudaFuncAttributes fa;
  if (cudaDeviceGetAttribute(&per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) !=
          cudaSuccess ||
      cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev) !=
          cudaSuccess ||
      cudaFuncGetAttributes(&fa, kern) != cudaSuccess)
    return 0;
  const size_t per_block = static_cast<size_t>(per_sm) / kBlocksPerSm;
  const size_t fixed = fa.sharedSizeBytes + static_cast<size_t>(reserved);
  return per_block > fixed ? (per_block - fixed) & ~static_cast<size_t>(127) : 0;
}

}  // namespace

bool small_t_supported(int H, int I) { return H <= kMaxH && I <= kMaxI; }

namespace {

std::mutex g_setup_mu;
uint64_t g_ready_mask = 0;
int g_grid_of[64] = {};
size_t g_budget_of[64] = {};

// Once per device: the shared-memory budget all four instantiations can
// use and the cooperative grid (the CTAs both kernels keep resident on
// every SM: the grid barrier needs every CTA resident at once).
cudaError_t small_t_setup(int dev) {
  std::lock_guard<std::mutex> lock(g_setup_mu);
  if ((g_ready_mask >> dev) & 1) return cudaSuccess;
  int sms = 0;
  cudaError_t e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const auto kerns = {small_t_kernel<1, false>, small_t_kernel<kMaxT, false>,
                      small_t_kernel<1, true>, small_t_kernel<kMaxT, true>};
  size_t smem = ~static_cast<size_t>(0);
  for (auto kern : kerns)
    smem = std::min(smem, smem_budget(dev, reinterpret_cast<const void *>(kern)));
  if (smem < 16384) return cudaErrorInvalidValue;
  int per_sm = kBlocksPerSm;
  for (auto kern : kerns) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    int n = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, kThreads, smem);
    if (e != cudaSuccess) return e;
    per_sm = std::min(per_sm, n);
  }
  if (per_sm < 1) return cudaErrorCooperativeLaunchTooLarge;
  g_budget_of[dev] = smem;
  g_grid_of[dev] = per_sm * sms;
  g_ready_mask |= 1ull << dev;
  return cudaSuccess;
}

}  // namespace

cudaError_t small_t_fits(int64_t T, int H, int I, int E, int k, bool fp8, bool *fits) {
  *fits = false;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if ((e = small_t_setup(dev)) != cudaSuccess) return e;
  if (!small_t_supported(H, I) || T < 1 || T > kMaxT || T * k > kMaxPairs) return cudaSuccess;
  // scales are staged only when they fit, so the bf16-sized layout decides
  const SmallTConfig cfg = small_t_config(static_cast<int>(T), static_cast<int>(T) * k, H, I, E,
                                          g_grid_of[dev], g_budget_of[dev], fp8 ? 1 : 2, 0);
  *fits = cfg.smem <= g_budget_of[dev];
  return cudaSuccess;
}

cudaError_t launch_small_t(const uint16_t *hidden, const void *w1, const void *w2,
                           const float *w1_scale, const float *w2_scale, int block,
                           const float *b1, const float *b2, int act_kind,
                           const float *topk_weights, const int32_t *topk_ids, float *act,
                           float *out, int64_t T, int H, int I, int E, int k, uint32_t *status,
                           unsigned long long *grid_sync, uint64_t wait_limit_ns,
                           cudaStream_t s, const StageHook &hook, uint64_t *timeline,
                           int64_t timeline_cap) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (!small_t_supported(H, I) || dev < 0 || dev >= 64 || T < 1 || T > kMaxT || T * k > kMaxPairs)
    return cudaErrorInvalidValue;
  if ((e = small_t_setup(dev)) != cudaSuccess) return e;
  const int grid = g_grid_of[dev];
  const bool fp8 = block > 0;
  if (fp8 && (w1_scale == nullptr || w2_scale == nullptr || block % 16 != 0 || H % block != 0 ||
              I % block != 0))
    return cudaErrorInvalidValue;
  const SmallTConfig cfg = small_t_config(static_cast<int>(T), static_cast<int>(T) * k, H, I, E,
                                          grid, g_budget_of[dev], fp8 ? 1 : 2,
                                          fp8 ? I / block : 0);
  if (cfg.smem > g_budget_of[dev]) return cudaErrorInvalidValue;
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(grid);
  lc.blockDim = dim3(kThreads);
  lc.dynamicSmemBytes = cfg.smem;
  lc.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  lc.attrs = attr;
  lc.numAttrs = 1;
  hook.begin(fp8 ? "small_t_fp8" : "small_t");
  auto kern = fp8 ? (T == 1 ? small_t_kernel<1, true> : small_t_kernel<kMaxT, true>)
                  : (T == 1 ? small_t_kernel<1, false> : small_t_kernel<kMaxT, false>);
  e = cudaLaunchKernelEx(&lc, kern, reinterpret_cast<const uint4 *>(hidden),
                         reinterpret_cast<const uint4 *>(w1), reinterpret_cast<const uint4 *>(w2),
                         w1_scale, w2_scale, block, b1, b2, act_kind, topk_weights, topk_ids, act, out, static_cast<int>(T), k, H, I, E,
                         cfg.rows_per_cta, cfg.slots, cfg.cache_act, cfg.stage_scl, status,
                         grid_sync, wait_limit_ns, timeline, timeline_cap);
  return hook.end(e);
}

}  // namespace moe
