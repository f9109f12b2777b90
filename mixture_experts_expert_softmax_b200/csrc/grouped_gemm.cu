// grouped_gemm.cu -- the two expert GEMMs of the fused MoE forward as
// persistent, warp-specialised tcgen05 kernels (sm_100a).
//
//   GEMM1 (+SwiGLU): for the rows of expert e in expert-sorted order,
//     g = x . w1[e, 0:I, :]^T, u = x . w1[e, I:2I, :]^T  (fp32 in TMEM),
//     act = silu(g) * u, stored as bf16 [rows, I].  Variants (the 0.13.2
//     version of the page below): gelu (tanh form) or swigluoai in place of
//     silu, and a bias b1[e] added to g and u before the activation.
//   GEMM2: y = act . w2[e]^T (fp32 in TMEM), plus the bias b2[e] when given
//     (before the top-k weight).  For top-k <= 2 the epilogue
//     adds w_j * y_j of each row straight into out[token] with bulk
//     reductions at L2 (out was zeroed first); out[t] = 0 + a + b is the
//     same in either arrival order, so the result is still deterministic.
//     For larger k it stores y as fp32 rows of P in the same expert-sorted
//     order and combine.cu forms sum_j w_j * y_j in fixed j order.
// This is the expert FFN of ref_moe on the page "tpu_inference/kernels/
// fused_moe/v1/kernel.py" (gate = w1, up = w3, then act . w2) in the weight
// layout of atrex-bench #009 (w1 [E, 2I, H], w2 [E, H, I], both applied as
// F.linear, i.e. K-major).
//
// Work unit: an m-tile of one expert's rows times one 256-column n-tile of
// the accumulator.  Tiles run expert-major, then n-tile, then m-tile, so
// CTAs working together share a weight tile through L2; the grid is
// persistent and loops over tiles.
//
// Three kernels share the code (MODE):
//   kModeFused   one launch on CTA pairs (a cluster of 2, M = 256,
//                cta_group::2) that runs every GEMM1 tile and then every
//                GEMM2 tile.  Its A rows come from copies in expert-sorted
//                order (hidden rows gathered by gather_rows_kernel, and act),
//                so rank r of the pair loads A rows 128r..128r+127 and half
//                of the B tile with TMA into its own shared memory; rank 0
//                issues the MMAs and each CTA receives its 128 accumulator
//                rows in its own TMEM.  For GEMM1 rank 0 loads the n-tile's
//                128 gate rows of w1 and rank 1 the matching 128 up rows, so
//                one accumulator holds gate and up side by side.  A GEMM2
//                tile waits (bounded) until the epilogues of all GEMM1 tiles
//                of its m-tile have published their act rows through a
//                per-m-tile counter: the static tile order puts every GEMM1
//                tile of a CTA before its GEMM2 tiles, so no wait can form a
//                cycle, and GEMM2 tiles fill the last, partial wave of GEMM1.
//                This needs every CTA of the grid resident at once (the grid
//                never exceeds the occupancy query's cluster count): work that
//                another stream keeps on the SMs meanwhile can hold CTAs back
//                until a bounded wait gives up (MOE_STATUS_TIMEOUT).
//   kModeGemm1   GEMM1 alone on single CTAs (M = 128, cta_group::1) that
//                gather their A rows by token index with cp.async (whose
//                completion can only be signalled to the CTA's own barriers)
//                and load gate and up rows themselves: no row copy needed.
//   kModeGemm2   GEMM2 alone on CTA pairs, after kModeGemm1.
// The GEMM2 epilogue stages each warp's 32 rows x 32 columns in shared
// memory and writes them with one asynchronous TMA tile store into P (a
// block that straddles the end of an expert's rows is written row by row
// instead), or, fused with the combine, scales row r by its top-k weight
// and issues one 128-byte bulk reduce-add per row into out[token]: large
// operations, because the TMA engine's cost per operation, not the bytes,
// bounds this epilogue.
//
// Shared memory: the barriers and the expert / tile offset tables sit in
// front, then (1024-byte aligned, as the 128-byte swizzle needs) the stage
// ring and the epilogue staging.  The number of stages is chosen at launch:
// as many as fit, up to kMaxStages, given the expert count.
//
// Warp roles (416 threads per CTA):
//   warps 0-3  producers.  kModeGemm1: the 128 threads gather the A rows with
//              16-byte cp.async into the 128-byte-swizzled K-major layout and
//              arrive on the stage barrier asynchronously when they land;
//              thread 0 issues the two TMA boxes of w1.  CTA pairs: thread 0
//              of each CTA issues TMA for its A rows and half of B, counted
//              on rank 0's barrier.
//   warp 4     allocates 512 TMEM columns (two accumulators); one thread (on
//              rank 0) issues the MMAs and commits each stage back to the
//              producers and each finished tile to the epilogues.
//   warps 5-12 epilogue, two warps per 32-lane TMEM quarter (a warp can only
//              read the quarter warp_id % 4), each taking half of the tile's
//              columns: tcgen05.ld, SwiGLU + bf16 store, or the fp32 TMA
//              store / bulk reductions, then release the accumulator.
// Every wait is bounded; a wait that gives up raises the timeout bit of the
// status word and makes every role of the CTA leave its loop.
#include <algorithm>
#include <mutex>

#include "moe_internal.h"

namespace moe {
namespace {

constexpr int BM = 128;  // rows per CTA
constexpr int BK = 64;   // K per stage: one 128-byte swizzle row of bf16
constexpr int kProducerThreads = 128;
constexpr int kMmaWarp = 4;
constexpr int kEpiWarps = 8;  // warps 5..12
constexpr int kThreads = (5 + kEpiWarps) * 32;
constexpr int kAccN = 256;            // UMMA N = accumulator columns per tile
constexpr int kTmemCols = 2 * kAccN;  // double-buffered accumulator
constexpr int kABytes = BM * BK * 2;  // 16 KB
constexpr int kMaxE = 1024;
constexpr int kMaxStages = 6;
constexpr uint16_t kBothCtas = 0x3;
// Per-warp staging of the GEMM2 epilogue: one 32-row x 32-column fp32 block,
// 128-byte swizzled for the TMA store, or 32 plain rows at a 144-byte pitch
// for the reductions (16-byte writes of 8 consecutive lanes then hit 8
// different bank groups: bank conflicts here would take shared-memory
// bandwidth from the tensor core's operand reads).  A 1024-byte multiple
// keeps every warp's block swizzle-aligned.
constexpr int kRedPitch = 144;
constexpr int kEpiWarpBytes = 5 * 1024;
static_assert(32 * kRedPitch <= kEpiWarpBytes, "staging");
// The CTA's last tile of the combine-fused GEMM2 stages whole 128-column
// half rows (512 bytes, at a 528-byte pitch: 8 consecutive lanes again hit
// 8 different bank groups) in the idle operand ring, one reduction per row.
constexpr int kBigPitch = 528;
constexpr size_t kSmemMax = 232448;  // opt-in maximum per block on sm_100
// act rows of an m-tile are complete when every epilogue warp of both CTAs
// has published each of its n-tiles
constexpr int kReadyPerTile = 2 * kEpiWarps;

enum { kModeGemm1 = 0, kModeGemm2 = 1, kModeFused = 2 };

template <int MODE>
struct Cfg;
template <>
struct Cfg<kModeGemm1> {
  static constexpr int CG = 1;        // CTAs per MMA
  static constexpr int kBRows = 256;  // B rows this CTA loads per stage
  static constexpr int kEpiBytes = 0;
};
template <>
struct Cfg<kModeGemm2> {
  static constexpr int CG = 2;
  static constexpr int kBRows = 128;
  static constexpr int kEpiBytes = kEpiWarps * kEpiWarpBytes;
};
template <>
struct Cfg<kModeFused> {
  static constexpr int CG = 2;
  static constexpr int kBRows = 128;  // GEMM1: gate rows on rank 0, up rows on rank 1
  static constexpr int kEpiBytes = kEpiWarps * kEpiWarpBytes;
};

template <int MODE>
constexpr int tile_m() { return BM * Cfg<MODE>::CG; }
template <int MODE>
constexpr int b_bytes() { return Cfg<MODE>::kBRows * BK * 2; }

struct __align__(8) Bars {
  uint64_t full[kMaxStages];   // stage landed (rank 0's counts both CTAs)
  uint64_t empty[kMaxStages];  // the MMAs finished reading the stage
  uint64_t acc_full[2];        // accumulator ready for the epilogue
  uint64_t acc_empty[2];       // epilogues (of both CTAs) drained the accumulator
  uint64_t drain;              // every MMA has completed
  uint32_t tmem_base;
  int abort_flag;
  int32_t scan[32];            // per-warp partial sums of build_tile_offsets
};

// Bytes in front of the aligned region: barriers, then exp_off and tile_off
// (E + 1 entries each).
__host__ __device__ constexpr size_t front_bytes(int E) {
  return sizeof(Bars) + 2 * static_cast<size_t>(E + 1) * sizeof(int32_t);
}

// Dynamic shared memory for `stages` stages (with the GEMM2 epilogue's
// staging when `gemm2`); 1008 bytes cover the padding to the next 1024-byte
// boundary from any 16-byte aligned base.
template <int MODE>
constexpr size_t smem_bytes(int E, int stages, bool gemm2 = true) {
  return front_bytes(E) + 1008 + static_cast<size_t>(stages) * (kABytes + b_bytes<MODE>()) +
         (gemm2 ? Cfg<MODE>::kEpiBytes : 0);
}

template <int MODE>
int stages_for(int E, bool gemm2 = true) {
  int st = kMaxStages;
  while (st > 2 && smem_bytes<MODE>(E, st, gemm2) > kSmemMax) --st;
  return st;
}
static_assert(smem_bytes<kModeGemm1>(kMaxE, 4) <= kSmemMax, "shared memory budget");
static_assert(smem_bytes<kModeGemm2>(kMaxE, 5) <= kSmemMax, "shared memory budget");
static_assert(smem_bytes<kModeFused>(kMaxE, 5) <= kSmemMax, "shared memory budget");

struct Params {
  const __nv_bfloat16 *hidden;
  const int32_t *sorted_rows;
  const int32_t *expert_offsets;
  __nv_bfloat16 *act;
  float *P;
  int H, I, E, k;
  int nt1, nt2;  // n-tiles per m-tile of GEMM1 (I / 128) and GEMM2 (ceil(H / 256))
  int stages;    // depth of the operand ring (<= kMaxStages)
  int run_gemm2; // kModeFused: 0 runs the GEMM1 tiles only (GEMM2 follows as
                 // its own kModeGemm2 launch)
  uint32_t *status;
  uint64_t wait_limit_ns;
  // float4 count of out to zero before GEMM2 adds into it (0: none)
  float4 *zero_out;
  int64_t zero_n4;
  // GEMM2 fused with the combine: out [T, H] and the top-k weights [T, k]
  float *out;
  const float *topk_weights;
  int fuse_combine;
  // kModeFused: per-m-tile act counters and the count of epilogue warps
  // that finished zeroing out (both zero at launch)
  int *ready;
  int *zero_done;
  // epilogue variant: activation (kAct*) and optional fp32 biases
  // b1 [E, 2I] (gate, then up) and b2 [E, H]
  const float *b1;
  const float *b2;
  int act_kind;
  // debug timeline (see timeline_rec): null when off; this launch's records
  // start at slot tl_base, kTlPerTile per tile
  uint64_t *tl_buf;
  int64_t tl_cap;
  int64_t tl_base;
  uint32_t tl_kind;
};

struct Tile {
  int e, mt, nt, row0, rows;  // row0/rows: the whole m-tile (both CTAs of a pair)
};

// Tile t -> (expert, m-tile, n-tile).  tile_off[e] counts the m-tiles of
// experts < e, so expert e owns tiles [tile_off[e] * NT, tile_off[e+1] * NT).
template <int TM>
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
  tl.row0 = exp_off[lo] + tl.mt * TM;
  tl.rows = min(TM, exp_off[lo + 1] - tl.row0);
  return tl;
}

// exp_off[0..E] -> tile_off[0..E]: exclusive prefix sum of ceil(count / TM),
// computed by the whole CTA (E <= 1024, kThreads threads).
template <int TM>
__device__ void build_tile_offsets(const int32_t *exp_off, int32_t *tile_off, int E,
                                   int32_t *scratch /* >= 32 ints */) {
  constexpr int kPer = (kMaxE + kThreads - 1) / kThreads;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int local[kPer];
  int sum = 0;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int e = tid * kPer + i;
    local[i] = e < E ? (exp_off[e + 1] - exp_off[e] + TM - 1) / TM : 0;
    sum += local[i];
  }
  int incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int x = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += x;
  }
  if (lane == 31) scratch[warp] = incl;
  __syncthreads();
  int before = 0;
  for (int w = 0; w < warp; ++w) before += scratch[w];
  int run = before + incl - sum;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int e = tid * kPer + i;
    if (e <= E) tile_off[e] = run;  // e == E receives the total
    run += local[i];
  }
}

__device__ __forceinline__ void give_up(const Params &p, volatile int *abort_flag) {
  *abort_flag = 1;
  atomicOr(p.status, kStatusTimeout);
}

__device__ __forceinline__ float as_f32(uint32_t u) { return __uint_as_float(u); }

// v[c] += b[c] for 32 fp32 values held as bits; b is 16-byte aligned and
// the same for every lane (a broadcast load)
__device__ __forceinline__ void add_bias32(uint32_t (&v)[32], const float *b) {
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float4 bb = __ldg(reinterpret_cast<const float4 *>(b) + j);
    v[4 * j] = __float_as_uint(as_f32(v[4 * j]) + bb.x);
    v[4 * j + 1] = __float_as_uint(as_f32(v[4 * j + 1]) + bb.y);
    v[4 * j + 2] = __float_as_uint(as_f32(v[4 * j + 2]) + bb.z);
    v[4 * j + 3] = __float_as_uint(as_f32(v[4 * j + 3]) + bb.w);
  }
}

// act = ACT(g, u) for 32 columns, packed to bf16 pairs
template <int ACT>
__device__ __forceinline__ void gated_pack32(const uint32_t (&g)[32], const uint32_t (&u)[32],
                                             uint32_t (&pk)[16]) {
#pragma unroll
  for (int v = 0; v < 16; ++v)
    pk[v] = pack_bf16x2(gated_f<ACT>(as_f32(g[2 * v]), as_f32(u[2 * v])),
                        gated_f<ACT>(as_f32(g[2 * v + 1]), as_f32(u[2 * v + 1])));
}

// What one tile of the static schedule is: GEMM1 or GEMM2 (phase 1 or 2),
// its place, and its global m-tile index.
struct Work {
  int phase;
  int mi;
  Tile tl;
};

template <int MODE>
__device__ __forceinline__ Work get_work(int t, int total1, const Params &p,
                                         const int32_t *tile_off, const int32_t *exp_off) {
  Work w;
  int local = t, nt = p.nt1;
  w.phase = 1;
  if (MODE == kModeGemm2 || (MODE == kModeFused && t >= total1)) {
    w.phase = 2;
    nt = p.nt2;
    if (MODE == kModeFused) local = t - total1;
  }
  w.tl = decode_tile<tile_m<MODE>()>(local, nt, p.E, tile_off, exp_off);
  w.mi = tile_off[w.tl.e] + w.tl.mt;
  return w;
}

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tm_a1,
                        const __grid_constant__ CUtensorMap tm_b1,
                        const __grid_constant__ CUtensorMap tm_a2,
                        const __grid_constant__ CUtensorMap tm_b2,
                        const __grid_constant__ CUtensorMap tm_out, const Params p) {
  using C = Cfg<MODE>;
  constexpr int CG = C::CG;
  constexpr int TM = tile_m<MODE>();
  constexpr int kBBytes = b_bytes<MODE>();
  constexpr bool kGather = MODE == kModeGemm1;  // A rows by cp.async
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const int kStages = p.stages;
  Bars *bars = reinterpret_cast<Bars *>(smem_raw);
  int32_t *s_tile_off = reinterpret_cast<int32_t *>(bars + 1);
  int32_t *s_exp_off = s_tile_off + (p.E + 1);
  uint8_t *sA = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + front_bytes(p.E) + 1023) &
      ~static_cast<uintptr_t>(1023));
  uint8_t *sB = sA + kStages * kABytes;
  uint8_t *sEpi = sB + kStages * kBBytes;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = CG == 2 ? cluster_rank() : 0;
  const bool leader = rank == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      // kModeGemm1: 128 cp.async arrivals + the expect_tx arrival; pairs:
      // rank 0's expect_tx arrival (both CTAs' TMA bytes are counted on it)
      mbar_init(&bars->full[s], kGather ? kProducerThreads + 1 : 1);
      mbar_init(&bars->empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&bars->acc_full[a], 1);
      mbar_init(&bars->acc_empty[a], kEpiWarps * CG);  // every epilogue warp of the pair
    }
    mbar_init(&bars->drain, 1);
    bars->abort_flag = 0;
    fence_mbar_init();
    if (MODE != kModeGemm2) prefetch_tmap(&tm_b1);
    if (MODE == kModeFused) prefetch_tmap(&tm_a1);
    if (MODE != kModeGemm1) {
      prefetch_tmap(&tm_a2);
      prefetch_tmap(&tm_b2);
      if (!p.fuse_combine) prefetch_tmap(&tm_out);
    }
  }
  if (warp == kMmaWarp) {
    if (CG == 2) {
      tmem_alloc_pair(&bars->tmem_base, kTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(&bars->tmem_base, kTmemCols);
      tmem_relinquish();
    }
  }
  // both CTAs' barriers exist before any traffic crosses the pair
  if (CG == 2) cluster_sync();
  // Everything above overlaps the previous kernel under PDL; the routing
  // permutation (and the A rows) are read only after this point.
  grid_dep_wait();
  grid_dep_launch();
  for (int i = threadIdx.x; i <= p.E; i += blockDim.x) s_exp_off[i] = p.expert_offsets[i];
  __syncthreads();
  build_tile_offsets<TM>(s_exp_off, s_tile_off, p.E, bars->scan);
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();

  const uint32_t tmem_base = bars->tmem_base;
  const int m_tiles = s_tile_off[p.E];
  const int total1 = MODE == kModeGemm2 ? 0 : m_tiles * p.nt1;
  const int total =
      total1 + (MODE == kModeGemm1 || (MODE == kModeFused && !p.run_gemm2) ? 0 : m_tiles * p.nt2);
  const int unit = CG == 2 ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int nunits = CG == 2 ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);
  volatile int *abort_flag = &bars->abort_flag;
  const uint64_t limit = p.wait_limit_ns;
  // rank 0's barriers as seen from this CTA
  const uint32_t full0 = CG == 2 ? map_to_rank(smem_addr(&bars->full[0]), 0) : 0u;
  const uint32_t acc_empty0 = CG == 2 ? map_to_rank(smem_addr(&bars->acc_empty[0]), 0) : 0u;

  if (warp < 4) {
    // ------------------------------------------------------------ producers
    if (kGather) {
      const int c = threadIdx.x & 7;      // 16-byte chunk of the 128-byte row
      const int rsub = threadIdx.x >> 3;  // rows rsub, rsub+16, ..., rsub+112
      const int KB = p.H / BK;
      int s = 0;  // ring slot and its phase parity, advanced per k-block
      uint32_t ph = 0;
      bool stop = false;
      for (int t = unit; t < total && !stop; t += nunits) {
        const uint64_t tl_t0 = p.tl_buf ? global_timer_ns() : 0;
        const Tile tl = get_work<MODE>(t, total1, p, s_tile_off, s_exp_off).tl;
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
        const int b_row = tl.e * 2 * p.I + tl.nt * (kAccN / 2);
        for (int kb = 0; kb < KB; ++kb, s = s + 1 == kStages ? 0 : s + 1, ph ^= s == 0) {
          if (!mbar_wait(&bars->empty[s], ph ^ 1, limit, abort_flag)) {
            give_up(p, abort_flag);
            stop = true;
            break;
          }
          if (threadIdx.x == 0) {
            mbar_arrive_expect_tx(&bars->full[s], kBBytes);
            uint8_t *b = sB + s * kBBytes;
            tma_load_2d(b, &tm_b1, &bars->full[s], kb * BK, b_row);                       // gate
            tma_load_2d(b + kBBytes / 2, &tm_b1, &bars->full[s], kb * BK, b_row + p.I);  // up
          }
          const uint32_t a_base = smem_addr(sA + s * kABytes);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int r = rsub + 16 * i;
            cp_async_16(a_base + r * 128 + ((c ^ (r & 7)) << 4), src[i] + kb * BK, nbytes[i]);
          }
          // counts as this thread's arrival on full[s] once its copies land
          cp_async_arrive_noinc(&bars->full[s]);
        }
        if (threadIdx.x == 0)
          timeline_rec(p.tl_buf, p.tl_cap, p.tl_base + int64_t{t} * kTlPerTile + rank, p.tl_kind,
                       kTlProducer, rank, t, tl_t0, global_timer_ns());
      }
      cp_async_wait_all();
      if (stop && threadIdx.x == 0) {
        // let TMA copies already issued land before the CTA can exit
        const uint64_t t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 200000) {
        }
      }
    } else if (threadIdx.x == 0) {
      int s = 0;  // ring slot and its phase parity, advanced per k-block
      uint32_t ph = 0;
      bool stop = false;
      for (int t = unit; t < total && !stop; t += nunits) {
        const uint64_t tl_t0 = p.tl_buf ? global_timer_ns() : 0;
        const Work w = get_work<MODE>(t, total1, p, s_tile_off, s_exp_off);
        if (MODE == kModeFused && w.phase == 2) {
          // the act rows of this m-tile come from other CTAs' GEMM1 epilogues
          if (!wait_geq(p.ready + w.mi, kReadyPerTile * p.nt1, limit, abort_flag)) {
            give_up(p, abort_flag);
            break;
          }
          fence_proxy_async_global();
        }
        const bool g1 = w.phase == 1;
        const CUtensorMap *am = g1 ? &tm_a1 : &tm_a2;
        const CUtensorMap *bm = g1 ? &tm_b1 : &tm_b2;
        const int KB = (g1 ? p.H : p.I) / BK;
        const int a_row = w.tl.row0 + static_cast<int>(rank) * BM;
        // GEMM1: rank 0 the n-tile's gate rows, rank 1 its up rows;
        // GEMM2: rank r rows 128r.. of the n-tile's 256 rows of w2
        const int b_row = g1 ? w.tl.e * 2 * p.I + static_cast<int>(rank) * p.I +
                                   w.tl.nt * (kAccN / 2)
                             : w.tl.e * p.H + w.tl.nt * kAccN + static_cast<int>(rank) * C::kBRows;
        for (int kb = 0; kb < KB; ++kb, s = s + 1 == kStages ? 0 : s + 1, ph ^= s == 0) {
          if (!mbar_wait(&bars->empty[s], ph ^ 1, limit, abort_flag)) {
            give_up(p, abort_flag);
            stop = true;
            break;
          }
          if (leader) mbar_arrive_expect_tx(&bars->full[s], CG * (kABytes + kBBytes));
          tma_load_2d_pair(sA + s * kABytes, am, full0 + 8u * s, kb * BK, a_row);
          tma_load_2d_pair(sB + s * kBBytes, bm, full0 + 8u * s, kb * BK, b_row);
        }
        timeline_rec(p.tl_buf, p.tl_cap, p.tl_base + int64_t{t} * kTlPerTile + rank, p.tl_kind,
                     kTlProducer, rank, t, tl_t0, global_timer_ns());
      }
      if (*abort_flag) {
        const uint64_t t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 200000) {
        }
      }
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0 && leader) {
      // ---------------------------------------------------------- MMA issuer
      const uint32_t idesc = idesc_bf16_f32(TM, kAccN);
      int s = 0, acc_it = 0;  // ring slot and its phase parity, advanced per k-block
      uint32_t ph = 0;
      bool stop = false;
      for (int t = unit; t < total && !stop; t += nunits, ++acc_it) {
        const int KB = (get_work<MODE>(t, total1, p, s_tile_off, s_exp_off).phase == 1 ? p.H : p.I) / BK;
        const int a = acc_it & 1;
        const uint32_t aph = (acc_it >> 1) & 1;
        if (!mbar_wait(&bars->acc_empty[a], aph ^ 1, limit, abort_flag)) {
          give_up(p, abort_flag);
          break;
        }
        tc_fence_after_sync();
        const uint64_t tl_t0 = p.tl_buf ? global_timer_ns() : 0;
        const uint32_t d_tmem = tmem_base + a * kAccN;
        for (int kb = 0; kb < KB; ++kb, s = s + 1 == kStages ? 0 : s + 1, ph ^= s == 0) {
          if (!mbar_wait(&bars->full[s], ph, limit, abort_flag)) {
            give_up(p, abort_flag);
            stop = true;
            break;
          }
          tc_fence_after_sync();
          // A rows may have been written by cp.async: order them before the
          // tensor core's (async-proxy) reads
          if (kGather) fence_proxy_async_smem();
          const uint64_t a_desc = smem_desc_sw128(smem_addr(sA + s * kABytes));
          const uint64_t b_desc = smem_desc_sw128(smem_addr(sB + s * kBBytes));
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            // +32 bytes of K per step, in 16-byte units of the start address
            if (CG == 2)
              umma_f16_pair(d_tmem, a_desc + 2 * kk, b_desc + 2 * kk, idesc, (kb | kk) != 0);
            else
              umma_f16(d_tmem, a_desc + 2 * kk, b_desc + 2 * kk, idesc, (kb | kk) != 0);
          }
          if (CG == 2)
            umma_commit_pair(&bars->empty[s], kBothCtas);
          else
            umma_commit(&bars->empty[s]);
        }
        if (!stop) {
          if (CG == 2)
            umma_commit_pair(&bars->acc_full[a], kBothCtas);
          else
            umma_commit(&bars->acc_full[a]);
        }
        timeline_rec(p.tl_buf, p.tl_cap, p.tl_base + int64_t{t} * kTlPerTile + 2, p.tl_kind, kTlMma,
                     0, t, tl_t0, global_timer_ns());
      }
      // every MMA must be complete before TMEM is released
      if (CG == 2)
        umma_commit_pair(&bars->drain, kBothCtas);
      else
        umma_commit(&bars->drain);
      if (!mbar_wait(&bars->drain, 0, limit)) give_up(p, abort_flag);
    } else if (lane == 0) {
      // rank 1 of a pair: wait for the pair's MMAs to finish with this TMEM
      if (!mbar_wait(&bars->drain, 0, limit)) give_up(p, abort_flag);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - (kMmaWarp + 1);  // 0..7
    const int q = warp & 3;                 // TMEM lane quarter accessible to this warp
    const int half = ew >> 2;               // which half of the tile's columns
    const int row = q * 32 + lane;
    uint8_t *ebuf = sEpi + ew * kEpiWarpBytes;  // GEMM2: this warp's staging buffer
    if (MODE != kModeGemm2 && p.zero_n4 > 0) {
      // out must read zero before GEMM2 adds into it; this runs while the
      // first tiles' MMAs are in flight
      const int64_t nw = static_cast<int64_t>(gridDim.x) * kEpiWarps;
      const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int64_t i = (static_cast<int64_t>(blockIdx.x) * kEpiWarps + ew) * 32 + lane;
           i < p.zero_n4; i += nw * 32)
        p.zero_out[i] = z;
      if (MODE == kModeFused && p.run_gemm2) {
        // publish: GEMM2 tiles of any CTA add into out only after every
        // epilogue warp of the grid has zeroed its part
        __threadfence();
        __syncwarp();
        if (lane == 0) atomicAdd(p.zero_done, 1);
      }
    }
    bool zero_seen = MODE != kModeFused || p.zero_n4 == 0 || !p.run_gemm2;
    int acc_it = 0;
    for (int t = unit; t < total; t += nunits, ++acc_it) {
      const Work w = get_work<MODE>(t, total1, p, s_tile_off, s_exp_off);
      const Tile &tl = w.tl;
      const int a = acc_it & 1;
      const uint32_t aph = (acc_it >> 1) & 1;
      if (!mbar_wait(&bars->acc_full[a], aph, limit, abort_flag)) {
        give_up(p, abort_flag);
        break;
      }
      tc_fence_after_sync();
      const uint64_t tl_t0 = p.tl_buf && ew == 0 ? global_timer_ns() : 0;
      const int my_row0 = tl.row0 + static_cast<int>(rank) * BM;
      const int my_rows = min(BM, max(0, tl.rows - static_cast<int>(rank) * BM));
      const bool valid = row < my_rows;
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + a * kAccN;
      if (w.phase == 1) {
        __nv_bfloat16 *dst =
            p.act + static_cast<size_t>(my_row0 + (valid ? row : 0)) * p.I + tl.nt * (kAccN / 2);
        const float *bg =
            p.b1 ? p.b1 + static_cast<size_t>(tl.e) * 2 * p.I + tl.nt * (kAccN / 2) : nullptr;
#pragma unroll 1
        for (int c0 = half * (kAccN / 4); c0 < (half + 1) * (kAccN / 4); c0 += 32) {
          uint32_t g[32], u[32];
          tmem_ld_32cols(tbase + c0, g);
          tmem_ld_32cols(tbase + kAccN / 2 + c0, u);
          tmem_ld_wait();
          if (valid) {
            if (bg) {
              add_bias32(g, bg + c0);
              add_bias32(u, bg + p.I + c0);
            }
            uint32_t pk[16];
            if (p.act_kind == kActGeluTanh)
              gated_pack32<kActGeluTanh>(g, u, pk);
            else if (p.act_kind == kActSwigluOai)
              gated_pack32<kActSwigluOai>(g, u, pk);
            else
              gated_pack32<kActSilu>(g, u, pk);
            uint4 *d4 = reinterpret_cast<uint4 *>(dst + c0);
#pragma unroll
            for (int v = 0; v < 4; ++v)
              d4[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
          }
          __syncwarp();
        }
      } else if (p.fuse_combine) {
        if (!zero_seen) {
          if (!wait_geq(p.zero_done, static_cast<int>(gridDim.x) * kEpiWarps, limit, abort_flag))
            give_up(p, abort_flag);
          fence_proxy_async_global();
          zero_seen = true;
        }
        // row -> (token, weight); each lane stages and reduces its own row,
        // so the lanes need no synchronisation with one another
        float wgt = 0.f;
        float *orow = p.out;
        if (valid) {
          const int slot = p.sorted_rows[my_row0 + row];
          wgt = p.topk_weights[slot];
          orow = p.out + static_cast<size_t>(slot / p.k) * p.H;
        }
        uint8_t *srow = ebuf + lane * kRedPitch;
        const float *b2row = p.b2 ? p.b2 + static_cast<size_t>(tl.e) * p.H : nullptr;
        // The CTA's last tile: no MMA follows to hide this epilogue behind,
        // and the TMA engine's cost per operation bounds it.  Every MMA has
        // completed (acc_full) and every operand load has landed (each was
        // consumed by one of those MMAs), so the operand ring is idle: each
        // lane stages its row's 128 columns there and adds them with one
        // 512-byte reduction instead of four 128-byte ones.
        const int colh = tl.nt * kAccN + half * (kAccN / 2);
        const bool wide = t + nunits >= total && colh + kAccN / 2 <= p.H &&
                          kStages * (kABytes + kBBytes) >= kEpiWarps * 32 * kBigPitch;
        if (wide) {
          uint8_t *brow = sA + (ew * 32 + lane) * kBigPitch;
#pragma unroll 1
          for (int c0 = 0; c0 < kAccN / 2; c0 += 32) {
            uint32_t v[32];
            tmem_ld_32cols(tbase + half * (kAccN / 2) + c0, v);
            tmem_ld_wait();
            if (b2row) add_bias32(v, b2row + colh + c0);
#pragma unroll
            for (int j = 0; j < 8; ++j)
              *reinterpret_cast<float4 *>(brow + 4 * c0 + 16 * j) =
                  make_float4(wgt * as_f32(v[4 * j]), wgt * as_f32(v[4 * j + 1]),
                              wgt * as_f32(v[4 * j + 2]), wgt * as_f32(v[4 * j + 3]));
          }
          if (valid && !*abort_flag) {
            fence_proxy_async_smem();
            bulk_reduce_add_f32(orow + colh, brow, 4 * (kAccN / 2));
            bulk_commit_group();
          }
          __syncwarp();
        }
#pragma unroll 1
        for (int c0 = half * (kAccN / 2); !wide && c0 < (half + 1) * (kAccN / 2); c0 += 32) {
          uint32_t v[32];
          tmem_ld_32cols(tbase + c0, v);
          tmem_ld_wait();
          const int col = tl.nt * kAccN + c0;
          if (b2row && col < p.H) add_bias32(v, b2row + col);
          if (col < p.H && valid && !*abort_flag) {
            // the previous reduction from this row must have read it
            bulk_wait_group_read<0>();
#pragma unroll
            for (int j = 0; j < 8; ++j)
              *reinterpret_cast<float4 *>(srow + 16 * j) =
                  make_float4(wgt * as_f32(v[4 * j]), wgt * as_f32(v[4 * j + 1]),
                              wgt * as_f32(v[4 * j + 2]), wgt * as_f32(v[4 * j + 3]));
            fence_proxy_async_smem();
            bulk_reduce_add_f32(orow + col, srow, 128);
            bulk_commit_group();
          }
          __syncwarp();
        }
      } else {
        // this warp's 32 rows: whole blocks go out through TMA stores
        const bool whole = q * 32 + 32 <= my_rows;
        const float *b2row = p.b2 ? p.b2 + static_cast<size_t>(tl.e) * p.H : nullptr;
#pragma unroll 1
        for (int c0 = half * (kAccN / 2); c0 < (half + 1) * (kAccN / 2); c0 += 32) {
          uint32_t v[32];
          tmem_ld_32cols(tbase + c0, v);
          tmem_ld_wait();
          const int col = tl.nt * kAccN + c0;
          if (b2row && col < p.H) add_bias32(v, b2row + col);
          if (col < p.H && whole) {
            // the previous store from this buffer must have read it
            if (lane == 0) bulk_wait_group_read<0>();
            __syncwarp();
            // row `lane` as 8 chunks of 16 bytes, 128-byte swizzle
#pragma unroll
            for (int j = 0; j < 8; ++j)
              *reinterpret_cast<uint4 *>(ebuf + lane * 128 + ((j ^ (lane & 7)) << 4)) =
                  make_uint4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&tm_out, ebuf, col, my_row0 + q * 32);
              bulk_commit_group();
            }
          } else if (col < p.H && valid) {
            // the block crosses the end of the expert's rows: plain stores
            float4 *d4 = reinterpret_cast<float4 *>(
                p.P + static_cast<size_t>(my_row0 + row) * p.H + col);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              d4[i] = make_float4(as_f32(v[4 * i]), as_f32(v[4 * i + 1]), as_f32(v[4 * i + 2]),
                                  as_f32(v[4 * i + 3]));
          }
          __syncwarp();
        }
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) {
        if (CG == 2)
          mbar_arrive_cluster(acc_empty0 + 8u * a);
        else
          mbar_arrive(&bars->acc_empty[a]);
        if (ew == 0)
          timeline_rec(p.tl_buf, p.tl_cap, p.tl_base + int64_t{t} * kTlPerTile + 3 + rank,
                       p.tl_kind, kTlEpilogue, rank, t, tl_t0, global_timer_ns());
      }
      if (MODE == kModeFused && w.phase == 1 && p.run_gemm2) {
        // publish this warp's act rows of the m-tile to GEMM2 tiles (after
        // the accumulator is released, so the fence does not hold up MMAs)
        __threadfence();
        __syncwarp();
        if (lane == 0) atomicAdd(p.ready + w.mi, 1);
      }
    }
    if (MODE != kModeGemm1) bulk_wait_group_all();
  }

  tc_fence_before_sync();
  __syncthreads();
  // neither CTA may leave (or free TMEM) while its peer can still reach it
  if (CG == 2) cluster_sync();
  if (warp == kMmaWarp) {
    tc_fence_after_sync();
    if (CG == 2)
      tmem_dealloc_pair(tmem_base, kTmemCols);
    else
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

// Row-major matrix [outer, inner] as a 2-D tensor map with a
// (box_inner x box_rows) box and the 128-byte swizzle.
bool make_map(CUtensorMap *m, CUtensorMapDataType dtype, int elem_bytes, const void *base,
              uint64_t inner, uint64_t outer, uint32_t box_inner, uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {inner * elem_bytes};
  const cuuint32_t box[2] = {box_inner, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, dtype, 2, const_cast<void *>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_bf16_map(CUtensorMap *m, const void *base, uint64_t inner, uint64_t outer,
                   uint32_t box_rows) {
  return make_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, inner, outer, BK, box_rows);
}

int g_max_pairs[64] = {};  // 2-CTA clusters resident at once, per device

template <int MODE>
int grid_for(const GroupedGemmArgs &a, int n_tiles_n, int device) {
  constexpr int CG = Cfg<MODE>::CG;
  const int64_t rows = a.T * a.k;
  const int64_t max_tiles = ((rows + tile_m<MODE>() - 1) / tile_m<MODE>() + a.E) * n_tiles_n;
  // never more units than can be resident together: the fused kernel's
  // GEMM2 tiles wait for other CTAs' GEMM1 tiles
  int units = a.num_sms / CG;
  if (CG == 2 && device >= 0 && device < 64 && g_max_pairs[device] > 0)
    units = std::min(units, g_max_pairs[device]);
  if (max_tiles < units) units = static_cast<int>(max_tiles);
  return CG * (units > 0 ? units : 1);
}

Params base_params(const GroupedGemmArgs &a) {
  Params p = {};
  p.hidden = reinterpret_cast<const __nv_bfloat16 *>(a.hidden);
  p.sorted_rows = a.sorted_rows;
  p.expert_offsets = a.expert_offsets;
  p.act = reinterpret_cast<__nv_bfloat16 *>(a.act);
  p.P = a.P;
  p.H = a.H;
  p.I = a.I;
  p.E = a.E;
  p.k = a.k;
  p.nt1 = a.I / (kAccN / 2);
  p.nt2 = (a.H + kAccN - 1) / kAccN;  // H % 128 == 0: a last half tile is masked
  p.status = a.status;
  p.wait_limit_ns = a.wait_limit_ns;
  p.fuse_combine = a.P == nullptr ? 1 : 0;
  if (p.fuse_combine) {
    p.out = a.out;
    p.topk_weights = a.topk_weights;
    p.zero_out = reinterpret_cast<float4 *>(a.out);
    p.zero_n4 = a.T * a.H / 4;
  }
  p.ready = a.counters + kCounterReady;
  p.zero_done = a.counters + kCounterZeroDone;
  p.b1 = a.b1;
  p.b2 = a.b2;
  p.act_kind = a.act_kind;
  p.tl_buf = a.timeline;
  p.tl_cap = a.timeline_cap;
  return p;
}

template <int MODE>
cudaLaunchConfig_t launch_config(int grid, size_t smem, cudaStream_t s, bool pdl,
                                 cudaLaunchAttribute (&attr)[3]) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  int n = 0;
  if (Cfg<MODE>::CG == 2) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = 2;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  if (pdl) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cfg;
}

template <int MODE>
cudaError_t set_smem_attr() {
  return cudaFuncSetAttribute(grouped_gemm_kernel<MODE>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(kSmemMax));
}

template <int MODE>
cudaError_t max_pairs(int *clusters) {
  cudaLaunchAttribute attr[3];
  cudaLaunchConfig_t cfg = launch_config<MODE>(2, kSmemMax, nullptr, false, attr);
  return cudaOccupancyMaxActiveClusters(clusters, grouped_gemm_kernel<MODE>, &cfg);
}

// The maps GEMM2 uses: act [T*k, I] and w2 [E*H, I] with 64 x 128-row boxes,
// and P [T*k, H] fp32 in 32 x 32 blocks (a stand-in map over act when P is
// not written).
bool gemm2_maps(const GroupedGemmArgs &a, CUtensorMap *tm_act, CUtensorMap *tm_w2,
                CUtensorMap *tm_p) {
  const uint64_t rows = static_cast<uint64_t>(a.T) * a.k;
  if (!make_bf16_map(tm_act, a.act, static_cast<uint64_t>(a.I), rows, BM) ||
      !make_bf16_map(tm_w2, a.w2, static_cast<uint64_t>(a.I), static_cast<uint64_t>(a.E) * a.H,
                     Cfg<kModeGemm2>::kBRows))
    return false;
  if (a.P == nullptr) {
    *tm_p = *tm_act;
    return true;
  }
  return make_map(tm_p, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, a.P, static_cast<uint64_t>(a.H), rows,
                  32, 32);
}

// w1 [E*2I, H], box 64 x 128 rows (128 gate or 128 up rows of an n-tile)
bool w1_map(const GroupedGemmArgs &a, CUtensorMap *tm_w1) {
  return make_bf16_map(tm_w1, a.w1, static_cast<uint64_t>(a.H),
                       static_cast<uint64_t>(a.E) * 2 * a.I, kAccN / 2);
}

}  // namespace

cudaError_t grouped_gemm_setup(int device) {
  static std::mutex mu;
  static uint64_t done_mask = 0;
  std::lock_guard<std::mutex> lock(mu);
  if (device >= 0 && device < 64 && (done_mask >> device) & 1) return cudaSuccess;
  cudaError_t e = set_smem_attr<kModeGemm1>();
  if (e == cudaSuccess) e = set_smem_attr<kModeGemm2>();
  if (e == cudaSuccess) e = set_smem_attr<kModeFused>();
  if (e != cudaSuccess) return e;
  if (encode_fn() == nullptr) return cudaErrorNotSupported;
  // how many 2-CTA clusters can be resident at once (both pair kernels take
  // one CTA per SM; the smaller count is used for both)
  int c2 = 0, cf = 0;
  e = max_pairs<kModeGemm2>(&c2);
  if (e == cudaSuccess) e = max_pairs<kModeFused>(&cf);
  const int clusters = std::min(c2, cf);
  if (e != cudaSuccess || clusters < 1) {
    cudaGetLastError();
    return e != cudaSuccess ? e : cudaErrorNotSupported;
  }
  if (device >= 0 && device < 64) {
    g_max_pairs[device] = clusters;
    done_mask |= 1ull << device;
  }
  return cudaSuccess;
}

cudaError_t launch_gemm1_swiglu(const GroupedGemmArgs &a, cudaStream_t s, const StageHook &hook) {
  CUtensorMap tm_w1;
  if (!w1_map(a, &tm_w1)) return cudaErrorInvalidValue;
  int dev = 0;
  cudaGetDevice(&dev);
  Params p = base_params(a);
  p.tl_kind = kTlGemm1;
  p.stages = stages_for<kModeGemm1>(a.E);
  cudaLaunchAttribute attr[3];
  const cudaLaunchConfig_t cfg =
      launch_config<kModeGemm1>(grid_for<kModeGemm1>(a, p.nt1, dev),
                                smem_bytes<kModeGemm1>(a.E, p.stages), s, hook.pdl, attr);
  hook.begin("gemm1_swiglu");
  cudaError_t e = cudaLaunchKernelEx(&cfg, grouped_gemm_kernel<kModeGemm1>, tm_w1, tm_w1, tm_w1,
                                     tm_w1, tm_w1, p);
  return hook.end(e);
}

cudaError_t launch_gemm2(const GroupedGemmArgs &a, cudaStream_t s, const StageHook &hook) {
  CUtensorMap tm_act, tm_w2, tm_p;
  if (!gemm2_maps(a, &tm_act, &tm_w2, &tm_p)) return cudaErrorInvalidValue;
  int dev = 0;
  cudaGetDevice(&dev);
  Params p = base_params(a);
  p.zero_out = nullptr;  // zeroed by GEMM1
  p.zero_n4 = 0;
  p.tl_kind = kTlGemm2;
  // after the first launch's records: at most (m-tiles) * (GEMM1 n-tiles) tiles
  p.tl_base = ((a.T * a.k + 255) / 128 + 2 * a.E) * (a.I / (kAccN / 2)) * kTlPerTile;
  p.stages = stages_for<kModeGemm2>(a.E);
  cudaLaunchAttribute attr[3];
  const cudaLaunchConfig_t cfg =
      launch_config<kModeGemm2>(grid_for<kModeGemm2>(a, p.nt2, dev),
                                smem_bytes<kModeGemm2>(a.E, p.stages), s, hook.pdl, attr);
  hook.begin("gemm2");
  cudaError_t e = cudaLaunchKernelEx(&cfg, grouped_gemm_kernel<kModeGemm2>, tm_act, tm_w2, tm_act,
                                     tm_w2, tm_p, p);
  return hook.end(e);
}

cudaError_t launch_fused_gemm(const GroupedGemmArgs &a, bool with_gemm2, cudaStream_t s,
                              const StageHook &hook) {
  if (a.xs == nullptr || (with_gemm2 && a.counters == nullptr)) return cudaErrorInvalidValue;
  CUtensorMap tm_xs, tm_w1, tm_act, tm_w2, tm_p;
  if (!make_bf16_map(&tm_xs, a.xs, static_cast<uint64_t>(a.H), static_cast<uint64_t>(a.T) * a.k,
                     BM) ||
      !w1_map(a, &tm_w1) || !gemm2_maps(a, &tm_act, &tm_w2, &tm_p))
    return cudaErrorInvalidValue;
  int dev = 0;
  cudaGetDevice(&dev);
  Params p = base_params(a);
  p.tl_kind = with_gemm2 ? kTlFused : kTlGemm1;
  p.run_gemm2 = with_gemm2 ? 1 : 0;
  p.stages = stages_for<kModeFused>(a.E, with_gemm2);
  cudaLaunchAttribute attr[3];
  const cudaLaunchConfig_t cfg = launch_config<kModeFused>(
      grid_for<kModeFused>(a, with_gemm2 ? p.nt1 + p.nt2 : p.nt1, dev),
      smem_bytes<kModeFused>(a.E, p.stages, with_gemm2), s, hook.pdl, attr);
  hook.begin(with_gemm2 ? "gemm_fused" : "gemm1_swiglu");
  cudaError_t e = cudaLaunchKernelEx(&cfg, grouped_gemm_kernel<kModeFused>, tm_xs, tm_w1, tm_act,
                                     tm_w2, tm_p, p);
  return hook.end(e);
}

cudaError_t launch_wait_probe(uint32_t *status, uint64_t limit_ns, cudaStream_t s) {
  wait_probe_kernel<<<1, 32, 0, s>>>(status, limit_ns);
  return cudaGetLastError();
}

}  // namespace moe
