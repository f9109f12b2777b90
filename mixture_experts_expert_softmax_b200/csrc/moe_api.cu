// moe_api.cu -- the extern "C" boundary of libmoe.so (declared in
// include/moe.h): argument checks, the per-device workspace, dispatch
// between the small-T GEMV path and the grouped-GEMM path, per-kernel
// profiling events and the debug switches.
#include <algorithm>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "moe.h"
#include "moe_internal.h"

namespace {

constexpr int kMaxDevices = 64;
constexpr int kMaxExperts = 1024;
constexpr int kMaxTopK = 16;
// above this many waves of GEMM tiles (per resident CTA pair) the two GEMMs
// run as separate launches
constexpr int64_t kFusedMaxWaves = 12;

std::mutex g_mu;  // guards the per-device state and the profiler

struct DeviceState {
  bool checked = false;
  bool usable = false;
  int num_sms = 0;
  uint32_t *status = nullptr;  // 256 B: status word at 0, small-T grid counter at 64
  void *ws = nullptr;          // grow-only workspace
  size_t ws_bytes = 0;
  void *wq = nullptr;          // grow-only: bf16 copies of FP8 weights (GEMM path)
  size_t wq_bytes = 0;
};
DeviceState g_dev[kMaxDevices];

int g_small_t_max = -1;  // -1: not read from the environment yet
int g_sync_each = -1;
int64_t g_wait_limit_ns = 2000000000LL;
uint64_t *g_timeline = nullptr;  // debug timeline buffer (moe_timeline), device
int64_t g_timeline_cap = 0;
thread_local const char *g_failed_stage = "";

// ---- profiler
struct ProfEvent {
  const char *name;
  cudaEvent_t a, b;
};
bool g_prof = false;
std::vector<ProfEvent> g_prof_pending;
std::vector<std::string> g_prof_names;
std::vector<int64_t> g_prof_count;
std::vector<double> g_prof_ms;
std::vector<cudaEvent_t> g_event_pool;

cudaEvent_t get_event() {
  if (!g_event_pool.empty()) {
    cudaEvent_t e = g_event_pool.back();
    g_event_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

int small_t_max() {
  if (g_small_t_max < 0) {
    const char *v = std::getenv("MOE_SMALL_T_MAX");
    // up to 8 tokens the GEMV path streams the chosen experts' weights
    // faster than the grouped GEMMs; at 16 the GEMMs win (B200 timings of
    // the E = 8 / top-2 and E = 128 / top-8 shapes)
    g_small_t_max = v ? std::max(0, std::atoi(v)) : 8;
    if (g_small_t_max > 16) g_small_t_max = 16;
  }
  return g_small_t_max;
}

bool sync_each() {
  if (g_sync_each < 0) {
    const char *v = std::getenv("MOE_SYNC_EACH_STAGE");
    g_sync_each = (v && std::atoi(v) != 0) ? 1 : 0;
  }
  return g_sync_each != 0;
}

struct CallCtx {
  cudaStream_t stream;
  const char *cur;
  cudaEvent_t ev0;
};

// Every stage is also an NVTX range named after it (pushed before its
// launch, popped after), so that a timeline tool attached to the process
// groups each kernel under its stage; without a tool the calls do nothing.
void hook_begin(void *c, const char *name) {
  CallCtx *ctx = static_cast<CallCtx *>(c);
  nvtxRangePushA(name);
  ctx->cur = name;
  ctx->ev0 = nullptr;
  if (g_prof) {
    ctx->ev0 = get_event();
    cudaEventRecord(ctx->ev0, ctx->stream);
  }
}

cudaError_t hook_end(void *c, cudaError_t err) {
  CallCtx *ctx = static_cast<CallCtx *>(c);
  if (err == cudaSuccess && g_prof && ctx->ev0 != nullptr) {
    cudaEvent_t ev1 = get_event();
    cudaEventRecord(ev1, ctx->stream);
    g_prof_pending.push_back({ctx->cur, ctx->ev0, ev1});
  }
  if (err == cudaSuccess && sync_each()) {
    err = cudaStreamSynchronize(ctx->stream);
    if (err == cudaSuccess) err = cudaGetLastError();
  }
  if (err != cudaSuccess) g_failed_stage = ctx->cur;
  nvtxRangePop();
  return err;
}

moe::StageHook make_hook(CallCtx *ctx) {
  moe::StageHook h;
  h.ctx = ctx;
  h.on_begin = hook_begin;
  h.on_end = hook_end;
  // event records between launches would break programmatic serialisation
  h.pdl = !g_prof && !sync_each();
  return h;
}

// Current device, checked once for sm_100 and given its status word.
int current_device(DeviceState **out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return MOE_ERR_NO_DEVICE;
  }
  DeviceState &d = g_dev[dev];
  if (!d.checked) {
    d.checked = true;
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) {
      cudaGetLastError();
      return MOE_ERR_NO_DEVICE;
    }
    if (prop.major != 10 || prop.minor != 0) return MOE_ERR_NO_DEVICE;
    d.num_sms = prop.multiProcessorCount;
    if (cudaMalloc(&d.status, 256) != cudaSuccess || cudaMemset(d.status, 0, 256) != cudaSuccess ||
        moe::grouped_gemm_setup(dev) != cudaSuccess || moe::group_setup() != cudaSuccess) {
      cudaGetLastError();
      return MOE_ERR_CUDA;
    }
    d.usable = true;
  }
  if (!d.usable) return MOE_ERR_NO_DEVICE;
  *out = &d;
  return MOE_OK;
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Make a grow-only device buffer at least `bytes` large.
int ensure_buffer(void *&buf, size_t &have, size_t bytes) {
  if (bytes <= have) return MOE_OK;
  if (buf != nullptr) {
    cudaFree(buf);  // synchronises the device
    buf = nullptr;
    have = 0;
  }
  const size_t want = align256(bytes);
  if (cudaMalloc(&buf, want) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_OOM;
  }
  have = want;
  return MOE_OK;
}

int ensure_workspace(DeviceState &d, size_t bytes) { return ensure_buffer(d.ws, d.ws_bytes, bytes); }

struct Carver {
  char *base;
  size_t off = 0;
  template <typename T>
  T *take(size_t count) {
    T *p = reinterpret_cast<T *>(base + off);
    off = align256(off + count * sizeof(T));
    return p;
  }
};

size_t permute_ws_bytes(int64_t n, int E) {
  const size_t chunks = static_cast<size_t>(moe::permute_num_chunks(n));
  return align256(std::max<size_t>(chunks, 1) * E * sizeof(int32_t)) +
         2 * align256((E + 1) * sizeof(int32_t)) + align256(std::max<int64_t>(n, 1) * 4);
}

int to_code(cudaError_t e) {
  if (e == cudaSuccess) return MOE_OK;
  cudaGetLastError();
  return MOE_ERR_CUDA;
}

}  // namespace

extern "C" {

const char *moe_error_string(int code) {
  switch (code) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument (null pointer, negative size or k outside [1, E])";
    case MOE_ERR_UNSUPPORTED: return "unsupported shape (needs H % 128 == 0, I % 128 == 0, E <= 1024, k <= 16)";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_TIMEOUT: return "a bounded device-side wait expired";
    case MOE_ERR_NO_DEVICE: return "no usable sm_100 device is current";
    case MOE_ERR_OOM: return "workspace allocation failed";
    case MOE_ERR_SCRATCH_LIMIT:
      return "request exceeds the fixed scratch of moe_forward_small_noalloc "
             "(T <= MOE_NOALLOC_MAX_T, T*k*I <= MOE_NOALLOC_MAX_ACT)";
    default: return "unknown error code";
  }
}

int moe_route(const float *logits, int64_t T, int E, int k, int renorm, int32_t *topk_ids,
              float *topk_weights, void *stream) {
  if (T < 0 || E < 1 || k < 1 || k > E) return MOE_ERR_INVALID_ARG;
  if (T > 0 && (logits == nullptr || topk_ids == nullptr || topk_weights == nullptr))
    return MOE_ERR_INVALID_ARG;
  if (E > kMaxExperts) return MOE_ERR_UNSUPPORTED;
  if (T == 0) return MOE_OK;
  if (T / 8 >= (static_cast<int64_t>(1) << 31) - 1) return MOE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState *d = nullptr;
  int rc = current_device(&d);
  if (rc != MOE_OK) return rc;
  CallCtx ctx{static_cast<cudaStream_t>(stream), "", nullptr};
  moe::StageHook hook = make_hook(&ctx);
  hook.begin("route");
  cudaError_t e = moe::launch_route(logits, T, E, k, renorm, topk_ids, topk_weights, ctx.stream);
  return to_code(hook.end(e));
}

int moe_permute_ex(const int32_t *topk_ids, int64_t T, int k, int E, int32_t *sorted_rows,
                   int32_t *expert_offsets, int32_t *inv, const uint16_t *hidden, int H,
                   uint16_t *xs, int kernel, void *stream) {
  if (T < 0 || k < 1 || E < 1) return MOE_ERR_INVALID_ARG;
  if (expert_offsets == nullptr || (T > 0 && (topk_ids == nullptr || sorted_rows == nullptr)))
    return MOE_ERR_INVALID_ARG;
  if (kernel != MOE_PERMUTE_AUTO && kernel != MOE_PERMUTE_SINGLE && kernel != MOE_PERMUTE_MULTI)
    return MOE_ERR_INVALID_ARG;
  if ((hidden == nullptr) != (xs == nullptr)) return MOE_ERR_INVALID_ARG;
  if (xs != nullptr && (H < 1 || !aligned16(hidden) || !aligned16(xs)))
    return MOE_ERR_INVALID_ARG;
  if (E > kMaxExperts || (xs != nullptr && H % 128 != 0)) return MOE_ERR_UNSUPPORTED;
  const int64_t n = T * k;
  if (n >= (static_cast<int64_t>(1) << 31)) return MOE_ERR_UNSUPPORTED;
  const bool single = kernel == MOE_PERMUTE_SINGLE ||
                      (kernel == MOE_PERMUTE_AUTO && moe::group_supported(n));
  if (single && !moe::group_supported(n)) return MOE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState *d = nullptr;
  int rc = current_device(&d);
  if (rc != MOE_OK) return rc;
  // chunk counts of the three-kernel grouping
  if ((rc = ensure_workspace(*d, permute_ws_bytes(n, E))) != MOE_OK) return rc;
  Carver cv{static_cast<char *>(d->ws)};
  int32_t *chunk_counts = cv.take<int32_t>(std::max(moe::permute_num_chunks(n), 1) * static_cast<size_t>(E));
  CallCtx ctx{static_cast<cudaStream_t>(stream), "", nullptr};
  moe::StageHook hook = make_hook(&ctx);
  cudaError_t e;
  if (single) {
    e = moe::launch_group(topk_ids, n, E, k, expert_offsets, sorted_rows, inv, nullptr, hidden, H,
                          xs, nullptr, 0, d->num_sms, ctx.stream, hook);
  } else {
    e = moe::launch_permute(topk_ids, n, E, chunk_counts, expert_offsets, sorted_rows, inv,
                            nullptr, nullptr, 0, ctx.stream, hook);
    if (e == cudaSuccess && xs != nullptr)
      e = moe::launch_gather_rows(hidden, H, k, sorted_rows, expert_offsets, E, n, d->num_sms, xs,
                                  nullptr, 0, ctx.stream, hook);
  }
  return to_code(e);
}

int moe_permute(const int32_t *topk_ids, int64_t T, int k, int E, int32_t *sorted_rows,
                int32_t *expert_offsets, void *stream) {
  return moe_permute_ex(topk_ids, T, k, E, sorted_rows, expert_offsets, nullptr, nullptr, 0,
                        nullptr, MOE_PERMUTE_AUTO, stream);
}

}  // extern "C"

namespace {

static_assert(MOE_ACT_SILU == moe::kActSilu && MOE_ACT_GELU_TANH == moe::kActGeluTanh &&
                  MOE_ACT_SWIGLUOAI == moe::kActSwigluOai,
              "activation codes of the ABI and the kernels agree");

// FP8 E4M3 weights: codes in the layouts of w1 and w2, fp32 scales per row
// and block of `block` contraction elements.
struct Fp8Weights {
  const float *s1, *s2;
  int block;
};

// moe_forward, moe_forward_ex and moe_forward_fp8: the variant is (b1, b2,
// act); b1 and b2 may be null; fp8 non-null means w1/w2 hold E4M3 codes.
int forward_impl(const void *hidden_, const void *w1_, const void *w2_, const float *b1,
                 const float *b2, int act_kind, const float *topk_weights,
                 const int32_t *topk_ids, float *out, int64_t T, int H, int I, int E, int k,
                 void *stream, const Fp8Weights *fp8 = nullptr) {
  const uint16_t *hidden = static_cast<const uint16_t *>(hidden_);
  const uint16_t *w1 = static_cast<const uint16_t *>(w1_);
  const uint16_t *w2 = static_cast<const uint16_t *>(w2_);
  if (T < 0 || H < 1 || I < 1 || E < 1 || k < 1 || k > E) return MOE_ERR_INVALID_ARG;
  if (act_kind != MOE_ACT_SILU && act_kind != MOE_ACT_GELU_TANH && act_kind != MOE_ACT_SWIGLUOAI)
    return MOE_ERR_INVALID_ARG;
  if (T > 0 && (hidden == nullptr || w1 == nullptr || w2 == nullptr || topk_weights == nullptr ||
                topk_ids == nullptr || out == nullptr))
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(hidden) || !aligned16(w1) || !aligned16(w2) || !aligned16(out) ||
      !aligned16(b1) || !aligned16(b2))
    return MOE_ERR_INVALID_ARG;
  if (H % 128 != 0 || I % 128 != 0 || E > kMaxExperts || k > kMaxTopK) return MOE_ERR_UNSUPPORTED;
  if (fp8 != nullptr) {
    if (T > 0 && (fp8->s1 == nullptr || fp8->s2 == nullptr)) return MOE_ERR_INVALID_ARG;
    if (fp8->block < 1) return MOE_ERR_INVALID_ARG;
    if (fp8->block % 128 != 0 || H % fp8->block != 0 || I % fp8->block != 0)
      return MOE_ERR_UNSUPPORTED;
  }
  const int64_t n = T * k;
  if (n >= (static_cast<int64_t>(1) << 31)) return MOE_ERR_UNSUPPORTED;
  if (T == 0) return MOE_OK;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState *d = nullptr;
  int rc = current_device(&d);
  if (rc != MOE_OK) return rc;
  CallCtx ctx{static_cast<cudaStream_t>(stream), "", nullptr};
  moe::StageHook hook = make_hook(&ctx);

  bool small = false;
  if (T <= small_t_max() && moe::small_t_supported(H, I)) {
    cudaError_t e = moe::small_t_fits(T, H, I, E, k, fp8 != nullptr, &small);
    if (e != cudaSuccess) return to_code(e);
  }
  if (small) {
    const size_t need = align256(static_cast<size_t>(n) * I * sizeof(float));
    if ((rc = ensure_workspace(*d, need)) != MOE_OK) return rc;
    Carver cv{static_cast<char *>(d->ws)};
    float *act = cv.take<float>(static_cast<size_t>(n) * I);
    return to_code(moe::launch_small_t(
        hidden, w1, w2, fp8 ? fp8->s1 : nullptr, fp8 ? fp8->s2 : nullptr, fp8 ? fp8->block : 0,
        b1, b2, act_kind, topk_weights, topk_ids, act, out, T, H, I, E, k,
        d->status,
        reinterpret_cast<unsigned long long *>(reinterpret_cast<char *>(d->status) + 64),
        static_cast<uint64_t>(g_wait_limit_ns), ctx.stream, hook, g_timeline, g_timeline_cap));
  }

  cudaError_t e;
  // top-k <= 2: GEMM2 adds its rows straight into out and no P is needed
  const bool fuse_combine = k <= 2;
  // Copying the hidden rows into expert-sorted order costs k row copies per
  // token and lets GEMM1 run on CTA pairs with TMA operands; with few slots
  // per token that pays off.
  const bool gather_rows = k <= 2;
  const int64_t n_counters = moe::gemm_counter_count(n, E);
  const size_t need = permute_ws_bytes(n, E) + align256(static_cast<size_t>(n) * 4) +
                      align256(static_cast<size_t>(n) * I * 2) +
                      align256(static_cast<size_t>(n_counters) * 4) +
                      (gather_rows ? align256(static_cast<size_t>(n) * H * 2) : 0) +
                      (fuse_combine ? 0 : align256(static_cast<size_t>(n) * H * sizeof(float)));
  if ((rc = ensure_workspace(*d, need)) != MOE_OK) return rc;
  Carver cv{static_cast<char *>(d->ws)};
  int32_t *chunk_counts =
      cv.take<int32_t>(std::max(moe::permute_num_chunks(n), 1) * static_cast<size_t>(E));
  int32_t *sorted_rows = cv.take<int32_t>(std::max<int64_t>(n, 1));
  int32_t *inv = cv.take<int32_t>(std::max<int64_t>(n, 1));
  int32_t *expert_offsets = cv.take<int32_t>(E + 1);
  uint16_t *act = cv.take<uint16_t>(static_cast<size_t>(n) * I);
  int *counters = cv.take<int>(static_cast<size_t>(n_counters));
  uint16_t *xs = gather_rows ? cv.take<uint16_t>(static_cast<size_t>(n) * H) : nullptr;
  float *P = fuse_combine ? nullptr : cv.take<float>(static_cast<size_t>(n) * H);

  // grouping (and the sorted row copy): one kernel up to 8192 entries, the
  // three-kernel grouping and a separate copy above; either zeroes the
  // GEMMs' counters
  if (moe::group_supported(n)) {
    e = moe::launch_group(topk_ids, n, E, k, expert_offsets, sorted_rows, inv, d->status, hidden,
                          H, xs, counters, static_cast<int>(n_counters), d->num_sms, ctx.stream,
                          hook);
    if (e != cudaSuccess) return to_code(e);
  } else {
    e = moe::launch_permute(topk_ids, n, E, chunk_counts, expert_offsets, sorted_rows, inv,
                            d->status, counters, static_cast<int>(n_counters), ctx.stream, hook);
    if (e != cudaSuccess) return to_code(e);
    if (gather_rows &&
        (e = moe::launch_gather_rows(hidden, H, k, sorted_rows, expert_offsets, E, n, d->num_sms,
                                     xs, nullptr, 0, ctx.stream, hook)) != cudaSuccess)
      return to_code(e);
  }
  if (fp8 != nullptr) {
    // the grouped GEMMs run on bf16 copies of the chosen experts' weights
    // (the others are left as they are: no row of theirs is read)
    const size_t n1 = static_cast<size_t>(E) * 2 * I * H, n2 = static_cast<size_t>(E) * H * I;
    if ((rc = ensure_buffer(d->wq, d->wq_bytes, (n1 + n2) * 2)) != MOE_OK) return rc;
    uint16_t *wd1 = static_cast<uint16_t *>(d->wq), *wd2 = wd1 + n1;
    if ((e = moe::launch_dequant_e4m3(reinterpret_cast<const uint8_t *>(w1), fp8->s1,
                                      static_cast<int64_t>(E) * 2 * I, H, fp8->block, wd1,
                                      d->num_sms, ctx.stream, hook, expert_offsets,
                                      2 * I)) != cudaSuccess ||
        (e = moe::launch_dequant_e4m3(reinterpret_cast<const uint8_t *>(w2), fp8->s2,
                                      static_cast<int64_t>(E) * H, I, fp8->block, wd2,
                                      d->num_sms, ctx.stream, hook, expert_offsets, H)) !=
            cudaSuccess)
      return to_code(e);
    w1 = wd1;
    w2 = wd2;
  }
  moe::GroupedGemmArgs ga = {};
  ga.hidden = hidden;
  ga.w1 = w1;
  ga.w2 = w2;
  ga.sorted_rows = sorted_rows;
  ga.expert_offsets = expert_offsets;
  ga.xs = xs;
  ga.act = act;
  ga.out = out;
  ga.topk_weights = topk_weights;
  ga.P = P;
  ga.counters = counters;
  ga.T = T;
  ga.H = H;
  ga.I = I;
  ga.E = E;
  ga.k = k;
  ga.num_sms = d->num_sms;
  ga.status = d->status;
  ga.wait_limit_ns = static_cast<uint64_t>(g_wait_limit_ns);
  ga.timeline = g_timeline;
  ga.timeline_cap = g_timeline_cap;
  ga.b1 = b1;
  ga.b2 = b2;
  ga.act_kind = act_kind;
  if (gather_rows) {
    // One launch for both GEMMs fills GEMM1's last partial wave with GEMM2
    // tiles; with many waves that gain is small and two launches, each with
    // the deepest operand ring its shared memory allows, run faster.
    const int64_t tiles = ((n + 255) / 256) * (I / 128 + (H + 255) / 256);
    const bool one_launch = tiles <= kFusedMaxWaves * std::max(1, d->num_sms / 2);
    if ((e = moe::launch_fused_gemm(ga, one_launch, ctx.stream, hook)) != cudaSuccess)
      return to_code(e);
    if (!one_launch && (e = moe::launch_gemm2(ga, ctx.stream, hook)) != cudaSuccess)
      return to_code(e);
  } else {
    if ((e = moe::launch_gemm1_swiglu(ga, ctx.stream, hook)) != cudaSuccess) return to_code(e);
    if ((e = moe::launch_gemm2(ga, ctx.stream, hook)) != cudaSuccess) return to_code(e);
  }
  if (fuse_combine) return MOE_OK;
  e = moe::launch_combine(P, inv, topk_weights, out, T, H, k, d->status, ctx.stream, hook);
  return to_code(e);
}

}  // namespace

extern "C" {

int moe_forward(const uint16_t *hidden, const uint16_t *w1, const uint16_t *w2,
                const float *topk_weights, const int32_t *topk_ids, float *out, int64_t T, int H,
                int I, int E, int k, void *stream) {
  return forward_impl(hidden, w1, w2, nullptr, nullptr, MOE_ACT_SILU, topk_weights, topk_ids,
                      out, T, H, I, E, k, stream);
}

int moe_forward_fp8(const uint16_t *hidden, const uint8_t *w1, const float *w1_scale,
                    const uint8_t *w2, const float *w2_scale, int block,
                    const float *topk_weights, const int32_t *topk_ids, float *out, int64_t T,
                    int H, int I, int E, int k, void *stream) {
  const Fp8Weights q{w1_scale, w2_scale, block};
  return forward_impl(hidden, w1, w2, nullptr, nullptr, MOE_ACT_SILU, topk_weights, topk_ids,
                      out, T, H, I, E, k, stream, &q);
}

int moe_forward_ex(const uint16_t *hidden, const uint16_t *w1, const uint16_t *w2,
                   const float *b1, const float *b2, int act, const float *topk_weights,
                   const int32_t *topk_ids, float *out, int64_t T, int H, int I, int E, int k,
                   void *stream) {
  return forward_impl(hidden, w1, w2, b1, b2, act, topk_weights, topk_ids, out, T, H, I, E, k,
                      stream);
}

// ---------------------------------------------------------------- expert parallelism

int moe_ep_dispatch_plan(const int32_t *topk_ids, int64_t T, int k, int E, int world,
                         int32_t *send_rows, int32_t *send_offsets, int32_t *inv, void *stream) {
  if (T < 0 || k < 1 || E < 1 || world < 1 || k > E) return MOE_ERR_INVALID_ARG;
  if (send_offsets == nullptr ||
      (T > 0 && (topk_ids == nullptr || send_rows == nullptr || inv == nullptr)))
    return MOE_ERR_INVALID_ARG;
  if (E > kMaxExperts || world > moe::kEpMaxWorld || E % world != 0) return MOE_ERR_UNSUPPORTED;
  const int64_t n = T * k;
  if (n >= (static_cast<int64_t>(1) << 31)) return MOE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState *d = nullptr;
  int rc = current_device(&d);
  if (rc != MOE_OK) return rc;
  if ((rc = ensure_workspace(*d, permute_ws_bytes(n, world) +
                                     align256(static_cast<size_t>(std::max<int64_t>(n, 1)) * 4))) !=
      MOE_OK)
    return rc;
  Carver cv{static_cast<char *>(d->ws)};
  int32_t *chunk_counts =
      cv.take<int32_t>(std::max(moe::permute_num_chunks(n), 1) * static_cast<size_t>(world));
  int32_t *owner = cv.take<int32_t>(std::max<int64_t>(n, 1));
  CallCtx ctx{static_cast<cudaStream_t>(stream), "", nullptr};
  moe::StageHook hook = make_hook(&ctx);
  cudaError_t e = cudaSuccess;
  if (n > 0) e = moe::launch_ep_owner(topk_ids, n, E, world, owner, ctx.stream, hook);
  // the (token, slot) rows grouped by owner rank, stable: the send order
  if (e == cudaSuccess) {
    if (moe::group_supported(n))
      e = moe::launch_group(owner, n, world, k, send_offsets, send_rows, inv, d->status, nullptr,
                            0, nullptr, nullptr, 0, d->num_sms, ctx.stream, hook);
    else
      e = moe::launch_permute(owner, n, world, chunk_counts, send_offsets, send_rows, inv,
                              d->status, nullptr, 0, ctx.stream, hook);
  }
  return to_code(e);
}

namespace {

// Host route tables of moe_ep_pack / moe_ep_return into the kernels' form.
int ep_routes(int world, const int64_t *offsets, const int64_t *row0, moe::EpRoutes *r) {
  if (world < 1 || world > moe::kEpMaxWorld || offsets == nullptr || row0 == nullptr)
    return MOE_ERR_INVALID_ARG;
  *r = moe::EpRoutes{};
  for (int i = 0; i <= world; ++i) {
    if (offsets[i] < 0 || (i > 0 && offsets[i] < offsets[i - 1])) return MOE_ERR_INVALID_ARG;
    r->off[i] = offsets[i];
  }
  if (offsets[0] != 0) return MOE_ERR_INVALID_ARG;
  for (int i = 0; i < world; ++i) {
    if (row0[i] < 0) return MOE_ERR_INVALID_ARG;
    r->row0[i] = row0[i];
  }
  return MOE_OK;
}

}  // namespace

int moe_ep_pack(const uint16_t *hidden, int H, const int32_t *topk_ids, int64_t T, int k, int E,
                int world, const int32_t *send_rows, const int64_t *send_offsets,
                uint16_t *const *dst_x, int32_t *const *dst_eid, const int64_t *dst_row0,
                void *stream) {
  if (T < 0 || H < 1 || k < 1 || E < 1 || world < 1 || dst_x == nullptr || dst_eid == nullptr)
    return MOE_ERR_INVALID_ARG;
  if (H % 128 != 0 || world > moe::kEpMaxWorld || E % world != 0) return MOE_ERR_UNSUPPORTED;
  moe::EpRoutes r;
  int rc = ep_routes(world, send_offsets, dst_row0, &r);
  if (rc != MOE_OK) return rc;
  if (r.off[world] > T * k) return MOE_ERR_INVALID_ARG;
  if (r.off[world] == 0) return MOE_OK;
  if (hidden == nullptr || topk_ids == nullptr || send_rows == nullptr || !aligned16(hidden))
    return MOE_ERR_INVALID_ARG;
  for (int i = 0; i < world; ++i) {
    if (r.off[i + 1] == r.off[i]) continue;
    if (dst_x[i] == nullptr || dst_eid[i] == nullptr || !aligned16(dst_x[i]))
      return MOE_ERR_INVALID_ARG;
    r.x[i] = dst_x[i];
    r.eid[i] = dst_eid[i];
  }
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState *d = nullptr;
  if ((rc = current_device(&d)) != MOE_OK) return rc;
  CallCtx ctx{static_cast<cudaStream_t>(stream), "", nullptr};
  moe::StageHook hook = make_hook(&ctx);
  return to_code(moe::launch_ep_pack(hidden, H, topk_ids, k, E, world, send_rows, r, d->num_sms,
                                     ctx.stream, hook));
}

int moe_ep_return(const float *y, int H, int world, const int64_t *recv_offsets,
                  float *const *dst_y, const int64_t *dst_row0, void *stream) {
  if (H < 1 || world < 1 || dst_y == nullptr) return MOE_ERR_INVALID_ARG;
  if (H % 128 != 0 || world > moe::kEpMaxWorld) return MOE_ERR_UNSUPPORTED;
  moe::EpRoutes r;
  int rc = ep_routes(world, recv_offsets, dst_row0, &r);
  if (rc != MOE_OK) return rc;
  if (r.off[world] == 0) return MOE_OK;
  if (y == nullptr || !aligned16(y)) return MOE_ERR_INVALID_ARG;
  for (int i = 0; i < world; ++i) {
    if (r.off[i + 1] == r.off[i]) continue;
    if (dst_y[i] == nullptr || !aligned16(dst_y[i])) return MOE_ERR_INVALID_ARG;
    r.y[i] = dst_y[i];
  }
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState *d = nullptr;
  if ((rc = current_device(&d)) != MOE_OK) return rc;
  CallCtx ctx{static_cast<cudaStream_t>(stream), "", nullptr};
  moe::StageHook hook = make_hook(&ctx);
  return to_code(moe::launch_ep_return(y, H, world, r, d->num_sms, ctx.stream, hook));
}

int moe_ep_combine(const float *y_back, const int32_t *inv, const float *topk_weights, float *out,
                   int64_t T, int H, int k, void *stream) {
  if (T < 0 || H < 1 || k < 1) return MOE_ERR_INVALID_ARG;
  if (T > 0 && (y_back == nullptr || inv == nullptr || topk_weights == nullptr || out == nullptr))
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(y_back) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
  if (H % 128 != 0 || k > kMaxTopK) return MOE_ERR_UNSUPPORTED;
  if (T == 0) return MOE_OK;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState *d = nullptr;
  int rc = current_device(&d);
  if (rc != MOE_OK) return rc;
  CallCtx ctx{static_cast<cudaStream_t>(stream), "", nullptr};
  moe::StageHook hook = make_hook(&ctx);
  return to_code(moe::launch_combine(y_back, inv, topk_weights, out, T, H, k, d->status,
                                     ctx.stream, hook));
}

int moe_get_device_status(void *stream, uint32_t *status) {
  if (status == nullptr) return MOE_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState *d = nullptr;
  int rc = current_device(&d);
  if (rc != MOE_OK) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t v = 0;
  cudaError_t e = cudaStreamSynchronize(s);
  if (e == cudaSuccess) e = cudaMemcpy(&v, d->status, sizeof(v), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemset(d->status, 0, sizeof(v));
  if (e != cudaSuccess) return to_code(e);
  *status = v;
  return MOE_OK;
}

int moe_set_small_t_max(int n) {
  std::lock_guard<std::mutex> lock(g_mu);
  const int prev = small_t_max();
  g_small_t_max = std::min(16, std::max(0, n));
  return prev;
}

int moe_set_sync_each_stage(int on) {
  std::lock_guard<std::mutex> lock(g_mu);
  const int prev = sync_each() ? 1 : 0;
  g_sync_each = on ? 1 : 0;
  return prev;
}

int64_t moe_set_wait_limit_ns(int64_t ns) {
  std::lock_guard<std::mutex> lock(g_mu);
  const int64_t prev = g_wait_limit_ns;
  g_wait_limit_ns = ns > 0 ? ns : 2000000000LL;
  return prev;
}

const char *moe_last_failed_stage(void) { return g_failed_stage; }

int moe_timeline(void *buf, int64_t capacity) {
  if (buf != nullptr && (capacity < 1 || (reinterpret_cast<uintptr_t>(buf) & 7u) != 0))
    return MOE_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(g_mu);
  g_timeline = static_cast<uint64_t *>(buf);
  g_timeline_cap = buf != nullptr ? capacity : 0;
  return MOE_OK;
}

int moe_debug_wait_timeout(int64_t limit_ns, void *stream) {
  if (limit_ns <= 0 || limit_ns > 10000000000LL) return MOE_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState *d = nullptr;
  int rc = current_device(&d);
  if (rc != MOE_OK) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = moe::launch_wait_probe(d->status, static_cast<uint64_t>(limit_ns), s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  uint32_t v = 0;
  if (e == cudaSuccess) e = cudaMemcpy(&v, d->status, sizeof(v), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return to_code(e);
  return (v & MOE_STATUS_TIMEOUT) ? MOE_ERR_TIMEOUT : MOE_OK;
}

int moe_profile_enable(int on) {
  std::lock_guard<std::mutex> lock(g_mu);
  const int prev = g_prof ? 1 : 0;
  g_prof = on != 0;
  return prev;
}

static void profile_collect() {
  if (g_prof_pending.empty()) return;
  cudaDeviceSynchronize();
  for (const ProfEvent &pe : g_prof_pending) {
    float ms = 0.f;
    cudaEventElapsedTime(&ms, pe.a, pe.b);
    size_t i = 0;
    while (i < g_prof_names.size() && g_prof_names[i] != pe.name) ++i;
    if (i == g_prof_names.size()) {
      g_prof_names.emplace_back(pe.name);
      g_prof_count.push_back(0);
      g_prof_ms.push_back(0.0);
    }
    g_prof_count[i] += 1;
    g_prof_ms[i] += ms;
    g_event_pool.push_back(pe.a);
    g_event_pool.push_back(pe.b);
  }
  g_prof_pending.clear();
  cudaGetLastError();
}

int moe_profile_reset(void) {
  std::lock_guard<std::mutex> lock(g_mu);
  profile_collect();
  g_prof_names.clear();
  g_prof_count.clear();
  g_prof_ms.clear();
  return MOE_OK;
}

int moe_profile_read(int max_names, char (*names)[64], int64_t *launches, double *total_ms) {
  std::lock_guard<std::mutex> lock(g_mu);
  profile_collect();
  const int n = static_cast<int>(g_prof_names.size());
  for (int i = 0; i < n && i < max_names; ++i) {
    if (names != nullptr) {
      std::strncpy(names[i], g_prof_names[i].c_str(), 63);
      names[i][63] = '\0';
    }
    if (launches != nullptr) launches[i] = g_prof_count[i];
    if (total_ms != nullptr) total_ms[i] = g_prof_ms[i];
  }
  return n;
}

}  // extern "C"
