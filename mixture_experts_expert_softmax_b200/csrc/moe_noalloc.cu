// moe_noalloc.cu -- moe_forward_small_noalloc: the small-batch (GEMV) form
// of moe_forward that never allocates device memory.
//
// Who needs it: callers whose device memory is planned up front and must not
// change afterwards -- a serving runtime that carves every buffer out of one
// reservation at start-up, or a latency-critical decode loop that cannot
// afford the device-wide synchronisation that cudaFree performs when the
// regular entry points grow their workspace.  Such callers pass inputs and
// outputs as usual; the only scratch this path needs (the bf16 SwiGLU
// intermediate of at most MOE_NOALLOC_MAX_ACT values, plus a status word)
// lives in a fixed __device__ array of this file, which every GPU that loads
// the library keeps until the process exits.
//
// Host code cannot use the array's name as a device address (on the host it
// names a stand-in object), so the first call on each device looks the
// address up with cudaGetSymbolAddress while that device is current and
// caches it; later calls reuse the cached address.
#include <mutex>

#include "moe.h"
#include "moe_internal.h"

namespace {

constexpr int kNoAllocMaxDevices = 64;
constexpr size_t kStatusBytes = 256;
constexpr size_t kScratchBytes =
    kStatusBytes + static_cast<size_t>(MOE_NOALLOC_MAX_ACT) * sizeof(float);

// [0, 256): status word the kernel may raise bits in (not reported back) at
// byte 0, and at byte 64 the kernel's grid-barrier counter, which starts at
// zero when the module loads and only ever advances (each launch adds its
// grid size and derives its own barrier target from the value it reads);
// [256, ...): the act scratch, T*k*I fp32 values.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

std::mutex g_noalloc_mu;
void *g_noalloc_addr[kNoAllocMaxDevices] = {};

}  // namespace

extern "C" int moe_forward_small_noalloc(const uint16_t *hidden, const uint16_t *w1,
                                         const uint16_t *w2, const float *topk_weights,
                                         const int32_t *topk_ids, float *out, int64_t T, int H,
                                         int I, int E, int k, void *stream) {
  if (T < 0 || H < 1 || I < 1 || E < 1 || k < 1 || k > E) return MOE_ERR_INVALID_ARG;
  if (T > 0 && (hidden == nullptr || w1 == nullptr || w2 == nullptr || topk_weights == nullptr ||
                topk_ids == nullptr || out == nullptr))
    return MOE_ERR_INVALID_ARG;
  // the kernel moves rows with 16-byte bulk copies and vector accesses
  if (((reinterpret_cast<uintptr_t>(hidden) | reinterpret_cast<uintptr_t>(w1) |
        reinterpret_cast<uintptr_t>(w2) | reinterpret_cast<uintptr_t>(out)) &
       15u) != 0)
    return MOE_ERR_INVALID_ARG;
  if (H % 128 != 0 || I % 128 != 0 || E > 1024 || k > 16 || !moe::small_t_supported(H, I))
    return MOE_ERR_UNSUPPORTED;
  if (T > MOE_NOALLOC_MAX_T ||
      T * static_cast<int64_t>(k) * static_cast<int64_t>(I) > MOE_NOALLOC_MAX_ACT)
    return MOE_ERR_SCRATCH_LIMIT;
  if (T == 0) return MOE_OK;

  int dev = -1, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoAllocMaxDevices ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_NO_DEVICE;
  }
  if (major != 10 || minor != 0) return MOE_ERR_NO_DEVICE;

  // shapes whose token vectors and per-CTA buffers do not fit the kernel's
  // shared memory are not a CUDA failure but a limit of this path
  bool fits = false;
  if (moe::small_t_fits(T, H, I, E, k, false, &fits) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  if (!fits) return MOE_ERR_UNSUPPORTED;

  void *base = nullptr;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  {
    if (g_noalloc_addr[dev] == nullptr) {
      void *p = nullptr;
      if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
      }
      g_noalloc_addr[dev] = p;
    }
    base = g_noalloc_addr[dev];
  }
  // Nothing has to be cleared between calls: every act value the second
  // phase reads is written by the first phase of the same call, and the
  // grid-barrier counter only ever advances by whole grids.
  uint32_t *status = static_cast<uint32_t *>(base);
  unsigned long long *grid_sync =
      reinterpret_cast<unsigned long long *>(static_cast<char *>(base) + 64);
  float *act = reinterpret_cast<float *>(static_cast<char *>(base) + kStatusBytes);
  moe::StageHook hook;
  hook.pdl = true;
  const cudaError_t e =
      moe::launch_small_t(hidden, w1, w2, nullptr, nullptr, 0, nullptr, nullptr, moe::kActSilu,
                          topk_weights,
                          topk_ids, act, out, T, H, I, E, k, status,
                          grid_sync, 2000000000ull, static_cast<cudaStream_t>(stream), hook);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}
