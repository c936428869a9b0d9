// noalloc.cu -- cc3d_forward_noalloc: the tensor-core causal conv for
// callers that cannot allocate device memory.
//
// Some callers must never call cudaMalloc: a serving process that hands out
// all device memory from a budget it reserved at start-up, a framework whose
// own caching allocator owns the device, or a latency-critical loop that
// cannot afford the implicit device synchronisation an allocation brings.
// cc3d_plan_create allocates (it keeps re-tiled weights in device memory),
// so those callers get this entry point instead: it keeps its only scratch,
// the re-tiled weights, in one fixed file-scope device array and allocates
// nothing.  The caller still passes every input and output.
//
// Limits and sharing rules (also stated in include/cc3d.h):
//   * the scratch is 8 MiB of re-tiled weights plus 16 KiB for a zero bias;
//     every GPU that loads the library holds it until the process exits;
//   * weights needing more than 8 MiB are refused with CC3D_ERR_TOO_LARGE;
//   * all calls on a device share the array, which keeps the last call's
//     contents; calls that overlap on the GPU race on it;
//   * the first call on a device looks up the array's device address; make
//     it before any stream capture.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <mutex>

#include "cc3d.h"
#include "internal.h"

namespace cc3d {
namespace {

constexpr size_t kNoAllocWeightBytes = size_t(8) << 20;  // re-tiled weights
constexpr size_t kNoAllocBiasBytes = size_t(16) << 10;   // zero bias, <= 4096 channels
constexpr size_t kNoAllocScratchBytes = kNoAllocWeightBytes + kNoAllocBiasBytes;

// The scratch itself.  In host code this name is only a stand-in for the
// symbol, never a device address: the address comes from
// cudaGetSymbolAddress, once per device, with that device current.
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
uint8_t *g_noalloc_ptr[64] = {nullptr};
int g_noalloc_sms[64] = {0};

// Device address of the scratch on the current device (set-up on first use).
cc3d_status scratch_for_current_device(uint8_t **ptr, int *sms) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return CC3D_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return CC3D_ERR_CUDA;
    if (major != 10 || minor != 0) return CC3D_ERR_UNSUPPORTED;
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return CC3D_ERR_CUDA;
    int n_sm = 0;
    if (cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return CC3D_ERR_CUDA;
    if (umma_prepare() != cudaSuccess) return CC3D_ERR_CUDA;
    if (!device_status_word()) return CC3D_ERR_CUDA;
    g_noalloc_sms[dev] = n_sm;
    g_noalloc_ptr[dev] = static_cast<uint8_t *>(p);
  }
  *ptr = g_noalloc_ptr[dev];
  *sms = g_noalloc_sms[dev];
  return CC3D_OK;
}

bool al16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlap(const void *a, size_t na, const void *b, size_t nb) {
  if (!a || !b || na == 0 || nb == 0) return false;
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

}  // namespace
}  // namespace cc3d

using namespace cc3d;

extern "C" cc3d_status cc3d_forward_noalloc(const cc3d_desc *d, const void *x, int t,
                                            const void *cache_in, void *y, void *cache_out,
                                            const void *residual, const void *next_cache_in,
                                            void *next_cache_out, void *stream_v) {
  // ---- descriptor: the bf16 tensor-core cases only --------------------------------
  if (!d || !d->weight || !x || !y) return CC3D_ERR_INVALID_ARG;
  if (d->n < 1 || d->c_in < 1 || d->c_out < 1 || d->h < 1 || d->w < 1 || d->max_t < 1 ||
      d->kt < 1 || d->kh < 1 || d->kw < 1 || t < 1 || t > d->max_t)
    return CC3D_ERR_INVALID_ARG;
  if (d->epi < CC3D_EPI_BIAS || d->epi > CC3D_EPI_BIAS_RMS) return CC3D_ERR_INVALID_ARG;
  const bool rms = d->epi == CC3D_EPI_BIAS_RMS_SILU || d->epi == CC3D_EPI_BIAS_RMS;
  if (rms && !d->gamma) return CC3D_ERR_INVALID_ARG;
  if ((d->epi == CC3D_EPI_BIAS_RESIDUAL) != (residual != nullptr)) return CC3D_ERR_INVALID_ARG;
  if (!rms && (next_cache_in || next_cache_out))
    return CC3D_ERR_INVALID_ARG;
  if (d->stride_t < 1 || d->stride_t > 2 || d->stride_h != 1 || d->stride_w != 1 ||
      d->dil_t != 1 || d->dil_h != 1 || d->dil_w != 1 || d->groups != 1 ||
      d->dtype != CC3D_BF16)
    return CC3D_ERR_UNSUPPORTED;
  if (d->kh != d->kw || (d->kh != 1 && d->kh != 3) || d->kt > 3 || d->pad_h != d->kh / 2 ||
      d->pad_w != d->kw / 2)
    return CC3D_ERR_UNSUPPORTED;
  if (d->c_in % 32 != 0 || d->c_out % 16 != 0) return CC3D_ERR_UNSUPPORTED;
  if (rms && d->c_out > 256 && (d->c_out > 512 || d->c_out % 32 != 0))
    return CC3D_ERR_UNSUPPORTED;
  const int taps = d->kt * d->kh * d->kw;
  const size_t wbytes = size_t(2) * d->c_out * d->c_in * taps;
  if (wbytes > kNoAllocWeightBytes || size_t(4) * d->c_out > kNoAllocBiasBytes)
    return CC3D_ERR_TOO_LARGE;

  // ---- pointers -------------------------------------------------------------------------
  if (!al16(x) || !al16(y) || !al16(cache_in) || !al16(cache_out) || !al16(residual) ||
      !al16(next_cache_in) || !al16(next_cache_out))
    return CC3D_ERR_ALIGNMENT;
  const int front = d->kt - 1;
  const size_t in_frame = size_t(d->h) * d->w * d->c_in * 2;
  const size_t out_frame = size_t(d->h) * d->w * d->c_out * 2;
  const int t_out = (t - 1) / d->stride_t + 1;  // frames of y
  const size_t xb = in_frame * d->n * t, yb = out_frame * d->n * t_out;
  const size_t cb = in_frame * d->n * front, ncb = out_frame * d->n * 2;
  if (overlap(cache_out, cb, cache_in, cb) || overlap(cache_out, cb, x, xb) ||
      overlap(cache_out, cb, y, yb) || overlap(next_cache_out, ncb, next_cache_in, ncb) ||
      overlap(next_cache_out, ncb, y, yb) || overlap(next_cache_out, ncb, x, xb) ||
      overlap(y, yb, x, xb))
    return CC3D_ERR_ALIAS;

  uint8_t *scratch = nullptr;
  int n_sm = 0;
  cc3d_status st = scratch_for_current_device(&scratch, &n_sm);
  if (st != CC3D_OK) return st;
  int *status = device_status_word();
  cudaStream_t stream = static_cast<cudaStream_t>(stream_v);

  // ---- tiles: the same choice cc3d_plan_create makes --------------------------------
  UmmaLayer L;
  std::memset(&L, 0, sizeof L);
  if (!choose_umma_config(d->n, d->c_in, d->c_out, d->h, d->w, d->kt, d->kh,
                          rms, (d->max_t - 1) / d->stride_t + 1, n_sm,
                          &L.cfg))
    return CC3D_ERR_UNSUPPORTED;
  const UmmaConfig &cfg = L.cfg;
  if (cfg.pair || cfg.xs == 2) {
    L.max_clusters = umma_max_clusters(cfg, d->kh);
    if (L.max_clusters < 1) return CC3D_ERR_CUDA;
  }
  const int kc = cfg.kc, nt = cfg.nt;

  // ---- scratch: re-tiled weights (every call), zero bias when none is given --------
  uint8_t *wimg = scratch;
  float *zero_bias = reinterpret_cast<float *>(scratch + kNoAllocWeightBytes);
  cudaError_t e = launch_repack_umma(static_cast<const __nv_bfloat16 *>(d->weight), wimg,
                                     d->c_out, d->c_in, taps, nt, kc, cfg.pair,
                                     taps * (d->c_in / kc), 0, stream);
  if (e == cudaSuccess && !d->bias)
    e = cudaMemsetAsync(zero_bias, 0, sizeof(float) * d->c_out, stream);
  if (e != cudaSuccess) return CC3D_ERR_CUDA;
  CUtensorMap mw;
  if (cfg.pair && !encode_weight_map(&mw, wimg,
                                     static_cast<long long>(d->c_out) * taps * (d->c_in / 64),
                                     nt / 2))
    return CC3D_ERR_CUDA;

  // ---- the conv (one kernel, which also writes cache_out and next_cache_out) ---------
  L.n = d->n; L.c_in = d->c_in; L.c_out = d->c_out; L.h = d->h; L.w = d->w;
  L.kt = d->kt; L.kh = d->kh; L.kw = d->kw; L.pad_h = d->pad_h; L.pad_w = d->pad_w;
  L.stride_t = d->stride_t;
  L.s2 = 0;
  L.epi = static_cast<int>(d->epi);
  L.sm_count = n_sm;
  L.wimg = wimg;
  L.map_w = &mw;
  L.bias = d->bias ? d->bias : zero_bias;
  L.gamma = d->gamma;
  L.beta = d->beta;
  UmmaCall c{};
  c.x = x; c.t = t; c.cache_in = cache_in; c.y = y; c.cache_out = cache_out;
  c.residual = residual; c.ncache_in = next_cache_in; c.ncache_out = next_cache_out;
  c.x_sc = nullptr;
  uint64_t tiles = 0;
  e = run_umma_layer(L, c, status, stream, &tiles);
  return e == cudaSuccess ? CC3D_OK : CC3D_ERR_CUDA;
}
