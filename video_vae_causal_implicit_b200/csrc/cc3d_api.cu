// cc3d_api.cu -- the C ABI of libcc3d.so (declared in include/cc3d.h):
// descriptor validation, plan-time weight re-tiling, TMA tensor-map
// encoding, kernel selection and launch, the residual block, route
// counters and the device status word.
//
// Gating mirrors the fast-path rule of the "cache-aware video decoder
// lowering" summary (5-D tensors, temporal stride 1, one group): anything
// else is refused with CC3D_ERR_UNSUPPORTED -- there is no fallback path.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include "cc3d.h"
#include "internal.h"

namespace cc3d {

// Device status word: non-zero after a bounded device wait ran out.
__device__ int g_status_word;

namespace {

std::atomic<uint64_t> g_launches{0};

std::mutex g_mu;
int *g_status_ptr[64] = {nullptr};

int *status_ptr() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_status_ptr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return nullptr;
    g_status_ptr[dev] = static_cast<int *>(p);
  }
  return g_status_ptr[dev];
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }();
  return fn;
}

bool is_sm100() {
  int dev = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return false;
  if (cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return false;
  return major == 10 && minor == 0;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlaps(const void *a, size_t na, const void *b, size_t nb) {
  if (!a || !b || na == 0 || nb == 0) return false;
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

// 5-D tensor map over an NDHWC buffer of bf16 (esz 2) or FP8 E4M3 bytes
// (esz 1): dims (C, W, H, T, N), a box of box_c channels x box_w x box_h x
// 1 x 1, zero fill out of bounds.  Boxes of 128-byte pixel rows (64 bf16 or
// 128 E4M3 channels) land 128-byte swizzled, 8-channel bf16 boxes plain.
bool encode_act_map(CUtensorMap *m, const void *base, int c, int w, int h, int t, int n,
                    int box_w, int box_h, int box_c, int esz = 2) {
  const bool sw = box_c * esz == 128;
  if (!(esz == 2 && (box_c == 8 || box_c == 64)) && !(esz == 1 && box_c == 128)) return false;
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t e = static_cast<cuuint64_t>(esz);
  cuuint64_t dims[5] = {(cuuint64_t)c, (cuuint64_t)w, (cuuint64_t)h, (cuuint64_t)t,
                        (cuuint64_t)n};
  cuuint64_t strides[4] = {(cuuint64_t)c * e, (cuuint64_t)c * e * w, (cuuint64_t)c * e * w * h,
                           (cuuint64_t)c * e * w * h * t};
  cuuint32_t box[5] = {(cuuint32_t)box_c, (cuuint32_t)box_w, (cuuint32_t)box_h, 1, 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(m, esz == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                  5, const_cast<void *>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE,
                  sw ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// The same map walking every other pixel in W and H (element strides 2):
// a box of box_c channels x box_w x box_h pixels of the stride-2 lattice
// that starts at the box's first pixel.
bool encode_act_map_s2(CUtensorMap *m, const void *base, int c, int w, int h, int t, int n,
                       int box_w, int box_h, int box_c) {
  if (box_c != 8 && box_c != 64) return false;
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[5] = {(cuuint64_t)c, (cuuint64_t)w, (cuuint64_t)h, (cuuint64_t)t,
                        (cuuint64_t)n};
  cuuint64_t strides[4] = {(cuuint64_t)c * 2, (cuuint64_t)c * 2 * w, (cuuint64_t)c * 2 * w * h,
                           (cuuint64_t)c * 2 * w * h * t};
  // (the box counts traversed elements: 2 * box pixels at stride 2)
  cuuint32_t box[5] = {(cuuint32_t)box_c, 2u * (cuuint32_t)box_w, 2u * (cuuint32_t)box_h, 1, 1};
  cuuint32_t estr[5] = {1, 2, 2, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void *>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  box_c == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 4-D bf16 tensor map over an NDHWC buffer with few channels: dims
// (W*C, H, T, N), a box of `row` elements x `box_h` rows x 1 x 1.
bool encode_thin_map(CUtensorMap *m, const void *base, int c, int w, int h, int t, int n,
                     int row, int box_h) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t wc = static_cast<cuuint64_t>(w) * c;
  cuuint64_t dims[4] = {wc, (cuuint64_t)h, (cuuint64_t)t, (cuuint64_t)n};
  cuuint64_t strides[3] = {wc * 2, wc * 2 * h, wc * 2 * h * t};
  cuuint32_t box[4] = {(cuuint32_t)row, (cuuint32_t)box_h, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Store map over y (NDHWC bf16): dims (C, W, H, T, N), a box of 32 channels
// x 8 columns x 16 rows with the 64-byte swizzle.
bool encode_store_map(CUtensorMap *m, const void *base, int c, int w, int h, int t, int n) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[5] = {(cuuint64_t)c, (cuuint64_t)w, (cuuint64_t)h, (cuuint64_t)t,
                        (cuuint64_t)n};
  cuuint64_t strides[4] = {(cuuint64_t)c * 2, (cuuint64_t)c * 2 * w, (cuuint64_t)c * 2 * w * h,
                           (cuuint64_t)c * 2 * w * h * t};
  cuuint32_t box[5] = {32, 8, 16, 1, 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void *>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                  CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

// Bound of every device-side wait, read once per process from
// CC3D_WAIT_LIMIT_US (microseconds; default 2 s).
unsigned long long wait_limit_ns() {
  static unsigned long long v = [] {
    const char *s = std::getenv("CC3D_WAIT_LIMIT_US");
    unsigned long long us = s ? std::strtoull(s, nullptr, 10) : 0ull;
    if (us == 0) us = 2000000ull;
    return us * 1000ull;
  }();
  return v;
}

cudaError_t run_umma_layer(const UmmaLayer &L, const UmmaCall &c, int *status,
                           cudaStream_t stream, uint64_t *tiles_out) {
  const UmmaConfig &cfg = L.cfg;
  CUtensorMap mx, mc;
  const int front = L.kt - 1;  // frames of the causal cache (0 for the stride-2 spatial conv)
  const int tile_w = umma_tile_w() * cfg.sub;
  // the kernel's spatial kernel: kh x kw, or for stride 2 the 2 x 2 views
  // of the input's four stride-2 phases
  const int ks = L.s2 ? 2 : L.kh;
  const int h_out = L.s2 ? L.h / 2 : L.h, w_out = L.s2 ? L.w / 2 : L.w;
  const int t_out = (c.t - 1) / L.stride_t + 1;
  // (a pair's CTA loads the halo of its own 8-column half)
  const int box_w = umma_halo_box_w(cfg.kc, cfg.pair ? 1 : cfg.sub, ks);
  const int box_h = umma_tile_h() + ks - 1;
  const int box_c = umma_halo_box_c(cfg.kc);
  const int esz = L.e4m3 ? 1 : 2;  // bytes per input element
  if (!(L.s2 ? encode_act_map_s2(&mx, c.x, L.c_in, L.w, L.h, c.t, L.n, box_w, box_h, box_c)
             : encode_act_map(&mx, c.x, L.c_in, L.w, L.h, c.t, L.n, box_w, box_h, box_c, esz)))
    return cudaErrorInvalidValue;
  const bool has_cache = c.cache_in && front > 0;
  if (has_cache) {
    if (!encode_act_map(&mc, c.cache_in, L.c_in, L.w, L.h, front, L.n, box_w, box_h, box_c, esz))
      return cudaErrorInvalidValue;
  } else {
    mc = mx;
  }
  CUtensorMap msc = mx;  // the conv_shortcut's input: same boxes, c_sc channels
  if (L.c_sc > 0 && !encode_act_map(&msc, c.x_sc, L.c_sc, L.w, L.h, c.t, L.n, box_w, box_h, box_c))
    return cudaErrorInvalidValue;
  UmmaArgs a;
  std::memset(&a, 0, sizeof a);
  a.wimg = L.wimg;
  a.bias = L.bias;
  a.gamma = L.gamma;
  a.beta = L.beta;
  a.residual = static_cast<const __nv_bfloat16 *>(c.residual);
  a.y = static_cast<__nv_bfloat16 *>(c.y);
  a.status = status;
  a.wait_limit_ns = wait_limit_ns();
  a.n = L.n; a.t = t_out; a.h = h_out; a.w = w_out; a.c_in = L.c_in; a.c_out = L.c_out;
  a.kt = L.s2 ? 4 : L.kt; a.kh = ks; a.kw = ks; a.pad_h = L.pad_h; a.pad_w = L.pad_w;
  a.stride_t = L.stride_t;
  a.s2 = L.s2;
  a.vec32 = (reinterpret_cast<uintptr_t>(c.y) & 31u) == 0 ? 1 : 0;
  a.b_resident = cfg.b_resident;
  a.c_sc = L.c_sc;
  a.n_cc_sc = L.n_cc_sc;
  a.nt = cfg.nt; a.n_ntiles = cfg.n_ntiles;
  a.sub = cfg.sub; a.nbuf = cfg.nbuf; a.g_taps = cfg.g_taps; a.pair = cfg.pair;
  a.tiles_w = (w_out + tile_w - 1) / tile_w;
  a.tiles_h = (h_out + umma_tile_h() - 1) / umma_tile_h();
  a.na = cfg.na; a.nb = cfg.nb; a.tmem_cols = cfg.tmem_cols;
  a.epi = c.y2 ? 4 : L.epi;
  a.has_cache = has_cache ? 1 : 0;
  // the frame caches, written by the kernel's epilogue
  a.x_in = static_cast<const uint8_t *>(c.x);
  a.t_in = c.t;
  a.cache_frames = front;
  a.cache_in = static_cast<const uint8_t *>(has_cache ? c.cache_in : nullptr);
  a.cache_out = front > 0 ? static_cast<uint8_t *>(c.cache_out) : nullptr;
  a.in_esz = esz;
  a.oscale = L.e4m3 ? L.oscale : nullptr;
  a.ncache_in = static_cast<const __nv_bfloat16 *>(c.ncache_in);
  a.ncache_out = static_cast<__nv_bfloat16 *>(c.ncache_out);
  a.nc_vec32 = (reinterpret_cast<uintptr_t>(c.ncache_out) & 31u) == 0 ? 1 : 0;
  a.xs = cfg.xs;
  a.y2 = static_cast<__nv_bfloat16 *>(c.y2);
  a.y2_vec32 = (reinterpret_cast<uintptr_t>(c.y2) & 31u) == 0 ? 1 : 0;
  if (c.y2) {
    a.gamma = c.gamma2;
    a.beta = nullptr;
  }
  const uint64_t tiles = static_cast<uint64_t>(L.n) * t_out * a.tiles_h * a.tiles_w * a.n_ntiles;
  uint64_t grid;
  if (cfg.pair || cfg.xs == 2) {
    // one cluster per tile (pair) or per M tile (xs: its two N tiles), at
    // most as many clusters as fit at once
    const uint64_t need = cfg.pair ? tiles : tiles / 2;
    const uint64_t clusters = static_cast<uint64_t>(L.max_clusters);
    grid = (need < clusters ? need : clusters) * 2;
  } else {
    const uint64_t slots = static_cast<uint64_t>(L.sm_count) * cfg.ctas_per_sm;
    grid = tiles < slots ? tiles : slots;
  }
  *tiles_out = tiles;
  const cudaError_t e = launch_conv_umma(mx, mc, cfg.pair ? *L.map_w : mx, msc, a, cfg.kc,
                                         static_cast<unsigned>(grid), stream);
  count_launch();
  return e;
}

int *device_status_word() { return status_ptr(); }

bool encode_activation_map(CUtensorMap *m, const void *base, int c, int w, int h, int t, int n,
                           int box_w, int box_h, int box_c) {
  return encode_act_map(m, base, c, w, h, t, n, box_w, box_h, box_c);
}

// 2-D tensor map over a weight image of `rows` rows of 128 bytes (64 bf16
// or 128 E4M3 channels): boxes of box_rows rows, 128-byte swizzled.
bool encode_weight_map(CUtensorMap *m, const void *img, long long rows, int box_rows, bool e4m3) {
  auto fn = encode_fn();
  if (!fn || rows < 1 || box_rows < 1 || box_rows > 256) return false;
  const cuuint64_t per_row = e4m3 ? 128 : 64;
  cuuint64_t dims[2] = {per_row, static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {128};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(per_row), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, e4m3 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                  const_cast<void *>(img), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace cc3d

using namespace cc3d;

struct cc3d_plan {
  cc3d_desc d;
  int variant;
  int device;
  // UMMA: the layer as the shared launcher sees it
  UmmaLayer layer;
  CUtensorMap map_w;  // pair: the weight image as 128-byte swizzled rows
  uint8_t *wimg;
  // Calls of one output frame (streamed chunks) run with the tiles chosen
  // for one frame when those differ from the plan's (chosen for max_t):
  // their own layer and weight image.  Every tile shape sums each output's
  // taps in the same order, so both give the same bytes.
  bool has_layer1;
  // per call shape [output frames][with a cache]: whether layer1 finishes it
  // sooner (the plan's tiles are chosen for max_t frames with a cache; a
  // call without one has cheap first frames, which may favour layer1's)
  std::vector<uint8_t> use_layer1;
  bool whole_rows;  // tiles hold whole C_out rows (an RMS epilogue may run)
  UmmaLayer layer1;
  CUtensorMap map_w1;
  uint8_t *wimg1;
  int c_sc;           // the residual block's fused 1x1x1 conv_shortcut (0: none)
  // fp32 / thin
  void *wraw;
  int kpad, thin_spec, nt, tmem_cols, sm_count, ctas_per_sm;
  float *bias, *gamma, *beta;
  float *oscale;  // FP8: s_x * s_w[c] per output channel
  cc3d_stats st;
  std::mutex mu;
  // cc3d_forward_host: staging slots (x and y of max_t frames each), an
  // upload and a download stream and their events, created on first use.
  // Three slots: a call's conv then waits only for the download of the
  // call three before it, which a long download (a whole sequence's y)
  // has usually finished by then.
  static constexpr int kHostSlots = 3;
  struct HostPipe {
    void *x[kHostSlots] = {};
    void *y[kHostSlots] = {};
    size_t x_frame = 0, y_frame = 0;  // bytes per frame (all n images)
    cudaStream_t up = nullptr, down = nullptr;
    cudaEvent_t entry = nullptr;
    cudaEvent_t up_done[kHostSlots] = {};
    cudaEvent_t conv_done[kHostSlots] = {};
    cudaEvent_t down_done[kHostSlots] = {};
    bool ready = false;
  } host;
};

struct cc3d_block {
  int n, c_in, c_out, h, w, max_t;
  int fused_rms;    // conv1 applies RMS_norm + SiLU in its epilogue (c_out <= 512)
  int shortcut;     // conv2 carries the 1x1x1 conv_shortcut of x (else y += x)
  cc3d_plan *conv1, *conv2;
  float *g1, *g2;   // g2: the stand-alone RMS_norm after conv1 when not fused
  __nv_bfloat16 *a0, *a1, *h1;  // h1: conv1's output before that RMS_norm
};

namespace {

cc3d_status from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return CC3D_OK;
  if (e == cudaErrorMemoryAllocation) return CC3D_ERR_OOM;
  return CC3D_ERR_CUDA;
}

void free_host_pipe(cc3d_plan::HostPipe &h) {
  for (int s = 0; s < cc3d_plan::kHostSlots; ++s) {
    cudaFree(h.x[s]);
    cudaFree(h.y[s]);
    if (h.up_done[s]) cudaEventDestroy(h.up_done[s]);
    if (h.conv_done[s]) cudaEventDestroy(h.conv_done[s]);
    if (h.down_done[s]) cudaEventDestroy(h.down_done[s]);
  }
  if (h.entry) cudaEventDestroy(h.entry);
  if (h.up) cudaStreamDestroy(h.up);
  if (h.down) cudaStreamDestroy(h.down);
  h = cc3d_plan::HostPipe();
}

void free_plan(cc3d_plan *p) {
  if (!p) return;
  if (p->host.up) cudaStreamSynchronize(p->host.up);
  if (p->host.down) cudaStreamSynchronize(p->host.down);
  free_host_pipe(p->host);
  cudaFree(p->wimg);
  cudaFree(p->wimg1);
  cudaFree(p->wraw);
  cudaFree(p->bias);
  cudaFree(p->gamma);
  cudaFree(p->beta);
  cudaFree(p->oscale);
  delete p;
}

cc3d_status copy_vec(float **dst, const float *src, int c, bool zero_if_null) {
  *dst = nullptr;
  if (!src && !zero_if_null) return CC3D_OK;
  cudaError_t e = cudaMalloc(dst, sizeof(float) * c);
  if (e != cudaSuccess) return CC3D_ERR_OOM;
  if (src)
    e = cudaMemcpy(*dst, src, sizeof(float) * c, cudaMemcpyDeviceToDevice);
  else
    e = cudaMemset(*dst, 0, sizeof(float) * c);
  return from_cuda(e);
}

// Validation that needs no GPU: returns CC3D_OK when a kernel covers desc.
cc3d_status check_desc(const cc3d_desc *d, int *variant) {
  if (!d || !d->weight) return CC3D_ERR_INVALID_ARG;
  if (d->n < 1 || d->c_in < 1 || d->c_out < 1 || d->h < 1 || d->w < 1 || d->max_t < 1)
    return CC3D_ERR_INVALID_ARG;
  if (d->kt < 1 || d->kh < 1 || d->kw < 1) return CC3D_ERR_INVALID_ARG;
  // temporal stride 2: the downsample path's time_conv; spatial stride 2:
  // its per-frame 3x3 conv (both on the tensor-core path)
  const bool s2 = d->stride_h == 2 && d->stride_w == 2;
  if (d->stride_t < 1 || d->stride_t > 2 || !(s2 || (d->stride_h == 1 && d->stride_w == 1)) ||
      d->dil_t != 1 || d->dil_h != 1 || d->dil_w != 1 || d->groups != 1)
    return CC3D_ERR_UNSUPPORTED;
  if (s2) {
    // ZeroPad2d(0, 1, 0, 1) + 3x3 stride 2 on each frame (pad_h = pad_w = 0:
    // no zero rows or columns before the frame, one after): H/2 x W/2 out
    if (d->kt != 1 || d->kh != 3 || d->kw != 3 || d->pad_h != 0 || d->pad_w != 0 ||
        d->stride_t != 1 || d->h % 2 != 0 || d->w % 2 != 0 || d->dtype != CC3D_BF16 ||
        d->c_in % 32 != 0)
      return CC3D_ERR_UNSUPPORTED;
  } else if (d->kh % 2 == 0 || d->kw % 2 == 0 || d->pad_h != d->kh / 2 ||
             d->pad_w != d->kw / 2) {
    return CC3D_ERR_UNSUPPORTED;
  }
  if (d->kt > 3 || d->kh > 3 || d->kw > 3) return CC3D_ERR_UNSUPPORTED;
  if (d->epi < CC3D_EPI_BIAS || d->epi > CC3D_EPI_BIAS_RMS) return CC3D_ERR_INVALID_ARG;
  const bool rms = d->epi == CC3D_EPI_BIAS_RMS_SILU || d->epi == CC3D_EPI_BIAS_RMS;
  if (rms && !d->gamma) return CC3D_ERR_INVALID_ARG;
  if (d->dtype == CC3D_FP32) {
    if (d->epi != CC3D_EPI_BIAS || d->stride_t != 1) return CC3D_ERR_UNSUPPORTED;
    *variant = CC3D_VARIANT_FP32;
    return CC3D_OK;
  }
  if (d->dtype == CC3D_FP8_E4M3) {
    // FP8 operands on the tensor-core path: 128-channel chunks, per-channel
    // weight scales and one activation scale, bias or residual epilogue
    if (!d->w_scale || !(d->x_scale > 0.f)) return CC3D_ERR_INVALID_ARG;
    if (d->c_in % 128 != 0 || d->c_out % 16 != 0 || d->kh != d->kw || s2 || rms)
      return CC3D_ERR_UNSUPPORTED;
    *variant = CC3D_VARIANT_UMMA;
    return CC3D_OK;
  }
  if (d->dtype != CC3D_BF16) return CC3D_ERR_INVALID_ARG;
  if (d->c_out % 16 != 0) return CC3D_ERR_UNSUPPORTED;
  if (d->c_in <= 8) {
    // thin path: whole K gathered per pixel, one N tile, bias epilogue
    if (d->epi != CC3D_EPI_BIAS || d->c_out > 256 || d->stride_t != 1)
      return CC3D_ERR_UNSUPPORTED;
    if (d->kt * d->kh * d->kw * d->c_in > 256) return CC3D_ERR_UNSUPPORTED;
    *variant = CC3D_VARIANT_THIN;
    return CC3D_OK;
  }
  if (d->c_in % 32 == 0) {
    if (d->kh != d->kw) return CC3D_ERR_UNSUPPORTED;
    // an RMS row: up to 256 channels on one CTA, or up to 512 (steps of 32)
    // split over the two CTAs of a cluster
    if (rms && d->c_out > 256 && (d->c_out > 512 || d->c_out % 32 != 0))
      return CC3D_ERR_UNSUPPORTED;
    *variant = CC3D_VARIANT_UMMA;
    return CC3D_OK;
  }
  return CC3D_ERR_UNSUPPORTED;
}

}  // namespace

namespace {
cc3d_status plan_create_impl(const cc3d_desc *desc, int c_sc, const void *w_sc,
                             const float *b_sc, cc3d_plan **out, bool whole_rows = false);
}  // namespace

extern "C" {

const char *cc3d_status_string(cc3d_status s) {
  switch (s) {
    case CC3D_OK: return "ok";
    case CC3D_ERR_INVALID_ARG: return "invalid argument";
    case CC3D_ERR_UNSUPPORTED: return "unsupported descriptor (no kernel covers it)";
    case CC3D_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case CC3D_ERR_ALIAS: return "cache_out overlaps cache_in, x or y";
    case CC3D_ERR_OOM: return "device allocation failed";
    case CC3D_ERR_CUDA: return "CUDA error";
    case CC3D_ERR_TIMEOUT: return "device wait timed out";
    case CC3D_ERR_TOO_LARGE: return "problem exceeds the fixed no-allocation scratch";
  }
  return "unknown status";
}

uint64_t cc3d_launch_count(void) { return g_launches.load(); }

cc3d_status cc3d_plan_create(const cc3d_desc *desc, cc3d_plan **out) {
  return plan_create_impl(desc, 0, nullptr, nullptr, out);
}

}  // extern "C"

namespace {

// A plan, optionally with the residual block's 1x1x1 conv_shortcut fused in
// (c_sc > 0: w_sc [c_out][c_sc] bf16 and b_sc [c_out] fp32, device): its
// channel chunks become extra K stages of the same accumulator, its bias is
// added to the conv's.  Only for bf16 3x3x3 stride-1 convs with the bias
// epilogue (the block's conv2).  whole_rows: tiles that hold whole C_out
// rows, as an RMS epilogue needs, although the plan's own epilogue has none
// (a block's conv2, whose calls may also apply the next block's first norm).
cc3d_status plan_create_impl(const cc3d_desc *desc, int c_sc, const void *w_sc,
                             const float *b_sc, cc3d_plan **out, bool whole_rows) {
  if (!out) return CC3D_ERR_INVALID_ARG;
  int variant = 0;
  cc3d_status s = check_desc(desc, &variant);
  if (s != CC3D_OK) return s;
  if (c_sc < 0 || (c_sc > 0 && !w_sc)) return CC3D_ERR_INVALID_ARG;
  if (c_sc > 0 && (variant != CC3D_VARIANT_UMMA || desc->kh != 3 || desc->kw != 3 ||
                   desc->stride_t != 1 || desc->stride_h != 1 || desc->epi != CC3D_EPI_BIAS ||
                   c_sc % 16 != 0))
    return CC3D_ERR_UNSUPPORTED;
  if (!is_sm100()) return CC3D_ERR_UNSUPPORTED;
  cc3d_plan *p = new cc3d_plan();
  p->d = *desc;
  p->d.weight = nullptr;
  p->d.bias = p->d.gamma = p->d.beta = nullptr;
  p->variant = variant;
  cudaGetDevice(&p->device);
  std::memset(&p->st, 0, sizeof(p->st));
  p->st.variant = variant;
  p->st.k_split = 1;
  p->st.mma_ctas = 1;
  p->st.row_ctas = 1;
  p->st.one_frame_mma_ctas = 1;
  const int taps = desc->kt * desc->kh * desc->kw;
  cudaError_t e = cudaSuccess;
  if ((s = copy_vec(&p->bias, desc->bias, desc->c_out, true)) != CC3D_OK) goto fail;
  if (c_sc > 0 && b_sc) {
    // one bias: the conv's plus the shortcut's
    std::vector<float> hb(desc->c_out), hs(desc->c_out);
    e = cudaMemcpy(hb.data(), p->bias, sizeof(float) * desc->c_out, cudaMemcpyDeviceToHost);
    if (e == cudaSuccess)
      e = cudaMemcpy(hs.data(), b_sc, sizeof(float) * desc->c_out, cudaMemcpyDeviceToHost);
    for (int i = 0; i < desc->c_out; ++i) hb[i] += hs[i];
    if (e == cudaSuccess)
      e = cudaMemcpy(p->bias, hb.data(), sizeof(float) * desc->c_out, cudaMemcpyHostToDevice);
    if (e != cudaSuccess) { s = from_cuda(e); goto fail; }
  }
  if ((s = copy_vec(&p->gamma, desc->gamma, desc->c_out, false)) != CC3D_OK) goto fail;
  if ((s = copy_vec(&p->beta, desc->beta, desc->c_out, false)) != CC3D_OK) goto fail;
  if (variant == CC3D_VARIANT_THIN) {
    if (!status_ptr()) { s = CC3D_ERR_CUDA; goto fail; }
    if (cudaDeviceGetAttribute(&p->sm_count, cudaDevAttrMultiProcessorCount, p->device) !=
        cudaSuccess)
      p->sm_count = 148;
    p->kpad = (taps * desc->c_in + 15) / 16 * 16;
    // RGB input with a 3x3x3 kernel: segment-ordered K (see conv_thin.cu)
    p->thin_spec = (desc->c_in == 3 && desc->kt == 3 && desc->kh == 3 && desc->kw == 3 &&
                    desc->pad_h == 1 && desc->pad_w == 1 && p->kpad == 96)
                       ? 1
                       : 0;
    p->nt = desc->c_out;
    int cols = 32;
    while (cols < 2 * desc->c_out) cols *= 2;
    p->tmem_cols = cols;
    {
      ThinArgs probe;
      std::memset(&probe, 0, sizeof probe);
      probe.kpad = p->kpad; probe.c_out = desc->c_out; probe.kt = desc->kt;
      probe.kh = desc->kh; probe.kw = desc->kw; probe.c_in = desc->c_in;
      probe.pad_w = desc->pad_w; probe.use_tma = 1; probe.spec_rgb333 = 0; probe.store_boxes = 1;
      int per_sm = static_cast<int>((228 * 1024) / (thin_smem_bytes(probe) + 1024));
      if (per_sm > 512 / cols) per_sm = 512 / cols;
      if (per_sm > 2) per_sm = 2;
      p->ctas_per_sm = per_sm < 1 ? 1 : per_sm;
    }
    p->st.tile_h = umma_tile_h();
    p->st.tile_w = umma_tile_w();
    p->st.n_tile = p->nt;
    p->st.one_frame_n_tile = p->nt;
    p->st.k_chunk = p->kpad;
    const size_t bytes = sizeof(__nv_bfloat16) * p->kpad * desc->c_out;
    if (cudaMalloc(&p->wraw, bytes) != cudaSuccess) { s = CC3D_ERR_OOM; goto fail; }
    e = launch_repack_thin(static_cast<const __nv_bfloat16 *>(desc->weight),
                           static_cast<uint8_t *>(p->wraw), desc->c_out, desc->c_in, taps,
                           p->kpad, p->thin_spec, 0);
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    if (e != cudaSuccess) { s = from_cuda(e); goto fail; }
  } else if (variant == CC3D_VARIANT_FP32) {
    const size_t bytes = sizeof(float) * desc->c_out * desc->c_in * taps;
    if (cudaMalloc(&p->wraw, bytes) != cudaSuccess) { s = CC3D_ERR_OOM; goto fail; }
    e = cudaMemcpy(p->wraw, desc->weight, bytes, cudaMemcpyDeviceToDevice);
    if (e != cudaSuccess) { s = from_cuda(e); goto fail; }
  } else {
    if (!encode_fn()) { s = CC3D_ERR_CUDA; goto fail; }
    e = umma_prepare();
    if (e != cudaSuccess) { s = from_cuda(e); goto fail; }
    if (!status_ptr()) { s = CC3D_ERR_CUDA; goto fail; }
    {
      UmmaLayer &L = p->layer;
      std::memset(&L, 0, sizeof L);
      if (cudaDeviceGetAttribute(&L.sm_count, cudaDevAttrMultiProcessorCount, p->device) !=
          cudaSuccess)
        L.sm_count = 148;
      L.n = desc->n; L.c_in = desc->c_in; L.c_out = desc->c_out; L.h = desc->h; L.w = desc->w;
      L.kt = desc->kt; L.kh = desc->kh; L.kw = desc->kw;
      L.pad_h = desc->pad_h; L.pad_w = desc->pad_w;
      L.stride_t = desc->stride_t;
      // spatial stride 2 runs as nine 1x1 taps over the output frame
      L.s2 = desc->stride_h == 2 ? 1 : 0;
      L.epi = static_cast<int>(desc->epi);
      // Tile configuration (N split, sub-tiles, CTA pair, weight grouping,
      // pipeline depths): a function of (n, c_in, c_out, h, w, epilogue,
      // max_t), and a second one for one-frame calls.
      UmmaConfig &cfg = L.cfg;
      const bool e4m3 = desc->dtype == CC3D_FP8_E4M3;
      L.e4m3 = e4m3 ? 1 : 0;
      const int max_out = (desc->max_t - 1) / desc->stride_t + 1;  // largest call's frames
      // (the stride-2 conv: four phase stages seen through 2 x 2 views)
      const int kt_eff = L.s2 ? 4 : desc->kt, ks_eff = L.s2 ? 2 : desc->kh;
      const int h_out = desc->h / desc->stride_h, w_out = desc->w / desc->stride_w;
      const bool rms_epi = desc->epi == CC3D_EPI_BIAS_RMS_SILU ||
                           desc->epi == CC3D_EPI_BIAS_RMS || whole_rows;
      p->whole_rows = rms_epi;
      if (!choose_umma_config(desc->n, desc->c_in, desc->c_out, h_out, w_out, kt_eff, ks_eff,
                              rms_epi, max_out, L.sm_count, &cfg, e4m3)) {
        s = CC3D_ERR_UNSUPPORTED;
        goto fail;
      }
      // the tiles for one-frame calls, when they differ
      UmmaConfig cfg1;
      p->has_layer1 = max_out > 1 &&
                      choose_umma_config(desc->n, desc->c_in, desc->c_out, h_out, w_out, kt_eff,
                                         ks_eff, rms_epi, 1, L.sm_count, &cfg1, e4m3) &&
                      std::memcmp(&cfg1, &cfg, sizeof cfg) != 0;
      p->st.tile_h = umma_tile_h();
      p->st.tile_w = umma_tile_w() * cfg.sub;
      p->st.n_tile = cfg.nt;
      p->st.k_chunk = cfg.kc;
      p->st.k_split = 1;
      p->st.mma_ctas = cfg.pair ? 2 : 1;
      p->st.row_ctas = cfg.xs == 2 ? 2 : 1;
      p->st.w_resident = cfg.b_resident;
      p->st.one_frame_mma_ctas = (p->has_layer1 ? cfg1.pair : cfg.pair) ? 2 : 1;
      p->st.one_frame_n_tile = p->has_layer1 ? cfg1.nt : cfg.nt;
      p->c_sc = c_sc;
      L.c_sc = c_sc;
      L.bias = p->bias;
      L.gamma = p->gamma;
      L.beta = p->beta;
      if (e4m3 && (s = copy_vec(&p->oscale, desc->w_scale, desc->c_out, false)) != CC3D_OK)
        goto fail;
      if (p->has_layer1) {
        p->layer1 = L;
        p->layer1.cfg = cfg1;
      }
      // weight image of a layer: per N tile, the conv's taps * c_in / kc
      // stages, then the shortcut's ceil(c_sc / kc) (its channels past c_sc
      // zero); pairs read it through a tensor map of 128-byte rows
      auto build = [&](UmmaLayer &Ly, uint8_t **img, CUtensorMap *map) -> cc3d_status {
        const UmmaConfig &cf = Ly.cfg;
        if (cf.pair || cf.xs == 2) {
          Ly.max_clusters = umma_max_clusters(cf, ks_eff);
          if (Ly.max_clusters < 1) return CC3D_ERR_CUDA;
        }
        Ly.n_cc_sc = c_sc > 0 ? (c_sc + cf.kc - 1) / cf.kc : 0;
        const int conv_stages = taps * (desc->c_in / cf.kc);
        const int stages = conv_stages + Ly.n_cc_sc;
        // (a stage row is 128 bytes: 64 bf16 or 128 E4M3 channels per 64 / 128)
        const size_t bytes = static_cast<size_t>(desc->c_out) * stages * cf.kc *
                             (e4m3 ? 1 : sizeof(__nv_bfloat16));
        if (cudaMalloc(img, bytes) != cudaSuccess) return CC3D_ERR_OOM;
        cudaError_t err;
        if (e4m3) {
          // E4M3 weights, quantised here with the per-channel scales (p->oscale
          // still holds s_w); the epilogue multiplies by s_x * s_w[c]
          err = launch_repack_umma_e4m3(static_cast<const __nv_bfloat16 *>(desc->weight),
                                        p->oscale, *img, desc->c_out, desc->c_in, taps, cf.nt,
                                        cf.pair, 0);
        } else {
          err = launch_repack_umma(static_cast<const __nv_bfloat16 *>(desc->weight), *img,
                                   desc->c_out, desc->c_in, taps, cf.nt, cf.kc, cf.pair, stages,
                                   0, 0);
        }
        if (err == cudaSuccess && c_sc > 0)
          err = launch_repack_umma(static_cast<const __nv_bfloat16 *>(w_sc), *img, desc->c_out,
                                   c_sc, 1, cf.nt, cf.kc, cf.pair, stages, conv_stages, 0);
        if (err == cudaSuccess) err = cudaDeviceSynchronize();
        if (err != cudaSuccess) return from_cuda(err);
        // (a pair's CTA loads half of each weight stage's rows per box)
        if (cf.pair && !encode_weight_map(map, *img, static_cast<long long>(desc->c_out) * stages,
                                          cf.nt / 2, e4m3))
          return CC3D_ERR_CUDA;
        Ly.wimg = *img;
        Ly.map_w = map;
        return CC3D_OK;
      };
      if ((s = build(L, &p->wimg, &p->map_w)) != CC3D_OK) goto fail;
      if (p->has_layer1 && (s = build(p->layer1, &p->wimg1, &p->map_w1)) != CC3D_OK) goto fail;
      if (e4m3) {
        e = launch_scale_vector(p->oscale, desc->c_out, desc->x_scale, 0);
        if (e == cudaSuccess) e = cudaDeviceSynchronize();
        if (e != cudaSuccess) { s = from_cuda(e); goto fail; }
      }
      L.oscale = p->oscale;
      if (p->has_layer1) {
        p->layer1.oscale = p->oscale;
        p->use_layer1.assign(2 * static_cast<size_t>(max_out + 1), 1);
        for (int to = 2; to <= max_out; ++to)
          for (int cached = 0; cached < 2; ++cached)
            p->use_layer1[2 * to + cached] =
                umma_deal_cost(cfg1, desc->n, to, h_out, w_out, desc->kt, desc->stride_t,
                               cached != 0, L.sm_count) <
                umma_deal_cost(cfg, desc->n, to, h_out, w_out, desc->kt, desc->stride_t,
                               cached != 0, L.sm_count);
      }
    }
  }
  *out = p;
  return CC3D_OK;
fail:
  free_plan(p);
  return s;
}

}  // namespace

extern "C" {

cc3d_status cc3d_plan_destroy(cc3d_plan *plan) {
  if (!plan) return CC3D_ERR_INVALID_ARG;
  free_plan(plan);
  return CC3D_OK;
}

cc3d_status cc3d_get_stats(const cc3d_plan *plan, cc3d_stats *out) {
  if (!plan || !out) return CC3D_ERR_INVALID_ARG;
  *out = plan->st;
  return CC3D_OK;
}

// cc3d_forward, plus the input of a fused conv_shortcut (x_sc: [n][t][h][w]
// [c_sc] bf16, required exactly when the plan has one), plus an optional
// second output of a bias / residual plan with whole-row tiles: y2 =
// SiLU(RMS_norm(y; gamma2)) with its 2-frame history in next_cache_*.
static cc3d_status forward_impl(cc3d_plan *p, const void *x, int t, const void *cache_in, void *y,
                                void *cache_out, const void *residual, const void *next_cache_in,
                                void *next_cache_out, const void *x_sc, void *stream_v,
                                void *y2 = nullptr, const float *gamma2 = nullptr) {
  if (!p) return CC3D_ERR_INVALID_ARG;
  const cc3d_desc &d = p->d;
  auto reject = [&](cc3d_status s) {
    std::lock_guard<std::mutex> lk(p->mu);
    p->st.rejected++;
    return s;
  };
  if (!x || !y || t < 1 || t > d.max_t) return reject(CC3D_ERR_INVALID_ARG);
  if ((d.epi == CC3D_EPI_BIAS_RESIDUAL) != (residual != nullptr))
    return reject(CC3D_ERR_INVALID_ARG);
  if (d.epi != CC3D_EPI_BIAS_RMS_SILU && d.epi != CC3D_EPI_BIAS_RMS && !y2 &&
      (next_cache_in || next_cache_out))
    return reject(CC3D_ERR_INVALID_ARG);
  // the second output: a bias or residual plan on tiles with whole rows
  if (y2 && (!gamma2 || !p->whole_rows || p->variant != CC3D_VARIANT_UMMA ||
             (d.epi != CC3D_EPI_BIAS && d.epi != CC3D_EPI_BIAS_RESIDUAL)))
    return reject(CC3D_ERR_INVALID_ARG);
  if (!aligned16(y2)) return reject(CC3D_ERR_ALIGNMENT);
  if ((p->c_sc > 0) != (x_sc != nullptr)) return reject(CC3D_ERR_INVALID_ARG);
  if (!aligned16(x_sc)) return reject(CC3D_ERR_ALIGNMENT);
  // The thin path reads x and the caches with 2-byte loads (or TMA when they
  // happen to be 16-byte aligned), so a chunk of a 3-channel video may start
  // anywhere on a bf16 boundary; everything else needs 16 bytes.
  const bool thin = p->variant == CC3D_VARIANT_THIN;
  auto in_ok = [&](const void *q) {
    return thin ? (reinterpret_cast<uintptr_t>(q) & 1u) == 0 : aligned16(q);
  };
  if (!in_ok(x) || !aligned16(y) || !in_ok(cache_in) || !in_ok(cache_out) ||
      !aligned16(residual) || !aligned16(next_cache_in) || !aligned16(next_cache_out))
    return reject(CC3D_ERR_ALIGNMENT);
  // bytes per element of x / caches and of y: fp32, bf16, or E4M3 in -> bf16 out
  const size_t esz = d.dtype == CC3D_FP32 ? 4 : 2;
  const size_t in_esz = d.dtype == CC3D_FP8_E4M3 ? 1 : esz;
  const int front = d.kt - 1;
  const int t_out = (t - 1) / d.stride_t + 1;  // frames of y (and of residual)
  const size_t in_frame = static_cast<size_t>(d.h) * d.w * d.c_in * in_esz;
  const size_t out_frame =
      static_cast<size_t>(d.h / d.stride_h) * (d.w / d.stride_w) * d.c_out * esz;
  const size_t x_bytes = in_frame * d.n * t, y_bytes = out_frame * d.n * t_out;
  const size_t c_bytes = in_frame * d.n * front;
  const size_t nc_bytes = out_frame * d.n * 2;
  if (overlaps(cache_out, c_bytes, cache_in, c_bytes) || overlaps(cache_out, c_bytes, x, x_bytes) ||
      overlaps(cache_out, c_bytes, y, y_bytes) ||
      overlaps(next_cache_out, nc_bytes, next_cache_in, nc_bytes) ||
      overlaps(next_cache_out, nc_bytes, y, y_bytes) ||
      overlaps(next_cache_out, nc_bytes, x, x_bytes) || overlaps(y, y_bytes, x, x_bytes) ||
      overlaps(y, y_bytes, x_sc, static_cast<size_t>(d.h) * d.w * p->c_sc * 2 * d.n * t) ||
      overlaps(y2, y_bytes, y, y_bytes) || overlaps(y2, y_bytes, x, x_bytes) ||
      overlaps(y2, y_bytes, residual, y_bytes) || overlaps(y2, y_bytes, next_cache_in, nc_bytes) ||
      overlaps(y2, y_bytes, next_cache_out, nc_bytes) || overlaps(y2, y_bytes, cache_out, c_bytes))
    return reject(CC3D_ERR_ALIAS);
  int dev = -1;
  cudaGetDevice(&dev);
  if (dev != p->device) return reject(CC3D_ERR_INVALID_ARG);
  cudaStream_t stream = static_cast<cudaStream_t>(stream_v);
  int *status = status_ptr();
  if (!status) return reject(CC3D_ERR_CUDA);
  cudaError_t e = cudaSuccess;
  uint64_t tiles = 0;
  if (p->variant == CC3D_VARIANT_FP32) {
    Fp32Args a;
    a.x = static_cast<const float *>(x);
    a.cache = static_cast<const float *>(cache_in);
    a.w = static_cast<const float *>(p->wraw);
    a.bias = p->bias;
    a.y = static_cast<float *>(y);
    a.n = d.n; a.t = t; a.h = d.h; a.w_ = d.w; a.c_in = d.c_in; a.c_out = d.c_out;
    a.kt = d.kt; a.kh = d.kh; a.kw = d.kw; a.pad_h = d.pad_h; a.pad_w = d.pad_w;
    e = launch_conv_fp32(a, stream);
    tiles = 1;
  } else if (p->variant == CC3D_VARIANT_THIN) {
    ThinArgs a;
    a.x = static_cast<const uint16_t *>(x);
    a.cache = static_cast<const uint16_t *>(cache_in);
    a.wimg = static_cast<const uint8_t *>(p->wraw);
    a.bias = p->bias;
    a.y = static_cast<__nv_bfloat16 *>(y);
    a.status = status;
    a.wait_limit_ns = wait_limit_ns();
    a.n = d.n; a.t = t; a.h = d.h; a.w = d.w; a.c_in = d.c_in; a.c_out = d.c_out;
    a.kt = d.kt; a.kh = d.kh; a.kw = d.kw; a.pad_h = d.pad_h; a.pad_w = d.pad_w;
    a.kpad = p->kpad;
    a.tiles_w = (d.w + umma_tile_w() - 1) / umma_tile_w();
    a.tiles_h = (d.h + umma_tile_h() - 1) / umma_tile_h();
    a.n_tiles = d.n * t * a.tiles_h * a.tiles_w;
    a.tmem_cols = p->tmem_cols;
    // TMA halo when both inputs can be described by a tensor map
    a.use_tma = (static_cast<long long>(d.w) * d.c_in % 8 == 0 && aligned16(x) &&
                 (!cache_in || aligned16(cache_in)))
                    ? 1
                    : 0;
    CUtensorMap mx, mc;
    std::memset(&mx, 0, sizeof mx);
    std::memset(&mc, 0, sizeof mc);
    if (a.use_tma) {
      const int row = thin_tma_row(a), box_h = umma_tile_h() + d.kh - 1;
      if (row > 256 || !encode_thin_map(&mx, x, d.c_in, d.w, d.h, t, d.n, row, box_h))
        a.use_tma = 0;
      else if (cache_in && front > 0 &&
               !encode_thin_map(&mc, cache_in, d.c_in, d.w, d.h, front, d.n, row, box_h))
        a.use_tma = 0;
      else if (!(cache_in && front > 0))
        mc = mx;
    }
    a.spec_rgb333 = p->thin_spec;
    CUtensorMap my_map;
    std::memset(&my_map, 0, sizeof my_map);
    a.store_boxes = (d.c_out % 32 == 0 && umma_tile_w() == 8 && umma_tile_h() == 16 &&
                     encode_store_map(&my_map, y, d.c_out, d.w, d.h, t, d.n))
                        ? 1
                        : 0;
    tiles = static_cast<uint64_t>(a.n_tiles);
    const uint64_t slots = static_cast<uint64_t>(p->sm_count) * p->ctas_per_sm;
    e = launch_conv_thin(mx, mc, my_map, a, static_cast<unsigned>(tiles < slots ? tiles : slots),
                         stream);
  } else {
    UmmaCall c{};
    c.x = x; c.t = t; c.cache_in = cache_in; c.y = y; c.cache_out = cache_out;
    c.residual = residual; c.ncache_in = next_cache_in; c.ncache_out = next_cache_out;
    c.x_sc = x_sc;
    c.y2 = y2;
    c.gamma2 = gamma2;
    const bool use1 =
        p->has_layer1 && p->use_layer1[2 * t_out + (cache_in && front > 0 ? 1 : 0)] != 0;
    e = run_umma_layer(use1 ? p->layer1 : p->layer, c, status, stream, &tiles);
    if (e == cudaSuccess && use1) {
      std::lock_guard<std::mutex> lk(p->mu);
      p->st.second_tile_calls++;
    }
  }
  // (the tensor-core conv writes both caches itself)
  if (p->variant == CC3D_VARIANT_UMMA) {
    cache_out = nullptr;
    next_cache_out = nullptr;
  }
  if (e == cudaSuccess && cache_out && front > 0)
    e = launch_cache_update(cache_in, x, cache_out, d.n, t, front, in_frame, stream);
  if (e == cudaSuccess && next_cache_out)
    e = launch_cache_update(next_cache_in, y, next_cache_out, d.n, t_out, 2, out_frame, stream);
  if (e != cudaSuccess) return reject(from_cuda(e));
  std::lock_guard<std::mutex> lk(p->mu);
  p->st.calls++;
  p->st.tiles += tiles;
  return CC3D_OK;
}

cc3d_status cc3d_forward(cc3d_plan *p, const void *x, int t, const void *cache_in, void *y,
                         void *cache_out, const void *residual, const void *next_cache_in,
                         void *next_cache_out, void *stream_v) {
  if (p && p->c_sc > 0) return CC3D_ERR_INVALID_ARG;  // (a block-internal plan)
  return forward_impl(p, x, t, cache_in, y, cache_out, residual, next_cache_in, next_cache_out,
                      nullptr, stream_v);
}

}  // extern "C"

namespace {
// The staging slots, streams and events of cc3d_forward_host (first use).
cc3d_status host_pipe_init(cc3d_plan *p) {
  cc3d_plan::HostPipe &h = p->host;
  if (h.ready) return CC3D_OK;
  const cc3d_desc &d = p->d;
  const size_t esz = d.dtype == CC3D_FP32 ? 4 : 2;
  const size_t in_esz = d.dtype == CC3D_FP8_E4M3 ? 1 : esz;
  h.x_frame = static_cast<size_t>(d.n) * d.h * d.w * d.c_in * in_esz;
  h.y_frame = static_cast<size_t>(d.n) * (d.h / d.stride_h) * (d.w / d.stride_w) * d.c_out * esz;
  const int max_out = (d.max_t - 1) / d.stride_t + 1;
  cudaError_t e = cudaSuccess;
  for (int s = 0; s < cc3d_plan::kHostSlots && e == cudaSuccess; ++s) {
    e = cudaMalloc(&h.x[s], h.x_frame * d.max_t);
    if (e == cudaSuccess) e = cudaMalloc(&h.y[s], h.y_frame * max_out);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&h.up_done[s], cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&h.conv_done[s], cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&h.down_done[s], cudaEventDisableTiming);
  }
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&h.entry, cudaEventDisableTiming);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&h.up, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&h.down, cudaStreamNonBlocking);
  if (e != cudaSuccess) {
    free_host_pipe(h);
    return from_cuda(e);
  }
  h.ready = true;
  return CC3D_OK;
}
}  // namespace

extern "C" {

cc3d_status cc3d_forward_host(cc3d_plan *p, const cc3d_host_call *calls, int ncalls,
                              void *stream_v) {
  if (!p || !calls || ncalls < 1 || p->c_sc > 0) return CC3D_ERR_INVALID_ARG;
  const cc3d_desc &d = p->d;
  // the next caches of an RMS epilogue have no host form
  if (d.epi == CC3D_EPI_BIAS_RMS_SILU || d.epi == CC3D_EPI_BIAS_RMS) return CC3D_ERR_INVALID_ARG;
  int dev = -1;
  cudaGetDevice(&dev);
  if (dev != p->device) return CC3D_ERR_INVALID_ARG;
  // everything cc3d_forward would check on these calls, before any enqueue
  // (x and y are the plan's own staging slots)
  const bool thin = p->variant == CC3D_VARIANT_THIN;
  auto in_ok = [&](const void *q) {
    return thin ? (reinterpret_cast<uintptr_t>(q) & 1u) == 0 : aligned16(q);
  };
  const size_t in_esz = d.dtype == CC3D_FP8_E4M3 ? 1 : (d.dtype == CC3D_FP32 ? 4 : 2);
  const size_t c_bytes = static_cast<size_t>(d.n) * (d.kt - 1) * d.h * d.w * d.c_in * in_esz;
  for (int i = 0; i < ncalls; ++i) {
    const cc3d_host_call &c = calls[i];
    if (!c.x_host || !c.y_host || c.t < 1 || c.t > d.max_t ||
        (d.epi == CC3D_EPI_BIAS_RESIDUAL) != (c.residual != nullptr))
      return CC3D_ERR_INVALID_ARG;
    if (!in_ok(c.cache_in) || !in_ok(c.cache_out) || !aligned16(c.residual))
      return CC3D_ERR_ALIGNMENT;
    if (overlaps(c.cache_out, c_bytes, c.cache_in, c_bytes)) return CC3D_ERR_ALIAS;
  }
  cc3d_status s = host_pipe_init(p);
  if (s != CC3D_OK) return s;
  cc3d_plan::HostPipe &h = p->host;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_v);
  // the uploads start after the work already on `stream`
  cudaError_t e = cudaEventRecord(h.entry, stream);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(h.up, h.entry, 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(h.down, h.entry, 0);
  for (int i = 0; i < ncalls && e == cudaSuccess; ++i) {
    const cc3d_host_call &c = calls[i];
    const int sl = i % cc3d_plan::kHostSlots;
    const bool reused = i >= cc3d_plan::kHostSlots;
    const int t_out = (c.t - 1) / d.stride_t + 1;
    // slot sl was last used by call i - kHostSlots: its x is free once that
    // conv has run, its y once that download has run
    if (reused) e = cudaStreamWaitEvent(h.up, h.conv_done[sl], 0);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(h.x[sl], c.x_host, h.x_frame * c.t, cudaMemcpyHostToDevice, h.up);
    if (e == cudaSuccess) e = cudaEventRecord(h.up_done[sl], h.up);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(stream, h.up_done[sl], 0);
    if (e == cudaSuccess && reused) e = cudaStreamWaitEvent(stream, h.down_done[sl], 0);
    if (e != cudaSuccess) break;
    s = forward_impl(p, h.x[sl], c.t, c.cache_in, h.y[sl], c.cache_out, c.residual, nullptr,
                     nullptr, nullptr, stream_v);
    if (s != CC3D_OK) return s;
    e = cudaEventRecord(h.conv_done[sl], stream);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(h.down, h.conv_done[sl], 0);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(c.y_host, h.y[sl], h.y_frame * t_out, cudaMemcpyDeviceToHost, h.down);
    if (e == cudaSuccess) e = cudaEventRecord(h.down_done[sl], h.down);
  }
  // `stream` waits for every download (the last one of each slot)
  for (int sl = 0; sl < cc3d_plan::kHostSlots && sl < ncalls && e == cudaSuccess; ++sl)
    e = cudaStreamWaitEvent(stream, h.down_done[sl], 0);
  return from_cuda(e);
}

}  // extern "C"

namespace {
// RMS_norm over channels (+ SiLU when `silu`), with its 2-frame cache.
cc3d_status rms_pass(const void *x, const float *gamma, const float *beta, int n, int t, int h,
                     int w, int c, void *y, const void *cache_in, void *cache_out, bool silu,
                     void *stream_v) {
  if (!x || !gamma || !y || n < 1 || t < 1 || h < 1 || w < 1 || c < 8) return CC3D_ERR_INVALID_ARG;
  if (c % 8 != 0 || c > 1024) return CC3D_ERR_UNSUPPORTED;
  if (!aligned16(x) || !aligned16(y) || !aligned16(cache_in) || !aligned16(cache_out))
    return CC3D_ERR_ALIGNMENT;
  const size_t frame = static_cast<size_t>(h) * w * c * 2;
  const size_t xb = frame * n * t, cb = frame * n * 2;
  if (overlaps(cache_out, cb, cache_in, cb) || overlaps(cache_out, cb, y, xb) ||
      overlaps(cache_out, cb, x, xb))
    return CC3D_ERR_ALIAS;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_v);
  // one kernel: the normalised activation and its 2-frame cache
  const cudaError_t e = launch_rmsnorm_silu(
      static_cast<const __nv_bfloat16 *>(x), gamma, beta, n, t, static_cast<long long>(h) * w, c,
      static_cast<__nv_bfloat16 *>(y), static_cast<const __nv_bfloat16 *>(cache_in),
      static_cast<__nv_bfloat16 *>(cache_out), silu, stream);
  return from_cuda(e);
}
}  // namespace

extern "C" {

cc3d_status rmsnorm_silu(const void *x, const float *gamma, const float *beta, int n, int t,
                         int h, int w, int c, void *y, const void *cache_in, void *cache_out,
                         void *stream) {
  return rms_pass(x, gamma, beta, n, t, h, w, c, y, cache_in, cache_out, true, stream);
}

cc3d_status rms_norm(const void *x, const float *gamma, const float *beta, int n, int t, int h,
                     int w, int c, void *y, const void *cache_in, void *cache_out, void *stream) {
  return rms_pass(x, gamma, beta, n, t, h, w, c, y, cache_in, cache_out, false, stream);
}

cc3d_status cc3d_quantize_e4m3(const void *x, size_t count, float scale, void *q, void *stream) {
  if (!x || !q || count % 8 != 0 || !(scale > 0.f)) return CC3D_ERR_INVALID_ARG;
  if (!aligned16(x) || (reinterpret_cast<uintptr_t>(q) & 7u) != 0) return CC3D_ERR_ALIGNMENT;
  if (overlaps(x, count * 2, q, count)) return CC3D_ERR_ALIAS;
  if (count == 0) return CC3D_OK;
  return from_cuda(launch_quantize_e4m3(static_cast<const __nv_bfloat16 *>(x), count, scale,
                                        static_cast<uint8_t *>(q),
                                        static_cast<cudaStream_t>(stream)));
}

cc3d_status cc3d_block_create2(int n, int c_in, int c_out, int h, int w, int max_t,
                               const void *w1, const float *b1, const float *g1, const void *w2,
                               const float *b2, const float *g2, const void *w_sc,
                               const float *b_sc, cc3d_block **out) {
  if (!out || !w1 || !w2 || !g1 || !g2 || n < 1 || h < 1 || w < 1 || max_t < 1)
    return CC3D_ERR_INVALID_ARG;
  if (!w_sc && (c_in != c_out || b_sc)) return CC3D_ERR_INVALID_ARG;
  if (c_in < 32 || c_in > 1024 || c_in % 32 != 0 || c_out < 32 || c_out > 1024 ||
      c_out % 32 != 0)
    return CC3D_ERR_UNSUPPORTED;
  cc3d_desc d;
  std::memset(&d, 0, sizeof d);
  d.n = n; d.h = h; d.w = w; d.max_t = max_t;
  d.kt = d.kh = d.kw = 3; d.pad_h = d.pad_w = 1;
  d.stride_t = d.stride_h = d.stride_w = 1; d.dil_t = d.dil_h = d.dil_w = 1; d.groups = 1;
  d.dtype = CC3D_BF16;
  cc3d_block *b = new cc3d_block();
  std::memset(b, 0, sizeof *b);
  b->n = n; b->c_in = c_in; b->c_out = c_out; b->h = h; b->w = w; b->max_t = max_t;
  // conv1's RMS epilogue covers rows up to 512 channels (wider than 256:
  // split over a cluster); wider blocks run conv1 with the bias epilogue and
  // the stand-alone RMS_norm + SiLU after it.
  b->fused_rms = c_out <= 256 || (c_out <= 512 && c_out % 32 == 0);
  b->shortcut = w_sc != nullptr;
  cc3d_status s;
  const size_t vox = static_cast<size_t>(n) * max_t * h * w;
  d.c_in = c_in; d.c_out = c_out;
  d.weight = w1; d.bias = b1;
  d.epi = b->fused_rms ? CC3D_EPI_BIAS_RMS_SILU : CC3D_EPI_BIAS;
  d.gamma = b->fused_rms ? g2 : nullptr;
  d.beta = nullptr;
  if ((s = cc3d_plan_create(&d, &b->conv1)) != CC3D_OK) goto fail;
  d.c_in = c_out;
  d.weight = w2; d.bias = b2; d.gamma = nullptr;
  d.epi = b->shortcut ? CC3D_EPI_BIAS : CC3D_EPI_BIAS_RESIDUAL;
  // conv2 on whole-row tiles where that costs nothing (up to 256 channels:
  // the same tiles), so that in a chain its epilogue can also apply the next
  // block's first norm.  (Wider rows would need the cluster-split tiles,
  // whose conv2 runs slower than its own CTA-pair tiles by more than the
  // stand-alone norm pass costs: there the hand-over is that pass.)
  if ((s = plan_create_impl(&d, b->shortcut ? c_in : 0, w_sc, b_sc, &b->conv2,
                            c_out <= 256)) != CC3D_OK)
    goto fail;
  if ((s = copy_vec(&b->g1, g1, c_in, false)) != CC3D_OK) goto fail;
  if (!b->fused_rms && (s = copy_vec(&b->g2, g2, c_out, false)) != CC3D_OK) goto fail;
  if (cudaMalloc(&b->a0, vox * c_in * 2) != cudaSuccess ||
      cudaMalloc(&b->a1, vox * c_out * 2) != cudaSuccess ||
      (!b->fused_rms && cudaMalloc(&b->h1, vox * c_out * 2) != cudaSuccess)) {
    s = CC3D_ERR_OOM;
    goto fail;
  }
  *out = b;
  return CC3D_OK;
fail:
  cc3d_block_destroy(b);
  return s;
}

cc3d_status cc3d_block_create(int n, int c, int h, int w, int max_t, const void *w1,
                              const float *b1, const float *g1, const void *w2, const float *b2,
                              const float *g2, cc3d_block **out) {
  return cc3d_block_create2(n, c, c, h, w, max_t, w1, b1, g1, w2, b2, g2, nullptr, nullptr, out);
}

cc3d_status cc3d_block_destroy(cc3d_block *b) {
  if (!b) return CC3D_ERR_INVALID_ARG;
  if (b->conv1) cc3d_plan_destroy(b->conv1);
  if (b->conv2) cc3d_plan_destroy(b->conv2);
  cudaFree(b->g1);
  cudaFree(b->g2);
  cudaFree(b->a0);
  cudaFree(b->a1);
  cudaFree(b->h1);
  delete b;
  return CC3D_OK;
}

cc3d_status cc3d_resblock_forward(cc3d_block *b, const void *x, int t, const void *cache1_in,
                                  const void *cache2_in, void *y, void *cache1_out,
                                  void *cache2_out, void *stream) {
  return cc3d_resblock_forward_fused(b, x, nullptr, t, cache1_in, cache2_in, y, cache1_out,
                                     cache2_out, nullptr, nullptr, nullptr, nullptr, stream);
}

cc3d_status cc3d_resblock_forward_fused(cc3d_block *b, const void *x, const void *a0_in, int t,
                                        const void *cache1_in, const void *cache2_in, void *y,
                                        void *cache1_out, void *cache2_out, const float *g_next,
                                        void *a0_next, const void *a0_next_cache_in,
                                        void *a0_next_cache_out, void *stream) {
  if (!b || !x || !y || t < 1 || t > b->max_t) return CC3D_ERR_INVALID_ARG;
  if ((g_next != nullptr) != (a0_next != nullptr) ||
      (!g_next && (a0_next_cache_in || a0_next_cache_out)))
    return CC3D_ERR_INVALID_ARG;
  const size_t fin = static_cast<size_t>(b->h) * b->w * b->c_in * 2;
  const size_t fout = static_cast<size_t>(b->h) * b->w * b->c_out * 2;
  const size_t xb = fin * b->n * t, yb = fout * b->n * t;
  const size_t c1 = fin * b->n * 2, c2 = fout * b->n * 2;  // cache1: a0 frames, cache2: a1
  if (overlaps(x, xb, y, yb) || overlaps(a0_in, xb, y, yb)) return CC3D_ERR_ALIAS;
  if (overlaps(cache1_out, c1, cache1_in, c1) || overlaps(cache2_out, c2, cache2_in, c2) ||
      overlaps(cache1_out, c1, x, xb) || overlaps(cache1_out, c1, y, yb) ||
      overlaps(cache2_out, c2, x, xb) || overlaps(cache2_out, c2, y, yb) ||
      overlaps(cache1_out, c1, cache2_out, c2) || overlaps(cache1_out, c1, cache2_in, c2) ||
      overlaps(cache2_out, c2, cache1_in, c1) || overlaps(cache1_out, c1, a0_in, xb) ||
      overlaps(cache2_out, c2, a0_in, xb))
    return CC3D_ERR_ALIAS;
  if (!aligned16(x) || !aligned16(y) || !aligned16(a0_in) || !aligned16(a0_next) ||
      !aligned16(cache1_in) || !aligned16(cache1_out) || !aligned16(cache2_in) ||
      !aligned16(cache2_out) || !aligned16(a0_next_cache_in) || !aligned16(a0_next_cache_out))
    return CC3D_ERR_ALIGNMENT;
  if (overlaps(a0_next, yb, x, xb) || overlaps(a0_next, yb, y, yb) ||
      overlaps(a0_next, yb, a0_in, xb) ||
      overlaps(a0_next, yb, cache1_in, c1) || overlaps(a0_next, yb, cache1_out, c1) ||
      overlaps(a0_next, yb, cache2_in, c2) || overlaps(a0_next, yb, cache2_out, c2) ||
      overlaps(a0_next_cache_out, c2, cache1_out, c1) ||
      overlaps(a0_next_cache_out, c2, cache2_out, c2) ||
      overlaps(a0_next_cache_out, c2, a0_next_cache_in, c2) ||
      overlaps(a0_next_cache_out, c2, a0_next, yb) || overlaps(a0_next_cache_out, c2, y, yb) ||
      overlaps(a0_next_cache_out, c2, x, xb))
    return CC3D_ERR_ALIAS;
  cc3d_status s = CC3D_OK;
  // a0 = SiLU(RMS(x; g1)), unless the previous block's conv2 produced it;
  // conv1's cache is a0's history (written by the norm pass, or else by
  // conv1 itself from its cache_in and a0)
  const void *a0 = a0_in;
  if (!a0_in) {
    s = rmsnorm_silu(x, b->g1, nullptr, b->n, t, b->h, b->w, b->c_in, b->a0, cache1_in,
                     cache1_out, stream);
    if (s != CC3D_OK) return s;
    a0 = b->a0;
  }
  void *conv1_cache_out = a0_in ? cache1_out : nullptr;
  // a1 = SiLU(RMS(conv1(a0) + b1; g2)); conv2's cache is a1's history.
  if (b->fused_rms) {
    s = cc3d_forward(b->conv1, a0, t, cache1_in, b->a1, conv1_cache_out, nullptr, cache2_in,
                     cache2_out, stream);
  } else {
    s = cc3d_forward(b->conv1, a0, t, cache1_in, b->h1, conv1_cache_out, nullptr, nullptr,
                     nullptr, stream);
    if (s == CC3D_OK)
      s = rmsnorm_silu(b->h1, b->g2, nullptr, b->n, t, b->h, b->w, b->c_out, b->a1, cache2_in,
                       cache2_out, stream);
  }
  if (s != CC3D_OK) return s;
  // y = conv2(a1) + b2 + (x | conv_shortcut(x) + b_sc), fused in conv2; with
  // g_next, the same epilogue also writes the next block's a0 (up to 256
  // channels; wider, a norm pass over y follows)
  const bool hand_over_in_epilogue = g_next && b->c_out <= 256;
  s = forward_impl(b->conv2, b->a1, t, cache2_in, y, nullptr, b->shortcut ? nullptr : x,
                   hand_over_in_epilogue ? a0_next_cache_in : nullptr,
                   hand_over_in_epilogue ? a0_next_cache_out : nullptr, b->shortcut ? x : nullptr,
                   stream, hand_over_in_epilogue ? a0_next : nullptr,
                   hand_over_in_epilogue ? g_next : nullptr);
  if (s != CC3D_OK || !g_next || hand_over_in_epilogue) return s;
  return rmsnorm_silu(y, g_next, nullptr, b->n, t, b->h, b->w, b->c_out, a0_next,
                      a0_next_cache_in, a0_next_cache_out, stream);
}

cc3d_status cc3d_sync_status(void *stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return CC3D_ERR_CUDA;
  int v = 0;
  e = cudaMemcpyFromSymbol(&v, g_status_word, sizeof v);
  if (e != cudaSuccess) return CC3D_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    cudaMemcpyToSymbol(g_status_word, &zero, sizeof zero);
    return CC3D_ERR_TIMEOUT;
  }
  return CC3D_OK;
}

}  // extern "C"
