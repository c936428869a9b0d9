// conv_thin.cu -- causal Conv3D for inputs with very few channels (the
// encoder's first layer, RGB video: C_in = 3), on tcgen05 tensor cores.
//
// Operation: the same causal conv as conv_umma.cu ("Cosmos3 Wan VAE --
// engine size vs context memory", §10.3), but with C_in so small that one
// pixel is 6 bytes: TMA boxes cannot start on such pixels and one tap holds
// only C_in useful K values.  The whole K = kt * kh * kw * C_in (81 for a
// 3x3x3 kernel on RGB) is instead gathered per output pixel ("im2col" in
// shared memory), zero-padded to a multiple of 16, and multiplied in
// K / 16 MMAs.  The layer moves ~40 MB in and writes C_out values per input
// pixel (1.3 GB at 17 x 480 x 832 x 96), so it is bound by the HBM write of
// y; the design keeps every other step off that critical path.
//
// Persistent CTAs (one or two per SM), 320 threads:
//   warp  5    halo loader: one TMA box per frame brings the tile's input
//              halo (kt frames x (16 + kh - 1) rows x a 16-byte aligned
//              run of (8 + kw - 1) * C_in elements) into a double-buffered
//              shared buffer -- from the cache when the frame precedes the
//              chunk; out-of-image and absent-cache reads are TMA zero fill;
//   warps 0-3  builders: write the A operand from the halo as K-major core
//              matrices (double buffered): in general the 128 x K_pad im2col
//              tile; for RGB with a 3x3x3 kernel only the (kt, kw, ci) part
//              of it, one 32-value row per halo row and tile column, which
//              the MMAs of the three kernel rows kh read at start addresses
//              kh halo rows apart.  When the input cannot be described by a
//              tensor map (unaligned chunk start, W * C_in not a multiple of
//              8) they stage the halo themselves with plain loads;
//   warp  4    tensor memory owner and MMA issuer (one thread);
//   warps 6-9  epilogue: tensor memory -> +bias -> bf16 -> global.
// The weights ([K_pad/8][C_out][8] core matrices) stay in shared memory for
// the life of the CTA; two accumulators in tensor memory let the epilogue
// of one tile overlap the build and MMAs of the next.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "internal.h"
#include "ptx.cuh"

namespace cc3d {
namespace {

constexpr int kTW = 8, kTH = 16, kM = kTW * kTH;
constexpr int kBuilders = 128;  // warps 0-3
constexpr int kMmaWarp = 4;
constexpr int kLoadWarp = 5;    // halo TMA producer
constexpr int kThreads = 320;   // + epilogue warps 6-9
constexpr int kNH = 3;          // halo ring depth (loader runs ahead)
// Bound of the drain waits at exit (copies / MMAs already issued finish in
// microseconds; this only guards against a broken pipeline).
constexpr unsigned long long kDrainLimitNs = 100ull * 1000000ull;

// Halo geometry of one tile.  Frames are [kt] slabs of `kt_stride`
// elements; a slab holds (16 + kh - 1) rows of `row` elements; the pixel
// (w0 - pad_w) starts at element `rem` of each row.
struct HaloGeom {
  int row, rem, kt_stride;
};

__host__ __device__ inline uint32_t rup(uint32_t v, uint32_t a) { return (v + a - 1) / a * a; }

__host__ __device__ inline HaloGeom halo_geom(const ThinArgs &a) {
  // One halo row is a run of the flattened (W * C_in) image row that starts
  // on a 16-byte boundary: the first element, (w0 - pad_w) * C_in, is
  // rounded down to a multiple of 8 (w0 is a multiple of 8, so the
  // remainder `rem` is the same for every tile).  The TMA box and the
  // plain-load staging fill exactly this shape, zero outside the image.
  HaloGeom g;
  const int hh = kTH + a.kh - 1, hw = kTW + a.kw - 1;
  g.rem = ((-a.pad_w * a.c_in) % 8 + 8) % 8;
  g.row = static_cast<int>(rup(g.rem + hw * a.c_in, 8));
  g.kt_stride = static_cast<int>(rup(g.row * hh * 2, 128) / 2);
  return g;
}

struct ThinLayout {
  uint32_t b_off, a_off, a_bytes, halo_off, halo_bytes, koff_off, bias_off, stage_off,
      stage_pitch, bar_off, total;
};

// RGB 3x3x3: the A buffer holds one 32-value row of K for each of the
// (16 + 2) halo rows and 8 tile columns, as [halo row][4 K groups of 8][8
// columns][8] bf16 -- 512 bytes per halo row.
constexpr uint32_t kRgbRowBytes = 4u * 128u;

__host__ __device__ inline ThinLayout thin_layout(const ThinArgs &a) {
  ThinLayout L;
  const HaloGeom g = halo_geom(a);
  L.b_off = 0;
  const uint32_t b_bytes = static_cast<uint32_t>(a.kpad) * a.c_out * 2u;
  L.a_off = rup(b_bytes, 1024u);
  L.a_bytes = a.spec_rgb333 ? rup(static_cast<uint32_t>(kTH + a.kh - 1) * kRgbRowBytes, 1024u)
                            : rup(static_cast<uint32_t>(a.kpad) * kM * 2u, 1024u);
  L.halo_off = L.a_off + 2 * L.a_bytes;
  L.halo_bytes = rup(static_cast<uint32_t>(a.kt) * g.kt_stride * 2u, 128u);  // per buffer
  L.koff_off = L.halo_off + kNH * L.halo_bytes;  // int32 halo offset per K index
  L.bias_off = rup(L.koff_off + 4u * a.kpad, 16u);  // fp32 bias copy
  // output staging: 128 pixels, each c_out * 2 bytes plus one spare 16-byte
  // chunk so eight consecutive pixels start in eight different bank quads
  L.stage_pitch = static_cast<uint32_t>(a.c_out) * 2u + 16u;
  L.stage_off = rup(L.bias_off + 4u * a.c_out, 1024u);
  L.bar_off = rup(L.stage_off + kM * L.stage_pitch, 64u);
  // b_full, a_full[2], a_empty[2], acc_full[2], acc_empty[2],
  // halo_full[kNH], halo_empty[kNH], drain, tmem slot + flags
  L.total = L.bar_off + 8u * (10 + 2 * kNH) + 16u;
  return L;
}

struct Tile {
  int n, t, h0, w0;
};

__device__ __forceinline__ Tile thin_tile(int tile, const ThinArgs &p) {
  Tile c;
  const int tw = tile % p.tiles_w;
  int r = tile / p.tiles_w;
  const int th = r % p.tiles_h;
  r /= p.tiles_h;
  c.t = r % p.t;
  c.n = r / p.t;
  c.w0 = tw * kTW;
  c.h0 = th * kTH;
  return c;
}

__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap *map, uint64_t *bar,
                                            int c0, int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3),
      "r"(smem_u32(bar))
      : "memory");
}

// One row of the RGB 3x3x3 A buffer: the 27 values of halo row `row` of
// the three frames at tile column c, k = kt * 9 + kw * 3 + ci, then five
// zeros.  With kernel row kh at K offset 32 * kh of the weights, output
// pixel (r, c) meets rows r, r + 1, r + 2 of this buffer in three MMA
// steps of K = 32.  A frame's nine values are consecutive halo elements
// (three pixels of three channels): five aligned 32-bit words, realigned
// with funnel shifts.  `hbits` points at frame 0's first value; frames are
// 768 elements apart (even), so all three share the realignment.
__device__ __forceinline__ void build_row_rgb333(const uint16_t *hbits, uint8_t *dst) {
  const uintptr_t e0 = reinterpret_cast<uintptr_t>(hbits);
  const uint32_t *w32 = reinterpret_cast<const uint32_t *>(e0 & ~static_cast<uintptr_t>(3));
  const uint32_t sh = (e0 & 2) ? 16u : 0u;
  uint32_t v[27];  // the 27 values, one per register (low 16 bits)
#pragma unroll
  for (int kt = 0; kt < 3; ++kt) {
    uint32_t w[5];
#pragma unroll
    for (int i = 0; i < 5; ++i) w[i] = w32[kt * 384 + i];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t pr = __funnelshift_r(w[i], w[i + 1], sh);  // values 2i, 2i + 1
      v[kt * 9 + 2 * i] = pr & 0xffffu;
      v[kt * 9 + 2 * i + 1] = pr >> 16;
    }
    v[kt * 9 + 8] = (w[4] >> sh) & 0xffffu;
  }
  uint32_t out[16];
#pragma unroll
  for (int q = 0; q < 16; ++q) {
    const uint32_t lo = 2 * q < 27 ? v[2 * q] : 0u;
    const uint32_t hi = 2 * q + 1 < 27 ? v[2 * q + 1] : 0u;
    out[q] = lo | (hi << 16);
  }
#pragma unroll
  for (int k8 = 0; k8 < 4; ++k8)
    *reinterpret_cast<uint4 *>(dst + k8 * 128) =
        make_uint4(out[4 * k8], out[4 * k8 + 1], out[4 * k8 + 2], out[4 * k8 + 3]);
}

__global__ void __launch_bounds__(kThreads, 2)
    conv_thin_kernel(const __grid_constant__ CUtensorMap map_x,
                     const __grid_constant__ CUtensorMap map_cache,
                     const __grid_constant__ CUtensorMap map_y, ThinArgs p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const ThinLayout L = thin_layout(p);
  const HaloGeom G = halo_geom(p);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L.bar_off);
  uint64_t *b_full = bars;
  uint64_t *a_full = bars + 1;       // [2]
  uint64_t *a_empty = bars + 3;      // [2]
  uint64_t *acc_full = bars + 5;     // [2]
  uint64_t *acc_empty = bars + 7;    // [2]
  uint64_t *halo_full = bars + 9;          // [kNH]
  uint64_t *halo_empty = bars + 9 + kNH;   // [kNH]
  uint64_t *drain = bars + 9 + 2 * kNH;    // MMA completion before TMEM is freed
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 10 + 2 * kNH);
  float *sbias = reinterpret_cast<float *>(smem + L.bias_off);
  volatile uint32_t *go_flag = tmem_slot + 1;
  volatile uint32_t *epi_flag = tmem_slot + 2;
  int *koff = reinterpret_cast<int *>(smem + L.koff_off);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int n_tiles = p.n * p.t * p.tiles_h * p.tiles_w;
  const int hh = kTH + p.kh - 1;
  const int K = p.kt * p.kh * p.kw * p.c_in;
  const uint32_t smem_base = smem_u32(smem);

  if (threadIdx.x == 0) {
    mbar_init(b_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&a_full[i], kBuilders);
      mbar_init(&a_empty[i], 1);
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 4);
    }
    for (int i = 0; i < kNH; ++i) {
      mbar_init(&halo_full[i], 1);
      mbar_init(&halo_empty[i], 1);
    }
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  for (int i = threadIdx.x; i < p.c_out; i += kThreads) sbias[i] = p.bias[i];
  // halo offset of each K index k = ((kt * kh + ih) * kw + iw) * c_in + ci,
  // relative to the output pixel's own halo position; -1 pads K to kpad
  for (int k = threadIdx.x; k < p.kpad; k += kThreads) {
    int off = -1;
    if (k < K) {
      int q = k;
      const int ci = q % p.c_in;
      q /= p.c_in;
      const int iw = q % p.kw;
      q /= p.kw;
      const int ih = q % p.kh;
      const int kt = q / p.kh;
      off = kt * G.kt_stride + ih * G.row + iw * p.c_in + ci;
    }
    koff[k] = off;
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, p.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  bool ok = true;

  if (warp < 4) {
    // ------------------------------ builders -----------------------------------
    const int m = threadIdx.x;  // A row built by this thread
    const int r = m / kTW, c = m % kTW;
    if (threadIdx.x == 0) {
      // weights: one bulk copy for the life of the CTA
      const uint32_t wbytes = static_cast<uint32_t>(p.kpad) * p.c_out * 2u;
      mbar_arrive_expect_tx(b_full, wbytes);
      bulk_load(smem_base + L.b_off, p.wimg, wbytes, b_full);
    }
    int it = 0;
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++it) {
      const int buf = it & 1;
      const int hb = p.use_tma ? it % kNH : 0;
      const uint32_t hph = static_cast<uint32_t>((it / kNH) & 1);
      uint16_t *halo = reinterpret_cast<uint16_t *>(smem + L.halo_off + hb * L.halo_bytes);
      if (!p.use_tma) {
        // stage the halo box with plain loads (zero outside the image): the
        // same shape the TMA box has; batches of loads are issued together
        const Tile tc = thin_tile(tile, p);
        const int helems = p.kt * hh * G.row;
        const long long wc = static_cast<long long>(p.w) * p.c_in;
        const long long x0 = static_cast<long long>(tc.w0 - p.pad_w) * p.c_in - G.rem;
        for (int i0 = 0; i0 < helems; i0 += 8 * kBuilders) {
          uint16_t v[8];
          int dst[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int i = i0 + u * kBuilders + threadIdx.x;
            v[u] = 0;
            dst[u] = -1;
            if (i < helems) {
              const int pos = i % G.row;
              const int q = i / G.row;
              const int rr = q % hh;
              const int kt = q / hh;
              dst[u] = kt * G.kt_stride + rr * G.row + pos;
              const int tau = tc.t + kt - (p.kt - 1);
              const int h = tc.h0 - p.pad_h + rr;
              const long long e = x0 + pos;
              if (h >= 0 && h < p.h && e >= 0 && e < wc) {
                const uint16_t *src = nullptr;
                if (tau >= 0)
                  src = p.x + (static_cast<size_t>(tc.n) * p.t + tau) * p.h * wc;
                else if (p.cache)
                  src = p.cache + (static_cast<size_t>(tc.n) * (p.kt - 1) + tau + (p.kt - 1)) *
                                      p.h * wc;
                if (src) v[u] = src[static_cast<size_t>(h) * wc + e];
              }
            }
          }
#pragma unroll
          for (int u = 0; u < 8; ++u)
            if (dst[u] >= 0) halo[dst[u]] = v[u];
        }
      }
      // thread 0 waits for: this A buffer free (MMAs of two tiles ago done)
      // and, with TMA, this tile's halo landed
      if (threadIdx.x == 0) {
        bool g = mbar_wait_bounded(&a_empty[buf], ((it >> 1) & 1) ^ 1, p.wait_limit_ns, p.status,
                                   11);
        if (g && p.use_tma)
          g = mbar_wait_bounded(&halo_full[hb], hph, p.wait_limit_ns, p.status, 16);
        *go_flag = g ? 1u : 0u;
      }
      asm volatile("bar.sync 1, %0;" ::"n"(kBuilders) : "memory");
      if (!*go_flag) {  // every builder reads the same flag: all leave together
        ok = false;
        break;
      }
      uint8_t *a_buf = smem + L.a_off + buf * L.a_bytes;
      if (p.spec_rgb333) {
        // rows (halo row, column) v = m and, for the last two halo rows,
        // v = 128 + m
        for (int v = m; v < (kTH + 2) * kTW; v += kBuilders)
          build_row_rgb333(halo + (v / kTW) * G.row + G.rem + (v % kTW) * 3,
                           a_buf + (v / kTW) * kRgbRowBytes + (v % kTW) * 16);
      } else {
        uint8_t *a_row = a_buf + (m / 8) * 128 + (m % 8) * 16;
        const uint16_t *hbits = halo + r * G.row + G.rem + c * p.c_in;
        // build row m of A (zero where koff is -1)
        for (int k8 = 0; k8 < p.kpad / 8; ++k8) {
          uint32_t packed[4];
#pragma unroll
          for (int e2 = 0; e2 < 4; ++e2) {
            const int o0 = koff[k8 * 8 + e2 * 2], o1 = koff[k8 * 8 + e2 * 2 + 1];
            const uint32_t lo = o0 >= 0 ? hbits[o0] : 0u;
            const uint32_t hi = o1 >= 0 ? hbits[o1] : 0u;
            packed[e2] = lo | (hi << 16);
          }
          *reinterpret_cast<uint4 *>(a_row + k8 * (kM * 16)) =
              make_uint4(packed[0], packed[1], packed[2], packed[3]);
        }
      }
      // make the generic-proxy writes visible to the tensor core, then signal
      fence_proxy_async_smem();
      mbar_arrive(&a_full[buf]);
      asm volatile("bar.sync 1, %0;" ::"n"(kBuilders) : "memory");  // halo fully read
      if (p.use_tma && threadIdx.x == 0) mbar_arrive(&halo_empty[hb]);
    }
    // Drain: the weight copy issued by thread 0 lands before the CTA may exit.
    if (threadIdx.x == 0) mbar_wait_bounded(b_full, 0, kDrainLimitNs, nullptr, 0);
  } else if (warp == kLoadWarp) {
    // ------------------------------ halo loader (TMA) ----------------------------
    if (p.use_tma && lane == 0) {
      const uint32_t box_bytes = static_cast<uint32_t>(G.row) * hh * 2u;
      uint32_t h_used = 0, h_par = 0;  // ring slots issued, parity of their last issue
      int it = 0;
      for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++it) {
        const int hb = it % kNH;
        if (!mbar_wait_bounded(&halo_empty[hb], ((it / kNH) & 1) ^ 1, p.wait_limit_ns, p.status,
                               17)) {
          ok = false;
          break;
        }
        const Tile tc = thin_tile(tile, p);
        mbar_arrive_expect_tx(&halo_full[hb], box_bytes * p.kt);
        h_used |= 1u << hb;
        h_par = (h_par & ~(1u << hb)) | (static_cast<uint32_t>((it / kNH) & 1) << hb);
        const uint32_t dst = smem_base + L.halo_off + hb * L.halo_bytes;
        const int x0 = (tc.w0 - p.pad_w) * p.c_in - G.rem;  // multiple of 8 elements
        for (int kt = 0; kt < p.kt; ++kt) {
          const int tau = tc.t + kt - (p.kt - 1);
          const bool from_cache = tau < 0 && p.cache;
          tma_load_4d(dst + kt * G.kt_stride * 2, from_cache ? &map_cache : &map_x,
                      &halo_full[hb], x0, tc.h0 - p.pad_h, from_cache ? tau + (p.kt - 1) : tau,
                      tc.n);
        }
      }
      // Drain: every halo load issued here lands before the CTA may exit.
      for (int i = 0; i < kNH; ++i)
        if (h_used >> i & 1u)
          mbar_wait_bounded(&halo_full[i], h_par >> i & 1u, kDrainLimitNs, nullptr, 0);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------ MMA issuer ----------------------------------
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kM, p.c_out);
      // A, im2col tile: [kpad/8][16 row groups][8 rows][8], K core matrices
      // 16 * 128 B apart, M groups 128 B.  RGB 3x3x3: [halo row][4][8][8],
      // K core matrices 128 B apart, M groups (tile rows) 512 B; the K step
      // j of 16 (kernel row kh = j / 2) starts kh rows and (j % 2) * 256 B
      // further on.
      const uint64_t adesc0 =
          p.spec_rgb333 ? smem_desc_noswizzle(smem_base + L.a_off, 128u, kRgbRowBytes)
                        : smem_desc_noswizzle(smem_base + L.a_off, kM * 16u, 128u);
      // B: [kpad/8][c_out][8]: K step c_out*16 B, N step 128 B
      const uint32_t b_lbo = static_cast<uint32_t>(p.c_out) * 16u;
      const uint64_t bdesc0 = smem_desc_noswizzle(smem_base + L.b_off, b_lbo, 128u);
      if (!mbar_wait_bounded(b_full, 0, p.wait_limit_ns, p.status, 12)) ok = false;
      int it = 0;
      for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x, ++it) {
        const int buf = it & 1;
        const uint32_t ph = (it >> 1) & 1;
        if (!mbar_wait_bounded(&acc_empty[buf], ph ^ 1, p.wait_limit_ns, p.status, 13) ||
            !mbar_wait_bounded(&a_full[buf], ph, p.wait_limit_ns, p.status, 14)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t a_st = adesc0 + ((buf * L.a_bytes) >> 4);
        for (int j = 0; j < p.kpad / 16; ++j) {
          const uint32_t a_step = p.spec_rgb333 ? (j / 2) * (kRgbRowBytes / 16) + (j % 2) * 16u
                                                : 2 * j * (kM * 16 / 16);
          umma_bf16(tmem_base + buf * p.c_out, a_st + a_step, bdesc0 + 2 * j * (b_lbo >> 4), idesc,
                    j > 0 ? 1u : 0u);
        }
        umma_commit(&a_empty[buf]);
        umma_commit(&acc_full[buf]);
      }
      // Drain: all MMAs issued here are complete before tensor memory is freed.
      umma_commit(drain);
      mbar_wait_bounded(drain, 0, kDrainLimitNs, nullptr, 0);
    }
  } else {
    // ------------------------------ epilogue (warps 6-9) -------------------------
    // Each thread owns one output pixel (its tensor-memory lane): TMEM ->
    // +bias -> bf16 -> shared staging -> global through the TMA engine.
    //  * store_boxes (c_out % 32 == 0): the tile is staged as c_out / 32
    //    boxes of [128 pixels][32 channels] with the 64-byte swizzle (eight
    //    consecutive pixels write eight different bank quads), and one thread
    //    stores each box with a TMA tensor store, which also clips the tile
    //    at the image edge;
    //  * otherwise each thread bulk-copies its own pixel from a padded slot.
    const int q = warp % 4;
    const int m = q * 32 + lane;
    const int r = m / kTW, c = m % kTW;
    const int et = threadIdx.x - 6 * 32;  // 0..127
    uint8_t *stage = smem + L.stage_off;
    uint8_t *my = stage + m * L.stage_pitch;
    const uint32_t pix_bytes = static_cast<uint32_t>(p.c_out) * 2u;
    int it = 0;
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++it) {
      const int buf = it & 1;
      const Tile tc = thin_tile(tile, p);
      // one thread waits (and, with box stores, lets its previous stores
      // finish reading the staging); the four warps agree through shared
      // memory so all of them take the named barriers or all leave
      if (et == 0) {
        if (p.store_boxes) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
        *epi_flag =
            mbar_wait_bounded(&acc_full[buf], (it >> 1) & 1, p.wait_limit_ns, p.status, 15) ? 1u
                                                                                            : 0u;
      }
      asm volatile("bar.sync 2, %0;" ::"n"(128) : "memory");
      if (!*epi_flag) break;
      tc_fence_after();
      const uint32_t taddr =
          tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(buf * p.c_out);
      if (!p.store_boxes) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
      for (int j0 = 0; j0 < p.c_out; j0 += 48) {
        // up to three 16-column loads in flight, one wait
        const int nld = (p.c_out - j0) >= 48 ? 3 : (p.c_out - j0) / 16;
        uint32_t raw[48];
        __syncwarp();
#pragma unroll
        for (int u = 0; u < 3; ++u)
          if (u < nld) tmem_ld16_nowait(taddr + j0 + 16 * u, raw + 16 * u);
        tmem_wait_ld();
        tmem_regs_after_wait<48>(raw);
        if (j0 + 48 >= p.c_out) {
          // last read of this accumulator: hand the buffer back to the MMA warp
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc_empty[buf]);
        }
#pragma unroll
        for (int u = 0; u < 3; ++u) {
          if (u >= nld) continue;
          const int j = j0 + 16 * u;
          const float4 *b4 = reinterpret_cast<const float4 *>(sbias + j);
          uint32_t o[8];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float4 t4 = b4[i];
            o[2 * i] = pack_bf16x2(__uint_as_float(raw[16 * u + 4 * i]) + t4.x,
                                   __uint_as_float(raw[16 * u + 4 * i + 1]) + t4.y);
            o[2 * i + 1] = pack_bf16x2(__uint_as_float(raw[16 * u + 4 * i + 2]) + t4.z,
                                       __uint_as_float(raw[16 * u + 4 * i + 3]) + t4.w);
          }
          if (p.store_boxes) {
            // channels j..j+15 = chunks (j % 32) / 8 and +1 of box j / 32
            uint8_t *box = stage + (j / 32) * (kM * 64) + m * 64;
            const int ch0 = (j % 32) / 8, sw = (m >> 1) & 3;
            *reinterpret_cast<uint4 *>(box + ((ch0 ^ sw) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
            *reinterpret_cast<uint4 *>(box + (((ch0 + 1) ^ sw) << 4)) =
                make_uint4(o[4], o[5], o[6], o[7]);
          } else {
            reinterpret_cast<uint4 *>(my + j * 2)[0] = make_uint4(o[0], o[1], o[2], o[3]);
            reinterpret_cast<uint4 *>(my + j * 2)[1] = make_uint4(o[4], o[5], o[6], o[7]);
          }
        }
      }
      fence_proxy_async_smem();  // staged bytes, written by this thread, to the TMA engine
      if (p.store_boxes) {
        asm volatile("bar.sync 2, %0;" ::"n"(128) : "memory");
        if (et == 0) {
          for (int bx = 0; bx < p.c_out / 32; ++bx)
            asm volatile(
                "cp.async.bulk.tensor.5d.global.shared::cta.tile.bulk_group"
                " [%0, {%1, %2, %3, %4, %5}], [%6];" ::"l"(reinterpret_cast<uint64_t>(&map_y)),
                "r"(bx * 32), "r"(tc.w0), "r"(tc.h0), "r"(tc.t), "r"(tc.n),
                "r"(smem_u32(stage + bx * (kM * 64)))
                : "memory");
          asm volatile("cp.async.bulk.commit_group;" ::: "memory");
        }
      } else {
        const int h = tc.h0 + r, w = tc.w0 + c;
        if (h < p.h && w < p.w) {
          __nv_bfloat16 *dst =
              p.y + (((static_cast<size_t>(tc.n) * p.t + tc.t) * p.h + h) * p.w + w) * p.c_out;
          asm volatile(
              "cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst),
              "r"(smem_u32(my)), "r"(pix_bytes)
              : "memory");
          asm volatile("cp.async.bulk.commit_group;" ::: "memory");
        }
      }
    }
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, p.tmem_cols);
  }
  (void)ok;
}

__global__ void repack_thin_kernel(const __nv_bfloat16 *__restrict__ w, __nv_bfloat16 *img,
                                   int c_out, int c_in, int taps, int kpad, int spec) {
  // img[k8][co][e] = W[co][ci][tap] at K index k = k8 * 8 + e; 0 past K.
  // Generic order: k = tap * c_in + ci.  RGB 3x3x3 order (spec): three
  // kernel rows of 32, k = kh * 32 + kt * 9 + kw * 3 + ci, 27..31 zero.
  const int total = kpad * c_out;
  const int K = taps * c_in;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < total; i += gridDim.x * blockDim.x) {
    const int e = i % 8;
    const int co = (i / 8) % c_out;
    const int k8 = i / (8 * c_out);
    const int k = k8 * 8 + e;
    __nv_bfloat16 v = __float2bfloat16_rn(0.f);
    if (spec) {
      const int kh = k / 32, j = k % 32;
      if (j < 27) {
        const int kt = j / 9, kw = (j % 9) / 3, ci = j % 3;
        v = w[(static_cast<size_t>(co) * 3 + ci) * 27 + (kt * 3 + kh) * 3 + kw];
      }
    } else if (k < K) {
      const int tap = k / c_in, ci = k % c_in;
      v = w[(static_cast<size_t>(co) * c_in + ci) * taps + tap];
    }
    img[i] = v;
  }
}

}  // namespace

size_t thin_smem_bytes(const ThinArgs &a) { return thin_layout(a).total + 1024; }

int thin_tma_row(const ThinArgs &a) { return halo_geom(a).row; }

cudaError_t launch_repack_thin(const __nv_bfloat16 *w, uint8_t *img, int c_out, int c_in,
                               int taps, int kpad, int spec, cudaStream_t stream) {
  const int total = kpad * c_out;
  repack_thin_kernel<<<(total + 255) / 256, 256, 0, stream>>>(
      w, reinterpret_cast<__nv_bfloat16 *>(img), c_out, c_in, taps, kpad, spec);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_conv_thin(const CUtensorMap &map_x, const CUtensorMap &map_cache,
                             const CUtensorMap &map_y, const ThinArgs &args, unsigned grid,
                             cudaStream_t stream) {
  const size_t smem = thin_smem_bytes(args);
  if (smem > 227 * 1024) return cudaErrorInvalidValue;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(conv_thin_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  conv_thin_kernel<<<grid, kThreads, smem, stream>>>(map_x, map_cache, map_y, args);
  count_launch();
  return cudaGetLastError();
}

}  // namespace cc3d
