// kernels_misc.cu -- the memory-bound kernels around the tensor-core conv:
//   * weight re-tiling into the UMMA shared-memory image (plan time),
//   * the frame-cache update (last kt-1 frames of concat(cache_in, src)),
//   * stand-alone channel RMS_norm + SiLU ("Cosmos3 Wan VAE -- engine size
//     vs context memory", §10.2 WanRMS_norm, §10.4 SiLU), one pass over
//     HBM: bf16 in, fp32 math, bf16 out,
//   * the fp32 SIMT direct causal conv (§10.3) for fp32 plans.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "internal.h"
#include "ptx.cuh"

namespace cc3d {

namespace {

__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&p);
}

__global__ void repack_umma_kernel(const __nv_bfloat16 *__restrict__ w, __nv_bfloat16 *img,
                                   int c_out, int c_in, int taps, int nt, int kc, int rows,
                                   int stages_per_ntile, int stage0) {
  const int n_cc = (c_in + kc - 1) / kc;  // channels past c_in are zero
  const long long total = static_cast<long long>(c_out) * n_cc * kc * taps;
  const long long stage_elems = static_cast<long long>(nt) * kc;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    // image order: ntile, tap, cchunk, then within the stage either
    // slab (kc/8), row (nt), element (8)  -- no-swizzle core matrices -- or
    // (rows) row (nt), channel (kc)       -- plain rows for a tensor map
    long long r = i;
    int e, nl, s;
    if (rows) {
      e = r % kc;
      r /= kc;
      nl = r % nt;
      r /= nt;
      s = 0;
    } else {
      e = r % 8;
      r /= 8;
      nl = r % nt;
      r /= nt;
      s = r % (kc / 8);
      r /= (kc / 8);
    }
    const int cc = r % n_cc;
    r /= n_cc;
    const int tap = r % taps;
    const int ntile = static_cast<int>(r / taps);
    const int co = ntile * nt + nl;
    const int ci = cc * kc + s * 8 + e;
    const long long dst =
        (static_cast<long long>(ntile) * stages_per_ntile + stage0 + tap * n_cc + cc) *
            stage_elems +
        i % stage_elems;
    img[dst] = ci < c_in ? w[(static_cast<long long>(co) * c_in + ci) * taps + tap]
                         : __float2bfloat16(0.f);
  }
}

// The FP8 E4M3 weight image: 128 one-byte channels per chunk, laid out like
// repack_umma_kernel's (rows: [ntile][tap][cchunk][NT][128]; else no-swizzle
// core matrices [ntile][tap][cchunk][8][NT][16]), each weight divided by its
// output channel's scale in fp32 (an IEEE division) and rounded to E4M3.
__global__ void repack_umma_e4m3_kernel(const __nv_bfloat16 *__restrict__ w,
                                        const float *__restrict__ w_scale, uint8_t *img,
                                        int c_out, int c_in, int taps, int nt, int rows) {
  constexpr int kc = 128;
  const int n_cc = c_in / kc;
  const long long total = static_cast<long long>(c_out) * n_cc * kc * taps;
  const long long stage_elems = static_cast<long long>(nt) * kc;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    long long r = i;
    int e, nl, s;
    if (rows) {
      e = r % kc;
      r /= kc;
      nl = r % nt;
      r /= nt;
      s = 0;
    } else {
      e = r % 16;
      r /= 16;
      nl = r % nt;
      r /= nt;
      s = r % (kc / 16);
      r /= (kc / 16);
    }
    const int cc = r % n_cc;
    r /= n_cc;
    const int tap = r % taps;
    const int ntile = static_cast<int>(r / taps);
    const int co = ntile * nt + nl;
    const int ci = cc * kc + s * 16 + e;
    const float q = __fdiv_rn(__bfloat162float(w[(static_cast<long long>(co) * c_in + ci) * taps + tap]),
                              w_scale[co]);
    const long long dst =
        (static_cast<long long>(ntile) * taps * n_cc + tap * n_cc + cc) * stage_elems +
        i % stage_elems;
    img[dst] = static_cast<uint8_t>(pack_e4m3x2(q, 0.f) & 0xFFu);
  }
}

__global__ void scale_vector_kernel(float *v, int count, float s) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < count) v[i] *= s;
}

// q = E4M3(x / scale), 8 elements per thread (16 bytes in, 8 out).
__global__ void quantize_e4m3_kernel(const __nv_bfloat16 *__restrict__ x, long long groups,
                                     float scale, uint8_t *__restrict__ q) {
  for (long long g = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; g < groups;
       g += static_cast<long long>(gridDim.x) * blockDim.x) {
    const uint4 raw = __ldcs(reinterpret_cast<const uint4 *>(x) + g);
    const __nv_bfloat16 *b = reinterpret_cast<const __nv_bfloat16 *>(&raw);
    uint16_t h[4];
#pragma unroll
    for (int k = 0; k < 4; ++k)
      h[k] = pack_e4m3x2(__fdiv_rn(__bfloat162float(b[2 * k]), scale),
                         __fdiv_rn(__bfloat162float(b[2 * k + 1]), scale));
    uint2 out;
    out.x = static_cast<uint32_t>(h[0]) | (static_cast<uint32_t>(h[1]) << 16);
    out.y = static_cast<uint32_t>(h[2]) | (static_cast<uint32_t>(h[3]) << 16);
    __stcs(reinterpret_cast<uint2 *>(q) + g, out);
  }
}

// out[b][i] = concat(cache_in[b] (frames), src[b] (t))[t + i], i < frames.
// 16-byte path: each thread moves U chunks per pass, all loads issued before
// the stores, so enough bytes are in flight to stream at HBM speed.
template <int U>
__global__ void copy_frames16_kernel(const uint8_t *__restrict__ cache_in,
                                     const uint8_t *__restrict__ src, uint8_t *__restrict__ out,
                                     int n, int t, int frames, size_t frame_bytes) {
  const size_t per_frame = frame_bytes / 16;
  const size_t total = static_cast<size_t>(n) * frames * per_frame;
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  for (size_t k0 = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; k0 < total;
       k0 += stride * U) {
    uint4 v[U];
    uint4 *to[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const size_t k = k0 + u * stride;
      to[u] = nullptr;
      v[u] = make_uint4(0, 0, 0, 0);
      if (k < total) {
        const size_t off = k % per_frame;
        const size_t fi = k / per_frame;
        const int i = static_cast<int>(fi % frames);
        const int b = static_cast<int>(fi / frames);
        const int ci = t + i;  // index into concat
        const uint8_t *from = nullptr;
        if (ci < frames) {
          if (cache_in) from = cache_in + (static_cast<size_t>(b) * frames + ci) * frame_bytes;
        } else {
          from = src + (static_cast<size_t>(b) * t + (ci - frames)) * frame_bytes;
        }
        if (from) v[u] = __ldcs(reinterpret_cast<const uint4 *>(from) + off);
        to[u] = reinterpret_cast<uint4 *>(out + (static_cast<size_t>(b) * frames + i) * frame_bytes) +
                off;
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u)
      if (to[u]) *to[u] = v[u];
  }
}

// 2-byte path for frames whose size or start is not 16-byte aligned.
__global__ void copy_frames2_kernel(const uint8_t *__restrict__ cache_in,
                                    const uint8_t *__restrict__ src, uint8_t *__restrict__ out,
                                    int n, int t, int frames, size_t frame_bytes) {
  const size_t per_frame = frame_bytes / 2;
  const size_t total = static_cast<size_t>(n) * frames * per_frame;
  for (size_t k = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; k < total;
       k += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const size_t off = k % per_frame;
    const size_t fi = k / per_frame;
    const int i = static_cast<int>(fi % frames);
    const int b = static_cast<int>(fi / frames);
    const int ci = t + i;
    const uint8_t *from = nullptr;
    if (ci < frames) {
      if (cache_in) from = cache_in + (static_cast<size_t>(b) * frames + ci) * frame_bytes;
    } else {
      from = src + (static_cast<size_t>(b) * t + (ci - frames)) * frame_bytes;
    }
    uint8_t *to = out + (static_cast<size_t>(b) * frames + i) * frame_bytes;
    const uint16_t v = from ? reinterpret_cast<const uint16_t *>(from)[off] : 0;
    reinterpret_cast<uint16_t *>(to)[off] = v;
  }
}

// The frame cache of an RMS_norm + SiLU pass over t frames of hw pixels:
// cache_out [n][2][hw][c] = the last two frames of concat(cache_in or
// zeros, y).  The thread that writes a voxel's output (chunk `g` of 8
// channels) also writes it to the cache when its frame is one of the last
// two, and with a single frame copies cache_in's second frame into the
// first cache frame.
struct RmsCache {
  const __nv_bfloat16 *in;  // [n][2][hw][c] or null (zeros)
  __nv_bfloat16 *out;       // [n][2][hw][c] or null (not written)
  long long hw;             // pixels per frame
  int t;                    // frames of the call
};

__device__ __forceinline__ void rms_cache_store(const RmsCache &k, long long v, int c, int g,
                                                const uint4 &w) {
  const long long per_img = k.hw * k.t;
  const long long img = v / per_img, rem = v - img * per_img;
  const int tt = static_cast<int>(rem / k.hw);
  const long long pix = rem - static_cast<long long>(tt) * k.hw;
  const int f = tt - (k.t - 2);  // frame of the cache this output lands in
  if (f < 0) return;
  __stcs(reinterpret_cast<uint4 *>(k.out + ((img * 2 + f) * k.hw + pix) * c) + g, w);
  if (k.t == 1) {
    const uint4 prev = k.in ? __ldcs(reinterpret_cast<const uint4 *>(
                                         k.in + ((img * 2 + 1) * k.hw + pix) * c) + g)
                            : make_uint4(0, 0, 0, 0);
    __stcs(reinterpret_cast<uint4 *>(k.out + (img * 2 * k.hw + pix) * c) + g, prev);
  }
}

// Packed fp32 pairs (the f32x2 forms of sm_100): two lanes of math per
// instruction.
__device__ __forceinline__ unsigned long long f2_make(float lo, float hi) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_split(unsigned long long v, float &lo, float &hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ unsigned long long f2_mul(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ unsigned long long f2_fma(unsigned long long a, unsigned long long b,
                                                     unsigned long long c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
// two bf16 (low half first) as an fp32 pair
__device__ __forceinline__ unsigned long long f2_from_bf16x2(uint32_t u) {
  return f2_make(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
}

// Lane-mapped RMS_norm + SiLU for channel counts whose 8-channel groups
// split evenly over a power-of-two number of lanes: LPV lanes share a voxel,
// each lane owning GPL groups (GPL = c / 8 / LPV, e.g. C = 192: 8 lanes x 3
// groups, four voxels per warp).  A warp's loads cover 32 * GPL consecutive
// 16-byte chunks (fully coalesced, every lane busy); UNR warp passes are
// loaded before any is used (one: more warps cover the loads' latency
// better than more passes per warp).  Gamma (and beta, when given) sit in
// shared memory as pre-halved fp32 pairs, which keeps the thread at 64
// registers: four CTAs per SM, 32 warps (with them in registers and two
// passes, two CTAs of 128-register threads).  The arithmetic runs on
// packed fp32 pairs (the kernel issues about as many instructions as it
// moves bytes, so halving the multiplies and adds shows).  The sum of
// squares is kept as two pair halves, added, then reduced with a fixed xor
// butterfly over the LPV lanes, so the result does not depend on
// scheduling.
template <int GPL, int UNR, bool BETA>
__global__ void __launch_bounds__(256, UNR == 1 ? 4 : 3)
    rmsnorm_silu_lanes_kernel(const __nv_bfloat16 *__restrict__ x,
                              const float *__restrict__ gamma, const float *__restrict__ beta,
                              long long voxels, int c, int lpv,
                              __nv_bfloat16 *__restrict__ y, RmsCache cache, bool silu) {
  const int lane = threadIdx.x % 32;
  const int vpw = 32 / lpv;                 // voxels per warp pass
  const int sub = lane % lpv, vloc = lane / lpv;
  const long long warp0 = (blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x) / 32;
  const long long nwarps = static_cast<long long>(gridDim.x) * blockDim.x / 32;
  const float scale = sqrtf(static_cast<float>(c));
  // gamma (and beta), halved for SiLU's h = a / 2 (SiLU(a) = h + h *
  // tanh(h)), as fp32 pairs in shared memory: read where they are used, so
  // that three CTAs fit per SM (kept in registers they cost 24-48 of them)
  __shared__ unsigned long long s_g[512], s_b[BETA ? 512 : 1];
  const float half = silu ? 0.5f : 1.0f;
  for (int i = threadIdx.x; i < c / 2; i += blockDim.x) {
    s_g[i] = f2_make(half * __ldg(gamma + 2 * i), half * __ldg(gamma + 2 * i + 1));
    if (BETA) s_b[i] = f2_make(half * __ldg(beta + 2 * i), half * __ldg(beta + 2 * i + 1));
  }
  __syncthreads();
  for (long long vb = warp0 * vpw * UNR; vb < voxels; vb += nwarps * vpw * UNR) {
    uint4 raw[UNR][GPL];
#pragma unroll
    for (int u = 0; u < UNR; ++u) {
      const long long v = vb + u * vpw + vloc;
#pragma unroll
      for (int k = 0; k < GPL; ++k)
        raw[u][k] = v < voxels
                        ? __ldcs(reinterpret_cast<const uint4 *>(x + v * c) + sub + k * lpv)
                        : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < UNR; ++u) {
      const long long v = vb + u * vpw + vloc;
      unsigned long long ss2 = 0ull;
#pragma unroll
      for (int k = 0; k < GPL; ++k) {
        const uint32_t w4[4] = {raw[u][k].x, raw[u][k].y, raw[u][k].z, raw[u][k].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const unsigned long long f = f2_from_bf16x2(w4[q]);
          ss2 = f2_fma(f, f, ss2);
        }
      }
      float s0, s1;
      f2_split(ss2, s0, s1);
      float ss = s0 + s1;
      for (int o = lpv / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      const float inv = scale / fmaxf(sqrtf(ss), 1e-12f);
      if (v >= voxels) continue;
      const unsigned long long inv2 = f2_make(inv, inv);
#pragma unroll
      for (int k = 0; k < GPL; ++k) {
        const int g = sub + k * lpv;
        const uint32_t w4[4] = {raw[u][k].x, raw[u][k].y, raw[u][k].z, raw[u][k].w};
        uint32_t ow[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          // h = x / rms * gamma (+ beta), halved when SiLU follows
          const unsigned long long h =
              f2_fma(f2_mul(f2_from_bf16x2(w4[q]), inv2), s_g[g * 4 + q], BETA ? s_b[g * 4 + q] : 0ull);
          float h0, h1;
          f2_split(h, h0, h1);
          if (silu) {
            float t0, t1;
            asm("tanh.approx.f32 %0, %1;" : "=f"(t0) : "f"(h0));
            asm("tanh.approx.f32 %0, %1;" : "=f"(t1) : "f"(h1));
            f2_split(f2_fma(h, f2_make(t0, t1), h), h0, h1);
          }
          ow[q] = pack2(h0, h1);
        }
        const uint4 w = make_uint4(ow[0], ow[1], ow[2], ow[3]);
        __stcs(reinterpret_cast<uint4 *>(y + v * c) + g, w);
        if (cache.out) rms_cache_store(cache, v, c, g, w);
      }
    }
  }
}

// A CTA normalises a contiguous run of voxels: its 256 threads load the
// run's consecutive 16-byte chunks (8 channels each, CPT per thread, all
// issued before any use), write each chunk's sum of squares to shared
// memory, then one thread per voxel adds its chunks' partial sums in
// channel order (a fixed order: the result does not depend on scheduling),
// and every thread scales, applies SiLU and stores its chunks.
template <int CPT>
__global__ void __launch_bounds__(256)
    rmsnorm_silu_kernel(const __nv_bfloat16 *__restrict__ x, const float *__restrict__ gamma,
                        const float *__restrict__ beta, long long voxels, int c,
                        __nv_bfloat16 *__restrict__ y, RmsCache cache, bool silu) {
  __shared__ float partial[256 * CPT];
  __shared__ float inv_s[256 * CPT];
  const int groups = c / 8;
  const int vpb = (256 * CPT) / groups;  // voxels per CTA pass
  const float scale = sqrtf(static_cast<float>(c));
  for (long long v0 = static_cast<long long>(blockIdx.x) * vpb; v0 < voxels;
       v0 += static_cast<long long>(gridDim.x) * vpb) {
    const int nv = static_cast<int>(voxels - v0 < vpb ? voxels - v0 : vpb);
    const int nch = nv * groups;
    const uint4 *src = reinterpret_cast<const uint4 *>(x + v0 * c);
    uint4 raw[CPT];
#pragma unroll
    for (int k = 0; k < CPT; ++k) {
      const int idx = threadIdx.x + 256 * k;
      raw[k] = idx < nch ? __ldcs(src + idx) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int k = 0; k < CPT; ++k) {
      const int idx = threadIdx.x + 256 * k;
      const __nv_bfloat16 *b = reinterpret_cast<const __nv_bfloat16 *>(&raw[k]);
      float ss = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float f = __bfloat162float(b[e]);
        ss = fmaf(f, f, ss);
      }
      if (idx < nch) partial[idx] = ss;
    }
    __syncthreads();
    for (int v = threadIdx.x; v < nv; v += 256) {
      float ss = 0.f;
      for (int g = 0; g < groups; ++g) ss += partial[v * groups + g];
      inv_s[v] = scale / fmaxf(sqrtf(ss), 1e-12f);
    }
    __syncthreads();
    uint4 *dst = reinterpret_cast<uint4 *>(y + v0 * c);
#pragma unroll
    for (int k = 0; k < CPT; ++k) {
      const int idx = threadIdx.x + 256 * k;
      if (idx < nch) {
        const int v = idx / groups, g = idx - (idx / groups) * groups;
        const float inv = inv_s[v];
        const float4 g0 = __ldg(reinterpret_cast<const float4 *>(gamma + g * 8));
        const float4 g1 = __ldg(reinterpret_cast<const float4 *>(gamma + g * 8) + 1);
        const float gm[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
        const __nv_bfloat16 *b = reinterpret_cast<const __nv_bfloat16 *>(&raw[k]);
        float o[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          float a = __bfloat162float(b[e]) * inv * gm[e];
          if (beta) a += __ldg(beta + g * 8 + e);
          o[e] = silu ? silu_fast(a) : a;
        }
        uint4 w;
        w.x = pack2(o[0], o[1]);
        w.y = pack2(o[2], o[3]);
        w.z = pack2(o[4], o[5]);
        w.w = pack2(o[6], o[7]);
        __stcs(dst + idx, w);
        if (cache.out) rms_cache_store(cache, v0 + v, c, g, w);
      }
    }
    __syncthreads();  // partial / inv_s are rewritten by the next pass
  }
}

// fp32 direct causal conv: one thread per output element, NDHWC, c_out
// fastest so a warp shares its input pixels.  Accumulation order: c_in,
// kt, kh, kw; bias last.
__global__ void conv_fp32_kernel(Fp32Args a) {
  const long long total = static_cast<long long>(a.n) * a.t * a.h * a.w_ * a.c_out;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    long long r = i;
    const int co = r % a.c_out;
    r /= a.c_out;
    const int w = r % a.w_;
    r /= a.w_;
    const int h = r % a.h;
    r /= a.h;
    const int t = r % a.t;
    const int n = static_cast<int>(r / a.t);
    float acc = 0.f;
    const int front = a.kt - 1;
    for (int ci = 0; ci < a.c_in; ++ci)
      for (int kt = 0; kt < a.kt; ++kt) {
        const int tau = t + kt - front;
        const float *base;
        if (tau >= 0) {
          base = a.x + (static_cast<long long>(n) * a.t + tau) * a.h * a.w_ * a.c_in;
        } else if (a.cache) {
          base = a.cache + (static_cast<long long>(n) * front + tau + front) * a.h * a.w_ * a.c_in;
        } else {
          continue;
        }
        for (int kh = 0; kh < a.kh; ++kh) {
          const int hh = h + kh - a.pad_h;
          if (hh < 0 || hh >= a.h) continue;
          for (int kw = 0; kw < a.kw; ++kw) {
            const int ww = w + kw - a.pad_w;
            if (ww < 0 || ww >= a.w_) continue;
            const float xv = base[(static_cast<long long>(hh) * a.w_ + ww) * a.c_in + ci];
            const float wv = a.w[(((static_cast<long long>(co) * a.c_in + ci) * a.kt + kt) * a.kh +
                                  kh) * a.kw + kw];
            acc = fmaf(wv, xv, acc);
          }
        }
      }
    a.y[i] = acc + a.bias[co];
  }
}

int grid_for(long long work, int block) {
  long long g = (work + block - 1) / block;
  if (g > 148LL * 16) g = 148LL * 16;
  if (g < 1) g = 1;
  return static_cast<int>(g);
}

}  // namespace

cudaError_t launch_repack_umma(const __nv_bfloat16 *w, uint8_t *img, int c_out, int c_in,
                               int taps, int nt, int kc, int rows, int stages_per_ntile,
                               int stage0, cudaStream_t stream) {
  const long long total = static_cast<long long>(c_out) * ((c_in + kc - 1) / kc) * kc * taps;
  repack_umma_kernel<<<grid_for(total, 256), 256, 0, stream>>>(
      w, reinterpret_cast<__nv_bfloat16 *>(img), c_out, c_in, taps, nt, kc, rows,
      stages_per_ntile, stage0);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_repack_umma_e4m3(const __nv_bfloat16 *w, const float *w_scale, uint8_t *img,
                                    int c_out, int c_in, int taps, int nt, int rows,
                                    cudaStream_t stream) {
  if (c_in % 128 != 0 || nt < 1 || c_out % nt != 0) return cudaErrorInvalidValue;
  const long long total = static_cast<long long>(c_out) * c_in * taps;
  repack_umma_e4m3_kernel<<<grid_for(total, 256), 256, 0, stream>>>(w, w_scale, img, c_out, c_in,
                                                                     taps, nt, rows);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_scale_vector(float *v, int count, float s, cudaStream_t stream) {
  scale_vector_kernel<<<(count + 255) / 256, 256, 0, stream>>>(v, count, s);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_quantize_e4m3(const __nv_bfloat16 *x, size_t count, float scale, uint8_t *q,
                                 cudaStream_t stream) {
  if (count % 8 != 0) return cudaErrorInvalidValue;
  const long long groups = static_cast<long long>(count / 8);
  long long g = (groups + 255) / 256;
  if (g > 148LL * 16) g = 148LL * 16;
  if (g < 1) g = 1;
  quantize_e4m3_kernel<<<static_cast<int>(g), 256, 0, stream>>>(x, groups, scale, q);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_cache_update(const void *cache_in, const void *src, void *cache_out, int n,
                                int t, int frames, size_t frame_bytes, cudaStream_t stream) {
  if (frames <= 0) return cudaSuccess;
  const bool vec16 = frame_bytes % 16 == 0 && (reinterpret_cast<uintptr_t>(src) % 16) == 0 &&
                     (reinterpret_cast<uintptr_t>(cache_out) % 16) == 0 &&
                     (reinterpret_cast<uintptr_t>(cache_in) % 16) == 0;
  const auto *ci = static_cast<const uint8_t *>(cache_in);
  const auto *sr = static_cast<const uint8_t *>(src);
  auto *co = static_cast<uint8_t *>(cache_out);
  if (vec16) {
    constexpr int kU = 4;
    const long long work = static_cast<long long>(n) * frames * (frame_bytes / 16);
    long long g = (work / kU + 255) / 256;
    if (g > 148LL * 8) g = 148LL * 8;
    if (g < 1) g = 1;
    copy_frames16_kernel<kU><<<static_cast<int>(g), 256, 0, stream>>>(ci, sr, co, n, t, frames,
                                                                        frame_bytes);
  } else {
    const long long work = static_cast<long long>(n) * frames * (frame_bytes / 2);
    copy_frames2_kernel<<<grid_for(work, 256), 256, 0, stream>>>(ci, sr, co, n, t, frames,
                                                                 frame_bytes);
  }
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_rmsnorm_silu(const __nv_bfloat16 *x, const float *gamma, const float *beta,
                                int n, int t, long long hw, int c, __nv_bfloat16 *y,
                                const __nv_bfloat16 *cache_in, __nv_bfloat16 *cache_out,
                                bool silu, cudaStream_t stream) {
  const int groups = c / 8;
  if (groups < 1 || n < 1 || t < 1 || hw < 1) return cudaErrorInvalidValue;
  const long long voxels = static_cast<long long>(n) * t * hw;
  RmsCache cache;
  cache.in = cache_in;
  cache.out = cache_out;
  cache.hw = hw;
  cache.t = t;
  // lanes per voxel: the largest power of two (<= 32) dividing the groups
  int lpv = 1;
  while (lpv < 32 && groups % (lpv * 2) == 0) lpv *= 2;
  const int gpl = groups / lpv;
  if (gpl <= 4) {
    constexpr int kUnr = 1;
    const long long per_warp = static_cast<long long>(32 / lpv) * kUnr;
    long long warps = (voxels + per_warp - 1) / per_warp;
    long long g = (warps * 32 + 255) / 256;
    if (g > 148LL * 16) g = 148LL * 16;
    if (g < 1) g = 1;
    const int grid = static_cast<int>(g);
    switch (gpl) {
#define CC3D_RMS_LANES(G)                                                                     \
  (beta ? rmsnorm_silu_lanes_kernel<G, kUnr, true><<<grid, 256, 0, stream>>>(                  \
              x, gamma, beta, voxels, c, lpv, y, cache, silu)                                   \
        : rmsnorm_silu_lanes_kernel<G, kUnr, false><<<grid, 256, 0, stream>>>(                 \
              x, gamma, beta, voxels, c, lpv, y, cache, silu))
      case 1: CC3D_RMS_LANES(1); break;
      case 2: CC3D_RMS_LANES(2); break;
      case 3: CC3D_RMS_LANES(3); break;
      default: CC3D_RMS_LANES(4); break;
#undef CC3D_RMS_LANES
    }
  } else {
    constexpr int kCpt = 12;  // 16-byte chunks per thread and pass
    if (groups > 256 * kCpt) return cudaErrorInvalidValue;
    const int vpb = (256 * kCpt) / groups;
    long long g = (voxels + vpb - 1) / vpb;
    if (g > 148LL * 8) g = 148LL * 8;
    if (g < 1) g = 1;
    rmsnorm_silu_kernel<kCpt><<<static_cast<int>(g), 256, 0, stream>>>(x, gamma, beta, voxels,
                                                                       c, y, cache, silu);
  }
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_conv_fp32(const Fp32Args &a, cudaStream_t stream) {
  const long long total = static_cast<long long>(a.n) * a.t * a.h * a.w_ * a.c_out;
  conv_fp32_kernel<<<grid_for(total, 128), 128, 0, stream>>>(a);
  count_launch();
  return cudaGetLastError();
}

}  // namespace cc3d
