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

namespace cc3d {

namespace {

__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&p);
}

__global__ void repack_umma_kernel(const __nv_bfloat16 *__restrict__ w, __nv_bfloat16 *img,
                                   int c_out, int c_in, int taps, int nt, int kc) {
  const long long total = static_cast<long long>(c_out) * c_in * taps;
  const int n_cc = c_in / kc;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    // image order: ntile, tap, cchunk, slab (kc/8), row (nt), element (8)
    long long r = i;
    const int e = r % 8;
    r /= 8;
    const int nl = r % nt;
    r /= nt;
    const int s = r % (kc / 8);
    r /= (kc / 8);
    const int cc = r % n_cc;
    r /= n_cc;
    const int tap = r % taps;
    const int ntile = static_cast<int>(r / taps);
    const int co = ntile * nt + nl;
    const int ci = cc * kc + s * 8 + e;
    img[i] = w[(static_cast<long long>(co) * c_in + ci) * taps + tap];
  }
}

__global__ void copy_frames_kernel(const uint8_t *__restrict__ cache_in,
                                   const uint8_t *__restrict__ src, uint8_t *__restrict__ out,
                                   int n, int t, int frames, size_t frame_bytes, int vec16) {
  // out[b][i] = concat(cache_in[b] (frames), src[b] (t))[t + i], i < frames
  const size_t per_frame = vec16 ? frame_bytes / 16 : frame_bytes / 2;
  const size_t total = static_cast<size_t>(n) * frames * per_frame;
  for (size_t k = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; k < total;
       k += static_cast<size_t>(gridDim.x) * blockDim.x) {
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
    uint8_t *to = out + (static_cast<size_t>(b) * frames + i) * frame_bytes;
    if (vec16) {
      uint4 v = from ? reinterpret_cast<const uint4 *>(from)[off] : make_uint4(0, 0, 0, 0);
      reinterpret_cast<uint4 *>(to)[off] = v;
    } else {
      uint16_t v = from ? reinterpret_cast<const uint16_t *>(from)[off] : 0;
      reinterpret_cast<uint16_t *>(to)[off] = v;
    }
  }
}

// A warp normalises VPW voxels per iteration; lane l owns channel groups
// l, l+32, ... of 8 channels (16 bytes) of each.  All loads of the VPW
// voxels are issued before any reduction so enough bytes are in flight to
// keep HBM busy.  The sum of squares is reduced with a fixed xor butterfly,
// so the result does not depend on scheduling.
template <int CPL, int VPW>
__global__ void rmsnorm_silu_kernel(const __nv_bfloat16 *__restrict__ x,
                                    const float *__restrict__ gamma,
                                    const float *__restrict__ beta, long long voxels, int c,
                                    __nv_bfloat16 *__restrict__ y) {
  const int lane = threadIdx.x % 32;
  const long long warp0 = (blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x) / 32;
  const long long nwarps = static_cast<long long>(gridDim.x) * blockDim.x / 32;
  const int groups = c / 8;
  const float scale = sqrtf(static_cast<float>(c));
  for (long long v0 = warp0 * VPW; v0 < voxels; v0 += nwarps * VPW) {
    uint4 raw[VPW][CPL];
#pragma unroll
    for (int u = 0; u < VPW; ++u)
#pragma unroll
      for (int k = 0; k < CPL; ++k) {
        const int g = lane + 32 * k;
        raw[u][k] = make_uint4(0, 0, 0, 0);
        if (v0 + u < voxels && g < groups)
          raw[u][k] = __ldcs(reinterpret_cast<const uint4 *>(x + (v0 + u) * c) + g);
      }
    float inv[VPW];
#pragma unroll
    for (int u = 0; u < VPW; ++u) {
      float ss = 0.f;
#pragma unroll
      for (int k = 0; k < CPL; ++k) {
        const __nv_bfloat16 *b = reinterpret_cast<const __nv_bfloat16 *>(&raw[u][k]);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float f = __bfloat162float(b[e]);
          ss = fmaf(f, f, ss);
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      inv[u] = scale / fmaxf(sqrtf(ss), 1e-12f);
    }
#pragma unroll
    for (int u = 0; u < VPW; ++u)
#pragma unroll
      for (int k = 0; k < CPL; ++k) {
        const int g = lane + 32 * k;
        if (v0 + u < voxels && g < groups) {
          const __nv_bfloat16 *b = reinterpret_cast<const __nv_bfloat16 *>(&raw[u][k]);
          float o[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int ch = g * 8 + e;
            float a = __bfloat162float(b[e]) * inv[u] * __ldg(gamma + ch);
            if (beta) a += __ldg(beta + ch);
            o[e] = a / (1.0f + __expf(-a));
          }
          uint4 w;
          w.x = pack2(o[0], o[1]);
          w.y = pack2(o[2], o[3]);
          w.z = pack2(o[4], o[5]);
          w.w = pack2(o[6], o[7]);
          __stcs(reinterpret_cast<uint4 *>(y + (v0 + u) * c) + g, w);
        }
      }
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
                               int taps, int nt, int kc, cudaStream_t stream) {
  const long long total = static_cast<long long>(c_out) * c_in * taps;
  repack_umma_kernel<<<grid_for(total, 256), 256, 0, stream>>>(
      w, reinterpret_cast<__nv_bfloat16 *>(img), c_out, c_in, taps, nt, kc);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_cache_update(const void *cache_in, const void *src, void *cache_out, int n,
                                int t, int frames, size_t frame_bytes, cudaStream_t stream) {
  if (frames <= 0) return cudaSuccess;
  const int vec16 = (frame_bytes % 16 == 0 && (reinterpret_cast<uintptr_t>(src) % 16) == 0 &&
                     (reinterpret_cast<uintptr_t>(cache_out) % 16) == 0 &&
                     (reinterpret_cast<uintptr_t>(cache_in) % 16) == 0)
                        ? 1
                        : 0;
  const long long work =
      static_cast<long long>(n) * frames * (vec16 ? frame_bytes / 16 : frame_bytes / 2);
  copy_frames_kernel<<<grid_for(work, 256), 256, 0, stream>>>(
      static_cast<const uint8_t *>(cache_in), static_cast<const uint8_t *>(src),
      static_cast<uint8_t *>(cache_out), n, t, frames, frame_bytes, vec16);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_rmsnorm_silu(const __nv_bfloat16 *x, const float *gamma, const float *beta,
                                long long voxels, int c, __nv_bfloat16 *y, cudaStream_t stream) {
  const int groups = c / 8;
  const int cpl = (groups + 31) / 32;
  constexpr int kVpw = 4;
  const int block = 256;
  long long warps = (voxels + kVpw - 1) / kVpw;
  long long g = (warps * 32 + block - 1) / block;
  if (g > 148LL * 16) g = 148LL * 16;
  if (g < 1) g = 1;
  const int grid = static_cast<int>(g);
  switch (cpl) {
    case 1: rmsnorm_silu_kernel<1, kVpw><<<grid, block, 0, stream>>>(x, gamma, beta, voxels, c, y); break;
    case 2: rmsnorm_silu_kernel<2, kVpw><<<grid, block, 0, stream>>>(x, gamma, beta, voxels, c, y); break;
    case 3: rmsnorm_silu_kernel<3, kVpw><<<grid, block, 0, stream>>>(x, gamma, beta, voxels, c, y); break;
    case 4: rmsnorm_silu_kernel<4, kVpw><<<grid, block, 0, stream>>>(x, gamma, beta, voxels, c, y); break;
    default: return cudaErrorInvalidValue;
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
