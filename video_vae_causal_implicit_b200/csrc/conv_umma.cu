// conv_umma.cu -- bf16 implicit-GEMM causal Conv3D on tcgen05 tensor cores.
//
// Operation ("Cosmos3 Wan VAE -- engine size vs context memory", §10.3
// WanCausalConv3d and its implicit-GEMM view): M = output voxels,
// N = C_out, K = C_in * kt * kh * kw; every tap is summed into one fp32
// accumulator held in tensor memory; bias is added once in the epilogue
// ("cache-aware video decoder lowering" summary: bias after the sum).
//
// Tiling.  An output tile is TW = 8 columns x TH = 16 rows of one frame
// (M = 128 rows of the GEMM, row m = 8 * r + c) by NT output channels.  The
// kernel is persistent: one CTA per SM walks the tiles round-robin.  The K
// loop of a tile runs over (kt, channel chunk of KC, kh, kw).
//
// A operand: for each (kt, channel chunk) one TMA box brings the input
// halo of the tile -- (TH + kh - 1) x (TW + kw - 1) pixels x KC channels --
// from the current chunk x (frame tau = t + kt - (kt_size - 1) >= 0) or the
// frame cache (tau < 0).  Spatial padding is TMA out-of-bounds zero fill,
// and a frame before the chunk with no cache (all zeros) is skipped: its
// stage is neither loaded nor multiplied.  No padded copy exists anywhere.  For 64-channel
// chunks the halo is one TMA box with the 128-byte swizzle,
//     [halo rows][halo cols][64 channels = 128 bytes],
// and the A matrix of spatial tap (kh, kw) is the same buffer seen from a
// start address shifted by (kh * halo_cols + kw) whole 128-byte rows: the
// tensor core un-swizzles by absolute shared-memory address, so a row-shifted
// view reads correctly (checked on B200).  One load serves all kh * kw taps.
// 32- and 96-channel chunks use no-swizzle core matrices instead,
//     [KC/8 slabs][halo rows][halo cols][8 channels],
// loaded as one 8-channel box per slab, where a pixel shift is 16 bytes.
//
// B operand: the weights, re-tiled at plan time into the exact shared
// memory image of each (N tile, tap, channel chunk) stage
//     [KC/8][NT][8 channels]   (K-major core matrices),
// fetched with one 1-D bulk copy per stage.
//
// Warp roles (192 threads): warp 0 issues the loads, warp 1 owns tensor
// memory and issues tcgen05.mma from one thread, warps 2..5 run the
// epilogue (tensor memory -> registers -> bias / residual / RMS+SiLU ->
// bf16 -> global).  Two accumulators live in tensor memory, so the
// epilogue of one tile overlaps the MMAs of the next.  Stages are handed
// over with mbarriers; every wait is bounded and reports through the status
// word instead of hanging.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "internal.h"
#include "ptx.cuh"

namespace cc3d {

namespace {

constexpr int kTW = 8;    // tile columns (one core matrix of rows)
constexpr int kTH = 16;   // tile rows -> M = 128
constexpr int kM = kTW * kTH;
constexpr int kThreads = 192;
constexpr int kEpiWarps = 4;
// Bound of the drain waits at exit (loads / MMAs already issued finish in
// microseconds; this only guards against a broken pipeline).
constexpr unsigned long long kDrainLimitNs = 100ull * 1000000ull;

struct SmemLayout {
  uint32_t a_off, a_stage, slab, b_off, b_stage, bar_off, total;
  int na, nb;
};

__host__ __device__ inline uint32_t round_up(uint32_t v, uint32_t a) { return (v + a - 1) / a * a; }

__host__ __device__ inline SmemLayout make_layout(int kc, int nt, int kh, int kw, int na, int nb) {
  SmemLayout L;
  const uint32_t hh = kTH + kh - 1, hw = kTW + kw - 1;
  L.slab = round_up(hh * hw * 16u, 128u);
  L.a_stage = (kc / 8) * L.slab;
  L.b_stage = static_cast<uint32_t>(nt) * kc * 2u;
  L.na = na;
  L.nb = nb;
  L.a_off = 0;
  L.b_off = round_up(L.a_off + na * L.a_stage, 1024u);
  L.bar_off = round_up(L.b_off + nb * L.b_stage, 64u);
  // full_a, empty_a, full_b, empty_b, acc_full[2], acc_empty[2], drain, tmem slot
  L.total = L.bar_off + 8u * (2 * na + 2 * nb + 5) + 16u;
  return L;
}

struct TileCoord {
  int ntile, n, t, h0, w0;
};

// Tile order: N tile fastest (CTAs sharing an input halo run together),
// then tile column, tile row, frame, batch image.
__device__ __forceinline__ TileCoord decode_tile(int tile, const UmmaArgs &p) {
  TileCoord c;
  c.ntile = tile % p.n_ntiles;
  int mt = tile / p.n_ntiles;
  const int tw = mt % p.tiles_w;
  mt /= p.tiles_w;
  const int th = mt % p.tiles_h;
  mt /= p.tiles_h;
  c.t = mt % p.t;
  c.n = mt / p.t;
  c.w0 = tw * kTW;
  c.h0 = th * kTH;
  return c;
}

template <int KC, int KS>
__global__ void __launch_bounds__(kThreads, 1)
    conv_umma_kernel(const __grid_constant__ CUtensorMap map_x,
                     const __grid_constant__ CUtensorMap map_cache, UmmaArgs p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // Align the dynamic shared window to 1 KiB ourselves (the attribute is a
  // request, not a guarantee).
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const SmemLayout L = make_layout(KC, p.nt, KS, KS, p.na, p.nb);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L.bar_off);
  uint64_t *full_a = bars;
  uint64_t *empty_a = full_a + L.na;
  uint64_t *full_b = empty_a + L.na;
  uint64_t *empty_b = full_b + L.nb;
  uint64_t *acc_full = empty_b + L.nb;   // [2]
  uint64_t *acc_empty = acc_full + 2;    // [2]
  uint64_t *drain = acc_empty + 2;       // MMA completion before TMEM is freed
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  const int n_cc = p.c_in / KC;   // channel chunks
  const int n_a = p.kt * n_cc;    // A stages per tile
  const uint32_t halo_w = kTW + KS - 1;
  const int n_tiles = p.n * p.t * p.tiles_h * p.tiles_w * p.n_ntiles;

  if (threadIdx.x == 0) {
    for (int i = 0; i < L.na; ++i) {
      mbar_init(&full_a[i], 1);
      mbar_init(&empty_a[i], 1);
    }
    for (int i = 0; i < L.nb; ++i) {
      mbar_init(&full_b[i], 1);
      mbar_init(&empty_b[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], kEpiWarps);
    }
    mbar_init(drain, 1);
    fence_mbar_init();
    prefetch_tmap(&map_x);
    if (p.has_cache) prefetch_tmap(&map_cache);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, p.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t smem_base = smem_u32(smem);
  bool ok = true;

  if (warp == 0) {
    // ------------------------------ producer ------------------------------------
    if (lane == 0) {
      const uint32_t a_bytes = (KC / 8) * (8u * 2u * halo_w * (kTH + KS - 1));
      int sa = 0, sb = 0;
      uint32_t pa = 0, pb = 0;
      // stages issued at least once, and the phase parity of their last issue
      uint32_t a_used = 0, a_par = 0, b_used = 0, b_par = 0;
      for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x) {
        const TileCoord tc0 = decode_tile(tile, p);
        const uint8_t *wsrc =
            p.wimg + static_cast<size_t>(tc0.ntile) * p.kt * KS * KS * n_cc * L.b_stage;
        for (int ia = 0; ia < n_a && ok; ++ia) {
          const int kt = ia / n_cc, cc = ia % n_cc;
          // A frame before the chunk with no cache is all zeros: its stage
          // (and its taps' weights) is skipped here and by the MMA issuer.
          if (tc0.t + kt - (p.kt - 1) < 0 && !p.has_cache) continue;
          if (!mbar_wait_bounded(&empty_a[sa], pa ^ 1, p.wait_limit_ns, p.status, 1)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full_a[sa], a_bytes);
          a_used |= 1u << sa;
          a_par = (a_par & ~(1u << sa)) | (pa << sa);
          const int tau = tc0.t + kt - (p.kt - 1);
          const bool from_cache = tau < 0;  // (zero frames were skipped above)
          const CUtensorMap *map = from_cache ? &map_cache : &map_x;
          const int tcoord = from_cache ? tau + (p.kt - 1) : tau;
          const uint32_t dst = smem_base + L.a_off + sa * L.a_stage;
#pragma unroll
          for (int s = 0; s < KC / 8; ++s)
            tma_load_5d(dst + s * L.slab, map, &full_a[sa], cc * KC + s * 8, tc0.w0 - KS / 2,
                        tc0.h0 - KS / 2, tcoord, tc0.n);
          if (++sa == L.na) { sa = 0; pa ^= 1; }
#pragma unroll 1
          for (int ts = 0; ts < KS * KS; ++ts) {
            if (!mbar_wait_bounded(&empty_b[sb], pb ^ 1, p.wait_limit_ns, p.status, 2)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&full_b[sb], L.b_stage);
            b_used |= 1u << sb;
            b_par = (b_par & ~(1u << sb)) | (pb << sb);
            const size_t stage_idx = static_cast<size_t>(kt * KS * KS + ts) * n_cc + cc;
            bulk_load(smem_base + L.b_off + sb * L.b_stage, wsrc + stage_idx * L.b_stage,
                      L.b_stage, &full_b[sb]);
            if (++sb == L.nb) { sb = 0; pb ^= 1; }
          }
        }
      }
      // Drain: every load this thread issued lands before the CTA may exit
      // (after a timeout elsewhere the consumer may not have waited for it).
      for (int i = 0; i < L.na; ++i)
        if (a_used >> i & 1u)
          mbar_wait_bounded(&full_a[i], a_par >> i & 1u, kDrainLimitNs, nullptr, 0);
      for (int i = 0; i < L.nb; ++i)
        if (b_used >> i & 1u)
          mbar_wait_bounded(&full_b[i], b_par >> i & 1u, kDrainLimitNs, nullptr, 0);
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer ----------------------------------
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kM, p.nt);
      const uint32_t a_sbo = halo_w * 16u;
      const uint32_t b_lbo = static_cast<uint32_t>(p.nt) * 16u;
      // Descriptors of stage 0; other stages, taps and K steps only move the
      // start address (low 14 bits, 16-byte units), so they are additions.
      // A 16-element K step is two 8-channel slabs (A) or two core-matrix
      // columns (B) further on; a halo pixel is 16 bytes.
      const uint64_t adesc0 = smem_desc_noswizzle(smem_base + L.a_off, L.slab, a_sbo);
      const uint64_t bdesc0 = smem_desc_noswizzle(smem_base + L.b_off, b_lbo, 128u);
      const uint32_t astep16 = 2u * (L.slab >> 4);
      const uint32_t bstep16 = 2u * (b_lbo >> 4);
      const uint32_t pix16 = 1u;
      int sa = 0, sb = 0;
      uint32_t pa = 0, pb = 0;
      int it = 0;
      for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x, ++it) {
        const int buf = it & 1;
        // wait until the epilogue has drained this accumulator buffer
        if (!mbar_wait_bounded(&acc_empty[buf], ((it >> 1) & 1) ^ 1, p.wait_limit_ns, p.status,
                               6)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * p.nt;
        const TileCoord tcm = decode_tile(tile, p);
        uint32_t accumulate = 0;
        for (int ia = 0; ia < n_a && ok; ++ia) {
          // the same zero-frame stages the producer skipped; adding their
          // exact zeros would not change the accumulator
          if (tcm.t + ia / n_cc - (p.kt - 1) < 0 && !p.has_cache) continue;
          if (!mbar_wait_bounded(&full_a[sa], pa, p.wait_limit_ns, p.status, 3)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t a_st = adesc0 + ((sa * L.a_stage) >> 4);
#pragma unroll
          for (int ts = 0; ts < KS * KS; ++ts) {
            if (!mbar_wait_bounded(&full_b[sb], pb, p.wait_limit_ns, p.status, 4)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint64_t a_tap = a_st + ((ts / KS) * halo_w + (ts % KS)) * pix16;
            const uint64_t b_st = bdesc0 + ((sb * L.b_stage) >> 4);
#pragma unroll
            for (int j = 0; j < KC / 16; ++j) {
              umma_bf16(d_tmem, a_tap + j * astep16, b_st + j * bstep16, idesc, accumulate);
              accumulate = 1;
            }
            umma_commit(&empty_b[sb]);  // frees the B stage when these MMAs finish
            if (++sb == L.nb) { sb = 0; pb ^= 1; }
          }
          umma_commit(&empty_a[sa]);
          if (++sa == L.na) { sa = 0; pa ^= 1; }
        }
        umma_commit(&acc_full[buf]);  // accumulator ready for the epilogue
      }
      // Drain: all MMAs issued here are complete before tensor memory is freed.
      umma_commit(drain);
      mbar_wait_bounded(drain, 0, kDrainLimitNs, nullptr, 0);
    }
  } else {
    // ------------------------------ epilogue ------------------------------------
    const int q = warp % 4;  // tensor-memory lane quarter this warp may read
    const int m = q * 32 + lane;
    const int r = m / kTW, c = m % kTW;
    int it = 0;
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++it) {
      const int buf = it & 1;
      const TileCoord tc0 = decode_tile(tile, p);
      const int h = tc0.h0 + r, w = tc0.w0 + c;
      const bool valid = (h < p.h) && (w < p.w);
      uint32_t got = 0;
      if (lane == 0)
        got = mbar_wait_bounded(&acc_full[buf], (it >> 1) & 1, p.wait_limit_ns, p.status, 5)
                  ? 1u
                  : 0u;
      got = __shfl_sync(0xffffffffu, got, 0);
      if (!got) break;
      tc_fence_after();
      const uint32_t taddr =
          tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(buf * p.nt);
      const int n0 = tc0.ntile * p.nt;
      const size_t pix = ((static_cast<size_t>(tc0.n) * p.t + tc0.t) * p.h + h) * p.w + w;
      __nv_bfloat16 *yrow = p.y + pix * p.c_out + n0;
      const __nv_bfloat16 *rrow = p.residual ? p.residual + pix * p.c_out + n0 : nullptr;
      float inv = 1.0f;
      if (p.epi == 2) {
        // pass 1: sum of squares of the biased row (three loads in flight)
        float ss = 0.f;
        for (int j0 = 0; j0 < p.nt; j0 += 48) {
          const int nld = (p.nt - j0) >= 48 ? 3 : (p.nt - j0) / 16;
          uint32_t raw[48];
          __syncwarp();
#pragma unroll
          for (int u = 0; u < 3; ++u)
            if (u < nld) tmem_ld16_nowait(taddr + j0 + 16 * u, raw + 16 * u);
          tmem_wait_ld();
          tmem_regs_after_wait<48>(raw);
#pragma unroll
          for (int u = 0; u < 3; ++u) {
            if (u >= nld) continue;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float hv = __uint_as_float(raw[16 * u + i]) + p.bias[n0 + j0 + 16 * u + i];
              ss = fmaf(hv, hv, ss);
            }
          }
        }
        inv = sqrtf(static_cast<float>(p.c_out)) / fmaxf(sqrtf(ss), 1e-12f);
      }
      // pass 2: bias (+ residual | RMS scale + SiLU) -> bf16 -> global
      for (int j0 = 0; j0 < p.nt; j0 += 48) {
        const int nld = (p.nt - j0) >= 48 ? 3 : (p.nt - j0) / 16;
        uint4 res[6];
        if (p.epi == 1 && valid) {
          // residual loads first, so their latency overlaps the TMEM reads
#pragma unroll
          for (int u = 0; u < 3; ++u)
            if (u < nld) {
              const uint4 *rr = reinterpret_cast<const uint4 *>(rrow + j0 + 16 * u);
              res[2 * u] = rr[0];
              res[2 * u + 1] = rr[1];
            }
        }
        uint32_t raw[48];
        __syncwarp();
#pragma unroll
        for (int u = 0; u < 3; ++u)
          if (u < nld) tmem_ld16_nowait(taddr + j0 + 16 * u, raw + 16 * u);
        tmem_wait_ld();
        tmem_regs_after_wait<48>(raw);
        if (j0 + 48 >= p.nt) {
          // last read of this accumulator: hand the buffer back to the MMA warp
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc_empty[buf]);
        }
#pragma unroll
        for (int u = 0; u < 3; ++u) {
          if (u >= nld) continue;
          const int j = j0 + 16 * u;
          float v[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(raw[16 * u + i]) + p.bias[n0 + j + i];
          if (p.epi == 1 && valid) {
            const __nv_bfloat16 *rb0 = reinterpret_cast<const __nv_bfloat16 *>(&res[2 * u]);
            const __nv_bfloat16 *rb1 = reinterpret_cast<const __nv_bfloat16 *>(&res[2 * u + 1]);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              v[i] += __bfloat162float(rb0[i]);
              v[8 + i] += __bfloat162float(rb1[i]);
            }
          } else if (p.epi == 2) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              float a = v[i] * inv * p.gamma[n0 + j + i];
              if (p.beta) a += p.beta[n0 + j + i];
              v[i] = silu_fast(a);
            }
          }
          if (valid) {
            uint4 o0, o1;
            o0.x = pack_bf16x2(v[0], v[1]);
            o0.y = pack_bf16x2(v[2], v[3]);
            o0.z = pack_bf16x2(v[4], v[5]);
            o0.w = pack_bf16x2(v[6], v[7]);
            o1.x = pack_bf16x2(v[8], v[9]);
            o1.y = pack_bf16x2(v[10], v[11]);
            o1.z = pack_bf16x2(v[12], v[13]);
            o1.w = pack_bf16x2(v[14], v[15]);
            uint4 *dst = reinterpret_cast<uint4 *>(yrow + j);
            dst[0] = o0;
            dst[1] = o1;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, p.tmem_cols);
  }
}

}  // namespace

size_t umma_smem_bytes(int kc, int nt, int kh, int kw, int na, int nb) {
  return make_layout(kc, nt, kh, kw, na, nb).total + 1024;  // + alignment slack
}

int umma_tile_w() { return kTW; }
int umma_tile_h() { return kTH; }

template <int KC, int KS>
cudaError_t set_smem_attr() {
  return cudaFuncSetAttribute(conv_umma_kernel<KC, KS>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
}

cudaError_t umma_prepare() {
  // Opt in to the largest dynamic shared memory window once per process.
  cudaError_t e = set_smem_attr<64, 3>();
  if (e == cudaSuccess) e = set_smem_attr<32, 3>();
  if (e == cudaSuccess) e = set_smem_attr<96, 3>();
  if (e == cudaSuccess) e = set_smem_attr<64, 1>();
  if (e == cudaSuccess) e = set_smem_attr<32, 1>();
  if (e == cudaSuccess) e = set_smem_attr<96, 1>();
  return e;
}

size_t umma_launch_smem(int kc, int nt, int ks, int na, int nb, int tmem_cols) {
  size_t smem = umma_smem_bytes(kc, nt, ks, ks, na, nb);
  // A CTA that holds more than half of tensor memory must have its SM to
  // itself; asking for more than half the shared memory guarantees that.
  if (tmem_cols > 256 && smem < 116 * 1024) smem = 116 * 1024;
  return smem;
}

cudaError_t launch_conv_umma(const CUtensorMap &map_x, const CUtensorMap &map_cache,
                             const UmmaArgs &args, int kc, unsigned grid, cudaStream_t stream) {
  if (args.kh != args.kw || (args.kh != 1 && args.kh != 3)) return cudaErrorInvalidValue;
  const size_t smem = umma_launch_smem(kc, args.nt, args.kh, args.na, args.nb, args.tmem_cols);
  if (smem > 227 * 1024) return cudaErrorInvalidValue;
#define CC3D_LAUNCH(KC_, KS_)                                                              \
  if (kc == KC_ && args.kh == KS_) {                                                       \
    conv_umma_kernel<KC_, KS_><<<grid, kThreads, smem, stream>>>(map_x, map_cache, args); \
    return cudaGetLastError();                                                             \
  }
  CC3D_LAUNCH(64, 3)
  CC3D_LAUNCH(32, 3)
  CC3D_LAUNCH(96, 3)
  CC3D_LAUNCH(64, 1)
  CC3D_LAUNCH(32, 1)
  CC3D_LAUNCH(96, 1)
#undef CC3D_LAUNCH
  return cudaErrorInvalidValue;
}

}  // namespace cc3d
