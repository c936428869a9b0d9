// conv_umma.cu -- bf16 implicit-GEMM causal Conv3D on tcgen05 tensor cores.
//
// Operation ("Cosmos3 Wan VAE -- engine size vs context memory", §10.3
// WanCausalConv3d and its implicit-GEMM view): M = output voxels,
// N = C_out, K = C_in * kt * kh * kw; every tap is summed into one fp32
// accumulator held in tensor memory; bias is added once in the epilogue
// ("cache-aware video decoder lowering" summary: bias after the sum).
//
// Tiling.  An MMA tile is TW = 8 columns x TH = 16 rows of one frame
// (M = 128 rows of the GEMM, row m = 8 * r + c) by NT output channels.  A
// CTA tile is SUB = 1 or 2 such MMA tiles side by side (8 or 16 columns);
// with two, every weight stage feeds two MMAs.  The kernel is persistent:
// one CTA per SM walks the tiles round-robin.  The K loop of a tile runs
// over (kt, channel chunk of KC, kh, kw).
//
// A operand: for each (kt, channel chunk) the input halo of the tile --
// (TH + kh - 1) x (SUB * TW + kw - 1) pixels x KC channels -- arrives by TMA
// from the current chunk x (frame tau = t + kt - (kt_size - 1) >= 0) or the
// frame cache (tau < 0), as no-swizzle core matrices,
//     [KC/8 slabs][halo rows][halo cols][8 channels],
// one 8-channel box per slab.  Spatial padding is TMA out-of-bounds zero
// fill, and a frame before the chunk with no cache (all zeros) is skipped:
// its stage is neither loaded nor multiplied.  No padded copy exists.  The
// A matrix of spatial tap (kh, kw) and of sub-tile s is the same buffer seen
// from a start address shifted by (kh * halo_cols + kw + 8 s) pixels of 16
// bytes, so one load serves every tap.
//
// B operand: the weights, re-tiled at plan time into the exact shared
// memory image of each (N tile, tap, channel chunk) stage
//     [KC/8][NT][8 channels]   (K-major core matrices),
// fetched with one 1-D bulk copy per stage.
//
// Temporal split.  When a frame has too few tiles to occupy the GPU, the
// kernel runs as clusters of kt CTAs that all take the same tile: CTA r
// multiplies temporal tap r only.  The senders (r < kt - 1) write their fp32
// partial sums, 16 accumulator columns at a time, straight into receive
// slots in the last CTA's shared memory (st.async, counted as transaction
// bytes on its mbarrier); the last CTA adds them to its own accumulator in
// a fixed order and runs the epilogue on the sums.
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
// Temporal split: the kXC-column chunks of a tile's accumulator meet in one
// CTA of the cluster (the owner, the last rank); the other CTAs send their
// partial sums of each chunk there, and the owner adds them and runs the
// epilogue for those columns.  Each epilogue warp of each CTA has
// kXSlots receive slots, each holding one kXC-column piece (32 lanes x kXC
// fp32 = kXPieceBytes) per sending rank.
constexpr int kXC = 16;
constexpr int kXSlots = 2;
constexpr uint32_t kXPieceBytes = 32u * kXC * 4u;
// x_ready[warp][slot] and x_free[warp][owner rank][slot]
__host__ __device__ constexpr int x_bar_count(int split) {
  return kEpiWarps * kXSlots * (1 + split);
}
__host__ __device__ constexpr uint32_t x_bytes(int split) {
  return split > 1 ? kEpiWarps * kXSlots * static_cast<uint32_t>(split - 1) * kXPieceBytes : 0u;
}

struct SmemLayout {
  uint32_t a_off, a_stage, slab, b_off, b_stage, x_off, bar_off, p_off, total;
  int na, nb;
};

// Epilogue parameters staged in shared memory: bias[c_out] (and, for the
// RMS epilogue, gamma[c_out], beta[c_out]).
__host__ __device__ constexpr int param_floats(int c_out, int epi) {
  return c_out * (epi == 2 ? 3 : 1);
}

__host__ __device__ inline uint32_t round_up(uint32_t v, uint32_t a) { return (v + a - 1) / a * a; }

// 64-channel chunks stage the A halo with the 128-byte swizzle: one TMA box
// of 128-byte pixel rows, its columns padded to a multiple of 8 so that an
// image row of the halo spans whole 1024-byte swizzle atoms.  Other chunk
// widths use 8-channel no-swizzle slabs (16-byte rows, 8 boxes for 64
// channels: many more TMA requests per stage).
__host__ __device__ constexpr bool uses_sw128(int kc) { return kc == 64; }
__host__ __device__ inline int halo_cols(int kc, int sub, int kw) {
  const int hw = kTW * sub + kw - 1;
  return uses_sw128(kc) ? (hw + 7) / 8 * 8 : hw;
}

__host__ __device__ inline SmemLayout make_layout(int kc, int nt, int kh, int kw, int na, int nb,
                                                  int sub, int split, bool pair, int params) {
  SmemLayout L;
  const uint32_t hh = kTH + kh - 1, hw = static_cast<uint32_t>(halo_cols(kc, sub, kw));
  if (uses_sw128(kc)) {
    L.slab = hh * hw * 128u;  // the whole halo; a multiple of 1024
    L.a_stage = L.slab;
  } else {
    L.slab = round_up(hh * hw * 16u, 128u);
    L.a_stage = (kc / 8) * L.slab;
  }
  // (a CTA pair: this CTA's half of the N rows, 128-byte swizzled rows)
  L.b_stage = static_cast<uint32_t>(pair ? nt / 2 : nt) * kc * 2u;
  L.na = na;
  L.nb = nb;
  L.a_off = 0;
  L.b_off = round_up(L.a_off + na * L.a_stage, 1024u);
  L.x_off = round_up(L.b_off + nb * L.b_stage, 128u);
  L.bar_off = round_up(L.x_off + x_bytes(split), 64u);
  // full_a, empty_a, full_b, empty_b, acc_full[2], acc_empty[2], drain,
  // (split: x_ready[4][2], x_free[4][2]), tmem slot
  L.p_off = round_up(
      L.bar_off + 8u * (2 * na + 2 * nb + 5 + (split > 1 ? x_bar_count(split) : 0)) + 16u, 16u);
  L.total = L.p_off + 4u * static_cast<uint32_t>(params);
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
  c.w0 = tw * kTW * p.sub;
  c.h0 = th * kTH;
  return c;
}

// 16 consecutive fp32 parameters (bias / gamma / beta, staged in shared
// memory at the 16-byte-aligned address `src`) as four 16-byte loads; every
// lane of a warp reads the same address (a broadcast).  Volatile, so that
// the compiler issues them where they are used instead of hoisting every
// group's parameters into registers at once.
__device__ __forceinline__ void ld_param16(uint32_t src, float (&v)[16]) {
#pragma unroll
  for (int u = 0; u < 4; ++u)
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v[4 * u]), "=f"(v[4 * u + 1]), "=f"(v[4 * u + 2]), "=f"(v[4 * u + 3])
                 : "r"(src + 16u * u));
}

// 16 bf16 values (two 16-byte halves) to global memory: one 256-bit store
// when the destination is 32-byte aligned, else two 128-bit stores.
__device__ __forceinline__ void store_bf16x16(__nv_bfloat16 *dst, const uint4 &lo, const uint4 &hi,
                                              int vec32) {
  if (vec32) {
    st_global_v8(dst, lo, hi);
  } else {
    uint4 *d = reinterpret_cast<uint4 *>(dst);
    d[0] = lo;
    d[1] = hi;
  }
}

template <int KC, int KS, int SUB, bool PAIR>
__global__ void __launch_bounds__(kThreads, 1)
    conv_umma_kernel(const __grid_constant__ CUtensorMap map_x,
                     const __grid_constant__ CUtensorMap map_cache,
                     const __grid_constant__ CUtensorMap map_w,
                     const __grid_constant__ CUtensorMap map_sc, UmmaArgs p) {
  static_assert(!PAIR || (SUB == 1 && uses_sw128(KC)), "CTA pairs take 64-channel chunks");
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // Align the dynamic shared window to 1 KiB ourselves (the attribute is a
  // request, not a guarantee).
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const SmemLayout L =
      make_layout(KC, p.nt, KS, KS, p.na, p.nb, SUB, p.split, PAIR, param_floats(p.c_out, p.epi));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L.bar_off);
  uint64_t *full_a = bars;
  uint64_t *empty_a = full_a + L.na;
  uint64_t *full_b = empty_a + L.na;
  uint64_t *empty_b = full_b + L.nb;
  uint64_t *acc_full = empty_b + L.nb;   // [2]
  uint64_t *acc_empty = acc_full + 2;    // [2]
  uint64_t *drain = acc_empty + 2;       // MMA completion before TMEM is freed
  const bool split = p.split > 1;
  // split: x_ready[q][slot] (as owner: its own arrival, one arrival per
  // other rank, and the bytes they store) and x_free[q][o][slot] (as sender
  // to owner rank o: one arrival from o once it has read the slot)
  uint64_t *x_ready = drain + 1;
  uint64_t *x_free = x_ready + (split ? kEpiWarps * kXSlots : 0);
  uint32_t *tmem_slot =
      reinterpret_cast<uint32_t *>(x_ready + (split ? x_bar_count(p.split) : 0));

  // Cluster geometry.  Without a split every CTA is its own cluster.  With
  // one, the CTAs of a cluster walk the same tiles; CTA `rank` multiplies
  // temporal tap kt = rank only, and the partial results meet chunk by chunk
  // in the chunk's owner, which adds them in a fixed order (tap kt-1 -- the
  // current frame, never a causal zero frame -- then kt-2 .. 0) and runs the
  // epilogue for those columns.
  //
  // With PAIR, a cluster of two CTAs (on one SM pair) takes a 16 x 16 pixel
  // tile: CTA `rank` holds the 8 x 16 half at columns 8 * rank and half of
  // each weight stage's N rows, and the leader (rank 0) issues M = 256
  // tcgen05 MMAs over both CTAs' shared memory into both CTAs' tensor memory.
  const int csize = PAIR ? 2 : p.split;
  const int rank = (split || PAIR) ? static_cast<int>(cluster_ctarank()) : 0;
  const int cid = static_cast<int>(blockIdx.x) / csize;
  const int ncl = static_cast<int>(gridDim.x) / csize;
  const bool pair_leader = !PAIR || rank == 0;
  const int kt_lo = split ? rank : 0;
  const int n_kt = split ? 1 : p.kt;

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  const int n_cc = p.c_in / KC;   // channel chunks
  const int n_a = n_kt * n_cc;    // A stages per tile (of this CTA)
  // weight stages of the conv per N tile, and the shortcut's chunks after them
  const int n_conv_stages = p.kt * KS * KS * n_cc;
  const int n_sc = (p.c_sc > 0 && !split) ? p.n_cc_sc : 0;
  const int stages_per_ntile = n_conv_stages + (p.c_sc > 0 ? p.n_cc_sc : 0);  // weight image
  constexpr bool kSw = uses_sw128(KC);
  const uint32_t halo_w = static_cast<uint32_t>(halo_cols(KC, SUB, KS));
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
      mbar_init(&acc_empty[i], PAIR ? 2 * kEpiWarps : kEpiWarps);  // (pair: both CTAs)
    }
    mbar_init(drain, 1);
    if (split) {
      for (int i = 0; i < kEpiWarps * kXSlots; ++i) mbar_init(&x_ready[i], p.split);
      for (int i = 0; i < kEpiWarps * p.split * kXSlots; ++i) mbar_init(&x_free[i], 1);
    }
    fence_mbar_init();
    prefetch_tmap(&map_x);
    if (p.has_cache) prefetch_tmap(&map_cache);
    if (PAIR) prefetch_tmap(&map_w);
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      tmem_alloc_pair(tmem_slot, p.tmem_cols);  // same columns in both CTAs
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, p.tmem_cols);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  // (in a cluster, no CTA may arrive on a peer's barriers before the peer
  // has initialised them)
  if (split || PAIR)
    cluster_sync();
  else
    __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t smem_base = smem_u32(smem);
  bool ok = true;

  if (warp == 0) {
    // ------------------------------ producer ------------------------------------
    if (lane == 0) {
      const uint32_t a_tx = kSw ? L.a_stage : (KC / 8) * (16u * halo_w * (kTH + KS - 1));
      // PAIR: both CTAs' loads complete on the leader's full barriers, which
      // the leader arms for the bytes of both halves
      const uint32_t lead_full_a = PAIR ? mapa_shared(smem_u32(full_a), 0u) : 0u;
      const uint32_t lead_full_b = PAIR ? mapa_shared(smem_u32(full_b), 0u) : 0u;
      int sa = 0, sb = 0;
      uint32_t pa = 0, pb = 0;
      // stages issued at least once, and the phase parity of their last issue
      uint32_t a_used = 0, a_par = 0, b_used = 0, b_par = 0;
      // weight stage `stage_idx` (tap-major, then channel chunk) of N tile
      // `ntile` into B slot `slot`: the whole stage, or this CTA's half of
      // its N rows on a pair
      auto load_b = [&](int slot, size_t stage_idx, int ntile) {
        if (pair_leader)
          mbar_arrive_expect_tx(&full_b[slot], PAIR ? 2u * L.b_stage : L.b_stage);
        if constexpr (PAIR) {
          // rows of the weight image [ntile][tap][cchunk][NT][64]
          const int row = static_cast<int>(
              ((static_cast<size_t>(ntile) * stages_per_ntile + stage_idx) * p.nt) +
              rank * (p.nt / 2));
          tma_load_2d_pair(smem_base + L.b_off + slot * L.b_stage, &map_w,
                           lead_full_b + 8u * slot, 0, row);
        } else {
          const uint8_t *wsrc =
              p.wimg + static_cast<size_t>(ntile) * stages_per_ntile * L.b_stage;
          bulk_load(smem_base + L.b_off + slot * L.b_stage, wsrc + stage_idx * L.b_stage,
                    L.b_stage, &full_b[slot]);
        }
      };
      // channels c0 .. c0+KC-1 of the box of `map` that starts at column
      // wc, row hc of frame `tcoord` of image `n`, into A slot `slot`
      auto load_a_at = [&](const CUtensorMap *map, int slot, int c0, int wc, int hc, int tcoord,
                           int n) {
        const uint32_t dst = smem_base + L.a_off + slot * L.a_stage;
        if constexpr (PAIR) {
          tma_load_5d_pair(dst, map, lead_full_a + 8u * slot, c0, wc, hc, tcoord, n);
        } else if constexpr (kSw) {
          tma_load_5d(dst, map, &full_a[slot], c0, wc, hc, tcoord, n);
        } else {
#pragma unroll
          for (int s = 0; s < KC / 8; ++s)
            tma_load_5d(dst + s * L.slab, map, &full_a[slot], c0 + s * 8, wc, hc, tcoord, n);
        }
      };
      // the tile's halo of channels c0 .. c0+KC-1 of frame `tcoord` of `map`
      // into A slot `slot` (this CTA's half of the tile on a pair)
      auto load_a = [&](const CUtensorMap *map, int slot, int c0, int tcoord,
                        const TileCoord &tc) {
        // (only a pair's CTAs hold different columns: a temporal split's
        // CTAs all load the whole tile)
        load_a_at(map, slot, c0, tc.w0 + (PAIR ? kTW * rank : 0) - KS / 2, tc.h0 - KS / 2, tcoord,
                  tc.n);
      };
      if (KS == 1 && p.b_resident) {
        // one N tile and every weight stage in a slot of its own: loaded
        // once here, read in place by the MMAs of every tile
        for (int st = 0; st < L.nb; ++st) load_b(st, static_cast<size_t>(st), 0);
        b_used = L.nb >= 32 ? 0xffffffffu : (1u << L.nb) - 1u;
      }
      for (int tile = cid; tile < n_tiles && ok; tile += ncl) {
        const TileCoord tc0 = decode_tile(tile, p);
        for (int ia = 0; ia < n_a && ok; ++ia) {
          const int kt = kt_lo + ia / n_cc, cc = ia % n_cc;
          // A frame before the chunk with no cache is all zeros: its stage
          // (and its taps' weights) is skipped here and by the MMA issuer.
          if (!(KS == 1 && p.s2) && p.stride_t * tc0.t + kt - (p.kt - 1) < 0 && !p.has_cache)
            continue;
          if (!mbar_wait_bounded(&empty_a[sa], pa ^ 1, p.wait_limit_ns, p.status, 1)) {
            ok = false;
            break;
          }
          if (pair_leader) mbar_arrive_expect_tx(&full_a[sa], PAIR ? 2u * a_tx : a_tx);
          a_used |= 1u << sa;
          a_par = (a_par & ~(1u << sa)) | (pa << sa);
          if (KS == 1 && p.s2) {
            // stride 2 in H and W: stage `kt` is spatial tap (kh, kw) =
            // (kt / 3, kt % 3); the map walks every other pixel, so the box
            // of output pixel (h, w) starts at input (2h + kh, 2w + kw)
            load_a_at(&map_x, sa, cc * KC, 2 * (tc0.w0 + (PAIR ? kTW * rank : 0)) + kt % 3 - p.pad_w,
                      2 * tc0.h0 + kt / 3 - p.pad_h, tc0.t, tc0.n);
          } else {
            const int tau = p.stride_t * tc0.t + kt - (p.kt - 1);  // input frame
            const bool from_cache = tau < 0;  // (zero frames were skipped above)
            load_a(from_cache ? &map_cache : &map_x, sa, cc * KC,
                   from_cache ? tau + (p.kt - 1) : tau, tc0);
          }
          if (++sa == L.na) { sa = 0; pa ^= 1; }
          if (KS == 1 && p.b_resident) continue;
#pragma unroll 1
          for (int ts = 0; ts < KS * KS; ++ts) {
            if (!mbar_wait_bounded(&empty_b[sb], pb ^ 1, p.wait_limit_ns, p.status, 2)) {
              ok = false;
              break;
            }
            b_used |= 1u << sb;
            b_par = (b_par & ~(1u << sb)) | (pb << sb);
            load_b(sb, static_cast<size_t>(kt * KS * KS + ts) * n_cc + cc, tc0.ntile);
            if (++sb == L.nb) { sb = 0; pb ^= 1; }
          }
        }
        // the residual block's 1x1x1 conv_shortcut: each channel chunk of
        // the block input at the output frame (a halo like the conv's, read
        // at its centre tap) against one weight stage stored after the
        // conv's, into the same accumulator
        for (int c2 = 0; c2 < n_sc && ok; ++c2) {
          if (!mbar_wait_bounded(&empty_a[sa], pa ^ 1, p.wait_limit_ns, p.status, 1)) {
            ok = false;
            break;
          }
          if (pair_leader) mbar_arrive_expect_tx(&full_a[sa], PAIR ? 2u * a_tx : a_tx);
          a_used |= 1u << sa;
          a_par = (a_par & ~(1u << sa)) | (pa << sa);
          load_a(&map_sc, sa, c2 * KC, tc0.t, tc0);
          if (++sa == L.na) { sa = 0; pa ^= 1; }
          if (!mbar_wait_bounded(&empty_b[sb], pb ^ 1, p.wait_limit_ns, p.status, 2)) {
            ok = false;
            break;
          }
          b_used |= 1u << sb;
          b_par = (b_par & ~(1u << sb)) | (pb << sb);
          load_b(sb, static_cast<size_t>(n_conv_stages + c2), tc0.ntile);
          if (++sb == L.nb) { sb = 0; pb ^= 1; }
        }
      }
      // Drain: every load this thread issued lands before the CTA may exit
      // (after a timeout elsewhere the consumer may not have waited for it).
      // A pair's leader drains for both CTAs: their loads complete on its
      // barriers, and the follower waits at the final cluster barrier.
      if (!pair_leader) a_used = b_used = 0;
      for (int i = 0; i < L.na; ++i)
        if (a_used >> i & 1u)
          mbar_wait_bounded(&full_a[i], a_par >> i & 1u, kDrainLimitNs, nullptr, 0);
      for (int i = 0; i < L.nb; ++i)
        if (b_used >> i & 1u)
          mbar_wait_bounded(&full_b[i], b_par >> i & 1u, kDrainLimitNs, nullptr, 0);
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer ----------------------------------
    // (a pair's follower issues nothing: the leader's MMAs cover both CTAs)
    if (lane == 0 && pair_leader) {
      const uint32_t idesc = idesc_bf16_f32(PAIR ? 2 * kM : kM, p.nt);
      const uint32_t b_lbo = static_cast<uint32_t>(p.nt) * 16u;
      // Descriptors of stage 0; other stages, taps, sub-tiles and K steps
      // only move the start address (low 14 bits, 16-byte units), so they
      // are additions.  A halo pixel is 128 bytes (swizzled) or 16 bytes (an
      // 8-channel slab); a 16-element K step is 32 bytes along the swizzled
      // row, or two slabs / two B core-matrix columns further on.
      const uint64_t adesc0 =
          kSw ? smem_desc_sw128(smem_base + L.a_off, halo_w * 128u)
              : smem_desc_noswizzle(smem_base + L.a_off, L.slab, halo_w * 16u);
      // B: [NT][KC/8][8] no-swizzle core matrices, or (pair) this CTA's
      // NT/2 rows of 128 swizzled bytes
      const uint64_t bdesc0 = PAIR ? smem_desc_sw128(smem_base + L.b_off, 1024u)
                                   : smem_desc_noswizzle(smem_base + L.b_off, b_lbo, 128u);
      const uint32_t astep16 = kSw ? 2u : 2u * (L.slab >> 4);
      const uint32_t bstep16 = PAIR ? 2u : 2u * (b_lbo >> 4);
      const uint32_t pix16 = kSw ? 8u : 1u;
      int sa = 0, sb = 0;
      uint32_t pa = 0, pb = 0;
      int it = 0;
      for (int tile = cid; tile < n_tiles && ok; tile += ncl, ++it) {
        const int buf = it % p.nbuf;
        const uint32_t use_par = static_cast<uint32_t>((it / p.nbuf) & 1);
        // wait until the epilogue (of both CTAs of a pair) has drained this
        // accumulator buffer
        if (!(PAIR ? mbar_wait_bounded_cluster(&acc_empty[buf], use_par ^ 1, p.wait_limit_ns,
                                               p.status, 6)
                   : mbar_wait_bounded(&acc_empty[buf], use_par ^ 1, p.wait_limit_ns, p.status,
                                       6))) {
          ok = false;
          break;
        }
        tc_fence_after();
        // sub-tile s of this buffer accumulates at columns (buf * SUB + s) * nt
        const uint32_t d_tmem = tmem_base + buf * SUB * p.nt;
        const TileCoord tcm = decode_tile(tile, p);
        uint32_t accumulate = 0;
        // the MMAs of weight slot `slot` (phase parity `par`) against the
        // halo at `a_st` seen through spatial tap `ts`
        auto issue_b = [&](uint64_t a_st, int slot, uint32_t par, int ts) -> bool {
          if (!mbar_wait_bounded(&full_b[slot], par, p.wait_limit_ns, p.status, 4)) return false;
          tc_fence_after();
          const uint64_t a_tap = a_st + ((ts / KS) * halo_w + (ts % KS)) * pix16;
          const uint64_t b_st = bdesc0 + ((static_cast<uint32_t>(slot) * L.b_stage) >> 4);
#pragma unroll
          for (int j = 0; j < KC / 16; ++j) {
            // every sub-tile (8 pixels further along the halo row) reuses
            // this weight stage
#pragma unroll
            for (int sbt = 0; sbt < SUB; ++sbt) {
              if constexpr (PAIR)
                umma_bf16_pair(d_tmem, a_tap + j * astep16, b_st + j * bstep16, idesc,
                               accumulate);
              else
                umma_bf16(d_tmem + sbt * p.nt, a_tap + sbt * kTW * pix16 + j * astep16,
                          b_st + j * bstep16, idesc, accumulate);
            }
            accumulate = 1;
          }
          return true;
        };
        for (int ia = 0; ia < n_a && ok; ++ia) {
          // the same zero-frame stages the producer skipped; adding their
          // exact zeros would not change the accumulator
          if (!(KS == 1 && p.s2) && p.stride_t * tcm.t + kt_lo + ia / n_cc - (p.kt - 1) < 0 &&
              !p.has_cache)
            continue;
          if (!mbar_wait_bounded(&full_a[sa], pa, p.wait_limit_ns, p.status, 3)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t a_st = adesc0 + ((sa * L.a_stage) >> 4);
          if (KS == 1 && p.b_resident) {
            // resident weights: stage (kt, cc) sits in slot kt * n_cc + cc,
            // loaded once (its first phase stays complete) and never freed
            if (!issue_b(a_st, kt_lo * n_cc + ia, 0u, 0)) {
              ok = false;
              break;
            }
          } else {
#pragma unroll
            for (int ts = 0; ts < KS * KS; ++ts) {
              if (!issue_b(a_st, sb, pb, ts)) {
                ok = false;
                break;
              }
              // frees the B stage (in both CTAs of a pair) when these MMAs finish
              if constexpr (PAIR) umma_commit_pair(&empty_b[sb], 3);
              else umma_commit(&empty_b[sb]);
              if (++sb == L.nb) { sb = 0; pb ^= 1; }
            }
          }
          if constexpr (PAIR) umma_commit_pair(&empty_a[sa], 3);
          else umma_commit(&empty_a[sa]);
          if (++sa == L.na) { sa = 0; pa ^= 1; }
        }
        // the conv_shortcut's chunks: the centre tap of each halo
        for (int c2 = 0; c2 < n_sc && ok; ++c2) {
          if (!mbar_wait_bounded(&full_a[sa], pa, p.wait_limit_ns, p.status, 3)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (!issue_b(adesc0 + ((sa * L.a_stage) >> 4), sb, pb, (KS / 2) * KS + KS / 2)) {
            ok = false;
            break;
          }
          if constexpr (PAIR) {
            umma_commit_pair(&empty_b[sb], 3);
            umma_commit_pair(&empty_a[sa], 3);
          } else {
            umma_commit(&empty_b[sb]);
            umma_commit(&empty_a[sa]);
          }
          if (++sb == L.nb) { sb = 0; pb ^= 1; }
          if (++sa == L.na) { sa = 0; pa ^= 1; }
        }
        // accumulator ready for the epilogue(s)
        if constexpr (PAIR) umma_commit_pair(&acc_full[buf], 3);
        else umma_commit(&acc_full[buf]);
      }
      // Drain: all MMAs issued here are complete before tensor memory is freed.
      if constexpr (PAIR) umma_commit_pair(drain, 1);
      else umma_commit(drain);
      mbar_wait_bounded(drain, 0, kDrainLimitNs, nullptr, 0);
    }
  } else {
    // ------------------------------ epilogue ------------------------------------
    const int q = warp % 4;  // tensor-memory lane quarter this warp may read
    const int m = q * 32 + lane;
    const int r = m / kTW, c = m % kTW;
    int it = 0;
    // split: chunks of each owner rank exchanged by this warp so far
    uint32_t xc0 = 0, xc1 = 0, xc2 = 0, xc3 = 0;
    // this warp's receive slots: [slot][sending rank index][quad of 4
    // columns][lane][4 fp32]; x_lane(slot, sender) is this lane's quad 0
    const int n_send = p.split - 1;
    // bias (and gamma, beta) of every output channel, staged once: the
    // per-column reads below are then shared-memory broadcasts
    float *sp = reinterpret_cast<float *>(smem + L.p_off);
    for (int i = static_cast<int>(threadIdx.x) - 64; i < p.c_out; i += 32 * kEpiWarps) {
      sp[i] = p.bias[i];
      if (p.epi == 2) {
        sp[p.c_out + i] = p.gamma[i];
        sp[2 * p.c_out + i] = p.beta ? p.beta[i] : 0.f;
      }
    }
    named_barrier_sync(1, 32 * kEpiWarps);  // (the epilogue warps only)
    // (shared addresses of the three vectors)
    const uint32_t s_bias = smem_u32(sp), s_gamma = s_bias + 4u * static_cast<uint32_t>(p.c_out),
                   s_beta = s_gamma + 4u * static_cast<uint32_t>(p.c_out);
    auto x_lane = [&](uint32_t slot, int sender) -> uint32_t {
      return smem_base + L.x_off +
             ((static_cast<uint32_t>(q) * kXSlots + slot) * static_cast<uint32_t>(n_send) +
              static_cast<uint32_t>(sender)) * kXPieceBytes +
             static_cast<uint32_t>(lane) * 16u;
    };
    for (int tile = cid; tile < n_tiles; tile += ncl, ++it) {
      const int buf = it % p.nbuf;
      const uint32_t use_par = static_cast<uint32_t>((it / p.nbuf) & 1);
      const TileCoord tc0 = decode_tile(tile, p);
      uint32_t got = 0;
      if (lane == 0)
        got = mbar_wait_bounded(&acc_full[buf], use_par, p.wait_limit_ns, p.status, 5) ? 1u : 0u;
      got = __shfl_sync(0xffffffffu, got, 0);
      if (!got) break;
      tc_fence_after();
      if (split) {
        // ---- the partial sums of the cluster meet in the owner CTA ----
        uint32_t live = 0;  // ranks whose tap is not a causal zero frame
        for (int rr = 0; rr < p.split; ++rr)
          if (p.has_cache || p.stride_t * tc0.t + rr - (p.kt - 1) >= 0) live |= 1u << rr;
        const bool own_live = (live >> rank) & 1u;
        const int n0 = tc0.ntile * p.nt;
        const int chunks_per_sub = p.nt / kXC;
        bool xok = true;
        for (int sbt = 0; sbt < SUB && xok; ++sbt) {
          const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                 static_cast<uint32_t>((buf * SUB + sbt) * p.nt);
          const int h = tc0.h0 + r, w = tc0.w0 + sbt * kTW + c;
          const bool valid = (h < p.h) && (w < p.w);
          const size_t pix = ((static_cast<size_t>(tc0.n) * p.t + tc0.t) * p.h + h) * p.w + w;
          for (int jc = 0; jc < chunks_per_sub; ++jc) {
            const int j0 = jc * kXC;
            // the last CTA (tap kt-1, the current frame) owns every chunk:
            // the senders then run ahead of it by the receive slots
            const int owner = p.split - 1;
            uint32_t k;  // (counters in registers: no indexed local array)
            if (owner == 0) k = xc0++;
            else if (owner == 1) k = xc1++;
            else if (owner == 2) k = xc2++;
            else k = xc3++;
            const uint32_t slot = k % kXSlots, ph = (k / kXSlots) & 1u;
            uint32_t raw[kXC];
            if (owner != rank) {
              // sender: this chunk's partial goes to its owner's slot
              if (own_live) {
                __syncwarp();
                tmem_ld16_nowait(taddr + j0, raw);
                tmem_wait_ld();
                tmem_regs_after_wait<kXC>(raw);
              }
              uint32_t free_ok = 0;
              if (lane == 0)
                free_ok = mbar_wait_bounded_cluster(&x_free[(q * p.split + owner) * kXSlots + slot],
                                                    ph ^ 1u, p.wait_limit_ns, p.status, 7)
                              ? 1u
                              : 0u;
              free_ok = __shfl_sync(0xffffffffu, free_ok, 0);
              if (!free_ok) {
                xok = false;
                break;
              }
              const uint32_t bar =
                  mapa_shared(smem_u32(&x_ready[q * kXSlots + slot]), static_cast<uint32_t>(owner));
              if (own_live) {
                const int sidx = rank < owner ? rank : rank - 1;
                const uint32_t dst = mapa_shared(x_lane(slot, sidx), static_cast<uint32_t>(owner));
#pragma unroll
                for (int u = 0; u < kXC / 4; ++u) st_async_v4(dst + u * 512u, raw + 4 * u, bar);
              }
              // every rank arrives once per chunk, live or not, so that no
              // rank's barrier phases run ahead of another's
              __syncwarp();
              if (lane == 0) mbar_arrive_remote_relaxed(bar);
              continue;
            }
            // owner: add the partials in a fixed order, then the epilogue
            uint4 res[2];
            if (p.epi == 1 && valid) {
              const uint4 *rr = reinterpret_cast<const uint4 *>(p.residual + pix * p.c_out + n0 + j0);
              res[0] = rr[0];
              res[1] = rr[1];
            }
            if (own_live) {
              __syncwarp();
              tmem_ld16_nowait(taddr + j0, raw);
            }
            uint32_t ready = 0;
            if (lane == 0) {
              mbar_arrive_expect_tx(&x_ready[q * kXSlots + slot],
                                    static_cast<uint32_t>(__popc(live & ~(1u << rank))) *
                                        kXPieceBytes);
              ready = mbar_wait_bounded_cluster(&x_ready[q * kXSlots + slot], ph, p.wait_limit_ns,
                                                p.status, 8)
                          ? 1u
                          : 0u;
            }
            ready = __shfl_sync(0xffffffffu, ready, 0);
            if (own_live) {
              tmem_wait_ld();
              tmem_regs_after_wait<kXC>(raw);
            }
            if (!ready) {
              xok = false;
              break;
            }
            float v[kXC];
            bool first = true;
            for (int src_rank = p.split - 1; src_rank >= 0; --src_rank) {
              if (!((live >> src_rank) & 1u)) continue;  // no partial: a causal zero frame
              float t16[kXC];
              if (src_rank == rank) {
#pragma unroll
                for (int i = 0; i < kXC; ++i) t16[i] = __uint_as_float(raw[i]);
              } else {
                const uint32_t src = x_lane(slot, src_rank < rank ? src_rank : src_rank - 1);
#pragma unroll
                for (int u = 0; u < kXC / 4; ++u)
                  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                               : "=f"(t16[4 * u]), "=f"(t16[4 * u + 1]), "=f"(t16[4 * u + 2]),
                                 "=f"(t16[4 * u + 3])
                               : "r"(src + u * 512u)
                               : "memory");
              }
#pragma unroll
              for (int i = 0; i < kXC; ++i) v[i] = first ? t16[i] : v[i] + t16[i];
              first = false;
            }
            // the slot's values are in registers: the senders may refill it
            __syncwarp();
            if (lane == 0)
              for (int dst_rank = 0; dst_rank < p.split; ++dst_rank)
                if (dst_rank != rank)
                  mbar_arrive_remote_relaxed(
                      mapa_shared(smem_u32(&x_free[(q * p.split + rank) * kXSlots + slot]),
                                  static_cast<uint32_t>(dst_rank)));
            {
              float bv[16];
              ld_param16(s_bias + 4u * static_cast<uint32_t>(n0 + j0), bv);
#pragma unroll
              for (int i = 0; i < kXC; ++i) v[i] += bv[i];
            }
            if (p.epi == 1 && valid) {
              const __nv_bfloat16 *rb0 = reinterpret_cast<const __nv_bfloat16 *>(&res[0]);
              const __nv_bfloat16 *rb1 = reinterpret_cast<const __nv_bfloat16 *>(&res[1]);
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                v[i] += __bfloat162float(rb0[i]);
                v[8 + i] += __bfloat162float(rb1[i]);
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
              store_bf16x16(p.y + pix * p.c_out + n0 + j0, o0, o1, p.vec32);
            }
          }
        }
        // every tensor-memory read of this tile is done
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[buf]);
        if (!xok) break;
        continue;
      }
      for (int sbt = 0; sbt < SUB; ++sbt) {
        // (a pair's CTA holds the 8 columns at 8 * rank of the 16-wide tile)
        const int h = tc0.h0 + r, w = tc0.w0 + (PAIR ? rank : sbt) * kTW + c;
        const bool valid = (h < p.h) && (w < p.w);
        const bool last_sub = sbt == SUB - 1;
        const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                               static_cast<uint32_t>((buf * SUB + sbt) * p.nt);
        const int n0 = tc0.ntile * p.nt;
        const size_t pix = ((static_cast<size_t>(tc0.n) * p.t + tc0.t) * p.h + h) * p.w + w;
        __nv_bfloat16 *yrow = p.y + pix * p.c_out + n0;
        const __nv_bfloat16 *rrow = p.residual ? p.residual + pix * p.c_out + n0 : nullptr;
        float inv = 1.0f;
        if (p.epi == 2) {
          // pass 1: sum of squares of the biased row h1 (three loads in
          // flight).  h1 is a bf16 activation, as it is when conv1 writes it
          // out for a separate RMS_norm: it is rounded before it is used.
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
              float bv[16];
              ld_param16(s_bias + 4u * static_cast<uint32_t>(n0 + j0 + 16 * u), bv);
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const float hv = round_to_bf16(__uint_as_float(raw[16 * u + i]) + bv[i]);
                ss = fmaf(hv, hv, ss);
              }
            }
          }
          inv = sqrtf(static_cast<float>(p.c_out)) / fmaxf(sqrtf(ss), 1e-12f);
        }
        // pass 2: bias (+ residual | RMS scale + SiLU) -> bf16 -> global, in
        // groups of 32 columns; the next group's tensor-memory loads are in
        // flight while this group is converted and stored
        const int n_groups = (p.nt + 31) / 32;
        auto load_group = [&](int j0, uint32_t(&dst)[32]) {
          const int nld = (p.nt - j0) >= 32 ? 2 : 1;
          __syncwarp();
#pragma unroll
          for (int u = 0; u < 2; ++u)
            if (u < nld) tmem_ld16_nowait(taddr + j0 + 16 * u, dst + 16 * u);
        };
        uint32_t raw[32];
        load_group(0, raw);
        tmem_wait_ld();
        tmem_regs_after_wait<32>(raw);
        for (int g = 0; g < n_groups; ++g) {
          const int j0 = 32 * g;
          const int nld = (p.nt - j0) >= 32 ? 2 : 1;
          const bool more = g + 1 < n_groups;
          uint4 res[4];
          if (p.epi == 1 && valid) {
#pragma unroll
            for (int u = 0; u < 2; ++u)
              if (u < nld) {
                const uint4 *rr = reinterpret_cast<const uint4 *>(rrow + j0 + 16 * u);
                res[2 * u] = rr[0];
                res[2 * u + 1] = rr[1];
              }
          }
          uint32_t nxt[32];
          if (more) {
            load_group(j0 + 32, nxt);
          } else if (last_sub) {
            // every read of this accumulator buffer has completed: hand it
            // back to the MMA warp (a pair's follower: to the leader's)
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
              if (PAIR && rank != 0)
                mbar_arrive_remote(mapa_shared(smem_u32(&acc_empty[buf]), 0u));
              else
                mbar_arrive(&acc_empty[buf]);
            }
          }
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            if (u >= nld) continue;
            const int j = j0 + 16 * u;
            float v[16];
            {
              float bv[16];
              ld_param16(s_bias + 4u * static_cast<uint32_t>(n0 + j), bv);
#pragma unroll
              for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(raw[16 * u + i]) + bv[i];
            }
            if (p.epi == 1 && valid) {
              const __nv_bfloat16 *rb0 = reinterpret_cast<const __nv_bfloat16 *>(&res[2 * u]);
              const __nv_bfloat16 *rb1 = reinterpret_cast<const __nv_bfloat16 *>(&res[2 * u + 1]);
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                v[i] += __bfloat162float(rb0[i]);
                v[8 + i] += __bfloat162float(rb1[i]);
              }
            } else if (p.epi == 2) {
              float gv[16], be[16];
              ld_param16(s_gamma + 4u * static_cast<uint32_t>(n0 + j), gv);
              ld_param16(s_beta + 4u * static_cast<uint32_t>(n0 + j), be);
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                float a = round_to_bf16(v[i]) * inv * gv[i];
                a += be[i];
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
              store_bf16x16(yrow + j, o0, o1, p.vec32);
            }
          }
          if (more) {
            tmem_wait_ld();
            tmem_regs_after_wait<32>(nxt);
#pragma unroll
            for (int i = 0; i < 32; ++i) raw[i] = nxt[i];
          }
        }
      }  // sub-tiles
    }
  }

  tc_fence_before();
  __syncthreads();
  // no CTA leaves while a peer may still write its shared or tensor memory
  // or arrive on its barriers
  if (split || PAIR) cluster_sync();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    if constexpr (PAIR)
      tmem_dealloc_pair(tmem_base, p.tmem_cols);
    else
      tmem_dealloc(tmem_base, p.tmem_cols);
  }
}

}  // namespace

size_t umma_smem_bytes(int kc, int nt, int kh, int kw, int na, int nb, int sub, int split,
                       int pair, int params) {
  // (a pair's CTA holds one 8 x 16 MMA tile: sub counts tile widths)
  return make_layout(kc, nt, kh, kw, na, nb, pair ? 1 : sub, split, pair != 0, params).total +
         1024;  // + alignment slack
}

namespace {
// Buffers, pipeline depths and residency of one tile shape.
bool finish_config(int ks, int kt, int c_in, UmmaConfig &c) {
  const int cta_sub = c.pair ? 1 : c.sub;  // MMA tiles whose accumulators one CTA holds
  c.nbuf = (2 * cta_sub * c.nt <= 512) ? 2 : 1;  // double-buffered accumulators when they fit
  c.tmem_cols = 32;
  while (c.tmem_cols < c.nbuf * cta_sub * c.nt) c.tmem_cols *= 2;
  if (c.tmem_cols > 512) return false;
  // A 3 x 3 halo stage feeds nine weight stages, so two of them keep the
  // tensor pipe busy; with a 1 x 1 spatial kernel every weight stage needs
  // a halo stage of its own, and both rings are as deep as the budget allows
  // (two would leave the MMAs waiting on each load's round trip).
  c.nb = 8;
  c.na = ks == 1 ? c.nb : 2;
  // (a split's exchange staging gets room of its own above the usual
  // budget, and so do the staged epilogue parameters)
  const size_t budget = (c.split > 1 ? 216 : 200) * 1024 + 4 * static_cast<size_t>(c.params);
  while (c.nb > 2 && umma_smem_bytes(c.kc, c.nt, ks, ks, c.na, c.nb, c.sub, c.split, c.pair,
                                     c.params) > budget) {
    --c.nb;
    if (ks == 1) c.na = c.nb;
  }
  // A short K (a 1 x 1 spatial kernel) with a single N tile: every weight
  // stage of the CTA fits in shared memory beside a halo ring of at least
  // three stages, so the weights are loaded once per launch instead of once
  // per tile (they were most of the bytes moved into shared memory).
  c.b_resident = 0;
  if (ks == 1 && c.split == 1 && c.n_ntiles == 1 && kt * (c_in / c.kc) <= 32) {
    const int stages = kt * (c_in / c.kc);
    const size_t budget_r = 216 * 1024 + 4 * static_cast<size_t>(c.params);
    int na = 8;
    while (na > 3 && umma_smem_bytes(c.kc, c.nt, 1, 1, na, stages, c.sub, 1, c.pair,
                                     c.params) > budget_r)
      --na;
    if (umma_smem_bytes(c.kc, c.nt, 1, 1, na, stages, c.sub, 1, c.pair, c.params) <= budget_r) {
      c.b_resident = 1;
      c.na = na;
      c.nb = stages;
    }
  }
  const size_t smem =
      umma_launch_smem(c.kc, c.nt, ks, c.na, c.nb, c.tmem_cols, c.sub, c.split, c.pair, c.params);
  if (smem > 227 * 1024) return false;
  int per_sm = static_cast<int>((228 * 1024) / (smem + 1024));
  if (per_sm > 512 / c.tmem_cols) per_sm = 512 / c.tmem_cols;
  if (per_sm > 2) per_sm = 2;
  if (c.pair) per_sm = 1;
  c.ctas_per_sm = per_sm < 1 ? 1 : per_sm;
  return true;
}

// Cycles one SM spends on one 128-pixel x nt x 16 MMA step, from the two
// limits measured on B200: the tensor pipe's issue time (48 cycles up to
// N = 64, 56 up to 96, N / 2 beyond) and shared-memory traffic at ~120
// bytes per cycle -- the MMA's operand reads (A: 4 KiB; B: nt x 32 bytes,
// or half of it on a CTA pair) plus the TMA writes of the weights (a stage
// is written once per CTA and shared by its sub-tiles) and of the halo.
long long mma_cycles(const UmmaConfig &c) {
  const long long math = c.nt <= 64 ? 48 : c.nt <= 96 ? 56 : c.nt / 2;
  const long long b_rows = c.pair ? c.nt / 2 : c.nt;
  const long long b_read = 32 * b_rows;
  const long long b_write = c.b_resident ? 0 : 32 * b_rows / (c.pair ? 1 : c.sub);
  const long long bytes = 4096 + b_read + b_write + 1000;
  const long long smem = (bytes + 119) / 120;
  return math > smem ? math : smem;
}

// Relative time of one frame of n images (or of n frames): whole waves of
// tiles over the GPU (SMs, or SM pairs for a pair), each as long as one
// tile's MMA steps.
long long frame_cost(const UmmaConfig &c, int n, int h, int w, int sm_count) {
  const long long tiles = static_cast<long long>(n) * ((h + kTH - 1) / kTH) *
                          ((w + c.sub * kTW - 1) / (c.sub * kTW)) * c.n_ntiles;
  const long long slots = c.pair ? sm_count / 2 : static_cast<long long>(sm_count) * c.ctas_per_sm;
  const long long share = (!c.pair && tiles > sm_count) ? c.ctas_per_sm : 1;
  const long long steps = c.pair ? 1 : c.sub;  // MMA steps per SM per K step
  return (tiles + slots - 1) / slots * share * steps * mma_cycles(c);
}
}  // namespace

bool choose_umma_config(int n, int c_in, int c_out, int h, int w, int kt, int ks, bool rms_epi,
                        bool shortcut, int max_t, int sm_count, UmmaConfig *cfg) {
  // N tile: the largest split of c_out that is a multiple of 16 and at most
  // `cap` (256 is the tcgen05 N limit); the RMS epilogue needs the whole row
  // in one CTA.
  auto largest_nt = [&](int cap) {
    for (int nt = cap; nt >= 16; nt -= 16)
      if (c_out % nt == 0 && (!rms_epi || nt == c_out)) return nt;
    return 0;
  };
  // Every choice below depends on (n, c, h, w, epilogue) and the plan's
  // max_t -- never on a call's t -- so streamed and whole-sequence calls of
  // one plan run identical arithmetic.
  UmmaConfig one;
  one.kc = (c_in % 64 == 0) ? 64 : (c_in % 96 == 0) ? 96 : 32;
  one.sub = 1;
  one.split = 1;
  one.pair = 0;
  one.nt = largest_nt(256);
  if (!one.nt) return false;
  one.n_ntiles = c_out / one.nt;
  one.params = param_floats(c_out, rms_epi ? 2 : 0);
  if (!finish_config(ks, kt, c_in, one)) return false;
  *cfg = one;
  const long long tiles1 = static_cast<long long>(n) * ((h + kTH - 1) / kTH) *
                           ((w + kTW - 1) / kTW) * one.n_ntiles;
  // Temporal split: when even kt CTAs per tile fit one wave, a frame has too
  // few tiles to occupy the GPU (a one-frame chunk of a latent-resolution
  // decoder layer), and its time is the length of one tile's K loop.  Each
  // CTA of a cluster of kt then runs one temporal tap, and the partial sums
  // meet through distributed shared memory in the last CTA.  Not with the
  // RMS epilogue, which needs whole rows in one CTA.  Taken only if it also
  // wins for the plan's largest call (max_t frames): there the split's
  // clusters (about 9/10 of sm_count / kt fit at once) take whole rounds of
  // one-tap work plus the exchange (measured at ~0.4 of a tap's MMAs),
  // against rounds of kt taps over all SMs.
  if (kt >= 2 && kt <= 4 && !rms_epi && !shortcut) {
    UmmaConfig sp = one;
    sp.split = kt;
    const long long calls_tiles = tiles1 * (max_t > 0 ? max_t : 1);
    const long long clusters = sm_count * 9 / (10 * kt);
    const long long slots = static_cast<long long>(sm_count) * one.ctas_per_sm;
    const long long cost_one = (calls_tiles + slots - 1) / slots * kt * 10;
    const long long cost_split = clusters > 0 ? (calls_tiles + clusters - 1) / clusters * 14 : 0;
    if (clusters > 0 && finish_config(ks, kt, c_in, sp) &&
        tiles1 * kt <= static_cast<long long>(sm_count) * sp.ctas_per_sm && cost_split < cost_one) {
      *cfg = sp;
      return true;
    }
  }
  // the tile shapes are compared on the plan's largest call: max_t frames
  // of n images tile like n * max_t images
  const int nt_frames = n * (max_t > 0 ? max_t : 1);
  long long best = frame_cost(one, nt_frames, h, w, sm_count);
  // Two sub-tiles (a 16 x 16 pixel CTA tile, two 8 x 16 MMA tiles) share
  // every weight stage, halving the weight bytes written per MMA.  Only with
  // N <= 128, where both sub-tiles still fit two accumulator buffers (a
  // single buffer stalls the MMAs behind the epilogue).
  UmmaConfig two = one;
  two.sub = 2;
  two.nt = largest_nt(128);
  if (two.nt) {
    two.n_ntiles = c_out / two.nt;
    if (finish_config(ks, kt, c_in, two) && two.nbuf == 2) {
      const long long cost = frame_cost(two, nt_frames, h, w, sm_count);
      if (cost < best) {
        best = cost;
        *cfg = two;
      }
    }
  }
  // A CTA pair (2-SM MMAs, M = 256): each SM holds half of every weight
  // stage, which cuts the shared-memory traffic per MMA enough to reach the
  // tensor pipe's own rate.  64-channel chunks (the 128-byte swizzled halo
  // and weight rows).
  if (one.kc == 64) {
    UmmaConfig pr = one;
    pr.pair = 1;
    pr.sub = 2;  // the tile is two MMA tiles wide
    if (finish_config(ks, kt, c_in, pr) && pr.nbuf == 2) {
      const long long cost = frame_cost(pr, nt_frames, h, w, sm_count);
      if (cost <= best) {
        best = cost;
        *cfg = pr;
      }
    }
  }
  return true;
}

int umma_tile_w() { return kTW; }
int umma_halo_box_w(int kc, int sub, int kw) { return halo_cols(kc, sub, kw); }
int umma_halo_box_c(int kc) { return uses_sw128(kc) ? 64 : 8; }
int umma_tile_h() { return kTH; }

template <int KC, int KS>
cudaError_t set_smem_attr() {
  cudaError_t e = cudaFuncSetAttribute(conv_umma_kernel<KC, KS, 1, false>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(conv_umma_kernel<KC, KS, 2, false>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
  if (e == cudaSuccess && uses_sw128(KC))
    e = cudaFuncSetAttribute(conv_umma_kernel<KC, KS, 1, uses_sw128(KC)>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
  return e;
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

size_t umma_launch_smem(int kc, int nt, int ks, int na, int nb, int tmem_cols, int sub,
                        int split, int pair, int params) {
  size_t smem = umma_smem_bytes(kc, nt, ks, ks, na, nb, sub, split, pair, params);
  // A CTA that holds more than half of tensor memory must have its SM to
  // itself; asking for more than half the shared memory guarantees that.
  if (tmem_cols > 256 && smem < 116 * 1024) smem = 116 * 1024;
  return smem;
}

namespace {
using UmmaKernel = void (*)(const CUtensorMap, const CUtensorMap, const CUtensorMap,
                            const CUtensorMap, UmmaArgs);

UmmaKernel umma_kernel_for(int kc, int ks, int sub, int pair) {
#define CC3D_PICK(KC_, KS_)                                                         \
  if (kc == KC_ && ks == KS_) {                                                     \
    if (pair) return uses_sw128(KC_) ? conv_umma_kernel<KC_, KS_, 1, uses_sw128(KC_)> : nullptr; \
    return sub == 2 ? conv_umma_kernel<KC_, KS_, 2, false>                          \
                    : conv_umma_kernel<KC_, KS_, 1, false>;                         \
  }
  CC3D_PICK(64, 3)
  CC3D_PICK(32, 3)
  CC3D_PICK(96, 3)
  CC3D_PICK(64, 1)
  CC3D_PICK(32, 1)
  CC3D_PICK(96, 1)
#undef CC3D_PICK
  return nullptr;
}

cudaLaunchConfig_t umma_launch_config(unsigned grid, size_t smem, int csize, cudaStream_t stream,
                                      cudaLaunchAttribute *attr) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  attr->id = cudaLaunchAttributeClusterDimension;
  attr->val.clusterDim.x = static_cast<unsigned>(csize);
  attr->val.clusterDim.y = 1;
  attr->val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = csize > 1 ? 1 : 0;
  return cfg;
}
}  // namespace

int umma_max_clusters(const UmmaConfig &c, int ks) {
  const int csize = c.pair ? 2 : c.split;
  if (csize <= 1) return 0;
  UmmaKernel k = umma_kernel_for(c.kc, ks, c.sub, c.pair);
  if (!k) return 0;
  const size_t smem =
      umma_launch_smem(c.kc, c.nt, ks, c.na, c.nb, c.tmem_cols, c.sub, c.split, c.pair, c.params);
  cudaLaunchAttribute attr;
  const cudaLaunchConfig_t cfg =
      umma_launch_config(static_cast<unsigned>(csize), smem, csize, nullptr, &attr);
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, reinterpret_cast<const void *>(k), &cfg) != cudaSuccess) {
    (void)cudaGetLastError();
    return 0;
  }
  return n;
}

cudaError_t launch_conv_umma(const CUtensorMap &map_x, const CUtensorMap &map_cache,
                             const CUtensorMap &map_w, const CUtensorMap &map_sc,
                             const UmmaArgs &args, int kc, unsigned grid, cudaStream_t stream) {
  if (args.kh != args.kw || (args.kh != 1 && args.kh != 3)) return cudaErrorInvalidValue;
  const size_t smem =
      umma_launch_smem(kc, args.nt, args.kh, args.na, args.nb, args.tmem_cols, args.sub,
                       args.split, args.pair, param_floats(args.c_out, args.epi));
  if (smem > 227 * 1024 || (args.sub != 1 && args.sub != 2) || args.nbuf < 1 || args.nbuf > 2)
    return cudaErrorInvalidValue;
  if (args.split != 1 && (args.split != args.kt || args.split > 4 || grid % args.split != 0 ||
                          args.epi == 2 || args.sub != 1 || args.pair))
    return cudaErrorInvalidValue;
  if (args.pair && (kc != 64 || args.sub != 2 || grid % 2 != 0 || args.nt % 16 != 0))
    return cudaErrorInvalidValue;
  if (args.b_resident && (args.split != 1 || args.n_ntiles != 1 || args.nb > 32 ||
                          args.nb != args.kt * args.kh * args.kw * (args.c_in / kc)))
    return cudaErrorInvalidValue;
  if (args.c_sc < 0 ||
      (args.c_sc > 0 && (args.split != 1 || args.b_resident || args.c_sc % 8 != 0 ||
                         args.n_cc_sc != (args.c_sc + kc - 1) / kc)))
    return cudaErrorInvalidValue;
  UmmaKernel k = umma_kernel_for(kc, args.kh, args.sub, args.pair);
  if (!k) return cudaErrorInvalidValue;
  cudaLaunchAttribute attr;
  const cudaLaunchConfig_t cfg =
      umma_launch_config(grid, smem, args.pair ? 2 : args.split, stream, &attr);
  return cudaLaunchKernelEx(&cfg, k, map_x, map_cache, map_w, map_sc, args);
}

}  // namespace cc3d
