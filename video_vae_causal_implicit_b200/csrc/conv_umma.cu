// conv_umma.cu -- bf16 implicit-GEMM causal Conv3D on tcgen05 tensor cores.
//
// Operation ("Cosmos3 Wan VAE -- engine size vs context memory", §10.3
// WanCausalConv3d and its implicit-GEMM view): M = output voxels,
// N = C_out, K = C_in * kt * kh * kw; every tap of an output is summed into
// one fp32 accumulator held in tensor memory; bias is added once in the
// epilogue ("cache-aware video decoder lowering" summary: bias after the
// sum).
//
// Tiling.  An MMA tile is TW = 8 columns x TH = 16 rows of one frame
// (M = 128 rows of the GEMM, row m = 8 * r + c) by NT output channels.  A
// CTA tile is SUB = 1 or 2 such MMA tiles side by side (8 or 16 columns);
// with two, every weight stage feeds two MMAs.  A CTA pair (cluster of two
// CTAs on one SM pair) takes a 16 x 16 tile with 2-SM MMAs (M = 256).  The
// kernel is persistent: one CTA (or pair) per SM takes its tiles in rounds,
// last frame first and serpentine over the clusters (TileOrder).  The K loop
// of a tile runs over (kt, channel chunk of KC, kh, kw).
//
// A operand: for each (kt, channel chunk) the input halo of the tile --
// (TH + kh - 1) x (SUB * TW + kw - 1) pixels x KC channels -- arrives by TMA
// from the current chunk x (frame tau = s * t + kt - (kt_size - 1) >= 0) or
// the frame cache (tau < 0).  Spatial padding is TMA out-of-bounds zero
// fill, and a frame before the chunk with no cache (all zeros) is skipped:
// its stage is neither loaded nor multiplied.  No padded copy exists.  The
// A matrix of spatial tap (kh, kw) and of sub-tile s is the same buffer seen
// from a start address shifted by whole pixels, so one load serves every
// tap.
//
// B operand: the weights, re-tiled at plan time into the exact shared
// memory image of each (N tile, tap, channel chunk) stage.  The taps of one
// kernel row (kh fixed, kw = 0 .. kw_size-1) travel together as one weight
// slot: one wait, kw * KC / 16 MMAs and one commit per slot, so the single
// MMA-issuing thread spends its time issuing MMAs rather than waiting on
// and releasing barriers.
//
// Epilogue.  Four warps read the accumulator from tensor memory and apply
// bias (once), then the residual add, or RMS_norm over the whole C_out row
// followed by SiLU, and store bf16 (or, for a residual block in a chain,
// store y and also SiLU(RMS_norm(y)) for the next block).  The same warps write the frame caches
// of the call: the input cache (the last kt-1 frames of concat(cache_in,
// x)) is copied tile by tile by the tiles of the last output frame, and the
// RMS epilogue's own output frames go to next_cache_out as they are
// stored.  No separate copy kernel runs.
//
// Warp roles (192 threads): warp 0 issues the loads, warp 1 owns tensor
// memory and issues tcgen05.mma from one thread, warps 2..5 run the
// epilogue.  Two accumulators live in tensor memory when they fit, so the
// epilogue of one tile overlaps the MMAs of the next.  Stages are handed
// over with mbarriers; every wait is bounded and reports through the status
// word instead of hanging.  Launches overlap: after its setup a CTA lets the
// stream's next conv start (programmatic dependent launch), and it waits for
// the previous kernel only before touching memory that kernel may write.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <vector>

#include "internal.h"
#include "ptx.cuh"

namespace cc3d {

namespace {

constexpr int kTW = 8;    // tile columns (one core matrix of rows)
constexpr int kTH = 16;   // tile rows -> M = 128
constexpr int kM = kTW * kTH;
constexpr int kThreads = 192;
constexpr int kEpiWarps = 4;
// Largest dynamic shared memory a CTA may request (the opt-in maximum).
constexpr size_t kSmemLimit = 227 * 1024;
// Bound of the drain waits at exit (loads / MMAs already issued finish in
// microseconds; this only guards against a broken pipeline).
constexpr unsigned long long kDrainLimitNs = 100ull * 1000000ull;

struct SmemLayout {
  uint32_t a_off, a_stage, slab, b_off, b_stage, b_slot, x_off, bar_off, p_off, total;
  int na, nb;
};

// A row split over the two CTAs of a cluster (xs = 2): each epilogue warp
// receives its 32 rows' partial sums of squares from the peer into one of
// two slots (tile parity).
constexpr uint32_t kXsBytes = 2u * 4u * 32u * 4u;

// RMS_norm epilogues: 2 with SiLU after it, 3 without, 4 the biased (and,
// with a residual, summed) output stored as y and, as a second output y2,
// RMS_norm + SiLU of it (the next residual block's first norm).
__host__ __device__ constexpr bool rms_epilogue(int epi) { return epi == 2 || epi == 3 || epi == 4; }

// 16 bf16 values at `src` as fp32 (zeros when `valid` is false).
__device__ __forceinline__ void load_bf16x16(const __nv_bfloat16 *src, bool valid, float (&v)[16]) {
  uint4 a = make_uint4(0, 0, 0, 0), b = make_uint4(0, 0, 0, 0);
  if (valid) {
    a = reinterpret_cast<const uint4 *>(src)[0];
    b = reinterpret_cast<const uint4 *>(src)[1];
  }
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

// Epilogue parameters staged in shared memory: bias[c_out] (and, for the
// RMS epilogues, gamma[c_out], beta[c_out]; for FP8 operands the output
// scale[c_out] = s_x * s_w[c_out]).
__host__ __device__ constexpr int param_floats(int c_out, int epi, bool scaled) {
  return c_out * ((rms_epilogue(epi) ? 3 : 1) + (scaled ? 1 : 0));
}

// A channel chunk of 128 means FP8 E4M3 operands: 128 one-byte channels
// per 128-byte pixel row, the same bytes as a 64-channel bf16 chunk.
__host__ __device__ constexpr bool is_e4m3(int kc) { return kc == 128; }
__host__ __device__ constexpr int kc_bytes(int kc) { return is_e4m3(kc) ? kc : 2 * kc; }

__host__ __device__ inline uint32_t round_up(uint32_t v, uint32_t a) { return (v + a - 1) / a * a; }

// 64-channel chunks stage the A halo with the 128-byte swizzle: one TMA box
// of 128-byte pixel rows, its columns padded to a multiple of 8 so that an
// image row of the halo spans whole 1024-byte swizzle atoms.  Other chunk
// widths use 8-channel no-swizzle slabs (16-byte rows, 8 boxes for 64
// channels: many more TMA requests per stage).
__host__ __device__ constexpr bool uses_sw128(int kc) { return kc == 64 || kc == 128; }
__host__ __device__ inline int halo_cols(int kc, int sub, int kw) {
  const int hw = kTW * sub + kw - 1;
  return uses_sw128(kc) ? (hw + 7) / 8 * 8 : hw;
}

// g_taps: weight stages (taps) per B slot; xs: 2 when a row is split over
// the two CTAs of a cluster.
__host__ __device__ inline SmemLayout make_layout(int kc, int nt, int kh, int kw, int na, int nb,
                                                  int sub, int g_taps, bool pair, int params,
                                                  int xs) {
  SmemLayout L;
  const uint32_t hh = kTH + kh - 1, hw = static_cast<uint32_t>(halo_cols(kc, sub, kw));
  if (uses_sw128(kc)) {
    L.slab = hh * hw * 128u;  // the whole halo; a multiple of 1024
    L.a_stage = L.slab;
  } else {
    L.slab = round_up(hh * hw * 16u, 128u);
    L.a_stage = (kc / 8) * L.slab;
  }
  // (a CTA pair: this CTA's half of the N rows, 128-byte swizzled rows, so
  // a stage is a multiple of 1024 bytes as the swizzle atoms require)
  L.b_stage = static_cast<uint32_t>(pair ? nt / 2 : nt) * static_cast<uint32_t>(kc_bytes(kc));
  L.b_slot = static_cast<uint32_t>(g_taps) * L.b_stage;
  L.na = na;
  L.nb = nb;
  L.a_off = 0;
  L.b_off = round_up(L.a_off + na * L.a_stage, 1024u);
  L.x_off = round_up(L.b_off + nb * L.b_slot, 128u);
  L.bar_off = round_up(L.x_off + (xs == 2 ? kXsBytes : 0u), 64u);
  // full_a, empty_a, full_b, empty_b, acc_full[2], acc_empty[2], drain,
  // (xs: x_full[2][4]), tmem slot
  L.p_off = round_up(L.bar_off + 8u * (2 * na + 2 * nb + 5 + (xs == 2 ? 8 : 0)) + 16u, 16u);
  L.total = L.p_off + 4u * static_cast<uint32_t>(params);
  return L;
}

struct TileCoord {
  int ntile, n, t, h0, w0;
};

// Tile order: N tile fastest (CTAs sharing an input halo run together),
// then tile column, tile row, frame, batch image.
// The stride-2 3x3 conv as four phases: output pixel (h, w), tap (kh, kw)
// reads input (2h + kh, 2w + kw) = phase (kh % 2, kw % 2) of the input --
// the pixels (2i + kh % 2, 2j + kw % 2) -- at (i, j) = (h + kh / 2,
// w + kw / 2).  Phase q = 2 * (kh % 2) + kw % 2 serves 4, 2, 2, 1 taps.
__host__ __device__ constexpr int phase_tap_count(int q) { return q == 0 ? 4 : (q == 3 ? 1 : 2); }
// The j-th tap of phase q, as kh * 3 + kw.
__host__ __device__ constexpr int phase_tap(int q, int j) {
  return ((q >> 1) + 2 * (j / ((q & 1) ? 1 : 2))) * 3 + (q & 1) + 2 * (j % ((q & 1) ? 1 : 2));
}

// The tiles of one CTA, round by round.  In round k its cluster takes unit
// (a pixel tile, at each N tile the cluster covers) number k * ncl + slot,
// counting units from the last one -- the last frames first, because a
// chunk's first frames skip their causal zero taps and cost less -- and the
// slot runs over the clusters forwards in even rounds and backwards in odd
// ones, so that the clusters that drew the cheapest units of one round draw
// the dearest of the next (a serpentine deal: with a few more units than
// clusters, the spare ones pair up with cheap ones instead of full ones).
struct TileOrder {
  int n_units, ncl, cid, per, rank;
  __device__ __forceinline__ int rounds() const { return (n_units + ncl - 1) / ncl; }
  // this CTA's tile in round k, or -1 if its cluster has none that round
  __device__ __forceinline__ int at(int k) const {
    const int slot = (k & 1) ? ncl - 1 - cid : cid;
    const int u = k * ncl + slot;
    return u < n_units ? (n_units - 1 - u) * per + rank : -1;
  }
};

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

// One pixel's 16-byte chunks [q0, q1) from `src` (null: zeros) to `dst`;
// both point at the pixel's first byte.
__device__ __forceinline__ void copy_pixel_chunks(const uint8_t *src, uint8_t *dst, int q0,
                                                  int q1) {
  const uint4 *s = reinterpret_cast<const uint4 *>(src);
  uint4 *d = reinterpret_cast<uint4 *>(dst);
  int q = q0;
  for (; q + 4 <= q1; q += 4) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) v[u] = s ? __ldcg(s + q + u) : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int u = 0; u < 4; ++u) d[q + u] = v[u];
  }
  for (; q < q1; ++q) d[q] = s ? __ldcg(s + q) : make_uint4(0, 0, 0, 0);
}

template <int KC, int KS, int SUB, bool PAIR>
__global__ void __launch_bounds__(kThreads, 1)
    conv_umma_kernel(const __grid_constant__ CUtensorMap map_x,
                     const __grid_constant__ CUtensorMap map_cache,
                     const __grid_constant__ CUtensorMap map_w,
                     const __grid_constant__ CUtensorMap map_sc, UmmaArgs p) {
  static_assert(!PAIR || (SUB == 1 && uses_sw128(KC)), "CTA pairs take 128-byte chunks");
  // K steps of one stage: 16 bf16 or 32 E4M3 elements (32 bytes) each
  constexpr int kSteps = kc_bytes(KC) / 32;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // Align the dynamic shared window to 1 KiB ourselves (the attribute is a
  // request, not a guarantee).
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const SmemLayout L = make_layout(KC, p.nt, KS, KS, p.na, p.nb, SUB, p.g_taps, PAIR,
                                   param_floats(p.c_out, p.epi, p.oscale != nullptr), p.xs);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L.bar_off);
  uint64_t *full_a = bars;
  uint64_t *empty_a = full_a + L.na;
  uint64_t *full_b = empty_a + L.na;
  uint64_t *empty_b = full_b + L.nb;
  uint64_t *acc_full = empty_b + L.nb;   // [2]
  uint64_t *acc_empty = acc_full + 2;    // [2]
  uint64_t *drain = acc_empty + 2;       // MMA completion before TMEM is freed
  uint64_t *x_full = drain + 1;          // xs: [tile parity][epilogue warp]
  const bool xs = p.xs == 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(x_full + (xs ? 8 : 0));

  // With PAIR, a cluster of two CTAs (on one SM pair) takes a 16 x 16 pixel
  // tile: CTA `rank` holds the 8 x 16 half at columns 8 * rank and half of
  // each weight stage's N rows, and the leader (rank 0) issues M = 256
  // tcgen05 MMAs over both CTAs' shared memory into both CTAs' tensor memory.
  // With xs, a cluster of two CTAs takes the same pixels: CTA `rank` the
  // output channels of N tile `rank` (its half of an RMS row).
  const int csize = PAIR ? 2 : (xs ? 2 : 1);
  const int rank = (PAIR || xs) ? static_cast<int>(cluster_ctarank()) : 0;
  const int cid = static_cast<int>(blockIdx.x) / csize;
  const int ncl = static_cast<int>(gridDim.x) / csize;
  const bool pair_leader = !PAIR || rank == 0;

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  const int n_cc = p.c_in / KC;   // channel chunks
  const int n_a = p.kt * n_cc;    // A stages per tile
  // weight stages of the conv per N tile, and the shortcut's chunks after them
  // (the stride-2 phase conv: four phase stages against the nine taps'
  // weight stages)
  const bool phases = KS == 2 && p.s2;
  const int n_conv_stages = (phases ? 9 : p.kt * KS * KS) * n_cc;
  const int n_sc = p.c_sc > 0 ? p.n_cc_sc : 0;
  // A 1x1 spatial kernel feeds only kSteps MMAs per halo stage, too few to
  // hide a stage's barrier wait and commit: with resident weights (no weight
  // waits at all) `a_grp` consecutive channel chunks of one frame (in
  // consecutive A slots) share the first slot's full and empty barriers, one
  // wait and one commit per group.  (With streamed weights the longer groups
  // keep fewer halos in flight and cost more than they save.)
  // With streamed weights the plan may group them the same way: g_taps (2
  // or 3) consecutive chunks share one weight slot of g_taps stages beside
  // a group of as many halo slots (b_grouped).
  const bool b_grouped = KS == 1 && !p.b_resident && n_sc == 0 && p.g_taps > 1;
  const int a_grp = (KS == 1 && p.b_resident && n_sc == 0)
                        ? ((n_cc % 3 == 0 && L.na % 3 == 0)   ? 3
                           : (n_cc % 2 == 0 && L.na % 2 == 0) ? 2
                                                              : 1)
                        : (b_grouped ? p.g_taps : 1);
  const int stages_per_ntile = n_conv_stages + n_sc;  // weight image
  // weight slots per A stage: one per group of g_taps spatial taps
  const int g_taps = p.g_taps;
  const int n_groups = b_grouped ? 1 : KS * KS / g_taps;
  constexpr bool kSw = uses_sw128(KC);
  const uint32_t halo_w = static_cast<uint32_t>(halo_cols(KC, SUB, KS));
  const int n_tiles = p.n * p.t * p.tiles_h * p.tiles_w * p.n_ntiles;
  // this CTA's tiles (xs: the M tiles of its cluster, each at N tile `rank`)
  const TileOrder order{xs ? n_tiles / 2 : n_tiles, ncl, cid, xs ? 2 : 1, xs ? rank : 0};
  // A stage whose input frame lies before a chunk that has no cache reads
  // only zeros (not for the stride-2 spatial conv, whose kt counts its
  // phases or taps).
  auto zero_frame = [&](int t, int kt) {
    return !p.s2 && !p.has_cache && p.stride_t * t + kt - (p.kt - 1) < 0;
  };

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
    if (xs)
      for (int i = 0; i < 8; ++i) mbar_init(&x_full[i], 32);  // (the peer warp's lanes)
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
  // (in a cluster, no CTA may arrive on its peer's barriers before the peer
  // has initialised them)
  if (PAIR || xs)
    cluster_sync();
  else
    __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t smem_base = smem_u32(smem);
  bool ok = true;
  // The setup above touched only this CTA's own memories: the next conv of
  // the stream may start its setup now, on the SMs this launch leaves free.
  // Before their first access to memory that earlier kernels write (x, the
  // caches, the residual, y), the producer and the epilogue wait for them;
  // the plan's constants (weights, bias, gamma) need no wait.
  griddep_launch_dependents();

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
      // slots issued at least once, and the phase parity of their last issue
      uint32_t a_used = 0, a_par = 0, b_used = 0, b_par = 0;
      // weight stage `stage_idx` (tap-major, then channel chunk) of N tile
      // `ntile` into part `part` of B slot `slot`: the whole stage, or this
      // CTA's half of its N rows on a pair
      auto load_b = [&](int slot, int part, size_t stage_idx, int ntile) {
        const uint32_t dst = smem_base + L.b_off + slot * L.b_slot + part * L.b_stage;
        if constexpr (PAIR) {
          // rows of the weight image [ntile][tap][cchunk][NT][64]: this
          // CTA's half of the stage's rows
          const int row0 = static_cast<int>(
              (static_cast<size_t>(ntile) * stages_per_ntile + stage_idx) * p.nt);
          tma_load_2d_pair(dst, &map_w, lead_full_b + 8u * slot, 0, row0 + rank * (p.nt / 2));
        } else {
          const uint8_t *wsrc =
              p.wimg + static_cast<size_t>(ntile) * stages_per_ntile * L.b_stage;
          bulk_load(dst, wsrc + stage_idx * L.b_stage, L.b_stage, &full_b[slot]);
        }
      };
      // arm B slot `slot` for `parts` stages (the leader arms for both CTAs
      // of a pair)
      auto arm_b = [&](int slot, int parts) {
        if (pair_leader)
          mbar_arrive_expect_tx(&full_b[slot],
                                static_cast<uint32_t>(parts) * (PAIR ? 2u : 1u) * L.b_stage);
        b_used |= 1u << slot;
        b_par = (b_par & ~(1u << slot)) | (pb << slot);
      };
      // channels c0 .. c0+KC-1 of the box of `map` that starts at column
      // wc, row hc of frame `tcoord` of image `n`, into A slot `slot`
      // (completing on the barrier of slot `bar`: the first of its group)
      auto load_a_at = [&](const CUtensorMap *map, int slot, int c0, int wc, int hc, int tcoord,
                           int n, int bar) {
        const uint32_t dst = smem_base + L.a_off + slot * L.a_stage;
        if constexpr (PAIR) {
          tma_load_5d_pair(dst, map, lead_full_a + 8u * bar, c0, wc, hc, tcoord, n);
        } else if constexpr (kSw) {
          tma_load_5d(dst, map, &full_a[bar], c0, wc, hc, tcoord, n);
        } else {
#pragma unroll
          for (int s = 0; s < KC / 8; ++s)
            tma_load_5d(dst + s * L.slab, map, &full_a[bar], c0 + s * 8, wc, hc, tcoord, n);
        }
      };
      // the tile's halo of channels c0 .. c0+KC-1 of frame `tcoord` of `map`
      // into A slot `slot` (on a pair, this CTA's 8-column half of the tile)
      auto load_a = [&](const CUtensorMap *map, int slot, int c0, int tcoord,
                        const TileCoord &tc, int bar) {
        load_a_at(map, slot, c0, tc.w0 + (PAIR ? kTW * rank : 0) - KS / 2, tc.h0 - KS / 2, tcoord,
                  tc.n, bar);
      };
      // wait for A slot `sa` to be free and arm it
      auto take_a = [&]() -> bool {
        if (!mbar_wait_bounded(&empty_a[sa], pa ^ 1, p.wait_limit_ns, p.status, 1)) return false;
        if (pair_leader)
          mbar_arrive_expect_tx(&full_a[sa],
                                (PAIR ? 2u : 1u) * static_cast<uint32_t>(a_grp) * a_tx);
        a_used |= 1u << sa;
        a_par = (a_par & ~(1u << sa)) | (pa << sa);
        return true;
      };
      if (KS == 1 && p.b_resident) {
        // one N tile and every weight stage in a slot of its own: loaded
        // once here, read in place by the MMAs of every tile
        for (int st = 0; st < L.nb; ++st) {
          arm_b(st, 1);
          load_b(st, 0, static_cast<size_t>(st), 0);
        }
      }
      // the weight slots of a group of A stages (chunks cc0 .. of frame kt)
      auto load_weights = [&](int kt, int cc0, const TileCoord &tc0) -> bool {
        if (b_grouped) {
          // one slot: the stages (kt, cc0 .. cc0 + a_grp - 1) of the 1 x 1 kernel
          if (!mbar_wait_bounded(&empty_b[sb], pb ^ 1, p.wait_limit_ns, p.status, 2)) return false;
          arm_b(sb, a_grp);
          for (int v = 0; v < a_grp; ++v)
            load_b(sb, v, static_cast<size_t>(kt) * n_cc + cc0 + v, tc0.ntile);
          if (++sb == L.nb) { sb = 0; pb ^= 1; }
          return true;
        }
        for (int u = 0; u < a_grp; ++u) {
          const int cc = cc0 + u;
          // this A stage's weight slots: g_taps consecutive taps each (a
          // phase stage: one slot per tap it serves)
          const int n_w = phases ? phase_tap_count(kt) : n_groups;
#pragma unroll 1
          for (int g = 0; g < n_w; ++g) {
            if (!mbar_wait_bounded(&empty_b[sb], pb ^ 1, p.wait_limit_ns, p.status, 2))
              return false;
            arm_b(sb, g_taps);
            for (int v = 0; v < g_taps; ++v)
              load_b(sb, v,
                     static_cast<size_t>(phases ? phase_tap(kt, g)
                                                : kt * KS * KS + g * g_taps + v) * n_cc + cc,
                     tc0.ntile);
            if (++sb == L.nb) { sb = 0; pb ^= 1; }
          }
        }
        return true;
      };
      bool dep_waited = false;  // (griddep_wait issued)
      for (int k = 0; k < order.rounds() && ok; ++k) {
        const int tile = order.at(k);
        if (tile < 0) continue;
        const TileCoord tc0 = decode_tile(tile, p);
        for (int ia = 0; ia < n_a && ok; ia += a_grp) {
          const int kt = ia / n_cc, cc0 = ia % n_cc;
          // A frame before the chunk with no cache is all zeros: its stage
          // (and its taps' weights) is skipped here and by the MMA issuer.
          if (zero_frame(tc0.t, kt)) continue;
          // The first stage's weights (plan constants) go out before the
          // wait for the previous kernel of the stream when the ring holds
          // them all without the MMAs freeing a slot; its halo after it.
          const bool streamed = !(KS == 1 && p.b_resident);
          const bool early_w =
              !dep_waited && streamed &&
              (b_grouped ? 1 : a_grp * (phases ? phase_tap_count(kt) : n_groups)) <= L.nb;
          if (early_w && !load_weights(kt, cc0, tc0)) {
            ok = false;
            break;
          }
          if (!dep_waited) {
            griddep_wait();
            dep_waited = true;
          }
          // the group's a_grp stages (chunks cc0 .. of frame kt) complete on
          // the barrier of its first slot
          if (!take_a()) {
            ok = false;
            break;
          }
          const int bar = sa;
          for (int u = 0; u < a_grp; ++u) {
            if (phases) {
              // stride 2 in H and W, stage `kt` = phase (a, b) = (kt / 2, kt %
              // 2): the map walks every other pixel from input (2 w0 + b,
              // 2 h0 + a), a halo one row and column wider than the tile
              load_a_at(&map_x, sa + u, cc0 * KC,
                        2 * (tc0.w0 + (PAIR ? kTW * rank : 0)) + (kt & 1), 2 * tc0.h0 + (kt >> 1),
                        tc0.t, tc0.n, bar);
            } else {
              const int tau = p.stride_t * tc0.t + kt - (p.kt - 1);  // input frame
              const bool from_cache = tau < 0;  // (zero frames were skipped above)
              load_a(from_cache ? &map_cache : &map_x, sa + u, (cc0 + u) * KC,
                     from_cache ? tau + (p.kt - 1) : tau, tc0, bar);
            }
          }
          sa += a_grp;
          if (sa == L.na) { sa = 0; pa ^= 1; }
          if (!streamed || early_w) continue;
          if (!load_weights(kt, cc0, tc0)) {
            ok = false;
            break;
          }
        }
        // the residual block's 1x1x1 conv_shortcut: each channel chunk of
        // the block input at the output frame (a halo like the conv's, read
        // at its centre tap) against one weight stage stored after the
        // conv's, into the same accumulator
        if (n_sc > 0 && !dep_waited) {
          griddep_wait();
          dep_waited = true;
        }
        for (int c2 = 0; c2 < n_sc && ok; ++c2) {
          if (!take_a()) {
            ok = false;
            break;
          }
          load_a(&map_sc, sa, c2 * KC, tc0.t, tc0, sa);
          if (++sa == L.na) { sa = 0; pa ^= 1; }
          if (!mbar_wait_bounded(&empty_b[sb], pb ^ 1, p.wait_limit_ns, p.status, 2)) {
            ok = false;
            break;
          }
          arm_b(sb, 1);
          load_b(sb, 0, static_cast<size_t>(n_conv_stages + c2), tc0.ntile);
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
      const uint32_t idesc = is_e4m3(KC) ? idesc_e4m3_f32(PAIR ? 2 * kM : kM, p.nt)
                                         : idesc_bf16_f32(PAIR ? 2 * kM : kM, p.nt);
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
      const uint32_t bstage16 = L.b_stage >> 4, bslot16 = L.b_slot >> 4;
      int sa = 0, sb = 0;
      uint32_t pa = 0, pb = 0;
      uint32_t b_seen = 0;  // resident weight slots already seen loaded
      int it = 0;
      for (int k = 0; k < order.rounds() && ok; ++k) {
        const int tile = order.at(k);
        if (tile < 0) continue;
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
        // (the epilogue's tensor-memory reads are ordered before these MMAs)
        tc_fence_after();
        // sub-tile s of this buffer accumulates at columns (buf * SUB + s) * nt
        const uint32_t d_tmem = tmem_base + buf * SUB * p.nt;
        const TileCoord tcm = decode_tile(tile, p);
        uint32_t accumulate = 0;
        // the MMAs of one weight stage (descriptor start b_st) against the
        // halo at `a_st` seen through spatial tap `ts`.  The operands were
        // written by TMA and handed over by the full barriers, whose
        // completion the tensor core's reads observe without a fence.
        // (the issuing thread is the throughput limit of the big convs:
        // the loops below unroll completely)
        auto mma_stage = [&](uint64_t a_st, uint64_t b_st, int ts) {
          const uint64_t a_tap = a_st + ((ts / KS) * halo_w + (ts % KS)) * pix16;
#pragma unroll
          for (int j = 0; j < kSteps; ++j) {
            // every sub-tile (8 pixels further along the halo row) reuses
            // this weight stage
#pragma unroll
            for (int sbt = 0; sbt < SUB; ++sbt) {
              const uint32_t d = d_tmem + (PAIR ? 0 : sbt * p.nt);
              const uint64_t a = a_tap + (PAIR ? 0 : sbt * kTW * pix16) + j * astep16;
              const uint64_t b = b_st + j * bstep16;
              if constexpr (PAIR && is_e4m3(KC)) umma_e4m3_pair(d, a, b, idesc, accumulate);
              else if constexpr (PAIR) umma_bf16_pair(d, a, b, idesc, accumulate);
              else if constexpr (is_e4m3(KC)) umma_e4m3(d, a, b, idesc, accumulate);
              else umma_bf16(d, a, b, idesc, accumulate);
            }
            accumulate = 1;
          }
        };
        // arrive on `bar` (in both CTAs of a pair) once the MMAs issued so
        // far have completed
        auto release = [&](uint64_t *bar) {
          if constexpr (PAIR) umma_commit_pair(bar, 3);
          else umma_commit(bar);
        };
        for (int ia = 0; ia < n_a && ok; ia += a_grp) {
          // the same zero-frame stages the producer skipped; adding their
          // exact zeros would not change the accumulator
          if (zero_frame(tcm.t, ia / n_cc)) continue;
          // (a group of a_grp stages: one wait, one release)
          if (!mbar_wait_bounded(&full_a[sa], pa, p.wait_limit_ns, p.status, 3)) {
            ok = false;
            break;
          }
          for (int u = 0; u < a_grp && ok; ++u) {
          const int is = ia + u;  // this stage: (kt, cc) = (is / n_cc, is % n_cc)
          const uint64_t a_st = adesc0 + (((sa + u) * L.a_stage) >> 4);
          if (KS == 1 && p.b_resident) {
            // resident weights: stage (kt, cc) sits in slot kt * n_cc + cc,
            // loaded once (its first phase stays complete) and never freed,
            // so it is waited for once (a bit per slot: at most 32 slots)
            if (!(b_seen >> is & 1u)) {
              if (!mbar_wait_bounded(&full_b[is], 0u, p.wait_limit_ns, p.status, 4)) {
                ok = false;
                break;
              }
              b_seen |= 1u << is;
            }
            mma_stage(a_st, bdesc0 + static_cast<uint32_t>(is) * bslot16, 0);
          } else if (b_grouped) {
            // the group's weight slot: stage u of it against halo slot sa + u
            if (u == 0 && !mbar_wait_bounded(&full_b[sb], pb, p.wait_limit_ns, p.status, 4)) {
              ok = false;
              break;
            }
            mma_stage(a_st, bdesc0 + static_cast<uint32_t>(sb) * bslot16 +
                                static_cast<uint32_t>(u) * bstage16,
                      0);
            if (u == a_grp - 1) {
              release(&empty_b[sb]);
              if (++sb == L.nb) { sb = 0; pb ^= 1; }
            }
          } else {
            const int q = is / n_cc;  // (a phase stage's phase)
            const int n_w = phases ? phase_tap_count(q) : n_groups;
#pragma unroll 1
            for (int g = 0; g < n_w; ++g) {
              if (!mbar_wait_bounded(&full_b[sb], pb, p.wait_limit_ns, p.status, 4)) {
                ok = false;
                break;
              }
              const uint64_t b_slot = bdesc0 + static_cast<uint32_t>(sb) * bslot16;
              if (phases) {
                // tap (kh, kw) reads its phase at (kh / 2, kw / 2): view
                // (dh, dw) of the 2 x 2 halo
                const int tap = phase_tap(q, g);
                mma_stage(a_st, b_slot, ((tap / 3) >> 1) * KS + ((tap % 3) >> 1));
              } else if (g_taps == KS) {
                // one kernel row: taps (g, 0 .. KS-1)
#pragma unroll
                for (int u = 0; u < KS; ++u)
                  mma_stage(a_st, b_slot + static_cast<uint32_t>(u) * bstage16, g * KS + u);
              } else {
                mma_stage(a_st, b_slot, g);
              }
              // frees the weight slot (in both CTAs of a pair) once these
              // MMAs have read it
              release(&empty_b[sb]);
              if (++sb == L.nb) { sb = 0; pb ^= 1; }
            }
            if (!ok) break;
          }
          }  // the group's stages
          if (!ok) break;
          release(&empty_a[sa]);
          sa += a_grp;
          if (sa == L.na) { sa = 0; pa ^= 1; }
        }
        // the conv_shortcut's chunks: the centre tap of each halo
        for (int c2 = 0; c2 < n_sc && ok; ++c2) {
          if (!mbar_wait_bounded(&full_a[sa], pa, p.wait_limit_ns, p.status, 3) ||
              !mbar_wait_bounded(&full_b[sb], pb, p.wait_limit_ns, p.status, 4)) {
            ok = false;
            break;
          }
          mma_stage(adesc0 + ((sa * L.a_stage) >> 4), bdesc0 + static_cast<uint32_t>(sb) * bslot16,
                    (KS / 2) * KS + KS / 2);
          release(&empty_b[sb]);
          release(&empty_a[sa]);
          if (++sb == L.nb) { sb = 0; pb ^= 1; }
          if (++sa == L.na) { sa = 0; pa ^= 1; }
        }
        // accumulator ready for the epilogue(s)
        release(&acc_full[buf]);
        ++it;
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
    // xs: the peer's partial sums of squares, [tile parity][quarter][lane]
    const float *xbuf = reinterpret_cast<const float *>(smem + L.x_off);
    const uint32_t xbuf_u32 = smem_u32(xbuf);
    bool epi_ok = true;
    // bias (and gamma, beta) of every output channel, staged once: the
    // per-column reads below are then shared-memory broadcasts
    float *sp = reinterpret_cast<float *>(smem + L.p_off);
    const int scale_at = rms_epilogue(p.epi) ? 3 * p.c_out : p.c_out;  // (FP8 output scale)
    for (int i = static_cast<int>(threadIdx.x) - 64; i < p.c_out; i += 32 * kEpiWarps) {
      sp[i] = p.bias[i];
      if (rms_epilogue(p.epi)) {
        sp[p.c_out + i] = p.gamma[i];
        sp[2 * p.c_out + i] = p.beta ? p.beta[i] : 0.f;
      }
      if (p.oscale) sp[scale_at + i] = p.oscale[i];
    }
    griddep_wait();
    named_barrier_sync(1, 32 * kEpiWarps);  // (the epilogue warps only)
    // (shared addresses of the three vectors)
    const uint32_t s_bias = smem_u32(sp), s_gamma = s_bias + 4u * static_cast<uint32_t>(p.c_out),
                   s_beta = s_gamma + 4u * static_cast<uint32_t>(p.c_out),
                   s_scale = s_bias + 4u * static_cast<uint32_t>(scale_at);
    // elements of one input frame and one output frame
    const size_t in_frame = static_cast<size_t>(p.h) * p.w * p.c_in;
    const size_t out_frame = static_cast<size_t>(p.h) * p.w * p.c_out;
    // The call's frame caches, written by the last output frame's tiles:
    // plain copies of the tile's pixels (each N tile takes its share of the
    // channels), made while the tile's MMAs run.
    auto copy_caches = [&](const TileCoord &tc) {
      for (int sbt = 0; sbt < SUB; ++sbt) {
        const int h = tc.h0 + r, w = tc.w0 + (PAIR ? rank : sbt) * kTW + c;
        if (h >= p.h || w >= p.w) continue;
        const size_t pix_img = static_cast<size_t>(h) * p.w + w;
        const int cf = p.cache_frames;
        if (p.cache_out && cf > 0) {
          // cache_out[f] = concat(cache_in or zeros, x)[t_in + f]  (bytes:
          // in_esz per input element)
          const size_t pix_bytes = static_cast<size_t>(p.c_in) * p.in_esz;
          const size_t frame_bytes = in_frame * p.in_esz;
          const int q_all = static_cast<int>(pix_bytes / 16);
          const int q0 = tc.ntile * q_all / p.n_ntiles;
          const int q1 = (tc.ntile + 1) * q_all / p.n_ntiles;
          for (int f = 0; f < cf; ++f) {
            const int src_f = p.t_in + f;  // index into the concatenation
            const uint8_t *src = nullptr;
            if (src_f >= cf)
              src = p.x_in + (static_cast<size_t>(tc.n) * p.t_in + (src_f - cf)) * frame_bytes;
            else if (p.cache_in)
              src = p.cache_in + (static_cast<size_t>(tc.n) * cf + src_f) * frame_bytes;
            uint8_t *dst = p.cache_out + (static_cast<size_t>(tc.n) * cf + f) * frame_bytes;
            copy_pixel_chunks(src ? src + pix_img * pix_bytes : nullptr, dst + pix_img * pix_bytes,
                              q0, q1);
          }
        }
        if (p.ncache_out && p.t < 2) {
          // one output frame: next_cache_out[0] = next_cache_in[1] (or
          // zeros); frame 1 is this tile's output, stored with it
          const int n0 = tc.ntile * p.nt;
          const __nv_bfloat16 *src =
              p.ncache_in ? p.ncache_in + (static_cast<size_t>(tc.n) * 2 + 1) * out_frame +
                                pix_img * p.c_out
                          : nullptr;
          __nv_bfloat16 *dst =
              p.ncache_out + static_cast<size_t>(tc.n) * 2 * out_frame + pix_img * p.c_out;
          copy_pixel_chunks(reinterpret_cast<const uint8_t *>(src), reinterpret_cast<uint8_t *>(dst),
                            n0 / 8, (n0 + p.nt) / 8);
        }
      }
    };
    // this thread's pixel rows of the residual for tile `tc` into L2 (its
    // first reads come from HBM, and the epilogue waits for each of them)
    auto prefetch_residual = [&](const TileCoord &tc) {
      for (int sbt = 0; sbt < SUB; ++sbt) {
        const int h = tc.h0 + r, w = tc.w0 + (PAIR ? rank : sbt) * kTW + c;
        if (h >= p.h || w >= p.w) continue;
        const size_t pix = (static_cast<size_t>(tc.n) * p.t + tc.t) * p.h * p.w +
                           static_cast<size_t>(h) * p.w + w;
        bulk_prefetch_l2(p.residual + pix * p.c_out + tc.ntile * p.nt,
                         static_cast<uint32_t>(p.nt) * 2u);
      }
    };
    for (int k = 0; k < order.rounds(); ++k) {
      const int tile = order.at(k);
      if (tile < 0) continue;
      const int buf = it % p.nbuf;
      const uint32_t use_par = static_cast<uint32_t>((it / p.nbuf) & 1);
      const TileCoord tc0 = decode_tile(tile, p);
      if (p.residual) {
        // this tile's rows (the first tile only) and the next tile's, read
        // one tile from now
        if (it == 0) prefetch_residual(tc0);
        const int next = order.at(k + 1);
        if (next >= 0) prefetch_residual(decode_tile(next, p));
      }
      if (tc0.t == p.t - 1) copy_caches(tc0);
      uint32_t got = 0;
      if (lane == 0)
        got = mbar_wait_bounded(&acc_full[buf], use_par, p.wait_limit_ns, p.status, 5) ? 1u : 0u;
      got = __shfl_sync(0xffffffffu, got, 0);
      if (!got) break;
      tc_fence_after();
      // the frame of next_cache_out (the last two frames of concat(
      // next_cache_in, y)) that this tile's output also goes to, or -1
      const int nc_frame = p.ncache_out ? tc0.t - (p.t - 2) : -1;
      for (int sbt = 0; sbt < SUB; ++sbt) {
        // (a pair's CTA holds the 8 columns at 8 * rank of the 16-wide tile)
        const int h = tc0.h0 + r, w = tc0.w0 + (PAIR ? rank : sbt) * kTW + c;
        const bool valid = (h < p.h) && (w < p.w);
        const bool last_sub = sbt == SUB - 1;
        const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                               static_cast<uint32_t>((buf * SUB + sbt) * p.nt);
        const int n0 = tc0.ntile * p.nt;
        const size_t pix_img = static_cast<size_t>(h) * p.w + w;  // within a frame
        const size_t pix = (static_cast<size_t>(tc0.n) * p.t + tc0.t) * p.h * p.w + pix_img;
        __nv_bfloat16 *yrow = p.y + pix * p.c_out + n0;
        // epi 4: the normalised activation goes to y2, the residual sum to y
        __nv_bfloat16 *outrow = p.epi == 4 ? p.y2 + pix * p.c_out + n0 : yrow;
        const __nv_bfloat16 *rrow = p.residual ? p.residual + pix * p.c_out + n0 : nullptr;
        __nv_bfloat16 *ncrow =
            nc_frame >= 0 ? p.ncache_out + (static_cast<size_t>(tc0.n) * 2 + nc_frame) * out_frame +
                                pix_img * p.c_out + n0
                          : nullptr;
        float inv = 1.0f;
        if (rms_epilogue(p.epi)) {
          // pass 1: sum of squares of the biased row h1 (three loads in
          // flight).  h1 is a bf16 activation, as it is when conv1 writes it
          // out for a separate RMS_norm: it is rounded before it is used.
          // (epi 4: h1 is the residual sum y, the block output)
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
              if (p.epi == 4 && p.residual) {
                float rv[16];
                load_bf16x16(rrow + j0 + 16 * u, valid, rv);
#pragma unroll
                for (int i = 0; i < 16; ++i) bv[i] += rv[i];
              }
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const float hv = round_to_bf16(__uint_as_float(raw[16 * u + i]) + bv[i]);
                ss = fmaf(hv, hv, ss);
              }
            }
          }
          if (xs) {
            // the row's other half is the peer CTA's: swap partial sums
            // through its shared memory (slot: tile parity, this warp's
            // quarter, this lane's row) and add them in rank order, so that
            // both CTAs compute the same norm
            const int slot = ((it & 1) * 4 + q);
            const uint32_t peer = static_cast<uint32_t>(rank ^ 1);
            st_cluster_b32(mapa_shared(xbuf_u32 + 4u * static_cast<uint32_t>(slot * 32 + lane), peer),
                           __float_as_uint(ss));
            mbar_arrive_remote(mapa_shared(smem_u32(&x_full[slot]), peer));
            uint32_t got_x = 0;
            if (lane == 0)
              got_x = mbar_wait_bounded_cluster(&x_full[slot], static_cast<uint32_t>((it >> 1) & 1),
                                                p.wait_limit_ns, p.status, 7)
                          ? 1u
                          : 0u;
            got_x = __shfl_sync(0xffffffffu, got_x, 0);
            if (!got_x) {
              epi_ok = false;
              break;
            }
            const float other = xbuf[slot * 32 + lane];
            ss = rank == 0 ? ss + other : other + ss;
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
          const bool add_res = (p.epi == 1 || (p.epi == 4 && p.residual)) && valid;
          if (add_res) {
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
              if (p.oscale) {
                // FP8 operands: the accumulator times s_x * s_w[c], then bias
                float sv[16];
                ld_param16(s_scale + 4u * static_cast<uint32_t>(n0 + j), sv);
#pragma unroll
                for (int i = 0; i < 16; ++i) v[i] = fmaf(__uint_as_float(raw[16 * u + i]), sv[i], bv[i]);
              } else {
#pragma unroll
                for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(raw[16 * u + i]) + bv[i];
              }
            }
            if (add_res) {
              const __nv_bfloat16 *rb0 = reinterpret_cast<const __nv_bfloat16 *>(&res[2 * u]);
              const __nv_bfloat16 *rb1 = reinterpret_cast<const __nv_bfloat16 *>(&res[2 * u + 1]);
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                v[i] += __bfloat162float(rb0[i]);
                v[8 + i] += __bfloat162float(rb1[i]);
              }
            }
            if (p.epi == 4 && valid) {
              // the block output, before the next block's norm
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
            if (rms_epilogue(p.epi)) {
              float gv[16], be[16];
              ld_param16(s_gamma + 4u * static_cast<uint32_t>(n0 + j), gv);
              ld_param16(s_beta + 4u * static_cast<uint32_t>(n0 + j), be);
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                float a = round_to_bf16(v[i]) * inv * gv[i];
                a += be[i];
                v[i] = p.epi != 3 ? silu_fast(a) : a;
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
              store_bf16x16(outrow + j, o0, o1, p.epi == 4 ? p.y2_vec32 : p.vec32);
              if (ncrow) store_bf16x16(ncrow + j, o0, o1, p.nc_vec32);
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
      if (!epi_ok) break;
      ++it;
    }
  }

  tc_fence_before();
  __syncthreads();
  // no CTA leaves while its peer may still write its shared or tensor memory
  // or arrive on its barriers
  if (PAIR || xs) cluster_sync();
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

size_t umma_smem_bytes(int kc, int nt, int kh, int kw, int na, int nb, int sub, int g_taps,
                       int pair, int params, int xs) {
  // (a pair's CTA holds one 8 x 16 MMA tile: sub counts tile widths)
  return make_layout(kc, nt, kh, kw, na, nb, pair ? 1 : sub, g_taps, pair != 0, params, xs)
             .total +
         1024;  // + alignment slack
}

namespace {
// Buffers, pipeline depths, weight grouping and residency of one tile shape.
bool finish_config(int ks, int kt, int c_in, UmmaConfig &c) {
  const int cta_sub = c.pair ? 1 : c.sub;  // MMA tiles whose accumulators one CTA holds
  c.nbuf = (2 * cta_sub * c.nt <= 512) ? 2 : 1;  // double-buffered accumulators when they fit
  c.tmem_cols = 32;
  while (c.tmem_cols < c.nbuf * cta_sub * c.nt) c.tmem_cols *= 2;
  if (c.tmem_cols > 512) return false;
  auto smem = [&](int na, int nb, int g) {
    return umma_launch_smem(c.kc, c.nt, ks, na, nb, c.tmem_cols, c.sub, g, c.pair, c.params,
                            c.xs);
  };
  // A 3 x 3 halo stage feeds nine weight stages, so two of them keep the
  // tensor pipe busy.  Its weights travel as three slots of one kernel row
  // each when two such slots fit beside the two halo stages (as many slots
  // as fit, up to four), else as single stages (up to eight).  With a 1 x 1
  // spatial kernel every weight stage needs a halo stage of its own, and
  // both rings are as deep as the budget allows (two would leave the MMAs
  // waiting on each load's round trip).
  c.b_resident = 0;
  if (ks == 1) {
    c.g_taps = 1;
    c.nb = 8;
    c.na = 8;
    const size_t budget = 200 * 1024 + 4 * static_cast<size_t>(c.params);
    while (c.nb > 2 && smem(c.na, c.nb, 1) > budget) c.na = --c.nb;
    // Two channel chunks per weight slot and per halo group (one wait and
    // one commit per 2 * KC / 16 MMAs instead of per KC / 16) when the
    // chunks pair up and at least three such slots fit beside two halo
    // groups (the deepest of these ring shapes that fits).
    const int n_cc = c_in / c.kc;
    if (n_cc % 2 == 0) {
      const int shapes[5][2] = {{8, 4}, {6, 4}, {8, 3}, {6, 3}, {4, 3}};
      for (const auto &s : shapes) {
        if (smem(s[0], s[1], 2) <= budget) {
          c.g_taps = 2;
          c.na = s[0];
          c.nb = s[1];
          break;
        }
      }
    }
  } else if (ks == 2) {
    // the stride-2 phase conv: a phase halo serves one to four taps, each
    // tap a weight slot of its own
    c.g_taps = 1;
    c.na = 2;
    c.nb = 8;
    const size_t budget = 200 * 1024 + 4 * static_cast<size_t>(c.params);
    while (c.nb > 2 && smem(c.na, c.nb, 1) > budget) --c.nb;
  } else {
    c.na = 2;
    c.g_taps = ks;
    c.nb = 4;
    while (c.nb > 2 && smem(c.na, c.nb, c.g_taps) > kSmemLimit) --c.nb;
    if (smem(c.na, c.nb, c.g_taps) > kSmemLimit) {
      c.g_taps = 1;
      c.nb = 8;
      const size_t budget = 200 * 1024 + 4 * static_cast<size_t>(c.params);
      while (c.nb > 2 && smem(c.na, c.nb, 1) > budget) --c.nb;
    }
  }
  // A short K (a 1 x 1 spatial kernel) with a single N tile: every weight
  // stage of the CTA fits in shared memory beside a halo ring of at least
  // three stages, so the weights are loaded once per launch instead of once
  // per tile (they were most of the bytes moved into shared memory).
  if (ks == 1 && c.n_ntiles == 1 && kt * (c_in / c.kc) <= 32) {
    const int stages = kt * (c_in / c.kc);
    const size_t budget_r = 216 * 1024 + 4 * static_cast<size_t>(c.params);
    int na = 8;
    while (na > 3 && smem(na, stages, 1) > budget_r) --na;
    if (smem(na, stages, 1) <= budget_r) {
      c.b_resident = 1;
      c.g_taps = 1;
      c.na = na;
      c.nb = stages;
    }
  }
  const size_t bytes = smem(c.na, c.nb, c.g_taps);
  if (bytes > kSmemLimit) return false;
  int per_sm = static_cast<int>((228 * 1024) / (bytes + 1024));
  if (per_sm > 512 / c.tmem_cols) per_sm = 512 / c.tmem_cols;
  if (per_sm > 2) per_sm = 2;
  if (c.pair) per_sm = 1;
  c.ctas_per_sm = per_sm < 1 ? 1 : per_sm;
  return true;
}

// Cycles one SM spends on one 128-pixel x nt x 16 MMA step, from the limits
// measured on B200: the tensor pipe (N / 2 cycles), shared-memory traffic at
// ~120 bytes per cycle -- the MMA's operand reads (A: 4 KiB; B: nt x 32
// bytes, or half of it on a CTA pair) plus the TMA writes of the weights (a
// stage is written once per CTA and shared by its sub-tiles) and of the
// halo -- and the issuing thread, which needs ~60 cycles per MMA
// instruction whatever its size (an instruction of a CTA pair covers both
// SMs).
long long mma_cycles(const UmmaConfig &c) {
  const long long math = c.nt / 2;
  const long long b_rows = c.pair ? c.nt / 2 : c.nt;
  const long long b_read = 32 * b_rows;
  const long long b_write = c.b_resident ? 0 : 32 * b_rows / (c.pair ? 1 : c.sub);
  const long long bytes = 4096 + b_read + b_write + 1000;
  const long long smem = (bytes + 119) / 120;
  const long long issue = c.pair ? 30 : 60;
  const long long t = math > smem ? math : smem;
  return t > issue ? t : issue;
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

long long umma_deal_cost(const UmmaConfig &c, int n, int t_out, int h, int w, int kt,
                         int stride_t, bool cached, int sm_count) {
  const long long tiles_w = (w + c.sub * kTW - 1) / (c.sub * kTW), tiles_h = (h + kTH - 1) / kTH;
  const long long per_frame = tiles_h * tiles_w * (c.xs == 2 ? c.n_ntiles / 2 : c.n_ntiles);
  const long long units = static_cast<long long>(n) * t_out * per_frame;
  const bool clusters = c.pair || c.xs == 2;
  const long long slots =
      clusters ? sm_count / 2 : static_cast<long long>(sm_count) * c.ctas_per_sm;
  const long long workers = std::min(units, slots);
  if (workers < 1 || per_frame < 1) return 0;
  // one unit with all kt taps live (two CTAs of a plan with two per SM
  // share it: each runs at half the rate)
  const long long share = (!clusters && units > sm_count) ? c.ctas_per_sm : 1;
  const long long unit = share * (c.pair ? 1 : c.sub) * mma_cycles(c);
  std::vector<long long> load(static_cast<size_t>(workers), 0);
  for (long long i = 0; i < units; ++i) {
    // the kernel's TileOrder: the i-th unit dealt is unit units-1-i, to
    // worker i % workers in even rounds and from the other end in odd ones
    const long long k = i / workers, slot = i % workers;
    const long long wk = (k & 1) ? workers - 1 - slot : slot;
    const long long t = ((units - 1 - i) / per_frame) % t_out;
    int live = kt;
    if (!cached)
      for (int j = 0; j < kt; ++j)
        if (stride_t * t + j - (kt - 1) < 0) --live;
    load[static_cast<size_t>(wk)] += unit * live;
  }
  return *std::max_element(load.begin(), load.end());
}

bool choose_umma_config(int n, int c_in, int c_out, int h, int w, int kt, int ks, bool rms_epi,
                        int max_t, int sm_count, UmmaConfig *cfg, bool e4m3) {
  // N tile: the largest split of c_out that is a multiple of 16 and at most
  // `cap` (256 is the tcgen05 N limit); the RMS epilogue needs the whole row
  // in one CTA.
  auto largest_nt = [&](int cap) {
    for (int nt = cap; nt >= 16; nt -= 16)
      if (c_out % nt == 0 && (!rms_epi || nt == c_out)) return nt;
    return 0;
  };
  // An RMS row wider than one MMA (257 to 512 channels): the two CTAs of a
  // cluster each take one half of the row (N = c_out / 2) for the same
  // pixels, each into two accumulator buffers (a tile's epilogue runs under
  // the next tile's MMAs), and swap each row's partial sum of squares
  // through shared memory.
  const bool wide_rms = rms_epi && c_out > 256;
  if (wide_rms && (c_out > 512 || c_out % 32 != 0)) return false;
  // Every choice below depends on (n, c, h, w, epilogue) and the plan's
  // max_t -- never on a call's t.  Whatever the shape, every output sums
  // its taps into one fp32 accumulator in the same order: the shapes differ
  // in which CTA computes which outputs, not in how.
  UmmaConfig one{};
  // channel chunk: 128 E4M3 channels, or 64 / 96 / 32 bf16 channels
  if (e4m3 && c_in % 128 != 0) return false;
  one.kc = e4m3 ? 128 : (c_in % 64 == 0) ? 64 : (c_in % 96 == 0) ? 96 : 32;
  one.sub = 1;
  one.pair = 0;
  one.nt = wide_rms ? c_out / 2 : largest_nt(256);
  if (!one.nt) return false;
  one.n_ntiles = c_out / one.nt;
  one.xs = wide_rms ? 2 : 0;
  one.params = param_floats(c_out, rms_epi ? 2 : 0, e4m3);
  if (!finish_config(ks, kt, c_in, one)) return false;
  *cfg = one;
  if (wide_rms) return one.nbuf == 2;
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
  // tensor pipe's own rate.  128-byte chunks (the 128-byte swizzled halo
  // and weight rows).
  if (uses_sw128(one.kc)) {
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
int umma_halo_box_c(int kc) { return is_e4m3(kc) ? 128 : uses_sw128(kc) ? 64 : 8; }
int umma_tile_h() { return kTH; }

template <int KC, int KS>
cudaError_t set_smem_attr() {
  cudaError_t e = cudaFuncSetAttribute(conv_umma_kernel<KC, KS, 1, false>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(conv_umma_kernel<KC, KS, 2, false>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit);
  if (e == cudaSuccess && uses_sw128(KC))
    e = cudaFuncSetAttribute(conv_umma_kernel<KC, KS, 1, uses_sw128(KC)>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit);
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
  if (e == cudaSuccess) e = set_smem_attr<128, 3>();
  if (e == cudaSuccess) e = set_smem_attr<128, 1>();
  // (2 x 2 views of a phase halo: the stride-2 conv)
  if (e == cudaSuccess) e = set_smem_attr<64, 2>();
  if (e == cudaSuccess) e = set_smem_attr<32, 2>();
  if (e == cudaSuccess) e = set_smem_attr<96, 2>();
  return e;
}

size_t umma_launch_smem(int kc, int nt, int ks, int na, int nb, int tmem_cols, int sub,
                        int g_taps, int pair, int params, int xs) {
  size_t smem = umma_smem_bytes(kc, nt, ks, ks, na, nb, sub, g_taps, pair, params, xs);
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
  CC3D_PICK(128, 3)
  CC3D_PICK(128, 1)
  CC3D_PICK(64, 2)
  CC3D_PICK(32, 2)
  CC3D_PICK(96, 2)
#undef CC3D_PICK
  return nullptr;
}

// attr: room for two attributes.  `overlap`: programmatic stream
// serialization (the kernel may start while the stream's previous kernel
// runs; it waits for it before reading what that kernel writes).
cudaLaunchConfig_t umma_launch_config(unsigned grid, size_t smem, int csize, cudaStream_t stream,
                                      cudaLaunchAttribute *attr, bool overlap = false) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  unsigned n = 0;
  if (csize > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = static_cast<unsigned>(csize);
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  if (overlap) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cfg;
}
}  // namespace

int umma_max_clusters(const UmmaConfig &c, int ks) {
  if (!c.pair && c.xs != 2) return 0;
  UmmaKernel k = umma_kernel_for(c.kc, ks, c.sub, c.pair);
  if (!k) return 0;
  const size_t smem = umma_launch_smem(c.kc, c.nt, ks, c.na, c.nb, c.tmem_cols, c.sub, c.g_taps,
                                       c.pair, c.params, c.xs);
  cudaLaunchAttribute attr[2];
  const cudaLaunchConfig_t cfg = umma_launch_config(2u, smem, 2, nullptr, attr);
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
  if (args.kh != args.kw || (args.kh != 1 && args.kh != 3 && !(args.kh == 2 && args.s2)))
    return cudaErrorInvalidValue;
  // weight slots: one tap, one kernel row, or (a 1 x 1 kernel with streamed
  // weights) g_taps channel chunks beside as many halo slots
  const bool chunk_slots = args.kh == 1 && args.g_taps > 1 && !args.b_resident &&
                           args.c_sc == 0 && (args.c_in / kc) % args.g_taps == 0 &&
                           args.na % args.g_taps == 0 && args.g_taps <= 3;
  if (args.g_taps != 1 && args.g_taps != args.kw && !chunk_slots) return cudaErrorInvalidValue;
  // the stride-2 phase conv: four phase stages per channel chunk, one tap
  // per weight slot
  if (args.kh == 2 && (args.kt != 4 || args.g_taps != 1 || args.b_resident))
    return cudaErrorInvalidValue;
  const size_t smem =
      umma_launch_smem(kc, args.nt, args.kh, args.na, args.nb, args.tmem_cols, args.sub,
                       args.g_taps, args.pair,
                       param_floats(args.c_out, args.epi, args.oscale != nullptr), args.xs);
  if (smem > kSmemLimit || (args.sub != 1 && args.sub != 2) || args.nbuf < 1 || args.nbuf > 2 ||
      args.na < 1 || args.na > 32 || args.nb < 1 || args.nb > 32)
    return cudaErrorInvalidValue;
  if (args.pair && (!uses_sw128(kc) || args.sub != 2 || grid % 2 != 0 || args.nt % 16 != 0))
    return cudaErrorInvalidValue;
  // a valid MMA N: a multiple of 16, at most 256 (on a pair each CTA's half
  // of it whole 8-row swizzle atoms)
  if (args.nt % 16 != 0 || args.nt > 256) return cudaErrorInvalidValue;
  // an RMS row split over a cluster: one MMA tile per CTA, two N tiles (one
  // per CTA), two accumulator buffers, whole clusters
  if (args.xs != 0 && (args.xs != 2 || args.pair || args.sub != 1 || args.n_ntiles != 2 ||
                       !rms_epilogue(args.epi) || grid % 2 != 0))
    return cudaErrorInvalidValue;
  if (args.b_resident && (args.n_ntiles != 1 || args.g_taps != 1 ||
                          args.nb != args.kt * args.kh * args.kw * (args.c_in / kc)))
    return cudaErrorInvalidValue;
  if (args.c_sc < 0 ||
      (args.c_sc > 0 && (args.b_resident || args.c_sc % 8 != 0 ||
                         args.n_cc_sc != (args.c_sc + kc - 1) / kc)))
    return cudaErrorInvalidValue;
  // epi 4 (the residual sum and its next-block norm) needs both outputs
  if (args.epi < 0 || args.epi > 4 || (args.epi == 4) != (args.y2 != nullptr))
    return cudaErrorInvalidValue;
  // FP8 operands (128-channel chunks) come with their output scale and a
  // bias or residual epilogue
  if (is_e4m3(kc) != (args.oscale != nullptr) || (is_e4m3(kc) && rms_epilogue(args.epi)) ||
      (args.in_esz != (is_e4m3(kc) ? 1 : 2)))
    return cudaErrorInvalidValue;
  // the frame caches the epilogue writes: whole 16-byte chunks per pixel
  if ((args.cache_out && (args.cache_frames < 1 || (args.c_in * args.in_esz) % 16 != 0 ||
                          !args.x_in || args.t_in < 1 || args.s2)) ||
      (args.ncache_out && (!rms_epilogue(args.epi) || args.nt % 8 != 0)))
    return cudaErrorInvalidValue;
  UmmaKernel k = umma_kernel_for(kc, args.kh, args.sub, args.pair);
  if (!k) return cudaErrorInvalidValue;
  cudaLaunchAttribute attr[2];
  const cudaLaunchConfig_t cfg =
      umma_launch_config(grid, smem, (args.pair || args.xs == 2) ? 2 : 1, stream, attr, true);
  return cudaLaunchKernelEx(&cfg, k, map_x, map_cache, map_w, map_sc, args);
}

}  // namespace cc3d
