// internal.h -- declarations shared by the kernels and the C-ABI layer of
// libcc3d.so (not part of the public interface).
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

namespace cc3d {

// Arguments of the tcgen05 implicit-GEMM conv kernel.
struct UmmaArgs {
  const uint8_t *wimg;            // re-tiled weights, [ntile][tap][cchunk][KC/8][NT][8] bf16
  const float *bias;              // [c_out] fp32 (never null; zeros when absent)
  const float *gamma;             // [c_out] (RMS epilogue)
  const float *beta;              // [c_out] or null
  const __nv_bfloat16 *residual;  // [n][t][h][w][c_out] or null
  __nv_bfloat16 *y;               // [n][t][h][w][c_out]
  int *status;                    // device status word
  unsigned long long wait_limit_ns;
  int n, t, h, w, c_in, c_out;    // t: output frames of this call
  int kt, kh, kw, pad_h, pad_w;
  int stride_t;                   // output frame t reads input frames stride_t * t + kt - (kt - 1)
  int nt, n_ntiles, tiles_w, tiles_h;
  int na, nb;                     // pipeline depths (A halo stages, B weight stages)
  int tmem_cols;
  int epi;                        // 0 bias, 1 bias + residual, 2 bias + RMS + SiLU,
                                  // 3 bias + RMS, 4 bias + residual -> y, and RMS + SiLU
                                  // of that sum -> y2 (the next block's first norm)
  int has_cache;
  int sub;                        // MMA sub-tiles (8 x 16 px) per CTA tile, side by side: 1 or 2
  int nbuf;                       // accumulator buffers in tensor memory: 1 or 2
  int g_taps;                     // weight stages (spatial taps) per weight slot: 1, or kw
                                  // (one kernel row)
  int pair;                       // 1: a cluster of 2 CTAs runs 2-SM MMAs on a 16 x 16 px
                                  // tile (sub is then 2: the tile width in MMA tiles)
  int vec32;                      // 1: y and residual are 32-byte aligned (256-bit stores)
  int b_resident;                 // 1: one N tile, every weight stage (nb = kt*kh*kw*c_in/KC)
                                  // in shared memory for the whole launch
  int c_sc;                       // > 0: the residual block's 1x1x1 conv_shortcut of a
                                  // c_sc-channel input (map_sc), summed into the accumulator
  int n_cc_sc;                    // its channel chunks, ceil(c_sc / KC) (tail zero-filled)
  int s2;                         // 1: stride 2 in H and W (the downsample path's 3x3 conv
                                  // per frame): kt = 4 stages per channel chunk, the
                                  // input's four stride-2 phases, each read through a map
                                  // that walks every other pixel and seen through 2 x 2
                                  // views (kh = kw = 2) by the taps it serves; h, w are
                                  // the output frame's
  // Frame caches written by the epilogue (null: not written).
  //   cache_out [n][cache_frames][h][w][c_in] = the last cache_frames frames of
  //   concat(cache_in or zeros, x_in), x_in having t_in frames;
  //   ncache_out [n][2][h][w][c_out] = the last two frames of concat(ncache_in
  //   or zeros, y) (the RMS epilogue's output history).
  const uint8_t *x_in;
  const uint8_t *cache_in;
  uint8_t *cache_out;
  int cache_frames, t_in;
  int in_esz;                     // bytes per input element: 2 (bf16) or 1 (FP8 E4M3)
  const float *oscale;            // FP8 operands: [c_out] output scale s_x * s_w[c] (else null)
  const __nv_bfloat16 *ncache_in;
  __nv_bfloat16 *ncache_out;
  int nc_vec32;                   // 1: ncache_out is 32-byte aligned (256-bit stores)
  __nv_bfloat16 *y2;              // epi 4: [n][t][h][w][c_out], the normalised sum
  int y2_vec32;                   // 1: y2 is 32-byte aligned
  int xs;                         // 2: the two CTAs of a cluster take the same M tiles, CTA
                                  // `rank` N tile `rank` (n_ntiles == 2): an RMS row split
                                  // in halves whose partial sums of squares the CTAs swap
                                  // through shared memory; else 0
};

// Tile configuration of the UMMA conv for a plan (chosen from n, c_in, c_out,
// h, w, the epilogue and the plan's max_t -- never from a call's t).
struct UmmaConfig {
  int kc, nt, n_ntiles, sub, nbuf, g_taps, pair, na, nb, tmem_cols, ctas_per_sm;
  int params;      // epilogue parameters staged in shared memory (floats)
  int b_resident;  // every weight stage resident in shared memory (nb of them)
  int xs;          // 2: an RMS row split over the two CTAs of a cluster (UmmaArgs::xs)
};
// e4m3: FP8 E4M3 operands (128-channel chunks; c_in % 128 == 0).
bool choose_umma_config(int n, int c_in, int c_out, int h, int w, int kt, int ks, bool rms_epi,
                        int max_t, int sm_count, UmmaConfig *cfg, bool e4m3 = false);
// Relative time of a call of t_out output frames of n images (h x w) on the
// tiles of `cfg`, dealt to the CTAs (or clusters) as the kernel deals them;
// without a cache (`cached` false) an output frame's temporal taps that read
// the frames before the chunk are skipped.  kt, stride_t: the temporal
// kernel size and stride.  For choosing a plan's layer per call.
long long umma_deal_cost(const UmmaConfig &cfg, int n, int t_out, int h, int w, int kt,
                         int stride_t, bool cached, int sm_count);
// Clusters of two CTAs that can be resident at once (cfg.pair or cfg.xs),
// for sizing the grid; 0 when the query fails.
int umma_max_clusters(const UmmaConfig &cfg, int ks);

size_t umma_smem_bytes(int kc, int nt, int kh, int kw, int na, int nb, int sub, int g_taps,
                       int pair, int params, int xs);
cudaError_t umma_prepare();
// Dynamic shared memory a launch requests (with the one-CTA-per-SM rule).
size_t umma_launch_smem(int kc, int nt, int ks, int na, int nb, int tmem_cols, int sub,
                        int g_taps, int pair, int params, int xs);
int umma_tile_w();
// TMA box of the A halo: columns (padded for the 128-byte swizzle) and
// channels (64: swizzled pixel rows; 8: no-swizzle slabs).
int umma_halo_box_w(int kc, int sub, int kw);
int umma_halo_box_c(int kc);
int umma_tile_h();
// map_w: the weights' tensor map (plain-rows image) for pair launches;
// map_sc: the conv_shortcut's input (c_sc > 0).  Unused maps may be any
// valid map.
cudaError_t launch_conv_umma(const CUtensorMap &map_x, const CUtensorMap &map_cache,
                             const CUtensorMap &map_w, const CUtensorMap &map_sc,
                             const UmmaArgs &args, int kc, unsigned grid, cudaStream_t stream);

// Weight re-tiling for the UMMA kernel (plan time):
// W[c_out][c_in][kt][kh][kw] (bf16) -> image[ntile][tap][cchunk][kc/8][nt][8].
// rows: 0 = [ntile][tap][cchunk][kc/8][nt][8] (no-swizzle stage images for
// a bulk copy), 1 = [ntile][tap][cchunk][nt][kc] (plain rows for a tensor map)
// stages_per_ntile / stage0: the image holds stages_per_ntile stages per N
// tile and this weight fills stages stage0 .. stage0 + taps*ceil(c_in/kc) - 1
// of each (channels past c_in are zero).
cudaError_t launch_repack_umma(const __nv_bfloat16 *w, uint8_t *img, int c_out, int c_in,
                               int taps, int nt, int kc, int rows, int stages_per_ntile,
                               int stage0, cudaStream_t stream);

// The same image for FP8 E4M3 weights (128-channel chunks, one byte per
// channel): W[c_out][c_in][taps] / w_scale[c_out] rounded to E4M3 in fp32
// (saturated to +-448); rows as for launch_repack_umma, one stage per
// (tap, chunk), stages_per_ntile = taps * c_in / 128.
cudaError_t launch_repack_umma_e4m3(const __nv_bfloat16 *w, const float *w_scale, uint8_t *img,
                                    int c_out, int c_in, int taps, int nt, int rows,
                                    cudaStream_t stream);
// v[i] *= s for i < count (device vector).
cudaError_t launch_scale_vector(float *v, int count, float s, cudaStream_t stream);
// q[i] = E4M3(x[i] / scale) for i < count: bf16 in, one byte out, the
// quotient in fp32, rounded to nearest even and saturated to +-448.
cudaError_t launch_quantize_e4m3(const __nv_bfloat16 *x, size_t count, float scale, uint8_t *q,
                                 cudaStream_t stream);

// Thin first-layer conv (c_in small): weights to [tap*c_in padded to kpad][c_out]
// image and the kernel itself.
struct ThinArgs {
  const uint16_t *x;              // [n][t][h][w][c_in] bf16 bits
  const uint16_t *cache;          // [n][kt-1][h][w][c_in] or null
  const uint8_t *wimg;            // [kpad/8][c_out][8] bf16 core-matrix image
  const float *bias;              // [c_out]
  __nv_bfloat16 *y;               // [n][t][h][w][c_out]
  int *status;
  unsigned long long wait_limit_ns;
  int n, t, h, w, c_in, c_out, kt, kh, kw, pad_h, pad_w;
  int kpad;                       // K padded to a multiple of 16
  int tiles_w, tiles_h, n_tiles;
  int tmem_cols;
  int use_tma;                    // halo by TMA (x and cache 16-byte aligned, w*c_in % 8 == 0)
  int spec_rgb333;                // RGB 3x3x3 pad 1: segment-ordered K (set at plan time)
  int store_boxes;                // y written by TMA tensor stores (c_out % 32 == 0)
};
cudaError_t launch_repack_thin(const __nv_bfloat16 *w, uint8_t *img, int c_out, int c_in,
                               int taps, int kpad, int spec, cudaStream_t stream);
size_t thin_smem_bytes(const ThinArgs &a);
// Elements per halo row of the TMA box (the box's inner extent).
int thin_tma_row(const ThinArgs &a);
cudaError_t launch_conv_thin(const CUtensorMap &map_x, const CUtensorMap &map_cache,
                             const CUtensorMap &map_y, const ThinArgs &args, unsigned grid,
                             cudaStream_t stream);

// fp32 SIMT direct convolution.
struct Fp32Args {
  const float *x, *cache, *w, *bias;
  float *y;
  int n, t, h, w_, c_in, c_out, kt, kh, kw, pad_h, pad_w;
};
cudaError_t launch_conv_fp32(const Fp32Args &a, cudaStream_t stream);

// cache_out = last (kt-1) frames of concat(cache_in or zeros, src[0..t)).
cudaError_t launch_cache_update(const void *cache_in, const void *src, void *cache_out, int n,
                                int t, int frames, size_t frame_bytes, cudaStream_t stream);

// RMS_norm + SiLU over channels of n x t frames of hw pixels, bf16 in/out;
// cache_out (null: not written) = the last two frames of concat(cache_in or
// zeros, y), written by the same kernel.
// silu: apply SiLU after the RMS_norm (else the RMS_norm alone).
cudaError_t launch_rmsnorm_silu(const __nv_bfloat16 *x, const float *gamma, const float *beta,
                                int n, int t, long long hw, int c, __nv_bfloat16 *y,
                                const __nv_bfloat16 *cache_in, __nv_bfloat16 *cache_out,
                                bool silu, cudaStream_t stream);

// One tensor-core conv layer as planned: its tile configuration, geometry
// and device-resident operands (the plan's, or the no-allocation scratch).
struct UmmaLayer {
  UmmaConfig cfg;
  int n, c_in, c_out, h, w;        // input frame geometry
  int kt, kh, kw, pad_h, pad_w;    // kernel as declared (kt, kh, kw of the descriptor)
  int stride_t, s2;                // temporal stride; s2: stride 2 in H and W
  int epi;                         // 0 bias, 1 bias + residual, 2 bias + RMS + SiLU, 3 bias + RMS
  int c_sc, n_cc_sc;               // fused 1x1x1 conv_shortcut (0: none)
  int sm_count, max_clusters;      // grid sizing (max_clusters: CTA pairs)
  int e4m3;                        // FP8 E4M3 operands (x, caches, weights)
  const float *oscale;             // e4m3: [c_out] output scale s_x * s_w[c]
  const uint8_t *wimg;             // re-tiled weights
  const CUtensorMap *map_w;        // the weights as 128-byte swizzled rows (pairs)
  const float *bias, *gamma, *beta;
};
// The pointers of one call (device; null where absent).  t: input frames.
struct UmmaCall {
  const void *x;
  int t;
  const void *cache_in;
  void *y;
  void *cache_out;
  const void *residual;
  const void *ncache_in;
  void *ncache_out;
  const void *x_sc;
  // a residual plan's call that also writes y2 = RMS_norm + SiLU(y; gamma2)
  // (epilogue 4; the plan's tiles must hold whole rows): null = no y2
  void *y2;
  const float *gamma2;
};
// Encodes the call's tensor maps and launches the conv (one kernel, which
// also writes cache_out and ncache_out).  Arguments are assumed validated.
// *tiles: output tiles of the launch.
cudaError_t run_umma_layer(const UmmaLayer &L, const UmmaCall &c, int *status,
                           cudaStream_t stream, uint64_t *tiles);

// Bound of every device-side wait in nanoseconds (CC3D_WAIT_LIMIT_US, else
// 2 s), read once per process.
unsigned long long wait_limit_ns();

// Host-side launch counter (all kernels of this library).
void count_launch();

// Device address of the status word on the current device (null on error).
int *device_status_word();
// 5-D bf16 activation tensor map (dims C, W, H, T, N; boxes of box_c = 8
// plain or 64 swizzled channels).
bool encode_activation_map(CUtensorMap *m, const void *base, int c, int w, int h, int t, int n,
                           int box_w, int box_h, int box_c);
// 2-D tensor map over a plain-rows weight image (rows of 128 bytes: 64 bf16,
// or 128 E4M3 codes), boxes of box_rows rows, 128-byte swizzled.
bool encode_weight_map(CUtensorMap *m, const void *img, long long rows, int box_rows,
                       bool e4m3 = false);

}  // namespace cc3d
