/*
 * cc3d.h -- C ABI of libcc3d.so: the Wan-style causal Conv3D
 * (WanCausalConv3d) and the residual block built around it, for NVIDIA
 * B200 (sm_100a).
 *
 * What is computed
 * ----------------
 * Causal Conv3D ("Cosmos3 Wan VAE -- engine size vs context memory",
 * §10.3, WanCausalConv3d, "causal padding"):
 *
 *   y[n,t,h,w,co] = b[co] + sum_{ci,kt,kh,kw} W[co,ci,kt,kh,kw] *
 *                   xt[n, t+kt, h+kh-pad_h, w+kw-pad_w, ci]
 *
 * where xt = concat(cache_in, x) along t and cache_in holds the kt-1 frames
 * before this chunk (zeros when cache_in is NULL: the causal front pad).
 * Spatially out-of-range reads are zero.  Stride 1, dilation 1, one group.
 * The bias is added once, after all taps ("cache-aware video decoder
 * lowering" summary, the section on per-slice Conv2D: bias after the sum).
 * Chunked evaluation that carries cache_out into the next call's cache_in
 * gives the same outputs as one whole-sequence call (§10.3, cache_x
 * concatenated in front of t; §8.5, CACHE_T = 2).
 *
 * RMS_norm + SiLU (§10.2 WanRMS_norm, §10.4 SiLU):
 *   a[v,c] = SiLU( x[v,c] / max(||x[v,:]||_2, 1e-12) * sqrt(C) * gamma[c]
 *                  (+ beta[c]) ),  computed in fp32, rounded once to bf16.
 *
 * Residual block (§10.4 WanResidualBlock, dropout = identity at inference):
 *   a0 = RMS_SiLU(x; g1);  a1 = RMS_SiLU(conv1(a0) + b1; g2);
 *   y  = conv2(a1) + b2 + s,
 * s = x (identity shortcut, C_in == C_out), or s = conv_shortcut(x) + b_sc,
 * the block's 1x1x1 causal conv, when the channel count changes.
 *
 * Layout
 * ------
 * Activations are channels-last NDHWC ([N][T][H][W][C], C fastest), bf16
 * (fp32 for CC3D_FP32 plans).  Caches are [N][kt-1][H][W][C] in the same
 * dtype.  A caller holding NCTHW tensors permutes them first.
 *
 * Conventions
 * -----------
 *  - Every pointer argument named x, y, cache*, residual, weight, bias,
 *    gamma, beta is a DEVICE pointer on the current device.  The caller owns
 *    all of them; plans and blocks copy what they keep.
 *  - Calls are stream-ordered and asynchronous.  A validation error returns
 *    before anything is launched.  Device-side waits are bounded: a wait
 *    that runs out sets a device status word that cc3d_sync_status()
 *    reports as CC3D_ERR_TIMEOUT (kernels never trap).
 *  - Activation pointers must be 16-byte aligned.  cache_out must not
 *    overlap cache_in, x or y (CC3D_ERR_ALIAS); callers ping-pong two cache
 *    buffers.
 *  - There is no CPU fallback.  A descriptor the kernels do not cover
 *    returns CC3D_ERR_UNSUPPORTED, and the plan's counters record which
 *    kernel served each call.
 */
#ifndef CC3D_H_
#define CC3D_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  CC3D_OK = 0,
  CC3D_ERR_INVALID_ARG = 1,  /* null pointer, bad size, t out of [1, max_t] */
  CC3D_ERR_UNSUPPORTED = 2,  /* spatial stride, dilation or groups != 1, a temporal
                                stride other than 1 or 2, channel counts or
                                kernel sizes no kernel covers, no sm_100 GPU */
  CC3D_ERR_ALIGNMENT = 3,    /* pointer not 16-byte aligned */
  CC3D_ERR_ALIAS = 4,        /* cache_out overlaps cache_in, x or y */
  CC3D_ERR_OOM = 5,          /* device allocation failed in a create call */
  CC3D_ERR_CUDA = 6,         /* a CUDA runtime/driver call failed */
  CC3D_ERR_TIMEOUT = 7,      /* a device-side bounded wait ran out */
  CC3D_ERR_TOO_LARGE = 8     /* cc3d_forward_noalloc: weights exceed its
                                fixed scratch                              */
} cc3d_status;

/* CC3D_FP8_E4M3: FP8 operands ("Cosmos3 Wan VAE", §9 names low-precision
 * conv quantisation without fixing one; this is the E4M3 form the tensor
 * cores take).  x and the caches are E4M3 codes (one byte per element, see
 * cc3d_quantize_e4m3) standing for x_scale * code; the weights are given in
 * bf16 and quantised at plan time to w / w_scale[c_out]; y (and residual)
 * stay bf16:  y = x_scale * w_scale[co] * conv(q_x, q_w) + b[co]. */
typedef enum { CC3D_BF16 = 0, CC3D_FP32 = 1, CC3D_FP8_E4M3 = 2 } cc3d_dtype;

/* Epilogue fused into the conv (§10.4: bias, residual add, next RMS+SiLU). */
typedef enum {
  CC3D_EPI_BIAS = 0,          /* y = conv + b                                  */
  CC3D_EPI_BIAS_RESIDUAL = 1, /* y = conv + b + residual                       */
  CC3D_EPI_BIAS_RMS_SILU = 2, /* y = SiLU(RMS(h; gamma) (+ beta)), h = conv + b
                                 rounded to bf16 first (the block's conv1
                                 output is a bf16 activation); c_out <= 256
                                 (one CTA owns each row), or up to 512 in
                                 steps of 32 (the row's halves on the two
                                 CTAs of a cluster)                         */
  CC3D_EPI_BIAS_RMS = 3       /* y = RMS(h; gamma) (+ beta), the same without
                                 SiLU: the WanRMS_norm after the downsample
                                 path's convs (§10.5)                        */
} cc3d_epilogue;

/* Kernel that served a call (the plan's route counters). */
typedef enum {
  CC3D_VARIANT_NONE = 0,
  CC3D_VARIANT_UMMA = 1,     /* tcgen05 implicit GEMM, TMA halo tiles       */
  CC3D_VARIANT_THIN = 2,     /* c_in = 3 first layer, tcgen05, gathered A   */
  CC3D_VARIANT_FP32 = 3      /* fp32 SIMT direct convolution               */
} cc3d_variant;

typedef struct {
  int n, c_in, c_out, h, w, max_t;   /* max_t: largest frame count per call  */
  int kt, kh, kw;                    /* kernel size; causal front pad = kt-1 */
  int pad_h, pad_w;                  /* spatial zero padding (kh/2, kw/2)    */
  int stride_t;        /* temporal stride: 1, or 2 (the downsample path's
                          time_conv; bf16 tensor-core descriptors only).
                          Output frame t reads input frames
                          stride_t*t + kt - (kt-1); a call of t input frames
                          writes (t-1)/stride_t + 1 output frames (y and
                          residual have that many).  Streamed chunks of a
                          multiple of stride_t frames give the whole
                          sequence's outputs.                               */
  int stride_h, stride_w;  /* 1, or both 2: the downsample path's spatial
                              step (§10.5): each frame zero-padded by one
                              row and column after it, then a 3x3 conv with
                              stride 2 -- kt = 1, kh = kw = 3, pad_h = pad_w
                              = 0, h and w even, bf16 with c_in % 32 == 0,
                              bias or residual epilogue.  y (and residual)
                              are [n][t][h/2][w/2][c_out].                  */
  int dil_t, dil_h, dil_w;           /* must be 1                            */
  int groups;                        /* must be 1                            */
  cc3d_dtype dtype;
  const void *weight;  /* device [c_out][c_in][kt][kh][kw] (PyTorch order),
                          dtype; copied (and re-tiled) at create             */
  const float *bias;   /* device [c_out] fp32, nullable (= 0); copied        */
  cc3d_epilogue epi;
  const float *gamma;  /* device [c_out] fp32, RMS epilogues only; copied    */
  const float *beta;   /* device [c_out] fp32, nullable; copied               */
  const float *w_scale; /* CC3D_FP8_E4M3 only: device [c_out] fp32 per-output-
                           channel weight scales (> 0); copied               */
  float x_scale;        /* CC3D_FP8_E4M3 only: the activation scale (> 0) of x
                           and the caches                                   */
} cc3d_desc;

typedef struct {
  uint64_t calls;          /* successful cc3d_forward launches               */
  uint64_t rejected;       /* calls refused by validation                    */
  uint64_t tiles;          /* output tiles launched in total                 */
  int variant;             /* cc3d_variant chosen at create                  */
  int tile_h, tile_w;      /* output tile (rows x cols of one frame)         */
  int n_tile;              /* output channels per CTA                        */
  int k_chunk;             /* input channels per pipeline stage              */
  int k_split;             /* always 1: every output sums all of its taps in
                              one accumulator of one CTA (no split-K)       */
  int mma_ctas;            /* CTAs (SMs) per tensor-core MMA: 1, or 2 for a
                              CTA pair issuing 2-SM MMAs (M = 256)          */
  int w_resident;          /* 1: the weights stay in shared memory for the
                              whole launch (short K, one N tile), 0: they
                              stream through a ring, once per tile          */
  int row_ctas;            /* CTAs that share one output pixel's channels: 1,
                              or 2 when an RMS row wider than 256 channels
                              is split over a cluster of two CTAs (each one
                              half, the row's sum of squares exchanged
                              between them through shared memory)          */
  int one_frame_mma_ctas;  /* mma_ctas of the tiles that calls of one output
                              frame use: a plan for max_t > 1 keeps a second
                              tile choice (and weight image) for them when
                              the best tiles for one frame differ; every
                              tile shape gives the same bytes              */
  int one_frame_n_tile;    /* n_tile of those tiles                          */
  uint64_t second_tile_calls; /* calls that ran on that second tile choice:
                              every one-frame call, and the longer calls it
                              finishes sooner (e.g. a call without a cache,
                              whose first frames skip their causal zero
                              taps)                                         */
} cc3d_stats;

typedef struct cc3d_plan cc3d_plan;
typedef struct cc3d_block cc3d_block;

/* Validate desc, pick a kernel, copy and re-tile the weights (and bias,
 * gamma, beta) into plan-owned device memory.  Synchronous.  Returns
 * CC3D_ERR_UNSUPPORTED for dilation/groups != 1, strides other than those
 * stride_t / stride_h / stride_w document, even kernel sizes, or channel
 * counts no kernel covers.  FP8 E4M3 covers c_in % 128 == 0, c_out % 16 ==
 * 0, kh == kw in {1, 3}, kt <= 3, temporal stride 1 or 2, bias or residual
 * epilogue.  bf16 covers c_out % 16 == 0 with
 * either c_in % 32 == 0 (kh == kw in {1, 3}, kt <= 3; N tiles of at most
 * 256 channels) or c_in <= 8 (the thin first-layer path: bias epilogue,
 * c_out <= 256, kt*kh*kw*c_in <= 256); fp32 covers any channel count with
 * the bias epilogue.  *out is set only on CC3D_OK. */
cc3d_status cc3d_plan_create(const cc3d_desc *desc, cc3d_plan **out);
cc3d_status cc3d_plan_destroy(cc3d_plan *plan);

/* One causal conv over a chunk of t frames (1 <= t <= max_t).
 *   x         [n][t][h][w][c_in]       input chunk
 *   cache_in  [n][kt-1][h][w][c_in]    frames before the chunk, oldest
 *                                      first; NULL = zero frames
 *   y         [n][t'][h][w][c_out]     output, t' = (t-1)/stride_t + 1
 *                                      (t' = t at temporal stride 1)
 *   cache_out [n][kt-1][h][w][c_in]    nullable: the last kt-1 frames of
 *                                      concat(cache_in, x), for the next call
 *                                      (written by the conv kernel itself on
 *                                      the tensor-core path: no extra launch)
 *   residual  [n][t'][h][w][c_out]     EPI_BIAS_RESIDUAL only, else NULL
 *   next_cache_in / next_cache_out     RMS epilogues only, nullable:
 *                                      [n][2][h][w][c_out]; next_cache_out
 *                                      receives the last 2 frames of
 *                                      concat(next_cache_in, y) -- the cache
 *                                      of the conv that consumes y.
 *   stream    a cudaStream_t (NULL = legacy default stream). */
cc3d_status cc3d_forward(cc3d_plan *plan, const void *x, int t,
                         const void *cache_in, void *y, void *cache_out,
                         const void *residual, const void *next_cache_in,
                         void *next_cache_out, void *stream);

/* One call of cc3d_forward_host: x and y in host memory, the rest as in
 * cc3d_forward (device pointers, same shapes and rules). */
typedef struct {
  const void *x_host;     /* [n][t][h][w][c_in] host memory                 */
  int t;                  /* frames of x, 1 <= t <= max_t                    */
  const void *cache_in;   /* device, nullable                                */
  void *cache_out;        /* device, nullable                                */
  const void *residual;   /* device, EPI_BIAS_RESIDUAL only                  */
  void *y_host;           /* [n][t'][h][w][c_out] host memory                */
} cc3d_host_call;

/* cc3d_forward over host buffers, for callers whose video lives in host
 * memory: `ncalls` calls of one plan run in order, each as upload of x ->
 * conv -> download of y, overlapped across calls: call i+1's upload and
 * call i-1's download run while call i's conv runs.  The uploads use a
 * stream of the plan, the convs run on `stream`, the downloads on a second
 * stream of the plan; the data pass through three device staging slots of
 * max_t frames of x and of y that the plan allocates on first use (freed
 * by cc3d_plan_destroy).  The first upload starts after the work enqueued
 * on `stream` before the call; on return every copy and conv is enqueued
 * and `stream` waits for the last download, so work enqueued on `stream`
 * afterwards, or a synchronize of it, sees every y_host complete.  Host
 * buffers should be pinned (cudaHostAlloc / cudaHostRegister) for the
 * copies to overlap; pageable memory works, with the copies serialised.
 * A call's y_host must not overlap another call's x_host or y_host.  The
 * calls are validated before anything is enqueued: CC3D_ERR_INVALID_ARG
 * (null host pointers, ncalls < 1, t out of range, a residual that does
 * not match the epilogue, an RMS-epilogue plan -- its next caches have no
 * host form), CC3D_ERR_ALIGNMENT / CC3D_ERR_ALIAS for the device pointers
 * as in cc3d_forward; CC3D_ERR_OOM when the staging slots cannot be
 * allocated.  Not safe to call on one plan from two threads at once. */
cc3d_status cc3d_forward_host(cc3d_plan *plan, const cc3d_host_call *calls, int ncalls,
                              void *stream);

/* FP8 E4M3 codes of bf16 values: q[i] = E4M3(x[i] / scale), the quotient
 * an IEEE fp32 division, rounded to nearest even and saturated to +-448
 * (the activation side of a CC3D_FP8_E4M3 plan).  x (device, 16-byte
 * aligned) holds `count` bf16 values, q (device, 8-byte aligned) receives
 * `count` bytes; count % 8 == 0, scale > 0, else CC3D_ERR_INVALID_ARG. */
cc3d_status cc3d_quantize_e4m3(const void *x, size_t count, float scale, void *q,
                               void *stream);

/* Stand-alone channel RMS_norm + SiLU (§10.2, §10.4), bf16 in / bf16 out.
 *   x, y      [n][t][h][w][c]; gamma [c] fp32; beta [c] fp32 nullable
 *   cache_in / cache_out  nullable, [n][2][h][w][c]: cache_out receives the
 *             last 2 frames of concat(cache_in (or zeros), y), written by
 *             the same kernel.
 * c must be a multiple of 8 and at most 1024. */
cc3d_status rmsnorm_silu(const void *x, const float *gamma, const float *beta,
                         int n, int t, int h, int w, int c, void *y,
                         const void *cache_in, void *cache_out, void *stream);

/* Stand-alone channel RMS_norm without SiLU (§10.2 WanRMS_norm; the norms
 * around the downsample path's convs, §10.5), bf16 in / bf16 out:
 *   y[v,c] = x[v,c] / max(||x[v,:]||_2, 1e-12) * sqrt(C) * gamma[c] (+ beta[c]).
 * Arguments, layout, caches and errors as for rmsnorm_silu. */
cc3d_status rms_norm(const void *x, const float *gamma, const float *beta, int n,
                     int t, int h, int w, int c, void *y, const void *cache_in,
                     void *cache_out, void *stream);

/* Residual block with c channels and the identity shortcut (§10.4):
 * cc3d_block_create2(n, c, c, ..., w_sc = b_sc = NULL, out). */
cc3d_status cc3d_block_create(int n, int c, int h, int w, int max_t,
                              const void *w1, const float *b1, const float *g1,
                              const void *w2, const float *b2, const float *g2,
                              cc3d_block **out);

/* Residual block from c_in to c_out channels (§10.4).  Device arguments,
 * all copied: w1 [c_out][c_in][3][3][3] and w2 [c_out][c_out][3][3][3] bf16;
 * g1 [c_in], b1, g2, b2 [c_out] fp32 (b1, b2 nullable); w_sc
 * [c_out][c_in][1][1][1] bf16 and b_sc [c_out] fp32 (nullable): the
 * conv_shortcut, required when c_in != c_out (NULL: identity shortcut).
 * The shortcut runs inside conv2 as extra K steps of the same accumulator
 * (the shortcut's bias is added to b2); conv1's epilogue applies the
 * RMS_norm + SiLU (up to c_out = 512; wider blocks write conv1's biased
 * output and run a separate RMS_norm + SiLU pass).  In every block conv1's
 * output is rounded to bf16 before its RMS_norm.
 * c_in, c_out multiples of 32 in [32, 1024], else CC3D_ERR_UNSUPPORTED;
 * CC3D_ERR_INVALID_ARG for a NULL weight or gamma, or c_in != c_out without
 * w_sc.  The block owns its activation buffers (max_t frames each). */
cc3d_status cc3d_block_create2(int n, int c_in, int c_out, int h, int w,
                               int max_t, const void *w1, const float *b1,
                               const float *g1, const void *w2,
                               const float *b2, const float *g2,
                               const void *w_sc, const float *b_sc,
                               cc3d_block **out);
cc3d_status cc3d_block_destroy(cc3d_block *block);

/* y = block(x) for a chunk of t frames: x [n][t][h][w][c_in], y
 * [n][t][h][w][c_out].  cache1_* is conv1's history (a0 frames,
 * [n][2][h][w][c_in]), cache2_* conv2's (a1 frames, [n][2][h][w][c_out]);
 * *_in nullable (zeros), *_out nullable.  All bf16. */
cc3d_status cc3d_resblock_forward(cc3d_block *block, const void *x, int t,
                                  const void *cache1_in, const void *cache2_in,
                                  void *y, void *cache1_out, void *cache2_out,
                                  void *stream);

/* cc3d_resblock_forward for chains of blocks, with the next block's first
 * RMS_norm + SiLU moved into this block's conv2 epilogue (§10.4: in a stage
 * of residual blocks, block k+1 starts with SiLU(RMS_norm(y_k; g1 of k+1))).
 * Up to c_out = 256 conv2's epilogue computes it from the accumulator row it
 * stores as y; wider blocks hand over through a norm pass over y after
 * conv2 (the whole-row tiles such rows need make conv2 slower than that
 * pass costs).  Either way the next block skips its own first norm.
 *   a0_in        nullable; else this block's a0 = SiLU(RMS_norm(x; g1)),
 *                [n][t][h][w][c_in], as the previous block's call wrote it
 *                into its a0_next: the block's own first norm is skipped
 *                (x is still read: residual or conv_shortcut input), and
 *                cache1_out is written by conv1 from cache1_in and a0_in.
 *   g_next       nullable: device [c_out] fp32, the next block's g1.  With
 *                it, the call writes y (unchanged) and also
 *   a0_next      [n][t][h][w][c_out] = SiLU(RMS_norm(y; g_next)), computed
 *                from y rounded to bf16, with its history
 *   a0_next_cache_in / a0_next_cache_out  nullable, [n][2][h][w][c_out]:
 *                the next block's cache1 (last two frames of
 *                concat(a0_next_cache_in or zeros, a0_next)).
 * The result equals cc3d_resblock_forward of each block in turn up to the
 * rounding order of the fused norm's sum of squares.  a0_next without
 * g_next, or the reverse, or a0_next_cache_* without them, is
 * CC3D_ERR_INVALID_ARG; a0_next must not overlap x, y, a0_in or any cache
 * (CC3D_ERR_ALIAS); every pointer is 16-byte aligned (CC3D_ERR_ALIGNMENT).
 * These checks run before any launch. */
cc3d_status cc3d_resblock_forward_fused(cc3d_block *block, const void *x,
                                        const void *a0_in, int t,
                                        const void *cache1_in,
                                        const void *cache2_in, void *y,
                                        void *cache1_out, void *cache2_out,
                                        const float *g_next, void *a0_next,
                                        const void *a0_next_cache_in,
                                        void *a0_next_cache_out, void *stream);

/* Synchronise `stream` and report (then clear) the device status word:
 * CC3D_ERR_TIMEOUT if a kernel's bounded wait ran out since the last call,
 * CC3D_ERR_CUDA on a CUDA error, else CC3D_OK. */
cc3d_status cc3d_sync_status(void *stream);

/* Copy the plan's counters. */
cc3d_status cc3d_get_stats(const cc3d_plan *plan, cc3d_stats *out);

/* Static description of a status code. */
const char *cc3d_status_string(cc3d_status s);

/* Number of kernel launches made by this library in this process (all
 * entry points).  Lets callers count device work. */
uint64_t cc3d_launch_count(void);

/* cc3d_forward without a plan and without any device allocation.
 *
 * The pages have no counterpart to this entry point; it exists for callers
 * that cannot call cudaMalloc: code that must hand all device memory out of
 * its own fixed pool (a serving process that reserves its budget up front,
 * a framework whose allocator owns the device), and latency-critical loops
 * where an allocation's implicit synchronisation is not acceptable.
 *
 * It computes exactly what cc3d_plan_create(desc) + cc3d_forward(...) would
 * (same kernel, same tiles), for bf16 descriptors that the tensor-core path
 * covers.  desc->weight / bias / gamma / beta are read on every call (bias
 * and gamma/beta directly, the weights after re-tiling); desc->max_t bounds
 * t as usual.  The re-tiled weights live in one fixed, file-scope device
 * array of 8 MiB + 16 KiB that every GPU which loads the library holds until
 * the process exits.  A descriptor whose weights need more than 8 MiB
 * (c_out * c_in * kt * kh * kw * 2 bytes; 384 x 384 x 3 x 3 x 3 fits)
 * returns CC3D_ERR_TOO_LARGE before anything is launched.
 *
 * All calls on a device share that array and it keeps the last call's
 * contents; calls that overlap on the GPU (different streams, no ordering
 * between them) race on it and give wrong results.  Serialise them.
 * The first call on a device looks the array's device address up (and
 * prepares the kernels); make that first call before any stream capture.
 * Arguments and errors are those of cc3d_forward. */
cc3d_status cc3d_forward_noalloc(const cc3d_desc *desc, const void *x, int t,
                                 const void *cache_in, void *y, void *cache_out,
                                 const void *residual, const void *next_cache_in,
                                 void *next_cache_out, void *stream);

#ifdef __cplusplus
}
#endif
#endif /* CC3D_H_ */
