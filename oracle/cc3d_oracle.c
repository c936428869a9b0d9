/*
 * cc3d_oracle.c -- plain fp64 CPU oracle for the Wan-style causal Conv3D,
 * the channel RMS_norm, SiLU and the residual block built from them.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the checker the CUDA library is
 * compared against.  Only the tests, the smoke check and the benchmark's CPU
 * baseline leg may load it.  It shares no code, header, table or helper with
 * the CUDA library, and the library never calls it.
 *
 * Every function is the plain definition written out, in the pages' own
 * notation and layout (logical NCTHW indexing, [B, C, T, H, W]):
 *
 *   - causal Conv3D ("Cosmos3 Wan VAE -- engine size vs context memory",
 *     §10.3 "WanCausalConv3d": standard Conv3D y = b + sum W.x over
 *     (c_in, kt, kh, kw); spatial padding symmetric; the time axis padded
 *     only on the past side with 2*T_pad frames, or fed from cache_x, the
 *     last frames of the previous chunk, concatenated in front of t), also
 *     with a temporal stride s (same page, §10.5: the downsample path's
 *     time_conv is a CausalConv3d with stride (2,1,1)): output frame t reads
 *     the padded sequence at s*t + kt, and ceil(T / s) frames come out;
 *   - bias added once, after every tap has been summed ("cache-aware video
 *     decoder lowering" summary, section on turning Conv3D into batched
 *     Conv2D);
 *   - WanRMS_norm (same page, §10.2: v / ||v||_2 over C, times sqrt(C)
 *     times gamma[c], plus bias[c]); the denominator is max(||v||_2, 1e-12),
 *     the documented default of the F.normalize call the page prints;
 *   - SiLU (same page, §10.4: x * sigmoid(x));
 *   - WanResidualBlock (same page, §10.4: norm1 -> SiLU -> conv1 -> norm2
 *     -> SiLU -> dropout (identity at inference) -> conv2, plus the
 *     shortcut, which is the identity when C_in == C_out).
 *
 * Arithmetic is fp64 throughout.  The only rounding is the optional
 * round-to-nearest-even to bfloat16 of the block's conv operands a0 and a1,
 * which models that both convs take bf16 operands (the block runs in bf16
 * on the page).  Accumulation order per output is fixed: c_in, then kt,
 * then kh, then kw; bias last.
 *
 * Inputs are read through a strided 5-D view so the same buffer can be
 * passed in any memory layout; element types are double, float or raw
 * bfloat16 bit patterns (exactly representable in double).
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_F64 0
#define ORC_F32 1
#define ORC_BF16 2

typedef struct {
  const void *data;
  int dtype;             /* ORC_F64, ORC_F32 or ORC_BF16 */
  long long stride[5];   /* element strides of logical dims (n, c, t, h, w) */
} orc_tensor;

/* Exact value of one bfloat16 bit pattern: the pattern is the top 16 bits
 * of an IEEE binary32. */
static double bf16_bits_to_double(uint16_t b) {
  uint32_t u = ((uint32_t)b) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

static double orc_get(const orc_tensor *a, long long i0, long long i1,
                      long long i2, long long i3, long long i4) {
  long long off = i0 * a->stride[0] + i1 * a->stride[1] + i2 * a->stride[2] +
                  i3 * a->stride[3] + i4 * a->stride[4];
  switch (a->dtype) {
    case ORC_F64: return ((const double *)a->data)[off];
    case ORC_F32: return (double)((const float *)a->data)[off];
    default: return bf16_bits_to_double(((const uint16_t *)a->data)[off]);
  }
}

/* Round a double to the nearest bfloat16 value, ties to even.
 * bfloat16 keeps 8 significant bits (1 implicit + 7 stored) and the binary32
 * exponent range: normal numbers down to 2^-126, subnormals spaced 2^-133,
 * largest finite (2 - 2^-7) * 2^127. */
double orc_round_bf16(double v) {
  if (v != v || v == 0.0 || isinf(v)) return v;
  double a = fabs(v);
  double r;
  if (a < ldexp(1.0, -126)) {
    /* subnormal range: a fixed grid of spacing 2^-133 */
    r = nearbyint(ldexp(a, 133));
    r = ldexp(r, -133);
  } else {
    int e;
    double m = frexp(a, &e);            /* a = m * 2^e, m in [0.5, 1) */
    r = nearbyint(ldexp(m, 8));         /* 8 significant bits, RNE */
    r = ldexp(r, e - 8);
    if (r > ldexp(255.0, 120)) r = INFINITY; /* beyond (2-2^-7)*2^127 */
  }
  return v < 0 ? -r : r;
}

/* FP8 E4M3 ("e4m3fn": 4 exponent bits, bias 7, 3 mantissa bits, no
 * infinities, largest finite 448 = 1.75 * 2^8, smallest subnormal 2^-9):
 * v clamped to [-448, 448], then rounded to the nearest E4M3 value, ties to
 * the even mantissa.  The quantiser of a low-precision conv (the pages name
 * INT8 / NVFP4 conv quantisation without giving one; this is the FP8 form
 * the tensor cores take). */
double orc_round_e4m3(double v) {
  if (v != v || v == 0.0) return v;
  double a = fabs(v);
  if (a > 448.0) a = 448.0;
  double r;
  if (a < ldexp(1.0, -6)) {
    /* subnormal range: a fixed grid of spacing 2^-9 */
    r = ldexp(nearbyint(ldexp(a, 9)), -9);
  } else {
    int e;
    double m = frexp(a, &e);            /* a = m * 2^e, m in [0.5, 1) */
    r = ldexp(nearbyint(ldexp(m, 4)), e - 4);  /* 4 significant bits, RNE */
  }
  return v < 0 ? -r : r;
}

/* orc_round_e4m3 over an array, in place. */
void orc_round_e4m3_array(double *v, long long count) {
  for (long long i = 0; i < count; ++i) v[i] = orc_round_e4m3(v[i]);
}

/* One output of the causal Conv3D, straight from the definition.
 * Input frame for output frame t and temporal tap kt is
 * tau = t + kt - (KT - 1): KT - 1 frames of causal front padding.  A frame
 * with tau < 0 comes from the cache (which holds the KT - 1 frames before
 * this chunk, oldest first) or is zero when there is no cache. */
static double conv_at(const orc_tensor *x, const orc_tensor *cache, int Cin,
                      int H, int W, const orc_tensor *wt, int KT, int KH,
                      int KW, int pad_h, int pad_w, int stride_t,
                      const double *bias, int n, int co, int t, int h, int w) {
  double acc = 0.0;
  for (int ci = 0; ci < Cin; ++ci)
    for (int kt = 0; kt < KT; ++kt) {
      /* padded frame stride_t * t + kt, i.e. input frame tau */
      int tau = stride_t * t + kt - (KT - 1);
      if (tau < 0 && cache == NULL) continue; /* zero frame */
      for (int kh = 0; kh < KH; ++kh) {
        int hh = h + kh - pad_h;
        if (hh < 0 || hh >= H) continue;      /* zero padding */
        for (int kw = 0; kw < KW; ++kw) {
          int ww = w + kw - pad_w;
          if (ww < 0 || ww >= W) continue;    /* zero padding */
          double xv = tau >= 0 ? orc_get(x, n, ci, tau, hh, ww)
                               : orc_get(cache, n, ci, tau + (KT - 1), hh, ww);
          acc += orc_get(wt, co, ci, kt, kh, kw) * xv;
        }
      }
    }
  if (bias) acc += bias[co]; /* bias once, after all taps */
  return acc;
}

/* Full causal Conv3D with temporal stride stride_t (>= 1).  T is the input
 * frame count; y is contiguous [N][Cout][Tout][H][W] with
 * Tout = (T - 1) / stride_t + 1.  Output spatial size equals input size
 * (pad = (k - 1) / 2 is what the callers use; any pad_h, pad_w in [0, k) is
 * accepted and the output keeps H x W).  Returns 0, or -1 on a bad
 * argument. */
int orc_causal_conv3d_s(const orc_tensor *x, const orc_tensor *cache, int N,
                        int Cin, int T, int H, int W, const orc_tensor *wt,
                        int Cout, int KT, int KH, int KW, int pad_h, int pad_w,
                        int stride_t, const double *bias, double *y) {
  if (!x || !wt || !y || N < 1 || Cin < 1 || Cout < 1 || T < 1 || H < 1 ||
      W < 1 || KT < 1 || KH < 1 || KW < 1 || stride_t < 1)
    return -1;
  const int Tout = (T - 1) / stride_t + 1;
  long long total = (long long)N * Cout * Tout * H;
#pragma omp parallel for schedule(dynamic, 1)
  for (long long idx = 0; idx < total; ++idx) {
    int h = (int)(idx % H);
    int t = (int)((idx / H) % Tout);
    int co = (int)((idx / ((long long)H * Tout)) % Cout);
    int n = (int)(idx / ((long long)H * Tout * Cout));
    for (int w = 0; w < W; ++w)
      y[(((long long)n * Cout + co) * Tout + t) * H * W + (long long)h * W +
        w] = conv_at(x, cache, Cin, H, W, wt, KT, KH, KW, pad_h, pad_w,
                     stride_t, bias, n, co, t, h, w);
  }
  return 0;
}

/* The same with stride 1 (Tout = T). */
int orc_causal_conv3d(const orc_tensor *x, const orc_tensor *cache, int N,
                      int Cin, int T, int H, int W, const orc_tensor *wt,
                      int Cout, int KT, int KH, int KW, int pad_h, int pad_w,
                      const double *bias, double *y) {
  return orc_causal_conv3d_s(x, cache, N, Cin, T, H, W, wt, Cout, KT, KH, KW,
                             pad_h, pad_w, 1, bias, y);
}

/* The causal Conv3D (temporal stride stride_t) at P chosen output voxels:
 * pts holds P rows (n, t, h, w), t an output frame; y is [P][Cout]. */
int orc_causal_conv3d_points_s(const orc_tensor *x, const orc_tensor *cache,
                               int N, int Cin, int T, int H, int W,
                               const orc_tensor *wt, int Cout, int KT, int KH,
                               int KW, int pad_h, int pad_w, int stride_t,
                               const double *bias, int P, const int *pts,
                               double *y) {
  if (!x || !wt || !y || !pts || P < 0 || stride_t < 1) return -1;
  const int Tout = (T - 1) / stride_t + 1;
  for (int p = 0; p < P; ++p) {
    const int *q = pts + 4 * p;
    if (q[0] < 0 || q[0] >= N || q[1] < 0 || q[1] >= Tout || q[2] < 0 ||
        q[2] >= H || q[3] < 0 || q[3] >= W)
      return -1;
  }
#pragma omp parallel for schedule(dynamic, 1)
  for (long long pc = 0; pc < (long long)P * Cout; ++pc) {
    int p = (int)(pc / Cout), co = (int)(pc % Cout);
    const int *q = pts + 4 * p;
    y[pc] = conv_at(x, cache, Cin, H, W, wt, KT, KH, KW, pad_h, pad_w,
                    stride_t, bias, q[0], co, q[1], q[2], q[3]);
  }
  return 0;
}

int orc_causal_conv3d_points(const orc_tensor *x, const orc_tensor *cache,
                             int N, int Cin, int T, int H, int W,
                             const orc_tensor *wt, int Cout, int KT, int KH,
                             int KW, int pad_h, int pad_w, const double *bias,
                             int P, const int *pts, double *y) {
  return orc_causal_conv3d_points_s(x, cache, N, Cin, T, H, W, wt, Cout, KT,
                                    KH, KW, pad_h, pad_w, 1, bias, P, pts, y);
}

/* The downsample path's spatial step ("Cosmos3 Wan VAE" page, section 10.5,
 * WanResample in downsample mode): every frame on its own goes through
 * ZeroPad2d(pad_l, pad_r, pad_t, pad_b) and a KH x KW Conv2d with stride
 * (sh, sw), bias once:
 *   y[n,co,t,i,j] = b[co] + sum_{ci,kh,kw} W[co,ci,0,kh,kw] *
 *                   xp[n,ci,t, sh*i + kh, sw*j + kw],
 *   xp[.., r, c] = x[.., r - pad_t, c - pad_l] inside the frame, else 0.
 * wt is [Cout][Cin][1][KH][KW]; y is contiguous [N][Cout][T][Ho][Wo] with
 * Ho = (H + pad_t + pad_b - KH) / sh + 1 and Wo likewise.  Returns 0, or -1
 * on a bad argument. */
int orc_conv2d_frames(const orc_tensor *x, int N, int Cin, int T, int H,
                      int W, const orc_tensor *wt, int Cout, int KH, int KW,
                      int sh, int sw, int pad_l, int pad_r, int pad_t,
                      int pad_b, const double *bias, double *y) {
  if (!x || !wt || !y || N < 1 || Cin < 1 || Cout < 1 || T < 1 || H < 1 ||
      W < 1 || KH < 1 || KW < 1 || sh < 1 || sw < 1 || pad_l < 0 ||
      pad_r < 0 || pad_t < 0 || pad_b < 0)
    return -1;
  if (H + pad_t + pad_b < KH || W + pad_l + pad_r < KW) return -1;
  const int Ho = (H + pad_t + pad_b - KH) / sh + 1;
  const int Wo = (W + pad_l + pad_r - KW) / sw + 1;
  const long long total = (long long)N * Cout * T * Ho;
#pragma omp parallel for schedule(dynamic, 1)
  for (long long idx = 0; idx < total; ++idx) {
    const int i = (int)(idx % Ho);
    const int t = (int)((idx / Ho) % T);
    const int co = (int)((idx / ((long long)Ho * T)) % Cout);
    const int n = (int)(idx / ((long long)Ho * T * Cout));
    for (int j = 0; j < Wo; ++j) {
      double acc = 0.0;
      for (int ci = 0; ci < Cin; ++ci)
        for (int kh = 0; kh < KH; ++kh) {
          const int r = sh * i + kh - pad_t; /* row of the unpadded frame */
          if (r < 0 || r >= H) continue;
          for (int kw = 0; kw < KW; ++kw) {
            const int c = sw * j + kw - pad_l;
            if (c < 0 || c >= W) continue;
            acc += orc_get(wt, co, ci, 0, kh, kw) * orc_get(x, n, ci, t, r, c);
          }
        }
      if (bias) acc += bias[co];
      y[(((long long)n * Cout + co) * T + t) * Ho * Wo + (long long)i * Wo + j] = acc;
    }
  }
  return 0;
}

/* SiLU(z) = z * sigmoid(z) = z / (1 + e^-z). */
double orc_silu(double z) { return z / (1.0 + exp(-z)); }

/* RMS_norm of one channel vector v[0..C), written to r[0..C):
 * r[c] = v[c] / max(||v||_2, 1e-12) * sqrt(C) * gamma[c] (+ beta[c]). */
static void rms_vec(const double *v, int C, const double *gamma,
                    const double *beta, double *r) {
  double s = 0.0;
  for (int c = 0; c < C; ++c) s += v[c] * v[c];
  double den = sqrt(s);
  if (den < 1e-12) den = 1e-12;
  double scale = sqrt((double)C);
  for (int c = 0; c < C; ++c)
    r[c] = v[c] / den * scale * gamma[c] + (beta ? beta[c] : 0.0);
}

/* Channel RMS_norm, optionally followed by SiLU, over every (n, t, h, w).
 * y is contiguous [N][C][T][H][W]. */
int orc_rms_norm(const orc_tensor *x, int N, int C, int T, int H, int W,
                 const double *gamma, const double *beta, int apply_silu,
                 double *y) {
  if (!x || !gamma || !y || N < 1 || C < 1 || T < 1 || H < 1 || W < 1)
    return -1;
  long long vox = (long long)N * T * H * W;
#pragma omp parallel
  {
    double *v = (double *)malloc(sizeof(double) * 2 * C);
    double *r = v + C;
#pragma omp for schedule(static)
    for (long long i = 0; i < vox; ++i) {
      int w = (int)(i % W);
      int h = (int)((i / W) % H);
      int t = (int)((i / ((long long)W * H)) % T);
      int n = (int)(i / ((long long)W * H * T));
      for (int c = 0; c < C; ++c) v[c] = orc_get(x, n, c, t, h, w);
      rms_vec(v, C, gamma, beta, r);
      for (int c = 0; c < C; ++c) {
        double o = apply_silu ? orc_silu(r[c]) : r[c];
        y[(((long long)n * C + c) * T + t) * H * W + (long long)h * W + w] = o;
      }
    }
    free(v);
  }
  return 0;
}

static orc_tensor contiguous_ncthw(const double *d, int C, int T, int H,
                                   int W) {
  orc_tensor t;
  t.data = d;
  t.dtype = ORC_F64;
  t.stride[4] = 1;
  t.stride[3] = W;
  t.stride[2] = (long long)H * W;
  t.stride[1] = (long long)T * H * W;
  t.stride[0] = (long long)C * T * H * W;
  return t;
}

/* WanResidualBlock, 3x3x3 convs, spatial pad 1, causal front pad 2, from
 * C_in to C_out channels:
 *   a0 = SiLU(RMS(x; g1))               C_in channels  [bf16 if round_bf16]
 *   h1 = conv1(a0) + b1                 C_out channels [bf16 if round_h1]
 *   a1 = SiLU(RMS(h1; g2))              C_out channels [bf16 if round_bf16]
 *   y  = conv2(a1) + b2 + s,   s = x                      (C_in == C_out, wsc NULL)
 *                              s = conv_1x1x1(x; wsc) + bsc  (the conv_shortcut)
 * conv1 and conv2 take their causal history from cache1 / cache2 (the two
 * a0 / a1 frames before this chunk; NULL = zero frames); the shortcut reads
 * the current frame only.  wsc is [C_out][C_in][1][1][1].
 * y, and the optional a0_out / a1_out, are contiguous [N][C][T][H][W]. */
int orc_resblock2(const orc_tensor *x, const orc_tensor *cache1,
                  const orc_tensor *cache2, int N, int Cin, int Cout, int T,
                  int H, int W, const orc_tensor *w1, const double *b1,
                  const double *g1, const orc_tensor *w2, const double *b2,
                  const double *g2, const orc_tensor *wsc, const double *bsc,
                  int round_bf16, int round_h1, double *y, double *a0_out,
                  double *a1_out) {
  if (!x || !w1 || !w2 || !g1 || !g2 || !y) return -1;
  if (!wsc && Cin != Cout) return -1;
  const long long vox = (long long)N * T * H * W;
  double *a0 = (double *)malloc(sizeof(double) * vox * Cin);
  double *h1 = (double *)malloc(sizeof(double) * vox * Cout);
  double *a1 = (double *)malloc(sizeof(double) * vox * Cout);
  if (!a0 || !h1 || !a1) {
    free(a0); free(h1); free(a1);
    return -2;
  }
  int rc = orc_rms_norm(x, N, Cin, T, H, W, g1, NULL, 1, a0);
  if (round_bf16)
    for (long long i = 0; i < vox * Cin; ++i) a0[i] = orc_round_bf16(a0[i]);
  orc_tensor ta0 = contiguous_ncthw(a0, Cin, T, H, W);
  if (!rc)
    rc = orc_causal_conv3d(&ta0, cache1, N, Cin, T, H, W, w1, Cout, 3, 3, 3, 1,
                           1, b1, h1);
  if (round_h1)
    for (long long i = 0; i < vox * Cout; ++i) h1[i] = orc_round_bf16(h1[i]);
  orc_tensor th1 = contiguous_ncthw(h1, Cout, T, H, W);
  if (!rc) rc = orc_rms_norm(&th1, N, Cout, T, H, W, g2, NULL, 1, a1);
  if (round_bf16)
    for (long long i = 0; i < vox * Cout; ++i) a1[i] = orc_round_bf16(a1[i]);
  orc_tensor ta1 = contiguous_ncthw(a1, Cout, T, H, W);
  if (!rc)
    rc = orc_causal_conv3d(&ta1, cache2, N, Cout, T, H, W, w2, Cout, 3, 3, 3,
                           1, 1, b2, y);
  if (!rc) {
    for (int n = 0; n < N; ++n)
      for (int c = 0; c < Cout; ++c)
        for (int t = 0; t < T; ++t)
          for (int h = 0; h < H; ++h)
            for (int w = 0; w < W; ++w) {
              double sc;
              if (wsc) {
                sc = bsc ? bsc[c] : 0.0;
                for (int ci = 0; ci < Cin; ++ci)
                  sc += orc_get(wsc, c, ci, 0, 0, 0) * orc_get(x, n, ci, t, h, w);
              } else {
                sc = orc_get(x, n, c, t, h, w);
              }
              y[(((long long)n * Cout + c) * T + t) * H * W + (long long)h * W +
                w] += sc;
            }
    if (a0_out) memcpy(a0_out, a0, sizeof(double) * vox * Cin);
    if (a1_out) memcpy(a1_out, a1, sizeof(double) * vox * Cout);
  }
  free(a0); free(h1); free(a1);
  return rc;
}

/* The identity-shortcut block (C_in == C_out == C). */
int orc_resblock(const orc_tensor *x, const orc_tensor *cache1,
                 const orc_tensor *cache2, int N, int C, int T, int H, int W,
                 const orc_tensor *w1, const double *b1, const double *g1,
                 const orc_tensor *w2, const double *b2, const double *g2,
                 int round_bf16, double *y, double *a0_out, double *a1_out) {
  return orc_resblock2(x, cache1, cache2, N, C, C, T, H, W, w1, b1, g1, w2, b2,
                       g2, NULL, NULL, round_bf16, 0, y, a0_out, a1_out);
}

/* a0 = SiLU(RMS(x[n, :, t, h, w]; g1)) at one voxel, optionally rounded. */
static void block_a0_at(const orc_tensor *x, int C, const double *g1,
                        int round_bf16, int n, int t, int h, int w,
                        double *v, double *out) {
  for (int c = 0; c < C; ++c) v[c] = orc_get(x, n, c, t, h, w);
  rms_vec(v, C, g1, NULL, out);
  for (int c = 0; c < C; ++c) {
    out[c] = orc_silu(out[c]);
    if (round_bf16) out[c] = orc_round_bf16(out[c]);
  }
}

/* The residual block at P chosen output voxels (pts rows are n, t, h, w);
 * y is [P][C_out].  Same definition as orc_resblock2, evaluated only on the
 * receptive field of each requested voxel: a0 on a 5x5x5 window, a1 on the
 * 3x3x3 window, then y. */
int orc_resblock2_points(const orc_tensor *x, const orc_tensor *cache1,
                         const orc_tensor *cache2, int N, int Cin, int Cout,
                         int T, int H, int W, const orc_tensor *w1,
                         const double *b1, const double *g1,
                         const orc_tensor *w2, const double *b2,
                         const double *g2, const orc_tensor *wsc,
                         const double *bsc, int round_bf16, int round_h1,
                         int P, const int *pts, double *y) {
  if (!x || !w1 || !w2 || !g1 || !g2 || !y || !pts || P < 0) return -1;
  if (!wsc && Cin != Cout) return -1;
  for (int p = 0; p < P; ++p) {
    const int *q = pts + 4 * p;
    if (q[0] < 0 || q[0] >= N || q[1] < 0 || q[1] >= T || q[2] < 0 ||
        q[2] >= H || q[3] < 0 || q[3] >= W)
      return -1;
  }
  const int Cmax = Cin > Cout ? Cin : Cout;
  int fail = 0;
#pragma omp parallel for schedule(dynamic, 1)
  for (int p = 0; p < P; ++p) {
    const int n = pts[4 * p], t0 = pts[4 * p + 1], h0 = pts[4 * p + 2],
              w0 = pts[4 * p + 3];
    /* a0 window: frames t0-4..t0, rows h0-2..h0+2, cols w0-2..w0+2.
     * present[] marks voxels that exist (frame >= 0 or taken from cache1,
     * row/col inside the image). */
    double *a0w = (double *)calloc((size_t)125 * Cin, sizeof(double));
    char present0[125];
    double *a1w = (double *)calloc((size_t)27 * Cout, sizeof(double));
    char present1[27];
    double *v = (double *)malloc(sizeof(double) * 2 * Cmax);
    double *hv = v + Cmax;
    if (!a0w || !a1w || !v) {
      free(a0w); free(a1w); free(v);
#pragma omp atomic write
      fail = 1;
      continue;
    }
    for (int dt = 0; dt < 5; ++dt)
      for (int dh = 0; dh < 5; ++dh)
        for (int dw = 0; dw < 5; ++dw) {
          int i = (dt * 5 + dh) * 5 + dw;
          int tt = t0 - 4 + dt, hh = h0 - 2 + dh, ww = w0 - 2 + dw;
          double *o = a0w + (size_t)i * Cin;
          present0[i] = 0;
          if (hh < 0 || hh >= H || ww < 0 || ww >= W) continue;
          if (tt >= 0) {
            block_a0_at(x, Cin, g1, round_bf16, n, tt, hh, ww, v, o);
            present0[i] = 1;
          } else if (tt >= -2 && cache1) {
            for (int c = 0; c < Cin; ++c) o[c] = orc_get(cache1, n, c, tt + 2, hh, ww);
            present0[i] = 1;
          }
        }
    /* a1 window: frames t0-2..t0, rows h0-1..h0+1, cols w0-1..w0+1. */
    for (int dt = 0; dt < 3; ++dt)
      for (int dh = 0; dh < 3; ++dh)
        for (int dw = 0; dw < 3; ++dw) {
          int i = (dt * 3 + dh) * 3 + dw;
          int tt = t0 - 2 + dt, hh = h0 - 1 + dh, ww = w0 - 1 + dw;
          double *o = a1w + (size_t)i * Cout;
          present1[i] = 0;
          if (hh < 0 || hh >= H || ww < 0 || ww >= W) continue;
          if (tt < 0) {
            if (tt >= -2 && cache2) {
              for (int c = 0; c < Cout; ++c) o[c] = orc_get(cache2, n, c, tt + 2, hh, ww);
              present1[i] = 1;
            }
            continue;
          }
          /* h1 = conv1(a0) at (tt, hh, ww): window offset of a0 index is
           * (tt - (t0-4)) + kt - 2 etc. */
          for (int co = 0; co < Cout; ++co) {
            double acc = 0.0;
            for (int ci = 0; ci < Cin; ++ci)
              for (int kt = 0; kt < 3; ++kt)
                for (int kh = 0; kh < 3; ++kh)
                  for (int kw = 0; kw < 3; ++kw) {
                    int it = (tt + kt - 2) - (t0 - 4);
                    int ih = (hh + kh - 1) - (h0 - 2);
                    int iw = (ww + kw - 1) - (w0 - 2);
                    int j = (it * 5 + ih) * 5 + iw;
                    if (!present0[j]) continue;
                    acc += orc_get(w1, co, ci, kt, kh, kw) * a0w[(size_t)j * Cin + ci];
                  }
            hv[co] = acc + (b1 ? b1[co] : 0.0);
            if (round_h1) hv[co] = orc_round_bf16(hv[co]);
          }
          rms_vec(hv, Cout, g2, NULL, o);
          for (int c = 0; c < Cout; ++c) {
            o[c] = orc_silu(o[c]);
            if (round_bf16) o[c] = orc_round_bf16(o[c]);
          }
          present1[i] = 1;
        }
    for (int co = 0; co < Cout; ++co) {
      double acc = 0.0;
      for (int ci = 0; ci < Cout; ++ci)
        for (int kt = 0; kt < 3; ++kt)
          for (int kh = 0; kh < 3; ++kh)
            for (int kw = 0; kw < 3; ++kw) {
              int j = (kt * 3 + kh) * 3 + kw;
              if (!present1[j]) continue;
              acc += orc_get(w2, co, ci, kt, kh, kw) * a1w[(size_t)j * Cout + ci];
            }
      acc += b2 ? b2[co] : 0.0;
      double sc;
      if (wsc) {
        sc = bsc ? bsc[co] : 0.0;
        for (int ci = 0; ci < Cin; ++ci)
          sc += orc_get(wsc, co, ci, 0, 0, 0) * orc_get(x, n, ci, t0, h0, w0);
      } else {
        sc = orc_get(x, n, co, t0, h0, w0);
      }
      y[(size_t)p * Cout + co] = acc + sc;
    }
    free(a0w); free(a1w); free(v);
  }
  return fail ? -2 : 0;
}

int orc_resblock_points(const orc_tensor *x, const orc_tensor *cache1,
                        const orc_tensor *cache2, int N, int C, int T, int H,
                        int W, const orc_tensor *w1, const double *b1,
                        const double *g1, const orc_tensor *w2,
                        const double *b2, const double *g2, int round_bf16,
                        int P, const int *pts, double *y) {
  return orc_resblock2_points(x, cache1, cache2, N, C, C, T, H, W, w1, b1, g1,
                              w2, b2, g2, NULL, NULL, round_bf16, 0, P, pts, y);
}
