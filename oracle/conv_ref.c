/*
 * conv_ref.c -- CPU oracle for the convolution forward pass (TEST INFRASTRUCTURE).
 *
 * This file is the checker, not the product.  Only the test-suite, the
 * package's smoke check and the CPU-baseline leg of the benchmark may load it.
 * It shares no code, header or constant with the CUDA library: its index
 * arithmetic, its half/bfloat16 decoders and its round-to-nearest encoders are
 * written here from their definitions.
 *
 * What it computes (the plain definition, no blocking, no reordering):
 *
 *   "Convolutions" tutorial, section 1 ("What is it?"): a small filter slides
 *   over the input and every output is the dot product of the filter with the
 *   window under it.  Section 4 ("Tiny example") spells this out as the loop
 *   out[i][j] += x[i+di][j+dj] * k[di][dj] -- a cross-correlation (the filter
 *   is NOT flipped).  The same page's "Convolution variants" table adds
 *   grouped convolution (channels split into G groups) and dilation ("gaps in
 *   the kernel"); section 7 fixes channels-last (NHWC) layout.  The MLX pull
 *   request "Add implicit matmul pathway for mx.conv3d" (benchmark table
 *   header) fixes the 3-D layouts: input (N, D, H, W, C), weight
 *   (O, kD, kH, kW, C/groups), one stride / pad per spatial dimension.
 *
 *   y[n,od,oh,ow,o] = sum_{kd,kh,kw,c} x[n, od*sd-pd+kd*dd, oh*sh-ph+kh*dh,
 *                                        ow*sw-pw+kw*dw, g*Cg+c]
 *                                     * w[o, kd, kh, kw, c]
 *   with g = o / Og, Cg = C/G, Og = O/G, and x = 0 outside [0,D)x[0,H)x[0,W)
 *   (zero padding, the same pad on both sides of a dimension).
 *
 *   Output extent per dimension: floor((I + 2p - dil*(k-1) - 1) / s) + 1.
 *   The tutorial's ResNet-50 example (224x224 input, 7x7, stride 2, giving a
 *   112x112 output in its FLOP count) is consistent with this at pad 3.
 *
 *   Two options are also provided, each in its plainest reading.  Flip (the
 *   MLX pull request's "What changed" list: its input loader handles a
 *   "correct flip" of the filter) reads the filter reversed in every spatial
 *   dimension, w[o, kD-1-kd, kH-1-kh, kW-1-kw, c] -- a true convolution
 *   instead of the cross-correlation.  Per-side padding is the general form
 *   of the padding above: p_lo below and p_hi above a dimension (the index
 *   origin is -p_lo; the extent uses p_lo + p_hi in place of 2p).  With
 *   p_lo = p_hi = p and no flip they reduce to the definition above.
 *
 * Alongside y the oracle returns S = sum |x*w| over the same receptive field;
 * the parity tolerance is expressed relative to S.
 *
 * Precision: every product of two binary16/bfloat16/binary32 values is exact
 * in binary64 and the fp64 sum of a few thousand such terms is exact to about
 * 1e-13 relative to S, so y is the exact result for practical purposes.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORACLE_F32 = 0, ORACLE_F16 = 1, ORACLE_BF16 = 2 };

/* ---- element decoders (IEEE 754 binary16 and the bfloat16 truncation of
 *      binary32), written from the bit-field definitions ------------------ */

double oracle_f16_to_f64(uint16_t h) {
  int sign = (h >> 15) & 1;
  int e = (h >> 10) & 0x1f;
  int m = h & 0x3ff;
  double v;
  if (e == 0) {
    v = ldexp((double)m, -24);                  /* subnormal: m * 2^-24 */
  } else if (e == 31) {
    v = m ? NAN : INFINITY;
  } else {
    v = ldexp((double)(1024 + m), e - 25);      /* (1.m) * 2^(e-15) */
  }
  return sign ? -v : v;
}

double oracle_bf16_to_f64(uint16_t b) {
  int sign = (b >> 15) & 1;
  int e = (b >> 7) & 0xff;
  int m = b & 0x7f;
  double v;
  if (e == 0) {
    v = ldexp((double)m, -133);                 /* subnormal: m * 2^-133 */
  } else if (e == 255) {
    v = m ? NAN : INFINITY;
  } else {
    v = ldexp((double)(128 + m), e - 134);      /* (1.m) * 2^(e-127) */
  }
  return sign ? -v : v;
}

static double load_elem(const void* p, int64_t i, int dtype) {
  if (dtype == ORACLE_F16) return oracle_f16_to_f64(((const uint16_t*)p)[i]);
  if (dtype == ORACLE_BF16) return oracle_bf16_to_f64(((const uint16_t*)p)[i]);
  return (double)((const float*)p)[i];
}

/* ---- correctly rounded binary64 -> binary16 / bfloat16 (round to nearest,
 *      ties to even), used to express "the oracle value rounded to the
 *      output type" ----------------------------------------------------- */

/* Generic encoder for a binary format with `mbits` stored significand bits,
 * minimum normal exponent `emin`, maximum exponent `emax` and exponent bias
 * `bias`. */
static uint32_t encode_rn(double v, int mbits, int emin, int emax, int bias,
                          int ebits) {
  uint32_t sign = signbit(v) ? 1u : 0u;
  uint32_t inf_bits = ((1u << ebits) - 1u) << mbits;
  uint32_t out;
  if (isnan(v)) return (sign << (mbits + ebits)) | inf_bits | (1u << (mbits - 1));
  double a = fabs(v);
  if (isinf(a)) return (sign << (mbits + ebits)) | inf_bits;
  if (a == 0.0) return sign << (mbits + ebits);
  int e2;
  frexp(a, &e2);                 /* a = f * 2^e2, f in [0.5, 1) */
  int E = e2 - 1;                /* a in [2^E, 2^(E+1)) */
  if (E < emin) E = emin;        /* subnormal range shares emin's quantum */
  double q = ldexp(1.0, E - mbits);
  double r = rint(a / q);        /* exact scaling, RNE in default mode */
  double rv = r * q;
  /* overflow: anything that rounds to >= 2^(emax+1) becomes infinity */
  if (rv >= ldexp(1.0, emax + 1)) return (sign << (mbits + ebits)) | inf_bits;
  if (rv == 0.0) return sign << (mbits + ebits);
  frexp(rv, &e2);
  E = e2 - 1;
  if (E < emin) {                /* subnormal: exponent field 0 */
    uint32_t mant = (uint32_t)(rv / ldexp(1.0, emin - mbits));
    out = mant;
  } else {
    uint32_t mant = (uint32_t)(rv / ldexp(1.0, E - mbits)) - (1u << mbits);
    out = ((uint32_t)(E + bias) << mbits) | mant;
  }
  return (sign << (mbits + ebits)) | out;
}

uint16_t oracle_f64_to_f16_rn(double v) {
  return (uint16_t)encode_rn(v, 10, -14, 15, 15, 5);
}

uint16_t oracle_f64_to_bf16_rn(double v) {
  return (uint16_t)encode_rn(v, 7, -126, 127, 127, 8);
}

/* ---- output extent ---------------------------------------------------- */

static int64_t extent(int64_t in, int k, int s, int p_lo, int p_hi, int d) {
  int64_t num = in + (int64_t)p_lo + (int64_t)p_hi - (int64_t)d * (k - 1) - 1;
  if (num < 0) return 0;
  return num / s + 1;
}

/* Output extents with padding p_lo below and p_hi above each dimension. */
int oracle_out_dims_ex(int D, int H, int W, int kD, int kH, int kW,
                       const int stride[3], const int pad_lo[3],
                       const int pad_hi[3], const int dil[3], int out[3]) {
  const int in[3] = {D, H, W};
  const int k[3] = {kD, kH, kW};
  for (int i = 0; i < 3; ++i) {
    if (in[i] <= 0 || k[i] <= 0 || stride[i] <= 0 || dil[i] <= 0 ||
        pad_lo[i] < 0 || pad_hi[i] < 0)
      return -1;
    int64_t e = extent(in[i], k[i], stride[i], pad_lo[i], pad_hi[i], dil[i]);
    if (e <= 0 || e > 0x7fffffff) return -1;
    out[i] = (int)e;
  }
  return 0;
}

int oracle_out_dims(int D, int H, int W, int kD, int kH, int kW,
                    const int stride[3], const int pad[3], const int dil[3],
                    int out[3]) {
  return oracle_out_dims_ex(D, H, W, kD, kH, kW, stride, pad, pad, dil, out);
}

/* ---- the direct sum ---------------------------------------------------- */

typedef struct {
  int N, D, H, W, C, O, kD, kH, kW, G;
  int Do, Ho, Wo;
  int s[3], p[3], d[3];  /* p: the padding below (the index origin is -p) */
  int flip;              /* read the filter reversed in every spatial dimension */
} shape_t;

static int make_shape(shape_t* sh, int N, int D, int H, int W, int C, int O,
                      int kD, int kH, int kW, const int stride[3],
                      const int pad_lo[3], const int pad_hi[3],
                      const int dil[3], int groups, int flip) {
  int out[3];
  if (N <= 0 || C <= 0 || O <= 0 || groups <= 0) return -1;
  if (C % groups || O % groups) return -1;
  if (flip != 0 && flip != 1) return -1;
  if (oracle_out_dims_ex(D, H, W, kD, kH, kW, stride, pad_lo, pad_hi, dil, out))
    return -1;
  sh->N = N; sh->D = D; sh->H = H; sh->W = W; sh->C = C; sh->O = O;
  sh->kD = kD; sh->kH = kH; sh->kW = kW; sh->G = groups;
  sh->Do = out[0]; sh->Ho = out[1]; sh->Wo = out[2];
  for (int i = 0; i < 3; ++i) {
    sh->s[i] = stride[i]; sh->p[i] = pad_lo[i]; sh->d[i] = dil[i];
  }
  sh->flip = flip;
  return 0;
}

/* One output element, reading x and w through `fetch` so that both the
 * pre-decoded (double) and the raw (typed) inputs share this loop. */
#define ORACLE_POINT_BODY(XAT, WAT)                                          \
  do {                                                                       \
    const int Cg = sh->C / sh->G, Og = sh->O / sh->G;                        \
    const int g = o / Og;                                                    \
    double acc = 0.0, mag = 0.0;                                             \
    for (int kd = 0; kd < sh->kD; ++kd) {                                    \
      int64_t id = (int64_t)od * sh->s[0] - sh->p[0] + (int64_t)kd * sh->d[0]; \
      if (id < 0 || id >= sh->D) continue;                                   \
      for (int kh = 0; kh < sh->kH; ++kh) {                                  \
        int64_t ih = (int64_t)oh * sh->s[1] - sh->p[1] + (int64_t)kh * sh->d[1]; \
        if (ih < 0 || ih >= sh->H) continue;                                 \
        for (int kw = 0; kw < sh->kW; ++kw) {                                \
          int64_t iw = (int64_t)ow * sh->s[2] - sh->p[2] + (int64_t)kw * sh->d[2]; \
          if (iw < 0 || iw >= sh->W) continue;                               \
          int64_t xb = ((((int64_t)n * sh->D + id) * sh->H + ih) * sh->W + iw) \
                       * sh->C + (int64_t)g * Cg;                            \
          const int fd = sh->flip ? sh->kD - 1 - kd : kd;                    \
          const int fh = sh->flip ? sh->kH - 1 - kh : kh;                    \
          const int fw = sh->flip ? sh->kW - 1 - kw : kw;                    \
          int64_t wb = ((((int64_t)o * sh->kD + fd) * sh->kH + fh) * sh->kW + fw) \
                       * Cg;                                                 \
          for (int c = 0; c < Cg; ++c) {                                     \
            double t = XAT(xb + c) * WAT(wb + c);                            \
            acc += t;                                                        \
            mag += fabs(t);                                                  \
          }                                                                  \
        }                                                                    \
      }                                                                      \
    }                                                                        \
    *py = acc;                                                               \
    *ps = mag;                                                               \
  } while (0)

static void point_f64(const shape_t* sh, const double* x, const double* w,
                      int n, int od, int oh, int ow, int o, double* py,
                      double* ps) {
#define XD(i) x[i]
#define WD(i) w[i]
  ORACLE_POINT_BODY(XD, WD);
#undef XD
#undef WD
}

static void point_raw(const shape_t* sh, const void* x, const void* w,
                      int dtype, int n, int od, int oh, int ow, int o,
                      double* py, double* ps) {
#define XR(i) load_elem(x, i, dtype)
#define WR(i) load_elem(w, i, dtype)
  ORACLE_POINT_BODY(XR, WR);
#undef XR
#undef WR
}

static double* decode_all(const void* p, int64_t n, int dtype) {
  double* out = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
  if (!out) return NULL;
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = load_elem(p, i, dtype);
  return out;
}

/* Full output.  x: NDHWC [N,D,H,W,C]; w: [O,kD,kH,kW,C/groups]; y and s:
 * [N,Do,Ho,Wo,O] doubles.  dtype: 0 = binary32, 1 = binary16, 2 = bfloat16.
 * Returns 0, or -1 on an invalid shape, -2 on an unknown dtype, -3 when out
 * of host memory. */
int oracle_conv_fwd_ex(const void* x, const void* w, int dtype, int N, int D,
                       int H, int W, int C, int O, int kD, int kH, int kW,
                       const int stride[3], const int pad_lo[3],
                       const int pad_hi[3], const int dil[3], int groups,
                       int flip, double* y, double* s) {
  shape_t sh;
  if (dtype < 0 || dtype > 2) return -2;
  if (make_shape(&sh, N, D, H, W, C, O, kD, kH, kW, stride, pad_lo, pad_hi, dil,
                 groups, flip))
    return -1;
  int64_t nx = (int64_t)N * D * H * W * C;
  int64_t nw = (int64_t)O * kD * kH * kW * (C / groups);
  double* xd = decode_all(x, nx, dtype);
  double* wd = decode_all(w, nw, dtype);
  if (!xd || !wd) { free(xd); free(wd); return -3; }
  const shape_t* shp = &sh;
#pragma omp parallel for collapse(3) schedule(dynamic, 1)
  for (int n = 0; n < sh.N; ++n)
    for (int od = 0; od < sh.Do; ++od)
      for (int oh = 0; oh < sh.Ho; ++oh)
        for (int ow = 0; ow < shp->Wo; ++ow)
          for (int o = 0; o < shp->O; ++o) {
            int64_t q = ((((int64_t)n * shp->Do + od) * shp->Ho + oh) * shp->Wo + ow)
                        * shp->O + o;
            point_f64(shp, xd, wd, n, od, oh, ow, o, &y[q], &s[q]);
          }
  free(xd);
  free(wd);
  return 0;
}

/* Selected outputs only: idx[i] is a flat index into [N,Do,Ho,Wo,O].
 * Reads x and w in their storage type, so it needs no copy of the input.
 * Returns 0, -1 (shape), -2 (dtype) or -4 (an index out of range). */
int oracle_conv_fwd_points_ex(const void* x, const void* w, int dtype, int N,
                              int D, int H, int W, int C, int O, int kD, int kH,
                              int kW, const int stride[3], const int pad_lo[3],
                              const int pad_hi[3], const int dil[3], int groups,
                              int flip, const int64_t* idx, int64_t npts,
                              double* y, double* s) {
  shape_t sh;
  if (dtype < 0 || dtype > 2) return -2;
  if (make_shape(&sh, N, D, H, W, C, O, kD, kH, kW, stride, pad_lo, pad_hi, dil,
                 groups, flip))
    return -1;
  int64_t total = (int64_t)sh.N * sh.Do * sh.Ho * sh.Wo * sh.O;
  for (int64_t i = 0; i < npts; ++i)
    if (idx[i] < 0 || idx[i] >= total) return -4;
  const shape_t* shp = &sh;
#pragma omp parallel for schedule(dynamic, 64)
  for (int64_t i = 0; i < npts; ++i) {
    int64_t q = idx[i];
    int o = (int)(q % shp->O); q /= shp->O;
    int ow = (int)(q % shp->Wo); q /= shp->Wo;
    int oh = (int)(q % shp->Ho); q /= shp->Ho;
    int od = (int)(q % shp->Do); q /= shp->Do;
    int n = (int)q;
    point_raw(shp, x, w, dtype, n, od, oh, ow, o, &y[i], &s[i]);
  }
  return 0;
}

/* The symmetric-padding, unflipped forms (the definition above). */
int oracle_conv_fwd(const void* x, const void* w, int dtype, int N, int D,
                    int H, int W, int C, int O, int kD, int kH, int kW,
                    const int stride[3], const int pad[3], const int dil[3],
                    int groups, double* y, double* s) {
  return oracle_conv_fwd_ex(x, w, dtype, N, D, H, W, C, O, kD, kH, kW, stride,
                            pad, pad, dil, groups, 0, y, s);
}

int oracle_conv_fwd_points(const void* x, const void* w, int dtype, int N,
                           int D, int H, int W, int C, int O, int kD, int kH,
                           int kW, const int stride[3], const int pad[3],
                           const int dil[3], int groups, const int64_t* idx,
                           int64_t npts, double* y, double* s) {
  return oracle_conv_fwd_points_ex(x, w, dtype, N, D, H, W, C, O, kD, kH, kW,
                                   stride, pad, pad, dil, groups, 0, idx, npts,
                                   y, s);
}

/* ---- transposed convolution ----------------------------------------------
 *
 * "Convolutions" tutorial, "Convolution variants worth knowing": the
 * transposed ("upsampling") convolution of decoders and diffusion models.  The
 * page gives no formula; its plainest reading, and the one every framework
 * uses, is the adjoint of the forward pass above: with the same weight tensor
 * w[Cin, kD, kH, kW, Cout/G] (the forward pass's [O, k, C/G] with O = Cin
 * input and C = Cout output channels), every input element x[n, i, ci]
 * scatters x * w[ci, k, c] onto the output position q = i*s - p + k*d:
 *
 *   y[n, q, g*Cog + c] = sum over taps k and input channels ci of group g
 *                        with q = i*s - p + k*d, 0 <= i < I, of
 *                        x[n, i, ci] * w[ci, k, c]          (per dimension)
 *
 * where Cog = Cout/G and group g holds input channels [g*Cin/G, (g+1)*Cin/G).
 * Output extent per dimension: (I-1)*s - 2p + d*(k-1) + 1 + op, op (the
 * output padding) in [0, max(s, d)) extending the high end.  Written here as
 * a sum per output element: the i that reach q through tap k are those with
 * q + p - k*d divisible by s.
 */

static int64_t extent_t(int64_t in, int k, int s, int p, int op, int d) {
  return (in - 1) * s - 2 * (int64_t)p + (int64_t)d * (k - 1) + 1 + op;
}

int oracle_convT_out_dims(int D, int H, int W, int kD, int kH, int kW,
                          const int stride[3], const int pad[3],
                          const int out_pad[3], const int dil[3], int out[3]) {
  const int in[3] = {D, H, W};
  const int k[3] = {kD, kH, kW};
  for (int i = 0; i < 3; ++i) {
    if (in[i] <= 0 || k[i] <= 0 || stride[i] <= 0 || dil[i] <= 0 ||
        pad[i] < 0 || out_pad[i] < 0)
      return -1;
    if (out_pad[i] >= stride[i] && out_pad[i] >= dil[i]) return -1;
    int64_t e = extent_t(in[i], k[i], stride[i], pad[i], out_pad[i], dil[i]);
    if (e <= 0 || e > 0x7fffffff) return -1;
    out[i] = (int)e;
  }
  return 0;
}

typedef struct {
  int N, D, H, W, Ci, Co, kD, kH, kW, G;
  int Qd, Qh, Qw;
  int s[3], p[3], d[3];
} tshape_t;

static int make_tshape(tshape_t* t, int N, int D, int H, int W, int Cin,
                       int Cout, int kD, int kH, int kW, const int stride[3],
                       const int pad[3], const int out_pad[3],
                       const int dil[3], int groups) {
  int out[3];
  if (N <= 0 || Cin <= 0 || Cout <= 0 || groups <= 0) return -1;
  if (Cin % groups || Cout % groups) return -1;
  if (oracle_convT_out_dims(D, H, W, kD, kH, kW, stride, pad, out_pad, dil,
                            out))
    return -1;
  t->N = N; t->D = D; t->H = H; t->W = W; t->Ci = Cin; t->Co = Cout;
  t->kD = kD; t->kH = kH; t->kW = kW; t->G = groups;
  t->Qd = out[0]; t->Qh = out[1]; t->Qw = out[2];
  for (int i = 0; i < 3; ++i) {
    t->s[i] = stride[i]; t->p[i] = pad[i]; t->d[i] = dil[i];
  }
  return 0;
}

/* The input index i that reaches output q through tap k, or -1. */
static int64_t src_index(int64_t q, int k, int s, int p, int d, int64_t in) {
  int64_t num = q + p - (int64_t)k * d;
  if (num < 0 || num % s) return -1;
  num /= s;
  return num < in ? num : -1;
}

#define ORACLE_TPOINT_BODY(XAT, WAT)                                         \
  do {                                                                       \
    const int Cig = t->Ci / t->G, Cog = t->Co / t->G;                        \
    const int g = c / Cog, cl = c - g * Cog;                                 \
    double acc = 0.0, mag = 0.0;                                             \
    for (int kd = 0; kd < t->kD; ++kd) {                                     \
      int64_t id = src_index(qd, kd, t->s[0], t->p[0], t->d[0], t->D);       \
      if (id < 0) continue;                                                  \
      for (int kh = 0; kh < t->kH; ++kh) {                                   \
        int64_t ih = src_index(qh, kh, t->s[1], t->p[1], t->d[1], t->H);     \
        if (ih < 0) continue;                                                \
        for (int kw = 0; kw < t->kW; ++kw) {                                 \
          int64_t iw = src_index(qw, kw, t->s[2], t->p[2], t->d[2], t->W);   \
          if (iw < 0) continue;                                              \
          int64_t xb = ((((int64_t)n * t->D + id) * t->H + ih) * t->W + iw)  \
                       * t->Ci + (int64_t)g * Cig;                           \
          for (int ci = 0; ci < Cig; ++ci) {                                 \
            int64_t wi = (((((int64_t)g * Cig + ci) * t->kD + kd) * t->kH + kh) \
                          * t->kW + kw) * Cog + cl;                          \
            double v = XAT(xb + ci) * WAT(wi);                               \
            acc += v;                                                        \
            mag += fabs(v);                                                  \
          }                                                                  \
        }                                                                    \
      }                                                                      \
    }                                                                        \
    *py = acc;                                                               \
    *ps = mag;                                                               \
  } while (0)

static void tpoint_f64(const tshape_t* t, const double* x, const double* w,
                       int n, int qd, int qh, int qw, int c, double* py,
                       double* ps) {
#define XD(i) x[i]
#define WD(i) w[i]
  ORACLE_TPOINT_BODY(XD, WD);
#undef XD
#undef WD
}

static void tpoint_raw(const tshape_t* t, const void* x, const void* w,
                       int dtype, int n, int qd, int qh, int qw, int c,
                       double* py, double* ps) {
#define XR(i) load_elem(x, i, dtype)
#define WR(i) load_elem(w, i, dtype)
  ORACLE_TPOINT_BODY(XR, WR);
#undef XR
#undef WR
}

/* Full output of the transposed convolution.  x: [N,D,H,W,Cin]; w:
 * [Cin,kD,kH,kW,Cout/G]; y and s: [N,Qd,Qh,Qw,Cout] doubles.  Returns 0, -1
 * (shape), -2 (dtype) or -3 (out of host memory). */
int oracle_conv_transpose(const void* x, const void* w, int dtype, int N,
                          int D, int H, int W, int Cin, int Cout, int kD,
                          int kH, int kW, const int stride[3],
                          const int pad[3], const int out_pad[3],
                          const int dil[3], int groups, double* y, double* s) {
  tshape_t ts;
  if (dtype < 0 || dtype > 2) return -2;
  if (make_tshape(&ts, N, D, H, W, Cin, Cout, kD, kH, kW, stride, pad, out_pad,
                  dil, groups))
    return -1;
  int64_t nx = (int64_t)N * D * H * W * Cin;
  int64_t nw = (int64_t)Cin * kD * kH * kW * (Cout / groups);
  double* xd = decode_all(x, nx, dtype);
  double* wd = decode_all(w, nw, dtype);
  if (!xd || !wd) { free(xd); free(wd); return -3; }
  const tshape_t* t = &ts;
#pragma omp parallel for collapse(3) schedule(dynamic, 1)
  for (int n = 0; n < ts.N; ++n)
    for (int qd = 0; qd < ts.Qd; ++qd)
      for (int qh = 0; qh < ts.Qh; ++qh)
        for (int qw = 0; qw < t->Qw; ++qw)
          for (int c = 0; c < t->Co; ++c) {
            int64_t q = ((((int64_t)n * t->Qd + qd) * t->Qh + qh) * t->Qw + qw)
                        * t->Co + c;
            tpoint_f64(t, xd, wd, n, qd, qh, qw, c, &y[q], &s[q]);
          }
  free(xd);
  free(wd);
  return 0;
}

/* Selected outputs (flat indices into [N,Qd,Qh,Qw,Cout]), read in the storage
 * type.  Returns 0, -1, -2 or -4 (an index out of range). */
int oracle_conv_transpose_points(const void* x, const void* w, int dtype,
                                 int N, int D, int H, int W, int Cin, int Cout,
                                 int kD, int kH, int kW, const int stride[3],
                                 const int pad[3], const int out_pad[3],
                                 const int dil[3], int groups,
                                 const int64_t* idx, int64_t npts, double* y,
                                 double* s) {
  tshape_t ts;
  if (dtype < 0 || dtype > 2) return -2;
  if (make_tshape(&ts, N, D, H, W, Cin, Cout, kD, kH, kW, stride, pad, out_pad,
                  dil, groups))
    return -1;
  int64_t total = (int64_t)ts.N * ts.Qd * ts.Qh * ts.Qw * ts.Co;
  for (int64_t i = 0; i < npts; ++i)
    if (idx[i] < 0 || idx[i] >= total) return -4;
  const tshape_t* t = &ts;
#pragma omp parallel for schedule(dynamic, 64)
  for (int64_t i = 0; i < npts; ++i) {
    int64_t q = idx[i];
    int c = (int)(q % t->Co); q /= t->Co;
    int qw = (int)(q % t->Qw); q /= t->Qw;
    int qh = (int)(q % t->Qh); q /= t->Qh;
    int qd = (int)(q % t->Qd); q /= t->Qd;
    int n = (int)q;
    tpoint_raw(t, x, w, dtype, n, qd, qh, qw, c, &y[i], &s[i]);
  }
  return 0;
}

/* ---- weight gradient ------------------------------------------------------
 *
 * The gradient of the forward pass above with respect to its weights, given
 * the gradient dy of its output (the third of the convolution's three passes;
 * the data gradient is the transposed convolution above):
 *
 *   dw[o, kd, kh, kw, c] = sum over n, od, oh, ow of
 *       dy[n, od, oh, ow, o] * x[n, od*sd - pd + kd*dd, oh*sh - ph + kh*dh,
 *                                ow*sw - pw + kw*dw, g*Cg + c]
 *
 * with g = o / Og, x = 0 outside the input, padding p_lo below (the index
 * origin) and the output extent fixed by p_lo + p_hi as in the forward pass.
 * Written as the plain sum per weight element; S = sum |dy * x| alongside.
 */
int oracle_conv_wgrad(const void* x, const void* dy, int dtype, int N, int D,
                      int H, int W, int C, int O, int kD, int kH, int kW,
                      const int stride[3], const int pad_lo[3],
                      const int pad_hi[3], const int dil[3], int groups,
                      double* dw, double* s) {
  shape_t sh;
  if (dtype < 0 || dtype > 2) return -2;
  if (make_shape(&sh, N, D, H, W, C, O, kD, kH, kW, stride, pad_lo, pad_hi, dil,
                 groups, 0))
    return -1;
  int64_t nx = (int64_t)N * D * H * W * C;
  int64_t ny = (int64_t)N * sh.Do * sh.Ho * sh.Wo * O;
  double* xd = decode_all(x, nx, dtype);
  double* yd = decode_all(dy, ny, dtype);
  if (!xd || !yd) { free(xd); free(yd); return -3; }
  const shape_t* t = &sh;
  const int Cg = C / groups, Og = O / groups;
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
  for (int o = 0; o < O; ++o)
    for (int kd = 0; kd < kD; ++kd)
      for (int kh = 0; kh < t->kH; ++kh)
        for (int kw = 0; kw < t->kW; ++kw)
          for (int c = 0; c < Cg; ++c) {
            const int g = o / Og;
            double acc = 0.0, mag = 0.0;
            for (int n = 0; n < t->N; ++n)
              for (int od = 0; od < t->Do; ++od) {
                int64_t id = (int64_t)od * t->s[0] - t->p[0] + (int64_t)kd * t->d[0];
                if (id < 0 || id >= t->D) continue;
                for (int oh = 0; oh < t->Ho; ++oh) {
                  int64_t ih = (int64_t)oh * t->s[1] - t->p[1] + (int64_t)kh * t->d[1];
                  if (ih < 0 || ih >= t->H) continue;
                  for (int ow = 0; ow < t->Wo; ++ow) {
                    int64_t iw = (int64_t)ow * t->s[2] - t->p[2] + (int64_t)kw * t->d[2];
                    if (iw < 0 || iw >= t->W) continue;
                    double gy = yd[((((int64_t)n * t->Do + od) * t->Ho + oh) * t->Wo + ow) * t->O + o];
                    double xv = xd[((((int64_t)n * t->D + id) * t->H + ih) * t->W + iw) * t->C +
                                   (int64_t)g * Cg + c];
                    acc += gy * xv;
                    mag += fabs(gy * xv);
                  }
                }
              }
            int64_t q = ((((int64_t)o * kD + kd) * t->kH + kh) * t->kW + kw) * Cg + c;
            dw[q] = acc;
            s[q] = mag;
          }
  free(xd);
  free(yd);
  return 0;
}

int oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

void oracle_set_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}
