/*
 * conv3d_oracle.c -- plain fp64 direct 3D convolution (cross-correlation).
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the oracle that the CUDA path is
 * checked against.  Only tests/, __graft_entry__.smoke() and the CPU-baseline
 * leg of bench.py may load it.  It shares no code, header, table or helper
 * with the CUDA library, and it is deliberately slow and literal.
 *
 * What it computes (engineering.drawthings.ai, "Metal conv3d" post: the
 * implicit-GEMM conv3d reaches the result of a plain 3D convolution, only
 * faster; "Video VAE" section of the Qwen Image post: causal 3D convolution in
 * which the frames before the first one are padding):
 *
 *   y[n,to,ho,wo,co] = bias[co] + residual[n,to,ho,wo,co]
 *     + sum_{it<kt} sum_{ih<kh} sum_{iw<kw} sum_{ci<Cin}
 *         w[co,it,ih,iw,ci] * Xpad[n, to*st+it-pf, ho*sh+ih-ph, wo*sw+iw-pw, ci]
 *
 * Layouts: x is NDHWC [N,D,H,W,Cin]; w is [Cout,kt,kh,kw,Cin]; y and residual
 * are [N,Do,Ho,Wo,Cout].  Xpad is x extended by padding:
 *   - spatially: 0 outside [0,H) x [0,W);
 *   - temporally, mode 0 (zero):            pf = pb = pt, 0 outside [0,D);
 *   - temporally, mode 1 (causal replicate): pf = kt-1, pb = 0, frames f<0
 *                                            read frame 0;
 *   - temporally, mode 2 (causal zero):      pf = kt-1, pb = 0, frames f<0
 *                                            are 0 (the Wan first-frame rule);
 *   - temporally, mode 3 (causal, cached):   pf = kt-1, pb = 0, frames f<0
 *                                            are the cached frames of the
 *                                            previous chunk, prev[n, kt-1+f]
 *                                            (prev is [N, kt-1, H, W, Cin]).
 * Do = (D + pf + pb - kt)/st + 1, Ho = (H + 2ph - kh)/sh + 1,
 * Wo = (W + 2pw - kw)/sw + 1.
 *
 * Inputs are the raw 16-bit patterns (bf16 or fp16) that the GPU is given;
 * they are decoded exactly to double.  The sum is accumulated in double and
 * NOT rounded to the 16-bit output type.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <string.h>

#define ORACLE_F16 0
#define ORACLE_BF16 1

/* bf16 is the top half of an IEEE binary32: widen and reinterpret. */
static double oracle_bf16_to_double(uint16_t h) {
  uint32_t u = ((uint32_t)h) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* IEEE 754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
static double oracle_f16_to_double(uint16_t h) {
  int sign = (h >> 15) & 1;
  int e = (h >> 10) & 0x1f;
  int m = h & 0x3ff;
  double v;
  if (e == 0) {
    v = ldexp((double)m, -24); /* subnormal: m * 2^-14 * 2^-10 */
  } else if (e == 31) {
    v = (m == 0) ? INFINITY : NAN;
  } else {
    v = ldexp((double)(1024 + m), e - 25); /* (1 + m/1024) * 2^(e-15) */
  }
  return sign ? -v : v;
}

static double oracle_decode(uint16_t h, int dtype) {
  return dtype == ORACLE_BF16 ? oracle_bf16_to_double(h) : oracle_f16_to_double(h);
}

/* Exposed so the tests can pin the decoders against numpy for all 65536 codes. */
void oracle_decode16(const uint16_t* in, double* out, int64_t n, int dtype) {
  for (int64_t i = 0; i < n; ++i) out[i] = oracle_decode(in[i], dtype);
}

/* Output extents.  Returns 0 on success, -1 when the problem is empty or
 * ill-formed.  out[0..2] = Do, Ho, Wo. */
int oracle_output_shape(int D, int H, int W, int kt, int kh, int kw, int st, int sh, int sw,
                        int pt, int ph, int pw, int tpad_mode, int* out) {
  int pf, pb;
  if (tpad_mode == 0) {
    pf = pt;
    pb = pt;
  } else {
    pf = kt - 1;
    pb = 0;
  }
  if (st <= 0 || sh <= 0 || sw <= 0) return -1;
  int nd = D + pf + pb - kt, nh = H + 2 * ph - kh, nw = W + 2 * pw - kw;
  if (nd < 0 || nh < 0 || nw < 0) return -1;
  out[0] = nd / st + 1;
  out[1] = nh / sh + 1;
  out[2] = nw / sw + 1;
  return 0;
}

/*
 * Evaluate the definition above at the output pixels listed in rows[] (each a
 * flat index m = ((n*Do + to)*Ho + ho)*Wo + wo), all Cout channels each, and
 * write y_out[r*Cout + co].  rows == NULL means every output pixel in order.
 * bias and residual may be NULL (treated as 0).  The residual, when given, is
 * indexed by the same m.  OpenMP splits the list of pixels; each output value
 * is one sequential sum in the fixed order (it, ih, iw, ci).
 * Returns 0, or -1 on an ill-formed problem.
 */
int oracle_conv3d_f64(const uint16_t* x, const uint16_t* prev, const uint16_t* w,
                      const uint16_t* bias, const uint16_t* residual, int dtype, int N, int Cin,
                      int D, int H, int W, int Cout, int kt, int kh, int kw, int st, int sh, int sw,
                      int pt, int ph, int pw, int tpad_mode, const int64_t* rows, int64_t n_rows,
                      double* y_out) {
  int od[3];
  if (oracle_output_shape(D, H, W, kt, kh, kw, st, sh, sw, pt, ph, pw, tpad_mode, od) != 0)
    return -1;
  if (tpad_mode < 0 || tpad_mode > 3) return -1;
  if (tpad_mode == 3 && prev == NULL && kt > 1) return -1;
  const int Do = od[0], Ho = od[1], Wo = od[2];
  const int pf = (tpad_mode == 0) ? pt : kt - 1;
  const int64_t M = (int64_t)N * Do * Ho * Wo;
  const int64_t count = rows ? n_rows : M;

#pragma omp parallel for schedule(dynamic, 16)
  for (int64_t r = 0; r < count; ++r) {
    const int64_t m = rows ? rows[r] : r;
    if (m < 0 || m >= M) continue;
    int64_t q = m;
    const int wo = (int)(q % Wo); q /= Wo;
    const int ho = (int)(q % Ho); q /= Ho;
    const int to = (int)(q % Do); q /= Do;
    const int n = (int)q;
    for (int co = 0; co < Cout; ++co) {
      double acc = 0.0;
      for (int it = 0; it < kt; ++it) {
        int f = to * st + it - pf;
        const uint16_t* src = x;          /* frames of x, or of prev   */
        int64_t src_frames = D;
        if (f < 0) {
          if (tpad_mode == 1) {
            f = 0;                        /* causal replicate: frame 0 */
          } else if (tpad_mode == 3) {
            src = prev;                   /* cached previous frames    */
            src_frames = kt - 1;
            f = kt - 1 + f;
          } else {
            continue;                     /* zero / causal zero        */
          }
        } else if (f >= D) {
          continue;                       /* back padding is zero      */
        }
        for (int ih = 0; ih < kh; ++ih) {
          const int hi = ho * sh + ih - ph;
          if (hi < 0 || hi >= H) continue;
          for (int iw = 0; iw < kw; ++iw) {
            const int wi = wo * sw + iw - pw;
            if (wi < 0 || wi >= W) continue;
            const uint16_t* xp = src + ((((int64_t)n * src_frames + f) * H + hi) * W + wi) * Cin;
            const uint16_t* wp = w + ((((int64_t)co * kt + it) * kh + ih) * kw + iw) * Cin;
            for (int ci = 0; ci < Cin; ++ci)
              acc += oracle_decode(wp[ci], dtype) * oracle_decode(xp[ci], dtype);
          }
        }
      }
      if (bias) acc += oracle_decode(bias[co], dtype);
      if (residual) acc += oracle_decode(residual[m * Cout + co], dtype);
      y_out[r * Cout + co] = acc;
    }
  }
  return 0;
}

/* Number of threads OpenMP will use for the next parallel region. */
#ifdef _OPENMP
#include <omp.h>
int oracle_num_threads(void) { return omp_get_max_threads(); }
#else
int oracle_num_threads(void) { return 1; }
#endif

/*
 * GroupNorm followed by SiLU, the normalisation and activation in front of
 * every decoder convolution (stable-diffusion.cpp discussion "Exe Heavy
 * Metal": a GROUP_NORM kernel; news.bugfactory.tech: a fused GroupNorm + SiLU
 * kernel).  Standard GroupNorm: for sample n (and, with per_frame, frame d)
 * and group g (channels [g*C/G, (g+1)*C/G)), over every element of the group:
 *   mu = mean(x), var = mean((x - mu)^2)       (biased variance, two passes)
 *   z  = (x - mu) / sqrt(var + eps) * gamma[c] + beta[c]
 *   y  = z / (1 + exp(-z))                      (SiLU; silu == 0 returns z)
 * x is [N, D, H, W, C] (16-bit patterns); gamma, beta are [C] (16-bit, may be
 * NULL for 1 and 0); y is fp64, unrounded.  Returns 0, or -1 if C % G != 0.
 */
int oracle_groupnorm_silu_f64(const uint16_t* x, const uint16_t* gamma, const uint16_t* beta,
                              int dtype, int N, int D, int H, int W, int C, int G,
                              int per_frame, double eps, int silu, double* y) {
  if (G <= 0 || C % G != 0) return -1;
  const int cg = C / G;
  const int64_t pixels = (int64_t)D * H * W;
  const int sets = per_frame ? N * D : N;             /* statistic sets per group */
  const int64_t set_pixels = per_frame ? (int64_t)H * W : pixels;
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
  for (int s = 0; s < sets; ++s) {
    for (int g = 0; g < G; ++g) {
      const int64_t p0 = (int64_t)s * set_pixels;      /* first pixel of the set */
      double sum = 0.0;
      for (int64_t p = 0; p < set_pixels; ++p)
        for (int j = 0; j < cg; ++j) sum += oracle_decode(x[(p0 + p) * C + g * cg + j], dtype);
      const double count = (double)set_pixels * cg;
      const double mu = sum / count;
      double ss = 0.0;
      for (int64_t p = 0; p < set_pixels; ++p)
        for (int j = 0; j < cg; ++j) {
          const double d = oracle_decode(x[(p0 + p) * C + g * cg + j], dtype) - mu;
          ss += d * d;
        }
      const double rstd = 1.0 / sqrt(ss / count + eps);
      for (int64_t p = 0; p < set_pixels; ++p)
        for (int j = 0; j < cg; ++j) {
          const int c = g * cg + j;
          const double ga = gamma ? oracle_decode(gamma[c], dtype) : 1.0;
          const double be = beta ? oracle_decode(beta[c], dtype) : 0.0;
          const int64_t i = (p0 + p) * C + c;
          const double z = (oracle_decode(x[i], dtype) - mu) * rstd * ga + be;
          y[i] = silu ? z / (1.0 + exp(-z)) : z;
        }
    }
  }
  return 0;
}

/*
 * Backward pass of the convolution above (the pages' on-device LoRA/LoCon
 * fine-tuning trains convolution layers: engineering.drawthings.ai, LoRA
 * post).  Both are the adjoints of the forward definition, written as the
 * same loop with the accumulation reversed: every forward product
 *     w[co,it,ih,iw,ci] * Xpad[n, f, hi, wi, ci]   (f after the padding rule)
 * that lands in y[n,to,ho,wo,co] sends dy[n,to,ho,wo,co] * w[...] to
 * dx[n, f, hi, wi, ci] and dy * Xpad[...] to dw[co,it,ih,iw,ci].  Taps that
 * read zero padding contribute nothing; with causal replicate padding the
 * frames before the first are frame 0, so their gradient lands on frame 0.
 *   dx [N,D,H,W,Cin], dw [Cout,kt,kh,kw,Cin], dbias [Cout] = sum of dy.
 * dy holds 16-bit patterns of y's shape; outputs are fp64 and unrounded.
 * Serial loops (the scatter into dx would race under threads).
 */
int oracle_conv3d_backward_f64(const uint16_t* x, const uint16_t* w, const uint16_t* dy,
                               int dtype, int N, int Cin, int D, int H, int W, int Cout, int kt,
                               int kh, int kw, int st, int sh, int sw, int pt, int ph, int pw,
                               int tpad_mode, double* dx, double* dw, double* dbias) {
  int od[3];
  if (tpad_mode < 0 || tpad_mode > 2) return -1;
  if (oracle_output_shape(D, H, W, kt, kh, kw, st, sh, sw, pt, ph, pw, tpad_mode, od) != 0)
    return -1;
  const int Do = od[0], Ho = od[1], Wo = od[2];
  const int pf = (tpad_mode == 0) ? pt : kt - 1;
  if (dx) memset(dx, 0, sizeof(double) * (size_t)N * D * H * W * Cin);
  if (dw) memset(dw, 0, sizeof(double) * (size_t)Cout * kt * kh * kw * Cin);
  if (dbias) memset(dbias, 0, sizeof(double) * (size_t)Cout);
  for (int n = 0; n < N; ++n)
    for (int to = 0; to < Do; ++to)
      for (int ho = 0; ho < Ho; ++ho)
        for (int wo = 0; wo < Wo; ++wo) {
          const int64_t m = (((int64_t)n * Do + to) * Ho + ho) * Wo + wo;
          for (int co = 0; co < Cout; ++co) {
            const double g = oracle_decode(dy[m * Cout + co], dtype);
            if (dbias) dbias[co] += g;
            for (int it = 0; it < kt; ++it) {
              int f = to * st + it - pf;
              if (f < 0) {
                if (tpad_mode == 1) f = 0;
                else continue;
              }
              if (f >= D) continue;
              for (int ih = 0; ih < kh; ++ih) {
                const int hi = ho * sh + ih - ph;
                if (hi < 0 || hi >= H) continue;
                for (int iw = 0; iw < kw; ++iw) {
                  const int wi = wo * sw + iw - pw;
                  if (wi < 0 || wi >= W) continue;
                  const int64_t xo = ((((int64_t)n * D + f) * H + hi) * W + wi) * Cin;
                  const int64_t wo_ = ((((int64_t)co * kt + it) * kh + ih) * kw + iw) * Cin;
                  for (int ci = 0; ci < Cin; ++ci) {
                    if (dx) dx[xo + ci] += g * oracle_decode(w[wo_ + ci], dtype);
                    if (dw) dw[wo_ + ci] += g * oracle_decode(x[xo + ci], dtype);
                  }
                }
              }
            }
          }
        }
  return 0;
}

/*
 * The adjoints of the cached-frames chunk mode (mode 3; Qwen Image post,
 * "Video VAE": the frames before a chunk are the previous chunk's last kt-1
 * frames): the same reversed forward loop, in which a tap that reads frame
 * f < 0 reads prev[n, kt-1+f], so its product sends dy * w to
 * dprev[n, kt-1+f] and dy * prev[...] to dw.
 *   dx [N,D,H,W,Cin], dprev [N,kt-1,H,W,Cin], dw [Cout,kt,kh,kw,Cin], dbias [Cout].
 * Serial loops, fp64, unrounded; any output pointer may be NULL.
 */
int oracle_conv3d_backward_cached_f64(const uint16_t* x, const uint16_t* prev, const uint16_t* w,
                                      const uint16_t* dy, int dtype, int N, int Cin, int D, int H,
                                      int W, int Cout, int kt, int kh, int kw, int st, int sh,
                                      int sw, int ph, int pw, double* dx, double* dprev,
                                      double* dw, double* dbias) {
  int od[3];
  if (oracle_output_shape(D, H, W, kt, kh, kw, st, sh, sw, 0, ph, pw, 3, od) != 0) return -1;
  if (kt > 1 && prev == NULL) return -1;
  const int Do = od[0], Ho = od[1], Wo = od[2];
  const int pf = kt - 1;
  const int P = kt - 1; /* cached frames per sample */
  if (dx) memset(dx, 0, sizeof(double) * (size_t)N * D * H * W * Cin);
  if (dprev && P > 0) memset(dprev, 0, sizeof(double) * (size_t)N * P * H * W * Cin);
  if (dw) memset(dw, 0, sizeof(double) * (size_t)Cout * kt * kh * kw * Cin);
  if (dbias) memset(dbias, 0, sizeof(double) * (size_t)Cout);
  for (int n = 0; n < N; ++n)
    for (int to = 0; to < Do; ++to)
      for (int ho = 0; ho < Ho; ++ho)
        for (int wo = 0; wo < Wo; ++wo) {
          const int64_t m = (((int64_t)n * Do + to) * Ho + ho) * Wo + wo;
          for (int co = 0; co < Cout; ++co) {
            const double g = oracle_decode(dy[m * Cout + co], dtype);
            if (dbias) dbias[co] += g;
            for (int it = 0; it < kt; ++it) {
              const int f = to * st + it - pf;
              if (f >= D) continue;
              /* the frame read: x[n, f], or the cached prev[n, P + f] */
              const uint16_t* src = f < 0 ? prev : x;
              double* dsrc = f < 0 ? dprev : dx;
              const int64_t frame = f < 0 ? (int64_t)n * P + (P + f) : (int64_t)n * D + f;
              for (int ih = 0; ih < kh; ++ih) {
                const int hi = ho * sh + ih - ph;
                if (hi < 0 || hi >= H) continue;
                for (int iw = 0; iw < kw; ++iw) {
                  const int wi = wo * sw + iw - pw;
                  if (wi < 0 || wi >= W) continue;
                  const int64_t xo = ((frame * H + hi) * W + wi) * Cin;
                  const int64_t wo_ = ((((int64_t)co * kt + it) * kh + ih) * kw + iw) * Cin;
                  for (int ci = 0; ci < Cin; ++ci) {
                    if (dsrc) dsrc[xo + ci] += g * oracle_decode(w[wo_ + ci], dtype);
                    if (dw) dw[wo_ + ci] += g * oracle_decode(src[xo + ci], dtype);
                  }
                }
              }
            }
          }
        }
  return 0;
}

/*
 * The same two adjoints, evaluated one element at a time for large problems
 * whose full backward the serial loop above cannot finish quickly.  Each
 * element is the plain sum that defines it, over every forward product it
 * receives:
 *   dx[n,f,hi,wi,ci] = sum over (to, it, ih, iw, co) with src(to,it) == f,
 *                      to*st+it-pf mapped by the padding rule, ho*sh+ih-ph == hi
 *                      and wo*sw+iw-pw == wi, of dy[n,to,ho,wo,co] * w[co,it,ih,iw,ci];
 *   dw[co,it,ih,iw,ci] = sum over (n, to, ho, wo) whose tap reads a real pixel
 *                      of dy[n,to,ho,wo,co] * x[n, src(to,it), ho*sh+ih-ph, wo*sw+iw-pw, ci].
 * pixels: flat input-pixel indices ((n*D + f)*H + hi)*W + wi; dx_out [n_pix][Cin].
 * entries: flat indices into dw [Cout,kt,kh,kw,Cin]; dw_out [n_entries].
 * Elements are independent, so the loops over them run in parallel threads.
 */
static int oracle_source_frame(int to, int it, int st, int pf, int D, int tpad_mode) {
  int f = to * st + it - pf;
  if (f < 0) {
    if (tpad_mode != 1) return -1;
    f = 0;
  }
  return f < D ? f : -1;
}

int oracle_conv3d_dx_at_f64(const uint16_t* w, const uint16_t* dy, int dtype, int N, int Cin,
                            int D, int H, int W, int Cout, int kt, int kh, int kw, int st, int sh,
                            int sw, int pt, int ph, int pw, int tpad_mode, const int64_t* pixels,
                            int64_t n_pix, double* dx_out) {
  int od[3];
  if (tpad_mode < 0 || tpad_mode > 2) return -1;
  if (oracle_output_shape(D, H, W, kt, kh, kw, st, sh, sw, pt, ph, pw, tpad_mode, od) != 0)
    return -1;
  const int Do = od[0], Ho = od[1], Wo = od[2];
  const int pf = (tpad_mode == 0) ? pt : kt - 1;
  for (int64_t q = 0; q < n_pix; ++q)
    if (pixels[q] < 0 || pixels[q] >= (int64_t)N * D * H * W) return -1;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t q = 0; q < n_pix; ++q) {
    const int64_t pix = pixels[q];
    const int wi = (int)(pix % W);
    const int hi = (int)((pix / W) % H);
    const int f = (int)((pix / ((int64_t)W * H)) % D);
    const int n = (int)(pix / ((int64_t)W * H * D));
    double* acc = dx_out + q * Cin;
    for (int ci = 0; ci < Cin; ++ci) acc[ci] = 0.0;
    for (int to = 0; to < Do; ++to)
      for (int it = 0; it < kt; ++it) {
        if (oracle_source_frame(to, it, st, pf, D, tpad_mode) != f) continue;
        for (int ih = 0; ih < kh; ++ih) {
          const int hs = hi + ph - ih;           /* = ho * sh */
          if (hs < 0 || hs % sh != 0 || hs / sh >= Ho) continue;
          const int ho = hs / sh;
          for (int iw = 0; iw < kw; ++iw) {
            const int ws = wi + pw - iw;         /* = wo * sw */
            if (ws < 0 || ws % sw != 0 || ws / sw >= Wo) continue;
            const int wo = ws / sw;
            const int64_t m = (((int64_t)n * Do + to) * Ho + ho) * Wo + wo;
            for (int co = 0; co < Cout; ++co) {
              const double g = oracle_decode(dy[m * Cout + co], dtype);
              const int64_t wo_ = ((((int64_t)co * kt + it) * kh + ih) * kw + iw) * Cin;
              for (int ci = 0; ci < Cin; ++ci) acc[ci] += g * oracle_decode(w[wo_ + ci], dtype);
            }
          }
        }
      }
  }
  return 0;
}

int oracle_conv3d_dw_at_f64(const uint16_t* x, const uint16_t* dy, int dtype, int N, int Cin,
                            int D, int H, int W, int Cout, int kt, int kh, int kw, int st, int sh,
                            int sw, int pt, int ph, int pw, int tpad_mode, const int64_t* entries,
                            int64_t n_entries, double* dw_out) {
  int od[3];
  if (tpad_mode < 0 || tpad_mode > 2) return -1;
  if (oracle_output_shape(D, H, W, kt, kh, kw, st, sh, sw, pt, ph, pw, tpad_mode, od) != 0)
    return -1;
  const int Do = od[0], Ho = od[1], Wo = od[2];
  const int pf = (tpad_mode == 0) ? pt : kt - 1;
  for (int64_t q = 0; q < n_entries; ++q)
    if (entries[q] < 0 || entries[q] >= (int64_t)Cout * kt * kh * kw * Cin) return -1;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t q = 0; q < n_entries; ++q) {
    int64_t e = entries[q];
    const int ci = (int)(e % Cin); e /= Cin;
    const int iw = (int)(e % kw); e /= kw;
    const int ih = (int)(e % kh); e /= kh;
    const int it = (int)(e % kt);
    const int co = (int)(e / kt);
    double acc = 0.0;
    for (int n = 0; n < N; ++n)
      for (int to = 0; to < Do; ++to) {
        const int f = oracle_source_frame(to, it, st, pf, D, tpad_mode);
        if (f < 0) continue;
        for (int ho = 0; ho < Ho; ++ho) {
          const int hi = ho * sh + ih - ph;
          if (hi < 0 || hi >= H) continue;
          for (int wo = 0; wo < Wo; ++wo) {
            const int wi = wo * sw + iw - pw;
            if (wi < 0 || wi >= W) continue;
            const int64_t m = (((int64_t)n * Do + to) * Ho + ho) * Wo + wo;
            const int64_t xo = ((((int64_t)n * D + f) * H + hi) * W + wi) * Cin + ci;
            acc += oracle_decode(dy[m * Cout + co], dtype) * oracle_decode(x[xo], dtype);
          }
        }
      }
    dw_out[q] = acc;
  }
  return 0;
}
