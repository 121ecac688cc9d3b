/*
 * Oracle for the Flash EQ-Linear layer -- TEST INFRASTRUCTURE ONLY.
 *
 * This file is a plain, slow, float64 CPU statement of what the layer computes.
 * It exists so the tests, the smoke check and the benchmark's CPU baseline can
 * compare the CUDA library against something obviously correct.  Nothing in the
 * product path may call it, and it shares no code with the CUDA sources: no
 * header, table, helper or constant generator.
 *
 * Source of the definitions ("Flash EQ-Linear" technical summary,
 * gist.science/ko/paper/2607.21271):
 *   - "Key insight": the EQ-Linear weight matrix is group-circulant, built by
 *     cyclically shifting and replicating one learnable parameter set; the layer
 *     is a circular operation over the group axis combined with a linear map over
 *     channels.
 *   - The operator written out (feature index c*T+t on the input, d*T+s on the
 *     output):  Y[n,d,s] = bias[d] + sum_{c,t} W[d,c,(t-s) mod T] * X[n,c,t].
 *   - "Algorithmic approach", items 1-3: DFT over the group axis, pointwise
 *     products per frequency, only the non-redundant half of the spectrum
 *     (conjugate symmetry), MAC count falling from NDC to about 2NDC/T.
 *   - "Specialisation for p4", bullet 3: six real GEMMs for T=4 (16/6 = 2.67x).
 *   - "Contributions", item 2: the method is exact (DFT invertibility plus the
 *     convolution theorem), up to floating-point rounding.
 *
 * The pages state the backward kernels exist ("Implementation", bullet 1) but
 * not their formulas; the three backward functions below are the gradients of
 * the forward definition, written out term by term.
 *
 * Layouts (all row-major, contiguous, float64):
 *   X   [N][C*T]   feature index c*T+t
 *   W   [D][C][T]
 *   bias[D]        (may be NULL: treated as zero)
 *   Y   [N][D*T]   feature index d*T+s
 *
 * Parity pins (tests that fix this oracle to something other than itself) live
 * in tests/test_oracle_pins.py: brute force against the explicitly replicated
 * dense matrix, cyclic-shift equivariance, numpy's FFT convolution theorem,
 * exact MAC counts, closed-form special cases and hand-worked values.
 */
#include <complex.h>
#include <math.h>
#include <stddef.h>
#include <stdint.h>

#ifndef M_PI
#define M_PI 3.14159265358979323846
#endif

static long wrap(long i, long T) { return ((i % T) + T) % T; }

#ifdef _OPENMP
#include <omp.h>
#endif

/* Threads of the parallel loops that follow (timing only; no effect on any
 * result, every loop writes disjoint outputs in a fixed order). */
void eqlo_set_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

/* Forward, the plain definition.  Returns the number of real multiply-adds. */
int64_t eqlo_forward(int T, int64_t N, int64_t C, int64_t D, const double* X, const double* W,
                     const double* bias, double* Y) {
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t d = 0; d < D; ++d) {
      for (int s = 0; s < T; ++s) {
        double acc = 0.0;
        for (int64_t c = 0; c < C; ++c) {
          for (int t = 0; t < T; ++t) {
            acc += W[(d * C + c) * T + wrap(t - s, T)] * X[n * C * T + c * T + t];
          }
        }
        Y[n * D * T + d * T + s] = acc + (bias ? bias[d] : 0.0);
      }
    }
  }
  return N * D * T * C * T;
}

/* The EQ-MLP block's activation, applied elementwise to a forward output:
 * GELU(y) = y * Phi(y) = 0.5 * y * (1 + erf(y / sqrt(2))), the exact (erf) form.
 * A pointwise function of each output feature commutes with the cyclic shift of
 * the group axis, so the block stays equivariant ("Key insight"; the pages'
 * network-level models are ViT/Swin, whose MLP blocks use this activation). */
void eqlo_gelu(int64_t n, double* y) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) y[i] = 0.5 * y[i] * (1.0 + erf(y[i] / sqrt(2.0)));
}

/* Gradient of the forward with respect to X:
 *   dX[n,c,t] = sum_{d,s} dY[n,d,s] * W[d,c,(t-s) mod T]. */
int64_t eqlo_backward_input(int T, int64_t N, int64_t C, int64_t D, const double* dY,
                            const double* W, double* dX) {
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t c = 0; c < C; ++c) {
      for (int t = 0; t < T; ++t) {
        double acc = 0.0;
        for (int64_t d = 0; d < D; ++d) {
          for (int s = 0; s < T; ++s) {
            acc += dY[n * D * T + d * T + s] * W[(d * C + c) * T + wrap(t - s, T)];
          }
        }
        dX[n * C * T + c * T + t] = acc;
      }
    }
  }
  return N * C * T * D * T;
}

/* Gradient with respect to W and bias:
 *   dW[d,c,u] = sum_{n,s} dY[n,d,s] * X[n,c,(s+u) mod T]
 *   dbias[d]  = sum_{n,s} dY[n,d,s]                  (dbias may be NULL). */
int64_t eqlo_backward_weight(int T, int64_t N, int64_t C, int64_t D, const double* X,
                             const double* dY, double* dW, double* dbias) {
#pragma omp parallel for schedule(static)
  for (int64_t d = 0; d < D; ++d) {
    for (int64_t c = 0; c < C; ++c) {
      for (int u = 0; u < T; ++u) {
        double acc = 0.0;
        for (int64_t n = 0; n < N; ++n) {
          for (int s = 0; s < T; ++s) {
            acc += dY[n * D * T + d * T + s] * X[n * C * T + c * T + wrap(s + u, T)];
          }
        }
        dW[(d * C + c) * T + u] = acc;
      }
    }
    if (dbias) {
      double acc = 0.0;
      for (int64_t n = 0; n < N; ++n)
        for (int s = 0; s < T; ++s) acc += dY[n * D * T + d * T + s];
      dbias[d] = acc;
    }
  }
  return N * D * C * T * T;
}

/* Sampled weight gradient: dW[d,c,:] only for the listed (d,c) pairs, written to
 * out[i*T + u].  Same sum as eqlo_backward_weight, one pair at a time. */
void eqlo_backward_weight_pairs(int T, int64_t N, int64_t C, int64_t D, const double* X,
                                const double* dY, int64_t npairs, const int64_t* pd,
                                const int64_t* pc, double* out) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < npairs; ++i) {
    const int64_t d = pd[i], c = pc[i];
    for (int u = 0; u < T; ++u) {
      double acc = 0.0;
      for (int64_t n = 0; n < N; ++n)
        for (int s = 0; s < T; ++s)
          acc += dY[n * D * T + d * T + s] * X[n * C * T + c * T + wrap(s + u, T)];
      out[i * T + u] = acc;
    }
  }
}

/*
 * The method's own route, step by step ("Algorithmic approach" items 1-3), in
 * float64 complex arithmetic, with a counter of real multiply-adds in the
 * per-frequency products:
 *   1. DFT of every length-T group vector: Xh[k] = sum_t x[t] e^{-2 pi i k t / T}
 *      and Wh[k] = sum_u w[u] e^{-2 pi i k u / T}.
 *   2. Because the operator correlates (index t-s), the per-frequency product is
 *      Yh[k] = sum_c conj(Wh[d,c,k]) * Xh[n,c,k]  (the correlation form of the
 *      convolution theorem).
 *   3. Only k = 0 .. floor(T/2) is computed (conjugate symmetry of real input);
 *      a real frequency (k = 0, and k = T/2 for even T) costs 1 real MAC per
 *      (n,d,c), a complex one costs 4.
 *   4. Inverse DFT over the full spectrum, the missing half filled in as
 *      Yh[T-k] = conj(Yh[k]), then the bias.
 * Returns the product-stage MAC count.
 */
int64_t eqlo_forward_spectral(int T, int64_t N, int64_t C, int64_t D, const double* X,
                              const double* W, const double* bias, double* Y) {
  const int K = T / 2 + 1; /* non-redundant frequencies 0..floor(T/2) */
  int64_t macs = 0;

#pragma omp parallel for schedule(static) reduction(+ : macs)
  for (int64_t n = 0; n < N; ++n) {
    double complex yh[64]; /* T <= 126 keeps K <= 64 */
    for (int64_t d = 0; d < D; ++d) {
      for (int k = 0; k < K; ++k) yh[k] = 0.0;
      for (int64_t c = 0; c < C; ++c) {
        for (int k = 0; k < K; ++k) {
          double complex xs = 0.0, ws = 0.0;
          for (int t = 0; t < T; ++t) {
            const double complex e = cexp(-2.0 * M_PI * I * (double)k * (double)t / (double)T);
            xs += X[n * C * T + c * T + t] * e;
            ws += W[(d * C + c) * T + t] * e;
          }
          if (k == 0 || 2 * k == T) {
            /* real frequency: both spectra are real here, one real MAC */
            yh[k] += creal(ws) * creal(xs);
            macs += 1;
          } else {
            /* complex frequency: conj(ws) * xs is four real MACs */
            yh[k] += conj(ws) * xs;
            macs += 4;
          }
        }
      }
      for (int s = 0; s < T; ++s) {
        double complex acc = 0.0;
        for (int k = 0; k < T; ++k) {
          const double complex yk = (k < K) ? yh[k] : conj(yh[T - k]);
          acc += yk * cexp(2.0 * M_PI * I * (double)k * (double)s / (double)T);
        }
        Y[n * D * T + d * T + s] = creal(acc) / (double)T + (bias ? bias[d] : 0.0);
      }
    }
  }
  return macs;
}

/*
 * The p4 transform pair of "Specialisation for p4" (T = 4), as real 4x4
 * matrices acting on one group vector.  Rows of the forward matrix F produce
 * (Re Xh0, Re Xh2, Re Xh1, Im Xh1) with Xh[k] = sum_t x[t] e^{-2 pi i k t/4};
 * the inverse G maps those four numbers back to x, using Xh3 = conj(Xh1).
 * Both are filled from the defining exponentials, not typed in, so the tests can
 * check that every entry lands on 0, +-1, +-1/2 or +-1/4 and that G F = I.
 */
void eqlo_p4_transform_matrices(double* F, double* G) {
  const int T = 4;
  for (int t = 0; t < T; ++t) {
    const double complex e0 = cexp(-2.0 * M_PI * I * 0.0 * t / T);
    const double complex e2 = cexp(-2.0 * M_PI * I * 2.0 * t / T);
    const double complex e1 = cexp(-2.0 * M_PI * I * 1.0 * t / T);
    F[0 * T + t] = creal(e0);
    F[1 * T + t] = creal(e2);
    F[2 * T + t] = creal(e1);
    F[3 * T + t] = cimag(e1);
  }
  /* x[s] = (1/4) sum_k Xh[k] e^{+2 pi i k s/4}; write it as a real combination of
   * (Re Xh0, Re Xh2, Re Xh1, Im Xh1). */
  for (int s = 0; s < T; ++s) {
    const double complex p1 = cexp(2.0 * M_PI * I * 1.0 * s / T);
    const double complex p2 = cexp(2.0 * M_PI * I * 2.0 * s / T);
    G[s * T + 0] = 1.0 / T;
    G[s * T + 1] = creal(p2) / T;
    /* Xh1 p1 + conj(Xh1) conj(p1) = 2 (Re Xh1 Re p1 - Im Xh1 Im p1) */
    G[s * T + 2] = 2.0 * creal(p1) / T;
    G[s * T + 3] = -2.0 * cimag(p1) / T;
  }
  /* cexp leaves round-off such as 6e-17 where the exact value is 0; snap each
   * entry to the nearest multiple of 1/4 when it is within 1e-12 of it.  The
   * tests then check exactness and G F = I on the snapped values. */
  for (int i = 0; i < T * T; ++i) {
    const double qf = nearbyint(F[i] * 4.0), qg = nearbyint(G[i] * 4.0);
    if (fabs(F[i] * 4.0 - qf) < 1e-12) F[i] = qf / 4.0;
    if (fabs(G[i] * 4.0 - qg) < 1e-12) G[i] = qg / 4.0;
  }
}

/*
 * Group-circulant convolution, the plain definition (the pages name equivariant
 * convolution as the natural next operator for the per-frequency method,
 * "Limitations and future work"; they give no formula).  Reading: the
 * EQ-Linear's group-circulant channel mixing at every tap of a KH x KW kernel,
 * stride 1, zero padding (ph, pw):
 *   Y[n][oy][ox][d*T+s] = bias[d] + sum_{i<KH, j<KW} sum_{c,t}
 *       Wc[i][j][d][c][(t-s) mod T] * X[n][oy+i-ph][ox+j-pw][c*T+t]
 * with X zero outside the H x Wd image.  A cyclic shift of every pixel's group
 * axis shifts the output's group axis the same way, as for the EQ-Linear, and
 * the operator commutes with translations away from the border.
 * Layouts: X [N][H][Wd][C*T], Wc [KH][KW][D][C][T], bias [D] or NULL,
 * Y [N][Ho][Wo][D*T] with Ho = H + 2 ph - KH + 1, Wo = Wd + 2 pw - KW + 1.
 * Returns the number of real multiply-adds taken inside the image.
 */
int64_t eqlo_conv_forward(int T, int64_t N, int64_t H, int64_t Wd, int64_t C, int64_t D,
                          int KH, int KW, int ph, int pw, const double* X, const double* Wc,
                          const double* bias, double* Y) {
  const int64_t Ho = H + 2 * ph - KH + 1, Wo = Wd + 2 * pw - KW + 1;
  if (Ho <= 0 || Wo <= 0) return 0;
  int64_t macs = 0;
#pragma omp parallel for collapse(2) schedule(static) reduction(+ : macs)
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t oy = 0; oy < Ho; ++oy) {
      for (int64_t ox = 0; ox < Wo; ++ox) {
        double* y = Y + ((n * Ho + oy) * Wo + ox) * D * T;
        for (int64_t d = 0; d < D; ++d) {
          for (int s = 0; s < T; ++s) {
            double acc = 0.0;
            for (int i = 0; i < KH; ++i) {
              const int64_t iy = oy + i - ph;
              if (iy < 0 || iy >= H) continue;
              for (int j = 0; j < KW; ++j) {
                const int64_t ix = ox + j - pw;
                if (ix < 0 || ix >= Wd) continue;
                const double* x = X + ((n * H + iy) * Wd + ix) * C * T;
                const double* w = Wc + (((int64_t)i * KW + j) * D + d) * C * T;
                for (int64_t c = 0; c < C; ++c)
                  for (int t = 0; t < T; ++t) acc += w[c * T + wrap(t - s, T)] * x[c * T + t];
                macs += C * T;
              }
            }
            y[d * T + s] = acc + (bias ? bias[d] : 0.0);
          }
        }
      }
    }
  }
  return macs;
}

/*
 * Gradients of the group-circulant convolution (the definition above,
 * differentiated term by term; taps outside the image contribute nothing):
 *   dX[n][y][x][c*T+t] = sum_{i,j,d,s} Wc[i][j][d][c][(t-s) mod T]
 *                                      * dY[n][y-i+ph][x-j+pw][d*T+s]
 *   dWc[i][j][d][c][u] = sum_{n,oy,ox,s} dY[n][oy][ox][d*T+s]
 *                                       * X[n][oy+i-ph][ox+j-pw][c*T + (s+u) mod T]
 *   dbias[d]           = sum_{n,oy,ox,s} dY[n][oy][ox][d*T+s]
 * dY is [N][Ho][Wo][D*T] with Ho = H + 2 ph - KH + 1, Wo = Wd + 2 pw - KW + 1.
 */
void eqlo_conv_backward_input(int T, int64_t N, int64_t H, int64_t Wd, int64_t C, int64_t D,
                              int KH, int KW, int ph, int pw, const double* dY, const double* Wc,
                              double* dX) {
  const int64_t Ho = H + 2 * ph - KH + 1, Wo = Wd + 2 * pw - KW + 1;
#pragma omp parallel for collapse(2) schedule(static)
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t y = 0; y < H; ++y) {
      for (int64_t x = 0; x < Wd; ++x) {
        double* dx = dX + ((n * H + y) * Wd + x) * C * T;
        for (int64_t c = 0; c < C; ++c) {
          for (int t = 0; t < T; ++t) {
            double acc = 0.0;
            for (int i = 0; i < KH; ++i) {
              const int64_t oy = y - i + ph;
              if (oy < 0 || oy >= Ho) continue;
              for (int j = 0; j < KW; ++j) {
                const int64_t ox = x - j + pw;
                if (ox < 0 || ox >= Wo) continue;
                const double* dy = dY + ((n * Ho + oy) * Wo + ox) * D * T;
                for (int64_t d = 0; d < D; ++d) {
                  const double* w = Wc + (((int64_t)i * KW + j) * D + d) * C * T + c * T;
                  for (int s = 0; s < T; ++s) acc += w[wrap(t - s, T)] * dy[d * T + s];
                }
              }
            }
            dx[c * T + t] = acc;
          }
        }
      }
    }
  }
}

void eqlo_conv_backward_weight(int T, int64_t N, int64_t H, int64_t Wd, int64_t C, int64_t D,
                               int KH, int KW, int ph, int pw, const double* X, const double* dY,
                               double* dWc, double* dbias) {
  const int64_t Ho = H + 2 * ph - KH + 1, Wo = Wd + 2 * pw - KW + 1;
#pragma omp parallel for collapse(3) schedule(static)
  for (int i = 0; i < KH; ++i) {
    for (int j = 0; j < KW; ++j) {
      for (int64_t d = 0; d < D; ++d) {
        for (int64_t c = 0; c < C; ++c) {
          for (int u = 0; u < T; ++u) {
            double acc = 0.0;
            for (int64_t n = 0; n < N; ++n)
              for (int64_t oy = 0; oy < Ho; ++oy) {
                const int64_t iy = oy + i - ph;
                if (iy < 0 || iy >= H) continue;
                for (int64_t ox = 0; ox < Wo; ++ox) {
                  const int64_t ix = ox + j - pw;
                  if (ix < 0 || ix >= Wd) continue;
                  const double* dy = dY + ((n * Ho + oy) * Wo + ox) * D * T + d * T;
                  const double* x = X + ((n * H + iy) * Wd + ix) * C * T + c * T;
                  for (int s = 0; s < T; ++s) acc += dy[s] * x[wrap(s + u, T)];
                }
              }
            dWc[((((int64_t)i * KW + j) * D + d) * C + c) * T + u] = acc;
          }
        }
      }
    }
  }
  for (int64_t d = 0; d < D; ++d) {
    double acc = 0.0;
    for (int64_t q = 0; q < N * Ho * Wo; ++q)
      for (int s = 0; s < T; ++s) acc += dY[q * D * T + d * T + s];
    dbias[d] = acc;
  }
}

/*
 * EQ-Linear over the dihedral group D4 (p4m: the four 90-degree rotations and
 * their compositions with a mirror), the reflection group the pages name as the
 * natural generalisation of the p4 method ("Limitations and future work"; no
 * formula is given).  Reading: the same group-circulant weight structure with
 * the cyclic shift replaced by the group law, i.e. a group cross-correlation
 * over the regular representation:
 *   Y[n][d*8+g] = bias[d] + sum_{c,h} W[d][c][g^-1 h] * X[n][c*8+h]
 * Group elements are indexed g = a + 4 b for r^a m^b (a = 0..3 quarter turns,
 * b = 1 with the mirror), with m r m = r^-1, so
 *   (r^a m^b)(r^c m^e) = r^(a + (-1)^b c) m^(b+e),   (r^a m^b)^-1 = r^(-(-1)^b a) m^b.
 * With W[d][c][u] = 0 for mirrored u and X zero on mirrored h, the rotation
 * outputs equal the cyclic T = 4 layer.  Returns the number of real
 * multiply-adds (N * D * C * 64).
 */
static int d4_mul(int g, int h) {
  const int a = g & 3, b = g >> 2, c = h & 3, e = h >> 2;
  const int rot = (a + (b ? -c : c)) & 3;
  return rot + 4 * (b ^ e);
}
static int d4_inv(int g) {
  const int a = g & 3, b = g >> 2;
  return (b ? a : ((4 - a) & 3)) + 4 * b;
}

int64_t eqlo_d4_forward(int64_t N, int64_t C, int64_t D, const double* X, const double* W,
                        const double* bias, double* Y) {
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t d = 0; d < D; ++d) {
      for (int g = 0; g < 8; ++g) {
        const int gi = d4_inv(g);
        double acc = 0.0;
        for (int64_t c = 0; c < C; ++c)
          for (int h = 0; h < 8; ++h) acc += W[(d * C + c) * 8 + d4_mul(gi, h)] * X[(n * C + c) * 8 + h];
        Y[(n * D + d) * 8 + g] = acc + (bias ? bias[d] : 0.0);
      }
    }
  }
  return N * D * C * 64;
}

/*
 * Gradients of the D4 layer (the definition above, differentiated term by term):
 *   dX[n][c*8+h] = sum_{d,g} W[d][c][g^-1 h] * dY[n][d*8+g]
 *   dW[d][c][u]  = sum_{n,g} dY[n][d*8+g] * X[n][c*8+g u]     (h = g u)
 *   dbias[d]     = sum_{n,g} dY[n][d*8+g]
 * Each returns the number of real multiply-adds (N * D * C * 64).
 */
int64_t eqlo_d4_backward_input(int64_t N, int64_t C, int64_t D, const double* dY,
                               const double* W, double* dX) {
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t c = 0; c < C; ++c) {
      for (int h = 0; h < 8; ++h) {
        double acc = 0.0;
        for (int64_t d = 0; d < D; ++d)
          for (int g = 0; g < 8; ++g)
            acc += W[(d * C + c) * 8 + d4_mul(d4_inv(g), h)] * dY[(n * D + d) * 8 + g];
        dX[(n * C + c) * 8 + h] = acc;
      }
    }
  }
  return N * D * C * 64;
}

int64_t eqlo_d4_backward_weight(int64_t N, int64_t C, int64_t D, const double* X,
                                const double* dY, double* dW, double* dbias) {
#pragma omp parallel for schedule(static)
  for (int64_t dc = 0; dc < D * C; ++dc) {
    const int64_t d = dc / C, c = dc % C;
    for (int u = 0; u < 8; ++u) {
      double acc = 0.0;
      for (int64_t n = 0; n < N; ++n)
        for (int g = 0; g < 8; ++g)
          acc += dY[(n * D + d) * 8 + g] * X[(n * C + c) * 8 + d4_mul(g, u)];
      dW[dc * 8 + u] = acc;
    }
  }
  for (int64_t d = 0; d < D; ++d) {
    double acc = 0.0;
    for (int64_t n = 0; n < N; ++n)
      for (int g = 0; g < 8; ++g) acc += dY[(n * D + d) * 8 + g];
    dbias[d] = acc;
  }
  return N * D * C * 64;
}
