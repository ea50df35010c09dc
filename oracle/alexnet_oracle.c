/*
 * alexnet_oracle.c -- plain CPU oracle for the AlexNet training hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  This file exists to check the CUDA library, not
 * to be used by it: only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg load it.  It shares no source, header, table or helper with
 * the CUDA library; the two never include or link each other.
 *
 * Arithmetic: every tensor is fp64 and every sum is accumulated in fp64, in
 * the plain order of the defining formula (direct nested loops, no blocking,
 * no fusion, no reordering).  OpenMP only splits independent outer loops
 * (images, output channels) across threads; each output is still summed by
 * one thread in the written order.
 *
 * Pages cited (by title, section, equation or listing):
 *   [S]  "ImageNet Classification with Deep Convolutional Neural Networks",
 *        the paper-graph-ui section-by-section summary page.
 *   [W]  "AlexNet and Deep CNNs" (fermi.ai wiki page).
 *   [P2] "AlexNet Part 2: Turning the Training Recipe into Testable Design
 *        Choices" (bloss0m paper-reading page).
 * Random numbers the method draws (dropout masks, crop offsets, flips, PCA
 * coefficients) come from Philox4x32-10, written here from its published
 * definition: J. Salmon, M. Moraes, R. Dror, D. Shaw, "Parallel Random
 * Numbers: As Easy as 1, 2, 3", SC'11, section 3.2 (the Philox S-box and key
 * schedule); normal deviates from G. Box and M. Muller, "A Note on the
 * Generation of Random Normal Deviates", 1958.
 *
 * Layouts (the same conventions the library documents for its parameter
 * blob, restated here independently):
 *   activations: NHWC, image-major, channels fastest.
 *   conv weight: [Cout][kh][kw][Cin/groups]; output channel o belongs to
 *                group o / (Cout/groups), which reads input channels
 *                g*(Cin/groups) ... (g+1)*(Cin/groups)-1.
 *   fc weight:   [out][in]; the FC6 input index is (h*W + w)*C + c, the
 *                H x W x C flattening of the last pooled map ([S] 3.4
 *                "Overall Architecture", Layer 6: 6x6x256 = 9216 inputs).
 *   parameter order: conv1.W conv1.b ... conv5.W conv5.b fc6.W fc6.b
 *                fc7.W fc7.b fc8.W fc8.b.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_API __attribute__((visibility("default")))

/* ------------------------------------------------------------------------ */
/* Philox4x32-10 (Salmon et al., SC'11, section 3.2).                        */
/* One round: two 32x32->64 multiplies of counter words 0 and 2 by the       */
/* multipliers, then the high halves are xor-ed with the other counter word  */
/* and a key word; the key is bumped by the Weyl constants between rounds.   */
/* ------------------------------------------------------------------------ */
static const uint32_t PHILOX_M0 = 0xD2511F53u;
static const uint32_t PHILOX_M1 = 0xCD9E8D57u;
static const uint32_t PHILOX_W0 = 0x9E3779B9u;
static const uint32_t PHILOX_W1 = 0xBB67AE85u;

ORACLE_API void oracle_philox4x32_10(const uint32_t ctr_in[4], const uint32_t key_in[2],
                                     uint32_t out[4]) {
  uint32_t c0 = ctr_in[0], c1 = ctr_in[1], c2 = ctr_in[2], c3 = ctr_in[3];
  uint32_t k0 = key_in[0], k1 = key_in[1];
  for (int round = 0; round < 10; ++round) {
    if (round > 0) {
      k0 += PHILOX_W0;
      k1 += PHILOX_W1;
    }
    uint64_t p0 = (uint64_t)PHILOX_M0 * (uint64_t)c0;
    uint64_t p1 = (uint64_t)PHILOX_M1 * (uint64_t)c2;
    uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
    uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
    uint32_t n0 = hi1 ^ c1 ^ k0;
    uint32_t n1 = lo1;
    uint32_t n2 = hi0 ^ c3 ^ k1;
    uint32_t n3 = lo0;
    c0 = n0; c1 = n1; c2 = n2; c3 = n3;
  }
  out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

static void philox_seeded(uint64_t seed, uint32_t a, uint32_t b, uint32_t c, uint32_t d,
                          uint32_t out[4]) {
  uint32_t ctr[4] = {a, b, c, d};
  uint32_t key[2] = {(uint32_t)(seed & 0xFFFFFFFFu), (uint32_t)(seed >> 32)};
  oracle_philox4x32_10(ctr, key, out);
}

/* Uniform on (0,1) from the top 24 bits of a word: (w>>8)*2^-24 + 2^-25.  */
static double word_to_open_unit(uint32_t w) {
  return (double)(w >> 8) * (1.0 / 16777216.0) + (1.0 / 33554432.0);
}

/* ------------------------------------------------------------------------ */
/* Convolution: [S] 3.4 "Overall Architecture" (layer shapes) and [W]        */
/* "Layer-by-layer structure" (stride/padding per layer).  Zero padding.     */
/* y[b,oh,ow,o] = bias[o] + sum_{kh,kw,ci} x[b, oh*s-p+kh, ow*s-p+kw,        */
/*                                          g*Cg+ci] * w[o,kh,kw,ci]         */
/* ------------------------------------------------------------------------ */
ORACLE_API int oracle_conv_out_size(int in, int k, int stride, int pad) {
  return (in + 2 * pad - k) / stride + 1;
}

ORACLE_API void oracle_conv_fwd(const double* x, int B, int H, int W, int C,
                                const double* w, const double* bias, int Cout, int K,
                                int stride, int pad, int groups, double* y) {
  const int Ho = oracle_conv_out_size(H, K, stride, pad);
  const int Wo = oracle_conv_out_size(W, K, stride, pad);
  const int Cg = C / groups, Og = Cout / groups;
#pragma omp parallel for collapse(2) schedule(static)
  for (int b = 0; b < B; ++b)
    for (int oh = 0; oh < Ho; ++oh)
      for (int ow = 0; ow < Wo; ++ow)
        for (int o = 0; o < Cout; ++o) {
          const int g = o / Og;
          double acc = bias ? bias[o] : 0.0;
          for (int kh = 0; kh < K; ++kh) {
            const int ih = oh * stride - pad + kh;
            if (ih < 0 || ih >= H) continue;
            for (int kw = 0; kw < K; ++kw) {
              const int iw = ow * stride - pad + kw;
              if (iw < 0 || iw >= W) continue;
              const double* xp = x + (((size_t)b * H + ih) * W + iw) * C + (size_t)g * Cg;
              const double* wp = w + (((size_t)o * K + kh) * K + kw) * Cg;
              for (int ci = 0; ci < Cg; ++ci) acc += xp[ci] * wp[ci];
            }
          }
          y[(((size_t)b * Ho + oh) * Wo + ow) * Cout + o] = acc;
        }
}

/* Backward of oracle_conv_fwd given dy = dL/d(pre-activation).  Each sum is
 * the transpose of the forward sum: dx gathers every (output, tap) that read
 * an input element, dw sums over all images and output positions, db sums dy.
 * dx may be NULL (the first layer's input needs no gradient). */
ORACLE_API void oracle_conv_bwd(const double* x, int B, int H, int W, int C,
                                const double* w, int Cout, int K, int stride, int pad,
                                int groups, const double* dy, double* dx, double* dw,
                                double* db) {
  const int Ho = oracle_conv_out_size(H, K, stride, pad);
  const int Wo = oracle_conv_out_size(W, K, stride, pad);
  const int Cg = C / groups, Og = Cout / groups;
  if (dx) {
#pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b)
      for (int ih = 0; ih < H; ++ih)
        for (int iw = 0; iw < W; ++iw)
          for (int c = 0; c < C; ++c) {
            const int g = c / Cg, ci = c % Cg;
            double acc = 0.0;
            for (int kh = 0; kh < K; ++kh) {
              const int t = ih + pad - kh;
              if (t < 0 || t % stride) continue;
              const int oh = t / stride;
              if (oh >= Ho) continue;
              for (int kw = 0; kw < K; ++kw) {
                const int u = iw + pad - kw;
                if (u < 0 || u % stride) continue;
                const int ow = u / stride;
                if (ow >= Wo) continue;
                const double* dyp = dy + (((size_t)b * Ho + oh) * Wo + ow) * Cout;
                for (int oo = 0; oo < Og; ++oo) {
                  const int o = g * Og + oo;
                  acc += dyp[o] * w[(((size_t)o * K + kh) * K + kw) * Cg + ci];
                }
              }
            }
            dx[(((size_t)b * H + ih) * W + iw) * C + c] = acc;
          }
  }
#pragma omp parallel for schedule(dynamic)
  for (int o = 0; o < Cout; ++o) {
    const int g = o / Og;
    double bacc = 0.0;
    for (int b = 0; b < B; ++b)
      for (int oh = 0; oh < Ho; ++oh)
        for (int ow = 0; ow < Wo; ++ow) bacc += dy[(((size_t)b * Ho + oh) * Wo + ow) * Cout + o];
    db[o] = bacc;
    for (int kh = 0; kh < K; ++kh)
      for (int kw = 0; kw < K; ++kw)
        for (int ci = 0; ci < Cg; ++ci) {
          double acc = 0.0;
          for (int b = 0; b < B; ++b)
            for (int oh = 0; oh < Ho; ++oh) {
              const int ih = oh * stride - pad + kh;
              if (ih < 0 || ih >= H) continue;
              for (int ow = 0; ow < Wo; ++ow) {
                const int iw = ow * stride - pad + kw;
                if (iw < 0 || iw >= W) continue;
                acc += dy[(((size_t)b * Ho + oh) * Wo + ow) * Cout + o] *
                       x[(((size_t)b * H + ih) * W + iw) * C + (size_t)g * Cg + ci];
              }
            }
          dw[(((size_t)o * K + kh) * K + kw) * Cg + ci] = acc;
        }
  }
}

/* Sampled forms for full-size checks: only the listed outputs are computed,
 * each by the same sum as above.  idx[i] indexes y (resp. dw) flat. */
ORACLE_API void oracle_conv_fwd_sampled(const double* x, int B, int H, int W, int C,
                                        const double* w, const double* bias, int Cout, int K,
                                        int stride, int pad, int groups, const int64_t* idx,
                                        int n, double* out) {
  const int Ho = oracle_conv_out_size(H, K, stride, pad);
  const int Wo = oracle_conv_out_size(W, K, stride, pad);
  const int Cg = C / groups, Og = Cout / groups;
  (void)B;
#pragma omp parallel for schedule(static)
  for (int i = 0; i < n; ++i) {
    int64_t e = idx[i];
    const int o = (int)(e % Cout); e /= Cout;
    const int ow = (int)(e % Wo); e /= Wo;
    const int oh = (int)(e % Ho); e /= Ho;
    const int b = (int)e;
    const int g = o / Og;
    double acc = bias ? bias[o] : 0.0;
    for (int kh = 0; kh < K; ++kh) {
      const int ih = oh * stride - pad + kh;
      if (ih < 0 || ih >= H) continue;
      for (int kw = 0; kw < K; ++kw) {
        const int iw = ow * stride - pad + kw;
        if (iw < 0 || iw >= W) continue;
        for (int ci = 0; ci < Cg; ++ci)
          acc += x[(((size_t)b * H + ih) * W + iw) * C + (size_t)g * Cg + ci] *
                 w[(((size_t)o * K + kh) * K + kw) * Cg + ci];
      }
    }
    out[i] = acc;
  }
}

ORACLE_API void oracle_conv_wgrad_sampled(const double* x, int B, int H, int W, int C,
                                          int Cout, int K, int stride, int pad, int groups,
                                          const double* dy, const int64_t* idx, int n,
                                          double* out) {
  const int Ho = oracle_conv_out_size(H, K, stride, pad);
  const int Wo = oracle_conv_out_size(W, K, stride, pad);
  const int Cg = C / groups, Og = Cout / groups;
#pragma omp parallel for schedule(dynamic)
  for (int i = 0; i < n; ++i) {
    int64_t e = idx[i];
    const int ci = (int)(e % Cg); e /= Cg;
    const int kw = (int)(e % K); e /= K;
    const int kh = (int)(e % K); e /= K;
    const int o = (int)e;
    const int g = o / Og;
    double acc = 0.0;
    for (int b = 0; b < B; ++b)
      for (int oh = 0; oh < Ho; ++oh) {
        const int ih = oh * stride - pad + kh;
        if (ih < 0 || ih >= H) continue;
        for (int ow = 0; ow < Wo; ++ow) {
          const int iw = ow * stride - pad + kw;
          if (iw < 0 || iw >= W) continue;
          acc += dy[(((size_t)b * Ho + oh) * Wo + ow) * Cout + o] *
                 x[(((size_t)b * H + ih) * W + iw) * C + (size_t)g * Cg + ci];
        }
      }
    out[i] = acc;
  }
}

/* ------------------------------------------------------------------------ */
/* ReLU f(x) = max(0, x): [S] 3.4 "ReLU Nonlinearity".  Its derivative is    */
/* taken as 1 for x > 0 and 0 otherwise (0 at x = 0).                        */
/* ------------------------------------------------------------------------ */
ORACLE_API void oracle_relu(double* x, int64_t n) {
  for (int64_t i = 0; i < n; ++i) x[i] = x[i] > 0.0 ? x[i] : 0.0;
}

/* dz = dy where the layer's output y = relu(z) is positive, else 0. */
ORACLE_API void oracle_relu_bwd(const double* y, double* d, int64_t n) {
  for (int64_t i = 0; i < n; ++i) d[i] = y[i] > 0.0 ? d[i] : 0.0;
}

/* ------------------------------------------------------------------------ */
/* Local response normalisation: [S] 3.4 "Local Response Normalization",    */
/* the b^i_{x,y} equation.  For each pixel and channel i of N channels:      */
/*   s_i = k + alpha * sum_{j=max(0,i-n/2)}^{min(N-1,i+n/2)} a_j^2           */
/*   b_i = a_i / s_i^beta                                                     */
/* n/2 is integer division; alpha is not divided by n.                        */
/* ------------------------------------------------------------------------ */
static double lrn_scale(const double* a, int N, int i, int n, double k, double alpha) {
  const int lo = i - n / 2 < 0 ? 0 : i - n / 2;
  const int hi = i + n / 2 > N - 1 ? N - 1 : i + n / 2;
  double sum = 0.0;
  for (int j = lo; j <= hi; ++j) sum += a[j] * a[j];
  return k + alpha * sum;
}

ORACLE_API void oracle_lrn_fwd(const double* a, int64_t P, int N, int n, double k, double alpha,
                               double beta, double* b) {
#pragma omp parallel for schedule(static)
  for (int64_t p = 0; p < P; ++p) {
    const double* ap = a + p * N;
    for (int i = 0; i < N; ++i) b[p * N + i] = ap[i] / pow(lrn_scale(ap, N, i, n, k, alpha), beta);
  }
}

/* Backward, derived from the forward by the chain rule:
 *   dL/da_j = g_j * s_j^-beta
 *             - 2*alpha*beta * a_j * sum_{i : j in window(i)} g_i * a_i * s_i^(-beta-1)
 * where g = dL/db and window(i) = [max(0,i-n/2), min(N-1,i+n/2)]. */
ORACLE_API void oracle_lrn_bwd(const double* a, const double* g, int64_t P, int N, int n,
                               double k, double alpha, double beta, double* da) {
#pragma omp parallel for schedule(static)
  for (int64_t p = 0; p < P; ++p) {
    const double* ap = a + p * N;
    const double* gp = g + p * N;
    for (int j = 0; j < N; ++j) {
      double cross = 0.0;
      for (int i = 0; i < N; ++i) {
        const int lo = i - n / 2 < 0 ? 0 : i - n / 2;
        const int hi = i + n / 2 > N - 1 ? N - 1 : i + n / 2;
        if (j < lo || j > hi) continue;
        const double s = lrn_scale(ap, N, i, n, k, alpha);
        cross += gp[i] * ap[i] * pow(s, -beta - 1.0);
      }
      const double sj = lrn_scale(ap, N, j, n, k, alpha);
      da[p * N + j] = gp[j] * pow(sj, -beta) - 2.0 * alpha * beta * ap[j] * cross;
    }
  }
}

/* ------------------------------------------------------------------------ */
/* Max pooling with window z x z and stride s, no padding, floor:            */
/* [S] 3.4 "Overlapping Pooling" (z = 3, s = 2).  argmax records the window   */
/* offset dy*z+dx of the first maximum in row-major window order (a later    */
/* element replaces it only if strictly greater).                            */
/* ------------------------------------------------------------------------ */
ORACLE_API int oracle_pool_out_size(int in, int z, int s) { return (in - z) / s + 1; }

ORACLE_API void oracle_maxpool_fwd(const double* x, int B, int H, int W, int C, int z, int s,
                                   double* y, uint8_t* argmax) {
  const int Ho = oracle_pool_out_size(H, z, s), Wo = oracle_pool_out_size(W, z, s);
#pragma omp parallel for collapse(2) schedule(static)
  for (int b = 0; b < B; ++b)
    for (int oh = 0; oh < Ho; ++oh)
      for (int ow = 0; ow < Wo; ++ow)
        for (int c = 0; c < C; ++c) {
          double best = 0.0;
          int arg = -1;
          for (int dy = 0; dy < z; ++dy)
            for (int dx = 0; dx < z; ++dx) {
              const double v = x[(((size_t)b * H + oh * s + dy) * W + ow * s + dx) * C + c];
              if (arg < 0 || v > best) {
                best = v;
                arg = dy * z + dx;
              }
            }
          const size_t o = (((size_t)b * Ho + oh) * Wo + ow) * C + c;
          y[o] = best;
          if (argmax) argmax[o] = (uint8_t)arg;
        }
}

/* Pooling with the window choice given (argmax from elsewhere, e.g. the
 * decision of an implementation that stores its maps in a lower precision):
 * y = x at the named window offset. */
ORACLE_API void oracle_maxpool_select(const double* x, const uint8_t* argmax, int B, int H, int W,
                                      int C, int z, int s, double* y) {
  const int Ho = oracle_pool_out_size(H, z, s), Wo = oracle_pool_out_size(W, z, s);
#pragma omp parallel for collapse(2) schedule(static)
  for (int b = 0; b < B; ++b)
    for (int oh = 0; oh < Ho; ++oh)
      for (int ow = 0; ow < Wo; ++ow)
        for (int c = 0; c < C; ++c) {
          const size_t o = (((size_t)b * Ho + oh) * Wo + ow) * C + c;
          const int a = argmax[o];
          y[o] = x[(((size_t)b * H + oh * s + a / z) * W + ow * s + a % z) * C + c];
        }
}

/* The gradient of each window goes to the input element its argmax names;
 * overlapping windows add their contributions. */
ORACLE_API void oracle_maxpool_bwd(const double* dy, const uint8_t* argmax, int B, int H, int W,
                                   int C, int z, int s, double* dx) {
  const int Ho = oracle_pool_out_size(H, z, s), Wo = oracle_pool_out_size(W, z, s);
  memset(dx, 0, sizeof(double) * (size_t)B * H * W * C);
#pragma omp parallel for schedule(static)
  for (int b = 0; b < B; ++b)
    for (int oh = 0; oh < Ho; ++oh)
      for (int ow = 0; ow < Wo; ++ow)
        for (int c = 0; c < C; ++c) {
          const size_t o = (((size_t)b * Ho + oh) * Wo + ow) * C + c;
          const int a = argmax[o];
          const int ih = oh * s + a / z, iw = ow * s + a % z;
          dx[(((size_t)b * H + ih) * W + iw) * C + c] += dy[o];
        }
}

/* ------------------------------------------------------------------------ */
/* Fully connected layer: y[b,o] = bias[o] + sum_i x[b,i] * w[o,i].         */
/* ------------------------------------------------------------------------ */
ORACLE_API void oracle_fc_fwd(const double* x, int B, int In, const double* w, const double* bias,
                              int Out, double* y) {
#pragma omp parallel for collapse(2) schedule(static)
  for (int b = 0; b < B; ++b)
    for (int o = 0; o < Out; ++o) {
      double acc = bias ? bias[o] : 0.0;
      for (int i = 0; i < In; ++i) acc += x[(size_t)b * In + i] * w[(size_t)o * In + i];
      y[(size_t)b * Out + o] = acc;
    }
}

ORACLE_API void oracle_fc_bwd(const double* x, int B, int In, const double* w, int Out,
                              const double* dz, double* dx, double* dw, double* db) {
  if (dx) {
#pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b)
      for (int i = 0; i < In; ++i) {
        double acc = 0.0;
        for (int o = 0; o < Out; ++o) acc += dz[(size_t)b * Out + o] * w[(size_t)o * In + i];
        dx[(size_t)b * In + i] = acc;
      }
  }
#pragma omp parallel for schedule(static)
  for (int o = 0; o < Out; ++o) {
    double bacc = 0.0;
    for (int b = 0; b < B; ++b) bacc += dz[(size_t)b * Out + o];
    db[o] = bacc;
    for (int i = 0; i < In; ++i) {
      double acc = 0.0;
      for (int b = 0; b < B; ++b) acc += dz[(size_t)b * Out + o] * x[(size_t)b * In + i];
      dw[(size_t)o * In + i] = acc;
    }
  }
}

/* ------------------------------------------------------------------------ */
/* Dropout: [S] 3.4 "Dropout" and [W] listing ALEXNET_FORWARD.  At training  */
/* time each hidden output is zeroed with probability p and kept unscaled;    */
/* at test time every output is kept and multiplied by 1 - p (0.5).          */
/* The pages do not say how the coin is drawn; the draw for element           */
/* e = b*Out + j of FC layer `layer` (6 or 7) at training step `step` is      */
/* word (e & 3) of Philox4x32-10(counter = (e >> 2, layer, step, 0),          */
/* key = (seed low 32, seed high 32)); the element is kept iff that word is   */
/* >= round(p * 2^32) (for p = 0.5: iff its top bit is set).  b is the       */
/* image's index in the whole minibatch: a part of a batch that starts at    */
/* image row0 draws the rows row0, row0 + 1, ... of the whole batch's mask.   */
/* ------------------------------------------------------------------------ */
ORACLE_API void oracle_dropout_mask_rows(uint64_t seed, uint32_t layer, uint32_t step, int row0,
                                         int B, int Out, double p, uint8_t* keep) {
  const double t = floor(p * 4294967296.0 + 0.5);
  const uint64_t thresh = (uint64_t)t;
  for (int64_t i = 0; i < (int64_t)B * Out; ++i) {
    const int64_t e = (int64_t)row0 * Out + i;
    uint32_t r[4];
    philox_seeded(seed, (uint32_t)(e >> 2), layer, step, 0u, r);
    keep[i] = (uint64_t)r[e & 3] >= thresh ? 1 : 0;
  }
}

ORACLE_API void oracle_dropout_mask(uint64_t seed, uint32_t layer, uint32_t step, int B, int Out,
                                    double p, uint8_t* keep) {
  oracle_dropout_mask_rows(seed, layer, step, 0, B, Out, p, keep);
}

/* ------------------------------------------------------------------------ */
/* Softmax over the classes and the multinomial logistic regression loss:    */
/* [S] 3.4 "Training Procedure Details", "Objective function": the mean over */
/* the mini-batch of -log p_label.  dlogits = (p - onehot(label)) / B.       */
/* ------------------------------------------------------------------------ */
ORACLE_API double oracle_softmax_ce(const double* z, const int32_t* labels, int B, int N,
                                    double* probs, double* dz) {
  double loss = 0.0;
  for (int b = 0; b < B; ++b) {
    const double* zb = z + (size_t)b * N;
    double m = zb[0];
    for (int j = 1; j < N; ++j) m = zb[j] > m ? zb[j] : m;
    double sum = 0.0;
    for (int j = 0; j < N; ++j) sum += exp(zb[j] - m);
    for (int j = 0; j < N; ++j) {
      const double pj = exp(zb[j] - m) / sum;
      if (probs) probs[(size_t)b * N + j] = pj;
      if (dz && labels) dz[(size_t)b * N + j] = (pj - (j == labels[b] ? 1.0 : 0.0)) / B;
    }
    if (labels) loss += -((zb[labels[b]] - m) - log(sum));
  }
  return labels ? loss / B : 0.0;
}

/* ------------------------------------------------------------------------ */
/* SGD with momentum and weight decay: [S] 3.4 "Training Procedure Details", */
/* update rule, and [W] listing TRAIN_STEP:                                   */
/*   v <- momentum*v - wd*lr*w - lr*g ;  w <- w + v                           */
/* applied to every parameter (biases included), in that order.               */
/* ------------------------------------------------------------------------ */
ORACLE_API void oracle_sgd(double* w, double* v, const double* g, int64_t n, double lr,
                           double momentum, double wd) {
  for (int64_t i = 0; i < n; ++i) {
    v[i] = momentum * v[i] - wd * lr * w[i] - lr * g[i];
    w[i] = w[i] + v[i];
  }
}

/* ------------------------------------------------------------------------ */
/* Network description.  The AlexNet defaults ([S] 3.4 "Overall Architecture"*/
/* and [W] "Layer-by-layer structure"): 227x227x3 input; conv 96@11x11/s4/p0, */
/* 256@5x5/p2, 384@3x3/p1, 384@3x3/p1, 256@3x3/p1; ReLU after each;           */
/* LRN after conv1, conv2; max-pool 3/2 after conv1, conv2, conv5; FC 4096,   */
/* 4096 with ReLU + dropout, FC 1000 + softmax.  groups = 2 on conv2, conv4,  */
/* conv5 expresses the two-GPU restricted connectivity ([S] 3.4 "Training on  */
/* Multiple GPUs"; [P2] "Reading Figure 2": 5x5x48 and 3x3x192 kernels).      */
/* A smaller instance with the same op sequence is used to check gradients.  */
/* ------------------------------------------------------------------------ */
typedef struct {
  int in_hw, in_c;
  int conv_c[5], conv_k[5], conv_s[5], conv_p[5], conv_g[5];
  int lrn_after[5], pool_after[5];
  int fc_n[3];
  int pool_z, pool_s;
  int lrn_n;
  double lrn_k, lrn_alpha, lrn_beta;
  int dropout_on;
  double dropout_p;
} oracle_net;

typedef struct {
  int hw[6];  /* spatial size entering conv l (hw[0] = input), hw[5] = flattened map side */
  int conv_out[5];
  int pool_out[5];
  int flat;
  int64_t w_off[8], b_off[8], w_len[8], b_len[8];
  int64_t n_params;
} oracle_shapes;

static void net_shapes(const oracle_net* net, oracle_shapes* s) {
  int hw = net->in_hw, c = net->in_c;
  int64_t off = 0;
  for (int l = 0; l < 5; ++l) {
    s->hw[l] = hw;
    const int o = oracle_conv_out_size(hw, net->conv_k[l], net->conv_s[l], net->conv_p[l]);
    s->conv_out[l] = o;
    hw = net->pool_after[l] ? oracle_pool_out_size(o, net->pool_z, net->pool_s) : o;
    s->pool_out[l] = hw;
    s->w_off[l] = off;
    s->w_len[l] = (int64_t)net->conv_c[l] * net->conv_k[l] * net->conv_k[l] * (c / net->conv_g[l]);
    off += s->w_len[l];
    s->b_off[l] = off;
    s->b_len[l] = net->conv_c[l];
    off += s->b_len[l];
    c = net->conv_c[l];
  }
  s->hw[5] = hw;
  s->flat = hw * hw * c;
  int in = s->flat;
  for (int f = 0; f < 3; ++f) {
    s->w_off[5 + f] = off;
    s->w_len[5 + f] = (int64_t)net->fc_n[f] * in;
    off += s->w_len[5 + f];
    s->b_off[5 + f] = off;
    s->b_len[5 + f] = net->fc_n[f];
    off += s->b_len[5 + f];
    in = net->fc_n[f];
  }
  s->n_params = off;
}

ORACLE_API int64_t oracle_param_count(const oracle_net* net) {
  oracle_shapes s;
  net_shapes(net, &s);
  return s.n_params;
}

/* offsets[16] = (w_off, w_len) for the 8 layers then (b_off, b_len) ... laid
 * out as w_off[8], w_len[8], b_off[8], b_len[8] (32 entries). */
ORACLE_API void oracle_param_layout(const oracle_net* net, int64_t* out32) {
  oracle_shapes s;
  net_shapes(net, &s);
  for (int l = 0; l < 8; ++l) {
    out32[l] = s.w_off[l];
    out32[8 + l] = s.w_len[l];
    out32[16 + l] = s.b_off[l];
    out32[24 + l] = s.b_len[l];
  }
}

/* Multiply-accumulates of one forward pass of one image (convolutions and
 * FC layers; [W] "Time complexity of one forward pass": per conv layer
 * Cin/groups * Cout * k * k * H' * W'). */
ORACLE_API int64_t oracle_forward_macs(const oracle_net* net) {
  oracle_shapes s;
  net_shapes(net, &s);
  int64_t macs = 0;
  int c = net->in_c;
  for (int l = 0; l < 5; ++l) {
    macs += (int64_t)(c / net->conv_g[l]) * net->conv_c[l] * net->conv_k[l] * net->conv_k[l] *
            s.conv_out[l] * s.conv_out[l];
    c = net->conv_c[l];
  }
  int in = s.flat;
  for (int f = 0; f < 3; ++f) {
    macs += (int64_t)in * net->fc_n[f];
    in = net->fc_n[f];
  }
  return macs;
}

/* Neurons per learned layer (output units of each conv and FC layer, before
 * pooling): out8[0..7]. */
ORACLE_API void oracle_neuron_counts(const oracle_net* net, int64_t* out8) {
  oracle_shapes s;
  net_shapes(net, &s);
  for (int l = 0; l < 5; ++l) out8[l] = (int64_t)s.conv_out[l] * s.conv_out[l] * net->conv_c[l];
  for (int f = 0; f < 3; ++f) out8[5 + f] = net->fc_n[f];
}

/* Activations kept between forward and backward. */
typedef struct {
  oracle_shapes s;
  double* conv_in[5];   /* input of conv l (conv_in[0] = x) */
  double* relu_out[5];  /* a_l = relu(conv_l) */
  double* lrn_out[5];   /* b_l (NULL if no LRN) */
  double* pool_out[5];  /* pooled map (NULL if no pool) */
  uint8_t* argmax[5];
  double* fc_in[3];
  double* fc_relu[2];   /* relu(FC6), relu(FC7) */
  double* fc_out[2];    /* after dropout / scaling */
  uint8_t* keep[2];
  double* logits;
  const uint8_t* relu_given[7];  /* optional ReLU decisions: conv1..5, FC6, FC7 */
  int keep_pre;                  /* store the pre-activations below */
  int row0;                      /* index of the first image in the whole minibatch (dropout) */
  double* pre[7];                /* conv1..5, FC6, FC7 before the ReLU (keep_pre only) */
} fwd_cache;

static double* dalloc(int64_t n) { return (double*)calloc((size_t)(n > 0 ? n : 1), sizeof(double)); }

static void cache_free(fwd_cache* c) {
  for (int l = 0; l < 5; ++l) {
    if (l > 0) free(c->conv_in[l]);
    free(c->relu_out[l]);
    free(c->lrn_out[l]);
    free(c->pool_out[l]);
    free(c->argmax[l]);
  }
  for (int f = 0; f < 2; ++f) {
    free(c->fc_relu[f]);
    free(c->fc_out[f]);
    free(c->keep[f]);
  }
  for (int i = 0; i < 7; ++i) free(c->pre[i]);
  free(c->logits);
}

/* mode: 0 = training (dropout masks drawn), 1 = inference (x (1-p)). */
static void net_forward_given(const oracle_net* net, const double* params, const double* x,
                              int B, int mode, uint64_t seed, uint32_t step,
                              const uint8_t* const* am_in, const uint8_t* const* relu_in,
                              fwd_cache* c);

static void net_forward(const oracle_net* net, const double* params, const double* x, int B,
                        int mode, uint64_t seed, uint32_t step, fwd_cache* c) {
  c->keep_pre = 0;
  c->row0 = 0;
  net_forward_given(net, params, x, B, mode, seed, step, NULL, NULL, c);
}

/* ReLU with the sign decision optionally given: out = z where the unit is
 * taken as active (given[e] != 0, or z > 0 when given is NULL), else 0. */
static void relu_decided(double* z, int64_t n, const uint8_t* given) {
  if (!given) {
    oracle_relu(z, n);
    return;
  }
  for (int64_t i = 0; i < n; ++i) z[i] = given[i] ? z[i] : 0.0;
}

/* The ReLU derivative with the same decision: d passes where active. */
static void relu_bwd_decided(const double* y, double* d, int64_t n, const uint8_t* given) {
  if (!given) {
    oracle_relu_bwd(y, d, n);
    return;
  }
  for (int64_t i = 0; i < n; ++i) d[i] = given[i] ? d[i] : 0.0;
}

/* am_in (nullable; entries nullable): window choices of the max-pools after
 * conv l, used instead of the oracle's own argmax.  relu_in (nullable;
 * entries nullable): ReLU sign decisions of conv1..conv5, FC6, FC7 used
 * instead of the oracle's own (z > 0). */
static void net_forward_given(const oracle_net* net, const double* params, const double* x,
                              int B, int mode, uint64_t seed, uint32_t step,
                              const uint8_t* const* am_in, const uint8_t* const* relu_in,
                              fwd_cache* c) {
  const int keep_pre = c->keep_pre, row0 = c->row0;
  memset(c, 0, sizeof(*c));
  c->keep_pre = keep_pre;
  c->row0 = row0;
  for (int i = 0; i < 7; ++i) c->relu_given[i] = relu_in ? relu_in[i] : NULL;
  net_shapes(net, &c->s);
  const oracle_shapes* s = &c->s;
  const double* in = x;
  int C = net->in_c;
  for (int l = 0; l < 5; ++l) {
    const int H = s->hw[l], O = s->conv_out[l], Co = net->conv_c[l];
    c->conv_in[l] = (double*)in;
    const int64_t n = (int64_t)B * O * O * Co;
    c->relu_out[l] = dalloc(n);
    oracle_conv_fwd(in, B, H, H, C, params + s->w_off[l], params + s->b_off[l], Co,
                    net->conv_k[l], net->conv_s[l], net->conv_p[l], net->conv_g[l],
                    c->relu_out[l]);
    if (c->keep_pre) {
      c->pre[l] = dalloc(n);
      memcpy(c->pre[l], c->relu_out[l], sizeof(double) * (size_t)n);
    }
    relu_decided(c->relu_out[l], n, c->relu_given[l]);
    const double* cur = c->relu_out[l];
    if (net->lrn_after[l]) {
      c->lrn_out[l] = dalloc(n);
      oracle_lrn_fwd(cur, (int64_t)B * O * O, Co, net->lrn_n, net->lrn_k, net->lrn_alpha,
                     net->lrn_beta, c->lrn_out[l]);
      cur = c->lrn_out[l];
    }
    if (net->pool_after[l]) {
      const int P = s->pool_out[l];
      const int64_t np = (int64_t)B * P * P * Co;
      c->pool_out[l] = dalloc(np);
      c->argmax[l] = (uint8_t*)calloc((size_t)np, 1);
      if (am_in && am_in[l]) {
        memcpy(c->argmax[l], am_in[l], (size_t)np);
        oracle_maxpool_select(cur, c->argmax[l], B, O, O, Co, net->pool_z, net->pool_s,
                              c->pool_out[l]);
      } else {
        oracle_maxpool_fwd(cur, B, O, O, Co, net->pool_z, net->pool_s, c->pool_out[l],
                           c->argmax[l]);
      }
      cur = c->pool_out[l];
    }
    if (l < 4) {
      /* the next conv reads this map; keep a private copy so the cache owns it */
      const int64_t nn = (int64_t)B * s->pool_out[l] * s->pool_out[l] * Co;
      double* cp = dalloc(nn);
      memcpy(cp, cur, sizeof(double) * (size_t)nn);
      in = cp;
    } else {
      c->fc_in[0] = (double*)cur;
    }
    C = Co;
  }
  int In = s->flat;
  for (int f = 0; f < 3; ++f) {
    const int Out = net->fc_n[f];
    double* z = dalloc((int64_t)B * Out);
    oracle_fc_fwd(c->fc_in[f], B, In, params + s->w_off[5 + f], params + s->b_off[5 + f], Out, z);
    if (f < 2) {
      if (c->keep_pre) {
        c->pre[5 + f] = dalloc((int64_t)B * Out);
        memcpy(c->pre[5 + f], z, sizeof(double) * (size_t)B * Out);
      }
      relu_decided(z, (int64_t)B * Out, c->relu_given[5 + f]);
      c->fc_relu[f] = z;
      double* d = dalloc((int64_t)B * Out);
      c->keep[f] = (uint8_t*)calloc((size_t)B * Out, 1);
      if (net->dropout_on && mode == 0) {
        oracle_dropout_mask_rows(seed, (uint32_t)(6 + f), step, c->row0, B, Out, net->dropout_p,
                                 c->keep[f]);
        for (int64_t e = 0; e < (int64_t)B * Out; ++e) d[e] = c->keep[f][e] ? z[e] : 0.0;
      } else if (net->dropout_on) {
        for (int64_t e = 0; e < (int64_t)B * Out; ++e) d[e] = z[e] * (1.0 - net->dropout_p);
      } else {
        for (int64_t e = 0; e < (int64_t)B * Out; ++e) d[e] = z[e];
      }
      c->fc_out[f] = d;
      c->fc_in[f + 1] = d;
    } else {
      c->logits = z;
    }
    In = Out;
  }
}

ORACLE_API void oracle_forward(const oracle_net* net, const double* params, const double* x,
                               int B, int mode, uint64_t seed, uint32_t step, double* logits,
                               double* probs) {
  fwd_cache c;
  net_forward(net, params, x, B, mode, seed, step, &c);
  const int N = net->fc_n[2];
  if (logits) memcpy(logits, c.logits, sizeof(double) * (size_t)B * N);
  if (probs) oracle_softmax_ce(c.logits, NULL, B, N, probs, NULL);
  cache_free(&c);
}

/* Intermediate maps of a forward pass, for per-op checks.  which:
 *   0..4  relu output of conv l      10..14 LRN output of conv l
 *   20..24 pooled map after conv l   30, 31 FC6/FC7 output after dropout
 *   40 logits */
/* Copy map `which` (codes of oracle_forward_probe) out of a forward cache. */
static void oracle_forward_probe_from(const oracle_net* net, const fwd_cache* c, int B, int which,
                                      double* out) {
  const oracle_shapes* s = &c->s;
  const double* src = NULL;
  int64_t n = 0;
  if (which >= 0 && which < 5) {
    src = c->relu_out[which];
    n = (int64_t)B * s->conv_out[which] * s->conv_out[which] * net->conv_c[which];
  } else if (which >= 10 && which < 15) {
    src = c->lrn_out[which - 10];
    n = (int64_t)B * s->conv_out[which - 10] * s->conv_out[which - 10] * net->conv_c[which - 10];
  } else if (which >= 20 && which < 25) {
    src = c->pool_out[which - 20];
    n = (int64_t)B * s->pool_out[which - 20] * s->pool_out[which - 20] * net->conv_c[which - 20];
  } else if (which == 30 || which == 31) {
    src = c->fc_out[which - 30];
    n = (int64_t)B * net->fc_n[which - 30];
  } else if (which == 40) {
    src = c->logits;
    n = (int64_t)B * net->fc_n[2];
  }
  if (src) memcpy(out, src, sizeof(double) * (size_t)n);
}

ORACLE_API void oracle_forward_probe(const oracle_net* net, const double* params,
                                     const double* x, int B, int mode, uint64_t seed,
                                     uint32_t step, int which, double* out) {
  fwd_cache c;
  net_forward(net, params, x, B, mode, seed, step, &c);
  oracle_forward_probe_from(net, &c, B, which, out);
  cache_free(&c);
}

/* Several intermediate maps of one forward pass, each copied to its own
 * output (which[i] -> out[i]):
 *   0..4, 10..14, 20..24, 30, 31, 40  as oracle_forward_probe;
 *   100+l  pre-activation of conv l (before the ReLU); 105, 106 FC6, FC7.
 * One pass instead of one per map: at the benchmark's batch a forward of
 * this oracle takes tens of seconds. */
ORACLE_API void oracle_forward_trace(const oracle_net* net, const double* params, const double* x,
                                     int B, int mode, uint64_t seed, uint32_t step, int n,
                                     const int* which, double* const* out) {
  fwd_cache c;
  c.keep_pre = 1;
  c.row0 = 0;
  net_forward_given(net, params, x, B, mode, seed, step, NULL, NULL, &c);
  const oracle_shapes* s = &c.s;
  for (int i = 0; i < n; ++i) {
    const int w = which[i];
    if (w < 100) {
      oracle_forward_probe_from(net, &c, B, w, out[i]);
    } else if (w >= 100 && w < 105) {
      const int l = w - 100;
      memcpy(out[i], c.pre[l],
             sizeof(double) * (size_t)B * s->conv_out[l] * s->conv_out[l] * net->conv_c[l]);
    } else if (w == 105 || w == 106) {
      memcpy(out[i], c.pre[w - 100], sizeof(double) * (size_t)B * net->fc_n[w - 105]);
    }
  }
  cache_free(&c);
}

/* One training step ([W] listing TRAIN_STEP; [S] 3.4 "Training Procedure
 * Details"): forward in training mode, mean cross-entropy, backpropagation
 * through every layer, then the SGD update of every parameter.  params and
 * velocity are updated in place; grads (nullable) receives dL/dparams at the
 * pre-update weights; logits (nullable) receives the forward logits.
 * Returns the loss. */
static double train_step_probe(const oracle_net* net, double* params, double* velocity,
                               const double* x, const int32_t* labels, int B, double lr,
                               double momentum, double wd, uint64_t seed, uint32_t step,
                               double* grads, double* logits, int probe, double* probe_out,
                               const uint8_t* const* am_in, const uint8_t* const* relu_in,
                               int row0);

ORACLE_API double oracle_train_step(const oracle_net* net, double* params, double* velocity,
                                    const double* x, const int32_t* labels, int B, double lr,
                                    double momentum, double wd, uint64_t seed, uint32_t step,
                                    double* grads, double* logits) {
  return train_step_probe(net, params, velocity, x, labels, B, lr, momentum, wd, seed, step,
                          grads, logits, -1, NULL, NULL, NULL, 0);
}

/* The same step with the max-pool window choices given (am1, am2, am5 for the
 * pools after conv1, conv2, conv5; each nullable) and the ReLU sign decisions
 * given (relu7: 7 nullable masks for conv1..conv5, FC6, FC7; nullable). */
ORACLE_API double oracle_train_step_given(const oracle_net* net, double* params, double* velocity,
                                          const double* x, const int32_t* labels, int B,
                                          double lr, double momentum, double wd, uint64_t seed,
                                          uint32_t step, double* grads, double* logits,
                                          const uint8_t* am1, const uint8_t* am2,
                                          const uint8_t* am5, const uint8_t* const* relu7) {
  const uint8_t* am_in[5] = {am1, am2, NULL, NULL, am5};
  return train_step_probe(net, params, velocity, x, labels, B, lr, momentum, wd, seed, step,
                          grads, logits, -1, NULL, am_in, relu7, 0);
}

/* The step of a part of a minibatch: B images that are images row0 ..
 * row0 + B - 1 of the whole batch (their dropout draws are those rows of the
 * whole batch's masks), the loss averaged over these B images.  With
 * row0 = 0 and the whole batch this is oracle_train_step. */
ORACLE_API double oracle_train_step_rows(const oracle_net* net, double* params, double* velocity,
                                         const double* x, const int32_t* labels, int B,
                                         double lr, double momentum, double wd, uint64_t seed,
                                         uint32_t step, int row0, double* grads, double* logits) {
  return train_step_probe(net, params, velocity, x, labels, B, lr, momentum, wd, seed, step,
                          grads, logits, -1, NULL, NULL, NULL, row0);
}

/* Intermediate gradients of a training step (no update is kept):
 *   50+l  dL/d(pre-activation of conv l)      60+l dL/d(pooled map of conv l)
 *   70+l  dL/d(LRN output of conv l)          80 dL/dlogits, 81/82 dL/d(FC7/FC6
 *   pre-activation) */
ORACLE_API void oracle_train_probe(const oracle_net* net, const double* params, const double* x,
                                   const int32_t* labels, int B, uint64_t seed, uint32_t step,
                                   int which, double* out, const uint8_t* am1,
                                   const uint8_t* am2, const uint8_t* am5,
                                   const uint8_t* const* relu7) {
  const uint8_t* am_in[5] = {am1, am2, NULL, NULL, am5};
  oracle_shapes s;
  net_shapes(net, &s);
  double* p = dalloc(s.n_params);
  double* v = dalloc(s.n_params);
  memcpy(p, params, sizeof(double) * (size_t)s.n_params);
  train_step_probe(net, p, v, x, labels, B, 0.0, 0.0, 0.0, seed, step, NULL, NULL, which, out,
                   am_in, relu7, 0);
  free(p);
  free(v);
}

static void probe_copy(int probe, int which, const double* src, int64_t n, double* out) {
  if (probe == which && out) memcpy(out, src, sizeof(double) * (size_t)n);
}

static double train_step_probe(const oracle_net* net, double* params, double* velocity,
                               const double* x, const int32_t* labels, int B, double lr,
                               double momentum, double wd, uint64_t seed, uint32_t step,
                               double* grads, double* logits, int probe, double* probe_out,
                               const uint8_t* const* am_in, const uint8_t* const* relu_in,
                               int row0) {
  fwd_cache c;
  c.keep_pre = 0;
  c.row0 = row0;
  net_forward_given(net, params, x, B, 0, seed, step, am_in, relu_in, &c);
  const oracle_shapes* s = &c.s;
  const int N = net->fc_n[2];
  if (logits) memcpy(logits, c.logits, sizeof(double) * (size_t)B * N);
  double* g = dalloc(s->n_params);
  double* dz = dalloc((int64_t)B * N);
  const double loss = oracle_softmax_ce(c.logits, labels, B, N, NULL, dz);
  probe_copy(probe, 80, dz, (int64_t)B * N, probe_out);

  /* FC8, FC7, FC6 */
  double* dcur = dz;
  for (int f = 2; f >= 0; --f) {
    const int Out = net->fc_n[f];
    const int In = f == 0 ? s->flat : net->fc_n[f - 1];
    double* dx = dalloc((int64_t)B * In);
    oracle_fc_bwd(c.fc_in[f], B, In, params + s->w_off[5 + f], Out, dcur,
                  dx, g + s->w_off[5 + f], g + s->b_off[5 + f]);
    free(dcur);
    dcur = dx;
    if (f > 0) {
      /* through dropout (same mask, or the test-time scale) and ReLU of FC(f-1) */
      const int64_t n = (int64_t)B * In;
      for (int64_t e = 0; e < n; ++e) {
        double d = dcur[e];
        if (net->dropout_on) d = c.keep[f - 1][e] ? d : 0.0;
        dcur[e] = d;
      }
      relu_bwd_decided(c.fc_relu[f - 1], dcur, n, c.relu_given[5 + f - 1]);
      probe_copy(probe, 80 + (3 - f), dcur, n, probe_out);
    }
  }
  /* conv5 ... conv1: dcur is dL/d(pooled or last map of layer l) */
  for (int l = 4; l >= 0; --l) {
    const int O = s->conv_out[l], Co = net->conv_c[l];
    const int64_t n = (int64_t)B * O * O * Co;
    if (net->pool_after[l]) {
      double* d = dalloc(n);
      probe_copy(probe, 60 + l, dcur, (int64_t)B * s->pool_out[l] * s->pool_out[l] * Co, probe_out);
      oracle_maxpool_bwd(dcur, c.argmax[l], B, O, O, Co, net->pool_z, net->pool_s, d);
      free(dcur);
      dcur = d;
    }
    if (net->lrn_after[l]) {
      double* d = dalloc(n);
      probe_copy(probe, 70 + l, dcur, n, probe_out);
      oracle_lrn_bwd(c.relu_out[l], dcur, (int64_t)B * O * O, Co, net->lrn_n, net->lrn_k,
                     net->lrn_alpha, net->lrn_beta, d);
      free(dcur);
      dcur = d;
    }
    relu_bwd_decided(c.relu_out[l], dcur, n, c.relu_given[l]);
    probe_copy(probe, 50 + l, dcur, n, probe_out);
    const int H = s->hw[l];
    const int Ci = l == 0 ? net->in_c : net->conv_c[l - 1];
    double* dx = l > 0 ? dalloc((int64_t)B * H * H * Ci) : NULL;
    oracle_conv_bwd(c.conv_in[l], B, H, H, Ci, params + s->w_off[l], Co, net->conv_k[l],
                    net->conv_s[l], net->conv_p[l], net->conv_g[l], dcur, dx,
                    g + s->w_off[l], g + s->b_off[l]);
    free(dcur);
    dcur = dx;
  }
  if (grads) memcpy(grads, g, sizeof(double) * (size_t)s->n_params);
  oracle_sgd(params, velocity, g, s->n_params, lr, momentum, wd);
  free(g);
  cache_free(&c);
  return loss;
}

/* Loss only (training-mode forward with the step's dropout masks): used for
 * finite-difference checks of oracle_train_step's gradients. */
ORACLE_API double oracle_loss(const oracle_net* net, const double* params, const double* x,
                              const int32_t* labels, int B, uint64_t seed, uint32_t step) {
  fwd_cache c;
  net_forward(net, params, x, B, 0, seed, step, &c);
  const double loss = oracle_softmax_ce(c.logits, labels, B, net->fc_n[2], NULL, NULL);
  cache_free(&c);
  return loss;
}

/* ------------------------------------------------------------------------ */
/* Training-time augmentation: [S] 3.4 "Data Augmentation", Form 1 (random   */
/* 224x224 patch of the 256x256 image and its horizontal reflection) and      */
/* Form 2 (add [p1 p2 p3][a1 l1, a2 l2, a3 l3]^T to every pixel, a_i drawn    */
/* once per image from N(0, 0.1^2)); the per-pixel training-set mean is       */
/* subtracted first ([S] 3.2 "Input preprocessing").                         */
/* Draws for image i at step t (key = seed):                                 */
/*   word 0 of Philox(i, 0xA0, t, 0): bits 0-4 row offset, bits 5-9 column    */
/*   offset (0..31 each), bit 10 reflection;                                  */
/*   the 4 words of Philox(i, 0xA1, t, 0) give a_1, a_2 (one Box-Muller pair  */
/*   from words 0, 1) and a_3 (the cosine branch of words 2, 3), times 0.1.  */
/* The 224x224 crop sits at the top-left of a 227x227 zero frame.            */
/* pca_vec is row-major 3x3 with column i = eigenvector p_i (RGB).           */
/* ------------------------------------------------------------------------ */
static void aug_draws(uint64_t seed, uint32_t img, uint32_t step, int* oy, int* ox, int* flip,
                      double alpha[3]) {
  uint32_t r[4];
  philox_seeded(seed, img, 0xA0u, step, 0u, r);
  *oy = (int)(r[0] & 31u);
  *ox = (int)((r[0] >> 5) & 31u);
  *flip = (int)((r[0] >> 10) & 1u);
  philox_seeded(seed, img, 0xA1u, step, 0u, r);
  const double two_pi = 6.283185307179586476925286766559;
  const double u1 = word_to_open_unit(r[0]), u2 = word_to_open_unit(r[1]);
  const double u3 = word_to_open_unit(r[2]), u4 = word_to_open_unit(r[3]);
  const double r1 = sqrt(-2.0 * log(u1)), r2 = sqrt(-2.0 * log(u3));
  alpha[0] = 0.1 * r1 * cos(two_pi * u2);
  alpha[1] = 0.1 * r1 * sin(two_pi * u2);
  alpha[2] = 0.1 * r2 * cos(two_pi * u4);
}

ORACLE_API void oracle_aug_draws(uint64_t seed, uint32_t img, uint32_t step, int32_t* oy_ox_flip,
                                 double* alpha) {
  int oy, ox, fl;
  aug_draws(seed, img, step, &oy, &ox, &fl, alpha);
  oy_ox_flip[0] = oy;
  oy_ox_flip[1] = ox;
  oy_ox_flip[2] = fl;
}

static void crop_one(const uint8_t* src, const double* mean, int oy, int ox, int flip,
                     const double add[3], double* out /* 227*227*3 */) {
  for (int y = 0; y < 227; ++y)
    for (int x = 0; x < 227; ++x)
      for (int c = 0; c < 3; ++c) {
        double v = 0.0;
        if (y < 224 && x < 224) {
          const int sy = oy + y;
          const int sx = flip ? ox + 223 - x : ox + x;
          const size_t si = ((size_t)sy * 256 + sx) * 3 + c;
          v = (double)src[si] - mean[si] + add[c];
        }
        out[((size_t)y * 227 + x) * 3 + c] = v;
      }
}

ORACLE_API void oracle_augment(const uint8_t* src, int B, const double* mean,
                               const double* pca_vec, const double* pca_val, uint64_t seed,
                               uint32_t step, double* out) {
#pragma omp parallel for schedule(static)
  for (int b = 0; b < B; ++b) {
    int oy, ox, fl;
    double a[3], add[3];
    aug_draws(seed, (uint32_t)b, step, &oy, &ox, &fl, a);
    for (int c = 0; c < 3; ++c) {
      add[c] = 0.0;
      for (int i = 0; i < 3; ++i) add[c] += pca_vec[c * 3 + i] * (a[i] * pca_val[i]);
    }
    crop_one(src + (size_t)b * 256 * 256 * 3, mean, oy, ox, fl, add,
             out + (size_t)b * 227 * 227 * 3);
  }
}

/* ------------------------------------------------------------------------ */
/* Ten-patch test-time averaging: [S] 3.4 "Data Augmentation" (test time):   */
/* the four corner 224x224 patches and the centre patch, plus their          */
/* reflections; the ten softmax outputs are averaged.  Patch order: TL, TR,  */
/* BL, BR, centre, then the same five reflected.  Top-k: descending          */
/* probability, ties to the lower class index ([S] 5 "Metrics": top-1/top-5).*/
/* ------------------------------------------------------------------------ */
static const int TEN_OY[5] = {0, 0, 32, 32, 16};
static const int TEN_OX[5] = {0, 32, 0, 32, 16};

ORACLE_API void oracle_tencrop_inputs(const uint8_t* src, int B, const double* mean,
                                      double* out /* [B*10, 227, 227, 3], image-major */) {
  const double zero[3] = {0.0, 0.0, 0.0};
#pragma omp parallel for schedule(static)
  for (int i = 0; i < B * 10; ++i) {
    const int b = i / 10, p = i % 10;
    crop_one(src + (size_t)b * 256 * 256 * 3, mean, TEN_OY[p % 5], TEN_OX[p % 5], p >= 5, zero,
             out + (size_t)i * 227 * 227 * 3);
  }
}

ORACLE_API void oracle_topk(const double* probs, int B, int N, int k, int32_t* idx) {
  for (int b = 0; b < B; ++b) {
    const double* p = probs + (size_t)b * N;
    for (int t = 0; t < k; ++t) {
      int best = -1;
      for (int j = 0; j < N; ++j) {
        int taken = 0;
        for (int u = 0; u < t; ++u) taken |= idx[(size_t)b * k + u] == j;
        if (taken) continue;
        if (best < 0 || p[j] > p[best]) best = j;
      }
      idx[(size_t)b * k + t] = best;
    }
  }
}

ORACLE_API void oracle_tencrop(const oracle_net* net, const double* params, const uint8_t* src,
                               int B, const double* mean, double* probs_avg, int32_t* top5) {
  const int N = net->fc_n[2];
  double* crops = dalloc((int64_t)B * 10 * 227 * 227 * 3);
  double* probs = dalloc((int64_t)B * 10 * N);
  oracle_tencrop_inputs(src, B, mean, crops);
  oracle_forward(net, params, crops, B * 10, 1, 0, 0, NULL, probs);
  for (int b = 0; b < B; ++b)
    for (int j = 0; j < N; ++j) {
      double acc = 0.0;
      for (int p = 0; p < 10; ++p) acc += probs[((size_t)b * 10 + p) * N + j];
      probs_avg[(size_t)b * N + j] = acc / 10.0;
    }
  oracle_topk(probs_avg, B, N, 5, top5);
  free(crops);
  free(probs);
}
