/* Plain C restatement of the oracle for small configurations: the NF4
 * codebook, block quantiser and dequantiser, one QLoRA projection forward and
 * hand-derived backward, and the gated MLP (SwiGLU, GeGLU-tanh) built from
 * three projections, written as loops in binary64.
 *
 * TEST INFRASTRUCTURE ONLY, like the rest of oracle/: nothing in the product
 * path links or calls it.  It shares no code with the CUDA path, nor with the
 * numpy oracle beside it (tests check that the two oracles agree, which pins
 * each against a second, independent statement of the same definitions).
 *
 * Sources, by page title and section:
 *  - "用 Unsloth 微调 Mistral，速度提升 14 倍", benchmark configuration block
 *    (QLoRA nf4 layers, rank 16, alpha 16) and item "10、11. 手动 Autograd"
 *    (the rank-r factor bracketed first in every chained product);
 *  - "Show HN: 80% faster, 50% less memory, 0% loss of accuracy Llama
 *    finetuning", highlight 1 (backward derived by hand), and the QLoRA paper
 *    the thread links for the NormalFloat format;
 *  - "使用 Unsloth 微调 Gemma：速度提升 2.4 倍，显存占用降低 58%", section
 *    "GeGLU 与 Swiglu 激活函数" (the gated MLP and its hand-derived derivatives).
 * Readings where the pages are silent (the same as the numpy oracle's): 16
 * levels from N(0, 1) quantiles with an exact zero, normalised to [-1, 1] and
 * stored as binary32; blocks of 64 along the input dimension with a binary32
 * absmax; even element of a pair in the high nibble; a value on a midpoint
 * takes the lower level; an all-zero block stores level 7 (zero); the
 * dequantised weight is the bf16 (round-to-nearest-even) of the binary32
 * product level x absmax.
 *
 * The N(0, 1) quantile here is Newton's method on the CDF written with the C
 * library's erfc, independent of the numpy oracle's statistics.NormalDist.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define NF4_BLOCK 64

static double std_normal_cdf(double x) { return 0.5 * erfc(-x / sqrt(2.0)); }

/* x with Phi(x) = p for 1/2 <= p < 1.  Phi is increasing and concave on
 * x >= 0, so Newton's iterates from x = 0 rise monotonically to the root. */
static double std_normal_quantile(double p) {
  const double inv_sqrt_2pi = 0.39894228040143267794;
  double x = 0.0;
  for (int it = 0; it < 200; ++it) {
    const double step = (std_normal_cdf(x) - p) / (inv_sqrt_2pi * exp(-0.5 * x * x));
    x -= step;
    if (fabs(step) <= 1e-16 * (1.0 + fabs(x))) break;
  }
  return x;
}

/* The 16 levels, ascending, each an exact binary32 value (returned as double). */
void oracle_c_nf4_codebook(double out[16]) {
  const double delta = 0.5 * ((1.0 - 1.0 / 30.0) + (1.0 - 1.0 / 32.0));
  double lv[16];
  int n = 0;
  /* positive half: 9 probabilities evenly spaced from delta to 1/2, the 1/2 end dropped */
  for (int i = 0; i < 8; ++i) lv[n++] = std_normal_quantile(delta + (0.5 - delta) * i / 8.0);
  /* negative half: 8 probabilities from delta to 1/2, the 1/2 end dropped, quantiles negated */
  for (int i = 0; i < 7; ++i) lv[n++] = -std_normal_quantile(delta + (0.5 - delta) * i / 7.0);
  lv[n++] = 0.0;
  /* sort ascending (insertion sort of 16 values) */
  for (int i = 1; i < 16; ++i) {
    const double v = lv[i];
    int j = i - 1;
    while (j >= 0 && lv[j] > v) {
      lv[j + 1] = lv[j];
      --j;
    }
    lv[j + 1] = v;
  }
  double scale = 0.0;
  for (int i = 0; i < 16; ++i)
    if (fabs(lv[i]) > scale) scale = fabs(lv[i]);
  for (int i = 0; i < 16; ++i) out[i] = (double)(float)(lv[i] / scale);
}

static double bf16_to_double(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* Round a binary32 value to bf16, round-to-nearest-even (finite inputs). */
static uint16_t float_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  const uint32_t lsb = (u >> 16) & 1u;
  u += 0x7FFFu + lsb;
  return (uint16_t)(u >> 16);
}

/* Quantise a bf16 weight [n_out, k_in] (bit patterns); k_in % 64 == 0.
 * codes: n_out * k_in / 2 bytes; absmax: n_out * k_in / 64 binary32. */
int oracle_c_nf4_quantize(const uint16_t* w, long n_out, long k_in, uint8_t* codes, float* absmax) {
  if (k_in % NF4_BLOCK) return 1;
  double lv[16], mid[15];
  oracle_c_nf4_codebook(lv);
  for (int i = 0; i < 15; ++i) mid[i] = 0.5 * (lv[i] + lv[i + 1]);
  const long nblocks = n_out * k_in / NF4_BLOCK;
  for (long b = 0; b < nblocks; ++b) {
    const uint16_t* wb = w + b * NF4_BLOCK;
    float am = 0.0f;
    for (int j = 0; j < NF4_BLOCK; ++j) {
      const float a = fabsf((float)bf16_to_double(wb[j]));
      if (a > am) am = a;
    }
    absmax[b] = am;
    int q[NF4_BLOCK];
    for (int j = 0; j < NF4_BLOCK; ++j) {
      if (am == 0.0f) {
        q[j] = 7;
        continue;
      }
      const float v = (float)bf16_to_double(wb[j]) / am; /* IEEE binary32 division */
      int idx = 0;
      for (int i = 0; i < 15; ++i)
        if ((double)v > mid[i]) ++idx;
      q[j] = idx;
    }
    for (int j = 0; j < NF4_BLOCK; j += 2) codes[(b * NF4_BLOCK + j) / 2] = (uint8_t)((q[j] << 4) | q[j + 1]);
  }
  return 0;
}

/* Dequantise to binary64 [n_out, k_in]: bf16(RN_binary32(level * absmax)). */
void oracle_c_nf4_dequantize(const uint8_t* codes, const float* absmax, long n_out, long k_in, double* w) {
  double lv[16];
  oracle_c_nf4_codebook(lv);
  const long n = n_out * k_in;
  for (long e = 0; e < n; ++e) {
    const uint8_t byte = codes[e / 2];
    const int q = (e % 2 == 0) ? (byte >> 4) : (byte & 0x0F);
    const float prod = (float)(lv[q] * (double)absmax[e / NF4_BLOCK]);
    w[e] = bf16_to_double(float_to_bf16_rne(prod));
  }
}

/* Forward of one projection, every operand row-major binary64:
 *   XA = X A [M, r],  Y = X W^T + s XA B [M, N];  X [M, K], W [N, K], A [K, r], B [r, N]. */
void oracle_c_linear_fwd(const double* X, const double* W, const double* A, const double* B, double s, long M,
                         long K, long N, long r, double* Y, double* XA) {
  for (long m = 0; m < M; ++m)
    for (long j = 0; j < r; ++j) {
      double acc = 0.0;
      for (long k = 0; k < K; ++k) acc += X[m * K + k] * A[k * r + j];
      XA[m * r + j] = acc;
    }
  for (long m = 0; m < M; ++m)
    for (long n = 0; n < N; ++n) {
      double acc = 0.0;
      for (long k = 0; k < K; ++k) acc += X[m * K + k] * W[n * K + k];
      double lora = 0.0;
      for (long j = 0; j < r; ++j) lora += XA[m * r + j] * B[j * N + n];
      Y[m * N + n] = acc + s * lora;
    }
}

/* Hand-derived backward, rank-r factor bracketed first, no gradient for W:
 *   G = dY B^T [M, r];  dX = dY W + s G A^T;  dA = s X^T G;  dB = s (X A)^T dY. */
void oracle_c_linear_bwd(const double* X, const double* W, const double* A, const double* B, double s,
                         const double* dY, long M, long K, long N, long r, double* dX, double* dA, double* dB,
                         double* G, double* XA) {
  for (long m = 0; m < M; ++m)
    for (long j = 0; j < r; ++j) {
      double g = 0.0, xa = 0.0;
      for (long n = 0; n < N; ++n) g += dY[m * N + n] * B[j * N + n];
      for (long k = 0; k < K; ++k) xa += X[m * K + k] * A[k * r + j];
      G[m * r + j] = g;
      XA[m * r + j] = xa;
    }
  for (long m = 0; m < M; ++m)
    for (long k = 0; k < K; ++k) {
      double acc = 0.0;
      for (long n = 0; n < N; ++n) acc += dY[m * N + n] * W[n * K + k];
      double lora = 0.0;
      for (long j = 0; j < r; ++j) lora += G[m * r + j] * A[k * r + j];
      dX[m * K + k] = acc + s * lora;
    }
  for (long k = 0; k < K; ++k)
    for (long j = 0; j < r; ++j) {
      double acc = 0.0;
      for (long m = 0; m < M; ++m) acc += X[m * K + k] * G[m * r + j];
      dA[k * r + j] = s * acc;
    }
  for (long j = 0; j < r; ++j)
    for (long n = 0; n < N; ++n) {
      double acc = 0.0;
      for (long m = 0; m < M; ++m) acc += XA[m * r + j] * dY[m * N + n];
      dB[j * N + n] = s * acc;
    }
}

/* ---------------------------------------------------------- gated MLP --
 * e = lin_g(X), g = lin_u(X), h = act(e) g, Y = lin_d(h), with act SiLU
 * (kind 0, e sigma(e)) or the tanh-approximate GELU (kind 1,
 * e/2 (1 + tanh(sqrt(2/pi) (e + 0.044715 e^3)))), as the Gemma blog's
 * "GeGLU 与 Swiglu 激活函数" section pairs them with the gated MLP.  The backward
 * is the chain rule: dh = dY W_d + s_d (dY B_d^T) A_d^T, de = dh g act'(e),
 * dg = dh act(e), dX = the gate backward of de plus the up backward of dg.
 * act' is differentiated here from the definitions:
 *   SiLU:      sigma + e sigma (1 - sigma);
 *   GELU-tanh: (1 + t)/2 + e/2 sech^2(u) du/de, sech^2 = 1 - t^2,
 *              u = c (e + 0.044715 e^3), du/de = c (1 + 3 * 0.044715 e^2). */
static double act_value(int kind, double e) {
  if (kind == 0) return e / (1.0 + exp(-e));
  const double c = sqrt(2.0 / acos(-1.0));
  return 0.5 * e * (1.0 + tanh(c * (e + 0.044715 * e * e * e)));
}

static double act_slope(int kind, double e) {
  if (kind == 0) {
    const double sig = 1.0 / (1.0 + exp(-e));
    return sig + e * sig * (1.0 - sig);
  }
  const double c = sqrt(2.0 / acos(-1.0));
  const double t = tanh(c * (e + 0.044715 * e * e * e));
  return 0.5 * (1.0 + t) + 0.5 * e * (1.0 - t * t) * c * (1.0 + 3.0 * 0.044715 * e * e);
}

/* One projection's operands: W [n_out, k_in], A [k_in, r], B [r, n_out], scale s. */
typedef struct {
  const double *W, *A, *B;
  double s;
} oracle_c_proj;

/* Forward: E, G, H [M, h], Y [M, d].  gate and up map d -> h, down maps h -> d.
 * Returns 0, or 1 if scratch memory could not be allocated. */
int oracle_c_mlp_fwd(int kind, const double* X, long M, long d, long h, long r, oracle_c_proj gate, oracle_c_proj up,
                     oracle_c_proj down, double* E, double* G, double* H, double* Y) {
  double* xa = malloc(sizeof(double) * (size_t)(M * r));
  if (!xa) return 1;
  oracle_c_linear_fwd(X, gate.W, gate.A, gate.B, gate.s, M, d, h, r, E, xa);
  oracle_c_linear_fwd(X, up.W, up.A, up.B, up.s, M, d, h, r, G, xa);
  for (long i = 0; i < M * h; ++i) H[i] = act_value(kind, E[i]) * G[i];
  oracle_c_linear_fwd(H, down.W, down.A, down.B, down.s, M, h, d, r, Y, xa);
  free(xa);
  return 0;
}

/* Backward from dY [M, d]: dX [M, d] and the six adapter gradients
 * dA_g, dA_u [d, r], dB_g, dB_u [r, h], dA_d [h, r], dB_d [r, d].
 * Recomputes the forward.  Returns 0, or 1 if scratch could not be allocated. */
int oracle_c_mlp_bwd(int kind, const double* X, long M, long d, long h, long r, oracle_c_proj gate, oracle_c_proj up,
                     oracle_c_proj down, const double* dY, double* dX, double* dA_g, double* dB_g, double* dA_u,
                     double* dB_u, double* dA_d, double* dB_d) {
  const size_t mh = (size_t)(M * h), md = (size_t)(M * d), mr = (size_t)(M * r);
  double* E = malloc(sizeof(double) * mh);
  double* G = malloc(sizeof(double) * mh);
  double* H = malloc(sizeof(double) * mh);
  double* Y = malloc(sizeof(double) * md);
  double* dH = malloc(sizeof(double) * mh);
  double* dE = malloc(sizeof(double) * mh);
  double* dG = malloc(sizeof(double) * mh);
  double* dXu = malloc(sizeof(double) * md);
  double* gs = malloc(sizeof(double) * mr);
  double* xa = malloc(sizeof(double) * mr);
  int rc = 1;
  if (E && G && H && Y && dH && dE && dG && dXu && gs && xa &&
      oracle_c_mlp_fwd(kind, X, M, d, h, r, gate, up, down, E, G, H, Y) == 0) {
    oracle_c_linear_bwd(H, down.W, down.A, down.B, down.s, dY, M, h, d, r, dH, dA_d, dB_d, gs, xa);
    for (size_t i = 0; i < mh; ++i) {
      dE[i] = dH[i] * G[i] * act_slope(kind, E[i]);
      dG[i] = dH[i] * act_value(kind, E[i]);
    }
    oracle_c_linear_bwd(X, gate.W, gate.A, gate.B, gate.s, dE, M, d, h, r, dX, dA_g, dB_g, gs, xa);
    oracle_c_linear_bwd(X, up.W, up.A, up.B, up.s, dG, M, d, h, r, dXu, dA_u, dB_u, gs, xa);
    for (size_t i = 0; i < md; ++i) dX[i] += dXu[i];
    rc = 0;
  }
  free(E);
  free(G);
  free(H);
  free(Y);
  free(dH);
  free(dE);
  free(dG);
  free(dXu);
  free(gs);
  free(xa);
  return rc;
}
