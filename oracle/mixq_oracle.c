/*
 * MixQ CPU oracle -- TEST INFRASTRUCTURE ONLY.
 *
 * Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline / reference
 * arm may load this library.  The product path (the CUDA library) never calls
 * it, and the two share no code, header, table or helper.
 *
 * It is a plain, slow, obviously-correct restatement of what the
 * outlier-decomposed mixed-precision linear layer computes.  Sources, cited by
 * page title and section/figure:
 *   [MixQ]   "一键部署LLM混合精度推理，端到端吞吐比AWQ最大提升6倍！" (MixQ, SC'24
 *            news article): 研究背景 Fig. 5 (matrix decomposition: low-bit dense
 *            part + FP16 outlier part, two products summed); MixQ的解决方案
 *            (outlier locality, Fig. 9; amax > threshold test; equivalent
 *            transformation, Fig. 10; order-preserved outlier matrix, Fig. 11;
 *            dequantize + scale + add of the low-precision result, Fig. 12).
 *   [QServe] "QServe W4A8KV4 Quantization and System Co-design" reading notes:
 *            渐进量化 (progressive group quantization: per-channel INT8 first,
 *            then the INT8 values group-quantized to 4 bits, so every product
 *            stays on INT8 tensor cores); group-wise (a scale s and zero z per
 *            g columns of a row); 寄存器压力和并行性 (weight dequantization in
 *            the mainloop; intermediates never overflow).
 *   [MixLLM] "MixLLM: Neuer Ansatz zur Optimierung der LLM-Quantisierung":
 *            "MixLLM: Ein neuer Ansatz" (8-bit symmetric activations, 4-bit
 *            asymmetric group-wise weights, two-stage dequantization on INT8
 *            tensor cores).
 *
 * Readings where the pages are silent (the same list is kept in the design notes):
 *   - scales are fp32; codes are symmetric in [-127, 127]; rounding is
 *     round-half-to-even of one fp32 multiply by the fp32 reciprocal 127/a;
 *   - the weight range a = max |W[n,:]| runs over ALL K columns;
 *   - "is there an outlier" is decided per token: mixed iff K_out > 0 and the
 *     token's amax is strictly greater than the threshold;
 *   - the outlier channel set used for arithmetic is the prepacked, sorted idx
 *     list (outlier locality); detection outside idx is only reported;
 *   - 4-bit level 2 uses integer scale s2 = max(1, ceil((hi-lo)/15)) and zero
 *     z2 = clamp(rint(-lo/s2), 0, 15), with q clamped so (q-z2)*s2 is int8;
 *   - 4-bit reading B quantizes the fp16 weights per group directly, with a
 *     real fp16 scale and an integer zero point over a range widened to hold
 *     0; its layer sums per-group INT32 partials of Xq * (q - z), each scaled
 *     by its group scale;
 *   - the final Y is evaluated in fp64 (the kernel's fp32 epilogue is checked
 *     against it within the stated tolerance);
 *   - the operation before the layer that the activation pass may absorb is
 *     the Llama RMSNorm x / sqrt(mean x^2 + eps) * g, evaluated in fp64 and
 *     rounded once to fp16 (a zero row with eps 0 stays zero).
 *
 * Floating point that decides an integer (a code, a threshold test, s2/z2) is
 * done in fp32 with single IEEE operations, the same precision the kernel
 * takes that decision in.  Build with -O2 -ffp-contract=off and no fast-math.
 *
 * fp16 values travel as raw IEEE binary16 bit patterns (uint16_t); conversion
 * uses the compiler's _Float16 type (exact widening, round-to-nearest-even
 * narrowing).
 *
 * Return codes: 0 ok, 1 invalid argument, 2 non-finite input, 3 int32 overflow.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_EINVAL 1
#define ORC_ENONFINITE 2
#define ORC_EOVERFLOW 3

static float h2f(uint16_t bits) {
  _Float16 h;
  memcpy(&h, &bits, sizeof h);
  return (float)h;
}

static uint16_t f2h_bits(double v) {
  _Float16 h = (_Float16)v;
  uint16_t bits;
  memcpy(&bits, &h, sizeof bits);
  return bits;
}

/* round half to even of an fp32 value (C rintf in the default rounding mode) */
static int32_t rint_even(float v) { return (int32_t)rintf(v); }

static int32_t clamp_i32(int32_t v, int32_t lo, int32_t hi) {
  return v < lo ? lo : (v > hi ? hi : v);
}

/* idx must be sorted ascending, unique, inside [0, K).  Fills mask[k] = 1 for
 * k in idx. [MixQ] Fig. 11: the outlier columns keep their original order. */
static int build_outlier_mask(const int32_t *idx, int K_out, int K, uint8_t *mask) {
  if (K_out < 0 || K_out > K) return ORC_EINVAL;
  memset(mask, 0, (size_t)K);
  for (int j = 0; j < K_out; ++j) {
    if (idx[j] < 0 || idx[j] >= K) return ORC_EINVAL;
    if (j > 0 && idx[j] <= idx[j - 1]) return ORC_EINVAL;
    mask[idx[j]] = 1;
  }
  return ORC_OK;
}

/* Symmetric per-row INT8 quantization of a real vector with range a:
 * s = a/127, code = clamp(rint(x * (127/a)), -127, 127), all codes 0 if a == 0. */
static float quant_scale(float a) { return a / 127.0f; }
static float quant_inv(float a) { return a > 0.0f ? 127.0f / a : 0.0f; }
static int8_t quant_code(float x, float inv) {
  float v = x * inv;
  return (int8_t)clamp_i32(rint_even(v), -127, 127);
}

/*
 * Weight prepack, 8-bit ([MixQ] Fig. 5: weights stored in low bits; per
 * output channel symmetric INT8), plus extraction of the outlier weight
 * columns in idx order ([MixQ] Fig. 11).
 *   W      [N][K] fp16 bits, row-major
 *   Wq     [N][K] int8 codes
 *   s_w    [N]    fp32 per-output-channel scale
 *   W_out  [N][K_out_pad] fp16 bits; column j < K_out is W[:, idx[j]], the
 *          rest is +0.0
 */
int oracle_prepack_w8(const uint16_t *W, int N, int K, const int32_t *idx, int K_out,
                      int K_out_pad, int8_t *Wq, float *s_w, uint16_t *W_out) {
  if (N < 0 || K <= 0 || K_out_pad < K_out) return ORC_EINVAL;
  uint8_t *mask = (uint8_t *)malloc((size_t)K);
  if (!mask) return ORC_EINVAL;
  int rc = build_outlier_mask(idx, K_out, K, mask);
  free(mask);
  if (rc) return rc;
  for (int n = 0; n < N; ++n) {
    const uint16_t *w = W + (size_t)n * K;
    float a = 0.0f;
    for (int k = 0; k < K; ++k) {
      float v = h2f(w[k]);
      if (!isfinite(v)) return ORC_ENONFINITE;
      float m = fabsf(v);
      if (m > a) a = m;
    }
    s_w[n] = quant_scale(a);
    float inv = quant_inv(a);
    for (int k = 0; k < K; ++k) Wq[(size_t)n * K + k] = quant_code(h2f(w[k]), inv);
    for (int j = 0; j < K_out_pad; ++j)
      W_out[(size_t)n * K_out_pad + j] = j < K_out ? w[idx[j]] : (uint16_t)0;
  }
  return ORC_OK;
}

/*
 * Weight prepack, 4-bit progressive level 2 ([QServe] 渐进量化 + group-wise;
 * [MixLLM] two-stage dequantization onto INT8 tensor cores).  Input is the
 * level-1 INT8 code matrix from oracle_prepack_w8.  For every row n and group
 * of G = 128 consecutive k:
 *   lo = min w8, hi = max w8
 *   s2 = max(1, ceil((hi - lo) / 15))                    (integer, <= 17)
 *   z2 = clamp(rint(-lo / s2), 0, 15)
 *   q  = clamp(rint(w8 / s2) + z2, qlo, qhi),
 *        qlo = max(0,  z2 + ceil(-128 / s2)), qhi = min(15, z2 + floor(127 / s2))
 *   w8eff = (q - z2) * s2                                 (always in [-128, 127])
 * Outputs are logical (unpacked) values:
 *   q [N][K], s2 [N][K/128], z2 [N][K/128], w8eff [N][K].
 */
#define ORC_GROUP 128
int oracle_prepack_w4(const int8_t *Wq8, int N, int K, uint8_t *q, uint8_t *s2, uint8_t *z2,
                      int8_t *w8eff) {
  if (N < 0 || K <= 0 || K % ORC_GROUP != 0) return ORC_EINVAL;
  const int ng = K / ORC_GROUP;
  for (int n = 0; n < N; ++n) {
    for (int g = 0; g < ng; ++g) {
      const int8_t *w = Wq8 + (size_t)n * K + (size_t)g * ORC_GROUP;
      int lo = 127, hi = -127;
      for (int i = 0; i < ORC_GROUP; ++i) {
        if (w[i] < lo) lo = w[i];
        if (w[i] > hi) hi = w[i];
      }
      int span = hi - lo; /* >= 0 */
      int scale = (span + 14) / 15;
      if (scale < 1) scale = 1;
      int zero = clamp_i32(rint_even(-(float)lo / (float)scale), 0, 15);
      int qlo = zero - 128 / scale; /* z2 + ceil(-128/s2) */
      if (qlo < 0) qlo = 0;
      int qhi = zero + 127 / scale; /* z2 + floor(127/s2) */
      if (qhi > 15) qhi = 15;
      s2[(size_t)n * ng + g] = (uint8_t)scale;
      z2[(size_t)n * ng + g] = (uint8_t)zero;
      for (int i = 0; i < ORC_GROUP; ++i) {
        int code = clamp_i32(rint_even((float)w[i] / (float)scale) + zero, qlo, qhi);
        size_t at = (size_t)n * K + (size_t)g * ORC_GROUP + i;
        q[at] = (uint8_t)code;
        w8eff[at] = (int8_t)((code - zero) * scale);
      }
    }
  }
  return ORC_OK;
}

/*
 * Weight prepack, 4-bit reading B ([MixLLM] "MixLLM: Ein neuer Ansatz": 4-bit
 * weights quantized asymmetrically per group, 8-bit activations, a two-step
 * dequantization that keeps the products on INT8 tensor cores, and a fast
 * integer-to-float conversion of the results).  Unlike reading A there is no
 * per-row INT8 level: the fp16 weights go to 4 bits directly, with a real
 * (fp16) scale and an integer zero point per row and group of G = 128 k.
 * Reading: the two-step dequantization must end in INT8 operands, so the
 * zero point is an integer subtracted before the product (step 1: q - z in
 * [-15, 15]); the real scale multiplies the group's INT32 partial sum after
 * it (step 2, converted to float).  The group range is widened to contain 0,
 * so z is always one of the 16 codes.  For every row n and group g:
 *   lo = min(0, min W), hi = max(0, max W)               (fp32, exact)
 *   s  = fp16( (hi - lo) / 15 )                          (fp32 ops, then fp16)
 *   if s == 0:  z = 0, q = 0                             (an all-zero group)
 *   else:       z = clamp(rint(-lo / s), 0, 15)
 *               q = clamp(rint(W / s) + z, 0, 15)        (s as stored, fp32)
 * The effective weight is s * (q - z).  Outputs are logical (unpacked):
 *   q [N][K] u8, s_g [N][K/128] fp16 bits, z_g [N][K/128] u8.
 */
int oracle_prepack_w4b(const uint16_t *W, int N, int K, uint8_t *q, uint16_t *s_g,
                       uint8_t *z_g) {
  if (N < 0 || K <= 0 || K % ORC_GROUP != 0) return ORC_EINVAL;
  const int ng = K / ORC_GROUP;
  for (int n = 0; n < N; ++n) {
    for (int g = 0; g < ng; ++g) {
      const uint16_t *w = W + (size_t)n * K + (size_t)g * ORC_GROUP;
      float lo = 0.0f, hi = 0.0f;
      for (int i = 0; i < ORC_GROUP; ++i) {
        float v = h2f(w[i]);
        if (!isfinite(v)) return ORC_ENONFINITE;
        if (v < lo) lo = v;
        if (v > hi) hi = v;
      }
      float range = hi - lo;
      uint16_t s_bits = f2h_bits((double)(range / 15.0f));
      float s = h2f(s_bits);
      int zero = 0;
      if (s > 0.0f) zero = clamp_i32(rint_even(-lo / s), 0, 15);
      s_g[(size_t)n * ng + g] = s_bits;
      z_g[(size_t)n * ng + g] = (uint8_t)zero;
      for (int i = 0; i < ORC_GROUP; ++i) {
        int code = s > 0.0f ? clamp_i32(rint_even(h2f(w[i]) / s) + zero, 0, 15) : 0;
        q[(size_t)n * K + (size_t)g * ORC_GROUP + i] = (uint8_t)code;
      }
    }
  }
  return ORC_OK;
}

/*
 * The layer with reading-B weights for rows [m0, m1) ([MixLLM] two-step
 * dequantization; [MixQ] Fig. 5 + Fig. 12 for the outlier part):
 *   P[m,n,g] = sum_{k in g} Xq[m,k] * (q[n,k] - z[n,g])     (exact integer)
 *   y[m,n]   = s_x[m] * sum_g s[n,g] * P[m,n,g]              (fp64)
 *            + sum_{j < K_out_pad} X_out[m,j] * W_out[n,j]    (fp64)
 * The activation codes and scales are those of the per-token activation
 * pass.  part (nullable) is [(m1-m0)][N][K/128]; y is [(m1-m0)][N].
 */
int oracle_linear_w4b(const int8_t *Xq, const float *s_x, const uint16_t *X_out,
                      const uint8_t *q, const uint16_t *s_g, const uint8_t *z_g,
                      const uint16_t *W_out, int M, int N, int K, int K_out_pad, int m0, int m1,
                      int32_t *part, double *y) {
  if (m0 < 0 || m1 > M || m0 > m1 || N < 0 || K <= 0 || K % ORC_GROUP != 0 || K_out_pad < 0)
    return ORC_EINVAL;
  const int ng = K / ORC_GROUP;
#pragma omp parallel for schedule(dynamic, 1)
  for (int m = m0; m < m1; ++m) {
    for (int n = 0; n < N; ++n) {
      double acc = 0.0;
      for (int g = 0; g < ng; ++g) {
        int64_t p = 0;
        const int z = z_g[(size_t)n * ng + g];
        for (int i = 0; i < ORC_GROUP; ++i) {
          size_t k = (size_t)g * ORC_GROUP + i;
          p += (int64_t)Xq[(size_t)m * K + k] * (int64_t)((int)q[(size_t)n * K + k] - z);
        }
        if (part) part[((size_t)(m - m0) * N + n) * ng + g] = (int32_t)p;
        acc += (double)h2f(s_g[(size_t)n * ng + g]) * (double)p;
      }
      double o = 0.0;
      for (int j = 0; j < K_out_pad; ++j)
        o += (double)h2f(X_out[(size_t)m * K_out_pad + j]) * (double)h2f(W_out[(size_t)n * K_out_pad + j]);
      y[(size_t)(m - m0) * N + n] = (double)s_x[m] * acc + o;
    }
  }
  return ORC_OK;
}

/*
 * Same as oracle_linear_w4b, but only at P sampled output points (ms[p],
 * ns[p]); part (nullable) is [P][K/128], y is [P].
 */
int oracle_linear_w4b_points(const int8_t *Xq, const float *s_x, const uint16_t *X_out,
                             const uint8_t *q, const uint16_t *s_g, const uint8_t *z_g,
                             const uint16_t *W_out, int M, int N, int K, int K_out_pad,
                             const int32_t *ms, const int32_t *ns, int P, int32_t *part,
                             double *y) {
  if (N < 0 || K <= 0 || K % ORC_GROUP != 0 || K_out_pad < 0 || P < 0) return ORC_EINVAL;
  for (int i = 0; i < P; ++i)
    if (ms[i] < 0 || ms[i] >= M || ns[i] < 0 || ns[i] >= N) return ORC_EINVAL;
  const int ng = K / ORC_GROUP;
#pragma omp parallel for schedule(static)
  for (int i = 0; i < P; ++i) {
    const int m = ms[i], n = ns[i];
    double acc = 0.0;
    for (int g = 0; g < ng; ++g) {
      int64_t sum = 0;
      const int z = z_g[(size_t)n * ng + g];
      for (int t = 0; t < ORC_GROUP; ++t) {
        size_t k = (size_t)g * ORC_GROUP + t;
        sum += (int64_t)Xq[(size_t)m * K + k] * (int64_t)((int)q[(size_t)n * K + k] - z);
      }
      if (part) part[(size_t)i * ng + g] = (int32_t)sum;
      acc += (double)h2f(s_g[(size_t)n * ng + g]) * (double)sum;
    }
    double o = 0.0;
    for (int j = 0; j < K_out_pad; ++j)
      o += (double)h2f(X_out[(size_t)m * K_out_pad + j]) * (double)h2f(W_out[(size_t)n * K_out_pad + j]);
    y[i] = (double)s_x[m] * acc + o;
  }
  return ORC_OK;
}

/*
 * RMS normalisation of each token: the operation before the layer, which the
 * activation pass can absorb ([MixQ] MixQ的解决方案: the amax of quantization
 * can be taken inside the preceding operation).  The pages give no formula for
 * that operation; reading: the Llama RMSNorm
 *   Y[m,k] = fp16( X[m,k] / sqrt(mean_k X[m,k]^2 + eps) * g[k] ),
 * evaluated in fp64 (sum, mean, square root, division, both products) and
 * rounded once to fp16, round to nearest even.
 *   X [M][ldx] fp16 bits, g [K] fp16 bits, eps >= 0, Y [M][K] fp16 bits.
 */
int oracle_rmsnorm(const uint16_t *X, int M, int K, int ldx, const uint16_t *g, double eps,
                   uint16_t *Y) {
  if (M < 0 || K <= 0 || ldx < K || !(eps >= 0.0) || !isfinite(eps)) return ORC_EINVAL;
  for (int k = 0; k < K; ++k)
    if (!isfinite(h2f(g[k]))) return ORC_ENONFINITE;
  for (int m = 0; m < M; ++m) {
    const uint16_t *x = X + (size_t)m * ldx;
    double ss = 0.0;
    for (int k = 0; k < K; ++k) {
      double v = (double)h2f(x[k]);
      if (!isfinite(v)) return ORC_ENONFINITE;
      ss += v * v;
    }
    double den = sqrt(ss / (double)K + eps);
    for (int k = 0; k < K; ++k) {
      double v = den > 0.0 ? (double)h2f(x[k]) / den * (double)h2f(g[k]) : 0.0;
      Y[(size_t)m * K + k] = f2h_bits(v);
    }
  }
  return ORC_OK;
}

/*
 * Activation quantization with outlier detection ([MixQ] MixQ的解决方案: the
 * amax taken for quantization tells whether outliers exist -- amax greater
 * than the threshold means yes; Fig. 10 equivalent transformation
 * X = X_dense + X_outlier; Fig. 11 order-preserved outlier matrix).
 * For each token m:
 *   aI = max_{k in idx} |x|,  aN = max_{k not in idx} |x|
 *   mixed = K_out > 0 && max(aI, aN) > T            (strictly greater)
 *   a = mixed ? aN : max(aI, aN);  s_x[m] = a / 127
 *   Xq[m,k] = (mixed && k in idx) ? 0 : clamp(rint(x * 127/a), -127, 127)
 *   X_out[m,j] = (mixed && j < K_out) ? X[m, idx[j]] : +0.0   (j < K_out_pad)
 * Over the whole matrix:
 *   bitmap bit k (word k/32, bit k%32) = max_m |X[m,k]| > T
 *   flags[0] = number of mixed tokens
 *   flags[1] = number of detected channels (bitmap) that are not in idx
 * X is [M][ldx] fp16 bits; Xq is [M][K]; X_out is [M][K_out_pad].
 */
int oracle_quantize_act(const uint16_t *X, int M, int K, int ldx, const int32_t *idx, int K_out,
                        int K_out_pad, float T, int8_t *Xq, float *s_x, uint16_t *X_out,
                        uint32_t *bitmap, int32_t *flags) {
  if (M < 0 || K <= 0 || ldx < K || K_out_pad < K_out) return ORC_EINVAL;
  uint8_t *mask = (uint8_t *)malloc((size_t)K);
  uint8_t *hit = (uint8_t *)calloc((size_t)K, 1);
  if (!mask || !hit) {
    free(mask);
    free(hit);
    return ORC_EINVAL;
  }
  int rc = build_outlier_mask(idx, K_out, K, mask);
  int32_t mixed_tokens = 0;
  for (int m = 0; m < M && rc == ORC_OK; ++m) {
    const uint16_t *x = X + (size_t)m * ldx;
    float aI = 0.0f, aN = 0.0f;
    for (int k = 0; k < K; ++k) {
      float v = h2f(x[k]);
      if (!isfinite(v)) {
        rc = ORC_ENONFINITE;
        break;
      }
      float mag = fabsf(v);
      if (mask[k]) {
        if (mag > aI) aI = mag;
      } else {
        if (mag > aN) aN = mag;
      }
      if (mag > T) hit[k] = 1;
    }
    if (rc) break;
    float amax = aI > aN ? aI : aN;
    int mixed = K_out > 0 && amax > T;
    float a = mixed ? aN : amax;
    s_x[m] = quant_scale(a);
    float inv = quant_inv(a);
    for (int k = 0; k < K; ++k)
      Xq[(size_t)m * K + k] = (mixed && mask[k]) ? (int8_t)0 : quant_code(h2f(x[k]), inv);
    for (int j = 0; j < K_out_pad; ++j)
      X_out[(size_t)m * K_out_pad + j] = (mixed && j < K_out) ? x[idx[j]] : (uint16_t)0;
    mixed_tokens += mixed;
  }
  if (rc == ORC_OK) {
    int words = (K + 31) / 32;
    int32_t outside = 0;
    for (int w = 0; w < words; ++w) bitmap[w] = 0;
    for (int k = 0; k < K; ++k) {
      if (hit[k]) {
        bitmap[k / 32] |= 1u << (k % 32);
        if (!mask[k]) ++outside;
      }
    }
    flags[0] = mixed_tokens;
    flags[1] = outside;
  }
  free(mask);
  free(hit);
  return rc;
}

/*
 * INT8 product of the dense part ([MixQ] Fig. 5, low-precision matmul):
 *   acc[m,n] = sum_k Xq[m,k] * Wq[n,k]   for rows m in [m0, m1)
 * accumulated in int64 and required to fit int32 (the kernel accumulates in
 * int32).  acc is [(m1-m0)][N].
 */
int oracle_gemm_i32(const int8_t *Xq, const int8_t *Wq, int M, int N, int K, int m0, int m1,
                    int32_t *acc) {
  if (m0 < 0 || m1 > M || m0 > m1 || N < 0 || K <= 0) return ORC_EINVAL;
  int overflow = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : overflow)
  for (int m = m0; m < m1; ++m) {
    for (int n = 0; n < N; ++n) {
      int64_t s = 0;
      for (int k = 0; k < K; ++k) s += (int64_t)Xq[(size_t)m * K + k] * (int64_t)Wq[(size_t)n * K + k];
      if (s > INT32_MAX || s < INT32_MIN) overflow = 1;
      acc[(size_t)(m - m0) * N + n] = (int32_t)s;
    }
  }
  return overflow ? ORC_EOVERFLOW : ORC_OK;
}

/*
 * The whole mixed-precision linear layer for rows [m0, m1) ([MixQ] Fig. 5 +
 * Fig. 12: the INT32 result is dequantized, scaled and added to the FP16
 * outlier product):
 *   acc[m,n] = sum_k Xq[m,k] * Wq[n,k]                         (exact integer)
 *   o[m,n]   = sum_{j < K_out_pad} X_out[m,j] * W_out[n,j]      (fp64)
 *   y[m,n]   = acc[m,n] * s_x[m] * s_w[n] + o[m,n]              (fp64)
 * Wq is the effective INT8 weight (level-1 codes for W8, w8eff for W4).
 * acc (nullable) and y are [(m1-m0)][N]; X_out/W_out may be NULL if
 * K_out_pad == 0.
 */
int oracle_linear(const int8_t *Xq, const float *s_x, const uint16_t *X_out, const int8_t *Wq,
                  const float *s_w, const uint16_t *W_out, int M, int N, int K, int K_out_pad,
                  int m0, int m1, int32_t *acc, double *y) {
  if (m0 < 0 || m1 > M || m0 > m1 || N < 0 || K <= 0 || K_out_pad < 0) return ORC_EINVAL;
  int overflow = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : overflow)
  for (int m = m0; m < m1; ++m) {
    for (int n = 0; n < N; ++n) {
      int64_t s = 0;
      for (int k = 0; k < K; ++k) s += (int64_t)Xq[(size_t)m * K + k] * (int64_t)Wq[(size_t)n * K + k];
      if (s > INT32_MAX || s < INT32_MIN) overflow = 1;
      double o = 0.0;
      for (int j = 0; j < K_out_pad; ++j)
        o += (double)h2f(X_out[(size_t)m * K_out_pad + j]) * (double)h2f(W_out[(size_t)n * K_out_pad + j]);
      size_t at = (size_t)(m - m0) * N + n;
      if (acc) acc[at] = (int32_t)s;
      y[at] = (double)s * (double)s_x[m] * (double)s_w[n] + o;
    }
  }
  return overflow ? ORC_EOVERFLOW : ORC_OK;
}

/*
 * Same as oracle_linear, but only at P sampled output points (ms[p], ns[p]);
 * used to check full-size launches element by element at sampled outputs.
 */
int oracle_linear_points(const int8_t *Xq, const float *s_x, const uint16_t *X_out,
                         const int8_t *Wq, const float *s_w, const uint16_t *W_out, int M, int N,
                         int K, int K_out_pad, const int32_t *ms, const int32_t *ns, int P,
                         int32_t *acc, double *y) {
  if (N < 0 || K <= 0 || K_out_pad < 0 || P < 0) return ORC_EINVAL;
  for (int p = 0; p < P; ++p)
    if (ms[p] < 0 || ms[p] >= M || ns[p] < 0 || ns[p] >= N) return ORC_EINVAL;
  int overflow = 0;
#pragma omp parallel for schedule(static) reduction(| : overflow)
  for (int p = 0; p < P; ++p) {
    int m = ms[p], n = ns[p];
    int64_t s = 0;
    for (int k = 0; k < K; ++k) s += (int64_t)Xq[(size_t)m * K + k] * (int64_t)Wq[(size_t)n * K + k];
    if (s > INT32_MAX || s < INT32_MIN) overflow = 1;
    double o = 0.0;
    for (int j = 0; j < K_out_pad; ++j)
      o += (double)h2f(X_out[(size_t)m * K_out_pad + j]) * (double)h2f(W_out[(size_t)n * K_out_pad + j]);
    if (acc) acc[p] = (int32_t)s;
    y[p] = (double)s * (double)s_x[m] * (double)s_w[n] + o;
  }
  return overflow ? ORC_EOVERFLOW : ORC_OK;
}

/* fp16 rounding of fp64 values (round to nearest even), as bit patterns. */
void oracle_round_f16(const double *v, long long n, uint16_t *out) {
  for (long long i = 0; i < n; ++i) out[i] = f2h_bits(v[i]);
}
