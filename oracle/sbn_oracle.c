/*
 * Sparse-BitLinear forward: CPU ORACLE.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, literal restatement of
 * what the Sparse-BitLinear forward computes.  It is used by the test-suite, by the
 * smoke check and by the benchmark's CPU-baseline leg, and by nothing else.  It
 * shares no code, header, table or helper with the CUDA library; neither side
 * includes or links the other.
 *
 * Sources (web pages; cited by title and section):
 *   [SBN-es]  "Sparse-BitNet: 1.58-bit LLMs are Naturally Friendly to Semi-Structured
 *             Sparsity", gist.science technical summary (Spanish), section
 *             "2. Metodología: Sparse-BitNet" (Sparse-BitLinear, mask generation,
 *             quant-then-mask order, dynamic recomputation).
 *   [SBN-ar]  Same paper, gist.science technical summary (Arabic), section 2
 *             "Methodology: Sparse-BitNet" (items 1-3 of the Sparse-BitLinear
 *             architecture; "mask generation" and "quant-then-mask order").
 *   [BitNet.cpp] "Marco de inferencia de Microsoft lleva modelos de lenguaje grande de
 *             1 bit a dispositivos locales" (unite.ai), section "Fundamento
 *             matemático", items 2 (activation quantisation) and 3 (BitLinear op).
 *   [BitNet-proj] "Introducción Detallada al Proyecto BitNet" (aibars.net), section
 *             "Especificaciones Técnicas" (W1.58A8, absmean weights, 8-bit activations,
 *             no bias).
 *
 * Readings where the pages are silent (each one is listed in the design notes):
 *   - gamma is per tensor, over all masters before masking, and the mean |W| is taken
 *     as an exact integer sum of trunc(|W| * 2^24) so that it does not depend on the
 *     summation order; eps is added in fp32.
 *   - round() is round-half-to-even; W/g and 127*x/s are IEEE fp32 divisions, because
 *     fp32 is the precision in which the GPU takes the same integer decisions.
 *   - M-groups run along the input dimension K inside one output row; the top-N rule
 *     ranks |W_master| and the lower index wins a tie.
 *   - Qb = 127, symmetric clip to [-127, 127]; the per-token scale is
 *     max(max|x|, 1e-5).
 *   - y = acc * g * s / 127 is evaluated in fp64 here (no rounding order is fixed by
 *     the pages); the GPU's fp32 result is compared to it with a relative tolerance.
 *
 * Build: gcc -O2 -ffp-contract=off -fno-fast-math -fopenmp -shared -fPIC.
 */
#include <fenv.h>
#include <math.h>
#include <stdint.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_ERR_W_NONFINITE 1
#define ORACLE_ERR_W_RANGE 2
#define ORACLE_ERR_X_NONFINITE 4
#define ORACLE_ERR_ACC_OVERFLOW 8

static float bf16_bits_to_float(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return f;
}

/* 1 when the host FPU rounds to nearest-even (every decision below assumes it). */
int oracle_rounding_is_nearest(void) { return fegetround() == FE_TONEAREST; }

int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/*
 * S1: per-tensor absmean scale [SBN-ar §2 item 1: gamma is the mean absolute value of
 * the weights; BitNet-proj: "absmean" weight quantisation].
 *   S     = sum_i trunc(|W_i| * 2^24)                 (exact, unsigned 64-bit)
 *   gamma = fp32( fp64(S) / (fp64(n) * 2^24) )
 *   g     = fp32( gamma + eps )
 * Elements that are NaN/Inf set ORACLE_ERR_W_NONFINITE, elements with |W| >= 256 set
 * ORACLE_ERR_W_RANGE; such elements are left out of S (the outputs are then
 * unspecified).  Returns the error bits.
 */
int oracle_weight_gamma(const uint16_t *W, int64_t n, float eps, uint64_t *S_out,
                        float *gamma_out, float *g_out) {
  uint64_t S = 0;
  int err = 0;
#pragma omp parallel for reduction(+ : S) reduction(| : err) schedule(static)
  for (int64_t i = 0; i < n; ++i) {
    float a = fabsf(bf16_bits_to_float(W[i]));
    if (!isfinite(a)) {
      err |= ORACLE_ERR_W_NONFINITE;
      continue;
    }
    if (a >= 256.0f) {
      err |= ORACLE_ERR_W_RANGE;
      continue;
    }
    double scaled = (double)a * 16777216.0; /* exact: 8-bit significand times 2^24 */
    S += (uint64_t)scaled;                  /* C conversion truncates toward zero */
  }
  float gamma = (float)((double)S / ((double)n * 16777216.0));
  float g = gamma + eps;
  if (S_out) *S_out = S;
  if (gamma_out) *gamma_out = gamma;
  if (g_out) *g_out = g;
  return err;
}

/*
 * S2: ternary code of one master weight [SBN-ar §2 item 1; BitNet-proj "Especificaciones
 * Técnicas"]: t = clamp(round(w / g), -1, 1) with an fp32 division and round-half-even.
 * A NaN quotient (only 0/0, when g == 0 and w == +-0) gives 0.
 */
static int8_t ternary_code(float w, float g) {
  float q = w / g;
  float r = rintf(q);
  if (r >= 1.0f) return 1;
  if (r <= -1.0f) return -1;
  return 0;
}

/*
 * S2 + S3 + S4(apply): codes, N:M mask and masked codes for a [O, K] master matrix.
 * Mask [SBN-es §2 "Generación de Máscara"; SBN-ar §2 "mask generation"]: inside each
 * group of M consecutive weights along K (aligned at multiples of M) keep position i iff
 *   #{ j in group : |W_j| > |W_i|  or  (|W_j| == |W_i| and j < i) }  <  N,
 * i.e. the N largest master magnitudes, lower index first on ties.
 * Order [SBN-es §2 "Orden de Operaciones"; SBN-ar §2 quant-then-mask]: the codes are
 * computed from all masters first, then the mask zeroes the pruned positions:
 *   ws = keep ? t : 0.
 * Outputs are [O, K] int8 / uint8 arrays (t, keep in {0,1}, ws); any may be NULL.
 */
void oracle_ternary_mask(const uint16_t *W, int64_t O, int64_t K, int N, int M, float g,
                         int8_t *t_out, uint8_t *keep_out, int8_t *ws_out) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < O; ++r) {
    for (int64_t base = 0; base < K; base += M) {
      float mag[8];
      for (int i = 0; i < M; ++i) mag[i] = fabsf(bf16_bits_to_float(W[r * K + base + i]));
      for (int i = 0; i < M; ++i) {
        int rank = 0;
        for (int j = 0; j < M; ++j) {
          if (j == i) continue;
          if (mag[j] > mag[i] || (mag[j] == mag[i] && j < i)) ++rank;
        }
        int64_t idx = r * K + base + i;
        uint8_t keep = (uint8_t)(rank < N);
        int8_t t = ternary_code(bf16_bits_to_float(W[idx]), g);
        if (t_out) t_out[idx] = t;
        if (keep_out) keep_out[idx] = keep;
        if (ws_out) ws_out[idx] = keep ? t : 0;
      }
    }
  }
}

/*
 * S4 (pack): the hardware format of the masked ternary matrix.  The pages ask for "2-bit
 * codes" with "well-defined N:M metadata on the discrete weights" [SBN-ar §2
 * quant-then-mask]; the layout below is this library's reading of it.
 *
 * Which positions the codes plane stores:
 *   pattern 2:4 (the pattern the sparse tensor cores consume): only the kept positions of
 *     each row, in ascending K order (K/2 stored elements per row);
 *   every other pattern: every position of the row in ascending K order, pruned positions
 *     holding the code of 0 (K stored elements per row).
 * Codes plane, row r: stored element e sits in the little-endian 32-bit word e/16 of the
 *   row; inside that word, with j = (e%16)/4 and k = e%4, it occupies bits
 *   [8k + 6 - 2j, 8k + 7 - 2j] (byte k, bit 6 - 2j).  A code is the 2-bit two's complement
 *   of the ternary value: 0 -> 00, +1 -> 01, -1 -> 11 (10 is never written).
 * Meta plane, row r, group g (M consecutive positions):
 *   pattern 2:4: the two kept positions i0 < i1 of the group as the nibble i0 | i1 << 2;
 *   other M == 4 patterns: the 4-bit keep mask (bit i = position i kept);
 *   M == 8: the 8-bit keep mask, one byte per group;
 *   nibbles: group 2h in the low nibble of byte h, group 2h+1 in the high nibble.
 * Rows are ldc / ldm bytes apart; every byte past a row's data is zero.
 * Returns 0, or -1 if some group does not keep exactly N positions.
 */
int oracle_pack(const int8_t *t, const uint8_t *keep, int64_t O, int64_t K, int N, int M,
                uint8_t *codes, int64_t ldc, uint8_t *meta, int64_t ldm) {
  int bad = 0;
  int compact = (N == 2 && M == 4);
  memset(codes, 0, (size_t)(O * ldc));
  memset(meta, 0, (size_t)(O * ldm));
#pragma omp parallel for reduction(| : bad) schedule(static)
  for (int64_t r = 0; r < O; ++r) {
    int64_t e = 0;
    for (int64_t k = 0; k < K; ++k) {
      int kept = keep[r * K + k];
      if (compact && !kept) continue;
      int8_t v = kept ? t[r * K + k] : 0;
      uint8_t code = (v == 0) ? 0u : (v == 1 ? 1u : 3u);
      int64_t byte = 4 * (e / 16) + e % 4;
      int shift = 6 - 2 * (int)((e % 16) / 4);
      if (byte >= ldc) { /* more stored elements than the plane holds */
        bad = 1;
        break;
      }
      codes[r * ldc + byte] |= (uint8_t)(code << shift);
      ++e;
    }
    for (int64_t gi = 0; gi < K / M; ++gi) {
      unsigned bits = 0, idx = 0;
      int kept = 0;
      for (int i = 0; i < M; ++i) {
        if (keep[r * K + gi * M + i]) {
          bits |= 1u << i;
          if (kept < 2) idx |= (unsigned)i << (2 * kept);
          ++kept;
        }
      }
      if (kept != N) bad = 1;
      if (M == 8)
        meta[r * ldm + gi] = (uint8_t)bits;
      else
        meta[r * ldm + gi / 2] |= (uint8_t)((compact ? idx : bits) << (4 * (gi % 2)));
    }
  }
  return bad ? -1 : 0;
}

/*
 * S5: per-token absmax int8 activations [BitNet.cpp "Fundamento matemático" item 2:
 * x_q = Clip(x * Qb / gamma_x, -Qb + eps, Qb - eps), gamma_x = max |x|; BitNet-proj
 * W1.58A8].  With Qb = 127:
 *   s = max(max_k |x_k|, 1e-5)                         (fp32)
 *   q = clamp(round_half_even((127 * x) / s), -127, 127)  (fp32 product is exact)
 * X is [T, K] bf16 bits; Xq is [T, K] int8; s_out is [T] fp32.  Returns error bits.
 */
int oracle_quant_acts(const uint16_t *X, int64_t T, int64_t K, int8_t *Xq, float *s_out) {
  int err = 0;
#pragma omp parallel for reduction(| : err) schedule(static)
  for (int64_t t = 0; t < T; ++t) {
    float a = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
      float v = fabsf(bf16_bits_to_float(X[t * K + k]));
      if (!isfinite(v)) {
        err |= ORACLE_ERR_X_NONFINITE;
        continue;
      }
      if (v > a) a = v;
    }
    float s = (a < 1e-5f) ? 1e-5f : a;
    s_out[t] = s;
    for (int64_t k = 0; k < K; ++k) {
      float x = bf16_bits_to_float(X[t * K + k]);
      float r = rintf((127.0f * x) / s);
      if (r > 127.0f) r = 127.0f;
      if (r < -127.0f) r = -127.0f;
      if (r != r) r = 0.0f; /* only reachable for non-finite x (flagged above) */
      Xq[t * K + k] = (int8_t)r;
    }
  }
  return err;
}

/*
 * S6: exact integer contraction [BitNet.cpp item 3; the ternary product is a signed sum]:
 *   acc[t, o] = sum_k Xq[t, k] * Ws[o, k]   (accumulated in int64, stored as int32)
 * Returns ORACLE_ERR_ACC_OVERFLOW if any sum leaves the int32 range.
 */
int oracle_contract(const int8_t *Xq, const int8_t *Ws, int64_t T, int64_t O, int64_t K,
                    int32_t *acc) {
  int err = 0;
#pragma omp parallel for reduction(| : err) schedule(static)
  for (int64_t o = 0; o < O; ++o) {
    for (int64_t t = 0; t < T; ++t) {
      int64_t sum = 0;
      for (int64_t k = 0; k < K; ++k) sum += (int64_t)Xq[t * K + k] * (int64_t)Ws[o * K + k];
      if (sum > INT32_MAX || sum < INT32_MIN) err |= ORACLE_ERR_ACC_OVERFLOW;
      acc[t * O + o] = (int32_t)sum;
    }
  }
  return err;
}

/*
 * S7: dequantising rescale [BitNet.cpp item 3: y = W x (beta * gamma / Qb)], here
 *   y[t, o] = acc[t, o] * g * s[t] / 127    evaluated in fp64.
 */
void oracle_rescale(const int32_t *acc, const float *s, float g, int64_t T, int64_t O,
                    double *y) {
  for (int64_t t = 0; t < T; ++t)
    for (int64_t o = 0; o < O; ++o)
      y[t * O + o] = (double)acc[t * O + o] * (double)g * (double)s[t] / 127.0;
}

/*
 * Mask statistics, by-products of S2-S3 that follow how the masks evolve in training.
 *
 * Natural zeros [SBN-es §3 "Contribuciones Clave" item 1 (the "quantisation valley": a
 * large share of the ternary weights is 0); SBN-ar §1, the hypothesis bullet]: the number
 * of positions whose ternary code t (S2, before the mask) is 0.
 */
int64_t oracle_count_zero_codes(const int8_t *t, int64_t n) {
  int64_t c = 0;
  for (int64_t i = 0; i < n; ++i)
    if (t[i] == 0) ++c;
  return c;
}

/*
 * Mask flips [SBN-es §2 "Recomputación Dinámica de Máscaras"; SBN-ar §2 dynamic
 * recomputation: the mask is rebuilt every step from the current masters, so the
 * topology moves]: the number of positions kept by one of two masks of the same tensor
 * and pruned by the other.
 */
int64_t oracle_count_mask_flips(const uint8_t *keep_a, const uint8_t *keep_b, int64_t n) {
  int64_t c = 0;
  for (int64_t i = 0; i < n; ++i)
    if ((keep_a[i] != 0) != (keep_b[i] != 0)) ++c;
  return c;
}

/*
 * Backward of the layer under the dual straight-through estimator [SBN-es §2 "Estrategia
 * de Entrenamiento", "Estimador de Paso Directo Dual": quantisation and mask selection
 * are not differentiable, so both are passed by straight-through estimators, and the
 * gradient reaches every master weight, the pruned ones included; SBN-ar §2, Sparse-BitLinear
 * item 3: the quantisation STE is the identity inside the clipping range, the mask STE
 * sends a dense gradient to all masters].  The forward's effective operands are
 *   W_eff[o, k] = g * Ws[o, k]            (the dequantised masked codes)
 *   X_eff[t, k] = s[t] / 127 * Xq[t, k]   (the dequantised activations)
 * and, in fp64,
 *   dX[t, k] = sum_o dY[t, o] * W_eff[o, k]
 *   dW[o, k] = pass[o, k] * sum_t dY[t, o] * X_eff[t, k]
 * where pass[o, k] is the quantisation STE: with round() taken as the identity the
 * quantiser is clip(W / g, -1, 1), whose derivative is 1 for |W / g| <= 1 and 0 outside
 * (the boundary included, as a clamp's gradient is).  The quotient is the fp32 one the
 * codes are decided from: pass = (fl32(|W| / g) <= 1).  The mask does not enter dW.
 * dY is [T, O] fp32; W holds the bf16 masters [O, K]; dX is [T, K] and dW is [O, K] fp64.
 */
int oracle_ste_pass(float w, float g) { return fabsf(w) / g <= 1.0f; }

void oracle_backward(const float *dY, const int8_t *Xq, const float *s, const int8_t *Ws,
                     const uint16_t *W, float g, int64_t T, int64_t O, int64_t K, double *dX,
                     double *dW) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; ++t)
    for (int64_t k = 0; k < K; ++k) {
      double acc = 0.0;
      for (int64_t o = 0; o < O; ++o)
        acc += (double)dY[t * O + o] * ((double)g * (double)Ws[o * K + k]);
      dX[t * K + k] = acc;
    }
#pragma omp parallel for schedule(static)
  for (int64_t o = 0; o < O; ++o)
    for (int64_t k = 0; k < K; ++k) {
      double acc = 0.0;
      for (int64_t t = 0; t < T; ++t)
        acc += (double)dY[t * O + o] * (((double)s[t]) / 127.0 * (double)Xq[t * K + k]);
      dW[o * K + k] = oracle_ste_pass(bf16_bits_to_float(W[o * K + k]), g) ? acc : 0.0;
    }
}

/*
 * Group quantisation [bitnet.cpp article, "Cuantización y normalización de grupos": instead
 * of one set of parameters for the whole weight matrix, weights and activations are split
 * into G groups, each with its own parameters, so that groups need no communication].
 * Reading: G equal blocks along the input dimension K (block j = inputs j*K/G ..
 * (j+1)*K/G - 1, K/G a multiple of 64), for the weights and for every token's activations;
 * each block is a Sparse-BitLinear of its own and the layer's output is their sum:
 *   S_j   = sum over the block's weights of trunc(|W| * 2^24)    (exact, all rows)
 *   g_j   = fp32( fp32( fp64(S_j) / (fp64(O * K / G) * 2^24) ) + eps )
 *   t     = clamp(round(W / g_j), -1, 1) for W in block j      (fp32 divide, half-even)
 *   mask  = the N:M rule on the master magnitudes (independent of the scales)
 *   s_tj  = max(max over the block of |x_t|, 1e-5)
 *   q     = clamp(round((127 x) / s_tj), -127, 127)
 *   acc_j = sum over the block of q * ws                       (exact)
 *   y     = sum_j acc_j * g_j * s_tj / 127                     (fp64, j ascending)
 * With G == 1 this is the per-tensor layer above.  The functions below implement each
 * step for all groups at once.
 */
int oracle_group_gamma(const uint16_t *W, int64_t O, int64_t K, int G, float eps,
                       uint64_t *S_out, float *gamma_out, float *g_out) {
  const int64_t kg = K / G;
  int err = 0;
  for (int j = 0; j < G; ++j) {
    uint64_t S = 0;
    for (int64_t r = 0; r < O; ++r)
      for (int64_t k = j * kg; k < (j + 1) * kg; ++k) {
        float a = fabsf(bf16_bits_to_float(W[r * K + k]));
        if (!isfinite(a)) {
          err |= ORACLE_ERR_W_NONFINITE;
          continue;
        }
        if (a >= 256.0f) {
          err |= ORACLE_ERR_W_RANGE;
          continue;
        }
        S += (uint64_t)((double)a * 16777216.0); /* exact product, truncating conversion */
      }
    const float gamma = (float)((double)S / ((double)O * (double)kg * 16777216.0));
    S_out[j] = S;
    gamma_out[j] = gamma;
    g_out[j] = gamma + eps;
  }
  return err;
}

/* Codes with the scale of each input's block, the N:M mask, and the masked codes. */
void oracle_group_ternary_mask(const uint16_t *W, int64_t O, int64_t K, int N, int M, int G,
                               const float *g, int8_t *t_out, uint8_t *keep_out,
                               int8_t *ws_out) {
  const int64_t kg = K / G;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < O; ++r) {
    for (int64_t base = 0; base < K; base += M) {
      for (int i = 0; i < M; ++i) {
        const int64_t idx = r * K + base + i;
        const float wi = bf16_bits_to_float(W[idx]);
        int ahead = 0; /* group members ranked before position i */
        for (int j = 0; j < M; ++j) {
          const float mj = fabsf(bf16_bits_to_float(W[r * K + base + j]));
          if (mj > fabsf(wi) || (mj == fabsf(wi) && j < i)) ++ahead;
        }
        const float q = wi / g[(base + i) / kg];
        const float rq = rintf(q);
        const int8_t t = rq >= 1.0f ? 1 : (rq <= -1.0f ? -1 : 0);
        const uint8_t keep = (uint8_t)(ahead < N);
        t_out[idx] = t;
        keep_out[idx] = keep;
        ws_out[idx] = (int8_t)(keep ? t : 0);
      }
    }
  }
}

/* s[t * G + j] and Xq for every token and block.  Returns error bits. */
int oracle_group_quant_acts(const uint16_t *X, int64_t T, int64_t K, int G, int8_t *Xq,
                            float *s_out) {
  const int64_t kg = K / G;
  int err = 0;
  for (int64_t t = 0; t < T; ++t)
    for (int j = 0; j < G; ++j) {
      float a = 0.0f;
      for (int64_t k = j * kg; k < (j + 1) * kg; ++k) {
        float v = fabsf(bf16_bits_to_float(X[t * K + k]));
        if (!isfinite(v)) {
          err |= ORACLE_ERR_X_NONFINITE;
          continue;
        }
        a = v > a ? v : a;
      }
      const float s = a < 1e-5f ? 1e-5f : a;
      s_out[t * G + j] = s;
      for (int64_t k = j * kg; k < (j + 1) * kg; ++k) {
        float r = rintf((127.0f * bf16_bits_to_float(X[t * K + k])) / s);
        r = r > 127.0f ? 127.0f : (r < -127.0f ? -127.0f : r);
        Xq[t * K + k] = (int8_t)(r != r ? 0.0f : r);
      }
    }
  return err;
}

/* acc[(j * T + t) * O + o] = the block-j sum; y[t * O + o] = sum_j acc * g_j * s_tj / 127. */
int oracle_group_contract_rescale(const int8_t *Xq, const int8_t *Ws, const float *s,
                                  const float *g, int64_t T, int64_t O, int64_t K, int G,
                                  int32_t *acc, double *y) {
  const int64_t kg = K / G;
  int err = 0;
#pragma omp parallel for reduction(| : err) schedule(static)
  for (int64_t o = 0; o < O; ++o)
    for (int64_t t = 0; t < T; ++t) {
      double yo = 0.0;
      for (int j = 0; j < G; ++j) {
        int64_t sum = 0;
        for (int64_t k = j * kg; k < (j + 1) * kg; ++k)
          sum += (int64_t)Xq[t * K + k] * (int64_t)Ws[o * K + k];
        if (sum > INT32_MAX || sum < INT32_MIN) err |= ORACLE_ERR_ACC_OVERFLOW;
        acc[(j * T + t) * O + o] = (int32_t)sum;
        yo += (double)sum * (double)g[j] * (double)s[t * G + j] / 127.0;
      }
      y[t * O + o] = yo;
    }
  return err;
}
