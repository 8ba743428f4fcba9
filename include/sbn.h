/*
 * sbn.h -- C ABI of the Sparse-BitLinear forward on NVIDIA B200 (sm_100a).
 *
 * The operation (Sparse-BitNet, "1.58-bit LLMs are Naturally Friendly to Semi-Structured
 * Sparsity", technical summaries on gist.science, section 2 "Methodology":
 * Sparse-BitLinear layer):
 *   1. gamma = mean |W| over the bf16 master weights of one tensor; g = gamma + eps;
 *   2. ternary codes t = clip(round(W / g), -1, 1)       (absmean quantisation);
 *   3. N:M mask = in every group of M consecutive inputs of a row, the N largest master
 *      magnitudes (ties: lower index), applied AFTER quantisation (quant-then-mask);
 *   4. the masked codes are packed as 2-bit codes plus per-group metadata;
 *   5. activations are quantised per token to int8 by absmax with Qb = 127
 *      ("Marco de inferencia de Microsoft lleva modelos de lenguaje grande de 1 bit a
 *      dispositivos locales", unite.ai, "Fundamento matemático", item 2);
 *   6. acc = Xq . Ws^T in exact int32; y = acc * g * s / 127 (same article, item 3:
 *      the BitLinear output is rescaled by the weight and activation scales over Qb).
 * Rounding of round() is half-to-even; W/g and 127*x/s are IEEE fp32 divisions.
 *
 * Conventions for every call below:
 *   - All tensor arguments are DEVICE pointers owned by the caller; the library keeps no
 *     state and allocates no memory.  Layouts are row-major and dense.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Every call only enqueues
 *     work on it and returns without synchronising.
 *   - Argument errors are detected on the host, before anything is launched, and
 *     returned as an sbn_status; nothing is written in that case.
 *   - Data errors (NaN/Inf or |W| >= 256 in the inputs) are found by the kernels, which
 *     OR the SBN_FLAG_* bits into *err_flag (an int32 in device memory that the caller
 *     zeroes; err_flag may be NULL to not report them).  Outputs are unspecified when a
 *     flag is raised.
 *   - Supported patterns: m in {4, 8}, 1 <= n <= m (n == m is the unmasked b1.58 layer).
 *     `in` (K) must be a positive multiple of 64; `out` (O) positive; tokens >= 0.
 *   - Device pointers must be 16-byte aligned.
 */
#ifndef SBN_H_
#define SBN_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SBN_API __attribute__((visibility("default")))
#else
#define SBN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum sbn_status {
  SBN_OK = 0,
  SBN_ERR_NULL = 1,    /* a required pointer is NULL */
  SBN_ERR_SHAPE = 2,   /* out <= 0, in <= 0, in % 64 != 0, tokens < 0, or too large */
  SBN_ERR_PATTERN = 3, /* m not in {4, 8} or n not in [1, m] */
  SBN_ERR_ALIGN = 4,   /* a device pointer is not 16-byte aligned */
  SBN_ERR_CUDA = 5,    /* a CUDA runtime call or a launch failed */
  SBN_ERR_ARG = 6      /* eps negative or not finite */
} sbn_status;

/* Data-error bits OR-ed into *err_flag by the kernels. */
#define SBN_FLAG_W_NONFINITE 1 /* a master weight is NaN or Inf */
#define SBN_FLAG_W_RANGE 2     /* a master weight has |W| >= 256 */
#define SBN_FLAG_X_NONFINITE 4 /* an activation is NaN or Inf */
#define SBN_FLAG_TIMEOUT 8     /* a tensor-core pipeline wait gave up (~1 s); Y unspecified */

/*
 * Packed weight format (sizes from sbn_linear_ref_dims).  Row r of each plane starts at
 * byte r * ld; bytes past a row's data up to ld are written as zero.
 *   codes plane: 2-bit codes (0 -> 00, +1 -> 01, -1 -> 11) of the row's stored elements:
 *     pattern 2:4 stores the kept positions only (K/2 per row, ascending K); every other
 *     pattern stores all K positions, pruned ones as 0.  Stored element e lives in the
 *     little-endian 32-bit word e/16 of the row, at bits [8k + 6 - 2j, 8k + 7 - 2j] with
 *     j = (e % 16) / 4 and k = e % 4, so (word << 2j) & 0xC0C0C0C0 holds 64 * code of
 *     elements 4j..4j+3 as four int8 lanes.
 *   meta plane: per group g of M inputs: 2:4 -> nibble i0 | i1 << 2 (the two kept
 *     positions, i0 < i1); other M == 4 -> 4-bit keep mask; M == 8 -> 8-bit keep mask
 *     (one byte per group).  Group 2h is the low nibble of byte h, 2h+1 the high one.
 */
typedef struct sbn_dims {
  int64_t codes_ld;             /* bytes between rows of the codes plane (multiple of 16) */
  int64_t meta_ld;              /* bytes between rows of the meta plane (multiple of 16) */
  int64_t codes_row_bytes;      /* data bytes per codes row (the rest is zero padding) */
  int64_t meta_row_bytes;       /* data bytes per meta row */
  int64_t codes_bytes;          /* out * codes_ld: size of the codes buffer */
  int64_t meta_bytes;           /* out * meta_ld: size of the meta buffer */
  int64_t pack_workspace_bytes; /* device workspace sbn_quantize_mask_pack_weights needs */
} sbn_dims;

/*
 * Host only, no CUDA call: validates (out, in, n, m) and fills *d with the plane sizes
 * and the workspace size.  Returns SBN_ERR_NULL / SHAPE / PATTERN on bad arguments.
 */
SBN_API sbn_status sbn_linear_ref_dims(int64_t out, int64_t in, int n, int m, sbn_dims *d);

/*
 * Steps 1-4 for one master tensor (Sparse-BitNet section 2: absmean ternary
 * quantisation, mask from the master magnitudes, quant-then-mask, packing).
 *   W          bf16 [out, in] master weights (bits of __nv_bfloat16), read only.
 *   eps        added to gamma in fp32 (finite, >= 0; 1e-5 is the usual value).
 *   codes      uint8 [dims.codes_bytes], written (including the zero padding).
 *   meta       uint8 [dims.meta_bytes], written.
 *   gamma_eff  one fp32: g = fp32(gamma + eps), where
 *              gamma = fp32( fp64(S) / (fp64(out * in) * 2^24) ),
 *              S = sum over all weights of trunc(|W| * 2^24)  (exact 64-bit integer sum,
 *              so the result does not depend on the order of summation).
 *   workspace  dims.pack_workspace_bytes of device memory for the reduction's per-CTA
 *              partial sums.  Its contents need no initialisation and may be reused by
 *              later calls; calls that share one workspace must not run concurrently.
 *   dense_dbg  optional int8 [out, in]: the masked ternary matrix (NULL to skip).
 *   err_flag   optional: SBN_FLAG_W_NONFINITE / SBN_FLAG_W_RANGE.
 * out * in must be below 2^31.
 */
SBN_API sbn_status sbn_quantize_mask_pack_weights(const void *W, int64_t out, int64_t in, int n,
                                          int m, float eps, uint8_t *codes, uint8_t *meta,
                                          float *gamma_eff, void *workspace,
                                          int8_t *dense_dbg, int32_t *err_flag,
                                          void *stream);

/*
 * Grouped pack: steps 1-4 for many master tensors in two launches, each tensor into one
 * pattern or into both of 6:8 and 2:4 (the training-step re-mask of Sparse-BitNet section 2,
 * "Recomputacion Dinamica": every step re-quantises and re-masks every linear from its
 * masters).  Every output bit is that of sbn_quantize_mask_pack_weights for the tensor and
 * pattern alone.  A tensor packed into two patterns is read twice in all (once for the
 * absmean sum, once for both patterns' codes and metadata), not twice per pattern.
 *
 * Use: sbn_pack_group_sizes -> allocate a HOST plan buffer (16-byte aligned) and a device
 * buffer of the same size, plus the device workspace, ZEROED once -> sbn_pack_group_plan
 * fills the host plan -> copy it to the device -> sbn_quantize_mask_pack_weights_group as
 * often as wanted (for instance after every optimizer step, masters updated in place).  The
 * plan records device pointers: the buffers must stay allocated and in place while it is
 * in use.
 */
typedef struct sbn_pack_group_tensor {
  const void *W;          /* bf16 [out, in] masters, read only */
  uint8_t *codes;         /* planes of the first pattern (n:m), sizes from sbn_linear_ref_dims */
  uint8_t *meta;
  uint8_t *codes2;        /* planes of the second pattern (n2:m2); NULL when m2 == 0 */
  uint8_t *meta2;
  float *gamma_eff;       /* one fp32, written: g, the same for both patterns */
  int8_t *dense_dbg;      /* optional int8 [out, in] masked ternary matrix, first pattern */
  int8_t *dense_dbg2;     /* optional, second pattern */
  int64_t out, in;        /* shape rules of sbn_quantize_mask_pack_weights */
  int32_t n, m;           /* 6:8 or 2:4 */
  int32_t n2, m2;         /* the other of 6:8 / 2:4, or 0, 0 for one pattern */
  float eps;              /* finite, >= 0 */
  int32_t reserved;       /* set to 0 */
} sbn_pack_group_tensor;

/*
 * Host only.  Validates the tensors (SBN_ERR_PATTERN for a pattern other than 6:8 / 2:4 or
 * two equal patterns; SBN_ERR_SHAPE / NULL / ALIGN / ARG as sbn_quantize_mask_pack_weights;
 * SBN_ERR_SHAPE for more than 65536 tensors) and returns the plan size and the device
 * workspace size (16 bytes per tensor).
 */
SBN_API sbn_status sbn_pack_group_sizes(const sbn_pack_group_tensor *tensors, int32_t count,
                                        int64_t *plan_bytes, int64_t *workspace_bytes);

/* Host only.  Writes the plan into the HOST buffer `plan` (16-byte aligned, plan_bytes). */
SBN_API sbn_status sbn_pack_group_plan(const sbn_pack_group_tensor *tensors, int32_t count,
                                       void *plan, int64_t plan_bytes);

/*
 * Steps 1-4 for every tensor of the plan.
 *   plan       the host plan; plan_dev the same bytes in device memory (16-byte aligned).
 *   workspace  workspace_bytes of device memory, ZEROED by the caller before its first use;
 *              every call leaves its counters at zero again, so it needs no clearing
 *              between calls.  Calls that share a workspace must not overlap on the GPU.
 *   err_flag   optional: SBN_FLAG_W_NONFINITE / SBN_FLAG_W_RANGE.
 * SBN_ERR_ARG if `plan` is not a plan from sbn_pack_group_plan.
 */
SBN_API sbn_status sbn_quantize_mask_pack_weights_group(const void *plan, const void *plan_dev,
                                                        void *workspace, int32_t *err_flag,
                                                        void *stream);

/*
 * The same computation as sbn_quantize_mask_pack_weights, for callers that cannot give
 * this library any device memory: plugin hosts that own every allocation and hand an
 * operator no workspace, or serving loops that forbid cudaMalloc/cudaFree on their hot
 * path because those calls can synchronise the device and fragment its memory.  (The
 * pages have no counterpart: this is an interface convenience, not part of the method.)
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.  The pack's
 *     scratch (the absmean partial sums) is a fixed 8448-byte array in the library's own
 *     device memory; every GPU that loads the library holds it until the process exits.
 *   - Sizes: the same limits as sbn_quantize_mask_pack_weights (out * in < 2^31,
 *     in <= 131072); anything larger is refused with SBN_ERR_SHAPE.
 *   - Each call looks up the array's address in the current device's context.  The
 *     first call on a device loads the library's device code there; make it before any
 *     stream capture.
 *   - Each call rewrites every part of the array it later reads, so nothing needs
 *     clearing.  All calls in the process share the one array per device: calls that
 *     overlap on the GPU (for instance on two streams) race and give wrong results.
 * Arguments and outputs are those of sbn_quantize_mask_pack_weights without `workspace`.
 */
SBN_API sbn_status sbn_quantize_mask_pack_weights_noalloc(const void *W, int64_t out,
                                                          int64_t in, int n, int m, float eps,
                                                          uint8_t *codes, uint8_t *meta,
                                                          float *gamma_eff, int8_t *dense_dbg,
                                                          int32_t *err_flag, void *stream);

/*
 * Step 5: per-token absmax int8 activations (bitnet.cpp article, "Fundamento
 * matemático", item 2, with Qb = 127):
 *   s[t] = max(max_k |X[t,k]|, 1e-5);  Xq[t,k] = clamp(rint((127 * X[t,k]) / s[t]), +-127).
 *   X       bf16 [tokens, in], read only.
 *   Xq      int8 [tokens, in], written.
 *   absmax  fp32 [tokens], written (s, after the 1e-5 floor).
 *   err_flag optional: SBN_FLAG_X_NONFINITE.
 * tokens == 0 is a no-op that returns SBN_OK before any pointer is checked (empty
 * tensors may have NULL data pointers).
 */
SBN_API sbn_status sbn_quantize_acts(const void *X, int64_t tokens, int64_t in, int8_t *Xq,
                             float *absmax, int32_t *err_flag, void *stream);

/*
 * Step 6: y[t, o] = (sum_k Xq[t,k] * Ws[o,k]) * c_t,  c_t = fp32(fp32(g * s[t]) / 127),
 * where Ws is the masked ternary matrix held by (codes, meta) and g = *gamma_eff.  The
 * sum is exact (int32).  The product acc * c_t is one fp32 multiply (no FMA); with
 * y_is_bf16 it is then rounded to bf16 (nearest-even).
 *   Xq, absmax       from sbn_quantize_acts (int8 [tokens, in], fp32 [tokens]).
 *   codes, meta      from sbn_quantize_mask_pack_weights for the same (out, in, n, m).
 *   gamma_eff        one fp32 on the device.
 *   Y                fp32 or bf16 [tokens, out], written.
 *   acc_dbg          optional int32 [tokens, out]: the exact integer sums (NULL to skip).
 *   err_flag         optional: SBN_FLAG_TIMEOUT if the tensor-core pipeline stalled.
 * tokens == 0 is a no-op that returns SBN_OK once the shapes and pattern are valid, before
 * any pointer is checked.
 */
SBN_API sbn_status sbn_linear(const int8_t *Xq, const float *absmax, const uint8_t *codes,
                      const uint8_t *meta, const float *gamma_eff, int64_t tokens,
                      int64_t out, int64_t in, int n, int m, void *Y, int y_is_bf16,
                      int32_t *acc_dbg, int32_t *err_flag, void *stream);

/*
 * Tensor-core operand (2:4): the packed planes expanded once into the form the sparse
 * tensor cores read, for contractions with many tokens (prefill).  The codes of each row
 * become int8 values t in {-1, 0, 1} (0.5 byte per weight) so that the contraction only
 * stages tiles with TMA and issues MMAs; the expansion costs one pass over the planes and
 * is done when the weights change (after sbn_quantize_mask_pack_weights), not per call.
 *
 * Layout (opaque to callers; described for completeness): with O_pad = out rounded up to
 * 256 and K_pad = in rounded up to 128, an int8 [O_pad][K_pad / 2] plane of the kept values
 * in K order (zero in the padding), then a uint8 [O_pad][K_pad / 8] copy of the metadata
 * plane (the index pair (0, 1) in the padding).
 */

/* Host only: *bytes = size of the operand of an (out, in) layer.  SBN_ERR_PATTERN unless
 * n:m is 2:4; the shape rules of sbn_linear_ref_dims. */
SBN_API sbn_status sbn_operand_bytes(int64_t out, int64_t in, int n, int m, int64_t *bytes);

/* Writes the operand (device memory of sbn_operand_bytes, 16-byte aligned) from the codes
 * and meta planes of sbn_quantize_mask_pack_weights (2:4).  One launch on `stream`. */
SBN_API sbn_status sbn_expand_operand(const uint8_t *codes, const uint8_t *meta, int64_t out,
                                      int64_t in, int n, int m, void *operand, void *stream);

/* Steps 6-7 from the operand: y[t, o] = (sum_k Xq[t,k] * Ws[o,k]) * c_t, exactly the result of
 * sbn_linear (every bit), with the other arguments as there.  Made for many tokens (tiles of
 * 224 tokens on CTA pairs); any tokens >= 0 is accepted. */
SBN_API sbn_status sbn_linear_operand(const int8_t *Xq, const float *absmax, const void *operand,
                                      const float *gamma_eff, int64_t tokens, int64_t out,
                                      int64_t in, int n, int m, void *Y, int y_is_bf16,
                                      int32_t *acc_dbg, int32_t *err_flag, void *stream);

/*
 * Grouped calls: steps 5-7 for many independent 2:4 layers of at most 32 tokens each (the
 * decode phase of a whole decoder stack) in one launch per step, instead of one launch
 * per layer.  Each layer is described by one sbn_group_linear; the arithmetic and every
 * output bit are those of sbn_quantize_acts and sbn_linear for that layer alone.
 *
 * Use: sbn_group_plan_sizes -> allocate a HOST plan buffer (128-byte aligned) and a device
 * buffer of the same size, plus the device workspace -> sbn_group_plan fills the host plan
 * -> copy it to the device buffer -> then, as often as wanted (for instance every decode
 * step, with new activations in the same X buffers):
 * sbn_quantize_acts_group and sbn_linear_group on a stream.  The plan records the device
 * pointers of every layer, so the buffers must stay allocated and in place while it is in
 * use; rebuild it when a pointer or a shape changes.
 */
typedef struct sbn_group_linear {
  const void *X;             /* bf16 [tokens, in] input of the grouped quantiser; may be
                                NULL if only sbn_linear_group is called (Xq given) */
  int8_t *Xq;                /* int8 [tokens, in] quantised activations */
  float *absmax;             /* fp32 [tokens] per-token scales s */
  const uint8_t *codes;      /* packed planes from sbn_quantize_mask_pack_weights (2:4) */
  const uint8_t *meta;
  const float *gamma_eff;    /* one fp32 on the device */
  void *Y;                   /* fp32 or bf16 [tokens, out], written */
  int32_t *acc_dbg;          /* optional int32 [tokens, out] exact sums (NULL to skip) */
  int64_t tokens;            /* 0..32; a layer with 0 tokens is skipped */
  int64_t out, in;           /* shape rules of sbn_linear */
  int32_t n, m;              /* must be 2 and 4 */
  int32_t y_is_bf16;
  int32_t reserved;          /* set to 0 */
  /* Row strides, 0 for the defaults.  A layer may be a K slice of a wider one (a block of
   * a group-quantised layer): X, Xq point at the slice's first column, `in` is the slice
   * width, and the strides are the wide layer's.
   *   ldx  elements between token rows of X and Xq (default in; a multiple of 16, >= in)
   *   ldc  bytes between rows of the codes plane (default that of sbn_linear_ref_dims for
   *        (out, in, 2, 4); a multiple of 16, >= in / 8)
   *   ldm  bytes between rows of the meta plane (likewise) */
  int64_t ldx, ldc, ldm;
} sbn_group_linear;

/*
 * Host only.  Validates the layers (SBN_ERR_PATTERN unless every n:m is 2:4; SBN_ERR_SHAPE
 * for tokens outside 0..32 or a bad shape; SBN_ERR_NULL / SBN_ERR_ALIGN for the pointers
 * of layers with tokens > 0, device pointers 16-byte aligned, absmax and gamma_eff 4-byte)
 * and returns the plan size and the device workspace size (0 when the schedule splits no
 * row tile over several work units).
 */
SBN_API sbn_status sbn_group_plan_sizes(const sbn_group_linear *lins, int32_t count,
                                        int64_t *plan_bytes, int64_t *workspace_bytes);

/*
 * Host only (queries the current device's SM count; no allocation, no synchronisation).
 * Writes the plan into the HOST buffer `plan` (128-byte aligned, plan_bytes from
 * sbn_group_plan_sizes): the TMA descriptors of every layer, the work units of the
 * contraction (128 weight rows x a range of K, spread over one CTA per SM) and the rows
 * of the activation quantiser.
 */
SBN_API sbn_status sbn_group_plan(const sbn_group_linear *lins, int32_t count, void *plan,
                                  int64_t plan_bytes);

/*
 * Step 5 for every layer of the plan (s and Xq of each layer's X), one launch.
 *   plan      the host plan; plan_dev the same bytes in device memory (128-byte aligned).
 *   err_flag  optional: SBN_FLAG_X_NONFINITE.
 * SBN_ERR_NULL if a layer of the plan has no X.
 */
SBN_API sbn_status sbn_quantize_acts_group(const void *plan, const void *plan_dev,
                                           int32_t *err_flag, void *stream);

/*
 * Steps 6-7 for every layer of the plan, one launch: Y = (Xq . Ws^T) * c_t exactly as
 * sbn_linear computes it.
 *   workspace  device memory of workspace_bytes (NULL allowed when that is 0), ZEROED by
 *              the caller before its first use; every call leaves it zeroed again, so it
 *              needs no clearing between calls.  After a call that raised
 *              SBN_FLAG_TIMEOUT it must be zeroed again.  Calls that share a workspace
 *              must not overlap on the GPU.
 *   err_flag   optional: SBN_FLAG_TIMEOUT if the tensor-core pipeline stalled.
 */
SBN_API sbn_status sbn_linear_group(const void *plan, const void *plan_dev, void *workspace,
                                    int32_t *err_flag, void *stream);

/*
 * The ordered sum of group quantisation: Y[i] = fp32 sum over j = 0..G-1 of part[j * n + i],
 * added in j order, stored fp32 or bf16 (RNE).  With the G blocks of group-quantised
 * layers as slices of a grouped call (each block's output y_j = fp32(acc_j * c_tj) written
 * into part), this completes their forward: the same bits as sbn_linear_gq.  Layers of
 * one G may share one call when their partial outputs and their Y are laid out back to
 * back (part as [G][n], Y as [n]).  n >= 0, 1 <= G <= 64; part and Y 16-byte aligned.
 */
SBN_API sbn_status sbn_gq_sum(const float *part, int64_t n, int32_t G, void *Y, int32_t y_is_bf16,
                              void *stream);

/*
 * Backward of the layer under the dual straight-through estimator (Sparse-BitNet summaries,
 * section 2 "Estimador de Paso Directo Dual" / Sparse-BitLinear item 3: the quantiser passes
 * the gradient as the identity inside its clip range; the mask passes it to every master
 * weight, the pruned ones included):
 *   dX[t, k] = g * sum_o dY[t, o] * Ws[o, k]
 *   dW[o, k] = pass[o, k] * sum_t dY[t, o] * (s[t] / 127) * Xq[t, k],
 *   pass[o, k] = (fl32(|W[o, k]| / g) <= 1)   (clip(W / g, -1, 1) has slope 1 there)
 * with Ws the masked ternary matrix of (codes, meta), g = *gamma_eff, s and Xq from the
 * forward's sbn_quantize_acts.  Computed on the tensor cores in bf16 x bf16 -> fp32 with
 * exact products (dY * Ws is exact; s / 127 is folded into dY and carried as two bf16
 * terms): the results differ from the exact sums only by fp32 accumulation and a relative
 * 2^-17 on the scaled dY.
 *   dY         bf16 [tokens, out], the upstream gradient.
 *   W          bf16 [out, in] masters (read for the clip gate; may be NULL if dW is NULL).
 *   dX         fp32 [tokens, in], written (NULL to skip).
 *   dW         fp32 [out, in], written (NULL to skip).
 *   workspace  device memory of sbn_backward_workspace_bytes (contents need no
 *              initialisation; calls sharing it must not overlap).
 *   err_flag   optional: SBN_FLAG_TIMEOUT.
 * Shapes: those of sbn_linear, and out % 8 == 0.  tokens == 0 is a no-op.
 */
SBN_API sbn_status sbn_backward_workspace_bytes(int64_t tokens, int64_t out, int64_t in,
                                                int64_t *bytes);
SBN_API sbn_status sbn_backward(const void *dY, const int8_t *Xq, const float *absmax,
                                const uint8_t *codes, const uint8_t *meta, const void *W,
                                const float *gamma_eff, int64_t tokens, int64_t out, int64_t in,
                                int n, int m, float *dX, float *dW, void *workspace,
                                int32_t *err_flag, void *stream);

/*
 * Steps 5-7 in one call: exactly sbn_quantize_acts followed by sbn_linear (every output bit,
 * Xq and absmax included).  For tokens <= 4 and in <= 16384 (decode) it is ONE launch: each
 * CTA of the GEMV quantises the few token rows into shared memory in its prologue (the
 * activation quantiser's launch and its round trip through global memory leave the
 * critical path); CTA 0 also writes Xq and absmax.  Otherwise the two launches of the
 * separate calls.  Arguments as in those two calls; Xq and absmax are required outputs.
 */
SBN_API sbn_status sbn_quantize_linear(const void *X, const uint8_t *codes, const uint8_t *meta,
                                       const float *gamma_eff, int64_t tokens, int64_t out,
                                       int64_t in, int n, int m, int8_t *Xq, float *absmax,
                                       void *Y, int y_is_bf16, int32_t *acc_dbg,
                                       int32_t *err_flag, void *stream);

/*
 * Group quantisation ("Marco de inferencia de Microsoft lleva modelos de lenguaje grande de
 * 1 bit a dispositivos locales", unite.ai, "Cuantización y normalización de grupos": weights
 * and activations split into G groups with parameters of their own, so that the groups need
 * no communication).  Here: G equal blocks along the input dimension; block j (inputs
 * j*in/G .. (j+1)*in/G - 1) is a Sparse-BitLinear of its own and the layer's output is the sum
 * of the blocks' outputs:
 *   g_j   = fp32(fp32(fp64(S_j) / (fp64(out * in / G) * 2^24)) + eps), S_j the exact sum of
 *           trunc(|W| * 2^24) over the block's weights (all rows)
 *   codes = clamp(round(W / g_j)) in block j; the N:M mask as in the per-tensor calls
 *   s_tj  = max(max |x_t| over block j, 1e-5); Xq by s_tj
 *   y[t,o]= sum_j fp32(acc_j[t,o] * c_tj), c_tj = fp32(fp32(g_j * s_tj) / 127), added in fp32
 *           in ascending j (acc_j the exact int32 sum over block j)
 * groups = 1 gives the per-tensor layer.  Shapes: 1 <= groups <= 64, in % groups == 0 and
 * (in / groups) % 128 == 0; the other rules and the packed planes are those of the per-tensor
 * calls (sbn_linear_ref_dims).  Scales: gamma_eff holds groups floats; absmax holds
 * groups * tokens floats, group-major (absmax[j * tokens + t]).
 */
/* Host only: *workspace_bytes = the contraction's scratch (groups * tokens * out fp32). */
SBN_API sbn_status sbn_gq_workspace_bytes(int64_t tokens, int64_t out, int64_t in, int groups,
                                          int64_t *workspace_bytes);
/* Steps 1-4 with per-group scales; workspace as for sbn_quantize_mask_pack_weights. */
SBN_API sbn_status sbn_quantize_mask_pack_weights_gq(const void *W, int64_t out, int64_t in,
                                                     int n, int m, int groups, float eps,
                                                     uint8_t *codes, uint8_t *meta,
                                                     float *gamma_eff, void *workspace,
                                                     int8_t *dense_dbg, int32_t *err_flag,
                                                     void *stream);
/* Step 5 with per-(token, group) scales. */
SBN_API sbn_status sbn_quantize_acts_gq(const void *X, int64_t tokens, int64_t in, int groups,
                                        int8_t *Xq, float *absmax, int32_t *err_flag,
                                        void *stream);
/* Steps 6-7: each block on the contraction kernels of sbn_linear, then the ordered sum.
 * acc_dbg (optional) is int32 [groups][tokens][out]: the blocks' exact sums. */
SBN_API sbn_status sbn_linear_gq(const int8_t *Xq, const float *absmax, const uint8_t *codes,
                                 const uint8_t *meta, const float *gamma_eff, int64_t tokens,
                                 int64_t out, int64_t in, int n, int m, int groups, void *Y,
                                 int y_is_bf16, void *workspace, int32_t *acc_dbg,
                                 int32_t *err_flag, void *stream);

/*
 * Mask statistics: by-products of steps 2-3 that follow how the masks evolve over training
 * steps (Sparse-BitNet summaries: section 3 "Contribuciones Clave" item 1, the large share
 * of ternary zeros; section 2, the mask recomputed every step from the current masters).
 * Both calls ADD their count into *count, one uint64 in device memory (8-byte aligned)
 * that the caller zeroes before the first call; several calls may accumulate into it.
 *
 * sbn_count_zero_codes: the number of weights of W (bf16 [out, in]) whose ternary code
 *   (step 2, before the mask) is 0, for g = *gamma_eff as written by
 *   sbn_quantize_mask_pack_weights for the same W.  Weights that are NaN, or a g that is
 *   not a finite positive number or zero, give an unspecified count.
 * sbn_count_mask_flips: the number of positions whose keep bit differs between two meta
 *   planes written by sbn_quantize_mask_pack_weights for the same (out, in, n, m) (for
 *   instance the masks of two training steps).
 * Shape, pattern and alignment rules are those of sbn_quantize_mask_pack_weights.
 */
SBN_API sbn_status sbn_count_zero_codes(const void *W, const float *gamma_eff, int64_t out,
                                        int64_t in, unsigned long long *count, void *stream);
SBN_API sbn_status sbn_count_mask_flips(const uint8_t *meta_a, const uint8_t *meta_b,
                                        int64_t out, int64_t in, int n, int m,
                                        unsigned long long *count, void *stream);

/* A static, human-readable name for a status code. */
SBN_API const char *sbn_status_string(sbn_status s);

#ifdef __cplusplus
}
#endif

#endif /* SBN_H_ */
