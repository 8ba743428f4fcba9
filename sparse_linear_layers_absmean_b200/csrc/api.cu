// The C ABI of sbn.h: host-side validation, buffer geometry and dispatch to the kernels.
// Nothing here allocates device memory or synchronises.
#include <cmath>

#include <cstring>

#include "common.cuh"
#include "group.cuh"
#include "kernels.cuh"

namespace {

constexpr int64_t kMaxIn = 131072;           // keeps 64 * 127 * in below 2^31
constexpr int64_t kMaxElems = (1ll << 31) - 1;  // out * in (one tensor)

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

sbn_status check_pattern(int n, int m) {
  if (m != 4 && m != 8) return SBN_ERR_PATTERN;
  if (n < 1 || n > m) return SBN_ERR_PATTERN;
  return SBN_OK;
}

sbn_status check_in(int64_t in) {
  if (in <= 0 || in % 64 != 0 || in > kMaxIn) return SBN_ERR_SHAPE;
  return SBN_OK;
}

void fill_dims(int64_t out, int64_t in, int n, int m, sbn_dims *d) {
  const bool compact = (n == 2 && m == 4);
  const int64_t stored = compact ? in / 2 : in;
  d->codes_row_bytes = stored / 4;
  d->meta_row_bytes = in / 8;
  d->codes_ld = (d->codes_row_bytes + 15) / 16 * 16;
  d->meta_ld = (d->meta_row_bytes + 15) / 16 * 16;
  d->codes_bytes = out * d->codes_ld;
  d->meta_bytes = out * d->meta_ld;
  d->pack_workspace_bytes = (int64_t)((sizeof(sbn::PackWorkspace) + 255) / 256 * 256);
}

sbn_status check_group(const sbn_group_linear *lins, int32_t count) {
  if (count < 0 || count > (1 << 20)) return SBN_ERR_SHAPE;
  if (count > 0 && !lins) return SBN_ERR_NULL;
  for (int32_t p = 0; p < count; ++p) {
    const sbn_group_linear &l = lins[p];
    if (l.n != 2 || l.m != 4) return SBN_ERR_PATTERN;
    sbn_dims d;
    sbn_status st = sbn_linear_ref_dims(l.out, l.in, l.n, l.m, &d);
    if (st != SBN_OK) return st;
    if (l.tokens < 0 || l.tokens > sbn::kGroupMaxTokens) return SBN_ERR_SHAPE;
    if (l.ldx < 0 || l.ldc < 0 || l.ldm < 0) return SBN_ERR_SHAPE;
    if ((l.ldx && (l.ldx < l.in || l.ldx % 16)) || (l.ldc && (l.ldc < d.codes_row_bytes || l.ldc % 16)) ||
        (l.ldm && (l.ldm < d.meta_row_bytes || l.ldm % 16)))
      return SBN_ERR_SHAPE;
    if (l.tokens == 0) continue;
    if (!l.Xq || !l.absmax || !l.codes || !l.meta || !l.gamma_eff || !l.Y) return SBN_ERR_NULL;
    if (!aligned16(l.Xq) || !aligned16(l.codes) || !aligned16(l.meta) || !aligned16(l.Y) ||
        (l.X && !aligned16(l.X)) || (l.acc_dbg && !aligned16(l.acc_dbg)) ||
        (reinterpret_cast<uintptr_t>(l.absmax) & 3u) ||
        (reinterpret_cast<uintptr_t>(l.gamma_eff) & 3u))
      return SBN_ERR_ALIGN;
  }
  return SBN_OK;
}

sbn_status check_groups(int64_t in, int groups) {
  if (groups < 1 || groups > 64 || in % groups != 0 || (in / groups) % 128 != 0)
    return SBN_ERR_SHAPE;
  return SBN_OK;
}

sbn_status check_plan(const void *plan, const void *plan_dev) {
  if (!plan || !plan_dev) return SBN_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(plan) & 127u) || (reinterpret_cast<uintptr_t>(plan_dev) & 127u))
    return SBN_ERR_ALIGN;
  const sbn::GroupHeader *hd = static_cast<const sbn::GroupHeader *>(plan);
  if (hd->magic != sbn::kGroupMagic || hd->version != sbn::kGroupVersion) return SBN_ERR_ARG;
  return SBN_OK;
}

bool fast_pattern(int n, int m) { return (n == 6 && m == 8) || (n == 2 && m == 4); }

sbn_status check_pack_group(const sbn_pack_group_tensor *ts, int32_t count) {
  if (count < 0 || count > sbn::kPackGroupMaxTensors) return SBN_ERR_SHAPE;
  if (count > 0 && !ts) return SBN_ERR_NULL;
  uint64_t total_q = 0;
  for (int32_t i = 0; i < count; ++i) {
    const sbn_pack_group_tensor &t = ts[i];
    sbn_dims d;
    sbn_status st = sbn_linear_ref_dims(t.out, t.in, t.n, t.m, &d);
    if (st != SBN_OK) return st;
    if (!fast_pattern(t.n, t.m)) return SBN_ERR_PATTERN;
    const bool two = t.m2 != 0 || t.n2 != 0;
    if (two && (!fast_pattern(t.n2, t.m2) || (t.n2 == t.n && t.m2 == t.m))) return SBN_ERR_PATTERN;
    if (!std::isfinite(t.eps) || t.eps < 0.0f) return SBN_ERR_ARG;
    if (!t.W || !t.codes || !t.meta || !t.gamma_eff) return SBN_ERR_NULL;
    if (two && (!t.codes2 || !t.meta2)) return SBN_ERR_NULL;
    if (!aligned16(t.W) || !aligned16(t.codes) || !aligned16(t.meta) ||
        (t.dense_dbg && !aligned16(t.dense_dbg)) ||
        (two && (!aligned16(t.codes2) || !aligned16(t.meta2) ||
                 (t.dense_dbg2 && !aligned16(t.dense_dbg2)))) ||
        (reinterpret_cast<uintptr_t>(t.gamma_eff) & 3u))
      return SBN_ERR_ALIGN;
    total_q += (uint64_t)((t.out * t.in / 64 + 7) / 8);
  }
  if (total_q >= (1ull << 32)) return SBN_ERR_SHAPE;
  return SBN_OK;
}

// One pattern's arguments for the shared per-lane pack routine.
sbn::FastPackArgs pack_args(const void *W, int64_t out, int64_t in, int n, int m, float eps,
                            uint8_t *codes, uint8_t *meta, int8_t *dense_dbg, float *gamma_eff) {
  sbn_dims d;
  fill_dims(out, in, n, m, &d);
  const uint32_t bpr = (uint32_t)(in / 64);
  return sbn::FastPackArgs{reinterpret_cast<const uint4 *>(W), out * in / 64, bpr,
                           sbn::make_fast_div(bpr), nullptr, codes, d.codes_ld,
                           d.codes_row_bytes, meta, d.meta_ld, d.meta_row_bytes, dense_dbg,
                           0, out * in, eps, gamma_eff};
}

}  // namespace

extern "C" {

const char *sbn_status_string(sbn_status s) {
  switch (s) {
    case SBN_OK: return "ok";
    case SBN_ERR_NULL: return "null pointer";
    case SBN_ERR_SHAPE: return "bad shape";
    case SBN_ERR_PATTERN: return "unsupported N:M pattern";
    case SBN_ERR_ALIGN: return "pointer not 16-byte aligned";
    case SBN_ERR_CUDA: return "CUDA error";
    case SBN_ERR_ARG: return "bad argument";
  }
  return "unknown status";
}

sbn_status sbn_linear_ref_dims(int64_t out, int64_t in, int n, int m, sbn_dims *d) {
  if (!d) return SBN_ERR_NULL;
  sbn_status st = check_pattern(n, m);
  if (st != SBN_OK) return st;
  if ((st = check_in(in)) != SBN_OK) return st;
  if (out <= 0 || out > kMaxElems / in) return SBN_ERR_SHAPE;
  fill_dims(out, in, n, m, d);
  return SBN_OK;
}

sbn_status sbn_quantize_mask_pack_weights(const void *W, int64_t out, int64_t in, int n, int m,
                                          float eps, uint8_t *codes, uint8_t *meta,
                                          float *gamma_eff, void *workspace, int8_t *dense_dbg,
                                          int32_t *err_flag, void *stream) {
  sbn_dims d;
  sbn_status st = sbn_linear_ref_dims(out, in, n, m, &d);
  if (st != SBN_OK) return st;
  if (!W || !codes || !meta || !gamma_eff || !workspace) return SBN_ERR_NULL;
  if (!std::isfinite(eps) || eps < 0.0f) return SBN_ERR_ARG;
  if (!aligned16(W) || !aligned16(codes) || !aligned16(meta) || !aligned16(workspace) ||
      (dense_dbg && !aligned16(dense_dbg)))
    return SBN_ERR_ALIGN;
  if ((reinterpret_cast<uintptr_t>(gamma_eff) & 3u) || (reinterpret_cast<uintptr_t>(err_flag) & 3u))
    return SBN_ERR_ALIGN;
  return sbn::launch_pack(W, out, in, n, m, eps, codes, d.codes_ld, d.codes_row_bytes, meta,
                          d.meta_ld, d.meta_row_bytes, gamma_eff,
                          static_cast<sbn::PackWorkspace *>(workspace), dense_dbg, err_flag,
                          static_cast<cudaStream_t>(stream));
}

sbn_status sbn_quantize_acts(const void *X, int64_t tokens, int64_t in, int8_t *Xq,
                             float *absmax, int32_t *err_flag, void *stream) {
  sbn_status st = check_in(in);
  if (st != SBN_OK) return st;
  if (tokens < 0 || tokens > (1ll << 31) - 1) return SBN_ERR_SHAPE;
  if (tokens == 0) return SBN_OK;  // empty batch: nothing to read or write
  if (!X || !Xq || !absmax) return SBN_ERR_NULL;
  if (!aligned16(X) || !aligned16(Xq) || (reinterpret_cast<uintptr_t>(absmax) & 3u) ||
      (reinterpret_cast<uintptr_t>(err_flag) & 3u))
    return SBN_ERR_ALIGN;
  return sbn::launch_act_quant(X, tokens, in, Xq, absmax, err_flag,
                               static_cast<cudaStream_t>(stream));
}

sbn_status sbn_linear(const int8_t *Xq, const float *absmax, const uint8_t *codes,
                      const uint8_t *meta, const float *gamma_eff, int64_t tokens, int64_t out,
                      int64_t in, int n, int m, void *Y, int y_is_bf16, int32_t *acc_dbg,
                      int32_t *err_flag, void *stream) {
  sbn_dims d;
  sbn_status st = sbn_linear_ref_dims(out, in, n, m, &d);
  if (st != SBN_OK) return st;
  if (tokens < 0 || tokens > (1ll << 31) - 1) return SBN_ERR_SHAPE;
  if (tokens == 0) return SBN_OK;  // empty batch: nothing to read or write
  if (!Xq || !absmax || !codes || !meta || !gamma_eff || !Y) return SBN_ERR_NULL;
  if (!aligned16(Xq) || !aligned16(codes) || !aligned16(meta) || !aligned16(Y) ||
      (acc_dbg && !aligned16(acc_dbg)) || (reinterpret_cast<uintptr_t>(absmax) & 3u) ||
      (reinterpret_cast<uintptr_t>(gamma_eff) & 3u) || (reinterpret_cast<uintptr_t>(err_flag) & 3u))
    return SBN_ERR_ALIGN;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (tokens <= sbn::kGemvMaxTokens)
    return sbn::launch_gemv(Xq, absmax, codes, meta, gamma_eff, tokens, out, in, in, n, m, d.codes_ld,
                            d.meta_ld, Y, y_is_bf16, acc_dbg, s);
  return sbn::launch_gemm_tc(Xq, absmax, codes, meta, gamma_eff, tokens, out, in, in, n, m,
                             d.codes_ld, d.meta_ld, Y, y_is_bf16, acc_dbg, err_flag, s);
}

sbn_status sbn_operand_bytes(int64_t out, int64_t in, int n, int m, int64_t *bytes) {
  if (!bytes) return SBN_ERR_NULL;
  sbn_dims d;
  sbn_status st = sbn_linear_ref_dims(out, in, n, m, &d);
  if (st != SBN_OK) return st;
  if (n != 2 || m != 4) return SBN_ERR_PATTERN;
  *bytes = sbn::operand_bytes(out, in);
  return SBN_OK;
}

sbn_status sbn_expand_operand(const uint8_t *codes, const uint8_t *meta, int64_t out, int64_t in,
                              int n, int m, void *operand, void *stream) {
  int64_t bytes = 0;
  sbn_status st = sbn_operand_bytes(out, in, n, m, &bytes);
  if (st != SBN_OK) return st;
  if (!codes || !meta || !operand) return SBN_ERR_NULL;
  if (!aligned16(codes) || !aligned16(meta) || !aligned16(operand)) return SBN_ERR_ALIGN;
  sbn_dims d;
  sbn_linear_ref_dims(out, in, n, m, &d);
  return sbn::launch_expand_operand(codes, meta, out, in, d.codes_ld, d.meta_ld, operand,
                                    static_cast<cudaStream_t>(stream));
}

sbn_status sbn_linear_operand(const int8_t *Xq, const float *absmax, const void *operand,
                              const float *gamma_eff, int64_t tokens, int64_t out, int64_t in,
                              int n, int m, void *Y, int y_is_bf16, int32_t *acc_dbg,
                              int32_t *err_flag, void *stream) {
  int64_t bytes = 0;
  sbn_status st = sbn_operand_bytes(out, in, n, m, &bytes);
  if (st != SBN_OK) return st;
  if (tokens < 0 || tokens > (1ll << 31) - 1) return SBN_ERR_SHAPE;
  if (tokens == 0) return SBN_OK;
  if (!Xq || !absmax || !operand || !gamma_eff || !Y) return SBN_ERR_NULL;
  if (!aligned16(Xq) || !aligned16(operand) || !aligned16(Y) ||
      (acc_dbg && !aligned16(acc_dbg)) || (reinterpret_cast<uintptr_t>(absmax) & 3u) ||
      (reinterpret_cast<uintptr_t>(gamma_eff) & 3u) || (reinterpret_cast<uintptr_t>(err_flag) & 3u))
    return SBN_ERR_ALIGN;
  return sbn::launch_gemm_operand(Xq, absmax, operand, gamma_eff, tokens, out, in, Y, y_is_bf16,
                                  acc_dbg, err_flag, static_cast<cudaStream_t>(stream));
}

sbn_status sbn_backward_workspace_bytes(int64_t tokens, int64_t out, int64_t in, int64_t *bytes) {
  if (!bytes) return SBN_ERR_NULL;
  sbn_dims d;
  sbn_status st = sbn_linear_ref_dims(out, in, 2, 4, &d);
  if (st != SBN_OK) return st;
  if (out % 8 != 0 || tokens < 0 || tokens > (1ll << 24)) return SBN_ERR_SHAPE;
  *bytes = sbn::backward_workspace_bytes(tokens, out, in);
  return SBN_OK;
}

sbn_status sbn_backward(const void *dY, const int8_t *Xq, const float *absmax, const uint8_t *codes,
                        const uint8_t *meta, const void *W, const float *gamma_eff, int64_t tokens,
                        int64_t out, int64_t in, int n, int m, float *dX, float *dW,
                        void *workspace, int32_t *err_flag, void *stream) {
  sbn_dims d;
  sbn_status st = sbn_linear_ref_dims(out, in, n, m, &d);
  if (st != SBN_OK) return st;
  if (out % 8 != 0 || tokens < 0 || tokens > (1ll << 24)) return SBN_ERR_SHAPE;
  if (tokens == 0 || (!dX && !dW)) return SBN_OK;
  if (!dY || !gamma_eff || !workspace) return SBN_ERR_NULL;
  if (dX && (!codes || !meta)) return SBN_ERR_NULL;
  if (dW && (!Xq || !absmax || !W)) return SBN_ERR_NULL;
  if (!aligned16(dY) || !aligned16(workspace) || (dX && (!aligned16(dX) || !aligned16(codes) ||
                                                         !aligned16(meta))) ||
      (dW && (!aligned16(dW) || !aligned16(W))) || (absmax && (reinterpret_cast<uintptr_t>(absmax) & 3u)) ||
      (reinterpret_cast<uintptr_t>(gamma_eff) & 3u) || (reinterpret_cast<uintptr_t>(err_flag) & 3u))
    return SBN_ERR_ALIGN;
  return sbn::launch_backward(dY, Xq, absmax, codes, meta, W, gamma_eff, tokens, out, in, n, m,
                              d.codes_ld, d.meta_ld, dX, dW, workspace, err_flag,
                              static_cast<cudaStream_t>(stream));
}

sbn_status sbn_group_plan_sizes(const sbn_group_linear *lins, int32_t count, int64_t *plan_bytes,
                                int64_t *workspace_bytes) {
  if (!plan_bytes || !workspace_bytes) return SBN_ERR_NULL;
  sbn_status st = check_group(lins, count);
  if (st != SBN_OK) return st;
  return sbn::group_plan_sizes(lins, count, plan_bytes, workspace_bytes);
}

sbn_status sbn_group_plan(const sbn_group_linear *lins, int32_t count, void *plan,
                          int64_t plan_bytes) {
  if (!plan) return SBN_ERR_NULL;
  if (reinterpret_cast<uintptr_t>(plan) & 127u) return SBN_ERR_ALIGN;
  sbn_status st = check_group(lins, count);
  if (st != SBN_OK) return st;
  return sbn::group_plan(lins, count, plan, plan_bytes);
}

sbn_status sbn_quantize_acts_group(const void *plan, const void *plan_dev, int32_t *err_flag,
                                   void *stream) {
  sbn_status st = check_plan(plan, plan_dev);
  if (st != SBN_OK) return st;
  if (reinterpret_cast<uintptr_t>(err_flag) & 3u) return SBN_ERR_ALIGN;
  if (!static_cast<const sbn::GroupHeader *>(plan)->has_x) return SBN_ERR_NULL;
  return sbn::launch_act_quant_group(plan, plan_dev, err_flag, static_cast<cudaStream_t>(stream));
}

sbn_status sbn_linear_group(const void *plan, const void *plan_dev, void *workspace,
                            int32_t *err_flag, void *stream) {
  sbn_status st = check_plan(plan, plan_dev);
  if (st != SBN_OK) return st;
  if (reinterpret_cast<uintptr_t>(err_flag) & 3u) return SBN_ERR_ALIGN;
  const sbn::GroupHeader *hd = static_cast<const sbn::GroupHeader *>(plan);
  if (hd->ws_bytes > 0 && !workspace) return SBN_ERR_NULL;
  if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 255u)) return SBN_ERR_ALIGN;
  return sbn::launch_linear_group(plan, plan_dev, workspace, err_flag,
                                  static_cast<cudaStream_t>(stream));
}

sbn_status sbn_quantize_linear(const void *X, const uint8_t *codes, const uint8_t *meta,
                               const float *gamma_eff, int64_t tokens, int64_t out, int64_t in,
                               int n, int m, int8_t *Xq, float *absmax, void *Y, int y_is_bf16,
                               int32_t *acc_dbg, int32_t *err_flag, void *stream) {
  sbn_dims d;
  sbn_status st = sbn_linear_ref_dims(out, in, n, m, &d);
  if (st != SBN_OK) return st;
  if (tokens < 0 || tokens > (1ll << 31) - 1) return SBN_ERR_SHAPE;
  if (tokens == 0) return SBN_OK;
  if (!X || !codes || !meta || !gamma_eff || !Xq || !absmax || !Y) return SBN_ERR_NULL;
  if (!aligned16(X) || !aligned16(Xq) || !aligned16(codes) || !aligned16(meta) || !aligned16(Y) ||
      (acc_dbg && !aligned16(acc_dbg)) || (reinterpret_cast<uintptr_t>(absmax) & 3u) ||
      (reinterpret_cast<uintptr_t>(gamma_eff) & 3u) || (reinterpret_cast<uintptr_t>(err_flag) & 3u))
    return SBN_ERR_ALIGN;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (tokens <= sbn::kGemvMaxTokens && in <= 16384)
    return sbn::launch_gemv_fused(X, codes, meta, gamma_eff, tokens, out, in, n, m, d.codes_ld,
                                  d.meta_ld, Y, y_is_bf16, Xq, absmax, acc_dbg, err_flag, s);
  if ((st = sbn::launch_act_quant(X, tokens, in, Xq, absmax, err_flag, s)) != SBN_OK) return st;
  return sbn_linear(Xq, absmax, codes, meta, gamma_eff, tokens, out, in, n, m, Y, y_is_bf16,
                    acc_dbg, err_flag, stream);
}

sbn_status sbn_gq_workspace_bytes(int64_t tokens, int64_t out, int64_t in, int groups,
                                  int64_t *workspace_bytes) {
  if (!workspace_bytes) return SBN_ERR_NULL;
  sbn_dims d;
  sbn_status st = sbn_linear_ref_dims(out, in, 2, 4, &d);
  if (st != SBN_OK) return st;
  if ((st = check_groups(in, groups)) != SBN_OK) return st;
  if (tokens < 0 || tokens > (1ll << 31) - 1) return SBN_ERR_SHAPE;
  *workspace_bytes = (int64_t)groups * tokens * out * 4;
  return SBN_OK;
}

sbn_status sbn_quantize_mask_pack_weights_gq(const void *W, int64_t out, int64_t in, int n, int m,
                                             int groups, float eps, uint8_t *codes, uint8_t *meta,
                                             float *gamma_eff, void *workspace, int8_t *dense_dbg,
                                             int32_t *err_flag, void *stream) {
  sbn_dims d;
  sbn_status st = sbn_linear_ref_dims(out, in, n, m, &d);
  if (st != SBN_OK) return st;
  if ((st = check_groups(in, groups)) != SBN_OK) return st;
  if (!W || !codes || !meta || !gamma_eff || !workspace) return SBN_ERR_NULL;
  if (!std::isfinite(eps) || eps < 0.0f) return SBN_ERR_ARG;
  if (!aligned16(W) || !aligned16(codes) || !aligned16(meta) || !aligned16(workspace) ||
      (dense_dbg && !aligned16(dense_dbg)) || (reinterpret_cast<uintptr_t>(gamma_eff) & 3u) ||
      (reinterpret_cast<uintptr_t>(err_flag) & 3u))
    return SBN_ERR_ALIGN;
  return sbn::launch_pack_gq(W, out, in, n, m, groups, eps, codes, d.codes_ld, d.codes_row_bytes,
                             meta, d.meta_ld, d.meta_row_bytes, gamma_eff,
                             static_cast<sbn::PackWorkspace *>(workspace), dense_dbg, err_flag,
                             static_cast<cudaStream_t>(stream));
}

sbn_status sbn_quantize_acts_gq(const void *X, int64_t tokens, int64_t in, int groups, int8_t *Xq,
                                float *absmax, int32_t *err_flag, void *stream) {
  sbn_status st = check_in(in);
  if (st != SBN_OK) return st;
  if ((st = check_groups(in, groups)) != SBN_OK) return st;
  if (tokens < 0 || tokens > (1ll << 31) - 1) return SBN_ERR_SHAPE;
  if (tokens == 0) return SBN_OK;
  if (!X || !Xq || !absmax) return SBN_ERR_NULL;
  if (!aligned16(X) || !aligned16(Xq) || (reinterpret_cast<uintptr_t>(absmax) & 3u) ||
      (reinterpret_cast<uintptr_t>(err_flag) & 3u))
    return SBN_ERR_ALIGN;
  return sbn::launch_act_quant_gq(X, tokens, in, groups, Xq, absmax, err_flag,
                                  static_cast<cudaStream_t>(stream));
}

sbn_status sbn_linear_gq(const int8_t *Xq, const float *absmax, const uint8_t *codes,
                         const uint8_t *meta, const float *gamma_eff, int64_t tokens, int64_t out,
                         int64_t in, int n, int m, int groups, void *Y, int y_is_bf16,
                         void *workspace, int32_t *acc_dbg, int32_t *err_flag, void *stream) {
  sbn_dims d;
  sbn_status st = sbn_linear_ref_dims(out, in, n, m, &d);
  if (st != SBN_OK) return st;
  if ((st = check_groups(in, groups)) != SBN_OK) return st;
  if (tokens < 0 || tokens > (1ll << 31) - 1) return SBN_ERR_SHAPE;
  if (tokens == 0) return SBN_OK;
  if (!Xq || !absmax || !codes || !meta || !gamma_eff || !Y || !workspace) return SBN_ERR_NULL;
  if (!aligned16(Xq) || !aligned16(codes) || !aligned16(meta) || !aligned16(Y) ||
      !aligned16(workspace) || (acc_dbg && !aligned16(acc_dbg)) ||
      (reinterpret_cast<uintptr_t>(absmax) & 3u) || (reinterpret_cast<uintptr_t>(gamma_eff) & 3u) ||
      (reinterpret_cast<uintptr_t>(err_flag) & 3u))
    return SBN_ERR_ALIGN;
  return sbn::launch_linear_gq(Xq, absmax, codes, meta, gamma_eff, tokens, out, in, n, m, groups,
                               d.codes_ld, d.meta_ld, Y, y_is_bf16,
                               static_cast<float *>(workspace), acc_dbg, err_flag,
                               static_cast<cudaStream_t>(stream));
}

sbn_status sbn_pack_group_sizes(const sbn_pack_group_tensor *tensors, int32_t count,
                               int64_t *plan_bytes, int64_t *workspace_bytes) {
  if (!plan_bytes || !workspace_bytes) return SBN_ERR_NULL;
  sbn_status st = check_pack_group(tensors, count);
  if (st != SBN_OK) return st;
  *plan_bytes = sbn::pack_group_plan_bytes(count);
  *workspace_bytes = (int64_t)count * (int64_t)sizeof(sbn::PackGroupSlot);
  return SBN_OK;
}

sbn_status sbn_pack_group_plan(const sbn_pack_group_tensor *tensors, int32_t count, void *plan,
                               int64_t plan_bytes) {
  if (!plan) return SBN_ERR_NULL;
  if (reinterpret_cast<uintptr_t>(plan) & 15u) return SBN_ERR_ALIGN;
  sbn_status st = check_pack_group(tensors, count);
  if (st != SBN_OK) return st;
  if (plan_bytes < sbn::pack_group_plan_bytes(count)) return SBN_ERR_ARG;
  auto *hd = static_cast<sbn::PackGroupHeader *>(plan);
  auto *T = reinterpret_cast<sbn::PackGroupTensor *>(hd + 1);
  std::memset(hd, 0, sizeof(*hd));
  uint32_t chunk = 0, q = 0;
  int mode = -2;  // not yet known
  for (int32_t i = 0; i < count; ++i) {
    const sbn_pack_group_tensor &t = tensors[i];
    sbn::PackGroupTensor e;
    std::memset(&e, 0, sizeof(e));
    if (t.m2 != 0) {  // both patterns: 6:8 into pa, 2:4 into pb, whichever order was asked
      const bool first68 = t.m == 8;
      e.pa = first68 ? pack_args(t.W, t.out, t.in, 6, 8, t.eps, t.codes, t.meta, t.dense_dbg,
                                 t.gamma_eff)
                     : pack_args(t.W, t.out, t.in, 6, 8, t.eps, t.codes2, t.meta2, t.dense_dbg2,
                                 t.gamma_eff);
      e.pb = first68 ? pack_args(t.W, t.out, t.in, 2, 4, t.eps, t.codes2, t.meta2, t.dense_dbg2,
                                 t.gamma_eff)
                     : pack_args(t.W, t.out, t.in, 2, 4, t.eps, t.codes, t.meta, t.dense_dbg,
                                 t.gamma_eff);
      e.pa_compact = 0;
      e.pb_compact = 1;
    } else {
      e.pa = pack_args(t.W, t.out, t.in, t.n, t.m, t.eps, t.codes, t.meta, t.dense_dbg,
                       t.gamma_eff);
      e.pa_compact = t.n == 2;
    }
    const int tmode = (t.dense_dbg || t.dense_dbg2) ? -1 : (t.m2 != 0 ? 2 : (t.n == 2 ? 1 : 0));
    mode = mode == -2 ? tmode : (mode == tmode ? mode : -1);
    e.nvec = t.out * t.in / 8;
    e.chunk_begin = chunk;
    e.nchunks = (uint32_t)((e.nvec + sbn::kPackGroupChunkVecs - 1) / sbn::kPackGroupChunkVecs);
    e.q_begin = q;
    e.nq = (uint32_t)((e.pa.nblocks + 7) / 8);
    chunk += e.nchunks;
    q += e.nq;
    std::memcpy(&T[i], &e, sizeof(e));
  }
  hd->magic = sbn::kPackGroupMagic;
  hd->count = count;
  hd->total_chunks = chunk;
  hd->total_q = q;
  hd->mode = mode < 0 ? -1 : mode;
  return SBN_OK;
}

sbn_status sbn_quantize_mask_pack_weights_group(const void *plan, const void *plan_dev,
                                                void *workspace, int32_t *err_flag,
                                                void *stream) {
  if (!plan || !plan_dev) return SBN_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(plan) & 15u) || (reinterpret_cast<uintptr_t>(plan_dev) & 15u) ||
      (reinterpret_cast<uintptr_t>(workspace) & 15u) || (reinterpret_cast<uintptr_t>(err_flag) & 3u))
    return SBN_ERR_ALIGN;
  const auto *hd = static_cast<const sbn::PackGroupHeader *>(plan);
  if (hd->magic != sbn::kPackGroupMagic) return SBN_ERR_ARG;
  if (hd->count == 0) return SBN_OK;
  if (!workspace) return SBN_ERR_NULL;
  return sbn::launch_pack_group(hd, plan_dev, static_cast<sbn::PackGroupSlot *>(workspace),
                                err_flag, static_cast<cudaStream_t>(stream));
}

sbn_status sbn_gq_sum(const float *part, int64_t n, int32_t G, void *Y, int32_t y_is_bf16,
                      void *stream) {
  if (n < 0 || G < 1 || G > 64) return SBN_ERR_SHAPE;
  if (n == 0) return SBN_OK;
  if (!part || !Y) return SBN_ERR_NULL;
  if (!aligned16(part) || !aligned16(Y)) return SBN_ERR_ALIGN;
  return sbn::launch_gq_sum(part, n, G, Y, y_is_bf16, static_cast<cudaStream_t>(stream));
}

sbn_status sbn_count_zero_codes(const void *W, const float *gamma_eff, int64_t out, int64_t in,
                                unsigned long long *count, void *stream) {
  sbn_dims d;
  sbn_status st = sbn_linear_ref_dims(out, in, 2, 4, &d);  // the shape rules of the pack
  if (st != SBN_OK) return st;
  if (!W || !gamma_eff || !count) return SBN_ERR_NULL;
  if (!aligned16(W) || (reinterpret_cast<uintptr_t>(gamma_eff) & 3u) ||
      (reinterpret_cast<uintptr_t>(count) & 7u))
    return SBN_ERR_ALIGN;
  return sbn::launch_count_zero_codes(W, out * in, gamma_eff, count,
                                      static_cast<cudaStream_t>(stream));
}

sbn_status sbn_count_mask_flips(const uint8_t *meta_a, const uint8_t *meta_b, int64_t out,
                                int64_t in, int n, int m, unsigned long long *count,
                                void *stream) {
  sbn_dims d;
  sbn_status st = sbn_linear_ref_dims(out, in, n, m, &d);
  if (st != SBN_OK) return st;
  if (!meta_a || !meta_b || !count) return SBN_ERR_NULL;
  if (!aligned16(meta_a) || !aligned16(meta_b) || (reinterpret_cast<uintptr_t>(count) & 7u))
    return SBN_ERR_ALIGN;
  return sbn::launch_count_mask_flips(meta_a, meta_b, d.meta_bytes, n == 2 && m == 4, count,
                                      static_cast<cudaStream_t>(stream));
}

}  // extern "C"
