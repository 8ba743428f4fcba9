// Internal launchers behind the C ABI (sbn.h).  Every launcher assumes its arguments were
// validated by the entry point and enqueues work on `st` without synchronising.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "sbn.h"

namespace sbn {

// Device workspace of the weight pack: one partial sum per CTA of the reduction.  The
// quant/mask/pack kernel that follows on the same stream reads them; nothing in the
// workspace needs clearing between calls.
constexpr int kPackMaxParts = 1024;
struct PackWorkspace {
  unsigned long long part[kPackMaxParts];  // one exact partial sum per k_abs_sum CTA
  unsigned int ticket;  // reserved (kept at zero)
  unsigned int thr;     // reserved
  float g;              // reserved
  unsigned int pad;
};

int num_sms();

// Exact b / d for b < 2^25 and 1 <= d <= 2^11: with L = ceil(log2 d) and
// M = ceil(2^(31+L) / d) < 2^32, b / d == (b * M) >> (31 + L): the error term
// b * (M*d - 2^(31+L)) stays below 2^(31+L) because b < 2^31.
struct FastDiv {
  uint32_t mul, shift;  // shift = L - 1, or 0xffffffff for d == 1
};

__device__ __forceinline__ uint32_t fast_div(uint32_t b, FastDiv f) {
  return f.shift == 0xffffffffu ? b : (__umulhi(b, f.mul) >> f.shift);
}

FastDiv make_fast_div(uint32_t d);

// Arguments of the 6:8 and 2:4 quant/mask/pack kernels (64-weight blocks, K % 64 == 0).
struct FastPackArgs {
  const uint4 *W;
  int64_t nblocks;
  uint32_t bpr;  // blocks per row
  FastDiv div_bpr;
  const PackWorkspace *ws;
  uint8_t *codes;
  int64_t ldc, codes_row_bytes;
  uint8_t *meta;
  int64_t ldm, meta_row_bytes;
  int8_t *dense_dbg;
  int nparts;       // partial sums left by k_abs_sum
  int64_t n;        // weights in the tensor
  float eps;
  float *gamma_eff;  // written by CTA 0
};

// 6:8 (compact false) and 2:4 (compact true): the keep masks, metadata and codes in one
// launch after k_abs_sum left a.nparts partial sums in a.ws.
sbn_status launch_fast_pack(const FastPackArgs &a, bool compact, cudaStream_t st);

// Grouped pack: many tensors, one or two of the fast patterns each, in two launches.
// Plan in device memory: a PackGroupHeader, then one PackGroupTensor per tensor.  The
// workspace holds one PackGroupSlot per tensor, zeroed before first use and left zeroed.
constexpr int kPackGroupMaxTensors = 1 << 16;
constexpr int64_t kPackGroupChunkVecs = 16384;  // 16-byte vectors per k_abs_sum_group chunk
constexpr uint32_t kPackGroupMagic = 0x31475053u;  // "SPG1"
struct PackGroupHeader {
  uint32_t magic;
  int32_t count;
  uint32_t total_chunks;  // k_abs_sum_group chunks over all tensors
  uint32_t total_q;       // k_qmp_group warp-iterations (8 blocks of 64 weights each)
  int32_t mode;           // every tensor 6:8 only (0), 2:4 only (1), both (2); mixed: -1
  uint32_t reserved[11];
};
static_assert(sizeof(PackGroupHeader) == 64, "plan header layout");
struct PackGroupTensor {
  FastPackArgs pa;      // first pattern (pa.W, pa.n, pa.eps, pa.gamma_eff used by both);
                        // 6:8 when the tensor packs both patterns
  FastPackArgs pb;      // second pattern (2:4); pb.codes == nullptr when the tensor has one
  int64_t nvec;         // 16-byte vectors of W
  uint32_t chunk_begin, nchunks;
  uint32_t q_begin, nq;
  int32_t pa_compact, pb_compact;  // 1: 2:4, 0: 6:8
};
static_assert(sizeof(PackGroupTensor) % 16 == 0, "plan entries stay 16-byte aligned");
struct PackGroupSlot {
  unsigned long long S;  // exact sum, accumulated by the chunks
  unsigned int done;     // chunks finished
  unsigned int thr;      // code threshold, written by the last chunk
};

int64_t pack_group_plan_bytes(int count);
sbn_status launch_pack_group(const PackGroupHeader *hdr_host, const void *plan_dev,
                             PackGroupSlot *slots, int32_t *err_flag, cudaStream_t st);

sbn_status launch_pack(const void *W, int64_t out, int64_t in, int n, int m, float eps,
                       uint8_t *codes, int64_t ldc, int64_t crow, uint8_t *meta, int64_t ldm,
                       int64_t mrow, float *gamma_eff, PackWorkspace *ws, int8_t *dense_dbg,
                       int32_t *err_flag, cudaStream_t st);

sbn_status launch_act_quant(const void *X, int64_t tokens, int64_t in, int8_t *Xq,
                            float *absmax, int32_t *err_flag, cudaStream_t st);

// CUDA-core contraction for few tokens.
sbn_status launch_gemv(const int8_t *Xq, const float *absmax, const uint8_t *codes,
                       const uint8_t *meta, const float *gamma_eff, int64_t tokens,
                       int64_t out, int64_t in, int64_t ldx, int n, int m, int64_t ldc, int64_t ldm,
                       void *Y, int y_is_bf16, int32_t *acc_dbg, cudaStream_t st);

// Steps 5-7 in one launch for at most kGemvMaxTokens tokens and in <= 16384 (gemv.cu).
sbn_status launch_gemv_fused(const void *X, const uint8_t *codes, const uint8_t *meta,
                             const float *gamma_eff, int64_t tokens, int64_t out, int64_t in,
                             int n, int m, int64_t ldc, int64_t ldm, void *Y, int y_is_bf16,
                             int8_t *Xq, float *absmax, int32_t *acc_dbg, int32_t *err_flag,
                             cudaStream_t st);

// Tensor-core (tcgen05, int8) contraction.
sbn_status launch_gemm_tc(const int8_t *Xq, const float *absmax, const uint8_t *codes,
                          const uint8_t *meta, const float *gamma_eff, int64_t tokens,
                          int64_t out, int64_t in, int64_t ldx, int n, int m, int64_t ldc, int64_t ldm,
                          void *Y, int y_is_bf16, int32_t *acc_dbg, int32_t *err_flag,
                          cudaStream_t st);

// Mask statistics (stats.cu): natural zeros of W for the scale *gamma_eff (n weights),
// and keep-bit differences between two meta planes of nbytes bytes each (index-pair
// nibbles for 2:4, keep masks otherwise).  Both add into *count.
sbn_status launch_count_zero_codes(const void *W, int64_t n, const float *gamma_eff,
                                   unsigned long long *count, cudaStream_t st);
sbn_status launch_count_mask_flips(const uint8_t *meta_a, const uint8_t *meta_b, int64_t nbytes,
                                   bool index_pairs, unsigned long long *count, cudaStream_t st);

// 2-D tensor map over a row-major uint8 matrix [rows, cols] with row stride `ld` bytes and
// a box of box_cols x box_rows bytes (zero fill outside the matrix); false on failure.
bool encode_u8(CUtensorMap *map, const void *base, int64_t cols, int64_t rows, int64_t ld,
               uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swz);

// Grouped calls (gemm_group.cu, act_quant.cu): host-side plan and the two launches.
sbn_status group_plan_sizes(const sbn_group_linear *lins, int count, int64_t *plan_bytes,
                            int64_t *workspace_bytes);
sbn_status group_plan(const sbn_group_linear *lins, int count, void *plan, int64_t plan_bytes);
sbn_status launch_act_quant_group(const void *plan_host, const void *plan_dev, int32_t *err_flag,
                                  cudaStream_t st);
sbn_status launch_linear_group(const void *plan_host, const void *plan_dev, void *workspace,
                               int32_t *err_flag, cudaStream_t st);

// Pre-expanded tensor-core operand of a 2:4 pack (gemm_operand.cu): size, expansion and the
// contraction that reads it (rows padded to 256, K to 128; see k_expand_operand).
int64_t operand_bytes(int64_t out, int64_t in);
sbn_status launch_expand_operand(const uint8_t *codes, const uint8_t *meta, int64_t out,
                                 int64_t in, int64_t ldc, int64_t ldm, void *operand,
                                 cudaStream_t st);
sbn_status launch_gemm_operand(const int8_t *Xq, const float *absmax, const void *operand,
                               const float *gamma_eff, int64_t T, int64_t O, int64_t K, void *Y,
                               int y_is_bf16, int32_t *acc_dbg, int32_t *err_flag,
                               cudaStream_t st);

// Dual-STE backward (backward.cu).
int64_t backward_workspace_bytes(int64_t tokens, int64_t out, int64_t in);
sbn_status launch_backward(const void *dY, const int8_t *Xq, const float *absmax,
                           const uint8_t *codes, const uint8_t *meta, const void *W,
                           const float *gamma_eff, int64_t T, int64_t O, int64_t K, int n, int m,
                           int64_t ldc, int64_t ldm, float *dX, float *dW, void *workspace,
                           int32_t *err_flag, cudaStream_t st);

// Group quantisation (pack.cu, act_quant.cu, group_quant.cu): G blocks along K.
sbn_status launch_pack_gq(const void *W, int64_t out, int64_t in, int n, int m, int G, float eps,
                          uint8_t *codes, int64_t ldc, int64_t crow, uint8_t *meta, int64_t ldm,
                          int64_t mrow, float *gamma_eff, PackWorkspace *ws, int8_t *dense_dbg,
                          int32_t *err_flag, cudaStream_t st);
sbn_status launch_act_quant_gq(const void *X, int64_t tokens, int64_t in, int G, int8_t *Xq,
                               float *absmax, int32_t *err_flag, cudaStream_t st);
// y[i] = fp32 sum over j of part[j * n + i] in j order (group quantisation).
sbn_status launch_gq_sum(const float *part, int64_t n, int G, void *Y, int y_is_bf16,
                         cudaStream_t st);

sbn_status launch_linear_gq(const int8_t *Xq, const float *absmax, const uint8_t *codes,
                            const uint8_t *meta, const float *gamma_eff, int64_t T, int64_t O,
                            int64_t K, int n, int m, int G, int64_t ldc, int64_t ldm, void *Y,
                            int y_is_bf16, float *part, int32_t *acc_dbg, int32_t *err_flag,
                            cudaStream_t st);

// Largest token count routed to the CUDA-core kernel; larger calls use the tensor cores.
constexpr int64_t kGemvMaxTokens = 4;

}  // namespace sbn
