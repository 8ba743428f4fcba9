// Group quantisation, contraction (the bitnet.cpp article's group quantisation: weights and
// activations in G groups with parameters of their own; here G blocks along K).  Block j is
// a Sparse-BitLinear of its own: its int32 sums acc_j (exact) are rescaled by
// c_tj = fp32(fp32(g_j * s_tj) / 127) into y_j = fp32(acc_j * c_tj) by the regular
// contraction kernels, run on the block's slice of the packed planes and of Xq (the TMA
// descriptors and the GEMV take the full row strides); k_gq_sum then adds the G partial
// outputs in group order in fp32 and stores fp32 or bf16.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

namespace sbn {

namespace {

__global__ void __launch_bounds__(256)
    k_gq_sum(const float *__restrict__ part, int64_t n, int G, void *__restrict__ Y,
             int y_is_bf16) {
  ptx::grid_dep_launch();
  ptx::grid_dep_wait();
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    float y = part[i];
    for (int j = 1; j < G; ++j) y = __fadd_rn(y, part[j * n + i]);
    if (y_is_bf16)
      reinterpret_cast<__nv_bfloat16 *>(Y)[i] = __float2bfloat16_rn(y);
    else
      reinterpret_cast<float *>(Y)[i] = y;
  }
}

}  // namespace

sbn_status launch_linear_gq(const int8_t *Xq, const float *absmax, const uint8_t *codes,
                            const uint8_t *meta, const float *gamma_eff, int64_t T, int64_t O,
                            int64_t K, int n, int m, int G, int64_t ldc, int64_t ldm, void *Y,
                            int y_is_bf16, float *part, int32_t *acc_dbg, int32_t *err_flag,
                            cudaStream_t st) {
  const bool compact = (n == 2 && m == 4);
  const int64_t kg = K / G;
  const int64_t cbytes = compact ? kg / 8 : kg / 4;  // code bytes of one block of one row
  for (int j = 0; j < G; ++j) {
    const int8_t *xj = Xq + j * kg;
    const uint8_t *cj = codes + j * cbytes;
    const uint8_t *mj = meta + j * (kg / 8);
    float *yj = part + (int64_t)j * T * O;
    int32_t *aj = acc_dbg ? acc_dbg + (int64_t)j * T * O : nullptr;
    const sbn_status s =
        T <= kGemvMaxTokens
            ? launch_gemv(xj, absmax + j * T, cj, mj, gamma_eff + j, T, O, kg, K, n, m, ldc, ldm,
                          yj, 0, aj, st)
            : launch_gemm_tc(xj, absmax + j * T, cj, mj, gamma_eff + j, T, O, kg, K, n, m, ldc,
                             ldm, yj, 0, aj, err_flag, st);
    if (s != SBN_OK) return s;
  }
  return launch_gq_sum(part, T * O, G, Y, y_is_bf16, st);
}

sbn_status launch_gq_sum(const float *part, int64_t n, int G, void *Y, int y_is_bf16,
                         cudaStream_t st) {
  int64_t grid = (n + 255) / 256;
  const int64_t cap = (int64_t)num_sms() * 8;
  if (grid > cap) grid = cap;
  return launch_pdl(k_gq_sum, dim3((unsigned)grid), dim3(256), 0, st, part, n, G, Y, y_is_bf16);
}

}  // namespace sbn
