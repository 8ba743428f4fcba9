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

// The same sum four outputs at a time (16-byte loads of every block's partials); for n a
// multiple of 4 with 16-byte aligned partials and 16- (fp32) or 8-byte (bf16) aligned Y.
__global__ void __launch_bounds__(256)
    k_gq_sum4(const float4 *__restrict__ part, int64_t n4, int G, void *__restrict__ Y,
              int y_is_bf16) {
  ptx::grid_dep_launch();
  ptx::grid_dep_wait();
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4;
       i += (int64_t)gridDim.x * blockDim.x) {
    float4 y = __ldg(part + i);
    for (int j = 1; j < G; ++j) {
      const float4 p = __ldg(part + j * n4 + i);
      y.x = __fadd_rn(y.x, p.x);
      y.y = __fadd_rn(y.y, p.y);
      y.z = __fadd_rn(y.z, p.z);
      y.w = __fadd_rn(y.w, p.w);
    }
    if (y_is_bf16) {
      const uint32_t lo = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(y.x)) |
                          ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(y.y)) << 16);
      const uint32_t hi = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(y.z)) |
                          ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(y.w)) << 16);
      reinterpret_cast<uint2 *>(Y)[i] = make_uint2(lo, hi);
    } else {
      reinterpret_cast<float4 *>(Y)[i] = y;
    }
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
  const int64_t cap = (int64_t)num_sms() * 8;
  const uintptr_t ya = reinterpret_cast<uintptr_t>(Y);
  if (n % 4 == 0 && (reinterpret_cast<uintptr_t>(part) & 15u) == 0 &&
      (ya & (y_is_bf16 ? 7u : 15u)) == 0) {
    int64_t grid = (n / 4 + 255) / 256;
    if (grid > cap) grid = cap;
    return launch_pdl(k_gq_sum4, dim3((unsigned)grid), dim3(256), 0, st,
                      reinterpret_cast<const float4 *>(part), n / 4, G, Y, y_is_bf16);
  }
  int64_t grid = (n + 255) / 256;
  if (grid > cap) grid = cap;
  return launch_pdl(k_gq_sum, dim3((unsigned)grid), dim3(256), 0, st, part, n, G, Y, y_is_bf16);
}

}  // namespace sbn
