// Shared device helpers of the Sparse-BitLinear kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "sbn.h"

namespace sbn {

constexpr int kWarp = 32;

// Magnitude bits of bf16 values: NaN/Inf have all exponent bits set (>= 0x7f80);
// 256.0 is 0x4380, the first magnitude outside the supported weight range.
constexpr uint32_t kBf16InfBits = 0x7f80u;
constexpr uint32_t kBf16Mag256Bits = 0x4380u;

__device__ __forceinline__ float bf16_lo_to_float(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi_to_float(uint32_t w) {
  return __uint_as_float(w & 0xffff0000u);
}

__device__ __forceinline__ uint4 ldg_v4(const void *p) {
  return __ldg(reinterpret_cast<const uint4 *>(p));
}

__device__ __forceinline__ unsigned long long warp_sum_u64(unsigned long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ uint32_t warp_max_u32(uint32_t v) {
  return __reduce_max_sync(0xffffffffu, v);
}

__device__ __forceinline__ uint32_t warp_or_u32(uint32_t v) {
  return __reduce_or_sync(0xffffffffu, v);
}

// Activation codes q = clamp(rint(fl(r / s)), -127, 127) of eight values r = fl(127 x) of one
// token, with the quotient rounded as the IEEE divide rounds it, from the products
// p = fl(r * inv), inv = fl(1 / s) (correctly rounded, once per token).  inv and the product
// each carry a relative error of at most 2^-24 and the rounded quotient another 2^-24, so
// for |r / s| < 128 the product is within 3 * 128 * 2^-24 < 2^-15 of the rounded quotient.
// rint changes value only at half-integers: a product farther than 2^-15 from every k + 1/2
// rounds to the same integer as the rounded quotient.  When one of the eight lies nearer
// (exact ties among them), all eight take the divide, on a branch of their own.  Past
// +-127.5 both sides clamp to the same code; NaN and infinity propagate through the product
// as through the divide.
__device__ __forceinline__ void act_codes8(const float (&r)[8], float s, float inv,
                                           int (&q)[8]) {
  float p[8];
  bool near = false;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    p[i] = __fmul_rn(r[i], inv);
    // distance to the nearest integer (exact); at least 1/2 - 2^-15 <=> within 2^-15 of a
    // half-integer.  NaN and infinity give NaN here and stay on the product.
    near |= fabsf(__fsub_rn(p[i], rintf(p[i]))) >= 0.5f - 0x1p-15f;
  }
  if (near) {
#pragma unroll
    for (int i = 0; i < 8; ++i) p[i] = __fdiv_rn(r[i], s);
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) q[i] = min(127, max(-127, __float2int_rn(p[i])));
}

// Eight bf16 activations (one 16-byte word) -> eight int8 codes, in order.
__device__ __forceinline__ uint2 act_codes_vec8(uint4 v, float s, float inv) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  float r[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    r[2 * i] = __fmul_rn(127.0f, bf16_lo_to_float(w[i]));
    r[2 * i + 1] = __fmul_rn(127.0f, bf16_hi_to_float(w[i]));
  }
  int q[8];
  act_codes8(r, s, inv, q);
  uint32_t o[2] = {0u, 0u};
#pragma unroll
  for (int i = 0; i < 8; ++i) o[i >> 2] |= ((uint32_t)q[i] & 0xffu) << (8 * (i & 3));
  return make_uint2(o[0], o[1]);
}

// Per-token activation scale and weight scale combined as the rescale factor
// c = fp32(fp32(g * s) / 127), then y = fp32(acc * c); no FMA contraction anywhere.
__device__ __forceinline__ float rescale_factor(float g, float s) {
  return __fdiv_rn(__fmul_rn(g, s), 127.0f);
}

}  // namespace sbn

// Host-side launch check shared by the entry points.
// Launch as a programmatic dependent of the previous kernel on the stream (programmatic
// stream serialisation): the launch and the kernel's prologue may overlap that kernel's
// tail; the kernel executes griddepcontrol.wait before it touches global memory, which
// returns once the previous kernel has completed and its writes are visible.
template <typename... KArgs, typename... Args>
inline sbn_status launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                             cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...) != cudaSuccess) {
    (void)cudaGetLastError();
    return SBN_ERR_CUDA;
  }
  return SBN_OK;
}

#define SBN_LAUNCH_CHECK()                                         \
  do {                                                             \
    if (cudaPeekAtLastError() != cudaSuccess) {                    \
      (void)cudaGetLastError();                                    \
      return SBN_ERR_CUDA;                                         \
    }                                                              \
  } while (0)
