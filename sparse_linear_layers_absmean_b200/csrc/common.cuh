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
