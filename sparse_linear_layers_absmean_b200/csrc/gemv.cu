// CUDA-core contraction for a few tokens (decode).  The packed codes are streamed once
// with 16-byte loads; each 32-bit code word turns into int8 lanes of 64 * t by one shift
// and one AND per four weights, and dp4a does the multiply-free signed sums that the
// pages describe for ternary weights (bitnet.cpp article, "Sistema de pesos ternarios":
// multiplications become additions and subtractions).  The int32 sum is divided by 64
// exactly at the end; y = acc * fp32(fp32(g * s) / 127).
//
// Work split: 8 lanes per output row (a warp owns 4 rows), lane i of a row takes the
// 64-weight chunks i, i+8, ...; the activations of all tokens sit in shared memory.
#include "common.cuh"
#include "kernels.cuh"

namespace sbn {

constexpr int kGvThreads = 256;

// prmt selector that gathers the kept activations of two 2:4 groups: meta byte
// (i0A | i1A << 2 | i0B << 4 | i1B << 6) -> byte selectors i0A, i1A, 4 + i0B, 4 + i1B.
__device__ __forceinline__ uint32_t pair_selector(uint32_t mb) {
  return (mb & 3u) | (((mb >> 2) & 3u) << 4) | ((((mb >> 4) & 3u) + 4u) << 8) |
         ((((mb >> 6) & 3u) + 4u) << 12);
}

template <int T, bool kCompact>
__global__ void __launch_bounds__(kGvThreads)
    k_gemv(const int8_t *__restrict__ Xq, const float *__restrict__ absmax,
           const uint8_t *__restrict__ codes, const uint8_t *__restrict__ meta,
           const float *__restrict__ gamma_eff, int64_t out, int64_t in, int64_t ldc,
           int64_t ldm, void *__restrict__ Y, int y_is_bf16, int32_t *__restrict__ acc_dbg) {
  extern __shared__ __align__(16) uint32_t xs[];  // [T][in/4] int8 words
  const int64_t kw = in / 4;
  for (int64_t i = threadIdx.x; i < T * kw / 4; i += blockDim.x)
    reinterpret_cast<uint4 *>(xs)[i] = __ldg(reinterpret_cast<const uint4 *>(Xq) + i);
  __syncthreads();

  const int lane = threadIdx.x & 31;
  const int sub = lane & 7;
  const int64_t nchunks = in / 64;
  const float g = __ldg(gamma_eff);
  const int64_t rows_per_pass = (int64_t)gridDim.x * (blockDim.x / 8);
  // all lanes of a warp iterate together (shuffles below); rows past the end do no loads
  for (int64_t row0 = (((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5) * 4; row0 < out;
       row0 += rows_per_pass) {
    const int64_t row = row0 + (lane >> 3);
    const bool valid = row < out;
    int acc[T];
#pragma unroll
    for (int t = 0; t < T; ++t) acc[t] = 0;
    if (valid) {
      if constexpr (!kCompact) {
        const uint4 *crow = reinterpret_cast<const uint4 *>(codes + row * ldc);
        for (int64_t c = sub; c < nchunks; c += 8) {
          uint4 cw = __ldg(crow + c);  // 64 positions
          uint32_t w4[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              int z = (int)((w4[q] << (2 * j)) & 0xC0C0C0C0u);
#pragma unroll
              for (int t = 0; t < T; ++t)
                acc[t] = __dp4a(z, (int)xs[t * kw + c * 16 + q * 4 + j], acc[t]);
            }
          }
        }
      } else {
        const uint2 *crow = reinterpret_cast<const uint2 *>(codes + row * ldc);
        const uint2 *mrow = reinterpret_cast<const uint2 *>(meta + row * ldm);
        for (int64_t c = sub; c < nchunks; c += 8) {
          uint2 cw = __ldg(crow + c);  // 32 stored codes = 64 positions
          uint2 mw = __ldg(mrow + c);  // 16 groups
          uint32_t w2[2] = {cw.x, cw.y}, m2[2] = {mw.x, mw.y};
#pragma unroll
          for (int q = 0; q < 2; ++q) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              int z = (int)((w2[q] << (2 * j)) & 0xC0C0C0C0u);
              uint32_t sel = pair_selector((m2[q] >> (8 * j)) & 0xffu);
              const int64_t xw = c * 16 + q * 8 + 2 * j;  // x words of the two groups
#pragma unroll
              for (int t = 0; t < T; ++t) {
                uint32_t xk = __byte_perm(xs[t * kw + xw], xs[t * kw + xw + 1], sel);
                acc[t] = __dp4a(z, (int)xk, acc[t]);
              }
            }
          }
        }
      }
    }
#pragma unroll
    for (int t = 0; t < T; ++t) {
      acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], 1);
      acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], 2);
      acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], 4);
    }
    if (valid && sub < T) {
      // lane `sub` writes token `sub` (T <= 8)
      int a = 0;
#pragma unroll
      for (int t = 0; t < T; ++t)
        if (t == sub) a = acc[t];
      a >>= 6;  // the code lanes carry 64 * t; the sum is an exact multiple of 64
      const float y = __fmul_rn((float)a, rescale_factor(g, __ldg(absmax + sub)));
      if (y_is_bf16)
        reinterpret_cast<__nv_bfloat16 *>(Y)[sub * out + row] = __float2bfloat16_rn(y);
      else
        reinterpret_cast<float *>(Y)[sub * out + row] = y;
      if (acc_dbg) acc_dbg[sub * out + row] = a;
    }
  }
}

template <int T>
static sbn_status gemv_t(const int8_t *Xq, const float *absmax, const uint8_t *codes,
                         const uint8_t *meta, const float *gamma_eff, int64_t out, int64_t in,
                         bool compact, int64_t ldc, int64_t ldm, void *Y, int y_is_bf16,
                         int32_t *acc_dbg, cudaStream_t st) {
  const size_t smem = (size_t)T * (size_t)in;
  const int64_t rows_per_cta = kGvThreads / 8;
  int64_t grid = (out + rows_per_cta - 1) / rows_per_cta;
  const int64_t cap = (int64_t)num_sms() * 8;
  if (grid > cap) grid = cap;
  auto kern = compact ? k_gemv<T, true> : k_gemv<T, false>;
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
          cudaSuccess)
    return SBN_ERR_CUDA;
  kern<<<(unsigned)grid, kGvThreads, smem, st>>>(Xq, absmax, codes, meta, gamma_eff, out, in,
                                                 ldc, ldm, Y, y_is_bf16, acc_dbg);
  SBN_LAUNCH_CHECK();
  return SBN_OK;
}

sbn_status launch_gemv(const int8_t *Xq, const float *absmax, const uint8_t *codes,
                       const uint8_t *meta, const float *gamma_eff, int64_t tokens,
                       int64_t out, int64_t in, int n, int m, int64_t ldc, int64_t ldm,
                       void *Y, int y_is_bf16, int32_t *acc_dbg, cudaStream_t st) {
  const bool compact = (n == 2 && m == 4);
  switch (tokens) {
    case 1:
      return gemv_t<1>(Xq, absmax, codes, meta, gamma_eff, out, in, compact, ldc, ldm, Y,
                       y_is_bf16, acc_dbg, st);
    case 2:
      return gemv_t<2>(Xq, absmax, codes, meta, gamma_eff, out, in, compact, ldc, ldm, Y,
                       y_is_bf16, acc_dbg, st);
    case 3:
      return gemv_t<3>(Xq, absmax, codes, meta, gamma_eff, out, in, compact, ldc, ldm, Y,
                       y_is_bf16, acc_dbg, st);
    case 4:
      return gemv_t<4>(Xq, absmax, codes, meta, gamma_eff, out, in, compact, ldc, ldm, Y,
                       y_is_bf16, acc_dbg, st);
    default:
      return SBN_ERR_SHAPE;
  }
}

}  // namespace sbn
