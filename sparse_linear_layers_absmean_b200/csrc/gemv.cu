// CUDA-core contraction for a few tokens (decode).  The packed codes are streamed once
// with 16-byte loads; each 32-bit code word turns into int8 lanes of 64 * t by one shift
// and one AND per four weights, and dp4a does the multiply-free signed sums that the
// pages describe for ternary weights (bitnet.cpp article, "Sistema de pesos ternarios":
// multiplications become additions and subtractions).  The int32 sum is divided by 64
// exactly at the end; y = acc * fp32(fp32(g * s) / 127).
//
// Work split: two output rows per warp; see k_gemv.
#include "common.cuh"
#include "kernels.cuh"

namespace sbn {

constexpr int kGvThreads = 128;

// prmt selector that gathers the kept activations of two 2:4 groups: meta byte
// (i0A | i1A << 2 | i0B << 4 | i1B << 6) -> byte selectors i0A, i1A, 4 + i0B, 4 + i1B.
__device__ __forceinline__ uint32_t pair_selector(uint32_t mb) {
  return (mb & 3u) | (((mb >> 2) & 3u) << 4) | ((((mb >> 4) & 3u) + 4u) << 8) |
         ((((mb >> 6) & 3u) + 4u) << 12);
}

// Two output rows per warp (rows 2w and 2w + 1), every row in one round: enough CTAs for
// all rows at once, so the whole codes plane is requested in one wave.  Lane l takes the
// 64-weight chunks l, l+32, ... (at most CPL per pass) of both rows; the per-token scales
// are requested first, then both rows' code (and 2:4 metadata) words, then the activation
// words (through L1: every warp of an SM reads the same few KB), each used for both rows.
// The warp reduces with shuffles and lane t writes token t of each row.
constexpr int kGvRows = 2;

template <int T, int CPL, bool kCompact>
__global__ void __launch_bounds__(kGvThreads)
    k_gemv(const int8_t *__restrict__ Xq, const float *__restrict__ absmax,
           const uint8_t *__restrict__ codes, const uint8_t *__restrict__ meta,
           const float *__restrict__ gamma_eff, int64_t out, int64_t in, int64_t ldc,
           int64_t ldm, void *__restrict__ Y, int y_is_bf16, int32_t *__restrict__ acc_dbg) {
  const int lane = threadIdx.x & 31;
  const int64_t row0 = kGvRows * (((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  if (row0 >= out) return;  // whole warps leave together
  const bool two = row0 + 1 < out;
  const float c = lane < T ? rescale_factor(__ldg(gamma_eff), __ldg(absmax + lane)) : 0.0f;
  const int nchunks = (int)(in / 64);
  int acc[kGvRows][T];
#pragma unroll
  for (int r = 0; r < kGvRows; ++r)
#pragma unroll
    for (int t = 0; t < T; ++t) acc[r][t] = 0;
  for (int c0 = 0; c0 < nchunks; c0 += 32 * CPL) {  // one pass unless in > 2048 * CPL
    if constexpr (!kCompact) {
      uint4 cw[kGvRows][CPL];
#pragma unroll
      for (int r = 0; r < kGvRows; ++r) {
        const uint4 *crow = reinterpret_cast<const uint4 *>(codes + (row0 + (two ? r : 0)) * ldc);
#pragma unroll
        for (int i = 0; i < CPL; ++i)
          cw[r][i] = c0 + lane + 32 * i < nchunks ? __ldg(crow + c0 + lane + 32 * i)
                                                  : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int i = 0; i < CPL; ++i) {
        const int ch = c0 + lane + 32 * i;
        if (ch >= nchunks) continue;
#pragma unroll
        for (int t = 0; t < T; ++t) {
          const uint4 *xs = reinterpret_cast<const uint4 *>(Xq + t * in + (int64_t)ch * 64);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint4 x4 = __ldg(xs + q);
            const uint32_t xw[4] = {x4.x, x4.y, x4.z, x4.w};
#pragma unroll
            for (int r = 0; r < kGvRows; ++r) {
              const uint32_t w4[4] = {cw[r][i].x, cw[r][i].y, cw[r][i].z, cw[r][i].w};
#pragma unroll
              for (int j = 0; j < 4; ++j)
                acc[r][t] = __dp4a((int)((w4[q] << (2 * j)) & 0xC0C0C0C0u), (int)xw[j], acc[r][t]);
            }
          }
        }
      }
    } else {
      uint2 cw[kGvRows][CPL], mw[kGvRows][CPL];
#pragma unroll
      for (int r = 0; r < kGvRows; ++r) {
        const int64_t row = row0 + (two ? r : 0);
        const uint2 *crow = reinterpret_cast<const uint2 *>(codes + row * ldc);
        const uint2 *mrow = reinterpret_cast<const uint2 *>(meta + row * ldm);
#pragma unroll
        for (int i = 0; i < CPL; ++i) {
          const bool ok = c0 + lane + 32 * i < nchunks;
          cw[r][i] = ok ? __ldg(crow + c0 + lane + 32 * i) : make_uint2(0, 0);
          mw[r][i] = ok ? __ldg(mrow + c0 + lane + 32 * i) : make_uint2(0, 0);
        }
      }
#pragma unroll
      for (int i = 0; i < CPL; ++i) {
        const int ch = c0 + lane + 32 * i;
        if (ch >= nchunks) continue;
#pragma unroll
        for (int t = 0; t < T; ++t) {
          const uint4 *xs = reinterpret_cast<const uint4 *>(Xq + t * in + (int64_t)ch * 64);
#pragma unroll
          for (int q = 0; q < 2; ++q) {  // 32 stored codes = 8 groups = 32 positions
            const uint4 xa = __ldg(xs + 2 * q), xb = __ldg(xs + 2 * q + 1);
            const uint32_t xw[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
#pragma unroll
            for (int r = 0; r < kGvRows; ++r) {
              const uint32_t w2 = q ? cw[r][i].y : cw[r][i].x, m2 = q ? mw[r][i].y : mw[r][i].x;
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const uint32_t sel = pair_selector((m2 >> (8 * j)) & 0xffu);
                const uint32_t xk = __byte_perm(xw[2 * j], xw[2 * j + 1], sel);
                acc[r][t] = __dp4a((int)((w2 << (2 * j)) & 0xC0C0C0C0u), (int)xk, acc[r][t]);
              }
            }
          }
        }
      }
    }
  }
#pragma unroll
  for (int r = 0; r < kGvRows; ++r)
#pragma unroll
    for (int t = 0; t < T; ++t) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc[r][t] += __shfl_xor_sync(0xffffffffu, acc[r][t], o);
    }
  if (lane < T) {
#pragma unroll
    for (int r = 0; r < kGvRows; ++r) {
      if (r == 1 && !two) break;
      const int64_t row = row0 + r;
      int a = 0;
#pragma unroll
      for (int t = 0; t < T; ++t)
        if (t == lane) a = acc[r][t];
      a >>= 6;  // the code lanes carry 64 * t; the sum is an exact multiple of 64
      const float y = __fmul_rn((float)a, c);
      if (y_is_bf16)
        reinterpret_cast<__nv_bfloat16 *>(Y)[lane * out + row] = __float2bfloat16_rn(y);
      else
        reinterpret_cast<float *>(Y)[lane * out + row] = y;
      if (acc_dbg) acc_dbg[lane * out + row] = a;
    }
  }
}

template <int T, int CPL>
static sbn_status gemv_tc(const int8_t *Xq, const float *absmax, const uint8_t *codes,
                          const uint8_t *meta, const float *gamma_eff, int64_t out, int64_t in,
                          bool compact, int64_t ldc, int64_t ldm, void *Y, int y_is_bf16,
                          int32_t *acc_dbg, cudaStream_t st) {
  const int64_t rows_per_cta = kGvRows * (kGvThreads / 32);
  const int64_t grid = (out + rows_per_cta - 1) / rows_per_cta;
  auto kern = compact ? k_gemv<T, CPL, true> : k_gemv<T, CPL, false>;
  kern<<<(unsigned)grid, kGvThreads, 0, st>>>(Xq, absmax, codes, meta, gamma_eff, out, in, ldc,
                                              ldm, Y, y_is_bf16, acc_dbg);
  SBN_LAUNCH_CHECK();
  return SBN_OK;
}

template <int T>
static sbn_status gemv_t(const int8_t *Xq, const float *absmax, const uint8_t *codes,
                         const uint8_t *meta, const float *gamma_eff, int64_t out, int64_t in,
                         bool compact, int64_t ldc, int64_t ldm, void *Y, int y_is_bf16,
                         int32_t *acc_dbg, cudaStream_t st) {
  const int64_t cpl = (in / 64 + 31) / 32;
  if (cpl <= 1)
    return gemv_tc<T, 1>(Xq, absmax, codes, meta, gamma_eff, out, in, compact, ldc, ldm, Y,
                         y_is_bf16, acc_dbg, st);
  if (cpl <= 2)
    return gemv_tc<T, 2>(Xq, absmax, codes, meta, gamma_eff, out, in, compact, ldc, ldm, Y,
                         y_is_bf16, acc_dbg, st);
  if (cpl <= 4)
    return gemv_tc<T, 4>(Xq, absmax, codes, meta, gamma_eff, out, in, compact, ldc, ldm, Y,
                         y_is_bf16, acc_dbg, st);
  return gemv_tc<T, 8>(Xq, absmax, codes, meta, gamma_eff, out, in, compact, ldc, ldm, Y,
                       y_is_bf16, acc_dbg, st);
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
