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
#include "ptx.cuh"

namespace sbn {

constexpr int kGvThreads = 128;

// prmt selectors that gather the kept activations of 2:4 groups, two at a time: each meta
// byte (i0A | i1A << 2 | i0B << 4 | i1B << 6) becomes the 16-bit selector with nibbles
// i0A, i1A, 4 + i0B, 4 + i1B.  For meta bytes b0, b1 in the low 16 bits of m, the result
// holds the selector of b0 in bits 0-15 and that of b1 in bits 16-31 (prmt reads the low
// 16 bits of its selector): every 2-bit field is spread to its own nibble.
__device__ __forceinline__ uint32_t pair_selectors(uint32_t m) {
  uint32_t x = m & 0xffffu;
  x = (x | (x << 8)) & 0x00ff00ffu;
  x = (x | (x << 4)) & 0x0f0f0f0fu;
  x = (x | (x << 2)) & 0x33333333u;
  return x + 0x44004400u;
}

// Two output rows per warp (rows 2w and 2w + 1), every row in one round: enough CTAs for
// all rows at once, so the whole codes plane is requested in one wave.  The row is cut
// into segments of 32 code words (one per lane): for 6:8 / dense codes a word holds 16
// weights and the lane's activations are the 16 bytes at 16 l of the 512-input segment;
// for 2:4 a word holds the 16 kept codes of 32 inputs with one metadata word beside it,
// and the lane's activations are the 32 bytes at 32 l of the 1024-input segment.  Both
// code and activation loads are contiguous across the warp.  SPL segments are requested
// per pass (the per-token scales first, then both rows' code and metadata words, then the
// activations, each used for both rows); the warp reduces with shuffles and lane t writes
// token t of each row.
constexpr int kGvRows = 2;

template <int T, int SPL, bool kCompact>
__global__ void __launch_bounds__(kGvThreads)
    k_gemv(const int8_t *__restrict__ Xq, const float *__restrict__ absmax,
           const uint8_t *__restrict__ codes, const uint8_t *__restrict__ meta,
           const float *__restrict__ gamma_eff, int nt, int64_t out, int64_t in, int64_t ldx,
           int64_t ldc, int64_t ldm, void *__restrict__ Y, int y_is_bf16,
           int32_t *__restrict__ acc_dbg) {
  // T: tokens the kernel is built for; nt <= T: tokens present (rows nt.. of Xq do not exist);
  // ldx: elements between Xq rows (in, or more for a slice of wider rows)
  const int lane = threadIdx.x & 31;
  const int64_t row0 = kGvRows * (((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  // launched as a programmatic dependent: everything read below comes from earlier kernels;
  // the next kernel on the stream may start its prologue (it waits for this one)
  ptx::grid_dep_launch();
  ptx::grid_dep_wait();
  if (row0 >= out) return;  // whole warps leave together
  const bool two = row0 + 1 < out;
  const float c = lane < nt ? rescale_factor(__ldg(gamma_eff), __ldg(absmax + lane)) : 0.0f;
  const int nwords = (int)(in / (kCompact ? 32 : 16));  // code words per row
  const uint32_t *crow[kGvRows], *mrow[kGvRows];
#pragma unroll
  for (int r = 0; r < kGvRows; ++r) {
    const int64_t row = row0 + (two ? r : 0);
    crow[r] = reinterpret_cast<const uint32_t *>(codes + row * ldc);
    mrow[r] = reinterpret_cast<const uint32_t *>(meta + row * ldm);
  }
  int acc[kGvRows][T];
#pragma unroll
  for (int r = 0; r < kGvRows; ++r)
#pragma unroll
    for (int t = 0; t < T; ++t) acc[r][t] = 0;
  for (int w0 = 0; w0 < nwords; w0 += 32 * SPL) {  // one pass for rows up to 32 * SPL words
    uint32_t cw[kGvRows][SPL], mw[kGvRows][SPL];
#pragma unroll
    for (int r = 0; r < kGvRows; ++r)
#pragma unroll
      for (int i = 0; i < SPL; ++i) {
        const int wi = w0 + 32 * i + lane;
        cw[r][i] = wi < nwords ? __ldg(crow[r] + wi) : 0u;
        if constexpr (kCompact) mw[r][i] = wi < nwords ? __ldg(mrow[r] + wi) : 0u;
      }
#pragma unroll
    for (int i = 0; i < SPL; ++i) {
      const int wi = w0 + 32 * i + lane;
      if (wi >= nwords) continue;
#pragma unroll
      for (int t = 0; t < T; ++t) {
        if (t >= nt) break;
        if constexpr (!kCompact) {
          const uint4 x4 = __ldg(reinterpret_cast<const uint4 *>(Xq + t * ldx + (int64_t)wi * 16));
          const uint32_t xw[4] = {x4.x, x4.y, x4.z, x4.w};
#pragma unroll
          for (int r = 0; r < kGvRows; ++r)
#pragma unroll
            for (int j = 0; j < 4; ++j)  // weights 4j..4j+3 sit in bits 7-2j..6-2j of the bytes
              acc[r][t] = __dp4a((int)((cw[r][i] << (2 * j)) & 0xC0C0C0C0u), (int)xw[j], acc[r][t]);
        } else {
          const uint4 *xs = reinterpret_cast<const uint4 *>(Xq + t * ldx + (int64_t)wi * 32);
          const uint4 xa = __ldg(xs), xb = __ldg(xs + 1);
          const uint32_t xw[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
#pragma unroll
          for (int r = 0; r < kGvRows; ++r) {
            // selectors of groups (0,1), (2,3) | (4,5), (6,7); the same for every token
            const uint32_t s01 = pair_selectors(mw[r][i]), s23 = pair_selectors(mw[r][i] >> 16);
            const uint32_t sel[4] = {s01, s01 >> 16, s23, s23 >> 16};
#pragma unroll
            for (int j = 0; j < 4; ++j) {  // groups 2j, 2j+1: stored codes 4j..4j+3
              const uint32_t xk = __byte_perm(xw[2 * j], xw[2 * j + 1], sel[j]);
              acc[r][t] = __dp4a((int)((cw[r][i] << (2 * j)) & 0xC0C0C0C0u), (int)xk, acc[r][t]);
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
  if (lane < nt) {
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

// Steps 5-7 in one launch for a few tokens: every CTA quantises the (small) token rows
// itself -- the per-token absmax by a block reduction over X (bf16, read from L2), then
// q = clamp(rint((127 x) / s), -127, 127) (rounded as the IEEE divide rounds the quotient)
// into shared memory -- and
// runs the GEMV above on them (two rows per warp, 8 warps per CTA, activations from shared
// memory).  CTA 0 also writes Xq and s to global memory.  Shared memory: T * in bytes
// (in <= 16384).
constexpr int64_t kFusedMaxIn = 16384;
// 8 warps (16 rows) per CTA: the row quantisation every CTA repeats is spread over 256
// threads and over 2x fewer CTAs than the GEMV's 8-row CTAs
constexpr int kGfThreads = 256;

template <int T, int SPL, bool kCompact>
__global__ void __launch_bounds__(kGfThreads)
    k_gemv_fused(const uint16_t *__restrict__ X, const uint8_t *__restrict__ codes,
                 const uint8_t *__restrict__ meta, const float *__restrict__ gamma_eff, int nt,
                 int64_t out, int64_t in, int64_t ldc, int64_t ldm, void *__restrict__ Y,
                 int y_is_bf16, int8_t *__restrict__ Xq_out, float *__restrict__ absmax_out,
                 int32_t *__restrict__ acc_dbg, int32_t *err_flag) {
  extern __shared__ __align__(16) uint8_t s_xq[];  // [T][in] int8
  __shared__ uint32_t s_red[T][kGfThreads / 32];
  __shared__ float s_scale[T];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  ptx::grid_dep_launch();
  ptx::grid_dep_wait();
  const int64_t nv = in / 8;  // 16-byte words (8 bf16) per token row
  // per-token absmax (as bf16 magnitude bits; max of bits is max of magnitudes)
  for (int t = 0; t < T; ++t) {
    if (t >= nt) break;
    const uint4 *row = reinterpret_cast<const uint4 *>(X + t * in);
    uint32_t mx = 0;
    for (int64_t i = threadIdx.x; i < nv; i += kGfThreads) {
      const uint4 v = __ldg(row + i);
      mx = __vmaxu2(mx, v.x & 0x7fff7fffu);
      mx = __vmaxu2(mx, v.y & 0x7fff7fffu);
      mx = __vmaxu2(mx, v.z & 0x7fff7fffu);
      mx = __vmaxu2(mx, v.w & 0x7fff7fffu);
    }
    const uint32_t m = warp_max_u32(max(mx & 0xffffu, mx >> 16));
    if (lane == 0) s_red[t][wid] = m;
  }
  __syncthreads();
  if (threadIdx.x < nt) {
    uint32_t m = 0;
#pragma unroll
    for (int w = 0; w < kGfThreads / 32; ++w) m = max(m, s_red[threadIdx.x][w]);
    if (m >= kBf16InfBits && blockIdx.x == 0 && err_flag) atomicOr(err_flag, SBN_FLAG_X_NONFINITE);
    const float sc = fmaxf(__uint_as_float(m << 16), 1e-5f);
    s_scale[threadIdx.x] = sc;
    if (blockIdx.x == 0 && absmax_out) absmax_out[threadIdx.x] = sc;
  }
  __syncthreads();
  for (int t = 0; t < T; ++t) {
    if (t >= nt) break;
    const float sc = s_scale[t];
    const float inv = __frcp_rn(sc);
    const uint4 *row = reinterpret_cast<const uint4 *>(X + t * in);
    uint2 *q = reinterpret_cast<uint2 *>(s_xq + t * in);
    uint2 *qg = Xq_out ? reinterpret_cast<uint2 *>(Xq_out + t * in) : nullptr;
    for (int64_t i = threadIdx.x; i < nv; i += kGfThreads) {
      const uint4 v = __ldg(row + i);
      const uint2 o = act_codes_vec8(v, sc, inv);
      q[i] = o;
      if (blockIdx.x == 0 && qg) qg[i] = o;
    }
  }
  __syncthreads();

  const int64_t row0 = kGvRows * (((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  if (row0 >= out) return;  // whole warps leave together
  const bool two = row0 + 1 < out;
  const float c = lane < nt ? rescale_factor(__ldg(gamma_eff), s_scale[lane]) : 0.0f;
  const int nwords = (int)(in / (kCompact ? 32 : 16));
  const uint32_t *crow[kGvRows], *mrow[kGvRows];
#pragma unroll
  for (int r = 0; r < kGvRows; ++r) {
    const int64_t row = row0 + (two ? r : 0);
    crow[r] = reinterpret_cast<const uint32_t *>(codes + row * ldc);
    mrow[r] = reinterpret_cast<const uint32_t *>(meta + row * ldm);
  }
  int acc[kGvRows][T];
#pragma unroll
  for (int r = 0; r < kGvRows; ++r)
#pragma unroll
    for (int t = 0; t < T; ++t) acc[r][t] = 0;
  for (int w0 = 0; w0 < nwords; w0 += 32 * SPL) {
    uint32_t cw[kGvRows][SPL], mw[kGvRows][SPL];
#pragma unroll
    for (int r = 0; r < kGvRows; ++r)
#pragma unroll
      for (int i = 0; i < SPL; ++i) {
        const int wi = w0 + 32 * i + lane;
        cw[r][i] = wi < nwords ? __ldg(crow[r] + wi) : 0u;
        if constexpr (kCompact) mw[r][i] = wi < nwords ? __ldg(mrow[r] + wi) : 0u;
      }
#pragma unroll
    for (int i = 0; i < SPL; ++i) {
      const int wi = w0 + 32 * i + lane;
      if (wi >= nwords) continue;
#pragma unroll
      for (int t = 0; t < T; ++t) {
        if (t >= nt) break;
        if constexpr (!kCompact) {
          const uint4 x4 = *reinterpret_cast<const uint4 *>(s_xq + t * in + (int64_t)wi * 16);
          const uint32_t xw[4] = {x4.x, x4.y, x4.z, x4.w};
#pragma unroll
          for (int r = 0; r < kGvRows; ++r)
#pragma unroll
            for (int j = 0; j < 4; ++j)
              acc[r][t] = __dp4a((int)((cw[r][i] << (2 * j)) & 0xC0C0C0C0u), (int)xw[j], acc[r][t]);
        } else {
          const uint4 *xs = reinterpret_cast<const uint4 *>(s_xq + t * in + (int64_t)wi * 32);
          const uint4 xa = xs[0], xb = xs[1];
          const uint32_t xw[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
#pragma unroll
          for (int r = 0; r < kGvRows; ++r) {
            const uint32_t s01 = pair_selectors(mw[r][i]), s23 = pair_selectors(mw[r][i] >> 16);
            const uint32_t sel[4] = {s01, s01 >> 16, s23, s23 >> 16};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const uint32_t xk = __byte_perm(xw[2 * j], xw[2 * j + 1], sel[j]);
              acc[r][t] = __dp4a((int)((cw[r][i] << (2 * j)) & 0xC0C0C0C0u), (int)xk, acc[r][t]);
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
  if (lane < nt) {
#pragma unroll
    for (int r = 0; r < kGvRows; ++r) {
      if (r == 1 && !two) break;
      const int64_t row = row0 + r;
      int a = 0;
#pragma unroll
      for (int t = 0; t < T; ++t)
        if (t == lane) a = acc[r][t];
      a >>= 6;
      const float y = __fmul_rn((float)a, c);
      if (y_is_bf16)
        reinterpret_cast<__nv_bfloat16 *>(Y)[lane * out + row] = __float2bfloat16_rn(y);
      else
        reinterpret_cast<float *>(Y)[lane * out + row] = y;
      if (acc_dbg) acc_dbg[lane * out + row] = a;
    }
  }
}

template <int T, int SPL>
static sbn_status gemv_fused_t(const void *X, const uint8_t *codes, const uint8_t *meta,
                               const float *gamma_eff, int nt, int64_t out, int64_t in,
                               bool compact, int64_t ldc, int64_t ldm, void *Y, int y_is_bf16,
                               int8_t *Xq, float *absmax, int32_t *acc_dbg, int32_t *err_flag,
                               cudaStream_t st) {
  const int64_t rows_per_cta = kGvRows * (kGfThreads / 32);
  const int64_t grid = (out + rows_per_cta - 1) / rows_per_cta;
  auto kern = compact ? k_gemv_fused<T, SPL, true> : k_gemv_fused<T, SPL, false>;
  const size_t smem = (size_t)T * (size_t)in;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)(T * kFusedMaxIn)) != cudaSuccess)
    return SBN_ERR_CUDA;
  return launch_pdl(kern, dim3((unsigned)grid), dim3(kGfThreads), smem, st,
                    static_cast<const uint16_t *>(X), codes, meta, gamma_eff, nt, out, in, ldc,
                    ldm, Y, y_is_bf16, Xq, absmax, acc_dbg, err_flag);
}

template <int T>
static sbn_status gemv_fused_spl(const void *X, const uint8_t *codes, const uint8_t *meta,
                                 const float *gamma_eff, int nt, int64_t out, int64_t in,
                                 bool compact, int64_t ldc, int64_t ldm, void *Y, int y_is_bf16,
                                 int8_t *Xq, float *absmax, int32_t *acc_dbg, int32_t *err_flag,
                                 cudaStream_t st) {
  const int64_t spl = (in / (compact ? 32 : 16) + 31) / 32;
  if (spl <= 2)
    return gemv_fused_t<T, 2>(X, codes, meta, gamma_eff, nt, out, in, compact, ldc, ldm, Y,
                              y_is_bf16, Xq, absmax, acc_dbg, err_flag, st);
  if (spl <= 4)
    return gemv_fused_t<T, 4>(X, codes, meta, gamma_eff, nt, out, in, compact, ldc, ldm, Y,
                              y_is_bf16, Xq, absmax, acc_dbg, err_flag, st);
  if (spl <= 6 || T > 2)
    return gemv_fused_t<T, 6>(X, codes, meta, gamma_eff, nt, out, in, compact, ldc, ldm, Y,
                              y_is_bf16, Xq, absmax, acc_dbg, err_flag, st);
  return gemv_fused_t<T, 8>(X, codes, meta, gamma_eff, nt, out, in, compact, ldc, ldm, Y,
                            y_is_bf16, Xq, absmax, acc_dbg, err_flag, st);
}

sbn_status launch_gemv_fused(const void *X, const uint8_t *codes, const uint8_t *meta,
                             const float *gamma_eff, int64_t tokens, int64_t out, int64_t in,
                             int n, int m, int64_t ldc, int64_t ldm, void *Y, int y_is_bf16,
                             int8_t *Xq, float *absmax, int32_t *acc_dbg, int32_t *err_flag,
                             cudaStream_t st) {
  const bool compact = (n == 2 && m == 4);
  const int nt = (int)tokens;
  if (in > kFusedMaxIn) return SBN_ERR_SHAPE;
#define SBN_GEMVF(TT)                                                                          \
  return gemv_fused_spl<TT>(X, codes, meta, gamma_eff, nt, out, in, compact, ldc, ldm, Y,    \
                            y_is_bf16, Xq, absmax, acc_dbg, err_flag, st)
  if (tokens == 1) SBN_GEMVF(1);
  if (tokens == 2) SBN_GEMVF(2);
  if (tokens == 3) SBN_GEMVF(3);
  if (tokens == 4) SBN_GEMVF(4);
#undef SBN_GEMVF
  return SBN_ERR_SHAPE;
}

template <int T, int SPL>
static sbn_status gemv_tc(const int8_t *Xq, const float *absmax, const uint8_t *codes,
                          const uint8_t *meta, const float *gamma_eff, int nt, int64_t out,
                          int64_t in, int64_t ldx,
                          bool compact, int64_t ldc, int64_t ldm, void *Y, int y_is_bf16,
                          int32_t *acc_dbg, cudaStream_t st) {
  const int64_t rows_per_cta = kGvRows * (kGvThreads / 32);
  const int64_t grid = (out + rows_per_cta - 1) / rows_per_cta;
  auto kern = compact ? k_gemv<T, SPL, true> : k_gemv<T, SPL, false>;
  // programmatic dependent launch: the GEMV's CTAs may be scheduled while the kernel before
  // it on the stream (the pack) drains; griddepcontrol.wait in the kernel keeps the order
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(kGvThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, Xq, absmax, codes, meta, gamma_eff, nt, out, in, ldx, ldc,
                         ldm, Y, y_is_bf16, acc_dbg) != cudaSuccess) {
    (void)cudaGetLastError();
    return SBN_ERR_CUDA;
  }
  return SBN_OK;
}

template <int T>
static sbn_status gemv_t(const int8_t *Xq, const float *absmax, const uint8_t *codes,
                         const uint8_t *meta, const float *gamma_eff, int nt, int64_t out,
                         int64_t in, int64_t ldx,
                         bool compact, int64_t ldc, int64_t ldm, void *Y, int y_is_bf16,
                         int32_t *acc_dbg, cudaStream_t st) {
  const int64_t words = in / (compact ? 32 : 16);  // code words per row
  const int64_t spl = (words + 31) / 32;
  if (spl <= 2)
    return gemv_tc<T, 2>(Xq, absmax, codes, meta, gamma_eff, nt, out, in, ldx, compact, ldc, ldm, Y,
                         y_is_bf16, acc_dbg, st);
  if (spl <= 4)
    return gemv_tc<T, 4>(Xq, absmax, codes, meta, gamma_eff, nt, out, in, ldx, compact, ldc, ldm, Y,
                         y_is_bf16, acc_dbg, st);
  if (spl <= 6 || T > 2)
    return gemv_tc<T, 6>(Xq, absmax, codes, meta, gamma_eff, nt, out, in, ldx, compact, ldc, ldm, Y,
                         y_is_bf16, acc_dbg, st);
  return gemv_tc<T, 8>(Xq, absmax, codes, meta, gamma_eff, nt, out, in, ldx, compact, ldc, ldm, Y,
                       y_is_bf16, acc_dbg, st);
}

sbn_status launch_gemv(const int8_t *Xq, const float *absmax, const uint8_t *codes,
                       const uint8_t *meta, const float *gamma_eff, int64_t tokens,
                       int64_t out, int64_t in, int64_t ldx, int n, int m, int64_t ldc, int64_t ldm,
                       void *Y, int y_is_bf16, int32_t *acc_dbg, cudaStream_t st) {
  const bool compact = (n == 2 && m == 4);
  const int nt = (int)tokens;
#define SBN_GEMV(TT)                                                                         \
  return gemv_t<TT>(Xq, absmax, codes, meta, gamma_eff, nt, out, in, ldx, compact, ldc, ldm, Y, \
                    y_is_bf16, acc_dbg, st)
  if (tokens == 1) SBN_GEMV(1);
  if (tokens == 2) SBN_GEMV(2);
  if (tokens == 3) SBN_GEMV(3);
  if (tokens == 4) SBN_GEMV(4);
#undef SBN_GEMV
  return SBN_ERR_SHAPE;
}

}  // namespace sbn
