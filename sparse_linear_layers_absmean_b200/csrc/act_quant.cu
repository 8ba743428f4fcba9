// Per-token absmax int8 activation quantisation ("Marco de inferencia de Microsoft lleva
// modelos de lenguaje grande de 1 bit a dispositivos locales", unite.ai, "Fundamento
// matemático" item 2; Qb = 127):
//   s = max(max_k |x_k|, 1e-5),  q_k = clamp(rint((127 * x_k) / s), -127, 127),
// the quotient rounded as the IEEE divide rounds it (act_codes8: products with the token's
// reciprocal, and the divide itself where a product lies near a half-integer).
// One CTA per token; rows of up to 16384 inputs stay in registers between the max pass and
// the quantise pass (one HBM read), longer rows are read twice.  Many tokens with rows of up
// to 1024 inputs: one warp per token (k_act_quant_warp).  Every kernel is
// launched as a programmatic dependent of the previous kernel on the stream and waits for
// it before reading X.
#include "common.cuh"
#include "group.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

namespace sbn {

constexpr int kAqThreads = 256;

// eight bf16 values -> eight int8 codes; inv = fl(1 / s)
__device__ __forceinline__ uint2 quant_vec8(uint4 v, float s, float inv) {
  return act_codes_vec8(v, s, inv);
}

__device__ __forceinline__ uint32_t vec8_absmax_bits(uint4 v, uint32_t mx) {
  mx = __vmaxu2(mx, v.x & 0x7fff7fffu);
  mx = __vmaxu2(mx, v.y & 0x7fff7fffu);
  mx = __vmaxu2(mx, v.z & 0x7fff7fffu);
  mx = __vmaxu2(mx, v.w & 0x7fff7fffu);
  return mx;
}

// Block-wide max of the per-thread packed magnitudes; returns the token's scale s.
__device__ __forceinline__ float block_scale(uint32_t mx, int32_t *err_flag) {
  __shared__ uint32_t s_mx[kAqThreads / 32];
  uint32_t m = warp_max_u32(max(mx & 0xffffu, mx >> 16));
  if ((threadIdx.x & 31) == 0) s_mx[threadIdx.x >> 5] = m;
  __syncthreads();
  m = 0;
#pragma unroll
  for (int w = 0; w < kAqThreads / 32; ++w) m = max(m, s_mx[w]);
  if (m >= kBf16InfBits && threadIdx.x == 0 && err_flag) atomicOr(err_flag, SBN_FLAG_X_NONFINITE);
  return fmaxf(__uint_as_float(m << 16), 1e-5f);
}

template <int R>
__global__ void __launch_bounds__(kAqThreads)
    k_act_quant_reg(const uint4 *__restrict__ X, int64_t nv, int8_t *__restrict__ Xq,
                    float *__restrict__ absmax, int32_t *err_flag) {
  ptx::grid_dep_launch();
  ptx::grid_dep_wait();
  const int64_t t = blockIdx.x;
  const uint4 *row = X + t * nv;
  uint4 v[R];
  uint32_t mx = 0;
#pragma unroll
  for (int r = 0; r < R; ++r) {
    int64_t i = threadIdx.x + (int64_t)r * kAqThreads;
    v[r] = i < nv ? __ldg(row + i) : make_uint4(0u, 0u, 0u, 0u);
    mx = vec8_absmax_bits(v[r], mx);
  }
  const float s = block_scale(mx, err_flag);
  const float inv = __frcp_rn(s);
  if (threadIdx.x == 0) absmax[t] = s;
  uint2 *qrow = reinterpret_cast<uint2 *>(Xq + t * nv * 8);
#pragma unroll
  for (int r = 0; r < R; ++r) {
    int64_t i = threadIdx.x + (int64_t)r * kAqThreads;
    if (i < nv) qrow[i] = quant_vec8(v[r], s, inv);
  }
}

__global__ void __launch_bounds__(kAqThreads)
    k_act_quant_loop(const uint4 *__restrict__ X, int64_t nv, int8_t *__restrict__ Xq,
                     float *__restrict__ absmax, int32_t *err_flag) {
  ptx::grid_dep_launch();
  ptx::grid_dep_wait();
  const int64_t t = blockIdx.x;
  const uint4 *row = X + t * nv;
  uint32_t mx = 0;
  for (int64_t i = threadIdx.x; i < nv; i += kAqThreads) mx = vec8_absmax_bits(__ldg(row + i), mx);
  const float s = block_scale(mx, err_flag);
  const float inv = __frcp_rn(s);
  if (threadIdx.x == 0) absmax[t] = s;
  uint2 *qrow = reinterpret_cast<uint2 *>(Xq + t * nv * 8);
  for (int64_t i = threadIdx.x; i < nv; i += kAqThreads) qrow[i] = quant_vec8(__ldg(row + i), s, inv);
}

// One warp per token for rows of up to 32 * 8 * R inputs: the whole row stays in the
// lane's registers (R 16-byte words each, all requested at once), the max is a shuffle
// reduction, and no CTA barrier is involved.
template <int R>
__global__ void __launch_bounds__(kAqThreads)
    k_act_quant_warp(const uint4 *__restrict__ X, int64_t tokens, int64_t nv,
                     int8_t *__restrict__ Xq, float *__restrict__ absmax, int32_t *err_flag) {
  ptx::grid_dep_launch();
  ptx::grid_dep_wait();
  const int lane = threadIdx.x & 31;
  const int64_t t = (int64_t)blockIdx.x * (kAqThreads / 32) + (threadIdx.x >> 5);
  if (t >= tokens) return;  // whole warps leave together
  const uint4 *row = X + t * nv;
  uint4 v[R];
  uint32_t mx = 0;
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int64_t i = lane + 32 * r;
    v[r] = i < nv ? __ldg(row + i) : make_uint4(0u, 0u, 0u, 0u);
  }
#pragma unroll
  for (int r = 0; r < R; ++r) mx = vec8_absmax_bits(v[r], mx);
  const uint32_t m = warp_max_u32(max(mx & 0xffffu, mx >> 16));
  if (m >= kBf16InfBits && lane == 0 && err_flag) atomicOr(err_flag, SBN_FLAG_X_NONFINITE);
  const float s = fmaxf(__uint_as_float(m << 16), 1e-5f);
  const float inv = __frcp_rn(s);
  if (lane == 0) absmax[t] = s;
  uint2 *qrow = reinterpret_cast<uint2 *>(Xq + t * nv * 8);
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int64_t i = lane + 32 * r;
    if (i < nv) qrow[i] = quant_vec8(v[r], s, inv);
  }
}

// Group quantisation: one CTA per (token t, group j) of G blocks along K; s is stored
// group-major, s[j * tokens + t], so that each group's scales are contiguous.  R > 0 keeps the
// block in registers (blocks of up to 8 * 256 * R inputs); R == 0 reads it twice.
template <int R>
__global__ void __launch_bounds__(kAqThreads)
    k_act_quant_gq(const uint4 *__restrict__ X, int64_t tokens, int64_t K, int G,
                   int8_t *__restrict__ Xq, float *__restrict__ absmax, int32_t *err_flag) {
  ptx::grid_dep_launch();
  ptx::grid_dep_wait();
  const int64_t t = blockIdx.x, j = blockIdx.y, kg = K / G, nv = kg / 8;
  const uint4 *row = X + (t * K + j * kg) / 8;
  uint2 *qrow = reinterpret_cast<uint2 *>(Xq + t * K + j * kg);
  if constexpr (R > 0) {
    uint4 v[R];
    uint32_t mx = 0;
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int64_t i = threadIdx.x + (int64_t)r * kAqThreads;
      v[r] = i < nv ? __ldg(row + i) : make_uint4(0u, 0u, 0u, 0u);
      mx = vec8_absmax_bits(v[r], mx);
    }
    const float s = block_scale(mx, err_flag);
    const float inv = __frcp_rn(s);
    if (threadIdx.x == 0) absmax[j * tokens + t] = s;
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int64_t i = threadIdx.x + (int64_t)r * kAqThreads;
      if (i < nv) qrow[i] = quant_vec8(v[r], s, inv);
    }
  } else {
    uint32_t mx = 0;
    for (int64_t i = threadIdx.x; i < nv; i += kAqThreads) mx = vec8_absmax_bits(__ldg(row + i), mx);
    const float s = block_scale(mx, err_flag);
    const float inv = __frcp_rn(s);
    if (threadIdx.x == 0) absmax[j * tokens + t] = s;
    for (int64_t i = threadIdx.x; i < nv; i += kAqThreads) qrow[i] = quant_vec8(__ldg(row + i), s, inv);
  }
}

sbn_status launch_act_quant_gq(const void *X, int64_t tokens, int64_t in, int G, int8_t *Xq,
                               float *absmax, int32_t *err_flag, cudaStream_t st) {
  const int64_t nv = in / G / 8;
  const uint4 *X4 = reinterpret_cast<const uint4 *>(X);
  const dim3 grid((unsigned)tokens, (unsigned)G), block(kAqThreads);
  if (nv <= 2 * kAqThreads)
    return launch_pdl(k_act_quant_gq<2>, grid, block, 0, st, X4, tokens, in, G, Xq, absmax, err_flag);
  if (nv <= 8 * kAqThreads)
    return launch_pdl(k_act_quant_gq<8>, grid, block, 0, st, X4, tokens, in, G, Xq, absmax, err_flag);
  return launch_pdl(k_act_quant_gq<0>, grid, block, 0, st, X4, tokens, in, G, Xq, absmax, err_flag);
}

// Grouped form: one CTA per (layer, token) row of a group plan.  R > 0 keeps the row in
// registers (rows of up to 8 * 256 * R inputs); R == 0 reads it twice.
template <int R>
__global__ void __launch_bounds__(kAqThreads)
    k_act_quant_group(const uint8_t *__restrict__ plan, int32_t *err_flag) {
  ptx::grid_dep_launch();
  ptx::grid_dep_wait();
  const GroupHeader &hd = *reinterpret_cast<const GroupHeader *>(plan);
  const GroupRow rw = reinterpret_cast<const GroupRow *>(plan + hd.off_rows)[blockIdx.x];
  const GroupProb &p = reinterpret_cast<const GroupProb *>(plan + hd.off_probs)[rw.prob];
  const int64_t nv = p.K / 8;
  // rows ldx elements apart (a multiple of 16): K, or more for a K slice of a wider row
  const uint4 *row = reinterpret_cast<const uint4 *>(p.X) + (int64_t)rw.token * (p.ldx / 8);
  uint2 *qrow = reinterpret_cast<uint2 *>(p.Xq + (int64_t)rw.token * p.ldx);
  if constexpr (R > 0) {
    uint4 v[R];
    uint32_t mx = 0;
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int64_t i = threadIdx.x + (int64_t)r * kAqThreads;
      v[r] = i < nv ? __ldg(row + i) : make_uint4(0u, 0u, 0u, 0u);
      mx = vec8_absmax_bits(v[r], mx);
    }
    const float s = block_scale(mx, err_flag);
    const float inv = __frcp_rn(s);
    if (threadIdx.x == 0) p.absmax[rw.token] = s;
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int64_t i = threadIdx.x + (int64_t)r * kAqThreads;
      if (i < nv) qrow[i] = quant_vec8(v[r], s, inv);
    }
  } else {
    uint32_t mx = 0;
    for (int64_t i = threadIdx.x; i < nv; i += kAqThreads) mx = vec8_absmax_bits(__ldg(row + i), mx);
    const float s = block_scale(mx, err_flag);
    const float inv = __frcp_rn(s);
    if (threadIdx.x == 0) p.absmax[rw.token] = s;
    for (int64_t i = threadIdx.x; i < nv; i += kAqThreads) qrow[i] = quant_vec8(__ldg(row + i), s, inv);
  }
}

sbn_status launch_act_quant_group(const void *plan_host, const void *plan_dev, int32_t *err_flag,
                                  cudaStream_t st) {
  const GroupHeader *hd = static_cast<const GroupHeader *>(plan_host);
  if (hd->nrows == 0) return SBN_OK;
  const uint8_t *P = static_cast<const uint8_t *>(plan_dev);
  const dim3 grid((unsigned)hd->nrows), block(kAqThreads);
  // When no row has more than 4096 inputs, rows stay in registers.  Otherwise every row is
  // read twice (the second read from L2): holding 8 words per thread keeps 4 CTAs per SM
  // resident, the two-pass form about twice as many, and with one short row per CTA the
  // number of rows in flight decides the time (the 160-layer, 16-token stack: 14.7 us with
  // 8 words per thread, 13.5 us in two passes).
  if (hd->max_nv <= 2 * kAqThreads)
    return launch_pdl(k_act_quant_group<2>, grid, block, 0, st, P, err_flag);
  return launch_pdl(k_act_quant_group<0>, grid, block, 0, st, P, err_flag);
}

sbn_status launch_act_quant(const void *X, int64_t tokens, int64_t in, int8_t *Xq,
                            float *absmax, int32_t *err_flag, cudaStream_t st) {
  const int64_t nv = in / 8;
  const uint4 *X4 = reinterpret_cast<const uint4 *>(X);
  const dim3 block(kAqThreads);
  if (tokens > 16 && nv <= 32 * 4) {
    // many tokens with rows of up to 1024 inputs: one warp each (a CTA-wide reduction per
    // token costs more than such a row).  Longer rows take a CTA per token: one warp per
    // token leaves each warp a long serial run of codes and the SMs mostly idle (2048 x 4096:
    // 11.4 us with a warp per token, 6.8 us with a CTA per token).
    const dim3 wgrid((unsigned)((tokens + kAqThreads / 32 - 1) / (kAqThreads / 32)));
    return launch_pdl(k_act_quant_warp<4>, wgrid, block, 0, st, X4, tokens, nv, Xq, absmax,
                      err_flag);
  }
  const dim3 grid((unsigned)tokens);
  if (nv <= 2 * kAqThreads)
    return launch_pdl(k_act_quant_reg<2>, grid, block, 0, st, X4, nv, Xq, absmax, err_flag);
  if (nv <= 8 * kAqThreads)
    return launch_pdl(k_act_quant_reg<8>, grid, block, 0, st, X4, nv, Xq, absmax, err_flag);
  return launch_pdl(k_act_quant_loop, grid, block, 0, st, X4, nv, Xq, absmax, err_flag);
}

}  // namespace sbn
