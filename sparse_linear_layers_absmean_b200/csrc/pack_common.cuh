// The absmean scale, shared by the quant/mask/pack kernels (pack.cu, pack_fast.cu): the
// exact fp64 accumulation k_abs_sum uses, and the prologue with which every CTA of the
// next kernel turns k_abs_sum's per-CTA partial sums into gamma, g = gamma + eps and the
// code threshold.
#pragma once

#include "common.cuh"
#include "kernels.cuh"

namespace sbn {

// ---------------------------------------------------------------------------------------
// Exact absmean sum S = sum trunc(|W| * 2^24) with one fp64 add per weight.
// ((h << 13) & 0x0fffe000) | 0x40000000, for the 15 magnitude bits h of a bf16 value, is
// the high word of the fp64 number |W| * 2^128 (bf16 exponent e -> fp64 exponent field
// e + 1024, the seven mantissa bits after it; zero and subnormals give values below 4).
// The accumulator starts at 2^156, where the fp64 spacing is 2^104, and every add rounds
// toward zero: with acc on that grid and 0 <= v, floor(acc + v) = acc + floor(v), so each
// add contributes exactly floor(|W| * 2^128 / 2^104) = trunc(|W| * 2^24).  The low 52 bits
// of the final accumulator are the sum (below 2^52 for any one thread's share).  Exact for
// |W| < 256, the supported range.
// ---------------------------------------------------------------------------------------
constexpr double kAccBias = 9.1343852333181432e46;  // 2^156

__device__ __forceinline__ double mag_lo_x2p128(uint32_t w) {
  return __hiloint2double((int)(((w << 13) & 0x0fffe000u) | 0x40000000u), 0);
}
__device__ __forceinline__ double mag_hi_x2p128(uint32_t w) {
  return __hiloint2double((int)(((w >> 3) & 0x0fffe000u) | 0x40000000u), 0);
}
__device__ __forceinline__ unsigned long long acc_value(double acc) {
  return (unsigned long long)__double_as_longlong(acc) & ((1ull << 52) - 1);
}

// Smallest bf16 magnitude (as bits) whose ternary code is non-zero for this g.
// round_half_even(x / g) != 0  <=>  fl(x / g) > 0.5, and fl(x / g) is non-decreasing in x,
// so the set of non-zero magnitudes is an up-set over the bit patterns (positive bf16
// values are ordered like their bits).  One warp searches it 32-ary: the predicate is
// false at 0 (0/g) and true at +Inf; each round keeps the sub-interval where it switches.
// Every division is an IEEE fp32 division.
__device__ __forceinline__ uint32_t code_threshold_warp(float g, int lane) {
  uint32_t lo = 0, hi = kBf16InfBits;
  while (hi - lo > 1) {
    const uint32_t step = (hi - lo + 31) / 32;
    uint32_t cand = lo + (uint32_t)(lane + 1) * step;
    if (cand > hi) cand = hi;
    const bool p = __fdiv_rn(__uint_as_float(cand << 16), g) > 0.5f;
    const uint32_t ballot = __ballot_sync(0xffffffffu, p || cand == hi);
    const int f = __ffs(ballot) - 1;  // first candidate where the predicate holds
    const uint32_t new_hi = __shfl_sync(0xffffffffu, cand, f);
    const uint32_t new_lo = f == 0 ? lo : __shfl_sync(0xffffffffu, cand, f > 0 ? f - 1 : 0);
    hi = new_hi;
    lo = new_lo;
  }
  return hi;
}

// g = fp32(gamma + eps) with gamma = fp32(fp64(S) / (fp64(n) * 2^24)), S the exact sum of
// trunc(|W| * 2^24) over the n weights, and the code threshold for that g.  Called by all
// 32 lanes of one warp; every lane returns both.
__device__ __forceinline__ uint32_t scale_from_sum(unsigned long long S, int64_t n, float eps,
                                                   int lane, float &g) {
  const double mean = __ddiv_rn(__ull2double_rn(S), (double)n * 16777216.0);
  g = __fadd_rn(__double2float_rn(mean), eps);
  return code_threshold_warp(g, lane);
}

// Run by every thread of a CTA at the start of a quant/mask/pack kernel.  Returns the code
// threshold; CTA 0 also publishes g = fp32(gamma + eps) to *gamma_eff, where
// gamma = fp32(fp64(S) / (fp64(n) * 2^24)) and S is the exact sum of the partials.  All
// threads load the partials (a few each, in one round of loads), warp 0 finishes.
__device__ __forceinline__ uint32_t pack_prologue(const PackWorkspace *ws, int nparts,
                                                  int64_t n, float eps, float *gamma_eff) {
  __shared__ unsigned long long s_part[32];
  __shared__ uint32_t s_thr;
  unsigned long long S = 0;
#pragma unroll 4
  for (int i = threadIdx.x; i < nparts; i += blockDim.x) S += ws->part[i];
  S = warp_sum_u64(S);
  if ((threadIdx.x & 31) == 0) s_part[threadIdx.x >> 5] = S;
  __syncthreads();
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    S = lane < (int)(blockDim.x >> 5) ? s_part[lane] : 0ull;
    S = warp_sum_u64(S);
    float g;
    const uint32_t thr = scale_from_sum(S, n, eps, lane, g);
    if (lane == 0) {
      s_thr = thr;
      if (blockIdx.x == 0) *gamma_eff = g;
    }
  }
  __syncthreads();
  return s_thr;
}

}  // namespace sbn
