// Backward of the Sparse-BitLinear layer under the dual straight-through estimator
// (Sparse-BitNet summaries, section 2: the quantiser and the mask are both passed straight
// through; the quantiser's estimator is the identity inside its clip range, the mask's
// sends a dense gradient to every master weight, pruned ones included):
//   dX[t, k] = g * sum_o dY[t, o] * Ws[o, k]                       (the forward's W_eff = g Ws)
//   dW[o, k] = pass[o, k] * sum_t dY[t, o] * (s_t / 127) * Xq[t, k] (the forward's X_eff)
//   pass[o, k] = (fl32(|W[o, k]| / g) <= 1)      (clip(W / g, -1, 1) has slope 1 there)
// Both are dense contractions and run on the tensor cores as bf16 x bf16 -> fp32 GEMMs
// (tcgen05.mma kind::f16) with products that are exact:
//   dX: A = dY (bf16 as given), B = Ws^T expanded to bf16 {-1, 0, 1} (k_bwd_expand_wt);
//   dW: the per-token factor c_t = fp32(s_t / 127) is folded into dY and the fp32 product is
//       split into two bf16 terms hi + lo (|dY c - hi - lo| <= 2^-16 |dY c|); A = [hi | lo]^T
//       and B = [Xq | Xq]^T (int8 values are exact in bf16) side by side along the reduction
//       (k_bwd_scale_dy, k_bwd_transpose_xq), so one GEMM over 2 T_pad sums both terms.
// The only other rounding is the fp32 accumulation of the tensor cores.
//
// k_gemm_bf16<EPI>: D[M x N] = A[M x R] . B[N x R]^T, A and B bf16 with the reduction R
// contiguous, 128 x 256 tiles, persistent over tiles, 4-stage TMA ring (128-byte swizzle,
// 64 bf16 per row and stage), two TMEM accumulators (columns 0 and 256) so that the
// epilogue of one tile overlaps the MMAs of the next.  192 threads: warp 0 TMA producer,
// warp 1 TMEM allocation + MMA thread, warps 2-5 epilogue (warp w reads TMEM lanes
// 32 (w mod 4) .. + 31).  Every wait is bounded and raises SBN_FLAG_TIMEOUT.
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

namespace sbn {

namespace {

constexpr long long kBwWaitCycles = 1ll << 31;
constexpr int kBwThreads = 192;
constexpr int kBwBM = 128, kBwBN = 256, kBwBK = 64;  // BK in bf16 elements (128 bytes)
constexpr int kBwStages = 4;
constexpr int kBwABytes = kBwBM * kBwBK * 2;  // 16 KB
constexpr int kBwBBytes = kBwBN * kBwBK * 2;  // 32 KB
constexpr int kBwStageBytes = kBwABytes + kBwBBytes;
constexpr size_t kBwSmem = 1024 + (size_t)kBwStages * kBwStageBytes + (2 * kBwStages + 5) * 8 + 64;
static_assert(kBwSmem <= 227 * 1024, "shared memory budget");

// Instruction descriptor: kind::f16, D = f32, A and B bf16, both K-major, M x N.
constexpr uint32_t idesc_bf16(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ bool bw_wait(uint64_t *bar, uint32_t parity, volatile int *abort) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    for (int i = 0; i < 64; ++i)
      if (ptx::mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if (clock64() - t0 > kBwWaitCycles) {
      *abort = 1;
      return false;
    }
  }
}

__device__ __forceinline__ bool bw_drain(uint64_t *bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!ptx::mbar_try_wait(bar, parity))
    if (clock64() - t0 > kBwWaitCycles) return false;
  return true;
}

__device__ __forceinline__ bool bw_bar_any(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.or.pred p, 1, 128, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred)
      : "memory");
  return r != 0;
}

// The smallest bf16 magnitude m (bits 0 .. 0x7f80) for which fl32(m / g) <= 1 is false;
// the clip-range test is then (|W| bits) < thr.  fl32(m / g) is monotone in m, so the set of
// passing magnitudes is a prefix (empty when g is 0 or NaN, as 0/0 and m/0 fail the test).
__device__ __forceinline__ uint32_t pass_threshold(float g) {
  uint32_t lo = 0, hi = 0x7f80u;  // answer in [lo, hi]
  while (lo < hi) {
    const uint32_t mid = (lo + hi) >> 1;
    const bool pass = __fdiv_rn(__uint_as_float(mid << 16), g) <= 1.0f;
    if (pass)
      lo = mid + 1;
    else
      hi = mid;
  }
  return lo;
}

struct EpiArgs {
  const float *gamma_eff;        // g
  const uint16_t *W;             // EPI 1: bf16 masters [M][N]
};

template <int EPI>
__global__ void __launch_bounds__(kBwThreads, 1)
    k_gemm_bf16(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                int64_t M, int64_t N, int64_t R, float *__restrict__ out, EpiArgs e,
                int32_t *err_flag) {
  constexpr int S = kBwStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + S * kBwStageBytes);
  uint64_t *empty = full + S;
  uint64_t *acc_full = empty + S;      // [2]
  uint64_t *acc_empty = acc_full + 2;  // [2]
  uint64_t *mma_done = acc_empty + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_done + 1);
  volatile int *s_abort = reinterpret_cast<volatile int *>(tmem_slot + 2);
  volatile uint32_t *s_thr = reinterpret_cast<volatile uint32_t *>(tmem_slot + 4);

  ptx::grid_dep_launch();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t n_m = (M + kBwBM - 1) / kBwBM, n_n = (N + kBwBN - 1) / kBwBN;
  const int64_t ntiles = n_m * n_n;
  const int nkb = (int)((R + kBwBK - 1) / kBwBK);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(&acc_full[b], 1);
      ptx::mbar_init(&acc_empty[b], 4);
    }
    ptx::mbar_init(mma_done, 1);
    *s_abort = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, 512);
    ptx::tmem_relinquish();
  }
  ptx::grid_dep_wait();
  if (EPI == 1 && threadIdx.x == 64) *s_thr = pass_threshold(__ldg(e.gamma_eff));
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      ptx::prefetch_tmap(&tmap_a);
      ptx::prefetch_tmap(&tmap_b);
      int64_t kg = 0, issued = 0;
      for (int64_t tile = blockIdx.x; tile < ntiles && !*s_abort; tile += gridDim.x) {
        const int32_t m0 = (int32_t)((tile % n_m) * kBwBM), n0 = (int32_t)((tile / n_m) * kBwBN);
        bool ok = true;
        for (int kb = 0; kb < nkb; ++kb, ++kg) {
          const int s = (int)(kg % S);
          const uint32_t ph = (uint32_t)(kg / S) & 1u;
          if (kg >= S && !bw_wait(&empty[s], ph ^ 1u, s_abort)) {
            ok = false;
            break;
          }
          uint8_t *st = smem + s * kBwStageBytes;
          ptx::mbar_arrive_expect_tx(&full[s], (uint32_t)kBwStageBytes);
          const int32_t x = kb * kBwBK * 2;  // the maps are byte-typed: x in bytes
          ptx::tma_load_2d(st, &tmap_a, &full[s], x, m0);
          ptx::tma_load_2d(st + kBwABytes, &tmap_b, &full[s], x, n0);
          ptx::tma_load_2d(st + kBwABytes + kBwBBytes / 2, &tmap_b, &full[s], x, n0 + kBwBN / 2);
          issued = kg + 1;
        }
        if (!ok) break;
      }
      for (int64_t q = issued - S < 0 ? 0 : issued - S; q < issued; ++q)
        if (!bw_drain(&full[q % S], (uint32_t)(q / S) & 1u)) *s_abort = 1;
    }
  } else if (warp == 1) {
    // ---------------- MMA thread ----------------
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(kBwBM, kBwBN);
      int64_t kg = 0;
      int i = 0;
      for (int64_t tile = blockIdx.x; tile < ntiles && !*s_abort; tile += gridDim.x, ++i) {
        const int buf = i & 1;
        if (i >= 2 && !bw_wait(&acc_empty[buf], ((uint32_t)(i >> 1) & 1u) ^ 1u, s_abort)) break;
        ptx::tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(buf * 256);
        bool ok = true;
        for (int kb = 0; kb < nkb; ++kb, ++kg) {
          const int s = (int)(kg % S);
          if (!bw_wait(&full[s], (uint32_t)(kg / S) & 1u, s_abort)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t a_addr = ptx::smem_u32(smem + s * kBwStageBytes);
          const uint32_t b_addr = a_addr + kBwABytes;
#pragma unroll
          for (int k = 0; k < kBwBK / 16; ++k)  // 16 bf16 (32 bytes) of K per MMA
            mma_bf16(d, ptx::smem_desc_sw128(a_addr + 32 * k), ptx::smem_desc_sw128(b_addr + 32 * k),
                     idesc, (kb | k) != 0);
          ptx::mma_commit(&empty[s]);
        }
        if (!ok) break;
        ptx::mma_commit(&acc_full[buf]);
      }
      ptx::mma_commit(mma_done);
      if (!bw_drain(mma_done, 0)) *s_abort = 1;
    }
  } else {
    // ---------------- epilogue (warps 2-5) ----------------
    const int q = warp & 3;
    const float g = __ldg(e.gamma_eff);
    const uint32_t thr = EPI == 1 ? *s_thr : 0u;
    bool failed = false;
    int i = 0;
    for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++i) {
      const int buf = i & 1;
      if (bw_bar_any(failed)) break;
      const int64_t m = (tile % n_m) * kBwBM + q * 32 + lane;
      const int64_t n0 = (tile / n_m) * kBwBN;
      failed = !__all_sync(0xffffffffu, !*s_abort && bw_wait(&acc_full[buf],
                                                              (uint32_t)(i >> 1) & 1u, s_abort));
      ptx::tc_fence_after();
      if (!failed) {
        const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * 256);
#pragma unroll 1
        for (int cb = 0; cb < kBwBN; cb += 32) {
          uint32_t v[32];
          ptx::tmem_ld_32(trow + cb, v);
          ptx::tmem_ld_wait();
          if (m >= M || n0 + cb >= N) continue;  // N is a multiple of 64: chunks are whole
          float4 *dst = reinterpret_cast<float4 *>(out + m * N + n0 + cb);
          if constexpr (EPI == 0) {
#pragma unroll
            for (int j = 0; j < 32; j += 4)
              dst[j / 4] = make_float4(__fmul_rn(__uint_as_float(v[j]), g),
                                       __fmul_rn(__uint_as_float(v[j + 1]), g),
                                       __fmul_rn(__uint_as_float(v[j + 2]), g),
                                       __fmul_rn(__uint_as_float(v[j + 3]), g));
          } else {
            const uint4 *wp = reinterpret_cast<const uint4 *>(e.W + m * N + n0 + cb);
#pragma unroll
            for (int j = 0; j < 32; j += 8) {
              const uint4 w8 = __ldg(wp + j / 8);
              const uint32_t wv[4] = {w8.x, w8.y, w8.z, w8.w};
              float o8[8];
#pragma unroll
              for (int h = 0; h < 4; ++h) {
                const bool p0 = (wv[h] & 0x7fffu) < thr, p1 = ((wv[h] >> 16) & 0x7fffu) < thr;
                o8[2 * h] = p0 ? __uint_as_float(v[j + 2 * h]) : 0.0f;
                o8[2 * h + 1] = p1 ? __uint_as_float(v[j + 2 * h + 1]) : 0.0f;
              }
              dst[j / 4] = make_float4(o8[0], o8[1], o8[2], o8[3]);
              dst[j / 4 + 1] = make_float4(o8[4], o8[5], o8[6], o8[7]);
            }
          }
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&acc_empty[buf]);
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && *s_abort && err_flag) atomicOr(err_flag, SBN_FLAG_TIMEOUT);
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 512);
  }
}

// ---- operand preparation --------------------------------------------------------------

__device__ __forceinline__ uint16_t bf16_of_code(uint32_t c) {
  // 2-bit code 00 -> 0, 01 -> +1, 11 -> -1 as bf16 bits
  return c == 1u ? (uint16_t)0x3f80u : c == 3u ? (uint16_t)0xbf80u : (uint16_t)0u;
}

// The operands of the two GEMMs are transposes of the inputs (Ws^T, dY'^T, Xq^T).  Each is
// built in tiles through shared memory: 8-byte loads along the rows of the input and 8-byte
// stores along the rows of the output, so both sides move whole 128-byte lines.

// 16 weights of row o, inputs 16c .. 16c + 15, as bf16 {-1, 0, +1} from the packed planes,
// two per word: v[j] holds inputs 16c + 2j (low half) and 16c + 2j + 1 (high half).
__device__ __forceinline__ void decode_chunk(const uint8_t *__restrict__ codes,
                                             const uint8_t *__restrict__ meta, int64_t o,
                                             int64_t c, int64_t ldc, int64_t ldm, int compact,
                                             uint32_t (&v)[8]) {
  if (!compact) {
    // stored element e = k: word e / 16, byte e % 4, bits 6 - 2j .. 7 - 2j, j = (e % 16) / 4
    const uint32_t w = __ldg(reinterpret_cast<const uint32_t *>(codes + o * ldc) + c);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e0 = 2 * j, e1 = 2 * j + 1;
      v[j] = (uint32_t)bf16_of_code((w >> (8 * (e0 % 4) + 6 - 2 * (e0 / 4))) & 3u) |
             ((uint32_t)bf16_of_code((w >> (8 * (e1 % 4) + 6 - 2 * (e1 / 4))) & 3u) << 16);
    }
  } else {
    // 2:4: the 8 kept codes of these 4 groups are stored elements 8c .. 8c + 7 (word c / 2,
    // half c % 2); group g's pair of positions is the nibble i0 | i1 << 2 of meta.  The
    // group's four bf16 are one 64-bit word: code 0 at position i0, code 1 at i1 (i0 wins
    // if the two are equal)
    const uint32_t w = __ldg(reinterpret_cast<const uint32_t *>(codes + o * ldc) + c / 2);
    const uint32_t mw = __ldg(reinterpret_cast<const uint16_t *>(meta + o * ldm) + c);
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      const uint32_t nib = (mw >> (4 * g)) & 15u;
      const uint32_t i0 = nib & 3u, i1 = nib >> 2;
      const int se0 = 8 * (int)(c % 2) + 2 * g;  // stored elements se0, se0 + 1 of the word
      const uint64_t c0 = bf16_of_code((w >> (8 * (se0 % 4) + 6 - 2 * (se0 / 4))) & 3u);
      const uint64_t c1 = bf16_of_code((w >> (8 * ((se0 + 1) % 4) + 6 - 2 * ((se0 + 1) / 4))) & 3u);
      const uint64_t q = (c0 << (16 * i0)) | (i1 != i0 ? c1 << (16 * i1) : 0ull);
      v[2 * g] = (uint32_t)q;
      v[2 * g + 1] = (uint32_t)(q >> 32);
    }
  }
}

// Ws^T [K][ldw] bf16 from the packed planes, in tiles of 64 rows o x 128 inputs: thread
// (row pair p, chunk q) decodes the tile's 16-input chunk q of rows 2p and 2p + 1 (8
// threads read a row's 32 contiguous bytes of codes), writes each input's two bf16 as one
// 32-bit word into the tile, and each of the tile's 128 input rows is stored as 64
// contiguous bf16.  K is a multiple of 64; O of 8.
__global__ void __launch_bounds__(256)
    k_bwd_expand_wt(const uint8_t *__restrict__ codes, const uint8_t *__restrict__ meta,
                    int64_t O, int64_t K, int64_t ldc, int64_t ldm, int compact,
                    uint16_t *__restrict__ wt, int64_t ldw) {
  __shared__ __align__(16) uint32_t tile[128][32 + 2];  // [k][o / 2]; rows 136 bytes apart
  ptx::grid_dep_launch();
  ptx::grid_dep_wait();
  const int64_t o0 = (int64_t)blockIdx.x * 64, k0 = (int64_t)blockIdx.y * 128;
  const int p = threadIdx.x >> 3, q = threadIdx.x & 7;
  const int64_t o = o0 + 2 * p, c = k0 / 16 + q;
  uint32_t va[8], vb[8];
  const bool cin = c < K / 16;
  if (cin && o < O) {
    decode_chunk(codes, meta, o, c, ldc, ldm, compact, va);
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) va[j] = 0;
  }
  if (cin && o + 1 < O) {
    decode_chunk(codes, meta, o + 1, c, ldc, ldm, compact, vb);
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) vb[j] = 0;
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    // inputs 16q + 2j (low halves) and 16q + 2j + 1 (high halves) of rows o, o + 1
    tile[16 * q + 2 * j][p] = (va[j] & 0xffffu) | (vb[j] << 16);
    tile[16 * q + 2 * j + 1][p] = (va[j] >> 16) | (vb[j] & 0xffff0000u);
  }
  __syncthreads();
  const int oc = 2 * (threadIdx.x & 15);  // word column: outputs 2 oc .. 2 oc + 3
#pragma unroll
  for (int pass = 0; pass < 8; ++pass) {
    const int kk = pass * 16 + (threadIdx.x >> 4);
    const int64_t k = k0 + kk, oo = o0 + 2 * oc;
    if (k < K && oo < O)
      *reinterpret_cast<uint2 *>(wt + k * ldw + oo) =
          *reinterpret_cast<const uint2 *>(&tile[kk][oc]);
  }
}

// dY'^T as two bf16 terms side by side: out[o][t] = hi, out[o][Tp + t] = lo, where
// dY' = fp32(dY[t][o] * fp32(s_t / 127)), hi = bf16(dY'), lo = bf16(dY' - hi); zero for
// t >= T.  Tiles of 64 tokens x 64 outputs: 4 bf16 per thread loaded along o, the scale of
// each token computed once per tile, 4 tokens per thread stored along t (O is a multiple of
// 8, Tp of 32).
__global__ void __launch_bounds__(256)
    k_bwd_scale_dy(const uint16_t *__restrict__ dY, const float *__restrict__ absmax, int64_t T,
                   int64_t O, int64_t Tp, uint16_t *__restrict__ out) {
  __shared__ float tile[64][64 + 1];  // [t][o]
  __shared__ float s_c[64];
  ptx::grid_dep_launch();
  ptx::grid_dep_wait();
  const int64_t o0 = (int64_t)blockIdx.x * 64, t0 = (int64_t)blockIdx.y * 64;
  if (threadIdx.x < 64) {
    const int64_t t = t0 + threadIdx.x;
    s_c[threadIdx.x] = t < T ? __fdiv_rn(__ldg(absmax + t), 127.0f) : 0.0f;
  }
  __syncthreads();
  const int c4 = 4 * (threadIdx.x & 15);
#pragma unroll
  for (int pass = 0; pass < 4; ++pass) {
    const int tt = pass * 16 + (threadIdx.x >> 4);
    const int64_t t = t0 + tt, o = o0 + c4;
    uint2 w = make_uint2(0u, 0u);
    if (t < T && o < O) w = __ldg(reinterpret_cast<const uint2 *>(dY + t * O + o));
    const float c = s_c[tt];
    tile[tt][c4 + 0] = __fmul_rn(__uint_as_float(w.x << 16), c);
    tile[tt][c4 + 1] = __fmul_rn(__uint_as_float(w.x & 0xffff0000u), c);
    tile[tt][c4 + 2] = __fmul_rn(__uint_as_float(w.y << 16), c);
    tile[tt][c4 + 3] = __fmul_rn(__uint_as_float(w.y & 0xffff0000u), c);
  }
  __syncthreads();
#pragma unroll
  for (int pass = 0; pass < 4; ++pass) {
    const int oo = pass * 16 + (threadIdx.x >> 4);
    const int64_t o = o0 + oo, t = t0 + c4;
    if (o >= O || t >= Tp) continue;
    uint32_t hi[2], lo[2];
#pragma unroll
    for (int p = 0; p < 2; ++p) {
      uint32_t h2 = 0, l2 = 0;
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const float v = tile[c4 + 2 * p + u][oo];
        const __nv_bfloat16 h = __float2bfloat16_rn(v);
        const __nv_bfloat16 l = __float2bfloat16_rn(__fsub_rn(v, __bfloat162float(h)));
        h2 |= (uint32_t)__bfloat16_as_ushort(h) << (16 * u);
        l2 |= (uint32_t)__bfloat16_as_ushort(l) << (16 * u);
      }
      hi[p] = h2;
      lo[p] = l2;
    }
    *reinterpret_cast<uint2 *>(out + o * (2 * Tp) + t) = make_uint2(hi[0], hi[1]);
    *reinterpret_cast<uint2 *>(out + o * (2 * Tp) + Tp + t) = make_uint2(lo[0], lo[1]);
  }
}

// Xq^T twice side by side as bf16: out[k][t] = out[k][Tp + t] = Xq[t][k]; zero for t >= T.
// Tiles of 64 tokens x 64 inputs: 4 int8 per thread loaded along k, 4 tokens per thread
// stored along t (K is a multiple of 64, Tp of 32).
__global__ void __launch_bounds__(256)
    k_bwd_transpose_xq(const int8_t *__restrict__ Xq, int64_t T, int64_t K, int64_t Tp,
                       uint16_t *__restrict__ out) {
  __shared__ float tile[64][64 + 1];  // [t][k]
  ptx::grid_dep_launch();
  ptx::grid_dep_wait();
  const int64_t k0 = (int64_t)blockIdx.x * 64, t0 = (int64_t)blockIdx.y * 64;
  const int c4 = 4 * (threadIdx.x & 15);
#pragma unroll
  for (int pass = 0; pass < 4; ++pass) {
    const int tt = pass * 16 + (threadIdx.x >> 4);
    const int64_t t = t0 + tt, k = k0 + c4;
    uint32_t w = 0;
    if (t < T && k < K) w = __ldg(reinterpret_cast<const uint32_t *>(Xq + t * K + k));
#pragma unroll
    for (int u = 0; u < 4; ++u) tile[tt][c4 + u] = (float)(int8_t)(w >> (8 * u));
  }
  __syncthreads();
#pragma unroll
  for (int pass = 0; pass < 4; ++pass) {
    const int kk = pass * 16 + (threadIdx.x >> 4);
    const int64_t k = k0 + kk, t = t0 + c4;
    if (k >= K || t >= Tp) continue;
    uint32_t b[2];
#pragma unroll
    for (int p = 0; p < 2; ++p)
      b[p] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(tile[c4 + 2 * p][kk])) |
             ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(tile[c4 + 2 * p + 1][kk])) << 16);
    *reinterpret_cast<uint2 *>(out + k * (2 * Tp) + t) = make_uint2(b[0], b[1]);
    *reinterpret_cast<uint2 *>(out + k * (2 * Tp) + Tp + t) = make_uint2(b[0], b[1]);
  }
}

bool encode_bf16(CUtensorMap *map, const void *base, int64_t cols, int64_t rows, int64_t ld_elems,
                 uint32_t box_rows) {
  // bf16 [rows][cols] with row stride ld_elems, box 64 x box_rows, 128-byte swizzle; the
  // maps are byte-typed (uint8) with twice the columns, which describes the same boxes
  return encode_u8(map, base, 2 * cols, rows, 2 * ld_elems, 2 * kBwBK, box_rows,
                   CU_TENSOR_MAP_SWIZZLE_128B);
}

template <int EPI>
sbn_status launch_gemm_bf16(const CUtensorMap &ta, const CUtensorMap &tb, int64_t M, int64_t N,
                            int64_t R, float *out, EpiArgs e, int32_t *err_flag,
                            cudaStream_t st) {
  auto kern = k_gemm_bf16<EPI>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kBwSmem) !=
      cudaSuccess)
    return SBN_ERR_CUDA;
  const int64_t tiles = ((M + kBwBM - 1) / kBwBM) * ((N + kBwBN - 1) / kBwBN);
  int64_t grid = num_sms();
  if (grid > tiles) grid = tiles;
  return launch_pdl(kern, dim3((unsigned)grid), dim3(kBwThreads), kBwSmem, st, ta, tb, M, N, R,
                    out, e, err_flag);
}

}  // namespace

int64_t backward_tokens_padded(int64_t tokens) { return (tokens + 31) / 32 * 32; }

int64_t backward_workspace_bytes(int64_t tokens, int64_t out, int64_t in) {
  const int64_t ldw = (out + 7) / 8 * 8, Tp = backward_tokens_padded(tokens);
  const int64_t wt = in * ldw * 2, dy = out * 2 * Tp * 2, xq = in * 2 * Tp * 2;
  return (wt + 255) / 256 * 256 + (dy + 255) / 256 * 256 + (xq + 255) / 256 * 256;
}

sbn_status launch_backward(const void *dY, const int8_t *Xq, const float *absmax,
                           const uint8_t *codes, const uint8_t *meta, const void *W,
                           const float *gamma_eff, int64_t T, int64_t O, int64_t K, int n, int m,
                           int64_t ldc, int64_t ldm, float *dX, float *dW, void *workspace,
                           int32_t *err_flag, cudaStream_t st) {
  const int64_t ldw = (O + 7) / 8 * 8, Tp = backward_tokens_padded(T);
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  uint16_t *wt = reinterpret_cast<uint16_t *>(ws);
  uint16_t *dyt = reinterpret_cast<uint16_t *>(ws + (K * ldw * 2 + 255) / 256 * 256);
  uint16_t *xqt = reinterpret_cast<uint16_t *>(reinterpret_cast<uint8_t *>(dyt) +
                                               (O * 2 * Tp * 2 + 255) / 256 * 256);
  EpiArgs e{gamma_eff, static_cast<const uint16_t *>(W)};
  sbn_status s = SBN_OK;
  if (dX) {
    s = launch_pdl(k_bwd_expand_wt, dim3((unsigned)((O + 63) / 64), (unsigned)((K + 127) / 128)),
                   dim3(256), 0, st, codes, meta, O, K, ldc, ldm, (int)(n == 2 && m == 4), wt, ldw);
    if (s != SBN_OK) return s;
    CUtensorMap ta, tb;
    if (!encode_bf16(&ta, dY, O, T, O, kBwBM) || !encode_bf16(&tb, wt, O, K, ldw, kBwBN / 2))
      return SBN_ERR_CUDA;
    s = launch_gemm_bf16<0>(ta, tb, T, K, O, dX, e, err_flag, st);
    if (s != SBN_OK) return s;
  }
  if (dW) {
    s = launch_pdl(k_bwd_scale_dy, dim3((unsigned)((O + 63) / 64), (unsigned)((Tp + 63) / 64)),
                   dim3(256), 0, st, static_cast<const uint16_t *>(dY), absmax, T, O, Tp, dyt);
    if (s != SBN_OK) return s;
    s = launch_pdl(k_bwd_transpose_xq, dim3((unsigned)((K + 63) / 64), (unsigned)((Tp + 63) / 64)),
                   dim3(256), 0, st, Xq, T, K, Tp, xqt);
    if (s != SBN_OK) return s;
    CUtensorMap ta, tb;
    if (!encode_bf16(&ta, dyt, 2 * Tp, O, 2 * Tp, kBwBM) ||
        !encode_bf16(&tb, xqt, 2 * Tp, K, 2 * Tp, kBwBN / 2))
      return SBN_ERR_CUDA;
    s = launch_gemm_bf16<1>(ta, tb, O, K, 2 * Tp, dW, e, err_flag, st);
  }
  return s;
}

}  // namespace sbn
