// Tensor-core contraction (prefill): Y[t, o] = (sum_k Xq[t,k] * Ws[o,k]) * c_t on the
// 5th-generation tensor cores (tcgen05.mma kind::i8, int32 accumulators in TMEM).
//
// Three kernels share the pipeline below: k_gemm_tc (dense codes, any N:M pattern; one
// tile per CTA), k_gemm_sp24 (2:4 on the sparse MMA; one tile per CTA, up to 128 tokens)
// and, for more tokens, k_gemm_sp24_pair (2:4, CTA pairs, persistent, double-buffered
// accumulators, the expanded weights and their metadata in TMEM).
//
// One CTA computes a 128 (outputs) x BN (tokens) tile with a multi-stage shared-memory
// pipeline over K in blocks of 128 (a stage holds one to four consecutive blocks: each
// hand-off between the roles has a fixed cost, so the narrow tiles move several blocks per
// hand-off).  Up to 32 tokens, k_gemm_sp24 may split a tile's K blocks over a cluster of
// CTAs when there are too few tiles to occupy the SMs; CTA 0 of the cluster receives the
// others' partial accumulators through distributed shared memory and stores the tile.
//   warp 4     TMA producer: per K block, the int8 activation tile (128-byte swizzle,
//              K-major) and the packed weight tile (codes, plus the 2:4 metadata) of the
//              CTA's 128 rows.
//   warps 0-3  weight expanders: thread r owns tile row r, reads its packed bytes from
//              shared memory, expands them to int8 lanes of 64 * t (one shift and one AND
//              per four weights; 2:4 codes are placed at their kept positions with a byte
//              permute) and stores them in the swizzled K-major layout the MMA reads;
//              then the epilogue.
//   warp 5     TMEM allocation and the single MMA-issuing thread.
// (k_gemm_sp24_pair has its own roles, described at its definition: two MMA-issuing
// threads, expanders writing TMEM, two producers.)
// The accumulator carries 64 * acc; the epilogue divides by 64 exactly, multiplies by
// c_t = fp32(fp32(g * s_t) / 127) and stores fp32 or bf16.
// Every mbarrier wait gives up after about a second (2^31 SM cycles) and raises
// SBN_FLAG_TIMEOUT.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

namespace sbn {

constexpr int kTcThreads = 192;
constexpr int kBM = 128;
constexpr int kBK = 128;
// Waits give up after 2^31 SM cycles (about 1 s at the 1965 MHz boost clock, 2 s at 1 GHz).
// The bound is kept with the SM's cycle counter: reading the global nanosecond timer costs
// about a tenth of a microsecond, which would sit on the critical path of every hand-off.
#ifdef SBN_TIMEOUT_TEST
// Test build only (tests/test_timeout_gpu.py): waits give up after 2^20 cycles (about half
// a millisecond), and in k_gemm_sp24 the first expander warp withholds its arrival for the
// second pipeline stage, so the MMA thread's wait on that stage runs out.
constexpr long long kWaitCycles = 1ll << 20;
#else
constexpr long long kWaitCycles = 1ll << 31;
#endif

// Bounded wait on an mbarrier phase; false on timeout.  (mbarrier.try_wait itself suspends
// the thread for a while when the phase is not yet complete.)
__device__ __forceinline__ bool wait_phase(uint64_t *bar, uint32_t parity) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    for (int i = 0; i < 64; ++i)
      if (ptx::mbar_try_wait(bar, parity)) return true;
    if (clock64() - t0 > kWaitCycles) return false;
  }
}

// Partial accumulators of a K-split tile, as CTA 0 of the cluster receives them: slot q
// holds [128 rows][BN] int32, the 16-byte chunks of row r XOR-swizzled by r so that a
// warp's chunk reads spread over the banks.
template <int BN>
__device__ __forceinline__ int red_word(int r, int col) {
  constexpr int kSwz = (BN / 4 < 8 ? BN / 4 : 8) - 1;
  return r * BN + ((((col >> 2) ^ (r & kSwz))) << 2) + (col & 3);
}

// One thread's chunk of an output row: y_i = fp32(acc_i * c_i) for the first nt of kCols
// accumulator columns (acc_i = v[i] / 64, exact), stored with stride O.  A full chunk has
// no per-column bound check; the pointer advances by O per column.
__device__ __forceinline__ void store_y(float *p, float y) { *p = y; }
__device__ __forceinline__ void store_y(__nv_bfloat16 *p, float y) { *p = __float2bfloat16_rn(y); }
template <int kCols, typename Out>
__device__ __forceinline__ void store_chunk(const uint32_t *v, const float *sc, int nt, Out *p,
                                            int64_t O, bool small_acc) {
  auto conv = [small_acc](uint32_t x) {
    const int a = ((int)x) >> 6;
    return small_acc ? __fsub_rn(__int_as_float(a + 0x4B400000), 12582912.0f) : __int2float_rn(a);
  };
  if (nt >= kCols) {
#pragma unroll
    for (int i = 0; i < kCols; ++i) {
      store_y(p, __fmul_rn(conv(v[i]), sc[i]));
      p += O;
    }
  } else {
#pragma unroll
    for (int i = 0; i < kCols; ++i) {
      if (i >= nt) break;
      store_y(p, __fmul_rn(conv(v[i]), sc[i]));
      p += O;
    }
  }
}

// Epilogue of the tensor-core kernels: warp w (0..3) owns accumulator lanes 32w..32w+31
// (output rows o), TMEM column j is token t0 + j and holds 64 * acc.  s_scale[j] holds
// c_t = fp32(fp32(g * s_t) / 127).  y = fp32(acc * c_t): acc is converted exactly (the
// magic-number addition is exact for |acc| < 2^22, a plain conversion is used otherwise)
// and multiplied once, the same rounding as acc * c_t.  With nred > 0 the nred partial
// accumulators in `red` (tile row r) are added first; integer sums, so the order of the
// parts does not change the result.
template <int BN>
__device__ __forceinline__ void store_tile(uint32_t trow, const float *s_scale, int64_t o,
                                           int64_t O, int64_t t0, int64_t T, bool small_acc,
                                           void *Y, int y_is_bf16, int32_t *acc_dbg,
                                           const uint32_t *red = nullptr, int nred = 0,
                                           int r = 0) {
  constexpr int kCols = BN < 32 ? BN : 32;
  const bool row_ok = o < O;
#pragma unroll 1
  for (int cb = 0; cb < BN; cb += 2 * kCols) {
    uint32_t va[32], vb[32];
    if constexpr (kCols == 32) {
      // BN is a multiple of 16: a chunk of 16 columns at the end is loaded at its own width,
      // so no load reads past the tile's accumulator columns
      if (BN - cb >= 32) {
        ptx::tmem_ld_32(trow + cb, va);
      } else {
        uint32_t v16[16];
        ptx::tmem_ld_16(trow + cb, v16);
#pragma unroll
        for (int i = 0; i < 16; ++i) va[i] = v16[i];
      }
      if (BN - cb - 32 >= 32) {
        ptx::tmem_ld_32(trow + cb + 32, vb);
      } else if (BN - cb - 32 > 0) {
        uint32_t v16[16];
        ptx::tmem_ld_16(trow + cb + 32, v16);
#pragma unroll
        for (int i = 0; i < 16; ++i) vb[i] = v16[i];
      }
    } else {
      uint32_t v16[16];
      ptx::tmem_ld_16(trow + cb, v16);
#pragma unroll
      for (int i = 0; i < 16; ++i) va[i] = v16[i];
    }
    ptx::tmem_ld_wait();
    for (int q = 0; q < nred; ++q) {
      const uint32_t *slot = red + q * (kBM * BN);
#pragma unroll
      for (int i = 0; i < kCols; i += 4) {
        if (cb + i < BN) {
          const uint4 p = *reinterpret_cast<const uint4 *>(slot + red_word<BN>(r, cb + i));
          va[i] += p.x, va[i + 1] += p.y, va[i + 2] += p.z, va[i + 3] += p.w;
        }
        if (cb + kCols + i < BN) {
          const uint4 p =
              *reinterpret_cast<const uint4 *>(slot + red_word<BN>(r, cb + kCols + i));
          vb[i] += p.x, vb[i + 1] += p.y, vb[i + 2] += p.z, vb[i + 3] += p.w;
        }
      }
    }
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int c0 = cb + half * kCols;
      if (c0 >= BN || !row_ok) continue;
      const uint32_t *v = half ? vb : va;
      // columns of this chunk that are real tokens of this tile
      const int nt = (int)min(T - (t0 + c0), (int64_t)(BN - c0));
      const int64_t off = (t0 + c0) * O + o;
      if (y_is_bf16)
        store_chunk<kCols>(v, s_scale + c0, nt, reinterpret_cast<__nv_bfloat16 *>(Y) + off, O,
                           small_acc);
      else
        store_chunk<kCols>(v, s_scale + c0, nt, reinterpret_cast<float *>(Y) + off, O,
                           small_acc);
      if (acc_dbg) {
#pragma unroll
        for (int i = 0; i < kCols; ++i) {
          if (i >= nt) break;
          acc_dbg[off + (int64_t)i * O] = ((int)v[i]) >> 6;
        }
      }
    }
  }
}

template <int BN, bool kCompact>
struct TcCfg {
  static constexpr int kABytes = kBM * kBK;
  static constexpr int kBBytes = BN * kBK;
  // packed weight bytes per row and K block: 2:4 -> 16 code + 16 meta, others -> 32 code
  static constexpr int kPackRow = kCompact ? 16 : 32;
  static constexpr int kPBytes = kBM * 32;
  static constexpr int kStageBytes = kABytes + kBBytes + kPBytes;
  static constexpr int kBudget = 225 * 1024 - BN * 4 - 512;
  static constexpr int kStages = (kBudget / kStageBytes) > 8 ? 8 : (kBudget / kStageBytes);
  static constexpr int kTmemCols = BN < 32 ? 32 : BN;
  static constexpr uint32_t kTxBytes = kBBytes + kPBytes;
  static constexpr size_t kSmem = 1024 + (size_t)kStages * kStageBytes +
                                  (size_t)(3 * kStages + 1) * 8 + 16 + (size_t)BN * 4;
};

// prmt selector placing the two kept 64*t bytes (bytes `b0`, `b0+1` of the code word) of a
// 2:4 group at positions i0 and i1 of a 4-byte word, zeros elsewhere (selector 4 picks a
// byte of the zero operand).
__device__ __forceinline__ uint32_t scatter_selector(uint32_t nib, uint32_t b0) {
  const uint32_t i0 = nib & 3u, i1 = nib >> 2;
  uint32_t sel = 0x4444u;
  sel = (sel & ~(0xfu << (4 * i0))) | (b0 << (4 * i0));
  sel = (sel & ~(0xfu << (4 * i1))) | ((b0 + 1u) << (4 * i1));
  return sel;
}

template <int BN, bool kCompact>
__global__ void __launch_bounds__(kTcThreads, 1)
    k_gemm_tc(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_c,
              const __grid_constant__ CUtensorMap tmap_m, const float *__restrict__ absmax,
              const float *__restrict__ gamma_eff, int64_t T, int64_t O, int64_t K,
              void *__restrict__ Y, int y_is_bf16, int32_t *__restrict__ acc_dbg,
              int32_t *err_flag) {
  using Cfg = TcCfg<BN, kCompact>;
  constexpr int S = Cfg::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *sA = smem;
  uint8_t *sB = smem + S * Cfg::kABytes;
  uint8_t *sP = sB + S * Cfg::kBBytes;
  uint64_t *full_a = reinterpret_cast<uint64_t *>(sP + S * Cfg::kPBytes);
  uint64_t *full_t = full_a + S;  // activation tile + packed weight tile landed
  uint64_t *empty = full_t + S;
  uint64_t *done = empty + S;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done + 1);
  float *s_scale = reinterpret_cast<float *>(tmem_slot + 4);

  // the next kernel on the stream may start its prologue; it waits for this one
  ptx::grid_dep_launch();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t o0 = (int64_t)blockIdx.x * kBM;
  const int64_t t0 = (int64_t)blockIdx.y * BN;
  const int nkb = (int)((K + kBK - 1) / kBK);
  bool timed_out = false;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      ptx::mbar_init(&full_a[s], 4);
      ptx::mbar_init(&full_t[s], 1);
      ptx::mbar_init(&empty[s], 1);
    }
    ptx::mbar_init(done, 1);
    ptx::fence_mbar_init();
  }
  if (warp == 5) {
    ptx::tmem_alloc(tmem_slot, Cfg::kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::grid_dep_wait();  // the previous kernel's outputs (activations, scales) are visible
  for (int i = threadIdx.x; i < BN; i += kTcThreads) {
    const int64_t t = t0 + i;
    s_scale[i] = t < T ? rescale_factor(__ldg(gamma_eff), __ldg(absmax + t)) : 0.0f;
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < 4) {
    // ---------------- weight expanders ----------------
    const int r = threadIdx.x;
    for (int kb = 0; kb < nkb; ++kb) {
      const int s = kb % S;
      const uint32_t ph = (uint32_t)(kb / S) & 1u;
      if ((kb >= S && !wait_phase(&empty[s], ph ^ 1u)) || !wait_phase(&full_t[s], ph)) {
        timed_out = true;
        break;
      }
      const uint8_t *prow = sP + s * Cfg::kPBytes;
      uint4 chunk[8];
      if constexpr (!kCompact) {
        const uint4 c0 = *reinterpret_cast<const uint4 *>(prow + r * 32);
        const uint4 c1 = *reinterpret_cast<const uint4 *>(prow + r * 32 + 16);
        const uint32_t w[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
        for (int c = 0; c < 8; ++c)
          chunk[c] = make_uint4(w[c] & 0xC0C0C0C0u, (w[c] << 2) & 0xC0C0C0C0u,
                                (w[c] << 4) & 0xC0C0C0C0u, (w[c] << 6) & 0xC0C0C0C0u);
      } else {
        const uint4 cw = *reinterpret_cast<const uint4 *>(prow + r * 16);
        const uint4 mw4 = *reinterpret_cast<const uint4 *>(prow + kBM * 16 + r * 16);
        const uint32_t w[4] = {cw.x, cw.y, cw.z, cw.w};
        const uint32_t mw[4] = {mw4.x, mw4.y, mw4.z, mw4.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t out[8];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint32_t z = (w[q] << (2 * j)) & 0xC0C0C0C0u;
            const uint32_t m8 = (mw[q] >> (8 * j)) & 0xffu;
            out[2 * j] = __byte_perm(z, 0u, scatter_selector(m8 & 15u, 0u));
            out[2 * j + 1] = __byte_perm(z, 0u, scatter_selector(m8 >> 4, 2u));
          }
          chunk[2 * q] = make_uint4(out[0], out[1], out[2], out[3]);
          chunk[2 * q + 1] = make_uint4(out[4], out[5], out[6], out[7]);
        }
      }
      uint8_t *dst = sA + s * Cfg::kABytes + r * 128;
#pragma unroll
      for (int c = 0; c < 8; ++c)
        *reinterpret_cast<uint4 *>(dst + ((c ^ (r & 7)) << 4)) = chunk[c];
      ptx::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&full_a[s]);
    }
  } else if (warp == 4) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      ptx::prefetch_tmap(&tmap_x);
      ptx::prefetch_tmap(&tmap_c);
      if constexpr (kCompact) ptx::prefetch_tmap(&tmap_m);
      int issued = 0;
      for (int kb = 0; kb < nkb; ++kb) {
        const int s = kb % S;
        const uint32_t ph = (uint32_t)(kb / S) & 1u;
        if (kb >= S && !wait_phase(&empty[s], ph ^ 1u)) {
          timed_out = true;
          break;
        }
        ptx::mbar_arrive_expect_tx(&full_t[s], Cfg::kTxBytes);
        ptx::tma_load_2d(sB + s * Cfg::kBBytes, &tmap_x, &full_t[s], kb * kBK, (int32_t)t0);
        uint8_t *p = sP + s * Cfg::kPBytes;
        ptx::tma_load_2d(p, &tmap_c, &full_t[s], kb * Cfg::kPackRow, (int32_t)o0);
        if constexpr (kCompact)
          ptx::tma_load_2d(p + kBM * 16, &tmap_m, &full_t[s], kb * 16, (int32_t)o0);
        issued = kb + 1;
      }
      // let every issued copy land before the CTA can exit (bounded)
      for (int kb = issued - S < 0 ? 0 : issued - S; kb < issued; ++kb)
        if (!wait_phase(&full_t[kb % S], (uint32_t)(kb / S) & 1u)) timed_out = true;
    }
  } else {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc = ptx::idesc_i8(kBM, BN);
      for (int kb = 0; kb < nkb; ++kb) {
        const int s = kb % S;
        const uint32_t ph = (uint32_t)(kb / S) & 1u;
        if (!wait_phase(&full_a[s], ph) || !wait_phase(&full_t[s], ph)) {
          timed_out = true;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t a_addr = ptx::smem_u32(sA + s * Cfg::kABytes);
        const uint32_t b_addr = ptx::smem_u32(sB + s * Cfg::kBBytes);
#pragma unroll
        for (int k = 0; k < kBK / 32; ++k)
          ptx::mma_i8(tmem, ptx::smem_desc_sw128(a_addr + 32 * k),
                      ptx::smem_desc_sw128(b_addr + 32 * k), idesc, (kb | k) != 0);
        ptx::mma_commit(&empty[s]);
      }
      ptx::mma_commit(done);
      // every MMA issued has completed before TMEM can be released, also after a timeout
      // (the epilogue skips its wait then)
      if (!wait_phase(done, 0)) timed_out = true;
    }
  }

  if (warp < 4) {
    // ---------------- epilogue ----------------
    __syncwarp();
    if (!timed_out && !wait_phase(done, 0)) timed_out = true;
    ptx::tc_fence_after();
    const int64_t o = o0 + warp * 32 + lane;
    const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
    // |acc| <= 127 * K < 2^22 for K <= 32768
    if (!timed_out)
      store_tile<BN>(trow, s_scale, o, O, t0, T, K <= 32768, Y, y_is_bf16, acc_dbg);
  }
  if (timed_out && err_flag) atomicOr(err_flag, SBN_FLAG_TIMEOUT);
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, Cfg::kTmemCols);
  }
}

// ---------------------------------------------------------------------------------------
// 2:4 on the sparse tensor cores (tcgen05.mma.sp kind::i8).
//
// A is the compressed weight tile: per row the 64 kept codes of a 128-wide K block, expanded
// to int8 lanes of 64 * t (no scatter: the kept codes are stored in order) into a 64-byte
// swizzled K-major tile.  The 2-bit metadata of the packed format (i0 | i1 << 2 per group,
// group 2h in the low nibble of byte h) is the sparse MMA's metadata as it stands: the TMA
// brings the 128 x 16-byte tile into shared memory and tcgen05.cp moves it to 4 TMEM
// columns; each K=64 MMA reads 2 of them.
// ---------------------------------------------------------------------------------------

template <int BN>
struct SpCfg {
  static constexpr int kKL = 128;                 // logical K of one block
  static constexpr int kABytes = kBM * kKL / 2;   // compressed int8: 64 bytes per row
  static constexpr int kBBytes = BN * kKL;        // activations: 128 bytes per token
  static constexpr int kPBytes = kBM * 16 * 2;    // packed codes + metadata, 16 B each per row
  static constexpr int kBlockBytes = kABytes + kBBytes + kPBytes;
  static constexpr int kBudget = 225 * 1024 - BN * 4 - 512;
  // kG consecutive K blocks share one set of pipeline barriers (a stage): every hand-off
  // between the roles has a fixed cost, so few tokens per tile move several blocks per
  // hand-off.  kSub block buffers in all, kStages = kSub / kG stages.
  static constexpr int kG = BN <= 32 ? 4 : BN <= 128 ? 2 : 1;
  static constexpr int kMaxSub = BN <= 32 ? 16 : 8;
  static constexpr int kFit = kBudget / kBlockBytes;
  static constexpr int kSub = ((kFit > kMaxSub ? kMaxSub : kFit) / kG) * kG;
  static constexpr int kStages = kSub / kG;
  static_assert(kStages >= 2, "at least two pipeline stages");
  static constexpr int kMetaCol = BN < 32 ? 32 : BN;  // first TMEM column of the metadata
  static constexpr int kNeedCols = kMetaCol + 4 * kSub;
  static constexpr int kTmemCols = kNeedCols <= 32 ? 32 : kNeedCols <= 64 ? 64
                                   : kNeedCols <= 128 ? 128 : kNeedCols <= 256 ? 256 : 512;
  static constexpr uint32_t kTxBytes = kBBytes + kPBytes;  // TMA bytes of one block
  static constexpr size_t kSmem = 1024 + (size_t)kSub * kBlockBytes +
                                  (size_t)(3 * kStages + 1) * 8 + 16 + (size_t)BN * 4;
  // K split over a cluster (BN <= 32): CTA 0 receives the other CTAs' partial tiles in its
  // block buffers
  static constexpr int kMaxSplit = BN <= 32 ? 8 : 1;
  static_assert((kMaxSplit - 1) * kBM * BN * 4 <= kSub * kBlockBytes,
                "the partial tiles of a split must fit in the stage memory");
};

template <int BN>
__global__ void __launch_bounds__(kTcThreads, 1)
    k_gemm_sp24(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_c,
                const __grid_constant__ CUtensorMap tmap_m, const float *__restrict__ absmax,
                const float *__restrict__ gamma_eff, int64_t T, int64_t O, int64_t K,
                void *__restrict__ Y, int y_is_bf16, int32_t *__restrict__ acc_dbg,
                int32_t *err_flag) {
  using Cfg = SpCfg<BN>;
  constexpr int S = Cfg::kStages, G = Cfg::kG, U = Cfg::kSub;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  // block buffer u = G * stage + g holds K block g of the stage
  uint8_t *sB = smem;                        // 1024-aligned blocks (128-byte swizzle)
  uint8_t *sA = sB + U * Cfg::kBBytes;       // 512-aligned blocks (64-byte swizzle)
  uint8_t *sP = sA + U * Cfg::kABytes;       // packed codes [128][16] then metadata [128][16]
  uint64_t *full_a = reinterpret_cast<uint64_t *>(sP + U * Cfg::kPBytes);
  uint64_t *full_t = full_a + S;
  uint64_t *empty = full_t + S;
  uint64_t *done = empty + S;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done + 1);
  float *s_scale = reinterpret_cast<float *>(tmem_slot + 4);

  // the next kernel on the stream may start its prologue; it waits for this one
  ptx::grid_dep_launch();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // A launch with clusters of C CTAs along x splits each tile's K blocks into C contiguous
  // ranges, one per CTA; CTA 0 of the cluster sums the partial accumulators and stores.
  const uint32_t csplit = ptx::cluster_nctarank();
  const uint32_t crank = csplit > 1 ? ptx::cluster_ctarank() : 0u;
  const int64_t o0 = (int64_t)(blockIdx.x / csplit) * kBM;
  const int64_t t0 = (int64_t)blockIdx.y * BN;
  const int nkb_all = (int)((K + Cfg::kKL - 1) / Cfg::kKL);
  const int kb0 = (int)((int64_t)nkb_all * crank / csplit);
  const int nkb = (int)((int64_t)nkb_all * (crank + 1) / csplit) - kb0;
  const int nst = (nkb + G - 1) / G;  // stages of this CTA; the last may hold fewer blocks
  bool timed_out = false;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      ptx::mbar_init(&full_a[s], 4);
      ptx::mbar_init(&full_t[s], 1);
      ptx::mbar_init(&empty[s], 1);
    }
    ptx::mbar_init(done, 1);
    ptx::fence_mbar_init();
  }
  if (warp == 5) {
    ptx::tmem_alloc(tmem_slot, Cfg::kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::grid_dep_wait();  // the previous kernel's outputs (activations, scales) are visible
  for (int i = threadIdx.x; i < BN; i += kTcThreads) {
    const int64_t t = t0 + i;
    s_scale[i] = t < T ? rescale_factor(__ldg(gamma_eff), __ldg(absmax + t)) : 0.0f;
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < 4) {
    // ---------------- compressed-weight expanders ----------------
    const int r = threadIdx.x;
    for (int j = 0; j < nst; ++j) {
      const int s = j % S;
      const uint32_t ph = (uint32_t)(j / S) & 1u;
      if ((j >= S && !wait_phase(&empty[s], ph ^ 1u)) || !wait_phase(&full_t[s], ph)) {
        timed_out = true;
        break;
      }
      const int nb = min(G, nkb - j * G);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        if (g >= nb) break;
        const int u = s * G + g;
        const int kb = kb0 + j * G + g;
        const uint4 cw = *reinterpret_cast<const uint4 *>(sP + u * Cfg::kPBytes + r * 16);
        const uint32_t w[4] = {cw.x, cw.y, cw.z, cw.w};
        // Groups past the matrix (rows >= O, or the second half of the last block when
        // K % 128 == 64) were zero-filled by the TMA; give them the valid index pair (0, 1)
        // so the MMA never sees a malformed metadata nibble (their codes are zero anyway).
        if (o0 + r >= O) {
          *reinterpret_cast<uint4 *>(sP + u * Cfg::kPBytes + kBM * 16 + r * 16) =
              make_uint4(0x44444444u, 0x44444444u, 0x44444444u, 0x44444444u);
        } else if ((int64_t)kb * Cfg::kKL + 64 >= K) {
          *reinterpret_cast<uint2 *>(sP + u * Cfg::kPBytes + kBM * 16 + r * 16 + 8) =
              make_uint2(0x44444444u, 0x44444444u);
        }
        uint8_t *dst = sA + u * Cfg::kABytes + r * 64;
#pragma unroll
        for (int c = 0; c < 4; ++c)  // 16 kept codes -> 16 int8 lanes, in order
          *reinterpret_cast<uint4 *>(dst + ((c ^ ((r >> 1) & 3)) << 4)) =
              make_uint4(w[c] & 0xC0C0C0C0u, (w[c] << 2) & 0xC0C0C0C0u,
                         (w[c] << 4) & 0xC0C0C0C0u, (w[c] << 6) & 0xC0C0C0C0u);
      }
      ptx::fence_proxy_async_smem();
      __syncwarp();
#ifdef SBN_TIMEOUT_TEST
      if (lane == 0 && !(warp == 0 && j == 1)) ptx::mbar_arrive(&full_a[s]);
#else
      if (lane == 0) ptx::mbar_arrive(&full_a[s]);
#endif
    }
  } else if (warp == 4) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      ptx::prefetch_tmap(&tmap_x);
      ptx::prefetch_tmap(&tmap_c);
      ptx::prefetch_tmap(&tmap_m);
      int issued = 0;
      for (int j = 0; j < nst; ++j) {
        const int s = j % S;
        const uint32_t ph = (uint32_t)(j / S) & 1u;
        if (j >= S && !wait_phase(&empty[s], ph ^ 1u)) {
          timed_out = true;
          break;
        }
        const int nb = min(G, nkb - j * G);
        ptx::mbar_arrive_expect_tx(&full_t[s], (uint32_t)nb * Cfg::kTxBytes);
        for (int g = 0; g < nb; ++g) {
          const int u = s * G + g;
          const int kb = kb0 + j * G + g;
          ptx::tma_load_2d(sB + u * Cfg::kBBytes, &tmap_x, &full_t[s], kb * Cfg::kKL,
                           (int32_t)t0);
          uint8_t *p = sP + u * Cfg::kPBytes;
          ptx::tma_load_2d(p, &tmap_c, &full_t[s], kb * 16, (int32_t)o0);
          ptx::tma_load_2d(p + kBM * 16, &tmap_m, &full_t[s], kb * 16, (int32_t)o0);
        }
        issued = j + 1;
      }
      for (int j = issued - S < 0 ? 0 : issued - S; j < issued; ++j)
        if (!wait_phase(&full_t[j % S], (uint32_t)(j / S) & 1u)) timed_out = true;
    }
  } else {
    // ---------------- metadata copy + sparse MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc = ptx::idesc_i8_sparse(kBM, BN);
      for (int j = 0; j < nst; ++j) {
        const int s = j % S;
        const uint32_t ph = (uint32_t)(j / S) & 1u;
        if (!wait_phase(&full_a[s], ph) || !wait_phase(&full_t[s], ph)) {
          timed_out = true;
          break;
        }
        ptx::tc_fence_after();
        const int nb = min(G, nkb - j * G);
        for (int g = 0; g < nb; ++g) {
          const int u = s * G + g;
          const uint32_t e_col = tmem + Cfg::kMetaCol + 4 * u;
          ptx::tmem_cp_128x128b(
              e_col, ptx::smem_desc_rows16(ptx::smem_u32(sP + u * Cfg::kPBytes + kBM * 16)));
          const uint32_t a_addr = ptx::smem_u32(sA + u * Cfg::kABytes);
          const uint32_t b_addr = ptx::smem_u32(sB + u * Cfg::kBBytes);
#pragma unroll
          for (int k = 0; k < 2; ++k)  // logical K 64 per MMA: 32 bytes of A, 64 of B
            ptx::mma_sp_i8(tmem, ptx::smem_desc_sw64(a_addr + 32 * k),
                           ptx::smem_desc_sw128(b_addr + 64 * k), e_col + 2 * k, idesc,
                           (j | g | k) != 0);
        }
        ptx::mma_commit(&empty[s]);
      }
      ptx::mma_commit(done);
      // every MMA issued has completed before TMEM can be released, also after a timeout
      // (the epilogue skips its wait then)
      if (!wait_phase(done, 0)) timed_out = true;
    }
  }

  const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
  if (warp < 4) {
    __syncwarp();
    if (!timed_out && !wait_phase(done, 0)) timed_out = true;
    ptx::tc_fence_after();
  }
  if (csplit > 1) {
    // ---------------- K-split reduction into CTA 0 ----------------
    // After the first cluster barrier every CTA's MMAs have completed, so CTA 0's stage
    // memory is free; CTAs 1.. store their partial tiles there; after the second, CTA 0
    // reads them.  A CTA that timed out sends what it has (the flag marks the output).
    ptx::fence_proxy_async_smem();
    __syncwarp();
    ptx::cluster_sync();
    if (warp < 4 && crank != 0) {
      const int r = threadIdx.x;
      const uint32_t slot = ptx::mapa_shared(ptx::smem_u32(smem), 0) +
                            (crank - 1) * (uint32_t)(kBM * BN * 4);
#pragma unroll
      for (int cb = 0; cb < BN; cb += 16) {
        uint32_t v[16];
        ptx::tmem_ld_16(trow + cb, v);
        ptx::tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; i += 4) {
          const uint4 p = nkb > 0 ? make_uint4(v[i], v[i + 1], v[i + 2], v[i + 3])
                                  : make_uint4(0u, 0u, 0u, 0u);
          ptx::st_cluster_v4(slot + 4u * (uint32_t)red_word<BN>(r, cb + i), p);
        }
      }
    }
    __syncwarp();
    ptx::cluster_sync();
  }
  if (warp < 4 && crank == 0) {
    // ---------------- epilogue ----------------
    const int64_t o = o0 + warp * 32 + lane;
    // |acc| <= 127 * K < 2^22 for K <= 32768
    if (!timed_out)
      store_tile<BN>(trow, s_scale, o, O, t0, T, K <= 32768, Y, y_is_bf16, acc_dbg,
                     reinterpret_cast<const uint32_t *>(smem), (int)csplit - 1, threadIdx.x);
  }
  if (timed_out && err_flag) atomicOr(err_flag, SBN_FLAG_TIMEOUT);
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, Cfg::kTmemCols);
  }
}

// ---------------------------------------------------------------------------------------
// Helpers of the persistent CTA-pair kernel below: every wait is bounded; a timeout anywhere
// raises a shared abort flag that ends all loops.
// ---------------------------------------------------------------------------------------

__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity, volatile int *abort) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    for (int i = 0; i < 64; ++i)
      if (ptx::mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if (clock64() - t0 > kWaitCycles) {
      *abort = 1;
      return false;
    }
  }
}

// bar.red.or over the `n` threads of named barrier `id`: every participant learns whether
// any of them passed true.
__device__ __forceinline__ bool bar_any(int id, int n, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.or.pred p, %2, %3, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}

// ---------------------------------------------------------------------------------------
// CTA-pair 2:4 kernel for large token counts.  A cluster of two CTAs computes 256 weight
// rows x BN tokens per tile with the pair form of the sparse MMA: each CTA stages and
// expands its own 128 rows and loads half of the activation tile (BN / 2 tokens), so every
// SM streams half the activation bytes of a single-CTA tile per unit of MMA work.  Two
// threads of CTA 0 issue the MMAs and the commits for both CTAs (commits reach the same
// barrier in both), alternate stages each; the expanders and the epilogue warps of both
// CTAs report to CTA 0's barriers.  Persistent over tiles with two TMEM accumulators
// (columns 0 and 256) per CTA: the epilogue warps drain tile i (and zero its accumulator)
// while the MMAs already accumulate tile i+1.
//
// A and its metadata live in TMEM: the expanders write each row's expanded codes (16
// columns per K block) and its metadata (4 columns) into their CTA's TMEM (tcgen05.st,
// lane = row), and the pair MMA reads A from there.  Shared memory then holds only B and
// the packed planes (17 KB per K block at 208 tokens), so the TMA ring is six stages of two
// blocks deep; the A ring lives in the TMEM columns the two accumulators leave free (two
// stages at 208 tokens).  Ring 1 (shared memory) is filled by the producers and freed by
// the MMA's commit of the stage; ring 2 (TMEM) is filled by the expanders, which wait for
// stage kg - S2's commit before they write stage kg's ring-2 slot.  The tile width 208 puts
// a 2048-token batch in 10 token tiles (six rounds of tiles on 74 pairs for 11008 rows); the
// host takes 192 where that needs no more rounds (4096 rows x 4096 tokens: 5 either way).
// ---------------------------------------------------------------------------------------
// 12 warps: expanders 0-3, producers 4 and 10, MMA threads in warps 5 and 11, epilogue 6-9
constexpr int kPairThreads = 384;

template <int BN>
struct PairCfg {
  static constexpr int kKL = 128;
  static constexpr int kBHalf = BN / 2;  // tokens per CTA
  static constexpr int kBBytes = kBHalf * kKL;
  static constexpr int kPBytes = kBM * 16;  // one plane (codes or meta) of a block
  static constexpr int kG = 2;              // K blocks per stage
  static constexpr int kSlot1 = kG * (kBBytes + 2 * kPBytes);
  static constexpr int kBudget = 225 * 1024 - BN * 4 - 1024;
  static constexpr int kS1 = (kBudget / kSlot1) / 2 * 2;  // even: two producers
  static_assert(kS1 >= 2, "at least two shared-memory stages");
  static_assert(kBBytes % 1024 == 0, "B blocks keep the 1024-byte swizzle alignment");
  // TMEM: accumulators at columns 0 and 256; each gap [BN, 256) holds kPerGap blocks of A
  // (16 columns each, from the gap's start) and their metadata (4 columns each, after them)
  static constexpr int kAccStride = 256;
  static constexpr int kPerGap = (256 - BN) / 20;
  // TMEM stages, even: the two MMA threads take alternate stages
  static constexpr int kS2 = (2 * kPerGap) / kG / 2 * 2;
  static_assert(kS2 % 2 == 0 && kS1 % 2 == 0, "rings of whole stage pairs");
  static_assert(kS2 >= 2, "at least two TMEM stages");
  static_assert(BN % 16 == 0 && BN <= 224, "pair tile width");
  static_assert(kBHalf % 8 == 0, "B tiles of whole 8-row swizzle atoms");
  __device__ static constexpr uint32_t a_col(int b) {  // b: block slot of ring 2
    return (uint32_t)((b / kPerGap) * kAccStride + BN + 16 * (b % kPerGap));
  }
  __device__ static constexpr uint32_t e_col(int b) {
    return (uint32_t)((b / kPerGap) * kAccStride + BN + 16 * kPerGap + 4 * (b % kPerGap));
  }
  static constexpr int kTmemCols = 512;
  static constexpr uint32_t kTxBytes = kBBytes + 2 * kPBytes;  // per block and CTA
  // barriers: full_t[S1], empty1[S1], full_a[S2], acc_full[2], acc_empty[2], mma_done;
  // then the TMEM address, the abort flag (32 bytes) and the per-token scales
  static constexpr size_t kSmem = 1024 + (size_t)kS1 * kSlot1 +
                                  (size_t)(2 * kS1 + kS2 + 5) * 8 + 32 + (size_t)BN * 4;
  static_assert(kS2 < kS1, "a stage's ring-2 slot is freed by the completion of stage kg - S2");
};

template <int BN>
__global__ void __launch_bounds__(kPairThreads, 1)
    k_gemm_sp24_pair(const __grid_constant__ CUtensorMap tmap_x,
                      const __grid_constant__ CUtensorMap tmap_c,
                      const __grid_constant__ CUtensorMap tmap_m,
                      const float *__restrict__ absmax, const float *__restrict__ gamma_eff,
                      int64_t T, int64_t O, int64_t K, void *__restrict__ Y, int y_is_bf16,
                      int32_t *__restrict__ acc_dbg, int32_t *err_flag) {
  using Cfg = PairCfg<BN>;
  constexpr int S1 = Cfg::kS1, S2 = Cfg::kS2, G = Cfg::kG;
  constexpr int kTileM = 2 * kBM;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  // ring-1 slot s: B of its G blocks, then their codes planes, then their meta planes
  uint8_t *ring1 = smem;
  uint64_t *full_t = reinterpret_cast<uint64_t *>(ring1 + (size_t)S1 * Cfg::kSlot1);  // own TMA
  // own stage done (the pair's commit of its MMAs): frees the ring-1 slot of stage kg, and
  // (S2 stages later) the ring-2 slot of stage kg
  uint64_t *empty1 = full_t + S1;
  uint64_t *full_a = empty1 + S1;     // CTA 0: both CTAs' expanders
  uint64_t *acc_full = full_a + S2;   // [2], own
  uint64_t *acc_empty = acc_full + 2;  // [2], CTA 0: both
  uint64_t *mma_done = acc_empty + 2;  // CTA 0: drain
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_done + 1);
  volatile int *s_abort = reinterpret_cast<volatile int *>(tmem_slot + 2);
  float *s_scale = reinterpret_cast<float *>(tmem_slot + 8);

  ptx::grid_dep_launch();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = ptx::cluster_ctarank();
  const int64_t pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int nkb = (int)((K + Cfg::kKL - 1) / Cfg::kKL);
  const int nst = (nkb + G - 1) / G;
  const int64_t n_o = (O + kTileM - 1) / kTileM, n_t = (T + BN - 1) / BN;
  const int64_t ntiles = n_o * n_t;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S1; ++s) {
      ptx::mbar_init(&full_t[s], 1);
      ptx::mbar_init(&empty1[s], 1);
    }
    for (int s = 0; s < S2; ++s)
      ptx::mbar_init(&full_a[s], 8);  // the expander warps of both CTAs (used in CTA 0)
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(&acc_full[b], 2);   // a commit of each MMA thread
      ptx::mbar_init(&acc_empty[b], 8);  // the epilogue warps of both CTAs
    }
    ptx::mbar_init(mma_done, 2);
    *s_abort = 0;
    ptx::fence_mbar_init();
  }
  ptx::cluster_sync();
  if (warp == 5) {
    ptx::tmem_alloc_pair(tmem_slot, Cfg::kTmemCols);
    ptx::tmem_relinquish_pair();
  }
  ptx::grid_dep_wait();
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t full_a0 = ptx::mapa_shared(ptx::smem_u32(full_a), 0);
  const uint32_t acc_empty0 = ptx::mapa_shared(ptx::smem_u32(acc_empty), 0);

  if (warp < 4) {
    // ---------------- expanders: this CTA's 128 rows into its TMEM ----------------
    const int r = threadIdx.x;
    const uint32_t lrow = (uint32_t)(warp * 32) << 16;
    // stage kg's slots and phases; (f1, fph) the ring-1 slot of stage kg - S2, whose
    // completion frees ring-2 slot s2
    int kg = 0, s1 = 0, s2 = 0, f1 = S1 - S2;
    uint32_t ph1 = 0, fph = 1;
    for (int64_t tile = pair;
         tile < ntiles && !__any_sync(0xffffffffu, *s_abort != 0); tile += npairs) {
      const int64_t o0 = (tile % n_o) * kTileM + (int64_t)rank * kBM;
      const bool row_ok = o0 + r < O;
      for (int j = 0; j < nst; ++j) {
        const bool ok = (kg < S2 || wait_or_abort(&empty1[f1], fph, s_abort)) &&
                        wait_or_abort(&full_t[s1], ph1, s_abort);
        if (!__all_sync(0xffffffffu, ok)) break;
        ptx::tc_fence_after();
        const uint8_t *slot = ring1 + (size_t)s1 * Cfg::kSlot1 + G * Cfg::kBBytes;
        const int nb = min(G, nkb - j * G);
#pragma unroll
        for (int g = 0; g < G; ++g) {
          if (g >= nb) break;
          const int kb = j * G + g;
          const int b2 = s2 * G + g;
          const uint4 cw = *reinterpret_cast<const uint4 *>(slot + g * Cfg::kPBytes + r * 16);
          uint4 m4 = *reinterpret_cast<const uint4 *>(slot + (G + g) * Cfg::kPBytes + r * 16);
          // groups outside the matrix get the valid index pair (0, 1); their codes are zero
          if (!row_ok) {
            m4 = make_uint4(0x44444444u, 0x44444444u, 0x44444444u, 0x44444444u);
          } else if ((int64_t)kb * Cfg::kKL + 64 >= K) {
            m4.z = 0x44444444u;
            m4.w = 0x44444444u;
          }
          ptx::tmem_st_4(tmem + lrow + Cfg::e_col(b2), m4);
          // 16 kept codes per word -> 16 int8 lanes of 64 * t, in K order: column 4c + q
          // holds the four values (w[c] << 2q) & 0xC0C0C0C0
          const uint32_t w[4] = {cw.x, cw.y, cw.z, cw.w};
          uint32_t a[16];
#pragma unroll
          for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int q = 0; q < 4; ++q) a[4 * c + q] = (w[c] << (2 * q)) & 0xC0C0C0C0u;
          ptx::tmem_st_16(tmem + lrow + Cfg::a_col(b2), a);
        }
        ptx::tmem_st_wait();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive_cluster(full_a0 + 8u * (uint32_t)s2);
        ++kg;
        if (++s1 == S1) s1 = 0, ph1 ^= 1u;
        if (++s2 == S2) s2 = 0;
        if (++f1 == S1) f1 = 0, fph ^= 1u;
      }
    }
  } else if (warp == 4 || warp == 10) {
    // ---------------- two TMA producers: stage kg by producer kg % 2 (S1 is even) --------
    if (lane == 0) {
      const int pt = warp == 4 ? 0 : 1;
      ptx::prefetch_tmap(&tmap_x);
      ptx::prefetch_tmap(&tmap_c);
      ptx::prefetch_tmap(&tmap_m);
      int64_t kg = 0, issued = -1;
      for (int64_t tile = pair; tile < ntiles && !*s_abort; tile += npairs) {
        const int64_t o0 = (tile % n_o) * kTileM + (int64_t)rank * kBM;
        const int64_t t0 = (tile / n_o) * BN + (int64_t)rank * Cfg::kBHalf;
        for (int j = 0; j < nst; ++j, ++kg) {
          if ((int)(kg & 1) != pt) continue;
          const int s = (int)(kg % S1);
          const uint32_t ph = (uint32_t)(kg / S1) & 1u;
          if (kg >= S1 && !wait_or_abort(&empty1[s], ph ^ 1u, s_abort)) break;
          const int nb = min(G, nkb - j * G);
          ptx::mbar_arrive_expect_tx(&full_t[s], (uint32_t)nb * Cfg::kTxBytes);
          uint8_t *slot = ring1 + (size_t)s * Cfg::kSlot1;
          for (int g = 0; g < nb; ++g) {
            const int kb = j * G + g;
            ptx::tma_load_2d(slot + g * Cfg::kBBytes, &tmap_x, &full_t[s], kb * Cfg::kKL,
                             (int32_t)t0);
            ptx::tma_load_2d(slot + G * Cfg::kBBytes + g * Cfg::kPBytes, &tmap_c, &full_t[s],
                             kb * 16, (int32_t)o0);
            ptx::tma_load_2d(slot + G * Cfg::kBBytes + (G + g) * Cfg::kPBytes, &tmap_m,
                             &full_t[s], kb * 16, (int32_t)o0);
          }
          issued = kg;
        }
      }
      // its last S1 / 2 stages, one per slot of its half, land before the CTA can exit
      for (int64_t q = issued, i = 0; q >= 0 && i < S1 / 2; q -= 2, ++i)
        if (!wait_phase(&full_t[q % S1], (uint32_t)(q / S1) & 1u)) *s_abort = 1;
    }
  } else if (warp == 5 || warp == 11) {
    // ---------------- CTA 0: the pair's MMAs, stage kg by MMA thread kg % 2 ----------------
    // Every MMA accumulates: the epilogue zeroes an accumulator before its tile (integer
    // sums, so the order in which the two threads' MMAs reach it does not matter).  A thread's
    // commit covers its own MMAs: stage kg's slots are freed by the thread that issued kg.
    if (rank == 0 && lane == 0) {
      const int mt = warp == 5 ? 0 : 1;
      constexpr uint32_t idesc = ptx::idesc_i8_sparse(kTileM, BN);
      // B descriptor of ring 1's first byte; a slot, block and K half add (offset >> 4)
      const uint64_t b_desc0 = ptx::smem_desc_sw128(ptx::smem_u32(ring1));
      // this thread's next stage kg = mt, mt + 2, ...: its ring slots (S1 and S2 are even)
      int s1 = mt, s2 = mt;
      uint32_t ph2 = 0;
      int64_t kg = 0;
      int i = 0;
      for (int64_t tile = pair; tile < ntiles && !*s_abort; tile += npairs, ++i) {
        const int buf = i & 1;
        if (!wait_or_abort(&acc_empty[buf], (uint32_t)(i >> 1) & 1u, s_abort)) break;
        ptx::tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(buf * Cfg::kAccStride);
        bool ok = true;
        for (int j = 0; j < nst; ++j, ++kg) {
          if ((int)(kg & 1) != mt) continue;
          // both CTAs expanded this stage, after their own B and planes had landed
          if (!wait_or_abort(&full_a[s2], ph2, s_abort)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const int nb = min(G, nkb - j * G);
          const uint64_t b_desc = b_desc0 + (uint64_t)((s1 * Cfg::kSlot1) >> 4);
          for (int g = 0; g < nb; ++g) {
            const int b2 = s2 * G + g;
#pragma unroll
            for (int k = 0; k < 2; ++k)
              ptx::mma_sp_i8_pair_tmem_a(d_tmem, tmem + Cfg::a_col(b2) + 8 * k,
                                         b_desc + (uint64_t)((g * Cfg::kBBytes + 64 * k) >> 4),
                                         tmem + Cfg::e_col(b2) + 2 * k, idesc, 1u);
          }
          ptx::mma_commit_pair(&empty1[s1], 0x3);
          if ((s1 += 2) >= S1) s1 -= S1;
          if ((s2 += 2) >= S2) s2 -= S2, ph2 ^= 1u;
        }
        if (!ok) break;
        ptx::mma_commit_pair(&acc_full[buf], 0x3);
      }
      ptx::mma_commit_pair(mma_done, 0x1);
      if (!wait_phase(mma_done, 0)) *s_abort = 1;
    }
  } else {
    // ---------------- epilogue (warps 6-9): this CTA's 128 rows ----------------
    const int q = warp & 3;
    const int et = threadIdx.x - 6 * 32;
    const float g = __ldg(gamma_eff);
    const uint32_t zero[16] = {};
    const uint32_t tlane = tmem + ((uint32_t)(q * 32) << 16);
    // both accumulators start at zero; each is zeroed again after its tile is read
#pragma unroll 1
    for (int b = 0; b < 2; ++b)
      for (int c = 0; c < BN; c += 16) ptx::tmem_st_16(tlane + b * Cfg::kAccStride + c, zero);
    ptx::tmem_st_wait();
    ptx::tc_fence_before();
    __syncwarp();
    if (lane == 0) {
      ptx::mbar_arrive_cluster(acc_empty0);
      ptx::mbar_arrive_cluster(acc_empty0 + 8u);
    }
    bool failed = false;
    int i = 0;
    for (int64_t tile = pair; tile < ntiles; tile += npairs, ++i) {
      const int buf = i & 1;
      const int64_t o0 = (tile % n_o) * kTileM + (int64_t)rank * kBM;
      const int64_t t0 = (tile / n_o) * BN;
      if (bar_any(1, 128, failed)) break;
      for (int c = et; c < BN; c += 128) {
        const int64_t t = t0 + c;
        s_scale[c] = t < T ? rescale_factor(g, __ldg(absmax + t)) : 0.0f;
      }
      asm volatile("bar.sync 1, 128;" ::: "memory");
      failed = !__all_sync(0xffffffffu, !*s_abort && wait_or_abort(&acc_full[buf],
                                                                   (uint32_t)(i >> 1) & 1u,
                                                                   s_abort));
      ptx::tc_fence_after();
      if (!failed) {
        const uint32_t trow = tlane + (uint32_t)(buf * Cfg::kAccStride);
        store_tile<BN>(trow, s_scale, o0 + q * 32 + lane, O, t0, T, K <= 32768, Y, y_is_bf16,
                       acc_dbg);
        for (int c = 0; c < BN; c += 16) ptx::tmem_st_16(trow + c, zero);
        ptx::tmem_st_wait();
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive_cluster(acc_empty0 + 8u * (uint32_t)buf);
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && *s_abort && err_flag) atomicOr(err_flag, SBN_FLAG_TIMEOUT);
  ptx::cluster_sync();
  if (warp == 5) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc_pair(tmem, Cfg::kTmemCols);
  }
}

// ---------------------------------------------------------------------------------------

static PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void *p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 2-D tensor map over a row-major uint8 matrix [rows, cols] with row stride `ld` bytes.
bool encode_u8(CUtensorMap *map, const void *base, int64_t cols, int64_t rows, int64_t ld,
                      uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swz) {
  auto encode = get_encode_fn();
  if (!encode) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ld};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides,
                box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// CTAs per tile along K for k_gemm_sp24<BN> (1 = no split).  The kernel holds one CTA per
// SM; a split trades longer-running tiles for more CTAs.  Estimated time in units of one
// K block's pipeline time (measured on B200 at 16 and 32 tokens: about 0.22 us per block,
// 4 us of fixed cost per CTA wave, 2.5 us for the cluster reduction):
// waves x (19 + K blocks per CTA) + 11 for a split.  The number of clusters that fit at
// once comes from the occupancy API (clusters stay inside a GPC) and is cached per device
// and split.
template <int BN, typename Kern>
static int sp24_split(Kern kern, int64_t tiles, int nkb) {
  using Cfg = SpCfg<BN>;
  if (Cfg::kMaxSplit <= 1 || nkb < 2) return 1;
  constexpr int kMaxDevices = 64;
  static int slots_cache[kMaxDevices][Cfg::kMaxSplit + 1] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    (void)cudaGetLastError();
    return 1;
  }
  int best = 1;
  double best_cost = 0.0;
  for (int c = 1; c <= Cfg::kMaxSplit && c <= nkb; ++c) {
    int &slots = slots_cache[dev][c];  // CTAs resident at once with clusters of c
    if (slots == 0) {
      if (c == 1) {
        int per_sm = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kTcThreads,
                                                          Cfg::kSmem) != cudaSuccess ||
            per_sm < 1) {
          (void)cudaGetLastError();
          per_sm = 1;
        }
        slots = per_sm * num_sms();
      } else {
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = (unsigned)c;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.gridDim = dim3((unsigned)(c * (num_sms() / c)));
        cfg.blockDim = dim3(kTcThreads);
        cfg.dynamicSmemBytes = Cfg::kSmem;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n < 1) {
          (void)cudaGetLastError();
          n = -1;  // not launchable with this cluster size
        }
        slots = n > 0 ? n * c : -1;
      }
    }
    if (slots <= 0) continue;
    const int64_t waves = (tiles * c + slots - 1) / slots;
    const double cost = (double)waves * (19.0 + (nkb + c - 1) / c) + (c > 1 ? 11.0 : 0.0);
    if (c == 1 || cost < best_cost) {
      best = c;
      best_cost = cost;
    }
  }
  return best;
}

template <int BN, bool kCompact>
static sbn_status gemm_tc_t(const int8_t *Xq, const float *absmax, const uint8_t *codes,
                            const uint8_t *meta, const float *gamma_eff, int64_t T, int64_t O,
                            int64_t K, int64_t ldx, int64_t ldc, int64_t ldm, void *Y, int y_is_bf16,
                            int32_t *acc_dbg, int32_t *err_flag, cudaStream_t st) {
  using Cfg = TcCfg<BN, kCompact>;
  CUtensorMap tx, tc, tm;
  const int64_t crow = kCompact ? K / 8 : K / 4;  // data bytes of a codes row
  if (!encode_u8(&tx, Xq, K, T, ldx, kBK, BN, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_u8(&tc, codes, crow, O, ldc, Cfg::kPackRow, kBM, CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !encode_u8(&tm, meta, K / 8, O, ldm, 16, kBM, CU_TENSOR_MAP_SWIZZLE_NONE))
    return SBN_ERR_CUDA;
  auto kern = k_gemm_tc<BN, kCompact>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Cfg::kSmem) !=
      cudaSuccess)
    return SBN_ERR_CUDA;
  const dim3 grid((unsigned)((O + kBM - 1) / kBM), (unsigned)((T + BN - 1) / BN));
  return launch_pdl(kern, grid, dim3(kTcThreads), Cfg::kSmem, st, tx, tc, tm, absmax, gamma_eff,
                    T, O, K, Y, y_is_bf16, acc_dbg, err_flag);
}

template <int BN>
static sbn_status gemm_sp24_t(const int8_t *Xq, const float *absmax, const uint8_t *codes,
                              const uint8_t *meta, const float *gamma_eff, int64_t T, int64_t O,
                              int64_t K, int64_t ldx, int64_t ldc, int64_t ldm, void *Y, int y_is_bf16,
                              int32_t *acc_dbg, int32_t *err_flag, cudaStream_t st) {
  using Cfg = SpCfg<BN>;
  CUtensorMap tx, tc, tm;
  if (!encode_u8(&tx, Xq, K, T, ldx, Cfg::kKL, BN, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_u8(&tc, codes, K / 8, O, ldc, 16, kBM, CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !encode_u8(&tm, meta, K / 8, O, ldm, 16, kBM, CU_TENSOR_MAP_SWIZZLE_NONE))
    return SBN_ERR_CUDA;
  auto kern = k_gemm_sp24<BN>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Cfg::kSmem) !=
      cudaSuccess)
    return SBN_ERR_CUDA;
  const int64_t row_tiles = (O + kBM - 1) / kBM, tok_tiles = (T + BN - 1) / BN;
  const int nkb = (int)((K + Cfg::kKL - 1) / Cfg::kKL);
  const int csplit = sp24_split<BN>(kern, row_tiles * tok_tiles, nkb);
  if (csplit > 1) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)csplit;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3((unsigned)(row_tiles * csplit), (unsigned)tok_tiles);
    cfg.blockDim = dim3(kTcThreads);
    cfg.dynamicSmemBytes = Cfg::kSmem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, tx, tc, tm, absmax, gamma_eff, T, O, K,
                                             Y, y_is_bf16, acc_dbg, err_flag);
    if (e == cudaSuccess) return SBN_OK;
    (void)cudaGetLastError();
    // only a cluster the device cannot place falls back to one CTA per tile (same results);
    // any other launch error is reported
    if (e != cudaErrorInvalidClusterSize && e != cudaErrorLaunchOutOfResources &&
        e != cudaErrorNotSupported)
      return SBN_ERR_CUDA;
  }
  return launch_pdl(kern, dim3((unsigned)row_tiles, (unsigned)tok_tiles), dim3(kTcThreads),
                    Cfg::kSmem, st, tx, tc, tm, absmax, gamma_eff, T, O, K, Y, y_is_bf16, acc_dbg,
                    err_flag);
}

template <int BN>
static sbn_status gemm_sp24_pair_t(const int8_t *Xq, const float *absmax, const uint8_t *codes,
                                   const uint8_t *meta, const float *gamma_eff, int64_t T,
                                   int64_t O, int64_t K, int64_t ldx, int64_t ldc, int64_t ldm, void *Y,
                                   int y_is_bf16, int32_t *acc_dbg, int32_t *err_flag,
                                   cudaStream_t st) {
  using Cfg = PairCfg<BN>;
  CUtensorMap tx, tc, tm;
  if (!encode_u8(&tx, Xq, K, T, ldx, Cfg::kKL, Cfg::kBHalf, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_u8(&tc, codes, K / 8, O, ldc, 16, kBM, CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !encode_u8(&tm, meta, K / 8, O, ldm, 16, kBM, CU_TENSOR_MAP_SWIZZLE_NONE))
    return SBN_ERR_CUDA;
  auto kern = k_gemm_sp24_pair<BN>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Cfg::kSmem) !=
      cudaSuccess)
    return SBN_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.blockDim = dim3(kPairThreads);
  cfg.dynamicSmemBytes = Cfg::kSmem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;  // the occupancy query takes the cluster shape only
  // as many pairs as can be resident at once (the kernel strides over the tiles); cached
  // per device
  constexpr int kMaxDevices = 64;
  static int pairs_cache[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    (void)cudaGetLastError();
    dev = 0;
  }
  int max_pairs = (dev >= 0 && dev < kMaxDevices) ? pairs_cache[dev] : 0;
  if (max_pairs == 0) {
    cfg.gridDim = dim3((unsigned)num_sms());
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n < 1) {
      (void)cudaGetLastError();
      n = num_sms() / 2;
    }
    max_pairs = n;
    if (dev >= 0 && dev < kMaxDevices) pairs_cache[dev] = n;
  }
  const int64_t ntiles = ((O + 2 * kBM - 1) / (2 * kBM)) * ((T + BN - 1) / BN);
  const int64_t npairs = ntiles < max_pairs ? ntiles : max_pairs;
  cfg.gridDim = dim3((unsigned)(2 * npairs));
  cfg.numAttrs = 2;  // and a programmatic dependent of the previous kernel
  if (cudaLaunchKernelEx(&cfg, kern, tx, tc, tm, absmax, gamma_eff, T, O, K, Y, y_is_bf16,
                         acc_dbg, err_flag) != cudaSuccess) {
    (void)cudaGetLastError();
    return SBN_ERR_CUDA;
  }
  return SBN_OK;
}

template <int BN>
static sbn_status gemm_tc_bn(bool compact, const int8_t *Xq, const float *absmax,
                             const uint8_t *codes, const uint8_t *meta, const float *gamma_eff,
                             int64_t T, int64_t O, int64_t K, int64_t ldx, int64_t ldc, int64_t ldm, void *Y,
                             int y_is_bf16, int32_t *acc_dbg, int32_t *err_flag, cudaStream_t st) {
  if (compact)
    return gemm_sp24_t<BN>(Xq, absmax, codes, meta, gamma_eff, T, O, K, ldx, ldc, ldm, Y, y_is_bf16,
                           acc_dbg, err_flag, st);
  return gemm_tc_t<BN, false>(Xq, absmax, codes, meta, gamma_eff, T, O, K, ldx, ldc, ldm, Y,
                              y_is_bf16, acc_dbg, err_flag, st);
}

sbn_status launch_gemm_tc(const int8_t *Xq, const float *absmax, const uint8_t *codes,
                          const uint8_t *meta, const float *gamma_eff, int64_t tokens,
                          int64_t out, int64_t in, int64_t ldx, int n, int m, int64_t ldc, int64_t ldm,
                          void *Y, int y_is_bf16, int32_t *acc_dbg, int32_t *err_flag,
                          cudaStream_t st) {
  const bool compact = (n == 2 && m == 4);
  if (compact && tokens > 128) {  // CTA pairs (every sm_100 device runs 2-CTA clusters)
    // tile width: 208 tokens, or 192 where that takes no more rounds of tiles over the
    // pairs (fewer activation bytes per tile; e.g. 4096 rows x 4096 tokens: 5 rounds either way)
    const int64_t pairs = num_sms() / 2 > 0 ? num_sms() / 2 : 1;
    const int64_t n_o = (out + 255) / 256;
    auto span = [&](int64_t bn) { return (n_o * ((tokens + bn - 1) / bn) + pairs - 1) / pairs * bn; };
    if (span(192) < span(208))
      return gemm_sp24_pair_t<192>(Xq, absmax, codes, meta, gamma_eff, tokens, out, in, ldx, ldc,
                                   ldm, Y, y_is_bf16, acc_dbg, err_flag, st);
    return gemm_sp24_pair_t<208>(Xq, absmax, codes, meta, gamma_eff, tokens, out, in, ldx, ldc, ldm, Y,
                                 y_is_bf16, acc_dbg, err_flag, st);
  }
  if (tokens > 128)
    return gemm_tc_bn<256>(compact, Xq, absmax, codes, meta, gamma_eff, tokens, out, in, ldx, ldc,
                           ldm, Y, y_is_bf16, acc_dbg, err_flag, st);
  if (tokens > 64)
    return gemm_tc_bn<128>(compact, Xq, absmax, codes, meta, gamma_eff, tokens, out, in, ldx, ldc,
                           ldm, Y, y_is_bf16, acc_dbg, err_flag, st);
  if (tokens > 32)
    return gemm_tc_bn<64>(compact, Xq, absmax, codes, meta, gamma_eff, tokens, out, in, ldx, ldc,
                          ldm, Y, y_is_bf16, acc_dbg, err_flag, st);
  if (tokens > 16)
    return gemm_tc_bn<32>(compact, Xq, absmax, codes, meta, gamma_eff, tokens, out, in, ldx, ldc,
                          ldm, Y, y_is_bf16, acc_dbg, err_flag, st);
  return gemm_tc_bn<16>(compact, Xq, absmax, codes, meta, gamma_eff, tokens, out, in, ldx, ldc, ldm,
                        Y, y_is_bf16, acc_dbg, err_flag, st);
}

}  // namespace sbn
