// Prefill contraction on a pre-expanded tensor-core operand (2:4).
//
// At many tokens the contraction is bound by the int8 tensor pipe, and any per-stage work
// between the weight load and the MMA (expanding 2-bit codes into int8 lanes) sits on the
// critical path of every pipeline stage.  Here the expansion is done once, ahead of the
// contraction, by k_expand_operand: the kept codes of each row become int8 values
// t in {-1, 0, 1} in K order, the compressed A operand of the sparse tensor cores
// ([out, in / 2] int8, 0.5 byte per weight).  The contraction then only moves tiles with
// TMA and issues MMAs:
//   k_gemm_sp24_operand<BN>: clusters of two CTAs (the two SMs of a pair), 256 weight rows x
//   BN tokens per tile, persistent over the tiles.  Per CTA (192 threads):
//     warp 0     TMA producer: per 128-deep K block its 128 rows of the operand (64 bytes
//                per row, 64-byte swizzle), its half of the activation tile (BN / 2 tokens,
//                128-byte swizzle) and its rows' metadata (16 bytes per row).
//     warp 1     CTA 0: metadata copies (tcgen05.cp) and the pair MMAs
//                (tcgen05.mma.sp.cta_group::2 kind::i8, M 256, N BN, two of logical K 64 per
//                block) into one of two TMEM accumulators; commits free the stage in both
//                CTAs.  CTA 1: relays "stage landed" of its own loads to CTA 0's barrier.
//     warps 2-5  epilogue: drain the accumulator of the previous tile while the next one
//                accumulates, rescale by c_t = fp32(fp32(g * s_t) / 127), store fp32/bf16.
// No TMA multicast; clusters only for the CTA pair.  Every wait is bounded (about 1 s) and
// raises SBN_FLAG_TIMEOUT through a shared abort flag; in-flight copies and MMAs are waited
// for and TMEM is freed on every path.
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

namespace sbn {

namespace {

constexpr long long kOpWaitCycles = 1ll << 31;
constexpr int kOpThreads = 192;
constexpr int kOpRows = 128;
constexpr int kOpKB = 128;

// ---- operand expansion -------------------------------------------------------------------

// The operand: rows padded to a multiple of 256 (one pair tile) and K to a multiple of 128
// (one K block), so the contraction's TMA loads never leave it:
//   A plane     int8 [O_pad][K_pad / 2]: the kept codes of each row as t in {-1, 0, 1}, in K
//               order; zero in the padding;
//   meta plane  uint8 [O_pad][K_pad / 8]: the pack's 2:4 metadata (i0 | i1 << 2 per group);
//               the valid index pair (0, 1) in the padding, whose codes are zero.
// One thread per (row, K block): 16 code bytes (64 kept codes) -> 64 int8 values, and the
// block's 16 metadata bytes.  Stored element e of a codes row lives in 32-bit word e / 16 at
// byte e % 4, bits 6 - 2j .. 7 - 2j with j = (e % 16) / 4; (word << 2j) & 0xC0C0C0C0 puts
// elements 4j .. 4j + 3 in the top two bits of four bytes, and per byte t = -sign | nonzero.
__global__ void __launch_bounds__(256)
    k_expand_operand(const uint8_t *__restrict__ codes, const uint8_t *__restrict__ meta,
                     int64_t O, int64_t K, int64_t ldc, int64_t ldm, int64_t kbp, int64_t total,
                     int8_t *__restrict__ A, uint8_t *__restrict__ M) {
  ptx::grid_dep_launch();
  ptx::grid_dep_wait();
  const int64_t lda = kbp * 64, ldmo = kbp * 16;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / kbp, kb = i - r * kbp;
    uint4 *dst = reinterpret_cast<uint4 *>(A + r * lda + kb * 64);
    uint4 *mdst = reinterpret_cast<uint4 *>(M + r * ldmo + kb * 16);
    if (r >= O || kb * 128 >= K) {
#pragma unroll
      for (int q = 0; q < 4; ++q) dst[q] = make_uint4(0u, 0u, 0u, 0u);
      *mdst = make_uint4(0x44444444u, 0x44444444u, 0x44444444u, 0x44444444u);
      continue;
    }
    // a last block with K % 128 == 64 reads the row's zero padding (the planes' rows are
    // padded to 16 bytes) for its second half
    const uint4 cw = __ldg(reinterpret_cast<const uint4 *>(codes + r * ldc + kb * 16));
    uint4 mw = __ldg(reinterpret_cast<const uint4 *>(meta + r * ldm + kb * 16));
    if (kb * 128 + 64 >= K) {
      mw.z = 0x44444444u;
      mw.w = 0x44444444u;
    }
    *mdst = mw;
    const uint32_t w[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t o[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t y = (w[q] << (2 * j)) & 0xC0C0C0C0u;
        const uint32_t nz = (y >> 6) & 0x01010101u, sg = (y >> 7) & 0x01010101u;
        o[j] = __vsub4(0u, sg) | nz;
      }
      dst[q] = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
}

// ---- the contraction ---------------------------------------------------------------------

template <int BN>
struct OpCfg {
  static constexpr int kBHalf = BN / 2;
  static constexpr int kABytes = kOpRows * kOpKB / 2;  // 8 KB
  static constexpr int kBBytes = kBHalf * kOpKB;
  static constexpr int kMBytes = kOpRows * 16;
  static constexpr int kStageBytes = kBBytes + kABytes + kMBytes;
  static constexpr int kBudget = 225 * 1024 - 1024;
  static constexpr int kFit = kBudget / kStageBytes;
  static constexpr int kStages = kFit > 12 ? 12 : kFit;
  static constexpr int kAccStride = 256;
  static constexpr int kGap = (256 - BN) / 4;
  static_assert(BN <= 256 && BN % 32 == 0, "pair tile width");
  static_assert(kBBytes % 1024 == 0 && kStageBytes % 1024 == 0, "swizzle alignment");
  static_assert(2 * kGap >= kStages, "two accumulators and the metadata fit in TMEM");
  static_assert(kStages >= 3, "pipeline depth");
  static constexpr int kTmemCols = 512;
  __device__ static constexpr uint32_t meta_col(int s) {
    return s < kGap ? (uint32_t)(BN + 4 * s) : (uint32_t)(kAccStride + BN + 4 * (s - kGap));
  }
  static constexpr uint32_t kTx = (uint32_t)kStageBytes;
  // barriers: full[S], peer[S], empty[S], acc_full[2], acc_empty[2], mma_done
  static constexpr size_t kSmem = 1024 + (size_t)kStages * kStageBytes +
                                  (size_t)(3 * kStages + 5) * 8 + 32 + (size_t)BN * 4;
};

__device__ __forceinline__ bool op_wait(uint64_t *bar, uint32_t parity, volatile int *abort) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    for (int i = 0; i < 64; ++i)
      if (ptx::mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if (clock64() - t0 > kOpWaitCycles) {
      *abort = 1;
      return false;
    }
  }
}

__device__ __forceinline__ bool op_drain(uint64_t *bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!ptx::mbar_try_wait(bar, parity))
    if (clock64() - t0 > kOpWaitCycles) return false;
  return true;
}

__device__ __forceinline__ bool op_bar_any(bool pred) {
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

// 32 columns of one output row: y_i = fp32(acc_i * c_i) for the first nt, stride O (a full
// chunk without per-column checks; the pointer advances by O per column).
__device__ __forceinline__ void op_store_y(float *p, float y) { *p = y; }
__device__ __forceinline__ void op_store_y(__nv_bfloat16 *p, float y) {
  *p = __float2bfloat16_rn(y);
}
template <typename Out>
__device__ __forceinline__ void op_store_chunk(const uint32_t *v, const float *sc, int nt, Out *p,
                                               int64_t O) {
  if (nt >= 32) {
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      op_store_y(p, __fmul_rn(__int2float_rn((int32_t)v[i]), sc[i]));
      p += O;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      if (i >= nt) break;
      op_store_y(p, __fmul_rn(__int2float_rn((int32_t)v[i]), sc[i]));
      p += O;
    }
  }
}

// Epilogue of one accumulator: warp quarter q holds rows 32q..32q+31 (TMEM lanes), column j
// is token t0 + j and holds the exact int32 sum; y = fp32(acc * c_t).
template <int BN>
__device__ __forceinline__ void op_store(uint32_t trow, const float *s_scale, int64_t o, int64_t O,
                                         int64_t t0, int64_t T, void *Y, int y_is_bf16,
                                         int32_t *acc_dbg) {
  const bool row_ok = o < O;
#pragma unroll 1
  for (int cb = 0; cb < BN; cb += 32) {
    uint32_t v[32];
    ptx::tmem_ld_32(trow + cb, v);
    ptx::tmem_ld_wait();
    if (!row_ok) continue;
    const int nt = (int)min(T - (t0 + cb), (int64_t)32);
    const int64_t off = (t0 + cb) * O + o;
    if (y_is_bf16)
      op_store_chunk(v, s_scale + cb, nt, reinterpret_cast<__nv_bfloat16 *>(Y) + off, O);
    else
      op_store_chunk(v, s_scale + cb, nt, reinterpret_cast<float *>(Y) + off, O);
    if (acc_dbg) {
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        if (i >= nt) break;
        acc_dbg[off + (int64_t)i * O] = (int32_t)v[i];
      }
    }
  }
}

template <int BN>
__global__ void __launch_bounds__(kOpThreads, 1)
    k_gemm_sp24_operand(const __grid_constant__ CUtensorMap tmap_x,
                        const __grid_constant__ CUtensorMap tmap_a,
                        const __grid_constant__ CUtensorMap tmap_m,
                        const float *__restrict__ absmax, const float *__restrict__ gamma_eff,
                        int64_t T, int64_t O, int64_t K, void *__restrict__ Y, int y_is_bf16,
                        int32_t *__restrict__ acc_dbg, int32_t *err_flag) {
  using Cfg = OpCfg<BN>;
  constexpr int S = Cfg::kStages;
  constexpr int kTileM = 2 * kOpRows;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *stages = smem;  // [S][B | A | meta]
  uint64_t *full = reinterpret_cast<uint64_t *>(stages + S * Cfg::kStageBytes);  // own loads
  uint64_t *peer = full + S;       // CTA 0: CTA 1's loads of the stage landed
  uint64_t *empty = peer + S;      // own stage free (commits from CTA 0)
  uint64_t *acc_full = empty + S;  // [2], own
  uint64_t *acc_empty = acc_full + 2;  // [2], CTA 0: the epilogue warps of both CTAs
  uint64_t *mma_done = acc_empty + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_done + 1);
  volatile int *s_abort = reinterpret_cast<volatile int *>(tmem_slot + 2);
  float *s_scale = reinterpret_cast<float *>(tmem_slot + 8);

  ptx::grid_dep_launch();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = ptx::cluster_ctarank();
  const int64_t pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int nkb = (int)((K + kOpKB - 1) / kOpKB);
  const int64_t n_o = (O + kTileM - 1) / kTileM, n_t = (T + BN - 1) / BN;
  const int64_t ntiles = n_o * n_t;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&peer[s], 1);
      ptx::mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(&acc_full[b], 1);
      ptx::mbar_init(&acc_empty[b], 8);
    }
    ptx::mbar_init(mma_done, 1);
    *s_abort = 0;
    ptx::fence_mbar_init();
  }
  ptx::cluster_sync();  // both CTAs' barriers exist before anyone arrives on a remote one
  if (warp == 1) {
    ptx::tmem_alloc_pair(tmem_slot, Cfg::kTmemCols);
    ptx::tmem_relinquish_pair();
  }
  ptx::grid_dep_wait();  // the previous kernel's outputs are visible
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t peer0 = ptx::mapa_shared(ptx::smem_u32(peer), 0);
  const uint32_t acc_empty0 = ptx::mapa_shared(ptx::smem_u32(acc_empty), 0);

  if (warp == 0) {
    // ---------------- TMA producer: this CTA's rows and half of the tokens ----------------
    if (lane == 0) {
      ptx::prefetch_tmap(&tmap_x);
      ptx::prefetch_tmap(&tmap_a);
      ptx::prefetch_tmap(&tmap_m);
      int64_t kg = 0, issued = 0;
      for (int64_t tile = pair; tile < ntiles && !*s_abort; tile += npairs) {
        const int32_t o0 = (int32_t)((tile % n_o) * kTileM + (int64_t)rank * kOpRows);
        const int32_t t0 = (int32_t)((tile / n_o) * BN + (int64_t)rank * Cfg::kBHalf);
        bool ok = true;
        for (int kb = 0; kb < nkb; ++kb, ++kg) {
          const int s = (int)(kg % S);
          const uint32_t ph = (uint32_t)(kg / S) & 1u;
          if (kg >= S && !op_wait(&empty[s], ph ^ 1u, s_abort)) {
            ok = false;
            break;
          }
          uint8_t *st = stages + s * Cfg::kStageBytes;
          ptx::mbar_arrive_expect_tx(&full[s], Cfg::kTx);
          ptx::tma_load_2d(st, &tmap_x, &full[s], kb * kOpKB, t0);
          ptx::tma_load_2d(st + Cfg::kBBytes, &tmap_a, &full[s], kb * (kOpKB / 2), o0);
          ptx::tma_load_2d(st + Cfg::kBBytes + Cfg::kABytes, &tmap_m, &full[s], kb * 16, o0);
          issued = kg + 1;
        }
        if (!ok) break;
      }
      for (int64_t q = issued - S < 0 ? 0 : issued - S; q < issued; ++q)
        if (!op_drain(&full[q % S], (uint32_t)(q / S) & 1u)) *s_abort = 1;
    }
  } else if (warp == 1) {
    if (rank == 1) {
      // ---------------- CTA 1: relay its stages' arrival to CTA 0 ----------------
      if (lane == 0) {
        int64_t kg = 0;
        for (int64_t tile = pair; tile < ntiles && !*s_abort; tile += npairs) {
          bool ok = true;
          for (int kb = 0; kb < nkb; ++kb, ++kg) {
            const int s = (int)(kg % S);
            if (!op_wait(&full[s], (uint32_t)(kg / S) & 1u, s_abort)) {
              ok = false;
              break;
            }
            ptx::mbar_arrive_cluster(peer0 + 8u * (uint32_t)s);
          }
          if (!ok) break;
        }
      }
    } else if (lane == 0) {
      // ---------------- CTA 0: metadata copies + pair MMAs ----------------
      constexpr uint32_t idesc = ptx::idesc_i8_sparse(kTileM, BN);
      int64_t kg = 0;
      int i = 0;
      for (int64_t tile = pair; tile < ntiles && !*s_abort; tile += npairs, ++i) {
        const int buf = i & 1;
        if (i >= 2 && !op_wait(&acc_empty[buf], ((uint32_t)(i >> 1) & 1u) ^ 1u, s_abort)) break;
        ptx::tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(buf * Cfg::kAccStride);
        bool ok = true;
        for (int kb = 0; kb < nkb; ++kb, ++kg) {
          const int s = (int)(kg % S);
          const uint32_t ph = (uint32_t)(kg / S) & 1u;
          if (!op_wait(&full[s], ph, s_abort) || !op_wait(&peer[s], ph, s_abort)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint8_t *st = stages + s * Cfg::kStageBytes;
          const uint32_t e_col = tmem + Cfg::meta_col(s);
          ptx::tmem_cp_128x128b_pair(
              e_col, ptx::smem_desc_rows16(ptx::smem_u32(st + Cfg::kBBytes + Cfg::kABytes)));
          const uint32_t a_addr = ptx::smem_u32(st + Cfg::kBBytes);
          const uint32_t b_addr = ptx::smem_u32(st);
#pragma unroll
          for (int k = 0; k < 2; ++k)
            ptx::mma_sp_i8_pair(d_tmem, ptx::smem_desc_sw64(a_addr + 32 * k),
                                ptx::smem_desc_sw128(b_addr + 64 * k), e_col + 2 * k, idesc,
                                (kb | k) != 0);
          ptx::mma_commit_pair(&empty[s], 0x3);
        }
        if (!ok) break;
        ptx::mma_commit_pair(&acc_full[buf], 0x3);
      }
      ptx::mma_commit_pair(mma_done, 0x1);
      if (!op_drain(mma_done, 0)) *s_abort = 1;
    }
  } else {
    // ---------------- epilogue (warps 2-5): this CTA's 128 rows ----------------
    const int q = warp & 3;
    const int et = threadIdx.x - 2 * 32;
    const float g = __ldg(gamma_eff);
    bool failed = false;
    int i = 0;
    for (int64_t tile = pair; tile < ntiles; tile += npairs, ++i) {
      const int buf = i & 1;
      const int64_t o0 = (tile % n_o) * kTileM + (int64_t)rank * kOpRows;
      const int64_t t0 = (tile / n_o) * BN;
      if (op_bar_any(failed)) break;
      for (int c = et; c < BN; c += 128) {
        const int64_t t = t0 + c;
        s_scale[c] = t < T ? rescale_factor(g, __ldg(absmax + t)) : 0.0f;
      }
      asm volatile("bar.sync 1, 128;" ::: "memory");
      failed = !__all_sync(0xffffffffu, !*s_abort && op_wait(&acc_full[buf],
                                                              (uint32_t)(i >> 1) & 1u, s_abort));
      ptx::tc_fence_after();
      if (!failed) {
        const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * Cfg::kAccStride);
        op_store<BN>(trow, s_scale, o0 + q * 32 + lane, O, t0, T, Y, y_is_bf16, acc_dbg);
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive_cluster(acc_empty0 + 8u * (uint32_t)buf);
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && *s_abort && err_flag) atomicOr(err_flag, SBN_FLAG_TIMEOUT);
  // neither CTA frees its TMEM or leaves while the pair's MMAs may still use it
  ptx::cluster_sync();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc_pair(tmem, Cfg::kTmemCols);
  }
}

}  // namespace

int64_t operand_rows(int64_t out) { return (out + 255) / 256 * 256; }
int64_t operand_kblocks(int64_t in) { return (in + 127) / 128; }
int64_t operand_bytes(int64_t out, int64_t in) {
  return operand_rows(out) * operand_kblocks(in) * (64 + 16);
}

sbn_status launch_expand_operand(const uint8_t *codes, const uint8_t *meta, int64_t out,
                                 int64_t in, int64_t ldc, int64_t ldm, void *operand,
                                 cudaStream_t st) {
  const int64_t rows = operand_rows(out), kbp = operand_kblocks(in);
  const int64_t total = rows * kbp;
  int64_t grid = (total + 255) / 256;
  const int64_t cap = (int64_t)num_sms() * 8;
  if (grid > cap) grid = cap;
  int8_t *A = static_cast<int8_t *>(operand);
  uint8_t *M = reinterpret_cast<uint8_t *>(A + rows * kbp * 64);
  return launch_pdl(k_expand_operand, dim3((unsigned)grid), dim3(256), 0, st, codes, meta, out,
                    in, ldc, ldm, kbp, total, A, M);
}

sbn_status launch_gemm_operand(const int8_t *Xq, const float *absmax, const void *operand,
                               const float *gamma_eff, int64_t T, int64_t O, int64_t K, void *Y,
                               int y_is_bf16, int32_t *acc_dbg, int32_t *err_flag,
                               cudaStream_t st) {
  constexpr int BN = 224;
  using Cfg = OpCfg<BN>;
  const int64_t rows = operand_rows(O), kbp = operand_kblocks(K);
  const int8_t *A = static_cast<const int8_t *>(operand);
  const uint8_t *M = reinterpret_cast<const uint8_t *>(A + rows * kbp * 64);
  CUtensorMap tx, ta, tm;
  if (!encode_u8(&tx, Xq, K, T, K, kOpKB, Cfg::kBHalf, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_u8(&ta, A, kbp * 64, rows, kbp * 64, kOpKB / 2, kOpRows,
                 CU_TENSOR_MAP_SWIZZLE_64B) ||
      !encode_u8(&tm, M, kbp * 16, rows, kbp * 16, 16, kOpRows, CU_TENSOR_MAP_SWIZZLE_NONE))
    return SBN_ERR_CUDA;
  auto kern = k_gemm_sp24_operand<BN>;
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
  cfg.blockDim = dim3(kOpThreads);
  cfg.dynamicSmemBytes = Cfg::kSmem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;  // the occupancy query takes the cluster shape only
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
      return SBN_ERR_CUDA;  // the device cannot run this cluster shape
    }
    max_pairs = n;
    if (dev >= 0 && dev < kMaxDevices) pairs_cache[dev] = n;
  }
  const int64_t ntiles = (rows / (2 * kOpRows)) * ((T + BN - 1) / BN);
  const int64_t npairs = ntiles < max_pairs ? ntiles : max_pairs;
  cfg.gridDim = dim3((unsigned)(2 * npairs));
  cfg.numAttrs = 2;
  if (cudaLaunchKernelEx(&cfg, kern, tx, ta, tm, absmax, gamma_eff, T, O, K, Y, y_is_bf16,
                         acc_dbg, err_flag) != cudaSuccess) {
    (void)cudaGetLastError();
    return SBN_ERR_CUDA;
  }
  return SBN_OK;
}

}  // namespace sbn
