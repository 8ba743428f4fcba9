// Grouped small-batch contraction: Y_p = (Xq_p . Ws_p^T) * c_t for many independent 2:4
// Sparse-BitLinear layers p of at most 32 tokens each, in ONE persistent launch on the
// sparse tensor cores (tcgen05.mma.sp kind::i8, int32 accumulators in TMEM).
//
// At a few tokens per layer the contraction streams the packed weights (0.25 bytes per
// weight) from HBM and does little arithmetic per byte, so what matters is that every SM
// keeps enough weight bytes in flight and that no launch, pipeline fill or drain repeats
// per layer.  The host plan (sbn_group_plan) cuts every layer into work units of 128 weight
// rows x a range of 128-deep K blocks and gives each CTA (one per SM) a contiguous run of
// units with about the same number of K blocks; the CTA walks its run as one pipeline in
// super-blocks of four 128-deep K blocks (every hand-off between the roles has a fixed cost,
// so each one moves four blocks):
//   warps 4, 15  two TMA producers on alternate super-blocks, each into its own half of ring 1
//              (the HBM stream, 6-8 slots; the issue of a TMA copy, not the copy engine,
//              limits one thread): per
//              super-block the packed
//              codes and the metadata of the unit's 128 rows as two boxes of 64 bytes x 128
//              rows (64-byte swizzle), and the four activation tiles (bn tokens x 128 inputs,
//              128-byte swizzle; L2 hits, all row tiles of a layer share them).
//   warps 0-3, 10-13  two groups of expanders taking alternate super-blocks, ring 2 in TMEM
//              (4 slots): thread r turns row r's kept codes into 64 int8 lanes of 64 * t per
//              block (the compressed A tile) and writes them with the block's metadata
//              (groups outside the matrix get the valid index pair (0, 1)) into TMEM lane r
//              with tcgen05.st; one wait and one arrival per super-block.  A never passes
//              through shared memory, and no tcgen05.cp is needed.
//   warps 5, 14, 16, 17  MMA threads (four at bn 16, two at bn 32) taking every fourth
//              (second) super-block (the issue of a tcgen05.mma of this small shape, not the
//              tensor pipe, sets the pace of one thread): per block two sparse MMAs (M 128,
//              N bn, logical K 64 each; A and the metadata read from TMEM, B from shared
//              memory) into the thread's accumulator chain(s); one commit frees both rings'
//              slots per super-block; at a unit's end all commit its accumulators to the
//              epilogue and the next unit starts in the other set (warp 5 also allocates
//              TMEM).  Every role picks super-blocks by the CTA's running counter, so each
//              ring slot has one producer and one consumer.
//   warps 6-9  epilogue: drain and add the chains (tcgen05.ld), release them, rescale by
//              c_t = fp32(fp32(g * s_t) / 127) and store fp32 or bf16.  The unit's layer
//              record and scales are fetched ahead (software-pipelined over the units), so
//              short units (K slices) do not wait on those loads after each drain.  A row tile whose K
//              blocks were split over several units writes its int32 partial to the
//              workspace; the unit that arrives last on the tile's counter adds the others
//              (integer sums: the split changes no result bit), stores the tile and resets
//              the counter to zero for the next call.
// Every mbarrier wait gives up after about a second and raises SBN_FLAG_TIMEOUT; a shared
// abort flag then ends every role's loop, in-flight copies and MMAs are waited for
// (bounded) and TMEM is freed.
#include <cuda.h>
#include <cuda_bf16.h>

#include <vector>

#include "common.cuh"
#include "group.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

namespace sbn {

namespace {

// 18 warps: two expander groups, two TMA producers, up to four MMA threads, the epilogue
constexpr int kGrpThreads = 576;
constexpr long long kGrpWaitCycles = 1ll << 31;  // about 1 s at 1.9 GHz
constexpr int kSuper = 4;  // K blocks per weight super-block (one 64-byte box per row)

template <int BN>
struct GrpCfg {
  // ring 1 in shared memory (the HBM stream), one slot per super-block of four 128-deep K
  // blocks: the packed codes and the metadata of 128 rows (64 bytes per row each, 64-byte
  // swizzle) and the four activation tiles (bn tokens x 128 inputs each, 128-byte swizzle)
  static constexpr int kPlane = kGroupRows * 16 * kSuper;  // 8 KB
  static constexpr int kBBytes = BN * kGroupKB;
  static constexpr int kSlot1 = 2 * kPlane + kSuper * kBBytes;
  static constexpr int kD1 = BN <= 16 ? 8 : 6;  // even: half the slots per producer
  // ring 2 in TMEM, one slot per super-block: per block the compressed A tile (lane r = row r,
  // 16 columns of four int8 values) and the metadata (4 columns)
  static constexpr int kD2 = BN <= 16 ? 4 : 2;
  static_assert(kD1 % (BN <= 16 ? 4 : 2) == 0 && kD2 % (BN <= 16 ? 4 : 2) == 0,
                "one consumer per ring slot: ring depths are multiples of the MMA threads");
  // kMma MMA threads take every kMma-th super-block (by the running counter, as the
  // producers and expanders do): each ring slot keeps one consumer because both rings'
  // depths are multiples of kMma.  Four threads at 16 tokens (each MMA of N 16 is short and
  // one thread issues one per ~100 cycles), two at 32 (the TMEM ring has two slots there).
  static constexpr int kMma = BN <= 16 ? 4 : 2;
  // accumulator chains per unit: each MMA thread owns kChains / kMma of them (block b of its
  // super-blocks into chain b mod kCpt); the epilogue adds the chains
  static constexpr int kChains = 4;
  static constexpr int kCpt = kChains / kMma;  // chains per MMA thread
  static constexpr int kAccCols = kChains * BN;         // one unit's accumulators
  static constexpr int kACol = 2 * kAccCols;            // A ring after the two units' accumulators
  static constexpr int kAColsPerSlot = kSuper * 16;
  static constexpr int kMetaCol = kACol + kD2 * kAColsPerSlot;
  static constexpr int kMColsPerSlot = kSuper * 4;
  static constexpr int kTmemCols = 512;
  static constexpr int kBars = 2 * kD1 + 2 * kD2 + 5;
  // this CTA's unit records, staged in shared memory at the start (units past the first
  // kUnitCache are read from global memory)
  static constexpr int kUnitCache = 256;
  static constexpr size_t kSmem = 1024 + (size_t)kD1 * kSlot1 + (size_t)kBars * 8 + 64 +
                                  (size_t)kUnitCache * sizeof(GroupUnit);
  static_assert(kSlot1 % 1024 == 0 && kBBytes % 1024 == 0, "tile alignment");
  static_assert(kMetaCol + kD2 * kMColsPerSlot <= kTmemCols, "TMEM columns");
  static_assert(kSmem <= 227 * 1024, "shared memory budget");
};

__device__ __forceinline__ bool grp_wait(uint64_t *bar, uint32_t parity, volatile int *abort) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    for (int i = 0; i < 64; ++i)
      if (ptx::mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if (clock64() - t0 > kGrpWaitCycles) {
      *abort = 1;
      return false;
    }
  }
}

// Bounded wait that ignores the abort flag: used to let in-flight copies and MMAs finish
// before the CTA exits.
__device__ __forceinline__ bool grp_drain(uint64_t *bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!ptx::mbar_try_wait(bar, parity))
    if (clock64() - t0 > kGrpWaitCycles) return false;
  return true;
}

__device__ __forceinline__ bool grp_bar_any(bool pred) {
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

__device__ __forceinline__ void grp_bar_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// Ring 1 is filled by two producers, super-block js by producer js % 2 into its own half of
// the slots (even / odd): no slot is ever shared between them, so each producer's copies and
// phases stay its own.  H = D1 / 2 slots per producer.
template <int D1>
__device__ __forceinline__ int ring1_slot(int64_t js) {
  return 2 * (int)((js >> 1) % (D1 / 2)) + (int)(js & 1);
}
template <int D1>
__device__ __forceinline__ uint32_t ring1_phase(int64_t js) {
  return (uint32_t)((js >> 1) / (D1 / 2)) & 1u;
}

template <int BN>
__global__ void __launch_bounds__(kGrpThreads, 1)
    k_gemm_group(const uint8_t *__restrict__ plan, uint8_t *__restrict__ ws,
                 int32_t *err_flag) {
  using Cfg = GrpCfg<BN>;
  constexpr int D1 = Cfg::kD1, D2 = Cfg::kD2, C = Cfg::kChains;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *ring1 = smem;  // [D1][codes | meta | 4 x B]
  uint64_t *full1 = reinterpret_cast<uint64_t *>(ring1 + D1 * Cfg::kSlot1);
  uint64_t *empty1 = full1 + D1;
  uint64_t *full2 = empty1 + D1;
  uint64_t *empty2 = full2 + D2;
  uint64_t *acc_full = empty2 + D2;   // [2]
  uint64_t *acc_empty = acc_full + 2;  // [2]
  uint64_t *mma_done = acc_empty + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_done + 1);
  volatile int *s_abort = reinterpret_cast<volatile int *>(tmem_slot + 2);
  volatile int *s_last = reinterpret_cast<volatile int *>(tmem_slot + 4);
  GroupUnit *s_units = reinterpret_cast<GroupUnit *>(tmem_slot + 16);  // 64 bytes past the slot

  ptx::grid_dep_launch();
  const GroupHeader &hd = *reinterpret_cast<const GroupHeader *>(plan);
  const GroupProb *probs = reinterpret_cast<const GroupProb *>(plan + hd.off_probs);
  const GroupUnit *units = reinterpret_cast<const GroupUnit *>(plan + hd.off_units);
  const int32_t *cta_begin = reinterpret_cast<const int32_t *>(plan + hd.off_cta);
  const int u0 = cta_begin[blockIdx.x], u1 = cta_begin[blockIdx.x + 1];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // the plan is written before the launch (not by the previous kernel): read it early
  const int ncache = min(u1 - u0, Cfg::kUnitCache);
  for (int i = threadIdx.x; i < ncache * 8; i += blockDim.x)
    reinterpret_cast<int32_t *>(s_units)[i] = reinterpret_cast<const int32_t *>(units + u0)[i];
  auto unit = [&](int u) -> GroupUnit {
    return u - u0 < Cfg::kUnitCache ? s_units[u - u0] : units[u];
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < D1; ++s) {
      ptx::mbar_init(&full1[s], 1);
      ptx::mbar_init(&empty1[s], 1);
    }
    for (int s = 0; s < D2; ++s) {
      ptx::mbar_init(&full2[s], 4);
      ptx::mbar_init(&empty2[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(&acc_full[b], Cfg::kMma);  // every MMA thread commits
      ptx::mbar_init(&acc_empty[b], 4);
    }
    ptx::mbar_init(mma_done, Cfg::kMma);
    *s_abort = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 5) {
    ptx::tmem_alloc(tmem_slot, Cfg::kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::grid_dep_wait();  // the activation quantiser's Xq and scales are visible
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < 4 || (warp >= 10 && warp < 14)) {
    // ---------------- expanders: two groups of four warps take alternate super-blocks;
    // warp w writes TMEM lanes 32 (w mod 4) .. + 31, i.e. tile rows of that quarter ----------
    const int grp = warp < 4 ? 0 : 1;
    const int qw = warp & 3;
    const int r = qw * 32 + lane;  // tile row
    const int swz = (r >> 1) & 3;  // 64-byte swizzle of row r's 16-byte chunks
    int64_t js = 0;  // super-block counter over this CTA's units
    bool stop = false;
    for (int u = u0; u < u1 && !stop; ++u) {
      const GroupUnit un = unit(u);
      const bool row_ok = un.row_tile * kGroupRows + r < un.O;
      const int64_t K = un.K;
      for (int b0 = 0; b0 < un.nkb; b0 += kSuper, ++js) {
        if ((int)(js & 1) != grp) continue;
        const int s1 = ring1_slot<D1>(js), s2 = (int)(js % D2);
        const uint32_t ph1 = ring1_phase<D1>(js), ph2 = (uint32_t)(js / D2) & 1u;
        const bool ok = grp_wait(&full1[s1], ph1, s_abort) &&
                        (js < D2 || grp_wait(&empty2[s2], ph2 ^ 1u, s_abort));
        if (!__all_sync(0xffffffffu, ok)) {
          stop = true;
          break;
        }
        const int nb = min(kSuper, un.nkb - b0);
        const uint8_t *slot1 = ring1 + s1 * Cfg::kSlot1;
        const uint32_t lrow = ((uint32_t)(qw * 32)) << 16;  // this warp's TMEM lanes
#pragma unroll
        for (int g = 0; g < kSuper; ++g) {
          if (g >= nb) break;
          const int off = r * 64 + ((g ^ swz) << 4);
          const uint4 cw = *reinterpret_cast<const uint4 *>(slot1 + off);
          uint4 m4 = *reinterpret_cast<const uint4 *>(slot1 + Cfg::kPlane + off);
          // metadata groups outside the matrix (rows >= O, or the second half of a last
          // block with K % 128 == 64) were zero-filled by the TMA: give them the valid index
          // pair (0, 1); their codes are zero
          if (!row_ok) {
            m4 = make_uint4(0x44444444u, 0x44444444u, 0x44444444u, 0x44444444u);
          } else if ((int64_t)(un.kb0 + b0 + g) * kGroupKB + 64 >= K) {
            m4.z = 0x44444444u;
            m4.w = 0x44444444u;
          }
          ptx::tmem_st_4(tmem + lrow + (uint32_t)(Cfg::kMetaCol + s2 * Cfg::kMColsPerSlot + 4 * g),
                         m4);
          // 16 kept codes per word -> 16 int8 lanes of 64 * t, in K order: column 4c + q holds
          // the four values (w[c] << 2q) & 0xC0C0C0C0
          const uint32_t w[4] = {cw.x, cw.y, cw.z, cw.w};
          uint32_t a[16];
#pragma unroll
          for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int q = 0; q < 4; ++q) a[4 * c + q] = (w[c] << (2 * q)) & 0xC0C0C0C0u;
          ptx::tmem_st_16(tmem + lrow + (uint32_t)(Cfg::kACol + s2 * Cfg::kAColsPerSlot + 16 * g),
                          a);
        }
        ptx::tmem_st_wait();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&full2[s2]);
      }
    }
  } else if (warp == 4 || warp == 15) {
    // ---------------- two TMA producers (ring 1: packed weights + activation tiles), taking
    // alternate super-blocks: the issue of a TMA copy, not the copy engine, sets the pace of
    // one thread ----------------
    if (lane == 0) {
      const int pt = warp == 4 ? 0 : 1;  // super-blocks js with js % 2 == pt
      int64_t js = 0, issued = -1;
      int last_prob = -1;
      for (int u = u0; u < u1 && !*s_abort; ++u) {
        const GroupUnit un = unit(u);
        const GroupProb &p = probs[un.prob];  // address only: the tensor maps stay in global memory
        if (un.prob != last_prob) {
          ptx::prefetch_tmap(&p.tc);
          ptx::prefetch_tmap(&p.tm);
          ptx::prefetch_tmap(&p.tx);
          last_prob = un.prob;
        }
        const int32_t row0 = un.row_tile * kGroupRows;
        bool ok = true;
        for (int b0 = 0; b0 < un.nkb; b0 += kSuper, ++js) {
          if ((int)(js & 1) != pt) continue;
          const int s1 = ring1_slot<D1>(js);
          const uint32_t ph1 = ring1_phase<D1>(js);
          if (js >= D1 && !grp_wait(&empty1[s1], ph1 ^ 1u, s_abort)) {
            ok = false;
            break;
          }
          const int nb = min(kSuper, un.nkb - b0);
          const int32_t kb = un.kb0 + b0;
          uint8_t *slot = ring1 + s1 * Cfg::kSlot1;
          ptx::mbar_arrive_expect_tx(&full1[s1], (uint32_t)(2 * Cfg::kPlane + nb * Cfg::kBBytes));
          ptx::tma_load_2d(slot, &p.tc, &full1[s1], kb * 16, row0);
          ptx::tma_load_2d(slot + Cfg::kPlane, &p.tm, &full1[s1], kb * 16, row0);
          for (int g = 0; g < nb; ++g)
            ptx::tma_load_2d(slot + 2 * Cfg::kPlane + g * Cfg::kBBytes, &p.tx, &full1[s1],
                             (kb + g) * kGroupKB, 0);
          issued = js;  // the last super-block this thread issued
        }
        if (!ok) break;
      }
      // every copy this thread issued lands before the CTA can exit (bounded, also after an
      // abort): the last D1 / 2 super-blocks it issued, one per slot of its half
      for (int64_t q = issued, i = 0; q >= 0 && i < D1 / 2; q -= 2, ++i)
        if (!grp_drain(&full1[ring1_slot<D1>(q)], ring1_phase<D1>(q))) *s_abort = 1;
    }
  } else if (warp == 5 || warp == 14 || warp >= 16) {
    // ---------------- kMma sparse-MMA threads (warps 5, 14, 16, 17) ----------------
    // Thread mt takes the super-blocks js with js % kMma == mt, so every ring slot has one
    // consumer and its uses stay in order.  Within a unit its first super-block is then one
    // of js0 .. js0 + kMma - 1 (js0: the unit's first); that one starts its chains.
    const int mt = warp == 5 ? 0 : warp == 14 ? 1 : warp - 14;
    if (lane == 0 && mt < Cfg::kMma) {
      constexpr uint32_t idesc = ptx::idesc_i8_sparse(kGroupRows, BN);
      int64_t js = 0;
      int i = 0;
      for (int u = u0; u < u1 && !*s_abort; ++u, ++i) {
        const int nkb = unit(u).nkb;
        const int64_t js0 = js;
        const int buf = i & 1;
        if (i >= 2 && !grp_wait(&acc_empty[buf], ((uint32_t)(i >> 1) & 1u) ^ 1u, s_abort))
          break;
        ptx::tc_fence_after();
        const uint32_t acc0 = tmem + (uint32_t)(buf * Cfg::kAccCols);
        bool ok = true;
        for (int b0 = 0; b0 < nkb; b0 += kSuper, ++js) {
          if ((int)(js % Cfg::kMma) != mt) continue;
          const int s1 = ring1_slot<D1>(js), s2 = (int)(js % D2);
          const uint32_t ph1 = ring1_phase<D1>(js), ph2 = (uint32_t)(js / D2) & 1u;
          if (!grp_wait(&full2[s2], ph2, s_abort) || !grp_wait(&full1[s1], ph1, s_abort)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint8_t *slot1 = ring1 + s1 * Cfg::kSlot1;
          const int nb = min(kSuper, nkb - b0);
          for (int g = 0; g < nb; ++g) {
            const uint32_t e_col = tmem + (uint32_t)(Cfg::kMetaCol + s2 * Cfg::kMColsPerSlot + 4 * g);
            const uint32_t a_col = tmem + (uint32_t)(Cfg::kACol + s2 * Cfg::kAColsPerSlot + 16 * g);
            const uint32_t b_addr = ptx::smem_u32(slot1 + 2 * Cfg::kPlane + g * Cfg::kBBytes);
            const uint32_t d = acc0 + (uint32_t)((mt * Cfg::kCpt + g % Cfg::kCpt) * BN);
            // the first blocks of this thread's first super-block of the unit start its chains
            const bool first = js - js0 < Cfg::kMma && g < Cfg::kCpt;
#pragma unroll
            for (int k = 0; k < 2; ++k)  // logical K 64 per MMA: 8 columns of A, 64 bytes of B
              ptx::mma_sp_i8_tmem_a(d, a_col + 8 * k, ptx::smem_desc_sw128(b_addr + 64 * k),
                                    e_col + 2 * k, idesc, (!first || k != 0) ? 1u : 0u);
          }
          ptx::mma_commit(&empty2[s2]);
          ptx::mma_commit(&empty1[s1]);
        }
        if (!ok) break;
        ptx::mma_commit(&acc_full[buf]);
      }
      // every MMA issued has completed before TMEM can be released (also after an abort)
      ptx::mma_commit(mma_done);
      if (!grp_drain(mma_done, 0)) *s_abort = 1;
    }
  } else {
    // ---------------- epilogue (warps 6-9) ----------------
    const int q = warp & 3;  // the TMEM lane quarter this warp may read
    const int et = q * 32 + lane;  // tile row
    const uint64_t part_off = (uint64_t)hd.ws_part_off;
    bool failed = false;
    int i = 0;
    int64_t js = 0;  // the super-block counter of the MMA threads
    // A unit's output description and scales are two pointer chases through the plan (the
    // layer record, then g and s_t), two L2 round trips that would otherwise sit between the
    // drain of one unit and the next.  At 16 tokens the record of unit u + 2 is loaded while
    // unit u is handled, and the scales of unit u + 1; at 32 tokens (no registers to spare
    // for that) both are loaded before the wait for the unit's accumulators.
    struct EpiRec {
      const float *absmax = nullptr, *gamma = nullptr;
      void *Y = nullptr;
      int32_t *acc_dbg = nullptr;
      int32_t T = 0, O = 0;  // at most 32 tokens; rows < 2^31 (checked by the plan)
      int32_t y_is_bf16 = 0, nparts = 1;
    };
    auto load_rec = [&](int u) {
      EpiRec r;
      if (u < u1) {
        const GroupProb &pp = probs[unit(u).prob];
        r.absmax = pp.absmax;
        r.gamma = pp.gamma_eff;
        r.Y = pp.Y;
        r.acc_dbg = pp.acc_dbg;
        r.T = (int32_t)pp.T;
        r.O = (int32_t)pp.O;
        r.y_is_bf16 = pp.y_is_bf16;
        r.nparts = pp.nparts;
      }
      return r;
    };
    auto load_scales = [&](const EpiRec &r, float &g, float &sa) {
      g = r.gamma ? __ldg(r.gamma) : 0.0f;
      sa = r.gamma && lane < r.T ? __ldg(r.absmax + lane) : 0.0f;
    };
    constexpr bool kAhead = BN <= 16;
    EpiRec rn, rnn;
    float gn = 0.0f, sn = 0.0f;
    if constexpr (kAhead) {
      rn = load_rec(u0);
      rnn = load_rec(u0 + 1);
      load_scales(rn, gn, sn);
    }
    for (int u = u0; u < u1; ++u, ++i) {
      const int buf = i & 1;
      // this unit's record and scales (and the loads for the next two units')
      EpiRec rc;
      float g, sa;
      if constexpr (kAhead) {
        rc = rn;
        g = gn;
        sa = sn;
        rn = rnn;
        rnn = load_rec(u + 2);
        load_scales(rn, gn, sn);
      } else {
        rc = load_rec(u);
        load_scales(rc, g, sa);
      }
      // all four warps stop together if any wait of the previous unit gave up
      if (grp_bar_any(failed)) break;
      const GroupUnit un = unit(u);
      const GroupProb &p = probs[un.prob];
      const int js0m = (int)(js % Cfg::kMma);  // the unit's first super-block, mod kMma
      js += (un.nkb + kSuper - 1) / kSuper;
      const int64_t T = rc.T, O = rc.O;
      const int y_is_bf16 = rc.y_is_bf16;
      void *const Yp = rc.Y;
      int32_t *const acc_dbg = rc.acc_dbg;
      const float c_lane = lane < T ? rescale_factor(g, sa) : 0.0f;
      failed = !__all_sync(0xffffffffu, !*s_abort && grp_wait(&acc_full[buf],
                                                              (uint32_t)(i >> 1) & 1u, s_abort));
      ptx::tc_fence_after();
      int32_t a[BN];
#pragma unroll
      for (int x = 0; x < BN; ++x) a[x] = 0;
      if (!failed) {
        const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * Cfg::kAccCols);
#pragma unroll
        for (int ch = 0; ch < C; ++ch) {
          // chain ch belongs to MMA thread t = ch / kCpt, whose first super-block of the unit
          // is the unit's local super-block (t - js0) mod kMma, and starts at its block
          // r = ch % kCpt
          const int jt = ((ch / Cfg::kCpt) - js0m + Cfg::kMma) % Cfg::kMma;
          if (kSuper * jt + ch % Cfg::kCpt >= un.nkb) continue;
#pragma unroll
          for (int c = 0; c < BN; c += 16) {
            uint32_t v[16];
            ptx::tmem_ld_16(taddr + ch * BN + c, v);
            ptx::tmem_ld_wait();
#pragma unroll
            for (int x = 0; x < 16; ++x) a[c + x] += (int32_t)v[x];
          }
        }
#pragma unroll
        for (int x = 0; x < BN; ++x) a[x] >>= 6;  // exact: the sums hold 64 * acc
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&acc_empty[buf]);
      if (grp_bar_any(failed)) {
        failed = true;
        break;
      }
      if (rc.nparts > 1) {
        // K split: publish this part, and let the last part to arrive finish the tile
        int32_t *parts = reinterpret_cast<int32_t *>(ws + part_off) +
                         (p.part_base + (int64_t)un.row_tile * p.nparts) * (kGroupRows * BN);
        unsigned int *ticket = reinterpret_cast<unsigned int *>(ws) + p.ticket_base + un.row_tile;
        int4 *mine = reinterpret_cast<int4 *>(parts + (int64_t)un.part * (kGroupRows * BN) +
                                              (int64_t)et * BN);
#pragma unroll
        for (int c = 0; c < BN; c += 4) __stcg(mine + c / 4, make_int4(a[c], a[c + 1], a[c + 2], a[c + 3]));
        __threadfence();
        grp_bar_sync();
        if (et == 0) *s_last = (atomicAdd(ticket, 1u) == (unsigned)(p.nparts - 1)) ? 1 : 0;
        grp_bar_sync();
        const bool last = *s_last != 0;
        if (!last) continue;
        __threadfence();
        for (int pt = 0; pt < p.nparts; ++pt) {
          if (pt == un.part) continue;
          const int4 *other = reinterpret_cast<const int4 *>(parts + (int64_t)pt * (kGroupRows * BN) +
                                                             (int64_t)et * BN);
#pragma unroll
          for (int c = 0; c < BN; c += 4) {
            const int4 o4 = __ldcg(other + c / 4);
            a[c] += o4.x, a[c + 1] += o4.y, a[c + 2] += o4.z, a[c + 3] += o4.w;
          }
        }
        if (et == 0) *ticket = 0u;  // ready for the next call
      }
      // rescale and store: lane t holds c_t for token t
      const int64_t o = (int64_t)un.row_tile * kGroupRows + et;
      float *yf = reinterpret_cast<float *>(Yp) + o;
      __nv_bfloat16 *yb = reinterpret_cast<__nv_bfloat16 *>(Yp) + o;
#pragma unroll
      for (int t = 0; t < BN; ++t) {
        const float c = __shfl_sync(0xffffffffu, c_lane, t);
        if (t < T && o < O) {
          const float y = __fmul_rn(__int2float_rn(a[t]), c);
          if (y_is_bf16)
            yb[(int64_t)t * O] = __float2bfloat16_rn(y);
          else
            yf[(int64_t)t * O] = y;
          if (acc_dbg) acc_dbg[(int64_t)t * O + o] = a[t];
        }
      }
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && *s_abort && err_flag) atomicOr(err_flag, SBN_FLAG_TIMEOUT);
  if (warp == 5) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, Cfg::kTmemCols);
  }
}

int64_t align_up(int64_t x, int64_t a) { return (x + a - 1) / a * a; }

struct PlanShape {
  int bn = 16;
  int split = 1;
  int64_t nunits = 0, nrows = 0, ntickets = 0, nparts_tiles = 0;
  int ncta = 0;
  int32_t max_nv = 0;
  bool has_x = true;
};

// Linear partition of the units (in order) over at most `ncta` CTAs so that every CTA gets
// about the same number of K blocks; returns the largest per-CTA cost (blocks + a fixed
// cost per unit) and fills `begin` (ncta + 1 entries, may end with empty CTAs trimmed).
int64_t partition_units(const std::vector<int32_t> &nkb, int ncta, int64_t unit_cost,
                        std::vector<int32_t> *begin) {
  int64_t total = 0;
  for (int32_t b : nkb) total += b + unit_cost;
  const int64_t n = (int64_t)nkb.size();
  if (ncta > n) ncta = (int)n;
  if (begin) begin->assign(1, 0);
  int64_t worst = 0, cum = 0, cur = 0;
  int c = 0;
  for (int64_t u = 0; u < n; ++u) {
    const int64_t w = nkb[u] + unit_cost;
    // start a new CTA when this unit's midpoint lies past the current CTA's share
    if (cur > 0 && c + 1 < ncta && 2 * (cum + w / 2) >= 2 * total * (c + 1) / ncta) {
      worst = cur > worst ? cur : worst;
      if (begin) begin->push_back((int32_t)u);
      ++c;
      cur = 0;
    }
    cur += w;
    cum += w;
  }
  worst = cur > worst ? cur : worst;
  if (begin) begin->push_back((int32_t)n);
  return worst;
}

void build_units(const sbn_group_linear *lins, int count, int split,
                 std::vector<GroupUnit> *units) {
  units->clear();
  for (int p = 0; p < count; ++p) {
    const sbn_group_linear &l = lins[p];
    if (l.tokens == 0) continue;
    const int nkb = (int)((l.in + kGroupKB - 1) / kGroupKB);
    const int parts = split < nkb ? split : nkb;
    const int tiles = (int)((l.out + kGroupRows - 1) / kGroupRows);
    for (int t = 0; t < tiles; ++t)
      for (int q = 0; q < parts; ++q) {
        GroupUnit u = {};
        u.prob = p;
        u.row_tile = t;
        u.kb0 = (int)((int64_t)nkb * q / parts);
        u.nkb = (int)((int64_t)nkb * (q + 1) / parts) - u.kb0;
        u.part = q;
        u.O = (int32_t)l.out;
        u.K = (int32_t)l.in;
        units->push_back(u);
      }
  }
}

// Cost model of the schedule in units of one K block's pipeline time: a unit adds a fixed
// cost (accumulator hand-off, epilogue), a split adds the partial write and read-back.
constexpr int64_t kUnitCost = 2;
constexpr int64_t kSplitCost = 6;

sbn_status plan_shape(const sbn_group_linear *lins, int count, PlanShape *ps,
                      std::vector<GroupUnit> *units, std::vector<int32_t> *begin) {
  int64_t maxT = 0;
  ps->max_nv = 0;
  ps->has_x = true;
  ps->nrows = 0;
  for (int p = 0; p < count; ++p) {
    const sbn_group_linear &l = lins[p];
    maxT = l.tokens > maxT ? l.tokens : maxT;
    if (l.tokens > 0) {
      ps->nrows += l.tokens;
      if ((int32_t)(l.in / 8) > ps->max_nv) ps->max_nv = (int32_t)(l.in / 8);
      if (!l.X) ps->has_x = false;
    }
  }
  ps->bn = maxT <= 16 ? 16 : 32;
  const int sms = num_sms();
  // the split factor (the same for every layer) with the smallest estimated makespan
  int best = 1;
  int64_t best_cost = -1;
  std::vector<GroupUnit> tmp;
  std::vector<int32_t> nkb;
  for (int split = 1; split <= 8; ++split) {
    build_units(lins, count, split, &tmp);
    if (tmp.empty()) break;
    nkb.resize(tmp.size());
    for (size_t u = 0; u < tmp.size(); ++u) nkb[u] = tmp[u].nkb;
    const int64_t cost =
        partition_units(nkb, sms, kUnitCost, nullptr) + (split > 1 ? kSplitCost : 0);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = split;
    }
  }
  ps->split = best;
  build_units(lins, count, best, units);
  ps->nunits = (int64_t)units->size();
  nkb.resize(units->size());
  for (size_t u = 0; u < units->size(); ++u) nkb[u] = (*units)[u].nkb;
  if (!units->empty()) {
    partition_units(nkb, sms, kUnitCost, begin);
    ps->ncta = (int)begin->size() - 1;
  } else {
    begin->assign(1, 0);
    ps->ncta = 0;
  }
  // split layers: one counter per row tile, nparts partial tiles per row tile
  ps->ntickets = 0;
  ps->nparts_tiles = 0;
  for (int p = 0; p < count; ++p) {
    const sbn_group_linear &l = lins[p];
    if (l.tokens == 0) continue;
    const int nkbp = (int)((l.in + kGroupKB - 1) / kGroupKB);
    const int parts = best < nkbp ? best : nkbp;
    if (parts <= 1) continue;
    const int64_t tiles = (l.out + kGroupRows - 1) / kGroupRows;
    ps->ntickets += tiles;
    ps->nparts_tiles += tiles * parts;
  }
  return SBN_OK;
}

struct PlanLayout {
  int64_t off_probs, off_units, off_cta, off_rows, bytes;
  int64_t ws_part_off, ws_bytes;
};

PlanLayout plan_layout(int count, const PlanShape &ps) {
  PlanLayout L;
  L.off_probs = 128;
  L.off_units = L.off_probs + (int64_t)count * (int64_t)sizeof(GroupProb);
  L.off_cta = align_up(L.off_units + ps.nunits * (int64_t)sizeof(GroupUnit), 128);
  L.off_rows = align_up(L.off_cta + (int64_t)(ps.ncta + 1) * 4, 128);
  L.bytes = align_up(L.off_rows + ps.nrows * (int64_t)sizeof(GroupRow), 128);
  if (ps.ntickets > 0) {
    L.ws_part_off = align_up(ps.ntickets * 4, 256);
    L.ws_bytes = L.ws_part_off + ps.nparts_tiles * (int64_t)(kGroupRows * ps.bn * 4);
  } else {
    L.ws_part_off = 0;
    L.ws_bytes = 0;
  }
  return L;
}

}  // namespace

sbn_status group_plan_sizes(const sbn_group_linear *lins, int count, int64_t *plan_bytes,
                            int64_t *workspace_bytes) {
  PlanShape ps;
  std::vector<GroupUnit> units;
  std::vector<int32_t> begin;
  sbn_status st = plan_shape(lins, count, &ps, &units, &begin);
  if (st != SBN_OK) return st;
  const PlanLayout L = plan_layout(count, ps);
  *plan_bytes = L.bytes;
  *workspace_bytes = L.ws_bytes;
  return SBN_OK;
}

sbn_status group_plan(const sbn_group_linear *lins, int count, void *plan, int64_t plan_bytes) {
  PlanShape ps;
  std::vector<GroupUnit> units;
  std::vector<int32_t> begin;
  sbn_status st = plan_shape(lins, count, &ps, &units, &begin);
  if (st != SBN_OK) return st;
  const PlanLayout L = plan_layout(count, ps);
  if (plan_bytes < L.bytes) return SBN_ERR_SHAPE;
  uint8_t *P = static_cast<uint8_t *>(plan);
  memset(P, 0, (size_t)L.bytes);
  GroupHeader *hd = reinterpret_cast<GroupHeader *>(P);
  hd->magic = kGroupMagic;
  hd->version = kGroupVersion;
  hd->count = count;
  hd->nunits = (int32_t)ps.nunits;
  hd->ncta = ps.ncta;
  hd->bn = ps.bn;
  hd->nrows = (int32_t)ps.nrows;
  hd->max_nv = ps.max_nv;
  hd->has_x = ps.has_x ? 1 : 0;
  hd->split = ps.split;
  hd->off_probs = L.off_probs;
  hd->off_units = L.off_units;
  hd->off_cta = L.off_cta;
  hd->off_rows = L.off_rows;
  hd->bytes = L.bytes;
  hd->ws_bytes = L.ws_bytes;
  hd->ntickets = ps.ntickets;
  hd->ws_part_off = L.ws_part_off;
  GroupProb *probs = reinterpret_cast<GroupProb *>(P + L.off_probs);
  GroupRow *rows = reinterpret_cast<GroupRow *>(P + L.off_rows);
  int64_t ticket = 0, part = 0, row = 0;
  for (int p = 0; p < count; ++p) {
    const sbn_group_linear &l = lins[p];
    GroupProb &g = probs[p];
    g.X = l.X;
    g.Xq = l.Xq;
    g.absmax = l.absmax;
    g.gamma_eff = l.gamma_eff;
    g.Y = l.Y;
    g.acc_dbg = l.acc_dbg;
    g.T = l.tokens;
    g.O = l.out;
    g.K = l.in;
    g.y_is_bf16 = l.y_is_bf16 ? 1 : 0;
    g.ldx = l.ldx ? l.ldx : l.in;
    if (l.tokens == 0) continue;
    // 2:4 planes: K/8 bytes per row, strides rounded up to 16 bytes (or the caller's, for a
    // K slice of a wider tensor's planes)
    const int64_t ldc = l.ldc ? l.ldc : (l.in / 8 + 15) / 16 * 16;
    const int64_t ldm = l.ldm ? l.ldm : (l.in / 8 + 15) / 16 * 16;
    if (!encode_u8(&g.tx, l.Xq, l.in, l.tokens, g.ldx, kGroupKB, (uint32_t)ps.bn,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_u8(&g.tc, l.codes, l.in / 8, l.out, ldc, 16 * kSuper, kGroupRows,
                   CU_TENSOR_MAP_SWIZZLE_64B) ||
        !encode_u8(&g.tm, l.meta, l.in / 8, l.out, ldm, 16 * kSuper, kGroupRows,
                   CU_TENSOR_MAP_SWIZZLE_64B))
      return SBN_ERR_CUDA;
    const int nkb = (int)((l.in + kGroupKB - 1) / kGroupKB);
    g.nparts = ps.split < nkb ? ps.split : nkb;
    if (g.nparts > 1) {
      const int64_t tiles = (l.out + kGroupRows - 1) / kGroupRows;
      g.ticket_base = ticket;
      g.part_base = part;
      ticket += tiles;
      part += tiles * g.nparts;
    }
    for (int64_t t = 0; t < l.tokens; ++t) rows[row++] = GroupRow{p, (int32_t)t};
  }
  memcpy(P + L.off_units, units.data(), units.size() * sizeof(GroupUnit));
  memcpy(P + L.off_cta, begin.data(), begin.size() * sizeof(int32_t));
  return SBN_OK;
}

sbn_status launch_linear_group(const void *plan_host, const void *plan_dev, void *workspace,
                               int32_t *err_flag, cudaStream_t st) {
  const GroupHeader *hd = static_cast<const GroupHeader *>(plan_host);
  if (hd->ncta == 0) return SBN_OK;
  const uint8_t *P = static_cast<const uint8_t *>(plan_dev);
  uint8_t *W = static_cast<uint8_t *>(workspace);
  if (hd->bn == 16) {
    auto kern = k_gemm_group<16>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)GrpCfg<16>::kSmem) != cudaSuccess)
      return SBN_ERR_CUDA;
    return launch_pdl(kern, dim3((unsigned)hd->ncta), dim3(kGrpThreads), GrpCfg<16>::kSmem, st,
                      P, W, err_flag);
  }
  auto kern = k_gemm_group<32>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)GrpCfg<32>::kSmem) != cudaSuccess)
    return SBN_ERR_CUDA;
  return launch_pdl(kern, dim3((unsigned)hd->ncta), dim3(kGrpThreads), GrpCfg<32>::kSmem, st, P,
                    W, err_flag);
}

}  // namespace sbn
