// Quant/mask/pack for the two patterns the pages use most, 6:8 and 2:4, with far fewer
// instructions per weight than the generic kernel (pack.cu).  Same results, bit for bit.
//
// The absmean sum needs all of W before any code is known, so W is read twice: k_abs_sum
// (pack.cu) streams it once at the full HBM bandwidth with little arithmetic per weight,
// then k_qmp here re-reads it (from L2 where W fits there), finishes the scale and does
// the heavy per-weight work - N:M selection, metadata and codes - in one pass.
//
// Each lane owns 16 consecutive weights (two 16-byte loads).  The arithmetic runs on the
// bf16 words as they are loaded (two weights per 32-bit register):
//   * N:M selection: the values of the M-N smallest magnitudes come from a min/max network
//     on both 16-bit halves at once (min.u16x2 / max.u16x2); a weight is pruned iff its
//     magnitude is <= the (M-N)-th smallest.  That set has exactly M-N members unless
//     magnitudes tie at the boundary; those groups (about one in a hundred) resolve the
//     tie inline with the rank rule's order (the lower index wins).
//   * code non-zero test: mag >= thr for both halves with one OR and one subtract
//     ((w | 0x80008000) - thr2 leaves each half's answer in its top bit, no borrow crosses).
//   * per-weight flags are collected with byte permutes into "byte-top" words (flag of
//     weight i in bit 8i+7) and shifted straight into the packed code layout.
#include "common.cuh"
#include "kernels.cuh"
#include "pack_common.cuh"
#include "ptx.cuh"

namespace sbn {

namespace {

__device__ __forceinline__ uint32_t vmin16(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("min.u16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
__device__ __forceinline__ uint32_t vmax16(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.u16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
__device__ __forceinline__ uint32_t swap16(uint32_t a) { return __byte_perm(a, a, 0x1032); }

constexpr uint32_t kTop = 0x80808080u;   // byte-top flag positions
constexpr uint32_t kHalf = 0x80008000u;  // bf16 sign positions
constexpr uint32_t kMag = 0x7fff7fffu;

// byte-top flags of two words (a: weights 0-3, b: weights 4-7) -> 8-bit mask
__device__ __forceinline__ uint32_t top_bits_to_byte(uint32_t a, uint32_t b) {
  const uint32_t x = ((a >> 7) & 0x01010101u) | ((b >> 3) & 0x10101010u);
  return (x * 0x01020408u) >> 24;
}
// 4-bit mask -> byte-top flags
__device__ __forceinline__ uint32_t nibble_to_top_bits(uint32_t k) {
  return ((k & 15u) * 0x10204080u) & kTop;
}
// byte-top "non-zero" and "negative" flags -> int8 lanes {0, +1, -1}
__device__ __forceinline__ uint32_t flags_to_i8(uint32_t lo, uint32_t hi) {
  return (lo >> 7) | ((hi >> 7) * 0xfeu);
}

// Highest set bit of x (x != 0) as a mask; 0 for x == 0.
__device__ __forceinline__ uint32_t top_bit(uint32_t x) {
  return x ? (0x80000000u >> __clz(x)) : 0u;
}

// Boundary ties.  With m2 the second smallest magnitude of a group, the pruned set is
// every weight below m2 (LT, at most one) plus, of the weights equal to m2 (EQ), the ones
// with the highest indices until two are pruned: the lower index wins a tie, as in the
// rank rule.  LE / LT / EQ are bit masks ordered like the weights, so the highest index
// is the highest set bit.
__device__ __forceinline__ uint32_t prune_with_ties(uint32_t le, uint32_t lt) {
  const uint32_t eq = le ^ lt;
  const uint32_t h1 = top_bit(eq);
  const uint32_t h2 = top_bit(eq ^ h1);
  return lt | h1 | (lt ? 0u : h2);
}

// 6:8 keep flags of one group (w[0..3]); KA/KB: byte-top flags of weights 0-3 / 4-7.
__device__ __forceinline__ void keep_6of8(const uint32_t *w, uint32_t &KA, uint32_t &KB) {
  const uint32_t M0 = w[0] & kMag, M1 = w[1] & kMag, M2 = w[2] & kMag, M3 = w[3] & kMag;
  // per half (even / odd weights): smallest c0 and second smallest c1 of its four
  const uint32_t a0 = vmin16(M0, M1), b0 = vmax16(M0, M1);
  const uint32_t a1 = vmin16(M2, M3), b1 = vmax16(M2, M3);
  const uint32_t c0 = vmin16(a0, a1), c1 = vmin16(vmax16(a0, a1), vmin16(b0, b1));
  // second smallest of all eight, in both halves
  const uint32_t m2 = vmin16(vmax16(c0, swap16(c0)), vmin16(c1, swap16(c1)));
  const uint32_t h = m2 | kHalf;
  // top bit of each half: mag <= m2 (exactly the pruned pair when the boundary has no tie)
  const uint32_t LA = __byte_perm(h - M0, h - M1, 0x7531) & kTop;
  const uint32_t LB = __byte_perm(h - M2, h - M3, 0x7531) & kTop;
  if (__popc(LA | (LB >> 1)) == 2) {
    KA = LA ^ kTop;
    KB = LB ^ kTop;
  } else {
    // mag <= m2 - 1 (nothing when m2 == 0: each half of hl is then 0x7fff)
    const uint32_t hl = h - 0x00010001u;
    const uint32_t TA = __byte_perm(hl - M0, hl - M1, 0x7531) & kTop;
    const uint32_t TB = __byte_perm(hl - M2, hl - M3, 0x7531) & kTop;
    const uint32_t keep =
        ~prune_with_ties(top_bits_to_byte(LA, LB), top_bits_to_byte(TA, TB)) & 0xffu;
    KA = nibble_to_top_bits(keep);
    KB = nibble_to_top_bits(keep >> 4);
  }
}

// 2:4 keep flags of one group (wa = weights 0,1; wb = weights 2,3) as byte-top flags.
__device__ __forceinline__ uint32_t keep_2of4(uint32_t wa, uint32_t wb) {
  const uint32_t Ma = wa & kMag, Mb = wb & kMag;
  const uint32_t a = vmin16(Ma, Mb), b = vmax16(Ma, Mb);  // sorted pairs (0,2) and (1,3)
  const uint32_t m2 = vmin16(vmax16(a, swap16(a)), vmin16(b, swap16(b)));
  const uint32_t h = m2 | kHalf;
  const uint32_t L = __byte_perm(h - Ma, h - Mb, 0x7531) & kTop;
  if (__popc(L) == 2) return L ^ kTop;
  const uint32_t hl = h - 0x00010001u;
  const uint32_t T = __byte_perm(hl - Ma, hl - Mb, 0x7531) & kTop;
  return prune_with_ties(L, T) ^ kTop;  // byte-top flags are ordered like the weights too
}

__device__ __forceinline__ uint32_t nonzero_flags(uint32_t w, uint32_t thr2) {
  return (w | kHalf) - thr2;  // top bit of each half: mag >= thr
}

}  // namespace


// For a keep byte (two 2:4 groups, 4 bits each): the meta byte (i0 | i1 << 2 per group)
// in bits 0-7, and in bits 8-23 the byte-permute selector that compacts the kept weights
// of the two groups (bytes 0-3 and 4-7 of a flag pair) into bytes 0-3.
__device__ uint32_t pair_entry(uint32_t keep8) {
  uint32_t meta = 0, sel = 0, slot = 0;
  for (int g = 0; g < 2; ++g) {
    uint32_t kept = 0;
    for (int i = 0; i < 4; ++i) {
      if ((keep8 >> (4 * g + i)) & 1u) {
        if (kept < 2) {
          meta |= (uint32_t)i << (4 * g + 2 * kept);
          sel |= (uint32_t)(4 * g + i) << (4 * slot);
          ++slot;
        }
        ++kept;
      }
    }
  }
  return meta | (sel << 8);
}

// Work split: warp-iteration q covers 64-weight blocks 8q .. 8q+7 (1 KB of W); lane l
// owns weights 16 (l & 3) .. +15 of block 8q + (l >> 2), loaded as two 16-byte words.
// Warps stride over q two iterations at a time (four 16-byte loads in flight per lane);
// four 256-thread CTAs per SM.
constexpr int kPkThreads = 256;
constexpr int kPkCtasPerSm = 4;

__device__ __forceinline__ void pk_load(const uint4 *W, uint32_t nb, uint32_t b, int s, uint4 &v0,
                                        uint4 &v1) {
  if (b < nb) {
    const uint4 *src = W + (uint64_t)b * 8 + 2 * s;
    v0 = __ldg(src);
    v1 = __ldg(src + 1);
  } else {
    v0 = v1 = make_uint4(0u, 0u, 0u, 0u);
  }
}

// One lane's 16 weights: keep masks, metadata, codes.
template <bool kCompact>
__device__ __forceinline__ void qmp_unit(const FastPackArgs &a, const uint32_t *s_pair, uint4 v0,
                                         uint4 v1, uint32_t b, int s, uint32_t thr2) {
  const bool valid = b < (uint32_t)a.nblocks;  // both lanes of a shuffle pair share the block
  const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
  // keep flags of weights 0-3, 4-7, 8-11, 12-15 (byte-top) and the metadata bits
  uint32_t K0, K1, K2, K3, meta16, selAB = 0, selCD = 0;
  if constexpr (kCompact) {
    K0 = keep_2of4(w[0], w[1]);
    K1 = keep_2of4(w[2], w[3]);
    K2 = keep_2of4(w[4], w[5]);
    K3 = keep_2of4(w[6], w[7]);
    const uint32_t eAB = s_pair[top_bits_to_byte(K0, K1)];
    const uint32_t eCD = s_pair[top_bits_to_byte(K2, K3)];
    meta16 = (eAB & 0xffu) | ((eCD & 0xffu) << 8);
    selAB = eAB >> 8;
    selCD = eCD >> 8;
  } else {
    keep_6of8(w, K0, K1);
    keep_6of8(w + 4, K2, K3);
    meta16 = top_bits_to_byte(K0, K1) | (top_bits_to_byte(K2, K3) << 8);
  }
  const uint32_t N0 = __byte_perm(nonzero_flags(w[0], thr2), nonzero_flags(w[1], thr2), 0x7531);
  const uint32_t N1 = __byte_perm(nonzero_flags(w[2], thr2), nonzero_flags(w[3], thr2), 0x7531);
  const uint32_t N2 = __byte_perm(nonzero_flags(w[4], thr2), nonzero_flags(w[5], thr2), 0x7531);
  const uint32_t N3 = __byte_perm(nonzero_flags(w[6], thr2), nonzero_flags(w[7], thr2), 0x7531);
  const uint32_t S0 = __byte_perm(w[0], w[1], 0x7531), S1 = __byte_perm(w[2], w[3], 0x7531);
  const uint32_t S2 = __byte_perm(w[4], w[5], 0x7531), S3 = __byte_perm(w[6], w[7], 0x7531);
  uint32_t word;
  if constexpr (kCompact) {
    // kept weights in order: stored elements 8s..8s+7 = (A.first, A.second, B.first,
    // B.second | C.first, ..., D.second): j = 2*(s&1) (+1 for C, D), byte k = position
    const int js = 4 * (s & 1);
    const uint32_t LAB = __byte_perm(N0, N1, selAB) & kTop;
    const uint32_t HAB = LAB & __byte_perm(S0, S1, selAB);
    const uint32_t LCD = __byte_perm(N2, N3, selCD) & kTop;
    const uint32_t HCD = LCD & __byte_perm(S2, S3, selCD);
    word = (HAB >> js) | (LAB >> (1 + js)) | (HCD >> (2 + js)) | (LCD >> (3 + js));
    word |= __shfl_xor_sync(0xffffffffu, word, 1);
  } else {
    const uint32_t L0 = N0 & K0, L1 = N1 & K1, L2 = N2 & K2, L3 = N3 & K3;
    const uint32_t H0 = L0 & S0, H1 = L1 & S1, H2 = L2 & S2, H3 = L3 & S3;
    // weights e = 0..15 of this lane are elements 16s+e of the block: word s, byte e%4,
    // bits (7,6) - 2*(e/4) for (negative, non-zero)
    word = H0 | (L0 >> 1) | (H1 >> 2) | (L1 >> 3) | (H2 >> 4) | (L2 >> 5) | (H3 >> 6) | (L3 >> 7);
  }
  if (!valid) return;
  const uint32_t row = fast_div(b, a.div_bpr);
  const uint32_t col = b - row * a.bpr;
  uint8_t *crow = a.codes + (int64_t)row * a.ldc;
  uint8_t *mrow = a.meta + (int64_t)row * a.ldm;
  if constexpr (kCompact) {
    if ((s & 1) == 0) reinterpret_cast<uint32_t *>(crow + col * 8)[s >> 1] = word;
  } else {
    reinterpret_cast<uint32_t *>(crow + col * 16)[s] = word;
  }
  reinterpret_cast<uint16_t *>(mrow + col * 8)[s] = (uint16_t)meta16;
  if (col == a.bpr - 1 && s == 0) {  // zero the row padding
    if (a.ldc > a.codes_row_bytes)
      *reinterpret_cast<uint2 *>(crow + a.codes_row_bytes) = make_uint2(0u, 0u);
    if (a.ldm > a.meta_row_bytes)
      *reinterpret_cast<uint2 *>(mrow + a.meta_row_bytes) = make_uint2(0u, 0u);
  }
  if (a.dense_dbg) {
    const uint32_t l0 = N0 & K0, l1 = N1 & K1, l2 = N2 & K2, l3 = N3 & K3;
    *reinterpret_cast<uint4 *>(a.dense_dbg + (uint64_t)b * 64 + 16 * s) =
        make_uint4(flags_to_i8(l0, l0 & S0), flags_to_i8(l1, l1 & S1), flags_to_i8(l2, l2 & S2),
                   flags_to_i8(l3, l3 & S3));
  }
}

// ---------------------------------------------------------------------------------------
// Keep masks, metadata and codes in one pass over W, after k_abs_sum (launched as its
// programmatic dependent: each lane requests its first W words before waiting for the
// partial sums, then the CTA finishes the scale in pack_prologue).
// ---------------------------------------------------------------------------------------
template <bool kCompact>
__global__ void __launch_bounds__(kPkThreads, kPkCtasPerSm) k_qmp(const FastPackArgs a) {
  __shared__ uint32_t s_pair[256];  // 2:4: keep byte -> meta byte | compaction selector << 8
  // a programmatic dependent (the contraction) may start launching; it waits for this
  // kernel's completion before reading the planes
  ptx::grid_dep_launch();
  if (kCompact) s_pair[threadIdx.x] = pair_entry(threadIdx.x);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int s = lane & 3;
  const uint32_t nb = (uint32_t)a.nblocks;
  const uint32_t bstep = 8 * gridDim.x * (kPkThreads / 32);
  const uint32_t first = 8 * (blockIdx.x * (kPkThreads / 32) + warp);  // warp-uniform
  const uint32_t sub = lane >> 2;
  uint4 p0, p1, q0, q1;
  pk_load(a.W, nb, first + sub, s, p0, p1);
  pk_load(a.W, nb, first + bstep + sub, s, q0, q1);
  ptx::grid_dep_wait();  // k_abs_sum complete: partial sums visible
  const uint32_t thr = pack_prologue(a.ws, a.nparts, a.n, a.eps, a.gamma_eff);  // syncs
  const uint32_t thr2 = thr | (thr << 16);
  for (uint32_t base = first;;) {
    qmp_unit<kCompact>(a, s_pair, p0, p1, base + sub, s, thr2);
    qmp_unit<kCompact>(a, s_pair, q0, q1, base + bstep + sub, s, thr2);
    base += 2 * bstep;
    if (base >= nb) break;
    pk_load(a.W, nb, base + sub, s, p0, p1);
    pk_load(a.W, nb, base + bstep + sub, s, q0, q1);
  }
}

sbn_status launch_fast_pack(const FastPackArgs &a, bool compact, cudaStream_t st) {
  // one wave: enough CTAs for one warp-iteration per warp, at most kPkCtasPerSm per SM
  const int64_t warp_iters = (a.nblocks + 7) / 8;
  int64_t grid = (warp_iters + kPkThreads / 32 - 1) / (kPkThreads / 32);
  const int64_t cap = (int64_t)num_sms() * kPkCtasPerSm;
  if (grid > cap) grid = cap;
  if (grid < 1) grid = 1;
  // launched as a programmatic dependent of k_abs_sum: it may start while k_abs_sum
  // drains and waits for its completion before reading the partial sums
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(kPkThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = compact ? cudaLaunchKernelEx(&cfg, k_qmp<true>, a)
                                : cudaLaunchKernelEx(&cfg, k_qmp<false>, a);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return SBN_ERR_CUDA;
  }
  return SBN_OK;
}

}  // namespace sbn
