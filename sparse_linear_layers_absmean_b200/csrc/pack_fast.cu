// Quant/mask/pack for the two patterns the pages use most, 6:8 and 2:4, with far fewer
// instructions per weight than the generic kernel (pack.cu).  Same results, bit for bit.
//
// Each lane owns 16 consecutive weights (two 16-byte loads).  The arithmetic runs on the
// bf16 words as they are loaded (two weights per 32-bit register):
//   * N:M selection: the values of the M-N smallest magnitudes come from a min/max network
//     on both 16-bit halves at once (min.u16x2 / max.u16x2); a weight is pruned iff its
//     magnitude is <= the (M-N)-th smallest.  That set has exactly M-N members unless
//     magnitudes tie at the boundary; those groups (rare) take the exact rank rule with
//     the lower index winning, the same rule as everywhere else.
//   * code non-zero test: mag >= thr for both halves with one OR and one subtract
//     ((w | 0x80008000) - thr2 leaves each half's answer in its top bit, no borrow crosses).
//   * per-weight flags are collected with byte permutes into "byte-top" words (flag of
//     weight i in bit 8i+7) and shifted straight into the packed code layout.
#include "common.cuh"
#include "kernels.cuh"
#include "pack_common.cuh"

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

// Exact rank rule for one group (the fallback when magnitudes tie at the boundary).
template <int N, int M>
__device__ __noinline__ uint32_t exact_keep(const uint32_t *w) {
  uint32_t key[M];
#pragma unroll
  for (int i = 0; i < M; ++i)
    key[i] = ((((w[i >> 1] >> (16 * (i & 1))) & 0x7fffu)) << 3) | (uint32_t)(M - 1 - i);
  uint32_t keep = 0;
#pragma unroll
  for (int i = 0; i < M; ++i) {
    int rank = 0;
#pragma unroll
    for (int j = 0; j < M; ++j) rank += (j != i) && (key[j] > key[i]);
    keep |= (uint32_t)(rank < N) << i;
  }
  return keep;
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
  // top bit of each half: mag <= m2 (pruned when the boundary has no tie)
  const uint32_t LA = __byte_perm(h - M0, h - M1, 0x7531) & kTop;
  const uint32_t LB = __byte_perm(h - M2, h - M3, 0x7531) & kTop;
  if (__popc(LA | (LB >> 1)) == 2) {
    KA = LA ^ kTop;
    KB = LB ^ kTop;
  } else {
    const uint32_t keep = exact_keep<6, 8>(w);
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
  const uint32_t w2[2] = {wa, wb};
  return nibble_to_top_bits(exact_keep<2, 4>(w2));
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

// This lane's 32 bytes of warp iteration q (zeros past the end).
__device__ __forceinline__ void load_lane(const FastPackArgs &a, int64_t q, int lane, uint4 &v0,
                                          uint4 &v1) {
  const int64_t b = 8 * q + (lane >> 2);
  if (b < a.nblocks) {
    const uint4 *src = a.W + b * 8 + 2 * (lane & 3);
    v0 = __ldg(src);
    v1 = __ldg(src + 1);
  } else {
    v0 = v1 = make_uint4(0u, 0u, 0u, 0u);
  }
}

__global__ void __launch_bounds__(256) k_qmp_6of8(const FastPackArgs a) {
  const int lane = threadIdx.x & 31;
  const int s = lane & 3;  // lane inside its 64-weight block
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
  const int64_t noct = (a.nblocks + 7) >> 3;  // 8 blocks per warp iteration
  const int64_t q0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  // the first weights are requested before the scale is finished, the next iteration's
  // before the current one is processed
  uint4 n0, n1;
  load_lane(a, q0, lane, n0, n1);
  const uint32_t thr = pack_prologue(a.ws, a.nparts, a.n, a.eps, a.gamma_eff);
  const uint32_t thr2 = thr | (thr << 16);
  for (int64_t q = q0; q < noct; q += nwarps) {
    const uint4 v0 = n0, v1 = n1;
    load_lane(a, q + nwarps, lane, n0, n1);
    const int64_t b = 8 * q + (lane >> 2);
    if (b >= a.nblocks) continue;  // no cross-lane exchange in this kernel
    const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
    uint32_t KGA, KGB, KHA, KHB;
    keep_6of8(w, KGA, KGB);
    keep_6of8(w + 4, KHA, KHB);
    const uint32_t NGA = __byte_perm(nonzero_flags(w[0], thr2), nonzero_flags(w[1], thr2), 0x7531);
    const uint32_t NGB = __byte_perm(nonzero_flags(w[2], thr2), nonzero_flags(w[3], thr2), 0x7531);
    const uint32_t NHA = __byte_perm(nonzero_flags(w[4], thr2), nonzero_flags(w[5], thr2), 0x7531);
    const uint32_t NHB = __byte_perm(nonzero_flags(w[6], thr2), nonzero_flags(w[7], thr2), 0x7531);
    const uint32_t LGA = NGA & KGA, LGB = NGB & KGB, LHA = NHA & KHA, LHB = NHB & KHB;
    const uint32_t HGA = LGA & __byte_perm(w[0], w[1], 0x7531);
    const uint32_t HGB = LGB & __byte_perm(w[2], w[3], 0x7531);
    const uint32_t HHA = LHA & __byte_perm(w[4], w[5], 0x7531);
    const uint32_t HHB = LHB & __byte_perm(w[6], w[7], 0x7531);
    // weights e = 0..15 of this lane are elements 16s+e of the block: word s, byte e%4,
    // bits (7,6) - 2*(e/4) for (negative, non-zero)
    const uint32_t word = HGA | (LGA >> 1) | (HGB >> 2) | (LGB >> 3) | (HHA >> 4) | (LHA >> 5) |
                          (HHB >> 6) | (LHB >> 7);
    const uint32_t meta16 = top_bits_to_byte(KGA, KGB) | (top_bits_to_byte(KHA, KHB) << 8);
    const uint32_t row = fast_div((uint32_t)b, a.div_bpr);
    const uint32_t col = (uint32_t)b - row * a.bpr;
    uint8_t *crow = a.codes + (int64_t)row * a.ldc;
    uint8_t *mrow = a.meta + (int64_t)row * a.ldm;
    reinterpret_cast<uint32_t *>(crow + col * 16)[s] = word;
    reinterpret_cast<uint16_t *>(mrow + col * 8)[s] = (uint16_t)meta16;
    if (col == a.bpr - 1 && s == 0 && a.ldm > a.meta_row_bytes)
      *reinterpret_cast<uint2 *>(mrow + a.meta_row_bytes) = make_uint2(0u, 0u);
    if (a.dense_dbg)
      *reinterpret_cast<uint4 *>(a.dense_dbg + b * 64 + 16 * s) =
          make_uint4(flags_to_i8(LGA, HGA), flags_to_i8(LGB, HGB), flags_to_i8(LHA, HHA),
                     flags_to_i8(LHB, HHB));
  }
}

__global__ void __launch_bounds__(256) k_qmp_2of4(const FastPackArgs a) {
  __shared__ uint32_t s_pair[256];
  s_pair[threadIdx.x] = pair_entry(threadIdx.x);
  const int lane = threadIdx.x & 31;
  const int s = lane & 3;
  const int js = 4 * (s & 1);  // 2j of stored elements 8s..8s+3 (j = 2*(s&1))
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
  const int64_t noct = (a.nblocks + 7) >> 3;
  const int64_t q0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  uint4 n0, n1;
  load_lane(a, q0, lane, n0, n1);
  const uint32_t thr = pack_prologue(a.ws, a.nparts, a.n, a.eps, a.gamma_eff);  // syncs
  const uint32_t thr2 = thr | (thr << 16);
  for (int64_t q = q0; q < noct; q += nwarps) {
    const uint4 v0 = n0, v1 = n1;
    load_lane(a, q + nwarps, lane, n0, n1);
    const int64_t b = 8 * q + (lane >> 2);
    const bool valid = b < a.nblocks;  // all lanes stay for the shuffle below
    const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
    const uint32_t KA = keep_2of4(w[0], w[1]), KB = keep_2of4(w[2], w[3]);
    const uint32_t KC = keep_2of4(w[4], w[5]), KD = keep_2of4(w[6], w[7]);
    const uint32_t eAB = s_pair[top_bits_to_byte(KA, KB)];
    const uint32_t eCD = s_pair[top_bits_to_byte(KC, KD)];
    const uint32_t NA = __byte_perm(nonzero_flags(w[0], thr2), nonzero_flags(w[1], thr2), 0x7531);
    const uint32_t NB = __byte_perm(nonzero_flags(w[2], thr2), nonzero_flags(w[3], thr2), 0x7531);
    const uint32_t NC = __byte_perm(nonzero_flags(w[4], thr2), nonzero_flags(w[5], thr2), 0x7531);
    const uint32_t ND = __byte_perm(nonzero_flags(w[6], thr2), nonzero_flags(w[7], thr2), 0x7531);
    const uint32_t SA = __byte_perm(w[0], w[1], 0x7531), SB = __byte_perm(w[2], w[3], 0x7531);
    const uint32_t SC = __byte_perm(w[4], w[5], 0x7531), SD = __byte_perm(w[6], w[7], 0x7531);
    // kept weights in order: stored elements 8s..8s+7 = (A.first, A.second, B.first,
    // B.second | C.first, ..., D.second): j = 2*(s&1) (+1 for C, D), byte k = position
    const uint32_t selAB = eAB >> 8, selCD = eCD >> 8;
    const uint32_t LAB = __byte_perm(NA, NB, selAB) & kTop;
    const uint32_t HAB = LAB & __byte_perm(SA, SB, selAB);
    const uint32_t LCD = __byte_perm(NC, ND, selCD) & kTop;
    const uint32_t HCD = LCD & __byte_perm(SC, SD, selCD);
    uint32_t word = (HAB >> js) | (LAB >> (1 + js)) | (HCD >> (2 + js)) | (LCD >> (3 + js));
    word |= __shfl_xor_sync(0xffffffffu, word, 1);
    if (!valid) continue;
    const uint32_t row = fast_div((uint32_t)b, a.div_bpr);
    const uint32_t col = (uint32_t)b - row * a.bpr;
    uint8_t *crow = a.codes + (int64_t)row * a.ldc;
    uint8_t *mrow = a.meta + (int64_t)row * a.ldm;
    if ((s & 1) == 0) reinterpret_cast<uint32_t *>(crow + col * 8)[s >> 1] = word;
    reinterpret_cast<uint16_t *>(mrow + col * 8)[s] = (uint16_t)((eAB & 0xffu) | ((eCD & 0xffu) << 8));
    if (col == a.bpr - 1 && s == 0) {
      if (a.ldc > a.codes_row_bytes)
        *reinterpret_cast<uint2 *>(crow + a.codes_row_bytes) = make_uint2(0u, 0u);
      if (a.ldm > a.meta_row_bytes)
        *reinterpret_cast<uint2 *>(mrow + a.meta_row_bytes) = make_uint2(0u, 0u);
    }
    if (a.dense_dbg) {
      const uint32_t la = NA & KA, lb = NB & KB, lc = NC & KC, ld = ND & KD;
      *reinterpret_cast<uint4 *>(a.dense_dbg + b * 64 + 16 * s) =
          make_uint4(flags_to_i8(la, la & SA), flags_to_i8(lb, lb & SB), flags_to_i8(lc, lc & SC),
                     flags_to_i8(ld, ld & SD));
    }
  }
}

}  // namespace sbn
