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

// The flags every pattern uses, from one lane's 16 weights (w[i] = weights 2i, 2i+1): N
// "code non-zero" and S "negative", byte-top, for weights 4i..4i+3 in N[i] / S[i].
struct LaneFlags {
  uint32_t N[4], S[4];
};
__device__ __forceinline__ LaneFlags lane_flags(const uint32_t *w, uint32_t thr2) {
  LaneFlags f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f.N[i] = __byte_perm(nonzero_flags(w[2 * i], thr2), nonzero_flags(w[2 * i + 1], thr2), 0x7531);
    f.S[i] = __byte_perm(w[2 * i], w[2 * i + 1], 0x7531);
  }
  return f;
}

// One pattern's result for a lane: keep flags (byte-top, weights 4i..4i+3 in K[i]), the
// lane's code word and its 16 metadata bits.
struct LanePack {
  uint32_t K[4], word, meta16;
};

// 2:4: the lane's 16 weights are two 8-weight halves of one 32-bit code word (kept elements
// 8s..8s+7 of the block); lanes s and s^1 exchange halves, so both hold the whole word.
__device__ __forceinline__ LanePack pack_lane_2of4(const uint32_t *w, const LaneFlags &f,
                                                   const uint32_t *s_pair, int s) {
  LanePack r;
  r.K[0] = keep_2of4(w[0], w[1]);
  r.K[1] = keep_2of4(w[2], w[3]);
  r.K[2] = keep_2of4(w[4], w[5]);
  r.K[3] = keep_2of4(w[6], w[7]);
  const uint32_t eAB = s_pair[top_bits_to_byte(r.K[0], r.K[1])];
  const uint32_t eCD = s_pair[top_bits_to_byte(r.K[2], r.K[3])];
  r.meta16 = (eAB & 0xffu) | ((eCD & 0xffu) << 8);
  const uint32_t selAB = eAB >> 8, selCD = eCD >> 8;
  // kept weights in order: stored elements 8s..8s+7 = (A.first, A.second, B.first,
  // B.second | C.first, ..., D.second): j = 2*(s&1) (+1 for C, D), byte k = position
  const int js = 4 * (s & 1);
  const uint32_t LAB = __byte_perm(f.N[0], f.N[1], selAB) & kTop;
  const uint32_t HAB = LAB & __byte_perm(f.S[0], f.S[1], selAB);
  const uint32_t LCD = __byte_perm(f.N[2], f.N[3], selCD) & kTop;
  const uint32_t HCD = LCD & __byte_perm(f.S[2], f.S[3], selCD);
  uint32_t word = (HAB >> js) | (LAB >> (1 + js)) | (HCD >> (2 + js)) | (LCD >> (3 + js));
  r.word = word | __shfl_xor_sync(0xffffffffu, word, 1);
  return r;
}

// 6:8: the lane's 16 weights are the 16 elements of one code word (word s of the block).
__device__ __forceinline__ LanePack pack_lane_6of8(const uint32_t *w, const LaneFlags &f) {
  LanePack r;
  keep_6of8(w, r.K[0], r.K[1]);
  keep_6of8(w + 4, r.K[2], r.K[3]);
  r.meta16 = top_bits_to_byte(r.K[0], r.K[1]) | (top_bits_to_byte(r.K[2], r.K[3]) << 8);
  const uint32_t L0 = f.N[0] & r.K[0], L1 = f.N[1] & r.K[1], L2 = f.N[2] & r.K[2],
                 L3 = f.N[3] & r.K[3];
  const uint32_t H0 = L0 & f.S[0], H1 = L1 & f.S[1], H2 = L2 & f.S[2], H3 = L3 & f.S[3];
  // weights e = 0..15 of this lane are elements 16s+e of the block: word s, byte e%4,
  // bits (7,6) - 2*(e/4) for (negative, non-zero)
  r.word = H0 | (L0 >> 1) | (H1 >> 2) | (L1 >> 3) | (H2 >> 4) | (L2 >> 5) | (H3 >> 6) | (L3 >> 7);
  return r;
}

// Where one pattern's planes go: the plane pointers and row strides (multiples of 16).
// Every row's data is a multiple of 8 bytes, so a row either fills its stride or ends 8
// bytes short of it; bit 0 of ldc / ldm marks the second case (those 8 bytes are zeroed).
struct PlaneOut {
  uint8_t *codes, *meta;
  uint32_t ldc, ldm;
};
__device__ __forceinline__ PlaneOut plane_out(const FastPackArgs &a) {
  return PlaneOut{a.codes, a.meta, (uint32_t)a.ldc | (a.codes_row_bytes != a.ldc ? 1u : 0u),
                  (uint32_t)a.ldm | (a.meta_row_bytes != a.ldm ? 1u : 0u)};
}

// Stores a lane's part of block (row, col) of one pattern: code word, metadata bits and
// the row padding (by the row's last block).
template <bool kCompact>
__device__ __forceinline__ void store_lane(const PlaneOut &o, const LanePack &r, uint32_t row,
                                           uint32_t col, bool row_end, int s) {
  const uint32_t ldc = o.ldc & ~1u, ldm = o.ldm & ~1u;
  uint8_t *crow = o.codes + (uint64_t)row * ldc;
  uint8_t *mrow = o.meta + (uint64_t)row * ldm;
  if constexpr (kCompact) {
    if ((s & 1) == 0) reinterpret_cast<uint32_t *>(crow + col * 8)[s >> 1] = r.word;
  } else {
    reinterpret_cast<uint32_t *>(crow + col * 16)[s] = r.word;
  }
  reinterpret_cast<uint16_t *>(mrow + col * 8)[s] = (uint16_t)r.meta16;
  if (row_end && s == 0) {
    if (o.ldc & 1u) *reinterpret_cast<uint2 *>(crow + ldc - 8) = make_uint2(0u, 0u);
    if (o.ldm & 1u) *reinterpret_cast<uint2 *>(mrow + ldm - 8) = make_uint2(0u, 0u);
  }
}

// The optional masked ternary matrix: the lane's 16 int8 values of block b.
__device__ __forceinline__ void store_dense(int8_t *dense, const LaneFlags &f, const LanePack &r,
                                            uint32_t b, int s) {
  const uint32_t l0 = f.N[0] & r.K[0], l1 = f.N[1] & r.K[1], l2 = f.N[2] & r.K[2],
                 l3 = f.N[3] & r.K[3];
  *reinterpret_cast<uint4 *>(dense + (uint64_t)b * 64 + 16 * s) =
      make_uint4(flags_to_i8(l0, l0 & f.S[0]), flags_to_i8(l1, l1 & f.S[1]),
                 flags_to_i8(l2, l2 & f.S[2]), flags_to_i8(l3, l3 & f.S[3]));
}

// One lane's 16 weights: keep masks, metadata, codes.
template <bool kCompact>
__device__ __forceinline__ void qmp_unit(const FastPackArgs &a, const uint32_t *s_pair, uint4 v0,
                                         uint4 v1, uint32_t b, int s, uint32_t thr2) {
  const bool valid = b < (uint32_t)a.nblocks;  // both lanes of a shuffle pair share the block
  const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
  const LaneFlags f = lane_flags(w, thr2);
  LanePack r;
  if constexpr (kCompact)
    r = pack_lane_2of4(w, f, s_pair, s);
  else
    r = pack_lane_6of8(w, f);
  if (!valid) return;
  const uint32_t row = fast_div(b, a.div_bpr);
  const uint32_t col = b - row * a.bpr;
  store_lane<kCompact>(plane_out(a), r, row, col, col == a.bpr - 1, s);
  if (a.dense_dbg) store_dense(a.dense_dbg, f, r, b, s);
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

// ---------------------------------------------------------------------------------------
// Grouped pack (many tensors, each packed into one or two of the patterns above).
//
// k_abs_sum_group streams every tensor's W in chunks of kPackGroupChunkVecs 16-byte
// vectors (256 KB), CTAs striding over the chunks of all tensors.  Each chunk's exact
// partial sum goes into its tensor's slot with one 64-bit atomic add (integer: the order
// of the adds cannot change S); the CTA that finishes a tensor's last chunk turns S into g
// and the code threshold, publishes them, and clears the slot for the next call.
// k_qmp_group then re-reads W once and writes both patterns' planes from the same words:
// a tensor asked for 6:8 and 2:4 is read twice in all, not four times.
// ---------------------------------------------------------------------------------------
constexpr int kAgThreads = 256;
constexpr int kAgLoads = 4;
static_assert(kPackGroupChunkVecs % (kAgThreads * kAgLoads) == 0, "whole iterations per chunk");

__global__ void __launch_bounds__(kAgThreads, 4)
    k_abs_sum_group(const PackGroupHeader *__restrict__ hdr, const PackGroupTensor *__restrict__ T,
                    PackGroupSlot *slots, int32_t *err_flag) {
  ptx::grid_dep_wait();  // the previous kernel on the stream may have written W
  ptx::grid_dep_launch();
  __shared__ unsigned long long s_sum[kAgThreads / 32];
  __shared__ uint32_t s_all[kAgThreads / 32], s_fin[kAgThreads / 32];
  __shared__ int s_last;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t total = hdr->total_chunks;
  int t = 0;  // chunks ascend per CTA, so the tensor index only moves forward
  for (uint32_t c = blockIdx.x; c < total; c += gridDim.x) {
    while (c >= T[t].chunk_begin + T[t].nchunks) ++t;
    const uint4 *W = T[t].pa.W;
    const int64_t v0 = (int64_t)(c - T[t].chunk_begin) * kPackGroupChunkVecs;
    const int64_t v1 = min(v0 + kPackGroupChunkVecs, T[t].nvec);
    double acc0 = kAccBias, acc1 = kAccBias;
    uint32_t mx = 0;
    for (int64_t i = v0 + threadIdx.x; i < v1; i += kAgLoads * kAgThreads) {
      uint4 v[kAgLoads];
#pragma unroll
      for (int u = 0; u < kAgLoads; ++u)
        v[u] = i + u * kAgThreads < v1 ? __ldg(W + i + u * kAgThreads) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
      for (int u = 0; u < kAgLoads; ++u) {
        const uint32_t w4[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          asm("max.u16x2 %0, %0, %1;" : "+r"(mx) : "r"(w4[q] & 0x7fff7fffu));
          acc0 = __dadd_rz(acc0, mag_lo_x2p128(w4[q]));
          acc1 = __dadd_rz(acc1, mag_hi_x2p128(w4[q]));
        }
      }
    }
    unsigned long long acc = acc_value(acc0) + acc_value(acc1);
    uint32_t mx_all = 0, mx_fin = 0;
    if (max(mx & 0xffffu, mx >> 16) >= kBf16Mag256Bits) {  // rare: tell NaN/Inf from range
      for (int64_t j = v0 + threadIdx.x; j < v1; j += kAgThreads) {
        const uint4 v = __ldg(W + j);
        const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
        for (int q = 0; q < 4; ++q)
          for (int h = 0; h < 2; ++h) {
            const uint32_t m = (w4[q] >> (16 * h)) & 0x7fffu;
            mx_all = max(mx_all, m);
            if (m < kBf16InfBits) mx_fin = max(mx_fin, m);
          }
      }
    }
    acc = warp_sum_u64(acc);
    mx_all = warp_max_u32(mx_all);
    mx_fin = warp_max_u32(mx_fin);
    if (lane == 0) {
      s_sum[warp] = acc;
      s_all[warp] = mx_all;
      s_fin[warp] = mx_fin;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      unsigned long long sum = 0;
      uint32_t a = 0, f = 0;
      for (int w = 0; w < kAgThreads / 32; ++w) {
        sum += s_sum[w];
        a = max(a, s_all[w]);
        f = max(f, s_fin[w]);
      }
      int flags = 0;
      if (a >= kBf16InfBits) flags |= SBN_FLAG_W_NONFINITE;
      if (f >= kBf16Mag256Bits) flags |= SBN_FLAG_W_RANGE;
      if (flags && err_flag) atomicOr(err_flag, flags);
      atomicAdd(&slots[t].S, sum);
      __threadfence();  // the add is visible before the chunk counts as done
      const unsigned int prev = atomicAdd(&slots[t].done, 1u);
      s_last = prev == T[t].nchunks - 1;
    }
    __syncthreads();
    if (s_last && warp == 0) {  // every chunk of tensor t is in S
      __threadfence();
      unsigned long long S = 0;
      if (lane == 0) S = atomicExch(&slots[t].S, 0ull);  // read and clear
      S = __shfl_sync(0xffffffffu, S, 0);
      float g;
      const uint32_t thr = scale_from_sum(S, T[t].pa.n, T[t].pa.eps, lane, g);
      if (lane == 0) {
        *T[t].pa.gamma_eff = g;
        slots[t].thr = thr;
        slots[t].done = 0u;
      }
    }
    __syncthreads();  // s_sum and s_last are reused by the next chunk
  }
}

__device__ __forceinline__ void qg_advance(const PackGroupTensor *__restrict__ T, int &t,
                                           uint32_t q) {
  while (q >= T[t].q_begin + T[t].nq) ++t;
}

__global__ void __launch_bounds__(kPkThreads, kPkCtasPerSm)
    k_qmp_group(const PackGroupHeader *__restrict__ hdr, const PackGroupTensor *__restrict__ T,
                const PackGroupSlot *__restrict__ slots) {
  __shared__ uint32_t s_pair[256];
  ptx::grid_dep_launch();
  s_pair[threadIdx.x] = pair_entry(threadIdx.x);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int s = lane & 3;
  const uint32_t sub = lane >> 2;
  const uint32_t nq = hdr->total_q;
  const uint32_t qstep = gridDim.x * (kPkThreads / 32);
  uint32_t q = blockIdx.x * (kPkThreads / 32) + warp;  // warp-uniform
  int t = 0;
  uint4 p0 = make_uint4(0u, 0u, 0u, 0u), p1 = p0;
  uint32_t b = 0;
  if (q < nq) {  // request the first words before waiting (W is final: k_abs_sum_group
                 // waited for its predecessor before it let this kernel launch)
    qg_advance(T, t, q);
    b = (q - T[t].q_begin) * 8 + sub;
    pk_load(T[t].pa.W, (uint32_t)T[t].pa.nblocks, b, s, p0, p1);
  }
  ptx::grid_dep_wait();  // k_abs_sum_group complete: thresholds and g published
  __syncthreads();       // s_pair
  while (q < nq) {
    const uint32_t qn = q + qstep;
    int tn = t;
    uint4 n0 = make_uint4(0u, 0u, 0u, 0u), n1 = n0;
    uint32_t bn = 0;
    if (qn < nq) {
      qg_advance(T, tn, qn);
      bn = (qn - T[tn].q_begin) * 8 + sub;
      pk_load(T[tn].pa.W, (uint32_t)T[tn].pa.nblocks, bn, s, n0, n1);
    }
    const PackGroupTensor &e = T[t];
    const uint32_t thr = slots[t].thr;
    const uint32_t thr2 = thr | (thr << 16);
    if (e.pa_compact)
      qmp_unit<true>(e.pa, s_pair, p0, p1, b, s, thr2);
    else
      qmp_unit<false>(e.pa, s_pair, p0, p1, b, s, thr2);
    if (e.pb.codes) {
      if (e.pb_compact)
        qmp_unit<true>(e.pb, s_pair, p0, p1, b, s, thr2);
      else
        qmp_unit<false>(e.pb, s_pair, p0, p1, b, s, thr2);
    }
    q = qn;
    t = tn;
    b = bn;
    p0 = n0;
    p1 = n1;
  }
}

// Fixed-pattern form of k_qmp_group, for plans whose tensors all pack the same patterns
// (kMode 0: 6:8, 1: 2:4, 2: 6:8 into pa and 2:4 into pb) and ask for no dense matrix.  A warp keeps its current
// tensor's geometry and output pointers in registers while its iterations stay in that
// tensor: the plan entry is read once per tensor, not once per iteration, and the flags,
// row and column of a block serve both patterns.  The words of the next iteration are
// requested before the current ones are packed.
constexpr int kQgCtasPerSm = 3;

template <int kMode>
__global__ void __launch_bounds__(kPkThreads, kQgCtasPerSm)
    k_qmp_group_fixed(const PackGroupHeader *__restrict__ hdr,
                      const PackGroupTensor *__restrict__ T,
                      const PackGroupSlot *__restrict__ slots) {
  __shared__ uint32_t s_pair[256];
  ptx::grid_dep_launch();
  if (kMode != 0) s_pair[threadIdx.x] = pair_entry(threadIdx.x);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int s = lane & 3;
  const uint32_t sub = lane >> 2;
  const uint32_t nq = hdr->total_q;
  const uint32_t qstep = gridDim.x * (kPkThreads / 32);
  uint32_t q = blockIdx.x * (kPkThreads / 32) + warp;  // warp-uniform
  // the load stream: tensor tl holds iterations [qbl, qel)
  int tl = -1;
  const uint4 *Wl = nullptr;
  uint32_t qbl = 0, qel = 0, nbl = 0;
  uint4 p0 = make_uint4(0u, 0u, 0u, 0u), p1 = p0;
  int tcur = -1;  // tensor of p0, p1
  if (q < nq) {
    do ++tl; while (q >= T[tl].q_begin + T[tl].nq);
    Wl = T[tl].pa.W;
    qbl = T[tl].q_begin;
    qel = qbl + T[tl].nq;
    nbl = (uint32_t)T[tl].pa.nblocks;
    tcur = tl;
    pk_load(Wl, nbl, (q - qbl) * 8 + sub, s, p0, p1);
  }
  ptx::grid_dep_wait();  // k_abs_sum_group complete: thresholds and g published
  __syncthreads();       // s_pair
  // the pack state of tensor tp
  int tp = -1;
  uint32_t qbp = 0, nbp = 0, bpr = 1, thr2 = 0;
  FastDiv div{};
  PlaneOut oa{}, ob{};
  while (q < nq) {
    const uint32_t qn = q + qstep;
    uint4 n0 = make_uint4(0u, 0u, 0u, 0u), n1 = n0;
    int tn = tcur;
    if (qn < nq) {
      if (qn >= qel) {
        do ++tl; while (qn >= T[tl].q_begin + T[tl].nq);
        Wl = T[tl].pa.W;
        qbl = T[tl].q_begin;
        qel = qbl + T[tl].nq;
        nbl = (uint32_t)T[tl].pa.nblocks;
      }
      tn = tl;
      pk_load(Wl, nbl, (qn - qbl) * 8 + sub, s, n0, n1);
    }
    if (tcur != tp) {
      tp = tcur;
      const PackGroupTensor &e = T[tp];
      qbp = e.q_begin;
      nbp = (uint32_t)e.pa.nblocks;
      bpr = e.pa.bpr;
      div = e.pa.div_bpr;
      oa = plane_out(e.pa);
      if (kMode == 2) ob = plane_out(e.pb);
      const uint32_t thr = slots[tp].thr;
      thr2 = thr | (thr << 16);
    }
    const uint32_t b = (q - qbp) * 8 + sub;
    const bool valid = b < nbp;
    const uint32_t row = fast_div(b, div);
    const uint32_t col = b - row * bpr;
    const bool row_end = col == bpr - 1;
    const uint32_t w[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
    const LaneFlags f = lane_flags(w, thr2);
    if constexpr (kMode == 0 || kMode == 2) {
      const LanePack r = pack_lane_6of8(w, f);
      if (valid) store_lane<false>(oa, r, row, col, row_end, s);
    }
    if constexpr (kMode == 1) {
      const LanePack r = pack_lane_2of4(w, f, s_pair, s);
      if (valid) store_lane<true>(oa, r, row, col, row_end, s);
    }
    if constexpr (kMode == 2) {
      const LanePack r = pack_lane_2of4(w, f, s_pair, s);
      if (valid) store_lane<true>(ob, r, row, col, row_end, s);
    }
    q = qn;
    tcur = tn;
    p0 = n0;
    p1 = n1;
  }
}

int64_t pack_group_plan_bytes(int count) {
  return (int64_t)sizeof(PackGroupHeader) + (int64_t)count * (int64_t)sizeof(PackGroupTensor);
}

sbn_status launch_pack_group(const PackGroupHeader *hdr_host, const void *plan_dev,
                             PackGroupSlot *slots, int32_t *err_flag, cudaStream_t st) {
  if (hdr_host->count == 0 || hdr_host->total_chunks == 0) return SBN_OK;
  const PackGroupHeader *hdr = static_cast<const PackGroupHeader *>(plan_dev);
  const PackGroupTensor *T = reinterpret_cast<const PackGroupTensor *>(hdr + 1);
  const int64_t cap = (int64_t)num_sms() * 4;
  int64_t g1 = hdr_host->total_chunks;
  if (g1 > cap) g1 = cap;
  sbn_status ls = launch_pdl(k_abs_sum_group, dim3((unsigned)g1), dim3(kAgThreads), 0, st, hdr, T,
                             slots, err_flag);
  if (ls != SBN_OK) return ls;
  const int per_sm = hdr_host->mode >= 0 ? kQgCtasPerSm : kPkCtasPerSm;
  int64_t g2 = ((int64_t)hdr_host->total_q + kPkThreads / 32 - 1) / (kPkThreads / 32);
  if (g2 > (int64_t)num_sms() * per_sm) g2 = (int64_t)num_sms() * per_sm;
  if (g2 < 1) g2 = 1;
  const dim3 grid2((unsigned)g2), block2(kPkThreads);
  switch (hdr_host->mode) {
    case 0: return launch_pdl(k_qmp_group_fixed<0>, grid2, block2, 0, st, hdr, T, slots);
    case 1: return launch_pdl(k_qmp_group_fixed<1>, grid2, block2, 0, st, hdr, T, slots);
    case 2: return launch_pdl(k_qmp_group_fixed<2>, grid2, block2, 0, st, hdr, T, slots);
    default: return launch_pdl(k_qmp_group, grid2, block2, 0, st, hdr, T, slots);
  }
}

}  // namespace sbn
