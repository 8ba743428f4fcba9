// Weight path of the Sparse-BitLinear forward: absmean scale, ternary codes, N:M mask
// from the master magnitudes applied after quantisation, and the 2-bit + metadata pack.
// (Sparse-BitNet technical summaries, section 2 "Methodology": Sparse-BitLinear items 1-2,
// mask generation from the BF16 masters, quant-then-mask order.)
//
// Two launches on the caller's stream.  6:8 and 2:4 use pack_fast.cu (keep masks and the
// sum in the first launch, codes in the second); every other N:M pattern uses:
//   k_abs_sum          exact integer sum S = sum trunc(|W| * 2^24), one partial per CTA in
//                      the workspace (eight 16-byte loads in flight per thread).
//   k_quant_mask_pack  every CTA first turns the partials into g and the code threshold
//                      (pack_common.cuh), then one pass over W: each lane owns 8
//                      consecutive weights, computes the keep mask of its group(s) and the
//                      codes, and the lanes of a 64-weight block assemble their packed
//                      words by shuffles.
#include "common.cuh"
#include "kernels.cuh"
#include "pack_common.cuh"
#include "ptx.cuh"

namespace sbn {

// ---------------------------------------------------------------------------------------
// S1: per-tensor absmean scale.
// ---------------------------------------------------------------------------------------

// One pass over W at the full HBM bandwidth: four CTAs of 256 threads per SM, four 16-byte
// loads in flight per thread, one fp64 add per weight (pack_common.cuh) and a packed
// 16-bit max for the range check.  One partial sum per CTA goes to the workspace.
constexpr int kAsThreads = 256;
constexpr int kAsLoads = 4;

__global__ void __launch_bounds__(kAsThreads, 4) k_abs_sum(const uint4 *__restrict__ W, int64_t nvec,
                                                         PackWorkspace *ws, int32_t *err_flag) {
  // A programmatic dependent of the previous kernel on the stream (which may write W): wait
  // for it first, then let the quant/mask/pack kernel launch.  That kernel requests W
  // before its own wait, so W must be final by the time it can start.
  ptx::grid_dep_wait();
  ptx::grid_dep_launch();
  double acc0 = kAccBias, acc1 = kAccBias;
  uint32_t mx = 0;  // largest magnitude bits seen, per 16-bit half
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const int64_t i0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  for (int64_t i = i0; i < nvec; i += kAsLoads * stride) {
    uint4 v[kAsLoads];
#pragma unroll
    for (int u = 0; u < kAsLoads; ++u)
      v[u] = i + u * stride < nvec ? __ldg(W + i + u * stride) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int u = 0; u < kAsLoads; ++u) {  // zero words add nothing
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
  // Rare path: some |W| >= 256 (or NaN/Inf).  Re-read this thread's weights to tell the
  // two error kinds apart.
  uint32_t mx_all = 0, mx_fin = 0;
  if (max(mx & 0xffffu, mx >> 16) >= kBf16Mag256Bits) {
    for (int64_t j = i0; j < nvec; j += stride) {
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
  __shared__ unsigned long long s_sum[kAsThreads / 32];
  __shared__ uint32_t s_all[kAsThreads / 32], s_fin[kAsThreads / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  acc = warp_sum_u64(acc);
  uint32_t ma = warp_max_u32(mx_all);
  uint32_t mf = warp_max_u32(mx_fin);
  if (lane == 0) {
    s_sum[warp] = acc;
    s_all[warp] = ma;
    s_fin[warp] = mf;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned long long sum = 0;
    uint32_t a = 0, f = 0;
    for (int w = 0; w < kAsThreads / 32; ++w) {
      sum += s_sum[w];
      a = max(a, s_all[w]);
      f = max(f, s_fin[w]);
    }
    ws->part[blockIdx.x] = sum;
    int flags = 0;
    if (a >= kBf16InfBits) flags |= SBN_FLAG_W_NONFINITE;
    if (f >= kBf16Mag256Bits) flags |= SBN_FLAG_W_RANGE;
    if (flags && err_flag) atomicOr(err_flag, flags);
  }
}

// ---------------------------------------------------------------------------------------
// S2-S4: codes, mask, pack.
// ---------------------------------------------------------------------------------------

// Keep mask of one group of M magnitudes: the N largest, the lower index winning ties.
// Keys (mag << 3) | (M-1-i) are distinct and order exactly like that rule.
template <int N, int M>
__device__ __forceinline__ uint32_t group_keep(const uint32_t *mag) {
  if constexpr (N == M) {
    return (1u << M) - 1u;
  } else {
    uint32_t key[M];
#pragma unroll
    for (int i = 0; i < M; ++i) key[i] = (mag[i] << 3) | (uint32_t)(M - 1 - i);
    uint32_t keep = 0;
    if constexpr (M - N <= N) {
      // drop the M-N smallest keys: tau = (M-N)-th smallest
      constexpr int D = M - N;
      uint32_t s[D];
#pragma unroll
      for (int d = 0; d < D; ++d) s[d] = 0xffffffffu;
#pragma unroll
      for (int i = 0; i < M; ++i) {
        uint32_t x = key[i];
#pragma unroll
        for (int d = 0; d < D; ++d) {
          uint32_t lo = min(s[d], x);
          x = max(s[d], x);
          s[d] = lo;
        }
      }
#pragma unroll
      for (int i = 0; i < M; ++i) keep |= (uint32_t)(key[i] > s[D - 1]) << i;
    } else {
      // keep the N largest keys: tau = N-th largest
      uint32_t s[N];
#pragma unroll
      for (int d = 0; d < N; ++d) s[d] = 0u;
#pragma unroll
      for (int i = 0; i < M; ++i) {
        uint32_t x = key[i];
#pragma unroll
        for (int d = 0; d < N; ++d) {
          uint32_t hi = max(s[d], x);
          x = min(s[d], x);
          s[d] = hi;
        }
      }
#pragma unroll
      for (int i = 0; i < M; ++i) keep |= (uint32_t)(key[i] >= s[N - 1]) << i;
    }
    return keep;
  }
}

// bits 0..3 of x -> bit 0 of bytes 0..3
__device__ __forceinline__ uint32_t spread4_to_bytes(uint32_t x) {
  return (x * 0x00204081u) & 0x01010101u;
}

// For a 2:4 keep nibble with exactly two bits set: the meta nibble i0 | i1 << 2.
// Table indexed by the keep nibble (4 bits per entry); other entries are unused.
constexpr unsigned long long kPairNibbleLut =
    (4ull << (4 * 0x3)) | (8ull << (4 * 0x5)) | (9ull << (4 * 0x6)) | (12ull << (4 * 0x9)) |
    (13ull << (4 * 0xA)) | (14ull << (4 * 0xC));

template <int N, int M>
struct QmpArgs {
  const uint4 *W;
  int64_t nblocks;
  uint32_t bpr;
  FastDiv div_bpr;
  const PackWorkspace *ws;
  uint8_t *codes;
  int64_t ldc, codes_row_bytes;
  uint8_t *meta;
  int64_t ldm, meta_row_bytes;
  int8_t *dense_dbg;
  int nparts;
  int64_t n;
  float eps;
  float *gamma_eff;
};

// One 64-weight block per 8 lanes: lane `sub` owns weights 8*sub .. 8*sub+7 of block b.
template <int N, int M>
__device__ __forceinline__ void qmp_block(const QmpArgs<N, M> &a, uint4 v, int64_t b, int sub,
                                          uint32_t thr) {
  constexpr bool kCompact = (N == 2 && M == 4);
  constexpr int kCodeBytesPerBlock = kCompact ? 8 : 16;  // 32 or 64 stored elements
  const bool valid = b < a.nblocks;
  const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
  uint32_t mag[8];
  uint32_t neg = 0;
#pragma unroll
  for (int p = 0; p < 8; ++p) {
    const uint32_t h = (w4[p >> 1] >> (16 * (p & 1))) & 0xffffu;
    mag[p] = h & 0x7fffu;
    neg |= (h >> 15) << p;
  }
  uint32_t keep;
  if constexpr (M == 8) {
    keep = group_keep<N, 8>(mag);
  } else {
    keep = group_keep<N, 4>(mag) | (group_keep<N, 4>(mag + 4) << 4);
  }
  uint32_t nz = 0;
#pragma unroll
  for (int p = 0; p < 8; ++p) nz |= (uint32_t)(mag[p] >= thr) << p;
  const uint32_t nzneg = nz & neg;

  uint32_t word, meta_byte;
  if constexpr (kCompact) {
    // stored elements 4*sub .. 4*sub+3 = (group A kept i0, i1, group B kept i0, i1);
    // they are j = sub % 4 of word sub / 4, bytes 0..3, bit 6 - 2j.
    const uint32_t nibA = (uint32_t)(kPairNibbleLut >> (4 * (keep & 15u))) & 15u;
    const uint32_t nibB = (uint32_t)(kPairNibbleLut >> (4 * (keep >> 4))) & 15u;
    const uint32_t pos0 = nibA & 3u, pos1 = nibA >> 2, pos2 = 4u + (nibB & 3u),
                   pos3 = 4u + (nibB >> 2);
    // bit 0 of byte k <- "non-zero" at the k-th kept position; bit 1 <- "negative"
    const uint32_t lo = ((nz >> pos0) & 1u) | (((nz >> pos1) & 1u) << 8) |
                        (((nz >> pos2) & 1u) << 16) | (((nz >> pos3) & 1u) << 24);
    const uint32_t hi = ((nzneg >> pos0) & 1u) | (((nzneg >> pos1) & 1u) << 8) |
                        (((nzneg >> pos2) & 1u) << 16) | (((nzneg >> pos3) & 1u) << 24);
    word = (lo | (hi << 1)) << (6 - 2 * (sub & 3));
    meta_byte = nibA | (nibB << 4);
    word |= __shfl_xor_sync(0xffffffffu, word, 1);
    word |= __shfl_xor_sync(0xffffffffu, word, 2);
  } else {
    // stored elements 8*sub + p: word sub/2, j = 2*(sub&1) + p/4, byte p%4;
    // pruned positions hold the code of 0
    const int jb = 2 * (sub & 1);
    const uint32_t kn = nz & keep, kneg = nzneg & keep;
    const uint32_t c_lo = spread4_to_bytes(kn & 15u) | (spread4_to_bytes(kneg & 15u) << 1);
    const uint32_t c_hi = spread4_to_bytes(kn >> 4) | (spread4_to_bytes(kneg >> 4) << 1);
    word = (c_lo << (6 - 2 * jb)) | (c_hi << (4 - 2 * jb));
    meta_byte = keep;  // M == 8: one group; M == 4: group A low nibble, B high nibble
    word |= __shfl_xor_sync(0xffffffffu, word, 1);
  }
  uint32_t mword = meta_byte << (8 * (sub & 3));
  mword |= __shfl_xor_sync(0xffffffffu, mword, 1);
  mword |= __shfl_xor_sync(0xffffffffu, mword, 2);
  if (!valid) return;
  const uint32_t row = fast_div((uint32_t)b, a.div_bpr);
  const uint32_t col = (uint32_t)b - row * a.bpr;
  uint8_t *crow = a.codes + (int64_t)row * a.ldc + col * kCodeBytesPerBlock;
  if constexpr (kCompact) {
    if ((sub & 3) == 0) reinterpret_cast<uint32_t *>(crow)[sub >> 2] = word;
  } else {
    if ((sub & 1) == 0) reinterpret_cast<uint32_t *>(crow)[sub >> 1] = word;
  }
  uint8_t *mrow = a.meta + (int64_t)row * a.ldm + col * 8;
  if ((sub & 3) == 0) reinterpret_cast<uint32_t *>(mrow)[sub >> 2] = mword;
  if (col == a.bpr - 1 && sub == 0) {
    // zero padding up to the 16-byte row stride (0 or 8 bytes)
    if (a.ldc > a.codes_row_bytes)
      *reinterpret_cast<uint2 *>(a.codes + (int64_t)row * a.ldc + a.codes_row_bytes) =
          make_uint2(0u, 0u);
    if (a.ldm > a.meta_row_bytes)
      *reinterpret_cast<uint2 *>(a.meta + (int64_t)row * a.ldm + a.meta_row_bytes) =
          make_uint2(0u, 0u);
  }
  if (a.dense_dbg) {
    // masked ternary values, one int8 per position
    const uint32_t kn = keep & nz, kneg = keep & nzneg;
    const uint32_t lo4 = spread4_to_bytes(kn & 15u) | (spread4_to_bytes(kneg & 15u) * 0xfeu);
    const uint32_t hi4 = spread4_to_bytes(kn >> 4) | (spread4_to_bytes(kneg >> 4) * 0xfeu);
    *reinterpret_cast<uint2 *>(a.dense_dbg + b * 64 + sub * 8) = make_uint2(lo4, hi4);
  }
}

template <int N, int M>
__global__ void __launch_bounds__(256) k_quant_mask_pack(const QmpArgs<N, M> a) {
  const uint32_t thr = pack_prologue(a.ws, a.nparts, a.n, a.eps, a.gamma_eff);
  const int lane = threadIdx.x & 31;
  const int sub = lane & 7;
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
  const int64_t nquads = (a.nblocks + 3) >> 2;
  const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
  // each warp takes quads q and q + nwarps per iteration: two 16-byte loads in flight
  for (int64_t q = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; q < nquads;
       q += 2 * nwarps) {
    const int64_t b0 = 4 * q + (lane >> 3);
    const int64_t b1 = b0 + 4 * nwarps;
    const uint4 v0 = b0 < a.nblocks ? __ldg(a.W + b0 * 8 + sub) : zero;
    const uint4 v1 = b1 < a.nblocks ? __ldg(a.W + b1 * 8 + sub) : zero;
    qmp_block<N, M>(a, v0, b0, sub, thr);
    if (q + nwarps < nquads) qmp_block<N, M>(a, v1, b1, sub, thr);
  }
}

// ---------------------------------------------------------------------------------------
// Group quantisation: G blocks along the input dimension K, each with its own absmean scale
// g_j.  k_gq_abs_sum leaves P exact partial sums per group (CTA (p, j) of the grid takes
// every P-th 64-weight block of group j); k_gq_quant_mask_pack turns them into the G
// scales and code thresholds in its prologue and packs as k_quant_mask_pack does, each
// 64-weight block with its group's threshold (K / G is a multiple of 64, so no block
// straddles two groups).
// ---------------------------------------------------------------------------------------
constexpr int kGqMaxGroups = 64;

__global__ void __launch_bounds__(kAsThreads)
    k_gq_abs_sum(const uint4 *__restrict__ W, int64_t O, int64_t K, int G,
                 PackWorkspace *ws, int32_t *err_flag) {
  ptx::grid_dep_wait();
  ptx::grid_dep_launch();
  const int j = blockIdx.y, P = gridDim.x;
  const int64_t bpg = K / G / 64;  // 64-weight blocks per row of a group
  const int64_t nb = O * bpg;
  double acc0 = kAccBias, acc1 = kAccBias;
  uint32_t mx = 0, mx_fin = 0, mx_all = 0;
  for (int64_t i = (int64_t)blockIdx.x * (blockDim.x / 8) + (threadIdx.x >> 3); i < nb;
       i += (int64_t)P * (blockDim.x / 8)) {
    const int64_t r = i / bpg, b = i - r * bpg;
    // 8 threads per block, one 16-byte word each
    const uint4 v = __ldg(W + (r * K + (int64_t)j * (K / G) + b * 64) / 8 + (threadIdx.x & 7));
    const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      asm("max.u16x2 %0, %0, %1;" : "+r"(mx) : "r"(w4[q] & 0x7fff7fffu));
      acc0 = __dadd_rz(acc0, mag_lo_x2p128(w4[q]));
      acc1 = __dadd_rz(acc1, mag_hi_x2p128(w4[q]));
      for (int h = 0; h < 2; ++h) {
        const uint32_t m = (w4[q] >> (16 * h)) & 0x7fffu;
        mx_all = max(mx_all, m);
        if (m < kBf16InfBits) mx_fin = max(mx_fin, m);
      }
    }
  }
  unsigned long long acc = warp_sum_u64(acc_value(acc0) + acc_value(acc1));
  const uint32_t ma = warp_max_u32(mx_all), mf = warp_max_u32(mx_fin);
  __shared__ unsigned long long s_sum[kAsThreads / 32];
  __shared__ uint32_t s_all[kAsThreads / 32], s_fin[kAsThreads / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) {
    s_sum[warp] = acc;
    s_all[warp] = ma;
    s_fin[warp] = mf;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned long long sum = 0;
    uint32_t a = 0, f = 0;
    for (int w = 0; w < kAsThreads / 32; ++w) {
      sum += s_sum[w];
      a = max(a, s_all[w]);
      f = max(f, s_fin[w]);
    }
    ws->part[j * P + blockIdx.x] = sum;
    int flags = 0;
    if (a >= kBf16InfBits) flags |= SBN_FLAG_W_NONFINITE;
    if (f >= kBf16Mag256Bits) flags |= SBN_FLAG_W_RANGE;
    if (flags && err_flag) atomicOr(err_flag, flags);
  }
  (void)mx;
}

template <int N, int M>
__global__ void __launch_bounds__(256)
    k_gq_quant_mask_pack(const QmpArgs<N, M> a, int G, int P, uint32_t bpg, FastDiv div_bpg) {
  __shared__ uint32_t s_thr[kGqMaxGroups];
  ptx::grid_dep_launch();
  ptx::grid_dep_wait();
  // prologue: warp w finishes groups w, w + 8, ...: exact sum of the group's P partials,
  // g_j = fp32(fp32(fp64(S_j) / (fp64(n / G) * 2^24)) + eps), code threshold of g_j
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int j = warp; j < G; j += blockDim.x >> 5) {
    unsigned long long S = 0;
    for (int i = lane; i < P; i += 32) S += a.ws->part[j * P + i];
    S = warp_sum_u64(S);
    const double mean = __ddiv_rn(__ull2double_rn(S), (double)(a.n / G) * 16777216.0);
    const float g = __fadd_rn(__double2float_rn(mean), a.eps);
    const uint32_t thr = code_threshold_warp(g, lane);
    if (lane == 0) {
      s_thr[j] = thr;
      if (blockIdx.x == 0) a.gamma_eff[j] = g;
    }
  }
  __syncthreads();
  const int sub = lane & 7;
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
  const int64_t nquads = (a.nblocks + 3) >> 2;
  const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
  auto thr_of = [&](int64_t b) -> uint32_t {
    if (b >= a.nblocks) return s_thr[0];
    const uint32_t row = fast_div((uint32_t)b, a.div_bpr);
    const uint32_t col = (uint32_t)b - row * a.bpr;
    return s_thr[fast_div(col, div_bpg)];
  };
  for (int64_t q = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; q < nquads;
       q += 2 * nwarps) {
    const int64_t b0 = 4 * q + (lane >> 3);
    const int64_t b1 = b0 + 4 * nwarps;
    const uint4 v0 = b0 < a.nblocks ? __ldg(a.W + b0 * 8 + sub) : zero;
    const uint4 v1 = b1 < a.nblocks ? __ldg(a.W + b1 * 8 + sub) : zero;
    qmp_block<N, M>(a, v0, b0, sub, thr_of(b0));
    if (q + nwarps < nquads) qmp_block<N, M>(a, v1, b1, sub, thr_of(b1));
  }
  (void)bpg;
}

// ---------------------------------------------------------------------------------------
// Host launchers
// ---------------------------------------------------------------------------------------

// SM count of the current device (cached per device; a concurrent first query stores the
// same value).
int num_sms() {
  constexpr int kMaxDevices = 64;
  static int cache[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) {
    (void)cudaGetLastError();
    return 148;
  }
  if (dev < kMaxDevices && cache[dev] > 0) return cache[dev];
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      sms < 1) {
    (void)cudaGetLastError();
    sms = 148;
  }
  if (dev < kMaxDevices) cache[dev] = sms;
  return sms;
}

FastDiv make_fast_div(uint32_t d) {
  FastDiv f;
  if (d == 1) {
    f.mul = 0;
    f.shift = 0xffffffffu;
    return f;
  }
  uint32_t L = 0;
  while ((1u << L) < d) ++L;
  f.mul = (uint32_t)(((1ull << (31 + L)) + d - 1) / d);
  f.shift = L - 1;
  return f;
}

template <int N, int M>
static void launch_qmp(const uint4 *W, int64_t nblocks, int64_t bpr, const PackWorkspace *ws,
                       uint8_t *codes, int64_t ldc, int64_t crow, uint8_t *meta, int64_t ldm,
                       int64_t mrow, int8_t *dense_dbg, int nparts, int64_t n, float eps,
                       float *gamma_eff, cudaStream_t st) {
  const int threads = 256;
  const int64_t nquads = (nblocks + 3) / 4;
  int64_t grid = (nquads + 15) / 16;  // 8 warps x 2 quads per CTA iteration
  const int64_t cap = (int64_t)num_sms() * 8;
  if (grid > cap) grid = cap;
  if (grid < 1) grid = 1;
  QmpArgs<N, M> a{W,    nblocks,   (uint32_t)bpr, make_fast_div((uint32_t)bpr), ws, codes, ldc,
                  crow, meta,      ldm,           mrow,          dense_dbg,    nparts, n,
                  eps,  gamma_eff};
  k_quant_mask_pack<N, M><<<(unsigned)grid, threads, 0, st>>>(a);
}

sbn_status launch_pack(const void *W, int64_t out, int64_t in, int n, int m, float eps,
                       uint8_t *codes, int64_t ldc, int64_t crow, uint8_t *meta, int64_t ldm,
                       int64_t mrow, float *gamma_eff, PackWorkspace *ws, int8_t *dense_dbg,
                       int32_t *err_flag, cudaStream_t st) {
  const int64_t nel = out * in;
  const uint4 *W4 = reinterpret_cast<const uint4 *>(W);
  const int64_t nblocks = nel / 64, bpr = in / 64;
  // S1 for every pattern: one exact partial sum per CTA
  const int64_t nvec = nel / 8;
  int64_t grid = (nvec + kAsThreads * kAsLoads - 1) / (kAsThreads * kAsLoads);
  const int64_t cap = (int64_t)num_sms() * 4;  // one wave of 4 CTAs per SM
  if (grid > cap) grid = cap;
  if (grid > kPackMaxParts) grid = kPackMaxParts;
  if (grid < 1) grid = 1;
  const int nparts = (int)grid;
  const sbn_status ls = launch_pdl(k_abs_sum, dim3((unsigned)grid), dim3(kAsThreads), 0, st, W4,
                                   nvec, ws, err_flag);
  if (ls != SBN_OK) return ls;
  if ((n == 6 && m == 8) || (n == 2 && m == 4)) {
    FastPackArgs fa{W4,  nblocks, (uint32_t)bpr, make_fast_div((uint32_t)bpr),
                    ws,  codes,   ldc,           crow,
                    meta, ldm,    mrow,          dense_dbg,
                    nparts, nel,  eps,           gamma_eff};
    return launch_fast_pack(fa, n == 2, st);
  }
#define SBN_QMP(NN, MM)                                                                    \
  case (NN * 16 + MM):                                                                     \
    launch_qmp<NN, MM>(W4, nblocks, bpr, ws, codes, ldc, crow, meta, ldm, mrow, dense_dbg, \
                       nparts, nel, eps, gamma_eff, st);                                   \
    break;
  switch (n * 16 + m) {
    SBN_QMP(1, 4)
    SBN_QMP(2, 4)
    SBN_QMP(3, 4)
    SBN_QMP(4, 4)
    SBN_QMP(1, 8)
    SBN_QMP(2, 8)
    SBN_QMP(3, 8)
    SBN_QMP(4, 8)
    SBN_QMP(5, 8)
    SBN_QMP(6, 8)
    SBN_QMP(7, 8)
    SBN_QMP(8, 8)
    default:
      return SBN_ERR_PATTERN;
  }
#undef SBN_QMP
  SBN_LAUNCH_CHECK();
  return SBN_OK;
}

template <int N, int M>
static sbn_status launch_gq_qmp(const uint4 *W, int64_t nblocks, int64_t bpr, int64_t bpg, int G,
                                int P, const PackWorkspace *ws, uint8_t *codes, int64_t ldc,
                                int64_t crow, uint8_t *meta, int64_t ldm, int64_t mrow,
                                int8_t *dense_dbg, int64_t n, float eps, float *gamma_eff,
                                cudaStream_t st) {
  const int64_t nquads = (nblocks + 3) / 4;
  int64_t grid = (nquads + 15) / 16;
  const int64_t cap = (int64_t)num_sms() * 8;
  if (grid > cap) grid = cap;
  if (grid < 1) grid = 1;
  QmpArgs<N, M> a{W,    nblocks,   (uint32_t)bpr, make_fast_div((uint32_t)bpr), ws, codes, ldc,
                  crow, meta,      ldm,           mrow,          dense_dbg,    P,  n,
                  eps,  gamma_eff};
  return launch_pdl(k_gq_quant_mask_pack<N, M>, dim3((unsigned)grid), dim3(256), 0, st, a, G, P,
                    (uint32_t)bpg, make_fast_div((uint32_t)bpg));
}

sbn_status launch_pack_gq(const void *W, int64_t out, int64_t in, int n, int m, int G, float eps,
                          uint8_t *codes, int64_t ldc, int64_t crow, uint8_t *meta, int64_t ldm,
                          int64_t mrow, float *gamma_eff, PackWorkspace *ws, int8_t *dense_dbg,
                          int32_t *err_flag, cudaStream_t st) {
  if (G < 1 || G > kGqMaxGroups) return SBN_ERR_SHAPE;
  const uint4 *W4 = reinterpret_cast<const uint4 *>(W);
  const int64_t nblocks = out * in / 64, bpr = in / 64, bpg = bpr / G;
  // P CTAs per group, at most kPackMaxParts partial sums in all
  int64_t P = ((int64_t)num_sms() * 4 + G - 1) / G;
  const int64_t per_group = (out * bpg + (kAsThreads / 8) - 1) / (kAsThreads / 8);
  if (P > per_group) P = per_group;
  if (P > kPackMaxParts / G) P = kPackMaxParts / G;
  if (P < 1) P = 1;
  sbn_status s = launch_pdl(k_gq_abs_sum, dim3((unsigned)P, (unsigned)G), dim3(kAsThreads), 0, st,
                            W4, out, in, G, ws, err_flag);
  if (s != SBN_OK) return s;
  const int64_t nel = out * in;
#define SBN_GQMP(NN, MM)                                                                       \
  case (NN * 16 + MM):                                                                         \
    return launch_gq_qmp<NN, MM>(W4, nblocks, bpr, bpg, G, (int)P, ws, codes, ldc, crow, meta, \
                                 ldm, mrow, dense_dbg, nel, eps, gamma_eff, st);
  switch (n * 16 + m) {
    SBN_GQMP(1, 4)
    SBN_GQMP(2, 4)
    SBN_GQMP(3, 4)
    SBN_GQMP(4, 4)
    SBN_GQMP(1, 8)
    SBN_GQMP(2, 8)
    SBN_GQMP(3, 8)
    SBN_GQMP(4, 8)
    SBN_GQMP(5, 8)
    SBN_GQMP(6, 8)
    SBN_GQMP(7, 8)
    SBN_GQMP(8, 8)
    default:
      return SBN_ERR_PATTERN;
  }
#undef SBN_GQMP
}

}  // namespace sbn
