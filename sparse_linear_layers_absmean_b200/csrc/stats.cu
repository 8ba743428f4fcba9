// Mask statistics: by-products of the weight path that follow how the masks evolve over
// training steps.  Natural zeros (the Sparse-BitNet summaries, section 3 "Contribuciones
// Clave" item 1: a large share of the ternary codes is 0) and mask flips (section 2,
// "Recomputación Dinámica de Máscaras": the mask is rebuilt every step from the current
// masters, so the kept positions move).  Both are single streaming reductions with one
// 64-bit atomic per CTA.
#include "common.cuh"
#include "kernels.cuh"
#include "pack_common.cuh"
#include "ptx.cuh"

namespace sbn {

namespace {

constexpr int kStThreads = 256;
constexpr int kStLoads = 4;

// Adds the CTA's per-thread counts into *count (one atomic per CTA).
__device__ __forceinline__ void add_cta_count(unsigned long long v, unsigned long long *count) {
  __shared__ unsigned long long s_part[kStThreads / 32];
  v = warp_sum_u64(v);
  if ((threadIdx.x & 31) == 0) s_part[threadIdx.x >> 5] = v;
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned long long t = 0;
    for (int w = 0; w < kStThreads / 32; ++w) t += s_part[w];
    if (t) atomicAdd(count, t);
  }
}

// The ternary code of a weight is 0 exactly when its magnitude bits are below the pack's
// code threshold for the same g (the smallest bf16 magnitude with fl(|W| / g) > 0.5), so
// every CTA derives that threshold once and compares bits.
__global__ void __launch_bounds__(kStThreads)
    k_count_zero_codes(const uint4 *__restrict__ W, int64_t nvec,
                       const float *__restrict__ gamma_eff, unsigned long long *count) {
  ptx::grid_dep_launch();
  ptx::grid_dep_wait();  // the previous kernel on the stream (the pack) wrote g
  __shared__ uint32_t s_thr;
  if (threadIdx.x < 32) {
    const uint32_t thr = code_threshold_warp(__ldg(gamma_eff), (int)threadIdx.x);
    if (threadIdx.x == 0) s_thr = thr;
  }
  __syncthreads();
  const uint32_t thr = s_thr;
  uint32_t c = 0;
  const int64_t stride = (int64_t)gridDim.x * kStThreads;
  for (int64_t i = (int64_t)blockIdx.x * kStThreads + threadIdx.x; i < nvec;
       i += kStLoads * stride) {
    uint4 v[kStLoads];
#pragma unroll
    for (int u = 0; u < kStLoads; ++u)  // past the end: infinities, never a zero code
      v[u] = i + u * stride < nvec ? __ldg(W + i + u * stride)
                                   : make_uint4(0x7f807f80u, 0x7f807f80u, 0x7f807f80u, 0x7f807f80u);
#pragma unroll
    for (int u = 0; u < kStLoads; ++u) {
      const uint32_t w4[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
      for (int q = 0; q < 4; ++q)
        c += (uint32_t)((w4[q] & 0x7fffu) < thr) + (uint32_t)(((w4[q] >> 16) & 0x7fffu) < thr);
    }
  }
  add_cta_count(c, count);
}

// A 2:4 metadata byte (two nibbles i0 | i1 << 2) -> its keep byte (bits i0 and i1 of each
// nibble).  A zero padding byte maps to the same keep byte in both planes.
__device__ __forceinline__ uint32_t keep_byte_of_index_pairs(uint32_t b) {
  const uint32_t n0 = b & 15u, n1 = (b >> 4) & 15u;
  return ((1u << (n0 & 3u)) | (1u << (n0 >> 2))) | (((1u << (n1 & 3u)) | (1u << (n1 >> 2))) << 4);
}

__device__ __forceinline__ uint32_t keep_word(const uint8_t *s_keep, uint32_t w) {
  return (uint32_t)s_keep[w & 255u] | ((uint32_t)s_keep[(w >> 8) & 255u] << 8) |
         ((uint32_t)s_keep[(w >> 16) & 255u] << 16) | ((uint32_t)s_keep[w >> 24] << 24);
}

__global__ void __launch_bounds__(kStThreads)
    k_count_mask_flips(const uint4 *__restrict__ a, const uint4 *__restrict__ b, int64_t nvec,
                       int index_pairs, unsigned long long *count) {
  __shared__ uint8_t s_keep[256];  // 2:4: metadata byte -> keep byte
  ptx::grid_dep_launch();
  s_keep[threadIdx.x] = (uint8_t)keep_byte_of_index_pairs(threadIdx.x);
  __syncthreads();
  ptx::grid_dep_wait();  // the previous kernel on the stream (the pack) wrote the planes
  uint32_t c = 0;
  const int64_t stride = (int64_t)gridDim.x * kStThreads;
  for (int64_t i = (int64_t)blockIdx.x * kStThreads + threadIdx.x; i < nvec; i += 2 * stride) {
    uint4 va[2], vb[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const bool in = i + u * stride < nvec;
      va[u] = in ? __ldg(a + i + u * stride) : make_uint4(0u, 0u, 0u, 0u);
      vb[u] = in ? __ldg(b + i + u * stride) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const uint32_t wa[4] = {va[u].x, va[u].y, va[u].z, va[u].w};
      const uint32_t wb[4] = {vb[u].x, vb[u].y, vb[u].z, vb[u].w};
#pragma unroll
      for (int q = 0; q < 4; ++q)
        c += index_pairs ? __popc(keep_word(s_keep, wa[q]) ^ keep_word(s_keep, wb[q]))
                         : __popc(wa[q] ^ wb[q]);
    }
  }
  add_cta_count(c, count);
}

int64_t stats_grid(int64_t nvec, int64_t per_thread) {
  int64_t grid = (nvec + kStThreads * per_thread - 1) / (kStThreads * per_thread);
  const int64_t cap = (int64_t)num_sms() * 8;
  if (grid > cap) grid = cap;
  return grid < 1 ? 1 : grid;
}

}  // namespace

sbn_status launch_count_zero_codes(const void *W, int64_t n, const float *gamma_eff,
                                   unsigned long long *count, cudaStream_t st) {
  const int64_t nvec = n / 8;  // n is a multiple of 64
  return launch_pdl(k_count_zero_codes, dim3((unsigned)stats_grid(nvec, kStLoads)),
                    dim3(kStThreads), 0, st, reinterpret_cast<const uint4 *>(W), nvec, gamma_eff,
                    count);
}

sbn_status launch_count_mask_flips(const uint8_t *meta_a, const uint8_t *meta_b, int64_t nbytes,
                                   bool index_pairs, unsigned long long *count, cudaStream_t st) {
  const int64_t nvec = nbytes / 16;  // rows are padded to 16 bytes
  return launch_pdl(k_count_mask_flips, dim3((unsigned)stats_grid(nvec, 2)), dim3(kStThreads), 0,
                    st, reinterpret_cast<const uint4 *>(meta_a),
                    reinterpret_cast<const uint4 *>(meta_b), nvec, index_pairs ? 1 : 0, count);
}

}  // namespace sbn
