// Allocation-free variant of the weight pack entry point.
//
// Some callers cannot hand this library any device memory of their own: plugin hosts
// that own every allocation and give an operator no workspace, and serving loops that
// forbid cudaMalloc/cudaFree on their hot path because those calls can synchronise the
// whole device and fragment its memory.  For them the pack's only scratch -- the per-CTA
// partial sums of the absmean reduction and the arrival counter -- lives in a fixed
// array in this library's own device memory instead of a caller workspace.
#include <mutex>

#include "common.cuh"
#include "kernels.cuh"

namespace {

// The scratch: one pack workspace (kPackMaxParts partial sums + counter + published
// values).  8448 bytes on every GPU that loads the library, held until the process exits.
constexpr size_t kNoallocScratchBytes = 8448;
static_assert(sizeof(sbn::PackWorkspace) <= kNoallocScratchBytes, "scratch too small");
static __device__ __align__(256) unsigned char g_pack_scratch[kNoallocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void *g_scratch_addr[kMaxDevices] = {};

// Device address of g_pack_scratch on the current device.  In host code the symbol
// itself is only a host-side stand-in, so the address is looked up once per device
// (with that device current) and cached.
sbn_status scratch_for_current_device(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SBN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_scratch_addr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_pack_scratch) != cudaSuccess || !p) return SBN_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return SBN_OK;
}

}  // namespace

extern "C" SBN_API sbn_status sbn_quantize_mask_pack_weights_noalloc(
    const void *W, int64_t out, int64_t in, int n, int m, float eps, uint8_t *codes,
    uint8_t *meta, float *gamma_eff, int8_t *dense_dbg, int32_t *err_flag, void *stream) {
  sbn_dims d;
  sbn_status st = sbn_linear_ref_dims(out, in, n, m, &d);
  if (st != SBN_OK) return st;
  // The reduction never uses more than kPackMaxParts partial sums, whatever the size, so
  // the fixed scratch always suffices; a build where it would not is refused here.
  if ((size_t)d.pack_workspace_bytes > kNoallocScratchBytes) return SBN_ERR_SHAPE;
  if (!W || !codes || !meta || !gamma_eff) return SBN_ERR_NULL;
  if (!(eps >= 0.0f) || eps > 3.4028235e38f) return SBN_ERR_ARG;
  const uintptr_t mis = reinterpret_cast<uintptr_t>(W) | reinterpret_cast<uintptr_t>(codes) |
                        reinterpret_cast<uintptr_t>(meta) | reinterpret_cast<uintptr_t>(dense_dbg);
  if ((mis & 15u) || (reinterpret_cast<uintptr_t>(gamma_eff) & 3u) ||
      (reinterpret_cast<uintptr_t>(err_flag) & 3u))
    return SBN_ERR_ALIGN;
  void *scratch = nullptr;
  if ((st = scratch_for_current_device(&scratch)) != SBN_OK) return st;
  // The array keeps whatever the previous call left; the arrival counter must start at 0.
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(static_cast<unsigned char *>(scratch) + offsetof(sbn::PackWorkspace, ticket),
                      0, sizeof(unsigned int), s) != cudaSuccess)
    return SBN_ERR_CUDA;
  return sbn_quantize_mask_pack_weights(W, out, in, n, m, eps, codes, meta, gamma_eff, scratch,
                                        dense_dbg, err_flag, stream);
}
