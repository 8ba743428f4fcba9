// Allocation-free variant of the weight pack entry point.
//
// Some callers cannot hand this library any device memory of their own: plugin hosts
// that own every allocation and give an operator no workspace, and serving loops that
// forbid cudaMalloc/cudaFree on their hot path because those calls can synchronise the
// whole device and fragment its memory.  For them the pack's only scratch -- the per-CTA
// partial sums of the absmean reduction and the arrival counter -- lives in a fixed
// array in this library's own device memory instead of a caller workspace.
#include "common.cuh"
#include "kernels.cuh"

namespace {

// The scratch: one pack workspace (kPackMaxParts partial sums + reserved words).  8448
// bytes on every GPU that loads the library, held until the process exits.
constexpr size_t kNoallocScratchBytes = 8448;
static_assert(sizeof(sbn::PackWorkspace) <= kNoallocScratchBytes, "scratch too small");
static __device__ __align__(256) unsigned char g_pack_scratch[kNoallocScratchBytes];

// Device address of g_pack_scratch in the current context.  In host code the symbol is
// only a host-side stand-in, so the address is looked up with the target device current.
// It is looked up on every call (no allocation, a host-side table lookup once the module
// is loaded) rather than cached: a cached address would go stale if the caller's context
// were destroyed and recreated (cudaDeviceReset) or a different context made current.
sbn_status scratch_for_current_device(void **out) {
  void *p = nullptr;
  if (cudaGetSymbolAddress(&p, g_pack_scratch) != cudaSuccess || !p) {
    (void)cudaGetLastError();
    return SBN_ERR_CUDA;
  }
  *out = p;
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
  // Nothing in the array needs clearing: the reduction kernel rewrites every partial sum
  // the quant/mask/pack kernel reads (one per CTA it launches), and the second kernel
  // waits for the first on the stream before reading them.
  return sbn_quantize_mask_pack_weights(W, out, in, n, m, eps, codes, meta, gamma_eff, scratch,
                                        dense_dbg, err_flag, stream);
}
