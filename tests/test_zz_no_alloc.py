"""The allocation-free weight pack, for callers that cannot give the library device
memory (plugin hosts that hand an operator no workspace, serving loops that forbid
cudaMalloc/cudaFree on the hot path).  It must produce exactly what the regular pack
entry point produces with a caller workspace.  Collected last on purpose: it touches the
library's process-wide scratch array."""
import ctypes

import numpy as np
import pytest
import torch

import sparse_linear_layers_absmean_b200 as sbn
import workloads

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def _vp(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _outputs(O, K, n, m):
    d = sbn.sbn_linear_ref_dims(O, K, n, m)
    return dict(codes=torch.empty((O, d.codes_ld), dtype=torch.uint8, device="cuda"),
                meta=torch.empty((O, d.meta_ld), dtype=torch.uint8, device="cuda"),
                g=torch.empty(1, dtype=torch.float32, device="cuda"),
                dense=torch.empty((O, K), dtype=torch.int8, device="cuda"),
                err=torch.zeros(1, dtype=torch.int32, device="cuda"))


def _regular(W, n, m, eps):
    O, K = W.shape
    o = _outputs(O, K, n, m)
    ws = sbn.new_workspace(O, K, n, m)
    st = sbn.lib().sbn_quantize_mask_pack_weights(
        _vp(W), O, K, n, m, ctypes.c_float(eps), _vp(o["codes"]), _vp(o["meta"]), _vp(o["g"]),
        _vp(ws), _vp(o["dense"]), _vp(o["err"]), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0
    return o


def _noalloc(W, n, m, eps):
    O, K = W.shape
    o = _outputs(O, K, n, m)
    st = sbn.lib().sbn_quantize_mask_pack_weights_noalloc(
        _vp(W), O, K, n, m, ctypes.c_float(eps), _vp(o["codes"]), _vp(o["meta"]), _vp(o["g"]),
        _vp(o["dense"]), _vp(o["err"]), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0
    return o


@pytest.mark.parametrize("n,m,O,K", [(2, 4, 300, 640), (6, 8, 6912, 2560), (3, 8, 37, 192)])
def test_noalloc_matches_regular_pack_twice(n, m, O, K):
    # two calls in a row on different masters: the second must not see the first's state
    for seed in (1, 2):
        W = workloads.torch_bf16(workloads.masters(O, K, seed=seed + 10 * n), "cuda")
        a = _noalloc(W, n, m, 1e-5)
        b = _regular(W, n, m, 1e-5)
        torch.cuda.synchronize()
        assert a["err"].item() == 0 and b["err"].item() == 0
        # gamma as fp32 bits; every integer output bit-exact
        assert a["g"].cpu().numpy().view(np.uint32)[0] == b["g"].cpu().numpy().view(np.uint32)[0]
        for k in ("codes", "meta", "dense"):
            assert torch.equal(a[k], b[k]), k


def test_noalloc_rejects_bad_arguments():
    L = sbn.lib()
    A = ctypes.c_void_p(0x10000)
    f = ctypes.c_float(1e-5)
    assert L.sbn_quantize_mask_pack_weights_noalloc(A, 8, 96, 2, 4, f, A, A, A, None, None,
                                                    None) == 2
    assert L.sbn_quantize_mask_pack_weights_noalloc(A, 2 ** 20, 4096, 2, 4, f, A, A, A, None,
                                                    None, None) == 2
    assert L.sbn_quantize_mask_pack_weights_noalloc(None, 8, 64, 2, 4, f, A, A, A, None, None,
                                                    None) == 1
    assert L.sbn_quantize_mask_pack_weights_noalloc(A, 8, 64, 2, 5, f, A, A, A, None, None,
                                                    None) == 3
