"""A tensor-core pipeline wait that runs out, on the GPU, without a fault or a hang.

The library's pipeline waits are bounded: after the limit a wait gives up, the kernel
raises SBN_FLAG_TIMEOUT, every role stops, the copies and MMAs already issued are waited
for, TMEM is freed and the call returns.  This test builds a test variant of the library
(define SBN_TIMEOUT_TEST: waits give up after about half a millisecond, and in the 2:4
small-batch kernel k_gemm_sp24 the first expander warp withholds its arrival for the second
pipeline stage, an arrival that therefore never comes), runs one contraction through it,
and checks that (1) the call returns and the flag is raised, (2) the CUDA context is still
usable: the regular library then computes a result equal to the oracle's on the same
device."""
import ctypes
import os
import subprocess

import numpy as np
import pytest
import torch

import gpu_path
import oracle
import sparse_linear_layers_absmean_b200 as sbn
import workloads
from sparse_linear_layers_absmean_b200 import build as sbn_build

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


@pytest.fixture(scope="module")
def timeout_lib(tmp_path_factory):
    out = str(tmp_path_factory.mktemp("timeout") / "libsbn_timeout.so")
    srcs = [os.path.join(sbn_build.CSRC, s) for s in sbn_build.SOURCES]
    subprocess.check_call([sbn_build._nvcc(), *sbn_build.NVCC_FLAGS, "-DSBN_TIMEOUT_TEST", "-I",
                           sbn_build.INCLUDE, "-I", sbn_build.CSRC, "-shared", "-o", out, *srcs])
    L = ctypes.CDLL(out)
    p, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    L.sbn_linear.argtypes = [p, p, p, p, p, i64, i64, i64, i32, i32, p, i32, p, p, p]
    L.sbn_linear.restype = i32
    return L


def test_wait_runs_out_and_device_stays_usable(timeout_lib):
    # 148 row tiles x 32 K blocks at 16 tokens: one CTA per tile, no K split, 8 pipeline
    # stages per CTA, so every CTA reaches the withheld stage
    O, K, T = 148 * 128, 4096, 16
    W = (torch.randn((O, K), device="cuda") * 0.02).bfloat16()
    X = torch.randn((T, K), device="cuda").bfloat16()
    w = sbn.pack_weights(W, 2, 4)
    Xq, s = sbn.quantize_acts(X)
    Y = torch.empty((T, O), dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = timeout_lib.sbn_linear(ctypes.c_void_p(Xq.data_ptr()), ctypes.c_void_p(s.data_ptr()),
                                ctypes.c_void_p(w.codes.data_ptr()),
                                ctypes.c_void_p(w.meta.data_ptr()),
                                ctypes.c_void_p(w.gamma_eff.data_ptr()), T, O, K, 2, 4,
                                ctypes.c_void_p(Y.data_ptr()), 0, None,
                                ctypes.c_void_p(err.data_ptr()),
                                ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0
    torch.cuda.synchronize()  # the call completed: no hang, no fault
    assert err.item() & sbn.FLAG_TIMEOUT

    # the same device, the regular library: parity with the oracle
    W_bits = workloads.masters(256, 640, seed=41)
    X_bits = workloads.activations(16, 640, seed=42)
    r = gpu_path.linear(X_bits, W_bits, 2, 4)
    ref = oracle.linear(X_bits, W_bits, 2, 4)
    assert r["err"] == 0
    assert np.array_equal(r["acc"], ref["acc"])
    gpu_path.assert_y_close(r["y"], ref["y"])
