"""Parity at the workloads' full sizes, in the launch configuration the benchmark uses.

Integer stages (codes, metadata, masked matrix, int8 activations, per-token scales, int32
sums) must match the CPU oracle bit for bit; fp32 outputs within 1e-5 relative.  Where a
full oracle product would take minutes, a seeded sample of tokens is compared."""
import numpy as np
import pytest
import torch

import gpu_path
import oracle
import workloads

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def _check_pack(W, n, m):
    got = gpu_path.pack(W, n, m)
    ref = oracle.quantize_mask_pack(W, n, m)
    assert got["err"] == 0
    assert got["g"].view(np.uint32) == np.float32(ref["g"]).view(np.uint32)
    assert np.array_equal(got["codes"], ref["codes"])
    assert np.array_equal(got["meta"], ref["meta"])
    assert np.array_equal(got["ws"], ref["ws"])
    return got, ref


def _linear_sampled(X, W, n, m, sample_tokens):
    got = gpu_path.linear(X, W, n, m)
    assert got["err"] == got["pack"]["err"] == got["quant"]["err"] == 0
    Xq, s, _ = oracle.quant_acts(X)
    assert np.array_equal(got["quant"]["Xq"], Xq)
    assert np.array_equal(got["quant"]["s"].view(np.uint32), s.view(np.uint32))
    ref = oracle.quantize_mask_pack(W, n, m)
    assert np.array_equal(got["pack"]["codes"], ref["codes"])
    assert np.array_equal(got["pack"]["meta"], ref["meta"])
    rows = np.arange(X.shape[0]) if sample_tokens is None else sample_tokens
    acc = oracle.contract(Xq[rows], ref["ws"])
    assert np.array_equal(got["acc"][rows], acc)
    y = oracle.rescale(acc, s[rows], ref["g"])
    gpu_path.assert_y_close(got["y"][rows], y)


def test_config1_tiny_full():
    c = workloads.TINY
    W = workloads.masters(c["O"], c["K"], seed=0, config=0)
    X = workloads.activations(c["T"], c["K"], seed=0, config=0, outliers=False)
    _linear_sampled(X, W, c["n"], c["m"], None)


def test_config2_decode_gemv_full():
    c = workloads.DECODE_GEMV
    W = workloads.masters(c["O"], c["K"], seed=0, config=1)
    X = workloads.activations(c["T"], c["K"], seed=0, config=1)
    _linear_sampled(X, W, c["n"], c["m"], None)


def test_config3_prefill_gemm_full():
    c = workloads.PREFILL_GEMM
    W = workloads.masters(c["O"], c["K"], seed=0, config=2)
    X = workloads.activations(c["T"], c["K"], seed=0, config=2)
    _linear_sampled(X, W, c["n"], c["m"], None)


@pytest.mark.parametrize("n,m", [(6, 8), (2, 4)])
def test_config4_training_step_one_layer(n, m):
    # one decoder layer (5 linears), step 0 and one perturbed step
    for t, (name, O, K) in enumerate(workloads.TRAIN_LAYER_SHAPES):
        W = workloads.masters(O, K, seed=0, config=3, tensor=t)
        _check_pack(W, n, m)
        if name in ("qkv", "down"):
            W1 = workloads.perturb(W, seed=0, config=3, tensor=t, step=0)
            _check_pack(W1, n, m)


def test_config5_stack_layer0_decode_and_prefill():
    shapes = dict((nm, (O, K)) for nm, O, K in workloads.STACK_LAYER_SHAPES)
    O, K = shapes["qkv"]
    W = workloads.masters(O, K, seed=0, config=4, tensor=0)
    X = workloads.student_t(workloads.STACK_DECODE_T, K, seed=0, config=4, tensor=100)
    _linear_sampled(X, W, 2, 4, None)
    O, K = shapes["down"]
    W = workloads.masters(O, K, seed=0, config=4, tensor=4)
    X = workloads.student_t(workloads.STACK_PREFILL_T, K, seed=0, config=4, tensor=104)
    rng = np.random.default_rng(5)
    sample = np.sort(rng.choice(workloads.STACK_PREFILL_T, size=256, replace=False))
    _linear_sampled(X, W, 2, 4, sample)
