"""Activation codes at exact quotient ties, on every quantiser path, vs the CPU oracle
(needs a B200).

q = clamp(rint((127 x) / s), -127, 127) rounds the quotient to nearest even at a tie.  The
kernels take q from a product with the token's reciprocal and use the IEEE divide only
where that product lies near a half-integer, so rows whose quotients are exact
half-integers are what exercises the divide.  Rows are built three ways (s is the row's
largest magnitude, put at one position):
  s = 127:     x = k + 1/2             -> 127 x / s = k + 1/2
  s = 254:     x odd integer           -> 127 x / s = x / 2
  s = 127/64:  x = (2k + 1) / 128      -> 127 x / s = k + 1/2
all exact in bf16, mixed with ordinary Student-t values.  Paths: one CTA per token, one
warp per token, two reads per token (K > 16384), the grouped quantiser, group
quantisation (G = 2, each block with its own s) and the quantiser in the fused decode
GEMV."""
import numpy as np
import pytest
import torch

import gpu_path
import oracle
import sparse_linear_layers_absmean_b200 as sbn
import workloads

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def tie_rows(T, K, seed, blocks=1):
    """bf16 bits [T, K]; each of `blocks` equal K slices of a row carries its own s."""
    rng = np.random.default_rng(seed)
    X = workloads.bf16_bits_to_f32(workloads.student_t(T, K, seed=seed, config=7, tensor=99))
    kb = K // blocks
    for t in range(T):
        kind = t % 3
        for j in range(blocks):
            sl = X[t, j * kb:(j + 1) * kb]
            if kind == 0:
                s, ties = 127.0, np.arange(-127, 127) + 0.5
            elif kind == 1:
                s, ties = 254.0, np.arange(-253, 254, 2).astype(np.float64)
            else:
                s, ties = 127.0 / 64.0, (2 * np.arange(-127, 127) + 1) / 128.0
            # ordinary values well inside the row's range, then ties at random positions
            sl[:] = sl / max(np.abs(sl).max(), 1e-3) * (s * 0.9)
            n = min(len(ties), kb // 2)
            pos = rng.choice(kb, size=n + 1, replace=False)
            sl[pos[:n]] = rng.choice(ties, size=n, replace=False)
            sl[pos[n]] = s if t % 2 == 0 else -s
    return workloads.to_bf16_bits(X)


@pytest.mark.parametrize("T,K", [(3, 512), (2, 11008), (40, 1024), (300, 4096), (2, 20480)])
def test_per_token_quantiser_ties(T, K):
    X = tie_rows(T, K, seed=T + K)
    got = gpu_path.quant(X)
    Xq, s, err = oracle.quant_acts(X)
    assert got["err"] == err == 0
    assert np.array_equal(got["s"].view(np.uint32), s.view(np.uint32))
    assert np.array_equal(got["Xq"], Xq)


def test_grouped_quantiser_ties():
    specs = [(128, 4096, 16), (96, 11008, 16), (64, 1024, 5)]
    layers, host = [], []
    dummy = torch.zeros(1 << 16, dtype=torch.uint8, device="cuda")
    gam = torch.ones(1, dtype=torch.float32, device="cuda")
    for i, (O, K, T) in enumerate(specs):
        X = tie_rows(T, K, seed=100 + i)
        w = sbn.PackedWeights(codes=dummy, meta=dummy, gamma_eff=gam, out=O, in_=K, n=2, m=4)
        layers.append(dict(X=workloads.torch_bf16(X, "cuda"),
                           Xq=torch.empty((T, K), dtype=torch.int8, device="cuda"),
                           s=torch.empty((T,), dtype=torch.float32, device="cuda"), w=w,
                           Y=torch.empty((T, O), dtype=torch.float32, device="cuda")))
        host.append(X)
    plan = sbn.GroupPlan(layers)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    plan.quantize_acts(err_flag=err)  # the quantiser only: the planes above are placeholders
    torch.cuda.synchronize()
    assert err.item() == 0
    for L, X in zip(layers, host):
        Xq, s, _ = oracle.quant_acts(X)
        assert np.array_equal(L["Xq"].cpu().numpy(), Xq)
        assert np.array_equal(L["s"].cpu().numpy().view(np.uint32), s.view(np.uint32))


def test_group_quantisation_ties():
    O, K, T, G = 128, 2048, 7, 2
    X = tie_rows(T, K, seed=7, blocks=G)
    W = workloads.masters(O, K, seed=8, config=7, tensor=0)
    ref = oracle.group_linear(X, W, 2, 4, G, 1e-5)
    Xq, s = sbn.quantize_acts_gq(workloads.torch_bf16(X, "cuda"), G)
    torch.cuda.synchronize()
    assert np.array_equal(Xq.cpu().numpy(), ref["Xq"])
    assert np.array_equal(s.cpu().numpy().T.view(np.uint32), ref["s"].view(np.uint32))


@pytest.mark.parametrize("T", [1, 4])
def test_fused_decode_quantiser_ties(T):
    O, K = 256, 2560
    X = tie_rows(T, K, seed=T)
    W = workloads.masters(O, K, seed=9, config=7, tensor=1)
    w = sbn.pack_weights(workloads.torch_bf16(W, "cuda"), 6, 8)
    Y, Xq, s = sbn.quantize_linear(workloads.torch_bf16(X, "cuda"), w)
    torch.cuda.synchronize()
    ref_q, ref_s, _ = oracle.quant_acts(X)
    assert np.array_equal(Xq.cpu().numpy(), ref_q)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), ref_s.view(np.uint32))
