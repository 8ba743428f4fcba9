"""Dual-STE backward (sbn_backward) vs the CPU oracle's fp64 backward (needs a B200).

Tolerances come from the arithmetic of the kernels (products exact in both GEMMs):
  dX = g * sum_o dY * Ws: fp32 accumulation of `out` exact products, then one multiply by g
       -> |dX - ref| <= (out + 2) 2^-24 * g * sum_o |dY * Ws|;
  dW = pass * sum_t dY * (s/127) * Xq: c_t = fp32(s_t / 127) and dY' = fp32(dY * c_t) round once
       each (2^-24), dY' is carried as hi + lo bf16 (residual <= 2^-18 |dY'|), and 2 T_pad
       exact products are accumulated in fp32
       -> |dW - ref| <= (2^-17 + (2 T_pad + 4) 2^-24) * sum_t |dY| |X_eff|;
  the clip gate is a decision: dW is exactly 0 wherever the oracle's gate is closed."""
import numpy as np
import pytest
import torch

import oracle
import sparse_linear_layers_absmean_b200 as sbn
import workloads

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def run(O, K, T, n, m, seed, token_rows=None, out_rows=None):
    W_bits = workloads.masters(O, K, seed=seed, config=6, tensor=0)
    X_bits = workloads.activations(T, K, seed=seed, config=6, tensor=1)
    rng = np.random.default_rng(seed)
    dY_bits = workloads.to_bf16_bits(rng.standard_normal((T, O)).astype(np.float32))
    W = workloads.torch_bf16(W_bits, "cuda")
    X = workloads.torch_bf16(X_bits, "cuda")
    dY = workloads.torch_bf16(dY_bits, "cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    w = sbn.pack_weights(W, n, m, 1e-5, err_flag=err)
    Xq, s = sbn.quantize_acts(X, err_flag=err)
    dX, dW = sbn.backward(dY, Xq, s, w, W, err_flag=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    ref = oracle.quantize_mask_pack(W_bits, n, m, 1e-5)
    Xq_h, s_h, _ = oracle.quant_acts(X_bits)
    dY_f = workloads.bf16_bits_to_f32(dY_bits)
    return dict(W=W_bits, dY=dY_f, Xq=Xq_h, s=s_h, ref=ref, dX=dX.cpu().numpy(),
                dW=dW.cpu().numpy())


def check_dx(r, rows):
    ref, g = r["ref"], float(r["ref"]["g"])
    O = ref["ws"].shape[0]
    dX_ref, _ = oracle.backward(r["dY"][rows], r["Xq"][rows], r["s"][rows], ref["ws"], r["W"],
                                ref["g"])
    bound = (O + 2) * 2.0 ** -24 * g * (np.abs(r["dY"][rows]).astype(np.float64) @
                                         np.abs(ref["ws"]).astype(np.float64))
    err = np.abs(r["dX"][rows].astype(np.float64) - dX_ref)
    assert (err <= bound + 1e-30).all(), float((err - bound).max())


def check_dw(r, rows):
    ref = r["ref"]
    T = r["dY"].shape[0]
    Tp = -(-T // 32) * 32
    _, dW_ref = oracle.backward(r["dY"][:, rows], r["Xq"], r["s"], ref["ws"][rows], r["W"][rows],
                                ref["g"])
    X_eff = r["Xq"].astype(np.float64) * (r["s"].astype(np.float64) / 127.0)[:, None]
    bound = (2.0 ** -17 + (2 * Tp + 4) * 2.0 ** -24) * (np.abs(r["dY"][:, rows]).T.astype(np.float64)
                                                        @ np.abs(X_eff))
    got = r["dW"][rows].astype(np.float64)
    closed = dW_ref == 0.0
    assert (got[closed & (bound > 0)] == 0.0).all()
    err = np.abs(got - dW_ref)
    assert (err <= bound + 1e-30).all(), float((err - bound).max())
    # the gate really closes somewhere and the mask does not: pruned weights get gradients
    assert closed.any() and (got[ref["keep"][rows] == 0] != 0).any()


@pytest.mark.parametrize("O,K,T,n,m", [(256, 512, 64, 2, 4), (200, 320, 37, 2, 4),
                                       (1024, 2048, 300, 6, 8), (136, 192, 5, 3, 8)])
def test_backward_small(O, K, T, n, m):
    r = run(O, K, T, n, m, seed=O + K + T)
    check_dx(r, slice(None))
    check_dw(r, slice(None))


def test_backward_prefill_shape_sampled():
    """The prefill configuration's shape (W 11008 x 4096 2:4, 2048 tokens): dX checked on 16
    sampled tokens, dW on 24 sampled rows, each against the oracle computed one by one."""
    cfg = workloads.PREFILL_GEMM
    r = run(cfg["O"], cfg["K"], cfg["T"], 2, 4, seed=0)
    rng = np.random.default_rng(3)
    check_dx(r, np.sort(rng.choice(cfg["T"], 16, replace=False)))
    check_dw(r, np.sort(rng.choice(cfg["O"], 24, replace=False)))
