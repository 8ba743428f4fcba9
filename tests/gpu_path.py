"""Runs the CUDA path through the C ABI on seeded inputs and returns numpy results."""
import numpy as np
import torch

import sparse_linear_layers_absmean_b200 as sbn
import workloads


def pack(W_bits, n, m, eps=1e-5, workspace=None):
    W = workloads.torch_bf16(W_bits, "cuda")
    O, K = W.shape
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    dense = torch.empty((O, K), dtype=torch.int8, device="cuda")
    w = sbn.pack_weights(W, n, m, eps, workspace=workspace, dense_dbg=dense, err_flag=err)
    torch.cuda.synchronize()
    return dict(w=w, codes=w.codes.cpu().numpy(), meta=w.meta.cpu().numpy(),
                g=np.float32(w.gamma_eff.item()), ws=dense.cpu().numpy(), err=int(err.item()))


def quant(X_bits):
    X = workloads.torch_bf16(X_bits, "cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    Xq, s = sbn.quantize_acts(X, err_flag=err)
    torch.cuda.synchronize()
    return dict(Xq_t=Xq, s_t=s, Xq=Xq.cpu().numpy(), s=s.cpu().numpy(), err=int(err.item()))


def linear(X_bits, W_bits, n, m, eps=1e-5, out_dtype=torch.float32):
    p = pack(W_bits, n, m, eps)
    q = quant(X_bits)
    T = X_bits.shape[0]
    acc = torch.empty((T, p["w"].out), dtype=torch.int32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    Y = sbn.linear(q["Xq_t"], q["s_t"], p["w"], out_dtype, acc_dbg=acc, err_flag=err)
    torch.cuda.synchronize()
    y = Y.float().cpu().numpy()
    return dict(pack=p, quant=q, acc=acc.cpu().numpy(), y=y, err=int(err.item()))


def assert_y_close(y, y_ref, bf16=False):
    """fp32 outputs: |y - y_ref| <= 1e-5 |y_ref|; bf16: <= 8e-3 |y_ref| (and y == 0 where the
    exact result is 0)."""
    tol = 8e-3 if bf16 else 1e-5
    y_ref = np.asarray(y_ref, np.float64)
    err = np.abs(y.astype(np.float64) - y_ref)
    bad = err > tol * np.abs(y_ref)
    assert not bad.any(), (int(bad.sum()), np.argwhere(bad)[:5], y[bad][:5], y_ref[bad][:5])
