"""sbn_quantize_linear (steps 5-7 in one call; one launch for <= 4 tokens) vs the CPU oracle
and vs the separate calls, through the C ABI (needs a B200).  Bit-exact Xq, s and int32
sums; fp32 y within 1e-5 relative (bf16: 8e-3); every output bit equal to
sbn_quantize_acts + sbn_linear."""
import numpy as np
import pytest
import torch

import gpu_path
import oracle
import sparse_linear_layers_absmean_b200 as sbn
import workloads

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def run(O, K, T, n, m, seed, out_dtype=torch.float32):
    W_bits = workloads.masters(O, K, seed=seed, config=2, tensor=0)
    X_bits = workloads.activations(T, K, seed=seed, config=2, tensor=1)
    W = workloads.torch_bf16(W_bits, "cuda")
    X = workloads.torch_bf16(X_bits, "cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    w = sbn.pack_weights(W, n, m, 1e-5, err_flag=err)
    acc = torch.empty((T, O), dtype=torch.int32, device="cuda")
    Y, Xq, s = sbn.quantize_linear(X, w, out_dtype, acc_dbg=acc, err_flag=err)
    Xq2, s2 = sbn.quantize_acts(X, err_flag=err)
    acc2 = torch.empty_like(acc)
    Y2 = sbn.linear(Xq2, s2, w, out_dtype, acc_dbg=acc2, err_flag=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    assert torch.equal(Xq, Xq2) and torch.equal(s, s2) and torch.equal(acc, acc2)
    assert torch.equal(Y, Y2)
    ref = oracle.linear(X_bits, W_bits, n, m, 1e-5)
    assert np.array_equal(Xq.cpu().numpy(), ref["Xq"])
    assert np.array_equal(s.cpu().numpy().view(np.uint32), np.asarray(ref["s"], np.float32).view(np.uint32))
    assert np.array_equal(acc.cpu().numpy(), ref["acc"])
    gpu_path.assert_y_close(Y.float().cpu().numpy(), ref["y"], bf16=out_dtype == torch.bfloat16)


@pytest.mark.parametrize("T", [1, 2, 3, 4])
@pytest.mark.parametrize("n,m", [(2, 4), (6, 8), (3, 8), (8, 8)])
@pytest.mark.parametrize("O,K", [(37, 192), (300, 2560), (9, 16384)])
def test_fused_small(T, n, m, O, K):
    run(O, K, T, n, m, seed=T * 7 + n + O)


def test_fused_bf16_out():
    run(129, 1024, 3, 6, 8, seed=5, out_dtype=torch.bfloat16)


@pytest.mark.parametrize("O,K,T", [(64, 16448, 2), (96, 512, 5)])
def test_unfused_paths(O, K, T):
    """Beyond the one-launch limits (in > 16384, or more than 4 tokens) the call is the two
    separate launches: same results."""
    run(O, K, T, 2, 4, seed=O + T)


def test_fused_decode_full_size():
    """The decode configuration: W 6912 x 2560 6:8, one token with outlier channels."""
    cfg = workloads.DECODE_GEMV
    run(cfg["O"], cfg["K"], cfg["T"], cfg["n"], cfg["m"], seed=0)
