"""The pre-expanded tensor-core operand (sbn_expand_operand) and the contraction that reads
it (sbn_linear_operand) vs the CPU oracle, through the C ABI (needs a B200).

The operand is checked byte for byte against one built from the oracle's masked codes and
metadata plane: the kept values of each row in K order, zero rows/blocks in the padding,
the metadata copied with the index pair (0, 1) in the padding.  The contraction: int32 sums
bit-exact, fp32 y within 1e-5 relative of the oracle's fp64 y (bf16: 8e-3), and every output
bit equal to sbn_linear's on the same inputs."""
import numpy as np
import pytest
import torch

import gpu_path
import oracle
import sparse_linear_layers_absmean_b200 as sbn
import workloads

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def expected_operand(ref, O, K):
    O_pad, K_pad = -(-O // 256) * 256, -(-K // 128) * 128
    A = np.zeros((O_pad, K_pad // 2), np.int8)
    for r in range(O):
        kept = ref["ws"][r][ref["keep"][r] != 0]
        assert kept.size == K // 2
        A[r, :K // 2] = kept
    M = np.full((O_pad, K_pad // 8), 0x44, np.uint8)
    M[:O, :K // 8] = ref["meta"][:, :K // 8]
    return np.concatenate([A.view(np.uint8).ravel(), M.ravel()])


def run(O, K, T, seed, out_dtype=torch.float32):
    W_bits = workloads.masters(O, K, seed=seed, config=3, tensor=0)
    X_bits = workloads.activations(T, K, seed=seed, config=3, tensor=1)
    W = workloads.torch_bf16(W_bits, "cuda")
    X = workloads.torch_bf16(X_bits, "cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    w = sbn.pack_weights(W, 2, 4, 1e-5, err_flag=err)
    op = sbn.expand_operand(w)
    Xq, s = sbn.quantize_acts(X, err_flag=err)
    acc = torch.empty((T, O), dtype=torch.int32, device="cuda")
    Y = sbn.linear_operand(Xq, s, w, op, out_dtype, acc_dbg=acc, err_flag=err)
    acc2 = torch.empty_like(acc)
    Y2 = sbn.linear(Xq, s, w, out_dtype, acc_dbg=acc2, err_flag=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    return dict(W=W_bits, X=X_bits, op=op, acc=acc, Y=Y, acc2=acc2, Y2=Y2)


@pytest.mark.parametrize("O,K,T", [(300, 640, 300), (256, 4160, 37), (513, 1024, 1),
                                   (64, 128, 224), (1000, 256, 449)])
def test_operand_linear_small(O, K, T):
    r = run(O, K, T, seed=O + K + T)
    ref = oracle.linear(r["X"], r["W"], 2, 4, 1e-5)
    assert np.array_equal(r["op"].cpu().numpy(), expected_operand(ref, O, K))
    assert np.array_equal(r["acc"].cpu().numpy(), ref["acc"])
    gpu_path.assert_y_close(r["Y"].cpu().numpy(), ref["y"])
    assert torch.equal(r["acc"], r["acc2"]) and torch.equal(r["Y"], r["Y2"])


def test_operand_linear_bf16():
    r = run(384, 512, 260, seed=9, out_dtype=torch.bfloat16)
    ref = oracle.linear(r["X"], r["W"], 2, 4, 1e-5)
    assert np.array_equal(r["acc"].cpu().numpy(), ref["acc"])
    gpu_path.assert_y_close(r["Y"].float().cpu().numpy(), ref["y"], bf16=True)
    assert torch.equal(r["Y"], r["Y2"])


def test_operand_prefill_full_size():
    """The prefill configuration (W 11008 x 4096 2:4, 2048 tokens with outlier channels),
    int32 sums compared in full with the oracle."""
    cfg = workloads.PREFILL_GEMM
    r = run(cfg["O"], cfg["K"], cfg["T"], seed=0)
    ref = oracle.linear(r["X"], r["W"], 2, 4, 1e-5)
    assert np.array_equal(r["acc"].cpu().numpy(), ref["acc"])
    gpu_path.assert_y_close(r["Y"].cpu().numpy(), ref["y"])
    assert torch.equal(r["Y"], r["Y2"])


def test_operand_rejects_other_patterns():
    with pytest.raises(sbn.SbnError):
        sbn.sbn_operand_bytes(128, 256, 6, 8)
