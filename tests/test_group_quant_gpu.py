"""Group quantisation (sbn_quantize_mask_pack_weights_gq, sbn_quantize_acts_gq,
sbn_linear_gq) vs the CPU oracle's group_linear, through the C ABI (needs a B200).

Bit-exact: the G scales (fp32 bits), codes and meta planes, the masked ternary matrix, Xq,
the per-(token, group) scales, every block's int32 sums.  y = sum_j fp32(acc_j * c_tj) added
in fp32: each term rounds twice (c_tj, the product) and the G - 1 additions once each, so
|y - y_ref| <= (G + 3) 2^-24 * sum_j |acc_j g_j s_tj / 127| (a bound on the absolute sum,
since the blocks' terms may cancel); bf16 output adds its own rounding, 2^-8 |y_ref|."""
import numpy as np
import pytest
import torch

import oracle
import sparse_linear_layers_absmean_b200 as sbn
import workloads

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def run(O, K, T, n, m, G, seed, out_dtype=torch.float32):
    W_bits = workloads.masters(O, K, seed=seed, config=7, tensor=0)
    X_bits = workloads.activations(T, K, seed=seed, config=7, tensor=1)
    # blocks with very different scales, so that a wrong block's scale shows
    Wf = workloads.bf16_bits_to_f32(W_bits)
    Wf[:, : K // G] *= 8.0
    W_bits = workloads.to_bf16_bits(Wf)
    W = workloads.torch_bf16(W_bits, "cuda")
    X = workloads.torch_bf16(X_bits, "cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    dense = torch.empty((O, K), dtype=torch.int8, device="cuda")
    w = sbn.pack_weights_gq(W, n, m, G, 1e-5, dense_dbg=dense, err_flag=err)
    Xq, s = sbn.quantize_acts_gq(X, G, err_flag=err)
    acc = torch.empty((G, T, O), dtype=torch.int32, device="cuda")
    Y = sbn.linear_gq(Xq, s, w, out_dtype, acc_dbg=acc, err_flag=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    ref = oracle.group_linear(X_bits, W_bits, n, m, G, 1e-5)
    assert np.array_equal(w.gamma_eff.cpu().numpy().view(np.uint32), ref["g"].view(np.uint32))
    assert np.array_equal(w.codes.cpu().numpy(), ref["codes"])
    assert np.array_equal(w.meta.cpu().numpy(), ref["meta"])
    assert np.array_equal(dense.cpu().numpy(), ref["ws"])
    assert np.array_equal(Xq.cpu().numpy(), ref["Xq"])
    assert np.array_equal(s.cpu().numpy().T.view(np.uint32), ref["s"].view(np.uint32))
    assert np.array_equal(acc.cpu().numpy(), ref["acc"])
    terms = (ref["acc"].astype(np.float64) * ref["g"].astype(np.float64)[:, None, None] *
             ref["s"].T.astype(np.float64)[:, :, None] / 127.0)
    bound = (G + 3) * 2.0 ** -24 * np.abs(terms).sum(axis=0)
    if out_dtype == torch.bfloat16:
        bound = bound + 2.0 ** -8 * np.abs(ref["y"])
    got = Y.float().cpu().numpy().astype(np.float64)
    assert (np.abs(got - ref["y"]) <= bound + 1e-30).all()
    return w, Y


@pytest.mark.parametrize("O,K,T,n,m,G", [(37, 256, 3, 2, 4, 2), (130, 512, 1, 6, 8, 4),
                                         (300, 1024, 16, 2, 4, 8), (64, 2048, 300, 2, 4, 2),
                                         (256, 768, 40, 6, 8, 3), (96, 4096, 5, 3, 8, 32)])
def test_group_quant(O, K, T, n, m, G):
    run(O, K, T, n, m, G, seed=O + K + G)


def test_group_quant_bf16():
    run(200, 1024, 2, 2, 4, 4, seed=3, out_dtype=torch.bfloat16)


def test_one_group_is_the_per_tensor_layer():
    O, K, T = 160, 512, 6
    W_bits = workloads.masters(O, K, seed=9)
    X_bits = workloads.activations(T, K, seed=10)
    W = workloads.torch_bf16(W_bits, "cuda")
    X = workloads.torch_bf16(X_bits, "cuda")
    wg = sbn.pack_weights_gq(W, 2, 4, 1)
    w = sbn.pack_weights(W, 2, 4)
    Xq_g, s_g = sbn.quantize_acts_gq(X, 1)
    Xq, s = sbn.quantize_acts(X)
    Yg = sbn.linear_gq(Xq_g, s_g, wg)
    Y = sbn.linear(Xq, s, w)
    torch.cuda.synchronize()
    assert torch.equal(wg.codes, w.codes) and torch.equal(wg.meta, w.meta)
    assert torch.equal(wg.gamma_eff, w.gamma_eff) and torch.equal(Xq_g, Xq)
    assert torch.equal(s_g[0], s) and torch.equal(Yg, Y)


def test_group_quant_rejects_bad_groups():
    W = torch.zeros((8, 384), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(sbn.SbnError):
        sbn.pack_weights_gq(W, 2, 4, 2)  # 384 / 2 = 192 is not a multiple of 128
    with pytest.raises(sbn.SbnError):
        sbn.pack_weights_gq(W, 2, 4, 5)
