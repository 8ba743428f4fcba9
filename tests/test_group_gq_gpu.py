"""Group quantisation on the grouped calls (GqGroupPlan: every block of every layer a K slice
of one grouped quantiser and one grouped contraction, then sbn_gq_sum) vs the CPU oracle's
group_linear and vs the one-layer calls (sbn_quantize_acts_gq + sbn_linear_gq), through the
C ABI (needs a B200).

Bit-exact: Xq, the per-(token, group) scales (fp32 bits), and y against the one-layer calls
(the same arithmetic: y_j = fp32(acc_j * c_tj) per block, added in block order in fp32).
Against the oracle's fp64 y the bound of the one-layer tests applies:
|y - y_ref| <= (G + 3) 2^-24 sum_j |acc_j g_j s_tj / 127| (+ 2^-8 |y_ref| for bf16)."""
import numpy as np
import pytest
import torch

import oracle
import sparse_linear_layers_absmean_b200 as sbn
import workloads

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def make(specs, G, seed):
    """specs: (O, K, T).  Blocks with different weight scales, Student-t(4) activations."""
    layers, host = [], []
    for i, (O, K, T) in enumerate(specs):
        W_bits = workloads.masters(O, K, seed=seed, config=7, tensor=2 * i)
        Wf = workloads.bf16_bits_to_f32(W_bits)
        Wf[:, : K // G] *= 8.0
        W_bits = workloads.to_bf16_bits(Wf)
        X_bits = workloads.student_t(T, K, seed=seed, config=7, tensor=2 * i + 1)
        w = sbn.pack_weights_gq(workloads.torch_bf16(W_bits, "cuda"), 2, 4, G, 1e-5)
        layers.append(dict(X=workloads.torch_bf16(X_bits, "cuda"), w=w))
        host.append((W_bits, X_bits))
    return layers, host


def check(plan, layers, host, G, bf16=False):
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    plan.quantize_acts(err_flag=err)
    plan.linear(err_flag=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    for i, (L, (W_bits, X_bits)) in enumerate(zip(layers, host)):
        if X_bits.shape[0] == 0:  # a layer with no tokens is skipped
            continue
        ref = oracle.group_linear(X_bits, W_bits, 2, 4, G, 1e-5)
        assert np.array_equal(plan.Xq[i].cpu().numpy(), ref["Xq"])
        assert np.array_equal(plan.s[i].cpu().numpy().T.view(np.uint32), ref["s"].view(np.uint32))
        terms = (ref["acc"].astype(np.float64) * ref["g"].astype(np.float64)[:, None, None] *
                 ref["s"].T.astype(np.float64)[:, :, None] / 127.0)
        bound = (G + 3) * 2.0 ** -24 * np.abs(terms).sum(axis=0)
        if bf16:
            bound = bound + 2.0 ** -8 * np.abs(ref["y"])
        got = plan.Y[i].float().cpu().numpy().astype(np.float64)
        assert (np.abs(got - ref["y"]) <= bound + 1e-30).all()
        # the one-layer calls give the same bits
        Xq, s = sbn.quantize_acts_gq(L["X"], G)
        Y1 = sbn.linear_gq(Xq, s, L["w"], plan.Y[i].dtype)
        torch.cuda.synchronize()
        assert torch.equal(Xq, plan.Xq[i]) and torch.equal(s, plan.s[i])
        assert torch.equal(Y1, plan.Y[i])


@pytest.mark.parametrize("G", [1, 2, 4])
def test_gq_grouped_mixed(G):
    specs = [(300, 1024, 16), (130, 512, 5), (37, 2048, 1), (513, 1024, 32), (128, 512, 0)]
    layers, host = make(specs, G, seed=G)
    plan = sbn.GqGroupPlan(layers)
    check(plan, layers, host, G)


def test_gq_grouped_bf16_and_one_k_block_per_group():
    # K / G = 128: every block is a single 128-deep K block of its slice
    layers, host = make([(200, 512, 7), (96, 1024, 12)], 4, seed=5)
    plan = sbn.GqGroupPlan(layers, out_dtype=torch.bfloat16)
    check(plan, layers, host, 4, bf16=True)


def test_gq_grouped_twice():
    """The plan, called again with new activations in the same X buffers."""
    layers, host = make([(256, 1024, 16), (384, 512, 8)], 2, seed=9)
    plan = sbn.GqGroupPlan(layers)
    check(plan, layers, host, 2)
    host2 = []
    for i, (L, (W_bits, _)) in enumerate(zip(layers, host)):
        X2 = workloads.student_t(*L["X"].shape, seed=10, config=7, tensor=i)
        L["X"].copy_(workloads.torch_bf16(X2, "cuda"))
        host2.append((W_bits, X2))
    check(plan, layers, host2, 2)


@pytest.mark.parametrize("G,n", [(1, 100), (2, 1 << 16), (5, 4096 + 3), (64, 257)])
def test_gq_sum(G, n):
    """sbn_gq_sum: y[i] = part[0, i] + part[1, i] + ... in that order, in fp32."""
    rng = np.random.default_rng(G + n)
    part = (rng.standard_normal((G, n)) * 10.0 ** rng.integers(-3, 4, (G, n))).astype(np.float32)
    ref = part[0].copy()
    for j in range(1, G):
        ref = (ref + part[j]).astype(np.float32)
    pt = torch.from_numpy(part).cuda()
    for dt in (torch.float32, torch.bfloat16):
        Y = torch.empty(n, dtype=dt, device="cuda")
        sbn.sbn_gq_sum(pt, n, G, Y)
        torch.cuda.synchronize()
        want = torch.from_numpy(ref).to(dt)
        assert torch.equal(Y.cpu(), want)
