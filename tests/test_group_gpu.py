"""Grouped calls (sbn_quantize_acts_group + sbn_linear_group) vs the CPU oracle, element by
element, through the C ABI (needs a B200).

Bit-exact: int8 activations, per-token scales (fp32 bits), int32 accumulators of every
layer.  Float: fp32 y within 1e-5 relative of the oracle's fp64 y; bf16 within 8e-3.
Shapes cover ragged row tiles (O % 128 != 0), K % 128 == 64, 1..32 tokens, layers with 0
tokens, a schedule that splits row tiles over several work units (called twice: the
split's arrival counters must be back at zero), the 4096-hidden stack layer at 16 tokens
compared in full, and the whole 160-linear stack in one plan on sampled linears and rows."""
import numpy as np
import pytest
import torch

import gpu_path
import oracle
import sparse_linear_layers_absmean_b200 as sbn
import workloads

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def make_layers(specs, seed, out_dtype=torch.float32):
    """specs: list of (O, K, T).  Masters N(0, 0.02^2), activations Student-t(4)."""
    layers, host = [], []
    for i, (O, K, T) in enumerate(specs):
        W_bits = workloads.masters(O, K, seed=seed, config=5, tensor=2 * i)
        X_bits = workloads.student_t(T, K, seed=seed, config=5, tensor=2 * i + 1)
        W = workloads.torch_bf16(W_bits, "cuda")
        w = sbn.pack_weights(W, 2, 4, 1e-5)
        layers.append(dict(X=workloads.torch_bf16(X_bits, "cuda"),
                           Xq=torch.empty((T, K), dtype=torch.int8, device="cuda"),
                           s=torch.empty((T,), dtype=torch.float32, device="cuda"), w=w,
                           Y=torch.empty((T, O), dtype=out_dtype, device="cuda"),
                           acc_dbg=torch.empty((T, O), dtype=torch.int32, device="cuda")))
        host.append((W_bits, X_bits))
    return layers, host


def run(plan):
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    plan.quantize_acts(err_flag=err)
    plan.linear(err_flag=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    return err


def check(layers, host, bf16=False):
    for L, (W_bits, X_bits) in zip(layers, host):
        T = X_bits.shape[0]
        if T == 0:
            continue
        ref = oracle.linear(X_bits, W_bits, 2, 4, 1e-5)
        assert np.array_equal(L["Xq"].cpu().numpy(), ref["Xq"])
        assert np.array_equal(L["s"].cpu().numpy().view(np.uint32),
                              np.asarray(ref["s"], np.float32).view(np.uint32))
        assert np.array_equal(L["acc_dbg"].cpu().numpy(), ref["acc"])
        gpu_path.assert_y_close(L["Y"].float().cpu().numpy(), ref["y"], bf16=bf16)


MIXED = [(300, 640, 16), (130, 192, 5), (256, 4160, 32), (37, 64, 1), (128, 128, 0),
         (513, 1024, 31), (1000, 320, 7)]


def test_group_mixed_shapes():
    layers, host = make_layers(MIXED, seed=1)
    plan = sbn.GroupPlan(layers)
    assert plan.bn == 32
    run(plan)
    check(layers, host)


def test_group_few_tokens_bf16():
    specs = [(640, 512, 16), (129, 256, 3), (64, 2112, 1)]
    layers, host = make_layers(specs, seed=2, out_dtype=torch.bfloat16)
    plan = sbn.GroupPlan(layers)
    assert plan.bn == 16
    run(plan)
    check(layers, host, bf16=True)


def test_group_split_twice():
    """One layer with two row tiles: the schedule splits K over several units per tile
    (partials through the workspace); a second call with new activations must see the
    arrival counters back at zero."""
    layers, host = make_layers([(256, 4096, 16)], seed=3)
    plan = sbn.GroupPlan(layers)
    assert plan.split > 1 and plan.workspace_bytes > 0
    run(plan)
    check(layers, host)
    assert not plan.workspace[:8].any()  # counters reset
    X2 = workloads.student_t(16, 4096, seed=33, config=5, tensor=1)
    layers[0]["X"].copy_(workloads.torch_bf16(X2, "cuda"))
    run(plan)
    check(layers, [(host[0][0], X2)])


def test_group_matches_single_layer_calls():
    """The same layers through sbn_linear one by one: identical int32 sums and outputs."""
    specs = [(384, 1024, 16), (200, 2048, 12), (128, 4096, 16)]
    layers, _ = make_layers(specs, seed=4)
    plan = sbn.GroupPlan(layers)
    run(plan)
    for L in layers:
        acc = torch.empty_like(L["acc_dbg"])
        Y = sbn.linear(L["Xq"], L["s"], L["w"], torch.float32, acc_dbg=acc)
        torch.cuda.synchronize()
        assert torch.equal(acc, L["acc_dbg"])
        assert torch.equal(Y, L["Y"])


def test_group_rejects_bad_layers():
    layers, _ = make_layers([(128, 256, 16)], seed=5)
    L = layers[0]
    bad = dict(L)
    bad["Xq"] = torch.empty((33, 256), dtype=torch.int8, device="cuda")  # 33 tokens
    with pytest.raises(sbn.SbnError):
        sbn.GroupPlan([bad])
    w68 = sbn.pack_weights(L["X"].new_zeros((128, 256)), 6, 8)
    with pytest.raises(sbn.SbnError):
        sbn.GroupPlan([dict(L, w=w68)])


def test_group_stack_layer_full_size():
    """Layer 0 of the 4096-hidden stack (QKV 12288x4096, O 4096x4096, gate/up 11008x4096,
    down 4096x11008) at 16 tokens, the decode configuration, compared in full."""
    specs = [(O, K, workloads.STACK_DECODE_T) for _, O, K in workloads.STACK_LAYER_SHAPES]
    layers, host = make_layers(specs, seed=0)
    plan = sbn.GroupPlan(layers)
    run(plan)
    check(layers, host)


# sampled linears of the full stack: first, middle and last layers, every projection kind,
# the last linear of the plan included (the end of the unit schedule)
STACK_SAMPLE = [0, 1, 2, 3, 4, 77, 83, 155, 159]


def test_group_full_stack_sampled():
    """All 160 linears of the 32-layer stack (hidden 4096, FFN 11008) at 16 tokens, 2:4, in
    one plan: the launch the benchmark times, with its seeded weights and activations.  The
    oracle checks every output of sampled linears on sampled rows (row tiles' first and last
    rows, the ragged end, random rows): codes and meta of those rows, Xq and s of the
    linear, int32 sums and y.  Every other output must be finite."""
    T = workloads.STACK_DECODE_T
    rng = np.random.default_rng(5)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    layers, sampled = [], {}
    for layer in range(workloads.STACK_LAYERS):
        for i, (_, O, K) in enumerate(workloads.STACK_LAYER_SHAPES):
            idx = 5 * layer + i
            W = workloads.masters_device(O, K, device="cuda", config=5, tensor=idx)
            w = sbn.pack_weights(W, 2, 4, 1e-5, err_flag=err)
            X_bits = workloads.student_t(T, K, config=5, tensor=10000 + idx)
            L = dict(X=workloads.torch_bf16(X_bits, "cuda"),
                     Xq=torch.empty((T, K), dtype=torch.int8, device="cuda"),
                     s=torch.empty((T,), dtype=torch.float32, device="cuda"), w=w,
                     Y=torch.empty((T, O), dtype=torch.float32, device="cuda"))
            if idx in STACK_SAMPLE:
                L["acc_dbg"] = torch.empty((T, O), dtype=torch.int32, device="cuda")
                W_bits = W.view(torch.int16).cpu().numpy().view(np.uint16)
                rows = np.unique(np.concatenate([[0, 127, 128, O - 1],
                                                 rng.choice(O, size=12, replace=False)]))
                sampled[idx] = (W_bits, X_bits, rows)
            layers.append(L)
            del W
    plan = sbn.GroupPlan(layers)
    run(plan)
    torch.cuda.synchronize()
    assert err.item() == 0
    for idx, (W_bits, X_bits, rows) in sampled.items():
        L = layers[idx]
        ri = torch.as_tensor(rows, device="cuda")
        _, _, g, werr = oracle.weight_gamma(W_bits, 1e-5)
        assert werr == 0
        assert L["w"].gamma_eff.cpu().numpy().view(np.uint32)[0] == np.float32(g).view(np.uint32)
        t, keep, ws = oracle.ternary_mask(W_bits[rows], 2, 4, g)
        codes, meta = oracle.pack(t, keep, 2, 4)
        assert np.array_equal(L["w"].codes[ri].cpu().numpy(), codes)
        assert np.array_equal(L["w"].meta[ri].cpu().numpy(), meta)
        Xq, s, xerr = oracle.quant_acts(X_bits)
        assert xerr == 0
        assert np.array_equal(L["Xq"].cpu().numpy(), Xq)
        assert np.array_equal(L["s"].cpu().numpy().view(np.uint32), s.view(np.uint32))
        acc = oracle.contract(Xq, ws)
        assert np.array_equal(L["acc_dbg"][:, ri].cpu().numpy(), acc)
        gpu_path.assert_y_close(L["Y"][:, ri].cpu().numpy(), oracle.rescale(acc, s, g))
    for L in layers:
        assert torch.isfinite(L["Y"]).all()


def test_group_odd_super_blocks_repeated():
    """Units with odd and even numbers of super-blocks (K = 384, 1152, 640, 5504: 1, 3, 2
    and 11 super-blocks of four 128-deep K blocks) follow one another on every CTA, and the
    plan runs 40 times back to back: which MMA thread consumes a ring slot must not depend
    on the units' lengths (no timeout flag; every call gives the single-layer results)."""
    Ks = [384, 1152, 640, 5504]
    T = 16
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    layers = []
    for i in range(64):
        O, K = 2048, Ks[i % 4]
        W = workloads.masters_device(O, K, device="cuda", config=5, tensor=i)
        w = sbn.pack_weights(W, 2, 4, 1e-5, err_flag=err)
        X = workloads.torch_bf16(workloads.student_t(T, K, config=5, tensor=1000 + i), "cuda")
        layers.append(dict(X=X, Xq=torch.empty((T, K), dtype=torch.int8, device="cuda"),
                           s=torch.empty((T,), dtype=torch.float32, device="cuda"), w=w,
                           Y=torch.empty((T, O), dtype=torch.float32, device="cuda")))
    plan = sbn.GroupPlan(layers)
    plan.quantize_acts(err_flag=err)
    torch.cuda.synchronize()
    refs = [sbn.linear(L["Xq"], L["s"], L["w"]) for L in layers]
    for _ in range(40):
        plan.linear(err_flag=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    for L, Y in zip(layers, refs):
        assert torch.equal(L["Y"], Y)
