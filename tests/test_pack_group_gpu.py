"""Grouped pack (sbn_pack_group_plan + sbn_quantize_mask_pack_weights_group) vs the CPU
oracle, through the C ABI (needs a B200).

Bit-exact: g (fp32 bits), the codes and meta planes of both patterns, the masked ternary
matrices.  Shapes cover tensors smaller than one 256 KB chunk, tensors whose last chunk and
last warp-iteration are partial, one-row and K = 64 tensors, one pattern or two in either
order, a second call after the masters changed in place (the workspace's counters must be
back at zero), the error flags, and the 130 tensors of the 26-layer training step in one plan (the
benchmark's launch) on sampled tensors and rows."""
import numpy as np
import pytest
import torch

import oracle
import sparse_linear_layers_absmean_b200 as sbn
import workloads

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

MIXED = [(1, 64), (37, 192), (300, 640), (130, 4160), (2100, 1024), (513, 2560), (64, 8640)]


def bits(W):
    return W.view(torch.int16).cpu().numpy().view(np.uint16)


def check(pg, Ws, rows=None, dense=None, which=None):
    """Tensors `which` (default: all) of the group against the oracle, on `rows` of each
    when given; Ws holds the masters of those tensors."""
    which = list(range(len(Ws))) if which is None else which
    for i, W in zip(which, Ws):
        W_bits = bits(W)
        _, _, g, err = oracle.weight_gamma(W_bits, 1e-5)
        assert err == 0
        r = np.arange(W.shape[0]) if rows is None else rows[which.index(i)]
        ri = torch.as_tensor(r, device=W.device)
        for j, (n, m) in enumerate(pg.patterns):
            pw = pg.packed[i][j]
            assert pw.gamma_eff.cpu().numpy().view(np.uint32)[0] == np.float32(g).view(np.uint32)
            t, keep, ws = oracle.ternary_mask(W_bits[r], n, m, g)
            codes, meta = oracle.pack(t, keep, n, m)
            assert np.array_equal(pw.codes[ri].cpu().numpy(), codes), (i, n, m)
            assert np.array_equal(pw.meta[ri].cpu().numpy(), meta), (i, n, m)
            if dense is not None:
                assert np.array_equal(dense[i][j][ri].cpu().numpy(), ws)


def counters_clear(pg):
    """The sum and chunk-count words of every workspace slot are back at zero (the third
    word, the code threshold, is rewritten by every call)."""
    slots = pg.workspace[:16 * len(pg.packed)].view(torch.int32).view(-1, 4)
    return not slots[:, :3].any()


def masters(specs, seed):
    return [workloads.torch_bf16(workloads.masters(O, K, seed=seed, config=4, tensor=i), "cuda")
            for i, (O, K) in enumerate(specs)]


@pytest.mark.parametrize("patterns", [((6, 8), (2, 4)), ((2, 4), (6, 8)), ((2, 4),), ((6, 8),)])
def test_pack_group_mixed(patterns):
    Ws = masters(MIXED, seed=1)
    dense = [[torch.empty(W.shape, dtype=torch.int8, device="cuda") for _ in patterns] for W in Ws]
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pg = sbn.PackGroup(Ws, patterns, dense_dbg=dense)
    pg.run(err_flag=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    check(pg, Ws, dense=dense)


@pytest.mark.parametrize("patterns", [((6, 8), (2, 4)), ((2, 4), (6, 8)), ((2, 4),), ((6, 8),)])
def test_pack_group_matches_single_tensor_calls(patterns):
    """Without dense matrices every plan here runs the fixed-pattern kernel."""
    Ws = masters(MIXED, seed=2)
    pg = sbn.PackGroup(Ws, patterns)
    assert pg.mode == (2 if len(patterns) == 2 else (1 if patterns[0] == (2, 4) else 0))
    pg.run()
    for i, W in enumerate(Ws):
        for j, (n, m) in enumerate(pg.patterns):
            w = sbn.pack_weights(W, n, m)
            torch.cuda.synchronize()
            pw = pg.packed[i][j]
            assert torch.equal(w.codes, pw.codes) and torch.equal(w.meta, pw.meta)
            assert torch.equal(w.gamma_eff, pw.gamma_eff)


def test_pack_group_second_call_after_update():
    """The masters change in place (one optimizer step's noise); the same plan and workspace
    pack the new values."""
    specs = MIXED[2:]
    Ws = masters(specs, seed=3)
    pg = sbn.PackGroup(Ws)
    pg.run()
    torch.cuda.synchronize()
    check(pg, Ws)
    for i, W in enumerate(Ws):
        W.copy_(workloads.torch_bf16(workloads.perturb(bits(W), seed=3, config=4, tensor=i),
                                     "cuda"))
    pg.run()
    torch.cuda.synchronize()
    assert counters_clear(pg)
    check(pg, Ws)


def test_pack_group_error_flags():
    Ws = masters([(64, 256), (64, 256), (64, 256)], seed=4)
    Ws[1][3, 5] = float("nan")
    Ws[2][7, 9] = 300.0
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pg = sbn.PackGroup(Ws)
    pg.run(err_flag=err)
    torch.cuda.synchronize()
    assert err.item() == 1 | 2
    check(pg, Ws[:1])  # the clean tensor is packed as usual
    err.zero_()
    Ws[1][3, 5] = 0.0
    Ws[2][7, 9] = 0.0
    pg.run(err_flag=err)
    torch.cuda.synchronize()
    assert err.item() == 0 and counters_clear(pg)
    check(pg, Ws)


TRAIN_SAMPLE = [0, 1, 2, 3, 4, 62, 129]


def test_pack_group_training_step_sampled():
    """The 130 linears of the 26-layer decoder (hidden 3200, FFN 8640), 6:8 and 2:4, in one
    plan, with the benchmark's seeded masters: every tensor equal to the single-tensor call,
    sampled tensors and rows (tile edges, the last row, random rows) against the oracle."""
    Ws = []
    for layer in range(workloads.TRAIN_LAYERS):
        for i, (_, O, K) in enumerate(workloads.TRAIN_LAYER_SHAPES):
            Ws.append(workloads.masters_device(O, K, device="cuda", config=4, tensor=5 * layer + i))
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pg = sbn.PackGroup(Ws)
    pg.run(err_flag=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    for i in range(0, len(Ws), 13):
        for j, (n, m) in enumerate(pg.patterns):
            w = sbn.pack_weights(Ws[i], n, m)
            torch.cuda.synchronize()
            assert torch.equal(w.codes, pg.packed[i][j].codes)
            assert torch.equal(w.meta, pg.packed[i][j].meta)
    rng = np.random.default_rng(7)
    rows = []
    for i in TRAIN_SAMPLE:
        O = Ws[i].shape[0]
        rows.append(np.unique(np.concatenate([[0, 127, 128, O - 1],
                                              rng.choice(O, size=12, replace=False)])))
    check(pg, [Ws[i] for i in TRAIN_SAMPLE], rows=rows, which=TRAIN_SAMPLE)
