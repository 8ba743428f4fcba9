"""CUDA path vs the CPU oracle, element by element, through the C ABI (needs a B200).

Bit-exact: gamma (as fp32 bits), codes and meta planes including the zero padding, the
masked ternary matrix, int8 activations, per-token scales, int32 accumulators.
Float: fp32 y within 1e-5 relative of the oracle's fp64 y; bf16 y within 8e-3."""
import numpy as np
import pytest
import torch

import gpu_path
import oracle
import workloads

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

PATTERNS = [(2, 4), (6, 8), (1, 4), (3, 4), (4, 4), (1, 8), (2, 8), (3, 8), (4, 8), (5, 8),
            (7, 8), (8, 8)]


def check_pack(W_bits, n, m, eps=1e-5):
    got = gpu_path.pack(W_bits, n, m, eps)
    ref = oracle.quantize_mask_pack(W_bits, n, m, eps)
    assert got["err"] == ref["err"] == 0
    assert got["g"].view(np.uint32) == np.float32(ref["g"]).view(np.uint32), (got["g"], ref["g"])
    assert np.array_equal(got["ws"], ref["ws"])
    assert np.array_equal(got["meta"], ref["meta"])
    assert np.array_equal(got["codes"], ref["codes"])
    return got, ref


@pytest.mark.parametrize("n,m", PATTERNS)
@pytest.mark.parametrize("O,K", [(1, 64), (37, 192), (130, 320), (9, 3200)])
def test_pack_small(n, m, O, K):
    check_pack(workloads.masters(O, K, seed=O * K + n * 8 + m), n, m)


def test_pack_ties_and_signed_zeros():
    rng = np.random.default_rng(0)
    vals = np.array([0.0, -0.0, 0.015625, -0.015625, 0.03125, -0.03125], np.float32)
    W = workloads.to_bf16_bits(rng.choice(vals, size=(64, 256)))
    for n, m in [(2, 4), (6, 8), (3, 8), (1, 4)]:
        check_pack(W, n, m)


def test_pack_exact_half_ties():
    # mean |W| = 0.5 exactly with eps = 0: 0.25 / 0.5 = 0.5 -> 0, 0.75 / 0.5 = 1.5 -> 1
    row = np.array([0.25, 0.75, 0.5, 0.5, -0.25, -0.75, -0.5, -0.5], np.float32)
    W = workloads.to_bf16_bits(np.tile(row, (16, 8)))
    got, ref = check_pack(W, 8, 8, eps=0.0)
    assert got["g"] == np.float32(0.5)


@pytest.mark.parametrize("n,m", [(2, 4), (6, 8), (3, 8)])
def test_pack_large_magnitudes(n, m):
    """Weights up to 255 (inside the supported range): 16 consecutive terms of
    trunc(|W| * 2^24) overflow 32 bits, so the exact sum must not depend on a narrow
    partial.  Rows of large values next to rows of ordinary ones, plus scattered 16.0 and
    15.9375 (the two sides of the narrow-partial bound)."""
    rng = np.random.default_rng(7)
    Wf = rng.normal(0.0, 0.02, size=(300, 512)).astype(np.float32)
    Wf[5] = rng.uniform(100.0, 255.0, size=512) * rng.choice([-1.0, 1.0], size=512)
    Wf[200, :64] = 255.0
    idx = rng.integers(0, Wf.size, size=40)
    Wf.flat[idx[:20]] = 16.0
    Wf.flat[idx[20:]] = -15.9375
    check_pack(workloads.to_bf16_bits(Wf), n, m)


def test_pack_all_zero_with_zero_eps():
    W = np.zeros((8, 128), np.uint16)
    got, ref = check_pack(W, 2, 4, eps=0.0)
    assert got["g"] == 0 and not got["ws"].any()


def test_pack_workspace_is_reusable():
    W1 = workloads.masters(64, 256, seed=1)
    W2 = workloads.masters(64, 256, seed=2)
    import sparse_linear_layers_absmean_b200 as sbn
    ws = sbn.new_workspace(64, 256, 2, 4)
    for W in (W1, W2, W1):
        got = gpu_path.pack(W, 2, 4, workspace=ws)
        ref = oracle.quantize_mask_pack(W, 2, 4)
        assert got["g"] == ref["g"] and np.array_equal(got["codes"], ref["codes"])
    # the reserved words after the 1024 partial sums are never written
    assert not ws[8192:8200].cpu().numpy().any()


def test_pack_workspace_many_sizes():
    """One workspace through calls of many sizes and both fast patterns (the reduction's
    grid size changes from call to call): every result exact, the reserved words after the
    partial sums untouched."""
    import sparse_linear_layers_absmean_b200 as sbn
    ws = sbn.new_workspace(8, 64, 2, 4)
    shapes = [(1, 64), (4096, 4096), (3, 192), (700, 2560), (1, 64), (6912, 2560), (130, 320)]
    for i, (O, K) in enumerate(shapes * 2):
        n, m = ((2, 4), (6, 8))[i % 2]
        W = workloads.masters(O, K, seed=100 + i)
        got = gpu_path.pack(W, n, m, workspace=ws)
        torch.cuda.synchronize()
        assert got["err"] == 0
        assert not ws[8192:8200].cpu().numpy().any()
        if O * K <= 1 << 22:
            ref = oracle.quantize_mask_pack(W, n, m)
            assert got["g"] == ref["g"] and np.array_equal(got["codes"], ref["codes"])
            assert np.array_equal(got["meta"], ref["meta"])


@pytest.mark.parametrize("bad,flag", [(np.nan, 1), (np.inf, 1), (-np.inf, 1), (300.0, 2),
                                      (-256.0, 2)])
def test_pack_flags_bad_weights(bad, flag):
    W = workloads.masters(16, 128, seed=3)
    W[5, 77] = workloads.to_bf16_bits(np.array([bad], np.float32))[0]
    got = gpu_path.pack(W, 2, 4)
    assert got["err"] == flag


@pytest.mark.parametrize("T,K", [(1, 64), (3, 256), (8, 2560), (37, 4096), (5, 11008),
                                 (2, 20480), (17, 64), (300, 1024), (101, 2048), (40, 4160),
                                 (1000, 3200)])
def test_act_quant(T, K):
    """Rows of more than 1024 inputs, and few tokens, take the one-CTA-per-token kernels
    (rows in registers, or read twice past 16384); many tokens with rows of up to 1024 the
    one-warp-per-token kernel (ragged last CTA)."""
    X = workloads.activations(T, K, seed=T * K)
    X[0, :7] = workloads.to_bf16_bits(np.array([0.5, -0.5, 1.5, 2.5, -2.5, 0, -0.0], np.float32))
    if T > 2:
        X[1] = 0
    got = gpu_path.quant(X)
    Xq, s, err = oracle.quant_acts(X)
    assert got["err"] == err == 0
    assert np.array_equal(got["s"].view(np.uint32), s.view(np.uint32))
    assert np.array_equal(got["Xq"], Xq)


@pytest.mark.parametrize("T", [4, 100])
def test_act_quant_flags_nonfinite(T):
    X = workloads.activations(T, 256, seed=5)
    X[2, 9] = workloads.to_bf16_bits(np.array([np.nan], np.float32))[0]
    assert gpu_path.quant(X)["err"] == 4
    X = workloads.activations(T, 256, seed=6)
    X[T - 1, 200] = workloads.to_bf16_bits(np.array([-np.inf], np.float32))[0]
    assert gpu_path.quant(X)["err"] == 4


def check_linear(T, O, K, n, m, seed, out_dtype=torch.float32, eps=1e-5):
    W = workloads.masters(O, K, seed=seed)
    X = workloads.activations(T, K, seed=seed + 1)
    got = gpu_path.linear(X, W, n, m, eps, out_dtype)
    ref = oracle.linear(X, W, n, m, eps)
    assert got["err"] == got["pack"]["err"] == got["quant"]["err"] == 0
    assert np.array_equal(got["quant"]["Xq"], ref["Xq"])
    assert np.array_equal(got["pack"]["codes"], ref["codes"])
    assert np.array_equal(got["acc"], ref["acc"]), np.argwhere(got["acc"] != ref["acc"])[:8]
    gpu_path.assert_y_close(got["y"], ref["y"], bf16=out_dtype == torch.bfloat16)


@pytest.mark.parametrize("n,m", [(2, 4), (6, 8), (4, 4), (1, 8)])
@pytest.mark.parametrize("T", [1, 2, 3, 4])
@pytest.mark.parametrize("O,K", [(37, 192), (300, 640), (129, 11008)])
def test_linear_cuda_cores(T, O, K, n, m):
    check_linear(T, O, K, n, m, seed=T + O + K + n)


@pytest.mark.parametrize("n,m", [(2, 4), (6, 8), (8, 8), (3, 4)])
@pytest.mark.parametrize("T", [5, 16, 17, 40, 100, 129, 300])
@pytest.mark.parametrize("O,K", [(300, 192), (130, 640)])
def test_linear_tensor_cores(T, O, K, n, m):
    check_linear(T, O, K, n, m, seed=T * 7 + O + K + n)


@pytest.mark.parametrize("T,O,K", [(1500, 6000, 320), (1000, 8000, 128), (500, 12000, 64),
                                   (1200, 5000, 1152), (700, 9000, 1664), (2048, 11008, 640)])
def test_linear_many_tiles_per_cta(T, O, K):
    """Enough 256-row output tiles that the persistent CTA-pair 2:4 kernel gives each pair
    several, so both TMEM accumulators and the stage rings wrap across tiles (ragged rows,
    tokens and K in each case); 2048 x 11008 takes 208-token tiles, the others 192.  Odd
    stage counts per tile (K = 128, 64, 1152, 1664, 640: 1, 1, 5, 7 and 3 stages of two K
    blocks) move the two MMA-issuing threads' share of stages from one tile to the next."""
    check_linear(T, O, K, 2, 4, seed=T + O + K)


@pytest.mark.parametrize("T,O,K", [(2048, 4096, 1152), (1500, 2000, 640), (4096, 4096, 512)])
def test_linear_pair_192_token_tiles(T, O, K):
    """Shapes where the CTA-pair kernel takes 192-token tiles (no more rounds of tiles over
    the pairs than 208 would take): ragged last token tile, odd stage counts (K = 1152, 640:
    5 and 3 stages of two K blocks), one or several tiles per pair."""
    check_linear(T, O, K, 2, 4, seed=T + O + K + 7)


@pytest.mark.parametrize("T,O,K", [(5, 4100, 4096), (16, 1000, 11008), (17, 300, 2048),
                                   (32, 130, 8192), (24, 4096, 576)])
def test_linear_few_tokens_long_k(T, O, K):
    """5-32 tokens on the 2:4 tensor-core kernel with long rows (up to 86 K blocks, so the
    stage ring wraps many times), ragged rows and a K that ends in half a block."""
    check_linear(T, O, K, 2, 4, seed=T * 3 + O + K)


@pytest.mark.parametrize("T,O,K,out", [(16, 4096, 4096, "f32"), (16, 12288, 4096, "f32"),
                                       (9, 260, 2048, "bf16"), (32, 1100, 11008, "f32"),
                                       (20, 4000, 4160, "bf16"), (7, 640, 704, "f32")])
def test_linear_split_k(T, O, K, out):
    """Up to 32 tokens with few row tiles and long rows: the 2:4 kernel splits each tile's
    K blocks over a cluster of 2-8 CTAs and CTA 0 adds the partial tiles (the decode
    shapes of a 4096-hidden layer, a K that ends in half a block, bf16 output)."""
    check_linear(T, O, K, 2, 4, seed=T + O + K,
                 out_dtype=torch.bfloat16 if out == "bf16" else torch.float32)


@pytest.mark.parametrize("T", [1, 3, 9, 300])
def test_linear_bf16_output(T):
    check_linear(T, 260, 256, 2, 4, seed=11, out_dtype=torch.bfloat16)
    check_linear(T, 260, 256, 6, 8, seed=12, out_dtype=torch.bfloat16)


def test_linear_zero_tokens_is_noop():
    import sparse_linear_layers_absmean_b200 as sbn
    w = sbn.pack_weights(workloads.torch_bf16(workloads.masters(8, 64), "cuda"), 2, 4)
    Xq = torch.empty((0, 64), dtype=torch.int8, device="cuda")
    s = torch.empty((0,), dtype=torch.float32, device="cuda")
    Y = sbn.linear(Xq, s, w)
    assert Y.shape == (0, 8)


def test_linear_zero_token_row_gives_zero():
    W = workloads.masters(140, 256, seed=4)
    X = workloads.activations(20, 256, seed=5)
    X[3] = 0
    got = gpu_path.linear(X, W, 2, 4)
    assert (got["y"][3] == 0).all() and (got["acc"][3] == 0).all()


@pytest.mark.parametrize("T,n,m", [(1, 6, 8), (8, 2, 4), (300, 2, 4), (40, 6, 8)])
def test_forward_public_api(T, n, m):
    """sbn.forward (activation quantiser on a side stream, pack on the caller's stream)
    against the oracle, on a non-default caller stream."""
    import sparse_linear_layers_absmean_b200 as sbn
    O, K = 300, 512
    W_bits = workloads.masters(O, K, seed=T + n)
    X_bits = workloads.activations(T, K, seed=T + m)
    ref = oracle.linear(X_bits, W_bits, n, m, 1e-5)
    st = torch.cuda.Stream()
    with torch.cuda.stream(st):
        W = workloads.torch_bf16(W_bits, "cuda")
        X = workloads.torch_bf16(X_bits, "cuda")
        Y = sbn.forward(X, W, n, m)
        del W, X  # freed while the side stream may still read X: record_stream keeps it
        y = Y.cpu().numpy()
    gpu_path.assert_y_close(y, ref["y"])


@pytest.mark.parametrize("n,m", [(2, 4), (6, 8), (1, 4), (3, 8), (8, 8)])
@pytest.mark.parametrize("O,K", [(1, 64), (37, 192), (300, 2560), (1000, 4096)])
def test_mask_stats(O, K, n, m):
    """Natural zeros and mask flips between two training steps (the masters plus small
    noise, and a copy with tie-heavy rows) against the oracle's counts."""
    import sparse_linear_layers_absmean_b200 as sbn
    W1 = workloads.masters(O, K, seed=O + K + n)
    rng = np.random.default_rng(O * K + m)
    W2f = workloads.bf16_bits_to_f32(W1) + rng.normal(0.0, 1e-3, size=(O, K)).astype(np.float32)
    W2 = workloads.to_bf16_bits(W2f.astype(np.float32))
    W2[::3] = workloads.to_bf16_bits(np.round(workloads.bf16_bits_to_f32(W1[::3]) * 64) / 64)
    r1 = oracle.quantize_mask_pack(W1, n, m)
    r2 = oracle.quantize_mask_pack(W2, n, m)
    Wd1, Wd2 = workloads.torch_bf16(W1, "cuda"), workloads.torch_bf16(W2, "cuda")
    p1, p2 = sbn.pack_weights(Wd1, n, m), sbn.pack_weights(Wd2, n, m)
    z1 = int(sbn.count_zero_codes(Wd1, p1).item())
    z2 = int(sbn.count_zero_codes(Wd2, p2).item())
    flips = int(sbn.count_mask_flips(p1, p2).item())
    assert z1 == oracle.count_zero_codes(r1["t"])
    assert z2 == oracle.count_zero_codes(r2["t"])
    assert flips == oracle.count_mask_flips(r1["keep"], r2["keep"])
    assert int(sbn.count_mask_flips(p1, p1).item()) == 0
    # the counts accumulate into a caller-zeroed counter
    c = torch.zeros(1, dtype=torch.int64, device="cuda")
    sbn.sbn_count_zero_codes(Wd1, p1.gamma_eff, c)
    sbn.sbn_count_zero_codes(Wd2, p2.gamma_eff, c)
    assert int(c.item()) == z1 + z2


def test_mask_stats_all_zero_tensor():
    """g = 0 (all-zero masters, eps = 0): every code is 0."""
    import sparse_linear_layers_absmean_b200 as sbn
    W = torch.zeros((16, 128), dtype=torch.bfloat16, device="cuda")
    w = sbn.pack_weights(W, 2, 4, eps=0.0)
    assert int(sbn.count_zero_codes(W, w).item()) == 16 * 128
