"""Checks that pin the CPU oracle to something other than itself.

Each check raises AssertionError on a mismatch.  They are run against the real oracle
(tests/test_oracle_pins.py) and against deliberately broken copies of it
(tests/test_oracle_mutants.py), which must each fail at least one check.

What pins what:
  hand_example        every stage, against values worked out by hand (golden file)
  mask_bruteforce     the top-N rule, against exhaustive search over all N-subsets
  gamma_closed_form   S1, against the exact rational mean |W| (fractions.Fraction)
  rounding_ties       round-half-to-even and the clip, on constructed exact ties
  dense_pattern       n == m reduces to the plain (unmasked) b1.58 BitLinear
  constant_magnitude  codes == sign(W) when all |W| are equal
  act_absmax          the absmax element of every token maps to +-127; 0-token -> 0
  contract_bruteforce S6, against an int64 sum written as a Python loop / numpy
  unpack_roundtrip    the packed planes decode (independent decoder) to the masked codes
  invariants          code range, no 0b10 pattern, N bits per group, zero padding
  scale_invariance    W -> 2W leaves the mask and codes unchanged and doubles gamma
  rescale_closed_form S7, against acc * g * s / 127 recomputed with Fraction
  mask_stats          natural-zero and mask-flip counts: hand-worked values (golden file),
                      a closed form, and the invariances of the mask (sign, power-of-two
                      scale, dense pattern)
  group_one           group quantisation with G = 1 is the per-tensor layer (every output)
  group_slices        G blocks: every block is the per-tensor layer on its K-slice (scales,
                      codes, mask, activations, sums) and y is the sum of the blocks' outputs
  group_hand          G = 2 on a hand-worked row (golden file)
  backward_hand       dual-STE backward on the hand-worked example (golden file): pruned
                      positions still receive their weight gradient, clipped ones none
  backward_adjoint    <dY, y> = <dX, X_eff> against the forward's y; <dW, V> = <dY,
                      X_eff (V * pass)^T> for a random V (the weight gradient is the adjoint
                      of the gated product); dW independent of the mask; the clip gate on
                      weights placed exactly at |W| = g and next to it
"""
import itertools
import math
import os
from fractions import Fraction

import numpy as np

import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    d = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, *v = line.split()
            d[k] = v
    return d


def _f32(bits):
    return workloads.bf16_bits_to_f32(bits)


def hand_example(o):
    g = _read_golden("hand_example_2of4.txt")
    n, m = int(g["n"][0]), int(g["m"][0])
    W = workloads.to_bf16_bits(np.array([[float(v) for v in g["W"]]], np.float32))
    X = workloads.to_bf16_bits(np.array([[float(v) for v in g["x"]]], np.float32))
    assert np.array_equal(_f32(W)[0], np.array([float(v) for v in g["W"]], np.float32))
    r = o.linear(X, W, n, m, eps=float(g["eps"][0]))
    assert r["err"] == 0 and r["xerr"] == 0
    assert r["S"] == int(g["S"][0]), r["S"]
    assert r["gamma"] == np.float32(float(g["gamma"][0])), r["gamma"]
    assert r["t"][0].tolist() == [int(v) for v in g["t"]], r["t"]
    assert r["keep"][0].tolist() == [int(v) for v in g["keep"]], r["keep"]
    assert r["ws"][0].tolist() == [int(v) for v in g["ws"]], r["ws"]
    assert r["codes"][0].tolist() == [int(v, 0) for v in g["codes"]], r["codes"]
    assert r["meta"][0].tolist() == [int(v, 0) for v in g["meta"]], r["meta"]
    assert r["s"][0] == np.float32(float(g["s"][0])), r["s"]
    assert r["Xq"][0].tolist() == [int(v) for v in g["q"]], r["Xq"]
    assert int(r["acc"][0, 0]) == int(g["acc"][0]), r["acc"]
    y_exact = float(g["y_num"][0]) / float(g["y_den"][0])
    assert abs(r["y"][0, 0] - y_exact) <= 1e-12 * abs(y_exact), r["y"]
    # eps = 1e-5 moves g but no code: y follows acc * fp32(gamma + eps) * s / 127.
    r2 = o.linear(X, W, n, m, eps=1e-5)
    assert r2["ws"][0].tolist() == [int(v) for v in g["ws"]]
    g2 = float(np.float32(np.float32(0.23046875) + np.float32(1e-5)))
    y2 = float(Fraction(-119) * Fraction(g2) * 8 / 127)
    assert abs(r2["y"][0, 0] - y2) <= 1e-12 * abs(y2), (r2["y"], y2)


def _tie_heavy_masters(rows, K, seed):
    rng = np.random.default_rng(seed)
    vals = np.array([0.0, -0.0, 0.25, -0.25, 0.5, -0.5, 0.0625, 1.0, -1.0], np.float32)
    a = rng.choice(vals, size=(rows, K))
    # sprinkle distinct magnitudes so groups mix ties and non-ties
    a += np.where(rng.random((rows, K)) < 0.3, rng.standard_normal((rows, K)) * 0.02, 0)
    return workloads.to_bf16_bits(a.astype(np.float32))


def mask_bruteforce(o):
    for (n, m) in [(1, 4), (2, 4), (3, 4), (4, 4), (1, 8), (2, 8), (4, 8), (6, 8), (7, 8)]:
        W = _tie_heavy_masters(6, 4 * m, seed=17 * n + m)
        _, keep, _ = o.ternary_mask(W, n, m, np.float32(0.1))
        mags = np.abs(_f32(W))
        for r in range(W.shape[0]):
            for base in range(0, W.shape[1], m):
                grp = mags[r, base:base + m]
                best = None
                for sub in itertools.combinations(range(m), n):
                    key = (sorted((float(grp[i]) for i in sub), reverse=True), [-i for i in sub])
                    if best is None or key > best[0]:
                        best = (key, sub)
                want = np.zeros(m, np.uint8)
                want[list(best[1])] = 1
                got = keep[r, base:base + m]
                assert np.array_equal(got, want), (n, m, r, base, grp, got, want)


def gamma_closed_form(o):
    for seed, (O, K) in enumerate([(7, 64), (64, 256), (33, 448)]):
        W = workloads.masters(O, K, seed=100 + seed)
        a = np.abs(_f32(W)).astype(np.float64)
        exact = sum((Fraction(float(v)) for v in a.ravel() if v >= 2.0 ** -17), Fraction(0))
        tiny = [float(v) for v in a.ravel() if 0 < v < 2.0 ** -17]
        # values below 2^-17 are truncated at 2^-24 by the stated definition
        exact += sum((Fraction(math.floor(v * 2 ** 24), 2 ** 24) for v in tiny), Fraction(0))
        mean = exact / W.size
        S, gamma, g, err = o.weight_gamma(W, 0.0)
        assert err == 0
        assert Fraction(S, 2 ** 24) == exact, (S, exact)
        # gamma is fp32(fp64(S) / (n 2^24)): within one fp32 ulp of the exact mean
        ulp = np.spacing(np.float32(float(mean)))
        assert abs(Fraction(float(gamma)) - mean) <= Fraction(float(ulp)), (gamma, float(mean))
        assert g == gamma
        S2, gamma2, g2, _ = o.weight_gamma(W, 1e-5)
        assert g2 == np.float32(gamma2 + np.float32(1e-5))
    # a mean that is exactly representable comes out exactly
    W = workloads.to_bf16_bits(np.array([[0.25, -0.75, 0.5, -0.5] * 16], np.float32))
    S, gamma, g, err = o.weight_gamma(W, 0.0)
    assert gamma == np.float32(0.5) and S == 32 * 2 ** 24
    # the stated truncation: magnitudes below 2^-24 contribute nothing
    W = workloads.to_bf16_bits(np.full((1, 64), 2.0 ** -30, np.float32))
    assert o.weight_gamma(W, 0.0)[0] == 0


def rounding_ties(o):
    # mean |W| = 0.5 exactly; 0.25/0.5 = 0.5 -> 0 (even), 0.75/0.5 = 1.5 -> 2 -> clip 1
    row = np.array([0.25, 0.75, 0.5, 0.5, -0.25, -0.75, -0.5, -0.5], np.float32)
    W = workloads.to_bf16_bits(np.tile(row, (2, 8)))
    S, gamma, g, _ = o.weight_gamma(W, 0.0)
    assert g == np.float32(0.5)
    t, keep, ws = o.ternary_mask(W, 8, 8, g)
    assert t[0, :8].tolist() == [0, 1, 1, 1, 0, -1, -1, -1], t[0, :8]
    # activations: absmax 127 -> q = x exactly; absmax 2 -> 127 x / 2 at exact .5 ties
    x = np.array([[1.0, 0.5, -0.5, 1.5, -1.5, 2.0, 0.0, -2.0]], np.float32)
    Xq, s, _ = o.quant_acts(workloads.to_bf16_bits(x))
    # 127*[1,.5,-.5,1.5,-1.5,2,0,-2]/2 = 63.5 31.75 -31.75 95.25 -95.25 127 0 -127
    assert Xq[0].tolist() == [64, 32, -32, 95, -95, 127, 0, -127], Xq
    x = np.array([[0.5, 127.0, 62.5, -62.5, 61.5, -0.5, 1.5, 2.5]], np.float32)
    Xq, s, _ = o.quant_acts(workloads.to_bf16_bits(x))
    assert s[0] == 127 and Xq[0].tolist() == [0, 127, 62, -62, 62, 0, 2, 2], Xq


def act_quotient_ties(o):
    # every exact tie of 127 x / s in three row scales; ties go to the even integer
    # (np.rint rounds half to even).  s = 127: the quotient is x; s = 254: x / 2 for odd x;
    # s = 127/64: 64 x for x = (2k + 1) / 128
    half = np.arange(-127, 127) + 0.5
    odd = np.arange(-253, 254, 2).astype(np.float64)
    for s, x, quot in [(127.0, half, half), (254.0, odd, odd / 2),
                       (127.0 / 64, (2 * np.arange(-127, 127) + 1) / 128.0, half)]:
        row = np.concatenate([[s], x, [-s / 2]]).astype(np.float32)[None, :]
        Xq, sc, err = o.quant_acts(workloads.to_bf16_bits(row))
        assert err == 0 and sc[0] == np.float32(s)
        want = np.rint(quot).astype(np.int64)
        assert np.array_equal(Xq[0, 1:1 + len(x)].astype(np.int64), want), (s, Xq[0, :8])
        assert Xq[0, 0] == 127


def dense_pattern(o):
    W = workloads.masters(5, 128, seed=5)
    for m in (4, 8):
        r = o.quantize_mask_pack(W, m, m, eps=1e-5)
        assert r["keep"].all()
        assert np.array_equal(r["ws"], r["t"])
        ldm = r["meta"].shape[1]
        assert (r["meta"][:, :128 // 8] == 0xFF).all() and (r["meta"][:, 128 // 8:ldm] == 0).all()
        # plain b1.58: codes = clip(round(W / g)) with no mask
        w = _f32(W)
        want = np.clip(np.rint(w / r["g"]), -1, 1).astype(np.int8)
        assert np.array_equal(r["t"], want)


def constant_magnitude(o):
    rng = np.random.default_rng(3)
    sign = np.where(rng.random((4, 64)) < 0.5, -1.0, 1.0).astype(np.float32)
    W = workloads.to_bf16_bits(sign * np.float32(0.0234375))
    for n, m in [(2, 4), (6, 8)]:
        r = o.quantize_mask_pack(W, n, m, eps=1e-5)
        assert np.array_equal(r["t"], sign.astype(np.int8))
        # all magnitudes tie: the first n positions of every group are kept
        assert (r["keep"].reshape(4, -1, m)[:, :, :n] == 1).all()
        assert (r["keep"].reshape(4, -1, m)[:, :, n:] == 0).all()


def act_absmax(o):
    X = workloads.activations(9, 256, seed=4)
    X[3] = 0  # an all-zero token
    Xq, s, err = o.quant_acts(X)
    x = _f32(X)
    assert err == 0
    for t in range(9):
        if t == 3:
            assert s[t] == np.float32(1e-5) and (Xq[t] == 0).all()
            continue
        j = int(np.argmax(np.abs(x[t])))
        assert s[t] == np.abs(x[t]).max()
        assert Xq[t, j] == (127 if x[t, j] > 0 else -127)
        assert np.abs(Xq[t]).max() == 127


def contract_bruteforce(o):
    rng = np.random.default_rng(9)
    Xq = rng.integers(-127, 128, size=(5, 96), dtype=np.int64).astype(np.int8)
    Ws = rng.integers(-1, 2, size=(7, 96), dtype=np.int64).astype(np.int8)
    acc = o.contract(Xq, Ws)
    for t in range(5):
        for j in range(7):
            want = 0
            for k in range(96):
                want += int(Xq[t, k]) * int(Ws[j, k])
            assert int(acc[t, j]) == want, (t, j)
    # a larger case against numpy's int64 matmul (operand order: tokens x outputs)
    Xq = rng.integers(-127, 128, size=(33, 640), dtype=np.int64).astype(np.int8)
    Ws = rng.integers(-1, 2, size=(65, 640), dtype=np.int64).astype(np.int8)
    assert np.array_equal(o.contract(Xq, Ws), Xq.astype(np.int64) @ Ws.astype(np.int64).T)


def unpack_planes(codes, meta, K, n, m):
    """Independent decoder of the packed format, written from its description: returns
    (ws, keep) with ws the masked ternary matrix and keep the mask."""
    O = codes.shape[0]
    compact = (n, m) == (2, 4)
    ws = np.zeros((O, K), np.int8)
    keep = np.zeros((O, K), np.uint8)

    def code_at(r, e):
        word = int.from_bytes(bytes(codes[r, 4 * (e // 16):4 * (e // 16) + 4]), "little")
        c = (word >> (8 * (e % 4) + 6 - 2 * ((e % 16) // 4))) & 3
        assert c != 2, "code 0b10 is never written"
        return {0: 0, 1: 1, 3: -1}[c]

    for r in range(O):
        for gi in range(K // m):
            if m == 8:
                field = int(meta[r, gi])
            else:
                field = (int(meta[r, gi // 2]) >> (4 * (gi % 2))) & 0xF
            if compact:
                i0, i1 = field & 3, field >> 2
                assert i0 < i1, "2:4 indices are stored in ascending order"
                kept = [i0, i1]
            else:
                kept = [i for i in range(m) if field >> i & 1]
            for i in kept:
                keep[r, gi * m + i] = 1
        e = 0
        for k in range(K):
            if compact:
                if keep[r, k]:
                    ws[r, k] = code_at(r, e)
                    e += 1
            else:
                v = code_at(r, k)
                assert keep[r, k] or v == 0, "pruned positions hold the code of 0"
                ws[r, k] = v
    return ws, keep


def unpack_roundtrip(o):
    for n, m, K in [(2, 4, 256), (6, 8, 192), (1, 8, 64), (3, 4, 64)]:
        W = workloads.masters(9, K, seed=K + n)
        r = o.quantize_mask_pack(W, n, m)
        ws, keep = unpack_planes(r["codes"], r["meta"], K, n, m)
        assert np.array_equal(ws, r["ws"]) and np.array_equal(keep, r["keep"])


def invariants(o):
    for n, m in [(2, 4), (6, 8), (3, 4), (4, 8)]:
        K = 320
        W = workloads.masters(64, K, seed=n * m)
        r = o.quantize_mask_pack(W, n, m)
        assert set(np.unique(r["t"]).tolist()) <= {-1, 0, 1}
        keep = r["keep"].reshape(64, -1, m)
        assert (keep.sum(-1) == n).all()
        assert ((r["ws"] != 0).reshape(64, -1, m).sum(-1) <= n).all()
        assert np.array_equal(r["ws"], r["t"] * r["keep"])
        stored = K // 2 if (n, m) == (2, 4) else K
        used_c = stored * 2 // 8
        used_m = K // 8
        assert (r["codes"][:, used_c:] == 0).all() and (r["meta"][:, used_m:] == 0).all()
        c = r["codes"][:, :used_c]
        for sh in (0, 2, 4, 6):
            assert ((c >> sh) & 3 != 2).all()
        mm = r["meta"][:, :used_m]
        if m == 4:
            nib = np.concatenate([mm & 0xF, mm >> 4])
            if n == 2:
                assert ((nib & 3) < (nib >> 2)).all()
            else:
                assert (np.unpackbits(nib[..., None], axis=-1).sum(-1) == n).all()
        else:
            assert (np.unpackbits(mm[..., None], axis=-1).sum(-1) == n).all()


def scale_invariance(o):
    W = workloads.masters(16, 256, seed=21)
    W2 = workloads.to_bf16_bits(_f32(W) * 2)
    for n, m in [(2, 4), (6, 8)]:
        a = o.quantize_mask_pack(W, n, m, eps=0.0)
        b = o.quantize_mask_pack(W2, n, m, eps=0.0)
        assert np.array_equal(a["keep"], b["keep"])
        assert np.array_equal(a["ws"], b["ws"])
        assert b["gamma"] == 2 * a["gamma"]


def rescale_closed_form(o):
    rng = np.random.default_rng(2)
    acc = rng.integers(-2 ** 20, 2 ** 20, size=(3, 5)).astype(np.int32)
    s = np.array([0.5, 3.25, 117.0], np.float32)
    g = np.float32(0.0171875)
    y = o.rescale(acc, s, g)
    for t in range(3):
        for j in range(5):
            want = Fraction(int(acc[t, j])) * Fraction(float(g)) * Fraction(float(s[t])) / 127
            assert abs(Fraction(float(y[t, j])) - want) <= abs(want) * Fraction(1, 2 ** 50)


def mask_stats(o):
    g = _read_golden("hand_example_2of4.txt")
    n, m = int(g["n"][0]), int(g["m"][0])
    W = workloads.to_bf16_bits(np.array([[float(v) for v in g["W"]]], np.float32))
    W2 = workloads.to_bf16_bits(np.array([[float(v) for v in g["W2"]]], np.float32))
    r1 = o.quantize_mask_pack(W, n, m, eps=float(g["eps"][0]))
    r2 = o.quantize_mask_pack(W2, n, m, eps=float(g["eps"][0]))
    assert o.count_zero_codes(r1["t"]) == int(g["zeros"][0])
    assert o.count_mask_flips(r1["keep"], r2["keep"]) == int(g["flips"][0])
    assert o.count_mask_flips(r2["keep"], r1["keep"]) == int(g["flips"][0])
    # closed form: three exact zeros and five weights of magnitude 1 give mean |W| = 5/8,
    # 1 / (5/8) = 1.6 -> code +-1, so exactly the three zeros are natural zeros
    Wc = workloads.to_bf16_bits(np.array([[0, 1, -1, 0, 1, 1, 0, -1]], np.float32))
    assert o.count_zero_codes(o.quantize_mask_pack(Wc, 2, 4, eps=0.0)["t"]) == 3
    # the mask depends on the master magnitudes only, and W -> 2W keeps their order: no
    # flips; with n == m every position is kept whatever the weights
    Wt = _tie_heavy_masters(6, 64, seed=11)
    W2x = workloads.to_bf16_bits(workloads.bf16_bits_to_f32(Wt) * np.float32(2.0))
    for (nn, mm) in [(2, 4), (6, 8), (3, 8), (1, 4)]:
        k = o.quantize_mask_pack(Wt, nn, mm)["keep"]
        assert o.count_mask_flips(k, o.quantize_mask_pack(Wt ^ np.uint16(0x8000), nn, mm)["keep"]) == 0
        assert o.count_mask_flips(k, o.quantize_mask_pack(W2x, nn, mm)["keep"]) == 0
    Wr = workloads.masters(6, 64, seed=12)
    assert o.count_mask_flips(o.quantize_mask_pack(Wt, 8, 8)["keep"],
                              o.quantize_mask_pack(Wr, 8, 8)["keep"]) == 0


def backward_hand(o):
    g = _read_golden("hand_example_2of4.txt")
    n, m = int(g["n"][0]), int(g["m"][0])
    W = workloads.to_bf16_bits(np.array([[float(v) for v in g["W"]]], np.float32))
    X = workloads.to_bf16_bits(np.array([[float(v) for v in g["x"]]], np.float32))
    r = o.linear(X, W, n, m, eps=float(g["eps"][0]))
    dY = np.array([[float(g["dY"][0])]], np.float32)
    dX, dW = o.backward(dY, r["Xq"], r["s"], r["ws"], W, r["g"])
    gamma = Fraction(g["gamma"][0])
    for k, v in enumerate(g["dX_over_gamma"]):
        assert Fraction(float(dX[0, k])) == gamma * int(v), (k, dX[0, k])
    den = int(g["dW_den"][0])
    for k, (v, p) in enumerate(zip(g["dW_num"], g["ste_pass"])):
        assert abs(Fraction(float(dW[0, k])) - Fraction(int(v), den)) <= Fraction(1, 2 ** 48)
        if p == "0":
            assert dW[0, k] == 0.0, (k, dW[0, k])


def backward_adjoint(o):
    rng = np.random.default_rng(21)
    T, O, K = 3, 5, 64
    W = _tie_heavy_masters(O, K, seed=22)
    X = workloads.activations(T, K, seed=23)
    r = o.linear(X, W, 2, 4)
    dY = rng.standard_normal((T, O)).astype(np.float32)
    dX, dW = o.backward(dY, r["Xq"], r["s"], r["ws"], W, r["g"])
    X_eff = r["Xq"].astype(np.float64) * (r["s"].astype(np.float64) / 127.0)[:, None]
    W_eff = r["ws"].astype(np.float64) * float(r["g"])
    lhs = float(np.sum(dY.astype(np.float64) * r["y"]))
    rhs = float(np.sum(dX * X_eff))
    assert abs(lhs - rhs) <= 1e-9 * max(1.0, abs(lhs)), (lhs, rhs)
    # dW is the adjoint of V -> X_eff (V * pass)^T, pass = the clip range of W / g; the
    # magnitudes of these masters straddle g, so both sides of the gate occur
    ratio = np.abs(workloads.bf16_bits_to_f32(W)) / np.float32(r["g"])
    gate = (ratio <= np.float32(1.0)).astype(np.float64)
    assert 0 < gate.sum() < gate.size
    for trial in range(3):
        V = rng.standard_normal((O, K))
        lhs = float(np.sum(dW * V))
        rhs = float(np.sum(dY.astype(np.float64) * (X_eff @ (V * gate).T)))
        assert abs(lhs - rhs) <= 1e-9 * max(1.0, abs(lhs)), (trial, lhs, rhs)
    assert np.all(dW[gate == 0] == 0)
    # the weight gradient does not depend on the mask (dense n == m gives the same dW)
    rd = o.linear(X, W, 4, 4)
    _, dWd = o.backward(dY, rd["Xq"], rd["s"], rd["ws"], W, rd["g"])
    assert np.array_equal(dW, dWd)
    assert np.any(dW[r["keep"] == 0] != 0)
    # the gate's boundary: one row of masters that are all +-m (so g = m + eps with eps = 0
    # gives |W| / g == 1 exactly: passes), and one with a single larger magnitude (that one
    # is clipped, the rest pass since the mean is above their magnitude)
    Wb = workloads.to_bf16_bits(np.array([[0.25, -0.25, 0.25, -0.25] * 16,
                                          [0.25, -0.25, 0.25, -0.25] * 15 + [4.0, 0.25, 0.25, 0.25]],
                                         np.float32))
    for row in range(2):
        rb = o.linear(X, Wb[row:row + 1], 2, 4, eps=0.0)
        dYb = np.ones((T, 1), np.float32)
        _, dWb = o.backward(dYb, rb["Xq"], rb["s"], rb["ws"], Wb[row:row + 1], rb["g"])
        full = X_eff.sum(axis=0)
        if row == 0:
            assert np.all(dWb[0] == full)
        else:
            assert dWb[0, 60] == 0.0 and np.all(np.delete(dWb[0], 60) == np.delete(full, 60))


def group_one(o):
    W = _tie_heavy_masters(12, 192, seed=31)
    X = workloads.activations(5, 192, seed=32)
    for (n, m) in [(2, 4), (6, 8), (3, 8)]:
        r1, r = o.group_linear(X, W, n, m, 1), o.linear(X, W, n, m)
        assert float(r1["g"][0]) == float(r["g"]) and int(r1["S"][0]) == int(r["S"])
        for k in ("t", "keep", "ws", "codes", "meta", "Xq"):
            assert np.array_equal(r1[k], r[k]), k
        assert np.array_equal(r1["s"][:, 0], r["s"])
        assert np.array_equal(r1["acc"][0], r["acc"]) and np.array_equal(r1["y"], r["y"])


def group_slices(o):
    rng = np.random.default_rng(33)
    O, K, T = 9, 256, 4
    W = workloads.masters(O, K, seed=34)
    X = workloads.activations(T, K, seed=35)
    # make the blocks' scales differ a lot: scale block 2 of W and block 1 of X by 4
    Wf = workloads.bf16_bits_to_f32(W)
    Wf[:, 128:192] *= 4.0
    W = workloads.to_bf16_bits(Wf)
    Xf = workloads.bf16_bits_to_f32(X)
    Xf[:, 64:128] *= 4.0
    X = workloads.to_bf16_bits(Xf)
    for (n, m, G) in [(2, 4, 4), (6, 8, 2), (1, 4, 4)]:
        r = o.group_linear(X, W, n, m, G)
        kg = K // G
        y = np.zeros((T, O))
        for j in range(G):
            sl = slice(j * kg, (j + 1) * kg)
            rj = o.linear(np.ascontiguousarray(X[:, sl]), np.ascontiguousarray(W[:, sl]), n, m)
            assert float(r["g"][j]) == float(rj["g"]) and int(r["S"][j]) == int(rj["S"])
            for k in ("t", "keep", "ws", "Xq"):
                assert np.array_equal(r[k][:, sl], rj[k]), (G, j, k)
            assert np.array_equal(r["s"][:, j], rj["s"])
            assert np.array_equal(r["acc"][j], rj["acc"])
            y = y + rj["y"]
        assert np.array_equal(r["y"], y)
    assert rng is not None


def group_hand(o):
    g = _read_golden("group_example_g2.txt")
    G, n, m = int(g["G"][0]), int(g["n"][0]), int(g["m"][0])
    W0 = np.array([float(v) for v in g["W0"]] * 8, np.float32)
    x0 = np.array([float(v) for v in g["x0"]] * 8, np.float32)
    W = workloads.to_bf16_bits(np.concatenate([W0, 2 * W0])[None, :])
    X = workloads.to_bf16_bits(np.concatenate([x0, x0 / 2])[None, :])
    r = o.group_linear(X, W, n, m, G, eps=float(g["eps"][0]))
    assert [float(v) for v in r["gamma"]] == [float(v) for v in g["gamma"]]
    ws = np.array([int(v) for v in g["ws"]] * 16, np.int8)
    assert np.array_equal(r["ws"][0], ws)
    assert [float(v) for v in r["s"][0]] == [float(v) for v in g["s"]]
    assert [int(v) for v in r["acc"][:, 0, 0]] == [int(v) for v in g["acc"]]
    y_ref = Fraction(g["y_num"][0]) / int(g["y_den"][0])
    assert abs(Fraction(float(r["y"][0, 0])) - y_ref) <= abs(y_ref) * Fraction(1, 2 ** 50)
    r1 = o.group_linear(X, W, n, m, 1, eps=float(g["eps"][0]))
    assert float(r1["gamma"][0]) == float(g["gamma_g1"][0]) and r1["t"][0, 1] == 0


ALL = [hand_example, mask_bruteforce, gamma_closed_form, rounding_ties, act_quotient_ties,
       dense_pattern,
       constant_magnitude, act_absmax, contract_bruteforce, unpack_roundtrip, invariants,
       scale_invariance, rescale_closed_form, mask_stats, group_one, group_slices, group_hand,
       backward_hand, backward_adjoint]
