"""CPU oracle of the Sparse-BitLinear forward.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by ``__graft_entry__.smoke()`` and by
the CPU-baseline leg of ``bench.py``; never by the product library.  The arithmetic lives
in ``sbn_oracle.c`` (plain scalar C, fp64 where the pages fix no precision, fp32 where an
fp32 decision produces an integer code); this module only marshals numpy arrays.

Every function cites the passage it restates; see ``sbn_oracle.c`` for the citations
(the Sparse-BitNet technical summaries, section 2 "Methodology"; the bitnet.cpp article,
"Fundamento matemático"; the BitNet project page, "Especificaciones Técnicas").
"""
import ctypes

import numpy as np

from . import build as _build

_DEFAULT = None

ERR_W_NONFINITE = 1
ERR_W_RANGE = 2
ERR_X_NONFINITE = 4
ERR_ACC_OVERFLOW = 8


def load_library(path):
    """Load a compiled oracle (the default one, or a test's deliberately broken copy)."""
    lib = ctypes.CDLL(path)
    p = ctypes.c_void_p
    i64 = ctypes.c_int64
    lib.oracle_rounding_is_nearest.restype = ctypes.c_int
    lib.oracle_num_threads.restype = ctypes.c_int
    lib.oracle_weight_gamma.argtypes = [p, i64, ctypes.c_float, p, p, p]
    lib.oracle_weight_gamma.restype = ctypes.c_int
    lib.oracle_ternary_mask.argtypes = [p, i64, i64, ctypes.c_int, ctypes.c_int,
                                        ctypes.c_float, p, p, p]
    lib.oracle_ternary_mask.restype = None
    lib.oracle_pack.argtypes = [p, p, i64, i64, ctypes.c_int, ctypes.c_int, p, i64, p, i64]
    lib.oracle_pack.restype = ctypes.c_int
    lib.oracle_quant_acts.argtypes = [p, i64, i64, p, p]
    lib.oracle_quant_acts.restype = ctypes.c_int
    lib.oracle_contract.argtypes = [p, p, i64, i64, i64, p]
    lib.oracle_contract.restype = ctypes.c_int
    lib.oracle_rescale.argtypes = [p, p, ctypes.c_float, i64, i64, p]
    lib.oracle_rescale.restype = None
    lib.oracle_count_zero_codes.argtypes = [p, i64]
    lib.oracle_count_zero_codes.restype = i64
    lib.oracle_count_mask_flips.argtypes = [p, p, i64]
    lib.oracle_count_mask_flips.restype = i64
    lib.oracle_backward.argtypes = [p, p, p, p, p, ctypes.c_float, i64, i64, i64, p, p]
    lib.oracle_backward.restype = None
    lib.oracle_group_gamma.argtypes = [p, i64, i64, ctypes.c_int, ctypes.c_float, p, p, p]
    lib.oracle_group_gamma.restype = ctypes.c_int
    lib.oracle_group_ternary_mask.argtypes = [p, i64, i64, ctypes.c_int, ctypes.c_int,
                                              ctypes.c_int, p, p, p, p]
    lib.oracle_group_ternary_mask.restype = None
    lib.oracle_group_quant_acts.argtypes = [p, i64, i64, ctypes.c_int, p, p]
    lib.oracle_group_quant_acts.restype = ctypes.c_int
    lib.oracle_group_contract_rescale.argtypes = [p, p, p, p, i64, i64, i64, ctypes.c_int, p, p]
    lib.oracle_group_contract_rescale.restype = ctypes.c_int
    if not lib.oracle_rounding_is_nearest():
        raise RuntimeError("oracle needs round-to-nearest-even on the host FPU")
    return lib


_OVERRIDE = None


def use_library(lib):
    """Route the functions below through ``lib`` (None restores the default build)."""
    global _OVERRIDE
    _OVERRIDE = lib


def _lib():
    global _DEFAULT
    if _OVERRIDE is not None:
        return _OVERRIDE
    if _DEFAULT is None:
        _DEFAULT = load_library(_build.build())
    return _DEFAULT


def _ptr(a):
    return ctypes.c_void_p(a.ctypes.data)


def num_threads() -> int:
    return int(_lib().oracle_num_threads())


def _bits(a):
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError("bf16 inputs are passed as their uint16 bit patterns")
    return a


def plane_dims(K: int, n: int, m: int):
    """Row strides (bytes) of the codes and meta planes, each row's data rounded up to 16
    bytes.  codes: 2 bits per stored element (K/2 kept elements for 2:4, K positions
    otherwise); meta: 4 bits per group for m == 4, 8 bits per group for m == 8."""
    stored = K // 2 if (n, m) == (2, 4) else K
    codes_bytes = -(-(stored * 2) // 8)
    meta_bytes = -(-((K // m) * (4 if m == 4 else 8)) // 8)
    return (-(-codes_bytes // 16) * 16, -(-meta_bytes // 16) * 16)


def weight_gamma(W_bits, eps: float):
    """S1: (S, gamma, g, err) for the whole tensor."""
    W = _bits(W_bits)
    S = ctypes.c_uint64()
    gamma = ctypes.c_float()
    g = ctypes.c_float()
    err = _lib().oracle_weight_gamma(_ptr(W), W.size, ctypes.c_float(eps), ctypes.byref(S),
                                     ctypes.byref(gamma), ctypes.byref(g))
    return int(S.value), np.float32(gamma.value), np.float32(g.value), int(err)


def ternary_mask(W_bits, n: int, m: int, g):
    """S2-S4(apply): (t, keep, ws), each [O, K]."""
    W = _bits(W_bits)
    O, K = W.shape
    t = np.empty((O, K), np.int8)
    keep = np.empty((O, K), np.uint8)
    ws = np.empty((O, K), np.int8)
    _lib().oracle_ternary_mask(_ptr(W), O, K, n, m, ctypes.c_float(float(g)), _ptr(t),
                               _ptr(keep), _ptr(ws))
    return t, keep, ws


def pack(t, keep, n: int, m: int):
    """S4(pack): (codes [O, ldc] u8, meta [O, ldm] u8)."""
    t = np.ascontiguousarray(t, np.int8)
    keep = np.ascontiguousarray(keep, np.uint8)
    O, K = t.shape
    ldc, ldm = plane_dims(K, n, m)
    codes = np.empty((O, ldc), np.uint8)
    meta = np.empty((O, ldm), np.uint8)
    bad = _lib().oracle_pack(_ptr(t), _ptr(keep), O, K, n, m, _ptr(codes), ldc, _ptr(meta), ldm)
    if bad:
        raise AssertionError("a group does not keep exactly n positions")
    return codes, meta


def quantize_mask_pack(W_bits, n: int, m: int, eps: float = 1e-5):
    """S1-S4 for one master tensor; returns a dict of every intermediate."""
    S, gamma, g, err = weight_gamma(W_bits, eps)
    t, keep, ws = ternary_mask(W_bits, n, m, g)
    codes, meta = pack(t, keep, n, m)
    return dict(S=S, gamma=gamma, g=g, err=err, t=t, keep=keep, ws=ws, codes=codes, meta=meta)


def quant_acts(X_bits):
    """S5: (Xq [T, K] int8, s [T] fp32, err)."""
    X = _bits(X_bits)
    T, K = X.shape
    Xq = np.empty((T, K), np.int8)
    s = np.empty((T,), np.float32)
    err = _lib().oracle_quant_acts(_ptr(X), T, K, _ptr(Xq), _ptr(s))
    return Xq, s, int(err)


def contract(Xq, Ws):
    """S6: acc [T, O] int32 (exact; raises if an int32 would overflow)."""
    Xq = np.ascontiguousarray(Xq, np.int8)
    Ws = np.ascontiguousarray(Ws, np.int8)
    T, K = Xq.shape
    O, K2 = Ws.shape
    assert K == K2
    acc = np.empty((T, O), np.int32)
    err = _lib().oracle_contract(_ptr(Xq), _ptr(Ws), T, O, K, _ptr(acc))
    if err:
        raise OverflowError("int32 accumulator overflow")
    return acc


def rescale(acc, s, g):
    """S7: y [T, O] fp64 = acc * g * s / 127."""
    acc = np.ascontiguousarray(acc, np.int32)
    s = np.ascontiguousarray(s, np.float32)
    T, O = acc.shape
    y = np.empty((T, O), np.float64)
    _lib().oracle_rescale(_ptr(acc), _ptr(s), ctypes.c_float(float(g)), T, O, _ptr(y))
    return y


def linear(X_bits, W_bits, n: int, m: int, eps: float = 1e-5):
    """The whole forward S1-S7; returns a dict with every intermediate and y (fp64)."""
    w = quantize_mask_pack(W_bits, n, m, eps)
    Xq, s, xerr = quant_acts(X_bits)
    acc = contract(Xq, w["ws"])
    y = rescale(acc, s, w["g"])
    w.update(Xq=Xq, s=s, xerr=xerr, acc=acc, y=y)
    return w


def count_zero_codes(t):
    """Natural zeros: positions whose ternary code (before the mask) is 0."""
    t = np.ascontiguousarray(t, np.int8)
    return int(_lib().oracle_count_zero_codes(_ptr(t), t.size))


def count_mask_flips(keep_a, keep_b):
    """Positions kept by one of two masks of the same tensor and pruned by the other."""
    a = np.ascontiguousarray(keep_a, np.uint8)
    b = np.ascontiguousarray(keep_b, np.uint8)
    assert a.shape == b.shape
    return int(_lib().oracle_count_mask_flips(_ptr(a), _ptr(b), a.size))


def backward(dY, Xq, s, Ws, W_bits, g):
    """Dual-STE backward: (dX [T, K], dW [O, K]) in fp64 for the forward's effective
    operands W_eff = g * Ws and X_eff = s / 127 * Xq.  dW reaches every master weight the
    mask pruned, and is zero where the quantiser clips (fl32(|W| / g) > 1)."""
    dY = np.ascontiguousarray(dY, np.float32)
    Xq = np.ascontiguousarray(Xq, np.int8)
    s = np.ascontiguousarray(s, np.float32)
    Ws = np.ascontiguousarray(Ws, np.int8)
    W_bits = np.ascontiguousarray(W_bits, np.uint16)
    T, O = dY.shape
    O2, K = Ws.shape
    assert O == O2 and Xq.shape == (T, K) and s.shape == (T,) and W_bits.shape == (O, K)
    dX = np.empty((T, K), np.float64)
    dW = np.empty((O, K), np.float64)
    _lib().oracle_backward(_ptr(dY), _ptr(Xq), _ptr(s), _ptr(Ws), _ptr(W_bits),
                           ctypes.c_float(float(g)), T, O, K, _ptr(dX), _ptr(dW))
    return dX, dW


def group_linear(X_bits, W_bits, n: int, m: int, G: int, eps: float = 1e-5):
    """Group-quantised forward (G blocks along K, each with its own weight scale g_j and
    per-token activation scale s_tj); a dict with every intermediate and y (fp64)."""
    W = np.ascontiguousarray(W_bits, np.uint16)
    X = np.ascontiguousarray(X_bits, np.uint16)
    O, K = W.shape
    T = X.shape[0]
    assert K % G == 0 and X.shape[1] == K
    S = np.empty(G, np.uint64)
    gamma = np.empty(G, np.float32)
    g = np.empty(G, np.float32)
    err = _lib().oracle_group_gamma(_ptr(W), O, K, G, ctypes.c_float(eps), _ptr(S), _ptr(gamma),
                                    _ptr(g))
    t = np.empty((O, K), np.int8)
    keep = np.empty((O, K), np.uint8)
    ws = np.empty((O, K), np.int8)
    _lib().oracle_group_ternary_mask(_ptr(W), O, K, n, m, G, _ptr(g), _ptr(t), _ptr(keep), _ptr(ws))
    codes, meta = pack(t, keep, n, m)
    Xq = np.empty((T, K), np.int8)
    s = np.empty((T, G), np.float32)
    xerr = _lib().oracle_group_quant_acts(_ptr(X), T, K, G, _ptr(Xq), _ptr(s))
    acc = np.empty((G, T, O), np.int32)
    y = np.empty((T, O), np.float64)
    if _lib().oracle_group_contract_rescale(_ptr(Xq), _ptr(ws), _ptr(s), _ptr(g), T, O, K, G,
                                            _ptr(acc), _ptr(y)):
        raise OverflowError("int32 accumulator overflow")
    return dict(S=S, gamma=gamma, g=g, err=int(err), t=t, keep=keep, ws=ws, codes=codes,
                meta=meta, Xq=Xq, s=s, xerr=int(xerr), acc=acc, y=y)
