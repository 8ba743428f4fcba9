"""The C ABI library loads, exports every entry point its header declares, and rejects bad
arguments on the host before touching a GPU (no GPU needed)."""
import ctypes
import os
import re

import pytest

import oracle
import sparse_linear_layers_absmean_b200 as sbn
from sparse_linear_layers_absmean_b200 import build as sbn_build

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                      "sbn.h")


@pytest.fixture(scope="module")
def L():
    sbn_build.build()
    return sbn.lib()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"SBN_API\s+[\w\s\*]+?\b(sbn_\w+)\s*\(", text)))


def test_header_declares_the_entry_points():
    assert set(sbn.EXPORTED) <= set(declared_symbols())


def test_every_declared_symbol_is_exported(L):
    for name in declared_symbols():
        assert hasattr(L, name), name
        assert ctypes.cast(getattr(L, name), ctypes.c_void_p).value


@pytest.mark.parametrize("n,m", [(2, 4), (6, 8), (1, 4), (3, 4), (4, 4), (1, 8), (5, 8), (8, 8)])
@pytest.mark.parametrize("out,in_", [(1, 64), (37, 192), (256, 256), (6912, 2560), (300, 3200),
                                     (7, 8640)])
def test_dims_match_the_oracle_geometry(L, n, m, out, in_):
    d = sbn.sbn_linear_ref_dims(out, in_, n, m)
    ldc, ldm = oracle.plane_dims(in_, n, m)
    assert (d.codes_ld, d.meta_ld) == (ldc, ldm)
    assert d.codes_bytes == out * ldc and d.meta_bytes == out * ldm
    stored = in_ // 2 if (n, m) == (2, 4) else in_
    assert d.codes_row_bytes == stored // 4 and d.meta_row_bytes == in_ // 8
    assert d.pack_workspace_bytes >= 8 * 1024 and d.pack_workspace_bytes % 256 == 0


@pytest.mark.parametrize("args,status", [
    ((0, 64, 2, 4), 2), ((-1, 64, 2, 4), 2), ((8, 0, 2, 4), 2), ((8, 96, 2, 4), 2),
    ((8, 32, 2, 4), 2), ((8, 64 * 3000, 2, 4), 2), ((2 ** 20, 4096, 2, 4), 2),
    ((8, 64, 2, 3), 3), ((8, 64, 0, 4), 3), ((8, 64, 5, 4), 3), ((8, 64, 9, 8), 3),
    ((8, 64, 2, 16), 3)])
def test_dims_rejects_bad_arguments(L, args, status):
    d = sbn.SbnDims()
    assert L.sbn_linear_ref_dims(*args, ctypes.byref(d)) == status
    assert L.sbn_linear_ref_dims(*args[:4], None) in (1, status)


def _p(v):
    return ctypes.c_void_p(v)


def test_entry_points_validate_before_launching(L):
    # Every call below fails validation on the host and returns before any CUDA call.
    A = _p(0x10000)   # a 16-byte aligned placeholder address, never dereferenced
    U = _p(0x10008)   # misaligned
    f = ctypes.c_float
    q = L.sbn_quantize_mask_pack_weights
    assert q(None, 8, 64, 2, 4, f(1e-5), A, A, A, A, None, None, None) == 1
    assert q(A, 8, 64, 2, 4, f(1e-5), None, A, A, A, None, None, None) == 1
    assert q(A, 8, 64, 2, 4, f(1e-5), A, A, A, None, None, None, None) == 1
    assert q(A, 8, 96, 2, 4, f(1e-5), A, A, A, A, None, None, None) == 2
    assert q(A, 8, 64, 3, 5, f(1e-5), A, A, A, A, None, None, None) == 3
    assert q(U, 8, 64, 2, 4, f(1e-5), A, A, A, A, None, None, None) == 4
    assert q(A, 8, 64, 2, 4, f(1e-5), A, A, A, A, U, None, None) == 4
    assert q(A, 8, 64, 2, 4, f(-1.0), A, A, A, A, None, None, None) == 6
    assert q(A, 8, 64, 2, 4, f(float("nan")), A, A, A, A, None, None, None) == 6
    assert q(A, 8, 64, 2, 4, f(float("inf")), A, A, A, A, None, None, None) == 6
    a = L.sbn_quantize_acts
    assert a(None, 4, 64, A, A, None, None) == 1
    assert a(A, 4, 65, A, A, None, None) == 2
    assert a(A, -1, 64, A, A, None, None) == 2
    assert a(U, 4, 64, A, A, None, None) == 4
    assert a(A, 0, 64, A, A, None, None) == 0  # empty: a valid no-op, nothing launched
    ln = L.sbn_linear
    assert ln(A, A, A, A, A, 4, 8, 64, 2, 4, None, 0, None, None, None) == 1
    assert ln(A, A, A, A, A, 4, 8, 64, 2, 7, A, 0, None, None, None) == 3
    assert ln(A, A, A, A, A, -2, 8, 64, 2, 4, A, 0, None, None, None) == 2
    assert ln(A, A, A, A, A, 4, 8, 64, 2, 4, U, 0, None, None, None) == 4
    assert ln(A, A, A, A, A, 0, 8, 64, 2, 4, A, 0, None, None, None) == 0


def test_statistics_entry_points_validate(L):
    A = _p(0x10000)
    U = _p(0x10004)   # 4-byte aligned only
    z = L.sbn_count_zero_codes
    assert z(None, A, 8, 64, A, None) == 1
    assert z(A, A, 8, 64, None, None) == 1
    assert z(A, A, 8, 96, A, None) == 2
    assert z(A, A, 0, 64, A, None) == 2
    assert z(U, A, 8, 64, A, None) == 4
    assert z(A, A, 8, 64, U, None) == 4   # the uint64 count must be 8-byte aligned
    f = L.sbn_count_mask_flips
    assert f(None, A, 8, 64, 2, 4, A, None) == 1
    assert f(A, A, 8, 64, 2, 4, None, None) == 1
    assert f(A, A, 8, 96, 2, 4, A, None) == 2
    assert f(A, A, 8, 64, 5, 4, A, None) == 3
    assert f(A, U, 8, 64, 2, 4, A, None) == 4
    assert f(A, A, 8, 64, 6, 8, U, None) == 4


def test_status_strings(L):
    for s in range(7):
        assert L.sbn_status_string(s)


def _group(specs, A=0x10000):
    """ctypes array of layers with placeholder (aligned, never dereferenced) pointers."""
    arr = (sbn.SbnGroupLinear * len(specs))()
    for i, (O, K, T, n, m) in enumerate(specs):
        arr[i] = sbn.SbnGroupLinear(X=A, Xq=A, absmax=A, codes=A, meta=A, gamma_eff=A, Y=A,
                                    acc_dbg=None, tokens=T, out=O, in_=K, n=n, m=m,
                                    y_is_bf16=0, reserved=0, ldx=0, ldc=0, ldm=0)
    return arr


def _sizes(L, arr):
    pb, wb = ctypes.c_int64(), ctypes.c_int64()
    st = L.sbn_group_plan_sizes(ctypes.cast(arr, ctypes.c_void_p), len(arr), ctypes.byref(pb),
                                ctypes.byref(wb))
    return st, pb.value, wb.value


def test_group_plan_sizes_validate(L):
    assert _sizes(L, _group([(128, 256, 16, 6, 8)]))[0] == 3      # 2:4 only
    assert _sizes(L, _group([(128, 256, 33, 2, 4)]))[0] == 2      # at most 32 tokens
    assert _sizes(L, _group([(128, 96, 16, 2, 4)]))[0] == 2       # in % 64
    assert _sizes(L, _group([(128, 256, 16, 2, 4)], A=0x10004))[0] == 4
    arr = _group([(128, 256, 16, 2, 4)])
    arr[0].Y = None
    assert _sizes(L, arr)[0] == 1
    arr = _group([(128, 256, 0, 2, 4)])
    arr[0].Y = None                                               # 0 tokens: not checked
    assert _sizes(L, arr)[0] == 0
    assert L.sbn_group_plan_sizes(None, 1, ctypes.byref(ctypes.c_int64()),
                                  ctypes.byref(ctypes.c_int64())) == 1
    A = _p(0x10000)
    assert L.sbn_group_plan(ctypes.cast(arr, ctypes.c_void_p), 1, _p(0x10040), 4096) == 4
    assert L.sbn_linear_group(None, A, A, None, None) == 1
    assert L.sbn_linear_group(A, _p(0x10040), A, None, None) == 4
    assert L.sbn_quantize_acts_group(A, None, None, None) == 1


def test_group_schedule_sizes(L):
    """Host-side schedule (SM count 148 without a device): the whole 4096-hidden stack at 16
    tokens has enough row tiles for every SM, so no split and no workspace; one small layer
    alone is split over several units and needs a workspace for its partials."""
    import workloads
    stack = [(O, K, 16, 2, 4) for _ in range(workloads.STACK_LAYERS)
             for _, O, K in workloads.STACK_LAYER_SHAPES]
    st, pb, wb = _sizes(L, _group(stack))
    assert st == 0 and wb == 0
    tiles = workloads.STACK_LAYERS * sum((O + 127) // 128 for _, O, _ in workloads.STACK_LAYER_SHAPES)
    assert pb >= 128 + 512 * len(stack) + 32 * tiles
    st, pb, wb = _sizes(L, _group([(256, 4096, 16, 2, 4)]))
    assert st == 0 and wb > 0


def _pack_group(specs, A=0x10000):
    """ctypes array of grouped-pack tensors with placeholder pointers; specs are
    (O, K, n, m, n2, m2)."""
    arr = (sbn.SbnPackGroupTensor * len(specs))()
    for i, (O, K, n, m, n2, m2) in enumerate(specs):
        two = m2 != 0
        arr[i] = sbn.SbnPackGroupTensor(W=A, codes=A, meta=A, codes2=A if two else None,
                                        meta2=A if two else None, gamma_eff=A, dense_dbg=None,
                                        dense_dbg2=None, out=O, in_=K, n=n, m=m, n2=n2, m2=m2,
                                        eps=1e-5, reserved=0)
    return arr


def _pack_sizes(L, arr):
    pb, wb = ctypes.c_int64(), ctypes.c_int64()
    st = L.sbn_pack_group_sizes(ctypes.cast(arr, ctypes.c_void_p), len(arr), ctypes.byref(pb),
                                ctypes.byref(wb))
    return st, pb.value, wb.value


def test_pack_group_sizes_validate(L):
    assert _pack_sizes(L, _pack_group([(128, 256, 6, 8, 2, 4)]))[0] == 0
    assert _pack_sizes(L, _pack_group([(128, 256, 2, 4, 0, 0)]))[0] == 0
    assert _pack_sizes(L, _pack_group([(128, 256, 1, 4, 0, 0)]))[0] == 3   # fast patterns only
    assert _pack_sizes(L, _pack_group([(128, 256, 6, 8, 6, 8)]))[0] == 3   # two equal patterns
    assert _pack_sizes(L, _pack_group([(128, 256, 6, 8, 3, 8)]))[0] == 3
    assert _pack_sizes(L, _pack_group([(128, 96, 6, 8, 2, 4)]))[0] == 2    # in % 64
    assert _pack_sizes(L, _pack_group([(1 << 16, 1 << 15, 2, 4, 0, 0)]))[0] == 2  # 2^31 weights
    assert _pack_sizes(L, _pack_group([(128, 256, 6, 8, 2, 4)], A=0x10008))[0] == 4
    arr = _pack_group([(128, 256, 6, 8, 2, 4)])
    arr[0].codes2 = None
    assert _pack_sizes(L, arr)[0] == 1
    arr = _pack_group([(128, 256, 6, 8, 2, 4)])
    arr[0].eps = float("nan")
    assert _pack_sizes(L, arr)[0] == 6
    assert L.sbn_pack_group_sizes(None, 1, ctypes.byref(ctypes.c_int64()),
                                  ctypes.byref(ctypes.c_int64())) == 1
    A = _p(0x10000)
    # a plan buffer that is not a plan: refused before any launch
    junk = (ctypes.c_uint8 * 64)()
    assert L.sbn_quantize_mask_pack_weights_group(ctypes.cast(junk, ctypes.c_void_p), A, A,
                                                  None, None) == 6
    assert L.sbn_quantize_mask_pack_weights_group(None, A, A, None, None) == 1
    assert L.sbn_quantize_mask_pack_weights_group(A, _p(0x10008), A, None, None) == 4


def test_pack_group_plan_layout(L):
    """The plan's chunk and warp-iteration bookkeeping for the training-step tensors plus
    ragged ones: 256 KB chunks of W per tensor, 8 blocks of 64 weights per iteration, both
    counted from each tensor's start."""
    import numpy as np
    import workloads
    specs = [(O, K, 6, 8, 2, 4) for _, O, K in workloads.TRAIN_LAYER_SHAPES]
    specs += [(1, 64, 2, 4, 6, 8), (37, 192, 6, 8, 0, 0), (130, 4160, 2, 4, 0, 0)]
    arr = _pack_group(specs)
    st, pb, wb = _pack_sizes(L, arr)
    assert st == 0 and wb == 16 * len(specs)
    entry = (pb - 64) // len(specs)
    assert pb == 64 + entry * len(specs) and entry % 16 == 0
    buf = (ctypes.c_uint8 * (pb + 16))()
    base = (ctypes.addressof(buf) + 15) // 16 * 16
    assert L.sbn_pack_group_plan(ctypes.cast(arr, ctypes.c_void_p), len(arr), _p(base), pb) == 0
    raw = np.frombuffer(buf, dtype=np.uint8)[base - ctypes.addressof(buf):][:pb]
    hdr = raw[:20].view(np.uint32)
    chunks = [-(-(O * K // 8) // 16384) for O, K, *_ in specs]
    iters = [-(-(O * K // 64) // 8) for O, K, *_ in specs]
    assert hdr[0] == 0x31475053 and hdr[1] == len(specs)
    assert hdr[2] == sum(chunks) and hdr[3] == sum(iters)
    assert hdr[4].view(np.int32) == -1  # mixed patterns: the general kernel
    for i, (O, K, n, m, n2, m2) in enumerate(specs):
        e = raw[64 + i * entry:64 + (i + 1) * entry]
        nvec = int(e[256:264].view(np.int64)[0])
        cb, nc, qb, nq, ca, cb2 = e[264:288].view(np.int32)
        assert nvec == O * K // 8
        assert (cb, nc) == (sum(chunks[:i]), chunks[i]) and (qb, nq) == (sum(iters[:i]), iters[i])
        # two patterns are stored 6:8 first, 2:4 second, whichever order was asked
        assert (ca, cb2) == (0, 1) if m2 else ca == (n == 2)


@pytest.mark.parametrize("specs,mode", [([(96, 256, 6, 8, 2, 4), (8, 64, 2, 4, 6, 8)], 2),
                                        ([(96, 256, 6, 8, 0, 0)] * 2, 0),
                                        ([(96, 256, 2, 4, 0, 0)] * 3, 1),
                                        ([(96, 256, 2, 4, 0, 0), (96, 256, 6, 8, 0, 0)], -1)])
def test_pack_group_plan_mode(L, specs, mode):
    """Plans whose tensors share their patterns (and ask for no dense matrix) name the
    fixed-pattern kernel; any other plan the general one."""
    import numpy as np
    for dense in (False, True):
        arr = _pack_group(specs)
        if dense:
            arr[0].dense_dbg = 0x10000
        st, pb, _ = _pack_sizes(L, arr)
        buf = (ctypes.c_uint8 * (pb + 16))()
        base = (ctypes.addressof(buf) + 15) // 16 * 16
        assert L.sbn_pack_group_plan(ctypes.cast(arr, ctypes.c_void_p), len(arr), _p(base),
                                     pb) == 0
        raw = np.frombuffer(buf, dtype=np.uint8)[base - ctypes.addressof(buf):][:pb]
        assert raw[16:20].view(np.int32)[0] == (-1 if dense else mode)


def test_group_strides_validate(L):
    """A layer may be a K slice of a wider one: strides at least the slice's row, multiples
    of 16; the ordered sum of group quantisation checks its arguments on the host."""
    arr = _group([(128, 256, 16, 2, 4)])
    arr[0].ldx, arr[0].ldc, arr[0].ldm = 1024, 128, 128
    assert _sizes(L, arr)[0] == 0
    for field, bad in (("ldx", 128), ("ldx", 1040 + 8), ("ldc", 16), ("ldc", 40), ("ldm", 24),
                       ("ldx", -16)):
        arr = _group([(128, 256, 16, 2, 4)])
        setattr(arr[0], field, bad)
        assert _sizes(L, arr)[0] == 2, (field, bad)
    A = _p(0x10000)
    assert L.sbn_gq_sum(A, 0, 4, A, 0, None) == 0            # nothing to add
    assert L.sbn_gq_sum(A, 16, 0, A, 0, None) == 2           # G in 1..64
    assert L.sbn_gq_sum(A, 16, 65, A, 0, None) == 2
    assert L.sbn_gq_sum(None, 16, 4, A, 0, None) == 1
    assert L.sbn_gq_sum(_p(0x10004), 16, 4, A, 0, None) == 4
