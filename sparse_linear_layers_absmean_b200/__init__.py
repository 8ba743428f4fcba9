"""Sparse-BitLinear forward on B200 (sm_100a): thin Python binding of libsbn.so.

The C ABI (include/sbn.h) does all the work in CUDA kernels; this module only marshals
arguments.  PyTorch provides device memory and streams.  The functions named like the
C entry points take torch tensors and forward their data pointers; the helpers at the end
(`pack_weights`, `quantize_acts`, `linear`, `forward`) allocate the output tensors with
torch and call them.

There is no CPU fallback: if libsbn.so cannot be loaded, or a tensor is not on a CUDA
device, the call raises.
"""
import contextlib
import ctypes
import os
from typing import NamedTuple, Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libsbn.so")

SBN_OK = 0
STATUS = {0: "SBN_OK", 1: "SBN_ERR_NULL", 2: "SBN_ERR_SHAPE", 3: "SBN_ERR_PATTERN",
          4: "SBN_ERR_ALIGN", 5: "SBN_ERR_CUDA", 6: "SBN_ERR_ARG"}
FLAG_W_NONFINITE = 1
FLAG_W_RANGE = 2
FLAG_X_NONFINITE = 4
FLAG_TIMEOUT = 8

EXPORTED = ("sbn_linear_ref_dims", "sbn_quantize_mask_pack_weights", "sbn_quantize_acts",
            "sbn_linear", "sbn_status_string", "sbn_quantize_mask_pack_weights_noalloc",
            "sbn_count_zero_codes", "sbn_count_mask_flips", "sbn_group_plan_sizes",
            "sbn_group_plan", "sbn_quantize_acts_group", "sbn_linear_group",
            "sbn_operand_bytes", "sbn_expand_operand", "sbn_linear_operand",
            "sbn_backward_workspace_bytes", "sbn_backward", "sbn_quantize_linear",
            "sbn_gq_workspace_bytes", "sbn_quantize_mask_pack_weights_gq", "sbn_quantize_acts_gq",
            "sbn_linear_gq", "sbn_pack_group_sizes", "sbn_pack_group_plan",
            "sbn_quantize_mask_pack_weights_group", "sbn_gq_sum")


class SbnError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {STATUS.get(status, status)}")
        self.status = status


class SbnDims(ctypes.Structure):
    _fields_ = [("codes_ld", ctypes.c_int64), ("meta_ld", ctypes.c_int64),
                ("codes_row_bytes", ctypes.c_int64), ("meta_row_bytes", ctypes.c_int64),
                ("codes_bytes", ctypes.c_int64), ("meta_bytes", ctypes.c_int64),
                ("pack_workspace_bytes", ctypes.c_int64)]


class SbnGroupLinear(ctypes.Structure):
    """One layer of a grouped call (sbn_group_linear in sbn.h)."""
    _fields_ = [("X", ctypes.c_void_p), ("Xq", ctypes.c_void_p), ("absmax", ctypes.c_void_p),
                ("codes", ctypes.c_void_p), ("meta", ctypes.c_void_p),
                ("gamma_eff", ctypes.c_void_p), ("Y", ctypes.c_void_p),
                ("acc_dbg", ctypes.c_void_p), ("tokens", ctypes.c_int64),
                ("out", ctypes.c_int64), ("in_", ctypes.c_int64), ("n", ctypes.c_int32),
                ("m", ctypes.c_int32), ("y_is_bf16", ctypes.c_int32),
                ("reserved", ctypes.c_int32), ("ldx", ctypes.c_int64), ("ldc", ctypes.c_int64),
                ("ldm", ctypes.c_int64)]


class SbnPackGroupTensor(ctypes.Structure):
    """One tensor of a grouped pack (sbn_pack_group_tensor in sbn.h)."""
    _fields_ = [("W", ctypes.c_void_p), ("codes", ctypes.c_void_p), ("meta", ctypes.c_void_p),
                ("codes2", ctypes.c_void_p), ("meta2", ctypes.c_void_p),
                ("gamma_eff", ctypes.c_void_p), ("dense_dbg", ctypes.c_void_p),
                ("dense_dbg2", ctypes.c_void_p), ("out", ctypes.c_int64), ("in_", ctypes.c_int64),
                ("n", ctypes.c_int32), ("m", ctypes.c_int32), ("n2", ctypes.c_int32),
                ("m2", ctypes.c_int32), ("eps", ctypes.c_float), ("reserved", ctypes.c_int32)]


_LIB = None


def lib():
    """Load libsbn.so (built in-tree by ``build.py``); raises if it is missing."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is not built; run sparse_linear_layers_absmean_b200/"
                               "build.py (or __graft_entry__.build())")
        L = ctypes.CDLL(LIB_PATH)
        p, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        L.sbn_linear_ref_dims.argtypes = [i64, i64, i32, i32, ctypes.POINTER(SbnDims)]
        L.sbn_linear_ref_dims.restype = i32
        L.sbn_quantize_mask_pack_weights.argtypes = [p, i64, i64, i32, i32, ctypes.c_float, p, p,
                                                     p, p, p, p, p]
        L.sbn_quantize_mask_pack_weights.restype = i32
        L.sbn_quantize_mask_pack_weights_noalloc.argtypes = [p, i64, i64, i32, i32,
                                                             ctypes.c_float, p, p, p, p, p, p]
        L.sbn_quantize_mask_pack_weights_noalloc.restype = i32
        L.sbn_quantize_acts.argtypes = [p, i64, i64, p, p, p, p]
        L.sbn_quantize_acts.restype = i32
        L.sbn_linear.argtypes = [p, p, p, p, p, i64, i64, i64, i32, i32, p, i32, p, p, p]
        L.sbn_linear.restype = i32
        L.sbn_count_zero_codes.argtypes = [p, p, i64, i64, p, p]
        L.sbn_count_zero_codes.restype = i32
        L.sbn_count_mask_flips.argtypes = [p, p, i64, i64, i32, i32, p, p]
        L.sbn_count_mask_flips.restype = i32
        L.sbn_gq_sum.argtypes = [p, i64, i32, p, i32, p]
        L.sbn_gq_sum.restype = i32
        L.sbn_pack_group_sizes.argtypes = [p, i32, p, p]
        L.sbn_pack_group_sizes.restype = i32
        L.sbn_pack_group_plan.argtypes = [p, i32, p, i64]
        L.sbn_pack_group_plan.restype = i32
        L.sbn_quantize_mask_pack_weights_group.argtypes = [p, p, p, p, p]
        L.sbn_quantize_mask_pack_weights_group.restype = i32
        L.sbn_group_plan_sizes.argtypes = [p, i32, p, p]
        L.sbn_group_plan_sizes.restype = i32
        L.sbn_group_plan.argtypes = [p, i32, p, i64]
        L.sbn_group_plan.restype = i32
        L.sbn_quantize_acts_group.argtypes = [p, p, p, p]
        L.sbn_quantize_acts_group.restype = i32
        L.sbn_linear_group.argtypes = [p, p, p, p, p]
        L.sbn_linear_group.restype = i32
        L.sbn_operand_bytes.argtypes = [i64, i64, i32, i32, p]
        L.sbn_operand_bytes.restype = i32
        L.sbn_expand_operand.argtypes = [p, p, i64, i64, i32, i32, p, p]
        L.sbn_expand_operand.restype = i32
        L.sbn_linear_operand.argtypes = [p, p, p, p, i64, i64, i64, i32, i32, p, i32, p, p, p]
        L.sbn_linear_operand.restype = i32
        L.sbn_backward_workspace_bytes.argtypes = [i64, i64, i64, p]
        L.sbn_backward_workspace_bytes.restype = i32
        L.sbn_backward.argtypes = [p, p, p, p, p, p, p, i64, i64, i64, i32, i32, p, p, p, p, p]
        L.sbn_backward.restype = i32
        L.sbn_quantize_linear.argtypes = [p, p, p, p, i64, i64, i64, i32, i32, p, p, p, i32, p, p,
                                          p]
        L.sbn_quantize_linear.restype = i32
        L.sbn_gq_workspace_bytes.argtypes = [i64, i64, i64, i32, p]
        L.sbn_gq_workspace_bytes.restype = i32
        L.sbn_quantize_mask_pack_weights_gq.argtypes = [p, i64, i64, i32, i32, i32, ctypes.c_float,
                                                        p, p, p, p, p, p, p]
        L.sbn_quantize_mask_pack_weights_gq.restype = i32
        L.sbn_quantize_acts_gq.argtypes = [p, i64, i64, i32, p, p, p, p]
        L.sbn_quantize_acts_gq.restype = i32
        L.sbn_linear_gq.argtypes = [p, p, p, p, p, i64, i64, i64, i32, i32, i32, p, i32, p, p, p, p]
        L.sbn_linear_gq.restype = i32
        L.sbn_status_string.argtypes = [i32]
        L.sbn_status_string.restype = ctypes.c_char_p
        _LIB = L
    return _LIB


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("sbn kernels take CUDA tensors only (no CPU path)")
    if not t.is_contiguous():
        raise ValueError("sbn kernels take contiguous tensors")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(status: int, what: str):
    if status != SBN_OK:
        raise SbnError(status, what)


# ---- the C entry points ------------------------------------------------------------------

def sbn_linear_ref_dims(out: int, in_: int, n: int, m: int) -> SbnDims:
    d = SbnDims()
    _check(lib().sbn_linear_ref_dims(out, in_, n, m, ctypes.byref(d)), "sbn_linear_ref_dims")
    return d


def sbn_quantize_mask_pack_weights(W, n, m, eps, codes, meta, gamma_eff, workspace,
                                   dense_dbg=None, err_flag=None, stream=None):
    out, in_ = W.shape
    _check(lib().sbn_quantize_mask_pack_weights(
        _ptr(W), out, in_, n, m, ctypes.c_float(eps), _ptr(codes), _ptr(meta), _ptr(gamma_eff),
        _ptr(workspace), _ptr(dense_dbg), _ptr(err_flag), _stream(stream)),
        "sbn_quantize_mask_pack_weights")


def sbn_quantize_mask_pack_weights_noalloc(W, n, m, eps, codes, meta, gamma_eff, dense_dbg=None,
                                           err_flag=None, stream=None):
    """Same outputs as sbn_quantize_mask_pack_weights, with no workspace argument: for
    callers that cannot provide device memory (the library uses a fixed array of its own;
    calls overlapping on the GPU race)."""
    out, in_ = W.shape
    _check(lib().sbn_quantize_mask_pack_weights_noalloc(
        _ptr(W), out, in_, n, m, ctypes.c_float(eps), _ptr(codes), _ptr(meta), _ptr(gamma_eff),
        _ptr(dense_dbg), _ptr(err_flag), _stream(stream)), "sbn_quantize_mask_pack_weights_noalloc")


def sbn_quantize_acts(X, Xq, absmax, err_flag=None, stream=None):
    tokens, in_ = X.shape
    _check(lib().sbn_quantize_acts(_ptr(X), tokens, in_, _ptr(Xq), _ptr(absmax), _ptr(err_flag),
                                   _stream(stream)), "sbn_quantize_acts")


def sbn_linear(Xq, absmax, codes, meta, gamma_eff, out, in_, n, m, Y, acc_dbg=None,
               err_flag=None, stream=None):
    tokens = Xq.shape[0]
    y_is_bf16 = 1 if Y.dtype == torch.bfloat16 else 0
    if Y.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError("Y must be float32 or bfloat16")
    _check(lib().sbn_linear(_ptr(Xq), _ptr(absmax), _ptr(codes), _ptr(meta), _ptr(gamma_eff),
                            tokens, out, in_, n, m, _ptr(Y), y_is_bf16, _ptr(acc_dbg),
                            _ptr(err_flag), _stream(stream)), "sbn_linear")


# ---- allocation helpers --------------------------------------------------------------------

class PackedWeights(NamedTuple):
    codes: torch.Tensor      # uint8 [out, codes_ld]
    meta: torch.Tensor       # uint8 [out, meta_ld]
    gamma_eff: torch.Tensor  # fp32 [1]
    out: int
    in_: int
    n: int
    m: int


def sbn_count_zero_codes(W, gamma_eff, count, stream=None):
    """Adds to count (int64 [1], caller-zeroed) the weights of W whose ternary code is 0."""
    out, in_ = W.shape
    _check(lib().sbn_count_zero_codes(_ptr(W), _ptr(gamma_eff), out, in_, _ptr(count),
                                      _stream(stream)), "sbn_count_zero_codes")


def sbn_count_mask_flips(meta_a, meta_b, out, in_, n, m, count, stream=None):
    """Adds to count (int64 [1], caller-zeroed) the positions whose keep bit differs between
    two meta planes of the same (out, in, n, m)."""
    _check(lib().sbn_count_mask_flips(_ptr(meta_a), _ptr(meta_b), out, in_, n, m, _ptr(count),
                                      _stream(stream)), "sbn_count_mask_flips")


def _alloc_stream(stream):
    """Context in which output tensors are allocated: the stream the kernel will run on,
    so that the caching allocator ties the memory to that stream (a tensor allocated on
    another stream could be handed out again while the kernel still writes it)."""
    if stream is None or not isinstance(stream, torch.cuda.Stream):
        return contextlib.nullcontext()
    return torch.cuda.stream(stream)


def new_workspace(out: int, in_: int, n: int, m: int, device="cuda") -> torch.Tensor:
    """Pack workspace (reusable by later calls on the same stream)."""
    d = sbn_linear_ref_dims(out, in_, n, m)
    return torch.zeros(d.pack_workspace_bytes, dtype=torch.uint8, device=device)


def pack_weights(W: torch.Tensor, n: int, m: int, eps: float = 1e-5,
                 workspace: Optional[torch.Tensor] = None, dense_dbg: Optional[torch.Tensor] = None,
                 err_flag: Optional[torch.Tensor] = None, stream=None) -> PackedWeights:
    out, in_ = W.shape
    d = sbn_linear_ref_dims(out, in_, n, m)
    with _alloc_stream(stream):
        codes = torch.empty((out, d.codes_ld), dtype=torch.uint8, device=W.device)
        meta = torch.empty((out, d.meta_ld), dtype=torch.uint8, device=W.device)
        gamma = torch.empty(1, dtype=torch.float32, device=W.device)
        if workspace is None:
            workspace = new_workspace(out, in_, n, m, W.device)
    sbn_quantize_mask_pack_weights(W, n, m, eps, codes, meta, gamma, workspace, dense_dbg,
                                   err_flag, stream)
    return PackedWeights(codes, meta, gamma, out, in_, n, m)


def quantize_acts(X: torch.Tensor, err_flag=None, stream=None):
    tokens, in_ = X.shape
    with _alloc_stream(stream):
        Xq = torch.empty((tokens, in_), dtype=torch.int8, device=X.device)
        s = torch.empty((tokens,), dtype=torch.float32, device=X.device)
    sbn_quantize_acts(X, Xq, s, err_flag, stream)
    return Xq, s


def linear(Xq: torch.Tensor, s: torch.Tensor, w: PackedWeights, out_dtype=torch.float32,
           acc_dbg=None, err_flag=None, stream=None) -> torch.Tensor:
    with _alloc_stream(stream):
        Y = torch.empty((Xq.shape[0], w.out), dtype=out_dtype, device=Xq.device)
    sbn_linear(Xq, s, w.codes, w.meta, w.gamma_eff, w.out, w.in_, w.n, w.m, Y, acc_dbg, err_flag,
               stream)
    return Y


_SIDE_STREAMS = {}


def count_zero_codes(W: torch.Tensor, w: "PackedWeights", stream=None) -> torch.Tensor:
    """Natural zeros of W (codes that are 0 before the mask) for the scale of its pack w;
    an int64 [1] device tensor."""
    count = torch.zeros(1, dtype=torch.int64, device=W.device)
    sbn_count_zero_codes(W, w.gamma_eff, count, stream)
    return count


def count_mask_flips(a: "PackedWeights", b: "PackedWeights", stream=None) -> torch.Tensor:
    """Positions kept by one of two packs of the same shape and pattern and pruned by the
    other; an int64 [1] device tensor."""
    if (a.out, a.in_, a.n, a.m) != (b.out, b.in_, b.n, b.m):
        raise ValueError("mask flips need two packs of the same shape and pattern")
    count = torch.zeros(1, dtype=torch.int64, device=a.meta.device)
    sbn_count_mask_flips(a.meta, b.meta, a.out, a.in_, a.n, a.m, count, stream)
    return count


def _side_stream(device: torch.device):
    """One auxiliary stream per device, for work that may overlap the weight pack."""
    key = device.index if device.index is not None else torch.cuda.current_device()
    if key not in _SIDE_STREAMS:
        _SIDE_STREAMS[key] = torch.cuda.Stream(device=key)
    return _SIDE_STREAMS[key]


def forward(X: torch.Tensor, W: torch.Tensor, n: int, m: int, eps: float = 1e-5,
            out_dtype=torch.float32, workspace=None, stream=None) -> torch.Tensor:
    """The whole Sparse-BitLinear forward: pack W, quantise X, contract and rescale.

    The activation quantiser does not depend on the weights: it runs on an auxiliary
    stream while the pack runs on `stream` (the current stream by default), and the
    contraction waits for both."""
    main = stream if stream is not None else torch.cuda.current_stream(X.device)
    side = _side_stream(X.device)
    side.wait_stream(main)  # X is ready on `main`
    with torch.cuda.stream(side):
        Xq, s = quantize_acts(X, stream=side)
    X.record_stream(side)
    w = pack_weights(W, n, m, eps, workspace=workspace, stream=main)
    main.wait_stream(side)
    Xq.record_stream(main)
    s.record_stream(main)
    return linear(Xq, s, w, out_dtype, stream=main)


# ---- grouped calls ---------------------------------------------------------------------------

def sbn_group_plan_sizes(lins):
    """(plan_bytes, workspace_bytes) for a ctypes array of SbnGroupLinear."""
    pb, wb = ctypes.c_int64(), ctypes.c_int64()
    _check(lib().sbn_group_plan_sizes(ctypes.cast(lins, ctypes.c_void_p), len(lins),
                                      ctypes.byref(pb), ctypes.byref(wb)), "sbn_group_plan_sizes")
    return pb.value, wb.value


def sbn_group_plan(lins, plan_host):
    """Fill plan_host (a 128-byte aligned uint8 CPU tensor) with the plan of `lins`."""
    _check(lib().sbn_group_plan(ctypes.cast(lins, ctypes.c_void_p), len(lins),
                                ctypes.c_void_p(plan_host.data_ptr()), plan_host.numel()),
           "sbn_group_plan")


def sbn_quantize_acts_group(plan_host, plan_dev, err_flag=None, stream=None):
    _check(lib().sbn_quantize_acts_group(ctypes.c_void_p(plan_host.data_ptr()), _ptr(plan_dev),
                                         _ptr(err_flag), _stream(stream)), "sbn_quantize_acts_group")


def sbn_linear_group(plan_host, plan_dev, workspace, err_flag=None, stream=None):
    _check(lib().sbn_linear_group(ctypes.c_void_p(plan_host.data_ptr()), _ptr(plan_dev),
                                  _ptr(workspace), _ptr(err_flag), _stream(stream)),
           "sbn_linear_group")


class GroupPlan:
    """A grouped call over many 2:4 layers of at most 32 tokens each: the plan (host and
    device copies) and the zeroed workspace.  `layers` is a list of dicts with the torch
    tensors X (bf16 [T, K], may be None), Xq (int8 [T, K]), s (fp32 [T]), w (PackedWeights),
    Y (fp32 or bf16 [T, O]) and optionally acc_dbg (int32 [T, O]).  The tensors must stay
    alive and in place while the plan is used."""

    def __init__(self, layers, device=None, _arr=None):
        self.layers = layers
        if _arr is None:
            arr = (SbnGroupLinear * len(layers))()
            for i, L in enumerate(layers):
                w = L["w"]
                Y = L["Y"]
                arr[i] = SbnGroupLinear(
                    X=_ptr(L.get("X")), Xq=_ptr(L["Xq"]), absmax=_ptr(L["s"]),
                    codes=_ptr(w.codes), meta=_ptr(w.meta), gamma_eff=_ptr(w.gamma_eff),
                    Y=_ptr(Y), acc_dbg=_ptr(L.get("acc_dbg")), tokens=L["Xq"].shape[0],
                    out=w.out, in_=w.in_, n=w.n, m=w.m,
                    y_is_bf16=1 if Y.dtype == torch.bfloat16 else 0, reserved=0, ldx=0, ldc=0,
                    ldm=0)
            _arr = arr
        arr = self._arr = _arr
        pb, wb = sbn_group_plan_sizes(arr)
        # 128-byte aligned host buffer
        raw = torch.empty(pb + 128, dtype=torch.uint8)
        off = (-raw.data_ptr()) % 128
        self.plan_host = raw[off:off + pb]
        self._raw = raw
        sbn_group_plan(arr, self.plan_host)
        device = device if device is not None else layers[0]["Xq"].device
        self.plan_dev = self.plan_host.to(device)
        self.workspace = torch.zeros(max(wb, 256), dtype=torch.uint8, device=device)
        self.workspace_bytes = wb
        hdr = self.plan_host[:48].numpy().view("int32")
        self.nunits, self.ncta, self.bn, self.nrows, self.split = (int(hdr[3]), int(hdr[4]),
                                                                   int(hdr[5]), int(hdr[6]),
                                                                   int(hdr[9]))

    def quantize_acts(self, err_flag=None, stream=None):
        sbn_quantize_acts_group(self.plan_host, self.plan_dev, err_flag, stream)

    def linear(self, err_flag=None, stream=None):
        sbn_linear_group(self.plan_host, self.plan_dev, self.workspace, err_flag, stream)


def sbn_gq_sum(part, n, G, Y, stream=None):
    """Y[i] = sum over j of part[j * n + i] in j order (fp32 adds), fp32 or bf16 Y."""
    _check(lib().sbn_gq_sum(_ptr(part), n, G, _ptr(Y), 1 if Y.dtype == torch.bfloat16 else 0,
                            _stream(stream)), "sbn_gq_sum")


class GqGroupPlan:
    """The decode step of many group-quantised 2:4 layers (each packed by pack_weights_gq
    with its own G) in three launches: the grouped quantiser (per-(token, group) scales,
    each block of a layer being a K slice of a grouped call), the grouped contraction (each
    block's y_j = fp32(acc_j * c_tj) into a partial buffer) and the ordered sum over the
    blocks.  All layers share one G.  `layers`: dicts with X (bf16 [T, K], T <= 32) and w
    (GqPackedWeights).  Allocates Xq, s ([G, T] per layer), the partials and Y (fp32 or
    bf16; layer i's output is ``self.Y[i]``)."""

    def __init__(self, layers, out_dtype=torch.float32, device=None):
        G = layers[0]["w"].groups
        if any(L["w"].groups != G for L in layers):
            raise ValueError("the layers of a GqGroupPlan share one G")
        device = device if device is not None else layers[0]["X"].device
        self.G = G
        # each layer's outputs start on a 16-byte boundary (the grouped call's rule for Y)
        ns = [-(-L["X"].shape[0] * L["w"].out // 8) * 8 for L in layers]
        self.n = sum(ns)
        self.part = torch.zeros((G, max(self.n, 8)), dtype=torch.float32, device=device)
        self.Yflat = torch.zeros(max(self.n, 8), dtype=out_dtype, device=device)
        self.Xq, self.s, self.Y, slices = [], [], [], []
        arr = (SbnGroupLinear * (G * len(layers)))()
        off = 0
        for i, L in enumerate(layers):
            X, w = L["X"], L["w"]
            T, K = X.shape
            if not X.is_cuda or not X.is_contiguous():
                raise ValueError("X: a contiguous CUDA tensor")
            kg = K // G
            Xq = torch.empty((T, K), dtype=torch.int8, device=device)
            s = torch.empty((G, T), dtype=torch.float32, device=device)
            self.Xq.append(Xq)
            self.s.append(s)
            self.Y.append(self.Yflat[off:off + T * w.out].view(T, w.out))
            for j in range(G):
                arr[i * G + j] = SbnGroupLinear(
                    X=X.data_ptr() + 2 * j * kg, Xq=Xq.data_ptr() + j * kg,
                    absmax=s.data_ptr() + 4 * j * T, codes=w.codes.data_ptr() + j * (kg // 8),
                    meta=w.meta.data_ptr() + j * (kg // 8), gamma_eff=w.gamma_eff.data_ptr() + 4 * j,
                    Y=self.part.data_ptr() + 4 * (j * self.part.shape[1] + off), acc_dbg=None,
                    tokens=T, out=w.out, in_=kg, n=w.n, m=w.m, y_is_bf16=0, reserved=0, ldx=K,
                    ldc=w.codes.shape[1], ldm=w.meta.shape[1])
            off += ns[i]
        self.layers = layers
        self.plan = GroupPlan([], device=device, _arr=arr) if len(layers) else None

    def quantize_acts(self, err_flag=None, stream=None):
        self.plan.quantize_acts(err_flag, stream)

    def linear(self, err_flag=None, stream=None):
        self.plan.linear(err_flag, stream)
        if self.n:
            sbn_gq_sum(self.part, self.part.shape[1], self.G, self.Yflat, stream)


# ---- grouped pack (many tensors, 6:8 and/or 2:4) -----------------------------------------

def sbn_pack_group_sizes(tensors):
    """(plan_bytes, workspace_bytes) for a ctypes array of SbnPackGroupTensor."""
    pb, wb = ctypes.c_int64(), ctypes.c_int64()
    _check(lib().sbn_pack_group_sizes(ctypes.cast(tensors, ctypes.c_void_p), len(tensors),
                                      ctypes.byref(pb), ctypes.byref(wb)), "sbn_pack_group_sizes")
    return pb.value, wb.value


def sbn_pack_group_plan(tensors, plan_host):
    """Fill plan_host (a 16-byte aligned uint8 CPU tensor) with the plan of `tensors`."""
    _check(lib().sbn_pack_group_plan(ctypes.cast(tensors, ctypes.c_void_p), len(tensors),
                                     ctypes.c_void_p(plan_host.data_ptr()), plan_host.numel()),
           "sbn_pack_group_plan")


def sbn_quantize_mask_pack_weights_group(plan_host, plan_dev, workspace, err_flag=None,
                                         stream=None):
    _check(lib().sbn_quantize_mask_pack_weights_group(
        ctypes.c_void_p(plan_host.data_ptr()), _ptr(plan_dev), _ptr(workspace), _ptr(err_flag),
        _stream(stream)), "sbn_quantize_mask_pack_weights_group")


class PackGroup:
    """A grouped pack: every master tensor of `Ws` (bf16 [O, K] CUDA tensors) into each
    pattern of `patterns` (one or two of (6, 8) and (2, 4)), in two launches per call.
    Allocates the outputs: ``packed[i][j]`` is tensor i's PackedWeights for patterns[j]
    (both patterns share one gamma_eff).  ``dense_dbg`` optionally gives, per tensor, a
    list of int8 [O, K] tensors (or None) per pattern.  The masters may change between
    calls (in place); the plan keeps their pointers."""

    def __init__(self, Ws, patterns=((6, 8), (2, 4)), eps=1e-5, dense_dbg=None, device=None):
        if len(patterns) not in (1, 2):
            raise ValueError("one or two patterns")
        device = device if device is not None else Ws[0].device
        self.Ws, self.patterns, self.packed = list(Ws), tuple(patterns), []
        arr = (SbnPackGroupTensor * len(self.Ws))()
        for i, W in enumerate(self.Ws):
            out, in_ = W.shape
            gamma = torch.empty(1, dtype=torch.float32, device=device)
            pw = []
            for (n, m) in self.patterns:
                d = sbn_linear_ref_dims(out, in_, n, m)
                pw.append(PackedWeights(
                    torch.empty((out, d.codes_ld), dtype=torch.uint8, device=device),
                    torch.empty((out, d.meta_ld), dtype=torch.uint8, device=device),
                    gamma, out, in_, n, m))
            self.packed.append(pw)
            dd = (dense_dbg[i] if dense_dbg is not None else None) or [None, None]
            two = len(pw) == 2
            arr[i] = SbnPackGroupTensor(
                W=_ptr(W), codes=_ptr(pw[0].codes), meta=_ptr(pw[0].meta),
                codes2=_ptr(pw[1].codes) if two else None, meta2=_ptr(pw[1].meta) if two else None,
                gamma_eff=_ptr(gamma), dense_dbg=_ptr(dd[0]),
                dense_dbg2=_ptr(dd[1]) if two and len(dd) > 1 else None, out=out, in_=in_,
                n=self.patterns[0][0], m=self.patterns[0][1],
                n2=self.patterns[1][0] if two else 0, m2=self.patterns[1][1] if two else 0,
                eps=eps, reserved=0)
        self._arr = arr
        pb, wb = sbn_pack_group_sizes(arr)
        raw = torch.empty(pb + 16, dtype=torch.uint8)
        off = (-raw.data_ptr()) % 16
        self.plan_host = raw[off:off + pb]
        self._raw = raw
        sbn_pack_group_plan(arr, self.plan_host)
        self.plan_dev = self.plan_host.to(device)
        self.workspace = torch.zeros(max(wb, 16), dtype=torch.uint8, device=device)
        hdr = self.plan_host[:20].numpy().view("int32")
        self.total_chunks, self.total_q = int(hdr[2]) & 0xffffffff, int(hdr[3]) & 0xffffffff
        self.mode = int(hdr[4])  # 0 / 1 / 2: the fixed-pattern kernel; -1: the general one

    def run(self, err_flag=None, stream=None):
        sbn_quantize_mask_pack_weights_group(self.plan_host, self.plan_dev, self.workspace,
                                             err_flag, stream)


# ---- tensor-core operand (2:4, many tokens) ----------------------------------------------

def sbn_operand_bytes(out, in_, n, m):
    b = ctypes.c_int64()
    _check(lib().sbn_operand_bytes(out, in_, n, m, ctypes.byref(b)), "sbn_operand_bytes")
    return b.value


def sbn_expand_operand(codes, meta, out, in_, n, m, operand, stream=None):
    _check(lib().sbn_expand_operand(_ptr(codes), _ptr(meta), out, in_, n, m, _ptr(operand),
                                    _stream(stream)), "sbn_expand_operand")


def sbn_linear_operand(Xq, absmax, operand, gamma_eff, out, in_, n, m, Y, acc_dbg=None,
                       err_flag=None, stream=None):
    if Y.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError("Y must be float32 or bfloat16")
    _check(lib().sbn_linear_operand(_ptr(Xq), _ptr(absmax), _ptr(operand), _ptr(gamma_eff),
                                    Xq.shape[0], out, in_, n, m, _ptr(Y),
                                    1 if Y.dtype == torch.bfloat16 else 0, _ptr(acc_dbg),
                                    _ptr(err_flag), _stream(stream)), "sbn_linear_operand")


def expand_operand(w: PackedWeights, stream=None) -> torch.Tensor:
    """The tensor-core operand of a 2:4 pack (uint8 device tensor)."""
    with _alloc_stream(stream):
        op = torch.empty(sbn_operand_bytes(w.out, w.in_, w.n, w.m), dtype=torch.uint8,
                         device=w.codes.device)
    sbn_expand_operand(w.codes, w.meta, w.out, w.in_, w.n, w.m, op, stream)
    return op


def linear_operand(Xq, s, w: PackedWeights, operand, out_dtype=torch.float32, acc_dbg=None,
                   err_flag=None, stream=None) -> torch.Tensor:
    with _alloc_stream(stream):
        Y = torch.empty((Xq.shape[0], w.out), dtype=out_dtype, device=Xq.device)
    sbn_linear_operand(Xq, s, operand, w.gamma_eff, w.out, w.in_, w.n, w.m, Y, acc_dbg, err_flag,
                       stream)
    return Y


# ---- dual-STE backward ---------------------------------------------------------------------

def sbn_backward_workspace_bytes(tokens, out, in_):
    b = ctypes.c_int64()
    _check(lib().sbn_backward_workspace_bytes(tokens, out, in_, ctypes.byref(b)),
           "sbn_backward_workspace_bytes")
    return b.value


def sbn_backward(dY, Xq, absmax, codes, meta, W, gamma_eff, out, in_, n, m, dX, dW, workspace,
                 err_flag=None, stream=None):
    _check(lib().sbn_backward(_ptr(dY), _ptr(Xq), _ptr(absmax), _ptr(codes), _ptr(meta), _ptr(W),
                              _ptr(gamma_eff), dY.shape[0], out, in_, n, m, _ptr(dX), _ptr(dW),
                              _ptr(workspace), _ptr(err_flag), _stream(stream)), "sbn_backward")


def backward(dY: torch.Tensor, Xq: torch.Tensor, s: torch.Tensor, w: PackedWeights,
             W: torch.Tensor, need_dX=True, need_dW=True, err_flag=None, stream=None):
    """(dX fp32 [T, in] or None, dW fp32 [out, in] or None) for the upstream gradient dY
    (bf16 [T, out]) of the forward that used Xq, s and the pack w of the masters W."""
    T = dY.shape[0]
    with _alloc_stream(stream):
        dX = torch.empty((T, w.in_), dtype=torch.float32, device=dY.device) if need_dX else None
        dW = torch.empty((w.out, w.in_), dtype=torch.float32, device=dY.device) if need_dW else None
        ws = torch.empty(max(256, sbn_backward_workspace_bytes(T, w.out, w.in_)), dtype=torch.uint8,
                         device=dY.device)
    sbn_backward(dY, Xq, s, w.codes, w.meta, W, w.gamma_eff, w.out, w.in_, w.n, w.m, dX, dW, ws,
                 err_flag, stream)
    return dX, dW


# ---- steps 5-7 in one call -------------------------------------------------------------------

def sbn_quantize_linear(X, codes, meta, gamma_eff, out, in_, n, m, Xq, absmax, Y, acc_dbg=None,
                        err_flag=None, stream=None):
    if Y.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError("Y must be float32 or bfloat16")
    _check(lib().sbn_quantize_linear(_ptr(X), _ptr(codes), _ptr(meta), _ptr(gamma_eff),
                                     X.shape[0], out, in_, n, m, _ptr(Xq), _ptr(absmax), _ptr(Y),
                                     1 if Y.dtype == torch.bfloat16 else 0, _ptr(acc_dbg),
                                     _ptr(err_flag), _stream(stream)), "sbn_quantize_linear")


def quantize_linear(X: torch.Tensor, w: PackedWeights, out_dtype=torch.float32, acc_dbg=None,
                    err_flag=None, stream=None):
    """Steps 5-7 (activation quantiser + contraction) in one call; (Y, Xq, s)."""
    T, K = X.shape
    with _alloc_stream(stream):
        Xq = torch.empty((T, K), dtype=torch.int8, device=X.device)
        s = torch.empty((T,), dtype=torch.float32, device=X.device)
        Y = torch.empty((T, w.out), dtype=out_dtype, device=X.device)
    sbn_quantize_linear(X, w.codes, w.meta, w.gamma_eff, w.out, w.in_, w.n, w.m, Xq, s, Y, acc_dbg,
                        err_flag, stream)
    return Y, Xq, s


# ---- group quantisation (G blocks along K) ---------------------------------------------------

class GqPackedWeights(NamedTuple):
    codes: torch.Tensor      # uint8 [out, codes_ld]
    meta: torch.Tensor       # uint8 [out, meta_ld]
    gamma_eff: torch.Tensor  # fp32 [groups]
    out: int
    in_: int
    n: int
    m: int
    groups: int


def pack_weights_gq(W, n, m, groups, eps=1e-5, dense_dbg=None, err_flag=None, stream=None):
    out, in_ = W.shape
    d = sbn_linear_ref_dims(out, in_, n, m)
    with _alloc_stream(stream):
        codes = torch.empty((out, d.codes_ld), dtype=torch.uint8, device=W.device)
        meta = torch.empty((out, d.meta_ld), dtype=torch.uint8, device=W.device)
        gamma = torch.empty(groups, dtype=torch.float32, device=W.device)
        ws = new_workspace(out, in_, n, m, W.device)
    _check(lib().sbn_quantize_mask_pack_weights_gq(
        _ptr(W), out, in_, n, m, groups, ctypes.c_float(eps), _ptr(codes), _ptr(meta), _ptr(gamma),
        _ptr(ws), _ptr(dense_dbg), _ptr(err_flag), _stream(stream)),
        "sbn_quantize_mask_pack_weights_gq")
    return GqPackedWeights(codes, meta, gamma, out, in_, n, m, groups)


def sbn_quantize_acts_gq(X, groups, Xq, absmax, err_flag=None, stream=None):
    T, K = X.shape
    _check(lib().sbn_quantize_acts_gq(_ptr(X), T, K, groups, _ptr(Xq), _ptr(absmax), _ptr(err_flag),
                                      _stream(stream)), "sbn_quantize_acts_gq")


def sbn_gq_workspace_bytes(tokens, out, in_, groups):
    b = ctypes.c_int64()
    _check(lib().sbn_gq_workspace_bytes(tokens, out, in_, groups, ctypes.byref(b)),
           "sbn_gq_workspace_bytes")
    return b.value


def sbn_linear_gq(Xq, absmax, codes, meta, gamma_eff, out, in_, n, m, groups, Y, workspace,
                  acc_dbg=None, err_flag=None, stream=None):
    if Y.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError("Y must be float32 or bfloat16")
    _check(lib().sbn_linear_gq(_ptr(Xq), _ptr(absmax), _ptr(codes), _ptr(meta), _ptr(gamma_eff),
                               Xq.shape[0], out, in_, n, m, groups, _ptr(Y),
                               1 if Y.dtype == torch.bfloat16 else 0, _ptr(workspace),
                               _ptr(acc_dbg), _ptr(err_flag), _stream(stream)), "sbn_linear_gq")


def quantize_acts_gq(X, groups, err_flag=None, stream=None):
    """(Xq int8 [T, K], s fp32 [groups, T])."""
    T, K = X.shape
    with _alloc_stream(stream):
        Xq = torch.empty((T, K), dtype=torch.int8, device=X.device)
        s = torch.empty((groups, T), dtype=torch.float32, device=X.device)
    sbn_quantize_acts_gq(X, groups, Xq, s, err_flag, stream)
    return Xq, s


def linear_gq(Xq, s, w: GqPackedWeights, out_dtype=torch.float32, acc_dbg=None, err_flag=None,
              stream=None):
    T = Xq.shape[0]
    with _alloc_stream(stream):
        Y = torch.empty((T, w.out), dtype=out_dtype, device=Xq.device)
        ws = torch.empty(max(sbn_gq_workspace_bytes(T, w.out, w.in_, w.groups), 16),
                         dtype=torch.uint8, device=Xq.device)
    sbn_linear_gq(Xq, s, w.codes, w.meta, w.gamma_eff, w.out, w.in_, w.n, w.m, w.groups, Y, ws,
                  acc_dbg, err_flag, stream)
    return Y
