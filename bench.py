"""Benchmark of the Sparse-BitLinear forward hot path on B200.

Default workload: the largest single-GPU configuration, a 32-layer decoder stack of
pre-packed 2:4 Sparse-BitLinear layers (hidden 4096, FFN 11008: QKV 4096->12288, O
4096->4096, gate and up 4096->11008, down 11008->4096; 160 layers, 6.48 G weights).
One step is the decode step of the whole stack at 16 tokens: the activation quantiser
(step 5) and the contraction with rescale (steps 6-7) of all 160 layers, each as one
grouped launch through the C ABI (sbn_quantize_acts_group, sbn_linear_group).  The
weights are packed once before timing, as a server does when it loads a model.

The same JSON line carries sub-records: the stack's 4096-token prefill (per-layer tensor-
core contraction, TOPS), and the single-tensor configurations -- decode GEMV (W 6912x2560
6:8, pack + act quant + GEMV per step), prefill GEMM (W 11008x4096 2:4, 2048 tokens) and
the training-step weight path (re-pack all 130 linears of a 26-layer decoder in 6:8 and
2:4).  Each has its own roofline and its own oracle leg.

Timing: W untimed warm-up steps, then exactly K steps captured in one CUDA graph and
replayed between a barrier + synchronize on both sides; the device time is the max over
ranks.  The stack's packed weights (1.62 GB) and the rotating input sets of the single-
tensor configurations exceed the 126 MB L2, so every step reads its weights from HBM.
Per-call durations come from a second graph of the same steps with CUDA events recorded
around every C-ABI call on the streams the calls run on.  nvidia-smi clocks are sampled
during the timed region.

`--impl reference` times the CPU oracle (test infrastructure) on a bounded sample of the
same workload instead.  `--gpus N` without torchrun relaunches itself under torchrun with
N local ranks; each rank runs its own replica of the workload on its own seeded inputs
(weak scaling, no collective in the data path).
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402
from sparse_linear_layers_absmean_b200 import dist  # noqa: E402

METRIC = "Sparse-BitLinear TOPS & packed-weight GB/s vs roofline; quant+mask GB/s"
L2_BYTES = 126 * 1024 * 1024
WORKLOADS = ("stack", "decode", "prefill", "train-step", "stack-prefill")


# ---- peaks, clocks -------------------------------------------------------------------------

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"],
                    bf16_sustained=d.get("bf16_tflops_sustained"), source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


def peak_source(peaks, key, value, what=""):
    """Where a roofline denominator came from: the measured-peaks file beside this script,
    or (when it is absent) an earlier measurement on B200s of the same kind."""
    if peaks["source"] == "measured":
        return f"{what}{key} of MEASURED_PEAKS.json: of measured"
    return (f"{what}{key} = {value} (MEASURED_PEAKS.json absent; an earlier measurement on "
            "B200): of fallback")


def hbm_roof(achieved, peaks, kernel, traffic=None, unit_note=""):
    return {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm"], "unit": "GB/s",
            "frac": achieved / peaks["hbm"], "traffic": traffic, "kernel": kernel,
            "peak_source": peak_source(peaks, "hbm_gbs", peaks["hbm"]) + unit_note}


def tensor_roof(achieved, peaks, kernel, traffic=None):
    # int8 dense tensor peak = 2 x the measured bf16 burst peak (the nominal int8/bf16 ratio
    # is 2); the burst figure because each contraction is timed per call, ~0.1 ms long
    peak = 2.0 * peaks["bf16"]
    return {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
            "frac": achieved / peak, "traffic": traffic, "kernel": kernel,
            "peak_source": peak_source(peaks, "bf16_tflops", peaks["bf16"], "2 x burst ")
                           + "; kept int8 ops"}


class ClockSampler:
    """Samples nvidia-smi clocks and throttle reasons while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm)}


def load_traffic(workload, call):
    """DRAM bytes per launch of a call from the committed ncu summary, if any."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    return d.get(workload, {}).get(call)


# ---- timing harness -----------------------------------------------------------------------

class Timer:
    """Captures `steps` steps in one CUDA graph and times its replay (barrier + synchronize
    on both sides, max over ranks), and a second graph of the same steps with external
    events around every call for the per-call durations."""

    def __init__(self, dev, local):
        self.dev, self.local = dev, local
        self.stream = torch.cuda.Stream(device=dev)

    def run(self, step, steps, warmup, calls=(), sample_clocks=True):
        """step(i, ev) runs step i; ev is None or a dict call -> (start, end) events to record
        around each call on the stream it runs on.  Returns (ms per step, per-call ms, clocks)."""
        with torch.cuda.stream(self.stream):
            for i in range(warmup):
                step(i, None)
        torch.cuda.synchronize(self.dev)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=self.stream):
            for i in range(steps):
                step(i, None)
        evs = [{c: (torch.cuda.Event(enable_timing=True, external=True),
                    torch.cuda.Event(enable_timing=True, external=True)) for c in calls}
               for _ in range(steps)]
        g_ev = None
        if calls:
            g_ev = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g_ev, stream=self.stream):
                for i in range(steps):
                    step(i, evs[i])
        with torch.cuda.stream(self.stream):
            g.replay()  # graph warm-up
        torch.cuda.synchronize(self.dev)
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        clk = ClockSampler(self.local) if sample_clocks else None
        if clk:
            clk.__enter__()
        try:
            dist.barrier(self.dev)
            with torch.cuda.stream(self.stream):
                t0.record()
                g.replay()
                t1.record()
            torch.cuda.synchronize(self.dev)
            dist.barrier(self.dev)
            ms = t0.elapsed_time(t1)
            # the per-call durations right after the timed steps, in the same thermal and
            # clock state (and inside the clock sampling)
            if g_ev is not None:
                with torch.cuda.stream(self.stream):
                    g_ev.replay()
                torch.cuda.synchronize(self.dev)
            if clk and ms < 300:  # keep the clocks sampled for at least ~0.3 s of load
                with torch.cuda.stream(self.stream):
                    for _ in range(max(1, int(300 / max(ms, 1e-3)))):
                        g.replay()
                torch.cuda.synchronize(self.dev)
        finally:
            if clk:
                clk.__exit__()
        per = {}
        if g_ev is not None:
            for c in calls:
                per[c] = sum(e[c][0].elapsed_time(e[c][1]) for e in evs) / steps
        del g, g_ev
        ms = dist.max_over_ranks(ms, self.dev)
        return ms / steps, per, (clk.summary() if clk else None)


# ---- the stack (configuration 5) ----------------------------------------------------------

STACK_LAYERS = workloads.STACK_LAYERS  # --stack-layers (profiling captures of a smaller stack)


def stack_layers(rank=0):
    """(index, name, O, K, tensor id) of the 160 layers of one replica of the stack; rank r
    draws its replica's weights and activations from tensor ids offset by 1000 r."""
    out = []
    for layer in range(STACK_LAYERS):
        for i, (name, O, K) in enumerate(workloads.STACK_LAYER_SHAPES):
            out.append((5 * layer + i, name, O, K, 5 * layer + i + 1000 * rank))
    return out


def build_stack(sbn, dev, rank, err):
    """Packs the 160 layers of the stack (2:4) on the GPU from seeded masters."""
    packed = []
    for idx, name, O, K, tid in stack_layers(rank):
        W = workloads.masters_device(O, K, device=dev, config=5, tensor=tid)
        packed.append(sbn.pack_weights(W, 2, 4, err_flag=err))
        del W
    return packed


def bench_stack_decode(args, sbn, dev, local, rank, world, peaks, timer, packed, err):
    T = workloads.STACK_DECODE_T
    lay = stack_layers(rank)
    # per-layer Student-t(4) activations, drawn on the host (seeded), one buffer each
    Xh = [workloads.torch_bf16(workloads.student_t(T, K, config=5, tensor=10000 + tid))
          for _, _, O, K, tid in lay]
    # every layer's X and Y are views of one device buffer each (offsets stay 16-byte
    # aligned: T K bf16 and T O fp32 with K, O multiples of 8), so that a step's inputs and
    # outputs cross PCIe as one copy each way
    nx = [T * K for _, _, _, K, _ in lay]
    ny = [T * O for _, _, O, _, _ in lay]
    Xall = torch.empty(sum(nx), dtype=torch.bfloat16, device=dev)
    Yall = torch.empty(sum(ny), dtype=torch.float32, device=dev)
    layers = []
    ox = oy = 0
    for (idx, name, O, K, tid), w, x, a, b in zip(lay, packed, Xh, nx, ny):
        X = Xall[ox:ox + a].view(T, K)
        X.copy_(x)
        layers.append(dict(X=X, Xq=torch.empty((T, K), dtype=torch.int8, device=dev),
                           s=torch.empty((T,), dtype=torch.float32, device=dev), w=w,
                           Y=Yall[oy:oy + b].view(T, O)))
        ox += a
        oy += b
    plan = sbn.GroupPlan(layers, device=dev)
    st = timer.stream

    def step(i, ev):
        if ev is not None:
            ev["act"][0].record(st)
        plan.quantize_acts(err, st)
        if ev is not None:
            ev["act"][1].record(st)
            ev["linear"][0].record(st)
        plan.linear(err, st)
        if ev is not None:
            ev["linear"][1].record(st)

    ms, per, clocks = timer.run(step, args.steps, args.warmup, calls=("act", "linear"))
    weights = sum(O * K for _, _, O, K, _ in lay)
    packed_b = weights // 4  # 2:4: K/8 code bytes + K/8 metadata bytes per row
    act_b = sum(2 * T * K + T * K + 4 * T for _, _, _, K, _ in lay)   # read X, write Xq, s
    lin_b = packed_b + sum(T * K + 4 * T + 4 * T * O for _, _, O, K, _ in lay)  # + read Xq, write Y
    total = act_b + lin_b
    roof = hbm_roof(packed_b / (per["linear"] * 1e-3) / 1e9, peaks,
                    "k_gemm_group (grouped 2:4 contraction, 160 layers, one launch)",
                    traffic=load_traffic("stack-decode", "linear"),
                    unit_note="; achieved on packed-weight bytes (0.25 B per weight)")
    rec = {
        "value": total * world / (ms * 1e-3) / 1e9, "unit": "GB/s", "ms_per_step": ms,
        "roofline": roof,
        "kernels": {
            "act_quant_group": {"ms": per["act"], "GB/s": act_b / (per["act"] * 1e-3) / 1e9,
                                "launches": 1},
            "linear_group": {"ms": per["linear"],
                             "packed_weight_GB/s": packed_b / (per["linear"] * 1e-3) / 1e9,
                             "all_bytes_GB/s": lin_b / (per["linear"] * 1e-3) / 1e9,
                             "TOPS": weights * T / (per["linear"] * 1e-3) / 1e12,
                             "launches": 1, "units": plan.nunits, "ctas": plan.ncta,
                             "split": plan.split}},
        "gpu_launches": 2 * args.steps, "clocks": clocks,
        "bytes_per_step": {"packed_weights": packed_b, "act_quant": act_b, "contraction": lin_b},
    }
    # e2e through the public API (GroupPlan) with pinned host buffers: every step copies its
    # 160 activation blocks in and its 160 outputs out and waits for them on the host.  The
    # stack runs as four plans of 40 layers (8 decoder layers) on three streams, so that a
    # chunk's output copy overlaps the next chunk's input copy and contraction (the two copy
    # directions use separate copy engines); every chunk crosses PCIe as one copy each way.
    hostX = torch.cat([x.flatten() for x in Xh]).pin_memory()
    hostY = torch.empty(Yall.shape, dtype=torch.float32).pin_memory()
    ke = min(args.steps, 20)
    nch = 4
    per_ch = (len(layers) + nch - 1) // nch
    chunks = []
    for c in range(0, len(layers), per_ch):
        sub = layers[c:c + per_ch]
        x0, y0 = sum(nx[:c]), sum(ny[:c])
        x1, y1 = x0 + sum(nx[c:c + per_ch]), y0 + sum(ny[c:c + per_ch])
        chunks.append((sbn.GroupPlan(sub, device=dev), slice(x0, x1), slice(y0, y1)))
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev_in = [torch.cuda.Event() for _ in chunks]
    ev_done = [torch.cuda.Event() for _ in chunks]

    def e2e_step():
        for (pl, xs, ys), ei, ed in zip(chunks, ev_in, ev_done):
            with torch.cuda.stream(s_in):
                Xall[xs].copy_(hostX[xs], non_blocking=True)
                ei.record(s_in)
            st.wait_event(ei)
            pl.quantize_acts(err, st)
            pl.linear(err, st)
            ed.record(st)
            s_out.wait_event(ed)
            with torch.cuda.stream(s_out):
                hostY[ys].copy_(Yall[ys], non_blocking=True)
        s_out.synchronize()  # every chunk's output copy waited for every earlier stage

    with torch.cuda.stream(st):
        for _ in range(3):
            e2e_step()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(s_in)
        for _ in range(ke):
            e2e_step()
        b.record(s_out)
    torch.cuda.synchronize(dev)
    e2e_ms = dist.max_over_ranks(a.elapsed_time(b) / ke, dev)
    # the outputs that crossed PCIe are the device's outputs, bit for bit
    e2e_same = bool(torch.equal(hostY, Yall.cpu()))
    h2d = sum(x.numel() * 2 for x in Xh)
    d2h = sum(L["Y"].numel() * 4 for L in layers)
    rec["e2e"] = {"value": total * world / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s",
                  "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                  "outputs_match_device": e2e_same,
                  "api": "GroupPlan.quantize_acts + GroupPlan.linear (sbn_quantize_acts_group, "
                         "sbn_linear_group) as 4 plans of 40 layers; weights resident, X in / Y "
                         "out over PCIe, one copy each way per plan, overlapped with the other "
                         "plans' contraction on three streams"}
    rec["config"] = {"workload": "stack-decode-32x4096-t16-2of4", "layers": len(lay),
                     "weights": weights, "packed_bytes": packed_b, "tokens": T,
                     "pattern": "2:4",
                     "step": "grouped act quant (S5) + grouped contraction/rescale (S6-S7) of "
                             "all 160 pre-packed layers",
                     "l2": "1.62 GB of packed weights per step > 126 MB L2",
                     "parallelism": f"replicas x{world} (one stack per GPU, own inputs)"}
    return rec, Xh, layers


def bench_stack_prefill(args, sbn, dev, local, rank, world, peaks, timer, packed, err):
    T = workloads.STACK_PREFILL_T
    lay = stack_layers(rank)
    Ks = sorted({K for _, _, _, K, _ in lay})
    Os = sorted({O for _, _, O, _, _ in lay})
    # Student-t(4) activations (seeded, host), one input per distinct K shared by its layers
    X = {K: workloads.torch_bf16(workloads.student_t(T, K, config=5, tensor=30000 + K + 1000 * rank),
                                 dev) for K in Ks}
    Xq = {K: torch.empty((T, K), dtype=torch.int8, device=dev) for K in Ks}
    sc = {K: torch.empty((T,), dtype=torch.float32, device=dev) for K in Ks}
    Y = {O: torch.empty((T, O), dtype=torch.float32, device=dev) for O in Os}
    st = timer.stream
    steps = min(args.steps, 10)

    def step(i, ev):
        for j, ((_, _, O, K, _), w) in enumerate(zip(lay, packed)):
            sbn.sbn_quantize_acts(X[K], Xq[K], sc[K], err, st)
            if ev is not None and j == 0:
                ev["linear"][0].record(st)
            sbn.sbn_linear(Xq[K], sc[K], w.codes, w.meta, w.gamma_eff, O, K, 2, 4, Y[O], None,
                           err, st)
            if ev is not None and j == 0:
                ev["linear"][1].record(st)

    ms, per, clocks = timer.run(step, steps, min(args.warmup, 3), calls=("linear",))
    weights = sum(O * K for _, _, O, K, _ in lay)
    ops = T * weights  # 2 x kept MACs = 2 T O K / 2
    qkv_ops = T * lay[0][2] * lay[0][3]
    return {"value": ops * world / (ms * 1e-3) / 1e12, "unit": "TOPS", "ms_per_step": ms,
            "steps": steps,
            "roofline": tensor_roof(qkv_ops / (per["linear"] * 1e-3) / 1e12, peaks,
                                    "k_gemm_sp24_pair<208> (QKV 12288x4096, 4096 tokens, per call)"),
            "whole_step_frac_of_int8_peak": ops / (ms * 1e-3) / 1e12 / (2.0 * peaks["bf16"]),
            "gpu_launches": 2 * len(lay) * steps, "clocks": clocks,
            "config": {"workload": "stack-prefill-32x4096-t4096-2of4", "tokens": T,
                       "kept_ops": ops, "step": "per layer: act quant + tensor-core contraction"}}


# ---- single-tensor configurations (2, 3) -------------------------------------------------

def step_accounting(cfg):
    O, K, T, n, m = cfg["O"], cfg["K"], cfg["T"], cfg["n"], cfg["m"]
    stored = K // 2 if (n, m) == (2, 4) else K
    codes_b, meta_b = O * (stored // 4), O * (K // 8)
    linear_w = codes_b + (meta_b if (n, m) == (2, 4) else 0)
    pack = 2 * O * K + codes_b + meta_b
    act = 2 * T * K + T * K + 4 * T
    linear = linear_w + T * K + 4 * T + 4 * T * O
    return dict(pack=pack, act=act, linear=linear, linear_weight=linear_w,
                ops=2 * T * O * K * n // m, total=pack + act + linear)


def bench_single(args, sbn, dev, local, rank, world, peaks, timer, cfg, err):
    O, K, T, n, m = cfg["O"], cfg["K"], cfg["T"], cfg["n"], cfg["m"]
    acct = step_accounting(cfg)
    set_bytes = 2 * O * K + 2 * T * K
    R = min(64, max(2, -(-2 * L2_BYTES // set_bytes))) if set_bytes < 2 * L2_BYTES else 1
    sets = []
    d = sbn.sbn_linear_ref_dims(O, K, n, m)
    for r in range(R):
        Wb = workloads.masters(O, K, seed=0, config=1, tensor=2 * (r + R * rank))
        Xb = workloads.activations(T, K, seed=0, config=1, tensor=2 * (r + R * rank) + 1)
        sets.append(dict(
            W=workloads.torch_bf16(Wb, dev), X=workloads.torch_bf16(Xb, dev),
            codes=torch.empty((O, d.codes_ld), dtype=torch.uint8, device=dev),
            meta=torch.empty((O, d.meta_ld), dtype=torch.uint8, device=dev),
            g=torch.empty(1, dtype=torch.float32, device=dev),
            Xq=torch.empty((T, K), dtype=torch.int8, device=dev),
            s=torch.empty((T,), dtype=torch.float32, device=dev),
            Y=torch.empty((T, O), dtype=torch.float32, device=dev)))
    ws = sbn.new_workspace(O, K, n, m, dev)
    main = timer.stream
    side = torch.cuda.Stream(device=dev)

    def step(i, ev):
        # the activation quantiser does not depend on the weights: side stream, overlapped
        # with the pack on the main stream; the contraction waits for both
        s = sets[i % R]
        if ev is not None:
            ev["pack"][0].record(main)
        side.wait_stream(main)
        if ev is not None:
            ev["act"][0].record(side)
        sbn.sbn_quantize_acts(s["X"], s["Xq"], s["s"], err, side)
        if ev is not None:
            ev["act"][1].record(side)
        sbn.sbn_quantize_mask_pack_weights(s["W"], n, m, 1e-5, s["codes"], s["meta"], s["g"], ws,
                                           None, err, main)
        if ev is not None:
            ev["pack"][1].record(main)
        main.wait_stream(side)
        if ev is not None:
            ev["linear"][0].record(main)
        sbn.sbn_linear(s["Xq"], s["s"], s["codes"], s["meta"], s["g"], O, K, n, m, s["Y"], None,
                       err, main)
        if ev is not None:
            ev["linear"][1].record(main)

    steps = args.steps
    ms, per, clocks = timer.run(step, steps, args.warmup, calls=("pack", "act", "linear"))
    dom = max(per, key=per.get)
    if dom == "linear" and T > 4:
        roof = tensor_roof(acct["ops"] / (per["linear"] * 1e-3) / 1e12, peaks,
                           "tensor-core contraction", load_traffic(cfg["name"], "linear"))
    else:
        b = {"pack": acct["pack"], "act": acct["act"], "linear": acct["linear"]}[dom]
        roof = hbm_roof(b / (per[dom] * 1e-3) / 1e9, peaks,
                        {"pack": "quant_mask_pack (k_abs_sum + k_qmp)", "act": "act_quant",
                         "linear": "GEMV"}[dom], load_traffic(cfg["name"], dom))
    return {"value": acct["total"] * world / (ms * 1e-3) / 1e9, "unit": "GB/s",
            "ms_per_step": ms, "steps": steps, "roofline": roof,
            "kernels": {"pack": {"ms": per["pack"], "GB/s": acct["pack"] / (per["pack"] * 1e-3) / 1e9},
                        "act_quant": {"ms": per["act"],
                                      "GB/s": acct["act"] / (per["act"] * 1e-3) / 1e9},
                        "linear": {"ms": per["linear"],
                                   "packed_weight_GB/s": acct["linear_weight"] / (per["linear"] * 1e-3) / 1e9,
                                   "TOPS": acct["ops"] / (per["linear"] * 1e-3) / 1e12}},
            "gpu_launches": 4 * steps, "clocks": clocks,
            "config": {"workload": cfg["name"], "O": O, "K": K, "tokens": T,
                       "pattern": f"{n}:{m}",
                       "step": "pack (S1-S4) | act quant (S5) on a side stream, then contract "
                               "(S6-S7)",
                       "l2": f"{R} rotating input sets ({R * set_bytes / 1e6:.0f} MB > 126 MB L2)"}}


# ---- training-step weight path (configuration 4) -----------------------------------------

def bench_train(args, sbn, dev, local, rank, world, peaks, timer, err):
    """Every linear of the 26-layer decoder re-packed from its masters in 6:8 and 2:4: one
    grouped pack (two launches for all 130 tensors, W read once for the absmean sums and
    once for both patterns' planes).  The per-tensor calls (two launches per tensor and
    pattern, the patterns on two streams) are timed beside it for comparison."""
    Ws = []
    for layer in range(workloads.TRAIN_LAYERS):
        for i, (name, O, K) in enumerate(workloads.TRAIN_LAYER_SHAPES):
            Ws.append(workloads.masters_device(O, K, device=dev, config=4,
                                               tensor=5 * layer + i + 1000 * rank))
    pg = sbn.PackGroup(Ws, ((6, 8), (2, 4)), device=dev)
    st = timer.stream

    def step(i, ev):
        pg.run(err, st)

    steps = min(args.steps, 10)
    ms, _, clocks = timer.run(step, steps, min(args.warmup, 3))

    # the per-tensor calls, into the same planes
    ws = {(6, 8): sbn.new_workspace(8, 64, 2, 4, dev), (2, 4): sbn.new_workspace(8, 64, 2, 4, dev)}
    side = torch.cuda.Stream(device=dev)

    def step_single(i, ev):
        side.wait_stream(st)
        for W, pw in zip(Ws, pg.packed):
            for w in pw:
                s_ = st if (w.n, w.m) == (6, 8) else side
                sbn.sbn_quantize_mask_pack_weights(W, w.n, w.m, 1e-5, w.codes, w.meta,
                                                   w.gamma_eff, ws[(w.n, w.m)], None, err, s_)
        st.wait_stream(side)

    ms_single, _, _ = timer.run(step_single, steps, min(args.warmup, 3))

    # mask statistics of the step: natural zeros of every tensor, and keep-bit flips of both
    # patterns against the previous step's masks (the masters before one update of
    # N(0, 1e-3^2) noise, packed once here)
    gen = torch.Generator(device=dev)
    gen.manual_seed(4000 + rank)
    Wp = [(W.float() + torch.randn(W.shape, device=dev, generator=gen) * 1e-3).to(torch.bfloat16)
          for W in Ws]
    pg_prev = sbn.PackGroup(Wp, ((6, 8), (2, 4)), device=dev)
    pg_prev.run(err, st)
    torch.cuda.synchronize(dev)
    pg_prev.Ws = []
    del Wp
    cnt = torch.zeros((len(Ws), 3), dtype=torch.int64, device=dev)
    # the 390 calls are independent (a counter each): four streams, forked from and joined
    # back to the timed stream, so that the small launches overlap
    sstreams = [torch.cuda.Stream(device=dev) for _ in range(4)]

    def step_stats(i, ev):
        cnt.zero_()
        for s_ in sstreams:
            s_.wait_stream(st)
        for k, (W, pw, pp) in enumerate(zip(Ws, pg.packed, pg_prev.packed)):
            sbn.sbn_count_zero_codes(W, pw[0].gamma_eff, cnt[k, 0:1], sstreams[k % 2])
            for j in range(2):
                sbn.sbn_count_mask_flips(pp[j].meta, pw[j].meta, pw[j].out, pw[j].in_, pw[j].n,
                                         pw[j].m, cnt[k, 1 + j:2 + j], sstreams[2 + j])
        for s_ in sstreams:
            st.wait_stream(s_)

    ms_stats, _, _ = timer.run(step_stats, steps, min(args.warmup, 3))
    tot = cnt.sum(dim=0).tolist()
    weights = sum(W.numel() for W in Ws)
    stats_bytes = weights * 2 + 2 * (weights // 8) + 2 * (weights // 8)
    stats = {"ms_per_step": ms_stats, "GB/s": stats_bytes / (ms_stats * 1e-3) / 1e9,
             "frac": stats_bytes / (ms_stats * 1e-3) / 1e9 / peaks["hbm"],
             "natural_zeros": tot[0] / weights, "flips_6of8": tot[1] / weights,
             "flips_2of4": tot[2] / weights, "launches_per_step": 3 * len(Ws),
             "bytes_per_step": stats_bytes,
             "what": "k_count_zero_codes on W (2 B/w) + k_count_mask_flips on both patterns' "
                     "meta planes of two steps (2 x 0.125 B/w each); the per-tensor calls on "
                     "four streams"}
    moved = weights * 2 * 2 + weights * 3 // 8 + weights // 4  # per pattern: read W + planes
    gbs = moved / (ms * 1e-3) / 1e9
    return {"value": gbs * world, "unit": "GB/s", "ms_per_step": ms, "steps": steps,
            "roofline": hbm_roof(gbs, peaks, "k_abs_sum_group + k_qmp_group, 130 tensors x "
                                 "(6:8, 2:4)",
                                 unit_note="; algorithmic bytes count W once per pattern"),
            "per_tensor_calls": {"ms_per_step": ms_single,
                                 "GB/s": moved / (ms_single * 1e-3) / 1e9,
                                 "launches_per_step": 2 * 2 * len(Ws)},
            "mask_stats": stats,
            "gpu_launches": 2 * steps, "clocks": clocks,
            "config": {"workload": "train-step-26x3200-6of8+2of4", "tensors": len(Ws),
                       "weights": weights, "bytes_per_step": moved,
                       "step": "grouped pack of every tensor into 6:8 and 2:4 (sbn_quantize_"
                               "mask_pack_weights_group)"}}


# ---- next rows: backward, group quantisation, one-launch decode ----------------------------

def bench_backward(args, sbn, dev, local, rank, world, peaks, timer, err):
    """The dual-STE backward on the prefill configuration's shape (W 11008 x 4096 2:4, 2048
    tokens): dX and the clip-gated dW, both tensor-core GEMMs.  Algorithmic flops: 2 T O K
    for each (dW's second bf16 term is an implementation cost, not counted)."""
    cfg = workloads.PREFILL_GEMM
    O, K, T = cfg["O"], cfg["K"], cfg["T"]
    W = workloads.masters_device(O, K, device=dev, config=6, tensor=0)
    X = workloads.torch_bf16(workloads.activations(T, K, seed=0, config=6, tensor=1), dev)
    g = torch.Generator(device=dev)
    g.manual_seed(6)
    dY = torch.randn((T, O), device=dev, generator=g).bfloat16()
    w = sbn.pack_weights(W, 2, 4, err_flag=err)
    Xq, s = sbn.quantize_acts(X, err_flag=err)
    dX = torch.empty((T, K), dtype=torch.float32, device=dev)
    dW = torch.empty((O, K), dtype=torch.float32, device=dev)
    ws = torch.empty(sbn.sbn_backward_workspace_bytes(T, O, K), dtype=torch.uint8, device=dev)
    st = timer.stream

    def step(i, ev):
        if ev is not None:
            ev["dX"][0].record(st)
        sbn.sbn_backward(dY, Xq, s, w.codes, w.meta, W, w.gamma_eff, O, K, 2, 4, dX, None, ws, err,
                         st)
        if ev is not None:
            ev["dX"][1].record(st)
            ev["dW"][0].record(st)
        sbn.sbn_backward(dY, Xq, s, w.codes, w.meta, W, w.gamma_eff, O, K, 2, 4, None, dW, ws, err,
                         st)
        if ev is not None:
            ev["dW"][1].record(st)

    steps = min(args.steps, 10)
    ms, per, clocks = timer.run(step, steps, min(args.warmup, 3), calls=("dX", "dW"))
    flops = 2 * T * O * K
    peak = peaks["bf16"]
    return {"value": 2 * flops * world / (ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": ms,
            "steps": steps,
            "roofline": {"bound": "tensor", "achieved": flops / (per["dX"] * 1e-3) / 1e12,
                         "peak": peak, "unit": "TFLOP/s",
                         "frac": flops / (per["dX"] * 1e-3) / 1e12 / peak, "traffic": None,
                         "kernel": "k_gemm_bf16<0> (dX = g dY Ws, bf16 x bf16 -> fp32)",
                         "peak_source": peak_source(peaks, "bf16_tflops", peaks["bf16"], "burst ")},
            "kernels": {"dX": {"ms": per["dX"], "TFLOP/s": flops / (per["dX"] * 1e-3) / 1e12},
                        "dW": {"ms": per["dW"], "TFLOP/s": flops / (per["dW"] * 1e-3) / 1e12,
                               "note": "two bf16 terms of the scaled dY: 2x the MMA work"}},
            "gpu_launches": 6 * steps, "clocks": clocks,
            "config": {"workload": "backward-11008x4096-t2048-2of4", "flops_per_gemm": flops}}


def bench_group_quant(args, sbn, dev, local, rank, world, peaks, timer, err):
    """Group quantisation (G = 2 blocks along K: the largest G that cuts every layer of the
    stack, K = 4096 or 11008 = 86 x 128, into whole 128-deep blocks): the 32-layer stack's
    decode step at 16 tokens with every layer packed with per-group scales, on the grouped
    calls (the grouped quantiser with per-(token, group) scales, the grouped contraction of
    every block of every layer, the ordered sum: 3 launches).  Beside it, one layer (QKV
    12288 x 4096) through the one-layer calls (a contraction per block + the sum)."""
    G, T = 2, workloads.STACK_DECODE_T
    layers = []
    for idx, name, O, K, tid in stack_layers(rank):
        W = workloads.masters_device(O, K, device=dev, config=7, tensor=tid)
        w = sbn.pack_weights_gq(W, 2, 4, G, err_flag=err)
        del W
        X = workloads.torch_bf16(workloads.student_t(T, K, config=7, tensor=10000 + tid), dev)
        layers.append(dict(X=X, w=w))
    plan = sbn.GqGroupPlan(layers, device=dev)
    st = timer.stream

    def step(i, ev):
        if ev is not None:
            ev["act"][0].record(st)
        plan.quantize_acts(err, st)
        if ev is not None:
            ev["act"][1].record(st)
            ev["linear"][0].record(st)
        plan.linear(err, st)
        if ev is not None:
            ev["linear"][1].record(st)

    steps = args.steps
    ms, per, clocks = timer.run(step, steps, args.warmup, calls=("act", "linear"))
    packed = sum(L["w"].out * L["w"].in_ // 4 for L in layers)
    xbytes = sum(L["X"].numel() * 3 + 4 * G * L["X"].shape[0] for L in layers)  # X in, Xq, s
    ybytes = plan.n * 4 * (G + G + 1)  # partials written and read, Y written
    gbs = packed / (per["linear"] * 1e-3) / 1e9

    # one layer through the one-layer calls (QKV), 8 rotating weight sets beyond L2
    O, K = 12288, 4096
    R = 8
    ws_ = [layers[5 * r]["w"] for r in range(R)]
    X = layers[0]["X"]
    Xq = torch.empty((T, K), dtype=torch.int8, device=dev)
    s1 = torch.empty((G, T), dtype=torch.float32, device=dev)
    Y1 = torch.empty((T, O), dtype=torch.float32, device=dev)
    part = torch.empty(G * T * O * 4, dtype=torch.uint8, device=dev)

    def step1(i, ev):
        w = ws_[i % R]
        sbn.sbn_quantize_acts_gq(X, G, Xq, s1, err, st)
        sbn.sbn_linear_gq(Xq, s1, w.codes, w.meta, w.gamma_eff, O, K, 2, 4, G, Y1, part, None,
                          err, st)

    ms1, _, _ = timer.run(step1, steps, args.warmup, sample_clocks=False)
    return {"value": (packed + xbytes + ybytes) * world / (ms * 1e-3) / 1e9, "unit": "GB/s",
            "ms_per_step": ms, "steps": steps,
            "roofline": hbm_roof(gbs, peaks, f"k_gemm_group over {G * len(layers)} layer blocks "
                                 "+ k_gq_sum",
                                 unit_note="; on packed-weight bytes"),
            "kernels": {"act_quant_group": {"ms": per["act"]},
                        "linear_group_and_sum": {"ms": per["linear"],
                                                 "packed_weight_GB/s": gbs}},
            "one_layer_calls": {"workload": f"12288x4096-t16-G{G}", "ms_per_step": ms1,
                                "packed_weight_GB/s": O * K / 4 / (ms1 * 1e-3) / 1e9,
                                "launches_per_step": 2 + G + 1},
            "gpu_launches": 3 * steps, "clocks": clocks,
            "config": {"workload": f"group-quant-stack-32x4096-t16-2of4-G{G}", "groups": G,
                       "layers": len(layers), "packed_bytes": packed,
                       "l2": f"{packed / 1e9:.2f} GB of packed weights per step > 126 MB L2"}}


def bench_fused_decode(args, sbn, dev, local, rank, world, peaks, timer, err):
    """One-launch decode (sbn_quantize_linear: activation quantiser in the GEMV prologue) on
    the decode configuration's pre-packed weights (W 6912 x 2560 6:8, 1 token), against the
    two separate launches; 8 rotating weight sets beyond L2."""
    cfg = workloads.DECODE_GEMV
    O, K, T, n, m = cfg["O"], cfg["K"], cfg["T"], cfg["n"], cfg["m"]
    R = 16
    packs = []
    for r in range(R):
        W = workloads.masters_device(O, K, device=dev, config=2, tensor=r)
        packs.append(sbn.pack_weights(W, n, m, err_flag=err))
        del W
    X = workloads.torch_bf16(workloads.activations(T, K, seed=0, config=2, tensor=1), dev)
    Xq = torch.empty((T, K), dtype=torch.int8, device=dev)
    s = torch.empty((T,), dtype=torch.float32, device=dev)
    Y = torch.empty((T, O), dtype=torch.float32, device=dev)
    st = timer.stream

    def fused(i, ev):
        w = packs[i % R]
        sbn.sbn_quantize_linear(X, w.codes, w.meta, w.gamma_eff, O, K, n, m, Xq, s, Y, None, err, st)

    def separate(i, ev):
        w = packs[i % R]
        sbn.sbn_quantize_acts(X, Xq, s, err, st)
        sbn.sbn_linear(Xq, s, w.codes, w.meta, w.gamma_eff, O, K, n, m, Y, None, err, st)

    ms_f, _, clocks = timer.run(fused, args.steps, args.warmup)
    ms_s, _, _ = timer.run(separate, args.steps, args.warmup, sample_clocks=False)
    codes_b = O * K // 4
    return {"value": codes_b * world / (ms_f * 1e-3) / 1e9, "unit": "GB/s", "ms_per_step": ms_f,
            "separate_ms_per_step": ms_s,
            "roofline": hbm_roof(codes_b / (ms_f * 1e-3) / 1e9, peaks,
                                 "k_gemv_fused (act quant in the GEMV prologue)",
                                 unit_note="; on the 0.25 B/w codes the GEMV reads"),
            "gpu_launches": args.steps, "clocks": clocks,
            "config": {"workload": "fused-decode-6912x2560-t1-6of8", "rotating_sets": R}}


# ---- the oracle (CPU baseline legs and the reference arm) ---------------------------------

_ORACLE_PREP = {}


def oracle_stack_decode(budget_s, steps=None):
    """The oracle on layer 0 of the stack at 16 tokens (weights packed by the oracle outside
    the timing, as the GPU step has them pre-packed): per layer quant_acts + contract +
    rescale.  Extrapolated x32 to the whole stack."""
    import oracle
    T = workloads.STACK_DECODE_T
    lay = stack_layers(0)[:5]
    if "stack_decode" not in _ORACLE_PREP:
        packs, xs = [], []
        for idx, name, O, K, tid in lay:
            Wb = workloads.masters(O, K, config=5, tensor=tid)
            packs.append(oracle.quantize_mask_pack(Wb, 2, 4, 1e-5))
            xs.append(workloads.student_t(T, K, config=5, tensor=10000 + tid))
        _ORACLE_PREP["stack_decode"] = (packs, xs)
    packs, xs = _ORACLE_PREP["stack_decode"]

    def one():
        for w, xb in zip(packs, xs):
            Xq, s, _ = oracle.quant_acts(xb)
            oracle.rescale(oracle.contract(Xq, w["ws"]), s, w["g"])

    one()
    done, t0 = 0, time.perf_counter()
    while True:
        one()
        done += 1
        el = time.perf_counter() - t0
        if (steps is not None and done >= steps) or (steps is None and el >= budget_s):
            break
    per_layer = el / done
    per_step = per_layer * workloads.STACK_LAYERS
    Ttok = T
    packed_b = sum(O * K for _, _, O, K, _ in lay) // 4
    act_b = sum(3 * Ttok * K + 4 * Ttok for _, _, _, K, _ in lay)
    lin_b = packed_b + sum(Ttok * K + 4 * Ttok + 4 * Ttok * O for _, _, O, K, _ in lay)
    total = (act_b + lin_b) * workloads.STACK_LAYERS
    return {"value": total / per_step / 1e9, "unit": "GB/s", "cores": oracle.num_threads(),
            "kind": "oracle", "ms_per_step": per_step * 1e3,
            "sample": f"layer 0 of 32 (5 layers, 16 tokens, quant_acts + contract + rescale), "
                      f"{done} runs in {el:.1f} s; step time extrapolated x32"}


def oracle_single(cfg, budget_s):
    import oracle
    acct = step_accounting(cfg)
    Wb = workloads.masters(cfg["O"], cfg["K"], seed=0, config=1, tensor=0)
    Xb = workloads.activations(cfg["T"], cfg["K"], seed=0, config=1, tensor=1)

    def one():
        w = oracle.quantize_mask_pack(Wb, cfg["n"], cfg["m"], 1e-5)
        Xq, s, _ = oracle.quant_acts(Xb)
        oracle.rescale(oracle.contract(Xq, w["ws"]), s, w["g"])

    one()
    done, t0 = 0, time.perf_counter()
    while True:
        one()
        done += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    return {"value": acct["total"] * done / el / 1e9, "unit": "GB/s",
            "cores": oracle.num_threads(), "kind": "oracle", "ms_per_step": el / done * 1e3,
            "sample": f"{done} whole steps of {cfg['name']} ({el:.1f} s)"}


def oracle_train(budget_s):
    """The oracle packs the 5 tensors of one layer in both patterns per sample, extrapolated
    x26 to the training step."""
    import oracle
    Ws = [workloads.masters(O, K, config=4, tensor=i)
          for i, (_, O, K) in enumerate(workloads.TRAIN_LAYER_SHAPES)]

    def one():
        for W in Ws:
            for (n, m) in ((6, 8), (2, 4)):
                oracle.quantize_mask_pack(W, n, m, 1e-5)

    done, t0 = 0, time.perf_counter()
    while True:
        one()
        done += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    weights = sum(O * K for _, O, K in workloads.TRAIN_LAYER_SHAPES)
    moved = weights * 4 + weights * 3 // 8 + weights // 4
    return {"value": moved * done / el / 1e9, "unit": "GB/s", "cores": oracle.num_threads(),
            "kind": "oracle", "ms_per_step": el / done * 1e3 * workloads.TRAIN_LAYERS,
            "sample": f"one layer (5 tensors x 6:8 and 2:4), {done} runs in {el:.1f} s; "
                      "step time extrapolated x26"}


def oracle_stack_prefill(budget_s):
    """The oracle on 128 of the 4096 tokens of layer 0 (per layer quant_acts + contract +
    rescale), in kept TOPS."""
    import oracle
    T = 128
    lay = stack_layers(0)[:5]
    packs, xs = [], []
    for idx, name, O, K, tid in lay:
        packs.append(oracle.quantize_mask_pack(workloads.masters(O, K, config=5, tensor=tid),
                                               2, 4, 1e-5))
        xs.append(workloads.student_t(T, K, config=5, tensor=20000 + tid))
    done, t0 = 0, time.perf_counter()
    while True:
        for w, xb in zip(packs, xs):
            Xq, s, _ = oracle.quant_acts(xb)
            oracle.rescale(oracle.contract(Xq, w["ws"]), s, w["g"])
        done += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    ops = T * sum(O * K for _, _, O, K, _ in lay) * done
    return {"value": ops / el / 1e12, "unit": "TOPS", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"128 of 4096 tokens of layer 0 (5 layers), {done} runs in {el:.1f} s"}


def run_reference(args):
    """The oracle as the reference arm, on the default workload's metric and unit: each step
    is layer 0 of the stack (5 layers, 16 tokens) -- a bounded sample of the stack's decode
    step -- timed on the host cores.  Under torchrun only rank 0 runs."""
    world, rank, _ = dist.env_world()
    if rank != 0:
        return
    import oracle
    for _ in range(args.warmup):
        oracle_stack_decode(0.0, steps=1)
    t0 = time.perf_counter()
    rec = oracle_stack_decode(0.0, steps=args.steps)
    el = time.perf_counter() - t0
    sample = (f"{args.steps} steps, each layer 0 of the 32-layer stack (5 layers, 16 tokens); "
              "the value counts the whole stack's bytes with the step time extrapolated x32")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": rec["value"], "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": rec["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int8xternary->int64, fp64 out", "data": "synthetic",
        "config": {"workload": "stack-decode-32x4096-t16-2of4", "tokens": 16, "pattern": "2:4"},
        "cpu_baseline": {"value": rec["value"], "unit": "GB/s", "cores": oracle.num_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": rec["value"], "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "wall_s": el}))


# ---- main ----------------------------------------------------------------------------------

def run_cuda(args):
    import sparse_linear_layers_absmean_b200 as sbn

    world, rank, local = dist.init("nccl")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    peaks = load_peaks()
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    timer = Timer(dev, local)
    result = None
    if args.workload in ("stack", "stack-prefill"):
        packed = build_stack(sbn, dev, rank, err)
        head, _, _ = bench_stack_decode(args, sbn, dev, local, rank, world, peaks, timer,
                                        packed, err)
        head_flag = int(err.item())  # the head line's own flag; the sub-records keep theirs
        err.zero_()
        if args.workload == "stack-prefill":
            head = bench_stack_prefill(args, sbn, dev, local, rank, world, peaks, timer, packed,
                                       err)
            subs = {}
        else:
            subs = {}
            if world == 1 and not args.no_sub:
                subs["stack_prefill"] = bench_stack_prefill(args, sbn, dev, local, rank, world,
                                                            peaks, timer, packed, err)
                subs["stack_prefill"]["err_flag"] = int(err.item())
                err.zero_()
        del packed
        torch.cuda.empty_cache()
        if world == 1 and not args.no_sub and args.workload == "stack":
            subs["decode_gemv"] = bench_single(args, sbn, dev, local, rank, world, peaks, timer,
                                               workloads.DECODE_GEMV, err)
            subs["decode_gemv"]["err_flag"] = int(err.item())
            err.zero_()
            subs["prefill_gemm"] = bench_single(args, sbn, dev, local, rank, world, peaks, timer,
                                                workloads.PREFILL_GEMM, err)
            subs["prefill_gemm"]["err_flag"] = int(err.item())
            err.zero_()
            subs["train_step"] = bench_train(args, sbn, dev, local, rank, world, peaks, timer,
                                             err)
            subs["train_step"]["err_flag"] = int(err.item())
            err.zero_()
            subs["backward"] = bench_backward(args, sbn, dev, local, rank, world, peaks, timer, err)
            subs["backward"]["err_flag"] = int(err.item())
            err.zero_()
            subs["group_quant"] = bench_group_quant(args, sbn, dev, local, rank, world, peaks,
                                                    timer, err)
            subs["group_quant"]["err_flag"] = int(err.item())
            err.zero_()
            subs["fused_decode"] = bench_fused_decode(args, sbn, dev, local, rank, world, peaks,
                                                      timer, err)
            subs["fused_decode"]["err_flag"] = int(err.item())
            err.zero_()
        # the line's flag: every flag raised anywhere in the run
        for rec in subs.values():
            head_flag |= rec.get("err_flag", 0)
        err.fill_(head_flag)
    elif args.workload == "decode":
        head, subs = bench_single(args, sbn, dev, local, rank, world, peaks, timer,
                                  workloads.DECODE_GEMV, err), {}
    elif args.workload == "prefill":
        head, subs = bench_single(args, sbn, dev, local, rank, world, peaks, timer,
                                  workloads.PREFILL_GEMM, err), {}
    else:
        head, subs = bench_train(args, sbn, dev, local, rank, world, peaks, timer, err), {}
    flag = int(err.item())
    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            b = args.cpu_seconds
            if args.workload == "stack":
                cpu = oracle_stack_decode(b)
                if "stack_prefill" in subs:
                    subs["stack_prefill"]["cpu_baseline"] = oracle_stack_prefill(b / 2)
                for key, cfg in (("decode_gemv", workloads.DECODE_GEMV),
                                 ("prefill_gemm", workloads.PREFILL_GEMM)):
                    if key in subs:
                        subs[key]["cpu_baseline"] = oracle_single(cfg, b / 2)
                if "train_step" in subs:
                    subs["train_step"]["cpu_baseline"] = oracle_train(b / 2)
            elif args.workload == "stack-prefill":
                cpu = oracle_stack_prefill(b)
            elif args.workload == "decode":
                cpu = oracle_single(workloads.DECODE_GEMV, b)
            elif args.workload == "prefill":
                cpu = oracle_single(workloads.PREFILL_GEMM, b)
            else:
                cpu = oracle_train(b)
        line = {
            "metric": METRIC, "value": head["value"], "unit": head["unit"], "n_gpus": world,
            "steps": head.get("steps", args.steps), "warmup": args.warmup,
            "ms_per_step": head["ms_per_step"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "int8 x ternary -> int32, fp32 out",
            "data": "synthetic (seeded: N(0,0.02) bf16 masters drawn on the GPU, packed once; "
                    "Student-t(4) bf16 activations)",
            "config": head["config"], "roofline": head["roofline"],
            "cpu_baseline": cpu, "e2e": head.get("e2e"), "gpu_launches": head["gpu_launches"],
            "clocks": head["clocks"], "kernels": head.get("kernels"), "err_flag": flag,
            "bytes_per_step": head.get("bytes_per_step"), "sub": subs,
            "peaks": {k: peaks[k] for k in ("hbm", "bf16", "bf16_sustained", "source")},
        }
        # the top record's own side measurements (per-tensor calls, mask statistics, ...)
        for key in ("per_tensor_calls", "mask_stats", "one_layer_calls"):
            if key in head:
                line[key] = head[key]
        print(json.dumps(line))
    dist.barrier(dev)
    dist.shutdown()
    if flag:
        sys.exit(1)


def run_only(args):
    """Profiling aid: one kind of C-ABI call on the workload's first inputs, `warmup + steps`
    times on one stream, nothing timed (for single-kernel ncu captures).  Prints one JSON
    line saying what ran."""
    import sparse_linear_layers_absmean_b200 as sbn

    dev = torch.device("cuda", 0)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    calls = args.warmup + args.steps
    if args.only == "backward" and args.workload != "prefill":
        sys.exit("--only backward takes the prefill workload (W 11008x4096 2:4, 2048 tokens)")
    if args.workload == "stack":
        packed = build_stack(sbn, dev, 0, err)
        T = workloads.STACK_DECODE_T
        layers = []
        for (idx, name, O, K, tid), w in zip(stack_layers(0), packed):
            X = workloads.torch_bf16(workloads.student_t(T, K, config=5, tensor=10000 + tid), dev)
            layers.append(dict(X=X, Xq=torch.empty((T, K), dtype=torch.int8, device=dev),
                               s=torch.empty((T,), dtype=torch.float32, device=dev), w=w,
                               Y=torch.empty((T, O), dtype=torch.float32, device=dev)))
        plan = sbn.GroupPlan(layers, device=dev)
        plan.quantize_acts(err)
        for _ in range(calls):
            if args.only == "act":
                plan.quantize_acts(err)
            else:
                plan.linear(err)
    elif args.workload == "train-step":
        if args.only != "pack":
            sys.exit("train-step --only takes pack (the grouped 6:8 + 2:4 pack)")
        Ws = [workloads.masters_device(O, K, device=dev, config=4, tensor=5 * layer + i)
              for layer in range(args.train_layers)
              for i, (name, O, K) in enumerate(workloads.TRAIN_LAYER_SHAPES)]
        pg = sbn.PackGroup(Ws, ((6, 8), (2, 4)), device=dev)
        for _ in range(calls):
            pg.run(err)
    elif args.only == "backward":
        cfg = workloads.PREFILL_GEMM
        O, K, T = cfg["O"], cfg["K"], cfg["T"]
        W = workloads.masters_device(O, K, device=dev, config=6, tensor=0)
        X = workloads.torch_bf16(workloads.activations(T, K, seed=0, config=6, tensor=1), dev)
        g = torch.Generator(device=dev)
        g.manual_seed(6)
        dY = torch.randn((T, O), device=dev, generator=g).bfloat16()
        w = sbn.pack_weights(W, 2, 4, err_flag=err)
        Xq, s = sbn.quantize_acts(X, err_flag=err)
        dX = torch.empty((T, K), dtype=torch.float32, device=dev)
        dW = torch.empty((O, K), dtype=torch.float32, device=dev)
        ws = torch.empty(sbn.sbn_backward_workspace_bytes(T, O, K), dtype=torch.uint8, device=dev)
        for _ in range(calls):
            sbn.sbn_backward(dY, Xq, s, w.codes, w.meta, W, w.gamma_eff, O, K, 2, 4, dX, None, ws,
                             err)
            sbn.sbn_backward(dY, Xq, s, w.codes, w.meta, W, w.gamma_eff, O, K, 2, 4, None, dW, ws,
                             err)
    else:
        cfg = {"decode": workloads.DECODE_GEMV, "prefill": workloads.PREFILL_GEMM}[args.workload]
        O, K, T, n, m = cfg["O"], cfg["K"], cfg["T"], cfg["n"], cfg["m"]
        W = workloads.torch_bf16(workloads.masters(O, K, seed=0, config=1, tensor=0), dev)
        X = workloads.torch_bf16(workloads.activations(T, K, seed=0, config=1, tensor=1), dev)
        w = sbn.pack_weights(W, n, m, err_flag=err)
        Xq, s = sbn.quantize_acts(X, err_flag=err)
        Y = torch.empty((T, O), dtype=torch.float32, device=dev)
        ws = sbn.new_workspace(O, K, n, m, dev)
        for _ in range(calls):
            if args.only == "pack":
                sbn.sbn_quantize_mask_pack_weights(W, n, m, 1e-5, w.codes, w.meta, w.gamma_eff,
                                                   ws, None, err)
            elif args.only == "act":
                sbn.sbn_quantize_acts(X, Xq, s, err)
            else:
                sbn.sbn_linear(Xq, s, w.codes, w.meta, w.gamma_eff, O, K, n, m, Y, None, err)
    torch.cuda.synchronize()
    flag = int(err.item())
    print(json.dumps({"only": args.only, "workload": args.workload, "calls": calls,
                      "err_flag": flag}))
    if flag:
        sys.exit(1)


def relaunch(args):
    """`--gpus N` outside torchrun: start N local ranks under torchrun and return its status."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={args.gpus}", "--master-addr=127.0.0.1",
           f"--master-port={29500 + os.getpid() % 1000}", os.path.abspath(__file__)] + sys.argv[1:]
    return subprocess.call(cmd)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--workload", default="stack", choices=WORKLOADS)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sub", action="store_true", help="headline only, no sub-records")
    ap.add_argument("--only", choices=["pack", "act", "linear", "backward"],
                    help="profiling aid: one kind of C-ABI call, untimed (decode, prefill, stack; "
                         "train-step: pack; prefill: backward, dX then dW)")
    ap.add_argument("--train-layers", type=int, default=workloads.TRAIN_LAYERS,
                    help="profiling aid with --only: decoder layers of the training step "
                         "(default 26)")
    ap.add_argument("--stack-layers", type=int, default=workloads.STACK_LAYERS,
                    help="profiling aid with --only: decoder layers of the stack (default 32)")
    args = ap.parse_args()
    if (args.stack_layers != workloads.STACK_LAYERS or
            args.train_layers != workloads.TRAIN_LAYERS) and not args.only:
        sys.exit("--stack-layers / --train-layers are profiling aids for --only runs")
    global STACK_LAYERS
    STACK_LAYERS = args.stack_layers
    if args.warmup < 3:
        args.warmup = 3
    world = int(os.environ.get("WORLD_SIZE", "0"))
    if args.gpus > 1 and world == 0:
        sys.exit(relaunch(args))
    if world and world != args.gpus:
        sys.exit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    if args.only:
        run_only(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_cuda(args)


if __name__ == "__main__":
    main()
