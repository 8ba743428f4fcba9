"""Seeded synthetic inputs for the Sparse-BitLinear forward.

This module only draws random numbers and rounds them to bf16 (round-to-nearest-even);
it holds none of the method's arithmetic.  It is the one module that both the CPU
oracle's callers and the CUDA path's callers share: the same bytes go to both sides.

Recipe (all seeds derive from numpy.random.SeedSequence([seed, config, tensor, step]),
PCG64):
  masters      W ~ N(0, 0.02^2), rounded to bf16;
  activations  X ~ N(0, 1); 0.5% of the channels (round(0.005*K) distinct columns) are
               multiplied by 20 ("outlier channels"), then rounded to bf16;
  student-t    X ~ t(nu=4) per element, rounded to bf16;
  noise        W_{s+1} = bf16(W_s + N(0, 1e-3^2)), the per-step master update.
The pages train Qwen2.5 models on RefineWeb and evaluate on downstream suites; none of
those are available here, so these tensors, with the shapes of the workloads below,
stand in for them.
"""
import numpy as np
import torch

# Workloads: (name, O, K, T, n, m, out_dtype)
TINY = dict(name="tiny-256x256-t8-2of4", O=256, K=256, T=8, n=2, m=4)
DECODE_GEMV = dict(name="decode-gemv-6912x2560-t1-6of8", O=6912, K=2560, T=1, n=6, m=8)
PREFILL_GEMM = dict(name="prefill-gemm-11008x4096-t2048-2of4", O=11008, K=4096, T=2048,
                    n=2, m=4)

# Training-step weight path: one decoder layer of a 26-layer model, hidden 3200, FFN 8640.
TRAIN_LAYER_SHAPES = [("qkv", 9600, 3200), ("o", 3200, 3200), ("gate", 8640, 3200),
                      ("up", 8640, 3200), ("down", 3200, 8640)]
TRAIN_LAYERS = 26
TRAIN_STEPS = 10

TRAIN_STEP = dict(name="train-step-26x3200-6of8+2of4", kind="train")

# Full 32-layer block stack, hidden 4096, FFN 11008.
STACK_LAYER_SHAPES = [("qkv", 12288, 4096), ("o", 4096, 4096), ("gate", 11008, 4096),
                      ("up", 11008, 4096), ("down", 4096, 11008)]
STACK_LAYERS = 32
STACK_DECODE_T = 16
STACK_PREFILL_T = 4096
STACK_DECODE = dict(name="stack-decode-32x4096-t16-2of4", kind="stack", T=STACK_DECODE_T)
STACK_PREFILL = dict(name="stack-prefill-32x4096-t4096-2of4", kind="stack",
                     T=STACK_PREFILL_T)


def rng(seed: int = 0, config: int = 0, tensor: int = 0, step: int = 0):
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, config, tensor,
                                                                       step])))


def to_bf16_bits(a) -> np.ndarray:
    """Round a float array to bf16 (RNE) and return the uint16 bit patterns."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def bf16_bits_to_f32(b) -> np.ndarray:
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def masters(O: int, K: int, *, seed=0, config=0, tensor=0, step=0, std=0.02) -> np.ndarray:
    r = rng(seed, config, tensor, step)
    return to_bf16_bits(r.standard_normal((O, K), dtype=np.float32) * np.float32(std))


def masters_device(O: int, K: int, *, device, seed=0, config=0, tensor=0, std=0.02):
    """bf16 masters N(0, std^2) drawn on the GPU from a seeded torch generator: for the
    multi-GB benchmark workloads (whole decoder stacks), where host generation would take
    minutes.  Not used by the parity tests, whose inputs come from `masters`."""
    g = torch.Generator(device=device)
    g.manual_seed(((seed * 1000003 + config) * 1000003 + tensor) & ((1 << 62) - 1))
    return (torch.randn((O, K), device=device, generator=g) * std).to(torch.bfloat16)


def activations(T: int, K: int, *, seed=0, config=0, tensor=1, step=0, outliers=True,
                outlier_frac=0.005, outlier_scale=20.0) -> np.ndarray:
    r = rng(seed, config, tensor, step)
    x = r.standard_normal((T, K), dtype=np.float32)
    if outliers:
        n_out = int(round(outlier_frac * K))
        cols = r.choice(K, size=n_out, replace=False)
        x[:, cols] *= np.float32(outlier_scale)
    return to_bf16_bits(x)


def student_t(T: int, K: int, *, seed=0, config=0, tensor=1, step=0, nu=4.0) -> np.ndarray:
    r = rng(seed, config, tensor, step)
    return to_bf16_bits(r.standard_t(nu, size=(T, K)).astype(np.float32))


def perturb(W_bits: np.ndarray, *, seed=0, config=0, tensor=0, step=0, std=1e-3) -> np.ndarray:
    """One master update of the training-step workload: W + N(0, std^2), back to bf16."""
    r = rng(seed, config, tensor, step + 1)
    w = bf16_bits_to_f32(W_bits)
    return to_bf16_bits(w + r.standard_normal(w.shape, dtype=np.float32) * np.float32(std))


def torch_bf16(bits: np.ndarray, device="cpu") -> torch.Tensor:
    """The same bytes as a torch bf16 tensor (on ``device``)."""
    t = torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16))
    return t.view(torch.bfloat16).to(device)
