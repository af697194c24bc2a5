"""Seeded synthetic workloads: parameter shapes, hyper-parameters and input draws.

This module holds no arithmetic of the optimizer. It only says which matrices
exist, which hyper-parameters each workload uses, and draws the seeded random
inputs (weights, per-worker gradients, drifting CacheMuon momenta, synthetic
Newton-Schulz outputs for the sign/vote tests). Both the CPU oracle tests and
the CUDA path's tests and benchmark take their inputs from here, so the two
sides always see the same numbers.

The shapes stand in for the training runs named on the pages (CIFAR-10 /
ResNet-50 and nanoGPT for Sign-Muon, "SignMuon: Communication-Efficient
Distributed Muon Optimization", section 4; GPT-2 Large for CacheMuon,
"CacheMuon" experiments section; GPT-2 Large shapes for LionMuon,
"LionMuon" results section). No dataset is involved: only the parameter shapes
are taken from the architectures.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

QUINTIC = (3.4445, -4.7750, 2.0315)
CUBIC = (1.5, -0.5, 0.0)


def resnet50_conv_shapes() -> list[tuple[int, int]]:
    """All 53 convolution weights of ResNet-50 as C_out x (C_in*k_h*k_w).

    Standard ImageNet stem (7x7, 3 -> 64), then bottleneck stages with
    (blocks, mid, out) = (3, 64, 256), (4, 128, 512), (6, 256, 1024),
    (3, 512, 2048); the first block of each stage has a 1x1 projection.
    """
    shapes = [(64, 3 * 7 * 7)]
    c_in = 64
    for blocks, mid, out in ((3, 64, 256), (4, 128, 512), (6, 256, 1024), (3, 512, 2048)):
        for blk in range(blocks):
            shapes.append((mid, c_in))          # 1x1 reduce
            shapes.append((mid, mid * 9))       # 3x3
            shapes.append((out, mid))           # 1x1 expand
            if blk == 0:
                shapes.append((out, c_in))      # 1x1 projection shortcut
            c_in = out
    return shapes


def gpt2_small_shapes() -> list[tuple[int, int]]:
    """12 transformer blocks x {qkv 768x2304, proj 768x768, fc 768x3072, fc-out 3072x768}."""
    return [s for _ in range(12) for s in ((768, 2304), (768, 768), (768, 3072), (3072, 768))]


def gpt2_large_shapes() -> list[tuple[int, int]]:
    """36 transformer blocks x {1280x3840, 1280x1280, 1280x5120, 5120x1280}."""
    return [s for _ in range(36) for s in ((1280, 3840), (1280, 1280), (1280, 5120), (5120, 1280))]


def resnet18_conv_shapes() -> list[tuple[int, int]]:
    """The 20 convolution weights of ResNet-18 as C_out x (C_in*k_h*k_w) (the
    vision run of the "CacheMuon" experiments): the 7x7 stem, then four stages
    of two basic blocks (two 3x3 convolutions each) with 64, 128, 256, 512
    channels, and a 1x1 projection in the first block of stages 2-4.
    11,166,912 parameters."""
    shapes = [(64, 3 * 7 * 7)]
    c_in = 64
    for stage, c in enumerate((64, 128, 256, 512)):
        for blk in range(2):
            shapes.append((c, c_in * 9))
            shapes.append((c, c * 9))
            if blk == 0 and stage > 0:
                shapes.append((c, c_in))
            c_in = c
    return shapes


# LLaMA-style decoder blocks at the 124M / 355M / 720M scales the "LionMuon"
# summary trains at: per block the attention projections q, k, v, o (d x d)
# and the gated MLP gate, up (h x d) and down (d x h). The pages give only the
# parameter counts; the widths are a reading: GPT-2's d and depth at 124M and
# 355M, d = 1536 with 24 blocks at 720M, and h = 8/3 d rounded up to a multiple
# of 256. Embeddings are not matrices the optimizer orthogonalises here.
LLAMA_DIMS = {"124m": (768, 12), "355m": (1024, 24), "720m": (1536, 24)}


def llama_shapes(size: str) -> list[tuple[int, int]]:
    d, layers = LLAMA_DIMS[size]
    h = -(-(8 * d // 3) // 256) * 256
    block = [(d, d)] * 4 + [(h, d), (h, d), (d, h)]
    return [s for _ in range(layers) for s in block]


@dataclass
class SignMuonWorkload:
    name: str
    shapes: list
    workers: int
    beta: float
    coeffs: tuple
    iters: int
    eta: float
    w_dtype: str            # "f32" | "bf16"
    w_init: str             # "normal002" | "he"
    grad_sigma: float
    vote: str               # "int8" | "popcount"
    tie_value: int = 0
    local_polar: bool = False
    steps: int = 1
    eps: float = 1e-7


SIGN_MUON_WORKLOADS = {
    "c1_256sq": SignMuonWorkload("c1_256sq", [(256, 256)], 3, 0.9, CUBIC, 5, 0.01, "f32",
                                 "normal002", 1.0, "popcount", 0, False, 1),
    "c2_resnet50": SignMuonWorkload("c2_resnet50", resnet50_conv_shapes(), 4, 0.9, QUINTIC, 1, 0.02,
                                    "f32", "he", 1e-2, "int8", 0, False, 10),
    "c3_gpt2s": SignMuonWorkload("c3_gpt2s", gpt2_small_shapes(), 8, 0.95, QUINTIC, 5, 0.02, "bf16",
                                 "normal002", 1.0, "popcount", 0, True, 20),
    # more layer sets for the same kernels: ResNet-18 with the ResNet-50 set's
    # hyper-parameters, the LLaMA-style sets with the GPT-2-small set's
    "resnet18": SignMuonWorkload("resnet18", resnet18_conv_shapes(), 4, 0.9, QUINTIC, 1, 0.02,
                                 "f32", "he", 1e-2, "int8", 0, False, 10),
    "llama124m": SignMuonWorkload("llama124m", llama_shapes("124m"), 8, 0.95, QUINTIC, 5, 0.02, "bf16",
                                  "normal002", 1.0, "popcount", 0, False, 20),
    "llama355m": SignMuonWorkload("llama355m", llama_shapes("355m"), 8, 0.95, QUINTIC, 5, 0.02, "bf16",
                                  "normal002", 1.0, "popcount", 0, False, 20),
    "llama720m": SignMuonWorkload("llama720m", llama_shapes("720m"), 8, 0.95, QUINTIC, 5, 0.02, "bf16",
                                  "normal002", 1.0, "popcount", 0, False, 20),
}


@dataclass
class CacheMuonWorkload:
    name: str
    shape: tuple
    gammas: tuple = (2.0, 15.0)
    drift: float = 0.01
    steps: int = 50
    coeffs: tuple = QUINTIC
    iters: int = 5
    seed0: int = 4242


CACHE_MUON_WORKLOADS = {
    "c4_4096sq": CacheMuonWorkload("c4_4096sq", (4096, 4096)),
    "c4_8192sq": CacheMuonWorkload("c4_8192sq", (8192, 8192)),
    "c4_4096x16384": CacheMuonWorkload("c4_4096x16384", (4096, 16384)),
}


@dataclass
class LionMuonWorkload:
    name: str
    shapes: list
    workers: int = 16
    beta1: float = 0.9
    beta2: float = 0.99
    period: int = 4
    coeffs: tuple = QUINTIC
    iters: int = 5
    eta: float = 3e-4
    tie_value: int = 0
    steps: int = 100
    w_dtype: str = "bf16"
    eps: float = 1e-7


LION_MUON_WORKLOADS = {
    "c5_gpt2l": LionMuonWorkload("c5_gpt2l", gpt2_large_shapes()),
}


# ----------------------------------------------------------------------------
# seeded draws
# ----------------------------------------------------------------------------

def _rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def weights(shapes, init: str, dtype: str = "f32", seed_base: int = 1000) -> list[np.ndarray]:
    """W_i ~ N(0, 0.02^2) or He-normal N(0, 2/fan_in); matrix i uses seed 1000 + i.

    bf16 weights are returned as float32 arrays whose values bf16 holds
    exactly, so both sides start from the same bf16 numbers.
    """
    out = []
    for i, (r, c) in enumerate(shapes):
        std = 0.02 if init == "normal002" else float(np.sqrt(2.0 / c))
        w = (_rng(seed_base + i).standard_normal((r, c), dtype=np.float32) * np.float32(std))
        if dtype == "bf16":
            w = _to_bf16_values(w)
        out.append(w)
    return out


def _to_bf16_values(x: np.ndarray) -> np.ndarray:
    """Draw-time quantisation of inputs to bf16-representable float32 values.

    Inputs only, not the method's rounding: the low 16 bits of the float32
    pattern are cleared (truncation toward zero), which always yields a value
    that bf16 holds exactly. Gaussian draws hold no NaN or Inf.
    """
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    return (u & np.uint32(0xFFFF0000)).view(np.float32)


class GradientStreams:
    """Per-worker gradient streams: worker m draws from a generator seeded m.

    Each call of ``next_step`` draws, for every worker, one gradient for every
    matrix in order (all layers of worker 0 first use worker 0's stream, and
    so on), scaled by sigma. Successive steps continue the same streams.
    """

    def __init__(self, shapes, workers: int, sigma: float, seed_base: int = 0):
        self.shapes = list(shapes)
        self.workers = workers
        self.sigma = np.float32(sigma)
        self.rngs = [_rng(seed_base + m) for m in range(workers)]

    def next_step(self) -> list[list[np.ndarray]]:
        """Returns grads[layer][worker] as float32 arrays."""
        per_worker = []
        for m in range(self.workers):
            g = self.rngs[m]
            per_worker.append([g.standard_normal(s, dtype=np.float32) * self.sigma for s in self.shapes])
        return [[per_worker[m][i] for m in range(self.workers)] for i in range(len(self.shapes))]


def cachemuon_momenta(shape, steps: int, drift: float = 0.01, seed0: int = 4242):
    """M_0 ~ N(0,1) from seed 4242; M_{t+1} = M_t + drift * N(0,1) drawn with seed 4243 + t.

    Yields float32 matrices M_0, M_1, ..., M_{steps-1}. The drift is applied
    in float32 (this is input generation, not the method).
    """
    m = _rng(seed0).standard_normal(shape, dtype=np.float32)
    yield m.copy()
    for t in range(steps - 1):
        m = m + np.float32(drift) * _rng(seed0 + 1 + t).standard_normal(shape, dtype=np.float32)
        yield m.copy()


def synthetic_polar_outputs(shape, workers: int, seed: int, dtype: str = "bf16",
                            zero_fraction: float = 0.0) -> list[np.ndarray]:
    """Stand-in Newton-Schulz outputs U^(m) for the sign/pack/vote/update tests.

    Both sides receive the same U (bf16-representable values when dtype is
    bf16); a fraction of exact zeros (and negative zeros) exercises the
    sign(0) convention.
    """
    g = _rng(seed)
    out = []
    for _ in range(workers):
        u = g.standard_normal(shape, dtype=np.float32) * np.float32(0.03)
        if zero_fraction > 0:
            mask = g.random(shape) < zero_fraction
            neg = g.random(shape) < 0.5
            u = np.where(mask, np.where(neg, np.float32(-0.0), np.float32(0.0)), u).astype(np.float32)
        if dtype == "bf16":
            u = _to_bf16_values(u)
        out.append(u)
    return out
