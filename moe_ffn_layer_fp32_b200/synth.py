"""Seeded synthetic inputs for the fused MoE FFN layer.

This module only draws random numbers and encodes them as the layer's input
types (BF16 activations, FP32 weights, FP32 router weights and bias).  It holds
none of the layer's arithmetic: quantisation, routing and the expert FFNs live
in the library (CUDA) and, independently, in the CPU oracle used by the tests.
Both sides receive the very same arrays from here.

Distributions (MobileMoE, "MoE preliminaries" and "QAT" sections, plus the
workload table of the layer benchmark):
  * router weight  W_r[d_model, 60]  ~ N(0, 0.02)   FP32
  * expert weights (gate, up [h, d_model]; down [d_model, h]) ~ N(0, 0.02) FP32,
    quantised later by Eq. (6)
  * activations    x[T, d_model]     ~ N(0, 1) rounded to BF16 (nearest-even)
  * optional skew bias b_e = c * ln(1 / (rank_e + 1)), rank_e the position of
    expert e in a random permutation of the 60 experts.

Draw order inside one PCG64 stream (seeded per layer): W_r, the permutation,
then experts 0..59 (gate, up, down) and the shared expert last.  Activations
come from their own PCG64 stream so that any number of tokens or decode steps
can be drawn without regenerating weights.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

N_ROUTED = 60
TOP_K = 4
GROUP = 32


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    d: int
    h: int
    E: int = N_ROUTED
    k: int = TOP_K
    bias_coef: float | None = None
    layers: int = 1
    weight_seed: int = 0
    x_seed: int = 1
    shared_hidden: int | None = None
    desc: str = ""

    @property
    def hs(self) -> int:
        return self.h if self.shared_hidden is None else self.shared_hidden


# The workloads of the layer benchmark.  Sizes are the ones the benchmark
# table states; c1's 24 layers use weight seeds 1000+l and decode step s
# draws its activations with seed 10**6 + s.
WORKLOADS: dict[str, Workload] = {
    "c0": Workload("c0", T=64, d=256, h=128,
                   desc="tiny layer: T=64, d_model=256, h=128"),
    "c1": Workload("c1", T=1, d=1024, h=512, layers=24, weight_seed=1000,
                   x_seed=10**6, desc="decode: T=1, d_model=1024, h=512, 24 layers"),
    "c1b8": Workload("c1b8", T=8, d=1024, h=512, layers=24, weight_seed=1000,
                     x_seed=10**6, desc="decode batch 8: T=8, d_model=1024, h=512, 24 layers"),
    "c2": Workload("c2", T=2048, d=1024, h=512,
                   desc="prefill, balanced: T=2048, d_model=1024, h=512"),
    "c3a": Workload("c3a", T=8192, d=1536, h=768, bias_coef=1.5,
                    desc="prefill, skewed (bias coefficient 1.5): T=8192, d_model=1536, h=768"),
    "c3b": Workload("c3b", T=8192, d=1536, h=768, bias_coef=0.25,
                    desc="prefill, skewed (bias coefficient 0.25): T=8192, d_model=1536, h=768"),
    "c4": Workload("c4", T=32768, d=2048, h=1024,
                   desc="large prefill: 4 x 8192 = 32768 tokens, d_model=2048, h=1024"),
    "c4dec": Workload("c4dec", T=64, d=2048, h=1024, x_seed=2,
                      desc="batched decode: T=64 on the d_model=2048, h=1024 weights"),
    # The MobileMoE-S layer shape: 60 routed SwiGLU experts of 768 x 384 and one
    # shared expert four times a routed one (hidden 1536), top-4.
    "s2048": Workload("s2048", T=2048, d=768, h=384, shared_hidden=1536, weight_seed=3, x_seed=4,
                      desc="MobileMoE-S layer, prefill: T=2048, d_model=768, h=384, shared hidden 1536"),
    "s1": Workload("s1", T=1, d=768, h=384, shared_hidden=1536, layers=24, weight_seed=2000, x_seed=3 * 10**6,
                   desc="MobileMoE-S layer, decode: T=1, d_model=768, h=384, shared hidden 1536, 24 layers"),
}


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round FP32 values to BF16 (nearest, ties to even); returns uint16 bit patterns."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    rounded = u + (np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1)))
    return (rounded >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclass
class LayerWeights:
    """FP32 weights of one MoE layer.  Index E (=60) of the expert axis is the shared expert."""
    d: int
    h: int
    hs: int
    E: int
    w_router: np.ndarray            # [d, E] float32
    router_bias: np.ndarray | None  # [E] float32 or None
    w_gate_up: list = field(default_factory=list)   # E+1 arrays [2*hid, d] float32 (gate rows, then up rows)
    w_down: list = field(default_factory=list)      # E+1 arrays [d, hid] float32


def draw_layer(d: int, h: int, *, E: int = N_ROUTED, seed: int = 0,
               bias_coef: float | None = None, shared_hidden: int | None = None,
               std: float = 0.02) -> LayerWeights:
    rng = np.random.Generator(np.random.PCG64(seed))
    sd = np.float32(std)
    w_router = rng.standard_normal((d, E), dtype=np.float32) * sd
    perm = rng.permutation(E)
    bias = None
    if bias_coef is not None:
        rank = np.empty(E, dtype=np.int64)
        rank[perm] = np.arange(E)
        bias = (bias_coef * np.log(1.0 / (rank + 1.0))).astype(np.float32)
    hs = h if shared_hidden is None else shared_hidden
    lw = LayerWeights(d=d, h=h, hs=hs, E=E, w_router=w_router, router_bias=bias)
    for g in range(E + 1):
        hid = h if g < E else hs
        gate = rng.standard_normal((hid, d), dtype=np.float32) * sd
        up = rng.standard_normal((hid, d), dtype=np.float32) * sd
        down = rng.standard_normal((d, hid), dtype=np.float32) * sd
        lw.w_gate_up.append(np.concatenate([gate, up], axis=0))
        lw.w_down.append(down)
    return lw


def draw_x(T: int, d: int, seed: int) -> np.ndarray:
    """Activations x[T, d] ~ N(0, 1), as BF16 bit patterns (uint16)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return f32_to_bf16_bits(rng.standard_normal((T, d), dtype=np.float32))


def workload_layer(w: Workload, layer: int = 0) -> LayerWeights:
    return draw_layer(w.d, w.h, E=w.E, seed=w.weight_seed + layer, bias_coef=w.bias_coef,
                      shared_hidden=w.shared_hidden)


def workload_x(w: Workload, step: int = 0, T: int | None = None) -> np.ndarray:
    return draw_x(w.T if T is None else T, w.d, w.x_seed + step)
