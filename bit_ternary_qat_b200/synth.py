"""Seeded synthetic inputs for the BitLinear hot path.

This module only draws random tensors with the shapes, dtypes and value
distributions of the five workloads below. It contains none of the layer's
arithmetic (no normalisation, no quantisation, no contraction), so both the
CUDA path and the CPU oracle can take their inputs from it without sharing
any of the method's code.

Every tensor is generated on the CPU with ``torch.Generator().manual_seed``
and then (for bf16 workloads) cast to bf16, so every consumer sees the same
bytes for the same seed.

Workloads (shapes follow the layer's nn.Linear convention: W is [d_out, d_in],
X is [tokens, d_in]):

* ``single``   - one BitLinear, X 64x256 fp32 ~N(0,1), W 512x256 fp32 ~N(0,0.02^2),
                 dY 64x512 fp32 ~N(0,1), gain 1, eps 1e-6, seed 0.
* ``square``   - one BitLinear, 4096 tokens, d_in = d_out = 2048, X bf16 ~N(0,1),
                 W fp32 ~N(0,0.02^2), dY bf16 ~N(0,(1e-2)^2), seed 2.
* ``mlp7b``    - two BitLinears of a 7B-shaped MLP (4096->11008 and 11008->4096),
                 8192 tokens, X bf16 ~N(0,1) (independent per layer),
                 W = 0.02 * StudentT(df=3), dY bf16 ~N(0,(1e-2)^2), seed 3.
* ``decode``   - packed-ternary decode GEMV, W 28672x8192 fp32 ~N(0,0.02^2),
                 activations [B x 8192] ~N(0,1) for B in (1, 4, 16), seed 4.
* ``layer7b``  - the seven projections of a 7B-shaped transformer layer
                 (q,k,v,o 4096x4096; gate, up 11008x4096; down 4096x11008),
                 16384 tokens, bf16 X and dY as in ``square``, seed 5.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional, Tuple

import torch

RMS_EPS = 1e-6
W_STD = 0.02
DY_STD_BF16 = 1e-2


@dataclass(frozen=True)
class LayerShape:
    """One BitLinear: ``d_out`` x ``d_in`` weight applied to ``tokens`` rows."""
    name: str
    tokens: int
    d_in: int
    d_out: int


@dataclass(frozen=True)
class Workload:
    name: str
    seed: int
    dtype: str                      # "f32" or "bf16" for X / dY / Y
    layers: Tuple[LayerShape, ...]
    w_dist: str = "normal"          # "normal" or "student_t3"
    dy_std: float = DY_STD_BF16
    decode_batches: Tuple[int, ...] = ()
    description: str = ""


WORKLOADS = {
    "single": Workload(
        "single", 0, "f32", (LayerShape("linear", 64, 256, 512),), dy_std=1.0,
        description="single BitLinear 256->512, 64 tokens, fp32"),
    "square": Workload(
        "square", 2, "bf16", (LayerShape("linear", 4096, 2048, 2048),),
        description="BitLinear 2048->2048, 4096 tokens, bf16 X/dY"),
    "mlp7b": Workload(
        "mlp7b", 3, "bf16",
        (LayerShape("up", 8192, 4096, 11008), LayerShape("down", 8192, 11008, 4096)),
        w_dist="student_t3",
        description="7B-shaped MLP BitLinears 4096->11008->4096, 8192 tokens, bf16"),
    "decode": Workload(
        "decode", 4, "f32", (LayerShape("decode", 16, 8192, 28672),),
        decode_batches=(1, 4, 16),
        description="packed-ternary decode GEMV, W 28672x8192, batch 1/4/16"),
    "layer7b": Workload(
        "layer7b", 5, "bf16",
        (LayerShape("q", 16384, 4096, 4096), LayerShape("k", 16384, 4096, 4096),
         LayerShape("v", 16384, 4096, 4096), LayerShape("o", 16384, 4096, 4096),
         LayerShape("gate", 16384, 4096, 11008), LayerShape("up", 16384, 4096, 11008),
         LayerShape("down", 16384, 11008, 4096)),
        description="all 7 projections of a 7B-shaped layer, 16384 tokens, bf16"),
}


def generator(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def normal(shape, std: float, gen: torch.Generator) -> torch.Tensor:
    return torch.randn(*shape, generator=gen, dtype=torch.float32) * std


def student_t3(shape, scale: float, gen: torch.Generator) -> torch.Tensor:
    """scale * Z / sqrt(V/3), Z ~ N(0,1), V ~ chi^2(3) drawn as a sum of three squared normals."""
    z = torch.randn(*shape, generator=gen, dtype=torch.float32)
    v = torch.zeros(*shape, dtype=torch.float32)
    for _ in range(3):
        e = torch.randn(*shape, generator=gen, dtype=torch.float32)
        v += e * e
    return (z / torch.sqrt(v / 3.0)) * scale


def to_dtype(t: torch.Tensor, dtype: str) -> torch.Tensor:
    if dtype == "bf16":
        return t.to(torch.bfloat16)
    if dtype == "f32":
        return t
    raise ValueError(dtype)


@dataclass
class LayerInputs:
    shape: LayerShape
    X: torch.Tensor       # [tokens, d_in], workload dtype
    W: torch.Tensor       # [d_out, d_in], fp32 latent weights
    dY: torch.Tensor      # [tokens, d_out], workload dtype
    g: Optional[torch.Tensor] = None   # RMSNorm gain, None = all ones


def layer_inputs(wl: Workload, layer: LayerShape, gen: torch.Generator,
                 tokens: Optional[int] = None) -> LayerInputs:
    t = layer.tokens if tokens is None else tokens
    if wl.w_dist == "student_t3":
        W = student_t3((layer.d_out, layer.d_in), W_STD, gen)
    else:
        W = normal((layer.d_out, layer.d_in), W_STD, gen)
    X = to_dtype(normal((t, layer.d_in), 1.0, gen), wl.dtype)
    dY = to_dtype(normal((t, layer.d_out), wl.dy_std, gen), wl.dtype)
    return LayerInputs(layer, X, W, dY, None)


def workload_inputs(name: str, tokens: Optional[int] = None, first: Optional[int] = None) -> List[LayerInputs]:
    """Inputs of every layer of a workload (or of its first `first` layers: the draws are
    sequential, so these equal the leading layers of the full list)."""
    wl = WORKLOADS[name]
    gen = generator(wl.seed)
    layers = wl.layers if first is None else wl.layers[:first]
    return [layer_inputs(wl, ly, gen, tokens) for ly in layers]


def decode_inputs(batch: int, d_out: int = 28672, d_in: int = 8192, seed: int = 4):
    """Latent weight [d_out, d_in] ~N(0,0.02^2) and activations [batch, d_in] ~N(0,1)."""
    gen = generator(seed)
    W = normal((d_out, d_in), W_STD, gen)
    x = normal((batch, d_in), 1.0, gen)
    return W, x


def random_case(T: int, K: int, N: int, seed: int, dtype: str = "bf16",
                w_dist: str = "normal", dy_std: float = DY_STD_BF16,
                with_gain: bool = False) -> LayerInputs:
    """A generic seeded case of arbitrary (ragged) size, for parity tests."""
    wl = Workload("case", seed, dtype, (LayerShape("case", T, K, N),), w_dist=w_dist, dy_std=dy_std)
    gen = generator(seed)
    li = layer_inputs(wl, wl.layers[0], gen)
    if with_gain:
        li.g = 1.0 + 0.25 * torch.randn(K, generator=gen, dtype=torch.float32)
    return li
