"""Seeded synthetic inputs for the packed-MXFP4 MoE expert FFN.

This module only draws random numbers and lays them out in the storage
formats of the path (packed E2M1 bytes, E8M0 exponent bytes, BF16 bit
patterns). It holds none of the method's arithmetic: no dequantisation, no
dot products, no routing, no rounding points of the FFN. Both the CPU oracle
(``oracle/``) and the CUDA path are fed from here, and nothing here imports
either of them.

Workloads (shapes from the model cards):

* ``tiny``      H=512,  I=384,  E=16, top-4, T=4.
* ``layer24b``  H=2048, I=1536, E=64, top-4, T=1: one MoE layer of
  LFM2.5-24B-A2B (hidden 2048, MoE intermediate 1536, 64 experts, top-4;
  "LFM2.5-24B-A2B on Your Own Hardware", section "Where do the 2.45B active
  parameters actually go?").
* ``stack24b``  38 such layers (the 38 MoE layers of the 40-layer model,
  "LFM2.5-24B-A2B — Packed MXFP4 Inference", table "Model and quantization").
* ``stack8b``   22 layers of E=32, H=2048, I=1536, router bias ~N(0,1)
  (the 8B-A1B family: 24 layers, the first two dense, 32-expert top-4 MoE
  after them; "LFM2.5-8B-A1B — Core AI", introduction).
* ``batched``   the 24B layer shape at T in {32, 64, 256} with externally
  drawn routing (uniform or Zipf(1.1) expert popularity).

Distributions: packed codes uniform over the 16 E2M1 nibble values (so each
byte is uniform over 0..255), E8M0 exponents uniform integers in [118, 124],
activations N(0, 1) rounded to BF16, router weights N(0, 0.02) rounded to
BF16.

Storage layout (the checkpoint's "custom packed layout" is not specified on
the model card; this is the layout the whole repository uses):

* codes  uint8 [E][3][rows][K/2]; matrix 0 = gate (rows=I, K=H),
  1 = up (rows=I, K=H), 2 = down (rows=H, K=I). Element 2i of a row is the
  low nibble of byte i, element 2i+1 the high nibble.
* scales uint8 [E][3][rows][K/32]; one E8M0 exponent per 32 consecutive
  K elements of a row.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

E8M0_LO, E8M0_HI = 118, 124


@dataclass(frozen=True)
class LayerShape:
    E: int
    H: int
    I: int
    top_k: int = 4

    @property
    def codes_per_matrix(self) -> int:
        return self.I * self.H // 2

    @property
    def scales_per_matrix(self) -> int:
        return self.I * self.H // 32

    @property
    def codes_per_expert(self) -> int:
        return 3 * self.codes_per_matrix

    @property
    def scales_per_expert(self) -> int:
        return 3 * self.scales_per_matrix


TINY = LayerShape(E=16, H=512, I=384, top_k=4)
L24B = LayerShape(E=64, H=2048, I=1536, top_k=4)
L8B = LayerShape(E=32, H=2048, I=1536, top_k=4)

WORKLOADS = {
    "tiny": dict(shape=TINY, layers=1, T=4, bias=False),
    "layer24b": dict(shape=L24B, layers=1, T=1, bias=False),
    "stack24b": dict(shape=L24B, layers=38, T=1, bias=False),
    "stack8b": dict(shape=L8B, layers=22, T=1, bias=True),
    "batched32": dict(shape=L24B, layers=1, T=32, bias=False),
    "prefill64": dict(shape=L24B, layers=1, T=64, bias=False),
    "batched256": dict(shape=L24B, layers=1, T=256, bias=False),
}


def rng_for(seed: int, *stream: int) -> np.random.Generator:
    """Independent, reproducible generator for (seed, stream...) (SFC64 bit
    generator seeded through a SeedSequence)."""
    return np.random.Generator(np.random.SFC64(np.random.SeedSequence([seed, *stream])))


def uniform_bytes(n: int, rng: np.random.Generator) -> np.ndarray:
    """n independent bytes uniform over 0..255."""
    words = rng.integers(0, 2 ** 64 - 1, size=(n + 7) // 8, dtype=np.uint64, endpoint=True)
    return words.view(np.uint8)[:n]


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to BF16 (round to nearest even); return the bits.

    Used only to store generated activations/router weights in BF16.
    """
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    nan = np.isnan(a)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)
    r[nan] = 0x7FC0
    return r


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def make_expert_weights(shape: LayerShape, rng: np.random.Generator):
    """Packed codes and E8M0 scales for all E experts of one layer.

    Returns (codes uint8 [E, 3*I*H/2], scales uint8 [E, 3*I*H/32]).
    """
    n_codes = shape.E * shape.codes_per_expert
    codes = uniform_bytes(n_codes, rng).reshape(shape.E, shape.codes_per_expert)
    scales = rng.integers(E8M0_LO, E8M0_HI + 1,
                          size=(shape.E, shape.scales_per_expert),
                          dtype=np.uint8)
    return codes, scales


def make_expert_weights_nvfp4(shape: LayerShape, rng: np.random.Generator):
    """NVFP4 experts of one layer: packed E2M1 codes (uniform bytes), one FP8
    E4M3 block scale per 16 K elements (positive normal values 2^-6 .. 1.875,
    uniform over exponent fields 1..7 and the 8 mantissas), and per expert two
    FP32 multipliers uniform in [0.01, 0.02] (gate/up shared, down).

    Returns (codes uint8 [E, 3*I*H/2], scales uint8 [E, 3*I*H/16],
    gscales float32 [E, 2]).
    """
    n_codes = shape.E * shape.codes_per_expert
    codes = uniform_bytes(n_codes, rng).reshape(shape.E, shape.codes_per_expert)
    n_sc = 3 * shape.I * shape.H // 16
    ex = rng.integers(1, 8, size=(shape.E, n_sc), dtype=np.uint8)
    man = rng.integers(0, 8, size=(shape.E, n_sc), dtype=np.uint8)
    scales = ((ex << 3) | man).astype(np.uint8)
    gscales = rng.uniform(0.01, 0.02, size=(shape.E, 2)).astype(np.float32)
    return codes, scales, gscales


def make_expert_weights_sym8(shape: LayerShape, rng: np.random.Generator):
    """sym8 experts of one layer: one int8 weight per element, uniform over
    the symmetric grid -127 .. 127, and one IEEE binary16 block scale per 32
    K elements, positive normal values 2^-13 .. 2^-9 (exponent fields 2..5,
    uniform 10-bit mantissas), so |w| <= 127 * 2^-9.

    Returns (q int8 [E, 3*I*H], scales uint16 [E, 3*I*H/32] binary16 bits).
    """
    n = 3 * shape.I * shape.H
    q = rng.integers(-127, 128, size=(shape.E, n), dtype=np.int16).astype(np.int8)
    ex = rng.integers(2, 6, size=(shape.E, n // 32), dtype=np.uint16)
    man = rng.integers(0, 1024, size=(shape.E, n // 32), dtype=np.uint16)
    scales = ((ex << 10) | man).astype(np.uint16)
    return q, scales


def make_activations(T: int, H: int, rng: np.random.Generator) -> np.ndarray:
    """x ~ N(0, 1) in BF16 bits, [T, H]."""
    return f32_to_bf16_bits(rng.standard_normal((T, H), dtype=np.float32))


def make_router(shape: LayerShape, rng: np.random.Generator) -> np.ndarray:
    """Router weight ~ N(0, 0.02) in BF16 bits, [E, H]."""
    w = rng.standard_normal((shape.E, shape.H), dtype=np.float32) * np.float32(0.02)
    return f32_to_bf16_bits(w)


def make_router_bias(shape: LayerShape, rng: np.random.Generator) -> np.ndarray:
    """Per-expert logit bias ~ N(0, 1), float32 [E] (skews expert popularity)."""
    return rng.standard_normal(shape.E).astype(np.float32)


def zipf_probs(E: int, s: float, rng: np.random.Generator) -> np.ndarray:
    """Zipf(s) popularity over E experts, assigned to experts by a random rank
    permutation."""
    p_rank = 1.0 / np.arange(1, E + 1, dtype=np.float64) ** s
    p_rank /= p_rank.sum()
    perm = rng.permutation(E)
    p = np.empty(E)
    p[perm] = p_rank
    return p


def make_routing(T: int, E: int, k: int, dist: str, rng: np.random.Generator):
    """Externally drawn routing for the batched workloads.

    Each token gets k distinct experts sampled without replacement from a
    uniform or Zipf(1.1) popularity; its k positive weights are normalised
    exponential draws sorted in descending order (slot 0 heaviest).
    Returns (ids int32 [T, k], w float32 [T, k]).
    """
    if dist == "uniform":
        p = None
    elif dist == "zipf":
        p = zipf_probs(E, 1.1, rng)
    else:
        raise ValueError(f"unknown routing distribution {dist!r}")
    ids = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float32)
    for t in range(T):
        ids[t] = rng.choice(E, size=k, replace=False, p=p)
        g = rng.exponential(size=k)
        g = np.sort(g / g.sum())[::-1]
        w[t] = g.astype(np.float32)
    return ids, w


@dataclass
class LayerInputs:
    shape: LayerShape
    codes: np.ndarray      # uint8 [E, 3*I*H/2]
    scales: np.ndarray     # uint8 [E, 3*I*H/32]
    router_w: np.ndarray   # uint16 (bf16) [E, H]
    router_b: np.ndarray | None  # float32 [E] or None
    gscales: np.ndarray | None = None  # NVFP4: float32 [E, 2]; scales are E4M3 [E, 3*I*H/16]
    fmt: str = "mxfp4"  # "mxfp4", "nvfp4" or "sym8" (codes int8 [E, 3*I*H], scales binary16 [E, 3*I*H/32])


def make_layer(shape: LayerShape, seed: int, layer: int = 0,
               bias: bool = False) -> LayerInputs:
    rng = rng_for(seed, 1, layer)
    codes, scales = make_expert_weights(shape, rng)
    router_w = make_router(shape, rng)
    router_b = make_router_bias(shape, rng) if bias else None
    return LayerInputs(shape, codes, scales, router_w, router_b)


def make_layer_nvfp4(shape: LayerShape, seed: int, layer: int = 0,
                     bias: bool = False) -> LayerInputs:
    rng = rng_for(seed, 5, layer)
    codes, scales, gscales = make_expert_weights_nvfp4(shape, rng)
    router_w = make_router(shape, rng)
    router_b = make_router_bias(shape, rng) if bias else None
    return LayerInputs(shape, codes, scales, router_w, router_b, gscales, fmt="nvfp4")


def make_layer_sym8(shape: LayerShape, seed: int, layer: int = 0,
                    bias: bool = False) -> LayerInputs:
    rng = rng_for(seed, 6, layer)
    q, scales = make_expert_weights_sym8(shape, rng)
    router_w = make_router(shape, rng)
    router_b = make_router_bias(shape, rng) if bias else None
    return LayerInputs(shape, q, scales, router_w, router_b, fmt="sym8")


def make_tokens(T: int, H: int, seed: int, stream: int = 0) -> np.ndarray:
    return make_activations(T, H, rng_for(seed, 2, stream))
