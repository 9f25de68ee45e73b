"""Seeded synthetic inputs for the flow-matching action-expert denoise loop.

This module is shared by the tests, the benchmark and the oracle's callers. It
draws random numbers and stores them in the input formats of the library (bf16
bit patterns for weights and the cached prefix K/V, fp32 for the action chunk).
It holds none of the method's arithmetic: no norm, no projection, no attention,
no quantiser.

Workload shapes follow the action expert of "LingBot-VLA on Thor (sm_110)"
(§1 Architecture / shapes: 36-layer expert, action chunk [1, 50, 75], 10/25/50
steps) and "LingBot-VLA v2 Examples" (50 x 55 chunk, 36-layer KV cache built per
request and reused by every denoise step).

Recipe (the pages print no inputs, so these are synthetic stand-ins):
  * weights ~ N(0, 0.02^2), drawn as fp32 normals, scaled in fp32, rounded to
    bf16 with round-to-nearest-even;
  * prefix K/V ~ N(0, 1), rounded to bf16 the same way;
  * x0 (the action chunk at t = 1) ~ N(0, 1) in fp32, not rounded.
Independent PCG64 streams are derived from one seed with
``np.random.SeedSequence([seed, stream])``: stream 0 = weights, 1 = prefix K/V,
2 = x0, 3 = the prefix K/V projection weights of the backbone, 4 = the prefix
hidden states those project.  Weight order: time_w1, time_w2, in_proj, out_proj, then per layer
(wq, wk, wv, wo, w_gate, w_up, w_down).  Prefix order: per layer K then V, each
[B, P, H_kv, hd].  Requests of a batch are drawn consecutively.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List

import numpy as np

TIME_DIM = 256          # width of the sinusoidal time feature
CHUNK_LEN = 50          # action horizon of every chunk

LAYER_KEYS = ("wq", "wk", "wv", "wo", "w_gate", "w_up", "w_down")


@dataclasses.dataclass(frozen=True)
class ExpertShape:
    """Shape of one action expert plus the workload knobs of one run."""
    n_layers: int
    d_model: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    d_ff: int
    action_dim: int
    prefix_len: int
    steps: int
    batch: int = 1
    chunk_len: int = CHUNK_LEN
    rms_eps: float = 1e-6
    rope_base: float = 10000.0
    weight_std: float = 0.02
    fp8: bool = False
    nvfp4_gu: bool = False     # E4M3 linears with an NVFP4 gate_up
    w8a8: bool = False         # E4M3 linears and per-token E4M3 linear inputs (batched path)

    @property
    def n_mod(self) -> int:
        """Modulation width: six d-wide vectors per layer plus a final pair."""
        return self.n_layers * 6 * self.d_model + 2 * self.d_model

    def weight_shapes(self) -> Dict[str, tuple]:
        d, hd = self.d_model, self.head_dim
        return {
            "time_w1": (d, TIME_DIM),
            "time_w2": (self.n_mod, d),
            "in_proj": (d, self.action_dim),
            "out_proj": (self.action_dim, d),
            "wq": (self.n_q_heads * hd, d),
            "wk": (self.n_kv_heads * hd, d),
            "wv": (self.n_kv_heads * hd, d),
            "wo": (d, self.n_q_heads * hd),
            "w_gate": (self.d_ff, d),
            "w_up": (self.d_ff, d),
            "w_down": (d, self.d_ff),
        }

    def weight_bytes_per_step(self, bytes_per_weight: float = 2.0) -> float:
        s = self.weight_shapes()
        per_layer = sum(int(np.prod(s[k])) for k in LAYER_KEYS)
        io = int(np.prod(s["in_proj"])) + int(np.prod(s["out_proj"]))
        return self.n_layers * per_layer * bytes_per_weight + io * 2.0


# Named workloads. Sizes follow the expert of the pages (36 layers, d 1024,
# 16/2 heads of 128, SwiGLU 4096, chunk 50 x 75 or 50 x 55).
WORKLOADS: Dict[str, ExpertShape] = {
    # 2 layers, d 256: small enough for a pure fp32/fp64 CPU check.
    "tiny": ExpertShape(2, 256, 4, 1, 64, 1024, 75, 64, 10),
    # LingBot-VLA-shaped expert, bf16, P = 256 (3 views x 64 patches + 64 text).
    "lingbot_p256_n10": ExpertShape(36, 1024, 16, 2, 128, 4096, 75, 256, 10),
    # Longer prefix, 50 steps, v2 action dim 55.
    "lingbot_p832_n50_a55": ExpertShape(36, 1024, 16, 2, 128, 4096, 55, 832, 50),
    # FP8 E4M3 per-output-channel weights, bf16 activations and KV.
    "lingbot_fp8_p256_n10": ExpertShape(36, 1024, 16, 2, 128, 4096, 75, 256, 10, fp8=True),
    # E4M3 linears with an NVFP4 gate_up (the Thor page's weight formats).
    "lingbot_nvfp4_p256_n10": ExpertShape(36, 1024, 16, 2, 128, 4096, 75, 256, 10, nvfp4_gu=True),
    # 64 independent requests on one GPU.
    "lingbot_b64_p256_n10": ExpertShape(36, 1024, 16, 2, 128, 4096, 75, 256, 10, batch=64),
    # Four layers of the LingBot-shaped expert: the profiling case (same layer
    # shape, ~200 MB on the device, weights still larger than L2).
    "lingbot_l4_p256_n10": ExpertShape(4, 1024, 16, 2, 128, 4096, 75, 256, 10),
    # The same four layers with 64 requests: the profiling case of the batched path.
    "lingbot_l4_b64_p256_n10": ExpertShape(4, 1024, 16, 2, 128, 4096, 75, 256, 10, batch=64),
    # 64 requests with E4M3 weights and per-token E4M3 activations (W8A8).
    "lingbot_w8a8_b64_p256_n10": ExpertShape(36, 1024, 16, 2, 128, 4096, 75, 256, 10, batch=64, w8a8=True),
    # Its four-layer profiling case.
    "lingbot_l4_w8a8_b64_p256_n10": ExpertShape(4, 1024, 16, 2, 128, 4096, 75, 256, 10, batch=64, w8a8=True),
}


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even); return the bit patterns."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to fp32 (exact)."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _stream(seed: int, stream: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, stream])))


def _bf16_normal(rng: np.random.Generator, shape, std: float) -> np.ndarray:
    x = rng.standard_normal(int(np.prod(shape)), dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return f32_to_bf16_bits(x).reshape(shape)


def make_weights(shape: ExpertShape, seed: int = 0, std: float | None = None) -> Dict:
    """All weights as bf16 bit arrays [out, in].

    Returns {"time_w1", "time_w2", "in_proj", "out_proj": arrays,
             "layers": [ {wq, wk, wv, wo, w_gate, w_up, w_down} ] }.
    """
    std = shape.weight_std if std is None else std
    rng = _stream(seed, 0)
    ws = shape.weight_shapes()
    out: Dict = {}
    for k in ("time_w1", "time_w2", "in_proj", "out_proj"):
        out[k] = _bf16_normal(rng, ws[k], std)
    layers: List[Dict[str, np.ndarray]] = []
    for _ in range(shape.n_layers):
        layers.append({k: _bf16_normal(rng, ws[k], std) for k in LAYER_KEYS})
    out["layers"] = layers
    return out


def make_prefix(shape: ExpertShape, seed: int = 0, batch: int | None = None,
                prefix_len: int | None = None):
    """Cached prefix K and V per layer, bf16 bits [B, P, H_kv, hd] (N(0,1))."""
    B = shape.batch if batch is None else batch
    P = shape.prefix_len if prefix_len is None else prefix_len
    rng = _stream(seed, 1)
    kshape = (B, P, shape.n_kv_heads, shape.head_dim)
    ks, vs = [], []
    for _ in range(shape.n_layers):
        ks.append(_bf16_normal(rng, kshape, 1.0))
        vs.append(_bf16_normal(rng, kshape, 1.0))
    return ks, vs


def make_prefix_builder(shape: ExpertShape, d_prefix: int, seed: int = 0):
    """Per-layer prefix K/V projection weights of the backbone: bf16 bits
    [H_kv * hd, d_prefix] each, N(0, 0.02^2); stream 3, layer by layer (wk, wv)."""
    rng = _stream(seed, 3)
    rows = shape.n_kv_heads * shape.head_dim
    return [(_bf16_normal(rng, (rows, d_prefix), shape.weight_std),
             _bf16_normal(rng, (rows, d_prefix), shape.weight_std)) for _ in range(shape.n_layers)]


def make_prefix_hidden(shape: ExpertShape, d_prefix: int, seed: int = 0, batch: int | None = None,
                       prefix_len: int | None = None):
    """Per-layer prefix hidden states, bf16 bits [B, P, d_prefix] ~ N(0, 1); stream 4."""
    B = shape.batch if batch is None else batch
    P = shape.prefix_len if prefix_len is None else prefix_len
    rng = _stream(seed, 4)
    return [_bf16_normal(rng, (B, P, d_prefix), 1.0) for _ in range(shape.n_layers)]


def make_x0(shape: ExpertShape, seed: int = 0, batch: int | None = None) -> np.ndarray:
    """Action chunk at t = 1: fp32 [B, chunk_len, action_dim] ~ N(0, 1)."""
    B = shape.batch if batch is None else batch
    rng = _stream(seed, 2)
    return rng.standard_normal((B, shape.chunk_len, shape.action_dim), dtype=np.float32)
