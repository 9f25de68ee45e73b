"""CPU oracle for the flow-matching action-expert denoise loop.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this module.  The library never calls
it, and it shares no code, table or constant generator with the CUDA path.

This is a plain, slow, fp64 (optionally fp32) restatement of what the denoise
loop computes, written from the pages' description of the action expert:

* "LingBot-VLA on Thor (sm_110)", §1 Architecture / shapes: a 36-layer
  flow-matching action expert runs a per-step denoise loop over an action
  chunk [1, 50, 75] with 10 / 25 / 50 steps.
* same page, §2 Build: the expert's own kernels are a fused AdaRMSNorm, a
  SwiGLU tail and QKV + RoPE; §3 FlashAttention-4: the denoise attention is
  grouped-query attention (``pack_gqa``).
* "LingBot-VLA v2 Examples", Configuration / CUDA Graph: the 36-layer prefix
  KV cache is built once per request and reused by every fixed-shape
  denoising step; the chunk is 50 x 55.

The pages print no formula, so the conventions below are the plainest readings
(each one is listed, with its reason, in the design notes of the repository):

  R1 time feature: 256 dims, [sin(2 pi t / p_i)] ++ [cos(2 pi t / p_i)],
     periods p_i geometric from 4e-3 to 4 (i = 0..127).
  R2 time MLP: exactly two bias-free linears with SiLU between them:
     m = SiLU(e W1^T) W2^T, split per layer into (s_a, b_a, g_a, s_f, b_f, g_f)
     then a final (s_o, b_o).
  R3 AdaRMSNorm: y = x (mean(x^2) + eps)^(-1/2) (1 + s) + b, no learned gain;
     gated residual h <- h + g * f(y).
  R4 RoPE: rotate-half pairs (j, j + hd/2), theta_j = base^(-2j/hd), applied to
     q and to the chunk's k at positions P .. P + T - 1; the cached prefix K is
     already rotated.
  R5 GQA: query head h reads KV head floor(h / (H_q / H_kv)); scale 1/sqrt(hd);
     no mask (the chunk attends to the whole prefix and to itself).
  R6 Euler from t = 1 to t = 0: t_k = 1 - k/n, dt = -1/n, x <- x + dt v(x, t_k).
  R7 in-proj and out-proj are bias-free; h is rebuilt from x every step; a final
     AdaRMSNorm (s_o, b_o), ungated, precedes the out-proj.  ``out_bias`` exists
     only to build a constant velocity field in tests.
  R8 FP8 weights: per output row c, s_c = absmax_c / 448 (fp32), q = E4M3
     nearest-even of (w / s_c) in fp32, saturated at 448; w' = q * s_c.
  R9 prefix cache rows: K = RoPE(x Wk^T) at positions 0 .. P-1, V = x Wv^T
     from each layer's prefix hidden states x, stored as bf16.
  R10 NVFP4 gate_up (with E4M3 R8 for the other linears): per tensor
     g = amax / (6 * 448) (fp32); per row and 16-column block
     s_b = E4M3 nearest-even of (amax_b / (6 g)) in fp32; codes = E2M1
     nearest-even of (w / (s_b g)) in fp32, saturated at 6; w' = q s_b g.
  R11 E4M3 activations (the batched path's W8A8 option; the pages fix FP8
     linears but no activation quantiser): each input row of the four
     per-layer linears, taken in fp32, is quantised per token with
     r = 448 / amax_row and s = amax_row / 448 (both fp32, 1 for a zero row):
     codes = E4M3(y r) with the product in fp32, y' = codes s (the cast
     multiplies by the fp32 factor fp8_max / amax, as the public FP8 recipes
     do, e.g. NVIDIA Transformer Engine's scale = fp8_max / amax).

Every function below is pinned by ``tests/test_oracle_pins.py`` against closed
forms, hand values, brute force or independent library routines.
"""
from __future__ import annotations

import math
from typing import Callable, Dict, List, Optional

import numpy as np

TIME_DIM = 256
MIN_PERIOD = 4e-3
MAX_PERIOD = 4.0
E4M3_MAX = 448.0


# ----------------------------------------------------------------------------
# input decoding (the oracle's own copy; it does not use the library's)
# ----------------------------------------------------------------------------
def decode_bf16(bits: np.ndarray, dtype=np.float64) -> np.ndarray:
    """bf16 bit patterns -> floating values (exact widening)."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(dtype)


# ----------------------------------------------------------------------------
# time conditioning (R1, R2)
# ----------------------------------------------------------------------------
def time_schedule(n: int):
    """Euler grid of R6: times t_0..t_{n-1} (t_k = 1 - k/n) and the step dt."""
    if n <= 0:
        raise ValueError("n must be positive")
    ts = np.array([1.0 - k / n for k in range(n)], dtype=np.float64)
    return ts, -1.0 / n


def sinusoid(t: np.ndarray, dim: int = TIME_DIM, dtype=np.float64) -> np.ndarray:
    """Sinusoidal time feature of R1 for each time in ``t`` -> [len(t), dim]."""
    half = dim // 2
    frac = np.arange(half, dtype=np.float64) / (half - 1)
    period = MIN_PERIOD * (MAX_PERIOD / MIN_PERIOD) ** frac
    ang = 2.0 * math.pi * np.asarray(t, dtype=np.float64)[:, None] / period[None, :]
    return np.concatenate([np.sin(ang), np.cos(ang)], axis=1).astype(dtype)


def silu(x: np.ndarray) -> np.ndarray:
    """SiLU(x) = x * sigmoid(x)."""
    return x / (1.0 + np.exp(-x))


def time_modulation(ts: np.ndarray, w1: np.ndarray, w2: np.ndarray, dtype=np.float64) -> np.ndarray:
    """Modulation rows m_k = SiLU(e_k W1^T) W2^T for every time t_k (R2)."""
    e = sinusoid(ts, w1.shape[1], dtype)
    h1 = silu(e @ w1.T)
    return h1 @ w2.T


def split_modulation(m: np.ndarray, n_layers: int, d: int):
    """Cut one modulation row into per-layer (s_a, b_a, g_a, s_f, b_f, g_f) and (s_o, b_o)."""
    per = [tuple(m[(6 * l + i) * d:(6 * l + i + 1) * d] for i in range(6)) for l in range(n_layers)]
    base = 6 * n_layers * d
    return per, (m[base:base + d], m[base + d:base + 2 * d])


# ----------------------------------------------------------------------------
# per-op definitions (R3, R4, R5)
# ----------------------------------------------------------------------------
def ada_rms(x: np.ndarray, s: np.ndarray, b: np.ndarray, eps: float) -> np.ndarray:
    """AdaRMSNorm of R3 over the last axis."""
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * (1.0 + s) + b


def rope(x: np.ndarray, pos: np.ndarray, base: float) -> np.ndarray:
    """Rotate-half rotary embedding of R4.  x: [T, H, hd], pos: [T]."""
    hd = x.shape[-1]
    half = hd // 2
    theta = base ** (-2.0 * np.arange(half, dtype=np.float64) / hd)
    ang = np.asarray(pos, dtype=np.float64)[:, None] * theta[None, :]
    c = np.cos(ang)[:, None, :].astype(x.dtype)
    s = np.sin(ang)[:, None, :].astype(x.dtype)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def softmax(z: np.ndarray) -> np.ndarray:
    """Max-subtracted softmax over the last axis."""
    z = z - np.max(z, axis=-1, keepdims=True)
    e = np.exp(z)
    return e / np.sum(e, axis=-1, keepdims=True)


def gqa_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray) -> np.ndarray:
    """Grouped-query attention of R5.

    q: [T, H_q, hd]; k, v: [S, H_kv, hd] -> o: [T, H_q, hd]; no mask.
    """
    T, Hq, hd = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    o = np.empty_like(q)
    for h in range(Hq):
        g = h // G
        p = softmax((q[:, h, :] @ k[:, g, :].T) / math.sqrt(hd))
        o[:, h, :] = p @ v[:, g, :]
    return o


# ----------------------------------------------------------------------------
# the expert
# ----------------------------------------------------------------------------
class Weights:
    """Decoded weights of one expert (float arrays, [out, in])."""

    def __init__(self, raw: Dict, dtype=np.float64, fp8: bool = False, nvfp4_gu: bool = False):
        self.dtype = dtype
        self.time_w1 = decode_bf16(raw["time_w1"], dtype)
        self.time_w2 = decode_bf16(raw["time_w2"], dtype)
        self.in_proj = decode_bf16(raw["in_proj"], dtype)
        self.out_proj = decode_bf16(raw["out_proj"], dtype)
        self.layers: List[Dict[str, np.ndarray]] = []
        for lw in raw["layers"]:
            d = {}
            for key, bits in lw.items():
                w = decode_bf16(bits, np.float64)
                if nvfp4_gu and key in ("w_gate", "w_up"):
                    w = nvfp4_dequantize(*nvfp4_quantize(bits))
                elif fp8 or nvfp4_gu:
                    codes, scale = fp8_quantize_rows(bits)
                    w = fp8_dequantize_rows(codes, scale)
                d[key] = w.astype(dtype)
            self.layers.append(d)


def expert_velocity(x: np.ndarray, m: np.ndarray, W: Weights, k_prefix: List[np.ndarray],
                    v_prefix: List[np.ndarray], eps: float, rope_base: float,
                    n_q_heads: int, n_kv_heads: int, out_bias: Optional[np.ndarray] = None,
                    trace: Optional[List[Dict[str, np.ndarray]]] = None, act_fp8: bool = False) -> np.ndarray:
    """Velocity v(x, t) of one request's chunk.

    x: [T, A]; m: modulation row for this t; k_prefix / v_prefix: per layer
    [P, H_kv, hd] (already rotated).  If ``trace`` is a list, one dict of
    intermediates per layer is appended, then a final dict.  ``act_fp8``
    quantises the input rows of the four per-layer linears per token (R11).
    """
    aq = fp8_quant_act if act_fp8 else (lambda a: a)
    dt_ = W.dtype
    T = x.shape[0]
    L = len(W.layers)
    d = W.in_proj.shape[0]
    per, (s_o, b_o) = split_modulation(m.astype(dt_), L, d)
    h = x.astype(dt_) @ W.in_proj.T
    for l, lw in enumerate(W.layers):
        s_a, b_a, g_a, s_f, b_f, g_f = per[l]
        kp = k_prefix[l].astype(dt_)
        vp = v_prefix[l].astype(dt_)
        P, _, hd = kp.shape
        rec = {"h_in": h.copy()} if trace is not None else None
        y = aq(ada_rms(h, s_a, b_a, eps))
        q = (y @ lw["wq"].T).reshape(T, n_q_heads, hd)
        kc = (y @ lw["wk"].T).reshape(T, n_kv_heads, hd)
        vc = (y @ lw["wv"].T).reshape(T, n_kv_heads, hd)
        pos = P + np.arange(T)
        q = rope(q, pos, rope_base)
        kc = rope(kc, pos, rope_base)
        K = np.concatenate([kp, kc], axis=0)
        V = np.concatenate([vp, vc], axis=0)
        o = gqa_attention(q, K, V).reshape(T, n_q_heads * hd)
        h = h + g_a * (aq(o) @ lw["wo"].T)
        if rec is not None:
            rec.update(q=q, k=kc, v=vc, o=o, h_mid=h.copy())
        y = aq(ada_rms(h, s_f, b_f, eps))
        u = silu(y @ lw["w_gate"].T) * (y @ lw["w_up"].T)
        h = h + g_f * (aq(u) @ lw["w_down"].T)
        if rec is not None:
            rec.update(u=u, h_out=h.copy())
            trace.append(rec)
    v = ada_rms(h, s_o, b_o, eps) @ W.out_proj.T
    if out_bias is not None:
        v = v + np.asarray(out_bias, dtype=dt_)
    if trace is not None:
        trace.append({"v": v})
    return v


def euler(x0: np.ndarray, n: int, velocity: Callable[[np.ndarray, int, float], np.ndarray],
          record: Optional[List[np.ndarray]] = None) -> np.ndarray:
    """Explicit Euler of R6: x <- x + dt * v(x, t_k) for k = 0..n-1."""
    ts, dt = time_schedule(n)
    x = np.array(x0, dtype=np.float64, copy=True)
    for k in range(n):
        v = velocity(x, k, ts[k])
        if record is not None:
            record.append(np.array(v, copy=True))
        x = x + dt * v
    return x


def denoise(x0: np.ndarray, n: int, raw_weights: Dict, k_prefix, v_prefix, shape,
            dtype=np.float64, out_bias=None, W: Optional[Weights] = None,
            velocities: Optional[List[np.ndarray]] = None, act_fp8: Optional[bool] = None) -> np.ndarray:
    """Denoise a batch of chunks: x0 [B, T, A] -> x_n [B, T, A].

    k_prefix / v_prefix: per layer bf16 bits [B, P, H_kv, hd].  All requests
    share the modulation rows (same t grid); each has its own prefix and x0.
    Without W, the weights follow the shape's formats; act_fp8 None follows
    the shape's W8A8 flag (R11).
    """
    w8a8 = bool(getattr(shape, "w8a8", False))
    if act_fp8 is None:
        act_fp8 = w8a8
    if W is None:
        W = Weights(raw_weights, dtype, fp8=shape.fp8 or w8a8, nvfp4_gu=bool(getattr(shape, "nvfp4_gu", False)))
    ts, _ = time_schedule(n)
    M = time_modulation(ts, W.time_w1, W.time_w2, dtype)
    x0 = np.asarray(x0, dtype=np.float64)
    out = np.empty_like(x0)
    for b in range(x0.shape[0]):
        kp = [decode_bf16(k[b], dtype) for k in k_prefix]
        vp = [decode_bf16(v[b], dtype) for v in v_prefix]

        def vel(x, k, t, kp=kp, vp=vp):
            return expert_velocity(x, M[k], W, kp, vp, shape.rms_eps, shape.rope_base,
                                   shape.n_q_heads, shape.n_kv_heads, out_bias, act_fp8=act_fp8).astype(np.float64)

        rec = [] if velocities is not None else None
        out[b] = euler(x0[b], n, vel, rec)
        if velocities is not None:
            velocities.append(rec)
    return out


# ----------------------------------------------------------------------------
# prefix K/V construction (R9)
# ----------------------------------------------------------------------------
def prefix_kv(x: np.ndarray, wk: np.ndarray, wv: np.ndarray, n_kv_heads: int, base: float):
    """R9: one layer's prefix cache rows from that layer's prefix hidden states
    ("LingBot-VLA v2 Examples", Configuration / CUDA Graph: the 36-layer
    KV-cache construction runs once per request before the denoise steps).

    x: [P, d_prefix]; wk, wv: [H_kv * hd, d_prefix].  K = RoPE(x Wk^T) at
    positions 0 .. P-1 (R4), V = x Wv^T; both [P, H_kv, hd].
    """
    P = x.shape[0]
    hd = wk.shape[0] // n_kv_heads
    k = (x @ wk.T).reshape(P, n_kv_heads, hd)
    v = (x @ wv.T).reshape(P, n_kv_heads, hd)
    return rope(k, np.arange(P), base), v


def bf16_round_bits(x: np.ndarray) -> np.ndarray:
    """Nearest-even bf16 bit patterns of float64 values (via their fp32
    rounding, as a kernel storing an fp32 result as bf16 does)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    return ((u + (((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF))) >> np.uint32(16)).astype(np.uint16)


# ----------------------------------------------------------------------------
# FP8 E4M3 weight quantiser (R8)
# ----------------------------------------------------------------------------
def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """E4M3 (no infinities, 0x7F / 0xFF = NaN) codes -> float64 values."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    mnt = c & 0x7
    val = np.where(e == 0, mnt * 2.0 ** -9, (1.0 + mnt / 8.0) * np.exp2(e - 7.0))
    val = np.where((c & 0x7F) == 0x7F, np.nan, val)
    return sign * val


def e4m3_encode(v: np.ndarray) -> np.ndarray:
    """Nearest E4M3 code (ties to even), saturating at +-448.  v: float32 values."""
    v = np.asarray(v, dtype=np.float32).astype(np.float64)
    sign = np.signbit(v)
    a = np.minimum(np.abs(v), E4M3_MAX)
    code = np.zeros(a.shape, dtype=np.int64)
    sub = a < 2.0 ** -6
    code[sub] = np.rint(a[sub] / 2.0 ** -9).astype(np.int64)          # 0..8, 8 == min normal
    nrm = ~sub
    if np.any(nrm):
        _, ex = np.frexp(a[nrm])           # a = f * 2^ex, f in [0.5, 1)
        e = ex - 1                         # a in [2^e, 2^(e+1))
        q = np.rint(a[nrm] / np.exp2(e - 3.0)).astype(np.int64)       # 8..16
        carry = q == 16
        e = np.where(carry, e + 1, e)
        q = np.where(carry, 8, q)
        code[nrm] = ((e + 7) << 3) | (q - 8)
    code = np.minimum(code, 0x7E)
    return (code | np.where(sign, 0x80, 0)).astype(np.uint8)


def fp8_quantize_rows(w_bits: np.ndarray):
    """R8 on bf16 weight bits [out, in] -> (codes uint8 [out, in], scale float32 [out])."""
    w = decode_bf16(w_bits, np.float32)
    amax = np.max(np.abs(w), axis=1).astype(np.float32)
    scale = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    ratio = (w / scale[:, None]).astype(np.float32)
    return e4m3_encode(ratio), scale


def fp8_quantize_act(y: np.ndarray):
    """R11: per-token E4M3 of activation rows (last axis) of the fp32 values:
    r = 448 / amax_row and s = amax_row / 448 in fp32 (both 1 for an all-zero
    row), codes = E4M3(y r) with the product in fp32.  Returns (codes uint8,
    s float32)."""
    y32 = np.asarray(y, dtype=np.float32)
    amax = np.max(np.abs(y32), axis=-1)
    nz = amax > 0
    safe = np.where(nz, amax, np.float32(1.0)).astype(np.float32)
    s = np.where(nz, safe / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    r = np.where(nz, np.float32(E4M3_MAX) / safe, np.float32(1.0)).astype(np.float32)
    codes = e4m3_encode((y32 * r[..., None]).astype(np.float32))
    return codes, s


def fp8_quant_act(y: np.ndarray) -> np.ndarray:
    """R11 as the linears see it: the rows quantised, returned dequantised in
    float64, y' = E4M3(y / s) s."""
    codes, s = fp8_quantize_act(y)
    return e4m3_decode(codes) * s[..., None].astype(np.float64)


def fp8_dequantize_rows(codes: np.ndarray, scale: np.ndarray) -> np.ndarray:
    """w' = decode(q) * s_c in float64."""
    return e4m3_decode(codes) * np.asarray(scale, dtype=np.float64)[:, None]


# ----------------------------------------------------------------------------
# NVFP4 weight quantiser (R10): E2M1 elements, 16-element E4M3 block scales,
# one fp32 scale per tensor
# ----------------------------------------------------------------------------
E2M1_VALUES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
NVFP4_BLOCK = 16


def e2m1_decode(codes: np.ndarray) -> np.ndarray:
    """4-bit E2M1 codes (bit 3 = sign) -> float64 values."""
    c = np.asarray(codes).astype(np.int64)
    return np.where(c & 8, -1.0, 1.0) * E2M1_VALUES[c & 7]


def e2m1_encode(v: np.ndarray) -> np.ndarray:
    """Nearest E2M1 code of fp32 values, ties to the even code, saturating at 6."""
    a = np.abs(np.asarray(v, dtype=np.float32).astype(np.float64))
    # distance to every magnitude; ties go to the even index
    d = np.abs(a[..., None] - E2M1_VALUES)
    best = np.zeros(a.shape, dtype=np.int64)
    bd = d[..., 0]
    for i in range(1, 8):
        take = (d[..., i] < bd) | ((d[..., i] == bd) & (i % 2 == 0))
        best = np.where(take, i, best)
        bd = np.where(take, d[..., i], bd)
    best = np.where(a >= 6.0, 7, best)
    sign = np.signbit(np.asarray(v, dtype=np.float32)) & (best > 0)
    return (best | np.where(sign, 8, 0)).astype(np.uint8)


def nvfp4_quantize(w_bits: np.ndarray):
    """R10 on bf16 weight bits [rows, K] (K a multiple of 16) ->
    (codes uint8 [rows, K] in 0..15, block scales uint8 E4M3 [rows, K/16], g float32)."""
    w = decode_bf16(w_bits, np.float32)
    rows, K = w.shape
    amax = np.float32(np.max(np.abs(w)))
    g = np.float32(amax / np.float32(6.0 * E4M3_MAX)) if amax > 0 else np.float32(1.0)
    blocks = w.reshape(rows, K // NVFP4_BLOCK, NVFP4_BLOCK)
    bmax = np.max(np.abs(blocks), axis=2).astype(np.float32)
    sb = e4m3_encode((bmax / (np.float32(6.0) * g)).astype(np.float32))
    sbv = e4m3_decode(sb).astype(np.float32)
    denom = (sbv * g).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = np.where(denom[:, :, None] > 0, (blocks / denom[:, :, None]).astype(np.float32), np.float32(0.0))
    codes = e2m1_encode(ratio).reshape(rows, K)
    return codes, sb, g


def nvfp4_dequantize(codes: np.ndarray, sb: np.ndarray, g) -> np.ndarray:
    """w' = e2m1(q) * e4m3(s_b) * g in float64."""
    rows, K = codes.shape
    q = e2m1_decode(codes).reshape(rows, K // NVFP4_BLOCK, NVFP4_BLOCK)
    return (q * e4m3_decode(sb)[:, :, None] * float(g)).reshape(rows, K)
