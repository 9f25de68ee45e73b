"""Pins of the oracle's layer composition: hand-worked one-layer experts run
through ``expert_velocity`` (no GPU).

The op-level pins fix each definition (AdaRMSNorm, RoPE, softmax, GQA,
SwiGLU, Euler); these cases fix how the expert wires them together, as the
readings R2-R7 state it ("LingBot-VLA on Thor (sm_110)", §2 Build: fused
AdaRMSNorm, SwiGLU tail, QKV + RoPE; §3: GQA denoise attention):

  * the modulation row is cut per layer into (s_a, b_a, g_a, s_f, b_f, g_f)
    and a final (s_o, b_o) -- each slot below has its own value and its own
    visible effect;
  * h = x W_in^T; y = AdaRMSNorm(h; s_a, b_a); q, k, v = y W^T (head-major
    columns); RoPE on q and the chunk's k at positions P .. P+T-1, the cached
    prefix keys untouched; attention over [prefix ; chunk] keys;
    h += g_a * (o W_o^T); y = AdaRMSNorm(h; s_f, b_f);
    h += g_f * ((SiLU(y W_gate^T) * (y W_up^T)) W_down^T);
    v = AdaRMSNorm(h; s_o, b_o) W_out^T.

Each expected value is worked out by hand below from those statements, as
scalar arithmetic on the case's numbers (eps = 0 so every norm is exact).
The weights are one-hot or tiny matrices chosen so that a wiring mistake
(gate and up swapped, g_a and g_f swapped, s and b swapped, the chunk
rotated at 0 .. T-1, the prefix keys rotated again, a transposed
projection, a missing 1/sqrt(hd), a (1 + g) gate) changes the velocity by
far more than rounding.  The last test plants each such mistake in a copy of
the oracle and checks that at least one case fails on it.
"""
import math
import os
import types

import numpy as np
import pytest

from oracle import fm_oracle as O

ORACLE_SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "fm_oracle.py")


def silu(z: float) -> float:
    return z / (1.0 + math.exp(-z))


def modulation(d, s_a, b_a, g_a, s_f, b_f, g_f, s_o, b_o):
    """One layer's modulation row in the slot order of R2."""
    m = np.concatenate([s_a, b_a, g_a, s_f, b_f, g_f, s_o, b_o]).astype(np.float64)
    assert m.size == 8 * d
    return m


class _W:
    """A Weights-like holder of float64 matrices for expert_velocity."""

    def __init__(self, in_proj, out_proj, layer):
        self.dtype = np.float64
        self.in_proj = np.asarray(in_proj, dtype=np.float64)
        self.out_proj = np.asarray(out_proj, dtype=np.float64)
        self.layers = [{k: np.asarray(v, dtype=np.float64) for k, v in layer.items()}]


def _run(mod, case):
    return mod.expert_velocity(case["x"], case["m"], case["W"], [case["kp"]], [case["vp"]], 0.0, 1e4,
                               case["hq"], case["hkv"])


# --------------------------------------------------------------------------- case 1: FFN path
def case_ffn():
    """d = A = 2, one token.  Attention weights are zero (o = 0); the FFN has
    one hidden unit: gate reads y_0, up reads y_1, down writes h_0."""
    x = np.array([[-13.0, 7.0]])
    w_in = np.array([[1.0, 2.0], [0.0, 1.0]])          # h = (x0 + 2 x1, x1) = (1, 7)
    w_out = np.array([[1.0, 0.0], [1.0, 1.0]])         # v = (y0, y0 + y1)
    layer = dict(wq=np.zeros((2, 2)), wk=np.zeros((2, 2)), wv=np.zeros((2, 2)), wo=np.eye(2),
                 w_gate=np.array([[1.0, 0.0]]), w_up=np.array([[0.0, 1.0]]), w_down=np.array([[1.0], [0.0]]))
    m = modulation(2, s_a=[3.0, -0.75], b_a=[0.3, 0.7], g_a=[7.0, -3.0],
                   s_f=[1.0, 0.5], b_f=[0.5, -0.25], g_f=[2.0, 5.0],
                   s_o=[0.5, -0.5], b_o=[0.1, -0.2])
    kp = np.zeros((1, 1, 2))
    vp = np.zeros((1, 1, 2))
    # by hand: h = (1, 7), mean(h^2) = 25, h / rms = (0.2, 1.4)
    # FFN norm: y = (0.2 * 2 + 0.5, 1.4 * 1.5 - 0.25) = (0.9, 1.85)
    u = silu(0.9) * 1.85
    h0, h1 = 1.0 + 2.0 * u, 7.0                        # g_f[0] gates the one FFN output
    r = math.sqrt((h0 * h0 + h1 * h1) / 2.0)
    y0, y1 = h0 / r * 1.5 + 0.1, h1 / r * 0.5 - 0.2
    expect = np.array([[y0, y0 + y1]])
    return dict(x=x, m=m, W=_W(w_in, w_out, layer), kp=kp, vp=vp, hq=1, hkv=1), expect


# --------------------------------------------------------------------------- case 2: attention path
def case_attention():
    """d = A = hd = 2, one head, one token, P = 2 cached keys; the FFN is
    zero.  Key 0 scores 0, key 1 is (1, 0) (already rotated: it must not be
    rotated again), the chunk's own key is 0; every weight stays visible."""
    x = np.array([[-13.0, 7.0]])
    w_in = np.array([[1.0, 2.0], [0.0, 1.0]])          # h = (1, 7)
    w_out = np.array([[1.0, 0.0], [1.0, 1.0]])
    layer = dict(wq=np.eye(2), wk=np.zeros((2, 2)), wv=np.array([[0.0, 1.0], [1.0, 0.0]]),
                 wo=np.array([[1.0, 0.0], [1.0, 1.0]]),
                 w_gate=np.zeros((1, 2)), w_up=np.zeros((1, 2)), w_down=np.zeros((2, 1)))
    m = modulation(2, s_a=[1.0, 0.5], b_a=[0.5, -0.25], g_a=[0.5, 2.0],
                   s_f=[-0.5, 2.0], b_f=[1.0, 1.0], g_f=[9.0, 9.0],
                   s_o=[0.0, 0.0], b_o=[0.0, 0.0])
    kp = np.array([[[0.0, 0.0]], [[1.0, 0.0]]])        # [P = 2, H_kv = 1, hd = 2]
    vp = np.array([[[4.0, 0.0]], [[0.0, 8.0]]])
    # by hand: y = (0.9, 1.85) (attention norm); q = y, rotated by angle
    # P + 0 = 2 (hd = 2: theta_0 = 1); k_chunk = 0; v_chunk = (y1, y0)
    c, s = math.cos(2.0), math.sin(2.0)
    q0 = 0.9 * c - 1.85 * s
    s1 = q0 * 1.0 / math.sqrt(2.0)                     # score of key 1; keys 0 and chunk score 0
    e1 = math.exp(s1)
    w0, w1, wc = 1.0 / (2.0 + e1), e1 / (2.0 + e1), 1.0 / (2.0 + e1)
    o0 = w0 * 4.0 + w1 * 0.0 + wc * 1.85
    o1 = w0 * 0.0 + w1 * 8.0 + wc * 0.9
    a0, a1 = o0, o0 + o1                               # o W_o^T
    h0, h1 = 1.0 + 0.5 * a0, 7.0 + 2.0 * a1            # g_a gates the attention branch
    r = math.sqrt((h0 * h0 + h1 * h1) / 2.0)
    n0, n1 = h0 / r, h1 / r                            # s_o = b_o = 0
    expect = np.array([[n0, n0 + n1]])
    return dict(x=x, m=m, W=_W(w_in, w_out, layer), kp=kp, vp=vp, hq=1, hkv=1), expect


# --------------------------------------------------------------------------- case 3: heads
def case_heads():
    """d = A = 4, two query heads sharing one KV head (hd = 2), one token,
    P = 1.  Head 0's query is zero (uniform weights over the prefix key and
    the chunk key); head 1's query is (200, 0) before RoPE, which makes the
    prefix key dominant (score ~76: weight 1 - 7e-34)."""
    x = np.ones((1, 4))
    wq = np.zeros((4, 4))
    wq[2, 0] = 200.0                                   # column 2 = head 1, dim 0 (head-major)
    layer = dict(wq=wq, wk=np.zeros((2, 4)), wv=np.zeros((2, 4)), wo=np.eye(4),
                 w_gate=np.zeros((1, 4)), w_up=np.zeros((1, 4)), w_down=np.zeros((4, 1)))
    z = [0.0] * 4
    m = modulation(4, s_a=z, b_a=z, g_a=[1.0] * 4, s_f=z, b_f=z, g_f=z, s_o=z, b_o=z)
    kp = np.array([[[1.0, 0.0]]])                      # [P = 1, 1, 2]
    vp = np.array([[[2.0, 3.0]]])
    # by hand: h = y = (1, 1, 1, 1); head 0: o = ((2, 3) + 0) / 2; head 1: o = (2, 3)
    h = [1.0 + 1.0, 1.0 + 1.5, 1.0 + 2.0, 1.0 + 3.0]
    r = math.sqrt(sum(t * t for t in h) / 4.0)
    expect = np.array([[t / r for t in h]])
    return dict(x=x, m=m, W=_W(np.eye(4), np.eye(4), layer), kp=kp, vp=vp, hq=2, hkv=1), expect


# --------------------------------------------------------------------------- case 4: two tokens
def case_two_tokens():
    """d = A = hd = 2, one head, T = 2 chunk tokens, P = 3 cached zero keys
    with zero values (they take softmax weight but add nothing): the chunk
    attends to itself without a mask, token
    i's query and key are rotated by P + i.  Token 0 has q = k = (1, 0)
    before RoPE, token 1 has q = k = (0, 1); v = y."""
    x = np.array([[5.0, 0.0], [0.0, 5.0]])
    layer = dict(wq=np.eye(2), wk=np.eye(2), wv=np.eye(2), wo=np.eye(2),
                 w_gate=np.zeros((1, 2)), w_up=np.zeros((1, 2)), w_down=np.zeros((2, 1)))
    z = [0.0, 0.0]
    m = modulation(2, s_a=z, b_a=z, g_a=[1.0, 1.0], s_f=z, b_f=z, g_f=z, s_o=z, b_o=z)
    P = 3
    kp = np.zeros((P, 1, 2))
    vp = np.zeros((P, 1, 2))
    # by hand: y_0 = (sqrt2, 0), y_1 = (0, sqrt2) (rms of (5, 0) is 5/sqrt2).
    # rotated q_i = k_i = R(P + i) y_i; score(i, j) = y_i . R(j - i) y_j / sqrt2
    # (rotation by P + j then the transpose of P + i), so
    # score(0,0) = score(1,1) = 2 / sqrt2; score(0,1) = y_0 . R(1) y_1 / sqrt2
    # = sqrt2 * (-sin 1) * sqrt2 / sqrt2 = -sqrt2 sin 1, and score(1,0) is the
    # same (q = k here, so the score matrix is symmetric).
    r2 = math.sqrt(2.0)
    out = []
    for i in range(2):
        sc = [0.0] * P + ([r2, -r2 * math.sin(1.0)] if i == 0 else [-r2 * math.sin(1.0), r2])
        mx = max(sc)
        e = [math.exp(t - mx) for t in sc]
        tot = sum(e)
        w = [t / tot for t in e]
        o = [w[P] * r2 + w[P + 1] * 0.0, w[P] * 0.0 + w[P + 1] * r2]
        h = [x[i][0] + o[0], x[i][1] + o[1]]
        rr = math.sqrt((h[0] ** 2 + h[1] ** 2) / 2.0)
        out.append([h[0] / rr, h[1] / rr])
    return dict(x=x, m=m, W=_W(np.eye(2), np.eye(2), layer), kp=kp, vp=vp, hq=1, hkv=1), np.array(out)


CASES = {"ffn": case_ffn, "attention": case_attention, "heads": case_heads, "two_tokens": case_two_tokens}


@pytest.mark.parametrize("name", sorted(CASES))
def test_expert_velocity_hand_worked(name):
    case, expect = CASES[name]()
    got = _run(O, case)
    assert got.shape == expect.shape
    assert np.allclose(got, expect, rtol=0, atol=1e-12), (got, expect)


def test_cases_are_sensitive():
    """Every case moves with its inputs: a different modulation row changes
    the velocity by far more than the 1e-12 bar."""
    for name, make in CASES.items():
        case, expect = make()
        m2 = case["m"].copy()
        m2[:] += 0.125
        case["m"] = m2
        assert np.max(np.abs(_run(O, case) - expect)) > 1e-3, name


# --------------------------------------------------------------------------- planted mistakes
MUTATIONS = {
    "gate_up_swapped": ('silu(y @ lw["w_gate"].T) * (y @ lw["w_up"].T)',
                        'silu(y @ lw["w_up"].T) * (y @ lw["w_gate"].T)'),
    "g_a_g_f_swapped": ("s_a, b_a, g_a, s_f, b_f, g_f = per[l]", "s_a, b_a, g_f, s_f, b_f, g_a = per[l]"),
    "s_b_swapped": ("s_a, b_a, g_a, s_f, b_f, g_f = per[l]", "b_a, s_a, g_a, b_f, s_f, g_f = per[l]"),
    "s_b_swapped_attn_only": ("s_a, b_a, g_a, s_f, b_f, g_f = per[l]", "b_a, s_a, g_a, s_f, b_f, g_f = per[l]"),
    "s_b_swapped_final": ("per, (s_o, b_o) = split_modulation", "per, (b_o, s_o) = split_modulation"),
    "attn_norm_uses_ffn_slot": ("y = aq(ada_rms(h, s_a, b_a, eps))", "y = aq(ada_rms(h, s_f, b_f, eps))"),
    "ffn_norm_uses_attn_slot": ("y = aq(ada_rms(h, s_f, b_f, eps))", "y = aq(ada_rms(h, s_a, b_a, eps))"),
    "chunk_rotated_from_zero": ("pos = P + np.arange(T)", "pos = np.arange(T)"),
    "prefix_rotated_again": ("K = np.concatenate([kp, kc], axis=0)",
                             "K = np.concatenate([rope(kp, np.arange(P), rope_base), kc], axis=0)"),
    "q_not_rotated": ("q = rope(q, pos, rope_base)", "q = q"),
    "gate_one_plus_g_attn": ("h = h + g_a * (", "h = h + (1.0 + g_a) * ("),
    "gate_one_plus_g_ffn": ("h = h + g_f * (", "h = h + (1.0 + g_f) * ("),
    "in_proj_transposed": ("h = x.astype(dt_) @ W.in_proj.T", "h = x.astype(dt_) @ W.in_proj"),
    "out_proj_transposed": ("@ W.out_proj.T", "@ W.out_proj"),
    "wo_transposed": ('(aq(o) @ lw["wo"].T)', '(aq(o) @ lw["wo"])'),
    "wq_wk_swapped": ('q = (y @ lw["wq"].T)', 'q = (y @ lw["wk"].T)'),
    "no_attention_residual": ("h = h + g_a * (aq(o)", "h = h + 0.0 * g_a * (aq(o)"),
    "no_score_scale": ("p = softmax((q[:, h, :] @ k[:, g, :].T) / math.sqrt(hd))",
                       "p = softmax(q[:, h, :] @ k[:, g, :].T)"),
    "final_norm_dropped": ("v = ada_rms(h, s_o, b_o, eps) @ W.out_proj.T", "v = h @ W.out_proj.T"),
}


def _mutant(src: str, old: str, new: str):
    assert src.count(old) >= 1, f"pattern not found in the oracle: {old!r}"
    mod = types.ModuleType("fm_oracle_mutant")
    exec(compile(src.replace(old, new), ORACLE_SRC, "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_fails_a_case(name):
    with open(ORACLE_SRC) as f:
        src = f.read()
    mod = _mutant(src, *MUTATIONS[name])
    failed = []
    for cname, make in CASES.items():
        case, expect = make()
        try:
            got = _run(mod, case)
            ok = got.shape == expect.shape and np.allclose(got, expect, rtol=0, atol=1e-12)
        except Exception:
            ok = False
        if not ok:
            failed.append(cname)
    assert failed, f"mistake {name} passes every hand-worked case"
