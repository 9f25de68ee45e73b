"""Pins of the CPU oracle against closed forms, hand values, brute force and
independent library routines (no GPU).  Each group names the passage of the
pages, or the mathematical fact, that fixes the expected value."""
import math
import os

import numpy as np
import pytest

from oracle import fm_oracle as O
from vla_flow_matching_denoise_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --------------------------------------------------------------------------- time feature
def test_sinusoid_t0_is_zero_sines_unit_cosines():
    e = O.sinusoid(np.array([0.0]))[0]
    assert np.all(e[:128] == 0.0) and np.all(e[128:] == 1.0)


def test_sinusoid_extreme_periods_hand_values():
    # channel 127 has period 4: at t = 1 the angle is pi/2, at t = 0.5 it is pi/4
    e1 = O.sinusoid(np.array([1.0, 0.5, 1e-3]))
    assert abs(e1[0, 127] - 1.0) < 1e-15 and abs(e1[0, 255]) < 1e-15
    assert abs(e1[1, 127] - math.sqrt(0.5)) < 1e-15
    # channel 0 has period 4e-3: at t = 1e-3 the angle is pi/2
    assert abs(e1[2, 0] - 1.0) < 1e-12 and abs(e1[2, 128]) < 1e-12


def test_sinusoid_periods_geometric_and_unit_circle():
    t = np.array([1e-4])
    e = O.sinusoid(t)[0]
    assert np.allclose(e[:128] ** 2 + e[128:] ** 2, 1.0, atol=1e-14)
    ang = np.arctan2(e[:128], e[128:])            # small t: no wrap
    period = 2 * math.pi * t[0] / ang
    ratio = period[1:] / period[:-1]
    assert np.allclose(ratio, (4.0 / 4e-3) ** (1 / 127), rtol=1e-9)
    assert abs(period[0] - 4e-3) < 1e-12


def test_time_schedule_matches_euler_grid():
    ts, dt = O.time_schedule(10)
    assert ts[0] == 1.0 and abs(ts[-1] - 0.1) < 1e-15 and dt == -0.1
    with pytest.raises(ValueError):
        O.time_schedule(0)


def test_time_modulation_one_hot_mlp_hand_value():
    # W1 picks the cosine of channel 0 (== 1 at t = 0); W2 copies h1[0] and -h1[0]
    w1 = np.zeros((4, 256)); w1[0, 128] = 1.0; w1[1, 0] = 1.0
    w2 = np.zeros((3, 4)); w2[0, 0] = 1.0; w2[1, 0] = -1.0; w2[2, 1] = 1.0
    m = O.time_modulation(np.array([0.0]), w1, w2)[0]
    silu1 = 0.7310585786300049     # 1 / (1 + e^-1)
    assert abs(m[0] - silu1) < 1e-15 and abs(m[1] + silu1) < 1e-15 and m[2] == 0.0


def test_split_modulation_order():
    L, d = 3, 4
    m = np.arange(L * 6 * d + 2 * d, dtype=np.float64)
    per, (so, bo) = O.split_modulation(m, L, d)
    assert per[1][2][0] == (6 * 1 + 2) * d          # g_a of layer 1
    assert per[2][5][-1] == (6 * 2 + 6) * d - 1     # g_f of layer 2, last entry
    assert so[0] == 6 * L * d and bo[-1] == m[-1]


# --------------------------------------------------------------------------- AdaRMSNorm
def test_ada_rms_hand_value():
    eps = 1e-6
    y = O.ada_rms(np.array([3.0, 4.0]), np.zeros(2), np.zeros(2), eps)
    assert np.allclose(y, np.array([3.0, 4.0]) / math.sqrt(12.5 + eps), rtol=0, atol=1e-15)


def test_ada_rms_scale_minus_one_gives_shift_exactly():
    rng = np.random.default_rng(1)
    x, b = rng.standard_normal((5, 8)), rng.standard_normal(8)
    assert np.array_equal(O.ada_rms(x, -np.ones(8), b, 1e-6), np.broadcast_to(b, (5, 8)))


def test_ada_rms_scale_invariance_and_modulation():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((3, 16))
    s, b = rng.standard_normal(16), rng.standard_normal(16)
    y1 = O.ada_rms(x, s, b, 0.0)
    y2 = O.ada_rms(1e3 * x, s, b, 0.0)
    assert np.allclose(y1, y2, rtol=1e-13, atol=1e-13)
    # mean of squares of the un-modulated part is exactly 1 when eps = 0
    z = O.ada_rms(x, np.zeros(16), np.zeros(16), 0.0)
    assert np.allclose(np.mean(z * z, axis=1), 1.0, rtol=1e-14)


# --------------------------------------------------------------------------- SiLU / SwiGLU
def test_silu_values():
    assert O.silu(np.array(0.0)) == 0.0
    assert abs(O.silu(np.array(1.0)) - 0.7310585786300049) < 1e-16
    assert abs(O.silu(np.array(50.0)) - 50.0) < 1e-18 * 50 + 1e-12
    assert abs(O.silu(np.array(-50.0))) < 1e-19


# --------------------------------------------------------------------------- RoPE
def test_rope_position_zero_is_identity():
    x = np.random.default_rng(3).standard_normal((4, 2, 8))
    assert np.array_equal(O.rope(x, np.zeros(4), 1e4), x)


def test_rope_two_dim_rotation_hand_value():
    # hd = 2: one pair (x0, x1) rotated by angle pos * base^0 = pos
    x = np.array([[[1.0, 0.0]], [[0.0, 2.0]]])
    y = O.rope(x, np.array([0.3, 1.1]), 1e4)
    assert np.allclose(y[0, 0], [math.cos(0.3), math.sin(0.3)], atol=1e-15)
    assert np.allclose(y[1, 0], [-2 * math.sin(1.1), 2 * math.cos(1.1)], atol=1e-15)


def test_rope_pairs_are_j_and_j_plus_half_with_decreasing_frequency():
    hd = 8
    x = np.zeros((1, 1, hd)); x[0, 0, 1] = 1.0           # pair (1, 5), theta_1 = base^(-2/8)
    y = O.rope(x, np.array([2.0]), 100.0)
    th = 100.0 ** (-2.0 / hd)
    expect = np.zeros(hd); expect[1] = math.cos(2 * th); expect[5] = math.sin(2 * th)
    assert np.allclose(y[0, 0], expect, atol=1e-15)


def test_rope_preserves_pair_norms_and_is_relative():
    rng = np.random.default_rng(4)
    q = rng.standard_normal((1, 1, 16)); k = rng.standard_normal((1, 1, 16))
    y = O.rope(q, np.array([7.0]), 1e4)
    assert np.allclose(y[0, 0, :8] ** 2 + y[0, 0, 8:] ** 2, q[0, 0, :8] ** 2 + q[0, 0, 8:] ** 2)
    for m, n in [(300, 5), (40, 39), (3, 11)]:
        lhs = np.dot(O.rope(q, np.array([m]), 1e4)[0, 0], O.rope(k, np.array([n]), 1e4)[0, 0])
        rhs = np.dot(O.rope(q, np.array([m - n]), 1e4)[0, 0], k[0, 0])
        assert abs(lhs - rhs) < 1e-11


# --------------------------------------------------------------------------- softmax / attention
def test_softmax_two_token_closed_form_and_shift_invariance():
    for delta in (-3.0, 0.0, 0.7, 20.0):
        p = O.softmax(np.array([0.0, delta]))
        assert np.allclose(p, [1 / (1 + math.exp(delta)), math.exp(delta) / (1 + math.exp(delta))],
                           rtol=1e-14)
    z = np.random.default_rng(5).standard_normal(9)
    assert np.allclose(O.softmax(z), O.softmax(z + 1234.5), rtol=1e-12)
    assert np.all(np.isfinite(O.softmax(np.array([1e4, 0.0]))))


def _brute_attention(q, k, v):
    T, Hq, hd = q.shape
    S, Hkv, _ = k.shape
    o = np.zeros_like(q)
    for t in range(T):
        for h in range(Hq):
            g = h // (Hq // Hkv)
            sc = [sum(q[t, h, j] * k[s, g, j] for j in range(hd)) / math.sqrt(hd) for s in range(S)]
            mx = max(sc)
            w = [math.exp(a - mx) for a in sc]
            tot = sum(w)
            for j in range(hd):
                o[t, h, j] = sum(w[s] * v[s, g, j] for s in range(S)) / tot
    return o


def test_gqa_attention_matches_brute_force():
    rng = np.random.default_rng(6)
    q = rng.standard_normal((3, 4, 4)); k = rng.standard_normal((5, 2, 4)); v = rng.standard_normal((5, 2, 4))
    assert np.allclose(O.gqa_attention(q, k, v), _brute_attention(q, k, v), rtol=1e-12, atol=1e-13)


def test_attention_identical_keys_gives_mean_of_values():
    rng = np.random.default_rng(7)
    q = rng.standard_normal((4, 2, 8))
    k = np.broadcast_to(rng.standard_normal((1, 1, 8)), (6, 1, 8)).copy()
    v = rng.standard_normal((6, 1, 8))
    o = O.gqa_attention(q, k, v)
    assert np.allclose(o, np.broadcast_to(v.mean(axis=0), o.shape), rtol=1e-13, atol=1e-14)


def test_attention_dominant_key_returns_its_value():
    q = np.ones((1, 1, 4)); k = np.zeros((3, 1, 4)); k[1] = 100.0
    v = np.arange(12, dtype=np.float64).reshape(3, 1, 4)
    assert np.allclose(O.gqa_attention(q, k, v)[0, 0], v[1, 0])


def test_gqa_head_to_kv_map():
    # V of KV head g is the constant g + 1, keys identical: head h returns floor(h/G) + 1
    Hq, Hkv, hd = 8, 2, 4
    q = np.random.default_rng(8).standard_normal((3, Hq, hd))
    k = np.ones((5, Hkv, hd))
    v = np.stack([np.full((5, hd), g + 1.0) for g in range(Hkv)], axis=1)
    o = O.gqa_attention(q, k, v)
    for h in range(Hq):
        assert np.all(o[:, h, :] == h // (Hq // Hkv) + 1)


# --------------------------------------------------------------------------- Euler
def test_euler_constant_and_linear_fields():
    x0 = np.array([1.5, -2.0, 0.25])
    assert np.array_equal(O.euler(x0, 7, lambda x, k, t: np.zeros_like(x)), x0)
    c = np.array([0.5, -0.25, 2.0])
    assert np.array_equal(O.euler(x0, 16, lambda x, k, t: c), x0 - c)          # dt = -1/16 exact
    lam = 0.7
    xn = O.euler(x0, 10, lambda x, k, t: lam * x)
    assert np.allclose(xn, x0 * (1 - lam / 10) ** 10, rtol=1e-14)


def test_euler_passes_time_grid():
    seen = []
    O.euler(np.zeros(1), 4, lambda x, k, t: (seen.append((k, t)), np.zeros(1))[1])
    assert seen == [(0, 1.0), (1, 0.75), (2, 0.5), (3, 0.25)]


# --------------------------------------------------------------------------- whole expert
def _tiny_shape(**kw):
    base = dict(n_layers=2, d_model=16, n_q_heads=4, n_kv_heads=2, head_dim=4, d_ff=32,
                action_dim=3, prefix_len=5, steps=4)
    base.update(kw)
    return synth.ExpertShape(**base)


def _raw(shape, seed=0, std=0.3):
    return synth.make_weights(shape, seed, std=std)


def test_expert_zero_modulation_reduces_to_rms_of_in_proj():
    # time_w2 = 0 makes every scale/shift/gate 0: layers leave h unchanged and
    # v = rms(x W_in^T) W_out^T; with d = A = 2 and identity projections this is by hand
    shape = synth.ExpertShape(1, 2, 1, 1, 2, 4, 2, 3, 3)
    raw = _raw(shape)
    raw["time_w2"][:] = 0
    one = 0x3F80
    raw["in_proj"][:] = np.array([[one, 0], [0, one]], dtype=np.uint16)
    raw["out_proj"][:] = raw["in_proj"]
    W = O.Weights(raw)
    kp, vp = synth.make_prefix(shape, batch=1)
    v = O.expert_velocity(np.array([[3.0, 4.0]] * 50), np.zeros(shape.n_mod), W,
                          [O.decode_bf16(k[0]) for k in kp], [O.decode_bf16(x[0]) for x in vp],
                          1e-6, 1e4, 1, 1)
    assert np.allclose(v, np.array([[3.0, 4.0]] * 50) / math.sqrt(12.5 + 1e-6), atol=1e-15)


def test_expert_constant_velocity_integrates_exactly():
    shape = _tiny_shape(steps=16)
    raw = _raw(shape)
    raw["out_proj"][:] = 0
    kp, vp = synth.make_prefix(shape, batch=2)
    x0 = synth.make_x0(shape, batch=2).astype(np.float64)
    c = np.array([0.5, -2.0, 0.125])
    xn = O.denoise(x0, 16, raw, kp, vp, shape, out_bias=c)
    assert np.array_equal(xn, x0 - c)


def test_expert_zero_up_and_zero_o_leave_residual_stream():
    # W_up = 0 and W_o = 0: each layer adds exactly 0, so the trace's h is constant
    shape = _tiny_shape()
    raw = _raw(shape)
    for lw in raw["layers"]:
        lw["w_up"][:] = 0
        lw["wo"][:] = 0
    W = O.Weights(raw)
    kp, vp = synth.make_prefix(shape, batch=1)
    tr = []
    ts, _ = O.time_schedule(4)
    M = O.time_modulation(ts, W.time_w1, W.time_w2)
    O.expert_velocity(synth.make_x0(shape, batch=1)[0], M[1], W, [O.decode_bf16(k[0]) for k in kp],
                      [O.decode_bf16(v[0]) for v in vp], 1e-6, 1e4, 4, 2, trace=tr)
    for rec in tr[:-1]:
        assert np.array_equal(rec["h_in"], rec["h_out"])
        assert np.all(rec["u"] == 0)


def test_expert_fp32_and_fp64_agree():
    shape = _tiny_shape()
    raw = _raw(shape)
    kp, vp = synth.make_prefix(shape, batch=1)
    x0 = synth.make_x0(shape, batch=1)
    a = O.denoise(x0, 4, raw, kp, vp, shape, dtype=np.float64)
    b = O.denoise(x0, 4, raw, kp, vp, shape, dtype=np.float32)
    assert np.linalg.norm(a - b) / np.linalg.norm(a) < 1e-5


def test_expert_batch_requests_are_independent():
    shape = _tiny_shape()
    raw = _raw(shape)
    kp, vp = synth.make_prefix(shape, batch=3)
    x0 = synth.make_x0(shape, batch=3)
    full = O.denoise(x0, 3, raw, kp, vp, shape)
    perm = [2, 0, 1]
    permuted = O.denoise(x0[perm], 3, raw, [k[perm] for k in kp], [v[perm] for v in vp], shape)
    assert np.array_equal(full[perm], permuted)
    single = O.denoise(x0[1:2], 3, raw, [k[1:2] for k in kp], [v[1:2] for v in vp], shape)
    assert np.array_equal(full[1:2], single)


def test_expert_prefix_position_base_shifts_chunk_rope():
    # with an all-identical prefix the scores of chunk keys depend on P only
    # through RoPE positions; rotating q and k by the same extra offset leaves
    # every score unchanged, so P = 5 and P = 9 give identical chunks when the
    # prefix keys are zero (their scores stay 0 whatever the rotation).
    shape5 = _tiny_shape(prefix_len=5)
    shape9 = _tiny_shape(prefix_len=9)
    raw = _raw(shape5)
    x0 = synth.make_x0(shape5, batch=1)
    kp5, vp5 = synth.make_prefix(shape5, batch=1)
    kp9, vp9 = synth.make_prefix(shape9, batch=1)
    for k5, v5, k9, v9 in zip(kp5, vp5, kp9, vp9):
        k5[:] = 0; k9[:] = 0
        v5[:] = 0x3F80; v9[:] = 0x3F80            # V = 1 everywhere
    a = O.denoise(x0, 2, raw, kp5, vp5, shape5)
    b = O.denoise(x0, 2, raw, kp9, vp9, shape9)
    # prefix weight changes with P (5 vs 9 equal-score keys), so the chunks differ;
    # but the chunk-only scores are RoPE-relative: check that the first layer's
    # chunk-to-chunk score matrix is the same for both P
    W = O.Weights(raw)
    ts, _ = O.time_schedule(2)
    M = O.time_modulation(ts, W.time_w1, W.time_w2)
    per, _ = O.split_modulation(M[0], 2, 16)
    y = O.ada_rms(x0[0].astype(np.float64) @ W.in_proj.T, per[0][0], per[0][1], 1e-6)
    q = (y @ W.layers[0]["wq"].T).reshape(50, 4, 4)
    k = (y @ W.layers[0]["wk"].T).reshape(50, 2, 4)
    s5 = np.einsum("thd,sd->ts", O.rope(q, 5 + np.arange(50), 1e4)[:, :1], O.rope(k, 5 + np.arange(50), 1e4)[:, 0])
    s9 = np.einsum("thd,sd->ts", O.rope(q, 9 + np.arange(50), 1e4)[:, :1], O.rope(k, 9 + np.arange(50), 1e4)[:, 0])
    assert np.allclose(s5, s9, atol=1e-12)
    assert not np.array_equal(a, b)


# --------------------------------------------------------------------------- FP8 quantiser
def _golden_e4m3():
    rows = []
    with open(os.path.join(GOLDEN, "e4m3_codes.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                v, c = line.split()
                rows.append((float(v), int(c, 16)))
    return rows


def test_e4m3_spec_code_points():
    for v, c in _golden_e4m3():
        assert int(O.e4m3_encode(np.array([v], np.float32))[0]) == c, v
        assert O.e4m3_decode(np.array([c], np.uint8))[0] == v


def test_e4m3_encode_is_nearest_even_by_brute_force():
    codes = np.arange(0x7F, dtype=np.uint8)            # non-negative finite codes
    vals = O.e4m3_decode(codes)
    rng = np.random.default_rng(9)
    xs = np.concatenate([rng.uniform(0, 460, 20000), rng.uniform(0, 0.05, 20000),
                         (vals[:-1] + vals[1:]) / 2]).astype(np.float32)   # ties included
    got = O.e4m3_encode(xs)
    for x, g in zip(xs.astype(np.float64), got):
        d = np.abs(vals - min(x, 448.0))
        best = np.flatnonzero(d == d.min())
        want = best[0] if len(best) == 1 else [b for b in best if b % 2 == 0][0]
        assert g == want, (x, g, want)
    neg = O.e4m3_encode(-xs[:100])
    assert np.array_equal(neg, got[:100] | 0x80)


def test_e4m3_encode_agrees_with_torch_float8():
    torch = pytest.importorskip("torch")
    if not hasattr(torch, "float8_e4m3fn"):
        pytest.skip("no float8 in torch")
    xs = np.random.default_rng(10).uniform(-448, 448, 50000).astype(np.float32)
    ref = torch.from_numpy(xs).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(O.e4m3_encode(xs), ref)


def test_fp8_rows_scale_and_roundtrip():
    w = synth.f32_to_bf16_bits(np.random.default_rng(11).standard_normal((6, 64)).astype(np.float32) * 0.02)
    w[3] = 0
    codes, scale = O.fp8_quantize_rows(w)
    assert scale.dtype == np.float32 and scale[3] == 1.0 and np.all(codes[3] == 0)
    wf = O.decode_bf16(w, np.float32)
    amax = np.abs(wf).max(axis=1)
    for r in (0, 1, 2, 4, 5):
        assert scale[r] == np.float32(amax[r]) / np.float32(448.0)
        assert (codes[r] & 0x7F).max() == 0x7E            # the absmax lands on 448
    deq = O.fp8_dequantize_rows(codes, scale)
    err = np.abs(deq - wf.astype(np.float64))
    assert np.all(err <= np.abs(wf) * 2 ** -4 + 2 ** -9 * scale[:, None] + 1e-12)


# --------------------------------------------------------------------------- prefix K/V (R9)
def test_prefix_kv_one_hot_rows_pick_weight_columns_then_rotate():
    # x row p = e_j: K row p = RoPE(Wk[:, j]) at position p, V row p = Wv[:, j]
    rng = np.random.default_rng(21)
    Hkv, hd, dp = 2, 8, 5
    wk = rng.standard_normal((Hkv * hd, dp)); wv = rng.standard_normal((Hkv * hd, dp))
    x = np.zeros((3, dp)); x[0, 4] = 1.0; x[1, 0] = 1.0; x[2, 2] = 1.0
    k, v = O.prefix_kv(x, wk, wv, Hkv, 1e4)
    for p, j in enumerate((4, 0, 2)):
        assert np.allclose(v[p].reshape(-1), wv[:, j], atol=1e-15)
        col = wk[:, j].reshape(1, Hkv, hd)
        assert np.allclose(k[p], O.rope(col, np.array([p]), 1e4)[0], atol=1e-14)
    # position 0 is not rotated
    assert np.allclose(k[0].reshape(-1), wk[:, 4], atol=1e-15)


def test_prefix_kv_brute_force_small():
    rng = np.random.default_rng(22)
    Hkv, hd, dp, P = 1, 4, 3, 4
    wk = rng.standard_normal((hd, dp)); wv = rng.standard_normal((hd, dp)); x = rng.standard_normal((P, dp))
    k, v = O.prefix_kv(x, wk, wv, Hkv, 100.0)
    for p in range(P):
        for e in range(hd):
            assert abs(v[p, 0, e] - sum(x[p, i] * wv[e, i] for i in range(dp))) < 1e-13
        raw = [sum(x[p, i] * wk[e, i] for i in range(dp)) for e in range(hd)]
        for j in range(hd // 2):
            a = p * 100.0 ** (-2.0 * j / hd)
            assert abs(k[p, 0, j] - (raw[j] * math.cos(a) - raw[j + 2] * math.sin(a))) < 1e-13
            assert abs(k[p, 0, j + 2] - (raw[j + 2] * math.cos(a) + raw[j] * math.sin(a))) < 1e-13


def test_bf16_round_bits_ties_to_even_and_exact_values():
    vals = np.array([1.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -2.5, 0.0])
    bits = O.bf16_round_bits(vals)
    # 1 + 2^-8 is halfway between 1 and 1 + 2^-7: ties to even (1.0);
    # 1 + 3 * 2^-8 is halfway between 1 + 2^-7 and 1 + 2^-6: ties to even (1 + 2^-6)
    assert list(O.decode_bf16(bits)) == [1.0, 1.0, 1.0 + 2.0 ** -6, -2.5, 0.0]


# --------------------------------------------------------------------------- NVFP4 (R10)
def test_e2m1_table_and_ties_to_even():
    # the eight E2M1 magnitudes (1 exponent bias, 1 mantissa bit)
    assert list(O.e2m1_decode(np.arange(8))) == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert list(O.e2m1_decode(np.arange(8, 16))) == [-0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0]
    # exact values round trip; midpoints go to the even code
    for c in range(16):
        assert O.e2m1_encode(O.e2m1_decode(np.array([c]))) == (0 if c == 8 else c)
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    assert list(O.e2m1_encode(mids)) == [0, 2, 2, 4, 4, 6, 6]
    assert list(O.e2m1_encode(np.array([7.0, 100.0, -9.0]))) == [7, 7, 15]


def test_nvfp4_block_max_maps_to_six_and_zero_blocks():
    rng = np.random.default_rng(31)
    w = rng.standard_normal((3, 64)).astype(np.float32) * 0.02
    w[1, 16:32] = 0.0                                   # an all-zero block
    bits = O.bf16_round_bits(w)
    codes, sb, g = O.nvfp4_quantize(bits)
    wd = O.decode_bf16(bits)
    assert g == np.float32(np.float32(np.max(np.abs(wd))) / np.float32(2688.0))
    assert sb[1, 1] == 0 and not codes[1, 16:32].any()
    deq = O.nvfp4_dequantize(codes, sb, g)
    # every dequantised weight is a bf16 value times g: e2m1 x e4m3 needs <= 5 significant bits
    prod = O.e2m1_decode(codes).reshape(3, 4, 16) * O.e4m3_decode(sb)[:, :, None]
    assert np.array_equal(O.decode_bf16(O.bf16_round_bits(prod)), prod.astype(np.float32).astype(np.float64))
    # relative error per block is bounded by half an E2M1 step at the block's top (and the scale rounding)
    err = np.abs(deq - wd).reshape(3, 4, 16).max(axis=2)
    top = np.abs(wd).reshape(3, 4, 16).max(axis=2)
    assert np.all(err <= 0.35 * top + 1e-12)


# --------------------------------------------------------------------------- E4M3 activations (R11)
def test_fp8_quant_act_row_max_exact_zero_row_and_grid_round_trip():
    y = np.array([[3.0, -1.5, 0.25, 0.0], [0.0, 0.0, 0.0, 0.0], [-7.0, 1.0, 2.0, 3.5]])
    q = O.fp8_quant_act(y)
    # the row maximum maps to code 448, i.e. to 448 * s with s the fp32 quotient
    # amax / 448 (rounded, so 3/448 does not come back as exactly 3); a zero row stays zero
    assert q[0, 0] == 448.0 * float(np.float32(3.0) / np.float32(448.0))
    assert q[2, 0] == -7.0 and not q[1].any()
    # values on the row's E4M3 grid round-trip exactly: s = 1/64 here
    s = 7.0 / 448.0
    grid = O.e4m3_decode(np.array([0x7E, 0x40, 0x38, 0x31], dtype=np.uint8)) * s   # 448 s, 2 s, 1 s, 0.5625 s
    row = np.array([[-grid[0], grid[1], grid[2], grid[3]]])
    assert np.array_equal(O.fp8_quant_act(row), row)
    # relative error per entry is at most half an E4M3 step (2^-4) of its binade
    r = np.random.default_rng(41).standard_normal((5, 64))
    qr = O.fp8_quant_act(r)
    big = np.abs(r) > np.max(np.abs(r), axis=1, keepdims=True) * 2.0 ** -6
    assert np.all(np.abs(qr - r)[big] <= np.abs(r)[big] * 2.0 ** -4 + 1e-12)


def test_act_fp8_quantises_the_inputs_of_the_four_linears(monkeypatch):
    """R11 applies to the inputs of QKV, o_proj, gate_up and down, once each
    per layer; with quantisation the chunk stays close to the plain one."""
    s = synth.WORKLOADS["tiny"]
    raw = synth.make_weights(s)
    kp, vp = synth.make_prefix(s)
    x0 = synth.make_x0(s)
    seen = []
    real = O.fp8_quant_act
    W = O.Weights(raw, fp8=True)
    monkeypatch.setattr(O, "fp8_quant_act", lambda a: seen.append(a.shape) or real(a))
    M = O.time_modulation(np.array([1.0]), W.time_w1, W.time_w2)
    O.expert_velocity(x0[0], M[0], W, [O.decode_bf16(k[0]) for k in kp], [O.decode_bf16(v[0]) for v in vp],
                      s.rms_eps, s.rope_base,
                      s.n_q_heads, s.n_kv_heads, act_fp8=True)
    T, d, hq, F = s.chunk_len, s.d_model, s.n_q_heads * s.head_dim, s.d_ff
    assert seen == [(T, d), (T, hq), (T, d), (T, F)] * s.n_layers
    monkeypatch.setattr(O, "fp8_quant_act", real)
    a = O.denoise(x0, s.steps, raw, kp, vp, s, W=W)
    b = O.denoise(x0, s.steps, raw, kp, vp, s, W=W, act_fp8=True)
    assert not np.array_equal(a, b)
    c = np.dot(a.ravel(), b.ravel()) / np.linalg.norm(a) / np.linalg.norm(b)
    assert c > 0.99


def test_fp8_quantize_act_codes_ties_and_subnormals():
    """R11 codes: with amax = 448 the scale is exactly 1, so the codes are the
    E4M3 nearest-even codes of the values themselves: midpoints go to the even
    code, half the smallest subnormal flushes to zero, the sign bit is bit 7."""
    row = np.zeros(8, dtype=np.float32)
    row[:7] = [448.0, 1.0625, 1.1875, 2.0 ** -10, 3 * 2.0 ** -10, -1.0, -448.0]
    codes, s = O.fp8_quantize_act(row[None])
    assert s[0] == 1.0
    assert list(codes[0]) == [0x7E, 0x38, 0x3A, 0x00, 0x02, 0xB8, 0xFE, 0x00]
    codes, s = O.fp8_quantize_act(np.zeros((2, 16), dtype=np.float32))
    assert np.all(s == 1.0) and not codes.any()
