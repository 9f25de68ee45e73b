"""GPU parity of the whole path on the tiny expert (2 layers, d 256, 4/1 heads
of 64, SwiGLU 1024, P 64, chunk 50 x 75, 10 steps) and on small variants that
reach the edge cases: several KV groups, a ragged prefix, P = 0, a constant
velocity field.  Every call goes through the C ABI."""
import numpy as np
import pytest

from oracle import fm_oracle as O
from tests._metrics import cosine, max_abs, rel_l2
from vla_flow_matching_denoise_b200 import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

from vla_flow_matching_denoise_b200.binding import Expert  # noqa: E402

PER_OP_TOL = 1e-2      # per-op rel-L2 on the op's own (GPU) inputs, bf16 outputs
VEL_TOL = 1e-2         # per-step velocity rel-L2 (teacher-forced)


class Case:
    def __init__(self, shape, seed=0, std=None, out_bias=None):
        self.shape = shape
        self.raw = synth.make_weights(shape, seed, std=std)
        self.kp, self.vp = synth.make_prefix(shape, seed)
        self.x0 = synth.make_x0(shape, seed)
        self.out_bias = out_bias
        self.W = O.Weights(self.raw)

    def expert(self, **kw):
        e = Expert(self.shape, self.raw, out_bias=self.out_bias, **kw)
        e.set_prefix(self.kp, self.vp, self.shape.batch, self.shape.prefix_len)
        return e


@pytest.fixture(scope="module")
def tiny():
    c = Case(synth.WORKLOADS["tiny"])
    c.e = c.expert()
    return c


def test_geometry_is_whole_clusters(tiny):
    cs, nc, n = tiny.e.geometry()
    assert cs == 8 and n == 8 * nc and nc >= 1


def test_time_modulation_matches_oracle(tiny):
    s = tiny.shape
    m = tiny.e.time_modulation(s.steps)
    ts, _ = O.time_schedule(s.steps)
    ref = O.time_modulation(ts, tiny.W.time_w1, tiny.W.time_w2)
    assert rel_l2(m, ref) < 5e-3


def _oracle_ops(case, rec, m, l, P):
    s = case.shape
    per, _ = O.split_modulation(m.astype(np.float64), s.n_layers, s.d_model)
    s_a, b_a, g_a, s_f, b_f, g_f = per[l]
    lw = case.W.layers[l]
    T, hd = s.chunk_len, s.head_dim
    h_in = rec["h_in"].astype(np.float64)
    y = O.ada_rms(h_in, s_a, b_a, s.rms_eps)
    pos = P + np.arange(T)
    q = O.rope((y @ lw["wq"].T).reshape(T, s.n_q_heads, hd), pos, s.rope_base).reshape(T, -1)
    k = O.rope((y @ lw["wk"].T).reshape(T, s.n_kv_heads, hd), pos, s.rope_base).reshape(T, -1)
    v = y @ lw["wv"].T
    K = np.concatenate([O.decode_bf16(case.kp[l][0]), rec["k"].reshape(T, s.n_kv_heads, hd)])
    V = np.concatenate([O.decode_bf16(case.vp[l][0]), rec["v"].reshape(T, s.n_kv_heads, hd)])
    o = O.gqa_attention(rec["q"].astype(np.float64).reshape(T, s.n_q_heads, hd), K, V).reshape(T, -1)
    h_mid = h_in + g_a * (rec["o"].astype(np.float64) @ lw["wo"].T)
    yf = O.ada_rms(rec["h_mid"].astype(np.float64), s_f, b_f, s.rms_eps)
    u = O.silu(yf @ lw["w_gate"].T) * (yf @ lw["w_up"].T)
    h_out = rec["h_mid"].astype(np.float64) + g_f * (rec["u"].astype(np.float64) @ lw["w_down"].T)
    return dict(q=q, k=k, v=v, o=o, h_mid=h_mid, u=u, h_out=h_out)


def _check_trace(case, e, step=3):
    s = case.shape
    m_all = e.time_modulation(s.steps)
    x = case.x0[0]
    tr = e.trace_velocity(x, step, s.steps)
    # in-proj
    h0 = x.astype(np.float64) @ case.W.in_proj.T
    assert rel_l2(tr[0]["h_in"], h0) < 1e-5
    worst = {}
    for l in range(s.n_layers):
        ref = _oracle_ops(case, tr[l], m_all[step], l, s.prefix_len)
        for k, r in ref.items():
            err = rel_l2(tr[l][k], r)
            worst[k] = max(worst.get(k, 0.0), err)
            assert err < PER_OP_TOL, (l, k, err)
    per, (s_o, b_o) = O.split_modulation(m_all[step].astype(np.float64), s.n_layers, s.d_model)
    v = O.ada_rms(tr[-2]["h_out"].astype(np.float64), s_o, b_o, s.rms_eps) @ case.W.out_proj.T
    assert rel_l2(tr[-1]["v"], v) < 1e-5
    return worst


def test_per_op_parity_trace(tiny):
    _check_trace(tiny, tiny.e)


def test_per_op_parity_stress_weights():
    # weights N(0, 1/sqrt(fan_in))-like (std 0.06 at d 256) make every op matter
    c = Case(synth.WORKLOADS["tiny"], seed=1, std=0.0625)
    e = c.expert()
    _check_trace(c, e, step=0)


def test_velocity_teacher_forced(tiny):
    s = tiny.shape
    ts, dt = O.time_schedule(s.steps)
    M = O.time_modulation(ts, tiny.W.time_w1, tiny.W.time_w2)
    kp = [O.decode_bf16(k[0]) for k in tiny.kp]
    vp = [O.decode_bf16(v[0]) for v in tiny.vp]
    x = tiny.x0[0].astype(np.float64)
    for k in range(s.steps):
        v_ref = O.expert_velocity(x, M[k], tiny.W, kp, vp, s.rms_eps, s.rope_base, s.n_q_heads, s.n_kv_heads)
        v_gpu = tiny.e.velocity(x[None].astype(np.float32), k, s.steps)[0]
        assert rel_l2(v_gpu, v_ref) < VEL_TOL, (k, rel_l2(v_gpu, v_ref))
        x = x + dt * v_ref


def test_denoise_end_to_end(tiny):
    s = tiny.shape
    ref = O.denoise(tiny.x0, s.steps, tiny.raw, tiny.kp, tiny.vp, s, W=tiny.W)
    out = tiny.e.denoise(tiny.x0, s.steps)
    assert cosine(out, ref) >= 0.999
    assert max_abs(out, ref) <= 5e-2


def test_denoise_is_bit_reproducible_and_buffer_kind_independent(tiny):
    s = tiny.shape
    a = tiny.e.denoise(tiny.x0, s.steps)
    b = tiny.e.denoise(tiny.x0, s.steps)
    assert np.array_equal(a, b)
    xd = torch.from_numpy(tiny.x0).cuda()
    od = tiny.e.denoise(xd, s.steps)
    torch.cuda.synchronize()
    assert np.array_equal(od.cpu().numpy(), a)
    # in place (out aliases x0) on the device
    tiny.e.denoise(xd, s.steps, out=xd)
    torch.cuda.synchronize()
    assert np.array_equal(xd.cpu().numpy(), a)


def test_step_counts_and_graph_reuse(tiny):
    s = tiny.shape
    for n in (1, 4, 16):
        ref = O.denoise(tiny.x0, n, tiny.raw, tiny.kp, tiny.vp, s, W=tiny.W)
        out = tiny.e.denoise(tiny.x0, n)
        assert cosine(out, ref) >= 0.999, n


def test_prefix_change_reuses_graph_and_is_exact():
    # a ragged prefix (P = 37, not a multiple of 16), then P = 0, on the same handle
    shape = synth.WORKLOADS["tiny"]
    c = Case(shape)
    e = Expert(shape, c.raw, max_prefix=64)
    for P in (37, 0, 64):
        kp = [k[:, :P] .copy() for k in c.kp]
        vp = [v[:, :P].copy() for v in c.vp]
        e.set_prefix(kp, vp, 1, P)
        sP = synth.ExpertShape(**{**shape.__dict__, "prefix_len": P})
        ref = O.denoise(c.x0, 10, c.raw, kp, vp, sP, W=c.W)
        out = e.denoise(c.x0, 10)
        assert cosine(out, ref) >= 0.999, P
        assert max_abs(out, ref) <= 5e-2, P


def test_zero_and_constant_velocity_fields_are_exact():
    shape = synth.ExpertShape(**{**synth.WORKLOADS["tiny"].__dict__, "steps": 16})
    raw = synth.make_weights(shape)
    raw["out_proj"][:] = 0
    kp, vp = synth.make_prefix(shape)
    x0 = synth.make_x0(shape)
    e = Expert(shape, raw)
    e.set_prefix(kp, vp, 1, shape.prefix_len)
    assert np.array_equal(e.denoise(x0, 16), x0)          # v = 0 leaves x fixed
    c = np.array([0.5, -2.0, 0.125] * 25, dtype=np.float32)
    e2 = Expert(shape, raw, out_bias=c)
    e2.set_prefix(kp, vp, 1, shape.prefix_len)
    got = e2.denoise(x0, 16)
    # v = c exactly; each update x <- x + dt c rounds once in fp32 (dt c is exact),
    # so the exact reference is the fp32 recurrence, within 16 ulp of x0 - c
    want = x0.copy()
    for _ in range(16):
        want = (want + np.float32(-1 / 16) * c).astype(np.float32)
    assert np.array_equal(got, want)
    assert np.all(np.abs(got - (x0.astype(np.float64) - c)) <= 16 * np.spacing(np.abs(x0 - c) + 2.0))


def test_gqa_head_to_kv_group_map():
    # zero K everywhere => uniform attention; prefix V = g + 1 per KV head and
    # chunk V = 0 => head h returns P (g + 1) / (P + T) with g = h // G
    shape = synth.ExpertShape(1, 256, 4, 2, 64, 512, 75, 30, 2)
    raw = synth.make_weights(shape)
    raw["layers"][0]["wk"][:] = 0
    raw["layers"][0]["wv"][:] = 0
    kp, vp = synth.make_prefix(shape)
    kp[0][:] = 0
    for g in range(2):
        vp[0][:, :, g, :] = synth.f32_to_bf16_bits(np.float32(g + 1))
    e = Expert(shape, raw)
    e.set_prefix(kp, vp, 1, 30)
    o = e.trace_velocity(synth.make_x0(shape)[0], 0, 2)[0]["o"].reshape(50, 4, 64)
    for h in range(4):
        want = 30 * (h // 2 + 1) / 80
        assert np.all(np.abs(o[:, h] - want) <= want * 2 ** -8), h
    assert np.array_equal(o[:, 0], o[:, 1]) and np.array_equal(o[:, 2], o[:, 3])
