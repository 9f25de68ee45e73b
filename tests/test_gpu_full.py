"""GPU parity at the full workload sizes, in the launch configuration the
benchmark times (fm_denoise, graph replay):
  * LingBot-VLA-shaped expert, bf16, P 256, 10 steps, chunk 50 x 75;
  * the same expert with P 832, 50 steps, chunk 50 x 55;
  * 64 independent requests (oracle on requests 0, 1 and 63).
Bars: per-op rel-L2 on the op's own inputs, per-step (teacher-forced) velocity
rel-L2 <= 1e-2, final chunk cosine >= 0.999 and max-abs <= 5e-2."""
import numpy as np
import pytest

from oracle import fm_oracle as O
from tests._metrics import cosine, max_abs, rel_l2
from vla_flow_matching_denoise_b200 import synth

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

from vla_flow_matching_denoise_b200.binding import Expert  # noqa: E402
from tests.test_gpu_tiny import PER_OP_TOL, _oracle_ops  # noqa: E402

BASE = synth.WORKLOADS["lingbot_p256_n10"]


class Full:
    pass


@pytest.fixture(scope="module")
def full():
    f = Full()
    f.shape = BASE
    f.raw = synth.make_weights(BASE)
    f.W = O.Weights(f.raw)
    f.kp, f.vp = synth.make_prefix(BASE)
    f.x0 = synth.make_x0(BASE)
    f.e = Expert(BASE, f.raw, max_prefix=832, max_batch=64)
    f.e.set_prefix(f.kp, f.vp, 1, BASE.prefix_len)
    return f


def test_time_modulation_full(full):
    m = full.e.time_modulation(10)
    ts, _ = O.time_schedule(10)
    ref = O.time_modulation(ts, full.W.time_w1, full.W.time_w2)
    assert rel_l2(m, ref) < 5e-3


def test_per_op_parity_all_layers(full):
    s = full.shape
    m_all = full.e.time_modulation(s.steps)
    step = 4
    tr = full.e.trace_velocity(full.x0[0], step, s.steps)
    assert rel_l2(tr[0]["h_in"], full.x0[0].astype(np.float64) @ full.W.in_proj.T) < 1e-5

    class C:
        pass
    c = C()
    c.shape, c.W, c.kp, c.vp = s, full.W, full.kp, full.vp
    for l in range(s.n_layers):
        ref = _oracle_ops(c, tr[l], m_all[step], l, s.prefix_len)
        for k, r in ref.items():
            err = rel_l2(tr[l][k], r)
            assert err < PER_OP_TOL, (l, k, err)


def test_velocity_teacher_forced_full(full):
    s = full.shape
    ts, dt = O.time_schedule(s.steps)
    M = O.time_modulation(ts, full.W.time_w1, full.W.time_w2)
    kp = [O.decode_bf16(k[0]) for k in full.kp]
    vp = [O.decode_bf16(v[0]) for v in full.vp]
    x = full.x0[0].astype(np.float64)
    for k in range(s.steps):
        v_ref = O.expert_velocity(x, M[k], full.W, kp, vp, s.rms_eps, s.rope_base, s.n_q_heads, s.n_kv_heads)
        if k in (0, 5, 9):
            v_gpu = full.e.velocity(x[None].astype(np.float32), k, s.steps)[0]
            assert rel_l2(v_gpu, v_ref) < 1e-2, (k, rel_l2(v_gpu, v_ref))
        x = x + dt * v_ref


def test_denoise_full_p256(full):
    s = full.shape
    ref = O.denoise(full.x0, s.steps, full.raw, full.kp, full.vp, s, W=full.W)
    xd = torch.from_numpy(full.x0).cuda()
    out = full.e.denoise(xd, s.steps).cpu().numpy()
    assert cosine(out, ref) >= 0.999
    assert max_abs(out, ref) <= 5e-2
    again = full.e.denoise(xd, s.steps).cpu().numpy()
    assert np.array_equal(out, again)


def test_denoise_p832_n50_a55():
    s = synth.WORKLOADS["lingbot_p832_n50_a55"]
    raw = synth.make_weights(s)
    W = O.Weights(raw)
    kp, vp = synth.make_prefix(s)
    x0 = synth.make_x0(s)
    e = Expert(s, raw)
    e.set_prefix(kp, vp, 1, s.prefix_len)
    out = e.denoise(x0, s.steps)
    vels = []
    ref = O.denoise(x0, s.steps, raw, kp, vp, s, W=W, velocities=vels)
    assert cosine(out, ref) >= 0.999
    assert max_abs(out, ref) <= 5e-2
    # teacher-forced spot check of the per-step velocity at the last step
    ts, dt = O.time_schedule(s.steps)
    x = x0[0].astype(np.float64)
    for k in range(s.steps - 1):
        x = x + dt * vels[0][k]
    v_gpu = e.velocity(x[None].astype(np.float32), s.steps - 1, s.steps)[0]
    assert rel_l2(v_gpu, vels[0][-1]) < 1e-2


def test_denoise_batch64_sampled_requests(full):
    s = synth.WORKLOADS["lingbot_b64_p256_n10"]
    kp, vp = synth.make_prefix(s)
    x0 = synth.make_x0(s)
    full.e.set_prefix(kp, vp, 64, s.prefix_len)
    out = full.e.denoise(x0, s.steps)
    for b in (0, 1, 63):
        ref = O.denoise(x0[b:b + 1], s.steps, full.raw, [k[b:b + 1] for k in kp], [v[b:b + 1] for v in vp],
                        s, W=full.W)
        assert cosine(out[b], ref[0]) >= 0.999, b
        assert max_abs(out[b], ref[0]) <= 5e-2, b
    # requests are independent: a permuted batch permutes the outputs bit-exactly
    perm = np.random.default_rng(0).permutation(64)
    full.e.set_prefix([k[perm].copy() for k in kp], [v[perm].copy() for v in vp], 64, s.prefix_len)
    outp = full.e.denoise(np.ascontiguousarray(x0[perm]), s.steps)
    assert np.array_equal(outp, out[perm])
    full.e.set_prefix(full.kp, full.vp, 1, BASE.prefix_len)
