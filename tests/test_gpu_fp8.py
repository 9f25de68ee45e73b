"""GPU parity of the E4M3 weight variant ("LingBot-VLA on Thor (sm_110)", §2:
FP8 weights for the per-layer linears; the time MLP and the action in/out
projections stay bf16).

The handle quantises the per-layer linears itself (per output row
s = absmax / 448, codes = E4M3 nearest-even of w / s, saturating).  Checked:
  * the codes and row scales the handle streams, read back from its packed
    arena, equal the oracle's quantiser bit for bit, including rows that
    reach the E4M3 subnormals, an all-zero row and a single-outlier row;
  * per-op outputs on the op's own inputs against the oracle run on the
    dequantised weights q * s;
  * the final chunk against that oracle: cosine >= 0.995 (the bar for this
    variant), and per-step velocities (teacher-forced) at the bf16 bar.
Every call goes through the C ABI."""
import dataclasses

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
from tests.test_gpu_tiny import VEL_TOL, _check_trace  # noqa: E402

FP8_COS = 0.995        # final-chunk cosine bar of the E4M3 variant
LINEARS = ("wq", "wk", "wv", "wo", "w_gate", "w_up", "w_down")   # order of fm_get_fp8_weights' `which`


class Case:
    def __init__(self, shape, raw=None, seed=0):
        self.shape = shape
        self.raw = synth.make_weights(shape, seed) if raw is None else raw
        self.kp, self.vp = synth.make_prefix(shape, seed)
        self.x0 = synth.make_x0(shape, seed)
        self.W = O.Weights(self.raw, fp8=True)
        self.e = Expert(shape, self.raw)
        self.e.set_prefix(self.kp, self.vp, shape.batch, shape.prefix_len)


def _stress_weights(shape):
    """Seeded weights plus rows that reach the corners of the quantiser."""
    raw = synth.make_weights(shape, seed=3)
    rng = np.random.default_rng(11)
    lw = raw["layers"][0]
    wq = O.decode_bf16(lw["wq"], np.float32).copy()
    wq[0] = 0.0                                              # all-zero row: scale 1, codes 0
    wq[1] = rng.standard_normal(wq.shape[1]).astype(np.float32) * np.float32(2.0) ** rng.integers(-30, 0, wq.shape[1])
    wq[2] = 1e-3 * rng.standard_normal(wq.shape[1]).astype(np.float32)
    wq[2, 5] = -7.0                                          # one negative outlier: most codes subnormal
    wq[3] = np.float32(2.0) ** -100 * rng.standard_normal(wq.shape[1]).astype(np.float32)   # tiny row
    lw["wq"] = synth.f32_to_bf16_bits(wq)
    wd = O.decode_bf16(lw["w_down"], np.float32).copy()
    wd[:, ::7] *= 50.0                                       # columns far above the rest
    lw["w_down"] = synth.f32_to_bf16_bits(wd)
    return raw


@pytest.fixture(scope="module")
def tiny8():
    return Case(dataclasses.replace(synth.WORKLOADS["tiny"], fp8=True))


def _check_codes(case, layers):
    for l in layers:
        for which, key in enumerate(LINEARS):
            w = case.raw["layers"][l][key]
            codes, scale = case.e.get_fp8_weights(l, which, *w.shape)
            rc, rs = O.fp8_quantize_rows(w)
            assert np.array_equal(scale.view(np.uint32), rs.astype(np.float32).view(np.uint32)), (l, key)
            assert np.array_equal(codes, rc), (l, key, int(np.count_nonzero(codes != rc)))


def test_fp8_codes_and_scales_bit_exact(tiny8):
    _check_codes(tiny8, range(tiny8.shape.n_layers))


def test_fp8_codes_stress_rows():
    shape = dataclasses.replace(synth.WORKLOADS["tiny"], fp8=True)
    c = Case(shape, raw=_stress_weights(shape), seed=3)
    _check_codes(c, [0])
    codes, scale = c.e.get_fp8_weights(0, 0, *c.raw["layers"][0]["wq"].shape)
    assert scale[0] == 1.0 and not codes[0].any()
    assert np.any((codes[2] & 0x78) == 0) and np.any(codes[2] & 0x07)      # subnormal codes occur
    # the stressed expert still runs and matches its oracle
    s = c.shape
    ref = O.denoise(c.x0, s.steps, c.raw, c.kp, c.vp, s, W=c.W)
    out = c.e.denoise(c.x0, s.steps)
    assert cosine(out, ref) >= FP8_COS


def test_fp8_bf16_handle_rejects_codes_hook():
    shape = synth.WORKLOADS["tiny"]
    e = Expert(shape, synth.make_weights(shape))
    with pytest.raises(RuntimeError):
        e.get_fp8_weights(0, 0, shape.n_q_heads * shape.head_dim, shape.d_model)


def test_fp8_per_op_parity(tiny8):
    for k in (0, tiny8.shape.steps - 1):
        _check_trace(tiny8, tiny8.e, step=k)


def test_fp8_denoise_and_teacher_forced_velocity(tiny8):
    s = tiny8.shape
    vels = []
    ref = O.denoise(tiny8.x0, s.steps, tiny8.raw, tiny8.kp, tiny8.vp, s, W=tiny8.W, velocities=vels)
    out = tiny8.e.denoise(tiny8.x0, s.steps)
    assert cosine(out, ref) >= FP8_COS
    assert max_abs(out, ref) <= 5e-2
    ts, dt = O.time_schedule(s.steps)
    x = tiny8.x0[0].astype(np.float64)
    for k in range(s.steps):
        v = tiny8.e.velocity(x[None].astype(np.float32), k, s.steps)[0]
        assert rel_l2(v, vels[0][k]) < VEL_TOL, k
        x = x + dt * vels[0][k]
    again = tiny8.e.denoise(tiny8.x0, s.steps)
    assert np.array_equal(out, again)


@pytest.mark.slow
def test_fp8_full_size_p256():
    """The LingBot-shaped expert with E4M3 linears, in the benchmark's launch
    configuration: codes of two layers bit-exact, final chunk cosine, and the
    teacher-forced velocity of the first and last steps."""
    s = synth.WORKLOADS["lingbot_fp8_p256_n10"]
    c = Case(s)
    _check_codes(c, [0, s.n_layers - 1])
    vels = []
    ref = O.denoise(c.x0, s.steps, c.raw, c.kp, c.vp, s, W=c.W, velocities=vels)
    out = c.e.denoise(torch.from_numpy(c.x0).cuda(), s.steps).cpu().numpy()
    assert cosine(out, ref) >= FP8_COS
    assert max_abs(out, ref) <= 5e-2
    ts, dt = O.time_schedule(s.steps)
    x = c.x0[0].astype(np.float64)
    for k in range(s.steps):
        if k in (0, s.steps - 1):
            v = c.e.velocity(x[None].astype(np.float32), k, s.steps)[0]
            assert rel_l2(v, vels[0][k]) < VEL_TOL, k
        x = x + dt * vels[0][k]
