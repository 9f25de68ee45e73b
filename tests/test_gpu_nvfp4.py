"""GPU parity of the NVFP4 gate_up variant ("LingBot-VLA on Thor (sm_110)", §1:
FP8 weights with an FP4 gate_up): wq/wk/wv/wo/w_down in E4M3 with row scales
(R8), w_gate and w_up in NVFP4 (R10: E2M1 codes, one E4M3 scale per 16 inputs,
one fp32 scale per tensor).  The handle quantises on the device; the step
kernel widens the codes to bf16 in shared memory (exact) and applies the
tensor scale to the reduced fp32 sums.

Checked: codes, block scales and tensor scales read back from the packed arena
equal the oracle's quantiser bit for bit (the E4M3 linears too); per-op outputs
and per-step velocities against the oracle on the dequantised weights; the
final chunk at cosine >= 0.995 (the bar of the quantised variants)."""
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

COS = 0.995
FP8_LINEARS = {0: "wq", 1: "wk", 2: "wv", 3: "wo", 6: "w_down"}


class Case:
    def __init__(self, shape, seed=0):
        self.shape = shape
        self.raw = synth.make_weights(shape, seed)
        self.kp, self.vp = synth.make_prefix(shape, seed)
        self.x0 = synth.make_x0(shape, seed)
        self.W = O.Weights(self.raw, nvfp4_gu=True)
        self.e = Expert(shape, self.raw)
        self.e.set_prefix(self.kp, self.vp, shape.batch, shape.prefix_len)


def _check_codes(case, layers):
    for l in layers:
        for which, key in ((4, "w_gate"), (5, "w_up")):
            w = case.raw["layers"][l][key]
            codes, sb, g = case.e.get_nvfp4_weights(l, which, *w.shape)
            rc, rsb, rg = O.nvfp4_quantize(w)
            assert np.float32(g).view(np.uint32) == np.float32(rg).view(np.uint32), (l, key)
            assert np.array_equal(sb, rsb), (l, key, int(np.count_nonzero(sb != rsb)))
            assert np.array_equal(codes, rc), (l, key, int(np.count_nonzero(codes != rc)))
        for which, key in FP8_LINEARS.items():
            w = case.raw["layers"][l][key]
            codes, scale = case.e.get_fp8_weights(l, which, *w.shape)
            rc, rs = O.fp8_quantize_rows(w)
            assert np.array_equal(codes, rc) and np.array_equal(scale.view(np.uint32), rs.view(np.uint32)), (l, key)


@pytest.fixture(scope="module")
def tiny4():
    return Case(dataclasses.replace(synth.WORKLOADS["tiny"], nvfp4_gu=True))


def test_nvfp4_codes_scales_bit_exact(tiny4):
    _check_codes(tiny4, range(tiny4.shape.n_layers))
    with pytest.raises(RuntimeError):
        tiny4.e.get_fp8_weights(0, 4, *tiny4.raw["layers"][0]["w_gate"].shape)


def test_nvfp4_per_op_parity(tiny4):
    for k in (0, tiny4.shape.steps - 1):
        _check_trace(tiny4, tiny4.e, step=k)


def test_nvfp4_denoise_and_velocity(tiny4):
    s = tiny4.shape
    vels = []
    ref = O.denoise(tiny4.x0, s.steps, tiny4.raw, tiny4.kp, tiny4.vp, s, W=tiny4.W, velocities=vels)
    out = tiny4.e.denoise(tiny4.x0, s.steps)
    assert cosine(out, ref) >= COS
    assert max_abs(out, ref) <= 5e-2
    ts, dt = O.time_schedule(s.steps)
    x = tiny4.x0[0].astype(np.float64)
    for k in range(s.steps):
        v = tiny4.e.velocity(x[None].astype(np.float32), k, s.steps)[0]
        assert rel_l2(v, vels[0][k]) < VEL_TOL, k
        x = x + dt * vels[0][k]


@pytest.mark.slow
def test_nvfp4_full_size():
    s = synth.WORKLOADS["lingbot_nvfp4_p256_n10"]
    c = Case(s)
    _check_codes(c, [0, s.n_layers - 1])
    ref = O.denoise(c.x0, s.steps, c.raw, c.kp, c.vp, s, W=c.W)
    out = c.e.denoise(torch.from_numpy(c.x0).cuda(), s.steps).cpu().numpy()
    assert cosine(out, ref) >= COS
    assert max_abs(out, ref) <= 5e-2
