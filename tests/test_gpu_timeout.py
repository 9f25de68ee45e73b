"""Failure detection on the device: a bounded wait that runs out.

Every wait of the one-request loop kernel is bounded (hand-off counters,
mbarriers, the weight ring, the cluster exchanges).  fm_test_stall makes the
QKV -> attention hand-off expect one writer that does not exist and gives every
wait a budget of about 1 ms.  The launch must then end early, the next
synchronising call must return FM_ERR_TIMEOUT, the device context must stay
usable, and normal runs afterwards -- on the same handle with the knob off and
on a fresh handle -- must match the oracle.  Nothing here faults or hangs the
GPU: the stalled wait gives up on its own and the kernel returns."""
import time

import numpy as np
import pytest

from oracle import fm_oracle as O
from tests._metrics import cosine, max_abs, rel_l2
from vla_flow_matching_denoise_b200 import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

from vla_flow_matching_denoise_b200.binding import Expert, FmError  # noqa: E402

FM_ERR_TIMEOUT = 5
SPIN_CYCLES = 2_000_000        # ~1 ms at the B200's 1.9-2.0 GHz SM clock


def test_stalled_handoff_times_out_and_the_context_recovers():
    s = synth.WORKLOADS["tiny"]
    raw = synth.make_weights(s)
    kp, vp = synth.make_prefix(s)
    x0 = synth.make_x0(s)
    W = O.Weights(raw)
    e = Expert(s, raw)
    e.set_prefix(kp, vp, 1, s.prefix_len)

    e.test_stall(True, SPIN_CYCLES)
    t0 = time.time()
    with pytest.raises(FmError) as err:
        e.velocity(x0, 0, s.steps)
    assert err.value.status == FM_ERR_TIMEOUT, str(err.value)
    assert time.time() - t0 < 30.0
    # a stalled denoise reports the timeout at the next synchronising call
    with pytest.raises(FmError) as err:
        e.denoise(x0, s.steps)
    assert err.value.status == FM_ERR_TIMEOUT, str(err.value)

    # knob off: the same handle computes the oracle's velocity again
    e.test_stall(False)
    ts, _ = O.time_schedule(s.steps)
    M = O.time_modulation(ts, W.time_w1, W.time_w2)
    kl = [O.decode_bf16(k[0]) for k in kp]
    vl = [O.decode_bf16(v[0]) for v in vp]
    v_ref = O.expert_velocity(x0[0].astype(np.float64), M[0], W, kl, vl, s.rms_eps, s.rope_base,
                              s.n_q_heads, s.n_kv_heads)
    v_gpu = e.velocity(x0, 0, s.steps)[0]
    assert rel_l2(v_gpu, v_ref) < 1e-2
    e.close()

    # a fresh handle runs a whole denoise that matches the oracle
    f = Expert(s, raw)
    f.set_prefix(kp, vp, 1, s.prefix_len)
    out = f.denoise(x0, s.steps)
    ref = O.denoise(x0, s.steps, raw, kp, vp, s, W=W)
    assert cosine(out, ref) >= 0.999 and max_abs(out, ref) <= 5e-2
    f.close()


def test_stall_knob_rejects_a_negative_budget():
    s = synth.WORKLOADS["tiny"]
    e = Expert(s, synth.make_weights(s))
    with pytest.raises(FmError):
        e.test_stall(True, -1)
    e.close()
