"""Per-request prefix lengths (fm_set_prefix_varlen): the prefix K/V of a
batch is padded to p_pad rows and request b holds P_b valid rows ("LingBot-VLA
v2 Examples", Configuration / CUDA Graph: language padding masks reuse the
denoising graph; "api.py", state_prompt_mode "fixed": a device-side valid
length).  Request b must then equal the oracle run on its own P_b keys, with
chunk RoPE positions P_b .. P_b+T-1; the lengths live on the device, so new
lengths reuse the captured graph.  Covered on the batched path (bf16, B >= 2),
on the per-request latency path (E4M3 handle, B = 3) and at B = 1."""
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
from tests.test_gpu_tiny import VEL_TOL  # noqa: E402

P_PAD = 64


def _padded_prefix(shape, B, seed):
    s = dataclasses.replace(shape, batch=B, prefix_len=P_PAD)
    return synth.make_prefix(s, seed=seed)


def _check_requests(e, shape, raw, W, kp, vp, x0, lens, cos_bar=0.999):
    out = e.denoise(x0, shape.steps)
    for b, P in enumerate(lens):
        kb = [k[b:b + 1, :P] for k in kp]
        vb = [v[b:b + 1, :P] for v in vp]
        ref = O.denoise(x0[b:b + 1], shape.steps, raw, kb, vb, dataclasses.replace(shape, prefix_len=P), W=W)
        assert cosine(out[b], ref[0]) >= cos_bar, (b, P)
        assert max_abs(out[b], ref[0]) <= 5e-2, (b, P)
    return out


def test_varlen_batched_and_length_change_without_recapture():
    shape = synth.WORKLOADS["tiny"]
    B = 4
    raw = synth.make_weights(shape)
    W = O.Weights(raw)
    kp, vp = _padded_prefix(shape, B, seed=5)
    x0 = synth.make_x0(dataclasses.replace(shape, batch=B), seed=5)
    e = Expert(shape, raw, max_prefix=P_PAD, max_batch=B)
    lens = [64, 0, 37, 13]
    e.set_prefix_varlen(kp, vp, B, lens, P_PAD)
    _check_requests(e, shape, raw, W, kp, vp, x0, lens)
    # teacher-forced velocity of request 2 at the first and last steps
    vels = []
    O.denoise(x0[2:3], shape.steps, raw, [k[2:3, :37] for k in kp], [v[2:3, :37] for v in vp],
              dataclasses.replace(shape, prefix_len=37), W=W, velocities=vels)
    v0 = e.velocity(x0, 0, shape.steps)
    assert rel_l2(v0[2], vels[0][0]) < VEL_TOL
    # new lengths, same (batch, steps): the captured graph is reused
    lens2 = [1, 64, 50, 7]
    e.set_prefix_varlen(kp, vp, B, lens2, P_PAD)
    _check_requests(e, shape, raw, W, kp, vp, x0, lens2)


def test_varlen_equal_lengths_match_fixed_prefix_bit_exactly():
    shape = synth.WORKLOADS["tiny"]
    B = 3
    raw = synth.make_weights(shape)
    kp, vp = _padded_prefix(shape, B, seed=8)
    x0 = synth.make_x0(dataclasses.replace(shape, batch=B), seed=8)
    e = Expert(shape, raw, max_prefix=P_PAD, max_batch=B)
    e.set_prefix(kp, vp, B, P_PAD)
    a = e.denoise(x0, shape.steps)
    e.set_prefix_varlen(kp, vp, B, [P_PAD] * B, P_PAD)
    b = e.denoise(x0, shape.steps)
    assert np.array_equal(a, b)


def test_varlen_latency_path_e4m3_and_single_request():
    shape = dataclasses.replace(synth.WORKLOADS["tiny"], fp8=True)
    raw = synth.make_weights(shape)
    W = O.Weights(raw, fp8=True)
    B = 3
    kp, vp = _padded_prefix(shape, B, seed=9)
    x0 = synth.make_x0(dataclasses.replace(shape, batch=B), seed=9)
    e = Expert(shape, raw, max_prefix=P_PAD, max_batch=B)
    lens = [5, 64, 20]
    e.set_prefix_varlen(kp, vp, B, lens, P_PAD)
    _check_requests(e, shape, raw, W, kp, vp, x0, lens, cos_bar=0.995)
    # B = 1 (bf16) with a length below the padded one
    s1 = synth.WORKLOADS["tiny"]
    raw1 = synth.make_weights(s1)
    e1 = Expert(s1, raw1, max_prefix=P_PAD)
    e1.set_prefix_varlen([k[:1] for k in kp], [v[:1] for v in vp], 1, [29], P_PAD)
    _check_requests(e1, s1, raw1, O.Weights(raw1), [k[:1] for k in kp], [v[:1] for v in vp], x0[:1], [29])


def test_varlen_rejects_bad_lengths():
    shape = synth.WORKLOADS["tiny"]
    raw = synth.make_weights(shape)
    kp, vp = _padded_prefix(shape, 2, seed=1)
    e = Expert(shape, raw, max_prefix=P_PAD, max_batch=2)
    with pytest.raises(RuntimeError):
        e.set_prefix_varlen(kp, vp, 2, [10, 65], P_PAD)          # beyond p_pad
    with pytest.raises(RuntimeError):
        e.set_prefix_varlen(kp, vp, 2, [10, -1], P_PAD)
    with pytest.raises(RuntimeError):
        e.set_prefix_varlen(kp, vp, 2, [10, 10], P_PAD + 1)      # beyond max_prefix
