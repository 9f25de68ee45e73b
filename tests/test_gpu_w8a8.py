"""GPU parity of the W8A8 variant: E4M3 per-row weights (R8) and per-token
E4M3 inputs of the four per-layer linears (R11), every batch size on the
batched tensor-core path (tcgen05 kind::f8f6f4 GEMMs; "LingBot-VLA on Thor
(sm_110)", §2: FP8 linears).

Checked through the C ABI:
  * the E4M3 codes and row scales in the handle's tile arena equal the
    oracle's quantiser bit for bit;
  * the final chunk against the W8A8 oracle run per request: cosine >= 0.995
    (the bar of the FP8 variants), max-abs <= 5e-2, on batches with a ragged
    last 128-row tile, B = 1 included, and on an expert with LingBot's head
    and FFN widths; the teacher-forced velocity of every step;
  * the row quantiser the path runs on the attention and SwiGLU outputs
    gives R11's codes and scales bit for bit (zero, outlier, tiny, huge
    rows and exact ties);
  * determinism and request independence (a permuted batch permutes the
    outputs bit for bit);
  * the one-request trace hook is refused."""
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

W8A8_COS = 0.995
# per-step velocity bar, derived: the two sides quantise inputs that differ by
# the GPU's bf16 rounding (delta ~ 2^-9/sqrt(3) ~ 1.1e-3 RMS relative); with
# E4M3 steps of rho ~ 2^-3.5 ~ 0.088 of the value a code moves with
# probability delta/rho and then by rho, so the quantised inputs differ by
# sqrt(delta * rho) ~ 1.0e-2 RMS relative; the bar is twice that estimate
W8A8_VEL_TOL = 2e-2
LINEARS = ("wq", "wk", "wv", "wo", "w_gate", "w_up", "w_down")

TINY = dataclasses.replace(synth.WORKLOADS["tiny"], w8a8=True)
# LingBot's head and FFN widths (o_proj K = 2048, down K = 4096), 2 layers
WIDE = synth.ExpertShape(2, 256, 16, 2, 128, 4096, 75, 64, 10, w8a8=True)


def _request(kp, vp, b):
    return [k[b:b + 1] for k in kp], [v[b:b + 1] for v in vp]


def test_w8a8_codes_and_scales_bit_exact():
    s = dataclasses.replace(TINY, batch=2)
    raw = synth.make_weights(s, seed=5)
    e = Expert(s, raw, max_batch=2)
    for l in range(s.n_layers):
        for which, key in enumerate(LINEARS):
            w = raw["layers"][l][key]
            codes, scale = e.get_fp8_weights(l, which, *w.shape)
            rc, rs = O.fp8_quantize_rows(w)
            assert np.array_equal(scale.view(np.uint32), rs.astype(np.float32).view(np.uint32)), (l, key)
            assert np.array_equal(codes, rc), (l, key, int(np.count_nonzero(codes != rc)))
    with pytest.raises(RuntimeError):
        e.trace_velocity(synth.make_x0(s, batch=1)[0], 0, s.steps)


@pytest.mark.parametrize("base,B,P", [("tiny", 1, 64), ("tiny", 3, 37), ("tiny", 5, 0), ("wide", 3, 64)])
def test_w8a8_matches_oracle_per_request(base, B, P):
    s = dataclasses.replace(WIDE if base == "wide" else TINY, batch=B, prefix_len=P)
    raw = synth.make_weights(s)
    W = O.Weights(raw, fp8=True)
    kp, vp = synth.make_prefix(s, seed=B)
    x0 = synth.make_x0(s, seed=B)
    e = Expert(s, raw, max_prefix=64, max_batch=8)
    e.set_prefix(kp, vp, B, P)
    out = e.denoise(x0, s.steps)
    ts, dt = O.time_schedule(s.steps)
    refs = []
    for b in range(B):
        kb, vb = _request(kp, vp, b)
        vels = []
        ref = O.denoise(x0[b:b + 1], s.steps, raw, kb, vb, s, W=W, velocities=vels, act_fp8=True)
        assert cosine(out[b], ref[0]) >= W8A8_COS, b
        assert max_abs(out[b], ref[0]) <= 5e-2, b
        refs.append(vels[0])
    x = x0.astype(np.float64)
    for k in range(s.steps):
        v = e.velocity(x.astype(np.float32), k, s.steps)
        for b in range(B):
            assert rel_l2(v[b], refs[b][k]) < W8A8_VEL_TOL, (k, b)
            x[b] = x[b] + dt * refs[b][k]
    assert np.array_equal(out, e.denoise(x0, s.steps))


def _act_rows(M, K, seed):
    """bf16 rows that reach the corners of the per-token quantiser."""
    rng = np.random.default_rng(seed)
    y = rng.standard_normal((M, K)).astype(np.float32) * np.float32(2.0) ** rng.integers(-8, 8, (M, 1))
    y[0] = 0.0                                                   # zero row: scale 1, codes 0
    y[1] = 0.1 * rng.standard_normal(K).astype(np.float32)
    y[1, 7] = -1e4                                               # one outlier: most codes subnormal
    y[2] = 0.0
    y[2, :6] = [448.0, 1.0625, 1.1875, 2.0 ** -10, 3 * 2.0 ** -10, -3.0]   # s = 1: ties to even
    y[3] *= np.float32(2.0) ** -100                              # tiny row
    y[4] *= np.float32(1e30)                                     # huge row
    y[5] = -np.abs(y[5])
    return synth.f32_to_bf16_bits(y)


@pytest.mark.parametrize("M,K", [(130, 256), (6, 4096), (200, 2048)])
def test_w8a8_activation_quantiser_bit_exact(M, K):
    """The row-quantiser kernel the W8A8 path runs on o and u, through the
    C ABI, against R11's codes and scales, bit for bit."""
    s = dataclasses.replace(TINY, batch=1)
    e = Expert(s, synth.make_weights(s), max_batch=1)
    x = _act_rows(M, K, seed=M + K)
    codes, scales = e.quantize_act_e4m3(x)
    rc, rs = O.fp8_quantize_act(O.decode_bf16(x, np.float32))
    assert np.array_equal(scales.view(np.uint32), rs.view(np.uint32))
    assert np.array_equal(codes, rc), int(np.count_nonzero(codes != rc))
    assert scales[0] == 1.0 and not codes[0].any()
    assert np.count_nonzero(codes[1] & 0x78) < K // 2          # the outlier row is mostly subnormal / zero
    assert list(codes[2, :6]) == [0x7E, 0x38, 0x3A, 0x00, 0x02, 0xC4]


def test_w8a8_requests_are_independent():
    s = dataclasses.replace(TINY, batch=6)
    raw = synth.make_weights(s)
    kp, vp = synth.make_prefix(s, seed=7)
    x0 = synth.make_x0(s, seed=7)
    e = Expert(s, raw, max_batch=6)
    e.set_prefix(kp, vp, 6, s.prefix_len)
    out = e.denoise(x0, s.steps)
    perm = np.array([3, 0, 5, 1, 4, 2])
    e.set_prefix([k[perm].copy() for k in kp], [v[perm].copy() for v in vp], 6, s.prefix_len)
    outp = e.denoise(np.ascontiguousarray(x0[perm]), s.steps)
    assert np.array_equal(outp, out[perm])
    # one request alone gives the same rows as inside the batch
    e.set_prefix([k[:1].copy() for k in kp], [v[:1].copy() for v in vp], 1, s.prefix_len)
    one = e.denoise(np.ascontiguousarray(x0[:1]), s.steps)
    assert np.array_equal(one[0], out[0])


@pytest.mark.slow
def test_w8a8_full_size_b64_sampled():
    """The LingBot-shaped W8A8 expert with 64 requests, in the benchmark's
    launch configuration: codes of one layer bit-exact, and requests 0 and 63
    against the W8A8 oracle."""
    s = synth.WORKLOADS["lingbot_w8a8_b64_p256_n10"]
    raw = synth.make_weights(s)
    kp, vp = synth.make_prefix(s)
    x0 = synth.make_x0(s)
    e = Expert(s, raw)
    for which, key in enumerate(LINEARS):
        w = raw["layers"][s.n_layers - 1][key]
        codes, scale = e.get_fp8_weights(s.n_layers - 1, which, *w.shape)
        rc, rs = O.fp8_quantize_rows(w)
        assert np.array_equal(codes, rc) and np.array_equal(scale, rs.astype(np.float32)), key
    e.set_prefix(kp, vp, s.batch, s.prefix_len)
    out = e.denoise(torch.from_numpy(x0).cuda(), s.steps).cpu().numpy()
    W = O.Weights(raw, fp8=True)
    for b in (0, s.batch - 1):
        kb, vb = _request(kp, vp, b)
        ref = O.denoise(x0[b:b + 1], s.steps, raw, kb, vb, s, W=W, act_fp8=True)
        assert cosine(out[b], ref[0]) >= W8A8_COS, b
        assert max_abs(out[b], ref[0]) <= 5e-2, b
