"""The prefix cache builder (fm_set_prefix_builder / fm_build_prefix): each
layer's prefix K/V rows are computed on the device from that layer's prefix
hidden states, K = RoPE(x Wk^T) at positions 0 .. P-1 and V = x Wv^T ("LingBot-VLA
v2 Examples", Configuration / CUDA Graph: the 36-layer KV-cache construction
precedes the denoise steps).  Checked against the oracle's prefix_kv: the
stored bf16 rows (read back through fm_get_prefix_kv) and the denoised chunk
that attends to them."""
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

ROW_TOL = 4e-3      # rel-L2 of the stored bf16 rows (about one bf16 rounding)


def _oracle_cache(shape, builder, hidden, B, P):
    """Oracle K/V per layer, rounded to bf16 bits like the cache: [B, P, Hkv, hd]."""
    ks, vs, kf, vf = [], [], [], []
    for l, (wk, wv) in enumerate(builder):
        kl = np.empty((B, P, shape.n_kv_heads, shape.head_dim)); vl = np.empty_like(kl)
        for b in range(B):
            k, v = O.prefix_kv(O.decode_bf16(hidden[l][b]), O.decode_bf16(wk), O.decode_bf16(wv),
                               shape.n_kv_heads, shape.rope_base)
            kl[b], vl[b] = k, v
        kf.append(kl); vf.append(vl)
        ks.append(O.bf16_round_bits(kl)); vs.append(O.bf16_round_bits(vl))
    return ks, vs, kf, vf


def _run(shape, d_prefix, B, P, layers_checked, cos_bar=0.999, seed=0):
    raw = synth.make_weights(shape, seed)
    builder = synth.make_prefix_builder(shape, d_prefix, seed)
    hidden = synth.make_prefix_hidden(shape, d_prefix, seed, batch=B, prefix_len=P)
    x0 = synth.make_x0(dataclasses.replace(shape, batch=B), seed)
    e = Expert(shape, raw, max_prefix=max(P, 1), max_batch=B)
    e.set_prefix_builder(builder, d_prefix)
    e.build_prefix(hidden, B, P)
    ks, vs, kf, vf = _oracle_cache(shape, builder, hidden, B, P)
    for l in layers_checked:
        for b in range(B if P > 0 else 0):
            gk, gv = e.get_prefix_kv(l, b, P)
            assert rel_l2(O.decode_bf16(gk), kf[l][b]) < ROW_TOL, (l, b)
            assert rel_l2(O.decode_bf16(gv), vf[l][b]) < ROW_TOL, (l, b)
            # most stored rows round to exactly the oracle's bf16 value
            assert np.mean(gk == ks[l][b]) > 0.9 and np.mean(gv == vs[l][b]) > 0.9, (l, b)
    out = e.denoise(x0, shape.steps)
    W = O.Weights(raw)
    for b in range(B):
        ref = O.denoise(x0[b:b + 1], shape.steps, raw, [k[b:b + 1] for k in ks], [v[b:b + 1] for v in vs],
                        dataclasses.replace(shape, prefix_len=P), W=W)
        assert cosine(out[b], ref[0]) >= cos_bar, b
        assert max_abs(out[b], ref[0]) <= 5e-2, b
    return e


@pytest.mark.parametrize("B,P", [(1, 64), (3, 37), (2, 0)])
def test_build_prefix_tiny(B, P):
    shape = synth.WORKLOADS["tiny"]
    _run(shape, 192, B, P, range(shape.n_layers))


def test_build_prefix_wide_heads():
    # 16/2 heads of 128 (256-wide weight tiles: K heads then V heads), ragged rows
    shape = synth.ExpertShape(2, 256, 16, 2, 128, 1024, 75, 64, 10)
    _run(shape, 320, 2, 45, range(shape.n_layers))


def test_build_prefix_requires_builder():
    shape = synth.WORKLOADS["tiny"]
    e = Expert(shape, synth.make_weights(shape))
    hidden = synth.make_prefix_hidden(shape, 64, batch=1, prefix_len=8)
    with pytest.raises(RuntimeError):
        e.build_prefix(hidden, 1, 8)


@pytest.mark.slow
def test_build_prefix_full_size():
    """LingBot-shaped expert (36 layers) with a 2048-wide backbone, P = 256."""
    shape = synth.WORKLOADS["lingbot_p256_n10"]
    _run(shape, 2048, 1, shape.prefix_len, (0, shape.n_layers - 1))
