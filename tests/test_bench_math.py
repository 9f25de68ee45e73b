"""The benchmark's roofline arithmetic against figures worked out by hand
from the layer shapes (d 1024, 16/2 x 128 heads, F 4096, 36 layers, chunk
50 x 75, P 256, 10 Euler steps)."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from vla_flow_matching_denoise_b200 import synth  # noqa: E402

# per layer: wq 2048x1024, wk and wv 256x1024, wo 1024x2048, w_gate and w_up
# 4096x1024, w_down 1024x4096
PER_LAYER = 2048 * 1024 + 2 * 256 * 1024 + 1024 * 2048 + 2 * 4096 * 1024 + 1024 * 4096
ROWS = 2048 + 256 + 256 + 1024 + 4096 + 4096 + 1024          # output rows (one scale each)
IO = 2 * 1024 * 75                                              # in- and out-projection weights
KV = 36 * 2 * (256 + 50) * 2 * 128 * 2                          # one request's K and V, bf16


def test_hand_figures():
    assert PER_LAYER == 17_301_504 and ROWS == 12_800


def test_bf16_bytes_per_call():
    want = 10 * (36 * PER_LAYER * 2 + IO * 2 + KV)
    assert bench.loop_bytes(synth.WORKLOADS["lingbot_p256_n10"], 10, 1) == pytest.approx(want, rel=1e-12)
    assert want == pytest.approx(12.573e9, rel=1e-3)


def test_e4m3_bytes_per_call():
    want = 10 * (36 * (PER_LAYER + ROWS * 4) + IO * 2 + KV)
    assert bench.loop_bytes(synth.WORKLOADS["lingbot_fp8_p256_n10"], 10, 1) == pytest.approx(want, rel=1e-12)


def test_nvfp4_bytes_per_call():
    gu = 2 * 4096 * 1024
    rows8 = ROWS - 2 * 4096
    per_layer = (PER_LAYER - gu) + rows8 * 4 + gu * 0.5 + gu / 16 + 8
    want = 10 * (36 * per_layer + IO * 2 + KV)
    assert bench.loop_bytes(synth.WORKLOADS["lingbot_nvfp4_p256_n10"], 10, 1) == pytest.approx(want, rel=1e-12)


@pytest.mark.parametrize("name", ["lingbot_b64_p256_n10", "lingbot_w8a8_b64_p256_n10"])
def test_batched_flops_per_call(name):
    rows = 64 * 50
    lin = 2 * rows * (36 * PER_LAYER + IO)
    att = 4 * rows * 16 * (256 + 50) * 128 * 36
    want = 10 * (lin + att)
    assert bench.loop_flops(synth.WORKLOADS[name], 10, 64) == pytest.approx(want, rel=1e-12)
    assert want == pytest.approx(42.76e12, rel=1e-3)


def test_kernel_hash_ignores_comments_but_not_code(tmp_path, monkeypatch):
    # the traffic figure stays attached to an unchanged kernel across comment
    # edits, and is dropped when the code changes
    src = tmp_path / "vla_flow_matching_denoise_b200" / "csrc"
    src.mkdir(parents=True)
    names = ("fm_step.cu", "fm_ptx.cuh", "fm_internal.h")
    for n in names:
        (src / n).write_text("int f(int x) {\n  return x + 1;  // add one\n}\n/* block */\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.kernel_source_hash()
    (src / "fm_step.cu").write_text("// a new header\nint f(int x) {\n    return x + 1;  // plus one\n}\n")
    assert bench.kernel_source_hash() == h0
    (src / "fm_step.cu").write_text("int f(int x) {\n  return x + 2;\n}\n")
    assert bench.kernel_source_hash() != h0
