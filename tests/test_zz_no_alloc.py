"""The allocation-free entry point, fm_time_modulation_noalloc.

Some callers cannot allocate device memory when they need the time
conditioning: a control loop or runtime whose device memory is fixed and
audited at start-up, or an embedder that hands the library only the buffers
it owns.  fm_time_modulation_noalloc serves them: it takes the caller's device
buffers and keeps its one intermediate in a library-owned device array.

Here it is called through the C ABI twice in a row and checked against the
oracle's time modulation (R1, R2) and against the handle-based
fm_time_modulation on the same weights, from 10 steps up to the array's limit
of 64 steps x d_model 1024 (the shared-memory opt-in above 48 KB included);
free device memory must not change across the first call; misaligned
pointers and sizes beyond the array are refused.  This file is collected last
on purpose, and it passes alone in a fresh process as well as after the other
tests."""
import numpy as np
import pytest

from oracle import fm_oracle as O
from tests._metrics import rel_l2
from vla_flow_matching_denoise_b200 import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

from vla_flow_matching_denoise_b200.binding import Expert, load  # noqa: E402

TOL = 5e-3     # the tolerance of the time-modulation parity tests


def _dev_bits(a: np.ndarray):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()


def _oracle(raw, steps):
    ts, _ = O.time_schedule(steps)
    return O.time_modulation(ts, O.decode_bf16(raw["time_w1"]), O.decode_bf16(raw["time_w2"]))


@pytest.mark.parametrize("shape,steps,with_handle", [
    (synth.WORKLOADS["tiny"], 10, True),
    (synth.ExpertShape(2, 1024, 16, 2, 128, 4096, 75, 256, 10), 10, True),    # d = 1024
    (synth.ExpertShape(1, 1024, 16, 2, 128, 4096, 75, 256, 32), 32, False),   # 64 KB of shared memory
    (synth.ExpertShape(1, 1024, 16, 2, 128, 4096, 75, 256, 64), 64, False),   # the whole array
])
def test_noalloc_matches_oracle_and_handle_on_two_calls(shape, steps, with_handle):
    lib = load()
    raw = synth.make_weights(shape)
    ref_o = _oracle(raw, steps)
    ref_h = None
    if with_handle:
        e = Expert(shape, raw)
        ref_h = e.time_modulation(steps)
        e.close()
    w1, w2 = _dev_bits(raw["time_w1"]), _dev_bits(raw["time_w2"])
    n_mod = shape.n_mod
    outs = []
    for i in range(2):
        out = torch.full((steps, n_mod), float("nan"), dtype=torch.float32, device="cuda")
        torch.cuda.synchronize()
        free0 = torch.cuda.mem_get_info()[0]
        st = lib.fm_time_modulation_noalloc(w1.data_ptr(), w2.data_ptr(), shape.d_model, n_mod, steps,
                                            out.data_ptr(), torch.cuda.current_stream().cuda_stream)
        assert st == 0, lib.fm_last_error(None)
        torch.cuda.synchronize()
        assert torch.cuda.mem_get_info()[0] == free0, "free device memory changed across the call"
        got = out.cpu().numpy()
        assert np.all(np.isfinite(got))
        assert rel_l2(got, ref_o) < TOL
        if ref_h is not None:
            assert rel_l2(got, ref_h) < TOL
        outs.append(got)
    assert np.array_equal(outs[0], outs[1])


def test_noalloc_rejects_sizes_beyond_its_array_and_misaligned_pointers():
    lib = load()
    w = torch.zeros(64, dtype=torch.int16, device="cuda")
    out = torch.zeros(64, dtype=torch.float32, device="cuda")
    for d, steps in ((2048, 10), (1024, 65), (100, 10)):
        st = lib.fm_time_modulation_noalloc(w.data_ptr(), w.data_ptr(), d, 16, steps, out.data_ptr(), None)
        assert st == 1
        assert b"out of range" in lib.fm_last_error(None)
    assert lib.fm_time_modulation_noalloc(None, w.data_ptr(), 256, 16, 10, out.data_ptr(), None) == 1
    for a, b, o in ((w.data_ptr() + 2, w.data_ptr(), out.data_ptr()),
                    (w.data_ptr(), w.data_ptr() + 2, out.data_ptr()),
                    (w.data_ptr(), w.data_ptr(), out.data_ptr() + 2)):
        assert lib.fm_time_modulation_noalloc(a, b, 256, 16, 10, o, None) == 1
        assert b"aligned" in lib.fm_last_error(None)
