"""The allocation-free entry point, fm_time_modulation_noalloc.

Some callers cannot allocate device memory when they need the time
conditioning (a control loop or runtime whose device memory is fixed at
start-up).  fm_time_modulation_noalloc serves them: it takes the
caller's device buffers and keeps its one intermediate in a library-owned
device array.  Here it is called through the C ABI twice in a row and checked
against the handle-based fm_time_modulation on the same weights.  This file is
collected last on purpose, and it passes alone in a fresh process as well as
after the other tests."""
import ctypes

import numpy as np
import pytest

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


@pytest.mark.parametrize("shape", [
    synth.WORKLOADS["tiny"],
    synth.ExpertShape(2, 1024, 16, 2, 128, 4096, 75, 256, 10),    # full width d = 1024
])
def test_noalloc_matches_handle_entry_point_on_two_calls(shape):
    lib = load()
    raw = synth.make_weights(shape)
    e = Expert(shape, raw)
    steps = shape.steps
    ref = e.time_modulation(steps)
    e.close()
    w1, w2 = _dev_bits(raw["time_w1"]), _dev_bits(raw["time_w2"])
    n_mod = shape.n_mod
    outs = []
    for _ in range(2):
        out = torch.full((steps, n_mod), float("nan"), dtype=torch.float32, device="cuda")
        st = lib.fm_time_modulation_noalloc(w1.data_ptr(), w2.data_ptr(), shape.d_model, n_mod, steps,
                                            out.data_ptr(), torch.cuda.current_stream().cuda_stream)
        assert st == 0, lib.fm_last_error(None)
        torch.cuda.synchronize()
        got = out.cpu().numpy()
        assert np.all(np.isfinite(got))
        assert rel_l2(got, ref) < TOL
        outs.append(got)
    assert np.array_equal(outs[0], outs[1])


def test_noalloc_rejects_sizes_beyond_its_array():
    lib = load()
    w = torch.zeros(16, dtype=torch.int16, device="cuda")
    out = torch.zeros(16, dtype=torch.float32, device="cuda")
    for d, steps in ((2048, 10), (1024, 65), (100, 10)):
        st = lib.fm_time_modulation_noalloc(w.data_ptr(), w.data_ptr(), d, 16, steps, out.data_ptr(), None)
        assert st == 1
        assert b"out of range" in lib.fm_last_error(None)
    assert lib.fm_time_modulation_noalloc(None, w.data_ptr(), 256, 16, 10, out.data_ptr(), None) == 1
