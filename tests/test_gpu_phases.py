"""The loop kernel's phase timeline on the device (fm_profile_phases) and its
reduction: every CTA records every mark of every phase, in time order, and the
budget has a positive length for every phase kind."""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

from vla_flow_matching_denoise_b200 import phases  # noqa: E402


def test_phase_marks_are_ordered_and_reduce_to_a_budget():
    m = phases.collect("tiny", steps=1)
    C, NP, _ = m.shape
    assert NP >= 2 + 5 * 2
    rel = m[:, :, 5].astype(np.int64)
    # a phase's latest release never precedes the one before it
    last = rel.max(axis=0)
    assert np.all(np.diff(last) >= 0)
    # within a CTA that ran a phase, its start precedes its release
    ran = rel > 0
    assert np.all(m[:, :, 0][ran] <= rel[ran])
    b = phases.budget(m)
    for name, rows in b.items():
        assert dict(rows)["length"] > 0, name
