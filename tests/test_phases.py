"""The phase-budget reduction of the loop kernel's timeline (host logic, CPU).

A synthetic mark array with known gaps between marks must come back as those
gaps: per phase kind, the median over CTAs and layers 1..L-1 of the time
between consecutive marks, "start" measured from the previous phase's latest
release, and the release-to-release length."""
import numpy as np

from vla_flow_matching_denoise_b200 import phases

# mark slot -> gap (ns) after the previous mark of the same phase
GAPS = {0: 600, 12: 200, 1: 1600, 2: 900, 3: 200, 8: 100, 4: 1300, 13: 64, 14: 96, 5: 640}


def _synthetic(C=16, L=4, jitter=0):
    NP = 2 + 5 * L
    m = np.zeros((C, NP, 16), dtype=np.int64)
    rng = np.random.default_rng(0)
    t_release = 10_000
    for p in range(NP):
        last = t_release
        ends = []
        for c in range(C):
            t = last
            for slot, gap in GAPS.items():
                t += gap + (int(rng.integers(0, jitter + 1)) if jitter else 0)
                m[c, p, slot] = t
            ends.append(m[c, p, 5])
        t_release = max(ends)
    return m


def test_budget_returns_the_gaps_between_marks():
    m = _synthetic()
    b = phases.budget(m)
    assert list(b) == phases.PHASES
    for name, rows in b.items():
        got = dict(rows)
        assert abs(got["start"] - GAPS[0] / 1e3) < 1e-9, name
        assert abs(got["mma"] - GAPS[1] / 1e3) < 1e-9, name
        assert abs(got["release"] - GAPS[5] / 1e3) < 1e-9, name
        total = sum(GAPS.values()) / 1e3
        assert abs(got["length"] - total) < 1e-9, name


def test_last_writer_counts_cover_every_layer_but_the_first():
    m = _synthetic(C=16, L=4, jitter=50)
    counts = phases.last_writer_clusters(m, cluster=8)
    for name, cnt in counts.items():
        assert cnt.shape == (2,)
        assert cnt.sum() == 3, name   # layers 1..3


def test_format_lists_every_phase():
    text = phases.format_budget(phases.budget(_synthetic()))
    for name in phases.PHASES:
        assert name in text
