"""Phase timeline of the one-request loop kernel (fm_profile_phases).

fm_profile_phases runs one velocity evaluation per Euler step with every CTA
recording %globaltimer (32 ns resolution) at fixed points of every phase
(in-proj, then per layer QKV, attention, o_proj, gate_up, down, then the
out-projection).  This module runs it and reduces the marks to the per-phase
budget: for each phase kind, the median over CTAs and layers 1..L-1 of the
time between consecutive marks, where the first column is measured from the
previous phase's release (the latest writer's release add) to this CTA's
start.  The phase length is release to release.

    python -m vla_flow_matching_denoise_b200.phases lingbot_p256_n10

Marks (slot numbers of the kernel's phase record):
  0 start      the hand-off wait returned (activation copy requested)
  12 push      the compute warps reach the MMA-done wait
  1 mma        the MMAs of this CTA's K-slice are done
  2 pushed     split-K partials sent to their owners
  3 received   every partial of the owned columns arrived
  8 epi        epilogue starts
  4 epi_done   epilogue outputs stored
  13, 14       proxy fence, compute-warp barrier
  5 release    release add on the hand-off counter issued
The attention phase has no split-K marks (12, 8).
"""
from __future__ import annotations

import sys
from typing import Dict, List

import numpy as np

PHASES = ["qkv", "attn", "o_proj", "gate_up", "down"]
ORDER = [(0, "start"), (12, "push"), (1, "mma"), (2, "pushed"), (3, "received"), (8, "epi"),
         (4, "epi_done"), (13, "fenced"), (14, "synced"), (5, "release")]


def collect(workload: str = "lingbot_p256_n10", steps: int = 1, device: int = 0):
    """Runs fm_profile_phases twice (the first warms up) on the workload's
    synthetic inputs; returns the mark array [CTAs, phases, 16] (ns)."""
    from . import synth
    from .binding import Expert
    s = synth.WORKLOADS[workload]
    e = Expert(s, synth.make_weights(s), device=device)
    e.set_prefix(*synth.make_prefix(s), 1, s.prefix_len)
    for _ in range(2):
        m, _, _, _ = e.profile_phases(steps)
    e.close()
    return np.asarray(m)


def budget(m: np.ndarray) -> Dict[str, List[tuple]]:
    """Per phase kind: [(mark name, median µs since the previous mark)] and
    ('length', median release-to-release µs), over layers 1..L-1."""
    m = m.astype(np.int64)
    C, NP, _ = m.shape
    L = (NP - 2) // 5
    rel = m[:, :, 5]
    out: Dict[str, List[tuple]] = {}
    for k, name in enumerate(PHASES):
        ps = [1 + 5 * l + k for l in range(1, L)]
        R = np.array([rel[:, p - 1].max() for p in ps])
        rows = []
        prev = None
        for slot, label in ORDER:
            v = np.stack([m[:, p, slot] for p in ps], 1)
            if not (v > 0).any():
                continue
            if prev is None:
                dv, ok = v - R[None, :], v > 0
            else:
                dv, ok = v - prev, (v > 0) & (prev > 0)
            rows.append((label, float(np.median(dv[ok])) / 1e3))
            prev = v
        length = np.median([rel[:, p].max() - rel[:, p - 1].max() for p in ps]) / 1e3
        rows.append(("length", float(length)))
        out[name] = rows
    return out


def last_writer_clusters(m: np.ndarray, cluster: int = 8) -> Dict[str, np.ndarray]:
    """Per phase kind: how often each cluster held the phase's last release."""
    m = m.astype(np.int64)
    C, NP, _ = m.shape
    L = (NP - 2) // 5
    out = {}
    for k, name in enumerate(PHASES):
        cnt = np.zeros(C // cluster, dtype=int)
        for l in range(1, L):
            p = 1 + 5 * l + k
            r = m[:, p, 5]
            if (r > 0).any():
                cnt[int(np.argmax(np.where(r > 0, r, -1))) // cluster] += 1
        out[name] = cnt
    return out


def format_budget(b: Dict[str, List[tuple]]) -> str:
    lines = []
    for name, rows in b.items():
        lines.append(f"{name:8s} " + "  ".join(f"{lab} +{v:.2f}" if lab != "length" else f"| length {v:.2f}"
                                               for lab, v in rows))
    return "\n".join(lines)


def main(argv: List[str]) -> int:
    wl = argv[1] if len(argv) > 1 else "lingbot_p256_n10"
    steps = int(argv[2]) if len(argv) > 2 else 1
    m = collect(wl, steps)
    C, NP, _ = m.shape
    rel = m[:, :, 5].astype(np.int64)
    print(f"{wl}: {C} CTAs, {NP} phases; first to last release {(rel[:, -1].max() - rel[:, 0].max()) / 1e3:.1f} us")
    print(format_budget(budget(m)))
    for name, cnt in last_writer_clusters(m).items():
        print(f"last release by cluster ({name}): {cnt.tolist()}")
    return 0


if __name__ == "__main__":
    sys.exit(main(sys.argv))
