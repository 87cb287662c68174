"""Helpers shared by the GPU parity tests: device upload of generated inputs
and the comparison rules against the oracle.

Tolerances: per-value agreement within max(1e-3 absolute, 2e-3 relative) of
the fp64 oracle; selected sets (top-k tokens, top-h heads) identical except
for entries whose oracle score lies within 4x that tolerance of the
selection boundary (the k-th / h-th best oracle score).  Such boundary ties
are counted and returned so the tests can report them.
"""
from __future__ import annotations

import numpy as np

ABS_TOL = 1e-3
REL_TOL = 2e-3


def tol(x):
    return np.maximum(ABS_TOL, REL_TOL * np.abs(x))


def assert_close(gpu, ref, what=""):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (what, gpu.shape, ref.shape)
    err = np.abs(gpu - ref)
    bad = err > tol(ref)
    if bad.any():
        i = int(np.argmax(err - tol(ref)))
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} values out of tolerance; "
                             f"worst at {i}: gpu={gpu.flat[i]!r} oracle={ref.flat[i]!r}")


def compare_selection(gpu_sel, ref_sel, ref_score_of, n_keep, what=""):
    """Compare two selected sets (arrays with -1 padding).

    ref_score_of: callable token -> oracle score.  The boundary is the lowest
    oracle score inside the oracle's set.  Returns the number of boundary ties
    (entries in exactly one set); raises if any differing entry is farther
    than 4x the tolerance from the boundary, or if the padding differs.
    """
    g = [int(x) for x in gpu_sel if x >= 0]
    r = [int(x) for x in ref_sel if x >= 0]
    assert len(g) == len(set(g)), f"{what}: duplicate selections"
    assert len(g) == len(r), f"{what}: {len(g)} selected vs oracle {len(r)}"
    gs, rs = set(g), set(r)
    diff = gs ^ rs
    if not diff:
        return 0
    bound = min(ref_score_of(t) for t in rs)
    for t in diff:
        s = ref_score_of(t)
        assert abs(s - bound) <= 4 * float(tol(bound)), \
            f"{what}: token {t} (oracle score {s}) differs, boundary {bound}"
    return len(diff)


def to_device(inp, torch, device="cuda"):
    """Upload generator arrays; returns (KeyCache, Queries) of the binding."""
    from long_context_misa_b200 import misa as M
    return M.device_inputs(inp, device)
