"""Helpers shared by the GPU parity tests: tolerances and the near-tie rule for labels."""

import numpy as np

# Output tolerance at O(1) magnitudes: max-abs 2e-2, mean-abs 2e-3 against the fp64 oracle.
MAX_ABS = 2e-2
MEAN_ABS = 2e-3
# Two compressed scores closer than this (relative to the row's largest |score|) are a near tie.
NEAR_TIE_REL = 1e-5


def output_errors(gpu, ref):
    """(max-abs, mean-abs) over the entries the oracle computed (NaN marks rows outside a sample)."""
    g = np.asarray(gpu, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    ok = ~np.isnan(r)
    d = np.abs(g[ok] - r[ok])
    assert np.all(np.isfinite(g[ok])), "non-finite GPU output"
    return float(d.max()), float(d.mean())


def assert_outputs_close(gpu, ref, what=""):
    mx, mean = output_errors(gpu, ref)
    assert mx <= MAX_ABS and mean <= MEAN_ABS, f"{what}: max-abs {mx:.3e}, mean-abs {mean:.3e}"
    return mx, mean


def label_mismatches(gpu_mask, ref_mask, S, kc, kn, rows=None):
    """Count label mismatches and how many of them the near-tie rule excuses.

    A mismatch at block j of row i is excused iff S_ij lies within
    NEAR_TIE_REL * max_j |S_ij| of one of the scores on either side of the
    oracle's critical boundary (ranks kc-1, kc) or negligible boundary
    (ranks Nk-kn-1, Nk-kn).
    """
    gpu_mask = np.asarray(gpu_mask)
    ref_mask = np.asarray(ref_mask)
    Nk = ref_mask.shape[-1]
    flat_g = gpu_mask.reshape(-1, Nk)
    flat_r = ref_mask.reshape(-1, Nk)
    flat_s = np.asarray(S).reshape(-1, Nk)
    idx = range(flat_r.shape[0]) if rows is None else rows
    total = excused = 0
    for rix in idx:
        bad = np.nonzero(flat_g[rix] != flat_r[rix])[0]
        if len(bad) == 0:
            continue
        s = flat_s[rix]
        order = np.lexsort((np.arange(Nk), -s))
        ranked = s[order]
        bounds = []
        for rk in (kc - 1, kc, Nk - kn - 1, Nk - kn):
            if 0 <= rk < Nk:
                bounds.append(ranked[rk])
        tol = NEAR_TIE_REL * np.abs(s).max()
        for j in bad:
            total += 1
            if any(abs(s[j] - b) <= tol for b in bounds):
                excused += 1
    return total, excused
