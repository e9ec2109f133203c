"""Comparison of a GPU result with the oracle, shared by the GPU parity tests.

Two bounds, both in relative L2 error:
  - the whole tensor (the bar every entry point is held to: 1e-5 in fp32 mode, 1.5e-2 in
    bf16-input / fp32-accumulate mode);
  - every row on its own (the last axis is a row; a 1-D or per-token tensor such as `den`
    is compared element by element), at ten times that bar, so that one wrong row, tile
    border or segment start cannot hide inside a whole-tensor norm.  A row's error is taken
    relative to the larger of its own norm and 1e-3 of the median row norm (rows that are
    exactly zero on both sides, such as zero queries, then count as exact).
Every comparison is recorded with its achieved error; conftest prints the list at the end
of the run, so the margins appear in the log of a quiet pytest run.
"""
import numpy as np

MARGINS = []
ROW_FACTOR = 10.0


def rel_l2(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def row_errors(got, want, per_element=False, row_scale=None):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    if per_element or got.ndim < 2:
        g2, w2 = got.reshape(-1, 1), want.reshape(-1, 1)
    else:
        g2, w2 = got.reshape(-1, got.shape[-1]), want.reshape(-1, want.shape[-1])
    rn = np.linalg.norm(w2, axis=1)
    if row_scale is not None:
        rn = np.maximum(rn, np.asarray(row_scale, np.float64).reshape(-1))
    en = np.linalg.norm(g2 - w2, axis=1)
    floor = max(float(np.median(rn)) * 1e-3, 1e-300)
    return en / np.maximum(rn, floor)


def check(name, got, want, tol, per_element=False, row_factor=ROW_FACTOR, row_mask=None,
          row_scale=None):
    """Assert the whole-tensor and per-row bounds; returns (whole, worst row).  row_mask
    (boolean, one entry per row) restricts the per-row bound to the rows it selects; the
    whole-tensor bound always covers every row.  row_scale (one entry per row) replaces a
    row's own norm as the denominator of its error where it is larger (see
    gradient_row_scale)."""
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert got.shape == want.shape, (name, got.shape, want.shape)
    assert np.isfinite(got).all(), name + ": non-finite values"
    whole = rel_l2(got, want)
    rows = row_errors(got, want, per_element, row_scale)
    if row_mask is not None:
        rows = np.where(np.asarray(row_mask, bool).reshape(-1), rows, 0.0)
    worst = float(rows.max()) if rows.size else 0.0
    at = int(rows.argmax()) if rows.size else -1
    shape = got.shape if per_element or got.ndim < 2 else got.shape[:-1]
    where = tuple(int(i) for i in np.unravel_index(at, shape)) if rows.size else ()
    MARGINS.append("%-58s rel_l2 %.3e (%.1f%% of %.1e)  worst row %.3e at %s (%d rows)"
                   % (name, whole, 100.0 * whole / tol, tol, worst, where, rows.size))
    assert whole <= tol, "%s: rel L2 %.3e > %.1e" % (name, whole, tol)
    assert worst <= row_factor * tol, "%s: worst row %.3e > %.1e" % (name, worst,
                                                                      row_factor * tol)
    return whole, worst


UNIT_ROUNDOFF = {"f32": 2.0 ** -24, "bf16": 2.0 ** -9}


def gradient_row_scale(exact, perturbed, dtype):
    """Per-row size of the terms that cancel in a gradient row.

    dphi(q_i) = S_i dn_i + z_i delta_i (and likewise dphi(k_j)) is a difference of two terms
    far larger than itself when row i's attention sits on a few keys; any rounding in the
    mode's dtype -- of the stored `out` the backward receives, or of the bf16 operands of its
    products -- then moves the row by about the unit roundoff times those terms.  `exact` is
    the oracle's gradient, `perturbed` the oracle's gradient at its own forward output
    rounded to `dtype` (oracle.attn_causal_bwd_given): their difference divided by the unit
    roundoff measures the cancelling terms.  The per-row bound of check() divides a row's
    error by the larger of its norm and this scale; the whole-tensor bound is unchanged."""
    e = np.asarray(exact, np.float64)
    p = np.asarray(perturbed, np.float64)
    return np.maximum(np.linalg.norm(e, axis=-1),
                      np.linalg.norm(p - e, axis=-1) / UNIT_ROUNDOFF[dtype])
