"""Comparison helpers of the GPU parity tests (CUDA path against the fp64 oracle).

The tolerance metric is the relative L2 error over a whole flattened tensor,
computed separately for outputs and states; max-abs error is printed beside it
(shown with ``pytest -rP``).  On large tensors a handful of wrong rows can hide
under a whole-tensor norm, so the full-size tests also bound every row on its
own: a row is one (token, V head) output vector or one (sequence, V head) state
matrix.
"""

import numpy as np

TOL_F32 = 1e-4   # fp32 I/O, fp32 arithmetic throughout
TOL_BF16 = 1e-2  # bf16 I/O with fp32 state
# Per-row bound for bf16 I/O: rounding one 128-element row to bf16 alone gives a
# relative error of about 2e-3 to 4e-3; 5e-2 leaves room for the rows with the
# least favourable rounding while still failing any row that is wrong.
TOL_ROW_BF16 = 5e-2


def as_f64(x):
    if hasattr(x, "detach"):
        return x.detach().double().cpu().numpy()
    return np.asarray(x, np.float64)


def errs(x, ref):
    x, ref = as_f64(x), as_f64(ref)
    rel = float(np.linalg.norm(x - ref) / max(np.linalg.norm(ref), 1e-300))
    return rel, float(np.max(np.abs(x - ref))) if x.size else 0.0


def assert_close(x, ref, tol, what):
    rel, mx = errs(x, ref)
    print("%s: rel-L2 %.3e (tol %.0e), max-abs %.3e" % (what, rel, tol, mx))
    assert np.isfinite(rel) and rel <= tol, "%s: rel-L2 %.3e (tol %.0e), max-abs %.3e" % (what, rel, tol, mx)
    return rel, mx


def assert_rows_close(x, ref, row_dims, tol, what):
    """Relative L2 error of every row, rows being the first ``row_dims`` axes flattened.
    A row whose reference norm is below 0.1 of the median row norm is measured against that
    floor instead: a bf16 dot product of normalised vectors carries an absolute rounding
    error set by the vectors' scale, not by the product's value, so a row whose exact value
    is nearly zero (a query almost orthogonal to the only key left after a strong decay)
    has a large relative error that says nothing about the kernel.  A structurally wrong
    row (a missing or misplaced contribution) is off by the order of the median norm and
    still fails."""
    x, ref = as_f64(x), as_f64(ref)
    if x.size == 0:
        return 0.0
    nrows = int(np.prod(x.shape[:row_dims]))
    xr, rr = x.reshape(nrows, -1), ref.reshape(nrows, -1)
    rn = np.linalg.norm(rr, axis=1)
    floor = max(0.1 * float(np.median(rn)), 1e-300)
    rel = np.linalg.norm(xr - rr, axis=1) / np.maximum(rn, floor)
    worst = int(np.argmax(rel))
    idx = np.unravel_index(worst, x.shape[:row_dims])
    print("%s: worst row %s rel-L2 %.3e (tol %.0e)" % (what, tuple(int(i) for i in idx), rel[worst], tol))
    assert np.all(np.isfinite(rel)) and rel[worst] <= tol, \
        "%s: row %s rel-L2 %.3e > %.0e" % (what, tuple(int(i) for i in idx), rel[worst], tol)
    return float(rel[worst])
