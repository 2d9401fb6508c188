"""Comparison helpers shared by the parity tests (no method arithmetic here).

Score tolerance.  A score is a signed sum of H terms w_j * ReLU(x_j); near zero
a per-element relative error is meaningless, so the bound is taken against the
sum's own condition scale mag = sum_j |w_j| * |x_j| (the oracle returns it):

    |gpu - ref| <= rtol * mag + 1e-6 * max_s |ref[row, s]|

with rtol = 1e-2 for FP8/bf16 inputs and 1e-4 for the fp32 path (the
tolerances the target states for FP8 and fp32 inputs; bf16 is held to the FP8
figure).  Top-k sets must be identical except for swaps among entries whose
oracle scores lie within that same relative tolerance of the k-th selected
oracle score: |ref[i] - ref_kth| <= rtol * |ref_kth| for every entry that one
set holds and the other does not.
"""
import numpy as np


def assert_scores_close(gpu, ref, mag, rtol, visible=None):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    if visible is None:
        visible = np.isfinite(ref)
    rowmax = np.max(np.where(visible, np.abs(ref), 0.0), axis=1, keepdims=True)
    bound = rtol * mag + 1e-6 * rowmax
    err = np.where(visible, np.abs(gpu - ref), 0.0)
    bad = err > bound
    if bad.any():
        r, s = np.argwhere(bad)[0]
        raise AssertionError(f"{bad.sum()} scores out of tolerance; first at row {r} pos {s}: "
                             f"gpu={gpu[r, s]!r} ref={ref[r, s]!r} bound={bound[r, s]!r}")


def assert_topk_equivalent(gpu_idx, ref_idx, ref_scores, rtol, n_valid=None, report=None):
    """Row by row: same size, ascending unique indices, equal sets up to near-ties.

    A swap is allowed only between entries whose oracle scores both lie within
    rtol * |k-th oracle score| of the k-th oracle score.  Returns the number of
    swapped entries (positions the GPU selected that the oracle did not); when
    `report` is a list, (row, swaps) is appended for every row that has any."""
    gpu_idx = np.asarray(gpu_idx)
    ref_idx = np.asarray(ref_idx)
    swaps = 0
    for r in range(gpu_idx.shape[0]):
        g = gpu_idx[r]
        f = ref_idx[r]
        gs = g[g >= 0]
        fs = f[f >= 0]
        assert len(gs) == len(fs), (r, len(gs), len(fs))
        assert np.all(g[len(gs):] == -1), r
        assert np.all(np.diff(gs) > 0), r
        if n_valid is not None:
            assert np.all(gs < n_valid[r]), r
        sg, sf = set(gs.tolist()), set(fs.tolist())
        if sg == sf:
            continue
        row = np.asarray(ref_scores[r], np.float64)
        kth = np.min(row[fs])
        band = rtol * abs(kth)
        for i in sg.symmetric_difference(sf):
            assert abs(row[i] - kth) <= band, (r, i, row[i], kth, band)
        n = len(sg - sf)
        swaps += n
        if report is not None:
            report.append((r, n))
    return swaps
