"""Comparison helpers for the GPU-vs-oracle parity tests: the bf16-output, lse and score tolerances and
the accepted top-k boundary swaps."""
from __future__ import annotations

import logging

import numpy as np
import torch

log = logging.getLogger("csa.parity")

OUT_ATOL, OUT_RTOL = 1e-2, 2e-2          # attention / compressor bf16 outputs
LSE_ATOL, LSE_RTOL = 1e-3, 1e-4
SCORE_RTOL = 1e-4                         # index scores: |d| <= 1e-4 (|s| + max|s| of the row)
BOUNDARY_RTOL = 1e-3                      # accepted top-k swaps at the k-th score


def f64(t):
    """torch tensor (any dtype, any device) -> float64 numpy."""
    return t.detach().to("cpu").to(torch.float64).numpy()


def np_u8(t):
    return t.detach().to("cpu").numpy().astype(np.uint8)


def assert_close(got, ref, atol, rtol, what=""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    both_inf = np.isinf(got) & np.isinf(ref) & (np.sign(got) == np.sign(ref))
    both_nan = np.isnan(got) & np.isnan(ref)
    with np.errstate(invalid="ignore"):
        err = np.abs(got - ref)
    err[both_inf | both_nan] = 0.0
    bad = err > atol + rtol * np.abs(np.where(both_inf | both_nan, 0.0, ref))
    # a NaN (or an infinity) on one side only is always a mismatch: NaN compares False above
    bad |= np.isnan(got) != np.isnan(ref)
    bad |= (np.isinf(got) | np.isinf(ref)) & ~both_inf
    if np.any(bad):
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {bad.sum()} / {bad.size} elements out of tolerance; first at {tuple(i)}: "
                             f"got {got[tuple(i)]}, ref {ref[tuple(i)]}")


def check_topk_row(gpu_idx, ref_scores, ref_ids, k, what=""):
    """GPU top-k set against the oracle's scores for one row.  ref_scores/ref_ids: every candidate's
    oracle score (-inf = not a candidate).  Exact set, or swaps only at the boundary (oracle scores of
    the swapped keys within BOUNDARY_RTOL of the k-th score).  Returns the number of accepted swaps."""
    gpu_idx = np.asarray(gpu_idx, np.int64)
    valid = np.isfinite(ref_scores)
    s = np.asarray(ref_scores)[valid]
    ids = np.asarray(ref_ids)[valid]
    order = np.lexsort((ids, -s))
    k_eff = min(k, len(order))
    ref_set = set(ids[order[:k_eff]].tolist())
    got = gpu_idx[gpu_idx >= 0]
    assert len(got) == k_eff, f"{what}: {len(got)} selected, expected {k_eff}"
    # slot order is unspecified: every slot is a selected id or the padding -1, and exactly k - k_eff
    # slots (of the k written) are padding
    assert np.all((gpu_idx >= 0) | (gpu_idx == -1)), f"{what}: slots other than ids and -1"
    assert int(np.sum(gpu_idx == -1)) == len(gpu_idx) - k_eff, f"{what}: padding count"
    got_set = set(got.tolist())
    assert len(got_set) == len(got), f"{what}: duplicate ids"
    if got_set == ref_set:
        return 0
    score_of = dict(zip(ids.tolist(), s.tolist()))
    kth = s[order[k_eff - 1]]
    diff = (got_set - ref_set) | (ref_set - got_set)
    for i in diff:
        assert i in score_of, f"{what}: id {i} is not a visible candidate"
        si = score_of[i]
        assert abs(si - kth) <= BOUNDARY_RTOL * max(abs(kth), 1e-30), \
            f"{what}: id {i} score {si} not at the boundary {kth}"
    log.warning("%s: %d boundary swap(s) accepted (k-th score %g)", what, len(diff) // 2, kth)
    return len(diff) // 2
