"""Failure message for an expert-index mismatch between the GPU and the oracle.

A mismatch always fails the test.  The message says whether the oracle's own
selection was a near tie: the gap between its K-th and (K+1)-th largest logits below
1e-12 of the largest |logit| (the fp64 sums of both sides differ in order, so only
such a gap could make two correct implementations pick different experts).  |logit|
stands in for the sum of |w_c x_c| of the row, which it never exceeds, so the label
errs towards "not a tie".
"""
import numpy as np

NEAR_TIE_REL = 1e-12


def selection_gap(logits, K):
    """(gap between the K-th and (K+1)-th largest logits, largest |logit|), or
    (None, None) when there is no (K+1)-th expert."""
    l = np.sort(np.asarray(logits, dtype=np.float64))[::-1]
    if l.size <= K:
        return None, None
    return float(l[K - 1] - l[K]), float(np.max(np.abs(l)))


def index_mismatch(ctx, got, want, logits=None):
    msg = f"{ctx}: idx {[int(i) for i in got]} vs oracle {[int(i) for i in want]}"
    if logits is None:
        return msg
    gap, scale = selection_gap(logits, len(want))
    if gap is None:
        return msg
    kind = "a near tie" if gap < NEAR_TIE_REL * max(scale, 1e-300) else "not a tie"
    return msg + f"; oracle gap between logits K and K+1: {gap:.3e} ({kind})"
