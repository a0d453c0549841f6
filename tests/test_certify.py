"""The near-tie certificate the GPU selection tests rely on (parity_util.certify_near_ties)
is not vacuous: it accepts identical selections, accepts a swap at a genuine near-tie, and
rejects a selection that swaps a clear winner for a clear loser."""
import numpy as np
import pytest

from parity_util import certify_near_ties


def _scores(lm, q, G):
    B, Hkv, nC, hd = lm.shape
    s = np.empty((B, Hkv, nC))
    for b in range(B):
        for g in range(Hkv):
            s[b, g] = (lm[b, g] @ q[b, g * G:(g + 1) * G].T).max(axis=1)
    return s


def test_certificate_accepts_equal_and_rejects_clear_swaps():
    rng = np.random.default_rng(1)
    B, Hkv, G, hd, nC = 1, 1, 2, 64, 50
    lm = rng.standard_normal((B, Hkv, nC, hd))
    q = rng.standard_normal((B, Hkv * G, hd))
    s = _scores(lm, q, G)
    order = np.argsort(-s[0, 0], kind="stable")
    sel_o = np.sort(order[:5])[None, None]
    sel_bad = np.sort(np.r_[order[:4], order[40]])[None, None]
    assert certify_near_ties(lm, lm, q, sel_o, sel_o, s, G, 5, 0, 0) == 0
    with pytest.raises(AssertionError):
        certify_near_ties(lm, lm, q, sel_bad, sel_o, s, G, 5, 0, 0)


def test_certificate_accepts_a_swap_at_a_perturbed_near_tie():
    """Two chunks whose scores differ by less than the landmark change can swap."""
    rng = np.random.default_rng(2)
    B, Hkv, G, hd, nC = 1, 1, 1, 16, 20
    lm = rng.standard_normal((B, Hkv, nC, hd))
    q = rng.standard_normal((B, Hkv * G, hd))
    s = _scores(lm, q, G)
    order = np.argsort(-s[0, 0], kind="stable")
    k = 6
    a, c = order[k - 1], order[k]               # the k-th and the (k+1)-th
    lm_g = lm.copy()
    gap = s[0, 0, a] - s[0, 0, c]
    j = int(np.argmax(np.abs(q[0, 0])))
    lm_g[0, 0, c, j] += 1.01 * gap / q[0, 0, j]    # the GPU side's landmark lifts c over a
    s_g = _scores(lm_g, q, G)
    sel_g = np.sort(np.argsort(-s_g[0, 0], kind="stable")[:k])[None, None]
    sel_o = np.sort(order[:k])[None, None]
    assert not np.array_equal(sel_g, sel_o)
    assert certify_near_ties(lm_g, lm, q, sel_g, sel_o, s, G, k, 0, 0) == 1
    # the same swap without the landmark change behind it is rejected
    with pytest.raises(AssertionError):
        certify_near_ties(lm, lm, q, sel_g, sel_o, s, G, k, 0, 0)
