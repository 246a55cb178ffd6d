"""CPU checks of the top-k comparison rule used by the GPU parity tests: exact sets on the
oracle's float64 scores, with ties to the lower index, and an exemption only for pairs of
entries whose float64 scores differ by less than 1e-6 relative.  The planted case is built so
that the oracle's fp32 decision order (the one the kernel reproduces) and the float64 order
disagree at the boundary; a pair further apart than 1e-6 must not be exempt."""
import numpy as np

from tests import helpers as H


def test_planted_near_tie_separates_fp32_and_float64_orders(orc):
    n, k, a, b = 2048, 10, 500, 600
    ik, isc, q, w, big = H.planted_near_tie(n, k, a, b)
    s32, s64 = orc.indexer_scores(ik[0].numpy(), isc[0].numpy(), q[0].numpy(), w[0].numpy())
    assert s32[a] == s32[b] == 192.0                      # an fp32 tie ...
    assert s64[b] - s64[a] == 2.0 ** -26                  # ... that float64 resolves
    sel32 = orc.topk(s32, k)
    sel64 = orc.topk64(s64, k)
    assert np.array_equal(sel32, np.array(sorted(big + [a]), np.int32))
    assert np.array_equal(sel64, np.array(sorted(big + [b]), np.int32))
    assert H.near_tie_only(sel32, sel64, s64)
    seq = np.array([4 * n], np.int32)
    assert H.assert_topk_matches_f64(orc, sel32[None], ik.numpy(), isc.numpy(), seq, 4, q.numpy(), w.numpy(), k) == 1


def test_exemption_does_not_cover_distinct_scores(orc):
    s64 = np.array([5.0, 4.0, 3.0, 3.0 * (1 + 1e-4), 1.0])
    sel64 = orc.topk64(s64, 3)
    assert np.array_equal(sel64, [0, 1, 3])
    assert not H.near_tie_only(np.array([0, 1, 2], np.int32), sel64, s64)     # 1e-4 apart: a real error
    s64[3] = 3.0 * (1 + 1e-9)
    assert H.near_tie_only(np.array([0, 1, 2], np.int32), orc.topk64(s64, 3), s64)
    assert not H.near_tie_only(np.array([0, 1, 4], np.int32), orc.topk64(s64, 3), s64)   # wrong entry


def test_float64_rule_counts_and_padding(orc):
    """Short sequences: the GPU row must hold exactly min(k, n) entries and -1 padding."""
    ik = np.zeros((2, 16, 32), np.uint8)
    isc = np.ones((2, 16, 2), np.float32)
    q = np.ones((2, 4, 64), np.float32)
    w = np.ones((2, 4), np.float32)
    seq = np.array([4 * 3, 0], np.int32)
    good = np.array([[0, 1, 2, -1, -1], [-1] * 5], np.int32)
    assert H.assert_topk_matches_f64(orc, good, ik, isc, seq, 4, q, w, 5) == 0
    bad = np.array([[0, 1, -1, -1, -1], [-1] * 5], np.int32)
    try:
        H.assert_topk_matches_f64(orc, bad, ik, isc, seq, 4, q, w, 5)
    except AssertionError:
        return
    raise AssertionError("a short row was not flagged")
