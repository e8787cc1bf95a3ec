"""Pins of the chunk-overlap oracle (paper Sec. 7.2) by cases whose answer
is fixed by the definition: identical selections (Overlap 1, full reuse),
disjoint selections (Overlap 0, no reuse), a hand-counted small case, and
-1 padding ignored."""
import numpy as np

from oracle import overlap as ov


def test_identical_rows_overlap_one():
    M, K = 4, 3
    idx = np.tile(np.array([2, 5, 9], dtype=np.int32), (1, 1, 2 * M, 1))
    s, u, r = ov.block_counts(idx, M)
    assert (s == M * K).all() and (u == K).all()
    assert r[0, 0, 0] == 0 and r[0, 0, 1] == K
    np.testing.assert_allclose(ov.overlap(s, u, M, K), 1.0)


def test_disjoint_rows_overlap_zero():
    M, K = 4, 2
    idx = np.arange(2 * M * K, dtype=np.int32).reshape(1, 1, 2 * M, K)
    s, u, r = ov.block_counts(idx, M)
    assert (u == M * K).all() and (r == 0).all()
    np.testing.assert_allclose(ov.overlap(s, u, M, K), 0.0)


def test_hand_counted_block_and_padding():
    # block 0: {1,2},{2,3},{3,-1}: 5 entries, union {1,2,3};
    # block 1: {3,4}: union {3,4}, reuse {3}
    idx = np.array([[[[1, 2], [2, 3], [3, -1], [3, 4]]]], dtype=np.int32)
    s, u, r = ov.block_counts(idx, 3)
    assert s.tolist() == [[[5, 2]]]
    assert u.tolist() == [[[3, 2]]]
    assert r.tolist() == [[[0, 1]]]
    # a full block of M=2 rows, K=2: (4 - 3) / 2
    s2, u2, _ = ov.block_counts(idx[:, :, :2], 2)
    np.testing.assert_allclose(ov.overlap(s2, u2, 2, 2), [[[0.5]]])
