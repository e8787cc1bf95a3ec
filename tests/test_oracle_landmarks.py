"""Pins of the landmark-builder oracle (Prop. 3.1) against what the
mathematics fixes, independently of its own formulas:

* exactness at the Taylor point: the surrogate q'.k'/sqrt(d) + b' equals
  the exact chunk log-mass at q = q' (computed by scipy's logsumexp);
* gradient: d/dq log-mass at q' equals k'/sqrt(d) (central finite
  differences of the exact log-mass);
* b' lies in [0, log S]; equal keys give b' = log S and k' = that key;
  one dominant key gives b' -> 0 and k' -> that key;
* permuting the keys inside a chunk changes nothing;
* the shared per-kv-head query equals the per-chunk query repeated.
"""
import numpy as np
import pytest
from scipy.special import logsumexp

from oracle import landmarks as lm


def _rand(shape, seed, scale=1.0):
    return scale * np.random.default_rng(seed).standard_normal(shape)


@pytest.mark.parametrize("S,d", [(64, 128), (16, 8), (128, 64)])
def test_surrogate_is_exact_at_the_landmark_query(S, d):
    K = _rand((1, 2, 5 * S, d), 1)
    Q = _rand((1, 2, 5, d), 2, scale=2.0)
    klm, bias = lm.build_landmarks(K, Q, S)
    for g in range(2):
        for c in range(5):
            q = Q[0, g, c]
            exact = logsumexp(K[0, g, c * S:(c + 1) * S] @ q / np.sqrt(d))
            sur = q @ klm[0, g, c] / np.sqrt(d) + bias[0, g, c]
            assert sur == pytest.approx(exact, abs=1e-10)


def test_gradient_of_log_mass_is_the_landmark_key():
    S, d = 32, 16
    K = _rand((1, 1, 3 * S, d), 3)
    Q = _rand((1, 1, 3, d), 4)
    klm, _ = lm.build_landmarks(K, Q, S)
    eps = 1e-5
    for c in range(3):
        q = Q[0, 0, c]
        grad = np.empty(d)
        for k in range(d):
            e = np.zeros(d)
            e[k] = eps
            grad[k] = (lm.chunk_logmass(K[0, 0], q + e, c, S)
                       - lm.chunk_logmass(K[0, 0], q - e, c, S)) / (2 * eps)
        np.testing.assert_allclose(grad, klm[0, 0, c] / np.sqrt(d), atol=1e-7)


def test_entropy_bounds_and_extremes():
    S, d = 64, 32
    K = _rand((2, 3, 4 * S, d), 5)
    Q = _rand((2, 3, 4, d), 6, scale=3.0)
    _, bias = lm.build_landmarks(K, Q, S)
    assert (bias >= -1e-12).all() and (bias <= np.log(S) + 1e-12).all()
    # equal keys: uniform distribution
    k0 = _rand(d, 7)
    Keq = np.broadcast_to(k0, (1, 1, S, d)).copy()
    klm, b = lm.build_landmarks(Keq, _rand((1, 1, 1, d), 8), S)
    assert b[0, 0, 0] == pytest.approx(np.log(S), abs=1e-12)
    np.testing.assert_allclose(klm[0, 0, 0], k0, atol=1e-12)
    # one dominant key
    Kd = _rand((1, 1, S, d), 9, scale=0.01)
    u = _rand(d, 10)
    u /= np.linalg.norm(u)
    Kd[0, 0, 17] = 60.0 * u
    klm, b = lm.build_landmarks(Kd, (60.0 * u)[None, None, None, :], S)
    assert b[0, 0, 0] < 1e-6
    np.testing.assert_allclose(klm[0, 0, 0], Kd[0, 0, 17], atol=1e-6)


def test_permutation_inside_a_chunk_changes_nothing():
    S, d = 32, 16
    K = _rand((1, 1, 2 * S, d), 11)
    Q = _rand((1, 1, 2, d), 12)
    perm = np.random.default_rng(13).permutation(S)
    K2 = K.copy()
    K2[0, 0, S:2 * S] = K[0, 0, S + perm]
    a = lm.build_landmarks(K, Q, S)
    b = lm.build_landmarks(K2, Q, S)
    for x, y in zip(a, b):
        np.testing.assert_allclose(x, y, atol=1e-12)


def test_shared_query_is_the_per_chunk_query_repeated():
    S, d = 16, 8
    K = _rand((2, 3, 5 * S + 7, d), 14)            # ragged tail: no summary
    qs = _rand((3, d), 15)
    rep = np.broadcast_to(qs[None, :, None, :], (2, 3, 5, d))
    a = lm.build_landmarks(K, qs, S)
    b = lm.build_landmarks(K, rep, S)
    assert a[0].shape == (2, 3, 5, d)
    for x, y in zip(a, b):
        np.testing.assert_allclose(x, y, atol=0)
