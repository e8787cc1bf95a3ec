"""Pins of the fp64 backward oracle (oracle/backward.py) that do not depend
on it: central finite differences of the independent whole-tensor forward
(oracle/brute.py) with the selection held fixed, and closed forms."""
import numpy as np
import pytest

from oracle import brute
from oracle.backward import hils_backward


def _inputs(seed, B=1, Hq=2, Hkv=1, N=72, d=8, S=8, qs=False):
    r = np.random.default_rng(seed)
    Q = r.standard_normal((B, Hq, N, d))
    K = r.standard_normal((B, Hkv, N, d))
    V = r.standard_normal((B, Hkv, N, d))
    nC = N // S
    Klm = K[:, :, :nC * S].reshape(B, Hkv, nC, S, d).mean(3) + \
        0.1 * r.standard_normal((B, Hkv, nC, d))
    bias = 0.5 * r.standard_normal((B, Hkv, nC))
    dO = r.standard_normal((B, Hq, N, d))
    Qs = Q + 0.5 * r.standard_normal(Q.shape) if qs else None
    hm = [h * Hkv // Hq for h in range(Hq)]
    return dict(Q=Q, K=K, V=V, Klm=Klm, bias=bias, dO=dO, Qs=Qs, hm=hm)


def _loss(x, S, W, Kt, idx0):
    O, idx, _ = brute.hils_forward(x["Q"], x["K"], x["V"], x["Klm"], x["bias"],
                                   x["hm"], S, W, Kt, Qs=x["Qs"])
    return float((O * x["dO"]).sum()), np.array_equal(idx, idx0)


@pytest.mark.parametrize("qs", [False, True])
def test_backward_matches_finite_differences(qs):
    """Every tensor's gradient, on sampled coordinates, equals the central
    difference of sum(O * dO) through the brute forward (selection fixed:
    coordinates whose perturbation changes it are skipped)."""
    S, W, Kt = 8, 16, 2
    x = _inputs(11 + qs, qs=qs)
    O0, idx0, _ = brute.hils_forward(x["Q"], x["K"], x["V"], x["Klm"],
                                     x["bias"], x["hm"], S, W, Kt, Qs=x["Qs"])
    g = hils_backward(x["Q"], x["K"], x["V"], x["Klm"], x["bias"], x["hm"],
                      S, W, idx0, x["dO"], Qs=x["Qs"])
    np.testing.assert_allclose(g["O"], O0, rtol=0, atol=1e-12)
    r = np.random.default_rng(5)
    eps = 1e-6
    names = [("Q", "dQ"), ("K", "dK"), ("V", "dV"), ("Klm", "dKlm"),
             ("bias", "dbias")] + ([("Qs", "dQs")] if qs else [])
    checked = total = 0
    for name, gname in names:
        flat = x[name].reshape(-1)
        for f in r.choice(flat.size, size=min(24, flat.size), replace=False):
            total += 1
            old = flat[f]
            flat[f] = old + eps
            lp, okp = _loss(x, S, W, Kt, idx0)
            flat[f] = old - eps
            lm, okm = _loss(x, S, W, Kt, idx0)
            flat[f] = old
            if not (okp and okm):
                continue
            fd = (lp - lm) / (2 * eps)
            an = g[gname].reshape(-1)[f]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, f, fd, an)
            checked += 1
    assert checked >= 0.9 * total


def test_backward_constant_values():
    """V constant over the tokens: O does not depend on Q, K, k', b', so
    their gradients vanish; dV_j = sum of p_ij dO_i."""
    S, W, Kt = 8, 16, 2
    x = _inputs(3)
    x["V"][:] = np.array([0.5, -1.0, 2.0, 0.0, 1.5, -0.25, 3.0, 1.0])
    _, idx0, _ = brute.hils_forward(x["Q"], x["K"], x["V"], x["Klm"],
                                    x["bias"], x["hm"], S, W, Kt)
    g = hils_backward(x["Q"], x["K"], x["V"], x["Klm"], x["bias"], x["hm"],
                      S, W, idx0, x["dO"])
    for n in ("dQ", "dK", "dKlm", "dbias"):
        assert np.abs(g[n]).max() < 1e-12, n


def test_backward_value_gradient_sums_to_upstream():
    """The weights of a row sum to one, so summed over the tokens of a kv
    head, dV equals the sum of dO over the rows of its query heads."""
    S, W, Kt = 8, 16, 3
    x = _inputs(4, Hq=4, Hkv=2, N=96)
    _, idx0, _ = brute.hils_forward(x["Q"], x["K"], x["V"], x["Klm"],
                                    x["bias"], x["hm"], S, W, Kt)
    g = hils_backward(x["Q"], x["K"], x["V"], x["Klm"], x["bias"], x["hm"],
                      S, W, idx0, x["dO"])
    for gg in range(2):
        heads = [h for h in range(4) if x["hm"][h] == gg]
        want = x["dO"][0, heads].sum(axis=(0, 1))
        np.testing.assert_allclose(g["dV"][0, gg].sum(0), want, atol=1e-11)


MUTANTS = [
    ("ds[seg] = de[seg] - pi * U", "ds[seg] = de[seg]"),          # lz_c term lost
    ("dbias[b, g, c] += U", "dbias[b, g, c] += 2 * U"),            # bias scale
    ("de = p * (u - D)", "de = p * u"),                            # softmax Jacobian
    ("dKlm[b, g, c] += U * qs * sc", "dKlm[b, g, c] += U * q * sc"),  # Q-Cal query
    ("np.add.at(dV[b, g], allj, p[:, None] * go[None, :])",
     "np.add.at(dV[b, g], allj[::-1], p[:, None] * go[None, :])"),  # token order
]


@pytest.mark.parametrize("old,new", MUTANTS)
def test_backward_pins_catch_planted_mistakes(old, new, tmp_path):
    """A plausible mistake planted in a copy of the oracle fails a pin."""
    import importlib.util
    import os
    src = open(os.path.join(os.path.dirname(os.path.dirname(__file__)),
                            "oracle", "backward.py")).read()
    assert src.count(old) == 1
    path = tmp_path / "backward_mutant.py"
    path.write_text(src.replace(old, new))
    spec = importlib.util.spec_from_file_location("backward_mutant", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    global hils_backward
    saved = hils_backward
    hils_backward = mod.hils_backward
    fails = 0
    try:
        for fn, args in [(test_backward_matches_finite_differences, (False,)),
                         (test_backward_matches_finite_differences, (True,)),
                         (test_backward_constant_values, ()),
                         (test_backward_value_gradient_sums_to_upstream, ())]:
            try:
                fn(*args)
            except AssertionError:
                fails += 1
    finally:
        hils_backward = saved
    assert fails >= 1
