"""Pins of the fp64 oracle against what the pages and mathematics fix.

All CPU-only. Each pin is chosen so that a plausible mistake in the oracle
(a dropped bias, a wrong window bound, a wrong scale, a missing per-head
normalisation, a reversed tie rule, a transposed operand) fails at least one
of them; tests/test_oracle_mutants.py plants such mistakes and checks that.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import brute
import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _num(x):
    if isinstance(x, (int, float)):
        return float(x)
    env = {"e": math.e, "exp": math.exp, "log": math.log, "inf": math.inf,
           "ln3": math.log(3.0), "ln2": math.log(2.0), "sqrt": math.sqrt}
    return float(eval(x, {"__builtins__": {}}, env))


def _inp(Q, K, V, Klm, bias, head_map, S, W, Ktop, Qs=None):
    B, Hq, N, d = Q.shape
    sh = synth.Shape("f32", B, Hq, K.shape[1], d, N, S, W, Ktop)
    return dict(Q=Q, Qs=Qs, K=K, V=V, Klm=Klm, bias=bias,
                head_map=list(head_map), shape=sh)


# --------------------------------------------------------------- golden pins
def test_golden_toy_window_chunks():
    fx = json.load(open(os.path.join(GOLD, "toy_window_chunks.json")))
    x = fx["inputs"]
    N, S, W, K = x["N"], x["S"], x["W"], x["K"]
    f = lambda a: torch.tensor([_num(v) for v in a], dtype=torch.float32)
    Q = f(x["q"]).view(1, 1, N, 1)
    Kt = f(x["k"]).view(1, 1, N, 1)
    V = f(x["v"]).view(1, 1, N, 1)
    Klm = f(x["klm"]).view(1, 1, -1, 1)
    bias = f(x["bias"]).view(1, 1, -1)
    inp = _inp(Q, Kt, V, Klm, bias, [0], S, W, K)
    r = oracle.prefill_full(inp)
    exp_O = np.array([_num(v) for v in fx["expected"]["O"]])
    exp_idx = np.array(fx["expected"]["idx"])
    exp_gap = np.array([_num(v) for v in fx["expected"]["gap"]])
    np.testing.assert_allclose(r["O"][0, 0, :, 0], exp_O, rtol=1e-6)
    np.testing.assert_array_equal(r["idx"][0, 0], exp_idx)
    np.testing.assert_allclose(r["gap"][0, 0], exp_gap, rtol=1e-6)
    # the independent brute force agrees with the hand derivation too
    Ob, Ib, Gb = brute.hils_forward(Q, Kt, V, Klm, bias, [0], S, W, K)
    np.testing.assert_allclose(Ob[0, 0, :, 0], exp_O, rtol=1e-6)
    np.testing.assert_array_equal(Ib[0, 0], exp_idx)


def test_golden_gqa_group_rule():
    fx = json.load(open(os.path.join(GOLD, "gqa_group_rule.json")))
    x = fx["inputs"]
    N, S, W, K = x["N"], x["S"], x["W"], x["K"]
    p0 = [_num(v) for v in x["p_head0"]]
    p1 = [_num(v) for v in x["p_head1"]]
    off = x["offset_head1"]
    Q = torch.zeros(1, 2, N, 2)
    Q[0, 0, :, :] = torch.tensor(x["q_head0"], dtype=torch.float32)
    Q[0, 1, :, :] = torch.tensor(x["q_head1"], dtype=torch.float32)
    Klm = torch.zeros(1, 1, N, 2)
    for c in range(3):
        Klm[0, 0, c, 0] = math.sqrt(2) * math.log(p0[c])
        Klm[0, 0, c, 1] = math.sqrt(2) * (math.log(p1[c]) + off)
    bias = torch.zeros(1, 1, N)
    Kt = torch.tensor(x["k"], dtype=torch.float32).view(1, 1, N, 2)
    V = torch.tensor(x["v"], dtype=torch.float32).view(1, 1, N, 2)
    inp = _inp(Q, Kt, V, Klm, bias, [0, 0], S, W, K)
    r = oracle.prefill_full(inp)
    np.testing.assert_array_equal(r["idx"][0, 0, 1:4],
                                  np.array(fx["expected"]["idx_rows_1_2_3"]))
    np.testing.assert_allclose(r["O"][0, 0, 3], _num(fx["expected"]["O_row3_head0"]),
                               rtol=1e-5)
    np.testing.assert_allclose(r["O"][0, 1, 3], _num(fx["expected"]["O_row3_head1"]),
                               rtol=1e-5)
    _, Ib, _ = brute.hils_forward(Q, Kt, V, Klm, bias, [0, 0], S, W, K)
    np.testing.assert_array_equal(Ib[0, 0, 1:4],
                                  np.array(fx["expected"]["idx_rows_1_2_3"]))


# ------------------------------------------------- window bounds, closed form
@pytest.mark.parametrize("S,W", [(64, 128), (64, 1), (4, 7), (128, 2048), (2, 3)])
def test_window_bounds_closed_form(S, W):
    N = 3 * W + 5 * S
    w0, nc = brute.bounds(N, S, W)
    for i in range(N):
        # l(i) = floor((i-W+1)/S) * S, Python's // floors for negatives too
        l = ((i - W + 1) // S) * S
        assert w0[i] == max(l, 0)
        assert nc[i] == max(l // S, 0)
        assert w0[i] % S == 0 and w0[i] <= i
        # the window always covers at least W tokens once l(i) > 0
        if l > 0:
            assert i - w0[i] + 1 >= W and i - w0[i] + 1 <= W + S - 1


# ------------------------------------------------------ brute force vs oracle
CASES = [
    # (B, Hq, Hkv, d, N, S, W, K, structure, head_map)
    (1, 1, 1, 16, 96, 8, 16, 3, "plain", None),
    (2, 4, 2, 8, 77, 8, 9, 4, "plain", [1, 0, 1, 0]),   # ragged tail, permuted map
    (1, 4, 1, 8, 64, 4, 5, 40, "plain", None),          # K > |C_i| everywhere
    (1, 2, 2, 8, 70, 8, 1, 2, "qcal", None),            # W = 1, scoring query
    (1, 3, 1, 12, 90, 6, 20, 5, "temperature", None),
]


@pytest.mark.parametrize("case", CASES)
def test_brute_matches_oracle(case):
    B, Hq, Hkv, d, N, S, W, K, st, hm = case
    sh = synth.Shape("f32", B, Hq, Hkv, d, N, S, W, K, st)
    inp = synth.make_prefill(sh, seed=7 + N, head_map=hm)
    r = oracle.prefill_full(inp)
    Ob, Ib, Gb = brute.hils_forward(inp["Q"], inp["K"], inp["V"], inp["Klm"],
                                    inp["bias"], inp["head_map"], S, W, K,
                                    Qs=inp["Qs"])
    np.testing.assert_array_equal(r["idx"], Ib)
    np.testing.assert_allclose(r["O"], Ob, rtol=1e-11, atol=1e-12)
    fin = np.isfinite(Gb)
    np.testing.assert_array_equal(np.isfinite(r["gap"]), fin)
    np.testing.assert_allclose(r["gap"][fin], Gb[fin], rtol=1e-9, atol=1e-12)


def test_config1_brute_vs_oracle():
    """Config 1 in full (fp32, N=1024, S=64, W=128, K=4)."""
    sh = synth.PREFILL_CONFIGS[1]
    inp = synth.make_prefill(sh, seed=synth.seed_for(1))
    r = oracle.prefill_full(inp)
    Ob, Ib, _ = brute.hils_forward(inp["Q"], inp["K"], inp["V"], inp["Klm"],
                                   inp["bias"], inp["head_map"], sh.S, sh.W,
                                   sh.K)
    np.testing.assert_array_equal(r["idx"], Ib)
    np.testing.assert_allclose(r["O"], Ob, rtol=1e-10, atol=1e-12)


# --------------------------------------------- exact-score identity (Sec. 3)
@pytest.mark.parametrize("hm", [[0, 0, 1, 1], [0, 1, 0, 1]])
def test_exact_scores_equal_naive_bsa(hm):
    """With s^_ic = log Z_ic the hierarchical weights collapse to a plain
    softmax over the selected tokens (naive BSA, Sec. 2.1)."""
    sh = synth.Shape("f32", 1, 4, 2, 8, 80, 8, 12, 3, "plain")
    inp = synth.make_prefill(sh, seed=11, head_map=hm)
    r = oracle.prefill_full(inp, score_mode=oracle.SCORE_EXACT)
    On, In = brute.naive_bsa(inp["Q"], inp["K"], inp["V"], hm, sh.S, sh.W,
                             sh.K)
    np.testing.assert_array_equal(r["idx"], In)
    np.testing.assert_allclose(r["O"], On, rtol=1e-11, atol=1e-12)


def test_exact_landmarks_equal_naive_bsa():
    """Structure 'exact': chunks of identical keys with (k', b') = (k̄, log S)
    make the landmark score the exact log-mass, so the surrogate path itself
    must reproduce naive BSA."""
    sh = synth.Shape("f32", 1, 2, 1, 8, 72, 8, 10, 2, "exact")
    inp = synth.make_prefill(sh, seed=5)
    r = oracle.prefill_full(inp)
    On, In = brute.naive_bsa(inp["Q"], inp["K"], inp["V"], inp["head_map"],
                             sh.S, sh.W, sh.K)
    gap_ok = ~(np.abs(r["gap"]) < 1e-5)
    assert np.array_equal(r["idx"][gap_ok], In[gap_ok])
    np.testing.assert_allclose(r["O"], On, rtol=1e-6, atol=1e-7)


def _causal_sdpa(Q, K, V, head_map):
    Q, K, V = (torch.as_tensor(np.asarray(x, dtype=np.float64))
               if not isinstance(x, torch.Tensor) else x.double()
               for x in (Q, K, V))
    Kx = K[:, list(head_map)]
    Vx = V[:, list(head_map)]
    return torch.nn.functional.scaled_dot_product_attention(
        Q, Kx, Vx, is_causal=True).numpy()


@pytest.mark.parametrize("mode", ["exact_scores", "exact_structure"])
def test_reduces_to_full_causal(mode):
    """K >= |C_i| with exact scores: every earlier token is attended with its
    exact softmax weight -> textbook causal attention (torch SDPA, fp64)."""
    st = "exact" if mode == "exact_structure" else "plain"
    sh = synth.Shape("f32", 2, 4, 2, 16, 100, 8, 12, 64, st)
    inp = synth.make_prefill(sh, seed=3)
    sm = oracle.SCORE_EXACT if mode == "exact_scores" else oracle.SCORE_LANDMARK
    r = oracle.prefill_full(inp, score_mode=sm)
    ref = _causal_sdpa(inp["Q"], inp["K"], inp["V"], inp["head_map"])
    tol = 1e-11 if mode == "exact_scores" else 1e-6
    np.testing.assert_allclose(r["O"], ref, rtol=tol, atol=tol)


def test_empty_candidate_rows_are_causal():
    """Rows with C_i empty (l(i) <= 0) are exact causal attention for any
    landmark inputs."""
    sh = synth.Shape("f32", 1, 2, 1, 16, 64, 8, 20, 2, "plain")
    inp = synth.make_prefill(sh, seed=9)
    r = oracle.prefill_full(inp)
    ref = _causal_sdpa(inp["Q"], inp["K"], inp["V"], inp["head_map"])
    w0, nc = brute.bounds(sh.N, sh.S, sh.W)
    rows = np.where(nc == 0)[0]
    assert len(rows) >= 20
    np.testing.assert_allclose(r["O"][:, :, rows], ref[:, :, rows], rtol=1e-12,
                               atol=1e-12)
    assert (r["idx"][:, :, rows] == -1).all()


# ---------------------------------------------------------------- invariants
def _small(seed=21, st="plain", K=3):
    sh = synth.Shape("f32", 1, 4, 2, 8, 96, 8, 10, K, st)
    return synth.make_prefill(sh, seed=seed)


def test_constant_values_give_constant_output():
    inp = _small()
    inp["V"] = torch.ones_like(inp["V"])
    r = oracle.prefill_full(inp)
    np.testing.assert_allclose(r["O"], 1.0, rtol=0, atol=1e-13)


def test_output_inside_value_hull_of_attended_tokens():
    inp = _small()
    sh = inp["shape"]
    r = oracle.prefill_full(inp)
    V = inp["V"].double().numpy()
    w0, nc = brute.bounds(sh.N, sh.S, sh.W)
    for g in range(sh.Hkv):
        for h in oracle.group_heads(inp["head_map"], g):
            for i in range(sh.N):
                toks = list(range(w0[i], i + 1))
                for c in r["idx"][0, g, i]:
                    if c >= 0:
                        toks += list(range(c * sh.S, c * sh.S + sh.S))
                vv = V[0, g, toks]
                o = r["O"][0, h, i]
                assert (o <= vv.max(0) + 1e-12).all()
                assert (o >= vv.min(0) - 1e-12).all()


def test_bias_shift_keeps_selection():
    inp = _small()
    r0 = oracle.prefill_full(inp)
    inp2 = dict(inp)
    inp2["bias"] = inp["bias"] + torch.tensor([3.0, -2.0]).view(1, 2, 1)
    r1 = oracle.prefill_full(inp2)
    np.testing.assert_array_equal(r0["idx"], r1["idx"])


def test_permuting_tokens_inside_selected_chunk_keeps_output():
    inp = _small()
    sh = inp["shape"]
    r0 = oracle.prefill_full(inp)
    i = sh.N - 1
    c = int(r0["idx"][0, 0, i, 0])
    assert c >= 0
    perm = torch.randperm(sh.S, generator=torch.Generator().manual_seed(1))
    K2, V2 = inp["K"].clone(), inp["V"].clone()
    sl = slice(c * sh.S, (c + 1) * sh.S)
    K2[0, 0, sl] = inp["K"][0, 0, sl][perm]
    V2[0, 0, sl] = inp["V"][0, 0, sl][perm]
    inp2 = dict(inp, K=K2, V=V2)
    r1 = oracle.prefill_rows(inp2, [[0, 0, i]])
    r0r = oracle.prefill_rows(inp, [[0, 0, i]])
    np.testing.assert_array_equal(r0r["idx"], r1["idx"])
    np.testing.assert_allclose(r1["O"], r0r["O"], rtol=1e-12, atol=1e-13)


def test_planted_bias_forces_selection():
    inp = _small(K=3)
    sh = inp["shape"]
    planted = [1, 4, 6]
    b = inp["bias"].clone()
    b[0, :, planted] = 1e4
    inp2 = dict(inp, bias=b)
    r = oracle.prefill_full(inp2)
    w0, nc = brute.bounds(sh.N, sh.S, sh.W)
    rows = np.where(nc > max(planted))[0]
    assert len(rows) > 0
    for g in range(sh.Hkv):
        assert (r["idx"][0, g, rows] == np.array(planted)).all()


def test_tie_rule_lower_index():
    """Identical (k', b') for chunks 2 and 5 (and 3, 4 pushed down): with
    K = 1 and those two clearly best, the lower index wins."""
    inp = _small(K=1)
    sh = inp["shape"]
    Klm = inp["Klm"].clone()
    b = inp["bias"].clone()
    Klm[0, :, 5] = Klm[0, :, 2]
    b[0, :, 2] = 50.0
    b[0, :, 5] = 50.0
    r = oracle.prefill_full(dict(inp, Klm=Klm, bias=b))
    w0, nc = brute.bounds(sh.N, sh.S, sh.W)
    rows = np.where(nc > 5)[0]
    assert len(rows) > 0
    assert (r["idx"][0, :, rows, 0] == 2).all()
    assert (r["gap"][0, :, rows] == 0.0).all()


def test_imposed_selection_reproduces_own_selection():
    inp = _small()
    sh = inp["shape"]
    rows = np.array([[0, g, i] for g in range(sh.Hkv) for i in range(sh.N)])
    r0 = oracle.prefill_rows(inp, rows)
    r1 = oracle.prefill_rows(inp, rows, imposed_idx=r0["idx"])
    np.testing.assert_array_equal(r0["O"], r1["O"])


# -------------------------------------------------------------------- decode
def test_decode_matches_prefill_row():
    """A decode step is the prefill computation at i = cache_len-1."""
    sh = synth.Shape("f32", 3, 4, 2, 16, 256, 8, 24, 5)
    dec = synth.make_decode(sh, seed=17, cache_len=[256, 131, 40])
    r = oracle.decode(dec)
    for b, L in enumerate([256, 131, 40]):
        Qp = torch.zeros(1, sh.Hq, L, sh.d)
        Qp[0, :, L - 1] = dec["Q"][b]
        pre = dict(Q=Qp, Qs=None, K=dec["K"][b:b + 1, :, :L].contiguous(),
                   V=dec["V"][b:b + 1, :, :L].contiguous(),
                   Klm=dec["Klm"][b:b + 1, :, :L // sh.S].contiguous(),
                   bias=dec["bias"][b:b + 1, :, :L // sh.S].contiguous(),
                   head_map=dec["head_map"], shape=sh.with_(B=1, N=L))
        Ob, Ib, _ = brute.hils_forward(pre["Q"], pre["K"], pre["V"],
                                       pre["Klm"], pre["bias"],
                                       pre["head_map"], sh.S, sh.W, sh.K)
        np.testing.assert_array_equal(r["idx"][b], Ib[0, :, L - 1])
        np.testing.assert_allclose(r["O"][b], Ob[0, :, L - 1], rtol=1e-11,
                                   atol=1e-12)


def test_oracle_bf16_storage_widens_exactly():
    """bf16 inputs are widened bit-exactly: same result as the f32 copy."""
    sh = synth.Shape("bf16", 1, 2, 1, 8, 64, 8, 9, 2)
    inp = synth.make_prefill(sh, seed=2)
    r16 = oracle.prefill_full(inp)
    inp32 = dict(inp, **{k: inp[k].float() for k in ("Q", "K", "V", "Klm")},
                 shape=sh.with_(dtype="f32"))
    r32 = oracle.prefill_full(inp32)
    np.testing.assert_array_equal(r16["idx"], r32["idx"])
    np.testing.assert_array_equal(r16["O"], r32["O"])


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_group_topk_lies_in_union_of_per_split_per_head_topk(seed):
    """The group top-K (a_c = max_h (s^_hc - LSE_h), ties to the lower
    chunk) is contained in the union, over contiguous splits of the
    candidates and over heads, of each split's per-head top-K by s^ (same
    tie rule): a chunk outside its split's top-K for its maximising head has
    K chunks of that split ranked above it for every head's offset. This
    bounds what a split-local pre-selection may discard. Exact ties are
    planted so the tie rule is exercised."""
    r = np.random.default_rng(seed)
    G, nc, K = 4, 300, 16
    shat = np.round(r.standard_normal((G, nc)) * 4) / 4      # many exact ties
    idx, _ = brute.select(shat[:, None, :], np.array([nc]), K)
    chosen = set(int(c) for c in idx[0] if c >= 0)
    for nsplit in (1, 3, 7, 19):
        bounds_ = np.linspace(0, nc, nsplit + 1).astype(int)
        union = set()
        for a, b in zip(bounds_[:-1], bounds_[1:]):
            for h in range(G):
                c = np.arange(a, b)
                order = np.lexsort((c, -shat[h, a:b]))
                union.update(int(x) for x in c[order[:K]])
        assert chosen <= union, (nsplit, sorted(chosen - union))
