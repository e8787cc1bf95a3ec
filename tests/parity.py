"""Comparison of the CUDA path's outputs with the oracle, under the
acceptance rule for HiLS forward outputs:

* idx bit-exact, except at a (row, kv group) whose oracle gap between the
  K-th and (K+1)-th group score is below 1e-3 * max(1, |a_(K)|); there the
  GPU's own selection is imposed on the oracle and O is checked against that;
* float32 O: max|O - O_ref| / max|O_ref| <= 1e-5 over the compared tensor;
* bf16 O: max|O - O_ref| <= 2e-2 against fp64.
"""
import numpy as np
import torch

import oracle

F32_REL = 1e-5
BF16_ABS = 2e-2


def near_tie(gap, akth):
    return np.abs(gap) < 1e-3 * np.maximum(1.0, np.abs(akth))


def sample_positions(sh, n_random=48, seed=0):
    """Edge rows of the window / candidate structure plus random rows."""
    N, S, W, K = sh.N, sh.S, sh.W, sh.K
    first_cand = W + S - 1                  # first i with |C_i| = 1
    edges = [0, 1, S - 1, S, W - 1, W, first_cand - 1, first_cand,
             first_cand + 1, W - 1 + K * S, W + K * S, W - 1 + (K + 1) * S,
             N // 2, N - S - 1, N - S, N - 2, N - 1]
    rng = np.random.default_rng(seed)
    rnd = rng.integers(0, N, size=n_random)
    pos = sorted({int(p) for p in list(edges) + list(rnd) if 0 <= p < N})
    return np.asarray(pos, dtype=np.int64)


def sample_positions_dense(sh, n_total=2048, block=128, seed=0):
    """A few thousand query positions of a long prefill: whole blocks of
    `block` adjacent queries (the CTA tiles of both kernels are 128 queries
    for scoring and 128/G queries for attention) at the start, where the
    first candidate appears, where |C_i| first reaches K, in the middle and
    at the end; the edge rows of `sample_positions`; and random rows
    stratified over the chunk phase i mod S (every phase the same number of
    times) and over the whole length, so every candidate-count regime is
    represented."""
    N, S, W, K = sh.N, sh.S, sh.W, sh.K
    starts = [0, W + S - 1, W - 1 + K * S, N // 2, N - block]
    pos = set()
    for s in starts:
        s0 = max(0, min(N - block, (s // block) * block))
        pos.update(range(s0, min(N, s0 + block)))
    pos.update(int(p) for p in sample_positions(sh, n_random=0))
    rng = np.random.default_rng(seed)
    while len(pos) < min(n_total, N):
        phase = rng.permutation(S)
        chunk = rng.integers(0, max(1, (N - 1) // S + 1), size=S)
        for p, c in zip(phase, chunk):
            i = int(c) * S + int(p)
            if i < N:
                pos.add(i)
    return np.asarray(sorted(pos), dtype=np.int64)


def _gpu_group_view(sh, head_map, O_gpu, positions, groups):
    """O_gpu [B,Hq,N,d] -> [B,nG,P,G,d] float64 host, heads in group order."""
    pt = torch.as_tensor(positions, device=O_gpu.device)
    sub = O_gpu.index_select(2, pt).double().cpu().numpy()
    out = np.zeros((sh.B, len(groups), len(positions), sh.G, sh.d))
    for gi, g in enumerate(groups):
        for hh, h in enumerate(oracle.group_heads(head_map, g)):
            out[:, gi, :, hh] = sub[:, h]
    return out


def check_prefill(inp, O_gpu, idx_gpu, positions=None, sel_gpu=None,
                  threads=0, groups=None):
    """Compare O, idx (and s^ of the selected chunks) at `positions` of the
    kv groups `groups` (default: all) with the oracle."""
    sh = inp["shape"]
    if positions is None:
        positions = np.arange(sh.N)
    groups = list(range(sh.Hkv)) if groups is None else list(groups)
    bound = oracle.bind_at(inp, positions)
    ref = oracle.prefill_at(inp, positions, threads=threads, groups=groups,
                            bound=bound)
    pt = torch.as_tensor(positions, device=idx_gpu.device)
    gt = torch.as_tensor(groups, device=idx_gpu.device)
    gi = idx_gpu.index_select(1, gt).index_select(2, pt).cpu().numpy()
    tie = near_tie(ref["gap"], ref["akth"])
    bad = (gi != ref["idx"]).any(-1)
    assert not (bad & ~tie).any(), (
        "idx mismatch outside near-ties at (b,g,p): "
        f"{np.argwhere(bad & ~tie)[:8].tolist()}")
    O_ref = ref["O"]
    if (bad & tie).any():                       # re-evaluate with GPU's pick
        r2 = oracle.prefill_at(inp, positions, imposed_idx=gi,
                               threads=threads, groups=groups, bound=bound)
        O_ref = np.where((bad & tie)[..., None, None], r2["O"], O_ref)
    Og = _gpu_group_view(sh, inp["head_map"], O_gpu, positions, groups)
    err = np.abs(Og - O_ref)
    if sh.dtype == "f32":
        rel = err.max() / max(1e-30, np.abs(O_ref).max())
        assert rel <= F32_REL, f"f32 O rel err {rel:.3e}"
    else:
        assert err.max() <= BF16_ABS, f"bf16 O max-abs err {err.max():.3e}"
    if sel_gpu is not None:
        sg = sel_gpu.index_select(2, pt).double().cpu().numpy()
        for gi_, g in enumerate(groups):
            for hh, h in enumerate(oracle.group_heads(inp["head_map"], g)):
                ok = ~bad[:, gi_]
                a = sg[:, h][ok]
                b = ref["shat_sel"][:, gi_, :, hh][ok]
                fin = np.isfinite(b)
                assert np.array_equal(np.isfinite(a), fin)
                assert np.abs(a[fin] - b[fin]).max(initial=0) < 1e-3
    return dict(ties=int(tie.sum()), tie_mismatch=int((bad & tie).sum()),
                max_err=float(err.max()), rows=int(np.prod(tie.shape)))


def check_decode(inp, O_gpu, idx_gpu, threads=0):
    sh = inp["shape"]
    ref = oracle.decode(inp, threads=threads)
    gi = idx_gpu.cpu().numpy()
    tie = near_tie(ref["gap"], ref["akth"])
    bad = (gi != ref["idx"]).any(-1)
    assert not (bad & ~tie).any(), (
        f"decode idx mismatch at (b,g): {np.argwhere(bad & ~tie)[:8].tolist()}")
    O_ref = ref["O"]
    if (bad & tie).any():
        r2 = oracle.decode(inp, imposed_idx=gi, threads=threads)
        rows = np.zeros((sh.B, sh.Hq), dtype=bool)
        for b, g in np.argwhere(bad & tie):
            for h in oracle.group_heads(inp["head_map"], g):
                rows[b, h] = True
        O_ref = np.where(rows[..., None], r2["O"], O_ref)
    Og = O_gpu.double().cpu().numpy()
    err = np.abs(Og - O_ref)
    if sh.dtype == "f32":
        rel = err.max() / max(1e-30, np.abs(O_ref).max())
        assert rel <= F32_REL, f"f32 decode O rel err {rel:.3e}"
    else:
        assert err.max() <= BF16_ABS, f"bf16 decode O max-abs {err.max():.3e}"
    return dict(ties=int(tie.sum()), max_err=float(err.max()))
