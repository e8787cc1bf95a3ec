"""Whole-tensor numpy brute force of HiLS attention, for tiny problems.

TEST INFRASTRUCTURE ONLY (see the package docstring). Written separately from
``hils_oracle.c``: it builds the dense token-logit matrix and boolean masks
for a whole head at once and evaluates the hierarchical-softmax weights in
the ratio form of "Hierarchical Sparse Attention Done Right", Sec. 3
("Answering RQ2: Hierarchical softmax" display),

    w_ij = exp(s_ij) / Z_{i,c(j)} * Z^_{i,c(j)} / Z^_i,
    Z^_{i,c} = exp(s^_ic) for selected chunks, Z_swa for the window,

directly with exponentials (no log-domain shift), so keep |logits| small
(below ~300) when using it. Chunk selection follows Sec. 3 (surrogate score
and rank) and Sec. 4.1 "HiLS-Attention in GQA" (max over heads of the
per-head normalised chunk weights), with the readings listed in the C
oracle's header.
"""
from __future__ import annotations

import numpy as np


def _f64(x):
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().cpu().double().numpy()
    except ImportError:                                   # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


def bounds(N, S, W):
    """Per query position: aligned window start and candidate-chunk count.
    (Sec. 2.1: l(i) = floor((i-W+1)/S) S, C_i = {0..l(i)/S-1}.)"""
    i = np.arange(N)
    lq = np.floor_divide(i - W + 1, S)
    w0 = np.maximum(lq * S, 0)
    nc = np.maximum(lq, 0)
    return w0, nc


def _masked_lse(x, mask):
    """log sum exp over the last axis restricted to mask; -inf if empty."""
    xm = np.where(mask, x, -np.inf)
    m = xm.max(axis=-1, keepdims=True)
    m_safe = np.where(np.isfinite(m), m, 0.0)
    s = np.where(mask, np.exp(xm - m_safe), 0.0).sum(axis=-1)
    with np.errstate(divide="ignore"):
        return np.where(s > 0, np.log(s) + m_safe[..., 0], -np.inf)


def select(shat_heads, nc, K):
    """Group top-K. shat_heads: [G, N, nC] chunk scores of the group's heads.
    Returns idx [N, K] (ascending, -1 padded) and gap [N]."""
    G, N, nC = shat_heads.shape
    cand = np.arange(nC)[None, :] < nc[:, None]                  # [N,nC]
    lse = _masked_lse(shat_heads, cand[None])                    # [G,N]
    a = np.where(cand[None], shat_heads - lse[..., None], -np.inf).max(0)
    idx = np.full((N, K), -1, dtype=np.int64)
    gap = np.full(N, np.inf)
    for i in range(N):
        n = int(nc[i])
        if n == 0:
            continue
        c = np.arange(n)
        order = np.lexsort((c, -a[i, :n]))       # key: -a, then chunk index
        take = order[:K]
        idx[i, :len(take)] = np.sort(take)
        if n > K:
            gap[i] = a[i, order[K - 1]] - a[i, order[K]]
    return idx, gap


def hils_forward(Q, K, V, Klm, bias, head_map, S, W, Ktop, Qs=None,
                 exact_scores=False):
    """HiLS forward for a whole (tiny) problem.

    Q/Qs [B,Hq,N,d], K/V [B,Hkv,N,d], Klm [B,Hkv,nC,d], bias [B,Hkv,nC].
    exact_scores=True replaces s^_ic by the exact log Z_ic (identity check).
    Returns O [B,Hq,N,d], idx [B,Hkv,N,K], gap [B,Hkv,N].
    """
    Q, K, V, Klm, bias = map(_f64, (Q, K, V, Klm, bias))
    Qs = Q if Qs is None else _f64(Qs)
    B, Hq, N, d = Q.shape
    Hkv, nC = K.shape[1], Klm.shape[2]
    w0, nc = bounds(N, S, W)
    pos = np.arange(N)
    chunk_of = pos // S
    O = np.zeros((B, Hq, N, d))
    IDX = np.zeros((B, Hkv, N, Ktop), dtype=np.int64)
    GAP = np.zeros((B, Hkv, N))
    for b in range(B):
        for g in range(Hkv):
            heads = [h for h in range(Hq) if head_map[h] == g]
            s_all, shat_all = [], []
            for h in heads:
                s = Q[b, h] @ K[b, g].T / np.sqrt(d)                # [N,N]
                if exact_scores:
                    sc = s[:, :nC * S].reshape(N, nC, S)
                    shat = np.log(np.exp(sc).sum(-1))
                else:
                    shat = Qs[b, h] @ Klm[b, g].T / np.sqrt(d) + bias[b, g]
                s_all.append(s)
                shat_all.append(shat)
            idx, gap = select(np.stack(shat_all), nc, Ktop)
            IDX[b, g], GAP[b, g] = idx, gap
            for hh, h in enumerate(heads):
                s, shat = s_all[hh], shat_all[hh]
                es = np.exp(s)
                for i in range(N):
                    win = (pos >= w0[i]) & (pos <= i)
                    z_swa = es[i, win].sum()
                    sel = idx[i][idx[i] >= 0]
                    zhat_sel = np.exp(shat[i, sel])
                    zhat_tot = zhat_sel.sum() + z_swa
                    w = np.zeros(N)
                    w[win] = es[i, win] / z_swa * z_swa / zhat_tot
                    for c, zh in zip(sel, zhat_sel):
                        tok = chunk_of == c
                        zc = es[i, tok].sum()
                        w[tok] = es[i, tok] / zc * zh / zhat_tot
                    O[b, h, i] = w @ V[b, g]
    return O, IDX, GAP


def naive_bsa(Q, K, V, head_map, S, W, Ktop):
    """Naive block-sparse attention (Sec. 2.1): select by the exact chunk
    masses Z_ic (group rule of Sec. 4.1), then an ordinary softmax over the
    selected chunks' tokens and the window, every other token weight 0."""
    Q, K, V = map(_f64, (Q, K, V))
    B, Hq, N, d = Q.shape
    Hkv = K.shape[1]
    nC = N // S
    w0, nc = bounds(N, S, W)
    pos = np.arange(N)
    O = np.zeros((B, Hq, N, d))
    IDX = np.zeros((B, Hkv, N, Ktop), dtype=np.int64)
    for b in range(B):
        for g in range(Hkv):
            heads = [h for h in range(Hq) if head_map[h] == g]
            S_h = [Q[b, h] @ K[b, g].T / np.sqrt(d) for h in heads]
            logZ = np.stack([np.log(np.exp(s[:, :nC * S].reshape(N, nC, S))
                                    .sum(-1)) for s in S_h])
            idx, _ = select(logZ, nc, Ktop)
            IDX[b, g] = idx
            for hh, h in enumerate(heads):
                for i in range(N):
                    keep = (pos >= w0[i]) & (pos <= i)
                    for c in idx[i][idx[i] >= 0]:
                        keep |= (pos // S) == c
                    x = np.where(keep, S_h[hh][i], -np.inf)
                    p = np.exp(x - x.max())
                    O[b, h, i] = (p / p.sum()) @ V[b, g]
    return O, IDX
