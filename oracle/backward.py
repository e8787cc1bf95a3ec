"""fp64 oracle of the HiLS attention backward (gradients of the prefill
output), for a fixed selection.

TEST INFRASTRUCTURE ONLY: imported by the tests and the benchmark's
CPU-baseline leg, never by the product path. No code is shared with the
CUDA library.

"Hierarchical Sparse Attention Done Right", Sec. 3 (RQ2: the chunk-level
softmax fused with the intra-chunk softmax, so the language-model loss
reaches the landmark scores) and Sec. 4 (native sparse training of the
landmarks). The selection (top-K) is a discrete choice: it is held fixed,
and gradients flow through every continuous quantity of the fused output.

Forward for one row i and head h of kv group g (0-based positions; chunk c
holds tokens cS .. cS+S-1; the window is [w0, i]):
    s_j   = q . k_j / sqrt(d)
    sh_c  = qs . k'_c / sqrt(d) + b'_c              (qs = Q-Cal query, or q)
    lz_c  = log sum_{j in chunk c} exp(s_j)
    e_j   = s_j - lz_c + sh_c   (tokens of selected chunks)
    e_j   = s_j                 (window tokens)
    p     = softmax(e) over all attended tokens;  o = sum_j p_j v_j

Backward, with u_j = dO . v_j and D = dO . o = sum_j p_j u_j:
    dV_j   += p_j dO
    de_j    = p_j (u_j - D)
    chunk c: U_c = sum_{j in c} de_j = P_c (Ubar_c - D), where
             P_c = sum_{j in c} p_j = exp(sh_c - L) and
             Ubar_c = sum_{j in c} pi_j u_j, pi_j = exp(s_j - lz_c);
             the lz_c term gives ds_j = de_j - pi_j U_c = p_j (u_j - Ubar_c);
             dsh_c = U_c
    window:  ds_j = de_j
    dq     += sum_j ds_j k_j / sqrt(d);   dK_j += ds_j q / sqrt(d)
    dqs    += sum_c dsh_c k'_c / sqrt(d); dK'_c += dsh_c qs / sqrt(d);
    db'_c  += dsh_c
Without a separate scoring query, dqs is added into dQ.
"""
from __future__ import annotations

import numpy as np


def _f64(x):
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu", torch.float64).numpy()
    except ImportError:                               # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


def bounds(i, S, W):
    """Window start w0 = max(l, 0) and candidate count nc = max(l/S, 0),
    l = floor((i - W + 1) / S) * S (Sec. 2.1)."""
    lq = (i - W + 1) // S
    return max(lq * S, 0), max(lq, 0)


def _lse(x):
    m = np.max(x)
    return m + np.log(np.sum(np.exp(x - m)))


def hils_backward(Q, K, V, Klm, bias, head_map, S, W, idx, dO, Qs=None):
    """Gradients of sum(O * dO) for O = HiLS prefill forward with the
    selection `idx` [B,Hkv,N,Ktop] (ascending, -1 padded; entries outside
    C_i are ignored, as the forward ignores them).

    Q/Qs/dO [B,Hq,N,d], K/V [B,Hkv,N,d], Klm [B,Hkv,nC,d], bias [B,Hkv,nC].
    Returns dict dQ, dQs (None when Qs is None: folded into dQ), dK, dV,
    dKlm, dbias (float64) and O (the forward output, float64).
    """
    Q, K, V, Klm, bias, dO = map(_f64, (Q, K, V, Klm, bias, dO))
    sep = Qs is not None
    Qs = _f64(Qs) if sep else Q
    if hasattr(idx, "cpu"):
        idx = idx.cpu().numpy()
    idx = np.asarray(idx, dtype=np.int64)
    B, Hq, N, d = Q.shape
    nC = Klm.shape[2]
    sc = 1.0 / np.sqrt(d)
    dQ, dQs = np.zeros_like(Q), np.zeros_like(Qs)
    dK, dV = np.zeros_like(K), np.zeros_like(V)
    dKlm, dbias = np.zeros_like(Klm), np.zeros_like(bias)
    O = np.zeros_like(Q)
    for b in range(B):
        for h in range(Hq):
            g = head_map[h]
            for i in range(N):
                w0, nc = bounds(i, S, W)
                sel = [int(c) for c in idx[b, g, i] if 0 <= c < nc]
                q, qs, go = Q[b, h, i], Qs[b, h, i], dO[b, h, i]
                # attended tokens: the selected chunks, then the window
                toks = [np.arange(c * S, c * S + S) for c in sel]
                win = np.arange(w0, i + 1)
                allj = np.concatenate(toks + [win]).astype(np.int64)
                s = K[b, g, allj] @ q * sc
                sh = np.array([qs @ Klm[b, g, c] * sc + bias[b, g, c]
                               for c in sel])
                e = s.copy()
                lz = np.zeros(len(sel))
                for n, c in enumerate(sel):
                    seg = slice(n * S, n * S + S)
                    lz[n] = _lse(s[seg])
                    e[seg] = s[seg] - lz[n] + sh[n]
                p = np.exp(e - _lse(e))
                o = p @ V[b, g, allj]
                O[b, h, i] = o
                u = V[b, g, allj] @ go
                D = go @ o
                np.add.at(dV[b, g], allj, p[:, None] * go[None, :])
                de = p * (u - D)
                ds = de.copy()
                for n, c in enumerate(sel):
                    seg = slice(n * S, n * S + S)
                    pi = np.exp(s[seg] - lz[n])
                    U = de[seg].sum()
                    ds[seg] = de[seg] - pi * U
                    dQs[b, h, i] += U * Klm[b, g, c] * sc
                    dKlm[b, g, c] += U * qs * sc
                    dbias[b, g, c] += U
                dQ[b, h, i] += ds @ K[b, g, allj] * sc
                np.add.at(dK[b, g], allj, ds[:, None] * q[None, :] * sc)
    if not sep:
        dQ = dQ + dQs
        dQs = None
    return dict(dQ=dQ, dQs=dQs, dK=dK, dV=dV, dKlm=dKlm, dbias=dbias, O=O)
