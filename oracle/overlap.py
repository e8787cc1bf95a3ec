"""Oracle of the chunk-overlap diagnostics over a selection.

TEST INFRASTRUCTURE ONLY (tests, smoke check, benchmark CPU leg); shares no
code with the CUDA library.

"Hierarchical Sparse Attention Done Right", Sec. 7.2: for a block of M
adjacent queries with selected chunk sets I_1..I_M,

    Overlap = (M K - |I_1 u ... u I_M|) / ((M - 1) K),

and the share of a block's chunks that the previous block already loaded.
Per block (b, kv head, block of M consecutive query rows; the last block may
be shorter) this returns the raw counts the metrics are formed from:
  n_sel    sum over the block's rows of |I_m| (entries >= 0 of idx),
  n_union  |union of the block's I_m|,
  n_reuse  |that union intersected with the previous block's union| (0 for
           the first block).
Reading: rows with fewer than K candidates contribute their actual |I_m|;
Overlap is then (n_sel - n_union) / (n_sel - n_sel / M) for full blocks,
which is the printed formula when every row holds K chunks.
"""
from __future__ import annotations

import numpy as np


def block_counts(idx, M):
    """idx [B,Hkv,N,K] int (-1 padded). Returns n_sel, n_union, n_reuse,
    each [B,Hkv,ceil(N/M)] int64."""
    idx = np.asarray(idx)
    B, H, N, K = idx.shape
    nb = (N + M - 1) // M
    n_sel = np.zeros((B, H, nb), dtype=np.int64)
    n_union = np.zeros_like(n_sel)
    n_reuse = np.zeros_like(n_sel)
    for b in range(B):
        for h in range(H):
            prev = set()
            for k in range(nb):
                rows = idx[b, h, k * M:(k + 1) * M]
                vals = rows[rows >= 0]
                cur = set(int(v) for v in vals)
                n_sel[b, h, k] = vals.size
                n_union[b, h, k] = len(cur)
                n_reuse[b, h, k] = len(cur & prev)
                prev = cur
    return n_sel, n_union, n_reuse


def overlap(n_sel, n_union, M, K):
    """The printed metric per full block whose rows all hold K chunks
    (NaN elsewhere)."""
    n_sel = np.asarray(n_sel, dtype=np.float64)
    n_union = np.asarray(n_union, dtype=np.float64)
    full = n_sel == M * K
    out = np.full(n_sel.shape, np.nan)
    out[full] = (M * K - n_union[full]) / ((M - 1) * K)
    return out
