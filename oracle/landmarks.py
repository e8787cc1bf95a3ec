"""fp64 oracle of the landmark summary builder (Prop. 3.1).

TEST INFRASTRUCTURE ONLY: used by the tests, the smoke check and the
benchmark's CPU leg, never by the product path; shares no code with the
CUDA library.

"Hierarchical Sparse Attention Done Right", Sec. 3 (answering RQ1, the
surrogate of Eq. 7): a landmark query q'_c induces an attention
distribution over the S keys of chunk c,

    p_j = softmax_j(q'_c . k_j / sqrt(d)),  j in T_c = {cS, ..., cS+S-1},

and the chunk summary is computed as Attn(q'_c, K_c, K_c):

    k'_c = sum_j p_j k_j          (the weighted sum of the chunk's keys)
    b'_c = -sum_j p_j log p_j     (the entropy of that distribution).

Readings (where the pages leave a step open):
  * one landmark query per (batch, kv head, chunk), shape [B,Hkv,nC,d], the
    shape the surrogate score takes its k' in; the pages' "shared learnable
    query per layer" variant (Sec. 4.1, landmark-token-free alternative) is
    the same computation with one query per kv head, [Hkv,d], broadcast
    over batch and chunks;
  * only full chunks (nC = floor(N/S)) get a summary; a trailing partial
    chunk can only lie in a query's window;
  * the entropy is evaluated as LSE - sum_j p_j s_j (equal to -sum p log p
    for p = softmax(s)), which stays finite when some p_j underflow.
"""
from __future__ import annotations

import numpy as np


def build_landmarks(K, Qlm, S):
    """K [B,Hkv,N,d]; Qlm [B,Hkv,nC,d] or [Hkv,d] (shared per kv head).

    Returns (k' [B,Hkv,nC,d], b' [B,Hkv,nC]) in float64.
    """
    K = np.asarray(K, dtype=np.float64)
    B, Hkv, N, d = K.shape
    nC = N // S
    Q = np.asarray(Qlm, dtype=np.float64)
    if Q.ndim == 2:                                   # shared query per kv head
        Q = np.broadcast_to(Q[None, :, None, :], (B, Hkv, nC, d))
    Kc = K[:, :, :nC * S, :].reshape(B, Hkv, nC, S, d)
    s = np.einsum("bhcd,bhcjd->bhcj", Q, Kc) / np.sqrt(d)   # [B,Hkv,nC,S]
    m = s.max(axis=-1, keepdims=True)
    e = np.exp(s - m)
    z = e.sum(axis=-1, keepdims=True)
    p = e / z
    lse = (m + np.log(z))[..., 0]
    klm = np.einsum("bhcj,bhcjd->bhcd", p, Kc)
    bias = lse - (p * s).sum(axis=-1)
    return klm, bias


def chunk_logmass(K, q, c, S):
    """log sum_{j in T_c} exp(q . k_j / sqrt(d)) for one query vector q and
    one chunk c of one [N,d] key matrix (the exact quantity the surrogate of
    Eq. 7 approximates)."""
    K = np.asarray(K, dtype=np.float64)
    d = K.shape[-1]
    s = K[c * S:(c + 1) * S] @ np.asarray(q, dtype=np.float64) / np.sqrt(d)
    m = s.max()
    return float(m + np.log(np.exp(s - m).sum()))
