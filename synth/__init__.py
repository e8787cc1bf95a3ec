"""Seeded synthetic inputs for HiLS attention (prefill and decode).

This module only draws numbers: it holds none of the attention method's
arithmetic and is shared, unchanged, by the CUDA path's tests/bench and by
the oracle's tests. Every tensor is produced from a torch generator seeded
with an explicit integer, on the device the caller asks for.

Workload recipes (the pages measure on RULER / LongBench / PPL corpora that
are not available here; the "planted needle" and "per-chunk temperature"
structures below stand in for the attention patterns of those suites):

* plain        Q, K, V ~ N(0, 1); landmark key k'_c = mean of chunk c's keys
               + N(0, 0.1^2); chunk bias b'_c ~ N(0, 0.5^2).
* needles      as plain, plus per kv head a unit direction u and needle
               chunks; one token of each needle chunk gets k = 8u + N(0,0.1^2)
               and every query after the first needle gets q += 4u (peaked
               logits). ``needle_every`` tokens per needle region, or
               ``n_needles`` chunks drawn uniformly.
* temperature  as plain, but every chunk's keys are scaled by a temperature
               drawn uniformly from {0.1, 1, 4} before k' is formed, mixing
               near-uniform and single-token-dominant chunks.
* exact        every complete chunk holds S copies of one key k̄_c, and the
               landmark is (k'_c, b'_c) = (k̄_c, log S): then the surrogate
               score equals the exact chunk log-mass for every query.
* qcal         as plain, plus a separate scoring query Q̂ = Q + 0.5 N(0,1)
               (stands in for the low-rank query calibration output).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import torch

__all__ = [
    "Shape", "PREFILL_CONFIGS", "DECODE_CONFIGS", "CONFIG_TEXT",
    "make_prefill", "make_decode", "default_head_map", "seed_for",
]


@dataclass(frozen=True)
class Shape:
    """Problem shape. ``N`` is the sequence length (prefill) or the cache
    capacity Lmax (decode)."""
    dtype: str          # "f32" or "bf16"
    B: int
    Hq: int
    Hkv: int
    d: int
    N: int
    S: int
    W: int
    K: int
    structure: str = "plain"
    needle_every: int = 0
    n_needles: int = 0
    extra: dict = field(default_factory=dict, compare=False, hash=False)

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def nC(self) -> int:
        return self.N // self.S

    def with_(self, **kw) -> "Shape":
        return replace(self, **kw)


# The five benchmark workloads (1: small f32 check; 2, 3, 5: prefill at
# 32K, 128K, 512K; 4: batch-8 decode over 512K caches).
PREFILL_CONFIGS = {
    1: Shape("f32", 1, 1, 1, 64, 1024, 64, 128, 4, "plain"),
    2: Shape("bf16", 1, 32, 8, 128, 32768, 64, 512, 16, "needles", n_needles=8),
    3: Shape("bf16", 1, 32, 8, 128, 131072, 64, 1024, 32, "temperature"),
    5: Shape("bf16", 1, 32, 8, 128, 524288, 128, 2048, 32, "needles",
             needle_every=65536),
}
DECODE_CONFIGS = {
    4: Shape("bf16", 8, 32, 8, 128, 524288, 64, 512, 32, "plain"),
}
CONFIG_TEXT = {
    1: "prefill f32 B=1 H=1 d=64 N=1024 S=64 W=128 K=4 (plain)",
    2: "prefill bf16 B=1 Hq=32 Hkv=8 d=128 N=32768 S=64 W=512 K=16 (needles)",
    3: "prefill bf16 B=1 Hq=32 Hkv=8 d=128 N=131072 S=64 W=1024 K=32 (temperature)",
    4: "decode bf16 B=8 Hq=32 Hkv=8 d=128 L=524288 S=64 W=512 K=32 (plain)",
    5: "prefill bf16 B=1 Hq=32 Hkv=8 d=128 N=524288 S=128 W=2048 K=32 (needles every 64K)",
}


def seed_for(config_id: int, rep: int = 0) -> int:
    return config_id * 1000 + rep


def default_head_map(Hq: int, Hkv: int) -> list[int]:
    """Standard GQA grouping: query head h reads kv head h // (Hq/Hkv)."""
    G = Hq // Hkv
    return [h // G for h in range(Hq)]


def _torch_dtype(name: str) -> torch.dtype:
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


class _Rng:
    def __init__(self, seed: int, device):
        self.device = torch.device(device)
        self.g = torch.Generator(device=self.device)
        self.g.manual_seed(seed)

    def randn(self, *shape):
        return torch.randn(*shape, generator=self.g, device=self.device,
                           dtype=torch.float32)

    def randint(self, lo, hi, shape):
        return torch.randint(lo, hi, shape, generator=self.g,
                             device=self.device)


def _landmarks_from_keys(rng: _Rng, Kf: torch.Tensor, S: int, nC: int,
                         noise: float = 0.1):
    """k'_c = mean of the chunk's keys + N(0, noise^2); Kf [B,H,N,d] fp32."""
    B, H, _, d = Kf.shape
    klm = torch.empty(B, H, nC, d, device=Kf.device, dtype=torch.float32)
    step = max(1, (1 << 24) // max(1, S * d))       # chunks per slice
    for c0 in range(0, nC, step):
        c1 = min(nC, c0 + step)
        blk = Kf[:, :, c0 * S:c1 * S, :].reshape(B, H, c1 - c0, S, d)
        klm[:, :, c0:c1, :] = blk.mean(dim=3)
    klm += noise * rng.randn(B, H, nC, d)
    return klm


def make_prefill(shape: Shape, seed: int, device="cpu", head_map=None,
                 bias_std: float = 0.5):
    """Inputs of one prefill problem.

    Returns a dict with Q, Qs (None unless structure == 'qcal'), K, V, Klm,
    bias (float32), head_map (list of Hq ints) and shape. Q/Qs are
    [B,Hq,N,d], K/V [B,Hkv,N,d], Klm [B,Hkv,nC,d], bias [B,Hkv,nC]; all
    contiguous, in ``shape.dtype`` except bias (float32).
    """
    sh = shape
    rng = _Rng(seed, device)
    B, Hq, Hkv, d, N, S = sh.B, sh.Hq, sh.Hkv, sh.d, sh.N, sh.S
    nC = N // S
    hm = list(head_map) if head_map is not None else default_head_map(Hq, Hkv)
    dt = _torch_dtype(sh.dtype)

    Q = rng.randn(B, Hq, N, d)
    Kf = rng.randn(B, Hkv, N, d)
    V = rng.randn(B, Hkv, N, d).to(dt)
    Qs = None

    if sh.structure == "needles":
        u = rng.randn(B, Hkv, d)
        u /= u.norm(dim=-1, keepdim=True)
        if sh.needle_every:
            regions = max(1, N // sh.needle_every)
            per = sh.needle_every // S
            base = torch.arange(regions, device=rng.device) * per
            offs = rng.randint(0, per, (B, Hkv, regions))
            chunks = base.view(1, 1, -1) + offs
        else:
            chunks = rng.randint(0, max(1, nC), (B, Hkv, max(1, sh.n_needles)))
        tok = rng.randint(0, S, tuple(chunks.shape))
        pos = chunks * S + tok                       # [B,Hkv,n]
        noise = rng.randn(*pos.shape, d)
        first = pos.min(dim=-1).values              # [B,Hkv]
        for b in range(B):
            for g in range(Hkv):
                for n in range(pos.shape[-1]):
                    p = int(pos[b, g, n])
                    if p < N:
                        Kf[b, g, p] = 8.0 * u[b, g] + 0.1 * noise[b, g, n]
        for h in range(Hq):
            g = hm[h]
            for b in range(B):
                f = int(first[b, g])
                Q[b, h, f + 1:] += 4.0 * u[b, g]
    elif sh.structure == "temperature":
        taus = torch.tensor([0.1, 1.0, 4.0], device=rng.device)
        pick = rng.randint(0, 3, (B, Hkv, nC))
        t = taus[pick]                               # [B,Hkv,nC]
        Kf[:, :, :nC * S, :] *= t.repeat_interleave(S, dim=2).unsqueeze(-1)
    elif sh.structure == "exact":
        kbar = rng.randn(B, Hkv, nC, d).to(dt).float()
        Kf[:, :, :nC * S, :] = kbar.repeat_interleave(S, dim=2)
    elif sh.structure == "qcal":
        Qs = (Q + 0.5 * rng.randn(B, Hq, N, d)).to(dt)
    elif sh.structure != "plain":
        raise ValueError(f"unknown structure {sh.structure!r}")

    Kq = Kf.to(dt)
    if sh.structure == "exact":
        Klm = Kq[:, :, :nC * S:S, :].contiguous() if nC else \
            torch.empty(B, Hkv, 0, d, device=rng.device, dtype=dt)
        bias = torch.full((B, Hkv, nC), math.log(S), device=rng.device,
                          dtype=torch.float32)
    else:
        Klm = _landmarks_from_keys(rng, Kq.float(), S, nC).to(dt)
        bias = bias_std * rng.randn(B, Hkv, nC)
    del Kf
    return dict(Q=Q.to(dt).contiguous(), Qs=Qs, K=Kq.contiguous(),
                V=V.contiguous(), Klm=Klm.contiguous(),
                bias=bias.contiguous(), head_map=hm, shape=sh)


def make_decode(shape: Shape, seed: int, device="cpu", head_map=None,
                cache_len=None, bias_std: float = 0.5):
    """Inputs of one decode step: B sequences with one query each.

    Q [B,Hq,d]; K/V caches [B,Hkv,Lmax,d]; Klm [B,Hkv,Lmax/S,d]; bias
    [B,Hkv,Lmax/S] float32; cache_len int32 [B] (default: every sequence
    full, Lmax). Chunks at or beyond a sequence's length hold random values
    that a correct kernel never reads into the result.
    """
    sh = shape
    rng = _Rng(seed, device)
    B, Hq, Hkv, d, L, S = sh.B, sh.Hq, sh.Hkv, sh.d, sh.N, sh.S
    nC = L // S
    hm = list(head_map) if head_map is not None else default_head_map(Hq, Hkv)
    dt = _torch_dtype(sh.dtype)
    Q = rng.randn(B, Hq, d).to(dt)
    Kc = torch.empty(B, Hkv, L, d, device=rng.device, dtype=dt)
    Vc = torch.empty(B, Hkv, L, d, device=rng.device, dtype=dt)
    Klm = torch.empty(B, Hkv, nC, d, device=rng.device, dtype=dt)
    for b in range(B):                               # bound the fp32 temps
        kf = rng.randn(1, Hkv, L, d)
        Kc[b] = kf[0].to(dt)
        Vc[b] = rng.randn(Hkv, L, d).to(dt)
        Klm[b] = _landmarks_from_keys(rng, Kc[b:b + 1].float(), S, nC)[0].to(dt)
        del kf
    bias = bias_std * rng.randn(B, Hkv, nC)
    if cache_len is None:
        cl = torch.full((B,), L, dtype=torch.int32, device=rng.device)
    else:
        cl = torch.as_tensor(cache_len, dtype=torch.int32).to(rng.device)
    return dict(Q=Q.contiguous(), K=Kc, V=Vc, Klm=Klm, bias=bias.contiguous(),
                cache_len=cl, head_map=hm, shape=sh)
