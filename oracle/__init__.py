"""fp64 CPU oracle of HiLS attention forward (prefill and decode).

TEST INFRASTRUCTURE ONLY: imported by the tests, by the smoke check and by
the benchmark's CPU-baseline leg, never by the product path. It shares no
code with the CUDA library.

Two independent implementations live here:

* ``hils_oracle.c`` (loaded through ctypes): the method step by step, in
  plain C loops, double precision, OpenMP over query rows. See its header
  for the passages of "Hierarchical Sparse Attention Done Right" it follows
  and the readings it fixes.
* ``brute.py``: a whole-tensor numpy restatement for tiny problems, written
  separately (dense score matrices and masks instead of per-row loops), used
  to pin the C oracle.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hils_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

SCORE_LANDMARK = 0
SCORE_EXACT = 1


def build(force: bool = False) -> str:
    """Compile hils_oracle.c into liboracle.so (gcc, -O2, no fast-math)."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
           "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    return _LIB


class _Problem(ctypes.Structure):
    _fields_ = [
        ("dtype", ctypes.c_int), ("B", ctypes.c_int), ("Hq", ctypes.c_int),
        ("Hkv", ctypes.c_int), ("d", ctypes.c_int), ("S", ctypes.c_int),
        ("W", ctypes.c_int), ("K", ctypes.c_int), ("q_rows", ctypes.c_int),
        ("kv_rows", ctypes.c_int), ("nC", ctypes.c_int),
        ("head_map", ctypes.c_void_p), ("Q", ctypes.c_void_p),
        ("Qs", ctypes.c_void_p), ("Kc", ctypes.c_void_p),
        ("V", ctypes.c_void_p), ("Klm", ctypes.c_void_p),
        ("bias", ctypes.c_void_p),
    ]


def load_library(path):
    """Open a compiled oracle library and declare its entry points."""
    lib = ctypes.CDLL(path)
    lib.oracle_rows.restype = ctypes.c_int
    lib.oracle_rows.argtypes = [
        ctypes.POINTER(_Problem), ctypes.c_int64,
        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
        ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p,
        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
    lib.oracle_max_threads.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            _lib = load_library(_LIB)
    return _lib


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def _host(x):
    """torch tensor / numpy array -> contiguous host numpy array holding the
    same bits (bf16 becomes uint16 storage)."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().contiguous()
            if x.dtype == torch.bfloat16:
                return x.view(torch.int16).numpy().view(np.uint16), 1
            if x.dtype == torch.float32:
                return x.numpy(), 0
            return x.numpy(), -1
    except ImportError:                                   # pragma: no cover
        pass
    x = np.ascontiguousarray(x)
    if x.dtype == np.float32:
        return x, 0
    if x.dtype == np.uint16:
        return x, 1
    return x, -1


def _ptr(a):
    return None if a is None else a.ctypes.data


class _Bound:
    """Host copies of one problem's arrays + the C struct that points at them."""

    def __init__(self, Q, Qs, K, V, Klm, bias, head_map, S, W, Kt, q_rows):
        self.Q, dt = _host(Q)
        self.Qs = _host(Qs)[0] if Qs is not None else None
        self.K, dk = _host(K)
        self.V, dv = _host(V)
        self.Klm, dl = _host(Klm)
        if not (dt == dk == dv == dl) or dt not in (0, 1):
            raise TypeError("Q, K, V, Klm must share one dtype (f32 or bf16)")
        self.bias = np.ascontiguousarray(_host(bias)[0], dtype=np.float32)
        self.hm = np.ascontiguousarray(np.asarray(head_map, dtype=np.int32))
        B, Hkv, kv_rows, d = self.K.shape
        Hq = self.Q.shape[1]
        nC = self.Klm.shape[2]
        self.dims = dict(B=B, Hq=Hq, Hkv=Hkv, d=d, kv_rows=kv_rows, nC=nC,
                         S=S, W=W, K=Kt, G=Hq // Hkv)
        self.p = _Problem(dt, B, Hq, Hkv, d, S, W, Kt, q_rows, kv_rows, nC,
                          _ptr(self.hm), _ptr(self.Q), _ptr(self.Qs),
                          _ptr(self.K), _ptr(self.V), _ptr(self.Klm),
                          _ptr(self.bias))

    def rows(self, rb, rg, ri, rr, score_mode=SCORE_LANDMARK,
             imposed_idx=None, threads=0):
        lib = _load()
        rb = np.ascontiguousarray(rb, dtype=np.int32)
        rg = np.ascontiguousarray(rg, dtype=np.int32)
        ri = np.ascontiguousarray(ri, dtype=np.int64)
        rr = np.ascontiguousarray(rr, dtype=np.int32)
        n = rb.shape[0]
        G, d, K = self.dims["G"], self.dims["d"], self.dims["K"]
        O = np.zeros((n, G, d), dtype=np.float64)
        idx = np.zeros((n, K), dtype=np.int32)
        shat = np.zeros((n, G, K), dtype=np.float64)
        gap = np.zeros((n,), dtype=np.float64)
        akth = np.zeros((n,), dtype=np.float64)
        lse = np.zeros((n, G), dtype=np.float64)
        imp = None
        if imposed_idx is not None:
            imp = np.ascontiguousarray(imposed_idx, dtype=np.int32)
            assert imp.shape == (n, K)
        fails = lib.oracle_rows(ctypes.byref(self.p), n, _ptr(rb), _ptr(rg),
                                _ptr(ri), _ptr(rr), int(score_mode), _ptr(imp),
                                _ptr(O), _ptr(idx), _ptr(shat), _ptr(gap),
                                _ptr(akth), _ptr(lse), int(threads))
        if fails:
            raise RuntimeError(f"oracle failed on {fails} rows")
        return dict(O=O, idx=idx, shat_sel=shat, gap=gap, akth=akth,
                    lse=lse)


def group_heads(head_map, g):
    return [h for h, x in enumerate(head_map) if x == g]


def prefill_rows(inp, rows, score_mode=SCORE_LANDMARK, imposed_idx=None,
                 threads=0, bound=None):
    """Oracle on selected prefill rows.

    inp: dict from ``synth.make_prefill`` (Q, Qs, K, V, Klm, bias, head_map,
    shape). rows: int array [n, 3] of (b, g, i). Returns per-row arrays:
    O [n,G,d] (float64), idx [n,K], shat_sel [n,G,K], gap [n], akth [n]
    (a_(K), the lowest selected group score), lse [n,G].
    """
    sh = inp["shape"]
    bd = bound or _Bound(inp["Q"], inp.get("Qs"), inp["K"], inp["V"],
                         inp["Klm"], inp["bias"], inp["head_map"], sh.S,
                         sh.W, sh.K, q_rows=sh.N)
    rows = np.asarray(rows, dtype=np.int64).reshape(-1, 3)
    return bd.rows(rows[:, 0], rows[:, 1], rows[:, 2], rows[:, 2],
                   score_mode, imposed_idx, threads)


def bind_prefill(inp):
    sh = inp["shape"]
    return _Bound(inp["Q"], inp.get("Qs"), inp["K"], inp["V"], inp["Klm"],
                  inp["bias"], inp["head_map"], sh.S, sh.W, sh.K,
                  q_rows=sh.N)


def prefill_full(inp, score_mode=SCORE_LANDMARK, threads=0):
    """Oracle on every (b, g, i). Returns O [B,Hq,N,d] float64,
    idx [B,Hkv,N,K], shat_sel [B,Hq,N,K], gap [B,Hkv,N]."""
    sh = inp["shape"]
    B, Hkv, N = sh.B, sh.Hkv, sh.N
    bb, gg, ii = np.meshgrid(np.arange(B), np.arange(Hkv), np.arange(N),
                             indexing="ij")
    rows = np.stack([bb.ravel(), gg.ravel(), ii.ravel()], axis=1)
    r = prefill_rows(inp, rows, score_mode=score_mode, threads=threads)
    return scatter_prefill(inp, rows, r)


def scatter_prefill(inp, rows, r):
    sh = inp["shape"]
    hm = inp["head_map"]
    O = np.full((sh.B, sh.Hq, sh.N, sh.d), np.nan)
    shat = np.full((sh.B, sh.Hq, sh.N, sh.K), np.nan)
    idx = np.full((sh.B, sh.Hkv, sh.N, sh.K), -2, dtype=np.int32)
    gap = np.full((sh.B, sh.Hkv, sh.N), np.nan)
    akth = np.full((sh.B, sh.Hkv, sh.N), np.nan)
    for g in range(sh.Hkv):
        heads = group_heads(hm, g)
        m = rows[:, 1] == g
        b, i = rows[m, 0], rows[m, 2]
        idx[b, g, i] = r["idx"][m]
        gap[b, g, i] = r["gap"][m]
        akth[b, g, i] = r["akth"][m]
        for hh, h in enumerate(heads):
            O[b, h, i] = r["O"][m, hh]
            shat[b, h, i] = r["shat_sel"][m, hh]
    return dict(O=O, idx=idx, shat_sel=shat, gap=gap, akth=akth)


def decode(inp, score_mode=SCORE_LANDMARK, imposed_idx=None, threads=0,
           batches=None):
    """Oracle for one decode step: query i = cache_len[b]-1 of each sequence.

    Returns O [B,Hq,d] float64, idx [B,Hkv,K], shat_sel [B,Hq,K],
    gap [B,Hkv], akth [B,Hkv], lse [B,Hq]. ``batches`` restricts the evaluated sequences
    (others are left NaN / -2). ``imposed_idx``: [B,Hkv,K] or None.
    """
    sh = inp["shape"]
    B, Hkv, G, K = sh.B, sh.Hkv, sh.G, sh.K
    Q = inp["Q"]
    q4 = Q.reshape(Q.shape[0], Q.shape[1], 1, Q.shape[2])
    bd = _Bound(q4, None, inp["K"], inp["V"], inp["Klm"], inp["bias"],
                inp["head_map"], sh.S, sh.W, K, q_rows=1)
    cl = np.asarray(_host(inp["cache_len"])[0], dtype=np.int64)
    bs = list(range(B)) if batches is None else list(batches)
    rb = np.repeat(np.asarray(bs), Hkv)
    rg = np.tile(np.arange(Hkv), len(bs))
    ri = cl[rb] - 1
    rr = np.zeros_like(rb)
    imp = None
    if imposed_idx is not None:
        imp = np.asarray(imposed_idx, dtype=np.int32)[rb, rg]
    r = bd.rows(rb, rg, ri, rr, score_mode, imp, threads)
    O = np.full((B, sh.Hq, sh.d), np.nan)
    shat = np.full((B, sh.Hq, K), np.nan)
    lse = np.full((B, sh.Hq), np.nan)
    idx = np.full((B, Hkv, K), -2, dtype=np.int32)
    gap = np.full((B, Hkv), np.nan)
    akth = np.full((B, Hkv), np.nan)
    hm = inp["head_map"]
    for n in range(len(rb)):
        b, g = rb[n], rg[n]
        idx[b, g] = r["idx"][n]
        gap[b, g] = r["gap"][n]
        akth[b, g] = r["akth"][n]
        for hh, h in enumerate(group_heads(hm, g)):
            O[b, h] = r["O"][n, hh]
            shat[b, h] = r["shat_sel"][n, hh]
            lse[b, h] = r["lse"][n, hh]
    return dict(O=O, idx=idx, shat_sel=shat, gap=gap, akth=akth, lse=lse)


def prefill_at(inp, positions, score_mode=SCORE_LANDMARK, imposed_idx=None,
               threads=0, groups=None, bound=None):
    """Oracle at chosen query positions of a (possibly huge) prefill problem.

    Only the Q / Qs rows at ``positions`` are copied to the host; K, V, Klm
    and bias are copied whole (or taken from ``bound``, a ``bind_at`` result
    for the same positions). ``groups`` restricts the kv groups evaluated
    (default: all, in order). Returns per-(b, g, position) arrays shaped
    O [B,nG,P,G,d], idx [B,nG,P,K], shat_sel [B,nG,P,G,K], gap/akth
    [B,nG,P], nG = len(groups). ``imposed_idx``: [B,nG,P,K] or None.
    """
    sh = inp["shape"]
    pos = np.asarray(positions, dtype=np.int64)
    P = len(pos)
    gs = np.arange(sh.Hkv) if groups is None else np.asarray(groups)
    nG = len(gs)
    bd = bound or bind_at(inp, pos)
    bb, gg, pp = np.meshgrid(np.arange(sh.B), gs, np.arange(P), indexing="ij")
    rb, rg, rp = bb.ravel(), gg.ravel(), pp.ravel()
    imp = None
    if imposed_idx is not None:
        imp = np.asarray(imposed_idx, dtype=np.int32).reshape(-1, sh.K)
    r = bd.rows(rb, rg, pos[rp], rp, score_mode, imp, threads)
    G, d, K = sh.G, sh.d, sh.K
    return dict(O=r["O"].reshape(sh.B, nG, P, G, d),
                idx=r["idx"].reshape(sh.B, nG, P, K),
                shat_sel=r["shat_sel"].reshape(sh.B, nG, P, G, K),
                gap=r["gap"].reshape(sh.B, nG, P),
                akth=r["akth"].reshape(sh.B, nG, P))


def bind_at(inp, positions):
    """Host copies for ``prefill_at`` at ``positions``: the Q / Qs rows at
    those positions, K, V, Klm and bias whole."""
    import torch
    sh = inp["shape"]
    pos = np.asarray(positions, dtype=np.int64)
    pt = torch.as_tensor(pos, device=inp["Q"].device)
    Qsub = inp["Q"].index_select(2, pt)
    Qssub = inp["Qs"].index_select(2, pt) if inp.get("Qs") is not None \
        else None
    return _Bound(Qsub, Qssub, inp["K"], inp["V"], inp["Klm"], inp["bias"],
                  inp["head_map"], sh.S, sh.W, sh.K, q_rows=len(pos))
