"""Thin Python binding of libhils (include/hils.h): HiLS attention forward.

Argument marshalling only: every step of the computation runs in the CUDA
kernels of libhils.so. PyTorch supplies device memory and the stream. There
is no CPU fallback: if the library cannot be loaded, or a tensor is not on a
CUDA device, the call raises.

    O, idx = fwd_prefill(Q, K, V, Klm, bias, head_map, S=64, W=512, topk=16)
    O, idx = fwd_decode(Q, Kc, Vc, Klm, bias, cache_len, head_map, S, W, topk)
"""
from __future__ import annotations

import ctypes
import os
import threading

__all__ = [
    "HilsError", "lib", "library_path", "symbols", "status_string",
    "fwd_prefill", "fwd_decode", "prefill_workspace_size",
    "decode_workspace_size", "PrefillArgs", "DecodeArgs", "STATUS",
    "launch_count", "fwd_decode_noalloc", "build_landmarks", "LandmarkArgs",
    "chunk_overlap", "fwd_decode_paged", "DecodePagedArgs",
    "fwd_decode_multi", "DecodeMultiArgs", "bwd_prefill", "BackwardArgs",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_HERE, "libhils.so")

STATUS = {
    0: "HILS_OK", 1: "HILS_ERR_INVALID_ARG", 2: "HILS_ERR_UNSUPPORTED",
    3: "HILS_ERR_MISALIGNED", 4: "HILS_ERR_WORKSPACE_TOO_SMALL",
    5: "HILS_ERR_CUDA", 6: "HILS_ERR_DEVICE_TIMEOUT",
    7: "HILS_ERR_DEVICE_BAD_LENGTH",
}
F32, BF16 = 0, 1

# Every function include/hils.h declares.
symbols = [
    "hils_status_string", "hils_version", "hils_prefill_workspace_size",
    "hils_decode_workspace_size", "hils_fwd_prefill", "hils_fwd_decode",
    "hils_prefill_select", "hils_prefill_attend", "hils_decode_select",
    "hils_decode_attend", "hils_launch_count", "hils_fwd_decode_noalloc",
    "hils_build_landmarks", "hils_chunk_overlap",
    "hils_decode_paged_workspace_size", "hils_fwd_decode_paged",
    "hils_decode_multi_workspace_size", "hils_fwd_decode_multi",
    "hils_bwd_prefill_workspace_size", "hils_bwd_prefill",
]


class HilsError(RuntimeError):
    def __init__(self, code, where=""):
        self.code = int(code)
        super().__init__(f"{where}: {STATUS.get(self.code, self.code)}")


_p = ctypes.c_void_p
_i = ctypes.c_int32


class PrefillArgs(ctypes.Structure):
    _fields_ = [("dtype", _i), ("B", _i), ("Hq", _i), ("Hkv", _i), ("N", _i),
                ("d", _i), ("S", _i), ("W", _i), ("K", _i),
                ("head_map", _p), ("Q", _p), ("Qs", _p), ("Kc", _p),
                ("V", _p), ("Klm", _p), ("bias", _p), ("O", _p), ("idx", _p),
                ("sel_score", _p), ("workspace", _p),
                ("workspace_bytes", ctypes.c_size_t), ("status", _p)]


class DecodeArgs(ctypes.Structure):
    _fields_ = [("dtype", _i), ("B", _i), ("Hq", _i), ("Hkv", _i),
                ("Lmax", _i), ("d", _i), ("S", _i), ("W", _i), ("K", _i),
                ("head_map", _p), ("Q", _p), ("Qs", _p), ("Kc", _p),
                ("V", _p), ("Klm", _p), ("bias", _p), ("cache_len", _p),
                ("O", _p), ("idx", _p), ("sel_score", _p), ("workspace", _p),
                ("workspace_bytes", ctypes.c_size_t), ("status", _p)]


class DecodePagedArgs(ctypes.Structure):
    _fields_ = [("base", DecodeArgs), ("block_table", _p), ("n_pages", _i)]


class BackwardArgs(ctypes.Structure):
    _fields_ = [("dtype", _i), ("B", _i), ("Hq", _i), ("Hkv", _i), ("N", _i),
                ("d", _i), ("S", _i), ("W", _i), ("K", _i), ("head_map", _p),
                ("Q", _p), ("Qs", _p), ("Kc", _p), ("V", _p), ("Klm", _p),
                ("bias", _p), ("dO", _p), ("idx", _p), ("dQ", _p),
                ("dQs", _p), ("dK", _p), ("dV", _p), ("dKlm", _p),
                ("dbias", _p), ("workspace", _p),
                ("workspace_bytes", ctypes.c_size_t), ("status", _p)]


class DecodeMultiArgs(ctypes.Structure):
    _fields_ = [("base", DecodeArgs), ("T", _i), ("block_table", _p),
                ("n_pages", _i)]


class LandmarkArgs(ctypes.Structure):
    _fields_ = [("dtype", _i), ("B", _i), ("Hkv", _i), ("N", _i), ("d", _i),
                ("S", _i), ("Kc", _p), ("Qlm", _p), ("shared_query", _i),
                ("Klm", _p), ("bias", _p)]


_lib = None
_lock = threading.Lock()


def lib():
    """The loaded libhils.so (raises if it is missing: no fallback)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(library_path):
                raise ImportError(
                    f"libhils.so not built ({library_path}); run "
                    "python -m chunk_sparse_long_landmark_b200.build")
            L = ctypes.CDLL(library_path)
            L.hils_status_string.restype = ctypes.c_char_p
            L.hils_status_string.argtypes = [ctypes.c_int]
            L.hils_version.restype = ctypes.c_int32
            for n, T in (("prefill", PrefillArgs), ("decode", DecodeArgs)):
                f = getattr(L, f"hils_{n}_workspace_size")
                f.restype = ctypes.c_int
                f.argtypes = [ctypes.POINTER(T), ctypes.POINTER(ctypes.c_size_t)]
                for fn in (f"hils_fwd_{n}", f"hils_{n}_select",
                           f"hils_{n}_attend"):
                    f = getattr(L, fn)
                    f.restype = ctypes.c_int
                    f.argtypes = [ctypes.POINTER(T), ctypes.c_void_p]
            L.hils_launch_count.restype = ctypes.c_uint64
            L.hils_fwd_decode_noalloc.restype = ctypes.c_int
            L.hils_fwd_decode_noalloc.argtypes = [ctypes.POINTER(DecodeArgs),
                                                  ctypes.c_void_p]
            L.hils_build_landmarks.restype = ctypes.c_int
            L.hils_build_landmarks.argtypes = [ctypes.POINTER(LandmarkArgs),
                                               ctypes.c_void_p]
            L.hils_decode_paged_workspace_size.restype = ctypes.c_int
            L.hils_decode_paged_workspace_size.argtypes = [
                ctypes.POINTER(DecodePagedArgs), ctypes.POINTER(ctypes.c_size_t)]
            L.hils_fwd_decode_paged.restype = ctypes.c_int
            L.hils_fwd_decode_paged.argtypes = [ctypes.POINTER(DecodePagedArgs),
                                                ctypes.c_void_p]
            L.hils_decode_multi_workspace_size.restype = ctypes.c_int
            L.hils_decode_multi_workspace_size.argtypes = [
                ctypes.POINTER(DecodeMultiArgs), ctypes.POINTER(ctypes.c_size_t)]
            L.hils_fwd_decode_multi.restype = ctypes.c_int
            L.hils_fwd_decode_multi.argtypes = [ctypes.POINTER(DecodeMultiArgs),
                                                ctypes.c_void_p]
            L.hils_bwd_prefill_workspace_size.restype = ctypes.c_int
            L.hils_bwd_prefill_workspace_size.argtypes = [
                ctypes.POINTER(BackwardArgs), ctypes.POINTER(ctypes.c_size_t)]
            L.hils_bwd_prefill.restype = ctypes.c_int
            L.hils_bwd_prefill.argtypes = [ctypes.POINTER(BackwardArgs),
                                           ctypes.c_void_p]
            L.hils_chunk_overlap.restype = ctypes.c_int
            L.hils_chunk_overlap.argtypes = [_p] + [_i] * 6 + [_p] * 4
            _lib = L
    return _lib


def status_string(code: int) -> str:
    return lib().hils_status_string(int(code)).decode()


def _dtype_code(t):
    import torch
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _ptr(t):
    return None if t is None else t.data_ptr()


def _dev(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("libhils needs CUDA tensors (no CPU fallback)")


def _stream_handle(stream):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _head_map_array(head_map, Hq):
    hm = list(head_map)
    arr = (ctypes.c_int32 * max(1, len(hm)))(*hm)
    return arr


def _prefill_struct(Q, K, V, Klm, bias, head_map, S, W, topk, Qs=None,
                    O=None, idx=None, sel_score=None, workspace=None,
                    status=None):
    B, Hq, N, d = Q.shape
    Hkv = K.shape[1]
    hm = _head_map_array(head_map, Hq)
    a = PrefillArgs(_dtype_code(Q), B, Hq, Hkv, N, d, S, W, topk,
                    ctypes.cast(hm, ctypes.c_void_p), _ptr(Q), _ptr(Qs),
                    _ptr(K), _ptr(V), _ptr(Klm), _ptr(bias), _ptr(O),
                    _ptr(idx), _ptr(sel_score), _ptr(workspace),
                    0 if workspace is None else workspace.numel() *
                    workspace.element_size(), _ptr(status))
    return a, hm


def prefill_workspace_size(Q, K, V, Klm, bias, head_map, S, W, topk,
                           with_sel_score=False) -> int:
    a, hm = _prefill_struct(Q, K, V, Klm, bias, head_map, S, W, topk)
    if with_sel_score:
        a.sel_score = 16
    n = ctypes.c_size_t(0)
    rc = lib().hils_prefill_workspace_size(ctypes.byref(a), ctypes.byref(n))
    if rc:
        raise HilsError(rc, "hils_prefill_workspace_size")
    return int(n.value)


def launch_count() -> int:
    """Kernel launches libhils has enqueued in this process so far."""
    return int(lib().hils_launch_count())


_STAGE_FN = {"both": "hils_fwd_{}", "select": "hils_{}_select",
             "attend": "hils_{}_attend"}


def fwd_prefill(Q, K, V, Klm, bias, head_map, S, W, topk, Qs=None, out=None,
                idx=None, sel_score=None, workspace=None, status=None,
                stream=None, stage="both"):
    """HiLS prefill forward through hils_fwd_prefill. Returns (O, idx).

    stage="select" / "attend" calls hils_prefill_select / _attend instead
    (attend needs the idx and scores of a select call: pass sel_score, or the
    same workspace, to both).

    Q/Qs [B,Hq,N,d], K/V [B,Hkv,N,d], Klm [B,Hkv,N//S,d] (same dtype),
    bias [B,Hkv,N//S] float32, head_map: Hq ints. Outputs are allocated with
    torch when not given; the workspace too (torch's caching allocator).
    """
    import torch
    _dev(Q, K, V, Klm, bias, Qs, out, idx, sel_score, workspace, status)
    B, Hq, N, d = Q.shape
    Hkv = K.shape[1]
    if out is None:
        out = torch.empty_like(Q)
    if idx is None:
        idx = torch.empty(B, Hkv, N, topk, dtype=torch.int32, device=Q.device)
    if workspace is None:
        n = prefill_workspace_size(Q, K, V, Klm, bias, head_map, S, W, topk,
                                   with_sel_score=sel_score is not None)
        workspace = torch.empty(n, dtype=torch.uint8, device=Q.device)
    a, hm = _prefill_struct(Q, K, V, Klm, bias, head_map, S, W, topk, Qs,
                            out, idx, sel_score, workspace, status)
    fn = _STAGE_FN[stage].format("prefill")
    rc = getattr(lib(), fn)(ctypes.byref(a), _stream_handle(stream))
    if rc:
        raise HilsError(rc, fn)
    return out, idx


def _decode_struct(Q, K, V, Klm, bias, cache_len, head_map, S, W, topk,
                   Qs=None, O=None, idx=None, sel_score=None, workspace=None,
                   status=None):
    B, Hq, d = Q.shape
    Hkv, Lmax = K.shape[1], K.shape[2]
    hm = _head_map_array(head_map, Hq)
    a = DecodeArgs(_dtype_code(Q), B, Hq, Hkv, Lmax, d, S, W, topk,
                   ctypes.cast(hm, ctypes.c_void_p), _ptr(Q), _ptr(Qs),
                   _ptr(K), _ptr(V), _ptr(Klm), _ptr(bias), _ptr(cache_len),
                   _ptr(O), _ptr(idx), _ptr(sel_score), _ptr(workspace),
                   0 if workspace is None else workspace.numel() *
                   workspace.element_size(), _ptr(status))
    return a, hm


def decode_workspace_size(Q, K, V, Klm, bias, cache_len, head_map, S, W,
                          topk, with_sel_score=False) -> int:
    a, hm = _decode_struct(Q, K, V, Klm, bias, cache_len, head_map, S, W,
                           topk)
    if with_sel_score:
        a.sel_score = 16
    n = ctypes.c_size_t(0)
    rc = lib().hils_decode_workspace_size(ctypes.byref(a), ctypes.byref(n))
    if rc:
        raise HilsError(rc, "hils_decode_workspace_size")
    return int(n.value)


def fwd_decode(Q, K, V, Klm, bias, cache_len, head_map, S, W, topk, Qs=None,
               out=None, idx=None, sel_score=None, workspace=None,
               status=None, stream=None, stage="both"):
    """HiLS decode step through hils_fwd_decode. Returns (O, idx).

    Q/Qs [B,Hq,d]; K/V caches [B,Hkv,Lmax,d]; Klm [B,Hkv,Lmax//S,d];
    bias [B,Hkv,Lmax//S] float32; cache_len int32 [B] on the device.
    """
    import torch
    _dev(Q, K, V, Klm, bias, cache_len, Qs, out, idx, sel_score, workspace,
         status)
    B, Hq, d = Q.shape
    Hkv = K.shape[1]
    if out is None:
        out = torch.empty_like(Q)
    if idx is None:
        idx = torch.empty(B, Hkv, topk, dtype=torch.int32, device=Q.device)
    if workspace is None:
        n = decode_workspace_size(Q, K, V, Klm, bias, cache_len, head_map, S,
                                  W, topk, with_sel_score=sel_score is not None)
        workspace = torch.empty(n, dtype=torch.uint8, device=Q.device)
    a, hm = _decode_struct(Q, K, V, Klm, bias, cache_len, head_map, S, W,
                           topk, Qs, out, idx, sel_score, workspace, status)
    fn = _STAGE_FN[stage].format("decode")
    rc = getattr(lib(), fn)(ctypes.byref(a), _stream_handle(stream))
    if rc:
        raise HilsError(rc, fn)
    return out, idx


def fwd_decode_noalloc(Q, K, V, Klm, bias, cache_len, head_map, S, W, topk,
                       Qs=None, out=None, idx=None, sel_score=None,
                       status=None, stream=None):
    """Decode step through hils_fwd_decode_noalloc: no workspace is passed;
    the library's fixed device scratch is used. Returns (O, idx). Outputs are
    allocated with torch here only when not given."""
    import torch
    _dev(Q, K, V, Klm, bias, cache_len, Qs, out, idx, sel_score, status)
    B, Hq, d = Q.shape
    Hkv = K.shape[1]
    if out is None:
        out = torch.empty_like(Q)
    if idx is None:
        idx = torch.empty(B, Hkv, topk, dtype=torch.int32, device=Q.device)
    a, hm = _decode_struct(Q, K, V, Klm, bias, cache_len, head_map, S, W,
                           topk, Qs, out, idx, sel_score, None, status)
    rc = lib().hils_fwd_decode_noalloc(ctypes.byref(a), _stream_handle(stream))
    if rc:
        raise HilsError(rc, "hils_fwd_decode_noalloc")
    return out, idx


def build_landmarks(K, Qlm, S, out=None, stream=None):
    """Landmark summaries (k', b') of every full chunk through
    hils_build_landmarks: K [B,Hkv,N,d]; Qlm [B,Hkv,N//S,d] (one landmark
    query per chunk) or [Hkv,d] (one shared query per kv head). Returns
    (Klm [B,Hkv,N//S,d] in K's dtype, bias [B,Hkv,N//S] float32)."""
    import torch
    _dev(K, Qlm)
    B, Hkv, N, d = K.shape
    nC = N // S
    shared = 1 if Qlm.dim() == 2 else 0
    if Qlm.dtype != K.dtype:
        raise TypeError("Qlm must have K's dtype")
    if not (K.is_contiguous() and Qlm.is_contiguous()):
        raise ValueError("K and Qlm must be contiguous")
    if out is None:
        out = (torch.empty(B, Hkv, nC, d, dtype=K.dtype, device=K.device),
               torch.empty(B, Hkv, nC, dtype=torch.float32, device=K.device))
    Klm, bias = out
    a = LandmarkArgs(_dtype_code(K), B, Hkv, N, d, S, _ptr(K), _ptr(Qlm),
                     shared, _ptr(Klm), _ptr(bias))
    rc = lib().hils_build_landmarks(ctypes.byref(a), _stream_handle(stream))
    if rc != 0:
        raise HilsError(rc, "hils_build_landmarks")
    return Klm, bias


def chunk_overlap(idx, nC, M, stream=None):
    """Per block of M consecutive query rows of idx [B,Hkv,N,K] (int32, as
    the select stage writes it): (n_sel, n_union, n_reuse), each
    [B,Hkv,ceil(N/M)] int32, through hils_chunk_overlap."""
    import torch
    _dev(idx)
    if idx.dtype != torch.int32 or not idx.is_contiguous():
        raise ValueError("idx must be a contiguous int32 tensor")
    B, Hkv, N, K = idx.shape
    nb = (N + M - 1) // M
    outs = [torch.empty(B, Hkv, nb, dtype=torch.int32, device=idx.device)
            for _ in range(3)]
    rc = lib().hils_chunk_overlap(_ptr(idx), B, Hkv, N, K, int(nC), int(M),
                                  *[_ptr(t) for t in outs],
                                  _stream_handle(stream))
    if rc != 0:
        raise HilsError(rc, "hils_chunk_overlap")
    return tuple(outs)


def fwd_decode_paged(Q, Kpool, Vpool, Klm, bias, cache_len, block_table,
                     head_map, S, W, topk, Qs=None, out=None, idx=None,
                     sel_score=None, workspace=None, status=None,
                     stream=None):
    """HiLS decode step over a paged cache (page = chunk) through
    hils_fwd_decode_paged. Returns (O, idx).

    Kpool/Vpool [n_pages,Hkv,S,d]; block_table int32 [B, Lmax//S] on the
    device (page of each logical chunk); Klm [B,Hkv,Lmax//S,d] and bias
    [B,Hkv,Lmax//S] per sequence; cache_len int32 [B] on the device."""
    import torch
    _dev(Q, Kpool, Vpool, Klm, bias, cache_len, block_table, Qs, out, idx,
         sel_score, workspace, status)
    if block_table.dtype != torch.int32 or not block_table.is_contiguous():
        raise ValueError("block_table must be a contiguous int32 tensor")
    B, Hq, d = Q.shape
    P, Hkv = Kpool.shape[0], Kpool.shape[1]
    Lmax = block_table.shape[1] * S
    hm = _head_map_array(head_map, Hq)
    if out is None:
        out = torch.empty_like(Q)
    if idx is None:
        idx = torch.empty(B, Hkv, topk, dtype=torch.int32, device=Q.device)

    def record(ws):
        base = DecodeArgs(_dtype_code(Q), B, Hq, Hkv, Lmax, d, S, W, topk,
                          ctypes.cast(hm, ctypes.c_void_p), _ptr(Q), _ptr(Qs),
                          _ptr(Kpool), _ptr(Vpool), _ptr(Klm), _ptr(bias),
                          _ptr(cache_len), _ptr(out), _ptr(idx),
                          _ptr(sel_score), _ptr(ws),
                          0 if ws is None else ws.numel() * ws.element_size(),
                          _ptr(status))
        return DecodePagedArgs(base, _ptr(block_table), P)

    if workspace is None:
        n = ctypes.c_size_t(0)
        rc = lib().hils_decode_paged_workspace_size(ctypes.byref(record(None)),
                                                    ctypes.byref(n))
        if rc:
            raise HilsError(rc, "hils_decode_paged_workspace_size")
        workspace = torch.empty(max(n.value, 1), dtype=torch.uint8,
                                device=Q.device)
    a = record(workspace)
    rc = lib().hils_fwd_decode_paged(ctypes.byref(a), _stream_handle(stream))
    if rc:
        raise HilsError(rc, "hils_fwd_decode_paged")
    return out, idx


def fwd_decode_multi(Q, Kc, V, Klm, bias, cache_len, head_map, S, W, topk,
                     block_table=None, Qs=None, out=None, idx=None,
                     sel_score=None, workspace=None, status=None,
                     stream=None):
    """Multi-token (speculative) decode through hils_fwd_decode_multi.
    Returns (O, idx).

    Q [B,T,Hq,d] (token-major): token t of sequence b sits at position
    cache_len[b]-T+t. Kc/V [B,Hkv,Lmax,d], or the page pool [n_pages,Hkv,S,d]
    when block_table (int32 [B, Lmax//S], device) is given. Klm
    [B,Hkv,Lmax//S,d], bias [B,Hkv,Lmax//S], cache_len int32 [B] on the
    device. O [B,T,Hq,d], idx [B,T,Hkv,topk]."""
    import torch
    _dev(Q, Kc, V, Klm, bias, cache_len, block_table, Qs, out, idx,
         sel_score, workspace, status)
    B, T, Hq, d = Q.shape
    Hkv = Kc.shape[1]
    if block_table is not None:
        if block_table.dtype != torch.int32 or not block_table.is_contiguous():
            raise ValueError("block_table must be a contiguous int32 tensor")
        Lmax = block_table.shape[1] * S
        n_pages = Kc.shape[0]
    else:
        Lmax = Kc.shape[2]
        n_pages = 0
    hm = _head_map_array(head_map, Hq)
    if out is None:
        out = torch.empty_like(Q)
    if idx is None:
        idx = torch.empty(B, T, Hkv, topk, dtype=torch.int32, device=Q.device)

    def record(ws):
        base = DecodeArgs(_dtype_code(Q), B, Hq, Hkv, Lmax, d, S, W, topk,
                          ctypes.cast(hm, ctypes.c_void_p), _ptr(Q), _ptr(Qs),
                          _ptr(Kc), _ptr(V), _ptr(Klm), _ptr(bias),
                          _ptr(cache_len), _ptr(out), _ptr(idx),
                          _ptr(sel_score), _ptr(ws),
                          0 if ws is None else ws.numel() * ws.element_size(),
                          _ptr(status))
        return DecodeMultiArgs(base, T, _ptr(block_table), n_pages)

    if workspace is None:
        n = ctypes.c_size_t(0)
        rc = lib().hils_decode_multi_workspace_size(ctypes.byref(record(None)),
                                                    ctypes.byref(n))
        if rc:
            raise HilsError(rc, "hils_decode_multi_workspace_size")
        workspace = torch.empty(max(n.value, 1), dtype=torch.uint8,
                                device=Q.device)
    a = record(workspace)
    rc = lib().hils_fwd_decode_multi(ctypes.byref(a), _stream_handle(stream))
    if rc:
        raise HilsError(rc, "hils_fwd_decode_multi")
    return out, idx


def bwd_prefill(Q, K, V, Klm, bias, head_map, S, W, idx, dO, Qs=None,
                grads=None, workspace=None, stream=None):
    """Backward of the prefill forward for a fixed selection, through
    hils_bwd_prefill. Returns a dict of float32 gradients dQ, dQs (None
    without Qs: folded into dQ), dK, dV, dKlm, dbias.

    Q/Qs/dO [B,Hq,N,d], K/V [B,Hkv,N,d], Klm [B,Hkv,N//S,d], bias
    [B,Hkv,N//S] (f32), idx [B,Hkv,N,topk] int32: the forward's selection.
    `grads` may hold preallocated outputs under the same keys."""
    import torch
    _dev(Q, K, V, Klm, bias, idx, dO, Qs, workspace)
    B, Hq, N, d = Q.shape
    Hkv = K.shape[1]
    topk = idx.shape[-1]
    hm = _head_map_array(head_map, Hq)
    f32 = dict(dtype=torch.float32, device=Q.device)
    g = dict(grads or {})
    g.setdefault("dQ", torch.empty(B, Hq, N, d, **f32))
    g.setdefault("dQs", torch.empty(B, Hq, N, d, **f32) if Qs is not None else None)
    g.setdefault("dK", torch.empty(B, Hkv, N, d, **f32))
    g.setdefault("dV", torch.empty(B, Hkv, N, d, **f32))
    g.setdefault("dKlm", torch.empty(B, Hkv, max(N // S, 1), d, **f32))
    g.setdefault("dbias", torch.empty(B, Hkv, max(N // S, 1), **f32))

    def record(ws):
        return BackwardArgs(_dtype_code(Q), B, Hq, Hkv, N, d, S, W, topk,
                            ctypes.cast(hm, ctypes.c_void_p), _ptr(Q),
                            _ptr(Qs), _ptr(K), _ptr(V), _ptr(Klm), _ptr(bias),
                            _ptr(dO), _ptr(idx), _ptr(g["dQ"]), _ptr(g["dQs"]),
                            _ptr(g["dK"]), _ptr(g["dV"]), _ptr(g["dKlm"]),
                            _ptr(g["dbias"]), _ptr(ws),
                            0 if ws is None else ws.numel() * ws.element_size())

    if workspace is None:
        n = ctypes.c_size_t(0)
        rc = lib().hils_bwd_prefill_workspace_size(ctypes.byref(record(None)),
                                                   ctypes.byref(n))
        if rc:
            raise HilsError(rc, "hils_bwd_prefill_workspace_size")
        workspace = torch.empty(max(n.value, 1), dtype=torch.uint8,
                                device=Q.device)
    rc = lib().hils_bwd_prefill(ctypes.byref(record(workspace)),
                                _stream_handle(stream))
    if rc:
        raise HilsError(rc, "hils_bwd_prefill")
    return g
