"""Host-only checks of the C ABI: the library loads, exports every function
include/hils.h declares, and rejects bad arguments before launching anything.
No GPU work is done here (every call below fails validation on the host or
only sizes the workspace)."""
import ctypes
import os
import re

import pytest

import chunk_sparse_long_landmark_b200 as hils
from chunk_sparse_long_landmark_b200 import build as hbuild

HDR = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include",
                   "hils.h")


@pytest.fixture(scope="module")
def L():
    hbuild.build()
    return hils.lib()


def header_functions():
    txt = open(HDR).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(hils_[a-z_0-9]+)\s*\(", txt)))


def test_header_symbols_exported(L):
    names = header_functions()
    assert names, "no functions parsed from include/hils.h"
    assert sorted(hils.symbols) == names
    for n in names:
        assert hasattr(L, n), f"libhils.so does not export {n}"


def test_status_strings(L):
    for code, name in hils.STATUS.items():
        assert hils.status_string(code) == name
    assert hils.status_string(99) == "HILS_ERR_UNKNOWN"
    assert L.hils_version() >= 100


def _pf(**kw):
    hm = (ctypes.c_int32 * 32)(*[h // 4 for h in range(32)])
    base = dict(dtype=1, B=1, Hq=32, Hkv=8, N=4096, d=128, S=64, W=512, K=16,
                head_map=ctypes.cast(hm, ctypes.c_void_p).value)
    fake = 1 << 40                               # never dereferenced
    ptrs = dict(Q=fake, Kc=fake + 4096, V=fake + 8192, Klm=fake + 12288,
                bias=fake + 16384, O=fake + 20480, idx=fake + 24576,
                workspace=fake + 28672, workspace_bytes=1 << 40)
    base.update(ptrs)
    base.update(kw)
    a = hils.PrefillArgs()
    for k, v in base.items():
        setattr(a, k, v)
    return a, hm


def _ws(L, a):
    n = ctypes.c_size_t(0)
    rc = L.hils_prefill_workspace_size(ctypes.byref(a), ctypes.byref(n))
    return rc, n.value


def test_workspace_size_valid(L):
    a, hm = _pf()
    rc, n = _ws(L, a)
    assert rc == 0 and n >= 4 * 32 * 4096 * 16     # s^ of selected chunks
    a2, hm2 = _pf(sel_score=1 << 41)
    rc2, n2 = _ws(L, a2)
    assert rc2 == 0 and n2 < n


@pytest.mark.parametrize("field,value,code", [
    ("dtype", 7, 1), ("B", 0, 1), ("Hq", 0, 1), ("N", 0, 1), ("S", 0, 1),
    ("W", 0, 1), ("K", 0, 1), ("K", 65, 2), ("Hkv", 5, 1), ("d", 256, 2),
    ("d", 12, 2), ("head_map", 0, 1),
])
def test_workspace_size_rejects(L, field, value, code):
    a, hm = _pf(**{field: value})
    rc, _ = _ws(L, a)
    assert rc == code, (field, value, hils.STATUS.get(rc))


def test_bad_head_map_rejected(L):
    hm = (ctypes.c_int32 * 32)(*([0] * 5 + [h // 4 for h in range(5, 32)]))
    a, _ = _pf(head_map=ctypes.cast(hm, ctypes.c_void_p).value)
    rc, _ = _ws(L, a)
    assert rc == 1
    hm2 = (ctypes.c_int32 * 32)(*([9] + [h // 4 for h in range(1, 32)]))
    a2, _ = _pf(head_map=ctypes.cast(hm2, ctypes.c_void_p).value)
    assert _ws(L, a2)[0] == 1


@pytest.mark.parametrize("field", ["Q", "Kc", "V", "O", "idx", "bias", "Klm"])
def test_fwd_prefill_rejects_null(L, field):
    a, hm = _pf(**{field: 0})
    assert L.hils_fwd_prefill(ctypes.byref(a), None) == 1


@pytest.mark.parametrize("field", ["Q", "Kc", "V", "O", "idx", "Klm",
                                   "workspace"])
def test_fwd_prefill_rejects_misaligned(L, field):
    a, hm = _pf()
    setattr(a, field, getattr(a, field) + 8)
    assert L.hils_fwd_prefill(ctypes.byref(a), None) == 3


def test_fwd_prefill_rejects_small_workspace(L):
    a, hm = _pf(workspace_bytes=1024)
    assert L.hils_fwd_prefill(ctypes.byref(a), None) == 4


def test_fwd_prefill_null_args(L):
    assert L.hils_fwd_prefill(None, None) == 1
    n = ctypes.c_size_t(0)
    assert L.hils_prefill_workspace_size(None, ctypes.byref(n)) == 1
    a, hm = _pf()
    assert L.hils_prefill_workspace_size(ctypes.byref(a), None) == 1


def _df(**kw):
    hm = (ctypes.c_int32 * 32)(*[h // 4 for h in range(32)])
    fake = 1 << 40
    base = dict(dtype=1, B=8, Hq=32, Hkv=8, Lmax=8192, d=128, S=64, W=512,
                K=32, head_map=ctypes.cast(hm, ctypes.c_void_p).value,
                Q=fake, Kc=fake + 4096, V=fake + 8192, Klm=fake + 12288,
                bias=fake + 16384, cache_len=fake + 20480, O=fake + 24576,
                idx=fake + 28672, workspace=fake + 32768,
                workspace_bytes=1 << 40)
    base.update(kw)
    a = hils.DecodeArgs()
    for k, v in base.items():
        setattr(a, k, v)
    return a, hm


def test_decode_validation(L):
    a, hm = _df()
    n = ctypes.c_size_t(0)
    assert L.hils_decode_workspace_size(ctypes.byref(a), ctypes.byref(n)) == 0
    assert n.value > 0
    a, hm = _df(cache_len=0)
    assert L.hils_fwd_decode(ctypes.byref(a), None) == 1
    a, hm = _df(Q=(1 << 40) + 4)
    assert L.hils_fwd_decode(ctypes.byref(a), None) == 3
    a, hm = _df(workspace_bytes=16)
    assert L.hils_fwd_decode(ctypes.byref(a), None) == 4
    a, hm = _df(Lmax=0)
    assert L.hils_fwd_decode(ctypes.byref(a), None) == 1


def test_binding_refuses_cpu_tensors(L):
    import torch
    Q = torch.zeros(1, 1, 8, 64)
    with pytest.raises(ValueError):
        hils.fwd_prefill(Q, Q, Q, Q[:, :, :1], torch.zeros(1, 1, 1), [0], 8,
                         8, 1)


def _lm_args(**kw):
    fake = 1 << 40                       # never dereferenced: refused first
    a = dict(dtype=hils.BF16, B=1, Hkv=2, N=1024, d=128, S=64, Kc=fake,
             Qlm=fake + 4096, shared_query=0, Klm=fake + 8192,
             bias=fake + 12288)
    a.update(kw)
    return hils.LandmarkArgs(**a)


@pytest.mark.parametrize("kw,code", [
    (dict(d=96), 2), (dict(S=48), 2), (dict(S=512), 2),
    (dict(N=32), 1), (dict(B=0), 1), (dict(dtype=7), 1),
    (dict(shared_query=2), 1), (dict(Kc=None), 1), (dict(bias=None), 1),
    (dict(Kc=(1 << 40) + 8), 3), (dict(Klm=(1 << 40) + 4), 3),
])
def test_build_landmarks_rejects_before_launch(L, kw, code):
    assert L.hils_build_landmarks(ctypes.byref(_lm_args(**kw)), None) == code


def test_build_landmarks_null_args(L):
    assert L.hils_build_landmarks(None, None) == 1


@pytest.mark.parametrize("args,code", [
    ((1, 2, 100, 16, 50, 1), 1), ((1, 2, 100, 65, 50, 16), 1),
    ((1, 2, 100, 16, 0, 16), 1), ((0, 2, 100, 16, 50, 16), 1),
    ((1, 2, 100, 16, 50, 129), 1),
])
def test_chunk_overlap_rejects_before_launch(L, args, code):
    fake = 1 << 40
    assert L.hils_chunk_overlap(fake, *args, fake, fake, fake, None) == code


def test_chunk_overlap_rejects_null(L):
    fake = 1 << 40
    assert L.hils_chunk_overlap(None, 1, 2, 100, 16, 50, 16, fake, fake,
                                fake, None) == 1
    assert L.hils_chunk_overlap(fake, 1, 2, 100, 16, 50, 16, fake, None,
                                fake, None) == 1


def _paged(**kw):
    fake = 1 << 40
    base = hils.DecodeArgs(hils.BF16, 2, 8, 2, 1024, 128, 64, 128, 8,
                           None, fake, None, fake, fake, fake, fake, fake,
                           fake, fake, None, fake, 1 << 30, None)
    a = dict(base=base, block_table=fake, n_pages=40)
    a.update(kw)
    return hils.DecodePagedArgs(**a)


def test_decode_paged_validation(L):
    hm = (ctypes.c_int32 * 8)(*[h // 4 for h in range(8)])
    a = _paged()
    a.base.head_map = ctypes.cast(hm, ctypes.c_void_p)
    n = ctypes.c_size_t(0)
    # without a CUDA driver (CPU-only host) the HBM kernels report
    # themselves unavailable: HILS_ERR_UNSUPPORTED; with one, a size
    rc = L.hils_decode_paged_workspace_size(ctypes.byref(a), ctypes.byref(n))
    assert rc in (0, 2)
    assert rc == 2 or n.value > 0
    for kw, code in [(dict(block_table=None), 1), (dict(n_pages=0), 1)]:
        b = _paged(**kw)
        b.base.head_map = ctypes.cast(hm, ctypes.c_void_p)
        assert L.hils_fwd_decode_paged(ctypes.byref(b), None) == code
    c = _paged()
    c.base.head_map = ctypes.cast(hm, ctypes.c_void_p)
    c.base.Lmax = 1000                    # not a multiple of S
    assert L.hils_fwd_decode_paged(ctypes.byref(c), None) == 1
    d = _paged()
    d.base.head_map = ctypes.cast(hm, ctypes.c_void_p)
    d.base.dtype = hils.F32               # no f32 paged kernels
    assert L.hils_fwd_decode_paged(ctypes.byref(d), None) == 2
    assert L.hils_fwd_decode_paged(None, None) == 1


def _multi(**kw):
    fake = 1 << 40
    base = hils.DecodeArgs(hils.BF16, 2, 8, 2, 1024, 128, 64, 128, 8,
                           None, fake, None, fake, fake, fake, fake, fake,
                           fake, fake, None, fake, 1 << 30, None)
    a = dict(base=base, T=4, block_table=None, n_pages=0)
    a.update(kw)
    return hils.DecodeMultiArgs(**a)


def test_decode_multi_validation(L):
    """Multi-token records are checked on the host before any launch (only
    records that fail a check are passed to the compute entry point)."""
    hm = (ctypes.c_int32 * 8)(*[h // 4 for h in range(8)])
    a = _multi()
    a.base.head_map = ctypes.cast(hm, ctypes.c_void_p)
    n = ctypes.c_size_t(0)
    rc = L.hils_decode_multi_workspace_size(ctypes.byref(a), ctypes.byref(n))
    assert rc in (0, 2)                   # 2 without a CUDA driver
    assert rc == 2 or n.value > 0
    fake = 1 << 40
    for kw, code in [(dict(T=0), 1), (dict(T=2000), 1), (dict(T=9), 2),
                     (dict(block_table=fake, n_pages=0), 1)]:
        b = _multi(**kw)
        b.base.head_map = ctypes.cast(hm, ctypes.c_void_p)
        assert L.hils_fwd_decode_multi(ctypes.byref(b), None) == code, kw
    d = _multi()
    d.base.head_map = ctypes.cast(hm, ctypes.c_void_p)
    d.base.dtype = hils.F32               # no f32 multi-token kernels
    assert L.hils_fwd_decode_multi(ctypes.byref(d), None) == 2
    assert L.hils_fwd_decode_multi(None, None) == 1


def _bwd(**kw):
    fake = 1 << 40
    hm = (ctypes.c_int32 * 8)(*[h // 4 for h in range(8)])
    a = dict(dtype=hils.BF16, B=1, Hq=8, Hkv=2, N=1024, d=128, S=64, W=128,
             K=8, head_map=ctypes.cast(hm, ctypes.c_void_p).value, Q=fake,
             Qs=None, Kc=fake, V=fake, Klm=fake, bias=fake, dO=fake, idx=fake,
             dQ=fake, dQs=None, dK=fake, dV=fake, dKlm=fake, dbias=fake,
             workspace=fake, workspace_bytes=1 << 40)
    a.update(kw)
    return hils.BackwardArgs(**a), hm


def test_backward_validation(L):
    """Backward records are checked on the host before any launch (only
    failing records reach the compute entry point)."""
    a, hm = _bwd()
    n = ctypes.c_size_t(0)
    assert L.hils_bwd_prefill_workspace_size(ctypes.byref(a), ctypes.byref(n)) == 0
    # per (row, head) L, D and per (row, head, slot) four floats; with the
    # tensor-core key side (a CUDA driver present) also the inverse index
    # (4 segments x 16 chunks + 1 offsets and N * K entries per kv group) and
    # the work units: an upper bound of 16 blocks + (pairs / 64 + 16) / ub
    # + 1 units of ub batches (pairs / 64 / 592, within [8, 256]), each with
    # room for partial dV, dK, dk', db'
    r256 = lambda x: (x + 255) // 256 * 256
    base = r256(4 * 8 * 1024 * 2) + r256(4 * 8 * 1024 * 8 * 4)
    pairs = 4 * (2 * 1024 * 8 + 16 * (128 + 128 - 1))
    ub = min(256, max(8, pairs // 64 // 592))
    units = 16 + (pairs // 64 + 16) // ub + 1
    tc = (r256(4 * 2 * (4 * 16 + 1)) + r256(4 * 2 * 1024 * 8) + r256(8 * units) +
          r256(4 * (2 * 16 + 1)) + r256(4 * units * (2 * 128 * 128 + 2 * 128 + 4)))
    assert n.value in (base, base + tc)
    fake = 1 << 40
    for kw, code in [(dict(S=32), 2), (dict(d=96), 2), (dict(K=65), 2),
                     (dict(dQ=None), 1), (dict(Qs=fake), 1),
                     (dict(workspace_bytes=16), 4), (dict(dK=fake + 8), 3),
                     (dict(Hkv=3), 1), (dict(dtype=5), 1)]:
        b, hm2 = _bwd(**kw)
        assert L.hils_bwd_prefill(ctypes.byref(b), None) == code, kw
    assert L.hils_bwd_prefill(None, None) == 1
