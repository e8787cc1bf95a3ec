"""The allocation-free decode entry point, hils_fwd_decode_noalloc.

It is meant for callers that cannot allocate device memory when they call
(memory reserved up front by a serving loop, latency paths that cannot take
cudaMalloc's implicit synchronisation, hosts that cannot own a workspace).
This file checks, through the C ABI, that two consecutive calls give the
same result as hils_fwd_decode (the entry point with a caller workspace),
under the tolerance the other parity tests use, and that a shape larger than
the fixed scratch is refused. Kept in its own file, collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

import chunk_sparse_long_landmark_b200 as hils
import oracle
import synth
from tests import parity

pytestmark = pytest.mark.gpu


def _noalloc(inp, O, idx):
    sh = inp["shape"]
    a, hm = hils._decode_struct(inp["Q"], inp["K"], inp["V"], inp["Klm"],
                                inp["bias"], inp["cache_len"],
                                inp["head_map"], sh.S, sh.W, sh.K, O=O,
                                idx=idx)
    s = torch.cuda.current_stream()
    return hils.lib().hils_fwd_decode_noalloc(ctypes.byref(a),
                                              ctypes.c_void_p(s.cuda_stream))


@pytest.mark.parametrize("dtype,lens", [
    ("bf16", [65536, 40000, 700, 1]),
    ("f32", [8192, 5000, 513, 64]),
])
def test_noalloc_matches_workspace_entry_point(dtype, lens, cuda_device):
    L = max(lens)
    sh = synth.Shape(dtype, len(lens), 32 if dtype == "bf16" else 8,
                     8 if dtype == "bf16" else 2, 128 if dtype == "bf16" else 64,
                     L, 64, 512, 32 if dtype == "bf16" else 8)
    inp = synth.make_decode(sh, seed=404, device=cuda_device, cache_len=lens)
    O_ref, idx_ref = hils.fwd_decode(inp["Q"], inp["K"], inp["V"], inp["Klm"],
                                     inp["bias"], inp["cache_len"],
                                     inp["head_map"], sh.S, sh.W, sh.K)
    torch.cuda.synchronize()
    gaps = oracle.decode(inp)
    tie = parity.near_tie(gaps["gap"], gaps["akth"])
    for call in range(2):
        O = torch.full_like(O_ref, float("nan"))
        idx = torch.full_like(idx_ref, -7)
        rc = _noalloc(inp, O, idx)
        assert rc == 0, hils.STATUS.get(rc, rc)
        torch.cuda.synchronize()
        a = idx.cpu().numpy()
        b = idx_ref.cpu().numpy()
        differ = (a != b).any(-1)
        assert not (differ & ~tie).any(), f"call {call}: idx differs"
        rows = np.ones(O.shape[:2], dtype=bool)
        for bb, g in np.argwhere(differ):
            for h in oracle.group_heads(inp["head_map"], g):
                rows[bb, h] = False
        err = (O.double() - O_ref.double()).abs().cpu().numpy()[rows]
        if dtype == "f32":
            ref = O_ref.double().abs().max().item()
            assert err.max() / ref <= parity.F32_REL, f"call {call}"
        else:
            assert err.max() <= parity.BF16_ABS, f"call {call}: {err.max()}"


def test_noalloc_refuses_shape_beyond_scratch(cuda_device):
    # 64M-token caches: one scoring block alone needs (G+1) * ~1M floats
    # (about 71 MB with G = 16), far beyond the fixed 8 MiB scratch. The
    # pointers are never dereferenced: the shape is refused on the host.
    sh = synth.Shape("bf16", 64, 128, 8, 64, 1 << 26, 64, 512, 64)
    fake = 1 << 40
    hm = (ctypes.c_int32 * sh.Hq)(*[h // 16 for h in range(sh.Hq)])
    a = hils.DecodeArgs(1, sh.B, sh.Hq, sh.Hkv, sh.N, sh.d, sh.S, sh.W, sh.K,
                        ctypes.cast(hm, ctypes.c_void_p), fake, None,
                        fake + 4096, fake + 8192, fake + 12288,
                        fake + 16384, fake + 20480, fake + 24576,
                        fake + 28672, None, None, 0, None)
    rc = hils.lib().hils_fwd_decode_noalloc(ctypes.byref(a), None)
    assert rc == 4          # HILS_ERR_WORKSPACE_TOO_SMALL, nothing enqueued
