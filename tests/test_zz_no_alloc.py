"""The allocation-free decode entry point, hils_fwd_decode_noalloc.

It is meant for callers that cannot allocate device memory when they call
(memory reserved up front by a serving loop, latency paths that cannot take
cudaMalloc's implicit synchronisation, hosts that cannot own a workspace).
This file checks, through the C ABI, that each of two consecutive calls
matches the fp64 oracle (idx exact outside near ties, O within the bf16 /
f32 bound) and gives the same result as hils_fwd_decode (the entry point with
a caller workspace), and that a shape larger than the fixed scratch is
refused. One case has more (sequence, kv head) units than scoring blocks fit
in the scratch, so the scoring grid is cut to what fits and its blocks loop
over the units. Kept in its own file, collected last.
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


SCRATCH_BYTES = 8 << 20        # the library's fixed scratch per device
SM_BLOCKS = 8                  # scoring blocks per SM the launch asks for

CASES = {
    "bf16_g4": (synth.Shape("bf16", 4, 32, 8, 128, 65536, 64, 512, 32),
                [65536, 40000, 700, 1]),
    "f32_g4": (synth.Shape("f32", 4, 8, 2, 64, 8192, 64, 512, 8),
               [8192, 5000, 513, 64]),
    # 64 (sequence, kv head) units; one scoring block needs (G+1) x 2040
    # floats (139 KB), so only 59 blocks fit in the scratch
    "bf16_g16_grid_cut": (synth.Shape("bf16", 8, 128, 8, 64, 131072, 64, 512,
                                      32),
                          [131072, 100000, 65536, 30000, 4096, 700, 64, 1]),
}


def _blocks_that_fit(sh):
    nc_max = max((sh.N - 1 - sh.W + 1) // sh.S, 1)
    per_block = 4 * (sh.G + 1) * nc_max
    sel = -(-4 * sh.B * sh.Hq * sh.K // 256) * 256     # sel_score not given
    return (SCRATCH_BYTES - sel) // per_block


@pytest.mark.parametrize("name", sorted(CASES))
def test_noalloc_matches_workspace_entry_point(name, cuda_device):
    sh, lens = CASES[name]
    dtype = sh.dtype
    if name.endswith("grid_cut"):
        units = sh.B * sh.Hkv
        assert _blocks_that_fit(sh) < min(units, SM_BLOCKS * torch.cuda.
                                          get_device_properties(0).
                                          multi_processor_count)
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
        parity.check_decode(inp, O, idx)            # against the oracle
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
