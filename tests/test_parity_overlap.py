"""GPU chunk-overlap counts (hils_chunk_overlap) against the oracle, bit
for bit, on selections made by the prefill select stage; and the MHA
setting of the pages' 345M model (G = 1, d = 64, S = 64, K = 32, W = 512)
through the whole prefill, with its overlap metric."""
import numpy as np
import pytest
import torch

import chunk_sparse_long_landmark_b200 as hils
import synth
from oracle import overlap as ov
from tests import parity

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M", [2, 16, 32, 100])
def test_overlap_counts_match_oracle(M, cuda_device):
    sh = synth.Shape("bf16", 2, 8, 2, 128, 6000, 64, 256, 16, "needles",
                     n_needles=4)
    inp = synth.make_prefill(sh, seed=31, device=cuda_device)
    _, idx = hils.fwd_prefill(inp["Q"], inp["K"], inp["V"], inp["Klm"],
                              inp["bias"], inp["head_map"], sh.S, sh.W, sh.K,
                              stage="select")
    got = hils.chunk_overlap(idx, sh.N // sh.S, M)
    torch.cuda.synchronize()
    want = ov.block_counts(idx.cpu().numpy(), M)
    for g, w in zip(got, want):
        np.testing.assert_array_equal(g.cpu().numpy(), w)


def test_overlap_of_identical_and_padded_rows(cuda_device):
    idx = torch.full((1, 1, 70, 4), -1, dtype=torch.int32, device=cuda_device)
    idx[0, 0, 10:] = torch.tensor([3, 8, 40, 41], dtype=torch.int32)
    got = [t.cpu().numpy() for t in hils.chunk_overlap(idx, 64, 16)]
    want = ov.block_counts(idx.cpu().numpy(), 16)
    for g, w in zip(got, want):
        np.testing.assert_array_equal(g, w)


def test_mha_345m_setting_prefill_and_overlap(cuda_device):
    """G = 1 (every query head its own kv head), d = 64, S = 64, K = 32,
    W = 512: the prefill matches the oracle, and adjacent queries share most
    of their chunks (the pages report high overlap for this setting)."""
    sh = synth.Shape("bf16", 1, 4, 4, 64, 8192, 64, 512, 32)
    inp = synth.make_prefill(sh, seed=32, device=cuda_device)
    sel = torch.empty(sh.B, sh.Hq, sh.N, sh.K, dtype=torch.float32,
                      device=cuda_device)
    O, idx = hils.fwd_prefill(inp["Q"], inp["K"], inp["V"], inp["Klm"],
                              inp["bias"], inp["head_map"], sh.S, sh.W, sh.K,
                              sel_score=sel)
    torch.cuda.synchronize()
    parity.check_prefill(inp, O, idx, positions=parity.sample_positions(sh),
                         sel_gpu=sel)
    M = 16
    n_sel, n_union, _ = hils.chunk_overlap(idx, sh.N // sh.S, M)
    o = ov.overlap(n_sel.cpu().numpy(), n_union.cpu().numpy(), M, sh.K)
    assert np.isfinite(o).sum() > 0 and np.nanmean(o) > 0.5
