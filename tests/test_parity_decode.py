"""GPU parity of hils_fwd_decode (through the C ABI) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import chunk_sparse_long_landmark_b200 as hils
import synth
from tests import parity

pytestmark = pytest.mark.gpu


def run_decode(inp, status=None):
    sh = inp["shape"]
    O, idx = hils.fwd_decode(inp["Q"], inp["K"], inp["V"], inp["Klm"],
                             inp["bias"], inp["cache_len"], inp["head_map"],
                             sh.S, sh.W, sh.K, status=status)
    torch.cuda.synchronize()
    return O, idx


CASES = {
    "f32_ragged": (synth.Shape("f32", 3, 4, 2, 64, 2048, 64, 128, 5), [2048, 1000, 70]),
    "bf16_ragged": (synth.Shape("bf16", 4, 32, 8, 128, 16384, 64, 512, 32), [16384, 9999, 600, 1]),
    "bf16_short": (synth.Shape("bf16", 2, 8, 2, 128, 4096, 64, 512, 32), [513, 575]),
    "bf16_d64_S128": (synth.Shape("bf16", 2, 8, 1, 64, 8192, 128, 300, 16), [8192, 5000]),
    "bf16_k64_g16": (synth.Shape("bf16", 1, 16, 1, 128, 32768, 64, 512, 64), [32768]),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_decode_small(name, cuda_device):
    sh, lens = CASES[name]
    inp = synth.make_decode(sh, seed=202, device=cuda_device, cache_len=lens)
    O, idx = run_decode(inp)
    parity.check_decode(inp, O, idx)


def test_decode_peaked(cuda_device):
    """Query scaled by 4 (exact in bf16): near one-hot attention, where the
    rounding of the weights to bf16 matters most for the output error."""
    sh = synth.Shape("bf16", 2, 32, 8, 128, 16384, 64, 512, 32)
    inp = synth.make_decode(sh, seed=203, device=cuda_device,
                            cache_len=[16384, 7001])
    inp = dict(inp, Q=inp["Q"] * 4)
    O, idx = run_decode(inp)
    parity.check_decode(inp, O, idx)


def test_decode_config4_full(cuda_device):
    """Batch of 8 sequences with 512K-token caches, every sequence checked."""
    sh = synth.DECODE_CONFIGS[4]
    inp = synth.make_decode(sh, seed=synth.seed_for(4), device=cuda_device)
    O, idx = run_decode(inp)
    for b in range(sh.B):                       # oracle one sequence at a time
        sub = dict(inp, Q=inp["Q"][b:b + 1], K=inp["K"][b:b + 1],
                   V=inp["V"][b:b + 1], Klm=inp["Klm"][b:b + 1],
                   bias=inp["bias"][b:b + 1],
                   cache_len=inp["cache_len"][b:b + 1],
                   shape=sh.with_(B=1))
        parity.check_decode(sub, O[b:b + 1], idx[b:b + 1])


def test_decode_bad_length_reported(cuda_device):
    """A cache_len outside [1, Lmax] is reported in the status word."""
    sh = synth.Shape("bf16", 2, 8, 2, 128, 2048, 64, 256, 8)
    inp = synth.make_decode(sh, seed=3, device=cuda_device,
                            cache_len=[2048, 4096])
    st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    O, idx = run_decode(inp, status=st)
    assert int(st.item()) == 7          # HILS_ERR_DEVICE_BAD_LENGTH
    # the valid sequence is still computed correctly
    sub = dict(inp, Q=inp["Q"][:1], K=inp["K"][:1], V=inp["V"][:1],
               Klm=inp["Klm"][:1], bias=inp["bias"][:1],
               cache_len=inp["cache_len"][:1], shape=sh.with_(B=1))
    parity.check_decode(sub, O[:1], idx[:1])


def test_decode_deterministic_and_graph(cuda_device):
    sh = synth.Shape("bf16", 4, 32, 8, 128, 65536, 64, 512, 32)
    inp = synth.make_decode(sh, seed=9, device=cuda_device)
    O1, i1 = run_decode(inp)
    O = torch.empty_like(O1)
    idx = torch.empty_like(i1)
    ws = torch.empty(hils.decode_workspace_size(
        inp["Q"], inp["K"], inp["V"], inp["Klm"], inp["bias"],
        inp["cache_len"], inp["head_map"], sh.S, sh.W, sh.K),
        dtype=torch.uint8, device=cuda_device)
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        hils.fwd_decode(inp["Q"], inp["K"], inp["V"], inp["Klm"],
                        inp["bias"], inp["cache_len"], inp["head_map"], sh.S,
                        sh.W, sh.K, out=O, idx=idx, workspace=ws, stream=s)
    s.synchronize()
    with torch.cuda.graph(g, stream=s):
        hils.fwd_decode(inp["Q"], inp["K"], inp["V"], inp["Klm"],
                        inp["bias"], inp["cache_len"], inp["head_map"], sh.S,
                        sh.W, sh.K, out=O, idx=idx, workspace=ws, stream=s)
    O.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(O, O1) and torch.equal(idx, i1)
    del g


@pytest.mark.parametrize("every", [80, 2])
def test_decode_exact_score_ties_take_lower_chunks(every, cuda_device):
    """Identical landmark keys; b' = 0 on chunks c % every == 0, -1 elsewhere.
    The tied chunks share one group score exactly, so the tie rule alone
    decides: idx must be the K lowest tied chunks of C_i, bit for bit.
    every=80 gives ~100 tied chunks (a short candidate list); every=2 ties
    half of all candidates (too many for a short list)."""
    sh = synth.Shape("bf16", 2, 32, 8, 128, 16384, 64, 512, 32)
    lens = [16384, 9000]
    inp = synth.make_decode(sh, seed=211, device=cuda_device, cache_len=lens)
    nC = sh.N // sh.S
    klm = inp["Klm"][:, :, :1, :].expand(-1, -1, nC, -1).contiguous()
    bias = torch.full((sh.B, sh.Hkv, nC), -1.0, dtype=torch.float32,
                      device=cuda_device)
    bias[:, :, 0::every] = 0.0
    inp = dict(inp, Klm=klm, bias=bias)
    O, idx = run_decode(inp)
    got = idx.cpu().numpy()
    for b, L in enumerate(lens):
        nc = max((L - 1 - sh.W + 1) // sh.S, 0)
        c = np.arange(nc)
        order = np.concatenate([c[c % every == 0], c[c % every != 0]])[:sh.K]
        want = np.sort(order)
        for g in range(sh.Hkv):
            np.testing.assert_array_equal(got[b, g], want)
    parity.check_decode(inp, O, idx)


def _to_pages(inp, sh, seed, spare=5):
    """Scatter the contiguous caches into a shuffled page pool (page = one
    chunk of every kv head) with a random block table, plus unused pages."""
    B, Hkv, L, d = inp["K"].shape
    npg = L // sh.S
    P = B * npg + spare
    g = torch.Generator(device="cpu").manual_seed(seed)
    perm = torch.randperm(P, generator=g)[:B * npg].view(B, npg)
    dev = inp["K"].device
    bt = perm.to(torch.int32).to(dev).contiguous()
    pools = []
    for name in ("K", "V"):
        pool = torch.randn(P, Hkv, sh.S, d, device=dev).to(inp[name].dtype)
        x = inp[name].view(B, Hkv, npg, sh.S, d).permute(0, 2, 1, 3, 4)
        pool[perm.reshape(-1).to(dev)] = x.reshape(B * npg, Hkv, sh.S, d)
        pools.append(pool.contiguous())
    return pools[0], pools[1], bt


@pytest.mark.parametrize("name", ["bf16_ragged", "bf16_d64_S128", "bf16_short"])
def test_decode_paged_equals_contiguous(name, cuda_device):
    """Same kernels, addressed through a block table: the paged step gives
    bit-identical O and idx to the contiguous one, and matches the oracle."""
    sh, lens = CASES[name]
    inp = synth.make_decode(sh, seed=205, device=cuda_device, cache_len=lens)
    O_ref, idx_ref = run_decode(inp)
    Kp, Vp, bt = _to_pages(inp, sh, seed=7)
    O, idx = hils.fwd_decode_paged(inp["Q"], Kp, Vp, inp["Klm"], inp["bias"],
                                   inp["cache_len"], bt, inp["head_map"],
                                   sh.S, sh.W, sh.K)
    torch.cuda.synchronize()
    assert torch.equal(idx, idx_ref)
    assert torch.equal(O, O_ref)
    parity.check_decode(inp, O, idx)


def test_decode_paged_bad_page_reported(cuda_device):
    """A page index outside the pool is reported in the status word (and
    read as zeros): no fault."""
    sh, lens = CASES["bf16_short"]
    inp = synth.make_decode(sh, seed=206, device=cuda_device, cache_len=lens)
    Kp, Vp, bt = _to_pages(inp, sh, seed=8)
    bt[0, (lens[0] - 1) // sh.S] = Kp.shape[0] + 3      # the query's own page
    st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    hils.fwd_decode_paged(inp["Q"], Kp, Vp, inp["Klm"], inp["bias"],
                          inp["cache_len"], bt, inp["head_map"], sh.S, sh.W,
                          sh.K, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 7          # HILS_ERR_DEVICE_BAD_LENGTH


# ---------------------------------------------------------------- multi-token
def _multi_inputs(name, T, seed, cuda_device):
    """Decode inputs plus T query tokens per sequence, token-major [B,T,Hq,d].
    cache_len counts the T new tokens (already in the cache)."""
    sh, lens = CASES[name]
    lens = [max(l, T) for l in lens]
    inp = synth.make_decode(sh, seed=seed, device=cuda_device, cache_len=lens)
    g = torch.Generator(device="cpu").manual_seed(seed + 17)
    Qm = torch.randn(sh.B, T, sh.Hq, sh.d, generator=g).to(inp["Q"].dtype)
    return sh, lens, inp, Qm.to(cuda_device).contiguous()


def _token_view(inp, sh, lens, Qm, T, t):
    """The plain decode record of token t: its query, the cache length that
    puts it at position cache_len - T + t."""
    cl = torch.tensor([l - (T - 1 - t) for l in lens], dtype=torch.int32,
                      device=inp["cache_len"].device)
    return dict(inp, Q=Qm[:, t].contiguous(), cache_len=cl)


def run_multi(inp, sh, Qm, block_table=None, K=None, V=None, status=None):
    O, idx = hils.fwd_decode_multi(Qm, inp["K"] if K is None else K,
                                   inp["V"] if V is None else V, inp["Klm"],
                                   inp["bias"], inp["cache_len"],
                                   inp["head_map"], sh.S, sh.W, sh.K,
                                   block_table=block_table, status=status)
    torch.cuda.synchronize()
    return O, idx


@pytest.mark.parametrize("name,T", [("bf16_ragged", 2), ("bf16_ragged", 4),
                                    ("bf16_short", 3), ("bf16_d64_S128", 4),
                                    ("bf16_ragged", 8)])
def test_decode_multi_matches_oracle_per_token(name, T, cuda_device):
    """Token t of a T-token step is the decode of a query at position
    cache_len - T + t: idx bit-exact (up to near ties) and O within the bf16
    bound against the oracle, and idx equal to the single-token step's."""
    sh, lens, inp, Qm = _multi_inputs(name, T, 301 + T, cuda_device)
    O, idx = run_multi(inp, sh, Qm)
    for t in range(T):
        sub = _token_view(inp, sh, lens, Qm, T, t)
        parity.check_decode(sub, O[:, t], idx[:, t])
        _, idx1 = run_decode(sub)
        assert torch.equal(idx[:, t], idx1), f"token {t}: idx differs from single-token decode"


def test_decode_multi_T1_equals_decode(cuda_device):
    """T = 1 runs exactly the plain decode step: bit-identical O and idx."""
    sh, lens, inp, Qm = _multi_inputs("bf16_ragged", 1, 311, cuda_device)
    O, idx = run_multi(inp, sh, Qm)
    O1, idx1 = run_decode(dict(inp, Q=Qm[:, 0].contiguous()))
    assert torch.equal(idx[:, 0], idx1)
    assert torch.equal(O[:, 0], O1)


def test_decode_multi_paged_equals_contiguous(cuda_device):
    """The multi-token step over a page pool gives bit-identical results."""
    T = 4
    sh, lens, inp, Qm = _multi_inputs("bf16_ragged", T, 321, cuda_device)
    O_ref, idx_ref = run_multi(inp, sh, Qm)
    Kp, Vp, bt = _to_pages(inp, sh, seed=9)
    O, idx = run_multi(inp, sh, Qm, block_table=bt, K=Kp, V=Vp)
    assert torch.equal(idx, idx_ref)
    assert torch.equal(O, O_ref)


def test_decode_multi_short_cache_reported(cuda_device):
    """cache_len below T is reported in the status word; other sequences are
    still computed."""
    T = 4
    sh, lens, inp, Qm = _multi_inputs("bf16_short", T, 331, cuda_device)
    inp = dict(inp, cache_len=torch.tensor([lens[0], 2], dtype=torch.int32,
                                           device=cuda_device))
    st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    O, idx = run_multi(inp, sh, Qm, status=st)
    assert int(st.item()) == 7          # HILS_ERR_DEVICE_BAD_LENGTH
    sub = _token_view(dict(inp, Q=inp["Q"][:1], K=inp["K"][:1], V=inp["V"][:1],
                           Klm=inp["Klm"][:1], bias=inp["bias"][:1],
                           shape=sh.with_(B=1)),
                      sh, lens[:1], Qm[:1], T, T - 1)
    parity.check_decode(sub, O[:1, T - 1], idx[:1, T - 1])
