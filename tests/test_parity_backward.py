"""GPU parity of hils_bwd_prefill (through the C ABI) against the fp64
backward oracle, on the selection the GPU forward made.

Tolerances, relative to the largest entry of each gradient:
- f32 arithmetic throughout (f32 inputs; dQs, dKlm, dbias for bf16 inputs):
  the GPU gets the same inputs as the oracle and differs only by f32
  rounding in sums of at most a few thousand terms, ~n * 2^-24 < 2e-4.
- dQ, dK, dV for bf16 inputs: the tensor-core kernels round the weights
  p_j and ds_j to bf16 before the products (relative error <= 2^-9 per
  term, independent across terms), so a sum's error is about 2^-9 times
  the root-sum-square of its terms, which for these random inputs is at
  most the sum's own scale; 2^-8 = 3.9e-3 leaves a factor of two."""
import numpy as np
import pytest
import torch

import chunk_sparse_long_landmark_b200 as hils
import synth
from oracle.backward import hils_backward

pytestmark = pytest.mark.gpu

REL = 2e-4
REL_BF16_TC = 2.0 ** -8


def _run(sh, seed, dev):
    inp = synth.make_prefill(sh, seed=seed, device=dev)
    O, idx = hils.fwd_prefill(inp["Q"], inp["K"], inp["V"], inp["Klm"],
                              inp["bias"], inp["head_map"], sh.S, sh.W, sh.K,
                              Qs=inp["Qs"])
    g0 = torch.Generator(device="cpu").manual_seed(seed + 1)
    dO = torch.randn(inp["Q"].shape, generator=g0).to(inp["Q"].dtype).to(dev)
    gr = hils.bwd_prefill(inp["Q"], inp["K"], inp["V"], inp["Klm"],
                          inp["bias"], inp["head_map"], sh.S, sh.W, idx, dO,
                          Qs=inp["Qs"])
    torch.cuda.synchronize()
    return inp, idx, dO, gr


def _check(inp, idx, dO, gr, sh):
    ref = hils_backward(inp["Q"], inp["K"], inp["V"], inp["Klm"], inp["bias"],
                        inp["head_map"], sh.S, sh.W, idx, dO, Qs=inp["Qs"])
    for name in ("dQ", "dQs", "dK", "dV", "dKlm", "dbias"):
        if ref[name] is None:
            assert gr[name] is None
            continue
        got = gr[name].double().cpu().numpy()
        want = ref[name]
        if want.size == 0:                       # no complete chunk (N < S)
            continue
        err = np.abs(got - want).max() / max(1e-30, np.abs(want).max())
        tol = REL
        if sh.dtype == "bf16" and name in ("dQ", "dK", "dV"):
            tol = REL_BF16_TC
        assert err <= tol, f"{name}: rel err {err:.3e} (tol {tol:.1e})"


CASES = {
    "f32_g4_d64": synth.Shape("f32", 1, 4, 1, 64, 1024, 64, 128, 4),
    "bf16_g4_d128": synth.Shape("bf16", 1, 8, 2, 128, 2048, 64, 256, 8),
    "bf16_mha_d64_ragged": synth.Shape("bf16", 2, 2, 2, 64, 1000, 64, 192, 5),
    "f32_qcal": synth.Shape("f32", 1, 2, 1, 128, 768, 64, 128, 3, "qcal"),
    "bf16_needles": synth.Shape("bf16", 1, 4, 1, 128, 2048, 64, 256, 8,
                                "needles", n_needles=3),
    # 128-token chunks
    "bf16_S128_g4_d128_ragged": synth.Shape("bf16", 1, 8, 2, 128, 2500, 128,
                                            300, 6),
    "f32_S128_qcal_d64": synth.Shape("f32", 1, 4, 1, 64, 1300, 128, 200, 4,
                                     "qcal"),
    # bf16 query calibration: the key side gathers the scoring rows too
    "bf16_qcal_d128": synth.Shape("bf16", 1, 4, 1, 128, 1300, 64, 200, 6,
                                  "qcal"),
    "bf16_S128_qcal_d64": synth.Shape("bf16", 1, 4, 1, 64, 1400, 128, 256, 4,
                                      "qcal"),
    # G = 8: eight pairs per row in a batch of 64
    "bf16_g8_d128": synth.Shape("bf16", 1, 8, 1, 128, 1000, 64, 128, 5),
    # G = 3 (128 % G != 0): the query side runs on the CUDA cores and feeds
    # the tensor-core key side
    "bf16_g3_d64": synth.Shape("bf16", 1, 6, 2, 64, 1100, 64, 160, 5),
    # N < S: no complete chunk, the key side sees window rows only
    "bf16_no_chunks": synth.Shape("bf16", 1, 4, 1, 64, 50, 64, 16, 2),
    # a single selected chunk per row
    "bf16_k1": synth.Shape("bf16", 1, 4, 1, 64, 700, 64, 64, 1),
    # many key blocks, rows selecting a chunk spread over several batches
    "bf16_g4_d128_long": synth.Shape("bf16", 1, 4, 1, 128, 3000, 64, 128, 12),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_backward_matches_oracle(name, cuda_device):
    sh = CASES[name]
    inp, idx, dO, gr = _run(sh, 401, cuda_device)
    _check(inp, idx, dO, gr, sh)


def test_backward_deterministic(cuda_device):
    """No floating-point atomics: two calls give bitwise equal gradients."""
    sh = CASES["bf16_g4_d128"]
    inp, idx, dO, g1 = _run(sh, 402, cuda_device)
    g2 = hils.bwd_prefill(inp["Q"], inp["K"], inp["V"], inp["Klm"],
                          inp["bias"], inp["head_map"], sh.S, sh.W, idx, dO)
    torch.cuda.synchronize()
    for k in ("dQ", "dK", "dV", "dKlm", "dbias"):
        assert torch.equal(g1[k], g2[k]), k


def test_backward_constant_values(cuda_device):
    """V constant over the tokens: the gradients of Q, K, k', b' vanish (up
    to f32 rounding of the softmax weights' sum)."""
    sh = synth.Shape("f32", 1, 4, 1, 64, 1024, 64, 128, 4)
    inp = synth.make_prefill(sh, seed=403, device=cuda_device)
    row = torch.linspace(-1, 1, sh.d, device=cuda_device)
    inp["V"] = row.expand_as(inp["V"]).contiguous()
    O, idx = hils.fwd_prefill(inp["Q"], inp["K"], inp["V"], inp["Klm"],
                              inp["bias"], inp["head_map"], sh.S, sh.W, sh.K)
    dO = torch.randn_like(inp["Q"])
    gr = hils.bwd_prefill(inp["Q"], inp["K"], inp["V"], inp["Klm"],
                          inp["bias"], inp["head_map"], sh.S, sh.W, idx, dO)
    torch.cuda.synchronize()
    for k in ("dQ", "dK", "dKlm", "dbias"):
        assert gr[k].abs().max().item() < 1e-4, k
