"""GPU parity of hils_build_landmarks (Prop. 3.1 landmark summaries)
against the fp64 oracle, through the C ABI, plus the exactness identity at
full size on sampled chunks and an end-to-end prefill fed with the built
landmarks.

Tolerances: k' is rounded to the key dtype; bf16 rounding is at most 2^-9
relative, so |k'_gpu - k'_ref| <= 2^-8 |k'_ref| + 1e-5 per element (fp32
accumulation adds ~1e-6). f32 k' within 1e-5 of max|k'_ref| (the f32 bar of
the hot path). b' is an fp32 log-sum-exp minus an fp32 weighted mean of at
most 256 terms: within 5e-5 absolute.
"""
import numpy as np
import pytest
import torch

import chunk_sparse_long_landmark_b200 as hils
import oracle
import synth
from oracle import landmarks as olm
from tests import parity

pytestmark = pytest.mark.gpu


def _inputs(dtype, B, Hkv, N, d, S, shared, seed, dev, qscale=1.0):
    g = torch.Generator(device=dev).manual_seed(seed)
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    K = torch.randn(B, Hkv, N, d, generator=g, device=dev).to(dt)
    nC = N // S
    shape = (Hkv, d) if shared else (B, Hkv, nC, d)
    Q = (qscale * torch.randn(*shape, generator=g, device=dev)).to(dt)
    return K, Q


def _check(K, Q, S, klm, bias):
    ref_k, ref_b = olm.build_landmarks(K.double().cpu().numpy(),
                                       Q.double().cpu().numpy(), S)
    gk = klm.double().cpu().numpy()
    gb = bias.double().cpu().numpy()
    if K.dtype == torch.bfloat16:
        assert (np.abs(gk - ref_k) <= 2.0 ** -8 * np.abs(ref_k) + 1e-5).all()
    else:
        assert np.abs(gk - ref_k).max() <= 1e-5 * np.abs(ref_k).max()
    assert np.abs(gb - ref_b).max() <= 5e-5


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("d,S", [(128, 64), (64, 128), (128, 32), (64, 256)])
@pytest.mark.parametrize("shared", [False, True])
def test_landmarks_match_oracle(dtype, d, S, shared, cuda_device):
    K, Q = _inputs(dtype, 2, 3, 5 * S + 17, d, S, shared, 11, cuda_device,
                   qscale=2.0)
    klm, bias = hils.build_landmarks(K, Q, S)
    torch.cuda.synchronize()
    _check(K, Q, S, klm, bias)


def test_landmarks_peaked_and_uniform_chunks(cuda_device):
    """A chunk of equal keys (b' = log S) and a chunk with one dominant key
    aligned with its query (b' ~ 0)."""
    S, d = 64, 128
    K, Q = _inputs("bf16", 1, 1, 2 * S, d, S, False, 12, cuda_device)
    K[0, 0, :S] = K[0, 0, 5]
    u = torch.randn(d, device=cuda_device)
    u = 24.0 * u / u.norm()
    K[0, 0, S + 9] = u.to(K.dtype)
    Q[0, 0, 1] = u.to(K.dtype)
    klm, bias = hils.build_landmarks(K, Q, S)
    torch.cuda.synchronize()
    _check(K, Q, S, klm, bias)
    assert abs(bias[0, 0, 0].item() - np.log(S)) < 5e-5
    assert bias[0, 0, 1].item() < 1e-3


def test_landmarks_full_size_exact_at_landmark_query(cuda_device):
    """128K-token keys (the 128K prefill workload's K shape): b' in
    [0, log S] everywhere; on sampled chunks the surrogate at q = q' equals
    the exact chunk log-mass (fp64 from the same bf16 inputs)."""
    sh = synth.PREFILL_CONFIGS[3]
    K, Q = _inputs("bf16", sh.B, sh.Hkv, sh.N, sh.d, sh.S, False, 13,
                   cuda_device)
    klm, bias = hils.build_landmarks(K, Q, sh.S)
    torch.cuda.synchronize()
    assert bool((bias >= -5e-5).all()) and bool((bias <= np.log(sh.S) + 5e-5).all())
    rng = np.random.default_rng(3)
    nC = sh.N // sh.S
    for _ in range(64):
        g, c = int(rng.integers(sh.Hkv)), int(rng.integers(nC))
        kc = K[0, g, c * sh.S:(c + 1) * sh.S].double().cpu().numpy()
        q = Q[0, g, c].double().cpu().numpy()
        exact = olm.chunk_logmass(kc, q, 0, sh.S)
        sur = float(q @ klm[0, g, c].double().cpu().numpy()) / np.sqrt(sh.d) \
            + float(bias[0, g, c])
        # k' in bf16: q.k' moves by up to 2^-9 |q||k'| / sqrt(d)
        tol = 2.0 ** -9 * np.linalg.norm(q) * float(
            klm[0, g, c].double().norm()) / np.sqrt(sh.d) + 1e-4
        assert abs(sur - exact) <= tol


def test_prefill_with_built_landmarks(cuda_device):
    """The hot path fed with landmarks from the builder (q'_c ~ N(0,1)):
    HiLS prefill still matches the oracle run on the same inputs."""
    sh = synth.Shape("bf16", 1, 8, 2, 128, 4096, 64, 512, 16)
    inp = synth.make_prefill(sh, seed=21, device=cuda_device)
    _, Q = _inputs("bf16", 1, 2, 4096, 128, 64, False, 22, cuda_device)
    klm, bias = hils.build_landmarks(inp["K"], Q, 64)
    inp = dict(inp, Klm=klm, bias=bias)
    sel = torch.empty(sh.B, sh.Hq, sh.N, sh.K, dtype=torch.float32,
                      device=cuda_device)
    O, idx = hils.fwd_prefill(inp["Q"], inp["K"], inp["V"], klm, bias,
                              inp["head_map"], sh.S, sh.W, sh.K,
                              sel_score=sel)
    torch.cuda.synchronize()
    parity.check_prefill(inp, O, idx, sel_gpu=sel)
