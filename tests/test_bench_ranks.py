"""The multi-GPU plumbing of bench.py on CPU: two gloo ranks.

Each rank runs its own replica of the workload (the path shards by (batch,
kv head) and has no exchange), so what has to be right is the barrier, the
max over ranks of the timed duration, and the whole-job rate computed from
it. Here two processes stand in for two GPUs with different step times.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
                      RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    ctx = bench.RankContext("gloo", timeout_s=60)
    ctx.barrier()
    my_ms = 10.0 * (rank + 1)               # rank 1 is the slow one
    ms = ctx.max(my_ms)
    rate = ctx.whole_job_rate(1000, ms)
    ctx.barrier()
    ctx.close()
    out.put((rank, ctx.world, ms, rate))


def test_two_gloo_ranks_agree_on_max_time_and_whole_job_rate():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q))
             for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, w, ms, rate in res:
        assert w == world
        assert ms == pytest.approx(20.0)        # the slower rank's time
        # both ranks' units over the slowest rank's time
        assert rate == pytest.approx(world * 1000 / 20e-3)


def test_single_process_needs_no_process_group():
    import bench
    for k in ("RANK", "WORLD_SIZE"):
        os.environ.pop(k, None)
    ctx = bench.RankContext("gloo")
    assert ctx.world == 1 and ctx.rank == 0
    assert ctx.max(3.5) == 3.5
    assert ctx.whole_job_rate(500, 5.0) == pytest.approx(1e5)
    ctx.close()


def test_decode_multi_bytes_reduces_to_single_token():
    """The multi-token bytes model with T = 1 is the decode bytes model, and
    tokens that share every chunk add only their Q / O / idx bytes."""
    import numpy as np

    import bench
    import synth
    sh = synth.Shape("bf16", 2, 8, 2, 128, 8192, 64, 512, 4)
    cl = [8192, 5000]
    rng = np.random.default_rng(0)
    idx1 = np.full((2, 1, 2, 4), -1, dtype=np.int64)
    for b, L in enumerate(cl):
        nc = (L - 1 - sh.W + 1) // sh.S
        for g in range(2):
            idx1[b, 0, g] = np.sort(rng.choice(nc, 4, replace=False))
    assert bench.decode_multi_bytes(sh, cl, 1, idx1) == bench.decode_bytes(sh, cl)
    # two tokens (positions L-2, L-1) with the same selection: the chunks and
    # the landmark scan are shared; the window union reaches back to the
    # earlier token's window start; each token adds its Q / O / idx bytes
    idx2 = np.repeat(idx1, 2, axis=1)
    extra = bench.decode_multi_bytes(sh, cl, 2, idx2) - bench.decode_bytes(sh, cl)
    esz = 2
    want = 0
    for L in cl:
        w0 = lambda i: max((i - sh.W + 1) // sh.S * sh.S, 0)
        want += (w0(L - 1) - w0(L - 2)) * sh.Hkv * 2 * sh.d * esz
        want += 2 * sh.Hq * sh.d * esz + sh.Hkv * sh.K * 4
    assert extra == want
