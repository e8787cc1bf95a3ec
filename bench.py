#!/usr/bin/env python
"""Benchmark of the HiLS attention forward path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl hils|reference] [--no-decode] [--no-cpu]

One step = one HiLS prefill forward (landmark scoring + group top-K +
gathered intra-chunk/window attention + chunk-softmax fusion) over the
workload's whole synthetic input, through the C ABI (hils_prefill_select then
hils_prefill_attend, exactly what hils_fwd_prefill runs), inputs resident in
HBM. The headline workload is the 512K prefill (B=1, Hq=32, Hkv=8, d=128,
S=128, W=2048, K=32, planted needles every 64K tokens); the 128K and 32K
prefills follow as their own legs ("prefill_128k", "prefill_32k"), each
with its roofline. The decode step of the 512K, batch-8 workload is measured
in the same run (as a CUDA graph) and reported under "decode". L2 is flushed
(256 MiB write) before every timed step.

Rank 0 prints one JSON line. Under torchrun each rank runs its own replica of
the workload on its own GPU (the path shards by (batch, kv head) with no
exchange), timed with CUDA events, max over ranks.

--impl reference times the fp64 CPU oracle (the reference arm of this
build) on a bounded sample of query positions per step.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = ("HiLS fwd prefill tokens/s & decode µs/token at 1 B200; "
          "% of tensor/HBM roofline")
WORKLOADS = {"prefill_32k": 2, "prefill_128k": 3, "prefill_512k": 5}
DECODE_WORKLOAD = ("decode_512k_b8", 4)
L2_FLUSH_BYTES = 256 << 20
# query positions per oracle batch (each evaluated for every kv group): 16
# positions x 8 groups keep 16 host cores busy in one batch
REF_POSITIONS = 16


# ------------------------------------------------------------ work counting
def prefill_work(sh):
    """Algorithmic work of one prefill forward (touched, not executed):
    select FLOPs = sum_rows Hq * 2d|C_i|; attend FLOPs = sum_rows Hq *
    4d(|I_i| S + i - w0 + 1); HBM bytes of the inputs read once and outputs
    written once."""
    i = np.arange(sh.N, dtype=np.int64)
    lq = np.floor_divide(i - sh.W + 1, sh.S)
    nc = np.maximum(lq, 0)
    w0 = np.maximum(lq * sh.S, 0)
    sel = np.minimum(nc, sh.K)
    toks = sel * sh.S + (i - w0 + 1)
    f_select = float(sh.B * sh.Hq * 2 * sh.d * nc.sum())
    f_attend = float(sh.B * sh.Hq * 4 * sh.d * toks.sum())
    return dict(select_flops=f_select, attend_flops=f_attend,
                tokens=sh.B * sh.N)


def union_stats(sh, idx):
    """Chunk-union diagnostics of the attention tiling, counted on the
    device by the library's hils_chunk_overlap.

    The attention kernel gives each block of M = 128/G adjacent queries one
    CTA that loads the union of their selected chunks. Returns the mean union
    size, the pages' chunk-overlap ratio (MK - |union|) / ((M-1)K) (Sec. 7.2)
    averaged over blocks whose queries all have K selected chunks, the share
    of a block's chunks the previous block already had, and the
    executed/touched ratio of the attention MMA work (union + window tiles
    for all 128 rows vs. the algorithmic 4d(|I_i| S + window) per row-head).
    """
    import torch

    import chunk_sparse_long_landmark_b200 as hils
    M = 128 // sh.G
    B, Hkv, N, K = idx.shape
    n_sel, n_union, n_reuse = (t.double() for t in
                               hils.chunk_overlap(idx, N // sh.S, M))
    nqb = n_union.shape[-1]
    full = n_sel == M * K
    ov = ((M * K - n_union) / ((M - 1) * K))[full]
    reuse = (n_reuse[..., 1:] / n_union[..., 1:].clamp(min=1)).mean()
    i0 = torch.arange(nqb, device=idx.device, dtype=torch.float64) * M
    il = torch.clamp(i0 + M - 1, max=N - 1)
    w0 = torch.clamp(torch.div(i0 - sh.W + 1, sh.S, rounding_mode="floor") * sh.S, min=0)
    wt = torch.div(il - w0, sh.S, rounding_mode="floor") + 1
    # one CTA = 128 rows (all G heads of M queries) x (union + window) tiles
    executed = ((n_union + wt.view(1, 1, -1)) * 128 * sh.S * sh.d * 4).sum().item()
    touched = prefill_work(sh)["attend_flops"]
    return {"mean_union_chunks": n_union.mean().item(),
            "overlap_M": M,
            "overlap_mean": ov.mean().item() if ov.numel() else None,
            "reuse_of_previous_block": reuse.item() if nqb > 1 else None,
            "attend_executed_over_touched": executed / touched}


def decode_bytes(sh, cache_len):
    """Touched HBM bytes of one decode step: k' and b' of every candidate,
    K and V of the selected chunks and the window, Q, O, idx."""
    tot = 0
    esz = 2 if sh.dtype == "bf16" else 4
    for L in cache_len:
        i = L - 1
        lq = (i - sh.W + 1) // sh.S
        nc = max(lq, 0)
        w0 = max(lq * sh.S, 0)
        toks = min(nc, sh.K) * sh.S + (i - w0 + 1)
        tot += nc * sh.Hkv * (sh.d * esz + 4)
        tot += toks * sh.Hkv * 2 * sh.d * esz
        tot += 2 * sh.Hq * sh.d * esz + sh.Hkv * sh.K * 4
    return float(tot)


def decode_multi_bytes(sh, cache_len, T, idx):
    """Touched HBM bytes of one T-token decode step: k' and b' of every
    candidate once per (sequence, kv head) (one shared scan), K and V of the
    union over the T tokens of their selected chunks and windows, Q, O, idx.
    idx is the step's [B, T, Hkv, K] selection (host array)."""
    tot = 0
    esz = 2 if sh.dtype == "bf16" else 4
    for b, L in enumerate(cache_len):
        i_last = L - 1
        nc_last = max((i_last - sh.W + 1) // sh.S, 0)
        tot += nc_last * sh.Hkv * (sh.d * esz + 4)
        for g in range(sh.Hkv):
            spans = []
            for t in range(T):
                i = L - T + t
                lq = (i - sh.W + 1) // sh.S
                spans.append((max(lq * sh.S, 0), i + 1))
                spans += [(int(c) * sh.S, int(c) * sh.S + sh.S)
                          for c in idx[b, t, g] if c >= 0]
            spans.sort()
            n, end = 0, -1
            for a, e in spans:                   # length of the union
                if e <= end:
                    continue
                n += e - max(a, end)
                end = e
            tot += n * 2 * sh.d * esz
        tot += T * (2 * sh.Hq * sh.d * esz + sh.Hkv * sh.K * 4)
    return float(tot)


# ------------------------------------------------------------------- clocks
class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled during a region.

    A reader thread polls NVML every 5 ms (read-only queries), so even a
    region of a few tens of milliseconds gets samples. The device is matched
    by UUID, which holds whatever CUDA_VISIBLE_DEVICES maps it to. Without
    NVML it falls back to `nvidia-smi -lms 200` on the same UUID."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,"
         "clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.rows = []
        self.proc = self.path = self.thread = None
        self.stop = None

    def _uuid(self):
        try:
            import torch
            u = str(torch.cuda.get_device_properties(self.index).uuid)
            return u if u.startswith("GPU-") else "GPU-" + u
        except Exception:
            return None

    def __enter__(self):
        import threading
        uuid = self._uuid()
        try:
            import pynvml as nv
            nv.nvmlInit()
            h = (nv.nvmlDeviceGetHandleByUUID(uuid) if uuid
                 else nv.nvmlDeviceGetHandleByIndex(self.index))
            smax = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons",
                                  None) or nv.nvmlDeviceGetCurrentClocksThrottleReasons
            bits = {"hw": 0x8, "hwt": 0x40, "swt": 0x20, "pcap": 0x4}
            self.stop = threading.Event()

            def run():
                while not self.stop.is_set():
                    try:
                        r = int(get_reasons(h))
                        row = dict(sm=float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)),
                                   smax=smax,
                                   power=nv.nvmlDeviceGetPowerUsage(h) / 1e3)
                        for k, bit in bits.items():
                            row[k] = "Active" if r & bit else "Not Active"
                        self.rows.append(row)
                    except Exception:
                        pass
                    self.stop.wait(0.005)

            self.thread = threading.Thread(target=run, daemon=True)
            self.thread.start()
            return self
        except Exception:
            self.thread = None
        import tempfile
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={uuid or self.index}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.thread is not None:
            self.stop.set()
            self.thread.join(timeout=5)
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = list(self.rows)
        if self.path and os.path.exists(self.path):
            for line in open(self.path):
                f = [x.strip() for x in line.split(",")]
                if len(f) < 9:
                    continue
                try:
                    rows.append(dict(sm=float(f[1]), smax=float(f[2]),
                                     power=float(f[3]), hw=f[5], hwt=f[6],
                                     swt=f[7], pcap=f[8]))
                except ValueError:
                    continue
            os.unlink(self.path)
        if not rows:
            return None
        reasons = set()
        for r in rows:
            for k, n in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                         ("swt", "sw_thermal_slowdown"),
                         ("pcap", "sw_power_cap")):
                if r[k].lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(r["sm"] for r in rows),
                "sm_max_mhz": max(r["smax"] for r in rows),
                "samples": len(rows), "reasons": sorted(reasons),
                "source": "nvml" if self.thread is not None else "nvidia-smi"}


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"],
                    bf16_sustained=d.get("bf16_tflops_sustained",
                                         d["bf16_tflops"]),
                    src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0,
                src="fallback")


def profiled_traffic(kernels, workload):
    """DRAM bytes per launch that one ncu capture recorded for `kernels`.

    Read from profiles/traffic.json (written from `ncu --set full` captures,
    one launch per kernel, dram__bytes_read.sum + dram__bytes_write.sum).
    Returns None when a kernel was not captured on this workload, or when
    its source file has changed since the capture (sha256 prefix differs).
    """
    import hashlib
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        tab = json.load(open(p))
    except (OSError, ValueError):
        return None
    total = 0
    for k in kernels:
        ent = tab.get(f"{k}@{workload}") or tab.get(k)
        if not ent or ent.get("workload") != workload:
            return None
        try:
            src = open(os.path.join(ROOT, ent["file"]), "rb").read()
        except OSError:
            return None
        if hashlib.sha256(src).hexdigest()[:16] != ent["source_sha256"]:
            return None
        total += int(ent["bytes_per_launch"])
    return total


# -------------------------------------------------------------- oracle arm
def oracle_sample(inp, budget_s, positions_per_batch=REF_POSITIONS, seed=0,
                  max_batches=None, bound=None):
    """Time the fp64 oracle on random query positions of the workload until
    `budget_s` seconds of work. Returns (tokens/s, positions, seconds,
    threads). `bound`: the inputs already copied to the host by
    oracle.bind_prefill (copied here otherwise, outside the timing)."""
    import oracle
    sh = inp["shape"]
    rng = np.random.default_rng(seed)
    bound = bound or oracle.bind_prefill(inp)
    done, t0 = 0, time.perf_counter()
    nb = 0
    while True:
        pos = rng.integers(0, sh.N, size=positions_per_batch)
        rows = np.array([[b, g, i] for b in range(sh.B)
                         for g in range(sh.Hkv) for i in pos])
        oracle.prefill_rows(inp, rows, bound=bound)
        done += len(pos) * sh.B
        nb += 1
        el = time.perf_counter() - t0
        if el >= budget_s or (max_batches and nb >= max_batches):
            break
    return done / el, done, el, oracle.max_threads()


def host_inputs(inp):
    import torch
    out = {}
    for k in ("Q", "K", "V", "Klm", "bias"):
        t = inp[k].cpu()
        out[k] = t.pin_memory() if torch.cuda.is_available() else t
    return out


def run_reference(args, sh, name):
    """The CPU oracle as the reference arm, on this arm's workload."""
    import synth
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import torch
    # the inputs are drawn on the GPU when there is one (the same numbers as
    # the GPU arm's) and copied to the host by the oracle's binding
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    inp = synth.make_prefill(sh, seed=synth.seed_for(WORKLOADS[name]),
                             device=dev)
    import oracle
    bound = oracle.bind_prefill(inp)
    per_step = []
    cnt = []
    for s in range(args.warmup + args.steps):
        v, n, el, thr = oracle_sample(inp, budget_s=0.0,
                                      positions_per_batch=REF_POSITIONS,
                                      seed=s, max_batches=1, bound=bound)
        if s >= args.warmup:
            per_step.append(el)
            cnt.append(n)
    tot = sum(per_step)
    val = sum(cnt) / tot
    line = {
        "impl": "reference", "metric": METRIC, "value": val,
        "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * tot / len(per_step),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic",
        "config": workload_config(sh, name),
        "cpu_baseline": {"value": val, "unit": "tokens/s", "cores": thr,
                         "kind": "oracle",
                         "sample": f"{REF_POSITIONS} random query positions "
                                   f"x {sh.Hkv} kv groups (all {sh.Hq} heads) "
                                   f"per step of the {name} workload"},
        "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_config(sh, name):
    return {"workload": name, "B": sh.B, "Hq": sh.Hq, "Hkv": sh.Hkv,
            "d": sh.d, "N": sh.N, "S": sh.S, "W": sh.W, "K": sh.K,
            "structure": sh.structure,
            "l2": "flushed by a 256 MiB write before every timed step",
            "parallelism": "one independent replica per GPU (shards by "
                           "(batch, kv head), no collective)"}


# ------------------------------------------------------------ rank plumbing
class RankContext:
    """One process per GPU, launched by torchrun (RANK / WORLD_SIZE / MASTER_*
    from the environment). Each rank runs its own replica of the workload
    (the path shards by (batch, kv head) with no exchange), so the only
    collectives are the barrier around the timed region and the max over
    ranks of the measured time. `backend` is "nccl" on GPUs; the same code
    runs on "gloo" with CPU tensors."""

    def __init__(self, backend="nccl", device=None, timeout_s=300):
        import torch
        import torch.distributed as dist
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.device = device if device is not None else torch.device("cpu")
        self._dist = None
        if self.world > 1:
            from datetime import timedelta
            kw = {"device_id": self.device} if backend == "nccl" else {}
            dist.init_process_group(backend, timeout=timedelta(seconds=timeout_s),
                                    **kw)
            self._dist = dist

    def barrier(self):
        if self._dist is not None:
            self._dist.barrier()

    def max(self, x):
        """Largest value of x over all ranks (a device-timed duration)."""
        import torch
        t = torch.tensor([float(x)], dtype=torch.float64, device=self.device)
        if self._dist is not None:
            self._dist.all_reduce(t, op=self._dist.ReduceOp.MAX)
        return float(t.item())

    def whole_job_rate(self, units_per_rank, ms_max):
        """Units all ranks processed per second, over the slowest rank's
        time (ms_max, already the max over ranks)."""
        return self.world * units_per_rank / (ms_max * 1e-3)

    def close(self):
        if self._dist is not None:
            self._dist.destroy_process_group()
            self._dist = None


# ---------------------------------------------------------------- GPU arm
def bench_prefill(args, name, dev, stream, flush, ranks, peaks, steps,
                  with_e2e, rank, seq_len=0):
    """Time one prefill workload through the C ABI (select then attend, as
    hils_fwd_prefill runs them), L2 flushed before every timed step.

    Returns the leg's dict: step time, stage times, the dominant kernel's
    roofline (algorithmic FLOPs of that stage / its mean event-timed
    duration), the whole step's fraction on the touched FLOPs of select +
    attend, chunk-union diagnostics and, if asked, the end-to-end figure
    (pinned host buffers, copies inside the timed region)."""
    import torch

    import chunk_sparse_long_landmark_b200 as hils
    import synth
    cfg_id = WORKLOADS[name]
    sh = synth.PREFILL_CONFIGS[cfg_id]
    if seq_len:
        sh = sh.with_(N=seq_len)
    inp = synth.make_prefill(sh, seed=synth.seed_for(cfg_id) + 17 * rank,
                             device=dev)
    work = prefill_work(sh)
    B, Hq, Hkv, N, K = sh.B, sh.Hq, sh.Hkv, sh.N, sh.K
    O = torch.empty_like(inp["Q"])
    idx = torch.empty(B, Hkv, N, K, dtype=torch.int32, device=dev)
    sel = torch.empty(B, Hq, N, K, dtype=torch.float32, device=dev)
    ws = torch.empty(max(1, hils.prefill_workspace_size(
        inp["Q"], inp["K"], inp["V"], inp["Klm"], inp["bias"],
        inp["head_map"], sh.S, sh.W, K, with_sel_score=True)),
        dtype=torch.uint8, device=dev)

    def call(stage):
        hils.fwd_prefill(inp["Q"], inp["K"], inp["V"], inp["Klm"],
                         inp["bias"], inp["head_map"], sh.S, sh.W, K,
                         out=O, idx=idx, sel_score=sel, workspace=ws,
                         stream=stream, stage=stage)

    for _ in range(args.warmup):
        call("select")
        call("attend")
    torch.cuda.synchronize()

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)]
           for _ in range(steps)]
    ranks.barrier()
    torch.cuda.synchronize()
    n0 = hils.launch_count()
    with ClockSampler(torch.cuda.current_device()) as clk:
        for s in range(steps):
            flush.zero_()
            evs[s][0].record(stream)
            call("select")
            evs[s][1].record(stream)
            call("attend")
            evs[s][2].record(stream)
        torch.cuda.synchronize()
    ranks.barrier()
    launches = hils.launch_count() - n0
    t_sel = [e[0].elapsed_time(e[1]) for e in evs]
    t_att = [e[1].elapsed_time(e[2]) for e in evs]
    t_step = [a + b for a, b in zip(t_sel, t_att)]
    ms_step = ranks.max(sum(t_step)) / steps
    value = ranks.whole_job_rate(work["tokens"], ms_step)

    # a region of more than 2 s of back-to-back kernels runs under the power
    # cap: it is compared with the sustained GEMM figure
    sustained = steps * ms_step > 2000
    peak = peaks["bf16_sustained"] if sustained else peaks["bf16"]
    a_ms, s_ms = statistics.mean(t_att), statistics.mean(t_sel)
    if a_ms >= s_ms:
        dom, dom_ms, dom_flops = "attend", a_ms, work["attend_flops"]
    else:
        dom, dom_ms, dom_flops = "select", s_ms, work["select_flops"]
    achieved = dom_flops / (dom_ms * 1e-3) / 1e12
    touched = work["select_flops"] + work["attend_flops"]
    step_ach = touched / (ms_step * 1e-3) / 1e12
    roof = {"bound": "tensor", "kernel": dom, "achieved": achieved,
            "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
            "peak_source": peaks["src"] + (" (sustained bf16 GEMM)" if sustained
                                           else " (burst bf16 GEMM)"),
            "algorithmic_flops_per_launch": dom_flops,
            "traffic": profiled_traffic(
                ["tc_attend" if dom == "attend" else "tc_select"], name),
            "whole_step": {
                "achieved": step_ach, "frac": step_ach / peak,
                "touched_flops": touched,
                "definition": "touched FLOPs of scoring + intra-chunk + "
                              "window attention (a2 + a5 + a6) / step time"},
            "stages": {
                "select": {"achieved": work["select_flops"] / (s_ms * 1e-3) / 1e12,
                           "frac": work["select_flops"] / (s_ms * 1e-3) / 1e12 / peak,
                           "flops": work["select_flops"]},
                "attend": {"achieved": work["attend_flops"] / (a_ms * 1e-3) / 1e12,
                           "frac": work["attend_flops"] / (a_ms * 1e-3) / 1e12 / peak,
                           "flops": work["attend_flops"]}}}
    leg = {"workload": name, "value": value, "unit": "tokens/s",
           "ms_per_step": ms_step, "steps": steps,
           "stages_ms": {"select": s_ms, "attend": a_ms},
           "roofline": roof, "gpu_launches": int(launches),
           "clocks": clk.summary(), "union": union_stats(sh, idx),
           "config": workload_config(sh, name + (f"_n{sh.N}" if seq_len else ""))}

    if with_e2e:
        # end to end through the C ABI with host buffers (pinned), per step:
        # H2D of Q, K, V, Klm, bias; the call; D2H of O and idx
        host = host_inputs(inp)
        Oh = torch.empty(O.shape, dtype=O.dtype).pin_memory()
        Ih = torch.empty(idx.shape, dtype=idx.dtype).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in host.values())
        d2h = Oh.numel() * Oh.element_size() + Ih.numel() * Ih.element_size()
        dvs = {k: torch.empty_like(inp[k]) for k in host}

        def e2e_step():
            for k, t in host.items():
                dvs[k].copy_(t, non_blocking=True)
            hils.fwd_prefill(dvs["Q"], dvs["K"], dvs["V"], dvs["Klm"],
                             dvs["bias"], inp["head_map"], sh.S, sh.W, K,
                             out=O, idx=idx, sel_score=sel, workspace=ws,
                             stream=stream)
            Oh.copy_(O, non_blocking=True)
            Ih.copy_(idx, non_blocking=True)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        ranks.barrier()
        ee = [(torch.cuda.Event(enable_timing=True),
               torch.cuda.Event(enable_timing=True))
              for _ in range(max(3, steps // 4))]
        for a, b in ee:
            flush.zero_()
            a.record(stream)
            e2e_step()
            b.record(stream)
        torch.cuda.synchronize()
        e_ms = ranks.max(sum(a.elapsed_time(b) for a, b in ee)) / len(ee)
        leg["e2e"] = {"value": ranks.world * work["tokens"] / (e_ms * 1e-3),
                      "unit": "tokens/s", "ms_per_step": e_ms,
                      "h2d_bytes_per_step": int(h2d),
                      "d2h_bytes_per_step": int(d2h)}
        del host, dvs, Oh, Ih
    del inp, O, idx, sel, ws
    torch.cuda.empty_cache()
    return leg


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="prefill_512k",
                    choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="hils", choices=["hils", "reference"])
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-legs", action="store_true",
                    help="skip the other prefill workloads' legs")
    ap.add_argument("--decode-only", action="store_true",
                    help="time only the decode step (prints its object)")
    ap.add_argument("--decode-batch", type=int, default=0,
                    help="run the decode legs with this many sequences instead "
                         "of the workload's (reduced cases for profilers)")
    ap.add_argument("--backward-workload", default="prefill_32k",
                    choices=sorted(WORKLOADS),
                    help="prefill workload of the backward leg")
    ap.add_argument("--backward-only", action="store_true",
                    help="time only the 32K prefill backward (prints its object)")
    ap.add_argument("--seq-len", type=int, default=0,
                    help="run the headline workload at this sequence length "
                         "instead of its own (reduced cases for profilers)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    import synth
    cfg_id = WORKLOADS[args.workload]
    sh = synth.PREFILL_CONFIGS[cfg_id]
    if args.impl == "reference":
        run_reference(args, sh, args.workload)
        return

    import torch

    import chunk_sparse_long_landmark_b200 as hils  # noqa: F401 (fails loudly)

    local = int(os.environ.get("LOCAL_RANK", "0"))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    ranks = RankContext("nccl", dev)
    world, rank = ranks.world, ranks.rank
    barrier, max_over_ranks = ranks.barrier, ranks.max

    peaks = measured_peaks()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    if args.backward_only:
        bw = bench_backward(args, dev, stream, flush, max_over_ranks, barrier,
                            rank)
        if rank == 0:
            print(json.dumps({"backward": bw}), flush=True)
        ranks.close()
        return
    if args.decode_only:
        d = bench_decode(args, dev, stream, flush, world, max_over_ranks,
                         barrier, rank, peaks)
        dm = bench_decode_multi(args, dev, stream, flush, world,
                                max_over_ranks, barrier, rank, peaks)
        if rank == 0:
            print(json.dumps({"decode": d, "decode_multi": dm}), flush=True)
        ranks.close()
        return

    head = bench_prefill(args, args.workload, dev, stream, flush, ranks,
                         peaks, args.steps, not args.no_e2e, rank,
                         seq_len=args.seq_len)
    line = {
        "metric": METRIC, "value": head["value"], "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": head["ms_per_step"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": head["config"],
        "stages_ms": head["stages_ms"], "roofline": head["roofline"],
        "gpu_launches": head["gpu_launches"], "clocks": head["clocks"],
        "union": head["union"],
    }
    if "e2e" in head:
        line["e2e"] = head["e2e"]

    if not args.no_legs:
        # the other prefill workloads, each with its own roofline
        for other in sorted(WORKLOADS, key=lambda n: -WORKLOADS[n]):
            if other == args.workload:
                continue
            line[other] = bench_prefill(args, other, dev, stream, flush, ranks,
                                        peaks, max(args.steps, 10), False,
                                        rank)

    if not args.no_decode:
        line["decode"] = bench_decode(args, dev, stream, flush, world,
                                      max_over_ranks, barrier, rank, peaks)
        line["decode_multi"] = bench_decode_multi(
            args, dev, stream, flush, world, max_over_ranks, barrier, rank,
            peaks)
        line["landmarks"] = bench_landmarks(args, dev, stream, flush,
                                            max_over_ranks, barrier, peaks)
        line["backward"] = bench_backward(args, dev, stream, flush,
                                          max_over_ranks, barrier, rank)

    if rank == 0 and world == 1 and not args.no_cpu:
        cinp = synth.make_prefill(sh, seed=synth.seed_for(cfg_id),
                                  device=dev)
        v, n, el, thr = oracle_sample(cinp, budget_s=15.0,
                                      positions_per_batch=REF_POSITIONS)
        line["cpu_baseline"] = {
            "value": v, "unit": "tokens/s", "cores": thr, "kind": "oracle",
            "sample": f"{n} random query positions (all {sh.Hq} heads, "
                      f"{REF_POSITIONS} positions x {sh.Hkv} kv groups per "
                      f"batch) of the {args.workload} workload, {el:.1f} s"}
        del cinp

    if rank == 0:
        print(json.dumps(line), flush=True)
    ranks.close()


def bench_landmarks(args, dev, stream, flush, max_over_ranks, barrier,
                    peaks):
    """Landmark summaries (Prop. 3.1) of the 128K-token key tensor of the
    128K prefill workload: one landmark query per chunk, L2 flushed before
    every call. HBM roofline on K + q' read and k' + b' written."""
    import torch

    import chunk_sparse_long_landmark_b200 as hils
    import synth
    sh = synth.PREFILL_CONFIGS[3]
    B, Hkv, N, d, S = sh.B, sh.Hkv, sh.N, sh.d, sh.S
    nC = N // S
    g = torch.Generator(device=dev).manual_seed(7)
    K = torch.randn(B, Hkv, N, d, generator=g, device=dev).to(torch.bfloat16)
    Q = torch.randn(B, Hkv, nC, d, generator=g, device=dev).to(torch.bfloat16)
    out = (torch.empty(B, Hkv, nC, d, dtype=torch.bfloat16, device=dev),
           torch.empty(B, Hkv, nC, dtype=torch.float32, device=dev))
    for _ in range(args.warmup):
        hils.build_landmarks(K, Q, S, out=out, stream=stream)
    steps = max(args.steps, 10)
    evs = [(torch.cuda.Event(enable_timing=True),
            torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    barrier()
    torch.cuda.synchronize()
    for a, b in evs:
        flush.zero_()
        a.record(stream)
        hils.build_landmarks(K, Q, S, out=out, stream=stream)
        b.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in evs)) / steps
    nbytes = 2 * (B * Hkv * N * d + 2 * B * Hkv * nC * d) + 4 * B * Hkv * nC
    ach = nbytes / (ms * 1e-3) / 1e9
    del K, Q, out
    torch.cuda.empty_cache()
    return {"workload": "landmarks_128k",
            "description": "Prop. 3.1 summaries of the 128K prefill keys, "
                           "one landmark query per chunk",
            "value": ms * 1e3, "unit": "us/call",
            "roofline": {"bound": "hbm", "achieved": ach,
                         "peak": peaks["hbm"], "unit": "GB/s",
                         "frac": ach / peaks["hbm"],
                         "peak_source": peaks["src"],
                         "algorithmic_bytes": nbytes,
                         "traffic": profiled_traffic(["landmarks"],
                                                     "landmarks_128k")},
            "config": {"B": B, "Hkv": Hkv, "N": N, "d": d, "S": S,
                       "l2": "flushed before every call"}}


def bench_decode(args, dev, stream, flush, world, max_over_ranks, barrier,
                 rank, peaks):
    import torch

    import chunk_sparse_long_landmark_b200 as hils
    import synth
    name, cid = DECODE_WORKLOAD
    sh = synth.DECODE_CONFIGS[cid]
    if getattr(args, "decode_batch", 0):
        sh = sh.with_(B=args.decode_batch)
        name = f"{name}_reduced_b{args.decode_batch}"
    inp = synth.make_decode(sh, seed=synth.seed_for(cid) + 17 * rank,
                            device=dev)
    O = torch.empty_like(inp["Q"])
    idx = torch.empty(sh.B, sh.Hkv, sh.K, dtype=torch.int32, device=dev)
    sel = torch.empty(sh.B, sh.Hq, sh.K, dtype=torch.float32, device=dev)
    ws = torch.empty(hils.decode_workspace_size(
        inp["Q"], inp["K"], inp["V"], inp["Klm"], inp["bias"],
        inp["cache_len"], inp["head_map"], sh.S, sh.W, sh.K,
        with_sel_score=True), dtype=torch.uint8, device=dev)
    side = torch.cuda.Stream(dev)

    def call(st, stage="both"):
        hils.fwd_decode(inp["Q"], inp["K"], inp["V"], inp["Klm"],
                        inp["bias"], inp["cache_len"], inp["head_map"], sh.S,
                        sh.W, sh.K, out=O, idx=idx, sel_score=sel,
                        workspace=ws, stream=st, stage=stage)

    with torch.cuda.stream(side):
        for _ in range(args.warmup):
            call(side)
    side.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        call(side)
    torch.cuda.synchronize()
    steps = max(args.steps, 20)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    barrier()
    evs = [(torch.cuda.Event(enable_timing=True),
            torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    cur = torch.cuda.current_stream(dev)
    for a, b in evs:
        flush.zero_()
        a.record(cur)
        g.replay()
        b.record(cur)
    torch.cuda.synchronize()
    times = [a.elapsed_time(b) for a, b in evs]
    ms = max_over_ranks(sum(times)) / steps
    med = statistics.median(times)
    # stage split (eager, separate events)
    ss = []
    for _ in range(5):
        e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        flush.zero_()
        e[0].record(cur)
        call(cur, "select")
        e[1].record(cur)
        call(cur, "attend")
        e[2].record(cur)
        torch.cuda.synchronize()
        ss.append((e[0].elapsed_time(e[1]), e[1].elapsed_time(e[2])))
    # end to end through the C ABI: the step's queries copied in from pinned
    # host memory and O, idx copied back, inside the timed region (the KV
    # cache and landmarks are resident state)
    hq = torch.empty(inp["Q"].shape, dtype=inp["Q"].dtype).pin_memory()
    hq.copy_(inp["Q"].cpu())
    hO = torch.empty(O.shape, dtype=O.dtype).pin_memory()
    hidx = torch.empty(idx.shape, dtype=idx.dtype).pin_memory()
    dq = torch.empty_like(inp["Q"])

    def e2e_step():
        dq.copy_(hq, non_blocking=True)
        hils.fwd_decode(dq, inp["K"], inp["V"], inp["Klm"], inp["bias"],
                        inp["cache_len"], inp["head_map"], sh.S, sh.W, sh.K,
                        out=O, idx=idx, sel_score=sel, workspace=ws,
                        stream=cur)
        hO.copy_(O, non_blocking=True)
        hidx.copy_(idx, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    ee = [(torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for a, b in ee:
        flush.zero_()
        a.record(cur)
        e2e_step()
        b.record(cur)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in ee)) / steps
    cl = inp["cache_len"].cpu().tolist()
    nbytes = decode_bytes(sh, cl)
    ach = nbytes / (ms * 1e-3) / 1e9
    del g
    out = {
        "workload": name, "value": ms * 1e3, "unit": "us/step",
        "note": f"one decode step = one new token for each of the B={sh.B} "
                "sequences (per-token latency of every sequence)",
        "median_us": med * 1e3, "tokens_per_s": world * sh.B / (ms * 1e-3),
        "stages_ms": {"select": statistics.mean(x[0] for x in ss),
                      "attend": statistics.mean(x[1] for x in ss)},
        "roofline": {"bound": "hbm", "kernel": "whole decode step (graph)",
                     "achieved": ach, "peak": peaks["hbm"], "unit": "GB/s",
                     "frac": ach / peaks["hbm"], "peak_source": peaks["src"],
                     "algorithmic_bytes_per_step": nbytes,
                     "traffic": profiled_traffic(
                         ["dec_score", "dec_select", "dec_attend"], name),
                     "traffic_covers": "dec_score + dec_select + dec_attend "
                                       "launches"},
        "e2e": {"value": e2e_ms * 1e3, "unit": "us/step",
                "h2d_bytes_per_step": hq.numel() * hq.element_size(),
                "d2h_bytes_per_step": hO.numel() * hO.element_size() +
                                      hidx.numel() * hidx.element_size(),
                "note": "queries in, O and idx out per step; caches resident"},
        "config": {"B": sh.B, "Hq": sh.Hq, "Hkv": sh.Hkv, "d": sh.d,
                   "L": sh.N, "S": sh.S, "W": sh.W, "K": sh.K,
                   "l2": "flushed before every timed step"},
    }
    del inp, O, idx, sel, ws, dq
    torch.cuda.empty_cache()
    return out


def bench_backward(args, dev, stream, flush, max_over_ranks, barrier, rank):
    """Backward of a prefill workload (32K unless --backward-workload says
    otherwise; selection from the forward, dO ~ N(0,1)), L2 flushed before
    every call. Its contractions (s, u, dq,
    dK, dV) run on the tensor cores in bf16 with f32 accumulation: roofline
    "tensor" against the measured bf16 peak, on the touched FLOPs: 10d per
    (row, head, attended token) plus 4d per (row, head, selected chunk) for
    dqs and dk'."""
    import torch

    import chunk_sparse_long_landmark_b200 as hils
    import synth
    wl = getattr(args, "backward_workload", "prefill_32k")
    cid = WORKLOADS[wl]
    sh = synth.PREFILL_CONFIGS[cid]
    inp = synth.make_prefill(sh, seed=synth.seed_for(cid) + 17 * rank + 3,
                             device=dev)
    _, idx = hils.fwd_prefill(inp["Q"], inp["K"], inp["V"], inp["Klm"],
                              inp["bias"], inp["head_map"], sh.S, sh.W, sh.K,
                              stream=stream)
    g0 = torch.Generator(device=dev).manual_seed(11)
    dO = torch.randn(inp["Q"].shape, generator=g0, device=dev).to(inp["Q"].dtype)
    grads = None

    def call():
        nonlocal grads
        grads = hils.bwd_prefill(inp["Q"], inp["K"], inp["V"], inp["Klm"],
                                 inp["bias"], inp["head_map"], sh.S, sh.W,
                                 idx, dO, grads=grads, stream=stream)

    for _ in range(max(1, min(args.warmup, 2))):
        call()
    steps = max(1, min(args.steps, 3))
    evs = [(torch.cuda.Event(enable_timing=True),
            torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    barrier()
    torch.cuda.synchronize()
    for a, b in evs:
        flush.zero_()
        a.record(stream)
        call()
        b.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in evs)) / steps
    i = np.arange(sh.N, dtype=np.int64)
    lq = np.floor_divide(i - sh.W + 1, sh.S)
    nc = np.maximum(lq, 0)
    w0 = np.maximum(lq * sh.S, 0)
    sel = np.minimum(nc, sh.K)
    toks = sel * sh.S + (i - w0 + 1)
    flops = float(sh.B * sh.Hq * sh.d * (10 * toks.sum() + 4 * sel.sum()))
    ach = flops / (ms * 1e-3) / 1e12
    peaks = measured_peaks()
    peak = peaks["bf16"]
    del inp, idx, dO, grads
    torch.cuda.empty_cache()
    return {"workload": f"{wl}_backward",
            "description": f"dQ, dK, dV, dk', db' of the {wl} prefill for "
                           "the forward's selection",
            "value": sh.B * sh.N / (ms * 1e-3), "unit": "tokens/s",
            "ms_per_step": ms, "steps": steps,
            "roofline": {"bound": "tensor", "achieved": ach, "peak": peak,
                         "unit": "TFLOP/s", "frac": ach / peak,
                         "peak_source": ("measured (burst bf16 GEMM)"
                                         if peaks["src"] == "measured"
                                         else "fallback (burst bf16)"),
                         "algorithmic_flops_per_call": flops,
                         "traffic": profiled_traffic(
                             ["bwd_rows_tc", "bwd_dqs", "bwd_keys_tc"],
                             f"{wl}_backward"),
                         "traffic_covers": "bwd_rows_tc + bwd_dqs + bwd_keys_tc "
                                           "(94% of the call; the landmark-score "
                                           "and index kernels not captured)"},
            "config": {"B": sh.B, "Hq": sh.Hq, "Hkv": sh.Hkv, "d": sh.d,
                       "N": sh.N, "S": sh.S, "W": sh.W, "K": sh.K,
                       "dtype": "bf16 inputs; bf16 tensor-core products (p and "
                                "ds rounded to bf16), f32 accumulation, f32 "
                                "gradients",
                       "l2": "flushed before every call"}}


DECODE_MULTI_T = 4


def bench_decode_multi(args, dev, stream, flush, world, max_over_ranks,
                       barrier, rank, peaks):
    """Speculative decode: the 512K batch-8 decode workload with T = 4 query
    tokens per sequence (positions L-4 .. L-1) in one step, as a CUDA graph,
    L2 flushed before every timed step. HBM roofline on the bytes the step
    must touch: one landmark scan per (sequence, kv head) and the union of
    the T tokens' chunks and windows."""
    import torch

    import chunk_sparse_long_landmark_b200 as hils
    import synth
    name, cid = DECODE_WORKLOAD
    sh = synth.DECODE_CONFIGS[cid]
    if getattr(args, "decode_batch", 0):
        sh = sh.with_(B=args.decode_batch)
    T = DECODE_MULTI_T
    inp = synth.make_decode(sh, seed=synth.seed_for(cid) + 17 * rank + 5,
                            device=dev)
    g0 = torch.Generator(device=dev).manual_seed(synth.seed_for(cid) + 29)
    Qm = torch.randn(sh.B, T, sh.Hq, sh.d, generator=g0,
                     device=dev).to(torch.bfloat16)
    O = torch.empty_like(Qm)
    idx = torch.empty(sh.B, T, sh.Hkv, sh.K, dtype=torch.int32, device=dev)
    sel = torch.empty(sh.B, T, sh.Hq, sh.K, dtype=torch.float32, device=dev)
    side = torch.cuda.Stream(dev)
    ws = None

    def call(st):
        nonlocal ws
        _, _ = hils.fwd_decode_multi(Qm, inp["K"], inp["V"], inp["Klm"],
                                     inp["bias"], inp["cache_len"],
                                     inp["head_map"], sh.S, sh.W, sh.K,
                                     out=O, idx=idx, sel_score=sel,
                                     workspace=ws, stream=st)

    n = ctypes_workspace_multi(hils, Qm, inp, sh, T)
    ws = torch.empty(n, dtype=torch.uint8, device=dev)
    with torch.cuda.stream(side):
        for _ in range(args.warmup):
            call(side)
    side.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        call(side)
    torch.cuda.synchronize()
    steps = max(args.steps, 20)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    barrier()
    evs = [(torch.cuda.Event(enable_timing=True),
            torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    cur = torch.cuda.current_stream(dev)
    for a, b in evs:
        flush.zero_()
        a.record(cur)
        g.replay()
        b.record(cur)
    torch.cuda.synchronize()
    times = [a.elapsed_time(b) for a, b in evs]
    ms = max_over_ranks(sum(times)) / steps
    cl = inp["cache_len"].cpu().tolist()
    nbytes = decode_multi_bytes(sh, cl, T, idx.cpu().numpy())
    ach = nbytes / (ms * 1e-3) / 1e9
    del g
    out = {
        "workload": f"{name}_T{T}", "value": ms * 1e3, "unit": "us/step",
        "note": f"one step = {T} speculative query tokens for each of the "
                f"B={sh.B} sequences (positions L-{T} .. L-1)",
        "median_us": statistics.median(times) * 1e3,
        "tokens_per_s": world * sh.B * T / (ms * 1e-3),
        "roofline": {"bound": "hbm", "kernel": "whole multi-token step (graph)",
                     "achieved": ach, "peak": peaks["hbm"], "unit": "GB/s",
                     "frac": ach / peaks["hbm"], "peak_source": peaks["src"],
                     "algorithmic_bytes_per_step": nbytes,
                     "bytes_model": "k', b' once per (sequence, kv head); K, V "
                                    "of the union of the tokens' chunks and "
                                    "windows",
                     "traffic": None},
        "config": {"B": sh.B, "T": T, "Hq": sh.Hq, "Hkv": sh.Hkv, "d": sh.d,
                   "L": sh.N, "S": sh.S, "W": sh.W, "K": sh.K,
                   "l2": "flushed before every timed step"},
    }
    del inp, Qm, O, idx, sel, ws
    torch.cuda.empty_cache()
    return out


def ctypes_workspace_multi(hils, Qm, inp, sh, T):
    """Workspace bytes of the multi-token step (with sel_score given)."""
    import ctypes
    hm = (ctypes.c_int32 * sh.Hq)(*inp["head_map"])
    fake = 1 << 40
    base = hils.DecodeArgs(hils.BF16, sh.B, sh.Hq, sh.Hkv, sh.N, sh.d, sh.S,
                           sh.W, sh.K, ctypes.cast(hm, ctypes.c_void_p), fake,
                           None, fake, fake, fake, fake, fake, fake, fake,
                           fake, None, 0, None)
    a = hils.DecodeMultiArgs(base, T, None, 0)
    n = ctypes.c_size_t(0)
    rc = hils.lib().hils_decode_multi_workspace_size(ctypes.byref(a),
                                                     ctypes.byref(n))
    if rc:
        raise hils.HilsError(rc, "hils_decode_multi_workspace_size")
    return max(n.value, 1)


if __name__ == "__main__":
    main()
