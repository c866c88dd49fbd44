"""Benchmark of the OCTOPUS codec on B200: encode + fused decode attention.

Headline workload (one GPU, the largest single-GPU decode workload):
batched long-context decode with OCTOPUS-QJL - batch 8, 32 query heads over
8 KV heads (GQA 4), head_dim 128, context 131072, bf16 keys (N(0,1), four
outlier channels x10, per-token lognormal(0, 0.5) scale), bf16 V and q ~
N(0,1), b = 4 plus the 1-bit residual sign sketch, joint rounding. One step
= encode the prefill cache (64 x 131072 keys) + one fused decode-attention
step (256 query heads over the whole cache).

Timing: CUDA events on the launching stream around each kernel; the step
loop is bracketed by a barrier and a device synchronize; the max over ranks
is reported. L2 (126 MB): two caches alternate, so each decode reads the
cache encoded one step earlier (2.95 GB of decode input, far larger than
L2, with the other cache's encode - 2.15 GB read, 0.8 GB written - in
between). Primary metric: decode-attention achieved HBM GB/s over the
algorithmic bytes (packed codes + gamma + sketch words + residual norms +
bf16 V + q + out); encode is reported in Mkeys/s.

The other decode workloads (LLM decode at context 32768 with b = 3, the
video/audio shape with d = 64, b = 2 and 8 query tokens) are timed over
caches the encoder wrote from keys of their recipe, with L2 flushed (a
512 MB buffer written) before every timed call.

``--gpus N`` without a launcher starts N ranks itself (one process per GPU,
each an independent batch, no collective on the data path); under torchrun
the ranks come from the environment. ``--impl reference`` times the CPU
oracle (the plain float64 restatement of the method) on a bounded sample of
the headline workload instead.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import socket
import subprocess
import sys
import threading
import time
from collections import namedtuple

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

SEED = 0
METRIC = "compressed-KV decode-attention HBM GB/s (% of ~8 TB/s); encode Mkeys/s"

Workload = namedtuple("Workload", "name B HQ HKV LQ D BITS N QJL keys")
QJL_LONG = Workload("qjl_long_context", 8, 32, 8, 1, 128, 4, 131072, True, "llm")
LLM_DECODE = Workload("llm_decode", 1, 32, 8, 1, 128, 3, 32768, False, "llm")
VIDEO_AUDIO = Workload("video_audio", 1, 16, 16, 8, 64, 2, 65536, False, "gauss")
LLM_DECODE_LARGE = Workload("llm_decode_large", 8, 32, 8, 1, 128, 3, 131072, False, "llm")
HEADLINE = QJL_LONG
OTHER_WORKLOADS = (LLM_DECODE, VIDEO_AUDIO, LLM_DECODE_LARGE)


def describe(w: Workload) -> str:
    keys = "bf16 keys N(0,1) x 4 outlier channels x10 x per-token lognormal(0,0.5)" if w.keys == "llm" else \
        "bf16 keys N(0,1)"
    return (f"{w.name}: B={w.B}, Hq={w.HQ}, Hkv={w.HKV}, Lq={w.LQ}, d={w.D}, ctx={w.N}, b={w.BITS}"
            f"{' + QJL sketch' if w.QJL else ''}, joint rounding, {keys}, bf16 V/q")


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return float(j.get("hbm_gbs", 6650.0)), "measured"
    return 6650.0, "fallback"


def unit_bytes(w: Workload, words: int) -> int:
    """Decode bytes of one (token, KV head): code words, gamma, bf16 V row (+ sketch words, residual norm)."""
    return 4 * words + 4 + 2 * w.D + ((4 * (w.D // 32) + 4) if w.QJL else 0)


def decode_bytes(w: Workload, words: int) -> int:
    units = w.B * w.HKV * w.N
    return units * unit_bytes(w, words) + w.B * w.HQ * w.LQ * w.D * (2 + 4)   # + q (bf16) + out (fp32)


def encode_bytes(w: Workload, words: int) -> int:
    per = 2 * w.D + 4 * words + 4 + ((4 * (w.D // 32) + 4) if w.QJL else 0)  # bf16 key in; codes, gamma (+ sketch) out
    return w.B * w.HKV * w.N * per


def _cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover - non-Linux
        return os.cpu_count() or 1


class ClockSampler:
    """Samples SM clocks and clock-event (throttle) reasons during the timed region.

    Polls NVML every ~1 ms from a thread; falls back to no samples if NVML is
    unavailable.
    """

    REASONS = {"hw_slowdown": "nvmlClocksEventReasonHwSlowdown",
               "hw_thermal_slowdown": "nvmlClocksEventReasonHwThermalSlowdown",
               "sw_thermal_slowdown": "nvmlClocksEventReasonSwThermalSlowdown",
               "sw_power_cap": "nvmlClocksEventReasonSwPowerCap",
               "hw_power_brake": "nvmlClocksEventReasonHwPowerBrakeSlowdown"}

    def __init__(self, torch_index: int):
        self.torch_index = torch_index
        self.samples = []
        self.stop = threading.Event()
        self.handle = None
        self.nv = None

    def _handle(self):
        import pynvml as nv
        import torch
        nv.nvmlInit()
        self.nv = nv
        try:
            p = torch.cuda.get_device_properties(self.torch_index)
            bus = f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
            return nv.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
            idx = int(vis.split(",")[self.torch_index]) if vis and vis.split(",")[0].isdigit() else self.torch_index
            return nv.nvmlDeviceGetHandleByIndex(idx)

    def _run(self):
        nv = self.nv
        while not self.stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM)
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
                self.samples.append((sm, r))
            except Exception:
                pass
            time.sleep(0.001)

    def __enter__(self):
        try:
            self.handle = self._handle()
            self.max_mhz = self.nv.nvmlDeviceGetMaxClockInfo(self.handle, self.nv.NVML_CLOCK_SM)
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
            time.sleep(0.005)
        except Exception:
            self.handle = None
        return self

    def __exit__(self, *exc):
        if self.handle is not None:
            self.stop.set()
            self.t.join(timeout=2)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        reasons = set()
        for _, r in self.samples:
            for name, attr in self.REASONS.items():
                bit = getattr(self.nv, attr, 0)
                if bit and (r & bit):
                    reasons.add(name)
        return {"sm_mhz": float(np.median([s for s, _ in self.samples])), "sm_max_mhz": float(self.max_mhz),
                "reasons": sorted(reasons), "samples": len(self.samples), "source": "nvml"}


# ------------------------------------------------------------------ ranks
def _dist_init():
    import torch
    import torch.distributed as dist
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1 and not dist.is_initialized():
        import datetime
        dist.init_process_group("nccl" if torch.cuda.is_available() else "gloo",
                                timeout=datetime.timedelta(seconds=120))
    return ws, rank, local


def _max_over_ranks(x: float, ws: int) -> float:
    if ws == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def _finish_ranks(ws):
    if ws > 1:
        import torch.distributed as dist
        if dist.is_initialized():
            dist.destroy_process_group()


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def spawn_ranks(n: int, argv, timeout_s: float = 1800.0) -> int:
    """Start ``n`` ranks of this script (one process per GPU, rank r on GPU r)
    with the rendezvous on 127.0.0.1. Rank 0's output is passed through (it
    alone prints the JSON line); the others' output is discarded. Returns the
    largest exit code."""
    port = _free_port()
    procs = []
    for r in range(n):
        env = dict(os.environ, RANK=str(r), LOCAL_RANK=str(r), WORLD_SIZE=str(n), LOCAL_WORLD_SIZE=str(n),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        out = None if r == 0 else subprocess.DEVNULL
        procs.append(subprocess.Popen([sys.executable, os.path.join(ROOT, "bench.py"), *argv], env=env, stdout=out,
                                      cwd=ROOT))
    rc = 0
    deadline = time.time() + timeout_s
    for p in procs:
        try:
            rc = max(rc, p.wait(timeout=max(1.0, deadline - time.time())))
        except subprocess.TimeoutExpired:
            p.kill()
            rc = max(rc, 124)
    return rc


def run_dry(args):
    """The rank logic without the GPU (a CPU check of the N-rank path): every
    rank takes its own batch, reports a made-up duration, and rank 0 prints
    the line with the whole-job units and the max over ranks."""
    ws, rank, _ = _dist_init()
    units = HEADLINE.B * HEADLINE.HKV * HEADLINE.N
    my_ms = 10.0 * (rank + 1)
    _barrier(ws)
    worst = _max_over_ranks(my_ms, ws)
    seeds = [SEED + 1000 * r for r in range(ws)]
    if rank == 0:
        print(json.dumps({"metric": METRIC, "dry_run": True, "n_gpus": ws, "value": ws * units / worst,
                          "unit": "units/ms", "max_ms": worst, "scaling": "weak",
                          "config": {"workload": describe(HEADLINE), "per_rank_seeds": seeds,
                                     "per_rank": "independent batch per GPU (no collective)"}}))
    _finish_ranks(ws)
    return 0


# ------------------------------------------------------------------ CPU oracle
def _oracle_head(job):
    """Oracle encode + decode attention of one KV head (runs in a worker)."""
    w, head, tokens, seed, one_thread = job
    if one_thread:  # a pool worker: one BLAS thread per process
        try:
            from threadpoolctl import threadpool_limits
            threadpool_limits(1)
        except Exception:
            pass
    from oracle import attention, codec, tables
    from rotation_preconditioned_quantization_b200 import inputs
    g = w.HQ // w.HKV
    tb = tables.as_f32(*tables.codebooks(w.D, w.BITS))
    lay = codec.Layout(w.D, w.BITS)
    signs = tables.rotation_signs(SEED, w.D, w.HKV)[head % w.HKV]
    S = tables.qjl_matrix(SEED + 0x517CC1, w.D, w.HKV)[head % w.HKV] if w.QJL else None
    if w.keys == "llm":
        keys = inputs.to_bf16(inputs.llm_keys(seed + 1, 1, tokens, w.D))[0]
    else:
        keys = inputs.to_bf16(inputs.gaussian_keys(seed + 1, 1, tokens, w.D))[0]
    V = inputs.to_bf16(inputs.normal(seed + 3, (tokens, w.D)))
    q = inputs.to_bf16(inputs.normal(seed + 2, (g * w.LQ, w.D)))
    t0 = time.perf_counter()
    e = codec.encode(keys.astype(np.float64), signs, tb, lay)
    qjl = None
    if w.QJL:
        uh = codec.decode_rotated(e.i_xi, e.i_eta, e.i_rho, tb, lay)
        bits, nu, _ = codec.qjl_encode(e.u_rot, uh, S)
        qjl = (bits, np.float32(nu).astype(np.float64), S)
    t1 = time.perf_counter()
    attention.decode_attention(q.astype(np.float64), e.gamma, e.i_xi, e.i_eta, e.i_rho, V.astype(np.float64), signs,
                               tb, lay, qjl=qjl)
    t2 = time.perf_counter()
    return t0, t1, t2  # CLOCK_MONOTONIC: comparable across the pool's processes


def cpu_baseline(w: Workload = HEADLINE, heads: int = 1, tokens: int = 8192, pool: int = 0):
    """Time the CPU oracle on a bounded sample of workload ``w``: oracle encode
    (+ sketch) and decode attention of ``heads`` KV heads (their query heads)
    over ``tokens`` tokens each. With ``pool`` > 0 the heads run in a process
    pool of that many workers (spawned: the caller may hold a CUDA context)."""
    from oracle import codec

    lay = codec.Layout(w.D, w.BITS)
    jobs = [(w, h, tokens, SEED + 101 * h, pool > 0) for h in range(heads)]
    if pool > 0:
        import multiprocessing as mp
        with mp.get_context("spawn").Pool(pool) as p:
            res = p.map(_oracle_head, jobs)
    else:
        res = [_oracle_head(j) for j in jobs]
    enc_s = float(sum(r[1] - r[0] for r in res))
    dec_s = float(sum(r[2] - r[1] for r in res))
    per = unit_bytes(w, lay.words)
    dec_bytes = heads * tokens * per + heads * (w.HQ // w.HKV) * w.LQ * w.D * 6
    if pool > 0:
        # the pool's span from the first encode start to the last decode end
        # (worker start-up and table set-up excluded), split in the ratio of
        # the summed encode and decode times
        span = max(r[2] for r in res) - min(r[0] for r in res)
        enc_s, dec_s = span * enc_s / (enc_s + dec_s), span * dec_s / (enc_s + dec_s)
    try:
        from threadpoolctl import threadpool_info
        blas = max([int(i.get("num_threads", 1)) for i in threadpool_info()] + [1])
    except Exception:
        blas = 1
    cores = _cores()
    used = min(pool, cores) if pool > 0 else min(blas, cores)
    return {
        "value": dec_bytes / dec_s / 1e9, "unit": "GB/s",
        "cores": used,
        "kind": "oracle",
        "sample": (f"{heads} KV head(s) x {tokens} tokens of {describe(w)}; oracle float64 numpy, "
                   + (f"{pool}-process pool (one head per task, one BLAS thread each) on {cores} affinity cores"
                      if pool > 0 else f"one process, {used} BLAS thread(s) on {cores} affinity cores")),
        "encode_mkeys_per_s": heads * tokens / enc_s / 1e6,
        "encode_s": enc_s, "decode_s": dec_s,
    }


def run_reference(args):
    # the oracle runs on rank 0 alone; it needs no process group
    if int(os.environ.get("RANK", "0")) != 0:
        return 0
    w, tokens = HEADLINE, 4096
    steps = []
    for i in range(args.warmup + args.steps):
        r = cpu_baseline(w, 1, tokens)
        if i >= args.warmup:
            steps.append(r)
    dec_s = float(np.mean([s["decode_s"] for s in steps]))
    enc_s = float(np.mean([s["encode_s"] for s in steps]))
    val = float(np.mean([s["value"] for s in steps]))
    line = {
        "impl": "reference", "metric": METRIC, "value": val,
        "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * (dec_s + enc_s), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic",
        "config": {"workload": describe(w), "sample": f"1 KV head x {tokens} tokens per step"},
        "encode_mkeys_per_s": float(np.mean([s["encode_mkeys_per_s"] for s in steps])),
        "cpu_baseline": {"value": val, "unit": "GB/s", "cores": steps[0]["cores"], "kind": "oracle",
                         "sample": steps[0]["sample"]},
        "e2e": {"value": val, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


# ------------------------------------------------------------------ GPU workloads
def setup(w: Workload, dev, seed: int, n_caches: int = 1, batch: int | None = None):
    """Device inputs of workload ``w`` (optionally another batch size): tables,
    keys, V, queries, ``n_caches`` empty caches, an output and a workspace."""
    import torch
    from rotation_preconditioned_quantization_b200 import api, inputs

    B = w.B if not batch else batch
    H = B * w.HKV
    lay = api.Layout(w.D, w.BITS, qjl=w.QJL)
    tabs = api.DeviceTables.build(lay, SEED, w.HKV, device=dev)
    if w.keys == "llm":
        keys = inputs.device_llm_keys(seed + 1, H, w.N, w.D, dev)
    else:
        keys = inputs.device_normal(seed + 1, (H, w.N, w.D), dev)
    V = inputs.device_normal(seed + 3, (H, w.N, w.D), dev)
    q = inputs.device_normal(seed + 2, (B, w.HQ, w.LQ, w.D), dev)
    caches = [api.Cache.empty(lay, H, w.N, dev) for _ in range(n_caches)]
    out = torch.empty((B, w.HQ, w.LQ, w.D), dtype=torch.float32, device=dev)
    wsp = api.Workspace(api.decode_attn_workspace_bytes(lay, B, w.HQ, w.HKV, w.LQ, w.N), dev)
    return dict(lay=lay, tabs=tabs, keys=keys, V=V, q=q, caches=caches, out=out, wsp=wsp, B=B)


def time_decode_flushed(w: Workload, dev, peak, iters: int = 6, batch: int | None = None):
    """Decode of workload ``w`` over a cache the encoder wrote from keys of its
    recipe; L2 flushed (512 MB written) before every timed call."""
    import torch
    from rotation_preconditioned_quantization_b200 import api

    s = setup(w, dev, SEED + 77, batch=batch)
    lay, cache = s["lay"], s["caches"][0]
    flush = torch.empty(512 * 1024 * 1024 // 4, device=dev)
    # the encode of the workload's keys (prefill into an empty cache), timed the same way
    te = []
    for i in range(iters + 2):
        flush.fill_(float(i))
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        api.encode(lay, s["tabs"], s["keys"], cache, 0)
        e1.record()
        torch.cuda.synchronize(dev)
        if i >= 2:
            te.append(e0.elapsed_time(e1))
    del s["keys"]
    ts = []
    for i in range(iters + 2):
        flush.fill_(float(i))
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        api.decode_attn(lay, s["tabs"], s["q"], cache, s["V"], w.HKV, out=s["out"], workspace=s["wsp"])
        e1.record()
        torch.cuda.synchronize(dev)
        if i >= 2:
            ts.append(e0.elapsed_time(e1))
    assert s["wsp"].status() == 0, "a bounded on-chip wait of the decode kernel expired"
    wb = w._replace(B=s["B"])
    nbytes = decode_bytes(wb, lay.words)
    ms = float(np.mean(ts))
    gbs = nbytes / (ms * 1e-3) / 1e9
    ems = float(np.mean(te))
    units = s["B"] * w.HKV * w.N
    return {"GB/s": gbs, "frac": gbs / peak, "ms": ms, "ms_min": float(np.min(ts)), "MB": nbytes / 1e6,
            "cache": "encoded by octo_encode", "l2": "flushed (512 MB written) before each call",
            "kernel": "tensor-core" if w.D <= 128 else "ffma",
            "encode": {"Mkeys/s": units / (ems * 1e-3) / 1e6, "ms": ems, "ms_min": float(np.min(te)),
                       "hbm_frac": encode_bytes(wb, lay.words) / (ems * 1e-3) / 1e9 / peak}}


def dequant_workload(dev, peak, iters=6):
    """octo_dequant (key reconstruction) of an LLM decode cache (8 KV heads x
    32768 tokens, d=128, b=3) into fp32 and bf16 rows. Algorithmic bytes per
    key: 4W + 4 read, 4d or 2d written."""
    import torch
    from rotation_preconditioned_quantization_b200 import api

    w = LLM_DECODE
    s = setup(w, dev, SEED + 5)
    lay, cache = s["lay"], s["caches"][0]
    api.encode(lay, s["tabs"], s["keys"], cache, 0)
    H, N, D = w.B * w.HKV, w.N, w.D
    flush = torch.empty(512 * 1024 * 1024 // 4, device=dev)  # > L2 between timed calls
    out = {}
    for name, dt, esz in (("f32", torch.float32, 4), ("bf16", torch.bfloat16, 2)):
        o = torch.empty((H, N, D), dtype=dt, device=dev)
        ts = []
        for i in range(iters + 2):
            flush.fill_(float(i))
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            api.dequant(lay, s["tabs"], cache, out=o)
            e1.record()
            torch.cuda.synchronize(dev)
            if i >= 2:
                ts.append(e0.elapsed_time(e1))
        nbytes = H * N * (4 * lay.words + 4 + esz * D)
        ms = float(np.mean(ts))
        gbs = nbytes / (ms * 1e-3) / 1e9
        out[name] = {"GB/s": gbs, "frac": gbs / peak, "ms": ms, "MB": nbytes / 1e6, "Mkeys/s": H * N / (ms * 1e-3) / 1e6}
    return out


def encode_sweep(dev, peak):
    """Encode throughput sweep: 2^22 fp32 keys ~ N(0,1) (8 heads x 2^19 tokens)
    streamed into the cache in appends of n ~ U{1..4096} tokens (one encode
    launch per append, all heads), for d in {64, 128, 256} x b in {2, 3, 4}.
    Keys are resident on the device; the time is the whole stream (CUDA
    events), launch gaps included. "Mkeys/s" replays the append stream as
    one CUDA graph (the GPU-side rate); "Mkeys/s_eager" issues the appends
    one by one from Python, whose per-call overhead then dominates."""
    import torch
    from rotation_preconditioned_quantization_b200 import api, inputs

    H, N = 8, 1 << 19
    lens = inputs.append_lengths(SEED + 17, N, 1, 4096)
    out = {}
    for d in (64, 128, 256):
        keys = torch.empty((H, N, d), dtype=torch.float32, device=dev)
        keys.normal_(generator=torch.Generator(device=dev).manual_seed(SEED + d))
        for b in (2, 3, 4):
            lay = api.Layout(d, b)
            tabs = api.DeviceTables.build(lay, SEED, H, device=dev)
            cache = api.Cache.empty(lay, H, N, dev)

            def stream_appends():
                cache.length = 0
                for n in lens:
                    s = cache.length
                    api.encode(lay, tabs, keys[:, s:s + n], cache)

            def timed(fn):
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record()
                fn()
                e1.record()
                torch.cuda.synchronize(dev)
                return e0.elapsed_time(e1)

            timed(stream_appends)  # warm-up (also fills the launch caches)
            ms_eager = timed(stream_appends)
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                stream_appends()
            graph.replay()
            torch.cuda.synchronize(dev)
            ms = timed(graph.replay)
            nbytes = H * N * (4 * d + 4 * lay.words + 4)
            out[f"d{d}_b{b}"] = {"Mkeys/s": H * N / (ms * 1e-3) / 1e6, "ms": ms, "appends": len(lens),
                                 "hbm_frac": nbytes / (ms * 1e-3) / 1e9 / peak,
                                 "Mkeys/s_eager": H * N / (ms_eager * 1e-3) / 1e6}
            del graph, cache
        del keys
    return out


def run_gpu(args):
    import torch
    from rotation_preconditioned_quantization_b200 import api

    ws, rank, local = _dist_init()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = HEADLINE
    seed = SEED + 1000 * rank  # an independent batch per rank
    s = setup(w, dev, seed, n_caches=2)
    lay, tabs, caches = s["lay"], s["tabs"], s["caches"]
    stream = torch.cuda.current_stream(dev)

    def step(i, ev=None):
        c_enc = caches[i % 2]
        c_dec = caches[(i - 1) % 2]
        if ev is not None:
            ev[0].record(stream)
        api.encode(lay, tabs, s["keys"], c_enc, 0)
        if ev is not None:
            ev[1].record(stream)
        api.decode_attn(lay, tabs, s["q"], c_dec, s["V"], w.HKV, kv_len=w.N, out=s["out"], workspace=s["wsp"])
        if ev is not None:
            ev[2].record(stream)

    # prime: both caches encoded once, then warm-up steps
    for c in caches:
        api.encode(lay, tabs, s["keys"], c, 0)
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize(dev)

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    _barrier(ws)
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        t_start.record(stream)
        for i in range(args.steps):
            step(args.warmup + i, evs[i])
        t_end.record(stream)
        torch.cuda.synchronize(dev)
    _barrier(ws)
    if s["wsp"].status() != 0:
        raise RuntimeError("a bounded on-chip wait of the decode kernel expired")
    total_ms = t_start.elapsed_time(t_end)
    enc_ms = [e[0].elapsed_time(e[1]) for e in evs]
    dec_ms = [e[1].elapsed_time(e[2]) for e in evs]
    # per step: encode, decode (+ the decode's query preparation for the sketch, d <= 128)
    launches = (3 if w.QJL and w.D <= 128 else 2) * args.steps

    total_ms_max = _max_over_ranks(total_ms, ws)
    dec_sum_max = _max_over_ranks(float(np.sum(dec_ms)), ws)
    enc_sum_max = _max_over_ranks(float(np.sum(enc_ms)), ws)
    dbytes = decode_bytes(w, lay.words)
    ebytes = encode_bytes(w, lay.words)
    units = w.B * w.HKV * w.N
    value = ws * dbytes * args.steps / (dec_sum_max * 1e-3) / 1e9
    enc_mkeys = ws * units * args.steps / (enc_sum_max * 1e-3) / 1e6

    # end to end through the public API from pinned host buffers: per step the
    # keys, V and queries go host -> device, then encode + decode, then the
    # output comes back. The copies run on their own stream into one of two
    # device input sets, so that step i + 1's inputs cross PCIe while step i
    # computes (the way a serving loop overlaps them); every step's copy is
    # inside the timed region.
    e2e_cache = caches[0]
    hk = s["keys"].cpu().pin_memory()
    hV = s["V"].cpu().pin_memory()
    hq = s["q"].cpu().pin_memory()
    hout = torch.empty_like(s["out"], device="cpu").pin_memory()
    sets = [(s["keys"], s["V"], s["q"]),
            (torch.empty_like(s["keys"]), torch.empty_like(s["V"]), torch.empty_like(s["q"]))]
    copy_stream = torch.cuda.Stream(dev)
    copied = [torch.cuda.Event() for _ in sets]
    freed = [torch.cuda.Event() for _ in sets]
    for ev in freed:
        ev.record(stream)

    def e2e_step(i):
        dk, dV, dq = sets[i % 2]
        with torch.cuda.stream(copy_stream):
            copy_stream.wait_event(freed[i % 2])  # the step that last read this set has finished
            dk.copy_(hk, non_blocking=True)
            dV.copy_(hV, non_blocking=True)
            dq.copy_(hq, non_blocking=True)
            copied[i % 2].record(copy_stream)
        stream.wait_event(copied[i % 2])
        api.encode(lay, tabs, dk, e2e_cache, 0)
        api.decode_attn(lay, tabs, dq, e2e_cache, dV, w.HKV, kv_len=w.N, out=s["out"], workspace=s["wsp"])
        freed[i % 2].record(stream)
        hout.copy_(s["out"], non_blocking=True)

    e2e_steps = max(1, min(args.steps, 10))
    for i in range(max(1, min(args.warmup, 3))):
        e2e_step(i)
    torch.cuda.synchronize(dev)
    _barrier(ws)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for ev in freed:  # no copy of the timed steps starts before e0
        ev.record(stream)
    for i in range(e2e_steps):
        e2e_step(i)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = _max_over_ranks(e0.elapsed_time(e1), ws)
    h2d = hk.numel() * 2 + hV.numel() * 2 + hq.numel() * 2
    d2h = hout.numel() * 4
    e2e_val = ws * dbytes * e2e_steps / (e2e_ms * 1e-3) / 1e9
    del hk, hV, sets

    peak, peak_kind = _peaks()
    dec_avg_s = float(np.mean(dec_ms)) * 1e-3
    achieved = dbytes / dec_avg_s / 1e9
    traffic = _ncu_traffic()
    if rank != 0:  # every collective is behind us; rank 0 alone reports
        _finish_ranks(ws)
        return 0
    del s
    torch.cuda.empty_cache()
    extra = None if args.no_extra else {describe(o): time_decode_flushed(o, dev, peak) for o in OTHER_WORKLOADS}
    dq = None if args.no_extra else dequant_workload(dev, peak)
    sweep = None if args.no_extra else encode_sweep(dev, peak)
    line = {
        "metric": METRIC,
        "value": value, "unit": "GB/s", "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": total_ms_max / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": describe(w), "per_rank": "independent batch per GPU (no collective)",
                   "l2": "inputs larger than L2: each decode reads 2.95 GB of cache + V, encoded one step earlier "
                         "into the other of two caches (the other cache's encode in between)"},
        "encode_mkeys_per_s": enc_mkeys,
        "encode_ms": float(np.mean(enc_ms)), "decode_ms": float(np.mean(dec_ms)),
        "decode_ms_min": float(np.min(dec_ms)),
        "decode_bytes_per_step": dbytes, "encode_bytes_per_step": ebytes,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic, "kernel": "octo_decode_attn (decode_tc_kernel<128,4,4,QJL>)",
                     "peak_source": f"{peak_kind} hbm_gbs (MEASURED_PEAKS.json)" if peak_kind == "measured" else "fallback 6650 GB/s",
                     "algorithmic_bytes": "per (token, KV head) 4W + 4 + 2d + 4d/32 + 4 = 352 B (W = 18), x 8.39 M units, + q + out"},
        "encode_roofline": {"bound": "alu", "hbm_achieved": ebytes / (float(np.mean(enc_ms)) * 1e-3) / 1e9,
                            "hbm_peak": peak, "unit": "GB/s",
                            "hbm_frac": ebytes / (float(np.mean(enc_ms)) * 1e-3) / 1e9 / peak},
        "e2e": {"value": e2e_val, "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e2e_ms / e2e_steps, "steps": e2e_steps,
                "method": "public API from pinned host memory; step i+1's host-to-device copy on a second stream "
                          "overlaps step i's encode + decode (two device input sets)"},
        "gpu_launches": launches,
        "other_workloads": extra,
        "dequant": dq,
        "encode_sweep": sweep,
        "clocks": clk.summary(),
    }
    if not args.no_cpu_baseline and ws == 1:
        one = cpu_baseline(w, 1, 8192)
        pool_n = min(_cores(), 8)
        many = cpu_baseline(w, pool_n, 8192, pool=pool_n)
        line["cpu_baseline"] = {k: v for k, v in many.items() if k not in ("encode_s", "decode_s")}
        line["cpu_baseline"]["single_process"] = {k: v for k, v in one.items() if k not in ("encode_s", "decode_s")}
    print(json.dumps(line))
    _finish_ranks(ws)
    return 0


DECODE_KERNEL_SOURCES = ("octo_common.cuh", "octo_decode_kernel.cuh", "octo_decode.cu")
DECODE_PROFILE = os.path.join(ROOT, "profiles", "decode_tc_kernel_qjl_long_context_h32x8_d128_ctx131072_b4qjl.md")


def _code_tokens(src: str) -> str:
    """C/C++/CUDA source with its comments removed and whitespace runs collapsed
    (string and character literals kept as they are)."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c in "\"'":
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def kernel_sources_digest(names=DECODE_KERNEL_SOURCES) -> str:
    """sha256 over the decode kernel's sources without their comments (detects
    a kernel changed since its ncu capture; a comment edit does not count)."""
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "rotation_preconditioned_quantization_b200", "csrc", n)) as f:
            h.update(_code_tokens(f.read()).encode())
    return h.hexdigest()


def _ncu_traffic():
    """DRAM bytes per headline decode launch from the committed ncu summary
    (captured on a smaller batch and scaled by the units processed), or None
    when the summary is missing or was taken on other kernel sources."""
    try:
        with open(DECODE_PROFILE) as f:
            text = f.read()
    except OSError:
        return None
    t = re.search(r"^traffic_bytes_per_launch:\s*(\d+)", text, re.M)
    d = re.search(r"^kernel_sources_sha256:\s*([0-9a-f]{64})", text, re.M)
    if not t or not d or d.group(1) != kernel_sources_digest():
        return None
    return int(t.group(1))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="octopus", choices=["octopus", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true", help="skip the other workloads, dequant and the encode sweep")
    ap.add_argument("--dry-run", action="store_true", help="rank logic only, no GPU (a CPU check of --gpus N)")
    ap.add_argument("--only", choices=["dequant", "encode_sweep", "decode_shape"],
                    help="time only this part (one GPU; prints its JSON)")
    ap.add_argument("--shape", default=HEADLINE.name,
                    help="with --only decode_shape: the decode workload to time (name prefix)")
    ap.add_argument("--batch", type=int, default=0,
                    help="with --only decode_shape: replace the workload's batch size (a smaller case to profile)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        return spawn_ranks(args.gpus, sys.argv[1:])
    if args.dry_run:
        return run_dry(args)
    if args.only:
        import torch

        dev = torch.device("cuda", 0)
        torch.cuda.set_device(dev)
        peak = _peaks()[0]
        if args.only == "dequant":
            print(json.dumps({"dequant": dequant_workload(dev, peak)}))
        elif args.only == "encode_sweep":
            print(json.dumps({"encode_sweep": encode_sweep(dev, peak)}))
        else:
            known = (HEADLINE, *OTHER_WORKLOADS)
            shapes = [w for w in known if w.name == args.shape] or [w for w in known if w.name.startswith(args.shape)]
            if len(shapes) != 1:
                raise SystemExit(f"--shape {args.shape!r} names {len(shapes)} workloads")
            w = shapes[0]
            b = args.batch if args.batch > 0 else None
            print(json.dumps({"decode_shape": {describe(w._replace(B=b or w.B)): time_decode_flushed(w, dev, peak,
                                                                                                        batch=b)}}))
        return 0
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
