"""Benchmark of the OCTOPUS codec on B200: encode + fused decode attention.

Workload (one GPU): LLM-shaped decode - batch 1, 32 query heads over 8 KV
heads (GQA 4), head_dim 128, context 32768, bf16 keys (N(0,1), four outlier
channels x10, per-token lognormal(0, 0.5) scale), bf16 V and q ~ N(0,1),
b = 3, joint rounding. One step = encode the prefill cache (8 x 32768 keys)
+ one fused decode-attention step (32 query heads over the whole cache).

Timing: CUDA events on the launching stream around each kernel; the step
loop is bracketed by a barrier and a device synchronize; the max over ranks
is reported. L2 (126 MB): inputs rotate over 3 independent copies of the
workload (~150 MB each) and each step decodes the cache that the previous
step encoded, so no decode input was touched within the last ~150 MB of
traffic. Primary metric: decode-attention achieved HBM GB/s over the
algorithmic bytes (packed codes + gamma + bf16 V + q + out); encode is
reported in Mkeys/s.

``--impl reference`` times the CPU oracle (the plain float64 restatement of
the method) on a bounded sample of the same workload instead.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

# workload
B, HQ, HKV, D, N, BITS = 1, 32, 8, 128, 32768, 3
SEED = 0
METRIC = "compressed-KV decode-attention HBM GB/s (% of ~8 TB/s); encode Mkeys/s"
WORKLOAD = "llm-decode: B=1, Hq=32, Hkv=8 (GQA 4), d=128, ctx=32768, bf16 K/V/q, b=3 joint"


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return float(j.get("hbm_gbs", 6650.0)), "measured"
    return 6650.0, "fallback"


def _bytes_decode(words):
    units = B * HKV * N
    per_unit = 4 * words + 4 + 2 * D            # packed words + gamma + bf16 V row
    return units * per_unit + B * HQ * D * 2 + B * HQ * D * 4   # + q (bf16) + out (fp32)


def _bytes_encode(words):
    return B * HKV * N * (2 * D + 4 * words + 4)


class ClockSampler:
    """Samples SM clocks and clock-event (throttle) reasons during the timed region.

    Polls NVML every ~1 ms from a thread (the timed region is only tens of
    milliseconds); falls back to no samples if NVML is unavailable.
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


def cpu_baseline(kv_heads: int = 1, tokens: int = N):
    """Time the CPU oracle on a bounded sample: oracle encode + decode attention of
    ``kv_heads`` KV heads (4 query heads each) over ``tokens`` tokens."""
    from oracle import attention, codec, tables
    from rotation_preconditioned_quantization_b200 import inputs
    try:
        from threadpoolctl import threadpool_info
        cores = max([int(i.get("num_threads", 1)) for i in threadpool_info()] + [1])
    except Exception:
        cores = os.cpu_count() or 1
    tb = tables.as_f32(*tables.codebooks(D, BITS))
    lay = codec.Layout(D, BITS)
    signs = tables.rotation_signs(SEED, D, HKV)
    keys = inputs.to_bf16(inputs.llm_keys(SEED + 1, kv_heads, tokens, D))
    V = inputs.to_bf16(inputs.normal(SEED + 3, (kv_heads, tokens, D)))
    q = inputs.to_bf16(inputs.normal(SEED + 2, (kv_heads, HQ // HKV, D)))
    t0 = time.perf_counter()
    encs = [codec.encode(keys[h].astype(np.float64), signs[h], tb, lay) for h in range(kv_heads)]
    t1 = time.perf_counter()
    for h in range(kv_heads):
        e = encs[h]
        attention.decode_attention(q[h].astype(np.float64), e.gamma, e.i_xi, e.i_eta, e.i_rho,
                                   V[h].astype(np.float64), signs[h], tb, lay)
    t2 = time.perf_counter()
    per_unit = 4 * lay.words + 4 + 2 * D
    dec_bytes = kv_heads * tokens * per_unit + kv_heads * (HQ // HKV) * D * 6
    return {
        "value": dec_bytes / (t2 - t1) / 1e9, "unit": "GB/s", "cores": cores, "kind": "oracle",
        "sample": f"{kv_heads} KV head(s) x {tokens} tokens (of {HKV} x {N}); oracle float64 numpy",
        "encode_mkeys_per_s": kv_heads * tokens / (t1 - t0) / 1e6,
        "encode_s": t1 - t0, "decode_s": t2 - t1,
    }


def run_reference(args):
    # the oracle runs on rank 0 alone; it needs no process group
    if int(os.environ.get("RANK", "0")) != 0:
        return 0
    tokens = 4096
    steps = []
    for i in range(args.warmup + args.steps):
        r = cpu_baseline(1, tokens)
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
        "config": {"workload": WORKLOAD, "sample": f"1 KV head x {tokens} tokens per step"},
        "encode_mkeys_per_s": float(np.mean([s["encode_mkeys_per_s"] for s in steps])),
        "cpu_baseline": {"value": val, "unit": "GB/s", "cores": steps[0]["cores"], "kind": "oracle",
                         "sample": steps[0]["sample"]},
        "e2e": {"value": val, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


# Decode throughput on the other workload shapes (reported next to the main
# metric). Codes, gammas, sketches, V and queries are drawn on the device:
# the decode's work and traffic do not depend on their values.
OTHER_WORKLOADS = (
    ("video_audio: B=1, 16/16 heads, d=64, ctx=65536, b=2, 8 query tokens", 1, 16, 16, 8, 64, 2, 65536, False),
    ("qjl_long_context: B=8, 32/8 heads, d=128, ctx=131072, b=4 + QJL sketch", 8, 32, 8, 1, 128, 4, 131072, True),
    ("llm_decode_large: B=8, 32/8 heads, d=128, ctx=131072, b=3", 8, 32, 8, 1, 128, 3, 131072, False),
)


def other_workloads(dev, peak, iters=6, shapes=OTHER_WORKLOADS):
    import torch
    from rotation_preconditioned_quantization_b200 import api

    out = {}
    flush = torch.empty(512 * 1024 * 1024 // 4, device=dev)  # > L2 between timed calls
    for name, B_, HQ_, HKV_, LQ_, D_, BITS_, N_, qjl in shapes:
        lay = api.Layout(D_, BITS_, qjl=qjl)
        H = B_ * HKV_
        tabs = api.DeviceTables.build(lay, SEED, HKV_, device=dev)
        g = torch.Generator(device=dev).manual_seed(SEED)
        cache = api.Cache.empty(lay, H, N_, dev)
        cache.packed.random_(generator=g)
        cache.gamma.uniform_(0.5, 2.0, generator=g)
        if qjl:
            cache.qjl_bits.random_(generator=g)
            cache.qjl_norm.uniform_(0.0, 0.3, generator=g)
        cache.length = N_
        V = torch.randn((H, N_, D_), device=dev, generator=g).to(torch.bfloat16)
        q = torch.randn((B_, HQ_, LQ_, D_), device=dev, generator=g).to(torch.bfloat16)
        o = torch.empty((B_, HQ_, LQ_, D_), device=dev)
        wsp = api.Workspace(api.decode_attn_workspace_bytes(lay, B_, HQ_, HKV_, LQ_, N_), dev)
        ts = []
        for i in range(iters + 2):
            flush.sum()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            api.decode_attn(lay, tabs, q, cache, V, HKV_, out=o, workspace=wsp)
            e1.record()
            torch.cuda.synchronize(dev)
            if i >= 2:
                ts.append(e0.elapsed_time(e1))
        unit = 4 * lay.words + 4 + 2 * D_ + (4 * (D_ // 32) + 4 if qjl else 0)
        nbytes = H * N_ * unit
        ms = float(np.mean(ts))
        gbs = nbytes / (ms * 1e-3) / 1e9
        out[name] = {"GB/s": gbs, "frac": gbs / peak, "ms": ms, "MB": nbytes / 1e6,
                     "kernel": "tensor-core" if D_ <= 128 else "ffma"}
        del cache, V
    return out


def dequant_workload(dev, peak, iters=6):
    """octo_dequant (key reconstruction) of the bench workload's cache
    (8 KV heads x 32768 tokens, d=128, b=3) into fp32 and bf16 rows.
    Algorithmic bytes per key: 4W + 4 read, 4d or 2d written."""
    import torch
    from rotation_preconditioned_quantization_b200 import api

    lay = api.Layout(D, BITS)
    H = B * HKV
    tabs = api.DeviceTables.build(lay, SEED, HKV, device=dev)
    g = torch.Generator(device=dev).manual_seed(SEED + 5)
    cache = api.Cache.empty(lay, H, N, dev)
    cache.packed.random_(generator=g)
    cache.gamma.uniform_(0.5, 2.0, generator=g)
    cache.length = N
    flush = torch.empty(512 * 1024 * 1024 // 4, device=dev)  # > L2 between timed calls
    out = {}
    for name, dt, esz in (("f32", torch.float32, 4), ("bf16", torch.bfloat16, 2)):
        o = torch.empty((H, N, D), dtype=dt, device=dev)
        ts = []
        for i in range(iters + 2):
            flush.sum()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            api.dequant(lay, tabs, cache, out=o)
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
    from rotation_preconditioned_quantization_b200 import api, inputs

    ws, rank, local = _dist_init()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    lay = api.Layout(D, BITS)
    tabs = api.DeviceTables.build(lay, SEED, HKV, device=dev)
    n_copies = 3

    # inputs: distinct per copy and per rank
    def make(copy):
        s = SEED + 1000 * rank + 10 * copy
        keys = torch.from_numpy(inputs.llm_keys(s + 1, B * HKV, N, D)).to(torch.bfloat16)
        V = torch.from_numpy(inputs.normal(s + 3, (B * HKV, N, D))).to(torch.bfloat16)
        q = torch.from_numpy(inputs.normal(s + 2, (B, HQ, 1, D))).to(torch.bfloat16)
        return keys, V, q

    host = [make(c) for c in range(n_copies)]
    devc = []
    for keys, V, q in host:
        devc.append(dict(keys=keys.to(dev), V=V.to(dev), q=q.to(dev), cache=api.Cache.empty(lay, B * HKV, N, dev),
                         out=torch.empty((B, HQ, 1, D), dtype=torch.float32, device=dev)))
    wsp = api.Workspace(api.decode_attn_workspace_bytes(lay, B, HQ, HKV, 1, N), dev)
    stream = torch.cuda.current_stream(dev)

    def step(i, ev=None):
        c_enc = devc[i % n_copies]
        c_dec = devc[(i - 1) % n_copies]
        if ev is not None:
            ev[0].record(stream)
        api.encode(lay, tabs, c_enc["keys"], c_enc["cache"], 0)
        if ev is not None:
            ev[1].record(stream)
        api.decode_attn(lay, tabs, c_dec["q"], c_dec["cache"], c_dec["V"], HKV, kv_len=N, out=c_dec["out"],
                        workspace=wsp)
        if ev is not None:
            ev[2].record(stream)

    # prime: every copy's cache encoded once, then warm-up steps
    for c in range(n_copies):
        api.encode(lay, tabs, devc[c]["keys"], devc[c]["cache"], 0)
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
    total_ms = t_start.elapsed_time(t_end)
    enc_ms = [e[0].elapsed_time(e[1]) for e in evs]
    dec_ms = [e[1].elapsed_time(e[2]) for e in evs]
    launches = 2 * args.steps

    total_ms_max = _max_over_ranks(total_ms, ws)
    dec_sum_max = _max_over_ranks(float(np.sum(dec_ms)), ws)
    enc_sum_max = _max_over_ranks(float(np.sum(enc_ms)), ws)
    dbytes = _bytes_decode(lay.words)
    ebytes = _bytes_encode(lay.words)
    value = ws * dbytes * args.steps / (dec_sum_max * 1e-3) / 1e9
    enc_mkeys = ws * B * HKV * N * args.steps / (enc_sum_max * 1e-3) / 1e6

    # end to end through the public API from pinned host buffers
    hk, hV, hq = (t.pin_memory() for t in host[0])
    hout = torch.empty((B, HQ, 1, D), dtype=torch.float32).pin_memory()
    e2e_cache = api.Cache.empty(lay, B * HKV, N, dev)
    dk = torch.empty_like(hk, device=dev)
    dV = torch.empty_like(hV, device=dev)
    dq = torch.empty_like(hq, device=dev)
    dout = torch.empty((B, HQ, 1, D), dtype=torch.float32, device=dev)

    def e2e_step():
        dk.copy_(hk, non_blocking=True)
        dV.copy_(hV, non_blocking=True)
        dq.copy_(hq, non_blocking=True)
        api.encode(lay, tabs, dk, e2e_cache, 0)
        api.decode_attn(lay, tabs, dq, e2e_cache, dV, HKV, kv_len=N, out=dout, workspace=wsp)
        hout.copy_(dout, non_blocking=True)

    for _ in range(max(1, args.warmup)):
        e2e_step()
    torch.cuda.synchronize(dev)
    _barrier(ws)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = _max_over_ranks(e0.elapsed_time(e1), ws)
    h2d = hk.numel() * 2 + hV.numel() * 2 + hq.numel() * 2
    d2h = hout.numel() * 4
    e2e_val = ws * dbytes * args.steps / (e2e_ms * 1e-3) / 1e9

    peak, peak_kind = _peaks()
    dec_avg_s = float(np.mean(dec_ms)) * 1e-3
    achieved = dbytes / dec_avg_s / 1e9
    traffic = _ncu_traffic()
    if rank != 0:  # every collective is behind us; rank 0 alone reports
        if ws > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return 0
    extra = None if args.no_extra else other_workloads(dev, peak)
    dq = None if args.no_extra else dequant_workload(dev, peak)
    sweep = None if args.no_extra else encode_sweep(dev, peak)
    line = {
        "metric": METRIC,
        "value": value, "unit": "GB/s", "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": total_ms_max / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": WORKLOAD, "per_rank": "independent batch per GPU (no collective)",
                   "l2": "3 rotating input copies (~150 MB each > 126 MB L2); decode reads the cache encoded one step earlier"},
        "encode_mkeys_per_s": enc_mkeys,
        "encode_ms": float(np.mean(enc_ms)), "decode_ms": float(np.mean(dec_ms)),
        "decode_bytes_per_step": dbytes, "encode_bytes_per_step": ebytes,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic, "kernel": "octo_decode_attn",
                     "peak_source": f"{peak_kind} hbm_gbs (MEASURED_PEAKS.json)" if peak_kind == "measured" else "fallback 6650 GB/s"},
        "encode_roofline": {"bound": "hbm", "achieved": ebytes / (float(np.mean(enc_ms)) * 1e-3) / 1e9, "peak": peak,
                            "unit": "GB/s", "frac": ebytes / (float(np.mean(enc_ms)) * 1e-3) / 1e9 / peak},
        "e2e": {"value": e2e_val, "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e2e_ms / args.steps},
        "gpu_launches": launches,
        "other_workloads": extra,
        "dequant": dq,
        "encode_sweep": sweep,
        "clocks": clk.summary(),
    }
    if not args.no_cpu_baseline and ws == 1:
        line["cpu_baseline"] = {k: v for k, v in cpu_baseline(1, N).items() if k not in ("encode_s", "decode_s")}
    print(json.dumps(line))
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


DECODE_KERNEL_SOURCES = ("octo_common.cuh", "octo_decode_kernel.cuh", "octo_decode.cu")
DECODE_PROFILE = os.path.join(ROOT, "profiles", "decode_tc_kernel_llm_decode_b1_h32x8_d128_ctx32768_b3.md")


def kernel_sources_digest(names=DECODE_KERNEL_SOURCES) -> str:
    """sha256 over the decode kernel's sources (detects a kernel changed since its ncu capture)."""
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "rotation_preconditioned_quantization_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def _ncu_traffic():
    """DRAM bytes per decode launch from the committed ncu summary, or None when
    the summary is missing or was taken on other kernel sources."""
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
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="octopus", choices=["octopus", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true", help="skip the decode timings of the other workload shapes")
    ap.add_argument("--only", choices=["dequant", "encode_sweep", "decode_shape"],
                    help="time only this part (one GPU; prints its JSON)")
    ap.add_argument("--shape", default="llm_decode_large",
                    help="with --only decode_shape: the other decode workload to time (name prefix)")
    ap.add_argument("--batch", type=int, default=0,
                    help="with --only decode_shape: replace the workload's batch size (a smaller case to profile)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    if args.only == "dequant":
        import torch

        dev = torch.device("cuda", 0)
        torch.cuda.set_device(dev)
        print(json.dumps({"dequant": dequant_workload(dev, _peaks()[0])}))
        return 0
    if args.only == "decode_shape":
        import torch

        dev = torch.device("cuda", 0)
        torch.cuda.set_device(dev)
        shapes = [w for w in OTHER_WORKLOADS if w[0].startswith(args.shape)]
        if len(shapes) != 1:
            raise SystemExit(f"--shape {args.shape!r} names {len(shapes)} workloads")
        w = list(shapes[0])
        if args.batch > 0 and args.batch != w[1]:
            w[0] = w[0].replace(f"B={w[1]},", f"B={args.batch},")
            w[1] = args.batch
        print(json.dumps({"decode_shape": other_workloads(dev, _peaks()[0], shapes=[tuple(w)])}))
        return 0
    if args.only == "encode_sweep":
        import torch

        dev = torch.device("cuda", 0)
        torch.cuda.set_device(dev)
        print(json.dumps({"encode_sweep": encode_sweep(dev, _peaks()[0])}))
        return 0
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
