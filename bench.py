#!/usr/bin/env python
"""Benchmark: KIVI 2-bit decode attention on B200.

One step = one decode step of one attention layer through the C ABI:
kivi_append_decode -- the new token's K/V into the residual window (the
window is flushed into the 2-bit store every R tokens, as its own launch)
and decode attention (fused dequant + q.K + online softmax + P.V over the
packed codes and the window, then the cross-split merge), one kernel launch
when no flush is due.  `--unfused` times kivi_append_token followed by
kivi_decode_attention instead (two launches per step).  The ragged workload
(per-sequence prompt lengths) times kivi_ragged_append_decode: the append
(each sequence flushing on its own) and the decode, two launches per step.

Headline workload: the Llama-2-13B-shaped layer (B=64, 40 heads, D=128,
context 8192, 2-bit, G=32, R=128; 2.81 GB of codes, scales and zeros per
decode call), the largest configuration that fits one GPU.  Beside it, under
"workloads", the Llama-2-7B layer, the Mistral-7B GQA layer, the streaming
workload's decode step and the 13B layer at 4 bits, each with its own rate
and roofline (headline and roofline passes only; `--no-extras` skips them).

L2 hygiene: `--layers` copies of the layer cache (default: enough for about
4 GB, at least two) are visited round-robin, so each step reads a cache that
is not L2-resident (inputs larger than the 126 MB L2).

Output: one JSON line (rank 0).  `value` = decode tokens/s over all ranks
(B tokens per step per rank) over K steps with nothing recorded between
launches; `roofline` = the decode kernel's algorithmic bytes / its CUDA-event
time vs measured HBM peak, from K further steps with events recorded around
each decode launch (events serialize consecutive launches, so this pass runs
apart from the headline one); `e2e` = the same loop with
the step's inputs copied from pinned host memory and the output copied back
inside the timed region (fused uniform steps: one `kivi_append_decode_host`
call per step, which does both copies); `cpu_baseline` = the CPU oracle on a bounded sample
of the same workload.  `--impl reference` times the CPU oracle alone.
Multi-GPU (torchrun): independent replicas, one per rank (no collective on
the data path); the barrier and max-over-ranks timing use torch.distributed.
"""
from __future__ import annotations

import argparse
import ctypes
import json
import math
import os
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from bit_asymmetric_kv_quantize_b200 import workloads as W  # noqa: E402

METRIC = "decode-attention tokens/s over 2-bit KV; achieved HBM GB/s vs B200 peak"
FALLBACK_HBM_GBS = 6650.0


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=4096)
    p.add_argument("--warmup", type=int, default=64)
    p.add_argument("--impl", choices=["kivi", "reference"], default="kivi")
    p.add_argument("--workload", default=W.LLAMA2_13B_2BIT.name, choices=sorted(W.ALL))
    p.add_argument("--layers", type=int, default=0,
                   help="layer caches visited round-robin (0: enough for ~4 GB, at least 2)")
    p.add_argument("--no-extras", action="store_true",
                   help="skip the other workloads reported beside the headline one")
    p.add_argument("--kernel", choices=["default", "simt"], default="default")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--unfused", action="store_true",
                   help="append and decode as two calls (kivi_append_token + decode)")
    p.add_argument("--cpu-budget-s", type=float, default=15.0)
    p.add_argument("--paged", choices=["shuffled", "sequential"], default=None,
                   help="ragged workloads: quantized store in pages of R tokens from a pool, "
                        "through a block table whose pages are shuffled over the pool or "
                        "consecutive per sequence")
    p.add_argument("--bits", type=int, choices=[1, 2, 3, 4], default=None,
                   help="code width other than the workload's (a format variant)")
    p.add_argument("--batch", type=int, default=None,
                   help="batch size other than the workload's (a smaller case of the same "
                        "kernel instance, e.g. for profiler captures)")
    p.add_argument("--outliers", default="0,0",
                   help="dense-and-sparse variant: entries kept exactly per key group and per "
                        "value group, 'k,v' (the inputs get 1%% spiked entries, x4)")
    p.add_argument("--meta", choices=["f32", "f16"], default="f32",
                   help="scale/zero storage: binary32, or the binary16 format variant "
                        "(fp16 workloads)")
    return p.parse_args()


DEFAULT_WORKLOAD = W.LLAMA2_13B_2BIT.name
# reported beside the headline, each with its own rate and roofline
EXTRA_WORKLOADS = (W.LLAMA2_7B.name, W.MISTRAL_7B.name, W.STREAMING.name, W.LLAMA2_13B_4BIT.name)


def bench_workload(args, name=None) -> W.Workload:
    """The workload named by --workload (or `name`) with the --meta storage;
    the streaming workload's decode loop is the step loop itself (steps = 0
    here)."""
    w = W.ALL[name or args.workload]
    if w.steps:
        w = w.with_(steps=0)
    if args.meta == "f16":
        w = w.with_(meta="f16", name=w.name + "-meta16")
    if getattr(args, "batch", None) and args.batch != w.B:
        w = w.with_(B=args.batch, name=f"{w.name}-batch{args.batch}")
    ko, vo = (int(x) for x in args.outliers.split(","))
    if ko or vo:
        w = w.with_(spike_frac=0.01, spike_scale=4.0, name=f"{w.name}-sparse{ko}x{vo}")
    if args.bits is not None and args.bits != w.bits:
        base = w.name[:-len("-2bit")] if w.name.endswith("-2bit") else w.name
        w = w.with_(bits=args.bits, name=f"{base}-{args.bits}bit")
    return w


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def max_over_ranks(value: float, world: int, device=None) -> float:
    """The largest `value` over all ranks (every rank gets it); identity for one rank."""
    if world <= 1:
        return value
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(world: int, batch: int, steps: int, ms_max: float) -> float:
    """Whole-job tokens/s of `world` independent replicas, each decoding `batch`
    sequences for `steps` steps, timed by the slowest rank."""
    return world * batch * steps / (ms_max * 1e-3)


def peak_hbm():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def profiled_traffic(w: W.Workload, alg_run: float):
    """DRAM bytes per decode launch (dram__bytes_read.sum + write) from the
    committed ncu summary of this workload, scaled from the capture's fill to
    this run's by the algorithmic bytes (the summary records both; traffic
    follows the bytes streamed), or None when there is no summary or the decode
    kernel's source changed since it was captured."""
    import hashlib
    prof = os.path.join(ROOT, "profiles", f"decode_stream_tc_{w.name.replace('-decode', '')}.md")
    csrc = os.path.join(ROOT, "bit_asymmetric_kv_quantize_b200", "csrc")
    try:
        text = open(prof).read()
        h = hashlib.sha256()
        for f in ("kivi_decode_tc.cuh", "kivi_decode_tc.cu", "kivi_internal.cuh"):
            h.update(open(os.path.join(csrc, f), "rb").read())
    except OSError:
        return None
    for line in text.splitlines():
        if line.startswith("traffic_bytes_per_launch:"):
            parts = line.replace("(", " ").replace(")", " ").split()
            if not parts or parts[-1] != h.hexdigest()[:16]:
                continue
            traffic = int(parts[1])
            if "algorithmic_bytes_per_launch:" in parts:
                alg_cap = int(parts[parts.index("algorithmic_bytes_per_launch:") + 1])
                return traffic * alg_run / alg_cap
            return float(traffic)
    return None


def algorithmic_bytes(w: W.Workload, n_q: int, r: int, outliers=(0, 0)) -> int:
    """Bytes one decode call must move: every code, scale and zero of the
    quantized store, the window tokens, q in and out (per unit: K codes
    n_q*D*b/8, K meta (n_q/G)*D*2*ms, V codes n_q*D*b/8, V meta
    n_q*(D/Gv)*2*ms, window r*D*2*es; plus B*Hq*D*es each for q and out;
    ms = 4, or 2 with binary16 scales and zeros)."""
    es = 2 if w.dtype == "f16" else 4
    ms = 2 if w.meta == "f16" else 4
    ko, vo = outliers  # dense-and-sparse lists: an int32 index and a binary32 value per entry

    def per_unit(nq, rr):
        return (2 * nq * w.D * w.bits // 8 + (nq // w.G) * w.D * 2 * ms
                + nq * (w.D // w.Gv) * 2 * ms + rr * w.D * 2 * es
                + 8 * ((nq // w.G) * w.D * ko + nq * (w.D // w.Gv) * vo))

    io = 2 * w.B * w.Hq * w.D * es
    if isinstance(n_q, (list, tuple)):  # ragged: one (n_q, r) per sequence
        return w.Hkv * sum(per_unit(nq, rr) for nq, rr in zip(n_q, r)) + io
    return w.B * w.Hkv * per_unit(n_q, r) + io


# --------------------------------------------------------------- clocks (NVML)

_REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
            0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
            0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
            0x100: "display_clock_setting"}


class ClockSampler:
    """Samples SM clock and clock-event reasons every ~5 ms while running."""

    def __init__(self, index: int):
        self.samples = []
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report it, keep going
            self.err = repr(e)
        self._stop = threading.Event()

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((sm, rs))
            except Exception:
                pass
            time.sleep(0.005)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok:
            return {"error": getattr(self, "err", "nvml unavailable")}
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        sms = [s for s, _ in self.samples]
        mask = 0
        for _, r in self.samples:
            mask |= r
        reasons = sorted(n for b, n in _REASONS.items() if mask & b and n != "gpu_idle")
        return {"sm_mhz": statistics.median(sms), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(sms)}


# ------------------------------------------------------------------ GPU arm

def run_kivi(args, rank, world, local):
    """The headline workload with every measurement, then (unless --no-extras)
    the other decode workloads with the headline and roofline passes only."""
    import torch.distributed as dist
    from datetime import timedelta

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=180), device_id=device)
    w = bench_workload(args)
    result = measure(args, w, rank, world, device, args.steps, args.warmup,
                     args.layers or default_layers(w), full=True)
    if not args.no_extras and args.workload == DEFAULT_WORKLOAD and not (
            args.bits or args.meta != "f32" or args.paged or args.unfused or args.kernel != "default"
            or args.batch or args.outliers != "0,0"):
        extra = {}
        for name in EXTRA_WORKLOADS:
            we = bench_workload(args, name)
            # each layer cache takes its first append in the warm-up: the
            # prefilled windows are full, so that append flushes (as the
            # headline's few layers do in its warm-up)
            nl = default_layers(we)
            r = measure(args, we, rank, world, device, min(args.steps, 1024), max(args.warmup, nl),
                        nl, full=False)
            if rank == 0:
                extra[we.name] = r
        if rank == 0:
            result["workloads"] = extra
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return result, w


def default_layers(w: W.Workload) -> int:
    """Layer caches visited round-robin: enough that the caches together are
    far larger than the 126 MB L2 (the 13B layer alone is 2.8 GB: two)."""
    per_layer = algorithmic_bytes(w, w.T, 0)
    return max(2, min(32, -(-4_000_000_000 // per_layer)))


def measure(args, w: W.Workload, rank, world, device, steps, warmup, n_layers, full):
    """Time `steps` steps of workload `w` (after `warmup`); full: also the
    prefill and append timings, e2e and clocks (the headline workload)."""
    import bit_asymmetric_kv_quantize_b200 as kivi
    import torch.distributed as dist

    ragged = w.len_min > 0
    outliers = tuple(int(x) for x in args.outliers.split(","))
    if args.paged:
        w = w.with_(name=f"{w.name}-paged-{args.paged}")
    if ragged and (args.kernel != "default" or args.unfused):
        raise SystemExit("ragged workloads run the fused tensor-core step only")
    if args.paged and not ragged:
        raise SystemExit("--paged needs a ragged workload")
    n_layers = max(1, n_layers)
    e2e_steps = 0 if (args.no_e2e or not full) else min(steps, 1024)
    per_layer = -(-(warmup + 2 * steps + e2e_steps) // n_layers) + 1
    capacity = -(-(w.T + per_layer) // w.R) * w.R
    Kp, Vp = W.prompt_kv(w, device=device)
    lens = W.seq_lengths(w)
    lens_dev = lens.to(device)
    caches, states = [], []
    # ragged: every layer's per-sequence counters, followed on the host for
    # the algorithmic bytes (the library keeps them on the device)
    host_len = []
    pps = capacity // w.R - 1
    pre_ev = []  # CUDA events around each layer's prefill
    for li in range(n_layers):
        if args.paged:
            # every layer its own pool with a shuffled table (distinct pages)
            g = torch.Generator().manual_seed(li)
            n_pages = w.B * pps
            order = (torch.randperm(n_pages, generator=g) if args.paged == "shuffled"
                     else torch.arange(n_pages))
            bt = order.to(torch.int32).view(w.B, pps)
            c = kivi.PagedKiviCache(w.B, w.Hkv, w.D, w.bits, pps, n_pages, bt.to(device).contiguous(),
                                    R=w.R, G=w.G, Gv=w.Gv, dtype=w.torch_dtype, device=device,
                                    meta=w.torch_meta)
        else:
            c = kivi.KiviCache(w.B, w.Hkv, w.D, w.bits, capacity, R=w.R, G=w.G, Gv=w.Gv,
                               dtype=w.torch_dtype, device=device, meta=w.torch_meta,
                               outliers=outliers)
        pe = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
        pe[0].record()
        if ragged:
            states.append(c.ragged_prefill(Kp, Vp, lens_dev))
            rr = [int((x - 1) % w.R) + 1 for x in lens.tolist()]
            host_len.append(([int(x) - y for x, y in zip(lens.tolist(), rr)], rr))
        else:
            c.prefill(Kp, Vp)
        pe[1].record()
        pre_ev.append(pe)
        caches.append(c)
    # append alone (host counters): 2R + 8 calls on a scratch cache of the
    # same shape, each between CUDA events, split into flush and plain steps
    append_times = None
    if not ragged and full:
        sc = kivi.KiviCache(w.B, w.Hkv, w.D, w.bits, -(-(w.T + 2 * w.R + 8) // w.R) * w.R, R=w.R,
                            G=w.G, Gv=w.Gv, dtype=w.torch_dtype, device=device, meta=w.torch_meta)
        sc.prefill(Kp, Vp)
        k0, v0 = W.step_kv(w, 0, device=device)
        evs_a = []
        for i in range(2 * w.R + 8):
            ea = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            flush = sc.r == sc.R
            # keep the GPU busy while the host enqueues the call, so that the
            # events bracket device time only (not the host's launch latency)
            torch.cuda._sleep(200_000)
            ea[0].record()
            sc.append(k0, v0)
            ea[1].record()
            evs_a.append((flush, ea))
        torch.cuda.synchronize(device)
        t_fl = [e[0].elapsed_time(e[1]) * 1e3 for f, e in evs_a[4:] if f]
        t_pl = [e[0].elapsed_time(e[1]) * 1e3 for f, e in evs_a[4:] if not f]
        append_times = {"call": "kivi_append_token", "plain_us": statistics.median(t_pl),
                        "flush_us": statistics.median(t_fl) if t_fl else None,
                        "flushes_timed": len(t_fl)}
        del sc
    torch.cuda.synchronize(device)
    pre_us = statistics.median(e0.elapsed_time(e1) * 1e3 for e0, e1 in pre_ev[1:] or pre_ev)
    es_in = 2 if w.dtype == "f16" else 4
    pre_tokens = int(lens.sum()) if ragged else w.B * w.T
    # bytes the prefill must move: the prompt's K and V in, the store and the
    # window out (the decode's per-unit byte count without q and out)
    io = 2 * w.B * w.Hq * w.D * es_in
    if ragged:
        r_pre = [(int(n) - 1) % w.R + 1 for n in lens.tolist()]
        written = algorithmic_bytes(w, [int(n) - x for n, x in zip(lens.tolist(), r_pre)], r_pre,
                                    outliers) - io
    else:
        r_pre = (w.T - 1) % w.R + 1
        written = algorithmic_bytes(w, w.T - r_pre, r_pre, outliers) - io
    pre_bytes = 2 * pre_tokens * w.Hkv * w.D * es_in + written
    prefill_times = {"call": "kivi_ragged_prefill" if ragged else "kivi_quantize_prefill",
                     "us": pre_us, "tokens_per_s": pre_tokens / (pre_us * 1e-6),
                     "input_GBps": 2 * pre_tokens * w.Hkv * w.D * es_in / (pre_us * 1e-6) / 1e9,
                     "hbm_bytes": pre_bytes,
                     "frac_of_hbm": pre_bytes / (pre_us * 1e-6) / 1e9 / peak_hbm()[0]}
    del Kp, Vp
    torch.cuda.empty_cache()
    P = 16
    ks, vs, qs = [], [], []
    for i in range(P):
        k, v = W.step_kv(w, i, device=device)
        ks.append(k)
        vs.append(v)
        qs.append(W.query(w, i, device=device))
    out = torch.empty(w.B, w.Hq, w.D, dtype=w.torch_dtype, device=device)
    # (ragged: zero-filled, shared by every layer's calls; the arrival
    # counters reset themselves)
    ws = caches[0]._ragged_ws(w.Hq) if ragged else caches[0].workspace(w.Hq)
    for c in caches[1:]:
        c._ws = ws
    L = kivi.lib()
    dec = L.kivi_decode_attention if args.kernel == "default" else L.kivi_decode_attention_simt
    stream = torch.cuda.current_stream(device)
    sh = stream.cuda_stream
    cstructs = [ctypes.byref(c._c) for c in caches]
    kp = [t.data_ptr() for t in ks]
    vp = [t.data_ptr() for t in vs]
    qp = [t.data_ptr() for t in qs]
    op, wp, wn = out.data_ptr(), ws.data_ptr(), ws.numel()

    fused = args.kernel == "default" and not args.unfused
    n_launch = [0]

    stp = [t.data_ptr() for t in states]

    def step_call(li, k_ptr, v_ptr, q_ptr):
        """One append + decode; returns the status and counts kernel launches."""
        c = caches[li]
        if ragged:
            n_launch[0] += 2  # the append (per-sequence flushes), then the decode
            nq, rr = host_len[li]
            for b in range(w.B):
                if rr[b] == w.R:
                    nq[b] += w.R
                    rr[b] = 1
                else:
                    rr[b] += 1
            return L.kivi_ragged_append_decode(cstructs[li], stp[li], k_ptr, v_ptr, q_ptr, w.Hq,
                                               1.0, op, wp, wn, sh)
        n_launch[0] += 1 if fused else 2  # fused: one launch, a due flush included
        if fused:
            return L.kivi_append_decode(cstructs[li], k_ptr, v_ptr, q_ptr, w.Hq, 1.0, op, wp, wn, sh)
        rc = L.kivi_append_token(cstructs[li], k_ptr, v_ptr, sh)
        return rc or dec(cstructs[li], q_ptr, w.Hq, 1.0, op, wp, wn, sh)

    def step(i, ev=None):
        li = i % n_layers
        if ev is not None:
            L.kivi_set_timing_events(ev[0], ev[1])
        rc = step_call(li, kp[i % P], vp[i % P], qp[i % P])
        if rc:
            raise RuntimeError(f"step: {L.kivi_status_string(rc)}")

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(device)

    # warm-up
    for i in range(warmup):
        step(i)
    barrier()

    # per-step events around the split kernel (created by one record each)
    evs = []
    for _ in range(steps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        e1.record(stream)
        evs.append((e0, e1))
    torch.cuda.synchronize(device)
    ev_handles = [(e0.cuda_event, e1.cuda_event) for e0, e1 in evs]
    # (1) the timed steps: nothing between consecutive launches, so a decode
    # launch may overlap the previous one's drain (programmatic serialization)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    n_launch[0] = 0
    with ClockSampler(device.index if device.index is not None else 0) as clk:
        t0.record(stream)
        h0 = time.perf_counter()
        for j in range(steps):
            step(warmup + j)
        host_us = (time.perf_counter() - h0) * 1e6 / steps
        t1.record(stream)
        timed_launches = n_launch[0]
        torch.cuda.synchronize(device)
    barrier()
    ms = t0.elapsed_time(t1)
    # (2) the roofline: as many further steps, CUDA events recorded by the
    # library around each decode launch (these serialize the launches)
    fills = []
    for j in range(steps):
        i = warmup + steps + j
        step(i, ev_handles[j])
        c = caches[i % n_layers]
        if ragged:
            nq, rr = host_len[i % n_layers]
            fills.append((list(nq), list(rr)))
        else:
            fills.append((c.n_q, c.r))
    torch.cuda.synchronize(device)
    L.kivi_set_timing_events(None, None)
    barrier()
    split_ms = [e0.elapsed_time(e1) for e0, e1 in evs]
    ms_max = max_over_ranks(ms, world, device)

    # roofline of the split kernel: algorithmic bytes / event time
    bytes_total = sum(algorithmic_bytes(w, nq, r, outliers) for nq, r in fills)
    # tokens attended per step (summed over sequences, per KV head), mean over the fills
    ctx_tokens = statistics.mean((sum(nq) + sum(r)) if isinstance(nq, list) else w.B * (nq + r)
                                 for nq, r in fills)
    split_total_ms = sum(split_ms)
    achieved = bytes_total / (split_total_ms * 1e-3) / 1e9
    peak, peak_src = peak_hbm()
    n_split = caches[0].num_splits(w.Hq)

    # e2e: the same loop, inputs from pinned host memory, output read back
    e2e = None
    if e2e_steps:
        # each step's k, v and q staged in one pinned host buffer and brought
        # over in one copy; k, v, q are views of one device buffer
        nk, nq_ = ks[0].numel(), qs[0].numel()
        hs = [torch.cat([ks[j].flatten(), vs[j].flatten(), qs[j].flatten()]).cpu().pin_memory()
              for j in range(P)]
        ho = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        dst = torch.empty_like(hs[0], device=device)
        dk = dst[:nk].view(ks[0].shape)
        dv = dst[nk:2 * nk].view(vs[0].shape)
        dq = dst[2 * nk:].view(qs[0].shape)
        h2d = hs[0].numel() * hs[0].element_size()
        d2h = out.numel() * out.element_size()
        n_e2e = e2e_steps
        base = warmup + 2 * steps
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        host_call = fused and not ragged  # the library's own host-buffer step
        if host_call:
            L.kivi_host_step_bytes.argtypes = [ctypes.POINTER(kivi.KiviCacheC), ctypes.c_int]
            L.kivi_host_step_bytes.restype = ctypes.c_size_t
            L.kivi_append_decode_host.argtypes = [ctypes.POINTER(kivi.KiviCacheC), ctypes.c_void_p,
                                                  ctypes.c_int, ctypes.c_float, ctypes.c_void_p,
                                                  ctypes.c_void_p, ctypes.c_size_t,
                                                  ctypes.c_void_p, ctypes.c_size_t,
                                                  ctypes.c_void_p]
            stg_n = int(L.kivi_host_step_bytes(cstructs[0], w.Hq))
            stg = torch.empty(stg_n, dtype=torch.uint8, device=device)
        for j in range(n_e2e):
            i = base + j
            li = i % n_layers
            if host_call:
                # k | v | q from pinned host memory, the fused step, out back:
                # one C-ABI call
                n_launch[0] += 1
                rc = L.kivi_append_decode_host(cstructs[li], hs[i % P].data_ptr(), w.Hq, 1.0,
                                               ho.data_ptr(), stg.data_ptr(), stg_n, wp, wn, sh)
            else:
                dst.copy_(hs[i % P], non_blocking=True)
                rc = step_call(li, dk.data_ptr(), dv.data_ptr(), dq.data_ptr())
                if not rc:
                    ho.copy_(out, non_blocking=True)
            if rc:
                raise RuntimeError("e2e step failed")
        e1.record(stream)
        torch.cuda.synchronize(device)
        e_ms = max_over_ranks(e0.elapsed_time(e1), world, device)
        e2e = {"value": replica_throughput(world, w.B, n_e2e, e_ms), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": n_e2e,
               "ms_per_step": e_ms / n_e2e,
               "call": "kivi_append_decode_host" if host_call else "copies + step call"}

    result = None
    if rank == 0:
        tokens_per_s = replica_throughput(world, w.B, steps, ms_max)
        result = {
            "metric": METRIC,
            "value": tokens_per_s,
            "unit": "tokens/s",
            "n_gpus": world,
            "steps": steps,
            "warmup": warmup,
            "ms_per_step": ms_max / steps,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "f32" if args.kernel == "simt" else "f16xf16+f32",
            "data": "synthetic",
            "config": {
                "workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "D": w.D,
                "context": w.T, "bits": w.bits, "G": w.G, "Gv": w.Gv, "R": w.R,
                "dtype_io": w.dtype, "meta": w.meta, "kernel": args.kernel,
                **({"outliers_per_group": {"keys": outliers[0], "values": outliers[1]}}
                   if any(outliers) else {}),
                **({"paged": f"pages of {w.R} tokens, {args.paged} block table"}
                   if args.paged else {}),
                "step": ("kivi_ragged_append_decode" if ragged else
                         "kivi_append_decode" if fused else "kivi_append_token+kivi_decode_attention"),
                "parallelism": f"replicas{world}",
                "layers_rotated": n_layers,
                "l2": f"inputs larger than L2: {n_layers} layer caches visited round-robin",
                "decode_splits": n_split,
                **({"lengths": {"min": int(lens.min()), "max": int(lens.max()),
                                "mean": float(lens.float().mean())}} if ragged else {}),
            },
            "roofline": {
                "kernel": "decode_stream_tc" if args.kernel == "default" else "decode_split_simt",
                "bound": "hbm", "achieved": achieved, "peak": peak,
                "peak_source": peak_src, "unit": "GB/s", "frac": achieved / peak,
                "traffic": (profiled_traffic(w, bytes_total / steps)
                            if args.kernel == "default" else None),
                "algorithmic_bytes_per_launch": bytes_total / steps,
                "avg_launch_us": split_total_ms * 1e3 / steps,
            },
            "context_tokens_per_s": ctx_tokens * w.Hkv / (ms_max / steps * 1e-3) * world,
            "prefill": prefill_times,
            "append": append_times,
            "e2e": e2e,
            "gpu_launches": timed_launches,
            "clocks": clk.summary(),
        }
        if not full:  # an extra workload: its own rate and roofline only
            keep = ("value", "unit", "steps", "warmup", "ms_per_step", "config", "roofline",
                    "context_tokens_per_s", "gpu_launches", "host_us_per_step")
            result["host_us_per_step"] = host_us
            result = {k: result[k] for k in keep}
        else:
            result["host_us_per_step"] = host_us
    del caches, states, ks, vs, qs, out, ws
    torch.cuda.empty_cache()
    return result


# --------------------------------------------------------------- CPU oracle arm

def oracle_sample(w: W.Workload, n_units: int, steps: int, threads: int):
    """Time `steps` decode steps (append + decode) of the CPU oracle on
    `n_units` units of the workload spread evenly over the batch (each at its
    sequence's prompt length); returns (seconds per step, units, factor that
    scales the sample's time to the whole batch by tokens held)."""
    import oracle
    from concurrent.futures import ThreadPoolExecutor

    total = w.B * w.Hkv
    n = max(1, min(n_units, total))
    picks = sorted({(i * total) // n for i in range(n)})
    units = [(u // w.Hkv, u % w.Hkv) for u in picks]
    lens = [int(x) for x in W.seq_lengths(w)]
    scale = (w.Hkv * sum(lens)) / sum(lens[b] for b, _ in units)
    cap = -(-(w.T + steps + 1) // w.R) * w.R
    oc = oracle.OracleCache(w.B, w.Hkv, w.D, w.bits, w.G, w.Gv, w.R, cap, units=units,
                            meta_f16=w.meta == "f16")
    g = w.with_(B=1, Hkv=1, Hq=w.gq)
    K, V = W.prompt_kv(g)
    Kf, Vf = K[0, 0].float().numpy(), V[0, 0].float().numpy()
    qs = W.query(w).float().numpy()
    step_in = [tuple(t.float().numpy() for t in W.step_kv(w, i)) for i in range(min(steps, 4))]
    gq = w.gq
    with ThreadPoolExecutor(threads) as ex:
        list(ex.map(lambda u: oc.prefill_unit(u[0], u[1], Kf[:lens[u[0]]], Vf[:lens[u[0]]]),
                    units))

        def one(u, i):
            b, h = u
            k, v = step_in[i % len(step_in)]
            oc.append_unit(b, h, k[b, h], v[b, h])
            oc.decode_unit(b, h, qs[b, h * gq:(h + 1) * gq], 1.0)

        t = time.perf_counter()
        for i in range(steps):
            list(ex.map(lambda u: one(u, i), units))
        dt = time.perf_counter() - t
    return dt / steps, len(units), scale


def cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_threads():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(w: W.Workload, budget_s: float):
    threads = cpu_threads()
    # calibrate on one step of a few units, then size the sample to the budget
    per_step, n, _ = oracle_sample(w, threads, 1, threads)
    per_unit_cpu = per_step * threads / n
    n_units = min(w.B * w.Hkv, max(threads, int(threads * 4)))
    steps = max(1, int(budget_s * threads / (per_unit_cpu * n_units)))
    per_step, n, scale = oracle_sample(w, n_units, steps, threads)
    full_step = per_step * scale
    # the same loop on one thread, over a fifth of the budget
    steps1 = max(1, int(budget_s / 5 / (per_unit_cpu * threads)))
    per1, n1, scale1 = oracle_sample(w, threads, steps1, 1)
    return {"value": w.B / full_step, "unit": "tokens/s", "cores": threads, "cpu_model": cpu_model(),
            "kind": "oracle",
            "sample": f"{steps} steps x {n} of {w.B * w.Hkv} (batch, KV head) units spread "
                      f"over the batch, append + decode, scaled to the full batch by tokens "
                      f"held; single oracle threads fanned out over units",
            "single_thread": {"value": w.B / (per1 * scale1), "unit": "tokens/s",
                              "sample": f"{steps1} steps x {n1} units on one thread, scaled "
                                        f"the same way"}}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    w = bench_workload(args)
    threads = cpu_threads()
    budget = 120.0  # seconds of wall time for warm-up + timed steps
    per_step, n, _ = oracle_sample(w, threads, 1, threads)
    n_units = max(1, min(w.B * w.Hkv,
                         int(budget / max(1, args.steps + args.warmup) / per_step * n)))
    oracle_sample(w, n_units, max(1, args.warmup), threads)
    per_step, n, scale = oracle_sample(w, n_units, args.steps, threads)
    full_step = per_step * scale
    value = w.B / full_step
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": full_step * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "D": w.D,
                   "context": w.T, "bits": w.bits, "G": w.G, "Gv": w.Gv, "R": w.R,
                   "meta": w.meta},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "cpu_model": cpu_model(), "kind": "oracle",
                         "sample": f"each step: append + decode on {n} of {w.B * w.Hkv} units, "
                                   f"scaled to the full batch"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    args = parse()
    rank, world, local = dist_env()
    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    res, w = run_kivi(args, rank, world, local)
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            res["cpu_baseline"] = cpu_baseline(w, args.cpu_budget_s)
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
