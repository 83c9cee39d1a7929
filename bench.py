"""Benchmark of the hybrid compressed attention path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload csa_prefill|hca_prefill|csa_decode|hybrid_decode|tiny]
                    [--secondary none|all]

Headline: CSA prefill tokens/s on one 65,536-token sequence (m=4 -> 16,384
entries, 64 heads x 128, indexer 8 x 64, top-k 1024). One step = compression
+ lightning indexer + top-k + sparse attention over the whole sequence, inputs
resident in HBM. With N ranks each rank runs its own sequence (independent
problems, weak scaling, no data-path collective); the JSON `value` is the
tokens of all ranks over the slowest rank's time. Between timed steps L2 is
flushed by writing a 512 MiB buffer (outside the timed events).

Also measured by default (secondary, same JSON line under "workloads"): HCA
prefill (1,048,576 tokens, m'=128) tokens/s, the CSA decode layer (64
sequences at 131,072 tokens of context, 32,768 entries each) and the hybrid
1M-context decode step (8 sequences, C,H,C,H) in microseconds per step.

--impl reference times the C++ CPU oracle (the plain float64 reference the
parity tests also pin) on this host's cores on a bounded sample of the same
workload.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from compressed_sparse_long_compress_b200 import workloads as W  # noqa: E402

L2_FLUSH_BYTES = 512 << 20


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi clock / throttle samples (every 50 ms) during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (FileNotFoundError, OSError):
            self.proc = None
        # start timing only once the sampler is live (its first line is written)
        t0 = time.time()
        while self.proc is not None and time.time() - t0 < 5.0:
            if os.path.getsize(self.path) > 0 or self.proc.poll() is not None:
                break
            time.sleep(0.02)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "samples": len(sm), "reasons": sorted(reasons)}


# ------------------------------------------------------------ dist helpers

def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    device = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(wid: int, rank: int) -> int:
    """Workload id whose seeded draws rank `rank` uses: every rank runs its own
    independent sequence (weak scaling, no data-path exchange)."""
    return wid + 10 * rank


def job_value(units_per_rank: int, max_ms: float, world: int) -> float:
    """Whole-job throughput: the units all ranks processed over the slowest
    rank's step time."""
    return world * units_per_rank / (max_ms * 1e-3)


# ---------------------------------------------------------------- workloads

def csa_selected_pairs(L, m, n_c, k):
    t = np.arange(L, dtype=np.int64)
    return int(np.minimum(k, np.minimum(n_c, (t + 1) // m)).sum())


def causal_visible_pairs(L, m, n_c):
    t = np.arange(L, dtype=np.int64)
    return int(np.minimum(n_c, (t + 1) // m).sum())


class CsaPrefill:
    name = "csa_prefill"

    def __init__(self, C, device, rank):
        wl = W.WORKLOADS["csa_prefill"]
        self.s = s = wl.csa
        self.C = C
        self.x = W.prefill_inputs(s, rank_seed(wl.wid, rank), device=device)
        self.e = torch.empty(s.B, s.n_c, 128, dtype=torch.bfloat16, device=device)
        self.idx = torch.empty(s.B, s.L, s.topk, dtype=torch.int32, device=device)
        self.out = torch.empty_like(self.x["q"])
        nb = C.indexer_topk_workspace_bytes(s.B, s.L, s.n_c, s.HI, s.topk)
        self.ws = torch.empty(max(nb, 16), dtype=torch.uint8, device=device)
        # score blocks, read off the workspace the library asks for: the whole
        # score tensor (one block), or two blocks of rows in flight
        full = s.B * s.L * s.n_c * 4
        self.rows_per_block = s.L if nb >= full else max(1, nb // (2 * s.B * s.n_c * 4))
        self.launches = 2 + 2 * math.ceil(s.L / self.rows_per_block)   # compress, attention, indexer + top-k per block
        self.pairs = csa_selected_pairs(s.L, s.m, s.n_c, s.topk)
        self.flops_attn = 4.0 * 128 * s.H * self.pairs            # QK^T + PV over selected pairs
        self.flops_indexer = 2.0 * 64 * s.HI * causal_visible_pairs(s.L, s.m, s.n_c)
        self.units = s.B * s.L

    def step(self, timer=None):
        s, x, C = self.s, self.x, self.C
        C.csa_compress(x["c"], x["z"], x["pos_bias"], m=s.m, out=self.e)
        C.csa_indexer_topk(x["q_idx"], x["w"], x["k_idx"], m=s.m, topk=s.topk, idx=self.idx, ws=self.ws)
        if timer:
            timer[0].record()
        C.csa_sparse_attn(x["q"], self.e, self.idx, s.scale, out=self.out)
        if timer:
            timer[1].record()

    def input_tensors(self):
        return [self.x[k] for k in ("c", "z", "pos_bias", "q", "q_idx", "w", "k_idx")]

    def output_tensors(self):
        return [self.out]

    def add_buffer_set(self):
        """A second set of device inputs and outputs, so that an end-to-end run
        can copy the next step's inputs in and the previous step's output out
        while a step runs."""
        self.sets = [(self.x, self.out),
                     ({k: torch.empty_like(v) for k, v in self.x.items()}, torch.empty_like(self.out))]

    def use_set(self, i):
        self.x, self.out = self.sets[i]

    def roofline(self, kernel_ms, peaks):
        ach = self.flops_attn / (kernel_ms * 1e-3) / 1e12
        return {"kernel": "csa_sparse_attn (sparse_attn_sm100_kernel<64>)", "bound": "tensor",
                "achieved": round(ach, 2), "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": round(ach / peaks["bf16_tflops"], 4),
                "traffic": measured_traffic("sparse", self.units),
                "algorithmic_flops_per_launch": self.flops_attn, "peak_source": peaks["source"] + " (burst)"}

    def config(self):
        return workload_config(self.name)


class HcaPrefill:
    name = "hca_prefill"

    def __init__(self, C, device, rank):
        wl = W.WORKLOADS["hca_prefill"]
        self.s = s = wl.hca
        self.C = C
        self.x = W.prefill_inputs(s, rank_seed(wl.wid, rank), device=device, with_indexer=False)
        self.e = torch.empty(s.B, s.n_c, 128, dtype=torch.bfloat16, device=device)
        self.out = torch.empty_like(self.x["q"])
        self.launches = 2
        self.pairs = causal_visible_pairs(s.L, s.m, s.n_c)
        self.flops_attn = 4.0 * 128 * s.H * self.pairs
        self.units = s.B * s.L

    def step(self, timer=None):
        s, x, C = self.s, self.x, self.C
        C.hca_compress(x["c"], x["z"], x["pos_bias"], m_prime=s.m, out=self.e)
        if timer:
            timer[0].record()
        C.hca_dense_attn(x["q"], self.e, m_prime=s.m, scale=s.scale, out=self.out)
        if timer:
            timer[1].record()

    def input_tensors(self):
        return [self.x[k] for k in ("c", "z", "pos_bias", "q")]

    def output_tensors(self):
        return [self.out]

    def roofline(self, kernel_ms, peaks):
        ach = self.flops_attn / (kernel_ms * 1e-3) / 1e12
        return {"kernel": "hca_dense_attn (dense_attn_sm100_kernel)", "bound": "tensor", "achieved": round(ach, 2),
                "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "frac": round(ach / peaks["bf16_tflops"], 4),
                "traffic": measured_traffic("dense", self.units), "algorithmic_flops_per_launch": self.flops_attn,
                "peak_source": peaks["source"] + " (burst)"}

    def config(self):
        return workload_config(self.name)


class FrontEnd:
    name = "front_end_prefill"

    def __init__(self, C, device, rank):
        wl = W.WORKLOADS[self.name]
        self.s = s = wl.front_end
        self.C = C
        self.x = W.front_end_inputs(s, rank_seed(wl.wid, rank), device=device)
        self.e = torch.empty(s.B, s.n_c, 128, dtype=torch.bfloat16, device=device)
        self.launches = 1
        self.flops = 2.0 * s.B * s.L * s.d_model * 128 * s.n_proj   # every token through the projections once
        self.units = s.B * s.L

    def step(self, timer=None):
        s, x = self.s, self.x
        if timer:
            timer[0].record()
        self.C.compress_front_end(x["h"], x["W"], x["pos_bias"], s.m, s.overlap, out=self.e)
        if timer:
            timer[1].record()

    def input_tensors(self):
        return [self.x["h"], self.x["W"], self.x["pos_bias"]]

    def output_tensors(self):
        return [self.e]

    def roofline(self, kernel_ms, peaks):
        ach = self.flops / (kernel_ms * 1e-3) / 1e12
        return {"kernel": "compress_front_end (front_end_sm100_kernel<true>)", "bound": "tensor",
                "achieved": round(ach, 2), "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": round(ach / peaks["bf16_tflops"], 4), "traffic": measured_traffic("front_end", self.units),
                "algorithmic_flops_per_launch": self.flops, "peak_source": peaks["source"] + " (burst)"}

    def config(self):
        return workload_config(self.name)


class Decode:
    def __init__(self, C, device, rank, name):
        self.name = name
        wl = W.WORKLOADS[name]
        self.d = d = wl.decode
        self.C = C
        self.layers, self.bytes = [], 0
        for li, kind in enumerate(d.kinds):
            x = W.decode_layer_inputs(d, li, rank_seed(wl.wid, rank), device=device)
            n = torch.full((d.B,), d.n_entries[li], dtype=torch.int32, device=device)
            nope, rope, sc = C.quantize_kv_mixed(x["kv"])
            del x["kv"]
            kw = {}
            if kind == "csa":
                kw = dict(q_idx=x["q_idx"], w=x["w"], k_idx=x["k_idx"], topk=d.topk)
                # indexer keys scanned once + selected mixed entries gathered + q
                self.bytes += d.B * d.n_entries[li] * 64 * 2 + d.B * min(d.topk, d.n_entries[li]) * 196
            else:
                self.bytes += d.B * d.n_entries[li] * 196
            self.bytes += d.B * d.H * 128 * 2 * 2      # q in, out
            self.layers.append(C.DecodeLayer(kind, x["q"], nope, rope, sc, n, d.scale, **kw))
        self.step_fn = C.DecodeStep(self.layers, HI=d.HI)
        # the library picks the CSA tail per batch (one cluster launch, or four
        # kernels); the count used in the line is measured (count_launches)
        self.launches = sum(5 if k == "csa" else 2 for k in d.kinds) + 1
        self.units = 1

    def step(self, timer=None):
        if timer:
            timer[0].record()
        self.step_fn()
        if timer:
            timer[1].record()

    def input_tensors(self):
        return [l.q for l in self.layers]

    def output_tensors(self):
        return [l.out for l in self.layers]

    def roofline(self, kernel_ms, peaks):
        ach = self.bytes / (kernel_ms * 1e-3) / 1e9
        return {"kernel": "whole decode step (cslc_decode_step)", "bound": "hbm", "achieved": round(ach, 1),
                "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(ach / peaks["hbm_gbs"], 4),
                "traffic": measured_traffic(self.name, 1),
                "algorithmic_bytes_per_launch": self.bytes, "peak_source": peaks["source"]}

    def config(self):
        return workload_config(self.name)


def workload_config(name):
    """The `config` object of a workload (no device needed; the reference arm
    reports the same one)."""
    wl = W.WORKLOADS[name]
    if name == "csa_prefill":
        s = wl.csa
        return {"workload": "csa_prefill: CSA prefill, batch 1, L=65536, m=4 -> 16384 entries, 64 heads x 128, "
                            "indexer 8 x 64, top-k 1024, causal",
                "global_batch": s.B, "seq_len": s.L, "heads": s.H, "head_dim": 128, "m": s.m, "topk": s.topk,
                "indexer_heads": s.HI, "l2": "flushed between steps (512 MiB write)"}
    if name == "hca_prefill":
        s = wl.hca
        return {"workload": "hca_prefill: HCA prefill, batch 1, L=1048576, m'=128 -> 8192 entries, 64 heads x 128, "
                            "dense causal", "global_batch": s.B, "seq_len": s.L, "heads": s.H, "m_prime": s.m,
                "l2": "inputs larger than L2 (q 16 GiB)"}
    if wl.front_end is not None:
        f = wl.front_end
        return {"workload": f"{name}: " + wl.description, "global_batch": f.B, "seq_len": f.L,
                "d_model": f.d_model, "m": f.m, "l2": "inputs larger than L2 (h 940 MB)"}
    if wl.decode is not None:
        d = wl.decode
        return {"workload": f"{name}: " + wl.description, "global_batch": d.B, "layers": list(d.kinds),
                "entries": list(d.n_entries), "heads": d.H, "topk": d.topk,
                "l2": "flushed between steps (512 MiB write)"}
    return {"workload": f"{name}: " + wl.description}


def make_workload(name, C, device, rank):
    if name == "csa_prefill":
        return CsaPrefill(C, device, rank)
    if name == "hca_prefill":
        return HcaPrefill(C, device, rank)
    if name == "front_end_prefill":
        return FrontEnd(C, device, rank)
    return Decode(C, device, rank, name)


# ------------------------------------------------------------------ timing

def time_device(wl, steps, warmup, world, flush):
    for _ in range(warmup):
        wl.step()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    step_ms, kern_ms = [], []
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i in range(steps):
        flush.zero_()
        a, b, k0, k1 = ev[i]
        a.record()
        wl.step(timer=(k0, k1))
        b.record()
    torch.cuda.synchronize()
    barrier(world)
    for a, b, k0, k1 in ev:
        step_ms.append(a.elapsed_time(b))
        kern_ms.append(k0.elapsed_time(k1))
    return step_ms, kern_ms


def time_e2e(wl, steps, world):
    """Host -> device copy of the step's inputs (pinned), the step, and the
    device -> host read of its outputs, every step. Workloads with a second
    buffer set run as a pipeline: step i's inputs are copied in on one stream
    and step i-1's output copied out on another while step i-1 / i runs."""
    if hasattr(wl, "add_buffer_set"):
        return time_e2e_pipelined(wl, steps, world)
    ins = wl.input_tensors()
    outs = wl.output_tensors()
    h_in = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in ins]
    for h, t in zip(h_in, ins):
        h.copy_(t)
    h_out = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in outs]
    torch.cuda.synchronize()
    barrier(world)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(steps):
        for h, t in zip(h_in, ins):
            t.copy_(h, non_blocking=True)
        wl.step()
        for h, t in zip(h_out, outs):
            h.copy_(t, non_blocking=True)
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / steps
    return ms, sum(t.numel() * t.element_size() for t in ins), sum(t.numel() * t.element_size() for t in outs)


def time_e2e_pipelined(wl, steps, world):
    wl.add_buffer_set()
    ins, outs = [], []
    for i in range(2):
        wl.use_set(i)
        ins.append(wl.input_tensors())
        outs.append(wl.output_tensors())
    wl.use_set(0)
    h_in = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in ins[0]]
    for h, t in zip(h_in, ins[0]):
        h.copy_(t)
    h_out = [[torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in o] for o in outs]
    comp = torch.cuda.current_stream()
    cin, cout = torch.cuda.Stream(), torch.cuda.Stream()
    in_ready = [torch.cuda.Event() for _ in range(2)]
    done = [torch.cuda.Event() for _ in range(2)]
    read = [torch.cuda.Event() for _ in range(2)]
    torch.cuda.synchronize()
    barrier(world)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(comp)
    cin.wait_stream(comp)
    for i in range(steps):
        k = i & 1
        with torch.cuda.stream(cin):
            if i >= 2:
                cin.wait_event(done[k])          # step i-2 has finished reading this set
            for h, t in zip(h_in, ins[k]):
                t.copy_(h, non_blocking=True)
            in_ready[k].record(cin)
        comp.wait_event(in_ready[k])
        if i >= 2:
            comp.wait_event(read[k])             # step i-2's output has been read out
        wl.use_set(k)
        wl.step()
        done[k].record(comp)
        with torch.cuda.stream(cout):
            cout.wait_event(done[k])
            for h, t in zip(h_out[k], outs[k]):
                h.copy_(t, non_blocking=True)
            read[k].record(cout)
    for k in range(min(2, steps)):
        comp.wait_event(read[k])
    b.record(comp)
    torch.cuda.synchronize()
    wl.use_set(0)
    wl.sets = None
    ms = a.elapsed_time(b) / steps
    return ms, sum(t.numel() * t.element_size() for t in ins[0]), sum(t.numel() * t.element_size() for t in outs[0])


def count_launches(wl, libs=("cslc",)):
    """This library's kernels launched by one (untimed) step, counted with the
    CUDA profiler; None when the profiler sees no kernel."""
    try:
        from torch.profiler import ProfilerActivity, profile
        torch.cuda.synchronize()
        with profile(activities=[ProfilerActivity.CUDA]) as prof:
            wl.step()
            torch.cuda.synchronize()
        names = [e.name for e in prof.events() if e.device_type == torch.autograd.DeviceType.CUDA]
    except Exception:   # no profiler support: the static count stands
        return None
    ours = [n for n in names if any(k in n for k in libs) or "_sm100_kernel" in n]
    return len(ours) if ours else None


def measure(name, C, args, world, rank, local, peaks, flush, with_e2e=True, min_timed_ms=0.0):
    """min_timed_ms > 0 (secondary workloads only) raises the number of timed
    steps until the timed region lasts about that long, so that the clock
    sampler sees it; the headline workload times exactly args.steps."""
    device = torch.device("cuda", local)
    wl = make_workload(name, C, device, rank)
    steps = args.steps
    if min_timed_ms > 0:
        probe, _ = time_device(wl, 2, 1, world, flush)
        per = max(1e-3, max_over_ranks(max(probe), world))
        steps = max(steps, int(min_timed_ms / per) + 1)
    with ClockSampler(local) as clk:
        step_ms, kern_ms = time_device(wl, steps, args.warmup, world, flush)
    clocks = clk.summary()
    ms = max_over_ranks(sum(step_ms) / len(step_ms), world)
    kms = max_over_ranks(sum(kern_ms) / len(kern_ms), world)
    res = {"ms_per_step": ms, "kernel_ms": kms, "clocks": clocks, "roofline": wl.roofline(kms, peaks),
           "gpu_launches": wl.launches * steps, "gpu_launches_per_step": wl.launches,
           "gpu_launches_counted": False, "config": wl.config(), "units": wl.units, "steps": steps}
    if wl.units > 1:
        res["value"] = job_value(wl.units, ms, world)
        res["unit"] = "tokens/s"
        res["higher_is_better"] = True
    else:
        res["value"] = ms * 1e3
        res["unit"] = "us/step"
        res["higher_is_better"] = False
    if with_e2e:
        pipelined = hasattr(wl, "add_buffer_set")
        e_ms, bi, bo = time_e2e(wl, max(2, min(args.steps, 10 if pipelined else 5)), world)
        e_ms = max_over_ranks(e_ms, world)
        e_val = job_value(wl.units, e_ms, world) if wl.units > 1 else e_ms * 1e3
        res["e2e"] = {"value": e_val, "unit": res["unit"], "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bo}
        if pipelined:
            res["e2e"]["pipeline"] = ("two device buffer sets: step i+1's inputs copied in and step i-1's "
                                      "output copied out on their own streams while step i runs")
    del wl
    torch.cuda.empty_cache()
    return res


def measure_indexer_variants(C, device, flush, reps=10):
    """The indexer + top-k of the 65,536-token CSA workload in its three forms
    (first page §1.4: a low-precision indexer): fp32 scores from bf16
    operands (the headline path), bf16-stored scores, and e4m3 operands with
    per-row scales (fp32 scores). CUDA-event medians with L2 flushed before
    each call; the e4m3 rows are quantised beforehand (their quantisation is
    timed on its own), and the recall of each variant's selection against the
    fp32 path's over every query row."""
    wl = W.WORKLOADS["csa_prefill"]
    s = wl.csa
    x = W.prefill_inputs(s, wl.wid, device=device)
    idx32 = torch.empty(s.B, s.L, s.topk, dtype=torch.int32, device=device)
    idx16 = torch.empty_like(idx32)
    idx8 = torch.empty_like(idx32)
    ws32 = torch.empty(max(16, C.indexer_topk_workspace_bytes(s.B, s.L, s.n_c, s.HI, s.topk)), dtype=torch.uint8,
                       device=device)
    ws16 = torch.empty(max(16, C.indexer_topk_bf16_workspace_bytes(s.B, s.L, s.n_c, s.HI, s.topk)), dtype=torch.uint8,
                       device=device)
    q8, qs = C.quantize_rows_e4m3(x["q_idx"])
    k8, ks = C.quantize_rows_e4m3(x["k_idx"])
    run32 = lambda: C.csa_indexer_topk(x["q_idx"], x["w"], x["k_idx"], m=s.m, topk=s.topk, idx=idx32, ws=ws32)
    run16 = lambda: C.csa_indexer_topk_bf16(x["q_idx"], x["w"], x["k_idx"], m=s.m, topk=s.topk, idx=idx16, ws=ws16)
    run8 = lambda: C.csa_indexer_topk_fp8(q8, qs, x["w"], k8, ks, m=s.m, topk=s.topk, idx=idx8, ws=ws32)
    quant = lambda: (C.quantize_rows_e4m3(x["q_idx"], q8, qs), C.quantize_rows_e4m3(x["k_idx"], k8, ks))
    out = {}
    for name, fn in (("fp32", run32), ("bf16_scores", run16), ("fp8_operands", run8), ("fp8_quantize", quant)):
        for _ in range(3):
            fn()
        ts = []
        for _ in range(reps):
            flush.zero_()
            a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a_.record()
            fn()
            b_.record()
            torch.cuda.synchronize()
            ts.append(a_.elapsed_time(b_))
        out[f"ms_{name}"] = sorted(ts)[len(ts) // 2]

    def recall(idx):   # |sel_fp32 & sel| / |sel_fp32| over all rows (selections ascending, -1 padded)
        kept = 0
        for r0 in range(0, s.L, 4096):
            a_ = idx32[0, r0:r0 + 4096].long()
            b_ = idx[0, r0:r0 + 4096].long()
            a_ = torch.where(a_ < 0, torch.full_like(a_, s.n_c + 1), a_)
            b_ = torch.where(b_ < 0, torch.full_like(b_, -1), b_)
            pos = torch.searchsorted(b_.contiguous(), a_.contiguous()).clamp(max=s.topk - 1)
            kept += int((torch.gather(b_, 1, pos) == a_).sum())
        return kept / max(1, int((idx32 >= 0).sum()))

    out["recall_bf16_scores_vs_fp32"] = recall(idx16)
    out["recall_fp8_operands_vs_fp32"] = recall(idx8)
    out["workload"] = "indexer + top-k of csa_prefill (L=65536, 16384 entries, 8 x 64, top-k 1024)"
    return out


# ------------------------------------------------------------ ncu cases

def profile_case(name):
    """One small case of a kernel for an ncu capture (inputs larger than L2,
    a few GB on the device): builds seeded inputs and calls the entry twice."""
    from compressed_sparse_long_compress_b200 import cslc as C
    dev = torch.device("cuda", 0)
    if name == "sparse_attn_L8192":
        L, H, n_c, k = 8192, 64, 16384, 1024
        q = W.randn_bf16((1, L, H, 128), 1, device=dev)
        e = W.randn_bf16((1, n_c, 128), 2, device=dev, std=0.4)
        g = torch.Generator(device=dev)
        g.manual_seed(3)
        idx = torch.sort(torch.rand(1, L, n_c, device=dev, generator=g).topk(k, dim=-1).indices.int(),
                         dim=-1).values.contiguous()
        out = torch.empty_like(q)
        for _ in range(2):
            C.csa_sparse_attn(q, e, idx, 1 / math.sqrt(128), out=out)
    elif name == "dense_attn_L65536":
        L, H = 65536, 64
        q = W.randn_bf16((1, L, H, 128), 1, device=dev)
        e = W.randn_bf16((1, L // 128, 128), 2, device=dev, std=0.4)
        out = torch.empty_like(q)
        for _ in range(2):
            C.hca_dense_attn(q, e, m_prime=128, scale=1 / math.sqrt(128), out=out)
    elif name == "topk_L8192":
        L, n_c, k = 8192, 16384, 1024
        scores = W.rand_f32((1, L, n_c), seed=4, device=dev)
        idx = torch.empty(1, L, k, dtype=torch.int32, device=dev)
        for _ in range(2):
            C.csa_topk(scores, m=4, topk=k, q_pos0=4 * n_c, idx=idx)   # every row sees all entries
    elif name == "indexer_L8192":
        L, n_c, HI = 8192, 16384, 8
        q_idx = W.randn_bf16((1, L, HI, 64), 5, device=dev)
        w = W.randn_bf16((1, L, HI), 6, device=dev)
        k_idx = W.randn_bf16((1, n_c, 64), 7, device=dev)
        scores = torch.empty(1, L, n_c, device=dev)
        idx = torch.empty(1, L, 1024, dtype=torch.int32, device=dev)
        for _ in range(2):   # the last 8192 query rows of a 65536-token sequence
            C.csa_indexer_topk(q_idx, w, k_idx, m=4, topk=1024, q_pos0=4 * n_c - L, scores=scores, idx=idx)
    elif name == "front_end_L16384":   # 16384 tokens of d_model 7168 (235 MB of hidden states)
        s = W.FrontEndShape(B=1, L=16384, d_model=7168)
        x = W.front_end_inputs(s, 6, device=dev)
        for _ in range(2):
            C.compress_front_end(x["h"], x["W"], x["pos_bias"], s.m, True)
    elif name == "dense_attn_steady":   # the last 16384 query rows of the 1,048,576-token HCA layer
        L, H, n_c = 16384, 64, 8192
        q = W.randn_bf16((1, L, H, 128), 1, device=dev)
        e = W.randn_bf16((1, n_c, 128), 2, device=dev, std=0.4)
        out = torch.empty_like(q)
        for _ in range(2):
            C.hca_dense_attn(q, e, m_prime=128, scale=1 / math.sqrt(128), q_pos0=128 * n_c - L, out=out)
    elif name in ("compress_L65536", "compress_hca_L1M"):   # the two prefill workloads' compression
        L, m, overlap = (65536, 4, True) if name == "compress_L65536" else (1 << 20, 128, False)
        c = W.randn_bf16((1, L, 128), 8, device=dev)
        z = W.randn_bf16((1, L, 128), 9, device=dev)
        bias = W.randn_bf16((2 * m if overlap else m, 128), 10, device=dev, std=0.1)
        for _ in range(2):
            if overlap:
                C.csa_compress(c, z, bias, m=m)
            else:
                C.hca_compress(c, z, bias, m_prime=m)
    elif name in ("csa_decode", "hybrid_decode"):   # the full decode workloads (about 1-1.4 GB on the device)
        wl = Decode(C, dev, 0, name)
        for _ in range(2):
            wl.step()
    else:
        raise SystemExit(f"unknown profile case {name}")
    torch.cuda.synchronize()
    C.sync_status()
    print("ok", name)


# DRAM bytes (read + write) per launch from one ncu capture of a smaller case
# (profiles/), scaled by the tokens a launch processes; valid only while the
# kernel source is the one that was measured.
MEASURED_TRAFFIC = {
    "sparse": {"src": "sparse_attn_sm100.cu",
               "sha256": "cda61cee7a0fdc35704200d66d5b4d744ea8af7d444108eee9d43312f00d39be",
               "bytes_per_token": (172.049920e6 + 100.580352e6) / 8192},
    "dense": {"src": "dense_attn_sm100.cu",
              "sha256": "c973b4b6687b01d616c69815ea7577dcb6608b99ea5a390f0bafd7de8f99b29a",
              "bytes_per_token": (271.014400e6 + 220.154624e6) / 16384},
    "front_end": {"src": "front_end_sm100.cu",
                  "sha256": "5690b1b7653aa1670ccd6b0fa5174caa3af789ce22d347caf149faa33f399ac7",
                  "bytes_per_token": (249.420800e6 + 3.766784e6) / 16384},
    # decode: the DRAM bytes of one whole step (all its launches, serialised
    # under ncu), so the unit is the step
    "csa_decode": {"src": "decode.cu",
                   "sha256": "79b227ff000d5a97fe43664dbc79b989fe701a21b6cf71614ea721f8ac94d586",
                   "bytes_per_token": 305214464.0},
    "hybrid_decode": {"src": "decode.cu",
                      "sha256": "79b227ff000d5a97fe43664dbc79b989fe701a21b6cf71614ea721f8ac94d586",
                      "bytes_per_token": 615825664.0},
}


def measured_traffic(kind, tokens):
    import hashlib
    t = MEASURED_TRAFFIC[kind]
    path = os.path.join(ROOT, "compressed_sparse_long_compress_b200", "csrc", t["src"])
    try:
        h = hashlib.sha256(open(path, "rb").read()).hexdigest()
    except OSError:
        return None
    return t["bytes_per_token"] * tokens if h == t["sha256"] else None


# ----------------------------------------------------------- CPU baseline

def oracle_sample(name, budget_s=10.0, one_thread_s=0.0):
    """The C++ float64 oracle (OpenMP over query rows / sequences), as it
    stands, on a bounded sample of the workload, on this host's cores.
    Returns a dict: value (the workload's unit), threads, sample description,
    and (when one_thread_s > 0) the same measure on one thread."""
    from oracle import cpp_oracle as CO
    f = lambda t: t.double().numpy()
    threads = CO.threads()

    def timed(fn):
        t0 = time.perf_counter()
        fn()
        return time.perf_counter() - t0

    res = {"threads": threads}
    if name in ("csa_prefill", "tiny"):
        wl = W.WORKLOADS[name]
        s = wl.csa
        x = W.prefill_inputs(s, wl.wid)
        c, z, bias, k_idx = f(x["c"]), f(x["z"]), f(x["pos_bias"]), f(x["k_idx"])
        box = {}
        t_comp = timed(lambda: box.setdefault("e", CO.compress(c, z, bias, s.m, True)))
        e = box["e"]
        rng = np.random.default_rng(5)

        def rows_batch(n_rows, budget):
            done, t = 0, 0.0
            while t < budget and done < s.L:
                rows = np.sort(rng.integers(0, s.L, n_rows))
                rt = torch.as_tensor(rows)
                qi, ww, qq = f(x["q_idx"][:, rt]), f(x["w"][:, rt]), f(x["q"][:, rt])
                t1 = time.perf_counter()
                sc = CO.indexer_scores(qi, ww, k_idx, s.m, rows=rows, compact=True)
                idx = CO.topk_select(sc, s.m, s.topk, rows=rows)
                CO.sparse_attention(qq, e, idx, s.scale)
                t += time.perf_counter() - t1
                done += n_rows
            return done, t

        done, t_rows = rows_batch(max(8, 8 * threads), budget_s)
        res["value"] = 1.0 / (t_rows / done + t_comp / s.L)
        res["unit"] = "tokens/s"
        res["sample"] = (f"C++ oracle: compression of all {s.L} tokens ({t_comp:.2f} s) + indexer, top-k and sparse "
                         f"attention for {done} uniformly drawn query rows ({t_rows:.1f} s); "
                         "tokens/s = 1 / (mean row time + compression time / L)")
        if one_thread_s > 0:
            CO.set_threads(1)
            t_comp1 = timed(lambda: CO.compress(c[:, :4096], z[:, :4096], bias, s.m, True)) * (s.L / 4096)
            done1, t1 = rows_batch(4, one_thread_s)
            CO.set_threads(threads)
            res["value_1thread"] = 1.0 / (t1 / done1 + t_comp1 / s.L)
        return res
    if name == "front_end_prefill":
        wl = W.WORKLOADS[name]
        s = wl.front_end
        x = W.front_end_inputs(s, wl.wid)
        Wt, bias = f(x["W"]), f(x["pos_bias"])
        rng = np.random.default_rng(7)
        done, t_e = 0, 0.0
        while t_e < budget_s:
            i = int(rng.integers(1, s.n_c))
            toks = f(x["h"][:, (i - 1) * s.m:(i + 1) * s.m])
            t1 = time.perf_counter()
            CO.compressor_front_end(toks, Wt, bias, s.m, True)
            t_e += time.perf_counter() - t1
            done += 1
        res["value"] = s.m / (t_e / done)   # every entry advances the sequence by m tokens
        res["unit"] = "tokens/s"
        res["sample"] = (f"C++ oracle: projections and compression of {done} uniformly drawn entries, each from its "
                         f"own 2m = {2 * s.m}-token window ({t_e:.1f} s); tokens/s = m / mean entry time (the 2x "
                         "projection overlap of adjacent windows is counted as work)")
        return res
    if name == "hca_prefill":
        wl = W.WORKLOADS[name]
        s = wl.hca
        n_tok = 65536   # compression timed on the first 65536 tokens and scaled to L
        c = f(W.randn_bf16((1, n_tok, 128), W.seed_of(wl.wid, W.T_C)))
        z = f(W.randn_bf16((1, n_tok, 128), W.seed_of(wl.wid, W.T_Z)))
        bias = f(W.randn_bf16((s.m, 128), W.seed_of(wl.wid, W.T_BIAS), std=0.1))
        t_comp = timed(lambda: CO.compress(c, z, bias, s.m, False)) * (s.L / n_tok)
        e = np.random.default_rng(1).standard_normal((1, s.n_c, 128)) * 0.4
        rng = np.random.default_rng(6)
        done, t_rows, batch = 0, 0.0, max(4, 2 * threads)
        while t_rows < budget_s:
            rows = np.sort(rng.integers(0, s.L, batch))
            qv = W.randn_bf16((1, batch, s.H, 128), 77 + done).double().numpy()
            t1 = time.perf_counter()
            CO.dense_causal_attention(qv, e, s.m, s.scale, rows=rows, compact=True)
            t_rows += time.perf_counter() - t1
            done += batch
        res["value"] = 1.0 / (t_rows / done + t_comp / s.L)
        res["unit"] = "tokens/s"
        res["sample"] = (f"C++ oracle: compression of {n_tok} tokens scaled to {s.L} ({t_comp:.1f} s scaled) + dense "
                         f"causal attention for {done} uniformly drawn query rows ({t_rows:.1f} s; q rows and "
                         "entries drawn N(0,1) / N(0,0.4^2) from their own seeds)")
        return res
    wl = W.WORKLOADS[name]
    d = wl.decode
    n_seq = min(d.B, 8 if d.B > 8 else 2)
    t_total = 0.0
    for li, kind in enumerate(d.kinds):
        sub = W.DecodeShape(B=n_seq, H=d.H, kinds=d.kinds, n_entries=d.n_entries, topk=d.topk)
        x = W.decode_layer_inputs(sub, li, wl.wid)   # the workload's first n_seq sequences
        codes, rope, scale = CO.quantize_kv_mixed(f(x["kv"]))
        hat = CO.dequantize_kv_mixed(codes, rope, scale)
        del codes, rope, x["kv"]
        n = [d.n_entries[li]] * n_seq
        if kind == "csa":
            qq, qi, ww, kk = f(x["q"]), f(x["q_idx"]), f(x["w"]), f(x["k_idx"])
            t_total += timed(lambda: CO.decode_csa_layer(qq, qi, ww, kk, hat, n, d.topk, d.scale))
        else:
            qq = f(x["q"])
            t_total += timed(lambda: CO.decode_hca_layer(qq, hat, n, d.scale))
        del hat
    res["value"] = t_total * (d.B / n_seq) * 1e6
    res["unit"] = "us/step"
    res["sample"] = (f"C++ oracle decode step (indexer, top-k and attention of every layer) for {n_seq} of the "
                     f"{d.B} sequences, scaled x{d.B // n_seq}; KV quantisation to the mixed layout not timed")
    return res


def cpu_baseline_entry(name, budget_s, one_thread_s=0.0):
    r = oracle_sample(name, budget_s, one_thread_s)
    out = {"value": r["value"], "unit": r["unit"], "cores": r["threads"], "kind": "oracle",
           "impl": "C++ float64 oracle, OpenMP", "sample": r["sample"]}
    if "value_1thread" in r:
        out["value_1thread"] = r["value_1thread"]
    return out


# the pages' own efficiency figures (model level, no hardware stated): context only
PAGES_CONTEXT = ("pages (first page intro; NARR 混合注意力革命): at 1M-token context DeepSeek-V4-Pro needs 27% of "
                 "V3.2's per-token inference FLOPs (FP8-equivalent) and 10% of its KV cache; V4-Flash 10% and 7%. "
                 "Model-level ratios, no hardware stated; not kernel numbers.")


# --------------------------------------------------------------------- main

def run_reference(args, world, rank):
    if rank != 0:
        return
    name = args.workload
    vals = []
    last = None
    budget = max(2.0, 60.0 / max(1, args.steps + args.warmup))
    for i in range(args.warmup + args.steps):
        r = oracle_sample(name, budget_s=budget)
        if i >= args.warmup:
            vals.append(r["value"])
        last = r
    v = float(np.mean(vals))
    unit = last["unit"]
    line = {"impl": "reference", "metric": "CSA+HCA prefill tokens/s and 1M-ctx decode us/step; % of TC/HBM roofline",
            "value": v, "unit": unit, "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "higher_is_better": unit == "tokens/s", "dtype": "f64", "data": "synthetic",
            "config": dict(workload_config(name), parallelism="rank 0 alone (host cores)"), "vs_baseline": None,
            "cpu_baseline": {"value": v, "unit": unit, "cores": last["threads"], "kind": "oracle",
                             "impl": "C++ float64 oracle, OpenMP", "sample": last["sample"]},
            "e2e": {"value": v, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=60)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="csa_prefill", choices=list(W.WORKLOADS))
    ap.add_argument("--secondary", default="all", choices=["none", "all"])
    ap.add_argument("--cpu-budget", type=float, default=12.0,
                    help="seconds of timed oracle work for the headline's CPU baseline (a third for each secondary)")
    ap.add_argument("--profile-case", default=None, choices=["sparse_attn_L8192", "dense_attn_L65536", "topk_L8192", "indexer_L8192",
                                                              "csa_decode", "hybrid_decode", "front_end_L16384", "dense_attn_steady",
                                                              "compress_L65536", "compress_hca_L1M"],
                    help="run one small kernel case for an ncu capture and exit")
    args = ap.parse_args()
    if args.profile_case:
        profile_case(args.profile_case)
        return
    if args.warmup < 3:
        args.warmup = 3

    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, world, rank)
        return

    from compressed_sparse_long_compress_b200 import cslc as C
    world, rank, local = dist_setup(args.gpus)
    peaks = load_peaks()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=torch.device("cuda", local))

    head = measure(args.workload, C, args, world, rank, local, peaks, flush)
    secondary = {}
    if args.secondary == "all" and args.workload == "csa_prefill":
        for name in ("hca_prefill", "front_end_prefill", "csa_decode", "hybrid_decode"):
            r = measure(name, C, args, world, rank, local, peaks, flush, with_e2e=False, min_timed_ms=500.0)
            secondary[name] = {k: r[k] for k in ("value", "unit", "ms_per_step", "kernel_ms", "roofline",
                                                  "clocks", "config", "steps", "gpu_launches",
                                                  "gpu_launches_per_step", "gpu_launches_counted")}
        secondary["indexer_topk_variants"] = measure_indexer_variants(C, torch.device("cuda", local), flush)

    # the launch counts, measured after all timing (the profiler stays out of
    # every timed region): one untimed step of each workload
    for res_name, res in [(args.workload, head)] + list(secondary.items()):
        if "gpu_launches_per_step" not in res:
            continue
        wl = make_workload(res_name, C, torch.device("cuda", local), rank)
        per_step = count_launches(wl)
        del wl
        torch.cuda.empty_cache()
        if per_step is not None:
            res["gpu_launches"] = per_step * res["steps"]
            res["gpu_launches_per_step"] = per_step
            res["gpu_launches_counted"] = True

    cpu = None
    if rank == 0 and world == 1:
        cpu = cpu_baseline_entry(args.workload, budget_s=args.cpu_budget, one_thread_s=args.cpu_budget / 4)
        for name in secondary:
            if name in W.WORKLOADS:   # the bf16-score entry is a variant of the headline's indexer
                secondary[name]["cpu_baseline"] = cpu_baseline_entry(name, budget_s=args.cpu_budget / 3)

    if rank == 0:
        line = {"metric": "CSA+HCA prefill tokens/s and 1M-ctx decode us/step; % of TC/HBM roofline",
                "value": head["value"], "unit": head["unit"], "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
                "higher_is_better": head["higher_is_better"], "scaling": "weak", "vs_baseline": None,
                "dtype": "bf16", "data": "synthetic (seeded N(0,1)/U(0,1) inputs of the workload's shapes)",
                "config": dict(head["config"], parallelism=f"independent sequences x{world}"),
                "e2e": head.get("e2e"), "gpu_launches": head["gpu_launches"],
                "gpu_launches_per_step": head["gpu_launches_per_step"],
                "gpu_launches_counted": head["gpu_launches_counted"], "clocks": head["clocks"],
                "roofline": head["roofline"], "cpu_baseline": cpu, "workloads": secondary,
                "peaks": peaks, "context": PAGES_CONTEXT}
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
