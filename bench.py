"""Benchmark of the MoE layer forward hot path (libmoe.so) on B200.

Default workload: the fine-grained MoE layer (T=4096, H=4096, E=256, k=8, I=2048, bf16,
capacity factor 1.25), the configuration the headline metric is quoted on. One step = one
moe_layer_forward (route -> align -> GEMM1 -> GEMM2 -> combine) over the whole batch.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 runs under torchrun as independent replicas (one process per GPU, no data-path
collective); timing is the max over ranks. Rank 0 prints one JSON line.

    python bench.py --sweep route-align-combine --workload skewed [--sweep-tokens 4096,...]

times the router, the grouping and the combine alone over a range of T (one GPU) and prints
one JSON line with each stage's HBM GB/s.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from expert_dispatch_gate_b200 import _lib as L  # noqa: E402
from expert_dispatch_gate_b200 import layer as M  # noqa: E402
from expert_dispatch_gate_b200 import workloads as W  # noqa: E402

METRIC = "MoE-layer tokens/s (E=256,k=8,T=4096,1 GPU); route+align+combine HBM GB/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
STAGES = ["route", "align", "gemm1", "gemm2", "combine"]
L2_BYTES = 126 << 20  # B200 L2


# ------------------------------------------------------------------ distributed plumbing

def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        kw = {"timeout": datetime.timedelta(seconds=120)}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, **kw)
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(value, world, device="cpu"):
    """Max of a per-rank float over all ranks (identity for one rank)."""
    if world == 1:
        return float(value)
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_throughput(units_per_rank, n_ranks, max_seconds):
    """Whole-job throughput: units processed by all ranks / the slowest rank's time."""
    return units_per_rank * n_ranks / max_seconds


# ------------------------------------------------------------------ clocks (NVML)

class ClockSampler:
    """Samples SM clock and throttle reasons through NVML every few ms while running."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting",
    }

    def __init__(self, index, period_s=0.005):
        self.index, self.period = index, period_s
        self.samples, self.reasons = [], 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:  # NVML missing: clocks reported as unavailable
            self.ok = False

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= int(self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._t is not None:
            self._t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples)}


# ------------------------------------------------------------------ algorithmic cost model

def stage_costs(wl, counts, hbm_peak, tc_peak, fp8_weights=False, fp8_acts=False):
    """Algorithmic bytes/flops per stage for one step, from the step's routing counts. With
    e4m3 expert weights a weight element is 1 byte, plus a float32 scale per output channel.
    With e4m3 activations too (W8A8), x is read once to be quantised, the GEMMs read e4m3 token
    rows, and the SwiGLU intermediate is stored once and read once as e4m3 (its bf16 copy before
    quantisation is implementation traffic)."""
    es = 2 if wl.dtype == "bf16" else 4
    T, H, E, k, I = wl.T, wl.H, wl.E, wl.k, wl.I
    A = T * k
    a_kept = int(counts.sum())
    used = int((counts > 0).sum())
    bias = E * 4 if wl.zipf_s > 0 else 0
    wes, ws_ = (1, 4) if fp8_weights else (es, 0)  # weight element bytes, scale bytes
    c = {
        "route": {"bytes": T * H * es + H * E * es + bias + T * k * 8, "flops": 2 * T * H * E},
        # read the expert ids once; write sorted_ids, slot_of and the drop mask; counts, offsets
        "align": {"bytes": A * 4 + A * (4 + 4 + 1) + E * 8, "flops": 0},
        "gemm1": {"bytes": used * 2 * H * I * wes + used * 2 * I * ws_ + a_kept * H * es
                           + a_kept * I * es,
                  "flops": 4 * a_kept * H * I},
        "gemm2": {"bytes": used * I * H * wes + used * H * ws_ + a_kept * I * es + a_kept * H * es,
                  "flops": 2 * a_kept * I * H},
        "combine": {"bytes": a_kept * H * es + T * k * 8 + T * H * es, "flops": 2 * a_kept * H},
    }
    if fp8_acts:
        c["gemm1"]["bytes"] = (used * 2 * H * I + used * 2 * I * 4 + T * H * es + a_kept * H
                               + a_kept * I)
        c["gemm2"]["bytes"] = used * I * H + used * H * 4 + a_kept * I + a_kept * H * es
    for v in c.values():
        v["t_hbm_us"] = v["bytes"] / (hbm_peak * 1e9) * 1e6
        v["t_tc_us"] = v["flops"] / (tc_peak * 1e12) * 1e6
    return c


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash():
    h = hashlib.sha256()
    for f in ("ffn_tc.cu", "common.cuh"):
        with open(os.path.join(ROOT, "expert_dispatch_gate_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel, workload):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on this source."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    ent = d.get(f"{kernel}@{workload}")
    if not ent or ent.get("source_hash") != kernel_source_hash():
        return None
    return ent.get("dram_bytes_per_launch")


# ------------------------------------------------------------------ CPU oracle timing

def oracle_sample_time(wl, host, weights, n_tokens, seed=0):
    """Time the oracle on a bounded sample: routing + capacity grouping over all T tokens
    (the grouping depends on every token), the expert FFN + combine on n_tokens sampled
    tokens. Returns (seconds_route_align, seconds_ffn_combine, tokens_sampled)."""
    from oracle import moe_oracle as orc
    t0 = time.perf_counter()
    logits = orc.router_logits(host["x"], host["w_router"], host["logit_bias"])
    idx = orc.select_topk(logits, wl.k)
    w = orc.route_weights(logits, idx)
    C = orc.capacity(wl.T, wl.k, wl.E, wl.capacity_factor)
    al = orc.align(idx, wl.E, C)
    t1 = time.perf_counter()
    rng = np.random.default_rng(seed)
    toks = sorted(rng.choice(wl.T, size=min(n_tokens, wl.T), replace=False).tolist())
    need = sorted({int(al["slot_of"][t * wl.k + j]) for t in toks for j in range(wl.k)
                   if al["slot_of"][t * wl.k + j] >= 0})
    y = orc.grouped_ffn_slots(host["x"], al["sorted_ids"], al["offsets"], wl.k, weights[0],
                              weights[1], weights[2], slots=need)
    orc.combine(y, al["slot_of"], w, tokens=toks)
    t2 = time.perf_counter()
    return t1 - t0, t2 - t1, len(toks)


class HostExperts:
    """Expert matrices of the sampled experts, copied to host memory in their own dtype before
    timing; the widening to float64 happens on access, inside the timed oracle call."""

    def __init__(self, w, experts):
        self.m = {int(e): w[int(e)].cpu() for e in experts}

    def __getitem__(self, e):
        return self.m[int(e)].double().numpy()


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def oracle_baseline(wl, dev, n_tokens, reps=1):
    from oracle import moe_oracle as orc
    host = {"x": dev["x"].float().cpu().numpy(), "w_router": dev["w_router"].float().cpu().numpy(),
            "logit_bias": None if dev["logit_bias"] is None else dev["logit_bias"].cpu().numpy()}
    # which experts the sample touches (routing recomputed inside the timed call)
    logits = orc.router_logits(host["x"], host["w_router"], host["logit_bias"])
    idx = orc.select_topk(logits, wl.k)
    rng = np.random.default_rng(0)
    toks = rng.choice(wl.T, size=min(n_tokens, wl.T), replace=False)
    experts = sorted(set(idx[toks].reshape(-1).tolist()))
    weights = [HostExperts(dev[n], experts) for n in ("w_gate", "w_up", "w_down")]
    best = None
    for _ in range(reps):
        r = oracle_sample_time(wl, host, weights, n_tokens)
        best = r if best is None or sum(r[:2]) < sum(best[:2]) else best
    t_ra, t_ffn, s = best
    per_token = t_ra / wl.T + t_ffn / s
    return {"value": 1.0 / per_token, "unit": "tokens/s", "cores": cpu_threads(),
            "kind": "oracle",
            "sample": (f"float64 NumPy oracle: routing + capacity grouping timed over all {wl.T} "
                       f"tokens ({t_ra:.2f} s), expert SwiGLU FFN + combine timed on {s} sampled "
                       f"tokens ({t_ffn:.2f} s); tokens/s = 1 / (t_route_align/T + t_ffn/{s})")}


# ------------------------------------------------------------------ the GPU arm

def route_ksplit(T, H, E):
    """K ranges of the tensor-core gate GEMM (the library's rule): split while about 128 CTAs
    or fewer run and each range keeps at least 4 k-blocks of 64."""
    kb_total = H // 64
    ctas = 2 * ((T + 255) // 256) if E % 128 == 0 else (T + 127) // 128
    ks = 1
    while (ks * 2 <= 16 and kb_total % (ks * 2) == 0 and kb_total // (ks * 2) >= 4
           and ctas * ks * 2 <= 128):
        ks *= 2
    return ks


def launches_per_step(wl, weights="bf16"):
    """Kernels one moe_layer_forward launches: router (tensor-core gate GEMM + top-k; one
    persistent kernel for both when E is 64, 128 or 256 and the hidden dimension is one K range;
    one CUDA-core kernel for E < 64 or f32), align (one launch; three past the cooperative grid's
    capacity of SMs x 1024 threads x 64 rounds of 32), the expert-major row copy (bf16), the
    W8A8 quantisations, the expert GEMMs, combine."""
    tc = wl.dtype == "bf16" and wl.E >= 64 and wl.E % 8 == 0
    fused = (tc and (wl.E == 64 or (wl.E % 128 == 0 and wl.E <= 256)) and wl.k <= 16
             and route_ksplit(wl.T, wl.H, wl.E) == 1)
    route = 2 if tc and not fused else 1
    align = 1 if wl.T * wl.k <= 148 * 1024 * 64 * 32 else 3
    # expert-major copy of the token rows before GEMM1: every bf16 layer (GEMM1 runs on CTA
    # pairs, and the e4m3-weight GEMM1 reads the copy too)
    copy = 1 if wl.dtype == "bf16" else 0
    # W8A8: the token rows and the SwiGLU rows are quantised by one launch each
    quant = 2 if weights == "w8a8" else 0
    # bf16 GEMM1 on CTA pairs with I % 256 == 128: the last 128 features on single CTAs
    gemm1 = 2 if (wl.dtype == "bf16" and weights == "bf16" and wl.I % 256 == 128
                  and wl.I >= 384) else 1
    return route + align + copy + quant + gemm1 + 1 + 1


def workload_of(args):
    wl = W.WORKLOADS.get(args.workload) or W.PROFILE_WORKLOADS[args.workload]
    return wl.with_tokens(args.tokens) if args.tokens else wl


def layer_config(wl, capacity, world, weights="bf16"):
    """The `config` object of a layer line; the reference arm prints the same keys."""
    fp8 = weights in ("fp8", "w8a8")
    wes = 1 if fp8 else (2 if wl.dtype == "bf16" else 4)
    wb = 3 * wl.E * wl.H * wl.I * wes
    return {"workload": wl.describe(), "T": wl.T, "H": wl.H, "E": wl.E, "k": wl.k, "I": wl.I,
            "capacity": int(capacity),
            "parallelism": "replicas" if world > 1 else "single-gpu",
            "expert_weights": {"fp8": "e4m3 codes + float32 per-channel scales (W8A16)",
                               "w8a8": "e4m3 codes + float32 per-channel scales, e4m3 "
                                       "activations with float32 per-row scales (W8A8)"}.get(
                                           weights, wl.dtype),
            "l2": (("inputs larger than L2: %.1f GB of expert weights streamed per step"
                    % (wb / 1e9)) if wb > L2_BYTES else
                   "inputs fit in L2 (%.1f MB of expert weights); L2 not flushed" % (wb / 1e6))}


class LayerRun:
    """One workload's layer on the device: inputs, outputs, workspace and the forward call."""

    def __init__(self, wl, dev, fp8=False, w8a8=False):
        self.wl, self.dev = wl, dev
        self.inp = W.make_inputs(wl, dev)
        self.shape = M.shape_of(wl.T, wl.H, wl.E, wl.k, wl.I, wl.capacity_factor, wl.dtype)
        self.ws = M.Workspace(self.shape, dev)
        self.outs = [torch.empty((wl.T, wl.H), dtype=wl.torch_dtype, device=dev),
                     torch.empty((wl.T, wl.k), dtype=torch.int32, device=dev),
                     torch.empty((wl.T, wl.k), dtype=torch.float32, device=dev),
                     torch.empty(wl.E, dtype=torch.int32, device=dev),
                     torch.empty(wl.T * wl.k, dtype=torch.uint8, device=dev)]
        self.stream = torch.cuda.current_stream(dev)
        self.fp8 = None
        self.w8a8 = None
        if fp8:
            # e4m3 expert weights, quantised once on the device before anything is timed
            self.fp8 = M.Fp8Weights(self.inp["w_gate"], self.inp["w_up"], self.inp["w_down"])
            torch.cuda.synchronize()
        if w8a8:
            # K-major e4m3 expert weights, packed once on the device before anything is timed
            self.w8a8 = M.W8A8Weights(self.inp["w_gate"], self.inp["w_up"], self.inp["w_down"])
            torch.cuda.synchronize()

    def forward(self, x, o):
        inp, ws = self.inp, self.ws
        if self.w8a8 is not None:
            L.moe_layer_forward_w8a8(self.shape, None, x, inp["w_router"], inp["logit_bias"],
                                     *self.w8a8.args(), o[0], None, o[1], o[2], o[3], o[4],
                                     ws.buf, ws.nbytes, self.stream)
        elif self.fp8 is not None:
            L.moe_layer_forward_w8(self.shape, None, x, inp["w_router"], inp["logit_bias"],
                                   *self.fp8.args(), o[0], None, o[1], o[2], o[3], o[4], ws.buf,
                                   ws.nbytes, self.stream)
        else:
            L.moe_layer_forward(self.shape, x, inp["w_router"], inp["logit_bias"], inp["w_gate"],
                                inp["w_up"], inp["w_down"], o[0], None, o[1], o[2], o[3], o[4],
                                ws.buf, ws.nbytes, self.stream)

    def step(self):
        self.forward(self.inp["x"], self.outs)

    def _stage_pass(self, steps):
        """`steps` layer calls with the library's stage events; mean ms per stage."""
        stream = self.stream
        starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        ev = [[torch.cuda.Event(enable_timing=True) for _ in STAGES] for _ in range(steps)]
        for e in ev:
            for x in e:
                x.record(stream)
        for s in starts:
            s.record(stream)
        torch.cuda.synchronize()
        for i in range(steps):
            starts[i].record(stream)
            L.moe_set_stage_events(ev[i])
            self.step()
        torch.cuda.synchronize()
        L.moe_set_stage_events(None)
        self.ws.check()
        st_ms = {s: 0.0 for s in STAGES}
        for i in range(steps):
            prev = starts[i]
            for j, s in enumerate(STAGES):
                st_ms[s] += prev.elapsed_time(ev[i][j]) / steps
                prev = ev[i][j]
        return st_ms

    def graph_time(self, steps, warmup, world):
        """The same layer call captured once in a CUDA graph (on a side stream) and replayed
        per step, as a serving loop for short batches would run it: the launches' host cost and
        the gaps between them leave the timed region. Returns ms per step (max over ranks)."""
        side = torch.cuda.Stream(self.dev)
        side.wait_stream(torch.cuda.current_stream(self.dev))
        saved = self.stream
        self.stream = side
        with torch.cuda.stream(side):
            self.step()  # first call on this stream: tensor maps and attributes set up
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=side):
            self.step()
        self.stream = saved
        for _ in range(warmup):
            graph.replay()
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize()
        a.record()
        for _ in range(steps):
            graph.replay()
        b.record()
        torch.cuda.synchronize()
        self.ws.check()
        del graph
        return max_over_ranks(a.elapsed_time(b), world, "cuda") / steps

    def time_stages(self, steps, warmup, world, local, peaks):
        """Device-resident timing. Pass 1, the timed region: total CUDA-event time over `steps`
        layer calls (max over ranks), the calls as a user makes them, so each kernel's launch
        still overlaps the end of the one before it (programmatic dependent launch). Pass 2
        (once before and once after pass 1, the smaller total kept): the same calls with the
        per-stage events the library records on its stream; an event between two kernels ends
        that overlap, so the stage times sum to a little more than pass 1's step. Returns the
        layer line's timing keys."""
        wl, stream = self.wl, self.stream
        for _ in range(warmup):
            self.step()
        torch.cuda.synchronize()
        self.ws.check()
        stages_before = self._stage_pass(steps)
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize()
        with ClockSampler(local) as clk:
            t_start.record(stream)
            for i in range(steps):
                # an NVTX range per layer call, for timeline profilers
                torch.cuda.nvtx.range_push(f"moe_layer_forward step {i}")
                self.step()
                torch.cuda.nvtx.range_pop()
            t_end.record(stream)
            torch.cuda.synchronize()
        barrier(world)
        ms = t_start.elapsed_time(t_end)
        self.ws.check()
        ms_max = max_over_ranks(ms, world, "cuda")
        value = aggregate_throughput(wl.T * steps, world, ms_max / 1e3)
        # pass 2, run once before and once after pass 1: per-stage events. A pass disturbed by
        # something outside the layer (the box's power or clock state) shows as a larger total;
        # the breakdown reported is the pass with the smaller total.
        stages_after = self._stage_pass(steps)
        st_ms = min(stages_before, stages_after, key=lambda d: sum(d.values()))
        cnt = self.outs[3].cpu().numpy()
        fp8 = self.fp8 is not None or self.w8a8 is not None
        # the tensor-core peak of the MMA's own operand type: e4m3 x e4m3 (W8A8) runs at the
        # nominal 2x of bf16 (4.5 against 2.25 PFLOP/s dense), so the measured bf16 peak x 2
        tc_ratio, tc_name = (2.0, "2 x bf16_tflops_sustained (e4m3 MMA)") \
            if self.w8a8 is not None else (1.0, "bf16_tflops_sustained")
        tc_peak = peaks["bf16_tflops_sustained"] * tc_ratio
        cost = stage_costs(wl, cnt, peaks["hbm_gbs"], tc_peak, fp8_weights=fp8,
                           fp8_acts=self.w8a8 is not None)
        kernels = {}
        for s in STAGES:
            t = st_ms[s] * 1e-3
            kernels[s] = {"us": round(st_ms[s] * 1e3, 2),
                          "gbs": round(cost[s]["bytes"] / t / 1e9, 1),
                          "tflops": round(cost[s]["flops"] / t / 1e12, 1),
                          "bytes": cost[s]["bytes"], "flops": cost[s]["flops"],
                          "frac_hbm": round(cost[s]["bytes"] / t / 1e9 / peaks["hbm_gbs"], 3)}
        dom = max(["gemm1", "gemm2"], key=lambda s: st_ms[s])
        t_dom = st_ms[dom] * 1e-3
        bound = "hbm" if cost[dom]["t_hbm_us"] >= cost[dom]["t_tc_us"] else "tensor"
        if bound == "hbm":
            ach, peak, unit = cost[dom]["bytes"] / t_dom / 1e9, peaks["hbm_gbs"], "GB/s"
        else:
            ach, peak, unit = cost[dom]["flops"] / t_dom / 1e12, tc_peak, "TFLOP/s"
        tflops_dom = cost[dom]["flops"] / t_dom / 1e12
        rac_bytes = sum(cost[s]["bytes"] for s in ("route", "align", "combine"))
        rac_t = sum(st_ms[s] for s in ("route", "align", "combine")) * 1e-3
        return {
            "value": value, "ms_max": ms_max, "cnt": cnt, "kernels": kernels, "clocks": clk.summary(),
            "roofline": {"kernel": dom, "bound": bound, "achieved": round(ach, 1), "peak": peak,
                         "unit": unit, "frac": round(ach / peak, 3),
                         "peak_source": "%s (%s)" % (peaks.get("_source", "measured"),
                                                     "hbm_gbs" if bound == "hbm" else tc_name),
                         "algorithmic_bytes": cost[dom]["bytes"],
                         "tensor_frac": round(tflops_dom / tc_peak, 3),
                         "tensor_frac_burst": round(tflops_dom / (peaks["bf16_tflops"] * tc_ratio),
                                                    3)},
            "route_align_combine_gbs": round(rac_bytes / rac_t / 1e9, 1),
            "route_align_combine_frac": round(rac_bytes / rac_t / 1e9 / peaks["hbm_gbs"], 3),
            # per-step sums of the two stage passes (before, after the timed pass), in ms
            "stage_passes_ms": [round(sum(stages_before.values()), 4),
                                round(sum(stages_after.values()), 4)],
        }

    def release(self):
        del self.inp, self.ws, self.outs, self.fp8, self.w8a8
        torch.cuda.empty_cache()


def other_workloads(args, dev, world, local, peaks):
    """The other layer configurations, timed the same way as the headline (device-resident
    inputs, stage events): Mixtral-shaped, skewed-load, and the decode sweep."""
    res = {}
    cases = [("mixtral", W.WORKLOADS["mixtral"]), ("skewed", W.WORKLOADS["skewed"])]
    cases += [(f"decode_T{t}", W.WORKLOADS["decode"].with_tokens(t)) for t in W.DECODE_TOKENS]
    for key, wl in cases:
        run = LayerRun(wl, dev)
        t = run.time_stages(args.steps, args.warmup, world, local, peaks)
        res[key] = {"workload": wl.describe(), "value": round(t["value"], 1), "unit": "tokens/s",
                    "ms_per_step": round(t["ms_max"] / args.steps, 4),
                    "stage_us": {s: t["kernels"][s]["us"] for s in STAGES},
                    "roofline": t["roofline"],
                    "route_align_combine_gbs": t["route_align_combine_gbs"],
                    "kept_assignments": int(t["cnt"].sum()),
                    "experts_used": int((t["cnt"] > 0).sum()),
                    "gpu_launches": launches_per_step(wl) * args.steps}
        if wl.T <= 256:
            # decode batches are launch-bound: also the call captured in a CUDA graph
            ms = run.graph_time(args.steps, args.warmup, world)
            res[key]["graph"] = {"value": round(aggregate_throughput(wl.T * args.steps, world,
                                                                     ms * args.steps / 1e3), 1),
                                 "unit": "tokens/s", "ms_per_step": round(ms, 4),
                                 "how": "the layer call captured once in a CUDA graph on a side "
                                        "stream and replayed per step; CUDA events around the "
                                        "replays"}
        run.release()
    return res


def run_ours(args, world, rank, local):
    wl = workload_of(args)
    dev = torch.device("cuda", local)
    peaks, peaks_src = load_peaks()
    peaks["_source"] = peaks_src
    run = LayerRun(wl, dev, fp8=args.weights == "fp8", w8a8=args.weights == "w8a8")
    inp, stream = run.inp, run.stream
    t = run.time_stages(args.steps, args.warmup, world, local, peaks)
    cnt = t["cnt"]
    dom = t["roofline"]["kernel"]
    t["roofline"]["traffic"] = recorded_traffic(
        dom + ("_w8" if run.fp8 is not None else "_w8a8" if run.w8a8 is not None else ""),
        args.workload)

    # End to end through the C ABI with host buffers: every step copies its x in from pinned host
    # memory and its outputs back out. Measured twice: serially (copy in, forward, copy out on one
    # stream) and as a throughput pipeline, where step i+1's copy in and step i-1's copy out run
    # on two copy streams while step i computes (x and the outputs double-buffered on the device).
    x_host = inp["x"].cpu().pin_memory()
    outs_dev = run.outs
    outs_host = [torch.empty(t_.shape, dtype=t_.dtype, pin_memory=True) for t_ in outs_dev]
    x_devs = [torch.empty_like(inp["x"]) for _ in range(2)]
    outs_devs = [outs_dev, [torch.empty_like(t_) for t_ in outs_dev]]
    fwd = run.forward

    def e2e_serial(n):
        for _ in range(n):
            x_devs[0].copy_(x_host, non_blocking=True)
            fwd(x_devs[0], outs_devs[0])
            for h, d in zip(outs_host, outs_devs[0]):
                h.copy_(d, non_blocking=True)

    h2d_stream, d2h_stream = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def e2e_pipelined(n):
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_fwd = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]
        begin = torch.cuda.Event()
        begin.record(stream)
        h2d_stream.wait_event(begin)
        d2h_stream.wait_event(begin)
        for i in range(n):
            b = i % 2
            with torch.cuda.stream(h2d_stream):
                if i >= 2:
                    h2d_stream.wait_event(ev_fwd[b])  # step i-2 has finished reading x_devs[b]
                x_devs[b].copy_(x_host, non_blocking=True)
                ev_in[b].record(h2d_stream)
            stream.wait_event(ev_in[b])
            if i >= 2:
                stream.wait_event(ev_out[b])  # step i-2's outputs have left outs_devs[b]
            fwd(x_devs[b], outs_devs[b])
            ev_fwd[b].record(stream)
            with torch.cuda.stream(d2h_stream):
                d2h_stream.wait_event(ev_fwd[b])
                for h, d in zip(outs_host, outs_devs[b]):
                    h.copy_(d, non_blocking=True)
                ev_out[b].record(d2h_stream)
        for e in ev_out[: min(n, 2)]:
            stream.wait_event(e)

    def timed(fn):
        fn(args.warmup)
        torch.cuda.synchronize()
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        fn(args.steps)
        e1.record(stream)
        torch.cuda.synchronize()
        return max_over_ranks(e0.elapsed_time(e1), world, "cuda")

    e2e_serial_ms = timed(e2e_serial)
    e2e_ms = timed(e2e_pipelined)
    run.ws.check()
    h2d = x_host.numel() * x_host.element_size()
    d2h = sum(t_.numel() * t_.element_size() for t_ in outs_host)

    per_step = launches_per_step(wl, args.weights)
    line = {
        "metric": METRIC,
        "value": round(t["value"], 1),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(t["ms_max"] / args.steps, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": wl.dtype,
        "data": "synthetic (seeded N(0,1) activations, N(0,1/fan_in) weights; no dataset)",
        "config": layer_config(wl, L.moe_capacity(run.shape), world, args.weights),
        "routing": {"kept_assignments": int(cnt.sum()), "experts_used": int((cnt > 0).sum())},
        "roofline": t["roofline"],
        "route_align_combine_gbs": t["route_align_combine_gbs"],
        "route_align_combine_frac": t["route_align_combine_frac"],
        "kernels": t["kernels"],
        "stage_passes_ms": t["stage_passes_ms"],
        "e2e": {"value": round(aggregate_throughput(wl.T * args.steps, world, e2e_ms / 1e3), 1),
                "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "copies": "each step's copies overlap the neighbouring steps' forward passes "
                          "(two copy streams, double-buffered device x and outputs)",
                "serial_value": round(aggregate_throughput(wl.T * args.steps, world,
                                                           e2e_serial_ms / 1e3), 1)},
        "gpu_launches": per_step * args.steps,
        "clocks": t["clocks"],
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = oracle_baseline(wl, inp, args.cpu_sample_tokens)
    run.release()
    del x_devs, outs_devs, outs_dev, inp
    if (world == 1 and args.workload == "fine" and not args.no_other_workloads
            and args.weights == "bf16" and not args.tokens):
        line["other_workloads"] = other_workloads(args, dev, world, local, peaks)
    return line


RAC_SWEEP_TOKENS = (4096, 8192, 16384, 32768, 65536, 131072)


def run_rac_sweep(args, local):
    """route -> align -> combine alone, through the C ABI, on one workload's shape with T swept:
    each stage's CUDA-event time and algorithmic HBM GB/s against the measured copy bandwidth.
    The combine reads seeded synthetic expert outputs (one row per assignment slot). Before
    every step a 256 MB buffer is written so that no stage starts from a warm L2."""
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peaks, peaks_src = load_peaks()
    base = W.WORKLOADS[args.workload]
    tokens = [int(t) for t in args.sweep_tokens.split(",")] if args.sweep_tokens else \
        list(RAC_SWEEP_TOKENS)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stages = ("route", "align", "combine")
    points = []
    with ClockSampler(local) as clk:
        for T in tokens:
            wl = base.with_tokens(T)
            inp = W.make_inputs(wl, dev, weights=False)
            y = W.make_y_slots(wl, dev)
            shape = M.shape_of(wl.T, wl.H, wl.E, wl.k, wl.I, wl.capacity_factor, wl.dtype)
            ws = M.Workspace(shape, dev)
            A = wl.T * wl.k
            idx = torch.empty((wl.T, wl.k), dtype=torch.int32, device=dev)
            wts = torch.empty((wl.T, wl.k), dtype=torch.float32, device=dev)
            counts = torch.empty(wl.E, dtype=torch.int32, device=dev)
            offsets = torch.empty(wl.E + 1, dtype=torch.int32, device=dev)
            sorted_ids = torch.empty(A, dtype=torch.int32, device=dev)
            slot_of = torch.empty(A, dtype=torch.int32, device=dev)
            drop = torch.empty(A, dtype=torch.uint8, device=dev)
            out = torch.empty((wl.T, wl.H), dtype=wl.torch_dtype, device=dev)

            def step(ev=None):
                flush.fill_(1)
                if ev is not None:
                    ev[0].record(stream)
                L.moe_route(shape, inp["x"], inp["w_router"], inp["logit_bias"], None, idx, wts,
                            ws.buf, ws.nbytes, stream)
                if ev is not None:
                    ev[1].record(stream)
                L.moe_align(shape, idx, counts, offsets, sorted_ids, slot_of, drop, ws.buf,
                            ws.nbytes, stream)
                if ev is not None:
                    ev[2].record(stream)
                L.moe_combine(shape, y, slot_of, wts, out, stream)
                if ev is not None:
                    ev[3].record(stream)

            for _ in range(args.warmup):
                step()
            torch.cuda.synchronize()
            evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)]
                   for _ in range(args.steps)]
            for ev in evs:
                step(ev)
            torch.cuda.synchronize()
            ws.check()
            us = {s_: statistics.median(ev[j].elapsed_time(ev[j + 1]) for ev in evs) * 1e3
                  for j, s_ in enumerate(stages)}
            cost = stage_costs(wl, counts.cpu().numpy(), peaks["hbm_gbs"],
                               peaks["bf16_tflops_sustained"])
            pt = {"T": T, "assignments": A, "kept": int(counts.sum().item())}
            for s_ in stages:
                gbs = cost[s_]["bytes"] / (us[s_] * 1e-6) / 1e9
                pt[s_] = {"us": round(us[s_], 2), "bytes": cost[s_]["bytes"],
                          "gbs": round(gbs, 1), "frac": round(gbs / peaks["hbm_gbs"], 3)}
            tot_b = sum(cost[s_]["bytes"] for s_ in stages)
            tot_us = sum(us[s_] for s_ in stages)
            pt["total"] = {"us": round(tot_us, 2), "bytes": tot_b,
                           "gbs": round(tot_b / (tot_us * 1e-6) / 1e9, 1),
                           "frac": round(tot_b / (tot_us * 1e-6) / 1e9 / peaks["hbm_gbs"], 3)}
            points.append(pt)
            del inp, y, ws, out
            torch.cuda.empty_cache()
    return {"sweep": "route_align_combine", "unit": "GB/s",
            "workload": base.describe().split(": ", 1)[1].replace(f"T={base.T} ", ""),
            "peak_hbm_gbs": peaks["hbm_gbs"], "peak_source": peaks_src,
            "timing": f"median of {args.steps} steps after {args.warmup} warm-up, CUDA events "
                      "around each stage, L2 overwritten (256 MB) before every step",
            "points": points, "clocks": clk.summary()}


def run_reference(args, world, rank, local):
    """The reference arm: the CPU oracle itself on the host cores, on the same workload and
    config. Each step is one bounded sample: routing and grouping over all T tokens (capacity
    ranks depend on every token), the expert FFN and combine on `--cpu-sample-tokens` sampled
    tokens (the same sample size as the GPU arm's cpu_baseline). `ms_per_step` is the measured
    wall time of one such sample; `value` extrapolates the sample to tokens/s over the whole
    batch. Under torchrun only rank 0 runs it."""
    if rank != 0:
        return None
    wl = workload_of(args)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    inp = W.make_inputs(wl, dev)
    n_tok = max(1, args.cpu_sample_tokens)
    from oracle import moe_oracle as orc
    host = {"x": inp["x"].float().cpu().numpy(), "w_router": inp["w_router"].float().cpu().numpy(),
            "logit_bias": None if inp["logit_bias"] is None else inp["logit_bias"].cpu().numpy()}
    logits = orc.router_logits(host["x"], host["w_router"], host["logit_bias"])
    idx = orc.select_topk(logits, wl.k)
    C = orc.capacity(wl.T, wl.k, wl.E, wl.capacity_factor)
    rng = np.random.default_rng(0)
    toks = rng.choice(wl.T, size=min(n_tok, wl.T), replace=False)
    experts = sorted(set(idx[toks].reshape(-1).tolist()))
    weights = [HostExperts(inp[n], experts) for n in ("w_gate", "w_up", "w_down")]
    del inp
    for _ in range(args.warmup):
        oracle_sample_time(wl, host, weights, n_tok)
    per, wall = [], []
    for _ in range(args.steps):
        w0 = time.perf_counter()
        t_ra, t_ffn, s = oracle_sample_time(wl, host, weights, n_tok)
        wall.append(time.perf_counter() - w0)
        per.append(t_ra / wl.T + t_ffn / s)
    per_token = sum(per) / len(per)
    value = 1.0 / per_token
    sample = (f"per step: float64 NumPy oracle, routing + capacity grouping over all {wl.T} "
              f"tokens, expert SwiGLU FFN + combine on {s} sampled tokens; tokens/s = "
              f"1 / (t_route_align/T + t_ffn/{s})")
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(sum(wall) / len(wall) * 1e3, 3),
        "ms_per_step_extrapolated_to_T": round(per_token * wl.T * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1) activations, N(0,1/fan_in) weights; no dataset)",
        "config": layer_config(wl, C, world),
        "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": cpu_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="fine",
                    choices=sorted(W.WORKLOADS) + sorted(W.PROFILE_WORKLOADS))
    ap.add_argument("--tokens", type=int, default=0, help="override T (decode sweep)")
    ap.add_argument("--cpu-sample-tokens", type=int, default=8)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-other-workloads", action="store_true",
                    help="time only the selected workload (by default a one-GPU run also times "
                         "the Mixtral-shaped, skewed and decode layers under other_workloads)")
    ap.add_argument("--weights", choices=["bf16", "fp8", "w8a8"], default="bf16",
                    help="expert weights: the layer dtype (default), e4m3 + per-channel scales "
                         "(fp8, bf16 activations), or e4m3 weights and activations (w8a8)")
    ap.add_argument("--sweep", choices=["route-align-combine"], default=None,
                    help="time route -> align -> combine alone over a range of T (HBM GB/s per "
                         "stage; one GPU) instead of the layer")
    ap.add_argument("--sweep-tokens", default="",
                    help="comma-separated T values for --sweep (default 4096 ... 131072)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world, rank, local = dist_setup()
    try:
        if args.sweep:
            if world > 1:
                ap.error("--sweep runs on one GPU")
            line = run_rac_sweep(args, local)
        elif args.impl == "reference":
            line = run_reference(args, world, rank, local)
        else:
            line = run_ours(args, world, rank, local)
        if rank == 0 and line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
