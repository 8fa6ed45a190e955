#!/usr/bin/env python
"""Benchmark of the MoM layer hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

A step is one MoM layer forward (router -> permute -> projections -> GDN
shared -> GDN routed -> combine) over the 380M-shape workload: 8 sequences
x 2048 tokens, d_model 1024, 4 heads of d_k = d_v = 256, 4 memories top-2
plus the shared memory, bf16 activations and weights, float32 state.  Inputs
are seeded synthetic tensors already resident in HBM; L2 is flushed (a
256 MiB write) before every timed step, outside its events.  The recurrent
decode step (256 sequences, 8 memories top-2, one new token per sequence,
float32 states of 2.4 GB, larger than L2) is timed in the same run and
reported under "decode".  The other forward workloads (the tiny float32
layer, the skewed-routing varlen batch and the 1.3B-shape 16-memory layer)
are timed the same way and reported under "configs".

With N > 1 (torchrun, one rank per GPU) every rank runs its own batch of
sequences: the layer shards by sequence with no collective on the data
path (weak scaling); the step time is the max over ranks.

`--impl reference` times the CPU oracle (fp64 numpy) on bounded samples of
the same workload instead: rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import time

# NCCL writes its version / debug lines to stdout when NCCL_DEBUG asks for
# them; the result line must be the only line on stdout, so they go to stderr
os.environ.setdefault("NCCL_DEBUG_FILE", "/dev/stderr")

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "MoM layer fwd tokens/s at 1 B200 and % of roofline; decode tokens/s"
UNIT = "tokens/s"
FWD = "mom380m"
DEC = "decode_b256"
# (workload, memory rule, per-memory gates): the other forward workloads, the
# 380M shape with the scalar-gated linear memories, and with per-memory gates
EXTRA = (("tiny_fp32", "gated_delta", False), ("mom380m_skew_varlen", "gated_delta", False),
         ("mom1p3b_m16", "gated_delta", False), ("mom380m", "gated_linear", False), ("mom380m", "gated_delta", True))


def extra_key(name, rule, mem_gates):
    return name + ("" if rule == "gated_delta" else "_" + rule) + ("_mem_gates" if mem_gates else "")
TIE_GAP = 1e-4
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def workload_desc(w):
    if w.varlen_total:
        toks = "%d packed tokens, sequence lengths U{%d..%d}" % (w.varlen_total, w.varlen_min, w.varlen_max)
    else:
        toks = "B=%d x T=%d tokens" % (w.batch, w.seq_len)
    bias = ", router bias +%g on memory 0" % w.router_bias0 if w.router_bias0 else ""
    types = "bf16 activations / fp32 state" if w.dtype == "bf16" else "float32 throughout"
    return ("MoM layer forward, %s shape: %s, d_model=%d, H=%d, d_k=d_v=%d, M=%d memories top-%d + shared%s, %s"
            % (w.name, toks, w.d_model, w.heads, w.d_head, w.n_mem, w.top_k, bias, types))


def load_peaks():
    """The roofline denominators: MEASURED_PEAKS.json's hbm_gbs, bf16_tflops
    and bf16_tflops_sustained where it has them (numbers, possibly under a
    "peaks" key), the fallback figures for any it lacks; "source" says which."""
    p = dict(FALLBACK_PEAKS)
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    got = []
    if os.path.exists(path):
        try:
            with open(path) as fh:
                m = json.load(fh)
        except (OSError, ValueError):
            m = {}
        if isinstance(m, dict) and isinstance(m.get("peaks"), dict):
            m = m["peaks"]
        for k in FALLBACK_PEAKS:
            v = m.get(k) if isinstance(m, dict) else None
            if isinstance(v, (int, float)) and v > 0:
                p[k] = float(v)
                got.append(k)
    p["source"] = ("measured" if len(got) == len(FALLBACK_PEAKS) else
                   "measured (%s), fallback otherwise" % ", ".join(got) if got else "fallback")
    return p


# ------------------------------------------------------------ algorithmic work
def step_work(w):
    """Algorithmic FLOPs / bytes of each of the six calls for one forward of
    workload w (minimum the method needs; intermediates not re-counted)."""
    N, D, H, d, M, K = w.n_tokens, w.d_model, w.heads, w.d_head, w.n_mem, w.top_k
    e = 2  # bf16
    return {
        "router": {"bound": "hbm", "bytes": N * D * e + M * D * e + N * K * 8},
        "permute": {"bound": "hbm", "bytes": 2 * N * K * 4 + N * K * 8},
        "proj": {"bound": "tensor", "flops": 2 * N * D * (3 * H * d + 2 * H) + 2 * N * K * D * 2 * H * d},
        "gdn": {"bound": "tensor", "flops": 6 * N * (1 + K) * H * d * d},
        "combine": {"bound": "hbm", "bytes": e * N * H * d * (2 + K) + N * K * 8},
    }


def layer_roofline(w, peaks, n_seq=None):
    """(FLOPs, bytes, roofline seconds) of one layer forward: the bytes are
    x, the weights, the output, every final state (one per sequence for the
    shared memory and for each routed memory) and the routing; n_seq is the
    number of sequences (default: the workload's fixed batch)."""
    N, D, H, d, M, K = w.n_tokens, w.d_model, w.heads, w.d_head, w.n_mem, w.top_k
    S = w.batch if n_seq is None else n_seq
    sw = step_work(w)
    flops = sw["proj"]["flops"] + sw["gdn"]["flops"] \
        + 2 * N * D * M + 2 * K * N * H * d
    weights = (M * D + 3 * H * d * D + 2 * H * D + M * 2 * H * d * D) * 2
    bytes_ = N * D * 2 + weights + N * H * d * 2 + (S + M * S) * H * d * d * 4 + N * K * 8
    t = max(flops / (peaks["bf16_tflops"] * 1e12), bytes_ / (peaks["hbm_gbs"] * 1e9))
    return flops, bytes_, t


def block_roofline(w, peaks, n_seq=None):
    """(FLOPs, bytes, roofline seconds) of one forward of the layer inside its
    Gated DeltaNet block: the layer's, plus the output gate's and the output
    projection's products, the short convolutions (W taps per channel of q,
    k, v and the routed k, v) and the gated norm; bytes: x, every weight
    (the block's included), the output y, the final states and the routing."""
    N, D, H, d, M, K, W = w.n_tokens, w.d_model, w.heads, w.d_head, w.n_mem, w.top_k, w.conv_width
    S = w.batch if n_seq is None else n_seq
    Hd = H * d
    lf, _, _ = layer_roofline(w, peaks, n_seq)
    flops = lf + 2 * N * D * Hd + 2 * N * Hd * D + 2 * W * (3 + 2 * K) * N * Hd + 8 * N * Hd
    weights = (M * D + 4 * Hd * D + 2 * H * D + M * 2 * Hd * D + D * Hd) * 2 + ((3 + 2 * M) * Hd * W + d) * 4
    bytes_ = N * D * 2 + weights + N * D * 2 + (S + M * S) * H * d * d * 4 + N * K * 8
    t = max(flops / (peaks["bf16_tflops"] * 1e12), bytes_ / (peaks["hbm_gbs"] * 1e9))
    return flops, bytes_, t


def backward_roofline(fwd_flops, peaks, ms):
    """The usual estimate of a backward's algorithmic work, twice its
    forward's FLOPs (an input and a weight gradient per product, the
    recurrence's reverse pass about twice its forward), against the bf16
    peak: {"flops", "roofline_ms", "frac"}."""
    flops = 2 * fwd_flops
    t_ms = flops / (peaks["bf16_tflops"] * 1e12) * 1e3
    return {"flops": flops, "roofline_ms": t_ms, "frac": t_ms / ms, "estimate": "2 x the forward's FLOPs"}


def block_bench(dev, steps, warmup, peaks, flush, name="mom380m_block"):
    """The 380M-shape layer inside its Gated DeltaNet block (short
    convolutions, gated norm, output projection), timed like the headline
    forward."""
    import torch
    from mixture_memories_layer_b200 import block as BL
    from mixture_memories_layer_b200 import synth
    w = synth.WORKLOADS[name]
    p = synth.make_problem(w)
    blk = BL.MoMBlock(BL.pack_block_weights(p, torch.bfloat16, dev), w.heads, w.d_head, w.top_k)
    x = torch.as_tensor(p["x"]).to(dev, torch.bfloat16)
    cu = torch.as_tensor(p["cu_seqlens"]).to(dev)
    for _ in range(warmup):
        blk.forward(x, cu)
    torch.cuda.synchronize()
    errs = blk.device_errors()
    if errs:
        raise SystemExit("device error records in %s: %s" % (name, errs))
    step_ms, per_call = time_forward(blk, x, cu, steps, flush)
    ms = sum(step_ms) / steps
    S = int(cu.numel()) - 1
    bf, bb, bt = block_roofline(w, peaks, n_seq=S)
    res = {"workload": workload_desc(w) + "; inside its Gated DeltaNet block (short convolutions of width %d, "
                                         "gated RMS norm, output projection)" % w.conv_width,
           "tokens": w.n_tokens, "sequences": S, "ms_per_step": ms, "value": w.n_tokens / (ms / 1e3), "unit": UNIT,
           "per_call_ms": per_call,
           "block_roofline": {"flops": bf, "bytes": bb, "roofline_ms": bt * 1e3, "frac": bt * 1e3 / ms}}
    return res, (blk, w, x, cu)


def block_backward_bench(blk, w, x, cu, flush, peaks, steps=3):
    """MoMBlock.backward after a forward on the same tokens (dy ~ N(0,1)):
    the output projection's and the gated norm's adjoints, the layer's
    reverse pass, the convolutions' adjoints and every weight's and the
    tokens' gradients."""
    import torch
    g = torch.Generator(device=x.device).manual_seed(3)
    dy = torch.randn((w.n_tokens, w.d_model), device=x.device, generator=g).to(x.dtype)
    blk.forward(x, cu)
    blk.backward(x, cu, dy)
    torch.cuda.synchronize()
    ms = []
    for _ in range(steps):
        blk.forward(x, cu)
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        blk.backward(x, cu, dy)
        e1.record()
        torch.cuda.synchronize()
        ms.append(e0.elapsed_time(e1))
    errs = blk.device_errors()
    if errs:
        raise SystemExit("device error records in the block backward: %s" % errs)
    t = sum(ms) / steps
    return {"workload": "backward of the %s block (all weight and token gradients), dy ~ N(0,1)" % w.name,
            "path": "output projection's adjoint on the tcgen05 tensor cores; gated norm and convolution adjoints "
                    "HBM-streamed; the layer's reverse pass as in layer_backward",
            "ms": t, "value": w.n_tokens / (t / 1e3), "unit": UNIT,
            "roofline": backward_roofline(block_roofline(w, peaks, int(cu.numel()) - 1)[0], peaks, t)}


def kernel_source_sha(name):
    path = os.path.join(ROOT, "mixture_memories_layer_b200", "csrc", name)
    if not os.path.exists(path):
        return None
    return hashlib.sha256(open(path, "rb").read()).hexdigest()[:16]


def measured_traffic(call):
    """(DRAM bytes per launch from a committed ncu capture, status): the
    bytes only while the kernel's source is unchanged since the capture was
    taken; status is "current", "stale" (a warning is printed) or "none"."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None, "none"
    with open(path) as fh:
        t = json.load(fh).get(call)
    if not t:
        return None, "none"
    if kernel_source_sha(t["source"]) != t.get("source_sha"):
        print("warning: profiles/traffic.json predates the current %s; roofline.traffic is null until it is "
              "re-captured" % t["source"], file=sys.stderr)
        return None, "stale"
    return t["bytes_per_launch"], "current"


# -------------------------------------------------------------------- clocks
class ClockSampler:
    """Polls NVML (read-only) every 10 ms in a thread while the timed region
    runs: SM clock, its maximum, and the active clock-event reasons."""
    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4}

    def __init__(self, torch_device, period=0.01):
        self.dev, self.period = torch_device, period
        self.samples = []
        self._stop = None
        self.error = None

    def _handle(self):
        import pynvml
        import torch
        pr = torch.cuda.get_device_properties(self.dev)
        try:   # NVML numbers GPUs differently from CUDA under CUDA_VISIBLE_DEVICES
            bus = "%08X:%02X:%02X.0" % (pr.pci_domain_id, pr.pci_bus_id, pr.pci_device_id)
            return pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return pynvml.nvmlDeviceGetHandleByIndex(self.dev.index or 0)

    def _run(self):
        import pynvml
        while not self._stop.is_set():
            try:
                sm = pynvml.nvmlDeviceGetClockInfo(self.h, pynvml.NVML_CLOCK_SM)
                rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((sm, rs))
            except Exception as e:          # keep the first failure for the report
                self.error = self.error or repr(e)
            self._stop.wait(self.period)

    def __enter__(self):
        import threading
        try:
            import pynvml
            pynvml.nvmlInit()
            self.h = self._handle()
            self.sm_max = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:
            self.sm_max, self.error = None, repr(e)
            return self
        self._stop = threading.Event()
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()
        return self

    def __exit__(self, *exc):
        if self._stop is not None:
            self._stop.set()
            self._t.join(timeout=2)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.sm_max, "reasons": ["unsampled"], "samples": 0,
                    "error": self.error}
        sm = [s for s, _ in self.samples]
        reasons = sorted({n for _, r in self.samples for n, bit in self.REASONS.items() if r & bit})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": self.sm_max, "reasons": reasons,
                "samples": len(sm)}


# ------------------------------------------------------------ ranks (N > 1)
class Ranks:
    """One process per GPU (torchrun's RANK / WORLD_SIZE / LOCAL_RANK).  The
    layer shards by sequence: every rank runs its own batch and nothing on
    the data path crosses ranks; the only collectives are a barrier around
    the timed region and the max over ranks of its duration.  `backend` is
    "nccl" for the bench and "gloo" for the CPU tests of this plumbing."""

    def __init__(self, backend="nccl", device=None, timeout_s=120):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.device = device
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            kw = {"device_id": device} if backend == "nccl" else {}
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)

    def barrier(self):
        if self.world > 1:
            import torch.distributed as dist
            dist.barrier()

    def max(self, v):
        if self.world == 1:
            return v
        import torch
        import torch.distributed as dist
        t = torch.tensor([v], dtype=torch.float64, device=self.device if self.device is not None else "cpu")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


def rank_problem(w, rank):
    """This rank's share of the job: the replicated weights and its own batch
    of sequences (rank 0: the workload's own tokens; rank r: tokens drawn
    from the seed w.seed * 1000 + r), so that per-GPU work is fixed as N
    grows."""
    from mixture_memories_layer_b200 import synth
    p = synth.make_problem(w)
    if rank:
        p["x"] = synth.make_tokens(w, np.random.default_rng(w.seed * 1000 + rank), w.n_tokens)
    return p


def aggregate_throughput(tokens_per_rank, world, steps, max_total_ms):
    """Whole-job tokens/s: every rank's tokens over the slowest rank's time."""
    return tokens_per_rank * world * steps / (max_total_ms / 1e3)


# ------------------------------------------------------------- the GPU arm
def time_forward(lay, x, cu, steps, flush):
    """`steps` layer forwards, L2 flushed before each outside its events.
    Returns (per-step ms list, mean ms per call of MoMLayer.STEPS)."""
    import torch
    names = type(lay).STEPS
    n_calls = len(names)
    marks = [[torch.cuda.Event(enable_timing=True) for _ in range(n_calls + 1)] for _ in range(steps)]
    torch.cuda.synchronize()
    for s in range(steps):
        flush.zero_()                          # evict L2 (outside the step's events)
        lay.forward(x, cu, marks=marks[s])
    torch.cuda.synchronize()
    step_ms = [marks[s][0].elapsed_time(marks[s][n_calls]) for s in range(steps)]
    per_call = {name: sum(marks[s][i].elapsed_time(marks[s][i + 1]) for s in range(steps)) / steps
                for i, name in enumerate(names)}
    return step_ms, per_call


def near_tie_tokens(x, w_r, b_r, top_k, gap=TIE_GAP):
    """Tokens whose k-th and (k+1)-th router logits (float32, on the device)
    lie within `gap`: rounding may flip their choice, so parity tests leave
    them out of the exact index check.  Reported, not used by the layer."""
    import torch
    if top_k >= w_r.shape[0]:
        return 0
    logits = x.float() @ w_r.float().t() + b_r.float()
    top = torch.topk(logits, top_k + 1, dim=-1).values
    return int(((top[:, top_k - 1] - top[:, top_k]) < gap).sum().item())


def config_bench(name, dev, steps, warmup, peaks, flush, rule="gated_delta", mem_gates=False):
    """One of the other forward workloads, timed like the headline one."""
    import dataclasses

    import torch
    from mixture_memories_layer_b200 import layer as L
    from mixture_memories_layer_b200 import synth
    w = dataclasses.replace(synth.WORKLOADS[name], mem_gates=mem_gates)
    p = synth.make_problem(w)
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    lay = L.MoMLayer(L.pack_weights(p, dt, dev), w.heads, w.d_head, w.top_k, rule=rule)
    x = torch.as_tensor(p["x"]).to(dev, dt)
    cu = torch.as_tensor(p["cu_seqlens"]).to(dev)
    for _ in range(warmup):
        lay.forward(x, cu)
    torch.cuda.synchronize()
    errs = lay.device_errors()
    if errs:
        raise SystemExit("device error records in %s (%s): %s" % (name, rule, errs))
    step_ms, per_call = time_forward(lay, x, cu, steps, flush)
    ms = sum(step_ms) / steps
    S = int(cu.numel()) - 1
    rows = lay.buffers(w.n_tokens, S)["mem_offset"].cpu().tolist()
    out = {"workload": workload_desc(w), "memory_rule": rule, "per_memory_gates": mem_gates, "dtype": w.dtype, "tokens": w.n_tokens, "sequences": S,
           "ms_per_step": ms, "value": w.n_tokens / (ms / 1e3), "unit": UNIT, "per_call_ms": per_call,
           "routed_rows_per_memory": [b - a for a, b in zip(rows[:-1], rows[1:])],
           "near_tie_tokens": near_tie_tokens(x, lay.w["w_r"], lay.w["b_r"], w.top_k)}
    if w.dtype == "bf16":
        lf, lb, lt = layer_roofline(w, peaks, n_seq=S)
        gdn = step_work(w)["gdn"]["flops"] / (per_call["gdn"] / 1e3) / 1e12
        out["layer_roofline"] = {"flops": lf, "bytes": lb, "roofline_ms": lt * 1e3, "frac": lt * 1e3 / ms}
        out["gdn_tflops"] = gdn
        out["gdn_frac"] = gdn / peaks["bf16_tflops"]
    else:
        out["layer_roofline"] = {"bound": "latency", "note": "float32 CUDA-core path; latency only"}
    return out


def gpu_arm(args):
    import torch

    from mixture_memories_layer_b200 import binding as B
    from mixture_memories_layer_b200 import layer as L
    from mixture_memories_layer_b200 import synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit("--gpus %d but WORLD_SIZE=%d (launch N>1 with torchrun)" % (args.gpus, world))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    ranks = Ranks("nccl", dev)
    rank = ranks.rank
    barrier, max_over_ranks = ranks.barrier, ranks.max

    peaks = load_peaks()
    w = synth.WORKLOADS[FWD]
    p = rank_problem(w, rank)
    dt = torch.bfloat16
    lay = L.MoMLayer(L.pack_weights(p, dt, dev), w.heads, w.d_head, w.top_k)
    x = torch.as_tensor(p["x"]).to(dev, dt)
    cu = torch.as_tensor(p["cu_seqlens"]).to(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    clocks = ClockSampler(dev).__enter__()     # sampled from warm-up to the end of decode
    for _ in range(args.warmup):
        lay.forward(x, cu)
    torch.cuda.synchronize()
    errs = lay.device_errors()
    if errs:
        raise SystemExit("device error records after warm-up: %s" % errs)

    launches0 = B.mom_launch_count()
    barrier()
    step_ms, per_call = time_forward(lay, x, cu, args.steps, flush)
    barrier()
    launches = B.mom_launch_count() - launches0
    total_ms = max_over_ranks(sum(step_ms))
    ms_per_step = total_ms / args.steps
    value = aggregate_throughput(w.n_tokens, world, args.steps, total_ms)

    # ---- roofline of the dominant call
    work = step_work(w)
    top = max(per_call, key=per_call.get)
    wk = work[top]
    sec = per_call[top] / 1e3
    if wk["bound"] == "tensor":
        achieved = wk["flops"] / sec / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": achieved / peaks["bf16_tflops"]}
    else:
        achieved = wk["bytes"] / sec / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"]}
    traffic, traffic_status = measured_traffic(top)
    roof.update({"kernel": top, "traffic": traffic, "traffic_record": traffic_status,
                 "peak_source": peaks["source"], "ms_per_launch": per_call[top]})
    lf, lb, lt = layer_roofline(w, peaks)
    layer_roof = {"flops": lf, "bytes": lb, "roofline_ms": lt * 1e3, "frac": (lt * 1e3) / ms_per_step}

    # ---- end to end through the C ABI with host buffers
    e2e = None
    if not args.no_e2e:
        e2e = e2e_bench(args, w, lay, x, cu, flush, stream, dt, world, max_over_ranks)
    decode = None if args.no_decode else decode_bench(args, dev, world, rank, max_over_ranks, barrier)
    configs = None
    if not args.no_configs and world == 1:
        want = None if args.configs is None else set(args.configs.split(","))
        on = lambda key: want is None or key in want
        configs = {extra_key(name, rule, mg): config_bench(name, dev, args.steps, args.warmup, peaks, flush, rule, mg)
                   for name, rule, mg in EXTRA if on(extra_key(name, rule, mg))}
        if on("block") or on("block_backward"):
            res, blk_run = block_bench(dev, args.steps, args.warmup, peaks, flush)
            if on("block"):
                configs["block"] = res
            if on("block_backward"):
                configs["block_backward"] = block_backward_bench(*blk_run, flush, peaks)
            del blk_run
        if on("block_decode"):
            configs["block_decode"] = block_decode_bench(dev, args.warmup)
        if on("recurrence_backward"):
            configs["recurrence_backward"] = backward_bench(lay, w, x, cu, flush)
        if on("layer_backward"):
            configs["layer_backward"] = layer_backward_bench(lay, w, x, cu, flush, peaks)
    clocks.__exit__(None, None, None)
    layer_roof["near_tie_tokens"] = near_tie_tokens(x, lay.w["w_r"], lay.w["b_r"], w.top_k)
    return finish(args, w, world, rank, value, ms_per_step, roof, layer_roof, per_call, e2e, launches, clocks, decode,
                  configs)


SETS = 2          # e2e buffer sets
E2E_STEPS = 64    # e2e steps at least


def e2e_bench(args, w, lay, x, cu, flush, stream, dt, world, max_over_ranks):
    """The same metric through the user-facing calls with host buffers:
    every step uploads its tokens from pinned host memory, runs the layer
    and reads its output back to pinned host memory.  Steps are pipelined
    the way a serving loop streams batches: SETS buffer sets (layer objects
    over the same weights), the upload of a later step and the download of
    an earlier one on their own streams beside a step's compute, so that the
    PCIe link (both directions at once) is the bound.  At least E2E_STEPS
    steps, so the pipeline's fill and drain (one upload, one download) are
    a small part of the timed region.  No L2 flush: a step touches ~0.6 GB,
    several times L2."""
    import torch
    from mixture_memories_layer_b200 import layer as L
    n = max(E2E_STEPS, args.steps)
    lays = [lay] + [L.MoMLayer(lay.w, w.heads, w.d_head, w.top_k) for _ in range(SETS - 1)]
    xs = [x] + [torch.empty_like(x) for _ in range(SETS - 1)]
    x_host = torch.empty(x.shape, dtype=dt, pin_memory=True)
    x_host.copy_(x.cpu())
    outs_host = [torch.empty((w.n_tokens, w.heads, w.d_head), dtype=dt, pin_memory=True) for _ in range(SETS)]
    for j in range(1, SETS):
        lays[j].forward(xs[0], cu)             # the other buffer sets, warm
    torch.cuda.synchronize()
    h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(n)]
    ev_fwd = [torch.cuda.Event() for _ in range(n)]
    ev_out = [torch.cuda.Event() for _ in range(n)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(h2d)
    for i in range(n):
        j = i % SETS
        if i >= SETS:
            h2d.wait_event(ev_fwd[i - SETS])   # the forward SETS steps back has read xs[j]
        with torch.cuda.stream(h2d):
            xs[j].copy_(x_host, non_blocking=True)
        ev_in[i].record(h2d)
        stream.wait_event(ev_in[i])
        if i >= SETS:
            stream.wait_event(ev_out[i - SETS])   # that step's output has left lays[j]'s buffer
        b = lays[j].forward(xs[j], cu, stream=stream)
        ev_fwd[i].record(stream)
        d2h.wait_event(ev_fwd[i])
        with torch.cuda.stream(d2h):
            outs_host[j].copy_(b["out"], non_blocking=True)
        ev_out[i].record(d2h)
    d2h.wait_stream(h2d)
    e1.record(d2h)
    e1.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1))
    return {"value": w.n_tokens * world * n / (e2e_ms / 1e3), "unit": UNIT,
            "h2d_bytes_per_step": x.numel() * x.element_size(),
            "d2h_bytes_per_step": outs_host[0].numel() * outs_host[0].element_size(),
            "steps": n, "pipelined": "uploads of later steps and downloads of earlier ones beside each step's compute "
                                      "(%d buffer sets, three streams); no L2 flush (each step touches ~0.6 GB)" % SETS}


def finish(args, w, world, rank, value, ms_per_step, roof, layer_roof, per_call, e2e, launches, clocks, decode,
           configs=None):
    import torch.distributed as dist
    result = None
    if rank == 0:
        cpu = cpu_baseline(w) if (world == 1 and not args.no_cpu_baseline) else None
        result = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic: seeded X~N(0,1), weights~N(0,1/d_model), A~U(0,2.7), b_a~U(-4,0)",
            "config": {"workload": workload_desc(w), "tokens_per_gpu": w.n_tokens, "global_tokens": w.n_tokens * world,
                       "seq_len": w.seq_len, "parallelism": "dp%d (sequences sharded, no collective)" % world,
                       "l2": "flushed before every timed step (256 MiB write, untimed)"},
            "roofline": roof, "layer_roofline": layer_roof,
            "per_call_ms": per_call, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": launches, "clocks": clocks.summary(), "decode": decode, "configs": configs,
        }
        print(json.dumps(result), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return result


def backward_bench(lay, w, x, cu, flush, steps=3):
    """The reverse pass of the layer's two recurrence problems (the shared
    memory over every token, the routed memories over their segments) on the
    layer's own q, k, v and gates, with a random output gradient: the first
    GPU path of the backward (token-serial float32 on CUDA cores)."""
    import torch
    from mixture_memories_layer_b200 import binding as B
    S = cu.numel() - 1
    b = lay.forward(x, cu)
    H, d = w.heads, w.d_head
    probs = {"shared": (b["q"], None, b["k_sh"], b["v_sh"], cu), "routed": (b["q"], b["perm"], b["k_p"], b["v_p"],
                                                                          b["seg_cu"])}
    out = {"workload": "reverse pass of the %s layer's recurrences (shared + routed), dout ~ N(0,1)" % w.name,
           "path": "token-serial float32 on CUDA cores (32 state rows per CTA, two CTAs per SM), states kept every 16 "
                   "tokens, chunks re-walked keeping a copy every 2"}
    total = 0.0
    g = torch.Generator(device=x.device).manual_seed(1)
    for name, (q, qidx, k, v, seg) in probs.items():
        n = k.shape[0]
        do = torch.randn((n, H, d), device=x.device, generator=g).to(x.dtype)
        bufs = [torch.empty((n, H, d), device=x.device) for _ in range(3)] + \
               [torch.empty((n, H), device=x.device) for _ in range(2)]
        dh0 = torch.empty((seg.numel() - 1, H, d, d), device=x.device)
        ws = B.new_workspace(B.mom_memory_chunk_bwd_workspace_size(n, seg.numel() - 1, H, d), x.device)
        call = lambda: B.mom_memory_chunk_bwd(q, qidx, k, v, b["beta"], b["log_alpha"], seg, lay.scale, lay.rule,
                                              None, do, None, *bufs, dh0, ws)
        call()
        torch.cuda.synchronize()
        ms = []
        for _ in range(steps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            call()
            e1.record()
            torch.cuda.synchronize()
            ms.append(e0.elapsed_time(e1))
        code, _ = B.mom_get_error(ws)
        if code:
            raise SystemExit("device error record in the recurrence reverse pass (%s): %d" % (name, code))
        out[name + "_ms"] = sum(ms) / steps
        total += out[name + "_ms"]
        del ws, bufs, dh0
    out["ms"] = total
    out["value"] = w.n_tokens / (total / 1e3)
    out["unit"] = UNIT
    return out


def layer_backward_bench(lay, w, x, cu, flush, peaks, steps=3):
    """MoMLayer.backward after a forward on the same tokens (dout ~ N(0,1)):
    every weight's and the tokens' gradients.  First path: the recurrences'
    reverse passes token-serial and the gradient GEMMs on CUDA cores, float32."""
    import torch
    g = torch.Generator(device=x.device).manual_seed(2)
    dout = torch.randn((w.n_tokens, w.heads, w.d_head), device=x.device, generator=g).to(x.dtype)
    lay.forward(x, cu)
    lay.backward(x, cu, dout)
    torch.cuda.synchronize()
    ms = []
    for _ in range(steps):
        lay.forward(x, cu)
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        lay.backward(x, cu, dout)
        e1.record()
        torch.cuda.synchronize()
        ms.append(e0.elapsed_time(e1))
    errs = lay.device_errors()
    if errs:
        raise SystemExit("device error records in the layer backward: %s" % errs)
    t = sum(ms) / steps
    return {"workload": "backward of the %s layer (all weight and token gradients), dout ~ N(0,1)" % w.name,
            "path": "recurrence reverse passes token-serial float32; gradient GEMMs on the tf32 tensor cores "
                    "(fp32 accumulation)",
            "ms": t, "value": w.n_tokens / (t / 1e3), "unit": UNIT,
            "roofline": backward_roofline(layer_roofline(w, peaks, int(cu.numel()) - 1)[0], peaks, t)}


def decode_bench(args, dev, world, rank, max_over_ranks, barrier):
    import torch

    from mixture_memories_layer_b200 import layer as L
    from mixture_memories_layer_b200 import synth

    w = synth.WORKLOADS[DEC]
    steps = w.decode_steps
    p = synth.make_decode_problem(w, steps=steps + args.warmup)
    dt = torch.bfloat16
    lay = L.MoMLayer(L.pack_weights(p, dt, dev), w.heads, w.d_head, w.top_k)
    b = lay.forward(torch.as_tensor(p["x_prefill"]).to(dev, dt), torch.as_tensor(p["cu_prefill"]).to(dev))
    state0 = torch.empty((w.batch, w.n_mem + 1, w.heads, w.d_head, w.d_head), dtype=torch.float32, device=dev)
    state0[:, :w.n_mem] = b["h_mem"].permute(1, 0, 2, 3, 4)
    state0[:, w.n_mem] = b["h_shared"]
    xs = torch.as_tensor(p["x_steps"]).to(dev, dt)
    state = state0.clone()
    for s in range(args.warmup):
        lay.decode_step(xs[steps + s], state)
    state.copy_(state0)
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for s in range(steps):
        lay.decode_step(xs[s], state)
    e1.record()
    torch.cuda.synchronize()
    barrier()
    ms = max_over_ranks(e0.elapsed_time(e1))
    state_bytes = (w.top_k + 1) * w.batch * w.heads * w.d_head * w.d_head * 4 * 2
    per_step = ms / steps
    hbm = load_peaks()["hbm_gbs"]
    return {"workload": "decode: B=%d sequences, d_model=%d, H=%d, d=%d, M=%d top-%d + shared, %d steps after a "
                        "%d-token prefill" % (w.batch, w.d_model, w.heads, w.d_head, w.n_mem, w.top_k, steps,
                                              w.prefill_len),
            "value": w.batch * world * steps / (ms / 1e3), "unit": "tokens/s", "ms_per_step": per_step,
            "state_bytes_per_step": state_bytes,
            "state_gbs": state_bytes / (per_step / 1e3) / 1e9,
            "frac_hbm": state_bytes / (per_step / 1e3) / 1e9 / hbm}


def block_decode_bench(dev, warmup, steps=128):
    """Decode through the Gated DeltaNet block: the decode workload's shape
    (256 sequences, 8 memories top-2 + shared) with the block, after a
    prefill through MoMBlock.forward and the windows it leaves."""
    import dataclasses

    import torch
    from mixture_memories_layer_b200 import block as BL
    from mixture_memories_layer_b200 import synth
    w = dataclasses.replace(synth.WORKLOADS[DEC], block=True)
    p = synth.make_decode_problem(w, steps=steps + warmup)
    blk = BL.MoMBlock(BL.pack_block_weights(p, torch.bfloat16, dev), w.heads, w.d_head, w.top_k)
    cu = torch.as_tensor(p["cu_prefill"]).to(dev)
    b = blk.forward(torch.as_tensor(p["x_prefill"]).to(dev, torch.bfloat16), cu)
    conv0 = blk.conv_state(b, cu)
    state0 = torch.empty((w.batch, w.n_mem + 1, w.heads, w.d_head, w.d_head), dtype=torch.float32, device=dev)
    state0[:, :w.n_mem] = b["h_mem"].permute(1, 0, 2, 3, 4)
    state0[:, w.n_mem] = b["h_shared"]
    xs = torch.as_tensor(p["x_steps"]).to(dev, torch.bfloat16)
    state, conv_sh, conv_mem = state0.clone(), conv0[0].clone(), conv0[1].clone()
    for s in range(warmup):
        blk.decode_step(xs[steps + s], state, conv_sh, conv_mem)
    state.copy_(state0)
    conv_sh.copy_(conv0[0])
    conv_mem.copy_(conv0[1])
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for s in range(steps):
        blk.decode_step(xs[s], state, conv_sh, conv_mem)
    e1.record()
    torch.cuda.synchronize()
    errs = blk.device_errors()
    if errs:
        raise SystemExit("device error records in the block decode: %s" % errs)
    ms = e0.elapsed_time(e1)
    return {"workload": "decode through the Gated DeltaNet block: B=%d sequences, d_model=%d, H=%d, d=%d, M=%d top-%d "
                        "+ shared, %d steps after a %d-token prefill" % (w.batch, w.d_model, w.heads, w.d_head,
                                                                         w.n_mem, w.top_k, steps, w.prefill_len),
            "value": w.batch * steps / (ms / 1e3), "unit": "tokens/s", "ms_per_step": ms / steps}


# --------------------------------------------------------- CPU oracle timing
# The oracle is plain single-threaded numpy per sequence; the sequences of a
# batch are independent, so the timed CPU legs run one sequence (or one
# window of it) per host process, each process with one BLAS thread.  The
# pool is started with "spawn" (never forked from a process that has used
# the GPU).
_ORACLE = {}


def _oracle_init(name):
    from threadpoolctl import threadpool_limits
    from mixture_memories_layer_b200 import synth
    _ORACLE["limit"] = threadpool_limits(1)
    w = synth.WORKLOADS[name]
    _ORACLE["w"], _ORACLE["p"] = w, synth.make_problem(w)


def _oracle_window(job):
    """Oracle layer forward on tokens [t0, t0 + n) of sequence s (states
    from zero); returns (tokens, seconds)."""
    from oracle import mom_oracle as orc
    s, t0, n = job
    w, p = _ORACLE["w"], _ORACLE["p"]
    a = int(p["cu_seqlens"][s]) + t0
    n = min(n, int(p["cu_seqlens"][s + 1]) - a)
    t = time.perf_counter()
    orc.mom_forward(p["x"][a:a + n], p, np.array([0, n]), w.top_k, w.heads, w.d_head)
    return n, time.perf_counter() - t


def _oracle_pool(name, procs):
    import multiprocessing as mp
    pool = mp.get_context("spawn").Pool(procs, initializer=_oracle_init, initargs=(name,))
    pool.map(_oracle_window, [(0, 0, 1)] * procs)      # every worker started and warm
    return pool


def _oracle_procs(w):
    return max(1, min(w.batch, os.cpu_count() or 1))


def cpu_baseline(w):
    """Whole sequences of the workload through the oracle, one per host
    process: tokens of all of them over the slowest one's time."""
    procs = _oracle_procs(w)
    pool = _oracle_pool(w.name, procs)
    try:
        res = pool.map(_oracle_window, [(s, 0, w.seq_len) for s in range(procs)], chunksize=1)
    finally:
        pool.close()
        pool.join()
    toks, sec = sum(n for n, _ in res), max(t for _, t in res)
    return {"value": toks / sec, "unit": UNIT, "cores": procs, "kind": "oracle",
            "sample": "%d whole %d-token sequences of the same workload, one per host process (one BLAS thread "
                      "each), fp64 numpy; tokens over the slowest process's %.1f s" % (procs, w.seq_len, sec)}


def memory_parallel_arm(args):
    """--parallel memory: the routed memories sharded over the ranks (each
    rank owns a block of memories and its own batch of sequences; routed rows
    go to their owners and back with NCCL all-to-alls).  The same timing
    rules as the data-parallel arm: warm-up, barriers, L2 flushed outside the
    events, max over ranks; the exchange's host reads of split sizes are
    inside the timed region."""
    import datetime

    import torch
    import torch.distributed as dist

    from mixture_memories_layer_b200 import binding as B
    from mixture_memories_layer_b200 import layer as L
    from mixture_memories_layer_b200 import synth
    from mixture_memories_layer_b200.mem_parallel import MemoryParallelMoM, Partition, TorchComm

    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit("--gpus %d but WORLD_SIZE=%d (launch N>1 with torchrun)" % (args.gpus, world))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world == 1:
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        os.environ.setdefault("MASTER_PORT", "29541")
        os.environ.setdefault("RANK", "0")
    dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev,
                            rank=int(os.environ.get("RANK", "0")), world_size=world)
    try:
        rank = dist.get_rank()
        w = synth.WORKLOADS[args.workload]
        p = rank_problem(w, rank)
        dt = torch.bfloat16
        full = L.pack_weights(p, dt, dev)
        part = Partition(w.n_mem, world)
        weights = {k: v for k, v in full.items() if k != "w_kv"}
        weights["w_kv"] = full["w_kv"][part.lo(rank):part.hi(rank)].contiguous()
        del full
        meta = dist.new_group(backend="gloo")
        layer = MemoryParallelMoM(weights, w.heads, w.d_head, w.top_k, w.n_mem, TorchComm(meta_group=meta))
        x = torch.as_tensor(p["x"]).to(dev, dt)
        cu = torch.as_tensor(p["cu_seqlens"]).to(dev)
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        for _ in range(args.warmup):
            layer.forward(x, cu)
        torch.cuda.synchronize()
        launches0 = B.mom_launch_count()
        dist.barrier()
        ms = []
        for _ in range(args.steps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            layer.forward(x, cu)
            b.record()
            torch.cuda.synchronize()
            ms.append(a.elapsed_time(b))
        dist.barrier()
        launches = B.mom_launch_count() - launches0
        t = torch.tensor([sum(ms)], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        total_ms = float(t.item())
        if rank == 0:
            value = aggregate_throughput(w.n_tokens, world, args.steps, total_ms)
            lf, lb, lt = layer_roofline(w, load_peaks())
            out = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
                   "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
                   "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                   "data": "synthetic: seeded, same generator as the data-parallel arm",
                   "config": {"workload": workload_desc(w), "tokens_per_gpu": w.n_tokens,
                              "global_tokens": w.n_tokens * world,
                              "parallelism": ("mp%d (memories sharded, routed rows to their owners and back by "
                                              "NCCL all-to-all)" % world) if world > 1 else
                                             "mp1 (every memory on the one rank: the row exchanges are the "
                                             "identity; the metadata still goes through the process group)",
                              "l2": "flushed before every timed step (256 MiB write, untimed)"},
                   "layer_roofline": {"flops": lf, "bytes": lb, "roofline_ms": lt * 1e3,
                                      "frac": lt * 1e3 / (total_ms / args.steps)},
                   "gpu_launches": launches}
            print(json.dumps(out), flush=True)
    finally:
        dist.destroy_process_group()


def reference_arm(args):
    if int(os.environ.get("RANK", "0")) != 0:
        return None
    from mixture_memories_layer_b200 import synth
    w = synth.WORKLOADS[FWD]
    T = 128                       # tokens per sequence per step: one bounded window
    n_win = w.seq_len // T
    procs = _oracle_procs(w)
    pool = _oracle_pool(w.name, procs)

    def step(i):
        return pool.map(_oracle_window, [(s, (i % n_win) * T, T) for s in range(procs)], chunksize=1)

    try:
        for i in range(args.warmup):
            step(i)
        t0 = time.perf_counter()
        for i in range(args.steps):
            step(args.warmup + i)
        sec = time.perf_counter() - t0
    finally:
        pool.close()
        pool.join()
    value = procs * T * args.steps / sec
    sample = ("each step: the oracle layer forward on a %d-token window (state from zero) of each of %d "
              "sequences of the same workload, one sequence per host process (one BLAS thread each)" % (T, procs))
    out = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3 / max(args.steps, 1),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic: seeded, same generator as the GPU arm",
           "config": {"workload": workload_desc(w), "tokens_per_step": procs * T},
           "cpu_baseline": {"value": value, "unit": UNIT, "cores": procs, "kind": "oracle", "sample": sample},
           "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end timing")
    ap.add_argument("--no-decode", action="store_true", help="skip the decode timing")
    ap.add_argument("--no-configs", action="store_true", help="skip the other forward workloads")
    ap.add_argument("--configs", default=None,
                    help="comma-separated subset of the other workloads to run (names as in the JSON line's "
                         "configs; default: all)")
    ap.add_argument("--parallel", default="data", choices=["data", "memory"],
                    help="data: every rank runs the whole layer on its own sequences; memory: the routed "
                         "memories are sharded over the ranks")
    ap.add_argument("--workload", default=None, help="forward workload of --parallel memory (default: the "
                    "16-memory 1.3B shape)")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        reference_arm(args)
    elif args.parallel == "memory":
        args.workload = args.workload or "mom1p3b_m16"
        memory_parallel_arm(args)
    else:
        gpu_arm(args)


if __name__ == "__main__":
    main()
