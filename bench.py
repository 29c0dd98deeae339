"""Gated-prefill benchmark: one step = gate score + top-K + compaction + gated
attention for one synthetic prompt batch, through libtokengate's C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload qwen_16k]
    python bench.py --impl reference ...      # the CPU oracle, timed on host cores

Prints one JSON line (rank 0).  Multi-GPU runs (torchrun, one process per GPU)
are weak-scaling replicas: every rank processes its own prompt batch (its own
seed), no data moves between GPUs, and the reported time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

DEFAULT_WORKLOAD = "qwen_16k"
L2_FLUSH_BYTES = 256 << 20
METRIC = "gated-prefill input tok/s"
# the libtokengate kernel each stage launches on the tensor-core path (the attention
# kernel depends on the batch: tg.attention_kernel names it)
KERNELS = {"gate": "gate_tc2_kernel", "topk": "topk_kernel", "gather": "gather_bulk_kernel"}
KERNELS_FP32 = {**KERNELS, "gate": "gate_simt_kernel"}  # fp32 gates run on the CUDA cores
HOLD_CYCLES = 40_000_000  # ~20 ms of device time before each timed batch is queued
FP32_FMA_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12  # nominal FP32 FMA peak (CUDA-core fp32 path)


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return dict(hbm=float(d["hbm_gbs"]), bf16=float(d["bf16_tflops"]),
                    bf16_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


class ClockSampler:
    """Polls SM clock and throttle reasons through NVML while the timed region runs."""

    REASONS = {0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, device_index, period_s=0.002):
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._period = period_s
        try:
            import pynvml

            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:  # noqa: BLE001 - clocks are reported as unavailable
            self._nv = None
        self._t = threading.Thread(target=self._loop, daemon=True)

    def _loop(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                bits = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for b, name in self.REASONS.items():
                    if bits & b:
                        self.reasons.add(name)
            except Exception:  # noqa: BLE001
                pass
            time.sleep(self._period)

    def __enter__(self):
        if self._nv is not None:
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._nv is not None:
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0}
        return {"sm_mhz": float(np.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def _dist_init(n_gpus):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world > 1:
        if world != n_gpus:
            raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE={world}")
        local = int(os.environ.get("LOCAL_RANK", "0"))
        torch.cuda.set_device(local)
        import datetime

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
        return dist.get_rank(), world, local
    return 0, 1, 0


def _traffic(kernel, workload):
    """DRAM bytes per launch from a committed ncu capture, or None once the kernel's
    source has changed since the capture."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    rec = json.load(open(path)).get(kernel, {}).get(workload)
    if not rec:
        return None
    src = os.path.join(ROOT, "learned_token_pruning_gate_b200", "csrc", rec["source"])
    if not os.path.exists(src) or _sha(src) != rec["sha256"]:
        return None
    return rec["bytes_per_launch"]


def _sha(path):
    return hashlib.sha256(open(path, "rb").read()).hexdigest()[:16]


DTYPES = {"bf16": "bf16", "fp32": "f32"}
# every other configuration measured in the same process after the headline one:
# (name, the workload whose inputs it reuses); the 32k budget sweep shares its inputs
OTHER_WORKLOADS = [("tiny_fp32", "tiny_fp32"), ("qwen_32k_k1024", "qwen_32k_k1024"),
                   ("qwen_32k_k4096", "qwen_32k_k1024"), ("qwen_32k_k8192", "qwen_32k_k1024"),
                   ("qwen_128k", "qwen_128k"), ("ragged_4", "ragged_4")]


def _make_layer(tg, inp, w, dev):
    from learned_token_pruning_gate_b200.pipeline import GatedLayer

    d = lambda t: t.to(dev).contiguous()  # noqa: E731
    return GatedLayer(d(inp.h), d(inp.q), d(inp.k), d(inp.v), d(inp.W1), d(inp.b1), d(inp.w2),
                      inp.b2, d(inp.gain), d(inp.temp), inp.cu_seqlens, inp.doc_begin,
                      inp.doc_end, np.asarray(w.budgets, np.int32), rope_theta=w.rope_theta,
                      algo=tg.ALGO_AUTO)


def _time_steps(graph, flush, stream, K, warmup, settle_s=0.3):
    """K CUDA-graph replays, each bracketed by CUDA events on the launching stream,
    with an L2 flush between them (outside the events).  Returns per-step ms."""
    import torch

    t_warm = time.time()
    for _ in range(max(warmup, 3)):
        flush.zero_()
        graph.replay()
    while time.time() - t_warm < settle_s:  # let the clocks settle before timing
        flush.zero_()
        graph.replay()
        torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(K)]
    # hold the stream for a moment so the host queues launches ahead of the GPU:
    # the timed intervals then hold device work only, not host launch latency
    torch.cuda._sleep(HOLD_CYCLES)
    for i in range(K):
        flush.zero_()
        ev[i][0].record(stream)
        graph.replay()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in ev]


def _time_stages(layer, flush, stream, n):
    """Per-kernel times inside the step: the four launches captured in one CUDA
    graph with an event record before and after each (on the launching stream),
    replayed n times with an L2 flush between replays; a stage's time is the
    interval between the events around its launch (mean over the replays).  The
    records sit between the kernels, so the next launch cannot start early under
    them: the sum of the stages is a little above the step time."""
    import ctypes

    import torch

    stages = layer.STAGES
    evs = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(len(stages) + 1)]
    side = torch.cuda.Stream()
    side.wait_stream(stream)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        st = ctypes.c_void_p(side.cuda_stream)
        evs[0].record(side)
        for j, s in enumerate(stages):
            getattr(layer, s)(st)
            evs[j + 1].record(side)
    torch.cuda.synchronize()
    acc = {s: [] for s in stages}
    for i in range(n + 2):  # two untimed replays first
        flush.zero_()
        g.replay()
        torch.cuda.synchronize()
        if i >= 2:
            for j, s in enumerate(stages):
                acc[s].append(evs[j].elapsed_time(evs[j + 1]))
    del g
    return {s: float(np.mean(v)) for s, v in acc.items()}


def _stages_and_roofline(tg, layer, w, name, stage_ms, pk):
    """Per-stage achieved rates and the roofline object of the dominant kernel."""
    work = layer.work()
    kernels = KERNELS if w.dtype == "bf16" else KERNELS_FP32
    us = {s: stage_ms[s] * 1e3 for s in stage_ms}
    stages = {
        "gate": {"us": us["gate"], "tflops": work["gate_flops"] / us["gate"] / 1e6,
                 "gbs": work["gate_bytes"] / us["gate"] / 1e3},
        "topk": {"us": us["topk"], "gbs": work["topk_bytes"] / us["topk"] / 1e3},
        "gather": {"us": us["gather"], "gbs": work["gather_bytes"] / us["gather"] / 1e3},
        "attention": {"us": us["attention"],
                      "tflops": work["attn_flops"] / us["attention"] / 1e6},
    }
    for s in stages.values():
        if "tflops" in s:
            s["frac_tensor"] = s["tflops"] / pk["bf16"]
        if "gbs" in s:
            s["frac_hbm"] = s["gbs"] / pk["hbm"]
    tg_us = us["topk"] + us["gather"]
    stages["topk+gather"] = {"us": tg_us,
                             "gbs": (work["topk_bytes"] + work["gather_bytes"]) / tg_us / 1e3}
    stages["topk+gather"]["frac_hbm"] = stages["topk+gather"]["gbs"] / pk["hbm"]
    dominant = max(("gate", "topk", "gather", "attention"), key=lambda s: us[s])
    attn_kernel = tg.attention_kernel(layer.cu_kept_host, w.n_q_heads, w.n_kv_heads, w.head_dim,
                                      dtype=w.dtype, with_workspace=layer.workspace is not None)
    attn_kernel = attn_kernel.split(" ")[0]
    stages["attention"]["kernel"] = attn_kernel
    if dominant == "attention" and w.dtype == "bf16":
        roof = {"kernel": attn_kernel, "bound": "tensor",
                "achieved": stages["attention"]["tflops"], "peak": pk["bf16"], "unit": "TFLOP/s"}
    elif dominant == "attention":  # fp32 runs on the CUDA cores: FP32 FMA peak
        roof = {"kernel": attn_kernel, "bound": "alu", "achieved": stages["attention"]["tflops"],
                "peak": FP32_FMA_TFLOPS, "unit": "TFLOP/s"}
    elif dominant == "gate":
        t_flop = work["gate_flops"] / (pk["bf16"] * 1e12)
        t_byte = work["gate_bytes"] / (pk["hbm"] * 1e9)
        if t_flop >= t_byte:
            roof = {"kernel": kernels["gate"], "bound": "tensor",
                    "achieved": stages["gate"]["tflops"], "peak": pk["bf16"], "unit": "TFLOP/s"}
        else:
            roof = {"kernel": kernels["gate"], "bound": "hbm", "achieved": stages["gate"]["gbs"],
                    "peak": pk["hbm"], "unit": "GB/s"}
    else:
        roof = {"kernel": kernels[dominant], "bound": "hbm",
                "achieved": stages[dominant]["gbs"], "peak": pk["hbm"], "unit": "GB/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = _traffic(roof["kernel"], name)
    roof["peak_source"] = f"{pk['source']} (burst)" if roof["bound"] != "alu" else \
        "nominal FP32 FMA: 148 SMs x 128 lanes x 2 flop x 1.965 GHz"
    return stages, roof


def _other_workloads(tg, gen, dev, stream, flush, pk, K):
    """Every configuration besides the headline one, timed the same way (graph
    replay, L2 flushed, CUDA events), fewer steps; buffers freed in between."""
    import torch

    res, cache = {}, {}
    for name, src in OTHER_WORKLOADS:
        w = gen.WORKLOADS[name]
        if src not in cache:
            cache.clear()
            cache[src] = gen.make_inputs(gen.WORKLOADS[src])
        inp = cache[src]
        layer = _make_layer(tg, inp, w, dev)
        graph = layer.capture()
        with ClockSampler(dev.index or 0) as clocks:
            step_ms = _time_steps(graph, flush, stream, K, 3, settle_s=0.1)
        stage_ms = _time_stages(layer, flush, stream, min(K, 10))
        if tg.device_status() != 0:
            raise SystemExit(f"{name}: a kernel reported a timed-out wait")
        stages, roof = _stages_and_roofline(tg, layer, w, name, stage_ms, pk)
        ms = float(np.mean(step_ms))
        res[name] = {"ms_per_step": ms, "tok_s": w.total_tokens / ms * 1e3, "steps": K,
                     "dtype": DTYPES[w.dtype], "tokens": w.total_tokens,
                     "kept_M": w.kept_lengths(), "stages": stages, "roofline": roof,
                     "clocks": clocks.summary()}
        del graph, layer
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
    return res


def run_gpu(args):
    import torch

    import learned_token_pruning_gate_b200 as tg
    from learned_token_pruning_gate_b200 import inputs as gen
    from learned_token_pruning_gate_b200 import dist as tgd

    rank, world, local = _dist_init(args.gpus)
    torch.cuda.set_device(local)
    # weak scaling: rank r draws its own prompt batch (same shapes, its own seed)
    w = tgd.rank_workload(gen.WORKLOADS[args.workload], rank)
    inp = gen.make_inputs(w)
    dev = torch.device("cuda", local)
    layer = _make_layer(tg, inp, w, dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    graph = layer.capture()

    # ---- device-timed steps (inputs resident in HBM), CUDA graph replay --------
    K = args.steps
    tgd.barrier()
    with ClockSampler(local) as clocks:
        step_ms = _time_steps(graph, flush, stream, K, args.warmup)
    tgd.barrier()
    total_ms = tgd.max_over_ranks(float(np.sum(step_ms)), device=dev)
    if tg.device_status() != 0:
        raise SystemExit("a kernel reported a timed-out wait")

    # ---- per-kernel times for the roofline (same launches, one event pair each) --
    stage_ms = _time_stages(layer, flush, stream, min(K, 50))

    # ---- end to end: pinned host inputs -> device -> 4 C-ABI calls -> host -----
    pinned = {n: getattr(inp, n).pin_memory() for n in ("h", "q", "k", "v")}
    out_host = torch.empty(layer.out.shape, dtype=layer.out.dtype, pin_memory=True)
    kept_host = torch.empty(layer.kept_idx.shape, dtype=torch.int32, pin_memory=True)
    h2d = sum(t.numel() * t.element_size() for t in pinned.values())
    d2h = out_host.numel() * out_host.element_size() + kept_host.numel() * 4
    n_e2e = max(min(K, 20), 3)

    def e2e_step():
        layer.h.copy_(pinned["h"], non_blocking=True)
        layer.q.copy_(pinned["q"], non_blocking=True)
        layer.k.copy_(pinned["k"], non_blocking=True)
        layer.v.copy_(pinned["v"], non_blocking=True)
        layer.run(stream.cuda_stream)
        out_host.copy_(layer.out, non_blocking=True)
        kept_host.copy_(layer.kept_idx, non_blocking=True)

    for _ in range(3):
        e2e_step()
    tgd.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(n_e2e):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = tgd.max_over_ranks(e0.elapsed_time(e1), device=dev)
    tgd.barrier()

    # ---- report -------------------------------------------------------------------
    tokens = w.total_tokens
    value = tgd.aggregate_throughput(tokens, K, total_ms, world)
    pk = _peaks()
    stages, roof = _stages_and_roofline(tg, layer, w, args.workload, stage_ms, pk)
    e2e_value = tgd.aggregate_throughput(tokens, n_e2e, e2e_ms, world)

    result = {
        "metric": METRIC, "value": value, "unit": "tok/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": total_ms / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": DTYPES[w.dtype], "data": "synthetic",
        "config": {**_workload_config(args.workload, w, world),
                   "l2": f"flushed between timed steps ({L2_FLUSH_BYTES >> 20} MiB write)",
                   "timing": "CUDA events per step around a CUDA-graph replay of the 4 launches"},
        "gpu_launches": 4 * K,
        "e2e": {"value": e2e_value, "unit": "tok/s", "h2d_bytes_per_step": int(h2d),
                "d2h_bytes_per_step": int(d2h), "steps": n_e2e},
        "roofline": roof,
        "stages": stages,
        "clocks": clocks.summary(),
    }
    del graph, layer, pinned
    torch.cuda.empty_cache()
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(inp, seconds=args.cpu_seconds)
    del inp
    if world == 1 and not args.headline_only:
        result["workloads"] = _other_workloads(tg, gen, dev, stream, flush, pk,
                                               max(3, min(K, args.other_steps)))
        result["gpu_launches_workloads"] = 4 * sum(
            v["steps"] + 3 for v in result["workloads"].values())
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


def cpu_baseline(inp, seconds=15.0, repeats=1):
    """The oracle, as it stands, on the host cores over a bounded sample of the
    workload, extrapolated to the whole step by the work it does."""
    import oracle

    w = inp.w
    N = w.total_tokens
    rng = np.random.default_rng(0)
    h32, W1 = inp.f32("h"), inp.f32("W1")
    t_gate_row = None
    n_rows = 256
    while True:  # size the gate sample to ~1/3 of the budget
        rows = rng.integers(0, N, n_rows)
        t0 = time.perf_counter()
        oracle.gate_score(h32, W1, inp.b1.numpy(), inp.w2.numpy(), inp.b2, rows=rows)
        dt = time.perf_counter() - t0
        t_gate_row = dt / n_rows
        if dt > seconds / 3 or n_rows >= N:
            break
        n_rows = min(N, int(n_rows * max(2.0, (seconds / 3) / max(dt, 1e-3))))
    gate_rows = n_rows
    # top-K and compaction run whole on scores drawn for the sample
    z = np.random.default_rng(1).standard_normal(N).astype(np.float32)  # score-shaped input
    t0 = time.perf_counter()
    kept, cu_kept = oracle.topk_select(z, inp.cu_seqlens, inp.doc_begin, inp.doc_end, inp.budget)
    t_topk = time.perf_counter() - t0
    t0 = time.perf_counter()
    qc = oracle.gather_rows(kept, inp.cu_seqlens, inp.f32("q"), w.n_q_heads, w.head_dim,
                            w.rope_theta)
    kc = oracle.gather_rows(kept, inp.cu_seqlens, inp.f32("k"), w.n_kv_heads, w.head_dim,
                            w.rope_theta)
    vc = oracle.gather_rows(kept, inp.cu_seqlens, inp.f32("v"))
    hc = oracle.gather_rows(kept, inp.cu_seqlens, h32)
    ls = oracle.logsig(kept, inp.cu_seqlens, inp.doc_begin, inp.doc_end, z)
    t_gather = time.perf_counter() - t0
    del hc
    # attention: a sample of query rows, extrapolated by visible-key count
    M = len(kept)
    lens = np.diff(cu_kept)
    vis_total = float(np.sum(lens * (lens + 1) / 2.0))
    n_q = 32
    while True:
        rows = np.sort(rng.integers(0, M, n_q))
        b_of = np.searchsorted(cu_kept, rows, side="right") - 1
        vis = float(np.sum(rows - cu_kept[b_of] + 1))
        t0 = time.perf_counter()
        oracle.gated_attention(qc, kc, vc, cu_kept, ls, inp.gain.numpy(), inp.temp.numpy(),
                               rows=rows)
        dt = time.perf_counter() - t0
        if dt > seconds / 3 or n_q >= M:
            break
        n_q = min(M, int(n_q * max(2.0, (seconds / 3) / max(dt, 1e-3))))
    t_attn = dt * vis_total / max(vis, 1.0)
    total = t_gate_row * N + t_topk + t_gather + t_attn
    return {"value": N / total, "unit": "tok/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": (f"gate on {gate_rows} of {N} tokens, top-K and compaction whole, "
                       f"attention on {n_q} of {M} query rows (all heads); extrapolated by "
                       f"tokens and by visible keys"),
            "seconds_per_step_extrapolated": total}


def _workload_config(name, w, world):
    """The workload keys of the bench line's config (shared by both arms)."""
    return {"workload": name, "prompts_per_gpu": w.batch, "seq_len": list(w.seqlens),
            "question": list(w.question), "budget_K": list(w.budgets), "kept_M": w.kept_lengths(),
            "d_model": w.d_model, "gate": f"{w.d_model}->{w.d_hidden}->1",
            "heads": f"{w.n_q_heads}q/{w.n_kv_heads}kv x {w.head_dim}",
            "parallelism": f"replicas x{world} (independent prompts, no collective)"}


def run_reference(args):
    """Reference arm: the CPU oracle on this workload, on the host cores."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    from learned_token_pruning_gate_b200 import inputs as gen

    w = gen.WORKLOADS[args.workload]
    inp = gen.make_inputs(w)
    per_step = max(2.0, min(20.0, 120.0 / max(args.steps + args.warmup, 1)))
    for _ in range(args.warmup):
        cpu_baseline(inp, seconds=per_step / 4)
    vals = []
    t0 = time.perf_counter()
    for _ in range(args.steps):
        vals.append(cpu_baseline(inp, seconds=per_step))
    wall = time.perf_counter() - t0
    value = float(np.median([v["value"] for v in vals]))
    cb = dict(vals[-1])
    cb["value"] = value
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tok/s",
        "n_gpus": int(os.environ.get("WORLD_SIZE", args.gpus)), "device": "host cores",
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": w.total_tokens / value * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {**_workload_config(args.workload, w, int(os.environ.get("WORLD_SIZE", args.gpus))),
                   "timing": "wall clock of the fp64 oracle on rank 0's host cores; each step a "
                             "bounded sample of the workload, extrapolated to all of it"},
        "cpu_baseline": cb,
        "e2e": {"value": value, "unit": "tok/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "wall_s": wall, "oracle_threads": oracle.num_threads()}), flush=True)


def run_ncu_case(args):
    """Untimed: build the workload and run `--steps` plain steps (for ncu captures)."""
    import torch

    import learned_token_pruning_gate_b200 as tg
    from learned_token_pruning_gate_b200 import inputs as gen
    from learned_token_pruning_gate_b200.pipeline import GatedLayer

    w = gen.WORKLOADS[args.workload]
    inp = gen.make_inputs(w)
    d = lambda t: t.cuda().contiguous()  # noqa: E731
    layer = GatedLayer(d(inp.h), d(inp.q), d(inp.k), d(inp.v), d(inp.W1), d(inp.b1), d(inp.w2),
                       inp.b2, d(inp.gain), d(inp.temp), inp.cu_seqlens, inp.doc_begin,
                       inp.doc_end, inp.budget, rope_theta=w.rope_theta)
    bwd = None
    if args.backward:
        o, lse = tg.gated_attention(layer.q_c, layer.k_c, layer.v_c, layer.cu_kept_host, layer.logsig,
                                    layer.gain, layer.temp, want_lse=True)
        dout = gen.attention_output_grad(layer.M, w.n_q_heads, w.head_dim, w.seed, w.dtype).cuda()
        bwd = lambda: tg.gated_attention_backward(  # noqa: E731
            layer.q_c, layer.k_c, layer.v_c, layer.cu_kept_host, layer.logsig, layer.gain,
            layer.temp, o, lse, dout)
    delta = None
    if args.delta:
        # a gated-delta-rule layer over the kept rows (one state head per query head)
        _, dq, dkk, dvv, dla, dbeta = gen.delta_inputs([layer.M], w.n_q_heads, w.head_dim, w.seed,
                                                       w.dtype)
        dq, dkk, dvv, dla, dbeta = (d(x) for x in (dq, dkk, dvv, dla, dbeta))
        dws = torch.empty(tg.delta_scan_workspace_bytes(layer.cu_kept_host, w.n_q_heads, w.head_dim),
                          dtype=torch.uint8, device="cuda")
        delta = lambda: tg.gated_delta_scan(dq, dkk, dvv, layer.cu_kept_host, dla, dbeta,  # noqa: E731
                                            algo=args.delta_algo, workspace=dws)
    for _ in range(args.steps):
        layer.run()
        if bwd:
            bwd()
        if delta:
            delta()
    torch.cuda.synchronize()
    if tg.device_status() != 0:
        raise SystemExit("a kernel reported a timed-out wait")
    print(json.dumps({"ncu_case": args.workload, "steps": args.steps, "N": layer.N,
                      "M": layer.M}))


def _library_baselines(layer, inp, w, res, timed):
    """Library calls doing each stage's operation (or its main part) on the same
    shapes and buffers, timed like the stages (L2 flushed, CUDA events): context
    beside the stage times, never on the layer's path.  gate: the cuBLAS GEMM of
    the residual with W1 alone (no GELU, w2 or bias); top-K: torch.topk over each
    prompt's document span; gather: torch.index_select of the four tensors, and
    one device copy of the same bytes; attention: PyTorch SDPA (cuDNN, flash)
    causal over each prompt's kept rows, without the key bias.  The 1-element
    add is the floor of this timing method."""
    import torch
    import torch.nn.functional as F
    from torch.nn.attention import SDPBackend, sdpa_kernel

    h, q, k, v, W1 = res[0], res[1], res[2], res[3], res[4]
    dev = h.device
    out = {}
    tiny = torch.zeros(1, device=dev)
    out["floor_1_element_add_us"] = timed(lambda: tiny.add_(1), 20)
    w1t = W1.t() if W1.shape[0] != h.shape[1] else W1
    out["cublas_gemm_residual_w1_us"] = timed(lambda: torch.matmul(h, w1t), 20)
    cu = np.asarray(inp.cu_seqlens)
    spans = [(int(cu[b] + inp.doc_begin[b]), int(cu[b] + inp.doc_end[b]), int(kb))
             for b, kb in enumerate(inp.budget)]
    spans = [(a, e, min(kb, e - a)) for a, e, kb in spans if e > a and kb > 0]
    z = layer.z
    out["torch_topk_us"] = timed(lambda: [torch.topk(z[a:e], kb) for a, e, kb in spans], 20)
    kept = layer.kept_idx.long()
    M = int(kept.numel())
    dst = [torch.empty((M,) + tuple(t.shape[1:]), dtype=t.dtype, device=dev) for t in (h, q, k, v)]
    out["torch_index_select_x4_us"] = timed(
        lambda: [torch.index_select(t, 0, kept, out=o) for t, o in zip((h, q, k, v), dst)], 20)
    nb = sum(o.numel() * o.element_size() for o in dst)
    c_src = torch.empty(nb, dtype=torch.uint8, device=dev)
    c_dst = torch.empty_like(c_src)
    out["torch_copy_same_bytes_us"] = timed(lambda: c_dst.copy_(c_src), 20)
    del dst, c_src, c_dst
    hq, hkv, dh = w.n_q_heads, w.n_kv_heads, w.head_dim
    ck = np.asarray(layer.cu_kept_host)
    per = []
    for b in range(len(ck) - 1):
        a, e = int(ck[b]), int(ck[b + 1])
        if e <= a:
            continue
        heads = lambda t, n: t[a:e].reshape(e - a, n, dh).transpose(0, 1).unsqueeze(0)  # noqa: E731
        per.append((heads(layer.q_c, hq).contiguous(),
                    heads(layer.k_c, hkv).repeat_interleave(hq // hkv, dim=1).contiguous(),
                    heads(layer.v_c, hkv).repeat_interleave(hq // hkv, dim=1).contiguous()))
    for name, be in (("cudnn", SDPBackend.CUDNN_ATTENTION), ("flash", SDPBackend.FLASH_ATTENTION)):
        key = f"sdpa_{name}_causal_no_bias_us"
        try:
            with sdpa_kernel([be]):
                out[key] = timed(lambda: [F.scaled_dot_product_attention(a_, b_, c_, is_causal=True)
                                          for a_, b_, c_ in per], 20)
        except RuntimeError:
            out[key] = None
    del per
    torch.cuda.synchronize()
    return {key: (round(val, 2) if val is not None else None) for key, val in out.items()}


def run_extras(args):
    """Supplementary layer-level figures for one workload (one JSON line; not the
    bench line): the bias overhead of the gated attention (logsig vs none), the
    ungated full-N causal attention over every token of the same prompts, the
    gated step's stages for comparison, and the live device memory of one gated
    layer vs a full-N layer."""
    import torch

    import learned_token_pruning_gate_b200 as tg
    from learned_token_pruning_gate_b200 import inputs as gen
    from learned_token_pruning_gate_b200.pipeline import GatedLayer

    w = gen.WORKLOADS[args.workload]
    inp = gen.make_inputs(w)
    dev = torch.device("cuda", 0)
    d = lambda t: t.to(dev).contiguous()  # noqa: E731
    res = [d(x) for x in (inp.h, inp.q, inp.k, inp.v, inp.W1, inp.b1, inp.w2, inp.gain, inp.temp)]
    torch.cuda.synchronize()
    base = torch.cuda.memory_allocated()  # inputs resident: count what the step allocates
    torch.cuda.reset_peak_memory_stats()
    layer = GatedLayer(*res[:7], inp.b2, res[7], res[8], inp.cu_seqlens, inp.doc_begin,
                       inp.doc_end, inp.budget, rope_theta=w.rope_theta, algo=tg.ALGO_AUTO)
    layer.run()
    torch.cuda.synchronize()
    gated_peak = torch.cuda.max_memory_allocated() - base
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def timed(fn, reps):
        for _ in range(2):
            fn()
        torch.cuda.synchronize()
        ms = []
        for _ in range(reps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda._sleep(HOLD_CYCLES // 4)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            ms.append(a.elapsed_time(b))
        return float(np.median(ms)) * 1e3  # us

    import ctypes
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    stage_us = {s: timed(lambda s=s: getattr(layer, s)(st), 20) for s in GatedLayer.STAGES}
    library = _library_baselines(layer, inp, w, res, timed)
    # selection variants on the layer's scores: an 8-budget sweep in one launch vs
    # eight single-budget launches, and random-K from caller-drawn keys
    n_doc = np.asarray(inp.doc_end) - np.asarray(inp.doc_begin)
    sweep = [[max(1, int(f * nd)) for nd in n_doc]
             for f in (0.01, 0.02, 0.05, 0.0625, 0.1, 0.125, 0.25, 0.5)]
    sweep_one = timed(lambda: tg.topk_select_multi(layer.z, inp.cu_seqlens, inp.doc_begin,
                                                   inp.doc_end, sweep), 20)
    sweep_sep = timed(lambda: [tg.topk_select(layer.z, inp.cu_seqlens, inp.doc_begin, inp.doc_end,
                                              k) for k in sweep], 20)
    keys = torch.from_numpy(gen.random_keys(w.total_tokens, seed=w.seed).view(np.int32)).to(dev)
    rand_us = timed(lambda: tg.random_select(keys, inp.cu_seqlens, inp.doc_begin, inp.doc_end,
                                             inp.budget), 20)
    ws = layer.workspace
    with_bias = timed(lambda: tg.gated_attention(layer.q_c, layer.k_c, layer.v_c, layer.cu_kept_host,
                                                 layer.logsig, layer.gain, layer.temp,
                                                 out=layer.out, workspace=ws), 20)
    no_bias = timed(lambda: tg.gated_attention(layer.q_c, layer.k_c, layer.v_c, layer.cu_kept_host,
                                               None, layer.gain, layer.temp, out=layer.out,
                                               workspace=ws), 20)
    # backward of the gated attention w.r.t. log-gates, gains, temperatures (training the
    # gate): S and dP over the causal triangle, the same flop count as the forward
    Mk = sum(w.kept_lengths())
    o_f, lse_f = tg.gated_attention(layer.q_c, layer.k_c, layer.v_c, layer.cu_kept_host,
                                    layer.logsig, layer.gain, layer.temp, want_lse=True,
                                    workspace=ws)
    dout = gen.attention_output_grad(Mk, w.n_q_heads, w.head_dim, w.seed, w.dtype).to(dev)
    bws = torch.empty(tg.attention_backward_workspace_bytes(layer.cu_kept_host, w.n_q_heads),
                      dtype=torch.uint8, device=dev)
    bwd_us = timed(lambda: tg.gated_attention_backward(
        layer.q_c, layer.k_c, layer.v_c, layer.cu_kept_host, layer.logsig, layer.gain, layer.temp,
        o_f, lse_f, dout, workspace=bws), 20)
    kept_flops = float(sum(2.0 * w.head_dim * w.n_q_heads * m * (m + 1) for m in w.kept_lengths()))
    # a stack of 4 Qwen3-1.7B-shaped upper layers over the kept rows (random init):
    # shared kept set and log-gates, per-layer gain and temperature, compacted KV cache
    stack = None
    if w.dtype == "bf16":
        from learned_token_pruning_gate_b200.pipeline import GatedStack
        n_up = 4
        _, _, _, _, sl = gen.stack_inputs([1] * len(w.kept_lengths()), n_up, w.d_model, w.n_q_heads,
                                          w.n_kv_heads, w.head_dim, 6144, w.seed, w.dtype)
        sl = [{k_: v_.to(dev) for k_, v_ in ly.items()} for ly in sl]
        st_ = GatedStack(sl, w.n_q_heads, w.n_kv_heads, w.head_dim, inp.cu_seqlens,
                         layer.cu_kept_host, layer.kept_idx, layer.logsig, rope_theta=w.rope_theta)
        xs = layer.h_c.clone()
        stack_us = timed(lambda: st_.run(xs), 10)
        # the same layers' attention alone (per layer, shared q/k/v buffers)
        att_us = timed(lambda: [tg.gated_attention(st_.q, st_.cache_k[i], st_.cache_v[i],
                                                   layer.cu_kept_host, layer.logsig, ly["gain"],
                                                   ly["temp"], out=st_.o, workspace=st_.ws)
                                for i, ly in enumerate(sl)], 10)
        kv_c = int(st_.cache_k.numel() + st_.cache_v.numel()) * 2
        stack = {"layers": n_up, "us": round(stack_us, 2), "us_per_layer": round(stack_us / n_up, 2),
                 "attention_us": round(att_us, 2),
                 "kv_cache_bytes": kv_c, "kv_cache_full_n_bytes": int(kv_c * w.total_tokens / Mk),
                 "note": "Qwen3-1.7B-shaped (d 2048, 16/8 x 128, MLP 6144), random init; GEMMs "
                         "cuBLAS, other steps libtokengate"}
        del st_, xs, sl
    # a Gated DeltaNet layer of a hybrid backbone over the same kept rows: the gated
    # delta rule, sequential over each prompt's rows, fp32 state per (prompt, head)
    dcu, dq, dkk, dvv, dla, dbeta = gen.delta_inputs(w.kept_lengths(), w.n_q_heads, w.head_dim,
                                                     w.seed, w.dtype)
    dq, dkk, dvv, dla, dbeta = (d(x) for x in (dq, dkk, dvv, dla, dbeta))
    d_out = torch.empty_like(dvv)
    d_state = torch.empty((len(dcu) - 1, w.n_q_heads, w.head_dim, w.head_dim), dtype=torch.float32,
                          device=dev)
    rec_us = timed(lambda: tg.gated_delta_scan(dq, dkk, dvv, dcu, dla, dbeta, out=d_out,
                                               state=d_state, algo="recurrent"), 10)
    dws = torch.empty(tg.delta_scan_workspace_bytes(dcu, w.n_q_heads, w.head_dim), dtype=torch.uint8,
                      device=dev)
    delta_us = timed(lambda: tg.gated_delta_scan(dq, dkk, dvv, dcu, dla, dbeta, out=d_out,
                                                 state=d_state, algo="chunked", workspace=dws), 10)
    # per row and head, as the recurrence counts it: S k, the rank-1 update (scale
    # + FMA) and S q over d x d -- the chunked form does about as many flops
    delta_flops = 7.0 * w.head_dim ** 2 * w.n_q_heads * Mk
    fp32_peak = FP32_FMA_TFLOPS
    delta = {"us": round(delta_us, 2), "recurrent_us": round(rec_us, 2),
             "rows_per_s": round(Mk / delta_us * 1e6),
             "tflops_fp32": round(delta_flops / delta_us / 1e6, 3),
             "frac_alu_nominal": round(delta_flops / delta_us / 1e6 / fp32_peak, 4),
             "heads": w.n_q_heads, "head_dim": w.head_dim, "workspace_bytes": int(dws.numel()),
             "note": "chunked scan (64-row chunks: parallel per-chunk solve, then the state "
                     "passed chunk to chunk over 16-row blocks); recurrent_us: row by row"}
    del dq, dkk, dvv, dla, dbeta, d_out, d_state, dws
    del layer, o_f, lse_f, dout, bws
    torch.cuda.synchronize()
    # ungated: every token of every prompt attends causally, no bias (the layer without a gate)
    q, k, v = res[1], res[2], res[3]
    base = torch.cuda.memory_allocated()
    torch.cuda.reset_peak_memory_stats()
    out = torch.empty_like(q)
    lens = np.diff(np.asarray(inp.cu_seqlens))
    full_ws = tg.attention_workspace_bytes(inp.cu_seqlens, w.n_q_heads, w.n_kv_heads, w.head_dim)
    fws = torch.empty(full_ws, dtype=torch.uint8, device=dev) if full_ws else None
    gain, temp = res[7], res[8]
    reps = 3 if w.total_tokens > 40000 else 10
    ungated = timed(lambda: tg.gated_attention(q, k, v, inp.cu_seqlens, None, gain, temp, out=out,
                                               workspace=fws), reps)
    torch.cuda.synchronize()
    full_peak = torch.cuda.max_memory_allocated() - base
    hq, dh = w.n_q_heads, w.head_dim
    esz = 2 if w.dtype == "bf16" else 4
    full_flops = float(sum(2.0 * dh * hq * n * (n + 1) for n in lens))
    gated_total = sum(stage_us.values())
    print(json.dumps({
        "extras": args.workload, "tokens": w.total_tokens, "kept": w.kept_lengths(),
        "stage_us": {s: round(v, 2) for s, v in stage_us.items()},
        "gated_layer_us": round(gated_total, 2),
        "library_same_shapes_us": library,
        "bias_overhead": {"with_bias_us": round(with_bias, 2), "no_bias_us": round(no_bias, 2),
                          "ratio": round(with_bias / no_bias, 4)},
        "ungated_attention": {"us": round(ungated, 2), "tflops": round(full_flops / ungated / 1e6, 1),
                              "frac_measured_bf16": round(full_flops / ungated / 1e6 / _peaks()["bf16"], 4)},
        "speedup_vs_ungated_attention": round(ungated / gated_total, 2),
        "upper_stack": stack,
        "delta_scan": delta,
        "attention_backward": {"us": round(bwd_us, 2),
                               "tflops": round(kept_flops / bwd_us / 1e6, 1),
                               "frac_measured_bf16": round(kept_flops / bwd_us / 1e6 / _peaks()["bf16"], 4),
                               "grads": "log-gates (and kept scores), gains, temperatures"},
        "selection": {"budget_sweep_8_one_launch_us": round(sweep_one, 2),
                      "budget_sweep_8_separate_launches_us": round(sweep_sep, 2),
                      "random_k_us": round(rand_us, 2), "topk_us": round(stage_us["topk"], 2)},
        "memory_bytes": {
            "gated_step_allocated": int(gated_peak), "ungated_step_allocated": int(full_peak),
            "kv_gated": int(2 * sum(w.kept_lengths()) * w.n_kv_heads * dh * esz),
            "kv_ungated": int(2 * w.total_tokens * w.n_kv_heads * dh * esz),
            "attention_live_gated": int(sum(w.kept_lengths()) * (2 * hq + 2 * w.n_kv_heads) * dh * esz),
            "attention_live_ungated": int(w.total_tokens * (2 * hq + 2 * w.n_kv_heads) * dh * esz)},
        "note": "one layer: ungated = causal attention over all N tokens (q,k,v already resident); "
                "gated = gate + top-K + compaction + gated attention; *_step_allocated = device "
                "memory each step allocates with its inputs resident (gated: z, kept rows, "
                "compacted h/q/k/v, bias, output, workspace; ungated: output); kv_* and "
                "attention_live_* (q, k, v, o) are the tensor sizes the layer holds",
    }), flush=True)



def main():
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--headline-only", action="store_true",
                    help="skip the other configurations' block (workloads)")
    ap.add_argument("--other-steps", type=int, default=20,
                    help="timed steps per configuration in the workloads block")
    ap.add_argument("--extras", action="store_true",
                    help="print bias overhead, ungated full-N attention and memory figures")
    ap.add_argument("--ncu-case", action="store_true",
                    help="untimed: run --steps plain steps of the workload (profiling)")
    ap.add_argument("--delta", action="store_true",
                    help="with --ncu-case: also run the gated-delta-rule scan over the kept rows")
    ap.add_argument("--delta-algo", default="chunked", choices=["chunked", "recurrent"],
                    help="with --ncu-case --delta: which form of the scan")
    ap.add_argument("--backward", action="store_true",
                    help="with --ncu-case: also run the attention backward after each step")
    args = ap.parse_args()
    if args.ncu_case:
        run_ncu_case(args)
    elif args.extras:
        run_extras(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
