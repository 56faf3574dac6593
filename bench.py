#!/usr/bin/env python
"""Joint-block throughput of the NVFP4 / FP8 FLUX-3-Image-Klein-style joint
transformer block on B200.

A step is one forward pass of the whole block (LN1+adaLN+NVFP4, QKV GEMM with
RoPE, FP8 cast, joint attention, NVFP4 of O, output GEMM with gated residual,
LN2+adaLN+NVFP4, MLP-up GEMM with SwiGLU, NVFP4 of h, MLP-down GEMM with gated
residual) over one image's token sequence, inputs resident in HBM.  The
default workload is the 1024x1024 text-to-image block: 512 text + 4,096 image
tokens (4,608), hidden 3072, 24 heads, MLP 9216, FP8 attention
(token counts: "Welcome FLUX.3 Image Klein in Diffusers", The VAE and
Tokenization; "FLUX.3 Image Klein Brings 2-Second AI Image Generation to
Diffusers", Summary).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...     # the CPU oracle as the reference arm

Prints one JSON line (rank 0).  Under torchrun every rank runs its own image's
block (data parallel over images, no collective on the data path): weak
scaling; timing is the max over ranks of device time.
"""

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

from synth import MOD_NAMES, WORKLOADS, block_inputs  # noqa: E402

METRIC = "joint-block tokens/s & % of dense FP4/FP8 tensor peak, 1024² T2I and I2I"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}
# dense tensor-core ratios to bf16 (nominal B200: bf16 2.25, fp8 4.5, fp4 9 PFLOP/s)
RATIO = {"fp4": 4.0, "fp8": 2.0, "bf16": 1.0}
STAGES = ("ln1", "qkv_gemm", "fp8_cast", "attention", "quant_o", "out_gemm", "ln2", "mlp_up_gemm", "quant_h",
          "mlp_down_gemm")
KERNELS_PER_STAGE = {"ln1": 2, "qkv_gemm": 1, "fp8_cast": 1, "attention": 1, "quant_o": 1, "out_gemm": 1, "ln2": 2,
                     "mlp_up_gemm": 1, "quant_h": 1, "mlp_down_gemm": 1}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        d["source"] = "measured"
        return d
    return dict(FALLBACK_PEAKS)


def stage_work(wl):
    """Algorithmic work per stage: ("flop", n, dtype) or ("byte", n)."""
    T, D, H, F = wl.n_tokens, wl.hidden, wl.heads, wl.mlp_hidden
    nv = 2 + 0.5 + 1 / 16          # bf16 read + NVFP4 codes + scales, bytes per element
    att_dtype = "fp8" if wl.attn == "fp8" else "bf16"
    return {
        "ln1": ("byte", T * D * nv),
        "qkv_gemm": ("flop", 2.0 * T * 3 * D * D, "fp4"),
        "fp8_cast": ("byte", T * 3 * D * 3.0),
        "attention": ("flop", 4.0 * T * T * H * 128, att_dtype),
        "quant_o": ("byte", T * D * nv),
        "out_gemm": ("flop", 2.0 * T * D * D, "fp4"),
        "ln2": ("byte", T * D * nv),
        "mlp_up_gemm": ("flop", 2.0 * T * 2 * F * D, "fp4"),
        "quant_h": ("byte", T * F * nv),
        "mlp_down_gemm": ("flop", 2.0 * T * D * F, "fp4"),
    }


def committed_traffic(wl, stage):
    """DRAM bytes per launch of a stage's kernel from the committed ncu capture
    (profiles/dram_traffic_<workload>.json), or None when there is none or the
    kernel source changed since it was taken."""
    import hashlib

    path = os.path.join(ROOT, "profiles", f"dram_traffic_{wl.name}.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    ent = d.get(stage)
    if not ent:
        return None
    src = os.path.join(ROOT, "diffusion_transformer_image_nvfp4_b200", "csrc", ent["source"])
    if not os.path.exists(src) or hashlib.sha1(open(src, "rb").read()).hexdigest() != ent["sha1"]:
        return None
    return ent["bytes"]


def tensor_peak_key(clk):
    """Burst bf16 peak when the timed region ran at full clock (no power cap
    pulled the SM clock down), the sustained one otherwise."""
    if clk and clk.get("sm_mhz") and clk.get("sm_max_mhz") and clk["sm_mhz"] >= 0.9 * clk["sm_max_mhz"]:
        return "bf16_tflops"
    return "bf16_tflops_sustained"


def roofline_entry(work, ms, peaks, peak_key="bf16_tflops_sustained"):
    if ms <= 0:
        return None
    if work[0] == "flop":
        ach = work[1] / (ms * 1e-3) / 1e12
        peak = peaks[peak_key] * RATIO[work[2]]
        return {"bound": "tensor", "achieved": round(ach, 2), "peak": round(peak, 1), "unit": "TFLOP/s",
                "frac": round(ach / peak, 4), "dtype": work[2]}
    ach = work[1] / (ms * 1e-3) / 1e9
    peak = peaks["hbm_gbs"]
    return {"bound": "hbm", "achieved": round(ach, 1), "peak": round(peak, 1), "unit": "GB/s",
            "frac": round(ach / peak, 4)}


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples taken during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None

        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        mx = [num(r[2]) for r in rows if num(r[2]) is not None]
        reasons = set()
        for r in rows:
            for name, val in zip(("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"),
                                 r[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(rows)}


def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus and world > 1:
        raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE {world}")
    return world, rank, local


# ------------------------------------------------ multi-rank host logic
# The same functions serve the NCCL run (device tensors) and the gloo CPU
# tests of the N > 1 path.
def rank_barrier(world, device=None):
    """Barrier over the ranks (when there are several), then a device sync."""
    if world > 1:
        import torch.distributed as dist

        dist.barrier()
    if device is not None and device.type == "cuda":
        torch.cuda.synchronize(device)


def rank_max(v, world, device):
    """max over ranks of a per-rank number (the job's time is its slowest rank)."""
    if world == 1:
        return float(v)
    import torch.distributed as dist

    t = torch.tensor([float(v)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_value(world, tokens_per_rank, steps, total_ms):
    """Weak scaling: every rank runs its own image's block; the job processes
    world * tokens_per_rank tokens per step in the slowest rank's time."""
    return world * tokens_per_rank * steps / (total_ms * 1e-3)


def config_of(wl, extra=None):
    c = {"workload": wl.name, "tokens": wl.n_tokens, "text_tokens": wl.n_text,
         "image_grid": f"{wl.grid_h}x{wl.grid_w}", "reference_images": wl.n_ref, "hidden": wl.hidden,
         "heads": wl.heads, "head_dim": 128, "mlp_hidden": wl.mlp_hidden, "attention": wl.attn,
         "weights": "NVFP4 (E2M1, UE4M3 per 16, fp32 global), random N(0,0.02)",
         "activations": "NVFP4 GEMM inputs, bf16 residual stream N(0,1)"}
    if extra:
        c.update(extra)
    return c


# --------------------------------------------------------------------- oracle
def oracle_sample(wl, n_text, grid_rows):
    """Inputs of a bounded slice of the workload for the CPU oracle: the first
    n_text text tokens and the first grid_rows rows of the image grid, full
    widths, the workload's own weights and modulation vectors."""
    import numpy as np

    from oracle import block, nvfp4

    inp = block_inputs(wl)
    x = inp["x"].float().numpy()
    rows = np.concatenate([np.arange(n_text), wl.n_text + np.arange(grid_rows * wl.grid_w)])
    lay = block.TokenLayout(n_text, grid_rows, wl.grid_w, 0)
    w = {n: nvfp4.quantize(inp[n].float().numpy()) for n in ("wqkv", "wo", "w1", "w2")}
    mod = {n: inp[n].float().numpy() for n in MOD_NAMES}
    return x[rows], mod, w, lay


def oracle_threads():
    try:
        from threadpoolctl import threadpool_info

        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def _oracle_block_seconds(wl, n_text, grid_rows):
    from oracle import block

    x, mod, w, lay = oracle_sample(wl, n_text, grid_rows)
    attn = "fp8" if wl.attn == "fp8" else "exact"
    t0 = time.perf_counter()
    block.block_forward(x, mod, w, lay, wl.heads, attn=attn)
    return time.perf_counter() - t0, lay.n_tokens


def cpu_baseline(wl, n_text=256, grid_rows=4):
    """The oracle on the host cores: a bounded slice of the workload with all
    BLAS threads, plus single-thread figures (the whole tiny block, and a
    128-token slice of this workload)."""
    dt, T = _oracle_block_seconds(wl, n_text, grid_rows)
    out = {"value": round(T / dt, 3), "unit": UNIT, "cores": oracle_threads(), "kind": "oracle",
           "sample": f"{T}-token slice of {wl.name} ({n_text} text + {grid_rows} grid rows x {wl.grid_w}), "
                     f"full widths, weights pre-encoded (untimed), one block forward: {dt:.1f} s"}
    try:
        from threadpoolctl import threadpool_limits
    except Exception:
        return out
    single = {}
    with threadpool_limits(limits=1):
        tiny = WORKLOADS["tiny"]
        dt1, T1 = _oracle_block_seconds(tiny, tiny.n_text, tiny.grid_h)
        single["tiny"] = {"value": round(T1 / dt1, 3), "unit": UNIT, "cores": 1,
                          "sample": f"the whole tiny block ({T1} tokens): {dt1:.1f} s"}
        dt2, T2 = _oracle_block_seconds(wl, 64, 1)
        single[wl.name] = {"value": round(T2 / dt2, 3), "unit": UNIT, "cores": 1,
                           "sample": f"{T2}-token slice of {wl.name} (64 text + 1 grid row), full widths: {dt2:.1f} s"}
    out["single_thread"] = single
    return out


def run_reference(args, wl):
    world, rank, _ = dist_setup(args.gpus)
    if rank != 0:
        return
    from oracle import block

    n_text, grid_rows = 64, 1
    x, mod, w, lay = oracle_sample(wl, n_text, grid_rows)
    attn = "fp8" if wl.attn == "fp8" else "exact"
    for _ in range(args.warmup):
        block.block_forward(x, mod, w, lay, wl.heads, attn=attn)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        block.block_forward(x, mod, w, lay, wl.heads, attn=attn)
        times.append(time.perf_counter() - t0)
    T = lay.n_tokens
    total = sum(times)
    value = T * args.steps / total
    sample = (f"each step: {T}-token slice of {wl.name} ({n_text} text + {grid_rows} grid row x {wl.grid_w}), "
              f"full widths, through the fp64 CPU oracle")
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * total / args.steps, 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded N(0,1) activations, N(0,0.02) weights, N(0,0.1) modulation)",
            "config": config_of(wl, {"sample_tokens": T}),
            "cpu_baseline": {"value": round(value, 3), "unit": UNIT, "cores": oracle_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 3), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------ ours
GATE_CYCLES = 20_000_000   # ~10 ms at B200 clocks: covers enqueueing a chunk of steps
CHUNK = 16


def gated(n_steps, body):
    """Enqueue the steps in chunks behind a short GPU sleep, so the queue is
    already full when the GPU reaches them and host-side enqueue time never
    shows up as device time."""
    for c0 in range(0, n_steps, CHUNK):
        torch.cuda._sleep(GATE_CYCLES)
        for i in range(c0, min(n_steps, c0 + CHUNK)):
            body(i)


def block_setup(kl, wl, dev):
    inp = block_inputs(wl)
    T, D, H, F = wl.n_tokens, wl.hidden, wl.heads, wl.mlp_hidden
    d = {k: v.to(dev) for k, v in inp.items()}
    W = kl.prepare_block_weights(d["wqkv"], d["wo"], d["w1"], d["w2"])
    cs = kl.rope_table(wl.n_text, wl.grid_h, wl.grid_w, wl.n_ref, device=dev)
    mod = {n: d[n] for n in MOD_NAMES}
    out = torch.empty_like(d["x"])
    ws = torch.empty(kl.block_workspace_size(T, D, H, F, wl.attn), dtype=torch.uint8, device=dev)
    return inp, W, cs, d["x"], mod, out, ws


def measure_block(kl, wl, dev, steps, warmup, flush, world, peaks, clocks=None, e2e=False):
    """One workload's block: graph-replay tokens/s (L2 flushed before every
    step), per-stage device times from direct launches with library-recorded
    events, roofline fractions; with ``e2e`` also the end-to-end number
    through kl_joint_block_forward_host on pinned host buffers."""
    inp, W, cs, x, mod, out, ws = block_setup(kl, wl, dev)
    T, D, H, F = wl.n_tokens, wl.hidden, wl.heads, wl.mlp_hidden
    for _ in range(warmup):
        kl.joint_block_forward(W, x, mod, cs, H, F, attn=wl.attn, out=out, workspace=ws)
    torch.cuda.synchronize()
    st = kl.device_status()
    if st != "KL_OK":
        raise SystemExit(f"{wl.name}: device status after warm-up: {st}")

    # value: the block captured once in a CUDA graph and replayed; every step
    # an L2 flush, then one replay bracketed by events on the stream
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        kl.joint_block_forward(W, x, mod, cs, H, F, attn=wl.attn, out=out, workspace=ws)
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]

    def graph_step(i):
        flush.zero_()
        starts[i].record()
        graph.replay()
        ends[i].record()

    rank_barrier(world, dev)
    if clocks is not None:
        clocks.start()
    gated(steps, graph_step)
    rank_barrier(world, dev)
    clk = clocks.stop() if clocks is not None else None
    total_ms = rank_max(sum(a.elapsed_time(b) for a, b in zip(starts, ends)), world, dev)
    del graph

    # per-stage breakdown: the same steps launched directly, the library
    # recording an event between the stages of every step
    stage_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(STAGES) + 1)] for _ in range(steps)]
    for row in stage_ev:
        for e in row:
            e.record()

    def eager_step(i):
        flush.zero_()
        kl.joint_block_forward(W, x, mod, cs, H, F, attn=wl.attn, out=out, workspace=ws, stage_events=stage_ev[i])

    rank_barrier(world, dev)
    gated(steps, eager_step)
    rank_barrier(world, dev)
    stage_ms = {s: sum(row[j].elapsed_time(row[j + 1]) for row in stage_ev) / steps for j, s in enumerate(STAGES)}
    eager_ms = sum(row[0].elapsed_time(row[-1]) for row in stage_ev) / steps

    res = {"workload": wl.name, "tokens": T, "steps": steps, "total_ms": total_ms, "clk": clk,
           "stage_ms": stage_ms, "eager_ms": eager_ms}
    if e2e:
        # end to end through the C ABI with host buffers: every step one
        # kl_joint_block_forward_host call (pinned x and modulation copied in,
        # the block, out copied back), all inside the timed events.  Steps
        # rotate over three streams, each with its own device workspace and
        # pinned output: a stream runs its step's copy in, block and copy out
        # in order, so with three in flight the copies of two steps overlap
        # the block of the third (independent images, as a caller with a
        # queue of them runs the API).  Each step moves several hundred MB
        # through HBM, more than the L2 holds, so nothing carries over in L2
        # between steps.
        x_h = inp["x"].pin_memory()
        mod_h = {n: inp[n].pin_memory() for n in MOD_NAMES}
        nstr = 3
        out_h = [torch.empty_like(x_h).pin_memory() for _ in range(nstr)]
        ws_h = [torch.empty(kl.lib().kl_block_host_workspace_size(T, D, H, F, kl.ATTN[wl.attn]), dtype=torch.uint8,
                            device=dev) for _ in range(nstr)]
        streams = [torch.cuda.Stream(device=dev) for _ in range(nstr)]
        main_s = torch.cuda.current_stream()

        def e2e_run(n):
            for i in range(n):
                with torch.cuda.stream(streams[i % nstr]):
                    kl.joint_block_forward_host(W, x_h, mod_h, cs, H, F, attn=wl.attn, out_host=out_h[i % nstr],
                                                workspace=ws_h[i % nstr])

        for s_ in streams:
            s_.wait_stream(main_s)
        e2e_run(max(warmup, nstr))
        torch.cuda.synchronize()
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        rank_barrier(world, dev)
        torch.cuda._sleep(GATE_CYCLES)  # the host enqueues the steps while the GPU sleeps
        start.record(main_s)
        for s_ in streams:
            s_.wait_stream(main_s)
        e2e_run(steps)
        for s_ in streams:
            main_s.wait_stream(s_)
        end.record(main_s)
        torch.cuda.synchronize()
        rank_barrier(world, dev)
        res["e2e_ms"] = rank_max(start.elapsed_time(end), world, dev)
        res["h2d"] = T * D * 2 + len(MOD_NAMES) * D * 2
        res["d2h"] = T * D * 2
        for o_h in out_h:
            if not torch.equal(o_h.to(dev), out):
                raise SystemExit(f"{wl.name}: host-buffer entry point disagrees with the device one")
    st = kl.device_status()
    if st != "KL_OK":
        raise SystemExit(f"{wl.name}: device status after timing: {st}")
    return res


def summarize(wl, res, peaks, pk, world):
    """tokens/s, TFLOP/s, per-stage roofline entries and the GEMM / attention
    fractions of one measured workload."""
    steps, total_ms, stage_ms = res["steps"], res["total_ms"], res["stage_ms"]
    work = stage_work(wl)
    stages = {}
    for s in STAGES:
        if wl.attn != "fp8" and s == "fp8_cast":
            continue
        ent = roofline_entry(work[s], stage_ms[s], peaks, pk) or {}
        ent["ms"] = round(stage_ms[s], 4)
        stages[s] = ent
    gemms = ("qkv_gemm", "out_gemm", "mlp_up_gemm", "mlp_down_gemm")
    gemm_ms = sum(stage_ms[s] for s in gemms)
    gemm_flop = sum(work[s][1] for s in gemms)
    fp4_peak = peaks[pk] * RATIO["fp4"]
    att_peak = peaks[pk] * RATIO["fp8" if wl.attn == "fp8" else "bf16"]
    return {"workload": wl.name, "tokens": wl.n_tokens,
            "value": round(whole_job_value(world, wl.n_tokens, steps, total_ms), 1), "unit": UNIT,
            "ms_per_step": round(total_ms / steps, 4), "steps": steps,
            "tflops": round((gemm_flop + work["attention"][1]) / (total_ms / steps * 1e-3) / 1e12, 2),
            "gemm_fp4_frac": round(gemm_flop / (gemm_ms * 1e-3) / 1e12 / fp4_peak, 4),
            "attention_frac": round(work["attention"][1] / (stage_ms["attention"] * 1e-3) / 1e12 / att_peak, 4),
            "ms_per_step_direct_launch": round(res["eager_ms"], 4), "stages": stages}


# secondary workloads measured after the main line (the metric names the
# 1024^2 T2I and I2I blocks; the multi-reference block is the stress case)
SECONDARY = {"t2i_1024": ("i2i_1024", "multiref_1024")}


def run_ours(args, wl):
    import diffusion_transformer_image_nvfp4_b200 as kl

    world, rank, local = dist_setup(args.gpus)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
    kl.lib()
    peaks = load_peaks()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)   # > 126 MB L2
    clocks = ClockSampler(local)
    res = measure_block(kl, wl, dev, args.steps, args.warmup, flush, world, peaks, clocks=clocks, e2e=True)
    clk = res["clk"]
    pk = tensor_peak_key(clk)
    main = summarize(wl, res, peaks, pk, world)
    stages = main["stages"]
    dom = max(stages, key=lambda s: stages[s]["ms"])
    roof = {k: stages[dom][k] for k in ("bound", "achieved", "peak", "unit", "frac")}
    roof["kernel"] = dom
    roof["traffic"] = committed_traffic(wl, dom)
    kind = "burst" if pk == "bf16_tflops" else "sustained"
    roof["peak_source"] = (f"{peaks['source']} ({kind} bf16 x nominal dense ratio)" if roof["bound"] == "tensor"
                           else f"{peaks['source']} (copy)")
    launches = sum(KERNELS_PER_STAGE[s] for s in stages) * args.steps

    line = {"metric": METRIC, "value": main["value"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": main["ms_per_step"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "nvfp4 (e2m1 x e2m1, fp32 acc) + e4m3 attention",
            "data": "synthetic (seeded N(0,1) activations, N(0,0.02) weights, N(0,0.1) modulation)",
            "config": config_of(wl, {"parallelism": f"dp{world} (one image per GPU)" if world > 1 else "single GPU",
                                     "l2": "flushed between timed steps (256 MiB write, outside the timed events)",
                                     "launch": "block captured once in a CUDA graph, replayed per step"}),
            "tflops": main["tflops"], "gemm_fp4_frac": main["gemm_fp4_frac"],
            "attention_frac": main["attention_frac"], "roofline": roof, "stages": stages, "gpu_launches": launches,
            "ms_per_step_direct_launch": main["ms_per_step_direct_launch"],
            "e2e": {"value": round(whole_job_value(world, wl.n_tokens, args.steps, res["e2e_ms"]), 1), "unit": UNIT,
                    "h2d_bytes_per_step": res["h2d"], "d2h_bytes_per_step": res["d2h"],
                    "via": "kl_joint_block_forward_host per step (pinned host x/modulation in, out back), steps "
                           "rotating over three streams with a workspace each, so the copies of two steps overlap "
                           "the block of the third; no L2 flush (each step moves more than the L2 holds)"},
            "clocks": clk}
    sec = []
    for name in (() if args.no_secondary else SECONDARY.get(wl.name, ())):
        w2 = WORKLOADS[name]
        r2 = measure_block(kl, w2, dev, min(args.steps, 50), args.warmup, flush, world, peaks)
        sec.append(summarize(w2, r2, peaks, pk, world))
        torch.cuda.empty_cache()
    if sec:
        line["secondary"] = sec
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.barrier()
        dist.destroy_process_group()


# ------------------------------------------------------------ DiT loop (c4)
def run_dit(args):
    """Per-image latency of the synthetic DiT loop (5 per-mode + 28 joint
    blocks at the 1024^2 T2I shape, 16 Euler steps), the 16 steps captured in
    one CUDA graph; weights and inputs drawn on the GPU (seeded)."""
    import diffusion_transformer_image_nvfp4_b200 as kl
    from synth import DIT_CONFIGS, dit_inputs

    cfg = DIT_CONFIGS["dit_t2i_1024"]
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    d = dit_inputs(cfg, device=dev, mods=args.mods)
    blocks = lambda bl: [kl.prepare_block_weights(b["wqkv"], b["wo"], b["w1"], b["w2"]) for b in bl]
    W = kl.DitWeights(kl.quantize_nvfp4(d["w_in"]), blocks(d["mode_text"]), blocks(d["mode_image"]),
                      blocks(d["joint"]), kl.quantize_nvfp4(d["w_out"]))
    for k in ("w_in", "w_out", "mode_text", "mode_image", "joint"):
        del d[k]
    torch.cuda.empty_cache()
    shape = kl.DitShape(cfg.n_text, cfg.grid_h, cfg.grid_w, cfg.channels, cfg.hidden, cfg.heads, cfg.mlp_hidden,
                        cfg.n_mode, cfg.n_joint, cfg.attn)
    ropes = (kl.rope_table(cfg.n_text, 0, 0, device=dev), kl.rope_table(0, cfg.grid_h, cfg.grid_w, device=dev),
             kl.rope_table(cfg.n_text, cfg.grid_h, cfg.grid_w, device=dev))
    ws = torch.empty(kl.dit_workspace_size(shape), dtype=torch.uint8, device=dev)
    w_abi = W.abi()
    # flow-matching timesteps from 1 to 0, optionally time-shifted
    ts = [args.shift * t / (1.0 + (args.shift - 1.0) * t) for t in (1.0 - i / cfg.n_steps for i in range(cfg.n_steps + 1))]
    mods = [(d["mod_mode"][i].contiguous(), d["mod_joint"][i].contiguous(), d["mod_final"][i].contiguous())
            for i in range(cfg.n_steps)]
    lat0 = d["latent"].contiguous()
    lat = lat0.clone()
    # Cache-DiT: the skip of blocks 1.. is a conditional node in the graph
    cache = kl.DitCache(shape, device=dev) if args.cache is not None else None

    def image():
        for i in range(cfg.n_steps):
            tau = args.sol_tau if i >= args.sol_dense_steps else 0.0  # Sol-Attention after the dense steps
            if cache is None:
                kl.dit_step(shape, W, lat, d["text"], *mods[i], *ropes, ts[i + 1] - ts[i], workspace=ws, w_abi=w_abi,
                            sol_tau=tau)
            else:
                kl.dit_step_cached(shape, W, cache, args.cache, lat, d["text"], *mods[i], *ropes, ts[i + 1] - ts[i],
                                   workspace=ws, w_abi=w_abi, sol_tau=tau)

    image()  # warm-up (eager)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        image()
    times = []
    for _ in range(args.warmup + args.steps):
        lat.copy_(lat0)
        if cache is not None:
            cache.reset()  # a new generation
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        graph.replay()
        b.record()
        times.append((a, b))
    torch.cuda.synchronize()
    ms = [a.elapsed_time(b) for a, b in times[args.warmup:]]
    st = kl.device_status()
    fin = bool(torch.isfinite(lat).all().item())
    blocks_per_image = cfg.n_steps * (2 * cfg.n_mode + cfg.n_joint)
    extra = {}
    if cache is not None:
        h = cache.header()  # the last replay's generation
        extra = {"cache_threshold": args.cache, "cached_steps_per_image": h["hits"], "steps_seen": h["steps"],
                 "last_residual_diff": h["diff"]}
    print(json.dumps({"metric": "per-image DiT latency, synthetic 1024^2 T2I loop", "value": round(statistics.median(ms), 3),
                      "unit": "ms", "higher_is_better": False, "images": args.steps, "warmup": args.warmup,
                      "config": {"workload": cfg.name, "steps": cfg.n_steps, "per_mode_blocks": cfg.n_mode,
                                 "joint_blocks": cfg.n_joint, "tokens": cfg.n_text + cfg.grid_h * cfg.grid_w,
                                 "latent": [2 * cfg.grid_h, 2 * cfg.grid_w, cfg.channels],
                                 "block_calls_per_image": blocks_per_image,
                                 "launch": "16 Euler steps captured in one CUDA graph", "time_shift": args.shift,
                                 "modulations": args.mods, "sol_tau": args.sol_tau,
                                 "sol_dense_steps": args.sol_dense_steps},
                      "min_ms": round(min(ms), 3), "device_status": st, "latent_finite": fin, **extra}), flush=True)


def run_sol(args):
    """Sol-Attention at the 1024^2 T2I attention shape (4,608 tokens, 24
    heads, FP8): device time of key-tile selection + sparse attention against
    dense attention, on seeded inputs with tile structure (synth
    sparse_attention_qkv), inputs resident, L2 flushed between steps."""
    import diffusion_transformer_image_nvfp4_b200 as kl
    from synth import sparse_attention_qkv

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    T, H = 4608, 24
    D = H * 128
    qkv = sparse_attention_qkv(T, H, seed=5).to(dev)
    amax = qkv.float().abs().view(T, 3, H, 128).amax(dim=(0, 3)).reshape(-1).contiguous()
    x8, sc = kl.cast_fp8_per_head(qkv, amax)
    q, k, v = x8, x8[:, D:], x8[:, 2 * D:]
    scales = dict(sq=sc[:H], sk=sc[H:2 * H], sv=sc[2 * H:])
    out = torch.empty((T, D), dtype=torch.bfloat16, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    lst = kl.sol_select(q, k, T, H, 3 * D, args.sol, "fp8", sq=scales["sq"], sk=scales["sk"])
    ws_sol = torch.empty(kl.lib().kl_sol_workspace_size(T, H, kl.ATTN["fp8"]), dtype=torch.uint8, device=dev)

    def select_step():
        kl._check(kl.lib().kl_sol_select(q.data_ptr(), k.data_ptr(), 3 * D, scales["sq"].data_ptr(),
                                         scales["sk"].data_ptr(), T, H, kl.ATTN["fp8"], float(args.sol),
                                         lst.data_ptr(), ws_sol.data_ptr(), ws_sol.numel(), kl._stream()),
                  "kl_sol_select")

    def sparse_step():  # selection into the preallocated list, then attention over it
        select_step()
        kl.joint_attention_sparse(q, k, v, T, H, 3 * D, lst, "fp8", out=out, **scales)

    def dense_step():
        kl.joint_attention(q, k, v, T, H, 3 * D, "fp8", out=out, **scales)

    def timed(fn):
        # device time of one graph replay (no host launch gaps inside the events)
        fn()
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            fn()
        for _ in range(args.warmup):
            graph.replay()
        ms = []
        for _ in range(args.steps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            graph.replay()
            b.record()
            ms.append((a, b))
        torch.cuda.synchronize()
        return statistics.median([a.elapsed_time(b) for a, b in ms])

    sparse_step()
    torch.cuda.synchronize()
    nkt = -(-T // 128)
    kept = float(lst[:, :, 0].float().mean().item()) / nkt
    t_sparse, t_dense, t_select = timed(sparse_step), timed(dense_step), timed(select_step)
    flops_dense = 4.0 * T * T * H * 128
    print(json.dumps({"metric": "Sol-Attention device time (selection + sparse FP8 attention), 1024^2 T2I shape",
                      "value": round(t_sparse * 1000, 1), "unit": "us", "higher_is_better": False,
                      "dense_us": round(t_dense * 1000, 1), "speedup": round(t_dense / t_sparse, 3),
                      "selection_us": round(t_select * 1000, 1),
                      "kept_tile_fraction": round(kept, 4), "tau": args.sol,
                      "kept_work_tflops": round(flops_dense * kept / (t_sparse * 1e-3) / 1e12, 1),
                      "config": {"workload": "sol_attention_t2i_1024", "tokens": T, "heads": H, "query_block": 256,
                                 "key_tile": 128, "inputs": "synth.sparse_attention_qkv(seed 5)",
                                 "launch": "each leg captured in a CUDA graph, replayed per step",
                                 "l2": "flushed between timed steps (256 MiB write, outside the timed events)"},
                      "steps": args.steps, "warmup": args.warmup, "device_status": kl.device_status()}), flush=True)


def run_vc(args):
    """VC-Attention repair at the 1024^2 T2I attention shape (4,608 tokens, 24
    heads, FP8): device time of the selection + FP8 pass + BF16 pass over the
    repaired pairs + merge, against dense FP8 attention, on seeded inputs with
    tile structure (synth sparse_attention_qkv), inputs resident, L2 flushed
    between steps."""
    import diffusion_transformer_image_nvfp4_b200 as kl
    from synth import sparse_attention_qkv

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    T, H = 4608, 24
    D = H * 128
    qkv = sparse_attention_qkv(T, H, seed=5).to(dev)
    amax = qkv.float().abs().view(T, 3, H, 128).amax(dim=(0, 3)).reshape(-1).contiguous()
    x8, sc = kl.cast_fp8_per_head(qkv, amax)
    q8, k8, v8 = x8, x8[:, D:], x8[:, 2 * D:]
    scales = dict(sq=sc[:H], sk=sc[H:2 * H], sv=sc[2 * H:])
    out = torch.empty((T, D), dtype=torch.bfloat16, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    l8, l16 = kl.vc_select(qkv, qkv[:, D:], T, H, 3 * D, args.vc)

    def vc_step():
        kl.vc_select(qkv, qkv[:, D:], T, H, 3 * D, args.vc)
        kl.joint_attention_vc(q8, k8, v8, 3 * D, scales["sq"], scales["sk"], scales["sv"], qkv, qkv[:, D:],
                              qkv[:, 2 * D:], 3 * D, T, H, l8, l16, out=out)

    def dense_step():
        kl.joint_attention(q8, k8, v8, T, H, 3 * D, "fp8", out=out, **scales)

    def timed(fn):
        fn()
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            fn()
        for _ in range(args.warmup):
            graph.replay()
        ms = []
        for _ in range(args.steps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            graph.replay()
            b.record()
            ms.append((a, b))
        torch.cuda.synchronize()
        return statistics.median([a.elapsed_time(b) for a, b in ms])

    t_vc, t_dense = timed(vc_step), timed(dense_step)
    repaired = int((l16[:, 0::2, 0] if l16.shape[1] > 1 else l16[:, :, 0]).sum().item())
    print(json.dumps({"metric": "VC-Attention device time (selection + FP8 pass + repaired BF16 pass + merge), "
                                "1024^2 T2I shape", "value": round(t_vc * 1000, 1), "unit": "us",
                      "higher_is_better": False, "dense_fp8_us": round(t_dense * 1000, 1),
                      "overhead": round(t_vc / t_dense, 3), "budget": args.vc, "repaired_pairs": repaired,
                      "pairs": int(H * l8.shape[1] * (l8.shape[2] - 1)),
                      "config": {"workload": "vc_attention_t2i_1024", "tokens": T, "heads": H, "query_block": 256,
                                 "key_tile": 128, "inputs": "synth.sparse_attention_qkv(seed 5)",
                                 "launch": "each leg captured in a CUDA graph, replayed per step",
                                 "l2": "flushed between timed steps (256 MiB write, outside the timed events)"},
                      "steps": args.steps, "warmup": args.warmup, "device_status": kl.device_status()}), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default="t2i_1024", choices=sorted(WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-secondary", action="store_true", help="skip the secondary workloads' lines (profiling runs)")
    ap.add_argument("--dit", action="store_true", help="time the synthetic DiT loop instead (one JSON line)")
    ap.add_argument("--shift", type=float, default=1.0, help="--dit: flow-matching time shift (1: linear)")
    ap.add_argument("--cache", type=float, default=None,
                    help="--dit: Cache-DiT residual-difference threshold (e.g. 0.24); default off")
    ap.add_argument("--sol", type=float, default=None,
                    help="time Sol-Attention (selection + sparse attention) at this tau against dense attention")
    ap.add_argument("--vc", type=float, default=None,
                    help="time VC-Attention repair (selection + both passes + merge) at this budget against dense")
    ap.add_argument("--sol-tau", type=float, default=0.0, help="--dit: Sol-Attention tau for every block (0: dense)")
    ap.add_argument("--sol-dense-steps", type=int, default=0, help="--dit: the first N steps stay dense")
    ap.add_argument("--mods", choices=("independent", "smooth"), default="independent",
                    help="--dit: modulations drawn per step, or smooth in t (m0 + t m1)")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    wl = WORKLOADS[args.workload]
    if args.dit:
        run_dit(args)
        return
    if args.sol is not None:
        run_sol(args)
        return
    if args.vc is not None:
        run_vc(args)
        return
    if args.impl == "reference":
        run_reference(args, wl)
    else:
        run_ours(args, wl)


if __name__ == "__main__":
    main()
