"""Benchmark of the CCA / CCGQA prefill block on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

One step = one pass of the whole block (down-projection, preprocessing,
attention, output projection) over one batch of synthetic input, through the
C ABI. Default workload: the CCGQA long prefill (B=1, S=16384, E=2048, C=4,
4 query heads x 128, 2 KV heads, seq-conv kernel 4), the configuration the
headline metric is quoted on. With N ranks (torchrun) every rank runs its own
independent sequence batch (weak scaling, no data-path collective); the
timing is the max over ranks.

Prints one JSON line (rank 0). `--impl reference` times the float64 CPU
oracle instead, on bounded samples of the same workload.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import tempfile
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "CCA prefill tokens/s and attention TFLOP/s (% bf16 peak) at S=16k, 1 B200"
DEFAULT_WORKLOAD = "ccgqa_16k_bf16"
DATASHEET_BF16_TFLOPS = 2250.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20
E2E_LANES = 3  # requests in flight in the end-to-end timing (streams with their own buffers)
ATTN_KERNEL_SRC = os.path.join(ROOT, "compressed_latent_space_cca_b200", "csrc", "attn_tc.cu")


# ------------------------------------------------------------ host logic --
def rank_workload(shape: workloads.BlockShape, rank: int) -> workloads.BlockShape:
    """Weak scaling: each rank owns an independent batch of the same shape,
    drawn with its own seed."""
    return shape.replace(seed=shape.seed + 1000 * rank)


def aggregate(elapsed_ms: float, tokens_per_rank: int, steps: int, world: int, reduce_max=None):
    """Whole-job throughput from this rank's timed region: the max elapsed
    time over ranks covers every rank's tokens."""
    t = elapsed_ms
    if reduce_max is not None:
        t = reduce_max(t)
    ms_per_step = t / steps
    value = tokens_per_rank * world / (ms_per_step / 1e3)
    return value, ms_per_step


def algorithmic_work(shape: workloads.BlockShape):
    B, S, E = shape.batch, shape.seq_len, shape.hidden
    T = B * S
    Lq, Lkv, d = shape.latent_q, shape.latent_kv, shape.head_dim
    Nlat = Lq + 2 * Lkv
    eb = 2 if shape.dtype == "bf16" else 4
    # bf16 blocks also write fp16 copies of k and v for the attention and an fp16 copy of W_o: bytes
    # this design moves beyond the method's own
    extra = (2 * T * Lkv * 2 + 2 * E * Lq * 2) if shape.dtype == "bf16" else 0
    return {
        "down_proj_flops": 2.0 * T * E * Nlat,
        "attention_flops": 2.0 * B * shape.n_q_heads * S * S * d,   # causal half, 2 GEMMs
        "out_proj_flops": 2.0 * T * Lq * E,
        # algorithmic: read q~k~v~, write q and the K/V cache (the roofline's bytes)
        "preproc_bytes": float(T * (Nlat + Lq + 2 * Lkv) * eb),
        # moved by this design: plus the fp16 attention copies of k and v and the W_o copy
        "preproc_bytes_moved": float(T * (Nlat + Lq + 2 * Lkv) * eb + extra),
    }


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def file_sha(path):
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def traffic_record(workload):
    """DRAM bytes per attention launch from the committed ncu summary, valid only
    for the workload it was captured on and while the kernel source is unchanged
    since the counters were taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p) or not os.path.exists(ATTN_KERNEL_SRC):
        return None
    with open(p) as f:
        rec = json.load(f)
    if rec.get("source_sha") != file_sha(ATTN_KERNEL_SRC) or rec.get("workload") != workload:
        return None
    return rec


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during timing."""

    FIELDS = ["clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, index: int, device_id: str = None):
        self.index = index
        # nvidia-smi numbers GPUs without regard to CUDA_VISIBLE_DEVICES, so the sampled GPU is named
        # by the UUID of the CUDA device when it is known
        self.device_id = device_id or str(index)
        self.proc = None
        # the raw samples: $CCA_BENCH_CLOCKS_DIR if set, else the system temporary directory
        d = os.environ.get("CCA_BENCH_CLOCKS_DIR") or tempfile.gettempdir()
        self.path = os.path.join(d, f"cca_bench_clocks_rank{index}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.device_id}", "--query-gpu=" + ",".join(self.FIELDS),
                 "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.fh, stderr=subprocess.DEVNULL)
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
        self.fh.close()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < len(self.FIELDS):
                    continue
                try:
                    sm.append(float(parts[0]))
                    mx = float(parts[1])
                except ValueError:
                    continue
                for n, v in zip(names, parts[4:8]):
                    if v.lower() == "active":
                        reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "gpu": self.device_id}


def cuda_device_uuid(dev) -> str:
    """nvidia-smi's name for the CUDA device ("GPU-<uuid>"), or None if torch does not report it."""
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        return None
    if not u:
        return None
    return u if u.startswith("GPU-") else "GPU-" + u


# ---------------------------------------------------------- oracle timing --
def oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [p.get("num_threads", 0) for p in threadpool_info() if p.get("user_api") == "blas"]
        if n:
            return max(n)
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def oracle_call(shape, inp64, rows):
    import oracle
    t0 = time.perf_counter()
    oracle.cca_block(inp64, shape.n_q_heads, shape.n_kv_heads, shape.head_dim, qk_mean_mode=shape.qk_mean_mode,
                     use_value_shift=bool(shape.value_shift), use_rope=bool(shape.use_rope),
                     rope_base=shape.rope_base, softmax_scale=shape.softmax_scale, rows=rows)
    return time.perf_counter() - t0


ROW_SAMPLES = (2048, 16384)  # at S = 16384 the second sample is the whole block


def spaced_rows(S, n):
    return np.unique(np.linspace(0, S - 1, n).round().astype(np.int64))


def oracle_extrapolated(shape):
    return len(spaced_rows(shape.seq_len, ROW_SAMPLES[1])) < shape.seq_len


def oracle_sample_text(shape):
    text = (f"oracle (numpy float64) on the {shape.name} inputs: every per-token stage over all "
            f"{shape.tokens} tokens, attention and output projection for {ROW_SAMPLES[0]} and "
            f"{ROW_SAMPLES[1]} evenly spaced query rows per sequence")
    if oracle_extrapolated(shape):
        return text + "; full-block time extrapolated linearly in the number of query rows"
    return text + " (the second sample is the whole block, whose time is reported)"


def oracle_extrapolate(times_by_rows, S):
    """Full-block time from two row counts (linear in the rows evaluated). When the
    sequence is shorter than the samples both calls already ran the full block."""
    (r1, t1), (r2, t2) = times_by_rows
    if r2 <= r1:
        return 0.5 * (t1 + t2)
    per_row = max(0.0, (t2 - t1) / (r2 - r1))
    return t1 + per_row * (S - r1)


def cpu_baseline(shape, inputs, repeats=2):
    inp64 = workloads.as_float64(inputs)
    pts = []
    for r in ROW_SAMPLES:
        rows = spaced_rows(shape.seq_len, r)
        t = min(oracle_call(shape, inp64, rows) for _ in range(repeats))
        pts.append((len(rows), t))
    t_full = oracle_extrapolate(pts, shape.seq_len)
    return {"value": shape.tokens / t_full, "unit": "tokens/s", "cores": oracle_threads(), "kind": "oracle",
            "sample": oracle_sample_text(shape), "extrapolated": oracle_extrapolated(shape),
            "sample_seconds": round(repeats * sum(t for _, t in pts), 2)}


REF_MAX_ROWS = 16384  # query rows of one reference step; at S <= 16384 a step is the whole block


def run_reference(args, shape):
    """The oracle as the reference arm: every step (warm-up and timed) is one oracle call on the
    same inputs. At S <= 16384 the call is the whole block, so `ms_per_step` is the block's time.
    Longer sequences run every per-token stage over all S tokens and attention and the output
    projection for 16384 evenly spaced query rows; the whole-block time is then extrapolated
    linearly in rows from one more call of 2048 rows (made after the timed steps) and labelled."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    inputs = workloads.make_inputs(shape)
    inp64 = workloads.as_float64(inputs)
    rows = spaced_rows(shape.seq_len, min(shape.seq_len, REF_MAX_ROWS))
    full = len(rows) == shape.seq_len
    times = []
    for i in range(args.warmup + args.steps):
        t = oracle_call(shape, inp64, None if full else rows)
        if i >= args.warmup:
            times.append(t)
    t_step = statistics.mean(times)
    if full:
        t_full = t_step
        sample = (f"oracle (numpy float64) on the {shape.name} inputs: the whole block, all "
                  f"{shape.tokens} tokens, every step")
    else:
        small = spaced_rows(shape.seq_len, ROW_SAMPLES[0])
        t_small = oracle_call(shape, inp64, small)
        t_full = oracle_extrapolate([(len(small), t_small), (len(rows), t_step)], shape.seq_len)
        sample = (f"oracle (numpy float64) on the {shape.name} inputs: every per-token stage over all "
                  f"{shape.tokens} tokens, attention and output projection for {len(rows)} evenly spaced query "
                  f"rows per step; the whole-block time extrapolated linearly in rows (one more call of "
                  f"{len(small)} rows)")
    value = shape.tokens / t_full
    cores = oracle_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_step * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_dict(shape), "path": "oracle",
        "full_block_ms": t_full * 1e3, "full_block_extrapolated": not full,
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": sample, "extrapolated": not full},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_dict(shape):
    """The workload, identical in both arms (the kernels that ran are the line's `path`)."""
    return {"workload": shape.name, "batch": shape.batch, "seq_len": shape.seq_len, "hidden": shape.hidden,
            "C": shape.compression, "n_q_heads": shape.n_q_heads, "n_kv_heads": shape.n_kv_heads,
            "head_dim": shape.head_dim, "conv_kernel": shape.conv_kernel, "qk_mean_mode": shape.qk_mean_mode,
            "value_shift": shape.value_shift, "rope_base": shape.rope_base,
            "l2": "flushed between timed steps (256 MiB write)"}


# ----------------------------------------------------------------- ours --
def run_ours(args, shape):
    import torch.distributed as dist

    import compressed_latent_space_cca_b200 as cca

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    my_shape = rank_workload(shape, rank)
    inputs_cpu = workloads.make_inputs(my_shape)
    cfg = cca.config_from_shape(my_shape)
    inputs = {k: v.to(dev) for k, v in inputs_cpu.items()}
    out = cca.alloc_outputs(cfg, dev)
    ws = cca.alloc_workspace(cfg, dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def barrier():
        if world > 1:
            dist.barrier()

    def reduce_max(v):
        if world == 1:
            return v
        t = torch.tensor([v], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    # which kernels run (tcgen05 or SIMT per stage) and how many launches a step makes
    path = PREPROC_PATHS[args.preproc]
    plan = cca.plan(cfg, path)
    if args.decode_only:
        # one prefill writes the cache, then only the decode step is timed (profiling runs)
        cca.prefill(cfg, inputs, out=out, workspace=ws, path=path)
        torch.cuda.synchronize()
        if rank == 0:
            res = run_decode(cca, dev, my_shape, inputs, out, load_peaks()[0], steps=args.steps,
                             warmup=args.warmup)
            print(json.dumps({"mode": "decode-only", "workload": my_shape.name, "decode": res}, default=float),
                  flush=True)
        if world > 1:
            dist.destroy_process_group()
        return 0
    if args.backward_only:
        # only the backward pass (cca_backward) is timed (profiling runs)
        if rank == 0:
            res = run_backward(cca, dev, my_shape, inputs, load_peaks()[0], steps=args.steps, warmup=args.warmup)
            print(json.dumps({"mode": "backward-only", "workload": my_shape.name, "backward": res}, default=float),
                  flush=True)
        if world > 1:
            dist.destroy_process_group()
        return 0
    path_tensor = plan["attention_tensor"]
    launches_per_step = plan["launches"]

    for _ in range(args.warmup):
        flush.zero_()
        cca.prefill(cfg, inputs, out=out, workspace=ws, path=path)
    torch.cuda.synchronize()
    st = cca.poll_device_status()
    if st != 0:
        raise SystemExit(f"device status {st} after warm-up")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    sampler = ClockSampler(local, cuda_device_uuid(dev))
    sampler.start()
    time.sleep(0.3)
    barrier()
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.zero_()
        cca.prefill(cfg, inputs, out=out, workspace=ws, stage_events=evs[i], path=path)
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop()
    st = cca.poll_device_status()
    if st != 0:
        raise SystemExit(f"device status {st} after timing")

    stage = np.array([[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(4)] for i in range(args.steps)])
    elapsed = float(stage.sum())
    value, ms_per_step = aggregate(elapsed, my_shape.tokens, args.steps, world, reduce_max)
    stage_ms = stage.mean(axis=0)
    work = algorithmic_work(my_shape)

    # end to end: x from pinned host memory, y back to pinned host memory, one C call per step
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(cca, cfg, args, inputs_cpu, inputs, out, ws, stream, my_shape, world, barrier, reduce_max)

    peaks, peak_src = load_peaks()
    attn_s = stage_ms[2] / 1e3
    attn_tflops = work["attention_flops"] / attn_s / 1e12
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    traffic = traffic_record(args.workload)
    roofline = {
        "kernel": "attention (tcgen05)" if path_tensor else "attention (SIMT)",
        "bound": "tensor", "achieved": attn_tflops, "peak": peak, "unit": "TFLOP/s",
        "frac": attn_tflops / peak, "peak_source": f"{peak_src} bf16 (burst)",
        "frac_of_datasheet_2250": attn_tflops / DATASHEET_BF16_TFLOPS,
        "traffic": traffic["dram_bytes_per_launch"] if traffic else None,
        "algorithmic_flops_per_launch": work["attention_flops"],
    }
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    kernels = {
        "down_proj": {"ms": stage_ms[0], "tflops": work["down_proj_flops"] / (stage_ms[0] / 1e3) / 1e12,
                      "frac": work["down_proj_flops"] / (stage_ms[0] / 1e3) / 1e12 / peak},
        "preproc": {"ms": stage_ms[1], "gbs": work["preproc_bytes"] / (stage_ms[1] / 1e3) / 1e9,
                    "frac": work["preproc_bytes"] / (stage_ms[1] / 1e3) / 1e9 / hbm,
                    "bytes_algorithmic": work["preproc_bytes"], "bytes_moved": work["preproc_bytes_moved"],
                    "gbs_moved": work["preproc_bytes_moved"] / (stage_ms[1] / 1e3) / 1e9},
        "attention": {"ms": stage_ms[2], "tflops": attn_tflops, "frac": attn_tflops / peak},
        "out_proj": {"ms": stage_ms[3], "tflops": work["out_proj_flops"] / (stage_ms[3] / 1e3) / 1e12,
                     "frac": work["out_proj_flops"] / (stage_ms[3] / 1e3) / 1e12 / peak},
    }
    line = None
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": config_dict(shape), "path": plan_name(plan),
            "attention_tflops": attn_tflops,
            "roofline": roofline,
            "kernels": kernels,
            "e2e": e2e,
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clocks,
        }
        if world == 1 and not args.no_backward and cca.backward_workspace_size(cfg) > 0:
            line["backward"] = run_backward(cca, dev, my_shape, inputs, peaks)
        if (world == 1 and not args.no_mha and my_shape.dtype == "bf16" and my_shape.conv_kernel > 0 and
                my_shape.hidden % 128 == 0):
            line["mha_baseline"] = run_mha_baseline(cca, dev, my_shape, ms_per_step, line.get("backward"), peaks)
        if world == 1 and not args.no_decode and cca.decode_workspace_size(cfg) > 0:
            line["decode"] = run_decode(cca, dev, my_shape, inputs, out, peaks)
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(my_shape, inputs_cpu)
        print(json.dumps(line, default=float), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def mha_shape(shape: workloads.BlockShape) -> workloads.BlockShape:
    """The uncompressed baseline of a block: plain multi-head attention (C = 1, heads of 128, no
    convolutions, QK-mean or value shift) with the same batch, sequence length and width."""
    base = workloads.WORKLOADS["mha_16k_bf16"]
    nh = shape.hidden // base.head_dim
    return base.replace(name=f"mha_b{shape.batch}_s{shape.seq_len}_e{shape.hidden}", batch=shape.batch,
                        seq_len=shape.seq_len, hidden=shape.hidden, n_q_heads=nh, n_kv_heads=nh)


def run_mha_baseline(cca, dev, shape, cca_ms_per_step, cca_backward=None, peaks=None, steps=10, warmup=3):
    """Times the plain multi-head block of the same shape with the same method (L2 flushed between
    steps, CUDA events around each stage) and returns its numbers and the CCA block's speedup; with
    the CCA block's backward timing given, the MHA block's backward too."""
    mshape = mha_shape(shape)
    cfg = cca.config_from_shape(mshape)
    inputs = {k: v.to(dev) for k, v in workloads.make_inputs(mshape).items()}
    out = cca.alloc_outputs(cfg, dev)
    ws = cca.alloc_workspace(cfg, dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    for _ in range(warmup):
        flush.zero_()
        cca.prefill(cfg, inputs, out=out, workspace=ws)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(steps)]
    torch.cuda.synchronize()
    for i in range(steps):
        flush.zero_()
        cca.prefill(cfg, inputs, out=out, workspace=ws, stage_events=evs[i])
    torch.cuda.synchronize()
    if cca.poll_device_status() != 0:
        raise SystemExit("device status error in the MHA baseline")
    stage = np.array([[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(4)] for i in range(steps)])
    ms = float(stage.sum(axis=1).mean())
    stage_ms = stage.mean(axis=0)
    work = algorithmic_work(mshape)
    del out, ws, flush
    torch.cuda.empty_cache()
    bwd = None
    if cca_backward is not None and cca.backward_workspace_size(cfg) > 0:
        bwd = run_backward(cca, dev, mshape, inputs, peaks if peaks is not None else load_peaks()[0])
        bwd["cca_backward_speedup"] = bwd["ms_per_step"] / cca_backward["ms_per_step"]
        if bwd.get("saved_forward") and cca_backward.get("saved_forward"):
            bwd["saved_forward"]["cca_backward_speedup"] = (bwd["saved_forward"]["ms_per_step"] /
                                                            cca_backward["saved_forward"]["ms_per_step"])
    del inputs
    torch.cuda.empty_cache()
    return {
        "workload": mshape.name, "n_q_heads": mshape.n_q_heads, "n_kv_heads": mshape.n_kv_heads,
        "head_dim": mshape.head_dim, "C": mshape.compression, "steps": steps, "warmup": warmup,
        "ms_per_step": ms, "tokens_per_s": mshape.tokens / (ms / 1e3),
        "attention_tflops": work["attention_flops"] / (stage_ms[2] / 1e3) / 1e12,
        "kernels_ms": {"down_proj": stage_ms[0], "rope_cache": stage_ms[1], "attention": stage_ms[2],
                       "out_proj": stage_ms[3]},
        "cca_speedup": ms / cca_ms_per_step,
        "backward": bwd,
    }


def backward_flops(shape: workloads.BlockShape):
    """Algorithmic FLOPs of cca_backward: the forward it recomputes, then per projection two GEMMs of
    the forward's size (the input and the weight gradients) and, for the causal attention, five
    products of the forward's QK^T size (S and dP recomputed, dV, dK, dQ)."""
    w = algorithmic_work(shape)
    fwd = w["down_proj_flops"] + w["attention_flops"] + w["out_proj_flops"]
    attn_bwd = 2.5 * w["attention_flops"]
    gemm_bwd = 2.0 * (w["down_proj_flops"] + w["out_proj_flops"])
    return {"forward": fwd, "attention_backward": attn_bwd, "projections_backward": gemm_bwd,
            "total": fwd + attn_bwd + gemm_bwd}


def run_backward(cca, dev, shape, inputs, peaks, steps=5, warmup=3):
    """cca_backward (the forward recomputed, then every gradient) at the workload, dL/dy seeded,
    timed with CUDA events around each call with L2 flushed before it."""
    cfg = cca.config_from_shape(shape)
    dy = workloads.make_dy(shape).to(dev)
    ws = torch.empty(cca.backward_workspace_size(cfg), dtype=torch.uint8, device=dev)
    grads = {n: torch.empty(tuple(inputs[n].shape), dtype=torch.float32, device=dev)
             for n in cca.GRAD_NAMES if n in inputs}  # a plain block has no conv weights
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    for _ in range(warmup):
        flush.zero_()
        cca.backward(cfg, inputs, dy, grads=grads, workspace=ws)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream(dev)
    for i in range(steps):
        flush.zero_()
        evs[i][0].record(stream)
        cca.backward(cfg, inputs, dy, grads=grads, workspace=ws)
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    if cca.poll_device_status() != 0:
        raise SystemExit("device status error in the backward timing")
    ms = float(np.mean([a.elapsed_time(b) for a, b in evs]))
    fl = backward_flops(shape)
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    tflops = fl["total"] / (ms / 1e3) / 1e12
    # the backward of a training step whose forward (prefill_train) kept its activations: no recompute
    saved = None
    try:
        cca.prefill_train(cfg, inputs, workspace=ws)
    except cca.CcaError:
        pass  # a block the saved forward does not take (fp32, CUDA-core attention)
    else:
        for _ in range(warmup):
            flush.zero_()
            cca.backward(cfg, inputs, dy, grads=grads, workspace=ws, saved=True)
        torch.cuda.synchronize()
        for i in range(steps):
            flush.zero_()
            evs[i][0].record(stream)
            cca.backward(cfg, inputs, dy, grads=grads, workspace=ws, saved=True)
            evs[i][1].record(stream)
        torch.cuda.synchronize()
        if cca.poll_device_status() != 0:
            raise SystemExit("device status error in the saved-forward backward timing")
        sms = float(np.mean([a.elapsed_time(b) for a, b in evs]))
        sfl = fl["attention_backward"] + fl["projections_backward"]
        saved = {"ms_per_step": sms, "includes": "all gradients from prefill_train's saved activations",
                 "flops": sfl, "tflops": sfl / (sms / 1e3) / 1e12,
                 "frac_of_bf16_peak": sfl / (sms / 1e3) / 1e12 / peak}
    del ws, grads, flush, dy
    torch.cuda.empty_cache()
    return {"ms_per_step": ms, "tokens_per_s": shape.tokens / (ms / 1e3), "steps": steps, "warmup": warmup,
            "includes": "forward recompute + all gradients", "flops": fl, "tflops": tflops,
            "frac_of_bf16_peak": tflops / peak, "timing": "CUDA events, L2 flushed before each call",
            "saved_forward": saved}


def decode_bytes(shape: workloads.BlockShape, t: int) -> float:
    """Bytes one decode step must move at position t: every weight once, the cache rows 0..t-1
    read and row t written, the conv state read and written, x_t read and y_t written."""
    B, E, d, K = shape.batch, shape.hidden, shape.head_dim, shape.conv_kernel
    Lq, Lkv = shape.latent_q, shape.latent_kv
    eb = 2 if shape.dtype == "bf16" else 4
    w = (Lq + 2 * Lkv) * E + E * Lq + (Lq + Lkv) * K + (shape.n_q_heads + shape.n_kv_heads) * d * d * (K > 0)
    state = (K - 1) * (Lq + Lkv) + Lkv if K > 0 else 0
    per_seq = 2 * (t + 1) * Lkv + 2 * state + 2 * E
    return float((w + B * per_seq) * eb)


def run_decode(cca, dev, shape, inputs, out, peaks, steps=50, warmup=5):
    """One decode step (cca_decode) at the last position of the workload, t = S - 1, reading the
    cache the timed prefill wrote. The step is captured once in a CUDA graph, as a serving loop
    runs it, and each replay is timed with CUDA events, L2 flushed before each. The host cost of
    one direct call (argument checks, four launches) is reported on its own."""
    t = shape.seq_len - 1
    cfg = cca.config_from_shape(shape)  # seq_len = t + 1
    B = shape.batch
    weights = {k: v for k, v in inputs.items() if k != "x"}
    x_t = inputs["x"][:, t].contiguous()
    K = shape.conv_kernel
    cs = None
    if K > 0:
        n = (K - 1) * (shape.latent_q + shape.latent_kv) + shape.latent_kv
        cs = torch.zeros((B, n), dtype=out["k_cache"].dtype, device=dev)
    y = torch.empty((B, shape.hidden), dtype=out["y"].dtype, device=dev)
    ws = torch.empty(cca.decode_workspace_size(cfg), dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def step(stream=None):
        cca.decode(cfg, x_t, weights, out["k_cache"], out["v_cache"], cs, y=y, workspace=ws, stream=stream)

    side = torch.cuda.Stream(device=dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):
        for _ in range(warmup):
            step()
    torch.cuda.current_stream(dev).wait_stream(side)
    torch.cuda.synchronize()
    # host cost of a direct call: wall clock over calls queued behind one long flush
    flush.zero_()
    h0 = time.perf_counter()
    for _ in range(20):
        step()
    host_us = (time.perf_counter() - h0) / 20 * 1e6
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    stream = torch.cuda.current_stream(dev)
    for _ in range(warmup):
        flush.zero_()
        graph.replay()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    torch.cuda.synchronize()
    for i in range(steps):
        flush.zero_()
        evs[i][0].record(stream)
        graph.replay()
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    if cca.poll_device_status() != 0:
        raise SystemExit("device status error in the decode timing")
    del graph
    us = np.array([a.elapsed_time(b) * 1e3 for a, b in evs])
    nbytes = decode_bytes(shape, t)
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    mean_us = float(us.mean())
    gemv_launches = 2 * ((B + 7) // 8)
    return {
        "position": t, "batch": B, "steps": steps, "warmup": warmup, "us_per_step": mean_us,
        "us_median": float(np.median(us)), "tokens_per_s": B / (mean_us / 1e6),
        "bytes_per_step": nbytes, "gbs": nbytes / (mean_us / 1e6) / 1e9,
        "frac_hbm": nbytes / (mean_us / 1e6) / 1e9 / hbm, "timing": "CUDA graph replay",
        "host_us_per_call": host_us, "launches_per_step": gemv_launches + 1 + (K > 0),
        "l2": "flushed before each step (256 MiB write)",
    }


def run_e2e(cca, cfg, args, inputs_cpu, inputs, out, ws, stream, shape, world, barrier, reduce_max):
    """Same metric through cca_prefill_host: every step copies its x from pinned host memory
    and its y back to pinned host memory inside the timed region (the KV cache stays on the
    device). Steps rotate over E2E_LANES streams, each with its own device buffers, so the copies
    of one step overlap the kernels and copies of the others, as a serving loop with that many
    requests in flight would run them: with three, the host-to-device copy engine no longer waits
    for a lane's device-to-host copy before the next input can start."""
    dev = inputs["x"].device
    x_host = inputs_cpu["x"].pin_memory()
    weights = {k: v for k, v in inputs.items() if k != "x"}
    lanes = []
    for i in range(E2E_LANES):
        o = cca.alloc_outputs(cfg, dev) if i else out
        lanes.append({
            "stream": torch.cuda.Stream(device=dev) if i else stream,
            "x_dev": torch.empty_like(inputs["x"]),
            "y_host": torch.empty(tuple(out["y"].shape), dtype=out["y"].dtype).pin_memory(),
            "out": o,
            "ws": cca.alloc_workspace(cfg, dev) if i else ws,
        })

    def step(i):
        ln = lanes[i % E2E_LANES]
        o = ln["out"]
        cca.prefill_host(cfg, x_host, weights, ln["x_dev"], o["y"], ln["y_host"], o["k_cache"], o["v_cache"],
                         ln["ws"], stream=ln["stream"])

    steps = max(2 * E2E_LANES, min(args.steps, 21))
    for i in range(E2E_LANES):
        step(i)
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for ln in lanes[1:]:
        ln["stream"].wait_event(e0)
    for i in range(steps):
        step(i)
    for ln in lanes[1:]:
        done = torch.cuda.Event()
        done.record(ln["stream"])
        stream.wait_event(done)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    value, _ = aggregate(e0.elapsed_time(e1), shape.tokens, steps, world, reduce_max)
    return {"value": value, "unit": "tokens/s", "steps": steps, "streams": E2E_LANES,
            "h2d_bytes_per_step": int(x_host.numel() * x_host.element_size()),
            "d2h_bytes_per_step": int(lanes[0]["y_host"].numel() * lanes[0]["y_host"].element_size())}


def plan_name(plan):
    k = lambda b: "tcgen05" if b else "simt"  # noqa: E731
    return (f"down_proj={k(plan['down_proj_tensor'])},"
            f"preproc={plan['preproc_kind']},attention={k(plan['attention_tensor'])},"
            f"out_proj={k(plan['out_proj_tensor'])}" + (",value_shift=down_proj_epilogue" if plan.get("value_shift_fused")
                                                          else ""))


# --preproc: which preprocessing kernel the timed block runs (the other stages on their tensor-core
# kernels where the shape allows them)
PREPROC_PATHS = {"auto": 0, "mma": 0x100 | 1 | 2 | 4 | 8, "tcgen05": 0x100 | 1 | 2 | 4 | 16,
                 "tcgen05+vshift": 0x100 | 1 | 2 | 4 | 16 | 32}


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the oracle timing (rank 0, N=1)")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end timing")
    ap.add_argument("--no-mha", action="store_true",
                    help="skip timing the plain multi-head block of the same shape (the uncompressed baseline)")
    ap.add_argument("--no-decode", action="store_true", help="skip timing one decode step at position S - 1")
    ap.add_argument("--no-backward", action="store_true", help="skip timing the backward pass (cca_backward)")
    ap.add_argument("--backward-only", action="store_true",
                    help="time only cca_backward at the workload (for profiling)")
    ap.add_argument("--decode-only", action="store_true",
                    help="time only the decode step at position S - 1 after one prefill (profiling runs)")
    ap.add_argument("--preproc", choices=sorted(PREPROC_PATHS), default="auto",
                    help="preprocessing kernel of the timed block (auto: the library's choice)")
    ap.add_argument("--batch", type=int, default=None, help="override the workload's batch (profiling cases)")
    ap.add_argument("--seq-len", type=int, default=None, help="override the workload's sequence length")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    shape = workloads.WORKLOADS[args.workload]
    if args.batch is not None or args.seq_len is not None:
        shape = shape.replace(batch=args.batch or shape.batch, seq_len=args.seq_len or shape.seq_len,
                              name=f"{shape.name}(B={args.batch or shape.batch},S={args.seq_len or shape.seq_len})")
    if args.impl == "reference":
        return run_reference(args, shape)
    return run_ours(args, shape)


if __name__ == "__main__":
    sys.exit(main())
