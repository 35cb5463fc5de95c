"""Benchmark: joint-attention TFLOPS on the 2048x2048 Base T2I workload.

One step = one pass of the whole hot path over one batch: jattn_rope_qkv_hp
(joint-sequence assembly + 2D axial RoPE, range scales, correction rows)
followed by jattn_fwd_bf16_hp -- the BF16 path that meets the BF16 error bars
--, with the plain fp16-operand pair, the e4m3 pair and the next-row paths
reported beside it.  TFLOPS = 4 * B * H * S^2 * d / step time.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With one GPU the whole batch runs on it.  Under torchrun (N > 1) the batch is
partitioned the way the multi-GPU mode of the page does it: the two
classifier-free-guidance branches (batch entries) on separate rank groups,
each branch's sequence over the ranks of its group with Ulysses sequence
parallelism (two NCCL all-to-alls around the unchanged device path).  The
total work is fixed (strong scaling); the step time is the max over ranks.
``--impl reference`` times the FP64 oracle on the host cores instead (rank 0
only), on bounded samples of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from diffusion_transformer_joint_jattn_b200 import workloads as W  # noqa: E402

WORKLOAD = "t2i_2048_base"
# DRAM bytes per launch of the forward kernels on t2i_2048_base: the ncu
# captures of the same kernels on t2i_1024_base (dram__bytes_read.sum +
# dram__bytes_write.sum: 170.01 + 39.44 MB with fp16 operands, 85.07 + 28.12
# MB with e4m3 operands, 184.22 + 38.92 MB for the high-precision instance,
# the headline's forward) scaled by the token count 16896 / 4608 (the
# traffic is Q, K, V and O once each, linear in tokens).
FWD_TRAFFIC_BYTES = (170.01e6 + 39.44e6) * 16896 / 4608
FWD_FP8_TRAFFIC_BYTES = (85.07e6 + 28.12e6) * 16896 / 4608
FWD_HP_TRAFFIC_BYTES = (184.22e6 + 38.92e6) * 16896 / 4608
METRIC = "joint-attention TFLOPS and % of B200 tensor peak (BF16/FP8), 2048^2 shape"
UNIT = "TFLOPS"
# Per-sample time of the oracle on the host cores (both CPU legs use the same
# sample shape, so their rates agree).
ORACLE_SAMPLE_S = 6.0


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=WORKLOAD)
    ap.add_argument("--no-fp8", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the FP8-with-repair, query/key-norm prologue and other-workload measurements")
    ap.add_argument("--rho", type=float, default=0.005, help="token-repair budget of the FP8-with-repair block")
    ap.add_argument("--tau", type=float, default=1.0, help="sparsity of the block-sparse block (0 = dense)")
    return ap.parse_args(argv)


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def max_over_ranks(x: float, world: int, device) -> float:
    """Max of a per-rank scalar over all ranks (identity for one rank)."""
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(flops_total: int, ms_per_step: float) -> float:
    """Aggregate throughput: the whole batch's FLOPs over the slowest rank's
    step time."""
    return flops_total / ms_per_step / 1e9


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            pk = json.load(f)
        return pk, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (FileNotFoundError, OSError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, val in zip(names, f[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


def tensor_roofline(flops: int, fwd_ms: float, peaks, peak_src: str, fp8: bool, traffic, kernel: str):
    """Roofline of one forward launch: algorithmic FLOPs / its CUDA-event
    duration against the measured burst cuBLAS bf16 rate (the forward is a
    few-millisecond kernel timed in a sub-second region); FP8 against twice
    that (the nominal fp8 / bf16 ratio)."""
    mult = 2.0 if fp8 else 1.0
    achieved = flops / fwd_ms / 1e9
    peak = mult * peaks["bf16_tflops"]
    return {"bound": "tensor", "achieved": round(achieved, 2), "peak": round(peak, 1), "unit": "TFLOP/s",
            "frac": round(achieved / peak, 4),
            "peak_note": (f"{'2 x ' if fp8 else ''}{peak_src} cuBLAS bf16 burst (MEASURED_PEAKS.json bf16_tflops)"
                          + (", nominal fp8 / bf16 ratio" if fp8 else "")),
            "frac_of_sustained": round(achieved / (mult * peaks["bf16_tflops_sustained"]), 4),
            "frac_of_nominal": round(achieved / (4500.0 if fp8 else 2250.0), 4),
            "traffic": None if traffic is None else round(traffic),
            "traffic_note": "ncu capture on t2i_1024_base scaled by tokens (see profiles/)",
            "kernel": kernel}


def prologue_bytes(w, out_bytes: int) -> int:
    """Algorithmic bytes of one prologue call: read 3*B*S*H*d bf16, write the
    same count in the output type (+ scales, negligible)."""
    n = 3 * w.B * w.S * w.H * w.d
    return n * 2 + n * out_bytes


class Ctx:
    """What the timing helpers share: device, stream, world size, barrier."""

    def __init__(self, dev, world):
        self.dev = dev
        self.world = world
        self.stream = torch.cuda.current_stream()

    def barrier(self):
        if self.world > 1:
            import torch.distributed as dist
            dist.barrier()

    def max_ranks(self, x: float) -> float:
        return max_over_ranks(x, self.world, self.dev)


def time_calls(ctx: Ctx, fn, steps: int, warmup: int, marks: int = 0):
    """Run ``fn(ev)`` warmup times untimed, then ``steps`` times between two
    events on the stream; ``fn`` records ``marks`` inner events (``ev`` list)
    around the kernels it launches.  Returns (ms per call, per-call inner
    intervals [steps][marks-1] in ms), max over ranks."""
    for _ in range(warmup):
        fn(None)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(marks)] for _ in range(steps)]
    ctx.barrier()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(ctx.stream)
    for i in range(steps):
        fn(evs[i] if marks else None)
    t1.record(ctx.stream)
    torch.cuda.synchronize()
    ctx.barrier()
    inner = [[e[k].elapsed_time(e[k + 1]) for k in range(marks - 1)] for e in evs] if marks else []
    return ctx.max_ranks(t0.elapsed_time(t1) / steps), inner


def path_step(jattn, w, dinp, path: str, dev, stream):
    """Buffers and a step function for one whole-path step (prologue +
    forward) of workload w; the step records 3 events when given them."""
    B, H, S, d = w.B, w.H, w.S, w.d
    ws = None
    if path == "bf16":
        q = torch.empty(B, H, S, d, dtype=torch.float16, device=dev)
        bufs = (q, torch.empty_like(q), torch.empty_like(q), None)
    elif path == "bf16_hp":
        q = torch.empty(B, H, S, d, dtype=torch.float16, device=dev)
        bufs = (q, torch.empty_like(q), torch.empty_like(q),
                torch.empty(3, B, H, jattn.n_blocks(S), dtype=torch.float32, device=dev),
                torch.empty(B, H, S, jattn.CORR_COLS, dtype=torch.float16, device=dev),
                torch.empty(B, H, S, jattn.CORR_COLS, dtype=torch.float16, device=dev))
        ws = torch.empty(jattn.rope_qkv_hp_workspace_bytes(B, H, w.S_txt, w.S_img, w.S_ref, d), dtype=torch.uint8,
                         device=dev)
    else:
        q = torch.empty(B, H, S, d, dtype=torch.float8_e4m3fn, device=dev)
        bufs = (q, torch.empty_like(q), torch.empty_like(q),
                torch.empty(3, B, H, jattn.n_blocks(S), dtype=torch.float32, device=dev))
    o = torch.empty(B, S, H, d, dtype=torch.bfloat16, device=dev)

    def step(ev):
        if ev is not None:
            ev[0].record(stream)
        if path == "bf16_hp":
            jattn.rope_qkv_hp(dinp["qkv_txt"], dinp["qkv_img"], dinp["qkv_ref"], dinp["pos"], w.split, w.theta,
                              out=bufs, workspace=ws, stream=stream)
        else:
            jattn.rope_qkv(dinp["qkv_txt"], dinp["qkv_img"], dinp["qkv_ref"], dinp["pos"], w.split, w.theta,
                           "fp16" if path == "bf16" else "e4m3", out=bufs, stream=stream)
        if ev is not None:
            ev[1].record(stream)
        if path == "bf16":
            jattn.fwd_bf16(bufs[0], bufs[1], bufs[2], o=o, stream=stream)
        elif path == "bf16_hp":
            jattn.fwd_bf16_hp(*bufs, o=o, stream=stream)
        else:
            jattn.fwd_fp8(bufs[0], bufs[1], bufs[2], bufs[3], o=o, stream=stream)
        if ev is not None:
            ev[2].record(stream)

    return step


def measure_path(jattn, ctx: Ctx, w, dinp, path: str, steps: int, warmup: int):
    """Whole-path steps of one workload: (ms per step, mean prologue ms, mean
    forward ms, median forward ms, min forward ms), max over ranks."""
    step = path_step(jattn, w, dinp, path, ctx.dev, ctx.stream)
    ms, inner = time_calls(ctx, step, steps, warmup, marks=3)
    code, bits = jattn.device_status(clear=True)
    if code != jattn.OK:
        raise RuntimeError(f"device status {code} bits {bits} after the {path} run of {w.name}")
    pro = [x[0] for x in inner]
    fwd = [x[1] for x in inner]
    return (ms, ctx.max_ranks(float(np.mean(pro))), ctx.max_ranks(float(np.mean(fwd))),
            ctx.max_ranks(float(np.median(fwd))), ctx.max_ranks(float(np.min(fwd))))


def run_ours(args, rank, world, local):
    if world > 1:
        return run_partition(args, rank, world, local)
    from diffusion_transformer_joint_jattn_b200 import jattn

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    ctx = Ctx(dev, world)
    w = W.BY_NAME[args.workload]
    B, H, S, d = w.B, w.H, w.S, w.d
    flops = w.flops
    inp = W.make_inputs(w, seed=0)
    dinp = {k: (None if v is None else v.to(dev)) for k, v in inp.items()}
    peaks, peak_src = load_peaks()
    full = args.workload == WORKLOAD

    # The headline BF16 path is the high-precision one (range scales and
    # split-precision Q.K^T): the one that meets the BF16 error bars on every
    # workload.  The plain fp16-operand path is reported beside it.
    sampler = ClockSampler(local)
    sampler.start()
    ms, pro_ms, fwd_ms, fwd_med, fwd_min = measure_path(jattn, ctx, w, dinp, "bf16_hp", args.steps, args.warmup)
    clocks = sampler.stop()
    msf, prof, fwdf, fwdf_med, fwdf_min = measure_path(jattn, ctx, w, dinp, "bf16", args.steps, args.warmup)
    fast = {"value": round(whole_job_tflops(flops, msf), 2), "unit": UNIT, "ms_per_step": round(msf, 4),
            "prologue_ms": round(prof, 4), "fwd_ms": round(fwdf, 4), "fwd_ms_median": round(fwdf_med, 4),
            "fwd_ms_min": round(fwdf_min, 4), "gpu_launches_per_step": 2,
            "path": "jattn_rope_qkv (fp16) + jattn_fwd_bf16: fp16 operands, no range scales, no Q.K^T correction "
                    "(max-abs above 2e-2 on the outlier workloads)",
            "roofline": tensor_roofline(flops, fwdf, peaks, peak_src, False, FWD_TRAFFIC_BYTES if full else None,
                                        "attn_fwd_kernel<128, fp16 operands>")}
    fp8 = None
    if not args.no_fp8:
        ms8, pro8, fwd8, fwd8_med, fwd8_min = measure_path(jattn, ctx, w, dinp, "fp8", args.steps, args.warmup)
        fp8 = {"value": round(whole_job_tflops(flops, ms8), 2), "unit": UNIT, "ms_per_step": round(ms8, 4),
               "prologue_ms": round(pro8, 4), "fwd_ms": round(fwd8, 4), "fwd_ms_median": round(fwd8_med, 4),
               "fwd_ms_min": round(fwd8_min, 4),
               "roofline": tensor_roofline(flops, fwd8, peaks, peak_src, True,
                                           FWD_FP8_TRAFFIC_BYTES if full else None,
                                           "attn_fwd_kernel<128, e4m3 operands>")}

    extras = {}
    if not args.no_extras:
        extras = measure_extras(jattn, ctx, w, dinp, args, flops)
        extras["workloads"] = measure_other_workloads(jattn, ctx, args)

    e2e = None
    if not args.no_e2e:
        e2e = measure_e2e(jattn, ctx, w, inp, min(args.steps, 10), 2, flops)

    line = {
        "metric": METRIC, "value": round(whole_job_tflops(flops, ms), 2), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True,
        "scaling": "strong", "vs_baseline": None, "dtype": "fp16", "data": "synthetic",
        "config": {"workload": w.name, "B": B, "H": H, "S": S, "S_txt": w.S_txt, "S_img": w.S_img,
                   "S_ref": w.S_ref, "d": d, "rope_split": list(w.split), "theta": w.theta,
                   "path": "bf16 in/out; jattn_rope_qkv_hp + jattn_fwd_bf16_hp: fp16 MMA operands with "
                           "power-of-two block range scales and split-precision Q.K^T on 4 channel pairs per head, "
                           "fp32 accumulate",
                   "l2": "inputs larger than L2 (623 MB qkv streams, 622 MB laid-out q/k/v)",
                   "parallelism": "single GPU"},
        "prologue_ms": round(pro_ms, 4), "fwd_ms": round(fwd_ms, 4), "fwd_ms_median": round(fwd_med, 4),
        "fwd_ms_min": round(fwd_min, 4),
        "roofline": tensor_roofline(flops, fwd_ms, peaks, peak_src, False, FWD_HP_TRAFFIC_BYTES if full else None,
                                    "attn_fwd_kernel<128, fp16 operands, high precision>"),
        "prologue_roofline": {"bound": "hbm", "achieved": round(prologue_bytes(w, 2) / prof / 1e6, 1),
                              "peak": peaks["hbm_gbs"], "unit": "GB/s",
                              "frac": round(prologue_bytes(w, 2) / prof / 1e6 / peaks["hbm_gbs"], 4),
                              "peak_note": f"{peak_src} HBM copy bandwidth",
                              "kernel": "rope_qkv_kernel<128, fp16 out> (the fast path's prologue, one launch); "
                                        "the headline's prologue stage (prologue with range scales and pair "
                                        "statistics, pair selection, correction rows) is prologue_ms"},
        "gpu_launches": 4 * args.steps,
        "clocks": clocks,
    }
    line["bf16_fast"] = fast
    if fp8 is not None:
        line["fp8"] = fp8
    line.update(extras)
    if e2e is not None:
        line["e2e"] = e2e
    if rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w)
    if rank == 0:
        print(json.dumps(line), flush=True)


def measure_extras(jattn, ctx: Ctx, w, dinp, args, flops):
    """The next-row paths on the headline workload, timed the same way
    (device events around the call, inputs resident, workspace allocated
    beforehand):
    * FP8 attention with token repair (the whole call: prologue, selection,
      gather, fp16 pass, masked FP8 pass merging both), in alternation with the
      plain FP8 step;
    * the prologue with the query/key RMSNorm fused in, against the same
      prologue without it."""
    out = {"fp8_repair": measure_repair(jattn, ctx, w, dinp, args.rho, args.steps, args.warmup)}
    out["block_sparse"] = measure_block_sparse(jattn, ctx, w, dinp, args.tau, args.steps, args.warmup)
    out["torch_sdpa"] = measure_torch_sdpa(jattn, ctx, w, dinp, args.steps, args.warmup)
    B, H, S, d = w.B, w.H, w.S, w.d
    q = torch.empty(B, H, S, d, dtype=torch.float16, device=ctx.dev)
    bufs = (q, torch.empty_like(q), torch.empty_like(q), None)
    nw = W.norm_weights(d, 0).to(ctx.dev)
    res = {}
    for name, norm in (("plain", None), ("qk_norm", nw)):
        res[name], _ = time_calls(
            ctx, lambda ev: jattn.rope_qkv(dinp["qkv_txt"], dinp["qkv_img"], dinp["qkv_ref"], dinp["pos"], w.split,
                                           w.theta, "fp16", out=bufs, stream=ctx.stream, norm_w=norm),
            args.steps, args.warmup)
    nbytes = prologue_bytes(w, 2)
    out["prologue_qk_norm"] = {"ms": round(res["qk_norm"], 4), "ms_without_norm": round(res["plain"], 4),
                               "achieved_GBps": round(nbytes / res["qk_norm"] / 1e6, 1),
                               "note": "fp16 output; back-to-back calls (no flush between them)"}
    return out


def measure_block_sparse(jattn, ctx: Ctx, w, dinp, tau, steps, warmup):
    """Block-sparse forward at tau on the fp16 operands of the prologue: the
    call (block means, selection, sparse forward) timed alone; TFLOPS on the
    dense FLOP count (the work the call stands in for) and on the kept
    blocks' own FLOPs."""
    B, H, S, d = w.B, w.H, w.S, w.d
    q, k, v, _ = jattn.rope_qkv(dinp["qkv_txt"], dinp["qkv_img"], dinp["qkv_ref"], dinp["pos"], w.split, w.theta,
                                "fp16")
    o = torch.empty(B, S, H, d, dtype=torch.bfloat16, device=ctx.dev)
    ws = torch.empty(jattn.load().jattn_fwd_block_sparse_workspace(
        jattn.ctypes.byref(jattn.make_shape(B, H, S, 0, 0, d))), dtype=torch.uint8, device=ctx.dev)
    _, kl, kc = jattn.fwd_block_sparse(q, k, v, tau, o=o, want_blocks=True, workspace=ws)
    ms, _ = time_calls(ctx, lambda ev: jattn.fwd_block_sparse(q, k, v, tau, o=o, workspace=ws, stream=ctx.stream),
                       steps, warmup)
    code, bits = jattn.device_status(clear=True)
    if code != jattn.OK:
        raise RuntimeError(f"device status {code} bits {bits} after the block-sparse run")
    # FLOPs of the kept (query tile, key tile) pairs: each 256-row block of
    # full query rows times the kept keys (tails counted at their length)
    n_qb, n_kb = kc.shape[-1], jattn.n_blocks(S)
    klen = torch.full((n_kb,), 128, dtype=torch.float64)
    klen[-1] = S - 128 * (n_kb - 1)
    qlen = torch.full((n_qb,), 256, dtype=torch.float64)
    qlen[-1] = S - 256 * (n_qb - 1)
    kept_keys = torch.zeros(B, H, n_qb, dtype=torch.float64)
    kl, kc = kl.cpu(), kc.cpu()
    for b in range(B):
        for h in range(H):
            for i in range(n_qb):
                kept_keys[b, h, i] = klen[kl[b, h, i, :kc[b, h, i]].long()].sum()
    kept_flops = float(4 * d * (kept_keys * qlen).sum())
    return {"tau": tau, "ms": round(ms, 4), "kept_fraction": round(kept_flops / w.flops, 4),
            "dense_equivalent_tflops": round(w.flops / ms / 1e9, 2),
            "kept_tflops": round(kept_flops / ms / 1e9, 2), "gpu_launches_per_call": 3,
            "operands": "fp16 from jattn_rope_qkv (prologue not timed)"}


def measure_torch_sdpa(jattn, ctx: Ctx, w, dinp, steps, warmup):
    """Context only (never an oracle, never the product path): PyTorch's
    scaled_dot_product_attention, whichever fused backend it picks, on the
    same rotated fp16 operands laid out [B, H, S, d] by jattn_rope_qkv, beside
    this library's plain fp16-operand forward on the same operands, timed the
    same way (device events, inputs resident)."""
    import torch.nn.functional as F
    q, k, v, _ = jattn.rope_qkv(dinp["qkv_txt"], dinp["qkv_img"], dinp["qkv_ref"], dinp["pos"], w.split, w.theta,
                                "fp16")
    o = torch.empty(w.B, w.S, w.H, w.d, dtype=torch.bfloat16, device=ctx.dev)
    with torch.cuda.stream(ctx.stream):
        ms_t, _ = time_calls(ctx, lambda ev: F.scaled_dot_product_attention(q, k, v), steps, warmup)
    ms_j, _ = time_calls(ctx, lambda ev: jattn.fwd_bf16(q, k, v, o=o, stream=ctx.stream), steps, warmup)
    return {"ms": round(ms_t, 4), "tflops": round(w.flops / ms_t / 1e9, 2),
            "jattn_fwd_bf16_ms": round(ms_j, 4), "jattn_fwd_bf16_tflops": round(w.flops / ms_j / 1e9, 2),
            "torch": torch.__version__, "note": "context only: torch SDPA on the same fp16 [B, H, S, d] operands"}


def measure_repair(jattn, ctx: Ctx, w, dinp, rho, steps, warmup):
    """FP8 with token repair, timed in alternation with the plain FP8 step
    (one of each per round, each between its own events) so that the
    overhead compares calls made under the same clock and power state."""
    B, H, S, d = w.B, w.H, w.S, w.d
    n = jattn.repair_count(B, H, w.S_txt, w.S_img, w.S_ref, d, rho)
    ws = torch.empty(jattn.repair_workspace_bytes(B, H, w.S_txt, w.S_img, w.S_ref, d, rho), dtype=torch.uint8,
                     device=ctx.dev)
    o = torch.empty(B, S, H, d, dtype=torch.bfloat16, device=ctx.dev)
    plain = path_step(jattn, w, dinp, "fp8", ctx.dev, ctx.stream)

    def repair():
        jattn.fwd_fp8_repair(dinp["qkv_txt"], dinp["qkv_img"], dinp["qkv_ref"], dinp["pos"], w.split, w.theta,
                             rho=rho, workspace=ws, o=o, stream=ctx.stream)

    for _ in range(warmup):
        plain(None)
        repair()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    ctx.barrier()
    torch.cuda.synchronize()
    for e in ev:
        e[0].record(ctx.stream)
        plain(None)
        e[1].record(ctx.stream)
        e[2].record(ctx.stream)
        repair()
        e[3].record(ctx.stream)
    torch.cuda.synchronize()
    ctx.barrier()
    code, bits = jattn.device_status(clear=True)
    if code != jattn.OK:
        raise RuntimeError(f"device status {code} bits {bits} after the FP8-with-repair run")
    ms_p = ctx.max_ranks(float(np.mean([e[0].elapsed_time(e[1]) for e in ev])))
    ms = ctx.max_ranks(float(np.mean([e[2].elapsed_time(e[3]) for e in ev])))
    return {"value": round(whole_job_tflops(w.flops, ms), 2), "unit": UNIT, "ms_per_step": round(ms, 4),
            "rho": rho, "repaired_per_head": n, "workspace_bytes": ws.numel(), "gpu_launches_per_step": 5 if n else 2,
            "plain_fp8_ms_interleaved": round(ms_p, 4), "overhead_vs_fp8": round(ms / ms_p - 1, 4)}


def measure_other_workloads(jattn, ctx: Ctx, args):
    """Throughput on the other 2048x2048 workloads: the distilled T2I (B = 1,
    FP8 plain and with token repair) and the I2I with one reference image
    (S = 33280, BF16 and FP8).  Fewer steps: each is a few-second run."""
    peaks, peak_src = load_peaks()
    steps, warmup = max(3, min(args.steps, 10)), 3
    out = {}
    for name, paths in (("t2i_2048_distilled", ("fp8",)), ("i2i_2048_base", ("bf16", "fp8"))):
        w = W.BY_NAME[name]
        dinp = {k: (None if v is None else v.to(ctx.dev)) for k, v in W.make_inputs(w, 0).items()}
        res = {"B": w.B, "S": w.S, "flops_per_call": w.flops}
        for path in paths:
            ms, pro, fwd, _, _ = measure_path(jattn, ctx, w, dinp, path, steps, warmup)
            res[path] = {"value": round(whole_job_tflops(w.flops, ms), 2), "unit": UNIT, "ms_per_step": round(ms, 4),
                         "prologue_ms": round(pro, 4), "fwd_ms": round(fwd, 4),
                         "roofline": tensor_roofline(w.flops, fwd, peaks, peak_src, path == "fp8", None,
                                                     f"attn_fwd_kernel<128, {'e4m3' if path == 'fp8' else 'fp16'} "
                                                     "operands>")}
        if name == "t2i_2048_distilled":
            res["fp8_repair"] = measure_repair(jattn, ctx, w, dinp, args.rho, steps, warmup)
        out[name] = res
        del dinp
        torch.cuda.empty_cache()
    return out


def measure_e2e(jattn, ctx: Ctx, w, inp, steps, warmup, flops):
    """Public one-call API with host (pinned) buffers: H2D of the step's
    inputs, the path, D2H of the output, all inside the timed region."""
    host = {k: (None if v is None else v.pin_memory()) for k, v in inp.items()}
    out_host = torch.empty(w.B, w.S, w.H, w.d, dtype=torch.bfloat16).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in host.values() if v is not None)
    d2h = out_host.numel() * out_host.element_size()
    ms, _ = time_calls(ctx, lambda ev: jattn.joint_attention(host["qkv_txt"], host["qkv_img"], host["qkv_ref"],
                                                             host["pos"], w.split, w.theta, out=out_host),
                       steps, warmup)
    return {"value": round(whole_job_tflops(flops, ms), 2), "unit": UNIT, "ms_per_step": round(ms, 3),
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "api": "jattn.joint_attention -> jattn_joint_attention_host (C ABI, pinned host in/out, the "
                   "high-precision pair, copies pipelined with the kernels in (batch entry, 2-head) chunks on "
                   "copy streams)"}


# --------------------------------------------------------------------------- N > 1

def run_partition(args, rank, world, local):
    """The page's multi-GPU arrangement on `world` ranks: cfg_size x
    ulysses_size (batch entries over rank groups, each entry's sequence over
    its group), the whole batch fixed (strong scaling)."""
    import datetime
    import torch.distributed as dist
    from diffusion_transformer_joint_jattn_b200 import jattn, ulysses

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(seconds=120))
    ctx = Ctx(dev, world)
    w = W.BY_NAME[args.workload]
    lens = [w.S_txt, w.S_img, w.S_ref]
    cfg, uly = ulysses.cfg_ulysses_layout(world, w.B, w.H, [n for n in lens if n])
    groups = [dist.new_group(g) for g in ulysses.cfg_ulysses_groups(world, cfg, uly)]
    bsl, g, r = ulysses.rank_work(rank, w.B, cfg, uly)
    inp = W.make_inputs(w, seed=0)
    streams = [None if t is None else t[bsl] for t in (inp["qkv_txt"], inp["qkv_img"], inp["qkv_ref"])]
    host_shards = [None if t is None else t.pin_memory() for t in ulysses.shard_streams(streams, uly, r)]
    shards = [None if t is None else t.to(dev) for t in host_shards]
    pos_host = inp["pos"].pin_memory()
    pos = pos_host.to(dev)

    def step(ev):
        ulysses.ulysses_attention(shards, pos, w.split, w.theta, group=groups[g], precise=True)

    sampler = ClockSampler(local)
    sampler.start()
    ms, _ = time_calls(ctx, step, args.steps, args.warmup)
    clocks = sampler.stop()
    code, bits = jattn.device_status(clear=True)
    if code != jattn.OK:
        raise RuntimeError(f"device status {code} bits {bits} on rank {rank}")

    # End to end: every step copies this rank's input shards in from pinned
    # host memory, runs the same exchange + attention, and copies its output
    # shards back out (all on the timed stream).
    outs = ulysses.ulysses_attention(shards, pos, w.split, w.theta, group=groups[g], precise=True)
    out_host = [None if o is None else torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in outs]

    def e2e_step(ev):
        for hs, ds in zip(host_shards, shards):
            if hs is not None:
                ds.copy_(hs, non_blocking=True)
        pos.copy_(pos_host, non_blocking=True)
        res = ulysses.ulysses_attention(shards, pos, w.split, w.theta, group=groups[g], precise=True)
        for o, oh in zip(res, out_host):
            if o is not None:
                oh.copy_(o, non_blocking=True)

    ms_e2e, _ = time_calls(ctx, e2e_step, args.steps, args.warmup)
    code, bits = jattn.device_status(clear=True)
    if code != jattn.OK:
        raise RuntimeError(f"device status {code} bits {bits} on rank {rank} (end to end)")
    h2d = world * (sum(t.numel() * t.element_size() for t in host_shards if t is not None)
                   + pos_host.numel() * pos_host.element_size())
    d2h = world * sum(t.numel() * t.element_size() for t in out_host if t is not None)
    line = {
        "metric": METRIC, "value": round(whole_job_tflops(w.flops, ms), 2), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True,
        "scaling": "strong", "vs_baseline": None, "dtype": "fp16", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "S": w.S, "d": w.d,
                   "path": "bf16 in/out; ulysses_attention per rank: NCCL all-to-all, jattn_rope_qkv_hp + "
                           "jattn_fwd_bf16_hp, all-to-all",
                   "l2": "inputs larger than L2",
                   "parallelism": f"cfg{cfg} x ulysses{uly}"},
        "gpu_launches": 4 * args.steps,
        "clocks": clocks,
        "e2e": {"value": round(whole_job_tflops(w.flops, ms_e2e), 2), "unit": UNIT, "ms_per_step": round(ms_e2e, 4),
                "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                "api": "ulysses.ulysses_attention on every rank (high-precision pair), each rank's pinned host "
                       "input shards copied in and its output shards copied out within the step; bytes summed "
                       "over ranks"},
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    ctx.barrier()
    for grp in groups:
        dist.destroy_process_group(grp)
    dist.destroy_process_group()


# --------------------------------------------------------------------------- oracle on the host

def oracle_sample(w, rows_per_head: int, heads: int, seed: int = 0):
    """Run the FP64 oracle on `heads` (b, h) pairs x `rows_per_head` query
    rows of workload w.  Returns (seconds, flops, worker threads)."""
    import oracle
    from threadpoolctl import threadpool_limits
    sub = w.with_batch_heads(B=1, H=heads)
    inp = W.make_inputs(sub, seed)
    rows = W.sample_rows(sub, rows_per_head, seed)
    # One worker thread per host core, each with a single-threaded BLAS, so
    # the threads used are exactly `workers`.
    workers = host_workers()
    with threadpool_limits(1):
        t = time.perf_counter()
        oracle.joint_attention(inp["qkv_txt"], inp["qkv_img"], inp["qkv_ref"], inp["pos"], sub.split, sub.theta,
                               rows=rows, workers=workers)
        dt = time.perf_counter() - t
    return dt, 4 * heads * rows.shape[-1] * w.S * w.d, workers


def cpu_model() -> str:
    """The host CPU's model name (Linux /proc/cpuinfo), for the oracle timings."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def host_workers() -> int:
    """Worker threads of the oracle timing: one per host core."""
    return max(1, os.cpu_count() or 1)


def round_heads(w, n: float, workers: int) -> int:
    """A head count for a sample: the oracle runs one head per worker thread,
    so a multiple of the worker count (at most B*H) keeps every core busy."""
    return int(max(1, min(w.B * w.H, -(-int(math.ceil(n)) // workers) * workers)))


def sample_shape(w, target_s: float):
    """(heads, rows) of one oracle sample of about ``target_s`` seconds: one
    head per worker thread, rows fitted from two timed probes (a fixed cost
    per head -- rotating its keys -- plus a cost per row)."""
    workers = host_workers()
    heads = round_heads(w, 1, workers)
    r0, r1 = min(64, w.S), min(256, w.S)
    t0, _, _ = oracle_sample(w, r0, heads)
    if r1 == r0:
        return heads, r0
    t1, _, _ = oracle_sample(w, r1, heads)
    per_row = max((t1 - t0) / (r1 - r0), 1e-9)
    fixed = max(t0 - per_row * r0, 0.0)
    rows = int((target_s - fixed) / per_row)
    return heads, int(max(32, min(w.S, rows)))


def cpu_baseline(w, target_s: float = ORACLE_SAMPLE_S, samples: int = 2):
    """The FP64 oracle on the host cores, on `samples` samples of the shape
    the reference arm times per step."""
    heads, rows = sample_shape(w, target_s)
    dts, fl, workers = [], 0, host_workers()
    for i in range(samples):
        dt, fl, workers = oracle_sample(w, rows, heads, seed=i)
        dts.append(dt)
    dt = float(np.mean(dts))
    return {"value": round(fl / dt / 1e12, 6), "unit": UNIT, "cores": workers, "blas_threads_per_worker": 1,
            "kind": "oracle", "cpu_model": cpu_model(),
            "sample": f"{heads} heads x {rows} sampled query rows of {w.name} (S={w.S}, d={w.d}), FP64 numpy "
                      f"oracle incl. RoPE, mean of {samples} samples of {dt:.1f} s"}


def run_reference(args, rank, world):
    if rank != 0:
        return
    w = W.BY_NAME[args.workload]
    per_step_s = min(ORACLE_SAMPLE_S, max(0.5, 150.0 / max(1, args.steps + args.warmup)))
    heads, rows = sample_shape(w, per_step_s)
    times, fl, workers = [], 0, host_workers()
    for i in range(args.warmup + args.steps):
        dt, fl, workers = oracle_sample(w, rows, heads, seed=i)
        if i >= args.warmup:
            times.append(dt)
    sec = float(np.mean(times))
    value = fl / sec / 1e12
    ms_full = w.flops / (fl / sec) * 1e3
    line = {"metric": METRIC, "value": round(value, 6), "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_full, 1), "higher_is_better": True, "scaling": "strong",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": w.name, "B": w.B, "H": w.H, "S": w.S, "d": w.d,
                       "note": "each step = FP64 oracle on %d heads x %d sampled rows; ms_per_step extrapolated "
                               "to the full call from the sampled rate" % (heads, rows)},
            "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": workers, "blas_threads_per_worker": 1,
                             "kind": "oracle", "cpu_model": cpu_model(),
                             "sample": f"{heads} heads x {rows} query rows per step"},
            "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    rank, world, local = dist_env()
    if args.impl == "reference":
        run_reference(args, rank, world)
    else:
        run_ours(args, rank, world, local)


if __name__ == "__main__":
    main()
