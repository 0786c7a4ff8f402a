"""Benchmark of the FlashDecoder streaming step on B200.

One step = one latent frame through the whole per-frame step (embed, every
block's QKV / attention / O-proj / MLP, final projection + unpatchify), i.e.
one replay of the library's CUDA graph via fd_decode_frame. The warm-up
steps also fill the rolling cache, so every timed step runs with the full
(W+1)-frame window. Each latent frame yields r_t = 4 pixel frames.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME]
  python bench.py --impl reference ...   (the CPU oracle on a bounded sample)

Rank 0 prints one JSON line. With N > 1 (torchrun) every rank decodes its
own independent video on its own GPU (replicas: the step has no exchange),
the timed region is bracketed by barriers and the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import fd_synth  # noqa: E402

METRIC = "decoded pixel frames/s at 1080p; p50 per-latent-frame latency; % of bf16 TC peak"
UNIT = "pixel frames/s"
DEFAULT_CONFIG = "1080p_wan22"

# DRAM traffic of one attention launch (one block, full window) measured by
# ncu (dram__bytes_read.sum + dram__bytes_write.sum), see
# profiles/attention_1080p_ncu.md. Keyed by the sha256 of the kernel source:
# when the kernel changes the figure no longer applies and is reported as null.
NCU_ATTN_TRAFFIC = {
    ("1080p_wan22", "1034ad4e5f3acab874932dac0e62d5b31664d64097e8713c2afd4bba88c521b3"):
        163608064 + 58525440,
}


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def is_paper(cfg) -> bool:
    return getattr(cfg, "head", "linear") == "paper"


def refine_batched(cfg) -> bool:
    """The library runs all r_t sub-frames through each refinement block in one
    launch per kernel for bf16 storage with L_frm a multiple of 8 (the ring
    layout the decoder reports through ring_layout), else one at a time."""
    return is_paper(cfg) and cfg.dtype == "bf16" and cfg.L_frm % 8 == 0


def describe(cfg) -> str:
    streams = f"{cfg.batch} video streams per step, " if getattr(cfg, "batch", 1) > 1 else ""
    head = (f"paper head (upsample x{cfg.r_t}, {cfg.n_refine} refinement blocks over "
            f"{cfg.r_t * (cfg.window + 1)} sub-frames, spatial MLP)" if is_paper(cfg)
            else "linear head")
    return (f"{cfg.name}: {streams}latent {cfg.latent_ch}ch {cfg.grid_h}x{cfg.grid_w}, patch {cfg.patch} "
            f"({cfg.L_frm} tokens/frame), d={cfg.d_model}, {cfg.n_heads} heads x {cfg.head_dim}"
            f" / {cfg.n_kv_heads} KV groups, {cfg.n_blocks} blocks, MLP {cfg.mlp_ratio}x, "
            f"W={cfg.window}, {head}{', FP8 E4M3 MLPs' if getattr(cfg, 'mlp_fp8', 0) else ''}; "
            f"each latent frame -> "
            f"{cfg.out_ch}x{cfg.r_t}x{cfg.out_shape[2]}x{cfg.out_shape[3]} px")


def attn_flops_per_launch(cfg):
    """FLOPs of each attention launch of one steady-state frame, in launch
    order: the backbone blocks (window of W+1 frames), then with the paper
    head the refinement launches (window of r_t (W+1) sub-frames): one per
    block covering all r_t sub-frames, or r_t x n_refine of one sub-frame."""
    L, hd, B = cfg.L_frm, cfg.n_heads * cfg.head_dim, getattr(cfg, "batch", 1)
    out = [B * 4 * L * ((cfg.window + 1) * L) * hd] * cfg.n_blocks
    if is_paper(cfg):
        sub = B * 4 * L * (cfg.r_t * (cfg.window + 1) * L) * hd
        if refine_batched(cfg):
            out += [cfg.r_t * sub] * cfg.n_refine
        else:
            out += [sub] * (cfg.r_t * cfg.n_refine)
    return out


def kind_flops(cfg):
    """FLOPs of one launch of each GEMM kind (2 per MAC), all B streams."""
    L, D = cfg.L_frm * getattr(cfg, "batch", 1), cfg.d_model
    f = {"qkv": 2 * L * D * cfg.qkv_dim, "oproj": 2 * L * cfg.n_heads * cfg.head_dim * D,
         "mlp_up": 2 * L * D * cfg.d_ff, "mlp_down": 2 * L * D * cfg.d_ff,
         "embed": 2 * L * cfg.c_in * D}
    if is_paper(cfg):
        f.update(upsample=2 * L * D * cfg.r_t * D, spatial=2 * L * D * D,
                 final=2 * L * D * cfg.c_px)
    else:
        f["final"] = 2 * L * D * cfg.c_out
    return f


def frame_kind_flops(cfg):
    """FLOPs of each GEMM kind summed over the launches of one frame."""
    k = kind_flops(cfg)
    blocks = cfg.n_blocks + (cfg.r_t * cfg.n_refine if is_paper(cfg) else 0)
    out = {n: blocks * k[n] for n in ("qkv", "oproj", "mlp_up", "mlp_down")}
    out["embed"] = k["embed"]
    if is_paper(cfg):
        out.update(upsample=k["upsample"], spatial=cfg.r_t * k["spatial"],
                   final=cfg.r_t * k["final"])
    else:
        out["final"] = k["final"]
    return out


def kernels_per_frame(cfg) -> int:
    per_block = 5 + (1 if getattr(cfg, "mlp_fp8", 0) else 0)   # FP8: + MLP-input quantization
    n = 2 + per_block * cfg.n_blocks                    # step_begin, embed, backbone
    if is_paper(cfg):
        sub = 1 if refine_batched(cfg) else cfg.r_t     # launches per refinement kernel
        return n + 1 + sub * (per_block * cfg.n_refine + 2)  # upsample, refinement, spatial MLP
    return n + 1                                        # final


def flops_per_frame(cfg):
    """Algorithmic FLOPs of one steady-state latent frame; returns (total,
    attention part)."""
    k = kind_flops(cfg)
    block = k["qkv"] + k["oproj"] + k["mlp_up"] + k["mlp_down"]
    attn = sum(attn_flops_per_launch(cfg))
    gemm = k["embed"] + cfg.n_blocks * block
    if is_paper(cfg):
        gemm += k["upsample"] + cfg.r_t * (cfg.n_refine * block + k["spatial"] + k["final"])
    else:
        gemm += k["final"]
    return gemm + attn, attn


def file_sha(path):
    return hashlib.sha256(open(path, "rb").read()).hexdigest()


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        rows = [r.split(",") for r in out.strip().splitlines() if r.count(",") >= 8]
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        pw = [float(r[3]) for r in rows if r[3].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4)
                          if r[5 + i].strip().lower() == "active"})
        load = [s for s in sm if mx and s > 0.3 * max(mx)] or sm
        return {"sm_mhz": float(np.median(load)) if load else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows),
                # SM clock range and power under load: per-step latency drift
                # over the timed region follows the clock when the power cap acts
                "sm_mhz_range": [min(load), max(load)] if load else None,
                "power_w_max": max(pw) if pw else None,
                "sm_mhz_by_sample": [int(x) for x in load][:400]}


# ------------------------------------------------------------------ dist
def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        local = int(os.environ.get("LOCAL_RANK", "0"))
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
        return dist, dist.get_rank(), world, local
    return None, 0, 1, 0


def barrier(dist):
    if dist is not None:
        dist.barrier()


def _reduce(dist, v, op):
    import torch
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=op)
    return float(t.item())


def max_over_ranks(dist, v):
    """Timing of a replicated step: the slowest rank's time."""
    return v if dist is None else _reduce(dist, v, dist.ReduceOp.MAX)


def sum_over_ranks(dist, v):
    """Work of a replicated step: the units all ranks processed."""
    return v if dist is None else _reduce(dist, v, dist.ReduceOp.SUM)


def replica_throughput(r_t, frames_all_ranks, max_ms, batch=1):
    """Whole-job pixel frames per second of N independent decoders, each
    decoding `batch` video streams per step."""
    return r_t * batch * frames_all_ranks / (max_ms / 1e3)


# ------------------------------------------------------------------ oracle
def one_block_weights(cfg, weights):
    """Weights of the same decoder with its first backbone block only."""
    return {k: v for k, v in weights.items()
            if not (k.startswith("b") and not k.startswith("b0."))}


def time_backbone_block(dec, z_t):
    """Seconds of one backbone block of the oracle on a full window (the
    block's cache is left as it was)."""
    import collections
    x = dec.embed(z_t)
    dq = collections.deque(dec.cache[0])
    t0 = time.perf_counter()
    dec._block("b0.", dq, dec.cfg.window + 1, x)
    return time.perf_counter() - t0


def oracle_sample_seconds(cfg, weights_1blk, z):
    """Time the CPU oracle on a bounded sample: frames 0..W of a decoder with
    one backbone block at the workload's full width (untimed set-up), then
    frame W+1 (full window, head included) timed, and one more backbone block
    timed alone. Returns (seconds per latent frame of the full-depth decoder,
    detail) = frame + (n_blocks - 1) x block."""
    import oracle
    dec = oracle.OracleDecoder(cfg.replace(n_blocks=1), weights_1blk)
    for t in range(cfg.window + 1):
        dec.decode_frame(z[t])
    t0 = time.perf_counter()
    dec.decode_frame(z[cfg.window + 1])
    t_one = time.perf_counter() - t0
    t_block = time_backbone_block(dec, z[0])
    per_frame = t_one + (cfg.n_blocks - 1) * t_block
    return per_frame, dict(t_block_s=t_block, t_frame_1blk_s=t_one)


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def run_reference(args):
    # the CPU oracle: rank 0 alone runs it; other ranks exit without work
    if int(os.environ.get("RANK", "0")) != 0:
        return 0
    cfg = fd_synth.CONFIGS[args.config]
    w1 = one_block_weights(cfg, fd_synth.make_weights(cfg))
    frames = args.warmup + args.steps + cfg.window + 2
    z = fd_synth.make_latents(cfg, frames=frames)
    import oracle
    dec = oracle.OracleDecoder(cfg.replace(n_blocks=1), w1)
    for t in range(cfg.window + 1):                     # fill the window (not a step)
        dec.decode_frame(z[t])
    t = cfg.window + 1
    for _ in range(args.warmup):
        dec.decode_frame(z[t]); t += 1
    t_block = time_backbone_block(dec, z[0])
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        dec.decode_frame(z[t]); t += 1
        times.append(time.perf_counter() - t0)
    per_frame = float(np.mean(times)) + (cfg.n_blocks - 1) * t_block
    value = cfg.r_t / per_frame
    sample = (f"each step: one full-window latent frame of the decoder with 1 backbone block at "
              f"the workload's full width ({cfg.L_frm} tokens, {(cfg.window + 1) * cfg.L_frm}-"
              f"token window), head included; per-frame time = that + {cfg.n_blocks - 1} x one "
              f"backbone block ({t_block:.2f} s, timed once)")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": per_frame * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": describe(cfg), "latent_frame_per_step": 1},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ main arm
def run_flashdec(args):
    import torch
    from streaming_transformer_video_b200 import FlashDecoder
    dist, rank, world, local = dist_setup(args.gpus)
    torch.cuda.set_device(local)
    cfg = fd_synth.CONFIGS[args.config].replace(batch=args.batch)
    if args.blocks > 0:
        cfg = cfg.replace(n_blocks=args.blocks)
    td = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    weights = fd_synth.make_weights(cfg)
    n_frames = args.warmup + args.steps
    B = cfg.batch
    # [T][B][C'][H'][W']: one video per stream, seeded per rank and stream
    z = np.stack([fd_synth.make_latents(cfg, frames=n_frames, seed=1 + rank * B + b)
                  for b in range(B)], axis=1)
    out_shape = (B,) + tuple(cfg.out_shape)
    if args.mlp_fp8:
        # static calibration (paper Sec. 4.6): the warm-up frames through the
        # bf16 decoder, recording each block's MLP input / hidden ranges
        cal = FlashDecoder(cfg, weights, record_mlp_amax=True)
        cal.reset()
        lat_c = torch.from_numpy(z[:args.warmup]).to(td).cuda()
        out_c = torch.empty(out_shape, dtype=td, device="cuda")
        for t in range(args.warmup):
            cal.decode_frame(lat_c[t], out_c)
        weights = {**weights, **cal.mlp_fp8_scales()}
        cal.close()
        del lat_c, out_c
        cfg = cfg.replace(mlp_fp8=1)
    # events only around the attention launches (the roofline kernel): an
    # event record node per kernel would cost ~1 us each inside the step
    dec = FlashDecoder(cfg, weights, kernel_timing=2)
    stream = torch.cuda.Stream()
    lat = torch.from_numpy(z).to(td).cuda()
    outs = [torch.empty(out_shape, dtype=td, device="cuda") for _ in range(2)]
    with torch.cuda.stream(stream):
        dec.reset(stream)
        for t in range(args.warmup):
            dec.decode_frame(lat[t], outs[t % 2], stream)
    stream.synchronize()
    assert dec.status() == 0

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    kern = {}
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    barrier(dist)
    torch.cuda.synchronize()
    mem_before = torch.cuda.mem_get_info()[0]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for i in range(args.steps):
        t = args.warmup + i
        ev[i][0].record(stream)
        dec.decode_frame(lat[t], outs[t % 2], stream)
        ev[i][1].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize()
    mem_after = torch.cuda.mem_get_info()[0]
    # device time of every attention launch of the last timed frame (CUDA
    # events recorded inside the graph; each replay overwrites them, so only
    # the last frame's are readable without syncing between frames)
    attn_launch_ms = [ms for kind, ms in dec.kernel_ms() if kind == "attn"]
    barrier(dist)
    clk = clocks.stop()
    assert dec.status() == 0
    total_ms = t_start.elapsed_time(t_end)
    total_ms = max_over_ranks(dist, total_ms)
    lat_ms = [a.elapsed_time(b) for a, b in ev]
    frames_all = sum_over_ranks(dist, args.steps)
    value = replica_throughput(cfg.r_t, frames_all, total_ms, cfg.batch)
    launches = kernels_per_frame(cfg)

    # ---- end to end: host buffers through fd_decode_frame_host
    lat_h = [torch.from_numpy(z[t]).to(td).pin_memory() for t in range(n_frames)]
    out_h = torch.empty(out_shape, dtype=td).pin_memory()
    e2e_steps = args.steps
    dec2 = FlashDecoder(cfg, weights)
    with torch.cuda.stream(stream):
        dec2.reset(stream)
        for t in range(args.warmup):
            dec2.decode_frame_host(lat_h[t], out_h, stream)
    stream.synchronize()
    barrier(dist)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(e2e_steps):
        dec2.decode_frame_host(lat_h[args.warmup + i], out_h, stream)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(dist)
    assert dec2.status() == 0
    e2e_ms = max_over_ranks(dist, e0.elapsed_time(e1))
    e2e_value = cfg.r_t * cfg.batch * sum_over_ranks(dist, e2e_steps) / (e2e_ms / 1e3)
    h2d = int(np.prod(lat.shape[1:])) * (2 if td == torch.bfloat16 else 4)
    d2h = int(np.prod(outs[0].shape)) * (2 if td == torch.bfloat16 else 4)
    dev_bytes = dec.device_bytes()
    dec2.close()

    # ---- per-kernel breakdown (informational, a separate short pass after
    # the timed region with events around every kernel)
    dec3 = FlashDecoder(cfg, weights, kernel_timing=1)
    with torch.cuda.stream(stream):
        dec3.reset(stream)
        for t in range(min(n_frames, cfg.window + 3)):
            dec3.decode_frame(lat[t], outs[t % 2], stream)
    stream.synchronize()
    for kind, ms in dec3.kernel_ms():
        kern.setdefault(kind, []).append(ms)
    dec3.close()

    # ---- roofline of the dominant kernel (attention) and of the whole step
    peaks, peak_src = measured_peaks()
    peak = float(peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops")))
    attn_fl = attn_flops_per_launch(cfg)
    assert len(attn_fl) == len(attn_launch_ms)
    attn_tf = sum(attn_fl) / (sum(attn_launch_ms) * 1e-3) / 1e12
    src = os.path.join(ROOT, "streaming_transformer_video_b200", "csrc", "fd_attn_tc.cuh")
    traffic = NCU_ATTN_TRAFFIC.get((args.config, file_sha(src)))
    step_flops, _ = flops_per_frame(cfg)
    step_tf = step_flops / (total_ms / args.steps * 1e-3) / 1e12

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not args.mlp_fp8:
        # the oracle decodes one stream at a time: stream 0's video
        per_frame, detail = oracle_sample_seconds(cfg.replace(batch=1),
                                                  one_block_weights(cfg, weights), z[:, 0])
        cpu = {"value": cfg.r_t / per_frame, "unit": UNIT, "cores": blas_threads(),
               "kind": "oracle",
               "sample": (f"frame {cfg.window + 1} (full {cfg.window + 1}-frame window) of the "
                          f"decoder with 1 backbone block at full width, head included "
                          f"({detail['t_frame_1blk_s']:.2f} s), after frames 0..{cfg.window} "
                          f"untimed; per-frame time = that + {cfg.n_blocks - 1} x one backbone "
                          f"block ({detail['t_block_s']:.2f} s)")}

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": ("bf16+e4m3-mlp" if args.mlp_fp8 else "bf16") if cfg.dtype == "bf16" else "f32",
        "data": "synthetic",
        "config": {"workload": describe(cfg), "latent_frame_per_step": 1,
                   "streams_per_gpu": cfg.batch, "replicas": world,
                   "l2": "no flush: every step streams ~%.1f GB (weights + ring cache) > 126 MB L2"
                         % (dev_bytes / 1e9)},
        "p50_ms": float(np.percentile(lat_ms, 50)), "p99_ms": float(np.percentile(lat_ms, 99)),
        "latency_ms_by_step": [round(x, 4) for x in lat_ms],
        "tc_frac_step": step_tf / peak,
        "step_tflops": step_tf,
        "roofline": {"bound": "tensor", "kernel": "tc_attn_kernel", "achieved": attn_tf,
                     "peak": peak, "unit": "TFLOP/s", "frac": attn_tf / peak,
                     "traffic": traffic,
                     "peak_source": f"{peak_src} bf16 sustained (kernel timed inside a long step)"},
        "kernels_ms": {k: float(np.mean(v)) for k, v in kern.items()},
        "kernels_tflops": {},
        "clocks": clk,
        "gpu_launches": launches * args.steps,
        "device_bytes": dev_bytes,
        # free device memory right before and after the timed steps: the
        # decoder allocates nothing per frame, so the two are equal
        "device_free_bytes_before_after": [int(mem_before), int(mem_after)],
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
    }
    # per kind: its FLOPs in one frame over its launches' time in the last frame
    for k, f in frame_kind_flops(cfg).items():
        if k in kern and k != "embed":
            line["kernels_tflops"][k] = f / (float(np.sum(kern[k])) * 1e-3) / 1e12
    # attention launches of the last frame of the breakdown pass, in launch order
    per_frame_attn = kern["attn"][-len(attn_fl):]
    line["kernels_tflops"]["attn"] = sum(attn_fl) / (sum(per_frame_attn) * 1e-3) / 1e12
    if cpu is not None:
        line["cpu_baseline"] = cpu
    dec.close()
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=60)
    ap.add_argument("--warmup", type=int, default=4)
    ap.add_argument("--impl", default="flashdec", choices=["flashdec", "reference"])
    ap.add_argument("--config", default=DEFAULT_CONFIG, choices=sorted(fd_synth.CONFIGS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--batch", type=int, default=1,
                    help="video streams decoded together per step (each its own video)")
    ap.add_argument("--blocks", type=int, default=0,
                    help="profiling only: override the number of Transformer blocks "
                         "(a shallower decoder of the same width, for short ncu captures; "
                         "its line is not the workload's measurement)")
    ap.add_argument("--mlp-fp8", action="store_true",
                    help="FP8 E4M3 MLP GEMMs with static scales calibrated on the warm-up "
                         "frames by a bf16 handle that records the MLP ranges")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_flashdec(args)


if __name__ == "__main__":
    sys.exit(main())
