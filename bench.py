"""Benchmark of the FlashHead Lite DiT slice sampler on B200.

Workload (one "step" = one slice): the 4-step Euler flow sampler (sigmas 1, .75,
.5, .25, 0) over the 30-block, width-1536 network on a 5 x 16 x 16 latent (1280
tokens, 512 x 512 frames), batch 1, motion frames 0-1 pinned, fresh seeded audio
tokens per slice; each slice yields 24 output frames. Metric: output frames/s
(24 x slices / device time), with DiT TFLOP/s against the dense BF16 peak beside
it. Inputs are synthetic and seeded; weights are the seeded synthetic network.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

N > 1 (under torch.distributed.run) runs N independent replicas, one per GPU
(the sampler has no exchange step); value = all ranks' frames / max rank time.
--impl reference times the CPU oracle (the only other implementation there is)
on a bounded sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth_inputs as si  # noqa: E402

METRIC = "output frames/sec per 4-step 30-block slice at 512x512; DiT TFLOP/s vs BF16 peak"
UNIT = "frames/s"
SIGMAS = [1.0, 0.75, 0.5, 0.25, 0.0]
FRAMES_PER_SLICE = 24
NET_SEED = 1002          # the Lite network shared by the full-width configurations
INPUT_SEED = 1003        # the sampler configuration's inputs
C, F, H, W, A, D, NB, FF, L = 128, 5, 16, 16, 32, 1536, 30, 8960, 1280


def slice_tflop() -> float:
    """Matmul + attention flops of one slice (cross-attention keys/values computed once per slice)."""
    gemm_block = 2 * L * D * (3 * D) + 2 * L * D * D * 3 + 2 * L * D * FF * 2   # qkv, o/cq/co, ffn
    attn = 4 * L * L * D                      # self-attention: QK^T and PV over all heads
    xattn = 4 * L * A * D                     # per-frame cross-attention
    patch_head = 2 * L * (2 * C) * D + 2 * L * D * C
    per_step = NB * (gemm_block + attn + xattn) + patch_head
    ckv = 2 * (F * A) * D * (2 * D) * NB
    return (4 * per_step + ckv) / 1e12


# launches per class inside one slice, and each launch's algorithmic flops
CLASS_NAMES = {1: "gated-residual GEMMs (O-proj, cross-O, FFN2): gemm_tc2s_kernel<256,EPI_RESID> "
                  "(split-K on clusters of four CTAs, two cta_group::2 pairs, eight epilogue warps)",
               2: "gemm_tc2_kernel<224,EPI_GELU> (CTA pair; FFN1)"}


def class_flops_per_launch(cls: int) -> float:
    if cls == 1:   # O-proj and cross-O (K = D) and FFN2 (K = FF), equally often
        return (2 * L * D * D * 2 + 2 * L * FF * D) / 3.0
    if cls == 2:
        return 2.0 * L * D * FF
    raise ValueError(cls)


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for f in ("gemm_tc.cu", "epilogue.cuh", "common.cuh"):
        h.update(open(os.path.join(ROOT, "audio_driven_talking_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def measured_traffic(cls: int):
    """Per-launch DRAM bytes of the timed kernel from the committed ncu summary, if the kernel is unchanged."""
    p = os.path.join(ROOT, "profiles", "gemm_tc_cfg3_traffic.md")
    if not os.path.exists(p):
        return None
    text = open(p).read()
    m = re.search(r"class %d traffic_bytes_per_launch: (\d+) source_sha256: ([0-9a-f]+)" % cls, text)
    if not m or m.group(2) != kernel_source_hash():
        return None
    return int(m.group(1))


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d.get("bf16_tflops", 1630.0), d.get("bf16_tflops_sustained", 1371.8), "of measured"
    return 1590.0, 1400.0, "of fallback"


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
             "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
             "clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = max(mx, float(parts[2]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


class OracleSample:
    """The oracle, as it stands, on a bounded sample of the workload: whole blocks of the
    1280-token network in the oracle's plain float32 mode (the parity reference of the bf16
    paths); a slice is 4 steps x 30 blocks of them."""

    PREC = "f32"

    def __init__(self):
        from oracle import model as om
        self.om = om
        cfg = om.CFG3
        self.W = om.make_weights(cfg, NET_SEED, blocks=[0, 1, 2, 3])
        self.x, self.a, t = si.block_inputs(INPUT_SEED, 1, cfg.tokens, cfg.dim, cfg.frames, cfg.audio_tokens, True)
        _, self.e0 = om.time_conditioning(self.W, t, self.PREC)
        self.ang = om.rope_angles(cfg)
        self.n = 0

    def block(self):
        self.x = self.om.block_forward(self.W, self.n % 4, self.x, self.a, self.e0, self.PREC, ang=self.ang)
        self.n += 1

    @staticmethod
    def cores():
        cores = len(os.sched_getaffinity(0))
        try:
            from threadpoolctl import threadpool_info
            th = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
            if th:
                cores = int(max(th))
        except Exception:
            pass
        return cores


def cpu_baseline(target_s: float = 15.0):
    """(frames/s, cores, sample text) of the oracle timed for about target_s seconds."""
    o = OracleSample()
    n, t0 = 0, time.perf_counter()
    while True:
        o.block()
        n += 1
        el = time.perf_counter() - t0
        if el >= target_s or n >= 64:
            break
    per_block = el / n
    return FRAMES_PER_SLICE / (per_block * 4 * NB), o.cores(), \
        f"{n} blocks of the 1280-token network (numpy float32 oracle), {per_block:.3f} s/block, " \
        f"scaled x{4 * NB} blocks per slice"


def run_reference(args, rank, world):
    """The CPU oracle timed as the reference arm. Each step is ONE BLOCK of the network (a
    bounded sample of a slice, which is 4 x 30 blocks): `steps` counts blocks and
    `ms_per_step` is milliseconds per block; `value` is the frames/s of whole slices that
    this block time implies, and `slice_extrapolation` states the scaling."""
    if rank != 0:
        return
    o = OracleSample()
    for _ in range(args.warmup):
        o.block()
    steps = max(1, args.steps)
    t0 = time.perf_counter()
    for _ in range(steps):
        o.block()
    el = time.perf_counter() - t0
    per_block = el / steps
    fps = FRAMES_PER_SLICE / (per_block * 4 * NB)
    sample = f"{steps} blocks of the 1280-token network (numpy float32 oracle), {per_block:.3f} s/block, " \
             f"scaled x{4 * NB} blocks per slice"
    cfg = workload_config(1, steps)
    cfg["step_unit"] = "one block of the network (a slice is 4 steps x 30 blocks)"
    line = {"impl": "reference", "metric": METRIC, "value": fps, "unit": UNIT, "n_gpus": args.gpus, "steps": steps,
            "warmup": args.warmup, "ms_per_step": 1000.0 * per_block, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": cfg,
            "slice_extrapolation": {"blocks_per_slice": 4 * NB, "ms_per_slice": 1000.0 * per_block * 4 * NB,
                                    "frames_per_slice": FRAMES_PER_SLICE},
            "cpu_baseline": {"value": fps, "unit": UNIT, "cores": o.cores(), "kind": "oracle", "sample": sample},
            "e2e": {"value": fps, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def rank_env():
    """(world, rank, local_rank) of this process, from the variables torchrun sets (1, 0, 0 alone)."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def max_over_ranks(value, world, device):
    """The largest of every rank's `value` (a device time in ms), on every rank: the
    job's time is its slowest replica's. Every rank must call it at the same point."""
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_frames_per_s(slices_per_rank, world, ms_max):
    """Whole-job throughput: the frames every replica produced over the slowest one's time."""
    return FRAMES_PER_SLICE * slices_per_rank * world / (ms_max / 1000.0)


def workload_config(world, steps):
    return {"workload": "slice sampler: 4 Euler steps over 30 blocks x 1536 (12 heads x 128), latent 5x16x16 = "
                        "1280 tokens (512x512), batch 1, motion frames pinned, fresh audio per slice",
            "slices_per_gpu": steps, "tokens": L, "batch": 1, "parallelism": f"replicas x{world}",
            "l2": "no flush: each slice streams 11.1 GB of weights (2.79 GB per flow step), far above the 126 MB L2",
            "tflop_per_slice": round(slice_tflop(), 4)}


def run_gpu(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    import audio_driven_talking_b200 as fh

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    m = fh.DiT(fh.LITE, NET_SEED, device=local_rank)
    ws = m.workspace(1)
    K, Wm = args.steps, args.warmup
    noise, ref, motion, _ = si.slice_inputs(INPUT_SEED, 1, C, F, H, W, A, D, True)
    # every slice's inputs resident in HBM before timing; audio seeded per slice
    audios = [torch.from_numpy(si.audio_tokens(INPUT_SEED + j, 1, F, A, D, True)).to(torch.bfloat16).to(dev)
              for j in range(K + Wm)]
    nd, rd, md = (torch.from_numpy(t).to(dev) for t in (noise, ref, motion))
    out = torch.empty_like(nd)
    timing_class = args.timing_class
    stream = torch.cuda.current_stream()

    for j in range(Wm):
        m.sample_slice(nd, rd, md, audios[K + j], SIGMAS, ws, out=out)
    m.sync()
    launches_per_slice = m.last_launch_count

    def timed(nslices):
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record(stream)
        for j in range(nslices):
            m.sample_slice(nd, rd, md, audios[j], SIGMAS, ws, out=out)
        ev1.record(stream)
        torch.cuda.synchronize()
        m.sync()
        if world > 1:
            dist.barrier()
        return ev0.elapsed_time(ev1)

    with ClockSampler(local_rank) as clk:
        ms = timed(K)
    ms_max = max_over_ranks(ms, world, dev)

    # roofline pass: the same slices again with CUDA events around every launch of one
    # kernel class (events recorded inside the graph; kept out of the headline timing)
    m.set_timing(timing_class)
    m.sample_slice(nd, rd, md, audios[-1], SIGMAS, ws, out=out)   # records the instrumented graph
    m.sync()
    kernel_us, kernel_n = [], 0
    if world > 1:
        dist.barrier()
    for j in range(min(K, 4)):
        m.sample_slice(nd, rd, md, audios[j], SIGMAS, ws, out=out)
        m.sync()
        us, n = m.get_timing()
        kernel_us.append(us)
        kernel_n += n
    kernel_us = float(np.mean(kernel_us)) if kernel_us else 0.0
    m.set_timing(0)

    # end to end through the C ABI with host buffers (pinned), copies inside the timed region
    pin = lambda a, dt=None: (torch.from_numpy(a).to(dt) if dt else torch.from_numpy(a)).pin_memory()
    hn, hr, hm = pin(noise), pin(ref), pin(motion)
    haud = [pin(si.audio_tokens(INPUT_SEED + j, 1, F, A, D, True), torch.bfloat16) for j in range(K)]
    hout = torch.empty(noise.shape, dtype=torch.float32).pin_memory()
    m.sample_slice_host(hn, hr, hm, haud[0], SIGMAS, ws, hout)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for j in range(K):
        m.sample_slice_host(hn, hr, hm, haud[j], SIGMAS, ws, hout)
    e1.record(stream)
    torch.cuda.synchronize()
    te_max = max_over_ranks(e0.elapsed_time(e1), world, dev)
    if world > 1:
        dist.barrier()
    h2d = hn.nbytes + hr.nbytes + hm.nbytes + haud[0].numel() * haud[0].element_size()
    d2h = hout.nbytes

    # the re-noising sampler (reading R12 of the update for distilled checkpoints) on the
    # same slices: one buffer of seeded draws per slice workload, refilled in place
    eps = torch.from_numpy(si.renoise_draws(INPUT_SEED, len(SIGMAS) - 1, 1, C, F, H, W)).to(dev)
    m.sample_slice_renoise(nd, rd, md, audios[0], SIGMAS, eps, ws, out=out)   # records its graph
    m.sync()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    r0, r1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    r0.record(stream)
    for j in range(K):
        m.sample_slice_renoise(nd, rd, md, audios[j], SIGMAS, eps, ws, out=out)
    r1.record(stream)
    torch.cuda.synchronize()
    m.sync()
    tr_max = max_over_ranks(r0.elapsed_time(r1), world, dev)
    if world > 1:
        dist.barrier()

    if rank == 0:
        value = job_frames_per_s(K, world, ms_max)
        burst, sustained, src = peaks()
        tflops = slice_tflop() * K * world / (ms_max / 1000.0)
        achieved = class_flops_per_launch(timing_class) / (kernel_us * 1e-6) / 1e12 if kernel_n else None
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": Wm,
            "ms_per_step": ms_max / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic (seeded latents, audio tokens and weights)",
            "config": workload_config(world, K),
            "tflops": tflops, "tflops_frac_burst": tflops / burst, "peak_note": src,
            "e2e": {"value": job_frames_per_s(K, world, te_max), "unit": UNIT,
                    "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)},
            # the burst peak: the step's SM clock stays at its maximum (the clocks field below),
            # so the power-capped sustained figure would flatter the kernel; its fraction is kept
            # beside for reference
            "roofline": {"bound": "tensor", "kernel": CLASS_NAMES[timing_class], "achieved": achieved,
                         "peak": burst, "unit": "TFLOP/s",
                         "frac": (achieved / burst) if achieved else None,
                         "frac_of_sustained": (achieved / sustained) if achieved else None,
                         "traffic": measured_traffic(timing_class), "launches_timed": kernel_n,
                         "mean_launch_us": kernel_us, "peak_kind": f"bf16 burst ({src})",
                         "flops_per_launch": class_flops_per_launch(timing_class)},
            "renoise_sampler": {"value": job_frames_per_s(K, world, tr_max), "unit": UNIT,
                                "ms_per_step": tr_max / K,
                                "note": "same workload, re-noising update with seeded fresh draws per step"},
            "gpu_launches": launches_per_slice * K,
            "clocks": clk.summary(),
        }
        if world == 1 and not args.no_cpu_baseline:
            fps, cores, sample = cpu_baseline()
            line["cpu_baseline"] = {"value": fps, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample}
        print(json.dumps(line), flush=True)
    m.close()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--timing-class", type=int, default=1, choices=[1, 2])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    world, rank, local_rank = rank_env()
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        run_gpu(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
