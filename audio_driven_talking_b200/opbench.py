"""Operator-level timing of the library's kernels through the C ABI, for roofline figures and
for ncu captures of one kernel on a case of a chosen size.

    python -m audio_driven_talking_b200.opbench row_norm --rows 65536
    python -m audio_driven_talking_b200.opbench attention --tokens 1280
    python -m audio_driven_talking_b200.opbench linear --m 1280 --n 1536 --k 1536
    python -m audio_driven_talking_b200.opbench cross_attention --tokens 1280
    python -m audio_driven_talking_b200.opbench slice --blocks 2 --iters 3 [--renoise]
    python -m audio_driven_talking_b200.opbench slice_kernels --blocks 30

Each prints one JSON line: the operator, its shape, the average time per launch in
microseconds (CUDA events on the launching stream, after warm-up launches, synchronised on
both sides; with --graph the launches are replayed from one CUDA graph, so host work per
call does not separate them) and the algorithmic bytes or FLOPs per launch with the rate they give. Inputs are
synthetic (seeded normal values on the device). Inputs of `row_norm` at the default size
(65536 rows of 1536 floats, 402 MB read) exceed the 126 MB L2, so consecutive launches read
them from HBM; the other operators' inputs stay in L2, as they do inside a block.
"""
import argparse
import json
import math

import audio_driven_talking_b200 as fh


GRAPH = False  # set by --graph: time the launches replayed from one CUDA graph


def _time(fn, iters, warmup):
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    run, n = fn, iters
    if GRAPH:
        # `iters` launches recorded once and replayed: the device time of back-to-back kernels
        # without the host's per-call work (argument checks, tensor-map encoding) in between
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(iters):
                fn()
        g.replay()
        torch.cuda.synchronize()
        run, n = g.replay, 3
    st = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(n):
        run()
    e1.record(st)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) * 1000.0 / (n * (iters if GRAPH else 1))


def _gen(seed):
    import torch
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    return g


def row_norm(a):
    import torch
    g = _gen(1)
    M, D = a.rows, a.dim
    x = torch.randn((M, D), device="cuda", generator=g)
    sc = 0.1 * torch.randn((D,), device="cuda", generator=g)
    sh = 0.1 * torch.randn((D,), device="cuda", generator=g)
    out = torch.empty((M, D), dtype=torch.bfloat16, device="cuda")
    us = _time(lambda: fh.row_norm(x, a.mode, sc, sh, 0, M, out=out), a.iters, a.warmup)
    nbytes = M * D * 4 + M * D * 2
    return {"op": "row_norm", "kernel": "norm_rows_kernel", "rows": M, "dim": D, "mode": a.mode, "us": us,
            "bytes": nbytes, "gb_per_s": nbytes / us / 1e3}


def attention(a):
    import torch
    g = _gen(2)
    B, NH, L = a.batch, a.heads, a.tokens
    q = torch.randn((B, NH, L, 128), device="cuda", generator=g).to(torch.bfloat16)
    k = torch.randn((B, NH, L, 128), device="cuda", generator=g).to(torch.bfloat16)
    v = torch.randn((B, NH, L, 128), device="cuda", generator=g).to(torch.float16)
    ssq = 128.0 * torch.rand((B * L, 2 * NH), device="cuda", generator=g) + 64.0
    us = _time(lambda: fh.attention(q, k, v, ssq), a.iters, a.warmup)
    flops = 4.0 * B * NH * L * L * 128
    return {"op": "attention", "kernel": "attn_tc_kernel", "batch": B, "heads": NH, "tokens": L, "us": us,
            "flop": flops, "tflop_per_s": flops / us / 1e6}


def linear(a):
    import torch
    g = _gen(3)
    M, N, K = a.m, a.n, a.k
    A = torch.randn((M, K), device="cuda", generator=g).to(torch.bfloat16)
    W = (torch.randn((N, K), device="cuda", generator=g) / math.sqrt(K)).to(torch.bfloat16)
    b = torch.randn((N,), device="cuda", generator=g)
    us = _time(lambda: fh.linear(A, W, b), a.iters, a.warmup)
    flops = 2.0 * M * N * K
    return {"op": "linear", "m": M, "n": N, "k": K, "us": us, "flop": flops, "tflop_per_s": flops / us / 1e6}


def cross_attention(a):
    import torch
    g = _gen(4)
    B, NH, F, L = a.batch, a.heads, a.frames, a.tokens
    D = NH * 128
    q = torch.randn((B, L, D), device="cuda", generator=g).to(torch.bfloat16)
    kv = torch.randn((B, F, 32, 2 * D), device="cuda", generator=g).to(torch.bfloat16)
    sq = 128.0 * torch.rand((B * L, NH), device="cuda", generator=g) + 64.0
    sk = 128.0 * torch.rand((B * F * 32, NH), device="cuda", generator=g) + 64.0
    us = _time(lambda: fh.cross_attention(q, sq, kv, sk, F), a.iters, a.warmup)
    nbytes = B * L * D * 2 * 2 + B * F * 32 * 2 * D * 2 + B * L * NH * 4
    return {"op": "cross_attention", "kernel": "xattn_tc_kernel", "batch": B, "heads": NH, "frames": F, "tokens": L,
            "us": us, "bytes": nbytes, "gb_per_s": nbytes / us / 1e3}


def slice_(a):
    """The whole sampler on a model of `blocks` blocks (the kernels of the 30-block model on a
    small device footprint): one launch each of the small per-step kernels per step."""
    import torch
    cfg = fh.LITE.replace(blocks=a.blocks)
    m = fh.DiT(cfg, 1002)
    ws = m.workspace(1)
    g = _gen(5)
    C, F, H, W, A, D = cfg.latent_ch, cfg.frames, cfg.lat_h, cfg.lat_w, cfg.audio_tokens, cfg.dim
    noise = torch.randn((1, C, F, H, W), device="cuda", generator=g)
    ref = torch.randn((1, C, F, H, W), device="cuda", generator=g)
    motion = torch.randn((1, C, 2, H, W), device="cuda", generator=g)
    audio = torch.randn((1, F, A, D), device="cuda", generator=g).to(torch.bfloat16)
    sig = [1.0, 0.75, 0.5, 0.25, 0.0]
    out = torch.empty_like(noise)
    if a.renoise:  # the re-noising sampler, with its fresh draws per step
        eps = torch.randn((len(sig) - 1,) + tuple(noise.shape), device="cuda", generator=g)
        run = lambda: m.sample_slice_renoise(noise, ref, motion, audio, sig, eps, ws, out=out)
    else:
        run = lambda: m.sample_slice(noise, ref, motion, audio, sig, ws, out=out)
    us = _time(run, a.iters, a.warmup)
    m.close()
    return {"op": "slice", "blocks": a.blocks, "steps": len(sig) - 1, "renoise": bool(a.renoise), "us": us}


def slice_kernels(a):
    """One sampler slice of a model of `blocks` blocks replayed from its CUDA graph under the
    CUDA profiler (CUPTI): per kernel, the spacing of consecutive kernel ends on the stream,
    i.e. what each kernel adds to the slice once programmatic launches overlap its prologue
    with its predecessor. Median and total per kernel name."""
    import collections
    import statistics
    import torch
    from torch.profiler import ProfilerActivity, profile
    cfg = fh.LITE.replace(blocks=a.blocks)
    m = fh.DiT(cfg, 1002)
    ws = m.workspace(1)
    g = _gen(5)
    C, F, H, W, A, D = cfg.latent_ch, cfg.frames, cfg.lat_h, cfg.lat_w, cfg.audio_tokens, cfg.dim
    noise = torch.randn((1, C, F, H, W), device="cuda", generator=g)
    ref = torch.randn((1, C, F, H, W), device="cuda", generator=g)
    motion = torch.randn((1, C, 2, H, W), device="cuda", generator=g)
    audio = torch.randn((1, F, A, D), device="cuda", generator=g).to(torch.bfloat16)
    sig = [1.0, 0.75, 0.5, 0.25, 0.0]
    out = torch.empty_like(noise)
    run = lambda: m.sample_slice(noise, ref, motion, audio, sig, ws, out=out)
    us = _time(run, a.iters, a.warmup)
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        run()
        torch.cuda.synchronize()
    ks = sorted((e.time_range.start, e.time_range.end, e.name) for e in prof.events()
                if e.device_type == torch.autograd.DeviceType.CUDA)
    inc = collections.defaultdict(list)
    for i in range(1, len(ks)):
        name = ks[i][2].replace("(anonymous namespace)::", "").replace("fh::", "").replace("void ", "")
        inc[name.split("(")[0]].append(ks[i][1] - ks[i - 1][1])
    m.close()
    per = {n: {"launches": len(v), "median_us": statistics.median(v), "total_us": sum(v)}
           for n, v in sorted(inc.items(), key=lambda kv: -sum(kv[1]))}
    return {"op": "slice_kernels", "blocks": a.blocks, "steps": len(sig) - 1, "us": us, "kernels": per}


def parser():
    p = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    p.add_argument("op", choices=["row_norm", "attention", "linear", "cross_attention", "slice", "slice_kernels"])
    p.add_argument("--rows", type=int, default=65536)
    p.add_argument("--dim", type=int, default=1536)
    p.add_argument("--mode", type=int, default=0)
    p.add_argument("--batch", type=int, default=1)
    p.add_argument("--heads", type=int, default=12)
    p.add_argument("--tokens", type=int, default=1280)
    p.add_argument("--frames", type=int, default=5)
    p.add_argument("--m", type=int, default=1280)
    p.add_argument("--n", type=int, default=1536)
    p.add_argument("--k", type=int, default=1536)
    p.add_argument("--blocks", type=int, default=2)
    p.add_argument("--renoise", action="store_true")
    p.add_argument("--iters", type=int, default=20)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--graph", action="store_true", help="replay the launches from a CUDA graph")
    return p


def main(argv=None):
    a = parser().parse_args(argv)
    global GRAPH
    GRAPH = a.graph and not a.op.startswith("slice")  # the sampler records its own graph
    import torch
    torch.cuda.set_device(0)
    fn = {"row_norm": row_norm, "attention": attention, "linear": linear, "cross_attention": cross_attention,
          "slice": slice_, "slice_kernels": slice_kernels}[a.op]
    r = fn(a)
    r["graph"] = GRAPH
    print(json.dumps(r))


if __name__ == "__main__":
    main()
