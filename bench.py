#!/usr/bin/env python
"""GPTQ layer-quantization throughput on B200: weights quantized per second.

Workload (one "step" = the whole hot path on one layer): a Llama-7B-shaped q_proj,
W 4096 x 4096 fp16 (1% outlier columns x10), X = 262,144 calibration tokens (bf16, low rank
256 + noise with Student-t(3) feature scales), 4-bit asymmetric grids per 128 columns, lazy
blocks of 128.  A step runs the four C-ABI calls: Hessian accumulation over all tokens,
preparation of R (dead features, damping, factorization), column-wise quantization with lazy
trailing updates, and packing.  Inputs are synthetic and seeded (workloads/synth.py).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (torchrun, one process per GPU) every rank quantizes its own independent layer
(weak scaling, no data-path collective); value = all ranks' weights / max-over-ranks time.
Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "GPTQ weights quantized/sec per layer (4-bit g128) on 1 B200; % of roofline"
UNIT = "weights/s"


GRID_MODES = {"static": 0, "dynamic": 2}  # the library's grid_given argument


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--chunk", type=int, default=262144, help="tokens per accumulate call")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--scale", type=float, default=1.0,
                    help="shrink the layer (tests only); the bench line is for 1.0")
    ap.add_argument("--grid", choices=sorted(GRID_MODES), default="static",
                    help="static groups (the default line) or dynamic groups (grid refitted per "
                         "processing group on the GPU)")
    ap.add_argument("--w4a16", choices=["q_proj", "fc2"], default=None,
                    help="instead of the quantization step, time the W4A16 product X Ŵᵀ over "
                         "packed 4-bit g128 codes of this layer shape (one call = one step)")
    ap.add_argument("--w4a16-tokens", type=int, default=1)
    ap.add_argument("--w4a16-layout", choices=["rows", "tiles"], default="rows",
                    help="codes in gptq_pack's row layout, or re-laid into 16 KB tiles first "
                         "(gptq_retile_codes, outside the timed region)")
    ap.add_argument("--n-tokens", type=int, default=0,
                    help="calibration tokens (profiling captures only; the bench line uses all)")
    return ap.parse_args()


def workload(scale: float, n_tokens: int = 0):
    import dataclasses
    from workloads.synth import CONFIGS
    spec = CONFIGS[2][0]
    if scale != 1.0:
        spec = spec.scaled(max(32, int(spec.m * scale)), max(128, int(spec.d * scale)),
                           max(512, int(spec.n_tokens * scale)))
    if n_tokens:
        spec = dataclasses.replace(spec, n_tokens=n_tokens)
    return spec


def workload_config(spec, chunk, grid="static"):
    return {"workload": f"q_proj {spec.m}x{spec.d} fp16 W, N={spec.n_tokens} bf16 tokens, "
                        f"{spec.bits}-bit g{spec.group}" +
                        (" (dynamic groups)" if grid == "dynamic" else "") +
                        f", block {spec.block}",
            "grid": grid,
            "m": spec.m, "d": spec.d, "n_tokens": spec.n_tokens, "bits": spec.bits,
            "group": spec.group, "block": spec.block, "act_order": spec.act_order,
            "chunk_tokens": min(chunk, spec.n_tokens),
            "l2": "flushed between timed steps (256 MiB write)"}


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
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
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        import statistics
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for n, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": float(rows[0][2]) if rows[0][2].replace(".", "").isdigit() else None,
                "reasons": sorted(reasons), "samples": len(rows)}


# ----------------------------------------------------------------------------- helpers
def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return j.get("bf16_tflops", 1590.0), j.get("hbm_gbs", 6650.0), "measured"
    return 1590.0, 6650.0, "fallback"


def kernel_source_digest(files):
    """Hash of the code of `files` with comments and whitespace removed, so that the committed
    ncu counters stay tied to the kernel and not to its comments."""
    import re
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), encoding="utf-8") as fh:
            src = fh.read()
        src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
        src = re.sub(r"//[^\n]*", " ", src)
        h.update(" ".join(src.split()).encode())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str, digest: str, per_launch_scale: float = 1.0):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on this exact
    kernel source; else None."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        j = json.load(f)
    e = j.get(kernel)
    if not e or e.get("source_digest") != digest:
        return None
    return e["dram_bytes_per_launch"] * per_launch_scale


def dist_setup(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """Maximum of a per-rank time over all ranks (NCCL: on the GPU; gloo: on the host)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(rank: int) -> int:
    """Every rank quantizes its own, independently drawn layer."""
    return 1 + rank


def weak_scaling_value(world: int, m: int, d: int, per_step_s: float) -> float:
    """Whole-job weights per second: every rank quantizes m x d weights per step, and the job
    takes as long as its slowest rank."""
    return world * m * d / per_step_s


# ----------------------------------------------------------------------------- oracle leg
def oracle_sample(spec, seed: int, n_tok: int, rows: int, grid: str = "static"):
    """The CPU oracle on a bounded sample of the layer: H from `n_tok` tokens at full d,
    preparation at full d, lazy-block quantization of `rows` rows.  Returns (seconds for the
    sample, seconds extrapolated to the whole layer, description)."""
    import numpy as np
    import torch
    from oracle import gptq_oracle as O
    from workloads.synth import XSource, make_weight

    W = make_weight(spec, seed, "cpu")[:rows].float().double().numpy()
    xs = XSource(spec.scaled(spec.m, spec.d, n_tok, chunk=n_tok), seed, "cpu")
    Xt = xs.chunk(0).float().double().numpy()
    t0 = time.perf_counter()
    H = O.hessian_tokens(Xt)
    t1 = time.perf_counter()
    prep = O.prepare_with_retry(H, spec.percdamp, spec.act_order)
    t2 = time.perf_counter()
    Wp = W[:, prep["perm"]]
    if grid == "dynamic":
        sc, ze = O.dynamic_grid_arrays(rows, spec.d, spec.group)
        O.gptq_lazy(Wp, prep["R"], sc, ze, np.arange(spec.d) // spec.group, spec.bits,
                    spec.block, dynamic=spec.group)
    else:
        sc, ze = O.fit_grid(W, spec.bits, spec.group)
        gcol = (prep["perm"] // spec.group) if spec.group != -1 else np.zeros(spec.d, int)
        O.gptq_lazy(Wp, prep["R"], sc, ze, gcol, spec.bits, spec.block)
    t3 = time.perf_counter()
    full = (t1 - t0) * (spec.n_tokens / n_tok) + (t2 - t1) + (t3 - t2) * (spec.m / rows)
    desc = (f"H from {n_tok} of {spec.n_tokens} tokens (time x{spec.n_tokens / n_tok:g}), "
            f"prepare at full d={spec.d}, quantize {rows} of {spec.m} rows "
            f"(time x{spec.m / rows:g}); extrapolated to the whole layer")
    return t3 - t0, full, desc


def cores_used():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count()


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    spec = workload(args.scale, args.n_tokens)
    n_tok, rows = min(2048, spec.n_tokens), min(16, spec.m)
    for _ in range(args.warmup):
        oracle_sample(spec, 1, n_tok, rows, args.grid)
    fulls = []
    desc = ""
    t_start = time.perf_counter()
    for _ in range(args.steps):
        _, full, desc = oracle_sample(spec, 1, n_tok, rows, args.grid)
        fulls.append(full)
    wall = time.perf_counter() - t_start
    per_layer = sum(fulls) / len(fulls)
    value = spec.m * spec.d / per_layer
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": per_layer * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(spec, args.chunk, args.grid),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores_used(),
                             "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
            "sample_wall_s": wall}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- our path
def run_ours(args):
    import torch
    import post_weight_quantization_17_b200 as G
    from workloads.synth import XSource, make_weight

    world, rank, local = dist_setup(args)
    spec = workload(args.scale, args.n_tokens)
    seed = rank_seed(rank)
    dev = torch.device("cuda", torch.cuda.current_device())
    W = make_weight(spec, seed, dev)
    # the data do not depend on --chunk: 8192-token chunks are generated and regrouped
    xs = XSource(spec, seed, dev)
    per = max(1, args.chunk // spec.chunk)
    chunks = []
    group = []
    for c in xs.chunks():
        group.append(c)
        if len(group) == per:
            chunks.append(torch.cat(group) if per > 1 else group[0])
            group = []
    if group:
        chunks.append(torch.cat(group))
    del group
    stream = torch.cuda.Stream(dev)
    ctx = G.Context(m_max=spec.m, d_max=spec.d, act_order=spec.act_order, stream=stream)
    bufs = G.LayerBuffers(spec.m, spec.d, spec.bits, spec.group, dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    syrk_ev = []

    def step(record=False):
        n = 0
        for xc in chunks:
            if record:
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                a.record(stream)
            n = G.gptq_hessian_accumulate(ctx, xc, bufs.S, n)
            if record:
                b.record(stream)
                syrk_ev.append((a, b))
        G.gptq_prepare_hinv(ctx, bufs.S, n, spec.percdamp, spec.act_order, bufs.R, bufs.perm,
                            bufs.dead)
        G.gptq_quantize_layer(ctx, W, bufs.R, bufs.perm if spec.act_order else None, bufs.dead,
                              spec.bits, spec.group, spec.block, GRID_MODES[args.grid],
                              bufs.scales, bufs.zeros,
                              bufs.codes, bufs.W_hat, bufs.col_loss)
        G.gptq_pack(ctx, bufs.codes, spec.bits, bufs.packed)

    clocks = ClockSampler(local)
    clocks.start()  # sampling covers the warm-up and the timed steps (nvidia-smi needs ~0.2 s)
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
        G.gptq_sync_status(ctx)
        torch.cuda.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        launches0 = G.gptq_kernel_launches(ctx)
        step_ev = []
        for _ in range(args.steps):
            flush.zero_()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            step(record=True)
            b.record(stream)
            step_ev.append((a, b))
        torch.cuda.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        clk = clocks.stop()
        launches = G.gptq_kernel_launches(ctx) - launches0
        G.gptq_sync_status(ctx)
    step_ms = [a.elapsed_time(b) for a, b in step_ev]
    syrk_ms = sum(a.elapsed_time(b) for a, b in syrk_ev) / args.steps
    total_s = max_over_ranks(sum(step_ms) / 1e3, world)
    per_step_s = total_s / args.steps
    value = weak_scaling_value(world, spec.m, spec.d, per_step_s)

    # roofline of the dominant kernel (Hessian accumulation): algorithmic flops per launch
    bf16_peak, hbm_peak, peak_src = measured_peaks()
    syrk_flops = float(spec.n_tokens) * spec.d * (spec.d + 1)   # lower triangle incl. diagonal
    n_launch = len(chunks)
    achieved = syrk_flops / (syrk_ms / 1e3) / 1e12
    digest = kernel_source_digest(["post_weight_quantization_17_b200/csrc/k_syrk.cu",
                                   "post_weight_quantization_17_b200/csrc/gemm_simt.cuh",
                                   "post_weight_quantization_17_b200/csrc/tc_util.cuh"])
    roofline = {"kernel": "hessian_accumulate (S += X^T X)", "bound": "tensor",
                "achieved": achieved, "peak": bf16_peak, "unit": "TFLOP/s",
                "frac": achieved / bf16_peak, "peak_source": f"{peak_src} bf16 burst",
                "traffic": ncu_traffic("hessian_accumulate", digest, 1.0 / n_launch),
                "algorithmic_flops_per_step": syrk_flops, "launches_per_step": n_launch,
                "kernel_ms_per_step": syrk_ms, "source_digest": digest}

    # end to end through the public API with host buffers (pinned), copies inside the region:
    # X goes up in 16384-token slabs on a copy stream, double-buffered, and each slab's Hessian
    # update runs while the next slab is in flight; then prepare, quantize, pack, and the packed
    # codes with their grid come back to the host
    e2e = None
    if not args.no_e2e:
        import post_weight_quantization_17_b200 as G
        X_host = torch.cat([c.cpu() for c in chunks]).pin_memory()
        W_host = W.cpu().pin_memory()
        out_host = [torch.empty_like(t, device="cpu").pin_memory() for t in
                    (bufs.packed, bufs.scales, bufs.zeros)]
        h2d = X_host.numel() * X_host.element_size() + W_host.numel() * W_host.element_size()
        d2h = sum(t.numel() * t.element_size() for t in out_host)
        slab = 16384
        n_tok = X_host.shape[0]
        slabs = [(a0, min(n_tok, a0 + slab)) for a0 in range(0, n_tok, slab)]
        dbuf = [torch.empty(slab, spec.d, dtype=X_host.dtype, device=dev) for _ in range(2)]
        copy_stream = torch.cuda.Stream()
        e2e_steps = max(3, min(args.steps, 10))
        with torch.cuda.stream(stream):
            torch.cuda.synchronize()
            barrier(world)
            t_ev = []
            for _ in range(e2e_steps):
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                landed = [torch.cuda.Event(), torch.cuda.Event()]
                free = [torch.cuda.Event(), torch.cuda.Event()]
                a.record(stream)
                W.copy_(W_host, non_blocking=True)
                copy_stream.wait_event(a)
                n_total = 0
                for k, (a0, a1) in enumerate(slabs):
                    u = k % 2
                    with torch.cuda.stream(copy_stream):
                        if k >= 2:
                            copy_stream.wait_event(free[u])
                        dbuf[u][:a1 - a0].copy_(X_host[a0:a1], non_blocking=True)
                        landed[u].record(copy_stream)
                    stream.wait_event(landed[u])
                    n_total = G.gptq_hessian_accumulate(ctx, dbuf[u][:a1 - a0], bufs.S, n_total)
                    free[u].record(stream)
                G.gptq_prepare_hinv(ctx, bufs.S, n_total, spec.percdamp, spec.act_order, bufs.R,
                                    bufs.perm, bufs.dead)
                G.gptq_quantize_layer(ctx, W, bufs.R, bufs.perm if spec.act_order else None,
                                      bufs.dead, spec.bits, spec.group, spec.block,
                                      GRID_MODES[args.grid],
                                      bufs.scales, bufs.zeros, bufs.codes, bufs.W_hat,
                                      bufs.col_loss)
                G.gptq_pack(ctx, bufs.codes, spec.bits, bufs.packed)
                for hd, dv in zip(out_host, (bufs.packed, bufs.scales, bufs.zeros)):
                    hd.copy_(dv, non_blocking=True)
                b.record(stream)
                b.synchronize()
                t_ev.append((a, b))
            barrier(world)
        e2e_s = max_over_ranks(sum(a.elapsed_time(b) for a, b in t_ev) / 1e3 / e2e_steps, world)
        e2e = {"value": weak_scaling_value(world, spec.m, spec.d, e2e_s), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": e2e_s * 1e3, "h2d_slab_tokens": slab}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        n_tok, rows = min(131072, spec.n_tokens), min(3072, spec.m)
        sample_s, full_s, desc = oracle_sample(spec, seed, n_tok, rows, args.grid)
        cpu = {"value": spec.m * spec.d / full_s, "unit": UNIT, "cores": cores_used(),
               "kind": "oracle", "sample": desc, "sample_seconds": sample_s}

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_step_s * 1e3,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "bf16 products, f32 accumulate/factor/quantize",
                "data": "synthetic (seeded; workloads/synth.py)",
                "config": workload_config(spec, args.chunk, args.grid),
                "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "clocks": clk,
                "gpu_launches": launches, "gpu_launches_per_step": launches / args.steps,
                "step_ms_min": min(step_ms), "step_ms_max": max(step_ms)}
        print(json.dumps(line), flush=True)
    ctx.close()
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def oracle_w4a16_sample(m: int, d: int, T: int, rows: int, g: int = 128):
    """The CPU oracle's W4A16 product (unpack, dequantize, multiply in fp64) on `rows` of the m
    rows; returns (seconds for the sample, seconds extrapolated to all m rows, description)."""
    import numpy as np
    from oracle import gptq_oracle as O
    rng = np.random.default_rng(1)
    packed = rng.integers(0, 2 ** 32, size=(rows, d // 8), dtype=np.uint64).astype(np.uint32)
    scales = rng.uniform(1e-3, 2.1e-2, (rows, d // g)).astype(np.float32)
    zeros = rng.integers(0, 16, (rows, d // g))
    X = rng.normal(size=(T, d)).astype(np.float32).astype(np.float64)
    t0 = time.perf_counter()
    O.dequant_matmul(X, packed, d, 4, scales, zeros, g)
    dt = time.perf_counter() - t0
    desc = (f"the oracle's product on {rows} of {m} rows (time x{m / rows:g}), T={T}; "
            "extrapolated to the whole layer")
    return dt, dt * m / rows, desc


def run_w4a16(args):
    """The consumer of the packed format on one GPU: Y [T, m] = X [T, d] Ŵᵀ with X bf16 and
    random valid 4-bit codes (g = 128).  Small T is bound by reading the codes from HBM, large T
    by the tensor cores; the line reports the bound that applies."""
    import torch
    import post_weight_quantization_17_b200 as G
    m, d = {"q_proj": (4096, 4096), "fc2": (12288, 49152)}[args.w4a16]
    T, g = args.w4a16_tokens, 128
    torch.cuda.set_device(0)
    gen = torch.Generator(device="cuda").manual_seed(1)
    packed = torch.randint(-2 ** 31, 2 ** 31 - 1, (m, d // 8), dtype=torch.int32, device="cuda",
                           generator=gen)
    scales = torch.rand(m, d // g, device="cuda", generator=gen) * 0.02 + 1e-3
    zeros = torch.randint(0, 16, (m, d // g), dtype=torch.int32, device="cuda", generator=gen)
    X = torch.randn(T, d, device="cuda", generator=gen).to(torch.bfloat16)
    Y = torch.empty(T, m, device="cuda")
    ctx = G.Context(m_max=4096, d_max=4096, act_order=True)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    if args.w4a16_layout == "tiles":
        tiled = torch.empty(G.gptq_tiled_words(m, d), dtype=torch.int32, device="cuda")
        G.gptq_retile_codes(ctx, packed, d, tiled)

        def product():
            G.gptq_dequant_matmul_tiled(ctx, X, tiled, m, g, scales, zeros, Y)

        # the tiled product must equal the row-layout product (same definition; the split of K
        # may differ, so the sums agree to rounding) before it is timed
        Y_rows = torch.empty_like(Y)
        G.gptq_dequant_matmul(ctx, X, packed, d, 4, g, scales, zeros, Y_rows)
        product()
        G.gptq_sync_status(ctx)
        rel = float((Y - Y_rows).norm() / Y_rows.norm())
        if not rel <= 1e-5:
            raise RuntimeError(f"tiled W4A16 product differs from the row-layout one: rel {rel:.2e}")
        del Y_rows
    else:
        def product():
            G.gptq_dequant_matmul(ctx, X, packed, d, 4, g, scales, zeros, Y)
    for _ in range(max(3, args.warmup)):
        product()
    G.gptq_sync_status(ctx)
    torch.cuda.synchronize()
    clocks = ClockSampler(0)
    clocks.start()
    times = []
    launches0 = G.gptq_kernel_launches(ctx)
    for _ in range(args.steps):
        flush.zero_()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        product()
        b.record(stream)
        torch.cuda.synchronize()
        times.append(a.elapsed_time(b) * 1e-3)
    clk = clocks.stop()
    launches = G.gptq_kernel_launches(ctx) - launches0
    G.gptq_sync_status(ctx)
    t = sum(times) / len(times)
    tflops_peak, hbm_peak, src = measured_peaks()
    nbytes = m * d // 2 + m * (d // g) * 8 + T * d * 2 + T * m * 4
    flops = 2.0 * T * m * d
    hbm_bound = nbytes / (hbm_peak * 1e9) >= flops / (tflops_peak * 1e12)
    if hbm_bound:
        ach = nbytes / t / 1e9
        roof = {"bound": "hbm", "achieved": ach, "peak": hbm_peak, "unit": "GB/s",
                "frac": ach / hbm_peak, "traffic": None, "peak_source": src}
    else:
        ach = flops / t / 1e12
        roof = {"bound": "tensor", "achieved": ach, "peak": tflops_peak, "unit": "TFLOP/s",
                "frac": ach / tflops_peak, "traffic": None, "peak_source": src}
    line = {"metric": "W4A16 product X W_hat^T from packed 4-bit g128 codes, weights per second",
            "value": m * d / t, "unit": "weights/s", "n_gpus": 1, "steps": args.steps,
            "warmup": max(3, args.warmup), "ms_per_step": t * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16 X, exact (c - z), f32 accumulate",
            "data": "synthetic (random valid codes, seeded)",
            "config": {"workload": f"{args.w4a16} {m}x{d}, T={T} tokens, {args.w4a16_layout} "
                                   "layout", "m": m, "d": d, "T": T, "layout": args.w4a16_layout,
                       "group": g, "l2": "flushed between timed calls (256 MiB write)"},
            "roofline": roof, "clocks": clk, "gpu_launches": launches}
    if not args.no_cpu_baseline:
        sample_s, full_s, desc = oracle_w4a16_sample(m, d, T, 512 if d > 8192 else m)
        line["cpu_baseline"] = {"value": m * d / full_s, "unit": "weights/s",
                                "cores": cores_used(), "kind": "oracle", "sample": desc,
                                "sample_seconds": sample_s}
    print(json.dumps(line), flush=True)
    ctx.close()


def main():
    args = parse()
    if args.w4a16:
        run_w4a16(args)
        return
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
