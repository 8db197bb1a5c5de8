#!/usr/bin/env python
"""GPTQ layer-quantization throughput on B200: weights quantized per second.

One "step" is the whole hot path on the configuration's layers: Hessian accumulation over all
calibration tokens, preparation of R (dead features, damping, factorization), column-wise
quantization with lazy trailing updates, and packing, through the four C-ABI calls.  Inputs
are synthetic and seeded (workloads/synth.py).

Default workload (the largest single-GPU configuration): a 175B-shaped fc2, W 12288 x 49152
fp16 with 0.5 % outlier columns, X = 65,536 calibration tokens (bf16, ReLU of a rank-1024
mixture plus noise) accumulated in 8192-token chunks, 4-bit asymmetric grids per 128 columns,
lazy blocks of 128 (--bits 2 for its 2-bit line).  --config 2 / 3 / 4 time the q_proj, the
act-order down_proj and the 7B decoder block (seven matrices over four shared inputs).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--config C]

With N > 1 every rank quantizes its own independent layer (weak scaling, no data-path
collective); value = all ranks' weights / max-over-ranks time.  Without a launcher's
environment, --gpus N > 1 starts the N ranks itself.  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import os
import socket
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "GPTQ weights quantized/sec per layer (4-bit g128) on 1 B200; % of roofline"
UNIT = "weights/s"

GRID_MODES = {"static": 0, "dynamic": 2}  # the library's grid_given argument


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", type=int, choices=[2, 3, 4, 5], default=5,
                    help="5: 175B fc2 (default); 2: q_proj; 3: act-order down_proj; 4: 7B block")
    ap.add_argument("--bits", type=int, choices=[2, 3, 4], default=0,
                    help="override the configuration's bit width (the fc2's 2-bit line: 2)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-stage-profile", action="store_true",
                    help="skip the extra, untimed step that times every kernel by stage")
    ap.add_argument("--scale", type=float, default=1.0,
                    help="shrink the layers (tests only); the bench line is for 1.0")
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
    ap.add_argument("--probe", choices=["factor", "tail", "hessian"], default=None,
                    help="profiling captures only: run one library call at a chosen size and exit "
                         "(factor: gptq_prepare_hinv on an SPD H of d = --probe-d; tail: that plus "
                         "gptq_quantize_layer of a 12288 x d layer; hessian: one "
                         "gptq_hessian_accumulate of 8192 tokens x d)")
    ap.add_argument("--probe-d", type=int, default=16384)
    return ap.parse_args(argv)


def run_probe(args):
    """One library call at a chosen size, for an ncu capture of its kernels (no timing, no JSON
    line).  Inputs are seeded random data generated on the device."""
    import torch
    import post_weight_quantization_17_b200 as G
    torch.cuda.set_device(0)
    d, dev = args.probe_d, torch.device("cuda")
    g = torch.Generator(device=dev).manual_seed(0)
    if args.probe in ("factor", "tail"):
        A = torch.randn(d, 2 * d, device=dev, generator=g) / (2 * d) ** 0.5
        S = A @ A.T
        del A
        S += 0.1 * torch.eye(d, device=dev)
        ctx = G.Context(m_max=12288, d_max=d, act_order=False)
        R = torch.empty(d, d, device=dev)
        perm = torch.empty(d, dtype=torch.int32, device=dev)
        dead = torch.empty(d, dtype=torch.uint8, device=dev)
        G.gptq_prepare_hinv(ctx, S, 0, 0.01, False, R, perm, dead)
        if args.probe == "tail":
            m = 12288
            W = (torch.randn(m, d, device=dev, generator=g) * 0.01).half()
            b = G.LayerBuffers(m, d, 4, 128, dev, with_factor=False)
            G.gptq_quantize_layer(ctx, W, R, None, dead, 4, 128, 128, 0, b.scales, b.zeros,
                                  b.codes, b.W_hat, b.col_loss)
    else:
        X = torch.randn(8192, d, device=dev, generator=g).to(torch.bfloat16)
        S = torch.empty(d, d, device=dev)
        ctx = G.Context(m_max=8, d_max=d, act_order=False)
        G.gptq_hessian_accumulate(ctx, X, S, 0)
    G.gptq_sync_status(ctx)
    ctx.close()
    torch.cuda.synchronize()
    print(f"probe {args.probe} d={d} done", flush=True)


@dataclasses.dataclass
class Group:
    """One calibration input (one Hessian, one factorization) and the matrices that share it."""
    name: str
    x_spec: object                  # LayerSpec whose d, N and X recipe define the input
    mats: list                      # LayerSpecs quantized with this input's R
    seed: int


def workload(config: int, scale: float = 1.0, n_tokens: int = 0, bits: int = 0, seed: int = 1):
    """The configuration's layer groups (config 4: seven matrices over four inputs)."""
    from workloads.synth import BLOCK7B_SHARED_INPUT, CONFIGS

    def adjust(spec):
        if config != 5:
            # only the fc2 configuration streams its tokens in chunks; the others are one
            # accumulation over all calibration tokens
            spec = dataclasses.replace(spec, chunk=spec.n_tokens)
        if bits:
            spec = dataclasses.replace(spec, bits=bits)
        if scale != 1.0:
            spec = spec.scaled(max(32, int(spec.m * scale)), max(128, int(spec.d * scale)),
                               max(512, int(spec.n_tokens * scale)))
        if n_tokens:
            spec = dataclasses.replace(spec, n_tokens=n_tokens, chunk=min(spec.chunk, n_tokens))
        return spec

    if config == 4:
        specs = {s.name.split("_")[0]: adjust(s) for s in CONFIGS[4]}
        return [Group(g, specs[members[0]], [specs[n] for n in members], 100 * seed + k)
                for k, (g, members) in enumerate(BLOCK7B_SHARED_INPUT.items())]
    spec = adjust(CONFIGS[config][0])
    return [Group(spec.name, spec, [spec], seed)]


def workload_name(config: int, groups) -> str:
    s = groups[0].mats[0]
    if config == 4:
        return (f"7B decoder block: 7 fp16 matrices (q,k,v,o 4096x4096; gate,up 11008x4096; down "
                f"4096x11008) over 4 shared inputs, N={s.n_tokens} bf16 tokens each, "
                f"{s.bits}-bit g{s.group}, block {s.block}")
    kind = {2: "q_proj", 3: "down_proj", 5: "175B fc2"}[config]
    ao = ", act-order" if s.act_order else ""
    return (f"{kind} {s.m}x{s.d} fp16 W, N={s.n_tokens} bf16 tokens in {s.chunk}-token chunks, "
            f"{s.bits}-bit g{s.group}{ao}, block {s.block}")


def workload_config(config, groups, grid="static"):
    s = groups[0].mats[0]
    return {"workload": workload_name(config, groups) +
                        (" (dynamic groups)" if grid == "dynamic" else ""),
            "config": config, "grid": grid,
            "matrices": [[t.m, t.d] for g in groups for t in g.mats],
            "n_tokens": s.n_tokens, "chunk_tokens": s.chunk, "bits": s.bits,
            "group": s.group, "block": s.block, "act_order": s.act_order,
            "weights_per_step": weights_per_step(groups),
            "l2": "flushed between timed steps (256 MiB write); X is larger than L2"}


def weights_per_step(groups) -> int:
    return sum(t.m * t.d for g in groups for t in g.mats)


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
    """Roofline denominators from MEASURED_PEAKS.json (measured on this machine's B200s):
    bf16 TFLOP/s burst and sustained, HBM GB/s; else the recipe's fallback."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return {"bf16": j.get("bf16_tflops", 1590.0),
                "bf16_sustained": j.get("bf16_tflops_sustained", 1400.0),
                "hbm": j.get("hbm_gbs", 6650.0), "source": "measured"}
    return {"bf16": 1590.0, "bf16_sustained": 1400.0, "hbm": 6650.0, "source": "fallback"}


def measure_tf32_peak(device) -> float:
    """Dense TF32 tensor throughput of this GPU, measured the way the bf16 peak was: one cuBLAS
    matmul of 8192^3 in fp32 with TF32 allowed, best of 10, CUDA events (TFLOP/s)."""
    import torch
    n = 8192
    prev = torch.backends.cuda.matmul.allow_tf32
    torch.backends.cuda.matmul.allow_tf32 = True
    try:
        g = torch.Generator(device=device).manual_seed(0)
        a = torch.randn(n, n, device=device, generator=g)
        b = torch.randn(n, n, device=device, generator=g)
        c = torch.empty(n, n, device=device)
        for _ in range(3):
            torch.matmul(a, b, out=c)
        best = float("inf")
        for _ in range(10):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            torch.matmul(a, b, out=c)
            e1.record()
            e1.synchronize()
            best = min(best, e0.elapsed_time(e1))
    finally:
        torch.backends.cuda.matmul.allow_tf32 = prev
    del a, b, c
    torch.cuda.empty_cache()
    return 2.0 * n ** 3 / (best * 1e-3) / 1e12


def measure_tf32_sustained(device, seconds: float = 3.0) -> float:
    """Dense TF32 tensor throughput under the power cap, taken the way the sustained bf16 figure
    was: the same 8192^3 matmul back to back for `seconds`; the rate over the second half."""
    import torch
    n = 8192
    prev = torch.backends.cuda.matmul.allow_tf32
    torch.backends.cuda.matmul.allow_tf32 = True
    try:
        g = torch.Generator(device=device).manual_seed(0)
        a = torch.randn(n, n, device=device, generator=g)
        b = torch.randn(n, n, device=device, generator=g)
        c = torch.empty(n, n, device=device)
        batches, elapsed = [], 0.0
        while elapsed < seconds * 1e3:
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(5):
                torch.matmul(a, b, out=c)
            e1.record()
            e1.synchronize()
            ms = e0.elapsed_time(e1)
            batches.append(ms)
            elapsed += ms
        late = batches[len(batches) // 2:]
    finally:
        torch.backends.cuda.matmul.allow_tf32 = prev
    del a, b, c
    torch.cuda.empty_cache()
    return 5 * len(late) * 2.0 * n ** 3 / (sum(late) * 1e-3) / 1e12


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


def ncu_traffic(key: str, digest: str):
    """DRAM bytes (read + write) per step of a stage's kernels from the committed ncu launch
    list (profiles/ncu_traffic.json, keyed "<stage>@config<k>"), if it was taken on this exact
    kernel source; else None."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        j = json.load(f)
    e = j.get(key)
    if not e or e.get("source_digest") != digest:
        return None
    return e["dram_bytes_per_step"]


def dist_setup(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
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


def weak_scaling_value(world: int, weights: int, per_step_s: float) -> float:
    """Whole-job weights per second: every rank quantizes `weights` weights per step, and the
    job takes as long as its slowest rank."""
    return world * weights / per_step_s


def self_launch(args, argv) -> int:
    """--gpus N > 1 without a launcher: start N ranks of this script with torch.distributed.run
    on this node (rendezvous on 127.0.0.1) and return its exit status."""
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={args.gpus}", "--master-addr=127.0.0.1",
           f"--master-port={port}", os.path.abspath(__file__), *argv]
    return subprocess.call(cmd, cwd=ROOT)


def cores_used():
    """Threads the oracle's numpy BLAS runs with (its parallel part), else the CPUs this process
    may run on."""
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n and max(n) > 0:
            return int(max(n))
    except Exception:
        pass
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count()


# ----------------------------------------------------------------------------- oracle leg
def oracle_instance(W, x_chunks, spec, cols: int, grid: str = "static", layer_d: int = 0):
    """The CPU oracle, timed, on a leading block of one layer: the first `cols` input features
    (columns of W and the matching rows of X) with every row of W and every token given.  W is
    a torch tensor [m, d], x_chunks an iterable of token-major torch chunks [C, d] (any device);
    layer_d: the whole layer's input features, for the description (default spec.d).
    Returns (seconds, weights quantized, description)."""
    import numpy as np
    from oracle import gptq_oracle as O
    Wn = W[:, :cols].float().cpu().double().numpy()
    m = Wn.shape[0]
    t0 = time.perf_counter()
    S = np.zeros((cols, cols))
    n = 0
    for c in x_chunks:
        xc = c[:, :cols].float().cpu().double().numpy()
        S += xc.T @ xc                           # the statistic, chunk by chunk ([T] §9.4)
        n += xc.shape[0]
    H = (2.0 / n) * S
    prep = O.prepare_with_retry(H, spec.percdamp, spec.act_order)
    Wp = Wn.copy()
    Wp[:, prep["dead"]] = 0.0
    Wp = Wp[:, prep["perm"]]
    if grid == "dynamic":
        sc, ze = O.dynamic_grid_arrays(m, cols, spec.group)
        O.gptq_lazy(Wp, prep["R"], sc, ze, np.arange(cols) // spec.group, spec.bits,
                    spec.block, dynamic=spec.group)
    else:
        sc, ze = O.fit_grid(Wn, spec.bits, spec.group)
        gcol = (prep["perm"] // spec.group) if spec.group != -1 else np.zeros(cols, int)
        codes, _, _ = O.gptq_lazy(Wp, prep["R"], sc, ze, gcol, spec.bits, spec.block)
        O.pack(codes, spec.bits)
    dt = time.perf_counter() - t0
    desc = (f"the whole hot path (H over {n} tokens, prepare, lazy-block quantization, pack) on "
            f"the layer's first {cols} of {layer_d or spec.d} input features: {m}x{cols} weights, timed "
            "in full, not extrapolated")
    return dt, m * cols, desc


def baseline_cols(d: int, n_tokens: int) -> int:
    """Leading input features of the CPU baseline's instance: the largest power of two (at most
    d) with n_tokens * cols^2 <= 2.75e11, which keeps the oracle's fp64 Hessian near 5e11 flop
    and the whole instance at about 10-30 s on a 16-core host (2048 columns at 65536 tokens)."""
    if n_tokens * d * d <= 2.75e11:
        return d
    cols = 1
    while cols * 2 <= d and n_tokens * (cols * 2) ** 2 <= 2.75e11:
        cols *= 2
    return min(cols, d)


def run_reference(args):
    """The oracle as it stands on the host cores, one bounded sample of the workload per step:
    the first 512 input features of the configuration's first matrix (all its rows) over its
    first 8192 tokens.  value = the weights of the sample / its measured time."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from workloads.synth import XSource, make_weight
    groups = workload(args.config, args.scale, args.n_tokens, args.bits)
    spec = groups[0].mats[0]
    cols, ntok = min(512, spec.d), min(8192, spec.n_tokens)
    sub = spec.scaled(spec.m, cols, ntok, chunk=ntok)
    W = make_weight(sub, 1, "cpu")
    X = XSource(sub, 1, "cpu").chunk(0)
    for _ in range(args.warmup):
        oracle_instance(W, [X], sub, cols, args.grid, spec.d)
    times = []
    desc, n_w = "", 0
    t_start = time.perf_counter()
    for _ in range(args.steps):
        dt, n_w, desc = oracle_instance(W, [X], sub, cols, args.grid, spec.d)
        times.append(dt)
    wall = time.perf_counter() - t_start
    per = sum(times) / len(times)
    value = n_w / per
    desc = ("a sample of the same recipe per step: " + desc +
            f"; the per-weight cost grows with d and N, so this rate is above the full layer's")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": per * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(args.config, groups, args.grid),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores_used(),
                             "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
            "sample_wall_s": wall}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- our path
_CS = "post_weight_quantization_17_b200/csrc/"
STAGE_KERNEL_FILES = {
    "a1_hessian": [_CS + "k_syrk.cu", _CS + "tc_util.cuh"],
    "a3_factor_gemm": [_CS + "k_factor.cu", _CS + "k_gemm_pair.cu", _CS + "k_gemm_tc.cu",
                       _CS + "gemm_simt.cuh", _CS + "tc_util.cuh", _CS + "tile_upper.h"],
    "a6_update": [_CS + "k_gemm_pair.cu", _CS + "k_gemm_tc.cu", _CS + "tc_util.cuh",
                  _CS + "tile_upper.h"],
}


def peak_regime(clk) -> str:
    """The regime the timed steps ran in, from the clocks sampled over them: "sustained" when the
    power cap held the median SM clock below 90 % of its maximum (the kernels then take the
    sustained peaks: bf16 from the peaks file, TF32 measured the same way), else "burst"."""
    if clk and clk.get("sm_mhz") and clk.get("sm_max_mhz") and \
            clk["sm_mhz"] < 0.9 * clk["sm_max_mhz"]:
        return "sustained"
    return "burst"


def stage_rooflines(groups, stage_ms, kern, peaks, tf32, regime="burst"):
    """Per-stage roofline entries: algorithmic work of the stage (flop or bytes, per step) over
    its time per step, against the peak of the unit that bounds it.  stage_ms: event times of the
    ABI calls in the timed steps; kern: per-stage kernel times of the profiled step (or None).
    3xTF32 stages count fp32-accurate flops against a third of the TF32 peak (three tf32 products
    per fp32-accurate product).  regime "sustained" (the timed steps ran with the power cap
    holding the SM clock down) takes the sustained bf16 figure and a TF32 peak measured the same
    way; "burst" the best-of-10 figures."""
    mats = [t for g in groups for t in g.mats]
    f_syrk = sum(float(g.x_spec.n_tokens) * g.x_spec.d * (g.x_spec.d + 1) for g in groups)
    f_fact = sum(2.0 / 3.0 * float(g.x_spec.d) ** 3 for g in groups)
    f_upd = sum(float(t.m) * t.d * t.d for t in mats)
    b_col = sum(19.0 * t.m * t.d for t in mats)       # W fp16 in, working copy, q, E, codes
    b_grid = sum(2.0 * t.m * t.d + 8.0 * t.m * t.n_groups for t in mats)
    b_pack = sum(t.m * t.d * (1.0 + t.bits / 8.0) for t in mats)
    fp32_peak = tf32 / 3.0
    out = {}

    def tensor(name, flops, ms, peak, src, time_src):
        if not ms:
            return
        ach = flops / (ms * 1e-3) / 1e12
        out[name] = {"bound": "tensor", "work": flops, "work_unit": "flop", "ms_per_step": ms,
                     "achieved": ach, "peak": peak, "unit": "TFLOP/s", "frac": ach / peak,
                     "peak_source": src, "time": time_src}

    def hbm(name, nbytes, ms):
        if not ms:
            return
        ach = nbytes / (ms * 1e-3) / 1e9
        out[name] = {"bound": "hbm", "work": nbytes, "work_unit": "byte", "ms_per_step": ms,
                     "achieved": ach, "peak": peaks["hbm"], "unit": "GB/s",
                     "frac": ach / peaks["hbm"], "peak_source": f"{peaks['source']} copy",
                     "time": "kernel events (profiled step)"}

    if regime == "sustained":
        bf16_peak, bf16_src = peaks["bf16_sustained"], f"{peaks['source']} bf16 sustained"
        tf_src = ("TF32 peak measured live (cuBLAS 8192^3 back to back for 3 s, under the power "
                  "cap) / 3 for 3xTF32")
    else:
        bf16_peak, bf16_src = peaks["bf16"], f"{peaks['source']} bf16 burst"
        tf_src = "TF32 peak measured live (cuBLAS 8192^3, best of 10) / 3 for 3xTF32"
    tensor("a1_hessian", f_syrk, stage_ms.get("hessian"), bf16_peak, bf16_src,
           "ABI-call events (timed steps)")
    tensor("a3_factor", f_fact, stage_ms.get("prepare"), fp32_peak, tf_src,
           "ABI-call events of gptq_prepare_hinv (timed steps; includes a2)")
    if kern:
        k = lambda n: kern.get(n, (0.0, 0))[0]
        tensor("a3_factor_gemm", f_fact, k("factor_gemm"), fp32_peak, tf_src,
               "kernel events (profiled step, run on one stream so that no two launches overlap)")
        tensor("a6_update", f_upd, k("update"), fp32_peak, tf_src, "kernel events (profiled step)")
        hbm("a4_grid", b_grid, k("grid"))
        hbm("a5_column", b_col, k("column"))
        hbm("a8_pack", b_pack, k("pack"))
    return out


def run_ours(args):
    import torch
    import post_weight_quantization_17_b200 as G
    from workloads.synth import XSource, make_weight

    world, rank, local = dist_setup(args)
    seed = rank_seed(rank)
    groups = workload(args.config, args.scale, args.n_tokens, args.bits, seed)
    dev = torch.device("cuda", torch.cuda.current_device())
    peaks = measured_peaks()
    tf32 = measure_tf32_peak(dev)
    stream = torch.cuda.Stream(dev)
    m_max = max(t.m for g in groups for t in g.mats)
    d_max = max(g.x_spec.d for g in groups)
    ao = any(t.act_order for g in groups for t in g.mats)
    ctx = G.Context(m_max=m_max, d_max=d_max, act_order=ao, stream=stream)
    data = []
    for g in groups:
        chunks = list(XSource(g.x_spec, g.seed, dev).chunks())
        Ws = [make_weight(t, g.seed * 10 + k, dev) for k, t in enumerate(g.mats)]
        d = g.x_spec.d
        S = torch.empty(d, d, device=dev)
        R = torch.empty(d, d, device=dev)
        perm = torch.empty(d, dtype=torch.int32, device=dev)
        dead = torch.empty(d, dtype=torch.uint8, device=dev)
        outs = [G.LayerBuffers(t.m, d, t.bits, t.group, dev, with_factor=False)
                for t in g.mats]
        data.append((g, chunks, Ws, S, R, perm, dead, outs))
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    W_total = weights_per_step(groups)
    STAGE_CALLS = ("hessian", "prepare", "quantize", "pack")

    def step(ev=None):
        """One pass of the hot path over every group; ev: per-call event pairs to fill."""
        def mark(name):
            if ev is None:
                return None
            a = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            return (name, a)

        def done(m):
            if m is not None:
                b = torch.cuda.Event(enable_timing=True)
                b.record(stream)
                ev.append((m[0], m[1], b))

        for g, chunks, Ws, S, R, perm, dead, outs in data:
            mk = mark("hessian")
            n = 0
            for xc in chunks:
                n = G.gptq_hessian_accumulate(ctx, xc, S, n)
            done(mk)
            mk = mark("prepare")
            G.gptq_prepare_hinv(ctx, S, n, g.x_spec.percdamp, g.x_spec.act_order, R, perm, dead)
            done(mk)
            for t, W, o in zip(g.mats, Ws, outs):
                mk = mark("quantize")
                G.gptq_quantize_layer(ctx, W, R, perm if t.act_order else None, dead, t.bits,
                                      t.group, t.block, GRID_MODES[args.grid], o.scales, o.zeros,
                                      o.codes, o.W_hat, o.col_loss)
                done(mk)
                mk = mark("pack")
                G.gptq_pack(ctx, o.codes, t.bits, o.packed)
                done(mk)

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
        step_ev, call_ev = [], []
        for _ in range(args.steps):
            flush.zero_()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            step(call_ev)
            b.record(stream)
            step_ev.append((a, b))
        torch.cuda.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        clk = clocks.stop()
        launches = G.gptq_kernel_launches(ctx) - launches0
        G.gptq_sync_status(ctx)
        # one more step, untimed, with every kernel bracketed by events, for the per-stage
        # kernel times (the events serialize the launches, so this step is not a bench value)
        kern = None
        if not args.no_stage_profile:
            flush.zero_()
            G.gptq_timing_enable(ctx, True)
            step()
            kern = G.gptq_timing_read(ctx)
            G.gptq_timing_enable(ctx, False)
            G.gptq_sync_status(ctx)
    step_ms = [a.elapsed_time(b) for a, b in step_ev]
    stage_ms = {k: 0.0 for k in STAGE_CALLS}
    for name, a, b in call_ev:
        stage_ms[name] += a.elapsed_time(b) / args.steps
    total_s = max_over_ranks(sum(step_ms) / 1e3, world)
    per_step_s = total_s / args.steps
    value = weak_scaling_value(world, W_total, per_step_s)

    regime = peak_regime(clk)
    tf32_sus = measure_tf32_sustained(dev) if regime == "sustained" else None
    stages = stage_rooflines(groups, stage_ms, kern, peaks, tf32_sus or tf32, regime)
    # the headline roofline: the stage that takes the longest
    main_name = max((n for n in ("a1_hessian", "a3_factor_gemm", "a6_update") if n in stages),
                    key=lambda n: stages[n]["ms_per_step"], default="a1_hessian")
    roofline = dict(stages.get(main_name, {}))
    if roofline:
        roofline["stage"] = main_name
        roofline["kernel"] = {"a1_hessian": "k_syrk_tc2 (S += X^T X)",
                              "a3_factor_gemm": "k_gemm_pair + k_gemm_tc + k_gemm_small "
                                                "(factorization products)",
                              "a6_update": "k_gemm_pair + k_gemm_tc (lazy trailing updates)"}[
            main_name]
        digest = kernel_source_digest(STAGE_KERNEL_FILES[main_name])
        roofline["source_digest"] = digest
        launches_main = (kern or {}).get({"a1_hessian": "hessian", "a3_factor_gemm": "factor_gemm",
                                          "a6_update": "update"}[main_name], (0, 0))[1]
        roofline["launches_per_step"] = launches_main
        tr = ncu_traffic(f"{main_name}@config{args.config}", digest)
        roofline["traffic"] = tr
        roofline["traffic_per"] = "step" if tr is not None else None

    # end to end through the public API with host buffers (pinned), copies inside the region:
    # X goes up in slabs on a copy stream, double-buffered, each slab's Hessian update running
    # while the next slab is in flight; W goes up behind the slabs; then prepare, quantize, pack,
    # and the packed codes with their grid come back to the host
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, G, ctx, stream, data, world, W_total)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        g0, chunks0, Ws0 = data[0][0], data[0][1], data[0][2]
        cols = baseline_cols(g0.x_spec.d, g0.x_spec.n_tokens)
        dt, nw, desc = oracle_instance(Ws0[0], chunks0, g0.mats[0], cols, args.grid)
        cpu = {"value": nw / dt, "unit": UNIT, "cores": cores_used(), "kind": "oracle",
               "sample": desc, "sample_seconds": dt}

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_step_s * 1e3,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "bf16 products, f32 accumulate/factor/quantize",
                "data": "synthetic (seeded; workloads/synth.py)",
                "config": workload_config(args.config, groups, args.grid),
                "roofline": roofline, "stages": stages,
                "stage_ms_per_step": stage_ms,
                "kernel_ms_profiled_step": {k: v[0] for k, v in (kern or {}).items()},
                "kernel_launches_profiled_step": {k: v[1] for k, v in (kern or {}).items()},
                "tf32_tflops_measured": tf32, "tf32_tflops_sustained_measured": tf32_sus,
                "peak_regime": regime,
                "cpu_baseline": cpu, "e2e": e2e, "clocks": clk,
                "gpu_launches": launches, "gpu_launches_per_step": launches / args.steps,
                "step_ms_min": min(step_ms), "step_ms_max": max(step_ms)}
        print(json.dumps(line), flush=True)
    ctx.close()
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_e2e(args, G, ctx, stream, data, world, W_total):
    import torch
    host = []
    h2d = d2h = 0
    for g, chunks, Ws, S, R, perm, dead, outs in data:
        X_host = [c.cpu().pin_memory() for c in chunks]
        W_host = [W.cpu().pin_memory() for W in Ws]
        o_host = [[torch.empty_like(t, device="cpu").pin_memory()
                   for t in (o.packed, o.scales, o.zeros)] for o in outs]
        h2d += sum(x.numel() * x.element_size() for x in X_host)
        h2d += sum(w.numel() * w.element_size() for w in W_host)
        d2h += sum(t.numel() * t.element_size() for oh in o_host for t in oh)
        host.append((X_host, W_host, o_host))
    dev = stream.device
    slab = max(c.shape[0] for d in data for c in d[1])
    d_max = max(d[0].x_spec.d for d in data)
    xdt = data[0][1][0].dtype
    dbuf = [torch.empty(slab * d_max, dtype=xdt, device=dev) for _ in range(2)]
    copy_stream = torch.cuda.Stream(dev)
    e2e_steps = max(3, min(args.steps, 5))
    with torch.cuda.stream(stream):
        torch.cuda.synchronize()
        barrier(world)
        t_ev = []
        for _ in range(e2e_steps):
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            copy_stream.wait_event(a)
            landed = [torch.cuda.Event(), torch.cuda.Event()]
            free = [torch.cuda.Event(), torch.cuda.Event()]
            k = 0
            for (g, chunks, Ws, S, R, perm, dead, outs), (X_host, W_host, o_host) in zip(data, host):
                d = g.x_spec.d
                n_total = 0
                for xh in X_host:
                    u = k % 2
                    rows = xh.shape[0]
                    buf = dbuf[u][:rows * d].view(rows, d)
                    with torch.cuda.stream(copy_stream):
                        if k >= 2:
                            copy_stream.wait_event(free[u])
                        buf.copy_(xh, non_blocking=True)
                        landed[u].record(copy_stream)
                    stream.wait_event(landed[u])
                    n_total = G.gptq_hessian_accumulate(ctx, buf, S, n_total)
                    free[u].record(stream)
                    k += 1
                # W goes up behind the slabs (it is needed only after the factorization), so the
                # first slab lands as early as it can
                for W, Wh in zip(Ws, W_host):
                    with torch.cuda.stream(copy_stream):
                        W.copy_(Wh, non_blocking=True)
                w_landed = torch.cuda.Event()
                w_landed.record(copy_stream)
                G.gptq_prepare_hinv(ctx, S, n_total, g.x_spec.percdamp, g.x_spec.act_order, R,
                                    perm, dead)
                stream.wait_event(w_landed)
                for t, W, o, oh in zip(g.mats, Ws, outs, o_host):
                    G.gptq_quantize_layer(ctx, W, R, perm if t.act_order else None, dead, t.bits,
                                          t.group, t.block, GRID_MODES[args.grid], o.scales,
                                          o.zeros, o.codes, o.W_hat, o.col_loss)
                    G.gptq_pack(ctx, o.codes, t.bits, o.packed)
                    for hd, dv in zip(oh, (o.packed, o.scales, o.zeros)):
                        hd.copy_(dv, non_blocking=True)
            b.record(stream)
            b.synchronize()
            t_ev.append((a, b))
        barrier(world)
    G.gptq_sync_status(ctx)
    e2e_s = max_over_ranks(sum(a.elapsed_time(b) for a, b in t_ev) / 1e3 / e2e_steps, world)
    return {"value": weak_scaling_value(world, W_total, e2e_s), "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": e2e_s * 1e3, "h2d_slab_tokens": slab, "steps": e2e_steps}


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
    pk = measured_peaks()
    tflops_peak, hbm_peak, src = pk["bf16"], pk["hbm"], pk["source"]
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
    argv = sys.argv[1:]
    args = parse(argv)
    if args.probe:
        run_probe(args)
        return
    if args.w4a16:
        run_w4a16(args)
        return
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        sys.exit(self_launch(args, argv))
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
