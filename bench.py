"""Throughput of the DeltaQuant W4A4 linear layer on B200.

One step = one forward of the whole layer (cube statistics, cube encode,
kernel-token product, main FP4 product with the low-rank slab and the
scatter epilogue) over one synthetic activation tensor X resident in HBM.
Default workload: the Wan-like 720p FFN down-projection (T=21, H=45, W=80,
N=75600 tokens, Ci=13824 -> Co=5120, rank 32, cube 1x2x2), the largest
layer that fits one GPU; --workload picks another.

Prints one JSON line (rank 0).  `value` is whole-job TFLOP/s with
F = 2 N Ci Co + 2 K Ci Co + 2 N r (Ci + Co) (main + kernel-token + low-rank
products, real rows only) per step; tokens/s and the per-stage breakdown are
extra keys.

Several GPUs (one process each, under torchrun): by default ONE layer is
sharded by cubes (slabs of whole cube layers along T, the weight replicated,
one 4-byte NCCL all-reduce(max) of the delta amax between the statistics and
encode stages), so the total work is fixed ("strong" scaling);
--parallelism replicas runs an independent layer per GPU instead ("weak").

--ffn fused|separate times the 720p feed-forward block instead (one GPU): the
up-projection (5120 -> 13824, cube 2x2x2) with GELU in its main product's
epilogue, then the down-projection (13824 -> 5120, cube 1x2x2); `fused` forms the
down-projection's statistics pass in that epilogue, `separate` runs it on its own.

--impl reference times the CPU oracle instead: each step a bounded slice of
the same seeded cube sample as the GPU arm's cpu_baseline, under the delta
scale of a whole-tensor statistics pass.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "W4A4 DeltaQuant linear TFLOPS & tokens/s; % of dense FP4 / HBM roofline"
FP4_PER_BF16 = 4.0  # nominal dense FP4 : BF16 tensor throughput on B200 (9 : 2.25 PFLOP/s)
FP8_PER_BF16 = 2.0  # nominal dense FP8 : BF16 (4.5 : 2.25 PFLOP/s)


def layer_flops(wl, K):
    return 2.0 * wl.N * wl.Ci * wl.Co + 2.0 * K * wl.Ci * wl.Co + 2.0 * wl.N * wl.rank * (wl.Ci + wl.Co)


def stage_model(wl, K, slab, kernel_group=0, fp8=False, pow2=False):
    """Algorithmic work per launch of each stage (bytes that must cross HBM,
    tensor FLOPs).  Stage 1 reads X twice (statistics, then encode: the
    per-tensor delta scale needs every delta first).  fp8: the FP8 kernel-token
    product reads q8 and the FP8 weight (1 byte each) plus one exponent per 32."""
    N, Ci, Co, r = wl.N, wl.Ci, wl.Co, wl.rank
    q8_copy = 0 if fp8 else (4 if kernel_group else 2)   # BF16 operand of the exact product (hi + lo when grouped)
    quant_bytes = ((2.0 if pow2 else 4.0) * N * Ci  # X read by a1 and a2 (once by the single-read quantiser)
                   + (N * Ci / 64 * 2 + N * Ci / 16 * 2 if pow2 else 0.0)  # provisional exponents, scale fix-up
                   + N * Ci / 2 + N * Ci / 16        # delta codes + scales
                   + K * Ci * (1 + q8_copy)          # q8 (E4M3) + the product's BF16 operand
                   + N * r * 4 * 2                   # X L1 partials (write + read)
                   + N * slab * 2 + 2 * r * Ci)      # U hi/lo, L1
    kernel_flops = 2.0 * K * Ci * Co
    if fp8:
        kernel_bytes = K * Ci + Co * Ci + Co * Ci / 32 + K * Co * 4
    else:
        kernel_bytes = K * Ci * (4 if kernel_group else 2) + Co * Ci * 2 + K * Co * 4
    main_flops = 2.0 * N * Ci * Co + 2.0 * N * slab * Co
    main_bytes = N * Ci * 9 / 16 + Co * Ci * 9 / 16 + N * slab * 2 + Co * slab * 2 + K * Co * 4 + N * Co * 2
    return dict(quantize=dict(bytes=quant_bytes, flops=2.0 * N * Ci * r),
                kernel_gemm=dict(bytes=kernel_bytes, flops=kernel_flops),
                main_gemm=dict(bytes=main_bytes, flops=main_flops))


def max_over_ranks(x, dist=None, device="cpu"):
    """The largest of every rank's `x` (one all-reduce that every rank takes part in);
    `x` itself with no process group."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([float(x)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tflops(flops_per_rank_step, world, ms_max):
    """Whole-job throughput under weak scaling: every rank's FLOPs over the slowest rank's step time."""
    return flops_per_rank_step * world / (ms_max * 1e-3) / 1e12


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return dict(hbm=float(d["hbm_gbs"]), bf16=float(d["bf16_tflops"]), source="measured")
    except Exception:
        return dict(hbm=6650.0, bf16=1590.0, source="fallback")


def committed_traffic(wl, stage):
    """DRAM bytes per launch of `stage` from the committed ncu summary, or None
    when the workload differs or the kernel's source has changed since the
    counters were taken."""
    try:
        d = json.load(open(os.path.join(ROOT, "profiles", f"traffic_{wl.name}.json")))
        s = d["stages"][stage]
        if wl.N != s["full_tokens"]:
            return None
        src = open(os.path.join(ROOT, s["source"]), "rb").read()
        if hashlib.sha256(src).hexdigest() != s["source_sha256"]:
            return None
        return float(s["bytes_per_launch"])
    except (OSError, KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "100", "-i", str(self.index)], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return dict(sm_mhz=statistics.median(sm), sm_max_mhz=mx, reasons=sorted(reasons), samples=len(sm))


def parse_cube(s):
    return tuple(int(v) for v in s.split(",")) if s else None


# --------------------------------------------------------------------------- CPU oracle (baseline and reference arm)

SAMPLE_CUBES = 512        # seeded cube sample of the CPU baseline (layers too large for a full oracle run)
SAMPLE_SEED = 0x5A3D
REFERENCE_SLICE = 64      # cubes per reference-arm step (a slice of the same sample)


def oracle_sample_cubes(wl, cube):
    """All cubes for layers the oracle finishes in reasonable time on the whole tensor
    (the tiny case and the 480p projection), else a seeded sample of SAMPLE_CUBES cubes."""
    import oracle
    K = oracle.num_cubes(wl.T, wl.H, wl.W, *cube)
    if wl.name in ("tiny", "wan480p_proj") or K <= SAMPLE_CUBES:
        return np.arange(K, dtype=np.int64), True
    return np.sort(np.random.default_rng(SAMPLE_SEED).choice(K, size=SAMPLE_CUBES, replace=False)), False


class OracleLayer:
    """The oracle's weight side and whole-tensor statistics pass of one workload, and
    timed runs over sets of its cubes."""

    def __init__(self, wl, cube, X, L1, L2, wq, pow2=False):
        import oracle
        self.oracle, self.wl, self.cube, self.X, self.L1, self.L2, self.wq = oracle, wl, cube, X, L1, L2, wq
        t0 = time.perf_counter()
        # S_delta needs the max |delta| of the whole tensor: the oracle's statistics pass over all cubes
        amax = oracle.delta_amax(X, wl.T, wl.H, wl.W, cube)
        self.S = oracle.pow2_scale(amax) if pow2 else oracle.tensor_scale(amax)
        self.stats_s = time.perf_counter() - t0
        self.K = oracle.num_cubes(wl.T, wl.H, wl.W, *cube)
        self.threads = oracle.num_threads()

    def run(self, cubes):
        """Quantise the cubes (means, FP8 kernel tokens, FP4 deltas under S) and compute
        their Y rows in fp64; returns (seconds, tokens)."""
        o, wl = self.oracle, self.wl
        t0 = time.perf_counter()
        sub = o.quantize_cubes(self.X, wl.T, wl.H, wl.W, self.cube, cubes, self.S)
        o.output_rows(sub, self.wq, self.X, self.L1, self.L2, sub["rows"])
        return time.perf_counter() - t0, int(sub["rows"].size)

    def full_seconds(self, sample_s, sample_tokens):
        """Whole-layer oracle time: the statistics pass plus the sample's time scaled by tokens."""
        return self.stats_s + sample_s * self.wl.N / sample_tokens


def bench_config(wl, cube, K, kernel_group, world, parallelism, fp8=False, pow2=False):
    """The `config` object of the JSON line, identical for the GPU arm and the reference arm."""
    return dict(workload=wl.name, T=wl.T, H=wl.H, W=wl.W, N=wl.N, Ci=wl.Ci, Co=wl.Co, rank=wl.rank, cube=list(cube),
                K=K, kernel_scale="per-token" if not kernel_group else f"group{kernel_group}",
                kernel_product="fp8 (restricted-scale C2 weights)" if fp8 else "bf16 (exact)",
                delta_scale="power of two (single read of X)" if pow2 else "amax / 2688 (two reads of X)",
                parallelism=(f"cube-sharded x{world} (T-slabs of whole cube layers, NCCL all-reduce(max) of the "
                             f"delta amax)" if parallelism == "sharded" and world > 1
                             else f"dp{world} (independent layer per GPU)"),
                l2="inputs larger than L2 (X %.0f MB, Y %.0f MB)" % (wl.N * wl.Ci * 2 / 1e6, wl.N * wl.Co * 2 / 1e6))


def run_reference(args, wl, cube):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    oracle.build()
    X = synth.activations(wl)
    Wb = synth.weight(wl)
    L1, L2, _ = oracle.lowrank_factors(Wb, wl.rank)
    fp8 = args.kernel_product == "fp8"
    pow2 = args.delta_scale == "pow2"
    wq = oracle.quantize_weight(Wb, L1, L2, c2=fp8)
    layer = OracleLayer(wl, cube, X, L1, L2, wq, pow2)
    cubes, full = oracle_sample_cubes(wl, cube)
    if wl.name == "tiny":
        slices = [cubes]
    else:
        slices = [cubes[i:i + REFERENCE_SLICE] for i in range(0, cubes.size, REFERENCE_SLICE)]
    for i in range(args.warmup):
        layer.run(slices[i % len(slices)])
    secs, toks = [], []
    for i in range(args.steps):
        dt, n = layer.run(slices[i % len(slices)])
        secs.append(dt)
        toks.append(n)
    sample_s, sample_tok = sum(secs), sum(toks)
    t_full = layer.full_seconds(sample_s, sample_tok)
    K = layer.K
    F = layer_flops(wl, K)
    value = F / t_full / 1e12
    sample = (f"{args.steps} steps over slices of {REFERENCE_SLICE} cubes of a seeded {cubes.size}-cube sample "
              f"({sample_tok} tokens, {sample_s:.1f} s) under the whole tensor's delta scale (statistics pass "
              f"{layer.stats_s:.1f} s); value = whole-layer FLOPs / (statistics pass + sample time x N / sample "
              f"tokens) = {t_full:.0f} s extrapolated")
    line = dict(metric=METRIC, value=value, unit="TFLOP/s", impl="reference", n_gpus=args.gpus, steps=args.steps,
                warmup=args.warmup, ms_per_step=sample_s / args.steps * 1e3, higher_is_better=True,
                scaling="weak" if args.gpus == 1 or args.parallelism == "replicas" else "strong",
                vs_baseline=None, dtype="f64", data="synthetic",
                config=bench_config(wl, cube, K, args.kernel_group, args.gpus, args.parallelism, fp8, pow2),
                tokens_per_s=wl.N / t_full, sample_tflops=sum(layer_flops_rows(wl, K, n) for n in toks) / sample_s / 1e12,
                cpu_baseline=dict(value=value, unit="TFLOP/s", cores=layer.threads, kind="oracle", sample=sample,
                                  sample_seconds=sample_s, extrapolated_full_seconds=t_full),
                e2e=dict(value=value, unit="TFLOP/s", h2d_bytes_per_step=0, d2h_bytes_per_step=0))
    print(json.dumps(line), flush=True)
    return 0


def layer_flops_rows(wl, K, rows):
    """FLOPs of `rows` output rows of the layer, with the kernel-token product counted
    once per cube (K / N of it per row)."""
    return rows * (2.0 * wl.Ci * wl.Co * (1.0 + K / wl.N) + 2.0 * wl.rank * (wl.Ci + wl.Co))


# --------------------------------------------------------------------------- GPU arm

def run_ffn(args):
    """The feed-forward block through dq_ffn_forward: one JSON line with the block's TFLOP/s and the six
    stage times (each layer's quantise, kernel-token product and main product)."""
    import torch
    import video_diffusion_w4a4_b200 as dq
    if int(os.environ.get("WORLD_SIZE", "1")) > 1:
        raise SystemExit("--ffn runs on one GPU")
    up, down = synth.WORKLOADS["wan720p_ffn_up"], synth.WORKLOADS["wan720p_ffn_down"]
    if args.frames:
        shrink = lambda wl: synth.Workload(f"{wl.name}_T{args.frames}", args.frames, wl.H, wl.W, wl.Ci, wl.Co, wl.rank,
                                           wl.cube, (args.frames,) + tuple(wl.grid[1:]), wl.x_outliers, wl.w_outliers,
                                           wl.gelu)
        up, down = shrink(up), shrink(down)
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    X = synth.activations(up)
    fp8 = args.kernel_product == "fp8"
    if fp8:
        # the FP8 kernel-token product in both layers: restricted-scale (C2) weights
        def pack(Wb, r):
            L1f, L2f = dq.dq_lowrank_factors(Wb, r)
            return dq.dq_pack_weight_factors(Wb, L1f, L2f, pack_flags=dq.DQ_PACK_C2)[:3]
    else:
        pack = dq.dq_pack_weight
    pu, L1u, L2u = pack(synth.weight(up), up.rank)
    pd, L1d, L2d = pack(synth.weight(down), down.rank)
    opts = dict(kernel_product=dq.DQ_KERNEL_PRODUCT_FP8 if fp8 else dq.DQ_KERNEL_PRODUCT_BF16)
    t16 = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev)
    Xd, L1u, L2u, L1d, L2d = t16(X), t16(L1u), t16(L2u), t16(L1d), t16(L2d)
    Pu, Pd = torch.from_numpy(pu).to(dev), torch.from_numpy(pd).to(dev)
    Hd = torch.empty((up.N, up.Co), dtype=torch.int16, device=dev)
    Yd = torch.empty((up.N, down.Co), dtype=torch.int16, device=dev)
    lu = dq.dq_workspace_layout_opts(up.T, up.H, up.W, *up.cube, up.Ci, up.Co, up.rank, **opts)
    ld = dq.dq_workspace_layout_opts(down.T, down.H, down.W, *down.cube, down.Ci, down.Co, down.rank, **opts)
    wsu = torch.zeros(lu.total_bytes, dtype=torch.uint8, device=dev)
    wsd = torch.zeros(ld.total_bytes, dtype=torch.uint8, device=dev)
    st = torch.cuda.current_stream(dev)
    flags = 0 if args.ffn == "fused" else dq.DQ_FFN_SEPARATE_STATISTICS
    fused = args.ffn == "fused" and dq.dq_ffn_fused_statistics(up.T, up.H, up.W, up.cube, down.cube)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(8)] for _ in range(args.steps)]
    for row in evs:
        for e in row:
            e.record(st)
    def step(ev=None):
        dq.dq_ffn_forward_opts(Xd, up.T, up.H, up.W, up.cube, down.cube, up.Ci, up.Co, down.Co, up.rank, down.rank,
                               Pu, L1u, L2u, Pd, L1d, L2d, Hd, Yd, wsu, lu.total_bytes, wsd, ld.total_bytes, flags, ev,
                               st, opts_up=opts, opts_down=opts)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    for ws in (wsu, wsd):
        status = dq.dq_read_device_status(ws, st, clear=True)
        if status != 0:
            raise RuntimeError(f"device status after warm-up: {dq.dq_status_string(status)}")
    with ClockSampler(0) as clk:
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record(st)
        for i in range(args.steps):
            step(evs[i])
        end.record(st)
        torch.cuda.synchronize(dev)
    ms = start.elapsed_time(end) / args.steps
    names = ("up_quantize", "up_kernel_gemm", "up_main_gemm_gelu", None, "down_quantize", "down_kernel_gemm",
             "down_main_gemm")
    stage_ms = {n: statistics.mean(evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(args.steps))
                for j, n in enumerate(names) if n}
    Ku, Kd = int(lu.K), int(ld.K)
    F = layer_flops(up, Ku) + layer_flops(down, Kd)
    peaks = load_peaks()
    fp4_peak = peaks["bf16"] * FP4_PER_BF16
    mu, md = stage_model(up, Ku, lu.slab, fp8=fp8), stage_model(down, Kd, ld.slab, fp8=fp8)
    dom = max(("up_main_gemm_gelu", "down_main_gemm"), key=stage_ms.get)
    m = mu if dom.startswith("up") else md
    ach = m["main_gemm"]["flops"] / (stage_ms[dom] * 1e-3) / 1e12
    line = dict(metric=METRIC, value=F / (ms * 1e-3) / 1e12, unit="TFLOP/s", n_gpus=1, steps=args.steps,
                warmup=args.warmup, ms_per_step=ms, higher_is_better=True, scaling="weak", vs_baseline=None,
                dtype="e2m1/e4m3->f32", data="synthetic",
                config=dict(workload="wan720p_ffn_block" + (f"_T{args.frames}" if args.frames else ""), T=up.T, H=up.H,
                            W=up.W, N=up.N, Ci=up.Ci, Cf=up.Co, Co=down.Co, rank=[up.rank, down.rank],
                            cube_up=list(up.cube), cube_down=list(down.cube), activation="GELU (erf form) in the "
                            "up-projection's main-product epilogue",
                            kernel_product="fp8 (restricted-scale C2 weights)" if fp8 else "bf16 (exact)",
                            down_statistics=("formed in the up-projection's epilogue (the down-projection runs "
                                             "no statistics pass; its encode pass forms X L1)" if fused
                                             else "separate pass"),
                            l2="inputs larger than L2"),
                tokens_per_s=up.N / (ms * 1e-3), stages={n: dict(ms=v) for n, v in stage_ms.items()},
                roofline=dict(kernel="k_gemm<3> (main FP4 product, feed-forward epilogue)" if dom.startswith("up")
                              else "k_gemm<1> (main FP4 product)", bound="tensor", achieved=ach, peak=fp4_peak,
                              unit="TFLOP/s", frac=ach / fp4_peak, traffic=None,
                              peak_source=peaks["source"] + " bf16 x 4 (nominal FP4:BF16)"),
                e2e=None, gpu_launches=8 * args.steps)
    clk_sum = clk.summary()
    if clk_sum:
        line["clocks"] = clk_sum
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="dq", choices=["dq", "reference"])
    ap.add_argument("--workload", default="wan720p_ffn_down", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--cube", default=None, help="override the cube, e.g. 2,2,2")
    ap.add_argument("--frames", type=int, default=None, help="override T (smaller cases for profiling)")
    ap.add_argument("--kernel-group", type=int, default=0, choices=[0, 64],
                    help="FP8 kernel-token scales: 0 = one per token, 64 = one per 64 channels")
    ap.add_argument("--kernel-product", default="bf16", choices=["bf16", "fp8"],
                    help="kernel-token product: exact BF16 operands (default) or FP8 on restricted-scale (C2) weights")
    ap.add_argument("--delta-scale", default="amax", choices=["amax", "pow2"],
                    help="per-tensor delta scale: amax / 2688 (default, two reads of X) or its power of two "
                         "(single-read quantiser)")
    ap.add_argument("--parallelism", default="sharded", choices=["sharded", "replicas"],
                    help="with several GPUs: one layer sharded by cubes (default) or one layer per GPU")
    ap.add_argument("--ffn", default=None, choices=["fused", "separate"],
                    help="time the 720p feed-forward block (up-projection + GELU + down-projection) instead, with the "
                         "down-projection's statistics fused into the up-projection's epilogue or as their own pass")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=5)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    wl = synth.WORKLOADS[args.workload]
    cube = parse_cube(args.cube) or wl.cube
    wl = wl.with_cube(cube)
    if args.frames:
        wl = synth.Workload(wl.name if args.frames == wl.T else f"{wl.name}_T{args.frames}", args.frames, wl.H, wl.W,
                            wl.Ci, wl.Co, wl.rank, cube, (args.frames,) + tuple(wl.grid[1:]), wl.x_outliers,
                            wl.w_outliers, wl.gelu)
    if args.impl == "reference":
        return run_reference(args, wl, cube)
    if args.ffn:
        return run_ffn(args)

    import torch
    import video_diffusion_w4a4_b200 as dq
    from video_diffusion_w4a4_b200 import shard

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    sharded = world > 1 and args.parallelism == "sharded"
    kg = args.kernel_group
    fp8 = args.kernel_product == "fp8"
    kp = dq.DQ_KERNEL_PRODUCT_FP8 if fp8 else dq.DQ_KERNEL_PRODUCT_BF16
    pow2 = args.delta_scale == "pow2"
    ds = dq.DQ_DELTA_SCALE_POW2 if pow2 else dq.DQ_DELTA_SCALE_AMAX
    if pow2 and kg:
        ap.error("the single-read quantiser takes per-token kernel scales")
    if sharded and (kg or fp8 or pow2):
        ap.error("the cube-sharded layer takes the default options")
    if fp8 and kg:
        ap.error("the FP8 kernel-token product takes per-token kernel scales")

    t, h, w = cube
    K = dq.dq_cube_count(wl.T, wl.H, wl.W, t, h, w)
    # inputs: replicas give each rank its own activation tensor (a different denoising step);
    # the sharded layer gives every rank the same tensor, of which it keeps its slab of frames
    X = synth.activations(wl, tau=0 if sharded else rank)
    Wb = synth.weight(wl)
    t0 = time.perf_counter()
    if fp8:
        L1f, L2f = dq.dq_lowrank_factors(Wb, wl.rank)
        packed, L1m, L2s, _ = dq.dq_pack_weight_factors(Wb, L1f, L2f, pack_flags=dq.DQ_PACK_C2)
    else:
        packed, L1m, L2s = dq.dq_pack_weight(Wb, wl.rank)
    pack_s = time.perf_counter() - t0
    if sharded:
        f0, f1 = shard.slab_frames(wl.T, t, world, rank)
        Ts = f1 - f0
        ts, hs, ws_ = shard.slab_cube(cube, Ts)
        X_mine = X[f0 * wl.H * wl.W:f1 * wl.H * wl.W]
    else:
        Ts, (ts, hs, ws_), X_mine = wl.T, cube, X
    Nm = Ts * wl.H * wl.W
    Xd = torch.from_numpy(X_mine.view(np.int16)).to(dev)
    Pd = torch.from_numpy(packed).to(dev)
    L1d = torch.from_numpy(L1m.view(np.int16)).to(dev)
    L2d = torch.from_numpy(L2s.view(np.int16)).to(dev)
    Yd = torch.empty((Nm, wl.Co), dtype=torch.int16, device=dev)
    lay = dq.dq_workspace_layout_opts(Ts, wl.H, wl.W, ts, hs, ws_, wl.Ci, wl.Co, wl.rank, kernel_group=kg,
                                      kernel_product=kp, delta_scale=ds)
    ws = torch.zeros(lay.total_bytes, dtype=torch.uint8, device=dev)
    st = torch.cuda.current_stream(dev)

    def allreduce_max(a):
        dist.all_reduce(a, op=dist.ReduceOp.MAX)

    def step(events=None, pre=None):
        if not sharded:
            dq.dq_linear_forward_opts(Xd, Ts, wl.H, wl.W, ts, hs, ws_, wl.Ci, wl.Co, wl.rank, Pd, L1d, L2d, Yd, ws,
                                      lay.total_bytes, dq.DQ_STAGE_ALL, events, st, kernel_group=kg, kernel_product=kp,
                                      delta_scale=ds)
            return
        # the cube-sharded layer: statistics of this slab, the one exchanged scalar (NCCL), then
        # encode and both products
        shard.forward_sharded(Xd, Ts, wl.H, wl.W, cube, wl.Ci, wl.Co, wl.rank, Pd, L1d, L2d, Yd, ws, allreduce_max,
                              st, events, pre)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    status = dq.dq_read_device_status(ws, st, clear=True)
    if status != 0:
        raise RuntimeError(f"device status after warm-up: {dq.dq_status_string(status)}")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    for row in evs:          # torch creates CUDA events lazily; create them before handing them to the library
        for e in row:
            e.record(st)
    if dist:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        start.record(st)
        for i in range(args.steps):
            step(evs[i][1:], evs[i][0])
        end.record(st)
        torch.cuda.synchronize(dev)
    if dist:
        dist.barrier()
    ms = start.elapsed_time(end) / args.steps
    stage_ms = {n: statistics.mean(evs[i][j + 1].elapsed_time(evs[i][j + 2]) for i in range(args.steps))
                for j, n in enumerate(("quantize", "kernel_gemm", "main_gemm"))}
    if sharded:
        # statistics pass + all-reduce, before the encode stage's first event; the quantise stage
        # below counts both halves (statistics, all-reduce and encode)
        stage_ms["stats_allreduce"] = statistics.mean(evs[i][0].elapsed_time(evs[i][1]) for i in range(args.steps))
        stage_ms["quantize"] += stage_ms["stats_allreduce"]
    status = dq.dq_read_device_status(ws, st, clear=True)
    if status != 0:
        raise RuntimeError(f"device status after timing: {dq.dq_status_string(status)}")
    ms = max_over_ranks(ms, dist, dev)

    # end to end through the public API with host buffers: pinned X in, Y out, copies inside the timed region
    Xh = torch.from_numpy(X_mine.view(np.int16)).pin_memory()
    Yh = torch.empty((Nm, wl.Co), dtype=torch.int16).pin_memory()
    Xd2, Yd2 = torch.empty_like(Xd), torch.empty_like(Yd)

    def e2e_step(overlap=True):
        if not sharded:
            # each step's copy of X in may overlap the previous step's products and copy of Y out
            dq.dq_linear_forward_host_ex(Xh, Ts, wl.H, wl.W, ts, hs, ws_, wl.Ci, wl.Co, wl.rank, Pd, L1d, L2d, Yh,
                                         Xd2, Yd2, ws, lay.total_bytes,
                                         dq.DQ_HOST_OVERLAP_PREVIOUS if overlap else 0, st)
            return
        Xd2.copy_(Xh, non_blocking=True)
        shard.forward_sharded(Xd2, Ts, wl.H, wl.W, cube, wl.Ci, wl.Co, wl.rank, Pd, L1d, L2d, Yd2, ws, allreduce_max,
                              st)
        Yh.copy_(Yd2, non_blocking=True)

    e2e_ms = None
    if not kg and not fp8 and not pow2:   # the host-buffer entry point takes the default options
        e2e_step()
        torch.cuda.synchronize(dev)
        if dist:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(st)
        for i in range(args.e2e_steps):
            e2e_step(overlap=i > 0)   # the first timed copy waits for the start event
        e1.record(st)
        torch.cuda.synchronize(dev)
        e2e_ms = e0.elapsed_time(e1) / args.e2e_steps
    if dist and e2e_ms is not None:
        e2e_ms = max_over_ranks(e2e_ms, dist, dev)
        dist.barrier()

    F = layer_flops(wl, K)
    # whole-job FLOPs per step: the one layer (sharded) or one layer per GPU (replicas)
    value = (F / (ms * 1e-3) / 1e12) if sharded else job_tflops(F, world, ms)
    peaks = load_peaks()
    fp4_peak = peaks["bf16"] * FP4_PER_BF16
    # per-stage work model of this rank's share (its slab when sharded)
    wl_mine = wl if not sharded else synth.Workload(wl.name, Ts, wl.H, wl.W, wl.Ci, wl.Co, wl.rank, (ts, hs, ws_),
                                                    wl.grid, wl.x_outliers, wl.w_outliers, wl.gelu)
    model = stage_model(wl_mine, int(lay.K), lay.slab, kg, fp8, pow2)
    # dominant kernel = the stage with the largest share of the step
    dom = max(("quantize", "kernel_gemm", "main_gemm"), key=stage_ms.get)
    if dom == "quantize":
        ach = model[dom]["bytes"] / (stage_ms[dom] * 1e-3) / 1e9
        roof = dict(kernel="k_cube_stats<.,.>+k_cube_encode", bound="hbm", achieved=ach, peak=peaks["hbm"], unit="GB/s")
    else:
        # the kernel-token product's own kind: BF16, or FP8 at 2 x the BF16 rate (nominal 4.5 : 2.25)
        pk = fp4_peak if dom == "main_gemm" else peaks["bf16"] * (FP8_PER_BF16 if fp8 else 1.0)
        ach = model[dom]["flops"] / (stage_ms[dom] * 1e-3) / 1e12
        roof = dict(kernel="k_gemm<1> (main FP4 product)" if dom == "main_gemm" else
                    ("k_gemm<2> (FP8 kernel-token product)" if fp8 else "k_gemm<0> (kernel-token product)"),
                    bound="tensor", achieved=ach, peak=pk, unit="TFLOP/s")
    roof["frac"] = roof["achieved"] / roof["peak"]
    same_cube = tuple(cube) == tuple(synth.WORKLOADS[args.workload].cube)
    roof["traffic"] = committed_traffic(wl_mine, dom) if same_cube and not kg and not fp8 and not pow2 else None
    roof["peak_source"] = ("measured" if peaks["source"] == "measured" else "fallback") + (
        " bf16 x 4 (nominal FP4:BF16)" if roof["unit"] == "TFLOP/s" and dom == "main_gemm" else
        " bf16 x 2 (nominal FP8:BF16)" if roof["unit"] == "TFLOP/s" and fp8 else "")
    stages = {}
    for n, tms in stage_ms.items():
        if n not in model:
            stages[n] = dict(ms=tms)
            continue
        m = model[n]
        stages[n] = dict(ms=tms, tflops=m["flops"] / (tms * 1e-3) / 1e12, gbs=m["bytes"] / (tms * 1e-3) / 1e9)
    stages["quantize"]["frac_hbm"] = stages["quantize"]["gbs"] / peaks["hbm"]
    stages["kernel_gemm"]["frac_bf16"] = stages["kernel_gemm"]["tflops"] / peaks["bf16"]
    if fp8:
        stages["kernel_gemm"]["frac_fp8"] = stages["kernel_gemm"]["tflops"] / (peaks["bf16"] * FP8_PER_BF16)
    stages["main_gemm"]["frac_fp4"] = stages["main_gemm"]["tflops"] / fp4_peak
    layer_bytes = sum(m["bytes"] for m in model.values())
    F_mine = layer_flops(wl_mine, int(lay.K))
    layer_roof_ms = max(F_mine / (fp4_peak * 1e12), layer_bytes / (peaks["hbm"] * 1e9)) * 1e3
    launches = (5 if t * h * w > 128 else 4)
    line = dict(metric=METRIC, value=value, unit="TFLOP/s", n_gpus=world, steps=args.steps, warmup=args.warmup,
                ms_per_step=ms, higher_is_better=True, scaling="strong" if sharded else "weak", vs_baseline=None,
                dtype="e2m1/e4m3->f32", data="synthetic",
                config=bench_config(wl, cube, K, kg, world, args.parallelism, fp8, pow2),
                tokens_per_s=wl.N * (1 if sharded else world) / (ms * 1e-3),
                layer_roofline_frac=layer_roof_ms / ms,
                roofline=roof, stages=stages,
                e2e=None if e2e_ms is None else dict(
                    value=(F / (e2e_ms * 1e-3) / 1e12) if sharded else job_tflops(F, world, e2e_ms), unit="TFLOP/s",
                    h2d_bytes_per_step=Nm * wl.Ci * 2, d2h_bytes_per_step=Nm * wl.Co * 2, ms_per_step=e2e_ms),
                gpu_launches=launches * args.steps, pack_seconds=pack_s)
    if sharded:
        line["shard"] = dict(frames=[f0, f1], tokens=Nm, cubes=int(lay.K))
    clk_sum = clk.summary()
    if clk_sum:
        line["clocks"] = clk_sum
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # the oracle on the machine's host cores: the whole tensor for the small layers, else a seeded
        # sample of whole cubes under the whole tensor's delta scale, extrapolated by tokens
        import oracle
        oracle.build()
        L1, L2 = dq.dq_lowrank_factors(Wb, wl.rank)
        wq = oracle.quantize_weight(Wb, L1, L2, c2=fp8)
        layer = OracleLayer(wl, cube, X, L1, L2, wq, pow2)
        cubes, full = oracle_sample_cubes(wl, cube)
        dt, n = layer.run(cubes)
        t_full = dt if full else layer.full_seconds(dt, n)
        if full:
            t_full += layer.stats_s
        what = (f"the whole tensor ({n} tokens, {dt + layer.stats_s:.1f} s)" if full else
                f"a seeded {cubes.size}-cube sample ({n} tokens, {dt:.1f} s) under the whole tensor's delta scale "
                f"(statistics pass {layer.stats_s:.1f} s), extrapolated by tokens to {t_full:.0f} s for the layer")
        line["cpu_baseline"] = dict(value=F / t_full / 1e12, unit="TFLOP/s", cores=layer.threads, kind="oracle",
                                    sample=f"oracle over {what}; {wl.name}, Ci={wl.Ci}, Co={wl.Co}, r={wl.rank}",
                                    sample_seconds=dt, extrapolated_full_seconds=None if full else t_full)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
