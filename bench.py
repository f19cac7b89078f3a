"""Benchmark of the ConvRot int8 linear layer on B200.

One step = the int8-compute forward (rotate + per-token int8 quantize, int8
GEMM with the fused rescale/bias epilogue) of every linear of the workload, on
inputs resident in HBM.  The headline value is int8 linear TOPS,
sum(2 M N K) / step time.  The default path's weight decode (dequantize +
derotate) of the same weights is timed in the same run and reported under
"derotate".

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...   # the CPU oracle on the host cores

Multi-GPU runs (torchrun, one process per GPU) are weak-scaled replicas: each
rank runs the whole workload on its own tokens; the layer needs no exchange, so
there is no collective on the data path.  Time is the max over ranks.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

MEASURED_PEAKS = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
INT8_PER_BF16 = 2.0  # nominal dense int8 : bf16 tensor throughput (4.5 : 2.25 POPS)

# DRAM bytes per launch from ncu (dram__bytes_read.sum + dram__bytes_write.sum),
# averaged over the GEMM launches of one step of a workload, valid only for the
# kernel source they were taken on (first 16 hex digits of its sha256).
NCU_TRAFFIC = {
    ("int8_gemm_tcgen05", "zimage_dit_block"): ((62.16e6 + 69.42e6) + (57.17e6 + 54.22e6) + (143.70e6 + 21.10e6)) / 3,
    ("int8_gemm_tcgen05", "wan22_a14b_video_dit"):
        ((187.12e6 + 217.64e6) + (173.47e6 + 193.75e6) + (565.78e6 + 70.48e6)) / 3,
}
NCU_TRAFFIC_SOURCE_SHA = {
    ("int8_gemm_tcgen05", "zimage_dit_block"): "15eac4e6bc70d2f3",
    ("int8_gemm_tcgen05", "wan22_a14b_video_dit"): "15eac4e6bc70d2f3",
}


def source_sha(rel: str) -> str:
    with open(os.path.join(ROOT, rel), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def load_peaks():
    try:
        with open(MEASURED_PEAKS) as f:
            p = json.load(f)
        return (float(p["hbm_gbs"]), float(p["bf16_tflops"]),
                float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), "measured")
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.1)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        rows = []
        try:
            with open(self.path) as f:
                for line in f:
                    parts = [p.strip() for p in line.split(",")]
                    if len(parts) >= 9:
                        rows.append(parts)
        except Exception:
            pass
        finally:
            if self.path and os.path.exists(self.path):
                os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        def num(v):
            try:
                return float(v)
            except ValueError:
                return None
        # samples under load: power draw in the upper half between the lowest
        # and highest draw seen (the idle samples around the region drop out)
        power = [num(r[3]) for r in rows]
        known = [w for w in power if w is not None]
        cut = (min(known) + max(known)) / 2 if known and max(known) - min(known) > 50 else None
        loaded = [r for r, w in zip(rows, power) if cut is None or (w is not None and w >= cut)]
        sm = [num(r[1]) for r in loaded if num(r[1]) is not None]
        mx = [num(r[2]) for r in rows if num(r[2]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows), "samples_under_load": len(loaded),
                "max_power_w": max(known) if known else None}


# ---------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------
def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and n_gpus != world:
        raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE={world}")
    return world, rank, local


def init_pg(world: int, backend: str):
    import datetime

    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return dist


def max_over_ranks(value: float, world: int, device) -> float:
    """The largest `value` over all ranks (host-side timing plumbing)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_throughput(ops_per_rank_step: float, steps: int, local_ms: float, world: int,
                            device) -> tuple[float, float]:
    """Whole-job throughput of weak-scaled replicas: every rank processed
    `steps` steps of `ops_per_rank_step` operations; the job took as long as the
    slowest rank.  Returns (TOP/s, max-over-ranks milliseconds)."""
    total_ms = max_over_ranks(local_ms, world, device)
    return ops_per_rank_step * steps * world / (total_ms * 1e-3) / 1e12, total_ms


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------------------
# CPU baseline: the oracle on a bounded sample of the same workload
# ---------------------------------------------------------------------------
def oracle_sample_rate(lins, rows_per_linear: int, budget_s: float):
    """int8 linear TOPS of the oracle (rotate+quantize, GEMM, epilogue) on
    `rows_per_linear` tokens of each linear, repeated until `budget_s`."""
    import oracle
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = os.cpu_count() or 1
    prepared = []
    for i, lin in enumerate(lins):
        inp = workloads.make_layer_inputs(lin, 1, M=rows_per_linear)
        Wq, s_w = oracle.quantize_weight(inp.W, inp.R)
        prepared.append((lin, inp, Wq, s_w))
    ops = 0.0
    t0 = time.perf_counter()
    reps = 0
    while True:
        for lin, inp, Wq, s_w in prepared:
            oracle.linear_int8(inp.x, Wq, s_w, inp.R, inp.bias)
            ops += 2.0 * rows_per_linear * lin.N * lin.K
        reps += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    return ops / dt / 1e12, cores, dt, reps


def run_reference(args, lins):
    world, rank, local = dist_setup(args.gpus)
    if rank != 0:
        return 0
    rows = args.ref_rows
    step_s = []
    rates = []
    cores = 1
    for k in range(args.warmup + args.steps):
        tops, cores, dt, _ = oracle_sample_rate(lins, rows, budget_s=0.0)
        if k >= args.warmup:
            step_s.append(dt)
            rates.append(tops)
    value = statistics.mean(rates)
    sample = (f"{rows} tokens of each of the {len(lins)} linears of {args.workload} "
              f"per step (rotate+quantize, int8 GEMM, epilogue; float64 numpy)")
    line = {
        "impl": "reference", "metric": "int8 ConvRot linear TOPS (rotate+quant+GEMM)",
        "value": value, "unit": "TOPS", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * statistics.mean(step_s),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_dict(args, lins, gpu=False),
        "cpu_baseline": {"value": value, "unit": "TOPS", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TOPS", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


def config_dict(args, lins, gpu=True):
    cfg = {
        "workload": args.workload,
        "linears": [f"{l.name}:M{l.M}xK{l.K}->N{l.N}" for l in lins],
        "G": lins[0].G, "rotation": "sylvester-hadamard",
        "activations": getattr(args, "dtype", "bf16"),
    }
    if gpu:
        cfg.update({
            "l2": "flushed between timed steps (256 MiB write + 256 MiB read, untimed)",
            "launch": "each step enqueued behind a 0.2 ms GPU spin, so host launch gaps are not timed",
            "timing": "step: CUDA events at step start and end only (kernels chained as in use); "
                      "per-kernel times and the roofline: an extra step after each timed step, "
                      "with events between kernels",
        })
    return cfg


# ---------------------------------------------------------------------------
# the GPU arm
# ---------------------------------------------------------------------------
def run_ours(args, lins):
    import torch

    world, rank, local = dist_setup(args.gpus)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    init_pg(world, "nccl")
    import activation_quantized_linear_b200 as cr

    hbm_gbs, bf16_tflops, bf16_sust, peak_src = load_peaks()
    int8_peak = bf16_tflops * INT8_PER_BF16

    rot = cr.Rotation(workloads.sylvester_rotation(lins[0].G))
    layers = []
    for i, lin in enumerate(lins):
        act = torch.float16 if args.dtype == "f16" else torch.bfloat16
        inp = workloads.make_layer_inputs(lin, 1 + rank, dtype=act)  # every rank its own tokens
        W = inp.W.to(dev)
        Wq, s_w = cr.quantize_weight(W, rot)
        del W
        layers.append(dict(
            lin=lin, x=inp.x.to(dev), x_host=inp.x.pin_memory(), Wq=Wq, s_w=s_w,
            bias=inp.bias.to(dev),
            xq=torch.empty((lin.M, lin.K), dtype=torch.int8, device=dev),
            s_tok=torch.empty(lin.M, dtype=torch.float32, device=dev),
            y=torch.empty((lin.M, lin.N), dtype=act, device=dev),
            y_host=torch.empty((lin.M, lin.N), dtype=act).pin_memory(),
            W_hat=torch.empty((lin.N, lin.K), dtype=act, device=dev),
            ws=torch.empty(cr.workspace_bytes(lin.M, lin.N, lin.K), dtype=torch.uint8,
                           device=dev),
        ))
    # L2 flush between timed steps: write 256 MiB (evicts everything), then read
    # another 256 MiB so that the dirty flush lines are written back before the
    # next step starts rather than during its first kernel.
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flush_rd = torch.ones(64 << 20, dtype=torch.float32, device=dev)

    def flush_l2(k):
        flush.fill_(k & 0xFF)
        flush_rd.sum()
        # Hold the GPU for ~0.2 ms so the host enqueues the whole step before
        # the first timed kernel starts: the events then time the kernels, not
        # the host's per-launch overhead.
        torch.cuda._sleep(400_000)
    stream = torch.cuda.current_stream()
    n_lin = len(layers)

    def ev():
        return torch.cuda.Event(enable_timing=True)

    def step(record=None):
        """One pass of the hot path; with `record`, events between the kernels."""
        for i, L in enumerate(layers):
            if record:
                record[i][0].record(stream)
            cr.rotate_quant_act(L["x"], rot, xq=L["xq"], s_tok=L["s_tok"])
            if record:
                record[i][1].record(stream)
            cr.int8_gemm(L["xq"], L["s_tok"], L["Wq"], L["s_w"], L["bias"], out=L["y"])
            if record:
                record[i][2].record(stream)

    # ---------------- warm-up
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    cr.check_status()

    # ---------------- timed: int8-compute forward.  Each timed step is
    # bracketed by two events only, so consecutive kernels overlap as they do
    # in use; every timed step is followed by a breakdown step with events
    # between the kernels (same clocks and power state), whose per-kernel
    # times give the roofline.
    steps_ev = [(ev(), ev()) for _ in range(args.steps)]
    recs = [[(ev(), ev(), ev()) for _ in range(n_lin)] for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        for k in range(args.steps):
            flush_l2(2 * k)
            steps_ev[k][0].record(stream)
            step()
            steps_ev[k][1].record(stream)
            flush_l2(2 * k + 1)
            step(recs[k])
        torch.cuda.synchronize()
    barrier(world)
    cr.check_status()
    clk = clocks.summary()

    rqa_ms = np.array([[r[i][0].elapsed_time(r[i][1]) for i in range(n_lin)] for r in recs])
    gemm_ms = np.array([[r[i][1].elapsed_time(r[i][2]) for i in range(n_lin)] for r in recs])
    step_ms = np.array([e0.elapsed_time(e1) for e0, e1 in steps_ev])
    ops_step = sum(2.0 * L["lin"].M * L["lin"].N * L["lin"].K for L in layers)
    value, total_ms = weak_scaling_throughput(ops_step, args.steps, float(step_ms.sum()), world, dev)

    gemm_mean = gemm_ms.mean(axis=0)
    gemm_ops = np.array([2.0 * L["lin"].M * L["lin"].N * L["lin"].K for L in layers])
    gemm_tops = float(gemm_ops.sum() / (gemm_mean.sum() * 1e-3) / 1e12)
    rqa_mean = rqa_ms.mean(axis=0)
    rqa_bytes = np.array([3.0 * L["lin"].M * L["lin"].K + 4.0 * L["lin"].M for L in layers])
    rqa_gbs = float(rqa_bytes.sum() / (rqa_mean.sum() * 1e-3) / 1e9)

    gemm_src = "activation_quantized_linear_b200/csrc/int8_gemm.cu"
    traffic = None
    key = ("int8_gemm_tcgen05", args.workload)
    if NCU_TRAFFIC.get(key) and NCU_TRAFFIC_SOURCE_SHA.get(key) == source_sha(gemm_src):
        traffic = NCU_TRAFFIC[key]

    # ---------------- timed: default-path weight decode (dequant + derotate)
    drecs = [[(ev(), ev()) for _ in range(n_lin)] for _ in range(args.steps)]
    for L in layers:
        cr.dequant_derotate(L["Wq"], L["s_w"], rot, out=L["W_hat"])
    torch.cuda.synchronize()
    for k in range(args.steps):
        flush_l2(k)
        for i, L in enumerate(layers):
            drecs[k][i][0].record(stream)
            cr.dequant_derotate(L["Wq"], L["s_w"], rot, out=L["W_hat"])
            drecs[k][i][1].record(stream)
    torch.cuda.synchronize()
    der_ms = np.array([[r[i][0].elapsed_time(r[i][1]) for i in range(n_lin)] for r in drecs])
    der_bytes = np.array([3.0 * L["lin"].N * L["lin"].K for L in layers])
    der_gbs = float(der_bytes.sum() / (der_ms.mean(axis=0).sum() * 1e-3) / 1e9)

    # ---------------- end to end through the public API with host buffers.
    # Per linear: pinned x -> device on an upload stream, convrot_linear_int8
    # on the compute stream once x has landed, y -> pinned host on a download
    # stream once it is computed; uploads, compute and downloads of
    # consecutive linears overlap (the copy engines run both directions).
    h2d = sum(L["x_host"].numel() * 2 for L in layers)
    d2h = sum(L["y_host"].numel() * 2 for L in layers)
    up, down = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    e2e_ms = []
    for k in range(max(2, min(args.steps, 5)) + 1):
        flush_l2(k)
        e0, e1 = ev(), ev()
        e0.record(stream)
        up.wait_stream(stream)
        down.wait_stream(stream)
        for L in layers:
            with torch.cuda.stream(up):
                L["x"].copy_(L["x_host"], non_blocking=True)
            stream.wait_stream(up)
            cr.linear_int8(L["x"], L["Wq"], L["s_w"], rot, L["bias"], out=L["y"], workspace=L["ws"])
            down.wait_stream(stream)
            with torch.cuda.stream(down):
                L["y_host"].copy_(L["y"], non_blocking=True)
        stream.wait_stream(down)
        e1.record(stream)
        torch.cuda.synchronize()
        if k:  # first pass warms the pinned-copy path
            e2e_ms.append(e0.elapsed_time(e1))
    e2e_value, e2e_total = weak_scaling_throughput(ops_step, 1, float(np.mean(e2e_ms)), world, dev)

    if rank != 0:
        return 0
    tops_frac = gemm_tops / int8_peak
    # the tensor cores' own int8 rate on this GPU (after the timed region):
    # context for the denominator, which stays the measured bf16 rate x 2
    issue_tops = issue_loop_tops()
    out = {
        "metric": "int8 ConvRot linear TOPS (rotate+quant+GEMM)",
        "value": value, "unit": "TOPS", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int8", "data": "synthetic", "config": config_dict(args, lins),
        "roofline": {
            "kernel": "int8_gemm_tcgen05", "bound": "tensor", "achieved": gemm_tops,
            "peak": int8_peak, "unit": "TFLOP/s", "frac": tops_frac, "traffic": traffic,
            "peak_source": f"{peak_src} bf16 {bf16_tflops} TFLOP/s (burst) x {INT8_PER_BF16} "
                           f"nominal int8:bf16",
            "int8_issue_loop_tops": issue_tops,
            "frac_of_issue_loop": gemm_tops / issue_tops if issue_tops else None,
            # context: the cuBLAS reference looped for seconds under the power cap
            "frac_of_sustained": gemm_tops / (bf16_sust * INT8_PER_BF16),
        },
        "kernels": {
            "rotate_quant_act": {"ms": rqa_mean.tolist(), "GB/s": rqa_gbs,
                                 "frac_hbm": rqa_gbs / hbm_gbs},
            "int8_gemm": {"ms": gemm_mean.tolist(), "TOPS": gemm_tops, "frac_int8_peak": tops_frac},
        },
        "derotate": {"metric": "dequant+derotate GB/s", "value": der_gbs, "unit": "GB/s",
                     "ms": der_ms.mean(axis=0).tolist(), "peak": hbm_gbs,
                     "frac": der_gbs / hbm_gbs, "bytes_per_element": 3},
        "e2e": {"value": e2e_value, "unit": "TOPS", "h2d_bytes_per_step": h2d,
                "pipeline": "pinned x uploads, convrot_linear_int8 and y downloads of "
                            "consecutive linears overlapped on three streams",
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_total},
        "gpu_launches": 2 * n_lin * args.steps,
        "clocks": clk,
    }
    if world == 1 and not args.no_cpu_baseline:
        tops, cores, dt, reps = oracle_sample_rate(lins, args.ref_rows, budget_s=args.cpu_budget)
        out["cpu_baseline"] = {
            "value": tops, "unit": "TOPS", "cores": cores, "kind": "oracle",
            "sample": f"{args.ref_rows} tokens of each linear, {reps} passes in {dt:.1f} s "
                      f"(rotate+quantize, int8 GEMM, epilogue; float64 numpy)"}
    print(json.dumps(out))
    return 0


def run_sweep(args):
    """Per-shape kernel times of the group-size / skinny-M sweep (K = N = 4096,
    G in {4, 16, 64, 256}, M in {1, 16, 128, 1024, 8192}) and of the standalone
    decode of a [12288, 3072] int8 weight at each G; one JSON line."""
    import torch

    import activation_quantized_linear_b200 as cr
    torch.cuda.set_device(0)
    hbm_gbs, bf16_tflops, _, _ = load_peaks()
    int8_peak = bf16_tflops * INT8_PER_BF16
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    flush_rd = torch.ones(64 << 20, dtype=torch.float32, device="cuda")

    def timed(fn, n):
        ts = []
        for k in range(n + 3):
            flush.fill_(k & 0xFF)
            flush_rd.sum()
            torch.cuda._sleep(400_000)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            if k >= 3:
                ts.append(e0.elapsed_time(e1))
        return statistics.median(ts)

    rows = []
    for G in workloads.GROUP_SIZES:
        rot = cr.Rotation(workloads.sylvester_rotation(G))
        for M in (1, 16, 128, 1024, 8192):
            lin = workloads.Linear("sweep", M, 4096, 4096, G=G)
            inp = workloads.make_layer_inputs(lin, 4)
            Wq, s_w = cr.quantize_weight(inp.W.cuda(), rot)
            x, bias = inp.x.cuda(), inp.bias.cuda()
            xq, s_tok = cr.rotate_quant_act(x, rot)
            y = cr.int8_gemm(xq, s_tok, Wq, s_w, bias)
            t_r = timed(lambda: cr.rotate_quant_act(x, rot, xq=xq, s_tok=s_tok), args.steps)
            t_g = timed(lambda: cr.int8_gemm(xq, s_tok, Wq, s_w, bias, out=y), args.steps)
            ops = 2.0 * M * 4096 * 4096
            gemm_bytes = M * 4096 + 4096 * 4096 + 2 * M * 4096
            rows.append({"G": G, "M": M, "rotate_ms": t_r, "rotate_GBps": (3 * M * 4096 + 4 * M) / t_r / 1e6,
                         "gemm_ms": t_g, "gemm_TOPS": ops / t_g / 1e9,
                         "gemm_frac_int8_peak": ops / t_g / 1e9 / int8_peak,
                         "gemm_GBps": gemm_bytes / t_g / 1e6,
                         "gemm_frac_hbm": gemm_bytes / t_g / 1e6 / hbm_gbs})
    # GEMMs launched back to back as in use (chained: each launch's set-up and
    # first weight loads overlap the previous launch's drain), each on its own
    # weight copy so that the weights stream from HBM; K = N = 4096
    gemm_chained = []
    rot = cr.Rotation(workloads.sylvester_rotation(256))
    for Mc in (1024, 8192):
        Ws = [torch.randint(-127, 128, (4096, 4096), dtype=torch.int8, device="cuda") for _ in range(6)]
        xq = torch.randint(-127, 128, (Mc, 4096), dtype=torch.int8, device="cuda")
        st = torch.rand(Mc, device="cuda") * 1e-3
        sw1 = torch.tensor([1e-3], device="cuda")
        bias = torch.zeros(4096, dtype=torch.bfloat16, device="cuda")
        y = torch.empty((Mc, 4096), dtype=torch.bfloat16, device="cuda")
        t = timed(lambda: [cr.int8_gemm(xq, st, W, sw1, bias, out=y) for W in Ws], args.steps) / len(Ws)
        ops = 2.0 * Mc * 4096 * 4096
        gemm_chained.append({"M": Mc, "gemm_ms": t, "gemm_TOPS": ops / t / 1e9,
                             "gemm_frac_int8_peak": ops / t / 1e9 / int8_peak})
        del Ws
    dec = []
    N, K = workloads.DEROTATE_SWEEP_SHAPE
    for G in workloads.GROUP_SIZES:
        rot = cr.Rotation(workloads.sylvester_rotation(G))
        Wq = torch.randint(-127, 128, (N, K), dtype=torch.int8, device="cuda")
        s_w = torch.tensor([1e-3], device="cuda")
        out = torch.empty((N, K), dtype=torch.bfloat16, device="cuda")
        t = timed(lambda: cr.dequant_derotate(Wq, s_w, rot, out=out), args.steps)
        dec.append({"G": G, "ms": t, "GBps": 3 * N * K / t / 1e6, "frac_hbm": 3 * N * K / t / 1e6 / hbm_gbs})
    # few tokens, launched back to back as in a model (chained launches), each
    # launch on its own weight copy so that the weights (8 x 16.8 MB) stream
    # from HBM, not L2
    # K = N = 4096 and the few-token forms of the workloads' wide and deep
    # linears (FLUX.1 fused in-projection, Z-Image QKV and FFN down)
    chained = []
    rot = cr.Rotation(workloads.sylvester_rotation(256))
    sw1 = torch.tensor([1e-3], device="cuda")
    for Kc, Nc, copies in ((4096, 4096, 8), (3072, 21504, 3), (3840, 11520, 4), (10240, 3840, 4)):
        Ws = [torch.randint(-127, 128, (Nc, Kc), dtype=torch.int8, device="cuda") for _ in range(copies)]
        for Mc in (1, 2, 16, 64, 128):  # 1-2 tokens: the dp4a product; more: swap-AB
            xq = torch.randint(-127, 128, (Mc, Kc), dtype=torch.int8, device="cuda")
            st = torch.rand(Mc, device="cuda") * 1e-3
            y = torch.empty((Mc, Nc), dtype=torch.bfloat16, device="cuda")
            t = timed(lambda: [cr.int8_gemm(xq, st, W, sw1, None, out=y) for W in Ws],
                      args.steps) / len(Ws)
            wbytes = Mc * Kc + Nc * Kc + 2 * Mc * Nc
            chained.append({"K": Kc, "N": Nc, "M": Mc, "gemm_ms": t, "gemm_GBps": wbytes / t / 1e6,
                            "gemm_frac_hbm": wbytes / t / 1e6 / hbm_gbs})
        del Ws
    # per-output-channel weight scales and fp16 activations/outputs, G = 256:
    # the GEMM at M = 8192 and the [12288, 3072] decode
    var = []
    rot = cr.Rotation(workloads.sylvester_rotation(256))
    M = 8192
    for fmt, per_channel in (("bf16", True), ("f16", False), ("f16", True)):
        act = torch.float16 if fmt == "f16" else torch.bfloat16
        inp = workloads.make_layer_inputs(workloads.Linear("sweep", M, 4096, 4096), 4, dtype=act)
        Wq, s_w = cr.quantize_weight(inp.W.cuda(), rot)
        if per_channel:
            s_w = (s_w * (1 + 0.1 * torch.rand(4096, device="cuda"))).contiguous()
        x, bias = inp.x.cuda(), inp.bias.cuda()
        xq, s_tok = cr.rotate_quant_act(x, rot)
        y = cr.int8_gemm(xq, s_tok, Wq, s_w, bias)
        t_r = timed(lambda: cr.rotate_quant_act(x, rot, xq=xq, s_tok=s_tok), args.steps)
        t_g = timed(lambda: cr.int8_gemm(xq, s_tok, Wq, s_w, bias, out=y), args.steps)
        Wd = torch.randint(-127, 128, (N, K), dtype=torch.int8, device="cuda")
        sd = (torch.rand(N, device="cuda") * 1e-3 + 1e-4) if per_channel else torch.tensor([1e-3], device="cuda")
        out = torch.empty((N, K), dtype=act, device="cuda")
        t_d = timed(lambda: cr.dequant_derotate(Wd, sd, rot, out=out), args.steps)
        ops = 2.0 * M * 4096 * 4096
        var.append({"activations": fmt, "s_w": "per_channel" if per_channel else "per_tensor",
                    "rotate_ms": t_r, "rotate_GBps": (3 * M * 4096 + 4 * M) / t_r / 1e6,
                    "gemm_ms": t_g, "gemm_TOPS": ops / t_g / 1e9,
                    "gemm_frac_int8_peak": ops / t_g / 1e9 / int8_peak,
                    "decode_12288x3072_ms": t_d, "decode_GBps": 3 * N * K / t_d / 1e6,
                    "decode_frac_hbm": 3 * N * K / t_d / 1e6 / hbm_gbs})
    # a dense (non-Hadamard) orthogonal R: the float64 FMA path
    dense = []
    for G in (64, 256):
        rot = cr.Rotation(workloads.qr_rotation(G))
        inp = workloads.make_layer_inputs(workloads.Linear("sweep", M, 4096, 4096, G=G), 4)
        x = inp.x.cuda()
        xq, s_tok = cr.rotate_quant_act(x, rot)
        t_r = timed(lambda: cr.rotate_quant_act(x, rot, xq=xq, s_tok=s_tok), max(3, args.steps // 4))
        Wd = torch.randint(-127, 128, (N, K), dtype=torch.int8, device="cuda")
        sd = torch.tensor([1e-3], device="cuda")
        out = torch.empty((N, K), dtype=torch.bfloat16, device="cuda")
        t_d = timed(lambda: cr.dequant_derotate(Wd, sd, rot, out=out), max(3, args.steps // 4))
        dense.append({"G": G, "rotate_ms": t_r, "rotate_GBps": (3 * M * 4096 + 4 * M) / t_r / 1e6,
                      "rotate_fp64_tflops": 2.0 * G * M * 4096 * 2 / t_r / 1e9,
                      "decode_12288x3072_ms": t_d, "decode_GBps": 3 * N * K / t_d / 1e6,
                      "decode_fp64_tflops": 2.0 * G * N * K / t_d / 1e9})
    print(json.dumps({"sweep": "group_size_and_skinny_M", "linears": rows, "decode_12288x3072": dec,
                      "gemm_chained_K4096": gemm_chained,
                      "variants_G256": var, "dense_R_M8192": dense,
                      "few_tokens_chained_G256": chained,
                      "peaks": {"hbm_gbs": hbm_gbs, "int8_tops": int8_peak}}))
    return 0


class Int8RateProbe:
    """The int8 tensor-core issue-rate probe: its own library
    (libconvrot_bench.so, built beside the layer's), which the layer's
    library does not export.  measure_int8_mma_rate(iters) -> TOP/s of one
    launch in which every SM issues iters x 4 tcgen05.mma.kind::i8 of
    128 x 256 x 32 on operands held in shared memory."""

    def __init__(self):
        import ctypes

        from activation_quantized_linear_b200 import build
        self._lib = ctypes.CDLL(build.BENCH_LIB_PATH)
        f = self._lib.convrot_bench_int8_mma_rate
        f.argtypes = [ctypes.c_int, ctypes.POINTER(ctypes.c_double), ctypes.c_void_p]
        f.restype = ctypes.c_int
        self._f = f

    def measure_int8_mma_rate(self, iters: int = 32768) -> float:
        import ctypes

        import torch
        tops = ctypes.c_double(0.0)
        st = self._f(int(iters), ctypes.byref(tops), torch.cuda.current_stream().cuda_stream)
        if st != 0:
            raise RuntimeError(f"int8 issue-rate probe failed with status {st}")
        return float(tops.value)


def issue_loop_tops(probe=None):
    """The int8 tensor cores' measured burst rate (TOP/s), or None if the
    measurement fails: it is context for the roofline, never a reason to
    lose the bench line."""
    try:
        probe = probe if probe is not None else Int8RateProbe()
        return probe.measure_int8_mma_rate(32768)
    except Exception as exc:  # noqa: BLE001
        print(f"int8 issue-rate measurement failed: {exc}", file=sys.stderr)
        return None


def run_default_path(args):
    """int8 compute against the pages' default path on the workload's linears
    (Invoke docs "int8 Compute": the default path decodes the weight and
    multiplies in 16 bits on every forward).  Per linear, CUDA events around one
    call on L2-flushed inputs: convrot_linear_int8 (rotate+quantize, int8 GEMM),
    convrot_linear_dequant (decode, 16-bit GEMM) and the 16-bit GEMM alone on a
    decoded weight; one JSON line."""
    import torch

    import activation_quantized_linear_b200 as cr
    torch.cuda.set_device(0)
    hbm_gbs, bf16_tflops, _, peak_kind = load_peaks()
    act = torch.float16 if args.dtype == "f16" else torch.bfloat16
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    flush_rd = torch.ones(64 << 20, dtype=torch.float32, device="cuda")

    def timed(fn, n):
        ts = []
        for k in range(n + 3):
            flush.fill_(k & 0xFF)
            flush_rd.sum()
            torch.cuda._sleep(400_000)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            if k >= 3:
                ts.append(e0.elapsed_time(e1))
        return statistics.median(ts)

    rows = []
    for i, lin in enumerate(workloads.WORKLOADS[args.workload]):
        inp = workloads.make_layer_inputs(lin, i, dtype=act)
        M, N, K = lin.M, lin.N, lin.K
        rot = cr.Rotation(inp.R)
        Wq, s_w = cr.quantize_weight(inp.W.cuda(), rot)
        x, b = inp.x.cuda(), inp.bias.cuda()
        y = torch.empty((M, N), dtype=act, device="cuda")
        ws_i8 = torch.empty(cr.workspace_bytes(M, N, K), dtype=torch.uint8, device="cuda")
        ws_dq = torch.empty(cr.workspace_bytes(M, N, K, op=cr.OP_LINEAR_DEQUANT),
                            dtype=torch.uint8, device="cuda")
        W_hat = cr.dequant_derotate(Wq, s_w, rot, dtype=act)
        t_i8 = timed(lambda: cr.linear_int8(x, Wq, s_w, rot, b, out=y, workspace=ws_i8), args.steps)
        t_dq = timed(lambda: cr.linear_dequant(x, Wq, s_w, rot, b, out=y, workspace=ws_dq),
                     args.steps)
        t_dense = timed(lambda: cr.dense_linear(x, W_hat, b, out=y), args.steps)
        # a library int8 GEMM for reference: torch._int_mm (int32 out, no epilogue)
        try:
            xq, _ = cr.rotate_quant_act(x, rot)
            Wt = Wq.t()  # [K, N] view of the [N, K] codes
            torch._int_mm(xq, Wt)
            t_intmm = timed(lambda: torch._int_mm(xq, Wt), args.steps)
            t_ours = timed(lambda: cr.int8_gemm_s32(xq, Wq), args.steps)
            intmm = {"torch_int_mm_ms": t_intmm, "torch_int_mm_tops": 2.0 * M * N * K / t_intmm / 1e9,
                     "int8_gemm_s32_ms": t_ours, "int8_gemm_s32_tops": 2.0 * M * N * K / t_ours / 1e9}
            del xq
        except Exception as exc:  # noqa: BLE001 (a reference point only)
            intmm = {"torch_int_mm": f"unavailable: {type(exc).__name__}: {exc}"[:200]}
        flops = 2.0 * M * N * K
        rows.append({"linear": f"{lin.name}:M{M}xK{K}->N{N}", "int8_ms": t_i8, "dequant_ms": t_dq,
                     "dense16_ms": t_dense, "int8_speedup_over_default": t_dq / t_i8,
                     "dense16_tflops": flops / t_dense / 1e9,
                     "dense16_frac_bf16_peak": flops / t_dense / 1e9 / bf16_tflops, **intmm})
        del Wq, W_hat, ws_i8, ws_dq, y
    issue_tops = issue_loop_tops()
    total_i8 = sum(r["int8_ms"] for r in rows)
    total_dq = sum(r["dequant_ms"] for r in rows)
    print(json.dumps({"compare": "int8_compute_vs_default_path", "workload": args.workload,
                      "dtype": args.dtype, "linears": rows,
                      "int8_speedup_over_default": total_dq / total_i8,
                      "bf16_peak_tflops": bf16_tflops, "peak": peak_kind,
                      "int8_issue_loop_tops": issue_tops,
                      "timing": "median of --steps single calls, CUDA events, L2 flushed before each"}))
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="wan22_a14b_video_dit",
                    choices=[k for k in workloads.WORKLOADS if k != "group_size_sweep"])
    ap.add_argument("--dtype", default="bf16", choices=["bf16", "f16"],
                    help="16-bit float format of activations, bias, outputs and the decoded weight")
    ap.add_argument("--ref-rows", type=int, default=64)
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--default-path", action="store_true",
                    help="time int8 compute against the default path (decode + 16-bit GEMM) instead")
    ap.add_argument("--sweep", action="store_true",
                    help="time the group-size / skinny-M sweep and the decode sweep instead")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.sweep:
        return run_sweep(args)
    if args.default_path:
        return run_default_path(args)
    lins = workloads.WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, lins)
    try:
        return run_ours(args, lins)
    finally:
        try:
            import torch.distributed as dist
            if dist.is_initialized():
                dist.destroy_process_group()
        except Exception:
            pass


if __name__ == "__main__":
    sys.exit(main())
