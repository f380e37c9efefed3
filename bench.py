"""Benchmark: one full Muon optimizer step on the Llama-7B-shaped parameter set.

Workload: 32 layers x {4 x 4096x4096, 2 x 4096x11008, 11008x4096} = 224 matrices,
6.476e9 parameters; bf16 weights ~ N(0, 0.02^2), bf16 gradients ~ N(0, 1e-3^2), fp32
momentum (zero at start); beta 0.95, lr 0.02, weight decay 0.1, Moonlight scale, 5
Newton-Schulz iterations with (3.4445, -4.7750, 2.0315).  A step is momentum + cast +
Frobenius scale + 15 grouped tcgen05 GEMM launches + update for all 224 matrices, through
the C ABI (muon_step_batched).  Synthetic data drawn on the device from a seeded
generator; the set (52 GB) is far larger than L2, so no flush is needed.

Multi-GPU (torchrun): every rank runs its own full parameter set (the step has no
exchange), value = ms per parameter set over the whole job, max over ranks.
`--impl reference` times the fp64 CPU oracle on a bounded sample instead.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

KJ = (3.4445, -4.7750, 2.0315)
LR, BETA, WD = 0.02, 0.95, 0.1
WORKLOAD = "llama7b_muon_step"


LAYERS = 32


def set_shapes():
    from matrix_orthogonalising_optimizer_02_b200 import workloads
    return workloads.llama7b_shapes(LAYERS)


def ns_flops_algorithmic(rows, cols, iters=5):
    """Symmetry-aware count per matrix: X X^T = r^2 s, A A = r^3, B X = 2 r^2 s per iteration."""
    r, s = min(rows, cols), max(rows, cols)
    return iters * (3.0 * r * r * s + float(r) ** 3)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["hbm_gbs"], d["bf16_tflops"], d.get("bf16_tflops_sustained", d["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def cpu_cores():
    try:
        from threadpoolctl import threadpool_info
        th = [i["num_threads"] for i in threadpool_info() if i.get("user_api") == "blas"]
        if th:
            return int(max(th))
    except Exception:
        pass
    return os.cpu_count() or 1


LAYER_SHAPES = ((4096, 4096), (4096, 11008), (11008, 4096))   # distinct shapes of one Llama layer


def layer_counts():
    """How many matrices of each distinct shape one layer holds (4 attention projections,
    2 up/gate, 1 down)."""
    from matrix_orthogonalising_optimizer_02_b200 import workloads
    layer = workloads.llama7b_shapes(1)
    return {sh: layer.count(sh) for sh in LAYER_SHAPES}


def oracle_shape_seconds(shape):
    """Seconds of one fp64 oracle Muon step (momentum, 5 Newton-Schulz iterations, update)
    on one matrix of `shape`, drawn like the set's (bf16 W ~ N(0, 0.02^2), G ~ N(0, 1e-3^2))."""
    import numpy as np
    import oracle as orc
    from matrix_orthogonalising_optimizer_02_b200 import workloads
    r = workloads.rng(1005)
    W = orc.round_to_bf16(r.standard_normal(shape) * 0.02)
    G = orc.round_to_bf16(r.standard_normal(shape) * 1e-3)
    M = np.zeros_like(G)
    t0 = time.perf_counter()
    orc.muon_step(W, G, M, lr=LR, beta=BETA, weight_decay=WD, schedule=orc.fixed_schedule(5))
    return time.perf_counter() - t0


def oracle_set_ms(per_shape_s):
    """The set's oracle time from per-shape step times: one layer is 4 x t(4096^2) +
    2 x t(4096 x 11008) + t(11008 x 4096), and the set is LAYERS such layers (matrices are
    stepped one after another, so their times add)."""
    counts = layer_counts()
    return 1e3 * LAYERS * sum(counts[sh] * per_shape_s[sh] for sh in LAYER_SHAPES)


def cpu_model():
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_baseline_object(per_shape_s, kind="oracle"):
    counts = layer_counts()
    parts = ", ".join(f"{r}x{c}: {per_shape_s[(r, c)]:.2f} s" for (r, c) in LAYER_SHAPES)
    return {"value": oracle_set_ms(per_shape_s), "unit": "ms", "cores": cpu_cores(), "kind": kind,
            "cpu_model": cpu_model(),
            "sample": "fp64 oracle full step (momentum, 5 NS iterations, update) timed on one matrix of each "
                      f"distinct shape of a Llama-7B layer ({parts}); one layer = "
                      + " + ".join(f"{counts[sh]} x t({sh[0]}x{sh[1]})" for sh in LAYER_SHAPES)
                      + f", extrapolated x{LAYERS} layers"}


def workload_config(shapes):
    """The `config` object both arms print for the parameter set `shapes`."""
    return {"workload": WORKLOAD if LAYERS == 32 else f"{WORKLOAD}_{LAYERS}layer", "matrices": len(shapes),
            "params": sum(r * c for r, c in shapes), "ns_iters": 5, "coeffs": list(KJ), "lr": LR, "beta": BETA,
            "weight_decay": WD, "scale": "moonlight", "l2": "inputs (52 GB) larger than L2; no flush"}


def recorded_traffic(layers_per_launch):
    """DRAM bytes per NS GEMM launch: the per-launch bytes ncu recorded on one layer (7
    independent matrices, so traffic grows in proportion), from profiles/tc_gemm_traffic.json,
    times the layers one launch covers -- if that capture was made on the kernel sources as
    they are now (else None)."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "tc_gemm_traffic.json")
    if not os.path.exists(path):
        return None
    rec = json.load(open(path))
    h = hashlib.sha256()
    for f in rec.get("kernel_sources", []):
        h.update(open(os.path.join(ROOT, f), "rb").read())
    if rec.get("kernel_source_sha256_16") != h.hexdigest()[:16] or "traffic_bytes_per_launch_one_layer" not in rec:
        return None
    return int(rec["traffic_bytes_per_launch_one_layer"] * layers_per_launch)


def set_flops():
    return sum(ns_flops_algorithmic(r, c) for (r, c) in set_shapes())


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.p = None

    def start(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                       "-lms", "200", "-i", str(self.dev)], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.p = None

    def stop(self):
        if self.p is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.p.terminate()
        self.p.wait()
        self.f.flush()
        rows = [ln.split(",") for ln in open(self.f.name).read().strip().splitlines() if ln.strip()]
        os.unlink(self.f.name)
        sm = [float(r[1]) for r in rows if len(r) >= 9 and r[1].strip().replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if len(r) >= 9 and r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows if len(r) >= 9 for i in range(4) if r[5 + i].strip() == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def _time_ms(fn, warmup, steps):
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps


def secondary_measurements(only=None):
    """The other parameter sets of the method, each timed on the device (CUDA events,
    warm-up first): a 64 x 1024^2 low-rank batch through ns_orthogonalize under the fixed and
    the hybrid schedule, the GPT-2-small set's full step, the 16 x 4096 x 1024 Stiefel step
    and the single 256 x 128 fp32 step."""
    import torch
    from matrix_orthogonalising_optimizer_02_b200 import binding as mb
    from matrix_orthogonalising_optimizer_02_b200 import workloads
    out = {}
    gen = torch.Generator(device="cuda")
    gen.manual_seed(1003)
    if only in (None, "lowrank"):
        out.update(_lowrank())
    if only in (None, "gpt2"):
        out.update(_gpt2(gen))
    if only in (None, "stiefel"):
        out.update(_stiefel(gen))
    if only in (None, "single"):
        out.update(_single())
    if only == "cublas":
        out.update(_cublas_reference())
    return out


def _cublas_reference():
    """Context, not the product path: the library GEMM (torch.matmul -> cuBLAS, bf16, fp32
    accumulate) on the dense equivalents of one Newton-Schulz iteration of one Llama layer
    (X X^T, A A, B X for 4 x 4096^2, 3 x 4096x11008), looped for a few seconds so the GPU
    settles at its power-capped clock.  Dense FLOP/s, and the NS chain time those rates
    imply for the full 224-matrix set."""
    import torch
    gen = torch.Generator(device="cuda")
    gen.manual_seed(7)
    shapes = [(4096, 4096)] * 4 + [(4096, 11008)] * 3
    Xs = [torch.empty(s, dtype=torch.bfloat16, device="cuda").normal_(0, 0.01, generator=gen) for s in shapes]
    As = [torch.empty((4096, 4096), dtype=torch.bfloat16, device="cuda").normal_(0, 0.01, generator=gen) for _ in shapes]

    def one_iteration():
        for X, A in zip(Xs, As):
            torch.matmul(X, X.t())
            torch.matmul(A, A)
            torch.matmul(A, X)

    dense = sum(2.0 * 4096 * 4096 * s[1] * 2 + 2.0 * 4096 ** 3 for s in shapes)
    ms = _time_ms(one_iteration, 5, 5)
    reps = max(1, int(3000.0 / ms))
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    ms = _time_ms(one_iteration, 0, reps)
    clk = clocks.stop()
    return {"cublas_dense_tflops": dense / (ms * 1e-3) / 1e12,
            "cublas_ns_chain_ms_for_set": ms * 5 * 32,
            "clocks": clk}


def _lowrank():
    import torch
    from matrix_orthogonalising_optimizer_02_b200 import binding as mb
    from matrix_orthogonalising_optimizer_02_b200 import workloads
    out = {}
    X = torch.tensor(workloads.low_rank_plus_noise(batch=64, n=1024)).to(torch.bfloat16).cuda()
    Y = torch.empty_like(X)
    for name, sch, iters in [("lowrank64_kj5_split2", mb.Schedule.fixed(5, n_split_iters=2), 5),
                             ("lowrank64_hybrid_split4", mb.Schedule.hybrid(n_split_iters=4), 10)]:
        ws = mb.workspace(mb.ns_workspace_size(64, 1024, 1024, sch))
        ms = _time_ms(lambda: mb.ns_orthogonalize(X, Y, sch, ws), 2, 5)
        fl = 64 * iters * 4.0 * 1024 ** 3
        out[name] = {"ms": ms, "algorithmic_tflops": fl / (ms * 1e-3) / 1e12}
        del ws
    return out


def _gpt2(gen):
    import torch
    from matrix_orthogonalising_optimizer_02_b200 import binding as mb
    from matrix_orthogonalising_optimizer_02_b200 import workloads
    out = {}
    mats = []
    for (rows, cols) in workloads.gpt2_small_shapes(12):
        mats.append(mb.Matrix(torch.empty((rows, cols), dtype=torch.bfloat16, device="cuda").normal_(0, 0.02, generator=gen),
                              torch.empty((rows, cols), dtype=torch.bfloat16, device="cuda").normal_(0, 1e-3, generator=gen),
                              torch.zeros((rows, cols), dtype=torch.float32, device="cuda")))
    hp = mb.hyper(lr=LR, beta=BETA, weight_decay=WD)
    ws = mb.workspace(mb.muon_step_workspace_size(mats, hp))
    ms = _time_ms(lambda: mb.muon_step_batched(mats, hp, ws), 3, 10)
    fl = sum(ns_flops_algorithmic(r, c) for r, c in workloads.gpt2_small_shapes(12))
    out["gpt2_small_step"] = {"ms": ms, "ns_algorithmic_tflops": fl / (ms * 1e-3) / 1e12}
    return out


def _stiefel(gen):
    import torch
    from matrix_orthogonalising_optimizer_02_b200 import binding as mb
    from matrix_orthogonalising_optimizer_02_b200 import workloads
    out = {}
    W = torch.tensor(workloads.stiefel_problem(batch=16, n=4096, k=1024), dtype=torch.float32, device="cuda")
    G = torch.empty_like(W).normal_(0, 1.0, generator=gen)
    ws = mb.workspace(mb.stiefel_workspace_size(16, 4096, 1024))
    mb.stiefel_cayley_step(W, G, 1e-2, ws)   # first launches load the kernels: keep them out of the timing
    torch.cuda.synchronize()
    mb.timing_reset()
    mb.timing_enable(True)
    mb.stiefel_cayley_step(W, G, 1e-2, ws)
    torch.cuda.synchronize()
    mb.timing_enable(False)
    kinds = {k: mb.timing_read(k) for k in ("tc_f32", "simt_gemm", "simt_gemm_f64", "lu", "misc")}
    work = sum(kinds[k][2] for k in ("tc_f32", "simt_gemm", "simt_gemm_f64", "lu"))
    ms = _time_ms(lambda: mb.stiefel_cayley_step(W, G, 1e-2, ws), 1, 3)
    # Rooflines, one per arithmetic type, from the unit counts at the maximum SM clock
    # (1965 MHz): 148 SMs x 128 fp32 FMA lanes x 2 FLOP = 74.4 TFLOP/s for the fp32 products;
    # 148 SMs x 64 fp64 lanes x 2 FLOP = 37.2 TFLOP/s for the fp64 LU and back-substitution
    # updates, which run on the fp64 tensor cores (the same peak as the fp64 FMA pipes here)
    def roof(kind, lanes, what):
        kms, _, kwork = kinds[kind]
        peak = 148 * lanes * 2 * 1.965e9 / 1e12
        ach = kwork / max(kms * 1e-3, 1e-12) / 1e12
        return {"bound": "alu" if lanes == 128 else "tensor", "kernel": what, "achieved": ach, "peak": peak,
                "unit": "TFLOP/s", "frac": ach / peak, "kernel_ms_per_step": kms,
                "peak_source": f"148 SMs x {lanes} lanes x 2 FLOP x 1965 MHz"}
    out["stiefel_16x4096x1024_step"] = {"ms": ms, "fma_tflops": work / (ms * 1e-3) / 1e12,
                                        "kernel_ms": {k: v[0] for k, v in kinds.items()},
                                        "tc_f32_tflops": kinds["tc_f32"][2] / max(kinds["tc_f32"][0] * 1e-3, 1e-12) / 1e12,
                                        "roofline_fp32": roof("simt_gemm", 128, "simt_gemm kernels, fp32 FMA products"),
                                        "roofline_fp64": roof("simt_gemm_f64", 64, "dmma_gemm_kernel, fp64 tensor-core LU and back-substitution updates")}
    return out


def _single():
    import torch
    from matrix_orthogonalising_optimizer_02_b200 import binding as mb
    from matrix_orthogonalising_optimizer_02_b200 import workloads
    out = {}
    Wn, Gn, Mn = workloads.single_fp32()
    one = [mb.Matrix(torch.tensor(Wn).cuda(), torch.tensor(Gn).cuda(), torch.tensor(Mn).cuda())]
    hp1 = mb.hyper(lr=0.02, beta=0.95, weight_decay=0.0, schedule=mb.Schedule.fixed(5, fp32_mode=True))
    ws = mb.workspace(mb.muon_step_workspace_size(one, hp1))
    out["single_256x128_fp32_step_us"] = 1e3 * _time_ms(lambda: mb.muon_step_batched(one, hp1, ws), 5, 50)
    # the device time of the step's kernels alone (events around each launch)
    mb.timing_reset()
    mb.timing_enable(True)
    for _ in range(20):
        mb.muon_step_batched(one, hp1, ws)
    torch.cuda.synchronize()
    mb.timing_enable(False)
    kern_ms = sum(mb.timing_read(k)[0] for k in mb.KERNEL_KINDS)
    launches = sum(mb.timing_read(k)[1] for k in mb.KERNEL_KINDS)
    out["single_256x128_fp32_kernel_us"] = 1e3 * kern_ms / 20
    out["single_256x128_fp32_launches"] = launches / 20
    # the same step replayed from a CUDA graph (no host work per step)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        mb.muon_step_batched(one, hp1, ws, stream=s)
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        mb.muon_step_batched(one, hp1, ws)
    out["single_256x128_fp32_graph_us"] = 1e3 * _time_ms(g.replay, 5, 50)
    return out


def run_reference(args, rank, world):
    """The oracle as it stands, on this host's cores.  Each step is one bounded sample: the
    full oracle step on one matrix of one of the layer's three distinct shapes, the shapes
    taken in turn.  The printed value is the set time composed from the mean time of each
    shape over the timed steps (a shape that no timed step reached is timed once more after
    them), exactly as the cpu_baseline of the device arm composes it."""
    if rank != 0:
        return
    times = {sh: [] for sh in LAYER_SHAPES}
    for i in range(args.warmup + args.steps):
        sh = LAYER_SHAPES[i % len(LAYER_SHAPES)]
        dt = oracle_shape_seconds(sh)
        if i >= args.warmup:
            times[sh].append(dt)
    for sh in LAYER_SHAPES:
        if not times[sh]:
            times[sh].append(oracle_shape_seconds(sh))
    per_shape = {sh: statistics.mean(v) for sh, v in times.items()}
    ms = oracle_set_ms(per_shape)
    base = cpu_baseline_object(per_shape)
    base["sample"] += f"; {args.steps} timed steps take the three shapes in turn"
    out = {"metric": "Muon full-step ms per param set (Llama-7B-shaped set)", "value": ms, "unit": "ms",
           "impl": "reference", "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
           "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic", "config": workload_config(set_shapes()),
           "cpu_baseline": base,
           "e2e": {"value": ms, "unit": "ms", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-secondary", action="store_true", help="skip the other parameter sets")
    ap.add_argument("--case", default=None, choices=["lowrank", "gpt2", "stiefel", "single", "cublas"],
                    help="time only one of the other parameter sets (for profiling); prints its figures")
    ap.add_argument("--layers", type=int, default=32,
                    help="Llama-7B layers in the set (32 = the full set; 1 = a profiling-sized case)")
    args = ap.parse_args()
    global LAYERS
    LAYERS = args.layers
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    assert args.warmup >= 3, "at least 3 warm-up steps"
    if args.case is not None:
        print(json.dumps(secondary_measurements(only=args.case)), flush=True)
        return

    import datetime
    import torch
    import torch.distributed as dist
    from matrix_orthogonalising_optimizer_02_b200 import binding as mb

    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    def barrier():
        if world > 1:
            dist.barrier()

    shapes = set_shapes()
    gen = torch.Generator(device="cuda")
    gen.manual_seed(1005 + 7919 * rank)
    mats = []
    for (rows, cols) in shapes:
        W = torch.empty((rows, cols), dtype=torch.bfloat16, device="cuda").normal_(0.0, 0.02, generator=gen)
        G = torch.empty((rows, cols), dtype=torch.bfloat16, device="cuda").normal_(0.0, 1e-3, generator=gen)
        M = torch.zeros((rows, cols), dtype=torch.float32, device="cuda")
        mats.append(mb.Matrix(W, G, M))
    hp = mb.hyper(lr=LR, beta=BETA, weight_decay=WD, scale_mode="moonlight", schedule=mb.Schedule.fixed(5, KJ))
    ws = mb.workspace(mb.muon_step_workspace_size(mats, hp))
    stream = torch.cuda.current_stream()

    def step():
        mb.muon_step_batched(mats, hp, ws, stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert mb.device_status(ws) == mb.MUON_OK

    # per-kernel-kind device times (events around every launch, on the launching stream)
    mb.timing_reset()
    mb.timing_enable(True)
    n_prof = 2
    for _ in range(n_prof):
        step()
    torch.cuda.synchronize()
    mb.timing_enable(False)
    prof = {k: mb.timing_read(k) for k in mb.KERNEL_KINDS}
    launches_per_step = sum(v[1] for v in prof.values()) / n_prof

    # timed region
    clocks = ClockSampler(local)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    ms_step = e0.elapsed_time(e1) / args.steps
    if world > 1:
        t = torch.tensor([ms_step], device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms_step = float(t.item())
    assert mb.device_status(ws) == mb.MUON_OK

    # end to end through the public API from host buffers: the gradients sit in pinned host
    # memory and the library streams them in every step (overlapped with the compute of
    # earlier chunks); the step's device status word is read back
    g_host = [m.G.cpu().pin_memory() for m in mats]
    h2d = sum(g.numel() * g.element_size() for g in g_host)
    host_mats = [mb.Matrix(m.W, g, m.M) for m, g in zip(mats, g_host)]
    ws_h = mb.workspace(mb.muon_step_host_grad_workspace_size(host_mats, hp))
    mb.muon_step_batched_host_grad(host_mats, hp, ws_h, stream)     # builds the per-chunk plans
    assert mb.device_status(ws_h, stream) == mb.MUON_OK
    barrier()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.e2e_steps):
        mb.muon_step_batched_host_grad(host_mats, hp, ws_h, stream)
        st = mb.device_status(ws_h, stream)
        assert st == mb.MUON_OK
    t1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = t0.elapsed_time(t1) / args.e2e_steps
    if world > 1:
        t = torch.tensor([e2e_ms], device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e_ms = float(t.item())
    del g_host, host_mats, ws_h

    hbm, tf_burst, tf_sust, peak_src = peaks()
    ns_ms, ns_launches, ns_flops = prof["ns_gemm"]
    ns_tflops = ns_flops / (ns_ms * 1e-3) / 1e12
    mom_ms, _, mom_bytes = prof["momentum"]
    upd_ms, _, upd_bytes = prof["update"]
    ew_gbs = (mom_bytes + upd_bytes) / ((mom_ms + upd_ms) * 1e-3) / 1e9
    total_flops = set_flops()
    step_ns_share = ns_ms / n_prof / ms_step

    out = {
        "metric": "Muon full-step ms per param set (Llama-7B-shaped set)",
        "value": ms_step / world,
        "unit": "ms",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_step,
        "higher_is_better": False,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded on-device normal draws, Llama-7B shapes)",
        "config": workload_config(shapes),
        "gpu_launches": int(round(launches_per_step * args.steps)),
        "matrices_per_s": len(shapes) * world / (ms_step * 1e-3),
        "ns_tflops": ns_tflops,
        "ns_frac_of_bf16_peak": ns_tflops / tf_sust,
        "ns_share_of_step": step_ns_share,
        "elementwise_gbs": ew_gbs,
        "elementwise_frac_of_hbm": ew_gbs / hbm,
        "momentum_gbs": mom_bytes / (mom_ms * 1e-3) / 1e9 if mom_ms else None,
        "update_gbs": upd_bytes / (upd_ms * 1e-3) / 1e9 if upd_ms else None,
        "roofline": {"bound": "tensor", "kernel": "tc_gemm_kernel (NS Gram/polynomial/apply)",
                     "achieved": ns_tflops, "peak": tf_sust, "unit": "TFLOP/s", "frac": ns_tflops / tf_sust,
                     "peak_source": f"{peak_src} bf16 sustained (kernel timed inside a long step)",
                     "work_per_launch": ns_flops / max(ns_launches, 1),
                     "traffic": recorded_traffic(LAYERS * 15 * n_prof / max(ns_launches, 1)),
                     "traffic_unit": "bytes per launch (ncu dram__bytes_read+write on one layer, scaled by the layers one launch covers)"},
        "e2e": {"value": e2e_ms / world, "unit": "ms", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": 4},
        "clocks": clk,
        "total_ns_flops_per_set": total_flops,
    }
    if rank == 0 and world == 1 and not args.no_secondary and LAYERS == 32:
        del mats, ws
        torch.cuda.empty_cache()
        out["secondary"] = secondary_measurements()
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline_object({sh: oracle_shape_seconds(sh) for sh in LAYER_SHAPES})
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
