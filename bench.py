#!/usr/bin/env python
"""Benchmark of the VC-Attention forward hot path on B200.

One step = the whole path on one batch of synthetic input already resident in
HBM: V-Smooth prep (k-means, cluster sort, block means, residual codes), Q/K
per-block FP8 quantisation, and the fused ExpCast FP8 attention. The metric is
FP8 TFLOP/s of the full call, counting the dense attention work 4*B*H*S^2*D
("VC-Attention: Value Smoothing and Softmax Casting for Low-bit Attention",
Abstract: low-bit tensor cores run the two matrix products).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...     # the CPU oracle, timed on host cores

Under torchrun (N > 1) every rank runs its own independent problem of the same
size on its own GPU (weak scaling); the only collectives are a barrier and the
max over ranks of the measured time. Rank 0 prints one JSON line.
"""
import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "VC-attn FP8 TFLOP/s and % of FP8 peak at S=73397,D=128; rel-L2 vs FP64"
UNIT = "TFLOP/s"
DEFAULT_WORKLOAD = "minimax_h56"
ATTN_SRC = os.path.join(ROOT, "bit_fp8_attention_prep_b200", "csrc", "vc_attn_fwd.cu")
# the kernel the roofline line describes: one E4M3 V plane, or the two exact
# E4M3 planes of an NVFP4 residual (the forward stage then also runs the
# plane split, nvfp4_planes_kernel)
ATTN_KERNEL = {"e4m3": "vc_attn_fwd_kernel<1>", "nvfp4": "vc_attn_fwd_kernel<2>"}
# DRAM bytes (read + write) of one attention launch on the default workload, from
# the ncu capture summarised in profiles/; valid only while the kernel source
# hashes to the recorded value (otherwise traffic is reported as null).
ATTN_TRAFFIC = {"sha256_16": "2b726db56ae51685", "bytes_per_launch": 8 * (200.098304e6 + 103.392e6)}
FALLBACK_BF16_TFLOPS_SUSTAINED = 1400.0
FALLBACK_HBM_GBS = 6650.0


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--k-p", type=int, default=8)
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the SDPA comparison, accuracy, e2e and CPU-baseline legs")
    ap.add_argument("--extras", default="all",
                    help="comma-separated extra legs after the timed region: accuracy, energy, smoothk, exp2, "
                         "sdpa, e2e, cpu, ties, formats, repair (default all; --no-extras = none)")
    ap.add_argument("--head-chunk", type=int, default=4,
                    help="heads per chunk of the host-buffer pipeline timed by the e2e leg")
    ap.add_argument("--sweep", choices=["nvfp4"], default=None,
                    help="instead of the benchmark line: the NVFP4-V vs E4M3-V sweep over S (H=24), one JSON "
                         "line per S")
    return ap.parse_args()


# ----------------------------------------------------------------- helpers
def flops_of(cfg):
    return 4.0 * cfg["B"] * cfg["H"] * float(cfg["S"]) ** 2 * 128


def max_over_ranks(x, world, device="cpu"):
    """The largest of the ranks' values of x (every rank gets it); x itself when
    there is one rank. The timed region of a multi-GPU run is the slowest rank's."""
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tflops(world, flops_per_rank, ms_per_step):
    """Whole-job throughput of a weak-scaling run: every rank runs its own
    problem of flops_per_rank, the step takes the slowest rank's time."""
    return world * flops_per_rank / (ms_per_step * 1e-3) / 1e12


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return dict(bf16_sustained=float(p["bf16_tflops_sustained"]), bf16_burst=float(p["bf16_tflops"]),
                    hbm=float(p["hbm_gbs"]), source="measured")
    except (OSError, KeyError, ValueError):
        return dict(bf16_sustained=FALLBACK_BF16_TFLOPS_SUSTAINED, bf16_burst=1590.0, hbm=FALLBACK_HBM_GBS,
                    source="fallback")


def src_hash(path):
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        self.dev = device_index

    def start(self):
        try:
            import torch
            uuid = str(torch.cuda.get_device_properties(self.dev).uuid)
            ident = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self.proc = subprocess.Popen(["nvidia-smi", "--id=" + ident, "--query-gpu=" + self.FIELDS,
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, AttributeError, RuntimeError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) != 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for n, v in zip(names, parts[3:]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------- CPU oracle legs
def oracle_sample(cfg, S_sample, rows, seed=0):
    """Time the oracle as it stands on one (b, h) slice: V-Smooth prep and Q/K
    quantisation of the first ``S_sample`` tokens, then ``rows`` query rows
    against all of them. Returns (seconds for the full workload, extrapolated
    per head and per row, the measured seconds, a description)."""
    import numpy as np
    import oracle as O
    from bit_fp8_attention_prep_b200 import synth
    Q, K, V = synth.make_qkv(1, S_sample, 1, recipe=cfg["recipe"], seed=seed)
    q, k, v = (X[0, :, 0].float().numpy() for X in (Q, K, V))
    t0 = time.perf_counter()
    prep = O.prepare_v_head(v, cfg["k"], cfg["iters"], 0, 0, fmt=cfg["fmt"])
    qc, qs, kc, ks = O.quant_qk_head(q, k, prep["perm"])
    t1 = time.perf_counter()
    r = np.linspace(0, S_sample - 1, rows).astype(np.int64)
    O.vc_attention_rows(qc, qs, kc, ks, prep["vres"], prep["mu"], S_sample, r, 1.0 / math.sqrt(128))
    t2 = time.perf_counter()
    S, BH = cfg["S"], cfg["B"] * cfg["H"]
    # prep and quantisation are linear in S; each output row costs O(S)
    full = BH * ((t1 - t0) * S / S_sample + (t2 - t1) * (S / rows) * (S / S_sample))
    desc = (f"one (b,h) slice: V-Smooth prep + Q/K quantisation of {S_sample} tokens and {rows} query rows "
            f"of VC-attention against them; extrapolated x{BH} slices, linearly in S for prep and per row "
            f"for attention")
    return full, t2 - t0, desc


def oracle_cores():
    """Host cores the oracle legs use: one process per core."""
    return max(1, os.cpu_count() or 1)


def _oracle_worker_init():
    # one BLAS thread per process (set before the worker first imports numpy)
    for var in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
        os.environ[var] = "1"


def _oracle_job(cfg, S_sample, rows, seed):
    return oracle_sample(cfg, S_sample, rows, seed=seed)


def oracle_sample_cores(cfg, S_sample, rows):
    """The oracle as it stands on every host core: one process per core (spawned,
    one BLAS thread each), each timing oracle_sample on its own seeded slice at
    the same time. The workload's slices would be shared among the processes, so
    its time is the mean per-process estimate over the process count.
    Returns (seconds for the full workload, measured seconds per process,
    description, processes)."""
    n = oracle_cores()
    if n == 1:
        full, took, desc = oracle_sample(cfg, S_sample, rows)
        return full, took, desc + "; 1 process", 1
    import multiprocessing as mp
    with mp.get_context("spawn").Pool(n, initializer=_oracle_worker_init) as pool:
        res = pool.starmap(_oracle_job, [(cfg, S_sample, rows, seed) for seed in range(n)])
    full = statistics.mean(r[0] for r in res) / n
    took = statistics.mean(r[1] for r in res)
    return full, took, res[0][2] + f"; {n} processes at once (one BLAS thread each), slices shared among them", n


def run_reference(args, cfg):
    """--impl reference: the CPU oracle as it stands, on the host cores."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    flops = flops_of(cfg)
    # each step a bounded sample, sized so that the whole run stays within a few minutes
    budget = 150.0 / max(1, args.steps + args.warmup)
    S_sample = int(min(cfg["S"], max(1024, 8192 * budget / 1.3)))   # ~1.3 s per 8192 tokens here
    for _ in range(args.warmup):
        oracle_sample_cores(cfg, S_sample, 64)
    est, meas = [], 0.0
    for _ in range(args.steps):
        full, took, desc, cores = oracle_sample_cores(cfg, S_sample, 64)
        est.append(full)
        meas += took
    t_full = statistics.mean(est)
    value = flops / t_full / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_full * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(cfg, args),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": desc + f"; measured {meas / max(1, args.steps):.2f} s per step"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


def config_of(cfg, args):
    return {"workload": cfg["name"], "B": cfg["B"], "S": cfg["S"], "H": cfg["H"], "D": 128,
            "kmeans_k": cfg["k"], "lloyd_iters": cfg["iters"], "residual": cfg["fmt"], "k_p": args.k_p,
            "layout": "[B,S,H,128] bf16 in, bf16 out", "non_causal": True,
            "l2": "inputs larger than L2 (bf16 Q/K/V %.2f GB per GPU)" % (3 * cfg["B"] * cfg["S"] * cfg["H"] * 256 / 1e9),
            "parallelism": f"independent problem per GPU x{args.gpus}"}


# ----------------------------------------------------------------- GPU leg
def run_ours(args, cfg):
    import torch
    import torch.distributed as dist
    from bit_fp8_attention_prep_b200 import synth, vc_attn

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    B, S, H = cfg["B"], cfg["S"], cfg["H"]
    Q, K, V = synth.make_workload(cfg["name"], seed=rank, device=dev)[1:]
    plan = vc_attn.Plan(B, S, H, k=cfg["k"], iters=cfg["iters"], fmt=cfg["fmt"], k_p=args.k_p, device=dev)
    stream = torch.cuda.current_stream(dev)
    flops = flops_of(cfg)

    for _ in range(args.warmup):
        plan.run(Q, K, V)
    torch.cuda.synchronize(dev)
    if int(plan.status.item()) != 0:
        raise RuntimeError(f"device status {int(plan.status.item())} after warm-up")

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    clocks = ClockSampler(local)
    n0 = vc_attn.launch_count()
    barrier()
    torch.cuda.synchronize(dev)
    clocks.start()
    for i in range(args.steps):
        e = ev[i]
        e[0].record(stream)
        plan.prepare_v(V)
        e[1].record(stream)
        plan.quant_qk(Q, K)
        e[2].record(stream)
        plan.forward()
        e[3].record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    clk = clocks.stop()
    launches = vc_attn.launch_count() - n0
    total_ms = ev[0][0].elapsed_time(ev[-1][3])
    prep_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ev)
    qk_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in ev)
    fwd_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in ev)
    status = int(plan.status.item())
    total_ms = max_over_ranks(total_ms, world, dev)
    ms_per_step = total_ms / args.steps
    value = job_tflops(world, flops, ms_per_step)

    peaks = load_peaks()
    # FP8 peak: the measured bf16 cuBLAS figure times the nominal FP8:BF16 ratio of
    # 2. The step lasts tens of milliseconds, so the burst figure is the one taken;
    # the sustained one (seconds under the power cap) is given beside it
    fp8_peak = 2.0 * peaks["bf16_burst"]
    fp8_peak_sustained = 2.0 * peaks["bf16_sustained"]
    attn_tflops = flops / (fwd_ms * 1e-3) / 1e12
    traffic = None
    if ATTN_TRAFFIC["sha256_16"] and ATTN_TRAFFIC["sha256_16"] == src_hash(ATTN_SRC) and \
            cfg["name"] == DEFAULT_WORKLOAD:
        traffic = ATTN_TRAFFIC["bytes_per_launch"]
    nb = (S + 127) // 128
    # algorithmic bytes: read bf16 V once, write codes + perm + means (prep);
    # read bf16 Q, K once, read perm, write codes + scales (Q/K)
    vres_bytes = 128 * nb * 128 if cfg["fmt"] == "e4m3" else 128 * nb * 128 // 2 + 128 * nb * 8
    prep_bytes = B * H * (S * 256 + vres_bytes + S * 4 + nb * 512)
    # the bytes the multi-pass prep must move: V once per Lloyd pass, once for the
    # first pass's cluster sums, once for the block statistics and once for the
    # residual codes (iters + 3 passes), plus the outputs
    passes = cfg["iters"] + 3
    prep_pass_bytes = B * H * (passes * S * 256 + vres_bytes + S * 4 + nb * 512)
    qk_bytes = B * H * (2 * S * 256 + S * 4 + 2 * nb * 128 * 128 + 2 * nb * 4)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "e4m3", "data": "synthetic",
        "config": config_of(cfg, argparse.Namespace(k_p=args.k_p, gpus=world)),
        "roofline": {"bound": "tensor", "kernel": ATTN_KERNEL[cfg["fmt"]], "achieved": attn_tflops,
                     "peak": fp8_peak, "unit": "TFLOP/s", "frac": attn_tflops / fp8_peak, "traffic": traffic,
                     "peak_source": f"2 x {peaks['source']} burst bf16 cuBLAS ({peaks['bf16_burst']:.1f})",
                     "frac_of_sustained_peak": attn_tflops / fp8_peak_sustained},
        "stages_ms": {"prepare_v": prep_ms, "quant_qk": qk_ms, "forward": fwd_ms},
        "forward_only_tflops": attn_tflops,
        "frac_of_fp8_peak_full_call": (value / world) / fp8_peak,
        "prep_hbm": {"algorithmic_bytes": prep_bytes, "achieved_gbs": prep_bytes / (prep_ms * 1e-3) / 1e9,
                     "peak_gbs": peaks["hbm"], "frac": prep_bytes / (prep_ms * 1e-3) / 1e9 / peaks["hbm"],
                     "passes_over_v": passes, "pass_bytes": prep_pass_bytes,
                     "pass_gbs": prep_pass_bytes / (prep_ms * 1e-3) / 1e9,
                     "pass_frac": prep_pass_bytes / (prep_ms * 1e-3) / 1e9 / peaks["hbm"],
                     "what": "frac: V read once and the outputs written, over the prep time; pass_frac: the "
                             "bytes of the multi-pass scheme (V once per Lloyd pass, for the first pass's sums, "
                             "the block statistics and the residual), over the same time"},
        "quant_qk_hbm": {"algorithmic_bytes": qk_bytes, "achieved_gbs": qk_bytes / (qk_ms * 1e-3) / 1e9,
                         "peak_gbs": peaks["hbm"], "frac": qk_bytes / (qk_ms * 1e-3) / 1e9 / peaks["hbm"]},
        "gpu_launches": launches,
        "device_status": status,
        "clocks": clk,
    }
    legs = set() if args.no_extras else (
        {"accuracy", "energy", "smoothk", "exp2", "sdpa", "e2e", "cpu", "ties", "formats", "repair"}
        if args.extras == "all" else set(args.extras.split(",")))
    if world > 1:
        # the same problem split by heads over the ranks (strong scaling), beside
        # the independent problem per rank that `value` reports
        del plan
        line["head_split"] = run_head_split(args, cfg, dev, world, rank, barrier)
        plan = None
    if legs and plan is not None:
        line.update(extras(args, cfg, plan, Q, K, V, dev, stream, flops, world, fwd_ms, ms_per_step, rank, legs))
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def head_slice(X, h0, h1):
    """Heads [h0, h1) of a [B, S, H, 128] (or [S, H, 128]) tensor, as a dense tensor."""
    return (X[:, h0:h1] if X.dim() == 3 else X[:, :, h0:h1]).contiguous()


def run_head_split(args, cfg, dev, world, rank, barrier):
    """One problem (the workload drawn with seed 0 on every rank) split by heads:
    rank r runs heads vc_attn.head_range(H, r, N) through a plan that seeds its
    k-means as those heads of the whole problem, so the N ranks together compute
    exactly the single-GPU result, with no exchange between them. Timed like the
    main region (barrier and synchronize on both sides, max over ranks); the
    value counts the whole problem's FLOPs once."""
    import torch
    from bit_fp8_attention_prep_b200 import synth, vc_attn
    B, S, H = cfg["B"], cfg["S"], cfg["H"]
    h0, h1 = vc_attn.head_range(H, rank, world)
    Qf, Kf, Vf = synth.make_workload(cfg["name"], seed=0, device=dev)[1:]
    Q, K, V = (head_slice(X, h0, h1) for X in (Qf, Kf, Vf))
    del Qf, Kf, Vf
    plan = vc_attn.Plan(B, S, h1 - h0, k=cfg["k"], iters=cfg["iters"], fmt=cfg["fmt"], k_p=args.k_p, device=dev,
                        h_base=h0, H_total=H)
    for _ in range(args.warmup):
        plan.run(Q, K, V)
    stream = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    e0.record(stream)
    for _ in range(args.steps):
        plan.run(Q, K, V)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev) / args.steps
    status = int(plan.status.item())
    del plan, Q, K, V
    return {"value": flops_of(cfg) / (ms * 1e-3) / 1e12, "unit": UNIT, "ms_per_step": ms, "scaling": "strong",
            "heads": [list(vc_attn.head_range(H, r, world)) for r in range(world)], "device_status": status,
            "what": "one problem split by heads over the ranks (vc_attn_prepare_v_shard seeds each shard's "
                    "k-means as those heads of the whole problem); whole-problem FLOPs over the slowest rank"}


def extras(args, cfg, plan, Q, K, V, dev, stream, flops, world, fwd_ms, ms_per_step, rank, legs):
    import torch
    import torch.nn.functional as F
    from torch.nn.attention import SDPBackend, sdpa_kernel

    from bit_fp8_attention_prep_b200 import vc_attn
    out = {}
    B, S, H = cfg["B"], cfg["S"], cfg["H"]
    # accuracy on sampled rows of two heads: rel-L2 against exact attention in fp64
    o = plan.run(Q, K, V).float()
    rows = torch.linspace(0, S - 1, 64, device=dev).long()
    o_naive = None
    if "accuracy" in legs:
        # the unsmoothed baseline: the same call with V quantised as it is (one scale per head)
        naive = vc_attn.Plan(B, S, H, k=cfg["k"], iters=cfg["iters"], fmt=cfg["fmt"], k_p=args.k_p, device=dev,
                             mode="naive")
        o_naive = naive.run(Q, K, V).float()[0, rows]
        del naive
    num = den = num_naive = 0.0
    for h in (0, H - 1):
        q = Q[0, rows, h].double()
        k, v = K[0, :, h].double(), V[0, :, h].double()
        p = torch.softmax((q @ k.t()) / math.sqrt(128), dim=-1)
        ref = p @ v
        num += float(((o[0, rows, h].double() - ref) ** 2).sum())
        den += float((ref ** 2).sum())
        if o_naive is not None:
            num_naive += float(((o_naive[:, h].double() - ref) ** 2).sum())
        del k, v, p
    if "accuracy" in legs:
        out["rel_l2_vs_fp64"] = math.sqrt(num / den)
        out["naive_v_rel_l2_vs_fp64"] = math.sqrt(num_naive / den)
        out["accuracy_sample"] = ("64 query rows x heads {0, H-1} of batch 0, exact fp64 softmax attention on the "
                                  "GPU; naive_v: the same path with V-Smooth off (V itself, one E4M3 scale per head)")
    if "energy" in legs:
        # residual energy per head: in the V-Smooth order with its block means, in
        # the original order with block means, and of V itself; the share of the
        # energy that the token ordering removes, over the heads of batch 0
        torch.cuda.synchronize(dev)
        pm = vc_attn.prepare_v(V, k=cfg["k"], iters=cfg["iters"], fmt=cfg["fmt"], mode="meanonly")
        e_vs = vc_attn.residual_energy(V, plan.perm, plan.mu)
        e_mo = vc_attn.residual_energy(V, pm["perm"], pm["mu"])
        e_v = vc_attn.residual_energy(V)
        cur = torch.cuda.current_stream(dev)
        n = max(3, min(args.steps, 10))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        e0.record(cur)
        for _ in range(n):
            vc_attn.residual_energy(V, plan.perm, plan.mu)
        e1.record(cur)
        torch.cuda.synchronize(dev)
        ms_e = e0.elapsed_time(e1) / n
        nb = (S + 127) // 128
        alg_bytes = B * H * (S * (128 * V.element_size() + 4) + nb * 128 * 4)
        f_sort = (1.0 - e_vs / e_mo)[0].cpu().numpy()
        out["residual_energy"] = {
            "removed_by_sort_mean": float(f_sort.mean()), "removed_by_sort_min": float(f_sort.min()),
            "removed_by_sort_max": float(f_sort.max()),
            "left_of_v_sorted": float((e_vs / e_v)[0].mean()), "left_of_v_meanonly": float((e_mo / e_v)[0].mean()),
            "kernel_ms": ms_e, "kernel_gbs": alg_bytes / (ms_e * 1e-3) / 1e9,
            "what": "per head of batch 0: 1 - E(cluster order, block means) / E(original order, block means), "
                    "E = fp64 sum of ||v - mu_block||^2; left_of_v_*: E / ||V||^2; kernel: one "
                    "vc_attn_residual_energy call (V gathered through perm, 128 x 2 B + 4 B per token-head)"}
        del pm
    if "smoothk" in legs and cfg["fmt"] == "e4m3":
        # K smoothing on keys with a per-(head, channel) offset (the synthetic K of
        # the workload has none): rel-L2 against exact fp64 attention with and
        # without the token-mean subtraction, and the time of the two Q/K calls
        gen = torch.Generator(device=dev).manual_seed(11)
        off = torch.randn((H, 128), generator=gen, device=dev) * 6.0
        Ko = (K.float() + off).to(K.dtype)
        pv = dict(perm=plan.perm, mu=plan.mu, v_codes=plan.v_codes, v_scales=None, s_v=plan.s_v)
        cur = torch.cuda.current_stream(dev)
        res = {}
        for sm in (False, True):
            qk = vc_attn.quant_qk(Q, Ko, plan.perm, smooth_k=sm)
            ok = vc_attn.forward(qk, pv, plan.shape, plan.softmax_scale, plan.k_p).float()
            n = max(3, min(args.steps, 10))
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize(dev)
            e0.record(cur)
            for _ in range(n):
                qk = vc_attn.quant_qk(Q, Ko, plan.perm, smooth_k=sm)
            e1.record(cur)
            torch.cuda.synchronize(dev)
            num = den = 0.0
            for h in (0, H - 1):
                q = Q[0, rows, h].double()
                k, v = Ko[0, :, h].double(), V[0, :, h].double()
                ref = torch.softmax((q @ k.t()) / math.sqrt(128), dim=-1) @ v
                num += float(((ok[0, rows, h].double() - ref) ** 2).sum())
                den += float((ref ** 2).sum())
                del k, v, ref
            res[sm] = (math.sqrt(num / den), e0.elapsed_time(e1) / n)
            del qk, ok
        out["k_smoothing"] = {"rel_l2_vs_fp64_plain": res[False][0], "rel_l2_vs_fp64_smoothed": res[True][0],
                              "quant_qk_ms_plain": res[False][1], "quant_qk_ms_smoothed": res[True][1],
                              "what": "K + N(0, 6^2) offset per (head, channel); vc_attn_quant_qk vs "
                                      "vc_attn_quant_qk_smoothk, same prepared V, same forward; 64 rows x heads "
                                      "{0, H-1} against exact fp64 attention"}
        del Ko
    def rel_l2_rows(of):
        # rel-L2 of output rows `rows` of heads {0, H-1} against exact fp64 attention
        num = den = 0.0
        for h in (0, H - 1):
            q = Q[0, rows, h].double()
            k, v = K[0, :, h].double(), V[0, :, h].double()
            ref = torch.softmax((q @ k.t()) / math.sqrt(128), dim=-1) @ v
            num += float(((of[0, rows, h].double() - ref) ** 2).sum())
            den += float((ref ** 2).sum())
            del k, v, ref
        return math.sqrt(num / den)

    def time_ms(fn, n):
        cur = torch.cuda.current_stream(dev)
        fn()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        e0.record(cur)
        for _ in range(n):
            fn()
        e1.record(cur)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / n

    if "formats" in legs and cfg["fmt"] == "e4m3":
        # the other residual formats on the same inputs: E4M3 with one scale per
        # channel, and MX-style FP4 (E2M1, a power of two per channel and 32 tokens)
        # with its block-scaled FP8 x FP4 PV; prep and forward timed separately
        res = {}
        n = max(3, min(args.steps, 5))
        for fmt in ("e4m3c", "mxfp4"):
            pf = vc_attn.Plan(B, S, H, k=cfg["k"], iters=cfg["iters"], fmt=fmt, k_p=args.k_p, device=dev)
            of = pf.run(Q, K, V).float()
            ms_p = time_ms(lambda: pf.prepare_v(V), n)
            ms_f = time_ms(lambda: pf.forward(), n)
            res[fmt] = {"prepare_v_ms": ms_p, "forward_ms": ms_f, "forward_tflops": flops / (ms_f * 1e-3) / 1e12,
                        "rel_l2_vs_fp64": rel_l2_rows(of), "device_status": int(pf.status.item())}
            del pf, of
        res["what"] = ("e4m3c: vc_attn_prepare_v(VC_RESIDUAL_E4M3_PER_CHANNEL) + vc_attn_forward_e4m3_per_channel; "
                       "mxfp4: vc_attn_prepare_v(VC_RESIDUAL_MXFP4) + vc_attn_forward_mxfp4v; same rows as "
                       "rel_l2_vs_fp64 (the per-head E4M3 path)")
        out["residual_formats"] = res
    if "repair" in legs and cfg["fmt"] == "e4m3":
        # the V residual repair: the prep with the repair planes, the two-plane
        # forward, and the error against exact fp64 attention at three budgets
        res = {}
        n = max(3, min(args.steps, 5))
        qk = dict(q_codes=plan.q_codes, q_scales=plan.q_scales, k_codes=plan.k_codes, k_scales=plan.k_scales)
        for budget in (0.0, 0.005, 0.05):
            pr = vc_attn.prepare_v_repair(V, budget=budget, k=cfg["k"], iters=cfg["iters"])
            ms_p = time_ms(lambda: vc_attn.prepare_v_repair(V, budget=budget, k=cfg["k"], iters=cfg["iters"]), n)
            plan.quant_qk(Q, K)      # the same permutation: the repair's k-means is the plain prep's
            orr = torch.empty_like(plan.o)
            st = torch.zeros(1, dtype=torch.int32, device=dev)
            ms_f = time_ms(lambda: vc_attn.forward_repair(qk, pr, plan.shape, plan.softmax_scale, plan.k_p, out=orr,
                                                          status=st), n)
            res[str(budget)] = {"prepare_v_repair_ms": ms_p, "forward_repair_ms": ms_f,
                                "forward_repair_tflops": flops / (ms_f * 1e-3) / 1e12,
                                "rel_l2_vs_fp64": rel_l2_rows(orr.float()), "device_status": int(st.item()),
                                "kept_tokens_head0": int(pr["kept"][0, 0].sum().item())}
            del pr, orr
        res["what"] = ("vc_attn_prepare_v_repair (prep + per-token error, radix select of the kept tokens, "
                       "correction plane) and vc_attn_forward_repair (two-plane FP8 PV); budget = share of the "
                       "tokens of each head repaired; same rows as rel_l2_vs_fp64")
        out["residual_repair"] = res
    # the comparison kernel: the same fused attention with the probabilities made
    # by exp2 on the special function unit and an E4M3 conversion instead of
    # ExpCast (same prepared inputs, same stream)
    if cfg["fmt"] == "e4m3" and "exp2" in legs:
        qk = dict(q_codes=plan.q_codes, q_scales=plan.q_scales, k_codes=plan.k_codes, k_scales=plan.k_scales)
        pv = dict(perm=plan.perm, mu=plan.mu, v_codes=plan.v_codes, v_scales=None, s_v=plan.s_v)
        ox = torch.empty_like(plan.o)
        for _ in range(2):
            vc_attn.test_forward_exp2(qk, pv, plan.shape, plan.softmax_scale, plan.k_p, out=ox)
        n = max(2, min(args.steps, 5))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        e0.record(stream)
        for _ in range(n):
            vc_attn.test_forward_exp2(qk, pv, plan.shape, plan.softmax_scale, plan.k_p, out=ox)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        ms_x = e0.elapsed_time(e1) / n
        oxf = ox.float()
        num = den = 0.0
        for h in (0, H - 1):
            q = Q[0, rows, h].double()
            k, v = K[0, :, h].double(), V[0, :, h].double()
            ref = torch.softmax((q @ k.t()) / math.sqrt(128), dim=-1) @ v
            num += float(((oxf[0, rows, h].double() - ref) ** 2).sum())
            den += float((ref ** 2).sum())
            del k, v, ref
        out["exp2_comparison"] = {"ms": ms_x, "tflops": flops / (ms_x * 1e-3) / 1e12, "expcast_speedup": ms_x / fwd_ms,
                                  "rel_l2_vs_fp64": math.sqrt(num / den),
                                  "what": "same fused kernel, P = E4M3(ex2.approx(c t - F + k_P)) instead of ExpCast"}
        del ox, oxf
    # BF16 cuDNN SDPA on the same inputs, same stream
    try:
        if "sdpa" not in legs:
            raise StopIteration
        qt, kt, vt = (X.transpose(1, 2) for X in (Q, K, V))
        with sdpa_kernel([SDPBackend.CUDNN_ATTENTION]):
            for _ in range(2):
                F.scaled_dot_product_attention(qt, kt, vt)
            n = max(2, min(args.steps, 5))
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize(dev)
            e0.record(stream)
            for _ in range(n):
                F.scaled_dot_product_attention(qt, kt, vt)
            e1.record(stream)
            torch.cuda.synchronize(dev)
        sdpa_ms = e0.elapsed_time(e1) / n
        out["sdpa_bf16_cudnn"] = {"ms": sdpa_ms, "tflops": flops / (sdpa_ms * 1e-3) / 1e12,
                                  "speedup_forward": sdpa_ms / fwd_ms, "speedup_full_call": sdpa_ms / ms_per_step}
    except StopIteration:
        pass
    except RuntimeError as exc:  # cuDNN backend not available for this shape
        out["sdpa_bf16_cudnn"] = {"unavailable": str(exc).splitlines()[0][:200]}
    if "e2e" in legs:
        # end to end through the public API with host buffers: vc_attn_run_host
        # copies Q, K, V in from pinned host memory and O back, head chunk by head
        # chunk, overlapped with the compute; everything inside the timed region
        hq, hk, hv = (X.cpu().pin_memory() for X in (Q, K, V))
        ho = torch.empty(plan.o.shape, dtype=plan.o.dtype).pin_memory()
        hp = vc_attn.HostPlan(B, S, H, k=cfg["k"], iters=cfg["iters"], fmt=cfg["fmt"], k_p=args.k_p,
                              head_chunk=args.head_chunk, device=dev)

        def timed(step, n):
            step()
            torch.cuda.synchronize(dev)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(n):
                step()
            e1.record(stream)
            torch.cuda.synchronize(dev)
            return max_over_ranks(e0.elapsed_time(e1) / n, world, dev)

        n = max(2, min(args.steps, 5))
        e2e_ms = timed(lambda: hp.run(hq, hk, hv, ho), n)
        plan.run(Q, K, V)
        torch.cuda.synchronize(dev)
        same = bool(torch.equal(ho.view(torch.int16), plan.o.cpu().view(torch.int16)))
        out["e2e"] = {"value": job_tflops(world, flops, e2e_ms), "unit": UNIT,
                      "h2d_bytes_per_step": 3 * Q.numel() * Q.element_size(),
                      "d2h_bytes_per_step": plan.o.numel() * plan.o.element_size(), "ms_per_step": e2e_ms,
                      "api": "vc_attn_run_host", "head_chunk": args.head_chunk,
                      "status": int(hp.status.item()), "output_equals_device_path": same}
        # the same copies done one after the other around the three device calls
        dq, dk, dv = torch.empty_like(Q), torch.empty_like(K), torch.empty_like(V)

        def serial_step():
            dq.copy_(hq, non_blocking=True)
            dk.copy_(hk, non_blocking=True)
            dv.copy_(hv, non_blocking=True)
            plan.run(dq, dk, dv)
            ho.copy_(plan.o, non_blocking=True)

        serial_ms = timed(serial_step, n)
        out["e2e_serial_copies"] = {"value": job_tflops(world, flops, serial_ms), "unit": UNIT,
                                    "ms_per_step": serial_ms}
        del hq, hk, hv, ho, dq, dk, dv, hp
    # k-means near ties: head 0 of this run's input through the GPU prep with its
    # per-pass assignments recorded, then the oracle in lock-step on the host
    if world == 1 and rank == 0 and "ties" in legs:
        import numpy as np
        import oracle as O
        from bit_fp8_attention_prep_b200 import vc_attn
        v0 = V[:, :, 0:1].contiguous()
        pv0 = vc_attn.prepare_v(v0, k=cfg["k"], iters=cfg["iters"], fmt=cfg["fmt"], history=True)
        torch.cuda.synchronize(dev)
        adopt = [pv0["history"][t, 0, 0].cpu().numpy() for t in range(cfg["iters"])]
        ref = O.prepare_v_head(v0[0, :, 0].float().cpu().numpy(), cfg["k"], cfg["iters"], 0, 0, fmt=cfg["fmt"],
                               adopt=adopt)
        out["kmeans_lockstep"] = {
            "near_ties": int(ref["stats"]["near_ties"]), "mismatches": int(ref["stats"]["mismatches"]),
            "perm_bit_exact": bool(np.array_equal(pv0["perm"][0, 0].cpu().numpy(), ref["perm"])),
            "sample": f"head 0: {S} tokens, k={cfg['k']}, {cfg['iters']} passes; a near tie is a disagreement "
                      f"whose relative distance gap is below 1e-6 (adopted); anything else is a mismatch"}
        del pv0, v0
    # the oracle on the host cores, rank 0 at N = 1 only
    if world == 1 and rank == 0 and "cpu" in legs:
        full, took, desc, cores = oracle_sample_cores(cfg, min(S, 73397), 256)
        out["cpu_baseline"] = {"value": flops / full / 1e12, "unit": UNIT, "cores": cores,
                               "kind": "oracle", "sample": desc + f"; measured {took:.1f} s"}
    return out


def run_sweep(args):
    """E4M3-V, NVFP4-V and MX-style FP4 V over S (the NVFP4 sweep workloads: B=1,
    H=24): forward FP8 TFLOP/s of each and rel-L2 against exact fp64 attention on
    sampled rows of two heads. One JSON line per S (not the benchmark line)."""
    import torch
    from bit_fp8_attention_prep_b200 import synth, vc_attn
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    for S in (1024, 4096, 16384, 32768, 65536, 131072):
        cfg = synth.workload(f"nvfp4_s{S}")
        B, H = cfg["B"], cfg["H"]
        Q, K, V = synth.make_workload(cfg["name"], seed=0, device=dev)[1:]
        rows = torch.linspace(0, S - 1, 32, device=dev).long()
        refs = {}
        for h in (0, H - 1):
            q = Q[0, rows, h].double()
            k, v = K[0, :, h].double(), V[0, :, h].double()
            refs[h] = torch.softmax((q @ k.t()) / math.sqrt(128), dim=-1) @ v
            del k, v
        line = {"sweep": "v_residual_formats", "S": S, "B": B, "H": H, "k_p": args.k_p}
        for fmt in ("e4m3", "nvfp4", "mxfp4"):
            plan = vc_attn.Plan(B, S, H, k=cfg["k"], iters=cfg["iters"], fmt=fmt, k_p=args.k_p, device=dev)
            plan.run(Q, K, V)
            for _ in range(2):
                plan.forward()
            n = 5
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize(dev)
            e0.record()
            for _ in range(n):
                plan.forward()
            e1.record()
            torch.cuda.synchronize(dev)
            ms = e0.elapsed_time(e1) / n
            o = plan.o.float()
            num = sum(float(((o[0, rows, h].double() - refs[h]) ** 2).sum()) for h in refs)
            den = sum(float((refs[h] ** 2).sum()) for h in refs)
            line[fmt] = {"forward_ms": ms, "tflops": flops_of(cfg) / (ms * 1e-3) / 1e12,
                         "rel_l2_vs_fp64": math.sqrt(num / den), "device_status": int(plan.status.item())}
            del plan, o
        print(json.dumps(line), flush=True)
        del Q, K, V, refs


def main():
    args = parse_args()
    from bit_fp8_attention_prep_b200 import synth
    if args.sweep:
        run_sweep(args)
        return
    cfg = synth.workload(args.workload)
    if args.impl == "reference":
        run_reference(args, cfg)
    else:
        run_ours(args, cfg)


if __name__ == "__main__":
    main()
