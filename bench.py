#!/usr/bin/env python
"""Benchmark of the triangle attention block on B200.

One step = the starting-node block on the pair tensor, then the ending-node
block on its output (the two orientations of triangle attention, chained as a
structure model applies them), on the N = 1536 bf16 workload (pair tensor
604 MB, larger than the 126 MB L2, so no L2 flush is needed between steps).

Prints ONE JSON line (rank 0).  `value` is attention TFLOP/s of the whole job:
the algorithmic attention FLOPs of a step, 2 x 4 N^2 N_valid H d (QK^T and PV
of both orientations; masked keys and tile padding not counted), times the
steps of all ranks, over the max-over-ranks device time of the timed steps.
`roofline` reports the dominant kernel (tri_attn_fwd) against the measured
bf16 dense tensor peak; `e2e` repeats the step through the host-buffer entry
point with the PCIe copies inside the timed region; `cpu_baseline` times the
fp64 CPU oracle on a bounded sample of the same workload.

Multi-GPU (torchrun): every rank runs its own instance of the workload (an
independent pair tensor; weak scaling); the only collectives are the barrier
and the max-reduction of the timings.

--impl reference runs the CPU oracle instead (the only reference this method
has), rank 0 only, each step a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

WORKLOAD = 3
METRIC = "triangle-attn TFLOP/s at N=1536 bf16; % of B200 bf16 dense tensor peak"
UNIT = "TFLOP/s"
DATASHEET_BF16_TFLOPS = 2250.0
EX2_PER_CLK_SM = 16      # special-function unit exp2 rate, measured with a probe on the B200
EX2_SHARE = 0.75         # the attention kernel evaluates one exponential pair in four on the FMA pipe
NUM_SMS = 148
SM_MAX_MHZ = 1965.0

# DRAM bytes per tri_attn_fwd launch at N = 1536, from one ncu capture of this
# kernel source at N = 768 (457.8 MB read + 133.4 MB written)
# scaled by the ratio of pairs (4): Q, K, V read once, O written once, and the
# logit bias all grow with N^2.  Valid only for the source with this hash;
# otherwise reported as null.
TRAFFIC = {"tri_attn_fwd.cuh": "cb382a5e25ef7893", "bytes_per_launch": 4 * (457.797888e6 + 133.481472e6),
           "measured_at": "N=768, scaled x4 to N=1536"}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=16)
    ap.add_argument("--workload", type=int, default=WORKLOAD,
                    help="workload index (the metric is quoted on the default; others are for profiling)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--backward", action="store_true",
                    help="time the attention-core backward (bf16, tensor cores) instead; one JSON line")
    ap.add_argument("--backward-f32", action="store_true",
                    help="with --backward: the fp32 SIMT kernels instead of the tensor-core ones")
    return ap.parse_args()


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), float(d["hbm_gbs"]), "measured"
    except Exception:
        return 1590.0, 6650.0, "fallback"


def src_hash(name):
    path = os.path.join(ROOT, "protein_pair_representation_layernorm_b200", "csrc", name)
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


# ----------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.path = tempfile.mktemp(prefix="clocks_", suffix=".csv")
        self.proc = None
        self.gpu = gpu_index
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(gpu_index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx.append(float(parts[2]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


# ----------------------------------------------------------------- distributed
def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64,
                     device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ----------------------------------------------------------------- CPU oracle
def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def run_oracle_sample(inp, target_s: float):
    """Time the fp64 oracle on a bounded sample of lines of both orientations.
    Returns (flops, seconds, description, threads).  The all-pairs bias the
    sample needs is timed too and prorated to the share of lines evaluated."""
    import numpy as np
    import oracle
    N = inp.N
    f64 = lambda t: t.detach().to(torch.float64).numpy()
    prob = oracle.Problem(
        Z=inp.Z.view(torch.int16).numpy().view(np.uint16), gamma=f64(inp.gamma),
        beta=f64(inp.beta), Wq=f64(inp.Wq), Wk=f64(inp.Wk), Wv=f64(inp.Wv), Wg=f64(inp.Wg),
        Wb=f64(inp.Wb), Wo=f64(inp.Wo), bg=f64(inp.bg), bo=f64(inp.bo),
        mask=None if inp.mask is None else inp.mask.numpy().astype(np.uint8))
    n_valid = N if inp.mask is None else int(inp.mask.sum())
    per_line = 4.0 * N * n_valid * 4 * 32
    t0 = time.perf_counter()
    bias = oracle.bias_all(prob)
    t_bias = time.perf_counter() - t0
    threads = oracle.num_threads()
    # calibrate on one batch of `threads` lines per orientation, then size the sample
    rng = np.random.default_rng(12345)
    lines_done, t_lines = 0, 0.0
    batch = max(1, threads)
    budget = max(1.0, target_s - t_bias)
    while True:
        lines = rng.choice(N, size=min(N, batch), replace=False).astype(np.int32)
        t0 = time.perf_counter()
        oracle.tri_attn(prob, 0, lines, bias=bias)
        oracle.tri_attn(prob, 1, lines, bias=bias)
        t_lines += time.perf_counter() - t0
        lines_done += 2 * len(lines)
        if t_lines >= budget or lines_done >= 2 * N:
            break
        rate = t_lines / lines_done
        batch = int(min(N, max(batch, (budget - t_lines) / rate / 2)))
    frac = lines_done / (2.0 * N)
    secs = t_lines + t_bias * frac
    flops = per_line * lines_done
    desc = (f"{lines_done} sampled lines (rows for the starting node, columns for the ending "
            f"node) of the N={N} workload, fp64, {threads} OpenMP threads; all-pairs bias "
            f"({t_bias:.2f} s) prorated by {frac:.4f}")
    return flops, secs, desc, threads


# ----------------------------------------------------------------- main arms
def run_reference(args, world, rank):
    if rank != 0:
        return
    from protein_pair_representation_layernorm_b200 import workloads
    inp = workloads.workload_inputs(WORKLOAD)
    w = workloads.WORKLOADS[WORKLOAD]
    times, flops_all = [], []
    desc, cores = "", cpu_cores()
    per_step_s = 2.0
    for k in range(args.warmup + args.steps):
        flops, secs, desc, thr = run_oracle_sample(inp, per_step_s)
        if k >= args.warmup:
            times.append(secs)
            flops_all.append(flops)
    value = sum(flops_all) / sum(times) / 1e12
    ms = 1e3 * sum(times) / len(times)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "N": w.N, "c_z": 128, "heads": 4, "head_dim": 32,
                   "orientations": list(w.orientations), "parallelism": "cpu oracle, rank 0"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": thr, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_ours(args, world, rank, local):
    from protein_pair_representation_layernorm_b200 import binding, workloads
    assert torch.cuda.is_available(), "bench.py needs a CUDA device"
    w = workloads.WORKLOADS[args.workload]
    inp = workloads.workload_inputs(args.workload)
    N = inp.N
    n_valid = N if inp.mask is None else int(inp.mask.sum())
    H, d = 4, 32
    flops_attn = 4.0 * N * N * n_valid * H * d          # one orientation
    exps_attn = float(N) * N * n_valid * H                # one exp2 per score
    flops_step = 2 * flops_attn
    blk = binding.TriangleAttention(inp.weights(), dtype=torch.bfloat16)
    st = torch.cuda.Stream()
    Z = inp.Z.cuda()
    mask = None if inp.mask is None else inp.mask.cuda()
    out1 = torch.empty_like(Z)
    out2 = torch.empty_like(Z)
    TIME = binding.TRI_ATTN_FLAG_TIME_KERNELS

    def step(flags):
        blk.forward(Z, binding.TRI_ATTN_STARTING, mask, out=out1, stream=st, flags=flags)
        blk.forward(out1, binding.TRI_ATTN_ENDING, mask, out=out2, stream=st, flags=flags)

    with torch.cuda.stream(st):
        for _ in range(args.warmup):
            step(0)
    st.synchronize()
    rc = blk.status(st)
    assert rc == binding.TRI_ATTN_OK, binding.tri_attn_status_string(rc)
    blk.kernel_times()  # reset the per-kernel record

    clocks = ClockSampler(local) if torch.cuda.is_available() else None
    barrier(world)
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(st)
    for _ in range(args.steps):
        step(TIME)
    ev1.record(st)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop() if clocks else None
    t_ms = ev0.elapsed_time(ev1)
    t_ms_max = max_over_ranks(t_ms, world)
    kms, kn = blk.kernel_times()
    rc = blk.status(st)
    assert rc == binding.TRI_ATTN_OK, binding.tri_attn_status_string(rc)
    # each orientation's kernels on their own, outside the timed region: 20
    # blocks of one orientation at a time, per-kernel CUDA events
    by_orient = {}
    for name, orient, src, dst in (("starting", binding.TRI_ATTN_STARTING, Z, out1),
                                   ("ending", binding.TRI_ATTN_ENDING, out1, out2)):
        with torch.cuda.stream(st):
            for _ in range(20):
                blk.forward(src, orient, mask, out=dst, stream=st, flags=TIME)
        st.synchronize()
        oms, on = blk.kernel_times()
        by_orient[name] = {k: oms[i] / max(on[i], 1)
                           for i, k in enumerate(("pair_ln_proj", "tri_attn_fwd", "gate_out"))}

    value = world * flops_step * args.steps / (t_ms_max / 1e3) / 1e12
    peak_tf, peak_gbs, peak_src = measured_peaks()
    attn_ms = kms[1] / max(kn[1], 1)
    attn_tf = flops_attn / (attn_ms / 1e3) / 1e12
    pairs = N * N
    proj_ms = kms[0] / max(kn[0], 1)
    gate_ms = kms[2] / max(kn[2], 1)
    # pair_ln_proj reads z (256 B a pair) and writes q, k, v (768 B) and the bias;
    # gate_out reads o and z (512 B) and writes out (256 B)
    proj_bytes = pairs * (256 + 768) + 4 * N * ((N + 63) // 64 * 64) * 2
    gate_bytes = pairs * (512 + 256)
    traffic = None
    if TRAFFIC["tri_attn_fwd.cuh"] == src_hash("tri_attn_fwd.cuh"):
        traffic = TRAFFIC["bytes_per_launch"]

    # ---- end to end through the host-buffer entry point (pinned memory): a
    # stream of e2e_steps independent problems, each uploaded from pinned host
    # memory, run through both blocks and downloaded, enqueued back to back with
    # tri_attn_forward_host_async so that one problem's upload and download
    # overlap another's computation; timed from before the first upload to
    # after the last download (CUDA events on the calls' stream, the end one
    # recorded once tri_attn_host_wait has returned).
    z_host = inp.Z.clone().pin_memory()
    o_host = torch.empty_like(z_host).pin_memory()
    mask_host = None if inp.mask is None else inp.mask.clone()
    if args.e2e_steps > 0:
        for _ in range(3):  # warm-up: allocates the three staging buffers
            blk.forward_host_async(z_host, [0, 1], mask_host, out=o_host, stream=st)
        assert blk.host_wait() == binding.TRI_ATTN_OK
    e_ms = 0.0
    if args.e2e_steps > 0:
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        a.record(st)
        for _ in range(args.e2e_steps):
            blk.forward_host_async(z_host, [0, 1], mask_host, out=o_host, stream=st)
        rc = blk.host_wait()
        assert rc == binding.TRI_ATTN_OK, binding.tri_attn_status_string(rc)
        b.record(st)
        b.synchronize()
        e_ms = max_over_ranks(a.elapsed_time(b) / args.e2e_steps, world)
    e2e_value = world * flops_step / (e_ms / 1e3) / 1e12 if args.e2e_steps > 0 else None
    h2d = Z.numel() * Z.element_size() + (0 if mask is None else N)
    d2h = Z.numel() * Z.element_size()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        flops, secs, desc, thr = run_oracle_sample(inp, 15.0)
        cpu = {"value": flops / secs / 1e12, "unit": UNIT, "cores": thr, "kind": "oracle",
               "sample": desc}

    launches = int(sum(kn))
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": t_ms_max / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "N": N, "c_z": 128, "heads": H, "head_dim": d,
                   "orientations": ["starting", "ending"],
                   "step": "starting-node block, then ending-node block on its output",
                   "global_batch": world, "l2": "inputs larger than L2 (Z is 604 MB)",
                   "parallelism": f"independent instance per GPU x{world}"},
        "pct_of_peak": {f"{peak_src}_bf16_{peak_tf:g}": 100.0 * value / world / peak_tf,
                        "datasheet_bf16_2250": 100.0 * value / world / DATASHEET_BF16_TFLOPS},
        "roofline": {"kernel": "tri_attn_fwd", "bound": "tensor", "achieved": attn_tf,
                     "peak": peak_tf, "unit": "TFLOP/s", "frac": attn_tf / peak_tf,
                     "peak_source": f"{peak_src} bf16_tflops (burst)", "traffic": traffic,
                     "traffic_source": (f"ncu dram__bytes_read.sum + dram__bytes_write.sum, "
                                        f"{TRAFFIC['measured_at']}") if traffic else None,
                     "algorithmic_flops_per_launch": flops_attn,
                     "launch_ms": attn_ms,
                     # the unit that caps the kernel at head width 32: one exp2 per
                     # score, three in four of them on the special-function unit (16
                     # per clock per SM, measured with a probe), at the maximum SM clock
                     "limiter": {"unit_name": "exp2 (special-function unit)",
                                 "achieved": EX2_SHARE * exps_attn / (attn_ms / 1e3),
                                 "peak": EX2_PER_CLK_SM * NUM_SMS * SM_MAX_MHZ * 1e6,
                                 "unit": "ex2/s",
                                 "frac": EX2_SHARE * exps_attn / (attn_ms / 1e3)
                                 / (EX2_PER_CLK_SM * NUM_SMS * SM_MAX_MHZ * 1e6),
                                 "peak_derivation": "16 ex2/clk/SM x 148 SMs x 1965 MHz; "
                                                    "3/4 of the exponentials on that unit"}},
        "kernels": {
            "pair_ln_proj": {"ms": proj_ms, "launches": kn[0],
                             "GB/s": proj_bytes / (proj_ms / 1e3) / 1e9,
                             "frac_hbm": proj_bytes / (proj_ms / 1e3) / 1e9 / peak_gbs},
            "tri_attn_fwd": {"ms": attn_ms, "launches": kn[1], "TFLOP/s": attn_tf,
                             "pair_rows_per_s": N / (attn_ms / 1e3)},
            "gate_out": {"ms": gate_ms, "launches": kn[2],
                         "GB/s": gate_bytes / (gate_ms / 1e3) / 1e9,
                         "frac_hbm": gate_bytes / (gate_ms / 1e3) / 1e9 / peak_gbs},
            "ms_by_orientation": by_orient,
        },
        "pair_rows_per_s": world * 2 * N * args.steps / (t_ms_max / 1e3),
        "clocks": clk,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e_ms,
                "steps": args.e2e_steps,
                "api": ("tri_attn_forward_host_async x e2e_steps + tri_attn_host_wait (pinned host "
                        "buffers, orientations [starting, ending]; consecutive problems' uploads "
                        "and downloads overlap each other's computation)")},
        "gpu_launches": launches,
        "cpu_baseline": cpu,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    blk.close()


def run_backward(args, rank):
    """Time the attention-core backward on the workload's N with every row, on
    synthetic q, k, v, dO and bias; prints one JSON line.  Default: the
    tensor-core path (tri_attn_attention_backward_bf16, after one
    tri_attn_attention_forward_bf16 for o and lse); --backward-f32: the fp32
    SIMT kernels (tri_attn_attention_backward).  Algorithmic work: 10 d flop
    per (row, head, query, unmasked key) score (S and dP, 2 d each, once;
    dQ, dK and dV, 2 d each)."""
    if rank != 0:
        return
    import ctypes

    from protein_pair_representation_layernorm_b200 import binding, workloads
    w = workloads.WORKLOADS[args.workload]
    inp = workloads.workload_inputs(args.workload)
    N = inp.N
    rows = N
    H, d = 4, 32
    tc = not args.backward_f32
    dt = torch.bfloat16 if tc else torch.float32
    gen = torch.Generator(device="cuda").manual_seed(17)
    Q, K, V, dO = (torch.randn(rows, H, N, d, device="cuda", generator=gen).to(dt)
                   for _ in range(4))
    bias = torch.randn(H, N, N, device="cuda", generator=gen).to(dt)
    mask = None if inp.mask is None else inp.mask.cuda().to(torch.uint8).contiguous()
    n_valid = N if inp.mask is None else int(inp.mask.sum())
    f32 = dict(dtype=torch.float32, device="cuda")
    dQ, dK, dV = (torch.empty(rows, H, N, d, **f32) for _ in range(3))
    dB = torch.empty(H, N, N, **f32)
    st = torch.cuda.Stream()
    P = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())  # noqa: E731
    sp = ctypes.c_void_p(st.cuda_stream)
    if tc:
        nbytes = binding.tri_attn_attention_bf16_workspace_bytes(rows, N)
        ws = torch.empty((nbytes + 15) // 16 * 4, **f32)
        O = torch.empty_like(Q)
        lse = torch.empty(rows, H, N, **f32)
        rc = binding.tri_attn_attention_forward_bf16(P(Q), P(K), P(V), P(bias), P(mask), rows, N,
                                                     P(O), P(lse), P(ws), nbytes, sp,
                                                     binding.TRI_ATTN_FLAG_SYNC)
        assert rc == binding.TRI_ATTN_OK, binding.tri_attn_status_string(rc)

        def step():
            rc = binding.tri_attn_attention_backward_bf16(
                P(Q), P(K), P(V), P(bias), P(mask), P(O), P(lse), P(dO), rows, N, P(dQ), P(dK),
                P(dV), P(dB), P(ws), nbytes, sp, 0)
            assert rc == binding.TRI_ATTN_OK, binding.tri_attn_status_string(rc)
        launches = 6  # prep_q, prep_bias, prep_rows, dQ, dK dV, dbias
    else:
        nbytes = binding.tri_attn_attention_backward_workspace_bytes(rows, N)
        ws = torch.empty(nbytes // 4, **f32)

        def step():
            rc = binding.tri_attn_attention_backward(P(Q), P(K), P(V), P(bias), P(mask), P(dO),
                                                     rows, N, P(dQ), P(dK), P(dV), P(dB), P(ws),
                                                     nbytes, sp, 0)
            assert rc == binding.TRI_ATTN_OK, binding.tri_attn_status_string(rc)
        launches = 4

    for _ in range(max(args.warmup, 1)):
        step()
    st.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(st)
    for _ in range(args.steps):
        step()
    ev1.record(st)
    ev1.synchronize()
    ms = ev0.elapsed_time(ev1) / args.steps
    flops = 10.0 * d * rows * N * n_valid * H
    tf = flops / (ms / 1e3) / 1e12
    if tc:
        peak_tf, _, peak_src = measured_peaks()
        roof = {"bound": "tensor", "achieved": tf, "peak": peak_tf, "unit": "TFLOP/s",
                "frac": tf / peak_tf, "peak_source": f"{peak_src} bf16_tflops (burst)"}
    else:
        # fp32 FFMA peak: 148 SMs x 128 lanes x 2 flop x 1965 MHz
        peak = 148 * 128 * 2 * 1.965e9 / 1e12
        roof = {"bound": "alu", "achieved": tf, "peak": peak, "unit": "TFLOP/s",
                "frac": tf / peak,
                "peak_derivation": "fp32 FFMA: 148 SMs x 128 lanes x 2 flop x 1965 MHz"}
    print(json.dumps({
        "metric": "attention-core backward TFLOP/s (algorithmic: 10 d flop per unmasked score)",
        "value": tf, "unit": "TFLOP/s", "ms_per_step": ms, "steps": args.steps,
        "warmup": max(args.warmup, 1), "higher_is_better": True,
        "dtype": "bf16" if tc else "f32", "data": "synthetic",
        "config": {"workload": w.name, "N": N, "rows": rows, "heads": H, "head_dim": d,
                   "path": "tensor cores (tcgen05)" if tc else "fp32 SIMT"},
        "roofline": roof, "gpu_launches": launches * args.steps}), flush=True)


def main():
    args = parse()
    world, rank, local = dist_setup(args)
    try:
        if args.backward:
            run_backward(args, rank)
        elif args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
