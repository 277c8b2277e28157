#!/usr/bin/env python
"""Benchmark of the W4A16 linear layer on B200.

Headline workload: the M=1 decode GEMV of the 8B MLP-up shape (M=1, K=4096,
N=14336, G=128, symmetric zp_bias=8, A ~ N(0,1), scales U[0.002, 0.02]).
One step = one w4a16_gemm call (host checks, kernel, split-K reduce, fp16
epilogue) on one batch of synthetic input. Metric: achieved HBM GB/s over the
algorithmic bytes (packed weights + scales + zeros + activations + output).

Timing: inputs are resident in HBM; each step reads a different copy of the
weights, R copies rotating with R * bytes > 2x L2, so every step streams its
weights from HBM (no L2 flush needed). Steps run back to back from a CUDA graph,
as the layers of a decode step would, with programmatic dependent launch: a step
may start streaming its weights while the previous one finishes, and reads its
activations only after it (--no-pdl turns this off; the line also reports the
per-step time without it). CUDA events on the launching stream bracket exactly
K steps, with a barrier and a device synchronize on both sides; the max over
ranks is taken.

Multi-GPU: the layer is run as independent replicas, one per GPU (weak scaling);
there is no collective on the data path.

--impl reference times the CPU oracle (the only other implementation) on this
machine's host cores, on the same workload, metric and unit.
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

import synth  # noqa: E402

METRIC = "W4A16 achieved HBM GB/s (M=1) and TFLOP/s (M=32) as fraction of roofline"
WORKLOADS = {
    "decode_m1": "decode GEMV M=1 K=4096 N=14336 G=128 sym zp_bias=8 (8B MLP-up shape)",
    "batch32": "batch-32 GEMM M=32 K=4096 N=14336 G=128 asym, weights repacked from [N,K/8]",
}
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 * 1024 * 1024


def alg_bytes(M, K, N, G, asym):
    return K * N // 2 + (K // G) * N * 2 + ((K // G) * N // 2 if asym else 0) + M * K * 2 + M * N * 2


def alg_flops(M, K, N):
    return 2 * M * K * N


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def code_only(text):
    """C/CUDA source with its comments removed and every run of whitespace outside string and
    character literals made one space, so that a change to comments or layout alone does not count
    as a change of the code (literals, inline assembly included, are kept as written)."""
    parts, code, i, n = [], [], 0, len(text)

    def flush():
        parts.append(" ".join("".join(code).split()))
        code.clear()

    while i < n:
        c = text[i]
        if c in "\"'":                                   # string or character literal, kept whole
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            flush()
            parts.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
            code.append(" ")
        else:
            code.append(c)
            i += 1
    flush()
    return " ".join(p for p in parts if p)


def csrc_hash(files=None):
    """Hash of the code (comments and layout ignored) of the library sources a kernel is compiled
    from (all of csrc/ when files is None)."""
    h = hashlib.sha256()
    d = os.path.join(ROOT, "weight_only_int4_08_b200", "csrc")
    for f in sorted(files or os.listdir(d)):
        h.update(code_only(open(os.path.join(d, f), encoding="utf-8").read()).encode())
    return h.hexdigest()[:16]


def traffic_from_profiles(kernel_key):
    """DRAM bytes per launch from the committed ncu summary, if the sources of that kernel (its
    translation unit and the headers it includes) are the ones it was taken on."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    e = d.get(kernel_key)
    if not e or e.get("csrc_hash") != csrc_hash(e.get("files")):
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        fd, self.path = tempfile.mkstemp(prefix=f"w4a16_clocks_rank{index}_", suffix=".csv")
        os.close(fd)

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
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
        self.f.close()
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 9 and parts[1].replace(".", "").isdigit():
                rows.append(parts)
        try:
            os.remove(self.path)
        except OSError:
            pass
        if not rows:
            return None
        sm = [float(r[1]) for r in rows]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for n, v in zip(names, r[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": float(rows[0][2]), "samples": len(rows),
                "reasons": sorted(reasons)}


# ----------------------------------------------------------------------------- GPU arm

def to_dev(x, torch):
    x = np.ascontiguousarray(x)
    if x.dtype == np.float16:
        return torch.from_numpy(x).cuda()
    return torch.from_numpy(x.view(np.int32)).cuda()


class Problem:
    """One GEMM shape resident on the device with R rotating weight copies."""

    def __init__(self, w, torch, case, copies, b=None):
        self.w, self.torch = w, torch
        self.M, self.K, self.N, self.G = case["M"], case["K"], case["N"], case["G"]
        self.zp = case["zp_bias"]
        self.asym = case["z"] is not None
        self.a = to_dev(case["a"], torch)
        b0 = b if b is not None else to_dev(case["b"], torch)
        s0, z0 = to_dev(case["s"], torch), (to_dev(case["z"], torch) if self.asym else None)
        self.bs = [b0] + [b0.clone() for _ in range(copies - 1)]
        self.ss = [s0] + [s0.clone() for _ in range(copies - 1)]
        self.zs = [z0] * copies if z0 is None else [z0] + [z0.clone() for _ in range(copies - 1)]
        self.out = torch.empty((self.M, self.N), dtype=torch.float32 if self.out_f32 else torch.float16,
                               device="cuda")
        self.ws = w.alloc_workspace(self.M, self.N, self.K, self.G)
        self.i = 0
        self.bytes = alg_bytes(self.M, self.K, self.N, self.G, self.asym)
        self.flops = alg_flops(self.M, self.K, self.N)

    pdl = True  # back-to-back steps read weights no step writes: programmatic dependent launch is valid
    out_f32 = False  # a row shard of a tensor-parallel layer writes fp32 partials

    def step(self, stream=None):
        j = self.i % len(self.bs)
        self.i += 1
        self.w.w4a16_gemm(self.a, self.bs[j], self.ss[j], self.zs[j], self.G, self.zp, out=self.out,
                          workspace=self.ws, stream=stream, pdl=self.pdl, out_f32=self.out_f32)

    def launches_per_step(self):
        # The library's automatic choice: tensor-core GEMM (one launch per 128 rows) above 16 rows,
        # otherwise the GEMV (one launch).
        return (self.M + 127) // 128 if uses_tc(self.M, self.N, self.K) else (self.M + 15) // 16


def copies_for(bytes_per_copy):
    return max(2, int(np.ceil(2 * L2_BYTES / bytes_per_copy)) + 1)


def uses_tc(M, N, K=4096):
    """The library's automatic kernel choice for an aligned problem (see w4a16_api.cu): the
    tensor-core GEMM above 16 rows, for any N and K that meet its shape rules."""
    return M > 16


def capture(torch, fn, n):
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()  # make sure everything is initialised outside capture
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    with torch.cuda.graph(g):
        for _ in range(n):
            fn()
    return g


def time_graph(torch, g, reps):
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record()
    for _ in range(reps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / 1e3


def measure_problem(torch, prob, steps_per_graph, reps):
    g = capture(torch, prob.step, steps_per_graph)
    time_graph(torch, g, 3)
    t = time_graph(torch, g, reps)
    per = t / (reps * steps_per_graph)
    del g
    return per


def summary(prob, per_step_s, peaks, tensor_bound):
    gbs = prob.bytes / per_step_s / 1e9
    tfs = prob.flops / per_step_s / 1e12
    # every path multiplies on the tensor cores (mma.sync for M <= 32, tcgen05 above)
    t_hbm = prob.bytes / (peaks["hbm_gbs"] * 1e9)
    t_tc = prob.flops / (peaks["bf16_tflops"] * 1e12)
    t_roof = max(t_hbm, t_tc)
    return {"us": round(per_step_s * 1e6, 3), "GB/s": round(gbs, 1), "TFLOP/s": round(tfs, 2),
            "roofline_us": round(t_roof * 1e6, 3), "frac_of_roofline": round(t_roof / per_step_s, 4)}


def max_over_ranks(dist, world, seconds, device):
    """The job's time: the largest of the ranks' local times, returned on every rank."""
    if world <= 1:
        return seconds
    import torch
    t = torch.tensor([seconds], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbs(world, steps, bytes_per_step, seconds):
    """Whole-job throughput: each of the `world` ranks ran `steps` steps of `bytes_per_step`."""
    return world * steps * bytes_per_step / seconds / 1e9


def run_gpu(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))

    def barrier():
        if world > 1:
            dist.barrier()

    import weight_only_int4_08_b200 as w
    peaks, peak_src = load_peaks()
    Problem.pdl = args.pdl

    if args.workload == "batch32":
        # batch-32 asymmetric GEMM (tensor cores), weights repacked from the checkpoint layout
        case = synth.config4()
        b_kn8 = w.w4a16_repack(to_dev(case["ckpt"], torch), case["N"], case["K"])
        prob = Problem(w, torch, case, copies_for(alg_bytes(32, case["K"], case["N"], case["G"], True)), b=b_kn8)
    else:
        case = synth.config2()
        prob = Problem(w, torch, case, copies_for(alg_bytes(1, case["K"], case["N"], case["G"], False)))
    K_steps, W_steps = args.steps, args.warmup

    # warm-up: W untimed steps
    for _ in range(W_steps):
        prob.step()
    torch.cuda.synchronize()

    chunk = min(K_steps, 256)
    g_main = capture(torch, prob.step, chunk)
    tail = K_steps % chunk
    g_tail = capture(torch, prob.step, tail) if tail else None
    # The first replay of a graph uploads it to the device; do that outside the timed region.
    g_main.replay()
    if g_tail is not None:
        g_tail.replay()
    torch.cuda.synchronize()

    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(K_steps // chunk):
        g_main.replay()
    if g_tail is not None:
        g_tail.replay()
    e1.record()
    torch.cuda.synchronize()
    barrier()
    t_local = e0.elapsed_time(e1) / 1e3
    # keep the same work running so the clock record has samples under load
    t_keep = time.time()
    while time.time() - t_keep < max(0.0, 1.0 - t_local):
        for _ in range(16):
            g_main.replay()
        torch.cuda.synchronize()
    clocks = sampler.stop()

    t_max = max_over_ranks(dist, world, t_local, "cuda")
    per_step = t_max / K_steps
    value = whole_job_gbs(world, K_steps, prob.bytes, t_max)

    # e2e: through the public API with pinned host buffers; H2D of the step's
    # activations and D2H of its output inside the timed region, every step.
    a_host = torch.from_numpy(np.ascontiguousarray(case["a"])).pin_memory()
    out_host = torch.empty((case["M"], case["N"]), dtype=torch.float16).pin_memory()
    a_dev = torch.empty_like(prob.a)
    e2e_steps = min(max(K_steps, 50), 2000)

    def e2e_step():
        a_dev.copy_(a_host, non_blocking=True)
        j = prob.i % len(prob.bs)
        prob.i += 1
        w.w4a16_gemm(a_dev, prob.bs[j], prob.ss[j], prob.zs[j], prob.G, prob.zp, out=prob.out, workspace=prob.ws)
        out_host.copy_(prob.out, non_blocking=True)

    for _ in range(5):
        e2e_step()
    torch.cuda.synchronize()
    barrier()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record()
    for _ in range(e2e_steps):
        e2e_step()
    f1.record()
    torch.cuda.synchronize()
    barrier()
    te = max_over_ranks(dist, world, f0.elapsed_time(f1) / 1e3, "cuda")
    e2e_value = whole_job_gbs(world, e2e_steps, prob.bytes, te)

    # kernel duration for the roofline: graph of back-to-back launches, CUDA events
    per_launch = measure_problem(torch, prob, 256, 40)
    # the same without programmatic dependent launch (each call waits for the previous to end)
    Problem.pdl = False
    per_launch_plain = measure_problem(torch, prob, 256, 40)
    Problem.pdl = args.pdl
    achieved = prob.bytes / per_launch / 1e9
    hbm_peak = float(peaks["hbm_gbs"])
    kernel_name = "tc_gemm_kernel<32, true>" if args.workload == "batch32" else "gemv_sk_kernel<8, 1, true>"
    traffic = traffic_from_profiles("tc_m32_k4096_n14336" if args.workload == "batch32" else "gemv_m1_k4096_n14336")
    if traffic is not None:  # per step, like `achieved`
        traffic = traffic * prob.launches_per_step()

    extras = {}
    if rank == 0 and not args.no_extras:
        extras = run_extras(torch, w, peaks)

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC,
        "value": round(value, 1),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": K_steps,
        "warmup": W_steps,
        "ms_per_step": round(per_step * 1e3, 6),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "fp16 in, fp32 accumulate (int4 weights)",
        "data": "synthetic (seeded; shapes and distributions of the 8B MLP-up decode GEMV)",
        "config": {"workload": WORKLOADS[args.workload],
                   "parallelism": f"replicas x{world}",
                   "l2": f"inputs larger than L2: {len(prob.bs)} rotating weight copies "
                         f"({len(prob.bs) * prob.bytes / 1e6:.0f} MB)",
                   "timing": "CUDA graph of back-to-back steps, CUDA events on the launching stream"},
        "no_pdl": {"us_per_step": round(per_launch_plain * 1e6, 3),
                   "GB/s": round(prob.bytes / per_launch_plain / 1e9, 1)},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm_peak, "unit": "GB/s",
                     "frac": round(achieved / hbm_peak, 4), "traffic": traffic,
                     "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)" if peak_src == "measured" else peak_src,
                     "kernel": kernel_name, "alg_bytes_per_launch": prob.bytes,
                     "us_per_launch": round(per_launch * 1e6, 3)},
        "e2e": {"value": round(e2e_value, 1), "unit": "GB/s", "h2d_bytes_per_step": int(a_host.numel() * 2),
                "d2h_bytes_per_step": int(out_host.numel() * 2), "steps": e2e_steps},
        "gpu_launches": K_steps * prob.launches_per_step(),
        "clocks": clocks,
    }
    if extras:
        line["extra"] = extras
    if args.cpu_baseline and world == 1:
        line["cpu_baseline"] = cpu_baseline(case, seconds=args.cpu_seconds)
    print(json.dumps(line), flush=True)


def run_extras(torch, w, peaks):
    """The other workloads: small-batch sweep, batch-32 with repack (and the whole-layer load), 32-layer stack."""
    ex = {}
    for M in (1, 2, 4, 8, 16):
        c = synth.config3(M)
        p = Problem(w, torch, c, copies_for(alg_bytes(M, 4096, 4096, 128, True)))
        ex[f"config3_M{M}"] = summary(p, measure_problem(torch, p, 64, 20), peaks, tensor_bound=M >= 9)
        del p
    c = synth.config4()
    ck = to_dev(c["ckpt"], torch)
    bkn = torch.empty((c["K"], c["N"] // 8), dtype=torch.int32, device="cuda")
    cks = [ck] + [ck.clone() for _ in range(3)]
    outs = [bkn] + [bkn.clone() for _ in range(3)]
    state = {"i": 0}

    def rp():
        j = state["i"] % 4
        state["i"] += 1
        w.w4a16_repack(cks[j], c["N"], c["K"], out=outs[j])

    per = measure_problem(torch, type("P", (), {"step": staticmethod(rp)})(), 16, 10)
    rbytes = 2 * c["N"] * c["K"] // 2
    ex["config4_repack"] = {"us": round(per * 1e6, 3), "GB/s": round(rbytes / per / 1e9, 1),
                            "frac_of_roofline": round(rbytes / (peaks["hbm_gbs"] * 1e9) / per, 4)}
    del cks, outs
    ex["config4_load_ct"] = measure_load_ct(torch, w, peaks)
    p = Problem(w, torch, c, copies_for(alg_bytes(32, 4096, 14336, 128, True)), b=bkn)
    ex["config4_M32"] = summary(p, measure_problem(torch, p, 16, 20), peaks, tensor_bound=True)
    del p
    # larger batches on the same layer (tensor-core GEMM)
    for M in (64, 128, 256):
        cm = synth.make_case(M, 4096, 14336, 128, sym=False, seed=3)
        p = Problem(w, torch, cm, copies_for(alg_bytes(M, 4096, 14336, 128, True)))
        ex[f"config4_M{M}"] = summary(p, measure_problem(torch, p, 16, 20), peaks, tensor_bound=True)
        del p
    ex.update(run_tp(torch, w, peaks))
    ex.update(run_stack(torch, w, peaks))
    return ex


def run_tp(torch, w, peaks):
    """One rank's share of the decode layer (M=1, K=4096, N=14336, G=128) under P-way tensor
    parallelism, for P = 2, 4, 8: its column shard (N/P output columns), its row shard (K/P rows,
    fp32 partial) and the reduction of P partials that closes a row-parallel layer. The
    collective that brings the partials together is not part of it (one GPU here)."""
    res = {}
    c = synth.config2()
    K, N, G = c["K"], c["N"], c["G"]
    for P in (2, 4, 8):
        nc, kr = N // P, K // P
        col = dict(c, N=nc, b=c["b"][:, :nc // 8], s=c["s"][:, :nc])
        row = dict(c, K=kr, a=np.ascontiguousarray(c["a"][:, :kr]), b=c["b"][:kr], s=c["s"][:kr // G])
        pc = Problem(w, torch, col, copies_for(alg_bytes(1, K, nc, G, False)))
        t_col = measure_problem(torch, pc, 64, 20)
        del pc
        Problem.out_f32 = True
        try:
            pr = Problem(w, torch, row, copies_for(alg_bytes(1, kr, N, G, False)))
            t_row = measure_problem(torch, pr, 64, 20)
        finally:
            Problem.out_f32 = False
        del pr
        parts = [torch.randn((1, N), dtype=torch.float32, device="cuda") for _ in range(P)]
        red_out = torch.empty((1, N), dtype=torch.float16, device="cuda")

        def red(parts=parts, red_out=red_out):
            w.w4a16_reduce_partials(parts, out=red_out)

        t_red = measure_problem(torch, type("P", (), {"step": staticmethod(red)})(), 64, 20)
        roof_col = alg_bytes(1, K, nc, G, False) / (peaks["hbm_gbs"] * 1e9)
        roof_row = alg_bytes(1, kr, N, G, False) / (peaks["hbm_gbs"] * 1e9)
        res[f"tp{P}_decode_rank"] = {"col_shard_us": round(t_col * 1e6, 3),
                                     "col_frac_of_roofline": round(roof_col / t_col, 4),
                                     "row_shard_us": round(t_row * 1e6, 3),
                                     "row_frac_of_roofline": round(roof_row / t_row, 4),
                                     "reduce_us": round(t_red * 1e6, 3),
                                     "row_plus_reduce_us": round((t_row + t_red) * 1e6, 3)}
    return res


def measure_load_ct(torch, w, peaks):
    """The batch-32 workload's layer loaded from the checkpoint layout (weight, scales, zeros) in one launch;
    four copies rotate so every call reads and writes 30 MB that are not in L2."""
    K, N, G = 4096, 14336, 128
    c = synth.ct_checkpoint(K, N, G, sym=False, seed=3)
    ins = [(to_dev(c["ckpt"], torch), to_dev(c["s_ng"], torch), to_dev(c["z_n8g"], torch)) for _ in range(4)]
    outs = [(torch.empty((K, N // 8), dtype=torch.int32, device="cuda"),
             torch.empty((K // G, N), dtype=torch.float16, device="cuda"),
             torch.empty((K // G, N // 8), dtype=torch.int32, device="cuda")) for _ in range(4)]
    state = {"i": 0}

    def ld():
        j = state["i"] % 4
        state["i"] += 1
        w.w4a16_load_ct(*ins[j], N, K, G, out=outs[j])

    per = measure_problem(torch, type("P", (), {"step": staticmethod(ld)})(), 16, 10)
    nbytes = 2 * (N * K // 2 + N * (K // G) * 2 + (N // 8) * (K // G) * 4)   # read + write of each tensor
    return {"us": round(per * 1e6, 3), "GB/s": round(nbytes / per / 1e9, 1),
            "frac_of_roofline": round(nbytes / (peaks["hbm_gbs"] * 1e9) / per, 4)}


def run_stack(torch, w, peaks):
    """32 layers x (qkv, o, gate_up, down) linears, one CUDA graph per pass, M = 1 and 32."""
    res = {}
    layers = []
    for layer in range(synth.N_LAYERS):
        row = []
        for idx in range(4):
            c = synth.config5_linear(layer, idx, 1)
            row.append((to_dev(c["b"], torch), to_dev(c["s"], torch), c["K"], c["N"]))
        layers.append(row)
    for M in (1, 32):
        acts = [[to_dev(synth.config5_linear(0, idx, M)["a"], torch) for idx in range(4)]]
        outs = [torch.empty((M, n), dtype=torch.float16, device="cuda") for (_, _, _, n) in layers[0]]
        wss = [w.alloc_workspace(M, n, k, 128) for (_, _, k, n) in layers[0]]

        def one_pass():
            for row in layers:
                for idx, (b, s, k, n) in enumerate(row):
                    w.w4a16_gemm(acts[0][idx], b, s, None, 128, 8, out=outs[idx], workspace=wss[idx], pdl=True)

        g = capture(torch, one_pass, 1)
        time_graph(torch, g, 2)
        t = time_graph(torch, g, 10) / 10
        del g
        # Gap analysis: each linear alone, its 32 layers back to back (the same calls as in the pass);
        # t_sum is what the pass would take if the four shapes cost what they cost alone.
        per_linear = {}
        for idx, name in enumerate(("qkv", "o", "gate_up", "down")):
            def one_linear(idx=idx):
                for row in layers:
                    b, s, k, n = row[idx]
                    w.w4a16_gemm(acts[0][idx], b, s, None, 128, 8, out=outs[idx], workspace=wss[idx], pdl=True)
            gl = capture(torch, one_linear, 1)
            time_graph(torch, gl, 2)
            per_linear[name] = time_graph(torch, gl, 10) / 10 / synth.N_LAYERS
            del gl
        t_sum = synth.N_LAYERS * sum(per_linear.values())
        byts = sum(alg_bytes(M, k, n, 128, False) for row in layers for (_, _, k, n) in row)
        flops = sum(alg_flops(M, k, n) for row in layers for (_, _, k, n) in row)
        t_roof = max(byts / (peaks["hbm_gbs"] * 1e9), flops / (peaks["bf16_tflops"] * 1e12))
        res[f"config5_stack_M{M}"] = {"us": round(t * 1e6, 1), "GB/s": round(byts / t / 1e9, 1),
                                      "TFLOP/s": round(flops / t / 1e12, 2), "roofline_us": round(t_roof * 1e6, 1),
                                      "frac_of_roofline": round(t_roof / t, 4), "launches": 128,
                                      "t_sum_us": round(t_sum * 1e6, 1),
                                      "per_linear_us": {k: round(v * 1e6, 2) for k, v in per_linear.items()}}
    return res


# ----------------------------------------------------------------------------- CPU oracle

def host_cpu_model():
    """The host CPU's model name (from /proc/cpuinfo), or the platform's processor string."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.lower().startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown CPU"


def cpu_baseline(case, seconds=10.0):
    import oracle
    # the batch workload's weights are drawn in the checkpoint layout: the oracle repacks them
    b = case["b"] if case.get("b") is not None else oracle.repack(case["ckpt"], case["N"], case["K"])
    oracle.gemm(case["a"], b, case["s"], case["z"], case["G"], case["zp_bias"])  # load/build
    n, t0 = 0, time.perf_counter()
    while True:
        oracle.gemm(case["a"], b, case["s"], case["z"], case["G"], case["zp_bias"])
        n += 1
        if time.perf_counter() - t0 >= seconds:
            break
    dt = (time.perf_counter() - t0) / n
    byts = alg_bytes(case["M"], case["K"], case["N"], case["G"], case["z"] is not None)
    return {"value": round(byts / dt / 1e9, 3), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"{n} full GEMMs of the M={case['M']} K={case['K']} N={case['N']} workload, "
                      f"{dt * 1e3:.1f} ms each, 1 thread of {os.cpu_count()} host cores ({host_cpu_model()})"}


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    case = synth.config2()
    oracle.gemm(case["a"], case["b"], case["s"], case["z"], case["G"], case["zp_bias"])
    for _ in range(args.warmup):
        oracle.gemm(case["a"], case["b"], case["s"], case["z"], case["G"], case["zp_bias"])
    # each step: the full M=1 workload once (about 0.7 s on one core); bounded step count
    steps = max(1, min(args.steps, 30))
    t0 = time.perf_counter()
    for _ in range(steps):
        oracle.gemm(case["a"], case["b"], case["s"], case["z"], case["G"], case["zp_bias"])
    dt = time.perf_counter() - t0
    byts = alg_bytes(1, case["K"], case["N"], case["G"], False)
    value = steps * byts / dt / 1e9
    line = {"metric": METRIC, "value": round(value, 3), "unit": "GB/s", "impl": "reference", "n_gpus": world,
            "steps": steps, "warmup": args.warmup, "ms_per_step": round(dt / steps * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "fp32 (CPU oracle)",
            "data": "synthetic", "config": {"workload": "decode GEMV M=1 K=4096 N=14336 G=128 sym zp_bias=8 (8B MLP-up shape)"},
            "cpu_baseline": {"value": round(value, 3), "unit": "GB/s", "cores": 1, "kind": "oracle",
                             "sample": f"{steps} full GEMMs of the workload on 1 of {os.cpu_count()} host cores "
                                       f"({host_cpu_model()})"},
            "e2e": {"value": round(value, 3), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-extras", action="store_true")
    ap.add_argument("--no-pdl", dest="pdl", action="store_false",
                    help="launch every step only after the previous one has finished")
    ap.add_argument("--no-cpu-baseline", dest="cpu_baseline", action="store_false")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--workload", default="decode_m1", choices=["decode_m1", "batch32"],
                    help="headline problem: the M=1 decode GEMV (default) or the batch-32 GEMM")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
