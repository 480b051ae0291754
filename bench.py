"""Benchmark: Gated DeltaNet forward + backward tokens/s on B200.

One step = gdn_fwd + gdn_bwd (the whole hot path) over one batch of the
workload B=4, T=4096, H=16, d_k=d_v=128, bf16 inputs, fp32 gates/state, with
inputs resident in HBM.  Each rank runs its own seeded batch (independent
problems, no collective on the data path): weak scaling.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line on rank 0.  ``--impl reference`` times the fp64 CPU
oracle (the only other implementation of this layer here) on the host cores
over a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "GDN fwd+bwd tokens/s (B=4,T=4K,H=16,d=128 bf16); % of TC/HBM roofline"
WORKLOAD = dict(B=4, T=4096, H=16, K=128, V=128, dtype="bf16", gate_scale=0.1, h0_std=0.02,
                seed=2, bwd=True)
C = 64


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--mode", choices=("fwdbwd", "decode", "report"), default="fwdbwd",
                    help="decode: the recurrent decode step; report: every workload's "
                         "throughput (neither is the headline line)")
    ap.add_argument("--shape", default=None,
                    help="B,T,H override of the workload (profiling and size sweeps only)")
    return ap.parse_args()


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return dict(hbm=p["hbm_gbs"], tc=p["bf16_tflops"], tc_sus=p["bf16_tflops_sustained"],
                    sm_mhz=p.get("sm_max_mhz", 1965.0), src="measured")
    except Exception:
        return dict(hbm=6650.0, tc=1590.0, tc_sus=1400.0, sm_mhz=1965.0, src="fallback")


# ------------------------------------------------------------------ roofline
def kernel_work(name, w, n_chunks):
    """Algorithmic work of one launch of a kernel on workload w: (bound, amount, unit).
    Bytes are the tensors the step must move for that kernel; flops the
    chunkwise products the kernel is defined to compute (per chunk-head unit
    times chunk-heads)."""
    K, V, H = w["K"], w["V"], w["H"]
    ch = n_chunks * H
    f2 = lambda m, n, k: 2.0 * m * n * k
    table = {
        "simt_prep": f2(C, C, K) + C ** 3 / 3 + f2(C, K, C) + f2(C, V, C),
        "simt_state_fwd": f2(C, V, K) + f2(K, V, C),
        "simt_out": f2(C, C, K) + f2(C, V, K) + f2(C, V, C),
        "simt_duloc": f2(C, C, K) + f2(C, V, C),
        "simt_state_bwd": f2(C, V, K) + 2 * f2(K, V, C),
        "simt_grads": 8 * f2(C, C, K) + 3 * f2(C, C, V) + 3 * f2(C, K, V) + 2 * f2(C, C, C),
    }
    if name in table:
        return "alu", table[name] * ch, "flop"
    th = w["B"] * w["T"] * w["H"]  # token-heads
    # tensor-core path: HBM-facing kernels report the tensors the method must
    # move through them (bytes per token-head), chain kernels their MMA flops
    hbm = {"tc_grads": 4 * 2 * K + 8 + 3 * 2 * K + 8,   # q,k,v,do + g,b in; dq,dk,dv + dg,db out
           "tc_prep": 2 * (2 * K + V) + 8,              # q, k, v, g, b
           "tc_prep_local": 2 * (2 * K + V) + 8,        # the same step in the backward
           "tc_out": 2 * V}                             # o out (its inputs are intermediates)
    if name in hbm:
        return "hbm", float(hbm[name]) * th, "B"
    # the forward chain also forms the output: O^T = S Qg^T + U^T P^T per chunk
    chain = {"tc_state_fwd": 2 * f2(C, V, K) + f2(C, V, K) + f2(C, V, C),
             "tc_chains": 5 * f2(C, V, K)}
    if name in chain:
        return "tensor", chain[name] * ch, "flop"
    return None, None, None


def _code_only(text: str) -> str:
    """C/C++ source without its comments and blank lines (string literals kept)."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c in "\"'":  # a literal, escapes included
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            while i < n and text[i] != "\n":
                i += 1
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    lines = [ln.rstrip() for ln in "".join(out).splitlines()]
    return "\n".join(ln for ln in lines if ln)


def csrc_hash() -> str:
    """Hash of the code (comments and blank lines aside) of the CUDA sources and the
    ABI header: ties recorded ncu traffic to a build."""
    import glob
    import hashlib
    h = hashlib.sha1()
    files = sorted(glob.glob(os.path.join(ROOT, "gated_delta_rule_99_b200", "csrc", "*.cu")) +
                   glob.glob(os.path.join(ROOT, "gated_delta_rule_99_b200", "csrc", "*.cuh")) +
                   glob.glob(os.path.join(ROOT, "include", "*.h")))
    for f in files:
        h.update(os.path.basename(f).encode())
        with open(f, encoding="utf-8") as fh:
            h.update(_code_only(fh.read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes of all of a kernel's launches in one step, from profiles/traffic.md,
    or None if the sources changed since the capture."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.md")) as f:
            lines = f.read().splitlines()
    except OSError:
        return None
    cur = csrc_hash()
    for ln in lines:
        cells = [c.strip() for c in ln.strip().strip("|").split("|")]
        if len(cells) == 5 and cells[0] == kernel and cells[3] == cur and cells[4] == workload:
            return int(cells[1]) + int(cells[2])
    return None


def alu_peak_tflops(sm_mhz):
    # 148 SMs x 128 fp32 lanes x 2 flop (FMA) per clock
    return 148 * 128 * 2 * sm_mhz * 1e6 / 1e12


def step_roofline(w, pk):
    """Whole-step binding roofline (method flops and bytes per token-head)."""
    K, V = w["K"], w["V"]
    th = w["B"] * w["T"] * w["H"]
    fwd_f = 2 * C * (3 * K + 2 * V) + 6 * K * V + C * C / 3
    bwd_f = 9 * 2 * C * K + 5 * 2 * C * V + 8 * 2 * K * V + 4 * C * C
    flops = (fwd_f + bwd_f) * th
    bytes_ = (1032 + 1808) * th + 3 * w["B"] * w["H"] * K * V * 4
    # the burst tensor peak: a step lasts about a millisecond, far from the seconds-long
    # loop the sustained figure was measured over
    t_tc = flops / (pk["tc"] * 1e12)
    t_hbm = bytes_ / (pk["hbm"] * 1e9)
    return dict(flops=flops, bytes=bytes_, t_tc_s=t_tc, t_hbm_s=t_hbm,
                bound="tensor" if t_tc > t_hbm else "hbm", t_bound_s=max(t_tc, t_hbm))


# ------------------------------------------------------------------ clocks
class ClockSampler:
    def __init__(self, uuid):
        self.uuid, self.proc, self.lines = uuid, None, []

    def __enter__(self):
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        cmd = ["nvidia-smi", "--query-gpu=" + q, "--format=csv,noheader,nounits", "-lms", "100"]
        if self.uuid:
            cmd += ["-i", self.uuid]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        return False

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": ["unavailable"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ CPU oracle
_ORACLE_INPUTS = {}


def cpu_oracle_sample(units_n, min_s=0.0, max_passes=1):
    """Time the fp64 oracle (fwd + bwd) on `units_n` (row, head) units of the
    workload, repeated in passes until `min_s` seconds have run (at most
    `max_passes`); returns (seconds, units processed, threads, tokens-equivalent)."""
    import oracle
    from gated_delta_rule_99_b200.inputs import make_inputs
    w = dict(WORKLOAD)
    if "inp" not in _ORACLE_INPUTS:  # drawn once, outside every timed call
        _ORACLE_INPUTS["inp"] = make_inputs(**w)
    inp = _ORACLE_INPUTS["inp"]
    allu = [(b, h) for b in range(w["B"]) for h in range(w["H"])]
    units = allu[:units_n]
    threads = oracle.default_threads()
    oracle.build()
    t0 = time.perf_counter()
    passes = 0
    while True:
        oracle.gdn_fwd(inp.q, inp.k, inp.v, inp.g, inp.beta, h0=inp.h0, units=units,
                       nthreads=threads)
        oracle.gdn_bwd(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.do, h0=inp.h0, dhT=inp.dhT,
                       units=units, nthreads=threads)
        passes += 1
        dt = time.perf_counter() - t0
        if dt >= min_s or passes >= max_passes:
            break
    n = passes * len(units)
    tokens = n * w["T"] / w["H"]  # one token of the metric spans H heads
    return dt, n, threads, tokens


def oracle_units_for_cores():
    import oracle
    return max(1, min(64, oracle.default_threads()))


# ------------------------------------------------------------------ ranks
def rank_seed(rank: int) -> int:
    """Each rank draws its own batch: independent problems, no data exchange."""
    return WORKLOAD["seed"] + rank


def max_over_ranks(value_ms: float, world: int, device) -> float:
    """The job's time is the slowest rank's (a MAX all-reduce; identity at N = 1)."""
    import torch
    t = torch.tensor([value_ms], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(tokens_per_rank: int, world: int, steps: int, max_ms: float) -> float:
    """Whole-job throughput: every rank's tokens over the max-over-ranks time."""
    return world * tokens_per_rank * steps / (max_ms / 1e3)


# ------------------------------------------------------------------ main arms
def run_reference(args, rank, world):
    if rank != 0:
        return
    n_units = oracle_units_for_cores()
    for _ in range(max(0, args.warmup)):
        cpu_oracle_sample(n_units)
    times, tokens, threads = [], 0.0, 1
    for _ in range(args.steps):
        dt, nu, threads, tk = cpu_oracle_sample(n_units)
        times.append(dt)
        tokens += tk
    total = sum(times)
    val = tokens / total
    sample = ("%d (row, head) units of 4096 tokens, fp64 token-recurrence forward+backward per "
              "step; tokens/s counts units*T/H" % n_units)
    line = {"metric": METRIC, "value": val, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": "gdn_fwdbwd_bf16_B4_T4096_H16_d128", "global_batch": 4,
                       "seq_len": 4096, "heads": 16, "head_dim": 128, "parallelism": "none"},
            "cpu_baseline": {"value": val, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import gated_delta_rule_99_b200 as gdn
    from gated_delta_rule_99_b200.inputs import make_inputs

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = dict(WORKLOAD)
    if args.shape:
        w["B"], w["T"], w["H"] = (int(x) for x in args.shape.split(","))
    w["seed"] = rank_seed(rank)
    inp = make_inputs(device="cpu", **w)
    d = inp.to(dev)
    B, T, H, K, V = w["B"], w["T"], w["H"], w["K"], w["V"]
    desc = gdn.make_desc(B, T, H, K, V)
    ws = gdn.alloc_workspace(max(gdn.fwd_workspace_size(desc), gdn.bwd_workspace_size(desc)), dev)
    o = torch.empty(B, T, H, V, dtype=torch.bfloat16, device=dev)
    hT = torch.empty(B, H, K, V, dtype=torch.float32, device=dev)
    grads = (torch.empty_like(d.q), torch.empty_like(d.k), torch.empty_like(d.v),
             torch.empty_like(d.g), torch.empty_like(d.beta), torch.empty_like(d.h0))
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        gdn.gdn_fwd(d.q, d.k, d.v, d.g, d.beta, h0=d.h0, o=o, hT=hT, workspace=ws)
        gdn.gdn_bwd(d.q, d.k, d.v, d.g, d.beta, d.do, h0=d.h0, dhT=d.dhT, grads=grads,
                    workspace=ws)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    if gdn.device_status(ws) != 0:
        raise RuntimeError("device status not ok after warm-up")

    n_chunks = B * ((T + C - 1) // C)
    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    trace = gdn.LaunchTrace(capacity=64 * args.steps)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(uuid if rank == 0 else None) as clk:
        with trace:
            for i in range(args.steps):
                flush.zero_()  # L2 flush (256 MiB > 126 MB L2), outside the step events
                evs[i][0].record(stream)
                step()
                evs[i][1].record(stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
    step_ms = [a.elapsed_time(b) for a, b in evs]
    tot_ms = max_over_ranks(sum(step_ms), world, dev)
    status = gdn.device_status(ws)
    if status != 0:
        raise RuntimeError("device status %d after timed steps" % status)
    per_kernel = trace.per_kernel()
    launches = trace.count

    # ---- e2e: host buffers, H2D + fwd + bwd + D2H of every step inside the timed region.
    # Pipelined as a training loop would be: the inputs of step i+1 go up and the results
    # of step i-1 come down (on their own streams) while step i computes; device buffers
    # are double-buffered and ordered with events.
    e2e = None
    if not args.no_e2e:
        pin = lambda x: x.cpu().pin_memory()
        names = ("q", "k", "v", "g", "beta", "h0", "do", "dhT")
        hin = [pin(getattr(inp, nm)) for nm in names]
        h2d = sum(x.numel() * x.element_size() for x in hin)
        dev_in = [[torch.empty_like(getattr(d, nm)) for nm in names] for _ in range(2)]
        dev_out = [((torch.empty_like(o), torch.empty_like(hT)) +
                    tuple(torch.empty_like(x) for x in grads)) for _ in range(2)]
        houts = [[torch.empty(x.shape, dtype=x.dtype, pin_memory=True) for x in dev_out[0]]
                 for _ in range(2)]
        d2h = sum(x.numel() * x.element_size() for x in houts[0])
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev = lambda: torch.cuda.Event()
        e_in = [ev(), ev()]
        e_comp = [ev(), ev()]
        e_out = [ev(), ev()]
        first = [True, True]

        def upload(i):
            b = i % 2
            with torch.cuda.stream(s_in):
                if not first[b]:
                    s_in.wait_event(e_comp[b])  # step i-2 finished reading this input set
                for hsrc, ddst in zip(hin, dev_in[b]):
                    ddst.copy_(hsrc, non_blocking=True)
                e_in[b].record(s_in)

        def compute(i):
            b = i % 2
            stream.wait_event(e_in[b])
            if not first[b]:
                stream.wait_event(e_out[b])  # step i-2's results are down
            x = dev_in[b]
            out = dev_out[b]
            gdn.gdn_fwd(x[0], x[1], x[2], x[3], x[4], h0=x[5], o=out[0], hT=out[1], workspace=ws)
            gdn.gdn_bwd(x[0], x[1], x[2], x[3], x[4], x[6], h0=x[5], dhT=x[7], grads=out[2:],
                        workspace=ws)
            e_comp[b].record(stream)

        def download(i):
            b = i % 2
            with torch.cuda.stream(s_out):
                s_out.wait_event(e_comp[b])
                for dsrc, hdst in zip(dev_out[b], houts[b]):
                    hdst.copy_(dsrc, non_blocking=True)
                e_out[b].record(s_out)
            first[b] = False

        def run(n):
            for i in range(n + 1):
                if i < n:
                    upload(i)
                if i >= 1:
                    download(i - 1)
                if i < n:
                    compute(i)
            torch.cuda.current_stream().wait_stream(s_out)

        run(2)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        s_in.wait_event(e0)
        s_out.wait_event(e0)
        run(args.steps)
        e1.record(stream)
        torch.cuda.synchronize()
        te = max_over_ranks(e0.elapsed_time(e1), world, dev)
        e2e = {"value": job_tokens_per_s(B * T, world, args.steps, te), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "overlap": "H2D of step i+1 and D2H of step i-1 on their own streams while "
                          "step i computes"}

    if rank != 0:
        return
    pk = peaks()
    value = job_tokens_per_s(B * T, world, args.steps, tot_ms)
    # dominant kernel roofline
    dom = max(per_kernel.items(), key=lambda kv: kv[1][1]) if per_kernel else None
    roof = None
    if dom:
        # a kernel may launch several times per step (the forward runs in parts of every
        # row): the work of all its launches in a step over their summed event time
        name, (n, ms) = dom
        per_launch_s = ms / n / 1e3
        per_step = n / args.steps
        bound, amount, unit = kernel_work(name, w, n_chunks)
        if amount is not None:  # algorithmic work of one launch: the passes a step makes
            # over the whole workload (the fp32 path's prep and forward chain run in both
            # gdn_fwd and gdn_bwd) spread over the step's launches
            amount *= {"simt_prep": 2, "simt_state_fwd": 2}.get(name, 1) / per_step
        if bound == "alu":
            peak = alu_peak_tflops(pk["sm_mhz"])
            ach = amount / per_launch_s / 1e12
            roof = {"kernel": name, "bound": "alu", "achieved": ach, "peak": peak,
                    "unit": "TFLOP/s", "frac": ach / peak, "traffic": None,
                    "peak_source": "derived: 148 SM x 128 fp32 lanes x 2 x %.0f MHz" % pk["sm_mhz"],
                    "ms_per_launch": per_launch_s * 1e3}
        elif bound in ("hbm", "tensor"):
            peak = pk["hbm"] if bound == "hbm" else pk["tc"]
            ach = amount / per_launch_s / (1e9 if bound == "hbm" else 1e12)
            wl = ("gdn_fwdbwd_bf16_B4_T4096_H16_d128" if not args.shape else
                  "gdn_fwdbwd_bf16_B%d_T%d_H%d_d128" % (B, T, H))
            tr = recorded_traffic(name, wl)
            roof = {"kernel": name, "bound": bound, "achieved": ach, "peak": peak,
                    "unit": "GB/s" if bound == "hbm" else "TFLOP/s", "frac": ach / peak,
                    "traffic": None if tr is None else tr / per_step,
                    "algorithmic": amount, "peak_source": pk["src"],
                    "ms_per_launch": per_launch_s * 1e3, "launches_per_step": per_step}
    sr = step_roofline(w, pk)
    cpu = None
    if not args.no_cpu_baseline and world == 1:
        # every (row, head) unit of the workload, in passes until >= 10 s of CPU work
        dt, nu, threads, tk = cpu_oracle_sample(WORKLOAD["B"] * WORKLOAD["H"], min_s=10.0,
                                                max_passes=16)
        cpu = {"value": tk / dt, "unit": "tokens/s", "cores": threads, "kind": "oracle",
               "sample": "%d (row, head) units x %d tokens (the whole workload in passes), "
                         "fp64 fwd+bwd, %.1f s; tokens/s = units*T/H / s" % (nu, WORKLOAD["T"], dt)}
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": ("gdn_fwdbwd_bf16_B4_T4096_H16_d128" if not args.shape else
                                "gdn_fwdbwd_bf16_B%d_T%d_H%d_d128" % (B, T, H)),
                   "global_batch": B * world,
                   "seq_len": T, "heads": H, "head_dim": K, "parallelism": "dp%d" % world,
                   "l2": "256 MiB memset before each step, outside the step events"},
        "roofline": roof,
        "step_roofline": {"bound": sr["bound"], "t_bound_us": sr["t_bound_s"] * 1e6,
                          "frac": sr["t_bound_s"] / (tot_ms / args.steps / 1e3),
                          "flops": sr["flops"], "bytes": sr["bytes"],
                          "peaks": "%s (hbm %.0f GB/s, bf16 burst %.0f TFLOP/s)"
                                   % (pk["src"], pk["hbm"], pk["tc"])},
        "kernels_ms_per_step": {k: v[1] / args.steps for k, v in per_kernel.items()},
        "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches,
        "clocks": clk.summary(),
    }
    print(json.dumps(line), flush=True)


def run_decode(args, rank, world, local_rank):
    """Recurrent decode step: B sequences x H heads advance one token each; HBM
    bound by the fp32 state (read and written once per step)."""
    import torch

    import gated_delta_rule_99_b200 as gdn
    from gated_delta_rule_99_b200.inputs import make_inputs
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    B, H, K, V = 256, 16, 128, 128
    if args.shape:
        B, _, H = (int(x) for x in args.shape.split(","))
    inp = make_inputs(B=B, T=1, H=H, K=K, V=V, dtype="bf16", seed=50 + rank, bwd=False)
    d = inp.to(dev)
    state = d.h0.clone()
    o = torch.empty_like(d.v)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    for _ in range(max(3, args.warmup)):
        gdn.gdn_decode(d.q, d.k, d.v, d.g, d.beta, state, o=o)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    torch.cuda.synchronize()
    with ClockSampler(None) as clk:
        for i in range(args.steps):
            flush.zero_()
            evs[i][0].record(stream)
            gdn.gdn_decode(d.q, d.k, d.v, d.g, d.beta, state, o=o)
            evs[i][1].record(stream)
        torch.cuda.synchronize()
    tot_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in evs), world, dev)
    if rank != 0:
        return
    pk = peaks()
    per = tot_ms / args.steps / 1e3
    bytes_ = B * H * (2 * K * V * 4 + 2 * (2 * K + 2 * V) + 8)
    ach = bytes_ / per / 1e9
    print(json.dumps({
        "metric": "GDN recurrent decode tokens/s (B=%d sequences, H=%d, d=128, bf16, fp32 state)"
                  % (B, H),
        "value": world * B / per, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": per * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "gdn_decode_bf16_B%d_H%d_d128" % (B, H),
                   "l2": "256 MiB memset before each step, outside the step events"},
        "roofline": {"kernel": "decode", "bound": "hbm", "achieved": ach, "peak": pk["hbm"],
                     "unit": "GB/s", "frac": ach / pk["hbm"], "traffic": None,
                     "algorithmic": bytes_, "peak_source": pk["src"]},
        "gpu_launches": args.steps, "clocks": clk.summary()}), flush=True)


def run_report(args, rank, world, local_rank):
    """Throughput of every workload on one GPU: forward tokens/s for the forward
    workloads, forward+backward for the others, each with its whole-call
    roofline (method flops and bytes against the measured peaks).  One JSON
    line per workload."""
    import torch

    import gated_delta_rule_99_b200 as gdn
    from gated_delta_rule_99_b200.inputs import WORKLOADS, make_inputs, workload
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    pk = peaks()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    # every workload; the long row also with the piece scan; the benchmark workload also with
    # the layer's own q/k normalisation (raw q, k); head dim 64 dense and packed (tensor cores)
    d64 = dict(WORKLOADS[2], K=64, V=64, name="gdn_fwdbwd_bf16_B4_T4096_H16_d64")
    p64 = dict(WORKLOADS[3], K=64, V=64, name=WORKLOADS[3]["name"].replace("d128", "d64"))
    # a long single row forward + backward (a quarter of the long-context row, which is
    # a forward workload), with and without the piece scan of both chains
    lrow = dict(WORKLOADS[4], T=1 << 18, bwd=True, name="gdn_fwdbwd_bf16_B1_T262144_H8_d128")
    # head dim 256 (fp32 CUDA-core kernels): the benchmark's token count per head, 8 heads
    d256 = dict(WORKLOADS[2], B=1, H=8, K=256, V=256, name="gdn_fwdbwd_bf16_B1_T4096_H8_d256")
    runs = ([(i, dict(WORKLOADS[i]), False, False) for i in sorted(WORKLOADS)] +
            [(4, dict(WORKLOADS[4]), True, False), (2, dict(WORKLOADS[2]), False, True),
             (None, d64, False, False), (None, p64, False, False),
             (None, lrow, False, False), (None, lrow, True, False),
             (None, d256, False, False)])
    for idx, w, piece, l2 in runs:
        if idx is not None and not l2:
            inp = workload(idx, device="cuda" if idx == 4 else "cpu")
        else:
            inp = make_inputs(**dict(w, raw_qk=l2, device="cuda" if w["T"] > 100000 else "cpu"))
        d = inp.to(dev)
        cu = inp.cu_seqlens
        cu_dev = None if cu is None else cu.to(dev)
        bwd = w["bwd"]
        B, T, H, K, V = w["B"], w["T"], w["H"], w["K"], w["V"]
        n = inp.n_seqs
        flags = (gdn.GDN_FLAG_PIECE_SCAN if piece else 0) | (gdn.GDN_FLAG_QK_L2NORM if l2 else 0)
        desc = gdn.make_desc(B, T, H, K, V, 0 if cu is None else n,
                             gdn.GDN_BF16 if w["dtype"] == "bf16" else gdn.GDN_FP32, flags=flags)
        ws = gdn.alloc_workspace(max(gdn.fwd_workspace_size(desc),
                                     gdn.bwd_workspace_size(desc) if bwd else 0), dev)
        o = torch.empty_like(d.v)
        hT = torch.empty(n, H, K, V, dtype=torch.float32, device=dev)
        grads = None
        if bwd:
            grads = (torch.empty_like(d.q), torch.empty_like(d.k), torch.empty_like(d.v),
                     torch.empty_like(d.g), torch.empty_like(d.beta),
                     torch.empty(n, H, K, V, dtype=torch.float32, device=dev))

        def step():
            gdn.gdn_fwd(d.q, d.k, d.v, d.g, d.beta, cu_seqlens=cu_dev, cu_seqlens_host=cu,
                        h0=d.h0, o=o, hT=hT, workspace=ws, piece_scan=piece, qk_l2norm=l2)
            if bwd:
                gdn.gdn_bwd(d.q, d.k, d.v, d.g, d.beta, d.do, cu_seqlens=cu_dev,
                            cu_seqlens_host=cu, h0=d.h0, dhT=d.dhT, grads=grads, workspace=ws,
                            qk_l2norm=l2, piece_scan=piece)

        for _ in range(3):
            step()
        torch.cuda.synchronize()
        if gdn.device_status(ws) != 0:
            raise RuntimeError("device status not ok after warm-up (%s)" % w["name"])
        steps = 3 if T > 100000 else max(5, args.steps)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(steps)]
        torch.cuda.synchronize()
        for i in range(steps):
            flush.zero_()
            evs[i][0].record(stream)
            step()
            evs[i][1].record(stream)
        torch.cuda.synchronize()
        if gdn.device_status(ws) != 0:  # a wait that gave up would make the time meaningless
            raise RuntimeError("device status not ok after the timed calls (%s)" % w["name"])
        ms = sum(a.elapsed_time(b) for a, b in evs) / steps
        th = B * T * H
        fwd_f = 2 * C * (3 * K + 2 * V) + 6 * K * V + C * C / 3
        bwd_f = 9 * 2 * C * K + 5 * 2 * C * V + 8 * 2 * K * V + 4 * C * C
        flops = (fwd_f + (bwd_f if bwd else 0)) * th
        el = 2 if w["dtype"] == "bf16" else 4
        fwd_b = (3 * el * K if K == V else el * (2 * K + V)) + 8 + el * V
        bwd_b = el * (2 * K + 2 * V) + 8 + el * (2 * K + V) + 8
        bytes_ = (fwd_b + (bwd_b if bwd else 0)) * th
        # the fp32 path (fp32 inputs, or a head dim of 256) runs on the CUDA cores: its
        # flops are bound by the fp32 FMA peak, the tensor-core path's by the bf16 MMA peak
        cuda_core = w["dtype"] != "bf16" or K > 128 or V > 128
        fpeak = alu_peak_tflops(pk["sm_mhz"]) if cuda_core else pk["tc"]
        t_bound = max(flops / (fpeak * 1e12), bytes_ / (pk["hbm"] * 1e9))
        if rank == 0:
            print(json.dumps({
                "workload": w["name"] + ("+piece_scan" if piece else "") + ("+qk_l2norm" if l2 else ""),
                "pass": "fwd+bwd" if bwd else "fwd",
                "tokens_per_s": B * T / (ms / 1e3), "ms_per_call": ms,
                "roofline_frac": t_bound * 1e3 / ms, "roofline_us": t_bound * 1e6,
                "path": "cuda-core fp32" if cuda_core else "tensor-core",
                "peaks": pk["src"]}), flush=True)
        del d, ws, o, hT, grads
        torch.cuda.empty_cache()


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        if args.mode == "decode":
            run_decode(args, rank, world, local_rank)
            return
        if args.mode == "report":
            run_report(args, rank, world, local_rank)
            return
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
