"""Benchmark of the sliced r-bit linear layer (MatQuant / MatGPTQ true-prefix slicing) on B200.

Workload (default, ``--workload ffn8b_decode``): the Llama-3.1-8B-shaped FFN at decode
batch sizes.  One step runs, for every width r in {2, 3, 4, 6, 8} and every batch
M in {1, 4, 16}, one FFN forward through the sliced linears:
    a    = silu(x . W_gate,r^T) * (x . W_up,r^T)   [M, 14336]   (ONE matq_linear call over the
           row-interleaved [gate; up] pack, MATQ_OUT_SILU_GATED: the gated product is formed
           in the epilogue from the fp32 results)
    y    = a . W_down,r^T           [M, 4096]
with group-128 parent codes of N(0, 0.02) weights (synthetic, seeded) and N(0, 1) bf16
activations.  ``value`` = algorithmic bytes of the sliced linears (planes of width r,
fp16 scales, uint8 zeros, x, y) over the device time of the step -> GB/s.

``--workload ffn8b_prefill``: the same FFN at M = 2048 with 1% outlier channels x20,
r in {3, 4, 8}; ``value`` = 2*M*N*K flops of the sliced linears over the step time -> TFLOP/s.

L2 (126 MB) is defeated by rotating through several device copies of the packed layer
(working set > 1 GB), so every call streams its planes from HBM.

Multi-GPU (torchrun, one rank per GPU): replicas / weak scaling -- every rank serves its own
batches with its own copy of the weights; there is no exchange step on this path.  The
step time is the max over ranks (device events, all-reduced).

``--impl reference``: the fp64 CPU oracle (the only reference this method has here), timed
on a bounded sample of the same workload on the host cores.
"""

from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np

WIDTHS = (2, 3, 4, 6, 8)
D_MODEL, D_FF, GROUP = 4096, 14336, 128
METRIC = "sliced r-bit linear: decode weight GB/s vs HBM peak; prefill TFLOP/s per r"
# arithmetic each path computes in (not a precision claim): decode multiplies the exact fp16
# weight levels with fp16 activations, prefill fp16 dequantised weight and activation tiles; both
# accumulate in fp32
DTYPES = {"GB/s": "f16-operands/f32-acc (bf16 in/out)", "TFLOP/s": "f16-operands/f32-acc (bf16 in/out)"}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="ffn8b_decode",
                    choices=["ffn8b_decode", "ffn8b_prefill", "stack32", "ffn9b_sweep", "linear1024"])
    ap.add_argument("--copies", type=int, default=6, help="device copies of the packed layer (L2 rotation)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", action="store_true",
                    help="decode workload only: leave out the prefill sub-record of the default line")
    ap.add_argument("--no-ep", action="store_true",
                    help="decode workload only: leave out the Extra-Precision sub-record of the default line")
    ap.add_argument("--case", choices=["decode", "prefill", "pack", "choose", "speedup", "ep"], default=None,
                    help="profiling aid: run a few single sliced-linear calls on the 8B gate matrix and exit")
    ap.add_argument("--r", type=int, default=2)
    ap.add_argument("--m", type=int, default=1)
    ap.add_argument("--calls", type=int, default=8)
    return ap.parse_args()


def workload_spec(name):
    if name == "ffn8b_decode":
        return dict(widths=WIDTHS, batches=(1, 4, 16), outlier=0.0, unit="GB/s")
    return dict(widths=(3, 4, 8), batches=(2048,), outlier=0.01, unit="TFLOP/s")


def workload_config(args, spec, world):
    """The workload both arms report (the reference arm adds where it runs)."""
    gu = ("gated product in the epilogue" if gated_epilogue(spec)
          else "both halves written, gated product by matq_silu_mul_gu")
    return {"workload": args.workload,
            "shapes": f"gate+up [28672,4096] (two [14336,4096] row-interleaved, {gu}), down [4096,14336], group 128",
            "widths": list(spec["widths"]), "batches": list(spec["batches"]),
            "parallelism": f"replicas x{world}"}


def linear_bytes(M, N, K, r, group=GROUP, out_cols=None):
    G = K // group
    return N * K * r // 8 + N * G * 3 + M * K * 2 + M * (N if out_cols is None else out_cols) * 2


# the sliced-linear calls of one FFN: gate+up over the row-interleaved pack, then down
FFN_CALLS = (("gate_up", (2 * D_FF, D_MODEL)), ("down", (D_MODEL, D_FF)))


def gated_epilogue(spec):
    """The gated product is fused into the gate+up call (both workloads)."""
    return True


def out_cols(spec, name):
    if name == "gate_up":
        return D_FF if gated_epilogue(spec) else 2 * D_FF
    return D_MODEL


def step_units(spec):
    """(algorithmic bytes, flops) of one step."""
    b = f = 0
    for r in spec["widths"]:
        for M in spec["batches"]:
            for name, (N, K) in FFN_CALLS:
                b += linear_bytes(M, N, K, r, out_cols=out_cols(spec, name))
                f += 2 * M * N * K
    return b, f


# ---------------------------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------------------------

def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def maybe_init_pg(world, backend):
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(world, value, device):
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_value(unit, step_bytes, step_flops, world, ms_step):
    """Whole-job throughput: every rank runs the same step on its own batches (weak scaling),
    so the job moves world x the per-rank units in the slowest rank's step time."""
    if unit == "GB/s":
        return step_bytes * world / (ms_step * 1e-3) / 1e9
    return step_flops * world / (ms_step * 1e-3) / 1e12


# ---------------------------------------------------------------------------------------------
# clocks
# ---------------------------------------------------------------------------------------------

class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "20"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in getattr(self, "lines", []):
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------------------------
# CPU oracle baseline (bounded sample)
# ---------------------------------------------------------------------------------------------

def cpu_oracle_rate(spec, weights_host, budget_s=12.0, rows=256):
    """Time the fp64 oracle (as it stands) on a bounded sample of the workload: the first
    `rows` rows of the three FFN matrices at each (r, M), scaled to the metric's unit per
    second.  At least one pass over every (r, M) is made."""
    import oracle as O
    done_b = done_f = 0.0
    t0 = time.perf_counter()
    rng = np.random.default_rng(0)
    n_iter = 0
    while time.perf_counter() - t0 < budget_s or n_iter == 0:
        for r in spec["widths"]:
            for M in spec["batches"]:
                for name, (N, K) in (("gate", (D_FF, D_MODEL)), ("up", (D_FF, D_MODEL)), ("down", (D_MODEL, D_FF))):
                    q, s, z = weights_host[name]
                    Mi = min(M, 64)
                    x = rng.standard_normal((Mi, K))
                    O.linear(x, q[:rows], s[:rows], z[:rows], r, GROUP)
                    done_b += linear_bytes(Mi, rows, K, r)
                    done_f += 2 * Mi * rows * K
        n_iter += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    cores = os.cpu_count()
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        cores = max((i.get("num_threads", 1) for i in info), default=cores)
    except Exception:
        pass
    val = done_b / dt / 1e9 if spec["unit"] == "GB/s" else done_f / dt / 1e12
    sample = (f"first {rows} rows of gate/up/down at every (r, M) of the workload "
              f"(M capped at 64), {n_iter} pass(es), {dt:.1f} s")
    return {"value": val, "unit": spec["unit"], "cores": cores, "kind": "oracle", "sample": sample, "seconds": dt}


def host_weights():
    from nested_bit_weight_msb_b200 import synth
    return {name: synth.parent_weights(N, K, GROUP, seed=0, layer=0, proj=name)
            for name, (N, K) in (("gate", (D_FF, D_MODEL)), ("up", (D_FF, D_MODEL)), ("down", (D_MODEL, D_FF)))}


def interleave_rows(a, b):
    out = np.empty((2 * a.shape[0],) + a.shape[1:], dtype=a.dtype)
    out[0::2] = a
    out[1::2] = b
    return out


def fused_weights(w):
    """gate and up read the same x: their codes, scales and zero points are interleaved by
    row (2i: gate row i, 2i + 1: up row i) into one [2F, D] matrix served by one call whose
    epilogue forms silu(gate) * up."""
    gu = tuple(interleave_rows(w["gate"][i], w["up"][i]) for i in range(3))
    return {"gate_up": gu, "down": w["down"]}


# ---------------------------------------------------------------------------------------------
# reference arm: the oracle on the host
# ---------------------------------------------------------------------------------------------

def reference_sampler(args, world):
    """(sample(budget_s, rows) -> rate record, unit, config) of the oracle for a workload; the
    config is the one our arm reports for the same workload."""
    if args.workload == "stack32":
        from nested_bit_weight_msb_b200 import synth
        w = host_weights()
        widths = [int(v) for v in synth.mixnmatch_widths(0, layers=STACK_LAYERS)]
        return (lambda b, rows: cpu_stack_rate(w, budget_s=b, rows=min(rows, 128)), "GB/s",
                stack_config(widths, world))
    if args.workload in SWEEPS:
        sw = SWEEPS[args.workload]
        mats = sweep_mats(sw)
        dec = [M for M in sw["batches"] if M <= 16]
        return (lambda b, rows: cpu_sweep_rate(mats, sw["group"], dec, sw["widths"], budget_s=b, rows=min(rows, 128)),
                "GB/s", sweep_config(args, sw, {k: list(v[0].shape) for k, v in mats.items()}, world))
    spec = workload_spec(args.workload)
    w = host_weights()
    return (lambda b, rows: cpu_oracle_rate(spec, w, budget_s=b, rows=rows), spec["unit"],
            workload_config(args, spec, world))


def run_reference(args):
    world, rank, local = dist_setup()
    if rank != 0:
        return 0
    sample, unit, config = reference_sampler(args, world)
    # each step is a bounded sample, sized so that warm-up + steps stay within ~3 minutes
    budget = min(5.0, 150.0 / max(1, args.steps + args.warmup))
    rows = 256 if budget >= 2.0 else 32
    for _ in range(args.warmup):
        sample(budget, rows)
    vals = []
    for _ in range(args.steps):
        vals.append(sample(budget, rows))
    v = float(np.mean([c["value"] for c in vals]))
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": unit, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup,
        # measured: the wall time of one step, i.e. of one bounded sample of the workload (value is
        # that sample's rate); a whole workload step on the oracle would take far longer
        "ms_per_step": float(np.mean([c["seconds"] for c in vals])) * 1e3,
        "step_is_bounded_sample": True,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": dict(config, device="host cores (fp64 oracle)"),
        "cpu_baseline": {"kind": "oracle", "cores": vals[0]["cores"], "sample": vals[0]["sample"], "value": v,
                         "unit": unit},
        "e2e": {"value": v, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------------------------

class FfnBench:
    """Device state of one workload's FFN step: the packed weights (rotating device copies), the
    workload's activations, output buffers, a workspace, and the call helpers."""

    def __init__(self, args, spec, packed, meta, dev, rank):
        import torch
        from nested_bit_weight_msb_b200 import matq, synth
        self.args, self.spec, self.packed, self.meta, self.dev = args, spec, packed, meta, dev
        self.matq = matq
        self.batches = spec["batches"]
        self.xs = {}
        for M in self.batches:
            xb, _ = synth.activations(M, D_MODEL, seed=rank, outlier_frac=spec["outlier"])
            self.xs[M] = torch.from_numpy(xb.view(np.int16)).to(dev).view(torch.bfloat16)
        Mmax = max(self.batches)
        self.ws = torch.zeros(max(matq.workspace_bytes(Mmax, K, N, GROUP) for _, (N, K) in FFN_CALLS),
                              dtype=torch.uint8, device=dev)
        self.gated = gated_epilogue(spec)
        self.a_buf = {M: torch.empty((M, D_FF), dtype=torch.bfloat16, device=dev) for M in self.batches}
        self.gu_buf = {M: torch.empty((M, out_cols(spec, "gate_up")), dtype=torch.bfloat16, device=dev)
                       for M in self.batches}
        self.y_buf = {M: torch.empty((M, D_MODEL), dtype=torch.bfloat16, device=dev) for M in self.batches}
        self.calls = [(r, M) for r in spec["widths"] for M in self.batches]

    def linear(self, name, copy, x, r, out):
        s, z, N, K = self.meta[name]
        mode = self.matq.MATQ_OUT_SILU_GATED if (name == "gate_up" and self.gated) else self.matq.MATQ_OUT_BF16
        self.matq.linear(x, self.packed[name][copy], 8, s, z, N, r, GROUP, y=out, y_mode=mode, workspace=self.ws)

    def ffn(self, x, M, r, copy, y=None):
        if self.gated:
            self.linear("gate_up", copy, x, r, self.a_buf[M])
        else:
            self.linear("gate_up", copy, x, r, self.gu_buf[M])
            self.matq.silu_mul_gu(self.gu_buf[M], out=self.a_buf[M])
        self.linear("down", copy, self.a_buf[M], r, self.y_buf[M] if y is None else y)

    def step(self, base=0):
        for i, (r, M) in enumerate(self.calls):
            self.ffn(self.xs[M], M, r, (base + i) % self.args.copies)


def graph_us_per_call(fn, stream, n=24):
    """Device microseconds per call of fn(i) in steady state: a CUDA graph of n back-to-back calls
    (rotating weight copies, so every call streams from HBM), median of 5 replays."""
    import torch
    with torch.cuda.stream(stream):
        for i in range(3):
            fn(i)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(n):
                fn(i)
        g.replay()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        reps = []
        for _ in range(5):
            e0.record(stream)
            g.replay()
            e1.record(stream)
            torch.cuda.synchronize()
            reps.append(e0.elapsed_time(e1) / n)
    del g
    return float(np.median(reps)) * 1e3


def per_call_table(fb, stream):
    """Per width and batch: each sliced-linear call of the FFN (gate+up with the gated epilogue,
    down) timed on its own as back-to-back launches, with its roofline fraction (decode: GB/s of
    algorithmic bytes over the measured HBM peak; prefill: TFLOP/s over the burst bf16 peak)."""
    peaks = load_peaks()
    rows = []
    for r in fb.spec["widths"]:
        for M in fb.batches:
            row = {"r": r, "M": M}
            tot_us = 0.0
            for name, (N, K) in FFN_CALLS:
                x = fb.xs[M] if name == "gate_up" else fb.a_buf[M]
                out = fb.a_buf[M] if name == "gate_up" else fb.y_buf[M]
                us = graph_us_per_call(lambda i: fb.linear(name, i % fb.args.copies, x, r, out), stream)
                tot_us += us
                if fb.spec["unit"] == "GB/s":
                    b = linear_bytes(M, N, K, r, out_cols=out_cols(fb.spec, name))
                    v = b / (us * 1e-6) / 1e9
                    row[name] = {"us": round(us, 2), "GB/s": round(v, 1), "frac": round(v / peaks["hbm_gbs"], 3)}
                else:
                    v = 2 * M * N * K / (us * 1e-6) / 1e12
                    row[name] = {"us": round(us, 2), "TFLOP/s": round(v, 1), "frac": round(v / peaks["bf16_tflops"], 3)}
            if fb.spec["unit"] == "GB/s":
                b = sum(linear_bytes(M, N, K, r, out_cols=out_cols(fb.spec, name)) for name, (N, K) in FFN_CALLS)
                row["ffn"] = {"us": round(tot_us, 2), "GB/s": round(b / (tot_us * 1e-6) / 1e9, 1)}
            else:
                f = sum(2 * M * N * K for _, (N, K) in FFN_CALLS)
                row["ffn"] = {"us": round(tot_us, 2), "TFLOP/s": round(f / (tot_us * 1e-6) / 1e12, 1)}
            rows.append(row)
    return rows


def measure(args, spec, fb, stream, world, local, dev):
    """Time the workload's step (device events around K graph replays after W warm-up replays,
    max over ranks), then the dominant kernel's roofline, the per-call table and the end-to-end
    step through the public calls with host buffers."""
    import torch
    with torch.cuda.stream(stream):
        fb.step()
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            fb.step()
        for _ in range(args.warmup):
            graph.replay()
        torch.cuda.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        with ClockSampler(local) as clk:
            e0.record(stream)
            for _ in range(args.steps):
                graph.replay()
            e1.record(stream)
            torch.cuda.synchronize()
        barrier(world)
        torch.cuda.synchronize()
    # a timed run whose device-side waits ran out prints no number
    st = fb.matq.workspace_status(fb.ws)
    if st != 0:
        raise RuntimeError(f"device status {st} after the timed region: the timed calls did not complete normally")
    ms_total = max_over_ranks(world, e0.elapsed_time(e1), dev)
    ms_step = ms_total / args.steps
    b, f = step_units(spec)
    value = whole_job_value(spec["unit"], b, f, world, ms_step)
    rl = roofline(args, spec, fb.linear, fb.xs, fb.a_buf if fb.gated else fb.gu_buf, stream, dev)
    table = per_call_table(fb, stream)
    e2e = end_to_end(args, spec, fb.ffn, fb.calls, fb.xs, fb.y_buf, stream, dev, world)
    del graph
    return {"value": value, "ms_per_step": ms_step, "roofline": rl, "per_r": table, "e2e": e2e,
            "clocks": clk.summary(),
            # per FFN: gated gate+up and down, one kernel each on the decode path, activation
            # conversion + GEMM each on the prefill path
            "gpu_launches": args.steps * len(fb.calls) * len(FFN_CALLS) * (1 if spec["unit"] == "GB/s" else 2)}


EP_WIDTHS = (2, 3, 4)


def ep_table(packed, meta, dev, stream, peaks):
    """Extra-Precision MatQuant ("Matryoshka Quantization | Summary" §7 Errata) per call at M = 1
    on the 8B FFN matrices: each matrix's rounded slice extracted once from its parent pack (the
    clamped levels, r bits a weight, plus the list of weights whose rounded level is 2^r), then
    served by matq_linear_rounded (gate+up with the gated output, down with bf16 output).
    Algorithmic bytes: the level planes, scales and zeros, 2 bytes per listed weight and the
    row pointers, x and y.  Each call timed as back-to-back launches over rotating copies."""
    import torch
    from nested_bit_weight_msb_b200 import matq, synth
    out = []
    for r in EP_WIDTHS:
        row = {"r": r, "M": 1}
        for name in ("gate_up", "down"):
            s, z, N, K = meta[name]
            levels, row_ptr, cols = matq.round_extract(packed[name][0], N, K, 8, r)
            nnz = int(row_ptr[-1].item())
            n_copies = int(min(8, max(2, (256 << 20) // levels.numel() + 1)))
            lv = [levels] + [levels.clone() for _ in range(n_copies - 1)]
            lists = [(row_ptr, cols)] + [(row_ptr.clone(), cols.clone()) for _ in range(n_copies - 1)]
            xb, _ = synth.activations(1, K, seed=0)
            x = torch.from_numpy(xb.view(np.int16)).to(dev).view(torch.bfloat16)
            gated = name == "gate_up"
            ycols = N // 2 if gated else N
            y = torch.empty((1, ycols), dtype=torch.bfloat16, device=dev)
            mode = matq.MATQ_OUT_SILU_GATED if gated else matq.MATQ_OUT_BF16
            ws = matq.rounded_workspace(1, K, N, GROUP, device=dev)
            us = graph_us_per_call(lambda i: matq.linear_rounded(x, lv[i % n_copies], r, s, z, N, GROUP,
                                                                 lists[i % n_copies][0], lists[i % n_copies][1],
                                                                 y=y, y_mode=mode, workspace=ws), stream)
            if matq.workspace_status(ws) != 0:
                raise RuntimeError("device status after the Extra-Precision calls: a call did not complete normally")
            b = linear_bytes(1, N, K, r, out_cols=ycols) + 2 * nnz + 4 * (N + 1)
            gbs = b / (us * 1e-6) / 1e9
            row[name] = {"us": round(us, 2), "GB/s": round(gbs, 1), "frac": round(gbs / peaks["hbm_gbs"], 3),
                         "listed_fraction": round(nnz / (N * K), 5), "bytes": b}
            del lv, lists, ws
        out.append(row)
    torch.cuda.empty_cache()
    return out


def run_ours(args):
    import torch
    world, rank, local = dist_setup()
    maybe_init_pg(world, "nccl")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    from nested_bit_weight_msb_b200 import matq

    spec = workload_spec(args.workload)
    weights = host_weights()
    # pack once per matrix (one-time), then clone into rotating copies
    packed = {}
    meta = {}
    for name, (q, s, z) in fused_weights(weights).items():
        dq = torch.from_numpy(q).to(dev)
        p = matq.pack(dq, r_keep=8)
        packed[name] = [p] + [p.clone() for _ in range(args.copies - 1)]
        meta[name] = (torch.from_numpy(s.view(np.int16)).to(dev), torch.from_numpy(z).to(dev), q.shape[0], q.shape[1])
        del dq
    torch.cuda.synchronize()
    stream = torch.cuda.Stream(device=dev)
    res = measure(args, spec, FfnBench(args, spec, packed, meta, dev, rank), stream, world, local, dev)
    # the default decode line also carries the prefill half of the metric (TFLOP/s per r)
    pre = None
    if args.workload == "ffn8b_decode" and not args.no_prefill:
        pspec = workload_spec("ffn8b_prefill")
        pfb = FfnBench(args, pspec, packed, meta, dev, rank)
        pre = measure(args, pspec, pfb, stream, world, local, dev)
        del pfb
        torch.cuda.empty_cache()

    ep = None
    if args.workload == "ffn8b_decode" and not args.no_ep:
        ep = ep_table(packed, meta, dev, stream, load_peaks())

    if rank == 0:
        peaks = load_peaks()
        line = {
            "metric": METRIC, "value": res["value"], "unit": spec["unit"], "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": res["ms_per_step"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": DTYPES[spec["unit"]], "data": "synthetic",
            "config": dict(workload_config(args, spec, world),
                           l2=f"rotating {args.copies} device copies of the packed layer (> L2)",
                           timing="CUDA graph replay, CUDA events"),
            "roofline": res["roofline"],
            "e2e": res["e2e"],
            "gpu_launches": res["gpu_launches"] + (pre["gpu_launches"] if pre else 0),
            "clocks": res["clocks"],
            "peaks_source": peaks.get("_source"),
            "per_r": res["per_r"],
        }
        if pre is not None:
            pspec = workload_spec("ffn8b_prefill")
            line["prefill"] = {
                "workload": "ffn8b_prefill", "value": pre["value"], "unit": pspec["unit"],
                "ms_per_step": pre["ms_per_step"], "dtype": DTYPES[pspec["unit"]],
                "config": dict(workload_config(argparse.Namespace(workload="ffn8b_prefill"), pspec, world),
                               l2=f"rotating {args.copies} device copies of the packed layer (> L2)",
                               timing="CUDA graph replay, CUDA events"),
                "roofline": pre["roofline"], "e2e": pre["e2e"], "clocks": pre["clocks"], "per_r": pre["per_r"],
                "gpu_launches": pre["gpu_launches"],
            }
        if ep is not None:
            line["extra_precision"] = {"widths": list(EP_WIDTHS), "per_r": ep,
                                       "note": "rounded slices served from the clamped-level pack plus the list of "
                                               "weights at level 2^r; the true-prefix calls are in per_r"}
        if not args.no_cpu_baseline and world == 1:
            line["cpu_baseline"] = cpu_oracle_rate(spec, weights)
            if pre is not None:
                line["prefill"]["cpu_baseline"] = cpu_oracle_rate(workload_spec("ffn8b_prefill"), weights)
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        d["_source"] = "measured"
        return d
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "_source": "fallback"}


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one launch of the roofline
# kernel, from an ncu capture, with the SHA-256 of the kernel's sources at capture time; the
# figure is reported only while the sources are unchanged.  Captures: profiles/.
_KERNEL_SOURCES = {
    "decode": ("decode.cu", "common.cuh", "operands.cuh", "sync.cuh"),
    "prefill": ("prefill.cu", "common.cuh", "operands.cuh", "sync.cuh"),
}
NCU_TRAFFIC = {  # kernel kind -> capture (sources hash, launch it was taken on, bytes)
    "decode": {"sha256": "e36c5d58b8a2ddfb8fd710e0b1ce6860a5b0438193844aad612da8f2c94a8978", "launch": "gate_up gated 28672x4096 r=2 M=1",
               "bytes": 32_188_672 + 0},
    "prefill": {"sha256": "58199cae351b8d6212fb20b4465a2ca14b7fd9a967156d6ed4862827fef8cb53", "launch": "gate_up gated 28672x4096 r=4 M=2048",
                "bytes": 78_321_664 + 30_037_760},
}


def kernel_source_sha(path_kind):
    import hashlib
    h = hashlib.sha256()
    for f in _KERNEL_SOURCES[path_kind]:
        with open(os.path.join(ROOT, "nested_bit_weight_msb_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def measured_traffic(path_kind, launch):
    rec = NCU_TRAFFIC[path_kind]
    if rec["bytes"] is None or rec.get("launch") != launch or rec["sha256"] != kernel_source_sha(path_kind):
        return None
    return rec["bytes"]


def roofline(args, spec, linear, xs, gu_buf, stream, dev):
    """Average device time per launch of the dominant kernel in steady state: a CUDA graph of
    back-to-back sliced-linear calls on the gate matrix (rotating weight copies, so every call
    streams from HBM), timed with CUDA events on the launching stream; total / launches."""
    import torch
    peaks = load_peaks()
    M = max(spec["batches"]) if spec["unit"] == "TFLOP/s" else 1
    r = 2 if spec["unit"] == "GB/s" else 4
    n = 24
    with torch.cuda.stream(stream):
        for i in range(3):
            linear("gate_up", i % args.copies, xs[M], r, gu_buf[M])
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(n):
                linear("gate_up", i % args.copies, xs[M], r, gu_buf[M])
        g.replay()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        reps = []
        for _ in range(5):
            e0.record(stream)
            g.replay()
            e1.record(stream)
            torch.cuda.synchronize()
            reps.append(e0.elapsed_time(e1) / n)
    del g
    avg_ms = float(np.median(reps))
    N = 2 * D_FF
    launch = f"gate_up {'gated ' if gated_epilogue(spec) else ''}{N}x{D_MODEL} r={r} M={M}"
    if spec["unit"] == "GB/s":
        units = linear_bytes(M, N, D_MODEL, r, out_cols=out_cols(spec, "gate_up"))
        ach = units / (avg_ms * 1e-3) / 1e9
        peak = peaks["hbm_gbs"]
        return {"bound": "hbm", "achieved": ach, "peak": peak, "unit": "GB/s", "frac": ach / peak,
                "traffic": measured_traffic("decode", launch), "algorithmic_bytes": units,
                "kernel": f"decode_kernel via matq_linear ({launch})",
                "avg_us": avg_ms * 1e3, "launches_timed": n, "peak_source": peaks.get("_source")}
    flops = 2 * M * N * D_MODEL
    ach = flops / (avg_ms * 1e-3) / 1e12
    peak = peaks["bf16_tflops"]
    return {"bound": "tensor", "achieved": ach, "peak": peak, "unit": "TFLOP/s", "frac": ach / peak,
            "traffic": measured_traffic("prefill", launch), "algorithmic_flops": flops,
            "kernel": f"prefill_kernel (+ activation pre-pass) via matq_linear ({launch})",
            "avg_us": avg_ms * 1e3, "launches_timed": n, "peak_source": peaks.get("_source")}


COPY_GROUP_BYTES = 4 << 20  # smallest host<->device copy the end-to-end step pipelines on its own


def copy_groups(sizes, min_bytes=COPY_GROUP_BYTES):
    """Split the calls of a step (their input bytes, in order) into runs of consecutive calls
    whose inputs move in one copy each way: a run closes once it holds min_bytes (the last run
    may hold less).  Small inputs (decode) make one run per step; large ones (prefill) one run
    per call, so a call's copies overlap the other calls' kernels."""
    groups, cur, acc = [], [], 0
    for i, b in enumerate(sizes):
        cur.append(i)
        acc += b
        if acc >= min_bytes:
            groups.append(cur)
            cur, acc = [], 0
    if cur:
        groups.append(cur)
    return groups


def end_to_end(args, spec, ffn, calls, xs, y_buf, stream, dev, world):
    """The same step through the public calls, with the step's activations copied in from
    pinned host memory and its outputs copied back to pinned host memory inside the timed
    region.  Copies run on their own streams (host->device and device->host use separate copy
    engines), one per run of calls (`copy_groups`): a run's kernels wait for its inputs, its
    outputs leave as soon as its kernels finish.  Two sets of device buffers alternate between
    steps, so one step's copies overlap the neighbouring steps' kernels; a buffer is refilled
    only after the step that last used it has read its inputs and copied its outputs out.  The
    first step's copies start after the opening event and the last step's outputs are on the
    host before the closing one."""
    import torch
    offs, o = [], 0
    for (_, M) in calls:
        offs.append(o)
        o += M
    rows = o
    host_x = torch.empty((rows, D_MODEL), dtype=torch.bfloat16).pin_memory()
    for (_, M), off in zip(calls, offs):
        host_x[off:off + M].copy_(xs[M].cpu())
    host_y = torch.empty((rows, D_MODEL), dtype=torch.bfloat16).pin_memory()
    nbuf = 2
    dev_x = [torch.empty((rows, D_MODEL), dtype=torch.bfloat16, device=dev) for _ in range(nbuf)]
    dev_y = [torch.empty((rows, D_MODEL), dtype=torch.bfloat16, device=dev) for _ in range(nbuf)]
    h2d = host_x.numel() * 2
    d2h = host_y.numel() * 2
    groups = copy_groups([M * D_MODEL * 2 for (_, M) in calls])
    span = [(offs[g[0]], offs[g[-1]] + calls[g[-1]][1]) for g in groups]
    h2d_s = torch.cuda.Stream(device=dev)
    d2h_s = torch.cuda.Stream(device=dev)

    def events():
        return [[torch.cuda.Event() for _ in groups] for _ in range(nbuf)]

    landed, used, out = events(), events(), events()  # inputs in; run done; outputs copied out
    fresh = [[True] * len(groups) for _ in range(nbuf)]

    def step(k, start):
        b = k % nbuf
        h2d_s.wait_event(start)
        with torch.cuda.stream(h2d_s):
            for gi, (lo, hi) in enumerate(span):
                if not fresh[b][gi]:
                    h2d_s.wait_event(used[b][gi])
                dev_x[b][lo:hi].copy_(host_x[lo:hi], non_blocking=True)
                landed[b][gi].record(h2d_s)
        for gi, (g, (lo, hi)) in enumerate(zip(groups, span)):
            stream.wait_event(landed[b][gi])
            if not fresh[b][gi]:
                stream.wait_event(out[b][gi])
            for i in g:
                (r, M), off = calls[i], offs[i]
                ffn(dev_x[b][off:off + M], M, r, (k + i) % args.copies, y=dev_y[b][off:off + M])
            used[b][gi].record(stream)
            d2h_s.wait_event(used[b][gi])
            with torch.cuda.stream(d2h_s):
                host_y[lo:hi].copy_(dev_y[b][lo:hi], non_blocking=True)
            out[b][gi].record(d2h_s)
            fresh[b][gi] = False

    def run(n, start):
        for k in range(n):
            step(k, start)
        done = torch.cuda.Event()
        done.record(d2h_s)  # copies on d2h_s run in issue order: every output is on the host
        stream.wait_event(done)

    with torch.cuda.stream(stream):
        s0 = torch.cuda.Event()
        s0.record(stream)
        run(max(1, args.warmup), s0)
        torch.cuda.synchronize()
        barrier(world)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        run(args.steps, e0)
        e1.record(stream)
        torch.cuda.synchronize()
        # every step computes the same outputs (the weight copies are identical and the kernels
        # deterministic): the pipelined copies must have brought back exactly those of a plain
        # step with no overlap
        want = torch.empty_like(dev_y[0])
        xin = host_x.to(dev)
        for i, ((r, M), off) in enumerate(zip(calls, offs)):
            ffn(xin[off:off + M], M, r, i % args.copies, y=want[off:off + M])
        torch.cuda.synchronize()
    same = torch.equal(want.cpu().view(torch.int16), host_y.view(torch.int16))
    ms = max_over_ranks(world, e0.elapsed_time(e1), dev) / args.steps  # every rank takes part
    if not same:
        raise RuntimeError("end-to-end step: outputs copied back differ from a serial step's")
    b, f = step_units(spec)
    v = whole_job_value(spec["unit"], b, f, world, ms)
    return {"value": v, "unit": spec["unit"], "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": ms, "copy_runs_per_step": len(groups), "buffers": nbuf, "outputs_checked": True}


def run_pack_case(args):
    """The one-time int8 -> plane-layout pack of every 8B and 9B FFN matrix (all planes,
    r_keep = 8), timed with CUDA events over 20 back-to-back packs each (inputs > L2):
    GB/s of its N*K bytes read + N*K bytes written."""
    import torch
    from nested_bit_weight_msb_b200 import matq
    torch.cuda.set_device(0)
    rng = np.random.default_rng(0)
    out = {}
    for name, (N, K) in (("8b gate/up", (14336, 4096)), ("8b down", (4096, 14336)),
                         ("9b gate/up", (14336, 3584)), ("9b down", (3584, 14336))):
        codes = [torch.from_numpy(rng.integers(0, 256, (N, K), dtype=np.uint8)).cuda() for _ in range(3)]
        planes = torch.empty(matq.matq_packed_bytes(N, K, 8), dtype=torch.uint8, device="cuda")
        stream = torch.cuda.current_stream()
        for i in range(3):
            matq.check(matq.matq_pack(codes[i].data_ptr(), N, K, 8, planes.data_ptr(), planes.numel(),
                                      stream.cuda_stream), "matq_pack")
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        n = 20
        e0.record()
        for i in range(n):
            matq.check(matq.matq_pack(codes[i % 3].data_ptr(), N, K, 8, planes.data_ptr(), planes.numel(),
                                      stream.cuda_stream), "matq_pack")
        e1.record()
        torch.cuda.synchronize()
        us = e0.elapsed_time(e1) / n * 1e3
        out[name] = {"us": round(us, 2), "GB/s": round(2 * N * K / us / 1e3, 1)}
    print(json.dumps({"case": "pack", "r_keep": 8, "results": out}))
    return 0


def cpu_choose_rate(budget_s=10.0, rows=8):
    """The oracle's parent-code choice (as it stands: fp32 brute force over all 256 codes) timed
    on the host cores on a bounded sample: the first `rows` rows of the 8B gate matrix, widths
    {3, 4, 8}, equal lambdas, centred reconstruction, repeated until `budget_s` is spent."""
    import oracle as O
    from nested_bit_weight_msb_b200 import synth
    w, s, z = synth.float_weights(rows, D_MODEL, GROUP, seed=0)
    done, n_iter = 0, 0
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < budget_s or n_iter == 0:
        O.choose_codes(w, s, z, GROUP, (3, 4, 8))
        done += w.size
        n_iter += 1
    dt = time.perf_counter() - t0
    cores = os.cpu_count()
    try:
        import threadpoolctl
        cores = max((i.get("num_threads", 1) for i in threadpoolctl.threadpool_info()), default=cores)
    except Exception:
        pass
    return {"value": done / dt / 1e9, "unit": "Gweights/s", "cores": cores, "kind": "oracle",
            "sample": f"first {rows} rows of the 8B gate matrix (x {D_MODEL} inputs), {n_iter} pass(es), {dt:.1f} s"}


def run_choose_case(args):
    """The parent-code choice for several widths (matq_choose_codes) on every 8B and 9B FFN
    matrix: widths {3, 4, 8} with equal lambdas (the pages' width set), centred and truncated
    reconstruction, timed with CUDA events over 10 back-to-back calls each (the fp32 weights,
    > 200 MB a matrix, exceed L2).  Reports weights per second and GB/s of the call's bytes
    (4 B of w read + 1 B of code written per weight, 3 B of scale and zero point per group)
    against the measured copy peak; the search itself is fp32 ALU work."""
    import torch
    from nested_bit_weight_msb_b200 import matq, synth
    torch.cuda.set_device(0)
    peaks = load_peaks()
    out = {}
    for name, (N, K, g) in (("8b gate/up", (14336, 4096, 128)), ("8b down", (4096, 14336, 128)),
                            ("9b gate/up", (14336, 3584, 64)), ("9b down", (3584, 14336, 64))):
        w, s, z = synth.float_weights(N, K, g, seed=0)
        dw = torch.from_numpy(w).cuda()
        ds = torch.from_numpy(s.view(np.int16)).cuda()
        dz = torch.from_numpy(z).cuda()
        codes = torch.empty((N, K), dtype=torch.uint8, device="cuda")
        for mode, mname in ((matq.MATQ_SLICE_TRUE_PREFIX, "true_prefix"), (matq.MATQ_SLICE_TRUNCATE, "truncate")):
            def call():
                matq.choose_codes(dw, ds, dz, g, (3, 4, 8), None, mode, out=codes)
            for _ in range(3):
                call()
            torch.cuda.synchronize()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            n = 10
            e0.record()
            for _ in range(n):
                call()
            e1.record()
            torch.cuda.synchronize()
            us = e0.elapsed_time(e1) / n * 1e3
            nbytes = N * K * 5 + N * (K // g) * 3
            out[f"{name} {mname}"] = {"us": round(us, 1), "Gweights/s": round(N * K / us / 1e3, 1),
                                      "GB/s": round(nbytes / us / 1e3, 1),
                                      "frac_of_copy_peak": round(nbytes / us / 1e3 / peaks["hbm_gbs"], 3)}
    line = {"case": "choose", "widths": [3, 4, 8], "lambdas": "equal", "results": out,
            "peak_hbm_gbs": peaks["hbm_gbs"], "peaks_source": peaks["_source"]}
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_choose_rate()
    print(json.dumps(line))
    return 0


def run_speedup_case(args):
    """The pages' own comparison: the sliced linear layer against torch.matmul (cuBLAS) in bf16
    on a dense weight of the same shape, at the decode batch sizes.  For each 8B FFN matrix and
    M in {1, 4, 16}: microseconds per call of torch.matmul(x, W^T) and of matq.linear at every
    width, both as CUDA graphs of 20 back-to-back calls over rotating weight copies (> L2), and
    the ratio.  Dense weight values do not change cuBLAS's time, so random bf16 values stand in
    for the dequantised W."""
    import torch
    from nested_bit_weight_msb_b200 import matq, synth
    torch.cuda.set_device(0)
    copies, calls = 3, 20

    def graph_us(fn):
        st = torch.cuda.Stream()
        with torch.cuda.stream(st):
            for i in range(3):
                fn(i)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(calls):
                fn(i)
        g.replay()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        g.replay()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / calls * 1e3

    out = {}
    for name, (N, K) in (("8b gate/up", (D_FF, D_MODEL)), ("8b down", (D_MODEL, D_FF))):
        dense = [torch.randn((N, K), dtype=torch.bfloat16, device="cuda") for _ in range(copies)]
        q, s, z = synth.parent_weights(N, K, GROUP, seed=0)
        p0 = matq.pack(torch.from_numpy(q).cuda(), 8)
        packs = [p0] + [p0.clone() for _ in range(copies - 1)]
        ds = torch.from_numpy(s.view(np.int16)).cuda()
        dz = torch.from_numpy(z).cuda()
        for M in (1, 4, 16):
            xb, _ = synth.activations(M, K, seed=0)
            x = torch.from_numpy(xb.view(np.int16)).cuda().view(torch.bfloat16)
            y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
            ws = matq.workspace(M, K, N, GROUP)
            t_ref = graph_us(lambda i: torch.matmul(x, dense[i % copies].t(), out=y))
            row = {"torch.matmul bf16 us": round(t_ref, 2)}
            for r in WIDTHS:
                t = graph_us(lambda i: matq.linear(x, packs[i % copies], 8, ds, dz, N, r, GROUP, y=y, workspace=ws))
                row[f"r={r} us"] = round(t, 2)
                row[f"r={r} speedup"] = round(t_ref / t, 2)
            out[f"{name} M={M}"] = row
        del dense, packs
        torch.cuda.empty_cache()
    print(json.dumps({"case": "speedup", "baseline": "torch.matmul bf16 (cuBLAS), dense weight of the same shape",
                      "results": out}))
    return 0


# ---------------------------------------------------------------------------------------------
# the Mix'n'Match stack: 32 FFN layers of 8B shape, a width per layer
# ---------------------------------------------------------------------------------------------
STACK_LAYERS = 32
STACK_BATCHES = (1, 16, 512)


def stack_perms(layers=STACK_LAYERS):
    """Seeded row permutations that make the stack's layers distinct matrices with the base
    layer's statistics: gate/up by row pairs (a gate row stays next to its up row), down by rows."""
    out = []
    for l in range(layers):
        rng = np.random.default_rng([7, l])
        out.append((rng.permutation(D_FF), rng.permutation(D_MODEL)))
    return out


def stack_rows(perm_pairs):
    return np.stack([2 * perm_pairs, 2 * perm_pairs + 1], axis=1).reshape(-1)


def stack_layer_host(fused, perms, l):
    """Host (codes, scales, zeros) of layer l's gate+up and down matrices."""
    pp, pd = perms[l]
    idx = stack_rows(pp)
    return tuple(a[idx] for a in fused["gate_up"]), tuple(a[pd] for a in fused["down"])


def stack_units(M, widths):
    """(algorithmic bytes, flops) of one pass: per layer the gated gate+up call (bf16 in and out)
    and the down call accumulating into the fp32 residual (read and written: 8 bytes per
    element); the RMSNorm is not counted."""
    b = f = 0
    G = D_MODEL // GROUP
    for r in widths:
        b += linear_bytes(M, 2 * D_FF, D_MODEL, r, out_cols=D_FF)
        b += D_MODEL * D_FF * r // 8 + D_MODEL * (D_FF // GROUP) * 3 + M * D_FF * 2 + M * D_MODEL * 8
        f += 2 * M * (2 * D_FF * D_MODEL + D_MODEL * D_FF)
    del G
    return b, f


class StackBench:
    """Device state of the 32-layer stack: every layer packed keeping only its width's planes
    (deployment mode A), the residual stream h (fp32), and the pass h <- h + FFN_l(RMSNorm(h))."""

    def __init__(self, weights, dev, rank):
        import torch
        from nested_bit_weight_msb_b200 import matq, synth
        self.matq = matq
        self.widths = [int(w) for w in synth.mixnmatch_widths(0, layers=STACK_LAYERS)]
        fused = fused_weights(weights)
        perms = stack_perms()
        q_gu = torch.from_numpy(fused["gate_up"][0]).to(dev)
        s_gu = torch.from_numpy(fused["gate_up"][1].view(np.int16)).to(dev)
        z_gu = torch.from_numpy(fused["gate_up"][2]).to(dev)
        q_d = torch.from_numpy(fused["down"][0]).to(dev)
        s_d = torch.from_numpy(fused["down"][1].view(np.int16)).to(dev)
        z_d = torch.from_numpy(fused["down"][2]).to(dev)
        self.layers = []
        for l, r in enumerate(self.widths):
            pp, pd = perms[l]
            idx = torch.from_numpy(stack_rows(pp)).to(dev)
            pdt = torch.from_numpy(pd).to(dev)
            self.layers.append({
                "r": r,
                "gu": (matq.pack(q_gu.index_select(0, idx), r_keep=r), s_gu.index_select(0, idx).contiguous(),
                       z_gu.index_select(0, idx).contiguous()),
                "d": (matq.pack(q_d.index_select(0, pdt), r_keep=r), s_d.index_select(0, pdt).contiguous(),
                      z_d.index_select(0, pdt).contiguous()),
            })
        del q_gu, q_d
        self.h0, self.h, self.n, self.a = {}, {}, {}, {}
        for M in STACK_BATCHES:
            _, xv = synth.activations(M, D_MODEL, seed=rank, outlier_frac=0.01 if M > 16 else 0.0)
            self.h0[M] = torch.from_numpy(np.ascontiguousarray(xv, dtype=np.float32)).to(dev)
            self.h[M] = torch.empty((M, D_MODEL), dtype=torch.float32, device=dev)
            self.n[M] = torch.empty((M, D_MODEL), dtype=torch.bfloat16, device=dev)
            self.a[M] = torch.empty((M, D_FF), dtype=torch.bfloat16, device=dev)
        Mmax = max(STACK_BATCHES)
        self.ws = torch.zeros(max(matq.workspace_bytes(Mmax, K, N, GROUP) for _, (N, K) in FFN_CALLS),
                              dtype=torch.uint8, device=dev)
        torch.cuda.synchronize()

    def layer(self, lay, M, h):
        m = self.matq
        m.rmsnorm(h, eps=1e-5, out=self.n[M])
        p, s, z = lay["gu"]
        m.linear(self.n[M], p, lay["r"], s, z, 2 * D_FF, lay["r"], GROUP, y=self.a[M],
                 y_mode=m.MATQ_OUT_SILU_GATED, workspace=self.ws)
        p, s, z = lay["d"]
        m.linear(self.a[M], p, lay["r"], s, z, D_MODEL, lay["r"], GROUP, y=h, y_mode=m.MATQ_OUT_F32_ACCUM,
                 workspace=self.ws)

    def run(self, M, h=None, h0=None):
        """One pass through the 32 layers, starting from h0 (the batch's activations)."""
        h = self.h[M] if h is None else h
        h.copy_(self.h0[M] if h0 is None else h0)
        for lay in self.layers:
            self.layer(lay, M, h)


def cpu_stack_rate(weights, budget_s=12.0, rows=128):
    """The fp64 oracle on a bounded sample of the stack: the first `rows` rows of each matrix of
    the first layers at M = 1, teacher-forced from N(0, 1) inputs; GB/s of algorithmic bytes."""
    import oracle as O
    from nested_bit_weight_msb_b200 import synth
    fused = fused_weights(weights)
    perms = stack_perms()
    widths = synth.mixnmatch_widths(0, layers=STACK_LAYERS)
    rng = np.random.default_rng(0)
    done = 0.0
    t0 = time.perf_counter()
    n_layers = 0
    while time.perf_counter() - t0 < budget_s or n_layers == 0:
        l = n_layers % STACK_LAYERS
        gu, d = stack_layer_host(fused, perms, l)
        r = int(widths[l])
        x = rng.standard_normal((1, D_MODEL))
        O.gated_product(O.linear(x, gu[0][0:rows:2], gu[1][0:rows:2], gu[2][0:rows:2], r, GROUP),
                        O.linear(x, gu[0][1:rows:2], gu[1][1:rows:2], gu[2][1:rows:2], r, GROUP))
        O.linear(rng.standard_normal((1, D_FF)), d[0][:rows], d[1][:rows], d[2][:rows], r, GROUP)
        done += linear_bytes(1, rows, D_MODEL, r) + linear_bytes(1, rows, D_FF, r)
        n_layers += 1
    dt = time.perf_counter() - t0
    return {"value": done / dt / 1e9, "unit": "GB/s", "cores": _oracle_cores(), "kind": "oracle",
            "sample": f"first {rows} rows of gate+up and down of {n_layers} stack layer(s) at M = 1, {dt:.1f} s",
            "seconds": dt}


def _oracle_cores():
    cores = os.cpu_count()
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        cores = max((i.get("num_threads", 1) for i in info), default=cores)
    except Exception:
        pass
    return cores


def stack_config(widths, world):
    return {"workload": "stack32", "layers": STACK_LAYERS, "widths": list(widths),
            "mean_bits": float(np.mean(widths)), "batches": list(STACK_BATCHES),
            "shapes": "per layer: gate+up [28672,4096] (gated product in the epilogue), down [4096,14336] "
                      "into the fp32 residual, group 128; layers are row-permuted copies of one seeded "
                      "8B FFN layer, each packed with only its width's planes",
            "parallelism": f"replicas x{world}", "l2": "32 distinct layers (2+ GB of planes) > L2",
            "timing": "one CUDA graph per pass, CUDA events"}


def run_stack(args):
    """--workload stack32: the Mix'n'Match stack.  One step = one pass through the 32 layers at
    each decode batch (M = 1 and 16), each pass one CUDA graph; the M = 512 pass (prefill path) is
    timed the same way and reported beside it.  value = algorithmic bytes of the decode passes
    over their device time."""
    import torch
    world, rank, local = dist_setup()
    maybe_init_pg(world, "nccl")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    weights = host_weights()
    sb = StackBench(weights, dev, rank)
    stream = torch.cuda.Stream(device=dev)
    peaks = load_peaks()
    graphs = {}
    with torch.cuda.stream(stream):
        for M in STACK_BATCHES:
            sb.run(M)
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                sb.run(M)
            graphs[M] = g
        for _ in range(args.warmup):
            for M in STACK_BATCHES:
                graphs[M].replay()
        torch.cuda.synchronize()
    if sb.matq.workspace_status(sb.ws) != 0:
        raise RuntimeError("device status after warm-up: the stack did not complete normally")
    per_m = {}
    clk = None
    for M in STACK_BATCHES:
        with torch.cuda.stream(stream):
            barrier(world)
            torch.cuda.synchronize()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            with ClockSampler(local) as c:
                e0.record(stream)
                for _ in range(args.steps):
                    graphs[M].replay()
                e1.record(stream)
                torch.cuda.synchronize()
            if M == 1:
                clk = c.summary()
        per_m[M] = max_over_ranks(world, e0.elapsed_time(e1), dev) / args.steps
    if sb.matq.workspace_status(sb.ws) != 0:
        raise RuntimeError("device status after the timed region: the stack did not complete normally")
    dec = [M for M in STACK_BATCHES if M <= 16]
    b_dec = sum(stack_units(M, sb.widths)[0] for M in dec)
    ms_step = sum(per_m[M] for M in dec)
    value = b_dec * world / (ms_step * 1e-3) / 1e9
    table = []
    for M in STACK_BATCHES:
        b, f = stack_units(M, sb.widths)
        row = {"M": M, "us": round(per_m[M] * 1e3, 1)}
        if M <= 16:
            v = b / (per_m[M] * 1e-3) / 1e9
            row.update({"GB/s": round(v, 1), "frac": round(v / peaks["hbm_gbs"], 3)})
        else:
            v = f / (per_m[M] * 1e-3) / 1e12
            row.update({"TFLOP/s": round(v, 1), "frac": round(v / peaks["bf16_tflops"], 3)})
        table.append(row)
    b1 = stack_units(1, sb.widths)[0]
    ach = b1 / (per_m[1] * 1e-3) / 1e9
    rl = {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": ach / peaks["hbm_gbs"],
          "traffic": None, "algorithmic_bytes": b1, "avg_us": per_m[1] * 1e3,
          "kernel": "one 32-layer pass at M = 1 (per layer: RMSNorm, gated gate+up, down into the fp32 residual)",
          "peak_source": peaks.get("_source")}
    # end to end: the decode passes through the public calls, the batches' activations copied in
    # from pinned host memory and the final residual streams copied back, every step
    host_in = {M: sb.h0[M].cpu().pin_memory() for M in dec}
    host_out = {M: torch.empty((M, D_MODEL), dtype=torch.float32).pin_memory() for M in dec}
    dev_in = {M: torch.empty_like(sb.h0[M]) for M in dec}
    with torch.cuda.stream(stream):
        def e2e_step():
            for M in dec:
                dev_in[M].copy_(host_in[M], non_blocking=True)
                sb.run(M, h0=dev_in[M])
                host_out[M].copy_(sb.h[M], non_blocking=True)
        for _ in range(max(1, args.warmup)):
            e2e_step()
        torch.cuda.synchronize()
        barrier(world)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
    ms_e2e = max_over_ranks(world, e0.elapsed_time(e1), dev) / args.steps
    for M in dec:
        if not torch.equal(host_out[M].to(dev), sb.h[M]):
            raise RuntimeError("end-to-end stack: the copied-back residual differs from the device one")
    e2e = {"value": b_dec * world / (ms_e2e * 1e-3) / 1e9, "unit": "GB/s",
           "h2d_bytes_per_step": sum(M * D_MODEL * 4 for M in dec), "d2h_bytes_per_step": sum(M * D_MODEL * 4 for M in dec),
           "ms_per_step": ms_e2e}
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": DTYPES["GB/s"], "data": "synthetic",
            "config": stack_config(sb.widths, world),
            "roofline": rl, "per_M": table, "e2e": e2e,
            "gpu_launches": args.steps * sum(STACK_LAYERS * (3 if M <= 16 else 5) for M in dec),
            "clocks": clk, "peaks_source": peaks.get("_source"),
        }
        if not args.no_cpu_baseline and world == 1:
            line["cpu_baseline"] = cpu_stack_rate(weights)
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


# ---------------------------------------------------------------------------------------------
# matrix sweeps: the Gemma-2-9B-shaped FFN over batch sizes, the 1024 x 1024 layer
# ---------------------------------------------------------------------------------------------
SWEEPS = {
    "ffn9b_sweep": {"d_model": 3584, "d_ff": 14336, "group": 64, "batches": (1, 8, 32, 128, 512, 2048),
                    "widths": WIDTHS, "ffn": True},
    "linear1024": {"n": 1024, "k": 1024, "group": 128, "batches": (1,), "widths": WIDTHS, "ffn": False},
}


def sweep_mats(sw):
    """Host (codes, scales, zeros) of a sweep's matrices: the 9B FFN's gate and up row-interleaved
    into one gated matrix plus down, or the single 1024 x 1024 layer."""
    from nested_bit_weight_msb_b200 import synth
    g = sw["group"]
    if sw["ffn"]:
        d, f = sw["d_model"], sw["d_ff"]
        w = {name: synth.parent_weights(N, K, g, seed=0, layer=0, proj=name)
             for name, (N, K) in (("gate", (f, d)), ("up", (f, d)), ("down", (d, f)))}
        return {"gate_up": tuple(interleave_rows(w["gate"][i], w["up"][i]) for i in range(3)), "down": w["down"]}
    return {"linear": synth.parent_weights(sw["n"], sw["k"], g, seed=0, layer=0, proj="gate")}


def sweep_config(args, sw, shapes, world):
    return {"workload": args.workload, "group": sw["group"], "batches": list(sw["batches"]),
            "widths": list(sw["widths"]), "shapes": shapes,
            "parallelism": f"replicas x{world}", "l2": "rotating device copies of each pack (> 2x L2)",
            "timing": "each call: CUDA graph of back-to-back launches, median of 5 replays"}


def run_sweep(args):
    """--workload ffn9b_sweep (Gemma-2-9B-shaped FFN: gate+up [28672, 3584] with the gated epilogue,
    down [3584, 14336], group 64, M in {1, 8, 32, 128, 512, 2048}, every width, and the one-time
    pack of each matrix) and --workload linear1024 (one 1024 x 1024 layer, group 128, M = 1, every
    width).  Every sliced-linear call is timed on its own as back-to-back launches over rotating
    weight copies (> 2x L2), with its roofline: decode batches (M <= 16) against the HBM copy peak,
    larger ones against min(bf16 peak, arithmetic intensity x HBM peak).  value = algorithmic bytes
    of the decode-batch calls over their device time."""
    import torch
    from nested_bit_weight_msb_b200 import matq, synth
    world, rank, local = dist_setup()
    maybe_init_pg(world, "nccl")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    sw = SWEEPS[args.workload]
    g = sw["group"]
    peaks = load_peaks()
    mats = sweep_mats(sw)
    state = {}
    for name, (q, sc, z) in mats.items():
        N, K = q.shape
        p0 = matq.pack(torch.from_numpy(q).to(dev), r_keep=8)
        copies = int(min(256, max(2, (512 << 20) // p0.numel() + 1)))
        state[name] = {"N": N, "K": K, "packs": [p0] + [p0.clone() for _ in range(copies - 1)],
                       "s": torch.from_numpy(sc.view(np.int16)).to(dev), "z": torch.from_numpy(z).to(dev),
                       "gated": name == "gate_up"}
    Mmax = max(sw["batches"])
    ws = torch.zeros(max(matq.workspace_bytes(Mmax, st["K"], st["N"], g) for st in state.values()),
                     dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream(device=dev)
    table, dec_b, dec_us = [], 0, 0.0
    total_us = 0.0
    with ClockSampler(local) as clk:
        for M in sw["batches"]:
            xs = {}
            for name, st in state.items():
                K = st["K"]
                xb, _ = synth.activations(M, K, seed=rank, outlier_frac=0.01 if M > 16 else 0.0)
                xs[name] = torch.from_numpy(xb.view(np.int16)).to(dev).view(torch.bfloat16)
            for r in sw["widths"]:
                row = {"M": M, "r": r}
                for name, st in state.items():
                    N, K = st["N"], st["K"]
                    cols = N // 2 if st["gated"] else N
                    y = torch.empty((M, cols), dtype=torch.bfloat16, device=dev)
                    mode = matq.MATQ_OUT_SILU_GATED if st["gated"] else matq.MATQ_OUT_BF16
                    n = len(st["packs"])
                    us = graph_us_per_call(lambda i: matq.linear(xs[name], st["packs"][i % n], 8, st["s"], st["z"], N, r,
                                                                 g, y=y, y_mode=mode, workspace=ws), stream,
                                           n=24)
                    b = linear_bytes(M, N, K, r, group=g, out_cols=cols)
                    fl = 2 * M * N * K
                    gbs, tfs = b / (us * 1e-6) / 1e9, fl / (us * 1e-6) / 1e12
                    if M <= 16:
                        roof, frac = "hbm", gbs / peaks["hbm_gbs"]
                        dec_b += b
                        dec_us += us
                    else:
                        lim = min(peaks["bf16_tflops"], fl / b * peaks["hbm_gbs"] / 1e3)
                        roof, frac = ("tensor" if lim == peaks["bf16_tflops"] else "hbm"), tfs / lim
                    total_us += us
                    row[name] = {"us": round(us, 2), "GB/s": round(gbs, 1), "TFLOP/s": round(tfs, 1),
                                 "bound": roof, "frac": round(frac, 3)}
                table.append(row)
    if matq.workspace_status(ws) != 0:
        raise RuntimeError("device status after the sweep: a call did not complete normally")
    # the one-time pack of each matrix (all planes), 20 back-to-back packs over 3 code copies
    pack = {}
    if sw["ffn"]:
        rng = np.random.default_rng(0)
        for name, st in state.items():
            N, K = st["N"], st["K"]
            codes = [torch.from_numpy(rng.integers(0, 256, (N, K), dtype=np.uint8)).to(dev) for _ in range(3)]
            planes = torch.empty(matq.matq_packed_bytes(N, K, 8), dtype=torch.uint8, device=dev)
            us = graph_us_per_call(lambda i: matq.check(
                matq.matq_pack(codes[i % 3].data_ptr(), N, K, 8, planes.data_ptr(), planes.numel(),
                               torch.cuda.current_stream().cuda_stream), "matq_pack"), stream, n=20)
            gbs = 2 * N * K / (us * 1e-6) / 1e9
            pack[name] = {"N": N, "K": K, "us": round(us, 2), "GB/s": round(gbs, 1),
                          "frac": round(gbs / peaks["hbm_gbs"], 3)}
            del codes, planes
    value = dec_b * world / (dec_us * 1e-6) / 1e9
    first = table[0]
    name0 = "gate_up" if sw["ffn"] else "linear"
    dom = [r for r in table if r["M"] == min(sw["batches"]) and r["r"] == 2][0][name0]
    rl = {"bound": "hbm", "achieved": dom["GB/s"], "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": dom["frac"],
          "traffic": None, "avg_us": dom["us"], "kernel": f"decode_kernel via matq_linear ({name0} r=2 M={first['M']})",
          "peak_source": peaks.get("_source")}
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": 1, "warmup": 3,
            "ms_per_step": total_us / 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": DTYPES["GB/s"], "data": "synthetic",
            "config": sweep_config(args, sw, {k: [v["N"], v["K"]] for k, v in state.items()}, world),
            "roofline": rl, "per_call": table, "pack": pack, "clocks": clk.summary(),
            "e2e": None, "e2e_note": "per-call sweep: the end-to-end form is measured on the FFN workloads",
            "peaks_source": peaks.get("_source"),
        }
        if not args.no_cpu_baseline and world == 1:
            line["cpu_baseline"] = cpu_sweep_rate(mats, g, [M for M in sw["batches"] if M <= 16], sw["widths"])
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def cpu_sweep_rate(mats, group, batches, widths, budget_s=12.0, rows=128):
    """The fp64 oracle on a bounded sample of a sweep's decode calls: the first `rows` rows of each
    matrix at every width and decode batch; GB/s of algorithmic bytes."""
    import oracle as O
    rng = np.random.default_rng(0)
    done = 0.0
    t0 = time.perf_counter()
    passes = 0
    while time.perf_counter() - t0 < budget_s or passes == 0:
        for r in widths:
            for M in batches:
                for q, s, z in mats.values():
                    K = q.shape[1]
                    O.linear(rng.standard_normal((M, K)), q[:rows], s[:rows], z[:rows], r, group)
                    done += linear_bytes(M, rows, K, r, group=group)
        passes += 1
    dt = time.perf_counter() - t0
    return {"value": done / dt / 1e9, "unit": "GB/s", "cores": _oracle_cores(), "kind": "oracle",
            "sample": f"first {rows} rows of each matrix at every width and decode batch, {passes} pass(es), {dt:.1f} s",
            "seconds": dt}


def run_case(args):
    """A few single calls of the gate+up projection (28672 x 4096 row-interleaved, group 128,
    gated-product epilogue, as in the workloads) at width r and batch m, rotating through
    device copies of the pack (> L2); used for ncu captures.
    `--case pack` times the one-time pack instead; `--case ep` makes the same calls on the
    Extra-Precision slice (clamped-level pack plus overflow list) of width r."""
    if args.case == "choose":
        return run_choose_case(args)
    if args.case == "speedup":
        return run_speedup_case(args)
    if args.case == "pack":
        return run_pack_case(args)
    import torch
    from nested_bit_weight_msb_b200 import matq, synth
    torch.cuda.set_device(0)
    q, s, z = fused_weights(host_weights())["gate_up"]
    N = q.shape[0]
    p0 = matq.pack(torch.from_numpy(q).cuda(), r_keep=8)
    packs = [p0] + [p0.clone() for _ in range(args.copies - 1)]
    ds = torch.from_numpy(s.view(np.int16)).cuda()
    dz = torch.from_numpy(z).cuda()
    xb, _ = synth.activations(args.m, D_MODEL, seed=0, outlier_frac=0.01 if args.case == "prefill" else 0.0)
    dx = torch.from_numpy(xb.view(np.int16)).cuda().view(torch.bfloat16)
    ws = matq.workspace(args.m, D_MODEL, N, GROUP)
    gated = True
    y = torch.empty((args.m, N // 2 if gated else N), dtype=torch.bfloat16, device="cuda")
    mode = matq.MATQ_OUT_SILU_GATED if gated else matq.MATQ_OUT_BF16
    if args.case == "ep":
        slices = [matq.round_extract(p, N, D_MODEL, 8, args.r) for p in packs]
        ws = matq.rounded_workspace(args.m, D_MODEL, N, GROUP)
        for i in range(args.calls):
            lv, rp, cl = slices[i % len(slices)]
            matq.linear_rounded(dx, lv, args.r, ds, dz, N, GROUP, rp, cl, y=y, y_mode=mode, workspace=ws)
    for i in range(args.calls if args.case != "ep" else 0):
        matq.linear(dx, packs[i % len(packs)], 8, ds, dz, N, args.r, GROUP, y=y, y_mode=mode, workspace=ws)
    torch.cuda.synchronize()
    assert matq.workspace_status(ws) == 0
    print(json.dumps({"case": args.case, "r": args.r, "m": args.m, "calls": args.calls, "ok": True}))
    return 0


def main():
    args = parse()
    if args.case:
        return run_case(args)
    if args.impl == "reference":
        return run_reference(args)
    if args.workload == "stack32":
        return run_stack(args)
    if args.workload in SWEEPS:
        return run_sweep(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
