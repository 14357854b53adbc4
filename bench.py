#!/usr/bin/env python
"""Benchmark of the fused int8 GroupedMatmul + MoeFinalizeRouting op on B200.

One step = one ``qgmm_finalize`` call (output init + persistent grouped GEMM
with the fused dequant/combine epilogue; plus the per-token quant prologue on
workloads that have one) over one batch of seeded synthetic inputs already
resident in HBM.  Default workload: the large prefill (tokens=16384, topK=8,
m=131072, e=256, k=2048, n=7168, Dirichlet(0.3) routing, bf16 sharedInput),
atomic combine.  The metric is effective INT8 TOPS = 2 * sum_g m_g * k * n / t.

Multi-GPU (torchrun, one process per GPU): the op's output columns are split
across the GPUs (whole 256-column tiles, as evenly as the tile count allows);
every rank holds x1 and the routing in full and its own columns of the weights,
scale, bias and sharedInput, and computes its own output columns -- no
collective on the data path (strong scaling: the total work is the one
workload).  ``value`` is the whole workload's work over the slowest rank's
device time.

``--impl reference`` times the CPU oracle instead, on a bounded sample of the
same workload's output rows (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "effective INT8 TOPS and % of B200 dense INT8 peak; HBM GB/s at decode m"
NOMINAL_INT8_TOPS = 4500.0
NOMINAL_HBM_GBS = 8000.0
KERNEL_SOURCES = ["quantized_moe_grouped_persistent_b200/csrc/kernels.cuh",
                  "quantized_moe_grouped_persistent_b200/csrc/ptx_sm100.cuh"]
TRAFFIC_SUMMARY = {
    "large_prefill": "profiles/grouped_gemm_large_prefill.md",
    "decode": "profiles/grouped_gemm_decode.md",
    "w4a8_prologue": "profiles/grouped_gemm_w4a8.md",
    "w4a8_mx": "profiles/grouped_gemm_w4a8_mx.md",
    "mid_prefill": "profiles/grouped_gemm_mid_prefill.md",
}


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="large_prefill")
    ap.add_argument("--deterministic", action="store_true", help="time the fixed-order combine instead")
    ap.add_argument("--no-extras", action="store_true", help="skip the decode / deterministic / e2e side runs")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="target oracle time for cpu_baseline")
    ap.add_argument("--tokens", type=int, default=None, help="shrink the workload (profiling proxies)")
    ap.add_argument("--experts", type=int, default=None, help="shrink the workload (profiling proxies)")
    ap.add_argument("--transpose-x2", action="store_true",
                    help="store the int8 / E4M3 weights (e, n, k) instead of (e, k, n); same result")
    return ap.parse_args()


# ----------------------------------------------------------------------------- helpers
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return dict(hbm_gbs=d["hbm_gbs"], bf16=d["bf16_tflops"], bf16_sustained=d["bf16_tflops_sustained"],
                    source="measured")
    return dict(hbm_gbs=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


def kernel_sources_sha():
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        h.update(open(os.path.join(ROOT, rel), "rb").read())
    return h.hexdigest()[:16]


def committed_traffic(workload):
    """DRAM bytes per launch of the grouped GEMM from the committed ncu summary, if still current."""
    rel = TRAFFIC_SUMMARY.get(workload)
    if not rel or not os.path.exists(os.path.join(ROOT, rel)):
        return None
    text = open(os.path.join(ROOT, rel)).read()
    m_sha = re.search(r"kernel_sources_sha256:\s*([0-9a-f]+)", text)
    m_b = re.search(r"dram_bytes_per_launch:\s*([0-9]+)", text)
    if not m_sha or not m_b or m_sha.group(1) != kernel_sources_sha():
        return None
    return int(m_b.group(1))


def total_rows(p):
    return int(p.counts.sum())


def int_ops(p):
    return 2.0 * total_rows(p) * p.k * p.n


def algorithmic_bytes(p):
    """Bytes the step must move at least once: the used experts' weights (and their
    scale/bias rows), x1 (or the bf16 activations), the per-row vectors, the output
    written once, and the sharedInput read once."""
    used = int((p.counts > 0).sum())
    w_bytes = p.k * p.n // 2 if p.weight in ("int4", "mxfp4") else p.k * p.n
    scale_bytes = p.n * p.k // 32 if p.weight == "mxfp4" else 4 * p.n     # E8M0 per 32 k, or f32 per column
    per_expert = w_bytes + scale_bytes + (4 * p.n if p.bias is not None else 0)
    b = used * per_expert
    m = total_rows(p)
    if p.x1 is not None:
        b += m * p.k
    elif p.weight == "mxfp4":   # the FP8 cast reads bf16, writes E4M3 + a scale byte per 32; the GEMM reads both
        b += m * p.k * 2 + 2 * (m * p.k + m * p.k // 32)
    else:                       # the int8 prologue reads bf16, writes int8 + a scale; the GEMM reads both
        b += m * p.k * 2 + m * p.k + 4 * m
    b += m * (4 + 4 + p.row_index.dtype.itemsize)
    b += p.output_bs * p.n * 4
    if p.shared is not None:
        b += p.shared.size * 2
    return float(b)


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        self.ident = str(device_index)
        try:
            import torch
            u = getattr(torch.cuda.get_device_properties(device_index), "uuid", None)
            if u is not None:
                s = str(u)
                self.ident = s if s.startswith("GPU-") else "GPU-" + s
        except Exception:
            pass

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.ident, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = []
        for line in out.strip().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) != 7:
                continue
            try:
                rows.append((float(parts[0]), float(parts[1]), parts[3:]))
            except ValueError:
                continue
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i, v in enumerate(r) if v.lower().startswith("active")})
        sm = sorted(x[0] for x in rows)
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": max(x[1] for x in rows), "reasons": reasons,
                "samples": len(rows)}


# ----------------------------------------------------------------------------- ranks
def rank_problem(p_full, world: int, rank: int):
    """Rank `rank`'s share of the workload: its block of output columns (the whole
    problem on one GPU).  Every rank draws the same seeded problem and keeps its
    columns of x2, scale, bias and sharedInput."""
    from quantized_moe_grouped_persistent_b200.shard import column_block, slice_columns
    c0, c1 = column_block(p_full.n, world, rank)
    if c1 == c0:
        raise SystemExit(f"{world} GPUs exceed the {p_full.n // 256} column tiles of the workload")
    return (p_full if world == 1 else slice_columns(p_full, c0, c1)), (c0, c1)


def max_over_ranks(values, dist=None, device="cpu"):
    """Element-wise max of per-rank timings (every rank takes part; all get the result)."""
    import torch
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if dist is not None:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def strong_scaling_value(total_work: float, ms_max: float) -> float:
    """Whole-job rate: the whole workload's work (ops, or bytes for the decode line)
    over the slowest rank's time, per second, in units of 1e12."""
    return total_work / (ms_max * 1e-3) / 1e12


# ----------------------------------------------------------------------------- device timing
def time_steps(d, steps, warmup, deterministic, dist=None, per_step=None):
    """Device time of `steps` back-to-back calls (CUDA events on the launch stream),
    and the grouped-GEMM kernel's own average duration from events recorded by the
    library around its launch.  If `per_step` is a dict it receives the median and
    the best single-step time (events between consecutive steps)."""
    import torch
    from quantized_moe_grouped_persistent_b200 import finalize_profiled
    stream = torch.cuda.current_stream()
    prob = d.problem(deterministic)
    ws = d.workspace(deterministic)

    def step(b, e):
        d.quantize()
        finalize_profiled(prob, d.x1, d.x2, d.scale, d.pts, d.group_list, d.logit, d.row_index, d.bias, d.shared,
                          d.out, ws, b, e, stream=stream)

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for b, e in ev:            # torch creates the underlying cudaEvent_t on first record
        b.record(stream)
        e.record(stream)
    for _ in range(warmup):
        step(*ev[0])
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    marks = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
    marks[0].record(stream)
    for s in range(steps):
        step(*ev[s])
        marks[s + 1].record(stream)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    ms = marks[0].elapsed_time(marks[-1]) / steps
    gemm_ms = sum(b.elapsed_time(e) for b, e in ev) / steps
    if per_step is not None:
        each = sorted(marks[s].elapsed_time(marks[s + 1]) for s in range(steps))
        gemm_each = sorted(b.elapsed_time(e) for b, e in ev)
        per_step.update(ms_median=each[len(each) // 2], ms_best=each[0],
                        gemm_ms_median=gemm_each[len(gemm_each) // 2], gemm_ms_best=gemm_each[0])
    return ms, gemm_ms


def time_e2e(d, p, steps, warmup, deterministic):
    """Same call through host buffers.  Every step copies its inputs (activations,
    routing, sharedInput) from pinned host memory, runs the op and reads the whole
    output back into pinned host memory; weights stay resident like a served layer's
    parameters.  Steps are double-buffered the way a serving loop runs them: step i's
    input copy (copy stream), op (compute stream) and output copy (second copy stream)
    overlap step i-1's, ordered by events, so the host-to-device and device-to-host
    links both stay busy.  Returns (ms per step, bytes in, bytes out)."""
    import numpy as np
    import torch
    compute = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()

    def pin(a):
        if a is None:
            return None
        if a.dtype == np.uint16:
            a = a.view(np.int16)
        return torch.from_numpy(np.ascontiguousarray(a)).pin_memory()

    host = {"x_bf16": pin(p.x_bf16)} if d.prologue else {"x1": pin(p.x1), "pts": pin(p.pertoken_scale)}
    host.update(group_list=pin(p.group_list.astype(np.int64)), logit=pin(p.logit), row_index=pin(p.row_index))
    if p.shared is not None:
        host["shared"] = pin(p.shared)
    sets = [d, d.io_copy()]
    for sd in sets:
        sd.workspace(deterministic)                        # allocate before timing
    host_out = [torch.empty(tuple(d.out.shape), dtype=torch.float32).pin_memory() for _ in sets]
    h2d = sum(h.numel() * h.element_size() for h in host.values())
    d2h = host_out[0].numel() * 4
    ev = [{k: torch.cuda.Event() for k in ("in", "done", "out")} for _ in sets]
    for e_ in ev:                                          # first waits find completed events
        for x in e_.values():
            x.record(compute)

    def step(i):
        b = i % 2
        sd, e_ = sets[b], ev[b]
        s_in.wait_event(e_["done"])                        # the op of step i-2 has read these inputs
        with torch.cuda.stream(s_in):
            for name, h in host.items():
                getattr(sd, name).copy_(h, non_blocking=True)
        e_["in"].record(s_in)
        compute.wait_event(e_["in"])
        compute.wait_event(e_["out"])                      # step i-2's output has been read back
        sd.run(deterministic=deterministic, stream=compute)
        e_["done"].record(compute)
        s_out.wait_event(e_["done"])
        with torch.cuda.stream(s_out):
            host_out[b].copy_(sd.out, non_blocking=True)
        e_["out"].record(s_out)

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(compute)
    for i in range(steps):
        step(warmup + i)
    for e_ in ev:
        compute.wait_event(e_["out"])                      # the last read-backs are inside the timed region
    t1.record(compute)
    torch.cuda.synchronize()
    return t0.elapsed_time(t1) / steps, h2d, d2h


def gemm_kernel_label(plan, weight="int8"):
    """Which grouped-GEMM kernel(s) a call runs, from the library's own plan (qgmm_plan)."""
    if weight == "mxfp4":
        return "grouped_gemm_mx_kernel"
    if not plan["pair"]:
        return "grouped_gemm_kernel"
    if plan["gemm_launches"] == 2:
        return "grouped GEMM (grouped_gemm_pair_kernel + tail launch)"
    return "grouped_gemm_pair_kernel"


def line_unit(workload, p):
    """The JSON line's unit, and the factor taking int8 TOPS of this workload to it:
    decode is HBM-bound and reports algorithmic GB/s (a sample that does a fraction
    of the ops is credited the same fraction of the workload's algorithmic bytes)."""
    if workload == "decode":
        return "GB/s", 1e3 * algorithmic_bytes(p) / int_ops(p)
    if p.weight in ("fp8", "mxfp4"):
        return "TFLOPS", 1.0
    return "TOPS", 1.0


# ----------------------------------------------------------------------------- CPU oracle timing
def oracle_sample_time(p, target_s, seed):
    """Time the oracle on a seeded sample of output rows sized to about target_s seconds."""
    import numpy as np
    import oracle
    from synth import sample_rows
    threads = oracle.default_threads()
    counts = np.bincount(p.row_index, minlength=p.output_bs)
    kw = {}
    if p.x1 is None:
        q, s = oracle.per_token_quant(p.x_bf16)
        kw = dict(x1=q, pertoken_scale=s)

    def run(nrows, sd):
        rows = sample_rows(sd, p.output_bs, nrows)
        t = time.perf_counter()
        oracle.problem_finalize(p, dest_rows=rows, want32=False, threads=threads, **kw)
        return time.perf_counter() - t, 2.0 * float(counts[rows].sum()) * p.k * p.n, rows.size

    t_cal, _, n_cal = run(max(2, threads // 2), seed)
    per_row = max(t_cal / n_cal, 1e-6)
    nrows = int(max(threads, min(p.output_bs, target_s / per_row)))
    t, ops, nr = run(nrows, seed + 1)
    return t, ops, nr, threads


def reference_arm(args, p, spec_desc):
    """The oracle as the reference arm: each step times a bounded sample of output rows."""
    import numpy as np
    import oracle
    from synth import sample_rows
    threads = oracle.default_threads()
    counts = np.bincount(p.row_index, minlength=p.output_bs)
    kw = {}
    if p.x1 is None:
        q, s = oracle.per_token_quant(p.x_bf16)
        kw = dict(x1=q, pertoken_scale=s)
    # size one step to about two seconds of host work
    rows = sample_rows(7, p.output_bs, max(2, threads // 2))
    t0 = time.perf_counter()
    oracle.problem_finalize(p, dest_rows=rows, want32=False, threads=threads, **kw)
    per_row = max((time.perf_counter() - t0) / rows.size, 1e-6)
    nrows = int(max(1, min(p.output_bs, 2.0 / per_row)))
    for w in range(args.warmup):
        oracle.problem_finalize(p, dest_rows=sample_rows(100 + w, p.output_bs, max(1, nrows // 8)), want32=False,
                                threads=threads, **kw)
    total_t, total_ops = 0.0, 0.0
    for s in range(args.steps):
        rows = sample_rows(1000 + s, p.output_bs, nrows)
        t0 = time.perf_counter()
        oracle.problem_finalize(p, dest_rows=rows, want32=False, threads=threads, **kw)
        total_t += time.perf_counter() - t0
        total_ops += 2.0 * float(counts[rows].sum()) * p.k * p.n
    unit, factor = line_unit(args.workload, p)
    value = factor * total_ops / total_t / 1e12
    sample = (f"{nrows} of {p.output_bs} output rows per step (every contributing source row in full), "
              f"{args.steps} steps")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": unit, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total_t / args.steps,
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "int8", "data": "synthetic",
        "config": {"workload": spec_desc, "mode": "deterministic order (oracle)"},
        "cpu_baseline": {"value": value, "unit": unit, "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- main
def time_ep(mode, world, rank, dist, steps, warmup, int8_peak):
    """The expert-parallel step of page "aclnnAlltoAllvQuantGroupedMatMul" on this
    rank's card: AlltoAllv (NCCL send/recv between ranks; device copies for a card's
    own chunks) with the permute folded in, the grouped matmul over the card's
    experts and the shared expert's matmul on a side stream.  Inputs resident on the
    device; per-card work fixed (weak scaling).  Returns a dict for the JSON line."""
    import numpy as np
    import torch
    from quantized_moe_grouped_persistent_b200 import finalize_launches
    from quantized_moe_grouped_persistent_b200.ep import EpGroupedMatmul
    from synth.ep import EP_BENCH, make_ep_problem
    cfg = dict(EP_BENCH)
    e = min(cfg.pop("e"), 256 // world)            # page 2: e * epWorldSize <= 256
    p = make_ep_problem(world=world, e=e, mode=mode, ranks=[rank], **cfg)
    c = p.cards[rank]
    m = EpGroupedMatmul(mode, world, rank, e, c.w, c.w_scale, c.mm_w, c.mm_w_scale)
    dev = m.device
    x = torch.from_numpy(c.x).to(dev)
    mm_x = torch.from_numpy(c.mm_x).to(dev)
    if mode == "mx":
        xs = torch.from_numpy(np.ascontiguousarray(c.x_scale)).to(dev)
        mms = torch.from_numpy(np.ascontiguousarray(c.mm_x_scale)).to(dev)
    else:
        xs, mms = c.x_scale, c.mm_x_scale
    stream = torch.cuda.current_stream()

    def step(events=None, check=False):
        return m.forward(x, xs, c.send_counts, c.recv_counts, mm_x, mms, check_counts=check, events=events)

    res = step(check=True)                          # first call: counts checked across ranks, workspaces
    torch.cuda.synchronize()
    a = int(res["permute_out"].shape[0])
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for b, en in ev:
        b.record(stream)
        en.record(stream)
    for _ in range(warmup):
        step(ev[0])
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    marks = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
    marks[0].record(stream)
    for s_ in range(steps):
        step(ev[s_])
        marks[s_ + 1].record(stream)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    ms = marks[0].elapsed_time(marks[-1]) / steps
    gemm_ms = sum(b.elapsed_time(en) for b, en in ev) / steps
    gmm_flops = 2.0 * a * p.h1 * p.n1
    mm_flops = 2.0 * p.tokens * p.h2 * p.n2
    flops = gmm_flops + mm_flops
    ms_max, gemm_max = max_over_ranks([ms, gemm_ms], dist, device="cuda")
    total = flops
    if dist is not None:
        t = torch.tensor([flops], dtype=torch.float64, device="cuda")
        dist.all_reduce(t)
        total = float(t.item())
    launches = (finalize_launches(m._problem(a, p.h1, p.n1, e))
                + finalize_launches(m._problem(p.tokens, p.h2, p.n2, 1)))
    achieved = gmm_flops / (gemm_ms * 1e-3) / 1e12
    quant = "E4M3 x E2M1 with E8M0 scales per 32" if mode == "mx" else "E4M3, per-tensor scales"
    return {
        "workload": (f"ep_{mode}: page 2's AlltoAllv + grouped matmul + shared-expert matmul, {world} card(s), "
                     f"e={e} experts per card, BS={p.tokens} tokens per card, topK={p.topk}, H1={p.h1}, N1={p.n1}, "
                     f"H2={p.h2}, N2={p.n2}; {quant}"),
        "value": total / (ms_max * 1e-3) / 1e12, "unit": "TFLOPS", "ms_per_step": ms_max,
        "gemm_ms": gemm_max, "rows_received_rank0": a, "flops_rank0": flops,
        "roofline": {"bound": "tensor", "kernel": "grouped GEMM over the card's experts", "achieved": achieved,
                     "peak": int8_peak, "unit": "TFLOPS", "frac": achieved / int8_peak, "traffic": None,
                     "kernel_ms": gemm_ms},
        "gpu_launches_per_step": launches,
    }


def ep_main(args, world, rank, local_rank):
    """``--workload ep_mx`` / ``ep_pertensor``: the expert-parallel step as the line."""
    mode = args.workload[len("ep_"):]
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps({"impl": "reference", "unavailable": "the expert-parallel workload has no timed CPU "
                              "leg; its oracle runs in the tests only"}), flush=True)
        return
    import torch
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as tdist
        torch.cuda.set_device(local_rank)
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
        dist = tdist
    else:
        torch.cuda.set_device(0)
    peaks = load_peaks()
    sampler = ClockSampler(torch.cuda.current_device())
    sampler.start()
    r = time_ep(mode, world, rank, dist, args.steps, args.warmup, 2.0 * peaks["bf16"])
    clocks = sampler.stop()
    if rank == 0:
        line = {"metric": "expert-parallel AlltoAllv + quantised grouped matmul + shared-expert matmul TFLOPS",
                "value": r["value"], "unit": "TFLOPS", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": r["ms_per_step"], "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "e4m3", "data": "synthetic",
                "config": {"workload": r["workload"], "l2": "inputs larger than L2, no flush",
                           "parallelism": f"expert parallel over {world} GPU(s)"},
                "roofline": r["roofline"], "gpu_launches": r["gpu_launches_per_step"] * args.steps,
                "clocks": clocks, "e2e": None}
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def main():
    args = parse_args()
    from synth import CONFIGS, make_problem

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.workload in ("ep_mx", "ep_pertensor"):
        return ep_main(args, world, rank, local_rank)
    spec = CONFIGS[args.workload]
    mode = "deterministic" if args.deterministic else "atomic"
    spec_desc = f"{args.workload}: {spec.description}; {mode} combine"

    if args.impl == "reference":
        if rank != 0:
            return
        p = make_problem(args.workload)
        reference_arm(args, p, spec_desc)
        return

    import torch
    from quantized_moe_grouped_persistent_b200 import finalize_launches, plan
    from quantized_moe_grouped_persistent_b200.device import DeviceProblem
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as tdist
        torch.cuda.set_device(local_rank)
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
        dist = tdist
    else:
        torch.cuda.set_device(0)
    dev_index = torch.cuda.current_device()

    p_full = make_problem(args.workload, tokens=args.tokens, e=args.experts)
    if args.transpose_x2:
        import numpy as np
        p_full.x2 = np.ascontiguousarray(np.swapaxes(p_full.x2, 1, 2))
        p_full.transpose_x2 = True
        spec_desc += "; weights stored (e, n, k)"
    if args.tokens or args.experts:
        spec_desc += f" (reduced: tokens={p_full.tokens}, e={p_full.e})"
    p, (c0, c1) = rank_problem(p_full, world, rank)
    d = DeviceProblem(p)
    ops = int_ops(p)
    peaks = load_peaks()
    # dense int8 = 2 x dense bf16 (nominal ratio).  The timed region is tens of ms,
    # so the burst figure (a cuBLAS GEMM timed alone) is the roofline denominator;
    # the sustained one (seconds under the power cap) is reported beside it.
    int8_peak = 2.0 * peaks["bf16"]
    int8_peak_sustained = 2.0 * peaks["bf16_sustained"]

    sampler = ClockSampler(dev_index)
    d.run(deterministic=args.deterministic)                # first call: module load, tensor maps
    torch.cuda.synchronize()
    flags = d.status(args.deterministic)
    sampler.start()
    per_step = {}
    ms, gemm_ms = time_steps(d, args.steps, args.warmup, args.deterministic, dist, per_step)
    clocks = sampler.stop()
    ms_max, gemm_max = max_over_ranks([ms, gemm_ms], dist, device="cuda")
    # the int8 tensor rate this device reaches with no memory traffic (CTA-pair
    # kind::i8 MMAs back to back), timed right after the op on the same GPU
    from quantized_moe_grouped_persistent_b200 import probe
    mma_probe = probe.mma_i8_rate()
    # decode is HBM-bound: its line reports algorithmic GB/s against the measured copy
    # bandwidth; the prefill-shaped workloads report int8 TOPS against the tensor peak
    unit, factor = line_unit(args.workload, p_full)
    hbm_line = unit == "GB/s"
    work = factor * ops / 1e12            # this rank's columns (the whole workload on one GPU)

    def rate(step_ms):
        return work / (step_ms * 1e-3)

    value = strong_scaling_value(factor * int_ops(p_full), ms_max)
    op_launches = finalize_launches(d.problem(args.deterministic))
    launches_per_step = op_launches + (1 if d.prologue else 0)
    sms = torch.cuda.get_device_properties(dev_index).multi_processor_count
    gemm_kernel = gemm_kernel_label(plan(d.problem(args.deterministic), sms), p.weight)

    extras = {}
    if not args.no_extras:
        # every rank copies its own inputs in and its own output columns out; the
        # whole job's rate is over the slowest rank
        e2e_ms, h2d, d2h = time_e2e(d, p, max(4, args.steps // 2), 2, args.deterministic)
        if dist is not None:
            dist.barrier()
        (e2e_max,) = max_over_ranks([e2e_ms], dist, device="cuda")
        extras["e2e"] = {"value": strong_scaling_value(factor * int_ops(p_full), e2e_max), "unit": unit,
                         "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_max,
                         "bytes_of_rank": rank}
    if world == 1 and not args.no_extras:
        if not args.deterministic:
            dms, dgemm = time_steps(d, max(3, args.steps // 2), 2, True)
            extras["deterministic"] = {"ms_per_step": dms, "value": rate(dms), "unit": unit, "gemm_ms": dgemm}
    del d
    torch.cuda.empty_cache()
    if world == 1 and not args.no_extras and args.workload != "decode":
        pd = make_problem("decode")
        dd = DeviceProblem(pd)
        dd.run()
        torch.cuda.synchronize()
        dms, dgemm = time_steps(dd, max(10, args.steps), 3, False)
        dbytes = algorithmic_bytes(pd)
        extras["decode"] = {
            "workload": "decode: " + CONFIGS["decode"].description + "; atomic combine",
            "value": dbytes / (dms * 1e-3) / 1e9, "unit": "GB/s", "ms_per_step": dms,
            "algorithmic_bytes": dbytes,
            "roofline": {"bound": "hbm", "achieved": dbytes / (dgemm * 1e-3) / 1e9, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": dbytes / (dgemm * 1e-3) / 1e9 / peaks["hbm_gbs"],
                         "traffic": committed_traffic("decode"), "kernel_ms": dgemm,
                         "peak_source": peaks["source"] + " copy bandwidth"},
            "pct_of_nominal_8tbs": 100.0 * dbytes / (dms * 1e-3) / 1e9 / NOMINAL_HBM_GBS,
        }
        del dd
        torch.cuda.empty_cache()
    if world == 1 and not args.no_extras and args.workload == "large_prefill":
        # the other prefill-shaped workloads, atomic combine, with their own int8 roofline
        for name in ("mid_prefill", "w4a8_prologue", "w4a8_mx"):
            ps = make_problem(name)
            ds = DeviceProblem(ps)
            ds.run()
            torch.cuda.synchronize()
            sms_, sgemm = time_steps(ds, max(10, args.steps), 3, False)
            sops = int_ops(ps)
            sunit, _ = line_unit(name, ps)
            extras[name] = {
                "workload": f"{name}: " + CONFIGS[name].description + "; atomic combine",
                "value": sops / (sms_ * 1e-3) / 1e12, "unit": sunit, "ms_per_step": sms_, "gemm_ms": sgemm,
                "roofline": {"bound": "tensor", "achieved": sops / (sgemm * 1e-3) / 1e12, "peak": int8_peak,
                             "unit": sunit, "frac": sops / (sgemm * 1e-3) / 1e12 / int8_peak,
                             "traffic": committed_traffic(name), "kernel_ms": sgemm},
            }
            del ds
            torch.cuda.empty_cache()
        extras["ep_mx"] = time_ep("mx", 1, 0, None, max(10, args.steps), 3, int8_peak)
        torch.cuda.empty_cache()

    cpu = None
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        t, sops, nr, threads = oracle_sample_time(p, args.cpu_seconds, 4242)
        cpu = {"value": factor * sops / t / 1e12, "unit": unit, "cores": threads, "kind": "oracle",
               "sample": f"{nr} of {p.output_bs} output rows of the same workload (every contributing source "
                         f"row in full, double-precision dequant/combine), {t:.1f} s"}

    if rank == 0:
        achieved = rate(gemm_max)
        if hbm_line:
            rates = {"pct_of_nominal_8tbs": 100.0 * value / world / NOMINAL_HBM_GBS}
            roofline = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                        "frac": achieved / peaks["hbm_gbs"], "traffic": committed_traffic(args.workload),
                        "kernel": gemm_kernel, "kernel_ms": gemm_max, "algorithmic_bytes": algorithmic_bytes(p),
                        "peak_source": peaks["source"] + " copy bandwidth"}
        else:
            rates = {"pct_of_dense_int8_peak": {"nominal_4500": 100.0 * value / world / NOMINAL_INT8_TOPS,
                                                "measured_burst": 100.0 * value / world / int8_peak,
                                                "measured_sustained": 100.0 * value / world / int8_peak_sustained}}
            roofline = {"bound": "tensor", "achieved": achieved, "peak": int8_peak, "unit": unit,
                        "frac": achieved / int8_peak, "traffic": committed_traffic(args.workload),
                        "kernel": gemm_kernel, "kernel_ms": gemm_max,
                        "frac_of_sustained": achieved / int8_peak_sustained,
                        "peak_source": f"{peaks['source']} bf16 burst x 2 (dense int8 : bf16 nominal ratio), "
                                       f"of measured",
                        "probe_int8_tops": mma_probe["tops"], "frac_of_probe": achieved / mma_probe["tops"],
                        "probe": dict(mma_probe, what="CTA-pair tcgen05.mma kind::i8 M=256 N=256 K=32 back to "
                                                      "back, no memory traffic, median of launches")}
        line = {
            "metric": METRIC, "value": value, "unit": unit, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_max,
            "step_ms": {"mean": ms_max, "median": per_step["ms_median"], "best": per_step["ms_best"],
                        "value_at_median": strong_scaling_value(factor * int_ops(p_full), per_step["ms_median"]),
                        "gemm_mean": gemm_max, "gemm_median": per_step["gemm_ms_median"],
                        "gemm_best": per_step["gemm_ms_best"], "of_rank": rank},
            "higher_is_better": True, "scaling": "strong",
            "vs_baseline": None, "dtype": "e4m3" if p.weight == "fp8" else "int8", "data": "synthetic",
            "config": {"workload": spec_desc, "tokens": p.tokens, "topk": p.topk, "m": p.m, "e": p.e, "k": p.k,
                       "n": p_full.n, "output_bs": p.output_bs, "mode": mode,
                       "l2": "inputs larger than L2 (x2 %.2f GB on rank 0), no flush" % (p.x2.nbytes / 1e9),
                       "parallelism": (f"column split over {world} GPUs: rank 0 owns columns [{c0}, {c1}) of "
                                       f"{p_full.n}; no data-path collective" if world > 1 else "1 GPU")},
            **rates,
            "roofline": roofline,
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clocks,
            "device_status": flags,
        }
        if cpu is not None:
            line["cpu_baseline"] = cpu
        line.update(extras)
        if "e2e" not in line:
            line["e2e"] = None
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
