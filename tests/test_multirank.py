"""The multi-GPU plumbing of bench.py, run as two gloo ranks on the CPU.

Every rank takes the same collective steps; every rank draws the same seeded
workload and keeps its own block of output columns (strong scaling, no
data-path collective); the reported time is the max over ranks and the value
the whole workload's work over that time.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import datetime
    import torch.distributed as dist
    import bench
    from synth import make_problem
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        mine = [1.0 + rank, 10.0 - rank]                    # different per-rank timings
        got = bench.max_over_ranks(mine, dist, device="cpu")
        p, cols = bench.rank_problem(make_problem("tiny"), world, rank)
        dist.barrier()
        import hashlib
        out.put((rank, got, cols, hashlib.sha256(p.x1.tobytes()).hexdigest(),
                 hashlib.sha256(p.x2.tobytes()).hexdigest(), p.x2.shape))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_max_and_split_the_columns():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for pr in procs:
        pr.start()
    results = [q.get(timeout=120) for _ in range(world)]
    for pr in procs:
        pr.join(timeout=60)
        assert pr.exitcode == 0
    results.sort()
    for _, got, _, _, _, _ in results:
        assert got == [2.0, 10.0]                          # max over ranks, on every rank
    assert [r[2] for r in results] == [(0, 256), (256, 512)]   # tiny: n = 512, one tile each
    assert results[0][3] == results[1][3]                  # x1 (row side) replicated
    assert results[0][4] != results[1][4]                  # x2: each rank its own columns
    assert results[0][5] == results[1][5] == (4, 256, 256)


def test_strong_scaling_value_and_rank_problems():
    import bench
    from synth import make_problem
    assert bench.strong_scaling_value(8e12, 2.0) == pytest.approx(4000.0)
    assert bench.max_over_ranks([3.0, 1.5]) == [3.0, 1.5]  # single process: unchanged
    p = make_problem("mid_prefill", tokens=16, e=4, k=128, n=768)
    whole, cols = bench.rank_problem(p, 1, 0)
    assert whole is p and cols == (0, 768)
    blocks = [bench.rank_problem(p, 2, r) for r in range(2)]
    assert [c for _, c in blocks] == [(0, 512), (512, 768)]
    np.testing.assert_array_equal(np.concatenate([q.x2 for q, _ in blocks], axis=2), p.x2)
    assert sum(bench.int_ops(q) for q, _ in blocks) == bench.int_ops(p)
    with pytest.raises(SystemExit):
        bench.rank_problem(p, 4, 3)                        # 3 tiles, 4 GPUs: rank 3 would get nothing


def test_line_unit_decode_is_bytes_prefill_is_tops():
    """Decode lines report algorithmic GB/s: the factor takes the workload's int8
    ops to its algorithmic bytes; prefill-shaped lines stay in TOPS."""
    import bench
    from synth import make_problem
    p = make_problem("decode", tokens=4, e=8, k=128, n=256)
    unit, factor = bench.line_unit("decode", p)
    assert unit == "GB/s"
    assert factor * bench.int_ops(p) / 1e12 == pytest.approx(bench.algorithmic_bytes(p) / 1e9)
    assert bench.line_unit("mid_prefill", make_problem("mid_prefill", tokens=8, e=4, k=128, n=256)) == ("TOPS", 1.0)


def _run_bench(args, env_extra=None):
    import json
    import subprocess
    import sys
    env = dict(os.environ, **(env_extra or {}))
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True, text=True,
                       env=env, timeout=240, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    return [json.loads(l) for l in lines]


def test_reference_arm_line_contract():
    """bench.py --impl reference times the oracle and prints one line with the
    contract's keys; its cpu_baseline and e2e restate the line's own value."""
    (line,) = _run_bench(["--impl", "reference", "--workload", "tiny", "--steps", "2", "--warmup", "1"])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config"):
        assert key in line, key
    assert line["impl"] == "reference" and line["unit"] == "TOPS" and line["value"] > 0
    assert line["steps"] == 2 and line["warmup"] == 1 and line["higher_is_better"] is True
    assert line["config"]["workload"].startswith("tiny")
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["cores"] >= 1 and cb["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_print_nothing():
    assert _run_bench(["--impl", "reference", "--workload", "tiny", "--steps", "1", "--warmup", "0"],
                      {"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"}) == []


def test_gemm_kernel_label_follows_the_plan(monkeypatch):
    import bench
    import quantized_moe_grouped_persistent_b200 as q
    monkeypatch.delenv("QGMM_PAIR_TAILS", raising=False)
    label = lambda m, e, **kw: bench.gemm_kernel_label(q.plan(q.make_problem(m, 2048, 7168, e, max(1, m // 8), **kw),
                                                              148))
    assert label(131072, 256) == "grouped GEMM (grouped_gemm_pair_kernel + tail launch)"
    assert label(8192, 32) == "grouped_gemm_pair_kernel"                    # tails inside the pair launch
    assert label(128, 256) == "grouped_gemm_kernel"                         # decode: 16-row tiles
    assert label(32768, 128, weight_type=q.QGMM_W_INT4_PACKED_INT32) == "grouped_gemm_kernel"
