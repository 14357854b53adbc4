"""Expert-parallel AlltoAllv + grouped matmul + shared-expert matmul (page
"aclnnAlltoAllvQuantGroupedMatMul"), host side.

- The oracle's dispatch, pinned to a hand-worked two-card example (tests/golden):
  rows leave each card in (destination card, expert) order and land on the
  destination expert-major, then by source card.  A source-major permute, a
  dropped chunk or an off-by-one offset fails it.
- The oracle's two dequant modes on hand-worked rows: pertensor (acc * weight
  scale) * the row's source-card scale, and mx with one 32-block.
- ``qgmm_ep_plan`` (C ABI, a host call) against the same example, against a
  placement of every chunk compared with the oracle's dispatch over random counts
  (also property-based over drawn domains), and on its limits (page 2: e <= 32,
  e * epWorldSize <= 256, 0 < BSK < 52428800, no negative count).
- The exchange over gloo with 2 and 3 ranks (random counts, empty chunks, a card
  that receives nothing): every rank's permuted rows and scales equal the
  oracle's dispatch of all ranks' buffers, byte for byte; mismatched counts raise
  before any transfer.
"""
import json
import os
import socket
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
GOLDEN = json.load(open(os.path.join(ROOT, "tests", "golden", "ep_dispatch_example.json")))


def _col(rows):
    return np.array(rows, np.int64).reshape(-1, 1)


def test_oracle_dispatch_matches_the_hand_worked_example():
    from oracle import ep
    g = GOLDEN
    got = ep.dispatch([_col(r) for r in g["send_rows"]], [np.array(c) for c in g["send_counts"]], g["e"])
    for r in range(g["world"]):
        rows, counts = got[r]
        assert rows[:, 0].tolist() == g["permuted"][r]
        assert counts.tolist() == g["group_counts"][r]
    src = ep.source_cards([np.array(c) for c in g["send_counts"]], g["e"])
    assert src[0].tolist() == [0, 1, 1, 0, 0] and src[1].tolist() == [0, 1, 0, 1]


def test_oracle_dispatch_keeps_every_row_once():
    from oracle import ep
    rng = np.random.default_rng(5)
    world, e = 3, 4
    counts = [rng.integers(0, 4, world * e) for _ in range(world)]
    bufs = [_col(np.arange(int(c.sum())) + 1000 * s) for s, c in enumerate(counts)]
    got = ep.dispatch(bufs, counts, e)
    every = np.sort(np.concatenate([rows[:, 0] for rows, _ in got]))
    np.testing.assert_array_equal(every, np.sort(np.concatenate([b[:, 0] for b in bufs])))
    for r, (rows, gc) in enumerate(got):
        assert gc.tolist() == [sum(int(counts[s][r * e + j]) for s in range(world)) for j in range(e)]
        # inside one expert the source cards come in order, and a chunk keeps its order
        src = rows[:, 0] // 1000
        off = 0
        for j in range(e):
            seg = src[off:off + gc[j]]
            assert (np.diff(seg) >= 0).all()
            off += gc[j]


def _e4m3(v):
    from oracle import e4m3_encode
    return np.vectorize(e4m3_encode)(np.asarray(v, np.float32)).astype(np.uint8)


def test_oracle_pertensor_dequant_worked_example():
    from oracle import ep
    g = GOLDEN["pertensor_worked"]
    x = _e4m3(g["x_values"])
    w = _e4m3(g["w_values"])[None]
    out64, _, out32 = ep.grouped_matmul("pertensor", x, np.array(g["row_scale"], np.float32), [2], w,
                                        np.array([g["w_scale"]], np.float32), want32=True)
    np.testing.assert_array_equal(out64, np.array(g["y"]))
    np.testing.assert_array_equal(out32, np.array(g["y"], np.float32))


def test_oracle_mx_shared_matmul_worked_example():
    from oracle import ep
    x = np.full((1, 32), 0x38, np.uint8)
    sfa = np.array([[127]], np.uint8)
    w = np.full((256, 16), 0x11, np.uint8)           # 256 output columns, each 32 weights of 0.5
    sfb = np.full((256, 1), 128, np.uint8)
    out64, _, _ = ep.shared_matmul("mx", x, sfa, w, sfb)
    assert out64.shape == (1, 256)
    assert (out64 == GOLDEN["mx_worked"]["y"]).all()


def test_ep_plan_matches_the_hand_worked_example(qgmm):
    g = GOLDEN
    for r in range(g["world"]):
        plan = qgmm.ep_plan(g["world"], g["e"], g["send_counts"][r], g["recv_counts"][r])
        assert plan["send_offsets"].tolist() == g["send_offsets"][r]
        assert plan["recv_offsets"].tolist() == g["recv_offsets"][r]
        assert plan["group_counts"].tolist() == g["group_counts"][r]
        assert plan["bsk"] == g["bsk"][r] and plan["a"] == g["a"][r]


def test_ep_plan_places_every_chunk_where_the_oracle_does(qgmm):
    from oracle import ep
    rng = np.random.default_rng(11)
    for world, e in ((1, 1), (1, 32), (2, 3), (4, 8), (8, 32), (3, 5)):
        counts = [rng.integers(0, 5, world * e) for _ in range(world)]
        counts = [np.where(rng.random(world * e) < 0.3, 0, c) for c in counts]
        for c in counts:
            c[0] += 1                                  # BSK >= 1 on every card
        bufs = [_col(np.arange(int(c.sum())) + 10000 * s) for s, c in enumerate(counts)]
        want = ep.dispatch(bufs, counts, e)
        for r in range(world):
            recv = np.array([counts[s][r * e + j] for s in range(world) for j in range(e)])
            plan = qgmm.ep_plan(world, e, counts[r], recv)
            rows = np.full(int(recv.sum()), -1, np.int64)
            for s in range(world):               # place every chunk by the plan's offsets
                sp = qgmm.ep_plan(world, e, counts[s], np.array(
                    [counts[t][s * e + j] for t in range(world) for j in range(e)]))
                for j in range(e):
                    cnt = int(counts[s][r * e + j])
                    src = bufs[s][int(sp["send_offsets"][r * e + j]):int(sp["send_offsets"][r * e + j]) + cnt, 0]
                    ro = int(plan["recv_offsets"][s * e + j])
                    rows[ro:ro + cnt] = src
            np.testing.assert_array_equal(rows, want[r][0][:, 0])
            np.testing.assert_array_equal(plan["group_counts"], want[r][1])


def test_ep_plan_limits(qgmm):
    ok = [1] * 4
    assert qgmm.ep_plan(2, 2, ok, ok)["a"] == 4
    bad = [
        (0, 1, [], []),                              # no card
        (1, 0, [], []),                              # no expert
        (1, 33, [1] * 33, [1] * 33),                 # e > 32
        (9, 32, [1] * 288, [1] * 288),               # e * world > 256
        (2, 2, [0, 0, 0, 0], ok),                    # BSK = 0
        (2, 2, [1, -1, 1, 1], ok),                   # a negative count
        (2, 2, ok, [1, 1, -1, 1]),
        (1, 1, [52428800], [1]),                     # BSK at the page's bound
    ]
    for world, e, sc, rc in bad:
        with pytest.raises(qgmm.QgmmError) as ei:
            qgmm.ep_plan(world, e, sc, rc)
        assert ei.value.code == qgmm.QGMM_ERR_SHAPE, (world, e)
    assert qgmm.ep_plan(1, 1, [52428799], [0])["bsk"] == 52428799
    assert qgmm.ep_plan(8, 32, [1] * 256, [0] * 256)["a"] == 0     # a card may receive nothing


def test_ep_plan_null_pointers(qgmm):
    import ctypes as C
    a = (C.c_int64 * 4)(1, 1, 1, 1)
    o = (C.c_int64 * 4)()
    assert qgmm.lib().qgmm_ep_plan(2, 2, None, a, o, o, o, o) == qgmm.QGMM_ERR_NULL_PTR
    assert qgmm.lib().qgmm_ep_plan(2, 2, a, a, o, o, o, None) == qgmm.QGMM_ERR_NULL_PTR


def test_ep_permute_rows_host_checks(qgmm):
    import ctypes as C
    L = qgmm.lib()
    t = (C.c_int64 * 2)(0, 4)
    z = (C.c_int64 * 2)(0, 0)
    neg = (C.c_int64 * 2)(-1, 0)
    assert L.qgmm_ep_permute_rows(None, None, 16, 2, t, t, z, None) == qgmm.QGMM_OK     # nothing to move
    assert L.qgmm_ep_permute_rows(None, None, 16, 2, None, t, z, None) == qgmm.QGMM_ERR_NULL_PTR
    assert L.qgmm_ep_permute_rows(None, None, 16, 33, t, t, z, None) == qgmm.QGMM_ERR_SHAPE
    assert L.qgmm_ep_permute_rows(None, None, 6, 2, t, t, z, None) == qgmm.QGMM_ERR_SHAPE     # row_bytes % 4
    assert L.qgmm_ep_permute_rows(None, None, 16, 2, t, t, neg, None) == qgmm.QGMM_ERR_SHAPE
    assert L.qgmm_ep_permute_rows(None, None, 16, 2, t, t, t, None) == qgmm.QGMM_ERR_NULL_PTR  # rows, no buffers


# ---------------------------------------------------------------- gloo exchange
def _cpu_local(src, dst, src_rows, dst_rows, counts):
    """The card's own chunks on CPU tensors (the library's copy kernel takes device tensors)."""
    for a, b, n in zip(src_rows, dst_rows, counts):
        dst[int(b):int(b) + int(n)] = src[int(a):int(a) + int(n)]


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _counts_for(world, e, seed):
    rng = np.random.default_rng(seed)
    counts = [rng.integers(0, 6, world * e) for _ in range(world)]
    counts = [np.where(rng.random(world * e) < 0.35, 0, c) for c in counts]
    for c in counts:
        c[0] += 1
    if world >= 3:                                   # card 1 receives nothing
        for s in range(world):
            counts[s][1 * e:2 * e] = 0
    return counts


def _exchange_main(rank, world, e, seed, port, out, mode):
    sys.path.insert(0, ROOT)
    import datetime
    import torch
    import torch.distributed as dist
    from quantized_moe_grouped_persistent_b200 import ep_plan
    from quantized_moe_grouped_persistent_b200.ep import Exchange
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        counts = _counts_for(world, e, seed)
        send = counts[rank]
        recv = np.array([counts[s][rank * e + j] for s in range(world) for j in range(e)], np.int64)
        if mode == "mismatch" and rank == 0:
            recv = recv.copy()
            recv[-1] += 1
        bsk = int(send.sum())
        rng = np.random.default_rng(seed + 1 + rank)
        x = torch.from_numpy(rng.integers(0, 256, (bsk, 64), dtype=np.uint8))
        sf = torch.from_numpy(rng.integers(100, 140, (bsk, 2), dtype=np.uint8))
        ex = Exchange(world, rank, e, local=_cpu_local)
        try:
            ex.check_counts(send, recv, "cpu")
        except Exception as err:                      # every rank sees the same gathered counts
            out.put((rank, "raised", str(err)))
            return
        plan = ep_plan(world, e, send, recv)
        px = torch.empty((plan["a"], 64), dtype=torch.uint8)
        psf = torch.empty((plan["a"], 2), dtype=torch.uint8)
        ex.run([(x, px), (sf, psf)], plan, send, recv)
        out.put((rank, x.numpy(), sf.numpy(), px.numpy(), psf.numpy(), plan["group_counts"]))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _run_ranks(world, e, seed, mode="ok"):
    import torch.multiprocessing as mp
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_exchange_main, args=(r, world, e, seed, port, q, mode)) for r in range(world)]
    for pr in procs:
        pr.start()
    res = sorted([q.get(timeout=180) for _ in range(world)], key=lambda t: t[0])
    for pr in procs:
        pr.join(timeout=60)
        assert pr.exitcode == 0
    return res


@pytest.mark.parametrize("world,e,seed", [(2, 3, 21), (3, 4, 22)])
def test_gloo_exchange_lands_every_chunk_in_its_permuted_place(world, e, seed):
    from oracle import ep
    res = _run_ranks(world, e, seed)
    counts = _counts_for(world, e, seed)
    xs = ep.dispatch([r[1] for r in res], counts, e)
    sfs = ep.dispatch([r[2] for r in res], counts, e)
    for r in range(world):
        np.testing.assert_array_equal(res[r][3], xs[r][0])
        np.testing.assert_array_equal(res[r][4], sfs[r][0])
        np.testing.assert_array_equal(res[r][5], xs[r][1])
    if world >= 3:
        assert res[1][3].shape[0] == 0


def test_gloo_exchange_rejects_mismatched_counts():
    res = _run_ranks(2, 2, 23, mode="mismatch")
    assert all(r[1] == "raised" for r in res)
    assert all("expects other counts" in r[2] for r in res)


def test_ep_plan_against_the_oracle_over_drawn_domains(qgmm):
    """Hypothesis: drawn domains (1-8 cards, 1-32 experts per card, at most 256 in all,
    chunk counts 0-6 with empty cards allowed on the receive side): every card's plan
    places each chunk where the oracle's dispatch puts its rows."""
    hyp = pytest.importorskip("hypothesis")
    st = pytest.importorskip("hypothesis.strategies")
    from oracle import ep

    @hyp.settings(max_examples=60, deadline=None, derandomize=True)
    @hyp.given(st.integers(1, 8), st.integers(1, 32), st.integers(0, 2 ** 31 - 1))
    def check(world, e, seed):
        hyp.assume(world * e <= 256)
        rng = np.random.default_rng(seed)
        counts = [rng.integers(0, 7, world * e) for _ in range(world)]
        for c in counts:
            c[rng.integers(0, world * e)] += 1                 # BSK >= 1 on every card
        bufs = [_col(np.arange(int(c.sum())) + 100000 * s) for s, c in enumerate(counts)]
        want = ep.dispatch(bufs, counts, e)
        plans = [qgmm.ep_plan(world, e, counts[r],
                              np.array([counts[s][r * e + j] for s in range(world) for j in range(e)]))
                 for r in range(world)]
        for r in range(world):
            rows = np.full(plans[r]["a"], -1, np.int64)
            for s in range(world):
                for j in range(e):
                    cnt = int(counts[s][r * e + j])
                    so = int(plans[s]["send_offsets"][r * e + j])
                    ro = int(plans[r]["recv_offsets"][s * e + j])
                    rows[ro:ro + cnt] = bufs[s][so:so + cnt, 0]
            np.testing.assert_array_equal(rows, want[r][0][:, 0])
            np.testing.assert_array_equal(plans[r]["group_counts"], want[r][1])
            assert plans[r]["bsk"] == int(counts[r].sum())

    check()
