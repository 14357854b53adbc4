"""GPU parity of the expert-parallel AlltoAllv + grouped matmul + shared-expert matmul
(page "aclnnAlltoAllvQuantGroupedMatMul") against the oracle.

- One card (epWorldSize 1): the whole call through ``EpGroupedMatmul.forward`` -- the
  dispatch (every chunk a device copy to its permuted place), the grouped matmul
  over the card's experts and the shared expert's matmul on the side stream.  The
  permuted rows and scales equal the oracle's byte for byte; the outputs are
  within the f32 bound of the E4M3 / MxA8W4 modes, 2 (k/32) 2^-24 of the sum of
  |scaled products|, plus 1e-5 of it for the f32 dequant.
- Several cards on one GPU, one after the other: each card's grouped matmul and
  shared-expert matmul run on the GPU over the permuted rows the oracle's dispatch
  gives that card (the exchange between processes is covered by the gloo tests).
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu


def acc_tol(k: int) -> float:
    return 2.0 * (k / 32) * 2.0 ** -24 + 1e-5


@pytest.fixture(scope="module")
def ep_mod(qgmm):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from quantized_moe_grouped_persistent_b200 import ep
    return ep


def _close(got, ref, k, what):
    out64, sabs, _ = ref
    err = np.abs(got.astype(np.float64) - out64) / np.where(sabs > 0, sabs, 1.0)
    assert err.max() <= acc_tol(k), (what, err.max(), acc_tol(k))


def _card(ep_mod, p, c):
    return ep_mod.EpGroupedMatmul(p.mode, p.world, c.rank, p.e, c.w, c.w_scale, c.mm_w, c.mm_w_scale)


@pytest.mark.parametrize("mode", ["pertensor", "mx"])
@pytest.mark.parametrize("shape", [dict(e=4, tokens=96, topk=2, h1=256, n1=512, h2=256, n2=256),
                                   dict(e=8, tokens=300, topk=4, h1=512, n1=768, h2=384, n2=512)])
def test_one_card_forward_matches_oracle(ep_mod, oracle, mode, shape):
    from oracle import ep as oep
    from synth.ep import make_ep_problem
    p = make_ep_problem(world=1, mode=mode, seed={"pertensor": 700, "mx": 750}[mode] + shape["e"], **shape)
    c = p.cards[0]
    ref = oep.reference(p)[0]
    m = _card(ep_mod, p, c)
    res = m.forward(c.x, c.x_scale, c.send_counts, c.recv_counts, c.mm_x, c.mm_x_scale)
    np.testing.assert_array_equal(res["permute_out"].cpu().numpy(), ref["permute_out"])
    np.testing.assert_array_equal(res["permute_scale"].cpu().numpy(), ref["permute_scale"])
    np.testing.assert_array_equal(res["group_counts"], ref["group_counts"])
    _close(res["gmm_y"].cpu().numpy(), ref["gmm"], p.h1, "gmm")
    _close(res["mm_y"].cpu().numpy(), ref["mm"], p.h2, "mm")
    from quantized_moe_grouped_persistent_b200 import device_status
    assert device_status(m._ws["gmm"]) == 0 and device_status(m._ws["mm"]) == 0


@pytest.mark.parametrize("mode", ["pertensor", "mx"])
@pytest.mark.parametrize("world,e", [(2, 4), (4, 8)])
def test_each_card_of_a_domain_matches_oracle(ep_mod, oracle, mode, world, e):
    from oracle import ep as oep
    from synth.ep import make_ep_problem
    p = make_ep_problem(world=world, e=e, tokens=128, topk=4, h1=256, n1=256, h2=256, n2=256, mode=mode,
                        routing="zipf", routing_param=1.0, seed=800 + world + e)
    refs = oep.reference(p)
    for c, ref in zip(p.cards, refs):
        m = _card(ep_mod, p, c)
        if ref["permute_out"].shape[0] > 0:
            x = torch.from_numpy(ref["permute_out"]).cuda()
            s = torch.from_numpy(np.ascontiguousarray(ref["permute_scale"])).cuda()
            gmm_y = m.grouped(x, s, ref["group_counts"])
            _close(gmm_y.cpu().numpy(), ref["gmm"], p.h1, f"gmm card {c.rank}")
        mm_y = m.shared(c.mm_x, c.mm_x_scale)
        m.join()
        _close(mm_y.cpu().numpy(), ref["mm"], p.h2, f"mm card {c.rank}")


def test_grouped_matmul_with_no_rows_launches_nothing(ep_mod):
    from synth.ep import make_ep_problem
    p = make_ep_problem(world=1, e=2, tokens=16, topk=1, h1=256, n1=256, mode="mx", seed=901)
    c = p.cards[0]
    m = _card(ep_mod, p, c)
    out, sc, plan = m.dispatch(c.x, c.x_scale, c.send_counts, c.recv_counts)
    assert out.shape[0] == plan["a"] == int(c.recv_counts.sum())
    assert m.grouped(out[:0], sc[:0], np.zeros(p.e, np.int64)) is None


@pytest.mark.parametrize("row_bytes", [7168, 224, 12, 4])
def test_permute_rows_kernel(ep_mod, row_bytes):
    from quantized_moe_grouped_persistent_b200 import ep_permute_rows
    rng = np.random.default_rng(row_bytes)
    counts = rng.integers(0, 40, 32)
    counts[3] = 0
    total = int(counts.sum())
    src_rows = np.concatenate([[0], np.cumsum(counts)[:-1]])
    order = rng.permutation(32)                         # destination order of the chunks
    dst_rows = np.zeros(32, np.int64)
    dst_rows[order] = np.concatenate([[0], np.cumsum(counts[order])[:-1]])
    src = rng.integers(0, 256, (total, row_bytes), dtype=np.uint8)
    want = np.zeros_like(src)
    for a, b, n in zip(src_rows, dst_rows, counts):
        want[b:b + n] = src[a:a + n]
    dsrc = torch.from_numpy(src).cuda()
    ddst = torch.zeros_like(dsrc)
    ep_permute_rows(dsrc, ddst, src_rows, dst_rows, counts)
    np.testing.assert_array_equal(ddst.cpu().numpy(), want)
