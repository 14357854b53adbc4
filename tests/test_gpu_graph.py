"""qgmm_finalize inside a CUDA graph.

The call allocates nothing and never synchronises: it encodes tensor maps on the
host and launches kernels on the caller's stream.  So a serving loop can capture
it once and replay it, here on both the single-CTA path (16-row tiles) and the
CTA-pair path (256-row tiles plus the tail launch), in both combine modes.  Each
replay must match the oracle like an ordinary call.  One ordinary call runs
before capture, so the library's per-device setup is not captured.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

ATOMIC_TOL = 2e-5


@pytest.fixture(scope="module")
def dev(qgmm):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from quantized_moe_grouped_persistent_b200 import device
    return device


@pytest.mark.parametrize("hint", [0, 200])
@pytest.mark.parametrize("deterministic", [True, False])
def test_captured_call_replays_exactly(dev, oracle, problem_cache, hint, deterministic):
    p = problem_cache("mid_prefill", tokens=96, e=8, k=512, n=768)
    d = dev.DeviceProblem(p, expected_m_per_expert=hint)
    o64, sabs, o32 = oracle.problem_finalize(p)
    d.run(deterministic=deterministic)              # per-device setup outside the capture
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        with torch.cuda.graph(g, stream=side):
            d.run(deterministic=deterministic)
    torch.cuda.synchronize()
    for _ in range(3):
        d.out.fill_(float("nan"))                   # each replay rewrites the whole output
        g.replay()
        torch.cuda.synchronize()
        out = d.out.cpu().numpy()
        assert d.status(deterministic) == 0
        if deterministic:
            np.testing.assert_array_equal(out, o32)
        else:
            err = np.abs(out.astype(np.float64) - o64) / np.where(sabs > 0, sabs, 1.0)
            assert err.max() <= ATOMIC_TOL
    del g
