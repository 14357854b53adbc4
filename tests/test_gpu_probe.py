"""The int8 tensor-rate probe (libqgmm_probe.so) on the device: its bounded wait
completes and the rate it reports is physically possible -- at most the tensor
pipe's 8192 int8 MACs per clock per SM at the clock the probe itself read, and
well above half of it (no memory traffic, no handshake in the issue loop)."""
import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu


def test_probe_rate_is_within_the_tensor_pipe(qgmm):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from quantized_moe_grouped_persistent_b200 import probe
    r = probe.mma_i8_rate(iters=4096, launches=5, warmup=1)
    assert 4096 < r["mac_per_clk_per_sm"] <= 8192 * 1.01, r
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert 0.5 < r["sm_ghz"] < 2.1, r
    assert r["tops"] <= 2 * 8192 * sms * 2.1e9 / 1e12, r
