"""Bounded device waits: a wait that nothing completes gives up, records
QLORA_ERR_TIMEOUT in the device status word, and leaves the context usable."""
import pytest
import torch

pytestmark = pytest.mark.gpu

q4 = pytest.importorskip("parameter_efficient_fine_nf4_b200")


def test_bounded_wait_reports_timeout_and_context_survives():
    assert q4.qlora_get_device_status() == 0
    q4.qlora_selftest_wait_timeout(20000)          # 20 ms limit on a barrier nobody completes
    assert q4.qlora_get_device_status() == q4.QLORA_ERR_TIMEOUT
    assert q4.qlora_get_device_status() == 0      # reading clears it
    # the context still works: a normal call succeeds afterwards
    W = torch.randn(64, 128, device="cuda", dtype=torch.float32)
    qw = q4.qlora_nf4_quantize(W)
    Wd = q4.qlora_nf4_dequantize(qw)
    torch.cuda.synchronize()
    assert torch.isfinite(Wd.float()).all()
    assert q4.qlora_get_device_status() == 0


def test_launch_counter_and_profiler():
    n0 = q4.qlora_launch_count()
    q4.qlora_profile_begin()
    W = torch.randn(128, 256, device="cuda", dtype=torch.float32)
    qw = q4.qlora_nf4_quantize(W)
    q4.qlora_nf4_dequantize(qw)
    stats = q4.qlora_profile_end()
    assert q4.qlora_launch_count() - n0 == 3
    names = {s["name"] for s in stats}
    assert {"nf4_quantize_phase1", "nf4_quantize_dq", "nf4_dequantize"} <= names
    assert all(s["total_ms"] > 0 for s in stats)
