"""The pipe-throughput probe (needs a B200) that backs the SFU roofline's derived peak.

The scan's roofline is stated against 148 SMs x 16 SFU results per clock x the maximum
SM clock.  The probe measures that rate directly (8 independent ex2.approx chains per
thread, 64 warps per SM), and the fp32 FMA rate beside it; the measured rates must lie
between half the derived figure and 10% above it (a rate far above would mean the
derived peak understates the hardware and every SFU fraction reported overstates the
kernels).  The packed fp32x2 FMA is only required to be positive and at most twice the
scalar FMA's derived rate, since whether pairing doubles fp32 throughput is what the
probe reports.
"""
import json
import os

import pytest
import torch

from selective_state_space_56_b200 import ops

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _max_sm_mhz():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f).get("sm_max_mhz", 1965.0))
    except (OSError, ValueError):
        return 1965.0


def _rate(kind, blocks, iters, sink):
    ops.diag_throughput(kind, blocks, 64, sink)
    best = float("inf")
    for _ in range(3):
        a, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        n = ops.diag_throughput(kind, blocks, iters, sink)
        e.record()
        e.synchronize()
        best = min(best, a.elapsed_time(e))
    assert torch.isfinite(sink).all()
    return n / (best * 1e-3)


def test_measured_pipe_rates_match_the_derived_peaks(cuda_ok):
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    mhz = _max_sm_mhz()
    blocks = sms * 8
    sink = torch.empty(blocks * 256, dtype=torch.float32, device="cuda")
    sfu = _rate("sfu_ex2", blocks, 4096, sink)
    ffma = _rate("ffma", blocks, 32768, sink)
    ffma2 = _rate("ffma2", blocks, 16384, sink)
    ops.check_device_error()
    sfu_derived = sms * 16 * mhz * 1e6
    fma_derived = sms * 128 * mhz * 1e6
    assert 0.5 * sfu_derived <= sfu <= 1.1 * sfu_derived, (sfu, sfu_derived)
    assert 0.5 * fma_derived <= ffma <= 1.1 * fma_derived, (ffma, fma_derived)
    assert 0.0 < ffma2 <= 2.2 * fma_derived, (ffma2, fma_derived)


def test_probe_writes_one_finite_value_per_thread(cuda_ok):
    sink = torch.full((2 * 256 + 7,), float("nan"), dtype=torch.float32, device="cuda")
    for kind in ops.THROUGHPUT_KINDS:
        sink.fill_(float("nan"))
        n = ops.diag_throughput(kind, 2, 3, sink)
        torch.cuda.synchronize()
        assert n == 2 * 256 * 3 * (16 if kind == "ffma2" else 8)
        assert torch.isfinite(sink[:512]).all(), kind
        assert torch.isnan(sink[512:]).all(), kind  # nothing past blocks * 256
    with pytest.raises(ValueError):
        ops.diag_throughput("ffma", 4, 3, sink)  # sink too small for 4 blocks
