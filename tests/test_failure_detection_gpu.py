"""Failure detection without a GPU fault (needs a B200): a device-side wait that nothing
completes gives up after its cycle limit, sets the library's device error word, the host
reads it as MAMBA_ERR_TIMEOUT, clearing works, and the context stays usable for the next
scan.  The wait is bounded (about a millisecond here); no trap, fault or endless loop."""
import pytest
import torch

from selective_state_space_56_b200 import inputs, ops

pytestmark = pytest.mark.gpu


def test_bounded_wait_timeout_is_reported_and_cleared(cuda_ok):
    ops.check_device_error(clear=True)
    ops.diag_wait_timeout(2_000_000)  # about 1 ms of SM clocks
    with pytest.raises(ops.MambaError) as e:
        ops.check_device_error(clear=False)
    assert e.value.status == -7
    with pytest.raises(ops.MambaError):  # still set: reading without clearing keeps it
        ops.check_device_error(clear=True)
    ops.check_device_error(clear=True)  # cleared by the previous read
    # the context is still usable
    p = inputs.scan_inputs(1, 16, 16, 64, torch.float32, seed=3, device="cuda")
    y = ops.selective_scan_fwd(p["u"], p["delta"], p["A"], p["B"], p["C"], D=p["D"], z=p["z"],
                               delta_bias=p["delta_bias"])
    torch.cuda.synchronize()
    assert torch.isfinite(y).all()
    ops.check_device_error(clear=True)
