"""The device watchdog: a bounded wait that can never complete gives up after its
time limit, records E4B_ERR_TIMEOUT in the status word (read and cleared by
e4b_device_status), and leaves the context usable.  Nothing faults or hangs."""
import time

import pytest
import torch

pytestmark = pytest.mark.gpu


def test_watchdog_times_out_and_context_stays_usable():
    import bit_quantized_mixture_nf4_b200 as e4b
    assert e4b.e4b_device_status() == e4b.E4B_OK
    t0 = time.perf_counter()
    e4b.e4b_watchdog_selftest()
    st = e4b.e4b_device_status()          # synchronizes, reads and clears the word
    elapsed = time.perf_counter() - t0
    assert st == e4b.E4B_ERR_TIMEOUT
    assert 1.5 <= elapsed <= 30.0          # the wait's limit is 2 s
    assert e4b.e4b_device_status() == e4b.E4B_OK   # cleared
    # the context still runs the library's kernels
    w = torch.randn(2, 64, 128, device="cuda") * 0.02
    packed, absmax = e4b.e4b_quantize_nf4(w)
    out = e4b.e4b_dequantize_nf4(packed, absmax, w.shape)
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all()
    assert e4b.e4b_device_status() == e4b.E4B_OK
