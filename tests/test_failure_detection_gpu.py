"""Failure detection on the GPU without a fault: a kernel waits on an on-chip barrier
that nothing completes.  The bounded wait every kernel of the library uses must give
up after about a second, record the timeout in the device status word, and leave
the context usable; the host reads the status and clears it."""
import time

import pytest
import torch

from exact_attention_108_b200 import binding
from gpu_common import gpu_inputs

pytestmark = pytest.mark.gpu


def test_bounded_wait_runs_out_and_is_reported():
    torch.cuda.synchronize()
    assert binding.device_status(clear=True) == binding.FATTN_OK
    t0 = time.perf_counter()
    binding.selftest_wait_timeout()
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert 0.5 <= elapsed <= 30.0, elapsed  # the wait limit is one second
    assert binding.device_status(clear=False) == binding.FATTN_ERR_DEVICE_TIMEOUT
    assert binding.device_status(clear=True) == binding.FATTN_ERR_DEVICE_TIMEOUT
    assert binding.device_status(clear=False) == binding.FATTN_OK
    # the context is still usable: an attention call runs and reports no timeout
    _, (q, k, v, _) = gpu_inputs(1, 1, 256, 64, 90, with_do=False)
    o, lse = binding.fwd(q, k, v, causal=True)
    torch.cuda.synchronize()
    assert binding.device_status(clear=True) == binding.FATTN_OK
    assert torch.isfinite(o.float()).all()
