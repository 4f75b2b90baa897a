"""Device-side failure detection, exercised without faulting the GPU.

Every wait inside the kernels is bounded; when one runs out, the kernel records
FA_ERR_TIMEOUT in a device status word and returns normally. Here a self-test kernel
waits on a barrier that nothing completes, with a short limit; the host must read the
timeout back, the read must clear it, and the context must still run attention.
"""

import math

import pytest

from exact_io_aware_69_b200 import fa
from exact_io_aware_69_b200.inputs import BF16, make_inputs

from helpers import to_device

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    import torch
    lib = fa.load()
    assert fa.device_status() == fa.FA_OK
    # ~10 ms at B200 clocks
    assert lib.fa_selftest_wait_timeout(20_000_000, fa._stream_handle(None)) == fa.FA_OK
    assert fa.device_status() == fa.FA_ERR_TIMEOUT
    assert fa.device_status() == fa.FA_OK  # reading cleared it
    inp = make_inputs(1, 1, 256, 64, BF16, seed=3)
    q, k, v = (to_device(getattr(inp, n), BF16) for n in ("q", "k", "v"))
    o, L, _ = fa.forward(q, k, v, causal=True, scale=1 / math.sqrt(64))
    torch.cuda.synchronize()
    assert fa.device_status() == fa.FA_OK
    assert torch.isfinite(o.float()).all() and torch.isfinite(L).all()
