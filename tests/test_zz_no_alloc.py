"""fa_bwd_noalloc: the backward for callers that cannot allocate device memory.

Some callers cannot allocate device memory where they run the backward -- a plugin
whose host application owns the device allocator, a service that must not allocate
in its steady state -- and so cannot hand fa_bwd its workspace. fa_bwd_noalloc runs
the same kernels on a scratch array built into the library instead. These tests call
it through the C ABI, twice in a row on the same inputs, and hold each result to
fa_bwd's with the tolerance the other GPU tests use; they also check that a problem
larger than the scratch array is refused before anything runs.

The file is named to be collected last, so that a run stopping at the first failure
has already run every other test.
"""

import pytest

from exact_io_aware_69_b200 import fa
from exact_io_aware_69_b200.inputs import BF16, FP16, make_inputs

from helpers import assert_close, to_device, to_f64

pytestmark = pytest.mark.gpu


def _noalloc(lib, q, k, v, o, o_res, do, L, dq, dk, dv, causal, scale):
    B, H, N, d = q.shape
    return lib.fa_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                              o_res.data_ptr(), do.data_ptr(), L.data_ptr(), dq.data_ptr(),
                              dk.data_ptr(), dv.data_ptr(), B, H, N, d, int(causal),
                              float(scale), fa._dtype_code(q), fa._stream_handle(None))


@pytest.mark.parametrize("dtype,causal,shape", [
    (BF16, True, (1, 2, 512, 128)),
    (FP16, False, (2, 2, 384, 64)),
])
def test_noalloc_matches_workspace_backward(dtype, causal, shape):
    import torch
    lib = fa.load()
    B, H, N, d = shape
    scale = d ** -0.5
    inp = make_inputs(B, H, N, d, dtype, seed=77)
    q, k, v, do = (to_device(getattr(inp, n), dtype) for n in ("q", "k", "v", "do"))
    o, L, o_res = fa.forward(q, k, v, causal=causal, scale=scale)
    want = fa.backward(q, k, v, o, L, do, causal=causal, scale=scale, o_res=o_res)
    torch.cuda.synchronize()
    for call in (1, 2):
        dq, dk, dv = (torch.full_like(q, float("nan")) for _ in range(3))
        rc = _noalloc(lib, q, k, v, o, o_res, do, L, dq, dk, dv, causal, scale)
        assert rc == fa.FA_OK, fa.status_string(rc)
        torch.cuda.synchronize()
        assert fa.device_status() == fa.FA_OK
        for name, got, ref in (("dq", dq, want[0]), ("dk", dk, want[1]), ("dv", dv, want[2])):
            assert_close(f"{name} (call {call})", to_f64(got), to_f64(ref), dtype)


def test_noalloc_refuses_problems_beyond_its_scratch():
    lib = fa.load()
    P = 0x7F0000000000  # never dereferenced: the size check comes first
    args = [P, P, P, P, None, P, P, P, P, P]
    # 64,640 rows at d = 128 need 33.6 MB of scratch, more than the 32 MiB array
    assert lib.fa_bwd_noalloc(*args, 1, 1, 64640, 128, 1, 0.088, fa.FA_BF16, None) == \
        fa.FA_ERR_UNSUPPORTED
    assert lib.fa_bwd_noalloc(*args, 2, 4, 16384, 64, 0, 0.125, fa.FA_BF16, None) == \
        fa.FA_ERR_UNSUPPORTED
    assert lib.fa_bwd_noalloc(*args, -1, 1, 128, 64, 0, 0.125, fa.FA_BF16, None) == \
        fa.FA_ERR_INVALID
