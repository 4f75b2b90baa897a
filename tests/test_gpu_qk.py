"""Different query and key lengths (fa_fwd_qk / fa_bwd_qk through the binding) vs the
fp64 oracle, element by element.

Causal masking is bottom-right aligned: query i sees keys j <= i + Nk - Nq. The shapes
cover one query against many keys, more queries than keys (the first Nq - Nk queries
see no key: O = 0, L = -inf, dQ = 0), fewer queries than keys, and lengths that are
not multiples of 128 on either side.
"""

import math

import numpy as np
import pytest

import oracle
from exact_io_aware_69_b200 import fa
from exact_io_aware_69_b200.inputs import BF16, FP16, make_inputs

from helpers import TOL_L, assert_close, to_device, to_f64

pytestmark = pytest.mark.gpu

SHAPES = [  # (B, H, Nq, Nk, d)
    (1, 2, 1, 300, 64),
    (2, 1, 200, 77, 128),
    (1, 2, 128, 384, 128),
    (1, 1, 333, 256, 64),
    (1, 1, 77, 600, 128),
    (1, 2, 640, 256, 128),
]


def _inputs(B, H, Nq, Nk, d, dtype, seed):
    a = make_inputs(B, H, Nq, d, dtype, seed)       # q and dO
    b = make_inputs(B, H, Nk, d, dtype, seed + 1)   # k and v
    return a, b


def _check_L(got, ref):
    """L = -inf exactly on the rows that see no key; elsewhere within TOL_L."""
    got = np.asarray(got, np.float64)
    empty = np.isneginf(ref)
    assert np.array_equal(np.isneginf(got), empty), "L: -inf rows differ"
    assert np.all(np.isfinite(got[~empty])), "L: non-finite values"
    if (~empty).any():
        mx = float(np.max(np.abs(got[~empty] - ref[~empty])))
        assert mx <= TOL_L, f"L: max-abs {mx:.3e} (tol {TOL_L:.0e})"


@pytest.mark.parametrize("dtype", [BF16, FP16])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "B{}H{}Nq{}Nk{}d{}".format(*s))
def test_qk_fwd_bwd_vs_oracle(shape, causal, dtype):
    import torch
    B, H, Nq, Nk, d = shape
    if dtype == FP16 and shape not in (SHAPES[1], SHAPES[3]):
        pytest.skip("fp16 on two shapes only (the arithmetic is the same)")
    scale = 1.0 / math.sqrt(d)
    a, b = _inputs(B, H, Nq, Nk, d, dtype, seed=1000 + Nq * 7 + Nk)
    q, do = to_device(a.q, dtype), to_device(a.do, dtype)
    k, v = to_device(b.k, dtype), to_device(b.v, dtype)
    o, L, o_res = fa.forward(q, k, v, causal=causal, scale=scale)
    dq, dk, dv = fa.backward(q, k, v, o, L, do, causal=causal, scale=scale, o_res=o_res)
    torch.cuda.synchronize()
    assert fa.device_status() == fa.FA_OK
    ref = oracle.attn_bwd(a.widened("q"), b.widened("k"), b.widened("v"), a.widened("do"),
                          causal, scale)
    _check_L(to_f64(L), ref["L"])
    for name, got in (("o", o), ("dq", dq), ("dk", dk), ("dv", dv)):
        assert_close(name, to_f64(got), ref[name], dtype)
    if causal and Nq > Nk:  # rows that see no key: exactly zero
        e = Nq - Nk
        assert torch.count_nonzero(o[:, :, :e]).item() == 0
        assert torch.count_nonzero(dq[:, :, :e]).item() == 0


def test_qk_square_matches_fa_fwd():
    """Nq = Nk through fa_fwd_qk is the same computation as fa_fwd."""
    import torch
    lib = fa.load()
    a = make_inputs(1, 2, 384, 128, BF16, seed=3)
    q, k, v = (to_device(getattr(a, n), BF16) for n in ("q", "k", "v"))
    o1, L1, r1 = fa.forward(q, k, v, causal=True)
    o2, L2 = torch.empty_like(q), torch.empty_like(L1)
    rc = lib.fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o2.data_ptr(), None, L2.data_ptr(),
                    1, 2, 384, 128, 1, 128 ** -0.5, fa.FA_BF16, fa._stream_handle(None))
    assert rc == fa.FA_OK
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(L1, L2)
