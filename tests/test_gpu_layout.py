"""[B, N, H, d] tensors (FA_LAYOUT_BNHD) through fa_fwd_ex / fa_bwd_ex.

The same inputs in the two layouts must give the same results: O, L, dK and dV bit for
bit (the same arithmetic in the same order), dQ within the parity bar (its partial
sums are added in no fixed order), and both against the fp64 oracle.
"""

import math

import pytest

import oracle
from exact_io_aware_69_b200 import fa
from exact_io_aware_69_b200.inputs import BF16, FP16, make_inputs

from helpers import assert_close, assert_close_L, to_device, to_f64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", [BF16, FP16])
@pytest.mark.parametrize("B,H,Nq,Nk,d,window", [
    (2, 3, 384, 384, 128, (-1, 0)),
    (1, 4, 333, 333, 64, (-1, -1)),
    (2, 2, 200, 520, 128, (100, 20)),
])
def test_bnhd_matches_bhnd_and_oracle(B, H, Nq, Nk, d, window, dtype):
    import torch
    scale = 1.0 / math.sqrt(d)
    a = make_inputs(B, H, Nq, d, dtype, seed=60 + Nq)
    b = make_inputs(B, H, Nk, d, dtype, seed=61 + Nq)
    q, do = to_device(a.q, dtype), to_device(a.do, dtype)
    k, v = to_device(b.k, dtype), to_device(b.v, dtype)

    def bnhd(t):
        return t.transpose(1, 2).contiguous()

    o1, L1, r1 = fa.forward(q, k, v, scale=scale, window=window)
    g1 = fa.backward(q, k, v, o1, L1, do, scale=scale, o_res=r1, window=window)
    q2, k2, v2, do2 = bnhd(q), bnhd(k), bnhd(v), bnhd(do)
    o2, L2, r2 = fa.forward(q2, k2, v2, scale=scale, window=window, layout="bnhd")
    g2 = fa.backward(q2, k2, v2, o2, L2, do2, scale=scale, o_res=r2, window=window,
                     layout="bnhd")
    torch.cuda.synchronize()
    assert fa.device_status() == fa.FA_OK
    assert o2.shape == (B, Nq, H, d) and L2.shape == (B, H, Nq)
    assert torch.equal(bnhd(o1), o2) and torch.equal(L1, L2) and torch.equal(bnhd(r1), r2)
    assert torch.equal(bnhd(g1[1]), g2[1]) and torch.equal(bnhd(g1[2]), g2[2])
    ref = oracle.attn_window(a.widened("q"), b.widened("k"), b.widened("v"), a.widened("do"),
                             window, scale)
    assert_close_L(to_f64(L2), ref["L"])
    for name, t in (("o", o2), ("dq", g2[0]), ("dk", g2[1]), ("dv", g2[2])):
        assert_close(name, to_f64(t.transpose(1, 2)), ref[name], dtype)
