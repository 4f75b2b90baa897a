"""Sliding-window (key band) attention through fa_fwd_ex / fa_bwd_ex vs the fp64 oracle.

Query i sees keys j with i + Nk - Nq - left <= j <= i + Nk - Nq + right (negative =
unbounded). The cases cover one-key and one-tile bands, bands that end exactly on a
tile edge (127, 128), wide bands, one-sided bands, square / ragged / Nq != Nk shapes,
key tiles that no query sees (dK = dV = 0 there) and query rows that see no key
(O = 0, L = -inf).
"""

import math

import numpy as np
import pytest

import oracle
from exact_io_aware_69_b200 import fa
from exact_io_aware_69_b200.inputs import BF16, FP16, make_inputs

from helpers import TOL_L, assert_close, to_device, to_f64

pytestmark = pytest.mark.gpu


def _check_L(got, ref):
    got = np.asarray(got, np.float64)
    empty = np.isneginf(ref)
    assert np.array_equal(np.isneginf(got), empty), "L: -inf rows differ"
    assert np.all(np.isfinite(got[~empty])), "L: non-finite values"
    if (~empty).any():
        mx = float(np.max(np.abs(got[~empty] - ref[~empty])))
        assert mx <= TOL_L, f"L: max-abs {mx:.3e} (tol {TOL_L:.0e})"


def _run(B, H, Nq, Nk, d, dtype, window, seed):
    import torch
    scale = 1.0 / math.sqrt(d)
    a = make_inputs(B, H, Nq, d, dtype, seed)        # q and dO
    b = make_inputs(B, H, Nk, d, dtype, seed + 1)    # k and v
    q, do = to_device(a.q, dtype), to_device(a.do, dtype)
    k, v = to_device(b.k, dtype), to_device(b.v, dtype)
    o, L, o_res = fa.forward(q, k, v, scale=scale, window=window)
    dq, dk, dv = fa.backward(q, k, v, o, L, do, scale=scale, o_res=o_res, window=window)
    torch.cuda.synchronize()
    assert fa.device_status() == fa.FA_OK
    ref = oracle.attn_window(a.widened("q"), b.widened("k"), b.widened("v"), a.widened("do"),
                             window, scale)
    got = {"o": o, "L": L, "dq": dq, "dk": dk, "dv": dv}
    return {n: to_f64(t) for n, t in got.items()}, ref


CASES = [  # (B, H, Nq, Nk, d, (left, right))
    (1, 2, 512, 512, 64, (0, 0)),
    (1, 2, 512, 512, 128, (1, 1)),
    (1, 1, 640, 640, 128, (127, 0)),
    (1, 1, 640, 640, 64, (128, 0)),
    (2, 1, 768, 768, 128, (300, 5)),
    (1, 2, 700, 700, 64, (128, 128)),
    (1, 1, 1000, 1000, 128, (-1, 128)),
    (1, 1, 1000, 1000, 64, (300, -1)),
    (1, 2, 333, 333, 128, (1, 127)),
    (1, 1, 256, 1024, 128, (0, 0)),       # key tiles 0-5 seen by no query
    (1, 1, 200, 900, 64, (127, 300)),
    (1, 1, 900, 200, 128, (-1, 0)),       # the first 700 queries see no key
    (1, 1, 900, 300, 64, (50, 1)),        # queries that see no key, and a band
    (1, 2, 1, 600, 128, (300, 0)),        # one query (decode-like) with a band
    (1, 1, 130, 130, 128, (0, -1)),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B{}H{}Nq{}Nk{}d{}-w{}_{}".format(
    *c[:5], *c[5]))
def test_window_fwd_bwd_vs_oracle(case):
    B, H, Nq, Nk, d, window = case
    got, ref = _run(B, H, Nq, Nk, d, BF16, window, seed=500 + Nq + 3 * Nk + window[0])
    _check_L(got["L"], ref["L"])
    for name in ("o", "dq", "dk", "dv"):
        assert_close(name, got[name], ref[name], BF16)


@pytest.mark.parametrize("case", [CASES[2], CASES[4], CASES[10]],
                         ids=lambda c: "B{}H{}Nq{}Nk{}d{}-w{}_{}".format(*c[:5], *c[5]))
def test_window_fp16_vs_oracle(case):
    B, H, Nq, Nk, d, window = case
    got, ref = _run(B, H, Nq, Nk, d, FP16, window, seed=900 + Nq + Nk)
    _check_L(got["L"], ref["L"])
    for name in ("o", "dq", "dk", "dv"):
        assert_close(name, got[name], ref[name], FP16)


def test_unseen_key_tiles_get_exact_zero_gradients():
    got, ref = _run(1, 1, 256, 1024, 128, BF16, (0, 0), seed=77)
    # queries 0..255 see keys 768..1023 only
    assert np.count_nonzero(got["dk"][0, 0, :768]) == 0
    assert np.count_nonzero(got["dv"][0, 0, :768]) == 0


def test_window_equals_causal_and_unmasked_calls():
    """(-1, 0) is the causal mask and a window wider than every row is no mask at all:
    both must give the same bits as the causal / unmasked calls."""
    import torch
    a = make_inputs(1, 2, 640, 128, BF16, seed=5)
    q, k, v = (to_device(getattr(a, n), BF16) for n in ("q", "k", "v"))
    for causal, window in ((True, (-1, 0)), (False, (-1, -1)), (False, (5000, 5000))):
        o1, L1, _ = fa.forward(q, k, v, causal=causal)
        o2, L2, _ = fa.forward(q, k, v, window=window)
        torch.cuda.synchronize()
        assert torch.equal(o1, o2) and torch.equal(L1, L2), window
