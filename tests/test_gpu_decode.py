"""The split-KV decode path (fa_decode) vs the fp64 oracle.

A few query rows per head (1 to 16) against key sequences from one key to 128k keys:
one split (short sequences, O written by the split kernel itself) and many splits
merged by log-sum-exp; causal (bottom-right aligned), unmasked and windowed rows; rows
that see no key; both layouts and both 16-bit types. Also: repeated calls give the
same bits, and the tensor-core forward agrees within the parity bar.
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


def _run(B, H, Nq, Nk, d, dtype, window, seed, layout="bhnd"):
    import torch
    scale = 1.0 / math.sqrt(d)
    a = make_inputs(B, H, Nq, d, dtype, seed, with_do=False)
    b = make_inputs(B, H, Nk, d, dtype, seed + 1, with_do=False)
    q = to_device(a.q, dtype)
    k, v = to_device(b.k, dtype), to_device(b.v, dtype)
    if layout == "bnhd":
        q, k, v = (t.transpose(1, 2).contiguous() for t in (q, k, v))
    o, L = fa.decode(q, k, v, scale=scale, window=window, layout=layout)
    torch.cuda.synchronize()
    assert fa.device_status() == fa.FA_OK
    if layout == "bnhd":
        o = o.transpose(1, 2)
    ref = oracle.attn_window(a.widened("q"), b.widened("k"), b.widened("v"), None, window, scale)
    return to_f64(o), to_f64(L), ref, (q, k, v, scale)


CASES = [  # (B, H, Nq, Nk, d, window)
    (2, 3, 1, 1, 128, (-1, 0)),
    (1, 4, 1, 100, 64, (-1, -1)),
    (2, 2, 4, 128, 128, (-1, 0)),
    (1, 2, 1, 4133, 128, (-1, 0)),
    (1, 3, 3, 5000, 64, (-1, 0)),
    (1, 2, 16, 9000, 128, (-1, 0)),
    (1, 2, 9, 2049, 128, (-1, -1)),
    (1, 1, 16, 3000, 64, (700, 0)),
    (1, 2, 7, 6000, 128, (1000, 3)),
    (1, 1, 4, 2, 128, (-1, 0)),          # queries 0 and 1 see no key
    (1, 1, 16, 20000, 128, (10, 0)),     # windows far inside one tile pair
    (2, 2, 2, 3000, 128, (-1, 0)),       # the fewest rows the tensor-core form takes
]


@pytest.mark.parametrize("dtype", [BF16, FP16])
@pytest.mark.parametrize("case", CASES, ids=lambda c: "B{}H{}Nq{}Nk{}d{}-w{}_{}".format(
    *c[:5], *c[5]))
def test_decode_vs_oracle(case, dtype):
    B, H, Nq, Nk, d, window = case
    if dtype == FP16 and case not in (CASES[3], CASES[5], CASES[8]):
        pytest.skip("fp16 on three cases (the arithmetic is the same)")
    o, L, ref, _ = _run(B, H, Nq, Nk, d, dtype, window, seed=40 + Nq + Nk)
    _check_L(L, ref["L"])
    assert_close("o", o, ref["o"], dtype)


@pytest.mark.parametrize("Nq", [1, 4, 16])
def test_decode_long_context_128k(Nq):
    """128k keys, one head pair: many splits merged by log-sum-exp."""
    o, L, ref, _ = _run(1, 2, Nq, 131072, 128, BF16, (-1, 0), seed=11 + Nq)
    _check_L(L, ref["L"])
    assert_close("o", o, ref["o"], BF16)


def test_decode_bnhd_layout():
    o, L, ref, _ = _run(2, 3, 5, 3333, 128, BF16, (-1, 0), seed=5, layout="bnhd")
    _check_L(L, ref["L"])
    assert_close("o", o, ref["o"], BF16)


def test_decode_repeatable_and_agrees_with_the_forward():
    import torch
    _, _, ref, (q, k, v, scale) = _run(2, 4, 8, 20000, 128, BF16, (-1, 0), seed=3)
    o1, L1 = fa.decode(q, k, v, causal=True, scale=scale)
    o2, L2 = fa.decode(q, k, v, causal=True, scale=scale)
    of, Lf, _ = fa.forward(q, k, v, causal=True, scale=scale)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(L1, L2)
    assert_close("decode vs forward", to_f64(o1), to_f64(of), BF16)
    assert float((L1 - Lf).abs().max()) <= TOL_L
