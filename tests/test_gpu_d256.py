"""Head dimension 256: the forward (fa_fwd / fa_fwd_ex, one query tile per CTA, two score
buffers) against the fp64 oracle, element by element.

The cases cover square, ragged (N not a multiple of 128) and N_q != N_k shapes, the
causal mask and key windows (rows that see no key: O = 0, L = -inf), both tensor
layouts, bf16 and fp16, the rounding residual O_res, and sampled rows of a larger
causal problem. The backward has no d = 256 kernel and says so.
"""

import math

import numpy as np
import pytest

import oracle
from exact_io_aware_69_b200 import fa
from exact_io_aware_69_b200.inputs import BF16, FP16, make_inputs

from helpers import TOL_L, assert_close, to_device, to_f64

pytestmark = pytest.mark.gpu

D = 256


def _check_L(got, ref):
    got = np.asarray(got, np.float64)
    empty = np.isneginf(ref)
    assert np.array_equal(np.isneginf(got), empty), "L: -inf rows differ"
    assert np.all(np.isfinite(got[~empty])), "L: non-finite values"
    if (~empty).any():
        mx = float(np.max(np.abs(got[~empty] - ref[~empty])))
        assert mx <= TOL_L, f"L: max-abs {mx:.3e} (tol {TOL_L:.0e})"


def _forward(B, H, Nq, Nk, dtype, window, seed, layout="bhnd"):
    import torch
    scale = 1.0 / math.sqrt(D)
    a = make_inputs(B, H, Nq, D, dtype, seed)
    b = make_inputs(B, H, Nk, D, dtype, seed + 1)
    q, k, v = to_device(a.q, dtype), to_device(b.k, dtype), to_device(b.v, dtype)
    if layout == "bnhd":
        q, k, v = (t.transpose(1, 2).contiguous() for t in (q, k, v))
    o, L, o_res = fa.forward(q, k, v, scale=scale, window=window, layout=layout)
    torch.cuda.synchronize()
    assert fa.device_status() == fa.FA_OK
    if layout == "bnhd":
        o, o_res = o.transpose(1, 2), o_res.transpose(1, 2)
    ref = oracle.attn_window(a.widened("q"), b.widened("k"), b.widened("v"), None, window,
                             scale)
    return o, L, o_res, ref


CASES = [  # (B, H, Nq, Nk, window)
    (1, 2, 256, 256, (-1, -1)),
    (1, 2, 384, 384, (-1, 0)),
    (2, 1, 300, 300, (-1, -1)),     # ragged last tile
    (1, 1, 333, 333, (-1, 0)),
    (1, 1, 200, 520, (-1, -1)),     # Nq < Nk
    (1, 2, 130, 700, (-1, 0)),
    (1, 1, 700, 200, (-1, 0)),      # the first 500 queries see no key
    (1, 1, 640, 640, (127, 0)),     # a band ending on a tile edge
    (1, 2, 512, 512, (100, 30)),
    (1, 1, 1, 900, (-1, -1)),       # one query
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B{}H{}Nq{}Nk{}-w{}_{}".format(
    c[0], c[1], c[2], c[3], *c[4]))
def test_d256_forward_vs_oracle(case):
    import torch
    B, H, Nq, Nk, window = case
    o, L, o_res, ref = _forward(B, H, Nq, Nk, BF16, window, seed=9000 + Nq + 3 * Nk)
    _check_L(to_f64(L), ref["L"])
    assert_close("o", to_f64(o), ref["o"], BF16)
    empty = np.isneginf(ref["L"])
    if empty.any():
        assert torch.count_nonzero(o[torch.as_tensor(empty).to(o.device)]).item() == 0


@pytest.mark.parametrize("case", [CASES[1], CASES[4], CASES[8]],
                         ids=["square-causal", "Nq<Nk", "band"])
def test_d256_forward_fp16_vs_oracle(case):
    B, H, Nq, Nk, window = case
    o, L, o_res, ref = _forward(B, H, Nq, Nk, FP16, window, seed=9100 + Nq)
    _check_L(to_f64(L), ref["L"])
    assert_close("o", to_f64(o), ref["o"], FP16)


def test_d256_residual_is_the_rounding_of_o():
    """O_res = bf16(O_fp32 - O) is at most half an ulp of O (<= 2^-8 |O| in bf16), and
    O + O_res is closer to the exact O than O alone (what remains is the error of the
    16-bit P weights, which O_res does not carry)."""
    o, L, o_res, ref = _forward(1, 2, 384, 384, BF16, (-1, 0), seed=9200)
    o64, r64 = to_f64(o), to_f64(o_res)
    assert np.all(np.abs(r64) <= 2.0 ** -8 * np.abs(o64) + 1e-30)
    e1 = np.abs(o64 - ref["o"]).max()
    e2 = np.abs(o64 + r64 - ref["o"]).max()
    assert e2 < e1 / 2, (e1, e2)


def test_d256_bnhd_matches_bhnd():
    import torch
    o1, L1, r1, ref = _forward(2, 2, 300, 300, BF16, (-1, 0), seed=9300)
    o2, L2, r2, _ = _forward(2, 2, 300, 300, BF16, (-1, 0), seed=9300, layout="bnhd")
    assert torch.equal(o1, o2) and torch.equal(L1, L2) and torch.equal(r1, r2)
    assert_close("o", to_f64(o2), ref["o"], BF16)


def test_d256_sampled_rows_larger_causal():
    """B1 H4 N4096 causal: 256 sampled (head, row) pairs against the oracle's rows."""
    import torch
    B, H, N = 1, 4, 4096
    scale = 1.0 / math.sqrt(D)
    a = make_inputs(B, H, N, D, BF16, 9400)
    q, k, v = to_device(a.q, BF16), to_device(a.k, BF16), to_device(a.v, BF16)
    o, L, _ = fa.forward(q, k, v, causal=True, scale=scale)
    torch.cuda.synchronize()
    assert fa.device_status() == fa.FA_OK
    rng = np.random.default_rng(9401)
    bh = rng.integers(0, B * H, 256)
    rows = rng.integers(0, N, 256)
    rows[:4] = [0, 127, 128, N - 1]
    ref = oracle.attn_rows(a.widened("q"), a.widened("k"), a.widened("v"), None, True, scale,
                           bh, rows)
    o_got = to_f64(o).reshape(B * H, N, D)[bh, rows]
    L_got = to_f64(L).reshape(B * H, N)[bh, rows]
    assert_close("o", o_got, ref["o"], BF16)
    assert float(np.abs(L_got - ref["L"]).max()) <= TOL_L


def test_d256_backward_is_unsupported():
    import torch
    q = torch.zeros((1, 1, 128, D), dtype=torch.bfloat16, device="cuda")
    o, L, o_res = fa.forward(q, q, q)
    with pytest.raises(Exception, match="UNSUPPORTED"):
        fa.backward(q, q, q, o, L, q, o_res=o_res)
