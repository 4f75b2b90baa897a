"""The deterministic backward (fa_bwd_ex with deterministic = 1).

dQ is formed by its own pass, one CTA per query tile summing the key tiles in a
fixed order, so repeated calls must give identical bits; dK and dV come from the same
dK/dV kernel as the default mode (without its dQ work) and must equal the default
mode's bit for bit; and every gradient must meet the parity bar against the oracle.
"""

import math

import numpy as np
import pytest

import oracle
from exact_io_aware_69_b200 import fa
from exact_io_aware_69_b200.inputs import BF16, FP16, WORKLOADS, make_inputs

from helpers import assert_close, to_device, to_f64

pytestmark = pytest.mark.gpu

CASES = [  # (B, H, Nq, Nk, d, window, layout)
    (1, 2, 512, 512, 128, (-1, 0), "bhnd"),
    (2, 1, 384, 384, 64, (-1, -1), "bhnd"),
    (1, 2, 333, 333, 128, (-1, 0), "bhnd"),
    (1, 1, 200, 700, 64, (-1, 0), "bhnd"),
    (1, 1, 700, 200, 128, (-1, 0), "bhnd"),    # queries that see no key
    (1, 2, 640, 640, 128, (128, 5), "bhnd"),
    (1, 1, 256, 1024, 64, (0, 0), "bhnd"),     # query tiles and key tiles outside the band
    (2, 3, 300, 300, 128, (-1, 0), "bnhd"),
]


def _inputs(B, H, Nq, Nk, d, dtype, layout, seed):
    a = make_inputs(B, H, Nq, d, dtype, seed)
    b = make_inputs(B, H, Nk, d, dtype, seed + 1)
    q, do = to_device(a.q, dtype), to_device(a.do, dtype)
    k, v = to_device(b.k, dtype), to_device(b.v, dtype)
    if layout == "bnhd":
        q, k, v, do = (t.transpose(1, 2).contiguous() for t in (q, k, v, do))
    return a, b, q, k, v, do


def _back(t, layout):
    return t.transpose(1, 2) if layout == "bnhd" else t


@pytest.mark.parametrize("dtype", [BF16, FP16])
@pytest.mark.parametrize("case", CASES, ids=lambda c: "B{}H{}Nq{}Nk{}d{}-w{}_{}-{}".format(
    *c[:5], *c[5], c[6]))
def test_deterministic_backward(case, dtype):
    import torch
    B, H, Nq, Nk, d, window, layout = case
    if dtype == FP16 and case not in (CASES[0], CASES[4], CASES[5]):
        pytest.skip("fp16 on three cases (the arithmetic is the same)")
    scale = 1.0 / math.sqrt(d)
    a, b, q, k, v, do = _inputs(B, H, Nq, Nk, d, dtype, layout, seed=800 + Nq + Nk)
    o, L, r = fa.forward(q, k, v, scale=scale, window=window, layout=layout)
    runs = [fa.backward(q, k, v, o, L, do, scale=scale, o_res=r, window=window, layout=layout,
                        deterministic=True) for _ in range(3)]
    plain = fa.backward(q, k, v, o, L, do, scale=scale, o_res=r, window=window, layout=layout)
    torch.cuda.synchronize()
    assert fa.device_status() == fa.FA_OK
    for g in runs[1:]:
        assert torch.equal(g[0], runs[0][0]), "dQ differs between repeated calls"
        assert torch.equal(g[1], runs[0][1]) and torch.equal(g[2], runs[0][2])
    assert torch.equal(runs[0][1], plain[1]) and torch.equal(runs[0][2], plain[2])
    ref = oracle.attn_window(a.widened("q"), b.widened("k"), b.widened("v"), a.widened("do"),
                             window, scale)
    for name, t in (("dq", runs[0][0]), ("dk", runs[0][1]), ("dv", runs[0][2])):
        assert_close(name, to_f64(_back(t, layout)), ref[name], dtype)


def test_deterministic_workspace_is_row_statistics_only():
    lib = fa.load()
    B, H, N, d = 2, 3, 1000, 128
    n_pad = 1024
    assert lib.fa_bwd_ex_workspace_size(B, H, N, N, d, 1) == B * H * n_pad * 8
    assert lib.fa_bwd_ex_workspace_size(B, H, N, N, d, 0) == B * H * n_pad * 8 + B * H * N * d * 4


def test_deterministic_config3_rows_and_repeat():
    """The headline workload: bit-identical dQ on a repeat, and dQ rows against the
    oracle on two heads."""
    import torch
    w = WORKLOADS["c3"]
    inp = w.make()
    q, k, v, do = (to_device(getattr(inp, n), w.dtype) for n in ("q", "k", "v", "do"))
    o, L, r = fa.forward(q, k, v, causal=True, scale=w.scale)
    g1 = fa.backward(q, k, v, o, L, do, causal=True, scale=w.scale, o_res=r, deterministic=True)
    dq1 = g1[0].clone()
    del g1
    g2 = fa.backward(q, k, v, o, L, do, causal=True, scale=w.scale, o_res=r, deterministic=True)
    torch.cuda.synchronize()
    assert fa.device_status() == fa.FA_OK
    assert torch.equal(dq1, g2[0])
    BH = w.B * w.H
    got = to_f64(g2[0]).reshape(BH, w.N, w.d)
    wide = {n: inp.widened(n).reshape(BH, w.N, w.d) for n in ("q", "k", "v", "do")}
    rng = np.random.default_rng(31)
    for h in (0, BH - 1):
        rows = np.array(sorted(set(rng.choice(w.N, 12, replace=False).tolist()) |
                               {0, 127, 128, w.N - 1}))
        ref = oracle.attn_rows(*(wide[n][h:h + 1].astype(np.float64) for n in ("q", "k", "v", "do")),
                               True, w.scale, np.zeros(len(rows)), rows)
        assert_close(f"dq[head {h}]", got[h, rows], ref["dq"], w.dtype)
