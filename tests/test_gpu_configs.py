"""The five named workloads at full size, in the launch configuration bench.py times.

Where the oracle cannot afford a whole workload, the check is on outputs it can
compute one by one -- whole heads, single query rows (O, L, dQ are per-row
quantities), single keys near the end of a causal sequence (dK, dV of key j need
only the rows i >= j) -- plus identities that hold at any size: sum_j dK_j = 0 and
sum_j dV_j = sum_i dO_i for every head.
"""

import math

import numpy as np
import pytest

import oracle
from exact_io_aware_69_b200 import fa
from exact_io_aware_69_b200.inputs import BF16, WORKLOADS, sweep_workloads

from helpers import assert_close, assert_close_L, to_device, to_f64

pytestmark = pytest.mark.gpu


def _run(w):
    import torch
    inp = w.make()
    q, k, v, do = (to_device(getattr(inp, n), w.dtype) for n in ("q", "k", "v", "do"))
    o, L, o_res = fa.forward(q, k, v, causal=w.causal, scale=w.scale)
    dq, dk, dv = fa.backward(q, k, v, o, L, do, causal=w.causal, scale=w.scale, o_res=o_res)
    torch.cuda.synchronize()
    assert fa.device_status() == fa.FA_OK
    BH = w.B * w.H
    got = {n: to_f64(t).reshape(BH, w.N, w.d) for n, t in
           (("o", o), ("dq", dq), ("dk", dk), ("dv", dv))}
    got["L"] = to_f64(L).reshape(BH, w.N)
    del q, k, v, do, o, L, dq, dk, dv
    torch.cuda.empty_cache()
    inp.wide = {n: inp.widened(n).reshape(BH, w.N, w.d) for n in ("q", "k", "v", "do")}
    return inp, got


def _head(inp, w, h):
    return [inp.wide[n][h:h + 1].astype(np.float64) for n in ("q", "k", "v", "do")]


def _relative(w):
    """The relative reading of the max bar applies to the large-logit workload only."""
    return w.large_frac > 0


def _check_heads(w, inp, got, heads):
    for h in heads:
        ref = oracle.attn_bwd(*_head(inp, w, h), w.causal, w.scale)
        assert_close_L(got["L"][h], ref["L"][0])
        for n in ("o", "dq", "dk", "dv"):
            assert_close(f"{n}[head {h}]", got[n][h], ref[n][0], w.dtype, _relative(w))


def _check_rows(w, inp, got, heads, rows_per_head, rng, extra_rows=None):
    for h in heads:
        rows = set(rng.choice(w.N, size=rows_per_head, replace=False).tolist())
        rows |= {0, 1, 127, 128, w.N - 1}
        if extra_rows is not None:
            rows |= set(int(r) for r in extra_rows[h][:8])
        rows = np.array(sorted(rows))
        ref = oracle.attn_rows(*_head(inp, w, h), w.causal, w.scale, np.zeros(len(rows)), rows)
        assert_close_L(got["L"][h, rows], ref["L"])
        assert_close(f"o[head {h}]", got["o"][h, rows], ref["o"], w.dtype, _relative(w))
        assert_close(f"dq[head {h}]", got["dq"][h, rows], ref["dq"], w.dtype, _relative(w))


def _check_keys(w, inp, got, heads, keys):
    keys = np.array(sorted(set(int(x) for x in keys)))
    for h in heads:
        ref = oracle.attn_keys(*_head(inp, w, h), w.causal, w.scale, np.zeros(len(keys)), keys)
        assert_close(f"dk[head {h}]", got["dk"][h, keys], ref["dk"], w.dtype, _relative(w))
        assert_close(f"dv[head {h}]", got["dv"][h, keys], ref["dv"], w.dtype, _relative(w))


def _heavy_keys(w, inp, h, count):
    """The keys that the scaled-up (large-logit) query rows of head h weight most: for
    each such row its highest-scoring visible key, ranked by that key's probability
    (numpy on the 16-bit inputs; a row's probabilities need only its own scores)."""
    q, k = inp.wide["q"][h].astype(np.float64), inp.wide["k"][h].astype(np.float64)
    best = []
    for i in np.sort(inp.large_rows[h]):
        s = (k[:i + 1] @ q[i]) * w.scale if w.causal else (k @ q[i]) * w.scale
        j = int(np.argmax(s))
        best.append((float(1.0 / np.exp(s - s[j]).sum()), j))
    best.sort(reverse=True)
    return [j for _, j in best[:count]]


def _check_identities(w, inp, got):
    """sum over keys of dK is 0 and of dV is sum over queries of dO (per head), up to
    the 16-bit roundings the method makes: each output (2^-9 relative), P and dS as
    MMA operands (2^-9 relative), and O as stored for D = dO . O (D off by up to
    2^-9 * sum_t |dO_it O_it|, which leaves sum_j dS_ij = -dD_i instead of 0). The
    bound is four times the root-sum-square of those terms."""
    do = inp.wide["do"].astype(np.float64)
    q = inp.wide["q"].astype(np.float64)
    u = 2.0 ** -9
    dD = u * np.abs(do * got["o"]).sum(axis=2)                        # [BH, N]
    sk = np.abs(got["dk"].sum(axis=1))                                # [BH, d]
    # rounding of dS_ij: |sum_j err_ij| <= 2^-9 sum_j |dS_ij| <= 2^-8 |dO_i| max_j |v_j|
    v = inp.wide["v"].astype(np.float64)
    vmax = np.sqrt((v ** 2).sum(axis=2)).max(axis=1)                   # [BH]
    eS = 2 * u * np.sqrt((do ** 2).sum(axis=2)) * vmax[:, None]        # [BH, N]
    bk = 4 * (u * np.sqrt((got["dk"] ** 2).sum(axis=1))
              + w.scale * np.sqrt(((q * dD[..., None]) ** 2).sum(axis=1))
              + w.scale * np.sqrt(((q * eS[..., None]) ** 2).sum(axis=1)))
    sv = np.abs(got["dv"].sum(axis=1) - do.sum(axis=1))
    bv = 4 * (u * np.sqrt((got["dv"] ** 2).sum(axis=1)) + u * np.sqrt((do ** 2).sum(axis=1)))
    assert np.all(sk <= bk + 1e-6), float((sk / (bk + 1e-6)).max())
    assert np.all(sv <= bv + 1e-6), float((sv / (bv + 1e-6)).max())


def test_config1_full():
    w = WORKLOADS["c1"]
    inp, got = _run(w)
    _check_heads(w, inp, got, [0])


@pytest.mark.parametrize("name", ["c2", "c2c"])
def test_config2(name):
    w = WORKLOADS[name]
    inp, got = _run(w)
    BH = w.B * w.H
    _check_heads(w, inp, got, [0, 21, BH - 1])
    _check_rows(w, inp, got, range(BH), 4, np.random.default_rng(2))
    _check_identities(w, inp, got)


def test_config3():
    w = WORKLOADS["c3"]
    inp, got = _run(w)
    BH = w.B * w.H
    _check_heads(w, inp, got, [0, BH - 1])
    _check_rows(w, inp, got, range(BH), 4, np.random.default_rng(3))
    _check_identities(w, inp, got)


def test_config4_long_context_large_logits():
    w = WORKLOADS["c4"]
    inp, got = _run(w)
    BH = w.B * w.H
    rng = np.random.default_rng(4)
    _check_rows(w, inp, got, range(BH), 6, rng, extra_rows=inp.large_rows)
    # head 0: key tile 0 (the CTA with the longest loop: every query tile sees it), the
    # keys that the x8 rows weight most, and the last keys; one pass of the oracle's
    # row statistics over the whole head serves all of them
    heavy = _heavy_keys(w, inp, 0, 16)
    _check_keys(w, inp, got, [0], list(range(128)) + heavy + list(range(w.N - 130, w.N)))
    # last head: keys of the last tiles, which need only the rows behind them
    _check_keys(w, inp, got, [BH - 1], list(range(w.N - 130, w.N)) + [w.N - 1000])
    _check_identities(w, inp, got)


@pytest.mark.parametrize("w", sweep_workloads(), ids=lambda w: w.name.replace(" ", "-"))
def test_config5_sweep(w):
    inp, got = _run(w)
    BH = w.B * w.H
    rng = np.random.default_rng(5)
    if w.N <= 2048:
        _check_heads(w, inp, got, [0, BH - 1])
    else:
        _check_rows(w, inp, got, [0, BH - 1], 8, rng)
        if w.causal:
            _check_keys(w, inp, got, [0], list(range(w.N - 130, w.N)))
        else:
            _check_keys(w, inp, got, [BH - 1], rng.choice(w.N, size=16, replace=False))
    _check_identities(w, inp, got)
