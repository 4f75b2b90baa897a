"""Pins of the fp64 oracle to facts that do not come from the oracle itself.

The pages print no worked numbers, so each pin is one of: a hand-worked tiny case
(tests/golden/hand_worked.json), a closed form, an invariant, brute force on tiny
inputs, central finite differences, or the pages' own per-row online recurrence
restated independently (oracle/recurrence.py). Each is chosen so that a plausible
slip in the oracle -- a dropped term, a wrong sign, a transposed operand, a missing
scale, a mask off by one -- fails at least one of them.
"""

import json
import math
import os

import numpy as np
import pytest

import oracle
from oracle.recurrence import online_row, random_split
from exact_io_aware_69_b200.inputs import BF16, make_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_worked.json")


def _ev(expr):
    return float(eval(expr, {"__builtins__": {}}, {"ln": math.log}))


def _evarr(x):
    if isinstance(x, list):
        return np.array([_evarr(e) for e in x], dtype=np.float64)
    return _ev(x)


def _rand(BH, N, d, seed, with_do=True):
    inp = make_inputs(1, BH, N, d, BF16, seed, with_do=with_do)
    f = lambda a: inp.widened(a).reshape(BH, N, d).astype(np.float64)
    return f("q"), f("k"), f("v"), f("do")


def _golden_cases():
    with open(GOLDEN) as fh:
        data = json.load(fh)
    out = []
    for case in data["cases"]:
        for mode in ("noncausal", "causal"):
            out.append(pytest.param(case, mode, id=f"{case['name']}-{mode}"))
    return out


@pytest.mark.parametrize("case,mode", _golden_cases())
def test_hand_worked_cases(case, mode):
    """Tiny cases computed by hand from the three-step definition."""
    q, k, v, do = (np.array(case[n], dtype=np.float64)[None] for n in ("q", "k", "v", "do"))
    exp = case[mode]
    out = oracle.attn_bwd(q, k, v, do, causal=(mode == "causal"), scale=_ev(case["scale"]))
    for name in ("o", "dq", "dk", "dv"):
        np.testing.assert_allclose(out[name][0], _evarr(exp[name]), rtol=0, atol=1e-12, err_msg=name)
    np.testing.assert_allclose(out["L"][0], _evarr(exp["L"]), rtol=0, atol=1e-12)
    np.testing.assert_allclose(out["D"][0], _evarr(exp["D"]), rtol=0, atol=1e-12)
    o_f, L_f = oracle.attn_fwd(q, k, v, causal=(mode == "causal"), scale=_ev(case["scale"]))
    np.testing.assert_allclose(o_f[0], _evarr(exp["o"]), rtol=0, atol=1e-12)
    np.testing.assert_allclose(L_f[0], _evarr(exp["L"]), rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N,d,scale", [(37, 8, 1 / math.sqrt(8)), (128, 64, 1 / 8), (65, 16, 1.7)])
def test_online_recurrence_equals_two_pass(N, d, scale, causal):
    """The pages' block-by-block recurrence reaches the two-pass softmax result."""
    q, k, v, _ = _rand(2, N, d, seed=11 + N)
    o, L = oracle.attn_fwd(q, k, v, causal, scale)
    rng = np.random.default_rng(5)
    for bh in range(2):
        for i in list(range(0, N, max(1, N // 9))) + [N - 1]:
            nvis = i + 1 if causal else N
            split = random_split(nvis, rng)
            o_r, L_r = online_row(q[bh, i], k[bh, :nvis], v[bh, :nvis], scale, split)
            np.testing.assert_allclose(o_r, o[bh, i], rtol=1e-12, atol=1e-13)
            assert abs(L_r - L[bh, i]) <= 1e-12 * max(1.0, abs(L_r))
            # one block of everything, and blocks of one key, are the extremes
            for split2 in ([nvis], [1] * nvis):
                o_r2, L_r2 = online_row(q[bh, i], k[bh, :nvis], v[bh, :nvis], scale, split2)
                np.testing.assert_allclose(o_r2, o[bh, i], rtol=1e-12, atol=1e-13)
                assert abs(L_r2 - L[bh, i]) <= 1e-12 * max(1.0, abs(L_r2))


@pytest.mark.parametrize("causal", [False, True])
def test_rows_of_P_sum_to_one(causal):
    """With every value vector equal to 1, each output entry is the row sum of P."""
    q, k, _, _ = _rand(3, 300, 32, seed=3)
    ones = np.ones_like(q)
    o, _ = oracle.attn_fwd(q, k, ones, causal, 1 / math.sqrt(32))
    assert np.max(np.abs(o - 1.0)) <= 1e-13


def test_single_key():
    """N = 1: O = V, L = scale q.k, dV = dO, dQ = dK = 0."""
    q, k, v, do = _rand(4, 1, 16, seed=4)
    scale = 0.25
    out = oracle.attn_bwd(q, k, v, do, False, scale)
    np.testing.assert_allclose(out["o"], v, rtol=0, atol=1e-15)
    for bh in range(4):
        s = scale * math.fsum(float(a) * float(b) for a, b in zip(q[bh, 0], k[bh, 0]))
        assert abs(out["L"][bh, 0] - s) <= 1e-13 * max(1.0, abs(s))
    np.testing.assert_allclose(out["dv"], do, rtol=0, atol=1e-15)
    assert np.max(np.abs(out["dq"])) <= 1e-15
    assert np.max(np.abs(out["dk"])) <= 1e-15


def test_identical_keys():
    """All keys equal: O = mean of V, L = s + ln N, dQ = 0 (P does not depend on q)."""
    N, d, scale = 50, 8, 0.3
    q, k, v, do = _rand(2, N, d, seed=6)
    k[:] = k[:, :1, :]
    out = oracle.attn_bwd(q, k, v, do, False, scale)
    for bh in range(2):
        np.testing.assert_allclose(out["o"][bh], np.broadcast_to(v[bh].mean(0), (N, d)),
                                   rtol=1e-12, atol=1e-13)
        s = scale * (q[bh] @ k[bh, 0])
        np.testing.assert_allclose(out["L"][bh], s + math.log(N), rtol=1e-12, atol=1e-12)
    assert np.max(np.abs(out["dq"])) <= 1e-13


@pytest.mark.parametrize("causal", [False, True])
def test_zero_queries(causal):
    """Q = 0: every score is 0, so the output is a (prefix) mean of V."""
    N, d = 40, 8
    _, k, v, do = _rand(2, N, d, seed=7)
    q = np.zeros_like(k)
    out = oracle.attn_bwd(q, k, v, do, causal, 0.5)
    for bh in range(2):
        if causal:
            cnt = np.arange(1, N + 1, dtype=np.float64)
            o_exp = np.cumsum(v[bh], axis=0) / cnt[:, None]
            L_exp = np.log(cnt)
            # dV_j = sum_{i >= j} dO_i / (i + 1)
            w = do[bh] / cnt[:, None]
            dv_exp = np.cumsum(w[::-1], axis=0)[::-1]
        else:
            o_exp = np.broadcast_to(v[bh].mean(0), (N, d))
            L_exp = np.full(N, math.log(N))
            dv_exp = np.broadcast_to(do[bh].sum(0) / N, (N, d))
        np.testing.assert_allclose(out["o"][bh], o_exp, rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(out["L"][bh], L_exp, rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(out["dv"][bh], dv_exp, rtol=1e-12, atol=1e-13)
    assert np.max(np.abs(out["dk"])) <= 1e-15  # dK_j = scale * sum_i dS_ij q_i with q = 0


def test_permutation_equivariance():
    """Non-causal attention is a function of the key/value SET and equivariant in queries."""
    N, d, scale = 33, 8, 0.35
    q, k, v, do = _rand(2, N, d, seed=8)
    base = oracle.attn_bwd(q, k, v, do, False, scale)
    rng = np.random.default_rng(1)
    pk = rng.permutation(N)
    out = oracle.attn_bwd(q, k[:, pk], v[:, pk], do, False, scale)
    for name in ("o", "dq", "L"):
        np.testing.assert_allclose(out[name], base[name], rtol=1e-12, atol=1e-13)
    for name in ("dk", "dv"):
        np.testing.assert_allclose(out[name], base[name][:, pk], rtol=1e-12, atol=1e-13)
    pq = rng.permutation(N)
    out = oracle.attn_bwd(q[:, pq], k, v, do[:, pq], False, scale)
    for name in ("o", "dq", "L"):
        np.testing.assert_allclose(out[name], base[name][:, pq], rtol=1e-12, atol=1e-13)
    for name in ("dk", "dv"):
        np.testing.assert_allclose(out[name], base[name], rtol=1e-12, atol=1e-13)
    # transposing the roles of Q and K changes the answer (guards against a swapped operand)
    swapped = oracle.attn_fwd(k, q, v, False, scale)[0]
    assert np.max(np.abs(swapped - base["o"])) > 1e-3


def _fd_grads(q, k, v, do, causal, scale, h=1e-6):
    def loss(qq, kk, vv):
        o, _ = oracle.attn_fwd(qq, kk, vv, causal, scale)
        return math.fsum((o * do).ravel())

    grads = []
    for which in range(3):
        args = [q, k, v]
        base = args[which]
        g = np.zeros_like(base)
        for idx in np.ndindex(base.shape):
            plus = base.copy(); plus[idx] += h
            minus = base.copy(); minus[idx] -= h
            ap = list(args); ap[which] = plus
            am = list(args); am[which] = minus
            g[idx] = (loss(*ap) - loss(*am)) / (2 * h)
        grads.append(g)
    return grads


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N,d", [(1, 1), (2, 2), (3, 4), (5, 8), (17, 2), (17, 8)])
def test_finite_differences(N, d, causal):
    """Analytic dQ, dK, dV equal central differences of sum(O * dO)."""
    rng = np.random.default_rng(100 + 10 * N + d)
    q, k, v, do = (rng.standard_normal((1, N, d)) for _ in range(4))
    scale = 1 / math.sqrt(d) if d > 1 else 0.9
    out = oracle.attn_bwd(q, k, v, do, causal, scale)
    fd = _fd_grads(q, k, v, do, causal, scale)
    for name, g in zip(("dq", "dk", "dv"), fd):
        err = np.linalg.norm(out[name] - g)
        assert err <= 1e-6 * max(np.linalg.norm(g), 1.0), (name, err)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 2, 5, 8])
def test_textbook_softmax_brute_force(N, causal):
    """For small logits, exp(s)/sum exp(s) without max subtraction, in pure Python."""
    d = 4
    rng = np.random.default_rng(200 + N)
    q, k, v = (rng.standard_normal((1, N, d)) * 0.5 for _ in range(3))
    scale = 0.5
    o, L = oracle.attn_fwd(q, k, v, causal, scale)
    for i in range(N):
        keys = range(i + 1) if causal else range(N)
        e = [math.exp(scale * math.fsum(q[0, i, t] * k[0, j, t] for t in range(d))) for j in keys]
        tot = math.fsum(e)
        for t in range(d):
            ref = math.fsum(e[n] * v[0, j, t] for n, j in enumerate(keys)) / tot
            assert abs(o[0, i, t] - ref) <= 1e-12
        assert abs(L[0, i] - math.log(tot)) <= 1e-12


def test_large_logits_stay_finite_and_exact():
    """Rows scaled x8 (and one x1024, whose exp would overflow without max subtraction)."""
    N, d = 64, 64
    inp = make_inputs(1, 1, N, d, BF16, seed=9, large_frac=0.1, large_factor=8.0)
    q = inp.widened("q").reshape(1, N, d).astype(np.float64)
    k = inp.widened("k").reshape(1, N, d).astype(np.float64)
    v = inp.widened("v").reshape(1, N, d).astype(np.float64)
    q[0, 5] *= 1024.0
    scale = 1 / 8
    for causal in (False, True):
        o, L = oracle.attn_fwd(q, k, v, causal, scale)
        assert np.all(np.isfinite(o)) and np.all(np.isfinite(L))
        for i in [5] + [int(r) for r in inp.large_rows[0][:3]] + [N - 1]:
            keys = range(i + 1) if causal else range(N)
            s = [scale * math.fsum(q[0, i] * k[0, j]) for j in keys]
            m = max(s)
            e = [math.exp(x - m) for x in s]
            tot = math.fsum(e)
            assert abs(L[0, i] - (m + math.log(tot))) <= 1e-12 * max(1.0, abs(m))
            for t in range(0, d, 7):
                ref = math.fsum(e[n] * v[0, j, t] for n, j in enumerate(keys)) / tot
                assert abs(o[0, i, t] - ref) <= 1e-12
    assert abs(L[0, 5]) > 700  # the x1024 row's logits are beyond exp's double range


@pytest.mark.parametrize("causal", [False, True])
def test_sampled_rows_and_keys_match_full(causal):
    """The per-row and per-key entry points agree with the full backward."""
    BH, N, d, scale = 3, 70, 16, 0.25
    q, k, v, do = _rand(BH, N, d, seed=10)
    full = oracle.attn_bwd(q, k, v, do, causal, scale)
    bh = np.array([0, 1, 2, 2, 0, 1])
    idx = np.array([0, 69, 33, 1, 64, 5])
    rows = oracle.attn_rows(q, k, v, do, causal, scale, bh, idx)
    keys = oracle.attn_keys(q, k, v, do, causal, scale, bh, idx)
    for r in range(len(bh)):
        np.testing.assert_allclose(rows["o"][r], full["o"][bh[r], idx[r]], rtol=0, atol=1e-14)
        np.testing.assert_allclose(rows["dq"][r], full["dq"][bh[r], idx[r]], rtol=0, atol=1e-14)
        assert abs(rows["L"][r] - full["L"][bh[r], idx[r]]) <= 1e-14
        assert abs(rows["D"][r] - full["D"][bh[r], idx[r]]) <= 1e-14
        np.testing.assert_allclose(keys["dk"][r], full["dk"][bh[r], idx[r]], rtol=0, atol=1e-14)
        np.testing.assert_allclose(keys["dv"][r], full["dv"][bh[r], idx[r]], rtol=0, atol=1e-14)
    fwd_rows = oracle.attn_rows(q, k, v, None, causal, scale, bh, idx)
    np.testing.assert_allclose(fwd_rows["o"], rows["o"], rtol=0, atol=0)


@pytest.mark.parametrize("causal", [False, True])
def test_gradient_identities(causal):
    """sum_j dK_j = 0, sum_j dV_j = sum_i dO_i, and D_i = dO_i . O_i."""
    q, k, v, do = _rand(2, 96, 16, seed=12)
    out = oracle.attn_bwd(q, k, v, do, causal, 0.25)
    assert np.max(np.abs(out["dk"].sum(axis=1))) <= 1e-12
    np.testing.assert_allclose(out["dv"].sum(axis=1), do.sum(axis=1), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(out["D"], np.einsum("bnd,bnd->bn", do, out["o"]), rtol=1e-12,
                               atol=1e-12)


def test_causal_row_is_prefix_attention():
    """Causal row i equals non-causal attention of that row over keys 0..i."""
    N, d, scale = 24, 8, 0.4
    q, k, v, _ = _rand(1, N, d, seed=13)
    o_c, L_c = oracle.attn_fwd(q, k, v, True, scale)
    for i in (0, 1, 11, N - 1):
        o_p, L_p = oracle.attn_fwd(q[:, :i + 1], k[:, :i + 1], v[:, :i + 1], False, scale)
        np.testing.assert_allclose(o_c[0, i], o_p[0, i], rtol=1e-13, atol=1e-14)
        assert abs(L_c[0, i] - L_p[0, i]) <= 1e-13


def test_scale_enters_scores():
    """scale multiplies q.k: scale 2 on Q equals scale 1 on 2Q."""
    q, k, v, _ = _rand(1, 20, 8, seed=14)
    o1, L1 = oracle.attn_fwd(2 * q, k, v, False, 1.0)
    o2, L2 = oracle.attn_fwd(q, k, v, False, 2.0)
    np.testing.assert_allclose(o1, o2, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(L1, L2, rtol=1e-13, atol=1e-14)


# ---------------------------------------------------------------- N_q != N_k
# Bottom-right causal alignment (query i sees keys j <= i + N_k - N_q) and rows that
# see no key, pinned to independent results: SciPy's softmax for a single query, and
# the square causal oracle (pinned above) through the identities below.

def _qkv(nq, nk, d, seed, bh=2):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((bh, nq, d))
    k = rng.standard_normal((bh, nk, d))
    v = rng.standard_normal((bh, nk, d))
    do = rng.standard_normal((bh, nq, d))
    return q, k, v, do


@pytest.mark.parametrize("causal", [False, True])
def test_single_query_is_library_softmax(causal):
    """N_q = 1: the query sees every key either way; O = softmax(scale K q) V and
    L = logsumexp(scale K q) by SciPy."""
    from scipy.special import logsumexp, softmax
    q, k, v, _ = _qkv(1, 37, 16, seed=5)
    scale = 0.3
    o, L = oracle.attn_fwd(q, k, v, causal, scale)
    for h in range(q.shape[0]):
        s = scale * k[h] @ q[h, 0]
        np.testing.assert_allclose(o[h, 0], softmax(s) @ v[h], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(L[h, 0], logsumexp(s), rtol=1e-13)


def test_non_causal_rows_are_independent():
    """Without a mask each query row is its own single-query problem."""
    q, k, v, _ = _qkv(5, 23, 8, seed=6)
    o, L = oracle.attn_fwd(q, k, v, False, 0.4)
    for i in range(q.shape[1]):
        oi, Li = oracle.attn_fwd(q[:, i:i + 1], k, v, False, 0.4)
        np.testing.assert_array_equal(o[:, i:i + 1], oi)
        np.testing.assert_array_equal(L[:, i:i + 1], Li)


@pytest.mark.parametrize("nq,nk", [(3, 11), (7, 8), (1, 5)])
def test_bottom_right_causal_is_suffix_of_square(nq, nk):
    """N_q < N_k, causal: the rows equal the last N_q rows of the square causal problem
    whose queries are [any N_k - N_q rows; Q]; with dO = [0; dO] the extra rows add
    nothing to dK and dV either."""
    q, k, v, do = _qkv(nq, nk, 8, seed=nq * 31 + nk)
    rng = np.random.default_rng(99)
    extra = rng.standard_normal((q.shape[0], nk - nq, q.shape[2]))
    q_sq = np.concatenate([extra, q], axis=1)
    do_sq = np.concatenate([np.zeros_like(extra), do], axis=1)
    got = oracle.attn_bwd(q, k, v, do, True, 0.35)
    sq = oracle.attn_bwd(q_sq, k, v, do_sq, True, 0.35)
    for name in ("o", "dq"):
        np.testing.assert_allclose(got[name], sq[name][:, nk - nq:], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(got["L"], sq["L"][:, nk - nq:], rtol=1e-13)
    for name in ("dk", "dv"):
        np.testing.assert_allclose(got[name], sq[name], rtol=1e-11, atol=1e-13)


@pytest.mark.parametrize("nq,nk", [(9, 4), (6, 1)])
def test_queries_that_see_no_key(nq, nk):
    """N_q > N_k, causal: the first N_q - N_k queries see no key (O = 0, L = -inf,
    dQ = 0, D = 0, nothing added to dK, dV); the others are the square causal problem
    on the last N_k queries."""
    q, k, v, do = _qkv(nq, nk, 8, seed=nq * 7 + nk)
    got = oracle.attn_bwd(q, k, v, do, True, 0.5)
    e = nq - nk
    assert np.all(got["o"][:, :e] == 0) and np.all(got["dq"][:, :e] == 0)
    assert np.all(got["L"][:, :e] == -np.inf) and np.all(got["D"][:, :e] == 0)
    sq = oracle.attn_bwd(q[:, e:], k, v, do[:, e:], True, 0.5)
    for name in ("o", "dq", "L", "D"):
        np.testing.assert_array_equal(got[name][:, e:], sq[name])
    for name in ("dk", "dv"):
        np.testing.assert_allclose(got[name], sq[name], rtol=1e-13, atol=1e-15)


# ------------------------------------------------------------- key windows
# (left, right) windows, the next mask variant. Pinned to the unmasked and causal
# oracles, to a closed form, to single-query attention over the key slice, and to
# central finite differences of the windowed forward.

@pytest.mark.parametrize("nq,nk", [(6, 6), (4, 9), (9, 4)])
def test_window_unbounded_and_causal_equal_the_plain_masks(nq, nk):
    q, k, v, do = _qkv(nq, nk, 8, seed=300 + nq * 10 + nk)
    for window, causal in (((-1, -1), False), ((-1, 0), True)):
        got = oracle.attn_window(q, k, v, do, window, 0.4)
        ref = oracle.attn_bwd(q, k, v, do, causal, 0.4)
        for name in ("o", "L", "dq", "dk", "dv", "D"):
            np.testing.assert_allclose(got[name], ref[name], rtol=1e-13, atol=1e-15,
                                       err_msg=f"{name} window {window}")


def test_window_of_one_key():
    """(0, 0) with Nq = Nk: query i sees key i only, so O_i = v_i, L_i = s_ii, D_i =
    dO_i . v_i, dV_i = dO_i and dQ = dK = 0 (P = 1, so dS = dP - D = 0)."""
    q, k, v, do = _qkv(7, 7, 8, seed=17)
    got = oracle.attn_window(q, k, v, do, (0, 0), 0.5)
    np.testing.assert_array_equal(got["o"], v)
    np.testing.assert_allclose(got["L"], 0.5 * np.einsum("bid,bid->bi", q, k), rtol=1e-14)
    np.testing.assert_allclose(got["D"], np.einsum("bid,bid->bi", do, v), rtol=1e-14)
    np.testing.assert_array_equal(got["dv"], do)
    assert np.all(got["dq"] == 0) and np.all(got["dk"] == 0)


@pytest.mark.parametrize("window", [(2, 1), (0, 3), (3, -1), (1, 0)])
def test_window_rows_are_single_queries_over_the_slice(window):
    nq, nk = 8, 11
    q, k, v, _ = _qkv(nq, nk, 8, seed=41 + window[0] * 5 + window[1])
    got = oracle.attn_window(q, k, v, None, window, 0.3)
    off = nk - nq
    for i in range(nq):
        lo = 0 if window[0] < 0 else max(0, i + off - window[0])
        hi = nk if window[1] < 0 else min(nk, i + off + window[1] + 1)
        if hi <= lo:
            assert np.all(got["o"][:, i] == 0) and np.all(got["L"][:, i] == -np.inf)
            continue
        o1, L1 = oracle.attn_fwd(q[:, i:i + 1], k[:, lo:hi], v[:, lo:hi], False, 0.3)
        np.testing.assert_allclose(got["o"][:, i], o1[:, 0], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(got["L"][:, i], L1[:, 0], rtol=1e-13)


def test_window_gradients_are_finite_differences():
    """dQ, dK, dV of the windowed backward against central differences of
    f = sum(O * dO) from the windowed forward."""
    nq, nk, d, window, scale = 5, 7, 4, (2, 1), 0.45
    q, k, v, do = _qkv(nq, nk, d, seed=77, bh=1)
    got = oracle.attn_window(q, k, v, do, window, scale)

    def f(qq, kk, vv):
        return float(np.sum(oracle.attn_window(qq, kk, vv, None, window, scale)["o"] * do))

    h = 1e-6
    for name, arr in (("dq", q), ("dk", k), ("dv", v)):
        num = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            plus, minus = arr.copy(), arr.copy()
            plus[idx] += h
            minus[idx] -= h
            args = {"dq": (q, k, v), "dk": (q, k, v), "dv": (q, k, v)}[name]
            a_p = [plus if x is arr else x for x in args]
            a_m = [minus if x is arr else x for x in args]
            num[idx] = (f(*a_p) - f(*a_m)) / (2 * h)
        np.testing.assert_allclose(got[name], num, rtol=1e-6, atol=1e-8, err_msg=name)


# ---------------------------------------------------------------- split and merge
@pytest.mark.parametrize("nq", [1, 4, 16])
@pytest.mark.parametrize("nk", [1, 37, 300])
@pytest.mark.parametrize("window", [(-1, -1), (-1, 0), (20, 3), (0, 0)])
def test_split_keys_then_merge_equals_the_definition(nq, nk, window):
    """Cutting the keys into blocks, attending within each block and merging the
    blocks' (o, L) by their log-sum-exps gives the plain definition back (decode's
    split-KV path), for every split, including blocks in which a row sees no key."""
    from oracle.recurrence import attn_fwd_split, random_split
    rng = np.random.default_rng(nq * 1000 + nk)
    d = 8
    q = rng.standard_normal((nq, d))
    k = rng.standard_normal((nk, d))
    v = rng.standard_normal((nk, d))
    ref = oracle.attn_window(q[None], k[None], v[None], None, window, 0.7)
    for _ in range(3):
        O, L = attn_fwd_split(q, k, v, window, 0.7, random_split(nk, rng))
        empty = np.isneginf(ref["L"][0])
        assert np.array_equal(np.isneginf(L), empty)
        np.testing.assert_allclose(L[~empty], ref["L"][0][~empty], rtol=0, atol=1e-12)
        np.testing.assert_allclose(O, ref["o"][0], rtol=0, atol=1e-12)


def test_merge_is_order_free_and_ignores_empty_blocks():
    from oracle.recurrence import merge_partials
    rng = np.random.default_rng(7)
    o = rng.standard_normal((5, 4))
    L = rng.standard_normal(5) * 10
    o1, L1 = merge_partials(o, L)
    perm = rng.permutation(5)
    o2, L2 = merge_partials(o[perm], L[perm])
    np.testing.assert_allclose(o2, o1, atol=1e-13)
    assert abs(L2 - L1) < 1e-13
    # merging two merged groups = merging all at once (the merge is associative)
    oa, La = merge_partials(o[:2], L[:2])
    ob, Lb = merge_partials(o[2:], L[2:])
    o3, L3 = merge_partials([oa, ob], [La, Lb])
    np.testing.assert_allclose(o3, o1, atol=1e-13)
    assert abs(L3 - L1) < 1e-13
    # an extra block with no visible key (L = -inf, any o) changes nothing
    o4, L4 = merge_partials(np.vstack([o, np.full((1, 4), 1e30)]), np.append(L, -np.inf))
    np.testing.assert_allclose(o4, o1, atol=1e-13)
    assert L4 == L1
    # no block saw a key: O = 0, L = -inf
    o5, L5 = merge_partials(np.ones((2, 4)), [-np.inf, -np.inf])
    assert np.all(o5 == 0) and L5 == -np.inf
    # closed form for two equal blocks: L = L_s + ln 2, o = mean of the two outputs
    o6, L6 = merge_partials(o[:2], [1.5, 1.5])
    np.testing.assert_allclose(o6, o[:2].mean(axis=0), atol=1e-14)
    assert abs(L6 - (1.5 + math.log(2))) < 1e-14
