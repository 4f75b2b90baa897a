"""The seeded input generator: rounding, determinism and the large-logit rows."""

import numpy as np
import torch

from exact_io_aware_69_b200.inputs import (BF16, FP16, WORKLOADS, make_inputs, round_to_bf16_bits,
                                           round_to_fp16_bits, sweep_workloads, widen)


def test_bf16_round_to_nearest_even_ties():
    # ulp(1) in bf16 is 2^-7: 1 + 2^-8 ties to 1 (even), 1 + 3*2^-8 ties up to 1 + 2^-6
    x = np.array([1 + 2**-8, 1 + 3 * 2**-8, -(1 + 2**-8), 1 + 2**-8 + 2**-20], np.float32)
    got = widen(round_to_bf16_bits(x), BF16)
    np.testing.assert_array_equal(got, np.array([1.0, 1 + 2**-6, -1.0, 1 + 2**-7], np.float32))


def test_rounding_matches_torch_conversions():
    x = np.random.default_rng(0).standard_normal(100000).astype(np.float32) * 3
    ref_bf = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(round_to_bf16_bits(x), ref_bf)
    ref_h = torch.from_numpy(x).to(torch.float16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(round_to_fp16_bits(x), ref_h)


def test_deterministic_and_distinct_streams():
    a = make_inputs(1, 2, 64, 16, BF16, seed=7)
    b = make_inputs(1, 2, 64, 16, BF16, seed=7)
    c = make_inputs(1, 2, 64, 16, BF16, seed=8)
    for name in ("q", "k", "v", "do"):
        np.testing.assert_array_equal(getattr(a, name), getattr(b, name))
    assert not np.array_equal(a.q, c.q)
    assert not np.array_equal(a.q, a.k)


def test_large_rows_are_scaled_by_eight():
    base = make_inputs(1, 2, 1000, 8, BF16, seed=3)
    big = make_inputs(1, 2, 1000, 8, BF16, seed=3, large_frac=0.01, large_factor=8.0)
    assert big.large_rows.shape == (2, 10)
    qb = base.widened("q").reshape(2, 1000, 8)
    qg = big.widened("q").reshape(2, 1000, 8)
    for bh in range(2):
        rows = big.large_rows[bh]
        assert len(set(rows.tolist())) == 10
        np.testing.assert_array_equal(qg[bh, rows], 8 * qb[bh, rows])
        others = np.setdiff1d(np.arange(1000), rows)
        np.testing.assert_array_equal(qg[bh, others], qb[bh, others])


def test_workload_table():
    assert WORKLOADS["c3"].N == 8192 and WORKLOADS["c3"].d == 128 and WORKLOADS["c3"].causal
    assert WORKLOADS["c4"].large_frac == 0.01
    sw = sweep_workloads()
    assert len(sw) == 6 * 2 * 2 * 2
    assert all(w.B * w.N == 16384 and w.H == 16 for w in sw)
    assert {w.dtype for w in sw} == {BF16, FP16}
