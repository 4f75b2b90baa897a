"""Why the max-abs bar is read relative to |ref| above 1 (CPU only).

The parity bar for bf16 results is max-abs 2e-2 and mean-abs 2e-3. This test takes
the exact computation and rounds only what the method itself must round to 16 bits:
the operands P and dS of the gradient products, and the outputs. On inputs whose
query rows are scaled x8 (large logits), the exact result then already misses 2e-2
in absolute terms on dK, whose entries reach ~10. Measured relative to max(1, |ref|)
it is far inside the bar. So the GPU parity tests apply the max bar that way; for
entries with |ref| <= 1 it is the literal absolute bar.
"""

import math

import numpy as np

import oracle
from exact_io_aware_69_b200.inputs import BF16, make_inputs, round_to_bf16_bits, widen

from helpers import errors


def _bf16(x):
    return widen(round_to_bf16_bits(np.asarray(x, np.float32)), BF16).astype(np.float64)


def test_exact_bf16_operand_pipeline_needs_relative_max_bar():
    N, d = 512, 128
    inp = make_inputs(1, 2, N, d, BF16, seed=4242, large_frac=0.05)
    q, k, v, do = (inp.widened(n).reshape(2, N, d).astype(np.float64) for n in ("q", "k", "v", "do"))
    scale = 1 / math.sqrt(d)
    ref = oracle.attn_bwd(q, k, v, do, False, scale)
    dk = np.empty_like(ref["dk"])
    for bh in range(2):
        P = np.exp(scale * q[bh] @ k[bh].T - ref["L"][bh][:, None])
        dS = P * (do[bh] @ v[bh].T - ref["D"][bh][:, None])
        dk[bh] = _bf16(scale * (_bf16(dS).T @ q[bh]))
    absolute = np.abs(dk - ref["dk"]).max()
    _, rel_max, mean = errors(dk, ref["dk"])
    assert np.abs(ref["dk"]).max() > 8
    assert absolute > 2e-2          # the literal absolute bar is out of reach ...
    assert rel_max < 2e-2 / 2       # ... the relative reading leaves margin
    assert mean < 2e-3


def test_d_from_16_bit_O_alone_misses_the_bar():
    """D = rowsum(dO * O) with O rounded to bf16 moves dK of large-logit rows by ~5e-2
    even under the relative reading, which is why the forward also hands the backward
    O's rounding residual (O + O_res is O to ~2^-17)."""
    N, d = 512, 128
    inp = make_inputs(1, 2, N, d, BF16, seed=4242, large_frac=0.05)
    q, k, v, do = (inp.widened(n).reshape(2, N, d).astype(np.float64) for n in ("q", "k", "v", "do"))
    scale = 1 / math.sqrt(d)
    ref = oracle.attn_bwd(q, k, v, do, False, scale)
    for use_residual, ok in ((False, False), (True, True)):
        dk = np.empty_like(ref["dk"])
        for bh in range(2):
            o16 = _bf16(ref["o"][bh])
            o = o16 + _bf16(ref["o"][bh] - o16) if use_residual else o16
            D = (do[bh] * o).sum(axis=1)
            P = np.exp(scale * q[bh] @ k[bh].T - ref["L"][bh][:, None])
            dS = P * (do[bh] @ v[bh].T - D[:, None])
            dk[bh] = _bf16(scale * (_bf16(dS).T @ q[bh]))
        _, rel_max, _ = errors(dk, ref["dk"])
        assert (rel_max <= 2e-2) == ok, (use_residual, rel_max)
