"""The pages' per-row online-softmax recurrence, restated in fp64 (test infrastructure).

josueisai.com "flash-attention", section "El truco: trocear y llevar la cuenta del
softmax": one query row walks over K/V in blocks and carries two running
statistics, the largest score seen so far (m) and the running sum of exponentials
(l), plus a partial output (o). When a block brings a larger maximum, what has been
accumulated so far is rescaled to the new reference; after the last block o is
divided by l once. The section states that the result then equals the softmax of
the whole row. kerneldigest.dev "FlashAttention" (first paragraph) calls the same
idea online log-sum-exp scaling.

This is written from that description, independently of the C oracle, so that the
tests can hold the two against each other: the C oracle materialises the full row
and takes the two-pass softmax, this walks the row block by block.

Scale and mask are readings, not on the pages: scores are ``scale * q.k`` and a
causal row passes only its visible keys.
"""

from __future__ import annotations

import math

import numpy as np


def online_row(q_row, keys, values, scale, block_sizes):
    """Attention output and log-sum-exp of one query row, consuming keys block by block.

    ``block_sizes`` is any sequence of positive ints summing to len(keys): the split is
    arbitrary, which is the point of the recurrence.
    Returns (o, L) with L = m + ln l in natural-log units of the scaled score.
    """
    q_row = np.asarray(q_row, dtype=np.float64)
    keys = np.asarray(keys, dtype=np.float64)
    values = np.asarray(values, dtype=np.float64)
    if sum(block_sizes) != keys.shape[0] or any(b <= 0 for b in block_sizes):
        raise ValueError("block sizes must be positive and cover every key")
    m = -math.inf
    l = 0.0
    o = np.zeros(values.shape[1], dtype=np.float64)
    start = 0
    for size in block_sizes:
        kb = keys[start:start + size]
        vb = values[start:start + size]
        start += size
        s = scale * (kb @ q_row)
        block_max = float(s.max())
        m_next = max(m, block_max)
        # weight of everything accumulated so far, relative to the new reference
        carry = math.exp(m - m_next) if m != -math.inf else 0.0
        e = np.exp(s - m_next)
        l = l * carry + float(e.sum())
        o = o * carry + e @ vb
        m = m_next
    return o / l, m + math.log(l)


def random_split(n, rng):
    """A random composition of n into positive block sizes (uneven, possibly size 1)."""
    sizes = []
    left = n
    while left > 0:
        b = int(rng.integers(1, left + 1))
        sizes.append(b)
        left -= b
    return sizes
