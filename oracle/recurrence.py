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


# ---------------------------------------------------------------------------------
# Split keys, then merge: the same recurrence applied to whole blocks at once.
#
# The running state of the recurrence after a block of keys is (m, l, o); carrying it
# into the next block rescales what has been accumulated by exp(m_old - m_new). Two
# states over disjoint key blocks combine the same way, whichever order they are
# merged in. Written in log-sum-exp form -- each block's normalised output o_s and
# L_s = ln(sum over the block's visible keys of exp(score)) -- the merge is
#     L = ln(sum_s exp(L_s)),    o = sum_s exp(L_s - L) o_s,
# which is what a decode path that splits a long key sequence across processors and
# merges their partial results computes. A block in which the row sees no key has
# L_s = -inf and drops out.


def merge_partials(o_parts, L_parts):
    """Merge per-block results of one query row: o_parts [S, d], L_parts [S] (natural
    log units; -inf for a block with no visible key). Returns (o, L); (0, -inf) when no
    block saw a key."""
    o_parts = np.asarray(o_parts, dtype=np.float64)
    L_parts = np.asarray(L_parts, dtype=np.float64)
    if np.all(np.isneginf(L_parts)):
        return np.zeros(o_parts.shape[1]), -math.inf
    m = float(L_parts.max())
    w = np.exp(L_parts - m)               # exp(-inf) = 0 for empty blocks
    total = float(w.sum())
    return (w[:, None] * o_parts).sum(axis=0) / total, m + math.log(total)


def _visible(i, j, nq, nk, window):
    """Query i sees key j under the (left, right) key window, bottom-right aligned
    (negative = that side unbounded)."""
    off = nk - nq
    left, right = window
    return (left < 0 or j >= i + off - left) and (right < 0 or j <= i + off + right)


def attn_fwd_split(q, k, v, window, scale, block_sizes):
    """Forward attention of the query rows q [Nq, d] against k, v [Nk, d] with the keys
    cut into consecutive blocks of the given sizes: each block's (o_s, L_s) is the plain
    definition restricted to that block's visible keys, then the blocks are merged.
    Returns (O [Nq, d], L [Nq])."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    nq, nk = q.shape[0], k.shape[0]
    if sum(block_sizes) != nk or any(b <= 0 for b in block_sizes):
        raise ValueError("block sizes must be positive and cover every key")
    O = np.zeros((nq, v.shape[1]))
    L = np.full(nq, -math.inf)
    for i in range(nq):
        o_parts, L_parts = [], []
        start = 0
        for size in block_sizes:
            keys = [j for j in range(start, start + size) if _visible(i, j, nq, nk, window)]
            start += size
            if not keys:
                o_parts.append(np.zeros(v.shape[1]))
                L_parts.append(-math.inf)
                continue
            s = scale * (k[keys] @ q[i])
            mx = float(s.max())
            e = np.exp(s - mx)
            o_parts.append(e @ v[keys] / e.sum())
            L_parts.append(mx + math.log(float(e.sum())))
        O[i], L[i] = merge_partials(o_parts, L_parts)
    return O, L
