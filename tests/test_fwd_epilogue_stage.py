"""The forward kernel's epilogue stages O's rounding residual in the K stage of key tile
J1 - 2 + g (g: the warpgroup, J1: one past the CTA's last key tile) when its rule allows.
This replays, for every CTA of many shapes and masks, the MMA issuer's order (step j:
P V of tile j - 1 then S of tile j, warpgroup 0 first) and the K-load schedule (tile T
into stage (T - J0) mod 3), and checks that a stage the rule picks is never read by an
S MMA issued after that warpgroup's last P V, never refilled by a later K load, was
filled before, and differs from the other warpgroup's. Key ranges come from the
library's own tile schedule (fa_tile_range)."""
import itertools

import pytest

from exact_io_aware_69_b200 import fa

K_STAGES = 3
TILE = 128


def _res_stage_rule(g, ga, gn, J0, J1):
    """The kernel's condition for staging O_res in a K stage, and the tile whose stage."""
    res_tile = J1 - 2 + g
    ok = gn > 0 and res_tile >= J0 and (ga + gn == J1 if g == 1 else ga + gn >= J1 - 1)
    return ok, res_tile


def _check(Nq, Nk, window):
    ntq, ntk = -(-Nq // TILE), -(-Nk // TILE)
    used = 0
    for pair in range((ntq + 1) // 2):
        a, n = [0, 0], [0, 0]
        for g in range(2):
            t = 2 * pair + g
            if t < ntq:
                a[g], n[g] = (0, ntk) if window is None else fa.tile_range(True, t, Nq, Nk, window)
        if n[0] + n[1] == 0:
            continue
        J0 = a[1] if n[0] == 0 else (a[0] if n[1] == 0 else min(a[0], a[1]))
        J1 = max(a[0] + n[0] if n[0] else 0, a[1] + n[1] if n[1] else 0)
        seq = []
        for j in range(J0, J1 + 1):
            for g in range(2):
                if a[g] <= j - 1 < a[g] + n[g]:
                    seq.append(("PV", g, j - 1))
                if a[g] <= j < a[g] + n[g]:
                    seq.append(("S", g, j))
        stages = {}
        for g in range(2):
            ok, res_tile = _res_stage_rule(g, a[g], n[g], J0, J1)
            if not ok:
                continue
            used += 1
            s = (res_tile - J0) % K_STAGES
            stages[g] = s
            last_pv = max(i for i, x in enumerate(seq) if x[0] == "PV" and x[1] == g)
            for x in seq[last_pv + 1:]:
                assert not (x[0] == "S" and (x[2] - J0) % K_STAGES == s), (Nq, Nk, window, pair, g)
            for T in range(res_tile + 1, J1):  # K loads after the staged tile's
                assert (T - J0) % K_STAGES != s, (Nq, Nk, window, pair, g, T)
            reads = [i for i, x in enumerate(seq) if x[0] == "S" and x[2] == res_tile]
            assert reads and all(i < last_pv for i in reads), (Nq, Nk, window, pair, g)
        if len(stages) == 2:
            assert stages[0] != stages[1], (Nq, Nk, window, pair)
    return used


WINDOWS = [None, (-1, 0), (0, 0), (128, 0), (255, 0), (300, 10), (-1, 129), (1000, 1000), (64, -1)]


@pytest.mark.parametrize("window", WINDOWS, ids=str)
def test_residual_stage_is_idle(window):
    used = 0
    for Nq, Nk in itertools.product((128, 256, 300, 384, 640, 1000, 1024, 2048),
                                    (128, 256, 384, 500, 1024, 2048, 3000)):
        used += _check(Nq, Nk, window)
    assert used > 0  # the rule is taken on every mask


def test_rule_falls_back_when_a_range_ends_early():
    # warpgroup 1's range ending before J1, or warpgroup 0's before J1 - 1, keeps O_res
    # in the Q buffer
    assert not _res_stage_rule(1, 0, 3, 0, 5)[0]
    assert not _res_stage_rule(0, 0, 3, 0, 5)[0]
    assert _res_stage_rule(0, 0, 4, 0, 5) == (True, 3)
    assert _res_stage_rule(1, 0, 5, 0, 5) == (True, 4)
    assert not _res_stage_rule(0, 0, 1, 0, 1)[0]  # a single key tile: no tile J1 - 2
