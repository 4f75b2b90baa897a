"""band_order (fa_band.cuh), the block -> (head, rank) order of band launches, compiled
for the host: every work item is visited exactly once, items go rank-major within each
group of heads (a rank is started for every head of the group before the next rank),
groups follow one another, and group = 1 is plain head-major order. Also band_group's
sizing: at least one head, at most all of them, fewer heads for longer sequences."""
import os
import subprocess
import tempfile

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "exact_io_aware_69_b200", "csrc")

PROGRAM = r'''
#include <cstdio>
#define __host__
#define __device__
#include "fa_band.cuh"
int main() {
  int per_head, BH, group;
  while (std::scanf("%d %d %d", &per_head, &BH, &group) == 3) {
    for (int b = 0; b < per_head * BH; ++b) {
      int bh, rank;
      fa::band_order(b, per_head, BH, group, &bh, &rank);
      std::printf("%d %d ", bh, rank);
    }
    std::printf("\n");
  }
  return 0;
}
'''

GROUP_PROGRAM = r'''
#include <cstdio>
#define __host__
#define __device__
#include "fa_band.cuh"
int main() {
  long BH, bytes, mg, budget;
  while (std::scanf("%ld %ld %ld %ld", &BH, &bytes, &mg, &budget) == 4)
    std::printf("%d\n", fa::band_group(BH, bytes, mg, budget));
  return 0;
}
'''


def _build(src, name, tmp):
    path = os.path.join(tmp, name + ".cpp")
    exe = os.path.join(tmp, name)
    with open(path, "w") as fh:
        fh.write(src)
    subprocess.run(["g++", "-std=c++17", "-O1", "-I", CSRC, path, "-o", exe], check=True)
    return exe


@pytest.fixture(scope="module")
def exes():
    with tempfile.TemporaryDirectory() as tmp:
        yield _build(PROGRAM, "order", tmp), _build(GROUP_PROGRAM, "group", tmp)


CASES = [(32, 64, 12), (32, 64, 1), (32, 64, 64), (64, 5, 3), (1, 7, 2), (7, 1, 1), (3, 10, 4),
         (16, 13, 5)]


def test_band_order_is_a_grouped_rank_major_permutation(exes):
    order, _ = exes
    inp = "".join(f"{p} {bh} {g}\n" for p, bh, g in CASES)
    out = subprocess.run([order], input=inp, capture_output=True, text=True, check=True).stdout
    for (per_head, BH, group), line in zip(CASES, out.strip().split("\n")):
        v = list(map(int, line.split()))
        items = list(zip(v[0::2], v[1::2]))
        assert len(items) == per_head * BH
        assert sorted(items) == [(h, r) for h in range(BH) for r in range(per_head)]
        expect = []
        for g0 in range(0, BH, group):
            heads = list(range(g0, min(BH, g0 + group)))
            expect += [(h, r) for r in range(per_head) for h in heads]
        assert items == expect, (per_head, BH, group)
        if group == 1:
            assert items == [(h, r) for h in range(BH) for r in range(per_head)]


def _groups(exe, cases):
    inp = "".join(f"{bh} {b} {mg} {bud}\n" for bh, b, mg, bud in cases)
    return list(map(int, subprocess.run([exe], input=inp, capture_output=True, text=True,
                                        check=True).stdout.split()))


def test_band_group_sizing(exes):
    _, group = exes
    fwd, bwd = (3, 88 << 20), (1, 48 << 20)
    cases = [(64, 4 * 8192 * 128, *fwd), (16, 4 * 65536 * 128, *fwd), (64, 4 * 2048 * 64, *fwd),
             (3, 4 * 512 * 64, *fwd), (64, 8 * 8192 * 128, *bwd), (1, 256, *fwd), (5, 0, *fwd),
             (2, 1 << 30, *fwd), (16, 8 * 65536 * 128, *bwd), (16, 4 * 32768 * 128, *fwd),
             (16, 4 * 16384 * 128, *fwd), (7, 40 << 20, *fwd)]
    out = _groups(group, cases)
    for (bh, per_head, mg, budget), g in zip(cases, out):
        assert 1 <= g <= bh
        ng = min(bh, max(mg, -(-bh * per_head // budget)))
        cap = max(1, budget // per_head) if per_head else bh
        assert g == min(-(-bh // ng), cap), (bh, per_head, g)
        assert -(-bh // g) >= min(mg, bh)  # at least min_groups groups
        assert g == 1 or g * per_head <= budget  # a group's bytes stay within the budget
    assert out[0] == 22  # forward, B2 H32 N8192 d128: 3 groups (22, 22 and 20 heads; 88 MiB)
    assert out[1] == 2   # forward, N = 65536: 32 MiB of K and V per head (3 would be 96 MiB)
    assert out[9] == 5   # forward, N = 32768: 16 MiB per head, 5 heads = 80 MiB
    assert out[10] == 6  # forward, N = 16384: 3 groups of 6 heads, 48 MiB
    assert out[4] == 6   # dK/dV kernel at c3: 8 MiB per head with the fp32 dQ accumulator
    assert out[8] == 1   # dK/dV kernel at N = 65536: one head already takes 64 MiB
    assert out[11] == 2  # 7 heads of 40 MiB: 3 groups would round up to 3 heads (120 MiB)
