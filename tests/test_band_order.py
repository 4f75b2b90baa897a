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
  long BH; int n, d;
  while (std::scanf("%ld %d %d", &BH, &n, &d) == 3) std::printf("%d\n", fa::band_group(BH, n, d));
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


def test_band_group_sizing(exes):
    _, group = exes
    cases = [(64, 8192, 128), (16, 65536, 128), (64, 2048, 64), (3, 512, 64), (64, 8192, 256),
             (1, 1, 64)]
    inp = "".join(f"{bh} {n} {d}\n" for bh, n, d in cases)
    out = list(map(int, subprocess.run([group], input=inp, capture_output=True, text=True,
                                       check=True).stdout.split()))
    budget = 48 << 20
    for (bh, n, d), g in zip(cases, out):
        assert 1 <= g <= bh
        per_head = 4 * n * d
        assert g == max(1, min(bh, budget // per_head))
    assert out[0] == 12  # B2 H32 N8192 d128: 4 MB streamed per head
    assert out[1] == 1   # N = 65536: one head's K and V already take 32 MB
