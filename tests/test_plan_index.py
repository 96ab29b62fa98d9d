"""The backward's closed-form position of a key tile in its query tile's plan
(`plan_index` in csrc/ps_ranges.cuh, used to find a pair's dS tile without a search) equals
that key tile's position in the oracle's brute-force plan, for every pair a key-tile item of
the backward visits.  CPU only: the header's host/device functions are compiled with g++."""
import os
import shutil
import subprocess

import numpy as np
import pytest

import oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
B = 128
CASES = [(1, 0, 1), (129, 7, 1), (300, 100, 64), (1000, 0, 128), (1000, 127, 129),
         (2500, 256, 1000), (4096, 128, 2048), (8192, 256, 2048), (8191, 1000, 5000),
         (3000, 300, 10000), (640, 129, 127),
         # L_prefix reaching or passing the sequence's end, tile-edge lengths
         (129, 134, 12), (1, 6, 129), (127, 127, 256), (129, 129, 2), (128, 128, 1),
         (256, 256, 129), (675, 489, 128), (129, 1, 256), (255, 127, 215), (509, 129, 129)]

_DRIVER = r"""
#include <cstdio>
#include "ps_ranges.cuh"
int main() {
  long long seq; int lp, w;
  while (std::scanf("%lld %d %d", &seq, &lp, &w) == 3) {
    for (long long kt = 0; kt * @B@ < seq; ++kt) {
      int64_t qlo, qhi;
      if (!ps::ktile_qrange(kt, seq, lp, w, @B@, &qlo, &qhi)) continue;
      for (int64_t qt = qlo; qt <= qhi; ++qt)
        std::printf("%lld %d %d %lld %lld %lld\n", seq, lp, w, (long long)qt, kt,
                    (long long)ps::plan_index(qt, kt, lp, w, @B@));
    }
  }
  return 0;
}
"""


@pytest.fixture(scope="module")
def driver(tmp_path_factory):
    gxx = shutil.which("g++")
    if gxx is None:
        pytest.skip("g++ not available")
    d = tmp_path_factory.mktemp("plan_index")
    src = d / "drv.cpp"
    src.write_text(_DRIVER.replace("@B@", str(B)))
    exe = d / "drv"
    subprocess.run([gxx, "-O1", "-std=c++17",
                    "-I" + os.path.join(ROOT, "prefix_sliding_window_b200", "csrc"),
                    "-I" + os.path.join(ROOT, "include"), str(src), "-o", str(exe)],
                   check=True)
    return str(exe)


def test_plan_index_matches_oracle_plan(driver):
    inp = "".join(f"{s} {lp} {w}\n" for s, lp, w in CASES)
    out = subprocess.run([driver], input=inp, capture_output=True, text=True, check=True).stdout
    got = {}
    for line in out.splitlines():
        s, lp, w, qt, kt, idx = map(int, line.split())
        got[(s, lp, w, qt, kt)] = idx
    n = 0
    for s, lp, w in CASES:
        plan = O.tile_plan(s, lp, w, B, B)
        pos = {}
        for q in np.unique(plan[:, 0]):
            row = plan[plan[:, 0] == q]
            for i, k in enumerate(row[:, 1]):
                pos[(int(q), int(k))] = i
        visited = {(qt, kt) for (s2, lp2, w2, qt, kt) in got if (s2, lp2, w2) == (s, lp, w)}
        # the backward visits exactly the planned pairs
        assert visited == set(pos), (s, lp, w)
        for (qt, kt), i in pos.items():
            assert got[(s, lp, w, qt, kt)] == i, (s, lp, w, qt, kt)
            n += 1
    assert n > 3000
