"""The decode kernel's tiling of the visible rows (`visible_ranges`, `make_tiling`,
`make_tiling_paged`, `tiling_tile` in csrc/ps_ranges.cuh) against the oracle's visible set
(eq. A(i)) mapped to prefix rows and ring slots: the tiles' [lo, hi) rows cover every visible
row exactly once and nothing else.  Contiguous store: no 64-row box reads an in-bounds row
outside its segment (out-of-bounds rows are zero-filled by TMA, without traffic).  Paged
store: every tile is one whole 64-row block.  CPU only: the header's host/device functions
are compiled with g++."""
import os
import shutil
import subprocess

import numpy as np
import pytest

import oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
TILE = 64

_DRIVER = r"""
#include <cstdio>
#include "ps_ranges.cuh"
int main() {
  long long p; int lp, w, paged;
  while (std::scanf("%d %d %lld %d", &lp, &w, &p, &paged) == 4) {
    const ps::VisibleRanges r = ps::visible_ranges(p, lp, w);
    const ps::DecodeTiling t = paged ? ps::make_tiling_paged(r) : ps::make_tiling(r, lp, w);
    std::printf("case %d %d %lld %d %d\n", lp, w, p, paged, t.total);
    for (int i = 0; i < t.total; ++i) {
      const ps::DecodeTile d = ps::tiling_tile(t, i);
      std::printf("%d %d %d %d\n", d.map_id, d.row0, d.lo, d.hi);
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
    d = tmp_path_factory.mktemp("decode_tiling")
    src = d / "drv.cpp"
    src.write_text(_DRIVER)
    exe = d / "drv"
    subprocess.run([gxx, "-O1", "-std=c++17",
                    "-I" + os.path.join(ROOT, "prefix_sliding_window_b200", "csrc"),
                    "-I" + os.path.join(ROOT, "include"), str(src), "-o", str(exe)],
                   check=True)
    return str(exe)


def _cases(paged):
    lps = [0, 1, 63, 64, 65, 100, 128, 130, 300]
    ws = [64, 128, 256, 512, 4096] if paged else [1, 2, 63, 64, 65, 100, 128, 256, 4096]
    rng = np.random.default_rng(5 if paged else 3)
    out = []
    for lp in lps:
        for w in ws:
            ps = {0, 1, max(lp - 1, 0), lp, lp + 1, lp + w - 1, lp + w, lp + w + 1,
                  lp + 2 * w - 1, lp + 2 * w + 5, lp + 3 * w + 63}
            ps |= set(int(x) for x in rng.integers(0, lp + 3 * w + 64, size=12))
            out += [(lp, w, p) for p in sorted(ps)]
    return out


def _run(driver, cases, paged):
    inp = "".join(f"{lp} {w} {p} {int(paged)}\n" for lp, w, p in cases)
    lines = subprocess.run([driver], input=inp, capture_output=True, text=True,
                           check=True).stdout.splitlines()
    res, i = {}, 0
    while i < len(lines):
        _, lp, w, p, _, total = lines[i].split()
        tiles = [tuple(map(int, ln.split())) for ln in lines[i + 1:i + 1 + int(total)]]
        res[(int(lp), int(w), int(p))] = tiles
        i += 1 + int(total)
    return res


def _expected(lp, w, p):
    vis = O.visible_positions(p, lp, w)
    return {(0, int(k)) if k < lp else (1, int((k - lp) % w)) for k in vis}


@pytest.mark.parametrize("paged", [False, True])
def test_tiles_cover_exactly_the_visible_rows(driver, paged):
    cases = _cases(paged)
    got = _run(driver, cases, paged)
    assert len(got) == len(cases)
    for (lp, w, p), tiles in got.items():
        covered = []
        for map_id, row0, lo, hi in tiles:
            assert 0 <= lo < hi <= TILE, (lp, w, p, row0, lo, hi)
            covered += [(map_id, row0 + i) for i in range(lo, hi)]
            dim = lp if map_id == 0 else w
            if paged:
                assert row0 % TILE == 0 and 0 <= row0 < dim, (lp, w, p, row0)
            else:
                # rows of the box inside the tensor but outside [lo, hi) would be loaded
                for i in range(TILE):
                    if 0 <= row0 + i < dim:
                        assert lo <= i < hi, (lp, w, p, map_id, row0, lo, hi, i)
        assert len(covered) == len(set(covered)), (lp, w, p)
        assert set(covered) == _expected(lp, w, p), (lp, w, p)


def _expected_intervals(lp, w, p):
    """The same set as _expected, from the two intervals of eq. A(i) (prefix [0, min(p+1,
    Lp)), window [max(Lp, p+1-W), p]), for positions too large to enumerate every earlier
    key; test_oracle_pins ties the brute-force set to these intervals at small p."""
    pre = {(0, k) for k in range(min(p + 1, lp))}
    win = {(1, (k - lp) % w) for k in range(max(lp, p + 1 - w), p + 1)}
    return pre | win


@pytest.mark.parametrize("paged", [False, True])
def test_tiles_at_large_positions(driver, paged):
    """Ring offsets (window start - Lp) on both sides of 2^31 and 2^32 and far past them: the
    32-bit remainder and its 64-bit fallback in visible_ranges give the visible rows, once
    each, with the window starting at its oldest key's slot."""
    ws = [64, 100, 4096] if not paged else [64, 128, 4096]
    offs = [2 ** 31 - 1, 2 ** 31, 2 ** 32 - 1, 2 ** 32, 2 ** 32 + 1, 2 ** 32 + 63,
            2 ** 33 + 12345, 2 ** 40 + 7]
    cases = [(lp, w, lp + w - 1 + x) for lp in (0, 100, 300) for w in ws for x in offs]
    got = _run(driver, cases, paged)
    assert len(got) == len(cases)
    for (lp, w, p), tiles in got.items():
        covered = []
        for map_id, row0, lo, hi in tiles:
            assert 0 <= lo < hi <= TILE, (lp, w, p, row0, lo, hi)
            covered += [(map_id, row0 + i) for i in range(lo, hi)]
        assert len(covered) == len(set(covered)), (lp, w, p)
        assert set(covered) == _expected_intervals(lp, w, p), (lp, w, p)
        # a full window covers every slot whatever the start, so also check the order: the
        # window's first covered row is the slot of its oldest key
        first = next(row0 + lo for map_id, row0, lo, hi in tiles if map_id == 1)
        assert first == (max(lp, p + 1 - w) - lp) % w, (lp, w, p, first)
