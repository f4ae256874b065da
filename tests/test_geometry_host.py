"""Host-side checks of the CUDA library's block <-> token map (csrc/geometry.cuh), compiled for the
CPU with g++: every block's tokens against the oracle's independent s3r_ref_block_tokens, and the
per-step slot bitmask the selection kernel masks with against the per-slot map."""
import os
import subprocess
import tempfile

import numpy as np
import pytest

from oracle import oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "sparse_global_attention_s3r_b200", "csrc")

PROGRAM = r"""
#define __host__
#define __device__
#define __forceinline__ inline
#include <cstdio>
#include <cstdlib>
#include <initializer_list>
#include "geometry.cuh"
using namespace s3r;
int main(int argc, char** argv) {
  // L b two_d special gh gw wh
  BlockGeo g{};
  g.L = std::atoll(argv[1]); g.b = std::atoi(argv[2]); g.two_d = std::atoi(argv[3]);
  int64_t nb;
  if (g.two_d) {
    g.special = std::atoi(argv[4]); g.gh = std::atoi(argv[5]); g.gw = std::atoi(argv[6]);
    g.wh = std::atoi(argv[7]);
    const int ww = g.b / g.wh;
    while ((1 << g.lww) < ww) ++g.lww;
    g.P = g.special + static_cast<int64_t>(g.gh) * g.gw;
    g.cols = (g.gw + ww - 1) / ww;
    g.per_view = (g.special > 0) + ((g.gh + g.wh - 1) / g.wh) * g.cols;
    nb = (g.L / g.P) * g.per_view;
  } else {
    nb = (g.L + g.b - 1) / g.b;
  }
  int bad = 0;
  for (int64_t j = 0; j < nb; ++j) {
    const BlockOrigin bo = block_origin(g, j);
    std::printf("%lld", static_cast<long long>(j));
    bool full = true;
    for (int o = 0; o < g.b; ++o) {
      const int64_t t = origin_token(g, bo, o);
      if (t != slot_token(g, j, o)) ++bad;
      if (t >= 0) std::printf(" %lld", static_cast<long long>(t)); else full = false;
    }
    std::printf("\n");
    if (full != block_full(g, j)) ++bad;
    for (int n : {32, 64}) {
      if (n > g.b) continue;
      for (int o0 = 0; o0 + n <= g.b; ++o0) {
        uint64_t want = 0;
        for (int i = 0; i < n; ++i) if (origin_token(g, bo, o0 + i) >= 0) want |= 1ull << i;
        if (slot_bits(g, bo, o0, n) != want) ++bad;
      }
    }
  }
  std::printf("bad %d\n", bad);
  return 0;
}
"""

GEOMETRIES = [  # (N views or L, b, special, gh, gw, wh); gh == 0: 1-D blocks over L = first entry
    (1000, 64, 0, 0, 0, 0), (1000, 32, 0, 0, 0, 0), (1300, 128, 0, 0, 0, 0), (17, 64, 0, 0, 0, 0),
    (3, 64, 5, 37, 37, 8), (3, 32, 3, 10, 13, 4), (2, 128, 0, 20, 35, 8), (1, 64, 2, 3, 5, 8),
    (3, 32, 32, 6, 9, 4), (2, 32, 1, 7, 9, 8), (2, 128, 4, 5, 300, 1), (2, 64, 0, 9, 9, 64),
]


@pytest.fixture(scope="module")
def exe():
    d = tempfile.mkdtemp()
    src = os.path.join(d, "geo.cc")
    with open(src, "w") as f:
        f.write(PROGRAM)
    out = os.path.join(d, "geo")
    subprocess.run(["g++", "-std=c++17", "-O1", "-I", CSRC, src, "-o", out], check=True)
    return out


@pytest.mark.parametrize("geo", GEOMETRIES)
def test_block_token_map_matches_oracle_and_masks_match_slots(exe, geo):
    first, b, special, gh, gw, wh = geo
    if gh == 0:
        L, args, pb = first, [str(first), str(b), "0"], O.Problem(first, 1, 64, b, 1)
    else:
        L = first * (special + gh * gw)
        args = [str(L), str(b), "1", str(special), str(gh), str(gw), str(wh)]
        pb = O.Problem(L, 1, 64, b, 1, grid_h=gh, grid_w=gw, special=special, win_h=wh)
    res = subprocess.run([exe] + args, check=True, capture_output=True, text=True).stdout.split("\n")
    assert res[-2] == "bad 0", res[-2]
    rows = [r.split() for r in res[:-2]]
    assert len(rows) == pb.nb
    for r in rows:
        j = int(r[0])
        got = np.array([int(x) for x in r[1:]], np.int64)
        np.testing.assert_array_equal(np.sort(got), pb.block_tokens(j))
