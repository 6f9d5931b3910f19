"""The query kernel's weighted stream-K split, host side (no GPU needed).

The kernel and the host plan share two functions from csrc/arl2_kernels.h: split_start
(first unit of CTA c) and split_owner (the CTA holding unit u). This compiles a small host
program against that header with nvcc and checks, for the 480p layer, the sweep shapes, the
growing-KV-cache baseline and small ragged cases, that the ranges tile the units in order,
that the owner of every unit is the CTA whose range holds it, that no range is empty when the
weighted share spans a whole unit of the largest weight, and that a head unit (key tile 0)
moves the boundaries as its weight says.
"""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "softmax_attention_ar_b200", "csrc")

PROGRAM = r"""
#include <cstdio>
#include <cstdlib>
#include "arl2_kernels.h"
using namespace arl2;
int main(int argc, char** argv) {
  const long long units = atoll(argv[1]);
  const int nkv = atoi(argv[2]), hw = atoi(argv[3]), P = atoi(argv[4]);
  for (int c = 0; c <= P; ++c) printf("%lld%c", split_start(c, units, nkv, hw, P), c == P ? '\n' : ' ');
  for (long long u = 0; u < units; ++u) printf("%d%c", split_owner(u, units, nkv, hw, P), u + 1 == units ? '\n' : ' ');
  return 0;
}
"""


@pytest.fixture(scope="module")
def split_tool(tmp_path_factory):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not available")
    d = tmp_path_factory.mktemp("split")
    src, exe = d / "split.cu", d / "split"
    src.write_text(PROGRAM)
    subprocess.run([nvcc, "-std=c++17", "-I", CSRC, "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)],
                   check=True, capture_output=True)
    return str(exe)


def run_split(tool, units, nkv, hw, P):
    out = subprocess.run([tool, str(units), str(nkv), str(hw), str(P)], check=True, capture_output=True,
                         text=True).stdout.split("\n")
    return [int(x) for x in out[0].split()], [int(x) for x in out[1].split()]


def weight_before(u, nkv, hw):
    return 4 * u + hw * ((u + nkv - 1) // nkv)


# (B * H * nq query tiles, nkv key tiles per query tile, CTAs): 480p, B=4 480p, T=390 and
# T=3600, the KV-cache baseline at 60 frames, small ragged cases.
SHAPES = [(156, 13, 148), (624, 13, 148), (48, 4, 148), (348, 29, 148), (156, 780, 148), (3, 2, 5), (7, 3, 4),
          (1, 1, 1), (8, 29, 148)]


@pytest.mark.parametrize("qtiles,nkv,P", SHAPES)
@pytest.mark.parametrize("hw", [0, 10])
def test_ranges_tile_the_units_and_owner_agrees(split_tool, qtiles, nkv, P, hw):
    units = qtiles * nkv
    P = min(P, units)
    wtot = qtiles * (4 * nkv + hw)
    if hw and wtot // P < 4 + hw + 1:
        pytest.skip("the plan uses no head weight for this split")
    starts, owners = run_split(split_tool, units, nkv, hw, P)
    assert starts[0] == 0 and starts[-1] == units
    assert all(a < b for a, b in zip(starts, starts[1:])), "a range is empty or out of order"
    for u, c in enumerate(owners):
        assert starts[c] <= u < starts[c + 1], (u, c)
    # Each range starts at the first unit whose weighted start reaches c * W / P.
    for c in range(P):
        target = c * wtot // P
        u = starts[c]
        assert weight_before(u, nkv, hw) >= target
        assert u == 0 or weight_before(u - 1, nkv, hw) < target


def test_head_weight_gives_fewer_units_to_ranges_with_more_heads(split_tool):
    # T = 3600 (29 key tiles a query tile): with the head weight, a range holding more key
    # tile 0 units holds fewer units in all.
    qtiles, nkv, P = 348, 29, 148
    starts, _ = run_split(split_tool, qtiles * nkv, nkv, 10, P)
    by_heads = {}
    for c in range(P):
        u0, u1 = starts[c], starts[c + 1]
        heads = sum(1 for u in range(u0, u1) if u % nkv == 0)
        by_heads.setdefault(heads, []).append(u1 - u0)
    ks = sorted(by_heads)
    assert len(ks) >= 2
    mean = {k: sum(v) / len(v) for k, v in by_heads.items()}
    assert mean[ks[-1]] < mean[ks[0]] - 1   # 2.5 units a head, less the rounding
    # Every range's weight is the share c W / P to within one unit of the largest weight.
    share = qtiles * (4 * nkv + 10) / P
    for c in range(P):
        w = weight_before(starts[c + 1], nkv, 10) - weight_before(starts[c], nkv, 10)
        assert abs(w - share) <= 4 + 10 + 1, (c, w, share)
