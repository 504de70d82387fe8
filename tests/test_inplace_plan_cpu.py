"""The In-Place tensor-core kernel's tile schedule, checked on the CPU.

A small host program includes the kernel's source (for its file-local plan builder and list
rotation), links the library for the rest, and prints every plan; the test checks that each
chunk's tiles appear exactly once across the lists (one list per CTA with 128-row tiles, per
SM pair with 256-row tiles), that the longest list stays within a few percent of the mean by
the plan's own cost model, that each list runs its TARGET tiles, then its UPDATE tiles, then
its APPLY tiles, and that the rotation between rounds is coprime to the list count."""

import json
import math
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "chunked_weight_layers_b200", "csrc")

HARNESS = r"""
#include "inplace_tc.cu"
#include <cstdio>
int main() {
  using namespace ttt;
  struct Case { int lists, tm, d, f, C, au, tg; } cases[] = {
      {148, 128, 2560, 9728, 1024, 1, 0}, {148, 128, 2560, 9728, 1024, 1, 1}, {148, 128, 2560, 9728, 1024, 0, 1},
      {148, 128, 200, 328, 128, 1, 0},    {148, 128, 392, 520, 256, 1, 1},    {148, 128, 256, 256, 128, 1, 0},
      {74, 256, 2560, 9728, 1024, 1, 0},  {74, 256, 2560, 9728, 1024, 1, 1},  {74, 256, 2560, 9728, 1024, 0, 1},
      {72, 256, 512, 328, 256, 1, 1},     {74, 256, 256, 256, 512, 1, 0}};
  printf("[");
  bool first = true;
  for (const Case& c : cases) {
    Plan p = make_plan(c.lists, c.tm, c.d, c.f, c.C, c.au != 0, c.tg != 0);
    printf("%s{\"lists\":%d,\"tm\":%d,\"d\":%d,\"f\":%d,\"C\":%d,\"au\":%d,\"tg\":%d,\"grid\":%d,"
           "\"rotate\":%d,\"plan\":[",
           first ? "" : ",", c.lists, c.tm, c.d, c.f, c.C, c.au, c.tg, p.grid, list_rotation(p.grid));
    for (size_t i = 0; i < p.host.size(); ++i) printf("%s%d", i ? "," : "", p.host[i]);
    printf("]}");
    first = false;
  }
  printf("]\n");
  return 0;
}
"""

APPLY, UPDATE, TARGET = 0, 1, 2


@pytest.fixture(scope="module")
def plans(tmp_path_factory):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not available")
    from chunked_weight_layers_b200 import build
    lib = build.build()
    d = tmp_path_factory.mktemp("plan")
    src = d / "plan_main.cu"
    src.write_text(HARNESS)
    exe = d / "plan_main"
    libdir = os.path.dirname(lib)
    subprocess.run([nvcc, "-std=c++17", "-O1", "-gencode", "arch=compute_100a,code=sm_100a", "-I", CSRC, "-I",
                    os.path.join(ROOT, "include"), str(src), "-o", str(exe), "-L", libdir, "-lttt",
                    f"-Xlinker=-rpath,{libdir}"], check=True, capture_output=True, timeout=600)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True, timeout=60).stdout
    return json.loads(out)


def _cost(code, c):
    t = (code >> 28) & 3
    if t == APPLY:
        return (c["f"] + 63) // 64 + 2
    if t == UPDATE:
        return max(c["C"] // 64, 20)
    return (c["d"] + 63) // 64 + 2


def test_every_tile_once_balanced_and_ordered(plans):
    for c in plans:
        grid, plan = c["grid"], c["plan"]
        offs, codes = plan[:grid + 1], plan[grid + 1:]
        assert offs[0] == 0 and offs[-1] == len(codes)
        tm = c["tm"]
        mt_tok, nt_d = c["C"] // tm, (c["d"] + 255) // 256
        want = set()
        if c["au"]:
            want |= {(APPLY << 28) | (m << 14) | n for m in range(mt_tok) for n in range(nt_d)}
            want |= {(UPDATE << 28) | (m << 14) | n for m in range((c["d"] + tm - 1) // tm)
                     for n in range((c["f"] + 255) // 256)}
        if c["tg"]:
            want |= {(TARGET << 28) | (m << 14) | n for m in range(mt_tok) for n in range(nt_d)}
        assert sorted(codes) == sorted(want) and len(codes) == len(want), c
        assert grid == min(c["lists"], len(want))
        rot = c["rotate"]
        assert math.gcd(rot, grid) == 1 and (grid < 4 or 2 * rot >= grid - 4), (grid, rot)
        loads = []
        for i in range(grid):
            lst = codes[offs[i]:offs[i + 1]]
            order = [{TARGET: 0, UPDATE: 1, APPLY: 2}[(x >> 28) & 3] for x in lst]
            assert order == sorted(order), (c["d"], c["f"], i)
            loads.append(sum(_cost(x, c) for x in lst))
        if len(want) >= 4 * grid:  # enough tiles for the longest-first assignment to even out
            assert max(loads) <= 1.1 * (sum(loads) / grid), (c["d"], c["f"], max(loads), sum(loads) / grid)
