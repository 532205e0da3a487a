"""The item order of the fused pool-and-route kernel (csrc/fv_plan.h), on the CPU.

The kernel's waits end only because every item it waits on comes earlier in its queue.
A small C++ program built from the same header decodes every item index and checks,
for a range of slice and block counts:
* every (kind, slice, index) occurs exactly once, and the indices per kind and slice
  are 0 .. count - 1;
* each logits item of slice s comes after all pool items of s, and each select item
  of s after all logits items of s;
* the logits of slice s come after the pool items of slice s + 1, when it exists, so
  that the pool items they wait on had a slice's worth of items to finish in.
"""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "free_adaptive_block_b200", "csrc")

HARNESS = r"""
#include <cstdio>
#include <vector>
#include "fv_plan.h"

static int check(int S, int nB) {
  const fv::PrPlan pl = fv::pr_plan(S, nB);
  const int per[3] = {pl.nP, pl.nL, pl.nS};
  std::vector<std::vector<long long>> first(3, std::vector<long long>(S, -1)), last(3, std::vector<long long>(S, -1));
  std::vector<std::vector<int>> seen(3, std::vector<int>(S, 0));
  std::vector<std::vector<char>> hit;
  for (int k = 0; k < 3; ++k)
    for (int s = 0; s < S; ++s) hit.push_back(std::vector<char>(per[k], 0));
  for (long long t = 0; t < pl.total; ++t) {
    int kind = -1, slice = -1, idx = -1;
    fv::pr_decode(pl, t, kind, slice, idx);
    if (kind < 0 || kind > 2 || slice < 0 || slice >= S || idx < 0 || idx >= per[kind]) {
      std::printf("bad item %lld: kind %d slice %d idx %d (S %d nB %d)\n", t, kind, slice, idx, S, nB);
      return 1;
    }
    char& h = hit[kind * S + slice][idx];
    if (h) { std::printf("item twice: %d %d %d\n", kind, slice, idx); return 1; }
    h = 1;
    if (first[kind][slice] < 0) first[kind][slice] = t;
    last[kind][slice] = t;
    ++seen[kind][slice];
  }
  for (int k = 0; k < 3; ++k)
    for (int s = 0; s < S; ++s)
      if (seen[k][s] != per[k]) { std::printf("count %d %d: %d of %d\n", k, s, seen[k][s], per[k]); return 1; }
  for (int s = 0; s < S; ++s) {
    if (first[1][s] <= last[0][s]) { std::printf("logits before pool, slice %d\n", s); return 1; }
    if (first[2][s] <= last[1][s]) { std::printf("select before logits, slice %d\n", s); return 1; }
    if (s + 1 < S && first[1][s] <= last[0][s + 1]) { std::printf("no lag, slice %d\n", s); return 1; }
  }
  return 0;
}

int main() {
  const int Ss[] = {1, 2, 3, 4, 7, 12, 40, 257};
  const int nBs[] = {1, 8, 27, 63, 64, 65, 336, 630, 768};
  int bad = 0;
  for (int S : Ss)
    for (int nB : nBs) bad |= check(S, nB);
  // the item count of the 480p layer: 12 slices x (672 pool + 36 logits + 42 select)
  if (fv::pr_plan(12, 336).total != 12LL * (672 + 36 + 42)) { std::printf("480p total\n"); bad = 1; }
  std::printf(bad ? "FAIL\n" : "OK\n");
  return bad;
}
"""


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_item_order(tmp_path):
    src = tmp_path / "plan.cpp"
    src.write_text(HARNESS)
    exe = tmp_path / "plan"
    subprocess.run(["g++", "-std=c++17", "-O1", "-Wall", "-Werror", "-I", CSRC, str(src), "-o", str(exe)],
                   check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip().endswith("OK"), r.stdout[-2000:]
