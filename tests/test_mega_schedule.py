"""The one-launch layer's hand-over from attention to the FFN side
(csrc/layer_mega.cuh), on the CPU.

The out-projection tiles of row group g wait until the group's counter reaches
4 x (the group's 128-row tiles) x heads; the attention epilogue raises the
counter of the group holding each warp's 32 rows once those rows of one head
are stored. Checked here on the headers' own functions (compiled by nvcc into
a host program): the work items cover every (sequence, head, query-tile pair)
exactly once, and every group receives exactly the count its tiles wait for --
no more (a wait released early would read rows not yet written) and no fewer (a
wait never released).
"""

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "blockwise_attn_ffn_bpt_b200", "csrc")
INCLUDE = os.path.join(ROOT, "include")

HARNESS = r"""
#include <cstdio>
#include <set>
#include <tuple>
#include <vector>
#include "layer_mega.cuh"
using namespace bpt;
int check(int b, int s, int heads, int gm) {
  AttnArgs a{};
  a.s = s; a.heads = heads; a.beta0 = 0; a.t_start = 0; a.t_len = s;
  a.n_pairs = (s + 2 * ATT_BM - 1) / (2 * ATT_BM);
  a.grp_rows = gm * 128;
  ChainArgs c{};
  c.M = (long long)b * s;
  c.m_tiles = (int)((c.M + 127) / 128);
  c.gm = gm;
  c.groups = (c.m_tiles + gm - 1) / gm;
  std::vector<long long> cnt(c.groups, 0);
  std::set<std::tuple<int, int, int>> seen;
  const int n_att = b * a.n_pairs * heads;
  for (int item = 0; item < n_att; ++item) {
    int beta, head, pair;
    mega_item_coords(a, item, beta, head, pair);
    if (beta < 0 || beta >= b || head < 0 || head >= heads || pair < 0 || pair >= a.n_pairs) {
      std::printf("FAIL range %d\n", item);
      return 1;
    }
    if (!seen.emplace(beta, head, pair).second) { std::printf("FAIL duplicate %d\n", item); return 1; }
    for (int q = 0; q < 2; ++q) {
      const int tq0 = pair * 2 * ATT_BM + q * ATT_BM;
      if (tq0 >= s) continue;  // the pair's second tile past the sequence: no rows, no epilogue
      for (int quarter = 0; quarter < 4; ++quarter) {
        const long long g = mega_warp_row(a, beta, tq0, quarter) / a.grp_rows;
        if (g < 0 || g >= c.groups) { std::printf("FAIL group %d\n", item); return 1; }
        ++cnt[g];
      }
    }
  }
  for (int g = 0; g < c.groups; ++g)
    if (cnt[g] != 4LL * chain_group_mt(c, g) * heads) {
      std::printf("FAIL count g=%d: %lld vs %lld\n", g, cnt[g], 4LL * chain_group_mt(c, g) * heads);
      return 1;
    }
  return 0;
}
int main() {
  const int cases[][4] = {{1, 32768, 32, 16}, {2, 4096, 2, 16}, {1, 1152, 4, 4}, {3, 384, 2, 1}, {2, 1280, 3, 4},
                          {1, 8192, 16, 16}, {4, 128, 5, 2}, {2, 2176, 1, 8}};
  for (const auto& k : cases)
    if (check(k[0], k[1], k[2], k[3])) { std::printf("case b=%d s=%d heads=%d gm=%d\n", k[0], k[1], k[2], k[3]); return 1; }
  std::printf("OK\n");
  return 0;
}
"""


def nvcc():
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    return None


def test_attention_counts_match_what_the_ffn_tiles_wait_for(tmp_path):
    exe = nvcc()
    if exe is None:
        pytest.skip("nvcc not available")
    src = tmp_path / "mega_schedule.cu"
    src.write_text(HARNESS)
    out = tmp_path / "mega_schedule"
    r = subprocess.run([exe, "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-I", CSRC, "-I", INCLUDE,
                        "-o", str(out), str(src)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr[-2000:]
    run = subprocess.run([str(out)], capture_output=True, text=True)
    assert run.returncode == 0 and run.stdout.strip().endswith("OK"), run.stdout + run.stderr
