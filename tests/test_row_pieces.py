"""The split of a run of flat rows into attention launches
(csrc/row_pieces.h), on the CPU.

The host-memory entry runs attention wave by wave, one launch per piece of a
wave's rows: whole sequences, or one sequence's run of positions. Checked
here on the header's own function, compiled by g++ into a host program, for
every run of rows of several small batches: the pieces come in row order,
cover the run exactly once, stay inside the batch, never hold a partial
sequence together with another sequence, and merge consecutive whole
sequences into one piece (at most three pieces per run).
"""

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "blockwise_attn_ffn_bpt_b200", "csrc")

HARNESS = r"""
#include <cstdio>
#include <vector>
#include "row_pieces.h"
using namespace bpt;
static int fail(const char* what, int b, int s, long long r0, long long m) {
  std::printf("FAIL %s b=%d s=%d r0=%lld m=%lld\n", what, b, s, r0, m);
  return 1;
}
int check(int b, int s, long long r0, long long m) {
  std::vector<RowPiece> ps;
  const int st = for_each_row_piece(r0, m, b, s, [&](const RowPiece& p) { ps.push_back(p); return 0; });
  if (st != 0) return fail("status", b, s, r0, m);
  long long at = r0;
  int whole_runs = 0;
  for (size_t i = 0; i < ps.size(); ++i) {
    const RowPiece& p = ps[i];
    if (p.n_seq < 1 || p.t_len < 1 || p.beta < 0 || p.beta + p.n_seq > b) return fail("range", b, s, r0, m);
    if (p.t_start < 0 || p.t_start + p.t_len > s) return fail("positions", b, s, r0, m);
    if (p.n_seq > 1 && (p.t_start != 0 || p.t_len != s)) return fail("partial with others", b, s, r0, m);
    if ((long long)p.beta * s + p.t_start != at) return fail("order", b, s, r0, m);
    const bool whole = p.t_start == 0 && p.t_len == s;
    if (whole) {
      if (i > 0 && ps[i - 1].t_start == 0 && ps[i - 1].t_len == s) return fail("unmerged", b, s, r0, m);
      ++whole_runs;
    }
    at += (long long)p.n_seq * p.t_len;
  }
  if (at != r0 + m) return fail("cover", b, s, r0, m);
  if (ps.size() > 3 || whole_runs > 1) return fail("count", b, s, r0, m);
  // a stopping callback ends the walk with its status
  int calls = 0;
  const int st2 = for_each_row_piece(r0, m, b, s, [&](const RowPiece&) { return ++calls == 1 ? 7 : 0; });
  if (m > 0 && (st2 != 7 || calls != 1)) return fail("stop", b, s, r0, m);
  return 0;
}
int main() {
  long long runs = 0;
  const int ss[] = {1, 2, 7, 128, 130};
  for (int b = 1; b <= 5; ++b)
    for (int s : ss) {
      const long long tok = (long long)b * s;
      for (long long r0 = 0; r0 <= tok; ++r0)
        for (long long m = 0; r0 + m <= tok; ++m) {
          if (check(b, s, r0, m)) return 1;
          ++runs;
        }
    }
  std::printf("OK %lld\n", runs);
  return 0;
}
"""


def test_row_pieces_cover_each_run_once_in_order(tmp_path):
    cxx = shutil.which("g++") or shutil.which("c++")
    if cxx is None:
        pytest.skip("no C++ compiler")
    src = tmp_path / "pieces.cpp"
    src.write_text(HARNESS)
    exe = tmp_path / "pieces"
    r = subprocess.run([cxx, "-std=c++17", "-O1", "-I", CSRC, str(src), "-o", str(exe)], capture_output=True,
                       text=True)
    assert r.returncode == 0, r.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0 and run.stdout.startswith("OK"), run.stdout + run.stderr
