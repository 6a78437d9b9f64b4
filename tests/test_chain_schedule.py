"""The tile queue of the one-launch FFN side (csrc/ffn_chain.cuh), on the CPU.

The kernel's progress argument rests on properties of the queue, checked
here on the header's own functions (compiled by nvcc into a host program):
every output tile of the three GEMMs appears exactly once; every tile that a
tile waits for -- the out-projection tiles of its group before an FFN-up
tile, the FFN-up tiles of its group before an FFN-down tile, and the FFN-down
tiles of the group that last used a scratch slot before the slot is written
again -- comes earlier in the queue, so the smallest unfinished tile never
waits; and, along the queue, the groups each kind of tile waits for never
decrease, which is what lets a CTA skip a wait for a group it has already
seen complete.
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
#include <cstdlib>
#include <map>
#include <tuple>
#include <vector>
#include "ffn_chain.cuh"
using namespace bpt;
static int fail(const char* what, long long t) { std::printf("FAIL %s at %lld\n", what, t); return 1; }
int check(long long M, int h, int f, int gm, int hs, int us) {
  ChainArgs a{};
  a.M = M; a.h = h; a.f = f;
  a.m_tiles = (int)((M + 127) / 128);
  a.gm = gm;
  a.groups = (a.m_tiles + gm - 1) / gm;
  a.hid_slots = hs < a.groups ? hs : a.groups;
  a.u_slots = us < a.groups ? us : a.groups;
  a.n_op = (h + 255) / 256; a.n_up = (f + 255) / 256; a.n_dn = a.n_op;
  const long long n = chain_num_tiles(a);
  std::map<std::tuple<int, int, int>, long long> pos;  // (kind, M-tile, N-tile) -> queue index
  std::vector<long long> last(3 * (size_t)a.m_tiles, -1), first_dn_group(a.groups, -1), last_dn_group(a.groups, -1);
  std::vector<long long> first_op_group(a.groups, -1), first_up_group(a.groups, -1), first_up_mt(a.m_tiles, -1),
      first_dn_mt(a.m_tiles, -1);
  for (long long t = 0; t < n; ++t) {
    const ChainTile c = chain_tile(a, t);
    if (c.kind < 0 || c.kind > 2) return fail("kind", t);
    if (c.g < 0 || c.g >= a.groups || c.mt < 0 || c.mt >= chain_group_mt(a, c.g)) return fail("range", t);
    const int nmax = c.kind == CK_UP ? a.n_up : a.n_op;
    if (c.nt < 0 || c.nt >= nmax) return fail("nt", t);
    const int mtg = c.g * a.gm + c.mt;
    if (!pos.emplace(std::make_tuple(c.kind, mtg, c.nt), t).second) return fail("duplicate", t);
    long long& L = last[3 * (size_t)mtg + c.kind];
    if (t > L) L = t;
    if (c.kind == CK_DN) {
      if (last_dn_group[c.g] < t) last_dn_group[c.g] = t;
      if (first_dn_mt[mtg] < 0) first_dn_mt[mtg] = t;
    }
    if (c.kind == CK_UP) {
      if (first_up_mt[mtg] < 0) first_up_mt[mtg] = t;
      if (first_up_group[c.g] < 0) first_up_group[c.g] = t;
    }
    if (c.kind == CK_OP && first_op_group[c.g] < 0) first_op_group[c.g] = t;
  }
  if ((long long)pos.size() != (long long)a.m_tiles * (a.n_op + a.n_up + a.n_dn)) return fail("count", n);
  for (int m = 0; m < a.m_tiles; ++m) {
    if (!(last[3 * (size_t)m + CK_OP] < first_up_mt[m])) return fail("UP before its OP tiles", m);
    if (!(last[3 * (size_t)m + CK_UP] < first_dn_mt[m])) return fail("DN before its UP tiles", m);
  }
  // group-level waits: the whole group's OP (UP) tiles precede its first UP (DN) tile
  std::vector<long long> last_op_g(a.groups, -1), last_up_g(a.groups, -1), first_dn_g(a.groups, -1);
  int need_op = -1, need_up = -1, need_dn = -1;  // groups waited for, in queue order
  for (long long t = 0; t < n; ++t) {
    const ChainTile c = chain_tile(a, t);
    if (c.kind == CK_OP) {
      last_op_g[c.g] = t;
      if (c.g >= a.hid_slots) { if (c.g - a.hid_slots < need_dn) return fail("DN wait decreases", t); need_dn = c.g - a.hid_slots; }
    } else if (c.kind == CK_UP) {
      last_up_g[c.g] = t;
      if (c.g < need_op) return fail("OP wait decreases", t);
      need_op = c.g;
      if (c.g >= a.u_slots) { if (c.g - a.u_slots < need_dn) return fail("DN wait decreases", t); need_dn = c.g - a.u_slots; }
    } else {
      if (first_dn_g[c.g] < 0) first_dn_g[c.g] = t;
      if (c.g < need_up) return fail("UP wait decreases", t);
      need_up = c.g;
    }
  }
  for (int g = 0; g < a.groups; ++g) {
    if (!(last_op_g[g] < first_up_group[g])) return fail("UP before its group's OP tiles", g);
    if (!(last_up_g[g] < first_dn_g[g])) return fail("DN before its group's UP tiles", g);
  }
  for (int g = 0; g < a.groups; ++g) {
    if (g >= a.hid_slots && !(last_dn_group[g - a.hid_slots] < first_op_group[g])) return fail("hid slot reuse", g);
    if (g >= a.u_slots && !(last_dn_group[g - a.u_slots] < first_up_group[g])) return fail("U slot reuse", g);
  }
  std::printf("ok M=%lld h=%d f=%d gm=%d tiles=%lld\n", M, h, f, gm, n);
  return 0;
}
int main() {
  int bad = 0;
  const long long Ms[] = {1, 127, 128, 1000, 2048, 2049, 4096, 8192, 16384 + 128, 32768, 65536 + 640};
  const int hs[] = {128, 256, 1024, 4096};
  const int gms[] = {1, 2, 4, 8, 16};
  for (long long M : Ms)
    for (int h : hs)
      for (int gm : gms) {
        if (M * (long long)h > (1LL << 29) && gm < 16) continue;  // keep the big cases few
        bad |= check(M, h, 4 * h, gm, CHAIN_HID_SLOTS, CHAIN_U_SLOTS);
        if (gm == 4) bad |= check(M, h, 192, gm, CHAIN_HID_SLOTS, CHAIN_U_SLOTS);
      }
  return bad;
}
"""


def test_chain_queue_is_complete_and_every_wait_points_backwards(tmp_path):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not available")
    src = tmp_path / "chain_schedule.cu"
    src.write_text(HARNESS)
    exe = tmp_path / "chain_schedule"
    r = subprocess.run([nvcc, "-std=c++17", "-O2", "-gencode", "arch=compute_100a,code=sm_100a", "-I", CSRC, "-I",
                        INCLUDE, "-o", str(exe), str(src)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr[-3000:]
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout[-3000:]
    assert "FAIL" not in r.stdout
