"""Work schedule of the tensor-core backbone (csrc/dc_btsched.h), checked on the CPU.

The kernel and the host planner share this header; a small C++ program drives it for many layer
shapes, batch sizes and CTA counts and checks what the kernel relies on:

* every chunk of every unit belongs to exactly one CTA's range, and the ranges tile the sequence;
* bt_seg_at maps each chunk to a unit (linear, row tile, token block) with the right K, and the
  unit ids are distinct per (linear, tile, token block) and below the workspace's counter count;
* the contributors of each unit are exactly c0, c0 + step, ..., c1 (bt_cta_of of its first and
  last chunk, step 1 or the team size), which is how the last contributor finds the partials;
* with teams, all CTAs of a team cover the same (tile, k) chunks for their own token blocks.
"""
import shutil
import subprocess

import numpy as np
import pytest

from test_pager_policy import CSRC

DRIVER = r"""
#include "dc_btsched.h"
#include <cstdio>
#include <map>
#include <set>
#include <tuple>
#include <vector>
struct Lin { int d_out, d_in; };
struct FakeF {
  Lin lin[8];
  int n_lin, fp8;
  int order[8], tile_prefix[9];
  int64_t bt_chunk_prefix[9], bt_total, bt_ctb;
  int bt_ntb, bt_grid, bt_team, bt_gtiles[8];
};
// stdin per case: n_lin fp8 T nb max_ctas, then n_lin pairs d_out d_in.  stdout per case: "ok ..."
// or the first violation.
int main() {
  int n_lin, fp8, T, nb, maxc;
  while (std::scanf("%d %d %d %d %d", &n_lin, &fp8, &T, &nb, &maxc) == 5) {
    FakeF F = {};
    F.n_lin = n_lin;
    F.fp8 = fp8;
    for (int p = 0; p < n_lin; ++p) std::scanf("%d %d", &F.lin[p].d_out, &F.lin[p].d_in);
    bt_plan_order(F);
    bt_plan(F, T, nb, maxc);
    const int kc = fp8 ? 128 : 64;
    const int step = F.bt_team ? F.bt_team : 1;
    int64_t max_dim = 0;
    for (int p = 0; p < n_lin; ++p) max_dim = std::max<int64_t>(max_dim, std::max(F.lin[p].d_out, F.lin[p].d_in));
    const int64_t units_cap = (int64_t)n_lin * (((max_dim + 127) / 128 * 128) / 128) * F.bt_ntb;
    std::map<std::tuple<int, int, int>, int> uid;                 // (slot, tile, tb) -> unit id
    std::map<int, std::set<int>> contrib;                          // unit -> CTAs
    std::map<int, std::pair<int64_t, int>> ustart;                 // unit -> (first chunk, K)
    std::map<int, std::set<std::tuple<int, int, int>>> team_cover;  // team -> (slot, tile, k)
    std::set<std::pair<int, int>> seen;                            // (unit, k)
    int64_t covered = 0, prev_end = 0;
    bool bad = false;
    auto fail = [&](const char* what, long long a, long long b) {
      if (!bad) std::printf("fail %s %lld %lld\n", what, a, b);
      bad = true;
    };
    for (int c = 0; c < F.bt_grid && !bad; ++c) {
      int64_t g0, g1;
      bt_range(F, c, g0, g1);
      if (g1 < g0) fail("range", c, 0);
      if (!F.bt_team && g0 != prev_end) fail("tiling", c, g0);
      prev_end = g1;
      for (int64_t g = g0; g < g1 && !bad;) {
        const BtSeg S = bt_seg_at(F, g, g1);
        const int p = F.order[S.slot];
        if (S.K != F.lin[p].d_in / kc) fail("K", S.slot, S.K);
        if (S.ot < 0 || S.ot >= F.lin[p].d_out / 128) fail("tile", S.slot, S.ot);
        if (S.tb < 0 || S.tb >= F.bt_ntb) fail("token block", S.slot, S.tb);
        if (S.u < 0 || S.u >= units_cap) fail("unit id", S.u, units_cap);
        if (S.k0 < 0 || S.k1 > S.K || S.k0 >= S.k1) fail("k range", S.k0, S.k1);
        if (S.ustart + S.k0 != g) fail("start", g, S.ustart);
        auto key = std::make_tuple(S.slot, S.ot, S.tb);
        auto it = uid.find(key);
        if (it == uid.end()) {
          for (auto& kv : uid)
            if (kv.second == S.u) fail("unit id reused", S.u, 0);
          uid[key] = S.u;
        } else if (it->second != S.u) {
          fail("unit id changes", it->second, S.u);
        }
        auto us = ustart.find(S.u);
        if (us == ustart.end()) ustart[S.u] = {S.ustart, S.K};
        else if (us->second.first != S.ustart) fail("unit start", S.u, S.ustart);
        for (int k = S.k0; k < S.k1; ++k) {
          if (!seen.insert({S.u, k}).second) fail("chunk twice", S.u, k);
          if (bt_cta_of(F, S.ustart + k) != c) fail("cta_of", c, S.ustart + k);
          if (F.bt_team) team_cover[c / F.bt_team].insert(std::make_tuple(S.slot, S.ot, k));
        }
        covered += S.k1 - S.k0;
        contrib[S.u].insert(c);
        g = S.ustart + S.k1;
      }
    }
    if (!bad && covered != F.bt_total) fail("coverage", covered, F.bt_total);
    int64_t want_units = 0;
    for (int p = 0; p < n_lin; ++p) want_units += (int64_t)(F.lin[p].d_out / 128) * F.bt_ntb;
    if (!bad && (int64_t)uid.size() != want_units) fail("units", uid.size(), want_units);
    int max_contrib = 0;
    for (auto& kv : contrib) {
      if (bad) break;
      const auto st = ustart[kv.first];
      const int c0 = bt_cta_of(F, st.first), c1 = bt_cta_of(F, st.first + st.second - 1);
      std::set<int> want;
      for (int c = c0; c <= c1; c += step) want.insert(c);
      if (want != kv.second) fail("contributors", kv.first, (long long)kv.second.size());
      if ((c1 - c0) % step) fail("contributor step", c0, c1);
      max_contrib = std::max<int>(max_contrib, (int)kv.second.size());
    }
    if (F.bt_team && !bad) {  // every team covers the same (slot, tile, k) set for each of its blocks
      std::map<int, std::map<std::tuple<int, int, int>, int>> cnt;
      for (int c = 0; c < F.bt_grid; ++c) {
        int64_t g0, g1;
        bt_range(F, c, g0, g1);
        for (int64_t g = g0; g < g1;) {
          const BtSeg S = bt_seg_at(F, g, g1);
          for (int k = S.k0; k < S.k1; ++k) cnt[c / F.bt_team][std::make_tuple(S.slot, S.ot, k)]++;
          g = S.ustart + S.k1;
        }
      }
      for (auto& t : cnt)
        for (auto& kv : t.second)
          if (kv.second != F.bt_team) fail("team in step", t.first, kv.second);
    }
    if (!bad)
      std::printf("ok team=%d grid=%d ntb=%d units=%zu max_contrib=%d\n", F.bt_team, F.bt_grid, F.bt_ntb, uid.size(),
                  max_contrib);
  }
  return 0;
}
"""

LLAMA7B = [(4096, 4096)] * 4 + [(11008, 4096)] * 2 + [(4096, 11008)]
LLAMA13B = [(5120, 5120)] * 4 + [(13824, 5120)] * 2 + [(5120, 13824)]


def _nb(T):
    """Token block of the backbone for a batch of T tokens (the workspace layout's rule)."""
    return max(16, -(-T // 16) * 16) if T <= 256 else 256


def _cases():
    rng = np.random.default_rng(5)
    out = [(LLAMA7B, 0, 64, 148), (LLAMA7B, 1, 64, 148), (LLAMA13B, 0, 2048, 148), (LLAMA13B, 1, 2048, 148),
           (LLAMA7B, 0, 257, 148), (LLAMA13B, 0, 4096, 132), ([(384, 640)], 0, 300, 148),
           ([(128, 1152)], 0, 1000, 148), ([(256, 256)] * 4 + [(384, 256)] * 2 + [(256, 384)], 0, 300, 148),
           ([(128, 128)], 0, 1, 148), ([(640, 256)], 0, 3, 148), ([(512, 512)], 0, 40000, 148)]
    for _ in range(40):
        n_lin = int(rng.choice([1, 7]))
        shapes = [(128 * int(rng.integers(1, 40)), 128 * int(rng.integers(1, 40))) for _ in range(n_lin)]
        fp8 = int(rng.integers(0, 2))
        T = int(rng.choice([1, 7, 16, 64, 200, 256, 257, 300, 777, 2048, 3000]))
        out.append((shapes, fp8, T, int(rng.choice([148, 132, 64, 17]))))
    return out


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_backbone_schedule_partitions(tmp_path):
    src, exe = tmp_path / "sched.cpp", tmp_path / "sched"
    src.write_text(DRIVER)
    r = subprocess.run(["g++", "-std=c++17", "-O2", "-I", CSRC, str(src), "-o", str(exe)], capture_output=True,
                       text=True)
    assert r.returncode == 0, r.stderr
    cases = _cases()
    inp = ""
    for shapes, fp8, T, maxc in cases:
        inp += f"{len(shapes)} {fp8} {T} {_nb(T)} {maxc} " + " ".join(f"{a} {b}" for a, b in shapes) + "\n"
    r = subprocess.run([str(exe)], input=inp, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr
    lines = r.stdout.strip().splitlines()
    assert len(lines) == len(cases)
    for case, line in zip(cases, lines):
        assert line.startswith("ok"), (case, line)
    # the prefill-sized batches ran in teams, the decode-sized ones in stream-K
    assert "team=8" in lines[2] and "team=0" in lines[0]
    assert "team=0" in lines[11]  # more token blocks than CTAs: stream-K
