"""Residency policy of the tenant pager (csrc/dc_lru.h), checked on the CPU.

Frequently used tenants stay resident and long-tail ones are loaded on demand (page
"Delta-CoMe – 清华联合 OpenBMB 等高校开源的新型增量压缩算法", FAQ "多模型同机部署最该关注什么？").
The policy is least recently used over batches.  A small C++ program drives the header and
compares every plan with a plain Python model of the same rule (a free slot first, else the slot
whose tenant was used longest ago, never a tenant of the current batch), over random Zipf batches:
loads, victims, hit and miss counts and the resident set must agree step by step.
"""
import os
import shutil
import subprocess

import numpy as np
import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "tenant_mixed_precision_b200", "csrc")

DRIVER = r"""
#include "dc_lru.h"
#include <cstdio>
#include <vector>
// stdin: n_tenants n_slots n_batches, then per batch: k t_1 .. t_k (distinct tenants)
// stdout per batch: ok hits misses nloads (tenant slot evicted)* and the slot of every tenant
int main() {
  int nt, ns, nb;
  if (std::scanf("%d %d %d", &nt, &ns, &nb) != 3) return 2;
  DcLru lru(nt, ns);
  std::vector<DcLru::Load> loads;
  for (int b = 0; b < nb; ++b) {
    int k;
    if (std::scanf("%d", &k) != 1) return 2;
    std::vector<int32_t> d(k);
    for (int i = 0; i < k; ++i) std::scanf("%d", &d[i]);
    int64_t h = 0, m = 0;
    const bool ok = lru.plan(d, loads, h, m);
    std::printf("%d %lld %lld %zu", ok ? 1 : 0, (long long)h, (long long)m, loads.size());
    for (auto& L : loads) std::printf(" %d %d %d", L.tenant, L.slot, L.evicted);
    for (int t = 0; t < nt; ++t) std::printf(" %d", lru.slot_of(t));
    std::printf("\n");
  }
  return 0;
}
"""


class ModelLru:
    """The same rule written out in Python."""

    def __init__(self, nt, ns):
        self.slot_of = [-1] * nt
        self.stamp = [0] * nt
        self.tenant_in = [-1] * ns
        self.clock = 0

    def plan(self, distinct):
        if len(distinct) > len(self.tenant_in):
            return False, 0, 0, []
        self.clock += 1
        now = self.clock
        for t in distinct:
            self.stamp[t] = now
        hits = misses = 0
        loads = []
        for t in distinct:
            if self.slot_of[t] >= 0:
                hits += 1
                continue
            misses += 1
            free = [s for s, v in enumerate(self.tenant_in) if v < 0]
            if free:
                best = free[0]
            else:
                cands = [s for s, v in enumerate(self.tenant_in) if self.stamp[v] != now]
                best = min(cands, key=lambda s: (self.stamp[self.tenant_in[s]], s))
            v = self.tenant_in[best]
            if v >= 0:
                self.slot_of[v] = -1
            self.tenant_in[best] = t
            self.slot_of[t] = best
            loads.append((t, best, v))
        return True, hits, misses, loads


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_lru_policy_matches_the_rule(tmp_path):
    src, exe = tmp_path / "lru.cpp", tmp_path / "lru"
    src.write_text(DRIVER)
    r = subprocess.run(["g++", "-std=c++17", "-O1", "-I", CSRC, str(src), "-o", str(exe)], capture_output=True,
                       text=True)
    assert r.returncode == 0, r.stderr
    rng = np.random.default_rng(17)
    nt, ns, nb = 40, 9, 300
    p = np.arange(1, nt + 1, dtype=np.float64) ** -1.1
    p /= p.sum()
    batches = []
    for b in range(nb):
        T = int(rng.integers(1, 24))
        d = list(dict.fromkeys(int(x) for x in rng.choice(nt, size=T, p=p)))
        if b % 50 == 49:  # now and then a batch with more tenants than slots
            d = list(range(ns + 1))
        batches.append(d)
    inp = f"{nt} {ns} {nb}\n" + "\n".join(f"{len(d)} " + " ".join(map(str, d)) for d in batches) + "\n"
    r = subprocess.run([str(exe)], input=inp, capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    lines = r.stdout.strip().splitlines()
    assert len(lines) == nb
    model = ModelLru(nt, ns)
    total_h = total_m = 0
    for d, line in zip(batches, lines):
        f = list(map(int, line.split()))
        ok, h, m, nl = f[:4]
        loads = [tuple(f[4 + 3 * i: 7 + 3 * i]) for i in range(nl)]
        slots = f[4 + 3 * nl:]
        mok, mh, mm, mloads = model.plan(d)
        assert (bool(ok), h, m, loads) == (mok, mh, mm, mloads)
        assert slots == model.slot_of
        if ok:
            # every tenant of the batch is resident, in distinct slots, and no slot holds two tenants
            assert all(slots[t] >= 0 for t in d)
            res = [s for s in slots if s >= 0]
            assert len(res) == len(set(res)) <= ns
            total_h += h
            total_m += m
        else:
            assert (h, m, nl) == (0, 0, 0)
    assert total_h > 0 and total_m > 0
