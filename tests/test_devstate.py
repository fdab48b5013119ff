"""Per-device launch state of the serving library, checked on the CPU.

The SM count and each kernel's dynamic shared-memory limit belong to one device's context.  The
library keeps them in a table keyed by device index (csrc/dc_devstate.h).  This test compiles a
small C++ program against that header with fake query and setter functions and checks that:
every device gets its own attribute calls, a larger request raises the limit again, a failed
setter leaves nothing recorded, indexes out of range are refused, and concurrent threads on
several devices call the setter exactly once per (device, kernel).
"""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "tenant_mixed_precision_b200", "csrc")

PROGRAM = r"""
#include "dc_devstate.h"
#include <atomic>
#include <cstdio>
#include <thread>
#include <vector>

#define CHECK(c) do { if (!(c)) { std::printf("FAIL line %d: %s\n", __LINE__, #c); return 1; } } while (0)

int main() {
  DcDevState st;
  int calls = 0;
  auto ok = [&](size_t) { ++calls; return 0; };
  // device 0: first request sets, an equal or smaller one does not, a larger one sets again
  CHECK(st.ensure_smem(0, DC_K_UDELTA, 1000, ok) == 0 && calls == 1);
  CHECK(st.ensure_smem(0, DC_K_UDELTA, 1000, ok) == 0 && calls == 1);
  CHECK(st.ensure_smem(0, DC_K_UDELTA, 500, ok) == 0 && calls == 1);
  CHECK(st.ensure_smem(0, DC_K_UDELTA, 2000, ok) == 0 && calls == 2);
  CHECK(st.smem_limit(0, DC_K_UDELTA) == 2000);
  // device 1 is a different context: its first request sets the attribute there too
  CHECK(st.ensure_smem(1, DC_K_UDELTA, 1000, ok) == 0 && calls == 3);
  CHECK(st.smem_limit(1, DC_K_UDELTA) == 1000 && st.smem_limit(0, DC_K_UDELTA) == 2000);
  // another kernel on device 0 is independent
  CHECK(st.ensure_smem(0, DC_K_VSTAGE, 10, ok) == 0 && calls == 4);
  // a failed setter is reported and nothing is recorded
  auto bad = [&](size_t) { ++calls; return 98; };
  CHECK(st.ensure_smem(2, DC_K_BASE_TC, 4096, bad) == 98 && calls == 5);
  CHECK(st.smem_limit(2, DC_K_BASE_TC) == 0);
  CHECK(st.ensure_smem(2, DC_K_BASE_TC, 4096, ok) == 0 && calls == 6);
  // out of range
  CHECK(st.ensure_smem(-1, DC_K_BASE, 1, ok) == -1 && st.ensure_smem(DC_MAX_DEVICES, DC_K_BASE, 1, ok) == -1);
  CHECK(st.ensure_smem(0, DC_K_COUNT, 1, ok) == -1 && calls == 6);
  // SM count: queried once per device, a failed query is not kept
  int q = 0;
  CHECK(st.sm_count(0, [&](int d) { ++q; return 148 + d; }) == 148 && q == 1);
  CHECK(st.sm_count(0, [&](int d) { ++q; return 7; }) == 148 && q == 1);
  CHECK(st.sm_count(3, [&](int d) { ++q; return 0; }) == 148 && q == 2);
  CHECK(st.sm_count(3, [&](int d) { ++q; return 132; }) == 132 && q == 3);
  // threads on 4 devices: one setter call per (device, kernel)
  DcDevState st2;
  std::atomic<int> per_dev[4];
  for (auto& a : per_dev) a = 0;
  std::vector<std::thread> th;
  for (int t = 0; t < 16; ++t)
    th.emplace_back([&, t] {
      for (int i = 0; i < 1000; ++i) {
        const int d = (t + i) % 4;
        st2.ensure_smem(d, DC_K_UPRE, 200000, [&](size_t) { per_dev[d]++; return 0; });
      }
    });
  for (auto& x : th) x.join();
  for (int d = 0; d < 4; ++d) CHECK(per_dev[d] == 1 && st2.smem_limit(d, DC_K_UPRE) == 200000);
  std::printf("ok\n");
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_device_state_is_keyed_per_device(tmp_path):
    src = tmp_path / "devstate_check.cpp"
    exe = tmp_path / "devstate_check"
    src.write_text(PROGRAM)
    r = subprocess.run(["g++", "-std=c++17", "-O1", "-pthread", "-I", CSRC, str(src), "-o", str(exe)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stdout + r.stderr
