"""The launchers' per-device setup (csrc/kda_once.h), compiled with g++ and run on the host.

Sixteen threads call it for four device ordinals at once.  Setup must run exactly once per
ordinal, every caller must get that ordinal's value, a failed setup must not be recorded (the
next call runs it again), and an ordinal outside the table runs setup on every call.
"""
import os
import shutil
import subprocess

import pytest

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                    "chunked_kda_prefill_b200", "csrc")

PROGRAM = r"""
#include <atomic>
#include <cstdio>
#include <thread>
#include <vector>
#include "kda_once.h"

int main() {
  kda::PerDevice st;
  std::atomic<int> runs[4] = {};
  std::atomic<int> bad{0};
  std::vector<std::thread> threads;
  for (int t = 0; t < 16; ++t) {
    threads.emplace_back([&, t] {
      for (int i = 0; i < 2000; ++i) {
        const int dev = (t + i) % 4;
        int v = -1;
        const int e = kda::once_per_device(st, dev, &v, [&](int d, int* out) {
          runs[d].fetch_add(1);
          std::this_thread::yield();
          *out = 100 + d;
          return 0;
        });
        if (e != 0 || v != 100 + dev) bad.fetch_add(1);
      }
    });
  }
  for (auto& th : threads) th.join();
  for (int d = 0; d < 4; ++d)
    if (runs[d].load() != 1) { std::printf("device %d set up %d times\n", d, runs[d].load()); return 1; }
  if (bad.load()) { std::printf("%d wrong results\n", bad.load()); return 1; }

  // a failed setup is not recorded: the next call runs it again and then caches
  kda::PerDevice st2;
  int calls = 0, v = 0;
  auto failing = [&](int, int* out) { ++calls; *out = 7; return calls == 1 ? 3 : 0; };
  if (kda::once_per_device(st2, 5, &v, failing) != 3) return 2;
  if (kda::once_per_device(st2, 5, &v, failing) != 0 || v != 7 || calls != 2) return 3;
  if (kda::once_per_device(st2, 5, &v, failing) != 0 || v != 7 || calls != 2) return 4;

  // ordinals outside the table are never cached
  int outside = 0;
  for (int i = 0; i < 3; ++i)
    kda::once_per_device(st2, kda::kMaxDevices, &v, [&](int, int* out) { ++outside; *out = 1; return 0; });
  if (outside != 3) return 5;
  std::printf("ok\n");
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_once_per_device_threads(tmp_path):
    src = tmp_path / "once.cpp"
    exe = tmp_path / "once"
    src.write_text(PROGRAM)
    subprocess.run(["g++", "-std=c++17", "-O1", "-pthread", "-I", CSRC, str(src), "-o", str(exe)],
                   check=True, capture_output=True, text=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.strip() == "ok", (r.returncode, r.stdout, r.stderr)
