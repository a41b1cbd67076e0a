"""Counter comparisons across the uint32 wrap (host-compiled, no GPU).

Dependency counters are never reset between steps: a wait's target is
epoch x arrivals, and both the counter and the target wrap around 2^32 after
enough steps.  The interpreter compares them by signed difference
(``reached`` and ``later`` in mk_internal.h).  This test compiles those two
functions on the host with g++ and walks a counter through steps that cross
the wrap, for several arrival counts, checking at every arrival that the wait
is met exactly when the step's last arrival lands.
"""

import os
import shutil
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "moe_persistent_cta_b200", "csrc")

PROGRAM = r"""
#include <cstdio>
#include "mk_internal.h"
using mk::reached;
using mk::later;
int main() {
  const uint32_t ns[] = {1u, 7u, 32u, 148u, 1187u, 65535u};
  int bad = 0;
  for (uint32_t n : ns) {
    // epochs around the point where epoch * n first wraps, and around the
    // wrap of the epoch itself
    const uint64_t wrap_epoch = (uint64_t(1) << 32) / n;
    const uint64_t starts[] = {1, wrap_epoch - 2, (uint64_t(1) << 32) - 3};
    for (uint64_t e0 : starts) {
      for (uint64_t e = e0; e < e0 + 5; ++e) {
        const uint32_t epoch = (uint32_t)e;               // the host's epoch wraps too
        const uint32_t target = epoch * n;
        uint32_t ctr = (uint32_t)(epoch - 1u) * n;       // value left by the previous step
        for (uint32_t i = 0; i < n; ++i) {
          if (reached(ctr, target)) { ++bad; std::printf("early n=%u e=%llu i=%u\n", n, (unsigned long long)e, i); }
          ++ctr;
        }
        if (!reached(ctr, target)) { ++bad; std::printf("missed n=%u e=%llu\n", n, (unsigned long long)e); }
        // the loader's cache: a later wait on the same counter for more
        // arrivals of the same step is not satisfied by the cached target
        if (n > 1 && !later(target, target - 1u)) ++bad;
        if (later(target, target)) ++bad;
        // the dispenser: taken indices relative to the step's base
        const uint32_t base = (uint32_t)(epoch - 1u) * (n + 3u);
        const uint32_t raw = base + 5u;
        if ((int)(raw - base) != 5) ++bad;
      }
    }
  }
  std::printf("bad=%d\n", bad);
  return bad != 0;
}
"""


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs a host C++ compiler")
def test_counter_comparisons_across_wrap():
    with tempfile.TemporaryDirectory() as d:
        src = os.path.join(d, "wrap.cpp")
        exe = os.path.join(d, "wrap")
        with open(src, "w") as f:
            f.write(PROGRAM)
        subprocess.run(["g++", "-std=c++17", "-O1", "-I", CSRC, "-I",
                        os.path.join(ROOT, "include"), src, "-o", exe], check=True)
        res = subprocess.run([exe], capture_output=True, text=True)
        assert res.returncode == 0, res.stdout + res.stderr
        assert "bad=0" in res.stdout


def test_unsigned_comparison_would_fail_at_the_wrap():
    """The plain unsigned test the interpreter used before fails right after
    epoch * n wraps: a planted-mistake check of the walk above."""
    n = 148
    epoch = (1 << 32) // n + 1                  # first epoch whose target wraps
    target = (epoch * n) & 0xFFFFFFFF
    start = ((epoch - 1) * n) & 0xFFFFFFFF      # counter at the start of the step
    assert start >= target                      # unsigned: the wait would pass at once
    diff = (start - target) & 0xFFFFFFFF
    assert diff >= 1 << 31                      # signed: still n arrivals short
