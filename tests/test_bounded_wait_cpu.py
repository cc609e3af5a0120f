"""The host-side wait with a limit (``helix_stream_wait`` and its poll loop), on a CPU-only host.

The poll loop is header-only C++ (``csrc/bounded_wait.h``) with the completion query as a template
argument. These tests compile a small driver with g++ and hand it fake queries: one that never
completes (the wait must give up with HELIX_ERR_TIMEOUT after about its limit, not hang), one that
completes after a few polls, and one that reports a failure. Nothing here touches a GPU.
"""

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

DRIVER = r"""
#include <chrono>
#include <cstdio>
#include "bounded_wait.h"
using helix::PollResult;
int main() {
  using clk = std::chrono::steady_clock;
  // never completes: must return HELIX_ERR_TIMEOUT once 200 ms have passed
  long polls = 0;
  auto t0 = clk::now();
  helix_status a = helix::poll_with_limit([&] { ++polls; return PollResult::kPending; }, 200000);
  double ms = std::chrono::duration<double, std::milli>(clk::now() - t0).count();
  // completes on the fifth poll
  int n = 0;
  helix_status b = helix::poll_with_limit([&] { return ++n >= 5 ? PollResult::kDone : PollResult::kPending; }, 1000000);
  // the awaited work failed
  helix_status c = helix::poll_with_limit([] { return PollResult::kError; }, 1000000);
  // a zero limit polls exactly once
  int m = 0;
  helix_status d = helix::poll_with_limit([&] { ++m; return PollResult::kPending; }, 0);
  std::printf("%d %.1f %ld %d %d %d %d %d\n", (int)a, ms, polls, (int)b, n, (int)c, (int)d, m);
  return 0;
}
"""


@pytest.fixture(scope="module")
def driver(tmp_path_factory):
    gxx = shutil.which("g++")
    if gxx is None:
        pytest.skip("g++ not found")
    d = tmp_path_factory.mktemp("bounded_wait")
    src = d / "driver.cpp"
    src.write_text(DRIVER)
    exe = d / "driver"
    r = subprocess.run([gxx, "-std=c++17", "-O2", "-Wall", "-Werror", "-pthread",
                        "-I", os.path.join(ROOT, "include"),
                        "-I", os.path.join(ROOT, "long_context_decode_helix_b200", "csrc"),
                        str(src), "-o", str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=30)
    assert out.returncode == 0, out.stderr
    return out.stdout.split()


def test_never_completing_query_times_out(driver):
    status, ms, polls = int(driver[0]), float(driver[1]), int(driver[2])
    assert status == 5  # HELIX_ERR_TIMEOUT
    assert 200.0 <= ms < 2000.0, ms  # gave up after the limit, not long after
    assert polls > 64  # kept polling (with sleeps) until then


def test_completion_and_failure(driver):
    assert int(driver[3]) == 0 and int(driver[4]) == 5  # HELIX_OK on the fifth poll
    assert int(driver[5]) == 4  # HELIX_ERR_CUDA when the query reports a failure
    assert int(driver[6]) == 5 and int(driver[7]) == 1  # a zero limit: one poll, then timeout


def test_stream_wait_rejects_a_null_event():
    import long_context_decode_helix_b200 as hx

    # checked before any CUDA call, so it holds on a host without a GPU too
    assert hx.lib.helix_stream_wait(None, None, 1000) == 1  # HELIX_ERR_INVALID_ARG
