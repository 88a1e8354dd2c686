"""Host helpers of the library (csrc/host_common.h), compiled with the host
C++ compiler.  The once-per-device set-up, driven from many threads: every
device's set-up runs exactly once however many threads race for it, what the
set-up wrote is visible to every caller that returns, and a failed set-up is
retried rather than cached.  The size and overlap checks the entry points run
before any launch: half-open byte ranges, strided extents, and the 2^48-byte
bound at its edge and far beyond it."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "nvfp4_w4a4_quantized_09_b200", "csrc")
INCLUDE = os.path.join(ROOT, "include")
CUDA_INCLUDE = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "include")

PROGRAM = r"""
#include "host_common.h"

#include <chrono>
#include <cstdio>
#include <thread>
#include <vector>

using nvfp4::PerDeviceOnce;

int main() {
    constexpr int kDevs = 8, kThreads = 16, kRounds = 2000;
    static PerDeviceOnce once;
    static std::atomic<int> calls[kDevs];
    static long payload[kDevs];              // written by the set-up, not atomic
    std::atomic<int> bad{0};
    std::vector<std::thread> pool;
    for (int t = 0; t < kThreads; ++t) {
        pool.emplace_back([&, t] {
            for (int r = 0; r < kRounds; ++r) {
                const int dev = (r + t) % kDevs;
                const nvfp4_status st = once.run(dev, [&] {
                    calls[dev].fetch_add(1);
                    std::this_thread::sleep_for(std::chrono::microseconds(300));
                    payload[dev] = 1000 + dev;
                    return NVFP4_OK;
                });
                if (st != NVFP4_OK || payload[dev] != 1000 + dev) bad.fetch_add(1);
            }
        });
    }
    for (auto& th : pool) th.join();
    for (int d = 0; d < kDevs; ++d)
        if (calls[d].load() != 1) { std::printf("device %d set up %d times\n", d, calls[d].load()); return 1; }
    if (bad.load()) { std::printf("%d callers saw a missing set-up\n", bad.load()); return 2; }

    // a failure is reported and not cached; the first success is
    PerDeviceOnce retry;
    int n = 0;
    if (retry.run(3, [&] { ++n; return NVFP4_ERR_CUDA; }) != NVFP4_ERR_CUDA) return 3;
    if (retry.run(3, [&] { ++n; return NVFP4_ERR_CUDA; }) != NVFP4_ERR_CUDA) return 4;
    if (retry.run(3, [&] { ++n; return NVFP4_OK; }) != NVFP4_OK) return 5;
    if (retry.run(3, [&] { ++n; return NVFP4_ERR_CUDA; }) != NVFP4_OK) return 6;
    if (n != 3) return 7;
    // devices are independent
    if (retry.run(4, [&] { ++n; return NVFP4_OK; }) != NVFP4_OK || n != 4) return 8;
    std::printf("ok\n");
    return 0;
}
"""


@pytest.mark.skipif(shutil.which("g++") is None or not os.path.exists(CUDA_INCLUDE),
                    reason="needs g++ and the CUDA headers")
def test_per_device_once_under_contention(tmp_path):
    src = tmp_path / "once.cpp"
    exe = tmp_path / "once"
    src.write_text(PROGRAM)
    subprocess.check_call(["g++", "-std=c++17", "-O2", "-pthread", "-I", CSRC, "-I", INCLUDE,
                           "-I", CUDA_INCLUDE, "-o", str(exe), str(src)])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, out.stdout + out.stderr
    assert out.stdout.strip() == "ok"


HELPERS = r"""
#include "host_common.h"
#include <cstdio>

using namespace nvfp4;

int main() {
    char buf[64];
    // half-open byte ranges: touching is not overlapping
    if (!overlaps(buf, 4, buf + 3, 4) || !overlaps(buf + 3, 4, buf, 4)) return 1;
    if (overlaps(buf, 4, buf + 4, 4) || overlaps(buf + 4, 4, buf, 4)) return 2;
    if (!overlaps(buf + 10, 4, buf, 64) || overlaps(nullptr, 4, buf, 64)) return 3;
    // bytes of a strided matrix: (rows - 1) * ld + cols elements
    if (extent_bytes(4, 64, 32, 2) != (3 * 64 + 32) * 2) return 4;
    if (extent_bytes(0, 64, 32, 2) != 0 || extent_bytes(4, 64, 0, 2) != 0) return 5;
    // 2^48-byte bound, checked without overflow even for huge operands
    if (extent_too_large(1, int64_t(1) << 47, 2)) return 6;           // exactly 2^48 bytes
    if (!extent_too_large(2, int64_t(1) << 47, 2)) return 7;
    if (!extent_too_large(int64_t(1) << 62, int64_t(1) << 62, 8)) return 8;
    if (extent_too_large(0, int64_t(1) << 62, 2) || extent_too_large(32768, 34816, 2)) return 9;
    std::printf("ok\n");
    return 0;
}
"""


@pytest.mark.skipif(shutil.which("g++") is None or not os.path.exists(CUDA_INCLUDE),
                    reason="needs g++ and the CUDA headers")
def test_size_and_overlap_helpers(tmp_path):
    src = tmp_path / "helpers.cpp"
    exe = tmp_path / "helpers"
    src.write_text(HELPERS)
    subprocess.check_call(["g++", "-std=c++17", "-O2", "-I", CSRC, "-I", INCLUDE,
                           "-I", CUDA_INCLUDE, "-o", str(exe), str(src)])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0 and out.stdout.strip() == "ok", (out.returncode, out.stdout, out.stderr)
