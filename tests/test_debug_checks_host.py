"""The debug build's bounds predicates (csrc/debug_checks.h) compiled as
plain C++ with the host compiler and run on a table of in- and out-of-range
accesses.  The GPU side of the debug build (the same predicates guarding
every TMA copy and TMEM access of the real kernels) is covered by
tests/test_gpu_debug_build.py."""
import os
import shutil
import subprocess

import pytest

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                    "long_context_bidirectional_b200", "csrc")

PROGRAM = r'''
#include "debug_checks.h"
#include <cstdio>
using namespace b2a;
#define EXPECT(cond, want) do { if ((cond) != (want)) { std::printf("FAIL line %d\n", __LINE__); ++bad; } } while (0)
int main() {
  int bad = 0;
  // TMA box starts: x (fp16 elements) aligned to 16 bytes and inside the extent
  EXPECT(tma_coords_ok(0, 2, 128, 0, 32, 0, 256), true);
  EXPECT(tma_coords_ok(64, 2, 128, 31, 32, 255, 256), true);
  EXPECT(tma_coords_ok(128, 2, 128, 0, 32, 0, 256), false);   // x at the extent
  EXPECT(tma_coords_ok(4, 2, 128, 0, 32, 0, 256), false);     // 8 bytes: unaligned
  EXPECT(tma_coords_ok(8, 2, 128, 0, 32, 0, 256), true);      // 16 bytes
  EXPECT(tma_coords_ok(2, 4, 128, 0, 32, 0, 256), false);     // fp32, 8 bytes
  EXPECT(tma_coords_ok(-8, 2, 128, 0, 32, 0, 256), false);
  EXPECT(tma_coords_ok(0, 2, 128, 32, 32, 0, 256), false);    // head past H
  EXPECT(tma_coords_ok(0, 2, 128, -1, 32, 0, 256), false);
  EXPECT(tma_coords_ok(0, 2, 128, 0, 32, 256, 256), false);   // row past the launch's rows
  EXPECT(tma_coords_ok(0, 2, 128, 0, 32, -128, 256), false);
  EXPECT(tma_coords_ok(0, 2, 4096, 0, 1, 32767, 32768), true);
  // shared-memory destination
  EXPECT(smem_box_ok(1024, 16384, 1024, 200 * 1024), true);
  EXPECT(smem_box_ok(1024 + 200 * 1024 - 16384, 16384, 1024, 200 * 1024), true);
  EXPECT(smem_box_ok(1024 + 200 * 1024 - 16384 + 128, 16384, 1024, 200 * 1024), false);
  EXPECT(smem_box_ok(512, 16384, 1024, 200 * 1024), false);   // below the base
  EXPECT(smem_box_ok(1024 + 64, 128, 1024, 200 * 1024), false);  // not 128-byte aligned
  // tcgen05.ld / st: lane field of the warp's quarter, columns inside 512
  EXPECT(tmem_ldst_ok((32u << 16) | 480u, 32, 1), true);
  EXPECT(tmem_ldst_ok((32u << 16) | 481u, 32, 1), false);
  EXPECT(tmem_ldst_ok((64u << 16) | 0u, 32, 1), false);       // another quarter's lanes
  EXPECT(tmem_ldst_ok((96u << 16) | 496u, 16, 3), true);
  // MMA operands: lane 0, columns inside 512
  EXPECT(tmem_operand_ok(384u, 128), true);
  EXPECT(tmem_operand_ok(385u, 128), false);
  EXPECT(tmem_operand_ok((32u << 16) | 0u, 128), false);
  EXPECT(tmem_operand_ok(504u, 8), true);
  EXPECT(tmem_operand_ok(505u, 8), false);
  EXPECT(idesc_n((256u >> 3) << 17), 256);
  EXPECT(idesc_n(((128u >> 3) << 17) | (16u << 24) | (1u << 4)), 128);
  std::printf("%d failed\n", bad);
  return bad != 0;
}
'''


def test_debug_predicates_on_the_cpu(tmp_path):
    cxx = shutil.which("g++") or shutil.which("c++")
    if cxx is None:
        pytest.skip("no host C++ compiler")
    src = tmp_path / "checks.cpp"
    src.write_text(PROGRAM)
    exe = tmp_path / "checks"
    subprocess.run([cxx, "-std=c++17", "-O1", f"-I{CSRC}", str(src), "-o", str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stdout
