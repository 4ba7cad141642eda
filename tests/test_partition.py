"""Host check of the split of a call's tiles over the persistent CTAs (``tile_begin`` /
``cta_of_tile`` / ``max_records_per_unit`` in ``csrc/lowram_internal.cuh``, host-and-device
functions), compiled for the host with nvcc and run here over every (tiles, CTAs) pair up to
a few hundred, with units of every size the kernels meet.

What the attend and combine kernels rely on:
* every tile belongs to exactly one CTA, and ``cta_of_tile`` names it;
* no CTA with no tile sits between two CTAs that hold tiles (the combine reads the piece
  records of the CTA range ``cta_of_tile(first) .. cta_of_tile(last)`` of a unit, and a CTA
  without tiles writes no record);
* for the fixed-k layout (k tiles per unit, tiles >= CTAs), a unit's tiles touch at most
  ``max_records_per_unit`` CTAs.
"""

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "kv_cache_compression_lowram_b200", "csrc")

PROGRAM = r"""
#include <cstdio>
#include "lowram_internal.cuh"
using namespace lowram;
int main() {
  long long checked = 0;
  for (int P = 1; P <= 300; ++P)
    for (long long total = 0; total <= 700; ++total) {
      if (tile_begin(total, P, 0) != 0 || tile_begin(total, P, P) != total) { printf("ends %d %lld\n", P, total); return 1; }
      for (int c = 0; c < P; ++c)
        if (tile_begin(total, P, c) > tile_begin(total, P, c + 1)) { printf("order %d %lld\n", P, total); return 1; }
      for (long long x = 0; x < total; ++x) {
        const int c = cta_of_tile(total, P, x);
        if (c < 0 || c >= P || tile_begin(total, P, c) > x || x >= tile_begin(total, P, c + 1)) {
          printf("owner %d %lld %lld\n", P, total, x);
          return 1;
        }
      }
      const int last = total ? cta_of_tile(total, P, total - 1) : -1;
      for (int c = 0; c <= last; ++c)
        if (tile_begin(total, P, c) == tile_begin(total, P, c + 1)) { printf("gap %d %lld %d\n", P, total, c); return 1; }
      for (int k = 1; k <= 32 && total >= P; ++k) {
        if (total % k) continue;
        for (long long u = 0; u < total / k; ++u) {
          const int n = cta_of_tile(total, P, (u + 1) * k - 1) - cta_of_tile(total, P, u * k) + 1;
          if (n > max_records_per_unit(total, P, k)) { printf("records %d %lld %d\n", P, total, k); return 1; }
        }
      }
      ++checked;
    }
  printf("ok %lld\n", checked);
  return 0;
}
"""


def _nvcc():
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    return None


@pytest.mark.skipif(_nvcc() is None, reason="nvcc not found")
def test_tile_partition_invariants(tmp_path):
    src = tmp_path / "partition.cu"
    src.write_text(PROGRAM)
    exe = tmp_path / "partition"
    inc = os.path.join(ROOT, "include")
    subprocess.run([_nvcc(), "-std=c++17", "-O2", "-I", inc, "-I", CSRC, str(src), "-o", str(exe)],
                   check=True, capture_output=True)
    res = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert res.returncode == 0 and res.stdout.startswith("ok"), res.stdout + res.stderr
