"""The shared-memory layout of the 64x64 tile transposes (tile_chunk in
csrc/tile_transpose.cuh), run on the host: the header is compiled by nvcc
into a small host program that walks both phases of the kernel's thread
mapping.  It checks that the layout is a bijection onto the 8 KB tile, that
a load-phase store and a store-phase load address the same element, and that
no warp access has a bank conflict beyond the minimum for its size."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "sparse_moe_layer_limited_b200", "csrc")

PROGRAM = r"""
#include <cstdio>
#include <set>
#include <map>
#include "tile_transpose.cuh"
using moe::tile_chunk;
// byte address of element (source row i, feature c) as the load phase writes it
static unsigned put_addr(int i, int c) { return tile_chunk(c, i >> 3) + (i & 7) * 2; }
int main() {
  int bad = 0;
  std::set<unsigned> seen;
  for (int i = 0; i < 64; ++i)
    for (int c = 0; c < 64; ++c) {
      unsigned a = put_addr(i, c);
      if (a >= 8192 || !seen.insert(a).second) ++bad;
    }
  // the store phase reads destination row c, columns 8q..8q+7 as one 16-byte chunk
  for (int c = 0; c < 64; ++c)
    for (int q = 0; q < 8; ++q)
      for (int k = 0; k < 8; ++k)
        if (tile_chunk(c, q) + 2 * k != put_addr(8 * q + k, c)) ++bad;
  // bank conflicts: 256 threads, two items each; a warp's 32 lanes per access
  int worst_put = 0, worst_get = 0;
  for (int w = 0; w < 8; ++w)
    for (int rep = 0; rep < 2; ++rep) {
      for (int e = 0; e < 8; ++e) {   // load phase: 2-byte stores of feature 8p+e
        std::map<int, std::set<unsigned>> banks;
        for (int lane = 0; lane < 32; ++lane) {
          int it = w * 32 + lane + rep * 256, i = it >> 3, p = it & 7;
          unsigned word = put_addr(i, 8 * p + e) / 4;
          banks[word % 32].insert(word);
        }
        for (auto& b : banks) if ((int)b.second.size() > worst_put) worst_put = b.second.size();
      }
      std::map<int, std::set<unsigned>> banks;   // store phase: 16-byte loads
      for (int lane = 0; lane < 32; ++lane) {
        int it = w * 32 + lane + rep * 256, c = it >> 3, q = it & 7;
        for (int j = 0; j < 4; ++j) {
          unsigned word = tile_chunk(c, q) / 4 + j;
          banks[word % 32].insert(word);
        }
      }
      for (auto& b : banks) if ((int)b.second.size() > worst_get) worst_get = b.second.size();
    }
  printf("%d %d %d\n", bad, worst_put, worst_get);
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("nvcc") is None, reason="nvcc not installed")
def test_tile_layout_is_a_conflict_free_bijection(tmp_path):
    src = tmp_path / "swizzle.cu"
    exe = tmp_path / "swizzle"
    src.write_text(PROGRAM)
    subprocess.run(["nvcc", "-std=c++17", "-I", CSRC, "-o", str(exe), str(src)], check=True,
                   capture_output=True, timeout=300)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True, timeout=60)
    bad, worst_put, worst_get = map(int, out.stdout.split())
    assert bad == 0
    assert worst_put == 1          # every 2-byte store of a warp in a distinct bank (or word)
    assert worst_get == 4          # 512 bytes per warp: four wavefronts, the minimum
