"""The activation-tile layouts of the tensor-core kernels, on the host (no
GPU): the closed forms the kernels store with (a per-lane base plus a
compile-time offset per column) must equal the layouts' definitions -- the
K order of the fragment registers (mma_k_position) placed in B-fragment
order (xtile_offset) for the mma.sync kernel, and the canonical K-major
position of the permuted column for the tcgen05 kernel -- for every row,
lane and column, and each tile must be filled exactly once.  The kernel
headers' __host__ __device__ functions are compiled into a small host
program with nvcc."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "bit_gemv_bcq_b200", "csrc")

PROGRAM = r'''
#include <cstdio>
#include <cstdint>
#include <vector>
namespace bcq {
// (the tile stores' group sums use the kernels' fp16 unpacking, defined by
// the translation unit that includes these headers; not called here)
__device__ __forceinline__ void unpack8(const uint4&, float (&)[8]) {}
}
#include "bcq_mma.cuh"
#include "bcq_umma.cuh"
using namespace bcq;

// tcgen05 tile: column 8l + e8 of the K-block -> byte offset in row n's slice
static uint32_t umma_definition(int NN, int n, int l, int e8) {
  const int h = l >> 4, U = (l >> 2) & 3, t = 8 * (l & 3) + e8;
  const int bt = (t & ~7) | ((t + 7) & 7);
  const int e = bt >> 4;
  const int s = (e ? 31 : 15) - bt;
  const int j = 2 * (64 * h + 16 * U + s) + e;
  return (uint32_t)((n >> 3) * 128 + (n & 7) * 16 + (j >> 3) * (NN * 16) + (j & 7) * 2);
}
template <int NN>
static int check_umma() {
  int bad = 0;
  std::vector<int> seen(NN * 256, 0);
  for (int n = 0; n < NN; ++n)
    for (int l = 0; l < 32; ++l)
      for (int e8 = 0; e8 < 8; ++e8) {
        const int h = l >> 4, U = (l >> 2) & 3, e = (l >> 1) & 1;
        const uint32_t base = (uint32_t)((n >> 3) * 128 + (n & 7) * 16) +
                              (uint32_t)((16 * h + 4 * U) * NN * 16 + e * 2) -
                              (uint32_t)(l & 1) * (32u * NN);
        const uint32_t off = base + umma_xtile_col_off<NN>(e8);
        bad += off != umma_definition(NN, n, l, e8);
        if (off % 2 == 0 && off / 2 < (uint32_t)(NN * 256)) seen[off / 2]++;
        else ++bad;
      }
  for (int c : seen) bad += c != 1;
  return bad;
}
int main() {
  int bad = 0;
  std::vector<int> seen(16 * 256, 0);
  for (int n = 0; n < 16; ++n)
    for (int l = 0; l < 32; ++l)
      for (int e8 = 0; e8 < 8; ++e8) {
        const int h = l >> 4, U = (l >> 2) & 3, e = (l >> 1) & 1;
        const uint32_t base =
            (uint32_t)(((((h * 4 + U) * 2 + (n >> 3)) * 32 + (n & 7) * 4) * 16) + e * 2) -
            8u * (uint32_t)(l & 1);
        const uint32_t off = base + xtile_col_off(e8);
        bad += off != xtile_offset(n, mma_k_position(l * 8 + e8));
        if (off % 2 == 0 && off / 2 < 16u * 256u) seen[off / 2]++;
        else ++bad;
      }
  for (int c : seen) bad += c != 1;
  // the K order is a permutation of the K-block's 256 columns
  std::vector<int> kseen(256, 0);
  for (int c = 0; c < 256; ++c) kseen[mma_k_position(c)]++;
  for (int c : kseen) bad += c != 1;
  bad += check_umma<16>() + check_umma<64>();
  std::printf("mismatches %d\n", bad);
  return bad != 0;
}
'''


@pytest.mark.skipif(shutil.which(os.environ.get("NVCC", "nvcc")) is None, reason="no nvcc")
def test_tile_closed_forms_match_their_definitions(tmp_path):
    src = tmp_path / "layout_check.cu"
    src.write_text(PROGRAM)
    exe = tmp_path / "layout_check"
    nvcc = os.environ.get("NVCC", "nvcc")
    subprocess.run([nvcc, "-std=c++17", "--expt-relaxed-constexpr", "-gencode",
                    "arch=compute_100a,code=sm_100a", "-I", os.path.join(ROOT, "include"), "-I", CSRC,
                    str(src), "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, out.stdout + out.stderr
    assert "mismatches 0" in out.stdout
