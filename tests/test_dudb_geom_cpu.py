"""Host logic of the fused dU/dB kernel's geometry (csrc/dudb.cu, dudb_geom),
checked on the CPU: a small host program that includes the kernel's source
(its device code is compiled for sm_100a and never launched) prints the chosen
block shape for a grid of layer shapes, and every choice must keep the
kernel's invariants -- every CTA owns at least one token tile and one feature
chunk, the accumulators fit in tensor memory, the pipeline in shared memory,
and the partial sums cost no more than the second read of dY they replace."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "bit_nf4_quantized_20_b200", "csrc")

HARNESS = r"""
#include "dudb.cu"
#include <cstdio>
namespace qlora {
cudaError_t ensure_smem_optin(const void *, int) { return cudaSuccess; }
}
int main() {
  long long T, N;
  int r;
  while (std::scanf("%lld %lld %d", &T, &N, &r) == 3) {
    qlora::DuDbGeom g;
    if (!qlora::dudb_geom(T, N, r, 148, g)) {
      std::printf("%lld %lld %d none\n", T, N, r);
      continue;
    }
    std::printf("%lld %lld %d %d %d %d %d %d %d %d %d %zu %zu\n", T, N, r, g.tt, g.nn, g.t_ranges, g.n_ranges,
                g.rb, g.stages, g.smem, g.tmem_cols, qlora::dudb_part_u_bytes(g, T, r),
                qlora::dudb_partials_bytes(g, T, N, r));
  }
  return 0;
}
"""

SHAPES = [(T, N, r) for T in (1, 16, 300, 513, 1300, 2048, 2500, 4096, 8192, 150000)
          for N in (64, 136, 1024, 3080, 4096, 4104, 8192, 14336, 22016)
          for r in (1, 8, 13, 16, 24, 32, 36, 64, 65, 128)]


@pytest.fixture(scope="module")
def geoms(tmp_path_factory):
    nvcc = os.environ.get("NVCC", "nvcc")
    if shutil.which(nvcc) is None:
        pytest.skip("nvcc not found")
    d = tmp_path_factory.mktemp("dudb_geom")
    src = d / "main.cu"
    src.write_text(HARNESS)
    exe = d / "geom"
    subprocess.run([nvcc, "-O2", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
                    "-I", CSRC, "-I", os.path.join(ROOT, "include"), "-o", str(exe), str(src), "-lcuda"],
                   check=True, capture_output=True)
    inp = "".join(f"{T} {N} {r}\n" for T, N, r in SHAPES)
    out = subprocess.run([str(exe)], input=inp, capture_output=True, text=True, check=True).stdout
    res = {}
    for line in out.splitlines():
        f = line.split()
        key = (int(f[0]), int(f[1]), int(f[2]))
        res[key] = None if f[3] == "none" else tuple(int(v) for v in f[3:])
    assert len(res) == len(SHAPES)
    return res


def test_every_geometry_keeps_the_kernel_invariants(geoms):
    found = 0
    for (T, N, r), g in geoms.items():
        if r > 64:
            assert g is None, (T, N, r)
            continue
        if g is None:
            continue
        found += 1
        tt, nn, t_ranges, n_ranges, rb, stages, smem, tmem, part_u, part_all = g
        t_tiles, n_chunks = -(-T // 128), -(-N // 128)
        assert rb == (16 if r <= 16 else 32 if r <= 32 else 64)
        assert 1 <= tt <= 8 and 1 <= nn <= 32
        # the last range of each kind is not empty
        assert t_ranges == -(-t_tiles // tt) and (t_ranges - 1) * tt < t_tiles
        assert n_ranges == -(-n_chunks // nn) and (n_ranges - 1) * nn < n_chunks
        # dU: 64 columns per token tile; dB: 2 rb per feature chunk (hi and lo stacked)
        assert tt * 64 + nn * 2 * rb <= tmem <= 512 and tmem >= 32 and tmem & (tmem - 1) == 0
        assert 2 <= stages <= 8 and smem <= 220 * 1024
        r4 = (r + 3) & ~3
        assert part_u == -(-(n_ranges * T * r4 * 4) // 256) * 256
        assert part_all == part_u + t_ranges * N * r4 * 4
        assert part_all <= T * N          # at most half of dY's bytes
    assert found > 100


def test_the_bench_shapes(geoms):
    # the 8B block at T = 4096, r = 16: gate/up, q/o/down, k/v
    assert geoms[(4096, 14336, 16)][:4] == (3, 9, 11, 13)
    assert geoms[(4096, 4096, 16)][:4] == (2, 4, 16, 8)
    assert geoms[(4096, 1024, 16)][:4] == (1, 2, 32, 4)
    # the 65B stack's rank 64 keeps the two-launch path (partials too large)
    assert geoms[(2048, 8192, 64)] is None and geoms[(2048, 22016, 64)] is None
