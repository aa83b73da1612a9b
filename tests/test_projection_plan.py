"""The output projection's split-mode work partition
(csrc/projection_plan.h, used by projection_kernel and its reduce kernel),
checked exhaustively on the host against brute-force ownership of every
unit: g++ compiles the header into a small checker (no GPU)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER_DIR = os.path.join(ROOT, "sparse_latent_attention_absorb_b200", "csrc")

CHECKER = r"""
#include <cstdio>
#include <vector>
#include "projection_plan.h"
using namespace mla;

// One (tiles, upt, C) case: returns the number of violations.
template <typename I>
static long check(I tiles, I upt, I C) {
  const I U = tiles * upt;
  long bad = 0;
  std::vector<I> owner(U);
  if (proj_unit_begin<I>(0, U, C) != 0 || proj_unit_begin<I>(C, U, C) != U) ++bad;
  for (I c = 0; c < C; ++c) {
    const I b0 = proj_unit_begin<I>(c, U, C), b1 = proj_unit_begin<I>(c + 1, U, C);
    if (b1 <= b0) ++bad;                                   // every CTA owns a unit (C <= U)
    if ((b1 - 1) / upt - b0 / upt > 1) ++bad;              // at most two tiles: segments 0 and 1
    for (I x = b0; x < b1; ++x) owner[x] = c;
  }
  for (I x = 0; x < U; ++x)
    if (proj_cta_of_unit<I>(x, U, C) != owner[x]) ++bad;   // the owner, from the formula
  for (I t = 0; t < tiles; ++t) {
    I lo, hi;
    proj_tile_ctas<I>(t, upt, U, C, &lo, &hi);
    if (lo != owner[t * upt] || hi != owner[t * upt + upt - 1]) ++bad;
    for (I c = lo; c <= hi; ++c) {
      // the tile's index among c's tiles, as the kernel numbers segments
      const I seg = t - proj_unit_begin<I>(c, U, C) / upt;
      if (seg != (I)proj_segment_of<I>(c, t, upt, U, C)) ++bad;
    }
  }
  return bad;
}

int main() {
  long bad = 0, cases = 0;
  const int sms[] = {132, 148, 160};
  for (int upt : {64, 256})
    for (int tiles = 1; tiles < 160; ++tiles)
      for (int sm : sms) {
        if (tiles >= sm) continue;                        // direct mode: one CTA per tile
        const long units = (long)tiles * upt;
        const int C = (int)(units < sm ? units : sm);     // the host's plan
        bad += check<int>(tiles, upt, C) + check<long long>(tiles, upt, C);
        ++cases;
        for (int Cx = tiles + 1; Cx <= 300 && Cx <= units; Cx += 7) {  // other CTA counts
          bad += check<int>(tiles, upt, Cx) + check<long long>(tiles, upt, Cx);
          ++cases;
        }
      }
  std::printf("%ld cases, %ld violations\n", cases, bad);
  return bad == 0 ? 0 : 1;
}
"""


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_projection_partition_is_exact(tmp_path):
    src = tmp_path / "plan_check.cpp"
    src.write_text(CHECKER)
    exe = tmp_path / "plan_check"
    subprocess.run(["g++", "-O2", "-std=c++17", "-I", HEADER_DIR, "-o", str(exe), str(src)], check=True)
    p = subprocess.run([str(exe)], capture_output=True, text=True, timeout=600)
    assert p.returncode == 0, p.stdout + p.stderr
    assert "0 violations" in p.stdout
