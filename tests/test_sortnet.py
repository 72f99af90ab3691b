"""The gate's sorting networks (csrc/sortnet.cuh) checked on the host (CPU),
for unsigned and fp32 keys:
the header is compiled with g++ as plain C++ and run exhaustively by the
0-1 principle -- a comparator network sorts every input iff it sorts every
0/1 input -- for the 16-key odd-even merge sort (all 2^16 inputs), and for the top-16 merge of two descending
lists over every pair of 0/1 lists, plus random keys against std::sort; and
the fp32 selection keys: the float order where scores differ beyond their
low 8 mantissa bits, ties (including +0 / -0) to the lower block, and
agreement in the other bits only within 2^-15 relative (2^-141 absolute
among subnormals)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "long_context_prefill_block_b200", "csrc")

PROGRAM = r"""
#define __host__
#define __device__
#define __forceinline__ inline
#include <algorithm>
#include <cmath>
#include <cstdio>
#include <functional>
#include <random>
#include "sortnet.cuh"

using namespace moba::net;

template <typename K>
static bool sorted_desc(const K* v) {
  for (int i = 0; i + 1 < 16; ++i) if (v[i] < v[i + 1]) return false;
  return true;
}

template <typename K>
static int check_networks(std::mt19937& rng) {
  // 0-1 principle for the sort
  for (uint32_t m = 0; m < (1u << 16); ++m) {
    K v[16];
    for (int i = 0; i < 16; ++i) v[i] = (K)((m >> i) & 1u);
    oe_sort16(v);
    if (!sorted_desc(v)) { printf("sort fails on mask %u\n", m); return 1; }
  }
  // merge: every pair of descending 0/1 lists (a ones, then zeros)
  for (int a = 0; a <= 16; ++a)
    for (int b = 0; b <= 16; ++b) {
      K l[16], g[16];
      for (int i = 0; i < 16; ++i) { l[i] = (K)(i < a); g[i] = (K)(i < b); }
      merge_top16(l, g);
      int ones = std::min(16, a + b);
      for (int i = 0; i < 16; ++i)
        if (l[i] != (K)(i < ones)) { printf("merge fails a=%d b=%d\n", a, b); return 1; }
    }
  // random keys: the top 16 of 8 groups of 16 against std::sort
  for (int trial = 0; trial < 2000; ++trial) {
    K all[128], list[16];
    for (int i = 0; i < 128; ++i) all[i] = (K)(rng() % (trial % 3 == 0 ? 7u : 0xFFFFFFu));
    for (int gi = 0; gi < 8; ++gi) {
      K g[16];
      for (int i = 0; i < 16; ++i) g[i] = all[16 * gi + i];
      oe_sort16(g);
      if (gi == 0) for (int i = 0; i < 16; ++i) list[i] = g[i];
      else merge_top16(list, g);
    }
    std::sort(all, all + 128, std::greater<K>());
    for (int i = 0; i < 16; ++i)
      if (list[i] != all[i]) { printf("random trial %d fails at %d\n", trial, i); return 1; }
  }
  return 0;
}

int main() {
  std::mt19937 rng(12345);
  if (check_networks<uint32_t>(rng)) return 1;
  if (check_networks<float>(rng)) return 1;
  // order keys: larger key = larger score; equal scores (also +0 / -0) -> lower block;
  // scores that differ in more than their low 8 mantissa bits keep the float order
  std::uniform_real_distribution<float> uf(-4.f, 4.f);
  for (int trial = 0; trial < 400000; ++trial) {
    float a = uf(rng), b = trial % 4 == 0 ? a : (trial % 4 == 1 ? -a : uf(rng));
    if (trial % 97 == 0) { a = 0.0f; b = -0.0f; }
    if (trial % 89 == 0) b = std::nextafter(a, 10.f);
    if (trial % 83 == 0) { a = std::ldexp(a, -140); b = std::ldexp(b, -140); }  // subnormals
    const int ia = rng() % 256, ib = rng() % 256;
    if (ia == ib) continue;
    const float ka = order_key(a, ia), kb = order_key(b, ib);
    if (key_block(ka) != ia || key_block(kb) != ib) { printf("key block\n"); return 1; }
    if (!(ka > -INFINITY) || std::isnan(ka)) { printf("empty key\n"); return 1; }
    const uint32_t ta = float_bits(a + 0.0f) & 0xFFFFFF00u, tb = float_bits(b + 0.0f) & 0xFFFFFF00u;
    if (a == b) {
      if ((ka > kb) != (ia < ib)) { printf("tie %g %g\n", a, b); return 1; }
    } else if (ta != tb) {
      if ((ka > kb) != (a > b)) { printf("order %g %g\n", a, b); return 1; }
    } else {
      const float big = std::max(std::fabs(a), std::fabs(b));
      if (std::fabs(a - b) > std::max(big * std::ldexp(1.f, -15), std::ldexp(1.f, -141))) {
        printf("band %g %g\n", a, b); return 1;
      }
    }
  }
  printf("ok\n");
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_sorting_networks_exhaustive(tmp_path):
    src = tmp_path / "t.cpp"
    src.write_text(PROGRAM)
    exe = tmp_path / "t"
    r = subprocess.run(["g++", "-std=c++17", "-O2", "-I", CSRC, str(src), "-o", str(exe)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.split() == ["ok"]
