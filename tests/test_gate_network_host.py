"""The ranking networks of the tensor-core gate (csrc/gate_tc.cu: sort_desc,
merge_top and the compare-exchange lists they apply, compiled for host and
device) checked on the CPU.  A host program includes the kernel source and

  - sorts every 0/1 input of K = 4, 8 and 16 entries with sort_desc (by the
    0-1 principle a comparator network that sorts all of them sorts every
    input);
  - merges every pair of sorted 0/1 lists with merge_top and compares the
    result with the top K of their union, sorted;
  - streams random candidate rows (up to 256 blocks, half of them drawn from a
    few values so that ties are common, with -inf for masked blocks) through
    the kernel's fold, one batch of K scores at a time sorted and merged into
    the running list, and checks that the list is the K largest scores in
    descending order, so that its m-th entry is the selection threshold.

A plausible slip in the networks (a missing stage, a wrong partner index, the
merge without reversing the second list) fails one of these.  No GPU is used."""
import os
import subprocess

from long_context_prefill_moba_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include "gate_tc.cu"
#include <algorithm>
#include <cmath>
#include <cstdio>
#include <functional>
#include <random>
#include <vector>

using namespace moba;

template <int K>
static int check_sort_01() {
  for (unsigned m = 0; m < (1u << K); ++m) {
    float v[K];
    for (int i = 0; i < K; ++i) v[i] = (m >> i) & 1u ? 1.f : 0.f;
    sort_desc<K>(v);
    for (int i = 1; i < K; ++i)
      if (v[i - 1] < v[i]) { printf("sort K=%d input %u\n", K, m); return 1; }
    int ones = 0;
    for (int i = 0; i < K; ++i) ones += v[i] == 1.f;
    if (ones != __builtin_popcount(m)) { printf("sort K=%d lost entries\n", K); return 1; }
  }
  return 0;
}

template <int K>
static int check_merge_01() {
  for (int x = 0; x <= K; ++x)
    for (int y = 0; y <= K; ++y) {
      float a[K], b[K];
      for (int i = 0; i < K; ++i) { a[i] = i < x ? 1.f : 0.f; b[i] = i < y ? 1.f : 0.f; }
      merge_top<K>(a, b);
      const int ones = std::min(K, x + y);
      for (int i = 0; i < K; ++i)
        if (a[i] != (i < ones ? 1.f : 0.f)) { printf("merge K=%d x=%d y=%d\n", K, x, y); return 1; }
    }
  return 0;
}

template <int K>
static int check_stream(std::mt19937& rng, int trials) {
  std::uniform_real_distribution<float> uni(-300.f, 300.f);
  for (int trial = 0; trial < trials; ++trial) {
    const int c = (int)(rng() % 257);
    const bool ties = rng() % 2;
    const int ncand = (c + 31) / 32 * 32;   // the kernel reads whole 32-column chunks
    std::vector<float> s(ncand, -INFINITY);
    for (int j = 0; j < c; ++j) {
      s[j] = ties ? (float)(rng() % 5) - 2.f : uni(rng);
      if (rng() % 64 == 0) s[j] = -INFINITY;
    }
    float a[K];
    for (int i = 0; i < K; ++i) a[i] = -INFINITY;
    for (int j0 = 0; j0 < ncand; j0 += K) {
      float bt[K];
      for (int i = 0; i < K; ++i) bt[i] = s[j0 + i];
      sort_desc<K>(bt);
      merge_top<K>(a, bt);
    }
    std::vector<float> want(s);
    std::sort(want.begin(), want.end(), std::greater<float>());
    for (int i = 0; i < K; ++i) {
      const float w = i < (int)want.size() ? want[i] : -INFINITY;
      if (!(a[i] == w)) { printf("stream K=%d trial %d entry %d: %g vs %g\n", K, trial, i, a[i], w); return 1; }
    }
  }
  return 0;
}

int main() {
  std::mt19937 rng(11);
  if (check_sort_01<4>() || check_sort_01<8>() || check_sort_01<16>()) return 1;
  if (check_merge_01<4>() || check_merge_01<8>() || check_merge_01<16>()) return 2;
  if (check_stream<4>(rng, 20000) || check_stream<8>(rng, 20000) || check_stream<16>(rng, 20000)) return 3;
  printf("ok\n");
  return 0;
}
"""


def test_gate_ranking_networks(tmp_path):
    src = tmp_path / "network_check.cu"
    src.write_text(PROGRAM)
    exe = tmp_path / "network_check"
    cmd = [B.nvcc(), *B.ARCH, "-O2", "-std=c++17", "--expt-relaxed-constexpr",
           "-I", os.path.join(ROOT, "include"), "-I", B.CSRC, str(src), "-o", str(exe), "-lcuda"]
    build = subprocess.run(cmd, capture_output=True, text=True)
    assert build.returncode == 0, build.stderr[-3000:]
    res = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert res.returncode == 0 and res.stdout.strip() == "ok", (res.returncode, res.stdout, res.stderr)
