"""The ranking code of the pooled-gate kernel (csrc/gate_pooled.cu: TopList and
write_union, compiled for host and device) against a brute force, on the
CPU.  A host program includes the kernel source, feeds random score streams
(half of them with many equal scores) through the same three lists the
kernel keeps, and compares the selection row it writes with the stable
descending sort of each ranking, their union, the current block and the -1
padding; it also checks each kept list's order.  No GPU is used."""
import os
import subprocess

from long_context_prefill_moba_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include "gate_pooled.cu"
#include <algorithm>
#include <cstdio>
#include <random>
#include <set>
#include <vector>

// the launchers gate_pooled.cu calls but this host program never runs
namespace moba {
bool gate_tc_pooled_supported(const Dims&, int) { return false; }
bool attn_tc_path(int, int) { return false; }
cudaError_t launch_gate_select_tc_pooled(const Dims&, int, int, const void*, const float*, const float*,
                                         const float*, int32_t*, int32_t*, int*, cudaStream_t) {
  return cudaErrorNotSupported;
}
cudaError_t launch_attn_passes(const Dims&, int, const void*, const void*, const void*, const int32_t*,
                               const int32_t*, const int32_t*, void*, float*, AttnWs, int, int,
                               cudaStream_t, int*) { return cudaErrorNotSupported; }
cudaError_t launch_gate_scan(const int32_t*, int32_t*, int64_t, int32_t, cudaStream_t) {
  return cudaErrorNotSupported;
}
}  // namespace moba

using namespace moba;

static std::vector<int> best(const std::vector<float>& s, int c, int m) {
  std::vector<int> idx(c);
  for (int i = 0; i < c; ++i) idx[i] = i;
  std::stable_sort(idx.begin(), idx.end(), [&](int a, int b) { return s[a] > s[b]; });
  idx.resize(std::min(m, c));
  return idx;
}

int main() {
  std::mt19937 rng(7);
  std::uniform_real_distribution<float> uni(-5.f, 5.f);
  for (int trial = 0; trial < 100000; ++trial) {
    const int topk = 1 + (int)(rng() % MOBA_MAX_TOPK);
    const int room = (MOBA_MAX_TOPK - topk) / 2;
    const int extra = room ? (int)(rng() % (room + 1)) : 0;
    const int W = topk + 2 * extra;
    const int c = (int)(rng() % 48);
    const bool ties = rng() % 2;
    std::vector<float> sa(c), sx(c), sn(c);
    for (int j = 0; j < c; ++j) {
      sa[j] = ties ? (float)(rng() % 4) : uni(rng);
      sx[j] = ties ? (float)(rng() % 3) : uni(rng);
      sn[j] = ties ? (float)(rng() % 5) : uni(rng);
    }
    TopList<kMeanCap> by_mean;
    TopList<kExtraCap> by_max, by_min;
    by_mean.init();
    by_max.init();
    by_min.init();
    for (int j = 0; j < c; ++j) {
      by_mean.offer(sa[j], j, topk - 1);
      by_max.offer(sx[j], j, extra);
      by_min.offer(sn[j], j, extra);
    }
    std::vector<int32_t> row(W, 12345);
    const int m = write_union(by_mean, by_max, by_min, c, W, row.data());
    std::set<int> chosen;
    for (int j : best(sa, c, topk - 1)) chosen.insert(j);
    for (int j : best(sx, c, extra)) chosen.insert(j);
    for (int j : best(sn, c, extra)) chosen.insert(j);
    std::vector<int32_t> want(chosen.begin(), chosen.end());
    want.push_back(c);
    while ((int)want.size() < W) want.push_back(-1);
    if (m != (int)chosen.size() || row != want) {
      printf("row mismatch: trial %d topk %d extra %d c %d\n", trial, topk, extra, c);
      return 1;
    }
    const std::vector<int> order = best(sa, c, topk - 1);
    for (size_t i = 0; i < order.size(); ++i)
      if (by_mean.j[i] != order[i]) {
        printf("order mismatch: trial %d\n", trial);
        return 2;
      }
  }
  printf("ok\n");
  return 0;
}
"""


def test_pooled_gate_ranking_code_against_brute_force(tmp_path):
    src = tmp_path / "ranking_check.cu"
    src.write_text(PROGRAM)
    exe = tmp_path / "ranking_check"
    cmd = [B.nvcc(), *B.ARCH, "-O2", "-std=c++17", "--expt-relaxed-constexpr",
           "-I", os.path.join(ROOT, "include"), "-I", B.CSRC, str(src), "-o", str(exe)]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    res = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert res.returncode == 0 and res.stdout.strip() == "ok", (res.returncode, res.stdout, res.stderr)
