"""The checks of moba_check_index (csrc/index_check.cu: sel_row_ok,
offsets_ok_at, group_of, row_entry_ok, compiled for host and device) on the
CPU.  A host program builds a valid query-per-block index for a small shape
by brute force (random selections obeying the gate's rules, grouped by
(pass, b, kv head, block)), runs every check the kernels run, and expects
them all to pass; then it plants one fault at a time (a block past the
current one, a missing current block, unsorted or duplicate entries, a bad
pad value, decreasing offsets, offsets past the capacity, a row id out of
range, a row in the wrong group, pass or batch entry, a row that did not
select the block) and expects at least one check to fail for each.  No GPU
is used."""
import os
import subprocess

from long_context_prefill_moba_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include "index_check.cu"
#include <algorithm>
#include <cstdio>
#include <random>
#include <vector>

using namespace moba;

struct Index {
  Dims dm;
  std::vector<int32_t> sel, offsets, rows;
  int64_t capacity;
};

static Index build_index(bool exact, unsigned seed) {
  Dims dm{};
  dm.batch = 2; dm.N = 300; dm.hq = 4; dm.hkv = 2; dm.d = 64; dm.B = 32; dm.topk = 4;
  dm.n = (dm.N + dm.B - 1) / dm.B; dm.G = dm.hq / dm.hkv; dm.chunk = 128;
  dm.nchunks = (dm.N + dm.chunk - 1) / dm.chunk; dm.t_lo = 0; dm.t_hi = dm.N;
  std::mt19937 rng(seed);
  Index ix{dm, {}, {}, {}, 0};
  const int64_t nrows = (int64_t)dm.batch * dm.N * dm.hq;
  const int64_t L = (int64_t)dm.nchunks * dm.batch * dm.hkv * dm.n;
  ix.sel.assign(nrows * dm.topk, -1);
  std::vector<std::vector<int32_t>> groups(L);
  for (int64_t r = 0; r < nrows; ++r) {
    const int h = (int)(r % dm.hq), t = (int)((r / dm.hq) % dm.N), b = (int)(r / ((int64_t)dm.hq * dm.N));
    const int c = t / dm.B;
    const int cap = std::min(dm.topk - 1, c);
    const int m = exact ? cap : (int)(rng() % (cap + 1));
    std::vector<int> pool(c);
    for (int j = 0; j < c; ++j) pool[j] = j;
    std::shuffle(pool.begin(), pool.end(), rng);
    pool.resize(m);
    std::sort(pool.begin(), pool.end());
    for (int i = 0; i < m; ++i) {
      ix.sel[r * dm.topk + i] = pool[i];
      const int64_t gi = (((int64_t)(t / dm.chunk) * dm.batch + b) * dm.hkv + h / dm.G) * dm.n + pool[i];
      groups[gi].push_back((int32_t)r);
    }
    ix.sel[r * dm.topk + m] = c;
    ix.capacity += cap;
  }
  ix.offsets.assign(L + 1, 0);
  for (int64_t g = 0; g < L; ++g) {
    std::shuffle(groups[g].begin(), groups[g].end(), rng);   // order within a group is free
    ix.offsets[g + 1] = ix.offsets[g] + (int32_t)groups[g].size();
    for (int32_t r : groups[g]) ix.rows.push_back(r);
  }
  ix.rows.resize(std::max<int64_t>(ix.capacity, 1), 0);
  return ix;
}

// every check of the kernels, on the host; true when all pass
static bool all_ok(const Index& ix, bool exact) {
  const Dims& dm = ix.dm;
  const int64_t L = (int64_t)dm.nchunks * dm.batch * dm.hkv * dm.n;
  for (int64_t i = 0; i <= L; ++i)
    if (!offsets_ok_at(ix.offsets.data(), L, ix.capacity, i)) return false;
  const int64_t nrows = (int64_t)dm.batch * dm.N * dm.hq;
  for (int64_t r = 0; r < nrows; ++r) {
    const int t = (int)((r / dm.hq) % dm.N);
    if (!sel_row_ok(ix.sel.data() + r * dm.topk, dm.topk, t / dm.B, dm.topk, exact)) return false;
  }
  for (int64_t p = 0; p < ix.capacity && p < ix.offsets[L]; ++p)
    if (!row_entry_ok(ix.rows[p], group_of(ix.offsets.data(), L, p), ix.sel.data(), dm)) return false;
  return true;
}

int main() {
  int failures = 0;
  for (int ex = 0; ex < 2; ++ex) {
    const bool exact = ex == 1;
    const Index good = build_index(exact, 11 + ex);
    if (!all_ok(good, exact)) { printf("valid index rejected (exact %d)\n", ex); return 1; }
    const Dims& dm = good.dm;
    const int W = dm.topk;
    // a row of the last pass (batch entry 1, kv head 1, token 256 or later) with at least two
    // earlier blocks selected, and its first entry in rows
    int64_t r0 = -1, p0 = -1;
    for (int t = 256; t < dm.N && r0 < 0; ++t) {
      const int64_t r = ((int64_t)1 * dm.N + t) * dm.hq + 3;
      if (good.sel[r * W + 1] >= 0 && good.sel[r * W + 1] < t / dm.B) r0 = r;
    }
    for (int64_t p = 0; r0 >= 0 && p < good.offsets.back(); ++p) if (good.rows[p] == r0) { p0 = p; break; }
    if (r0 < 0 || p0 < 0) { printf("no suitable row\n"); return 3; }
    const int64_t L = (int64_t)dm.nchunks * dm.batch * dm.hkv * dm.n;
    using Fault = void (*)(Index&, int64_t, int64_t, int);
    struct Case { const char* name; Fault f; };
    const Case cases[] = {
      {"future block", [](Index& x, int64_t r, int64_t, int w) { x.sel[r * w + 0] = 9; }},
      {"no current block", [](Index& x, int64_t r, int64_t, int w) {
         for (int i = w - 1; i >= 0; --i) if (x.sel[r * w + i] >= 0) { x.sel[r * w + i] = -1; break; } }},
      {"unsorted", [](Index& x, int64_t r, int64_t, int w) { std::swap(x.sel[r * w + 0], x.sel[r * w + 1]); }},
      {"duplicate", [](Index& x, int64_t r, int64_t, int w) { x.sel[r * w + 1] = x.sel[r * w + 0]; }},
      {"bad pad", [](Index& x, int64_t, int64_t, int w) { x.sel[0 * w + 1] = -7; }},
      {"offsets decrease", [](Index& x, int64_t, int64_t, int) { x.offsets[5] = x.offsets[6] + 1; }},
      {"offsets past capacity", [](Index& x, int64_t, int64_t, int) { x.offsets.back() = (int32_t)x.capacity + 1; }},
      {"row id out of range", [](Index& x, int64_t, int64_t p, int) { x.rows[p] = 1 << 30; }},
      {"negative row id", [](Index& x, int64_t, int64_t p, int) { x.rows[p] = -2; }},
      {"other kv head", [](Index& x, int64_t r, int64_t p, int) { x.rows[p] = (int32_t)(r - 3); }},
      {"other batch entry", [](Index& x, int64_t r, int64_t p, int) { x.rows[p] = (int32_t)(r - 300 * 4); }},
      {"other pass", [](Index& x, int64_t r, int64_t p, int) { x.rows[p] = (int32_t)(r - 130 * 4); }},
      {"block not selected", [](Index& x, int64_t r, int64_t p, int w) {
         // same pass, batch entry and head, a token whose row did not select this block
         const int t0 = (int)((r / 4) % 300);
         for (int t = 256; t < 300; ++t) {
           const int64_t r2 = r + (int64_t)(t - t0) * 4;
           bool has = false;
           for (int i = 0; i < w; ++i) has |= x.sel[r2 * w + i] == x.sel[r * w + 0];
           if (!has) { x.rows[p] = (int32_t)r2; return; }
         }
       }},
    };
    for (const Case& cs : cases) {
      Index bad = good;
      cs.f(bad, r0, p0, W);
      if (all_ok(bad, exact)) { printf("not detected: %s (exact %d)\n", cs.name, ex); ++failures; }
    }
    if (exact) {   // a row with fewer blocks than min(topk, c + 1) passes only without `exact`
      Index bad = good;
      bad.sel[r0 * W + 0] = bad.sel[r0 * W + 1];
      bad.sel[r0 * W + 1] = bad.sel[r0 * W + 2];
      bad.sel[r0 * W + 2] = bad.sel[r0 * W + 3];
      bad.sel[r0 * W + 3] = -1;
      if (all_ok(bad, true)) { printf("not detected: short row\n"); ++failures; }
    }
    (void)L;
  }
  if (failures) return 2;
  printf("ok\n");
  return 0;
}
"""


def test_index_checks_pass_a_valid_index_and_catch_planted_faults(tmp_path):
    src = tmp_path / "index_check_host.cu"
    src.write_text(PROGRAM)
    exe = tmp_path / "index_check_host"
    cmd = [B.nvcc(), *B.ARCH, "-O2", "-std=c++17", "--expt-relaxed-constexpr",
           "-I", os.path.join(ROOT, "include"), "-I", B.CSRC, str(src), "-o", str(exe)]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    res = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert res.returncode == 0 and res.stdout.strip() == "ok", (res.returncode, res.stdout, res.stderr)
