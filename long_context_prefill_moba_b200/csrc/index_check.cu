// Device-side validation of the query-per-block index (sel, offsets, rows)
// before an attention or backward call consumes it.
//
// The attention kernels index K/V, the partial results and the output with
// block ids from `sel` and row ids from `rows` without range checks of their
// own (the gate writes them, and checks would cost registers in the hot
// loops).  moba_check_index runs these checks as separate kernels, for index
// arrays from another gate or for debugging a change to the gate:
//   every sel row:     entries strictly ascending in [0, c], then -1; the last
//                      valid entry is c (the query's block); at most
//                      min(topk, c + 1) entries (exactly that many with `exact`);
//   offsets:           offsets[0] = 0, non-decreasing, offsets[last] <= the
//                      rows capacity;
//   every rows entry:  a row id of the shape, whose batch entry, kv head, and
//                      pass are those of its group (pass, b, g, j), with
//                      j < its block and j listed in its sel row.
// A failed check sets the status word to MOBA_ERR_INTERNAL; a last kernel
// then makes the index inert (offsets all 0, every sel row {c, -1, ...}), so
// a later attention or backward call reads no invalid index (its outputs are
// not meaningful).  Duplicate rows entries are not detected.
#include "launch.h"

namespace moba {

namespace {

constexpr int kThreads = 256;

#define MOBA_HD __host__ __device__ __forceinline__

// a selection row of width W for a query in block c
MOBA_HD bool sel_row_ok(const int32_t* row, int W, int c, int topk, bool exact) {
  int len = 0, prev = -1;
  bool ended = false;
  for (int i = 0; i < W; ++i) {
    const int e = row[i];
    if (e < 0) {
      if (e != -1) return false;
      ended = true;
      continue;
    }
    if (ended || e <= prev || e > c) return false;
    prev = e;
    ++len;
  }
  if (len == 0 || prev != c) return false;
  const int cap = topk < c + 1 ? topk : c + 1;
  return exact ? len == cap : len <= cap;
}

// group holding rows position p: the largest i < L with offsets[i] <= p
MOBA_HD int64_t group_of(const int32_t* offsets, int64_t L, int64_t p) {
  int64_t lo = 0, hi = L - 1;
  while (lo < hi) {
    const int64_t mid = (lo + hi + 1) >> 1;
    if (offsets[mid] <= p) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// rows entry r at a position of group gi = ((pass * batch + b) * hkv + g) * n + j
MOBA_HD bool row_entry_ok(int64_t r, int64_t gi, const int32_t* sel, const Dims& dm) {
  const int64_t nrows = (int64_t)dm.batch * dm.N * dm.hq;
  if (r < 0 || r >= nrows) return false;
  const int j = (int)(gi % dm.n);
  const int g = (int)((gi / dm.n) % dm.hkv);
  const int b = (int)((gi / ((int64_t)dm.n * dm.hkv)) % dm.batch);
  const int ch = (int)(gi / ((int64_t)dm.n * dm.hkv * dm.batch));
  const int h = (int)(r % dm.hq);
  const int t = (int)((r / dm.hq) % dm.N);
  const int rb = (int)(r / ((int64_t)dm.hq * dm.N));
  if (rb != b || h / dm.G != g || t / dm.chunk != ch || j >= t / dm.B) return false;
  const int32_t* row = sel + r * dm.topk;
  for (int i = 0; i < dm.topk; ++i)
    if (row[i] == j) return true;
  return false;
}

// entry i (0 <= i <= L) of the offsets of L groups
MOBA_HD bool offsets_ok_at(const int32_t* offsets, int64_t L, int64_t capacity, int64_t i) {
  bool ok = true;
  if (i == 0) ok = offsets[0] == 0;
  if (i < L) ok = ok && offsets[i] <= offsets[i + 1];
  if (i == L) ok = ok && offsets[L] <= capacity;
  return ok;
}

__global__ void __launch_bounds__(kThreads) check_offsets_kernel(const int32_t* __restrict__ offsets,
                                                                 int64_t L, int64_t capacity,
                                                                 int* __restrict__ status) {
  const int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  if (i <= L && !offsets_ok_at(offsets, L, capacity, i)) atomicExch(status, MOBA_ERR_INTERNAL);
}

__global__ void __launch_bounds__(kThreads) check_sel_kernel(const int32_t* __restrict__ sel, Dims dm,
                                                             int exact, int* __restrict__ status) {
  const int64_t r = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  if (r >= (int64_t)dm.batch * dm.N * dm.hq) return;
  const int t = (int)((r / dm.hq) % dm.N);
  if (!sel_row_ok(sel + r * dm.topk, dm.topk, t / dm.B, dm.topk, exact != 0))
    atomicExch(status, MOBA_ERR_INTERNAL);
}

// runs after check_offsets: with valid offsets, every position < offsets[L] is
// inside the rows capacity
__global__ void __launch_bounds__(kThreads) check_rows_kernel(const int32_t* __restrict__ sel,
                                                              const int32_t* __restrict__ offsets,
                                                              const int32_t* __restrict__ rows, int64_t L,
                                                              int64_t capacity, Dims dm,
                                                              int* __restrict__ status) {
  if (*(volatile int*)status != 0) return;   // offsets already rejected
  const int64_t p = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  if (p >= capacity || p >= offsets[L]) return;
  if (!row_entry_ok(rows[p], group_of(offsets, L, p), sel, dm)) atomicExch(status, MOBA_ERR_INTERNAL);
}

// after a failed check: offsets all 0 and every sel row {c, -1, ...}
__global__ void __launch_bounds__(kThreads) make_inert_kernel(int32_t* __restrict__ sel,
                                                              int32_t* __restrict__ offsets, int64_t L,
                                                              Dims dm, const int* __restrict__ status) {
  if (*(volatile const int*)status == 0) return;
  const int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  if (i <= L) offsets[i] = 0;
  if (i < (int64_t)dm.batch * dm.N * dm.hq) {
    const int t = (int)((i / dm.hq) % dm.N);
    int32_t* row = sel + i * dm.topk;
    row[0] = t / dm.B;
    for (int e = 1; e < dm.topk; ++e) row[e] = -1;
  }
}

unsigned grid_of(int64_t n) { return (unsigned)((n + kThreads - 1) / kThreads); }

}  // namespace

cudaError_t launch_index_check(const Dims& dm, int exact, int32_t* sel, int32_t* offsets,
                               const int32_t* rows, int64_t capacity, int* status, cudaStream_t stream,
                               int* launches) {
  const int64_t L = (int64_t)dm.nchunks * dm.batch * dm.hkv * dm.n;
  const int64_t nrows = (int64_t)dm.batch * dm.N * dm.hq;
  cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int), stream);
  if (e != cudaSuccess) return e;
  check_offsets_kernel<<<grid_of(L + 1), kThreads, 0, stream>>>(offsets, L, capacity, status);
  ++*launches;
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  check_sel_kernel<<<grid_of(nrows), kThreads, 0, stream>>>(sel, dm, exact, status);
  ++*launches;
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (capacity > 0) {
    check_rows_kernel<<<grid_of(capacity), kThreads, 0, stream>>>(sel, offsets, rows, L, capacity, dm,
                                                                  status);
    ++*launches;
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  make_inert_kernel<<<grid_of(nrows > L + 1 ? nrows : L + 1), kThreads, 0, stream>>>(sel, offsets, L, dm,
                                                                                     status);
  ++*launches;
  return cudaGetLastError();
}

}  // namespace moba
