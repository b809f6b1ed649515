// Gate variant that also routes blocks by max- and min-pooled keys, and the
// per-pass step that lets the attention kernels take its selections.
//
// "MoBA: Mixture of Block Attention for Long-Context LLMs", paperhub.cn
// OpenReview discussion page, the authors' rebuttals to W1 (block
// representation; the comparison with QUEST): besides the blocks the
// mean-pooled gate selects, the ablation also selects the top blocks under max
// pooling and under min pooling of the keys.  The page gives no formula; the
// reading implemented here:  a query at position t (current block c) attends
//     the top (topk - 1) earlier blocks by <q, mean K_j>        (the MoBA gate)
//   U the top `extra` earlier blocks by <q, max K_j>             (channel-wise)
//   U the top `extra` earlier blocks by <q, min K_j>             (channel-wise)
//   U {c},
// each ranking over the candidates j < c, equal scores to the lower block.
//
// The selection row is W = topk + 2 extra wide: the chosen earlier blocks in
// ascending order, then c, then -1.  The attention kernels run unchanged with
// W in place of topk (each row then owns W - 1 partial-result slots).  A row
// that chose fewer than min(W - 1, c) earlier blocks (the rankings overlap)
// leaves slots that no historical tile writes; pooled_fill marks them empty
// (log-sum-exp -inf, output 0) before each pass, so the merge, which reads
// min(W - 1, c) slots per row, adds nothing for them.
//
// Launches of the gate: maxminpool (once per layer, beside the mean-pool),
// the selection, the gate's prefix scan, pooled_scatter; of the attention:
// pooled_fill before the two attention kernels of every pass.  The selection
// runs on tensor cores (three passes of gate_select_tc, one per ranking; see
// gate_tc.cu) for bf16 with head_dim 128 when a row's candidate mask fits its
// sel entries, and on CUDA cores (pooled_select, below) otherwise.
#include <float.h>

#include "launch.h"

namespace moba {

namespace {

// ---- K1': channel-wise max and min of every block's keys ---------------------
// Same work split as the mean-pool: one CTA per (column slice, block, batch),
// 16-byte coalesced loads, each key byte read once.  max/min are exact, so the
// result does not depend on the reduction order.
constexpr int kPoolThreads = 256;

template <typename T>
__global__ void __launch_bounds__(kPoolThreads) maxminpool_kernel(const T* __restrict__ k,
                                                                  float* __restrict__ maxk,
                                                                  float* __restrict__ mink, int N,
                                                                  int W, int B, int n) {
  constexpr int V = Vec16<T>::kN;
  const int vecs_per_row = W / V;
  const int cols_cta = min(vecs_per_row, kPoolThreads);
  const int rows_per_pass = kPoolThreads / cols_cta;
  const int tid = threadIdx.x;
  const int cvec = blockIdx.x * cols_cta + (tid % cols_cta);
  const int rsub = tid / cols_cta;
  const int j = blockIdx.y;
  const int b = blockIdx.z;
  const int t0 = j * B;
  const int t1 = min(N, t0 + B);
  const bool active = (rsub < rows_per_pass) && (cvec < vecs_per_row);

  float mx[V], mn[V];
#pragma unroll
  for (int i = 0; i < V; ++i) { mx[i] = -INFINITY; mn[i] = INFINITY; }
  if (active) {
    const T* base = k + ((size_t)b * N) * W + (size_t)cvec * V;
#pragma unroll 4
    for (int t = t0 + rsub; t < t1; t += rows_per_pass) {
      float x[V];
      Vec16<T>::load(base + (size_t)t * W, x);
#pragma unroll
      for (int i = 0; i < V; ++i) { mx[i] = fmaxf(mx[i], x[i]); mn[i] = fminf(mn[i], x[i]); }
    }
  }
  __shared__ float red_mx[kPoolThreads * V];
  __shared__ float red_mn[kPoolThreads * V];
  if (rsub < rows_per_pass) {
#pragma unroll
    for (int i = 0; i < V; ++i) {
      red_mx[rsub * cols_cta * V + (tid % cols_cta) * V + i] = mx[i];
      red_mn[rsub * cols_cta * V + (tid % cols_cta) * V + i] = mn[i];
    }
  }
  __syncthreads();
  for (int e = tid; e < cols_cta * V; e += kPoolThreads) {
    const int col = blockIdx.x * cols_cta * V + e;
    if (col >= W) continue;
    float a = -INFINITY, z = INFINITY;
    for (int r = 0; r < rows_per_pass; ++r) {
      a = fmaxf(a, red_mx[r * cols_cta * V + e]);
      z = fminf(z, red_mn[r * cols_cta * V + e]);
    }
    maxk[((size_t)b * n + j) * W + col] = a;
    mink[((size_t)b * n + j) * W + col] = z;
  }
}

// ---- K2': three rankings and their union ----------------------------------------
constexpr int kRows = 128;                            // query rows per CTA (one thread each)
constexpr int kJChunk = 16;                           // blocks of each pool staged at a time
constexpr int kSmemHist = 4096;                       // blocks counted in shared memory
constexpr int kMeanCap = MOBA_MAX_TOPK - 1;           // slots of the mean ranking
constexpr int kExtraCap = (MOBA_MAX_TOPK - 1) / 2;    // slots of the max / min rankings
constexpr int kUnion = kMeanCap + 2 * kExtraCap;

#define MOBA_HD __host__ __device__ __forceinline__

// Descending list of the best K (<= CAP) candidates offered so far.  Candidates
// arrive in increasing block index and an equal score is placed after the
// entries already kept, so ties go to the lower block.
template <int CAP>
struct TopList {
  float s[CAP];
  int j[CAP];
  int kept;
  float thresh;   // smallest kept score once the list is full

  MOBA_HD void init() {
#pragma unroll
    for (int i = 0; i < CAP; ++i) { s[i] = -FLT_MAX; j[i] = -1; }
    kept = 0;
    thresh = -INFINITY;
  }
  MOBA_HD void offer(float v, int idx, int K) {
    if (K == 0 || (kept == K && !(v > thresh))) return;
    // insertion point: kept entries with a score >= v stay ahead
    int p = 0;
#pragma unroll
    for (int i = 0; i < CAP; ++i) p += (i < kept && s[i] >= v) ? 1 : 0;
#pragma unroll
    for (int i = CAP - 1; i >= 0; --i) {
      if (i < K) {
        if (i > p) {
          s[i] = s[i > 0 ? i - 1 : 0];
          j[i] = j[i > 0 ? i - 1 : 0];
        } else if (i == p) {
          s[i] = v;
          j[i] = idx;
        }
      }
    }
    kept = kept + 1 < K ? kept + 1 : K;
    if (kept == K) {
      thresh = INFINITY;
#pragma unroll
      for (int i = 0; i < CAP; ++i) thresh = fminf(thresh, i < K ? s[i] : INFINITY);
    }
  }
  MOBA_HD bool holds(int x) const {
    bool f = false;
#pragma unroll
    for (int i = 0; i < CAP; ++i) f |= (i < kept && j[i] == x);
    return f;
  }
};

// The selection row of a query in block c from its three lists: every chosen
// earlier block once, ascending, then c, then -1 up to the width W.  Returns
// the number of chosen earlier blocks (at most W - 1).
MOBA_HD int write_union(const TopList<kMeanCap>& by_mean, const TopList<kExtraCap>& by_max,
                        const TopList<kExtraCap>& by_min, int c, int W, int32_t* out) {
  int u[kUnion];
  bool keep[kUnion];
#pragma unroll
  for (int i = 0; i < kMeanCap; ++i) {
    u[i] = by_mean.j[i];
    keep[i] = i < by_mean.kept;
  }
#pragma unroll
  for (int i = 0; i < kExtraCap; ++i) {
    u[kMeanCap + i] = by_max.j[i];
    keep[kMeanCap + i] = i < by_max.kept && !by_mean.holds(by_max.j[i]);
    u[kMeanCap + kExtraCap + i] = by_min.j[i];
    keep[kMeanCap + kExtraCap + i] =
        i < by_min.kept && !by_mean.holds(by_min.j[i]) && !by_max.holds(by_min.j[i]);
  }
  int m = 0;
#pragma unroll
  for (int e = 0; e < kUnion; ++e) {
    if (keep[e]) {
      int rank = 0;
#pragma unroll
      for (int f = 0; f < kUnion; ++f) rank += (keep[f] && u[f] < u[e]) ? 1 : 0;
      out[rank] = u[e];
      ++m;
    }
  }
  out[m] = c;
  for (int i = m + 1; i < W; ++i) out[i] = -1;
  return m;
}

template <typename T, int D>
__global__ void __launch_bounds__(kRows) pooled_select_kernel(
    const T* __restrict__ q, const float* __restrict__ meank, const float* __restrict__ maxk,
    const float* __restrict__ mink, int32_t* __restrict__ sel, int32_t* __restrict__ counts, Dims dm,
    int km, int extra) {
  __shared__ __align__(16) float kb[3][kJChunk * D];
  __shared__ int hist[kSmemHist];
  const int tiles_per_seq = (dm.t_hi - dm.t_lo + kRows - 1) / kRows;
  const int tile = blockIdx.x % tiles_per_seq;
  const int bh = blockIdx.x / tiles_per_seq;
  const int h = bh % dm.hq;
  const int b = bh / dm.hq;
  const int g = h / dm.G;
  const int t_first = dm.t_lo + tile * kRows;
  const int t = t_first + threadIdx.x;
  const bool valid = t < dm.t_hi;
  const int c = valid ? t / dm.B : 0;
  const int t_last = min(dm.t_hi, t_first + kRows) - 1;
  const int c_max = t_last / dm.B;
  const bool use_hist = dm.n <= kSmemHist;
  const int j_lim = (km > 0 || extra > 0) ? c_max : 0;

  if (use_hist)
    for (int i = threadIdx.x; i < c_max; i += kRows) hist[i] = 0;

  float qv[D];
  if (valid) {
    const T* qp = q + ((size_t)(b * dm.N + t) * dm.hq + h) * D;
#pragma unroll
    for (int e = 0; e < D; e += Vec16<T>::kN) Vec16<T>::load(qp + e, qv + e);
  } else {
#pragma unroll
    for (int e = 0; e < D; ++e) qv[e] = 0.f;
  }

  TopList<kMeanCap> by_mean;
  TopList<kExtraCap> by_max, by_min;
  by_mean.init();
  by_max.init();
  by_min.init();

  const size_t pool_g = ((size_t)b * dm.n * dm.hkv + g) * D;   // block j at + j * hkv * D
  const float* pools[3] = {meank + pool_g, maxk + pool_g, mink + pool_g};
  for (int j0 = 0; j0 < j_lim; j0 += kJChunk) {
    const int jn = min(kJChunk, j_lim - j0);
    __syncthreads();
    for (int e = threadIdx.x * 4; e < jn * D; e += kRows * 4) {
      const int jj = e / D, col = e % D;
      const size_t src = (size_t)(j0 + jj) * dm.hkv * D + col;
#pragma unroll
      for (int p = 0; p < 3; ++p)
        *reinterpret_cast<float4*>(&kb[p][e]) = __ldg(reinterpret_cast<const float4*>(pools[p] + src));
    }
    __syncthreads();
    if (!valid) continue;
    const int jend = min(jn, c - j0);
    for (int jj = 0; jj < jend; ++jj) {
      const float4* ka = reinterpret_cast<const float4*>(&kb[0][jj * D]);
      const float4* kx = reinterpret_cast<const float4*>(&kb[1][jj * D]);
      const float4* kn = reinterpret_cast<const float4*>(&kb[2][jj * D]);
      float sa0 = 0.f, sa1 = 0.f, sx0 = 0.f, sx1 = 0.f, sn0 = 0.f, sn1 = 0.f;
#pragma unroll
      for (int e = 0; e < D / 4; ++e) {
        const float4 a = ka[e], x = kx[e], z = kn[e];
        sa0 = fmaf(qv[4 * e + 0], a.x, sa0);
        sa1 = fmaf(qv[4 * e + 1], a.y, sa1);
        sa0 = fmaf(qv[4 * e + 2], a.z, sa0);
        sa1 = fmaf(qv[4 * e + 3], a.w, sa1);
        sx0 = fmaf(qv[4 * e + 0], x.x, sx0);
        sx1 = fmaf(qv[4 * e + 1], x.y, sx1);
        sx0 = fmaf(qv[4 * e + 2], x.z, sx0);
        sx1 = fmaf(qv[4 * e + 3], x.w, sx1);
        sn0 = fmaf(qv[4 * e + 0], z.x, sn0);
        sn1 = fmaf(qv[4 * e + 1], z.y, sn1);
        sn0 = fmaf(qv[4 * e + 2], z.z, sn0);
        sn1 = fmaf(qv[4 * e + 3], z.w, sn1);
      }
      const int jidx = j0 + jj;
      by_mean.offer(sa0 + sa1, jidx, km);
      by_max.offer(sx0 + sx1, jidx, extra);
      by_min.offer(sn0 + sn1, jidx, extra);
    }
  }

  if (valid) {
    int32_t* out = sel + ((size_t)(b * dm.N + t) * dm.hq + h) * dm.topk;
    const int m = write_union(by_mean, by_max, by_min, c, dm.topk, out);
    const int ch = t / dm.chunk;
    int32_t* cnt_g = counts + ((size_t)(ch * dm.batch + b) * dm.hkv + g) * dm.n;
    for (int i = 0; i < m; ++i) {
      const int j = out[i];
      if (use_hist) atomicAdd(&hist[j], 1);
      else atomicAdd(&cnt_g[j], 1);
    }
  }
  if (use_hist) {
    __syncthreads();
    // a tile never straddles a pass boundary (the pass length is a multiple of 128)
    const int ch = t_first / dm.chunk;
    int32_t* cnt_g = counts + ((size_t)(ch * dm.batch + b) * dm.hkv + g) * dm.n;
    for (int i = threadIdx.x; i < c_max; i += kRows)
      if (hist[i]) atomicAdd(&cnt_g[i], hist[i]);
  }
}

// Places each (row, chosen earlier block) into its group's range of `rows`.
// The earlier blocks of a row are the prefix of its selection with entries in
// [0, c); there are at most W - 1 of them.
__global__ void __launch_bounds__(kRows) pooled_scatter_kernel(const int32_t* __restrict__ sel,
                                                               const int32_t* __restrict__ offsets,
                                                               int32_t* __restrict__ cursors,
                                                               int32_t* __restrict__ rows, Dims dm) {
  __shared__ int cnt[kSmemHist];
  __shared__ int base[kSmemHist];
  const int tiles_per_seq = (dm.t_hi - dm.t_lo + kRows - 1) / kRows;
  const int tile = blockIdx.x % tiles_per_seq;
  const int bh = blockIdx.x / tiles_per_seq;
  const int h = bh % dm.hq;
  const int b = bh / dm.hq;
  const int g = h / dm.G;
  const int t_first = dm.t_lo + tile * kRows;
  const int t = t_first + threadIdx.x;
  const bool valid = t < dm.t_hi;
  const int t_last = min(dm.t_hi, t_first + kRows) - 1;
  const int c_max = t_last / dm.B;
  const bool use_hist = dm.n <= kSmemHist;
  const int ch = t_first / dm.chunk;
  const size_t grp0 = ((size_t)(ch * dm.batch + b) * dm.hkv + g) * dm.n;
  const int32_t r = (b * dm.N + t) * dm.hq + h;

  constexpr int kH = MOBA_MAX_TOPK - 1;
  int js[kH];
  bool live[kH];
  int loc[kH];
  if (valid) {
    const int32_t* srow = sel + (size_t)r * dm.topk;
    const int c = t / dm.B;
#pragma unroll
    for (int i = 0; i < kH; ++i) {
      const int e = i < dm.topk - 1 ? srow[i] : -1;
      live[i] = e >= 0 && e < c;
      js[i] = live[i] ? e : 0;
    }
  } else {
#pragma unroll
    for (int i = 0; i < kH; ++i) { live[i] = false; js[i] = 0; }
  }
  if (use_hist) {
    for (int i = threadIdx.x; i < c_max; i += kRows) cnt[i] = 0;
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kH; ++i)
      if (live[i]) loc[i] = atomicAdd(&cnt[js[i]], 1);
    __syncthreads();
    for (int i = threadIdx.x; i < c_max; i += kRows)
      base[i] = cnt[i] ? atomicAdd(&cursors[grp0 + i], cnt[i]) : 0;
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kH; ++i)
      if (live[i]) rows[offsets[grp0 + js[i]] + base[js[i]] + loc[i]] = r;
  } else {
#pragma unroll
    for (int i = 0; i < kH; ++i)
      if (live[i]) rows[offsets[grp0 + js[i]] + atomicAdd(&cursors[grp0 + js[i]], 1)] = r;
  }
}

// One thread per (row of pass ch, partial slot): a slot the merge will read
// (slot < min(W - 1, c)) that no historical tile writes (slot >= the row's
// number of chosen earlier blocks) gets lse -inf and a zero output.
constexpr int kFillThreads = 256;

__global__ void __launch_bounds__(kFillThreads) pooled_fill_kernel(const int32_t* __restrict__ sel,
                                                                   float* __restrict__ part_o,
                                                                   float* __restrict__ part_lse, Dims dm,
                                                                   int ch, int part_elem_bytes) {
  const int KH = dm.topk - 1;
  const int t0 = ch * dm.chunk;
  const int len = min(dm.N, t0 + dm.chunk) - t0;
  const int64_t idx = (int64_t)blockIdx.x * kFillThreads + threadIdx.x;
  if (idx >= (int64_t)dm.batch * len * dm.hq * KH) return;
  const int slot = (int)(idx % KH);
  int64_t rest = idx / KH;
  const int h = (int)(rest % dm.hq);
  rest /= dm.hq;
  const int tt = (int)(rest % len);
  const int b = (int)(rest / len);
  const int t = t0 + tt;
  const int c = t / dm.B;
  if (slot >= min(KH, c)) return;
  const int32_t* srow = sel + ((size_t)(b * dm.N + t) * dm.hq + h) * dm.topk;
  int chosen = 0;
  for (int i = 0; i < KH; ++i) {
    const int e = srow[i];
    chosen += (e >= 0 && e < c) ? 1 : 0;
  }
  if (slot < chosen) return;
  const size_t pidx = (size_t)((b * dm.chunk + tt) * dm.hq + h) * KH + slot;
  part_lse[pidx] = -INFINITY;
  uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<char*>(part_o) + pidx * dm.d * part_elem_bytes);
  const int n16 = dm.d * part_elem_bytes / 16;
  for (int i = 0; i < n16; ++i) dst[i] = make_uint4(0u, 0u, 0u, 0u);
}

template <typename T>
cudaError_t launch_pooled_select(const Dims& dm, int km, int extra, const void* q, const float* meank,
                                 const float* maxk, const float* mink, int32_t* sel, int32_t* counts,
                                 cudaStream_t stream) {
  const int tiles = (dm.t_hi - dm.t_lo + kRows - 1) / kRows;
  dim3 grid(tiles * dm.batch * dm.hq);
  if (dm.d == 128)
    pooled_select_kernel<T, 128><<<grid, kRows, 0, stream>>>(static_cast<const T*>(q), meank, maxk, mink,
                                                             sel, counts, dm, km, extra);
  else
    pooled_select_kernel<T, 64><<<grid, kRows, 0, stream>>>(static_cast<const T*>(q), meank, maxk, mink,
                                                            sel, counts, dm, km, extra);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_maxminpool(const Dims& dm, int dtype, const void* k, float* maxk, float* mink,
                              cudaStream_t stream, int* launches) {
  const int W = dm.hkv * dm.d;
  const int V = dtype == MOBA_BF16 ? 8 : 4;
  const int vecs_per_row = W / V;
  const int cols_cta = vecs_per_row < kPoolThreads ? vecs_per_row : kPoolThreads;
  dim3 grid((vecs_per_row + cols_cta - 1) / cols_cta, dm.n, dm.batch);
  if (dtype == MOBA_BF16)
    maxminpool_kernel<__nv_bfloat16><<<grid, kPoolThreads, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(k), maxk, mink, dm.N, W, dm.B, dm.n);
  else
    maxminpool_kernel<float><<<grid, kPoolThreads, 0, stream>>>(static_cast<const float*>(k), maxk, mink,
                                                                 dm.N, W, dm.B, dm.n);
  ++*launches;
  return cudaGetLastError();
}

cudaError_t launch_gate_pooled(const Dims& dm, int dtype, int km, int extra, const void* q,
                               const float* meank, const float* maxk, const float* mink, int32_t* sel,
                               int32_t* offsets, int32_t* rows, GateWs ws, cudaStream_t stream,
                               int* launches) {
  const int64_t L = (int64_t)dm.nchunks * dm.batch * dm.hkv * dm.n;
  cudaError_t e = cudaMemsetAsync(ws.counts, 0, sizeof(int32_t) * L * 2, stream);  // counts+cursors
  if (e != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(ws.status, 0, sizeof(int), stream)) != cudaSuccess) return e;
  if (gate_tc_pooled_supported(dm, dtype)) {
    // three tensor-core passes (mean, max, min rankings), the union in the last
    e = launch_gate_select_tc_pooled(dm, km, extra, q, meank, maxk, mink, sel, ws.counts, ws.status, stream);
    *launches += 3;
  } else if (dtype == MOBA_BF16) {
    e = launch_pooled_select<__nv_bfloat16>(dm, km, extra, q, meank, maxk, mink, sel, ws.counts, stream);
    ++*launches;
  } else {
    e = launch_pooled_select<float>(dm, km, extra, q, meank, maxk, mink, sel, ws.counts, stream);
    ++*launches;
  }
  if (e != cudaSuccess) return e;
  if ((e = launch_gate_scan(ws.counts, offsets, L, 0, stream)) != cudaSuccess) return e;
  ++*launches;
  if (dm.topk > 1) {
    const int tiles = (dm.t_hi - dm.t_lo + kRows - 1) / kRows;
    pooled_scatter_kernel<<<tiles * dm.batch * dm.hq, kRows, 0, stream>>>(sel, offsets, ws.cursors,
                                                                          rows, dm);
    ++*launches;
    e = cudaGetLastError();
  }
  return e;
}

cudaError_t launch_attn_pooled(const Dims& dm, int dtype, const void* q, const void* k, const void* v,
                               const int32_t* sel, const int32_t* offsets, const int32_t* rows,
                               void* out, float* lse, AttnWs ws, cudaStream_t stream, int* launches) {
  cudaError_t e = cudaMemsetAsync(ws.status, 0, sizeof(int), stream);
  if (e != cudaSuccess) return e;
  const int KH = dm.topk - 1;
  // the partial outputs are bf16 for the tensor-core kernels, fp32 otherwise
  const int part_elem_bytes = attn_tc_path(dtype, dm.d) ? 2 : 4;
  for (int ch = 0; ch < dm.nchunks; ++ch) {
    if (KH > 0) {
      const int t0 = ch * dm.chunk;
      const int len = (dm.N < t0 + dm.chunk ? dm.N : t0 + dm.chunk) - t0;
      const int64_t total = (int64_t)dm.batch * len * dm.hq * KH;
      pooled_fill_kernel<<<(unsigned)((total + kFillThreads - 1) / kFillThreads), kFillThreads, 0, stream>>>(
          sel, ws.part_o, ws.part_lse, dm, ch, part_elem_bytes);
      ++*launches;
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    e = launch_attn_passes(dm, dtype, q, k, v, sel, offsets, rows, out, lse, ws, ch, ch + 1, stream,
                           launches);
    if (e != cudaSuccess) return e;
  }
  return e;
}

}  // namespace moba
