// K3 (fp32 inputs): the same two attention steps as the bf16 kernels, on CUDA
// cores in fp32, one warp per query row.  Used for fp32 layers (small parity
// workloads); the mathematics and the partial-result layout are those of the
// bf16 path ("MoBA: Mixture of Block Attention for Long-Context LLMs",
// paper-graph summary §3 "The Core MoBA Attention Equation", "Causality
// Enforcement", Implementation Steps 3-4).
#include "launch.h"

namespace moba {

namespace {

constexpr int kWarps = 4;

// online softmax over keys [u0, u1) of one kv head for the query in qs;
// o[] holds this lane's D/32 output columns (unnormalised), m and l the
// running max (log2 units) and sum
template <int D>
MOBA_DEV void attend_range(const float* qs, const float* kb, const float* vb, size_t kstride, int u0,
                           int u1, float sl2, float* o, float& m, float& l) {
  const int lane = threadIdx.x & 31;
  for (int base = u0; base < u1; base += 32) {
    const int u = base + lane;
    float z = -INFINITY;
    if (u < u1) {
      const float* kr = kb + (size_t)u * kstride;
      float s = 0.f;
#pragma unroll 8
      for (int e = 0; e < D; ++e) s = fmaf(qs[e], kr[e], s);
      z = s * sl2;
    }
    const float mx = warp_max(z);
    const float m_new = fmaxf(m, mx);
    const float corr = exp2f(m - m_new);
    const float p = exp2f(z - m_new);
    l = l * corr + warp_sum(p);
    m = m_new;
#pragma unroll
    for (int x = 0; x < D / 32; ++x) o[x] *= corr;
    const int lim = min(32, u1 - base);
    for (int i = 0; i < lim; ++i) {
      const float pi = __shfl_sync(0xffffffffu, p, i);
      const float* vr = vb + (size_t)(base + i) * kstride;
#pragma unroll
      for (int x = 0; x < D / 32; ++x) o[x] = fmaf(pi, vr[lane + 32 * x], o[x]);
    }
  }
}

template <int D>
__global__ void __launch_bounds__(kWarps * 32) attn_hist_f32_kernel(
    const float* __restrict__ q, const float* __restrict__ k, const float* __restrict__ v,
    const int32_t* __restrict__ sel, const int32_t* __restrict__ offsets,
    const int32_t* __restrict__ rows, float* __restrict__ part_o, float* __restrict__ part_lse,
    Dims dm, int ch, int nrows) {
  __shared__ float qsm[kWarps][D];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int w = blockIdx.x * kWarps + warp;
  if (w >= nrows) return;
  const int ngroups = dm.batch * dm.hkv * dm.n;
  const int32_t* off = offsets + (size_t)ch * ngroups;
  const int p = off[0] + w;
  if (p >= off[ngroups]) return;   // nrows may be an upper bound (pooled gate)
  int lo = 0, hi = ngroups - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (off[mid] <= p) lo = mid; else hi = mid - 1;
  }
  const int j = lo % dm.n, g = (lo / dm.n) % dm.hkv, b = lo / (dm.n * dm.hkv);
  const int r = rows[p];
  const int h = r % dm.hq, t = (r / dm.hq) % dm.N;
  const int KH = dm.topk - 1;
  const int slot = slot_of(sel + (size_t)r * dm.topk, dm.topk, j);
  const size_t pidx = (size_t)((b * dm.chunk + (t - ch * dm.chunk)) * dm.hq + h) * KH + slot;

  for (int e = lane; e < D; e += 32) qsm[warp][e] = q[(size_t)r * D + e];
  __syncwarp();
  const size_t kstride = (size_t)dm.hkv * D;
  const float* kb = k + ((size_t)b * dm.N * dm.hkv + g) * D;
  const float* vb = v + ((size_t)b * dm.N * dm.hkv + g) * D;
  float o[D / 32] = {};
  float m = -INFINITY, l = 0.f;
  attend_range<D>(qsm[warp], kb, vb, kstride, j * dm.B, (j + 1) * dm.B, dm.scale_log2, o, m, l);
  const float inv = 1.f / l;
#pragma unroll
  for (int x = 0; x < D / 32; ++x) part_o[pidx * D + lane + 32 * x] = o[x] * inv;
  if (lane == 0) part_lse[pidx] = m + log2f(l);
}

template <int D>
__global__ void __launch_bounds__(kWarps * 32) attn_cur_f32_kernel(
    const float* __restrict__ q, const float* __restrict__ k, const float* __restrict__ v,
    const float* __restrict__ part_o, const float* __restrict__ part_lse, float* __restrict__ out,
    float* __restrict__ lse, Dims dm, int ch) {
  __shared__ float qsm[kWarps][D];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = ch * dm.chunk;
  const int len = min(dm.N, t0 + dm.chunk) - t0;
  const int w = blockIdx.x * kWarps + warp;
  if (w >= len * dm.batch * dm.hq) return;
  const int t = t0 + w % len;
  const int h = (w / len) % dm.hq;
  const int b = w / (len * dm.hq);
  const int g = h / dm.G;
  const size_t r = (size_t)(b * dm.N + t) * dm.hq + h;
  for (int e = lane; e < D; e += 32) qsm[warp][e] = q[r * D + e];
  __syncwarp();
  const size_t kstride = (size_t)dm.hkv * D;
  const float* kb = k + ((size_t)b * dm.N * dm.hkv + g) * D;
  const float* vb = v + ((size_t)b * dm.N * dm.hkv + g) * D;
  float o[D / 32] = {};
  float m = -INFINITY, l = 0.f;
  const int c = t / dm.B;
  attend_range<D>(qsm[warp], kb, vb, kstride, c * dm.B, t + 1, dm.scale_log2, o, m, l);

  const int KH = dm.topk - 1;
  const int nh = min(KH, c);
  const size_t pbase = (size_t)((b * dm.chunk + (t - t0)) * dm.hq + h) * KH;
  const float lse_cur = m + log2f(l);
  float M = lse_cur;
  for (int s = 0; s < nh; ++s) M = fmaxf(M, part_lse[pbase + s]);
  const float wc = exp2f(lse_cur - M);
  float W = wc;
  float acc[D / 32];
#pragma unroll
  for (int x = 0; x < D / 32; ++x) acc[x] = o[x] * (wc / l);
  for (int s = 0; s < nh; ++s) {
    const float ws = exp2f(part_lse[pbase + s] - M);
    W += ws;
#pragma unroll
    for (int x = 0; x < D / 32; ++x) acc[x] = fmaf(ws, part_o[(pbase + s) * D + lane + 32 * x], acc[x]);
  }
#pragma unroll
  for (int x = 0; x < D / 32; ++x) out[r * D + lane + 32 * x] = acc[x] / W;
  if (lse != nullptr && lane == 0) lse[((size_t)b * dm.hq + h) * dm.N + t] = (M + log2f(W)) * kLn2;
}

}  // namespace

cudaError_t launch_attn_f32_hist(const Dims& dm, const void* q, const void* k, const void* v,
                                 const int32_t* sel, const int32_t* offsets, const int32_t* rows,
                                 const AttnWs& ws, int ch, int64_t nrows, cudaStream_t stream) {
  const int64_t grid = (nrows + kWarps - 1) / kWarps;
  if (dm.d == 128)
    attn_hist_f32_kernel<128><<<grid, kWarps * 32, 0, stream>>>(
        (const float*)q, (const float*)k, (const float*)v, sel, offsets, rows, ws.part_o,
        ws.part_lse, dm, ch, (int)nrows);
  else
    attn_hist_f32_kernel<64><<<grid, kWarps * 32, 0, stream>>>(
        (const float*)q, (const float*)k, (const float*)v, sel, offsets, rows, ws.part_o,
        ws.part_lse, dm, ch, (int)nrows);
  return cudaGetLastError();
}

cudaError_t launch_attn_f32_cur(const Dims& dm, const void* q, const void* k, const void* v,
                                const AttnWs& ws, void* out, float* lse, int ch,
                                cudaStream_t stream) {
  const int t0 = ch * dm.chunk;
  const int len = (dm.N < t0 + dm.chunk ? dm.N : t0 + dm.chunk) - t0;
  const int64_t total = (int64_t)len * dm.batch * dm.hq;
  const int64_t grid = (total + kWarps - 1) / kWarps;
  if (dm.d == 128)
    attn_cur_f32_kernel<128><<<grid, kWarps * 32, 0, stream>>>(
        (const float*)q, (const float*)k, (const float*)v, ws.part_o, ws.part_lse, (float*)out, lse,
        dm, ch);
  else
    attn_cur_f32_kernel<64><<<grid, kWarps * 32, 0, stream>>>(
        (const float*)q, (const float*)k, (const float*)v, ws.part_o, ws.part_lse, (float*)out, lse,
        dm, ch);
  return cudaGetLastError();
}

}  // namespace moba
