// Backward of the attention step (dq, dk, dv given dout) on CUDA cores in
// fp32, for every dtype and head size.
//
// "MoBA: Mixture of Block Attention for Long-Context LLMs", paper-graph summary
// §3 "The Core MoBA Attention Equation" (Softmax(q K[I]^T) V[I] over the key set
// I the gate chose) and "Causality Enforcement" (causal inside the current
// block).  The gate's selection is held fixed (its derivative is zero almost
// everywhere; the pages print no backward formula).  For a row r with logits
// z_u = scale <q_r, k_u> and the forward's log-sum-exp L_r:
//   p_ru = exp(z_u - L_r), D_r = <dout_r, out_r>, ds_ru = p_ru (<dout_r, v_u> - D_r),
//   dq_r = scale sum_u ds_ru k_u,  dk_u = scale sum_r ds_ru q_r,  dv_u = sum_r p_ru dout_r,
// where the sums over r run over every query row whose key set contains u:
// the rows of u's own block at or after u (all query heads of the kv group)
// and the rows the gate routed to u's block (the `rows` index of every pass).
//
// Three launches: bwd_delta (D_r), bwd_dq (one warp per query row), bwd_dkv
// (one warp per key).  Every output element is written once (no atomics), so
// for one gate index the result is bitwise reproducible.  bf16 layers with
// head_dim 128 run the tensor-core kernels of attn_bwd_tc.cu instead (after
// the same bwd_delta).
#include "launch.h"

namespace moba {

namespace {

constexpr int kWarps = 4;

template <typename T, int D>
MOBA_DEV void load_row(const T* src, float* dst) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int x = 0; x < D / 32; ++x) dst[lane + 32 * x] = to_f32(src[lane + 32 * x]);
}

// D_r = <dout_r, out_r>, one warp per row
template <typename T, int D>
__global__ void __launch_bounds__(kWarps * 32) bwd_delta_kernel(const T* __restrict__ out,
                                                                const T* __restrict__ dout,
                                                                float* __restrict__ delta, int64_t nrows) {
  const int lane = threadIdx.x & 31;
  const int64_t r = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (r >= nrows) return;
  float s = 0.f;
#pragma unroll
  for (int x = 0; x < D / 32; ++x) {
    const size_t e = (size_t)r * D + lane + 32 * x;
    s = fmaf(to_f32(out[e]), to_f32(dout[e]), s);
  }
  s = warp_sum(s);
  if (lane == 0) delta[r] = s;
}

// dq_r over the row's key set: keys of each selected earlier block and of the
// current block up to t; lanes take 32 keys at a time for the dot products,
// then every lane accumulates its D/32 columns of dq
template <typename T, int D>
__global__ void __launch_bounds__(kWarps * 32) bwd_dq_kernel(
    const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v, const T* __restrict__ dout,
    const float* __restrict__ lse, const float* __restrict__ delta, const int32_t* __restrict__ sel,
    T* __restrict__ dq, Dims dm) {
  __shared__ float qs[kWarps][D], ds_[kWarps][D];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t nrows = (int64_t)dm.batch * dm.N * dm.hq;
  const int64_t r = (int64_t)blockIdx.x * kWarps + warp;
  if (r >= nrows) return;
  const int h = (int)(r % dm.hq);
  const int t = (int)((r / dm.hq) % dm.N);
  const int b = (int)(r / ((int64_t)dm.hq * dm.N));
  const int g = h / dm.G;
  const int c = t / dm.B;
  load_row<T, D>(q + (size_t)r * D, qs[warp]);
  load_row<T, D>(dout + (size_t)r * D, ds_[warp]);
  __syncwarp();
  const float L2 = lse[((size_t)b * dm.hq + h) * dm.N + t] * kLog2e;
  const float Dr = delta[r];
  const size_t kstride = (size_t)dm.hkv * D;
  const T* kb = k + ((size_t)b * dm.N * dm.hkv + g) * D;
  const T* vb = v + ((size_t)b * dm.N * dm.hkv + g) * D;
  float acc[D / 32];
#pragma unroll
  for (int x = 0; x < D / 32; ++x) acc[x] = 0.f;
  const int32_t* srow = sel + (size_t)r * dm.topk;
  for (int i = 0; i < dm.topk; ++i) {
    const int j = srow[i];
    if (j < 0) break;
    const int u0 = j * dm.B;
    const int u1 = j == c ? t + 1 : min(dm.N, u0 + dm.B);
    for (int base = u0; base < u1; base += 32) {
      const int u = base + lane;
      float dsu = 0.f;
      if (u < u1) {
        const T* kr = kb + (size_t)u * kstride;
        const T* vr = vb + (size_t)u * kstride;
        float s = 0.f, dp = 0.f;
#pragma unroll 8
        for (int e = 0; e < D; ++e) {
          s = fmaf(qs[warp][e], to_f32(kr[e]), s);
          dp = fmaf(ds_[warp][e], to_f32(vr[e]), dp);
        }
        const float p = exp2f(s * dm.scale_log2 - L2);
        dsu = p * (dp - Dr);
      }
      const int lim = min(32, u1 - base);
      for (int i2 = 0; i2 < lim; ++i2) {
        const float w = __shfl_sync(0xffffffffu, dsu, i2);
        const T* kr = kb + (size_t)(base + i2) * kstride;
#pragma unroll
        for (int x = 0; x < D / 32; ++x) acc[x] = fmaf(w, to_f32(kr[lane + 32 * x]), acc[x]);
      }
    }
  }
  const float scale = dm.scale_log2 / kLog2e;
#pragma unroll
  for (int x = 0; x < D / 32; ++x) dq[(size_t)r * D + lane + 32 * x] = from_f32<T>(acc[x] * scale);
}

// dk_u, dv_u for one key u of kv head g: the rows of u's block at or after u
// (every query head of the group), then the rows every pass routed to u's block
template <typename T, int D>
__global__ void __launch_bounds__(kWarps * 32) bwd_dkv_kernel(
    const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v, const T* __restrict__ dout,
    const float* __restrict__ lse, const float* __restrict__ delta, const int32_t* __restrict__ offsets,
    const int32_t* __restrict__ rows, T* __restrict__ dk, T* __restrict__ dv, Dims dm) {
  __shared__ float ks[kWarps][D], vs[kWarps][D];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t nkeys = (int64_t)dm.batch * dm.N * dm.hkv;
  const int64_t key = (int64_t)blockIdx.x * kWarps + warp;   // (b * N + u) * hkv + g
  if (key >= nkeys) return;
  const int g = (int)(key % dm.hkv);
  const int u = (int)((key / dm.hkv) % dm.N);
  const int b = (int)(key / ((int64_t)dm.hkv * dm.N));
  const int j = u / dm.B;
  load_row<T, D>(k + (size_t)key * D, ks[warp]);
  load_row<T, D>(v + (size_t)key * D, vs[warp]);
  __syncwarp();
  float gk[D / 32], gv[D / 32];
#pragma unroll
  for (int x = 0; x < D / 32; ++x) gk[x] = gv[x] = 0.f;

  // one batch of up to 32 rows (lane i holds row ids[i]): dot products per
  // lane, then every lane accumulates its columns over the batch
  auto batch = [&](int64_t rr, bool live) {
    float p = 0.f, dsr = 0.f;
    if (live) {
      const int h = (int)(rr % dm.hq);
      const int t = (int)((rr / dm.hq) % dm.N);
      const T* qr = q + (size_t)rr * D;
      const T* dr = dout + (size_t)rr * D;
      float s = 0.f, dp = 0.f;
#pragma unroll 8
      for (int e = 0; e < D; ++e) {
        s = fmaf(to_f32(qr[e]), ks[warp][e], s);
        dp = fmaf(to_f32(dr[e]), vs[warp][e], dp);
      }
      p = exp2f(s * dm.scale_log2 - lse[((size_t)b * dm.hq + h) * dm.N + t] * kLog2e);
      dsr = p * (dp - delta[rr]);
    }
    for (int i = 0; i < 32; ++i) {
      const int64_t ri = __shfl_sync(0xffffffffu, rr, i);
      const float pi = __shfl_sync(0xffffffffu, p, i);
      const float si = __shfl_sync(0xffffffffu, dsr, i);
      if (__shfl_sync(0xffffffffu, (int)live, i) == 0) continue;
      const T* qr = q + (size_t)ri * D;
      const T* dr = dout + (size_t)ri * D;
#pragma unroll
      for (int x = 0; x < D / 32; ++x) {
        gk[x] = fmaf(si, to_f32(qr[lane + 32 * x]), gk[x]);
        gv[x] = fmaf(pi, to_f32(dr[lane + 32 * x]), gv[x]);
      }
    }
  };

  // the key's own block: tokens u .. block end, every query head of group g
  const int t_end = min(dm.N, (j + 1) * dm.B);
  const int64_t own = (int64_t)(t_end - u) * dm.G;
  for (int64_t base = 0; base < own; base += 32) {
    const int64_t i = base + lane;
    const bool live = i < own;
    const int t = u + (int)(live ? i / dm.G : 0);
    const int h = g * dm.G + (int)(live ? i % dm.G : 0);
    batch(((int64_t)b * dm.N + t) * dm.hq + h, live);
  }
  // rows routed to block j by every pass
  const int64_t ngroups = (int64_t)dm.batch * dm.hkv * dm.n;
  for (int ch = 0; ch < dm.nchunks; ++ch) {
    const int64_t gi = ch * ngroups + ((int64_t)b * dm.hkv + g) * dm.n + j;
    const int r0 = offsets[gi], r1 = offsets[gi + 1];
    for (int base = r0; base < r1; base += 32) {
      const int i = base + lane;
      const bool live = i < r1;
      batch(live ? (int64_t)rows[i] : 0, live);
    }
  }
  const float scale = dm.scale_log2 / kLog2e;
#pragma unroll
  for (int x = 0; x < D / 32; ++x) {
    dk[(size_t)key * D + lane + 32 * x] = from_f32<T>(gk[x] * scale);
    dv[(size_t)key * D + lane + 32 * x] = from_f32<T>(gv[x]);
  }
}

template <typename T, int D>
cudaError_t launch_all(const Dims& dm, const void* q, const void* k, const void* v, const void* out,
                       const void* dout, const float* lse, const int32_t* sel, const int32_t* offsets,
                       const int32_t* rows, void* dq, void* dk, void* dv, float* delta, cudaStream_t stream,
                       int* launches) {
  const int64_t nrows = (int64_t)dm.batch * dm.N * dm.hq;
  const int64_t nkeys = (int64_t)dm.batch * dm.N * dm.hkv;
  bwd_delta_kernel<T, D><<<(nrows + kWarps - 1) / kWarps, kWarps * 32, 0, stream>>>(
      (const T*)out, (const T*)dout, delta, nrows);
  ++*launches;
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  bwd_dq_kernel<T, D><<<(nrows + kWarps - 1) / kWarps, kWarps * 32, 0, stream>>>(
      (const T*)q, (const T*)k, (const T*)v, (const T*)dout, lse, delta, sel, (T*)dq, dm);
  ++*launches;
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  bwd_dkv_kernel<T, D><<<(nkeys + kWarps - 1) / kWarps, kWarps * 32, 0, stream>>>(
      (const T*)q, (const T*)k, (const T*)v, (const T*)dout, lse, delta, offsets, rows, (T*)dk, (T*)dv, dm);
  ++*launches;
  return cudaGetLastError();
}

}  // namespace

__global__ void attn_plan_kernel(const int32_t* __restrict__ offsets, int ngroups, int tm,
                                 int32_t* __restrict__ tile_start);
int attn_bwd_tc_rows_per_tile();
cudaError_t launch_bwd_kv_tc(const Dims& dm, const void* q, const void* k, const void* v, const void* dout,
                             const float* lse, const float* delta, const int32_t* offsets, const int32_t* rows,
                             void* dk, void* dv, int* status, cudaStream_t stream);
cudaError_t launch_bwd_q_tc(const Dims& dm, bool cur, const void* q, const void* k, const void* v,
                            const void* dout, const float* lse, const float* delta, const int32_t* offsets,
                            const int32_t* rows, const int32_t* tile_start, float* dqacc, int* status, int ch,
                            int64_t grid, cudaStream_t stream);
cudaError_t launch_dq_convert(const float* acc, void* dq, int64_t n, cudaStream_t stream);

bool attn_bwd_tc_path(const Dims& dm, int dtype) { return dtype == MOBA_BF16 && dm.d == 128; }

cudaError_t launch_attn_bwd(const Dims& dm, int dtype, const void* q, const void* k, const void* v,
                            const void* out, const void* dout, const float* lse, const int32_t* sel,
                            const int32_t* offsets, const int32_t* rows, void* dq, void* dk, void* dv,
                            BwdWs ws, cudaStream_t stream, int* launches) {
  if (attn_bwd_tc_path(dm, dtype)) {
    const int64_t nrows = (int64_t)dm.batch * dm.N * dm.hq;
    cudaError_t e = cudaMemsetAsync(ws.dqacc, 0, sizeof(float) * nrows * dm.d, stream);
    if (e != cudaSuccess) return e;
    bwd_delta_kernel<__nv_bfloat16, 128><<<(nrows + kWarps - 1) / kWarps, kWarps * 32, 0, stream>>>(
        (const __nv_bfloat16*)out, (const __nv_bfloat16*)dout, ws.delta, nrows);
    ++*launches;
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // dk, dv: one CTA per 128-key tile
    e = launch_bwd_kv_tc(dm, q, k, v, dout, lse, ws.delta, offsets, rows, dk, dv, ws.status, stream);
    ++*launches;
    if (e != cudaSuccess) return e;
    // dq of the routed rows, pass by pass (row tiles of one gate group), then of the own block
    const int KH = dm.topk - 1;
    const int ngroups = dm.batch * dm.hkv * dm.n;
    const int tm = attn_bwd_tc_rows_per_tile();
    for (int ch = 0; ch < dm.nchunks && KH > 0; ++ch) {
      const int t0 = ch * dm.chunk;
      const int t1 = dm.N < t0 + dm.chunk ? dm.N : t0 + dm.chunk;
      const int64_t nr = hist_rows_range(t0, t1, dm.B, KH) * dm.batch * dm.hq;
      if (nr == 0) continue;
      attn_plan_kernel<<<1, 1024, 0, stream>>>(offsets + (size_t)ch * ngroups, ngroups, tm, ws.tile_start);
      ++*launches;
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
      const int cmax = (t1 - 1) / dm.B;
      const int64_t active = (int64_t)dm.batch * dm.hkv * (cmax < dm.n ? cmax : dm.n);
      e = launch_bwd_q_tc(dm, false, q, k, v, dout, lse, ws.delta, offsets, rows, ws.tile_start, ws.dqacc,
                          ws.status, ch, nr / tm + active + 1, stream);
      ++*launches;
      if (e != cudaSuccess) return e;
    }
    e = launch_bwd_q_tc(dm, true, q, k, v, dout, lse, ws.delta, offsets, rows, ws.tile_start, ws.dqacc,
                        ws.status, 0, 0, stream);
    ++*launches;
    if (e != cudaSuccess) return e;
    e = launch_dq_convert(ws.dqacc, dq, nrows * dm.d, stream);
    ++*launches;
    return e;
  }
  if (dtype == MOBA_BF16)
    return dm.d == 128 ? launch_all<__nv_bfloat16, 128>(dm, q, k, v, out, dout, lse, sel, offsets, rows, dq,
                                                        dk, dv, ws.delta, stream, launches)
                       : launch_all<__nv_bfloat16, 64>(dm, q, k, v, out, dout, lse, sel, offsets, rows, dq,
                                                       dk, dv, ws.delta, stream, launches);
  return dm.d == 128 ? launch_all<float, 128>(dm, q, k, v, out, dout, lse, sel, offsets, rows, dq, dk, dv,
                                              ws.delta, stream, launches)
                     : launch_all<float, 64>(dm, q, k, v, out, dout, lse, sel, offsets, rows, dq, dk, dv,
                                             ws.delta, stream, launches);
}

}  // namespace moba
