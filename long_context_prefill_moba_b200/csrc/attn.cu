// Orchestration of the attention step: the query range is processed in passes
// of `chunk` tokens.  Each pass runs the historical-block kernel (partials into
// the workspace) and then the current-block kernel, which merges them.
#include "launch.h"

namespace moba {

// tile prefix of one pass: tile_start[i] = sum over groups i' < i of
// ceil(rows of group i' / tm), and tile_start[ngroups] = the pass's tile count
// (one block; a warp-shuffle scan per 1024 groups, carried across chunks)
__global__ void attn_plan_kernel(const int32_t* __restrict__ offsets, int ngroups, int tm,
                                 int32_t* __restrict__ tile_start) {
  __shared__ int32_t warp_tot[32];
  __shared__ int32_t carry;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  for (int base = 0; base < ngroups; base += blockDim.x) {
    const int i = base + threadIdx.x;
    const int32_t x = i < ngroups ? (offsets[i + 1] - offsets[i] + tm - 1) / tm : 0;
    int32_t incl = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int32_t y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) warp_tot[wid] = incl;
    __syncthreads();
    if (wid == 0) {
      int32_t w = lane < (int)(blockDim.x >> 5) ? warp_tot[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        int32_t y = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += y;
      }
      warp_tot[lane] = w;
    }
    __syncthreads();
    const int32_t before = carry + (wid > 0 ? warp_tot[wid - 1] : 0) + incl - x;
    if (i < ngroups) tile_start[i] = before;
    __syncthreads();
    if (threadIdx.x == blockDim.x - 1) carry = before + x;
    __syncthreads();
  }
  if (threadIdx.x == 0) tile_start[ngroups] = carry;
}

cudaError_t launch_attn_tc_hist(const Dims& dm, const void* q, const void* k, const void* v,
                                const int32_t* sel, const int32_t* offsets, const int32_t* rows,
                                const AttnWs& ws, int ch, int64_t grid, cudaStream_t stream);
cudaError_t launch_attn_tc_cur(const Dims& dm, const void* q, const void* k, const void* v,
                               const AttnWs& ws, void* out, float* lse, int ch,
                               cudaStream_t stream);
int attn_tc_rows_per_tile();
cudaError_t launch_attn_f32_hist(const Dims& dm, const void* q, const void* k, const void* v,
                                 const int32_t* sel, const int32_t* offsets, const int32_t* rows,
                                 const AttnWs& ws, int ch, int64_t nrows, cudaStream_t stream);
cudaError_t launch_attn_f32_cur(const Dims& dm, const void* q, const void* k, const void* v,
                                const AttnWs& ws, void* out, float* lse, int ch,
                                cudaStream_t stream);

int64_t hist_rows_range(int64_t t0, int64_t t1, int64_t B, int64_t KH) {
  int64_t total = 0;
  int64_t t = t0;
  while (t < t1) {
    const int64_t c = t / B;
    const int64_t e = (c + 1) * B < t1 ? (c + 1) * B : t1;
    total += (e - t) * (c < KH ? c : KH);
    t = e;
  }
  return total;
}

cudaError_t launch_attn_passes(const Dims& dm, int dtype, const void* q, const void* k,
                               const void* v, const int32_t* sel, const int32_t* offsets,
                               const int32_t* rows, void* out, float* lse, AttnWs ws, int ch_begin,
                               int ch_end, cudaStream_t stream, int* launches) {
  const int KH = dm.topk - 1;
  const int ngroups = dm.batch * dm.hkv * dm.n;
  cudaError_t e = cudaSuccess;
  // bf16 (head_dim 128 or 64): tensor-core (tcgen05) kernels for both attention
  // steps; fp32: the CUDA-core kernels
  const bool tc = attn_tc_path(dtype, dm.d);
  if (!tc && dtype == MOBA_BF16) return cudaErrorInvalidValue;
  const int tm = attn_tc_rows_per_tile();
  for (int ch = ch_begin; ch < ch_end; ++ch) {
    const int t0 = ch * dm.chunk;
    const int t1 = dm.N < t0 + dm.chunk ? dm.N : t0 + dm.chunk;
    const int64_t nrows = hist_rows_range(t0, t1, dm.B, KH) * dm.batch * dm.hq;
    if (nrows > 0) {
      if (tc) {
        attn_plan_kernel<<<1, 1024, 0, stream>>>(offsets + (size_t)ch * ngroups, ngroups, tm,
                                                 ws.tile_start);
        ++*launches;
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        const int cmax = (t1 - 1) / dm.B;
        const int64_t active = (int64_t)dm.batch * dm.hkv * (cmax < dm.n ? cmax : dm.n);
        const int64_t grid = nrows / tm + active + 1;
        e = launch_attn_tc_hist(dm, q, k, v, sel, offsets, rows, ws, ch, grid, stream);
      } else {
        e = launch_attn_f32_hist(dm, q, k, v, sel, offsets, rows, ws, ch, nrows, stream);
      }
      ++*launches;
      if (e != cudaSuccess) return e;
    }
    e = tc ? launch_attn_tc_cur(dm, q, k, v, ws, out, lse, ch, stream)
           : launch_attn_f32_cur(dm, q, k, v, ws, out, lse, ch, stream);
    ++*launches;
    if (e != cudaSuccess) return e;
  }
  return e;
}

cudaError_t launch_attn(const Dims& dm, int dtype, const void* q, const void* k, const void* v,
                        const int32_t* sel, const int32_t* offsets, const int32_t* rows, void* out,
                        float* lse, AttnWs ws, cudaStream_t stream, int* launches) {
  cudaError_t e = cudaMemsetAsync(ws.status, 0, sizeof(int), stream);
  if (e != cudaSuccess) return e;
  return launch_attn_passes(dm, dtype, q, k, v, sel, offsets, rows, out, lse, ws, 0, dm.nchunks,
                            stream, launches);
}

}  // namespace moba
