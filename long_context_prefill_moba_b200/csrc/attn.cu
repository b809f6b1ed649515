// Orchestration of the attention step: the query range is processed in passes
// of `chunk` tokens.  Each pass runs the historical-block kernel (partials into
// the workspace) and then the current-block kernel, which merges them.
#include "launch.h"

namespace moba {

__global__ void attn_plan_kernel(const int32_t* __restrict__ offsets, int ngroups, int tm,
                                 int32_t* __restrict__ tile_start);
cudaError_t launch_attn_mma_hist(const Dims& dm, const void* q, const void* k, const void* v,
                                 const int32_t* sel, const int32_t* offsets, const int32_t* rows,
                                 const AttnWs& ws, int ch, int64_t grid, cudaStream_t stream);
cudaError_t launch_attn_mma_cur(const Dims& dm, const void* q, const void* k, const void* v,
                                const AttnWs& ws, void* out, float* lse, int ch,
                                cudaStream_t stream);
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
  // bf16 with head_dim 128: tensor-core (tcgen05) kernels for both attention steps
  const bool tc = dtype == MOBA_BF16 && dm.d == 128;
  const int tm = tc ? attn_tc_rows_per_tile() : 64;
  for (int ch = ch_begin; ch < ch_end; ++ch) {
    const int t0 = ch * dm.chunk;
    const int t1 = dm.N < t0 + dm.chunk ? dm.N : t0 + dm.chunk;
    const int64_t nrows = hist_rows_range(t0, t1, dm.B, KH) * dm.batch * dm.hq;
    if (nrows > 0) {
      if (dtype == MOBA_BF16) {
        attn_plan_kernel<<<1, 1024, 0, stream>>>(offsets + (size_t)ch * ngroups, ngroups, tm,
                                                 ws.tile_start);
        ++*launches;
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        const int cmax = (t1 - 1) / dm.B;
        const int64_t active = (int64_t)dm.batch * dm.hkv * (cmax < dm.n ? cmax : dm.n);
        const int64_t grid = nrows / tm + active + 1;
        e = tc ? launch_attn_tc_hist(dm, q, k, v, sel, offsets, rows, ws, ch, grid, stream)
               : launch_attn_mma_hist(dm, q, k, v, sel, offsets, rows, ws, ch, grid, stream);
      } else {
        e = launch_attn_f32_hist(dm, q, k, v, sel, offsets, rows, ws, ch, nrows, stream);
      }
      ++*launches;
      if (e != cudaSuccess) return e;
    }
    e = tc ? launch_attn_tc_cur(dm, q, k, v, ws, out, lse, ch, stream)
           : dtype == MOBA_BF16 ? launch_attn_mma_cur(dm, q, k, v, ws, out, lse, ch, stream)
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
