// K1: block mean-pool of the keys.
//
// "MoBA: Mixture of Block Attention for Long-Context LLMs", paper-graph
// summary §3 "Affinity Scoring": each block is represented by the mean of its
// key rows, computed once per layer (Algorithm 1 Step 1, pooled keys n x h x d).
//
// HBM-bound: every key byte is read exactly once with 16-byte coalesced loads.
// One CTA reduces one (batch, block, column slice): the warps of the CTA walk
// disjoint rows of the block, sum runs of four rows in fp32 and the runs in
// fp64 registers, and combine through shared memory in a fixed order
// (deterministic result); the mean is rounded to fp32 once, so the pooled keys
// carry no error of a long fp32 running sum even for blocks of 40960 rows.
#include "launch.h"

namespace moba {

namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;   // the fp32 run below adds exactly four rows

template <typename T>
__global__ void __launch_bounds__(kThreads) meanpool_kernel(const T* __restrict__ k,
                                                            float* __restrict__ meank, int N, int W,
                                                            int B, int n, int j0) {
  constexpr int V = Vec16<T>::kN;            // elements per 16-byte load
  const int vecs_per_row = W / V;             // W = hkv * d is a multiple of V
  const int cols_cta = min(vecs_per_row, kThreads);
  const int rows_per_pass = kThreads / cols_cta;
  const int tid = threadIdx.x;
  const int cvec = blockIdx.x * cols_cta + (tid % cols_cta);
  const int rsub = tid / cols_cta;
  const int j = j0 + blockIdx.y;
  const int b = blockIdx.z;
  const int t0 = j * B;
  const int t1 = min(N, t0 + B);
  const bool active = (rsub < rows_per_pass) && (cvec < vecs_per_row);

  // runs of kUnroll rows are summed in fp32 (pairwise), the runs in fp64: the
  // pooled key is the fp32 rounding of a sum with ~1e-16 relative error, not
  // of a long fp32 running sum
  double acc[V];
#pragma unroll
  for (int i = 0; i < V; ++i) acc[i] = 0.0;

  if (active) {
    const T* base = k + ((size_t)b * N) * W + (size_t)cvec * V;
    int t = t0 + rsub;
    for (; t + (kUnroll - 1) * rows_per_pass < t1; t += kUnroll * rows_per_pass) {
      float x[kUnroll][V];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) Vec16<T>::load(base + (size_t)(t + u * rows_per_pass) * W, x[u]);
#pragma unroll
      for (int i = 0; i < V; ++i) acc[i] += (double)((x[0][i] + x[1][i]) + (x[2][i] + x[3][i]));
    }
    for (; t < t1; t += rows_per_pass) {
      float x[V];
      Vec16<T>::load(base + (size_t)t * W, x);
#pragma unroll
      for (int i = 0; i < V; ++i) acc[i] += (double)x[i];
    }
  }

  // combine the row-groups of the CTA: [rows_per_pass][cols_cta * V]
  __shared__ double red[kThreads * V];
  if (rsub < rows_per_pass) {
#pragma unroll
    for (int i = 0; i < V; ++i) red[rsub * cols_cta * V + (tid % cols_cta) * V + i] = acc[i];
  }
  __syncthreads();
  const double len = (double)(t1 - t0);
  for (int e = tid; e < cols_cta * V; e += kThreads) {
    const int col = blockIdx.x * cols_cta * V + e;
    if (col >= W) continue;
    double s = 0.0;
    for (int r = 0; r < rows_per_pass; ++r) s += red[r * cols_cta * V + e];
    meank[((size_t)b * n + j) * W + col] = (float)(s / len);
  }
}

}  // namespace

cudaError_t launch_meanpool_blocks(const Dims& dm, int dtype, const void* k, float* meank, int j0,
                                   int j1, cudaStream_t stream, int* launches) {
  if (j1 <= j0) return cudaSuccess;
  const int W = dm.hkv * dm.d;
  const int V = dtype == MOBA_BF16 ? 8 : 4;
  const int vecs_per_row = W / V;
  const int cols_cta = vecs_per_row < kThreads ? vecs_per_row : kThreads;
  dim3 grid((vecs_per_row + cols_cta - 1) / cols_cta, j1 - j0, dm.batch);
  if (dtype == MOBA_BF16)
    meanpool_kernel<__nv_bfloat16><<<grid, kThreads, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(k), meank, dm.N, W, dm.B, dm.n, j0);
  else
    meanpool_kernel<float><<<grid, kThreads, 0, stream>>>(static_cast<const float*>(k), meank, dm.N,
                                                           W, dm.B, dm.n, j0);
  ++*launches;
  return cudaGetLastError();
}

cudaError_t launch_meanpool(const Dims& dm, int dtype, const void* k, float* meank,
                            cudaStream_t stream, int* launches) {
  return launch_meanpool_blocks(dm, dtype, k, meank, 0, dm.n, stream, launches);
}

}  // namespace moba
