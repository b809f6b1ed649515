// K2: causal top-k gate and the query-per-block index.
//
// "MoBA: Mixture of Block Attention for Long-Context LLMs", paper-graph
// summary §3: "Affinity Scoring" (s_i = <q, mean_pool(K[I_i])>, no softmax
// scale), "Top-k Gating" (g_i = 1 iff s_i is among the top k; the current block
// is always routed, like a shared expert), "Causality Enforcement" mechanism 1
// (blocks that are not entirely in the past get s = -inf, g = 0) and the
// Implementation section, Algorithm 1 Steps 1-2 (S = Q meanK^T with a causal
// mask, top-k, then queries regrouped by the block they attend to).
//
// Three launches:
//   gate_select  one thread per query row: scores against the pooled keys of
//                all earlier blocks (fp32), running top-(topk-1) with ties to the
//                lower block index, writes the ascending selection list and
//                counts rows per (pass, b, kv head, block) through shared-memory
//                histograms (one global atomic per touched block per CTA).
//   gate_scan    exclusive prefix of the counts -> offsets.
//   gate_scatter one thread per query row: places each (row, earlier block)
//                into its group's range of `rows`.
#include <float.h>

#include "launch.h"

namespace moba {

namespace {

constexpr int kRows = 128;        // query rows (tokens of one (b, h)) per CTA
constexpr int kJChunk = 32;       // pooled keys staged in shared memory at a time
constexpr int kSmemHist = 4096;   // blocks counted in shared memory (else global)

template <typename T, int D>
__global__ void __launch_bounds__(kRows) gate_select_kernel(const T* __restrict__ q,
                                                            const float* __restrict__ meank,
                                                            int32_t* __restrict__ sel,
                                                            int32_t* __restrict__ counts, Dims dm) {
  __shared__ __align__(16) float kb[kJChunk * D];
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
  const int c_max = t_last / dm.B;              // largest current block in the tile
  const int KH = dm.topk - 1;                   // historical slots
  const bool use_hist = dm.n <= kSmemHist;
  const int j_lim = KH > 0 ? c_max : 0;         // topk == 1: nothing to score

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

  float ts[MOBA_MAX_TOPK];
  int ti[MOBA_MAX_TOPK];
#pragma unroll
  for (int i = 0; i < MOBA_MAX_TOPK; ++i) { ts[i] = -FLT_MAX; ti[i] = -1; }
  float thresh = -INFINITY;   // score of the last kept slot once the list is full
  int kept = 0;

  const float* kb_g = meank + ((size_t)b * dm.n * dm.hkv + g) * D;   // row j at + j*hkv*D
  for (int j0 = 0; j0 < j_lim; j0 += kJChunk) {
    const int jn = min(kJChunk, j_lim - j0);
    __syncthreads();
    for (int e = threadIdx.x * 4; e < jn * D; e += kRows * 4) {
      const int jj = e / D, col = e % D;
      *reinterpret_cast<float4*>(&kb[e]) =
          __ldg(reinterpret_cast<const float4*>(kb_g + (size_t)(j0 + jj) * dm.hkv * D + col));
    }
    __syncthreads();
    if (!valid) continue;
    const int jend = min(jn, c - j0);
    for (int jj = 0; jj < jend; ++jj) {
      const float4* kr = reinterpret_cast<const float4*>(&kb[jj * D]);
      float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
      for (int e = 0; e < D / 4; ++e) {
        float4 kv = kr[e];
        s0 = fmaf(qv[4 * e + 0], kv.x, s0);
        s1 = fmaf(qv[4 * e + 1], kv.y, s1);
        s2 = fmaf(qv[4 * e + 2], kv.z, s2);
        s3 = fmaf(qv[4 * e + 3], kv.w, s3);
      }
      const float s = (s0 + s1) + (s2 + s3);
      const int jidx = j0 + jj;
      // candidates arrive in increasing block index, so a tie never displaces
      // an entry already kept: the lower index wins
      if (kept < KH || s > thresh) {
        // insert into the descending list ts[0..KH): walk from the back
#pragma unroll
        for (int i = MOBA_MAX_TOPK - 1; i >= 0; --i) {
          if (i < KH) {
            const bool gt_prev = (i > 0) ? (s > ts[i > 0 ? i - 1 : 0]) : true;
            const bool gt_here = s > ts[i] || ti[i] < 0;
            if (i > 0 && gt_prev) {
              ts[i] = ts[i > 0 ? i - 1 : 0];
              ti[i] = ti[i > 0 ? i - 1 : 0];
            } else if (gt_here) {
              ts[i] = s;
              ti[i] = jidx;
            }
          }
        }
        kept = min(kept + 1, KH);
        // threshold = smallest kept score; a predicated min keeps indices compile-time
        thresh = INFINITY;
#pragma unroll
        for (int i = 0; i < MOBA_MAX_TOPK; ++i) thresh = fminf(thresh, i < KH ? ts[i] : INFINITY);
      }
    }
  }

  if (valid) {
    // ascending order of the kept blocks, then the current block, then -1
    int32_t* out = sel + ((size_t)(b * dm.N + t) * dm.hq + h) * dm.topk;
    const int m = min(KH, c);
    const int ch = t / dm.chunk;
    int32_t* cnt_g = counts + ((size_t)(ch * dm.batch + b) * dm.hkv + g) * dm.n;
#pragma unroll
    for (int i = 0; i < MOBA_MAX_TOPK; ++i) {
      if (i < m) {
        int rank = 0;
#pragma unroll
        for (int i2 = 0; i2 < MOBA_MAX_TOPK; ++i2)
          if (i2 < m && ti[i2] < ti[i]) ++rank;
        out[rank] = ti[i];
        if (use_hist) atomicAdd(&hist[ti[i]], 1);
        else atomicAdd(&cnt_g[ti[i]], 1);
      }
    }
    out[m] = c;
    for (int i = m + 1; i < dm.topk; ++i) out[i] = -1;
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

// Exclusive prefix sum of `in` (len L) plus `base` into out[0..L]; one CTA.
constexpr int kScanThreads = 1024;
__global__ void __launch_bounds__(kScanThreads) gate_scan_kernel(const int32_t* __restrict__ in,
                                                                 int32_t* __restrict__ out,
                                                                 int64_t L, int32_t base) {
  __shared__ int32_t warp_tot[32];
  __shared__ int32_t carry;
  if (threadIdx.x == 0) carry = base;
  __syncthreads();
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  for (int64_t base = 0; base < L; base += kScanThreads) {
    const int64_t i = base + threadIdx.x;
    const int32_t x = i < L ? in[i] : 0;
    int32_t incl = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int32_t y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) warp_tot[wid] = incl;
    __syncthreads();
    if (wid == 0) {
      int32_t w = warp_tot[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        int32_t y = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += y;
      }
      warp_tot[lane] = w;   // inclusive over warps
    }
    __syncthreads();
    const int32_t before = carry + (wid > 0 ? warp_tot[wid - 1] : 0) + incl - x;
    if (i < L) out[i] = before;
    __syncthreads();
    if (threadIdx.x == kScanThreads - 1) carry = before + x;
    __syncthreads();
  }
  if (threadIdx.x == 0) out[L] = carry;
}

__global__ void __launch_bounds__(kRows) gate_scatter_kernel(const int32_t* __restrict__ sel,
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
  const int KH = dm.topk - 1;
  const bool use_hist = dm.n <= kSmemHist;
  const int ch = t_first / dm.chunk;
  const size_t grp0 = ((size_t)(ch * dm.batch + b) * dm.hkv + g) * dm.n;
  const int32_t r = (b * dm.N + t) * dm.hq + h;

  int js[MOBA_MAX_TOPK];
  int loc[MOBA_MAX_TOPK];
  int m = 0;
  if (valid) {
    const int32_t* srow = sel + (size_t)r * dm.topk;
    m = min(KH, t / dm.B);
#pragma unroll
    for (int i = 0; i < MOBA_MAX_TOPK; ++i) js[i] = (i < m) ? srow[i] : 0;
  }
  if (use_hist) {
    for (int i = threadIdx.x; i < c_max; i += kRows) cnt[i] = 0;
    __syncthreads();
#pragma unroll
    for (int i = 0; i < MOBA_MAX_TOPK; ++i)
      if (i < m) loc[i] = atomicAdd(&cnt[js[i]], 1);
    __syncthreads();
    for (int i = threadIdx.x; i < c_max; i += kRows)
      base[i] = cnt[i] ? atomicAdd(&cursors[grp0 + i], cnt[i]) : 0;
    __syncthreads();
#pragma unroll
    for (int i = 0; i < MOBA_MAX_TOPK; ++i)
      if (i < m) rows[offsets[grp0 + js[i]] + base[js[i]] + loc[i]] = r;
  } else {
#pragma unroll
    for (int i = 0; i < MOBA_MAX_TOPK; ++i)
      if (i < m) rows[offsets[grp0 + js[i]] + atomicAdd(&cursors[grp0 + js[i]], 1)] = r;
  }
}

template <typename T>
cudaError_t launch_select(const Dims& dm, const void* q, const float* meank, int32_t* sel,
                          int32_t* counts, cudaStream_t stream) {
  const int tiles = (dm.t_hi - dm.t_lo + kRows - 1) / kRows;
  dim3 grid(tiles * dm.batch * dm.hq);
  if (dm.d == 128)
    gate_select_kernel<T, 128><<<grid, kRows, 0, stream>>>(static_cast<const T*>(q), meank, sel,
                                                           counts, dm);
  else
    gate_select_kernel<T, 64><<<grid, kRows, 0, stream>>>(static_cast<const T*>(q), meank, sel,
                                                          counts, dm);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gate_scan(const int32_t* in, int32_t* out, int64_t L, int32_t base,
                             cudaStream_t stream) {
  gate_scan_kernel<<<1, kScanThreads, 0, stream>>>(in, out, L, base);
  return cudaGetLastError();
}

cudaError_t launch_gate(const Dims& dm, int dtype, const void* q, const float* meank, int32_t* sel,
                        int32_t* offsets, int32_t* rows, GateWs ws, cudaStream_t stream,
                        int* launches) {
  const int64_t L = (int64_t)dm.nchunks * dm.batch * dm.hkv * dm.n;
  cudaError_t e = cudaMemsetAsync(ws.counts, 0, sizeof(int32_t) * L * 2, stream);  // counts+cursors
  if (e != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(ws.status, 0, sizeof(int), stream)) != cudaSuccess) return e;
  if (gate_tc_supported(dm, dtype))
    e = launch_gate_select_tc(dm, q, meank, sel, ws.counts, ws.status, stream);
  else if (dtype == MOBA_BF16)
    e = launch_select<__nv_bfloat16>(dm, q, meank, sel, ws.counts, stream);
  else
    e = launch_select<float>(dm, q, meank, sel, ws.counts, stream);
  ++*launches;
  if (e != cudaSuccess) return e;
  gate_scan_kernel<<<1, kScanThreads, 0, stream>>>(ws.counts, offsets, L, 0);
  ++*launches;
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (dm.topk > 1) {
    const int tiles = (dm.t_hi - dm.t_lo + kRows - 1) / kRows;
    gate_scatter_kernel<<<tiles * dm.batch * dm.hq, kRows, 0, stream>>>(sel, offsets, ws.cursors,
                                                                        rows, dm);
    ++*launches;
    e = cudaGetLastError();
  }
  return e;
}

cudaError_t launch_gate_pass(const Dims& dm_all, int dtype, const void* q, const float* meank,
                             int32_t* sel, int32_t* offsets, int32_t* rows, GateWs ws, int pass,
                             cudaStream_t stream, int* launches) {
  Dims dm = dm_all;
  dm.t_lo = pass * dm.chunk;
  dm.t_hi = dm.N < dm.t_lo + dm.chunk ? dm.N : dm.t_lo + dm.chunk;
  const int64_t G0 = (int64_t)dm.batch * dm.hkv * dm.n;   // groups of one pass
  // rows of the earlier passes: every token t contributes min(topk - 1, t / B) per (b, h)
  const int64_t before = hist_rows_range(0, dm.t_lo, dm.B, dm.topk - 1) * dm.batch * dm.hq;
  cudaError_t e;
  if (gate_tc_supported(dm, dtype))
    e = launch_gate_select_tc(dm, q, meank, sel, ws.counts, ws.status, stream);
  else if (dtype == MOBA_BF16)
    e = launch_select<__nv_bfloat16>(dm, q, meank, sel, ws.counts, stream);
  else
    e = launch_select<float>(dm, q, meank, sel, ws.counts, stream);
  ++*launches;
  if (e != cudaSuccess) return e;
  gate_scan_kernel<<<1, kScanThreads, 0, stream>>>(ws.counts + pass * G0, offsets + pass * G0, G0,
                                                   (int32_t)before);
  ++*launches;
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (dm.topk > 1) {
    const int tiles = (dm.t_hi - dm.t_lo + kRows - 1) / kRows;
    gate_scatter_kernel<<<tiles * dm.batch * dm.hq, kRows, 0, stream>>>(sel, offsets, ws.cursors,
                                                                        rows, dm);
    ++*launches;
    e = cudaGetLastError();
  }
  return e;
}

}  // namespace moba

// ---------------------------------------------------------------------------
// Allocation-free gate: the scratch counters live in a fixed device array of
// this file instead of caller-provided memory (see moba_gate_topk_noalloc).
// ---------------------------------------------------------------------------
#include <mutex>

namespace {

constexpr int kNoAllocMaxDevices = 64;
constexpr int64_t kNoAllocStatusIndex = 2 * (int64_t)MOBA_GATE_NOALLOC_MAX_GROUPS;
static __device__ __align__(256) int32_t g_gate_scratch[2 * MOBA_GATE_NOALLOC_MAX_GROUPS + 64];

std::mutex g_scratch_mu;
int32_t* g_scratch_ptr[kNoAllocMaxDevices] = {};

// Device address of g_gate_scratch on the current device (looked up once per
// device; the host-side symbol itself is not a device address).
cudaError_t scratch_for_current_device(int32_t** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kNoAllocMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_gate_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = static_cast<int32_t*>(p);
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace

namespace moba {

cudaError_t launch_gate_noalloc(const Dims& dm, int dtype, const void* q, const float* meank,
                                int32_t* sel, int32_t* offsets, int32_t* rows,
                                cudaStream_t stream, int* launches) {
  int32_t* scratch = nullptr;
  cudaError_t e = scratch_for_current_device(&scratch);
  if (e != cudaSuccess) return e;
  const int64_t L = (int64_t)dm.nchunks * dm.batch * dm.hkv * dm.n;
  // counts, cursors (launch_gate clears them) and the status word, which sits
  // at a fixed index whatever the shape so that moba_gate_noalloc_status finds it
  GateWs ws{scratch, scratch + L, scratch + kNoAllocStatusIndex};
  return launch_gate(dm, dtype, q, meank, sel, offsets, rows, ws, stream, launches);
}

cudaError_t gate_noalloc_status(int* host_status, cudaStream_t stream) {
  int32_t* scratch = nullptr;
  cudaError_t e = scratch_for_current_device(&scratch);
  if (e != cudaSuccess) return e;
  return cudaMemcpyAsync(host_status, scratch + kNoAllocStatusIndex, sizeof(int), cudaMemcpyDeviceToHost,
                         stream);
}

}  // namespace moba
