// Host-side launchers of the MoBA kernels (internal to the library).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "common.cuh"

namespace moba {

// Every launcher enqueues on `stream`, adds the kernels it launched to
// *launches and returns the first CUDA error seen (cudaSuccess otherwise).

// rows entries contributed by tokens [t0, t1) of one (b, h): sum min(KH, t / B)
int64_t hist_rows_range(int64_t t0, int64_t t1, int64_t B, int64_t KH);

cudaError_t launch_meanpool(const Dims& dm, int dtype, const void* k, float* meank,
                            cudaStream_t stream, int* launches);
// blocks [j0, j1) only
cudaError_t launch_meanpool_blocks(const Dims& dm, int dtype, const void* k, float* meank, int j0,
                                   int j1, cudaStream_t stream, int* launches);

struct GateWs {
  int32_t* counts;   // [ngroups] rows per (chunk, b, g, j)
  int32_t* cursors;  // [ngroups] scatter cursors
  int* status;       // device status word: 0, or MOBA_ERR_TIMEOUT after a bounded wait expired
};

// tensor-core scores + selection (bf16, head_dim 128, at most 256 blocks)
bool gate_tc_supported(const Dims& dm, int dtype);
cudaError_t launch_gate_select_tc(const Dims& dm, const void* q, const float* meank, int32_t* sel,
                                  int32_t* counts, int* status, cudaStream_t stream);
// the pooled variant's three rankings on tensor cores (mean, max, min), the
// union written as the W-wide sel row (dm.topk = W) with its counts; requires
// gate_tc_pooled_supported (the row's candidate mask must fit its sel entries)
bool gate_tc_pooled_supported(const Dims& dm, int dtype);
cudaError_t launch_gate_select_tc_pooled(const Dims& dm, int km, int extra, const void* q,
                                         const float* meank, const float* maxk, const float* mink,
                                         int32_t* sel, int32_t* counts, int* status,
                                         cudaStream_t stream);
cudaError_t launch_gate(const Dims& dm, int dtype, const void* q, const float* meank, int32_t* sel,
                        int32_t* offsets, int32_t* rows, GateWs ws, cudaStream_t stream,
                        int* launches);

// the gate of one query pass (tokens [pass * chunk, +chunk)): selection,
// offsets of that pass's groups (continuing the earlier passes' rows) and the
// scatter; the counters of ws must be zero beforehand
cudaError_t launch_gate_pass(const Dims& dm, int dtype, const void* q, const float* meank,
                             int32_t* sel, int32_t* offsets, int32_t* rows, GateWs ws, int pass,
                             cudaStream_t stream, int* launches);

// moba_gate_topk with the counters in the library's fixed device array
// (requires nchunks * batch * hkv * n <= MOBA_GATE_NOALLOC_MAX_GROUPS)
cudaError_t launch_gate_noalloc(const Dims& dm, int dtype, const void* q, const float* meank,
                                int32_t* sel, int32_t* offsets, int32_t* rows,
                                cudaStream_t stream, int* launches);
// copy of the allocation-free gate's device status word into host memory, on `stream`
cudaError_t gate_noalloc_status(int* host_status, cudaStream_t stream);

// exclusive prefix sum of in[0..L) plus `base` into out[0..L] (one CTA)
cudaError_t launch_gate_scan(const int32_t* in, int32_t* out, int64_t L, int32_t base,
                             cudaStream_t stream);

// gate variant with max- and min-pooled keys (dm.topk = the selection width
// W = km + 1 + 2 * extra; km = slots of the mean ranking)
cudaError_t launch_maxminpool(const Dims& dm, int dtype, const void* k, float* maxk, float* mink,
                              cudaStream_t stream, int* launches);
cudaError_t launch_gate_pooled(const Dims& dm, int dtype, int km, int extra, const void* q,
                               const float* meank, const float* maxk, const float* mink, int32_t* sel,
                               int32_t* offsets, int32_t* rows, GateWs ws, cudaStream_t stream,
                               int* launches);

struct AttnWs {
  int* status;          // device status word: 0, or MOBA_ERR_TIMEOUT after a bounded wait expired
  float* part_o;        // [b * C * hq * (topk-1), d]  normalised partial outputs
  float* part_lse;      // [b * C * hq * (topk-1)]     their log2-sum-exp2
  int32_t* tile_start;  // [b * hkv * n + 1]           tile prefix of one pass
};
cudaError_t launch_attn(const Dims& dm, int dtype, const void* q, const void* k, const void* v,
                        const int32_t* sel, const int32_t* offsets, const int32_t* rows, void* out,
                        float* lse, AttnWs ws, cudaStream_t stream, int* launches);
// passes [ch_begin, ch_end) only, without resetting the status word
cudaError_t launch_attn_passes(const Dims& dm, int dtype, const void* q, const void* k,
                               const void* v, const int32_t* sel, const int32_t* offsets,
                               const int32_t* rows, void* out, float* lse, AttnWs ws, int ch_begin,
                               int ch_end, cudaStream_t stream, int* launches);

// the attention step over the pooled gate's selections (rows with fewer
// chosen blocks than the width allows): launch_attn plus the per-pass fill of
// the partial slots no historical tile writes
cudaError_t launch_attn_pooled(const Dims& dm, int dtype, const void* q, const void* k, const void* v,
                               const int32_t* sel, const int32_t* offsets, const int32_t* rows,
                               void* out, float* lse, AttnWs ws, cudaStream_t stream, int* launches);

// backward of the attention step: dq, dk, dv (in the input dtype) given dout,
// the forward's out and lse and the gate's sel/offsets/rows
struct BwdWs {
  int* status;          // device status word
  float* delta;         // [b * N * hq]      <dout, out> per row
  float* dqacc;         // [b * N * hq, d]   fp32 dq accumulator (tensor-core path)
  int32_t* tile_start;  // [b * hkv * n + 1] row-tile prefix of one pass (tensor-core path)
};
bool attn_bwd_tc_path(const Dims& dm, int dtype);
// the forward attention steps run on tcgen05, with bf16 partial results
// (bf16 with head_dim 128 or 64)
bool attn_tc_path(int dtype, int d);
cudaError_t launch_attn_bwd(const Dims& dm, int dtype, const void* q, const void* k, const void* v,
                            const void* out, const void* dout, const float* lse, const int32_t* sel,
                            const int32_t* offsets, const int32_t* rows, void* dq, void* dk, void* dv,
                            BwdWs ws, cudaStream_t stream, int* launches);

// checks of sel / offsets / rows (moba_check_index): the status word becomes
// MOBA_ERR_INTERNAL on a violation, and the index is then made inert
cudaError_t launch_index_check(const Dims& dm, int exact, int32_t* sel, int32_t* offsets,
                               const int32_t* rows, int64_t capacity, int* status, cudaStream_t stream,
                               int* launches);

// a kernel whose only wait can never complete: it must time out (status word)
cudaError_t launch_bounded_wait_selftest(int* status, cudaStream_t stream);

}  // namespace moba
