// C ABI of the MoBA causal-prefill forward: argument validation, sizes and the
// three entry points declared in include/moba.h.
#include <math.h>

#include "launch.h"

namespace {

thread_local int g_last_cuda_error = 0;
thread_local int g_last_launches = 0;

constexpr int64_t kI32Max = 2147483647;
constexpr int64_t kGridYZMax = 65535;            // largest y or z extent of a CUDA grid
constexpr int64_t kPartialBudget = 8ll << 30;   // bytes of partials per pass (automatic chunk)

int64_t round_up(int64_t x, int64_t m) { return (x + m - 1) / m * m; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

int64_t nblocks(const moba_shape_t* s) { return ((int64_t)s->seqlen + s->block - 1) / s->block; }

int64_t chunk_of(const moba_shape_t* s) {
  const int64_t cap = round_up(s->seqlen, 128);
  if (s->query_chunk > 0) return s->query_chunk < cap ? s->query_chunk : cap;
  const int64_t KH = s->topk - 1;
  if (KH == 0) return cap;
  // bytes of one partial result: bf16 output and fp32 log-sum-exp on the
  // tensor-core path (bf16, head_dim 128 or 64), fp32 output and lse otherwise
  const int64_t slot = moba::attn_tc_path(s->dtype, s->head_dim) ? 2 * s->head_dim + 4
                                                                 : 4 * (s->head_dim + 1);
  const int64_t per_token = (int64_t)s->batch * s->hq * KH * slot;
  int64_t c = 128;
  while (c * 2 <= cap && c * 2 * per_token <= kPartialBudget) c *= 2;
  return c < cap ? c : cap;
}

int64_t nchunks_of(const moba_shape_t* s) {
  const int64_t c = chunk_of(s);
  return (s->seqlen + c - 1) / c;
}

int64_t ngroups_total(const moba_shape_t* s) {
  return nchunks_of(s) * s->batch * s->hkv * nblocks(s);
}

int64_t rows_total(const moba_shape_t* s) {
  return moba::hist_rows_range(0, s->seqlen, s->block, s->topk - 1) * s->batch * s->hq;
}

moba::Dims make_dims(const moba_shape_t* s) {
  moba::Dims d;
  d.batch = s->batch;
  d.N = s->seqlen;
  d.hq = s->hq;
  d.hkv = s->hkv;
  d.d = s->head_dim;
  d.B = s->block;
  d.topk = s->topk;
  d.n = (int)nblocks(s);
  d.G = s->hq / s->hkv;
  d.chunk = (int)chunk_of(s);
  d.nchunks = (int)nchunks_of(s);
  d.t_lo = 0;
  d.t_hi = s->seqlen;
  const float scale = s->scale > 0.f ? s->scale : 1.0f / sqrtf((float)s->head_dim);
  d.scale_log2 = scale * moba::kLog2e;
  return d;
}

size_t align_up(size_t x) { return (x + 255) & ~size_t(255); }

struct AttnLayout {
  size_t status, part_o, part_lse, tile_start, total;
};
AttnLayout attn_layout(const moba_shape_t* s) {
  const size_t KH = s->topk - 1;
  const size_t entries = (size_t)s->batch * chunk_of(s) * s->hq * KH;
  // the tensor-core kernels (bf16, head_dim 128 or 64) keep the partial
  // outputs in bf16; the others in fp32
  const size_t part_bytes = moba::attn_tc_path(s->dtype, s->head_dim) ? 2 : 4;
  AttnLayout L;
  L.status = 0;
  L.part_o = 256;
  L.part_lse = L.part_o + align_up(entries * s->head_dim * part_bytes);
  L.tile_start = L.part_lse + align_up(entries * sizeof(float));
  L.total = L.tile_start + align_up(((size_t)s->batch * s->hkv * nblocks(s) + 1) * sizeof(int32_t));
  return L;
}

// device workspace of moba_prefill_host: the device copies of q, k, v, out
// (and lse), then the intermediate arrays and the two step workspaces
struct HostLayout {
  size_t q, k, v, out, lse, meank, sel, offsets, rows, gate_ws, attn_ws, total;
};
HostLayout host_layout(const moba_shape_t* s, bool with_lse) {
  const size_t es = s->dtype == MOBA_BF16 ? 2 : 4;
  const size_t qbytes = (size_t)s->batch * s->seqlen * s->hq * s->head_dim * es;
  const size_t kbytes = (size_t)s->batch * s->seqlen * s->hkv * s->head_dim * es;
  HostLayout L;
  size_t at = 0;
  auto take = [&](size_t bytes) { const size_t here = at; at += align_up(bytes > 0 ? bytes : 1); return here; };
  L.q = take(qbytes);
  L.k = take(kbytes);
  L.v = take(kbytes);
  L.out = take(qbytes);
  L.lse = take(with_lse ? (size_t)s->batch * s->hq * s->seqlen * sizeof(float) : 0);
  L.meank = take((size_t)s->batch * nblocks(s) * s->hkv * s->head_dim * sizeof(float));
  L.sel = take((size_t)s->batch * s->seqlen * s->hq * s->topk * sizeof(int32_t));
  L.offsets = take(((size_t)ngroups_total(s) + 1) * sizeof(int32_t));
  L.rows = take((size_t)rows_total(s) * sizeof(int32_t));
  L.gate_ws = take(align_up(2 * (size_t)ngroups_total(s) * sizeof(int32_t)) + 256);
  L.attn_ws = take(attn_layout(s).total);
  L.total = at;
  return L;
}

moba_status_t finish(cudaError_t e, int launches) {
  g_last_launches = launches;
  if (e != cudaSuccess) {
    g_last_cuda_error = (int)e;
    return MOBA_ERR_CUDA;
  }
  return MOBA_OK;
}

}  // namespace

extern "C" {

MOBA_API moba_status_t moba_check_shape(const moba_shape_t* s) {
  if (s == nullptr) return MOBA_ERR_INVALID_ARG;
  if (s->batch < 1 || s->seqlen < 1 || s->hq < 1 || s->hkv < 1 || s->block < 1 || s->topk < 1 ||
      s->head_dim < 1)
    return MOBA_ERR_INVALID_ARG;
  if (s->hq % s->hkv != 0) return MOBA_ERR_INVALID_ARG;
  if (s->dtype != MOBA_BF16 && s->dtype != MOBA_F32) return MOBA_ERR_INVALID_ARG;
  if (isnan(s->scale) || isinf(s->scale)) return MOBA_ERR_INVALID_ARG;
  if (s->query_chunk < 0 || (s->query_chunk > 0 && s->query_chunk % 128 != 0))
    return MOBA_ERR_INVALID_ARG;
  if (s->head_dim != 64 && s->head_dim != 128) return MOBA_ERR_UNSUPPORTED;
  if (s->topk > MOBA_MAX_TOPK) return MOBA_ERR_UNSUPPORTED;
  // the pooling kernels put blocks and batch entries on the grid's y and z axes
  if (nblocks(s) > kGridYZMax || s->batch > kGridYZMax) return MOBA_ERR_UNSUPPORTED;
  if ((int64_t)s->batch * s->seqlen * s->hq > kI32Max) return MOBA_ERR_UNSUPPORTED;
  if (rows_total(s) > kI32Max) return MOBA_ERR_UNSUPPORTED;
  if (ngroups_total(s) + 1 > kI32Max) return MOBA_ERR_UNSUPPORTED;
  if ((int64_t)s->batch * chunk_of(s) * s->hq * (s->topk - 1) > kI32Max) return MOBA_ERR_UNSUPPORTED;
  return MOBA_OK;
}

MOBA_API int64_t moba_num_blocks(const moba_shape_t* s) {
  return moba_check_shape(s) == MOBA_OK ? nblocks(s) : -1;
}
MOBA_API int64_t moba_query_chunk(const moba_shape_t* s) {
  return moba_check_shape(s) == MOBA_OK ? chunk_of(s) : -1;
}
MOBA_API int64_t moba_num_chunks(const moba_shape_t* s) {
  return moba_check_shape(s) == MOBA_OK ? nchunks_of(s) : -1;
}
MOBA_API int64_t moba_meank_elems(const moba_shape_t* s) {
  return moba_check_shape(s) == MOBA_OK ? (int64_t)s->batch * nblocks(s) * s->hkv * s->head_dim : -1;
}
MOBA_API int64_t moba_sel_elems(const moba_shape_t* s) {
  return moba_check_shape(s) == MOBA_OK ? (int64_t)s->batch * s->seqlen * s->hq * s->topk : -1;
}
MOBA_API int64_t moba_offsets_elems(const moba_shape_t* s) {
  return moba_check_shape(s) == MOBA_OK ? ngroups_total(s) + 1 : -1;
}
MOBA_API int64_t moba_rows_elems(const moba_shape_t* s) {
  return moba_check_shape(s) == MOBA_OK ? rows_total(s) : -1;
}
MOBA_API size_t moba_gate_workspace_size(const moba_shape_t* s) {
  if (moba_check_shape(s) != MOBA_OK) return 0;
  return align_up(2 * (size_t)ngroups_total(s) * sizeof(int32_t)) + 256;   // counters + status word
}
MOBA_API size_t moba_attn_workspace_size(const moba_shape_t* s) {
  if (moba_check_shape(s) != MOBA_OK) return 0;
  return attn_layout(s).total;
}
MOBA_API size_t moba_workspace_size(const moba_shape_t* s) {
  if (moba_check_shape(s) != MOBA_OK) return 0;
  return moba_gate_workspace_size(s) + moba_attn_workspace_size(s);
}
MOBA_API int64_t moba_rows_capacity(const moba_shape_t* s) {
  return moba_check_shape(s) == MOBA_OK ? rows_total(s) : -1;
}

MOBA_API moba_status_t moba_block_meanpool(const moba_shape_t* s, const void* k, float* meank,
                                           moba_stream_t stream) {
  g_last_launches = 0;
  moba_status_t st = moba_check_shape(s);
  if (st != MOBA_OK) return st;
  if (k == nullptr || meank == nullptr || !aligned16(k) || !aligned16(meank))
    return MOBA_ERR_INVALID_ARG;
  int launches = 0;
  cudaError_t e = moba::launch_meanpool(make_dims(s), s->dtype, k, meank, (cudaStream_t)stream,
                                        &launches);
  return finish(e, launches);
}

MOBA_API moba_status_t moba_gate_topk(const moba_shape_t* s, const void* q, const float* meank,
                                      int32_t* sel, int32_t* offsets, int32_t* rows, void* ws,
                                      size_t ws_bytes, moba_stream_t stream) {
  g_last_launches = 0;
  moba_status_t st = moba_check_shape(s);
  if (st != MOBA_OK) return st;
  if (q == nullptr || meank == nullptr || sel == nullptr || offsets == nullptr || ws == nullptr)
    return MOBA_ERR_INVALID_ARG;
  if (rows == nullptr && rows_total(s) > 0) return MOBA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(meank) || !aligned4(sel) || !aligned4(offsets) ||
      (rows != nullptr && !aligned4(rows)) || !aligned16(ws))
    return MOBA_ERR_INVALID_ARG;
  if (ws_bytes < moba_gate_workspace_size(s)) return MOBA_ERR_WORKSPACE;
  const int64_t L = ngroups_total(s);
  moba::GateWs g{static_cast<int32_t*>(ws), static_cast<int32_t*>(ws) + L,
                 reinterpret_cast<int*>(static_cast<char*>(ws) + align_up(2 * (size_t)L * sizeof(int32_t)))};
  int launches = 0;
  cudaError_t e = moba::launch_gate(make_dims(s), s->dtype, q, meank, sel, offsets, rows, g,
                                    (cudaStream_t)stream, &launches);
  return finish(e, launches);
}

MOBA_API moba_status_t moba_attn_fwd(const moba_shape_t* s, const void* q, const void* k,
                                     const void* v, const int32_t* sel, const int32_t* offsets,
                                     const int32_t* rows, void* out, float* lse, void* ws,
                                     size_t ws_bytes, moba_stream_t stream) {
  g_last_launches = 0;
  moba_status_t st = moba_check_shape(s);
  if (st != MOBA_OK) return st;
  if (q == nullptr || k == nullptr || v == nullptr || sel == nullptr || offsets == nullptr ||
      out == nullptr || ws == nullptr)
    return MOBA_ERR_INVALID_ARG;
  if (rows == nullptr && rows_total(s) > 0) return MOBA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned4(sel) ||
      !aligned4(offsets) || (rows != nullptr && !aligned4(rows)) || !aligned16(ws) ||
      (lse != nullptr && !aligned4(lse)))
    return MOBA_ERR_INVALID_ARG;
  if (ws_bytes < moba_attn_workspace_size(s)) return MOBA_ERR_WORKSPACE;
  AttnLayout L = attn_layout(s);
  char* base = static_cast<char*>(ws);
  moba::AttnWs a{reinterpret_cast<int*>(base + L.status), reinterpret_cast<float*>(base + L.part_o),
                 reinterpret_cast<float*>(base + L.part_lse),
                 reinterpret_cast<int32_t*>(base + L.tile_start)};
  int launches = 0;
  cudaError_t e = moba::launch_attn(make_dims(s), s->dtype, q, k, v, sel, offsets, rows, out, lse, a,
                                    (cudaStream_t)stream, &launches);
  return finish(e, launches);
}

MOBA_API moba_status_t moba_gate_topk_noalloc(const moba_shape_t* s, const void* q,
                                              const float* meank, int32_t* sel, int32_t* offsets,
                                              int32_t* rows, moba_stream_t stream) {
  g_last_launches = 0;
  moba_status_t st = moba_check_shape(s);
  if (st != MOBA_OK) return st;
  if (ngroups_total(s) > MOBA_GATE_NOALLOC_MAX_GROUPS) return MOBA_ERR_UNSUPPORTED;
  if (q == nullptr || meank == nullptr || sel == nullptr || offsets == nullptr)
    return MOBA_ERR_INVALID_ARG;
  if (rows == nullptr && rows_total(s) > 0) return MOBA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(meank) || !aligned4(sel) || !aligned4(offsets) ||
      (rows != nullptr && !aligned4(rows)))
    return MOBA_ERR_INVALID_ARG;
  int launches = 0;
  cudaError_t e = moba::launch_gate_noalloc(make_dims(s), s->dtype, q, meank, sel, offsets, rows,
                                            (cudaStream_t)stream, &launches);
  return finish(e, launches);
}

MOBA_API moba_status_t moba_gate_noalloc_status(int* status, moba_stream_t stream) {
  g_last_launches = 0;
  if (status == nullptr) return MOBA_ERR_INVALID_ARG;
  return finish(moba::gate_noalloc_status(status, (cudaStream_t)stream), 0);
}

struct BwdLayout {
  size_t status, delta, dqacc, tile_start, total;
};
BwdLayout bwd_layout(const moba_shape_t* s) {
  const size_t nrows = (size_t)s->batch * s->seqlen * s->hq;
  const bool tc = moba::attn_bwd_tc_path(make_dims(s), s->dtype);
  BwdLayout L;
  L.status = 0;
  L.delta = 256;
  L.dqacc = L.delta + align_up(nrows * sizeof(float));
  L.tile_start = L.dqacc + (tc ? align_up(nrows * s->head_dim * sizeof(float)) : 0);
  L.total = L.tile_start + (tc ? align_up(((size_t)s->batch * s->hkv * nblocks(s) + 1) * sizeof(int32_t)) : 0);
  return L;
}

MOBA_API size_t moba_attn_bwd_workspace_size(const moba_shape_t* s) {
  if (moba_check_shape(s) != MOBA_OK) return 0;
  return bwd_layout(s).total;
}

MOBA_API moba_status_t moba_attn_bwd(const moba_shape_t* s, const void* q, const void* k, const void* v,
                                     const void* out, const void* dout, const float* lse,
                                     const int32_t* sel, const int32_t* offsets, const int32_t* rows,
                                     void* dq, void* dk, void* dv, void* ws, size_t ws_bytes,
                                     moba_stream_t stream) {
  g_last_launches = 0;
  moba_status_t st = moba_check_shape(s);
  if (st != MOBA_OK) return st;
  if (q == nullptr || k == nullptr || v == nullptr || out == nullptr || dout == nullptr ||
      lse == nullptr || sel == nullptr || offsets == nullptr || dq == nullptr || dk == nullptr ||
      dv == nullptr || ws == nullptr)
    return MOBA_ERR_INVALID_ARG;
  if (rows == nullptr && rows_total(s) > 0) return MOBA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(dout) ||
      !aligned4(lse) || !aligned4(sel) || !aligned4(offsets) || (rows != nullptr && !aligned4(rows)) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || !aligned16(ws))
    return MOBA_ERR_INVALID_ARG;
  if (ws_bytes < moba_attn_bwd_workspace_size(s)) return MOBA_ERR_WORKSPACE;
  char* base = static_cast<char*>(ws);
  const BwdLayout L = bwd_layout(s);
  moba::BwdWs w{reinterpret_cast<int*>(base + L.status), reinterpret_cast<float*>(base + L.delta),
                reinterpret_cast<float*>(base + L.dqacc), reinterpret_cast<int32_t*>(base + L.tile_start)};
  int launches = 0;
  cudaError_t e = cudaMemsetAsync(w.status, 0, sizeof(int), (cudaStream_t)stream);
  if (e == cudaSuccess)
    e = moba::launch_attn_bwd(make_dims(s), s->dtype, q, k, v, out, dout, lse, sel, offsets, rows, dq, dk,
                              dv, w, (cudaStream_t)stream, &launches);
  return finish(e, launches);
}

MOBA_API size_t moba_prefill_host_workspace_size(const moba_shape_t* s, int with_lse) {
  if (moba_check_shape(s) != MOBA_OK) return 0;
  return host_layout(s, with_lse != 0).total;
}

MOBA_API moba_status_t moba_prefill_host(const moba_shape_t* s, const void* q, const void* k,
                                         const void* v, void* out, float* lse, int* status,
                                         void* ws, size_t ws_bytes, moba_stream_t stream_) {
  g_last_launches = 0;
  moba_status_t st = moba_check_shape(s);
  if (st != MOBA_OK) return st;
  if (q == nullptr || k == nullptr || v == nullptr || out == nullptr || ws == nullptr)
    return MOBA_ERR_INVALID_ARG;
  if (!aligned16(ws)) return MOBA_ERR_INVALID_ARG;
  const HostLayout L = host_layout(s, lse != nullptr);
  if (ws_bytes < L.total) return MOBA_ERR_WORKSPACE;
  const moba::Dims dm = make_dims(s);
  const cudaStream_t stream = (cudaStream_t)stream_;
  char* base = static_cast<char*>(ws);
  void* qd = base + L.q;
  void* kd = base + L.k;
  void* vd = base + L.v;
  void* od = base + L.out;
  float* lsed = lse != nullptr ? reinterpret_cast<float*>(base + L.lse) : nullptr;
  float* meank = reinterpret_cast<float*>(base + L.meank);
  int32_t* sel = reinterpret_cast<int32_t*>(base + L.sel);
  int32_t* offsets = reinterpret_cast<int32_t*>(base + L.offsets);
  int32_t* rows = reinterpret_cast<int32_t*>(base + L.rows);
  const int64_t G = ngroups_total(s);
  moba::GateWs g{reinterpret_cast<int32_t*>(base + L.gate_ws),
                 reinterpret_cast<int32_t*>(base + L.gate_ws) + G,
                 reinterpret_cast<int*>(base + L.gate_ws + align_up(2 * (size_t)G * sizeof(int32_t)))};
  const AttnLayout AL = attn_layout(s);
  char* ab = base + L.attn_ws;
  moba::AttnWs a{reinterpret_cast<int*>(ab + AL.status), reinterpret_cast<float*>(ab + AL.part_o),
                 reinterpret_cast<float*>(ab + AL.part_lse), reinterpret_cast<int32_t*>(ab + AL.tile_start)};

  const size_t es = s->dtype == MOBA_BF16 ? 2 : 4;
  const size_t qrow = (size_t)s->hq * s->head_dim * es;       // bytes of one token of q / out
  const size_t kbytes = (size_t)s->batch * s->seqlen * s->hkv * s->head_dim * es;
  const int np = dm.nchunks;

  // copy-in and copy-out streams beside the caller's compute stream; every
  // object made here is released at the end (destroying a stream or event
  // with work pending is legal: it goes once that work is done)
  cudaStream_t s_in = nullptr, s_out = nullptr;
  cudaEvent_t ev_start = nullptr, ev_done = nullptr;
  cudaEvent_t* ev_q = new cudaEvent_t[np]();
  cudaEvent_t* ev_o = new cudaEvent_t[np]();
  int launches = 0;
  cudaError_t e = cudaStreamCreateWithFlags(&s_in, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&s_out, cudaStreamNonBlocking);
  for (cudaEvent_t* ev : {&ev_start, &ev_done})
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming);
  for (int p = 0; p < np && e == cudaSuccess; ++p) {
    e = cudaEventCreateWithFlags(&ev_q[p], cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ev_o[p], cudaEventDisableTiming);
  }
  // k and v stream in with the passes, so a tile that reaches past the copied
  // rows (masked, but multiplied by zero probabilities) must read finite
  // values: clear the device copies first
  if (e == cudaSuccess) e = cudaMemsetAsync(kd, 0, kbytes, stream);
  if (e == cudaSuccess) e = cudaMemsetAsync(vd, 0, kbytes, stream);
  // the copies start after the work already queued on the caller's stream
  if (e == cudaSuccess) e = cudaEventRecord(ev_start, stream);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(s_in, ev_start, 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(s_out, ev_start, 0);
  // host -> device one query pass at a time: the pass's k, v and q rows.  Every
  // step of pass p reads only tokens before the pass's end: the pooled keys of
  // complete blocks, the gate's candidate blocks (all earlier) and the
  // attention's keys.
  const size_t krow = (size_t)s->hkv * s->head_dim * es;
  for (int p = 0; p < np && e == cudaSuccess; ++p) {
    const int t0 = p * dm.chunk, t1 = dm.N < t0 + dm.chunk ? dm.N : t0 + dm.chunk;
    const size_t kp = (size_t)dm.N * krow;
    e = cudaMemcpy2DAsync(static_cast<char*>(kd) + (size_t)t0 * krow, kp, static_cast<const char*>(k) + (size_t)t0 * krow,
                          kp, (size_t)(t1 - t0) * krow, dm.batch, cudaMemcpyHostToDevice, s_in);
    if (e == cudaSuccess)
      e = cudaMemcpy2DAsync(static_cast<char*>(vd) + (size_t)t0 * krow, kp,
                            static_cast<const char*>(v) + (size_t)t0 * krow, kp, (size_t)(t1 - t0) * krow,
                            dm.batch, cudaMemcpyHostToDevice, s_in);
    const size_t pitch = (size_t)dm.N * qrow;
    if (e == cudaSuccess)
      e = cudaMemcpy2DAsync(static_cast<char*>(qd) + (size_t)t0 * qrow, pitch,
                            static_cast<const char*>(q) + (size_t)t0 * qrow, pitch, (size_t)(t1 - t0) * qrow,
                            dm.batch, cudaMemcpyHostToDevice, s_in);
    if (e == cudaSuccess) e = cudaEventRecord(ev_q[p], s_in);
  }
  // compute on the caller's stream, pass by pass as each pass's rows arrive:
  // mean-pool of the blocks the pass completes, gate, attention
  if (e == cudaSuccess) e = cudaMemsetAsync(g.counts, 0, sizeof(int32_t) * G * 2, stream);
  if (e == cudaSuccess) e = cudaMemsetAsync(g.status, 0, sizeof(int), stream);
  if (e == cudaSuccess) e = cudaMemsetAsync(a.status, 0, sizeof(int), stream);
  int pooled = 0;
  for (int p = 0; p < np && e == cudaSuccess; ++p) {
    const int t0 = p * dm.chunk, t1 = dm.N < t0 + dm.chunk ? dm.N : t0 + dm.chunk;
    e = cudaStreamWaitEvent(stream, ev_q[p], 0);
    const int upto = t1 == dm.N ? dm.n : t1 / dm.B;   // blocks complete once the pass is in
    if (e == cudaSuccess)
      e = moba::launch_meanpool_blocks(dm, s->dtype, kd, meank, pooled, upto, stream, &launches);
    pooled = upto > pooled ? upto : pooled;
    if (e == cudaSuccess)
      e = moba::launch_gate_pass(dm, s->dtype, qd, meank, sel, offsets, rows, g, p, stream, &launches);
    if (e == cudaSuccess)
      e = moba::launch_attn_passes(dm, s->dtype, qd, kd, vd, sel, offsets, rows, od, lsed, a, p, p + 1,
                                   stream, &launches);
    if (e == cudaSuccess) e = cudaEventRecord(ev_o[p], stream);
    // device -> host: this pass's output while the next pass computes
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s_out, ev_o[p], 0);
    if (e == cudaSuccess) {
      const size_t pitch = (size_t)dm.N * qrow;
      e = cudaMemcpy2DAsync(static_cast<char*>(out) + (size_t)t0 * qrow, pitch,
                            static_cast<const char*>(od) + (size_t)t0 * qrow, pitch,
                            (size_t)(t1 - t0) * qrow, dm.batch, cudaMemcpyDeviceToHost, s_out);
    }
    if (e == cudaSuccess && lse != nullptr)
      e = cudaMemcpy2DAsync(lse + t0, (size_t)dm.N * sizeof(float), lsed + t0, (size_t)dm.N * sizeof(float),
                            (size_t)(t1 - t0) * sizeof(float), (size_t)dm.batch * dm.hq,
                            cudaMemcpyDeviceToHost, s_out);
  }
  if (e == cudaSuccess && status != nullptr) {
    e = cudaMemcpyAsync(status, g.status, sizeof(int), cudaMemcpyDeviceToHost, s_out);
    if (e == cudaSuccess) e = cudaMemcpyAsync(status + 1, a.status, sizeof(int), cudaMemcpyDeviceToHost, s_out);
  }
  // the caller's stream completes only after the last copy-out
  if (e == cudaSuccess) e = cudaEventRecord(ev_done, s_out);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(stream, ev_done, 0);
  if (e != cudaSuccess) {
    // the caller's stream may not cover copies already queued on the private
    // streams: let them finish before the caller can release its buffers
    if (s_in != nullptr) cudaStreamSynchronize(s_in);
    if (s_out != nullptr) cudaStreamSynchronize(s_out);
  }
  for (int p = 0; p < np; ++p) {
    if (ev_q[p] != nullptr) cudaEventDestroy(ev_q[p]);
    if (ev_o[p] != nullptr) cudaEventDestroy(ev_o[p]);
  }
  delete[] ev_q;
  delete[] ev_o;
  for (cudaEvent_t ev : {ev_start, ev_done})
    if (ev != nullptr) cudaEventDestroy(ev);
  if (s_in != nullptr) cudaStreamDestroy(s_in);
  if (s_out != nullptr) cudaStreamDestroy(s_out);
  return finish(e, launches);
}

// ---- gate variant with max- and min-pooled keys ------------------------------

MOBA_API moba_status_t moba_pooled_wide_shape(const moba_shape_t* s, int32_t extra, moba_shape_t* wide) {
  if (wide == nullptr) return MOBA_ERR_INVALID_ARG;
  moba_status_t st = moba_check_shape(s);
  if (st != MOBA_OK) return st;
  if (extra < 0) return MOBA_ERR_INVALID_ARG;
  if ((int64_t)s->topk + 2 * (int64_t)extra > MOBA_MAX_TOPK) return MOBA_ERR_UNSUPPORTED;
  moba_shape_t w = *s;
  w.topk = s->topk + 2 * extra;
  if ((st = moba_check_shape(&w)) != MOBA_OK) return st;
  *wide = w;
  return MOBA_OK;
}

MOBA_API moba_status_t moba_block_maxminpool(const moba_shape_t* s, const void* k, float* maxk,
                                             float* mink, moba_stream_t stream) {
  g_last_launches = 0;
  moba_status_t st = moba_check_shape(s);
  if (st != MOBA_OK) return st;
  if (k == nullptr || maxk == nullptr || mink == nullptr || !aligned16(k) || !aligned16(maxk) ||
      !aligned16(mink))
    return MOBA_ERR_INVALID_ARG;
  int launches = 0;
  cudaError_t e = moba::launch_maxminpool(make_dims(s), s->dtype, k, maxk, mink, (cudaStream_t)stream,
                                          &launches);
  return finish(e, launches);
}

MOBA_API moba_status_t moba_gate_pooled(const moba_shape_t* s, int32_t extra, const void* q,
                                        const float* meank, const float* maxk, const float* mink,
                                        int32_t* sel, int32_t* offsets, int32_t* rows, void* ws,
                                        size_t ws_bytes, moba_stream_t stream) {
  g_last_launches = 0;
  moba_shape_t w;
  moba_status_t st = moba_pooled_wide_shape(s, extra, &w);
  if (st != MOBA_OK) return st;
  if (q == nullptr || meank == nullptr || maxk == nullptr || mink == nullptr || sel == nullptr ||
      offsets == nullptr || ws == nullptr)
    return MOBA_ERR_INVALID_ARG;
  if (rows == nullptr && rows_total(&w) > 0) return MOBA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(meank) || !aligned16(maxk) || !aligned16(mink) || !aligned4(sel) ||
      !aligned4(offsets) || (rows != nullptr && !aligned4(rows)) || !aligned16(ws))
    return MOBA_ERR_INVALID_ARG;
  if (ws_bytes < moba_gate_workspace_size(&w)) return MOBA_ERR_WORKSPACE;
  const int64_t L = ngroups_total(&w);
  moba::GateWs g{static_cast<int32_t*>(ws), static_cast<int32_t*>(ws) + L,
                 reinterpret_cast<int*>(static_cast<char*>(ws) + align_up(2 * (size_t)L * sizeof(int32_t)))};
  int launches = 0;
  cudaError_t e = moba::launch_gate_pooled(make_dims(&w), s->dtype, s->topk - 1, extra, q, meank, maxk,
                                           mink, sel, offsets, rows, g, (cudaStream_t)stream, &launches);
  return finish(e, launches);
}

MOBA_API moba_status_t moba_attn_fwd_pooled(const moba_shape_t* s, int32_t extra, const void* q,
                                            const void* k, const void* v, const int32_t* sel,
                                            const int32_t* offsets, const int32_t* rows, void* out,
                                            float* lse, void* ws, size_t ws_bytes, moba_stream_t stream) {
  g_last_launches = 0;
  moba_shape_t w;
  moba_status_t st = moba_pooled_wide_shape(s, extra, &w);
  if (st != MOBA_OK) return st;
  if (q == nullptr || k == nullptr || v == nullptr || sel == nullptr || offsets == nullptr ||
      out == nullptr || ws == nullptr)
    return MOBA_ERR_INVALID_ARG;
  if (rows == nullptr && rows_total(&w) > 0) return MOBA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned4(sel) ||
      !aligned4(offsets) || (rows != nullptr && !aligned4(rows)) || !aligned16(ws) ||
      (lse != nullptr && !aligned4(lse)))
    return MOBA_ERR_INVALID_ARG;
  if (ws_bytes < moba_attn_workspace_size(&w)) return MOBA_ERR_WORKSPACE;
  AttnLayout L = attn_layout(&w);
  char* base = static_cast<char*>(ws);
  moba::AttnWs a{reinterpret_cast<int*>(base + L.status), reinterpret_cast<float*>(base + L.part_o),
                 reinterpret_cast<float*>(base + L.part_lse),
                 reinterpret_cast<int32_t*>(base + L.tile_start)};
  int launches = 0;
  cudaError_t e = moba::launch_attn_pooled(make_dims(&w), s->dtype, q, k, v, sel, offsets, rows, out,
                                           lse, a, (cudaStream_t)stream, &launches);
  return finish(e, launches);
}

MOBA_API moba_status_t moba_check_index(const moba_shape_t* s, int32_t exact, int32_t* sel,
                                        int32_t* offsets, const int32_t* rows, int* status,
                                        moba_stream_t stream) {
  g_last_launches = 0;
  moba_status_t st = moba_check_shape(s);
  if (st != MOBA_OK) return st;
  if (sel == nullptr || offsets == nullptr || status == nullptr) return MOBA_ERR_INVALID_ARG;
  if (rows == nullptr && rows_total(s) > 0) return MOBA_ERR_INVALID_ARG;
  if (!aligned4(sel) || !aligned4(offsets) || (rows != nullptr && !aligned4(rows)) || !aligned4(status))
    return MOBA_ERR_INVALID_ARG;
  int launches = 0;
  cudaError_t e = moba::launch_index_check(make_dims(s), exact != 0, sel, offsets, rows, rows_total(s),
                                           status, (cudaStream_t)stream, &launches);
  return finish(e, launches);
}

MOBA_API const char* moba_status_string(moba_status_t st) {
  switch (st) {
    case MOBA_OK: return "MOBA_OK";
    case MOBA_ERR_INVALID_ARG: return "MOBA_ERR_INVALID_ARG: invalid argument";
    case MOBA_ERR_UNSUPPORTED: return "MOBA_ERR_UNSUPPORTED: shape or dtype not supported";
    case MOBA_ERR_WORKSPACE: return "MOBA_ERR_WORKSPACE: workspace too small";
    case MOBA_ERR_CUDA: return "MOBA_ERR_CUDA: CUDA launch or runtime error";
    case MOBA_ERR_INTERNAL: return "MOBA_ERR_INTERNAL: internal error";
    case MOBA_ERR_TIMEOUT: return "MOBA_ERR_TIMEOUT: device wait timed out";
  }
  return "unknown moba_status_t";
}

MOBA_API moba_status_t moba_selftest_bounded_wait(int* status, moba_stream_t stream) {
  g_last_launches = 0;
  if (status == nullptr || !aligned4(status)) return MOBA_ERR_INVALID_ARG;
  return finish(moba::launch_bounded_wait_selftest(status, (cudaStream_t)stream), 1);
}

MOBA_API int moba_last_cuda_error(void) { return g_last_cuda_error; }
MOBA_API int moba_last_launch_count(void) { return g_last_launches; }

}  // extern "C"
