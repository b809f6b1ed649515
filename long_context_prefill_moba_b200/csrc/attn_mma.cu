// K3 (bf16, warp-level MMA): block-sparse flash attention of MoBA.
//
// "MoBA: Mixture of Block Attention for Long-Context LLMs", paper-graph
// summary §3 "The Core MoBA Attention Equation" (Softmax(q K[I]^T) V[I]),
// "Causality Enforcement" mechanism 2 (causal mask inside the current block)
// and the Implementation section, Algorithm 1 Step 3 (historical blocks without
// a mask, current block causal, queries grouped per block so one load of a
// block serves all its queries) and Step 4 (online-softmax merge).
//
// attn_hist_mma: one CTA per tile of <= 64 query rows that all routed to the
//   same (b, kv head g, earlier block j); it streams the B keys of that block
//   through shared memory (cp.async, double buffered) and writes one partial
//   result per row: o normalised (fp32) and its log2-sum-exp2.
// attn_cur_mma: one CTA per 64 consecutive tokens of one (b, h); causal
//   attention over the tokens' own block, then the merge with the row's
//   partials, writing out (and lse).
//
// Both use mma.sync m16n8k16 (bf16 -> fp32); each warp owns 16 query rows.
#include <float.h>

#include "launch.h"

namespace moba {

namespace {

constexpr int kTM = 64;      // query rows per CTA
constexpr int kTK = 64;      // keys per tile
constexpr int kWarps = 4;

// byte offset of element (row, col) in a [rows x D] bf16 tile whose 16-byte
// chunks are XOR-swizzled by (row % 8) to keep ldmatrix conflict-free
template <int D>
MOBA_DEV uint32_t swz(int row, int col) {
  return (uint32_t)(row * (D * 2) + ((((col >> 3) ^ (row & 7))) << 4) + ((col & 7) << 1));
}

// copy one [64 x D] tile of rows (given by global row pointers) into smem
template <int D>
MOBA_DEV void load_tile(uint32_t smem, const __nv_bfloat16* const* rowp, const bool* ok) {
  constexpr int CH = D / 8;  // 16-byte chunks per row
  for (int i = threadIdx.x; i < kTM * CH; i += kWarps * 32) {
    const int r = i / CH, cchunk = i % CH;
    cp_async16(smem + swz<D>(r, cchunk * 8), rowp[r] + cchunk * 8, ok[r]);
  }
}

template <int D>
struct Frag {
  static constexpr int kDT = D / 8;   // 8-wide column tiles of the output
  static constexpr int kKS = D / 16;  // 16-deep k-steps over the head dim
};

// S[8][4] = Q_warp (16 x D) * K_tile^T (D x 64)
template <int D>
MOBA_DEV void qk_tile(float (*S)[4], const uint32_t (*qa)[4], uint32_t ks, int lane) {
#pragma unroll
  for (int n = 0; n < 8; ++n) S[n][0] = S[n][1] = S[n][2] = S[n][3] = 0.f;
  const int mi = lane >> 3;
#pragma unroll
  for (int kk = 0; kk < Frag<D>::kKS; ++kk) {
#pragma unroll
    for (int np = 0; np < 4; ++np) {
      uint32_t b0, b1, b2, b3;
      ldmatrix_x4(ks + swz<D>(np * 16 + (mi >> 1) * 8 + (lane & 7), kk * 16 + (mi & 1) * 8), b0, b1,
                  b2, b3);
      mma_bf16_16816(S[2 * np], qa[kk], b0, b1);
      mma_bf16_16816(S[2 * np + 1], qa[kk], b2, b3);
    }
  }
}

// O[DT][4] += P (16 x 64, from S registers) * V_tile (64 x D)
template <int D>
MOBA_DEV void pv_tile(float (*O)[4], const float (*S)[4], uint32_t vs, int lane) {
  const int mi = lane >> 3;
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
    uint32_t pa[4];
    pa[0] = pack_bf16x2(S[2 * kk][0], S[2 * kk][1]);
    pa[1] = pack_bf16x2(S[2 * kk][2], S[2 * kk][3]);
    pa[2] = pack_bf16x2(S[2 * kk + 1][0], S[2 * kk + 1][1]);
    pa[3] = pack_bf16x2(S[2 * kk + 1][2], S[2 * kk + 1][3]);
#pragma unroll
    for (int dp = 0; dp < Frag<D>::kDT / 2; ++dp) {
      uint32_t b0, b1, b2, b3;
      ldmatrix_x4_trans(vs + swz<D>(kk * 16 + (mi & 1) * 8 + (lane & 7), dp * 16 + (mi >> 1) * 8),
                        b0, b1, b2, b3);
      mma_bf16_16816(O[2 * dp], pa, b0, b1);
      mma_bf16_16816(O[2 * dp + 1], pa, b2, b3);
    }
  }
}

// online-softmax step on S (already scaled to log2 units and masked with
// -inf): updates row maxima m[2], thread-partial sums l[2] and rescales O;
// leaves p = exp2(s - m) in S
template <int D>
MOBA_DEV void softmax_step(float (*S)[4], float (*O)[4], float* m, float* l) {
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    float mx = -INFINITY;
#pragma unroll
    for (int n = 0; n < 8; ++n) mx = fmaxf(mx, fmaxf(S[n][2 * hr], S[n][2 * hr + 1]));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const float m_new = fmaxf(m[hr], mx);
    const float base = m_new == -INFINITY ? 0.f : m_new;
    const float corr = exp2f(m[hr] - base);       // m[hr] = -inf -> 0
    m[hr] = m_new;
    float rs = 0.f;
#pragma unroll
    for (int n = 0; n < 8; ++n) {
      S[n][2 * hr] = exp2f(S[n][2 * hr] - base);
      S[n][2 * hr + 1] = exp2f(S[n][2 * hr + 1] - base);
      rs += S[n][2 * hr] + S[n][2 * hr + 1];
    }
    l[hr] = l[hr] * corr + rs;
#pragma unroll
    for (int dt = 0; dt < Frag<D>::kDT; ++dt) {
      O[dt][2 * hr] *= corr;
      O[dt][2 * hr + 1] *= corr;
    }
  }
}

template <int D>
MOBA_DEV void load_q_frags(uint32_t (*qa)[4], uint32_t qs, int warp, int lane) {
#pragma unroll
  for (int kk = 0; kk < Frag<D>::kKS; ++kk)
    ldmatrix_x4(qs + swz<D>(warp * 16 + (lane & 15), kk * 16 + (lane >> 4) * 8), qa[kk][0], qa[kk][1],
                qa[kk][2], qa[kk][3]);
}

// ---------------------------------------------------------------------------
// historical blocks
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(kWarps * 32) attn_hist_mma_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
    const __nv_bfloat16* __restrict__ v, const int32_t* __restrict__ sel,
    const int32_t* __restrict__ offsets, const int32_t* __restrict__ rows,
    const int32_t* __restrict__ tile_start, float* __restrict__ part_o,
    float* __restrict__ part_lse, Dims dm, int ch) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int TILE_BYTES = kTM * D * 2;
  const uint32_t qs = smem_u32(smem);
  const uint32_t ks0 = qs + TILE_BYTES;           // K stages at ks0, ks0 + 2*TILE
  const uint32_t vs0 = ks0 + TILE_BYTES;          // V stages interleaved
  __shared__ const __nv_bfloat16* rowp[kTM];
  __shared__ bool rowok[kTM];
  __shared__ int pidx[kTM];

  const int ngroups = dm.batch * dm.hkv * dm.n;
  const int tile = blockIdx.x;
  if (tile >= tile_start[ngroups]) return;
  // group containing this tile: last i with tile_start[i] <= tile
  int lo = 0, hi = ngroups - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (tile_start[mid] <= tile) lo = mid; else hi = mid - 1;
  }
  const int grp = lo;
  const int j = grp % dm.n;
  const int g = (grp / dm.n) % dm.hkv;
  const int b = grp / (dm.n * dm.hkv);
  const size_t goff = (size_t)ch * ngroups + grp;
  const int r0 = offsets[goff] + (tile - tile_start[grp]) * kTM;
  const int cnt = min(kTM, offsets[goff + 1] - r0);
  const int KH = dm.topk - 1;
  const int t0 = ch * dm.chunk;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid < kTM) {
    const bool ok = tid < cnt;
    const int r = ok ? rows[r0 + tid] : 0;
    rowp[tid] = q + (size_t)r * D;
    rowok[tid] = ok;
    if (ok) {
      const int h = r % dm.hq;
      const int t = (r / dm.hq) % dm.N;
      const int slot = slot_of(sel + (size_t)r * dm.topk, dm.topk, j);
      pidx[tid] = ((b * dm.chunk + (t - t0)) * dm.hq + h) * KH + slot;
    }
  }
  __syncthreads();
  load_tile<D>(qs, rowp, rowok);
  cp_async_commit();

  // key rows of block j, kv head g
  const __nv_bfloat16* kbase = k + ((size_t)b * dm.N * dm.hkv + g) * D;
  const __nv_bfloat16* vbase = v + ((size_t)b * dm.N * dm.hkv + g) * D;
  const size_t kstride = (size_t)dm.hkv * D;
  const int key0 = j * dm.B;
  const int nkt = (dm.B + kTK - 1) / kTK;

  auto issue_kv = [&](int kt, int stage) {
    constexpr int CH = D / 8;
    const uint32_t kd = ks0 + stage * 2 * TILE_BYTES, vd = vs0 + stage * 2 * TILE_BYTES;
    for (int i = tid; i < kTK * CH; i += kWarps * 32) {
      const int rr = i / CH, cc = i % CH;
      const int kr = kt * kTK + rr;
      const bool ok = kr < dm.B;
      const size_t off = (size_t)(key0 + (ok ? kr : 0)) * kstride + cc * 8;
      cp_async16(kd + swz<D>(rr, cc * 8), kbase + off, ok);
      cp_async16(vd + swz<D>(rr, cc * 8), vbase + off, ok);
    }
  };
  issue_kv(0, 0);
  cp_async_commit();
  if (nkt > 1) issue_kv(1, 1);
  cp_async_commit();

  uint32_t qa[Frag<D>::kKS][4];
  float O[Frag<D>::kDT][4];
#pragma unroll
  for (int dt = 0; dt < Frag<D>::kDT; ++dt) O[dt][0] = O[dt][1] = O[dt][2] = O[dt][3] = 0.f;
  float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
  const float sl2 = dm.scale_log2;

  for (int kt = 0; kt < nkt; ++kt) {
    cp_async_wait<1>();
    __syncthreads();
    if (kt == 0) load_q_frags<D>(qa, qs, warp, lane);
    const int stage = kt & 1;
    float S[8][4];
    qk_tile<D>(S, qa, ks0 + stage * 2 * TILE_BYTES, lane);
    const int kvalid = dm.B - kt * kTK;          // keys of this tile inside the block
#pragma unroll
    for (int n = 0; n < 8; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int col = n * 8 + 2 * (lane & 3) + (e & 1);
        S[n][e] = col < kvalid ? S[n][e] * sl2 : -INFINITY;
      }
    softmax_step<D>(S, O, m, l);
    pv_tile<D>(O, S, vs0 + stage * 2 * TILE_BYTES, lane);
    __syncthreads();
    if (kt + 2 < nkt) issue_kv(kt + 2, stage);
    cp_async_commit();
  }

  // epilogue: normalise and store the partials
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    float lt = l[hr];
    lt += __shfl_xor_sync(0xffffffffu, lt, 1);
    lt += __shfl_xor_sync(0xffffffffu, lt, 2);
    const int row = warp * 16 + (lane >> 2) + hr * 8;
    if (row < cnt) {
      const float inv = 1.f / lt;
      const size_t p = pidx[row];
      float* dst = part_o + p * D;
#pragma unroll
      for (int dt = 0; dt < Frag<D>::kDT; ++dt) {
        const int col = dt * 8 + 2 * (lane & 3);
        *reinterpret_cast<float2*>(dst + col) = make_float2(O[dt][2 * hr] * inv, O[dt][2 * hr + 1] * inv);
      }
      if ((lane & 3) == 0) part_lse[p] = m[hr] + log2f(lt);
    }
  }
}

// ---------------------------------------------------------------------------
// current block (causal) + merge
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(kWarps * 32) attn_cur_mma_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
    const __nv_bfloat16* __restrict__ v, const float* __restrict__ part_o,
    const float* __restrict__ part_lse, __nv_bfloat16* __restrict__ out, float* __restrict__ lse,
    Dims dm, int ch) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int TILE_BYTES = kTM * D * 2;
  const uint32_t qs = smem_u32(smem);
  const uint32_t ks0 = qs + TILE_BYTES;
  const uint32_t vs0 = ks0 + TILE_BYTES;
  __shared__ const __nv_bfloat16* rowp[kTM];
  __shared__ bool rowok[kTM];

  const int t0 = ch * dm.chunk;
  const int t_end = min(dm.N, t0 + dm.chunk);
  const int tiles = (t_end - t0 + kTM - 1) / kTM;
  const int tile = blockIdx.x % tiles;
  const int bh = blockIdx.x / tiles;
  const int h = bh % dm.hq;
  const int b = bh / dm.hq;
  const int g = h / dm.G;
  const int t_first = t0 + tile * kTM;
  const int t_last = min(t_end, t_first + kTM) - 1;
  const int KH = dm.topk - 1;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid < kTM) {
    const int t = t_first + tid;
    rowok[tid] = t <= t_last;
    rowp[tid] = q + ((size_t)(b * dm.N + min(t, t_last)) * dm.hq + h) * D;
  }
  __syncthreads();
  load_tile<D>(qs, rowp, rowok);
  cp_async_commit();

  const __nv_bfloat16* kbase = k + ((size_t)b * dm.N * dm.hkv + g) * D;
  const __nv_bfloat16* vbase = v + ((size_t)b * dm.N * dm.hkv + g) * D;
  const size_t kstride = (size_t)dm.hkv * D;
  const int key0 = (t_first / dm.B) * dm.B;       // first key any row of the tile may see
  const int nkt = (t_last - key0) / kTK + 1;

  auto issue_kv = [&](int kt, int stage) {
    constexpr int CH = D / 8;
    const uint32_t kd = ks0 + stage * 2 * TILE_BYTES, vd = vs0 + stage * 2 * TILE_BYTES;
    for (int i = tid; i < kTK * CH; i += kWarps * 32) {
      const int rr = i / CH, cc = i % CH;
      const int u = key0 + kt * kTK + rr;
      const bool ok = u <= t_last;
      const size_t off = (size_t)(ok ? u : key0) * kstride + cc * 8;
      cp_async16(kd + swz<D>(rr, cc * 8), kbase + off, ok);
      cp_async16(vd + swz<D>(rr, cc * 8), vbase + off, ok);
    }
  };
  issue_kv(0, 0);
  cp_async_commit();
  if (nkt > 1) issue_kv(1, 1);
  cp_async_commit();

  uint32_t qa[Frag<D>::kKS][4];
  float O[Frag<D>::kDT][4];
#pragma unroll
  for (int dt = 0; dt < Frag<D>::kDT; ++dt) O[dt][0] = O[dt][1] = O[dt][2] = O[dt][3] = 0.f;
  float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
  const float sl2 = dm.scale_log2;
  int trow[2], tlo[2];
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    trow[hr] = t_first + warp * 16 + (lane >> 2) + hr * 8;
    tlo[hr] = (trow[hr] / dm.B) * dm.B;
  }

  for (int kt = 0; kt < nkt; ++kt) {
    cp_async_wait<1>();
    __syncthreads();
    if (kt == 0) load_q_frags<D>(qa, qs, warp, lane);
    const int stage = kt & 1;
    float S[8][4];
    qk_tile<D>(S, qa, ks0 + stage * 2 * TILE_BYTES, lane);
#pragma unroll
    for (int n = 0; n < 8; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int u = key0 + kt * kTK + n * 8 + 2 * (lane & 3) + (e & 1);
        const int hr = e >> 1;
        S[n][e] = (u <= trow[hr] && u >= tlo[hr]) ? S[n][e] * sl2 : -INFINITY;
      }
    softmax_step<D>(S, O, m, l);
    pv_tile<D>(O, S, vs0 + stage * 2 * TILE_BYTES, lane);
    __syncthreads();
    if (kt + 2 < nkt) issue_kv(kt + 2, stage);
    cp_async_commit();
  }

  // epilogue: merge with the historical partials of each row
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    float lt = l[hr];
    lt += __shfl_xor_sync(0xffffffffu, lt, 1);
    lt += __shfl_xor_sync(0xffffffffu, lt, 2);
    const int t = trow[hr];
    if (t > t_last) continue;
    const float lse_cur = m[hr] + log2f(lt);
    const int nh = min(KH, t / dm.B);
    const size_t pbase = (size_t)((b * dm.chunk + (t - t0)) * dm.hq + h) * KH;
    float M = lse_cur;
    for (int s = 0; s < nh; ++s) M = fmaxf(M, part_lse[pbase + s]);
    const float wc = exp2f(lse_cur - M);
    float W = wc;
    float acc[Frag<D>::kDT][2];
    const float ic = wc / lt;
#pragma unroll
    for (int dt = 0; dt < Frag<D>::kDT; ++dt) {
      acc[dt][0] = O[dt][2 * hr] * ic;
      acc[dt][1] = O[dt][2 * hr + 1] * ic;
    }
    for (int s = 0; s < nh; ++s) {
      const float w = exp2f(part_lse[pbase + s] - M);
      W += w;
      const float* src = part_o + (pbase + s) * D;
#pragma unroll
      for (int dt = 0; dt < Frag<D>::kDT; ++dt) {
        const float2 o2 = *reinterpret_cast<const float2*>(src + dt * 8 + 2 * (lane & 3));
        acc[dt][0] = fmaf(w, o2.x, acc[dt][0]);
        acc[dt][1] = fmaf(w, o2.y, acc[dt][1]);
      }
    }
    const float iw = 1.f / W;
    __nv_bfloat16* dst = out + ((size_t)(b * dm.N + t) * dm.hq + h) * D;
#pragma unroll
    for (int dt = 0; dt < Frag<D>::kDT; ++dt) {
      const uint32_t pk = pack_bf16x2(acc[dt][0] * iw, acc[dt][1] * iw);
      *reinterpret_cast<uint32_t*>(dst + dt * 8 + 2 * (lane & 3)) = pk;
    }
    if (lse != nullptr && (lane & 3) == 0)
      lse[((size_t)b * dm.hq + h) * dm.N + t] = (M + log2f(W)) * kLn2;
  }
}

template <int D>
constexpr int smem_bytes() { return 5 * kTM * D * 2; }   // Q + 2 x (K, V)

}  // namespace

// tile prefix of one pass: tile_start[i] = sum_{i' < i} ceil(count_i' / 64)
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

cudaError_t launch_attn_mma_hist(const Dims& dm, const void* q, const void* k, const void* v,
                                 const int32_t* sel, const int32_t* offsets, const int32_t* rows,
                                 const AttnWs& ws, int ch, int64_t grid, cudaStream_t stream) {
  if (dm.d == 128) {
    auto kern = attn_hist_mma_kernel<128>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes<128>());
    kern<<<grid, kWarps * 32, smem_bytes<128>(), stream>>>(
        (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v, sel, offsets,
        rows, ws.tile_start, ws.part_o, ws.part_lse, dm, ch);
  } else {
    auto kern = attn_hist_mma_kernel<64>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes<64>());
    kern<<<grid, kWarps * 32, smem_bytes<64>(), stream>>>(
        (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v, sel, offsets,
        rows, ws.tile_start, ws.part_o, ws.part_lse, dm, ch);
  }
  return cudaGetLastError();
}

cudaError_t launch_attn_mma_cur(const Dims& dm, const void* q, const void* k, const void* v,
                                const AttnWs& ws, void* out, float* lse, int ch,
                                cudaStream_t stream) {
  const int t0 = ch * dm.chunk;
  const int t_end = dm.N < t0 + dm.chunk ? dm.N : t0 + dm.chunk;
  const int tiles = (t_end - t0 + kTM - 1) / kTM;
  const int64_t grid = (int64_t)tiles * dm.batch * dm.hq;
  if (dm.d == 128) {
    auto kern = attn_cur_mma_kernel<128>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes<128>());
    kern<<<grid, kWarps * 32, smem_bytes<128>(), stream>>>(
        (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v, ws.part_o,
        ws.part_lse, (__nv_bfloat16*)out, lse, dm, ch);
  } else {
    auto kern = attn_cur_mma_kernel<64>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes<64>());
    kern<<<grid, kWarps * 32, smem_bytes<64>(), stream>>>(
        (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v, ws.part_o,
        ws.part_lse, (__nv_bfloat16*)out, lse, dm, ch);
  }
  return cudaGetLastError();
}

}  // namespace moba
