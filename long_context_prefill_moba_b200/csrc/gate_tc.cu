// K2 scores on tensor cores: S = Q meanK^T as a tcgen05 GEMM, then the causal
// top-k per query row straight out of TMEM.
//
// "MoBA: Mixture of Block Attention for Long-Context LLMs", paper-graph
// summary §3 "Affinity Scoring" (s_i = <q, mean_pool(K[I_i])>, no softmax
// scale), "Top-k Gating" (top-k blocks plus the always-routed current block),
// "Causality Enforcement" mechanism 1 (no block that is not entirely in the
// past), Implementation, Algorithm 1 Step 1 (S = Q meanK^T with the causal mask
// and top-k).  S never leaves the chip: each row ranks its candidates in
// registers and only the k block ids are written.
//
// Precision.  q is bf16 (exact).  The fp32 pooled keys are split into three
// bf16 terms, meanK = hi + mid + lo with hi = bf16(meanK), mid = bf16(meanK -
// hi), lo = bf16(meanK - hi - mid); 3 x 8 significant bits cover the 24 of an
// fp32 value, so the split is exact and the three products (lo, then mid,
// then hi) accumulate into one fp32 TMEM accumulator: the only error of a
// score is the fp32 accumulation itself.  The ranking compares the full fp32
// scores; ties go to the lower block index.
//
// Ranking.  Each selection thread owns one query row (one TMEM lane).  A pass
// over the row's candidates keeps the top KB scores (KB = topk - 1 rounded up
// to 4, 8 or 16) with sorting networks: each batch of KB scores is sorted
// (Batcher's odd-even merge sort) and merged into the running list (the top KB
// of two sorted lists are the elementwise maxima of one list and the other
// reversed, a bitonic sequence, which a bitonic merger sorts).  The (k-1)-th
// largest score T is the threshold; a second pass over the candidates sets the
// bit of every block with score >= T in a 256-bit mask, and rows with ties at T
// beyond the quota take the tied blocks in increasing index.  The selected
// blocks come out of the mask in increasing order, as the sel rows store them.
//
// One CTA = one (b, kv head g) and a range of at most kTokens tokens inside one
// query pass, for all G query heads of the group: the group's pooled keys are
// converted and staged in shared memory once, then 128-row Q tiles stream
// through by TMA.  A tile holds 128 / GT consecutive tokens of GT query heads
// (GT = G when G divides 128, else 1), rows interleaved token-major, so a warp's
// rows write neighbouring sel rows.  Roles:
//   warps 0-3  selection, even tiles (S buffer 0: TMEM columns 0..255)
//   warps 4-7  selection, odd tiles  (S buffer 1: TMEM columns 256..511)
//   warp 8     TMA producer of Q tiles (and TMEM allocation)
//   warp 9     single-thread tcgen05.mma issuer
// The MMA of one tile overlaps the selection of the other warpgroup's tile.
// Requires bf16, head_dim 128 and at most 256 blocks.
//
// The gate variant with max- and min-pooled keys (the OpenReview discussion,
// the authors' answer to W1 on block representations; reading G1: the union of
// the top (k-1) blocks by the mean-pooled keys and the top `extra` by each of
// the max- and min-pooled keys) runs the same kernel three times, once per
// ranking, with the row's candidate mask carried between the passes in the
// row's own sel entries (a W-wide row holds the ceil(c / 32) mask words): the
// mean pass stores its mask, the max pass ORs into it, and the min pass ORs its
// own, takes the union out of the mask in increasing order and counts it.  The
// max and min pools are bf16 values (maxima of bf16 keys), so one bf16 term
// represents them exactly.
#include <cudaTypedefs.h>
#include <float.h>

#include <utility>

#include "launch.h"
#include "sm100.cuh"

namespace moba {

namespace {

using namespace sm100;

constexpr int kD = 128;
constexpr int kRowsT = 128;              // rows per Q tile (TMEM lanes)
constexpr int kTokens = 1024;            // tokens per CTA (per head), at most
constexpr int kMaxBlocks = 256;          // one MMA of N <= 256
constexpr int kSelThreads = 256;         // two selection warpgroups
constexpr int kThreads = kSelThreads + 64;
constexpr int kTerms = 3;                // meanK = hi + mid + lo
constexpr uint32_t kQTile = kRowsT * kD * 2;       // 32 KB
constexpr uint32_t kHalfQ = kRowsT * 128;          // 16 KB (64 columns)
constexpr uint32_t kOffQ = 0;                      // one stage
constexpr uint32_t kOffKB = kQTile;                // terms hi, mid, lo; each 2 halves of kMaxBlocks x 128 B
constexpr uint32_t kKBHalf = kMaxBlocks * 128;     // 32 KB
constexpr uint32_t kKB = 2 * kKBHalf;              // 64 KB per term
constexpr uint32_t kSmemBytes = kOffKB + kTerms * kKB + 1024;

struct Ctl {
  uint64_t q_full, q_free, s_full[2], s_free[2], drain;
  uint32_t tmem_base;
  int abort;
  int hist[kMaxBlocks];
};

// what one launch ranks and writes (see the file comment)
struct GatePass {
  const float* pool;   // pooled keys [b, n, hkv, d] fp32
  int nterms;          // bf16 terms that represent them exactly: 3 (mean) or 1 (max, min)
  int slots;           // blocks this ranking selects per row: topk - 1, or extra
  int mode;            // kOutSel, kMaskStore, kMaskOr, kMaskUnion
};
constexpr int kOutSel = 0, kMaskStore = 1, kMaskOr = 2, kMaskUnion = 3;

MOBA_DEV uint32_t bar(const uint64_t* b) { return smem_u32(b); }
// AND of `v` over the 128 threads of selection warpgroup `wg` (named barrier 1 + wg)
MOBA_DEV bool selectors_all(bool v, int wg) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.and.pred q, %2, 128, p;\n"
      " selp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(1 + wg)
      : "memory");
  return r != 0;
}

// ---- sorting networks on registers (descending) --------------------------------
// compiled for the host as well, so that a host program can check them
#define MOBA_NET __host__ __device__ __forceinline__
MOBA_NET void cex(float& a, float& b) {
  const float hi = fmaxf(a, b);
  b = fminf(a, b);
  a = hi;
}
// Batcher's odd-even merge sort of v[0..K), K a power of two <= 16: the
// compare-exchange pairs are generated at compile time and applied by a fold
// expression, so every register index is a constant
struct CePairs {
  int n;
  unsigned char a[64], b[64];
};
constexpr CePairs oem_pairs(int K) {
  CePairs P{0, {}, {}};
  for (int p = 1; p < K; p <<= 1)
    for (int k = p; k >= 1; k >>= 1)
      for (int j = k % p; j + k < K; j += 2 * k)
        for (int i = 0; i < k; ++i)
          if (i + j + k < K && (i + j) / (2 * p) == (i + j + k) / (2 * p)) {
            P.a[P.n] = (unsigned char)(i + j);
            P.b[P.n] = (unsigned char)(i + j + k);
            ++P.n;
          }
  return P;
}
// the bitonic merger of K entries: stages of distance K/2, K/4, .., 1
constexpr CePairs bitonic_pairs(int K) {
  CePairs P{0, {}, {}};
  for (int j = K / 2; j >= 1; j >>= 1)
    for (int i = 0; i < K; ++i)
      if ((i & j) == 0) {
        P.a[P.n] = (unsigned char)i;
        P.b[P.n] = (unsigned char)(i + j);
        ++P.n;
      }
  return P;
}
static_assert(oem_pairs(16).n == 63 && oem_pairs(8).n == 19 && oem_pairs(4).n == 5, "network sizes");
static_assert(bitonic_pairs(16).n == 32, "merger size");

template <int K, bool Bitonic, size_t... I>
MOBA_NET void apply_pairs(float (&v)[K], std::index_sequence<I...>) {
  constexpr CePairs P = Bitonic ? bitonic_pairs(K) : oem_pairs(K);
  (cex(v[P.a[I]], v[P.b[I]]), ...);
}
template <int K>
MOBA_NET void sort_desc(float (&v)[K]) {
  apply_pairs<K, false>(v, std::make_index_sequence<oem_pairs(K).n>{});
}
// a <- the top K of a and b (both sorted descending), sorted descending
template <int K>
MOBA_NET void merge_top(float (&a)[K], const float (&b)[K]) {
#pragma unroll
  for (int i = 0; i < K; ++i) a[i] = fmaxf(a[i], b[K - 1 - i]);
  apply_pairs<K, true>(a, std::make_index_sequence<bitonic_pairs(K).n>{});
}

// bits [0, n) set, n clamped to [0, 32]
MOBA_DEV uint32_t low_bits(int n) { return n <= 0 ? 0u : n >= 32 ? ~0u : ((1u << n) - 1u); }

template <int KB>
__global__ void __launch_bounds__(kThreads, 1) gate_select_tc_kernel(
    const __grid_constant__ CUtensorMap tmQ, const GatePass gp, int32_t* __restrict__ sel,
    int32_t* __restrict__ counts, int* __restrict__ status, Dims dm) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ Ctl ctl;
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  // CTA -> (b, g, pass, range): ranges never straddle a query pass
  const int L = min(kTokens, dm.chunk);
  const int rpp = (dm.chunk + L - 1) / L;
  const int p0 = dm.t_lo / dm.chunk;
  const int np = (dm.t_hi - 1) / dm.chunk - p0 + 1;
  const int rg = blockIdx.x % rpp;
  const int pp = p0 + (blockIdx.x / rpp) % np;
  const int g = (blockIdx.x / (rpp * np)) % dm.hkv;
  const int b = blockIdx.x / (rpp * np * dm.hkv);
  const int t_begin = max(dm.t_lo, pp * dm.chunk + rg * L);
  const int t_stop = min(min(dm.t_hi, (pp + 1) * dm.chunk), pp * dm.chunk + (rg + 1) * L);
  if (t_begin >= t_stop) return;   // uniform over the CTA, before any barrier or TMEM use
  const int GT = (kRowsT % dm.G == 0) ? dm.G : 1;   // query heads per tile
  const int TT = kRowsT / GT;                       // tokens per tile
  const int nsub = dm.G / GT;
  const int ttiles = (t_stop - t_begin + TT - 1) / TT;
  const int ntiles = ttiles * nsub;                 // tile k: token tile k / nsub, heads (k % nsub) * GT..
  const int cmax_cta = (t_stop - 1) / dm.B;         // blocks [0, cmax_cta) may be candidates
  const int npad = max(16, (cmax_cta + 15) / 16 * 16);
  const int KH = gp.slots;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    mbar_init(bar(&ctl.q_full), 1);
    mbar_init(bar(&ctl.q_free), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(&ctl.s_full[s]), 1);
      mbar_init(bar(&ctl.s_free[s]), kRowsT);
    }
    mbar_init(bar(&ctl.drain), 1);
    ctl.abort = 0;
    fence_mbar_init();
  }
  for (int i = tid; i < kMaxBlocks; i += kThreads) ctl.hist[i] = 0;
  if (warp == 8) {
    tmem_alloc(smem_u32(&ctl.tmem_base), 512);
    tmem_relinquish();
  }
  // pooled keys of (b, g) for blocks < npad as three bf16 terms, K-major,
  // 128-byte swizzle
  const uint32_t khi = base + kOffKB, kmid = khi + kKB, klo = kmid + kKB;
  for (int i = tid; i < npad * 16; i += kThreads) {
    const int jr = i >> 4, c = i & 15;              // block row, 8-element chunk
    float x[8];
    if (jr < cmax_cta) {
      const float4* src = reinterpret_cast<const float4*>(
          gp.pool + (((size_t)b * dm.n + jr) * dm.hkv + g) * kD + c * 8);
      const float4 a = __ldg(src), e = __ldg(src + 1);
      x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = e.x; x[5] = e.y; x[6] = e.z; x[7] = e.w;
    } else {
#pragma unroll
      for (int u = 0; u < 8; ++u) x[u] = 0.f;
    }
    uint32_t hi[4], mid[4], lo[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float2 v = make_float2(x[2 * u], x[2 * u + 1]);
      const __nv_bfloat162 h2 = __floats2bfloat162_rn(v.x, v.y);
      const float2 hf = __bfloat1622float2(h2);
      const float2 r1 = make_float2(v.x - hf.x, v.y - hf.y);       // exact
      const __nv_bfloat162 m2 = __floats2bfloat162_rn(r1.x, r1.y);
      const float2 mf = __bfloat1622float2(m2);
      hi[u] = *reinterpret_cast<const uint32_t*>(&h2);
      mid[u] = *reinterpret_cast<const uint32_t*>(&m2);
      lo[u] = pack_bf16x2(r1.x - mf.x, r1.y - mf.y);               // exact residual, exact in bf16
    }
    const uint32_t off = (c >> 3) * kKBHalf + sw128_off(jr, c & 7);
    asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};\n" ::"r"(khi + off), "r"(hi[0]), "r"(hi[1]),
                 "r"(hi[2]), "r"(hi[3]) : "memory");
    if (gp.nterms > 1) {
      asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};\n" ::"r"(kmid + off), "r"(mid[0]), "r"(mid[1]),
                   "r"(mid[2]), "r"(mid[3]) : "memory");
      asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};\n" ::"r"(klo + off), "r"(lo[0]), "r"(lo[1]),
                   "r"(lo[2]), "r"(lo[3]) : "memory");
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = ctl.tmem_base;
  volatile int* abort_flag = &ctl.abort;

  if (warp < 8) {
    // ------------------------------------------------------------ selection
    const int wg = warp >> 2;
    const int rho = tid & 127;                       // row of the tile = TMEM lane
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tb + (uint32_t)wg * 256u + lane_off;
    const int tl = rho / GT, hl = rho % GT;
    bool ok = true;
    for (int k = wg; k < ntiles && ok; k += 2) {
      const int i_wg = k >> 1;                       // this warpgroup's tile count so far
      const int tt = t_begin + (k / nsub) * TT;
      const int h = g * dm.G + (k % nsub) * GT + hl;
      const int t = tt + tl;
      const bool valid = t < t_stop;
      const int c = valid ? t / dm.B : 0;
      const int m = min(KH, c);                      // historical blocks this row selects
      const int ctile = (min(t_stop, tt + TT) - 1) / dm.B;   // candidates of the tile: [0, ctile)
      const int jlim = KH > 0 ? ctile : 0;
      // the decision is uniform over the warpgroup, so the named barrier is
      // always reached by all four warps
      ok = selectors_all(mbar_wait(bar(&ctl.s_full[wg]), i_wg & 1, abort_flag), wg);
      if (!ok) break;
      tc_fence_after();
      // rows with at most topk - 1 candidates take all of them; the others are
      // ranked below
      uint32_t mw[kMaxBlocks / 32];
#pragma unroll
      for (int w = 0; w < kMaxBlocks / 32; ++w) mw[w] = c <= KH ? low_bits(c - 32 * w) : 0u;
      // rows with more candidates than slots rank them (warp-uniform branch)
      if (__any_sync(0xffffffffu, c > KH)) {
        const int cmin = __reduce_min_sync(0xffffffffu, (unsigned)c);
        float a[KB];
#pragma unroll
        for (int i = 0; i < KB; ++i) a[i] = -INFINITY;
        for (int j0 = 0; j0 < jlim; j0 += 32) {
          uint32_t sr[32];
          tmem_ld32(tS + j0, sr);
          tmem_wait_ld();
          float v[32];
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) v[jj] = __uint_as_float(sr[jj]) + 0.0f;   // -0 -> +0
          if (j0 + 32 > cmin) {
#pragma unroll
            for (int jj = 0; jj < 32; ++jj) v[jj] = j0 + jj < c ? v[jj] : -INFINITY;
          }
#pragma unroll
          for (int bi = 0; bi < 32 / KB; ++bi) {
            float bt[KB];
#pragma unroll
            for (int i = 0; i < KB; ++i) bt[i] = v[bi * KB + i];
            sort_desc<KB>(bt);
            merge_top<KB>(a, bt);
          }
        }
        // threshold: the m-th largest score (rows with m == 0 select nothing)
        float T = a[0];
#pragma unroll
        for (int i = 1; i < KB; ++i) T = i < m ? a[i] : T;
        int cnt = 0;
        const bool ranked = c > KH;
#pragma unroll
        for (int w = 0; w < kMaxBlocks / 32; ++w) {
          if (w * 32 < jlim) {
            uint32_t sr[32];
            tmem_ld32(tS + w * 32, sr);
            tmem_wait_ld();
            uint32_t bits = 0;
#pragma unroll
            for (int jj = 0; jj < 32; ++jj)
              if (__uint_as_float(sr[jj]) >= T) bits |= 1u << jj;
            if (ranked) mw[w] = bits & low_bits(c - 32 * w);
          }
          cnt += __popc(mw[w]);
        }
        // ties at T beyond the quota: take the tied blocks in increasing index
        if (__any_sync(0xffffffffu, ranked && cnt > m)) {
          int need = m;
#pragma unroll
          for (int i = 0; i < KB; ++i) need -= (i < m && a[i] > T) ? 1 : 0;
          const bool fix = ranked && cnt > m;
#pragma unroll
          for (int w = 0; w < kMaxBlocks / 32; ++w) {
            if (w * 32 < jlim) {
              uint32_t sr[32];
              tmem_ld32(tS + w * 32, sr);
              tmem_wait_ld();
              uint32_t bits = 0;
#pragma unroll
              for (int jj = 0; jj < 32; ++jj) {
                const float s = __uint_as_float(sr[jj]);
                const bool cand = w * 32 + jj < c;
                const bool take = cand && s == T && need > 0;
                need -= take ? 1 : 0;
                if (cand && (s > T || take)) bits |= 1u << jj;
              }
              if (fix) mw[w] = bits;
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(bar(&ctl.s_free[wg]));
      if (valid) {
        int32_t* outp = sel + ((size_t)(b * dm.N + t) * dm.hq + h) * dm.topk;
        if (gp.mode != kOutSel) {
          // the candidate mask travels between the passes in the row's sel entries
          const int nwc = (c + 31) >> 5;
          if (gp.mode != kMaskStore) {
#pragma unroll
            for (int w = 0; w < kMaxBlocks / 32; ++w)
              if (w < nwc) mw[w] |= (uint32_t)outp[w];
          }
          if (gp.mode != kMaskUnion) {
#pragma unroll
            for (int w = 0; w < kMaxBlocks / 32; ++w)
              if (w < nwc) outp[w] = (int32_t)mw[w];
          }
        }
        if (gp.mode == kOutSel || gp.mode == kMaskUnion) {
          int pos = 0;
#pragma unroll
          for (int w = 0; w < kMaxBlocks / 32; ++w) {
            uint32_t x = mw[w];
            while (x) {
              const int j = w * 32 + __ffs(x) - 1;
              x &= x - 1;
              outp[pos++] = j;
              atomicAdd(&ctl.hist[j], 1);
            }
          }
          // pos is m for the plain gate unless a score was NaN (then the row
          // keeps fewer blocks); for the union it is the size of the union
          outp[pos] = c;
          for (int i = pos + 1; i < dm.topk; ++i) outp[i] = -1;
        }
      }
    }
  } else if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      int issued = 0;
      for (int k = 0; k < ntiles; ++k) {
        if (k >= 1 && !mbar_wait(bar(&ctl.q_free), (k - 1) & 1, abort_flag)) break;
        const int tt = t_begin + (k / nsub) * TT;
        const int h0 = g * dm.G + (k % nsub) * GT;
        const uint32_t qs = base + kOffQ;
        mbar_arrive_expect_tx(bar(&ctl.q_full), kQTile);
        tma_load_3d(qs, &tmQ, 0, h0, b * dm.N + tt, bar(&ctl.q_full));
        tma_load_3d(qs + kHalfQ, &tmQ, 64, h0, b * dm.N + tt, bar(&ctl.q_full));
        issued = k + 1;
      }
      if (*abort_flag && issued > 0) {
        int never = 0;
        mbar_wait(bar(&ctl.q_full), (issued - 1) & 1, &never);
      }
    }
  } else {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = true;
      for (int k = 0; k < ntiles && ok; ++k) {
        const int s = k & 1;
        const int tt = t_begin + (k / nsub) * TT;
        const int ctile = (min(t_stop, tt + TT) - 1) / dm.B;
        const int nt = max(16, (ctile + 15) / 16 * 16);
        ok = mbar_wait(bar(&ctl.q_full), k & 1, abort_flag);
        if (ok && k >= 2) ok = mbar_wait(bar(&ctl.s_free[s]), ((k >> 1) - 1) & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
        if (ctile > 0 && KH > 0) {
          const uint32_t idesc = idesc_bf16(128, nt, false);
          const uint32_t qa = base + kOffQ;
          const uint32_t d = tb + s * 256u;
          // smallest term first: the accumulator is still small while the
          // low-order products are added (one term: hi only)
          const int t0 = kTerms - gp.nterms;
          for (int term = t0; term < kTerms; ++term) {
            const uint32_t kt = klo - term * kKB;   // lo, mid, hi
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t qo = (kk >> 2) * kHalfQ + (kk & 3) * 32;
              const uint32_t ko = (kk >> 2) * kKBHalf + (kk & 3) * 32;
              mma_ss(d, sdesc_sw128(qa + qo, 16, 1024), sdesc_sw128(kt + ko, 16, 1024), idesc,
                     (term > t0 || kk > 0) ? 1u : 0u);
            }
          }
        }
        mma_commit(bar(&ctl.s_full[s]));
        mma_commit(bar(&ctl.q_free));
      }
      if (!ok) {
        int never = 0;
        mma_commit(bar(&ctl.drain));
        mbar_wait(bar(&ctl.drain), 0, &never);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // rows per (pass, b, g, j) of the whole CTA (one pass)
  int32_t* cnt_g = counts + ((size_t)(pp * dm.batch + b) * dm.hkv + g) * dm.n;
  for (int i = tid; i < cmax_cta; i += kThreads) {
    const int v = ctl.hist[i];
    if (v) atomicAdd(&cnt_g[i], v);
  }
  if (warp == 8) tmem_dealloc(tb, 512);
  if (tid == 0 && ctl.abort) atomicExch(status, (int)MOBA_ERR_TIMEOUT);
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn_gate() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) == cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

int gate_ctas(const Dims& dm) {
  const int L = dm.chunk < kTokens ? dm.chunk : kTokens;
  const int rpp = (dm.chunk + L - 1) / L;
  const int np = (dm.t_hi - 1) / dm.chunk - dm.t_lo / dm.chunk + 1;
  return rpp * np * dm.hkv * dm.batch;
}

template <int KB>
cudaError_t run_select(const CUtensorMap& mq, const Dims& dm, const GatePass& gp, int32_t* sel,
                       int32_t* counts, int* status, cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(gate_select_tc_kernel<KB>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  gate_select_tc_kernel<KB><<<gate_ctas(dm), kThreads, kSmemBytes, stream>>>(mq, gp, sel, counts,
                                                                             status, dm);
  return cudaGetLastError();
}

cudaError_t run_pass(const Dims& dm, const void* q, const GatePass& gp, int32_t* sel, int32_t* counts,
                     int* status, cudaStream_t stream) {
  // q viewed as [b * N][hq][d]: a box of 64 columns x GT heads x 128 / GT tokens
  // lands in shared memory as 128 rows of 128 bytes, token-major
  const int GT = (kRowsT % dm.G == 0) ? dm.G : 1;
  CUtensorMap mq;
  cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)dm.hq, (cuuint64_t)dm.batch * dm.N};
  cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)dm.hq * kD * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)GT, (cuuint32_t)(kRowsT / GT)};
  cuuint32_t es[3] = {1, 1, 1};
  if (encode_fn_gate()(&mq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), dims, strides, box,
                       es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                       CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                       CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  // list length of the sorting networks: 4, 8 or 16 >= the ranking's slots
  return gp.slots <= 4   ? run_select<4>(mq, dm, gp, sel, counts, status, stream)
         : gp.slots <= 8 ? run_select<8>(mq, dm, gp, sel, counts, status, stream)
                         : run_select<16>(mq, dm, gp, sel, counts, status, stream);
}

}  // namespace

bool gate_tc_supported(const Dims& dm, int dtype) {
  return dtype == MOBA_BF16 && dm.d == kD && dm.n <= kMaxBlocks && encode_fn_gate() != nullptr;
}

cudaError_t launch_gate_select_tc(const Dims& dm, const void* q, const float* meank, int32_t* sel,
                                  int32_t* counts, int* status, cudaStream_t stream) {
  return run_pass(dm, q, GatePass{meank, kTerms, dm.topk - 1, kOutSel}, sel, counts, status, stream);
}

bool gate_tc_pooled_supported(const Dims& dm, int dtype) {
  // the candidate mask of a row (ceil(c / 32) words, c <= n - 1) must fit its W-wide sel row
  return gate_tc_supported(dm, dtype) && (dm.n - 1 + 31) / 32 <= dm.topk;
}

cudaError_t launch_gate_select_tc_pooled(const Dims& dm, int km, int extra, const void* q,
                                         const float* meank, const float* maxk, const float* mink,
                                         int32_t* sel, int32_t* counts, int* status,
                                         cudaStream_t stream) {
  cudaError_t e = run_pass(dm, q, GatePass{meank, kTerms, km, kMaskStore}, sel, counts, status, stream);
  if (e != cudaSuccess) return e;
  e = run_pass(dm, q, GatePass{maxk, 1, extra, kMaskOr}, sel, counts, status, stream);
  if (e != cudaSuccess) return e;
  return run_pass(dm, q, GatePass{mink, 1, extra, kMaskUnion}, sel, counts, status, stream);
}

}  // namespace moba
