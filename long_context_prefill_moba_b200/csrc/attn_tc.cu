// K3 on 5th-generation tensor cores (tcgen05 + TMEM + TMA): the two attention
// steps of MoBA for bf16, head_dim D = 128 or 64.
//
// "MoBA: Mixture of Block Attention for Long-Context LLMs", paper-graph summary
// §3 "The Core MoBA Attention Equation" (Softmax(q K[I]^T) V[I]), "Causality
// Enforcement" mechanism 2 (causal mask inside the current block) and the
// Implementation section, Algorithm 1 Step 3 (historical blocks without a
// mask, the queries that routed to a block gathered so the block's keys and
// values are loaded once for all of them; the current block causal) and Step 4
// (online-softmax merge of the partial results).
//
// Two modes of one kernel template:
//   kHist  one CTA = up to 256 query rows of one (b, kv head g, earlier block j)
//          group (taken from the gate's `rows` list), all B keys of block j,
//          no mask; writes each row's normalised partial (o, log2-sum-exp2).
//   kCur   one CTA = 128 consecutive tokens of two query heads of one kv group
//          (one head when the group size is odd and this is the last head);
//          keys from the start of the first token's block up to the last
//          token, causal inside each token's own block; the epilogue merges the
//          row's historical partials and writes out (and lse).
// The 256 rows are two 128-row tiles Q0 / Q1 (TMEM lanes = rows).  Roles:
//   warps 0-3  softmax for Q0        warps 4-7  softmax for Q1
//   warp 8     TMA producer of K/V tiles (and TMEM allocation)
//   warp 9     single-thread tcgen05.mma issuer      warps 10-11 idle
// The softmax warpgroups raise their register budget to 216 with setmaxnreg
// and the third warpgroup drops to 64 (384 x 168 at launch = 256 x 216 + 128 x 64
// + 1024 spare).
// Per 128-key tile i: S_w = Q_w K_i^T (SS MMA, fp32 in TMEM), the softmax warps
// read S_w, keep a lazily rescaled running max, write P_w = exp2(S - m) as bf16
// back over S_w, and O_w += P_w V_i runs as a TS MMA (A operand from TMEM).
// TMEM: S0 [0,128) S1 [128,256) O0 [256,256+D) O1 [384,384+D) columns.
// SMEM: Q0 Q1, K and V double buffered, each tile 128 rows x D (32 KB for
// D = 128, 16 KB for D = 64): 192 or 96 KB.  All tiles use the 128-byte
// swizzled K-major layout in 64-column halves (V is read MN-major).
//
// The MMA issue order per tile i is PV0_i, S0_{i+1}, PV1_i, S1_{i+1}; tcgen05
// operations of one thread execute in order and a commit covers every earlier
// operation, so when S_w(i+1) is signalled complete, PV_w(i) is complete too and
// the softmax warps may rescale O_w in place before releasing P_w(i+1).
//
// Every wait is bounded (2 s); on expiry the CTA drains what it issued, frees
// TMEM and reports MOBA_ERR_TIMEOUT through the status word.
#include <cudaTypedefs.h>

#include "launch.h"
#include "sm100.cuh"

namespace moba {

namespace {

using namespace sm100;

constexpr int kHist = 0, kCur = 1;

constexpr int kQT = 128;                 // rows per Q tile
constexpr int kBK = 128;                 // keys per K/V tile
constexpr int kRowsPerCta = 2 * kQT;
constexpr int kThreads = 384;
constexpr int kLaunchRegs = 168;         // registers per thread at launch (ptxas, 384 threads, 1 CTA/SM)
constexpr int kSoftmaxRegs = 216;
constexpr int kServiceRegs = 64;
static_assert(2 * 128 * kSoftmaxRegs + 128 * kServiceRegs <= kThreads * kLaunchRegs,
              "register split exceeds the launch allocation");
constexpr uint32_t kHalf = 16384;       // a 64-column half of a 128-row tile (128-byte rows)
constexpr float kRescaleThreshold = 8.f; // log2 units: rescale O only when the max grows by > 2^8
// A tile whose probabilities, taken against the row's current base, sum to at
// most 2^15 (so none exceeds 2^15) is accepted without computing its row max.
constexpr float kFastSumLimit = 32768.f;
// Of every 8 pairs of exponentials, this many run on the FMA pipe
// (exp2_poly2) and the rest on the special-function unit, whose 16 results
// per clock per SM alone would take as long as the tile's two MMAs.
#ifndef MOBA_POLY_OF8
#define MOBA_POLY_OF8 0
#endif
constexpr int kPolyOf8 = MOBA_POLY_OF8;
static_assert(kPolyOf8 >= 0 && kPolyOf8 <= 8, "pairs per 8");
// merge staging in the current-block epilogue: per softmax warp kMergeStages
// slots of 32 rows; the 8 warps' stages fill the Q/K/V buffers
constexpr int kMergeStages = 3;

// Shared-memory geometry for head_dim D (64 or 128).  Q, K and V tiles are 128
// rows of D bf16, stored as D / 64 column halves of 128-byte rows (16 KB
// each), 128-byte swizzled; Q0 Q1 at 0, K stages at 2 tiles, V stages at 4.
template <int D>
struct Geo {
  static_assert(D == 64 || D == 128, "head_dim 64 or 128");
  static constexpr uint32_t kTile = kBK * D * 2;
  static constexpr int kHalves = D / 64;
  static constexpr uint32_t kOffQ = 0, kOffK = 2 * kTile, kOffV = 4 * kTile;
  static constexpr uint32_t kSmem = 6 * kTile + 1024;
  static constexpr int kRowBytes = 2 * D;           // one bf16 row
  static constexpr int kChunks = D / 8;             // its 16-byte chunks
  static constexpr int kRowsPerOp = 32 / kChunks;   // rows one warp instruction covers
  static constexpr uint32_t kMergeSlot = 32 * kRowBytes;
  static constexpr uint32_t kMergeWarp = kMergeStages * kMergeSlot;
  static_assert(8 * kMergeWarp <= 6 * kTile, "merge staging exceeds the tile buffers");
};
// MUFU exponential: 1 = ex2.approx.ftz.f32 directly, 0 = exp2f
#ifndef MOBA_EX2_DIRECT
#define MOBA_EX2_DIRECT 1
#endif

struct Ctl {
  uint64_t q_full[2], k_full[2], v_full[2], k_free[2], v_free[2], s_full[2], p_full[2], o_full[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

MOBA_DEV uint32_t bar(const uint64_t* b) { return smem_u32(b); }
MOBA_DEV float ex2(float x) { return MOBA_EX2_DIRECT ? ex2_approx(x) : exp2f(x); }

struct Tile {
  int b, g, nq;
  int key0;        // sequence position of key tile 0
  int nkt;         // key tiles
  int j;           // kHist: the block
  int r0, cnt;     // kHist: rows[r0 .. r0 + cnt)
  int h0, t_first, t_last;   // kCur
};

// 32 rows of D bf16 staged in shared memory: 16-byte chunk c of row rr at
// rr * 2D + ((c ^ (rr mod D/8)) << 4), so that a warp writing one row per lane
// and reading whole rows (two or four per instruction) both spread over the banks
template <int D>
MOBA_DEV uint32_t stage_off(int rr, int c) {
  return (uint32_t)(rr * Geo<D>::kRowBytes + ((c ^ (rr & (Geo<D>::kChunks - 1))) << 4));
}
MOBA_DEV void st_shared_v4(uint32_t a, uint32_t x, uint32_t y, uint32_t z, uint32_t w) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};\n" ::"r"(a), "r"(x), "r"(y), "r"(z), "r"(w) : "memory");
}
// rows staged by the warp (lane i staged row i, destination row index `row`
// of `dst`, D bf16 per row) written whole rows at a time (two per instruction
// for D = 128, four for D = 64)
template <int D>
MOBA_DEV void store_rows_from_stage(uint32_t stg, __nv_bfloat16* dst, int64_t row, bool valid, int lane) {
  using G = Geo<D>;
  const int cc = lane % G::kChunks;
#pragma unroll
  for (int k2 = 0; k2 < 32 / G::kRowsPerOp; ++k2) {
    const int rl = G::kRowsPerOp * k2 + lane / G::kChunks;
    const int64_t rd = __shfl_sync(0xffffffffu, (long long)row, rl);
    const bool vd = __shfl_sync(0xffffffffu, valid, rl);
    uint32_t x, y, z, w;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];\n"
                 : "=r"(x), "=r"(y), "=r"(z), "=r"(w)
                 : "r"(stg + stage_off<D>(rl, cc)));
    if (vd) *reinterpret_cast<uint4*>(dst + rd * D + cc * 8) = make_uint4(x, y, z, w);
  }
}

template <int MODE>
MOBA_DEV bool decode_tile(Tile& w, const int32_t* tile_start, const int32_t* offsets, const Dims& dm,
                          int ch) {
  const int t0 = ch * dm.chunk;
  if (MODE == kHist) {
    const int ngroups = dm.batch * dm.hkv * dm.n;
    const int tile = blockIdx.x;
    if (tile >= tile_start[ngroups]) return false;
    int lo = 0, hi = ngroups - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (tile_start[mid] <= tile) lo = mid; else hi = mid - 1;
    }
    w.j = lo % dm.n;
    w.g = (lo / dm.n) % dm.hkv;
    w.b = lo / (dm.n * dm.hkv);
    const size_t goff = (size_t)ch * ngroups + lo;
    w.r0 = offsets[goff] + (tile - tile_start[lo]) * kRowsPerCta;
    w.cnt = min(kRowsPerCta, offsets[goff + 1] - w.r0);
    w.nq = w.cnt > kQT ? 2 : 1;
    w.key0 = w.j * dm.B;
    w.nkt = (dm.B + kBK - 1) / kBK;
  } else {
    const int t_end = min(dm.N, t0 + dm.chunk);
    const int ntile = (t_end - t0 + kQT - 1) / kQT;
    const int pairs = (dm.G + 1) / 2;
    int idx = blockIdx.x;
    // the last token tiles of a block (or of the sequence, with one block) have
    // the most keys: they start first, so the launch does not end on them
    const int tau = ntile - 1 - idx % ntile; idx /= ntile;
    const int p = idx % pairs; idx /= pairs;
    w.g = idx % dm.hkv;
    w.b = idx / dm.hkv;
    if (w.b >= dm.batch) return false;
    w.h0 = w.g * dm.G + 2 * p;
    w.nq = (2 * p + 1 < dm.G) ? 2 : 1;
    w.t_first = t0 + tau * kQT;
    w.t_last = min(t_end, w.t_first + kQT) - 1;
    w.key0 = (w.t_first / dm.B) * dm.B;
    w.nkt = (w.t_last - w.key0) / kBK + 1;
  }
  return true;
}

template <int MODE, int D>
__global__ void __launch_bounds__(kThreads, 1) attn_tc_kernel(
    const __nv_bfloat16* __restrict__ q, const __grid_constant__ CUtensorMap tmK,
    const __grid_constant__ CUtensorMap tmV, const int32_t* __restrict__ sel,
    const int32_t* __restrict__ offsets, const int32_t* __restrict__ rows,
    const int32_t* __restrict__ tile_start, float* __restrict__ part_o,
    float* __restrict__ part_lse, __nv_bfloat16* __restrict__ out, float* __restrict__ lse,
    int* __restrict__ status, Dims dm, int ch) {
  using G = Geo<D>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ Ctl ctl;
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;

  Tile wk;
  if (!decode_tile<MODE>(wk, tile_start, offsets, dm, ch)) return;
  const int b = wk.b, g = wk.g, nq = wk.nq, nkt = wk.nkt;
  const int KH = dm.topk - 1;
  const int t0 = ch * dm.chunk;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int w = 0; w < 2; ++w) {
      mbar_init(bar(&ctl.q_full[w]), kQT);
      mbar_init(bar(&ctl.p_full[w]), kQT);
      mbar_init(bar(&ctl.k_full[w]), 1);
      mbar_init(bar(&ctl.v_full[w]), 1);
      mbar_init(bar(&ctl.k_free[w]), 1);
      mbar_init(bar(&ctl.v_free[w]), 1);
      mbar_init(bar(&ctl.s_full[w]), 1);
      mbar_init(bar(&ctl.o_full[w]), 1);
    }
    mbar_init(bar(&ctl.drain), 1);
    ctl.abort = 0;
    fence_mbar_init();
  }
  if (warp == 8) {
    tmem_alloc(smem_u32(&ctl.tmem_base), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = ctl.tmem_base;
  volatile int* abort_flag = &ctl.abort;
  if (warp < 8)
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(kSoftmaxRegs));
  else
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(kServiceRegs));

  if (warp < 8) {
    // ------------------------------------------------------------ softmax
    const int w = warp >> 2;
    if (w < nq) {
      const int rho = tid & 127;
      bool valid;
      int r, t, h;
      if (MODE == kHist) {
        const int row_i = w * kQT + rho;
        valid = row_i < wk.cnt;
        r = valid ? rows[wk.r0 + row_i] : 0;
        h = r % dm.hq;
        t = (r / dm.hq) % dm.N;
      } else {
        t = wk.t_first + rho;
        valid = t <= wk.t_last;
        h = wk.h0 + w;
        r = valid ? (b * dm.N + t) * dm.hq + h : 0;
      }
      // the warp copies its 32 rows whole rows at a time: for D = 128 lanes
      // 0-15 take the 16 chunks of one row and lanes 16-31 those of the next
      // (four rows of 8 chunks for D = 64), so each copy instruction reads
      // whole rows instead of 16 bytes of 32 rows
      const uint32_t qs = base + G::kOffQ + w * G::kTile;
      {
        const int wrow0 = (warp & 3) * 32, cc = lane % G::kChunks;
#pragma unroll
        for (int k2 = 0; k2 < 32 / G::kRowsPerOp; ++k2) {
          const int rl = G::kRowsPerOp * k2 + lane / G::kChunks;
          const int rs = __shfl_sync(0xffffffffu, r, rl);
          const bool vs = __shfl_sync(0xffffffffu, valid, rl);
          cp_async16(qs + (cc >> 3) * kHalf + sw128_off(wrow0 + rl, cc & 7), q + (size_t)rs * D + cc * 8, vs);
        }
      }
      cp_async_commit();
      cp_async_wait<0>();
      fence_proxy_async_smem();
      mbar_arrive(bar(&ctl.q_full[w]));
      // causal window of this row in kCur: keys [lo_t, t]
      const int lo_t = (t / dm.B) * dm.B;
      const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
      const uint32_t tS = tb + (w ? 128u : 0u) + lane_off;
      const uint32_t tO = tb + (w ? 384u : 256u) + lane_off;
      const float sl2 = dm.scale_log2;
      float m_used = -INFINITY, l = 0.f;
      bool ok = true;
      // S tile i into registers, keys outside the row's window set to -inf
      auto load_s = [&](uint32_t (&sr)[128], int i) {
        tmem_ld32(tS + 0, sr);
        tmem_ld32(tS + 32, sr + 32);
        tmem_ld32(tS + 64, sr + 64);
        tmem_ld32(tS + 96, sr + 96);
        tmem_wait_ld();
        // keys of this tile valid for this row: positions [vlo, vhi] relative to the tile
        const int u0 = wk.key0 + i * kBK;
        int vlo, vhi;
        if (MODE == kHist) {
          vlo = 0;
          vhi = dm.B - i * kBK - 1;
        } else {
          vlo = lo_t - u0;
          vhi = t - u0;
        }
        if (!(vlo <= 0 && vhi >= kBK - 1)) {
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c < vlo || c > vhi) sr[c] = __float_as_uint(-INFINITY);
        }
      };
      // p = 2^(s * scale * log2(e) - mb) as bf16 pairs; returns the fp32 sum of p
      auto exp_tile = [&](const uint32_t (&sr)[128], float mb, uint32_t (&pk)[64]) -> float {
        const uint64_t sl2x2 = f2_pack(sl2, sl2), nmbx2 = f2_pack(-mb, -mb);
        uint64_t rs4[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const uint64_t x2 =
              f2_fma(f2_pack(__uint_as_float(sr[2 * c]), __uint_as_float(sr[2 * c + 1])), sl2x2, nmbx2);
          uint64_t p2;
          if (((c * kPolyOf8) & 7) < kPolyOf8) {
            p2 = exp2_poly2(x2);
          } else {
            float x0, x1;
            f2_unpack(x2, x0, x1);
            p2 = f2_pack(ex2(x0), ex2(x1));
          }
          rs4[c & 3] = f2_add(rs4[c & 3], p2);
          float p0, p1;
          f2_unpack(p2, p0, p1);
          pk[c] = pack_bf16x2(p0, p1);
        }
        float a0, a1;
        f2_unpack(f2_add(f2_add(rs4[0], rs4[1]), f2_add(rs4[2], rs4[3])), a0, a1);
        return a0 + a1;
      };
      for (int i = 0; i < nkt && ok; ++i) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar(&ctl.s_full[w]), i & 1, abort_flag));
        if (!ok) break;
        tc_fence_after();
        uint32_t sr[128], pk[64];
        float ts = 0.f;
        load_s(sr, i);
        // fast path: exponentials against the current base m_used, no row max;
        // taken back (S reloaded from TMEM) if any row of the warp sums above
        // the limit or has no base yet
        bool slow = __any_sync(0xffffffffu, m_used == -INFINITY);
        if (!slow) {
          ts = exp_tile(sr, m_used, pk);
          slow = __any_sync(0xffffffffu, !(ts <= kFastSumLimit));
          if (slow) load_s(sr, i);
        }
        if (slow) {
          // row max: four independent chains of three-input maxima, then a tree
          float mx4[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) mx4[u] = fmaxf(__uint_as_float(sr[2 * u]), __uint_as_float(sr[2 * u + 1]));
#pragma unroll
          for (int c = 8; c < 128; c += 8)
#pragma unroll
            for (int u = 0; u < 4; ++u)
              mx4[u] = max3(mx4[u], __uint_as_float(sr[c + 2 * u]), __uint_as_float(sr[c + 2 * u + 1]));
          const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
          const float mxs = mx * sl2;
          const bool need = mxs > m_used + kRescaleThreshold;
          if (i > 0 && __any_sync(0xffffffffu, need)) {
            // S_i complete implies PV_(i-1) complete (MMA issue order), so O is final here
            const float f = need ? exp2f(m_used - mxs) : 1.f;
#pragma unroll
            for (int cc = 0; cc < D / 32; ++cc) {
              uint32_t o[32];
              tmem_ld32(tO + cc * 32, o);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
              tmem_st32(tO + cc * 32, o);
            }
            tmem_wait_st();
          }
          if (need) {
            l *= exp2f(m_used - mxs);
            m_used = mxs;
          }
          // a row with no valid key yet keeps m_used = -inf: use 0 as the base (p = 0)
          ts = exp_tile(sr, m_used == -INFINITY ? 0.f : m_used, pk);
        }
        l += ts;
        tmem_st32(tS + 0, pk);
        tmem_st32(tS + 32, pk + 32);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(&ctl.p_full[w]));
      }
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(&ctl.o_full[w]), 0, abort_flag));
      if (ok) {
        tc_fence_after();
        const float lse2 = m_used + log2f(l);
        if (MODE == kHist) {
          size_t pidx = 0;
          if (valid) {
            const int slot = slot_of(sel + (size_t)r * dm.topk, dm.topk, wk.j);
            pidx = (size_t)((b * dm.chunk + (t - t0)) * dm.hq + h) * KH + slot;
          }
          const float inv = 1.f / l;
          // partials are kept in bf16 (the merge is done in fp32; the
          // rounding, 2^-9 relative of a normalised output, stays far below
          // the output tolerance) to halve their HBM traffic.  Every MMA has
          // completed, so each warp stages its 32 rows in its 8 KB of the Q
          // buffers and stores two whole rows per instruction.
          const uint32_t stg = base + G::kOffQ + (uint32_t)warp * (32u * G::kRowBytes);
#pragma unroll
          for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t o[32];
            tmem_ld32(tO + cc * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int e8 = 0; e8 < 4; ++e8)
              st_shared_v4(stg + stage_off<D>(lane, cc * 4 + e8),
                           pack_bf16x2(__uint_as_float(o[8 * e8 + 0]) * inv, __uint_as_float(o[8 * e8 + 1]) * inv),
                           pack_bf16x2(__uint_as_float(o[8 * e8 + 2]) * inv, __uint_as_float(o[8 * e8 + 3]) * inv),
                           pack_bf16x2(__uint_as_float(o[8 * e8 + 4]) * inv, __uint_as_float(o[8 * e8 + 5]) * inv),
                           pack_bf16x2(__uint_as_float(o[8 * e8 + 6]) * inv, __uint_as_float(o[8 * e8 + 7]) * inv));
          }
          __syncwarp();
          store_rows_from_stage<D>(stg, reinterpret_cast<__nv_bfloat16*>(part_o), (int64_t)pidx, valid, lane);
          if (valid) part_lse[pidx] = lse2;
        } else {
          // merge with the historical partials of the row (Algorithm 1 Step 4).
          // Every MMA has completed, so the Q/K/V buffers are free: each warp
          // stages the partials of its 32 rows there slot by slot (one cp.async
          // of the warp copies two rows' 256 contiguous bytes), kMergeStages
          // slots in flight, and each lane reads its own row back.
          const int nh = valid ? min(KH, t / dm.B) : 0;
          const size_t pbase = (size_t)((b * dm.chunk + (t - t0)) * dm.hq + h) * KH;
          float pl[MOBA_MAX_TOPK - 1];
          float M = lse2;
#pragma unroll
          for (int s = 0; s < MOBA_MAX_TOPK - 1; ++s) {
            pl[s] = s < nh ? part_lse[pbase + s] : -INFINITY;
            M = fmaxf(M, pl[s]);
          }
          const float wc = exp2f(lse2 - M);
          float W = wc;
#pragma unroll
          for (int s = 0; s < MOBA_MAX_TOPK - 1; ++s) W += exp2f(pl[s] - M);
          const float iw = 1.f / W;
          const float fc = wc / l * iw;
          float acc[D];
#pragma unroll
          for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t o[32];
            tmem_ld32(tO + cc * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) acc[cc * 32 + e] = __uint_as_float(o[e]) * fc;
          }
          fence_proxy_async_smem();
          const int nhw = __reduce_max_sync(0xffffffffu, nh);
          const uint32_t stage = base + (uint32_t)warp * G::kMergeWarp;
          const __nv_bfloat16* pb = reinterpret_cast<const __nv_bfloat16*>(part_o);
          // row rr of this warp is token t - lane + rr: its partials start rr * hq * KH slots later
          const size_t pbase0 = pbase - (size_t)lane * dm.hq * KH;
          auto issue = [&](int sl) {
            const uint32_t buf = stage + (uint32_t)(sl % kMergeStages) * G::kMergeSlot;
#pragma unroll
            for (int k = 0; k < 32 / G::kRowsPerOp; ++k) {
              const int rr = G::kRowsPerOp * k + lane / G::kChunks, c = lane % G::kChunks;
              const bool live = sl < __shfl_sync(0xffffffffu, nh, rr);
              const __nv_bfloat16* src = live ? pb + (pbase0 + (size_t)rr * dm.hq * KH + sl) * D + c * 8 : pb;
              cp_async16(buf + stage_off<D>(rr, c), src, live);
            }
          };
#pragma unroll
          for (int k = 0; k < kMergeStages - 1; ++k) {
            if (k < nhw) issue(k);
            cp_async_commit();
          }
          for (int sl = 0; sl < nhw; ++sl) {
            if (sl + kMergeStages - 1 < nhw) issue(sl + kMergeStages - 1);
            cp_async_commit();
            cp_async_wait<kMergeStages - 1>();
            __syncwarp();
            if (sl < nh) {
              const float ws = exp2f(part_lse[pbase + sl] - M) * iw;
              const uint32_t row = stage + (uint32_t)(sl % kMergeStages) * G::kMergeSlot;
#pragma unroll
              for (int c = 0; c < G::kChunks; ++c) {
                uint32_t w4[4];
                asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];\n"
                             : "=r"(w4[0]), "=r"(w4[1]), "=r"(w4[2]), "=r"(w4[3])
                             : "r"(row + stage_off<D>(lane, c)));
#pragma unroll
                for (int h2 = 0; h2 < 4; ++h2) {
                  const float2 f2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w4[h2]));
                  acc[8 * c + 2 * h2] = fmaf(ws, f2.x, acc[8 * c + 2 * h2]);
                  acc[8 * c + 2 * h2 + 1] = fmaf(ws, f2.y, acc[8 * c + 2 * h2 + 1]);
                }
              }
            }
            __syncwarp();
          }
          // out rows through the warp's (now idle) staging slot 0: two whole
          // rows per store instruction
#pragma unroll
          for (int e8 = 0; e8 < G::kChunks; ++e8)
            st_shared_v4(stage + stage_off<D>(lane, e8), pack_bf16x2(acc[8 * e8 + 0], acc[8 * e8 + 1]),
                         pack_bf16x2(acc[8 * e8 + 2], acc[8 * e8 + 3]), pack_bf16x2(acc[8 * e8 + 4], acc[8 * e8 + 5]),
                         pack_bf16x2(acc[8 * e8 + 6], acc[8 * e8 + 7]));
          __syncwarp();
          store_rows_from_stage<D>(stage, out, (int64_t)r, valid, lane);
          if (valid && lse != nullptr)
            lse[((size_t)b * dm.hq + h) * dm.N + t] = (M + log2f(W)) * kLn2;
        }
      }
    }
  } else if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      const int y0 = b * dm.N + wk.key0;
      const int x0 = g * D;
      int issued_k = 0, issued_v = 0;
      for (int i = 0; i < nkt; ++i) {
        const int s = i & 1;
        const uint32_t ks = base + G::kOffK + s * G::kTile, vs = base + G::kOffV + s * G::kTile;
        if (i >= 2 && !mbar_wait(bar(&ctl.k_free[s]), ((i >> 1) - 1) & 1, abort_flag)) break;
        mbar_arrive_expect_tx(bar(&ctl.k_full[s]), G::kTile);
#pragma unroll
        for (int hh = 0; hh < G::kHalves; ++hh)
          tma_load_2d(ks + hh * kHalf, &tmK, x0 + 64 * hh, y0 + i * kBK, bar(&ctl.k_full[s]));
        issued_k = i + 1;
        if (i >= 2 && !mbar_wait(bar(&ctl.v_free[s]), ((i >> 1) - 1) & 1, abort_flag)) break;
        mbar_arrive_expect_tx(bar(&ctl.v_full[s]), G::kTile);
#pragma unroll
        for (int hh = 0; hh < G::kHalves; ++hh)
          tma_load_2d(vs + hh * kHalf, &tmV, x0 + 64 * hh, y0 + i * kBK, bar(&ctl.v_full[s]));
        issued_v = i + 1;
      }
      if (*abort_flag) {
        // let the copies this thread issued land before the CTA exits
        int never = 0;
        for (int i = (issued_k > 2 ? issued_k - 2 : 0); i < issued_k; ++i)
          mbar_wait(bar(&ctl.k_full[i & 1]), (i >> 1) & 1, &never);
        for (int i = (issued_v > 2 ? issued_v - 2 : 0); i < issued_v; ++i)
          mbar_wait(bar(&ctl.v_full[i & 1]), (i >> 1) & 1, &never);
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idS = idesc_bf16(128, kBK, false);
      const uint32_t idO = idesc_bf16(128, D, true);
      // descriptor words precomputed once; each MMA adds a compile-time offset
      const uint32_t hi = sdesc_hi(1024);
      const uint32_t loQ = sdesc_lo(base + G::kOffQ, 16), loK = sdesc_lo(base + G::kOffK, 16),
                     loV = sdesc_lo(base + G::kOffV, kHalf);
      auto issue_s = [&](int w, int s) {
        const uint32_t qa = loQ + (w ? (G::kTile >> 4) : 0u), ka = loK + (s ? (G::kTile >> 4) : 0u);
        const uint32_t d = tb + (w ? 128u : 0u);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk >> 2) * kHalf + (kk & 3) * 32) >> 4;
          mma_ss(d, sdesc_join(qa + off, hi), sdesc_join(ka + off, hi), idS, kk > 0);
        }
      };
      auto issue_pv = [&](int w, int s, bool acc) {
        const uint32_t va = loV + (s ? (G::kTile >> 4) : 0u);
        const uint32_t d = tb + (w ? 384u : 256u), a = tb + (w ? 128u : 0u);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(d, a + kk * 8, sdesc_join(va + ((kk * 2048) >> 4), hi), idO, (acc || kk > 0) ? 1u : 0u);
      };
      bool ok = mbar_wait(bar(&ctl.q_full[0]), 0, abort_flag);
      if (ok && nq == 2) ok = mbar_wait(bar(&ctl.q_full[1]), 0, abort_flag);
      if (ok) ok = mbar_wait(bar(&ctl.k_full[0]), 0, abort_flag);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
        mma_commit(bar(&ctl.s_full[0]));
        if (nq == 2) {
          issue_s(1, 0);
          mma_commit(bar(&ctl.s_full[1]));
        }
        mma_commit(bar(&ctl.k_free[0]));
      }
      for (int i = 0; i < nkt && ok; ++i) {
        const int s = i & 1, s1 = (i + 1) & 1;
        const bool more = i + 1 < nkt;
        // the K/V tiles are normally resident long before P0: their barriers
        // are waited for first, so that PV0 and S0 go out back to back
        ok = mbar_wait(bar(&ctl.v_full[s]), (i >> 1) & 1, abort_flag) &&
             (!more || mbar_wait(bar(&ctl.k_full[s1]), ((i + 1) >> 1) & 1, abort_flag)) &&
             mbar_wait(bar(&ctl.p_full[0]), i & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
        issue_pv(0, s, i > 0);
        if (more) {
          issue_s(0, s1);
          mma_commit(bar(&ctl.s_full[0]));
        }
        if (nq == 2) {
          if (!(ok = mbar_wait(bar(&ctl.p_full[1]), i & 1, abort_flag))) break;
          tc_fence_after();
          issue_pv(1, s, i > 0);
          if (more) {
            issue_s(1, s1);
            mma_commit(bar(&ctl.s_full[1]));
          }
        }
        mma_commit(bar(&ctl.v_free[s]));
        if (more) mma_commit(bar(&ctl.k_free[s1]));
      }
      if (ok) {
        mma_commit(bar(&ctl.o_full[0]));
        if (nq == 2) mma_commit(bar(&ctl.o_full[1]));
      } else {
        // drain every MMA this thread issued before TMEM is released
        int never = 0;
        mma_commit(bar(&ctl.drain));
        mbar_wait(bar(&ctl.drain), 0, &never);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 8) tmem_dealloc(tb, 512);
  if (tid == 0 && ctl.abort) atomicExch(status, (int)MOBA_ERR_TIMEOUT);
}

}  // namespace

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

// 2-D map over a [batch*N, hkv*d] bf16 tensor, 128 rows x 64 columns per box,
// 128-byte swizzle; rows past the end read as zero.
bool make_kv_map(CUtensorMap* map, const void* base, const Dims& dm) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {(cuuint64_t)dm.hkv * dm.d, (cuuint64_t)dm.batch * dm.N};
  cuuint64_t strides[1] = {(cuuint64_t)dm.hkv * dm.d * 2};
  cuuint32_t box[2] = {64, kBK};
  cuuint32_t es[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {

// the setmaxnreg split is only safe if the kernel really launches with kLaunchRegs
template <int MODE, int D>
cudaError_t check_regs() {
  static int regs = -1;
  if (regs < 0) {
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, attn_tc_kernel<MODE, D>);
    if (e != cudaSuccess) return e;
    regs = fa.numRegs;
  }
  return regs >= kLaunchRegs ? cudaSuccess : cudaErrorInvalidConfiguration;
}

template <int MODE, int D>
cudaError_t launch_tc_d(const Dims& dm, const void* q, const void* k, const void* v,
                        const int32_t* sel, const int32_t* offsets, const int32_t* rows,
                        const AttnWs& ws, void* out, float* lse, int ch, int64_t grid,
                        cudaStream_t stream) {
  CUtensorMap mk, mv;
  if (!make_kv_map(&mk, k, dm) || !make_kv_map(&mv, v, dm)) return cudaErrorInvalidValue;
  cudaError_t e = check_regs<MODE, D>();
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(attn_tc_kernel<MODE, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           Geo<D>::kSmem);
  if (e != cudaSuccess) return e;
  attn_tc_kernel<MODE, D><<<grid, kThreads, Geo<D>::kSmem, stream>>>(
      (const __nv_bfloat16*)q, mk, mv, sel, offsets, rows, ws.tile_start, ws.part_o, ws.part_lse,
      (__nv_bfloat16*)out, lse, ws.status, dm, ch);
  return cudaGetLastError();
}

template <int MODE>
cudaError_t launch_tc(const Dims& dm, const void* q, const void* k, const void* v,
                      const int32_t* sel, const int32_t* offsets, const int32_t* rows,
                      const AttnWs& ws, void* out, float* lse, int ch, int64_t grid,
                      cudaStream_t stream) {
  if (dm.d == 128)
    return launch_tc_d<MODE, 128>(dm, q, k, v, sel, offsets, rows, ws, out, lse, ch, grid, stream);
  if (dm.d == 64)
    return launch_tc_d<MODE, 64>(dm, q, k, v, sel, offsets, rows, ws, out, lse, ch, grid, stream);
  return cudaErrorInvalidValue;
}

}  // namespace

int attn_tc_rows_per_tile() { return kRowsPerCta; }

// bf16 with head_dim 128 or 64 runs both attention steps on tcgen05 (with bf16
// partial results); fp32 on the CUDA-core kernels
bool attn_tc_path(int dtype, int d) { return dtype == MOBA_BF16 && (d == 128 || d == 64); }

// the CTA-pair historical kernel (csrc/attn_pair_tc.cu) takes the same 256-row tiles
bool attn_hist_pair_enabled();
cudaError_t launch_attn_pair_hist(const Dims& dm, const void* q, const void* k, const void* v,
                                  const int32_t* sel, const int32_t* offsets, const int32_t* rows,
                                  const AttnWs& ws, int ch, int64_t grid, cudaStream_t stream);

cudaError_t launch_attn_tc_hist(const Dims& dm, const void* q, const void* k, const void* v,
                                const int32_t* sel, const int32_t* offsets, const int32_t* rows,
                                const AttnWs& ws, int ch, int64_t grid, cudaStream_t stream) {
  if (dm.d == 128 && attn_hist_pair_enabled())
    return launch_attn_pair_hist(dm, q, k, v, sel, offsets, rows, ws, ch, grid, stream);
  return launch_tc<kHist>(dm, q, k, v, sel, offsets, rows, ws, nullptr, nullptr, ch, grid, stream);
}

cudaError_t launch_attn_tc_cur(const Dims& dm, const void* q, const void* k, const void* v,
                               const AttnWs& ws, void* out, float* lse, int ch,
                               cudaStream_t stream) {
  const int t0 = ch * dm.chunk;
  const int t_end = dm.N < t0 + dm.chunk ? dm.N : t0 + dm.chunk;
  const int64_t ntile = (t_end - t0 + kQT - 1) / kQT;
  const int64_t grid = ntile * ((dm.G + 1) / 2) * dm.hkv * dm.batch;
  return launch_tc<kCur>(dm, q, k, v, nullptr, nullptr, nullptr, ws, out, lse, ch, grid, stream);
}

}  // namespace moba
