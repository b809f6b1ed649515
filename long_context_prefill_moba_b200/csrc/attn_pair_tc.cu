// K3, historical blocks, on CTA pairs: two CTAs of a cluster share one
// tcgen05 MMA of M = 256 query rows (.cta_group::2), each holding 128 rows.
//
// "MoBA: Mixture of Block Attention for Long-Context LLMs", paper-graph summary
// §3 "The Core MoBA Attention Equation" (Softmax(q K[I]^T) V[I]) and the
// Implementation section, Algorithm 1 Step 3 (historical blocks without a
// mask; the queries routed to a block gathered so that the block's keys and
// values are loaded once for all of them).
//
// One pair = up to 256 rows of one (b, kv head g, earlier block j) group (from
// the gate's `rows`), all B keys of block j; each row's normalised partial (o
// in bf16, log2-sum-exp2 in fp32) goes to the merge of the current-block
// kernel.  CTA rank 0 ("leader") issues every MMA; rank 1 holds rows 128-255.
//
// Why pairs.  In the single-CTA kernel (two 128-row Q tiles per CTA) TMEM is
// full (S0, S1, O0, O1) and each Q tile's next scores can only be computed
// after its PV has read P out of the same columns, so softmax -> PV -> S is a
// serial chain per tile.  Here each CTA has one 128-row tile and TMEM holds
// two S buffers and O: S(i+2) is issued right after PV(i), so the scores of
// tile i+1 are ready while the softmax works on tile i.  The pair keeps the
// shared-memory traffic per query row of the two-tile kernel: each CTA loads
// half of every K tile (64 keys) and half of every V tile (64 of the d
// columns), and the MMA reads the peer's half from the peer.
//
// Roles (256 threads per CTA):
//   warps 0-3  softmax of the CTA's 128 rows (TMEM lanes), Q row gather,
//              epilogue
//   warp 4     TMA producer of this CTA's K/V halves; TMEM allocation
//   warp 5     leader: single-thread MMA issuer; rank 1: relays "my half of
//              K/V stage s landed" to the leader (each CTA's copies complete
//              on its own barrier, so each CTA can wait for its own copies)
// Barriers the MMA issuer waits on (q_full, p_full, k_peer, v_peer) live in the
// leader and are arrived on with cluster-scope release from either CTA; the
// MMA completions (s_full, pv_done, o_full, k_free, v_free) are committed to
// the same barrier in both CTAs.
//
// TMEM (512 columns allocated for the pair): S buffers at 0 and 128, O at
// 256; lanes = the CTA's rows.  P is written as bf16 over the first 64
// columns of its S buffer and read by the TS MMA.
// SMEM per CTA: Q 32 KB, 4 stages of K halves (64 keys x 128 d, 16 KB) and of
// V halves (128 keys x 64 d, 16 KB), all 128-byte swizzled (V read MN-major).
//
// Every wait is bounded (2 s); on expiry each CTA drains what it issued, the
// pair meets at a cluster barrier before TMEM is freed, and the status word
// gets MOBA_ERR_TIMEOUT.
#include <cudaTypedefs.h>
#include <stdlib.h>
#include <string.h>

#include "launch.h"
#include "sm100.cuh"

namespace moba {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn();
bool make_kv_map(CUtensorMap* map, const void* base, const Dims& dm);

namespace {

using namespace sm100;

constexpr int kD = 128;
constexpr int kQT = 128;                    // query rows per CTA
constexpr int kBK = 128;                    // keys per K/V tile (both halves)
constexpr int kRowsPerPair = 2 * kQT;
constexpr int kNS = 2;                      // S buffers in TMEM
constexpr int kStages = 4;                  // K and V half-tile buffers
constexpr uint32_t kQBytes = kQT * kD * 2;  // two 16 KB column halves of 128 rows
constexpr uint32_t kQHalf = 16384;
constexpr uint32_t kKHalf = 64 * kD * 2;    // 64 keys x 128 d: two 8 KB column halves
constexpr uint32_t kKCol = 8192;
constexpr uint32_t kVHalf = kBK * 64 * 2;   // 128 keys x 64 d
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = kQBytes;
constexpr uint32_t kOffV = kOffK + kStages * kKHalf;
constexpr uint32_t kSmemBytes = kOffV + kStages * kVHalf + 1024;
constexpr uint32_t kColO = kNS * 128;
static_assert(kColO + 128 <= 512, "TMEM columns");
constexpr float kRescaleThreshold = 8.f;    // log2 units: rescale O only when the max grows by > 2^8
constexpr float kFastSumLimit = 32768.f;    // a tile accepted without its row max sums to <= 2^15

struct PairCtl {
  uint64_t q_full;                          // leader: one arrival per softmax warp of both CTAs
  uint64_t k_full[kStages], v_full[kStages];  // this CTA's own copies (tx bytes)
  uint64_t k_peer[kStages], v_peer[kStages];  // leader: the peer's copies landed (relay)
  uint64_t k_free[kStages], v_free[kStages];  // MMA completions, both CTAs
  uint64_t s_full[kNS], p_full[kNS];        // s_full both CTAs; p_full leader, 8 warp arrivals
  uint64_t pv_done, o_full, drain;
  uint32_t tmem_base;
  int abort;
};

MOBA_DEV uint32_t bar(const uint64_t* b) { return smem_u32(b); }

MOBA_DEV void st_shared_v4(uint32_t a, uint32_t x, uint32_t y, uint32_t z, uint32_t w) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};\n" ::"r"(a), "r"(x), "r"(y), "r"(z), "r"(w) : "memory");
}

// OR of `v` over the 64 threads of named barrier `id` (the two warps of one
// TMEM lane quarter); also a barrier
MOBA_DEV bool pair_any(int id, bool v) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.or.pred q, %2, 64, p;\n"
      " selp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(id)
      : "memory");
  return r != 0;
}
MOBA_DEV void pair_sync(int id) { asm volatile("bar.sync %0, 64;\n" ::"r"(id) : "memory"); }

// HALVES = softmax warps per TMEM lane quarter: 1 (each warp takes all 128
// key columns of its 32 rows) or 2 (each takes 64 columns; the two warps of a
// quarter agree on every row's exponent base through a 64-thread named
// barrier, and one warp's TMEM loads and stores overlap the other's
// exponentials on the same SM sub-partition)
template <int HALVES>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(32 * (4 * HALVES + 2), 1) attn_pair_kernel(
    const __nv_bfloat16* __restrict__ q, const __grid_constant__ CUtensorMap tmK,
    const __grid_constant__ CUtensorMap tmV, const int32_t* __restrict__ sel,
    const int32_t* __restrict__ offsets, const int32_t* __restrict__ rows,
    const int32_t* __restrict__ tile_start, __nv_bfloat16* __restrict__ part_o,
    float* __restrict__ part_lse, int* __restrict__ status, Dims dm, int ch) {
  constexpr int kSmWarps = 4 * HALVES;
  constexpr int kProdWarp = kSmWarps, kMmaWarp = kSmWarps + 1;
  constexpr int kCols = kBK / HALVES;        // key columns of S per softmax warp
  constexpr int kOCols = kD / HALVES;        // columns of O per softmax warp
  constexpr int kRowBytes = kOCols * 2;      // bf16 bytes of a partial row per warp
  constexpr int kChunks = kRowBytes / 16;
  constexpr int kRowsPerSt = 32 / kChunks;   // rows per warp store instruction
  static_assert(kSmWarps * 32 * kRowBytes <= (int)kQBytes, "epilogue staging uses the Q buffer");
  extern __shared__ uint8_t smem_raw[];
  __shared__ PairCtl ctl;
  __shared__ float xchg[4][2][32];
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t rank = cluster_ctarank();
  const bool lead = rank == 0;

  // ---- work tile of the pair (both CTAs decode the same one)
  const int ngroups = dm.batch * dm.hkv * dm.n;
  const int tile = blockIdx.x >> 1;
  if (tile >= tile_start[ngroups]) return;
  int grp;
  {
    int lo = 0, hi = ngroups - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (tile_start[mid] <= tile) lo = mid; else hi = mid - 1;
    }
    grp = lo;
  }
  const int j = grp % dm.n, g = (grp / dm.n) % dm.hkv, b = grp / (dm.n * dm.hkv);
  const size_t goff = (size_t)ch * ngroups + grp;
  const int r0 = offsets[goff] + (tile - tile_start[grp]) * kRowsPerPair;
  const int cnt = min(kRowsPerPair, offsets[goff + 1] - r0);
  const int key0 = j * dm.B;
  const int nkt = (dm.B + kBK - 1) / kBK;
  const int KH = dm.topk - 1;
  const int t0 = ch * dm.chunk;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    mbar_init(bar(&ctl.q_full), 2 * kSmWarps);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(&ctl.k_full[s]), 1);
      mbar_init(bar(&ctl.v_full[s]), 1);
      mbar_init(bar(&ctl.k_peer[s]), 1);
      mbar_init(bar(&ctl.v_peer[s]), 1);
      mbar_init(bar(&ctl.k_free[s]), 1);
      mbar_init(bar(&ctl.v_free[s]), 1);
    }
    for (int x = 0; x < kNS; ++x) {
      mbar_init(bar(&ctl.s_full[x]), 1);
      mbar_init(bar(&ctl.p_full[x]), 2 * kSmWarps);
    }
    mbar_init(bar(&ctl.pv_done), 1);
    mbar_init(bar(&ctl.o_full), 1);
    mbar_init(bar(&ctl.drain), 1);
    ctl.abort = 0;
    fence_mbar_init();
  }
  if (warp == kProdWarp) {
    tmem_alloc_pair(smem_u32(&ctl.tmem_base), 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();   // the peer's barriers are initialised before anyone arrives on them
  tc_fence_after();
  const uint32_t tb = ctl.tmem_base;
  volatile int* abort_flag = &ctl.abort;

  if (warp < kSmWarps) {
    // ------------------------------------------------------------ softmax
    const int qd = warp & 3, hf = warp >> 2, pair = 1 + qd;
    const int rho = qd * 32 + lane;               // this CTA's row = TMEM lane
    const int row_i = (int)rank * kQT + rho;      // row of the pair's tile
    const bool valid = row_i < cnt;
    const int r = valid ? rows[r0 + row_i] : 0;
    const int h = r % dm.hq;
    const int t = (r / dm.hq) % dm.N;
    auto any_of = [&](bool v) -> bool {
      if constexpr (HALVES == 2) return pair_any(pair, v);
      else return __any_sync(0xffffffffu, v);
    };
    {
      // the quarter's 32 rows, two at a time (lanes 0-15 take the 16 chunks
      // of one row, lanes 16-31 those of the next), split between its warps
      const uint32_t qs = base + kOffQ;
      const int cc = lane & 15;
#pragma unroll
      for (int k2 = 0; k2 < 16 / HALVES; ++k2) {
        const int rl = hf * (32 / HALVES) + 2 * k2 + (lane >> 4);
        const int rs = __shfl_sync(0xffffffffu, r, rl);
        const bool vs = __shfl_sync(0xffffffffu, valid, rl);
        cp_async16(qs + (cc >> 3) * kQHalf + sw128_off(qd * 32 + rl, cc & 7), q + (size_t)rs * kD + cc * 8, vs);
      }
      cp_async_commit();
      cp_async_wait<0>();
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(bar(&ctl.q_full), 0));
    }
    const uint32_t lane_off = (uint32_t)(qd * 32) << 16;
    const uint32_t tO = tb + kColO + (uint32_t)(hf * kOCols) + lane_off;
    const float sl2 = dm.scale_log2;
    float m_used = -INFINITY, l = 0.f;
    bool fail = false;
    // this warp's key columns of S(i); keys outside block j set to -inf
    auto load_s = [&](uint32_t (&sr)[kCols], int i) {
      const uint32_t tS = tb + (uint32_t)(i % kNS) * 128u + (uint32_t)(hf * kCols) + lane_off;
#pragma unroll
      for (int c = 0; c < kCols; c += 32) tmem_ld32(tS + c, sr + c);
      tmem_wait_ld();
      const int vhi = dm.B - i * kBK - 1 - hf * kCols;
      if (vhi < kCols - 1) {
#pragma unroll
        for (int c = 0; c < kCols; ++c)
          if (c > vhi) sr[c] = __float_as_uint(-INFINITY);
      }
    };
    // p = 2^(s * scale * log2(e) - mb) as bf16 pairs; returns the fp32 sum of p
    auto exp_cols = [&](const uint32_t (&sr)[kCols], float mb, uint32_t (&pk)[kCols / 2]) -> float {
      const uint64_t sl2x2 = f2_pack(sl2, sl2), nmbx2 = f2_pack(-mb, -mb);
      uint64_t rs4[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
      for (int c = 0; c < kCols / 2; ++c) {
        const uint64_t x2 =
            f2_fma(f2_pack(__uint_as_float(sr[2 * c]), __uint_as_float(sr[2 * c + 1])), sl2x2, nmbx2);
        float x0, x1;
        f2_unpack(x2, x0, x1);
        const uint64_t p2 = f2_pack(ex2_approx(x0), ex2_approx(x1));
        rs4[c & 3] = f2_add(rs4[c & 3], p2);
        float p0, p1;
        f2_unpack(p2, p0, p1);
        pk[c] = pack_bf16x2(p0, p1);
      }
      float a0, a1;
      f2_unpack(f2_add(f2_add(rs4[0], rs4[1]), f2_add(rs4[2], rs4[3])), a0, a1);
      return a0 + a1;
    };
    const uint32_t p_full_lead = mapa_shared(bar(&ctl.p_full[0]), 0);   // + 8 x for buffer x
    for (int i = 0; i < nkt; ++i) {
      const int x = i % kNS;
      if (!fail) fail = !__all_sync(0xffffffffu, mbar_wait(bar(&ctl.s_full[x]), (i / kNS) & 1, abort_flag));
      uint32_t sr[kCols], pk[kCols / 2];
      float ts = 0.f;
      bool slowrow = true;
      if (!fail) {
        tc_fence_after();
        load_s(sr, i);
        // fast path: exponentials against the current base m_used, no row
        // max; taken back if any row's part sums above the limit (so no p can
        // exceed it) or has no base yet
        if (!__any_sync(0xffffffffu, m_used == -INFINITY)) {
          ts = exp_cols(sr, m_used, pk);
          slowrow = !(ts <= kFastSumLimit / HALVES);
        }
      }
      // one barrier of the quarter per tile: both warps have read S before
      // either writes P over it, and they agree on the slow path; a second
      // barrier, only when one is needed, tells a failure from a slow tile
      if (*abort_flag) fail = true;
      tc_fence_before();
      const bool slow = any_of(fail || slowrow);
      if (slow && any_of(fail)) {
        fail = true;
        break;
      }
      tc_fence_after();
      if (slow) {
        load_s(sr, i);
        float mx4[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) mx4[u] = fmaxf(__uint_as_float(sr[2 * u]), __uint_as_float(sr[2 * u + 1]));
#pragma unroll
        for (int c = 8; c < kCols; c += 8)
#pragma unroll
          for (int u = 0; u < 4; ++u)
            mx4[u] = max3(mx4[u], __uint_as_float(sr[c + 2 * u]), __uint_as_float(sr[c + 2 * u + 1]));
        float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
        if constexpr (HALVES == 2) {
          xchg[qd][hf][lane] = mx;
          pair_sync(pair);
          mx = fmaxf(xchg[qd][0][lane], xchg[qd][1][lane]);
        }
        const float mxs = mx * sl2;
        const bool need = mxs > m_used + kRescaleThreshold;
        if (i > 0 && __any_sync(0xffffffffu, need)) {
          // O may only be rescaled once PV(i-1) has completed (S(i) complete
          // implies PV(i-2) complete, so the parity names PV(i-1)); on a
          // timeout the next tile's barrier of the quarter sees the abort
          if (!__all_sync(0xffffffffu, mbar_wait(bar(&ctl.pv_done), (i - 1) & 1, abort_flag))) {
            fail = true;
            continue;
          }
          tc_fence_after();
          const float f = need ? exp2f(m_used - mxs) : 1.f;
#pragma unroll
          for (int cc = 0; cc < kOCols; cc += 32) {
            uint32_t o[32];
            tmem_ld32(tO + cc, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
            tmem_st32(tO + cc, o);
          }
          tmem_wait_st();
        }
        if (need) {
          l *= exp2f(m_used - mxs);
          m_used = mxs;
        }
        // a row with no valid key yet keeps m_used = -inf: use 0 as the base (p = 0)
        ts = exp_cols(sr, m_used == -INFINITY ? 0.f : m_used, pk);
      }
      l += ts;
      const uint32_t tP = tb + (uint32_t)x * 128u + (uint32_t)(hf * kCols / 2) + lane_off;
#pragma unroll
      for (int c = 0; c < kCols / 2; c += 32) tmem_st32(tP + c, pk + c);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(p_full_lead + 8u * (uint32_t)x);
    }
    // ---- epilogue: O / l as bf16 and lse, after the last PV
    if (!fail) fail = !__all_sync(0xffffffffu, mbar_wait(bar(&ctl.o_full), 0, abort_flag));
    if (*abort_flag) fail = true;
    tc_fence_before();
    // both warps of the quarter have left the tile loop and agree
    const bool bad = any_of(fail);
    tc_fence_after();
    if (!bad) {
      float L = l;
      if constexpr (HALVES == 2) {
        xchg[qd][hf][lane] = l;
        pair_sync(pair);
        L = xchg[qd][0][lane] + xchg[qd][1][lane];
      }
      const float inv = 1.f / L;
      size_t pidx = 0;
      if (valid) {
        const int slot = slot_of(sel + (size_t)r * dm.topk, dm.topk, j);
        pidx = (size_t)((b * dm.chunk + (t - t0)) * dm.hq + h) * KH + slot;
      }
      // every MMA of the pair has completed: the warp stages its rows' part
      // in the Q buffer (chunk c of row rr at rr * kRowBytes + ((c ^ (rr %
      // kChunks)) << 4): no bank conflicts either way) and stores kRowsPerSt
      // whole row parts per instruction
      const uint32_t stg = base + kOffQ + (uint32_t)warp * (32u * kRowBytes);
#pragma unroll
      for (int cc = 0; cc < kOCols; cc += 32) {
        uint32_t o[32];
        tmem_ld32(tO + cc, o);
        tmem_wait_ld();
#pragma unroll
        for (int e8 = 0; e8 < 4; ++e8) {
          const int c = cc / 8 + e8;
          st_shared_v4(stg + lane * kRowBytes + ((c ^ (lane % kChunks)) << 4),
                       pack_bf16x2(__uint_as_float(o[8 * e8 + 0]) * inv, __uint_as_float(o[8 * e8 + 1]) * inv),
                       pack_bf16x2(__uint_as_float(o[8 * e8 + 2]) * inv, __uint_as_float(o[8 * e8 + 3]) * inv),
                       pack_bf16x2(__uint_as_float(o[8 * e8 + 4]) * inv, __uint_as_float(o[8 * e8 + 5]) * inv),
                       pack_bf16x2(__uint_as_float(o[8 * e8 + 6]) * inv, __uint_as_float(o[8 * e8 + 7]) * inv));
        }
      }
      __syncwarp();
      const int cq = lane % kChunks;
#pragma unroll
      for (int k2 = 0; k2 < 32 / kRowsPerSt; ++k2) {
        const int rl = kRowsPerSt * k2 + lane / kChunks;
        const long long rd = __shfl_sync(0xffffffffu, (long long)pidx, rl);
        const bool vd = __shfl_sync(0xffffffffu, valid, rl);
        uint32_t x0, x1, x2, x3;
        asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];\n"
                     : "=r"(x0), "=r"(x1), "=r"(x2), "=r"(x3)
                     : "r"(stg + rl * kRowBytes + ((cq ^ (rl % kChunks)) << 4)));
        if (vd) *reinterpret_cast<uint4*>(part_o + rd * kD + hf * kOCols + cq * 8) = make_uint4(x0, x1, x2, x3);
      }
      if (valid && hf == 0) part_lse[pidx] = m_used + log2f(L);
    }
  } else if (warp == kProdWarp) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      const int y0 = b * dm.N + key0;
      const int x0 = g * kD;
      int issued_k = 0, issued_v = 0;
      for (int i = 0; i < nkt; ++i) {
        const int s = i % kStages, u = i / kStages;
        const uint32_t ks = base + kOffK + s * kKHalf, vs = base + kOffV + s * kVHalf;
        if (i >= kStages && !mbar_wait(bar(&ctl.k_free[s]), (u - 1) & 1, abort_flag)) break;
        mbar_arrive_expect_tx(bar(&ctl.k_full[s]), kKHalf);
        // keys [64 rank, +64) of the tile, all d columns
        tma_load_2d(ks, &tmK, x0, y0 + i * kBK + (int)rank * 64, bar(&ctl.k_full[s]));
        tma_load_2d(ks + kKCol, &tmK, x0 + 64, y0 + i * kBK + (int)rank * 64, bar(&ctl.k_full[s]));
        issued_k = i + 1;
        if (i >= kStages && !mbar_wait(bar(&ctl.v_free[s]), (u - 1) & 1, abort_flag)) break;
        mbar_arrive_expect_tx(bar(&ctl.v_full[s]), kVHalf);
        // all keys of the tile, d columns [64 rank, +64)
        tma_load_2d(vs, &tmV, x0 + (int)rank * 64, y0 + i * kBK, bar(&ctl.v_full[s]));
        issued_v = i + 1;
      }
      if (*abort_flag) {
        // let the copies this thread issued land before the CTA exits
        int never = 0;
        for (int i = (issued_k > kStages ? issued_k - kStages : 0); i < issued_k; ++i)
          mbar_wait(bar(&ctl.k_full[i % kStages]), (i / kStages) & 1, &never);
        for (int i = (issued_v > kStages ? issued_v - kStages : 0); i < issued_v; ++i)
          mbar_wait(bar(&ctl.v_full[i % kStages]), (i / kStages) & 1, &never);
      }
    }
  } else if (warp == kMmaWarp && lane == 0) {
    if (!lead) {
      // ---------------------------------------------------------- relay
      const uint32_t kp = mapa_shared(bar(&ctl.k_peer[0]), 0), vp = mapa_shared(bar(&ctl.v_peer[0]), 0);
      for (int i = 0; i < nkt; ++i) {
        const int s = i % kStages, u = i / kStages;
        if (!mbar_wait(bar(&ctl.k_full[s]), u & 1, abort_flag)) break;
        mbar_arrive_cluster(kp + 8u * s);
        if (!mbar_wait(bar(&ctl.v_full[s]), u & 1, abort_flag)) break;
        mbar_arrive_cluster(vp + 8u * s);
      }
    } else {
      // ---------------------------------------------------------- MMA issuer
      const uint32_t idS = idesc_bf16(2 * kQT, kBK, false);
      const uint32_t idO = idesc_bf16(2 * kQT, kD, true);
      const uint32_t hi = sdesc_hi(1024);
      const uint32_t loQ = sdesc_lo(base + kOffQ, 16), loK = sdesc_lo(base + kOffK, 16),
                     loV = sdesc_lo(base + kOffV, kVHalf);
      auto ready = [&](const uint64_t* own, const uint64_t* peer, int n) -> bool {
        const int s = n % kStages;
        const uint32_t ph = (n / kStages) & 1;
        return mbar_wait(bar(&own[s]), ph, abort_flag) && mbar_wait(bar(&peer[s]), ph, abort_flag);
      };
      auto issue_s = [&](int n) {
        const uint32_t ka = loK + (uint32_t)(n % kStages) * (kKHalf >> 4);
        const uint32_t d = tb + (uint32_t)(n % kNS) * 128u;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t offa = ((kk >> 2) * kQHalf + (kk & 3) * 32) >> 4;
          const uint32_t offb = ((kk >> 2) * kKCol + (kk & 3) * 32) >> 4;
          mma_ss_pair(d, sdesc_join(loQ + offa, hi), sdesc_join(ka + offb, hi), idS, kk > 0);
        }
      };
      auto issue_pv = [&](int i) {
        const uint32_t va = loV + (uint32_t)(i % kStages) * (kVHalf >> 4);
        const uint32_t a = tb + (uint32_t)(i % kNS) * 128u;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts_pair(tb + kColO, a + kk * 8, sdesc_join(va + ((kk * 2048) >> 4), hi), idO,
                      (i > 0 || kk > 0) ? 1u : 0u);
      };
      bool ok = mbar_wait(bar(&ctl.q_full), 0, abort_flag);
      for (int n = 0; n < kNS && n < nkt && ok; ++n) {
        if (!(ok = ready(ctl.k_full, ctl.k_peer, n))) break;
        tc_fence_after();
        issue_s(n);
        mma_commit_pair_both(bar(&ctl.s_full[n % kNS]));
        mma_commit_pair_both(bar(&ctl.k_free[n % kStages]));
      }
      for (int i = 0; i < nkt && ok; ++i) {
        ok = mbar_wait(bar(&ctl.p_full[i % kNS]), (i / kNS) & 1, abort_flag) &&
             ready(ctl.v_full, ctl.v_peer, i);
        if (!ok) break;
        tc_fence_after();
        issue_pv(i);
        mma_commit_pair_both(bar(&ctl.pv_done));
        mma_commit_pair_both(bar(&ctl.v_free[i % kStages]));
        // S(i + 2) into the buffer PV(i) has just read P(i) from (tcgen05
        // operations of one thread execute in order)
        const int n = i + kNS;
        if (n < nkt) {
          if (!(ok = ready(ctl.k_full, ctl.k_peer, n))) break;
          tc_fence_after();
          issue_s(n);
          mma_commit_pair_both(bar(&ctl.s_full[n % kNS]));
          mma_commit_pair_both(bar(&ctl.k_free[n % kStages]));
        }
      }
      if (ok) {
        mma_commit_pair_both(bar(&ctl.o_full));
      } else {
        // drain every MMA this thread issued before either CTA frees TMEM
        int never = 0;
        mma_commit_pair(bar(&ctl.drain));
        mbar_wait(bar(&ctl.drain), 0, &never);
      }
    }
  }

  __syncwarp();
  tc_fence_before();
  cluster_sync_all();   // neither CTA frees TMEM or leaves while the pair's MMAs may read it
  tc_fence_after();
  if (warp == kProdWarp) tmem_dealloc_pair(tb, 512);
  if (tid == 0 && ctl.abort) atomicExch(status, (int)MOBA_ERR_TIMEOUT);
}

// 2-D map over a [batch*N, hkv*d] bf16 tensor, 64 rows x 64 columns per box,
// 128-byte swizzle: half of a 128-key tile, one 64-column half of d
bool make_khalf_map(CUtensorMap* map, const void* base, const Dims& dm) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {(cuuint64_t)dm.hkv * kD, (cuuint64_t)dm.batch * dm.N};
  cuuint64_t strides[1] = {(cuuint64_t)dm.hkv * kD * 2};
  cuuint32_t box[2] = {64, kBK / 2};
  cuuint32_t es[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

// MOBA_HIST_KERNEL=pair selects this kernel instead of the single-CTA one
bool attn_hist_pair_enabled() {
  const char* e = getenv("MOBA_HIST_KERNEL");
  return e != nullptr && strcmp(e, "pair") == 0;
}

cudaError_t launch_attn_pair_hist(const Dims& dm, const void* q, const void* k, const void* v,
                                  const int32_t* sel, const int32_t* offsets, const int32_t* rows,
                                  const AttnWs& ws, int ch, int64_t grid, cudaStream_t stream) {
  CUtensorMap mk, mv;
  if (!make_khalf_map(&mk, k, dm) || !make_kv_map(&mv, v, dm)) return cudaErrorInvalidValue;
  // MOBA_PAIR_SOFTMAX_WARPS=4 selects one softmax warp per TMEM lane quarter
  const char* e4 = getenv("MOBA_PAIR_SOFTMAX_WARPS");
  const bool one = e4 != nullptr && strcmp(e4, "4") == 0;
  auto kern = one ? attn_pair_kernel<1> : attn_pair_kernel<2>;
  const int threads = one ? 32 * 6 : 32 * 10;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  kern<<<2 * grid, threads, kSmemBytes, stream>>>(
      (const __nv_bfloat16*)q, mk, mv, sel, offsets, rows, ws.tile_start,
      reinterpret_cast<__nv_bfloat16*>(ws.part_o), ws.part_lse, ws.status, dm, ch);
  return cudaGetLastError();
}

}  // namespace moba
