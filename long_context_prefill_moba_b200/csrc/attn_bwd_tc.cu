// Backward of the attention step on 5th-generation tensor cores (bf16,
// head_dim 128): the gradients of Softmax(q K[I]^T) V[I] ("MoBA: Mixture of
// Block Attention for Long-Context LLMs", paper-graph summary §3 "The Core MoBA
// Attention Equation", "Causality Enforcement"; Implementation, Algorithm 1
// Steps 2-3 for the grouping of query rows by the block they attend) with the
// gate's selection held fixed.  With the forward's lse L_r and
// D_r = <dout_r, out_r>, for a tile of rows against a tile of keys:
//   S = Q K^T, dP = dO V^T, P = exp(scale S - L), dS = P (dP - D),
//   dV += P^T dO, dK += scale dS^T Q, dQ += scale dS K.
// P needs no row max (the forward's L normalises it), so every element of a
// tile is independent and the softmax warps split the key columns freely.
//
// bwd_kv_tc_kernel: one CTA per 128-key tile of one (b, kv head g, block j).
//   dK and dV accumulate in TMEM over every query row that attends the tile:
//   the rows the gate routed to block j in every pass (gathered through
//   `rows`) and the rows of block j itself at or after the tile (causal, all G
//   query heads).  Per 128-row tile: S^T = K Q^T and dP^T = V dO^T (SS MMAs,
//   a key per TMEM lane), P^T and dS^T as bf16 back into TMEM, dV += P^T dO
//   and dK += dS^T Q (TS MMAs, dO and Q read MN-major); the next row tile's
//   q/dout rows load into the second stage meanwhile.  Each key's dk, dv is
//   written once.
// bwd_q_tc_kernel: one CTA per 128-row tile, like the forward: kHist takes up
//   to 128 rows of one gate group against all keys of block j, kCur 128
//   tokens of one head against its own block (causal).  Per 128-key tile: S and
//   dP, dS as bf16 into TMEM, dQ += dS K (TS MMA, K read MN-major).  The row
//   tile's dQ is added into an fp32 accumulator with one vector reduction per
//   row and 16 bytes (a row receives one per selected block).
//
// Every mbarrier wait is bounded (2 s); on expiry the CTA drains what it
// issued, frees TMEM and writes MOBA_ERR_TIMEOUT to the status word.
#include <cudaTypedefs.h>

#include "launch.h"
#include "sm100.cuh"

namespace moba {

bool make_kv_map(CUtensorMap* map, const void* base, const Dims& dm);

namespace {

using namespace sm100;

constexpr int kD = 128;
constexpr int kT = 128;                     // rows or keys per tile
constexpr uint32_t kTile = kT * kD * 2;     // 32 KB: two 16 KB column halves, 128-byte swizzle
constexpr uint32_t kHalf = 16384;
constexpr int kSoftmaxWarps = 8;

MOBA_DEV uint32_t bar(const uint64_t* b) { return smem_u32(b); }

MOBA_DEV void red_add_v4(float* dst, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};\n" ::"l"(dst), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}

// ============================================================================ dK, dV
// Transposed products: S^T = K Q^T and dP^T = V dO^T put a key on every TMEM
// lane, so P^T and dS^T stay in TMEM as bf16 and feed dV += P^T dO and
// dK += dS^T Q as TS MMAs.  Row tiles are 64 query rows:
//   TMEM   two stages of S^T | dP^T (64 columns each) and the dV, dK
//          accumulators (128 columns each): 512 columns;
//   SMEM   the K and V tiles and four stages of q | dout row tiles (16 KB each).
// The MMA issuer runs S^T, dP^T of row tile i and then dV, dK of tile i - 1,
// so the elementwise warps work on one tile while the tensor core computes
// the next.  Four gather warps copy the row tiles (cp.async) with their lse,
// D and causal limit: warp w owns shared-memory stage w and the tiles
// i = w mod 4, and publishes each tile as soon as its own copies have landed,
// so four tiles are in flight.
constexpr int kR = 64;                          // query rows per row tile
constexpr int kStages = 4;                      // q | dout row-tile stages
constexpr uint32_t kRHalf = kR * 128;           // 8 KB: one 64-column half of a row tile
constexpr uint32_t kRTile = 2 * kRHalf;         // 16 KB: q (or dout) of a row tile
constexpr uint32_t kRStage = 2 * kRTile;        // q then dout
constexpr int kGatherWarps = 4;
constexpr int kKvWarps = kSoftmaxWarps + kGatherWarps + 1;   // elementwise, gather, MMA issuer
constexpr int kKvThreads = kKvWarps * 32;
constexpr int kGatherWarp = kSoftmaxWarps;                    // first gather warp
constexpr int kMmaWarp = kSoftmaxWarps + kGatherWarps;
static_assert(kGatherWarps == kStages, "each gather warp owns one row-tile stage");
constexpr uint32_t kKvOffK = 0, kKvOffV = kTile, kKvOffQ = 2 * kTile;   // stage x at kKvOffQ + x kRStage
constexpr uint32_t kKvSmem = 2 * kTile + kStages * kRStage + 1024;

constexpr int kMaxPassPrefix = 256;    // passes whose row-tile prefix is kept in shared memory

struct KvCtl {
  uint64_t kv_full, q_full[kStages], q_free[kStages], s_full[2], p_full[2], mm_done, drain;
  int pass_tiles[kMaxPassPrefix + 1];   // routed row tiles of passes [0, p), this CTA's group
  int pass_r0[kMaxPassPrefix];          // first routed row of pass p's group
  int pass_r1[kMaxPassPrefix];          // end of pass p's group
  uint32_t tmem_base;
  int abort;
  float lse2[kStages][kR];   // per row of a stage: forward lse in log2 units (+inf: no row)
  float dlt[kStages][kR];    // D = <dout, out>
  int tmax[kStages][kR];     // last key the row may attend (its token for the block's own rows)
};

// the query rows of row tile i of this key tile: the gate's groups of block j
// over all passes, then block j's own tokens from the tile on, per query head
struct RowTile {
  bool own;          // block j's own rows (causal) or routed rows
  int r0, cnt;       // routed: rows[r0 .. r0 + cnt)
  int t0, h;         // own: tokens t0 .. t0 + kR - 1 of head h
};

MOBA_DEV int kv_tiles(const int32_t* offsets, const Dims& dm, int b, int g, int j, int key0, int key_end,
                      int& hist_tiles) {
  const int64_t ngroups = (int64_t)dm.batch * dm.hkv * dm.n;
  hist_tiles = 0;
  for (int ch = 0; ch < dm.nchunks; ++ch) {
    const int64_t gi = ch * ngroups + ((int64_t)b * dm.hkv + g) * dm.n + j;
    hist_tiles += (offsets[gi + 1] - offsets[gi] + kR - 1) / kR;
  }
  return hist_tiles + (key_end - key0 + kR - 1) / kR * dm.G;
}

MOBA_DEV RowTile kv_row_tile(int i, int hist_tiles, const int32_t* offsets, const Dims& dm, int b, int g, int j,
                             int key0, const int* pass_tiles, const int* pass_r0, const int* pass_r1) {
  RowTile rt{};
  if (i < hist_tiles && pass_tiles != nullptr) {
    // the pass holding tile i: largest p with pass_tiles[p] <= i (all in shared memory)
    int lo = 0, hi = dm.nchunks - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (pass_tiles[mid] <= i) lo = mid; else hi = mid - 1;
    }
    const int left = i - pass_tiles[lo];
    rt.own = false;
    rt.r0 = pass_r0[lo] + left * kR;
    rt.cnt = min(kR, pass_r1[lo] - rt.r0);
    return rt;
  }
  if (i < hist_tiles) {
    const int64_t ngroups = (int64_t)dm.batch * dm.hkv * dm.n;
    int left = i;
    for (int ch = 0; ch < dm.nchunks; ++ch) {
      const int64_t gi = ch * ngroups + ((int64_t)b * dm.hkv + g) * dm.n + j;
      const int r0 = offsets[gi], n = offsets[gi + 1] - r0;
      const int nt = (n + kR - 1) / kR;
      if (left < nt) {
        rt.own = false;
        rt.r0 = r0 + left * kR;
        rt.cnt = min(kR, n - left * kR);
        return rt;
      }
      left -= nt;
    }
  }
  const int k = i - hist_tiles;
  rt.own = true;
  rt.t0 = key0 + (k / dm.G) * kR;
  rt.h = g * dm.G + k % dm.G;
  return rt;
}

// AND of `v` over the 256 elementwise threads (named barrier 1)
MOBA_DEV bool elementwise_all(bool v) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.and.pred q, 1, 256, p;\n"
      " selp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(r)
      : "r"((uint32_t)v)
      : "memory");
  return r != 0;
}

__global__ void __launch_bounds__(kKvThreads, 1) bwd_kv_tc_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
    const __nv_bfloat16* __restrict__ v, const __nv_bfloat16* __restrict__ dout,
    const float* __restrict__ lse, const float* __restrict__ delta, const int32_t* __restrict__ offsets,
    const int32_t* __restrict__ rows, __nv_bfloat16* __restrict__ dk, __nv_bfloat16* __restrict__ dv,
    int* __restrict__ status, Dims dm) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ KvCtl ctl;
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const int tiles_per_block = (dm.B + kT - 1) / kT;
  int idx = blockIdx.x;
  const int kt = idx % tiles_per_block; idx /= tiles_per_block;
  const int j = idx % dm.n; idx /= dm.n;
  const int g = idx % dm.hkv;
  const int b = idx / dm.hkv;
  const int key0 = j * dm.B + kt * kT;
  const int key_end = min(dm.N, (j + 1) * dm.B);
  if (b >= dm.batch || key0 >= key_end) return;
  int hist_tiles;
  const int ntiles = kv_tiles(offsets, dm, b, g, j, key0, key_end, hist_tiles);   // >= G: own rows

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool prefix = dm.nchunks <= kMaxPassPrefix;
  if (prefix && tid == 0) {
    const int64_t ngroups = (int64_t)dm.batch * dm.hkv * dm.n;
    int acc = 0;
    for (int ch = 0; ch < dm.nchunks; ++ch) {
      const int64_t gi = ch * ngroups + ((int64_t)b * dm.hkv + g) * dm.n + j;
      ctl.pass_tiles[ch] = acc;
      ctl.pass_r0[ch] = offsets[gi];
      ctl.pass_r1[ch] = offsets[gi + 1];
      acc += (offsets[gi + 1] - offsets[gi] + kR - 1) / kR;
    }
    ctl.pass_tiles[dm.nchunks] = acc;
  }
  if (tid == 0) {
    mbar_init(bar(&ctl.kv_full), kGatherWarps);
    for (int x = 0; x < kStages; ++x) {
      mbar_init(bar(&ctl.q_full[x]), 1);
      mbar_init(bar(&ctl.q_free[x]), 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(bar(&ctl.s_full[x]), 1);
      mbar_init(bar(&ctl.p_full[x]), kSoftmaxWarps);
    }
    mbar_init(bar(&ctl.mm_done), 1);
    mbar_init(bar(&ctl.drain), 1);
    ctl.abort = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(&ctl.tmem_base), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const int* pt = prefix ? ctl.pass_tiles : nullptr;
  const int* pr = prefix ? ctl.pass_r0 : nullptr;
  const int* pe = prefix ? ctl.pass_r1 : nullptr;
  const uint32_t tb = ctl.tmem_base;
  volatile int* abort_flag = &ctl.abort;

  if (warp < kSoftmaxWarps) {
    // ------------------------------------------------------------ elementwise
    const int qd = warp & 3, hf = warp >> 2;
    const int rho = qd * 32 + lane;           // TMEM lane: a key of S^T, dP^T, dK, dV
    const uint32_t lane_off = (uint32_t)(qd * 32) << 16;
    const float sl2 = dm.scale_log2;
    const int u = key0 + rho;                  // this thread's key
    const bool key_ok = u < key_end;
    bool ok = true;
    for (int i = 0; i < ntiles && ok; ++i) {
      const int x = i & 1, st = i % kStages;
      ok = elementwise_all(mbar_wait(bar(&ctl.s_full[x]), (i >> 1) & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      // this warp's 32 rows of the tile: columns [32 hf, 32 hf + 32) of S^T_x and dP^T_x
      const uint32_t cS = 64u * x + 32u * hf, cP = 128u + 64u * x + 32u * hf;
      uint32_t sr[32], dr[32];
      tmem_ld32(tb + cS + lane_off, sr);
      tmem_ld32(tb + cP + lane_off, dr);
      tmem_wait_ld();
      uint32_t pp[16], ps[16];
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const int ra = 32 * hf + 2 * c, rb = ra + 1;   // rows of this column pair
        float p0 = ex2_approx(__uint_as_float(sr[2 * c]) * sl2 - ctl.lse2[st][ra]);
        float p1 = ex2_approx(__uint_as_float(sr[2 * c + 1]) * sl2 - ctl.lse2[st][rb]);
        p0 = (key_ok && u <= ctl.tmax[st][ra]) ? p0 : 0.f;
        p1 = (key_ok && u <= ctl.tmax[st][rb]) ? p1 : 0.f;
        pp[c] = pack_bf16x2(p0, p1);
        ps[c] = pack_bf16x2(p0 * (__uint_as_float(dr[2 * c]) - ctl.dlt[st][ra]),
                            p1 * (__uint_as_float(dr[2 * c + 1]) - ctl.dlt[st][rb]));
      }
      // P^T and dS^T over the first half of this warp's own columns (already read)
      tmem_st16(tb + cS + lane_off, pp);
      tmem_st16(tb + cP + lane_off, ps);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(&ctl.p_full[x]));
    }
    if (ok) ok = elementwise_all(mbar_wait(bar(&ctl.mm_done), 0, abort_flag));
    if (ok) {
      // dK, dV rows (lanes = keys) of this warp's 64 columns
      tc_fence_after();
      const float scale = sl2 / kLog2e;
      const size_t kr = ((size_t)b * dm.N + u) * dm.hkv + g;
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        uint32_t gvv[32], gkk[32];
        tmem_ld32(tb + 256u + 64u * hf + 32u * cc + lane_off, gvv);
        tmem_ld32(tb + 384u + 64u * hf + 32u * cc + lane_off, gkk);
        tmem_wait_ld();
        if (key_ok) {
          uint4* dvp = reinterpret_cast<uint4*>(dv + kr * kD + 64 * hf + 32 * cc);
          uint4* dkp = reinterpret_cast<uint4*>(dk + kr * kD + 64 * hf + 32 * cc);
#pragma unroll
          for (int e8 = 0; e8 < 4; ++e8) {
            dvp[e8] = make_uint4(
                pack_bf16x2(__uint_as_float(gvv[8 * e8 + 0]), __uint_as_float(gvv[8 * e8 + 1])),
                pack_bf16x2(__uint_as_float(gvv[8 * e8 + 2]), __uint_as_float(gvv[8 * e8 + 3])),
                pack_bf16x2(__uint_as_float(gvv[8 * e8 + 4]), __uint_as_float(gvv[8 * e8 + 5])),
                pack_bf16x2(__uint_as_float(gvv[8 * e8 + 6]), __uint_as_float(gvv[8 * e8 + 7])));
            dkp[e8] = make_uint4(
                pack_bf16x2(__uint_as_float(gkk[8 * e8 + 0]) * scale, __uint_as_float(gkk[8 * e8 + 1]) * scale),
                pack_bf16x2(__uint_as_float(gkk[8 * e8 + 2]) * scale, __uint_as_float(gkk[8 * e8 + 3]) * scale),
                pack_bf16x2(__uint_as_float(gkk[8 * e8 + 4]) * scale, __uint_as_float(gkk[8 * e8 + 5]) * scale),
                pack_bf16x2(__uint_as_float(gkk[8 * e8 + 6]) * scale, __uint_as_float(gkk[8 * e8 + 7]) * scale));
          }
        }
      }
    }
  } else if (warp < kMmaWarp) {
    // ------------------------------------------------------------ gather
    const int gw = warp - kGatherWarp;
    {
      // K and V of the tile: this warp's 32 keys, two per copy instruction
      // (lanes 0-15 the 16 chunks of one key's row, lanes 16-31 the next's)
      const int cc = lane & 15;
#pragma unroll
      for (int k2 = 0; k2 < 16; ++k2) {
        const int key = 32 * gw + 2 * k2 + (lane >> 4);
        const bool kok = key0 + key < key_end;
        const size_t kr = ((size_t)b * dm.N + (kok ? key0 + key : 0)) * dm.hkv + g;
        const uint32_t off = (cc >> 3) * kHalf + sw128_off(key, cc & 7);
        cp_async16(base + kKvOffK + off, k + kr * kD + cc * 8, kok);
        cp_async16(base + kKvOffV + off, v + kr * kD + cc * 8, kok);
      }
      cp_async_commit();
      cp_async_wait<0>();
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(&ctl.kv_full));
    }
    // Row tiles i = gw, gw + 4, ... into stage gw.  Lane l holds rows l and
    // l + 32 of the tile: id, lse, D and causal limit.  The row ids of the
    // warp's next tile (a read of `rows`) load while this tile is copied; each
    // copy instruction reads two whole 256-byte rows (lanes 0-15 one row's 16
    // chunks, lanes 16-31 the next row's).
    const int cc = lane & 15;
    struct RowOf {
      int r, t, h, tmax;
      bool valid;
    };
    auto row_of = [&](int i, int rr) -> RowOf {
      RowOf m{0, 0, 0, 0x7fffffff, false};
      if (i >= ntiles) return m;
      const RowTile rt = kv_row_tile(i, hist_tiles, offsets, dm, b, g, j, key0, pt, pr, pe);
      if (rt.own) {
        m.t = rt.t0 + rr;
        m.h = rt.h;
        m.valid = m.t < key_end;
        m.r = m.valid ? (b * dm.N + m.t) * dm.hq + m.h : 0;
        m.tmax = m.t;
      } else {
        m.valid = rr < rt.cnt;
        m.r = m.valid ? rows[rt.r0 + rr] : 0;   // t and h follow from r once it has arrived
        m.t = -1;
      }
      return m;
    };
    // lse (log2 units) and D of a row; +inf / 0 for no row
    auto scal_of = [&](RowOf& m, float& lse2, float& dl) {
      lse2 = INFINITY;
      dl = 0.f;
      if (!m.valid) return;
      if (m.t < 0) {
        m.h = m.r % dm.hq;
        m.t = (m.r / dm.hq) % dm.N;
      }
      lse2 = lse[((size_t)b * dm.hq + m.h) * dm.N + m.t] * kLog2e;
      dl = delta[m.r];
    };
    const uint32_t sq = base + kKvOffQ + (uint32_t)gw * kRStage, sdo = sq + kRTile;
    RowOf ra = row_of(gw, lane), rb = row_of(gw, lane + 32);
    bool ok = true;
    for (int i = gw, use = 0; i < ntiles && ok; i += kStages, ++use) {
      // the stage held this warp's previous tile: free once its dV, dK MMAs completed
      if (use >= 1) ok = __all_sync(0xffffffffu, mbar_wait(bar(&ctl.q_free[gw]), (use - 1) & 1, abort_flag));
      if (!ok) break;
      float la, da, lb, db;
      scal_of(ra, la, da);
      scal_of(rb, lb, db);
      const RowOf na = row_of(i + kStages, lane), nb = row_of(i + kStages, lane + 32);
#pragma unroll
      for (int k2 = 0; k2 < 32; ++k2) {
        const int rl = 2 * k2 + (lane >> 4);     // row of the tile; its data sit in lane rl & 31
        const int rsa = __shfl_sync(0xffffffffu, ra.r, rl & 31), rsb = __shfl_sync(0xffffffffu, rb.r, rl & 31);
        const bool vsa = __shfl_sync(0xffffffffu, ra.valid, rl & 31),
                   vsb = __shfl_sync(0xffffffffu, rb.valid, rl & 31);
        const int rs = rl < 32 ? rsa : rsb;
        const bool vs = rl < 32 ? vsa : vsb;
        const uint32_t off = (cc >> 3) * kRHalf + sw128_off(rl, cc & 7);
        cp_async16(sq + off, q + (size_t)rs * kD + cc * 8, vs);
        cp_async16(sdo + off, dout + (size_t)rs * kD + cc * 8, vs);
      }
      ctl.lse2[gw][lane] = la;
      ctl.dlt[gw][lane] = da;
      ctl.tmax[gw][lane] = ra.tmax;
      ctl.lse2[gw][lane + 32] = lb;
      ctl.dlt[gw][lane + 32] = db;
      ctl.tmax[gw][lane + 32] = rb.tmax;
      cp_async_commit();
      cp_async_wait<0>();
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(&ctl.q_full[gw]));
      ra = na;
      rb = nb;
    }
    cp_async_wait<0>();
  } else if (lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t idS = idesc_bf16(128, kR, false);     // A (K, V tile), B (q, dout rows) K-major
    const uint32_t idG = idesc_bf16(128, kD, true);      // A from TMEM, B (q, dout rows) MN-major
    const uint32_t hi = sdesc_hi(1024);
    const uint32_t loK = sdesc_lo(base + kKvOffK, 16), loV = sdesc_lo(base + kKvOffV, 16);
    // dV += P^T dO and dK += dS^T Q of row tile i (TMEM stage i & 1, smem stage i % kStages):
    // K runs over its 64 rows (rows 0-31 in columns 0-15 of P^T / dS^T, rows 32-63 in 32-47)
    auto issue_grad = [&](int i) {
      const int x = i & 1;
      const uint32_t sq = base + kKvOffQ + (uint32_t)(i % kStages) * kRStage, sdo = sq + kRTile;
      const uint32_t mnQ = sdesc_lo(sq, kRHalf), mnDO = sdesc_lo(sdo, kRHalf);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint32_t a = 64u * x + (kk < 2 ? kk * 8u : 32u + (kk - 2) * 8u);
        mma_ts(tb + 256u, tb + a, sdesc_join(mnDO + ((kk * 2048) >> 4), hi), idG, (i > 0 || kk > 0) ? 1u : 0u);
      }
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint32_t a = 128u + 64u * x + (kk < 2 ? kk * 8u : 32u + (kk - 2) * 8u);
        mma_ts(tb + 384u, tb + a, sdesc_join(mnQ + ((kk * 2048) >> 4), hi), idG, (i > 0 || kk > 0) ? 1u : 0u);
      }
      mma_commit(bar(&ctl.q_free[i % kStages]));
    };
    bool ok = mbar_wait(bar(&ctl.kv_full), 0, abort_flag);
    for (int i = 0; i < ntiles && ok; ++i) {
      const int x = i & 1, st = i % kStages;
      const uint32_t sq = base + kKvOffQ + (uint32_t)st * kRStage, sdo = sq + kRTile;
      const uint32_t loQ = sdesc_lo(sq, 16), loDO = sdesc_lo(sdo, 16);
      if (!(ok = mbar_wait(bar(&ctl.q_full[st]), (i / kStages) & 1, abort_flag))) break;
      tc_fence_after();
      // S^T_x, dP^T_x: stage x last held tile i - 2, whose dV, dK were issued before
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t offA = ((kk >> 2) * kHalf + (kk & 3) * 32) >> 4;
        const uint32_t offB = ((kk >> 2) * kRHalf + (kk & 3) * 32) >> 4;
        mma_ss(tb + 64u * x, sdesc_join(loK + offA, hi), sdesc_join(loQ + offB, hi), idS, kk > 0);
      }
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t offA = ((kk >> 2) * kHalf + (kk & 3) * 32) >> 4;
        const uint32_t offB = ((kk >> 2) * kRHalf + (kk & 3) * 32) >> 4;
        mma_ss(tb + 128u + 64u * x, sdesc_join(loV + offA, hi), sdesc_join(loDO + offB, hi), idS, kk > 0);
      }
      mma_commit(bar(&ctl.s_full[x]));
      if (i >= 1) {
        if (!(ok = mbar_wait(bar(&ctl.p_full[(i - 1) & 1]), ((i - 1) >> 1) & 1, abort_flag))) break;
        tc_fence_after();
        issue_grad(i - 1);
      }
    }
    if (ok) ok = mbar_wait(bar(&ctl.p_full[(ntiles - 1) & 1]), ((ntiles - 1) >> 1) & 1, abort_flag);
    if (ok) {
      tc_fence_after();
      issue_grad(ntiles - 1);
      mma_commit(bar(&ctl.mm_done));
    } else {
      int never = 0;
      mma_commit(bar(&ctl.drain));
      mbar_wait(bar(&ctl.drain), 0, &never);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tb, 512);
  if (tid == 0 && ctl.abort) atomicExch(status, (int)MOBA_ERR_TIMEOUT);
}

// ============================================================================ dQ
constexpr int kHist = 0, kCur = 1;
constexpr int kQThreads = (kSoftmaxWarps + 2) * 32;   // softmax, TMA producer, MMA issuer
// K tiles in three stages: K(i) is read by dQ(i), the last MMA of tile i, and
// K(i + 3) must already be arriving when S(i + 3) is issued during tile i + 2
constexpr int kQKStages = 3;
constexpr uint32_t kQOffQ = 0, kQOffDO = kTile, kQOffK = 2 * kTile, kQOffV = (2 + kQKStages) * kTile;
constexpr uint32_t kQSmem = (4 + kQKStages) * kTile + 1024;

struct QCtl {
  uint64_t q_full, k_full[kQKStages], v_full[2], k_free[kQKStages], v_free[2], s_full, s_read, p_full[2], o_full,
      drain;
  uint32_t tmem_base;
  int abort;
};

template <int MODE>
__global__ void __launch_bounds__(kQThreads, 1) bwd_q_tc_kernel(
    const __nv_bfloat16* __restrict__ q, const __grid_constant__ CUtensorMap tmK,
    const __grid_constant__ CUtensorMap tmV, const __nv_bfloat16* __restrict__ dout,
    const float* __restrict__ lse, const float* __restrict__ delta, const int32_t* __restrict__ offsets,
    const int32_t* __restrict__ rows, const int32_t* __restrict__ tile_start, float* __restrict__ dqacc,
    int* __restrict__ status, Dims dm, int ch) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ QCtl ctl;
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;

  // ---- the row tile and its keys
  int b, g, key0, nkt, r0 = 0, cnt = 0, t_first = 0, h_cur = 0;
  if (MODE == kHist) {
    const int ngroups = dm.batch * dm.hkv * dm.n;
    const int tile = blockIdx.x;
    if (tile >= tile_start[ngroups]) return;
    int lo = 0, hi = ngroups - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (tile_start[mid] <= tile) lo = mid; else hi = mid - 1;
    }
    const int j = lo % dm.n;
    g = (lo / dm.n) % dm.hkv;
    b = lo / (dm.n * dm.hkv);
    const size_t goff = (size_t)ch * ngroups + lo;
    r0 = offsets[goff] + (tile - tile_start[lo]) * kT;
    cnt = min(kT, offsets[goff + 1] - r0);
    key0 = j * dm.B;
    nkt = (dm.B + kT - 1) / kT;
  } else {
    const int ntile = (dm.N + kT - 1) / kT;
    int idx = blockIdx.x;
    const int tau = idx % ntile; idx /= ntile;
    h_cur = idx % dm.hq;
    b = idx / dm.hq;
    if (b >= dm.batch) return;
    g = h_cur / dm.G;
    t_first = tau * kT;
    const int t_last = min(dm.N, t_first + kT) - 1;
    key0 = (t_first / dm.B) * dm.B;
    nkt = (t_last - key0) / kT + 1;
  }

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    mbar_init(bar(&ctl.q_full), kSoftmaxWarps);
    for (int s = 0; s < kQKStages; ++s) {
      mbar_init(bar(&ctl.k_full[s]), 1);
      mbar_init(bar(&ctl.k_free[s]), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(&ctl.v_full[s]), 1);
      mbar_init(bar(&ctl.v_free[s]), 1);
    }
    mbar_init(bar(&ctl.s_full), 1);
    mbar_init(bar(&ctl.s_read), kSoftmaxWarps);
    mbar_init(bar(&ctl.p_full[0]), kSoftmaxWarps);
    mbar_init(bar(&ctl.p_full[1]), kSoftmaxWarps);
    mbar_init(bar(&ctl.o_full), 1);
    mbar_init(bar(&ctl.drain), 1);
    ctl.abort = 0;
    fence_mbar_init();
  }
  if (warp == kSoftmaxWarps) {
    tmem_alloc(smem_u32(&ctl.tmem_base), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = ctl.tmem_base;
  volatile int* abort_flag = &ctl.abort;

  if (warp < kSoftmaxWarps) {
    const int qd = warp & 3, hf = warp >> 2;
    const int rho = qd * 32 + lane;
    const uint32_t lane_off = (uint32_t)(qd * 32) << 16;
    const float sl2 = dm.scale_log2;
    bool valid;
    int r, t, h;
    if (MODE == kHist) {
      valid = rho < cnt;
      r = valid ? rows[r0 + rho] : 0;
      h = r % dm.hq;
      t = (r / dm.hq) % dm.N;
    } else {
      t = t_first + rho;
      valid = t < dm.N;
      h = h_cur;
      r = valid ? (b * dm.N + t) * dm.hq + h : 0;
    }
    {
      // this warp's 32 rows, half hf of each: four rows per copy instruction
      // (eight lanes take a row's eight chunks of the half)
      const int c8 = lane & 7;
#pragma unroll
      for (int k4 = 0; k4 < 8; ++k4) {
        const int rl = 4 * k4 + (lane >> 3);
        const int rs = __shfl_sync(0xffffffffu, r, rl);
        const bool vs = __shfl_sync(0xffffffffu, valid, rl);
        const uint32_t off = hf * kHalf + sw128_off(qd * 32 + rl, c8);
        cp_async16(base + kQOffQ + off, q + (size_t)rs * kD + hf * 64 + c8 * 8, vs);
        cp_async16(base + kQOffDO + off, dout + (size_t)rs * kD + hf * 64 + c8 * 8, vs);
      }
    }
    const float L2 = valid ? lse[((size_t)b * dm.hq + h) * dm.N + t] * kLog2e : INFINITY;
    const float Dr = valid ? delta[r] : 0.f;
    cp_async_commit();
    cp_async_wait<0>();
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(bar(&ctl.q_full));
    // keys valid for the row: [lo_u, hi_u]
    const int lo_u = MODE == kHist ? key0 : (t / dm.B) * dm.B;
    const int hi_u = MODE == kHist ? min(dm.N, key0 + dm.B) - 1 : t;
    bool ok = true;
    for (int i = 0; i < nkt && ok; ++i) {
      ok = __all_sync(0xffffffffu, mbar_wait(bar(&ctl.s_full), i & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      // dP(i), then dS(i), in columns [128, 256) for even i, [384, 512) for odd i
      const uint32_t tD = tb + ((i & 1) ? 384u : 128u) + 64u * hf + lane_off;
      uint32_t sr[64], dr[64];
      tmem_ld32(tb + 64u * hf + lane_off, sr);
      tmem_ld32(tb + 64u * hf + 32 + lane_off, sr + 32);
      tmem_ld32(tD, dr);
      tmem_ld32(tD + 32, dr + 32);
      tmem_wait_ld();
      // S(i) is in registers: the MMA issuer may compute S(i+1) over it
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(&ctl.s_read));
      const int u0 = key0 + i * kT + 64 * hf;     // key of column 0 of this warp's half
      const int vlo = lo_u - u0, vhi = hi_u - u0;
      uint32_t ps[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        float p0 = ex2_approx(__uint_as_float(sr[2 * c]) * sl2 - L2);
        float p1 = ex2_approx(__uint_as_float(sr[2 * c + 1]) * sl2 - L2);
        p0 = (2 * c >= vlo && 2 * c <= vhi) ? p0 : 0.f;
        p1 = (2 * c + 1 >= vlo && 2 * c + 1 <= vhi) ? p1 : 0.f;
        ps[c] = pack_bf16x2(p0 * (__uint_as_float(dr[2 * c]) - Dr), p1 * (__uint_as_float(dr[2 * c + 1]) - Dr));
      }
      // dS over this warp's own dP columns [64 hf, 64 hf + 32): already read
      tmem_st32(tD, ps);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(&ctl.p_full[i & 1]));
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(&ctl.o_full), 0, abort_flag));
    if (ok) {
      tc_fence_after();
      const float scale = sl2 / kLog2e;
      float* dst = dqacc + (size_t)r * kD + 64 * hf;
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        uint32_t o[32];
        tmem_ld32(tb + 256u + 64u * hf + 32u * cc + lane_off, o);
        tmem_wait_ld();
        if (valid) {
#pragma unroll
          for (int e4 = 0; e4 < 8; ++e4)
            red_add_v4(dst + 32 * cc + 4 * e4, __uint_as_float(o[4 * e4]) * scale,
                       __uint_as_float(o[4 * e4 + 1]) * scale, __uint_as_float(o[4 * e4 + 2]) * scale,
                       __uint_as_float(o[4 * e4 + 3]) * scale);
        }
      }
    }
  } else if (warp == kSoftmaxWarps) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      const int y0 = b * dm.N + key0;
      const int x0 = g * kD;
      int issued_k = 0, issued_v = 0;
      for (int i = 0; i < nkt; ++i) {
        const int sk = i % kQKStages, uk = i / kQKStages, s = i & 1;
        const uint32_t ks = base + kQOffK + sk * kTile, vs = base + kQOffV + s * kTile;
        if (i >= kQKStages && !mbar_wait(bar(&ctl.k_free[sk]), (uk - 1) & 1, abort_flag)) break;
        mbar_arrive_expect_tx(bar(&ctl.k_full[sk]), kTile);
        tma_load_2d(ks, &tmK, x0, y0 + i * kT, bar(&ctl.k_full[sk]));
        tma_load_2d(ks + kHalf, &tmK, x0 + 64, y0 + i * kT, bar(&ctl.k_full[sk]));
        issued_k = i + 1;
        if (i >= 2 && !mbar_wait(bar(&ctl.v_free[s]), ((i >> 1) - 1) & 1, abort_flag)) break;
        mbar_arrive_expect_tx(bar(&ctl.v_full[s]), kTile);
        tma_load_2d(vs, &tmV, x0, y0 + i * kT, bar(&ctl.v_full[s]));
        tma_load_2d(vs + kHalf, &tmV, x0 + 64, y0 + i * kT, bar(&ctl.v_full[s]));
        issued_v = i + 1;
      }
      if (*abort_flag) {
        int never = 0;
        for (int i = (issued_k > kQKStages ? issued_k - kQKStages : 0); i < issued_k; ++i)
          mbar_wait(bar(&ctl.k_full[i % kQKStages]), (i / kQKStages) & 1, &never);
        for (int i = (issued_v > 2 ? issued_v - 2 : 0); i < issued_v; ++i)
          mbar_wait(bar(&ctl.v_full[i & 1]), (i >> 1) & 1, &never);
      }
    }
  } else if (lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t idS = idesc_bf16(128, kT, false);
    const uint32_t idQ = idesc_bf16(128, kD, true);        // B (K tile) read MN-major
    const uint32_t hi = sdesc_hi(1024);
    const uint32_t loQ = sdesc_lo(base + kQOffQ, 16), loDO = sdesc_lo(base + kQOffDO, 16),
                   loK = sdesc_lo(base + kQOffK, 16), loV = sdesc_lo(base + kQOffV, 16),
                   mnK = sdesc_lo(base + kQOffK, kHalf);
    // S(n) into columns [0, 128) and dP(n) into its buffer, [128, 256) for even
    // n and [384, 512) for odd n (dQ accumulates in [256, 384))
    auto issue_sdp = [&](int n) {
      const uint32_t ko = (uint32_t)(n % kQKStages) * (kTile >> 4), vo = (n & 1) ? (kTile >> 4) : 0u;
      const uint32_t tdp = tb + ((n & 1) ? 384u : 128u);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t off = ((kk >> 2) * kHalf + (kk & 3) * 32) >> 4;
        mma_ss(tb, sdesc_join(loQ + off, hi), sdesc_join(loK + ko + off, hi), idS, kk > 0);
      }
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t off = ((kk >> 2) * kHalf + (kk & 3) * 32) >> 4;
        mma_ss(tdp, sdesc_join(loDO + off, hi), sdesc_join(loV + vo + off, hi), idS, kk > 0);
      }
    };
    auto kv_ready = [&](int n) -> bool {
      return mbar_wait(bar(&ctl.k_full[n % kQKStages]), (n / kQKStages) & 1, abort_flag) &&
             mbar_wait(bar(&ctl.v_full[n & 1]), (n >> 1) & 1, abort_flag);
    };
    bool ok = mbar_wait(bar(&ctl.q_full), 0, abort_flag) && kv_ready(0);
    if (ok) {
      tc_fence_after();
      issue_sdp(0);
      mma_commit(bar(&ctl.s_full));
      mma_commit(bar(&ctl.v_free[0]));
    }
    for (int i = 0; i < nkt && ok; ++i) {
      // S(i+1), dP(i+1) as soon as the softmax warps hold S(i) in registers: they
      // run on the tensor cores while dS(i) is computed (dP(i+1) goes to the
      // other buffer; the one it overwrites was last read by dQ(i-1), issued
      // before it)
      if (i + 1 < nkt) {
        if (!(ok = kv_ready(i + 1) && mbar_wait(bar(&ctl.s_read), i & 1, abort_flag))) break;
        tc_fence_after();
        issue_sdp(i + 1);
        mma_commit(bar(&ctl.s_full));
        mma_commit(bar(&ctl.v_free[(i + 1) & 1]));
      }
      if (!(ok = mbar_wait(bar(&ctl.p_full[i & 1]), (i >> 1) & 1, abort_flag))) break;
      tc_fence_after();
      // dQ += dS K: dS of keys 0-63 in the first 32 columns of its buffer, keys
      // 64-127 in columns 64-95
      const uint32_t ko = (uint32_t)(i % kQKStages) * (kTile >> 4);
      const uint32_t tds = tb + ((i & 1) ? 384u : 128u);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t a = tds + (kk < 4 ? kk * 8u : 64u + (kk - 4) * 8u);
        mma_ts(tb + 256u, a, sdesc_join(mnK + ko + ((kk * 2048) >> 4), hi), idQ, (i > 0 || kk > 0) ? 1u : 0u);
      }
      mma_commit(bar(&ctl.k_free[i % kQKStages]));
    }
    if (ok) {
      mma_commit(bar(&ctl.o_full));
    } else {
      int never = 0;
      mma_commit(bar(&ctl.drain));
      mbar_wait(bar(&ctl.drain), 0, &never);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kSoftmaxWarps) tmem_dealloc(tb, 512);
  if (tid == 0 && ctl.abort) atomicExch(status, (int)MOBA_ERR_TIMEOUT);
}

__global__ void dq_convert_kernel(const float* __restrict__ acc, __nv_bfloat16* __restrict__ dq, int64_t n4) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n4) return;
  const float4 x = reinterpret_cast<const float4*>(acc)[i];
  reinterpret_cast<uint2*>(dq)[i] = make_uint2(pack_bf16x2(x.x, x.y), pack_bf16x2(x.z, x.w));
}

}  // namespace

int attn_bwd_tc_rows_per_tile() { return kT; }

cudaError_t launch_bwd_kv_tc(const Dims& dm, const void* q, const void* k, const void* v, const void* dout,
                             const float* lse, const float* delta, const int32_t* offsets, const int32_t* rows,
                             void* dk, void* dv, int* status, cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(bwd_kv_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kKvSmem);
  if (e != cudaSuccess) return e;
  const int64_t grid = (int64_t)dm.batch * dm.hkv * dm.n * ((dm.B + kT - 1) / kT);
  bwd_kv_tc_kernel<<<grid, kKvThreads, kKvSmem, stream>>>(
      (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v, (const __nv_bfloat16*)dout,
      lse, delta, offsets, rows, (__nv_bfloat16*)dk, (__nv_bfloat16*)dv, status, dm);
  return cudaGetLastError();
}

cudaError_t launch_bwd_q_tc(const Dims& dm, bool cur, const void* q, const void* k, const void* v,
                            const void* dout, const float* lse, const float* delta, const int32_t* offsets,
                            const int32_t* rows, const int32_t* tile_start, float* dqacc, int* status, int ch,
                            int64_t grid, cudaStream_t stream) {
  CUtensorMap mk, mv;
  if (!make_kv_map(&mk, k, dm) || !make_kv_map(&mv, v, dm)) return cudaErrorInvalidValue;
  auto kern = cur ? bwd_q_tc_kernel<kCur> : bwd_q_tc_kernel<kHist>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kQSmem);
  if (e != cudaSuccess) return e;
  if (cur) grid = (int64_t)((dm.N + kT - 1) / kT) * dm.hq * dm.batch;
  kern<<<grid, kQThreads, kQSmem, stream>>>((const __nv_bfloat16*)q, mk, mv, (const __nv_bfloat16*)dout, lse,
                                            delta, offsets, rows, tile_start, dqacc, status, dm, ch);
  return cudaGetLastError();
}

cudaError_t launch_dq_convert(const float* acc, void* dq, int64_t n, cudaStream_t stream) {
  const int64_t n4 = n / 4;
  dq_convert_kernel<<<(n4 + 255) / 256, 256, 0, stream>>>(acc, (__nv_bfloat16*)dq, n4);
  return cudaGetLastError();
}

}  // namespace moba
