// K2 scores on tensor cores: S = Q meanK^T as a tcgen05 GEMM, then the causal
// top-k per query row straight out of TMEM.
//
// "MoBA: Mixture of Block Attention for Long-Context LLMs", paper-graph
// summary §3 "Affinity Scoring" (s_i = <q, mean_pool(K[I_i])>, no softmax
// scale), "Top-k Gating" (top-k blocks plus the always-routed current block),
// "Causality Enforcement" mechanism 1 (no block that is not entirely in the
// past), Implementation, Algorithm 1 Step 1 (S = Q meanK^T with the causal mask
// and top-k).  S never leaves the chip: each row keeps its running top-(k-1)
// in registers and only the k block ids are written.
//
// Precision: q is bf16 (exact); the fp32 pooled keys are split as
// meanK = hi + lo with hi = bf16(meanK) and lo = bf16(meanK - hi), and both
// products accumulate into the same fp32 TMEM columns, so the scores carry
// about 16 mantissa bits of meanK (error far below the 1e-3 score gap that
// decides ties in the parity tests).
//
// One CTA = one (b, kv head g) and a range of kTokens tokens, for all G query
// heads of the group: the group's pooled keys are converted and staged in
// shared memory once, then 128-row Q tiles stream through (TMA, double
// buffered) and the score tiles alternate between two TMEM buffers so the MMA
// of one tile overlaps the selection of the previous one.  Roles:
//   warps 0-3  selection (one thread per query row = TMEM lane)
//   warp 4     TMA producer of Q tiles (and TMEM allocation)
//   warp 5     single-thread tcgen05.mma issuer
// Requires bf16, head_dim 128 and at most 256 blocks (block ids fit 8 bits).
#include <cudaTypedefs.h>
#include <float.h>

#include "launch.h"
#include "sm100.cuh"

namespace moba {

namespace {

using namespace sm100;

constexpr int kD = 128;
constexpr int kRowsT = 128;              // rows per Q tile
constexpr int kTokens = 1024;            // tokens per CTA (per head)
constexpr int kMaxBlocks = 256;          // one MMA of N <= 256
constexpr int kThreads = 192;
constexpr uint32_t kQTile = kRowsT * kD * 2;       // 32 KB
constexpr uint32_t kHalfQ = kRowsT * 128;          // 16 KB
constexpr uint32_t kOffQ = 0;                      // two stages
constexpr uint32_t kOffKB = 2 * kQTile;            // hi then lo, each 2 halves of kMaxBlocks x 128 B
constexpr uint32_t kKBHalf = kMaxBlocks * 128;     // 32 KB
constexpr uint32_t kKB = 2 * kKBHalf;              // 64 KB per (hi | lo)
constexpr uint32_t kSmemBytes = kOffKB + 2 * kKB + 1024;

struct Ctl {
  uint64_t q_full[2], q_free[2], s_full[2], s_free[2], drain;
  uint32_t tmem_base;
  int abort;
  int hist[kMaxBlocks];
};

MOBA_DEV uint32_t bar(const uint64_t* b) { return smem_u32(b); }
MOBA_DEV void named_sync_selectors() { asm volatile("bar.sync 1, 128;\n" ::: "memory"); }
// AND of `v` over the 128 selection threads (all four warps reach it every tile)
MOBA_DEV bool selectors_all(bool v) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.and.pred q, 1, 128, p;\n"
      " selp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(r)
      : "r"((uint32_t)v)
      : "memory");
  return r != 0;
}

template <int KB>
__global__ void __launch_bounds__(kThreads, 1) gate_select_tc_kernel(
    const __grid_constant__ CUtensorMap tmQ, const float* __restrict__ meank,
    int32_t* __restrict__ sel, int32_t* __restrict__ counts, int* __restrict__ status, Dims dm) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ Ctl ctl;
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const int ranges = (dm.t_hi - dm.t_lo + kTokens - 1) / kTokens;
  const int rg = blockIdx.x % ranges;
  const int g = (blockIdx.x / ranges) % dm.hkv;
  const int b = blockIdx.x / (ranges * dm.hkv);
  const int t_begin = dm.t_lo + rg * kTokens;
  const int t_stop = min(dm.t_hi, t_begin + kTokens);
  const int ttiles = (t_stop - t_begin + kRowsT - 1) / kRowsT;
  const int ntiles = ttiles * dm.G;                 // tile k: token tile k / G, head g*G + k % G
  const int cmax_cta = (t_stop - 1) / dm.B;         // blocks [0, cmax_cta) may be candidates
  const int npad = max(16, (cmax_cta + 15) / 16 * 16);
  const int KH = dm.topk - 1;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(&ctl.q_full[s]), 1);
      mbar_init(bar(&ctl.q_free[s]), 1);
      mbar_init(bar(&ctl.s_full[s]), 1);
      mbar_init(bar(&ctl.s_free[s]), kRowsT);
    }
    mbar_init(bar(&ctl.drain), 1);
    ctl.abort = 0;
    fence_mbar_init();
  }
  for (int i = tid; i < kMaxBlocks; i += kThreads) ctl.hist[i] = 0;
  if (warp == 4) {
    tmem_alloc(smem_u32(&ctl.tmem_base), 512);
    tmem_relinquish();
  }
  // pooled keys of (b, g) for blocks < npad as bf16 hi / lo, K-major, 128-byte swizzle
  const uint32_t khi = base + kOffKB, klo = khi + kKB;
  for (int i = tid; i < npad * 16; i += kThreads) {
    const int jr = i >> 4, c = i & 15;              // block row, 8-element chunk
    float x[8];
    if (jr < cmax_cta) {
      const float4* src = reinterpret_cast<const float4*>(
          meank + (((size_t)b * dm.n + jr) * dm.hkv + g) * kD + c * 8);
      const float4 a = __ldg(src), e = __ldg(src + 1);
      x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = e.x; x[5] = e.y; x[6] = e.z; x[7] = e.w;
    } else {
#pragma unroll
      for (int u = 0; u < 8; ++u) x[u] = 0.f;
    }
    uint32_t hi[4], lo[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const __nv_bfloat162 h2 = __floats2bfloat162_rn(x[2 * u], x[2 * u + 1]);
      const float2 hf = __bfloat1622float2(h2);
      hi[u] = *reinterpret_cast<const uint32_t*>(&h2);
      lo[u] = pack_bf16x2(x[2 * u] - hf.x, x[2 * u + 1] - hf.y);
    }
    const uint32_t off = (c >> 3) * kKBHalf + sw128_off(jr, c & 7);
    asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};\n" ::"r"(khi + off), "r"(hi[0]), "r"(hi[1]),
                 "r"(hi[2]), "r"(hi[3]) : "memory");
    asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};\n" ::"r"(klo + off), "r"(lo[0]), "r"(lo[1]),
                 "r"(lo[2]), "r"(lo[3]) : "memory");
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = ctl.tmem_base;
  volatile int* abort_flag = &ctl.abort;

  if (warp < 4) {
    // ------------------------------------------------------------ selection
    const int rho = tid;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    bool ok = true;
    for (int k = 0; k < ntiles && ok; ++k) {
      const int tt = t_begin + (k / dm.G) * kRowsT;
      const int h = g * dm.G + k % dm.G;
      const int t = tt + rho;
      const bool valid = t < dm.t_hi;
      const int c = valid ? t / dm.B : 0;
      const int ctile = (min(dm.t_hi, tt + kRowsT) - 1) / dm.B;   // candidates of the tile: [0, ctile)
      // the decision is uniform over the four selection warps, so the named
      // barriers below are always reached by all of them
      ok = selectors_all(mbar_wait(bar(&ctl.s_full[k & 1]), (k >> 1) & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      // Running top-(k-1) as packed keys: the order-preserving bits of the
      // score with the low 8 bits replaced by 255 - j, so a larger key is a
      // larger score and, between scores that agree to 2^-15 relative (far
      // below the 1e-3 score gap the parity tests allow to differ), the lower
      // block index.  A branch-free insertion network keeps all rows of the
      // warp in lockstep.
      uint32_t a[KB];
#pragma unroll
      for (int i = 0; i < KB; ++i) a[i] = 0u;
      const uint32_t tS = tb + (k & 1) * 256u + lane_off;
      const int jlim = KH > 0 ? ctile : 0;
      for (int j0 = 0; j0 < jlim; j0 += 32) {
        uint32_t sr[32];
        tmem_ld32(tS + j0, sr);
        tmem_wait_ld();
#pragma unroll
        for (int jj = 0; jj < 32; ++jj) {
          const int jb = j0 + jj;
          const uint32_t u = sr[jj];
          const uint32_t ord = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
          const uint32_t key = jb < c ? ((ord & 0xFFFFFF00u) | (uint32_t)(255 - jb)) : 0u;
#pragma unroll
          for (int i = KB - 1; i > 0; --i) a[i] = max(a[i], min(a[i - 1], key));
          a[0] = max(a[0], key);
        }
      }
      tc_fence_before();
      mbar_arrive(bar(&ctl.s_free[k & 1]));
      if (valid) {
        int32_t* outp = sel + ((size_t)(b * dm.N + t) * dm.hq + h) * dm.topk;
        const int m = min(KH, c);
        int ti[KB];
#pragma unroll
        for (int i = 0; i < KB; ++i) ti[i] = 255 - (int)(a[i] & 0xFFu);
#pragma unroll
        for (int i = 0; i < KB; ++i) {
          if (i < m) {
            int rank = 0;
#pragma unroll
            for (int i2 = 0; i2 < KB; ++i2)
              if (i2 < m && ti[i2] < ti[i]) ++rank;
            outp[rank] = ti[i];
            atomicAdd(&ctl.hist[ti[i]], 1);
          }
        }
        outp[m] = c;
        for (int i = m + 1; i < dm.topk; ++i) outp[i] = -1;
      }
      // flush the tile's histogram (a tile never straddles a pass: the pass
      // length is a multiple of 128)
      named_sync_selectors();
      const int ch = tt / dm.chunk;
      int32_t* cnt_g = counts + ((size_t)(ch * dm.batch + b) * dm.hkv + g) * dm.n;
      for (int i = rho; i < ctile; i += kRowsT) {
        const int v = ctl.hist[i];
        if (v) {
          atomicAdd(&cnt_g[i], v);
          ctl.hist[i] = 0;
        }
      }
      named_sync_selectors();
    }
  } else if (warp == 4) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      int issued = 0;
      for (int k = 0; k < ntiles; ++k) {
        const int s = k & 1;
        if (k >= 2 && !mbar_wait(bar(&ctl.q_free[s]), ((k >> 1) - 1) & 1, abort_flag)) break;
        const int tt = t_begin + (k / dm.G) * kRowsT;
        const int h = g * dm.G + k % dm.G;
        const uint32_t qs = base + kOffQ + s * kQTile;
        mbar_arrive_expect_tx(bar(&ctl.q_full[s]), kQTile);
        tma_load_2d(qs, &tmQ, h * kD, b * dm.N + tt, bar(&ctl.q_full[s]));
        tma_load_2d(qs + kHalfQ, &tmQ, h * kD + 64, b * dm.N + tt, bar(&ctl.q_full[s]));
        issued = k + 1;
      }
      if (*abort_flag) {
        int never = 0;
        for (int k = (issued > 2 ? issued - 2 : 0); k < issued; ++k)
          mbar_wait(bar(&ctl.q_full[k & 1]), (k >> 1) & 1, &never);
      }
    }
  } else {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = true;
      for (int k = 0; k < ntiles && ok; ++k) {
        const int s = k & 1;
        const int tt = t_begin + (k / dm.G) * kRowsT;
        const int ctile = (min(dm.t_hi, tt + kRowsT) - 1) / dm.B;
        const int nt = max(16, (ctile + 15) / 16 * 16);
        ok = mbar_wait(bar(&ctl.q_full[s]), (k >> 1) & 1, abort_flag);
        if (ok && k >= 2) ok = mbar_wait(bar(&ctl.s_free[s]), ((k >> 1) - 1) & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
        if (ctile > 0 && KH > 0) {
          const uint32_t idesc = idesc_bf16(128, nt, false);
          const uint32_t qa = base + kOffQ + s * kQTile;
          const uint32_t d = tb + s * 256u;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t qo = (kk >> 2) * kHalfQ + (kk & 3) * 32;
            const uint32_t ko = (kk >> 2) * kKBHalf + (kk & 3) * 32;
            mma_ss(d, sdesc_sw128(qa + qo, 16, 1024), sdesc_sw128(khi + ko, 16, 1024), idesc, kk > 0);
            mma_ss(d, sdesc_sw128(qa + qo, 16, 1024), sdesc_sw128(klo + ko, 16, 1024), idesc, 1);
          }
        }
        mma_commit(bar(&ctl.s_full[s]));
        mma_commit(bar(&ctl.q_free[s]));
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
  if (warp == 4) tmem_dealloc(tb, 512);
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

template <int KB>
cudaError_t run_select(const CUtensorMap& mq, const Dims& dm, const float* meank, int32_t* sel,
                       int32_t* counts, int* status, cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(gate_select_tc_kernel<KB>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  const int ranges = (dm.t_hi - dm.t_lo + kTokens - 1) / kTokens;
  gate_select_tc_kernel<KB><<<(int64_t)ranges * dm.hkv * dm.batch, kThreads, kSmemBytes, stream>>>(
      mq, meank, sel, counts, status, dm);
  return cudaGetLastError();
}

}  // namespace

bool gate_tc_supported(const Dims& dm, int dtype) {
  return dtype == MOBA_BF16 && dm.d == kD && dm.n <= kMaxBlocks && encode_fn_gate() != nullptr;
}

cudaError_t launch_gate_select_tc(const Dims& dm, const void* q, const float* meank, int32_t* sel,
                                  int32_t* counts, int* status, cudaStream_t stream) {
  CUtensorMap mq;
  cuuint64_t dims[2] = {(cuuint64_t)dm.hq * kD, (cuuint64_t)dm.batch * dm.N};
  cuuint64_t strides[1] = {(cuuint64_t)dm.hq * kD * 2};
  cuuint32_t box[2] = {64, kRowsT};
  cuuint32_t es[2] = {1, 1};
  if (encode_fn_gate()(&mq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(q), dims, strides, box,
                       es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                       CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                       CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  const int kh = dm.topk - 1;   // slots of the insertion network: a multiple of 4 >= topk - 1
  return kh <= 4    ? run_select<4>(mq, dm, meank, sel, counts, status, stream)
         : kh <= 8  ? run_select<8>(mq, dm, meank, sel, counts, status, stream)
         : kh <= 12 ? run_select<12>(mq, dm, meank, sel, counts, status, stream)
                    : run_select<16>(mq, dm, meank, sel, counts, status, stream);
}

}  // namespace moba
