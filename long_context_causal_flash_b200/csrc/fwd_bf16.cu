// bf16 attention forward on the 5th-generation tensor cores (tcgen05 / TMEM), sm_100a.
//
// The bf16 path of kev PR #202 ("The change": a bf16 call keeps grouped-query
// attention on a flash kernel) and the 1M-token packed workloads of maxtext PR #4929
// run here.  QK^T and PV are dense contractions, so both go to tcgen05.mma with
// fp32 accumulators in tensor memory; the softmax runs on the CUDA cores between them.
//
// CTA = one tile of 128 query rows = (128 / G) positions x all G query heads that
// share one key/value head (the MMA's M = 128), so each K/V tile in shared memory
// serves G heads and K/V are never repeated in HBM.  192 threads, 1 CTA per SM:
//   warp 0    TMA producer: Q once (4 boxes of 64 d), K and V tiles of 64 keys into
//             2-stage rings, 128-byte swizzle.
//   warp 1    TMEM owner (512 columns) and MMA issuer (one thread):
//               S(t)  = Q K(t)^T    M128 N64  K256, into TMEM S buffer t % 2
//               O    += P(t) V(t)   M128 N256 K64,  into TMEM O (256 columns)
//             S(t+1) is issued before PV(t), so the tensor pipe works while the
//             softmax of tile t runs.  tcgen05.commit signals the mbarriers.
//   warps 2-5 softmax, one query row per thread (TMEM lane = row): load S(t) from
//             TMEM, mask (partial tiles), running max in base 2, P = exp2(S - m) as
//             bf16 into a 2-buffer shared-memory ring (K-major, swizzled), row sum.
//             The running max is only raised when it grows by more than 8 (log2),
//             rescaling O in TMEM then; otherwise P <= 2^8 is exact to accumulate.
//             Epilogue: O / l to bf16, LSE in fp32.
#include "internal.h"
#include "tcgen05.cuh"

#include <cuda_bf16.h>

namespace gqa {
namespace {

constexpr int kRows = kBf16Rows;  // 128
constexpr int kBc = kBf16Bc;      // 64 keys per tile
constexpr int kThreads = 192;
constexpr int kQBlock = kRows * 128;      // one 64-wide d block of Q: 16 KiB
constexpr int kQBytes = 4 * kQBlock;      // 64 KiB
constexpr int kKVBlock = kBc * 128;       // 64 keys x 64 d: 8 KiB
constexpr int kKVBytes = 4 * kKVBlock;    // 32 KiB per stage
constexpr int kPBytes = kRows * 128;      // 128 rows x 64 keys bf16: 16 KiB
constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + kQBytes;
constexpr int kOffV = kOffK + 2 * kKVBytes;
constexpr int kOffP = kOffV + 2 * kKVBytes;
constexpr int kOffBar = kOffP + 2 * kPBytes;
constexpr int kSmemBytes = kOffBar + 256 + 1024;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 0;    // columns [0, 256): O accumulator
constexpr uint32_t kTmemS = 256;  // columns [256, 384): two S buffers of 64
constexpr float kRescaleThreshold = 8.0f;  // log2 units: P stays <= 256 between rescales

// barrier indices (8 bytes each)
enum {
  kBarQ = 0,
  kBarKFull = 1,   // +stage
  kBarKEmpty = 3,  // +stage
  kBarVFull = 5,
  kBarVEmpty = 7,
  kBarSFull = 9,   // +buffer
  kBarSFree = 11,
  kBarPFull = 13,
  kBarPVDone = 15,
  kNumBars = 17
};
constexpr int kOffTmemSlot = kOffBar + 8 * kNumBars;
static_assert(kOffTmemSlot + 4 <= kOffBar + 256, "barrier area");
static_assert(kSmemBytes <= 232448, "shared memory per block");

__device__ __forceinline__ int classify(const FwdParams& p, int64_t i0, int64_t i1, SegBounds qb, int kt) {
  const int64_t j0 = int64_t(kt) * kBc;
  const int64_t j1 = min(p.Lk, j0 + kBc) - 1;
  SegBounds kb{0, 0};
  if (p.has_seg) kb = SegBounds{p.kv_bounds[2 * kt], p.kv_bounds[2 * kt + 1]};
  return tile_class(i0, i1, j0, j1, p.off, p.P0, p.has_seg != 0, qb, kb);
}

// Bounded wait taken by a whole warp: every lane sees the same outcome, so the
// warp stays converged for the warp-collective operations that follow.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, int64_t budget, int32_t* status) {
  return __all_sync(0xffffffffu, mbar_wait_bounded(bar, parity, budget, status));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ void sts128u(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

__global__ void __launch_bounds__(kThreads, 1)
fwd_bf16_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ FwdParams p) {
  extern __shared__ char smem_raw[];
  const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t sQ = sbase + kOffQ, sK = sbase + kOffK, sV = sbase + kOffV, sP = sbase + kOffP;
  const uint32_t bar = sbase + kOffBar;
  auto B = [&](int i) { return bar + 8u * uint32_t(i); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int per_qt = p.Hkv * p.B;
  const int qt = p.nq - 1 - int(blockIdx.x / per_qt);
  const int rem = int(blockIdx.x % per_qt);
  const int g = rem % p.Hkv;
  const int b = rem / p.Hkv;
  const int br = p.br;
  const int64_t q0 = int64_t(qt) * br;
  const int64_t i1 = min(p.Lq, q0 + br) - 1;
  SegBounds qb{0, 0};
  int kbeg, kend;
  if (p.has_seg) {
    qb = SegBounds{p.q_bounds[2 * qt], p.q_bounds[2 * qt + 1]};
    kbeg = p.q_ranges[2 * qt];
    kend = p.q_ranges[2 * qt + 1];
  } else {
    kv_range_no_seg(i1, p.off, kBc, p.nk, &kbeg, &kend);
  }

  if (threadIdx.x == 0) {
    mbar_init(B(kBarQ), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(B(kBarKFull + s), 1);
      mbar_init(B(kBarKEmpty + s), 1);
      mbar_init(B(kBarVFull + s), 1);
      mbar_init(B(kBarVEmpty + s), 1);
      mbar_init(B(kBarSFull + s), 1);
      mbar_init(B(kBarSFree + s), 4);
      mbar_init(B(kBarPFull + s), 4);
      mbar_init(B(kBarPVDone + s), 1);
    }
    fence_barrier_init();
  }
  if (warp == 1) umma::tmem_alloc(sbase + kOffTmemSlot, kTmemCols);
  umma::fence_before_sync();
  __syncthreads();
  umma::fence_after_sync();
  uint32_t tmem;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(tmem) : "r"(sbase + kOffTmemSlot));

  const int64_t budget = p.wait_budget_ns;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      const int qhead = b * p.Hq + g * p.G;
      const int kvhead = b * p.Hkv + g;
      mbar_arrive_expect_tx(B(kBarQ), kQBytes);
      for (int c = 0; c < 4; ++c) tma_load_3d(sQ + c * kQBlock, &tmQ, B(kBarQ), c * 64, int(q0), qhead);
      int nk_issued = 0, nv_issued = 0;
      for (int kt = kbeg; kt < kend; ++kt) {
        if (classify(p, q0, i1, qb, kt) == GQA_TILE_SKIP) continue;
        const int s = nk_issued & 1;
        const uint32_t par = ((uint32_t(nk_issued) >> 1) & 1u) ^ 1u;
        if (!mbar_wait_bounded(B(kBarKEmpty + s), par, budget, p.status)) break;
        mbar_arrive_expect_tx(B(kBarKFull + s), kKVBytes);
        for (int c = 0; c < 4; ++c)
          tma_load_3d(sK + s * kKVBytes + c * kKVBlock, &tmK, B(kBarKFull + s), c * 64, kt * kBc, kvhead);
        ++nk_issued;
        if (!mbar_wait_bounded(B(kBarVEmpty + s), par, budget, p.status)) break;
        mbar_arrive_expect_tx(B(kBarVFull + s), kKVBytes);
        for (int c = 0; c < 4; ++c)
          tma_load_3d(sV + s * kKVBytes + c * kKVBlock, &tmV, B(kBarVFull + s), c * 64, kt * kBc, kvhead);
        ++nv_issued;
      }
      // no copies may be in flight when the CTA ends
      mbar_wait_bounded(B(kBarQ), 0, budget, p.status);
      for (int i = nk_issued - 2; i < nk_issued; ++i)
        if (i >= 0) mbar_wait_bounded(B(kBarKFull + (i & 1)), (uint32_t(i) >> 1) & 1u, budget, p.status);
      for (int i = nv_issued - 2; i < nv_issued; ++i)
        if (i >= 0) mbar_wait_bounded(B(kBarVFull + (i & 1)), (uint32_t(i) >> 1) & 1u, budget, p.status);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t id_s = umma::idesc_bf16(kRows, kBc, 0, 0);
      constexpr uint32_t id_o = umma::idesc_bf16(kRows, 256, 0, 1);
      const uint64_t dq = umma::smem_desc(sQ, 16, 1024);
      int n_s = 0, n_pv = 0;
      bool ok = mbar_wait_bounded(B(kBarQ), 0, budget, p.status);
      // Tiles are enumerated twice in lockstep: `ks` for S issue (one ahead), `kp` for PV.
      int ks = kbeg, kp = kbeg;
      auto next_tile = [&](int kt) {
        while (kt < kend && classify(p, q0, i1, qb, kt) == GQA_TILE_SKIP) ++kt;
        return kt;
      };
      auto issue_s = [&](int t) -> bool {
        const int s = t & 1;
        const uint32_t ph = (uint32_t(t) >> 1) & 1u;
        if (!mbar_wait_bounded(B(kBarKFull + s), ph, budget, p.status)) return false;
        if (!mbar_wait_bounded(B(kBarSFree + s), ph ^ 1u, budget, p.status)) return false;
        umma::fence_after_sync();
        const uint64_t dk = umma::smem_desc(sK + s * kKVBytes, 16, 1024);
        const uint32_t d_tmem = tmem + kTmemS + uint32_t(s * kBc);
#pragma unroll
        for (int kk = 0; kk < 16; ++kk) {
          const uint32_t off_q = uint32_t((kk >> 2) * kQBlock + (kk & 3) * 32);
          const uint32_t off_k = uint32_t((kk >> 2) * kKVBlock + (kk & 3) * 32);
          umma::mma_ss(d_tmem, umma::desc_add(dq, off_q), umma::desc_add(dk, off_k), id_s, kk > 0);
        }
        umma::commit(B(kBarSFull + s));
        umma::commit(B(kBarKEmpty + s));
        return true;
      };
      if (ok) {
        ks = next_tile(ks);
        if (ks < kend) {
          ok = issue_s(n_s);
          if (ok) {
            ++n_s;
            ks = next_tile(ks + 1);
          }
        }
      }
      while (ok) {
        kp = next_tile(kp);
        if (kp >= kend) break;
        // S for the next tile first: the tensor pipe computes it during this tile's softmax.
        if (ks < kend) {
          if (!(ok = issue_s(n_s))) break;
          ++n_s;
          ks = next_tile(ks + 1);
        }
        const int t = n_pv, s = t & 1;
        const uint32_t ph = (uint32_t(t) >> 1) & 1u;
        if (!(ok = mbar_wait_bounded(B(kBarPFull + s), ph, budget, p.status))) break;
        if (!(ok = mbar_wait_bounded(B(kBarVFull + s), ph, budget, p.status))) break;
        umma::fence_after_sync();
        const uint64_t dp = umma::smem_desc(sP + s * kPBytes, 16, 1024);
        const uint64_t dv = umma::smem_desc(sV + s * kKVBytes, kKVBlock, 1024);
#pragma unroll
        for (int kk = 0; kk < kBc / 16; ++kk)
          umma::mma_ss(tmem + kTmemO, umma::desc_add(dp, uint32_t(kk * 32)), umma::desc_add(dv, uint32_t(kk * 2048)),
                       id_o, (t > 0 || kk > 0) ? 1u : 0u);
        umma::commit(B(kBarPVDone + s));
        umma::commit(B(kBarVEmpty + s));
        ++n_pv;
        ++kp;
      }
      // all issued MMAs must be complete before TMEM is released
      for (int i = n_s - 2; i < n_s; ++i)
        if (i >= 0) mbar_wait_bounded(B(kBarSFull + (i & 1)), (uint32_t(i) >> 1) & 1u, budget, p.status);
      for (int i = n_pv - 2; i < n_pv; ++i)
        if (i >= 0) mbar_wait_bounded(B(kBarPVDone + (i & 1)), (uint32_t(i) >> 1) & 1u, budget, p.status);
    }
  } else {
    // ---------------------------------------------------------------- softmax warps
    const int quarter = warp & 3;           // TMEM lane quarter this warp may access
    const int r = quarter * 32 + lane;      // query row of the tile = TMEM lane
    const uint32_t lane_addr = tmem + (uint32_t(quarter * 32) << 16);
    const int hh = r / br, pp = r % br;
    const int64_t qi = q0 + pp;
    const int64_t pos = qi + p.off;
    const int sq = p.has_seg ? p.seg_q[min(qi, p.Lq - 1)] : 0;
    float m_ref = -INFINITY;  // running max (log2 units), raised lazily
    float l = 0.f;
    int t = 0;
    bool ok = true;
    for (int kt = kbeg; kt < kend; ++kt) {
      const int cls = classify(p, q0, i1, qb, kt);
      if (cls == GQA_TILE_SKIP) continue;
      const int s = t & 1;
      const uint32_t ph = (uint32_t(t) >> 1) & 1u;
      if (!(ok = warp_wait(B(kBarSFull + s), ph, budget, p.status))) break;
      umma::fence_after_sync();
      float x[kBc];
      {
        float a[32], c[32];
        umma::tmem_ld32(lane_addr + kTmemS + uint32_t(s * kBc), a);
        umma::tmem_ld32(lane_addr + kTmemS + uint32_t(s * kBc + 32), c);
        umma::tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          x[i] = a[i];
          x[32 + i] = c[i];
        }
      }
      umma::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(B(kBarSFree + s));

      const int64_t j0 = int64_t(kt) * kBc;
      const bool need_mask = (cls == GQA_TILE_PARTIAL) || (j0 + kBc > p.Lk);
      float mx = -INFINITY;
#pragma unroll
      for (int i = 0; i < kBc; ++i) {
        float v = x[i] * p.scale_log2;
        if (need_mask) {
          const int64_t j = j0 + i;
          bool vis = j <= pos;
          if (p.has_seg) vis = vis && (j < p.P0 || sq == __ldg(p.seg_kv + min(j, p.Lk - 1)));
          if (!vis) v = -INFINITY;
        }
        x[i] = v;
        mx = fmaxf(mx, v);
      }
      const float m_old = m_ref;
      float alpha = 1.f;
      if (mx > m_ref + kRescaleThreshold) {  // also true for the first visible key
        alpha = exp2f(m_old - mx);             // 0 when m_old = -inf
        m_ref = mx;
      }
      const float m_use = m_ref == -INFINITY ? 0.f : m_ref;
      uint32_t pk[kBc / 2];
      float rs = 0.f;
#pragma unroll
      for (int i = 0; i < kBc; i += 2) {
        const float e0 = exp2f(x[i] - m_use), e1 = exp2f(x[i + 1] - m_use);
        pk[i / 2] = pack_bf16x2(e0, e1);
        __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162*>(&pk[i / 2]);
        rs += __low2float(h) + __high2float(h);  // sum what the MMA will see
      }
      l = l * alpha + rs;

      // P buffer s was read by PV(t-2); O is updated by PV(t-1).
      if (t >= 2)
        if (!(ok = warp_wait(B(kBarPVDone + s), ((uint32_t(t) - 2) >> 1) & 1u, budget, p.status))) break;
      const bool rescale = (alpha != 1.f) && (m_old != -INFINITY) && (t > 0);
      if (__any_sync(0xffffffffu, rescale)) {
        const int tp = t - 1;
        if (!(ok = warp_wait(B(kBarPVDone + (tp & 1)), (uint32_t(tp) >> 1) & 1u, budget, p.status))) break;
        umma::fence_after_sync();
#pragma unroll 1
        for (int c0 = 0; c0 < 256; c0 += 32) {
          float o[32];
          umma::tmem_ld32(lane_addr + kTmemO + uint32_t(c0), o);
          umma::tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= alpha;
          umma::tmem_st32(lane_addr + kTmemO + uint32_t(c0), o);
        }
        umma::tmem_wait_st();
      }
      // P row r, K-major with 128-byte swizzle: 16-byte chunk c at c ^ (r & 7).
      const uint32_t prow = sP + uint32_t(s * kPBytes + r * 128);
#pragma unroll
      for (int c = 0; c < 8; ++c)
        sts128u(prow + uint32_t((c ^ (r & 7)) << 4), pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      fence_proxy_async_smem();
      umma::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(B(kBarPFull + s));
      ++t;
    }
    // ------------------------------------------------------------ epilogue
    if (ok) {
      __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out);
      const int head = b * p.Hq + g * p.G + hh;
      const bool live = qi < p.Lq;
      uint4* dst = reinterpret_cast<uint4*>(out + (int64_t(head) * p.Lq + (live ? qi : 0)) * kHeadDim);
      const float inv = l > 0.f ? 1.f / l : 0.f;
      if (t > 0) {
        const int tl = t - 1;
        ok = warp_wait(B(kBarPVDone + (tl & 1)), (uint32_t(tl) >> 1) & 1u, budget, p.status);
        umma::fence_after_sync();
      }
      if (ok) {
#pragma unroll 1
        for (int c0 = 0; c0 < 256; c0 += 32) {
          float o[32];
          if (t > 0) {
            umma::tmem_ld32(lane_addr + kTmemO + uint32_t(c0), o);
            umma::tmem_wait_ld();
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = 0.f;
          }
          if (live) {
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4) {
              uint4 w;
              w.x = pack_bf16x2(o[8 * v4 + 0] * inv, o[8 * v4 + 1] * inv);
              w.y = pack_bf16x2(o[8 * v4 + 2] * inv, o[8 * v4 + 3] * inv);
              w.z = pack_bf16x2(o[8 * v4 + 4] * inv, o[8 * v4 + 5] * inv);
              w.w = pack_bf16x2(o[8 * v4 + 6] * inv, o[8 * v4 + 7] * inv);
              dst[c0 / 8 + v4] = w;
            }
          }
        }
        if (live) p.lse[int64_t(head) * p.Lq + qi] = l > 0.f ? (m_ref + log2f(l)) * kLn2 : -INFINITY;
      }
    }
    umma::fence_before_sync();
  }

  __syncthreads();
  if (warp == 1) {
    umma::fence_after_sync();
    umma::tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

int launch_fwd_bf16(const FwdTensors& t, const FwdParams& p, cudaStream_t stream) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return GQA_ERR_LAUNCH;
  CUtensorMap mq, mk, mv;
  const cuuint32_t estr[3] = {1, 1, 1};
  {
    const cuuint64_t dims[3] = {cuuint64_t(kHeadDim), cuuint64_t(p.Lq), cuuint64_t(p.B) * p.Hq};
    const cuuint64_t strides[2] = {cuuint64_t(kHeadDim) * 2, cuuint64_t(p.Lq) * kHeadDim * 2};
    const cuuint32_t box[3] = {64, cuuint32_t(p.br), cuuint32_t(p.G)};
    if (enc(&mq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(t.q), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return GQA_ERR_LAUNCH;
  }
  {
    const cuuint64_t dims[3] = {cuuint64_t(kHeadDim), cuuint64_t(p.Lk), cuuint64_t(p.B) * p.Hkv};
    const cuuint64_t strides[2] = {cuuint64_t(kHeadDim) * 2, cuuint64_t(p.Lk) * kHeadDim * 2};
    const cuuint32_t box[3] = {64, cuuint32_t(kBc), 1};
    if (enc(&mk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(t.k), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return GQA_ERR_LAUNCH;
    if (enc(&mv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(t.v), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return GQA_ERR_LAUNCH;
  }
  if (cudaFuncSetAttribute(fwd_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) != cudaSuccess)
    return GQA_ERR_LAUNCH;
  const int64_t units = int64_t(p.nq) * p.Hkv * p.B;
  if (units <= 0) return GQA_OK;
  if (units > 0x7fffffff) return GQA_ERR_UNSUPPORTED;
  fwd_bf16_kernel<<<unsigned(units), kThreads, kSmemBytes, stream>>>(mq, mk, mv, p);
  return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_LAUNCH;
}

}  // namespace gqa
