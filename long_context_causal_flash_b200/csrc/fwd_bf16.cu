// bf16 attention forward on the 5th-generation tensor cores (tcgen05 / TMEM), sm_100a.
//
// The bf16 path of kev PR #202 ("The change": a bf16 call keeps grouped-query
// attention on a flash kernel) and the 1M-token packed workloads of maxtext PR #4929
// run here.  QK^T and PV are dense contractions, so both go to tcgen05.mma with fp32
// accumulators in tensor memory; the softmax runs on the CUDA cores between them.
//
// CTA = one tile of 128 query rows = (128 / G) positions x all G query heads that
// share one key/value head (the MMA's M = 128), so each K/V tile in shared memory
// serves G heads and K/V are never repeated in HBM.  416 threads, 1 CTA per SM.
//
// Issue rate.  One thread issues a tcgen05.mma about every 200 cycles whatever its N
// (measured on B200), while an M128 x N256 x K16 MMA takes the tensor core about as
// long.  A 64-key tile needs 16 MMAs for S = Q K^T (N = 64) and 4 for O += P V
// (N = 256), so a single issuer would leave the tensor core idle most of the time.
// Three issuing warps on different SM sub-partitions share the work: two issue the
// two halves of the d = 256 contraction of S into separate accumulators (S_a, S_b,
// summed by the softmax), one issues PV.
//
// Tensor memory (512 columns x 128 lanes, lane = query row):
//   [  0, 256)  O accumulator, fp32
//   [256, 512)  two S buffers of 128 columns: S_a at +0, S_b at +64 (64 keys each)
// Shared memory: Q (64 KiB), 2-stage K and V rings (64 keys x 256 d, 32 KiB per
// stage) and a 2-buffer P ring (128 rows x 64 keys bf16, K-major), all with the
// 128-byte swizzle; Q, K and V are filled by TMA.
//
// Roles:
//   warp 0     TMA producer of Q (once) and the K tiles;  warp 10  of the V tiles.
//   warp 1     TMEM owner; issues S_a (d 0-127);  warp 11 issues S_b (d 128-255).
//   warp 12    issues O += P V.
//   warps 2-9  softmax, two warps per TMEM lane quarter (32 rows each): `half` 0 takes
//              S columns 0-31 and O columns 0-127, `half` 1 the rest.  Per tile: load
//              S_a + S_b, mask (partial tiles), row max exchanged within the pair,
//              P = 2^(S*scale - m) as bf16 into shared memory, row sum.  The running
//              max m is raised only when it grows by more than 8 (log2): P <= 2^8
//              then, and O is rescaled in TMEM only on those rare raises.
//              Epilogue: O / l to bf16, LSE in fp32.
#include "internal.h"
#include "tcgen05.cuh"

#include <cuda_bf16.h>

namespace gqa {
namespace {

constexpr int kRows = kBf16Rows;  // 128
constexpr int kBc = kBf16Bc;      // 64 keys per tile
constexpr int kThreads = 416;     // 13 warps
constexpr int kVWarp = 10, kSbWarp = 11, kPVWarp = 12;
constexpr int kStages = 2;              // K and V rings
constexpr int kQBlock = kRows * 128;    // 128 rows x 64 d bf16: 16 KiB
constexpr int kQBytes = 4 * kQBlock;    // 64 KiB
constexpr int kKVBlock = kBc * 128;     // 64 keys x 64 d bf16: 8 KiB
constexpr int kKVBytes = 4 * kKVBlock;  // one 64-key tile: 32 KiB
constexpr int kPBytes = kRows * 128;    // 128 rows x 64 keys bf16: 16 KiB
constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + kQBytes;
constexpr int kOffV = kOffK + kStages * kKVBytes;
constexpr int kOffP = kOffV + kStages * kKVBytes;
constexpr int kOffBar = kOffP + 2 * kPBytes;
constexpr int kOffRed = kOffBar + 256;                   // [tile parity][half][row] fp32 exchange
constexpr int kSmemBytes = kOffRed + 2 * 2 * kRows * 4;  // dynamic smem is 1024-byte aligned
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 0;
constexpr uint32_t kTmemS = 256;  // buffer b at +128 b: S_a at +0, S_b at +64
constexpr float kRescaleThreshold = 8.0f;  // log2 units: P stays <= 256 between rescales

// barrier indices (8 bytes each)
enum {
  kBarQ = 0,                          // Q tile landed
  kBarKFull = 1,                      // + stage
  kBarKEmpty = kBarKFull + kStages,   // + stage, 2 arrivals (S_a and S_b issuers)
  kBarVFull = kBarKEmpty + kStages,
  kBarVEmpty = kBarVFull + kStages,
  kBarSFull = kBarVEmpty + kStages,   // + S buffer, 2 arrivals
  kBarSFree = kBarSFull + 2,          // + S buffer, 8 arrivals (softmax read S)
  kBarPFull = kBarSFree + 2,          // + P buffer, 8 arrivals
  kBarPVDone = kBarPFull + 2,         // + P buffer
  kNumBars = kBarPVDone + 2
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

// Named barrier over the 64 threads of a softmax warp pair; returns the AND of
// `pred` over them, so both warps take the same branch afterwards.
__device__ __forceinline__ bool pair_and(uint32_t id, bool pred) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, 64, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(out)
      : "r"(uint32_t(pred)), "r"(id)
      : "memory");
  return out != 0;
}

// 2^x on the MUFU unit (PTX ex2.approx.ftz.f32): 2^-inf = 0, relative error ~2^-22.
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
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
  extern __shared__ __align__(1024) char smem_raw[];
  const uint32_t sbase = smem_u32(smem_raw);
  if (sbase & 1023u) {  // the swizzled tiles need 1024-byte alignment; never expected
    if (threadIdx.x == 0) set_status(p.status, GQA_ERR_LAUNCH);
    return;
  }
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
    for (int s = 0; s < kStages; ++s) {
      mbar_init(B(kBarKFull + s), 1);
      mbar_init(B(kBarKEmpty + s), 2);
      mbar_init(B(kBarVFull + s), 1);
      mbar_init(B(kBarVEmpty + s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(B(kBarSFull + s), 2);
      mbar_init(B(kBarSFree + s), 8);
      mbar_init(B(kBarPFull + s), 8);
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

  if (warp == 0 || warp == kVWarp) {
    // ---------------------------------------------------------------- TMA producers
    if (lane == 0) {
      const bool is_k = warp == 0;
      const CUtensorMap* map = is_k ? &tmK : &tmV;
      tma_prefetch_desc(map);
      const int kvhead = b * p.Hkv + g;
      const uint32_t ring = is_k ? sK : sV;
      const int bar_full = is_k ? kBarKFull : kBarVFull;
      const int bar_empty = is_k ? kBarKEmpty : kBarVEmpty;
      if (is_k) {
        tma_prefetch_desc(&tmQ);
        mbar_arrive_expect_tx(B(kBarQ), kQBytes);
        for (int c = 0; c < 4; ++c)
          tma_load_3d(sQ + c * kQBlock, &tmQ, B(kBarQ), c * 64, int(q0), b * p.Hq + g * p.G);
      }
      int issued = 0;
      for (int kt = kbeg; kt < kend; ++kt) {
        if (classify(p, q0, i1, qb, kt) == GQA_TILE_SKIP) continue;
        const int s = issued % kStages;
        const uint32_t par = (uint32_t(issued / kStages) & 1u) ^ 1u;  // first pass: free
        if (!mbar_wait_bounded(B(bar_empty + s), par, budget, p.status)) break;
        mbar_arrive_expect_tx(B(bar_full + s), kKVBytes);
        for (int c = 0; c < 4; ++c)
          tma_load_3d(ring + s * kKVBytes + c * kKVBlock, map, B(bar_full + s), c * 64, kt * kBc, kvhead);
        ++issued;
      }
      // no copies may be in flight when the CTA ends
      if (is_k) mbar_wait_bounded(B(kBarQ), 0, budget, p.status);
      for (int i = issued - kStages; i < issued; ++i)
        if (i >= 0) mbar_wait_bounded(B(bar_full + i % kStages), uint32_t(i / kStages) & 1u, budget, p.status);
    }
  } else if (warp == 1 || warp == kSbWarp) {
    // ---------------------------------------------------------------- S issuers
    // part 0 (warp 1): K-steps 0-7 into S_a;  part 1 (warp 11): K-steps 8-15 into S_b.
    if (lane == 0) {
      const int part = warp == 1 ? 0 : 1;
      constexpr uint32_t id_s = umma::idesc_bf16(kRows, kBc, 0, 0);
      const uint64_t dq = umma::smem_desc(sQ, 16, 1024);
      int t = 0;
      bool ok = mbar_wait_bounded(B(kBarQ), 0, budget, p.status);
      for (int kt = kbeg; ok && kt < kend; ++kt) {
        if (classify(p, q0, i1, qb, kt) == GQA_TILE_SKIP) continue;
        const int s = t % kStages, sb = t & 1;
        if (!(ok = mbar_wait_bounded(B(kBarKFull + s), uint32_t(t / kStages) & 1u, budget, p.status))) break;
        // S buffer sb was read by the softmax of tile t - 2
        if (!(ok = mbar_wait_bounded(B(kBarSFree + sb), ((uint32_t(t) >> 1) & 1u) ^ 1u, budget, p.status))) break;
        umma::fence_after_sync();
        const uint64_t dk = umma::smem_desc(sK + s * kKVBytes, 16, 1024);
        const uint32_t d_tmem = tmem + kTmemS + uint32_t(sb * 128 + part * 64);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const int k16 = part * 8 + kk;
          umma::mma_ss(d_tmem, umma::desc_add(dq, uint32_t((k16 >> 2) * kQBlock + (k16 & 3) * 32)),
                       umma::desc_add(dk, uint32_t((k16 >> 2) * kKVBlock + (k16 & 3) * 32)), id_s, kk > 0);
        }
        umma::commit(B(kBarSFull + sb));
        umma::commit(B(kBarKEmpty + s));
        ++t;
      }
      // this thread's MMAs must be complete before TMEM is released
      for (int i = t - 2; i < t; ++i)
        if (i >= 0) mbar_wait_bounded(B(kBarSFull + (i & 1)), (uint32_t(i) >> 1) & 1u, budget, p.status);
    }
  } else if (warp == kPVWarp) {
    // ---------------------------------------------------------------- PV issuer
    if (lane == 0) {
      constexpr uint32_t id_o = umma::idesc_bf16(kRows, 256, 0, 1);
      int t = 0;
      bool ok = true;
      for (int kt = kbeg; ok && kt < kend; ++kt) {
        if (classify(p, q0, i1, qb, kt) == GQA_TILE_SKIP) continue;
        const int s = t % kStages, pb = t & 1;
        if (!(ok = mbar_wait_bounded(B(kBarPFull + pb), (uint32_t(t) >> 1) & 1u, budget, p.status))) break;
        if (!(ok = mbar_wait_bounded(B(kBarVFull + s), uint32_t(t / kStages) & 1u, budget, p.status))) break;
        umma::fence_after_sync();
        const uint64_t dp = umma::smem_desc(sP + pb * kPBytes, 16, 1024);
        const uint64_t dv = umma::smem_desc(sV + s * kKVBytes, kKVBlock, 1024);
#pragma unroll
        for (int kk = 0; kk < kBc / 16; ++kk)
          umma::mma_ss(tmem + kTmemO, umma::desc_add(dp, uint32_t(kk * 32)), umma::desc_add(dv, uint32_t(kk * 2048)),
                       id_o, (t > 0 || kk > 0) ? 1u : 0u);
        umma::commit(B(kBarPVDone + pb));
        umma::commit(B(kBarVEmpty + s));
        ++t;
      }
      for (int i = t - 2; i < t; ++i)
        if (i >= 0) mbar_wait_bounded(B(kBarPVDone + (i & 1)), (uint32_t(i) >> 1) & 1u, budget, p.status);
    }
  } else {
    // ---------------------------------------------------------------- softmax warps
    // Every wait outcome is agreed on within the warp pair (bar.red.and) before any
    // pair barrier, so the two warps always leave the loop together.
    const int quarter = warp & 3;       // TMEM lane quarter this warp may access
    const int half = (warp - 2) >> 2;
    const int r = quarter * 32 + lane;  // query row of the tile = TMEM lane
    const uint32_t lane_addr = tmem + (uint32_t(quarter * 32) << 16);
    const uint32_t pair_bar = 1u + uint32_t(quarter);
    float* red = reinterpret_cast<float*>(smem_raw + kOffRed);
    const int hh = r / br, pp = r % br;
    const int64_t qi = q0 + pp;
    const bool live = qi < p.Lq;
    const int head = b * p.Hq + g * p.G + hh;
    const int64_t pos = qi + p.off;
    const int sq = p.has_seg ? p.seg_q[min(qi, p.Lq - 1)] : 0;

    float m_ref = -INFINITY;  // running max (log2 units), raised lazily; same in both halves
    float l = 0.f;            // this half's share of the row sum
    int t = 0;
    bool ok = true;
    for (int kt = kbeg; kt < kend; ++kt) {
      const int cls = classify(p, q0, i1, qb, kt);
      if (cls == GQA_TILE_SKIP) continue;
      const int sb = t & 1;
      const uint32_t s_col = kTmemS + uint32_t(sb * 128 + half * 32);
      float x[32];
      const bool ok_s = ok && warp_wait(B(kBarSFull + sb), (uint32_t(t) >> 1) & 1u, budget, p.status);
      if (ok_s) {
        float xb[32];
        umma::fence_after_sync();
        umma::tmem_ld32(lane_addr + s_col, x);
        umma::tmem_ld32(lane_addr + s_col + 64u, xb);
        umma::tmem_wait_ld();
        umma::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(B(kBarSFree + sb));
#pragma unroll
        for (int i = 0; i < 32; ++i) x[i] += xb[i];
      }
      const int64_t j0 = int64_t(kt) * kBc + half * 32;
      const bool need_mask = (cls == GQA_TILE_PARTIAL) || (int64_t(kt) * kBc + kBc > p.Lk);
      if (need_mask) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int64_t j = j0 + i;
          bool vis = j <= pos;
          if (p.has_seg) vis = vis && (j < p.P0 || sq == __ldg(p.seg_kv + min(j, p.Lk - 1)));
          if (!vis) x[i] = -INFINITY;
        }
      }
      float m4[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) m4[u] = x[u];
#pragma unroll
      for (int i = 4; i < 32; ++i) m4[i & 3] = fmaxf(m4[i & 3], x[i]);
      const float pm = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
      red[((t & 1) * 2 + half) * kRows + r] = pm;
      if (!pair_and(pair_bar, ok_s)) {
        ok = false;
        break;
      }
      const float other = red[((t & 1) * 2 + (half ^ 1)) * kRows + r];
      const float mx = fmaxf(pm, other) * p.scale_log2;
      const float m_old = m_ref;
      float alpha = 1.f;
      if (mx > m_ref + kRescaleThreshold) {  // also true for the first visible key
        alpha = ex2_approx(m_old - mx);      // 0 when m_old = -inf
        m_ref = mx;
      }
      const float neg_m = m_ref == -INFINITY ? 0.f : -m_ref;
      uint32_t pk[16];
      float r4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int i = 0; i < 32; i += 2) {
        const float e0 = ex2_approx(fmaf(x[i], p.scale_log2, neg_m));
        const float e1 = ex2_approx(fmaf(x[i + 1], p.scale_log2, neg_m));
        pk[i / 2] = pack_bf16x2(e0, e1);
        r4[(i / 2) & 3] += e0 + e1;
      }
      l = l * alpha + ((r4[0] + r4[1]) + (r4[2] + r4[3]));

      // P buffer sb was read by PV(t-2); O is updated by PV(t-1).
      if (t >= 2) ok = warp_wait(B(kBarPVDone + sb), ((uint32_t(t) - 2) >> 1) & 1u, budget, p.status);
      const bool rescale = (alpha != 1.f) && (m_old != -INFINITY) && (t > 0);
      if (ok && __any_sync(0xffffffffu, rescale)) {
        const int tp = t - 1;
        ok = warp_wait(B(kBarPVDone + (tp & 1)), (uint32_t(tp) >> 1) & 1u, budget, p.status);
        if (ok) {
          umma::fence_after_sync();
#pragma unroll 1
          for (int c0 = half * 128; c0 < half * 128 + 128; c0 += 32) {
            float o[32];
            umma::tmem_ld32(lane_addr + kTmemO + uint32_t(c0), o);
            umma::tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= alpha;
            umma::tmem_st32(lane_addr + kTmemO + uint32_t(c0), o);
          }
          umma::tmem_wait_st();
        }
      }
      if (ok) {
        // P row r, K-major with 128-byte swizzle: 16-byte chunk c at c ^ (r & 7).
        const uint32_t prow = sP + uint32_t(sb * kPBytes + r * 128);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int cc = half * 4 + c;
          sts128u(prow + uint32_t((cc ^ (r & 7)) << 4), pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        }
        fence_proxy_async_smem();
        umma::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(B(kBarPFull + sb));
      }
      ++t;
    }
    // ------------------------------------------------------------ epilogue
    // Row sum = both halves' shares; slot parity t & 1 was last read before tile t-1's barrier.
    red[((t & 1) * 2 + half) * kRows + r] = l;
    if (pair_and(pair_bar, ok)) {
      l += red[((t & 1) * 2 + (half ^ 1)) * kRows + r];
      __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out);
      uint4* dst = reinterpret_cast<uint4*>(out + (int64_t(head) * p.Lq + (live ? qi : 0)) * kHeadDim);
      const float inv = l > 0.f ? 1.f / l : 0.f;
      if (t > 0) {
        const int tl = t - 1;
        ok = warp_wait(B(kBarPVDone + (tl & 1)), (uint32_t(tl) >> 1) & 1u, budget, p.status);
        umma::fence_after_sync();
      }
      if (ok) {
#pragma unroll 1
        for (int c0 = half * 128; c0 < half * 128 + 128; c0 += 32) {
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
        if (live && half == 0) p.lse[int64_t(head) * p.Lq + qi] = l > 0.f ? (m_ref + log2f(l)) * kLn2 : -INFINITY;
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
  if (cudaFuncSetAttribute(fwd_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) != cudaSuccess)
    return GQA_ERR_LAUNCH;
  const int64_t units = int64_t(p.nq) * p.Hkv * p.B;
  if (units <= 0) return GQA_OK;
  if (units > 0x7fffffff) return GQA_ERR_UNSUPPORTED;
  fwd_bf16_kernel<<<unsigned(units), kThreads, kSmemBytes, stream>>>(mq, mk, mv, p);
  return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_LAUNCH;
}

}  // namespace gqa
