// bf16 attention forward on the 5th-generation tensor cores (tcgen05 / TMEM), sm_100a.
//
// The bf16 path of kev PR #202 ("The change": a bf16 call keeps grouped-query
// attention on a flash kernel) and the 1M-token packed workloads of maxtext PR #4929
// run here.  QK^T and PV are dense contractions, so both go to tcgen05.mma with fp32
// accumulators in tensor memory; the softmax runs on the CUDA cores between them.
//
// Work unit = a cluster of two CTAs on two SMs (a CTA pair) sharing one key/value
// head.  Each CTA owns a tile of 128 query rows = (128 / G) positions x the G query
// heads of that key/value head; the pair's MMAs are M = 256 pair instructions
// (tcgen05 cta_group::2) issued by one thread of the even CTA.  Each CTA stages only
// half of every K/V tile (K: 64 of the 128 keys, V: 128 of the 256 columns), so a
// K/V byte fetched into shared memory serves 256 query rows: on B200 the TMA feed into
// shared memory, not the tensor core, bounds a single-CTA version of this kernel.
// K/V are never repeated in HBM.  320 threads per CTA, 1 CTA per SM.
//
// Tile shape.  Key tiles hold 128 keys, so every MMA has N >= 128: S = Q K^T is 16
// pair MMAs of M256 N128 K16 and O += P V is 8 of M256 N256 K16; one issuing thread
// keeps the tensor cores of both SMs busy at these sizes (measured).
//
// Tensor memory of each CTA (512 columns x 128 lanes, lane = query row):
//   [  0, 256)  O accumulator, fp32
//   [256, 512)  two S buffers of 128 fp32 columns; P(t) (bf16 pairs) overwrites the
//               first 64 columns of its S buffer and is the A operand of O += P V,
//               so P never touches shared memory.
// Shared memory of each CTA: its Q tile (64 KiB, four 64-column blocks) and a ring of
// five 32 KiB slots that a TMA producer fills in the order the issuer consumes them:
// a K slot is this CTA's 64 keys x 256 d (four 64-column blocks, K-major), a V slot
// 128 keys x this CTA's 128 d (two 64-column blocks, MN-major); all 128-byte
// swizzled.  The slot barriers that the issuer waits on live in the even CTA and
// count both CTAs' bytes.
//
// Copy count.  One SM's TMA engine completes about one bulk tensor copy per ~650
// cycles whatever its size between 4 and 32 KiB (measured on B200), so each slot is
// filled by a single copy of a 4-D view (d within a 64-column block, key, block,
// head): two copies per key tile per CTA instead of one per 64-column block.
//
// Issue order: S(0), then for each tile t: S(t+1), O += P(t) V(t).  S(t+1) runs on
// the tensor cores while the softmax of tile t runs on the CUDA cores.  MMAs from one
// thread execute in issue order, so S(t+2) (issued after PV(t)) never overwrites P(t)
// before PV(t) has read it, and the completion of S(t) implies that PV(t-2) has
// finished reading S buffer t & 1.
//
// Roles (both CTAs unless noted):
//   warp 0     TMA producer (Q once, then this CTA's halves of the slot ring).
//   warp 1     TMEM owner; in the even CTA lane 0 issues every MMA of the pair.
//   warps 2-9  softmax of this CTA's 128 rows, two warps per TMEM lane quarter (32
//              rows each): `half` 0 takes S columns 0-63 and O columns 0-127, `half` 1
//              the rest.  Per tile: load S, mask (partial tiles), row max exchanged
//              within the pair of warps, P = 2^(S*scale - m) as bf16 into TMEM, row
//              sum.  The running max m is raised only when it grows by more than 8
//              (log2): P <= 2^8 then, and O is rescaled in TMEM only on those rare
//              raises.  Epilogue: O / l to bf16, LSE in fp32.
#include "internal.h"
#include "tcgen05.cuh"

#include <cuda_bf16.h>

namespace gqa {
namespace {

constexpr int kRows = kBf16Rows;  // 128 query rows per CTA
constexpr int kBc = kBf16Bc;      // 128 keys per tile
constexpr int kThreads = 320;     // 10 warps
constexpr int kSlots = 5;
constexpr int kSlotBytes = 32768;      // this CTA's half of a K or V tile
constexpr int kQBlock = kRows * 128;   // 128 rows x 64 d bf16: 16 KiB
constexpr int kQBytes = 4 * kQBlock;   // 64 KiB
constexpr int kKHalf = kBc / 2;        // keys of a K tile held by each CTA
constexpr int kKBlock = kKHalf * 128;  // 64 keys x 64 d bf16: 8 KiB
constexpr int kVBlock = kBc * 128;     // 128 keys x 64 d bf16: 16 KiB
constexpr int kOffQ = 0;
constexpr int kOffRing = kOffQ + kQBytes;
constexpr int kOffBar = kOffRing + kSlots * kSlotBytes;
constexpr int kOffRed = kOffBar + 512;                   // [tile parity][half][row] fp32 exchange
constexpr int kSmemBytes = kOffRed + 2 * 2 * kRows * 4;  // dynamic smem is 1024-byte aligned
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 0;
constexpr uint32_t kTmemS = 256;  // buffer b at +128 b
constexpr uint16_t kPairMask = 0x3;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: P stays <= 256 between rescales

static_assert(kBc == 128, "the issue schedule assumes 128-key tiles");
static_assert(4 * kKBlock == kSlotBytes && 2 * kVBlock == kSlotBytes, "slot geometry");

// barrier indices (8 bytes each); Q, Full, PFull and Drain are used in the even CTA only
enum {
  kBarQ = 0,                       // both Q tiles landed (bytes of both CTAs)
  kBarFull = 1,                    // + slot: both halves landed
  kBarEmpty = kBarFull + kSlots,   // + slot: MMAs reading it completed (each CTA)
  kBarSFull = kBarEmpty + kSlots,  // + S buffer (each CTA)
  kBarPFull = kBarSFull + 2,       // + S buffer: 16 arrivals, P written in both CTAs
  kBarPVDone = kBarPFull + 2,      // + S buffer (each CTA)
  kBarDrain = kBarPVDone + 2,      // every MMA of the pair completed
  kNumBars = kBarDrain + 1
};
constexpr int kOffTmemSlot = kOffBar + 8 * kNumBars;
static_assert(kOffTmemSlot + 4 <= kOffBar + 512, "barrier area");
static_assert(kSmemBytes <= 232448, "shared memory per block");

// One query tile of the pair: rows [i0, i1], its id bounds and its key-tile range.
// A tile index past the last query tile (odd tile count) has no rows.
struct QTile {
  int64_t i0, i1;
  SegBounds qb;
  int kbeg, kend;
};

__device__ __forceinline__ QTile query_tile(const FwdParams& p, int qt) {
  QTile q;
  q.qb = SegBounds{0, 0};
  if (qt >= p.nq) {
    q.i0 = q.i1 = 0;
    q.kbeg = q.kend = 0;
    return q;
  }
  q.i0 = int64_t(qt) * p.br;
  q.i1 = min(p.Lq, q.i0 + p.br) - 1;
  if (p.has_seg) {
    q.qb = SegBounds{p.q_bounds[2 * qt], p.q_bounds[2 * qt + 1]};
    q.kbeg = p.q_ranges[2 * qt];
    q.kend = p.q_ranges[2 * qt + 1];
  } else {
    kv_range_no_seg(q.i1, p.off, kBc, p.nk, &q.kbeg, &q.kend);
  }
  return q;
}

// Class of key tile kt for one query tile (SKIP outside the tile's key range).
__device__ __forceinline__ int classify(const FwdParams& p, const QTile& q, int kt) {
  if (kt < q.kbeg || kt >= q.kend) return GQA_TILE_SKIP;
  const int64_t j0 = int64_t(kt) * kBc;
  const int64_t j1 = min(p.Lk, j0 + kBc) - 1;
  SegBounds kb{0, 0};
  if (p.has_seg) kb = SegBounds{p.kv_bounds[2 * kt], p.kv_bounds[2 * kt + 1]};
  return tile_class(q.i0, q.i1, j0, j1, p.off, p.P0, p.has_seg != 0, q.qb, kb);
}

// Bounded wait taken by a whole warp: every lane sees the same outcome, so the
// warp stays converged for the warp-collective operations that follow.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, int64_t budget, int32_t* status) {
  return __all_sync(0xffffffffu, mbar_wait_bounded_cluster(bar, parity, budget, status));
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

// The slot ring is consumed in a fixed order: K(t0), K(t1), V(t0), K(t2), V(t1), ...,
// K(t_last), V(t_prev), V(t_last) over the pair's non-skipped tiles t0, t1, ...; each
// K or V tile takes one slot.  Slot use u lands in slot u % kSlots, phase
// (u / kSlots) & 1.
struct Ring {
  uint32_t u = 0;
  __device__ __forceinline__ int slot() const { return int(u % kSlots); }
  __device__ __forceinline__ uint32_t phase() const { return (u / kSlots) & 1u; }
};

__global__ void __launch_bounds__(kThreads, 1)
fwd_bf16_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ FwdParams p) {
  extern __shared__ __align__(1024) char smem_raw[];
  const uint32_t sbase = smem_u32(smem_raw);
  // The swizzled tiles need 1024-byte alignment (never expected to fail).  A CTA of a
  // pair must not leave early: on failure it only skips its role.
  const bool misaligned = (sbase & 1023u) != 0;
  const uint32_t sQ = sbase + kOffQ, sRing = sbase + kOffRing;
  const uint32_t bar = sbase + kOffBar;
  auto B = [&](int i) { return bar + 8u * uint32_t(i); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0: the even CTA, which issues the MMAs
  const uint32_t lead_bar = mapa_shared(bar, 0);
  auto LB = [&](int i) { return lead_bar + 8u * uint32_t(i); };

  // Unit: (query-tile pair, kv head, batch); pairs in descending order so the longest
  // causal rows start first.
  const int pair = int(blockIdx.x >> 1);
  const int per_qp = p.Hkv * p.B;
  const int npairs = (p.nq + 1) / 2;
  const int qp = npairs - 1 - pair / per_qp;
  const int rem = pair % per_qp;
  const int g = rem % p.Hkv;
  const int b = rem / p.Hkv;
  const int br = p.br;
  const QTile own = query_tile(p, 2 * qp + int(rank));
  const QTile t0 = query_tile(p, 2 * qp), t1 = query_tile(p, 2 * qp + 1);
  int kbeg = 0x7fffffff, kend = 0;  // union of the two tiles' key ranges
  if (t0.kbeg < t0.kend) kbeg = t0.kbeg, kend = t0.kend;
  if (t1.kbeg < t1.kend) kbeg = min(kbeg, t1.kbeg), kend = max(kend, t1.kend);
  if (kbeg >= kend) kbeg = kend = 0;
  const int64_t q0 = int64_t(2 * qp + int(rank)) * br;  // first row of this CTA (may be >= Lq)
  // The pair computes a key tile unless it is SKIP for both query tiles.
  auto pair_skip = [&](int kt) {
    return classify(p, t0, kt) == GQA_TILE_SKIP && classify(p, t1, kt) == GQA_TILE_SKIP;
  };

  if (threadIdx.x == 0) {
    mbar_init(B(kBarQ), 1);
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(B(kBarFull + s), 1);
      mbar_init(B(kBarEmpty + s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(B(kBarSFull + s), 1);
      mbar_init(B(kBarPFull + s), 16);
      mbar_init(B(kBarPVDone + s), 1);
    }
    mbar_init(B(kBarDrain), 1);
    fence_barrier_init();
    if (misaligned) set_status(p.status, GQA_ERR_LAUNCH);
  }
  if (warp == 1) umma::tmem_alloc_2sm(sbase + kOffTmemSlot, kTmemCols);
  umma::fence_before_sync();
  cluster_sync();  // both CTAs' barriers initialised and TMEM allocated
  umma::fence_after_sync();
  uint32_t tmem;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(tmem) : "r"(sbase + kOffTmemSlot));

  const int64_t budget = p.wait_budget_ns;
  const bool leader = rank == 0;

  if (misaligned) {
    // no role: fall through to the final cluster barrier
  } else if (warp == 0) {
    // ---------------------------------------------------------------- TMA producers
    // Each CTA loads its own Q tile and its halves of the K/V tiles; completion is
    // counted on the even CTA's barriers, which its producer arms with both halves' bytes.
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      if (leader) mbar_arrive_expect_tx(B(kBarQ), 2 * kQBytes);
      tma_load_4d_pair(sQ, &tmQ, LB(kBarQ), 0, int(q0), b * p.Hq + g * p.G, 0);
      const int kvhead = b * p.Hkv + g;
      Ring ring;
      // One slot: wait until the MMAs that read its previous contents completed.
      auto acquire = [&](int* s) {
        *s = ring.slot();
        if (!mbar_wait_bounded(B(kBarEmpty + *s), ring.phase() ^ 1u, budget, p.status)) return false;
        if (leader) mbar_arrive_expect_tx(B(kBarFull + *s), 2 * kSlotBytes);
        return true;
      };
      auto load_k = [&](int kt) {  // this CTA's 64 keys x 256 d
        int s;
        if (!acquire(&s)) return false;
        tma_load_4d_pair(sRing + s * kSlotBytes, &tmK, LB(kBarFull + s), 0, kt * kBc + int(rank) * kKHalf, 0, kvhead);
        ++ring.u;
        return true;
      };
      auto load_v = [&](int kt) {  // 128 keys x this CTA's 128 d
        int s;
        if (!acquire(&s)) return false;
        tma_load_4d_pair(sRing + s * kSlotBytes, &tmV, LB(kBarFull + s), 0, kt * kBc, 2 * int(rank), kvhead);
        ++ring.u;
        return true;
      };
      bool ok = true;
      int prev = -1;
      for (int kt = kbeg; ok && kt < kend; ++kt) {
        if (pair_skip(kt)) continue;
        ok = load_k(kt);
        if (ok && prev >= 0) ok = load_v(prev);
        prev = kt;
      }
      if (ok && prev >= 0) load_v(prev);
      // No copy may be in flight when the pair ends.  The even CTA's barriers count
      // both CTAs' copies; the final cluster barrier holds the odd CTA until these
      // waits are over.
      if (leader) {
        mbar_wait_bounded_cluster(B(kBarQ), 0, budget, p.status);
        for (uint32_t i = ring.u > uint32_t(kSlots) ? ring.u - kSlots : 0u; i < ring.u; ++i)
          mbar_wait_bounded_cluster(B(kBarFull + int(i % kSlots)), (i / kSlots) & 1u, budget, p.status);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer (even CTA)
    if (lane == 0 && leader) {
      constexpr uint32_t id_s = umma::idesc_bf16(2 * kRows, kBc, 0, 0);
      constexpr uint32_t id_o = umma::idesc_bf16(2 * kRows, 256, 0, 1);
      const uint64_t dq = umma::smem_desc(sQ, 16, 1024);
      Ring ring;
      // S(t) = Q K(t)^T into S buffer t & 1: one K slot, four 64-column blocks of four
      // K16 steps.
      auto issue_s = [&](int t) {
        const uint32_t d = tmem + kTmemS + uint32_t((t & 1) * 128);
        const int s = ring.slot();
        if (!mbar_wait_bounded_cluster(B(kBarFull + s), ring.phase(), budget, p.status)) return false;
        umma::fence_after_sync();
        const uint64_t dk = umma::smem_desc(sRing + s * kSlotBytes, 16, 1024);
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int k = 0; k < 4; ++k)
            umma::mma_ss_2sm(d, umma::desc_add(dq, uint32_t(c * kQBlock + k * 32)),
                             umma::desc_add(dk, uint32_t(c * kKBlock + k * 32)), id_s, (c | k) != 0 ? 1u : 0u);
        umma::commit_2sm_mc(B(kBarEmpty + s), kPairMask);
        ++ring.u;
        umma::commit_2sm_mc(B(kBarSFull + (t & 1)), kPairMask);
        return true;
      };
      // O += P(t) V(t): A = P(t) in TMEM, one V slot of eight K16 steps (16 keys each).
      auto issue_pv = [&](int t) {
        const int sb = t & 1;
        if (!mbar_wait_bounded_cluster(B(kBarPFull + sb), (uint32_t(t) >> 1) & 1u, budget, p.status)) return false;
        const uint32_t a = tmem + kTmemS + uint32_t(sb * 128);
        const int s = ring.slot();
        if (!mbar_wait_bounded_cluster(B(kBarFull + s), ring.phase(), budget, p.status)) return false;
        umma::fence_after_sync();
        const uint64_t dv = umma::smem_desc(sRing + s * kSlotBytes, kVBlock, 1024);
#pragma unroll
        for (int k = 0; k < kBc / 16; ++k)
          umma::mma_ts_2sm(tmem + kTmemO, a + uint32_t(k * 8), umma::desc_add(dv, uint32_t(k * 2048)), id_o,
                           (t > 0 || k > 0) ? 1u : 0u);
        umma::commit_2sm_mc(B(kBarEmpty + s), kPairMask);
        ++ring.u;
        umma::commit_2sm_mc(B(kBarPVDone + sb), kPairMask);
        return true;
      };
      auto next_tile = [&](int kt) {
        while (kt < kend && pair_skip(kt)) ++kt;
        return kt;
      };
      bool ok = mbar_wait_bounded_cluster(B(kBarQ), 0, budget, p.status);
      int cur = next_tile(kbeg);
      if (ok && cur < kend) ok = issue_s(0);
      for (int t = 0; ok && cur < kend; ++t) {
        const int nxt = next_tile(cur + 1);
        if (nxt < kend) ok = issue_s(t + 1);
        if (ok) ok = issue_pv(t);
        cur = nxt;
      }
      // every MMA of the pair must be complete before TMEM is released
      umma::commit_2sm(B(kBarDrain));
      mbar_wait_bounded_cluster(B(kBarDrain), 0, budget, p.status);
    }
    __syncwarp();
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
      if (pair_skip(kt)) continue;
      const int cls = classify(p, own, kt);
      const int sb = t & 1;
      const uint32_t s_col = kTmemS + uint32_t(sb * 128 + half * 64);
      float xa[32], xb[32];
      // S(t) must be complete even when none of it is used: P(t) overwrites its buffer.
      const bool ok_s = ok && warp_wait(B(kBarSFull + sb), (uint32_t(t) >> 1) & 1u, budget, p.status);
      if (ok_s && cls != GQA_TILE_SKIP) {
        umma::fence_after_sync();
        umma::tmem_ld32(lane_addr + s_col, xa);
        umma::tmem_ld32(lane_addr + s_col + 32u, xb);
        umma::tmem_wait_ld();
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) xa[i] = xb[i] = -INFINITY;
      }
      const int64_t j0 = int64_t(kt) * kBc + half * 64;
      const bool need_mask = (cls == GQA_TILE_PARTIAL) || (cls == GQA_TILE_FULL && int64_t(kt) * kBc + kBc > p.Lk);
      if (need_mask) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int64_t ja = j0 + i, jb = j0 + 32 + i;
          bool va = ja <= pos, vb = jb <= pos;
          if (p.has_seg) {
            va = va && (ja < p.P0 || sq == __ldg(p.seg_kv + min(ja, p.Lk - 1)));
            vb = vb && (jb < p.P0 || sq == __ldg(p.seg_kv + min(jb, p.Lk - 1)));
          }
          if (!va) xa[i] = -INFINITY;
          if (!vb) xb[i] = -INFINITY;
        }
      }
      float m4[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) m4[u] = fmaxf(xa[u], xb[u]);
#pragma unroll
      for (int i = 4; i < 32; ++i) m4[i & 3] = fmaxf(m4[i & 3], fmaxf(xa[i], xb[i]));
      const float pm = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
      red[((t & 1) * 2 + half) * kRows + r] = pm;
      // Both halves have loaded their S columns once this barrier passes, so P may
      // now overwrite the first 64 columns of the buffer.
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
      uint32_t pk[32];
      float r4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int i = 0; i < 32; i += 2) {
        const float e0 = ex2_approx(fmaf(xa[i], p.scale_log2, neg_m));
        const float e1 = ex2_approx(fmaf(xa[i + 1], p.scale_log2, neg_m));
        pk[i / 2] = pack_bf16x2(e0, e1);
        r4[(i / 2) & 3] += e0 + e1;
      }
#pragma unroll
      for (int i = 0; i < 32; i += 2) {
        const float e0 = ex2_approx(fmaf(xb[i], p.scale_log2, neg_m));
        const float e1 = ex2_approx(fmaf(xb[i + 1], p.scale_log2, neg_m));
        pk[16 + i / 2] = pack_bf16x2(e0, e1);
        r4[(i / 2) & 3] += e0 + e1;
      }
      l = l * alpha + ((r4[0] + r4[1]) + (r4[2] + r4[3]));

      // O was last updated by PV(t-1): rescale it only after that MMA completed.
      const bool rescale = (alpha != 1.f) && (m_old != -INFINITY) && (t > 0);
      if (__any_sync(0xffffffffu, rescale)) {
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
        }
      }
      if (ok) {
        // P row r: keys half*64 .. +63 as bf16 pairs in columns half*32 .. +31 of the buffer.
        umma::tmem_st32u(lane_addr + kTmemS + uint32_t(sb * 128 + half * 32), pk);
        umma::tmem_wait_st();
        umma::fence_before_sync();
        __syncwarp();
        if (lane == 0) {
          if (leader)
            mbar_arrive(B(kBarPFull + sb));
          else
            mbar_arrive_remote(LB(kBarPFull + sb));
        }
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
  }

  // Neither CTA may release TMEM or leave while the pair's MMAs or copies may still
  // touch its memory: the issuer and the even CTA's producer have drained by now.
  umma::fence_before_sync();
  cluster_sync();
  if (warp == 1) {
    umma::fence_after_sync();
    umma::tmem_dealloc_2sm(tmem, kTmemCols);
  }
}

}  // namespace

int launch_fwd_bf16(const FwdTensors& t, const FwdParams& p, cudaStream_t stream) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return GQA_ERR_LAUNCH;
  CUtensorMap mq, mk, mv;
  // 4-D views whose innermost dimension is one 64-column (128-byte) block of d, so one
  // copy fills several blocks; the block dimension has a 128-byte stride.
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const cuuint64_t row = cuuint64_t(kHeadDim) * 2;  // bytes per token row
  {
    // (d in block, position, head, block): box = 128 rows (G heads x br positions) x 4 blocks
    const cuuint64_t dims[4] = {64, cuuint64_t(p.Lq), cuuint64_t(p.B) * p.Hq, 4};
    const cuuint64_t strides[3] = {row, cuuint64_t(p.Lq) * row, 128};
    const cuuint32_t box[4] = {64, cuuint32_t(p.br), cuuint32_t(p.G), 4};
    if (enc(&mq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(t.q), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return GQA_ERR_LAUNCH;
  }
  // (d in block, key, block, kv head): K box = 64 keys x 4 blocks, V box = 128 keys x 2 blocks
  const cuuint64_t dims[4] = {64, cuuint64_t(p.Lk), 4, cuuint64_t(p.B) * p.Hkv};
  const cuuint64_t strides[3] = {row, 128, cuuint64_t(p.Lk) * row};
  const cuuint32_t box_k[4] = {64, cuuint32_t(kKHalf), 4, 1};
  const cuuint32_t box_v[4] = {64, cuuint32_t(kBc), 2, 1};
  if (enc(&mk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(t.k), dims, strides, box_k, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return GQA_ERR_LAUNCH;
  if (enc(&mv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(t.v), dims, strides, box_v, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return GQA_ERR_LAUNCH;
  if (cudaFuncSetAttribute(fwd_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) != cudaSuccess)
    return GQA_ERR_LAUNCH;
  // Two CTAs (one cluster) per pair of query tiles.
  const int64_t units = 2 * ((int64_t(p.nq) + 1) / 2) * p.Hkv * p.B;
  if (units <= 0) return GQA_OK;
  if (units > 0x7fffffff) return GQA_ERR_UNSUPPORTED;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(units), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, fwd_bf16_kernel, mq, mk, mv, p) != cudaSuccess) return GQA_ERR_LAUNCH;
  return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_LAUNCH;
}

}  // namespace gqa
