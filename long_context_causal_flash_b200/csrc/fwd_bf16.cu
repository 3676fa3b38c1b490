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
// K/V are never repeated in HBM.  640 threads per CTA, 1 CTA per SM.
//
// Tile shape.  Key tiles hold 128 keys, so every MMA has N >= 128: S = Q K^T is 16
// pair MMAs of M256 N128 K16 and O += P V is 8 of M256 N256 K16 (N = 64 MMAs reach
// about two thirds of the tensor cores' rate, measured).
//
// Tensor memory of each CTA (512 columns x 128 lanes, lane = query row):
//   [  0, 256)  O accumulator, fp32
//   [256, 512)  two S buffers of 128 fp32 columns; P(t) (bf16 pairs) overwrites the
//               first 64 columns of its S buffer and is the A operand of O += P V,
//               so P never touches shared memory.
// Shared memory of each CTA: its Q tile (64 KiB, four 64-column blocks) and five
// 32 KiB slots (a 2-slot K ring and a 3-slot V ring) that TMA producers fill: a K
// slot is this CTA's 64 keys x 256 d (four 64-column blocks, K-major), a V slot 128
// keys x this CTA's 128 d (two 64-column blocks, MN-major); all 128-byte swizzled.
// The slot barriers that the issuers wait on live in the even CTA and count both
// CTAs' bytes.
//
// Copy count.  One SM's TMA engine completes about one bulk tensor copy per ~650
// cycles whatever its size between 4 and 32 KiB (measured on B200), so each slot is
// filled by a single copy of a 4-D view (d within a 64-column block, key, block,
// head): two copies per key tile per CTA instead of one per 64-column block.
//
// Two issuing threads.  One thread issues every S(t) = Q K(t)^T, another every
// O += P(t) V(t) (a single thread cannot issue a pair MMA much faster than the tensor
// cores run an N = 128 one, so one issuer serialises its waits with the issue time).
// S(t) waits for PV(t-2), which read P(t-2) from the same S buffer; with two S
// buffers, S(t+1) then runs on the tensor cores while the softmax of tile t runs on
// the CUDA cores, and the PVs are ordered among themselves by their single thread.
//
// Roles (both CTAs unless noted):
//   warp 0     TMA producer of Q (once) and of this CTA's K halves (2-slot ring).
//   warp 3     TMA producer of this CTA's V halves (3-slot ring).
//   warp 1     TMEM owner; in the even CTA lane 0 issues every S MMA of the pair.
//   warp 2     in the even CTA lane 0 issues every PV MMA of the pair.
//   warps 4-19 softmax of this CTA's 128 rows, four warps per TMEM lane quarter (32
//              rows each), each with 32 of the 128 S columns and 64 of the 256 O
//              columns.  Per tile: load S, mask (partial tiles), P = 2^(S*scale - m)
//              as bf16 into TMEM, row sum.  The running max m is raised only when a
//              row's max grows by more than 8 (log2): P <= 2^8 then, and O is rescaled
//              in TMEM only on those rare raises.  Epilogue: O / l to bf16, LSE in fp32.
#include "internal.h"
#include "tcgen05.cuh"

#include <cuda_bf16.h>

namespace gqa {
namespace {

constexpr int kRows = kBf16Rows;  // 128 query rows per CTA
constexpr int kBc = kBf16Bc;      // 128 keys per tile
constexpr int kThreads = 640;     // 20 warps
constexpr int kKSlots = 2, kVSlots = 3;
constexpr int kSlotBytes = 32768;      // this CTA's half of a K or V tile
constexpr int kQBlock = kRows * 128;   // 128 rows x 64 d bf16: 16 KiB
constexpr int kQBytes = 4 * kQBlock;   // 64 KiB
constexpr int kKHalf = kBc / 2;        // keys of a K tile held by each CTA
constexpr int kKBlock = kKHalf * 128;  // 64 keys x 64 d bf16: 8 KiB
constexpr int kVBlock = kBc * 128;     // 128 keys x 64 d bf16: 16 KiB
constexpr int kOffQ = 0;
constexpr int kOffRing = kOffQ + kQBytes;
constexpr int kOffBar = kOffRing + (kKSlots + kVSlots) * kSlotBytes;
constexpr int kOffRed = kOffBar + 512;               // [part][row] fp32 exchange
constexpr int kSmemBytes = kOffRed + 4 * kRows * 4;  // dynamic smem is 1024-byte aligned
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 0;
constexpr uint32_t kTmemS = 256;  // buffer b at +128 b
constexpr uint16_t kPairMask = 0x3;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: P stays <= 256 between rescales

static_assert(kBc == 128, "the issue schedule assumes 128-key tiles");
static_assert(4 * kKBlock == kSlotBytes && 2 * kVBlock == kSlotBytes, "slot geometry");

// barrier indices (8 bytes each); Q, Full, PFull and Drain are used in the even CTA only
enum {
  kBarQ = 0,                          // both Q tiles landed (bytes of both CTAs)
  kBarKFull = 1,                      // + K slot: both halves landed
  kBarKEmpty = kBarKFull + kKSlots,   // + K slot: MMAs reading it completed (each CTA)
  kBarVFull = kBarKEmpty + kKSlots,   // + V slot
  kBarVEmpty = kBarVFull + kVSlots,   // + V slot (each CTA)
  kBarSFull = kBarVEmpty + kVSlots,   // + S buffer (each CTA)
  kBarPFull = kBarSFull + 2,          // + S buffer: 32 arrivals, P written in both CTAs
  kBarPVDone = kBarPFull + 2,         // + S buffer (each CTA)
  kBarDrain = kBarPVDone + 2,         // 2 arrivals: both issuers' MMAs completed
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
  return __all_sync(0xffffffffu, mbar_wait_inline(bar, parity, budget, status));
}

// Named barriers over the 128 threads (four warps) of one TMEM lane quarter.
__device__ __forceinline__ void quad_sync(uint32_t id) { asm volatile("bar.sync %0, 128;" ::"r"(id) : "memory"); }

// Number of the quarter's threads whose `pred` is true.
__device__ __forceinline__ uint32_t quad_popc(uint32_t id, bool pred) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.popc.u32 %0, %2, 128, p;\n\t}"
      : "=r"(out)
      : "r"(uint32_t(pred)), "r"(id)
      : "memory");
  return out;
}

// AND of `pred` over the quarter's threads, so all four warps take the same branch.
__device__ __forceinline__ bool quad_and(uint32_t id, bool pred) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, 128, p;\n\t"
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

__global__ void __launch_bounds__(kThreads, 1)
fwd_bf16_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ FwdParams p) {
  extern __shared__ __align__(1024) char smem_raw[];
  const uint32_t sbase = smem_u32(smem_raw);
  // The swizzled tiles need 1024-byte alignment (never expected to fail).  A CTA of a
  // pair must not leave early: on failure it only skips its role.
  const bool misaligned = (sbase & 1023u) != 0;
  const uint32_t sQ = sbase + kOffQ, sKRing = sbase + kOffRing, sVRing = sKRing + kKSlots * kSlotBytes;
  const uint32_t bar = sbase + kOffBar;
  auto B = [&](int i) { return bar + 8u * uint32_t(i); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0: the even CTA, which issues the MMAs
  const uint32_t lead_bar = mapa_shared(bar, 0);
  auto LB = [&](int i) { return lead_bar + 8u * uint32_t(i); };

  // Unit: (query-tile pair, kv head, batch[, key split]), ordered kv head by kv head
  // and, within one, pairs in descending order so the longest causal rows start
  // first.  The pairs resident together then share one kv head's K/V (62 MB in bf16
  // at L = 60,926, inside the L2) and sweep it a few tiles apart.
  const int splits = p.splits > 1 ? p.splits : 1;
  const int split = int(blockIdx.x >> 1) % splits;
  const int pair = int(blockIdx.x >> 1) / splits;
  const int npairs = (p.nq + 1) / 2;
  const int qp = npairs - 1 - pair % npairs;
  const int hb = pair / npairs;  // b * Hkv + g
  const int g = hb % p.Hkv;
  const int b = hb / p.Hkv;
  const int br = p.br;
  const QTile own = query_tile(p, 2 * qp + int(rank));
  const QTile t0 = query_tile(p, 2 * qp), t1 = query_tile(p, 2 * qp + 1);
  int kbeg = 0x7fffffff, kend = 0;  // union of the two tiles' key ranges
  if (t0.kbeg < t0.kend) kbeg = t0.kbeg, kend = t0.kend;
  if (t1.kbeg < t1.kend) kbeg = min(kbeg, t1.kbeg), kend = max(kend, t1.kend);
  if (kbeg >= kend) kbeg = kend = 0;
  split_range(split, splits, &kbeg, &kend);
  const int64_t q0 = int64_t(2 * qp + int(rank)) * br;  // first row of this CTA (may be >= Lq)
  // The pair computes a key tile unless it is SKIP for both query tiles.  Without
  // segment ids every tile of [kbeg, kend) holds a key visible to the last row.
  auto pair_skip = [&](int kt) {
    return p.has_seg && classify(p, t0, kt) == GQA_TILE_SKIP && classify(p, t1, kt) == GQA_TILE_SKIP;
  };

  if (threadIdx.x == 0) {
    mbar_init(B(kBarQ), 1);
    for (int s = 0; s < kKSlots; ++s) {
      mbar_init(B(kBarKFull + s), 1);
      mbar_init(B(kBarKEmpty + s), 1);
    }
    for (int s = 0; s < kVSlots; ++s) {
      mbar_init(B(kBarVFull + s), 1);
      mbar_init(B(kBarVEmpty + s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(B(kBarSFull + s), 1);
      mbar_init(B(kBarPFull + s), 32);
      mbar_init(B(kBarPVDone + s), 1);
    }
    mbar_init(B(kBarDrain), 2);
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
  } else if (warp == 0 || warp == 3) {
    // ---------------------------------------------------------------- TMA producers
    // Warp 0 loads Q and the K ring, warp 3 the V ring.  Each CTA loads its own Q tile
    // and its halves of the K/V tiles; completion is counted on the even CTA's
    // barriers, which its producers arm with both halves' bytes.
    if (lane == 0) {
      const bool is_k = warp == 0;
      const CUtensorMap* map = is_k ? &tmK : &tmV;
      tma_prefetch_desc(map);
      const int kvhead = b * p.Hkv + g;
      if (is_k) {
        tma_prefetch_desc(&tmQ);
        if (leader) mbar_arrive_expect_tx(B(kBarQ), 2 * kQBytes);
        tma_load_4d_pair(sQ, &tmQ, LB(kBarQ), 0, int(q0), b * p.Hq + g * p.G, 0);
      }
      const int nslots = is_k ? kKSlots : kVSlots;
      const int bar_full = is_k ? kBarKFull : kBarVFull;
      const int bar_empty = is_k ? kBarKEmpty : kBarVEmpty;
      const uint32_t ring = is_k ? sKRing : sVRing;
      uint32_t u = 0;  // fills issued
      for (int kt = kbeg; kt < kend; ++kt) {
        if (pair_skip(kt)) continue;
        const int s = int(u % uint32_t(nslots));
        // wait until the MMAs that read the slot's previous contents completed
        if (!mbar_wait_inline(B(bar_empty + s), ((u / uint32_t(nslots)) & 1u) ^ 1u, budget, p.status)) break;
        if (is_k && int(u) == p.test_skip_fill) {  // test hook: both CTAs skip this fill
          ++u;
          continue;
        }
        if (leader) mbar_arrive_expect_tx(B(bar_full + s), 2 * kSlotBytes);
        if (is_k)  // this CTA's 64 keys x 256 d
          tma_load_4d_pair(ring + s * kSlotBytes, map, LB(bar_full + s), 0, kt * kBc + int(rank) * kKHalf, 0, kvhead);
        else  // 128 keys x this CTA's 128 d
          tma_load_4d_pair(ring + s * kSlotBytes, map, LB(bar_full + s), 0, kt * kBc, 2 * int(rank), kvhead);
        ++u;
      }
      // No copy may be in flight when the pair ends.  The even CTA's barriers count
      // both CTAs' copies; the final cluster barrier holds the odd CTA until these
      // waits are over.
      if (leader) {
        if (is_k) mbar_wait_inline(B(kBarQ), 0, budget, p.status);
        for (uint32_t i = u > uint32_t(nslots) ? u - nslots : 0u; i < u; ++i)
          mbar_wait_inline(B(bar_full + int(i % uint32_t(nslots))), (i / uint32_t(nslots)) & 1u, budget,
                                    p.status);
      }
    }
    __syncwarp();
  } else if (warp == 1 || warp == 2) {
    // ---------------------------------------------------------------- MMA issuers (even CTA)
    // Warp 1 issues every S = Q K^T, warp 2 every O += P V.  MMAs of different threads
    // are not ordered, so S(t) waits for PV(t-2) to complete before it overwrites the
    // S buffer that held P(t-2); the PVs are ordered among themselves (one thread).
    if (lane == 0 && leader) {
      const bool is_s = warp == 1;
      constexpr uint32_t id_s = umma::idesc_bf16(2 * kRows, kBc, 0, 0);
      constexpr uint32_t id_o = umma::idesc_bf16(2 * kRows, 256, 0, 1);
      const uint64_t dq = umma::smem_desc(sQ, 16, 1024);
      bool ok = !is_s || mbar_wait_inline(B(kBarQ), 0, budget, p.status);
      int t = 0;
      for (int kt = kbeg; ok && kt < kend; ++kt) {
        if (pair_skip(kt)) continue;
        const int sb = t & 1;
        if (is_s) {
          // S(t) into S buffer t & 1: one K slot, four 64-column blocks of four K16 steps.
          const int s = t % kKSlots;
          if (!(ok = mbar_wait_inline(B(kBarKFull + s), uint32_t(t / kKSlots) & 1u, budget, p.status))) break;
          if (t >= 2 && !(ok = mbar_wait_inline(B(kBarPVDone + sb), (uint32_t(t - 2) >> 1) & 1u, budget,
                                                         p.status)))
            break;
          umma::fence_after_sync();
          const uint32_t d = tmem + kTmemS + uint32_t(sb * 128);
          const uint64_t dk = umma::smem_desc(sKRing + s * kSlotBytes, 16, 1024);
#pragma unroll
          for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int k = 0; k < 4; ++k)
              umma::mma_ss_2sm(d, umma::desc_add(dq, uint32_t(c * kQBlock + k * 32)),
                               umma::desc_add(dk, uint32_t(c * kKBlock + k * 32)), id_s, (c | k) != 0 ? 1u : 0u);
          umma::commit_2sm_mc(B(kBarKEmpty + s), kPairMask);
          umma::commit_2sm_mc(B(kBarSFull + sb), kPairMask);
        } else {
          // O += P(t) V(t): A = P(t) in TMEM, one V slot of eight K16 steps (16 keys each).
          const int s = t % kVSlots;
          if (!(ok = mbar_wait_inline(B(kBarPFull + sb), (uint32_t(t) >> 1) & 1u, budget, p.status))) break;
          if (!(ok = mbar_wait_inline(B(kBarVFull + s), uint32_t(t / kVSlots) & 1u, budget, p.status))) break;
          umma::fence_after_sync();
          const uint32_t a = tmem + kTmemS + uint32_t(sb * 128);
          const uint64_t dv = umma::smem_desc(sVRing + s * kSlotBytes, kVBlock, 1024);
#pragma unroll
          for (int k = 0; k < kBc / 16; ++k)
            umma::mma_ts_2sm(tmem + kTmemO, a + uint32_t(k * 8), umma::desc_add(dv, uint32_t(k * 2048)), id_o,
                             (t > 0 || k > 0) ? 1u : 0u);
          umma::commit_2sm_mc(B(kBarVEmpty + s), kPairMask);
          umma::commit_2sm_mc(B(kBarPVDone + sb), kPairMask);
        }
        ++t;
      }
      // every MMA of the pair must be complete before TMEM is released
      umma::commit_2sm(B(kBarDrain));
      mbar_wait_inline(B(kBarDrain), 0, budget, p.status);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- softmax warps
    // Four warps share each TMEM lane quarter (32 rows); `part` p takes S columns
    // 32p .. 32p+31 (keys), writes P columns 16p .. 16p+15 and owns O columns 64p ..
    // 64p+63.  The running max m_ref is raised only when a row's max grows by more
    // than kRescaleThreshold, so the exponentials are computed with the current m_ref
    // before the four warps compare notes: one counting barrier per tile tells whether
    // any row of the quarter needs a raise (rare; the row maxima are then exchanged
    // through shared memory and the tile recomputed) or any wait ran out.  The same
    // barrier guarantees that all four warps have loaded S before P overwrites it.
    const int quarter = warp & 3;       // TMEM lane quarter this warp may access
    const int part = (warp - 4) >> 2;   // 0..3
    const int r = quarter * 32 + lane;  // query row of the tile = TMEM lane
    const uint32_t lane_addr = tmem + (uint32_t(quarter * 32) << 16);
    const uint32_t quad_bar = 1u + uint32_t(quarter);
    float* red = reinterpret_cast<float*>(smem_raw + kOffRed);  // [part][row]
    const int hh = r / br, pp = r % br;
    const int64_t qi = q0 + pp;
    const bool live = qi < p.Lq;
    const int head = b * p.Hq + g * p.G + hh;
    // the last key this row sees: its position, or the block's last key when the key
    // block ends before it (a block of a sharded sequence)
    const int64_t pos = min(qi + p.off, p.Lk - 1);
    const int sq = p.has_seg ? p.seg_q[min(qi, p.Lq - 1)] : 0;

    float m_ref = -INFINITY;  // running max (log2 units), raised lazily; same in all parts
    float l = 0.f;            // this part's share of the row sum
    int t = 0;
    bool ok = true;
    for (int kt = kbeg; kt < kend; ++kt) {
      if (pair_skip(kt)) continue;
      const int cls = classify(p, own, kt);
      const int sb = t & 1;
      float x[32];
      // S(t) must be complete even when none of it is used: P(t) overwrites its buffer.
      const bool ok_s = ok && warp_wait(B(kBarSFull + sb), (uint32_t(t) >> 1) & 1u, budget, p.status);
      if (ok_s && cls != GQA_TILE_SKIP) {
        umma::fence_after_sync();
        umma::tmem_ld32(lane_addr + kTmemS + uint32_t(sb * 128 + part * 32), x);
        umma::tmem_wait_ld();
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) x[i] = -INFINITY;
      }
      const int64_t j0 = int64_t(kt) * kBc + part * 32;
      const bool need_mask = (cls == GQA_TILE_PARTIAL) || (cls == GQA_TILE_FULL && int64_t(kt) * kBc + kBc > p.Lk);
      if (need_mask) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int64_t j = j0 + i;
          bool vis = j <= pos;
          if (p.has_seg) vis = vis && (j < p.P0 || sq == __ldg(p.seg_kv + min(j, p.Lk - 1)));
          if (!vis) x[i] = -INFINITY;
        }
      }
      float m4[4] = {x[0], x[1], x[2], x[3]};
#pragma unroll
      for (int i = 4; i < 32; ++i) m4[i & 3] = fmaxf(m4[i & 3], x[i]);
      const float pm = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * p.scale_log2;
      // Exponentials with the current reference, before the quarter agrees on it.
      uint32_t pk[16];
      float rs;
      auto exps = [&](float m) {
        const float neg_m = m == -INFINITY ? 0.f : -m;
        float r4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const float e0 = ex2_approx(fmaf(x[i], p.scale_log2, neg_m));
          const float e1 = ex2_approx(fmaf(x[i + 1], p.scale_log2, neg_m));
          pk[i / 2] = pack_bf16x2(e0, e1);
          r4[(i / 2) & 3] += e0 + e1;
        }
        rs = (r4[0] + r4[1]) + (r4[2] + r4[3]);
      };
      exps(m_ref);
      const bool raise_here = pm > m_ref + kRescaleThreshold;  // also true for the first visible key
      float alpha = 1.f;
      const float m_old = m_ref;
      if (quad_popc(quad_bar, !ok_s || raise_here) != 0) {
        // Rare path: agree on the outcome of the waits, then on every row's maximum.
        red[part * kRows + r] = pm;
        if (!quad_and(quad_bar, ok_s)) {
          ok = false;
          break;
        }
        const float mx = fmaxf(fmaxf(red[r], red[kRows + r]), fmaxf(red[2 * kRows + r], red[3 * kRows + r]));
        if (mx > m_ref + kRescaleThreshold) {
          alpha = ex2_approx(m_ref - mx);  // 0 when m_ref = -inf
          m_ref = mx;
          exps(m_ref);
        }
      }
      l = l * alpha + rs;

      // O was last updated by PV(t-1): rescale it only after that MMA completed.
      const bool rescale = (alpha != 1.f) && (m_old != -INFINITY) && (t > 0);
      if (__any_sync(0xffffffffu, rescale)) {
        const int tp = t - 1;
        ok = warp_wait(B(kBarPVDone + (tp & 1)), (uint32_t(tp) >> 1) & 1u, budget, p.status);
        if (ok) {
          umma::fence_after_sync();
#pragma unroll 1
          for (int c0 = part * 64; c0 < part * 64 + 64; c0 += 32) {
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
        // P row r: keys 32*part .. +31 as bf16 pairs in columns 16*part .. +15 of the buffer.
        umma::tmem_st16u(lane_addr + kTmemS + uint32_t(sb * 128 + part * 16), pk);
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
    // Row sum = the four parts' shares.  The first barrier keeps every read of the
    // exchange buffer in the loop ahead of the writes below.
    if (quad_and(quad_bar, ok)) {
      red[part * kRows + r] = l;
      quad_sync(quad_bar);
      l = (red[r] + red[kRows + r]) + (red[2 * kRows + r] + red[3 * kRows + r]);
      // One key split writes its normalised partial output (fp32) and log-sum-exp.
      const int64_t row = int64_t(head) * p.Lq + (live ? qi : 0);
      const int64_t plane = int64_t(p.B) * p.Hq * p.Lq;
      __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out);
      uint4* dst = reinterpret_cast<uint4*>(out + row * kHeadDim);
      float4* dst_part = splits > 1 ? reinterpret_cast<float4*>(p.o_part + (split * plane + row) * kHeadDim) : nullptr;
      float* lse_out = splits > 1 ? p.lse_part + split * plane : p.lse;
      const float inv = l > 0.f ? 1.f / l : 0.f;
      if (t > 0) {
        const int tl = t - 1;
        ok = warp_wait(B(kBarPVDone + (tl & 1)), (uint32_t(tl) >> 1) & 1u, budget, p.status);
        umma::fence_after_sync();
      }
      if (ok) {
#pragma unroll 1
        for (int c0 = part * 64; c0 < part * 64 + 64; c0 += 32) {
          float o[32];
          if (t > 0) {
            umma::tmem_ld32(lane_addr + kTmemO + uint32_t(c0), o);
            umma::tmem_wait_ld();
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = 0.f;
          }
          if (live && splits > 1) {
#pragma unroll
            for (int v4 = 0; v4 < 8; ++v4)
              dst_part[c0 / 4 + v4] =
                  make_float4(o[4 * v4] * inv, o[4 * v4 + 1] * inv, o[4 * v4 + 2] * inv, o[4 * v4 + 3] * inv);
          } else if (live) {
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
        if (live && part == 0) lse_out[int64_t(head) * p.Lq + qi] = l > 0.f ? (m_ref + log2f(l)) * kLn2 : -INFINITY;
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
  const int64_t units = 2 * ((int64_t(p.nq) + 1) / 2) * p.Hkv * p.B * (p.splits > 1 ? p.splits : 1);
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
