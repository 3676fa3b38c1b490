// bf16 attention backward on the 5th-generation tensor cores (tcgen05 / TMEM), sm_100a.
//
// Training over packed long sequences (maxtext PR #4929, description: the splash
// kernel runs inside training steps on 1,048,576-token packed batches) needs dQ, dK
// and dV.  From the forward's log-sum-exp, with D_i = <dO_i, O_i>:
//     P = exp(scale * Q K^T - LSE),  dP = dO V^T,  dS = P * (dP - D),
//     dQ = scale * dS K,  dK = scale * dS^T Q,  dV = P^T dO   (summed over the group).
// Every product is a dense contraction with d = 256, so all of them run on tcgen05.mma
// with fp32 accumulators in tensor memory; P and dS are rounded to bf16 as the A
// operands of the accumulating products (the forward does the same with P).
//
// Tensor memory decides the split.  A 256-column fp32 accumulator (one row per TMEM
// lane) plus two 128-column tiles already fill the 512 columns, so one kernel cannot
// hold both dK and dV.  Three kernels, no atomics:
//   dQ: rows = a query tile,   columns = key tiles:   S, dP, dQ += dS K
//   dK: rows = a key tile,     columns = query tiles: S^T, dP^T, dK += dS^T Q
//   dV: rows = a key tile,     columns = query tiles: S^T, dV += P^T dO
// (8 GEMM-equivalents per visible block instead of 5; the FFMA version of this
// backward computes 7.)  One template covers the three.
//
// Work unit = a cluster of two CTAs on two SMs (a CTA pair): each CTA owns 128 rows
// and the pair issues M = 256 pair MMAs (cta_group::2) from the even CTA.  A query tile
// holds 128 rows = (128 / G) positions x the G query heads of one key/value head; a
// key tile 128 keys.  Shared memory of each CTA:
//   A1, A2  the row tile's two resident operands, 64 KiB each (dQ: Q and dO; dK: K
//           and V; dV: K only), four 64-column blocks of 128 rows, K-major.
//   B1, B2  this CTA's half (64 of the 128 columns) of the column tile's operands of
//           S and dP, 32 KiB each (dQ: K and V; dK: Q and dO; dV: Q), K-major.
//   B3      all 128 columns x this CTA's 128 of the 256 d of the accumulating
//           product's B operand, 32 KiB (dQ: K; dK: Q; dV: dO), MN-major.
// dQ / dK hold one slot of each B operand (224 KiB in all); dV two slots of B1 and
// B3.  Everything is 128-byte swizzled and filled by single 4-D TMA copies.
//
// Tensor memory of each CTA (128 lanes = rows):
//   [  0, 256)  accumulator (dQ, dK or dV), fp32
//   [256, 384), [384, 512)  two regions; column tile t lives in region t % 2: S(t),
//               then (dQ / dK) dP(t) over it once every elementwise thread holds S(t)
//               in registers, then dS(t) (P(t) for dV) as bf16 pairs, which the
//               accumulation of tile t reads.  Tile t + 2 reuses the region.
// The elementwise thread that read 32 columns of a row writes their 16 packed bf16
// columns over the first half of the same 32, so no other thread's data is touched.
//
// Issue.  One thread cannot issue N = 128 pair MMAs as fast as the tensor cores run
// them (about 88 cycles each against 64, measured on B200), so S, dP and the
// accumulating product have an issuing thread each (dV: two).  Hazards between them:
//   S(t)   waits until the accumulation of tile t-2 (same region) completed;
//   dP(t)  waits until every elementwise thread has loaded S(t);
//   acc(t) waits until dS(t) (P(t)) is written by both CTAs.
// So dP(t+1) does not wait for acc(t), and while the elementwise warps compute the
// exponentials of tile t the tensor cores run dP(t), acc(t-1) and S(t+1).
//
// Roles (both CTAs unless noted):
//   warp 0      TMA: lane 0 A1 (+A2) once, then the B1 ring; lane 1 the B2 and B3
//               rings (two producers in one warp keep the CTA at 20 warps, 5 per SM
//               sub-partition, and so at 96 registers per thread).
//   warp 1      TMEM owner; even CTA lane 0 issues S.
//   warp 2      even CTA lane 0 issues the accumulating product.
//   warp 3      even CTA lane 0 issues dP (dQ / dK only).
//   warps 4-19  elementwise: TMEM lane quarter warp % 4, columns 32 * ((warp - 4) / 4)
//               .. +31 of S / dP and 64 of the 256 accumulator columns.
#include "internal.h"
#include "tcgen05.cuh"

#include <cuda_bf16.h>

namespace gqa {
namespace {

enum { kModeDQ = 0, kModeDK = 1, kModeDV = 2 };

constexpr int kRows = 128;           // rows per CTA
constexpr int kCols = 128;           // columns per column tile
constexpr int kThreads = 640;        // 20 warps
constexpr int kABytes = 65536;       // 128 rows x 256 d bf16
constexpr int kABlock = 16384;       // 128 rows x 64 d
constexpr int kBBytes = 32768;       // one B slot
constexpr int kBHalfBlock = 8192;    // B1 / B2: 64 rows x 64 d
constexpr int kB3Block = 16384;      // B3: 128 rows x 64 d
constexpr int kColBytes = 1024;      // D and log2-LSE of the 128 columns of a query tile
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemAcc = 0, kTmemS = 256;  // two 128-column regions from kTmemS
constexpr uint16_t kPairMask = 0x3;

template <int kMode>
struct Geo {
  static constexpr bool kDP = kMode != kModeDV;  // dP and dS (dQ, dK)
  static constexpr int kNA = kDP ? 2 : 1;
  static constexpr int kS1 = kDP ? 1 : 2;  // slots of B1, B2, B3
  static constexpr int kS2 = kDP ? 1 : 0;
  static constexpr int kS3 = kDP ? 1 : 2;
  static constexpr int kOffA = 0;
  static constexpr int kOffB1 = kNA * kABytes;
  static constexpr int kOffB2 = kOffB1 + kS1 * kBBytes;
  static constexpr int kOffB3 = kOffB2 + kS2 * kBBytes;
  static constexpr int kOffBar = kOffB3 + kS3 * kBBytes;
  static constexpr int kOffCol = kOffBar + 512;  // dK / dV: 2 slots of a query tile's D and LSE
  static constexpr int kSmem = kOffCol + (kMode == kModeDQ ? 0 : 2 * kColBytes);
  static constexpr int kIssuers = kDP ? 3 : 2;
  static_assert(kSmem <= 232448, "shared memory per block");
};

// barrier indices (8 bytes each).  Full / SFree / PFull / DSReady / Drain and A are
// counted in the even CTA; Empty / SFull / DPFull / AccDone are signalled in both.
enum {
  kBarA = 0,
  kBarB1Full = 1,     // + slot (2)
  kBarB1Empty = 3,    // + slot (2)
  kBarB2Full = 5,
  kBarB2Empty = 6,
  kBarB3Full = 7,     // + slot (2)
  kBarB3Empty = 9,    // + slot (2)
  kBarSFull = 11,     // + region (2)
  kBarSFree = 13,     // + region (2), 32 arrivals: every elementwise warp of the pair loaded S
  kBarPFull = 15,     // + region (2), 32 arrivals: P written (dV)
  kBarDPFull = 17,    // + region (2)
  kBarDSReady = 19,   // + region (2), 32 arrivals: dS written
  kBarAccDone = 21,   // + region (2): the accumulation that read the region completed
  kBarDrain = 23,
  kBarColFull = 24,   // + slot (2): this CTA's copy of a query tile's column state landed
  kBarColEmpty = 26,  // + slot (2): 16 arrivals, this CTA's elementwise warps are done with it
  kNumBars = 28
};
constexpr int kOffTmemSlot = 8 * kNumBars;  // within the barrier area
constexpr int kOffRange = kOffTmemSlot + 8;
static_assert(kOffRange + 8 <= 512, "barrier area");

struct TcParams {
  __nv_bfloat16* dst;  // dq [B, Hq, Lq, d], or dk / dv [B, Hkv, Lk, d]
  const float* L2;     // [B * Hq][Lqp]: log2-domain LSE, +inf where a row takes no part
  const float* D;      // [B * Hq][Lqp]: rowsum(dO * O), 0 past Lq
  const int32_t* seg_q;
  const int32_t* seg_kv;
  const int32_t* q_bounds;   // plan at (br, 128) tiles, or null
  const int32_t* kv_bounds;
  const int32_t* q_ranges;
  int32_t* status;
  int64_t Lq, Lk, Lqp, off, P0, wait_budget_ns;
  int B, Hq, Hkv, G, br, nq, nk, has_seg;
  int test_skip_fill;  // test hook: the first producer lane skips its fill n of ring B1 (-1: off)
  float scale_log2, out_scale;
};

// Class of the block (query tile qt, key tile kt); SKIP outside the tile grid.
__device__ __forceinline__ int block_class(const TcParams& p, int qt, int kt) {
  if (qt < 0 || qt >= p.nq || kt < 0 || kt >= p.nk) return GQA_TILE_SKIP;
  const int64_t i0 = int64_t(qt) * p.br, i1 = min(p.Lq, i0 + p.br) - 1;
  const int64_t j0 = int64_t(kt) * kCols, j1 = min(p.Lk, j0 + kCols) - 1;
  SegBounds qb{0, 0}, kb{0, 0};
  if (p.has_seg) {
    qb = SegBounds{p.q_bounds[2 * qt], p.q_bounds[2 * qt + 1]};
    kb = SegBounds{p.kv_bounds[2 * kt], p.kv_bounds[2 * kt + 1]};
  }
  return tile_class(i0, i1, j0, j1, p.off, p.P0, p.has_seg != 0, qb, kb);
}

// Key-tile range [first, end) of query tile qt (empty past the last tile).
__device__ __forceinline__ void key_range(const TcParams& p, int qt, int* first, int* end) {
  *first = *end = 0;
  if (qt >= p.nq) return;
  if (p.has_seg) {
    *first = p.q_ranges[2 * qt];
    *end = p.q_ranges[2 * qt + 1];
  } else {
    kv_range_no_seg(min(p.Lq, int64_t(qt) * p.br + p.br) - 1, p.off, kCols, p.nk, first, end);
  }
}

__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, int64_t budget, int32_t* status) {
  return __all_sync(0xffffffffu, mbar_wait_inline(bar, parity, budget, status));
}

// 2^x on the MUFU unit (PTX ex2.approx.ftz.f32): 2^-inf = 0.
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// TMEM column (bf16 pairs) of K16 step k of the packed P / dS tile: the thread of
// part q packed keys 32q .. 32q+31 into columns 32q .. 32q+15.
__device__ __forceinline__ uint32_t packed_col(int k) { return uint32_t(32 * (k >> 1) + 8 * (k & 1)); }

// Arrival of one warp on a barrier counted in the even CTA.
__device__ __forceinline__ void arrive_leader(bool leader, uint32_t local, uint32_t remote) {
  if (leader)
    mbar_arrive(local);
  else
    mbar_arrive_remote(remote);
}

// D = rowsum(dO * O) and the log2-domain LSE of every query row, into arrays with a
// row stride of Lqp (Lq rounded up to 128) so that the dK / dV kernels load four
// consecutive query rows' values with one 16-byte load; padded rows take no part
// (L2 = +inf, D = 0), and so do rows without a visible key (LSE = -inf).  One warp
// per padded row.
__global__ void __launch_bounds__(256) bwd_rowstate_kernel(const __nv_bfloat16* __restrict__ out,
                                                           const __nv_bfloat16* __restrict__ dout,
                                                           const float* __restrict__ lse, float* __restrict__ L2,
                                                           float* __restrict__ D, int64_t Lq, int64_t Lqp,
                                                           int64_t rows) {
  const int64_t row = int64_t(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int lane = threadIdx.x & 31;
  const int64_t head = row / Lqp, qi = row % Lqp;
  if (qi >= Lq) {
    if (lane == 0) L2[row] = INFINITY, D[row] = 0.f;
    return;
  }
  const int64_t src = head * Lq + qi;
  const uint4 a = *reinterpret_cast<const uint4*>(dout + src * kHeadDim + lane * 8);
  const uint4 c = *reinterpret_cast<const uint4*>(out + src * kHeadDim + lane * 8);
  const __nv_bfloat162* ha = reinterpret_cast<const __nv_bfloat162*>(&a);
  const __nv_bfloat162* hc = reinterpret_cast<const __nv_bfloat162*>(&c);
  float acc = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 fa = __bfloat1622float2(ha[i]), fc = __bfloat1622float2(hc[i]);
    acc = fmaf(fa.x, fc.x, acc);
    acc = fmaf(fa.y, fc.y, acc);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) {
    const float l = lse[src];
    L2[row] = l == -INFINITY ? INFINITY : l * kLog2e;
    D[row] = acc;
  }
}

template <int kMode>
__global__ void __launch_bounds__(kThreads, 1)
bwd_tc_kernel(const __grid_constant__ CUtensorMap tmA1, const __grid_constant__ CUtensorMap tmA2,
              const __grid_constant__ CUtensorMap tmB1, const __grid_constant__ CUtensorMap tmB2,
              const __grid_constant__ CUtensorMap tmB3, const __grid_constant__ CUtensorMap tmC,
              const __grid_constant__ TcParams p) {
  using Gm = Geo<kMode>;
  constexpr bool kDQ = kMode == kModeDQ;
  constexpr bool kDP = Gm::kDP;
  extern __shared__ __align__(1024) char smem_raw[];
  const uint32_t sbase = smem_u32(smem_raw);
  // The swizzled tiles need 1024-byte alignment (never expected to fail).  A CTA of a
  // pair must not leave early: on failure it only skips its role.
  const bool misaligned = (sbase & 1023u) != 0;
  const uint32_t sA1 = sbase + Gm::kOffA, sA2 = sA1 + kABytes;
  const uint32_t sB1 = sbase + Gm::kOffB1, sB2 = sbase + Gm::kOffB2, sB3 = sbase + Gm::kOffB3;
  const uint32_t sCol = sbase + Gm::kOffCol;
  const uint32_t bar = sbase + Gm::kOffBar;
  auto B = [&](int i) { return bar + 8u * uint32_t(i); };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0: the even CTA, which issues the MMAs
  const bool leader = rank == 0;
  const uint32_t lead_bar = mapa_shared(bar, 0);
  auto LB = [&](int i) { return lead_bar + 8u * uint32_t(i); };
  int* range = reinterpret_cast<int*>(smem_raw + Gm::kOffBar + kOffRange);

  // Unit: (row-tile pair, kv head, batch), ordered kv head by kv head: the pairs
  // resident together then stream the same head's columns, which stay in L2.
  const int npairs = kDQ ? (p.nq + 1) / 2 : (p.nk + 1) / 2;  // row-tile pairs per kv head
  const int pair = int(blockIdx.x >> 1);
  const int local = pair % npairs;  // row-tile pair within the kv head
  const int g = (pair / npairs) % p.Hkv, b = (pair / npairs) / p.Hkv;
  const int br = p.br, br_shift = __ffs(br) - 1;
  const int kvhead = b * p.Hkv + g;
  const int qhead0 = b * p.Hq + g * p.G;
  int rt0;               // the pair's first row tile; this CTA's is rt0 + rank
  int cbeg = 0, cend = 0;  // column-tile range of the pair
  if (kDQ) {
    rt0 = 2 * (npairs - 1 - local);  // longest query rows first
    int f0, e0, f1, e1;
    key_range(p, rt0, &f0, &e0);
    key_range(p, rt0 + 1, &f1, &e1);
    if (f0 < e0) cbeg = f0, cend = e0;
    if (f1 < e1) {
      if (cbeg < cend) {
        cbeg = min(cbeg, f1);
        cend = max(cend, e1);
      } else {
        cbeg = f1;
        cend = e1;
      }
    }
  } else {
    rt0 = 2 * local;  // the earliest keys, seen by the most rows, first
    // Causally the first query tile holding a row at position >= the first key (every
    // tile for a key tile with shared-state keys); with segment ids the first and last
    // tile that is not SKIP for either key tile, found by the whole CTA.
    const int64_t j0 = int64_t(rt0) * kCols;
    cbeg = (j0 < p.P0 || j0 <= p.off) ? 0 : int(min(int64_t(p.nq), (j0 - p.off) / br));
    cend = p.nq;
    if (p.has_seg) {
      if (threadIdx.x == 0) range[0] = 0x7fffffff, range[1] = -1;
      __syncthreads();
      int lo = 0x7fffffff, hi = -1;
      for (int ct = cbeg + int(threadIdx.x); ct < cend; ct += kThreads)
        if (block_class(p, ct, rt0) != GQA_TILE_SKIP || block_class(p, ct, rt0 + 1) != GQA_TILE_SKIP) {
          lo = min(lo, ct);
          hi = max(hi, ct);
        }
      if (hi >= 0) {
        atomicMin(&range[0], lo);
        atomicMax(&range[1], hi);
      }
      __syncthreads();
      if (range[1] >= 0) {
        cbeg = range[0];
        cend = range[1] + 1;
      } else {
        cbeg = cend = 0;
      }
    }
  }
  const int rt = rt0 + int(rank);
  // Order of the column tiles.  dQ walks the key tiles upwards from 0; dK / dV walk the
  // query tiles downwards from the last, so the pairs of one key/value head running at
  // the same time read the same query tile at about the same time and it is fetched
  // from HBM about once (Q and dO are G times larger than K and V and exceed L2 at long
  // L; upwards, each pair would start at its own first visible tile).
  auto col_at_step = [&](int i) { return kDQ ? i : cbeg + cend - 1 - i; };
  // The pair computes a column tile unless it is SKIP for both row tiles; without
  // segment ids every tile of the range is visible to one of them.
  auto col_skip = [&](int ct) -> bool {
    if (!p.has_seg) return false;
    return kDQ ? (block_class(p, rt0, ct) == GQA_TILE_SKIP && block_class(p, rt0 + 1, ct) == GQA_TILE_SKIP)
               : (block_class(p, ct, rt0) == GQA_TILE_SKIP && block_class(p, ct, rt0 + 1) == GQA_TILE_SKIP);
  };

  if (threadIdx.x == 0) {
    mbar_init(B(kBarA), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(B(kBarB1Full + s), 1);
      mbar_init(B(kBarB1Empty + s), 1);
      mbar_init(B(kBarB3Full + s), 1);
      mbar_init(B(kBarB3Empty + s), 1);
      mbar_init(B(kBarSFull + s), 1);
      mbar_init(B(kBarSFree + s), 32);
      mbar_init(B(kBarPFull + s), 32);
      mbar_init(B(kBarDPFull + s), 1);
      mbar_init(B(kBarDSReady + s), 32);
      mbar_init(B(kBarAccDone + s), 1);
    }
    mbar_init(B(kBarB2Full), 1);
    mbar_init(B(kBarB2Empty), 1);
    mbar_init(B(kBarDrain), Gm::kIssuers);
    for (int s = 0; s < 2; ++s) {
      mbar_init(B(kBarColFull + s), 1);
      mbar_init(B(kBarColEmpty + s), 16);
    }
    fence_barrier_init();
    if (misaligned) set_status(p.status, GQA_ERR_LAUNCH);
  }
  if (warp == 1) umma::tmem_alloc_2sm(bar + kOffTmemSlot, kTmemCols);
  umma::fence_before_sync();
  cluster_sync();  // both CTAs' barriers initialised and TMEM allocated
  umma::fence_after_sync();
  uint32_t tmem;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(tmem) : "r"(bar + kOffTmemSlot));
  const int64_t budget = p.wait_budget_ns;

  if (misaligned) {
    // no role: fall through to the final cluster barrier
  } else if (warp == 0) {
    // ---------------------------------------------------------------- TMA producers
    // Each CTA loads its own row tile and its halves of the column tiles; completion
    // is counted on the even CTA's barriers, which its producers arm with both halves.
    if (lane < 2) {
      const bool first = lane == 0;
      // coordinates of column tile ct: (d in block, row, head or block, block or head)
      auto half_coords = [&](int ct, int* c) {  // B1 / B2: this CTA's 64 columns x 256 d
        if (kDQ) {
          c[1] = ct * kCols + int(rank) * 64, c[2] = 0, c[3] = kvhead;
        } else {
          c[1] = ct * br + (p.G == 1 ? int(rank) * 64 : 0);
          c[2] = qhead0 + (p.G > 1 ? int(rank) * (p.G / 2) : 0);
          c[3] = 0;
        }
      };
      auto dhalf_coords = [&](int ct, int* c) {  // B3: 128 columns x this CTA's 128 d
        if (kDQ)
          c[1] = ct * kCols, c[2] = 2 * int(rank), c[3] = kvhead;
        else
          c[1] = ct * br, c[2] = qhead0, c[3] = 2 * int(rank);
      };
      // One ring: wait for the slot to be free, arm, copy.
      auto fill = [&](uint32_t u, int nslots, int bar_full, int bar_empty, uint32_t ring, const CUtensorMap* map,
                      const int* c) -> bool {
        const int s = int(u % uint32_t(nslots));
        if (!mbar_wait_inline(B(bar_empty + s), ((u / uint32_t(nslots)) & 1u) ^ 1u, budget, p.status)) return false;
        if (leader) mbar_arrive_expect_tx(B(bar_full + s), 2 * kBBytes);
        tma_load_4d_pair(ring + uint32_t(s) * kBBytes, map, LB(bar_full + s), 0, c[1], c[2], c[3]);
        return true;
      };
      if (first) {
        tma_prefetch_desc(&tmA1);
        tma_prefetch_desc(&tmB1);
        if (leader) mbar_arrive_expect_tx(B(kBarA), 2u * Gm::kNA * kABytes);
        if (kDQ) {
          tma_load_4d_pair(sA1, &tmA1, LB(kBarA), 0, rt * br, qhead0, 0);
          tma_load_4d_pair(sA2, &tmA2, LB(kBarA), 0, rt * br, qhead0, 0);
        } else {
          tma_load_4d_pair(sA1, &tmA1, LB(kBarA), 0, rt * kCols, 0, kvhead);
          if (kDP) tma_load_4d_pair(sA2, &tmA2, LB(kBarA), 0, rt * kCols, 0, kvhead);
        }
      } else {
        if (kDP) tma_prefetch_desc(&tmB2);
        tma_prefetch_desc(&tmB3);
      }
      uint32_t u = 0;  // column tiles filled
      bool ok = true;
      for (int i = cbeg; ok && i < cend; ++i) {
        const int ct = col_at_step(i);
        if (col_skip(ct)) continue;
        int c[4];
        if (first) {
          if (!kDQ) {
            // this CTA's own copy of the query tile's D and log2-LSE (2 slots)
            const int s = int(u & 1u);
            ok = mbar_wait_inline(B(kBarColEmpty + s), ((u >> 1) & 1u) ^ 1u, budget, p.status);
            if (!ok) break;
            mbar_arrive_expect_tx(B(kBarColFull + s), kColBytes);
            tma_load_3d(sCol + uint32_t(s) * kColBytes, &tmC, B(kBarColFull + s), ct * br, qhead0, 0);
          }
          half_coords(ct, c);
          if (int(u) == p.test_skip_fill) {  // test hook: both CTAs skip this fill of ring B1
            const int s = int(u % uint32_t(Gm::kS1));
            ok = mbar_wait_inline(B(kBarB1Empty + s), ((u / uint32_t(Gm::kS1)) & 1u) ^ 1u, budget, p.status);
          } else {
            ok = fill(u, Gm::kS1, kBarB1Full, kBarB1Empty, sB1, &tmB1, c);
          }
        } else {
          if (kDP) {
            half_coords(ct, c);
            ok = fill(u, Gm::kS2, kBarB2Full, kBarB2Empty, sB2, &tmB2, c);
          }
          dhalf_coords(ct, c);
          ok = ok && fill(u, Gm::kS3, kBarB3Full, kBarB3Empty, sB3, &tmB3, c);
        }
        if (ok) ++u;
      }
      // No copy may be in flight when the pair ends.  The even CTA's barriers count
      // both CTAs' copies; the final cluster barrier holds the odd CTA until these
      // waits are over.
      if (leader) {
        auto drain = [&](int nslots, int bar_full) {
          for (uint32_t i = u > uint32_t(nslots) ? u - nslots : 0u; i < u; ++i)
            mbar_wait_inline(B(bar_full + int(i % uint32_t(nslots))), (i / uint32_t(nslots)) & 1u, budget, p.status);
        };
        if (first) {
          mbar_wait_inline(B(kBarA), 0, budget, p.status);
          drain(Gm::kS1, kBarB1Full);
        } else {
          if (kDP) drain(Gm::kS2, kBarB2Full);
          drain(Gm::kS3, kBarB3Full);
        }
      }
      if (first && !kDQ)  // each CTA's column-state copies complete on its own barriers
        for (uint32_t i = u > 2u ? u - 2u : 0u; i < u; ++i)
          mbar_wait_inline(B(kBarColFull + int(i & 1u)), (i >> 1) & 1u, budget, p.status);
    }
    __syncwarp();
  } else if (warp < 4) {
    // ---------------------------------------------------------------- MMA issuers (even CTA)
    const int role = warp == 1 ? 0 : (warp == 3 ? 1 : 2);  // 0: S, 1: dP, 2: accumulation
    if (lane == 0 && leader && (kDP || role != 1)) {
      constexpr uint32_t id_s = umma::idesc_bf16(2 * kRows, kCols, 0, 0);
      constexpr uint32_t id_acc = umma::idesc_bf16(2 * kRows, 256, 0, 1);
      bool ok = role == 2 || mbar_wait_inline(B(kBarA), 0, budget, p.status);
      int t = 0;
      for (int i = cbeg; ok && i < cend; ++i) {
        const int ct = col_at_step(i);
        if (col_skip(ct)) continue;
        const int sb = t & 1;  // TMEM region of column tile t
        if (role != 2) {
          // S(t) = A1 B1(t)^T, or dP(t) = A2 B2(t)^T, into region sb: 16 pair MMAs of
          // M256 N128 K16 (four 64-column blocks of four K16 steps).  S(t) waits until
          // the accumulation of tile t-2 has read that region; dP(t) until every
          // elementwise thread has S(t) in registers.
          const bool is_s = role == 0;
          const int ns = is_s ? Gm::kS1 : 1;
          const int s = t % ns;
          if (!(ok = mbar_wait_inline(B((is_s ? kBarB1Full : kBarB2Full) + s), uint32_t(t / ns) & 1u, budget,
                                      p.status)))
            break;
          if (is_s && t >= 2 &&
              !(ok = mbar_wait_inline(B(kBarAccDone + sb), (uint32_t(t - 2) >> 1) & 1u, budget, p.status)))
            break;
          if (!is_s && !(ok = mbar_wait_inline(B(kBarSFree + sb), (uint32_t(t) >> 1) & 1u, budget, p.status)))
            break;
          umma::fence_after_sync();
          const uint32_t d = tmem + kTmemS + uint32_t(sb * 128);
          const uint64_t da = umma::smem_desc(is_s ? sA1 : sA2, 16, 1024);
          const uint64_t db = umma::smem_desc((is_s ? sB1 : sB2) + uint32_t(s) * kBBytes, 16, 1024);
#pragma unroll
          for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int k = 0; k < 4; ++k)
              umma::mma_ss_2sm(d, umma::desc_add(da, uint32_t(c * kABlock + k * 32)),
                               umma::desc_add(db, uint32_t(c * kBHalfBlock + k * 32)), id_s, (c | k) != 0 ? 1u : 0u);
          umma::commit_2sm_mc(B((is_s ? kBarB1Empty : kBarB2Empty) + s), kPairMask);
          umma::commit_2sm_mc(B((is_s ? kBarSFull : kBarDPFull) + sb), kPairMask);
        } else {
          // acc += dS(t) B3(t) (P(t) B3(t) for dV): A = the packed tile in region sb,
          // eight pair MMAs of M256 N256 K16 over the 128 columns.
          const int s = t % Gm::kS3;
          if (!(ok = mbar_wait_inline(B((kDP ? kBarDSReady : kBarPFull) + sb), (uint32_t(t) >> 1) & 1u, budget,
                                      p.status)))
            break;
          if (!(ok = mbar_wait_inline(B(kBarB3Full + s), uint32_t(t / Gm::kS3) & 1u, budget, p.status))) break;
          umma::fence_after_sync();
          const uint32_t a = tmem + kTmemS + uint32_t(sb * 128);
          const uint64_t db = umma::smem_desc(sB3 + uint32_t(s) * kBBytes, kB3Block, 1024);
#pragma unroll
          for (int k = 0; k < kCols / 16; ++k)
            umma::mma_ts_2sm(tmem + kTmemAcc, a + packed_col(k), umma::desc_add(db, uint32_t(k * 2048)), id_acc,
                             (t > 0 || k > 0) ? 1u : 0u);
          umma::commit_2sm_mc(B(kBarB3Empty + s), kPairMask);
          umma::commit_2sm_mc(B(kBarAccDone + sb), kPairMask);
        }
        ++t;
      }
      // every MMA of the pair must be complete before TMEM is released
      umma::commit_2sm(B(kBarDrain));
      mbar_wait_inline(B(kBarDrain), 0, budget, p.status);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- elementwise warps
    const int quarter = warp & 3;       // TMEM lane quarter this warp may access
    const int part = (warp - 4) >> 2;   // columns 32 part .. +31
    const int r = quarter * 32 + lane;  // row of this CTA = TMEM lane
    const uint32_t lane_addr = tmem + (uint32_t(quarter * 32) << 16);
    const float sl2 = p.scale_log2;
    // Row state.  dQ: a query row (its log2-LSE, D, position, segment); dK / dV: a key.
    int64_t dst_row = -1, pos = 0, key = 0;
    float L2r = INFINITY, Dr = 0.f;
    int srow = 0;
    if (kDQ) {
      const int hh = r >> br_shift, pp = r & (br - 1);
      const int64_t qi = int64_t(rt) * br + pp;
      if (rt < p.nq && qi < p.Lq) {
        const int64_t hrow = int64_t(qhead0 + hh) * p.Lqp + qi;
        L2r = p.L2[hrow];
        Dr = p.D[hrow];
        dst_row = int64_t(qhead0 + hh) * p.Lq + qi;
        if (p.has_seg) srow = p.seg_q[qi];
      }
      pos = qi + p.off;
    } else {
      key = int64_t(rt) * kCols + r;
      if (rt < p.nk && key < p.Lk) {
        dst_row = int64_t(kvhead) * p.Lk + key;
        if (p.has_seg) srow = p.seg_kv[key];
      }
    }
    // Column state of a query tile (dK / dV), staged by TMA: D of column c at word c,
    // log2-LSE at word 128 + c; every lane of a warp reads the same 16 bytes.
    auto col_vec = [&](int slot, int word) -> float4 {
      float4 f;
      asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                   : "=f"(f.x), "=f"(f.y), "=f"(f.z), "=f"(f.w)
                   : "r"(sCol + uint32_t(slot * kColBytes + word * 4)));
      return f;
    };

    int t = 0;
    bool ok = true;
    for (int i = cbeg; i < cend; ++i) {
      const int ct = col_at_step(i);
      if (col_skip(ct)) continue;
      const int cls = kDQ ? block_class(p, rt, ct) : block_class(p, ct, rt);
      const int sb = t & 1;  // TMEM region of this column tile
      float x[32];
      const int cslot = t & 1;
      if (!warp_wait(B(kBarSFull + sb), (uint32_t(t) >> 1) & 1u, budget, p.status)) {
        ok = false;
        break;
      }
      umma::fence_after_sync();
      umma::tmem_ld32(lane_addr + kTmemS + uint32_t(sb * 128 + part * 32), x);
      umma::tmem_wait_ld();
      if (kDP) {
        // S is in registers: the tensor cores may overwrite it with dP(t).
        umma::fence_before_sync();
        __syncwarp();
        if (lane == 0) arrive_leader(leader, B(kBarSFree + sb), LB(kBarSFree + sb));
      }
      if (!kDQ && !warp_wait(B(kBarColFull + cslot), (uint32_t(t) >> 1) & 1u, budget, p.status)) {
        ok = false;
        break;
      }
      // P = 2^(S * scale * log2(e) - LSE * log2(e)), 0 where the pair is masked.
      if (cls == GQA_TILE_SKIP) {
#pragma unroll
        for (int i = 0; i < 32; ++i) x[i] = 0.f;
      } else if (kDQ) {
        // exponent arguments first (masked entries -inf), then the 32 exponentials
        const int64_t jb = int64_t(ct) * kCols + part * 32;
        const bool need_mask = cls == GQA_TILE_PARTIAL || int64_t(ct) * kCols + kCols > p.Lk;
#pragma unroll
        for (int i = 0; i < 32; ++i) x[i] = fmaf(x[i], sl2, -L2r);
        if (need_mask) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int64_t j = jb + i;
            bool vis = j <= pos && j < p.Lk;
            if (p.has_seg) vis = vis && (j < p.P0 || srow == __ldg(p.seg_kv + min(j, p.Lk - 1)));
            if (!vis) x[i] = -INFINITY;
          }
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) x[i] = ex2_approx(x[i]);
      } else {
        // exponent arguments first (masked entries -inf), then the 32 exponentials
        const bool need_mask = cls == GQA_TILE_PARTIAL;
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          const float4 f = col_vec(cslot, 128 + part * 32 + 4 * v);
          x[4 * v] = fmaf(x[4 * v], sl2, -f.x);
          x[4 * v + 1] = fmaf(x[4 * v + 1], sl2, -f.y);
          x[4 * v + 2] = fmaf(x[4 * v + 2], sl2, -f.z);
          x[4 * v + 3] = fmaf(x[4 * v + 3], sl2, -f.w);
        }
        if (need_mask) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int c = part * 32 + i;
            const int64_t qi = int64_t(ct) * br + (c & (br - 1));
            bool vis = key <= qi + p.off;
            if (p.has_seg) vis = vis && (key < p.P0 || srow == __ldg(p.seg_q + min(qi, p.Lq - 1)));
            if (!vis) x[i] = -INFINITY;
          }
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) x[i] = ex2_approx(x[i]);
      }
      uint32_t pk[16];
      if (!kDP) {
        // dV: P as bf16 pairs over the first 16 of this thread's 32 S columns.
#pragma unroll
        for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(x[2 * i], x[2 * i + 1]);
        umma::tmem_st16u(lane_addr + kTmemS + uint32_t(sb * 128 + part * 32), pk);
        umma::tmem_wait_st();
        umma::fence_before_sync();
        __syncwarp();
        if (lane == 0) {
          arrive_leader(leader, B(kBarPFull + sb), LB(kBarPFull + sb));
          mbar_arrive(B(kBarColEmpty + cslot));
        }
      } else {
        // dS = P (dP - D) as bf16 pairs over the first 16 of this thread's 32 dP columns.
        if (!warp_wait(B(kBarDPFull + sb), (uint32_t(t) >> 1) & 1u, budget, p.status)) {
          ok = false;
          break;
        }
        umma::fence_after_sync();
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          float y[16];
          float dc[16];
          umma::tmem_ld16(lane_addr + kTmemS + uint32_t(sb * 128 + part * 32 + h * 16), y);
          if (!kDQ) {
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              const float4 f = col_vec(cslot, part * 32 + h * 16 + 4 * v);
              dc[4 * v] = f.x, dc[4 * v + 1] = f.y, dc[4 * v + 2] = f.z, dc[4 * v + 3] = f.w;
            }
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) dc[i] = Dr;
          }
          umma::tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 8; ++i)
            pk[h * 8 + i] = pack_bf16x2(x[h * 16 + 2 * i] * (y[2 * i] - dc[2 * i]),
                                        x[h * 16 + 2 * i + 1] * (y[2 * i + 1] - dc[2 * i + 1]));
        }
        umma::tmem_st16u(lane_addr + kTmemS + uint32_t(sb * 128 + part * 32), pk);
        umma::tmem_wait_st();
        umma::fence_before_sync();
        __syncwarp();
        if (lane == 0) {
          arrive_leader(leader, B(kBarDSReady + sb), LB(kBarDSReady + sb));
          if (!kDQ) mbar_arrive(B(kBarColEmpty + cslot));
        }
      }
      ++t;
    }
    // ------------------------------------------------------------ epilogue
    // Row r of the accumulator, columns 64 part .. +63, scaled, as bf16.
    if (ok && t > 0) {
      const int tl = t - 1;
      ok = warp_wait(B(kBarAccDone + (tl & 1)), (uint32_t(tl) >> 1) & 1u, budget, p.status);
      umma::fence_after_sync();
    }
    if (ok) {
      uint4* dst = reinterpret_cast<uint4*>(p.dst + (dst_row >= 0 ? dst_row : 0) * kHeadDim);
#pragma unroll 1
      for (int c0 = part * 64; c0 < part * 64 + 64; c0 += 32) {
        float o[32];
        if (t > 0) {
          umma::tmem_ld32(lane_addr + kTmemAcc + uint32_t(c0), o);
          umma::tmem_wait_ld();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = 0.f;
        }
        if (dst_row >= 0) {
          const float sc = p.out_scale;
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4) {
            uint4 w;
            w.x = pack_bf16x2(o[8 * v4 + 0] * sc, o[8 * v4 + 1] * sc);
            w.y = pack_bf16x2(o[8 * v4 + 2] * sc, o[8 * v4 + 3] * sc);
            w.z = pack_bf16x2(o[8 * v4 + 4] * sc, o[8 * v4 + 5] * sc);
            w.w = pack_bf16x2(o[8 * v4 + 6] * sc, o[8 * v4 + 7] * sc);
            dst[c0 / 8 + v4] = w;
          }
        }
      }
    }
  }

  // Neither CTA may release TMEM or leave while the pair's MMAs or copies may still
  // touch its memory: the issuers and the even CTA's producers have drained by now.
  umma::fence_before_sync();
  cluster_sync();
  if (warp == 1) {
    umma::fence_after_sync();
    umma::tmem_dealloc_2sm(tmem, kTmemCols);
  }
}

// 4-D views with a 64-column (128-byte) block of d innermost, 128-byte swizzled.
// Query side [B * Hq][Lq][256]: (d in block, position, head, block).
bool encode_q(EncodeTiledFn enc, CUtensorMap* m, const void* ptr, int64_t Lq, int64_t heads, int box_pos,
              int box_heads, int box_blocks) {
  const cuuint64_t row = cuuint64_t(kHeadDim) * 2;
  const cuuint64_t dims[4] = {64, cuuint64_t(Lq), cuuint64_t(heads), 4};
  const cuuint64_t strides[3] = {row, cuuint64_t(Lq) * row, 128};
  const cuuint32_t box[4] = {64, cuuint32_t(box_pos), cuuint32_t(box_heads), cuuint32_t(box_blocks)};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Key side [B * Hkv][Lk][256]: (d in block, key, block, kv head).
bool encode_k(EncodeTiledFn enc, CUtensorMap* m, const void* ptr, int64_t Lk, int64_t heads, int box_keys,
              int box_blocks) {
  const cuuint64_t row = cuuint64_t(kHeadDim) * 2;
  const cuuint64_t dims[4] = {64, cuuint64_t(Lk), 4, cuuint64_t(heads)};
  const cuuint64_t strides[3] = {row, 128, cuuint64_t(Lk) * row};
  const cuuint32_t box[4] = {64, cuuint32_t(box_keys), cuuint32_t(box_blocks), 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int kMode>
int launch_mode(const CUtensorMap (&m)[6], const TcParams& p, int64_t units, cudaStream_t stream) {
  if (units <= 0) return GQA_OK;
  if (units > 0x7fffffff) return GQA_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(bwd_tc_kernel<kMode>, cudaFuncAttributeMaxDynamicSharedMemorySize, Geo<kMode>::kSmem) !=
      cudaSuccess)
    return GQA_ERR_LAUNCH;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(units), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = Geo<kMode>::kSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, bwd_tc_kernel<kMode>, m[0], m[1], m[2], m[3], m[4], m[5], p) != cudaSuccess)
    return GQA_ERR_LAUNCH;
  return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_LAUNCH;
}

}  // namespace

int launch_bwd_bf16(const BwdArgs& a, cudaStream_t stream) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return GQA_ERR_LAUNCH;
  TcParams p;
  p.L2 = a.L2;
  p.D = a.D;
  p.seg_q = a.seg_q;
  p.seg_kv = a.seg_kv;
  p.q_bounds = a.q_bounds;
  p.kv_bounds = a.kv_bounds;
  p.q_ranges = a.q_ranges;
  p.status = a.status;
  p.Lq = a.Lq;
  p.Lk = a.Lk;
  p.Lqp = a.ldD;
  p.off = a.off;
  p.P0 = a.P0;
  p.wait_budget_ns = a.wait_budget_ns;
  p.test_skip_fill = a.test_skip_fill;
  p.B = a.B;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.G = a.Hq / a.Hkv;
  p.br = kBf16Rows / p.G;
  p.nq = int((a.Lq + p.br - 1) / p.br);
  p.nk = int((a.Lk + kCols - 1) / kCols);
  p.has_seg = a.seg_q != nullptr;
  p.scale_log2 = a.scale * kLog2e;
  if (p.Lqp % 128 != 0 || p.Lqp < a.Lq) return GQA_ERR_INVALID_ARG;

  const int64_t rows = int64_t(a.B) * a.Hq * p.Lqp;
  if (rows > 0) {
    const int64_t blocks = (rows + 7) / 8;
    if (blocks > 0x7fffffff) return GQA_ERR_UNSUPPORTED;
    bwd_rowstate_kernel<<<unsigned(blocks), 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(a.out),
                                                              static_cast<const __nv_bfloat16*>(a.dout), a.lse,
                                                              a.L2, a.D, a.Lq, p.Lqp, rows);
    if (cudaGetLastError() != cudaSuccess) return GQA_ERR_LAUNCH;
  }
  const int64_t qheads = int64_t(a.B) * a.Hq, kheads = int64_t(a.B) * a.Hkv;
  const int G = p.G, br = p.br;
  const int G2 = G > 1 ? G / 2 : 1, br2 = 64 / G2;  // half a query tile: 64 columns
  CUtensorMap q_full, do_full, q_half, do_half, q_dhalf, do_dhalf, k_full, v_full, k_half, v_half, k_dhalf;
  if (!encode_q(enc, &q_full, a.q, a.Lq, qheads, br, G, 4) || !encode_q(enc, &do_full, a.dout, a.Lq, qheads, br, G, 4) ||
      !encode_q(enc, &q_half, a.q, a.Lq, qheads, br2, G2, 4) ||
      !encode_q(enc, &do_half, a.dout, a.Lq, qheads, br2, G2, 4) ||
      !encode_q(enc, &q_dhalf, a.q, a.Lq, qheads, br, G, 2) || !encode_q(enc, &do_dhalf, a.dout, a.Lq, qheads, br, G, 2) ||
      !encode_k(enc, &k_full, a.k, a.Lk, kheads, kCols, 4) || !encode_k(enc, &v_full, a.v, a.Lk, kheads, kCols, 4) ||
      !encode_k(enc, &k_half, a.k, a.Lk, kheads, 64, 4) || !encode_k(enc, &v_half, a.v, a.Lk, kheads, 64, 4) ||
      !encode_k(enc, &k_dhalf, a.k, a.Lk, kheads, kCols, 2))
    return GQA_ERR_LAUNCH;
  // Column state of the dK / dV kernels: the D and log2-LSE planes of the workspace as
  // one (position, head, plane) view; a box is one query tile's 128 columns of both.
  CUtensorMap col;
  {
    const int64_t plane = reinterpret_cast<const char*>(a.L2) - reinterpret_cast<const char*>(a.D);
    if (plane <= 0 || plane % 16 != 0) return GQA_ERR_INVALID_ARG;
    const cuuint64_t dims[3] = {cuuint64_t(p.Lqp), cuuint64_t(qheads), 2};
    const cuuint64_t strides[2] = {cuuint64_t(p.Lqp) * 4, cuuint64_t(plane)};
    const cuuint32_t box[3] = {cuuint32_t(br), cuuint32_t(G), 2};
    const cuuint32_t estr[3] = {1, 1, 1};
    if (enc(&col, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, a.D, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return GQA_ERR_LAUNCH;
  }
  const int64_t q_units = 2 * ((int64_t(p.nq) + 1) / 2) * kheads;
  const int64_t k_units = 2 * ((int64_t(p.nk) + 1) / 2) * kheads;
  int rc;
  {
    const CUtensorMap m[6] = {k_full, k_full, q_half, q_half, do_dhalf, col};
    p.dst = static_cast<__nv_bfloat16*>(a.dv);
    p.out_scale = 1.f;
    if ((rc = launch_mode<kModeDV>(m, p, k_units, stream)) != GQA_OK) return rc;
  }
  {
    const CUtensorMap m[6] = {k_full, v_full, q_half, do_half, q_dhalf, col};
    p.dst = static_cast<__nv_bfloat16*>(a.dk);
    p.out_scale = a.scale;
    if ((rc = launch_mode<kModeDK>(m, p, k_units, stream)) != GQA_OK) return rc;
  }
  const CUtensorMap m[6] = {q_full, do_full, k_half, v_half, k_dhalf, col};
  p.dst = static_cast<__nv_bfloat16*>(a.dq);
  p.out_scale = a.scale;
  return launch_mode<kModeDQ>(m, p, q_units, stream);
}

}  // namespace gqa
