// Attention backward (dQ, dK, dV from the saved LSE) on the FP32 pipe, sm_100a.
//
// Training over packed long sequences (maxtext PR #4929, description: the splash
// kernel runs inside training steps on 1,048,576-token packed batches) needs the
// gradients of the attention output.  With P = exp(scale * S - LSE) recomputed from
// the forward's log-sum-exp, D_i = <dO_i, O_i>, dP = dO V^T and dS = P * (dP - D):
//     dV_j = sum_{h in group} sum_i P_ij dO_i,   dK_j = scale * sum_{h in group} sum_i dS_ij Q_i,
//     dQ_i = scale * sum_j dS_ij K_j.
// Four kernels, no atomics:
//   bwd_rowdot_kernel   D = rowsum(dO * O), one warp per row.
//   bwd_ffma_kernel<R>  three instances of one design, each a CTA of 8 warps that keeps
//                       64 "resident" rows and accumulates a 64 x 256 gradient in
//                       registers while it streams tiles of 128 "streamed" rows:
//     R = DQ  resident: 64 query rows (64/G positions x the G heads of a kv head),
//             Q and dO; streamed: key tiles of the query tile's range (the plan's
//             block skipping); S = Q K^T, dP = dO V^T, dS, dQ += dS K.
//     R = DK  resident: 64 keys of a kv head, K and V; streamed: query tiles of 128
//             rows (128/G positions x the G heads) that see them; S^T = K Q^T,
//             dP^T = V dO^T, dS^T, dK += dS^T Q -- the G heads' contributions summed
//             on chip.
//     R = DV  resident: 64 keys, K; streamed: the same query tiles; S^T, P^T,
//             dV += P^T dO.
// The design is the forward FFMA kernel's (fwd_f32.cu).  Shared-memory wavefronts
// bound an FFMA contraction at d = 256: a warp's 128-bit shared load costs four
// wavefronts with distinct addresses and two when every lane reads one, and an SM
// moves one wavefront per cycle against two packed FMAs (fma.rn.f32x2).  So:
//   * the resident operands sit transposed in shared memory ([d][row]), written once
//     per CTA, so a row pair at one depth is a register pair, and every lane of warp
//     w reads the same fragment of its rows 8w .. 8w+7;
//   * "S-like" products (S, dP, S^T, dP^T): lane l takes streamed rows l + 32 m
//     (m < 4), one accumulator per product: per depth, 2 broadcast loads (4
//     wavefronts) and 4 streamed values (4) for 16 packed FMAs;
//   * accumulations: the weights (dS, P^T, dS^T) go through a warp-private slice
//     [streamed row][8 resident rows] and are read as broadcasts; lane l owns columns
//     4l.. and 128+4l.. of its 8 gradient rows: per streamed row, 2 broadcast loads
//     (4) and 2 per-lane loads (8) for 32 packed FMAs.
// Streamed operands arrive as 16 KiB chunks, each ONE TMA copy (128-byte swizzle),
// through a ring of 4 slots that the warp finishing a chunk last refills four chunks
// ahead: "d-chunks" [128 rows][32 d] for the S-like products and "row chunks"
// [16 rows][256 d] for the accumulation.  Per tile: DQ 8 K d-chunks, 8 V d-chunks,
// 8 K row chunks; DK 8 Q, 8 dO d-chunks, 8 Q row chunks; DV 8 Q d-chunks, 8 dO row
// chunks.  The resident rows land in the ring first and are transposed from there.
// Both dtypes' arithmetic is fp32 (bf16 calls use the tensor-core backward).
#include <cuda_bf16.h>

#include "internal.h"

namespace gqa {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = 8;
constexpr int kRes = 64;        // resident rows per CTA (8 per warp)
constexpr int kStream = 128;    // streamed rows per tile (4 per lane)
constexpr int kSlots = 4;
constexpr int kSlotBytes = 16384;
constexpr int kBoxCols = 32;    // fp32 per 128-byte swizzle row
constexpr int kResBox = kRes * 128;            // resident staging: 64 rows x 32 d (8 KiB)
constexpr int kRowChunkRows = 16;              // rows of a row chunk
constexpr int kRowBlock = kRowChunkRows * 128; // row chunk: 16 rows x 32 d per block (2 KiB)
constexpr int kWWarpBytes = kStream * 8 * 4;   // weight slice: [128 streamed rows][8 rows] fp32
constexpr int kOffX1 = 0;                      // X1^T [256 d][64 rows]
constexpr int kOffX2 = kOffX1 + kRes * kHeadDim * 4;
constexpr int kOffW = kOffX2 + kRes * kHeadDim * 4;
constexpr int kOffRing = kOffW + kWarps * kWWarpBytes;
constexpr int kOffBar = kOffRing + kSlots * kSlotBytes;
enum { kBarRes = 0, kBarSlot = 1 };
constexpr int kOffCnt = kOffBar + 8 * (1 + kSlots);
constexpr int kOffIss = kOffCnt + 4 * kSlots;
constexpr int kSmemBytes = kOffIss + 4 * kSlots + 1024;  // + slack to align to the 1024-byte swizzle atom

static_assert(kRes == 8 * kWarps && kStream == 4 * 32, "tile geometry");
static_assert(kStream * 128 == kSlotBytes && 8 * kRowBlock == kSlotBytes, "chunk geometry");
static_assert(4 * kSlotBytes == kRes * kHeadDim * 4, "the resident rows are staged in the ring");
static_assert(kSmemBytes <= 232448, "shared memory per block");

enum Role { kDQ = 0, kDK = 1, kDV = 2 };

struct BwdParams {
  const void* q;
  const void* k;
  const void* v;
  const void* out;
  const float* lse;
  const void* dout;
  void* dq;
  void* dk;
  void* dv;
  float* D;  // [B, Hq, Lq]
  const int32_t* seg_q;
  const int32_t* seg_kv;
  const int32_t* q_bounds;   // plan [nq][2] at (br, 128) tiles, or null
  const int32_t* kv_bounds;  // [nk][2] or null
  const int32_t* q_ranges;   // [nq][2] or null
  int32_t* status;
  int64_t Lq, Lk, off, P0, wait_budget_ns;
  int B, Hq, Hkv, G, br, nq, nk, has_seg, bf16;
  int bq2, nq2, nk64;  // query tiles of the key-side kernels: 128 / G positions; key tiles of 64
  int test_skip_fill;
  float scale, scale_log2;
};

// Eight consecutive elements (16-byte aligned in fp32, 16 bytes in bf16) widened to fp32.
__device__ __forceinline__ void ld8(const void* base, int64_t idx, bool bf16, float (&x)[8]) {
  if (bf16) {
    const uint4 u = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(base) + idx);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(h[i]);
      x[2 * i] = f.x;
      x[2 * i + 1] = f.y;
    }
  } else {
    const float4 a = *reinterpret_cast<const float4*>(static_cast<const float*>(base) + idx);
    const float4 b = *reinterpret_cast<const float4*>(static_cast<const float*>(base) + idx + 4);
    x[0] = a.x, x[1] = a.y, x[2] = a.z, x[3] = a.w, x[4] = b.x, x[5] = b.y, x[6] = b.z, x[7] = b.w;
  }
}

__device__ __forceinline__ float4 lds128(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr));
  return v;
}

__device__ __forceinline__ void sts128(uint32_t addr, float a, float b, float c, float d) {
  asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}

// c0, c1 += a0 * b0, a1 * b1 in one packed fp32x2 FMA (round to nearest).
__device__ __forceinline__ void ffma2(float& c0, float& c1, float a0, float a1, float b0, float b1) {
  asm("{\n\t.reg .b64 ra, rb, rc;\n\t"
      "mov.b64 ra, {%2, %3};\n\t"
      "mov.b64 rb, {%4, %5};\n\t"
      "mov.b64 rc, {%0, %1};\n\t"
      "fma.rn.f32x2 rc, ra, rb, rc;\n\t"
      "mov.b64 {%0, %1}, rc;\n\t}"
      : "+f"(c0), "+f"(c1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// Tiled TMA loads into this CTA's shared memory (no multicast).
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int c0, int c1,
                                            int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}
// Tensor maps of one kernel: the resident operands (X1, X2: 8 boxes of 64 rows x 32 d),
// the streamed d-chunks (Y1, Y2: 128 rows x 32 d) and row chunks (Z: 16 rows x 256 d).
struct Maps {
  CUtensorMap x1, x2, y1, y2, z;
};

template <int R>
__global__ void __launch_bounds__(kThreads, 1) bwd_ffma_kernel(const __grid_constant__ Maps maps,
                                                               const __grid_constant__ BwdParams p) {
  constexpr int kPhases = R == kDV ? 1 : 2;      // S-like products per tile
  constexpr int kChunks = 8 * kPhases + 8;        // chunks per tile
  static_assert(kChunks % (2 * kSlots) == 0, "a tile is an even number of uses of every slot");
  extern __shared__ char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  const uint32_t sX1 = sbase + kOffX1, sX2 = sbase + kOffX2, sW = sbase + kOffW, sRing = sbase + kOffRing;
  const uint32_t bar = sbase + kOffBar;
  auto slot_bar = [&](int s) { return bar + 8u * uint32_t(kBarSlot + s); };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool bf16 = p.bf16 != 0;

  // Unit: (resident tile, kv head, batch), kv head by kv head.  DQ: query tiles in
  // descending order (the longest key ranges first); DK / DV: key tiles ascending
  // (the earliest keys see the most queries).
  const int nres = R == kDQ ? p.nq : p.nk64;
  const int rt = R == kDQ ? nres - 1 - int(blockIdx.x % unsigned(nres)) : int(blockIdx.x % unsigned(nres));
  const int hb = int(blockIdx.x / unsigned(nres));
  const int g = hb % p.Hkv, b = hb / p.Hkv;
  const int qhead0 = b * p.Hq + g * p.G;
  const int kvhead = b * p.Hkv + g;

  // Resident rows: DQ rows r = head (r / br) x position q0 + r % br; DK / DV keys k0 + r.
  const int64_t q0 = R == kDQ ? int64_t(rt) * p.br : 0;
  const int64_t k0 = R == kDQ ? 0 : int64_t(rt) * kRes;

  // Range of streamed tiles.  DQ: key tiles (128 keys) of the plan's range; DK / DV:
  // query tiles of bq2 positions that can see keys [k0, k0 + 64): causally from the
  // first row at position >= k0 (every row for a shared-state key), and with segment
  // ids the first and last tile that is not SKIP, found by the whole CTA.
  __shared__ int range[2];
  auto class_kv = [&](int qt2) {  // DK / DV: class of (query tile qt2, keys [k0, k0 + 64))
    const int64_t i0 = int64_t(qt2) * p.bq2, i1 = min(p.Lq, i0 + p.bq2) - 1;
    const int64_t j1 = min(p.Lk, k0 + kRes) - 1;
    SegBounds qb{0, 0}, kb{0, 0};
    if (p.has_seg) {  // plan tiles: query tiles of br = bq2 / 2 positions, key tiles of 128
      const int a = 2 * qt2, c = min(2 * qt2 + 1, p.nq - 1);
      qb = SegBounds{min(p.q_bounds[2 * a], p.q_bounds[2 * c]), max(p.q_bounds[2 * a + 1], p.q_bounds[2 * c + 1])};
      const int kt = int(k0 / 128);
      kb = SegBounds{p.kv_bounds[2 * kt], p.kv_bounds[2 * kt + 1]};
    }
    return tile_class(i0, i1, k0, j1, p.off, p.P0, p.has_seg != 0, qb, kb);
  };
  auto class_q = [&](int kt) {  // DQ: class of (query tile rt, key tile kt)
    const int64_t i1 = min(p.Lq, q0 + p.br) - 1;
    const int64_t j0 = int64_t(kt) * kStream, j1 = min(p.Lk, j0 + kStream) - 1;
    SegBounds qb{0, 0}, kb{0, 0};
    if (p.has_seg) {
      qb = SegBounds{p.q_bounds[2 * rt], p.q_bounds[2 * rt + 1]};
      kb = SegBounds{p.kv_bounds[2 * kt], p.kv_bounds[2 * kt + 1]};
    }
    return tile_class(q0, i1, j0, j1, p.off, p.P0, p.has_seg != 0, qb, kb);
  };
  auto tile_class_of = [&](int st) { return R == kDQ ? class_q(st) : class_kv(st); };
  int tbeg, tend;
  if (R == kDQ) {
    if (p.has_seg) {
      tbeg = p.q_ranges[2 * rt];
      tend = p.q_ranges[2 * rt + 1];
    } else {
      kv_range_no_seg(min(p.Lq, q0 + p.br) - 1, p.off, kStream, p.nk, &tbeg, &tend);
    }
  } else {
    tbeg = (k0 < p.P0 || k0 <= p.off) ? 0 : int((k0 - p.off) / p.bq2);
    tend = p.nq2;
    if (p.has_seg) {
      if (threadIdx.x == 0) range[0] = p.nq2, range[1] = -1;
      __syncthreads();
      int lo = p.nq2, hi = -1;
      for (int qt2 = tbeg + int(threadIdx.x); qt2 < p.nq2; qt2 += kThreads)
        if (class_kv(qt2) != GQA_TILE_SKIP) lo = min(lo, qt2), hi = max(hi, qt2);
      if (hi >= 0) {
        atomicMin(&range[0], lo);
        atomicMax(&range[1], hi);
      }
      __syncthreads();
      tbeg = range[0];
      tend = range[1] + 1;
    }
  }

  uint32_t* cnt = reinterpret_cast<uint32_t*>(smem_raw + (sbase + kOffCnt - raw));
  uint32_t* iss = reinterpret_cast<uint32_t*>(smem_raw + (sbase + kOffIss - raw));
  if (threadIdx.x == 0) {
    mbar_init(bar + 8 * kBarRes, 1);
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(slot_bar(s), 1);
      cnt[s] = 0;
      iss[s] = 0;
    }
    fence_barrier_init();
  }
  __syncthreads();

  auto next_tile = [&](int st) {
    while (st < tend && tile_class_of(st) == GQA_TILE_SKIP) ++st;
    return st;
  };
  // Chunk c of streamed tile st into slot c % 4.  c < 8: Y1 block c; 8 <= c < 8 kPhases:
  // Y2 block c - 8; the last 8: row chunk c - 8 kPhases of Z.
  auto load_chunk = [&](int st, int c) {
    const int s = c & 3;
    const uint32_t u = atomicAdd(&iss[s], 1u);  // the u-th fill of slot s: chunk 4u + s of the stream
    if (int64_t(4) * u + s == p.test_skip_fill) return;  // test hook: never arrives
    mbar_arrive_expect_tx(slot_bar(s), kSlotBytes);
    const uint32_t dst = sRing + s * kSlotBytes;
    const int zc = c - 8 * kPhases;  // row chunk index when >= 0
    if (R == kDQ) {  // streamed rows: keys st*128 ..
      const int key0 = st * kStream;
      if (c < 8)
        tma_load_4d(dst, &maps.y1, slot_bar(s), 0, key0, c, kvhead);
      else if (zc < 0)
        tma_load_4d(dst, &maps.y2, slot_bar(s), 0, key0, c - 8, kvhead);
      else
        tma_load_4d(dst, &maps.z, slot_bar(s), 0, key0 + kRowChunkRows * zc, 0, kvhead);
    } else {  // streamed rows: (head, position) of query tile st
      const int pos0 = st * p.bq2;
      if (zc < 0) {
        const CUtensorMap* map = c < 8 ? &maps.y1 : &maps.y2;
        tma_load_3d(dst, map, slot_bar(s), kBoxCols * (c & 7), pos0, qhead0);
      } else {
        const int r0 = kRowChunkRows * zc;  // first row of the chunk within the tile
        tma_load_4d(dst, &maps.z, slot_bar(s), 0, pos0 + r0 % p.bq2, qhead0 + r0 / p.bq2, 0);
      }
    }
  };
  auto release = [&](int st, int c, uint32_t use) {
    __syncwarp();
    if (lane == 0) {
      __threadfence_block();
      const int s = c & 3;
      if (atomicAdd(&cnt[s], 1u) == uint32_t(kWarps) * (use + 1) - 1) {
        if (c + 4 < kChunks) {
          load_chunk(st, c + 4);
        } else {
          const int sn = next_tile(st + 1);
          if (sn < tend) load_chunk(sn, c + 4 - kChunks);
        }
      }
    }
  };

  // ---- resident rows: staged in the ring (8 boxes of 64 rows x 32 d), transposed
  // into X^T [d][row]; X1, then X2.
  bool ok = true;
  for (int x = 0; x < (R == kDV ? 1 : 2); ++x) {
    if (threadIdx.x == 0) {
      if (x == 0) {
        tma_prefetch_desc(&maps.x1);
        tma_prefetch_desc(&maps.y1);
        tma_prefetch_desc(&maps.z);
        if (R != kDV) {
          tma_prefetch_desc(&maps.x2);
          tma_prefetch_desc(&maps.y2);
        }
      } else {
        fence_proxy_async_smem();  // the first round's staging reads come before these copies
      }
      const CUtensorMap* map = x == 0 ? &maps.x1 : &maps.x2;
      mbar_arrive_expect_tx(bar + 8 * kBarRes, 4 * kSlotBytes);
      for (int c = 0; c < 8; ++c) {
        if (R == kDQ)
          tma_load_3d(sRing + c * kResBox, map, bar + 8 * kBarRes, kBoxCols * c, int(q0), qhead0);
        else
          tma_load_3d(sRing + c * kResBox, map, bar + 8 * kBarRes, kBoxCols * c, int(k0), kvhead);
      }
    }
    ok = ok && mbar_wait_bounded(bar + 8 * kBarRes, uint32_t(x), p.wait_budget_ns, p.status);
    if (ok) {
      const int r = threadIdx.x & 63;
      float* xt = reinterpret_cast<float*>(smem_raw + ((x == 0 ? sX1 : sX2) - raw));
#pragma unroll 4
      for (int cx = threadIdx.x >> 6; cx < 64; cx += kThreads / 64) {  // (block c, chunk q) of d
        const int c = cx >> 3, qq = cx & 7;
        const float4 v = lds128(sRing + c * kResBox + r * 128 + (uint32_t(qq ^ (r & 7)) << 4));
        const int d = 32 * c + 4 * qq;
        xt[(d + 0) * kRes + r] = v.x;
        xt[(d + 1) * kRes + r] = v.y;
        xt[(d + 2) * kRes + r] = v.z;
        xt[(d + 3) * kRes + r] = v.w;
      }
    }
    ok = __syncthreads_and(ok);
  }
  if (threadIdx.x == 0) {
    fence_proxy_async_smem();  // the staging reads above come before the copies below
    const int s0 = ok ? next_tile(tbeg) : tend;
    if (s0 < tend)
      for (int c = 0; c < 4; ++c) load_chunk(s0, c);
  }

  // ---- per-resident-row state (DQ: log2-domain LSE and D of the warp's 8 query rows)
  // (positions and keys fit int32: Lk = off + Lq < 2^31)
  float L2r[8], Dr[8];
  int posr[8];  // DQ: position of the query row (-1 past Lq); DK / DV: the key index (INT_MAX past Lk)
  int segr[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = 8 * warp + i;
    if (R == kDQ) {
      const int hh = r / p.br;
      const int64_t qi = q0 + r % p.br;
      const bool live = hh < p.G && qi < p.Lq;
      const int64_t row = (int64_t(qhead0 + hh)) * p.Lq + qi;
      const float l = live ? p.lse[row] : -INFINITY;
      L2r[i] = l == -INFINITY ? INFINITY : l * kLog2e;
      Dr[i] = live ? p.D[row] : 0.f;
      posr[i] = live ? int(qi + p.off) : -1;
      segr[i] = (live && p.has_seg) ? p.seg_q[qi] : 0;
    } else {
      const int64_t kj = k0 + r;
      L2r[i] = 0.f;
      Dr[i] = 0.f;
      posr[i] = kj < p.Lk ? int(kj) : 0x7fffffff;  // a key past Lk is seen by no row
      segr[i] = (kj < p.Lk && p.has_seg) ? p.seg_kv[kj] : 0;
    }
  }

  float acc[8][8];
#pragma unroll
  for (int r = 0; r < 8; ++r)
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[r][c] = 0.f;

  const uint32_t xw = 8 * warp * 4;  // the warp's rows in X^T
  const uint32_t kl = lane * 128 + ((lane & 7) << 4);
  uint32_t zoff[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) zoff[c] = (lane >> 3) * kRowBlock + c * 128 + (uint32_t(c ^ (lane & 7)) << 4);
  const uint32_t sWw = sW + warp * kWWarpBytes;

  uint32_t t = 0;  // tiles computed so far: slot uses (kChunks / 4) t ..
  for (int st = tbeg; st < tend && ok; ++st) {
    const int cls = tile_class_of(st);
    if (cls == GQA_TILE_SKIP) continue;
    const uint32_t use0 = uint32_t(kChunks / 4) * t;

    // ---- S-like products: X^T row pairs (uniform) x streamed rows l + 32 m.
    float s1[8][4], s2[8][4];
    auto sphase = [&](float (&s)[8][4], const uint32_t xt, const int ph) {
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int m = 0; m < 4; ++m) s[i][m] = 0.f;
      float4 fq[4][2];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        fq[e][0] = lds128(xt + e * 256);
        fq[e][1] = lds128(xt + e * 256 + 16);
      }
#pragma unroll 1
      for (int c = 0; c < 8; ++c) {
        const int cc = 8 * ph + c;
        ok = __all_sync(0xffffffffu,
                        mbar_wait_bounded(slot_bar(cc & 3), uint32_t(cc >> 2) & 1u, p.wait_budget_ns, p.status));
        if (!ok) break;
        const uint32_t kslot = sRing + (cc & 3) * kSlotBytes + kl;
        float4 fk[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) fk[m] = lds128(kslot + m * 4096);
#pragma unroll
        for (int x = 0; x < 8; ++x) {  // depth step: d = 32 c + 4 x + e
          const int nd = (32 * c + 4 * (x + 1)) & (kHeadDim - 1);  // the last step re-reads depth 0
#pragma unroll
          for (int e = 0; e < 4; ++e) {
#pragma unroll
            for (int m = 0; m < 4; ++m) {
              const float kv = e == 0 ? fk[m].x : e == 1 ? fk[m].y : e == 2 ? fk[m].z : fk[m].w;
              ffma2(s[0][m], s[1][m], fq[e][0].x, fq[e][0].y, kv, kv);
              ffma2(s[2][m], s[3][m], fq[e][0].z, fq[e][0].w, kv, kv);
              ffma2(s[4][m], s[5][m], fq[e][1].x, fq[e][1].y, kv, kv);
              ffma2(s[6][m], s[7][m], fq[e][1].z, fq[e][1].w, kv, kv);
              if (e == 3 && x < 7) fk[m] = lds128((kslot ^ (uint32_t(x + 1) << 4)) + m * 4096);
            }
            fq[e][0] = lds128(xt + (nd + e) * 256);
            fq[e][1] = lds128(xt + (nd + e) * 256 + 16);
          }
        }
        release(st, cc, use0 + uint32_t(cc >> 2));
      }
    };
    sphase(s1, sX1 + xw, 0);
    if (!ok) break;
    if (kPhases == 2) {
      sphase(s2, sX2 + xw, 1);
      if (!ok) break;
    }

    // ---- weights: DQ dS = P (dP - D); DK dS^T = P^T (dP^T - D); DV P^T, P = exp2(S c - L2)
    {
      const int64_t c0 = int64_t(st) * (R == kDQ ? kStream : p.bq2);  // DQ: first key; else first position
      const bool edge = cls == GQA_TILE_PARTIAL ||
                        (R == kDQ ? c0 + kStream > p.Lk : (c0 + p.bq2 > p.Lq || k0 + kRes > p.Lk));
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int cr = lane + 32 * m;  // streamed row of the tile
        // the streamed row's index (DQ: key; else the query row's index in Lq, head hh)
        int cj;
        float L2c = 0.f, Dc = 0.f;
        int segc = 0;
        bool clive;
        if (R == kDQ) {
          cj = int(c0 + cr);
          clive = cj < p.Lk;
          segc = (edge && clive && p.has_seg) ? p.seg_kv[cj] : 0;
        } else {
          const int hh = cr / p.bq2;
          cj = int(c0 + cr % p.bq2);
          clive = cj < p.Lq;
          const int64_t row = int64_t(qhead0 + hh) * p.Lq + (clive ? cj : 0);
          const float l = clive ? p.lse[row] : -INFINITY;
          L2c = l == -INFINITY ? INFINITY : l * kLog2e;
          if (R == kDK) Dc = clive ? p.D[row] : 0.f;
          segc = (edge && clive && p.has_seg) ? p.seg_q[cj] : 0;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          bool vis = true;
          if (edge) {
            if (R == kDQ) {  // row: query at posr[i]; column: key cj
              vis = clive && cj <= posr[i];
              if (p.has_seg) vis = vis && (cj < p.P0 || segr[i] == segc);
            } else {  // row: key posr[i]; column: query at position cj + off
              vis = clive && int64_t(posr[i]) <= cj + p.off;
              if (p.has_seg) vis = vis && (posr[i] < p.P0 || segr[i] == segc);
            }
          }
          const float L2 = R == kDQ ? L2r[i] : L2c;
          const float pr = vis ? exp2f(fmaf(s1[i][m], p.scale_log2, -L2)) : 0.f;
          if (R == kDV)
            s1[i][m] = pr;
          else
            s1[i][m] = pr * (s2[i][m] - (R == kDQ ? Dr[i] : Dc));
        }
      }
      // slice [streamed row][8 rows]; row k's 16-byte chunk h (rows 4h .. 4h+3) sits at
      // chunk h ^ ((k >> 2) & 1), so a quarter warp's eight stores hit distinct banks
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int k = lane + 32 * m;
        const uint32_t a = sWw + k * 32;
        const int sw = (k >> 2) & 1;
        sts128(a + ((0 ^ sw) << 4), s1[0][m], s1[1][m], s1[2][m], s1[3][m]);
        sts128(a + ((1 ^ sw) << 4), s1[4][m], s1[5][m], s1[6][m], s1[7][m]);
      }
      __syncwarp();
    }

    // ---- accumulation: acc[8 rows][8 cols] += W^T Z over the tile's 128 streamed rows
#pragma unroll 1
    for (int zc = 0; zc < 8; ++zc) {
      const int cc = 8 * kPhases + zc;
      ok = __all_sync(0xffffffffu,
                      mbar_wait_bounded(slot_bar(cc & 3), uint32_t(cc >> 2) & 1u, p.wait_budget_ns, p.status));
      if (!ok) break;
      const uint32_t zslot = sRing + (cc & 3) * kSlotBytes;
      const uint32_t wrow = sWw + zc * kRowChunkRows * 32;
      float4 fw[2][2], fz[2][2];
      fw[0][0] = lds128(wrow);
      fw[0][1] = lds128(wrow + 16);
      fz[0][0] = lds128(zslot + zoff[0]);
      fz[0][1] = lds128(zslot + zoff[0] + 4 * kRowBlock);
#pragma unroll
      for (int kk = 0; kk < kRowChunkRows; ++kk) {
        const int cur = kk & 1, nxt = cur ^ 1;
        const int nk = min(kk + 1, kRowChunkRows - 1);  // the last prefetch re-reads row 15
        const int nsw = (nk >> 2) & 1;                  // (zc*16 + nk) >> 2 & 1 = (nk >> 2) & 1
        fw[nxt][0] = lds128(wrow + nk * 32 + ((0 ^ nsw) << 4));
        fw[nxt][1] = lds128(wrow + nk * 32 + ((1 ^ nsw) << 4));
        const uint32_t zrow = zslot + zoff[nk & 7] + (nk & ~7) * 128;
        fz[nxt][0] = lds128(zrow);
        fz[nxt][1] = lds128(zrow + 4 * kRowBlock);
        const float w8[8] = {fw[cur][0].x, fw[cur][0].y, fw[cur][0].z, fw[cur][0].w,
                             fw[cur][1].x, fw[cur][1].y, fw[cur][1].z, fw[cur][1].w};
        const float z8[8] = {fz[cur][0].x, fz[cur][0].y, fz[cur][0].z, fz[cur][0].w,
                             fz[cur][1].x, fz[cur][1].y, fz[cur][1].z, fz[cur][1].w};
#pragma unroll
        for (int r = 0; r < 8; ++r)
#pragma unroll
          for (int c = 0; c < 8; c += 2) ffma2(acc[r][c], acc[r][c + 1], w8[r], w8[r], z8[c], z8[c + 1]);
      }
      release(st, cc, use0 + uint32_t(cc >> 2));
    }
    if (!ok) break;
    ++t;
  }

  // ---- epilogue: the 8 gradient rows of this warp (columns 4l.., 128+4l..)
  if (ok) {
    const float sc = R == kDV ? 1.f : p.scale;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int r = 8 * warp + i;
      int64_t row;
      void* dst;
      if (R == kDQ) {
        const int hh = r / p.br;
        const int64_t qi = q0 + r % p.br;
        if (hh >= p.G || qi >= p.Lq) continue;
        row = int64_t(qhead0 + hh) * p.Lq + qi;
        dst = p.dq;
      } else {
        const int64_t kj = k0 + r;
        if (kj >= p.Lk) continue;
        row = int64_t(kvhead) * p.Lk + kj;
        dst = R == kDK ? p.dk : p.dv;
      }
      float* o = static_cast<float*>(dst) + row * kHeadDim;
      *reinterpret_cast<float4*>(o + 4 * lane) =
          make_float4(acc[i][0] * sc, acc[i][1] * sc, acc[i][2] * sc, acc[i][3] * sc);
      *reinterpret_cast<float4*>(o + 128 + 4 * lane) =
          make_float4(acc[i][4] * sc, acc[i][5] * sc, acc[i][6] * sc, acc[i][7] * sc);
    }
  }
  (void)bf16;
  __syncthreads();
  if (threadIdx.x == 0) {  // no copy may be in flight when the CTA ends (returns at once normally)
    mbar_wait_bounded(bar + 8 * kBarRes, uint32_t(R == kDV ? 0 : 1), p.wait_budget_ns, p.status);
    for (int s = 0; s < kSlots; ++s) {
      const uint32_t n = iss[s];
      if (n) mbar_wait_bounded(slot_bar(s), (n - 1) & 1u, p.wait_budget_ns, p.status);
    }
  }
}

__global__ void __launch_bounds__(kThreads) bwd_rowdot_kernel(BwdParams p, int64_t rows) {
  const int64_t row = int64_t(blockIdx.x) * (kThreads / 32) + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int lane = threadIdx.x & 31;
  const bool bf16 = p.bf16 != 0;
  float a[8], c[8];
  ld8(p.dout, row * kHeadDim + lane * 8, bf16, a);
  ld8(p.out, row * kHeadDim + lane * 8, bf16, c);
  float acc = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) acc = fmaf(a[i], c[i], acc);
#pragma unroll
  for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) p.D[row] = acc;
}

// 3-D map (d, position or key, head) of a [heads][L][256] fp32 tensor with a box of
// 32 d x box1 x box2, 128-byte swizzled.
bool map3d(EncodeTiledFn enc, CUtensorMap* m, const void* base, int64_t L, int64_t heads, int box1, int box2) {
  const cuuint32_t estr[3] = {1, 1, 1};
  const cuuint64_t dims[3] = {cuuint64_t(kHeadDim), cuuint64_t(L), cuuint64_t(heads)};
  const cuuint64_t strides[2] = {cuuint64_t(kHeadDim) * 4, cuuint64_t(L) * kHeadDim * 4};
  const cuuint32_t box[3] = {cuuint32_t(kBoxCols), cuuint32_t(box1), cuuint32_t(box2)};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 4-D map (d within a 32-column block, key, block, head) of a [heads][L][256] tensor.
bool map4d(EncodeTiledFn enc, CUtensorMap* m, const void* base, int64_t L, int64_t heads, int box1, int box2) {
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const cuuint64_t dims[4] = {cuuint64_t(kBoxCols), cuuint64_t(L), cuuint64_t(kHeadDim / kBoxCols),
                              cuuint64_t(heads)};
  const cuuint64_t strides[3] = {cuuint64_t(kHeadDim) * 4, cuuint64_t(kBoxCols) * 4, cuuint64_t(L) * kHeadDim * 4};
  const cuuint32_t box[4] = {cuuint32_t(kBoxCols), cuuint32_t(box1), cuuint32_t(box2), 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 4-D map (d within a 32-column block, position, head, block) of a [heads][L][256]
// tensor: a box of bpos positions x bheads heads x all 8 blocks lands as
// [block][head][position][32 d], i.e. [block][16 rows][128 bytes].
bool map_rows(EncodeTiledFn enc, CUtensorMap* m, const void* base, int64_t L, int64_t heads, int bpos, int bheads) {
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const cuuint64_t dims[4] = {cuuint64_t(kBoxCols), cuuint64_t(L), cuuint64_t(heads),
                              cuuint64_t(kHeadDim / kBoxCols)};
  const cuuint64_t strides[3] = {cuuint64_t(kHeadDim) * 4, cuuint64_t(L) * kHeadDim * 4, cuuint64_t(kBoxCols) * 4};
  const cuuint32_t box[4] = {cuuint32_t(kBoxCols), cuuint32_t(bpos), cuuint32_t(bheads),
                             cuuint32_t(kHeadDim / kBoxCols)};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int R>
int launch_role(const Maps& maps, const BwdParams& p, int units, cudaStream_t stream) {
  if (cudaFuncSetAttribute(bwd_ffma_kernel<R>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) !=
      cudaSuccess)
    return GQA_ERR_LAUNCH;
  if (units > 0) bwd_ffma_kernel<R><<<unsigned(units), kThreads, kSmemBytes, stream>>>(maps, p);
  return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_LAUNCH;
}

}  // namespace

int launch_bwd(const BwdArgs& a, cudaStream_t stream) {
  if (a.bf16) return launch_bwd_bf16(a, stream);
  BwdParams p;
  p.q = a.q;
  p.k = a.k;
  p.v = a.v;
  p.out = a.out;
  p.lse = a.lse;
  p.dout = a.dout;
  p.dq = a.dq;
  p.dk = a.dk;
  p.dv = a.dv;
  p.D = a.D;
  p.seg_q = a.seg_q;
  p.seg_kv = a.seg_kv;
  p.q_bounds = a.q_bounds;
  p.kv_bounds = a.kv_bounds;
  p.q_ranges = a.q_ranges;
  p.status = a.status;
  p.Lq = a.Lq;
  p.Lk = a.Lk;
  p.off = a.off;
  p.P0 = a.P0;
  p.wait_budget_ns = a.wait_budget_ns;
  p.test_skip_fill = a.test_skip_fill;
  p.B = a.B;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.G = a.Hq / a.Hkv;
  p.br = kBwdRowsQ / p.G;
  p.nq = int((a.Lq + p.br - 1) / p.br);
  p.nk = int((a.Lk + kBwdKeys - 1) / kBwdKeys);
  p.bq2 = 2 * p.br;
  p.nq2 = int((a.Lq + p.bq2 - 1) / p.bq2);
  p.nk64 = int((a.Lk + kRes - 1) / kRes);
  p.has_seg = a.seg_q != nullptr;
  p.bf16 = 0;
  p.scale = a.scale;
  p.scale_log2 = a.scale * kLog2e;
  const int64_t rows = int64_t(a.B) * a.Hq * a.Lq;
  if (rows > 0) {
    const int64_t blocks = (rows + 7) / 8;
    if (blocks > 0x7fffffff) return GQA_ERR_UNSUPPORTED;
    bwd_rowdot_kernel<<<unsigned(blocks), kThreads, 0, stream>>>(p, rows);
    if (cudaGetLastError() != cudaSuccess) return GQA_ERR_LAUNCH;
  }
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return GQA_ERR_LAUNCH;
  const int64_t qh = int64_t(a.B) * a.Hq, kh = int64_t(a.B) * a.Hkv;
  const int64_t dq_units = int64_t(p.nq) * kh, kv_units = int64_t(p.nk64) * kh;
  if (dq_units > 0x7fffffff || kv_units > 0x7fffffff) return GQA_ERR_UNSUPPORTED;
  // Row chunks of a query tile: 16 rows = min(16, bq2) positions x the heads to fill 16.
  const int bpos = p.bq2 < kRowChunkRows ? p.bq2 : kRowChunkRows, bheads = kRowChunkRows / bpos;
  Maps mq, mk, mv;
  // dQ: resident Q, dO (64/G positions x G heads); streamed K, V d-chunks and K rows.
  if (!map3d(enc, &mq.x1, a.q, a.Lq, qh, p.br, p.G) || !map3d(enc, &mq.x2, a.dout, a.Lq, qh, p.br, p.G) ||
      !map4d(enc, &mq.y1, a.k, a.Lk, kh, kStream, 1) || !map4d(enc, &mq.y2, a.v, a.Lk, kh, kStream, 1) ||
      !map4d(enc, &mq.z, a.k, a.Lk, kh, kRowChunkRows, kHeadDim / kBoxCols))
    return GQA_ERR_LAUNCH;
  // dK: resident K, V (64 keys); streamed Q, dO d-chunks (bq2 positions x G heads), Q rows.
  if (!map3d(enc, &mk.x1, a.k, a.Lk, kh, kRes, 1) || !map3d(enc, &mk.x2, a.v, a.Lk, kh, kRes, 1) ||
      !map3d(enc, &mk.y1, a.q, a.Lq, qh, p.bq2, p.G) || !map3d(enc, &mk.y2, a.dout, a.Lq, qh, p.bq2, p.G) ||
      !map_rows(enc, &mk.z, a.q, a.Lq, qh, bpos, bheads))
    return GQA_ERR_LAUNCH;
  // dV: resident K; streamed Q d-chunks and dO rows.
  mv = mk;
  if (!map_rows(enc, &mv.z, a.dout, a.Lq, qh, bpos, bheads)) return GQA_ERR_LAUNCH;
  int rc = launch_role<kDQ>(mq, p, int(dq_units), stream);
  if (rc == GQA_OK) rc = launch_role<kDK>(mk, p, int(kv_units), stream);
  if (rc == GQA_OK) rc = launch_role<kDV>(mv, p, int(kv_units), stream);
  return rc;
}

}  // namespace gqa
