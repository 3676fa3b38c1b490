// Attention backward (dQ, dK, dV from the saved LSE) on the FP32 pipe, sm_100a.
//
// Training over packed long sequences (maxtext PR #4929, description: the splash
// kernel runs inside training steps on 1,048,576-token packed batches) needs the
// gradients of the attention output.  With P = exp(scale * S - LSE) recomputed from
// the forward's log-sum-exp, D_i = <dO_i, O_i>, dP = dO V^T and dS = P * (dP - D):
//     dV_j = sum_{h in group} sum_i P_ij dO_i,   dK_j = scale * sum_{h in group} sum_i dS_ij Q_i,
//     dQ_i = scale * sum_j dS_ij K_j.
// Three kernels, no atomics:
//   bwd_rowdot_kernel  D = rowsum(dO * O), one warp per row.
//   bwd_dq_kernel      64 resident query rows (64/G positions x the G heads of a kv
//                      head), Q and dO; streams the key tiles (128 keys) of the query
//                      tile's range (the plan's block skipping): S = Q K^T, dP = dO V^T,
//                      dS, dQ += dS K.
//   bwd_dkv_kernel     32 resident keys of a kv head, K and V; streams the query tiles
//                      (128 rows = 128/G positions x the G heads) that see them.  Warps
//                      0-3 compute S^T = K Q^T, P^T and dV += P^T dO; warps 4-7 dP^T =
//                      V dO^T, dS^T (with P^T handed over through shared memory) and
//                      dK += dS^T Q.  S^T is computed once for both gradients and the G
//                      query heads' contributions to their key/value head sum on chip.
// The design is the forward FFMA kernel's (fwd_f32.cu).  Shared-memory wavefronts
// bound an FFMA contraction at d = 256: a warp's 128-bit shared load costs four
// wavefronts with distinct addresses and two when every lane reads one, and an SM
// moves one wavefront per cycle against two packed FMAs (fma.rn.f32x2).  So:
//   * the resident operands sit transposed in shared memory ([d][row]), written once
//     per CTA, so a row pair at one depth is a register pair, and every lane of a
//     warp reads the same fragment of its 8 resident rows;
//   * score-like products (S, dP, S^T, dP^T): lane l takes streamed rows l + 32 m
//     (m < 4), one accumulator per product: per depth, 2 broadcast loads (4
//     wavefronts) and 4 streamed values (4) for 16 packed FMAs;
//   * accumulations: the weights (dS, P^T, dS^T) go through a warp-private slice
//     [streamed row][8 resident rows] and are read as broadcasts; lane l owns columns
//     4l.. and 128+4l.. of its 8 gradient rows: per streamed row, 2 broadcast loads
//     (4) and 2 per-lane loads (8) for 32 packed FMAs.
// Streamed operands arrive as 16 KiB chunks, each ONE TMA copy (128-byte swizzle),
// through a ring of slots that the warps finishing a chunk last refill with the chunk
// one ring length ahead: "d-chunks" [128 rows][32 d] for the score-like products and
// "row chunks" [16 rows][256 d] for the accumulations.  The resident rows land in the
// ring first and are transposed from there.  fp32 only (bf16 calls use the
// tensor-core backward).
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
  int B, Hq, Hkv, G, br, nq, nk, has_seg;
  int bq2, nq2, nk32;  // dK / dV: query tiles of 128 / G positions; key tiles of 32
  int test_skip_fill;
  float scale, scale_log2;
};

// Eight consecutive fp32 elements (32-byte aligned).
__device__ __forceinline__ void ld8(const void* base, int64_t idx, float (&x)[8]) {
  const float4 a = *reinterpret_cast<const float4*>(static_cast<const float*>(base) + idx);
  const float4 b = *reinterpret_cast<const float4*>(static_cast<const float*>(base) + idx + 4);
  x[0] = a.x, x[1] = a.y, x[2] = a.z, x[3] = a.w, x[4] = b.x, x[5] = b.y, x[6] = b.z, x[7] = b.w;
}

// 128-bit shared load and store inside the region [lo, lo + n) the address belongs to:
// a checked build (GQA_DEBUG_BOUNDS) verifies the range, skips an access outside it and
// records the failure; other builds ignore lo and n.
__device__ __forceinline__ float4 lds128(uint32_t addr, uint32_t lo, uint32_t n) {
  float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
  if (!debug_region_ok(addr, 16, lo, n)) return v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr));
  return v;
}

__device__ __forceinline__ void sts128(uint32_t addr, uint32_t lo, uint32_t n, float a, float b, float c,
                                       float d) {
  if (!debug_region_ok(addr, 16, lo, n)) return;
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
// Tensor maps of the dQ kernel: resident Q, dO (8 boxes of 64 rows x 32 d each), K and
// V d-chunks (128 keys x 32 d) and K row chunks (16 keys x 256 d).
struct MapsQ {
  CUtensorMap q, dout, kd, vd, kr;
};

__global__ void __launch_bounds__(kThreads, 1) bwd_dq_kernel(const __grid_constant__ MapsQ maps,
                                                             const __grid_constant__ BwdParams p) {
  constexpr int kChunks = 24;  // per key tile: 8 K d-chunks, 8 V d-chunks, 8 K row chunks
  static_assert(kChunks % (2 * kSlots) == 0, "a tile is an even number of uses of every slot");
  extern __shared__ char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  const uint32_t sX1 = sbase + kOffX1, sX2 = sbase + kOffX2, sW = sbase + kOffW, sRing = sbase + kOffRing;
  const uint32_t bar = sbase + kOffBar;
  auto slot_bar = [&](int s) { return bar + 8u * uint32_t(kBarSlot + s); };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Unit: (query tile, kv head, batch), kv head by kv head, query tiles in descending
  // order (the longest key ranges first).
  const int nres = p.nq;
  const int rt = nres - 1 - int(blockIdx.x % unsigned(nres));
  const int hb = int(blockIdx.x / unsigned(nres));
  const int g = hb % p.Hkv, b = hb / p.Hkv;
  const int qhead0 = b * p.Hq + g * p.G;
  const int kvhead = b * p.Hkv + g;

  // Resident rows r = head (r / br) x position q0 + r % br.
  const int64_t q0 = int64_t(rt) * p.br;

  // Key tiles (128 keys) of the query tile's range from the plan.
  auto class_q = [&](int kt) {  // class of (query tile rt, key tile kt)
    const int64_t i1 = min(p.Lq, q0 + p.br) - 1;
    const int64_t j0 = int64_t(kt) * kStream, j1 = min(p.Lk, j0 + kStream) - 1;
    SegBounds qb{0, 0}, kb{0, 0};
    if (p.has_seg) {
      qb = SegBounds{p.q_bounds[2 * rt], p.q_bounds[2 * rt + 1]};
      kb = SegBounds{p.kv_bounds[2 * kt], p.kv_bounds[2 * kt + 1]};
    }
    return tile_class(q0, i1, j0, j1, p.off, p.P0, p.has_seg != 0, qb, kb);
  };
  int tbeg, tend;
  if (p.has_seg) {
    tbeg = p.q_ranges[2 * rt];
    tend = p.q_ranges[2 * rt + 1];
  } else {
    kv_range_no_seg(min(p.Lq, q0 + p.br) - 1, p.off, kStream, p.nk, &tbeg, &tend);
  }

  uint32_t* cnt = reinterpret_cast<uint32_t*>(smem_raw + (sbase + kOffCnt - raw));
  uint32_t* iss = reinterpret_cast<uint32_t*>(smem_raw + (sbase + kOffIss - raw));
  if (threadIdx.x == 0) {
    debug_flag_reset();
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
    while (st < tend && class_q(st) == GQA_TILE_SKIP) ++st;
    return st;
  };
  // Chunk c of key tile st into slot c % 4: c < 8: K d-block c; c < 16: V d-block c - 8;
  // else K row chunk c - 16 (keys st*128 + 16 (c - 16) ..).
  auto load_chunk = [&](int st, int c) {
    const int s = c & 3;
    const uint32_t u = atomicAdd(&iss[s], 1u);  // the u-th fill of slot s: chunk 4u + s of the stream
    if (int64_t(4) * u + s == p.test_skip_fill) return;  // test hook: never arrives
    mbar_arrive_expect_tx(slot_bar(s), kSlotBytes);
    const uint32_t dst = sRing + s * kSlotBytes;
    const int key0 = st * kStream;
    if (c < 8)
      tma_load_4d(dst, &maps.kd, slot_bar(s), 0, key0, c, kvhead);
    else if (c < 16)
      tma_load_4d(dst, &maps.vd, slot_bar(s), 0, key0, c - 8, kvhead);
    else
      tma_load_4d(dst, &maps.kr, slot_bar(s), 0, key0 + kRowChunkRows * (c - 16), 0, kvhead);
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
  // into Q^T and dO^T [d][row], one after the other.
  bool ok = true;
  for (int x = 0; x < 2; ++x) {
    if (threadIdx.x == 0) {
      if (x == 0) {
        tma_prefetch_desc(&maps.q);
        tma_prefetch_desc(&maps.dout);
        tma_prefetch_desc(&maps.kd);
        tma_prefetch_desc(&maps.vd);
        tma_prefetch_desc(&maps.kr);
      } else {
        fence_proxy_async_smem();  // the first round's staging reads come before these copies
      }
      const CUtensorMap* map = x == 0 ? &maps.q : &maps.dout;
      mbar_arrive_expect_tx(bar + 8 * kBarRes, 4 * kSlotBytes);
      for (int c = 0; c < 8; ++c)
        tma_load_3d(sRing + c * kResBox, map, bar + 8 * kBarRes, kBoxCols * c, int(q0), qhead0);
    }
    ok = ok && mbar_wait_bounded(bar + 8 * kBarRes, uint32_t(x), p.wait_budget_ns, p.status);
    if (ok) {
      const int r = threadIdx.x & 63;
      float* xt = reinterpret_cast<float*>(smem_raw + ((x == 0 ? sX1 : sX2) - raw));
#pragma unroll 4
      for (int cx = threadIdx.x >> 6; cx < 64; cx += kThreads / 64) {  // (block c, chunk q) of d
        const int c = cx >> 3, qq = cx & 7;
        const float4 v = lds128(sRing + c * kResBox + r * 128 + (uint32_t(qq ^ (r & 7)) << 4), sRing, 8 * kResBox);
        const int d = 32 * c + 4 * qq;
        if (!debug_index_ok((d + 3) * kRes + r, kRes * kHeadDim)) continue;
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
  // the warp's 8 query rows: log2-domain LSE, D, position (-1 past Lq; positions fit
  // int32: Lk = off + Lq < 2^31), segment id
  float L2r[8], Dr[8];
  int posr[8], segr[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = 8 * warp + i;
    const int hh = r / p.br;
    const int64_t qi = q0 + r % p.br;
    const bool live = hh < p.G && qi < p.Lq;
    const int64_t row = (int64_t(qhead0 + hh)) * p.Lq + qi;
    const float l = live ? p.lse[row] : -INFINITY;
    L2r[i] = l == -INFINITY ? INFINITY : l * kLog2e;
    Dr[i] = live ? p.D[row] : 0.f;
    posr[i] = live ? int(qi + p.off) : -1;
    segr[i] = (live && p.has_seg) ? p.seg_q[qi] : 0;
  }

  float acc[8][8];
#pragma unroll
  for (int r = 0; r < 8; ++r)
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[r][c] = 0.f;

  const uint32_t xw = 8 * warp * 4;  // the warp's rows in Q^T / dO^T
  const uint32_t kl = lane * 128 + ((lane & 7) << 4);
  uint32_t zoff[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) zoff[c] = (lane >> 3) * kRowBlock + c * 128 + (uint32_t(c ^ (lane & 7)) << 4);
  const uint32_t sWw = sW + warp * kWWarpBytes;

  uint32_t t = 0;  // tiles computed so far: slot uses (kChunks / 4) t ..
  for (int st = tbeg; st < tend && ok; ++st) {
    const int cls = class_q(st);
    if (cls == GQA_TILE_SKIP) continue;
    const uint32_t use0 = uint32_t(kChunks / 4) * t;

    // ---- S and dP: Q^T / dO^T row pairs (uniform) x keys l + 32 m of K / V d-chunks.
    float s1[8][4], s2[8][4];
    auto sphase = [&](float (&s)[8][4], const uint32_t xt, const int ph) {
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int m = 0; m < 4; ++m) s[i][m] = 0.f;
      float4 fq[4][2];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        fq[e][0] = lds128(xt + e * 256, xt - (8 * warp) * 4, kRes * kHeadDim * 4);
        fq[e][1] = lds128(xt + e * 256 + 16, xt - (8 * warp) * 4, kRes * kHeadDim * 4);
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
        for (int m = 0; m < 4; ++m) fk[m] = lds128(kslot + m * 4096, kslot - kl, kSlotBytes);
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
              if (e == 3 && x < 7) fk[m] = lds128((kslot ^ (uint32_t(x + 1) << 4)) + m * 4096, kslot - kl, kSlotBytes);
            }
            fq[e][0] = lds128(xt + (nd + e) * 256, xt - (8 * warp) * 4, kRes * kHeadDim * 4);
            fq[e][1] = lds128(xt + (nd + e) * 256 + 16, xt - (8 * warp) * 4, kRes * kHeadDim * 4);
          }
        }
        release(st, cc, use0 + uint32_t(cc >> 2));
      }
    };
    sphase(s1, sX1 + xw, 0);  // S = Q K^T
    if (!ok) break;
    sphase(s2, sX2 + xw, 1);  // dP = dO V^T
    if (!ok) break;

    // ---- dS = P (dP - D), P = exp2(S c - L2)
    {
      const int64_t j0 = int64_t(st) * kStream;
      const bool edge = cls == GQA_TILE_PARTIAL || j0 + kStream > p.Lk;
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int cj = int(j0 + lane + 32 * m);  // key
        const bool clive = cj < p.Lk;
        const int segc = (edge && clive && p.has_seg) ? p.seg_kv[cj] : 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          bool vis = true;
          if (edge) {
            vis = clive && cj <= posr[i];
            if (p.has_seg) vis = vis && (cj < p.P0 || segr[i] == segc);
          }
          const float pr = vis ? exp2f(fmaf(s1[i][m], p.scale_log2, -L2r[i])) : 0.f;
          s1[i][m] = pr * (s2[i][m] - Dr[i]);
        }
      }
      // slice [key][8 rows]; row k's 16-byte chunk h (rows 4h .. 4h+3) sits at
      // chunk h ^ ((k >> 2) & 1), so a quarter warp's eight stores hit distinct banks
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int k = lane + 32 * m;
        const uint32_t a = sWw + k * 32;
        const int sw = (k >> 2) & 1;
        sts128(a + ((0 ^ sw) << 4), sWw, kWWarpBytes, s1[0][m], s1[1][m], s1[2][m], s1[3][m]);
        sts128(a + ((1 ^ sw) << 4), sWw, kWWarpBytes, s1[4][m], s1[5][m], s1[6][m], s1[7][m]);
      }
      __syncwarp();
    }

    // ---- dQ[8 rows][8 cols] += dS K over the tile's 128 keys (K row chunks)
#pragma unroll 1
    for (int zc = 0; zc < 8; ++zc) {
      const int cc = 16 + zc;
      ok = __all_sync(0xffffffffu,
                      mbar_wait_bounded(slot_bar(cc & 3), uint32_t(cc >> 2) & 1u, p.wait_budget_ns, p.status));
      if (!ok) break;
      const uint32_t zslot = sRing + (cc & 3) * kSlotBytes;
      const uint32_t wrow = sWw + zc * kRowChunkRows * 32;
      float4 fw[2][2], fz[2][2];
      fw[0][0] = lds128(wrow, sWw, kWWarpBytes);
      fw[0][1] = lds128(wrow + 16, sWw, kWWarpBytes);
      fz[0][0] = lds128(zslot + zoff[0], zslot, kSlotBytes);
      fz[0][1] = lds128(zslot + zoff[0] + 4 * kRowBlock, zslot, kSlotBytes);
#pragma unroll
      for (int kk = 0; kk < kRowChunkRows; ++kk) {
        const int cur = kk & 1, nxt = cur ^ 1;
        const int nk = min(kk + 1, kRowChunkRows - 1);  // the last prefetch re-reads row 15
        const int nsw = (nk >> 2) & 1;                  // (zc*16 + nk) >> 2 & 1 = (nk >> 2) & 1
        fw[nxt][0] = lds128(wrow + nk * 32 + ((0 ^ nsw) << 4), sWw, kWWarpBytes);
        fw[nxt][1] = lds128(wrow + nk * 32 + ((1 ^ nsw) << 4), sWw, kWWarpBytes);
        const uint32_t zrow = zslot + zoff[nk & 7] + (nk & ~7) * 128;
        fz[nxt][0] = lds128(zrow, zslot, kSlotBytes);
        fz[nxt][1] = lds128(zrow + 4 * kRowBlock, zslot, kSlotBytes);
        const float w8[8] = {fw[cur][0].x, fw[cur][0].y, fw[cur][0].z, fw[cur][0].w,
                             fw[cur][1].x, fw[cur][1].y, fw[cur][1].z, fw[cur][1].w};
        const float z8[8] = {fz[cur][0].x, fz[cur][0].y, fz[cur][0].z, fz[cur][0].w,
                             fz[cur][1].x, fz[cur][1].y, fz[cur][1].z, fz[cur][1].w};
        // column pair outermost: runs of eight packed FMAs share one register pair
#pragma unroll
        for (int c = 0; c < 8; c += 2)
#pragma unroll
          for (int r = 0; r < 8; ++r) ffma2(acc[r][c], acc[r][c + 1], w8[r], w8[r], z8[c], z8[c + 1]);
      }
      release(st, cc, use0 + uint32_t(cc >> 2));
    }
    if (!ok) break;
    ++t;
  }

  // ---- epilogue: dQ of the warp's 8 rows (columns 4l.., 128+4l..), scaled
  if (ok) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int r = 8 * warp + i;
      const int hh = r / p.br;
      const int64_t qi = q0 + r % p.br;
      if (hh >= p.G || qi >= p.Lq) continue;
      if (!debug_index_ok(int64_t(qhead0 + hh) * p.Lq + qi, int64_t(p.B) * p.Hq * p.Lq)) continue;
      float* o = static_cast<float*>(p.dq) + (int64_t(qhead0 + hh) * p.Lq + qi) * kHeadDim;
      *reinterpret_cast<float4*>(o + 4 * lane) =
          make_float4(acc[i][0] * p.scale, acc[i][1] * p.scale, acc[i][2] * p.scale, acc[i][3] * p.scale);
      *reinterpret_cast<float4*>(o + 128 + 4 * lane) =
          make_float4(acc[i][4] * p.scale, acc[i][5] * p.scale, acc[i][6] * p.scale, acc[i][7] * p.scale);
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {  // no copy may be in flight when the CTA ends (returns at once normally)
    mbar_wait_bounded(bar + 8 * kBarRes, 1u, p.wait_budget_ns, p.status);
    for (int s = 0; s < kSlots; ++s) {
      const uint32_t n = iss[s];
      if (n) mbar_wait_bounded(slot_bar(s), (n - 1) & 1u, p.wait_budget_ns, p.status);
    }
    debug_flag_report(p.status);
  }
}

// ---------------------------------------------------------------------------------
// dK and dV together: 32 resident keys of a kv head; warps 0-3 (half A) accumulate dV,
// warps 4-7 (half B) dK, and warps a and a + 4 share keys 8a .. 8a+7.  Per query tile
// (128 rows): A computes S^T = K Q^T over Q's d-chunks, P^T = exp2(S^T c - L2), hands
// P^T to B through its shared-memory slice and accumulates dV += P^T dO over dO's row
// chunks; B computes dP^T = V dO^T over dO's d-chunks, takes P^T, forms dS^T = P^T
// (dP^T - D) and accumulates dK += dS^T Q over Q's row chunks.  S^T is computed once
// for both gradients.  The hand-off uses two mbarriers per pair (P^T written / read),
// with bounded waits like every other wait.
constexpr int kResKV = 32;
constexpr int kSlotsKV = 8;          // even chunks (half A) in even slots, odd chunks (B) in odd slots
constexpr int kChunksKV = 32;        // per tile: 8 Q and 8 dO d-chunks interleaved, then 8 dO and 8 Q row chunks
constexpr int kResBoxKV = kResKV * 128;  // staging: 32 keys x 32 d (4 KiB)
constexpr int kOffKT = 0;                                   // K^T [256 d][32 keys]
constexpr int kOffVT = kOffKT + kResKV * kHeadDim * 4;      // V^T
constexpr int kOffWKV = kOffVT + kResKV * kHeadDim * 4;     // weight slices, 4 KiB per warp
constexpr int kOffRingKV = kOffWKV + kWarps * kWWarpBytes;
constexpr int kOffBarKV = kOffRingKV + kSlotsKV * kSlotBytes;
enum { kBarResKV = 0, kBarSlotKV = 1, kBarFullKV = 9, kBarEmptyKV = 13, kNumBarsKV = 17 };
constexpr int kOffCntKV = kOffBarKV + 8 * kNumBarsKV;
constexpr int kOffIssKV = kOffCntKV + 4 * kSlotsKV;
constexpr int kSmemBytesKV = kOffIssKV + 4 * kSlotsKV + 1024;
static_assert(kSmemBytesKV <= 232448, "shared memory per block");
static_assert(16 * kResBoxKV == 4 * kSlotBytes, "K and V staged in four ring slots");

struct MapsKV {
  CUtensorMap k, v, qd, dod, qr, dor;  // resident K, V; Q, dO d-chunks; Q, dO row chunks
};

__global__ void __launch_bounds__(kThreads, 1) bwd_dkv_kernel(const __grid_constant__ MapsKV maps,
                                                              const __grid_constant__ BwdParams p) {
  extern __shared__ char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  const uint32_t sKT = sbase + kOffKT, sVT = sbase + kOffVT, sW = sbase + kOffWKV, sRing = sbase + kOffRingKV;
  const uint32_t bar = sbase + kOffBarKV;
  auto B_ = [&](int i) { return bar + 8u * uint32_t(i); };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int half = warp >> 2, a = warp & 3;  // half 0: dV (S^T, P^T); half 1: dK (dP^T, dS^T)

  // Unit: (key tile of 32, kv head, batch), kv head by kv head, keys ascending (the
  // earliest keys see the most queries).
  const int nres = p.nk32;
  const int rt = int(blockIdx.x % unsigned(nres));
  const int hb = int(blockIdx.x / unsigned(nres));
  const int g = hb % p.Hkv, b = hb / p.Hkv;
  const int qhead0 = b * p.Hq + g * p.G;
  const int kvhead = b * p.Hkv + g;
  const int64_t k0 = int64_t(rt) * kResKV;

  __shared__ int range[2];
  auto class_kv = [&](int qt2) {  // class of (query tile qt2, keys [k0, k0 + 32))
    const int64_t i0 = int64_t(qt2) * p.bq2, i1 = min(p.Lq, i0 + p.bq2) - 1;
    const int64_t j1 = min(p.Lk, k0 + kResKV) - 1;
    SegBounds qb{0, 0}, kb{0, 0};
    if (p.has_seg) {  // plan tiles: query tiles of br = bq2 / 2 positions, key tiles of 128
      const int x0 = 2 * qt2, x1 = min(2 * qt2 + 1, p.nq - 1);
      qb = SegBounds{min(p.q_bounds[2 * x0], p.q_bounds[2 * x1]), max(p.q_bounds[2 * x0 + 1], p.q_bounds[2 * x1 + 1])};
      const int kt = int(k0 / 128);
      kb = SegBounds{p.kv_bounds[2 * kt], p.kv_bounds[2 * kt + 1]};
    }
    return tile_class(i0, i1, k0, j1, p.off, p.P0, p.has_seg != 0, qb, kb);
  };
  // Query tiles that can see keys [k0, k0 + 32): causally from the first row at
  // position >= k0 (every row for a shared-state key), and with segment ids the first
  // and last tile that is not SKIP, found by the whole CTA.
  int tbeg = (k0 < p.P0 || k0 <= p.off) ? 0 : int((k0 - p.off) / p.bq2);
  int tend = p.nq2;
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

  uint32_t* cnt = reinterpret_cast<uint32_t*>(smem_raw + (sbase + kOffCntKV - raw));
  uint32_t* iss = reinterpret_cast<uint32_t*>(smem_raw + (sbase + kOffIssKV - raw));
  if (threadIdx.x == 0) {
    debug_flag_reset();
    mbar_init(B_(kBarResKV), 1);
    for (int s = 0; s < kSlotsKV; ++s) {
      mbar_init(B_(kBarSlotKV + s), 1);
      cnt[s] = 0;
      iss[s] = 0;
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(B_(kBarFullKV + i), 1);
      mbar_init(B_(kBarEmptyKV + i), 1);
    }
    fence_barrier_init();
  }
  __syncthreads();

  auto next_tile = [&](int st) {
    while (st < tend && class_kv(st) == GQA_TILE_SKIP) ++st;
    return st;
  };
  // Chunk c of query tile st into slot c % 8: c < 16: d-block c / 2 of Q (even) or dO
  // (odd); c >= 16: row chunk (c - 16) / 2 of dO (even) or Q (odd).
  auto load_chunk = [&](int st, int c) {
    const int s = c & (kSlotsKV - 1);
    const uint32_t u = atomicAdd(&iss[s], 1u);  // the u-th fill of slot s: chunk 8u + s of the stream
    if (int64_t(kSlotsKV) * u + s == p.test_skip_fill) return;  // test hook: never arrives
    mbar_arrive_expect_tx(B_(kBarSlotKV + s), kSlotBytes);
    const uint32_t dst = sRing + s * kSlotBytes;
    const int pos0 = st * p.bq2;
    if (c < 16) {
      tma_load_3d(dst, (c & 1) ? &maps.dod : &maps.qd, B_(kBarSlotKV + s), kBoxCols * (c >> 1), pos0, qhead0);
    } else {
      const int r0 = kRowChunkRows * ((c - 16) >> 1);
      tma_load_4d(dst, (c & 1) ? &maps.qr : &maps.dor, B_(kBarSlotKV + s), 0, pos0 + r0 % p.bq2,
                  qhead0 + r0 / p.bq2, 0);
    }
  };
  // The last of the half's four warps done with chunk c issues chunk c + 8 (the same
  // half's next chunk in this slot).
  auto release = [&](int st, int c, uint32_t use) {
    __syncwarp();
    if (lane == 0) {
      __threadfence_block();
      const int s = c & (kSlotsKV - 1);
      if (atomicAdd(&cnt[s], 1u) == 4u * (use + 1) - 1) {
        if (c + kSlotsKV < kChunksKV) {
          load_chunk(st, c + kSlotsKV);
        } else {
          const int sn = next_tile(st + 1);
          if (sn < tend) load_chunk(sn, c + kSlotsKV - kChunksKV);
        }
      }
    }
  };

  // ---- resident keys: K and V staged in the ring (8 boxes of 32 keys x 32 d each),
  // transposed into K^T and V^T [d][key].
  if (threadIdx.x == 0) {
    tma_prefetch_desc(&maps.k);
    tma_prefetch_desc(&maps.v);
    tma_prefetch_desc(&maps.qd);
    tma_prefetch_desc(&maps.dod);
    tma_prefetch_desc(&maps.qr);
    tma_prefetch_desc(&maps.dor);
    mbar_arrive_expect_tx(B_(kBarResKV), 16 * kResBoxKV);
    for (int c = 0; c < 8; ++c) {
      tma_load_3d(sRing + c * kResBoxKV, &maps.k, B_(kBarResKV), kBoxCols * c, int(k0), kvhead);
      tma_load_3d(sRing + (8 + c) * kResBoxKV, &maps.v, B_(kBarResKV), kBoxCols * c, int(k0), kvhead);
    }
  }
  bool ok = mbar_wait_bounded(B_(kBarResKV), 0, p.wait_budget_ns, p.status);
  if (ok) {
    const int r = threadIdx.x & 31;
    for (int op = 0; op < 2; ++op) {
      float* xt = reinterpret_cast<float*>(smem_raw + ((op == 0 ? sKT : sVT) - raw));
      const uint32_t stage = sRing + op * 8 * kResBoxKV;
#pragma unroll 4
      for (int cx = threadIdx.x >> 5; cx < 64; cx += kThreads / 32) {  // (block c, chunk x) of d
        const int c = cx >> 3, x = cx & 7;
        const float4 v = lds128(stage + c * kResBoxKV + r * 128 + (uint32_t(x ^ (r & 7)) << 4), stage, 8 * kResBoxKV);
        const int d = 32 * c + 4 * x;
        if (!debug_index_ok((d + 3) * kResKV + r, kResKV * kHeadDim)) continue;
        xt[(d + 0) * kResKV + r] = v.x;
        xt[(d + 1) * kResKV + r] = v.y;
        xt[(d + 2) * kResKV + r] = v.z;
        xt[(d + 3) * kResKV + r] = v.w;
      }
    }
  }
  ok = __syncthreads_and(ok);
  if (threadIdx.x == 0) {
    fence_proxy_async_smem();  // the staging reads above come before the copies below
    const int s0 = ok ? next_tile(tbeg) : tend;
    if (s0 < tend)
      for (int c = 0; c < kSlotsKV; ++c) load_chunk(s0, c);
  }

  // keys 8a + i of this pair
  int posr[8], segr[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int64_t kj = k0 + 8 * a + i;
    posr[i] = kj < p.Lk ? int(kj) : 0x7fffffff;  // a key past Lk is seen by no row
    segr[i] = (kj < p.Lk && p.has_seg) ? p.seg_kv[kj] : 0;
  }
  float acc[8][8];
#pragma unroll
  for (int r = 0; r < 8; ++r)
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[r][c] = 0.f;

  const uint32_t xt = (half == 0 ? sKT : sVT) + 8 * a * 4;  // this pair's keys in K^T / V^T
  const uint32_t kl = lane * 128 + ((lane & 7) << 4);
  uint32_t zoff[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) zoff[c] = (lane >> 3) * kRowBlock + c * 128 + (uint32_t(c ^ (lane & 7)) << 4);
  const uint32_t sWw = sW + warp * kWWarpBytes;  // this warp's slice
  const uint32_t sWa = sW + a * kWWarpBytes;     // the pair's P^T (half A's slice)

  uint32_t t = 0;  // tiles computed so far: slot uses 4t .. 4t+3
  for (int st = tbeg; st < tend && ok; ++st) {
    const int cls = class_kv(st);
    if (cls == GQA_TILE_SKIP) continue;
    const uint32_t use0 = 4u * t;

    // ---- S^T (half A) or dP^T (half B): key pairs of K^T / V^T (uniform) x query rows
    // l + 32 m of Q / dO d-chunks
    float s[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int m = 0; m < 4; ++m) s[i][m] = 0.f;
    {
      float4 fq[4][2];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        fq[e][0] = lds128(xt + e * (kResKV * 4), xt - 8 * a * 4, kResKV * kHeadDim * 4);
        fq[e][1] = lds128(xt + e * (kResKV * 4) + 16, xt - 8 * a * 4, kResKV * kHeadDim * 4);
      }
#pragma unroll 1
      for (int j = 0; j < 8; ++j) {
        const int cc = 2 * j + half;
        const int slot = cc & (kSlotsKV - 1);
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(B_(kBarSlotKV + slot), uint32_t(cc >> 3) & 1u,
                                                        p.wait_budget_ns, p.status));
        if (!ok) break;
        const uint32_t kslot = sRing + slot * kSlotBytes + kl;
        float4 fk[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) fk[m] = lds128(kslot + m * 4096, kslot - kl, kSlotBytes);
#pragma unroll
        for (int x = 0; x < 8; ++x) {  // depth step: d = 32 j + 4 x + e
          const int nd = (32 * j + 4 * (x + 1)) & (kHeadDim - 1);  // the last step re-reads depth 0
#pragma unroll
          for (int e = 0; e < 4; ++e) {
#pragma unroll
            for (int m = 0; m < 4; ++m) {
              const float kv = e == 0 ? fk[m].x : e == 1 ? fk[m].y : e == 2 ? fk[m].z : fk[m].w;
              ffma2(s[0][m], s[1][m], fq[e][0].x, fq[e][0].y, kv, kv);
              ffma2(s[2][m], s[3][m], fq[e][0].z, fq[e][0].w, kv, kv);
              ffma2(s[4][m], s[5][m], fq[e][1].x, fq[e][1].y, kv, kv);
              ffma2(s[6][m], s[7][m], fq[e][1].z, fq[e][1].w, kv, kv);
              if (e == 3 && x < 7) fk[m] = lds128((kslot ^ (uint32_t(x + 1) << 4)) + m * 4096, kslot - kl, kSlotBytes);
            }
            fq[e][0] = lds128(xt + (nd + e) * (kResKV * 4), xt - 8 * a * 4, kResKV * kHeadDim * 4);
            fq[e][1] = lds128(xt + (nd + e) * (kResKV * 4) + 16, xt - 8 * a * 4, kResKV * kHeadDim * 4);
          }
        }
        release(st, cc, use0 + uint32_t(cc >> 3));
      }
    }
    if (!ok) break;

    // ---- weights.  Query row of this lane's column m: tile row l + 32 m = head hh,
    // position cj (index in Lq).
    const int64_t c0 = int64_t(st) * p.bq2;
    const bool edge = cls == GQA_TILE_PARTIAL || c0 + p.bq2 > p.Lq || k0 + kResKV > p.Lk;
    if (half == 0) {
      // P^T = exp2(S^T c - L2) into this warp's slice, once B has read the last one
      if (t > 0) {
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(B_(kBarEmptyKV + a), (t - 1) & 1u, p.wait_budget_ns,
                                                        p.status));
        if (!ok) break;
      }
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int cr = lane + 32 * m;
        const int hh = cr / p.bq2;
        const int cj = int(c0 + cr % p.bq2);
        const bool clive = cj < p.Lq;
        const int64_t row = int64_t(qhead0 + hh) * p.Lq + (clive ? cj : 0);
        const float l = clive ? p.lse[row] : -INFINITY;
        const float L2c = l == -INFINITY ? INFINITY : l * kLog2e;
        const int segc = (edge && clive && p.has_seg) ? p.seg_q[cj] : 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          bool vis = true;
          if (edge) {  // row: key posr[i]; column: query at position cj + off
            vis = clive && int64_t(posr[i]) <= cj + p.off;
            if (p.has_seg) vis = vis && (posr[i] < p.P0 || segr[i] == segc);
          }
          s[i][m] = vis ? exp2f(fmaf(s[i][m], p.scale_log2, -L2c)) : 0.f;
        }
      }
    } else {
      // dS^T = P^T (dP^T - D), P^T read from the pair's slice once A has written it
      ok = __all_sync(0xffffffffu, mbar_wait_bounded(B_(kBarFullKV + a), t & 1u, p.wait_budget_ns, p.status));
      if (!ok) break;
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int cr = lane + 32 * m;
        const int sw = (cr >> 2) & 1;
        const float4 p0 = lds128(sWa + cr * 32 + ((0 ^ sw) << 4), sWa, kWWarpBytes);
        const float4 p1 = lds128(sWa + cr * 32 + ((1 ^ sw) << 4), sWa, kWWarpBytes);
        const int hh = cr / p.bq2;
        const int cj = int(c0 + cr % p.bq2);
        const bool clive = cj < p.Lq;
        const float Dc = clive ? p.D[int64_t(qhead0 + hh) * p.Lq + cj] : 0.f;
        const float pv[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) s[i][m] = pv[i] * (s[i][m] - Dc);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(B_(kBarEmptyKV + a));  // the pair's P^T slice may be rewritten
    }
    // this warp's slice [query row][8 keys] (P^T for A, dS^T for B); row k's chunk h
    // (keys 4h .. 4h+3) sits at chunk h ^ ((k >> 2) & 1)
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const int k = lane + 32 * m;
      const uint32_t ad = sWw + k * 32;
      const int sw = (k >> 2) & 1;
      sts128(ad + ((0 ^ sw) << 4), sWw, kWWarpBytes, s[0][m], s[1][m], s[2][m], s[3][m]);
      sts128(ad + ((1 ^ sw) << 4), sWw, kWWarpBytes, s[4][m], s[5][m], s[6][m], s[7][m]);
    }
    __syncwarp();
    if (half == 0 && lane == 0) mbar_arrive(B_(kBarFullKV + a));  // P^T of this tile is in place

    // ---- accumulation over the half's row chunks: dV += P^T dO (A), dK += dS^T Q (B)
#pragma unroll 1
    for (int zc = 0; zc < 8; ++zc) {
      const int cc = 16 + 2 * zc + half;
      const int slot = cc & (kSlotsKV - 1);
      ok = __all_sync(0xffffffffu, mbar_wait_bounded(B_(kBarSlotKV + slot), uint32_t(cc >> 3) & 1u,
                                                      p.wait_budget_ns, p.status));
      if (!ok) break;
      const uint32_t zslot = sRing + slot * kSlotBytes;
      const uint32_t wrow = sWw + zc * kRowChunkRows * 32;
      float4 fw[2][2], fz[2][2];
      fw[0][0] = lds128(wrow, sWw, kWWarpBytes);
      fw[0][1] = lds128(wrow + 16, sWw, kWWarpBytes);
      fz[0][0] = lds128(zslot + zoff[0], zslot, kSlotBytes);
      fz[0][1] = lds128(zslot + zoff[0] + 4 * kRowBlock, zslot, kSlotBytes);
#pragma unroll
      for (int kk = 0; kk < kRowChunkRows; ++kk) {
        const int cur = kk & 1, nxt = cur ^ 1;
        const int nk = min(kk + 1, kRowChunkRows - 1);  // the last prefetch re-reads row 15
        const int nsw = (nk >> 2) & 1;
        fw[nxt][0] = lds128(wrow + nk * 32 + ((0 ^ nsw) << 4), sWw, kWWarpBytes);
        fw[nxt][1] = lds128(wrow + nk * 32 + ((1 ^ nsw) << 4), sWw, kWWarpBytes);
        const uint32_t zrow = zslot + zoff[nk & 7] + (nk & ~7) * 128;
        fz[nxt][0] = lds128(zrow, zslot, kSlotBytes);
        fz[nxt][1] = lds128(zrow + 4 * kRowBlock, zslot, kSlotBytes);
        const float w8[8] = {fw[cur][0].x, fw[cur][0].y, fw[cur][0].z, fw[cur][0].w,
                             fw[cur][1].x, fw[cur][1].y, fw[cur][1].z, fw[cur][1].w};
        const float z8[8] = {fz[cur][0].x, fz[cur][0].y, fz[cur][0].z, fz[cur][0].w,
                             fz[cur][1].x, fz[cur][1].y, fz[cur][1].z, fz[cur][1].w};
        // column pair outermost: runs of eight packed FMAs share one register pair
#pragma unroll
        for (int c = 0; c < 8; c += 2)
#pragma unroll
          for (int r = 0; r < 8; ++r) ffma2(acc[r][c], acc[r][c + 1], w8[r], w8[r], z8[c], z8[c + 1]);
      }
      release(st, cc, use0 + uint32_t(cc >> 3));
    }
    if (!ok) break;
    ++t;
  }

  // ---- epilogue: dV (half A) or dK (half B) of the pair's 8 keys
  if (ok) {
    const float sc = half == 0 ? 1.f : p.scale;
    float* dst = static_cast<float*>(half == 0 ? p.dv : p.dk);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int64_t kj = k0 + 8 * a + i;
      if (kj >= p.Lk) continue;
      if (!debug_index_ok(int64_t(kvhead) * p.Lk + kj, int64_t(p.B) * p.Hkv * p.Lk)) continue;
      float* o = dst + (int64_t(kvhead) * p.Lk + kj) * kHeadDim;
      *reinterpret_cast<float4*>(o + 4 * lane) =
          make_float4(acc[i][0] * sc, acc[i][1] * sc, acc[i][2] * sc, acc[i][3] * sc);
      *reinterpret_cast<float4*>(o + 128 + 4 * lane) =
          make_float4(acc[i][4] * sc, acc[i][5] * sc, acc[i][6] * sc, acc[i][7] * sc);
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {  // no copy may be in flight when the CTA ends (returns at once normally)
    mbar_wait_bounded(B_(kBarResKV), 0, p.wait_budget_ns, p.status);
    for (int s = 0; s < kSlotsKV; ++s) {
      const uint32_t n = iss[s];
      if (n) mbar_wait_bounded(B_(kBarSlotKV + s), (n - 1) & 1u, p.wait_budget_ns, p.status);
    }
    debug_flag_report(p.status);
  }
}

__global__ void __launch_bounds__(kThreads) bwd_rowdot_kernel(BwdParams p, int64_t rows) {
  const int64_t row = int64_t(blockIdx.x) * (kThreads / 32) + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int lane = threadIdx.x & 31;
  float a[8], c[8];
  ld8(p.dout, row * kHeadDim + lane * 8, a);
  ld8(p.out, row * kHeadDim + lane * 8, c);
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
  p.nk32 = int((a.Lk + kResKV - 1) / kResKV);
  p.has_seg = a.seg_q != nullptr;
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
  const int64_t dq_units = int64_t(p.nq) * kh, kv_units = int64_t(p.nk32) * kh;
  if (dq_units > 0x7fffffff || kv_units > 0x7fffffff) return GQA_ERR_UNSUPPORTED;
  // Row chunks of a query tile: 16 rows = min(16, bq2) positions x the heads to fill 16.
  const int bpos = p.bq2 < kRowChunkRows ? p.bq2 : kRowChunkRows, bheads = kRowChunkRows / bpos;
  MapsQ mq;
  // dQ: resident Q, dO (64/G positions x G heads); streamed K, V d-chunks and K rows.
  if (!map3d(enc, &mq.q, a.q, a.Lq, qh, p.br, p.G) || !map3d(enc, &mq.dout, a.dout, a.Lq, qh, p.br, p.G) ||
      !map4d(enc, &mq.kd, a.k, a.Lk, kh, kStream, 1) || !map4d(enc, &mq.vd, a.v, a.Lk, kh, kStream, 1) ||
      !map4d(enc, &mq.kr, a.k, a.Lk, kh, kRowChunkRows, kHeadDim / kBoxCols))
    return GQA_ERR_LAUNCH;
  // dK and dV: resident K, V (32 keys); streamed Q, dO d-chunks (bq2 positions x G heads)
  // and Q, dO row chunks.
  MapsKV mkv;
  if (!map3d(enc, &mkv.k, a.k, a.Lk, kh, kResKV, 1) || !map3d(enc, &mkv.v, a.v, a.Lk, kh, kResKV, 1) ||
      !map3d(enc, &mkv.qd, a.q, a.Lq, qh, p.bq2, p.G) || !map3d(enc, &mkv.dod, a.dout, a.Lq, qh, p.bq2, p.G) ||
      !map_rows(enc, &mkv.qr, a.q, a.Lq, qh, bpos, bheads) || !map_rows(enc, &mkv.dor, a.dout, a.Lq, qh, bpos, bheads))
    return GQA_ERR_LAUNCH;
  if (cudaFuncSetAttribute(bwd_dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) != cudaSuccess ||
      cudaFuncSetAttribute(bwd_dkv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytesKV) != cudaSuccess)
    return GQA_ERR_LAUNCH;
  if (dq_units > 0) bwd_dq_kernel<<<unsigned(dq_units), kThreads, kSmemBytes, stream>>>(mq, p);
  if (cudaGetLastError() != cudaSuccess) return GQA_ERR_LAUNCH;
  if (kv_units > 0) bwd_dkv_kernel<<<unsigned(kv_units), kThreads, kSmemBytesKV, stream>>>(mkv, p);
  const int rc = cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_LAUNCH;
  return rc;
}

}  // namespace gqa
