// fp32 attention forward on the FP32 pipe (FFMA), sm_100a.
//
// kev PR #202 ("Why fp32 fell to the L x L kernel", "The change") evaluates its
// models in fp32 with TF32 off and needs the fp32 path to run in memory linear in
// L without repeating the 4 key/value heads for the 16 query heads.  This kernel
// does both: one CTA owns a tile of 64 query rows = (64 / G) positions x all G
// query heads that share one key/value head, so every key/value tile it stages in
// shared memory serves G heads, and scores live only in registers.
//
// CTA = 8 warps (256 threads, 2 per SM sub-partition, up to 255 registers each;
// 1 CTA per SM).  Key tiles hold 256 keys.  Warp w owns query rows 8w .. 8w+7 for
// the whole key loop, every lane all 8 of them:
//   S = Q K^T   lane l: 8 rows x keys l + 32 m (m < 8); Q^T fragments warp-uniform
//   softmax     online, base 2, row max by warp shuffles over 32 lanes; each lane
//               keeps its own partial row sums (reduced once, at the end)
//   O += P V    lane l: 8 rows x cols 4l.., 128+4l.. (P fragments warp-uniform)
// P goes through a warp-private 4 KiB slice of shared memory (half a tile at a time),
// so warps never wait for one another inside the key loop.
//
// Why these register tiles.  Shared-memory bandwidth bounds an FFMA attention at
// d = 256: a warp's 128-bit shared load costs four data wavefronts when its lanes
// read distinct addresses and two when they all read one (ncu), the SM moves one
// wavefront per cycle, and its four sub-partitions retire two packed FMAs
// (fma.rn.f32x2) per cycle -- so a loop needs more than 2 packed FMAs per wavefront
// to leave the FP32 pipe the bound.  S pairs rows at one depth, (S[r][j], S[r+1][j]) +=
// (q[r], q[r+1]) * (k[j], k[j]): Q is kept transposed in shared memory ([d][row],
// written once per CTA), so the row pairs are natural register pairs and a score needs
// one accumulator register, which leaves room for 8 keys per lane: per depth, 2
// broadcast Q^T loads (4 wavefronts) and 8 keys' worth of K (8) feed 32 packed FMAs,
// 2.67 per wavefront.  PV takes, per key, 2 broadcast P loads (4) and 2 V loads (8)
// for 32 packed FMAs, also 2.67.  (Values stored once are duplicated into the (v, v)
// operand pairs in registers.)
//
// Key/value streaming.  A 256-key tile is 16 chunks of 32 KiB: K's eight 32-column
// blocks of d ([256 keys][32 d]) and then V's eight groups of 32 keys ([32 keys][256
// d]), each ONE 4-D TMA copy (128-byte swizzle) into a ring of 4 slots.  Chunk n of a
// CTA's stream goes to slot n % 4.  The warp that finishes a chunk last (an arrival
// count per slot) issues the chunk four places later into the freed slot, so copies
// run three chunks ahead of the warps and no warp ever blocks to issue one.  Q lands
// first in two ring slots and is transposed into Q^T before the K stream starts.
// Block skipping: the key-tile range per query tile comes from the plan; SKIP
// tiles are neither loaded nor computed, FULL tiles skip the per-element mask.
#include "internal.h"

namespace gqa {
namespace {

constexpr int kRows = kF32Rows;  // 64 query rows per CTA
constexpr int kBc = kF32Bc;      // 256 keys per tile
constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kBoxCols = 32;                  // fp32 per 128-byte swizzle row
constexpr int kQBox = kRows * 128;            // Q as loaded: 64 rows x 32 fp32 per 32-column block (8 KiB)
constexpr int kQBytes = 8 * kQBox;            // 64 rows x 256 fp32
constexpr int kSlots = 4;
constexpr int kSlotBytes = 32768;
constexpr int kChunks = 16;                   // per key tile: 8 K blocks of d, then 8 V groups of keys
constexpr int kVKeys = 32;                    // keys per V chunk
constexpr int kVBlock = kVKeys * 128;         // V chunk: 32 keys x 32 fp32 (4 KiB), eight per slot
constexpr int kPKeys = kBc / 2;               // keys of P held in shared memory at a time
constexpr int kPWarpBytes = kPKeys * 8 * 4;   // P^T slice: [128 keys][8 rows] fp32, swizzled
constexpr int kOffQT = 0;                     // Q^T: [256 d][64 rows] fp32
constexpr int kOffRing = kQBytes;
constexpr int kOffP = kOffRing + kSlots * kSlotBytes;
constexpr int kOffBar = kOffP + kWarps * kPWarpBytes;
// barriers: Q, then one per slot (8 bytes each); then per slot an arrival counter
// and the number of copies issued into it (read back at exit to drain copies)
enum { kBarQ = 0, kBarSlot = 1 };
constexpr int kOffCnt = kOffBar + 8 * (1 + kSlots);
constexpr int kOffIss = kOffCnt + 4 * kSlots;
constexpr int kSmemBytes = kOffIss + 4 * kSlots + 1024;  // + slack to align to the 1024-byte swizzle atom

static_assert(kRows == 8 * kWarps, "one warp per 8 query rows");
static_assert(kBc == 256 && kBc * 128 == kSlotBytes && 8 * kVBlock == kSlotBytes, "chunk geometry");
static_assert(kQBytes == 2 * kSlotBytes, "Q is staged in two ring slots");
static_assert(kSmemBytes <= 232448, "shared memory per block");

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

// c0, c1 += a0 * b0, a1 * b1 in one instruction (sm_100 packed fp32 FMA, round to
// nearest): half the issue slots of two FFMAs.
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

__device__ __forceinline__ void sts128(uint32_t addr, uint32_t lo, uint32_t n, float a, float b, float c,
                                       float d) {
  if (!debug_region_ok(addr, 16, lo, n)) return;
  asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}

// 4-D tiled TMA load into this CTA's shared memory (no multicast).
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int c0, int c1,
                                            int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}

struct TileCtx {
  int64_t i0, i1;  // query rows of the tile (clamped to Lq - 1)
  SegBounds qb;
};

__device__ __forceinline__ int classify(const FwdParams& p, const TileCtx& c, int kt) {
  const int64_t j0 = int64_t(kt) * kBc;
  const int64_t j1 = min(p.Lk, j0 + kBc) - 1;
  SegBounds kb{0, 0};
  if (p.has_seg) kb = SegBounds{p.kv_bounds[2 * kt], p.kv_bounds[2 * kt + 1]};
  return tile_class(c.i0, c.i1, j0, j1, p.off, p.P0, p.has_seg != 0, c.qb, kb);
}

__global__ void __launch_bounds__(kThreads, 1)
fwd_f32_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const __grid_constant__ FwdParams p) {
  extern __shared__ char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  const uint32_t sQT = sbase + kOffQT, sRing = sbase + kOffRing, sP = sbase + kOffP;
  const uint32_t bar = sbase + kOffBar;
  auto slot_bar = [&](int s) { return bar + 8u * uint32_t(kBarSlot + s); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // Unit: (query tile, kv head, batch[, key split]), ordered kv head by kv head and,
  // within one, query tiles in descending order so the longest causal rows start
  // first.  The CTAs resident together then belong to one kv head and sweep its key
  // tiles from 0 a few tiles apart, so a key/value tile one CTA fetched is still in
  // L2 when the next one reaches it (one kv head's K/V is 125 MB in fp32 at L =
  // 60,926; all four would be four times the L2).
  const int splits = p.splits > 1 ? p.splits : 1;
  const int split = int(blockIdx.x % unsigned(splits));
  const unsigned unit = blockIdx.x / unsigned(splits);
  const int qt = p.nq - 1 - int(unit % unsigned(p.nq));
  const int hb = int(unit / unsigned(p.nq));  // b * Hkv + g
  const int g = hb % p.Hkv;
  const int b = hb / p.Hkv;
  const int br = p.br;
  const int64_t q0 = int64_t(qt) * br;

  TileCtx ctx;
  ctx.i0 = q0;
  ctx.i1 = min(p.Lq, q0 + br) - 1;
  ctx.qb = SegBounds{0, 0};
  int kbeg, kend;
  if (p.has_seg) {
    ctx.qb = SegBounds{p.q_bounds[2 * qt], p.q_bounds[2 * qt + 1]};
    kbeg = p.q_ranges[2 * qt];
    kend = p.q_ranges[2 * qt + 1];
  } else {
    kv_range_no_seg(ctx.i1, p.off, kBc, p.nk, &kbeg, &kend);
  }
  split_range(split, splits, &kbeg, &kend);

  // generic views of the counters
  uint32_t* cnt = reinterpret_cast<uint32_t*>(smem_raw + (sbase + kOffCnt - raw));
  uint32_t* iss = reinterpret_cast<uint32_t*>(smem_raw + (sbase + kOffIss - raw));
  if (threadIdx.x == 0) {
    debug_flag_reset();
    mbar_init(bar + 8 * kBarQ, 1);
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(slot_bar(s), 1);
      cnt[s] = 0;
      iss[s] = 0;
    }
    fence_barrier_init();
  }
  __syncthreads();

  const int qhead = b * p.Hq + g * p.G;
  const int kvhead = b * p.Hkv + g;
  auto next_tile = [&](int kt) {
    while (kt < kend && classify(p, ctx, kt) == GQA_TILE_SKIP) ++kt;
    return kt;
  };
  // Chunk c of key tile kt goes to slot c % 4 (a tile's 16 chunks are 4 uses of each
  // slot): c < 8 is K's 32-column block c of d, [256 keys][32 d]; c >= 8 is V's keys
  // 32 (c - 8) .. +31, [32 keys][256 d].
  auto load_chunk = [&](int kt, int c) {
    const int s = c & 3;
    // the u-th fill of slot s is chunk 4u + s of this CTA's stream
    const uint32_t u = atomicAdd(&iss[s], 1u);
    if (int64_t(4) * u + s == p.test_skip_fill) return;  // test hook: never arrives
    mbar_arrive_expect_tx(slot_bar(s), kSlotBytes);
    const uint32_t dst = sRing + s * kSlotBytes;
    if (c < 8)
      tma_load_4d(dst, &tmK, slot_bar(s), 0, kt * kBc, c, kvhead);
    else
      tma_load_4d(dst, &tmV, slot_bar(s), 0, kt * kBc + kVKeys * (c - 8), 0, kvhead);
  };
  // The last warp done with chunk c of tile kt (the `use`-th use of its slot) issues
  // the chunk four places later.
  auto release = [&](int kt, int c, uint32_t use) {
    __syncwarp();
    if (lane == 0) {
      __threadfence_block();
      const int s = c & 3;
      if (atomicAdd(&cnt[s], 1u) == uint32_t(kWarps) * (use + 1) - 1) {
        if (c + 4 < kChunks) {
          load_chunk(kt, c + 4);
        } else {
          const int kn = next_tile(kt + 1);
          if (kn < kend) load_chunk(kn, c + 4 - kChunks);
        }
      }
    }
  };
  // Q lands in slots 0-1 and is transposed to Q^T [d][row] (the S loop below takes row
  // pairs at one depth as packed-FMA operands); the K stream starts after that.
  if (threadIdx.x == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    mbar_arrive_expect_tx(bar + 8 * kBarQ, kQBytes);
    for (int c = 0; c < 8; ++c)
      tma_load_3d(sRing + c * kQBox, &tmQ, bar + 8 * kBarQ, c * kBoxCols, int(q0), qhead);
  }
  bool ok = mbar_wait_bounded(bar + 8 * kBarQ, 0, p.wait_budget_ns, p.status);
  if (ok) {
    const int r = threadIdx.x & 63;
    float* qt_gen = reinterpret_cast<float*>(smem_raw + (sQT - raw));
#pragma unroll 4
    for (int cx = threadIdx.x >> 6; cx < 64; cx += kThreads / 64) {  // (block c, chunk x) of d
      const int c = cx >> 3, x = cx & 7;
      const float4 v = lds128(sRing + c * kQBox + r * 128 + (uint32_t(x ^ (r & 7)) << 4), sRing, kQBytes);
      const int d = 32 * c + 4 * x;
      if (!debug_index_ok((d + 3) * kRows + r, kQBytes / 4)) continue;
      qt_gen[(d + 0) * kRows + r] = v.x;
      qt_gen[(d + 1) * kRows + r] = v.y;
      qt_gen[(d + 2) * kRows + r] = v.z;
      qt_gen[(d + 3) * kRows + r] = v.w;
    }
  }
  ok = __syncthreads_and(ok);
  if (threadIdx.x == 0) {
    fence_proxy_async_smem();  // the staging reads above come before the copies below
    const int k0 = ok ? next_tile(kbeg) : kend;
    if (k0 < kend)
      for (int c = 0; c < 4; ++c) load_chunk(k0, c);
  }

  // ------------------------------------------------------------------ consumers
  const uint32_t sPw = sP + warp * kPWarpBytes;

  float o[8][8];
#pragma unroll
  for (int r = 0; r < 8; ++r)
#pragma unroll
    for (int c = 0; c < 8; ++c) o[r][c] = 0.f;
  // m: running max of each row (the same in every lane); l: this lane's share of the
  // row sum (its keys only), reduced over the warp in the epilogue.
  float m[8], l[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    m[i] = -INFINITY;
    l[i] = 0.f;
  }

  // Shared-memory addresses.  A 128-byte row r of a block lives at r*128, its 16-byte
  // chunk x at physical chunk x ^ (r & 7) (TMA 128-byte swizzle).
  //   Q^T depth d, rows 8w .. 8w+7: qtw + d*256 (+16 for rows 4-7), the same address in
  //     every lane;
  //   K chunk (one 32-column block of d): key l + 32 m (r & 7 = l & 7), chunk x at
  //     (kl ^ (x << 4)) + m*4K from the slot;
  //   V chunk: key kk, columns 4l.. in block l / 8 (chunk l & 7) and 128 + 4l.. in
  //     block 4 + l / 8: voff[kk & 7] + (kk & ~7)*128 from the slot (+ 4 blocks).
  const uint32_t qtw = sQT + (8 * warp) * 4;
  const uint32_t kl = lane * 128 + ((lane & 7) << 4);
  uint32_t voff[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) voff[c] = (lane >> 3) * kVBlock + c * 128 + (uint32_t(c ^ (lane & 7)) << 4);

  uint32_t t = 0;  // tiles computed so far: slot uses 4t .. 4t+3
  for (int kt = kbeg; kt < kend && ok; ++kt) {
    const int cls = classify(p, ctx, kt);
    if (cls == GQA_TILE_SKIP) continue;
    const int64_t j0 = int64_t(kt) * kBc;

    // ---- S = Q K^T: 8 rows x 8 keys (l + 32 m) per lane, depth 256 in eight chunks.
    // Rows are paired at one depth: (S[r][j], S[r+1][j]) += (q[r], q[r+1]) (k[j], k[j]),
    // one packed FMA, the key value duplicated into a register pair.
    float s[8][8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int m8 = 0; m8 < 8; ++m8) s[i][m8] = 0.f;
    // Q^T fragments of the four depths of a step rotate: depth e of the next step is
    // loaded once depth e of this one is consumed.  K fragments rotate the same way.
    float4 fq[4][2];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      fq[e][0] = lds128(qtw + e * 256, sQT, kQBytes);
      fq[e][1] = lds128(qtw + e * 256 + 16, sQT, kQBytes);
    }
#pragma unroll 1
    for (int c = 0; c < 8; ++c) {
      ok = __all_sync(0xffffffffu, mbar_wait_bounded(slot_bar(c & 3), uint32_t(c >> 2) & 1u, p.wait_budget_ns,
                                                      p.status));
      if (!ok) break;
      const uint32_t kslot = sRing + (c & 3) * kSlotBytes + kl;
      float4 fk[8];
#pragma unroll
      for (int m8 = 0; m8 < 8; ++m8) fk[m8] = lds128(kslot + m8 * 4096, kslot - kl, kSlotBytes);
#pragma unroll
      for (int x = 0; x < 8; ++x) {  // depth step: d = 32 c + 4 x + e
        // the next step's depths (the last step of the tile re-reads depth 0)
        const int nd = (32 * c + 4 * (x + 1)) & (kHeadDim - 1);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          // Order of the packed FMAs: runs of eight that share one (q_r, q_r+1) register
          // pair keep the FP32 pipe fuller than runs that share the duplicated key value
          // (a register-only loop reaches ~99 % of the nominal rate against ~85 %).  The
          // last depth of a step keeps the key-major order so that each key's fragment
          // for the next step is reloaded right after its last use.
          if (e < 3) {
#pragma unroll
            for (int rp = 0; rp < 4; ++rp) {
              const float qa = rp == 0 ? fq[e][0].x : rp == 1 ? fq[e][0].z : rp == 2 ? fq[e][1].x : fq[e][1].z;
              const float qb = rp == 0 ? fq[e][0].y : rp == 1 ? fq[e][0].w : rp == 2 ? fq[e][1].y : fq[e][1].w;
#pragma unroll
              for (int m8 = 0; m8 < 8; ++m8) {
                const float kv = e == 0 ? fk[m8].x : e == 1 ? fk[m8].y : fk[m8].z;
                ffma2(s[2 * rp][m8], s[2 * rp + 1][m8], qa, qb, kv, kv);
              }
            }
          } else {
#pragma unroll
            for (int m8 = 0; m8 < 8; ++m8) {
              const float kv = fk[m8].w;
              ffma2(s[0][m8], s[1][m8], fq[e][0].x, fq[e][0].y, kv, kv);
              ffma2(s[2][m8], s[3][m8], fq[e][0].z, fq[e][0].w, kv, kv);
              ffma2(s[4][m8], s[5][m8], fq[e][1].x, fq[e][1].y, kv, kv);
              ffma2(s[6][m8], s[7][m8], fq[e][1].z, fq[e][1].w, kv, kv);
              if (x < 7) fk[m8] = lds128((kslot ^ (uint32_t(x + 1) << 4)) + m8 * 4096, kslot - kl, kSlotBytes);
            }
          }
          fq[e][0] = lds128(qtw + (nd + e) * 256, sQT, kQBytes);
          fq[e][1] = lds128(qtw + (nd + e) * 256 + 16, sQT, kQBytes);
        }
      }
      // The last warp done with K block c issues chunk c + 4.
      release(kt, c, 4 * t + (c >> 2));
    }
    if (!ok) break;

    // ---- mask + online softmax (base 2)
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int m8 = 0; m8 < 8; ++m8) s[i][m8] *= p.scale_log2;
    if ((cls == GQA_TILE_PARTIAL) || (j0 + kBc > p.Lk)) {
#pragma unroll
      for (int m8 = 0; m8 < 8; ++m8) {
        const int64_t j = j0 + lane + 32 * m8;
        const int sk = p.has_seg ? p.seg_kv[min(j, p.Lk - 1)] : 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int r = 8 * warp + i;
          // the last key this row sees: its position, or the block's last key when the
          // key block ends before it (a block of a sharded sequence)
          const int64_t pos = min(q0 + (r % br) + p.off, p.Lk - 1);
          bool vis = j <= pos;
          if (p.has_seg) vis = vis && (p.seg_q[min(q0 + (r % br), p.Lq - 1)] == sk || j < p.P0);
          if (!vis) s[i][m8] = -INFINITY;
        }
      }
    }
    float mx[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      mx[i] = s[i][0];
#pragma unroll
      for (int m8 = 1; m8 < 8; ++m8) mx[i] = fmaxf(mx[i], s[i][m8]);
    }
    // The eight rows' reductions interleaved: five dependent shuffle steps, not forty.
#pragma unroll
    for (int sh = 16; sh >= 1; sh >>= 1)
#pragma unroll
      for (int i = 0; i < 8; ++i) mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], sh));
    float alpha[8];
    bool raised = false;  // the same in every lane: m and mx are
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float m_new = fmaxf(m[i], mx[i]);
      const float m_ref = (m_new == -INFINITY) ? 0.f : m_new;  // no visible key yet
      raised |= m_new != m[i];
      alpha[i] = exp2f(m[i] - m_ref);
      m[i] = m_new;
      float rs = 0.f;
#pragma unroll
      for (int m8 = 0; m8 < 8; ++m8) {
        s[i][m8] = exp2f(s[i][m8] - m_ref);
        rs += s[i][m8];
      }
      l[i] = l[i] * alpha[i] + rs;
    }
    // P^T slice, half a tile (128 keys) at a time: [key][8 rows]; key k's 16-byte chunk
    // h (rows 4h .. 4h+3) sits at chunk h ^ ((k >> 2) & 1), so a quarter warp's eight
    // stores hit distinct banks.  Half 1 (keys 128-255) is written after PV has read
    // half 0.
    auto store_p_half = [&](int hh) {
#pragma unroll
      for (int m4 = 0; m4 < 4; ++m4) {
        const int m8 = 4 * hh + m4;
        const int k = lane + 32 * m4;  // key within the half
        const uint32_t a = sPw + k * 32;
        const int sw = (k >> 2) & 1;
        sts128(a + ((0 ^ sw) << 4), sPw, kPWarpBytes, s[0][m8], s[1][m8], s[2][m8], s[3][m8]);
        sts128(a + ((1 ^ sw) << 4), sPw, kPWarpBytes, s[4][m8], s[5][m8], s[6][m8], s[7][m8]);
      }
      __syncwarp();
    };
    store_p_half(0);

    // ---- O = alpha * O + P V  (8 rows x 8 cols per lane); alpha is 1 in every row
    // unless a row's maximum rose, which the lanes see alike
    if (raised) {
#pragma unroll
      for (int r = 0; r < 8; ++r)
#pragma unroll
        for (int c = 0; c < 8; ++c) o[r][c] *= alpha[r];
    }
#pragma unroll 1
    for (int vc = 0; vc < 8; ++vc) {
      if (vc == 4) {
        __syncwarp();  // this warp's reads of half 0 are done
        store_p_half(1);
      }
      const int cn = 8 + vc;
      ok = __all_sync(0xffffffffu, mbar_wait_bounded(slot_bar(cn & 3), uint32_t(cn >> 2) & 1u, p.wait_budget_ns,
                                                      p.status));
      if (!ok) break;
      const uint32_t vslot = sRing + (cn & 3) * kSlotBytes;
      const uint32_t pkey = sPw + (vc & 3) * kVKeys * 32;
      // P and V fragments double-buffered over the chunk's 32 keys (the last prefetch
      // re-reads key 31 of the chunk).
      float4 fp[2][2], fv[2][2];
      fp[0][0] = lds128(pkey, sPw, kPWarpBytes);
      fp[0][1] = lds128(pkey + 16, sPw, kPWarpBytes);
      fv[0][0] = lds128(vslot + voff[0], vslot, kSlotBytes);
      fv[0][1] = lds128(vslot + voff[0] + 4 * kVBlock, vslot, kSlotBytes);
#pragma unroll 1
      for (int k8 = 0; k8 < kVKeys; k8 += 8) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const int cur = kk & 1, nxt = cur ^ 1;
          const int nk = min(k8 + kk + 1, kVKeys - 1);
          const int nkk = (kk + 1) & 7;                  // nk & 7 unless clamped
          const int nsw = (((kk + 1) & 7) >> 2) & 1;     // (nk >> 2) & 1 (k8 is a multiple of 8)
          fp[nxt][0] = lds128(pkey + nk * 32 + ((0 ^ nsw) << 4), sPw, kPWarpBytes);
          fp[nxt][1] = lds128(pkey + nk * 32 + ((1 ^ nsw) << 4), sPw, kPWarpBytes);
          const uint32_t vrow = vslot + voff[nkk] + (nk - nkk) * 128;
          fv[nxt][0] = lds128(vrow, vslot, kSlotBytes);
          fv[nxt][1] = lds128(vrow + 4 * kVBlock, vslot, kSlotBytes);
          const float pr[8] = {fp[cur][0].x, fp[cur][0].y, fp[cur][0].z, fp[cur][0].w,
                               fp[cur][1].x, fp[cur][1].y, fp[cur][1].z, fp[cur][1].w};
          const float vc8[8] = {fv[cur][0].x, fv[cur][0].y, fv[cur][0].z, fv[cur][0].w,
                                fv[cur][1].x, fv[cur][1].y, fv[cur][1].z, fv[cur][1].w};
          // column pair outermost: runs of eight packed FMAs share one (v_c, v_c+1) pair
#pragma unroll
          for (int c = 0; c < 8; c += 2)
#pragma unroll
            for (int r = 0; r < 8; ++r) ffma2(o[r][c], o[r][c + 1], pr[r], pr[r], vc8[c], vc8[c + 1]);
        }
      }
      // The last warp done with V group vc issues chunk 12 + vc (of the next tile past 3).
      release(kt, cn, 4 * t + (cn >> 2));
    }
    if (!ok) break;
    ++t;
  }
  // A wait that ran out leaves ok == false: the status word says so and this warp's
  // outputs are not written.  Every thread still meets the barrier at the end.
  if (ok) {
    // ---- epilogue: out = O / l, lse = (m + log2 l) ln 2, l summed over the lanes
#pragma unroll
    for (int sh = 16; sh >= 1; sh >>= 1)
#pragma unroll
      for (int i = 0; i < 8; ++i) l[i] += __shfl_xor_sync(0xffffffffu, l[i], sh);
    // One key split writes its normalised partial output and log-sum-exp.
    const int64_t plane = int64_t(p.B) * p.Hq * p.Lq;
    float* out = splits > 1 ? p.o_part + split * plane * kHeadDim : static_cast<float*>(p.out);
    float* lse_out = splits > 1 ? p.lse_part + split * plane : p.lse;
#pragma unroll
    for (int rr = 0; rr < 8; ++rr) {
      const int r = 8 * warp + rr;
      const int64_t qi = q0 + (r % br);
      if (qi >= p.Lq) continue;
      const int head = b * p.Hq + g * p.G + r / br;
      const float inv = l[rr] > 0.f ? 1.f / l[rr] : 0.f;
      if (!debug_index_ok(int64_t(head) * p.Lq + qi, plane)) continue;
      float* row = out + (int64_t(head) * p.Lq + qi) * kHeadDim;
      float4 w0 = make_float4(o[rr][0] * inv, o[rr][1] * inv, o[rr][2] * inv, o[rr][3] * inv);
      float4 w1 = make_float4(o[rr][4] * inv, o[rr][5] * inv, o[rr][6] * inv, o[rr][7] * inv);
      *reinterpret_cast<float4*>(row + 4 * lane) = w0;
      *reinterpret_cast<float4*>(row + 128 + 4 * lane) = w1;
      if (lane == rr) lse_out[int64_t(head) * p.Lq + qi] = l[rr] > 0.f ? (m[rr] + log2f(l[rr])) * kLn2 : -INFINITY;
    }
  }  // if (ok)
  __syncthreads();
  if (threadIdx.x == 0) {  // no copy may be in flight when the CTA ends (returns at once normally)
    mbar_wait_bounded(bar + 8 * kBarQ, 0, p.wait_budget_ns, p.status);
    for (int s = 0; s < kSlots; ++s) {
      const uint32_t n = iss[s];
      if (n) mbar_wait_bounded(slot_bar(s), (n - 1) & 1u, p.wait_budget_ns, p.status);
    }
    debug_flag_report(p.status);
  }
}

}  // namespace

int launch_fwd_f32(const FwdTensors& t, const FwdParams& p, cudaStream_t stream) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return GQA_ERR_LAUNCH;
  CUtensorMap mq, mk, mv;
  {
    const cuuint32_t estr[3] = {1, 1, 1};
    const cuuint64_t dims[3] = {cuuint64_t(kHeadDim), cuuint64_t(p.Lq), cuuint64_t(p.B) * p.Hq};
    const cuuint64_t strides[2] = {cuuint64_t(kHeadDim) * 4, cuuint64_t(p.Lq) * kHeadDim * 4};
    const cuuint32_t box[3] = {cuuint32_t(kBoxCols), cuuint32_t(p.br), cuuint32_t(p.G)};
    if (enc(&mq, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(t.q), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return GQA_ERR_LAUNCH;
  }
  {
    // K and V as 4-D views (d within a 32-column block, key, block, head): one copy
    // brings [keys][blocks] of one head, block by block, 128-byte swizzled.
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    const cuuint64_t dims[4] = {cuuint64_t(kBoxCols), cuuint64_t(p.Lk), cuuint64_t(kHeadDim / kBoxCols),
                                cuuint64_t(p.B) * p.Hkv};
    const cuuint64_t strides[3] = {cuuint64_t(kHeadDim) * 4, cuuint64_t(kBoxCols) * 4,
                                   cuuint64_t(p.Lk) * kHeadDim * 4};
    const cuuint32_t kbox[4] = {cuuint32_t(kBoxCols), cuuint32_t(kBc), 1, 1};       // K: 256 keys x 32 d
    const cuuint32_t vbox[4] = {cuuint32_t(kBoxCols), cuuint32_t(kVKeys), 8, 1};    // V: 32 keys x 256 d
    if (enc(&mk, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, const_cast<void*>(t.k), dims, strides, kbox, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return GQA_ERR_LAUNCH;
    if (enc(&mv, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, const_cast<void*>(t.v), dims, strides, vbox, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return GQA_ERR_LAUNCH;
  }
  if (cudaFuncSetAttribute(fwd_f32_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) !=
      cudaSuccess)
    return GQA_ERR_LAUNCH;
  const int64_t units = int64_t(p.nq) * p.Hkv * p.B * (p.splits > 1 ? p.splits : 1);
  if (units <= 0) return GQA_OK;
  if (units > 0x7fffffff) return GQA_ERR_UNSUPPORTED;
  fwd_f32_kernel<<<unsigned(units), kThreads, kSmemBytes, stream>>>(mq, mk, mv, p);
  return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_LAUNCH;
}

}  // namespace gqa
