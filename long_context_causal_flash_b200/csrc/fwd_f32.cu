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
// 1 CTA per SM).  Key tiles hold 128 keys.  Warp w owns query rows 8w .. 8w+7 for
// the whole key loop, every lane all 8 of them:
//   S = Q K^T   lane l: 8 rows x keys l, l+32, l+64, l+96 (Q fragments warp-uniform)
//   softmax     online, base 2, row max by warp shuffles over 32 lanes; each lane
//               keeps its own partial row sums (reduced once, at the end)
//   O += P V    lane l: 8 rows x cols 4l.., 128+4l.. (P fragments warp-uniform)
// P goes through a warp-private 4 KiB slice of shared memory, so warps never wait
// for one another inside the key loop.
//
// Why these register tiles.  Shared-memory bandwidth, not the FP32 pipe, bounded the
// earlier 64-key form: a warp's 128-bit load costs four data wavefronts (two when
// every lane reads one address), and the SM moves one wavefront per cycle while
// its four sub-partitions retire two packed FMAs (fma.rn.f32x2) per cycle.  Per
// depth step of 4, S here loads 8 broadcast Q fragments (16 wavefronts) and 4 K
// fragments (16) for 64 packed FMAs; PV loads, per key, 2 broadcast P fragments
// (4) and 2 V fragments (8) for 32: 2.3 packed FMAs per wavefront over a tile, where
// the FP32 pipe needs 2.  (P is stored once per value; the (p, p) operand pairs of
// the packed FMAs are formed in registers.)
//
// Key/value streaming.  A 128-key tile is 8 chunks of 32 KiB: K in four quarters
// of d ([128 keys][64 d], two 64-column blocks), V in four quarters of the keys
// ([32 keys][256 d], eight blocks), each ONE 4-D TMA copy (128-byte swizzle) into a
// ring of 4 slots.  Chunk n of a CTA's stream goes to slot n % 4: the K quarters of
// a tile fill slots 0-3 and its V quarters follow them in the same slots.  The warp
// that finishes a chunk last (an arrival count per slot) issues the chunk four
// places later into the freed slot, so the copy of V quarter q overlaps the rest of
// S, and K of the next tile overlaps PV.  No warp ever blocks to issue a copy.
// Block skipping: the key-tile range per query tile comes from the plan; SKIP
// tiles are neither loaded nor computed, FULL tiles skip the per-element mask.
#include "internal.h"

namespace gqa {
namespace {

constexpr int kRows = kF32Rows;  // 64 query rows per CTA
constexpr int kBc = kF32Bc;      // 128 keys per tile
constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kBoxCols = 32;                  // fp32 per 128-byte swizzle row
constexpr int kQBox = kRows * 128;            // Q: 64 rows x 32 fp32 per 64-column block... (8 KiB)
constexpr int kQBytes = 8 * kQBox;            // 64 rows x 256 fp32
constexpr int kSlots = 4;
constexpr int kSlotBytes = 32768;
constexpr int kKBlock = kBc * 128;            // K chunk: 128 keys x 32 fp32 (16 KiB), two per slot
constexpr int kVKeys = kBc / 4;               // keys per V chunk
constexpr int kVBlock = kVKeys * 128;         // V chunk: 32 keys x 32 fp32 (4 KiB), eight per slot
constexpr int kPWarpBytes = kBc * 8 * 4;      // P^T slice: [128 keys][8 rows] fp32, swizzled
constexpr int kOffQ = 0;
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
static_assert(kBc == 128 && 2 * kKBlock == kSlotBytes && 8 * kVBlock == kSlotBytes, "chunk geometry");
static_assert(kSmemBytes <= 232448, "shared memory per block");

__device__ __forceinline__ float4 lds128(uint32_t addr) {
  float4 v;
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

__device__ __forceinline__ void sts128(uint32_t addr, float a, float b, float c, float d) {
  asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(a), "f"(b), "f"(c),
               "f"(d)
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
  const uint32_t sQ = sbase + kOffQ, sRing = sbase + kOffRing, sP = sbase + kOffP;
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
  // Chunk `part` of key tile kt into slot part % 4: parts 0-3 are K's quarters of d,
  // parts 4-7 V's quarters of the keys.
  auto load_chunk = [&](int kt, int part) {
    const int s = part & 3;
    // the u-th fill of slot s is chunk 4u + s of this CTA's stream
    const uint32_t u = atomicAdd(&iss[s], 1u);
    if (int64_t(4) * u + s == p.test_skip_fill) return;  // test hook: never arrives
    mbar_arrive_expect_tx(slot_bar(s), kSlotBytes);
    const uint32_t dst = sRing + s * kSlotBytes;
    if (part < 4)
      tma_load_4d(dst, &tmK, slot_bar(s), 0, kt * kBc, 2 * part, kvhead);
    else
      tma_load_4d(dst, &tmV, slot_bar(s), 0, kt * kBc + kVKeys * (part - 4), 0, kvhead);
  };
  // The last warp done with chunk `part` of tile kt (the `use`-th use of its slot)
  // issues the chunk four places later.
  auto release = [&](int kt, int part, uint32_t use) {
    __syncwarp();
    if (lane == 0) {
      __threadfence_block();
      const int s = part & 3;
      if (atomicAdd(&cnt[s], 1u) == uint32_t(kWarps) * (use + 1) - 1) {
        if (part < 4) {
          load_chunk(kt, part + 4);
        } else {
          const int kn = next_tile(kt + 1);
          if (kn < kend) load_chunk(kn, part - 4);
        }
      }
    }
  };
  if (threadIdx.x == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    mbar_arrive_expect_tx(bar + 8 * kBarQ, kQBytes);
    for (int c = 0; c < 8; ++c)
      tma_load_3d(sQ + c * kQBox, &tmQ, bar + 8 * kBarQ, c * kBoxCols, int(q0), qhead);
    const int k0 = next_tile(kbeg);
    if (k0 < kend)
      for (int part = 0; part < 4; ++part) load_chunk(k0, part);
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

  bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(bar + 8 * kBarQ, 0, p.wait_budget_ns, p.status));

  // Shared-memory addresses.  A 128-byte row r of a block lives at r*128, its 16-byte
  // chunk x at physical chunk x ^ (r & 7) (TMA 128-byte swizzle).
  //   Q block c, row 8w + i (r & 7 = i): qrow + c*8K + i*128 + ((x ^ i) << 4), the
  //     same address in every lane;
  //   K chunk: block bb (d 64 part + 32 bb ..), key l + 32 jj (r & 7 = l & 7):
  //     (kl ^ (x << 4)) + bb*16K + jj*4K from the slot;
  //   V chunk: key kk, columns 4l.. in block l / 8 (chunk l & 7) and 128 + 4l.. in
  //     block 4 + l / 8: voff[kk & 7] + (kk & ~7)*128 from the slot (+ 4 blocks).
  const uint32_t qrow = sQ + (8 * warp) * 128;
  const uint32_t kl = lane * 128 + ((lane & 7) << 4);
  uint32_t voff[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) voff[c] = (lane >> 3) * kVBlock + c * 128 + (uint32_t(c ^ (lane & 7)) << 4);

  uint32_t t = 0;  // tiles computed so far: slot uses 2t (K) and 2t + 1 (V)
  for (int kt = kbeg; kt < kend && ok; ++kt) {
    const int cls = classify(p, ctx, kt);
    if (cls == GQA_TILE_SKIP) continue;
    const int64_t j0 = int64_t(kt) * kBc;

    // ---- S = Q K^T (8 rows x 4 keys per lane, depth 256 in four chunks of 64)
    // Each score is accumulated as two partial sums (even / odd elements of d) in a
    // register pair, so every pair of products is one packed FMA.
    float2 s2[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) s2[i][jj] = make_float2(0.f, 0.f);
    // Q fragments rotate: row i of the next depth step is loaded as soon as row i of
    // this one is consumed; K fragments are double-buffered within a chunk.
    float4 fq[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) fq[i] = lds128(qrow + i * 128 + (i << 4));
#pragma unroll 1
    for (int part = 0; part < 4; ++part) {
      ok = __all_sync(0xffffffffu, mbar_wait_bounded(slot_bar(part), 0u, p.wait_budget_ns, p.status));
      if (!ok) break;
      const uint32_t kslot = sRing + part * kSlotBytes + kl;
      float4 fk[2][4];
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) fk[0][jj] = lds128(kslot + jj * 4096);
#pragma unroll
      for (int st = 0; st < 16; ++st) {  // depth step: block bb = st / 8, chunk x = st % 8
        const int cur = st & 1, nxt = cur ^ 1;
        const int x = st & 7, bb = st >> 3;
        if (st < 15) {
          const int nx = (st + 1) & 7, nbb = (st + 1) >> 3;
#pragma unroll
          for (int jj = 0; jj < 4; ++jj)
            fk[nxt][jj] = lds128(((kslot + nbb * kKBlock) ^ (uint32_t(nx) << 4)) + jj * 4096);
        }
        // the next depth step's Q block (the last step of the tile re-reads block 7)
        const int nst = st + 1;
        const int nc = min(2 * part + (nst >> 3), 7);
        const int nqx = nst & 7;
        (void)x;
        (void)bb;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
#pragma unroll
          for (int jj = 0; jj < 4; ++jj)
            ffma2(s2[i][jj].x, s2[i][jj].y, fq[i].x, fq[i].y, fk[cur][jj].x, fk[cur][jj].y);
#pragma unroll
          for (int jj = 0; jj < 4; ++jj)
            ffma2(s2[i][jj].x, s2[i][jj].y, fq[i].z, fq[i].w, fk[cur][jj].z, fk[cur][jj].w);
          fq[i] = lds128(qrow + nc * kQBox + i * 128 + ((nqx ^ i) << 4));
        }
      }
      // The last warp done with K quarter `part` issues V quarter `part` of this tile.
      release(kt, part, 2 * t);
    }
    if (!ok) break;

    // ---- mask + online softmax (base 2)
    float s[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) s[i][jj] = (s2[i][jj].x + s2[i][jj].y) * p.scale_log2;
    if ((cls == GQA_TILE_PARTIAL) || (j0 + kBc > p.Lk)) {
      int sk[4];
      int64_t j[4];
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        j[jj] = j0 + lane + 32 * jj;
        sk[jj] = p.has_seg ? p.seg_kv[min(j[jj], p.Lk - 1)] : 0;
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int r = 8 * warp + i;
        // the last key this row sees: its position, or the block's last key when the
        // key block ends before it (a block of a sharded sequence)
        const int64_t pos = min(q0 + (r % br) + p.off, p.Lk - 1);
        const int sqi = p.has_seg ? p.seg_q[min(q0 + (r % br), p.Lq - 1)] : 0;
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          bool vis = j[jj] <= pos;
          if (p.has_seg) vis = vis && (sqi == sk[jj] || j[jj] < p.P0);
          if (!vis) s[i][jj] = -INFINITY;
        }
      }
    }
    float mx[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) mx[i] = fmaxf(fmaxf(s[i][0], s[i][1]), fmaxf(s[i][2], s[i][3]));
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
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) s[i][jj] = exp2f(s[i][jj] - m_ref);
      l[i] = l[i] * alpha[i] + ((s[i][0] + s[i][1]) + (s[i][2] + s[i][3]));
    }
    // P^T slice: [key][8 rows]; key k's 16-byte chunk h (rows 4h .. 4h+3) sits at
    // chunk h ^ ((k >> 2) & 1), so a quarter warp's eight stores hit distinct banks.
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      const int k = lane + 32 * jj;
      const uint32_t a = sPw + k * 32;
      const int sw = (k >> 2) & 1;
      sts128(a + ((0 ^ sw) << 4), s[0][jj], s[1][jj], s[2][jj], s[3][jj]);
      sts128(a + ((1 ^ sw) << 4), s[4][jj], s[5][jj], s[6][jj], s[7][jj]);
    }
    __syncwarp();

    // ---- O = alpha * O + P V  (8 rows x 8 cols per lane); alpha is 1 in every row
    // unless a row's maximum rose, which the lanes see alike
    if (raised) {
#pragma unroll
      for (int r = 0; r < 8; ++r)
#pragma unroll
        for (int c = 0; c < 8; ++c) o[r][c] *= alpha[r];
    }
#pragma unroll 1
    for (int vp = 0; vp < 4; ++vp) {
      ok = __all_sync(0xffffffffu, mbar_wait_bounded(slot_bar(vp), 1u, p.wait_budget_ns, p.status));
      if (!ok) break;
      const uint32_t vslot = sRing + vp * kSlotBytes;
      const uint32_t pkey = sPw + vp * kVKeys * 32;
      // P and V fragments double-buffered over the chunk's 32 keys (the last prefetch
      // re-reads key 31 of the chunk).
      float4 fp[2][2], fv[2][2];
      fp[0][0] = lds128(pkey);
      fp[0][1] = lds128(pkey + 16);
      fv[0][0] = lds128(vslot + voff[0]);
      fv[0][1] = lds128(vslot + voff[0] + 4 * kVBlock);
#pragma unroll 1
      for (int k8 = 0; k8 < kVKeys; k8 += 8) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const int cur = kk & 1, nxt = cur ^ 1;
          const int nk = min(k8 + kk + 1, kVKeys - 1);
          const int nkk = (kk + 1) & 7;                  // nk & 7 unless clamped
          const int nsw = (((kk + 1) & 7) >> 2) & 1;     // (nk >> 2) & 1 (k8 is a multiple of 8)
          fp[nxt][0] = lds128(pkey + nk * 32 + ((0 ^ nsw) << 4));
          fp[nxt][1] = lds128(pkey + nk * 32 + ((1 ^ nsw) << 4));
          const uint32_t vrow = vslot + voff[nkk] + (nk - nkk) * 128;
          fv[nxt][0] = lds128(vrow);
          fv[nxt][1] = lds128(vrow + 4 * kVBlock);
          const float pr[8] = {fp[cur][0].x, fp[cur][0].y, fp[cur][0].z, fp[cur][0].w,
                               fp[cur][1].x, fp[cur][1].y, fp[cur][1].z, fp[cur][1].w};
          const float vc[8] = {fv[cur][0].x, fv[cur][0].y, fv[cur][0].z, fv[cur][0].w,
                               fv[cur][1].x, fv[cur][1].y, fv[cur][1].z, fv[cur][1].w};
#pragma unroll
          for (int r = 0; r < 8; ++r)
#pragma unroll
            for (int c = 0; c < 8; c += 2) ffma2(o[r][c], o[r][c + 1], pr[r], pr[r], vc[c], vc[c + 1]);
        }
      }
      // The last warp done with V quarter vp issues K quarter vp of the next tile.
      release(kt, 4 + vp, 2 * t + 1);
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
    const cuuint32_t kbox[4] = {cuuint32_t(kBoxCols), cuuint32_t(kBc), 2, 1};       // K: 128 keys x 64 d
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
