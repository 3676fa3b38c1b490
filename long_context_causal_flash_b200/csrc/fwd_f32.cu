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
// 1 CTA per SM).  TMA loads of the Q tile (once) and of K and V tiles (64 keys x 256,
// fp32, 128-byte swizzle) go into one K and one V buffer: the warp that finishes
// S(t) = Q K(t)^T last (a shared-memory arrival count) issues K(t+1), which then
// streams in during softmax and O += P V(t); the last to finish PV(t) issues V(t+1),
// which streams in during S(t+1).  No warp ever blocks to issue a copy.
//   warp w owns query rows 8w .. 8w+7 for the whole key loop:
//     S = Q K^T   each lane a 4 x 4 register tile (4 rows x keys tc + 16 i)
//     softmax     online, base 2, row max / sum by warp shuffles over 16 lanes
//     O += P V    each lane an 8 x 8 register tile (8 rows x cols 4l.., 128+4l..)
//   P goes through a warp-private 2 KiB slice of shared memory, so warps never
//   wait for one another inside the key loop.
// Block skipping: the key-tile range per query tile comes from the plan; SKIP
// tiles are neither loaded nor computed, FULL tiles skip the per-element mask.
#include "internal.h"

namespace gqa {
namespace {

constexpr int kRows = kF32Rows;  // 64 query rows per CTA
constexpr int kBc = kF32Bc;      // 64 keys per tile
constexpr int kConsumerWarps = 8;
constexpr int kThreads = kConsumerWarps * 32;
constexpr int kBoxCols = 32;                  // fp32 per 128-byte swizzle row
constexpr int kBoxBytes = 64 * 128;           // 64 rows x 32 fp32
constexpr int kTileBytes = 8 * kBoxBytes;     // 64 rows x 256 fp32
constexpr int kPWarpBytes = kBc * 8 * 2 * 4;  // P^T slice: [64 keys][8 rows] fp32 pairs (p, p)
constexpr int kOffQ = 0;
constexpr int kOffK = kTileBytes;
constexpr int kOffV = 2 * kTileBytes;
constexpr int kOffP = 3 * kTileBytes;
constexpr int kOffBar = kOffP + kConsumerWarps * kPWarpBytes;
constexpr int kSmemBytes = kOffBar + 64 + 1024;  // + slack to align to the 1024-byte swizzle atom
// After the barriers (5 x 8 bytes): arrival counters for K and V, and the number of
// K and V loads issued (read back at exit to drain copies still in flight).
enum { kCntK = 40, kCntV = 44, kIssK = 48, kIssV = 52 };

static_assert(kRows == 8 * kConsumerWarps, "one consumer warp per 8 query rows");

enum { kBarQ = 0, kBarFullK = 1, kBarFullV = 2 };

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
  const uint32_t sQ = sbase + kOffQ, sK = sbase + kOffK, sV = sbase + kOffV, sP = sbase + kOffP;
  const uint32_t bar = sbase + kOffBar;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // Unit: (query tile, kv head, batch[, key split]); query tiles in descending order
  // so the longest causal rows start first.
  const int splits = p.splits > 1 ? p.splits : 1;
  const int split = int(blockIdx.x % unsigned(splits));
  const unsigned unit = blockIdx.x / unsigned(splits);
  const int per_qt = p.Hkv * p.B;
  const int qt = p.nq - 1 - int(unit / per_qt);
  const int rem = int(unit % per_qt);
  const int g = rem % p.Hkv;
  const int b = rem / p.Hkv;
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

  uint32_t* cnt = reinterpret_cast<uint32_t*>(smem_raw + (bar - raw));  // generic view of the barrier area
  if (threadIdx.x == 0) {
    mbar_init(bar + 8 * kBarQ, 1);
    mbar_init(bar + 8 * kBarFullK, 1);
    mbar_init(bar + 8 * kBarFullV, 1);
    cnt[kCntK / 4] = 0;
    cnt[kCntV / 4] = 0;
    cnt[kIssK / 4] = 0;
    cnt[kIssV / 4] = 0;
    fence_barrier_init();
  }
  __syncthreads();

  const int qhead = b * p.Hq + g * p.G;
  const int kvhead = b * p.Hkv + g;
  auto next_tile = [&](int kt) {
    while (kt < kend && classify(p, ctx, kt) == GQA_TILE_SKIP) ++kt;
    return kt;
  };
  auto load_k = [&](int kt) {
    mbar_arrive_expect_tx(bar + 8 * kBarFullK, kTileBytes);
    for (int c = 0; c < 8; ++c)
      tma_load_3d(sK + c * kBoxBytes, &tmK, bar + 8 * kBarFullK, c * kBoxCols, kt * kBc, kvhead);
    atomicAdd(&cnt[kIssK / 4], 1u);
  };
  auto load_v = [&](int kt) {
    mbar_arrive_expect_tx(bar + 8 * kBarFullV, kTileBytes);
    for (int c = 0; c < 8; ++c)
      tma_load_3d(sV + c * kBoxBytes, &tmV, bar + 8 * kBarFullV, c * kBoxCols, kt * kBc, kvhead);
    atomicAdd(&cnt[kIssV / 4], 1u);
  };
  if (threadIdx.x == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    mbar_arrive_expect_tx(bar + 8 * kBarQ, kTileBytes);
    for (int c = 0; c < 8; ++c)
      tma_load_3d(sQ + c * kBoxBytes, &tmQ, bar + 8 * kBarQ, c * kBoxCols, int(q0), qhead);
    const int k0 = next_tile(kbeg);
    if (k0 < kend) {
      load_k(k0);
      load_v(k0);
    }
  }

  // ------------------------------------------------------------------ consumers
  const int tr = lane >> 4;  // S tile: rows 4tr .. 4tr+3 of this warp
  const int tc = lane & 15;  // S tile: keys tc + 16 i
  const uint32_t sPw = sP + warp * kPWarpBytes;

  // Positions / segment ids of this lane's 4 S rows.
  int64_t pos[4];
  int sq[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = 8 * warp + 4 * tr + i;
    // the last key this row sees: its position, or the block's last key when the
    // key block ends before it (a block of a sharded sequence)
    pos[i] = min(q0 + (r % br) + p.off, p.Lk - 1);
    const int64_t qi = min(q0 + (r % br), p.Lq - 1);
    sq[i] = p.has_seg ? p.seg_q[qi] : 0;
  }

  float o[8][8];
#pragma unroll
  for (int r = 0; r < 8; ++r)
#pragma unroll
    for (int c = 0; c < 8; ++c) o[r][c] = 0.f;
  float m[4], l[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    m[i] = -INFINITY;
    l[i] = 0.f;
  }

  bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(bar + 8 * kBarQ, 0, p.wait_budget_ns, p.status));

  // Shared-memory addresses.  Row r of box c lives at c*8K + r*128, its 16-byte
  // chunk x at physical chunk x ^ (r & 7) (TMA 128-byte swizzle).  Q rows of this
  // lane are 4tr + i, so chunk pc of row i sits at (pc ^ i) ^ 4tr: the xor with
  // 4tr is +64 or -64 bytes depending on bit 2 of (pc ^ i), hence two bases.  K
  // rows are tc + 16 jj (row & 7 = tc & 7): one base per chunk.  Same for V rows k.
  const uint32_t qrow = sQ + (8 * warp + 4 * tr) * 128;
  const uint32_t q_up = qrow + 64 * tr, q_dn = qrow - 64 * tr;
  uint32_t kaddr[8], vaddr[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    kaddr[c] = sK + tc * 128 + (uint32_t(c ^ (tc & 7)) << 4);
    vaddr[c] = sV + (lane >> 3) * kBoxBytes + c * 128 + (uint32_t(c ^ (lane & 7)) << 4);
  }

  int t = 0;
  for (int kt = kbeg; kt < kend && ok; ++kt) {
    const int cls = classify(p, ctx, kt);
    if (cls == GQA_TILE_SKIP) continue;
    const uint32_t parity = uint32_t(t) & 1u;
    const int64_t j0 = int64_t(kt) * kBc;

    // ---- S = Q K^T (4 x 4 per lane, depth 256)
    ok = __all_sync(0xffffffffu, mbar_wait_bounded(bar + 8 * kBarFullK, parity, p.wait_budget_ns, p.status));
    if (!ok) break;
    // Each score is accumulated as two partial sums (even / odd elements of d) in a
    // register pair, so every pair of products is one packed FMA.
    float2 s2[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) s2[i][jj] = make_float2(0.f, 0.f);
    // Fragments are double-buffered: the loads for K-step n+1 are issued before the
    // 64 FFMAs of step n, so shared-memory latency hides behind arithmetic.
    float4 fa[2][4], fk[2][4];
#pragma unroll
    for (int i = 0; i < 4; ++i) fa[0][i] = lds128(((i & 4) ? q_dn : q_up) + i * 128 + (i << 4));
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) fk[0][jj] = lds128(kaddr[0] + jj * 16 * 128);
#pragma unroll 1
    for (int box = 0; box < 8; ++box) {
      const uint32_t bo = box * kBoxBytes;
      const uint32_t bn = box < 7 ? bo + kBoxBytes : bo;  // the last prefetch re-reads box 7
#pragma unroll
      for (int pc = 0; pc < 8; ++pc) {
        const int cur = pc & 1, nxt = cur ^ 1;
        const int npc = (pc + 1) & 7;
        const uint32_t nbo = pc == 7 ? bn : bo;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int x = npc ^ i;
          fa[nxt][i] = lds128(((x & 4) ? q_dn : q_up) + nbo + i * 128 + (x << 4));
        }
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) fk[nxt][jj] = lds128(kaddr[npc] + nbo + jj * 16 * 128);
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int jj = 0; jj < 4; ++jj)
            ffma2(s2[i][jj].x, s2[i][jj].y, fa[cur][i].x, fa[cur][i].y, fk[cur][jj].x, fk[cur][jj].y);
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int jj = 0; jj < 4; ++jj)
            ffma2(s2[i][jj].x, s2[i][jj].y, fa[cur][i].z, fa[cur][i].w, fk[cur][jj].z, fk[cur][jj].w);
      }
    }
    float s[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) s[i][jj] = s2[i][jj].x + s2[i][jj].y;
    // The last warp done with K(t) issues K of the next tile.
    __syncwarp();
    if (lane == 0) {
      __threadfence_block();
      if (atomicAdd(&cnt[kCntK / 4], 1u) == uint32_t(kConsumerWarps * (t + 1) - 1)) {
        const int kn = next_tile(kt + 1);
        if (kn < kend) load_k(kn);
      }
    }

    // ---- mask + online softmax (base 2)
    const bool need_mask = (cls == GQA_TILE_PARTIAL) || (j0 + kBc > p.Lk);
    int sk[4];
    if (need_mask && p.has_seg) {
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) sk[jj] = p.seg_kv[min(j0 + tc + 16 * jj, p.Lk - 1)];
    }
    float alpha[4], mx[4], rs[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      mx[i] = -INFINITY;
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        float x = s[i][jj] * p.scale_log2;
        if (need_mask) {
          const int64_t j = j0 + tc + 16 * jj;
          bool vis = j <= pos[i];
          if (p.has_seg) vis = vis && (sq[i] == sk[jj] || j < p.P0);
          if (!vis) x = -INFINITY;
        }
        s[i][jj] = x;
        mx[i] = fmaxf(mx[i], x);
      }
    }
    // The four rows' reductions interleaved: four dependent shuffle steps, not sixteen.
#pragma unroll
    for (int o = 1; o < 16; o <<= 1)
#pragma unroll
      for (int i = 0; i < 4; ++i) mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], o));
    float m_ref[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float m_new = fmaxf(m[i], mx[i]);
      m_ref[i] = (m_new == -INFINITY) ? 0.f : m_new;  // no visible key yet
      alpha[i] = exp2f(m[i] - m_ref[i]);
      m[i] = m_new;
      rs[i] = 0.f;
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const float e = exp2f(s[i][jj] - m_ref[i]);
        s[i][jj] = e;
        rs[i] += e;
      }
    }
#pragma unroll
    for (int o = 1; o < 16; o <<= 1)
#pragma unroll
      for (int i = 0; i < 4; ++i) rs[i] += __shfl_xor_sync(0xffffffffu, rs[i], o);
#pragma unroll
    for (int i = 0; i < 4; ++i) l[i] = l[i] * alpha[i] + rs[i];
    // P^T slice: [key][row] with each value stored twice, the (p, p) operand of
    // the packed FMAs below.
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      const uint32_t a = sPw + (tc + 16 * jj) * 64 + tr * 32;
      sts128(a, s[0][jj], s[0][jj], s[1][jj], s[1][jj]);
      sts128(a + 16, s[2][jj], s[2][jj], s[3][jj], s[3][jj]);
    }
    __syncwarp();

    // ---- O = alpha * O + P V  (8 rows x 8 cols per lane)
    {
      float a8[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float other = __shfl_xor_sync(0xffffffffu, alpha[i], 16);
        a8[i] = tr == 0 ? alpha[i] : other;
        a8[4 + i] = tr == 0 ? other : alpha[i];
      }
#pragma unroll
      for (int r = 0; r < 8; ++r)
#pragma unroll
        for (int c = 0; c < 8; ++c) o[r][c] *= a8[r];
    }
    ok = __all_sync(0xffffffffu, mbar_wait_bounded(bar + 8 * kBarFullV, parity, p.wait_budget_ns, p.status));
    if (!ok) break;
    {
      // Same double buffering for P and V; the last prefetch re-reads key 63.
      float4 fp[2][4], fv[2][2];
#pragma unroll
      for (int u = 0; u < 4; ++u) fp[0][u] = lds128(sPw + u * 16);
      fv[0][0] = lds128(vaddr[0]);
      fv[0][1] = lds128(vaddr[0] + 4 * kBoxBytes);
#pragma unroll 1
      for (int k8 = 0; k8 < kBc; k8 += 8) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const int cur = kk & 1, nxt = cur ^ 1;
          const int nk = min(k8 + kk + 1, kBc - 1);
          const int nkk = nk & 7, nk8 = nk & ~7;
#pragma unroll
          for (int u = 0; u < 4; ++u) fp[nxt][u] = lds128(sPw + nk * 64 + u * 16);
          fv[nxt][0] = lds128(vaddr[(kk + 1) & 7] + nk8 * 128 + (nkk - ((kk + 1) & 7)) * 128);
          fv[nxt][1] = lds128(vaddr[(kk + 1) & 7] + 4 * kBoxBytes + nk8 * 128 + (nkk - ((kk + 1) & 7)) * 128);
          const float vc[8] = {fv[cur][0].x, fv[cur][0].y, fv[cur][0].z, fv[cur][0].w,
                               fv[cur][1].x, fv[cur][1].y, fv[cur][1].z, fv[cur][1].w};
#pragma unroll
          for (int r = 0; r < 8; ++r) {
            const float4 pq = fp[cur][r >> 1];
            const float p0 = (r & 1) ? pq.z : pq.x, p1 = (r & 1) ? pq.w : pq.y;  // (p_r, p_r)
#pragma unroll
            for (int c = 0; c < 8; c += 2) ffma2(o[r][c], o[r][c + 1], p0, p1, vc[c], vc[c + 1]);
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) {
      __threadfence_block();
      if (atomicAdd(&cnt[kCntV / 4], 1u) == uint32_t(kConsumerWarps * (t + 1) - 1)) {
        const int kn = next_tile(kt + 1);
        if (kn < kend) load_v(kn);
      }
    }
    ++t;
  }
  // A wait that ran out leaves ok == false: the status word says so and this warp's
  // outputs are not written.  Every thread still meets the barrier at the end.
  if (ok) {
  // ---- epilogue: out = O / l, lse = (m + log2 l) ln 2
  float l8[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float other = __shfl_xor_sync(0xffffffffu, l[i], 16);
    l8[i] = tr == 0 ? l[i] : other;
    l8[4 + i] = tr == 0 ? other : l[i];
  }
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
    const float inv = l8[rr] > 0.f ? 1.f / l8[rr] : 0.f;
    float* row = out + (int64_t(head) * p.Lq + qi) * kHeadDim;
    float4 w0 = make_float4(o[rr][0] * inv, o[rr][1] * inv, o[rr][2] * inv, o[rr][3] * inv);
    float4 w1 = make_float4(o[rr][4] * inv, o[rr][5] * inv, o[rr][6] * inv, o[rr][7] * inv);
    *reinterpret_cast<float4*>(row + 4 * lane) = w0;
    *reinterpret_cast<float4*>(row + 128 + 4 * lane) = w1;
  }
  if (tc == 0) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = 8 * warp + 4 * tr + i;
      const int64_t qi = q0 + (r % br);
      if (qi >= p.Lq) continue;
      const int head = b * p.Hq + g * p.G + r / br;
      lse_out[int64_t(head) * p.Lq + qi] = l[i] > 0.f ? (m[i] + log2f(l[i])) * kLn2 : -INFINITY;
    }
  }
  }  // if (ok)
  __syncthreads();
  if (threadIdx.x == 0) {  // no copy may be in flight when the CTA ends (returns at once normally)
    mbar_wait_bounded(bar + 8 * kBarQ, 0, p.wait_budget_ns, p.status);
    const uint32_t nk = cnt[kIssK / 4], nv = cnt[kIssV / 4];
    if (nk) mbar_wait_bounded(bar + 8 * kBarFullK, (nk - 1) & 1u, p.wait_budget_ns, p.status);
    if (nv) mbar_wait_bounded(bar + 8 * kBarFullV, (nv - 1) & 1u, p.wait_budget_ns, p.status);
  }
}

}  // namespace

int launch_fwd_f32(const FwdTensors& t, const FwdParams& p, cudaStream_t stream) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return GQA_ERR_LAUNCH;
  CUtensorMap mq, mk, mv;
  const cuuint32_t estr[3] = {1, 1, 1};
  {
    const cuuint64_t dims[3] = {cuuint64_t(kHeadDim), cuuint64_t(p.Lq), cuuint64_t(p.B) * p.Hq};
    const cuuint64_t strides[2] = {cuuint64_t(kHeadDim) * 4, cuuint64_t(p.Lq) * kHeadDim * 4};
    const cuuint32_t box[3] = {cuuint32_t(kBoxCols), cuuint32_t(p.br), cuuint32_t(p.G)};
    if (enc(&mq, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(t.q), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return GQA_ERR_LAUNCH;
  }
  {
    const cuuint64_t dims[3] = {cuuint64_t(kHeadDim), cuuint64_t(p.Lk), cuuint64_t(p.B) * p.Hkv};
    const cuuint64_t strides[2] = {cuuint64_t(kHeadDim) * 4, cuuint64_t(p.Lk) * kHeadDim * 4};
    const cuuint32_t box[3] = {cuuint32_t(kBoxCols), cuuint32_t(kBc), 1};
    if (enc(&mk, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(t.k), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return GQA_ERR_LAUNCH;
    if (enc(&mv, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(t.v), dims, strides, box, estr,
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
