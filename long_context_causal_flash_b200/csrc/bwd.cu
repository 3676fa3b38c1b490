// Attention backward (dQ, dK, dV from the saved LSE) on the FP32 pipe, sm_100a.
//
// Training over packed long sequences (maxtext PR #4929, description: the splash
// kernel runs inside training steps on 1,048,576-token packed batches) needs the
// gradients of the attention output.  With P = exp(scale * S - LSE) recomputed from
// the forward's log-sum-exp, D_i = <dO_i, O_i>, dP = dO V^T and dS = P * (dP - D):
//     dV_j = sum_{h in group} sum_i P_ij dO_i,   dK_j = scale * sum_{h in group} sum_i dS_ij Q_i,
//     dQ_i = scale * sum_j dS_ij K_j.
// Three kernels, no atomics:
//   bwd_rowdot_kernel   D = rowsum(dO * O), one warp per row.
//   bwd_dkv_kernel      one CTA per (key tile of 32 keys, kv head, batch): dK and dV of
//                       the tile stay in registers while the CTA visits every query
//                       tile (64 rows = 64/G positions x the G heads of the kv head)
//                       that sees the key tile, so the G query heads' contributions
//                       to their shared key/value head are summed on chip.
//   bwd_dq_kernel       one CTA per (query tile, kv head, batch): dQ stays in
//                       registers while the CTA visits the key tiles of the query
//                       tile's range (the forward's block-skip plan at these tile
//                       sizes; SKIP tiles are never loaded).
// Both dtypes run here: bf16 inputs are widened to fp32 on load, all arithmetic is
// fp32, and the gradients are written in the input dtype (bf16 round-to-nearest-even).
// Tiles are staged in shared memory with rows padded to 260 floats, so eight rows
// read at the same column fall into different banks.
#include <cuda_bf16.h>

#include "internal.h"

namespace gqa {
namespace {

constexpr int kThreads = 256;
constexpr int kRowsQ = kBwdRowsQ;  // query rows per query tile (positions x heads)
constexpr int kKeys = kBwdKeys;    // keys per key tile
constexpr int kPad = 260;    // floats per staged row of d = 256
constexpr int kPStride = 36; // floats per row of the P / dS tiles (16-byte aligned)

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
  const int32_t* q_bounds;   // [nq][2] or null
  const int32_t* kv_bounds;  // [nk][2] or null
  const int32_t* q_ranges;   // [nq][2] or null
  int64_t Lq, Lk, off, P0;
  int B, Hq, Hkv, G, br, nq, nk, has_seg, bf16;
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

__device__ __forceinline__ void st4(void* base, int64_t idx, bool bf16, float a, float b, float c, float d) {
  if (bf16) {
    __nv_bfloat162 h[2] = {__floats2bfloat162_rn(a, b), __floats2bfloat162_rn(c, d)};
    *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(base) + idx) = *reinterpret_cast<const uint2*>(h);
  } else {
    *reinterpret_cast<float4*>(static_cast<float*>(base) + idx) = make_float4(a, b, c, d);
  }
}

// Stages `kRowsT` rows of 256 elements (global row index from `row_of`, -1 for none)
// into shared memory as fp32 with the padded stride.  Every load of the thread is
// issued before the first store, so their latencies overlap.
template <int kRowsT, typename RowOf>
__device__ __forceinline__ void stage_rows(float* dst, const void* src, bool bf16, RowOf row_of) {
  constexpr int kPer = kRowsT * 32 / kThreads;  // 8-element chunks per thread
  static_assert(kRowsT * 32 % kThreads == 0, "whole chunks per thread");
  uint4 raw[kPer][2];
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int e = threadIdx.x + i * kThreads;
    const int r = e >> 5, c8 = (e & 31) * 8;
    const int64_t gr = row_of(r);
    raw[i][0] = raw[i][1] = make_uint4(0u, 0u, 0u, 0u);
    if (gr >= 0) {
      if (bf16) {
        raw[i][0] = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(src) + gr * kHeadDim + c8);
      } else {
        const uint4* g = reinterpret_cast<const uint4*>(static_cast<const float*>(src) + gr * kHeadDim + c8);
        raw[i][0] = g[0];
        raw[i][1] = g[1];
      }
    }
  }
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int e = threadIdx.x + i * kThreads;
    const int r = e >> 5, c8 = (e & 31) * 8;
    float4* d = reinterpret_cast<float4*>(dst + r * kPad + c8);
    if (bf16) {
      const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw[i][0]);
      const float2 f0 = __bfloat1622float2(h[0]), f1 = __bfloat1622float2(h[1]);
      const float2 f2 = __bfloat1622float2(h[2]), f3 = __bfloat1622float2(h[3]);
      d[0] = make_float4(f0.x, f0.y, f1.x, f1.y);
      d[1] = make_float4(f2.x, f2.y, f3.x, f3.y);
    } else {
      d[0] = *reinterpret_cast<const float4*>(&raw[i][0]);
      d[1] = *reinterpret_cast<const float4*>(&raw[i][1]);
    }
  }
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

// 16 dot products per thread over d = 256 between two staged tiles: rows rg, rg + 16,
// rg + 32, rg + 48 of A (64 rows) and rows kg, kg + 8, kg + 16, kg + 24 of Bm (32 rows),
// for one half of the CTA (rg = (t % 128) / 8, kg = t % 8): one half computes S = Q K^T
// while the other computes dP = dO V^T.  Four rows x four keys per thread take 8
// fragment loads per 32 packed FMAs.  A warp's four row groups are consecutive rows,
// 4 banks apart in the 260-float padding, so the row fragments never conflict.  Each
// dot product is two partial sums (even / odd elements of d) so that every pair of
// products is one packed FMA.
__device__ __forceinline__ void dots_4x4(const float* A, const float* Bm, int rg, int kg, float (&acc)[4][4]) {
  float2 a2[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int m = 0; m < 4; ++m) a2[i][m] = make_float2(0.f, 0.f);
#pragma unroll 2
  for (int d4 = 0; d4 < kHeadDim / 4; ++d4) {
    float4 x[4], y[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) x[i] = reinterpret_cast<const float4*>(A + (rg + 16 * i) * kPad)[d4];
#pragma unroll
    for (int m = 0; m < 4; ++m) y[m] = reinterpret_cast<const float4*>(Bm + (kg + 8 * m) * kPad)[d4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int m = 0; m < 4; ++m) ffma2(a2[i][m].x, a2[i][m].y, x[i].x, x[i].y, y[m].x, y[m].y);
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int m = 0; m < 4; ++m) ffma2(a2[i][m].x, a2[i][m].y, x[i].z, x[i].w, y[m].z, y[m].w);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int m = 0; m < 4; ++m) acc[i][m] = a2[i][m].x + a2[i][m].y;
}

__device__ __forceinline__ int bwd_classify(const BwdParams& p, int qt, int kt) {
  const int64_t i0 = int64_t(qt) * p.br, i1 = min(p.Lq, i0 + p.br) - 1;
  const int64_t j0 = int64_t(kt) * kKeys, j1 = min(p.Lk, j0 + kKeys) - 1;
  SegBounds qb{0, 0}, kb{0, 0};
  if (p.has_seg) {
    qb = SegBounds{p.q_bounds[2 * qt], p.q_bounds[2 * qt + 1]};
    kb = SegBounds{p.kv_bounds[2 * kt], p.kv_bounds[2 * kt + 1]};
  }
  return tile_class(i0, i1, j0, j1, p.off, p.P0, p.has_seg != 0, qb, kb);
}

// Per-row state of a staged query tile: log2-domain LSE (+inf for rows that take no
// part: past Lq or without a visible key), D, position and segment id.
struct RowState {
  float* L2;
  float* D;
  int64_t* pos;
  int* seg;
};

__device__ __forceinline__ void stage_row_state(const BwdParams& p, RowState rs, int64_t q0, int b, int g) {
  for (int r = threadIdx.x; r < kRowsQ; r += kThreads) {
    const int hh = r / p.br, pp = r % p.br;
    const int64_t qi = q0 + pp;
    const bool live = hh < p.G && qi < p.Lq;
    const int64_t row = (int64_t(b) * p.Hq + g * p.G + hh) * p.Lq + qi;
    const float l = live ? p.lse[row] : -INFINITY;
    rs.L2[r] = l == -INFINITY ? INFINITY : l * kLog2e;
    rs.D[r] = live ? p.D[row] : 0.f;
    rs.pos[r] = live ? qi + p.off : -1;
    rs.seg[r] = (live && p.has_seg) ? p.seg_q[qi] : 0;
  }
}

// P of the 4 x 4 score block of an S thread (rows rg + 16 i, keys kg + 8 m of key
// tile j0), written to P[row][key].
__device__ __forceinline__ void store_probs(const BwdParams& p, const RowState& rs, int64_t j0, bool need_mask,
                                            int rg, int kg, const float (&s)[4][4], float* P) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = rg + 16 * i;
    const float L2 = rs.L2[r];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const int64_t j = j0 + kg + 8 * m;
      bool vis = true;
      if (need_mask) {
        vis = j < p.Lk && j <= rs.pos[r];
        if (p.has_seg) vis = vis && (j < p.P0 || rs.seg[r] == p.seg_kv[min(j, p.Lk - 1)]);
      }
      P[r * kPStride + kg + 8 * m] = vis ? exp2f(fmaf(s[i][m], p.scale_log2, -L2)) : 0.f;
    }
  }
}

// dS = P (dP - D) of the 4 x 4 block of a dP thread, from P[row][key]; written to dS
// (which may be P itself: each element is read and written by the same thread).
__device__ __forceinline__ void store_dscores(const RowState& rs, int rg, int kg, const float (&dp)[4][4],
                                              const float* P, float* dS) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = rg + 16 * i;
    const float D = rs.D[r];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const int idx = r * kPStride + kg + 8 * m;
      dS[idx] = P[idx] * (dp[i][m] - D);
    }
  }
}

// smem layout shared by both kernels (floats)
constexpr int kOffBig0 = 0;                        // Q tile [64][kPad]
constexpr int kOffBig1 = kOffBig0 + kRowsQ * kPad; // dO tile [64][kPad]
constexpr int kOffK = kOffBig1 + kRowsQ * kPad;    // K tile [32][kPad]
constexpr int kOffV = kOffK + kKeys * kPad;        // V tile [32][kPad]
constexpr int kOffP = kOffV + kKeys * kPad;        // P (or dS) [64][kPStride]
constexpr int kOffS = kOffP + kRowsQ * kPStride;   // dS [64][kPStride] (dK/dV kernel)
constexpr int kOffRow = kOffS + kRowsQ * kPStride; // L2[64], D[64], seg[64], pos[64] (int64)
constexpr int kSmemFloats = kOffRow + 3 * kRowsQ + 2 * kRowsQ;
constexpr size_t kSmemBytes = size_t(kSmemFloats) * 4;
static_assert(kSmemBytes <= 232448, "shared memory per block");

__device__ __forceinline__ RowState row_state(float* sm) {
  RowState rs;
  rs.L2 = sm + kOffRow;
  rs.D = rs.L2 + kRowsQ;
  rs.seg = reinterpret_cast<int*>(rs.D + kRowsQ);
  rs.pos = reinterpret_cast<int64_t*>(rs.seg + kRowsQ);
  return rs;
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

// dQ of one query tile (64 rows = br positions x G heads of kv head g) over the key
// tiles of its range.  Thread t owns rows 8 (t / 32) .. +7 and columns 4 (t % 32) .. +3
// and 128 + 4 (t % 32) .. +3 of dQ.
__global__ void __launch_bounds__(kThreads, 1) bwd_dq_kernel(const BwdParams p) {
  extern __shared__ __align__(16) float sm[];
  float *Qs = sm + kOffBig0, *dOs = sm + kOffBig1, *Ks = sm + kOffK, *Vs = sm + kOffV, *Ps = sm + kOffP;
  const RowState rs = row_state(sm);
  const bool bf16 = p.bf16 != 0;
  const int per_qt = p.Hkv * p.B;
  const int qt = p.nq - 1 - int(blockIdx.x / per_qt);  // longest rows first
  const int rem = int(blockIdx.x % per_qt);
  const int g = rem % p.Hkv, b = rem / p.Hkv;
  const int64_t q0 = int64_t(qt) * p.br;
  auto qrow = [&](int r) -> int64_t {
    const int hh = r / p.br;
    const int64_t qi = q0 + r % p.br;
    return (hh < p.G && qi < p.Lq) ? (int64_t(b) * p.Hq + g * p.G + hh) * p.Lq + qi : -1;
  };
  stage_rows<kRowsQ>(Qs, p.q, bf16, qrow);
  stage_rows<kRowsQ>(dOs, p.dout, bf16, qrow);
  stage_row_state(p, rs, q0, b, g);
  int kbeg, kend;
  if (p.has_seg) {
    kbeg = p.q_ranges[2 * qt];
    kend = p.q_ranges[2 * qt + 1];
  } else {
    kv_range_no_seg(min(p.Lq, q0 + p.br) - 1, p.off, kKeys, p.nk, &kbeg, &kend);
  }
  const int rbase = (threadIdx.x >> 5) * 8, c4 = (threadIdx.x & 31) * 4;
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[i][c] = 0.f;
  const int64_t kvbase = (int64_t(b) * p.Hkv + g) * p.Lk;
  for (int kt = kbeg; kt < kend; ++kt) {
    const int cls = bwd_classify(p, qt, kt);
    if (cls == GQA_TILE_SKIP) continue;
    const int64_t j0 = int64_t(kt) * kKeys;
    __syncthreads();  // the previous tile's K and dS are no longer read
    auto krow = [&](int r) -> int64_t { return j0 + r < p.Lk ? kvbase + j0 + r : -1; };
    stage_rows<kKeys>(Ks, p.k, bf16, krow);
    stage_rows<kKeys>(Vs, p.v, bf16, krow);
    __syncthreads();
    // Warps 0-3: S and P (into Ps); warps 4-7: dP, then dS = P (dP - D) over P.
    const bool s_half = threadIdx.x < kThreads / 2;
    const int rg = (threadIdx.x & 127) >> 3, kg = threadIdx.x & 7;
    float sc[4][4];
    dots_4x4(s_half ? Qs : dOs, s_half ? Ks : Vs, rg, kg, sc);
    const bool need_mask = cls == GQA_TILE_PARTIAL || j0 + kKeys > p.Lk;
    if (s_half) store_probs(p, rs, j0, need_mask, rg, kg, sc, Ps);
    __syncthreads();
    if (!s_half) store_dscores(rs, rg, kg, sc, Ps, Ps);
    __syncthreads();
    // dQ += dS K: four keys' weights per row in one load.
#pragma unroll 1
    for (int j4 = 0; j4 < kKeys; j4 += 4) {
      float4 w[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) w[i] = reinterpret_cast<const float4*>(Ps + (rbase + i) * kPStride + j4)[0];
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const float4 ka = reinterpret_cast<const float4*>(Ks + (j4 + jj) * kPad + c4)[0];
        const float4 kb = reinterpret_cast<const float4*>(Ks + (j4 + jj) * kPad + 128 + c4)[0];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float wv = jj == 0 ? w[i].x : jj == 1 ? w[i].y : jj == 2 ? w[i].z : w[i].w;
          acc[i][0] = fmaf(wv, ka.x, acc[i][0]);
          acc[i][1] = fmaf(wv, ka.y, acc[i][1]);
          acc[i][2] = fmaf(wv, ka.z, acc[i][2]);
          acc[i][3] = fmaf(wv, ka.w, acc[i][3]);
          acc[i][4] = fmaf(wv, kb.x, acc[i][4]);
          acc[i][5] = fmaf(wv, kb.y, acc[i][5]);
          acc[i][6] = fmaf(wv, kb.z, acc[i][6]);
          acc[i][7] = fmaf(wv, kb.w, acc[i][7]);
        }
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int64_t row = qrow(rbase + i);
    if (row < 0) continue;
    st4(p.dq, row * kHeadDim + c4, bf16, acc[i][0] * p.scale, acc[i][1] * p.scale, acc[i][2] * p.scale,
        acc[i][3] * p.scale);
    st4(p.dq, row * kHeadDim + 128 + c4, bf16, acc[i][4] * p.scale, acc[i][5] * p.scale, acc[i][6] * p.scale,
        acc[i][7] * p.scale);
  }
}

// dK and dV of one key tile (32 keys of kv head g) over every query tile that sees it.
// Warps 0-3 accumulate dV, warps 4-7 dK: thread t owns keys 8 ((t / 32) % 4) .. +7 and
// columns 4 (t % 32) .. +3 and 128 + 4 (t % 32) .. +3 of its accumulator.
__global__ void __launch_bounds__(kThreads, 1) bwd_dkv_kernel(const BwdParams p) {
  extern __shared__ __align__(16) float sm[];
  float *Qs = sm + kOffBig0, *dOs = sm + kOffBig1, *Ks = sm + kOffK, *Vs = sm + kOffV;
  float *Ps = sm + kOffP, *dSs = sm + kOffS;
  __shared__ int range[2];
  const RowState rs = row_state(sm);
  const bool bf16 = p.bf16 != 0;
  const int per_kt = p.Hkv * p.B;
  const int kt = int(blockIdx.x / per_kt);  // early keys see the most rows: first
  const int rem = int(blockIdx.x % per_kt);
  const int g = rem % p.Hkv, b = rem / p.Hkv;
  const int64_t j0 = int64_t(kt) * kKeys;
  const int64_t kvbase = (int64_t(b) * p.Hkv + g) * p.Lk;
  auto krow = [&](int r) -> int64_t { return j0 + r < p.Lk ? kvbase + j0 + r : -1; };
  stage_rows<kKeys>(Ks, p.k, bf16, krow);
  stage_rows<kKeys>(Vs, p.v, bf16, krow);
  // Query tiles that can see this key tile: causally from the first row at position
  // >= j0 (every row for a shared-state key tile); with segment ids the first and last
  // non-SKIP tile of that range, found by the whole CTA.
  int qa = (j0 < p.P0 || j0 <= p.off) ? 0 : int((j0 - p.off) / p.br);
  int qb = p.nq;
  if (p.has_seg) {
    if (threadIdx.x == 0) range[0] = p.nq, range[1] = -1;
    __syncthreads();
    int lo = p.nq, hi = -1;
    for (int qt = qa + int(threadIdx.x); qt < p.nq; qt += kThreads)
      if (bwd_classify(p, qt, kt) != GQA_TILE_SKIP) lo = min(lo, qt), hi = max(hi, qt);
    if (hi >= 0) {
      atomicMin(&range[0], lo);
      atomicMax(&range[1], hi);
    }
    __syncthreads();
    qa = range[0];
    qb = range[1] + 1;
  }
  const bool is_dk = threadIdx.x >= kThreads / 2;
  const int kbase = ((threadIdx.x >> 5) & 3) * 8, c4 = (threadIdx.x & 31) * 4;
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[i][c] = 0.f;
  for (int qt = qa; qt < qb; ++qt) {
    const int cls = bwd_classify(p, qt, kt);
    if (cls == GQA_TILE_SKIP) continue;
    const int64_t q0 = int64_t(qt) * p.br;
    auto qrow = [&](int r) -> int64_t {
      const int hh = r / p.br;
      const int64_t qi = q0 + r % p.br;
      return (hh < p.G && qi < p.Lq) ? (int64_t(b) * p.Hq + g * p.G + hh) * p.Lq + qi : -1;
    };
    __syncthreads();  // the previous query tile is no longer read
    stage_rows<kRowsQ>(Qs, p.q, bf16, qrow);
    stage_rows<kRowsQ>(dOs, p.dout, bf16, qrow);
    stage_row_state(p, rs, q0, b, g);
    __syncthreads();
    // Warps 0-3: S and P (into Ps); warps 4-7: dP, then dS = P (dP - D) into dSs.
    const bool s_half = threadIdx.x < kThreads / 2;
    const int rg = (threadIdx.x & 127) >> 3, kg = threadIdx.x & 7;
    float sc[4][4];
    dots_4x4(s_half ? Qs : dOs, s_half ? Ks : Vs, rg, kg, sc);
    const bool need_mask = cls == GQA_TILE_PARTIAL || j0 + kKeys > p.Lk;
    if (s_half) store_probs(p, rs, j0, need_mask, rg, kg, sc, Ps);
    __syncthreads();
    if (!s_half) store_dscores(rs, rg, kg, sc, Ps, dSs);
    __syncthreads();
    // dV += P^T dO (warps 0-3), dK += dS^T Q (warps 4-7): per row, 8 weights (broadcast
    // within the warp) times 8 columns (one contiguous 512-byte row slice per load).
    const float* W = is_dk ? dSs : Ps;
    const float* X = is_dk ? Qs : dOs;
#pragma unroll 2
    for (int r = 0; r < kRowsQ; ++r) {
      const float4 w0 = reinterpret_cast<const float4*>(W + r * kPStride + kbase)[0];
      const float4 w1 = reinterpret_cast<const float4*>(W + r * kPStride + kbase + 4)[0];
      const float4 xa = reinterpret_cast<const float4*>(X + r * kPad + c4)[0];
      const float4 xb = reinterpret_cast<const float4*>(X + r * kPad + 128 + c4)[0];
      const float w8[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
      const float x8[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[i][c] = fmaf(w8[i], x8[c], acc[i][c]);
    }
  }
  void* dst = is_dk ? p.dk : p.dv;
  const float sc = is_dk ? p.scale : 1.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int64_t row = krow(kbase + i);
    if (row < 0) continue;
    st4(dst, row * kHeadDim + c4, bf16, acc[i][0] * sc, acc[i][1] * sc, acc[i][2] * sc, acc[i][3] * sc);
    st4(dst, row * kHeadDim + 128 + c4, bf16, acc[i][4] * sc, acc[i][5] * sc, acc[i][6] * sc, acc[i][7] * sc);
  }
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
  p.Lq = a.Lq;
  p.Lk = a.Lk;
  p.off = a.off;
  p.P0 = a.P0;
  p.B = a.B;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.G = a.Hq / a.Hkv;
  p.br = kBwdRowsQ / p.G;
  p.nq = int((a.Lq + p.br - 1) / p.br);
  p.nk = int((a.Lk + kBwdKeys - 1) / kBwdKeys);
  p.has_seg = a.seg_q != nullptr;
  p.bf16 = a.bf16;
  p.scale = a.scale;
  p.scale_log2 = a.scale * kLog2e;
  const int64_t rows = int64_t(a.B) * a.Hq * a.Lq;
  if (rows > 0) {
    const int64_t blocks = (rows + 7) / 8;
    if (blocks > 0x7fffffff) return GQA_ERR_UNSUPPORTED;
    bwd_rowdot_kernel<<<unsigned(blocks), kThreads, 0, stream>>>(p, rows);
    if (cudaGetLastError() != cudaSuccess) return GQA_ERR_LAUNCH;
  }
  if (cudaFuncSetAttribute(bwd_dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kSmemBytes)) !=
          cudaSuccess ||
      cudaFuncSetAttribute(bwd_dkv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kSmemBytes)) !=
          cudaSuccess)
    return GQA_ERR_LAUNCH;
  const int64_t nq_units = int64_t(p.nq) * p.Hkv * p.B, nk_units = int64_t(p.nk) * p.Hkv * p.B;
  if (nq_units > 0x7fffffff || nk_units > 0x7fffffff) return GQA_ERR_UNSUPPORTED;
  if (nk_units > 0) bwd_dkv_kernel<<<unsigned(nk_units), kThreads, kSmemBytes, stream>>>(p);
  if (cudaGetLastError() != cudaSuccess) return GQA_ERR_LAUNCH;
  if (nq_units > 0) bwd_dq_kernel<<<unsigned(nq_units), kThreads, kSmemBytes, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_LAUNCH;
}

}  // namespace gqa
