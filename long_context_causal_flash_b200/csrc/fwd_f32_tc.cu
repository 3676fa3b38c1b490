// fp32 attention forward on the tensor cores (tcgen05 / TMEM) by operand splitting,
// sm_100a.
//
// kev PR #202 ("Measurements") evaluates its models in fp32 with TF32 off, and the
// fp32 contraction on the CUDA cores (fwd_f32.cu) runs at the FP32 pipe's ~75 TFLOP/s.
// Here both contractions of the fp32 attention run on the tensor cores instead.
// Every operand x (q, k, v and the probabilities p) is written as
//     x' = x * 2^e  (exact: e is a per-head power of two, max |x'| in [2^14, 2^15)),
//     hi = fp16(x'),  lo = fp16(x' - hi),
// so hi + lo holds x' to about 2^-22 relative (fp16 keeps 11 significant bits, and
// the scaling keeps lo out of fp16's subnormal range for all but negligible
// elements).  A product is then summed as hi*hi + hi*lo + lo*hi in the fp32
// accumulator (the lo*lo term is ~2^-22 of it and dropped): three fp16 MMAs per
// contraction step instead of one FFMA per multiply-add.  The scales come back out
// exactly: S' = S * 2^(eq+ek) is multiplied by 2^-(eq+ek) inside the exponent's
// scale, and 2^-ev joins 1/l in the epilogue.  The probabilities are formed as
// 2^(s - m + 6): the split of a probability whose lo term would be subnormal is off by
// at most 2^-25 (half of fp16's subnormal spacing), which is then 2^-31 of the row's
// largest term (>= 2^6) instead of 2^-25; the factor cancels between O and the row
// sum l.
//
// Two small kernels prepare the operands in the workspace: split_amax_kernel (max |x|
// per head of q, k and v) and split_planes_kernel (hi and lo planes, [term][head][L][d]
// fp16).  The attention kernel below is the CTA-pair kernel of fwd_bf16.cu with
// these changes:
//   * Q tile: hi and lo, 128 KiB per CTA, loaded once.
//   * One 3-slot ring of 32 KiB slots for K and V, filled by a single producer in the
//     order K(0) | K(1) V(0) | K(2) V(1) | ... | V(T-1), each tile's K and V in two
//     chunks: K chunk h = this CTA's 64 keys x d in [128h, 128h+128), V chunk c = keys
//     [64c, 64c+64) x this CTA's 128 columns, both terms in one 5-D TMA copy.  K(t+1)
//     is ahead of V(t) because S(t+1) runs on the tensor cores while the softmax of
//     tile t runs on the CUDA cores; PV(t) follows.  (Q 128 KiB + 3 x 32 KiB fills the
//     227 KiB of shared memory; a K and a V tile of both terms would need 128 KiB.)
//   * S(t) = 48 pair MMAs of M256 N128 K16 (3 terms x 16 steps), O += P V = 24 of
//     M256 N256 K16 (3 terms x 8), kind::f16 with fp16 operands.
//   * P(t) hi and lo overwrite the two halves of their S buffer in TMEM (64 columns
//     each) and are the A operands of the PV MMAs.
//   * out is fp32.
#include "internal.h"
#include "tcgen05.cuh"

#include <cuda_fp16.h>

namespace gqa {

// Exponent e of the power-of-two scale for a head whose max |x| has bit pattern
// `amax_bits`: max |x| * 2^e lies in [2^14, 2^15).  0 for an all-zero, infinite or NaN
// head; clamped to [-60, 60] so that 2^-(eq + ek) stays a normal fp32 number.
__host__ __device__ __forceinline__ int split_exponent(uint32_t amax_bits) {
  const int biased = int((amax_bits >> 23) & 0xffu);
  if (amax_bits == 0u || biased == 255) return 0;
  if (biased == 0) return 60;  // subnormal maximum
  const int e = 15 - (biased - 126);  // max |x| = f * 2^(biased - 126), f in [0.5, 1)
  return e < -60 ? -60 : (e > 60 ? 60 : e);
}

__device__ __forceinline__ float pow2f(int e) { return __int_as_float((127 + e) << 23); }  // |e| <= 126

namespace {

constexpr int kSplitRows = 64;       // rows of one head per block of the split kernels
constexpr int kSplitThreads = 256;

// Tensor y of the job without indexing the parameter array dynamically (which would
// copy it to local memory).
__device__ __forceinline__ SplitSrc pick(const SplitJob& job, unsigned y) {
  return y == 0 ? job.src[0] : (y == 1 ? job.src[1] : job.src[2]);
}

__global__ void __launch_bounds__(kSplitThreads) split_amax_kernel(SplitJob job) {
  const SplitSrc s = pick(job, blockIdx.y);
  const int64_t chunks = (s.L + kSplitRows - 1) / kSplitRows;
  if (int64_t(blockIdx.x) >= chunks * s.heads) return;
  const int head = int(blockIdx.x / chunks);
  const int64_t r0 = int64_t(blockIdx.x % chunks) * kSplitRows;
  const int64_t r1 = min(s.L, r0 + kSplitRows);
  const float4* x = reinterpret_cast<const float4*>(s.x) + (int64_t(head) * s.L + r0) * (kHeadDim / 4);
  const int64_t n4 = (r1 - r0) * (kHeadDim / 4);
  float m = 0.f;
  for (int64_t i = threadIdx.x; i < n4; i += kSplitThreads) {
    const float4 v = __ldg(x + i);
    m = fmaxf(m, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  __shared__ float wm[kSplitThreads / 32];
  if ((threadIdx.x & 31) == 0) wm[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float b = wm[0];
    for (int w = 1; w < kSplitThreads / 32; ++w) b = fmaxf(b, wm[w]);
    atomicMax(s.amax + head, __float_as_uint(b));  // order-preserving for b >= 0
  }
}

__global__ void __launch_bounds__(kSplitThreads) split_planes_kernel(SplitJob job) {
  const SplitSrc s = pick(job, blockIdx.y);
  const int64_t chunks = (s.L + kSplitRows - 1) / kSplitRows;
  if (int64_t(blockIdx.x) >= chunks * s.heads) return;
  const int head = int(blockIdx.x / chunks);
  const int64_t r0 = int64_t(blockIdx.x % chunks) * kSplitRows;
  const int64_t r1 = min(s.L, r0 + kSplitRows);
  const float scale = pow2f(split_exponent(s.amax[head]));
  const int64_t base4 = (int64_t(head) * s.L + r0) * (kHeadDim / 4);
  const float4* x = reinterpret_cast<const float4*>(s.x) + base4;
  uint2* hi = reinterpret_cast<uint2*>(s.planes) + base4;
  uint2* lo = hi + int64_t(s.heads) * s.L * (kHeadDim / 4);
  const int64_t n4 = (r1 - r0) * (kHeadDim / 4);
  for (int64_t i = threadIdx.x; i < n4; i += kSplitThreads) {
    const float4 v = __ldg(x + i);
    const float a[4] = {v.x * scale, v.y * scale, v.z * scale, v.w * scale};
    __half h[4], l[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      h[c] = __float2half_rn(a[c]);
      l[c] = __float2half_rn(a[c] - __half2float(h[c]));
    }
    uint2 wh, wl;
    wh.x = uint32_t(__half_as_ushort(h[0])) | (uint32_t(__half_as_ushort(h[1])) << 16);
    wh.y = uint32_t(__half_as_ushort(h[2])) | (uint32_t(__half_as_ushort(h[3])) << 16);
    wl.x = uint32_t(__half_as_ushort(l[0])) | (uint32_t(__half_as_ushort(l[1])) << 16);
    wl.y = uint32_t(__half_as_ushort(l[2])) | (uint32_t(__half_as_ushort(l[3])) << 16);
    hi[i] = wh;
    lo[i] = wl;
  }
}

}  // namespace

int launch_split_operands(const SplitJob& job, cudaStream_t stream) {
  int64_t blocks = 0;
  for (int t = 0; t < 3; ++t) {
    const int64_t b = (job.src[t].L + kSplitRows - 1) / kSplitRows * job.src[t].heads;
    blocks = b > blocks ? b : blocks;
  }
  if (blocks <= 0) return GQA_OK;
  if (blocks > 0x7fffffff) return GQA_ERR_UNSUPPORTED;
  const dim3 grid(unsigned(blocks), 3, 1);
  split_amax_kernel<<<grid, kSplitThreads, 0, stream>>>(job);
  split_planes_kernel<<<grid, kSplitThreads, 0, stream>>>(job);
  return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_LAUNCH;
}

namespace {

constexpr int kRows = kBf16Rows;  // 128 query rows per CTA
constexpr int kBc = kBf16Bc;      // 128 keys per tile
constexpr int kThreads = 640;     // 20 warps
constexpr int kSlots = 3;
constexpr int kSlotBytes = 32768;          // one K or V chunk of this CTA, both terms
constexpr int kQBlock = kRows * 128;       // 128 rows x 64 d fp16: 16 KiB
constexpr int kQTerm = 4 * kQBlock;        // one term of the Q tile: 64 KiB
constexpr int kQBytes = 2 * kQTerm;        // 128 KiB
constexpr int kChunkBlock = 64 * 128;      // 64 keys x 64 fp16: 8 KiB
constexpr int kChunkTerm = 2 * kChunkBlock;  // one term of a chunk: 16 KiB
constexpr int kOffQ = 0;
constexpr int kOffRing = kOffQ + kQBytes;
constexpr int kOffBar = kOffRing + kSlots * kSlotBytes;
constexpr int kOffRed = kOffBar + 512;               // [part][row] fp32 exchange
constexpr int kSmemBytes = kOffRed + 4 * kRows * 4;  // dynamic smem is 1024-byte aligned
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 0;
constexpr uint32_t kTmemS = 256;  // buffer b at +128 b; P hi / lo at +0 / +64 of it
constexpr uint16_t kPairMask = 0x3;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr float kPBias = 6.0f;             // P = 2^(s - m + 6) <= 2^14 between rescales

static_assert(kBc == 128, "the issue schedule assumes 128-key tiles");
static_assert(2 * kChunkTerm == kSlotBytes, "slot geometry");
static_assert(kRescaleThreshold + kPBias < 16.f, "P must stay below fp16's largest value");

enum {
  kBarQ = 0,                          // both Q tiles landed (bytes of both CTAs)
  kBarFull = 1,                       // + slot: both CTAs' chunks landed
  kBarEmpty = kBarFull + kSlots,      // + slot: MMAs reading it completed (each CTA)
  kBarSFull = kBarEmpty + kSlots,     // + S buffer (each CTA)
  kBarPFull = kBarSFull + 2,          // + S buffer: 32 arrivals, P written in both CTAs
  kBarPVDone = kBarPFull + 2,         // + S buffer (each CTA)
  kBarDrain = kBarPVDone + 2,         // 2 arrivals: both issuers' MMAs completed
  kNumBars = kBarDrain + 1
};
constexpr int kOffTmemSlot = kOffBar + 8 * kNumBars;
static_assert(kOffTmemSlot + 4 <= kOffBar + 512, "barrier area");
static_assert(kSmemBytes <= 232448, "shared memory per block");

// Position of the ring fills of tile t (t-th computed key tile of the pair):
// K(0) | K(1) V(0) | K(2) V(1) | ... | V(T-1), two chunks each.
__device__ __forceinline__ uint32_t seq_k(int t) { return t == 0 ? 0u : uint32_t(4 * t - 2); }
__device__ __forceinline__ uint32_t seq_v(int t, bool last) { return uint32_t(4 * t + (last ? 2 : 4)); }

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

__device__ __forceinline__ int classify(const FwdParams& p, const QTile& q, int kt) {
  if (kt < q.kbeg || kt >= q.kend) return GQA_TILE_SKIP;
  const int64_t j0 = int64_t(kt) * kBc;
  const int64_t j1 = min(p.Lk, j0 + kBc) - 1;
  SegBounds kb{0, 0};
  if (p.has_seg) kb = SegBounds{p.kv_bounds[2 * kt], p.kv_bounds[2 * kt + 1]};
  return tile_class(q.i0, q.i1, j0, j1, p.off, p.P0, p.has_seg != 0, q.qb, kb);
}

__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, int64_t budget, int32_t* status) {
  return __all_sync(0xffffffffu, mbar_wait_inline(bar, parity, budget, status));
}

__device__ __forceinline__ void quad_sync(uint32_t id) { asm volatile("bar.sync %0, 128;" ::"r"(id) : "memory"); }

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

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// hi = fp16 pair of (a, b) (a in the low half), lo = fp16 pair of the remainders.
__device__ __forceinline__ void split_pair(float a, float b, uint32_t& hi, uint32_t& lo) {
  const __half2 h = __floats2half2_rn(a, b);
  const float2 f = __half22float2(h);
  const __half2 l = __floats2half2_rn(a - f.x, b - f.y);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}

__global__ void __launch_bounds__(kThreads, 1)
fwd_f32_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ FwdParams p) {
  extern __shared__ __align__(1024) char smem_raw[];
  const uint32_t sbase = smem_u32(smem_raw);
  const bool misaligned = (sbase & 1023u) != 0;
  const uint32_t sQ = sbase + kOffQ, sRing = sbase + kOffRing;
  const uint32_t bar = sbase + kOffBar;
  auto B = [&](int i) { return bar + 8u * uint32_t(i); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0: the even CTA, which issues the MMAs
  const uint32_t lead_bar = mapa_shared(bar, 0);
  auto LB = [&](int i) { return lead_bar + 8u * uint32_t(i); };

  // Unit: (query-tile pair, kv head, batch[, key split]), ordered kv head by kv head
  // and, within one, longest causal rows first: the pairs resident together share
  // one kv head's operand planes in L2 (as in the bf16 kernel).
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
  int kbeg = 0x7fffffff, kend = 0;
  if (t0.kbeg < t0.kend) kbeg = t0.kbeg, kend = t0.kend;
  if (t1.kbeg < t1.kend) kbeg = min(kbeg, t1.kbeg), kend = max(kend, t1.kend);
  if (kbeg >= kend) kbeg = kend = 0;
  split_range(split, splits, &kbeg, &kend);
  const int64_t q0 = int64_t(2 * qp + int(rank)) * br;
  auto pair_skip = [&](int kt) {
    return p.has_seg && classify(p, t0, kt) == GQA_TILE_SKIP && classify(p, t1, kt) == GQA_TILE_SKIP;
  };
  auto next_tile = [&](int kt) {  // first computed key tile >= kt, or kend
    while (kt < kend && pair_skip(kt)) ++kt;
    return kt;
  };

  if (threadIdx.x == 0) {
    mbar_init(B(kBarQ), 1);
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(B(kBarFull + s), 1);
      mbar_init(B(kBarEmpty + s), 1);
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
  cluster_sync();
  umma::fence_after_sync();
  uint32_t tmem;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(tmem) : "r"(sbase + kOffTmemSlot));

  const int64_t budget = p.wait_budget_ns;
  const bool leader = rank == 0;
  const int kvhead = b * p.Hkv + g;

  if (misaligned) {
    // no role: fall through to the final cluster barrier
  } else if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    // Q once, then the ring in the order of seq_k / seq_v.  Completion is counted on
    // the even CTA's barriers, which its producer arms with both CTAs' bytes.
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      if (leader) mbar_arrive_expect_tx(B(kBarQ), 2 * kQBytes);
      tma_load_5d_pair(sQ, &tmQ, LB(kBarQ), 0, int(q0), b * p.Hq + g * p.G, 0, 0);
      uint32_t u = 0;  // fills issued
      auto fill = [&](const CUtensorMap* map, int key0, int blk0) {
        const int s = int(u % uint32_t(kSlots));
        if (!mbar_wait_inline(B(kBarEmpty + s), ((u / uint32_t(kSlots)) & 1u) ^ 1u, budget, p.status)) return false;
        if (int(u) == p.test_skip_fill) {  // test hook: both CTAs skip this fill
          ++u;
          return true;
        }
        if (leader) mbar_arrive_expect_tx(B(kBarFull + s), 2 * kSlotBytes);
        tma_load_5d_pair(sRing + uint32_t(s * kSlotBytes), map, LB(kBarFull + s), 0, key0, blk0, 0, kvhead);
        ++u;
        return true;
      };
      // K chunk h: this CTA's 64 keys, d blocks 2h, 2h+1.  V chunk c: keys 64c.., this
      // CTA's column blocks 2 rank, 2 rank + 1.
      auto fill_k = [&](int kt) {
        const int key0 = kt * kBc + int(rank) * 64;
        return fill(&tmK, key0, 0) && fill(&tmK, key0, 2);
      };
      auto fill_v = [&](int kt) { return fill(&tmV, kt * kBc, 2 * int(rank)) && fill(&tmV, kt * kBc + 64, 2 * int(rank)); };
      int kt = next_tile(kbeg);
      bool ok = kt >= kend || fill_k(kt);
      while (ok && kt < kend) {
        const int kn = next_tile(kt + 1);
        if (kn < kend) ok = fill_k(kn);
        if (ok) ok = fill_v(kt);
        kt = kn;
      }
      if (leader) {
        mbar_wait_inline(B(kBarQ), 0, budget, p.status);
        for (uint32_t i = u > uint32_t(kSlots) ? u - kSlots : 0u; i < u; ++i)
          mbar_wait_inline(B(kBarFull + int(i % uint32_t(kSlots))), (i / uint32_t(kSlots)) & 1u, budget, p.status);
      }
    }
    __syncwarp();
  } else if (warp == 1 || warp == 2) {
    // ---------------------------------------------------------------- MMA issuers (even CTA)
    if (lane == 0 && leader) {
      const bool is_s = warp == 1;
      constexpr uint32_t id_s = umma::idesc_f16(2 * kRows, kBc, 0, 0);
      constexpr uint32_t id_o = umma::idesc_f16(2 * kRows, 256, 0, 1);
      const uint64_t dq = umma::smem_desc(sQ, 16, 1024);
      bool ok = !is_s || mbar_wait_inline(B(kBarQ), 0, budget, p.status);
      int t = 0;
      for (int kt = next_tile(kbeg); ok && kt < kend; ++t) {
        const int kn = next_tile(kt + 1);
        const int sb = t & 1;
        if (is_s) {
          // S(t) = sum over the two K chunks (d halves) of hi*hi + hi*lo + lo*hi.
          if (t >= 2 && !(ok = mbar_wait_inline(B(kBarPVDone + sb), (uint32_t(t - 2) >> 1) & 1u, budget, p.status)))
            break;
          const uint32_t d = tmem + kTmemS + uint32_t(sb * 128);
          for (int h = 0; h < 2 && ok; ++h) {
            const uint32_t n = seq_k(t) + uint32_t(h);
            const int s = int(n % uint32_t(kSlots));
            if (!(ok = mbar_wait_inline(B(kBarFull + s), (n / uint32_t(kSlots)) & 1u, budget, p.status))) break;
            umma::fence_after_sync();
            const uint64_t dk = umma::smem_desc(sRing + uint32_t(s * kSlotBytes), 16, 1024);
#pragma unroll
            for (int c = 0; c < 2; ++c)
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const uint64_t a_hi = umma::desc_add(dq, uint32_t((2 * h + c) * kQBlock + k * 32));
                const uint64_t a_lo = umma::desc_add(a_hi, kQTerm);
                const uint64_t b_hi = umma::desc_add(dk, uint32_t(c * kChunkBlock + k * 32));
                const uint64_t b_lo = umma::desc_add(b_hi, kChunkTerm);
                umma::mma_ss_2sm(d, a_hi, b_hi, id_s, (h | c | k) != 0 ? 1u : 0u);
                umma::mma_ss_2sm(d, a_hi, b_lo, id_s, 1u);
                umma::mma_ss_2sm(d, a_lo, b_hi, id_s, 1u);
              }
            umma::commit_2sm_mc(B(kBarEmpty + s), kPairMask);
          }
          if (!ok) break;
          umma::commit_2sm_mc(B(kBarSFull + sb), kPairMask);
        } else {
          // O += P(t) V(t): A = P hi / lo in TMEM, the two V chunks (64 keys each).
          if (!(ok = mbar_wait_inline(B(kBarPFull + sb), (uint32_t(t) >> 1) & 1u, budget, p.status))) break;
          const uint32_t a_hi = tmem + kTmemS + uint32_t(sb * 128), a_lo = a_hi + 64u;
          const bool last = kn >= kend;
          for (int c = 0; c < 2 && ok; ++c) {
            const uint32_t n = seq_v(t, last) + uint32_t(c);
            const int s = int(n % uint32_t(kSlots));
            if (!(ok = mbar_wait_inline(B(kBarFull + s), (n / uint32_t(kSlots)) & 1u, budget, p.status))) break;
            umma::fence_after_sync();
            const uint64_t dv = umma::smem_desc(sRing + uint32_t(s * kSlotBytes), kChunkBlock, 1024);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const uint64_t b_hi = umma::desc_add(dv, uint32_t(k * 2048));
              const uint64_t b_lo = umma::desc_add(b_hi, kChunkTerm);
              const uint32_t ac = uint32_t((4 * c + k) * 8);  // 16 keys = 8 columns of fp16 pairs
              umma::mma_ts_2sm(tmem + kTmemO, a_hi + ac, b_hi, id_o, (t > 0 || c > 0 || k > 0) ? 1u : 0u);
              umma::mma_ts_2sm(tmem + kTmemO, a_hi + ac, b_lo, id_o, 1u);
              umma::mma_ts_2sm(tmem + kTmemO, a_lo + ac, b_hi, id_o, 1u);
            }
            umma::commit_2sm_mc(B(kBarEmpty + s), kPairMask);
          }
          if (!ok) break;
          umma::commit_2sm_mc(B(kBarPVDone + sb), kPairMask);
        }
        kt = kn;
      }
      umma::commit_2sm(B(kBarDrain));
      mbar_wait_inline(B(kBarDrain), 0, budget, p.status);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ---------------------------------------------------------------- softmax warps
    // As in the bf16 kernel: four warps per TMEM lane quarter, part q of them takes S
    // columns 32q .. 32q+31 and O columns 64q .. 64q+63; P hi goes to columns 16q ..
    // 16q+15 of the S buffer and P lo to 64 + 16q .., both after the quarter's counting
    // barrier (every part has loaded S by then).
    const int quarter = warp & 3;
    const int part = (warp - 4) >> 2;
    const int r = quarter * 32 + lane;
    const uint32_t lane_addr = tmem + (uint32_t(quarter * 32) << 16);
    const uint32_t quad_bar = 1u + uint32_t(quarter);
    float* red = reinterpret_cast<float*>(smem_raw + kOffRed);
    const int hh = r / br, pp = r % br;
    const int64_t qi = q0 + pp;
    const bool live = qi < p.Lq;
    const int head = b * p.Hq + g * p.G + hh;
    const int64_t pos = min(qi + p.off, p.Lk - 1);
    const int sq = p.has_seg ? p.seg_q[min(qi, p.Lq - 1)] : 0;
    // Scales of the split operands: S' = S * 2^(eq + ek), V' = V * 2^ev.
    const int nqh = p.B * p.Hq, nkh = p.B * p.Hkv;
    const int eq = split_exponent(p.amax[head]);
    const int ek = split_exponent(p.amax[nqh + kvhead]);
    const int ev = split_exponent(p.amax[nqh + nkh + kvhead]);
    const float sl2 = p.scale_log2 * pow2f(-(eq + ek));

    float m_ref = -INFINITY;
    float l = 0.f;
    int t = 0;
    bool ok = true;
    for (int kt = kbeg; kt < kend; ++kt) {
      if (pair_skip(kt)) continue;
      const int cls = classify(p, own, kt);
      const int sb = t & 1;
      float x[32];
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
      const float pm = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * sl2;
      uint32_t ph[16], pl[16];
      float rs;
      auto exps = [&](float m) {
        const float nb = (m == -INFINITY ? 0.f : -m) + kPBias;
        float r4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const float e0 = ex2_approx(fmaf(x[i], sl2, nb));
          const float e1 = ex2_approx(fmaf(x[i + 1], sl2, nb));
          split_pair(e0, e1, ph[i / 2], pl[i / 2]);
          r4[(i / 2) & 3] += e0 + e1;
        }
        rs = (r4[0] + r4[1]) + (r4[2] + r4[3]);
      };
      exps(m_ref);
      const bool raise_here = pm > m_ref + kRescaleThreshold;
      float alpha = 1.f;
      const float m_old = m_ref;
      if (quad_popc(quad_bar, !ok_s || raise_here) != 0) {
        red[part * kRows + r] = pm;
        if (!quad_and(quad_bar, ok_s)) {
          ok = false;
          break;
        }
        const float mx = fmaxf(fmaxf(red[r], red[kRows + r]), fmaxf(red[2 * kRows + r], red[3 * kRows + r]));
        if (mx > m_ref + kRescaleThreshold) {
          alpha = ex2_approx(m_ref - mx);
          m_ref = mx;
          exps(m_ref);
        }
      }
      l = l * alpha + rs;

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
        umma::tmem_st16u(lane_addr + kTmemS + uint32_t(sb * 128 + part * 16), ph);
        umma::tmem_st16u(lane_addr + kTmemS + uint32_t(sb * 128 + 64 + part * 16), pl);
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
    if (quad_and(quad_bar, ok)) {
      red[part * kRows + r] = l;
      quad_sync(quad_bar);
      l = (red[r] + red[kRows + r]) + (red[2 * kRows + r] + red[3 * kRows + r]);
      const int64_t row = int64_t(head) * p.Lq + (live ? qi : 0);
      const int64_t plane = int64_t(p.B) * p.Hq * p.Lq;
      float* dst_base = splits > 1 ? p.o_part + split * plane * kHeadDim : static_cast<float*>(p.out);
      float4* dst = reinterpret_cast<float4*>(dst_base + row * kHeadDim);
      float* lse_out = splits > 1 ? p.lse_part + split * plane : p.lse;
      // O' / l' = (O / l) * 2^ev: the 2^6 of P cancels, the V scale is undone here.
      const float inv = l > 0.f ? pow2f(-ev) / l : 0.f;
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
          if (live) {
#pragma unroll
            for (int v4 = 0; v4 < 8; ++v4)
              dst[c0 / 4 + v4] =
                  make_float4(o[4 * v4] * inv, o[4 * v4 + 1] * inv, o[4 * v4 + 2] * inv, o[4 * v4 + 3] * inv);
          }
        }
        if (live && part == 0)
          lse_out[int64_t(head) * p.Lq + qi] = l > 0.f ? (m_ref + log2f(l) - kPBias) * kLn2 : -INFINITY;
      }
    }
  }

  umma::fence_before_sync();
  cluster_sync();
  if (warp == 1) {
    umma::fence_after_sync();
    umma::tmem_dealloc_2sm(tmem, kTmemCols);
  }
}

}  // namespace

int launch_fwd_f32_tc(const FwdTensors& planes, const FwdParams& p, cudaStream_t stream) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return GQA_ERR_LAUNCH;
  CUtensorMap mq, mk, mv;
  // Planes [term][head][L][d] fp16.  5-D views whose innermost dimension is one
  // 64-column (128-byte) block of d; the block dimension has a 128-byte stride.
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  const cuuint64_t row = cuuint64_t(kHeadDim) * 2;
  {
    // (d in block, position, head, block, term): box = 128 rows (G heads x br
    // positions) x 4 blocks x 2 terms
    const cuuint64_t heads = cuuint64_t(p.B) * p.Hq;
    const cuuint64_t dims[5] = {64, cuuint64_t(p.Lq), heads, 4, 2};
    const cuuint64_t strides[4] = {row, cuuint64_t(p.Lq) * row, 128, heads * cuuint64_t(p.Lq) * row};
    const cuuint32_t box[5] = {64, cuuint32_t(p.br), cuuint32_t(p.G), 4, 2};
    if (enc(&mq, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 5, const_cast<void*>(planes.q), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return GQA_ERR_LAUNCH;
  }
  // (d in block, key, block, term, kv head): box = 64 keys x 2 blocks x 2 terms
  const cuuint64_t kvheads = cuuint64_t(p.B) * p.Hkv;
  const cuuint64_t dims[5] = {64, cuuint64_t(p.Lk), 4, 2, kvheads};
  const cuuint64_t strides[4] = {row, 128, kvheads * cuuint64_t(p.Lk) * row, cuuint64_t(p.Lk) * row};
  const cuuint32_t box[5] = {64, 64, 2, 2, 1};
  if (enc(&mk, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 5, const_cast<void*>(planes.k), dims, strides, box, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return GQA_ERR_LAUNCH;
  if (enc(&mv, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 5, const_cast<void*>(planes.v), dims, strides, box, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return GQA_ERR_LAUNCH;
  if (cudaFuncSetAttribute(fwd_f32_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) !=
      cudaSuccess)
    return GQA_ERR_LAUNCH;
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
  if (cudaLaunchKernelEx(&cfg, fwd_f32_tc_kernel, mq, mk, mv, p) != cudaSuccess) return GQA_ERR_LAUNCH;
  return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_LAUNCH;
}

}  // namespace gqa
