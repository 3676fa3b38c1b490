// Merges of partial attention results by their log-sum-exp, sm_100a: key splits of
// one call (split-KV) and the blocks of a context-parallel ring.
//
// With few query rows against a long key range (the branch rows after a shared state
// of system1-omni issue #27, item 3), query tiles alone leave most SMs idle, so the
// key range of each query tile is cut into `splits` chunks processed by separate
// CTAs.  Split s leaves its normalised partial output O_s = sum_j p_j v_j / l_s and
// its log-sum-exp lse_s = m_s + ln l_s.  The exact result is
//     lse = ln sum_s exp(lse_s),    out = sum_s exp(lse_s - lse) O_s,
// the same online-softmax identity that combines key tiles inside one CTA.  One warp
// per (batch, head, row); each lane owns 8 consecutive columns of d = 256.
#include <cuda_bf16.h>

#include "internal.h"

namespace gqa {
namespace {

template <bool kBf16>
__global__ void __launch_bounds__(256) merge_splits_kernel(const float* __restrict__ o_part,
                                                           const float* __restrict__ lse_part, void* out,
                                                           float* lse, int64_t rows, int splits) {
  const int64_t row = int64_t(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int lane = threadIdx.x & 31;
  float m = -INFINITY;
  for (int s = 0; s < splits; ++s) m = fmaxf(m, lse_part[s * rows + row]);
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  float wsum = 0.f;
  if (m != -INFINITY) {
    for (int s = 0; s < splits; ++s) {
      const float w = expf(lse_part[s * rows + row] - m);  // 0 for an empty split (lse_s = -inf)
      if (w == 0.f) continue;
      wsum += w;
      const float4* src = reinterpret_cast<const float4*>(o_part + (s * rows + row) * kHeadDim) + 2 * lane;
      const float4 a = src[0], b = src[1];
      acc[0] = fmaf(w, a.x, acc[0]);
      acc[1] = fmaf(w, a.y, acc[1]);
      acc[2] = fmaf(w, a.z, acc[2]);
      acc[3] = fmaf(w, a.w, acc[3]);
      acc[4] = fmaf(w, b.x, acc[4]);
      acc[5] = fmaf(w, b.y, acc[5]);
      acc[6] = fmaf(w, b.z, acc[6]);
      acc[7] = fmaf(w, b.w, acc[7]);
    }
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;  // a row with no visible key: out = 0
  if (kBf16) {
    __nv_bfloat162 h[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(acc[2 * i] * inv, acc[2 * i + 1] * inv);
    reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(out) + row * kHeadDim)[lane] =
        *reinterpret_cast<const uint4*>(h);
  } else {
    float4* dst = reinterpret_cast<float4*>(static_cast<float*>(out) + row * kHeadDim) + 2 * lane;
    dst[0] = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
    dst[1] = make_float4(acc[4] * inv, acc[5] * inv, acc[6] * inv, acc[7] * inv);
  }
  if (lane == 0) lse[row] = wsum > 0.f ? m + logf(wsum) : -INFINITY;
}

// Two partial results over disjoint key sets (the blocks of a context-parallel ring
// step), either of which may be absent (null: no visible key, lse = -inf):
//     lse = ln(exp(lse_a) + exp(lse_b)),   out = exp(lse_a - lse) o_a + exp(lse_b - lse) o_b.
// o_a is fp32; o_b and out are fp32 or bf16; out may be o_a itself (each lane reads
// its 8 columns before writing them, and the warp has read lse_a before lane 0
// overwrites it).  One warp per row.
template <bool kBBf16, bool kOutBf16>
__global__ void __launch_bounds__(256) merge_pair_kernel(const float* o_a, const float* lse_a, const void* o_b,
                                                         const float* lse_b, void* o_out, float* lse_out,
                                                         int64_t rows) {
  const int64_t row = int64_t(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int lane = threadIdx.x & 31;
  const float la = o_a ? lse_a[row] : -INFINITY;
  const float lb = o_b ? lse_b[row] : -INFINITY;
  const float m = fmaxf(la, lb);
  float wa = 0.f, wb = 0.f;
  if (m != -INFINITY) {
    wa = la == -INFINITY ? 0.f : expf(la - m);
    wb = lb == -INFINITY ? 0.f : expf(lb - m);
  }
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  if (wa > 0.f) {
    const float4* src = reinterpret_cast<const float4*>(o_a + row * kHeadDim) + 2 * lane;
    const float4 x = src[0], y = src[1];
    const float a8[8] = {x.x, x.y, x.z, x.w, y.x, y.y, y.z, y.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = wa * a8[i];
  }
  if (wb > 0.f) {
    float b8[8];
    if (kBBf16) {
      const uint4 u = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(o_b) + row * kHeadDim)[lane];
      const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(h[i]);
        b8[2 * i] = f.x;
        b8[2 * i + 1] = f.y;
      }
    } else {
      const float4* src = reinterpret_cast<const float4*>(static_cast<const float*>(o_b) + row * kHeadDim) + 2 * lane;
      const float4 x = src[0], y = src[1];
      b8[0] = x.x, b8[1] = x.y, b8[2] = x.z, b8[3] = x.w, b8[4] = y.x, b8[5] = y.y, b8[6] = y.z, b8[7] = y.w;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = fmaf(wb, b8[i], acc[i]);
  }
  const float wsum = wa + wb;
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;  // no visible key on either side: out = 0
  if (kOutBf16) {
    __nv_bfloat162 h[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(acc[2 * i] * inv, acc[2 * i + 1] * inv);
    reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(o_out) + row * kHeadDim)[lane] =
        *reinterpret_cast<const uint4*>(h);
  } else {
    float4* dst = reinterpret_cast<float4*>(static_cast<float*>(o_out) + row * kHeadDim) + 2 * lane;
    dst[0] = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
    dst[1] = make_float4(acc[4] * inv, acc[5] * inv, acc[6] * inv, acc[7] * inv);
  }
  __syncwarp();
  if (lane == 0) lse_out[row] = wsum > 0.f ? m + logf(wsum) : -INFINITY;
}

}  // namespace

int launch_merge_pair(const float* o_a, const float* lse_a, const void* o_b, const float* lse_b, bool b_bf16,
                      void* o_out, float* lse_out, bool out_bf16, int64_t rows, cudaStream_t stream) {
  if (rows <= 0) return GQA_OK;
  const int64_t blocks = (rows + 7) / 8;
  if (blocks > 0x7fffffff) return GQA_ERR_UNSUPPORTED;
  const unsigned g = unsigned(blocks);
  if (b_bf16 && out_bf16)
    merge_pair_kernel<true, true><<<g, 256, 0, stream>>>(o_a, lse_a, o_b, lse_b, o_out, lse_out, rows);
  else if (b_bf16)
    merge_pair_kernel<true, false><<<g, 256, 0, stream>>>(o_a, lse_a, o_b, lse_b, o_out, lse_out, rows);
  else if (out_bf16)
    merge_pair_kernel<false, true><<<g, 256, 0, stream>>>(o_a, lse_a, o_b, lse_b, o_out, lse_out, rows);
  else
    merge_pair_kernel<false, false><<<g, 256, 0, stream>>>(o_a, lse_a, o_b, lse_b, o_out, lse_out, rows);
  return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_LAUNCH;
}

int launch_merge_splits(const float* o_part, const float* lse_part, void* out, float* lse, int64_t rows,
                        int splits, bool bf16, cudaStream_t stream) {
  if (rows <= 0) return GQA_OK;
  const int64_t blocks = (rows + 7) / 8;
  if (blocks > 0x7fffffff) return GQA_ERR_UNSUPPORTED;
  if (bf16)
    merge_splits_kernel<true><<<unsigned(blocks), 256, 0, stream>>>(o_part, lse_part, out, lse, rows, splits);
  else
    merge_splits_kernel<false><<<unsigned(blocks), 256, 0, stream>>>(o_part, lse_part, out, lse, rows, splits);
  return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_LAUNCH;
}

}  // namespace gqa
