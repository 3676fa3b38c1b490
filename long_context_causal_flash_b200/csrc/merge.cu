// Merge of key-split partial results (split-KV), sm_100a.
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

}  // namespace

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
