// Measurement aid: the throughput ceiling of the packed fp32 FMA in the operand form
// the FFMA attention kernels issue, (s[r], s[r+1]) += (q[r], q[r+1]) * (k, k), in the
// two orders of a run of such FMAs (sharing the key value or the row pair).
//
// The attention kernels report their fraction of the FP32 pipe against the nominal
// peak (128 FMA lanes per SM x 2 flop x clock).  A loop of these packed FMAs alone,
// with every operand in registers and no shared-memory or global traffic, does not
// reach that nominal rate on a B200; timing it in the same run gives the attainable
// ceiling of the instruction form itself, the second denominator the bench reports.
#include "internal.h"

namespace gqa {
namespace {

constexpr int kProbeThreads = 256;

// c0, c1 += a0 * b0, a1 * b1 (fma.rn.f32x2), the same form as the attention kernels'.
__device__ __forceinline__ void probe_ffma2(float& c0, float& c1, float a0, float a1, float b0, float b1) {
  asm("{\n\t.reg .b64 ra, rb, rc;\n\t"
      "mov.b64 ra, {%2, %3};\n\t"
      "mov.b64 rb, {%4, %5};\n\t"
      "mov.b64 rc, {%0, %1};\n\t"
      "fma.rn.f32x2 rc, ra, rb, rc;\n\t"
      "mov.b64 {%0, %1}, rc;\n\t}"
      : "+f"(c0), "+f"(c1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// Each thread: 8 rows x 8 keys of accumulators, `iters` rounds of 64 FMAs, then one
// float (the sum of its accumulators) to out[global thread index].  FORM picks the
// operand form and the order of a round:
//   0  32 x (s_r, s_r+1) += (q_r, q_r+1) * (k_m, k_m), key outermost: runs of four
//      packed FMAs share the duplicated key value
//   1  the same FMAs, row pair outermost: runs of eight share the (q_r, q_r+1) pair
//      (the order the attention kernels use for most of their packed FMAs)
//   2  32 x (s_r,m, s_r+1,m+1) += (q_r, q_r+1) * (k_m, k_m+1), and the crossed pair
//      with (k_m+1, k_m): no duplicated operand
//   3  64 x scalar fma.rn.f32
template <int FORM>
__global__ void __launch_bounds__(kProbeThreads, 1) ffma2_probe_kernel(float* out, int iters) {
  float s[8][8], q[8], k[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    q[i] = 1e-3f * float((threadIdx.x + i) % 17);
    k[i] = 1e-3f * float((threadIdx.x + 3 * i) % 13);
#pragma unroll
    for (int j = 0; j < 8; ++j) s[i][j] = 0.f;
  }
  for (int it = 0; it < iters; ++it) {
    if (FORM == 0) {
#pragma unroll
      for (int m = 0; m < 8; ++m)
#pragma unroll
        for (int r = 0; r < 8; r += 2) probe_ffma2(s[r][m], s[r + 1][m], q[r], q[r + 1], k[m], k[m]);
    } else if (FORM == 1) {
#pragma unroll
      for (int r = 0; r < 8; r += 2)
#pragma unroll
        for (int m = 0; m < 8; ++m) probe_ffma2(s[r][m], s[r + 1][m], q[r], q[r + 1], k[m], k[m]);
    } else if (FORM == 2) {
#pragma unroll
      for (int r = 0; r < 8; r += 2)
#pragma unroll
        for (int m = 0; m < 8; m += 2) {
          probe_ffma2(s[r][m], s[r + 1][m + 1], q[r], q[r + 1], k[m], k[m + 1]);
          probe_ffma2(s[r][m + 1], s[r + 1][m], q[r], q[r + 1], k[m + 1], k[m]);
        }
    } else {
#pragma unroll
      for (int m = 0; m < 8; ++m)
#pragma unroll
        for (int r = 0; r < 8; ++r) s[r][m] = fmaf(q[r], k[m], s[r][m]);
    }
  }
  float acc = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc += s[i][j];
  out[int64_t(blockIdx.x) * kProbeThreads + threadIdx.x] = acc;
}

}  // namespace

int launch_probe_ffma2(float* out, int ctas, int iters, int form, cudaStream_t stream) {
  switch (form) {
    case 0: ffma2_probe_kernel<0><<<unsigned(ctas), kProbeThreads, 0, stream>>>(out, iters); break;
    case 1: ffma2_probe_kernel<1><<<unsigned(ctas), kProbeThreads, 0, stream>>>(out, iters); break;
    case 2: ffma2_probe_kernel<2><<<unsigned(ctas), kProbeThreads, 0, stream>>>(out, iters); break;
    case 3: ffma2_probe_kernel<3><<<unsigned(ctas), kProbeThreads, 0, stream>>>(out, iters); break;
    default: return GQA_ERR_INVALID_ARG;
  }
  return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_LAUNCH;
}

}  // namespace gqa
