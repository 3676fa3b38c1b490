// Host-side interfaces between the translation units of libgqa_attn.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace gqa {

// Geometry of the block-skip plan for one call.
struct PlanShape {
  int64_t Lq, Lk, off, P0;
  int br, bc, nq, nk, has_seg;
};

// Tile sizes per dtype: query rows per CTA tile (positions x heads) and keys per tile.
constexpr int kF32Rows = 64, kF32Bc = 256;
constexpr int kBf16Rows = 128, kBf16Bc = 128;

// Enqueues the per-tile bounds and per-query-tile ranges (segment ids only).
int launch_plan(const PlanShape& s, const int32_t* seg_q, const int32_t* seg_kv, char* ws,
                cudaStream_t stream);
// Enqueues the debug export (ranges + class matrix); launch_plan must precede it.
int launch_plan_export(const PlanShape& s, char* ws, uint8_t* classes, int32_t* kv_ranges,
                       cudaStream_t stream);

// Tensor-map encoder obtained from the driver at run time (no link-time libcuda).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled_fn();

struct FwdTensors {
  const void* q;
  const void* k;
  const void* v;
};

// Backward tile sizes: query rows per query tile (positions x heads), keys per key tile.
constexpr int kBwdRowsQ = 64, kBwdKeys = 128;

struct BwdArgs {
  const void *q, *k, *v, *out;
  const float* lse;
  const void* dout;
  void *dq, *dk, *dv;
  float* D;   // workspace [B * Hq][ldD]: rowsum(dO * O)
  float* L2;  // workspace [B * Hq][ldD]: log2-domain LSE (bf16 path only)
  int64_t ldD;  // row stride of D and L2: Lq (fp32 path) or Lq rounded up to 128 (bf16)
  const int32_t *seg_q, *seg_kv;
  const int32_t *q_bounds, *kv_bounds, *q_ranges;  // plan at the backward's tile sizes, or null
  int32_t* status;
  int64_t Lq, Lk, off, P0, wait_budget_ns;
  int test_skip_fill;  // test hook (see FwdParams); the bf16 kernels only
  int B, Hq, Hkv, bf16;
  float scale;
};

int launch_bwd(const BwdArgs& a, cudaStream_t stream);
// bf16 backward on the tensor cores (plan at (kBf16Rows / G, kBf16Bc) tiles).
int launch_bwd_bf16(const BwdArgs& a, cudaStream_t stream);
int launch_fwd_f32(const FwdTensors& t, const FwdParams& p, cudaStream_t stream);
int launch_fwd_bf16(const FwdTensors& t, const FwdParams& p, cudaStream_t stream);

// Split-operand fp32 path: one fp32 input tensor [heads][L][d] and its hi / lo fp16
// planes ([2][heads][L][d]); amax[heads] must be zero before launch_split_operands.
struct SplitSrc {
  const float* x;
  void* planes;
  int64_t L;
  int heads;
  uint32_t* amax;
};
struct SplitJob {
  SplitSrc src[3];  // q, k, v
};
// Enqueues the per-head max |x| and the hi / lo planes of the three tensors.
int launch_split_operands(const SplitJob& job, cudaStream_t stream);
// The attention kernel on the planes (FwdTensors = hi plane of q, k, v; p.amax set).
int launch_fwd_f32_tc(const FwdTensors& planes, const FwdParams& p, cudaStream_t stream);
int launch_selftest_wait(int32_t* status, int64_t budget_ns, cudaStream_t stream);
// The packed-FMA throughput probe: `ctas` CTAs of 256 threads, `iters` rounds each,
// operand form `form` (0 .. 3).
int launch_probe_ffma2(float* out, int ctas, int iters, int form, cudaStream_t stream);
// GQA_ERR_UNSUPPORTED unless the library was built with GQA_DEBUG_BOUNDS.
int launch_selftest_bounds(int32_t* status, int planted, cudaStream_t stream);
// Combines `splits` key-split partials ([splits][rows][d] fp32 and [splits][rows]) into
// out (fp32 or bf16) and lse ([rows]).
int launch_merge_splits(const float* o_part, const float* lse_part, void* out, float* lse, int64_t rows,
                        int splits, bool bf16, cudaStream_t stream);
// out = merge of (o_a, lse_a) (fp32, or absent) and (o_b, lse_b) (fp32 or bf16, or absent);
// o_out may alias o_a when it is fp32.
int launch_merge_pair(const float* o_a, const float* lse_a, const void* o_b, const float* lse_b, bool b_bf16,
                      void* o_out, float* lse_out, bool out_bf16, int64_t rows, cudaStream_t stream);

}  // namespace gqa
