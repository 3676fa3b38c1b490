// Block-skip plan on the device: per-tile [min, max] segment ids and, per query
// tile, the range of key tiles that hold any visible pair.
//
// The segmented splash kernel of maxtext PR #4929 ("Let splash attention exceed
// 524,288 tokens when packing is off", description) prefetches block-pair tables
// (2,097,152 bytes at 1M tokens) into 1 MiB of scalar memory and fails to build.
// Here the metadata is O(L / tile): two bounds per tile and two range ends per
// query tile, written to the caller's workspace.  The attention kernels classify
// each (query tile, key tile) pair on the fly from these bounds (tile_class in
// common.cuh) and never read a SKIP tile.
#include "internal.h"

namespace gqa {

namespace {

constexpr int kPlanWarps = 8;

// One warp per tile: [min, max] of the ids under it.  Tiles [0, nq) are query
// tiles of `br` rows, tiles [nq, nq + nk) key tiles of `bc` keys.
__global__ void __launch_bounds__(kPlanWarps * 32)
plan_bounds_kernel(const int32_t* __restrict__ seg_q, const int32_t* __restrict__ seg_kv,
                   int64_t Lq, int64_t Lk, int br, int bc, int nq, int nk,
                   int32_t* __restrict__ q_bounds, int32_t* __restrict__ kv_bounds) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t t = int64_t(blockIdx.x) * kPlanWarps + warp;
  if (t >= int64_t(nq) + nk) return;
  const bool is_q = t < nq;
  const int32_t* ids = is_q ? seg_q : seg_kv;
  const int64_t tile = is_q ? t : t - nq;
  const int64_t len = is_q ? Lq : Lk;
  const int size = is_q ? br : bc;
  const int64_t a = tile * size;
  const int64_t e = (a + size < len) ? a + size : len;
  int lo = INT32_MAX, hi = INT32_MIN;
  for (int64_t i = a + lane; i < e; i += 32) {
    const int x = ids[i];
    lo = min(lo, x);
    hi = max(hi, x);
  }
  lo = __reduce_min_sync(0xffffffffu, lo);
  hi = __reduce_max_sync(0xffffffffu, hi);
  if (lane == 0) {
    int32_t* dst = is_q ? q_bounds : kv_bounds;
    dst[2 * tile] = lo;
    dst[2 * tile + 1] = hi;
  }
}

struct PlanArgs {
  int64_t Lq, Lk, off, P0;
  int br, bc, nq, nk, has_seg;
  const int32_t* q_bounds;
  const int32_t* kv_bounds;
};

// One warp per query tile: first and last non-SKIP key tile.  Key tiles past the
// causal end are SKIP unless they hold state keys, and state keys lie below P0 <=
// i1 + off, so the scan stops at the causal end.
__global__ void __launch_bounds__(kPlanWarps * 32)
plan_ranges_kernel(PlanArgs a, int32_t* __restrict__ q_ranges) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = blockIdx.x * kPlanWarps + warp;
  if (qt >= a.nq) return;
  const int64_t i0 = int64_t(qt) * a.br;
  const int64_t i1 = min(a.Lq, i0 + a.br) - 1;
  int first, end;
  kv_range_no_seg(i1, a.off, a.bc, a.nk, &first, &end);
  if (a.has_seg) {
    const SegBounds qb{a.q_bounds[2 * qt], a.q_bounds[2 * qt + 1]};
    int lo = INT32_MAX, hi = -1;
    for (int kt = lane; kt < end; kt += 32) {
      const int64_t j0 = int64_t(kt) * a.bc;
      const int64_t j1 = min(a.Lk, j0 + a.bc) - 1;
      const SegBounds kb{a.kv_bounds[2 * kt], a.kv_bounds[2 * kt + 1]};
      if (tile_class(i0, i1, j0, j1, a.off, a.P0, true, qb, kb) != GQA_TILE_SKIP) {
        lo = min(lo, kt);
        hi = max(hi, kt);
      }
    }
    lo = __reduce_min_sync(0xffffffffu, lo);
    hi = __reduce_max_sync(0xffffffffu, hi);
    if (hi < 0) {
      first = 0;
      end = 0;
    } else {
      first = lo;
      end = hi + 1;
    }
  }
  if (lane == 0) {
    q_ranges[2 * qt] = first;
    q_ranges[2 * qt + 1] = end;
  }
}

// Debug export: the class of every (query tile, key tile) pair.
__global__ void plan_classes_kernel(PlanArgs a, uint8_t* __restrict__ classes) {
  const int64_t idx = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= int64_t(a.nq) * a.nk) return;
  const int qt = int(idx / a.nk), kt = int(idx % a.nk);
  const int64_t i0 = int64_t(qt) * a.br, i1 = min(a.Lq, i0 + a.br) - 1;
  const int64_t j0 = int64_t(kt) * a.bc, j1 = min(a.Lk, j0 + a.bc) - 1;
  SegBounds qb{0, 0}, kb{0, 0};
  if (a.has_seg) {
    qb = {a.q_bounds[2 * qt], a.q_bounds[2 * qt + 1]};
    kb = {a.kv_bounds[2 * kt], a.kv_bounds[2 * kt + 1]};
  }
  classes[idx] = uint8_t(tile_class(i0, i1, j0, j1, a.off, a.P0, a.has_seg != 0, qb, kb));
}

PlanArgs make_args(const PlanShape& s, const WsLayout& w, char* ws) {
  PlanArgs a;
  a.Lq = s.Lq;
  a.Lk = s.Lk;
  a.off = s.off;
  a.P0 = s.P0;
  a.br = s.br;
  a.bc = s.bc;
  a.nq = s.nq;
  a.nk = s.nk;
  a.has_seg = s.has_seg;
  a.q_bounds = s.has_seg ? reinterpret_cast<const int32_t*>(ws + w.q_bounds) : nullptr;
  a.kv_bounds = s.has_seg ? reinterpret_cast<const int32_t*>(ws + w.kv_bounds) : nullptr;
  return a;
}

}  // namespace

int launch_plan(const PlanShape& s, const int32_t* seg_q, const int32_t* seg_kv, char* ws,
                cudaStream_t stream) {
  if (!s.has_seg) return GQA_OK;
  const WsLayout w = ws_layout(s.nq, s.nk, true);
  const int64_t tiles = int64_t(s.nq) + s.nk;
  plan_bounds_kernel<<<unsigned((tiles + kPlanWarps - 1) / kPlanWarps), kPlanWarps * 32, 0, stream>>>(
      seg_q, seg_kv, s.Lq, s.Lk, s.br, s.bc, s.nq, s.nk, reinterpret_cast<int32_t*>(ws + w.q_bounds),
      reinterpret_cast<int32_t*>(ws + w.kv_bounds));
  if (cudaGetLastError() != cudaSuccess) return GQA_ERR_LAUNCH;
  plan_ranges_kernel<<<unsigned((s.nq + kPlanWarps - 1) / kPlanWarps), kPlanWarps * 32, 0, stream>>>(
      make_args(s, w, ws), reinterpret_cast<int32_t*>(ws + w.q_ranges));
  if (cudaGetLastError() != cudaSuccess) return GQA_ERR_LAUNCH;
  return GQA_OK;
}

int launch_plan_export(const PlanShape& s, char* ws, uint8_t* classes, int32_t* kv_ranges,
                       cudaStream_t stream) {
  const WsLayout w = ws_layout(s.nq, s.nk, s.has_seg != 0);
  const PlanArgs a = make_args(s, w, ws);
  plan_ranges_kernel<<<unsigned((s.nq + kPlanWarps - 1) / kPlanWarps), kPlanWarps * 32, 0, stream>>>(
      a, kv_ranges);
  if (cudaGetLastError() != cudaSuccess) return GQA_ERR_LAUNCH;
  const int64_t n = int64_t(s.nq) * s.nk;
  if (n > 0) {
    plan_classes_kernel<<<unsigned((n + 255) / 256), 256, 0, stream>>>(a, classes);
    if (cudaGetLastError() != cudaSuccess) return GQA_ERR_LAUNCH;
  }
  return GQA_OK;
}

}  // namespace gqa
