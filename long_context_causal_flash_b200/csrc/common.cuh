// Device helpers shared by the plan and attention kernels of libgqa_attn:
// mbarrier / TMA wrappers (inline PTX for sm_100a), bounded waits, the
// block-skip tile classes and the workspace layout.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gqa_attn.h"

namespace gqa {

constexpr int kHeadDim = 256;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// ----------------------------------------------------------------------------
// Workspace layout (bytes).  Offset 0 holds the status word that bounded waits
// write on timeout.  With segment ids: [min, max] of every query tile and key
// tile, then [first, last + 1) key-tile range of every query tile.  All O(L/tile).
// ----------------------------------------------------------------------------
struct WsLayout {
  size_t q_bounds = 0, kv_bounds = 0, q_ranges = 0, total = 0;
};

__host__ __device__ inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

__host__ __device__ inline WsLayout ws_layout(int64_t nq, int64_t nk, bool has_seg) {
  WsLayout w;
  size_t off = 256;
  if (has_seg) {
    w.q_bounds = off;
    off += round_up(size_t(nq) * 2 * sizeof(int32_t), 256);
    w.kv_bounds = off;
    off += round_up(size_t(nk) * 2 * sizeof(int32_t), 256);
    w.q_ranges = off;
    off += round_up(size_t(nq) * 2 * sizeof(int32_t), 256);
  }
  w.total = off;
  return w;
}

// ----------------------------------------------------------------------------
// Tile classes.  For query rows [i0, i1] (positions i + off), keys [j0, j1]:
//   causal_skip = j0 > i1 + off          causal_full = j1 <= i0 + off
//   all_state   = j1 < P0                any_state   = j0 < P0
//   seg_skip    = qmax < kmin || kmax < qmin,  seg_full = qmin == qmax == kmin == kmax
//   (without segment ids: seg_skip = false, seg_full = true)
//   SKIP iff !any_state && (causal_skip || seg_skip)
//   FULL iff all_state || (causal_full && seg_full);  PARTIAL otherwise.
// P0 is the shared-state length for the prefix-branch mask, 0 otherwise.  State
// keys are visible to every branch row (each sits at p >= P0), so a tile holding
// one is never skipped.  Bounds only: O(L / tile) metadata, never block pairs.
// ----------------------------------------------------------------------------
struct SegBounds {
  int lo, hi;
};

__host__ __device__ __forceinline__ int tile_class(int64_t i0, int64_t i1, int64_t j0, int64_t j1,
                                                   int64_t off, int64_t P0, bool has_seg,
                                                   SegBounds q, SegBounds k) {
  const bool causal_skip = j0 > i1 + off;
  const bool causal_full = j1 <= i0 + off;
  const bool all_state = j1 < P0;
  const bool any_state = j0 < P0;
  bool seg_skip = false, seg_full = true;
  if (has_seg) {
    seg_skip = (q.hi < k.lo) || (k.hi < q.lo);
    seg_full = (q.lo == q.hi) && (q.hi == k.lo) && (k.lo == k.hi);
  }
  if (!any_state && (causal_skip || seg_skip)) return GQA_TILE_SKIP;
  if (all_state || (causal_full && seg_full)) return GQA_TILE_FULL;
  return GQA_TILE_PARTIAL;
}

// Key-tile range of query tile [i0, i1] without segment ids: every tile up to the
// causal end (the first key tile always holds key 0 <= i1 + off).
__host__ __device__ __forceinline__ void kv_range_no_seg(int64_t i1, int64_t off, int bc, int nk,
                                                         int* first, int* end) {
  int64_t e = (i1 + off) / bc + 1;
  *first = 0;
  *end = int(e < nk ? e : nk);
}

// Key-split s of `splits` of the key-tile range [first, end): consecutive chunks of
// ceil(n / splits) tiles (the last ones may be short or empty).
__host__ __device__ __forceinline__ void split_range(int split, int splits, int* first, int* end) {
  if (splits <= 1) return;
  const int n = *end - *first;
  const int chunk = (n + splits - 1) / splits;
  const int b = *first + split * chunk;
  const int e = b + chunk < *end ? b + chunk : *end;
  *first = b < *end ? b : *end;
  *end = e > *first ? e : *first;
}

// ----------------------------------------------------------------------------
// PTX wrappers (sm_100a).
// ----------------------------------------------------------------------------
#if defined(__CUDACC__)

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Records the first device-side error of a call in the workspace status word.
__device__ __forceinline__ void set_status(int32_t* status, int code) {
  if (status) atomicCAS(reinterpret_cast<int*>(status), 0, code);
}

// Waits for phase `parity` of an mbarrier, giving up after `budget_ns`
// nanoseconds: then records GQA_ERR_DEVICE_TIMEOUT and returns false.  The polling
// loop is always a call.
static __device__ __noinline__ bool mbar_wait_slow(uint32_t bar, uint32_t parity, int64_t budget_ns, int32_t* status) {
  const uint64_t t0 = global_timer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (int64_t(global_timer_ns() - t0) > budget_ns) {
      set_status(status, GQA_ERR_DEVICE_TIMEOUT);
      return false;
    }
  }
}

// Called form (smaller code at each wait; the fp32 kernel is faster with it).
static __device__ __noinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity, int64_t budget_ns,
                                                      int32_t* status) {
  return mbar_try_wait(bar, parity) || mbar_wait_slow(bar, parity, budget_ns, status);
}

// Inline first test (the bf16 kernel's issuers and softmax warps are faster with it).
__device__ __forceinline__ bool mbar_wait_inline(uint32_t bar, uint32_t parity, int64_t budget_ns, int32_t* status) {
  return mbar_try_wait(bar, parity) || mbar_wait_slow(bar, parity, budget_ns, status);
}

// ----------------------------------------------------------------------------
// Checked builds (-DGQA_DEBUG_BOUNDS).  The FFMA kernels route their generic
// shared-memory accesses and global output rows through these checks; a failure
// skips the access and sets a flag kept in the last 16 bytes of the CTA's dynamic
// shared memory (spare in every kernel: their layouts end at least 16 bytes before
// the window's end), which the kernel turns into GQA_ERR_DEVICE_BOUNDS in the status
// word when it ends.  In normal builds every check compiles to nothing.
// ----------------------------------------------------------------------------
#if defined(GQA_DEBUG_BOUNDS)
extern __shared__ __align__(16) char gqa_dyn_smem[];
__device__ __forceinline__ uint32_t dyn_smem_size() {
  uint32_t n;
  asm volatile("mov.u32 %0, %%dynamic_smem_size;" : "=r"(n));
  return n;
}
__device__ __forceinline__ uint32_t debug_flag_addr() { return smem_u32(gqa_dyn_smem) + dyn_smem_size() - 16; }
__device__ __forceinline__ void debug_fail() {
  asm volatile("red.shared.or.b32 [%0], 1;" ::"r"(debug_flag_addr()) : "memory");
}
// Shared access of `bytes` at `addr`: inside the window, below the flag.
__device__ __forceinline__ bool debug_smem_ok(uint32_t addr, uint32_t bytes) {
  const uint32_t lo = smem_u32(gqa_dyn_smem);
  if (addr >= lo && addr + bytes <= debug_flag_addr() && (addr & (bytes - 1)) == 0) return true;
  debug_fail();
  return false;
}
// The same, and the access lies inside the region [lo, lo + n) it belongs to.
__device__ __forceinline__ bool debug_region_ok(uint32_t addr, uint32_t bytes, uint32_t lo, uint32_t n) {
  if (!debug_smem_ok(addr, bytes)) return false;
  if (addr >= lo && addr + bytes <= lo + n) return true;
  debug_fail();
  return false;
}
// Global element index i of a buffer of n elements.
__device__ __forceinline__ bool debug_index_ok(int64_t i, int64_t n) {
  if (i >= 0 && i < n) return true;
  debug_fail();
  return false;
}
// Thread 0 at kernel start (before the first barrier) and at kernel end (after the last).
__device__ __forceinline__ void debug_flag_reset() {
  asm volatile("st.shared.u32 [%0], 0;" ::"r"(debug_flag_addr()) : "memory");
}
__device__ __forceinline__ void debug_flag_report(int32_t* status) {
  uint32_t f;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(f) : "r"(debug_flag_addr()) : "memory");
  if (f) set_status(status, GQA_ERR_DEVICE_BOUNDS);
}
#else
__device__ __forceinline__ bool debug_smem_ok(uint32_t, uint32_t) { return true; }
__device__ __forceinline__ bool debug_region_ok(uint32_t, uint32_t, uint32_t, uint32_t) { return true; }
__device__ __forceinline__ bool debug_index_ok(int64_t, int64_t) { return true; }
__device__ __forceinline__ void debug_flag_reset() {}
__device__ __forceinline__ void debug_flag_report(int32_t*) {}
#endif

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 3-D tiled TMA load global -> shared, completion counted on `bar` in bytes.
// No multicast: every CTA fetches its own tiles.
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// ---- clusters (CTA pairs)

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Address of the same shared-memory offset in CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t out;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(out) : "r"(addr), "r"(rank));
  return out;
}

// Whole-cluster barrier (every thread of every CTA; release / acquire at cluster scope).
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Arrival on an mbarrier of another CTA of the cluster (default semantics, as for a
// local arrival).  What it publishes between the CTA pair is tensor-memory state,
// ordered by tcgen05 fences around the arrival and the wait; a cluster-scope release
// here costs about a thousand cycles per arrival on B200 (measured).
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// 4-D tiled TMA load into this CTA's shared memory whose completion is counted on an
// mbarrier of either CTA of the pair (`bar_cluster` is a shared::cluster address).
// No multicast: each CTA fetches its own half of a pair tile.
__device__ __forceinline__ void tma_load_4d_pair(uint32_t dst, const CUtensorMap* map, uint32_t bar_cluster, int c0,
                                                 int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}

// The 5-D form of tma_load_4d_pair.
__device__ __forceinline__ void tma_load_5d_pair(uint32_t dst, const CUtensorMap* map, uint32_t bar_cluster, int c0,
                                                 int c1, int c2, int c3, int c4) {
  asm volatile(
      "cp.async.bulk.tensor.5d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4)
      : "memory");
}

#endif  // __CUDACC__

// ----------------------------------------------------------------------------
// Kernel parameters shared by both dtypes.
// ----------------------------------------------------------------------------
struct FwdParams {
  const void* q;  // read directly by kernels that stage Q outside shared memory
  void* out;
  float* lse;
  const int32_t* seg_q;
  const int32_t* seg_kv;
  const int32_t* q_bounds;   // [nq][2] or null
  const int32_t* kv_bounds;  // [nk][2] or null
  const int32_t* q_ranges;   // [nq][2] or null
  int32_t* status;
  int64_t Lq, Lk, off, P0;
  int B, Hq, Hkv, G, br, bc, nq, nk;
  int has_seg;
  float scale_log2;  // (1/sqrt(d)) * log2(e)
  int64_t wait_budget_ns;
  // Fault-injection hook for tests (-1: off): the key/value producer of every CTA
  // skips its fill number `test_skip_fill` -- it neither arms the slot's barrier nor
  // copies -- so that the waits on that fill run out of budget and the kernel takes
  // its timeout exit.  Set from GQA_ATTN_TEST_SKIP_FILL by the host.
  int test_skip_fill;
  // Key splits: with splits > 1 the attention kernels write, for key split s, the
  // partial output O_s / l_s (fp32, [splits][B][Hq][Lq][d]) and its log-sum-exp
  // ([splits][B][Hq][Lq]) instead of out and lse; a merge kernel combines them.
  int splits;
  float* o_part;
  float* lse_part;
  // Split-operand fp32 path only: per-head max |x| bit patterns, [B*Hq] for q then
  // [B*Hkv] for k and for v; they fix the power-of-two scale of each head.
  const uint32_t* amax;
};

}  // namespace gqa
