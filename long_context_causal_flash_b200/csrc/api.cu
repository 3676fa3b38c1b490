// C ABI of libgqa_attn: argument validation, workspace sizing, dispatch by dtype.
// The operation, layouts and error conventions are documented in gqa_attn.h.
#include <cmath>
#include <cstdlib>
#include <cstring>

#include "internal.h"

namespace gqa {

EncodeTiledFn encode_tiled_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

namespace {

constexpr int64_t kDefaultWaitBudgetNs = 2000000000LL;  // 2 s: waits normally end in microseconds

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct Shape {
  int G, br, bc, nq, nk;
};

// Shape checks shared by every entry point.  Returns GQA_OK and fills `s`.
int check_shape(int B, int Hq, int Hkv, int64_t Lq, int64_t Lk, int d, int dtype, int mask_kind,
                int64_t off, int has_seg, Shape* s, bool any_key_count = false) {
  if (B < 1 || Hq < 1 || Hkv < 1 || Lq < 1 || Lk < 1 || off < 0) return GQA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return GQA_ERR_INVALID_ARG;
  // A key block of a sharded sequence may start anywhere before the queries.
  if (!any_key_count && Lk != off + Lq) return GQA_ERR_INVALID_ARG;
  if (off > (int64_t(1) << 40)) return GQA_ERR_INVALID_ARG;
  if (dtype != GQA_F32 && dtype != GQA_BF16 && dtype != GQA_F32_TC) return GQA_ERR_INVALID_ARG;
  if (mask_kind != GQA_MASK_CAUSAL && mask_kind != GQA_MASK_PREFIX_BRANCH) return GQA_ERR_INVALID_ARG;
  if (mask_kind == GQA_MASK_PREFIX_BRANCH && !has_seg) return GQA_ERR_INVALID_ARG;
  if (d != kHeadDim) return GQA_ERR_UNSUPPORTED;
  const int G = Hq / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8 && G != 16) return GQA_ERR_UNSUPPORTED;
  // TMA coordinates are int32 and the head index folds B in.
  if (Lk > (int64_t(1) << 31) - 1 || int64_t(B) * Hq > (int64_t(1) << 31) - 1) return GQA_ERR_UNSUPPORTED;
  const int rows = dtype == GQA_F32 ? kF32Rows : kBf16Rows;
  s->G = G;
  s->br = rows / G;
  s->bc = dtype == GQA_F32 ? kF32Bc : kBf16Bc;
  s->nq = int((Lq + s->br - 1) / s->br);
  s->nk = int((Lk + s->bc - 1) / s->bc);
  return GQA_OK;
}

PlanShape plan_shape(const Shape& s, int64_t Lq, int64_t Lk, int mask_kind, int64_t off, int has_seg) {
  PlanShape ps;
  ps.Lq = Lq;
  ps.Lk = Lk;
  ps.off = off;
  ps.P0 = mask_kind == GQA_MASK_PREFIX_BRANCH ? off : 0;
  ps.br = s.br;
  ps.bc = s.bc;
  ps.nq = s.nq;
  ps.nk = s.nk;
  ps.has_seg = has_seg;
  return ps;
}

// Workspace for key splits: the base layout, then [splits][B*Hq*Lq] fp32 log-sum-exps,
// then [splits][B*Hq*Lq][d] fp32 partial outputs.
struct SplitLayout {
  size_t lse_part = 0, o_part = 0, total = 0;
};

SplitLayout split_layout(const WsLayout& w, int64_t rows, int splits) {
  SplitLayout l;
  l.total = w.total;
  if (splits <= 1) return l;
  l.lse_part = w.total;
  l.o_part = l.lse_part + round_up(size_t(splits) * size_t(rows) * sizeof(float), 256);
  l.total = l.o_part + round_up(size_t(splits) * size_t(rows) * kHeadDim * sizeof(float), 256);
  return l;
}

// Split-operand fp32 path: after `base` bytes, the per-head max |x| words (q heads,
// then k heads, then v heads) and the hi / lo fp16 planes of q, k and v.
struct TcLayout {
  size_t amax = 0, amax_bytes = 0, q = 0, k = 0, v = 0, total = 0;
};

TcLayout tc_layout(size_t base, int B, int Hq, int Hkv, int64_t Lq, int64_t Lk) {
  TcLayout t;
  t.amax = base;
  t.amax_bytes = round_up((size_t(B) * Hq + 2 * size_t(B) * Hkv) * sizeof(uint32_t), 256);
  t.q = t.amax + t.amax_bytes;
  t.k = t.q + round_up(2 * size_t(B) * Hq * size_t(Lq) * kHeadDim * 2, 256);
  const size_t kv = round_up(2 * size_t(B) * Hkv * size_t(Lk) * kHeadDim * 2, 256);
  t.v = t.k + kv;
  t.total = t.v + kv;
  return t;
}

constexpr int kMaxSplits = 16;
constexpr int kB200Sms = 148;

// Test hook: GQA_ATTN_TEST_SKIP_FILL=n makes the key/value producer of every CTA
// skip its fill n (read at every call, so a test can clear it between calls).
int test_skip_fill() {
  if (const char* e = std::getenv("GQA_ATTN_TEST_SKIP_FILL")) {
    const long long v = std::atoll(e);
    if (v >= 0 && v < (1LL << 30)) return int(v);
  }
  return -1;
}

int64_t wait_budget_ns() {
  static int64_t budget = -1;
  if (budget < 0) {
    budget = kDefaultWaitBudgetNs;
    if (const char* e = std::getenv("GQA_ATTN_WAIT_BUDGET_NS")) {
      const long long v = std::atoll(e);
      if (v >= 1000000LL && v <= 10000000000LL) budget = v;
    }
  }
  return budget;
}

}  // namespace
}  // namespace gqa

using namespace gqa;

namespace gqa {
namespace {

// Backward geometry: the plan at the backward's tile sizes (fp32: the FFMA kernels'
// 64-row x 32-key tiles; bf16: the tensor-core kernels' 128 x 128) and the per-row
// D = rowsum(dO * O) (bf16 also the log2-domain LSE, rows padded to a multiple of 128),
// after the status word.
struct BwdLayout {
  PlanShape ps;
  WsLayout w;
  int64_t ldD = 0;
  size_t D = 0, L2 = 0, total = 0;
};

BwdLayout bwd_layout(int B, int Hq, int Hkv, int64_t Lq, int64_t Lk, int dtype, int mask_kind, int64_t off,
                     int has_seg) {
  BwdLayout l;
  const int G = Hq / Hkv;
  const bool bf16 = dtype == GQA_BF16;
  l.ps.Lq = Lq;
  l.ps.Lk = Lk;
  l.ps.off = off;
  l.ps.P0 = mask_kind == GQA_MASK_PREFIX_BRANCH ? off : 0;
  l.ps.br = (bf16 ? kBf16Rows : kBwdRowsQ) / G;
  l.ps.bc = bf16 ? kBf16Bc : kBwdKeys;
  l.ps.nq = int((Lq + l.ps.br - 1) / l.ps.br);
  l.ps.nk = int((Lk + l.ps.bc - 1) / l.ps.bc);
  l.ps.has_seg = has_seg;
  l.w = ws_layout(l.ps.nq, l.ps.nk, has_seg != 0);
  l.ldD = bf16 ? int64_t(round_up(size_t(Lq), 128)) : Lq;
  const size_t plane = round_up(size_t(B) * Hq * size_t(l.ldD) * sizeof(float), 256);
  l.D = l.w.total;
  l.L2 = l.D + plane;
  l.total = l.L2 + (bf16 ? plane : 0);
  return l;
}

}  // namespace
}  // namespace gqa

static int fwd_impl(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Hq, int Hkv,
                    int64_t Lq, int64_t Lk, int d, int dtype, int mask_kind, int64_t q_pos_offset,
                    const int32_t* segment_ids_q, const int32_t* segment_ids_kv, int splits, void* workspace,
                    size_t workspace_bytes, gqa_stream_t stream, bool any_key_count = false) {
  if (splits < 1 || splits > kMaxSplits) return GQA_ERR_INVALID_ARG;
  if (!q || !k || !v || !out || !lse) return GQA_ERR_INVALID_ARG;
  // Key blocks at an arbitrary offset take a 256-byte workspace: no room for planes.
  if (any_key_count && dtype == GQA_F32_TC) return GQA_ERR_UNSUPPORTED;
  if ((segment_ids_q == nullptr) != (segment_ids_kv == nullptr)) return GQA_ERR_INVALID_ARG;
  const int has_seg = segment_ids_q != nullptr;
  Shape s;
  int rc = check_shape(B, Hq, Hkv, Lq, Lk, d, dtype, mask_kind, q_pos_offset, has_seg, &s, any_key_count);
  if (rc != GQA_OK) return rc;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse))
    return GQA_ERR_MISALIGNED;
  const WsLayout w = ws_layout(s.nq, s.nk, has_seg);
  const int64_t rows = int64_t(B) * Hq * Lq;
  const SplitLayout sl = split_layout(w, rows, splits);
  const bool tc = dtype == GQA_F32_TC;
  const TcLayout tl = tc_layout(sl.total, B, Hq, Hkv, Lq, Lk);
  if (!workspace || workspace_bytes < (tc ? tl.total : sl.total)) return GQA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return GQA_ERR_MISALIGNED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  if (cudaMemsetAsync(ws, 0, 256, st) != cudaSuccess) return GQA_ERR_LAUNCH;
  const PlanShape ps = plan_shape(s, Lq, Lk, mask_kind, q_pos_offset, has_seg);
  rc = launch_plan(ps, segment_ids_q, segment_ids_kv, ws, st);
  if (rc != GQA_OK) return rc;

  FwdParams p;
  std::memset(&p, 0, sizeof(p));
  p.q = q;
  p.out = out;
  p.lse = lse;
  p.seg_q = segment_ids_q;
  p.seg_kv = segment_ids_kv;
  p.q_bounds = has_seg ? reinterpret_cast<const int32_t*>(ws + w.q_bounds) : nullptr;
  p.kv_bounds = has_seg ? reinterpret_cast<const int32_t*>(ws + w.kv_bounds) : nullptr;
  p.q_ranges = has_seg ? reinterpret_cast<const int32_t*>(ws + w.q_ranges) : nullptr;
  p.status = reinterpret_cast<int32_t*>(ws);
  p.Lq = Lq;
  p.Lk = Lk;
  p.off = q_pos_offset;
  p.P0 = ps.P0;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = s.G;
  p.br = s.br;
  p.bc = s.bc;
  p.nq = s.nq;
  p.nk = s.nk;
  p.has_seg = has_seg;
  p.scale_log2 = float(1.0 / std::sqrt(double(d)) * 1.4426950408889634);
  p.wait_budget_ns = wait_budget_ns();
  p.test_skip_fill = test_skip_fill();
  p.splits = splits;
  p.o_part = splits > 1 ? reinterpret_cast<float*>(ws + sl.o_part) : nullptr;
  p.lse_part = splits > 1 ? reinterpret_cast<float*>(ws + sl.lse_part) : nullptr;
  if (tc) {
    if (cudaMemsetAsync(ws + tl.amax, 0, tl.amax_bytes, st) != cudaSuccess) return GQA_ERR_LAUNCH;
    uint32_t* amax = reinterpret_cast<uint32_t*>(ws + tl.amax);
    SplitJob job;
    job.src[0] = SplitSrc{static_cast<const float*>(q), ws + tl.q, Lq, B * Hq, amax};
    job.src[1] = SplitSrc{static_cast<const float*>(k), ws + tl.k, Lk, B * Hkv, amax + B * Hq};
    job.src[2] = SplitSrc{static_cast<const float*>(v), ws + tl.v, Lk, B * Hkv, amax + B * Hq + B * Hkv};
    rc = launch_split_operands(job, st);
    if (rc != GQA_OK) return rc;
    p.amax = amax;
    rc = launch_fwd_f32_tc(FwdTensors{ws + tl.q, ws + tl.k, ws + tl.v}, p, st);
  } else {
    const FwdTensors t{q, k, v};
    rc = dtype == GQA_F32 ? launch_fwd_f32(t, p, st) : launch_fwd_bf16(t, p, st);
  }
  if (rc != GQA_OK || splits == 1) return rc;
  return launch_merge_splits(p.o_part, p.lse_part, out, lse, rows, splits, dtype == GQA_BF16, st);
}


extern "C" {

size_t gqa_attn_workspace_bytes(int B, int Hq, int Hkv, int64_t Lq, int64_t Lk, int d, int dtype,
                                int mask_kind, int has_segments) {
  Shape s;
  const int64_t off = Lk - Lq;
  if (check_shape(B, Hq, Hkv, Lq, Lk, d, dtype, mask_kind, off, has_segments != 0, &s) != GQA_OK) return 0;
  const size_t base = ws_layout(s.nq, s.nk, has_segments != 0).total;
  return dtype == GQA_F32_TC ? tc_layout(base, B, Hq, Hkv, Lq, Lk).total : base;
}

size_t gqa_attn_bwd_workspace_bytes(int B, int Hq, int Hkv, int64_t Lq, int64_t Lk, int d, int dtype,
                                    int mask_kind, int has_segments) {
  Shape s;
  const int64_t off = Lk - Lq;
  if (check_shape(B, Hq, Hkv, Lq, Lk, d, dtype, mask_kind, off, has_segments != 0, &s) != GQA_OK) return 0;
  if (dtype == GQA_F32_TC) return 0;
  return bwd_layout(B, Hq, Hkv, Lq, Lk, dtype, mask_kind, off, has_segments != 0).total;
}

static int bwd_impl(const void* q, const void* k, const void* v, const void* out, const float* lse, const void* dout,
                    void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int64_t Lq, int64_t Lk, int d, int dtype,
                    int mask_kind, int64_t q_pos_offset, const int32_t* segment_ids_q,
                    const int32_t* segment_ids_kv, void* workspace, size_t workspace_bytes, gqa_stream_t stream,
                    bool any_key_count) {
  if (!q || !k || !v || !out || !lse || !dout || !dq || !dk || !dv) return GQA_ERR_INVALID_ARG;
  if ((segment_ids_q == nullptr) != (segment_ids_kv == nullptr)) return GQA_ERR_INVALID_ARG;
  const int has_seg = segment_ids_q != nullptr;
  Shape s;
  int rc = check_shape(B, Hq, Hkv, Lq, Lk, d, dtype, mask_kind, q_pos_offset, has_seg, &s, any_key_count);
  if (rc != GQA_OK) return rc;
  if (dtype == GQA_F32_TC) return GQA_ERR_UNSUPPORTED;  // the fp32 backward is dtype GQA_F32
  for (const void* ptr : {q, k, v, out, static_cast<const void*>(lse), dout, static_cast<const void*>(dq),
                          static_cast<const void*>(dk), static_cast<const void*>(dv)})
    if (!aligned16(ptr)) return GQA_ERR_MISALIGNED;
  const BwdLayout l = bwd_layout(B, Hq, Hkv, Lq, Lk, dtype, mask_kind, q_pos_offset, has_seg);
  if (!workspace || workspace_bytes < l.total) return GQA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return GQA_ERR_MISALIGNED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  if (cudaMemsetAsync(ws, 0, 256, st) != cudaSuccess) return GQA_ERR_LAUNCH;
  rc = launch_plan(l.ps, segment_ids_q, segment_ids_kv, ws, st);
  if (rc != GQA_OK) return rc;
  BwdArgs a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.out = out;
  a.lse = lse;
  a.dout = dout;
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  a.D = reinterpret_cast<float*>(ws + l.D);
  a.L2 = dtype == GQA_BF16 ? reinterpret_cast<float*>(ws + l.L2) : nullptr;
  a.ldD = l.ldD;
  a.status = reinterpret_cast<int32_t*>(ws);
  a.wait_budget_ns = wait_budget_ns();
  a.test_skip_fill = test_skip_fill();
  a.seg_q = segment_ids_q;
  a.seg_kv = segment_ids_kv;
  a.q_bounds = has_seg ? reinterpret_cast<const int32_t*>(ws + l.w.q_bounds) : nullptr;
  a.kv_bounds = has_seg ? reinterpret_cast<const int32_t*>(ws + l.w.kv_bounds) : nullptr;
  a.q_ranges = has_seg ? reinterpret_cast<const int32_t*>(ws + l.w.q_ranges) : nullptr;
  a.Lq = Lq;
  a.Lk = Lk;
  a.off = q_pos_offset;
  a.P0 = l.ps.P0;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.bf16 = dtype == GQA_BF16;
  a.scale = float(1.0 / std::sqrt(double(d)));
  return launch_bwd(a, st);
}

int gqa_attn_bwd(const void* q, const void* k, const void* v, const void* out, const float* lse, const void* dout,
                 void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int64_t Lq, int64_t Lk, int d, int dtype,
                 int mask_kind, int64_t q_pos_offset, const int32_t* segment_ids_q, const int32_t* segment_ids_kv,
                 void* workspace, size_t workspace_bytes, gqa_stream_t stream) {
  return bwd_impl(q, k, v, out, lse, dout, dq, dk, dv, B, Hq, Hkv, Lq, Lk, d, dtype, mask_kind, q_pos_offset,
                  segment_ids_q, segment_ids_kv, workspace, workspace_bytes, stream, false);
}

int gqa_attn_bwd_offset(const void* q, const void* k, const void* v, const void* out, const float* lse,
                        const void* dout, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int64_t Lq, int64_t Lk,
                        int d, int dtype, int64_t q_pos_offset, void* workspace, size_t workspace_bytes,
                        gqa_stream_t stream) {
  return bwd_impl(q, k, v, out, lse, dout, dq, dk, dv, B, Hq, Hkv, Lq, Lk, d, dtype, GQA_MASK_CAUSAL, q_pos_offset,
                  nullptr, nullptr, workspace, workspace_bytes, stream, true);
}

int gqa_attn_tile_sizes(int dtype, int Hq, int Hkv, int* br, int* bc) {
  if (!br || !bc) return GQA_ERR_INVALID_ARG;
  Shape s;
  const int rc = check_shape(1, Hq, Hkv, 1, 1, kHeadDim, dtype, GQA_MASK_CAUSAL, 0, 0, &s);
  if (rc != GQA_OK) return rc;
  *br = s.br;
  *bc = s.bc;
  return GQA_OK;
}

int gqa_attn_fwd(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Hq,
                 int Hkv, int64_t Lq, int64_t Lk, int d, int dtype, int mask_kind, int64_t q_pos_offset,
                 const int32_t* segment_ids_q, const int32_t* segment_ids_kv, void* workspace,
                 size_t workspace_bytes, gqa_stream_t stream) {
  return fwd_impl(q, k, v, out, lse, B, Hq, Hkv, Lq, Lk, d, dtype, mask_kind, q_pos_offset, segment_ids_q,
                  segment_ids_kv, 1, workspace, workspace_bytes, stream);
}

int gqa_attn_split_hint(int B, int Hq, int Hkv, int64_t Lq, int64_t Lk, int dtype, int mask_kind,
                        int has_segments) {
  Shape s;
  const int64_t off = Lk - Lq;
  const int rc = check_shape(B, Hq, Hkv, Lq, Lk, kHeadDim, dtype, mask_kind, off, has_segments != 0, &s);
  if (rc != GQA_OK) return rc;
  // Work units (one CTA for fp32, one CTA pair on two SMs for bf16) and how many run
  // at once on a B200; key tiles per unit: the causal range of an average query row.
  const double units = dtype == GQA_F32 ? double(s.nq) * Hkv * B : double((s.nq + 1) / 2) * Hkv * B;
  const double per_wave = dtype == GQA_F32 ? kB200Sms : kB200Sms / 2;
  const double tiles = (double(off) + 0.5 * double(Lq)) / s.bc;
  auto efficiency = [&](int n) {  // busy fraction of the last wave's SMs, whole-wave model
    const double waves = units * n / per_wave;
    return waves / std::ceil(waves);
  };
  // The tensor-core kernels (bf16, and fp32 on split operands) are 10-25x faster per
  // key than the FFMA one, so their fp32 partial writes and the merge weigh more: they
  // split only a clearly under-filled GPU (measured: 8 x 256 branch rows after 30,468
  // tokens run 3 % slower with 4 splits in bf16 and 6 % slower in fp32 on the tensor
  // cores, 14 % faster with 2 on the FFMA kernel).
  const bool ffma = dtype == GQA_F32;
  const double start = ffma ? 0.9 : 0.6, target = ffma ? 0.9 : 0.8;
  int best = 1;
  double best_eff = efficiency(1);
  if (best_eff >= start) return 1;
  for (int n = 2; n <= kMaxSplits && best_eff < target; ++n) {
    if (tiles / n < 4.0) break;  // chunks this short cost more in the merge than they save
    const double e = efficiency(n);
    if (e > best_eff + 0.02) best = n, best_eff = e;
  }
  return best;
}

size_t gqa_attn_split_workspace_bytes(int B, int Hq, int Hkv, int64_t Lq, int64_t Lk, int d, int dtype,
                                      int mask_kind, int has_segments, int splits) {
  Shape s;
  const int64_t off = Lk - Lq;
  if (splits < 1 || splits > kMaxSplits) return 0;
  if (check_shape(B, Hq, Hkv, Lq, Lk, d, dtype, mask_kind, off, has_segments != 0, &s) != GQA_OK) return 0;
  const size_t base = split_layout(ws_layout(s.nq, s.nk, has_segments != 0), int64_t(B) * Hq * Lq, splits).total;
  return dtype == GQA_F32_TC ? tc_layout(base, B, Hq, Hkv, Lq, Lk).total : base;
}

int gqa_attn_fwd_split(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Hq,
                       int Hkv, int64_t Lq, int64_t Lk, int d, int dtype, int mask_kind, int64_t q_pos_offset,
                       const int32_t* segment_ids_q, const int32_t* segment_ids_kv, int splits, void* workspace,
                       size_t workspace_bytes, gqa_stream_t stream) {
  return fwd_impl(q, k, v, out, lse, B, Hq, Hkv, Lq, Lk, d, dtype, mask_kind, q_pos_offset, segment_ids_q,
                  segment_ids_kv, splits, workspace, workspace_bytes, stream);
}

int gqa_attn_fwd_offset(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Hq,
                        int Hkv, int64_t Lq, int64_t Lk, int d, int dtype, int64_t q_pos_offset, void* workspace,
                        size_t workspace_bytes, gqa_stream_t stream) {
  return fwd_impl(q, k, v, out, lse, B, Hq, Hkv, Lq, Lk, d, dtype, GQA_MASK_CAUSAL, q_pos_offset, nullptr, nullptr,
                  1, workspace, workspace_bytes, stream, true);
}

int gqa_attn_merge(const float* o_a, const float* lse_a, const void* o_b, const float* lse_b, void* o_out,
                   float* lse_out, int64_t rows, int d, int dtype_b, int dtype_out, gqa_stream_t stream) {
  if (rows < 1 || !o_out || !lse_out) return GQA_ERR_INVALID_ARG;
  if ((o_a == nullptr) != (lse_a == nullptr) || (o_b == nullptr) != (lse_b == nullptr)) return GQA_ERR_INVALID_ARG;
  if ((dtype_b != GQA_F32 && dtype_b != GQA_BF16) || (dtype_out != GQA_F32 && dtype_out != GQA_BF16))
    return GQA_ERR_INVALID_ARG;
  if (d != kHeadDim) return GQA_ERR_UNSUPPORTED;
  for (const void* ptr : {static_cast<const void*>(o_a), static_cast<const void*>(lse_a), o_b,
                          static_cast<const void*>(lse_b), static_cast<const void*>(o_out),
                          static_cast<const void*>(lse_out)})
    if (!aligned16(ptr)) return GQA_ERR_MISALIGNED;
  return launch_merge_pair(o_a, lse_a, o_b, lse_b, dtype_b == GQA_BF16, o_out, lse_out, dtype_out == GQA_BF16, rows,
                           reinterpret_cast<cudaStream_t>(stream));
}

int gqa_attn_tile_plan(int Hq, int Hkv, int64_t Lq, int64_t Lk, int dtype, int mask_kind,
                       int64_t q_pos_offset, const int32_t* segment_ids_q, const int32_t* segment_ids_kv,
                       void* workspace, size_t workspace_bytes, uint8_t* classes, int32_t* kv_ranges,
                       gqa_stream_t stream) {
  if (!classes || !kv_ranges) return GQA_ERR_INVALID_ARG;
  if ((segment_ids_q == nullptr) != (segment_ids_kv == nullptr)) return GQA_ERR_INVALID_ARG;
  const int has_seg = segment_ids_q != nullptr;
  Shape s;
  int rc = check_shape(1, Hq, Hkv, Lq, Lk, kHeadDim, dtype, mask_kind, q_pos_offset, has_seg, &s);
  if (rc != GQA_OK) return rc;
  const WsLayout w = ws_layout(s.nq, s.nk, has_seg);
  if (!workspace || workspace_bytes < w.total) return GQA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return GQA_ERR_MISALIGNED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  if (cudaMemsetAsync(ws, 0, 256, st) != cudaSuccess) return GQA_ERR_LAUNCH;
  const PlanShape ps = plan_shape(s, Lq, Lk, mask_kind, q_pos_offset, has_seg);
  rc = launch_plan(ps, segment_ids_q, segment_ids_kv, ws, st);
  if (rc != GQA_OK) return rc;
  return launch_plan_export(ps, ws, classes, kv_ranges, st);
}

int gqa_attn_status(const void* workspace, gqa_stream_t stream) {
  if (!workspace) return GQA_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int32_t word = 0;
  if (cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return GQA_ERR_LAUNCH;
  if (cudaStreamSynchronize(st) != cudaSuccess) return GQA_ERR_LAUNCH;
  return word;
}

int gqa_attn_selftest_wait(void* workspace, size_t workspace_bytes, int64_t budget_ns, gqa_stream_t stream) {
  if (!workspace || workspace_bytes < 256) return GQA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return GQA_ERR_MISALIGNED;
  if (budget_ns < 1000000LL || budget_ns > 10000000000LL) return GQA_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(workspace, 0, 256, st) != cudaSuccess) return GQA_ERR_LAUNCH;
  return launch_selftest_wait(static_cast<int32_t*>(workspace), budget_ns, st);
}

int gqa_attn_selftest_bounds(void* workspace, size_t workspace_bytes, int planted, gqa_stream_t stream) {
  if (!workspace || workspace_bytes < 256) return GQA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return GQA_ERR_MISALIGNED;
  if (planted != 0 && planted != 1) return GQA_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
#if defined(GQA_DEBUG_BOUNDS)
  if (cudaMemsetAsync(workspace, 0, 256, st) != cudaSuccess) return GQA_ERR_LAUNCH;
#endif
  return launch_selftest_bounds(static_cast<int32_t*>(workspace), planted, st);
}

int gqa_attn_probe_ffma2(float* out, int ctas, int iters, int form, gqa_stream_t stream) {
  if (!out) return GQA_ERR_INVALID_ARG;
  if (ctas < 1 || ctas > 65535 || iters < 1 || form < 0 || form > 3) return GQA_ERR_INVALID_ARG;
  if (!aligned16(out)) return GQA_ERR_MISALIGNED;
  return launch_probe_ffma2(out, ctas, iters, form, reinterpret_cast<cudaStream_t>(stream));
}

const char* gqa_attn_strerror(int status) {
  switch (status) {
    case GQA_OK: return "ok";
    case GQA_ERR_INVALID_ARG: return "invalid argument";
    case GQA_ERR_UNSUPPORTED: return "unsupported shape (d must be 256, Hq/Hkv in {1,2,4,8,16})";
    case GQA_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case GQA_ERR_WORKSPACE: return "workspace missing or too small";
    case GQA_ERR_LAUNCH: return "CUDA launch or API call failed";
    case GQA_ERR_DEVICE_TIMEOUT: return "a bounded device-side wait ran out";
    case GQA_ERR_DEVICE_BOUNDS: return "a device-side index check failed (checked build)";
    default: return "unknown status";
  }
}

}  // extern "C"
