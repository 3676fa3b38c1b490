/*
 * gqa_attn.h -- C ABI of libgqa_attn.so: exact causal grouped-query attention
 * forward for NVIDIA B200 (sm_100a).
 *
 *   out[b,h,i,:] = sum_j softmax_j( scale * <q[b,h,i,:], k[b,g,j,:]> + mask(i,j) ) * v[b,g,j,:]
 *   lse[b,h,i]   = ln sum_{visible j} exp( scale * <q[b,h,i,:], k[b,g,j,:]> )
 *
 * with g = h / (Hq / Hkv) and scale = 1/sqrt(d).
 *
 * Sources.  The operation is the attention that PyTorch's SDPA computes for a
 * grouped-query model: 16 query heads sharing 4 key/value heads (kev PR #202,
 * "Why fp32 fell to the L x L kernel"), head_dim 256 (system1-omni issue #27,
 * "The closest planned or implemented model").  The library computes it in memory
 * linear in L: the 16 x L x L score matrix that the L x L "math" kernel
 * materialises (69 GB at 32k, 275 GB at 64k per layer, same section) is never
 * formed, and keys/values are never repeated per query head (the 1 GiB per
 * tensor at 64k of kev PR #202, "The change").  Masks: causal; a shared state
 * followed by per-question branches (system1-omni issue #27, item 3: state once,
 * then one branch per question); and segment ids for block-causal packing
 * (maxtext PR #4929, description).  Like the model-agnostic kernel library of
 * system1-omni issue #27 ("The closest planned or implemented model"), this ABI
 * knows no model; unlike the attention entry point named there, it takes a mask.
 *
 * Conventions shared by every entry point
 * --------------------------------------
 * - Layouts are dense and contiguous, batch-major then head-major (SDPA's
 *   [B, H, L, d]):  q, out: [B, Hq, Lq, d];  k, v: [B, Hkv, Lk, d];
 *   lse: [B, Hq, Lq] fp32.  Element type of q, k, v and out is given by dtype
 *   (GQA_F32 = float, GQA_BF16 = bfloat16 stored as uint16, round-to-nearest-even
 *   on output).  Segment ids are int32 arrays of length Lq and Lk, shared by all
 *   batch entries and heads.
 * - Query row i sits at absolute position p = i + q_pos_offset and sees keys
 *   j <= p (so Lk must equal q_pos_offset + Lq).  With segment ids it also needs
 *   segment_ids_q[i] == segment_ids_kv[j].  With GQA_MASK_PREFIX_BRANCH the first
 *   q_pos_offset keys (the shared state) are visible to every query row whatever
 *   their ids; the remaining keys follow the segment (branch) rule.
 * - A query row with no visible key gets out = 0 and lse = -inf.
 * - Pointers named "device" must point to device memory of the current CUDA
 *   device (or be managed memory).  The caller owns every buffer and the stream;
 *   the library allocates, frees and synchronises nothing, except where an entry
 *   point says so.  Work is enqueued on `stream` (NULL = legacy default stream)
 *   and runs asynchronously; the return value reports host-side validation and
 *   launch errors only.  Errors detected on the device (a bounded wait that ran
 *   out) are recorded in the workspace and read with gqa_attn_status().
 * - Every entry point returns a gqa_status_t (0 on success, negative on error)
 *   unless stated otherwise, and leaves outputs untouched on a validation error.
 */
#ifndef GQA_ATTN_H_
#define GQA_ATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* The caller's cudaStream_t, passed through untouched. */
typedef struct CUstream_st *gqa_stream_t;

/*
 * Element types.  GQA_F32 and GQA_F32_TC both take and return fp32 (float)
 * tensors; they differ in how the two contractions run:
 *   GQA_F32     fp32 FFMA on the CUDA cores.
 *   GQA_F32_TC  the tensor cores (tcgen05, kind::f16) on a two-term fp16 split
 *               of every operand, x = hi + lo with hi = fp16(x'), lo = fp16(x' - hi)
 *               after an exact per-head power-of-two scaling x' = x * 2^e that puts
 *               max |x'| in [2^14, 2^15); each product is summed as
 *               hi*hi + hi*lo + lo*hi in fp32, so an element keeps about 22
 *               significant bits and a product about 21.  The scaled split
 *               operands live in the workspace (4 bytes per element of q, k and v).
 *               Forward entry points gqa_attn_fwd and gqa_attn_fwd_split only.
 *               The scale exponent is clamped to [-60, 60]: a head whose max |x| is
 *               2^75 or more (q and k that large overflow fp32 scores on any path; v
 *               is the case that matters) overflows fp16 -- use GQA_F32 there.
 * kev PR #202 ("Measurements") loads its models in fp32 with TF32 off: GQA_F32_TC
 * uses no TF32; its split operands carry twice TF32's 11 significant bits.
 */
typedef enum { GQA_F32 = 0, GQA_BF16 = 1, GQA_F32_TC = 2 } gqa_dtype_t;

typedef enum { GQA_MASK_CAUSAL = 0, GQA_MASK_PREFIX_BRANCH = 1 } gqa_mask_t;

typedef enum {
  GQA_OK = 0,
  GQA_ERR_INVALID_ARG = -1,    /* bad shape, null pointer, Lk != q_pos_offset + Lq, ... */
  GQA_ERR_UNSUPPORTED = -2,    /* d != 256, or Hq / Hkv not in {1, 2, 4, 8, 16}        */
  GQA_ERR_MISALIGNED = -3,     /* q/k/v/out/lse/workspace not 16-byte aligned            */
  GQA_ERR_WORKSPACE = -4,      /* workspace null or smaller than gqa_attn_workspace_bytes */
  GQA_ERR_LAUNCH = -5,         /* a CUDA launch or API call failed                       */
  GQA_ERR_DEVICE_TIMEOUT = -6, /* a bounded device-side wait ran out (see gqa_attn_status) */
  GQA_ERR_DEVICE_BOUNDS = -7   /* checked builds only: a shared- or global-memory index
                                  fell outside its buffer (the access was skipped)      */
} gqa_status_t;

/* Tile classes reported by gqa_attn_tile_plan. */
typedef enum { GQA_TILE_SKIP = 0, GQA_TILE_PARTIAL = 1, GQA_TILE_FULL = 2 } gqa_tile_class_t;

/*
 * Bytes of device workspace that gqa_attn_fwd / gqa_attn_tile_plan need for this
 * problem.  Linear in Lq + Lk: a status word plus, when segment ids are used,
 * the [min, max] segment id of every query tile and key tile and the key-tile
 * range of every query tile (maxtext PR #4929, description: block-pair mask
 * tables of O((L / block)^2) entries are what overflowed splash's scalar memory at
 * 1M tokens; this plan keeps O(L / block)).  GQA_F32_TC adds, after 256-byte
 * aligned sections, one fp32 word per query and key/value head (the per-head
 * maxima |x| that fix the split scales) and the split operands: 2 x 2 bytes per
 * element of q, k and v.  Returns 0 for arguments that gqa_attn_fwd would reject.
 * Host-only; touches no device.
 */
size_t gqa_attn_workspace_bytes(int B, int Hq, int Hkv, int64_t Lq, int64_t Lk, int d,
                                int dtype, int mask_kind, int has_segments);

/*
 * The attention forward (see the top of this file for the operation).
 *
 *   q, k, v        device, read-only, layouts above, 16-byte aligned.
 *   out            device, written, [B, Hq, Lq, d] of dtype, 16-byte aligned.
 *   lse            device, written, [B, Hq, Lq] fp32 (natural log of the scaled
 *                  scores' exp-sum; -inf for a row with no visible key).
 *   B, Hq, Hkv     batch and head counts; Hq % Hkv == 0, Hq / Hkv in {1,2,4,8,16}.
 *   Lq, Lk         query rows and keys, >= 1, Lk == q_pos_offset + Lq.
 *   d              head dimension; must be 256.
 *   dtype          GQA_F32 (fp32 FFMA kernel), GQA_BF16 (tcgen05 kernel) or
 *                  GQA_F32_TC (fp32 tensors, tcgen05 kernel on split operands).
 *   mask_kind      GQA_MASK_CAUSAL or GQA_MASK_PREFIX_BRANCH (needs segment ids).
 *   q_pos_offset   keys preceding query row 0 (a state before its branch rows).
 *   segment_ids_q, segment_ids_kv
 *                  device int32 [Lq] and [Lk], both NULL (no segments) or both set.
 *                  Arbitrary int32 values; nondecreasing ids skip the most tiles.
 *   workspace      device, >= gqa_attn_workspace_bytes(...), 16-byte aligned;
 *                  overwritten by the call.  Calls that share a workspace must be
 *                  ordered on one stream.
 *   stream         the caller's cudaStream_t.
 *
 * Returns GQA_OK once all kernels are enqueued, or an error code with nothing
 * enqueued (validation) or a partly enqueued call (GQA_ERR_LAUNCH).
 */
int gqa_attn_fwd(const void *q, const void *k, const void *v, void *out, float *lse,
                 int B, int Hq, int Hkv, int64_t Lq, int64_t Lk, int d, int dtype,
                 int mask_kind, int64_t q_pos_offset,
                 const int32_t *segment_ids_q, const int32_t *segment_ids_kv,
                 void *workspace, size_t workspace_bytes, gqa_stream_t stream);

/*
 * Split-KV forward for short query blocks.  The branch rows after a shared state
 * (system1-omni issue #27, item 3: the state is computed once, then one branch per
 * question) and kev PR #202's re-prefill per question ("End to end") put few query
 * rows against a long key range; their query tiles alone leave most of the GPU's SMs
 * idle.  gqa_attn_fwd_split cuts the key-tile range of every query tile into `splits`
 * consecutive chunks, runs each chunk as its own work unit writing a normalised
 * partial output and its log-sum-exp, and merges them exactly:
 *     lse = ln sum_s exp(lse_s),   out = sum_s exp(lse_s - lse) * O_s.
 * The result equals gqa_attn_fwd's up to fp32 rounding order (it is the same online
 * softmax with one more combination step).
 *
 * gqa_attn_split_hint: a split count for this shape on a B200 (148 SMs): 1 when the
 *   query tiles already keep the SMs busy (last wave of work units >= 90 % full for
 *   GQA_F32, >= 60 % for the tensor-core dtypes GQA_BF16 and GQA_F32_TC, whose fp32
 *   partials cost relatively more) or the key ranges are short, else the smallest
 *   count in [2, 16] whose last wave is at least 90 % (GQA_F32) / 80 % full.
 *   Returns a negative gqa_status_t for a shape gqa_attn_fwd rejects.  Host-only.
 * gqa_attn_split_workspace_bytes: device workspace for gqa_attn_fwd_split with this
 *   split count: gqa_attn_workspace_bytes(...) plus splits * B * Hq * Lq * (d + 1)
 *   fp32 values for the partials, 256-byte aligned sections.  0 for a rejected shape
 *   or splits outside [1, 16].  Host-only.
 * gqa_attn_fwd_split: arguments as gqa_attn_fwd, plus `splits` in [1, 16] (1 is
 *   gqa_attn_fwd itself) and a workspace of at least
 *   gqa_attn_split_workspace_bytes(...).  Enqueues the attention kernel and, for
 *   splits > 1, one merge kernel on `stream`.  Errors as gqa_attn_fwd
 *   (GQA_ERR_INVALID_ARG also for splits outside [1, 16]).
 */
int gqa_attn_split_hint(int B, int Hq, int Hkv, int64_t Lq, int64_t Lk, int dtype, int mask_kind,
                        int has_segments);
size_t gqa_attn_split_workspace_bytes(int B, int Hq, int Hkv, int64_t Lq, int64_t Lk, int d, int dtype,
                                      int mask_kind, int has_segments, int splits);
int gqa_attn_fwd_split(const void *q, const void *k, const void *v, void *out, float *lse,
                       int B, int Hq, int Hkv, int64_t Lq, int64_t Lk, int d, int dtype,
                       int mask_kind, int64_t q_pos_offset,
                       const int32_t *segment_ids_q, const int32_t *segment_ids_kv, int splits,
                       void *workspace, size_t workspace_bytes, gqa_stream_t stream);

/*
 * Context-parallel blocks.  maxtext PR #4929 trains at 1,048,576 tokens with context
 * parallelism ("Effect"), and its code review names the ring attention path
 * (use_tokamax_ring): the sequence is sharded across devices, each device's query
 * rows attend to every earlier device's key/value block in turn, and the partial
 * results are merged by their log-sum-exps.  These two calls are the per-device
 * compute of such a ring; the transport between devices is the caller's (the Python
 * package's `ring` module uses NCCL send / receive through torch.distributed).
 *
 * gqa_attn_fwd_offset: causal attention of Lq query rows against a block of Lk keys
 *   that starts q_pos_offset >= 0 positions before query row 0: row i sees key j iff
 *   j <= i + q_pos_offset.  Unlike gqa_attn_fwd, Lk is free (Lk <= q_pos_offset covers
 *   a block wholly before the queries, every key visible).  No segment ids, causal
 *   mask only.  Arguments, layouts, dtypes and errors otherwise as gqa_attn_fwd; the
 *   workspace needs 256 bytes (16-byte aligned), which is why dtype GQA_F32_TC (whose
 *   split operands live in the workspace) returns GQA_ERR_UNSUPPORTED here.  Every
 *   row sees key 0, so no row is empty.
 * gqa_attn_merge: exact combination of two partial results over disjoint key sets,
 *       lse = ln(exp(lse_a) + exp(lse_b)),
 *       out = exp(lse_a - lse) * o_a + exp(lse_b - lse) * o_b,
 *   row by row over `rows` rows of d = 256 columns.  o_a: device fp32 [rows][d] with
 *   lse_a [rows], or both NULL (an empty partial, lse = -inf); o_b: device fp32 or
 *   bf16 (dtype_b) with lse_b, or both NULL; o_out: device [rows][d] in dtype_out and
 *   lse_out [rows] fp32, written.  o_out / lse_out may be o_a / lse_a (in place,
 *   dtype_out = GQA_F32), not o_b.  A row empty on both sides gets out = 0, lse = -inf.
 *   All pointers 16-byte aligned.  Enqueues one kernel on `stream`.  Errors:
 *   GQA_ERR_INVALID_ARG (rows < 1, an output NULL, a half-given pair, a bad dtype),
 *   GQA_ERR_UNSUPPORTED (d != 256), GQA_ERR_MISALIGNED, GQA_ERR_LAUNCH.
 */
int gqa_attn_fwd_offset(const void *q, const void *k, const void *v, void *out, float *lse,
                        int B, int Hq, int Hkv, int64_t Lq, int64_t Lk, int d, int dtype,
                        int64_t q_pos_offset, void *workspace, size_t workspace_bytes,
                        gqa_stream_t stream);
int gqa_attn_merge(const float *o_a, const float *lse_a, const void *o_b, const float *lse_b,
                   void *o_out, float *lse_out, int64_t rows, int d, int dtype_b, int dtype_out,
                   gqa_stream_t stream);

/*
 * Attention backward: the gradients of sum(out * dout) with respect to q, k and v,
 * for training on packed long sequences (maxtext PR #4929, description: the splash
 * kernel runs inside training steps over 1,048,576-token packed batches).  With
 * P = exp(scale * S - lse) recomputed from the forward's saved log-sum-exp,
 * D_i = <dout_i, out_i>, dP = dout V^T and dS = P * (dP - D):
 *     dq = scale * dS K,   dk = scale * sum over the group's query heads of dS^T Q,
 *     dv = sum over the group's query heads of P^T dout.
 *
 *   q, k, v, out, lse   device, the forward's inputs and outputs (out and lse as
 *                       written by gqa_attn_fwd or gqa_attn_fwd_split for the same
 *                       arguments), layouts as for gqa_attn_fwd.
 *   dout                device, [B, Hq, Lq, d] of dtype: the upstream gradient.
 *   dq, dk, dv          device, written, shapes of q, k, v, of dtype (bf16 outputs are
 *                       rounded to nearest even from fp32 accumulation).
 *   dtype               GQA_F32 or GQA_BF16; GQA_F32_TC returns GQA_ERR_UNSUPPORTED
 *                       (the fp32 backward is dtype GQA_F32).
 *   other arguments     as for gqa_attn_fwd; every pointer 16-byte aligned.
 *   workspace           device, >= gqa_attn_bwd_workspace_bytes(...): status word,
 *                       block-skip plan at the backward's tile sizes (fp32: 64 query
 *                       rows x 32 keys; bf16: 128 / G positions x 128 keys), and the
 *                       fp32 row dot products D (bf16: also the log2-domain LSE; rows
 *                       padded to a multiple of 128).
 *
 * Rows with no visible key contribute nothing (their dq is 0).  Enqueues on `stream`:
 * GQA_F32 -- a row-dot kernel, the plan kernels (with segment ids), a dK/dV kernel and a
 * dQ kernel, fp32 arithmetic on the CUDA cores; GQA_BF16 -- a row-state kernel, the
 * plan kernels (with segment ids) and three tensor-core kernels (dV, dK, dQ; bf16
 * operands, fp32 accumulation).  Errors as gqa_attn_fwd.  gqa_attn_bwd_workspace_bytes
 * returns 0 for a shape gqa_attn_fwd rejects and for GQA_F32_TC.  Host-only.
 */
size_t gqa_attn_bwd_workspace_bytes(int B, int Hq, int Hkv, int64_t Lq, int64_t Lk, int d, int dtype,
                                    int mask_kind, int has_segments);
int gqa_attn_bwd(const void *q, const void *k, const void *v, const void *out, const float *lse,
                 const void *dout, void *dq, void *dk, void *dv, int B, int Hq, int Hkv, int64_t Lq,
                 int64_t Lk, int d, int dtype, int mask_kind, int64_t q_pos_offset,
                 const int32_t *segment_ids_q, const int32_t *segment_ids_kv, void *workspace,
                 size_t workspace_bytes, gqa_stream_t stream);

/*
 * gqa_attn_bwd_offset: the backward of one block of gqa_attn_fwd_offset (causal
 * attention of Lq query rows against a block of Lk keys that starts q_pos_offset >= 0
 * positions before query row 0; row i sees key j iff j <= i + q_pos_offset; Lk free),
 * for a sequence sharded into blocks (context-parallel training; maxtext PR #4929,
 * description and code review: 1,048,576-token training with a ring attention path).
 * `out` and `lse` are the WHOLE sequence's (the merged forward's rows), so
 * P = exp(scale * S - lse) is the block's share of each row's softmax and D = <dout,
 * out> is the full row's: the call writes the block's contributions to dq (over this
 * key block only), dk and dv (over these query rows only), which the caller sums over
 * the blocks.  Causal mask only, no segment ids; dtype GQA_F32 or GQA_BF16.  Workspace:
 * gqa_attn_bwd_workspace_bytes(B, Hq, Hkv, Lq, Lq, d, dtype, GQA_MASK_CAUSAL, 0) bytes
 * (it does not depend on Lk or the offset).  Other arguments and errors as gqa_attn_bwd.
 */
int gqa_attn_bwd_offset(const void *q, const void *k, const void *v, const void *out, const float *lse,
                        const void *dout, void *dq, void *dk, void *dv, int B, int Hq, int Hkv, int64_t Lq,
                        int64_t Lk, int d, int dtype, int64_t q_pos_offset, void *workspace,
                        size_t workspace_bytes, gqa_stream_t stream);

/*
 * Tile shape used by gqa_attn_fwd for this dtype and group size G = Hq / Hkv:
 * *br = query positions per query tile (each tile holds br positions of all G
 * heads of one key/value head), *bc = keys per key tile.  Host-only.
 */
int gqa_attn_tile_sizes(int dtype, int Hq, int Hkv, int *br, int *bc);

/*
 * Test and debug export of the block-skip plan that gqa_attn_fwd computes on the
 * device for the same arguments (same dtype and group size, hence same tiles).
 *
 *   classes     device, written, [nq, nk] uint8 gqa_tile_class_t, nq = ceil(Lq/br),
 *               nk = ceil(Lk/bc) (this matrix exists only in this export; the
 *               forward never forms it).
 *   kv_ranges   device, written, [nq, 2] int32: [first, last + 1) of the non-SKIP
 *               key tiles of each query tile, (0, 0) if none.
 *
 * The class of a (query tile, key tile) pair follows from the tiles' positions and
 * their [min, max] segment ids only; SKIP tiles hold no visible pair and are never
 * read, FULL tiles hold only visible pairs and skip the per-element mask.
 */
int gqa_attn_tile_plan(int Hq, int Hkv, int64_t Lq, int64_t Lk, int dtype, int mask_kind,
                       int64_t q_pos_offset, const int32_t *segment_ids_q,
                       const int32_t *segment_ids_kv, void *workspace, size_t workspace_bytes,
                       uint8_t *classes, int32_t *kv_ranges, gqa_stream_t stream);

/*
 * Device-side status of the last call that used this workspace: GQA_OK,
 * GQA_ERR_DEVICE_TIMEOUT (a bounded wait on an mbarrier ran out; the kernel
 * stopped, its outputs are undefined) or, in a library built with
 * GQA_DEBUG_BOUNDS, GQA_ERR_DEVICE_BOUNDS (an index check of the FFMA kernels
 * failed; the access was skipped, the outputs are undefined).  Synchronises `stream` (copies one word
 * back).  Returns GQA_ERR_LAUNCH if the copy itself fails.
 */
int gqa_attn_status(const void *workspace, gqa_stream_t stream);

/*
 * Self-test of the bounded-wait machinery: launches one CTA that waits on an
 * mbarrier nothing ever arrives on, with a budget of `budget_ns` nanoseconds
 * (1 ms .. 10 s).  The wait must give up and record GQA_ERR_DEVICE_TIMEOUT in
 * the workspace, which gqa_attn_status() then returns; the context stays usable.
 * `workspace` needs gqa_attn_workspace_bytes(...) >= 256 bytes.
 */
int gqa_attn_selftest_wait(void *workspace, size_t workspace_bytes, int64_t budget_ns,
                           gqa_stream_t stream);

/*
 * Self-test of the index checks of a checked build (compiled with GQA_DEBUG_BOUNDS:
 * the fp32 FFMA kernels then check each shared-memory access against the region it
 * belongs to and each output row against its buffer, skip a failing access and record
 * GQA_ERR_DEVICE_BOUNDS).  One CTA evaluates in-range checks and, with planted = 1,
 * one out-of-range shared address and global index as well; only the comparisons
 * run, no access is made.  Afterwards gqa_attn_status() returns GQA_OK (planted = 0)
 * or GQA_ERR_DEVICE_BOUNDS (planted = 1).  Returns GQA_ERR_UNSUPPORTED, launching
 * nothing, in a normal build (which is how a caller tells the two apart);
 * GQA_ERR_INVALID_ARG for planted other than 0 or 1.  `workspace`: >= 256 bytes,
 * 16-byte aligned.
 */
int gqa_attn_selftest_bounds(void *workspace, size_t workspace_bytes, int planted, gqa_stream_t stream);

/*
 * Measurement aid (no attention work): the throughput ceiling of fp32 FMAs with every
 * operand in registers, by operand form:
 *   form 0: fma.rn.f32x2 in the GQA_F32 kernels' operand form, (s_r, s_r+1) +=
 *           (q_r, q_r+1) * (k, k), consecutive FMAs sharing the duplicated k;
 *   form 1: the same FMAs, consecutive ones sharing the (q_r, q_r+1) pair (the order
 *           the kernels use for most of their packed FMAs);
 *   form 2: packed FMAs with no duplicated operand ((q_r, q_r+1) * (k_m, k_m+1) and
 *           the crossed pair);
 *   form 3: scalar fma.rn.f32.
 * Launches `ctas` CTAs of 256 threads; each thread runs `iters` rounds of 64 FMAs and
 * writes one float to out[cta * 256 + thread] (device, ctas * 256 floats, 16-byte
 * aligned, caller-owned).  Asynchronous on `stream`: time it with events; 2 x ctas x
 * 256 x iters x 64 flop over the time is the attainable FP32 rate of that form.  Form
 * 1 is the denominator the bench reports next to the nominal FP32 peak (kev PR #202,
 * "Measurements": the fp32 path is the one evaluated).  GQA_ERR_INVALID_ARG for a null
 * `out`, ctas outside 1 .. 65535, iters < 1 or form outside 0 .. 3;
 * GQA_ERR_MISALIGNED; GQA_ERR_LAUNCH.
 */
int gqa_attn_probe_ffma2(float *out, int ctas, int iters, int form, gqa_stream_t stream);

/*
 * Size of the device scratch behind gqa_attn_fwd_static_ws (2 MiB).  Calls without
 * segment ids need only the 256-byte status header, at any length.  With segment ids
 * the block-skip tables grow with the number of query tiles, Lq * G / 64 (GQA_F32) or
 * Lq * G / 128 (GQA_BF16) with G = Hq / Hkv: 1,048,576-token calls fit for G <= 4 in
 * GQA_F32 and G <= 8 in GQA_BF16; at G = 16 (and G = 8 in GQA_F32) they need more and
 * return GQA_ERR_WORKSPACE.  GQA_F32_TC keeps split operand planes as large as the
 * fp32 inputs in its workspace, so only tiny shapes fit this scratch.
 */
#define GQA_ATTN_STATIC_WORKSPACE_BYTES ((size_t)2 << 20)

/*
 * gqa_attn_fwd without a workspace argument, for callers that cannot allocate device
 * memory (no counterpart on the pages: this is an integration convenience).  Such
 * callers include plug-ins inside a host framework that owns all device memory and
 * exposes no allocator, services held to a fixed memory budget after start-up, and
 * latency-critical paths that must avoid the device synchronisation an allocation can
 * cause.  The caller still provides q, k, v, out, lse and the segment ids exactly as
 * for gqa_attn_fwd (same arguments, layouts, semantics and return codes).
 *
 * Scratch: a file-scope device array of GQA_ATTN_STATIC_WORKSPACE_BYTES in this
 * library, which every GPU that loads the library holds until the process exits.
 * Calls whose gqa_attn_workspace_bytes(...) exceeds that size return
 * GQA_ERR_WORKSPACE and enqueue nothing.  This call allocates and frees nothing and
 * calls no allocating routine.
 *
 * Set-up: the first call on each device (with that device current) looks up the
 * array's device address once; make that first call before any stream capture.
 * Sharing: every call on a device uses the same array and leaves the last call's
 * contents in it (each call resets what must start at zero), so calls that overlap
 * on the GPU -- on different streams, or from several host threads -- race; order
 * them on one stream.  gqa_attn_status() cannot read this scratch.
 */
int gqa_attn_fwd_static_ws(const void *q, const void *k, const void *v, void *out, float *lse,
                           int B, int Hq, int Hkv, int64_t Lq, int64_t Lk, int d, int dtype,
                           int mask_kind, int64_t q_pos_offset,
                           const int32_t *segment_ids_q, const int32_t *segment_ids_kv,
                           gqa_stream_t stream);

/* Static, human-readable text for a gqa_status_t; never NULL. */
const char *gqa_attn_strerror(int status);

#ifdef __cplusplus
}
#endif

#endif /* GQA_ATTN_H_ */
