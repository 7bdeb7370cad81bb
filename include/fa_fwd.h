/*
 * fa_fwd.h -- C ABI of the B200 (sm_100a) FlashAttention forward library,
 * libfa_fwd.so.
 *
 * The operation.  For every batch b, head h and query row i
 *
 *     O[b,h,i,:] = softmax_j( scale * q[b,h,i,:] . k[b,h,j,:]  [+ causal mask] ) * V[b,h,:,:]
 *     LSE[b,h,i] = ln( sum_j exp( scale * q[b,h,i,:] . k[b,h,j,:] ) )   over the visible keys j
 *
 * computed tile by tile with an online softmax (running row max and running
 * exp-sum, rescaled per key/value tile) so that the Sq x Sk score matrix never
 * reaches device memory.  Sources on the pages:
 *   - the standard attention it must equal, and the tiling + online-softmax
 *     method: page "FlashAttention: long-text inference without running out
 *     of memory" (ai6s.net/6a0d42d8), sections "the memory black hole" and
 *     "FlashAttention's answer: tiling + online normalisation";
 *   - the causal flag in place of a mask tensor: page "FlashAttention in
 *     ops-transformer on Ascend NPU" (ai6s.net/6a0d3bfb), section "how
 *     FlashAttention runs on the Ascend NPU" (causal=True, not a triu mask);
 *   - whole-tile skipping above the diagonal: page "catlass FlashAttention
 *     template tuning" (hwcomputing.csdn.net/6a0d4681), section "causal mask
 *     implementations", mode 2 (diagonal skip);
 *   - the per-row log-sum-exp [B, H, S] in natural log: page "64K
 *     long-sequence FlashAttention" (ai6s.net/6a140d07), section "layer 2:
 *     numerical stability";
 *   - the call shape flash_attention(q, k, v, head_num, input_layout, scale)
 *     and the BSND / BNSD layouts: page "ops-transformer FlashAttention on
 *     Atlas 800" (hwcomputing.csdn.net/6a0d4444), sections "minimal runnable
 *     code" and the error table; page hwcomputing.csdn.net/6a0d4681, section
 *     "data layout";
 *   - fp16 and bf16 as the two half-precision choices: page
 *     hwcomputing.csdn.net/6a0d4681, section "precision choice".
 *
 * Causal masking is aligned at the top-left corner: key j is visible to query
 * i iff j <= i (the pages only show the square case, triu(ones(S,S), 1)).
 * Every row therefore sees at least key 0.
 *
 * Arithmetic: q.k products accumulate in fp32 on the tensor cores; the
 * softmax runs in fp32; the probabilities are rounded to the input dtype
 * before P.V (fp32 accumulation); O is rounded to the input dtype once, at
 * the end; LSE is fp32.
 *
 * Besides the forward pass (fa_fwd, fa_fwd_ws, fa_fwd_opts, fa_fwd_heads,
 * fa_fwd_noalloc, fa_fwd_varlen, fa_fwd_splitkv) the library exports its backward pass
 * (fa_bwd, fa_bwd_atomic), the merge of
 * partial results that ring attention over several GPUs is built from
 * (fa_lse_merge), one ring step with that merge fused into the attention
 * (fa_fwd_ring_step), and the attention output projection (fa_out_proj,
 * fa_fwd_proj).  Each is described at its declaration below.
 */
#ifndef FA_FWD_H
#define FA_FWD_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Return codes.  No entry point crashes on a bad argument: it returns one of these. */
typedef enum fa_status {
    FA_OK = 0,
    FA_ERR_INVALID_ARG = 1,        /* null pointer, non-positive size, bad enum, non-finite scale, Sk = 0 */
    FA_ERR_UNSUPPORTED = 2,        /* head dim D not in {64, 128}, or a size beyond the 32-bit tile coordinates */
    FA_ERR_NOT_DEVICE_POINTER = 3, /* a tensor pointer is host memory (the pages: a CPU tensor segfaults; here it is refused) */
    FA_ERR_MISALIGNED = 4,         /* q, k, v or o not 16-byte aligned (TMA), or lse not 4-byte aligned */
    FA_ERR_ALIAS = 5,              /* o or lse overlaps q, k or v, or o overlaps lse */
    FA_ERR_CUDA = 6,               /* a CUDA runtime / driver call failed; see fa_last_cuda_error() */
    FA_ERR_TIMEOUT = 7             /* a kernel wait ran past its limit (reported by fa_device_status) */
} fa_status;

/* Tensor layouts.  "N" is the head axis: BSND == BSHD, BHSD == BNSD. */
typedef enum fa_layout {
    FA_BSND = 0,   /* q: [B, Sq, H, D], k and v: [B, Sk, H, D], o like q */
    FA_BHSD = 1    /* q: [B, H, Sq, D], k and v: [B, H, Sk, D], o like q */
} fa_layout;

/* Element type of q, k, v and o. */
typedef enum fa_dtype {
    FA_FP16 = 0,
    FA_BF16 = 1
} fa_dtype;

/*
 * fa_fwd -- the attention forward pass, asynchronous on `stream`.
 *
 * q, k, v   device pointers, dense and contiguous in `layout` (row-major,
 *           innermost axis D), element type `dtype`; read only.  16-byte
 *           aligned (they are read with TMA).
 * o         device pointer, same shape, layout and dtype as q; every element
 *           is overwritten.  16-byte aligned.
 * lse       device pointer to B*H*Sq fp32 values laid out [B, H, Sq]
 *           (head-major in both layouts); every element is overwritten with
 *           the natural-log log-sum-exp of the row's scaled, masked logits.
 * B, H      batch and head counts (>= 1).
 * Sq, Sk    query and key lengths.  Sq = 0 is a no-op returning FA_OK; Sk must
 *           be >= 1 (a softmax over no keys is undefined).  Neither needs to be
 *           a multiple of the tile: ragged tails are masked in the kernel.
 * D         head dimension, 64 or 128.
 * layout    FA_BSND or FA_BHSD.
 * causal    non-zero: key j is visible to query i iff j <= i.
 * scale     multiplies q.k before the softmax, used as given (any finite
 *           value, 0 included; the usual choice is 1/sqrt(D)).
 * dtype     FA_FP16 or FA_BF16.
 * stream    a cudaStream_t (passed as void*); NULL is the legacy default stream.
 *
 * Ownership: the caller allocates and owns every buffer; the library keeps no
 * pointer after the call returns and allocates no device memory.  o and lse
 * must not overlap q, k, v or each other.
 *
 * Errors: arguments are validated before anything is launched and every
 * failure is a return code.  FA_ERR_CUDA means a launch or driver call
 * failed; fa_last_cuda_error() gives the CUDA error number.  A kernel whose
 * internal wait exceeded its limit (which indicates a bug, never expected)
 * stops early, leaves o / lse unspecified, and is reported by the next
 * fa_device_status() call.
 *
 * The call does not synchronise.  It is safe to call from several host
 * threads on different streams.
 */
fa_status fa_fwd(const void *q, const void *k, const void *v, void *o, float *lse,
                 int64_t B, int64_t H, int64_t Sq, int64_t Sk, int64_t D,
                 fa_layout layout, int causal, float scale, fa_dtype dtype, void *stream);

/*
 * fa_fwd_ws -- fa_fwd with a dynamic work schedule: the same operation,
 * arguments and results (bit-identical: each work unit is computed the same
 * way), but the persistent CTAs take work units (two 128-row query tiles of
 * one batch and head) from a counter in `workspace`, longest first, instead
 * of a fixed round-robin share.  This balances causal workloads, whose units
 * differ in length (page "64K long-sequence FlashAttention"
 * (ai6s.net/6a140d07), section "multi-AI-Core load balancing": dynamic
 * scheduling of uneven per-core tile counts).
 *
 * workspace        device memory of at least fa_fwd_workspace_size() bytes,
 *                  16-byte aligned, owned by the caller; the library zeroes
 *                  it on `stream` before the launch and uses it as scratch
 *                  (a call with no more work units than the GPU has SMs
 *                  needs no counter: it neither zeroes nor uses it).
 *                  It must not overlap any tensor argument, and two calls
 *                  that may run at the same time need separate workspaces.
 * workspace_bytes  its size in bytes.
 *
 * Errors as for fa_fwd, plus FA_ERR_INVALID_ARG (null or too small
 * workspace), FA_ERR_MISALIGNED and FA_ERR_ALIAS for the workspace.
 */
fa_status fa_fwd_ws(const void *q, const void *k, const void *v, void *o, float *lse,
                    int64_t B, int64_t H, int64_t Sq, int64_t Sk, int64_t D,
                    fa_layout layout, int causal, float scale, fa_dtype dtype,
                    void *workspace, size_t workspace_bytes, void *stream);

/* Bytes of device workspace fa_fwd_ws needs (a small constant). */
size_t fa_fwd_workspace_size(void);

/*
 * fa_fwd_options -- settings of the online softmax's lazy rescale, and
 * optional statistics of it (for fa_fwd_opts).
 *
 * The pages' recurrence moves a row's running max, and rescales its running
 * sum and partial output, whenever a key tile holds a larger logit (page
 * "FlashAttention: long-text inference without running out of memory"
 * (ai6s.net/6a0d42d8), section "tiling + online normalisation").  The kernel
 * moves its reference max only when a tile's max exceeds it by more than
 * rescale_threshold_log2 (in log2 units of the scaled logits); until then the
 * tile's weights are taken against the older, smaller reference and may reach
 * 2^rescale_threshold_log2.  O, the sum and the LSE use the same reference, so
 * the result is the same softmax; only the rounding differs.  For bf16 a moved
 * reference is set bf16_headroom_log2 above the tile max (weights then start
 * at most 2^-headroom, so later tiles may rise further before the next move);
 * fp16 ignores the headroom.  Threshold 0 and headroom 0 is the pages'
 * recurrence taken literally.
 *
 * rescale_threshold_log2  in [0, 15] (fp16 holds weights up to 2^15); default 15.
 * bf16_headroom_log2      in [0, 16]; default 8.
 * branch_counts           NULL, or device memory for four 64-bit counters,
 *                         8-byte aligned, that the kernel INCREMENTS (zero them
 *                         first): per warp of 32 rows and key tile after a
 *                         work unit's first, [0] such warp-tiles, [1] with the
 *                         tile's speculative pass rejected (a weight above
 *                         2^threshold: the tile is recomputed against its
 *                         exact max), [2] with the rows' O rescaled, [3]
 *                         accepted with a weight above 2^(threshold - 1).
 */
typedef struct fa_fwd_options {
    float rescale_threshold_log2;
    float bf16_headroom_log2;
    unsigned long long *branch_counts;
} fa_fwd_options;

/* Fills *opts with the defaults fa_fwd uses (threshold 15, headroom 8, no counters). */
void fa_fwd_default_options(fa_fwd_options *opts);

/*
 * fa_fwd_opts -- fa_fwd (workspace NULL) or fa_fwd_ws (workspace given) with
 * the lazy rescale's settings and statistics taken from *opts (NULL: the
 * defaults).  FA_ERR_INVALID_ARG for settings outside their ranges,
 * FA_ERR_MISALIGNED / FA_ERR_NOT_DEVICE_POINTER / FA_ERR_ALIAS for the
 * counters as for a tensor; otherwise as fa_fwd / fa_fwd_ws.
 */
fa_status fa_fwd_opts(const void *q, const void *k, const void *v, void *o, float *lse,
                      int64_t B, int64_t H, int64_t Sq, int64_t Sk, int64_t D,
                      fa_layout layout, int causal, float scale, fa_dtype dtype,
                      const fa_fwd_options *opts, void *workspace, size_t workspace_bytes, void *stream);

/*
 * fa_fwd_heads -- the forward pass over a contiguous range of heads only:
 * the share of one GPU when the heads of one problem are split across GPUs
 * (page "64K long-sequence FlashAttention" (ai6s.net/6a140d07), section
 * "performance tuning tips", multi-card model parallelism; attention heads
 * are independent, so the split needs no exchange during the pass).
 *
 * q, k, v, o, lse, B .. dtype   as for fa_fwd: the WHOLE problem's tensors,
 *                  in place.  Only the heads g = b * H + h (flattened, batch
 *                  major) with head_begin <= g < head_begin + head_count are
 *                  read and computed; their rows of o and lse are written and
 *                  every other element of o and lse is left untouched.  So
 *                  several calls over disjoint ranges (on one GPU, or on
 *                  GPUs that each hold the tensors) together write the whole
 *                  result, bit-identical to one fa_fwd call: a head's result
 *                  does not depend on which launch computes it.
 * head_begin, head_count   0 <= head_begin, head_begin + head_count <= B * H
 *                  (else FA_ERR_INVALID_ARG); head_count = 0 is a no-op.
 * workspace, workspace_bytes   as for fa_fwd_ws (dynamic schedule), or NULL
 *                  and 0 for the static schedule of fa_fwd.
 *
 * Errors as for fa_fwd and fa_fwd_ws.  Asynchronous on `stream`; allocates
 * nothing.
 */
fa_status fa_fwd_heads(const void *q, const void *k, const void *v, void *o, float *lse,
                       int64_t B, int64_t H, int64_t Sq, int64_t Sk, int64_t D,
                       fa_layout layout, int causal, float scale, fa_dtype dtype,
                       int64_t head_begin, int64_t head_count,
                       void *workspace, size_t workspace_bytes, void *stream);

/*
 * fa_fwd_varlen -- the same forward pass over a batch of B sequences of
 * different lengths, packed row after row (the uneven-work case of page "64K
 * long-sequence FlashAttention" (ai6s.net/6a140d07), section "multi-AI-Core
 * load balancing"; work units of short sequences simply end sooner).
 * Sequence b owns query rows [cu_seqlens_q[b], cu_seqlens_q[b+1]) and key /
 * value rows [cu_seqlens_k[b], cu_seqlens_k[b+1]); it attends only to its own
 * keys, causal alignment is top-left within the sequence (key j visible to
 * query i iff j <= i, both counted from the sequence start).
 *
 * q, o           [total_q, H, D], fp16 / bf16, contiguous, 16-byte aligned
 * k, v           [total_k, H, D]
 * lse            [H, total_q] fp32: lse[h * total_q + row] (natural log)
 * cu_seqlens_q/k device int32 arrays of B + 1 offsets, non-decreasing, first
 *                0, last <= total_q / total_k, 4-byte aligned
 * max_seqlen_q/k upper bounds of the sequence lengths (they size the
 *                schedule); <= total_q / total_k
 * workspace      as for fa_fwd_ws, or NULL for the static schedule
 *
 * Every other argument is as for fa_fwd.  The offsets live on the device, so
 * the host cannot check them: a sequence whose offsets are out of range or
 * decreasing, longer than max_seqlen_q/k, or with queries but no keys, is
 * skipped (its o and lse rows are not written) and the next
 * fa_device_status() returns FA_ERR_INVALID_ARG.  Sequences with no query
 * rows are allowed.  Host-side errors are returned as for fa_fwd.
 */
fa_status fa_fwd_varlen(const void *q, const void *k, const void *v, void *o, float *lse,
                        const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                        int64_t B, int64_t H, int64_t total_q, int64_t total_k,
                        int64_t max_seqlen_q, int64_t max_seqlen_k, int64_t D,
                        int causal, float scale, fa_dtype dtype,
                        void *workspace, size_t workspace_bytes, void *stream);

/*
 * fa_bwd -- gradients of the forward pass: given q, k, v, the forward's o and
 * lse, and dout = dL/dO, writes dq, dk, dv (same shapes, layout and dtype as
 * q, k, v).  The weights are recomputed from q, k and lse (page "FlashAttention
 * in ops-transformer on Ascend NPU" (ai6s.net/6a0d3bfb), section "how FA runs
 * on the NPU": recomputation), then dV = P^T dO, dS = P * (dO V^T -
 * rowsum(dO * O)), dQ = scale dS K, dK = scale dS^T Q, with the forward's
 * causal mask.  Deterministic: every gradient row is accumulated by one CTA in
 * a fixed order, with no atomics (page "catlass FlashAttention template
 * tuning" (hwcomputing.csdn.net/6a0d4681): the backward's `deterministic`
 * switch).  fp32 accumulation; results rounded to the input dtype.
 *
 * q, k, v, o, dout, lse, B, H, Sq, Sk, D, layout, causal, scale, dtype, stream
 *                  as for fa_fwd (o and lse as fa_fwd wrote them)
 * dq, dk, dv       outputs, caller-owned, 16-byte aligned, fully overwritten
 * workspace        device memory of fa_bwd_workspace_size(B, H, Sq) bytes,
 *                  16-byte aligned, caller-owned scratch (per-row sums)
 *
 * Errors as for fa_fwd; the outputs and the workspace must not overlap each
 * other or any input (FA_ERR_ALIAS).  Sq = 0 sets dk = dv = 0.
 */
size_t fa_bwd_workspace_size(int64_t B, int64_t H, int64_t Sq);
fa_status fa_bwd(const void *q, const void *k, const void *v, const void *o, const void *dout,
                 const float *lse, void *dq, void *dk, void *dv,
                 int64_t B, int64_t H, int64_t Sq, int64_t Sk, int64_t D,
                 fa_layout layout, int causal, float scale, fa_dtype dtype,
                 void *workspace, size_t workspace_bytes, void *stream);

/*
 * fa_selftest_wait_timeout -- exercises the kernel's failure detection
 * without a fault.  The kernel is launched as by fa_fwd (same arguments and
 * validation), but its producer warp issues no loads and every wait is limited
 * to `wait_limit_us` microseconds (1,000 .. 1,000,000).  Every consumer's wait
 * for Q or K / V therefore runs out; the CTAs record the timeout in the device
 * error word, drain (nothing is in flight) and return.  q, k and v are not
 * read; o and lse are not written.  Returns FA_OK once launched (or the
 * argument error fa_fwd would return, FA_ERR_INVALID_ARG for a limit outside
 * the range); the next fa_device_status() then returns FA_ERR_TIMEOUT and
 * clears the word, and the CUDA context stays usable.  The pages have no
 * counterpart: this is a test hook for the bounded waits.
 */
fa_status fa_selftest_wait_timeout(const void *q, const void *k, const void *v, void *o, float *lse,
                                   int64_t B, int64_t H, int64_t Sq, int64_t Sk, int64_t D,
                                   fa_layout layout, int causal, float scale, fa_dtype dtype,
                                   uint32_t wait_limit_us, void *stream);

/*
 * fa_fwd_noalloc -- fa_fwd_ws for callers that cannot allocate device memory.
 * This entry point has no counterpart on the pages: it exists for callers
 * that own only their input and output buffers -- a plugin inside a host
 * framework that keeps every device allocation to itself, or a latency-bound
 * path that must not call the CUDA allocator (cudaMalloc can synchronise the
 * device and fragment a fixed memory budget).  It computes exactly what
 * fa_fwd_ws computes and allocates nothing.
 *
 * The dynamic schedule's scratch (its work counter, 16 bytes) lives in a
 * fixed 256-byte array inside the library, held by every GPU that loads the
 * library until the process exits.  The counter's size does not depend on
 * the call's sizes, so no size is too large for the array.  The first call
 * on a device looks up that array's device address (cudaGetSymbolAddress,
 * with the device current); make that first call before any stream capture.
 * Only a successful lookup is kept: a lookup that fails returns FA_ERR_CUDA
 * and is tried again by the next call.  After cudaDeviceReset the kept
 * address is checked, found stale and looked up again.  Every call that
 * needs the counter (see fa_fwd_ws) zeroes it on `stream` before its launch
 * and then uses it, so calls that
 * overlap on the same GPU (for example on two streams) race on it: serialise
 * them, or use fa_fwd_ws with separate workspaces.  Each GPU has its own copy
 * of the array.  Arguments, results and errors as for fa_fwd, checked in the
 * same order.
 */
fa_status fa_fwd_noalloc(const void *q, const void *k, const void *v, void *o, float *lse,
                         int64_t B, int64_t H, int64_t Sq, int64_t Sk, int64_t D,
                         fa_layout layout, int causal, float scale, fa_dtype dtype, void *stream);

/*
 * fa_bwd_atomic -- the backward pass's non-deterministic variant (page "catlass
 * FlashAttention template tuning" (hwcomputing.csdn.net/6a0d4681), section on
 * the backward: the `deterministic` switch, atomic adds when off).  Same
 * arithmetic and arguments as fa_bwd, D = 64 or 128.
 * One kernel per 128-key tile computes dK, dV and that tile's share of dQ;
 * the shares are added into an fp32 accumulator in the workspace by atomic
 * adds in whatever order the tiles finish, so dq may differ between runs by
 * fp32 rounding (dk and dv do not).  A last pass scales the
 * accumulator and rounds it into dq.
 *
 * workspace   device memory of fa_bwd_atomic_workspace_size(B, H, Sq, D)
 *             bytes, 16-byte aligned, caller-owned scratch (the per-row sums
 *             and the dQ accumulator, zeroed here on the stream)
 *
 * Everything else as for fa_bwd.
 */
size_t fa_bwd_atomic_workspace_size(int64_t B, int64_t H, int64_t Sq, int64_t D);
fa_status fa_bwd_atomic(const void *q, const void *k, const void *v, const void *o, const void *dout,
                        const float *lse, void *dq, void *dk, void *dv, int64_t B, int64_t H, int64_t Sq,
                        int64_t Sk, int64_t D, fa_layout layout, int causal, float scale, fa_dtype dtype,
                        void *workspace, size_t workspace_bytes, void *stream);

/*
 * fa_lse_merge -- merges one partial attention result into a running one.
 * Attention over a key range split into blocks (ring / context-parallel
 * attention: page "FlashAttention in ops-transformer on Ascend NPU"
 * (ai6s.net/6a0d3bfb), section "what else is in the ops-transformer
 * repository", ring attention for long sequences; page "64K long-sequence
 * FlashAttention" (ai6s.net/6a140d07), section "performance tuning tips",
 * multi-card parallelism) gives, per query row, a partial (O_i, LSE_i)
 * normalised over block i (what fa_fwd writes for that block).  The result over
 * the union of the blocks follows the online-normalisation update of page
 * "FlashAttention: long-text inference without running out of memory"
 * (ai6s.net/6a0d42d8), section on tiling and online normalisation, applied to
 * whole blocks:
 *     LSE = log(exp(LSE_acc) + exp(LSE_part))
 *     O   = exp(LSE_acc - LSE) O_acc + exp(LSE_part - LSE) O_part
 * A row with LSE = -inf (no visible key in the block) gets weight 0.
 *
 * o_part, lse_part  one block's partial: o_part like q (fp16 / bf16, layout
 *                   `layout`, [B, S, H, D] or [B, H, S, D]), lse_part fp32
 *                   [B, H, S]; read only
 * o_acc, lse_acc    the running result in fp32: o_acc with o_part's shape and
 *                   layout, lse_acc [B, H, S].  Read when flags has
 *                   FA_MERGE_ACCUMULATE; written (in place) unless flags has
 *                   FA_MERGE_FINAL.  May be NULL when neither is needed
 *                   (flags == FA_MERGE_FINAL: a copy of the partial).
 * o_out, lse_out    written instead of o_acc / lse_acc when flags has
 *                   FA_MERGE_FINAL: o_out like o_part (rounded to nearest),
 *                   lse_out fp32 [B, H, S]; else unused (may be NULL)
 * flags             0: running result = the partial (the first block);
 *                   FA_MERGE_ACCUMULATE: running result merged with the partial;
 *                   adding FA_MERGE_FINAL writes the outcome to o_out / lse_out
 *
 * The caller owns every buffer.  16-byte alignment for o_part, o_acc, o_out;
 * 4-byte for the LSE arrays.  D must be 64 or 128.  Outputs must not overlap
 * any other array (FA_ERR_ALIAS), except that o_acc / lse_acc are updated in
 * place.  S = 0 is a no-op.  Other errors as for fa_fwd.  Asynchronous on
 * `stream`.
 */
enum { FA_MERGE_ACCUMULATE = 1, FA_MERGE_FINAL = 2 };
fa_status fa_lse_merge(const void *o_part, const float *lse_part, float *o_acc, float *lse_acc,
                       void *o_out, float *lse_out, int64_t B, int64_t H, int64_t S, int64_t D,
                       fa_layout layout, fa_dtype dtype, int flags, void *stream);

/*
 * fa_fwd_ring_step -- one step of ring attention in one launch.  Ring
 * attention (page "FlashAttention in ops-transformer on Ascend NPU"
 * (ai6s.net/6a0d3bfb), section "what else is in the ops-transformer
 * repository"; page "64K long-sequence FlashAttention" (ai6s.net/6a140d07),
 * section "performance tuning tips", multi-card parallelism) gives each rank,
 * at each step, one or two blocks of its query rows against the key/value
 * chunks it holds at that step.  This call attends every such block (a
 * "segment") and merges the result into the running result of its rows in
 * the attention kernel's epilogue -- the update fa_lse_merge applies, without
 * the partial result's round trip through memory:
 *     LSE = log(exp(LSE_run) + exp(LSE_seg))
 *     O   = exp(LSE_run - LSE) O_run + exp(LSE_seg - LSE) O_seg
 *
 * q, o     this rank's query rows and output: [B, Sq, H, D] (FA_BSND) or
 *          [B, H, Sq, D] (FA_BHSD), fp16 / bf16, 16-byte aligned
 * k, v     the key/value rows held at this step, Sk of them, same layout and
 *          dtype, 16-byte aligned; read only
 * lse      fp32 [B, H, Sq]: the running LSE (read where a segment has
 *          first = 0) and the merged LSE (written for every segment row)
 * acc      fp32 like o: the running O, read where first = 0 and written where
 *          last = 0; may be NULL when every segment has first = last = 1.
 *          16-byte aligned
 * rows     query rows per segment (the same for every segment)
 * segs     nseg (1 or 2) segments with disjoint row ranges; segment s covers
 *          query rows [row0, row0 + rows) and keys [key0, key0 + keys) of
 *          k / v.  causal_offset >= 0: key c of the segment (counted from
 *          key0) is visible from its row r (counted from row0) iff
 *          c <= r + causal_offset, so every row sees key 0; causal_offset < 0:
 *          every key is visible.  first = 1: the rows have no earlier result
 *          (acc and lse are not read); last = 1: the merged result is final
 *          and written to o in the input dtype (rounded to nearest), else to
 *          acc in fp32.
 *
 * The work is scheduled as one persistent launch over both segments' work
 * units (longest first); workspace as for fa_fwd_ws (fa_fwd_workspace_size
 * bytes, zeroed on `stream` by the call).  The caller owns every buffer;
 * acc and the workspace must not overlap any other buffer, and o / lse none
 * of the inputs (FA_ERR_ALIAS).  FA_ERR_INVALID_ARG for a segment outside
 * the tensors, overlapping segments, flags other than 0 / 1, or a missing
 * acc or workspace.  Other errors as for fa_fwd.  Asynchronous on `stream`.
 */
typedef struct fa_ring_segment {
  int64_t row0;           /* first query row of q / o / lse */
  int64_t key0;           /* first key row of k / v */
  int64_t keys;           /* keys attended, >= 1 */
  int64_t causal_offset;  /* < 0: no mask; >= 0: key c visible from row r iff c <= r + causal_offset */
  int32_t first;          /* 1: no running result yet */
  int32_t last;           /* 1: write the final output */
} fa_ring_segment;
fa_status fa_fwd_ring_step(const void *q, const void *k, const void *v, void *o, float *acc, float *lse,
                           int64_t B, int64_t H, int64_t Sq, int64_t Sk, int64_t D, int64_t rows,
                           const fa_ring_segment *segs, int nseg, fa_layout layout, float scale,
                           fa_dtype dtype, void *workspace, size_t workspace_bytes, void *stream);

/*
 * fa_fwd_splitkv -- the forward pass without a mask for problems with few
 * work units (few heads and query rows: a short prompt, or decoding against a
 * long key sequence), with the keys split across CTAs as well.  The key range
 * is cut into up to nsplit ranges of whole 128-key tiles; every (query rows,
 * key range) pair is a work unit of the ring-step kernel, which writes the
 * range's result normalised over its own keys (fp32 O and LSE, in the
 * workspace); a second kernel merges a row's partial results by the update
 * of fa_lse_merge taken over all of them at once (page "FlashAttention: long-
 * text inference without running out of memory" (ai6s.net/6a0d42d8), section
 * on tiling and online normalisation, applied to whole key ranges):
 *     LSE = log(sum_s exp(LSE_s)),  O = sum_s exp(LSE_s - LSE) O_s
 * and writes O (rounded to nearest in dtype) and LSE as fa_fwd does.  The
 * result equals fa_fwd's within rounding (the partial results are fp32), not
 * bit for bit.
 *
 * Arguments as for fa_fwd with causal = 0 (no mask is applied), plus
 * nsplit     1..64 requested key ranges (fewer when Sk has fewer 128-key tiles)
 * workspace  fa_fwd_splitkv_workspace_size(B, H, Sq, D, nsplit) bytes of
 *            caller-owned device memory, 256-byte aligned, not overlapping
 *            any tensor (FA_ERR_ALIAS); overwritten by the call
 * Errors as for fa_fwd_ws; FA_ERR_INVALID_ARG for nsplit outside 1..64 or a
 * missing or short workspace.  Asynchronous on `stream`.
 */
size_t fa_fwd_splitkv_workspace_size(int64_t B, int64_t H, int64_t Sq, int64_t D, int nsplit);
fa_status fa_fwd_splitkv(const void *q, const void *k, const void *v, void *o, float *lse, int64_t B, int64_t H,
                         int64_t Sq, int64_t Sk, int64_t D, fa_layout layout, float scale, fa_dtype dtype,
                         int nsplit, void *workspace, size_t workspace_bytes, void *stream);

/*
 * fa_out_proj -- the attention output projection Y = O W^T (page "catlass
 * FlashAttention template tuning" (hwcomputing.csdn.net/6a0d4681), section on
 * graph fusion: the fused operator FusedAttnProj is FlashAttention followed by
 * the output MatMul).  Every token's heads form one row of inputs:
 *     y[b, s, n] = sum_{h, d} o[b, s, h, d] * w_o[n, h * D + d]
 * fp32 accumulation on the tensor cores, y rounded to nearest in dtype.
 *
 * o      attention output as fa_fwd writes it: [B, S, H, D] (FA_BSND) or
 *        [B, H, S, D] (FA_BHSD), fp16 / bf16, 16-byte aligned; read only
 * w_o    [E, H * D] row-major (a linear layer's weight: row n is output
 *        feature n), same dtype, 16-byte aligned; read only
 * y      [B, S, E] row-major, same dtype, 16-byte aligned, fully overwritten
 * E      output features, a positive multiple of 32
 *
 * Caller-owned buffers; y must not overlap o or w_o (FA_ERR_ALIAS).  S = 0 is
 * a no-op.  D must be 64 or 128 and E a multiple of 32 (else
 * FA_ERR_UNSUPPORTED).  Other errors as for fa_fwd.  Asynchronous on `stream`.
 */
fa_status fa_out_proj(const void *o, const void *w_o, void *y, int64_t B, int64_t H, int64_t S, int64_t D,
                      int64_t E, fa_layout layout, fa_dtype dtype, void *stream);

/*
 * fa_fwd_proj -- attention followed by its output projection in one call:
 * fa_fwd_ws (or fa_fwd when workspace is NULL) writes o and lse, then
 * fa_out_proj writes y = o w_o^T, stream-ordered on `stream`.  Arguments as
 * for those two calls (Sq for S); o is caller-owned and also an output (the
 * attention result, kept for a backward pass).  y and w_o must not overlap
 * any other array.
 */
fa_status fa_fwd_proj(const void *q, const void *k, const void *v, const void *w_o, void *o, float *lse, void *y,
                      int64_t B, int64_t H, int64_t Sq, int64_t Sk, int64_t D, int64_t E, fa_layout layout,
                      int causal, float scale, fa_dtype dtype, void *workspace, size_t workspace_bytes,
                      void *stream);

/*
 * fa_device_status -- synchronises `stream`, then reads and clears the
 * library's device-side error word on the current device.  Returns FA_OK,
 * FA_ERR_TIMEOUT if a kernel stopped at a wait limit since the last call,
 * else FA_ERR_INVALID_ARG if a variable-length batch had invalid sequence
 * offsets (fa_fwd_varlen), or FA_ERR_CUDA if the synchronisation itself failed.
 */
fa_status fa_device_status(void *stream);

/* FA_OK if (D, dtype) is supported by fa_fwd, FA_ERR_UNSUPPORTED otherwise. */
fa_status fa_query_support(int64_t D, fa_dtype dtype);

/* Human-readable name of a status code (static storage; never NULL). */
const char *fa_status_string(fa_status status);

/* The cudaError_t / CUresult number behind the last FA_ERR_CUDA on this host thread (0 if none). */
int fa_last_cuda_error(void);

/* Library version: major * 10000 + minor * 100 + patch. */
int fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_FWD_H */
