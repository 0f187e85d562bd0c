/*
 * fa.h -- C ABI of the B200 (sm_100a) exact-attention library, libfa_sm100.so.
 *
 * The library computes exact scaled-dot-product attention
 *
 *     O = softmax(scale * Q K^T [+ causal mask]) V
 *
 * and its gradient, tile by tile with an online softmax, so that the N x N
 * score and probability matrices never reach HBM.  Sources:
 *   - "FlashAttention-2: Faster Attention with Better Parallelism and Work
 *     Partitioning" (abstract): exact attention, no approximation; memory
 *     linear in the sequence length; work split over sequence, batch and heads.
 *   - iplexlaw blog "FlashAttention-2 GPU work partitioning", section "Tiling
 *     preserves the attention calculation": tiles are staged on chip and an
 *     online softmax rescales running statistics and partial outputs so the
 *     blocks add up to the globally normalised result; section "Three changes
 *     improve GPU utilisation": fewer non-matmul operations (rescaling, bounds
 *     and causal-mask handling), parallelism along the sequence dimension.
 * The log-sum-exp output and the backward algorithm (recompute P from LSE,
 * D = rowsum(dO * O), fp32 reduction of dQ) are the standard gradient of the
 * definition; the pages name gradients and training but print no formula.
 *
 * Conventions shared by every entry point
 *   - Tensors are contiguous row-major [B, H, N, d] in bf16 (Q, K, V, O, dO,
 *     dQ, dK, dV); row (b, h, n) starts at element ((b*H + h)*N + n)*d.
 *     LSE is [B, H, N] fp32.  N_q = N_k = N.
 *   - Every pointer is a DEVICE pointer on the current CUDA device, 16-byte
 *     aligned (TMA requirement).  The caller owns every buffer; the library
 *     allocates no device memory and keeps no state beyond a per-device error
 *     word and one-time kernel attributes.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Work is enqueued asynchronously; no call synchronises the
 *     host except fa_get_device_error.
 *   - A status other than FA_OK means nothing was enqueued.
 *   - Supported: d in {64, 128}; N >= 1; B, H >= 1; B*H <= 2^24, N <= 2^30
 *     and B*H*ceil(N/256) < 2^31 (grid and TMA coordinates are 32-bit);
 *     element offsets are 64-bit, so a tensor may exceed 2^31 elements;
 *     scale finite and > 0.
 *     causal: key j is visible to query i iff j <= i.
 *   - Device-side waits are bounded (about 2 s).  A kernel whose pipeline wait
 *     runs out records FA_ERR_TIMEOUT in the device error word and returns
 *     early; fa_get_device_error reports it.
 */
#ifndef FA_SM100_H
#define FA_SM100_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FA_OK = 0,
    FA_ERR_INVALID_ARG = 1,  /* null pointer, bad size, non-finite/<=0 scale */
    FA_ERR_UNSUPPORTED = 2,  /* d not in {64,128}, or no sm_100 device       */
    FA_ERR_MISALIGNED = 3,   /* a pointer is not 16-byte aligned             */
    FA_ERR_CUDA = 4,         /* a CUDA runtime/driver call failed            */
    FA_ERR_TIMEOUT = 5       /* a device-side pipeline wait ran out          */
} fa_status;

/*
 * fa_fwd -- forward pass.
 *   q, k, v  [B,H,N,d] bf16, read only.
 *   o        [B,H,N,d] bf16, written: O_i = sum_j P_ij v_j.
 *   lse      [B,H,N] fp32, written: LSE_i = ln sum_{j visible} exp(scale q_i.k_j)
 *            (natural log), the statistic fa_bwd consumes.
 *   causal   0: none; 1: key j visible to query i iff j <= i; 2: iff j < i
 *            (the causal mask without its diagonal, for the pairs of a
 *            striped ring whose key shard comes later in the sequence; row 0
 *            then sees no key and gets O = 0, LSE = -inf).
 *   scale    multiplies Q K^T (commonly 1/sqrt(d)).
 * Cites: FlashAttention-2 abstract (exact attention, tiled, sequence-parallel);
 * iplexlaw blog, "Tiling preserves the attention calculation" (online softmax).
 * Errors: FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_MISALIGNED,
 * FA_ERR_CUDA (launch failure).  o and lse may not alias the inputs.
 */
fa_status fa_fwd(const void* q, const void* k, const void* v, void* o,
                 float* lse, int B, int H, int N, int d, int causal,
                 float scale, void* stream);

/*
 * fa_fwd_qk8 -- forward pass with 8-bit float scores (low-precision attention
 * on Blackwell tensor cores, in the manner of SageAttention, whose
 * Blackwell work the pages cite: the QK^T product is quantised, P V stays in
 * 16 bits).
 *   q, k     [B,H,N,d] e4m3 (1 byte per element, OCP FP8 E4M3), read only,
 *            with per-tensor dequantisation factors q_descale, k_descale
 *            (finite, > 0): the attention is that of q_descale * q and
 *            k_descale * k.
 *   v        [B,H,N,d] bf16.  o, lse as fa_fwd.
 * S = Q K^T runs as tcgen05.mma kind::f8f6f4 (e4m3 x e4m3, fp32 accumulate,
 * exact products) at twice the bf16 rate; the descales fold into the softmax
 * scale; P is rounded to bf16 for P V exactly as in fa_fwd.  For inputs that
 * are e4m3 values, the result is fa_fwd's on the dequantised Q and K, within
 * the same tolerances.  Supported: d = 128.  Other conventions and errors as
 * fa_fwd (FA_ERR_UNSUPPORTED for d != 128).
 */
fa_status fa_fwd_qk8(const void* q, const void* k, const void* v,
                     float q_descale, float k_descale, void* o, float* lse,
                     int B, int H, int N, int d, int causal, float scale,
                     void* stream);

/*
 * fa_fwd_fp8 -- forward pass with both products in 8-bit floats (the next
 * step of the low-precision attention on Blackwell tensor cores the pages
 * cite): Q, K and V are e4m3, S = Q K^T and O += P V both run as
 * tcgen05.mma kind::f8f6f4.
 *   q, k, v  [B,H,N,d] e4m3 (OCP FP8 E4M3), read only, with per-tensor
 *            dequantisation factors q_descale, k_descale, v_descale (finite,
 *            > 0): the attention is that of the dequantised tensors.
 *   o        [B,H,N,d] bf16, written; lse as fa_fwd.
 * P is scaled by 2^6 and rounded to e4m3 in the softmax (the running maximum
 * is refreshed once a row's scores exceed it by 2 in log2 units, so the
 * scaled weights stay below e4m3's 448), and O is normalised by the sum of
 * the rounded weights, so O is an exact convex combination of V rows under
 * weights that each carry up to 2^-4 relative rounding (2^-3 after
 * normalising).  LSE uses the unrounded fp32 weights, as in fa_fwd.
 * Contract, per element, against the definition on the dequantised inputs:
 *   |O - O_ref| <= 2^-3 * sum_j P_ij |v_j - O_ref,i| + 2^-8 |O_ref| + 4e-3,
 *   relative L2 of O <= 6e-2, LSE max-abs <= 1e-3.
 * Supported: d = 128, causal 0 or 1.  Other conventions and errors as
 * fa_fwd_qk8 (FA_ERR_INVALID_ARG for a descale that is not finite and > 0).
 */
fa_status fa_fwd_fp8(const void* q, const void* k, const void* v,
                     float q_descale, float k_descale, float v_descale, void* o,
                     float* lse, int B, int H, int N, int d, int causal,
                     float scale, void* stream);

/*
 * Attention with an additive score bias: S_ij = scale * q_i.k_j + b_ij
 * (a prior added to the query-key scores, the "attention with bias" of
 * vision, language and protein-folding models that the pages cite), before
 * the causal mask and the softmax.
 *
 * fa_fwd_bias -- fa_fwd with a bias.
 *   bias     [Bb, Hb, N, N] bf16, read only: Bb = B if bias_batch else 1,
 *            Hb = H if bias_heads else 1 (a bias shared by the batch and/or
 *            the heads, e.g. a relative-position bias).  Row i, column j is
 *            the bias of query i and key j.  Each row needs at least one
 *            finite biased score among its visible keys (a bias of -inf
 *            masks a key).
 *   lse      includes the bias: LSE_i = ln sum_j exp(scale q_i.k_j + b_ij).
 *   Needs N % 8 == 0 (each bias row a multiple of 16 bytes), else
 *   FA_ERR_UNSUPPORTED.  Other arguments, conventions and errors as fa_fwd.
 */
fa_status fa_fwd_bias(const void* q, const void* k, const void* v,
                      const void* bias, void* o, float* lse, int B, int H,
                      int N, int d, int bias_batch, int bias_heads, int causal,
                      float scale, void* stream);

/*
 * fa_bwd_bias -- fa_bwd for fa_fwd_bias (same bias, flags, causal, scale),
 *   recomputing P = exp(scale q.k + b - LSE).
 *   dbias    [B, H, N, N] bf16, or NULL: receives the gradient of the bias,
 *            dS_ij = P_ij (dP_ij - D_i), for every batch and head (sum it over
 *            the batch / heads yourself when the bias is shared).  With the
 *            causal mask the hidden entries are written as 0.
 *   The other arguments, the workspace, conventions and errors are those of
 *   fa_bwd; N % 8 == 0 as for fa_fwd_bias.
 */
fa_status fa_bwd_bias(const void* q, const void* k, const void* v,
                      const void* bias, const void* o, const float* lse,
                      const void* dO, void* dq, void* dk, void* dv, void* dbias,
                      int B, int H, int N, int d, int bias_batch, int bias_heads,
                      int causal, float scale, void* workspace,
                      size_t workspace_bytes, void* stream);

/*
 * fa_bwd_workspace_size -- bytes of device workspace fa_bwd needs:
 * an fp32 dQ accumulator [B,H,Npad,d] plus two fp32 row vectors [B,H,Npad]
 * (log2-scaled LSE and D = rowsum(dO * O)), Npad = N rounded up to 128.
 * Linear in N (FlashAttention-2 abstract: memory linear, not quadratic).
 * Returns 0 for invalid sizes.
 */
size_t fa_bwd_workspace_size(int B, int H, int N, int d);

/*
 * fa_bwd -- backward pass.
 *   q, k, v, o, lse   as passed to / produced by one fa_fwd call (same
 *                     causal and scale).
 *   dO                [B,H,N,d] bf16 upstream gradient, read only.
 *   dq, dk, dv        [B,H,N,d] bf16, overwritten (not accumulated).
 *   workspace         device buffer of >= fa_bwd_workspace_size(B,H,N,d)
 *                     bytes, 256-byte aligned; contents need no
 *                     initialisation and are clobbered.
 * causal as for fa_fwd (0, 1 or 2).
 * Three launches on `stream`: preprocess (D, log2 LSE, zero dQ accumulator),
 * the main kernel (one CTA per key block; recomputes P from LSE; dK, dV per
 * key block; dQ by fp32 reduction), and the dQ conversion to bf16.
 * dQ is not bitwise deterministic (fp32 reduction order varies); dK and dV are.
 * Cites: iplexlaw blog, "Tiling preserves the attention calculation" (gradient
 * comparisons within tolerances) and "Why long inputs put pressure on memory"
 * (the N x N matrices are not stored, so P is recomputed); the gradient
 * formulas themselves are not on the pages (textbook softmax calculus).
 * Errors: as fa_fwd, plus FA_ERR_INVALID_ARG when the workspace is too small.
 */
fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o,
                 const float* lse, const void* dO, void* dq, void* dk,
                 void* dv, int B, int H, int N, int d, int causal, float scale,
                 void* workspace, size_t workspace_bytes, void* stream);

/*
 * The three stages fa_bwd runs, callable one by one on the same workspace
 * (for example to time the main kernel alone).  Same conventions as fa_bwd;
 * each returns FA_OK after enqueueing its launch.
 *
 * fa_bwd_preprocess -- D_i = sum_d dO_id * O_id (fp32), LSE_i * log2(e), and a
 *   zeroed fp32 dQ accumulator, all in `workspace`.  Reads o, lse, dO.
 */
fa_status fa_bwd_preprocess(const void* o, const float* lse, const void* dO,
                            int B, int H, int N, int d, void* workspace,
                            size_t workspace_bytes, void* stream);

/*
 * fa_bwd_main -- one CTA per (b, h, 128-row key block): recomputes P from the
 *   stored LSE, writes dK (times scale) and dV in bf16, and reduce-adds the
 *   unscaled dQ into the workspace accumulator.  Needs fa_bwd_preprocess's
 *   workspace contents.
 */
fa_status fa_bwd_main(const void* q, const void* k, const void* v,
                      const void* dO, void* dk, void* dv, int B, int H, int N,
                      int d, int causal, float scale, void* workspace,
                      size_t workspace_bytes, void* stream);

/*
 * fa_bwd_dq_convert -- dq = bf16(scale * accumulator).  Needs fa_bwd_main's
 *   workspace contents.
 */
fa_status fa_bwd_dq_convert(void* dq, int B, int H, int N, int d, float scale,
                            void* workspace, size_t workspace_bytes,
                            void* stream);

/*
 * Sequence sharding across devices (Ring Attention with Blockwise
 * Transformers, abstract: each device keeps its query block while key/value
 * blocks travel around a ring of devices, overlapped with the blockwise
 * attention).  Each (query shard, key/value shard) pair is an ordinary
 * fa_fwd / fa_bwd problem of the shard length; the calls below fold the
 * pairs' results together.
 *
 * fa_lse_merge -- fold one partial attention result into a running one.
 *   o_acc    [rows, d] fp32, read unless init, written: the running O.
 *   lse_acc  [rows] fp32 (natural log), likewise: the running LSE.
 *   o_part   [rows, d] bf16 and lse_part [rows] fp32: attention of the same
 *            query rows over a key set disjoint from the ones already folded
 *            in (as fa_fwd writes them).
 *   o_out    [rows, d] bf16 or NULL: receives bf16(merged O) as well.
 *   init     1: the accumulator takes the partial as it is; 0: merge,
 *            O = (w_a O_acc + w_b O_part) / (w_a + w_b), w = exp(LSE - max),
 *            LSE = max + log(w_a + w_b) (the online-softmax rescaling of
 *            iplexlaw blog "Tiling preserves the attention calculation").
 *   rows = number of query rows (e.g. B*H*N), d in {64, 128}.
 * Errors: FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_MISALIGNED,
 * FA_ERR_CUDA.
 */
fa_status fa_lse_merge(float* o_acc, float* lse_acc, const void* o_part,
                       const float* lse_part, void* o_out, long long rows,
                       int d, int init, void* stream);

/*
 * fa_bwd_main_accumulate -- fa_bwd_main that ADDS its dK (times scale) and
 * dV to fp32 accumulators instead of writing bf16: dk_acc, dv_acc
 * [B,H,N,d] fp32, 16-byte aligned, read-modify-written by bulk reductions.
 * With a workspace prepared by fa_bwd_preprocess from the FINAL O and LSE
 * of the query rows (over all key shards), calling it once per key/value
 * shard accumulates dQ (in the workspace) and each shard's dK, dV exactly as
 * the gradient over the union of the shards; fa_bwd_dq_convert then yields
 * dQ.  causal 0, 1 or 2 as for fa_fwd.  Other arguments and errors as
 * fa_bwd_main.
 */
fa_status fa_bwd_main_accumulate(const void* q, const void* k, const void* v,
                                 const void* dO, float* dk_acc, float* dv_acc,
                                 int B, int H, int N, int d, int causal,
                                 float scale, void* workspace,
                                 size_t workspace_bytes, void* stream);

/*
 * fa_convert_f32_bf16 -- dst[i] = bf16(src[i]) (round to nearest even) for
 * n elements, n a positive multiple of 8; both 16-byte aligned.
 */
fa_status fa_convert_f32_bf16(const float* src, void* dst, long long n,
                              void* stream);

/*
 * fa_bwd_noalloc -- fa_bwd for callers that cannot allocate device memory.
 * (No counterpart in the paper; it is a packaging choice of this library.)
 *   Some callers have no way to hand fa_bwd a workspace: a plugin inside a host
 *   application that owns all device memory through its own pool and gives
 *   extensions no allocator, or a serving path that forbids cudaMalloc after
 *   start-up because it can synchronise the device and take driver locks.
 *   This entry point takes the same arguments as fa_bwd minus the workspace
 *   and uses a fixed scratch array of FA_BWD_NOALLOC_MAX_WORKSPACE_BYTES that
 *   the library reserves, at load, on every GPU that loads it (held until the
 *   process exits).  It calls no allocator itself.
 *   - Problems whose fa_bwd_workspace_size exceeds that maximum are rejected
 *     with FA_ERR_INVALID_ARG before anything is enqueued (d outside {64, 128}
 *     gives FA_ERR_UNSUPPORTED).
 *   - The first call on a device looks up the scratch array's device address
 *     (a one-time set-up per device, done with that device current); make
 *     that first call before any stream capture.
 *   - All calls on a device share the one array, which keeps whatever the
 *     last call left in it; each call rewrites what it reads before reading
 *     it.  Calls whose GPU work overlaps (e.g. on two streams without
 *     ordering between them) race on the array and give wrong results:
 *     order them on one stream or with events.
 *   Other conventions, outputs and errors are those of fa_bwd.
 */
#define FA_BWD_NOALLOC_MAX_WORKSPACE_BYTES ((size_t)64 << 20)
fa_status fa_bwd_noalloc(const void* q, const void* k, const void* v,
                         const void* o, const float* lse, const void* dO,
                         void* dq, void* dk, void* dv, int B, int H, int N,
                         int d, int causal, float scale, void* stream);

/*
 * Decoding: N_q query rows against N_k >= N_q cached keys, N_q small.
 * iplexlaw blog "FlashAttention-2 GPU work partitioning", section "What the
 * paper measures": prefill and token-by-token decoding have different
 * bottlenecks and are measured apart.  Decoding reads every cached key and
 * value once for a few query rows, so it is bound by HBM bandwidth; the key
 * range is split across CTAs ("split-KV") and the partial results merged
 * with the log-sum-exp rule of the online softmax ("Tiling preserves the
 * attention calculation").
 *
 * fa_fwd_decode -- O = softmax(scale * Q K^T [+ causal mask]) V for
 *   q        [B,H,Nq,d] bf16, read only.
 *   k, v     [B,H,kv_rows,d] bf16, read only; the first Nk rows of every
 *            head are the keys (a cache allocated for kv_rows >= Nk rows).
 *   o        [B,H,Nq,d] bf16, written.
 *   lse      [B,H,Nq] fp32, written: natural-log LSE over the visible keys.
 *   causal   0 or 1.  The query rows are the LAST Nq positions of the
 *            sequence: query i (0-based) sees key j iff j <= i + Nk - Nq
 *            (needs Nk >= Nq); for Nq = Nk this is fa_fwd's mask.
 *   workspace  device buffer of >= fa_decode_workspace_size(B,H,Nq,Nk,d)
 *            bytes, 256-byte aligned, clobbered; may be NULL when that size
 *            is 0 (Nk <= 256).
 * Arithmetic: fp32 scores, weights and accumulation from the bf16 inputs.
 * Intended for Nq <= 16 (query rows are handled four at a time, and every
 * group of four re-reads the keys, mostly from L2); any Nq >= 1 is correct.
 * One launch, plus a merge launch when the keys were split.
 * Errors: as fa_fwd; FA_ERR_INVALID_ARG also for kv_rows < Nk, causal with
 * Nk < Nq, or a missing / too small workspace.
 */
size_t fa_decode_workspace_size(int B, int H, int Nq, int Nk, int d);
fa_status fa_fwd_decode(const void* q, const void* k, const void* v, void* o,
                        float* lse, int B, int H, int Nq, int Nk,
                        long long kv_rows, int d, int causal, float scale,
                        void* workspace, size_t workspace_bytes, void* stream);

/*
 * fa_decode_split_plan -- the work split fa_fwd_decode uses on a GPU with
 * `sm_count` SMs that holds `ctas_per_sm` decode CTAs each: query rows per
 * CTA (1, 2 or 4), the number of key splits per head, and the keys per split
 * (a multiple of 64, at least 256 when the keys are split).  Host
 * arithmetic only; touches no GPU.  Errors: FA_ERR_INVALID_ARG /
 * FA_ERR_UNSUPPORTED for sizes fa_fwd_decode would reject.
 */
fa_status fa_decode_split_plan(int B, int H, int Nq, int Nk, int d,
                               int sm_count, int ctas_per_sm,
                               int* qgroup_rows, int* n_splits, int* chunk);

/*
 * fa_get_device_error -- synchronises `stream`, then reads and clears the
 * current device's error word.  Returns FA_ERR_TIMEOUT if a kernel's bounded
 * pipeline wait ran out since the last call, FA_ERR_CUDA if the stream
 * reports a CUDA error, FA_OK otherwise.
 * Cites: not on the pages (failure reporting of this library).
 */
fa_status fa_get_device_error(void* stream);

/*
 * fa_selftest_wait_timeout -- exercises the failure path of the bounded
 * device waits without faulting or hanging the GPU: enqueues one tiny kernel
 * whose single wait, on an mbarrier that nothing arrives on, runs out after
 * `limit_us` microseconds (1 .. 2,000,000) and records FA_ERR_TIMEOUT in the
 * device error word, exactly as a stalled attention pipeline would.  The
 * following fa_get_device_error(stream) returns FA_ERR_TIMEOUT (and clears
 * the word); the context stays usable.  Errors: FA_ERR_INVALID_ARG for a
 * limit out of range, FA_ERR_UNSUPPORTED / FA_ERR_CUDA as for fa_fwd.
 * Cites: not on the pages (a test hook of this library's failure path).
 */
fa_status fa_selftest_wait_timeout(unsigned int limit_us, void* stream);

/* fa_strerror -- static, human-readable name of a status.
 * Cites: not on the pages. */
const char* fa_strerror(fa_status status);

#ifdef __cplusplus
}
#endif

#endif /* FA_SM100_H */
