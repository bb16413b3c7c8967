/*
 * lsh_attn.h -- C ABI of the LSH self-attention library (shared query-key,
 * forward and backward) for NVIDIA B200 (sm_100a).
 *
 * The operation is Reformer's LSH attention as described in the paper note
 * "Reformer" (eightmm.github.io, on Kitaev, Kaiser, Levskaya, "Reformer: The
 * Efficient Transformer", ICLR 2020):
 *   - section "LSH Attention": hash h(x) into buckets, candidate set
 *     N_LSH(i) = {j : h(q_i) = h(k_j)}, output
 *     y_i = sum_{j in N(i)} softmax_j(q_i . k_j / sqrt(d_k)) v_j;
 *   - section "Shared Query-Key Space": Q = K;
 *   - section "Sorting and Chunking": hash -> sort by bucket -> attention in
 *     chunks of nearby sorted positions;
 *   - section "Multiple Hash Rounds": N(i) is the union over R rounds;
 *   - section "Implementation Reading": the causal mask must survive the
 *     sort; whether a token may attend to its own position.
 *
 * Where the note leaves a step open this library fixes it as follows:
 *   hash      bucket = argmax over the n_buckets-vector [x R_r ; -x R_r]
 *             (0-based; the lowest index wins an exact tie), x as stored;
 *   sort      stable: inside a bucket, original positions increase;
 *   chunks    sorted slots are cut into chunks of `chunk`; a query in chunk
 *             c attends to the slots of chunks c-1 and c (chunk 0: itself
 *             only); there is no bucket-equality mask inside that window;
 *   keys      k_j = x_j / |x_j| (k_j = 0 when |x_j| = 0); queries are x_i as
 *             stored; scores are q_i . k_j / sqrt(d);
 *   self      a query never attends to its own position unless no other
 *             candidate is left, in which case it attends to itself alone;
 *   causal    key position <= query position, on ORIGINAL positions;
 *   rounds    y_i = sum_r softmax_r(lse_r,i) o_r,i, where o_r and lse_r are
 *             round r's output and natural-log logsumexp;
 *   backward  gradients w.r.t. x (query and key role) and v with the
 *             bucket assignment held fixed (it is piecewise constant);
 *             no gradient w.r.t. R.
 *
 * Conventions shared by every entry point
 *   - Every tensor argument is a DEVICE pointer owned by the caller,
 *     16-byte aligned, contiguous, row-major:
 *       qk, v, out, dout, dqk, dv   [B, H, L, d]      element type = dtype
 *       R                           [n_hashes, d, n_buckets/2], dtype,
 *                                   shared by every batch row and head
 *       lse                         [B, H, n_hashes, L]   float32
 *       perm                        [B, H, n_hashes, L]   int32: perm[s] is
 *                                   the original position at sorted slot s
 *       buckets                     [B, H, n_hashes, L]   uint16
 *   - workspace: a caller-owned device buffer of at least
 *     lsh_attn_workspace_size() bytes, 256-byte aligned.  The library never
 *     allocates or frees memory.  One workspace must not be used by two
 *     calls that may run at the same time.
 *   - stream: a cudaStream_t (NULL = legacy default stream).  Every call is
 *     asynchronous on that stream; arguments are checked on the host before
 *     anything is launched, so an error status means nothing was launched,
 *     except LSH_ERR_CUDA, which reports a launch failure.
 *   - Which kernels run is fixed by the dtype, never chosen at run time:
 *     fp32 inputs run on CUDA cores in fp32 (no TF32), any chunk with
 *     L % chunk == 0; bf16 inputs run on the tensor cores (bf16 operands,
 *     fp32 accumulation) and require chunk == 64 and L % 64 == 0.  A bf16
 *     descriptor outside that envelope is refused with LSH_ERR_UNSUPPORTED
 *     before anything is launched; there is no slower substitute path.
 *     d must be 64 for both.
 */
#ifndef LSH_ATTN_H
#define LSH_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define LSH_ATTN_ABI_VERSION 3

#if defined(__GNUC__)
#define LSH_API __attribute__((visibility("default")))
#else
#define LSH_API
#endif

typedef enum {
    LSH_OK = 0,
    LSH_ERR_ARG = -1,          /* null pointer or unknown enum value            */
    LSH_ERR_SHAPE = -2,        /* sizes inconsistent (e.g. L % chunk != 0)      */
    LSH_ERR_ALIGN = -3,        /* a pointer is not 16-byte aligned              */
    LSH_ERR_UNSUPPORTED = -4,  /* valid request outside what the kernels run     */
                               /* (d != 64; bf16 with chunk != 64 or L % 64 != 0) */
    LSH_ERR_CUDA = -5,         /* a CUDA launch or runtime call failed          */
    LSH_ERR_TIMEOUT = -6,      /* a bounded device-side wait gave up            */
    LSH_ERR_WORKSPACE = -7     /* workspace smaller than required               */
} lsh_status;

typedef enum { LSH_F32 = 0, LSH_BF16 = 1 } lsh_dtype;

/* Optional semantics (lsh_attn_desc.flags, bitwise OR; 0 = the defaults above).
 *   LSH_FLAG_BUCKET_MASK   strict candidate set of section "LSH Attention",
 *                          N_LSH(i) = {j : h(q_i) = h(k_j)}: inside the chunk
 *                          window a key is a candidate only if it shares the
 *                          query's bucket in that round.
 *   LSH_FLAG_SELF_PENALTY  the other answer to the same-token question of
 *                          "Implementation Reading": the query's own position is
 *                          always a candidate, with the fixed score
 *                          LSH_SELF_PENALTY_SCORE in place of q_i . k_i / sqrt(d),
 *                          so it carries weight only when nothing else is left.
 * Unknown bits are rejected with LSH_ERR_ARG. */
#define LSH_FLAG_BUCKET_MASK 1
#define LSH_FLAG_SELF_PENALTY 2
#define LSH_SELF_PENALTY_SCORE (-1.0e5f)

typedef struct {
    int32_t B, H, L, d;      /* batch, heads, sequence length, head dim (64)   */
    int32_t n_buckets;       /* even, 2 .. 65536                               */
    int32_t n_hashes;        /* rounds R >= 1                                  */
    int32_t chunk;           /* chunk length m >= 1, L % m == 0                */
    int32_t causal;          /* 0 or 1                                         */
    int32_t dtype;           /* lsh_dtype                                      */
    int32_t flags;           /* LSH_FLAG_* bits, 0 for the default semantics   */
} lsh_attn_desc;

/* Random rotations on the HOST ("LSH Attention": one random rotation per
 * round, entries N(0, 1)): fills R_host[n_hashes, d, n_buckets/2] (float32, or
 * bfloat16 bits as uint16 when desc->dtype is LSH_BF16; caller-owned host
 * memory of n_hashes * d * n_buckets/2 elements) from `seed` with
 * Philox4x32-10 and the Box-Muller transform, rounded to float32 and then,
 * for bf16, to bfloat16 (nearest, ties to even).  The same seed always gives
 * the same rotations.  Only the descriptor's dtype, d, n_buckets and n_hashes
 * are used.  Errors: LSH_ERR_ARG (null pointer, unknown dtype), LSH_ERR_SHAPE
 * (n_buckets odd, < 2 or > 65536; d or n_hashes < 1).  Nothing runs on the
 * device. */
LSH_API lsh_status lsh_attn_make_rotations(uint64_t seed, const lsh_attn_desc *desc, void *R_host);

/* Bytes of workspace needed by lsh_attn_fwd (for_backward = 0) or by
 * lsh_attn_bwd (for_backward = 1; includes what a recomputed hash and sort
 * need when perm is NULL).  Returns 0 for an invalid descriptor. */
LSH_API size_t lsh_attn_workspace_size(const lsh_attn_desc *desc, int for_backward);

/* Hash stage ("LSH Attention", hash equation): buckets[b,h,r,i] =
 * argmax([x_i R_r ; -x_i R_r]) for every round r. */
LSH_API lsh_status lsh_attn_hash(const lsh_attn_desc *desc, const void *qk, const void *R,
                         uint16_t *buckets, void *workspace, size_t ws_bytes, void *stream);

/* Sort stage ("Sorting and Chunking"): for every (b, h, r) segment, a stable
 * segmented radix sort of positions by bucket id; writes perm. */
LSH_API lsh_status lsh_attn_sort(const lsh_attn_desc *desc, const uint16_t *buckets, int32_t *perm,
                         void *workspace, size_t ws_bytes, void *stream);

/* Upper bound on the scratch that lsh_attn_sort_static can use (bytes, per
 * device). */
#define LSH_ATTN_SORT_STATIC_MAX_BYTES ((size_t)16 << 20)

/* Allocation-free sort.  The paper has no counterpart: it is a library
 * convenience, not a step of the method.  It computes exactly what
 * lsh_attn_sort computes (same kernels, same perm), but takes no workspace:
 * its scratch (first-pass keys and positions, per-tile digit counters) lives
 * in one fixed device array of LSH_ATTN_SORT_STATIC_MAX_BYTES per device,
 * which is part of the library's static device memory.
 *
 * Who needs it: a caller that must not allocate device memory when it sorts,
 * or has no allocator at hand.  Examples: code that runs inside a memory
 * pool's own callbacks (allocating there would re-enter the pool), a service
 * that fixes its memory footprint at start-up and forbids allocation
 * afterwards, or a plain C caller that holds device pointers handed to it by
 * another component but no way to obtain a workspace.  The call makes no
 * cudaMalloc/cudaFree and calls no library that allocates.
 *
 * Set-up: every call looks up the array's device address on the current
 * device (cudaGetSymbolAddress); nothing is cached, so a device reset or a
 * different current context leaves no stale address behind.  The first call
 * on a device may make the CUDA runtime load the library's device code, so
 * make it before any stream capture begins.
 *
 * Sizes: the scratch needed grows with B*H*n_hashes*L (6 bytes per position
 * when n_buckets > 256, plus a few counters per 2048 positions).  A
 * descriptor that needs more than LSH_ATTN_SORT_STATIC_MAX_BYTES is rejected
 * with LSH_ERR_WORKSPACE before anything is launched, and
 * lsh_attn_last_error() names the bytes needed and the limit; use
 * lsh_attn_sort with a workspace for such sizes.  Other argument errors are
 * those of lsh_attn_sort.
 *
 * Nothing in the scratch needs to start at zero: every pass writes each
 * counter and each slot before reading it.
 *
 * Concurrency: all calls on one device share the same array.  Two calls
 * whose kernels can overlap in time (different streams without ordering
 * between them, or different host threads on unordered streams) race on it
 * and produce wrong permutations.  Issue calls on one device in stream order.
 */
LSH_API lsh_status lsh_attn_sort_static(const lsh_attn_desc *desc, const uint16_t *buckets, int32_t *perm,
                                        void *stream);

/* Attention + round merge for a GIVEN permutation ("LSH Attention" output
 * equation, "Multiple Hash Rounds"): gathers rows in sorted order, runs the
 * chunked attention of every round, merges the rounds into out, and writes
 * the per-round logsumexp lse in original order.  perm must hold, for every
 * segment, a permutation of 0..L-1.  Entries outside [0, L) are ignored
 * and reported by lsh_attn_poll (LSH_ERR_ARG); a repeated entry is not
 * detected and gives undefined values at the positions involved. */
LSH_API lsh_status lsh_attn_fwd_sorted(const lsh_attn_desc *desc, const void *qk, const void *v,
                               const int32_t *perm, void *out, float *lse,
                               void *workspace, size_t ws_bytes, void *stream);

/* Full forward: hash, sort, attention, merge.  perm_out (nullable) receives
 * the permutation so that lsh_attn_bwd need not recompute it.
 *
 * Where a (batch, head, round) segment fits on chip (bf16, L <= 4096,
 * n_buckets <= 128, n_hashes <= 8; see lsh_attn_fused_forward_fits) the four
 * steps run as one kernel, one cluster of n_hashes CTAs per head ("Sorting and
 * Chunking": hash -> sort -> chunked attention with no HBM round trip for the
 * bucket ids, the permutation or the key norms; the rounds are merged inside
 * the cluster).  Its results are those of the staged kernels: the same
 * products, the same argmax tie rule, the same merge arithmetic. */
LSH_API lsh_status lsh_attn_fwd(const lsh_attn_desc *desc, const void *qk, const void *v, const void *R,
                        void *out, float *lse, int32_t *perm_out,
                        void *workspace, size_t ws_bytes, void *stream);

/* Backward of lsh_attn_fwd: given out, lse (from the forward) and dout,
 * writes dqk and dv.  perm may be NULL, in which case hash and sort are
 * recomputed from qk and R (R is ignored when perm is given). */
LSH_API lsh_status lsh_attn_bwd(const lsh_attn_desc *desc, const void *qk, const void *v, const void *R,
                        const void *out, const float *lse, const int32_t *perm, const void *dout,
                        void *dqk, void *dv, void *workspace, size_t ws_bytes, void *stream);

/* Local (non-hashed) chunk attention: the local self-attention of the page
 * "The Reformer - Pushing the limits of language modeling" (section "Approach
 * / What changed": input cut into chunks that attend with a preceding and a
 * following overlap).  No hashing or sort: positions keep their own order,
 * cut into chunks of desc->chunk, and a query in chunk c attends to chunks
 * c - 1, c and, when chunks_after = 1, c + 1, with the keys, self rule,
 * causal mask and self penalty of the LSH path (chunks_after = 0 is the LSH
 * window on unsorted positions; under the causal mask the following chunk
 * holds no candidate, so both values give the same result).
 *   desc      n_hashes must be 1; n_buckets is not used; LSH_FLAG_BUCKET_MASK
 *             is refused (LSH_ERR_ARG); the dtype envelope is that of
 *             lsh_attn_fwd.
 *   chunks_after  0 or 1 (other values: LSH_ERR_UNSUPPORTED).
 *   lse       [B, H, 1, L] float32: the logsumexp over the whole window.
 *   workspace at least lsh_attn_local_workspace_size() bytes, 256-byte aligned.
 * The backward takes out and lse from the forward and writes dqk, dv.
 * Errors and conventions as for lsh_attn_fwd / lsh_attn_bwd. */
LSH_API size_t lsh_attn_local_workspace_size(const lsh_attn_desc *desc, int32_t chunks_after, int for_backward);
LSH_API lsh_status lsh_attn_local_fwd(const lsh_attn_desc *desc, int32_t chunks_after, const void *qk,
                                      const void *v, void *out, float *lse, void *workspace, size_t ws_bytes,
                                      void *stream);
LSH_API lsh_status lsh_attn_local_bwd(const lsh_attn_desc *desc, int32_t chunks_after, const void *qk,
                                      const void *v, const void *out, const float *lse, const void *dout,
                                      void *dqk, void *dv, void *workspace, size_t ws_bytes, void *stream);

/* Reversible residual block with LSH attention as its first function
 * (paper note "Reformer", section "Reversible Residual Layers"):
 *   forward   y1 = x1 + F(x2),  y2 = x2 + G(y1)
 *   backward  from the OUTPUTS: x2 = y2 - G(y1), x1 = y1 - F(x2), so the
 *             block's inputs need not be kept; gradients
 *             dx1 = dy1 + J_G(y1)^T dy2,  dx2 = dy2 + J_F(x2)^T dx1.
 * F(x2) is LSH attention with x2 as both the shared query-key and the value
 * (hash, sort, chunked attention, round merge: the semantics of lsh_attn_fwd
 * with this descriptor; R as there).  G is the token-wise layer
 * G(u) = tanh(u Wg + bg), Wg [64, 64] row-major (input row, output column),
 * bg [64], float32.  x1, x2, y1, y2, dy1, dy2, dx1, dx2 are float32 [B, H, L,
 * 64] device buffers: the residual streams stay in fp32 so that the inverse
 * recovers x2 to fp32 rounding and F hashes it into the same buckets; F runs
 * in desc->dtype (x2 is rounded to it on the way in).  The backward returns
 * the recovered inputs in x1, x2 and the input gradients in dx1, dx2 (no
 * gradient for Wg, bg or R).  Workspace: lsh_rev_workspace_size() bytes,
 * 256-byte aligned.  Errors as for lsh_attn_fwd / lsh_attn_bwd. */
LSH_API size_t lsh_rev_workspace_size(const lsh_attn_desc *desc, int for_backward);
LSH_API lsh_status lsh_rev_fwd(const lsh_attn_desc *desc, const float *x1, const float *x2, const void *R,
                               const float *Wg, const float *bg, float *y1, float *y2, void *workspace,
                               size_t ws_bytes, void *stream);
LSH_API lsh_status lsh_rev_bwd(const lsh_attn_desc *desc, const float *y1, const float *y2, const float *dy1,
                               const float *dy2, const void *R, const float *Wg, const float *bg, float *x1,
                               float *x2, float *dx1, float *dx2, void *workspace, size_t ws_bytes, void *stream);

/* Forward, and backward when dout_h is given, on HOST buffers (the layouts of
 * lsh_attn_fwd / lsh_attn_bwd; qk_h, v_h, R_h, dout_h in; out_h, lse_h
 * (nullable), dqk_h, dv_h out).  The computation is that of lsh_attn_fwd
 * followed by lsh_attn_bwd with the forward's permutation.  The (batch, head)
 * slices are independent, so they are processed in chunks of heads_per_chunk
 * consecutive slices (<= 0: about an eighth of B*H, at least 1) through two
 * device slots in `scratch`: while one chunk is computed on streams[0], the
 * next is copied in on streams[1] and the previous copied out on streams[2],
 * so both copy directions overlap the kernels.  Host buffers should be
 * page-locked for the copies to be asynchronous.  streams: three cudaStream_t
 * (distinct for overlap; streams[0] is the one to synchronise: its work ends
 * after the last copy out).  scratch: a device buffer of at least
 * lsh_attn_step_host_scratch_size() bytes, 256-byte aligned; lsh_attn_poll
 * on it reports the device status of the call.  Creates and destroys six CUDA
 * events per call; allocates no memory. */
LSH_API size_t lsh_attn_step_host_scratch_size(const lsh_attn_desc *desc, int32_t heads_per_chunk,
                                               int with_backward);
LSH_API lsh_status lsh_attn_step_host(const lsh_attn_desc *desc, int32_t heads_per_chunk, const void *qk_h,
                                      const void *v_h, const void *R_h, const void *dout_h, void *out_h,
                                      float *lse_h, void *dqk_h, void *dv_h, void *scratch, size_t scratch_bytes,
                                      void *const *streams);

/* Parity bookkeeping: the number of (row, round) pairs of the last hash
 * (lsh_attn_hash, or the hash inside lsh_attn_fwd / lsh_attn_bwd) whose two
 * largest entries of [x R_r ; -x R_r] differ by less than 1e-6 of the
 * largest magnitude, so that a rounding difference could change the bucket.
 * Counted only in the tuning build (liblsh_attn_trace.so), where every hash
 * also runs a CUDA-core pass that recomputes the projections in fp32;
 * synchronises the device.  Returns -1 in the regular build, -2 on a CUDA
 * error. */
LSH_API int lsh_attn_last_near_ties(void);

/* Device-side status of the calls made with this workspace since the last
 * poll: synchronises `stream`, returns LSH_ERR_TIMEOUT if a bounded wait in a
 * kernel gave up, else LSH_ERR_ARG if a kernel read a permutation entry
 * outside [0, L) (such an entry is treated as an empty slot: nothing is read
 * or written at it, and positions it should have covered get no output), and
 * clears the word.  Call it after a call, not during. */
LSH_API lsh_status lsh_attn_poll(void *workspace, void *stream);

/* Stage timing.  lsh_attn_trace_begin(capacity) creates `capacity` pairs of
 * CUDA events and, until lsh_attn_trace_end, every entry point records one
 * pair around each stage it enqueues (process-wide; not for concurrent use
 * from several host threads).  lsh_attn_trace_end synchronises on the last
 * event, adds each recorded stage's elapsed milliseconds into ms[stage],
 * its invocation count into calls[stage] and the number of kernels it
 * launched into kernels[stage] (arrays of n >= LSH_STAGE_COUNT entries,
 * accumulated, not cleared), then destroys the events.  Stages beyond the
 * capacity are not recorded; the return value is then LSH_ERR_WORKSPACE. */
typedef enum {
    LSH_STAGE_HASH = 0,      /* lsh_hash: rotations + argmax                    */
    LSH_STAGE_SORT,          /* bucket_sort: radix passes                       */
    LSH_STAGE_NORMS,         /* 1/|x| per row                                   */
    LSH_STAGE_ATTN_FWD,      /* gather + chunk attention, per-round outputs     */
    LSH_STAGE_COMBINE,       /* unsort_combine: merge rounds                    */
    LSH_STAGE_BWD_PREP,      /* logsumexp over rounds, dY.Y, zero accumulators  */
    LSH_STAGE_ATTN_BWD,      /* chunk attention backward                        */
    LSH_STAGE_BWD_FINAL,     /* fp32 accumulators -> dqk, dv                    */
    LSH_STAGE_FUSED_FWD,     /* hash + sort + attention + merge in one kernel   */
    LSH_STAGE_COUNT
} lsh_stage;

LSH_API lsh_status lsh_attn_trace_begin(int32_t capacity);
LSH_API lsh_status lsh_attn_trace_end(float *ms, int32_t *calls, int32_t *kernels, int32_t n);

/* Which stages a trace records: bit s of `mask` for lsh_stage s (default: all).
 * Process-wide, takes effect for the stages enqueued after the call; a stage
 * left out is enqueued without events around it, so timing one kernel adds
 * only its own event pair to the stream.  Always returns LSH_OK. */
LSH_API lsh_status lsh_attn_trace_stages(uint32_t mask);

/* Single-kernel forward of short segments (lsh_attn_fwd, the reversible block
 * and lsh_attn_step_host).  mode = 1 (the default): used where a segment fits
 * and the B*H*n_hashes segments make one well-filled wave (one CTA per
 * segment: from three quarters of the SM count up to the SM count); otherwise
 * the staged kernels, which spread every tile over all SMs, are faster.  mode = 2:
 * used wherever a segment fits.  mode = 0: never (the staged kernels: hash,
 * sort, attention, merge).  Both forms give the same bits.  Process-wide;
 * takes effect for calls made after it.  Returns LSH_ERR_ARG for any other
 * value. */
LSH_API lsh_status lsh_attn_fused_forward(int32_t mode);

/* 1 if a forward with this descriptor runs as the single kernel under the
 * current setting (on the current device), 0 otherwise (also for an invalid
 * descriptor). */
LSH_API int32_t lsh_attn_fused_forward_fits(const lsh_attn_desc *desc);

/* Self-test of the bounded device-side waits: launches one CTA that waits on a
 * barrier nothing completes, for `budget_cycles` SM cycles (>= 0).  The wait
 * gives up, sets the timeout bit in the status word at the start of
 * `workspace` (any buffer of >= 256 bytes, 256-byte aligned) and the kernel
 * returns; lsh_attn_poll then reports LSH_ERR_TIMEOUT.  Nothing faults. */
LSH_API lsh_status lsh_attn_selftest_timeout(void *workspace, int64_t budget_cycles, void *stream);

/* Human-readable name of a status code; never NULL. */
LSH_API const char *lsh_attn_status_str(lsh_status status);

/* Text of the last CUDA error seen by this thread ("" if none). */
LSH_API const char *lsh_attn_last_error(void);

/* LSH_ATTN_ABI_VERSION of the loaded library. */
LSH_API int32_t lsh_attn_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LSH_ATTN_H */
