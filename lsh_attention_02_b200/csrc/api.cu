// C ABI of the LSH attention library: argument checks, workspace layout and
// the launch sequence of each entry point.  Every entry point checks its
// arguments on the host before launching anything and never allocates.
#include <stdio.h>
#include <string.h>

#include "common.cuh"

namespace lsh {

static thread_local char g_last_error[256] = "";

static lsh_status cuda_fail(cudaError_t e, const char *where)
{
    snprintf(g_last_error, sizeof(g_last_error), "%s: %s", where, cudaGetErrorString(e));
    return LSH_ERR_CUDA;
}

#define LSH_TRY(expr, where)                                        \
    do {                                                            \
        cudaError_t e_ = (expr);                                    \
        if (e_ != cudaSuccess) return cuda_fail(e_, where);         \
    } while (0)

static size_t align_up(size_t a, size_t b) { return (a + b - 1) / b * b; }

// ------------------------------------------------------------------ stage trace
struct Trace {
    bool on = false;
    int cap = 0, used = 0;
    bool overflow = false;
    cudaEvent_t *ev = nullptr;      // 2 per record
    int *stage = nullptr, *kernels = nullptr;
};
static Trace g_trace;
static uint32_t g_trace_mask = ~0u;  // stages recorded while a trace is on (bit = lsh_stage)

// Records one event pair around a stage; `fn` enqueues the stage's kernels.
template <typename F>
static cudaError_t staged(int stage, int n_kernels, cudaStream_t st, F fn)
{
    const bool sel = ((g_trace_mask >> stage) & 1u) != 0;
    const bool rec = g_trace.on && sel && g_trace.used < g_trace.cap;
    if (g_trace.on && sel && !rec) g_trace.overflow = true;
    if (rec) {
        cudaError_t e = cudaEventRecord(g_trace.ev[2 * g_trace.used], st);
        if (e != cudaSuccess) return e;
    }
    cudaError_t e = fn();
    if (e != cudaSuccess) return e;
    if (rec) {
        e = cudaEventRecord(g_trace.ev[2 * g_trace.used + 1], st);
        if (e != cudaSuccess) return e;
        g_trace.stage[g_trace.used] = stage;
        g_trace.kernels[g_trace.used] = n_kernels;
        ++g_trace.used;
    }
    return cudaSuccess;
}

Workspace plan_workspace(const Problem &p, bool backward, bool tc_attn, bool tc_hash, char *base)
{
    Workspace w{};
    size_t off = 0;
    auto take = [&](size_t bytes) -> char * {
        char *ptr = base ? base + off : nullptr;
        off = align_up(off + bytes, 256);
        return ptr;
    };
    const size_t S = (size_t)p.S(), L = (size_t)p.L, T = (size_t)p.tokens();
    const SortPlan sp = make_sort_plan(p.nb, p.L);
    w.status = (uint32_t *)take(256);
    w.rot = take(tc_hash ? hash_tc_scratch_bytes(p) : 0);
    w.invnorm = (float *)take(T * sizeof(float));
    w.buckets = (uint16_t *)take(S * L * sizeof(uint16_t));
    w.sort_keys = (uint16_t *)take(sp.passes > 1 ? S * L * sizeof(uint16_t) : 0);
    w.sort_vals = (int32_t *)take(sp.passes > 1 ? S * L * sizeof(int32_t) : 0);
    w.sort_counts = (uint32_t *)take(S * (size_t)sp.max_radix * sp.n_tiles * sizeof(uint32_t));
    w.perm = (int32_t *)take(S * L * sizeof(int32_t));
    if (!backward) {
        w.o_r = take(S * L * kDim * (tc_attn ? 2 : 4));
        w.lse_r = (float *)take(p.prev_mask ? S * L * sizeof(float) : 0);
    } else {
        w.lse_all = (float *)take(T * sizeof(float));
        w.delta = (float *)take(T * sizeof(float));
        w.own = (float *)take((p.flags & LSH_FLAG_SELF_PENALTY) ? T * sizeof(float) : 0);
        w.self_only = (uint8_t *)take(tc_attn ? 0 : S * L);
        w.dx_acc = (float *)take(T * kDim * sizeof(float));
        w.dv_acc = (float *)take(T * kDim * sizeof(float));
    }
    w.bytes = off;
    return w;
}

static lsh_status check_desc(const lsh_attn_desc *d, Problem *p)
{
    if (!d) return LSH_ERR_ARG;
    if (d->dtype != LSH_F32 && d->dtype != LSH_BF16) return LSH_ERR_ARG;
    if (d->causal != 0 && d->causal != 1) return LSH_ERR_ARG;
    if (d->flags & ~(LSH_FLAG_BUCKET_MASK | LSH_FLAG_SELF_PENALTY)) return LSH_ERR_ARG;
    if (d->B < 1 || d->H < 1 || d->L < 1 || d->n_hashes < 1 || d->chunk < 1) return LSH_ERR_SHAPE;
    if (d->n_buckets < 2 || d->n_buckets % 2 != 0 || d->n_buckets > 65536) return LSH_ERR_SHAPE;
    if (d->L % d->chunk != 0) return LSH_ERR_SHAPE;
    if (d->d != kDim) return LSH_ERR_UNSUPPORTED;
    long long segs = (long long)d->B * d->H * d->n_hashes;
    if (segs > 65535) return LSH_ERR_UNSUPPORTED;     // grid.y of the per-segment kernels
    p->B = d->B; p->H = d->H; p->L = d->L; p->d = d->d; p->nb = d->n_buckets;
    p->R = d->n_hashes; p->m = d->chunk; p->causal = d->causal; p->dtype = d->dtype; p->flags = d->flags;
    return LSH_OK;
}

// bf16 hash and attention run on the tensor-core kernels only; a request they
// do not cover is refused (the sort alone does not depend on the dtype).
static lsh_status check_envelope(const Problem &p)
{
    if (p.dtype == LSH_BF16 && !(attn_tc_supported(p) && hash_tc_supported(p))) return LSH_ERR_UNSUPPORTED;
    return LSH_OK;
}

// Which kernels run is fixed by the dtype: bf16 -> tensor cores, fp32 -> CUDA cores (no TF32).
struct Choice {
    bool tc_attn;
    bool tc_hash;
};
static Choice choose(const Problem &p)
{
    const bool tc = p.dtype == LSH_BF16;
    return Choice{tc, tc};
}

static bool aligned16(const void *ptr) { return ((uintptr_t)ptr & 15u) == 0; }

static lsh_status check_ptrs(std::initializer_list<const void *> ptrs)
{
    for (const void *q : ptrs) if (!q) return LSH_ERR_ARG;
    for (const void *q : ptrs) if (!aligned16(q)) return LSH_ERR_ALIGN;
    return LSH_OK;
}

static lsh_status check_ws(void *ws, size_t ws_bytes, size_t need)
{
    if (!ws) return LSH_ERR_ARG;
    if (((uintptr_t)ws & 255u) != 0) return LSH_ERR_ALIGN;
    if (ws_bytes < need) return LSH_ERR_WORKSPACE;
    return LSH_OK;
}

// hash + sort into perm (internal helper shared by fwd and bwd)
static lsh_status run_hash_sort(const Problem &p, const Choice &c, const void *qk, const void *R, int32_t *perm,
                                const Workspace &w, cudaStream_t st)
{
    LSH_TRY(staged(LSH_STAGE_HASH, c.tc_hash ? 2 : 1, st, [&] {
                return c.tc_hash ? launch_hash_tc(p, qk, R, w.buckets, w.rot, w.invnorm, w.status, st)
                                 : launch_hash_simt(p, qk, R, w.buckets, st);
            }), "hash");
    LSH_TRY(launch_near_ties(p, qk, R, st), "near-tie count");
    LSH_TRY(staged(LSH_STAGE_SORT, sort_kernel_count(p), st,
                   [&] { return launch_sort(p, w.buckets, perm, w, st); }), "sort");
    return LSH_OK;
}

// norms_ready: the tensor-core hash of this call already wrote w.invnorm
static lsh_status run_attn_fwd(const Problem &p, const Choice &c, const void *qk, const void *v,
                               const int32_t *perm, void *out, float *lse, const Workspace &w, cudaStream_t st,
                               bool norms_ready = false)
{
    if (!norms_ready)
        LSH_TRY(staged(LSH_STAGE_NORMS, 1, st, [&] { return launch_invnorm(p, qk, w.invnorm, st); }), "key norms");
    LSH_TRY(staged(LSH_STAGE_ATTN_FWD, 1, st, [&] {
                return c.tc_attn
                           ? launch_attn_fwd_tc(p, qk, v, perm, w.buckets, w.invnorm, (__nv_bfloat16 *)w.o_r, lse,
                                                w.status, st)
                           : launch_attn_fwd_simt(p, qk, v, perm, w.invnorm, w.buckets, (float *)w.o_r, lse,
                                                  w.status, st);
            }), "attention forward");
    LSH_TRY(staged(LSH_STAGE_COMBINE, 1, st, [&] {
                return launch_combine(p, w.o_r, c.tc_attn, lse, out, nullptr, st);
            }), "round merge");
    return LSH_OK;
}

// The whole forward from the rotations: one kernel per head's rounds where a
// segment fits on chip and the setting allows it, otherwise hash, sort,
// attention and merge as separate stages.  Setting 1 (the default) takes the
// single kernel only where its segments make one well-filled wave: it runs one
// CTA per segment, so with few segments most SMs idle while the staged kernels
// spread every tile over all of them, and a second wave doubles its time while
// the staged time grows less than linearly.  Measured at L = 4096 (64 buckets,
// 2 rounds; single kernel against staged, us): 4 segments 117 / 43, 64 116 /
// 85, 128 124 / 131, 160 227 / 164, 256 236 / 228.  So: at least three
// quarters as many segments as SMs, and no more than the SMs.  Setting 2 takes
// it wherever it fits (tests), 0 never.
static int g_fused_forward = 1;
static int sm_count()
{
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
                                                   cudaSuccess || sms <= 0) {
        cudaGetLastError();
        sms = 148;                          // no device: the B200's count
    }
    return sms;
}
static bool use_fused(const Problem &p, const Choice &c)
{
    if (g_fused_forward == 0 || !c.tc_attn || !fused_fwd_fits(p)) return false;
    if (g_fused_forward == 2) return true;
    const long long sms = sm_count(), S = p.S();
    return 4 * S >= 3 * sms && S <= sms;
}
static lsh_status run_forward(const Problem &p, const Choice &c, const void *qk, const void *v, const void *R,
                              int32_t *perm, void *out, float *lse, const Workspace &w, cudaStream_t st)
{
    if (use_fused(p, c)) {
        LSH_TRY(staged(LSH_STAGE_FUSED_FWD, 1, st, [&] {
                    return launch_fused_fwd_tc(p, qk, v, R, perm, w.buckets, w.invnorm, w.o_r, lse, out, w.status, st);
                }), "single-kernel forward");
        return LSH_OK;
    }
    lsh_status s;
    if ((s = run_hash_sort(p, c, qk, R, perm, w, st)) != LSH_OK) return s;
    return run_attn_fwd(p, c, qk, v, perm, out, lse, w, st, c.tc_hash);
}

// prologue, attention backward and epilogue for a given permutation (shared by
// lsh_attn_bwd and the reversible block)
static lsh_status run_attn_bwd(const Problem &p, const Choice &c, const void *qk, const void *v, const void *out,
                               const float *lse, const int32_t *perm, const void *dout, void *dqk, void *dv,
                               const Workspace &w, cudaStream_t st)
{
    float *own = (p.flags & LSH_FLAG_SELF_PENALTY) ? w.own : nullptr;
    // the tensor-core backward computes the key norms from its gathered rows
    if (!c.tc_attn)
        LSH_TRY(staged(LSH_STAGE_NORMS, 1, st, [&] { return launch_invnorm(p, qk, w.invnorm, st); }), "key norms");
    LSH_TRY(staged(LSH_STAGE_BWD_PREP, 1, st, [&] {
                return launch_bwd_prep(p, lse, out, dout, w.lse_all, w.delta, own, w.dx_acc, w.dv_acc, st);
            }), "backward prologue");
    LSH_TRY(staged(LSH_STAGE_ATTN_BWD, c.tc_attn ? 1 : 2, st, [&] {
                return c.tc_attn ? launch_attn_bwd_tc(p, qk, v, dout, perm, w.buckets, w.lse_all, w.delta, own,
                                                      w.dx_acc, w.dv_acc, w.status, st)
                                 : launch_attn_bwd_simt(p, qk, v, dout, perm, w.invnorm, w.buckets, w.lse_all,
                                                        w.delta, own, w.self_only, w.dx_acc, w.dv_acc, w.status, st);
            }), "attention backward");
    LSH_TRY(staged(LSH_STAGE_BWD_FINAL, 1, st,
                   [&] { return launch_bwd_finalize(p, w.dx_acc, w.dv_acc, dqk, dv, st); }),
            "backward epilogue");
    return LSH_OK;
}

}  // namespace lsh

using namespace lsh;

extern "C" {

size_t lsh_attn_workspace_size(const lsh_attn_desc *desc, int for_backward)
{
    Problem p;
    Choice c;
    if (check_desc(desc, &p) != LSH_OK) return 0;
    c = choose(p);
    return plan_workspace(p, for_backward != 0, c.tc_attn, c.tc_hash, nullptr).bytes;
}

lsh_status lsh_attn_hash(const lsh_attn_desc *desc, const void *qk, const void *R, uint16_t *buckets,
                         void *workspace, size_t ws_bytes, void *stream)
{
    Problem p;
    Choice c;
    lsh_status s;
    if ((s = check_desc(desc, &p)) != LSH_OK) return s;
    if ((s = check_envelope(p)) != LSH_OK) return s;
    c = choose(p);
    if ((s = check_ptrs({qk, R})) != LSH_OK) return s;
    if (!buckets) return LSH_ERR_ARG;
    Workspace w = plan_workspace(p, false, c.tc_attn, c.tc_hash, nullptr);
    if ((s = check_ws(workspace, ws_bytes, w.bytes)) != LSH_OK) return s;
    w = plan_workspace(p, false, c.tc_attn, c.tc_hash, (char *)workspace);
    cudaStream_t st = (cudaStream_t)stream;
    LSH_TRY(staged(LSH_STAGE_HASH, c.tc_hash ? 2 : 1, st, [&] {
                return c.tc_hash ? launch_hash_tc(p, qk, R, buckets, w.rot, nullptr, w.status, st)
                                 : launch_hash_simt(p, qk, R, buckets, st);
            }), "hash");
    LSH_TRY(launch_near_ties(p, qk, R, st), "near-tie count");
    return LSH_OK;
}

lsh_status lsh_attn_sort(const lsh_attn_desc *desc, const uint16_t *buckets, int32_t *perm, void *workspace,
                         size_t ws_bytes, void *stream)
{
    Problem p;
    Choice c;
    lsh_status s;
    if ((s = check_desc(desc, &p)) != LSH_OK) return s;
    c = choose(p);
    if (!buckets || !perm) return LSH_ERR_ARG;
    Workspace w = plan_workspace(p, false, c.tc_attn, c.tc_hash, nullptr);
    if ((s = check_ws(workspace, ws_bytes, w.bytes)) != LSH_OK) return s;
    w = plan_workspace(p, false, c.tc_attn, c.tc_hash, (char *)workspace);
    cudaStream_t st = (cudaStream_t)stream;
    LSH_TRY(staged(LSH_STAGE_SORT, sort_kernel_count(p), st,
                   [&] { return launch_sort(p, buckets, perm, w, st); }), "sort");
    return LSH_OK;
}

int lsh_attn_last_near_ties(void)
{
    const long long v = read_near_ties();
    return v > 0x7FFFFFFFLL ? 0x7FFFFFFF : (int)v;
}

lsh_status lsh_attn_sort_static(const lsh_attn_desc *desc, const uint16_t *buckets, int32_t *perm, void *stream)
{
    Problem p;
    lsh_status s;
    if ((s = check_desc(desc, &p)) != LSH_OK) return s;
    if (!buckets || !perm) return LSH_ERR_ARG;
    size_t need = 0;
    plan_sort_scratch(p, nullptr, &need);
    if (need > kStaticSortScratchBytes) {
        snprintf(g_last_error, sizeof(g_last_error),
                 "lsh_attn_sort_static: needs %zu bytes of scratch, limit is %zu; use lsh_attn_sort", need,
                 kStaticSortScratchBytes);
        return LSH_ERR_WORKSPACE;
    }
    void *base = nullptr;
    LSH_TRY(static_sort_scratch(&base), "lsh_attn_sort_static: scratch address");
    const Workspace w = plan_sort_scratch(p, (char *)base, nullptr);
    cudaStream_t st = (cudaStream_t)stream;
    LSH_TRY(staged(LSH_STAGE_SORT, sort_kernel_count(p), st,
                   [&] { return launch_sort(p, buckets, perm, w, st); }), "sort_static");
    return LSH_OK;
}

lsh_status lsh_attn_fwd_sorted(const lsh_attn_desc *desc, const void *qk, const void *v, const int32_t *perm,
                               void *out, float *lse, void *workspace, size_t ws_bytes, void *stream)
{
    Problem p;
    Choice c;
    lsh_status s;
    if ((s = check_desc(desc, &p)) != LSH_OK) return s;
    if ((s = check_envelope(p)) != LSH_OK) return s;
    c = choose(p);
    if ((s = check_ptrs({qk, v, out, lse})) != LSH_OK) return s;
    if (!perm) return LSH_ERR_ARG;
    if (p.flags & LSH_FLAG_BUCKET_MASK) return LSH_ERR_ARG;     // needs bucket ids: use lsh_attn_fwd
    Workspace w = plan_workspace(p, false, c.tc_attn, c.tc_hash, nullptr);
    if ((s = check_ws(workspace, ws_bytes, w.bytes)) != LSH_OK) return s;
    w = plan_workspace(p, false, c.tc_attn, c.tc_hash, (char *)workspace);
    cudaStream_t st = (cudaStream_t)stream;
    LSH_TRY(cudaMemsetAsync(w.status, 0, sizeof(uint32_t), st), "status reset");
    return run_attn_fwd(p, c, qk, v, perm, out, lse, w, st);
}

lsh_status lsh_attn_fwd(const lsh_attn_desc *desc, const void *qk, const void *v, const void *R, void *out,
                        float *lse, int32_t *perm_out, void *workspace, size_t ws_bytes, void *stream)
{
    Problem p;
    Choice c;
    lsh_status s;
    if ((s = check_desc(desc, &p)) != LSH_OK) return s;
    if ((s = check_envelope(p)) != LSH_OK) return s;
    c = choose(p);
    if ((s = check_ptrs({qk, v, R, out, lse})) != LSH_OK) return s;
    Workspace w = plan_workspace(p, false, c.tc_attn, c.tc_hash, nullptr);
    if ((s = check_ws(workspace, ws_bytes, w.bytes)) != LSH_OK) return s;
    w = plan_workspace(p, false, c.tc_attn, c.tc_hash, (char *)workspace);
    cudaStream_t st = (cudaStream_t)stream;
    int32_t *perm = perm_out ? perm_out : w.perm;
    LSH_TRY(cudaMemsetAsync(w.status, 0, sizeof(uint32_t), st), "status reset");
    return run_forward(p, c, qk, v, R, perm, out, lse, w, st);
}

lsh_status lsh_attn_bwd(const lsh_attn_desc *desc, const void *qk, const void *v, const void *R, const void *out,
                        const float *lse, const int32_t *perm, const void *dout, void *dqk, void *dv,
                        void *workspace, size_t ws_bytes, void *stream)
{
    Problem p;
    Choice c;
    lsh_status s;
    if ((s = check_desc(desc, &p)) != LSH_OK) return s;
    if ((s = check_envelope(p)) != LSH_OK) return s;
    c = choose(p);
    if ((s = check_ptrs({qk, v, out, lse, dout, dqk, dv})) != LSH_OK) return s;
    const bool mask = (p.flags & LSH_FLAG_BUCKET_MASK) != 0;
    if ((!perm || mask) && !R) return LSH_ERR_ARG;             // the hash is recomputed from R
    Workspace w = plan_workspace(p, true, c.tc_attn, c.tc_hash, nullptr);
    if ((s = check_ws(workspace, ws_bytes, w.bytes)) != LSH_OK) return s;
    w = plan_workspace(p, true, c.tc_attn, c.tc_hash, (char *)workspace);
    cudaStream_t st = (cudaStream_t)stream;
    LSH_TRY(cudaMemsetAsync(w.status, 0, sizeof(uint32_t), st), "status reset");
    if (!perm) {
        if ((s = run_hash_sort(p, c, qk, R, w.perm, w, st)) != LSH_OK) return s;
        perm = w.perm;
    } else if (mask) {
        // the bucket mask needs the bucket ids of this call's rounds
        LSH_TRY(staged(LSH_STAGE_HASH, c.tc_hash ? 2 : 1, st, [&] {
                    return c.tc_hash ? launch_hash_tc(p, qk, R, w.buckets, w.rot, nullptr, w.status, st)
                                     : launch_hash_simt(p, qk, R, w.buckets, st);
                }), "hash");
    }
    return run_attn_bwd(p, c, qk, v, out, lse, perm, dout, dqk, dv, w, st);
}

// ------------------------------------------------------------------ local attention
// Local (non-hashed) chunk attention reuses the attention kernels: round 0 is
// the positions in their own order with the usual window (previous chunk and
// own chunk); with a following chunk (non-causal only: under the causal mask
// it holds no candidate), round 1 runs on the reversed order with the window
// reduced to the previous chunk, which there is the following chunk.  The two
// candidate sets are disjoint, so the round merge gives the three-chunk window
// exactly, and its logsumexp is the window's.
static lsh_status local_problem(const lsh_attn_desc *desc, int chunks_after, Problem *p)
{
    if (!desc) return LSH_ERR_ARG;
    lsh_attn_desc d = *desc;
    d.n_buckets = 2;                                     // not used
    lsh_status s = check_desc(&d, p);
    if (s != LSH_OK) return s;
    if (p->R != 1) return LSH_ERR_SHAPE;                 // one set of outputs: lse is [B, H, 1, L]
    if (p->flags & LSH_FLAG_BUCKET_MASK) return LSH_ERR_ARG;    // no buckets without hashing
    if (chunks_after != 0 && chunks_after != 1) return LSH_ERR_UNSUPPORTED;
    const bool following = chunks_after == 1 && !p->causal;
    p->R = following ? 2 : 1;
    p->prev_mask = following ? 2 : 0;
    return LSH_OK;
}

size_t lsh_attn_local_workspace_size(const lsh_attn_desc *desc, int32_t chunks_after, int for_backward)
{
    Problem p;
    if (local_problem(desc, chunks_after, &p) != LSH_OK) return 0;
    const Choice c = choose(p);
    return plan_workspace(p, for_backward != 0, c.tc_attn, c.tc_hash, nullptr).bytes;
}

lsh_status lsh_attn_local_fwd(const lsh_attn_desc *desc, int32_t chunks_after, const void *qk, const void *v,
                              void *out, float *lse, void *workspace, size_t ws_bytes, void *stream)
{
    Problem p;
    lsh_status s;
    if ((s = local_problem(desc, chunks_after, &p)) != LSH_OK) return s;
    if ((s = check_envelope(p)) != LSH_OK) return s;
    const Choice c = choose(p);
    if ((s = check_ptrs({qk, v, out, lse})) != LSH_OK) return s;
    Workspace w = plan_workspace(p, false, c.tc_attn, c.tc_hash, nullptr);
    if ((s = check_ws(workspace, ws_bytes, w.bytes)) != LSH_OK) return s;
    w = plan_workspace(p, false, c.tc_attn, c.tc_hash, (char *)workspace);
    cudaStream_t st = (cudaStream_t)stream;
    LSH_TRY(cudaMemsetAsync(w.status, 0, sizeof(uint32_t), st), "status reset");
    LSH_TRY(launch_local_perm(p, w.perm, st), "local order");
    float *lse_rounds = p.R == 2 ? w.lse_r : lse;        // one part: its lse is the window's
    LSH_TRY(staged(LSH_STAGE_NORMS, 1, st, [&] { return launch_invnorm(p, qk, w.invnorm, st); }), "key norms");
    LSH_TRY(staged(LSH_STAGE_ATTN_FWD, 1, st, [&] {
                return c.tc_attn ? launch_attn_fwd_tc(p, qk, v, w.perm, nullptr, w.invnorm, (__nv_bfloat16 *)w.o_r,
                                                      lse_rounds, w.status, st)
                                 : launch_attn_fwd_simt(p, qk, v, w.perm, w.invnorm, nullptr, (float *)w.o_r,
                                                        lse_rounds, w.status, st);
            }), "local attention forward");
    LSH_TRY(staged(LSH_STAGE_COMBINE, 1, st, [&] {
                return launch_combine(p, w.o_r, c.tc_attn, lse_rounds, out, p.R == 2 ? lse : nullptr, st);
            }), "local merge");
    return LSH_OK;
}

lsh_status lsh_attn_local_bwd(const lsh_attn_desc *desc, int32_t chunks_after, const void *qk, const void *v,
                              const void *out, const float *lse, const void *dout, void *dqk, void *dv,
                              void *workspace, size_t ws_bytes, void *stream)
{
    Problem p;
    lsh_status s;
    if ((s = local_problem(desc, chunks_after, &p)) != LSH_OK) return s;
    if ((s = check_envelope(p)) != LSH_OK) return s;
    const Choice c = choose(p);
    if ((s = check_ptrs({qk, v, out, lse, dout, dqk, dv})) != LSH_OK) return s;
    Workspace w = plan_workspace(p, true, c.tc_attn, c.tc_hash, nullptr);
    if ((s = check_ws(workspace, ws_bytes, w.bytes)) != LSH_OK) return s;
    w = plan_workspace(p, true, c.tc_attn, c.tc_hash, (char *)workspace);
    cudaStream_t st = (cudaStream_t)stream;
    LSH_TRY(cudaMemsetAsync(w.status, 0, sizeof(uint32_t), st), "status reset");
    LSH_TRY(launch_local_perm(p, w.perm, st), "local order");
    if (!c.tc_attn)
        LSH_TRY(staged(LSH_STAGE_NORMS, 1, st, [&] { return launch_invnorm(p, qk, w.invnorm, st); }), "key norms");
    // lse holds the whole window's logsumexp already: the prologue's merge is over one set
    float *own = (p.flags & LSH_FLAG_SELF_PENALTY) ? w.own : nullptr;
    Problem p1 = p;
    p1.R = 1;
    LSH_TRY(staged(LSH_STAGE_BWD_PREP, 1, st, [&] {
                return launch_bwd_prep(p1, lse, out, dout, w.lse_all, w.delta, own, w.dx_acc, w.dv_acc, st);
            }), "local backward prologue");
    LSH_TRY(staged(LSH_STAGE_ATTN_BWD, c.tc_attn ? 1 : 2, st, [&] {
                return c.tc_attn ? launch_attn_bwd_tc(p, qk, v, dout, w.perm, nullptr, w.lse_all, w.delta, own,
                                                      w.dx_acc, w.dv_acc, w.status, st)
                                 : launch_attn_bwd_simt(p, qk, v, dout, w.perm, w.invnorm, nullptr, w.lse_all,
                                                        w.delta, own, w.self_only, w.dx_acc, w.dv_acc, w.status, st);
            }), "local attention backward");
    LSH_TRY(staged(LSH_STAGE_BWD_FINAL, 1, st,
                   [&] { return launch_bwd_finalize(p, w.dx_acc, w.dv_acc, dqk, dv, st); }),
            "local backward epilogue");
    return LSH_OK;
}

// ------------------------------------------------------------------ reversible block
// Workspace of the reversible block: one attention workspace first (forward,
// or the larger of forward and backward; its status word at offset 0 is the one
// lsh_attn_poll reads), then the block's own buffers at 256-byte boundaries.
struct RevPlan {
    void *xa, *f, *da, *dqk, *dv;     // [T, 64] in the attention dtype
    float *g;                         // [T, 64] fp32: G(y1)
    float *lse;                       // [S, L]
    int32_t *perm;                    // [S, L]
    char *attn;                       // the attention workspace
    size_t attn_bytes, bytes;
};
static RevPlan plan_rev(const Problem &p, const Choice &c, bool backward, char *base)
{
    RevPlan r{};
    size_t off = 0;
    auto take = [&](size_t n) -> char * {
        char *ptr = base ? base + off : nullptr;
        off = align_up(off + n, 256);
        return ptr;
    };
    const size_t T = (size_t)p.tokens(), e = p.dtype == LSH_BF16 ? 2 : 4, S = (size_t)p.S(), L = (size_t)p.L;
    const size_t af = plan_workspace(p, false, c.tc_attn, c.tc_hash, nullptr).bytes;
    const size_t ab = backward ? plan_workspace(p, true, c.tc_attn, c.tc_hash, nullptr).bytes : 0;
    r.attn_bytes = af > ab ? af : ab;
    r.attn = take(r.attn_bytes);
    r.xa = take(T * kDim * e);
    r.f = take(T * kDim * e);
    r.lse = (float *)take(S * L * sizeof(float));
    r.perm = (int32_t *)take(S * L * sizeof(int32_t));
    if (backward) {
        r.g = (float *)take(T * kDim * sizeof(float));
        r.da = take(T * kDim * e);
        r.dqk = take(T * kDim * e);
        r.dv = take(T * kDim * e);
    }
    r.bytes = off;
    return r;
}

size_t lsh_rev_workspace_size(const lsh_attn_desc *desc, int for_backward)
{
    Problem p;
    if (check_desc(desc, &p) != LSH_OK) return 0;
    return plan_rev(p, choose(p), for_backward != 0, nullptr).bytes;
}

lsh_status lsh_rev_fwd(const lsh_attn_desc *desc, const float *x1, const float *x2, const void *R, const float *Wg,
                       const float *bg, float *y1, float *y2, void *workspace, size_t ws_bytes, void *stream)
{
    Problem p;
    lsh_status s;
    if ((s = check_desc(desc, &p)) != LSH_OK) return s;
    if ((s = check_envelope(p)) != LSH_OK) return s;
    const Choice c = choose(p);
    if ((s = check_ptrs({x1, x2, R, Wg, bg, y1, y2})) != LSH_OK) return s;
    RevPlan r = plan_rev(p, c, false, nullptr);
    if ((s = check_ws(workspace, ws_bytes, r.bytes)) != LSH_OK) return s;
    r = plan_rev(p, c, false, (char *)workspace);
    const Workspace w = plan_workspace(p, false, c.tc_attn, c.tc_hash, r.attn);
    cudaStream_t st = (cudaStream_t)stream;
    LSH_TRY(cudaMemsetAsync(w.status, 0, sizeof(uint32_t), st), "status reset");
    LSH_TRY(launch_cast(p, x2, r.xa, st), "x2 to the attention dtype");
    if ((s = run_forward(p, c, r.xa, r.xa, R, r.perm, r.f, r.lse, w, st)) != LSH_OK) return s;   // F(x2)
    LSH_TRY(launch_axpy(p, x1, r.f, 1.f, y1, st), "y1 = x1 + F(x2)");
    LSH_TRY(launch_g_forward(p, y1, Wg, bg, x2, y2, nullptr, st), "y2 = x2 + G(y1)");
    return LSH_OK;
}

lsh_status lsh_rev_bwd(const lsh_attn_desc *desc, const float *y1, const float *y2, const float *dy1,
                       const float *dy2, const void *R, const float *Wg, const float *bg, float *x1, float *x2,
                       float *dx1, float *dx2, void *workspace, size_t ws_bytes, void *stream)
{
    Problem p;
    lsh_status s;
    if ((s = check_desc(desc, &p)) != LSH_OK) return s;
    if ((s = check_envelope(p)) != LSH_OK) return s;
    const Choice c = choose(p);
    if ((s = check_ptrs({y1, y2, dy1, dy2, R, Wg, bg, x1, x2, dx1, dx2})) != LSH_OK) return s;
    RevPlan r = plan_rev(p, c, true, nullptr);
    if ((s = check_ws(workspace, ws_bytes, r.bytes)) != LSH_OK) return s;
    r = plan_rev(p, c, true, (char *)workspace);
    const Workspace wf = plan_workspace(p, false, c.tc_attn, c.tc_hash, r.attn);
    const Workspace wb = plan_workspace(p, true, c.tc_attn, c.tc_hash, r.attn);
    cudaStream_t st = (cudaStream_t)stream;
    LSH_TRY(cudaMemsetAsync(wf.status, 0, sizeof(uint32_t), st), "status reset");
    // inverse of the G half: x2 = y2 - G(y1); gradient into y1: dy1 + J_G(y1)^T dy2
    LSH_TRY(launch_g_forward(p, y1, Wg, bg, nullptr, r.g, nullptr, st), "G(y1)");
    LSH_TRY(launch_sub(p, y2, r.g, x2, st), "x2 = y2 - G(y1)");
    LSH_TRY(launch_g_backward(p, r.g, dy2, Wg, dy1, dx1, st), "dx1 = dy1 + J_G^T dy2");
    // inverse of the F half: F(x2) again (hash, sort, attention), x1 = y1 - F(x2)
    LSH_TRY(launch_cast(p, x2, r.xa, st), "x2 to the attention dtype");
    if ((s = run_forward(p, c, r.xa, r.xa, R, r.perm, r.f, r.lse, wf, st)) != LSH_OK) return s;
    LSH_TRY(launch_axpy(p, y1, r.f, -1.f, x1, st), "x1 = y1 - F(x2)");
    // gradient through F, whose query-key and value inputs are both x2
    LSH_TRY(launch_cast(p, dx1, r.da, st), "dF to the attention dtype");
    // (the bucket ids of the forward above are still in place: the backward's
    // workspace fields that precede the per-round outputs coincide with the forward's)
    if ((s = run_attn_bwd(p, c, r.xa, r.xa, r.f, r.lse, r.perm, r.da, r.dqk, r.dv, wb, st)) != LSH_OK) return s;
    LSH_TRY(launch_sum3(p, dy2, r.dqk, r.dv, dx2, st), "dx2 = dy2 + dF/dx2");
    return LSH_OK;
}

// ------------------------------------------------------------------ host-buffer pipeline
// Forward (+ backward) on host buffers.  The (batch, head) slices are
// independent, so they go in chunks of consecutive slices through two
// device slots: while chunk i is computed, chunk i+1 is copied in and
// chunk i-1 copied out, each on its own stream, so both copy directions and
// the kernels overlap.  The rotations are copied once.
struct HostPlan {
    int chunk, n_chunks;
    size_t R_bytes;
    char *R;                          // device copy of the rotations
    struct Slot {
        char *ws;                     // attention workspace (fwd / bwd share it in turn)
        void *x, *v, *dy, *out, *dqk, *dv;
        float *lse;
        int32_t *perm;
    } slot[2];
    size_t ws_bytes, bytes;
};

static HostPlan plan_host(const Problem &p, const Choice &c, int heads_per_chunk, bool bwd, char *base)
{
    HostPlan h{};
    const long long BH = p.BH();
    h.chunk = heads_per_chunk > 0 ? (int)std::min<long long>(heads_per_chunk, BH)
                                  : (int)std::max<long long>(1, (BH + 7) / 8);
    h.n_chunks = (int)((BH + h.chunk - 1) / h.chunk);
    Problem pc = p;
    pc.B = 1;
    pc.H = h.chunk;
    const size_t wf = plan_workspace(pc, false, c.tc_attn, c.tc_hash, nullptr).bytes;
    const size_t wb = bwd ? plan_workspace(pc, true, c.tc_attn, c.tc_hash, nullptr).bytes : 0;
    h.ws_bytes = std::max(wf, wb);
    size_t off = 0;
    auto take = [&](size_t n) -> char * {
        char *ptr = base ? base + off : nullptr;
        off = align_up(off + n, 256);
        return ptr;
    };
    const size_t e = p.dtype == LSH_BF16 ? 2 : 4;
    const size_t rows = (size_t)h.chunk * p.L, seg = (size_t)h.chunk * p.R * p.L;
    for (int k = 0; k < 2; ++k) {
        HostPlan::Slot &sl = h.slot[k];
        sl.ws = take(h.ws_bytes);         // slot 0's status word is at offset 0
        sl.x = take(rows * kDim * e);
        sl.v = take(rows * kDim * e);
        sl.dy = take(bwd ? rows * kDim * e : 0);
        sl.out = take(rows * kDim * e);
        sl.dqk = take(bwd ? rows * kDim * e : 0);
        sl.dv = take(bwd ? rows * kDim * e : 0);
        sl.lse = (float *)take(seg * sizeof(float));
        sl.perm = (int32_t *)take(seg * sizeof(int32_t));
    }
    h.R_bytes = (size_t)p.R * kDim * (p.nb / 2) * e;
    h.R = take(h.R_bytes);
    h.bytes = off;
    return h;
}

size_t lsh_attn_step_host_scratch_size(const lsh_attn_desc *desc, int32_t heads_per_chunk, int with_backward)
{
    Problem p;
    if (check_desc(desc, &p) != LSH_OK) return 0;
    return plan_host(p, choose(p), heads_per_chunk, with_backward != 0, nullptr).bytes;
}

lsh_status lsh_attn_step_host(const lsh_attn_desc *desc, int32_t heads_per_chunk, const void *qk_h, const void *v_h,
                              const void *R_h, const void *dout_h, void *out_h, float *lse_h, void *dqk_h,
                              void *dv_h, void *scratch, size_t scratch_bytes, void *const *streams)
{
    Problem p;
    lsh_status s;
    if ((s = check_desc(desc, &p)) != LSH_OK) return s;
    if ((s = check_envelope(p)) != LSH_OK) return s;
    const Choice c = choose(p);
    if (!qk_h || !v_h || !R_h || !out_h || !streams) return LSH_ERR_ARG;
    const bool bwd = dout_h != nullptr;
    if (bwd && (!dqk_h || !dv_h)) return LSH_ERR_ARG;
    HostPlan h = plan_host(p, c, heads_per_chunk, bwd, nullptr);
    if ((s = check_ws(scratch, scratch_bytes, h.bytes)) != LSH_OK) return s;
    h = plan_host(p, c, heads_per_chunk, bwd, (char *)scratch);
    cudaStream_t cs = (cudaStream_t)streams[0], in_s = (cudaStream_t)streams[1], out_s = (cudaStream_t)streams[2];
    const size_t e = p.dtype == LSH_BF16 ? 2 : 4;
    const size_t slice = (size_t)p.L * kDim * e, seg = (size_t)p.R * p.L;
    cudaEvent_t ev[2][3];                 // per slot: inputs landed, computed, outputs read
    for (int k = 0; k < 2; ++k)
        for (int j = 0; j < 3; ++j) {
            cudaError_t er = cudaEventCreateWithFlags(&ev[k][j], cudaEventDisableTiming);
            if (er != cudaSuccess) {
                for (int kk = 0; kk <= k; ++kk)
                    for (int jj = 0; jj < (kk < k ? 3 : j); ++jj) cudaEventDestroy(ev[kk][jj]);
                return cuda_fail(er, "pipeline events");
            }
        }
    lsh_status rc = LSH_OK;
    auto fail = [&](cudaError_t er, const char *where) {
        if (er != cudaSuccess && rc == LSH_OK) rc = cuda_fail(er, where);
        return er != cudaSuccess;
    };
    // every slot's kernels report into slot 0's status word
    uint32_t *status = (uint32_t *)h.slot[0].ws;
    if (fail(cudaMemsetAsync(status, 0, sizeof(uint32_t), cs), "status reset")) goto done;
    if (fail(cudaMemcpyAsync(h.R, R_h, h.R_bytes, cudaMemcpyHostToDevice, in_s), "rotations in")) goto done;
    for (int i = 0; i < h.n_chunks && rc == LSH_OK; ++i) {
        const int k = i & 1;
        const HostPlan::Slot &sl = h.slot[k];
        const long long bh0 = (long long)i * h.chunk;
        const int nh = (int)std::min<long long>(h.chunk, p.BH() - bh0);
        const size_t nb = (size_t)nh * slice;
        // copy in (the slot's inputs are free once chunk i-2 is computed)
        if (i >= 2 && fail(cudaStreamWaitEvent(in_s, ev[k][1], 0), "wait")) break;
        if (fail(cudaMemcpyAsync(sl.x, (const char *)qk_h + bh0 * slice, nb, cudaMemcpyHostToDevice, in_s), "qk in") ||
            fail(cudaMemcpyAsync(sl.v, (const char *)v_h + bh0 * slice, nb, cudaMemcpyHostToDevice, in_s), "v in"))
            break;
        if (bwd && fail(cudaMemcpyAsync(sl.dy, (const char *)dout_h + bh0 * slice, nb, cudaMemcpyHostToDevice, in_s),
                        "dout in"))
            break;
        if (fail(cudaEventRecord(ev[k][0], in_s), "record")) break;
        // compute (after the inputs, and after chunk i-2's outputs were read out)
        if (fail(cudaStreamWaitEvent(cs, ev[k][0], 0), "wait")) break;
        if (i >= 2 && fail(cudaStreamWaitEvent(cs, ev[k][2], 0), "wait")) break;
        Problem pc = p;
        pc.B = 1;
        pc.H = nh;
        Workspace wf = plan_workspace(pc, false, c.tc_attn, c.tc_hash, sl.ws);
        wf.status = status;
        if ((rc = run_forward(pc, c, sl.x, sl.v, h.R, sl.perm, sl.out, sl.lse, wf, cs)) != LSH_OK) break;
        if (bwd) {
            Workspace wb = plan_workspace(pc, true, c.tc_attn, c.tc_hash, sl.ws);
            wb.status = status;
            if ((rc = run_attn_bwd(pc, c, sl.x, sl.v, sl.out, sl.lse, sl.perm, sl.dy, sl.dqk, sl.dv, wb, cs)) !=
                LSH_OK)
                break;
        }
        if (fail(cudaEventRecord(ev[k][1], cs), "record")) break;
        // copy out
        if (fail(cudaStreamWaitEvent(out_s, ev[k][1], 0), "wait")) break;
        if (fail(cudaMemcpyAsync((char *)out_h + bh0 * slice, sl.out, nb, cudaMemcpyDeviceToHost, out_s), "out"))
            break;
        if (lse_h && fail(cudaMemcpyAsync(lse_h + bh0 * seg, sl.lse, (size_t)nh * seg * sizeof(float),
                                          cudaMemcpyDeviceToHost, out_s), "lse out"))
            break;
        if (bwd && (fail(cudaMemcpyAsync((char *)dqk_h + bh0 * slice, sl.dqk, nb, cudaMemcpyDeviceToHost, out_s),
                         "dqk out") ||
                    fail(cudaMemcpyAsync((char *)dv_h + bh0 * slice, sl.dv, nb, cudaMemcpyDeviceToHost, out_s),
                         "dv out")))
            break;
        if (fail(cudaEventRecord(ev[k][2], out_s), "record")) break;
    }
    // the caller's stream (streams[0]) ends after the last copy out
    if (rc == LSH_OK && h.n_chunks > 0) fail(cudaStreamWaitEvent(cs, ev[(h.n_chunks - 1) & 1][2], 0), "join");
done:
    for (int k = 0; k < 2; ++k)
        for (int j = 0; j < 3; ++j) cudaEventDestroy(ev[k][j]);
    return rc;
}

lsh_status lsh_attn_poll(void *workspace, void *stream)
{
    if (!workspace) return LSH_ERR_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    uint32_t word = 0;
    LSH_TRY(cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost, st), "status read");
    LSH_TRY(cudaStreamSynchronize(st), "status read");
    LSH_TRY(cudaMemsetAsync(workspace, 0, sizeof(word), st), "status clear");
    if (word & kStatusTimeout) return LSH_ERR_TIMEOUT;
    return (word & kStatusBadPerm) ? LSH_ERR_ARG : LSH_OK;
}

lsh_status lsh_attn_selftest_timeout(void *workspace, int64_t budget_cycles, void *stream)
{
    if (!workspace) return LSH_ERR_ARG;
    if (((uintptr_t)workspace & 255u) != 0) return LSH_ERR_ALIGN;
    if (budget_cycles < 0) return LSH_ERR_ARG;
    LSH_TRY(launch_wait_selftest((uint32_t *)workspace, (long long)budget_cycles, (cudaStream_t)stream),
            "wait self-test");
    return LSH_OK;
}

lsh_status lsh_attn_trace_begin(int32_t capacity)
{
    if (capacity < 1 || g_trace.on) return LSH_ERR_ARG;
    Trace t;
    t.cap = capacity;
    t.ev = new cudaEvent_t[2 * (size_t)capacity];
    t.stage = new int[capacity];
    t.kernels = new int[capacity];
    for (int i = 0; i < 2 * capacity; ++i) {
        cudaError_t e = cudaEventCreate(&t.ev[i]);
        if (e != cudaSuccess) {
            for (int k = 0; k < i; ++k) cudaEventDestroy(t.ev[k]);
            delete[] t.ev; delete[] t.stage; delete[] t.kernels;
            return cuda_fail(e, "trace events");
        }
    }
    t.on = true;
    g_trace = t;
    return LSH_OK;
}

lsh_status lsh_attn_trace_stages(uint32_t mask)
{
    g_trace_mask = mask;
    return LSH_OK;
}

lsh_status lsh_attn_fused_forward(int32_t mode)
{
    if (mode < 0 || mode > 2) return LSH_ERR_ARG;
    g_fused_forward = mode;
    return LSH_OK;
}

int32_t lsh_attn_fused_forward_fits(const lsh_attn_desc *desc)
{
    Problem p;
    if (check_desc(desc, &p) != LSH_OK || check_envelope(p) != LSH_OK) return 0;
    return use_fused(p, choose(p)) ? 1 : 0;
}

lsh_status lsh_attn_trace_end(float *ms, int32_t *calls, int32_t *kernels, int32_t n)
{
    if (!g_trace.on) return LSH_ERR_ARG;
    if (!ms || !calls || !kernels || n < LSH_STAGE_COUNT) return LSH_ERR_ARG;
    Trace t = g_trace;
    g_trace = Trace();
    lsh_status rc = LSH_OK;
    if (t.used > 0) {
        cudaError_t e = cudaEventSynchronize(t.ev[2 * t.used - 1]);
        if (e != cudaSuccess) rc = cuda_fail(e, "trace sync");
    }
    for (int i = 0; rc == LSH_OK && i < t.used; ++i) {
        float x = 0.f;
        cudaError_t e = cudaEventElapsedTime(&x, t.ev[2 * i], t.ev[2 * i + 1]);
        if (e != cudaSuccess) { rc = cuda_fail(e, "trace elapsed"); break; }
        ms[t.stage[i]] += x;
        calls[t.stage[i]] += 1;
        kernels[t.stage[i]] += t.kernels[i];
    }
    for (int i = 0; i < 2 * t.cap; ++i) cudaEventDestroy(t.ev[i]);
    delete[] t.ev; delete[] t.stage; delete[] t.kernels;
    if (rc == LSH_OK && t.overflow) rc = LSH_ERR_WORKSPACE;
    return rc;
}

const char *lsh_attn_status_str(lsh_status status)
{
    switch (status) {
    case LSH_OK: return "ok";
    case LSH_ERR_ARG: return "invalid argument (null pointer or unknown enum value)";
    case LSH_ERR_SHAPE: return "inconsistent sizes";
    case LSH_ERR_ALIGN: return "pointer not aligned";
    case LSH_ERR_UNSUPPORTED: return "unsupported configuration";
    case LSH_ERR_CUDA: return "CUDA error";
    case LSH_ERR_TIMEOUT: return "device-side wait timed out";
    case LSH_ERR_WORKSPACE: return "workspace too small";
    }
    return "unknown status";
}

const char *lsh_attn_last_error(void) { return g_last_error; }

int32_t lsh_attn_abi_version(void) { return LSH_ATTN_ABI_VERSION; }

}  // extern "C"

// ------------------------------------------------------------------ tensor maps
#include <cudaTypedefs.h>
#include "tc_common.cuh"

namespace lsh {
namespace tc {

bool make_row_tmap(CUtensorMap *map, const void *base, long long rows, int box_rows)
{
    static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    if (!encode) {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !fn)
            return false;
        encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    const cuuint64_t dims[2] = {(cuuint64_t)kDim, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)kDim * 2};
    const cuuint32_t box[2] = {(cuuint32_t)kDim, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace tc
}  // namespace lsh

