// Shared device helpers and the internal launch interface of the LSH
// attention library.  Nothing here is part of the C ABI.
#pragma once

#include <algorithm>

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/lsh_attn.h"

namespace lsh {

constexpr int kDim = 64;              // head dimension supported by every kernel

// ---------------------------------------------------------------- problem
struct Problem {
    int B, H, L, d, nb, R, m, causal, dtype, flags;
    // Rounds whose window is the previous chunk alone (bit r set: round r), with
    // no self fallback; 0 for LSH attention.  Local attention with a following
    // chunk runs that part as round 1 on the reversed order.
    int prev_mask = 0;
    long long BH() const { return (long long)B * H; }
    long long S() const { return BH() * R; }         // (b, h, round) segments
    long long tokens() const { return BH() * L; }
};

// ---------------------------------------------------------------- sort plan
constexpr int kSortTile = 2048;       // positions per sort CTA
constexpr int kSortThreads = 256;     // 8 warps x 32 lanes x 8 iterations

struct SortPlan {
    int passes;                       // 1 or 2
    int shift[2];
    int bits[2];
    int n_tiles;
    int max_radix;
};
SortPlan make_sort_plan(int n_buckets, int L);
// Segments this short with this few buckets are sorted on chip by one CTA.
constexpr int kSegMaxL = 16384;
constexpr int kSegMaxBuckets = 512;
bool seg_sort_fits(const Problem &p);
// Kernels one sort launches (for the stage trace).
inline int sort_kernel_count(const Problem &p)
{
    return seg_sort_fits(p) ? 1 : 3 * make_sort_plan(p.nb, p.L).passes;
}

// ---------------------------------------------------------------- workspace
struct Workspace {
    uint32_t *status;                 // device status word (timeouts)
    void *rot;                        // rotations re-laid out for the tensor-core hash
    float *invnorm;                   // [BH, L]  1/|x| (0 for a zero row)
    uint16_t *buckets;                // [S, L]
    uint16_t *sort_keys;              // [S, L]   first-pass keys
    int32_t *sort_vals;               // [S, L]   first-pass positions
    uint32_t *sort_counts;            // [S, radix, tiles]
    int32_t *perm;                    // [S, L]   internal permutation
    void *o_r;                        // [S, L, 64] per-round outputs
    float *lse_r;                     // [S, L]   per-round logsumexp (local attention with two parts)
    float *lse_all;                   // [BH, L]  logsumexp over rounds
    float *delta;                     // [BH, L]  dY . Y
    float *own;                       // [BH, L]  penalised own entry's weight (self penalty only)
    uint8_t *self_only;               // [S, L]   per sorted slot
    float *dx_acc;                    // [BH, L, 64]
    float *dv_acc;                    // [BH, L, 64]
    size_t bytes;
};
// Lays the workspace out from `base` (or from 0 when base is null, to size it).
Workspace plan_workspace(const Problem &p, bool backward, bool tc_attn, bool tc_hash, char *base);

// Fixed-size sort scratch of lsh_attn_sort_static (bytes per device).
constexpr size_t kStaticSortScratchBytes = LSH_ATTN_SORT_STATIC_MAX_BYTES;
// Lays out only the sort fields (keys, values, counters) from `base`; *bytes = total.
Workspace plan_sort_scratch(const Problem &p, char *base, size_t *bytes);
// Device address of this device's fixed sort scratch (looked up on first use).
cudaError_t static_sort_scratch(void **ptr);

// ---------------------------------------------------------------- helpers
__device__ __forceinline__ float to_f(float a) { return a; }
__device__ __forceinline__ float to_f(__nv_bfloat16 a) { return __bfloat162float(a); }
template <typename T> __device__ __forceinline__ T from_f(float a);
template <> __device__ __forceinline__ float from_f<float>(float a) { return a; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float a) { return __float2bfloat16_rn(a); }

// Loads a 64-element row into registers as float.
__device__ __forceinline__ void load_row(const float *p, float *r)
{
    const float4 *q = reinterpret_cast<const float4 *>(p);
#pragma unroll
    for (int k = 0; k < 16; ++k) {
        float4 a = q[k];
        r[4 * k] = a.x; r[4 * k + 1] = a.y; r[4 * k + 2] = a.z; r[4 * k + 3] = a.w;
    }
}
__device__ __forceinline__ void load_row(const __nv_bfloat16 *p, float *r)
{
    const uint4 *q = reinterpret_cast<const uint4 *>(p);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        uint4 a = q[k];
        const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            r[8 * k + 2 * e] = __uint_as_float(w[e] << 16);
            r[8 * k + 2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
        }
    }
}

// Sequential fp32 dot product of two 64-vectors (fixed order, fused multiply-add).
__device__ __forceinline__ float dot64(const float *a, const float *b)
{
    float s = 0.f;
#pragma unroll
    for (int k = 0; k < 64; ++k) s = fmaf(a[k], b[k], s);
    return s;
}

__device__ __forceinline__ void store_row(float *p, const float *r)
{
    float4 *q = reinterpret_cast<float4 *>(p);
#pragma unroll
    for (int k = 0; k < 16; ++k) q[k] = make_float4(r[4 * k], r[4 * k + 1], r[4 * k + 2], r[4 * k + 3]);
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}
__device__ __forceinline__ void store_row(__nv_bfloat16 *p, const float *r)
{
    uint4 *q = reinterpret_cast<uint4 *>(p);
#pragma unroll
    for (int k = 0; k < 8; ++k)
        q[k] = make_uint4(pack_bf16x2(r[8 * k], r[8 * k + 1]), pack_bf16x2(r[8 * k + 2], r[8 * k + 3]),
                          pack_bf16x2(r[8 * k + 4], r[8 * k + 5]), pack_bf16x2(r[8 * k + 6], r[8 * k + 7]));
}

// ---------------------------------------------------------------- launchers
// Every launcher enqueues on `st` and returns cudaGetLastError().
cudaError_t launch_invnorm(const Problem &p, const void *x, float *invnorm, cudaStream_t st);
cudaError_t launch_hash_simt(const Problem &p, const void *x, const void *R, uint16_t *buckets, cudaStream_t st);
// Near-tie count of a hash (tuning build only; a no-op elsewhere) and its read-back
// (-1 when not compiled in, -2 on a CUDA error).
cudaError_t launch_near_ties(const Problem &p, const void *x, const void *R, cudaStream_t st);
long long read_near_ties();
// invnorm (nullable): receives 1/|x| per token [BH, L] (from the same reads of x)
cudaError_t launch_hash_tc(const Problem &p, const void *x, const void *R, uint16_t *buckets, void *scratch,
                           float *invnorm, uint32_t *status, cudaStream_t st);
bool hash_tc_supported(const Problem &p);
size_t hash_tc_scratch_bytes(const Problem &p);
cudaError_t launch_sort(const Problem &p, const uint16_t *buckets, int32_t *perm, const Workspace &ws,
                        cudaStream_t st);
// bkt: bucket ids by position [S, L], read only under LSH_FLAG_BUCKET_MASK (may be null otherwise)
cudaError_t launch_attn_fwd_simt(const Problem &p, const void *x, const void *v, const int32_t *perm,
                                 const float *invnorm, const uint16_t *bkt, float *o_r, float *lse,
                                 uint32_t *status, cudaStream_t st);
// xinv: 1/|x| per token [BH, L] (launch_invnorm)
cudaError_t launch_attn_fwd_tc(const Problem &p, const void *x, const void *v, const int32_t *perm,
                               const uint16_t *bkt, const float *xinv, __nv_bfloat16 *o_r, float *lse,
                               uint32_t *status, cudaStream_t st);
bool attn_tc_supported(const Problem &p);
// Single-kernel forward of short segments (hash, sort, attention and merge in one
// cluster of R CTAs per head): perm [S, L], bkt [S, L] (bucket ids by position),
// xinv [BH, L] (1/|x|) and lse [S, L] are outputs, o_r [S, L, 64] bf16 is
// scratch, out [BH, L, 64] bf16 the merged output.
bool fused_fwd_fits(const Problem &p);
cudaError_t launch_fused_fwd_tc(const Problem &p, const void *x, const void *v, const void *R, int32_t *perm,
                                uint16_t *bkt, float *xinv, void *o_r, float *lse, void *out, uint32_t *status,
                                cudaStream_t st);
// lse_out (nullable): receives logsumexp over the rounds, [BH, L]
cudaError_t launch_combine(const Problem &p, const void *o_r, bool o_r_bf16, const float *lse, void *out,
                           float *lse_out, cudaStream_t st);
// Local attention's slot orders ([S, L]: round 0 identity, round 1 reversed).
cudaError_t launch_local_perm(const Problem &p, int32_t *perm, cudaStream_t st);
// own (nullable): the weight of a lone query's penalised own entry, [BH, L]
cudaError_t launch_bwd_prep(const Problem &p, const float *lse, const void *out, const void *dout,
                            float *lse_all, float *delta, float *own, float *dx_acc, float *dv_acc, cudaStream_t st);
cudaError_t launch_attn_bwd_simt(const Problem &p, const void *x, const void *v, const void *dout,
                                 const int32_t *perm, const float *invnorm, const uint16_t *bkt,
                                 const float *lse_all, const float *delta, const float *own, uint8_t *self_only,
                                 float *dx_acc, float *dv_acc, uint32_t *status, cudaStream_t st);
cudaError_t launch_attn_bwd_tc(const Problem &p, const void *x, const void *v, const void *dout,
                               const int32_t *perm, const uint16_t *bkt, const float *lse_all,
                               const float *delta, const float *own, float *dx_acc, float *dv_acc, uint32_t *status,
                               cudaStream_t st);
cudaError_t launch_bwd_finalize(const Problem &p, const float *dx_acc, const float *dv_acc, void *dqk, void *dv,
                                cudaStream_t st);

cudaError_t launch_wait_selftest(uint32_t *status, long long budget, cudaStream_t st);

// Reversible block pieces (fp32 streams [tokens, 64]; `b`, `c` in the attention dtype).
cudaError_t launch_g_forward(const Problem &p, const float *u, const float *W, const float *b, const float *res,
                             float *out, float *g_out, cudaStream_t st);
cudaError_t launch_g_backward(const Problem &p, const float *g, const float *dy, const float *W, const float *base,
                              float *out, cudaStream_t st);
cudaError_t launch_axpy(const Problem &p, const float *a, const void *b, float s, float *out, cudaStream_t st);
cudaError_t launch_cast(const Problem &p, const float *a, void *out, cudaStream_t st);
cudaError_t launch_sum3(const Problem &p, const float *a, const void *b, const void *c, float *out, cudaStream_t st);
cudaError_t launch_sub(const Problem &p, const float *a, const float *b, float *out, cudaStream_t st);

// Status bits written by kernels into Workspace::status.
constexpr uint32_t kStatusTimeout = 1u;     // a bounded wait gave up
constexpr uint32_t kStatusBadPerm = 2u;     // a permutation entry outside [0, L) was read (and ignored)

}  // namespace lsh
