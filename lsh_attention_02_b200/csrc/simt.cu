// CUDA-core kernels: key norms, the fp32 hash, chunked attention forward and
// backward on CUDA cores, the round merge and the backward prologue/epilogue.
//
// These run every stage for fp32 inputs (no TF32 anywhere) and for shapes the
// tensor-core kernels do not cover; the merge, backward prologue and epilogue
// are memory-bound and serve both paths.
//
// Notation (paper note "Reformer"): x is the shared query-key ("Shared
// Query-Key Space", Q = K); tau = 1/sqrt(d) ("LSH Attention", output
// equation); a (b, h, r) segment holds one round's permutation.
#include <math.h>

#include "combine.cuh"

namespace lsh {

// ------------------------------------------------------------------ norms
// invnorm[row] = 1/|x_row| (fp32, IEEE sqrt and division), 0 for a zero row.
template <typename T>
__global__ void invnorm_kernel(const T *__restrict__ x, float *__restrict__ invnorm, long long rows)
{
    long long r = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (r >= rows) return;
    float a[kDim];
    load_row(x + r * kDim, a);
    float s = dot64(a, a);
    invnorm[r] = s > 0.f ? 1.0f / sqrtf(s) : 0.f;
}

// bf16 rows: a warp takes 16 consecutive rows, four per load instruction
// (eight lanes per 128-byte row, 512 contiguous bytes), all four loads in
// flight before any arithmetic; each row's eight partial sums of squares are
// added by shuffles.
constexpr int kNormRowsPerWarp = 16;
__global__ void invnorm_bf16_kernel(const __nv_bfloat16 *__restrict__ x, float *__restrict__ invnorm, long long rows)
{
    const long long w = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    const long long r0 = w * kNormRowsPerWarp + (lane >> 3);
    uint4 u[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const long long r = r0 + 4 * k;
        u[k] = r < rows ? __ldg(reinterpret_cast<const uint4 *>(x + r * kDim) + (lane & 7)) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const uint32_t wd[4] = {u[k].x, u[k].y, u[k].z, u[k].w};
        float s = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float a = __uint_as_float(wd[e] << 16), b = __uint_as_float(wd[e] & 0xFFFF0000u);
            s = fmaf(a, a, s);
            s = fmaf(b, b, s);
        }
        s += __shfl_xor_sync(0xffffffffu, s, 1);
        s += __shfl_xor_sync(0xffffffffu, s, 2);
        s += __shfl_xor_sync(0xffffffffu, s, 4);
        const long long r = r0 + 4 * k;
        if (r < rows && (lane & 7) == 0) invnorm[r] = s > 0.f ? 1.0f / sqrtf(s) : 0.f;
    }
}

cudaError_t launch_invnorm(const Problem &p, const void *x, float *invnorm, cudaStream_t st)
{
    const long long rows = p.tokens();
    if (p.dtype == LSH_BF16) {
        const long long warps = (rows + kNormRowsPerWarp - 1) / kNormRowsPerWarp;
        const unsigned grid = (unsigned)((warps * 32 + 255) / 256);
        invnorm_bf16_kernel<<<grid, 256, 0, st>>>((const __nv_bfloat16 *)x, invnorm, rows);
    } else {
        const unsigned grid = (unsigned)((rows + 127) / 128);
        invnorm_kernel<float><<<grid, 128, 0, st>>>((const float *)x, invnorm, rows);
    }
    return cudaGetLastError();
}

// ------------------------------------------------------------------ hash
// "LSH Attention", hash equation: bucket = argmax over [x R_r ; -x R_r].
// One thread per (row, round); projections in fp32, sequential fma over d.
// Exact ties keep the lowest index: +x R_r entries come before -x R_r ones.
template <typename T>
__global__ void hash_simt_kernel(const T *__restrict__ x, const T *__restrict__ R, uint16_t *__restrict__ buckets,
                                 long long BH, int L, int n_hashes, int half)
{
    long long row = (long long)blockIdx.x * blockDim.x + threadIdx.x;   // (bh, i)
    int r = blockIdx.y;
    if (row >= BH * L) return;
    float a[kDim];
    load_row(x + row * kDim, a);
    const T *Rr = R + (long long)r * kDim * half;
    float best_p = -INFINITY, best_n = -INFINITY;
    int idx_p = 0, idx_n = 0;
    for (int k = 0; k < half; ++k) {
        float s = 0.f;
#pragma unroll 16
        for (int t = 0; t < kDim; ++t) s = fmaf(a[t], to_f(Rr[(long long)t * half + k]), s);
        if (s > best_p) { best_p = s; idx_p = k; }
        if (-s > best_n) { best_n = -s; idx_n = k; }
    }
    int bucket = best_p >= best_n ? idx_p : half + idx_n;
    long long bh = row / L;
    int i = (int)(row % L);
    buckets[(bh * n_hashes + r) * L + i] = (uint16_t)bucket;
}

cudaError_t launch_hash_simt(const Problem &p, const void *x, const void *R, uint16_t *buckets, cudaStream_t st)
{
    if (p.dtype != LSH_F32) return cudaErrorInvalidValue;      // bf16 runs on the tensor-core hash
    long long rows = p.tokens();
    dim3 grid((unsigned)((rows + 127) / 128), p.R);
    hash_simt_kernel<float><<<grid, 128, 0, st>>>((const float *)x, (const float *)R, buckets, p.BH(), p.L, p.R,
                                                  p.nb / 2);
    return cudaGetLastError();
}

// ------------------------------------------------------------------ near ties
// Parity bookkeeping (compiled into the tuning build only): the number of
// (row, round) pairs whose two largest entries of [x R_r ; -x R_r] (fp32,
// sequential fma over d) differ by less than 1e-6 of the largest magnitude,
// i.e. whose bucket a rounding difference could flip.
#ifdef LSH_PHASE_TRACE
static __device__ unsigned long long g_near_ties;

__global__ void near_tie_reset_kernel() { g_near_ties = 0ull; }

template <typename T>
__global__ void near_tie_kernel(const T *__restrict__ x, const T *__restrict__ R, long long BH, int L, int half)
{
    long long row = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    int r = blockIdx.y;
    if (row >= BH * L) return;
    float a[kDim];
    load_row(x + row * kDim, a);
    const T *Rr = R + (long long)r * kDim * half;
    float t1 = -INFINITY, t2 = -INFINITY;                  // largest and second largest of [p ; -p]
    for (int k = 0; k < half; ++k) {
        float s = 0.f;
#pragma unroll 16
        for (int t = 0; t < kDim; ++t) s = fmaf(a[t], to_f(Rr[(long long)t * half + k]), s);
        const float hi = fmaxf(s, -s), lo = fminf(s, -s);
        if (hi > t1) { t2 = fmaxf(t1, lo); t1 = hi; }
        else { t2 = fmaxf(t2, hi); }
    }
    const float margin = (t1 - t2) / fmaxf(fabsf(t1), 1e-30f);
    if (margin < 1e-6f) atomicAdd(&g_near_ties, 1ull);
}
#endif

cudaError_t launch_near_ties(const Problem &p, const void *x, const void *R, cudaStream_t st)
{
#ifdef LSH_PHASE_TRACE
    near_tie_reset_kernel<<<1, 1, 0, st>>>();
    long long rows = p.tokens();
    dim3 grid((unsigned)((rows + 127) / 128), p.R);
    if (p.dtype == LSH_F32)
        near_tie_kernel<float><<<grid, 128, 0, st>>>((const float *)x, (const float *)R, p.BH(), p.L, p.nb / 2);
    else
        near_tie_kernel<__nv_bfloat16><<<grid, 128, 0, st>>>((const __nv_bfloat16 *)x, (const __nv_bfloat16 *)R,
                                                              p.BH(), p.L, p.nb / 2);
    return cudaGetLastError();
#else
    (void)p; (void)x; (void)R; (void)st;
    return cudaSuccess;
#endif
}

long long read_near_ties()
{
#ifdef LSH_PHASE_TRACE
    unsigned long long v = 0;
    if (cudaDeviceSynchronize() != cudaSuccess) return -2;
    if (cudaMemcpyFromSymbol(&v, g_near_ties, sizeof(v)) != cudaSuccess) return -2;
    return (long long)v;
#else
    return -1;
#endif
}

// ------------------------------------------------------------------ candidates
// Window of sorted slot s: chunks c-1 and c ("Sorting and Chunking").  A slot
// t != s is a candidate unless causal and its position exceeds the query's
// ("Implementation Reading": the mask uses original positions).
struct Window {
    int w0, w1;
};
// The window of sorted slot s: chunks c - 1 and c (c = s / m); `prev`: the
// previous chunk alone (the following-chunk part of local attention, run on
// the reversed order), empty for c = 0.
__device__ __forceinline__ Window window_of(int s, int m, int L, bool prev = false)
{
    int c = s / m;
    Window w;
    w.w0 = c > 0 ? (c - 1) * m : 0;
    w.w1 = prev ? c * m : min((c + 1) * m, L);
    return w;
}

// A permutation entry outside [0, L) marks an empty slot: it is skipped and
// reported in the status word.
__device__ __forceinline__ bool valid_pos(int j, int L, uint32_t *status)
{
    if ((unsigned)j < (unsigned)L) return true;
    atomicOr(status, kStatusBadPerm);
    return false;
}

// ------------------------------------------------------------------ candidates
// Optional readings (lsh_attn_desc.flags): `bkt` (nullable) holds the bucket id
// of every position of the segment, and only keys in the query's bucket are
// candidates (strict N_LSH, "LSH Attention"); `self_penalty` gives the query's
// own position the constant score kSelfPenalty instead of removing it.  When
// other candidates exist that entry's weight exp(kSelfPenalty - lse) is below
// 2^-149 for every |x_i| < 8e5, i.e. exactly 0 in fp32, so only a query with no
// other candidate uses it.
constexpr float kSelfPenalty = LSH_SELF_PENALTY_SCORE;

struct SlotView {
    const int32_t *P;
    const uint16_t *Bk;
    int L, causal;
    uint32_t *status;
    // key slot t (!= the query's slot) is a candidate of query position i in bucket bi
    __device__ __forceinline__ bool candidate(int t, int i, int bi, int &j) const
    {
        j = P[t];
        if (!valid_pos(j, L, status)) return false;
        if (causal && j > i) return false;
        return !Bk || Bk[j] == bi;
    }
};

// ------------------------------------------------------------------ forward
// One thread per (segment, sorted slot): full softmax over the window, output
// and logsumexp written at the query's original position.
template <typename T>
__global__ void attn_fwd_simt_kernel(const T *__restrict__ x, const T *__restrict__ v,
                                     const int32_t *__restrict__ perm, const float *__restrict__ invnorm,
                                     const uint16_t *__restrict__ bkt, float *__restrict__ o_r,
                                     float *__restrict__ lse, int L, int R, int m, int causal, int self_penalty,
                                     float tau, uint32_t prev_mask, uint32_t *__restrict__ status)
{
    const long long seg = blockIdx.y;
    const int s = blockIdx.x * blockDim.x + threadIdx.x;
    if (s >= L) return;
    const long long bh = seg / R;
    const SlotView sv{perm + seg * L, bkt ? bkt + seg * L : nullptr, L, causal, status};
    const T *X = x + bh * L * kDim;
    const T *V = v + bh * L * kDim;
    const float *IN = invnorm + bh * L;
    const int i = sv.P[s];
    if (!valid_pos(i, L, status)) return;          // an empty slot has no output
    const int bi = sv.Bk ? sv.Bk[i] : 0;
    float q[kDim], kv[kDim];
    load_row(X + (long long)i * kDim, q);
    const bool prev = (prev_mask >> (seg % R)) & 1u;
    const Window w = window_of(s, m, L, prev);
    float mx = -INFINITY;
    int cnt = 0;
    for (int t = w.w0; t < w.w1; ++t) {
        int j;
        if (t == s || !sv.candidate(t, i, bi, j)) continue;
        load_row(X + (long long)j * kDim, kv);
        float z = tau * (dot64(q, kv) * IN[j]);
        mx = fmaxf(mx, z);
        ++cnt;
    }
    float acc[kDim];
    float lse_i;
    if (cnt == 0 && prev) {               // nothing in the previous chunk: no contribution
        lse_i = -INFINITY;
#pragma unroll
        for (int k = 0; k < kDim; ++k) acc[k] = 0.f;
    } else if (cnt == 0) {                // self is the only candidate
        lse_i = self_penalty ? kSelfPenalty : tau * (dot64(q, q) * IN[i]);
        load_row(V + (long long)i * kDim, acc);
    } else {
#pragma unroll
        for (int k = 0; k < kDim; ++k) acc[k] = 0.f;
        float l = 0.f;
        for (int t = w.w0; t < w.w1; ++t) {
            int j;
            if (t == s || !sv.candidate(t, i, bi, j)) continue;
            load_row(X + (long long)j * kDim, kv);
            float e = expf(tau * (dot64(q, kv) * IN[j]) - mx);
            l += e;
            load_row(V + (long long)j * kDim, kv);
#pragma unroll
            for (int k = 0; k < kDim; ++k) acc[k] = fmaf(e, kv[k], acc[k]);
        }
        float inv = 1.0f / l;
#pragma unroll
        for (int k = 0; k < kDim; ++k) acc[k] *= inv;
        lse_i = mx + logf(l);
    }
    store_row(o_r + (seg * L + i) * kDim, acc);
    lse[seg * L + i] = lse_i;
}

cudaError_t launch_attn_fwd_simt(const Problem &p, const void *x, const void *v, const int32_t *perm,
                                 const float *invnorm, const uint16_t *bkt, float *o_r, float *lse,
                                 uint32_t *status, cudaStream_t st)
{
    if (p.dtype != LSH_F32) return cudaErrorInvalidValue;      // bf16 runs on the tensor-core kernels
    dim3 grid((p.L + 127) / 128, (unsigned)p.S());
    float tau = 1.0f / sqrtf((float)p.d);
    attn_fwd_simt_kernel<float><<<grid, 128, 0, st>>>(
        (const float *)x, (const float *)v, perm, invnorm, (p.flags & LSH_FLAG_BUCKET_MASK) ? bkt : nullptr, o_r,
        lse, p.L, p.R, p.m, p.causal, (p.flags & LSH_FLAG_SELF_PENALTY) ? 1 : 0, tau, (uint32_t)p.prev_mask, status);
    return cudaGetLastError();
}

// ------------------------------------------------------------------ merge
// "Multiple Hash Rounds": y_i = sum_r softmax_r(lse_r,i) o_r,i.
// 16 threads per token, four features each.
template <typename T, typename OT>
__global__ void combine_kernel(const OT *__restrict__ o_r, const float *__restrict__ lse, T *__restrict__ out,
                               float *__restrict__ lse_out, long long tokens, int L, int R)
{
    long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    long long tok = gid >> 4;
    int quad = (int)(gid & 15);
    if (tok >= tokens) return;
    long long bh = tok / L;
    int i = (int)(tok % L);
    // weights exp(lse_r - mx) / sum: computed relative to the largest lse, so that
    // lse values far from 0 (the self penalty) lose no precision
    float mx = -INFINITY;
    for (int r = 0; r < R; ++r) mx = fmaxf(mx, lse[(bh * R + r) * L + i]);
    float ssum = 0.f;
    for (int r = 0; r < R; ++r) ssum += expf(lse[(bh * R + r) * L + i] - mx);
    if (lse_out && quad == 0) lse_out[tok] = mx + logf(ssum);
    const float inv = 1.f / ssum;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int r = 0; r < R; ++r) {
        float wr = expf(lse[(bh * R + r) * L + i] - mx) * inv;
        const OT *o = o_r + ((bh * R + r) * L + i) * kDim + quad * 4;
#pragma unroll
        for (int k = 0; k < 4; ++k) acc[k] = fmaf(wr, to_f(o[k]), acc[k]);
    }
    T *y = out + tok * kDim + quad * 4;
#pragma unroll
    for (int k = 0; k < 4; ++k) y[k] = from_f<T>(acc[k]);
}

// bf16 round outputs: 8 threads per token, eight features each
// (combine_token_bf16).
template <int RMAX>
__global__ void combine_bf16_kernel(const __nv_bfloat16 *__restrict__ o_r, const float *__restrict__ lse,
                                    __nv_bfloat16 *__restrict__ out, float *__restrict__ lse_out, long long tokens,
                                    int L, int R)
{
    long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    long long tok = gid >> 3;
    int oct = (int)(gid & 7);
    if (tok >= tokens) return;
    long long bh = tok / L;
    int i = (int)(tok % L);
    const float *lp = lse + bh * R * (long long)L + i;
    const uint4 *orow = reinterpret_cast<const uint4 *>(o_r + (bh * R * (long long)L + i) * kDim) + oct;
    const long long rstride = (long long)L * kDim / 8;          // one round, in 16-byte units
    combine_token_bf16<RMAX, false>(orow, rstride, lp, L, R, reinterpret_cast<uint4 *>(out + tok * kDim) + oct,
                                    lse_out ? lse_out + tok : nullptr, oct);
}

cudaError_t launch_combine(const Problem &p, const void *o_r, bool o_r_bf16, const float *lse, void *out,
                           float *lse_out, cudaStream_t st)
{
    if (p.dtype == LSH_BF16) {
        if (!o_r_bf16) return cudaErrorInvalidValue;
        long long threads = p.tokens() * 8;
        const unsigned grid = (unsigned)((threads + 255) / 256);
        auto kern = p.R <= 4 ? combine_bf16_kernel<4> : p.R <= 8 ? combine_bf16_kernel<8> : combine_bf16_kernel<0>;
        kern<<<grid, 256, 0, st>>>((const __nv_bfloat16 *)o_r, lse, (__nv_bfloat16 *)out, lse_out, p.tokens(), p.L,
                                   p.R);
        return cudaGetLastError();
    }
    if (o_r_bf16) return cudaErrorInvalidValue;
    long long threads = p.tokens() * 16;
    unsigned grid = (unsigned)((threads + 255) / 256);
    combine_kernel<float, float><<<grid, 256, 0, st>>>((const float *)o_r, lse, (float *)out, lse_out, p.tokens(),
                                                       p.L, p.R);
    return cudaGetLastError();
}

// Slot orders of local attention: round 0 the positions in their own order,
// round 1 (its following-chunk part) in reversed order, so that the previous
// chunk of a slot there holds the following chunk of its position.
__global__ void local_perm_kernel(int32_t *__restrict__ perm, long long n, int L, int R)
{
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;   // over BH * R * L
    if (idx >= n) return;
    const int s = (int)(idx % L);
    const int r = (int)((idx / L) % R);
    perm[idx] = r == 0 ? s : L - 1 - s;
}

cudaError_t launch_local_perm(const Problem &p, int32_t *perm, cudaStream_t st)
{
    const long long n = p.S() * p.L;
    local_perm_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(perm, n, p.L, p.R);
    return cudaGetLastError();
}

// ------------------------------------------------------------------ backward prologue
// LSE_i = logsumexp over rounds of lse_r,i and delta_i = dY_i . Y_i; also
// zeroes the fp32 gradient accumulators.  16 threads per token.
//
// With P_rij = exp(z_rij - LSE_i) the merged output is y_i = sum_r,j P_rij v_j,
// so the backward of every round uses P_rij and dz_rij = P_rij (dY_i.v_j - delta_i).
// own (nullable, self penalty): the weight exp(kSelfPenalty - LSE_i) of a lone
// query's own entry, as exp(kSelfPenalty - mx) / sum_r exp(lse_r - mx) (mx the
// largest lse): LSE_i itself near -1e5 carries fp32 steps of 2^-7.
template <typename T>
__global__ void bwd_prep_kernel(const float *__restrict__ lse, const T *__restrict__ out, const T *__restrict__ dout,
                                float *__restrict__ lse_all, float *__restrict__ delta, float *__restrict__ own,
                                float *__restrict__ dx_acc, float *__restrict__ dv_acc, long long tokens, int L, int R)
{
    long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    long long tok = gid >> 4;
    int quad = (int)(gid & 15);
    bool valid = tok < tokens;
    float part = 0.f;
    if (valid) {
        const T *y = out + tok * kDim + quad * 4;
        const T *g = dout + tok * kDim + quad * 4;
#pragma unroll
        for (int k = 0; k < 4; ++k) part = fmaf(to_f(g[k]), to_f(y[k]), part);
        float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
        reinterpret_cast<float4 *>(dx_acc + tok * kDim)[quad] = z;
        reinterpret_cast<float4 *>(dv_acc + tok * kDim)[quad] = z;
    }
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    if (valid && quad == 0) {
        long long bh = tok / L;
        int i = (int)(tok % L);
        float mx = -INFINITY;
        for (int r = 0; r < R; ++r) mx = fmaxf(mx, lse[(bh * R + r) * L + i]);
        float ssum = 0.f;
        for (int r = 0; r < R; ++r) ssum += expf(lse[(bh * R + r) * L + i] - mx);
        lse_all[tok] = mx + logf(ssum);
        delta[tok] = part;
        if (own) own[tok] = expf(kSelfPenalty - mx) / ssum;
    }
}

__global__ void bwd_prep_bf16_kernel(const float *__restrict__ lse, const __nv_bfloat16 *__restrict__ out,
                                     const __nv_bfloat16 *__restrict__ dout, float *__restrict__ lse_all,
                                     float *__restrict__ delta, float *__restrict__ own, float *__restrict__ dx_acc,
                                     float *__restrict__ dv_acc, long long tokens, int L, int R)
{
    long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    long long tok = gid >> 3;
    int oct = (int)(gid & 7);
    bool valid = tok < tokens;
    float part = 0.f;
    if (valid) {
        const uint4 yu = reinterpret_cast<const uint4 *>(out + tok * kDim)[oct];
        const uint4 gu = reinterpret_cast<const uint4 *>(dout + tok * kDim)[oct];
        const uint32_t yw[4] = {yu.x, yu.y, yu.z, yu.w}, gw[4] = {gu.x, gu.y, gu.z, gu.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            part = fmaf(__uint_as_float(gw[e] << 16), __uint_as_float(yw[e] << 16), part);
            part = fmaf(__uint_as_float(gw[e] & 0xFFFF0000u), __uint_as_float(yw[e] & 0xFFFF0000u), part);
        }
        const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
        float4 *dxp = reinterpret_cast<float4 *>(dx_acc + tok * kDim) + 2 * oct;
        float4 *dvp = reinterpret_cast<float4 *>(dv_acc + tok * kDim) + 2 * oct;
        dxp[0] = z; dxp[1] = z; dvp[0] = z; dvp[1] = z;
    }
#pragma unroll
    for (int o = 4; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    if (valid && oct == 0) {
        long long bh = tok / L;
        int i = (int)(tok % L);
        const float *lp = lse + bh * R * (long long)L + i;
        float mx = -INFINITY;
        for (int r = 0; r < R; ++r) mx = fmaxf(mx, lp[(long long)r * L]);
        float ssum = 0.f;
        for (int r = 0; r < R; ++r) ssum += expf(lp[(long long)r * L] - mx);
        lse_all[tok] = mx + logf(ssum);
        delta[tok] = part;
        if (own) own[tok] = expf(kSelfPenalty - mx) / ssum;
    }
}

cudaError_t launch_bwd_prep(const Problem &p, const float *lse, const void *out, const void *dout,
                            float *lse_all, float *delta, float *own, float *dx_acc, float *dv_acc, cudaStream_t st)
{
    if (p.dtype == LSH_BF16) {
        long long threads = p.tokens() * 8;
        bwd_prep_bf16_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, st>>>(
            lse, (const __nv_bfloat16 *)out, (const __nv_bfloat16 *)dout, lse_all, delta, own, dx_acc, dv_acc,
            p.tokens(), p.L, p.R);
        return cudaGetLastError();
    }
    long long threads = p.tokens() * 16;
    unsigned grid = (unsigned)((threads + 255) / 256);
    bwd_prep_kernel<float><<<grid, 256, 0, st>>>(lse, (const float *)out, (const float *)dout, lse_all, delta, own,
                                                 dx_acc, dv_acc, p.tokens(), p.L, p.R);
    return cudaGetLastError();
}

// ------------------------------------------------------------------ backward, query role
// One thread per (segment, sorted slot s) with query position i:
//   dx_i += sum_j dz_ij tau k_j,   k_j = x_j invnorm_j.
// Also records whether the slot attends to itself alone (needed by the key pass).
// With the self penalty that lone entry has a constant score: no gradient to x.
template <typename T>
__global__ void attn_bwd_q_simt_kernel(const T *__restrict__ x, const T *__restrict__ v, const T *__restrict__ dout,
                                       const int32_t *__restrict__ perm, const float *__restrict__ invnorm,
                                       const uint16_t *__restrict__ bkt, const float *__restrict__ lse_all,
                                       const float *__restrict__ delta, uint8_t *__restrict__ self_only,
                                       float *__restrict__ dx_acc, int L, int R, int m, int causal,
                                       int self_penalty, float tau, uint32_t prev_mask, uint32_t *__restrict__ status)
{
    const long long seg = blockIdx.y;
    const int s = blockIdx.x * blockDim.x + threadIdx.x;
    if (s >= L) return;
    const long long bh = seg / R;
    const SlotView sv{perm + seg * L, bkt ? bkt + seg * L : nullptr, L, causal, status};
    const T *X = x + bh * L * kDim;
    const T *V = v + bh * L * kDim;
    const float *IN = invnorm + bh * L;
    const int i = sv.P[s];
    if (!valid_pos(i, L, status)) {
        self_only[seg * L + s] = 0;
        return;
    }
    const int bi = sv.Bk ? sv.Bk[i] : 0;
    float q[kDim], g[kDim], kv[kDim], dq[kDim];
    load_row(X + (long long)i * kDim, q);
    load_row(dout + (bh * L + i) * kDim, g);
#pragma unroll
    for (int k = 0; k < kDim; ++k) dq[k] = 0.f;
    const float big = lse_all[bh * L + i], dl = delta[bh * L + i];
    const bool prev = (prev_mask >> (seg % R)) & 1u;
    const Window w = window_of(s, m, L, prev);
    int cnt = 0;
    for (int t = w.w0; t < w.w1; ++t) {
        int j;
        if (t == s || !sv.candidate(t, i, bi, j)) continue;
        ++cnt;
        load_row(X + (long long)j * kDim, kv);
        float pij = expf(tau * (dot64(q, kv) * IN[j]) - big);
        float c = tau * IN[j];
        float kvv[kDim];
        load_row(V + (long long)j * kDim, kvv);
        float dz = pij * (dot64(g, kvv) - dl);
#pragma unroll
        for (int k = 0; k < kDim; ++k) dq[k] = fmaf(dz * c, kv[k], dq[k]);
    }
    if (cnt == 0 && !self_penalty && !prev) {
        float pij = expf(tau * (dot64(q, q) * IN[i]) - big);
        load_row(V + (long long)i * kDim, kv);
        float dz = pij * (dot64(g, kv) - dl);
        float c = tau * IN[i];
#pragma unroll
        for (int k = 0; k < kDim; ++k) dq[k] = dz * c * q[k];
    }
    self_only[seg * L + s] = cnt == 0 && !prev;
    float *dst = dx_acc + (bh * L + i) * kDim;
#pragma unroll
    for (int k = 0; k < kDim; ++k) atomicAdd(dst + k, dq[k]);
}

// ------------------------------------------------------------------ backward, key role
// One thread per (segment, sorted slot t) with key position j.  The queries
// whose window holds t sit in chunks c(t) and c(t)+1:
//   g_j  = sum_s dz_sj tau x_s          (gradient w.r.t. the unit key k_j)
//   dx_j += invnorm_j (g_j - k_j (k_j . g_j)),   dv_j += sum_s P_sj dY_s.
// A lone query's own entry with the self penalty has P = exp(kSelfPenalty - LSE)
// and a constant score: it adds to dv only.
template <typename T>
__global__ void attn_bwd_k_simt_kernel(const T *__restrict__ x, const T *__restrict__ v, const T *__restrict__ dout,
                                       const int32_t *__restrict__ perm, const float *__restrict__ invnorm,
                                       const uint16_t *__restrict__ bkt, const float *__restrict__ lse_all,
                                       const float *__restrict__ delta, const float *__restrict__ own,
                                       const uint8_t *__restrict__ self_only,
                                       float *__restrict__ dx_acc, float *__restrict__ dv_acc, int L, int R, int m,
                                       int causal, int self_penalty, float tau, uint32_t prev_mask,
                                       uint32_t *__restrict__ status)
{
    const long long seg = blockIdx.y;
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= L) return;
    const long long bh = seg / R;
    const int32_t *P = perm + seg * L;
    const uint16_t *Bk = bkt ? bkt + seg * L : nullptr;
    const T *X = x + bh * L * kDim;
    const float *IN = invnorm + bh * L;
    const int j = P[t];
    if (!valid_pos(j, L, status)) return;
    const int bj = Bk ? Bk[j] : 0;
    float kx[kDim], vj[kDim], gk[kDim], dvj[kDim], q[kDim], g[kDim];
    load_row(X + (long long)j * kDim, kx);
    load_row(v + (bh * L + j) * kDim, vj);
#pragma unroll
    for (int k = 0; k < kDim; ++k) { gk[k] = 0.f; dvj[k] = 0.f; }
    const float inj = IN[j];
    // queries whose window holds slot t: chunks c and c + 1 (c = t / m), or only
    // c + 1 when the window is the previous chunk alone
    const int c = t / m;
    const bool prev = (prev_mask >> (seg % R)) & 1u;
    const int s0 = (prev ? c + 1 : c) * m, s1 = min((c + 2) * m, L);
    for (int s = s0; s < s1; ++s) {
        int i = P[s];
        if (!valid_pos(i, L, status)) continue;
        if (s == t) {
            if (self_only[seg * L + s] == 0) continue;
            if (self_penalty) {
                load_row(dout + (bh * L + i) * kDim, g);
                const float pij = own[bh * L + i];                // exp(kSelfPenalty - LSE_i)
#pragma unroll
                for (int k = 0; k < kDim; ++k) dvj[k] = fmaf(pij, g[k], dvj[k]);
                continue;
            }
        } else {
            if (causal && j > i) continue;
            if (Bk && Bk[i] != bj) continue;
        }
        load_row(X + (long long)i * kDim, q);
        load_row(dout + (bh * L + i) * kDim, g);
        float pij = expf(tau * (dot64(q, kx) * inj) - lse_all[bh * L + i]);
        float dz = pij * (dot64(g, vj) - delta[bh * L + i]);
#pragma unroll
        for (int k = 0; k < kDim; ++k) {
            gk[k] = fmaf(dz * tau, q[k], gk[k]);
            dvj[k] = fmaf(pij, g[k], dvj[k]);
        }
    }
    // through k_j = x_j / |x_j|: dx_j = invnorm_j (g - k (k . g)), k = x_j invnorm_j
    float kg = 0.f;
#pragma unroll
    for (int k = 0; k < kDim; ++k) kg = fmaf(kx[k] * inj, gk[k], kg);
    float *dxd = dx_acc + (bh * L + j) * kDim;
    float *dvd = dv_acc + (bh * L + j) * kDim;
#pragma unroll
    for (int k = 0; k < kDim; ++k) {
        atomicAdd(dxd + k, inj * (gk[k] - kx[k] * inj * kg));
        atomicAdd(dvd + k, dvj[k]);
    }
}

cudaError_t launch_attn_bwd_simt(const Problem &p, const void *x, const void *v, const void *dout,
                                 const int32_t *perm, const float *invnorm, const uint16_t *bkt,
                                 const float *lse_all, const float *delta, const float *own, uint8_t *self_only,
                                 float *dx_acc, float *dv_acc, uint32_t *status, cudaStream_t st)
{
    if (p.dtype != LSH_F32) return cudaErrorInvalidValue;      // bf16 runs on the tensor-core kernels
    dim3 grid((p.L + 127) / 128, (unsigned)p.S());
    float tau = 1.0f / sqrtf((float)p.d);
    const uint16_t *bk = (p.flags & LSH_FLAG_BUCKET_MASK) ? bkt : nullptr;
    const int pen = (p.flags & LSH_FLAG_SELF_PENALTY) ? 1 : 0;
    attn_bwd_q_simt_kernel<float><<<grid, 128, 0, st>>>((const float *)x, (const float *)v, (const float *)dout,
                                                        perm, invnorm, bk, lse_all, delta, self_only, dx_acc, p.L,
                                                        p.R, p.m, p.causal, pen, tau, (uint32_t)p.prev_mask, status);
    attn_bwd_k_simt_kernel<float><<<grid, 128, 0, st>>>((const float *)x, (const float *)v, (const float *)dout,
                                                        perm, invnorm, bk, lse_all, delta, own, self_only, dx_acc,
                                                        dv_acc, p.L, p.R, p.m, p.causal, pen, tau,
                                                        (uint32_t)p.prev_mask, status);
    return cudaGetLastError();
}

// ------------------------------------------------------------------ backward epilogue
// Eight elements of each accumulator per thread: two 16-byte loads per array
// and one 16-byte store of eight bf16 (or two of fp32) per output.
template <typename T>
__global__ void bwd_finalize_kernel(const float *__restrict__ dx_acc, const float *__restrict__ dv_acc,
                                    T *__restrict__ dqk, T *__restrict__ dv, long long n8)
{
    long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n8) return;
    const float4 a0 = reinterpret_cast<const float4 *>(dx_acc)[2 * i], a1 = reinterpret_cast<const float4 *>(dx_acc)[2 * i + 1];
    const float4 b0 = reinterpret_cast<const float4 *>(dv_acc)[2 * i], b1 = reinterpret_cast<const float4 *>(dv_acc)[2 * i + 1];
    if constexpr (sizeof(T) == 2) {
        reinterpret_cast<uint4 *>(dqk)[i] = make_uint4(pack_bf16x2(a0.x, a0.y), pack_bf16x2(a0.z, a0.w),
                                                       pack_bf16x2(a1.x, a1.y), pack_bf16x2(a1.z, a1.w));
        reinterpret_cast<uint4 *>(dv)[i] = make_uint4(pack_bf16x2(b0.x, b0.y), pack_bf16x2(b0.z, b0.w),
                                                      pack_bf16x2(b1.x, b1.y), pack_bf16x2(b1.z, b1.w));
    } else {
        reinterpret_cast<float4 *>(dqk)[2 * i] = a0;
        reinterpret_cast<float4 *>(dqk)[2 * i + 1] = a1;
        reinterpret_cast<float4 *>(dv)[2 * i] = b0;
        reinterpret_cast<float4 *>(dv)[2 * i + 1] = b1;
    }
}

cudaError_t launch_bwd_finalize(const Problem &p, const float *dx_acc, const float *dv_acc, void *dqk, void *dv,
                                cudaStream_t st)
{
    long long n8 = p.tokens() * kDim / 8;
    unsigned grid = (unsigned)((n8 + 255) / 256);
    if (p.dtype == LSH_F32)
        bwd_finalize_kernel<float><<<grid, 256, 0, st>>>(dx_acc, dv_acc, (float *)dqk, (float *)dv, n8);
    else
        bwd_finalize_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(dx_acc, dv_acc, (__nv_bfloat16 *)dqk,
                                                                 (__nv_bfloat16 *)dv, n8);
    return cudaGetLastError();
}

}  // namespace lsh
