// unsort_combine for one token ("Multiple Hash Rounds", paper note
// "Reformer"): y_i = sum_r softmax_r(lse_r,i) o_r,i, with the rounds' outputs
// o_r,i (bf16, at the token's original position) and logsumexps lse_r,i.
// Used by the round-merge kernel and by the single-kernel forward, so both
// give the same bits.
#pragma once
#include "common.cuh"

namespace lsh {

// Eight threads per token, eight features each (16-byte loads and stores).
// orow: the token's round-0 row seen as 16-byte units, this thread's unit
// included (rstride units apart per round); lp: the token's round-0 lse (L
// apart per round).  L2ONLY: the rows were written by other CTAs of the same
// kernel, so they are read through L2 (ld.global.cg), not the read-only path.
template <int RMAX, bool L2ONLY>
__device__ __forceinline__ void combine_load(const uint4 *orow, long long rstride, const float *lp, int L, int R,
                                             uint4 (&u)[RMAX], float (&lr)[RMAX])
{
#pragma unroll
    for (int r = 0; r < RMAX; ++r) {
        u[r] = r < R ? (L2ONLY ? __ldcg(orow + r * rstride) : __ldg(orow + r * rstride)) : make_uint4(0, 0, 0, 0);
        lr[r] = r < R ? (L2ONLY ? __ldcg(lp + (long long)r * L) : __ldg(lp + (long long)r * L)) : -INFINITY;
    }
}

__device__ __forceinline__ void combine_accumulate(float (&acc)[8], float wr, const uint4 &u)
{
    const uint32_t wd[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        acc[2 * e] = fmaf(wr, __uint_as_float(wd[e] << 16), acc[2 * e]);
        acc[2 * e + 1] = fmaf(wr, __uint_as_float(wd[e] & 0xFFFF0000u), acc[2 * e + 1]);
    }
}

// The merge of R <= RMAX loaded rounds.  Weights exp(lse_r - max) / sum are
// computed relative to the largest lse, so that lse values far from 0 (the
// self penalty) lose no precision.  lse_out (nullable): the logsumexp over the
// rounds, written by the token's first thread.
template <int RMAX>
__device__ __forceinline__ uint4 combine_rows(const uint4 (&u)[RMAX], const float (&lr)[RMAX], int R,
                                              float *lse_out, int oct)
{
    float mx = -INFINITY;
#pragma unroll
    for (int r = 0; r < RMAX; ++r) mx = fmaxf(mx, lr[r]);
    float w[RMAX], ssum = 0.f;
#pragma unroll
    for (int r = 0; r < RMAX; ++r) {
        w[r] = r < R ? expf(lr[r] - mx) : 0.f;
        ssum += w[r];
    }
    const float inv = 1.f / ssum;
    if (lse_out && oct == 0) *lse_out = mx + logf(ssum);
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int r = 0; r < RMAX; ++r) combine_accumulate(acc, w[r] * inv, u[r]);
    return make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]), pack_bf16x2(acc[4], acc[5]),
                      pack_bf16x2(acc[6], acc[7]));
}

// One token: RMAX > 0 loads the R <= RMAX round rows before any arithmetic, so
// their memory latencies overlap; RMAX = 0 handles any R one round at a time
// (the same arithmetic in the same order).
template <int RMAX, bool L2ONLY>
__device__ __forceinline__ void combine_token_bf16(const uint4 *orow, long long rstride, const float *lp, int L, int R,
                                                   uint4 *yout, float *lse_out, int oct)
{
    if constexpr (RMAX > 0) {
        uint4 u[RMAX];
        float lr[RMAX];
        combine_load<RMAX, L2ONLY>(orow, rstride, lp, L, R, u, lr);
        *yout = combine_rows<RMAX>(u, lr, R, lse_out, oct);
    } else {
        float mx = -INFINITY;
        for (int r = 0; r < R; ++r) mx = fmaxf(mx, __ldg(lp + (long long)r * L));
        float ssum = 0.f;
        for (int r = 0; r < R; ++r) ssum += expf(__ldg(lp + (long long)r * L) - mx);
        if (lse_out && oct == 0) *lse_out = mx + logf(ssum);
        const float inv = 1.f / ssum;
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int r = 0; r < R; ++r)
            combine_accumulate(acc, expf(__ldg(lp + (long long)r * L) - mx) * inv, __ldg(orow + r * rstride));
        *yout = make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]), pack_bf16x2(acc[4], acc[5]),
                           pack_bf16x2(acc[6], acc[7]));
    }
}

}  // namespace lsh
