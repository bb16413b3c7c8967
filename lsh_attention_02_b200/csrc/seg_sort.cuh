// Stable sort of one segment's bucket ids by one CTA in shared memory
// ("Sorting and Chunking", paper note "Reformer": tokens sorted by bucket,
// original order kept inside a bucket).  Used by the on-chip segment sort
// kernel and by the single-kernel forward of short segments.
//
// Each warp counts the ids of its own contiguous run of positions, one
// exclusive scan in (bucket, warp) order gives every warp's first output slot
// per bucket, and each warp places its run in position order (equal ids inside
// a 32-position step ranked by lane, the lanes found with one ballot per id
// bit), so the result is the stable sort.  An id >= n_buckets (invalid input)
// is counted as n_buckets - 1, which keeps every access in bounds.
#pragma once
#include "common.cuh"

namespace lsh {

// Lanes of the warp whose key equals this lane's, from one ballot per key bit
// (keys below 2^nbits; a lane with key 2^nbits, an out-of-range marker, matches
// only lanes with the same marker).
__device__ __forceinline__ uint32_t peers_of(uint32_t key, int nbits)
{
    uint32_t peers = 0xffffffffu;
    for (int bit = 0; bit <= nbits; ++bit) {
        const bool set = (key >> bit) & 1u;
        const uint32_t bal = __ballot_sync(0xffffffffu, set);
        peers &= set ? bal : ~bal;
    }
    return peers;
}
__device__ __forceinline__ int bits_for(int n)      // smallest b with 2^b >= n
{
    int b = 0;
    while ((1 << b) < n) ++b;
    return b;
}

// Called by all NW * 32 threads of the CTA once `keys` [L] is complete in
// shared memory and visible (after a barrier).  Scratch in shared memory:
// wh [nb * NW], warp_tot [32].  Writes perm [L] (shared memory): perm[slot] =
// the position sorted to that slot.  Ends with a barrier.
template <int NW>
__device__ __forceinline__ void seg_sort_block(const uint16_t *keys, int L, int nb, uint32_t *wh, uint32_t *warp_tot,
                                               int32_t *perm)
{
    static_assert(NW <= 32, "one warp scans the warp totals");
    constexpr int kT = NW * 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t lt_mask = (1u << lane) - 1u;
    const int nbits = bits_for(nb);
    for (int e = threadIdx.x; e < nb * NW; e += kT) wh[e] = 0;
    __syncthreads();
    const int run = (L + kT - 1) / kT * 32;      // positions per warp, a multiple of 32
    const int p0 = warp * run;
    // A: per-warp counts of every bucket id, in position order
    for (int it = 0; it < run; it += 32) {
        const int pos = p0 + it + lane;
        const bool valid = pos < L;
        const uint32_t b = valid ? min((uint32_t)keys[pos], (uint32_t)(nb - 1)) : (1u << nbits);
        const uint32_t peers = peers_of(b, nbits);
        if (valid && (peers & lt_mask) == 0) wh[b * NW + warp] += __popc(peers);
        __syncwarp();
    }
    __syncthreads();
    // B: exclusive scan of wh in (bucket, warp) order; thread t scans a contiguous span
    const int n = nb * NW, per = (n + kT - 1) / kT;
    const int e0 = min(n, (int)threadIdx.x * per), e1 = min(n, e0 + per);
    uint32_t tot = 0;
    for (int e = e0; e < e1; ++e) tot += wh[e];
    uint32_t incl = tot;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const uint32_t wv = lane < NW ? warp_tot[lane] : 0u;
        uint32_t wi = wv;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t t = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += t;
        }
        if (lane < NW) warp_tot[lane] = wi - wv;
    }
    __syncthreads();
    uint32_t off = warp_tot[warp] + incl - tot;
    for (int e = e0; e < e1; ++e) {
        const uint32_t c = wh[e];
        wh[e] = off;
        off += c;
    }
    __syncthreads();
    // C: stable placement
    for (int it = 0; it < run; it += 32) {
        const int pos = p0 + it + lane;
        const bool valid = pos < L;
        const uint32_t b = valid ? min((uint32_t)keys[pos], (uint32_t)(nb - 1)) : (1u << nbits);
        const uint32_t peers = peers_of(b, nbits);
        const uint32_t slot = valid ? wh[b * NW + warp] + __popc(peers & lt_mask) : 0u;
        __syncwarp();
        if (valid && (peers & lt_mask) == 0) wh[b * NW + warp] += __popc(peers);
        __syncwarp();
        if (valid) perm[slot] = pos;
    }
    __syncthreads();
}

}  // namespace lsh
