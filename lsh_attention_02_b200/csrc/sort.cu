// Stable segmented radix sort of positions by bucket id.
//
// "Sorting and Chunking" (paper note "Reformer"): after hashing, tokens are
// sorted by bucket.  Inside a bucket the order is the original position
// order, so the sort is stable.  Each (batch, head, round) segment of L
// bucket ids is sorted independently.
//
// Segments of up to kSegMaxL positions with up to kSegMaxBuckets buckets are
// sorted by one CTA in shared memory (below).  Longer ones: a
// least-significant-digit radix sort with at most two passes of <= 8 bits
// (bucket ids have <= 16 bits).  Each pass is three kernels:
//   count   per 2048-position tile, a shared-memory histogram of the digit;
//           written digit-major: counts[seg][digit][tile];
//   scan    per segment, an exclusive scan over (digit, tile) in that order,
//           which is exactly the output offset of (digit, tile)'s first element;
//   scatter per tile, a stable rank of each element among equal digits
//           (warp-private histograms; inside a warp, the lanes holding the
//           same digit found with one ballot per digit bit), then the
//           element is written at offset + rank.
// Pass 0 reads the bucket ids in position order with the position as the
// value; the last pass writes only the values, i.e. the permutation.

#include "seg_sort.cuh"

namespace lsh {

SortPlan make_sort_plan(int n_buckets, int L)
{
    SortPlan sp{};
    int bits = 1;
    while ((1 << bits) < n_buckets) ++bits;
    sp.passes = bits <= 8 ? 1 : 2;
    sp.bits[0] = (bits + sp.passes - 1) / sp.passes;
    sp.bits[1] = bits - sp.bits[0];
    sp.shift[0] = 0;
    sp.shift[1] = sp.bits[0];
    sp.n_tiles = (L + kSortTile - 1) / kSortTile;
    sp.max_radix = 1 << sp.bits[0];
    return sp;
}


__global__ void __launch_bounds__(kSortThreads)
radix_count_kernel(const uint16_t *__restrict__ keys, uint32_t *__restrict__ counts, int L, int n_tiles,
                   int shift, int radix)
{
    __shared__ uint32_t hist[256];
    const long long seg = blockIdx.y;
    const int tile = blockIdx.x;
    for (int d = threadIdx.x; d < radix; d += blockDim.x) hist[d] = 0;
    __syncthreads();
    const uint16_t *k = keys + seg * L;
    for (int e = threadIdx.x; e < kSortTile; e += blockDim.x) {
        int pos = tile * kSortTile + e;
        if (pos < L) atomicAdd(&hist[(k[pos] >> shift) & (radix - 1)], 1u);
    }
    __syncthreads();
    for (int d = threadIdx.x; d < radix; d += blockDim.x)
        counts[(seg * radix + d) * n_tiles + tile] = hist[d];
}

// In-place exclusive scan of n counters per segment; one 1024-thread block per segment.
__global__ void __launch_bounds__(1024)
radix_scan_kernel(uint32_t *__restrict__ counts, int n)
{
    __shared__ uint32_t warp_tot[32];
    __shared__ uint32_t carry_s;
    uint32_t *p = counts + (long long)blockIdx.x * n;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (threadIdx.x == 0) carry_s = 0;
    __syncthreads();
    for (int base = 0; base < n; base += 1024) {
        int idx = base + threadIdx.x;
        uint32_t v = idx < n ? p[idx] : 0u;
        uint32_t incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += t;
        }
        if (lane == 31) warp_tot[warp] = incl;
        __syncthreads();
        if (warp == 0) {
            uint32_t w = warp_tot[lane];
            uint32_t wi = w;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                uint32_t t = __shfl_up_sync(0xffffffffu, wi, o);
                if (lane >= o) wi += t;
            }
            warp_tot[lane] = wi - w;           // exclusive prefix of warp totals
        }
        __syncthreads();
        uint32_t carry = carry_s;
        if (idx < n) p[idx] = carry + warp_tot[warp] + incl - v;
        __syncthreads();
        if (threadIdx.x == 1023) carry_s = carry + warp_tot[31] + incl;
        __syncthreads();
    }
}

__global__ void __launch_bounds__(kSortThreads)
radix_scatter_kernel(const uint16_t *__restrict__ keys_in, const int32_t *__restrict__ vals_in,
                     const uint32_t *__restrict__ offsets, uint16_t *__restrict__ keys_out,
                     int32_t *__restrict__ vals_out, int L, int n_tiles, int shift, int radix)
{
    constexpr int kWarps = kSortThreads / 32;
    constexpr int kPerWarp = kSortTile / kWarps;          // 256 consecutive positions per warp
    __shared__ uint32_t wh[kWarps][256];
    const long long seg = blockIdx.y;
    const int tile = blockIdx.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t lt_mask = (1u << lane) - 1u;
    const int rbits = bits_for(radix);
    for (int d = lane; d < radix; d += 32) wh[warp][d] = 0;
    __syncwarp();
    const uint16_t *kin = keys_in + seg * L;

    // A: per-warp digit counts, in position order
    for (int it = 0; it < kPerWarp / 32; ++it) {
        int pos = tile * kSortTile + warp * kPerWarp + it * 32 + lane;
        bool valid = pos < L;
        uint32_t dg = valid ? ((kin[pos] >> shift) & (radix - 1)) : (uint32_t)radix;
        uint32_t peers = peers_of(dg, rbits);
        if (valid && (peers & lt_mask) == 0) wh[warp][dg] += __popc(peers);
        __syncwarp();
    }
    __syncthreads();
    // B: warp base = tile offset of the digit + counts of earlier warps
    for (int d = threadIdx.x; d < radix; d += blockDim.x) {
        uint32_t run = offsets[(seg * radix + d) * n_tiles + tile];
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            uint32_t c = wh[w][d];
            wh[w][d] = run;
            run += c;
        }
    }
    __syncthreads();
    // C: stable scatter
    for (int it = 0; it < kPerWarp / 32; ++it) {
        int pos = tile * kSortTile + warp * kPerWarp + it * 32 + lane;
        bool valid = pos < L;
        uint16_t key = valid ? kin[pos] : 0;
        uint32_t dg = valid ? ((key >> shift) & (radix - 1)) : (uint32_t)radix;
        uint32_t peers = peers_of(dg, rbits);
        uint32_t rank = valid ? wh[warp][dg] + __popc(peers & lt_mask) : 0u;
        __syncwarp();
        if (valid && (peers & lt_mask) == 0) wh[warp][dg] += __popc(peers);
        __syncwarp();
        if (valid) {
            int32_t val = vals_in ? vals_in[seg * L + pos] : pos;
            vals_out[seg * L + rank] = val;
            if (keys_out) keys_out[seg * L + rank] = key;
        }
    }
}

// ------------------------------------------------------------ small segments
// A segment of at most kSegMaxL positions and kSegMaxBuckets buckets is sorted
// by one CTA entirely in shared memory (seg_sort_block: per-warp counts, one
// scan in (bucket, warp) order, stable placement); the permutation is
// assembled in shared memory and written out with coalesced stores.
constexpr int kSegThreads = 1024;
constexpr int kSegWarps = kSegThreads / 32;

// Shared memory sized to the problem (so that two CTAs share an SM when they
// fit): perm [L], warp_tot [32], wh [n_buckets][32 warps], keys [L].
struct SegSortSmem {
    int32_t *perm;
    uint32_t *warp_tot, *wh;
    uint16_t *keys;
};
__host__ __device__ inline size_t seg_sort_smem_bytes(int L, int nb)
{
    return (size_t)L * 4 + kSegWarps * 4 + (size_t)nb * kSegWarps * 4 + ((size_t)L * 2 + 15) / 16 * 16;
}
__device__ inline SegSortSmem seg_sort_layout(uint8_t *base, int L, int nb)
{
    SegSortSmem m;
    m.perm = reinterpret_cast<int32_t *>(base);
    m.warp_tot = reinterpret_cast<uint32_t *>(base + (size_t)L * 4);
    m.wh = m.warp_tot + kSegWarps;
    m.keys = reinterpret_cast<uint16_t *>(m.wh + (size_t)nb * kSegWarps);
    return m;
}

__global__ void __launch_bounds__(kSegThreads)
seg_sort_kernel(const uint16_t *__restrict__ buckets, int32_t *__restrict__ perm, int L, int nb)
{
    extern __shared__ __align__(16) uint8_t seg_smem[];
    const SegSortSmem sm = seg_sort_layout(seg_smem, L, nb);
    const long long seg = blockIdx.x;
    const uint16_t *k = buckets + seg * L;
    for (int e = threadIdx.x; e < L; e += kSegThreads) sm.keys[e] = k[e];
    __syncthreads();
    seg_sort_block<kSegWarps>(sm.keys, L, nb, sm.wh, sm.warp_tot, sm.perm);
    int32_t *out = perm + seg * L;
    for (int e = threadIdx.x; e < L; e += kSegThreads) out[e] = sm.perm[e];
}

bool seg_sort_fits(const Problem &p) { return p.L <= kSegMaxL && p.nb <= kSegMaxBuckets; }

cudaError_t launch_sort(const Problem &p, const uint16_t *buckets, int32_t *perm, const Workspace &ws,
                        cudaStream_t st)
{
    if (seg_sort_fits(p)) {
        const size_t smem = seg_sort_smem_bytes(p.L, p.nb);
        cudaError_t e = cudaFuncSetAttribute(seg_sort_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)seg_sort_smem_bytes(kSegMaxL, kSegMaxBuckets));
        if (e != cudaSuccess) return e;
        seg_sort_kernel<<<(unsigned)p.S(), kSegThreads, smem, st>>>(buckets, perm, p.L, p.nb);
        return cudaGetLastError();
    }
    const SortPlan sp = make_sort_plan(p.nb, p.L);
    const dim3 grid(sp.n_tiles, (unsigned)p.S());
    const uint16_t *kin = buckets;
    const int32_t *vin = nullptr;
    for (int pass = 0; pass < sp.passes; ++pass) {
        const int radix = 1 << sp.bits[pass];
        const bool last = pass == sp.passes - 1;
        radix_count_kernel<<<grid, kSortThreads, 0, st>>>(kin, ws.sort_counts, p.L, sp.n_tiles, sp.shift[pass], radix);
        radix_scan_kernel<<<(unsigned)p.S(), 1024, 0, st>>>(ws.sort_counts, radix * sp.n_tiles);
        radix_scatter_kernel<<<grid, kSortThreads, 0, st>>>(kin, vin, ws.sort_counts, last ? nullptr : ws.sort_keys,
                                                            last ? perm : ws.sort_vals, p.L, sp.n_tiles,
                                                            sp.shift[pass], radix);
        kin = ws.sort_keys;
        vin = ws.sort_vals;
    }
    return cudaGetLastError();
}

// ------------------------------------------------------------ fixed scratch
// Scratch of lsh_attn_sort_static: one array per device, part of this
// module's static device memory, so the entry point itself never allocates.
// The driver creates it when the module is loaded; its address is looked up
// on each call.
static __device__ __align__(256) unsigned char g_sort_scratch[kStaticSortScratchBytes];

Workspace plan_sort_scratch(const Problem &p, char *base, size_t *bytes)
{
    Workspace w{};
    size_t off = 0;
    auto take = [&](size_t n) -> char * {
        char *ptr = base ? base + off : nullptr;
        off = (off + n + 255) / 256 * 256;
        return ptr;
    };
    const size_t S = (size_t)p.S(), L = (size_t)p.L;
    const SortPlan sp = make_sort_plan(p.nb, p.L);
    const bool small = seg_sort_fits(p);                 // sorted on chip: no scratch
    w.sort_keys = (uint16_t *)take(!small && sp.passes > 1 ? S * L * sizeof(uint16_t) : 0);
    w.sort_vals = (int32_t *)take(!small && sp.passes > 1 ? S * L * sizeof(int32_t) : 0);
    w.sort_counts = (uint32_t *)take(small ? 0 : S * (size_t)sp.max_radix * sp.n_tiles * sizeof(uint32_t));
    w.bytes = off;
    if (bytes) *bytes = off;
    return w;
}

cudaError_t static_sort_scratch(void **ptr)
{
    // Looked up on every call, on the current device and context: the address
    // is not cached, so a device reset (which reloads the module) or another
    // current context never leaves a stale pointer.
    void *a = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&a, g_sort_scratch);
    if (e != cudaSuccess) return e;
    *ptr = a;
    return cudaSuccess;
}

}  // namespace lsh
