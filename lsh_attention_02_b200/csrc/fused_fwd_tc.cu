// Single-kernel forward of short segments: lsh_hash, bucket_sort, gather +
// chunk_attn and unsort_combine of one (batch, head) in one cluster of R CTAs,
// CTA r taking round r ("Sorting and Chunking", "Multiple Hash Rounds", paper
// note "Reformer").  The bucket ids, ranks, counts and the permutation stay in
// shared memory between the steps; the key norms pass through L2, and the
// rounds' outputs are read back by the merge (from L2 where they are still
// resident, otherwise from HBM).
//
// Per CTA (segment (bh, r), L <= kMaxL positions, n_buckets <= 2 kMaxHalf):
//   hash       split over the cluster: CTA r loads x tiles r, r + R, ... of the
//              head (TMA tile loads, 128 rows, 128-byte swizzle) into a ring laid
//              over the attention stages' memory and multiplies each by the
//              rotations of every round at once on the tensor cores (M = 128, N up
//              to 128 columns per MMA, into TMEM); two groups of four warps take
//              alternate products: per round the first maximum of
//              [x R_r ; -x R_r] ("LSH Attention", hash equation; the oracle's tie
//              rule), and for each warp's 32 consecutive positions their rank
//              among equal ids and the group's count per id (one ballot per id
//              bit), all written into that round's CTA (distributed shared
//              memory); 1/|x| of each row to global memory;
//   sort       a stable counting sort from those counts: one exclusive scan in
//              (bucket, group) order gives every group's first slot per bucket,
//              and each position goes to that slot plus its rank; the
//              permutation stays in shared memory, and it and the bucket ids
//              are also written to global memory (the backward takes them);
//   attention  the roles of attn_fwd_roles.cuh over the segment's tiles in
//              order, positions, norms and buckets read from shared memory; o_r
//              rows and lse_r are stored at the original positions;
//   merge      after a cluster barrier (every round's o_r and lse_r written),
//              CTA r merges rows [r L/R, (r+1) L/R) of the head
//              (combine_token_bf16, the merge kernel's arithmetic).
//
// Every wait on an mbarrier is bounded (the status word gets the timeout bit
// and every role unwinds); the cluster barrier is reached by every thread of
// every CTA on every path.
#include <cooperative_groups.h>

#include "attn_fwd_roles.cuh"
#include "combine.cuh"
#include "seg_sort.cuh"

namespace cg = cooperative_groups;

// Tuning build: the global timer (ns) of every CTA at its phase boundaries.
#ifdef LSH_PHASE_TRACE
static __device__ unsigned long long lsh_cta_trace[1024][6];
#define LSH_CTA_MARK(ev)                                                          \
    do {                                                                          \
        if (threadIdx.x == 0 && blockIdx.x < 1024) {                              \
            unsigned long long t_;                                                \
            asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_));                \
            lsh_cta_trace[blockIdx.x][ev] = t_;                                   \
        }                                                                         \
    } while (0)
extern "C" LSH_API int lsh_attn_cta_trace_fused(unsigned long long *out)
{
    return (int)cudaMemcpyFromSymbol(out, lsh_cta_trace, sizeof(lsh_cta_trace));
}
#else
#define LSH_CTA_MARK(ev) \
    do {                 \
    } while (0)
#endif

namespace lsh {

namespace {

using namespace fwd;

constexpr int kMaxL = 4096;             // positions per segment
constexpr int kMaxHalf = 64;            // n_buckets / 2
constexpr int kMaxRounds = 8;           // CTAs per cluster (portable cluster size)
constexpr int kRingStages = 4;
constexpr int kHashTiles = 8;           // at most this many x tiles of 128 rows (16 KB) in flight
constexpr int kAccBufs = 4;             // TMEM accumulators of 128 columns
constexpr int kAccCols = 128;
constexpr int kWarps = kThreads / 32;
constexpr int kHashProducerWarp = kSoftmaxWarps;   // TMA loads of the hash phase
constexpr uint32_t kTileBytes = 128 * 128;

struct FusedSmem {
    Ring<kRingStages> ring;                         // stage memory doubles as the hash's x tiles and tables
    alignas(16) uint16_t perm[kMaxL];               // sorted slot -> position
    alignas(16) uint8_t bkt[kMaxL];                 // bucket id by position
    uint32_t warp_tot[32];
    uint64_t a_full[kHashTiles], a_empty[kHashTiles];
    uint64_t acc_full[kAccBufs], acc_empty[kAccBufs];
};
static_assert(kAccBufs * kAccCols <= kTmemCols, "hash accumulators fit in tensor memory");

// Hash and sort scratch in the stage memory, during the hash: n_buf x tiles
// (16 KB each), then this CTA's round's count of each bucket in each group of
// 32 consecutive positions (u8, [bucket][group]) and each position's rank among
// the equal buckets of its group (u8), then the rotations of every round
// (R_r^T stacked: rows r * hp + n of 64 k, K-major SW128).  After the hash,
// over the x tiles: the first sorted slot of each (bucket, group) (u16, same
// order).
constexpr int kGroups = kMaxL / 32;
constexpr size_t kStageBytes = sizeof(Stage) * kRingStages;
constexpr size_t kCntBytes = (size_t)2 * kMaxHalf * kGroups;
constexpr size_t kTablesBytes = kCntBytes + kMaxL;
constexpr size_t kRotMaxBytes = (size_t)kMaxRounds * kMaxHalf * 128;
static_assert(kTablesBytes % 1024 == 0, "the rotation tile stays 1024-byte aligned");
static_assert(7 * kTileBytes + kTablesBytes + kRotMaxBytes <= kStageBytes, "at least 7 x tiles beside the tables");
static_assert(kCntBytes * 2 <= 7 * kTileBytes, "first slots fit over the x tiles");

__device__ __forceinline__ uint8_t *hash_tile(FusedSmem &sm, int b)
{
    return reinterpret_cast<uint8_t *>(sm.ring.st) + (size_t)b * kTileBytes;
}

// The bucket of one row from its NH projections v (columns >= half are zero
// padding): the first maximum of [v ; -v].  Pass 1 takes the largest and
// smallest value (3-input max/min, four independent chains); the larger of max
// and -min picks the side (+ wins an exact tie: its indices come first); pass 2
// finds the lowest column holding that extreme.  A padding column (exactly 0)
// never decides: max(v_j, -v_j) >= 0 for every real column, and real columns
// come first.  This is the hash kernel's rule, so both give the same ids.
// Called by whole warps.
template <int NH>
__device__ __forceinline__ int first_max_bucket(const float *v, int half)
{
    constexpr int Q = NH / 4;
    float mxq[4], mnq[4];
#pragma unroll
    for (int qq = 0; qq < 4; ++qq) {
        const int j0 = qq * Q;
        float a = fmaxf(v[j0], v[j0 + 1]), b = fminf(v[j0], v[j0 + 1]);
#pragma unroll
        for (int j = j0 + 2; j < j0 + Q; j += 2) {
            a = tc::max3f(a, v[j], v[j + 1]);
            b = tc::min3f(b, v[j], v[j + 1]);
        }
        mxq[qq] = a;
        mnq[qq] = b;
    }
    const float mx = fmaxf(fmaxf(mxq[0], mxq[1]), fmaxf(mxq[2], mxq[3]));
    const float mn = fminf(fminf(mnq[0], mnq[1]), fminf(mnq[2], mnq[3]));
    const bool pos = mx >= -mn;
    const float target = pos ? mx : mn;
    // pass 2 on the FMA pipe (pass 1 runs on the ALU pipe): U = |extreme| bounds
    // every |v_j|; with B = 2^(24 - e(U)), (U - side v_j) B is exactly 0 where v_j
    // is the extreme and at least 1 elsewhere, so a saturating FMA gives an exact
    // 0/1 flag; sixteen flags are summed as the bits of an integer held in the
    // mantissa of 2^23 + sum, and the first clear bit is the column.  Extremes
    // whose B would not be finite take the compare-and-select form.
    const float U = pos ? mx : -mn;
    const int be = (__float_as_int(U) >> 23) & 0xFF;
    int js;
    if (__any_sync(0xffffffffu, U != 0.f && be < 24)) {
        int jq[4];
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
            int jj = NH;
#pragma unroll
            for (int j = qq * Q + Q - 1; j >= qq * Q; --j) jj = (v[j] == target) ? j : jj;
            jq[qq] = jj;
        }
        js = min(min(jq[0], jq[1]), min(jq[2], jq[3]));
    } else {
        const float B = __int_as_float(min(278 - be, 253) << 23);
        const float nsB = pos ? -B : B;
        const float UB = U * B;
        constexpr int NC = NH / 16;
        float acc[NC];
#pragma unroll
        for (int c = 0; c < NC; ++c) acc[c] = 8388608.f;
#pragma unroll
        for (int k = 0; k < 16; ++k)
#pragma unroll
            for (int c = 0; c < NC; ++c) acc[c] = fmaf(tc::fma_sat(v[c * 16 + k], nsB, UB), (float)(1 << k), acc[c]);
        js = NH;
#pragma unroll
        for (int c = NC - 1; c >= 0; --c) {
            const uint32_t eq = ~__float_as_uint(acc[c]) & 0xFFFFu;
            js = eq ? c * 16 + __ffs((int)eq) - 1 : js;
        }
    }
    return (pos ? 0 : half) + js;
}

// The epilogue warp's TMEM reads of an accumulator are done: release it to the MMAs.
__device__ __forceinline__ void release_acc(uint64_t &bar, int lane)
{
    tc::tc_fence_before();
    __syncwarp();
    if (lane == 0) tc::mbar_arrive(&bar);
}

__device__ __forceinline__ void cluster_sync_all()
{
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Rows [i0, i1) of head bh merged over its R <= RMAX rounds, eight threads per
// row; every thread loads K rows' round data before merging any, so that K
// memory round trips overlap.
template <int RMAX, int K>
__device__ __forceinline__ void merge_rows(const __nv_bfloat16 *__restrict__ o_r, const float *__restrict__ lse,
                                           __nv_bfloat16 *__restrict__ out, long long bh, int L, int R, int i0, int i1)
{
    const long long rstride = (long long)L * kDim / 8;
    const int n = (i1 - i0) * 8;
    for (int base = threadIdx.x; base < n; base += K * kThreads) {
        uint4 u[K][RMAX];
        float lr[K][RMAX];
#pragma unroll
        for (int k = 0; k < K; ++k) {
            const int idx = min(base + k * kThreads, n - 1);
            const int i = i0 + (idx >> 3), oct = idx & 7;
            const uint4 *orow = reinterpret_cast<const uint4 *>(o_r + (bh * R * (long long)L + i) * kDim) + oct;
            combine_load<RMAX, true>(orow, rstride, lse + bh * R * (long long)L + i, L, R, u[k], lr[k]);
        }
#pragma unroll
        for (int k = 0; k < K; ++k) {
            const int idx = base + k * kThreads;
            if (idx < n) {
                const int i = i0 + (idx >> 3), oct = idx & 7;
                reinterpret_cast<uint4 *>(out + (bh * L + i) * kDim)[oct] = combine_rows<RMAX>(u[k], lr[k], R, nullptr, oct);
            }
        }
    }
}

template <bool CAUSAL, int FL>
__global__ void __launch_bounds__(kThreads, 1)
fused_fwd_tc_kernel(const __grid_constant__ CUtensorMap xmap, const __nv_bfloat16 *__restrict__ x,
                    const __nv_bfloat16 *__restrict__ v, const __nv_bfloat16 *__restrict__ rot,
                    int32_t *__restrict__ perm_out, uint16_t *__restrict__ bkt_out, float *__restrict__ xinv,
                    __nv_bfloat16 *__restrict__ o_r, float *__restrict__ lse,
                    __nv_bfloat16 *__restrict__ out, int L, int R, int nb, float tau, uint32_t *__restrict__ status)
{
    extern __shared__ uint8_t smem_raw[];
    FusedSmem &sm = *reinterpret_cast<FusedSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Ring<kRingStages> &ring = sm.ring;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long seg = blockIdx.x;               // (bh, r), r fastest: the cluster is one head's rounds
    const int r = (int)(seg % R);
    const long long bh = seg / R;
    const int half = nb / 2, hp = half <= 32 ? 32 : 64;        // rotation columns, zero beyond half
    const int n_mt = (L + 127) / 128;               // hash tiles
    const int n_k = (L + kQ - 1) / kQ;              // attention tiles
    // The hash is split over the cluster: CTA r loads x tiles t = r, r + R, ...
    // and hashes them for every round at once (all rounds' rotations side by side,
    // rg rounds per MMA of N = rg * hp <= 128 columns, n_rg MMAs per tile); each
    // round's bucket ids, ranks and counts go to that round's CTA.
    const int rg = kAccCols / hp, n_rg = (R + rg - 1) / rg;
    const int n_local = r < n_mt ? (n_mt - r + R - 1) / R : 0;
    const int n_items = n_local * n_rg;
    const size_t rot_bytes = (size_t)R * hp * 128;
    const int n_buf = (int)min((size_t)kHashTiles, (kStageBytes - kTablesBytes - rot_bytes) / kTileBytes);
    uint8_t *const stage_mem = reinterpret_cast<uint8_t *>(ring.st);
    uint8_t *const cnt = stage_mem + (size_t)n_buf * kTileBytes;
    uint8_t *const rank = cnt + kCntBytes;
    uint8_t *const rot_t = rank + kMaxL;
    uint16_t *const first = reinterpret_cast<uint16_t *>(stage_mem);
    const int n_groups = (L + 31) / 32, nbits = bits_for(nb);
    cg::cluster_group cluster = cg::this_cluster();

    if (threadIdx.x == 0) {
        ring_init(ring);
        for (int b = 0; b < kHashTiles; ++b) {
            tc::mbar_init(&sm.a_full[b], 1);
            tc::mbar_init(&sm.a_empty[b], 4 * n_rg);    // every item of the tile has read it
        }
        for (int a = 0; a < kAccBufs; ++a) {
            tc::mbar_init(&sm.acc_full[a], 1);
            tc::mbar_init(&sm.acc_empty[a], 4);
        }
        tc::fence_mbar_init();
    }
    if (warp == 0) tc::tmem_alloc(&ring.tmem_base, kTmemCols);
    for (int e = threadIdx.x; e < (nb * n_groups + 15) / 16; e += kThreads)   // within the 16 KB table
        reinterpret_cast<uint4 *>(cnt)[e] = make_uint4(0, 0, 0, 0);
    // R_r^T of every round into the K-major swizzled B layout; columns n >= half
    // of a round are zero (never a first maximum: see first_max_bucket)
    for (int e = threadIdx.x; e < R * hp * kDim; e += kThreads) {
        const int nn = e % (R * hp), k = e / (R * hp), rr = nn / hp, n = nn % hp;
        const __nv_bfloat16 val =
            n < half ? rot[((long long)rr * kDim + k) * half + n] : __float2bfloat16_rn(0.f);
        *reinterpret_cast<__nv_bfloat16 *>(rot_t + tc::sw128_offset((uint32_t)nn, (uint32_t)k)) = val;
    }
    tc::fence_async_smem();
    tc::tc_fence_before();
    cluster_sync_all();                 // every CTA's tables are zero before any peer writes into them
    tc::tc_fence_after();
    const uint32_t tmem = ring.tmem_base;
    if (threadIdx.x == 0) LSH_PHASE(0, 7, 0, 0);
    LSH_CTA_MARK(0);

    // ================= hash
    if (warp == kHashProducerWarp) {
        if (lane == 0) {
            tc::prefetch_tmap(&xmap);
            for (int u = 0; u < n_local; ++u) {
                const int b = u % n_buf, t = r + u * R;
                if (u >= n_buf &&
                    !tc::mbar_wait(&sm.a_empty[b], (uint32_t)((u / n_buf) - 1) & 1u, &ring.abort, status))
                    break;
                LSH_PHASE(0, 4, u, 0);
                tc::mbar_arrive_expect_tx(&sm.a_full[b], kTileBytes);
                tc::tma_load_2d(hash_tile(sm, b), &xmap, 0, (int)(bh * L + (long long)t * 128), &sm.a_full[b]);
            }
        }
    } else if (warp == kMmaWarp) {
        if (lane == 0) {
            const uint32_t rs = tc::smem_u32(rot_t);
            bool go = true;
            for (int u = 0; go && u < n_local; ++u) {
                const int b = u % n_buf;
                if (!tc::mbar_wait(&sm.a_full[b], (uint32_t)(u / n_buf) & 1u, &ring.abort, status)) break;
                LSH_PHASE(0, 5, u, 0);
                const uint64_t da = tc::sw128_desc(tc::smem_u32(hash_tile(sm, b)));
                for (int g = 0; g < n_rg; ++g) {
                    const int it = u * n_rg + g, a = it % kAccBufs;
                    if (it >= kAccBufs &&
                        !tc::mbar_wait(&sm.acc_empty[a], (uint32_t)((it / kAccBufs) - 1) & 1u, &ring.abort, status)) {
                        go = false;
                        break;
                    }
                    tc::tc_fence_after();
                    const int nr = min(rg, R - g * rg);
                    const uint32_t id = tc::idesc_bf16(128, nr * hp, 0, 0);
                    const uint64_t db = tc::sw128_desc(rs + (uint32_t)(g * rg * hp * 128));
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        tc::mma_bf16(tmem + (uint32_t)(a * kAccCols), tc::desc_add(da, kk * 32),
                                     tc::desc_add(db, kk * 32), id, kk > 0);
                    tc::mma_commit(&sm.acc_full[a]);
                }
                LSH_PHASE(0, 5, u, 1);
            }
            if (*reinterpret_cast<volatile int *>(&ring.abort)) tc::mma_drain(&ring.drain, status);
        }
    } else if (warp < kSoftmaxWarps) {
        // group eg takes items it = eg, eg + 2, ...; warp q of it reads TMEM lanes 32 q..
        const int eg = warp >> 2, q = warp & 3;
        const int row = q * 32 + lane;
        for (int it = eg; it < n_items; it += 2) {
            const int u = it / n_rg, g = it % n_rg, a = it % kAccBufs, b = u % n_buf;
            const int t = r + u * R, pos = t * 128 + row;
            const bool valid = pos < L;
            if (!tc::mbar_wait(&sm.acc_full[a], (uint32_t)(it / kAccBufs) & 1u, &ring.abort, status)) break;
            if (q == 0 && lane == 0) LSH_PHASE(0, 6, it, 0);
            tc::tc_fence_after();
            const uint32_t tacc = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(a * kAccCols);
            const int nr = min(rg, R - g * rg);
            for (int j = 0; j < nr; ++j) {
                const int rr = g * rg + j;
                int bi;
                if (hp == 32) {
                    float pv[32];
                    tc::tmem_ld32(tacc + (uint32_t)(j * 32), pv);
                    tc::tmem_ld_wait();
                    bi = first_max_bucket<32>(pv, half);
                } else {
                    float pv[64];
                    tc::tmem_ld64(tacc + (uint32_t)(j * 64), pv);
                    tc::tmem_ld_wait();
                    bi = first_max_bucket<64>(pv, half);
                }
                // the warp's 32 consecutive positions form one sort group of round rr:
                // each position's rank among the equal ids before it, and the group's
                // count per id, written into round rr's CTA
                const uint32_t peers = peers_of(valid ? (uint32_t)bi : (1u << nbits), nbits);
                const uint32_t before = peers & ((1u << lane) - 1u);
                if (valid) {
                    *cluster.map_shared_rank(&sm.bkt[pos], rr) = (uint8_t)bi;
                    *cluster.map_shared_rank(rank + pos, rr) = (uint8_t)__popc(before);
                    if (before == 0) *cluster.map_shared_rank(cnt + bi * n_groups + (pos >> 5), rr) = (uint8_t)__popc(peers);
                }
            }
            release_acc(sm.acc_empty[a], lane);
            if (g == 0) {
                // 1/|x| of the row, sum of squares in element order (as the norm pass)
                const uint8_t *A = hash_tile(sm, b);
                float ssq = 0.f;
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    const uint4 w4 = *reinterpret_cast<const uint4 *>(A + row * 128 + ((ch ^ (row & 7)) << 4));
                    const uint32_t wd[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float lo = __uint_as_float(wd[e] << 16), hi = __uint_as_float(wd[e] & 0xFFFF0000u);
                        ssq = fmaf(lo, lo, ssq);
                        ssq = fmaf(hi, hi, ssq);
                    }
                }
                if (valid) xinv[bh * L + pos] = ssq > 0.f ? 1.0f / sqrtf(ssq) : 0.f;
            }
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&sm.a_empty[b]);
            if (q == 0 && lane == 0) LSH_PHASE(0, 6, it, 1);
        }
    }
    tc::fence_async_smem();
    tc::tc_fence_before();
    cluster_sync_all();                 // every round's ids, ranks and counts and every norm are written
    tc::tc_fence_after();
    bool ok = true;                     // the same for every thread of the cluster
    for (int c = 0; c < R; ++c) ok = ok && *cluster.map_shared_rank(&ring.abort, c) == 0;
    if (threadIdx.x == 0) LSH_PHASE(0, 7, 0, 1);
    LSH_CTA_MARK(1);

    // ================= sort
    if (ok) {
        // stable counting sort: first slot of every (bucket, group) by an exclusive
        // scan in (bucket, group) order; a position goes to its group's first slot
        // for its bucket plus its rank there
        {
            const int n = nb * n_groups, per = (n + kThreads - 1) / kThreads;
            const int e0 = min(n, (int)threadIdx.x * per), e1 = min(n, e0 + per);
            uint32_t tot = 0;
            for (int e = e0; e < e1; ++e) tot += cnt[e];
            uint32_t incl = tot;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t v2 = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += v2;
            }
            if (lane == 31) sm.warp_tot[warp] = incl;
            __syncthreads();
            if (warp == 0) {
                const uint32_t wv = lane < kWarps ? sm.warp_tot[lane] : 0u;
                uint32_t wi = wv;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const uint32_t v2 = __shfl_up_sync(0xffffffffu, wi, o);
                    if (lane >= o) wi += v2;
                }
                if (lane < kWarps) sm.warp_tot[lane] = wi - wv;
            }
            __syncthreads();
            uint32_t off = sm.warp_tot[warp] + incl - tot;
            for (int e = e0; e < e1; ++e) {
                const uint32_t c = cnt[e];
                first[e] = (uint16_t)off;
                off += c;
            }
            __syncthreads();
            for (int p = threadIdx.x; p < L; p += kThreads)
                sm.perm[first[sm.bkt[p] * n_groups + (p >> 5)] + rank[p]] = (uint16_t)p;
            __syncthreads();
        }
        if (threadIdx.x == 0) LSH_PHASE(0, 7, 0, 2);
        LSH_CTA_MARK(2);
        int32_t *pg = perm_out + seg * L;
        uint16_t *bg = bkt_out + seg * L;
        for (int e = threadIdx.x; e < L; e += kThreads) {
            pg[e] = (int32_t)sm.perm[e];
            bg[e] = (uint16_t)sm.bkt[e];
        }

        // ================= attention
        if (warp >= kSoftmaxWarps && warp < kMmaWarp) {
            const SegmentTiles src{sm.perm, sm.bkt, xinv + bh * L, L, r, bh, seg};
            producer_role<CAUSAL, FL>(ring, src, n_k, x, v, tau * kLog2e, status);
        } else if (warp == kMmaWarp) {
            mma_role(ring, n_k, tmem, status);
        } else {
            softmax_role<CAUSAL, FL, kRingStages, true>(ring, n_k, tmem, o_r, lse, L, tau, 0u, status);
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0) LSH_PHASE(0, 7, 0, 3);
    LSH_CTA_MARK(3);

    // ================= merge: every round's o_r and lse_r of this head are written
    cluster_sync_all();
    if (threadIdx.x == 0) LSH_PHASE(0, 7, 0, 4);
    LSH_CTA_MARK(4);
    if (ok && *reinterpret_cast<volatile int *>(&ring.abort) == 0) {
        const int rows = (L + R - 1) / R, i0 = r * rows, i1 = min(L, i0 + rows);
        if (R <= 2)
            merge_rows<2, 8>(o_r, lse, out, bh, L, R, i0, i1);
        else if (R <= 4)
            merge_rows<4, 4>(o_r, lse, out, bh, L, R, i0, i1);
        else
            merge_rows<8, 2>(o_r, lse, out, bh, L, R, i0, i1);
    }
    if (threadIdx.x == 0) LSH_PHASE(0, 7, 0, 5);
    LSH_CTA_MARK(5);
    if (warp == 0) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace

bool fused_fwd_fits(const Problem &p)
{
    return p.dtype == LSH_BF16 && p.d == kDim && p.m == 64 && p.L % 64 == 0 && p.L <= kMaxL &&
           p.nb / 2 <= kMaxHalf && p.R <= kMaxRounds && p.prev_mask == 0 && p.tokens() >= 128 &&
           p.tokens() < (1LL << 31) - 128;
}

template <bool CAUSAL, int FL>
static cudaError_t launch_fused(const Problem &p, const CUtensorMap &xmap, const void *x, const void *v,
                                const void *R, int32_t *perm, uint16_t *bkt, float *xinv, __nv_bfloat16 *o_r,
                                float *lse, void *out, uint32_t *status, cudaStream_t st)
{
    static_assert(sizeof(FusedSmem) + 1024 <= 232448, "shared memory per CTA");
    const size_t smem = sizeof(FusedSmem) + 1024;
    auto kern = fused_fwd_tc_kernel<CAUSAL, FL>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)p.S(), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)p.R;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, xmap, (const __nv_bfloat16 *)x, (const __nv_bfloat16 *)v,
                              (const __nv_bfloat16 *)R, perm, bkt, xinv, o_r, lse, (__nv_bfloat16 *)out, p.L, p.R, p.nb,
                              1.0f / sqrtf((float)p.d), status);
}

cudaError_t launch_fused_fwd_tc(const Problem &p, const void *x, const void *v, const void *R, int32_t *perm,
                                uint16_t *bkt, float *xinv, void *o_r, float *lse, void *out, uint32_t *status,
                                cudaStream_t st)
{
    if (!fused_fwd_fits(p)) return cudaErrorInvalidValue;
    CUtensorMap xmap;
    if (!tc::make_row_tmap(&xmap, x, p.tokens(), 128)) return cudaErrorInvalidValue;
    __nv_bfloat16 *orb = (__nv_bfloat16 *)o_r;
    const int fl = p.flags & (kMask | kPen);
#define LSH_FUSED_CASE(C, F) return launch_fused<C, F>(p, xmap, x, v, R, perm, bkt, xinv, orb, lse, out, status, st)
    if (p.causal) {
        switch (fl) {
        case 0: LSH_FUSED_CASE(true, 0);
        case kMask: LSH_FUSED_CASE(true, kMask);
        case kPen: LSH_FUSED_CASE(true, kPen);
        default: LSH_FUSED_CASE(true, kMask | kPen);
        }
    }
    switch (fl) {
    case 0: LSH_FUSED_CASE(false, 0);
    case kMask: LSH_FUSED_CASE(false, kMask);
    case kPen: LSH_FUSED_CASE(false, kPen);
    default: LSH_FUSED_CASE(false, kMask | kPen);
    }
#undef LSH_FUSED_CASE
}

}  // namespace lsh

LSH_PHASE_EXPORT(fused)
