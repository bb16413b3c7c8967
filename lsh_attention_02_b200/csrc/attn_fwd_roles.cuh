// Warp roles of chunk_attn forward on the tensor cores (bf16, d = 64, m = 64),
// shared by the persistent kernel over every segment (attn_fwd_tc.cu) and the
// single-kernel forward of short segments (fused_fwd_tc.cu).
//
// "Sorting and Chunking" (paper note "Reformer"): after the sort, the sorted
// sequence is cut into chunks of m = 64 slots and chunk c attends to chunks
// c-1 and c.  One work tile = 128 sorted query slots (chunks 2k and 2k+1) of
// one (batch, head, round) segment, whose keys are the 192 slots of chunks
// 2k-1, 2k and 2k+1.  Shared query-key ("Shared Query-Key Space", Q = K):
// the 128 query rows are the last 128 rows of the gathered 192-row key tile,
// so one gathered tile serves as both MMA operands.
//
// Per tile:
//   gather   rows x[perm[s]] and v[perm[s]] of the 192 window slots, copied
//            straight into the 128-byte-swizzled layout the tensor core reads;
//   norms    1/|x_j| of the window rows, gathered with the positions;
//   S = Q K^T  tcgen05.mma M=128, N=192, K=64 into tensor memory (raw
//            dot products x_i . x_j, bf16 in, fp32 accumulate);
//   softmax  one query row per thread: s_ij = (x_i . x_j) / |x_j| / sqrt(d)
//            (unit keys), masked to the window of the row's chunk, to
//            earlier original positions when causal, optionally to the
//            query's bucket ("LSH Attention", strict candidate set), and
//            never the query's own position unless nothing else is left
//            ("Implementation Reading"); P is written as bf16 back into the
//            S columns;
//   O = P V  tcgen05.mma M=128, N=64, K=192 with A = P read from tensor
//            memory and V read MN-major from shared memory;
//   store    o_r and lse_r at the query's original position (the unsort),
//            o_r rows staged in shared memory and written as whole lines.
//
// Scores satisfy s_ij <= tau |x_i| (Cauchy-Schwarz with unit keys), so the
// softmax uses M = tau |x_i| in place of the row maximum: one sweep, no max
// pass.  A warp whose rows have tau |x_i| so large that exp(s - M) could leave
// the normal fp32 range first finds the exact maximum.  A query with no
// other candidate (its softmax sum is 0) keeps its own key, whose score is
// tau |x_i|, so p = 1 there and lse = tau |x_i|; with the self penalty its
// lse is the penalty score.  Where other candidates exist the penalised self
// entry's weight exp(penalty - lse) is 0 in fp32 (|x_i| < 8e5), so it is left
// out.
//
// Warp roles (12 warps):
//   warps 0-3, 4-7  two softmax groups working on alternate tiles, each with
//                   its own 256 TMEM columns (S/P 192, O 64), so one group's
//                   softmax overlaps the other's MMAs and stores;
//   warps 8-10      producer: positions and key norms (and, with the bucket
//                   mask, buckets) loaded a tile ahead; x and v rows by
//                   16-byte cp.async (eight threads per row, zero fill for a
//                   missing slot) into the shared-memory ring; a stage is
//                   published once the next stage's copies are in flight;
//   warp 11         MMA issuer.
#pragma once
#include "tc_common.cuh"

namespace lsh {
namespace fwd {

constexpr int kQ = 128;             // query slots per tile
constexpr int kW = 192;             // window rows (keys)
constexpr int kSoftmaxWarps = 8;   // two groups of four
constexpr int kProducerWarps = 3;
constexpr int kProducerThreads = kProducerWarps * 32;
constexpr int kMmaWarp = kSoftmaxWarps + kProducerWarps;
constexpr int kThreads = (kMmaWarp + 1) * 32;
static_assert(kW == 2 * kProducerThreads, "two window positions per producer thread");
static_assert(kW % (kProducerThreads / 8) == 0, "rows split evenly over the producer");
constexpr int kTmemCols = 512;
constexpr uint32_t kGroupCols = 256;
constexpr uint32_t kOCol = 192;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

struct TileCoord {
    int r, k;
    long long bh, seg;
};
// Tile order of the persistent kernel (bh, k, r): tiles in flight at the same
// time share a head's rows in L2.  Only the producer locates tiles (a tile
// ahead); the softmax groups read the coordinates from the stage.
__device__ __forceinline__ TileCoord tile_coord(long long tile, int R, int n_k)
{
    TileCoord c;
    c.r = (int)(tile % R);
    const long long bk = tile / R;
    c.k = (int)(bk % n_k);
    c.bh = bk / n_k;
    c.seg = c.bh * R + c.r;
    return c;
}

struct alignas(1024) Stage {
    uint8_t X[kW * 128];            // gathered x rows, K-major SW128 (24 KB)
    uint8_t V[kW * 128];            // gathered v rows (24 KB)
    alignas(16) int32_t pos[kW];    // original positions of the window slots (-1: none)
    alignas(16) float sinv[kW];     // tau * log2(e) / |x_j| (0 for a zero row or no row)
    alignas(16) float inv[kW];      // 1 / |x_j|
    alignas(16) int32_t kb[kW];     // bucket of each window slot (-1: none); bucket mask only
    TileCoord coord;                // the tile's coordinates
};

// Optional readings (template parameter FL, bits of lsh_attn_desc.flags).
constexpr int kMask = LSH_FLAG_BUCKET_MASK, kPen = LSH_FLAG_SELF_PENALTY;
constexpr float kSelfPenalty = LSH_SELF_PENALTY_SCORE;

// Key j (position kp, bucket kb) is a candidate of query position qpos (bucket
// qb): causal -- an earlier position (an empty slot, -1, never is); otherwise
// any other position; with the bucket mask also the same bucket.
template <bool CAUSAL, int FL>
__device__ __forceinline__ bool admit(int kp, int qpos, int kb, int qb)
{
    const bool ok = CAUSAL ? (unsigned)kp < (unsigned)qpos : kp != qpos;
    return (FL & kMask) ? ok && kb == qb : ok;
}

// The stage ring and the barriers of the roles; NST stages.
template <int NST>
struct Ring {
    Stage st[NST];
    uint64_t full[NST], empty[NST];
    uint64_t s_full[2], p_half[2], p_full[2], o_full[2], o_free[2];  // p_half: P of keys 0..63 written
    uint64_t drain;                 // timeout path: the MMA issuer's last products
    uint32_t tmem_base;
    int abort;
};

template <int NST>
__device__ __forceinline__ void ring_init(Ring<NST> &sm)
{
    for (int s = 0; s < NST; ++s) {
        tc::mbar_init(&sm.full[s], kProducerThreads);
        tc::mbar_init(&sm.empty[s], 4);
    }
    for (int g = 0; g < 2; ++g) {
        tc::mbar_init(&sm.s_full[g], 1);
        tc::mbar_init(&sm.p_half[g], 4);
        tc::mbar_init(&sm.p_full[g], 4);
        tc::mbar_init(&sm.o_full[g], 1);
        tc::mbar_init(&sm.o_free[g], 4);
    }
    tc::mbar_init(&sm.drain, 1);
    sm.abort = 0;
    tc::fence_mbar_init();
}

// Where a CTA's tiles and their positions, key norms and buckets come from.
// GridTiles: the persistent kernel's tiles blockIdx.x + it * gridDim.x of every
// segment, read from global memory.  SegmentTiles: the tiles of one segment in
// order, with its permutation and bucket ids in shared memory (positions below
// 65536, ids below 256) and its key norms in global memory.
struct GridTiles {
    const int32_t *perm;            // [S, L]
    const uint16_t *bkt;            // [S, L] (bucket mask only)
    const float *xinv;              // [B*H, L]
    int L, R, n_k;
    __device__ __forceinline__ TileCoord coord(int it) const
    {
        return tile_coord(blockIdx.x + (long long)it * gridDim.x, R, n_k);
    }
    __device__ __forceinline__ int slot_pos(const TileCoord &c, int sl) const { return perm[c.seg * L + sl]; }
    __device__ __forceinline__ int bucket(const TileCoord &c, int p) const { return (int)bkt[c.seg * L + p]; }
    __device__ __forceinline__ float inv(const TileCoord &c, int p) const { return xinv[c.bh * L + p]; }
};
struct SegmentTiles {
    const uint16_t *perm;           // [L], shared memory
    const uint8_t *bkt;             // [L], shared memory (by position)
    const float *xinv;              // [L], this head's norms (by position)
    int L, r;
    long long bh, seg;
    __device__ __forceinline__ TileCoord coord(int it) const { return TileCoord{r, it, bh, seg}; }
    __device__ __forceinline__ int slot_pos(const TileCoord &, int sl) const { return (int)perm[sl]; }
    __device__ __forceinline__ int bucket(const TileCoord &, int p) const { return (int)bkt[p]; }
    __device__ __forceinline__ float inv(const TileCoord &, int p) const { return xinv[p]; }
};

// Softmax of one query row (thread) over window columns [BASE, BASE + 128)
// (chunk 2k: BASE = 0, chunk 2k+1: BASE = 64).  FIRST: the segment's first
// tile, whose chunk -1 (window columns 0..63) does not exist.  P is written as
// packed bf16 pairs into the row's own S columns (key j -> column j/2), in
// place: each half of 64 scores is read before packed columns
// BASE/2 + [32h, 32h + 32) are written, and those never reach an unread half.
// Columns outside the row's window get zeros.  Returns l = sum of p.
//
// Candidates: see admit().  A row with none gets l = 0 here and is patched by
// the caller.
template <bool CAUSAL, int FL>
__device__ __forceinline__ float softmax_sweep(const Stage &st, uint32_t tl, int qpos, int qb, float shift2, int BASE,
                                               bool FIRST, bool PREV, uint64_t *half_done)
{
    float lsum = 0.f;
    const uint32_t z[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    // Keys 0..63 must be complete for every row after the first half-sweep: rows
    // of chunk 2k+1 (BASE 64) cannot see them and clear their packed columns
    // first (their S columns there are unused); rows of chunk 2k clear keys
    // 128..191 last, since those packed columns still hold S values they read.
    if (BASE != 0) {
#pragma unroll
        for (int c = 0; c < 4; ++c) tc::tmem_st8(tl + (uint32_t)(c * 8), z);
    }
#pragma unroll 1
    for (int h = 0; h < 2; ++h) {
        if ((FIRST && BASE == 0 && h == 0) || (PREV && h == 1)) {   // missing chunk -1, or own chunk left out
#pragma unroll
            for (int c = 0; c < 4; ++c) tc::tmem_st8(tl + (uint32_t)(BASE / 2 + h * 32 + c * 8), z);
        } else {
            float v[64];
            tc::tmem_ld64(tl + (uint32_t)(BASE + h * 64), v);
            tc::tmem_ld_wait();
    #pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t w[8];
    #pragma unroll
                for (int e4 = 0; e4 < 16; e4 += 4) {
                    const int j0 = h * 64 + c * 16 + e4;
                    const int4 kp = *reinterpret_cast<const int4 *>(&st.pos[BASE + j0]);
                    const float4 ks = *reinterpret_cast<const float4 *>(&st.sinv[BASE + j0]);
                    const int4 kb = (FL & kMask) ? *reinterpret_cast<const int4 *>(&st.kb[BASE + j0])
                                                 : make_int4(0, 0, 0, 0);
                    const int kpa[4] = {kp.x, kp.y, kp.z, kp.w};
                    const int kba[4] = {kb.x, kb.y, kb.z, kb.w};
                    const float ksa[4] = {ks.x, ks.y, ks.z, ks.w};
                    float pe[4];
    #pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const bool ok = admit<CAUSAL, FL>(kpa[e], qpos, kba[e], qb);
                        const float p = tc::fast_exp2(fmaf(v[c * 16 + e4 + e], ksa[e], -shift2));
                        pe[e] = ok ? p : 0.f;
                        lsum += pe[e];
                    }
                    w[e4 / 2] = pack_bf16x2(pe[0], pe[1]);
                    w[e4 / 2 + 1] = pack_bf16x2(pe[2], pe[3]);
                }
                tc::tmem_st8(tl + (uint32_t)(BASE / 2 + h * 32 + c * 8), w);
            }
        }
        if (h == 0) {
            tc::tmem_st_wait();
            tc::tc_fence_before();
            __syncwarp();
            if ((threadIdx.x & 31) == 0) tc::mbar_arrive(half_done);
        }
    }
    if (BASE == 0) {
#pragma unroll
        for (int c = 0; c < 4; ++c) tc::tmem_st8(tl + 64 + (uint32_t)(c * 8), z);
    }
    return lsum;
}

// Exact row maximum of the log2-domain scores (only for rows whose bound
// tau |x_i| is so loose that exp(s - bound) could leave the normal range).
template <bool CAUSAL, int FL>
__device__ __forceinline__ float exact_max(const Stage &st, uint32_t tl, int jlo, int jhi, int qpos, int qb, int BASE)
{
    float mx = -INFINITY;
#pragma unroll 1
    for (int c = 0; c < jhi / 16; ++c) {
        float v[16];
        tc::tmem_ld16(tl + (uint32_t)(BASE + c * 16), v);
        tc::tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const int j = c * 16 + e;
            const bool ok = (j >= jlo) && admit<CAUSAL, FL>(st.pos[BASE + j], qpos, st.kb[BASE + j], qb);
            mx = ok ? fmaxf(mx, v[e] * st.sinv[BASE + j]) : mx;
        }
    }
    return mx;
}

// A row has no candidate exactly when its sum l is 0: every admitted term is at
// least 2^-100 (exp2 of an argument >= -2 bound log2(e) >= -100 when the row is
// not wide, and the row maximum gives 1 when it is).  PREV: a round whose window
// is the previous chunk alone (the following-chunk part of local attention, in
// reversed order); a row left with no candidate there contributes nothing
// (lse = -inf, output 0) instead of attending to itself.
template <bool CAUSAL, int FL>
__device__ __forceinline__ void softmax_row(const Stage &st, uint32_t tl, int i, int qpos, int qb, float qinv,
                                            float tau, int BASE, bool FIRST, bool PREV, uint64_t *half_done,
                                            float &l, float &row_lse)
{
    const float bound = qinv > 0.f ? tau / qinv : 0.f;        // tau |x_i| >= every score of the row
    float shift2 = bound * kLog2e;                              // log2-domain offset
    const bool wide = 2.f * bound * kLog2e > 100.f;             // bound - s <= 2 bound
    if (__any_sync(0xffffffffu, wide)) {
        const float mx = exact_max<CAUSAL, FL>(st, tl, FIRST && BASE == 0 ? 64 : 0, PREV ? 64 : 128, qpos, qb, BASE);
        if (wide && mx > -INFINITY) shift2 = mx;
    }
    l = softmax_sweep<CAUSAL, FL>(st, tl, qpos, qb, shift2, BASE, FIRST, PREV, half_done);
    row_lse = kLn2 * (shift2 + log2f(l));
    const bool self_only = qpos >= 0 && l == 0.f && !PREV;
    if (__any_sync(0xffffffffu, self_only)) {
        // A row with no candidate attends to itself: p = 1 on its own key (window
        // row 64 + i), lse = tau x_i . (x_i / |x_i|) = tau |x_i| (with the self
        // penalty: lse = the penalty score).  The warp's 32 own keys occupy packed
        // columns 32 + i/2 - (lane/2); each lane edits its own row.
        const int lane = i & 31;
        const uint32_t col0 = (uint32_t)((64 + (i - lane)) >> 1);
        float w[16];
        tc::tmem_st_wait();
        tc::tmem_ld16(tl + col0, w);
        tc::tmem_ld_wait();
        uint32_t u[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
            const uint32_t one = (lane & 1) ? 0x3F800000u : 0x00003F80u;
            u[c] = (self_only && c == (lane >> 1)) ? one : __float_as_uint(w[c]);
        }
        tc::tmem_st16(tl + col0, u);
        if (self_only) {
            l = 1.f;
            row_lse = (FL & kPen) ? kSelfPenalty : bound;
        }
    }
}


// Producer (warps kSoftmaxWarps .. kMmaWarp - 1): positions, norms and buckets
// of a tile, loaded a tile ahead, and the x and v rows of its window by 16-byte
// cp.async into the stage ring.  n_mine: this CTA's tiles.
template <bool CAUSAL, int FL, int NST, class Src>
__device__ __forceinline__ void producer_role(Ring<NST> &sm, const Src &src, int n_mine,
                                              const __nv_bfloat16 *__restrict__ x,
                                              const __nv_bfloat16 *__restrict__ v, float sl2,
                                              uint32_t *__restrict__ status)
{
    const int ptid = threadIdx.x - kSoftmaxWarps * 32;
    const int L = src.L;
    // positions (and, with the bucket mask, buckets) of the next tile, loaded a
    // tile ahead (two slots per thread)
    int pn[2] = {-1, -1}, bn[2] = {-1, -1};
    float nn[2] = {0.f, 0.f};                   // 1/|x| of those positions
    // A slot outside [0, L) (chunk -1, or the missing chunk of a last tile
    // when L % 128 == 64) is empty (-1); so is a permutation entry outside
    // [0, L), which is also reported in the status word.
    TileCoord nc{};                             // coordinates of that tile
    auto load_pos = [&](int it) {
        const TileCoord c = src.coord(it);
        nc = c;
        const int slot0 = c.k * kQ - 64;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int e = ptid + j * kProducerThreads;     // kW = 2 * kProducerThreads
            const int sl = slot0 + e;
            const bool in = sl >= 0 && sl < L;
            const int pl = src.slot_pos(c, min(max(sl, 0), L - 1));
            const bool good = (unsigned)pl < (unsigned)L;
            if (in && !good) atomicOr(status, kStatusBadPerm);
            pn[j] = in && good ? pl : -1;
            if (FL & kMask) bn[j] = pn[j] >= 0 ? src.bucket(c, pn[j]) : -1;
            nn[j] = pn[j] >= 0 ? src.inv(c, pn[j]) : 0.f;
        }
    };
    if (n_mine > 0) load_pos(0);
    int prev_s = -1;
    for (int it = 0; it < n_mine; ++it) {
        const int s = it % NST;
        if (ptid == 0) LSH_PHASE(0, 0, it, 0);
        bool ok = it < NST ||
                  tc::mbar_wait(&sm.empty[s], (uint32_t)((it / NST) - 1) & 1u, &sm.abort, status);
        if (tc::named_bar_or(1, kProducerThreads, !ok)) { prev_s = -1; break; }
        if (ptid == 0) LSH_PHASE(0, 0, it, 1);
        Stage &st = sm.st[s];
        const TileCoord cc = nc;
        const long long rowbase = cc.bh * L;
        if (ptid == 0) st.coord = cc;
        st.pos[ptid] = pn[0];
        st.pos[ptid + kProducerThreads] = pn[1];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            st.inv[ptid + j * kProducerThreads] = nn[j];
            st.sinv[ptid + j * kProducerThreads] = nn[j] * sl2;
        }
        if (FL & kMask) {
            st.kb[ptid] = bn[0];
            st.kb[ptid + kProducerThreads] = bn[1];
        }
        tc::named_bar_sync(1, kProducerThreads);
        if (it + 1 < n_mine) load_pos(it + 1);   // overlaps the copies below
        if (ptid == 0) LSH_PHASE(0, 0, it, 2);
        // x and v rows: thread t copies 16-byte chunk t % 8 of rows t / 8 + 12 j
        // (zero fill for a missing slot); every position is read first for ILP
        {
            constexpr int kRowStep = kProducerThreads / 8;
            const int ch = ptid & 7, r0 = ptid >> 3;
            int pr[kW / kRowStep];
#pragma unroll
            for (int j = 0; j < kW / kRowStep; ++j) pr[j] = st.pos[r0 + kRowStep * j];
#pragma unroll
            for (int j = 0; j < kW / kRowStep; ++j) {
                const int row = r0 + kRowStep * j;
                const uint32_t off = (uint32_t)row * 128u + (uint32_t)((ch ^ (row & 7)) << 4);
                const long long src = (rowbase + max(pr[j], 0)) * kDim + ch * 8;
                const uint32_t nb = pr[j] >= 0 ? 16u : 0u;
                tc::cp_async16_zfill(st.X + off, x + src, nb);
                tc::cp_async16_zfill(st.V + off, v + src, nb);
            }
        }
        tc::cp_async_commit();
        if (ptid == 0) LSH_PHASE(0, 0, it, 3);
        if (prev_s >= 0) {
            // the previous stage's copies have landed: publish it
            tc::cp_async_wait<1>();
            tc::fence_async_smem();
            tc::mbar_arrive(&sm.full[prev_s]);
        }
        if (ptid == 0) LSH_PHASE(0, 0, it, 4);
        prev_s = s;
    }
    if (prev_s >= 0) {
        tc::cp_async_wait<0>();
        tc::fence_async_smem();
        tc::mbar_arrive(&sm.full[prev_s]);
    } else {
        tc::cp_async_wait<0>();         // given up: let this thread's copies land before the CTA ends
    }
}

// MMA issuer (warp kMmaWarp; lane 0 issues).
template <int NST>
__device__ __forceinline__ void mma_role(Ring<NST> &sm, int n_mine, uint32_t tmem, uint32_t *__restrict__ status)
{
    const int lane = threadIdx.x & 31;
    // S = Q K^T of a tile needs its stage loaded and its group's TMEM free;
    // O = P V needs the tile's P.  Whichever is ready is issued first, so a
    // late stage never holds back the O of the tile before it.
    if (lane == 0) {
        constexpr uint32_t id_s = tc::idesc_bf16(128, kW, 0, 0);
        constexpr uint32_t id_o = tc::idesc_bf16(128, kDim, 0, 1);
        int next_s = 0, next_oh = 0, next_o = 0;        // next tile (local index) for S, O's first keys, O
        long long t0 = clock64();
        while (next_o < n_mine) {
            bool progressed = false;
            if (next_s < n_mine && next_s <= next_o + 1) {
                const int it = next_s, s = it % NST, g = it & 1;
                if (tc::mbar_test_wait(&sm.full[s], (uint32_t)(it / NST) & 1u) &&
                    (it < 2 || tc::mbar_test_wait(&sm.o_free[g], (uint32_t)((it >> 1) - 1) & 1u))) {
                    LSH_PHASE(0, 1, it, 1);
                    tc::tc_fence_after();
                    const uint64_t dx = tc::sw128_desc(tc::smem_u32(sm.st[s].X));
                    const uint32_t d = tmem + (uint32_t)g * kGroupCols;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        tc::mma_bf16(d, tc::desc_add(dx, 64 * 128 + kk * 32), tc::desc_add(dx, kk * 32),
                                     id_s, kk > 0);
                    tc::mma_commit(&sm.s_full[g]);
                    LSH_PHASE(0, 1, it, 2);
                    ++next_s;
                    progressed = true;
                }
            }
            if (next_oh < next_s) {
                // keys 0..63 as soon as every row's P there is written
                const int it = next_oh, s = it % NST, g = it & 1;
                if (tc::mbar_test_wait(&sm.p_half[g], (uint32_t)(it >> 1) & 1u)) {
                    tc::tc_fence_after();
                    const uint64_t dv = tc::sw128_desc(tc::smem_u32(sm.st[s].V));
                    const uint32_t base = tmem + (uint32_t)g * kGroupCols;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        tc::mma_bf16_ts(base + kOCol, base + kk * 8, tc::desc_add(dv, kk * 16 * 128), id_o,
                                        kk > 0);
                    ++next_oh;
                    progressed = true;
                }
            }
            if (next_o < next_oh) {
                const int it = next_o, s = it % NST, g = it & 1;
                if (tc::mbar_test_wait(&sm.p_full[g], (uint32_t)(it >> 1) & 1u)) {
                    LSH_PHASE(0, 1, it, 3);
                    tc::tc_fence_after();
                    const uint64_t dv = tc::sw128_desc(tc::smem_u32(sm.st[s].V));
                    const uint32_t base = tmem + (uint32_t)g * kGroupCols;
#pragma unroll
                    for (int kk = 4; kk < 12; ++kk)
                        tc::mma_bf16_ts(base + kOCol, base + kk * 8, tc::desc_add(dv, kk * 16 * 128), id_o,
                                        true);
                    tc::mma_commit(&sm.o_full[g]);
                    LSH_PHASE(0, 1, it, 4);
                    ++next_o;
                    progressed = true;
                }
            }
            if (progressed) {
                t0 = clock64();
            } else {
                if (*reinterpret_cast<volatile int *>(&sm.abort)) break;
                if (clock64() - t0 > tc::kWaitCycles) {
                    sm.abort = 1;
                    atomicOr(status, kStatusTimeout);
                    break;
                }
                __nanosleep(20);
            }
        }
        if (*reinterpret_cast<volatile int *>(&sm.abort)) tc::mma_drain(&sm.drain, status);
    }
}

// A 16-byte store that asks L2 to keep the line (evict-last policy): for rows
// that the same kernel reads back soon.
__device__ __forceinline__ void st_keep_l2(void *p, const uint4 &u, uint64_t policy)
{
    asm volatile("st.global.L2::cache_hint.v4.b32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(p), "r"(u.x), "r"(u.y),
                 "r"(u.z), "r"(u.w), "l"(policy)
                 : "memory");
}

// Softmax groups (warps 0-3 and 4-7): group g takes the CTA's tiles it = g, g + 2, ...
// KEEP: o_r rows are stored with an L2 evict-last hint (read back by this kernel).
template <bool CAUSAL, int FL, int NST, bool KEEP = false>
__device__ __forceinline__ void softmax_role(Ring<NST> &sm, int n_mine, uint32_t tmem,
                                             __nv_bfloat16 *__restrict__ o_r, float *__restrict__ lse, int L,
                                             float tau, uint32_t prev_mask, uint32_t *__restrict__ status)
{
    uint64_t keep = 0;
    if (KEEP) asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(keep));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = warp >> 2, q = warp & 3;
    const int i = q * 32 + lane;                             // query row = TMEM lane
    const int gt = i;                                        // thread index inside the group
    const uint32_t tl = tmem + (uint32_t)g * kGroupCols + ((uint32_t)(q * 32) << 16);
    for (int it = g; it < n_mine; it += 2) {
        const int s = it % NST;
        const uint32_t gph = (uint32_t)(it >> 1) & 1u;
        const bool mark = gt == 0;
        if (mark) LSH_PHASE(0, 2 + g, it, 0);
        if (!tc::mbar_wait(&sm.full[s], (uint32_t)(it / NST) & 1u, &sm.abort, status)) break;
        if (mark) LSH_PHASE(0, 2 + g, it, 1);
        Stage &st = sm.st[s];
        if (!tc::mbar_wait(&sm.s_full[g], gph, &sm.abort, status)) break;
        if (mark) LSH_PHASE(0, 2 + g, it, 2);
        tc::tc_fence_after();
        const TileCoord tcd = st.coord;
        const int qpos = st.pos[64 + i];
        const int qb = (FL & kMask) ? st.kb[64 + i] : 0;
        const float qinv = st.inv[64 + i];
        const bool first = tcd.k == 0;
        float l, row_lse;
        // one run-time-parameterised copy of the row code for every warp (instruction cache)
        const bool prev = (prev_mask >> tcd.r) & 1u;    // this round's window: the previous chunk alone
        softmax_row<CAUSAL, FL>(st, tl, i, qpos, qb, qinv, tau, q >= 2 ? 64 : 0, first && q < 2, prev, &sm.p_half[g],
                                l, row_lse);
        tc::tmem_st_wait();
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&sm.p_full[g]);
        if (mark) LSH_PHASE(0, 2 + g, it, 3);
        if (!tc::mbar_wait(&sm.o_full[g], gph, &sm.abort, status)) break;
        if (mark) LSH_PHASE(0, 2 + g, it, 4);
        tc::tc_fence_after();
        float o[kDim];
#pragma unroll
        for (int c = 0; c < 4; ++c) tc::tmem_ld16(tl + kOCol + (uint32_t)(c * 16), o + c * 16);
        tc::tmem_ld_wait();
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&sm.o_free[g]);
        const float rl = l > 0.f ? 1.0f / l : 0.f;        // no candidate (previous-chunk round): output 0
        // o_r at the original positions: each warp stages its 32 rows (bf16, 16-byte
        // chunks swizzled by row) in this stage's v tile, which no product reads any
        // more, and stores them four rows per instruction, eight lanes per 128-byte
        // row, so every store instruction writes four whole lines.
        {
            uint8_t *wst = st.V + q * 32 * 128;
#pragma unroll
            for (int c = 0; c < 8; ++c)
                *reinterpret_cast<uint4 *>(wst + lane * 128 + ((c ^ (lane & 7)) << 4)) =
                    make_uint4(pack_bf16x2(o[8 * c] * rl, o[8 * c + 1] * rl),
                               pack_bf16x2(o[8 * c + 2] * rl, o[8 * c + 3] * rl),
                               pack_bf16x2(o[8 * c + 4] * rl, o[8 * c + 5] * rl),
                               pack_bf16x2(o[8 * c + 6] * rl, o[8 * c + 7] * rl));
            __syncwarp();
            const int ch = lane & 7;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const int rr = 4 * k + (lane >> 3);
                const int p = __shfl_sync(0xffffffffu, qpos, rr);
                const uint4 u = *reinterpret_cast<const uint4 *>(wst + rr * 128 + ((ch ^ (rr & 7)) << 4));
                if (p >= 0) {                // an empty query slot has no output
                    if (KEEP)
                        st_keep_l2(o_r + (tcd.seg * L + p) * kDim + ch * 8, u, keep);
                    else
                        *reinterpret_cast<uint4 *>(o_r + (tcd.seg * L + p) * kDim + ch * 8) = u;
                }
            }
            __syncwarp();
        }
        if (qpos >= 0) lse[tcd.seg * L + qpos] = row_lse;
        if (lane == 0) tc::mbar_arrive(&sm.empty[s]);
        if (mark) LSH_PHASE(0, 2 + g, it, 5);
    }
}

}  // namespace fwd
}  // namespace lsh
