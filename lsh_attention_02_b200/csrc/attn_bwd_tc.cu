// chunk_attn backward on the tensor cores (bf16, d = 64, m = 64).
//
// Merged output of the rounds ("Multiple Hash Rounds"): with LSE_i the
// logsumexp of every candidate score of query i over all rounds,
//   y_i = sum_r sum_j P_rij v_j,   P_rij = exp(s_rij - LSE_i),
// so each round's backward is an ordinary attention backward with LSE_i in
// place of the per-round logsumexp and delta_i = dY_i . y_i:
//   dv_j += P_ij dY_i,   ds_ij = P_ij (dY_i . v_j - delta_i),
//   s_ij = tau (x_i . x_j) inv_j  (inv_j = 1/|x_j|, unit keys, Q = K), so with
//   e_ij = tau inv_j ds_ij:
//   dx_i += sum_j e_ij x_j                                  (query role)
//   g_j   = sum_i e_ij x_i,  dx_j += g_j - inv_j^2 (g_j . x_j) x_j   (key role)
//
// Work tile = 128 sorted KEY slots (chunks 2k, 2k+1) of one segment; the
// queries that can see them are the 192 slots of chunks 2k..2k+2, whose
// first 128 rows are the keys themselves (shared query-key), so one gathered
// x tile feeds every product.  Keys sit on TMEM lanes (one key row per
// thread), queries on columns:
//   S^T  = Xk Xq^T   (M=128, N=192, K=64)      dP^T = Vk dYq^T  (M=128, N=192, K=64)
//   elementwise: P^T (bf16, into tensor memory), E^T = tau inv_j dS^T (bf16, shared memory)
//   dV   = P^T dYq   (A from TMEM, M=128, N=64, K=192)
//   G    = E^T Xq    (M=128, N=64, K=192)
//   dQ   = E Xk      (E^T read MN-major; two M=128 halves over the 192 queries: K=128
//                     keys for queries 0..127, K=64 (keys of chunk 2k+1) for 128..191)
// Query slot r < 128 is also key slot r, so G and the first dQ half accumulate
// into one TMEM block; the key-role correction needs g_j . x_j, which equals
// sum_i e_ij (x_i . x_j) and is summed from S^T during the elementwise step.
// Gradients of every round are added into fp32 accumulators with vector
// reductions (red.global.add.v4.f32); their summation order is not fixed.
//
// A query attends to itself only when no other candidate is left (causal:
// its position is the smallest in its window); that flag is recomputed here
// from the window minima of positions.
//
// Warp roles (persistent CTA, one per SM):
//   warps 0-7  compute: warp w owns TMEM lanes 32*(w%4).. (key rows) and query
//              columns half (w/4); elementwise step, then the epilogue;
//   warps 8-10 producer: positions, per-query LSE, delta and causal key
//              bounds into a 2-stage ring, and 16-byte cp.async gathers of
//              the x, v and dY rows straight into the swizzled operand
//              layout (key norms are computed by the compute warps);
//   warp 11    MMA issuer.
#include "tc_common.cuh"

namespace lsh {

namespace {

constexpr int kK = 128;             // key slots per tile
constexpr int kQ = 192;             // query slots per tile
constexpr int kStages = 2;
constexpr int kRun = 8;             // consecutive key tiles of one segment per work unit
constexpr int kComputeWarps = 8;
constexpr int kProducerWarps = 3;
constexpr int kProducerThreads = kProducerWarps * 32;
constexpr int kMmaWarp = kComputeWarps + kProducerWarps;
constexpr int kThreads = (kMmaWarp + 1) * 32;
constexpr int kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;

// TMEM columns.  Elementwise phase: S^T [0,192), P^T packed [192,288), dP^T [288,480).
constexpr uint32_t cS = 0, cPT = 192, cD = 288;
// After it: dV [0,64), G + dQ rows 0-127 [64,128), dQ rows 64-191 [288,352).
constexpr uint32_t cDV = 0, cDX = 64, cQb = 288;

struct alignas(1024) Stage {
    uint8_t X[kQ * 128];            // x rows of the query slots (first 128 = key slots)   24 KB
    uint8_t V[kK * 128];            // v rows of the key slots                              16 KB
    uint8_t G[kQ * 128];            // dY rows of the query slots                           24 KB
    alignas(16) int32_t pos[256];   // positions of slots [128k - 64, 128k + 192); -1 if none
    alignas(16) int32_t qpos[kQ];   // original position of each query slot (-1 if none)
    alignas(16) float qlse2[kQ];    // LSE * log2(e) (+inf if none)
    alignas(16) float qdelta[kQ];   // dY . y
    alignas(16) int32_t qlim[kQ];   // causal: key bound, position + 1 when the query attends to itself alone;
                                    // otherwise: the one key position it does not take (-2: none)
    alignas(16) int32_t bk[256];    // bucket of slots [128k - 64, 128k + 192) (-1 if none); bucket mask only
    alignas(16) float qown[kQ];     // self penalty: weight of the query's own entry when it is alone
    int32_t cmin[4];                // smallest position of chunks 2k-1 .. 2k+2 (INT_MAX if none)
};

// Optional readings (template parameter FL, bits of lsh_attn_desc.flags).
constexpr int kMask = LSH_FLAG_BUCKET_MASK, kPen = LSH_FLAG_SELF_PENALTY;

struct BwdSmem {
    Stage st[kStages];
    uint8_t ET[3][kK * 128];        // tau inv_j dS^T, 3 blocks of 64 queries (48 KB)
    uint8_t carry[2][64 * 256];     // fp32 dQ rows of chunk 2k+2 handed to the next tile (2 x 16 KB)
    uint64_t full[kStages], empty[kStages];
    uint64_t bar_s, bar_p, bar_o, bar_free;
    uint64_t gx_ready;              // the second half's partial sums of g . x are in gxh
    uint64_t epi_done;              // every compute warp finished the previous tile's epilogue
    float gxh[kK];
    alignas(16) int ridx[kComputeWarps][2][32];   // row indices of the staged rows, per warp
    uint64_t drain;                 // timeout path: the MMA issuer's last products
    uint32_t tmem_base;
    int abort;
};

// Nothing in the kernel reads the accumulators, so the reduction carries no
// memory clobber: shared-memory loads around it may be scheduled freely.
__device__ __forceinline__ void red_add_v4(float *addr, float a, float b, float c, float d)
{
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b), "f"(c), "f"(d));
}

// Adds each lane's 64-float row `a` to row `rowg` of `acc` (skipped when
// rowg < 0) with coalesced vector reductions: the warp's 32 rows go through
// its 8 KB staging buffer (16-byte chunks swizzled by row against bank
// conflicts) and their row indices through `ridx` (32 ints), then each
// reduction instruction covers two whole rows, r and r + 16.
__device__ __forceinline__ void stage_rows(uint8_t *stg, int *ridx, int lane, const float *a, int rowg)
{
#pragma unroll
    for (int c = 0; c < 16; ++c)
        *reinterpret_cast<float4 *>(stg + lane * 256 + ((c ^ (lane & 15)) << 4)) =
            make_float4(a[4 * c], a[4 * c + 1], a[4 * c + 2], a[4 * c + 3]);
    ridx[lane] = rowg;
    __syncwarp();
}
// `add` (nullable): 32 more rows in the same staged layout, added on the way.
__device__ __forceinline__ void reduce_rows(const uint8_t *stg, const int *ridx, int lane, float *acc,
                                            const uint8_t *add = nullptr)
{
    const int c = lane & 15, r0 = (lane >> 4) * 16;
#pragma unroll 1
    for (int k = 0; k < 4; ++k) {
        const int4 r4 = *reinterpret_cast<const int4 *>(ridx + r0 + 4 * k);
        const int rows[4] = {r4.x, r4.y, r4.z, r4.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int it = 4 * k + u;
            const uint32_t off = (r0 + it) * 256 + ((c ^ it) << 4);
            float4 val = *reinterpret_cast<const float4 *>(stg + off);
            if (add) {
                const float4 g = *reinterpret_cast<const float4 *>(add + off);
                val.x += g.x; val.y += g.y; val.z += g.z; val.w += g.w;
            }
            if (rows[u] >= 0) red_add_v4(acc + (long long)rows[u] * kDim + 4 * c, val.x, val.y, val.z, val.w);
        }
    }
    __syncwarp();
}
__device__ __forceinline__ void flush_rows(uint8_t *stg, int *ridx, int lane, const float *a, float *acc, int rowg,
                                           int ph_role = -1, int ph_it = 0, int ph_ev = 0,
                                           const uint8_t *add = nullptr)
{
    stage_rows(stg, ridx, lane, a, rowg);
    if (ph_role >= 0 && lane == 0) LSH_PHASE(1, ph_role, ph_it, ph_ev);
    reduce_rows(stg, ridx, lane, acc, add);
    if (ph_role >= 0 && lane == 0) LSH_PHASE(1, ph_role, ph_it, ph_ev + 1);
}

// Chunk `ch` (elements 8ch .. 8ch+7) of bf16 row `row` of a K-major SW128 tile.
__device__ __forceinline__ void smem_chunk(const uint8_t *tile, int row, int ch, float *out);

// 1/|x| of row `row` of a gathered K-major SW128 tile (sum of squares in element
// order; 0 for a zero row).
__device__ __forceinline__ float key_inv_norm(const uint8_t *X, int row)
{
    float ssq = 0.f;
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) {
        float xr[8];
        smem_chunk(X, row, ch, xr);
#pragma unroll
        for (int e = 0; e < 8; ++e) ssq = fmaf(xr[e], xr[e], ssq);
    }
    return ssq > 0.f ? 1.0f / sqrtf(ssq) : 0.f;
}

// Chunk `ch` (elements 8ch .. 8ch+7) of bf16 row `row` of a K-major SW128 tile.
__device__ __forceinline__ void smem_chunk(const uint8_t *tile, int row, int ch, float *out)
{
    const uint4 u = *reinterpret_cast<const uint4 *>(tile + row * 128 + ((ch ^ (row & 7)) << 4));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        out[2 * e] = __uint_as_float(w[e] << 16);
        out[2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
    }
}

// One step of 16 query columns [C0 + 16 STEP, +16) of key row kr (position
// kpos, bucket kb) from the S^T and dP^T values s, dp: P^T into TMEM, E^T into
// shared memory.  With the self penalty, a lone query's own entry has the
// constant score (LSH_SELF_PENALTY_SCORE): its P is exp(penalty - LSE), from the
// prologue, which computes it without forming LSE, and its E is 0.
template <bool CAUSAL, int FL, int STEP>
__device__ __forceinline__ void key_row_step(const Stage &st, uint8_t (*ET)[kK * 128], uint32_t tl, int kr, int kpos,
                                             int kb, int C0, float sc, float ec, const float *s, const float *dp,
                                             float &gx)
{
    uint32_t pw[8], ew[8];
#pragma unroll
    for (int j4 = 0; j4 < 16; j4 += 4) {
        const int q0 = C0 + STEP * 16 + j4;
        // causal: key admitted iff its position < qlim; otherwise iff it differs from qlim
        const int4 qp4 = *reinterpret_cast<const int4 *>(&st.qlim[q0]);
        const float4 ql4 = *reinterpret_cast<const float4 *>(&st.qlse2[q0]);
        const float4 qd4 = *reinterpret_cast<const float4 *>(&st.qdelta[q0]);
        const int4 qb4 = (FL & kMask) ? *reinterpret_cast<const int4 *>(&st.bk[64 + q0]) : make_int4(0, 0, 0, 0);
        const int4 qo4 = (FL & kPen) ? *reinterpret_cast<const int4 *>(&st.qpos[q0]) : make_int4(0, 0, 0, 0);
        const float4 qw4 = (FL & kPen) ? *reinterpret_cast<const float4 *>(&st.qown[q0]) : make_float4(0, 0, 0, 0);
        const int qp[4] = {qp4.x, qp4.y, qp4.z, qp4.w};
        const float ql[4] = {ql4.x, ql4.y, ql4.z, ql4.w};
        const float qd[4] = {qd4.x, qd4.y, qd4.z, qd4.w};
        const int qb[4] = {qb4.x, qb4.y, qb4.z, qb4.w};
        const int qo[4] = {qo4.x, qo4.y, qo4.z, qo4.w};
        const float qw[4] = {qw4.x, qw4.y, qw4.z, qw4.w};
        float pv[4], ev[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            bool ok = CAUSAL ? (kpos < qp[u]) : (kpos != qp[u]);
            if (FL & kMask) ok = ok && kb == qb[u];
            const bool own = (FL & kPen) && kpos == qo[u];
            const float e2 = tc::fast_exp2(fmaf(s[j4 + u], sc, -ql[u]));
            pv[u] = ok ? (own ? qw[u] : e2) : 0.f;
            ev[u] = own ? 0.f : ec * pv[u] * (dp[j4 + u] - qd[u]);
            gx = fmaf(ev[u], s[j4 + u], gx);
        }
        pw[j4 / 2] = pack_bf16x2(pv[0], pv[1]);
        pw[j4 / 2 + 1] = pack_bf16x2(pv[2], pv[3]);
        ew[j4 / 2] = pack_bf16x2(ev[0], ev[1]);
        ew[j4 / 2 + 1] = pack_bf16x2(ev[2], ev[3]);
    }
    tc::tmem_st8(tl + cPT + C0 / 2 + STEP * 8, pw);
    const int blk = C0 >> 6;
#pragma unroll
    for (int c2 = 0; c2 < 2; ++c2) {
        const int ch = STEP * 2 + c2;
        const uint32_t off = (uint32_t)kr * 128u + (uint32_t)((ch ^ (kr & 7)) << 4);
        *reinterpret_cast<uint4 *>(ET[blk] + off) = make_uint4(ew[4 * c2], ew[4 * c2 + 1], ew[4 * c2 + 2], ew[4 * c2 + 3]);
    }
}

// Elementwise step for key row kr over query columns [C0, C0 + 64): P^T (bf16)
// into TMEM columns cPT + C0/2, E^T into shared-memory block C0/64, in four
// steps of 16 columns whose tensor-memory loads run one step ahead.  A
// candidate is a query at a later original position (causal) or at any other
// position; a causal query with no other candidate takes its own key.  Query
// metadata is read four queries per vector load.  Returns this block's part of
// g . x = sum_i e_i (x_i . x_k).  C0 is a run-time value so that the warps of
// all three column blocks share one copy of the code.
template <bool CAUSAL, int FL>
__device__ __forceinline__ float key_row_block(const Stage &st, uint8_t (*ET)[kK * 128], uint32_t tl, int kr, int kpos,
                                               int kb, int C0, float kinv, float tau, bool mark = false,
                                               int it = 0)
{
    const float sc = tau * kinv * kLog2e;
    const float ec = tau * kinv;
    float gx = 0.f;
    float sa[16], da[16], sb[16], db[16];
    if (mark) LSH_PHASE(1, 5, it, 0);
    tc::tmem_ld16(tl + cS + C0, sa);
    tc::tmem_ld16(tl + cD + C0, da);
    tc::tmem_ld_wait();
    if (mark) LSH_PHASE(1, 5, it, 1);
    tc::tmem_ld16(tl + cS + C0 + 16, sb);
    tc::tmem_ld16(tl + cD + C0 + 16, db);
    key_row_step<CAUSAL, FL, 0>(st, ET, tl, kr, kpos, kb, C0, sc, ec, sa, da, gx);
    if (mark) LSH_PHASE(1, 5, it, 2);
    tc::tmem_ld_wait();
    if (mark) LSH_PHASE(1, 5, it, 3);
    tc::tmem_ld16(tl + cS + C0 + 32, sa);
    tc::tmem_ld16(tl + cD + C0 + 32, da);
    key_row_step<CAUSAL, FL, 1>(st, ET, tl, kr, kpos, kb, C0, sc, ec, sb, db, gx);
    if (mark) LSH_PHASE(1, 5, it, 4);
    tc::tmem_ld_wait();
    tc::tmem_ld16(tl + cS + C0 + 48, sb);
    tc::tmem_ld16(tl + cD + C0 + 48, db);
    key_row_step<CAUSAL, FL, 2>(st, ET, tl, kr, kpos, kb, C0, sc, ec, sa, da, gx);
    if (mark) LSH_PHASE(1, 5, it, 5);
    tc::tmem_ld_wait();
    if (mark) LSH_PHASE(1, 5, it, 6);
    key_row_step<CAUSAL, FL, 3>(st, ET, tl, kr, kpos, kb, C0, sc, ec, sb, db, gx);
    if (mark) LSH_PHASE(1, 5, it, 7);
    return gx;
}

// Zero P^T and E^T for query columns [C0, C0 + 64) of key row kr.
template <int C0>
__device__ __forceinline__ void zero_block(uint8_t (*ET)[kK * 128], uint32_t tl, int kr)
{
    const uint32_t z[16] = {0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0};
    tc::tmem_st16(tl + cPT + C0 / 2, z);
    tc::tmem_st16(tl + cPT + C0 / 2 + 16, z);
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) {
        const uint32_t off = (uint32_t)kr * 128u + (uint32_t)((ch ^ (kr & 7)) << 4);
        *reinterpret_cast<uint4 *>(ET[C0 / 64] + off) = make_uint4(0, 0, 0, 0);
    }
}

// Work unit u = (bh, run, r) with r fastest: key tiles k = kRun * run .. of
// segment (bh, r), taken in order by one CTA, so the dQ rows of chunk 2k+2
// that tile k computes can be handed to tile k+1 instead of being reduced
// twice.  Units in flight at the same time share one head's rows in L2.
// The iterator keeps the unit's coordinates, so the divisions that locate a
// unit run once per unit, not once per tile.
struct TileIter {
    long long unit;                 // >= n_units: done
    int j;                          // tile within the unit
    int r, k0;                      // round; first key tile of the unit's run
    long long bh, seg;
};
struct TileCoord {
    int r, k;
    long long bh, seg;
    bool next_adjacent;             // the CTA's next tile is (seg, k + 1)
};
__device__ __forceinline__ void tile_locate(TileIter &t, int R, int n_runs)
{
    t.r = (int)(t.unit % R);
    const long long br = t.unit / R;
    t.k0 = (int)(br % n_runs) * kRun;
    t.bh = br / n_runs;
    t.seg = t.bh * R + t.r;
}
__device__ __forceinline__ TileIter tile_begin(long long unit, int R, int n_runs)
{
    TileIter t;
    t.unit = unit;
    t.j = 0;
    tile_locate(t, R, n_runs);
    return t;
}
__device__ __forceinline__ TileCoord tile_coord(const TileIter &t, int n_k)
{
    TileCoord c;
    c.r = t.r;
    c.k = t.k0 + t.j;
    c.bh = t.bh;
    c.seg = t.seg;
    c.next_adjacent = t.j + 1 < kRun && c.k + 1 < n_k;
    return c;
}
__device__ __forceinline__ void tile_advance(TileIter &t, int R, int n_k, int n_runs)
{
    if (t.j + 1 < kRun && t.k0 + t.j + 1 < n_k) {
        ++t.j;
    } else {
        t.unit += gridDim.x;
        t.j = 0;
        tile_locate(t, R, n_runs);
    }
}

template <bool CAUSAL, int FL>
__global__ void __launch_bounds__(kThreads, 1)
attn_bwd_tc_kernel(const __nv_bfloat16 *__restrict__ x, const __nv_bfloat16 *__restrict__ v,
                   const __nv_bfloat16 *__restrict__ dout, const int32_t *__restrict__ perm,
                   const uint16_t *__restrict__ bkt, const float *__restrict__ lse_all,
                   const float *__restrict__ delta, const float *__restrict__ own, float *__restrict__ dx_acc,
                   float *__restrict__ dv_acc, int L,
                   int R, long long n_units, float tau, uint32_t prev_mask, uint32_t *__restrict__ status)
{
    extern __shared__ uint8_t smem_raw[];
    BwdSmem &sm = *reinterpret_cast<BwdSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n_k = (L + kK - 1) / kK;          // the last tile may hold one chunk only
    const int n_runs = (n_k + kRun - 1) / kRun;

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            tc::mbar_init(&sm.full[s], kProducerThreads);
            tc::mbar_init(&sm.empty[s], kComputeWarps);
        }
        tc::mbar_init(&sm.bar_s, 1);
        tc::mbar_init(&sm.bar_p, kComputeWarps);
        tc::mbar_init(&sm.bar_o, 1);
        tc::mbar_init(&sm.bar_free, kComputeWarps);
        tc::mbar_init(&sm.gx_ready, kComputeWarps / 2);
        tc::mbar_init(&sm.epi_done, kComputeWarps);
        tc::mbar_init(&sm.drain, 1);
        sm.abort = 0;
        tc::fence_mbar_init();
    }
    if (warp == 0) tc::tmem_alloc(&sm.tmem_base, kTmemCols);
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    if (warp >= kComputeWarps && warp < kMmaWarp) {
        // ================= producer group
        const int ptid = tid - kComputeWarps * 32, pw = ptid >> 5;
        // positions of slots [128k - 64, 128k + 192) of the next tile, loaded a tile ahead
        constexpr int kPosPer = (256 + kProducerThreads - 1) / kProducerThreads;
        int pn[kPosPer], bn[kPosPer];
        auto load_pos = [&](const TileIter &t) {
            const TileCoord c = tile_coord(t, n_k);
            const int32_t *P = perm + c.seg * L;
            const int slot0 = c.k * kK - 64;
#pragma unroll
            for (int j = 0; j < kPosPer; ++j) {
                const int e = ptid + j * kProducerThreads;
                const int sl = slot0 + e;
                const bool in = e < 256 && sl >= 0 && sl < L;
                const int pl = P[min(max(sl, 0), L - 1)];
                // a permutation entry outside [0, L) leaves its slot empty and is reported
                const bool good = (unsigned)pl < (unsigned)L;
                if (in && !good) atomicOr(status, kStatusBadPerm);
                pn[j] = in && good ? pl : -1;
                if (FL & kMask) bn[j] = pn[j] >= 0 ? (int)bkt[c.seg * L + pn[j]] : -1;
            }
        };
        TileIter ti = tile_begin(blockIdx.x, R, n_runs);
        if (ti.unit < n_units) load_pos(ti);
        for (int it = 0; ti.unit < n_units; ++it) {
            const int s = it % kStages;
            if (ptid == 0) LSH_PHASE(1, 0, it, 0);
            bool ok = it < kStages ||
                      tc::mbar_wait(&sm.empty[s], (uint32_t)((it / kStages) - 1) & 1u, &sm.abort, status);
            if (tc::named_bar_or(1, kProducerThreads, !ok)) break;
            if (ptid == 0) LSH_PHASE(1, 0, it, 1);
            Stage &st = sm.st[s];
            const long long rowbase = tile_coord(ti, n_k).bh * L;
#pragma unroll
            for (int j = 0; j < kPosPer; ++j) {
                const int e = ptid + j * kProducerThreads;
                if (e < 256) {
                    st.pos[e] = pn[j];
                    if (FL & kMask) st.bk[e] = bn[j];
                }
            }
            tc::named_bar_sync(1, kProducerThreads);
            const TileCoord pc = tile_coord(ti, n_k);
            const int tile_k = pc.k;
            const bool prev = (prev_mask >> pc.r) & 1u;     // previous chunk alone: no lone queries
            // per-query LSE and delta: loads issued now, used after the copies are issued
            static_assert(kQ == 2 * kProducerThreads, "two queries per producer thread");
            int qp[2];
            float ql[2], qd[2], qw[2] = {0.f, 0.f};
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int q = min(ptid + j * kProducerThreads, kQ - 1);
                qp[j] = st.pos[64 + q];
                const long long rp = rowbase + max(qp[j], 0);
                ql[j] = lse_all[rp];
                qd[j] = delta[rp];
                if (FL & kPen) qw[j] = own[rp];
            }
            // x, dY rows of the 192 query slots and v rows of the 128 key slots: thread t
            // copies chunk t % 8 of rows t / 8 + 12 j (zero fill for a missing slot)
            {
                constexpr int kRowStep = kProducerThreads / 8;
                const int ch = ptid & 7, r0 = ptid >> 3;
                int pr[kQ / kRowStep];
#pragma unroll
                for (int j = 0; j < kQ / kRowStep; ++j) pr[j] = st.pos[64 + r0 + kRowStep * j];
#pragma unroll
                for (int j = 0; j < kQ / kRowStep; ++j) {
                    const int row = r0 + kRowStep * j;
                    const uint32_t off = (uint32_t)row * 128u + (uint32_t)((ch ^ (row & 7)) << 4);
                    const long long src = (rowbase + max(pr[j], 0)) * kDim + ch * 8;
                    const uint32_t nb = pr[j] >= 0 ? 16u : 0u;
                    tc::cp_async16_zfill(st.X + off, x + src, nb);
                    tc::cp_async16_zfill(st.G + off, dout + src, nb);
                    if (row < kK) tc::cp_async16_zfill(st.V + off, v + src, nb);
                }
            }
            tc::cp_async_commit();
            if (ptid == 0) LSH_PHASE(1, 0, it, 2);
            // smallest position of chunks 2k-1 .. 2k+2 (warp w takes chunks w, w + 3)
            for (int c = pw; c < 4 && CAUSAL && !(FL & kMask); c += kProducerWarps) {
                const int a0 = st.pos[c * 64 + lane], a1 = st.pos[c * 64 + 32 + lane];
                int mn = min(a0 >= 0 ? a0 : INT_MAX, a1 >= 0 ? a1 : INT_MAX);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, o));
                if (lane == 0) st.cmin[c] = mn;
            }
            tc::named_bar_sync(1, kProducerThreads);
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int q = ptid + j * kProducerThreads;
                if (q < kQ) {
                    const int p = qp[j];
                    // Does the query attend to itself alone?  Causal, no mask: its position is
                    // the smallest of its window (chunks 2k-1+q/64 and 2k+q/64).  With the bucket
                    // mask: the stable sort keeps a bucket's slots contiguous and in position
                    // order, so it has a candidate iff the slot before it (or, non-causal, after
                    // it) lies in its window and holds the same bucket.  Non-causal, no mask: never.
                    bool lone = false;
                    if (prev) {
                    } else if (FL & kMask) {
                        const int e = 64 + q, slot = tile_k * kK + q, b = st.bk[e];
                        const bool prev = slot >= 1 && st.bk[e - 1] == b;
                        const bool next = !CAUSAL && (slot & 63) != 63 && st.bk[e + 1] == b;
                        lone = p >= 0 && !prev && !next;
                    } else if (CAUSAL) {
                        const int qa = q >> 6;
                        lone = p >= 0 && p == min(st.cmin[qa], st.cmin[qa + 1]);
                    }
                    st.qpos[q] = p;
                    st.qlse2[q] = p >= 0 ? ql[j] * kLog2e : INFINITY;
                    st.qdelta[q] = p >= 0 ? qd[j] : 0.f;
                    if (FL & kPen) st.qown[q] = p >= 0 ? qw[j] : 0.f;
                    st.qlim[q] = CAUSAL ? (lone ? p + 1 : p) : (lone ? -2 : p);
                }
            }
            tile_advance(ti, R, n_k, n_runs);
            if (ti.unit < n_units) load_pos(ti);
            if (ptid == 0) LSH_PHASE(1, 0, it, 3);
            // with two stages the producer cannot run further ahead: publish this stage now
            tc::cp_async_wait<0>();
            tc::fence_async_smem();
            tc::mbar_arrive(&sm.full[s]);
            if (ptid == 0) LSH_PHASE(1, 0, it, 4);
        }
    } else if (warp == kMmaWarp) {
        // ================= MMA issuer
        if (lane == 0) {
            constexpr uint32_t id_s = tc::idesc_bf16(128, kQ, 0, 0);
            constexpr uint32_t id_kv = tc::idesc_bf16(128, kDim, 0, 1);   // A K-major, B MN-major
            constexpr uint32_t id_q = tc::idesc_bf16(128, kDim, 1, 1);    // A MN-major, B MN-major
            const uint64_t de0 = tc::sw128_desc(tc::smem_u32(sm.ET[0])), de1 = tc::sw128_desc(tc::smem_u32(sm.ET[1])),
                           de2 = tc::sw128_desc(tc::smem_u32(sm.ET[2]));
            // E = (E^T)^T read MN-major: 64-query blocks 16 KB apart (leading byte offset)
            const uint64_t de0l = tc::sw128_desc(tc::smem_u32(sm.ET[0]), kK * 128),
                           de1l = tc::sw128_desc(tc::smem_u32(sm.ET[1]), kK * 128);
            TileIter ti = tile_begin(blockIdx.x, R, n_runs);
            for (int it = 0; ti.unit < n_units; ++it, tile_advance(ti, R, n_k, n_runs)) {
                const int s = it % kStages;
                const uint32_t ph = (uint32_t)it & 1u;
                LSH_PHASE(1, 1, it, 0);
                if (!tc::mbar_wait(&sm.full[s], (uint32_t)(it / kStages) & 1u, &sm.abort, status)) break;
                LSH_PHASE(1, 1, it, 1);
                if (it > 0 && !tc::mbar_wait(&sm.bar_free, ph ^ 1u, &sm.abort, status)) break;
                LSH_PHASE(1, 1, it, 2);
                tc::tc_fence_after();
                const Stage &st = sm.st[s];
                const uint64_t dxs = tc::sw128_desc(tc::smem_u32(st.X)), dvs = tc::sw128_desc(tc::smem_u32(st.V)),
                               dgs = tc::sw128_desc(tc::smem_u32(st.G));
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    tc::mma_bf16(tmem + cS, tc::desc_add(dxs, kk * 32), tc::desc_add(dxs, kk * 32), id_s, kk > 0);
                    tc::mma_bf16(tmem + cD, tc::desc_add(dvs, kk * 32), tc::desc_add(dgs, kk * 32), id_s, kk > 0);
                }
                tc::mma_commit(&sm.bar_s);
#ifdef LSH_PHASE_TRACE
                // tuning build: when the products complete, as the issuer sees it
                if (tc::mbar_wait(&sm.bar_s, ph, &sm.abort, status)) LSH_PHASE(1, 1, it, 5);
#endif
                if (!tc::mbar_wait(&sm.bar_p, ph, &sm.abort, status)) break;
                LSH_PHASE(1, 1, it, 3);
                tc::tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 12; ++kk) {
                    const uint64_t dea = tc::desc_add(kk < 4 ? de0 : kk < 8 ? de1 : de2, (kk & 3) * 32);
                    tc::mma_bf16_ts(tmem + cDV, tmem + cPT + kk * 8, tc::desc_add(dgs, kk * 2048), id_kv, kk > 0);
                    tc::mma_bf16(tmem + cDX, dea, tc::desc_add(dxs, kk * 2048), id_kv, kk > 0);
                }
                // E = (E^T)^T read MN-major: 64-query blocks 16 KB apart (leading byte offset).
                // The second half (queries 64..191) is read only for chunk 2k+2 (rows
                // 128..191), whose queries see the keys of chunk 2k+1 alone: its K range is
                // keys 64..127 (rows 64..127 of that product are never read).
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    tc::mma_bf16(tmem + cDX, tc::desc_add(de0l, kk * 2048), tc::desc_add(dxs, kk * 2048),
                                 id_q, true);
#pragma unroll
                for (int kk = 4; kk < 8; ++kk)
                    tc::mma_bf16(tmem + cQb, tc::desc_add(de1l, kk * 2048), tc::desc_add(dxs, kk * 2048),
                                 id_q, kk > 4);
                tc::mma_commit(&sm.bar_o);
                LSH_PHASE(1, 1, it, 4);
#ifdef LSH_PHASE_TRACE
                if (tc::mbar_wait(&sm.bar_o, ph, &sm.abort, status)) LSH_PHASE(1, 1, it, 6);
#endif
            }
            if (*reinterpret_cast<volatile int *>(&sm.abort)) tc::mma_drain(&sm.drain, status);
        }
    } else {
        // ================= compute warps
        const int quad = warp & 3, half = warp >> 2;
        const int kr = quad * 32 + lane;
        const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);
        TileIter ti = tile_begin(blockIdx.x, R, n_runs);
        bool carry_in = false;                       // this tile's chunk-2k rows hold a handed-over dQ part
        bool have_next_kinv = false;
        float next_kinv = 0.f;
        for (int it = 0; ti.unit < n_units; ++it, tile_advance(ti, R, n_k, n_runs)) {
            const int s = it % kStages;
            const uint32_t ph = (uint32_t)it & 1u;
            if (tid == 0) LSH_PHASE(1, 2, it, 0);
            if (!tc::mbar_wait(&sm.full[s], (uint32_t)(it / kStages) & 1u, &sm.abort, status)) break;
            if (tid == 0) LSH_PHASE(1, 2, it, 1);
            const Stage &st = sm.st[s];
            const TileCoord tcd = tile_coord(ti, n_k);
            const long long rowbase = tcd.bh * L;
            const int kpos = st.pos[64 + kr];
            const int kb = (FL & kMask) ? st.bk[64 + kr] : 0;
            // 1/|x_k| of this key row, unless computed while the previous tile's products ran
            const float kinv = have_next_kinv ? next_kinv : key_inv_norm(st.X, kr);
            if (!tc::mbar_wait(&sm.bar_s, ph, &sm.abort, status)) break;
            if (tid == 0) LSH_PHASE(1, 2, it, 2);
            tc::tc_fence_after();
            // ---- elementwise.  E^T and gxh are rewritten here: wait until no warp still
            // stages the previous tile's rows in them.
            if (it > 0 && !tc::mbar_wait(&sm.epi_done, (uint32_t)(it - 1) & 1u, &sm.abort, status)) break;
            const int erole_ev = warp == 0 ? 0 : warp == 4 ? 4 : -1;
            if (erole_ev >= 0 && lane == 0) LSH_PHASE(1, 7, it, erole_ev);
            float gx;                                // partial g . x of key row kr
            // keys of chunk 2k (quads 0, 1) see queries of chunks 2k, 2k+1 (columns 0..127),
            // keys of chunk 2k+1 those of chunks 2k+1, 2k+2 (64..191); each half takes 64
            // (a round whose window is the previous chunk alone: keys of chunk 2k+1 see
            // only the queries of chunk 2k+2, keys of chunk 2k only those of 2k+1, so
            // the lower column block is zero as well)
            const int c0 = quad < 2 ? half * 64 : 64 + half * 64;
            const bool prev = (prev_mask >> tcd.r) & 1u;
            if (prev && half == 0) {
                gx = 0.f;
                if (quad < 2) zero_block<0>(sm.ET, tl, kr);
                else zero_block<64>(sm.ET, tl, kr);
            } else {
                gx = key_row_block<CAUSAL, FL>(st, sm.ET, tl, kr, kpos, kb, c0, kinv, tau, tid == 0, it);
            }
            if (half == 0) {
                if (quad < 2) zero_block<128>(sm.ET, tl, kr);
                else zero_block<0>(sm.ET, tl, kr);
            }
            if (erole_ev >= 0 && lane == 0) LSH_PHASE(1, 7, it, erole_ev + 1);
            if (half == 1) sm.gxh[kr] = gx;
            tc::tmem_st_wait();
            if (erole_ev >= 0 && lane == 0) LSH_PHASE(1, 7, it, erole_ev + 2);
            tc::fence_async_smem();
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                tc::mbar_arrive(&sm.bar_p);
                if (half == 1) tc::mbar_arrive(&sm.gx_ready);
            }
            if (tid == 0) LSH_PHASE(1, 2, it, 3);
            // the next tile's key norm while this tile's products run
            have_next_kinv = false;
            {
                TileIter nx = ti;
                tile_advance(nx, R, n_k, n_runs);
                if (nx.unit < n_units) {
                    const int s2 = (it + 1) % kStages;
                    if (!tc::mbar_wait(&sm.full[s2], (uint32_t)((it + 1) / kStages) & 1u, &sm.abort, status)) break;
                    next_kinv = key_inv_norm(sm.st[s2].X, kr);
                    have_next_kinv = true;
                }
            }
            if (!tc::mbar_wait(&sm.bar_o, ph, &sm.abort, status)) break;
            if (tid == 0) LSH_PHASE(1, 2, it, 4);
            tc::tc_fence_after();
            // ---- epilogue: reductions into the fp32 accumulators.  The staging
            // buffers reuse memory the MMAs no longer read: E^T and this stage's v rows.
            uint8_t *stg = warp < 6 ? reinterpret_cast<uint8_t *>(sm.ET) + warp * 8192
                                    : const_cast<uint8_t *>(st.V) + (warp - 6) * 8192;
            const int krow = kpos >= 0 ? (int)rowbase + kpos : -1;
            // Every warp first moves its outputs from tensor memory to registers and
            // releases the columns, so the next tile's S^T and dP^T products run while
            // this tile's rows are reduced.
            float a[kDim];
            auto release_tmem = [&] {
                tc::tmem_ld_wait();
                tc::tc_fence_before();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&sm.bar_free);
            };
            if (half == 0) {
                // slot kr: query-role dQ plus key-role g, less inv^2 (g . x) x
                const int prole = warp == 0 ? 4 : -1;
                if (prole >= 0 && lane == 0) LSH_PHASE(1, prole, it, 0);
#pragma unroll
                for (int c = 0; c < 4; ++c) tc::tmem_ld16(tl + cDX + c * 16, a + c * 16);
                release_tmem();
                if (prole >= 0 && lane == 0) LSH_PHASE(1, prole, it, 1);
                if (!tc::mbar_wait(&sm.gx_ready, ph, &sm.abort, status)) break;
                const float cf = kinv * kinv * (gx + sm.gxh[kr]);
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    float xr[8];
                    smem_chunk(st.X, kr, ch, xr);
#pragma unroll
                    for (int e = 0; e < 8; ++e) a[ch * 8 + e] = fmaf(-cf, xr[e], a[ch * 8 + e]);
                }
                // chunk 2k rows: plus the previous tile's part of their dQ, when handed over
                const uint8_t *add = quad < 2 && carry_in ? sm.carry[(it - 1) & 1] + quad * 32 * 256 : nullptr;
                flush_rows(stg, sm.ridx[warp][0], lane, a, dx_acc, krow, prole, it, 2, add);
                if (prole >= 0 && lane == 0) LSH_PHASE(1, prole, it, 4);
            } else {
                if (tid == 128) LSH_PHASE(1, 3, it, 0);
                if (quad < 2) {
#pragma unroll
                    for (int c = 0; c < 4; ++c) tc::tmem_ld16(tl + cDV + c * 16, a + c * 16);
                    release_tmem();
                    flush_rows(stg, sm.ridx[warp][0], lane, a, dv_acc, krow);
                } else {
                    // the dV row (staged first), then query row 64 + kr (chunk 2k+2): handed
                    // to the next tile when that is k+1 of this segment, else reduced here,
                    // staged in this stage's dY rows, which the MMAs no longer read
#pragma unroll
                    for (int c = 0; c < 4; ++c) tc::tmem_ld16(tl + cDV + c * 16, a + c * 16);
                    tc::tmem_ld_wait();
                    stage_rows(stg, sm.ridx[warp][0], lane, a, krow);
#pragma unroll
                    for (int c = 0; c < 4; ++c) tc::tmem_ld16(tl + cQb + c * 16, a + c * 16);
                    release_tmem();
                    if (warp == 6 && lane == 0) LSH_PHASE(1, 6, it, 0);
                    uint8_t *stg2 = const_cast<uint8_t *>(st.G) + (quad - 2) * 8192;
                    if (tcd.next_adjacent) {
                        const int cr = kr - 64;
                        uint8_t *cb = sm.carry[it & 1] + cr * 256;
#pragma unroll
                        for (int c = 0; c < 16; ++c)
                            *reinterpret_cast<float4 *>(cb + ((c ^ (cr & 15)) << 4)) =
                                make_float4(a[4 * c], a[4 * c + 1], a[4 * c + 2], a[4 * c + 3]);
                    } else {
                        const int qp = st.qpos[64 + kr];
                        stage_rows(stg2, sm.ridx[warp][1], lane, a, qp >= 0 ? (int)rowbase + qp : -1);
                    }
                    reduce_rows(stg, sm.ridx[warp][0], lane, dv_acc);
                    if (warp == 6 && lane == 0) LSH_PHASE(1, 6, it, 1);
                    if (!tcd.next_adjacent) reduce_rows(stg2, sm.ridx[warp][1], lane, dx_acc);
                    if (warp == 6 && lane == 0) LSH_PHASE(1, 6, it, 2);
                }
                if (tid == 128) LSH_PHASE(1, 3, it, 1);
            }
            if (tid == 0) LSH_PHASE(1, 2, it, 5);
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                tc::mbar_arrive(&sm.empty[s]);
                tc::mbar_arrive(&sm.epi_done);
            }
            carry_in = tcd.next_adjacent;
        }
    }

    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace

template <bool CAUSAL, int FL>
static cudaError_t launch_bwd(const Problem &p, const void *x, const void *v, const void *dout, const int32_t *perm,
                              const uint16_t *bkt, const float *lse_all, const float *delta, const float *own,
                              float *dx_acc, float *dv_acc, uint32_t *status, cudaStream_t st)
{
    static_assert(sizeof(BwdSmem) + 1024 <= 232448, "shared memory per CTA");
    const size_t smem = sizeof(BwdSmem) + 1024;
    auto kern = attn_bwd_tc_kernel<CAUSAL, FL>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    const long long n_units = p.S() * (((p.L + kK - 1) / kK + kRun - 1) / kRun);
    const unsigned grid = (unsigned)std::min<long long>(n_units, (long long)sms);
    kern<<<grid, kThreads, smem, st>>>((const __nv_bfloat16 *)x, (const __nv_bfloat16 *)v,
                                       (const __nv_bfloat16 *)dout, perm, bkt, lse_all, delta, own, dx_acc, dv_acc,
                                       p.L,
                                       p.R, n_units, 1.0f / sqrtf((float)p.d), (uint32_t)p.prev_mask, status);
    return cudaGetLastError();
}

cudaError_t launch_attn_bwd_tc(const Problem &p, const void *x, const void *v, const void *dout, const int32_t *perm,
                               const uint16_t *bkt, const float *lse_all, const float *delta, const float *own,
                               float *dx_acc, float *dv_acc, uint32_t *status, cudaStream_t st)
{
    // key norms are computed in the kernel from the gathered rows
    const int fl = p.flags & (kMask | kPen);
#define LSH_BWD_CASE(C, F) \
    return launch_bwd<C, F>(p, x, v, dout, perm, bkt, lse_all, delta, own, dx_acc, dv_acc, status, st)
    if (p.causal) {
        switch (fl) {
        case 0: LSH_BWD_CASE(true, 0);
        case kMask: LSH_BWD_CASE(true, kMask);
        case kPen: LSH_BWD_CASE(true, kPen);
        default: LSH_BWD_CASE(true, kMask | kPen);
        }
    }
    switch (fl) {
    case 0: LSH_BWD_CASE(false, 0);
    case kMask: LSH_BWD_CASE(false, kMask);
    case kPen: LSH_BWD_CASE(false, kPen);
    default: LSH_BWD_CASE(false, kMask | kPen);
    }
#undef LSH_BWD_CASE
}

}  // namespace lsh

LSH_PHASE_EXPORT(bwd)
