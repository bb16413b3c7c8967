// gather_sorted + chunk_attn forward on the tensor cores (bf16, d = 64, m = 64).
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
//   gather   rows x[perm[s]] and v[perm[s]] for the 192 window slots, 16-byte
//            cp.async copies written straight into the 128-byte-swizzled
//            K-major layout the tensor core reads;
//   S = Q K^T  tcgen05.mma M=128, N=192, K=64 into tensor memory (raw
//            dot products x_i . x_j, bf16 in, fp32 accumulate);
//   softmax  one query row per thread: s_ij = (x_i . x_j) / |x_j| / sqrt(d)
//            (unit keys), masked to the window of the row's chunk, to
//            earlier original positions when causal, and never the query's
//            own position unless nothing else is left ("Implementation
//            Reading"); full softmax (the window fits), P written as bf16;
//   O = P V  tcgen05.mma M=128, N=64, K=192 (V read MN-major);
//   store    o_r and lse_r at the query's original position (the unsort).
//
// Two CTAs per SM (96 KB shared memory, 256 TMEM columns each) overlap one
// CTA's gather and MMAs with the other's softmax.
#include "tc_common.cuh"

namespace lsh {

namespace {

constexpr int kQ = 128;             // query slots per tile
constexpr int kW = 192;             // window rows (keys)
constexpr int kThreads = 128;
constexpr int kTmemCols = 256;      // S: 192 columns, O: 64 columns
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

struct FwdSmem {
    uint8_t X[kW * 128];            // gathered x rows, K-major SW128 (24 KB)
    uint8_t V[kW * 128];            // gathered v rows (24 KB)
    uint8_t P[3][kQ * 128];         // probabilities, 3 K-blocks of 64 keys (48 KB)
    alignas(16) int32_t pos[kW];
    alignas(16) float inv[kW];
    uint64_t bar_s, bar_o;
    uint32_t tmem_base;
    int abort;
};

// Softmax of one query row (thread) over the 128 window columns its chunk may
// see: window columns [BASE, BASE + 128) (chunk 2k: BASE = 0, chunk 2k+1:
// BASE = 64); `jlo` skips the missing chunk -1 of the first tile.  Writes the
// row of P (bf16, zeros elsewhere) into shared memory.
//
// Scores are s_j = tau (x_i . x_j) / |x_j| <= tau |x_i| (Cauchy-Schwarz), so
// M = tau |x_i| bounds the row maximum and p_j = exp(s_j - M) needs no max
// pass: one sweep over tensor memory gives P and l = sum p_j, and
// lse = M + log(l).  When the bound is so loose that every p_j would
// underflow (|x_i| in the hundreds) the warp redoes the row with the exact
// maximum.  A row with no candidate at all attends to itself (p = 1 there,
// lse = tau |x_i|).
template <int BASE>
__device__ __forceinline__ void softmax_row(FwdSmem &sm, uint32_t taddr, bool ok, int jlo, int i, int qpos, float qinv,
                                            int causal, float tau, float &l, float &row_lse)
{
    const float sl2 = tau * kLog2e;
    const float bound = qinv > 0.f ? tau / qinv : 0.f;      // tau |x_i|
    // pass over the 8 TMEM chunks of 16 columns; `shift` is the log2-domain offset
    auto sweep = [&](float shift, float &lsum, bool &any) {
        lsum = 0.f;
        any = false;
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
            float v[16];
            if (ok) {
                tc::tmem_ld16(taddr + (uint32_t)(BASE + c * 16), v);
                tc::tmem_ld_wait();
            }
            uint32_t w[8];
#pragma unroll
            for (int e4 = 0; e4 < 16; e4 += 4) {
                const int4 kp = *reinterpret_cast<const int4 *>(&sm.pos[BASE + c * 16 + e4]);
                const float4 kv = *reinterpret_cast<const float4 *>(&sm.inv[BASE + c * 16 + e4]);
                const int kpa[4] = {kp.x, kp.y, kp.z, kp.w};
                const float kva[4] = {kv.x, kv.y, kv.z, kv.w};
                float pe[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int j = c * 16 + e4 + e;
                    const bool valid = (j >= jlo) && (causal ? (kpa[e] < qpos) : (kpa[e] != qpos));
                    const float p = exp2f(fmaf(v[e4 + e], kva[e] * sl2, -shift));
                    pe[e] = valid ? p : 0.f;
                    any |= valid;
                    lsum += pe[e];
                }
                w[e4 / 2] = pack_bf16x2(pe[0], pe[1]);
                w[e4 / 2 + 1] = pack_bf16x2(pe[2], pe[3]);
            }
            // window column BASE + 16c .. +15 -> P block (BASE + 16c) / 64, chunks 2 at a time
            const int col = BASE + c * 16;
            uint8_t *blk = sm.P[col >> 6];
            const int ch0 = (col & 63) >> 3;
            *reinterpret_cast<uint4 *>(blk + i * 128 + ((ch0 ^ (i & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
            *reinterpret_cast<uint4 *>(blk + i * 128 + (((ch0 + 1) ^ (i & 7)) << 4)) = make_uint4(w[4], w[5], w[6], w[7]);
        }
    };
    float lsum;
    bool any;
    sweep(bound * kLog2e, lsum, any);
    l = lsum;
    row_lse = bound + kLn2 * log2f(lsum);
    // exact-maximum redo for rows whose bound underflowed every term
    const bool redo = any && !(lsum > 1e-30f);
    if (__any_sync(0xffffffffu, redo)) {
        float mx = -INFINITY;
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
            float v[16];
            if (ok) {
                tc::tmem_ld16(taddr + (uint32_t)(BASE + c * 16), v);
                tc::tmem_ld_wait();
            }
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const int j = c * 16 + e;
                const int kp = sm.pos[BASE + j];
                const bool valid = (j >= jlo) && (causal ? (kp < qpos) : (kp != qpos));
                if (valid) mx = fmaxf(mx, v[e] * sm.inv[BASE + j] * tau);
            }
        }
        // every thread of the warp takes part (tcgen05.ld is warp-wide); rows that
        // did not need the redo recompute exactly what they already wrote
        const float shift = redo ? mx * kLog2e : bound * kLog2e;
        float l2;
        bool any2;
        sweep(shift, l2, any2);
        if (redo) {
            l = l2;
            row_lse = mx + kLn2 * log2f(l2);
        }
    }
    // zero the columns outside [BASE, BASE + 128)
    {
        constexpr int zcol = BASE == 0 ? 128 : 0;
        uint8_t *blk = sm.P[zcol >> 6];
#pragma unroll
        for (int ch = 0; ch < 8; ++ch)
            *reinterpret_cast<uint4 *>(blk + i * 128 + ((ch ^ (i & 7)) << 4)) = make_uint4(0, 0, 0, 0);
    }
    if (!any) {
        // nothing but the query itself: p = 1 on its own column (window row 64 + i)
        const int col = 64 + i;
        uint8_t *blk = sm.P[col >> 6];
        const int cc = col & 63;
        const int ch = cc >> 3;
        uint32_t w[4] = {0, 0, 0, 0};
        const int e = cc & 7;
        w[e >> 1] = (e & 1) ? 0x3F800000u : 0x00003F80u;       // bf16 1.0 in the low or high half
        *reinterpret_cast<uint4 *>(blk + i * 128 + ((ch ^ (i & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
        l = 1.f;
        row_lse = bound;                                         // tau * x_i . (x_i / |x_i|)
    }
}

__global__ void __launch_bounds__(kThreads, 2)
attn_fwd_tc_kernel(const __nv_bfloat16 *__restrict__ x, const __nv_bfloat16 *__restrict__ v,
                   const int32_t *__restrict__ perm, const float *__restrict__ invnorm,
                   __nv_bfloat16 *__restrict__ o_r, float *__restrict__ lse, int L, int R, long long n_tiles,
                   int causal, float tau, uint32_t *__restrict__ status)
{
    extern __shared__ uint8_t smem_raw[];
    FwdSmem &sm = *reinterpret_cast<FwdSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n_k = L / kQ;

    if (tid == 0) {
        tc::mbar_init(&sm.bar_s, 1);
        tc::mbar_init(&sm.bar_o, 1);
        sm.abort = 0;
        tc::fence_mbar_init();
    }
    if (warp == 0) tc::tmem_alloc(&sm.tmem_base, kTmemCols);
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    const uint32_t tS = tmem, tO = tmem + kW;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    uint32_t phase = 0;

    for (long long tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, phase ^= 1u) {
        // tile order (bh, k, r): concurrent tiles share a head's rows in L2
        const int r = (int)(tile % R);
        const long long bk = tile / R;
        const int k = (int)(bk % n_k);
        const long long bh = bk / n_k;
        const long long seg = bh * R + r;
        const int32_t *P = perm + seg * L;
        const __nv_bfloat16 *X = x + bh * L * kDim;
        const __nv_bfloat16 *V = v + bh * L * kDim;
        const int slot0 = k * kQ - 64;          // window slot of row 0

        // ---- positions and key norms of the window
        for (int w = tid; w < kW; w += kThreads) {
            int s = slot0 + w;
            int p = s >= 0 ? P[s] : -1;
            sm.pos[w] = p;
            sm.inv[w] = p >= 0 ? invnorm[bh * L + p] : 0.f;
        }
        __syncthreads();
        // ---- gather rows into the swizzled operand tiles
        for (int c = tid; c < kW * 8; c += kThreads) {
            int w = c >> 3, ch = c & 7;
            uint32_t off = (uint32_t)w * 128u + (uint32_t)((ch ^ (w & 7)) << 4);
            int p = sm.pos[w];
            if (p >= 0) {
                tc::cp_async16(sm.X + off, X + (long long)p * kDim + ch * 8);
                tc::cp_async16(sm.V + off, V + (long long)p * kDim + ch * 8);
            } else {
                *reinterpret_cast<uint4 *>(sm.X + off) = make_uint4(0, 0, 0, 0);
                *reinterpret_cast<uint4 *>(sm.V + off) = make_uint4(0, 0, 0, 0);
            }
        }
        tc::cp_async_commit();
        tc::cp_async_wait<0>();
        tc::fence_async_smem();
        __syncthreads();

        // ---- S = Q K^T
        if (tid == 0) {
            tc::tc_fence_after();
            constexpr uint32_t idesc = tc::idesc_bf16(128, kW, 0, 0);
            const uint32_t xs = tc::smem_u32(sm.X);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                tc::mma_bf16(tS, tc::sw128_desc(xs + 64 * 128 + kk * 32), tc::sw128_desc(xs + kk * 32), idesc, kk > 0);
            tc::mma_commit(&sm.bar_s);
        }
        bool ok = tc::mbar_wait(&sm.bar_s, phase, &sm.abort, status);
        tc::tc_fence_after();

        // ---- softmax, one query row per thread
        const int i = warp * 32 + lane;                 // query row in tile = window row 64 + i
        const int qpos = sm.pos[64 + i];
        const float qinv = sm.inv[64 + i];
        float l = 1.f, row_lse = 0.f;
        if (warp < 2)
            softmax_row<0>(sm, tS + lane_off, ok, k == 0 ? 64 : 0, i, qpos, qinv, causal, tau, l, row_lse);
        else
            softmax_row<64>(sm, tS + lane_off, ok, 0, i, qpos, qinv, causal, tau, l, row_lse);
        tc::fence_async_smem();
        tc::tc_fence_before();
        __syncthreads();

        // ---- O = P V
        if (tid == 0 && ok) {
            tc::tc_fence_after();
            constexpr uint32_t idesc = tc::idesc_bf16(128, kDim, 0, 1);
            const uint32_t vs = tc::smem_u32(sm.V);
#pragma unroll
            for (int kk = 0; kk < 12; ++kk) {
                const uint32_t pa = tc::smem_u32(sm.P[kk >> 2]) + (kk & 3) * 32;
                tc::mma_bf16(tO, tc::sw128_desc(pa), tc::sw128_desc(vs + kk * 16 * 128), idesc, kk > 0);
            }
            tc::mma_commit(&sm.bar_o);
        }
        ok = ok && tc::mbar_wait(&sm.bar_o, phase, &sm.abort, status);
        tc::tc_fence_after();
        if (ok) {
            float o[kDim];
#pragma unroll
            for (int c = 0; c < 4; ++c) tc::tmem_ld16(tO + lane_off + (uint32_t)(c * 16), o + c * 16);
            tc::tmem_ld_wait();
            const float rl = 1.0f / l;
#pragma unroll
            for (int d = 0; d < kDim; ++d) o[d] *= rl;
            store_row(o_r + (seg * L + qpos) * kDim, o);
            lse[seg * L + qpos] = row_lse;
        }
        tc::tc_fence_before();
        if (__syncthreads_or(sm.abort != 0)) break;     // uniform exit after a timed-out wait
    }

    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace

bool attn_tc_supported(const Problem &p)
{
    return p.dtype == LSH_BF16 && p.d == kDim && p.m == 64 && p.L % kQ == 0;
}

cudaError_t launch_attn_fwd_tc(const Problem &p, const void *x, const void *v, const int32_t *perm,
                               const float *invnorm, __nv_bfloat16 *o_r, float *lse, uint32_t *status,
                               cudaStream_t st)
{
    const size_t smem = sizeof(FwdSmem) + 1024;
    cudaError_t e = cudaFuncSetAttribute(attn_fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long long n_tiles = p.S() * (p.L / kQ);
    const unsigned grid = (unsigned)std::min<long long>(n_tiles, 2LL * sms);
    attn_fwd_tc_kernel<<<grid, kThreads, smem, st>>>((const __nv_bfloat16 *)x, (const __nv_bfloat16 *)v, perm,
                                                     invnorm, o_r, lse, p.L, p.R, n_tiles, p.causal,
                                                     1.0f / sqrtf((float)p.d), status);
    return cudaGetLastError();
}

}  // namespace lsh
