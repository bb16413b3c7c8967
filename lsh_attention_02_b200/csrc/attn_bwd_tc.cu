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
//   elementwise: P^T, E^T = tau inv_j dS^T  -> bf16 in shared memory
//   dV   = P^T dYq   (M=128, N=64, K=192)      G    = E^T Xq    (M=128, N=64, K=192)
//   dQ   = E Xk      (two M=128 halves over the 192 queries, K=128)
// Gradients of every round are added into fp32 accumulators with vector
// reductions (red.global.add.v4.f32); their summation order is not fixed.
//
// A query attends to itself only when no other candidate is left (causal:
// its position is the smallest in its window); that flag is recomputed here
// from the window minima of positions.
#include "tc_common.cuh"

namespace lsh {

namespace {

constexpr int kK = 128;             // key slots per tile
constexpr int kQ = 192;             // query slots per tile
constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;

struct BwdSmem {
    uint8_t X[kQ * 128];            // x rows of the query slots (first 128 = key slots)   24 KB
    uint8_t V[kK * 128];            // v rows of the key slots                              16 KB
    uint8_t G[kQ * 128];            // dY rows of the query slots                           24 KB
    uint8_t PT[3][kK * 128];        // P^T, 3 blocks of 64 queries                          48 KB
    uint8_t ET[3][kK * 128];        // tau inv_j dS^T                                      48 KB
    alignas(16) int32_t pos[256];   // positions of slots [128k - 64, 128k + 192)
    alignas(16) float qlse[kQ];     // LSE_i * log2(e) (+inf for a missing query)
    alignas(16) float qdelta[kQ];
    alignas(16) int32_t qself[kQ];  // 1 if the query attends to itself alone
    alignas(16) float kinv[kK];
    int32_t cmin[4];
    uint64_t bar1, bar2;
    uint32_t tmem_base;
    int abort;
};

__device__ __forceinline__ void red_add_v4(float *addr, float a, float b, float c, float d)
{
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
                 : "memory");
}

// Adds a 64-float row to dst with 16 vector reductions.
__device__ __forceinline__ void red_row(float *dst, const float *r)
{
#pragma unroll
    for (int c = 0; c < 16; ++c) red_add_v4(dst + 4 * c, r[4 * c], r[4 * c + 1], r[4 * c + 2], r[4 * c + 3]);
}

// bf16 row `row` of a K-major SW128 tile -> 64 floats.
__device__ __forceinline__ void smem_row(const uint8_t *tile, int row, float *out)
{
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) {
        const uint4 u = *reinterpret_cast<const uint4 *>(tile + row * 128 + ((ch ^ (row & 7)) << 4));
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            out[ch * 8 + 2 * e] = __uint_as_float(w[e] << 16);
            out[ch * 8 + 2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
        }
    }
}

// Elementwise step for one key row over 64 query columns [C0, C0 + 64) of the
// tile, C0 a multiple of 64: P^T and E^T chunks written to shared memory.
template <int C0>
__device__ __forceinline__ void key_row_block(BwdSmem &sm, uint32_t tS, uint32_t tD, int kr, int kpos, float kinv,
                                              int causal, float tau)
{
    float s[64], dp[64];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        tc::tmem_ld16(tS + (uint32_t)(C0 + c * 16), s + c * 16);
        tc::tmem_ld16(tD + (uint32_t)(C0 + c * 16), dp + c * 16);
    }
    tc::tmem_ld_wait();
    const float sc = tau * kinv * kLog2e;      // score * log2(e) = raw * sc
    const float ec = tau * kinv;
    constexpr int blk = C0 / 64;
#pragma unroll
    for (int j8 = 0; j8 < 64; j8 += 8) {
        uint32_t pw[4], ew[4];
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
            float pv[2], ev[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int j = j8 + e + u;
                const int q = C0 + j;                        // query column in the tile
                const int qp = sm.pos[64 + q];
                const bool valid = (causal ? (kpos < qp) : (kpos != qp)) || (kpos == qp && sm.qself[q]);
                const float p = valid ? exp2f(s[j] * sc - sm.qlse[q]) : 0.f;
                pv[u] = p;
                ev[u] = ec * p * (dp[j] - sm.qdelta[q]);
            }
            pw[e / 2] = pack_bf16x2(pv[0], pv[1]);
            ew[e / 2] = pack_bf16x2(ev[0], ev[1]);
        }
        const int ch = j8 / 8;
        const uint32_t off = (uint32_t)kr * 128u + (uint32_t)((ch ^ (kr & 7)) << 4);
        *reinterpret_cast<uint4 *>(sm.PT[blk] + off) = make_uint4(pw[0], pw[1], pw[2], pw[3]);
        *reinterpret_cast<uint4 *>(sm.ET[blk] + off) = make_uint4(ew[0], ew[1], ew[2], ew[3]);
    }
}

__device__ __forceinline__ void zero_block(BwdSmem &sm, int blk, int kr)
{
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) {
        const uint32_t off = (uint32_t)kr * 128u + (uint32_t)((ch ^ (kr & 7)) << 4);
        *reinterpret_cast<uint4 *>(sm.PT[blk] + off) = make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4 *>(sm.ET[blk] + off) = make_uint4(0, 0, 0, 0);
    }
}

__global__ void __launch_bounds__(kThreads, 1)
attn_bwd_tc_kernel(const __nv_bfloat16 *__restrict__ x, const __nv_bfloat16 *__restrict__ v,
                   const __nv_bfloat16 *__restrict__ dout, const int32_t *__restrict__ perm,
                   const float *__restrict__ invnorm, const float *__restrict__ lse_all,
                   const float *__restrict__ delta, float *__restrict__ dx_acc, float *__restrict__ dv_acc, int L,
                   int R, long long n_tiles, int causal, float tau, uint32_t *__restrict__ status)
{
    extern __shared__ uint8_t smem_raw[];
    BwdSmem &sm = *reinterpret_cast<BwdSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, half = warp >> 2;
    const int n_k = L / kK;

    if (tid == 0) {
        tc::mbar_init(&sm.bar1, 1);
        tc::mbar_init(&sm.bar2, 1);
        sm.abort = 0;
        tc::fence_mbar_init();
    }
    if (warp == 0) tc::tmem_alloc(&sm.tmem_base, kTmemCols);
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    // TMEM columns: S^T [0,192), dP^T [256,448); after the elementwise step
    // dV [0,64), G [64,128), dQ rows 0-127 [128,192), dQ rows 64-191 [192,256).
    const uint32_t tS = tmem, tD = tmem + 256;
    const uint32_t tDV = tmem, tG = tmem + 64, tQa = tmem + 128, tQb = tmem + 192;
    uint32_t phase = 0;

    for (long long tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, phase ^= 1u) {
        const int r = (int)(tile % R);
        const long long bk = tile / R;
        const int k = (int)(bk % n_k);
        const long long bh = bk / n_k;
        const long long seg = bh * R + r;
        const int32_t *P = perm + seg * L;
        const long long rowbase = bh * L;
        const int slot0 = k * kK - 64;           // slot of pos[0]

        // ---- positions of slots [128k - 64, 128k + 192); -1 where missing
        for (int e = tid; e < 256; e += kThreads) {
            const int s = slot0 + e;
            sm.pos[e] = (s >= 0 && s < L) ? P[s] : -1;
        }
        __syncthreads();
        if (warp == 0) {
            // minimum position of each of the four chunks (2k-1 .. 2k+2)
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                int mn = INT_MAX;
                for (int e = lane; e < 64; e += 32) {
                    const int p = sm.pos[c * 64 + e];
                    if (p >= 0) mn = min(mn, p);
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, o));
                if (lane == 0) sm.cmin[c] = mn;
            }
        }
        __syncthreads();
        for (int q = tid; q < kQ; q += kThreads) {
            const int p = sm.pos[64 + q];
            const int qa = q >> 6;                   // query chunk 2k + qa, window = ext chunks qa, qa + 1
            const int wmin = min(sm.cmin[qa], sm.cmin[qa + 1]);
            sm.qself[q] = (p >= 0 && causal && p == wmin) ? 1 : 0;
            sm.qlse[q] = p >= 0 ? lse_all[rowbase + p] * kLog2e : INFINITY;
            sm.qdelta[q] = p >= 0 ? delta[rowbase + p] : 0.f;
            if (q < kK) sm.kinv[q] = p >= 0 ? invnorm[rowbase + p] : 0.f;
        }
        // ---- gather x (192 query slots), v (128 key slots), dY (192 query slots)
        for (int c = tid; c < kQ * 8; c += kThreads) {
            const int w = c >> 3, ch = c & 7;
            const uint32_t off = (uint32_t)w * 128u + (uint32_t)((ch ^ (w & 7)) << 4);
            const int p = sm.pos[64 + w];
            if (p >= 0) {
                tc::cp_async16(sm.X + off, x + (rowbase + p) * kDim + ch * 8);
                tc::cp_async16(sm.G + off, dout + (rowbase + p) * kDim + ch * 8);
                if (w < kK) tc::cp_async16(sm.V + off, v + (rowbase + p) * kDim + ch * 8);
            } else {
                *reinterpret_cast<uint4 *>(sm.X + off) = make_uint4(0, 0, 0, 0);
                *reinterpret_cast<uint4 *>(sm.G + off) = make_uint4(0, 0, 0, 0);
                if (w < kK) *reinterpret_cast<uint4 *>(sm.V + off) = make_uint4(0, 0, 0, 0);
            }
        }
        tc::cp_async_commit();
        tc::cp_async_wait<0>();
        tc::fence_async_smem();
        __syncthreads();

        // ---- S^T = Xk Xq^T, dP^T = Vk dYq^T
        if (tid == 0) {
            tc::tc_fence_after();
            constexpr uint32_t idesc = tc::idesc_bf16(128, kQ, 0, 0);
            const uint32_t xs = tc::smem_u32(sm.X), vs = tc::smem_u32(sm.V), gs = tc::smem_u32(sm.G);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                tc::mma_bf16(tS, tc::sw128_desc(xs + kk * 32), tc::sw128_desc(xs + kk * 32), idesc, kk > 0);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                tc::mma_bf16(tD, tc::sw128_desc(vs + kk * 32), tc::sw128_desc(gs + kk * 32), idesc, kk > 0);
            tc::mma_commit(&sm.bar1);
        }
        bool ok = tc::mbar_wait(&sm.bar1, phase, &sm.abort, status);
        tc::tc_fence_after();

        // ---- elementwise: thread = key row kr, 64 query columns per warp half
        const int kr = quad * 32 + lane;
        const int kpos = sm.pos[64 + kr];
        const float kinv = sm.kinv[kr];
        if (ok) {
            const uint32_t tSl = tS + lane_off, tDl = tD + lane_off;
            if (quad < 2) {                          // keys of chunk 2k: queries of chunks 2k, 2k+1
                if (half == 0) { key_row_block<0>(sm, tSl, tDl, kr, kpos, kinv, causal, tau); zero_block(sm, 2, kr); }
                else key_row_block<64>(sm, tSl, tDl, kr, kpos, kinv, causal, tau);
            } else {                                 // keys of chunk 2k+1: queries of chunks 2k+1, 2k+2
                if (half == 0) { key_row_block<64>(sm, tSl, tDl, kr, kpos, kinv, causal, tau); zero_block(sm, 0, kr); }
                else key_row_block<128>(sm, tSl, tDl, kr, kpos, kinv, causal, tau);
            }
        }
        tc::fence_async_smem();
        tc::tc_fence_before();
        __syncthreads();

        // ---- dV = P^T dYq, G = E^T Xq, dQ = E Xk (two halves)
        if (tid == 0 && ok) {
            tc::tc_fence_after();
            constexpr uint32_t id_kv = tc::idesc_bf16(128, kDim, 0, 1);   // A K-major, B MN-major
            constexpr uint32_t id_q = tc::idesc_bf16(128, kDim, 1, 1);    // A MN-major, B MN-major
            const uint32_t xs = tc::smem_u32(sm.X), gs = tc::smem_u32(sm.G);
#pragma unroll
            for (int kk = 0; kk < 12; ++kk) {
                const uint32_t pa = tc::smem_u32(sm.PT[kk >> 2]) + (kk & 3) * 32;
                const uint32_t ea = tc::smem_u32(sm.ET[kk >> 2]) + (kk & 3) * 32;
                tc::mma_bf16(tDV, tc::sw128_desc(pa), tc::sw128_desc(gs + kk * 2048), id_kv, kk > 0);
                tc::mma_bf16(tG, tc::sw128_desc(ea), tc::sw128_desc(xs + kk * 2048), id_kv, kk > 0);
            }
            // E = (E^T)^T read MN-major: 64-query blocks 16 KB apart (leading byte offset)
            const uint32_t e0 = tc::smem_u32(sm.ET[0]), e1 = tc::smem_u32(sm.ET[1]);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                tc::mma_bf16(tQa, tc::sw128_desc(e0 + kk * 2048, kK * 128), tc::sw128_desc(xs + kk * 2048), id_q, kk > 0);
                tc::mma_bf16(tQb, tc::sw128_desc(e1 + kk * 2048, kK * 128), tc::sw128_desc(xs + kk * 2048), id_q, kk > 0);
            }
            tc::mma_commit(&sm.bar2);
        }
        ok = ok && tc::mbar_wait(&sm.bar2, phase, &sm.abort, status);
        tc::tc_fence_after();

        // ---- epilogue: reductions into the fp32 accumulators
        if (ok) {
            float a[kDim];
            if (half == 0) {
                // dV row of key kr
#pragma unroll
                for (int c = 0; c < 4; ++c) tc::tmem_ld16(tDV + lane_off + (uint32_t)(c * 16), a + c * 16);
                tc::tmem_ld_wait();
                if (kpos >= 0) red_row(dv_acc + (rowbase + kpos) * kDim, a);
            } else {
                // key-role dx: g - inv^2 (g . x) x
#pragma unroll
                for (int c = 0; c < 4; ++c) tc::tmem_ld16(tG + lane_off + (uint32_t)(c * 16), a + c * 16);
                tc::tmem_ld_wait();
                float xr[kDim];
                smem_row(sm.X, kr, xr);
                float gx = 0.f;
#pragma unroll
                for (int d = 0; d < kDim; ++d) gx = fmaf(a[d], xr[d], gx);
                const float cf = kinv * kinv * gx;
#pragma unroll
                for (int d = 0; d < kDim; ++d) a[d] = fmaf(-cf, xr[d], a[d]);
                if (kpos >= 0) red_row(dx_acc + (rowbase + kpos) * kDim, a);
            }
            // query-role dx: rows 0-127 from the first half, rows 128-191 from lanes 64-127 of the second
            if (half == 0) {
#pragma unroll
                for (int c = 0; c < 4; ++c) tc::tmem_ld16(tQa + lane_off + (uint32_t)(c * 16), a + c * 16);
                tc::tmem_ld_wait();
                const int qp = sm.pos[64 + kr];
                if (qp >= 0) red_row(dx_acc + (rowbase + qp) * kDim, a);
            } else if (quad >= 2) {
#pragma unroll
                for (int c = 0; c < 4; ++c) tc::tmem_ld16(tQb + lane_off + (uint32_t)(c * 16), a + c * 16);
                tc::tmem_ld_wait();
                const int qp = sm.pos[64 + 64 + kr];          // query row 64 + kr, kr in [64, 128)
                if (qp >= 0) red_row(dx_acc + (rowbase + qp) * kDim, a);
            }
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

cudaError_t launch_attn_bwd_tc(const Problem &p, const void *x, const void *v, const void *dout, const int32_t *perm,
                               const float *invnorm, const float *lse_all, const float *delta, float *dx_acc,
                               float *dv_acc, uint32_t *status, cudaStream_t st)
{
    const size_t smem = sizeof(BwdSmem) + 1024;
    cudaError_t e = cudaFuncSetAttribute(attn_bwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long long n_tiles = p.S() * (p.L / kK);
    const unsigned grid = (unsigned)std::min<long long>(n_tiles, (long long)sms);
    attn_bwd_tc_kernel<<<grid, kThreads, smem, st>>>((const __nv_bfloat16 *)x, (const __nv_bfloat16 *)v,
                                                     (const __nv_bfloat16 *)dout, perm, invnorm, lse_all, delta,
                                                     dx_acc, dv_acc, p.L, p.R, n_tiles, p.causal,
                                                     1.0f / sqrtf((float)p.d), status);
    return cudaGetLastError();
}

}  // namespace lsh
