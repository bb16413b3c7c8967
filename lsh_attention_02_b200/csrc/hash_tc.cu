// lsh_hash on the tensor cores: bucket = argmax over [x R_r ; -x R_r]
// ("LSH Attention", hash equation; angular LSH with Gaussian rotations).
//
// For every round the rotation product x R_r is a dense [rows x 64] x
// [64 x n_buckets/2] GEMM; it runs as tcgen05.mma (bf16 in, fp32 accumulate
// in tensor memory) and the argmax is the epilogue, so the projections are
// never written to memory.
//
// Persistent CTAs (one per SM) walk blocks of 256 rows (two M=128 tiles);
// each block runs every round.  Warp roles:
//   warps 0-15 epilogue: warp w reads TMEM lanes 32*(w%4).. of M-tile (w/4)%2,
//              one row per thread, and one half of every N-tile's columns
//              (w/8), keeping the running argmax; the halves of a row merge
//              through shared memory at the end of each round;
//   warp 16    producer: the next block's x rows by two TMA tile loads into
//              the idle one of two A buffers, and one bulk copy per (round,
//              N-tile) of the rotation tile, pre-transposed and pre-swizzled
//              in global memory, into a 4-stage shared-memory ring;
//   warp 17    MMA issuer: 4 K-steps per M-tile and N-tile into one of two
//              TMEM accumulator buffers (double buffering lets the epilogue
//              of tile t overlap the MMAs of tile t+1), with a completion
//              barrier per M-tile so the two epilogue halves start apart and
//              their ALU- and FMA-heavy passes overlap;
//   warps 18-19 key norms: 1/|x| of the block's rows from the same shared-memory
//              tile (the attention kernels read them), so x is read once.
//
// Epilogue per N-tile of NT columns held in registers: pass 1 takes the
// max and min with 3-input min/max; the larger of max and -min decides the
// side ([+xR] wins an exact tie, as its indices come first); pass 2 finds the
// lowest column equal to that extreme with exact 0/1 flags from saturating
// FMAs (see the epilogue).  Tiles merge in index order, so the
// result is the first maximum of [xR ; -xR], the oracle's tie rule.
#include "tc_common.cuh"

namespace lsh {

namespace {

constexpr int kRows = 256;          // rows per block
constexpr int kMaxNT = 128;         // widest N-tile
constexpr int kStages = 4;          // rotation-tile ring
constexpr int kEpiWarps = 16;         // 4 lane quadrants x 2 M-tiles x 2 column halves
constexpr int kNormWarp = kEpiWarps + 2;   // first of kNormWarps
constexpr int kNormWarps = 2;
constexpr int kThreads = (kNormWarp + kNormWarps) * 32;
constexpr int kTmemCols = 512;      // 2 buffers x 2 M-tiles x kMaxNT

struct HashSmem {
    uint8_t A[2][kRows * 128];              // x rows of two row blocks, K-major SW128 (64 KB)
    uint8_t B[kStages][kMaxNT * 128];       // rotation tiles (64 KB)
    uint64_t full[kStages], empty[kStages];
    uint64_t a_full[2], a_empty[2];
    uint64_t acc_full[2][2], acc_empty[2];  // [buffer][M-tile]
    float mbest[2][kRows];                  // upper column half's running best, by round parity
    int mbkt[2][kRows];                     // ... and its bucket
    uint64_t drain;                         // timeout path: the MMA issuer's last products
    uint32_t tmem_base;
    int abort;
};

// R [R, 64, half] (k-major per column) -> Rs [R, hp, 64] rows of 64 k, with the
// 16-byte chunks of row n stored at position (chunk ^ (n & 7)): the shared-memory
// image of a K-major 128-byte-swizzled B operand, so one bulk copy lands a tile.
// Columns n >= half (padding up to hp, a multiple of the N-tile) are zero: their
// projections are exactly 0, which never displaces the first maximum of a real
// column (max(xR) >= 0 or -min(xR) > 0 decides the side with a real column, and
// real columns come first in index order).
__global__ void rot_swizzle_kernel(const __nv_bfloat16 *__restrict__ R, __nv_bfloat16 *__restrict__ Rs, int half,
                                   int hp, int rounds)
{
    long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;   // over rounds * hp * 64
    long long total = (long long)rounds * hp * kDim;
    if (idx >= total) return;
    int k = (int)(idx % kDim);
    long long rn = idx / kDim;
    int n = (int)(rn % hp);
    int r = (int)(rn / hp);
    __nv_bfloat16 val = n < half ? R[((long long)r * kDim + k) * half + n] : __float2bfloat16_rn(0.f);
    const uint32_t off = tc::sw128_offset((uint32_t)n, (uint32_t)k);
    *reinterpret_cast<__nv_bfloat16 *>(reinterpret_cast<uint8_t *>(Rs) + (long long)r * hp * 128 + off) = val;
}

template <int NT>
__global__ void __launch_bounds__(kThreads, 1)
hash_tc_kernel(const __grid_constant__ CUtensorMap xmap, const __nv_bfloat16 *__restrict__ Rs,
               uint16_t *__restrict__ buckets, float *__restrict__ invnorm, long long rows_total, int L, int rounds,
               int half, int hp, uint32_t *__restrict__ status)
{
    extern __shared__ uint8_t smem_raw[];
    HashSmem &sm = *reinterpret_cast<HashSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_nt = hp / NT;                  // hp: half rounded up to a whole N-tile
    const int items = rounds * n_nt;
    const long long n_blocks = (rows_total + kRows - 1) / kRows;
    if (threadIdx.x == 0) LSH_PHASE(0, 3, 0, 0);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) { tc::mbar_init(&sm.full[s], 1); tc::mbar_init(&sm.empty[s], 1); }
        for (int b = 0; b < 2; ++b) {
            tc::mbar_init(&sm.a_full[b], 1);
            tc::mbar_init(&sm.a_empty[b], 1 + kNormWarps);   // the MMAs and the norm warps
            tc::mbar_init(&sm.acc_full[b][0], 1);
            tc::mbar_init(&sm.acc_full[b][1], 1);
            tc::mbar_init(&sm.acc_empty[b], kEpiWarps);
        }
        tc::mbar_init(&sm.drain, 1);
        sm.abort = 0;
        tc::fence_mbar_init();
    }
    if (warp == 0) tc::tmem_alloc(&sm.tmem_base, kTmemCols);
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    if (threadIdx.x == 0) LSH_PHASE(0, 3, 0, 1);

    if (warp == kEpiWarps) {
        // ---------------- producer
        if (lane == 0) {
            tc::prefetch_tmap(&xmap);
            auto load_a = [&](long long blk, int bi) -> bool {
                const int ab = bi & 1;
                if (bi >= 2 && !tc::mbar_wait(&sm.a_empty[ab], (uint32_t)((bi >> 1) - 1) & 1u, &sm.abort, status))
                    return false;
                tc::mbar_arrive_expect_tx(&sm.a_full[ab], kRows * 128);
                tc::tma_load_2d(sm.A[ab], &xmap, 0, (int)(blk * kRows), &sm.a_full[ab]);
                tc::tma_load_2d(sm.A[ab] + 128 * 128, &xmap, 0, (int)(blk * kRows + 128), &sm.a_full[ab]);
                return true;
            };
            bool ok = blockIdx.x >= n_blocks || load_a(blockIdx.x, 0);
            int it = 0, bi = 0, r_issued = 0, a_issued = blockIdx.x < n_blocks ? 1 : 0;
            for (long long blk = blockIdx.x; ok && blk < n_blocks; blk += gridDim.x, ++bi) {
                const int prefetch_at = min(kStages, items) - 1;
                for (int i = 0, r = 0, nt = 0; i < items; ++i, ++it) {
                    const int s = it % kStages;
                    const uint32_t ph = (uint32_t)(it / kStages) & 1u;
                    LSH_PHASE(0, 1, it, 0);
                    if (it >= kStages && !tc::mbar_wait(&sm.empty[s], ph ^ 1u, &sm.abort, status)) { ok = false; break; }
                    LSH_PHASE(0, 1, it, 1);
                    const __nv_bfloat16 *src = Rs + ((long long)r * hp + (long long)nt * NT) * kDim;
                    if (++nt == n_nt) {
                        nt = 0;
                        ++r;
                    }
                    tc::mbar_arrive_expect_tx(&sm.full[s], NT * 128);
                    tc::bulk_g2s(sm.B[s], src, NT * 128, &sm.full[s]);
                    ++r_issued;
                    // the next block's rows, once this block's MMAs have started
                    if (i == prefetch_at && blk + gridDim.x < n_blocks) {
                        if (!load_a(blk + gridDim.x, bi + 1)) { ok = false; break; }
                        ++a_issued;
                    }
                }
            }
            if (!ok) {
                // given up: before the CTA ends, let the copies this thread started land
                // (bounded waits on the barriers that count their bytes)
                int stop = 0;
                const long long budget = 1000000;
                for (int j = r_issued > kStages ? r_issued - kStages : 0; j < r_issued; ++j)
                    tc::mbar_wait(&sm.full[j % kStages], (uint32_t)(j / kStages) & 1u, &stop, status, budget);
                for (int b = a_issued > 2 ? a_issued - 2 : 0; b < a_issued; ++b)
                    tc::mbar_wait(&sm.a_full[b & 1], (uint32_t)(b >> 1) & 1u, &stop, status, budget);
            }
        }
    } else if (warp == kEpiWarps + 1) {
        // ---------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = tc::idesc_bf16(128, NT, 0, 0);
            int it = 0, bi = 0;
            bool ok = true;
            for (long long blk = blockIdx.x; ok && blk < n_blocks; blk += gridDim.x, ++bi) {
                const int xa = bi & 1;
                if (!tc::mbar_wait(&sm.a_full[xa], (uint32_t)(bi >> 1) & 1u, &sm.abort, status)) break;
                const uint64_t da = tc::sw128_desc(tc::smem_u32(sm.A[xa]));
                for (int i = 0; i < items; ++i, ++it) {
                    const int s = it % kStages;
                    const uint32_t ph = (uint32_t)(it / kStages) & 1u;
                    const int ab = it & 1;
                    const uint32_t aph = (uint32_t)(it >> 1) & 1u;
                    LSH_PHASE(0, 2, it, 0);
                    if (!tc::mbar_wait(&sm.full[s], ph, &sm.abort, status)) { ok = false; break; }
                    LSH_PHASE(0, 2, it, 1);
                    if (it >= 2 && !tc::mbar_wait(&sm.acc_empty[ab], aph ^ 1u, &sm.abort, status)) { ok = false; break; }
                    LSH_PHASE(0, 2, it, 2);
                    tc::tc_fence_after();
                    const uint64_t db = tc::sw128_desc(tc::smem_u32(sm.B[s]));
#pragma unroll
                    for (int mt = 0; mt < 2; ++mt) {
                        const uint32_t d = tmem + (uint32_t)(ab * 2 * kMaxNT + mt * kMaxNT);
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            tc::mma_bf16(d, tc::desc_add(da, mt * 128 * 128 + k * 32), tc::desc_add(db, k * 32),
                                         idesc, k > 0);
                        tc::mma_commit(&sm.acc_full[ab][mt]);
                    }
                    tc::mma_commit(&sm.empty[s]);
                    LSH_PHASE(0, 2, it, 3);
                }
                if (ok) tc::mma_commit(&sm.a_empty[xa]);
            }
            if (*reinterpret_cast<volatile int *>(&sm.abort)) tc::mma_drain(&sm.drain, status);
        }
    } else if (warp >= kNormWarp) {
        // ---------------- key norms of each block's rows (norm warp w, lane l: rows 32 w + l,
        // + 64, ...), sum of squares in element order as the norm pass does; then the A
        // buffer may be refilled
        int bi = 0;
        for (long long blk = blockIdx.x; blk < n_blocks; blk += gridDim.x, ++bi) {
            const int xa = bi & 1;
            if (!tc::mbar_wait(&sm.a_full[xa], (uint32_t)(bi >> 1) & 1u, &sm.abort, status)) break;
            if (invnorm) {
                const uint8_t *A = sm.A[xa];
#pragma unroll 1
                for (int r = (warp - kNormWarp) * 32 + lane; r < kRows; r += 32 * kNormWarps) {
                    float ssq = 0.f;
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch) {
                        const uint4 u = *reinterpret_cast<const uint4 *>(A + r * 128 + ((ch ^ (r & 7)) << 4));
                        const uint32_t wd[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float a = __uint_as_float(wd[e] << 16), b = __uint_as_float(wd[e] & 0xFFFF0000u);
                            ssq = fmaf(a, a, ssq);
                            ssq = fmaf(b, b, ssq);
                        }
                    }
                    const long long g = blk * kRows + r;
                    if (g < rows_total) invnorm[g] = ssq > 0.f ? 1.0f / sqrtf(ssq) : 0.f;
                }
            }
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&sm.a_empty[xa]);
        }
    } else {
        // ---------------- epilogue: warp w reads TMEM lanes 32*(w%4).. of M-tile
        // (w/4)%2, one row per thread, and columns [NH*hf, NH*hf + NH) of every
        // N-tile (hf = w/8), so four epilogue warps share each scheduler.  The two
        // column halves of a row merge through shared memory once per round.
        constexpr int NH = NT / 2;
        const int q = warp & 3, mt = (warp >> 2) & 1, hf = warp >> 3;
        const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(mt * kMaxNT + hf * NH);
        const int prow = mt * 128 + q * 32 + lane;               // row within the 256-row block
        int it = 0, rd = 0;                                      // rd: rounds finished (merge slot parity)
        bool ok = true;
        for (long long blk = blockIdx.x; ok && blk < n_blocks; blk += gridDim.x) {
            const long long g = blk * kRows + prow;
            float best = -INFINITY;
            int bucket = 0;
            int r = 0, nt = 0;                               // item i = (round r, N-tile nt), no division
            for (int i = 0; i < items; ++i, ++it) {
                const int ab = it & 1;
                const uint32_t aph = (uint32_t)(it >> 1) & 1u;
                if (threadIdx.x == 0) LSH_PHASE(0, 0, it, 0);
                if (!tc::mbar_wait(&sm.acc_full[ab][mt], aph, &sm.abort, status)) { ok = false; break; }
                if (threadIdx.x == 0) LSH_PHASE(0, 0, it, 1);
                tc::tc_fence_after();
                float v[NH];
                if constexpr (NH == 64) {
                    tc::tmem_ld64(lane_base + (uint32_t)(ab * 2 * kMaxNT), v);
                } else if constexpr (NH == 32) {
                    tc::tmem_ld32(lane_base + (uint32_t)(ab * 2 * kMaxNT), v);
                } else {
#pragma unroll
                    for (int c = 0; c < NH / 16; ++c)
                        tc::tmem_ld16(lane_base + (uint32_t)(ab * 2 * kMaxNT + c * 16), v + c * 16);
                }
                tc::tmem_ld_wait();
                tc::tc_fence_before();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&sm.acc_empty[ab]);
                if (threadIdx.x == 0) LSH_PHASE(0, 0, it, 2);

                // pass 1: extremes of the half tile, four independent chains per extreme
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
                if (threadIdx.x == 0) LSH_PHASE(0, 0, it, 3);
                // pass 2: lowest column holding the extreme.  U = |extreme| bounds every
                // |v| of the half tile; with B = 2^(24 - e(U)), (U - side * v_j) * B is
                // exactly 0 where v_j is the extreme and at least 1 elsewhere (the closest
                // float below U is 2^(e(U) - 24) away), so a saturating FMA gives a 0/1
                // flag without a compare.  Sixteen flags per chain are summed as the bits
                // of an integer kept in the mantissa of 2^23 + sum (exact), and the first
                // clear bit is the column.  This runs on the FMA pipe while pass 1 uses
                // the ALU pipe.  Extremes below 2^-103 (B would not be finite) take the
                // compare-and-select form.
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
                        for (int c = 0; c < NC; ++c)
                            acc[c] = fmaf(tc::fma_sat(v[c * 16 + k], nsB, UB), (float)(1 << k), acc[c]);
                    js = NH;
#pragma unroll
                    for (int c = NC - 1; c >= 0; --c) {
                        const uint32_t eq = ~__float_as_uint(acc[c]) & 0xFFFFu;
                        js = eq ? c * 16 + __ffs((int)eq) - 1 : js;
                    }
                }
                const float tbest = pos ? mx : -mn;
                const int tb = (pos ? 0 : half) + nt * NT + hf * NH + js;
                if (tbest > best || (tbest == best && tb < bucket)) { best = tbest; bucket = tb; }
                if (threadIdx.x == 0) LSH_PHASE(0, 0, it, 4);
                if (nt == n_nt - 1) {
                    // the upper column half hands its (best, bucket) to the lower one, which
                    // keeps the larger value (the lower bucket on a tie) and writes the id;
                    // both warps of a pair wait on the same barriers, so both get here
                    const int slot = rd & 1;
                    if (hf == 1) {
                        sm.mbest[slot][prow] = best;
                        sm.mbkt[slot][prow] = bucket;
                    }
                    tc::named_bar_sync(1 + (warp & 7), 64);
                    if (hf == 0) {
                        const float ob = sm.mbest[slot][prow];
                        const int obk = sm.mbkt[slot][prow];
                        if (ob > best || (ob == best && obk < bucket)) { best = ob; bucket = obk; }
                        if (g < rows_total) {
                            const long long bh = g / L;
                            const int pos_i = (int)(g % L);
                            buckets[(bh * rounds + r) * L + pos_i] = (uint16_t)bucket;
                        }
                    }
                    ++rd;
                    best = -INFINITY;
                    bucket = 0;
                }
                if (++nt == n_nt) {
                    nt = 0;
                    ++r;
                }
            }
        }
    }

    tc::tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0) LSH_PHASE(0, 3, 0, 2);
    if (warp == 0) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, kTmemCols);
    }
}

template <int NT>
cudaError_t launch_nt(const Problem &p, const void *x, const __nv_bfloat16 *Rs, int hp, uint16_t *buckets,
                      float *invnorm, uint32_t *status, cudaStream_t st)
{
    // one CTA per SM: each holds all 512 TMEM columns
    const size_t smem = sizeof(HashSmem) + 1024;
    cudaError_t e = cudaFuncSetAttribute(hash_tc_kernel<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const long long rows = p.tokens();
    CUtensorMap xmap;
    if (!tc::make_row_tmap(&xmap, x, rows, 128)) return cudaErrorInvalidValue;
    int dev = 0, sms = 148;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    const long long blocks = (rows + kRows - 1) / kRows;
    const unsigned grid = (unsigned)std::min<long long>(blocks, sms);
    hash_tc_kernel<NT><<<grid, kThreads, smem, st>>>(xmap, Rs, buckets, invnorm, rows, p.L, p.R, p.nb / 2, hp,
                                                     status);
    return cudaGetLastError();
}

// N-tile width: the widest of 128, 96, 64 that divides n_buckets/2, else 32
// with the last tile padded by zero rotation columns.
int pick_nt(int half)
{
    if (half % 128 == 0) return 128;
    if (half % 96 == 0) return 96;
    if (half % 64 == 0) return 64;
    return 32;
}
int padded_half(int half)
{
    const int nt = pick_nt(half);
    return (half + nt - 1) / nt * nt;
}

}  // namespace

// Rows are addressed by 32-bit TMA coordinates in boxes of 128 rows.
bool hash_tc_supported(const Problem &p)
{
    return p.dtype == LSH_BF16 && p.d == kDim && p.tokens() >= 128 && p.tokens() < (1LL << 31) - kRows;
}

size_t hash_tc_scratch_bytes(const Problem &p)
{
    return (size_t)p.R * padded_half(p.nb / 2) * kDim * sizeof(__nv_bfloat16);
}

cudaError_t launch_hash_tc(const Problem &p, const void *x, const void *R, uint16_t *buckets, void *scratch,
                           float *invnorm, uint32_t *status, cudaStream_t st)
{
    const int half = p.nb / 2, hp = padded_half(half);
    __nv_bfloat16 *Rs = (__nv_bfloat16 *)scratch;
    const long long total = (long long)p.R * hp * kDim;
    rot_swizzle_kernel<<<(unsigned)((total + 255) / 256), 256, 0, st>>>((const __nv_bfloat16 *)R, Rs, half, hp,
                                                                        p.R);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    switch (pick_nt(half)) {
    case 128: return launch_nt<128>(p, x, Rs, hp, buckets, invnorm, status, st);
    case 96: return launch_nt<96>(p, x, Rs, hp, buckets, invnorm, status, st);
    case 64: return launch_nt<64>(p, x, Rs, hp, buckets, invnorm, status, st);
    default: return launch_nt<32>(p, x, Rs, hp, buckets, invnorm, status, st);
    }
}

}  // namespace lsh

LSH_PHASE_EXPORT(hash)
