// gather_sorted + chunk_attn forward on the tensor cores, persistent over
// every (batch, head, round) segment: one CTA per SM walks the tiles
// blockIdx.x, blockIdx.x + gridDim.x, ... in (bh, k, r) order.  The tile, the
// softmax and the warp roles are described in attn_fwd_roles.cuh; positions
// come from the sort's permutation and the key norms from the per-token norms
// written by the hash (or a norm pass), both in global memory.
#include "attn_fwd_roles.cuh"

namespace lsh {

namespace {

using namespace fwd;

constexpr int kStages = 4;

struct FwdSmem {
    Ring<kStages> ring;
};

template <bool CAUSAL, int FL>
__global__ void __launch_bounds__(kThreads, 1)
attn_fwd_tc_kernel(const __nv_bfloat16 *__restrict__ x, const __nv_bfloat16 *__restrict__ v,
                   const int32_t *__restrict__ perm, const uint16_t *__restrict__ bkt,
                   const float *__restrict__ xinv, __nv_bfloat16 *__restrict__ o_r, float *__restrict__ lse,
                   int L, int R, long long n_tiles, float tau, uint32_t prev_mask, uint32_t *__restrict__ status)
{
    extern __shared__ uint8_t smem_raw[];
    FwdSmem &smem = *reinterpret_cast<FwdSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Ring<kStages> &sm = smem.ring;
    const int warp = threadIdx.x >> 5;
    const int n_k = (L + kQ - 1) / kQ;          // the last tile may hold one chunk only
    const int n_mine = blockIdx.x < n_tiles ? (int)((n_tiles - 1 - blockIdx.x) / gridDim.x + 1) : 0;

    if (threadIdx.x == 0) ring_init(sm);
    if (warp == 0) tc::tmem_alloc(&sm.tmem_base, kTmemCols);
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    if (warp >= kSoftmaxWarps && warp < kMmaWarp) {
        const GridTiles src{perm, bkt, xinv, L, R, n_k};
        producer_role<CAUSAL, FL>(sm, src, n_mine, x, v, tau * kLog2e, status);
    } else if (warp == kMmaWarp) {
        mma_role(sm, n_mine, tmem, status);
    } else {
        softmax_role<CAUSAL, FL>(sm, n_mine, tmem, o_r, lse, L, tau, prev_mask, status);
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
    return p.dtype == LSH_BF16 && p.d == kDim && p.m == 64 && p.L % 64 == 0 && p.tokens() < (1LL << 31);
}

template <bool CAUSAL, int FL>
static cudaError_t launch_fwd(const Problem &p, const void *x, const void *v, const int32_t *perm,
                              const uint16_t *bkt, const float *xinv, __nv_bfloat16 *o_r, float *lse,
                              uint32_t *status, cudaStream_t st)
{
    const size_t smem = sizeof(FwdSmem) + 1024;
    auto kern = attn_fwd_tc_kernel<CAUSAL, FL>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    const long long n_tiles = p.S() * ((p.L + kQ - 1) / kQ);
    const unsigned grid = (unsigned)std::min<long long>(n_tiles, (long long)sms);
    kern<<<grid, kThreads, smem, st>>>((const __nv_bfloat16 *)x, (const __nv_bfloat16 *)v, perm, bkt, xinv, o_r,
                                       lse, p.L, p.R, n_tiles, 1.0f / sqrtf((float)p.d), (uint32_t)p.prev_mask, status);
    return cudaGetLastError();
}

cudaError_t launch_attn_fwd_tc(const Problem &p, const void *x, const void *v, const int32_t *perm,
                               const uint16_t *bkt, const float *xinv, __nv_bfloat16 *o_r, float *lse,
                               uint32_t *status, cudaStream_t st)
{
    const int fl = p.flags & (kMask | kPen);
    if (p.causal) {
        switch (fl) {
        case 0: return launch_fwd<true, 0>(p, x, v, perm, bkt, xinv, o_r, lse, status, st);
        case kMask: return launch_fwd<true, kMask>(p, x, v, perm, bkt, xinv, o_r, lse, status, st);
        case kPen: return launch_fwd<true, kPen>(p, x, v, perm, bkt, xinv, o_r, lse, status, st);
        default: return launch_fwd<true, kMask | kPen>(p, x, v, perm, bkt, xinv, o_r, lse, status, st);
        }
    }
    switch (fl) {
    case 0: return launch_fwd<false, 0>(p, x, v, perm, bkt, xinv, o_r, lse, status, st);
    case kMask: return launch_fwd<false, kMask>(p, x, v, perm, bkt, xinv, o_r, lse, status, st);
    case kPen: return launch_fwd<false, kPen>(p, x, v, perm, bkt, xinv, o_r, lse, status, st);
    default: return launch_fwd<false, kMask | kPen>(p, x, v, perm, bkt, xinv, o_r, lse, status, st);
    }
}

}  // namespace lsh

LSH_PHASE_EXPORT(fwd)
