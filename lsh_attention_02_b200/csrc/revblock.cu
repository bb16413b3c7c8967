// Token-wise kernels of the reversible residual block ("Reversible Residual
// Layers" of the paper note "Reformer": y1 = x1 + F(x2), y2 = x2 + G(y1), and
// the inverse x2 = y2 - G(y1), x1 = y1 - F(x2)).  F is LSH attention (the
// attention kernels); G is a token-wise layer G(u) = tanh(u W + b) with
// W [64, 64] and b [64] in fp32.  The residual streams are fp32, so that the
// inverse recovers x2 to fp32 rounding and hashing it again gives the same
// buckets.
#include "common.cuh"

namespace lsh {

namespace {

constexpr int kTok = 32;                 // tokens per CTA (one warp-row of outputs each)

// g = tanh(u W + b) for kTok tokens per CTA: thread (t, c) computes output
// column c of token t; W and b stay in shared memory.  Sequential fp32 fma over
// the 64 inputs.  With `res` given, out = res + g (a residual add) and g is
// also written to g_out when that is non-null.
__global__ void __launch_bounds__(256) g_forward_kernel(const float *__restrict__ u, const float *__restrict__ W,
                                                        const float *__restrict__ b, const float *__restrict__ res,
                                                        float *__restrict__ out, float *__restrict__ g_out,
                                                        long long tokens)
{
    __shared__ float sW[kDim * kDim];
    __shared__ float sb[kDim];
    __shared__ float su[kTok][kDim + 1];
    for (int i = threadIdx.x; i < kDim * kDim; i += blockDim.x) sW[i] = W[i];
    if (threadIdx.x < kDim) sb[threadIdx.x] = b[threadIdx.x];
    const long long t0 = (long long)blockIdx.x * kTok;
    for (int i = threadIdx.x; i < kTok * kDim; i += blockDim.x) {
        const long long t = t0 + i / kDim;
        su[i / kDim][i % kDim] = t < tokens ? u[t * kDim + i % kDim] : 0.f;
    }
    __syncthreads();
    const int c = threadIdx.x & 63;
    for (int tl = threadIdx.x >> 6; tl < kTok; tl += blockDim.x >> 6) {
        const long long t = t0 + tl;
        if (t >= tokens) break;
        float a = sb[c];
#pragma unroll 16
        for (int k = 0; k < kDim; ++k) a = fmaf(su[tl][k], sW[k * kDim + c], a);
        const float g = tanhf(a);
        if (g_out) g_out[t * kDim + c] = g;
        out[t * kDim + c] = res ? res[t * kDim + c] + g : g;
    }
}

// Backward of G through its saved output g: dpre = dy (1 - g^2),
// du = dpre W^T; out = base + du (base: the gradient already flowing into u).
__global__ void __launch_bounds__(256) g_backward_kernel(const float *__restrict__ g, const float *__restrict__ dy,
                                                         const float *__restrict__ W, const float *__restrict__ base,
                                                         float *__restrict__ out, long long tokens)
{
    __shared__ float sWt[kDim * (kDim + 1)];     // W transposed, padded rows: conflict-free both ways
    __shared__ float sd[kTok][kDim + 1];
    for (int i = threadIdx.x; i < kDim * kDim; i += blockDim.x) sWt[(i % kDim) * (kDim + 1) + i / kDim] = W[i];
    const long long t0 = (long long)blockIdx.x * kTok;
    for (int i = threadIdx.x; i < kTok * kDim; i += blockDim.x) {
        const long long t = t0 + i / kDim;
        float d = 0.f;
        if (t < tokens) {
            const float gv = g[t * kDim + i % kDim];
            d = dy[t * kDim + i % kDim] * (1.f - gv * gv);
        }
        sd[i / kDim][i % kDim] = d;
    }
    __syncthreads();
    const int k = threadIdx.x & 63;              // input column
    for (int tl = threadIdx.x >> 6; tl < kTok; tl += blockDim.x >> 6) {
        const long long t = t0 + tl;
        if (t >= tokens) break;
        float a = 0.f;
#pragma unroll 16
        for (int c = 0; c < kDim; ++c) a = fmaf(sd[tl][c], sWt[c * (kDim + 1) + k], a);
        out[t * kDim + k] = base[t * kDim + k] + a;
    }
}

// Elementwise pieces: out = a + s * to_f(b) over n floats (b in the attention
// dtype), and the cast of an fp32 stream to the attention dtype (nearest even).
template <typename T>
__global__ void axpy_kernel(const float *__restrict__ a, const T *__restrict__ b, float s, float *__restrict__ out,
                            long long n)
{
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) out[i] = a[i] + s * to_f(b[i]);
}
template <typename T>
__global__ void cast_kernel(const float *__restrict__ a, T *__restrict__ out, long long n)
{
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) out[i] = from_f<T>(a[i]);
}
// out = a + to_f(b) + to_f(c) (the two gradients of F's shared input plus the residual path)
template <typename T>
__global__ void sum3_kernel(const float *__restrict__ a, const T *__restrict__ b, const T *__restrict__ c,
                            float *__restrict__ out, long long n)
{
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) out[i] = a[i] + to_f(b[i]) + to_f(c[i]);
}

__global__ void sub_kernel(const float *__restrict__ a, const float *__restrict__ b, float *__restrict__ out,
                           long long n)
{
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) out[i] = a[i] - b[i];
}

unsigned blocks(long long n, int t) { return (unsigned)((n + t - 1) / t); }

}  // namespace

cudaError_t launch_g_forward(const Problem &p, const float *u, const float *W, const float *b, const float *res,
                             float *out, float *g_out, cudaStream_t st)
{
    const long long T = p.tokens();
    g_forward_kernel<<<blocks(T, kTok), 256, 0, st>>>(u, W, b, res, out, g_out, T);
    return cudaGetLastError();
}

cudaError_t launch_g_backward(const Problem &p, const float *g, const float *dy, const float *W, const float *base,
                              float *out, cudaStream_t st)
{
    const long long T = p.tokens();
    g_backward_kernel<<<blocks(T, kTok), 256, 0, st>>>(g, dy, W, base, out, T);
    return cudaGetLastError();
}

cudaError_t launch_axpy(const Problem &p, const float *a, const void *b, float s, float *out, cudaStream_t st)
{
    const long long n = p.tokens() * kDim;
    if (p.dtype == LSH_BF16)
        axpy_kernel<__nv_bfloat16><<<blocks(n, 256), 256, 0, st>>>(a, (const __nv_bfloat16 *)b, s, out, n);
    else
        axpy_kernel<float><<<blocks(n, 256), 256, 0, st>>>(a, (const float *)b, s, out, n);
    return cudaGetLastError();
}

cudaError_t launch_cast(const Problem &p, const float *a, void *out, cudaStream_t st)
{
    const long long n = p.tokens() * kDim;
    if (p.dtype == LSH_BF16)
        cast_kernel<__nv_bfloat16><<<blocks(n, 256), 256, 0, st>>>(a, (__nv_bfloat16 *)out, n);
    else
        cast_kernel<float><<<blocks(n, 256), 256, 0, st>>>(a, (float *)out, n);
    return cudaGetLastError();
}

cudaError_t launch_sum3(const Problem &p, const float *a, const void *b, const void *c, float *out, cudaStream_t st)
{
    const long long n = p.tokens() * kDim;
    if (p.dtype == LSH_BF16)
        sum3_kernel<__nv_bfloat16><<<blocks(n, 256), 256, 0, st>>>(a, (const __nv_bfloat16 *)b,
                                                                   (const __nv_bfloat16 *)c, out, n);
    else
        sum3_kernel<float><<<blocks(n, 256), 256, 0, st>>>(a, (const float *)b, (const float *)c, out, n);
    return cudaGetLastError();
}

cudaError_t launch_sub(const Problem &p, const float *a, const float *b, float *out, cudaStream_t st)
{
    const long long n = p.tokens() * kDim;
    sub_kernel<<<blocks(n, 256), 256, 0, st>>>(a, b, out, n);
    return cudaGetLastError();
}

}  // namespace lsh
