/* A plain C caller of the library: rotations from a seed, inputs from a small
 * generator, one forward through the C ABI on the GPU, and the result checked
 * against the CPU oracle run with the GPU's permutation.  Exit status 0 and
 * the line "ok" on success.  With --compile-check it only links and returns. */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime_api.h>

#include "lsh_attn.h"

/* test infrastructure: the oracle's forward for one (batch, head) */
int oracle_fwd_head_perm(const double *x, const double *v, long L, int d, const int32_t *perm, int n_hashes, int m,
                         int causal, double *y, double *lse);

static uint64_t g_state = 0x9E3779B97F4A7C15ull;
static float next_normal(void)
{
    /* splitmix64 uniforms, Box-Muller; any fixed sequence will do here */
    double u[2];
    for (int k = 0; k < 2; ++k) {
        uint64_t z = (g_state += 0x9E3779B97F4A7C15ull);
        z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
        z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
        z ^= z >> 31;
        u[k] = ((double)(z >> 11) + 0.5) / 9007199254740992.0;
    }
    return (float)(sqrt(-2.0 * log(u[0])) * cos(6.283185307179586 * u[1]));
}

#define CHECK(call)                                                          \
    do {                                                                     \
        int rc_ = (int)(call);                                               \
        if (rc_ != 0) {                                                      \
            fprintf(stderr, "%s failed: %d (%s)\n", #call, rc_, lsh_attn_last_error()); \
            return 1;                                                        \
        }                                                                    \
    } while (0)

int main(int argc, char **argv)
{
    if (argc > 1 && strcmp(argv[1], "--compile-check") == 0) return lsh_attn_abi_version() == LSH_ATTN_ABI_VERSION ? 0 : 1;
    const int B = 1, H = 2, L = 512, d = 64, nb = 16, nh = 2, m = 64, causal = 1;
    lsh_attn_desc desc = {B, H, L, d, nb, nh, m, causal, LSH_F32, LSH_IMPL_AUTO};
    const size_t n = (size_t)B * H * L * d, nr = (size_t)nh * d * (nb / 2), ns = (size_t)B * H * nh * L;
    float *x = malloc(n * 4), *v = malloc(n * 4), *R = malloc(nr * 4), *out = malloc(n * 4), *lse = malloc(ns * 4);
    int32_t *perm = malloc(ns * 4);
    if (!x || !v || !R || !out || !lse || !perm) return 1;
    for (size_t i = 0; i < n; ++i) x[i] = next_normal();
    for (size_t i = 0; i < n; ++i) v[i] = next_normal();
    CHECK(lsh_attn_make_rotations(42, &desc, R));

    void *dx, *dv, *dR, *dout, *dws;
    float *dlse;
    int32_t *dperm;
    const size_t ws = lsh_attn_workspace_size(&desc, 0);
    if (ws == 0) return 1;
    CHECK(cudaMalloc(&dx, n * 4));
    CHECK(cudaMalloc(&dv, n * 4));
    CHECK(cudaMalloc(&dR, nr * 4));
    CHECK(cudaMalloc(&dout, n * 4));
    CHECK(cudaMalloc((void **)&dlse, ns * 4));
    CHECK(cudaMalloc((void **)&dperm, ns * 4));
    CHECK(cudaMalloc(&dws, ws));
    CHECK(cudaMemcpy(dx, x, n * 4, cudaMemcpyHostToDevice));
    CHECK(cudaMemcpy(dv, v, n * 4, cudaMemcpyHostToDevice));
    CHECK(cudaMemcpy(dR, R, nr * 4, cudaMemcpyHostToDevice));
    CHECK(lsh_attn_fwd(&desc, dx, dv, dR, dout, dlse, dperm, dws, ws, NULL));
    CHECK(lsh_attn_poll(dws, NULL));
    CHECK(cudaMemcpy(out, dout, n * 4, cudaMemcpyDeviceToHost));
    CHECK(cudaMemcpy(lse, dlse, ns * 4, cudaMemcpyDeviceToHost));
    CHECK(cudaMemcpy(perm, dperm, ns * 4, cudaMemcpyDeviceToHost));

    /* oracle with the GPU's permutation, per (batch, head) */
    double *xd = malloc((size_t)L * d * 8), *vd = malloc((size_t)L * d * 8), *yd = malloc((size_t)L * d * 8),
           *ld = malloc((size_t)nh * L * 8);
    if (!xd || !vd || !yd || !ld) return 1;
    double err = 0.0, lerr = 0.0;
    for (int bh = 0; bh < B * H; ++bh) {
        for (size_t i = 0; i < (size_t)L * d; ++i) {
            xd[i] = x[(size_t)bh * L * d + i];
            vd[i] = v[(size_t)bh * L * d + i];
        }
        CHECK(oracle_fwd_head_perm(xd, vd, L, d, perm + (size_t)bh * nh * L, nh, m, causal, yd, ld));
        for (size_t i = 0; i < (size_t)L * d; ++i) err = fmax(err, fabs(yd[i] - out[(size_t)bh * L * d + i]));
        for (size_t i = 0; i < (size_t)nh * L; ++i) lerr = fmax(lerr, fabs(ld[i] - lse[(size_t)bh * nh * L + i]));
    }
    printf("max |out - oracle| = %.3e, max |lse - oracle| = %.3e\n", err, lerr);
    if (!(err <= 1e-4 && lerr <= 1e-4)) return 1;
    printf("ok\n");
    return 0;
}
