/* A plain C caller of the library: rotations from a seed, inputs from a small
 * generator, then through the C ABI on the GPU (a) one fp32 forward (CUDA-core
 * kernels) and (b) one bf16 forward and backward (tensor-core kernels), each
 * checked against the CPU oracle run with the GPU's permutation.  Exit status
 * 0 and the line "ok" on success.  With --compile-check it only links and
 * returns. */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime_api.h>

#include "lsh_attn.h"

/* test infrastructure: the oracle's forward for one (batch, head) */
int oracle_fwd_head_perm(const double *x, const double *v, long L, int d, const int32_t *perm, int n_hashes, int m,
                         int causal, const int32_t *bucket, int self_penalty, double *y, double *lse);
int oracle_bwd_head(const double *x, const double *v, const double *dy, long L, int d, const int32_t *perm,
                    int n_hashes, int m, int causal, const int32_t *bucket, int self_penalty, double *dx,
                    double *dv);

/* float -> bfloat16 bits, round to nearest even (finite inputs), and back */
static uint16_t to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}
static float from_bf16(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

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

static int run_f32(void)
{
    const int B = 1, H = 2, L = 512, d = 64, nb = 16, nh = 2, m = 64, causal = 1;
    lsh_attn_desc desc = {B, H, L, d, nb, nh, m, causal, LSH_F32, 0};
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
        CHECK(oracle_fwd_head_perm(xd, vd, L, d, perm + (size_t)bh * nh * L, nh, m, causal, NULL, 0, yd, ld));
        for (size_t i = 0; i < (size_t)L * d; ++i) err = fmax(err, fabs(yd[i] - out[(size_t)bh * L * d + i]));
        for (size_t i = 0; i < (size_t)nh * L; ++i) lerr = fmax(lerr, fabs(ld[i] - lse[(size_t)bh * nh * L + i]));
    }
    printf("fp32: max |out - oracle| = %.3e, max |lse - oracle| = %.3e\n", err, lerr);
    return err <= 1e-4 && lerr <= 1e-4 ? 0 : 1;
}

/* max-abs and relative-L2 error of n bf16 GPU values against the oracle */
static void bf16_errors(const uint16_t *got, const double *want, size_t n, double *max_abs, double *num,
                        double *den)
{
    for (size_t i = 0; i < n; ++i) {
        const double e = (double)from_bf16(got[i]) - want[i];
        if (fabs(e) > *max_abs) *max_abs = fabs(e);
        *num += e * e;
        *den += want[i] * want[i];
    }
}

static int run_bf16(void)
{
    const int B = 1, H = 2, L = 512, d = 64, nb = 64, nh = 2, m = 64, causal = 1;
    lsh_attn_desc desc = {B, H, L, d, nb, nh, m, causal, LSH_BF16, 0};
    const size_t n = (size_t)B * H * L * d, nr = (size_t)nh * d * (nb / 2), ns = (size_t)B * H * nh * L;
    uint16_t *x = malloc(n * 2), *v = malloc(n * 2), *g = malloc(n * 2), *R = malloc(nr * 2);
    uint16_t *out = malloc(n * 2), *dqk = malloc(n * 2), *dv = malloc(n * 2);
    int32_t *perm = malloc(ns * 4);
    if (!x || !v || !g || !R || !out || !dqk || !dv || !perm) return 1;
    for (size_t i = 0; i < n; ++i) x[i] = to_bf16(next_normal());
    for (size_t i = 0; i < n; ++i) v[i] = to_bf16(next_normal());
    for (size_t i = 0; i < n; ++i) g[i] = to_bf16(next_normal());
    CHECK(lsh_attn_make_rotations(7, &desc, R));

    void *d_x, *d_v, *d_g, *d_R, *d_out, *d_dqk, *d_dv, *d_wf, *d_wb;
    float *d_lse;
    int32_t *d_perm;
    const size_t wf = lsh_attn_workspace_size(&desc, 0), wb = lsh_attn_workspace_size(&desc, 1);
    if (wf == 0 || wb == 0) return 1;
    CHECK(cudaMalloc(&d_x, n * 2));
    CHECK(cudaMalloc(&d_v, n * 2));
    CHECK(cudaMalloc(&d_g, n * 2));
    CHECK(cudaMalloc(&d_R, nr * 2));
    CHECK(cudaMalloc(&d_out, n * 2));
    CHECK(cudaMalloc(&d_dqk, n * 2));
    CHECK(cudaMalloc(&d_dv, n * 2));
    CHECK(cudaMalloc((void **)&d_lse, ns * 4));
    CHECK(cudaMalloc((void **)&d_perm, ns * 4));
    CHECK(cudaMalloc(&d_wf, wf));
    CHECK(cudaMalloc(&d_wb, wb));
    CHECK(cudaMemcpy(d_x, x, n * 2, cudaMemcpyHostToDevice));
    CHECK(cudaMemcpy(d_v, v, n * 2, cudaMemcpyHostToDevice));
    CHECK(cudaMemcpy(d_g, g, n * 2, cudaMemcpyHostToDevice));
    CHECK(cudaMemcpy(d_R, R, nr * 2, cudaMemcpyHostToDevice));
    CHECK(lsh_attn_fwd(&desc, d_x, d_v, d_R, d_out, d_lse, d_perm, d_wf, wf, NULL));
    CHECK(lsh_attn_bwd(&desc, d_x, d_v, d_R, d_out, d_lse, d_perm, d_g, d_dqk, d_dv, d_wb, wb, NULL));
    CHECK(lsh_attn_poll(d_wf, NULL));
    CHECK(lsh_attn_poll(d_wb, NULL));
    CHECK(cudaMemcpy(out, d_out, n * 2, cudaMemcpyDeviceToHost));
    CHECK(cudaMemcpy(dqk, d_dqk, n * 2, cudaMemcpyDeviceToHost));
    CHECK(cudaMemcpy(dv, d_dv, n * 2, cudaMemcpyDeviceToHost));
    CHECK(cudaMemcpy(perm, d_perm, ns * 4, cudaMemcpyDeviceToHost));

    const size_t hd = (size_t)L * d;
    double *xd = malloc(hd * 8), *vd = malloc(hd * 8), *gd = malloc(hd * 8), *yd = malloc(hd * 8),
           *ld = malloc((size_t)nh * L * 8), *dxd = malloc(hd * 8), *dvd = malloc(hd * 8);
    if (!xd || !vd || !gd || !yd || !ld || !dxd || !dvd) return 1;
    double e_out = 0, e_dx = 0, e_dv = 0, n_out = 0, n_dx = 0, n_dv = 0, s_out = 0, s_dx = 0, s_dv = 0;
    for (int bh = 0; bh < B * H; ++bh) {
        for (size_t i = 0; i < hd; ++i) {
            xd[i] = from_bf16(x[bh * hd + i]);
            vd[i] = from_bf16(v[bh * hd + i]);
            gd[i] = from_bf16(g[bh * hd + i]);
        }
        const int32_t *pb = perm + (size_t)bh * nh * L;
        CHECK(oracle_fwd_head_perm(xd, vd, L, d, pb, nh, m, causal, NULL, 0, yd, ld));
        CHECK(oracle_bwd_head(xd, vd, gd, L, d, pb, nh, m, causal, NULL, 0, dxd, dvd));
        bf16_errors(out + bh * hd, yd, hd, &e_out, &n_out, &s_out);
        bf16_errors(dqk + bh * hd, dxd, hd, &e_dx, &n_dx, &s_dx);
        bf16_errors(dv + bh * hd, dvd, hd, &e_dv, &n_dv, &s_dv);
    }
    const double r_out = sqrt(n_out / s_out), r_dx = sqrt(n_dx / s_dx), r_dv = sqrt(n_dv / s_dv);
    printf("bf16: out max_abs %.3e rel_l2 %.3e; dqk max_abs %.3e rel_l2 %.3e; dv max_abs %.3e rel_l2 %.3e\n",
           e_out, r_out, e_dx, r_dx, e_dv, r_dv);
    return e_out <= 2e-2 && e_dx <= 2e-2 && e_dv <= 2e-2 && r_out <= 1e-2 && r_dx <= 1e-2 && r_dv <= 1e-2 ? 0 : 1;
}

int main(int argc, char **argv)
{
    if (argc > 1 && strcmp(argv[1], "--compile-check") == 0) return lsh_attn_abi_version() == LSH_ATTN_ABI_VERSION ? 0 : 1;
    if (run_f32() != 0) return 1;
    if (run_bf16() != 0) return 1;
    printf("ok\n");
    return 0;
}
