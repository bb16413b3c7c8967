// Host-side generator of the random rotations R[n_hashes, d, n_buckets/2]
// ("LSH Attention": angular LSH with a random rotation per round, entries
// drawn from N(0, 1)).
//
// Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as easy
// as 1, 2, 3", SC 2011): ten rounds of two 32x32->64-bit multiplies with the
// Weyl key schedule, counter = (block, 0, 0, 0) with a 64-bit block index, key
// = (low word of seed, 2 ^ high word of seed).  Each block gives four 32-bit
// words; word u becomes the uniform (u + 0.5) 2^-32 in (0, 1), and
// consecutive uniform pairs (u0, u1) become two standard normals by the
// Box-Muller transform, sqrt(-2 ln u0) (cos, sin)(2 pi u1), in double.  The
// normals are rounded to float32, then (bf16) to bfloat16 with
// round-to-nearest-even.  The same definition drives the repository's
// synthetic inputs, so a seed below 2^32 reproduces their rotations.
#include <math.h>
#include <stdint.h>
#include <string.h>

#include "../../include/lsh_attn.h"

namespace {

struct Philox {
    uint32_t k0, k1;
    void block(uint64_t ctr, uint32_t out[4]) const
    {
        uint32_t c0 = (uint32_t)ctr, c1 = (uint32_t)(ctr >> 32), c2 = 0, c3 = 0;
        uint32_t a = k0, b = k1;
        for (int r = 0; r < 10; ++r) {
            const uint64_t p0 = (uint64_t)0xD2511F53u * c0;
            const uint64_t p1 = (uint64_t)0xCD9E8D57u * c2;
            const uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
            const uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
            const uint32_t n0 = hi1 ^ c1 ^ a, n1 = lo1, n2 = hi0 ^ c3 ^ b, n3 = lo0;
            c0 = n0; c1 = n1; c2 = n2; c3 = n3;
            a += 0x9E3779B9u;
            b += 0xBB67AE85u;
        }
        out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
    }
    uint32_t word(uint64_t i) const
    {
        uint32_t w[4];
        block(i >> 2, w);
        return w[i & 3];
    }
};

uint16_t to_bf16_bits(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

}  // namespace

extern "C" LSH_API lsh_status lsh_attn_make_rotations(uint64_t seed, const lsh_attn_desc *desc, void *R_host)
{
    if (!desc || !R_host) return LSH_ERR_ARG;
    if (desc->dtype != LSH_F32 && desc->dtype != LSH_BF16) return LSH_ERR_ARG;
    if (desc->d < 1 || desc->n_hashes < 1) return LSH_ERR_SHAPE;
    if (desc->n_buckets < 2 || desc->n_buckets % 2 != 0 || desc->n_buckets > 65536) return LSH_ERR_SHAPE;
    const Philox g{(uint32_t)seed, 2u ^ (uint32_t)(seed >> 32)};
    const uint64_t n = (uint64_t)desc->n_hashes * (uint64_t)desc->d * (uint64_t)(desc->n_buckets / 2);
    const double two32 = 1.0 / 4294967296.0, two_pi = 6.283185307179586476925286766559;
    for (uint64_t i = 0; i < n; i += 2) {
        const double u0 = ((double)g.word(i) + 0.5) * two32;
        const double u1 = ((double)g.word(i + 1) + 0.5) * two32;
        const double rad = sqrt(-2.0 * log(u0)), ang = two_pi * u1;
        const double z[2] = {rad * cos(ang), rad * sin(ang)};
        for (int k = 0; k < 2 && i + k < n; ++k) {
            const float f = (float)z[k];
            if (desc->dtype == LSH_F32)
                static_cast<float *>(R_host)[i + k] = f;
            else
                static_cast<uint16_t *>(R_host)[i + k] = to_bf16_bits(f);
        }
    }
    return LSH_OK;
}
