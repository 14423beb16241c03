/*
 * Seeded N(0,1) input values for the synthetic decode workloads.
 *
 * Counter-based so that any thread count gives the same values:
 *   - Philox4x32-10 (Salmon, Moraes, Dror and Shaw, "Parallel Random Numbers:
 *     As Easy as 1, 2, 3", SC 2011): 10 rounds of the 4x32 Philox S-box with
 *     multipliers 0xD2511F53 / 0xCD9E8D57 and Weyl key increments
 *     0x9E3779B9 / 0xBB67AE85;
 *   - each counter value (index j, stream) gives four 32-bit words, turned into
 *     uniforms in (0, 1) and then into four normals by the Box-Muller
 *     transform (Box and Muller, 1958);
 *   - optional rounding of the float32 value to bfloat16, nearest-even.
 *
 * Input generation only: nothing here is part of what the attention computes.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

static void philox_round(uint32_t c[4], const uint32_t k[2])
{
    uint64_t p0 = (uint64_t)0xD2511F53u * c[0];
    uint64_t p1 = (uint64_t)0xCD9E8D57u * c[2];
    uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
    uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
    uint32_t n0 = hi1 ^ c[1] ^ k[0];
    uint32_t n2 = hi0 ^ c[3] ^ k[1];
    c[0] = n0;
    c[1] = lo1;
    c[2] = n2;
    c[3] = lo0;
}

void synth_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4])
{
    uint32_t c[4] = {ctr[0], ctr[1], ctr[2], ctr[3]};
    uint32_t k[2] = {key[0], key[1]};
    for (int r = 0; r < 10; ++r) {
        if (r > 0) {
            k[0] += 0x9E3779B9u;
            k[1] += 0xBB67AE85u;
        }
        philox_round(c, k);
    }
    memcpy(out, c, sizeof c);
}

static uint16_t to_bf16_rne(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

/* n normals for (seed, stream); element i comes from counter i / 4.
 * out_f32 (float*) or out_bf16 (uint16_t*): exactly one is non-null. */
void synth_normals(uint64_t seed, uint32_t stream, int64_t n, float *out_f32, uint16_t *out_bf16)
{
    const double two_pi = 6.283185307179586476925286766559;
    const double inv32 = 1.0 / 4294967296.0;
    int64_t nblk = (n + 3) / 4;
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < nblk; ++j) {
        uint32_t ctr[4] = {(uint32_t)j, (uint32_t)((uint64_t)j >> 32), stream, 0u};
        uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
        uint32_t w[4];
        synth_philox4x32_10(ctr, key, w);
        float z[4];
        for (int pr = 0; pr < 2; ++pr) {
            double u1 = ((double)w[2 * pr] + 0.5) * inv32;
            double u2 = ((double)w[2 * pr + 1] + 0.5) * inv32;
            double r = sqrt(-2.0 * log(u1));
            z[2 * pr] = (float)(r * cos(two_pi * u2));
            z[2 * pr + 1] = (float)(r * sin(two_pi * u2));
        }
        for (int e = 0; e < 4; ++e) {
            int64_t i = 4 * j + e;
            if (i >= n)
                break;
            if (out_f32)
                out_f32[i] = z[e];
            else
                out_bf16[i] = to_bf16_rne(z[e]);
        }
    }
}
