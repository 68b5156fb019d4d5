/*
 * Seeded synthetic-input generator (host C).  Holds no arithmetic of the
 * selective scan itself: it only turns (seed, stream, index) into numbers.
 *
 * Bits: Philox4x32-10, the counter-based generator of Salmon, Moraes, Dror and
 * Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3" (SC'11): ten rounds of
 *   (c0,c1,c2,c3) -> (hi(M1*c2)^c1^k0, lo(M1*c2), hi(M0*c0)^c3^k1, lo(M0*c0))
 * with the key bumped by the Weyl constants between rounds.
 *
 * Stream layout: element i of a tensor drawn on stream s with seed S takes
 * word (i mod 4) of the Philox block with key (lo32(S), hi32(S)) and counter
 * (lo32(i/4), hi32(i/4), s, 0).  Tensors drawn on different streams are
 * independent, and any element can be regenerated on its own.
 *
 * Normals: Box-Muller on word pairs (w0,w1) and (w2,w3) of a block, computed
 * in double with u = (w + 0.5) / 2^32 in (0, 1), then rounded to float (and to
 * bf16 by round-to-nearest-even on the float's bits when asked).
 * Uniforms: lo + (hi - lo) * u, in double, then rounded the same way.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define PHILOX_M0 0xD2511F53u
#define PHILOX_M1 0xCD9E8D57u
#define PHILOX_W0 0x9E3779B9u
#define PHILOX_W1 0xBB67AE85u

static void philox_round(uint32_t c[4], const uint32_t k[2])
{
    const uint64_t p0 = (uint64_t)PHILOX_M0 * c[0];
    const uint64_t p1 = (uint64_t)PHILOX_M1 * c[2];
    const uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
    const uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
    const uint32_t n0 = hi1 ^ c[1] ^ k[0];
    const uint32_t n2 = hi0 ^ c[3] ^ k[1];
    c[0] = n0;
    c[1] = lo1;
    c[2] = n2;
    c[3] = lo0;
}

void ssgen_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4])
{
    uint32_t c[4] = {ctr[0], ctr[1], ctr[2], ctr[3]};
    uint32_t k[2] = {key[0], key[1]};
    for (int r = 0; r < 10; ++r) {
        if (r > 0) {
            k[0] += PHILOX_W0;
            k[1] += PHILOX_W1;
        }
        philox_round(c, k);
    }
    memcpy(out, c, sizeof(c));
}

static inline double unit_open(uint32_t w)
{
    return ((double)w + 0.5) * (1.0 / 4294967296.0);
}

static inline uint16_t f32_to_bf16_rne(float f)
{
    uint32_t bits;
    memcpy(&bits, &f, sizeof(bits));
    if ((bits & 0x7fffffffu) > 0x7f800000u) /* NaN: keep it a quiet NaN */
        return (uint16_t)((bits >> 16) | 0x40u);
    const uint32_t lsb = (bits >> 16) & 1u;
    bits += 0x7fffu + lsb;
    return (uint16_t)(bits >> 16);
}

uint16_t ssgen_f32_to_bf16(float f) { return f32_to_bf16_rne(f); }

enum { SSGEN_NORMAL = 0, SSGEN_UNIFORM = 1 };
enum { SSGEN_F32 = 0, SSGEN_BF16 = 1 };

/*
 * Fill out[0..n) with draws of `kind` (normal: mean p0, std p1; uniform:
 * [p0, p1)), stored as float32 or bf16 bits.  Returns 0, or -1 on bad args.
 */
int ssgen_fill(uint64_t seed, uint32_t stream, int64_t n, int kind, double p0, double p1,
               int out_dtype, void *out, int nthreads)
{
    if (n < 0 || (n > 0 && !out) || (kind != SSGEN_NORMAL && kind != SSGEN_UNIFORM) ||
        (out_dtype != SSGEN_F32 && out_dtype != SSGEN_BF16))
        return -1;
    const uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    const int64_t nblocks = (n + 3) / 4;
    float *of = (float *)out;
    uint16_t *ob = (uint16_t *)out;
#ifdef _OPENMP
    if (nthreads <= 0)
        nthreads = omp_get_max_threads();
#pragma omp parallel for schedule(static) num_threads(nthreads)
#endif
    for (int64_t blk = 0; blk < nblocks; ++blk) {
        const uint32_t ctr[4] = {(uint32_t)blk, (uint32_t)((uint64_t)blk >> 32), stream, 0u};
        uint32_t w[4];
        ssgen_philox4x32_10(ctr, key, w);
        double v[4];
        if (kind == SSGEN_NORMAL) {
            for (int p = 0; p < 2; ++p) {
                const double r = sqrt(-2.0 * log(unit_open(w[2 * p])));
                const double t = 6.283185307179586476925 * unit_open(w[2 * p + 1]);
                v[2 * p] = p0 + p1 * (r * cos(t));
                v[2 * p + 1] = p0 + p1 * (r * sin(t));
            }
        } else {
            for (int j = 0; j < 4; ++j)
                v[j] = p0 + (p1 - p0) * unit_open(w[j]);
        }
        for (int j = 0; j < 4; ++j) {
            const int64_t i = blk * 4 + j;
            if (i >= n)
                break;
            const float f = (float)v[j];
            if (out_dtype == SSGEN_F32)
                of[i] = f;
            else
                ob[i] = f32_to_bf16_rne(f);
        }
    }
    return 0;
}
