/*
 * Seeded, counter-based input generator shared by the tests, the oracle
 * harness and the benchmark.  It holds none of the MoE layer's arithmetic:
 * only Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random numbers:
 * as easy as 1, 2, 3", SC'11) and the Box-Muller transform.
 *
 * Every element of a generated tensor is a pure function of
 * (seed, stream, element index), so chunked or multi-threaded generation
 * gives bit-identical results.
 *
 *   key     = (low 32 bits of seed, stream)
 *   counter = (block index low, block index high, 0, 0), block = element / 4
 *
 * Uniforms: u = (word + 0.5) * 2^-32, in (0, 1).
 * Normals:  words (0,1) and (2,3) of a block each give one Box-Muller pair,
 *           r = sqrt(-2 ln u_a), z = r cos(2 pi u_b) or r sin(2 pi u_b),
 *           evaluated in double, then scaled and rounded once to float.
 */
#include <math.h>
#include <stdint.h>

#define PHILOX_M0 0xD2511F53u
#define PHILOX_M1 0xCD9E8D57u
#define PHILOX_W0 0x9E3779B9u
#define PHILOX_W1 0xBB67AE85u

static inline void mulhilo32(uint32_t a, uint32_t b, uint32_t *hi, uint32_t *lo) {
    uint64_t p = (uint64_t)a * (uint64_t)b;
    *hi = (uint32_t)(p >> 32);
    *lo = (uint32_t)p;
}

void synth_philox4x32_10(const uint32_t ctr_in[4], const uint32_t key_in[2], uint32_t out[4]) {
    uint32_t c0 = ctr_in[0], c1 = ctr_in[1], c2 = ctr_in[2], c3 = ctr_in[3];
    uint32_t k0 = key_in[0], k1 = key_in[1];
    for (int round = 0; round < 10; ++round) {
        uint32_t hi0, lo0, hi1, lo1;
        mulhilo32(PHILOX_M0, c0, &hi0, &lo0);
        mulhilo32(PHILOX_M1, c2, &hi1, &lo1);
        uint32_t n0 = hi1 ^ c1 ^ k0;
        uint32_t n1 = lo1;
        uint32_t n2 = hi0 ^ c3 ^ k1;
        uint32_t n3 = lo0;
        c0 = n0; c1 = n1; c2 = n2; c3 = n3;
        k0 += PHILOX_W0;
        k1 += PHILOX_W1;
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

static inline void block_words(uint64_t seed, uint32_t stream, uint64_t block, uint32_t w[4]) {
    uint32_t ctr[4] = {(uint32_t)block, (uint32_t)(block >> 32), 0u, 0u};
    uint32_t key[2] = {(uint32_t)seed, stream};
    synth_philox4x32_10(ctr, key, w);
}

static inline double word_to_unit(uint32_t w) {
    return ((double)w + 0.5) * (1.0 / 4294967296.0);
}

/* out[i] = float(mean + sigma * z(start + i)), i in [0, n) */
void synth_normal_f32(uint64_t seed, uint32_t stream, uint64_t start, uint64_t n,
                      double sigma, double mean, float *out) {
    if (n == 0) return;
    const double two_pi = 6.283185307179586476925286766559;
    uint64_t b0 = start >> 2, b1 = (start + n - 1) >> 2;
    #pragma omp parallel for schedule(static)
    for (int64_t b = (int64_t)b0; b <= (int64_t)b1; ++b) {
        uint32_t w[4];
        block_words(seed, stream, (uint64_t)b, w);
        double z[4];
        for (int p = 0; p < 2; ++p) {
            double rad = sqrt(-2.0 * log(word_to_unit(w[2 * p])));
            double ang = two_pi * word_to_unit(w[2 * p + 1]);
            z[2 * p] = rad * cos(ang);
            z[2 * p + 1] = rad * sin(ang);
        }
        for (int r = 0; r < 4; ++r) {
            uint64_t e = ((uint64_t)b << 2) + (uint64_t)r;
            if (e >= start && e < start + n) out[e - start] = (float)(mean + sigma * z[r]);
        }
    }
}

/* out[i] = u(start + i) in (0, 1) */
void synth_uniform_f64(uint64_t seed, uint32_t stream, uint64_t start, uint64_t n, double *out) {
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < (int64_t)n; ++i) {
        uint64_t e = start + (uint64_t)i;
        uint32_t w[4];
        block_words(seed, stream, e >> 2, w);
        out[i] = word_to_unit(w[e & 3]);
    }
}
