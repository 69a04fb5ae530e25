/*
 * Seeded synthetic-input generator (host side).
 *
 * This file holds no arithmetic of the decoder itself: it only produces the
 * random-init weights and the synthetic token ids / activations that the
 * workloads are defined on (weights N(0, 0.02^2), gains 1, token ids uniform
 * in [0, V)).  It is shared by the fp64 oracle and the tests; the CUDA
 * library carries its own independent device implementation of the same
 * published generator.
 *
 * Generator, from its published definitions:
 *   - Philox4x32-10: Salmon, Moraes, Dror, Shaw, "Parallel random numbers:
 *     as easy as 1, 2, 3", SC'11.  Round function on a 128-bit counter
 *     (x0,x1,x2,x3) with a 64-bit key (k0,k1):
 *        (hi0,lo0) = mulhilo(0xD2511F53, x0), (hi1,lo1) = mulhilo(0xCD9E8D57, x2)
 *        x' = (hi1 ^ x1 ^ k0, lo1, hi0 ^ x3 ^ k1, lo0)
 *     ten rounds, the key advanced by the Weyl constants
 *     (0x9E3779B9, 0xBB67AE85) between consecutive rounds.
 *   - Box-Muller transform (Box & Muller, 1958): two uniforms u1 in (0,1],
 *     u2 in [0,1) give R cos(2 pi u2) and R sin(2 pi u2), R = sqrt(-2 ln u1).
 *
 * Element mapping (the contract both implementations follow):
 *   key      = (seed, tensor_id)
 *   element e of a tensor uses counter (e >> 2, 0, 0, 0) split as
 *            x0 = low 32 bits, x1 = high 32 bits of (e >> 2), x2 = x3 = 0
 *   lane j = e & 3 takes the pair p = j >> 1: a = r[2p], b = r[2p+1],
 *            u1 = (a + 1) * 2^-32,  u2 = b * 2^-32,
 *            z  = R cos(2 pi u2)  (j even)   or   R sin(2 pi u2)  (j odd)
 *   value    = scale * z in fp64, then rounded to nearest-even into the
 *              storage type (fp32 or bf16) directly from fp64.
 *   token t  = (r0 * V) >> 32 with counter (t, 0, 0, 0): integer exact.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define PHILOX_M0 0xD2511F53u
#define PHILOX_M1 0xCD9E8D57u
#define PHILOX_W0 0x9E3779B9u
#define PHILOX_W1 0xBB67AE85u

static inline void philox_round(uint32_t x[4], uint32_t k0, uint32_t k1) {
    uint64_t p0 = (uint64_t)PHILOX_M0 * x[0];
    uint64_t p1 = (uint64_t)PHILOX_M1 * x[2];
    uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
    uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
    uint32_t y0 = hi1 ^ x[1] ^ k0;
    uint32_t y2 = hi0 ^ x[3] ^ k1;
    x[0] = y0;
    x[1] = lo1;
    x[2] = y2;
    x[3] = lo0;
}

void synth_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]) {
    uint32_t x[4] = {ctr[0], ctr[1], ctr[2], ctr[3]};
    uint32_t k0 = key[0], k1 = key[1];
    for (int r = 0; r < 10; ++r) {
        if (r > 0) {
            k0 += PHILOX_W0;
            k1 += PHILOX_W1;
        }
        philox_round(x, k0, k1);
    }
    memcpy(out, x, sizeof(x));
}

static inline double normal_at(uint32_t seed, uint32_t tensor_id, uint64_t e) {
    uint32_t ctr[4] = {(uint32_t)(e >> 2), (uint32_t)(e >> 34), 0u, 0u};
    uint32_t key[2] = {seed, tensor_id};
    uint32_t r[4];
    synth_philox4x32_10(ctr, key, r);
    int j = (int)(e & 3u);
    int p = j >> 1;
    double u1 = ((double)r[2 * p] + 1.0) * 2.3283064365386963e-10; /* 2^-32 */
    double u2 = (double)r[2 * p + 1] * 2.3283064365386963e-10;
    double R = sqrt(-2.0 * log(u1));
    double t = 2.0 * 3.141592653589793 * u2;
    return (j & 1) ? R * sin(t) : R * cos(t);
}

/* fp64 -> bf16, round to nearest, ties to even, directly from fp64.
 * Finite inputs inside the fp32 normal range are all this generator makes;
 * the conversion goes through fp32 with round-to-odd, which (fp32 carrying
 * 16 more significand bits than bf16) gives the correctly rounded result. */
static inline uint16_t f64_to_bf16_rne(double x) {
    float f = (float)x;               /* nearest fp32 */
    if ((double)f != x) {
        /* truncate toward zero, then set the sticky (odd) bit */
        if (fabs((double)f) > fabs(x)) f = nextafterf(f, 0.0f);
        uint32_t b;
        memcpy(&b, &f, 4);
        b |= 1u;
        memcpy(&f, &b, 4);
    }
    uint32_t bits;
    memcpy(&bits, &f, 4);
    uint32_t lsb = (bits >> 16) & 1u;
    bits += 0x7FFFu + lsb;
    return (uint16_t)(bits >> 16);
}

uint16_t synth_f64_to_bf16(double x) { return f64_to_bf16_rne(x); }

/* Elements [first, first+count) computed four at a time: one Philox call and
 * one (u1 -> R) per pair of lanes serve all four; every element still gets
 * exactly the value normal_at(e) defines. */
static inline void normals_block(uint32_t seed, uint32_t tensor_id, uint64_t e4, double out[4]) {
    uint32_t ctr[4] = {(uint32_t)e4, (uint32_t)(e4 >> 32), 0u, 0u};
    uint32_t key[2] = {seed, tensor_id};
    uint32_t r[4];
    synth_philox4x32_10(ctr, key, r);
    for (int p = 0; p < 2; ++p) {
        double u1 = ((double)r[2 * p] + 1.0) * 2.3283064365386963e-10;
        double u2 = (double)r[2 * p + 1] * 2.3283064365386963e-10;
        double R = sqrt(-2.0 * log(u1));
        double t = 2.0 * 3.141592653589793 * u2;
        out[2 * p] = R * cos(t);
        out[2 * p + 1] = R * sin(t);
    }
}

static inline void normals_range(uint32_t seed, uint32_t tensor_id, uint64_t first, uint64_t count, double scale,
                                 double* out) {
    const int64_t b0 = (int64_t)(first >> 2), b1 = (int64_t)((first + count + 3) >> 2);
#pragma omp parallel for schedule(static)
    for (int64_t blk = b0; blk < b1; ++blk) {
        double z[4];
        normals_block(seed, tensor_id, (uint64_t)blk, z);
        for (int j = 0; j < 4; ++j) {
            const uint64_t e = ((uint64_t)blk << 2) + (uint64_t)j;
            if (e >= first && e < first + count) out[e - first] = scale * z[j];
        }
    }
}

/* out[i] = scale * z_{first+i}, fp64, unrounded */
void synth_normal_f64(uint32_t seed, uint32_t tensor_id, uint64_t first, uint64_t count,
                      double scale, double* out) {
    normals_range(seed, tensor_id, first, count, scale, out);
}

/* rounded to the storage type, returned as fp64 values (exactly representable) */
void synth_normal_stored_f64(uint32_t seed, uint32_t tensor_id, uint64_t first, uint64_t count,
                             double scale, int dtype_bf16, double* out) {
    normals_range(seed, tensor_id, first, count, scale, out);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < (int64_t)count; ++i) {
        double v = out[i];
        if (dtype_bf16) {
            uint32_t b = (uint32_t)f64_to_bf16_rne(v) << 16;
            float f;
            memcpy(&f, &b, 4);
            out[i] = (double)f;
        } else {
            out[i] = (double)(float)v;
        }
    }
}

void synth_normal_bf16(uint32_t seed, uint32_t tensor_id, uint64_t first, uint64_t count,
                       double scale, uint16_t* out) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < (int64_t)count; ++i)
        out[i] = f64_to_bf16_rne(scale * normal_at(seed, tensor_id, first + (uint64_t)i));
}

void synth_normal_f32(uint32_t seed, uint32_t tensor_id, uint64_t first, uint64_t count,
                      double scale, float* out) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < (int64_t)count; ++i)
        out[i] = (float)(scale * normal_at(seed, tensor_id, first + (uint64_t)i));
}

void synth_tokens(uint32_t seed, uint32_t tensor_id, uint64_t first, uint64_t count,
                  uint32_t vocab, int32_t* out) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < (int64_t)count; ++i) {
        uint64_t e = first + (uint64_t)i;
        uint32_t ctr[4] = {(uint32_t)e, (uint32_t)(e >> 32), 0u, 0u};
        uint32_t key[2] = {seed, tensor_id};
        uint32_t r[4];
        synth_philox4x32_10(ctr, key, r);
        out[i] = (int32_t)(((uint64_t)r[0] * (uint64_t)vocab) >> 32);
    }
}
