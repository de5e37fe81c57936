/*
 * Q4_0 decode oracle: plain, slow, obviously correct CPU reference.
 *
 * TEST INFRASTRUCTURE ONLY. Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library. The product (the CUDA
 * library under quantized_decode_q4_b200/) never includes, links or calls it,
 * and this file includes nothing from the product.
 *
 * What it computes, and where that comes from:
 *   - "Llamas on the Web" (gist.science technical summary of arXiv 2605.20706),
 *     section "Design di Shader Consapevole della Quantizzazione": quantised
 *     weights are kept as packed integer words and dequantised inside the
 *     matrix-vector product at decode time.
 *   - "MicroLLM Lab" (sitech.ge), section "Seven models, all in Q4": 16-bit
 *     weights are compressed to 4 bits per parameter.
 *   - The pages never spell out the Q4_0 bit layout. The library fixes it as
 *     llama.cpp's legacy Q4_0 (named by "Llamas on the Web", problem statement,
 *     "legacy schemes"): blocks of 32 consecutive weights of a row, one IEEE
 *     binary16 scale d, 4-bit codes q in 0..15, w = d*(q-8), 18 bytes per block
 *     stored as {uint16 d; uint8 qs[16]} with qs[j] = q[j] | q[j+16] << 4.
 *
 * Readings where the pages are silent (each is pinned by a test):
 *   - tie in max|w| inside a block: the lowest index wins;
 *   - d = m / -8 with m the signed element of largest magnitude, in binary32;
 *   - code rounding: multiply by the binary32 reciprocal of d, add 8.5, take
 *     the floor, clamp to 0..15 (llama.cpp's quantiser convention);
 *   - codes come from the binary32 d; only its binary16 rounding is stored;
 *   - an all-zero block has m = +0, so d = +0 / -8 = -0 in IEEE arithmetic:
 *     it stores d bits 0x8000 and every code 8, and decodes to zeros.
 *
 * Precision: binary32 for the pack (it decides integer codes, so it uses the
 * same precision as the library's pack kernel), exact binary32 for dequant,
 * binary64 accumulation in index order for the matrix-vector products.
 *
 * Build: gcc -O2 -std=c99 -fPIC -shared -ffp-contract=off -fno-fast-math.
 * -ffp-contract=off matters: a fused multiply-add in the pack would change
 * codes at rounding boundaries.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define ORACLE_QK 32          /* weights per block                       */
#define ORACLE_BLOCK_BYTES 18 /* 2 bytes of d + 16 bytes of packed codes  */

/* ------------------------------------------------------------------------ */
/* IEEE-754 binary16 <-> binary32, written from the format's definition.    */
/* ------------------------------------------------------------------------ */

static uint32_t f32_bits(float f) {
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return u;
}

/*
 * binary32 -> binary16, round to nearest, ties to even.
 * A finite nonzero binary32 is m * 2^(e-23) with a 24-bit integer m. Its
 * binary16 neighbours are integer multiples of the binary16 quantum
 * 2^(max(e,-14)-10). Rounding m to that quantum gives an integer k; because
 * binary16 encodings are monotone and contiguous, the result's bits are
 * k itself in the subnormal range and ((e+15)<<10) + (k-1024) in the normal
 * range, with a carry of k to 2048 moving into the exponent field on its own
 * and exponent 31 meaning infinity.
 */
uint16_t oracle_f32_to_f16(float f) {
    uint32_t x = f32_bits(f);
    uint16_t sign = (uint16_t)((x >> 16) & 0x8000u);
    uint32_t ax = x & 0x7fffffffu;
    if (ax > 0x7f800000u) return (uint16_t)(sign | 0x7e00u); /* NaN stays NaN */
    if (ax == 0x7f800000u) return (uint16_t)(sign | 0x7c00u); /* infinity     */
    if (ax == 0) return sign;                                 /* signed zero  */

    int e;       /* unbiased exponent of the binary32 value */
    uint64_t m;  /* 24-bit integer significand               */
    if ((ax >> 23) == 0) { /* binary32 subnormal: far below 2^-25, rounds to 0 */
        return sign;
    }
    e = (int)(ax >> 23) - 127;
    m = (uint64_t)((ax & 0x7fffffu) | 0x800000u);
    if (e >= 16) return (uint16_t)(sign | 0x7c00u); /* >= 65536: overflow */

    int q_exp = (e < -14 ? -14 : e) - 10; /* exponent of the binary16 quantum  */
    int r = q_exp - (e - 23);             /* bits to drop from m (>= 13)        */
    uint64_t k;
    if (r >= 40) {
        k = 0;
    } else {
        uint64_t kept = m >> r;
        uint64_t rem = m & ((1ull << r) - 1);
        uint64_t halfway = 1ull << (r - 1);
        if (rem > halfway || (rem == halfway && (kept & 1u))) kept += 1;
        k = kept;
    }
    uint32_t bits;
    if (e < -14) {
        bits = (uint32_t)k; /* subnormal (k == 1024 is the smallest normal) */
    } else {
        bits = ((uint32_t)(e + 15) << 10) + (uint32_t)k - 1024u;
    }
    return (uint16_t)(sign | bits);
}

/* binary16 -> binary32, exact: every binary16 value is a binary32 value. */
float oracle_f16_to_f32(uint16_t h) {
    int sign = (h >> 15) & 1;
    int ex = (h >> 10) & 0x1f;
    int mant = h & 0x3ff;
    double v;
    if (ex == 0) {
        v = ldexp((double)mant, -24);
    } else if (ex == 31) {
        v = mant ? NAN : INFINITY;
    } else {
        v = ldexp((double)(1024 + mant), ex - 25);
    }
    return (float)(sign ? -v : v);
}

/* ------------------------------------------------------------------------ */
/* Pack: row-major binary32 W[n][k] -> row-major Q4_0 blocks (18 B each).   */
/* ------------------------------------------------------------------------ */

/* One block of 32 weights -> d bits and 16 packed code bytes. */
static void pack_block(const float *w, uint8_t *out) {
    /* signed element of largest magnitude; strict '>' keeps the first index;
       m stays +0 for a block with no nonzero element */
    float amax = 0.0f;
    float m = 0.0f;
    for (int j = 0; j < ORACLE_QK; ++j) {
        float a = fabsf(w[j]);
        if (a > amax) {
            amax = a;
            m = w[j];
        }
    }
    volatile float d = m / -8.0f; /* volatile: keep each step in binary32 */
    volatile float id = (d != 0.0f) ? 1.0f / d : 0.0f;
    uint8_t q[ORACLE_QK];
    for (int j = 0; j < ORACLE_QK; ++j) {
        volatile float scaled = w[j] * id;
        volatile float shifted = scaled + 8.5f;
        int code = (int)floorf(shifted);
        if (code < 0) code = 0;
        if (code > 15) code = 15;
        q[j] = (uint8_t)code;
    }
    uint16_t dh = oracle_f32_to_f16(d);
    out[0] = (uint8_t)(dh & 0xff); /* little-endian binary16 */
    out[1] = (uint8_t)(dh >> 8);
    for (int j = 0; j < ORACLE_QK / 2; ++j) {
        out[2 + j] = (uint8_t)(q[j] | (q[j + ORACLE_QK / 2] << 4));
    }
}

/* Returns 0 on success, -1 if k is not a multiple of 32. */
int oracle_q4_pack(const float *w, int64_t n, int64_t k, uint8_t *blocks) {
    if (k % ORACLE_QK != 0 || n < 0 || k < 0) return -1;
    int64_t nb = k / ORACLE_QK;
    for (int64_t r = 0; r < n; ++r) {
        for (int64_t b = 0; b < nb; ++b) {
            pack_block(w + r * k + b * ORACLE_QK,
                       blocks + (r * nb + b) * ORACLE_BLOCK_BYTES);
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Block accessors used by dequant and the products.                        */
/* ------------------------------------------------------------------------ */

static float block_scale(const uint8_t *blk) {
    uint16_t dh = (uint16_t)(blk[0] | (blk[1] << 8));
    return oracle_f16_to_f32(dh);
}

/* code of weight j (0..31) of a block: low nibbles hold j < 16, high j >= 16 */
static int block_code(const uint8_t *blk, int j) {
    uint8_t byte = blk[2 + (j % 16)];
    return j < 16 ? (byte & 0x0f) : (byte >> 4);
}

/* Dequant: w_hat = d * (q - 8), exact in binary32 (11-bit d times |q-8| <= 8). */
int oracle_q4_dequant(const uint8_t *blocks, int64_t n, int64_t k, float *w_out) {
    if (k % ORACLE_QK != 0 || n < 0 || k < 0) return -1;
    int64_t nb = k / ORACLE_QK;
    for (int64_t r = 0; r < n; ++r) {
        for (int64_t b = 0; b < nb; ++b) {
            const uint8_t *blk = blocks + (r * nb + b) * ORACLE_BLOCK_BYTES;
            float d = block_scale(blk);
            for (int j = 0; j < ORACLE_QK; ++j) {
                w_out[r * k + b * ORACLE_QK + j] = d * (float)(block_code(blk, j) - 8);
            }
        }
    }
    return 0;
}

/*
 * y[r] = sum_k w_hat[r][k] * x[k], binary64, summed in index order.
 * abs_sum[r] = sum_k |w_hat[r][k] * x[k]| (the scale of the GEMV tolerance).
 * abs_sum may be NULL.
 */
int oracle_q4_gemv(const uint8_t *blocks, int64_t n, int64_t k, const float *x,
                   double *y, double *abs_sum) {
    if (k % ORACLE_QK != 0 || n < 0 || k < 0) return -1;
    int64_t nb = k / ORACLE_QK;
    for (int64_t r = 0; r < n; ++r) {
        double acc = 0.0, sabs = 0.0;
        for (int64_t b = 0; b < nb; ++b) {
            const uint8_t *blk = blocks + (r * nb + b) * ORACLE_BLOCK_BYTES;
            double d = (double)block_scale(blk);
            for (int j = 0; j < ORACLE_QK; ++j) {
                double w_hat = d * (double)(block_code(blk, j) - 8);
                double term = w_hat * (double)x[b * ORACLE_QK + j];
                acc += term;
                sabs += fabs(term);
            }
        }
        y[r] = acc;
        if (abs_sum) abs_sum[r] = sabs;
    }
    return 0;
}

/*
 * Small-batch product: Y[t][r] = sum_k w_hat[r][k] * X[t][k] for t < batch,
 * X row-major [batch][k], Y and abs_sum row-major [batch][n].
 */
int oracle_q4_gemv_batched(const uint8_t *blocks, int64_t n, int64_t k, const float *X,
                           int64_t batch, double *Y, double *abs_sum) {
    if (batch < 0) return -1;
    for (int64_t t = 0; t < batch; ++t) {
        int rc = oracle_q4_gemv(blocks, n, k, X + t * k, Y + t * n,
                                abs_sum ? abs_sum + t * n : (double *)0);
        if (rc) return rc;
    }
    return 0;
}

/*
 * Split row-major blocks into the two planes the device format uses:
 * qs[n][k/2] (the 16 code bytes of each block, in block order) and
 * d[n][k/32] (the binary16 scale bits). The bytes are unchanged.
 */
int oracle_blocks_to_planes(const uint8_t *blocks, int64_t n, int64_t k, uint8_t *qs,
                            uint16_t *d) {
    if (k % ORACLE_QK != 0 || n < 0 || k < 0) return -1;
    int64_t nblocks = n * (k / ORACLE_QK);
    for (int64_t i = 0; i < nblocks; ++i) {
        const uint8_t *blk = blocks + i * ORACLE_BLOCK_BYTES;
        d[i] = (uint16_t)(blk[0] | (blk[1] << 8));
        memcpy(qs + i * 16, blk + 2, 16);
    }
    return 0;
}
