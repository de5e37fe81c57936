// Integer dot product of Q4_0 codes with activations held in 31-bit block fixed
// point: the register-level core of the batch-1 kernel.
//
// A block of 32 activations is written x_j ~= s X_j with a power-of-two scale
// s = 2^e chosen so that max_j |x_j| / s lies in [2^29, 2^30), and integers
// X_j = rne(x_j / s). Dividing by a power of two is exact, so the only
// approximation is the rounding of x_j / s to an integer: an absolute error of
// at most s/2, relative error 2^-30 for the largest element but unbounded for an
// element much smaller than the block's largest. Every element whose rounding
// error exceeds kXRel = 2^-14 of its own magnitude marks the block as flagged;
// a flagged block is multiplied in binary32 instead (the exact path), so every
// element that reaches the integer path is within 2^-14 of itself. That makes the
// GEMV error at most 2^-14 sum |w x| (plus binary32 rounding of the block sums)
// for any input, whatever the spread of magnitudes inside a block: one outlier
// inflates the scale, its neighbours' rounding errors exceed the bound, and the
// block takes the exact path.
//
// Each X_j is split into two signed 16-bit digits X_j = 65536 D1_j + D0_j
// (D0_j in -32768..32767, |D1_j| <= 2^14), and the block sum over codes q_j in
// 0..15 is exact in integers:
//   sum_j (q_j - 8) X_j = 65536 S1 + S0,   Sp = sum_j q_j Dp_j - 8 sum_j Dp_j,
// each sum_j q_j Dp_j a chain of dp2a instructions (two 16-bit digits times two
// 8-bit codes per instruction). |S0| <= 2^23 and |S1| <= 2^22, so 16 S0 and
// 16 S1 (the form block_dot16 computes) convert to binary32 exactly and one
// fused multiply-add forms 16 times the block sum.
#pragma once

#include <cstdint>
#include <cmath>
#include <cstring>

#include <cuda_runtime.h>

namespace q4dev {

// Largest relative rounding error an element may carry into the integer path.
constexpr float kXRel = 1.0f / 16384.0f;  // 2^-14
// Blocks whose largest |x| lies outside [2^kXExpLo, 2^kXExpHi) are flagged (the
// power-of-two scale and its reciprocal must stay normal binary32 numbers).
constexpr int kXExpLo = -60;
constexpr int kXExpHi = 100;

__host__ __device__ __forceinline__ uint32_t f32_bits(float f) {
#ifdef __CUDA_ARCH__
    return __float_as_uint(f);
#else
    uint32_t u;
    memcpy(&u, &f, 4);
    return u;
#endif
}

__host__ __device__ __forceinline__ float bits_to_f32(uint32_t u) {
#ifdef __CUDA_ARCH__
    return __uint_as_float(u);
#else
    float f;
    memcpy(&f, &u, 4);
    return f;
#endif
}

// Scale of a block from the bit pattern of its largest |x| (a non-negative
// binary32): writes s = 2^e and 1/s, returns false if the block must be flagged
// (largest |x| not finite or outside the supported exponent range). A block of
// zeros gets s = 0, 1/s = 0 and is not flagged.
__host__ __device__ __forceinline__ bool xq_scale(uint32_t maxbits, float* s, float* inv) {
    if (maxbits == 0) {
        *s = 0.0f;
        *inv = 0.0f;
        return true;
    }
    const int E = (int)(maxbits >> 23);  // biased exponent (maxbits has no sign bit)
    if (E >= 255 || E - 127 < kXExpLo || E - 127 >= kXExpHi) {
        *s = 0.0f;
        *inv = 0.0f;
        return false;
    }
    // max in [2^(E-127), 2^(E-126)); max / s in [2^29, 2^30) for s = 2^(E-156)
    *s = bits_to_f32((uint32_t)(E - 29) << 23);
    *inv = bits_to_f32((uint32_t)(283 - E) << 23);
    return true;
}

// X = rne(x * inv) and whether the element keeps its rounding error within
// kXRel of itself. x * inv is exact (inv is a power of two and the product is a
// normal number or zero), and t - X is exact (for |t| >= 2^23, t is an integer).
__host__ __device__ __forceinline__ int32_t xq_int(float x, float inv, bool* ok) {
    const float t = x * inv;
#ifdef __CUDA_ARCH__
    const int32_t X = __float2int_rn(t);
#else
    const int32_t X = (int32_t)nearbyintf(t);
#endif
    const float r = t - (float)X;
    *ok = fabsf(r) <= kXRel * fabsf(t);
    return X;
}

// Signed 16-bit digits of |X| <= 2^30: X = 65536 d1 + d0, d0 in -32768..32767.
__host__ __device__ __forceinline__ void x_digits16(int32_t X, int32_t* d0, int32_t* d1) {
    const int32_t lo = (int32_t)(int16_t)(uint16_t)((uint32_t)X & 0xFFFFu);
    *d0 = lo;
    *d1 = (X - lo) >> 16;
}

__host__ __device__ __forceinline__ uint32_t pack16(int32_t a, int32_t b) {
    return ((uint32_t)a & 0xFFFFu) | ((uint32_t)b << 16);
}

// Sum over the low (mode lo) or high (mode hi) two bytes of u (unsigned bytes)
// times the two signed 16-bit halves of a, plus acc.
__host__ __device__ __forceinline__ int32_t dp2a_lo(uint32_t a, uint32_t u, int32_t acc) {
#ifdef __CUDA_ARCH__
    int32_t d;
    asm("dp2a.lo.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(u), "r"(acc));
    return d;
#else
    return acc + (int32_t)(int16_t)(a & 0xFFFFu) * (int32_t)(u & 0xFFu) +
           (int32_t)(int16_t)(a >> 16) * (int32_t)((u >> 8) & 0xFFu);
#endif
}

__host__ __device__ __forceinline__ int32_t dp2a_hi(uint32_t a, uint32_t u, int32_t acc) {
#ifdef __CUDA_ARCH__
    int32_t d;
    asm("dp2a.hi.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(u), "r"(acc));
    return d;
#else
    return acc + (int32_t)(int16_t)(a & 0xFFFFu) * (int32_t)((u >> 16) & 0xFFu) +
           (int32_t)(int16_t)(a >> 16) * (int32_t)(u >> 24);
#endif
}

// Digit planes of one activation block: word i of plane p holds the digits of
// elements 2i (low half) and 2i + 1 (high half); c0, c1 = -8 sum_j Dp_j.
struct XPlanes {
    uint32_t a0[16], a1[16];
    int32_t c0, c1;
};

// 16 sum_j (q_j - 8) X_j of one block from its 16 code bytes, as 4 words (word w
// holds bytes 4w..4w+3; byte m carries code 4w+m in its low nibble and code
// 16+4w+m in its high nibble). The high nibbles are multiplied in place (as
// bytes 16 q, no shift), so the low-nibble sums are scaled by 16 before the two
// are added: 16 Sp = 16 (sum_lo q Dp - 8 sum Dp) + sum_hi (16 q) Dp, with
// |16 S0| <= 2^27 and |16 S1| <= 2^26 (exact in binary32). Returned as binary32
// (one rounding).
__host__ __device__ __forceinline__ float block_dot16(const uint4 q, const XPlanes& x) {
    const uint32_t words[4] = {q.x, q.y, q.z, q.w};
    int32_t s0 = x.c0, s1 = x.c1, h0 = 0, h1 = 0;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        const uint32_t lo = words[w] & 0x0F0F0F0Fu;  // codes 4w .. 4w+3
        const uint32_t hi = words[w] & 0xF0F0F0F0u;  // 16 x codes 16+4w .. 16+4w+3
        s0 = dp2a_lo(x.a0[2 * w], lo, s0);
        s0 = dp2a_hi(x.a0[2 * w + 1], lo, s0);
        h0 = dp2a_lo(x.a0[8 + 2 * w], hi, h0);
        h0 = dp2a_hi(x.a0[9 + 2 * w], hi, h0);
        s1 = dp2a_lo(x.a1[2 * w], lo, s1);
        s1 = dp2a_hi(x.a1[2 * w + 1], lo, s1);
        h1 = dp2a_lo(x.a1[8 + 2 * w], hi, h1);
        h1 = dp2a_hi(x.a1[9 + 2 * w], hi, h1);
    }
    return fmaf((float)(s1 * 16 + h1), 65536.0f, (float)(s0 * 16 + h0));
}

// Quantise one block of 32 activations (host reference of the kernel's staging):
// fills the digit planes, returns the scale and whether the block is flagged.
__host__ __device__ inline bool xq_block(const float* x, XPlanes* out, float* scale) {
    uint32_t m = 0;
    for (int j = 0; j < 32; ++j) {
        const uint32_t b = f32_bits(x[j]) & 0x7FFFFFFFu;
        m = b > m ? b : m;
    }
    float s, inv;
    bool ok = xq_scale(m, &s, &inv);
    int32_t sum0 = 0, sum1 = 0;
    int32_t d0[32], d1[32];
    for (int j = 0; j < 32; ++j) {
        bool ej = true;
        const int32_t X = ok ? xq_int(x[j], inv, &ej) : 0;
        ok = ok && ej;
        x_digits16(X, &d0[j], &d1[j]);
        sum0 += d0[j];
        sum1 += d1[j];
    }
    for (int i = 0; i < 16; ++i) {
        out->a0[i] = pack16(d0[2 * i], d0[2 * i + 1]);
        out->a1[i] = pack16(d1[2 * i], d1[2 * i + 1]);
    }
    out->c0 = -8 * sum0;
    out->c1 = -8 * sum1;
    *scale = s;
    return !ok;
}

}  // namespace q4dev
