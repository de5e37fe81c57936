// Integer dot product of Q4_0 codes with activations held in 24-bit block fixed
// point: the register-level core of the batch-1 streaming kernel.
//
// Activations of one block of 32 are written x_j ~= s * X_j with one binary32
// scale s = max_j |x_j| / kXMax and integers |X_j| <= kXMax, split into three
// signed 8-bit digits X_j = 65536 a_j + 256 b_j + c_j (each digit in -128..127).
// For codes q_j in 0..15 the block sum is then exact in integers:
//   sum_j (q_j - 8) X_j = 65536 A + 256 B + C,
//   A = sum_j a_j q_j - 8 sum_j a_j   (likewise B, C),
// and each sum_j digit_j q_j is a chain of dp4a instructions on 4 codes at a
// time (the low nibbles of a code word are 4 codes, the high nibbles 4 more).
// The only approximation is x ~= s X: |x_j - s X_j| <= s / 2 (plus one binary32
// rounding of x_j / s), i.e. at most max|x| / (2 kXMax) = 2^-24 max|x| per
// element of the block.
#pragma once

#include <cstdint>
#include <cmath>
#include <cstring>

#include <cuda_runtime.h>

namespace q4dev {

// Largest |X| whose three balanced base-256 digits all lie in -128..127.
constexpr int32_t kXMax = 127 * 65536 + 127 * 256 + 127;  // 8,355,711

// Split an integer |X| <= kXMax into digits a, b, c in -128..127 with
// X = 65536 a + 256 b + c.
__host__ __device__ __forceinline__ void x_digits(int32_t X, int32_t* a, int32_t* b, int32_t* c) {
    const int32_t lo = ((X + 128) & 255) - 128;
    const int32_t y = (X - lo) >> 8;
    const int32_t mid = ((y + 128) & 255) - 128;
    *c = lo;
    *b = mid;
    *a = (y - mid) >> 8;
}

// Blocks whose largest |x| is below this are taken as zero (the reciprocal of
// the scale would overflow binary32; the absolute error is below 1e-30 per code
// step).
constexpr float kXTiny = 1e-30f;

// Scale of a block whose largest |x| is maxabs, and its reciprocal (both one
// binary32 rounding; a zero or tiny block has scale 0 and all X = 0).
__host__ __device__ __forceinline__ float xq_scale(float maxabs) {
    return maxabs >= kXTiny ? maxabs / (float)kXMax : 0.0f;
}
__host__ __device__ __forceinline__ float xq_inv(float maxabs) {
    return maxabs >= kXTiny ? (float)kXMax / maxabs : 0.0f;
}

// X = round-to-nearest-even(x / s), clamped to +-kXMax.
__host__ __device__ __forceinline__ int32_t xq_int(float x, float inv) {
    const float t = x * inv;
#ifdef __CUDA_ARCH__
    int32_t X = __float2int_rn(t);
#else
    int32_t X = (int32_t)nearbyintf(t);
#endif
    return X > kXMax ? kXMax : (X < -kXMax ? -kXMax : X);
}

// Sum over 4 byte lanes of (unsigned byte of u) * (signed byte of s), plus acc.
__host__ __device__ __forceinline__ int32_t dp4a_us(uint32_t u, uint32_t s, int32_t acc) {
#ifdef __CUDA_ARCH__
    int32_t d;
    asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(u), "r"(s), "r"(acc));
    return d;
#else
    for (int i = 0; i < 4; ++i)
        acc += (int32_t)((u >> (8 * i)) & 0xFFu) * (int32_t)(int8_t)((s >> (8 * i)) & 0xFFu);
    return acc;
#endif
}

// Digit words of one activation block: word w of digit plane p holds the digits
// of elements 4w..4w+3 (one per byte, element 4w in the low byte).
struct XDigits {
    uint32_t a[8], b[8], c[8];
};

// sum_j (q_j - 8) X_j for one block, from its 16 code bytes (as 4 words: word w
// holds bytes 4w..4w+3; byte m carries code 4w+m in its low nibble and code
// 16+4w+m in its high nibble) and the block's correction terms
// ca = -8 sum a_j, cb = -8 sum b_j, cc = -8 sum c_j. Returned as binary32
// (65536 A + 256 B + C, one rounding).
__host__ __device__ __forceinline__ float block_dot_int(const uint4 q, const XDigits& x, int32_t ca,
                                                        int32_t cb, int32_t cc) {
    const uint32_t words[4] = {q.x, q.y, q.z, q.w};
    // two chains per digit plane (low and high nibbles) halve the dependent
    // dp4a chain length
    int32_t A = ca, B = cb, C = cc, A2 = 0, B2 = 0, C2 = 0;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        const uint32_t lo = words[w] & 0x0F0F0F0Fu;         // codes 4w .. 4w+3
        const uint32_t hi = (words[w] >> 4) & 0x0F0F0F0Fu;  // codes 16+4w .. 16+4w+3
        A = dp4a_us(lo, x.a[w], A);
        A2 = dp4a_us(hi, x.a[w + 4], A2);
        B = dp4a_us(lo, x.b[w], B);
        B2 = dp4a_us(hi, x.b[w + 4], B2);
        C = dp4a_us(lo, x.c[w], C);
        C2 = dp4a_us(hi, x.c[w + 4], C2);
    }
    A += A2;
    B += B2;
    C += C2;
    return fmaf((float)A, 65536.0f, fmaf((float)B, 256.0f, (float)C));
}

}  // namespace q4dev
