// Register-level operand preparation of the batched tensor-core GEMV, compiled
// for the device and (for the host-side replay in q4_debug_check_tc) for the
// CPU from the same source.
//
// A operand: the 32 codes of one block become 16 words of bf16 pairs, the
// values (q - 8) exactly. A code nibble OR-ed into the bit pattern 0x4300 (bf16
// 128) gives the bf16 value 128 + q (q < 16 fits the 7 fraction bits at unit
// weight); subtracting bf16 136 leaves q - 8, exact since every value involved
// is a small integer. Column 2 i + s of chunk h2 holds nibble h2 of code bytes
// 4 i + s (low half) and 4 i + s + 2 (high half).
//
// B operand: each activation x is split into bf16 parts hi = rn(x) and
// lo = rn(x - hi); x - hi is exact in binary32 and |x - hi - lo| <= 2^-16 |x|.
// Eight consecutive elements e0..e7 fill one 16-byte core-matrix row in the
// position order of the A operand: (e0, e2), (e1, e3), (e4, e6), (e5, e7).
#pragma once

#include <cstdint>
#include <cstring>

#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace q4tm {

// bf16 bits of a binary32 value, round to nearest even (finite inputs).
__host__ __device__ __forceinline__ uint32_t bf16_bits_rn_host(float f) {
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (u + 0x7FFFu + ((u >> 16) & 1u)) >> 16;
}

__host__ __device__ __forceinline__ float bf16_value(uint32_t bits16) {
    const uint32_t u = bits16 << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

// One word of two bf16 values (q_lo - 8, q_hi - 8) from the nibbles at bits
// 0..3 and 16..19 of v (other bits ignored).
__host__ __device__ __forceinline__ uint32_t code_pair(uint32_t v) {
    const uint32_t m = (v & 0x000F000Fu) | 0x43004300u;
#ifdef __CUDA_ARCH__
    uint32_t r;
    asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(m), "r"(0x43084308u));
    return r;
#else
    // each half: bf16 (128 + q) - 136 = q - 8, an integer in [-8, 7], exact
    const float lo = bf16_value(m & 0xFFFFu) - 136.0f;
    const float hi = bf16_value(m >> 16) - 136.0f;
    return bf16_bits_rn_host(lo) | (bf16_bits_rn_host(hi) << 16);
#endif
}

// The 16 A-operand words (tensor-memory columns 0..15 of a slot) of one block.
__host__ __device__ __forceinline__ void dequant_block(const uint4 q, uint32_t (&a)[16]) {
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        a[2 * i] = code_pair(w[i]);               // low nibbles of bytes 4i, 4i+2
        a[2 * i + 1] = code_pair(w[i] >> 8);      // low nibbles of bytes 4i+1, 4i+3
        a[8 + 2 * i] = code_pair(w[i] >> 4);      // high nibbles of bytes 4i, 4i+2
        a[8 + 2 * i + 1] = code_pair(w[i] >> 12); // high nibbles of bytes 4i+1, 4i+3
    }
}

// bf16 pair word (a in the low half, b in the high half), round to nearest even.
__host__ __device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
#ifdef __CUDA_ARCH__
    const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    uint32_t u;
    memcpy(&u, &v, sizeof u);
    return u;
#else
    return bf16_bits_rn_host(a) | (bf16_bits_rn_host(b) << 16);
#endif
}

// hi and lo core-matrix rows of eight consecutive activations.
__host__ __device__ __forceinline__ void split_row(const float (&e)[8], uint4* hi, uint4* lo) {
    const float p[8] = {e[0], e[2], e[1], e[3], e[4], e[6], e[5], e[7]};
    uint32_t H[4], L[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        H[j] = pack_bf16(p[2 * j], p[2 * j + 1]);
        const float ra = p[2 * j] - bf16_value(H[j] & 0xFFFFu);   // exact
        const float rb = p[2 * j + 1] - bf16_value(H[j] >> 16);  // exact
        L[j] = pack_bf16(ra, rb);
    }
    *hi = make_uint4(H[0], H[1], H[2], H[3]);
    *lo = make_uint4(L[0], L[1], L[2], L[3]);
}

}  // namespace q4tm
