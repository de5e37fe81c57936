// Device helpers for the sm_100a Q4_0 kernels: shared-memory barriers, bulk
// (TMA engine) copies, programmatic dependent launch, bounded waits and the
// register-resident nibble unpack of the decode mat-vec.
#pragma once

#include <cstdint>
#include <cstring>
#include <cmath>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace q4dev {

// Time limit of every wait on an mbarrier (nanoseconds of %globaltimer). A wait
// that gives up records Q4_ERR_TIMEOUT in the workspace header and the kernel
// skips its math; copies of a few tens of KB normally land in microseconds.
constexpr uint64_t kWaitLimitNs = 20ull * 1000 * 1000;
// Longest a thread may sleep inside one try_wait before it re-checks the clock.
constexpr uint32_t kSuspendHintNs = 100000;

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
                 : "memory");
}

// Make a freshly initialised barrier visible to the async (TMA) proxy.
__device__ __forceinline__ void mbar_fence_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

// Returns true once the barrier's phase with the given parity has completed,
// false if it did not within kWaitLimitNs.
__device__ __forceinline__ bool mbar_try(uint32_t addr, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(done)
        : "r"(addr), "r"(parity), "r"(kSuspendHintNs)
        : "memory");
    return done != 0;
}

// Returns true once the barrier's phase with the given parity has completed,
// false if it did not within kWaitLimitNs. The clock is read only when the
// first try did not succeed.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity) {
    const uint32_t addr = smem_addr(bar);
    if (mbar_try(addr, parity)) return true;
    const uint64_t start = global_ns();
    while (true) {
        if (mbar_try(addr, parity)) return true;
        if (global_ns() - start > kWaitLimitNs) return false;
    }
}

// The same bounded wait with try_wait at the hardware's own short time limit (no
// suspend hint), so a waiting thread notices the phase change at once: for waits
// on the critical path of a pipeline.
__device__ __forceinline__ bool mbar_try_short(uint32_t addr, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(done)
        : "r"(addr), "r"(parity)
        : "memory");
    return done != 0;
}

__device__ __forceinline__ bool mbar_wait_short_bounded(uint64_t* bar, uint32_t parity) {
    const uint32_t addr = smem_addr(bar);
    if (mbar_try_short(addr, parity)) return true;
    const uint64_t start = global_ns();
    while (true) {
        if (mbar_try_short(addr, parity)) return true;
        if (global_ns() - start > kWaitLimitNs) return false;
    }
}

// Global -> shared bulk copy through the TMA engine, completing on `bar`.
// dst, src and bytes must be multiples of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes,
                                         uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(smem_addr(dst)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

// Bulk prefetch of [src, src + bytes) into L2 (no completion tracking). src and
// bytes must be multiples of 16.
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// Programmatic dependent launch: let the next kernel of the stream be scheduled,
// and wait for the previous kernel's completion and memory flush.
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__host__ __device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }

// Pairwise binary32 add / fused multiply-add: one packed f32x2 instruction on
// sm_100a, two scalar operations when the same code runs on the host.
__host__ __device__ __forceinline__ float2 add2(float2 a, float2 b) {
#ifdef __CUDA_ARCH__
    return __fadd2_rn(a, b);
#else
    return f2(a.x + b.x, a.y + b.y);
#endif
}

__host__ __device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
#ifdef __CUDA_ARCH__
    return __ffma2_rn(a, b, c);
#else
    return f2(fmaf(a.x, b.x, c.x), fmaf(a.y, b.y, c.y));
#endif
}

__host__ __device__ __forceinline__ float bits_f32(uint32_t u) {
#ifdef __CUDA_ARCH__
    return __uint_as_float(u);
#else
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
#endif
}

// The four weight pairs of one 32-bit word of codes, as exact binary32 (q - 8).
//
// A word holds bytes 4w..4w+3 of a block. Byte 4w+m carries weight 4w+m in its
// low nibble and weight 16+4w+m in its high nibble. A nibble at bit p of a
// binary32 significand (p <= 19, so that it stays clear of the exponent field at
// bits 23..30) becomes the value 2^(23-p) + q when OR-ed into the bit pattern of
// 2^(23-p): its bits land exactly on the units place. Subtracting 2^(23-p) + 8
// then gives q - 8 exactly. The nibbles at bits 20, 24 and 28 are read from the
// word shifted right by 12, where they sit at bits 8, 12 and 16.
//   lo01 = weights (4w,     4w+1)     bits 0, 8
//   lo23 = weights (4w+2,   4w+3)     bits 16, 24 (-> 12 after the shift)
//   hi01 = weights (16+4w,  16+4w+1)  bits 4, 12
//   hi23 = weights (16+4w+2, 16+4w+3) bits 20, 28 (-> 8, 16 after the shift)
struct Pairs {
    float2 lo01, lo23, hi01, hi23;
};

__host__ __device__ __forceinline__ float2 u64_f2(uint64_t v) {
    return f2(bits_f32((uint32_t)v), bits_f32((uint32_t)(v >> 32)));
}

// Each pair is formed by one 64-bit mask-and-OR whose two halves are single
// 32-bit logic operations writing the two registers of the pair directly.
__host__ __device__ __forceinline__ Pairs unpack_word(uint32_t q) {
    const uint32_t s = q >> 12;
    const uint64_t qq = ((uint64_t)q << 32) | q;
    const uint64_t sq = ((uint64_t)s << 32) | q;
    const uint64_t ss = ((uint64_t)s << 32) | s;
    Pairs p;
    // (2^23 + q, 2^15 + q)
    p.lo01 = add2(u64_f2((qq & 0x00000F000000000Full) | 0x470000004B000000ull),
                  f2(-8388616.0f, -32776.0f));
    // (2^7 + q, 2^11 + q)
    p.lo23 = add2(u64_f2((sq & 0x0000F000000F0000ull) | 0x4500000043000000ull),
                  f2(-136.0f, -2056.0f));
    // (2^19 + q, 2^11 + q)
    p.hi01 = add2(u64_f2((qq & 0x0000F000000000F0ull) | 0x4500000049000000ull),
                  f2(-524296.0f, -2056.0f));
    // (2^15 + q, 2^7 + q)
    p.hi23 = add2(u64_f2((ss & 0x000F000000000F00ull) | 0x4300000047000000ull),
                  f2(-32776.0f, -136.0f));
    return p;
}

// Constants of the register unpack: the magic exponents 2^23, 2^19, 2^15, 2^11,
// 2^7 and the four (2^e + 8) offset pairs, as bit patterns (held in registers).
struct UnpackConsts {
    uint32_t e23, e19, e15, e11, e7;
    unsigned long long lo01, lo23, hi01, hi23;
};

__host__ __device__ __forceinline__ UnpackConsts unpack_consts_default() {
    UnpackConsts k;
    k.e23 = 0x4B000000u;
    k.e19 = 0x49000000u;
    k.e15 = 0x47000000u;
    k.e11 = 0x45000000u;
    k.e7 = 0x43000000u;
    k.lo01 = 0xC7000800CB000008ull;  // (-(2^23 + 8), -(2^15 + 8))
    k.lo23 = 0xC5008000C3080000ull;  // (-(2^7 + 8),  -(2^11 + 8))
    k.hi01 = 0xC5008000C9000080ull;  // (-(2^19 + 8), -(2^11 + 8))
    k.hi23 = 0xC3080000C7000800ull;  // (-(2^15 + 8), -(2^7 + 8))
    return k;
}

// Sum over one block of (q - 8) * x, with x given as 8 float4 chunks (chunk i
// holds x[4i .. 4i+3] of the block), as two partial sums: binary32 products of
// the exact (q - 8) with x, two accumulator chains. On the device each pair is
// packed from two logic results and handled by one f32x2 add and one f32x2
// fused multiply-add; the host compiles the same arithmetic in C++ pairs (which
// the host-side unpack check exercises).
__host__ __device__ __forceinline__ float2 block_dot(const uint4 q, const float4 (&x)[8],
                                                     const UnpackConsts& k) {
    float2 acc = f2(0.0f, 0.0f);
    const uint32_t words[4] = {q.x, q.y, q.z, q.w};
    (void)k;
#if defined(__CUDA_ARCH__)
    unsigned long long a[2] = {0ull, 0ull};
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        const unsigned long long xlo01 = ((unsigned long long)__float_as_uint(x[w].y) << 32) | __float_as_uint(x[w].x);
        const unsigned long long xlo23 = ((unsigned long long)__float_as_uint(x[w].w) << 32) | __float_as_uint(x[w].z);
        const unsigned long long xhi01 = ((unsigned long long)__float_as_uint(x[w + 4].y) << 32) | __float_as_uint(x[w + 4].x);
        const unsigned long long xhi23 = ((unsigned long long)__float_as_uint(x[w + 4].w) << 32) | __float_as_uint(x[w + 4].z);
        asm("{\n"
            " .reg .b32 s, t0, t1;\n .reg .b64 p;\n"
            " shr.b32 s, %1, 12;\n"
            " lop3.b32 t0, %1, 0x0000000F, %6, 0xEA;\n"
            " lop3.b32 t1, %1, 0x00000F00, %8, 0xEA;\n"
            " mov.b64 p, {t0, t1};\n"
            " add.rn.f32x2 p, p, %11;\n fma.rn.f32x2 %0, p, %2, %0;\n"
            " lop3.b32 t0, %1, 0x000F0000, %10, 0xEA;\n"
            " lop3.b32 t1, s, 0x0000F000, %9, 0xEA;\n"
            " mov.b64 p, {t0, t1};\n"
            " add.rn.f32x2 p, p, %12;\n fma.rn.f32x2 %0, p, %3, %0;\n"
            " lop3.b32 t0, %1, 0x000000F0, %7, 0xEA;\n"
            " lop3.b32 t1, %1, 0x0000F000, %9, 0xEA;\n"
            " mov.b64 p, {t0, t1};\n"
            " add.rn.f32x2 p, p, %13;\n fma.rn.f32x2 %0, p, %4, %0;\n"
            " lop3.b32 t0, s, 0x00000F00, %8, 0xEA;\n"
            " lop3.b32 t1, s, 0x000F0000, %10, 0xEA;\n"
            " mov.b64 p, {t0, t1};\n"
            " add.rn.f32x2 p, p, %14;\n fma.rn.f32x2 %0, p, %5, %0;\n"
            "}\n"
            : "+l"(a[w & 1])
            : "r"(words[w]), "l"(xlo01), "l"(xlo23), "l"(xhi01), "l"(xhi23),
              "r"(k.e23), "r"(k.e19), "r"(k.e15), "r"(k.e11), "r"(k.e7),
              "l"(k.lo01), "l"(k.lo23), "l"(k.hi01), "l"(k.hi23));
    }
    acc = f2(__uint_as_float((uint32_t)a[0]) + __uint_as_float((uint32_t)a[1]),
             __uint_as_float((uint32_t)(a[0] >> 32)) + __uint_as_float((uint32_t)(a[1] >> 32)));
#else
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        const Pairs p = unpack_word(words[w]);
        acc = fma2(p.lo01, f2(x[w].x, x[w].y), acc);
        acc = fma2(p.lo23, f2(x[w].z, x[w].w), acc);
        acc = fma2(p.hi01, f2(x[w + 4].x, x[w + 4].y), acc);
        acc = fma2(p.hi23, f2(x[w + 4].z, x[w + 4].w), acc);
    }
#endif
    return acc;
}

#if defined(__CUDACC__)
// The four exact binary32 pairs (q - 8) of one code word, in the order block_dot
// uses them: (codes 4w, 4w+1), (4w+2, 4w+3), (16+4w, 16+4w+1), (16+4w+2,
// 16+4w+3) for word w of a block, each pair as the two halves of a 64-bit
// register (low half first). Several token rows reuse them.
__device__ __forceinline__ void code_pairs(uint32_t word, const UnpackConsts& k, uint64_t (&p)[4]) {
    asm("{\n"
        " .reg .b32 s, t0, t1;\n"
        " shr.b32 s, %4, 12;\n"
        " lop3.b32 t0, %4, 0x0000000F, %5, 0xEA;\n"
        " lop3.b32 t1, %4, 0x00000F00, %7, 0xEA;\n"
        " mov.b64 %0, {t0, t1};\n add.rn.f32x2 %0, %0, %10;\n"
        " lop3.b32 t0, %4, 0x000F0000, %9, 0xEA;\n"
        " lop3.b32 t1, s, 0x0000F000, %8, 0xEA;\n"
        " mov.b64 %1, {t0, t1};\n add.rn.f32x2 %1, %1, %11;\n"
        " lop3.b32 t0, %4, 0x000000F0, %6, 0xEA;\n"
        " lop3.b32 t1, %4, 0x0000F000, %8, 0xEA;\n"
        " mov.b64 %2, {t0, t1};\n add.rn.f32x2 %2, %2, %12;\n"
        " lop3.b32 t0, s, 0x00000F00, %7, 0xEA;\n"
        " lop3.b32 t1, s, 0x000F0000, %9, 0xEA;\n"
        " mov.b64 %3, {t0, t1};\n add.rn.f32x2 %3, %3, %13;\n"
        "}\n"
        : "=l"(p[0]), "=l"(p[1]), "=l"(p[2]), "=l"(p[3])
        : "r"(word), "r"(k.e23), "r"(k.e19), "r"(k.e15), "r"(k.e11), "r"(k.e7), "l"(k.lo01), "l"(k.lo23),
          "l"(k.hi01), "l"(k.hi23));
}

// c + a * b on both halves of 64-bit registers holding binary32 pairs.
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

__device__ __forceinline__ uint64_t pack2(float lo, float hi) {
    return ((uint64_t)__float_as_uint(hi) << 32) | __float_as_uint(lo);
}

// Sum of the four binary32 values in two pairs: (a.lo + b.lo) + (a.hi + b.hi).
__device__ __forceinline__ float sum_pairs(uint64_t a, uint64_t b) {
    return (__uint_as_float((uint32_t)a) + __uint_as_float((uint32_t)b)) +
           (__uint_as_float((uint32_t)(a >> 32)) + __uint_as_float((uint32_t)(b >> 32)));
}
#endif

}  // namespace q4dev
