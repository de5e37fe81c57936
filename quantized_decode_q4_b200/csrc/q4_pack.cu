// Q4_0 pack and dequant kernels for sm_100a.
//
// Pack: the "Q4 packer" of "MicroLLM Lab" (introduction), run once before
// decode: 16-bit-class weights become 4 bits per parameter ("Seven models, all
// in Q4"). Every binary32 step is an explicit round-to-nearest intrinsic, so no
// multiply-add contraction can move a code across a rounding boundary.
// Dequant: the dequantised tile of the mat-mat path ("Llamas on the Web",
// section 3), written out; w = d * (q - 8) is exact in binary32.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace q4k {

__device__ __forceinline__ uint32_t q4_code(float w, float inv_d) {
    const float t = __fadd_rn(__fmul_rn(w, inv_d), 8.5f);
    int c = static_cast<int>(floorf(t));
    c = c < 0 ? 0 : (c > 15 ? 15 : c);
    return static_cast<uint32_t>(c);
}

// One thread per block of 32 weights. Block i is row i / nb, block i % nb, so
// its codes go to qs + 16 i and its scale to d[i] in the row-major planes.
__global__ void __launch_bounds__(256) pack_kernel(const float* __restrict__ w,
                                                   uint8_t* __restrict__ qs,
                                                   uint16_t* __restrict__ d, int64_t nblocks) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nblocks; i += stride) {
        const float4* src = reinterpret_cast<const float4*>(w) + i * 8;
        float v[32];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const float4 t = src[c];
            v[4 * c + 0] = t.x;
            v[4 * c + 1] = t.y;
            v[4 * c + 2] = t.z;
            v[4 * c + 3] = t.w;
        }
        // signed weight of largest magnitude; strict '>' keeps the lowest index
        float amax = 0.0f, m = 0.0f;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const float a = fabsf(v[j]);
            if (a > amax) {
                amax = a;
                m = v[j];
            }
        }
        const float dd = __fdiv_rn(m, -8.0f);
        const float inv = dd != 0.0f ? __frcp_rn(dd) : 0.0f;
        uint32_t words[4] = {0u, 0u, 0u, 0u};
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const uint32_t byte = q4_code(v[j], inv) | (q4_code(v[j + 16], inv) << 4);
            words[j >> 2] |= byte << (8 * (j & 3));
        }
        reinterpret_cast<uint4*>(qs)[i] = make_uint4(words[0], words[1], words[2], words[3]);
        d[i] = __half_as_ushort(__float2half_rn(dd));
    }
}

// Eight threads per block, each writing four consecutive outputs as one 16-byte
// store, so a warp writes 512 contiguous bytes (four blocks). Thread g of a block
// writes outputs 4g .. 4g+3: for g < 4 these are the low nibbles of code word g,
// for g >= 4 the high nibbles of code word g - 4 (byte m of a word carries
// output 4w+m in its low nibble and output 16+4w+m in its high nibble).
__global__ void __launch_bounds__(256) dequant_kernel(const uint8_t* __restrict__ qs,
                                                      const uint16_t* __restrict__ d,
                                                      float* __restrict__ out, int64_t nblocks) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    const int64_t total = nblocks * 8;
    for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < total; t += stride) {
        const int64_t i = t >> 3;
        const int g = (int)(t & 7);
        const uint32_t word = reinterpret_cast<const uint32_t*>(qs)[i * 4 + (g & 3)];
        const uint32_t nib = g < 4 ? word : word >> 4;
        const float s = __half2float(__ushort_as_half(d[i]));
        float v[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) v[m] = __fmul_rn(s, (float)((int)((nib >> (8 * m)) & 0xFu) - 8));
        reinterpret_cast<float4*>(out)[t] = make_float4(v[0], v[1], v[2], v[3]);
    }
}

// Grids of at most 64 CTAs of 256 threads per multiprocessor (grid-stride loops).
cudaError_t launch_pack(const float* w, uint8_t* qs, uint16_t* d, int64_t nblocks, int num_sms,
                        cudaStream_t stream) {
    const int threads = 256;
    int64_t blocks = (nblocks + threads - 1) / threads;
    if (blocks > (int64_t)num_sms * 64) blocks = (int64_t)num_sms * 64;
    pack_kernel<<<(unsigned)blocks, threads, 0, stream>>>(w, qs, d, nblocks);
    return cudaGetLastError();
}

cudaError_t launch_dequant(const uint8_t* qs, const uint16_t* d, float* out, int64_t nblocks,
                           int num_sms, cudaStream_t stream) {
    const int threads = 256;
    int64_t blocks = (nblocks * 8 + threads - 1) / threads;
    if (blocks > (int64_t)num_sms * 64) blocks = (int64_t)num_sms * 64;
    dequant_kernel<<<(unsigned)blocks, threads, 0, stream>>>(qs, d, out, nblocks);
    return cudaGetLastError();
}

}  // namespace q4k
