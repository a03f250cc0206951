// NF4 and MXFP4 quantizers (test-input generation). One warp per 64 K elements:
// each lane owns two neighbouring elements, i.e. one output byte.
//
// NF4 follows the grouped-nf4-gemm README (0.11.0), "Try it on CPU right now",
// block 1; MXFP4 block 2 of the same section. The rounding steps are fixed so
// that the bytes equal the CPU oracle's bit for bit: IEEE fp32 division for the
// NF4 normalisation, exact power-of-two scaling for MXFP4.
#include <cstdint>
#include <cuda_runtime.h>

#include "gnf4_common.cuh"
#include "gnf4_kernels.h"

namespace gnf4 {

// NF4 values (QLoRA NF4 / bitsandbytes NF4), fp32, ascending.
__constant__ float c_nf4[16] = {
    -1.0f, -0.6961928009986877f, -0.5250730514526367f, -0.39491748809814453f,
    -0.28444138169288635f, -0.18477343022823334f, -0.09105003625154495f, 0.0f,
    0.07958029955625534f, 0.16093020141124725f, 0.24611230194568634f,
    0.33791524171829224f, 0.44070982933044434f, 0.5626170039176941f,
    0.7229568362236023f, 1.0f};

__device__ __forceinline__ uint32_t nf4_code(float x) {
    // nearest NF4 value, ties to the lower code: count fp32 midpoints below x
    uint32_t code = 0;
#pragma unroll
    for (int i = 0; i < 15; ++i) {
        const float mid = __fmul_rn(__fadd_rn(c_nf4[i], c_nf4[i + 1]), 0.5f);
        code += (x > mid) ? 1u : 0u;
    }
    return code;
}

__global__ void __launch_bounds__(256) quantize_nf4_kernel(const float* __restrict__ w,
                                                           int64_t nblocks, int64_t K,
                                                           uint8_t* __restrict__ packed,
                                                           float* __restrict__ absmax) {
    const int64_t blk = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (blk >= nblocks) return;
    const int lane = threadIdx.x & 31;
    const float2 v = __ldg(reinterpret_cast<const float2*>(w + blk * 64) + lane);
    float a = fmaxf(fabsf(v.x), fabsf(v.y));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    uint32_t c0 = 7u, c1 = 7u;                   // all-zero block: code 7 (0.0)
    if (a > 0.0f) {
        c0 = nf4_code(__fdiv_rn(v.x, a));
        c1 = nf4_code(__fdiv_rn(v.y, a));
    }
    packed[blk * 32 + lane] = (uint8_t)((c0 << 4) | c1);   // element 2j in the high nibble
    if (lane == 0) absmax[blk] = a;
    (void)K;
}

__device__ __forceinline__ uint32_t e2m1_code(float w, float inv_scale) {
    // |w| * 2^-E is exact for every normal result; results below 2^-126 give code 0
    const float a = fabsf(w) * inv_scale;
    uint32_t c = 0;
    c += (a > 0.25f) ? 1u : 0u;    // ties between codes i and i+1 go to the even code
    c += (a >= 0.75f) ? 1u : 0u;
    c += (a > 1.25f) ? 1u : 0u;
    c += (a >= 1.75f) ? 1u : 0u;
    c += (a > 2.5f) ? 1u : 0u;
    c += (a >= 3.5f) ? 1u : 0u;
    c += (a > 5.0f) ? 1u : 0u;     // and everything above 6 saturates to code 7
    return c | ((w < 0.0f) ? 8u : 0u);
}

__global__ void __launch_bounds__(256) quantize_mxfp4_kernel(const float* __restrict__ w,
                                                             int64_t nblocks32,
                                                             uint8_t* __restrict__ blocks,
                                                             uint8_t* __restrict__ scales) {
    // a warp covers two 32-element blocks; lanes 0..15 the first, 16..31 the second
    const int64_t pair = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    const int64_t blk = pair * 2 + (lane >> 4);
    const bool live = blk < nblocks32;
    float2 v = make_float2(0.f, 0.f);
    if (live) v = __ldg(reinterpret_cast<const float2*>(w + blk * 32) + (lane & 15));
    float a = fmaxf(fabsf(v.x), fabsf(v.y));
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    if (!live) return;
    // E = floor(log2 amax) - 2 from the exponent field, clamped to [-127, 127]
    const int ef = (int)((__float_as_uint(a) >> 23) & 0xFFu);
    int E = (ef > 0) ? ef - 127 - 2 : -127;
    E = max(-127, min(127, E));
    if (a == 0.0f) E = 0;
    const float inv = __uint_as_float((uint32_t)(127 - E) << 23);   // 2^-E, E in [-127, 125]
    const uint32_t c0 = e2m1_code(v.x, inv), c1 = e2m1_code(v.y, inv);
    blocks[blk * 16 + (lane & 15)] = (uint8_t)(c0 | (c1 << 4));      // element 2j in the low nibble
    if ((lane & 15) == 0) scales[blk] = (uint8_t)(E + 127);
}

cudaError_t launch_quantize_nf4(const float* w, int64_t rows, int64_t K, uint8_t* packed,
                                float* absmax, cudaStream_t s) {
    const int64_t nblocks = rows * (K / 64);
    if (nblocks == 0) return cudaSuccess;
    const int64_t grid = (nblocks + 7) / 8;
    quantize_nf4_kernel<<<(unsigned)grid, 256, 0, s>>>(w, nblocks, K, packed, absmax);
    return cudaGetLastError();
}

cudaError_t launch_quantize_mxfp4(const float* w, int64_t rows, int64_t K, uint8_t* blocks,
                                  uint8_t* scales, cudaStream_t s) {
    const int64_t nb = rows * (K / 32);
    if (nb == 0) return cudaSuccess;
    const int64_t pairs = (nb + 1) / 2;
    const int64_t grid = (pairs + 7) / 8;
    quantize_mxfp4_kernel<<<(unsigned)grid, 256, 0, s>>>(w, nb, blocks, scales);
    return cudaGetLastError();
}

}  // namespace gnf4
