// The two memory-bound steps either side of the grouped GEMM in a routed MoE
// layer: SwiGLU over the gate_up rows, and the top-k combine of the down rows
// into one row per token (the decode glue of the status page "MoE Software
// Status & Known Limits", section "grouped-nf4-gemm", "Correctness contracts").
//
// Both kernels stream rows in 16-byte vectors (8 bf16): a thread owns one
// vector of the output per iteration, consecutive threads own consecutive
// vectors, and a grid of a few CTAs per SM strides over the whole output.
//
// SwiGLU: out[r, j] = bf16_rn( silu(gate) * up ), gate = h[r, j], up = h[r, I + j],
// silu(g) = g * sigmoid(g) in fp32 from e = exp(-|g|) (base-2 hardware exponential)
// and a fast division by 1 + e: about 2^-17 relative error before the bf16 rounding,
// about ten instructions per element, so that the kernel stays bound by HBM.
//
// Combine: out[t, n] = bf16_rn( acc ), acc an fp32 running sum that starts at +0
// and adds, for s = 0 .. k-1 in that order, the fp32 product w(t,s) * y[src(t,s), n]
// (product and sum each rounded once: __fmul_rn / __fadd_rn keep the compiler
// from fusing them). A token's result depends only on its own k slots, so it has
// the same bits whatever the number of tokens in the call.
#include <cstdint>
#include <cuda_runtime.h>

#include "gnf4_kernels.h"

namespace gnf4 {

namespace {

constexpr int kGlueThreads = 256;
constexpr int kGlueCtasPerSm = 8;      // 2048 threads per SM
constexpr int kSlotBatch = 8;          // slot loads issued before the in-order sum
constexpr int kSwigluVecs = 4;         // 16-byte vectors per thread per pass of the SwiGLU

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// two fp32 -> one bf16x2 word (lo in the low half), round to nearest even
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t d;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
    return d;
}

__device__ __forceinline__ uint32_t swiglu_word(uint32_t g, uint32_t u) {
    return pack_bf16x2(silu_mul(bf16_lo(g), bf16_lo(u)), silu_mul(bf16_hi(g), bf16_hi(u)));
}

// IDX is uint32_t when the vector count fits, so that the row/column split is a
// 32-bit division. Each thread takes kSwigluVecs vectors per pass, kGlueThreads
// apart, and issues all their loads before the first expf.
template <typename IDX>
__global__ void __launch_bounds__(kGlueThreads) swiglu_kernel(const uint4* __restrict__ h,
                                                              uint4* __restrict__ out,
                                                              IDX I8, IDX total) {
    const IDX stride = (IDX)gridDim.x * (kGlueThreads * kSwigluVecs);
    for (IDX base = (IDX)blockIdx.x * (kGlueThreads * kSwigluVecs) + threadIdx.x; base < total;
         base += stride) {
        uint4 g[kSwigluVecs], u[kSwigluVecs];
#pragma unroll
        for (int j = 0; j < kSwigluVecs; ++j) {
            const IDX i = base + (IDX)j * kGlueThreads;
            if (i < total) {
                const IDX r = i / I8;
                const IDX c = i - r * I8;
                const uint4* row = h + (int64_t)r * 2 * I8;
                g[j] = __ldg(row + c);
                u[j] = __ldg(row + I8 + c);
            }
        }
#pragma unroll
        for (int j = 0; j < kSwigluVecs; ++j) {
            const IDX i = base + (IDX)j * kGlueThreads;
            if (i < total) {
                uint4 o;
                o.x = swiglu_word(g[j].x, u[j].x);
                o.y = swiglu_word(g[j].y, u[j].y);
                o.z = swiglu_word(g[j].z, u[j].z);
                o.w = swiglu_word(g[j].w, u[j].w);
                out[i] = o;
            }
        }
    }
}

__device__ __forceinline__ void add_word(float* acc, uint32_t v, float wt, bool weighted) {
    const float a = bf16_lo(v), b = bf16_hi(v);
    acc[0] = __fadd_rn(acc[0], weighted ? __fmul_rn(wt, a) : a);
    acc[1] = __fadd_rn(acc[1], weighted ? __fmul_rn(wt, b) : b);
}

template <typename IDX, bool GATHER, bool WEIGHTED>
__global__ void __launch_bounds__(kGlueThreads) combine_kernel(const uint4* __restrict__ y,
                                                               const int32_t* __restrict__ src,
                                                               const float* __restrict__ wts,
                                                               uint4* __restrict__ out, IDX N8,
                                                               IDX total, int k, int64_t R) {
    const IDX stride = (IDX)gridDim.x * kGlueThreads;
    for (IDX i = (IDX)blockIdx.x * kGlueThreads + threadIdx.x; i < total; i += stride) {
        const IDX t = i / N8;
        const IDX c = i - t * N8;
        float acc[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[j] = 0.0f;
        const int64_t slot0 = (int64_t)t * k;
        for (int s0 = 0; s0 < k; s0 += kSlotBatch) {
            // issue the batch's loads first, then add them in slot order
            uint4 v[kSlotBatch];
            float wt[kSlotBatch];
            bool ok[kSlotBatch];
#pragma unroll
            for (int j = 0; j < kSlotBatch; ++j) {
                const int s = s0 + j;
                ok[j] = false;
                wt[j] = 1.0f;
                v[j] = make_uint4(0, 0, 0, 0);
                if (s < k) {
                    const int64_t r = GATHER ? (int64_t)__ldg(src + slot0 + s) : slot0 + s;
                    ok[j] = (r >= 0 && r < R);     // a dropped slot contributes nothing
                    if (ok[j]) v[j] = __ldg(y + r * N8 + c);
                    if (WEIGHTED) wt[j] = __ldg(wts + slot0 + s);
                }
            }
#pragma unroll
            for (int j = 0; j < kSlotBatch; ++j) {
                if (!ok[j]) continue;
                add_word(acc + 0, v[j].x, wt[j], WEIGHTED);
                add_word(acc + 2, v[j].y, wt[j], WEIGHTED);
                add_word(acc + 4, v[j].z, wt[j], WEIGHTED);
                add_word(acc + 6, v[j].w, wt[j], WEIGHTED);
            }
        }
        uint4 o;
        o.x = pack_bf16x2(acc[0], acc[1]);
        o.y = pack_bf16x2(acc[2], acc[3]);
        o.z = pack_bf16x2(acc[4], acc[5]);
        o.w = pack_bf16x2(acc[6], acc[7]);
        out[i] = o;
    }
}

int glue_grid(int64_t total, int per_thread = 1) {
    const int64_t per_cta = (int64_t)kGlueThreads * per_thread;
    const int64_t want = (total + per_cta - 1) / per_cta;
    const int64_t cap = (int64_t)device_sm_count() * kGlueCtasPerSm;
    return (int)(want < cap ? want : cap);
}

template <typename IDX>
cudaError_t launch_combine_t(const uint4* y, const int32_t* src, const float* w, uint4* out,
                             int64_t N8, int64_t total, int k, int64_t R, cudaStream_t s) {
    const int grid = glue_grid(total);
    if (src && w)
        combine_kernel<IDX, true, true><<<grid, kGlueThreads, 0, s>>>(y, src, w, out, (IDX)N8, (IDX)total, k, R);
    else if (src)
        combine_kernel<IDX, true, false><<<grid, kGlueThreads, 0, s>>>(y, src, w, out, (IDX)N8, (IDX)total, k, R);
    else if (w)
        combine_kernel<IDX, false, true><<<grid, kGlueThreads, 0, s>>>(y, src, w, out, (IDX)N8, (IDX)total, k, R);
    else
        combine_kernel<IDX, false, false><<<grid, kGlueThreads, 0, s>>>(y, src, w, out, (IDX)N8, (IDX)total, k, R);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_swiglu(const void* h, int64_t R, int64_t I, void* out, cudaStream_t s) {
    const int64_t I8 = I / 8, total = R * I8;
    if (total == 0) return cudaSuccess;
    const int grid = glue_grid(total, kSwigluVecs);
    const uint4* hv = reinterpret_cast<const uint4*>(h);
    uint4* ov = reinterpret_cast<uint4*>(out);
    // the 32-bit index path needs base + stride and base + (kSwigluVecs-1)*kGlueThreads to fit
    if (total <= (int64_t)UINT32_MAX - (int64_t)grid * kGlueThreads * kSwigluVecs)
        swiglu_kernel<uint32_t><<<grid, kGlueThreads, 0, s>>>(hv, ov, (uint32_t)I8, (uint32_t)total);
    else
        swiglu_kernel<int64_t><<<grid, kGlueThreads, 0, s>>>(hv, ov, I8, total);
    return cudaGetLastError();
}

cudaError_t launch_combine_topk(const void* y, int64_t R, int64_t N, const int32_t* row_of_slot,
                                const float* slot_weight, int64_t T, int64_t k, void* out,
                                cudaStream_t s) {
    const int64_t N8 = N / 8, total = T * N8;
    if (total == 0) return cudaSuccess;
    const uint4* yv = reinterpret_cast<const uint4*>(y);
    uint4* ov = reinterpret_cast<uint4*>(out);
    if (total <= (int64_t)UINT32_MAX - (int64_t)glue_grid(total) * kGlueThreads)
        return launch_combine_t<uint32_t>(yv, row_of_slot, slot_weight, ov, N8, total, (int)k, R, s);
    return launch_combine_t<int64_t>(yv, row_of_slot, slot_weight, ov, N8, total, (int)k, R, s);
}

}  // namespace gnf4
