// Decode band of the grouped 4-bit GEMM: groups with few routed rows, where the
// packed weight bytes are the whole cost (the GEMV path of the solution page
// "How do I run a grouped GEMM directly on NF4 packed MoE expert weights,
// without dequantizing to bf16 first?", "Supported scope": one-token groups
// take the GEMV path).
//
// Work item = (active expert, 16 weight rows). A CTA of 8 warps takes one item
// at a time and splits K across its warps; each warp streams its share of the
// item's packed bytes straight from HBM into registers, decodes the nibbles with
// byte permutes (no shared-memory table), and multiplies through warp-level
// bf16 MMAs with the weights as the 16-row M side and up to 8 routed rows per
// MMA as the N side. Each MMA chain covers exactly one scale block (64 K for
// NF4, 32 K for MXFP4), so the block sum comes out of the tensor core in fp32
// and is scaled and accumulated in fp32 outside it. The 8 warp partials are
// summed in a fixed order through shared memory (deterministic), weighted, and
// stored as bf16 at the destination rows.
//
// MMA k-slot mapping: in m16n8k16, lane (g, t) supplies k-slots 2t, 2t+1,
// 2t+8, 2t+9 of both operands. Those slots are mapped to the four consecutive K
// positions base + (SB/4)*t + 4*s + {0,1,2,3} of step s, the same for A and B,
// so each lane reads contiguous bytes of the packed rows and of the activation
// rows.
#include <climits>
#include <cstdint>
#include <cuda_runtime.h>

#include "gnf4_common.cuh"
#include "gnf4_kernels.h"

namespace gnf4 {

constexpr int kDecodeWarps = 8;
constexpr int kMaxExperts = 2048;

template <int FMT, int GMAX>
__global__ void __launch_bounds__(kDecodeWarps * 32) decode_band_kernel(const GroupedArgs p) {
    constexpr int SB = (FMT == FMT_NF4) ? 64 : 32;   // K elements per scale block
    constexpr int STEPS = SB / 16;                   // k16 MMA steps per block
    constexpr int WPR = SB / 32;                     // packed words per lane per row per block
    constexpr int XW = SB / 8;                       // bf16x2 words of x per lane per block
    constexpr int CH = (FMT == FMT_NF4) ? 4 : 8;     // blocks loaded ahead per warp

    __shared__ int s_active[kMaxExperts];
    __shared__ int s_nact;
    __shared__ float4 s_red[kDecodeWarps][GMAX][32];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;

    // experts of this band, in id order (every CTA derives the same list)
    if (warp == 0) {
        int count = 0;
        for (int e0 = 0; e0 < p.E; e0 += 32) {
            const int e = e0 + lane;
            bool act = false;
            if (e < p.E) {
                const int64_t m = p.offsets[e + 1] - p.offsets[e];
                act = (m >= p.m_lo) && (m <= p.m_hi);
            }
            const unsigned bal = __ballot_sync(0xffffffffu, act);
            if (act) s_active[count + __popc(bal & ((1u << lane) - 1u))] = e;
            count += __popc(bal);
        }
        if (lane == 0) s_nact = count;
    }
    __syncthreads();

    const int nt = p.N >> 4;
    const int total = s_nact * nt;
    const int nb = p.K / SB;
    const int kb0 = warp * nb / kDecodeWarps;
    const int kb1 = (warp + 1) * nb / kDecodeWarps;
    const int64_t rowbytes = p.K >> 1;

    for (int item = blockIdx.x; item < total; item += gridDim.x) {
        const int e = s_active[item / nt];
        const int n0 = (item % nt) << 4;
        const int64_t r0 = p.offsets[e];
        const int m = (int)(p.offsets[e + 1] - r0);
        const int64_t row_g = (int64_t)e * p.N + n0 + g;          // weight row of lane group g
        const uint8_t* wp0 = p.W + row_g * rowbytes + t * (WPR * 4);
        const uint8_t* wp1 = wp0 + 8 * rowbytes;                   // row g + 8
        const int64_t sc0 = row_g * nb;
        const int64_t sc1 = sc0 + 8 * (int64_t)nb;

        for (int mc = 0; mc < m; mc += 8 * GMAX) {
            const int G = min(GMAX, (m - mc + 7) >> 3);
            const uint16_t* xr[GMAX];
#pragma unroll
            for (int j = 0; j < GMAX; ++j) {
                const int rr = mc + 8 * j + g;
                xr[j] = nullptr;
                if (j < G && rr < m) {
                    const int64_t r = r0 + rr;
                    const int64_t tk = p.row_token ? (int64_t)p.row_token[r] : r;
                    xr[j] = p.x + tk * p.K + t * (SB / 4);
                }
            }
            float acc[GMAX][4];
#pragma unroll
            for (int j = 0; j < GMAX; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;

            for (int kc = kb0; kc < kb1; kc += CH) {
                uint32_t a0[CH][WPR], a1[CH][WPR];
                float s0[CH], s1[CH];
#pragma unroll
                for (int c = 0; c < CH; ++c) {
                    const int b = kc + c;
                    if (b < kb1) {
                        if constexpr (WPR == 2) {
                            const uint2 u0 = __ldg(reinterpret_cast<const uint2*>(wp0 + b * (SB / 2)));
                            const uint2 u1 = __ldg(reinterpret_cast<const uint2*>(wp1 + b * (SB / 2)));
                            a0[c][0] = u0.x; a0[c][WPR - 1] = u0.y;
                            a1[c][0] = u1.x; a1[c][WPR - 1] = u1.y;
                        } else {
                            a0[c][0] = __ldg(reinterpret_cast<const uint32_t*>(wp0 + b * (SB / 2)));
                            a1[c][0] = __ldg(reinterpret_cast<const uint32_t*>(wp1 + b * (SB / 2)));
                        }
                        s0[c] = load_scale<FMT>(p.scales, sc0 + b);
                        s1[c] = load_scale<FMT>(p.scales, sc1 + b);
                    } else {
#pragma unroll
                        for (int q = 0; q < WPR; ++q) a0[c][q] = a1[c][q] = 0u;
                        s0[c] = s1[c] = 0.f;
                    }
                }
#pragma unroll
                for (int c = 0; c < CH; ++c) {
                    const int b = kc + c;
                    if (b < kb1) {
                        uint32_t d0[4 * WPR], d1[4 * WPR];
#pragma unroll
                        for (int q = 0; q < WPR; ++q) {
                            uint32_t o[4];
                            decode_word<FMT>(a0[c][q], p.lut, o);
                            d0[4 * q + 0] = o[0]; d0[4 * q + 1] = o[1];
                            d0[4 * q + 2] = o[2]; d0[4 * q + 3] = o[3];
                            decode_word<FMT>(a1[c][q], p.lut, o);
                            d1[4 * q + 0] = o[0]; d1[4 * q + 1] = o[1];
                            d1[4 * q + 2] = o[2]; d1[4 * q + 3] = o[3];
                        }
#pragma unroll
                        for (int j = 0; j < GMAX; ++j) {
                            if (j < G) {
                                uint32_t xw[XW];
                                if (xr[j] != nullptr) {
#pragma unroll
                                    for (int q = 0; q < XW / 4; ++q) {
                                        const uint4 v = __ldg(reinterpret_cast<const uint4*>(xr[j] + b * SB) + q);
                                        xw[4 * q + 0] = v.x; xw[4 * q + 1] = v.y;
                                        xw[4 * q + 2] = v.z; xw[4 * q + 3] = v.w;
                                    }
                                } else {
#pragma unroll
                                    for (int q = 0; q < XW; ++q) xw[q] = 0u;
                                }
                                float cb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                                for (int s = 0; s < STEPS; ++s)
                                    mma_bf16_16816(cb, d0[2 * s], d1[2 * s], d0[2 * s + 1], d1[2 * s + 1],
                                                   xw[2 * s], xw[2 * s + 1]);
                                acc[j][0] = fmaf(cb[0], s0[c], acc[j][0]);
                                acc[j][1] = fmaf(cb[1], s0[c], acc[j][1]);
                                acc[j][2] = fmaf(cb[2], s1[c], acc[j][2]);
                                acc[j][3] = fmaf(cb[3], s1[c], acc[j][3]);
                            }
                        }
                    }
                }
            }

            // sum the 8 warp partials in a fixed order, then the epilogue
#pragma unroll
            for (int j = 0; j < GMAX; ++j)
                if (j < G) s_red[warp][j][lane] = make_float4(acc[j][0], acc[j][1], acc[j][2], acc[j][3]);
            __syncthreads();
            for (int q = threadIdx.x; q < G * 128; q += kDecodeWarps * 32) {
                const int j = q >> 7, ln = (q >> 2) & 31, i = q & 3;
                float v = 0.f;
#pragma unroll
                for (int w = 0; w < kDecodeWarps; ++w) v += reinterpret_cast<const float*>(&s_red[w][j][ln])[i];
                const int slot = mc + 8 * j + 2 * (ln & 3) + (i & 1);   // C column 2t (+1)
                if (slot < m) {
                    const int64_t r = r0 + slot;
                    if (p.row_weight) v *= __ldg(p.row_weight + r);
                    const int64_t dst = p.row_dest ? (int64_t)p.row_dest[r] : r;
                    const int n = n0 + (ln >> 2) + ((i & 2) ? 8 : 0);      // C row g (+8)
                    p.out[dst * p.N + n] = f32_to_bf16_rne(v);
                }
            }
            __syncthreads();
        }
    }
}

template <int FMT, int GMAX>
static cudaError_t launch_db(const GroupedArgs& a, cudaStream_t s) {
    static int per_sm = -1;
    if (per_sm < 0) {
        cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(
            &per_sm, decode_band_kernel<FMT, GMAX>, kDecodeWarps * 32, 0);
        if (e != cudaSuccess) return e;
        if (per_sm < 1) per_sm = 1;
    }
    const int64_t groups_max = a.R < (int64_t)a.E ? a.R : (int64_t)a.E;
    const int64_t items_max = groups_max * (a.N / 16);
    int64_t grid = (int64_t)device_sm_count() * per_sm;
    if (items_max < grid) grid = items_max;
    if (grid < 1) return cudaSuccess;
    decode_band_kernel<FMT, GMAX><<<(unsigned)grid, kDecodeWarps * 32, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_decode_band(int fmt, const GroupedArgs& a, cudaStream_t s) {
    const int64_t mmax = a.R < (int64_t)a.m_hi ? a.R : (int64_t)a.m_hi;   // no group exceeds this
    if (fmt == FMT_NF4) {
        if (mmax <= 8) return launch_db<FMT_NF4, 1>(a, s);
        if (mmax <= 16) return launch_db<FMT_NF4, 2>(a, s);
        return launch_db<FMT_NF4, 4>(a, s);
    }
    if (mmax <= 8) return launch_db<FMT_MXFP4, 1>(a, s);
    if (mmax <= 16) return launch_db<FMT_MXFP4, 2>(a, s);
    return launch_db<FMT_MXFP4, 4>(a, s);
}

}  // namespace gnf4
