// Decode band of the grouped 4-bit GEMM: groups with few routed rows, where
// the packed weight bytes are the whole cost (the GEMV path of the solution page
// "How do I run a grouped GEMM directly on NF4 packed MoE expert weights,
// without dequantizing to bf16 first?", "Supported scope": one-token groups
// take the GEMV path).
//
// Work item = (active expert, 16 weight rows); each CTA takes a contiguous run
// of items (consecutive items share an expert, so its activation rows stay in
// L1). One producer warp streams every item's packed rows into a ring of
// shared-memory stages with 1-D bulk copies (cp.async.bulk, completion counted
// on an mbarrier), several items ahead of the consumers, so HBM sees many
// bytes in flight per SM regardless of what the consumers are doing. Eight
// consumer warps split each stage's K range; each decodes the nibbles with byte
// permutes (tables in registers) and multiplies through warp-level bf16 MMAs
// with the 16 weight rows as the M side and up to 8 routed rows per MMA as the
// N side. Every MMA chain covers exactly one scale block (64 K for NF4, 32 K for
// MXFP4), so the block sum leaves the tensor core in fp32 and is scaled and
// accumulated in fp32 outside it. The 8 warp partials are summed in a fixed
// order through shared memory (deterministic), weighted, rounded to bf16 and
// stored at the destination rows.
//
// MMA k-slot mapping: in m16n8k16, lane (g, t) supplies k-slots 2t, 2t+1,
// 2t+8, 2t+9 of both operands. They are mapped to the four consecutive K
// positions base + (SB/4)*t + 4*s + {0,1,2,3} of step s, the same for A and
// B, so each lane reads contiguous bytes of the packed rows and of x.
#include <climits>
#include <cstdint>
#include <cuda_runtime.h>

#include "gnf4_common.cuh"
#include "gnf4_kernels.h"

namespace gnf4 {

__device__ unsigned g_decode_error;

namespace db {

constexpr int kConsumers = 8;                    // consumer warps
constexpr int kThreads = (kConsumers + 1) * 32;  // + one producer warp
constexpr int kMaxExperts = 2048;
constexpr int kBlocksPerStage = 32;              // scale blocks per stage (4 per consumer warp)
constexpr long long kTimeoutCycles = 1LL << 32;

struct Plan {
    int kch;          // K elements per stage (a multiple of the scale block)
    int nch;          // stages per item pass
    int row_stride;   // bytes per weight row in a stage (chunk bytes + 16 of padding)
    int stage_bytes;  // 16 rows
    int nstages;
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
    return ok != 0;
}
// bounded wait: false after ~2^32 cycles (error recorded) or once another warp gave up
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
    if (mbar_try(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
        if (mbar_try(bar, parity)) return true;
        if (*abort_flag) return false;
        if (clock64() - t0 > kTimeoutCycles) {
            *abort_flag = 1;
            atomicOr(&g_decode_error, 1u);
            return false;
        }
    }
}

struct Pos {
    int item, pass, kc;
};

}  // namespace db

template <int FMT, int GMAX>
__global__ void __maxnreg__(112) decode_band_kernel(const GroupedArgs p, const db::Plan plan) {
    using namespace db;
    constexpr int SB = (FMT == FMT_NF4) ? 64 : 32;   // K elements per scale block
    constexpr int STEPS = SB / 16;                   // k16 MMA steps per block
    constexpr int BPL = SB / 8;                      // packed bytes per lane per row per block (8 or 4)
    constexpr int XW = SB / 8;                       // bf16x2 words of x per lane per block
    constexpr int BPW = kBlocksPerStage / kConsumers;  // blocks per consumer warp per stage (4)

    extern __shared__ __align__(128) uint8_t smem[];
    // layout: [stages][16 rows][row_stride] | red[8][GMAX][32] float4 | barriers | lists
    float4* red = reinterpret_cast<float4*>(smem + plan.nstages * plan.stage_bytes);
    uint8_t* tail = smem + plan.nstages * plan.stage_bytes + kConsumers * GMAX * 32 * sizeof(float4);
    uint64_t* bars = reinterpret_cast<uint64_t*>(tail);                 // full[ns], empty[ns]
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tail + 16 * 8 * 2);
    int* s_nact = reinterpret_cast<int*>(tail + 16 * 8 * 2 + 16);
    int* s_active = s_nact + 4;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ns = plan.nstages;

    if (warp == 0) {
        // experts of this band, in id order (every CTA derives the same list)
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
        if (lane == 0) s_nact[0] = count;
    } else if (warp == kConsumers && lane == 0) {
        for (int i = 0; i < ns; ++i) {
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(bars + i)) : "memory");
            asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bars + 16 + i)),
                         "r"(kConsumers) : "memory");
        }
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    const int nt = p.N >> 4;
    const int total = s_nact[0] * nt;
    const int i0 = (int)((int64_t)blockIdx.x * total / gridDim.x);
    const int i1 = (int)((int64_t)(blockIdx.x + 1) * total / gridDim.x);
    const int64_t rowbytes = p.K >> 1;
    const int nbk = p.K / SB;                        // scale blocks per weight row

    auto item_m = [&](int item) -> int {
        const int e = s_active[item / nt];
        return (int)(p.offsets[e + 1] - p.offsets[e]);
    };
    auto advance = [&](Pos q) -> Pos {
        if (++q.kc == plan.nch) {
            q.kc = 0;
            const int npass = (item_m(q.item) + 8 * GMAX - 1) / (8 * GMAX);
            if (++q.pass == npass) {
                q.pass = 0;
                ++q.item;
            }
        }
        return q;
    };

    if (warp == kConsumers) {
        // ================= producer: packed rows -> shared-memory stages =================
        if (lane == 0) {
            uint32_t ctr = 0;
            for (Pos q{i0, 0, 0}; q.item < i1; q = advance(q), ++ctr) {
                const uint32_t slot = ctr % ns, ph = ((ctr / ns) & 1u) ^ 1u;
                if (!mbar_wait(smem_u32(bars + 16 + slot), ph, abort_flag)) break;
                const int e = s_active[q.item / nt];
                const int n0 = (q.item % nt) << 4;
                const int kb = q.kc * plan.kch;
                const uint32_t bytes = (uint32_t)(min(plan.kch, p.K - kb) >> 1);
                const uint32_t full = smem_u32(bars + slot);
                asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(full), "r"(16u * bytes)
                             : "memory");
                const uint8_t* src = p.W + ((int64_t)e * p.N + n0) * rowbytes + (kb >> 1);
                const uint32_t dst = smem_u32(smem + slot * plan.stage_bytes);
                for (int r = 0; r < 16; ++r)
                    asm volatile(
                        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                        ::"r"(dst + r * plan.row_stride), "l"(src + r * rowbytes), "r"(bytes), "r"(full)
                        : "memory");
            }
        }
        __syncwarp();
    } else {
        // ================= consumers =================
        const int g = lane >> 2, t = lane & 3;
        uint32_t ctr = 0;
        float acc[GMAX][4];
        float sc0[BPW], sc1[BPW], nsc0[BPW], nsc1[BPW];
        auto load_scales = [&](const Pos& q, float (&s0)[BPW], float (&s1)[BPW]) {
            const int e = s_active[q.item / nt];
            const int n0 = (q.item % nt) << 4;
            const int nbc = min(plan.kch, p.K - q.kc * plan.kch) / SB;
            const int b0 = warp * nbc / kConsumers, b1 = (warp + 1) * nbc / kConsumers;
            const int64_t base0 = ((int64_t)e * p.N + n0 + g) * nbk + q.kc * (plan.kch / SB);
#pragma unroll
            for (int c = 0; c < BPW; ++c) {
                s0[c] = s1[c] = 0.f;
                if (b0 + c < b1) {
                    s0[c] = load_scale<FMT>(p.scales, base0 + b0 + c);
                    s1[c] = load_scale<FMT>(p.scales, base0 + 8 * (int64_t)nbk + b0 + c);
                }
            }
        };
        Pos cur{i0, 0, 0};
        if (cur.item < i1) load_scales(cur, nsc0, nsc1);
        while (cur.item < i1) {
            const int e = s_active[cur.item / nt];
            const int n0 = (cur.item % nt) << 4;
            const int64_t r0 = p.offsets[e];
            const int m = (int)(p.offsets[e + 1] - r0);
            const int mc = cur.pass * 8 * GMAX;
            const int G = min(GMAX, (m - mc + 7) >> 3);
#pragma unroll
            for (int c = 0; c < BPW; ++c) { sc0[c] = nsc0[c]; sc1[c] = nsc1[c]; }
            const Pos nxt = advance(cur);
            if (nxt.item < i1) load_scales(nxt, nsc0, nsc1);
            if (cur.kc == 0) {
#pragma unroll
                for (int j = 0; j < GMAX; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
            }
            const int kb = cur.kc * plan.kch;
            const int nbc = min(plan.kch, p.K - kb) / SB;
            const int b0 = warp * nbc / kConsumers, b1 = (warp + 1) * nbc / kConsumers;
            // activation row of this lane's token column g, per 8-row group (-1: none)
            int xtk[GMAX];
#pragma unroll
            for (int j = 0; j < GMAX; ++j) {
                const int rr = mc + 8 * j + g;
                xtk[j] = -1;
                if (j < G && rr < m) {
                    const int64_t r = r0 + rr;
                    xtk[j] = p.row_token ? __ldg(p.row_token + r) : (int)r;
                }
            }
            const uint16_t* xbase = p.x + kb + t * (SB / 4);
            // group 0's activation words for this warp's blocks, loaded before the wait
            uint32_t xw0[BPW][XW];
#pragma unroll
            for (int c = 0; c < BPW; ++c) {
#pragma unroll
                for (int q = 0; q < XW; ++q) xw0[c][q] = 0u;
                if (b0 + c < b1 && xtk[0] >= 0) {
#pragma unroll
                    for (int q = 0; q < XW / 4; ++q) {
                        const uint4 v = __ldg(reinterpret_cast<const uint4*>(
                            xbase + (int64_t)xtk[0] * p.K + (b0 + c) * SB) + q);
                        xw0[c][4 * q] = v.x; xw0[c][4 * q + 1] = v.y; xw0[c][4 * q + 2] = v.z; xw0[c][4 * q + 3] = v.w;
                    }
                }
            }
            const uint32_t slot = ctr % ns, ph = (ctr / ns) & 1u;
            ++ctr;
            if (!mbar_wait(smem_u32(bars + slot), ph, abort_flag)) break;
            const uint8_t* st = smem + slot * plan.stage_bytes;
#pragma unroll
            for (int c = 0; c < BPW; ++c) {
                if (b0 + c < b1) {
                    const int b = b0 + c;
                    uint32_t w0[BPL / 4], w1[BPL / 4];
                    const uint8_t* rp0 = st + g * plan.row_stride + b * (SB / 2) + t * BPL;
                    const uint8_t* rp1 = rp0 + 8 * plan.row_stride;
                    if constexpr (BPL == 8) {
                        const uint2 u0 = *reinterpret_cast<const uint2*>(rp0);
                        const uint2 u1 = *reinterpret_cast<const uint2*>(rp1);
                        w0[0] = u0.x; w0[BPL / 4 - 1] = u0.y;
                        w1[0] = u1.x; w1[BPL / 4 - 1] = u1.y;
                    } else {
                        w0[0] = *reinterpret_cast<const uint32_t*>(rp0);
                        w1[0] = *reinterpret_cast<const uint32_t*>(rp1);
                    }
                    uint32_t d0[2 * BPL / 2], d1[2 * BPL / 2];
#pragma unroll
                    for (int q = 0; q < BPL / 4; ++q) {
                        uint32_t o[4];
                        decode_word<FMT>(w0[q], p.lut, o);
                        d0[4 * q] = o[0]; d0[4 * q + 1] = o[1]; d0[4 * q + 2] = o[2]; d0[4 * q + 3] = o[3];
                        decode_word<FMT>(w1[q], p.lut, o);
                        d1[4 * q] = o[0]; d1[4 * q + 1] = o[1]; d1[4 * q + 2] = o[2]; d1[4 * q + 3] = o[3];
                    }
#pragma unroll
                    for (int j = 0; j < GMAX; ++j) {
                        if (j < G) {
                            uint32_t xw[XW];
                            if (j == 0) {
#pragma unroll
                                for (int q = 0; q < XW; ++q) xw[q] = xw0[c][q];
                            } else if (xtk[j] >= 0) {
#pragma unroll
                                for (int q = 0; q < XW / 4; ++q) {
                                    const uint4 v = __ldg(reinterpret_cast<const uint4*>(
                                        xbase + (int64_t)xtk[j] * p.K + b * SB) + q);
                                    xw[4 * q] = v.x; xw[4 * q + 1] = v.y; xw[4 * q + 2] = v.z; xw[4 * q + 3] = v.w;
                                }
                            } else {
#pragma unroll
                                for (int q = 0; q < XW; ++q) xw[q] = 0u;
                            }
                            float cb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                            for (int s = 0; s < STEPS; ++s)
                                mma_bf16_16816(cb, d0[2 * s], d1[2 * s], d0[2 * s + 1], d1[2 * s + 1], xw[2 * s],
                                               xw[2 * s + 1]);
                            acc[j][0] = fmaf(cb[0], sc0[c], acc[j][0]);
                            acc[j][1] = fmaf(cb[1], sc0[c], acc[j][1]);
                            acc[j][2] = fmaf(cb[2], sc1[c], acc[j][2]);
                            acc[j][3] = fmaf(cb[3], sc1[c], acc[j][3]);
                        }
                    }
                }
            }
            __syncwarp();
            if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bars + 16 + slot))
                                        : "memory");
            if (cur.kc == plan.nch - 1) {
                // sum the 8 warp partials in a fixed order, then the epilogue
#pragma unroll
                for (int j = 0; j < GMAX; ++j)
                    if (j < G) red[(warp * GMAX + j) * 32 + lane] = make_float4(acc[j][0], acc[j][1], acc[j][2], acc[j][3]);
                asm volatile("bar.sync 1, %0;" ::"n"(kConsumers * 32) : "memory");
                for (int q = threadIdx.x; q < G * 128; q += kConsumers * 32) {
                    const int j = q >> 7, ln = (q >> 2) & 31, i = q & 3;
                    float v = 0.f;
#pragma unroll
                    for (int w = 0; w < kConsumers; ++w)
                        v += reinterpret_cast<const float*>(&red[(w * GMAX + j) * 32 + ln])[i];
                    const int slot_row = mc + 8 * j + 2 * (ln & 3) + (i & 1);   // C column 2t (+1)
                    if (slot_row < m) {
                        const int64_t r = r0 + slot_row;
                        if (p.row_weight) v *= __ldg(p.row_weight + r);
                        const int64_t dst = p.row_dest ? (int64_t)__ldg(p.row_dest + r) : r;
                        const int n = n0 + (ln >> 2) + ((i & 2) ? 8 : 0);        // C row g (+8)
                        p.out[dst * p.N + n] = f32_to_bf16_rne(v);
                    }
                }
                asm volatile("bar.sync 1, %0;" ::"n"(kConsumers * 32) : "memory");
            }
            cur = nxt;
        }
    }
}

template <int FMT, int GMAX>
static cudaError_t launch_db(const GroupedArgs& a, cudaStream_t s) {
    using namespace db;
    constexpr int SB = (FMT == FMT_NF4) ? 64 : 32;
    Plan plan;
    plan.kch = kBlocksPerStage * SB;
    if (plan.kch > a.K) plan.kch = a.K;
    plan.nch = (a.K + plan.kch - 1) / plan.kch;
    plan.row_stride = plan.kch / 2 + 16;
    plan.stage_bytes = ((16 * plan.row_stride + 127) / 128) * 128;
    const int red_bytes = kConsumers * GMAX * 32 * (int)sizeof(float4);
    const int fixed = red_bytes + 16 * 8 * 2 + 16 + 16 + kMaxExperts * 4;
    int per_sm = 2;
    int budget = 113 * 1024;
    int nst = (budget - fixed) / plan.stage_bytes;
    if (nst < 2) {
        per_sm = 1;
        budget = 225 * 1024;
        nst = (budget - fixed) / plan.stage_bytes;
    }
    if (nst > 8) nst = 8;
    if (nst < 2) return cudaErrorInvalidValue;
    plan.nstages = nst;
    const int smem = nst * plan.stage_bytes + fixed;
    static int smem_set = 0;                 // largest dynamic shared memory opted in so far
    if (smem > smem_set) {
        cudaError_t e = cudaFuncSetAttribute(decode_band_kernel<FMT, GMAX>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        smem_set = smem;
    }
    const int64_t groups_max = a.R < (int64_t)a.E ? a.R : (int64_t)a.E;
    const int64_t items_max = groups_max * (a.N / 16);
    int64_t grid = (int64_t)device_sm_count() * per_sm;
    if (items_max < grid) grid = items_max;
    if (grid < 1) return cudaSuccess;
    decode_band_kernel<FMT, GMAX><<<(unsigned)grid, kThreads, smem, s>>>(a, plan);
    return cudaGetLastError();
}

cudaError_t launch_decode_band(int fmt, const GroupedArgs& a, cudaStream_t s) {
    const int64_t mmax = a.R < (int64_t)a.m_hi ? a.R : (int64_t)a.m_hi;   // no group exceeds this
    // up to 16 routed rows per pass over a weight tile; larger groups take several passes
    if (fmt == FMT_NF4) return mmax <= 8 ? launch_db<FMT_NF4, 1>(a, s) : launch_db<FMT_NF4, 2>(a, s);
    return mmax <= 8 ? launch_db<FMT_MXFP4, 1>(a, s) : launch_db<FMT_MXFP4, 2>(a, s);
}

unsigned take_decode_error(cudaError_t* err) {
    unsigned v = 0;
    const unsigned zero = 0;
    *err = cudaMemcpyFromSymbol(&v, g_decode_error, sizeof(unsigned));
    if (*err == cudaSuccess && v) *err = cudaMemcpyToSymbol(g_decode_error, &zero, sizeof(unsigned));
    return v;
}

}  // namespace gnf4
