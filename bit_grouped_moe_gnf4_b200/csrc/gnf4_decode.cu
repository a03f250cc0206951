// Decode band of the grouped 4-bit GEMM: groups with few routed rows, where
// the packed weight bytes are the whole cost (the GEMV path of the solution page
// "How do I run a grouped GEMM directly on NF4 packed MoE expert weights,
// without dequantizing to bf16 first?", "Supported scope": one-token groups
// take the GEMV path).
//
// One persistent CTA per SM takes a contiguous run of work items; an item is
// (active expert, 16 weight rows). The CTA's 16 consumer warps form 4 groups of
// 4 warps; group q takes items q, q+4, ... of the run. A producer warp (one
// lane per group) streams each item's packed rows, one K chunk of 512 at a
// time, into the group's ring of shared-memory stages with 1-D bulk copies
// (cp.async.bulk, completion counted on an mbarrier), several chunks ahead, so
// HBM always has many bytes in flight per SM.
//
// The 4 warps of a group split each chunk's scale blocks. Nibble pairs are
// decoded by a table in shared memory that maps each packed byte to its two
// bf16 values (one bf16x2 word), replicated per lane so that 32 lookups never
// conflict; a byte permute forms the lookup address. The products run on
// warp-level bf16 MMAs with the 16 weight rows as the M side and up to 8 routed
// rows per MMA as the N side. Every MMA chain covers exactly one scale block
// (64 K for NF4, 32 K for MXFP4), so the block sum leaves the tensor core in
// fp32 and is scaled and accumulated in fp32 outside it. After the last chunk
// the group's 4 partial sums are added in a fixed order through shared memory
// (deterministic), weighted, rounded to bf16 and stored at the destination rows.
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

constexpr int kMaxGroups = 4;                      // item groups per CTA (fewer when shared memory is short)
constexpr int kGroupWarps = 4;                     // consumer warps per group (split of each chunk)
constexpr int kMaxThreads = (kMaxGroups * kGroupWarps + 1) * 32;   // + one producer warp
constexpr int kMaxExperts = 2048;
constexpr int kChunkK = 512;                       // K per stage
constexpr int kLutBytes = 256 * 256;               // byte value b, lane l -> offset b*256 + l*4

struct Plan {
    int kch;          // K elements per stage
    int nch;          // stages per item pass
    int row_stride;   // bytes per weight row in a stage (chunk bytes + 16 of padding)
    int stage_bytes;  // 16 rows
    int scale_bytes;  // slot for one item's scales (16 rows x all blocks, contiguous in memory), rounded to 128
    int nstages;      // stages per group ring
    int nslots;       // item scale slots per group
    int ngroups;      // item groups in the CTA (consumer warps = 4 * ngroups, then the producer warp)
};

struct Pos {
    int item, pass, kc;
};

}  // namespace db

template <int FMT, int GMAX>
__global__ void __launch_bounds__(db::kMaxThreads, 1) decode_band_kernel(const GroupedArgs p, const db::Plan plan) {
    using namespace db;
    constexpr int SB = (FMT == FMT_NF4) ? 64 : 32;   // K elements per scale block
    constexpr int STEPS = SB / 16;                   // k16 MMA steps per block
    constexpr int BPL = SB / 8;                      // packed bytes per lane per row per block (8 or 4)
    constexpr int XW = SB / 8;                       // bf16x2 words of x per lane per block
    constexpr int BPW = (kChunkK / SB) / kGroupWarps;  // blocks per warp per full chunk (2 or 4)

    const int kGroups = plan.ngroups;
    const int kConsumers = kGroups * kGroupWarps;
    const int kThreads = (kConsumers + 1) * 32;

    extern __shared__ __align__(1024) uint8_t smem[];
    // [lut][rings: groups x stages x stage_bytes][scale slots: groups x stages x scale_bytes]
    // [red][barriers][abort, counts][active experts: id, first row, rows]
    uint8_t* lut = smem;                                            // [256][64] words
    uint8_t* rings = smem + kLutBytes;
    uint8_t* sslots = rings + kGroups * plan.nstages * plan.stage_bytes;
    float4* red = reinterpret_cast<float4*>(sslots + kGroups * plan.nslots * plan.scale_bytes);
    uint64_t* bars = reinterpret_cast<uint64_t*>(red + kConsumers * GMAX * 32);   // full[g][s], empty[g][s]
    int* tailw = reinterpret_cast<int*>(bars + 2 * kGroups * plan.nstages);
    volatile int* abort_flag = tailw;
    int* s_nact = tailw + 4;
    int64_t* s_r0 = reinterpret_cast<int64_t*>(tailw + 8);         // [E] first routed row
    int* s_active = reinterpret_cast<int*>(s_r0 + p.E);            // [E] expert id
    int* s_cnt = s_active + p.E;                                   // [E] routed rows

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ns = plan.nstages;

    // byte -> bf16x2 table, one copy per lane
    for (int i = threadIdx.x; i < 256 * 32; i += kThreads) {
        const int b = i >> 5, l = i & 31;
        *reinterpret_cast<uint32_t*>(lut + b * 256 + l * 4) = byte_bf16x2<FMT>((uint32_t)b, p.lut);
    }
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
            if (act) {
                const int idx = count + __popc(bal & ((1u << lane) - 1u));
                s_active[idx] = e;
                s_r0[idx] = p.offsets[e];
                s_cnt[idx] = (int)(p.offsets[e + 1] - p.offsets[e]);
            }
            count += __popc(bal);
        }
        if (lane == 0) s_nact[0] = count;
    } else if (warp == kConsumers && lane == 0) {
        for (int i = 0; i < kGroups * ns; ++i) {
            mbar_init(smem_addr(bars + i), 1);                                 // full: producer + tx bytes
            mbar_init(smem_addr(bars + kGroups * ns + i), kGroupWarps);        // empty: the group's warps
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

    auto advance = [&](Pos q) -> Pos {
        if (++q.kc == plan.nch) {
            q.kc = 0;
            const int m = s_cnt[q.item / nt];
            if (++q.pass == (m + 8 * GMAX - 1) / (8 * GMAX)) {
                q.pass = 0;
                q.item += kGroups;
            }
        }
        return q;
    };

    if (warp == kConsumers) {
        // ================= producer: lane q feeds group q's ring =================
        if (lane < kGroups) {
            const int q = lane;
            uint64_t* full = bars + q * ns;
            uint64_t* empty = bars + kGroups * ns + q * ns;
            uint8_t* ring = rings + q * ns * plan.stage_bytes;
            uint8_t* sring = sslots + q * plan.nslots * plan.scale_bytes;
            const int ssz = FMT == FMT_NF4 ? 4 : 1;
            uint32_t ctr = 0, jitem = 0;
            for (Pos ps{i0 + q, 0, 0}; ps.item < i1; ps = advance(ps), ++ctr) {
                const uint32_t slot = ctr % ns, ph = ((ctr / ns) & 1u) ^ 1u;
                if (!mbar_wait_bounded(smem_addr(empty + slot), ph, abort_flag, &g_decode_error, 1u)) break;
                const int e = s_active[ps.item / nt];
                const int n0 = (ps.item % nt) << 4;
                const int kb = ps.kc * plan.kch;
                const uint32_t bytes = (uint32_t)(min(plan.kch, p.K - kb) >> 1);
                const uint32_t fb = smem_addr(full + slot);
                const bool first = ps.kc == 0 && ps.pass == 0;
                const uint32_t sbytes = (uint32_t)(16 * nbk * ssz);      // exact, a multiple of 16
                mbar_arrive_tx(fb, 16u * bytes + (first ? sbytes : 0u));
                if (first) {
                    // the item's scales: 16 rows x all blocks, one contiguous range
                    const uint8_t* ssrc = reinterpret_cast<const uint8_t*>(p.scales) +
                                          ((int64_t)e * p.N + n0) * nbk * ssz;
                    asm volatile(
                        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                        ::"r"(smem_addr(sring + (jitem % plan.nslots) * plan.scale_bytes)), "l"(ssrc),
                          "r"(sbytes), "r"(fb) : "memory");
                    ++jitem;
                }
                const uint8_t* src = p.W + ((int64_t)e * p.N + n0) * rowbytes + (kb >> 1);
                const uint32_t dst = smem_addr(ring + slot * plan.stage_bytes);
                for (int r = 0; r < 16; ++r)
                    asm volatile(
                        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                        ::"r"(dst + r * plan.row_stride), "l"(src + r * rowbytes), "r"(bytes), "r"(fb)
                        : "memory");
            }
        }
        __syncwarp();
    } else {
        // ================= consumers =================
        const int q = warp / kGroupWarps, gw = warp % kGroupWarps;
        const int g = lane >> 2, t = lane & 3;
        uint64_t* full = bars + q * ns;
        uint64_t* empty = bars + kGroups * ns + q * ns;
        const uint8_t* ring = rings + q * ns * plan.stage_bytes;
        const uint8_t* sring = sslots + q * plan.nslots * plan.scale_bytes;
        float4* gred = red + q * kGroupWarps * GMAX * 32;
        const uint32_t lane_sel = (uint32_t)lane * 4u;   // lut offset of this lane's copy
        uint32_t ctr = 0, jitem = 0;
        float acc[GMAX][4];
        // activation row of this lane's token column g, per 8-row group (-1: none), for the
        // current and the next item; the next item's rows are prefetched into L1 early
        int xtk[GMAX], ntk[GMAX];
        auto tokens_of = [&](int item, int pass, int (&tk)[GMAX]) {
#pragma unroll
            for (int j = 0; j < GMAX; ++j) tk[j] = -1;
            if (item >= i1) return;
            const int a = item / nt;
            const int64_t r0 = s_r0[a];
            const int m = s_cnt[a];
            const int mc = pass * 8 * GMAX;
#pragma unroll
            for (int j = 0; j < GMAX; ++j) {
                const int rr = mc + 8 * j + g;
                if (rr < m) tk[j] = p.row_token ? __ldg(p.row_token + r0 + rr) : (int)(r0 + rr);
            }
        };
        auto prefetch_x = [&](const int (&tk)[GMAX]) {
            // this lane's 16-byte pieces of x for every block of this warp, all chunks
#pragma unroll
            for (int j = 0; j < GMAX; ++j) {
                if (tk[j] < 0) continue;
                const uint16_t* xr = p.x + (int64_t)tk[j] * p.K + t * (SB / 4);
                for (int kc = 0; kc < plan.nch; ++kc) {
                    const int kb = kc * plan.kch;
                    const int nbc = min(plan.kch, p.K - kb) / SB;
                    for (int b = gw * nbc / kGroupWarps; b < (gw + 1) * nbc / kGroupWarps; ++b)
                        asm volatile("prefetch.global.L1 [%0];" ::"l"(xr + kb + b * SB));
                }
            }
        };
        Pos cur{i0 + q, 0, 0};
        tokens_of(cur.item, 0, xtk);
        prefetch_x(xtk);
        tokens_of(cur.item + kGroups, 0, ntk);
        while (cur.item < i1) {
            const int a = cur.item / nt;
            const int n0 = (cur.item % nt) << 4;
            const int64_t r0 = s_r0[a];
            const int m = s_cnt[a];
            const int mc = cur.pass * 8 * GMAX;
            const int G = min(GMAX, (m - mc + 7) >> 3);
            const Pos nxt = advance(cur);
            if (cur.kc == 0) {
#pragma unroll
                for (int j = 0; j < GMAX; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
                if (cur.pass == 0) prefetch_x(ntk);       // next item's rows, one item ahead
            }
            const int kb = cur.kc * plan.kch;
            const int nbc = min(plan.kch, p.K - kb) / SB;
            const int b0 = gw * nbc / kGroupWarps, b1 = (gw + 1) * nbc / kGroupWarps;
            const uint16_t* xbase = p.x + kb + t * (SB / 4);
            const uint32_t slot = ctr % ns, ph = (ctr / ns) & 1u;
            ++ctr;
            if (!mbar_wait_bounded(smem_addr(full + slot), ph, abort_flag, &g_decode_error, 2u)) break;
            const uint8_t* st = ring + slot * plan.stage_bytes;
            const uint8_t* ss = sring + (jitem % plan.nslots) * plan.scale_bytes;
            const int bg0 = cur.kc * (plan.kch / SB);     // first scale block of the chunk
#pragma unroll
            for (int c = 0; c < BPW; ++c) {
                if (b0 + c < b1) {
                    const int b = b0 + c;
                    float s0, s1;
                    if constexpr (FMT == FMT_NF4) {
                        s0 = reinterpret_cast<const float*>(ss)[g * nbk + bg0 + b];
                        s1 = reinterpret_cast<const float*>(ss)[(g + 8) * nbk + bg0 + b];
                    } else {
                        s0 = e8m0_to_f32(ss[g * nbk + bg0 + b]);
                        s1 = e8m0_to_f32(ss[(g + 8) * nbk + bg0 + b]);
                    }
                    // this lane's packed bytes of rows g and g+8
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
                    // byte j -> bf16x2 word j (table lookup; address = byte*256 + lane*4)
                    uint32_t d0[BPL], d1[BPL];
#pragma unroll
                    for (int j = 0; j < BPL; ++j) {
                        const uint32_t sel = 0x5504u | ((uint32_t)(j & 3) << 4);
                        d0[j] = *reinterpret_cast<const uint32_t*>(lut + prmt(w0[j >> 2], lane_sel, sel));
                        d1[j] = *reinterpret_cast<const uint32_t*>(lut + prmt(w1[j >> 2], lane_sel, sel));
                    }
#pragma unroll
                    for (int j = 0; j < GMAX; ++j) {
                        if (j < G) {
                            uint32_t xw[XW];
                            if (xtk[j] >= 0) {
#pragma unroll
                                for (int w = 0; w < XW / 4; ++w) {
                                    const uint4 v = __ldg(reinterpret_cast<const uint4*>(
                                        xbase + (int64_t)xtk[j] * p.K + b * SB) + w);
                                    xw[4 * w] = v.x; xw[4 * w + 1] = v.y; xw[4 * w + 2] = v.z; xw[4 * w + 3] = v.w;
                                }
                            } else {
#pragma unroll
                                for (int w = 0; w < XW; ++w) xw[w] = 0u;
                            }
                            float cb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                            for (int s = 0; s < STEPS; ++s)
                                mma_bf16_16816(cb, d0[2 * s], d1[2 * s], d0[2 * s + 1], d1[2 * s + 1], xw[2 * s],
                                               xw[2 * s + 1]);
                            acc[j][0] = fmaf(cb[0], s0, acc[j][0]);
                            acc[j][1] = fmaf(cb[1], s0, acc[j][1]);
                            acc[j][2] = fmaf(cb[2], s1, acc[j][2]);
                            acc[j][3] = fmaf(cb[3], s1, acc[j][3]);
                        }
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_addr(empty + slot));
            if (cur.kc == plan.nch - 1) {
                // the group's 4 partial sums, added in a fixed order, then the epilogue
#pragma unroll
                for (int j = 0; j < GMAX; ++j)
                    if (j < G) gred[(gw * GMAX + j) * 32 + lane] = make_float4(acc[j][0], acc[j][1], acc[j][2], acc[j][3]);
                asm volatile("bar.sync %0, %1;" ::"r"(1 + q), "n"(kGroupWarps * 32) : "memory");
                const int tid = gw * 32 + lane;
                for (int qq = tid; qq < G * 128; qq += kGroupWarps * 32) {
                    const int j = qq >> 7, ln = (qq >> 2) & 31, i = qq & 3;
                    float v = 0.f;
#pragma unroll
                    for (int w = 0; w < kGroupWarps; ++w)
                        v += reinterpret_cast<const float*>(&gred[(w * GMAX + j) * 32 + ln])[i];
                    const int row = mc + 8 * j + 2 * (ln & 3) + (i & 1);   // C column 2t (+1)
                    if (row < m) {
                        const int64_t r = r0 + row;
                        if (p.row_weight) v *= __ldg(p.row_weight + r);
                        const int64_t dst = p.row_dest ? (int64_t)__ldg(p.row_dest + r) : r;
                        const int n = n0 + (ln >> 2) + ((i & 2) ? 8 : 0);   // C row g (+8)
                        p.out[dst * p.N + n] = f32_to_bf16_rne(v);
                    }
                }
                asm volatile("bar.sync %0, %1;" ::"r"(1 + q), "n"(kGroupWarps * 32) : "memory");
                // next pass of this item, or the next item
                if (nxt.item != cur.item) {
                    ++jitem;
#pragma unroll
                    for (int j = 0; j < GMAX; ++j) xtk[j] = ntk[j];
                    tokens_of(nxt.item + kGroups, 0, ntk);
                } else {
                    tokens_of(nxt.item, nxt.pass, xtk);
                }
            }
            cur = nxt;
        }
    }
}

template <int FMT, int GMAX>
static cudaError_t launch_db(const GroupedArgs& a, cudaStream_t s) {
    using namespace db;
    Plan plan;
    plan.kch = kChunkK < a.K ? kChunkK : a.K;
    plan.nch = (a.K + plan.kch - 1) / plan.kch;
    plan.row_stride = plan.kch / 2 + 16;
    plan.stage_bytes = ((16 * plan.row_stride + 127) / 128) * 128;
    const int SB = (FMT == FMT_NF4) ? 64 : 32;
    plan.scale_bytes = ((16 * (a.K / SB) * (FMT == FMT_NF4 ? 4 : 1) + 127) / 128) * 128;
    // largest group count whose rings fit in shared memory
    const int tables = 32 + 16 * a.E;
    int smem = 0;
    plan.ngroups = 0;
    for (int ng = kMaxGroups; ng >= 1 && plan.ngroups == 0; ng >>= 1) {
        const int red_bytes = ng * kGroupWarps * GMAX * 32 * (int)sizeof(float4);
        const int fixed = kLutBytes + red_bytes + 2 * ng * 8 * 8 + tables;
        for (int nst = 8; nst >= 3; --nst) {
            const int nsl = (nst - 1 + plan.nch - 1) / plan.nch + 1;   // items a group can have in flight
            const int need = fixed + ng * (nst * plan.stage_bytes + nsl * plan.scale_bytes);
            if (need <= 226 * 1024) {
                plan.ngroups = ng;
                plan.nstages = nst;
                plan.nslots = nsl;
                smem = need;
                break;
            }
        }
    }
    if (plan.ngroups == 0) return cudaErrorInvalidValue;
    static int smem_set = 0;                 // largest dynamic shared memory opted in so far
    if (smem > smem_set) {
        cudaError_t e = cudaFuncSetAttribute(decode_band_kernel<FMT, GMAX>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        smem_set = smem;
    }
    const int64_t groups_max = a.R < (int64_t)a.E ? a.R : (int64_t)a.E;
    const int64_t items_max = groups_max * (a.N / 16);
    int64_t grid = device_sm_count();
    if (items_max < grid) grid = items_max;
    if (grid < 1) return cudaSuccess;
    decode_band_kernel<FMT, GMAX><<<(unsigned)grid, (plan.ngroups * kGroupWarps + 1) * 32, smem, s>>>(a, plan);
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
