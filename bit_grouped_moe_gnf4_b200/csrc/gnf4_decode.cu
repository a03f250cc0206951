// Decode band of the grouped 4-bit GEMM: groups with few routed rows, where
// the packed weight bytes are the whole cost (the GEMV path of the solution page
// "How do I run a grouped GEMM directly on NF4 packed MoE expert weights,
// without dequantizing to bf16 first?", "Supported scope": one-token groups
// take the GEMV path).
//
// One persistent CTA per SM takes a contiguous run of work items; an item is
// (active expert, ROWS = 48 weight rows; fewer when K is very large). A producer
// thread streams each item's packed rows, one K chunk of 256 at a time, into a
// ring of 8 KB shared-memory stages with one 2-D TMA load per chunk (a box of
// 128 bytes x ROWS rows, 128B-swizzled); the stage holds nothing else, so the
// producer issues one copy per stage and the copy engine keeps HBM busy. The
// item's block scales (ROWS rows x all blocks, one contiguous range) land in a
// scale slot with a barrier of their own, issued one item ahead.
//
// 12 consumer warps: warp (rt, ks) owns row tile rt (16 rows of the item) and
// the K chunks kc with kc % nks == ks (nks = 4 for 48-row items, so K chunks
// of any multiple of 1024 split evenly), so each stage is read by ROWS/16 warps
// and stages are consumed in parallel. Ownership goes
// by K position only, so the fp32 grouping of a row's sum never depends on the
// other rows of the call. Because owners skip the stages of other warps, a ring
// slot carries a tag naming the chunk that was last issued into it; an owner
// reads the slot's barrier only once the tag shows its chunk, which keeps
// every parity wait within one phase.
//
// The activations of the routed rows are small and shared by every item of an
// expert, so the consumers read them straight from global memory through L1
// (prefetched into L1 before the wait for the chunk's weights). Nibbles are
// decoded by a table in shared memory that maps each packed byte to its two
// bf16 values (replicated per lane, so 32 lookups never conflict; a byte
// permute forms the address); for MXFP4, whose register decode is short, one
// of the lane's two rows goes through byte permutes on register tables instead,
// to spread the work over the shared-memory and ALU pipes. The products run on warp-level bf16 MMAs with 16
// weight rows as the M side and up to 8 routed rows per MMA as the N side.
// Every MMA chain covers exactly one scale block (64 K for NF4, 32 K for
// MXFP4), so the block sum leaves the tensor core in fp32 and is scaled and
// accumulated in fp32 outside it.
//
// At the end of each pass over an item the consumer warps hand their fp32
// partial sums to an epilogue warp through double-buffered slots (kept in the
// unused half of every 256-byte row of the lookup table) and go on; the
// epilogue warp adds the K splits in a fixed order (deterministic), applies the
// routing weight, rounds to bf16 and stores at the destination rows.
//
// MMA k-slot mapping: in m16n8k16, lane (g, t) supplies k-slots 2t, 2t+1,
// 2t+8, 2t+9 of both operands. They are mapped to the four consecutive K
// positions base + (SB/4)*t + 4*s + {0,1,2,3} of step s, the same for A and
// B, so each lane reads contiguous bytes of the packed rows and of x.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <climits>
#include <cstdint>

#include "gnf4_common.cuh"
#include "gnf4_kernels.h"

namespace gnf4 {

__device__ unsigned g_decode_error;

namespace db {

constexpr int kConsumers = 12;                     // consumer warps: 4 row tiles x 3 K-split owners
constexpr int kProducerWarp = kConsumers;          // one thread issues all copies
constexpr int kEpilogueWarp = kConsumers + 1;      // reduces and stores the partial sums
constexpr int kThreads = (kConsumers + 2) * 32;    // 14 warps: at most 4 per SM sub-partition,
constexpr int kRegBound = 512;                     // so 128 registers a thread (bounds for 16 warps)
constexpr int kChunkK = 256;                       // K per stage: 128 packed bytes per row = one TMA box
constexpr int kBoxBytes = 128;
constexpr int kLutBytes = 256 * 256;               // byte value b, lane l -> offset b*256 + l*4
constexpr int kMaxTableRows = 1024;                // routed rows whose metadata fits the CTA's table
constexpr int kMaxRowTiles = 4;                    // ROWS / 16 is at most 3

struct Plan {
    int rows;         // weight rows per item (48, 32 or 16)
    int nch;          // stages per item pass
    int stage_bytes;  // rows x 128 bytes (a multiple of 1024)
    int scale_bytes;  // slot for one item's scales (rows x all blocks), rounded to 128
    int nstages;      // ring stages
    int nslots;       // item scale slots
};

__device__ __forceinline__ void tma_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar) : "memory");
}
__device__ __forceinline__ void bulk_1d(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(dst), "l"(src), "r"(bytes), "r"(bar) : "memory");
}

// Wait until the ring slot's tag names chunk `want` (the producer has issued it,
// so the slot's previous fill was consumed). Bounded like mbar_wait_bounded.
__device__ __forceinline__ bool wait_tag(const int* tag, uint32_t want, volatile int* abort_flag, unsigned* err,
                                         unsigned code) {
    const uint32_t a = smem_addr(tag);
    uint32_t v;
    asm volatile("ld.acquire.cta.shared::cta.u32 %0, [%1];" : "=r"(v) : "r"(a) : "memory");
    if (v == want) return true;
    const long long t0 = clock64();
    for (uint32_t it = 1;; ++it) {
        __nanosleep(64);
        asm volatile("ld.acquire.cta.shared::cta.u32 %0, [%1];" : "=r"(v) : "r"(a) : "memory");
        if (v == want) return true;
        if ((it & 7u) == 0u) {
            if (*abort_flag) return false;
            if (clock64() - t0 > kWaitTimeoutCycles) {
                *abort_flag = 1;
                atomicOr(err, code);
                return false;
            }
        }
    }
}

__device__ __forceinline__ void prefetch_l1(const void* p) {
    asm volatile("prefetch.global.L1 [%0];" ::"l"(p));
}

// Partial-sum slot of unit u (= ((buffer * row tiles + rt) * nks + ks) * GMAX + j)
// for one lane: 512 bytes per unit, spread over four 128-byte holes of the lookup
// table (bytes 128..255 of each 256-byte row, which the table leaves unused).
__device__ __forceinline__ float4* red_slot(uint8_t* lut, int u, int lane) {
    return reinterpret_cast<float4*>(lut + (u * 4 + (lane >> 3)) * 256 + 128 + (lane & 7) * 16);
}

// The MMAs of one chunk for one consumer warp: 16 weight rows (ra = row g, rb =
// row g + 8 of the row tile) x NG groups of 8 routed rows x NBC scale blocks
// (only the first nbc when the chunk is the ragged end of K).
template <int FMT, int GMAX, int NG, bool FULL>
__device__ __forceinline__ void chunk_mma(const uint8_t* __restrict__ st, const uint8_t* __restrict__ ss,
                                          const uint8_t* __restrict__ lut, uint32_t lane_sel, const LutPlanes& L,
                                          const uint16_t* xr0, const uint16_t* xr1, int ra, int rb, int t, int nbk,
                                          int kc, int nbc, bool vec_scales, float (&acc)[GMAX][4]) {
    constexpr int SB = (FMT == FMT_NF4) ? 64 : 32;   // K elements per scale block
    constexpr int STEPS = SB / 16;                   // k16 MMA steps per block
    constexpr int BPL = SB / 8;                      // packed bytes per lane per row per block (8 or 4)
    constexpr int XW = SB / 8;                       // bf16x2 words of x per lane per block
    constexpr int NBC = kChunkK / SB;                // scale blocks in a full chunk (4 or 8)
    const int bg0 = kc * NBC;                        // first scale block of the chunk
    // block scales of rows ra and rb for this chunk: one vector load per row when the
    // rows' blocks are aligned for it, picked per block by selects (no local arrays)
    float4 va4 = make_float4(0.f, 0.f, 0.f, 0.f), vb4 = va4;
    uint2 va2 = make_uint2(0u, 0u), vb2 = va2;
    const bool vec = FULL && vec_scales;
    if (vec) {
        if constexpr (FMT == FMT_NF4) {
            va4 = *reinterpret_cast<const float4*>(ss + (ra * nbk + bg0) * 4);
            vb4 = *reinterpret_cast<const float4*>(ss + (rb * nbk + bg0) * 4);
        } else {
            va2 = *reinterpret_cast<const uint2*>(ss + ra * nbk + bg0);
            vb2 = *reinterpret_cast<const uint2*>(ss + rb * nbk + bg0);
        }
    }
#pragma unroll 2
    for (int b = 0; b < NBC; ++b) {
        if (FULL || b < nbc) {
            float sa, sb;
            if (vec) {
                if constexpr (FMT == FMT_NF4) {
                    const int i = b & 3;
                    sa = i == 0 ? va4.x : i == 1 ? va4.y : i == 2 ? va4.z : va4.w;
                    sb = i == 0 ? vb4.x : i == 1 ? vb4.y : i == 2 ? vb4.z : vb4.w;
                } else {
                    const uint32_t sh = 8u * (uint32_t)(b & 3);
                    sa = e8m0_to_f32(((b < 4 ? va2.x : va2.y) >> sh) & 0xFFu);
                    sb = e8m0_to_f32(((b < 4 ? vb2.x : vb2.y) >> sh) & 0xFFu);
                }
            } else {
                if constexpr (FMT == FMT_NF4) {
                    sa = reinterpret_cast<const float*>(ss)[ra * nbk + bg0 + b];
                    sb = reinterpret_cast<const float*>(ss)[rb * nbk + bg0 + b];
                } else {
                    sa = e8m0_to_f32(ss[ra * nbk + bg0 + b]);
                    sb = e8m0_to_f32(ss[rb * nbk + bg0 + b]);
                }
            }
            // this lane's packed bytes of rows ra and rb: byte o of the row's 128-byte
            // chunk sits in 16-byte piece (o/16) ^ (row%8) of the swizzled box row
            const int o = b * (SB / 2) + t * BPL;
            const int pc = o >> 4, po = o & 15;
            const uint8_t* rp0 = st + ra * kBoxBytes + ((pc ^ (ra & 7)) << 4) + po;
            const uint8_t* rp1 = st + rb * kBoxBytes + ((pc ^ (rb & 7)) << 4) + po;
            uint32_t w0[BPL / 4], w1[BPL / 4];
            if constexpr (BPL == 8) {
                const uint2 u0 = *reinterpret_cast<const uint2*>(rp0);
                const uint2 u1 = *reinterpret_cast<const uint2*>(rp1);
                w0[0] = u0.x; w0[BPL / 4 - 1] = u0.y;
                w1[0] = u1.x; w1[BPL / 4 - 1] = u1.y;
            } else {
                w0[0] = *reinterpret_cast<const uint32_t*>(rp0);
                w1[0] = *reinterpret_cast<const uint32_t*>(rp1);
            }
            // row ra by the shared-memory table; row rb by the table too (NF4) or by
            // byte permutes on register tables (MXFP4)
            uint32_t d0[BPL], d1[BPL];
#pragma unroll
            for (int j = 0; j < BPL; ++j) {
                const uint32_t sel = 0x5504u | ((uint32_t)(j & 3) << 4);
                d0[j] = *reinterpret_cast<const uint32_t*>(lut + prmt(w0[j >> 2], lane_sel, sel));
                if constexpr (FMT == FMT_NF4)
                    d1[j] = *reinterpret_cast<const uint32_t*>(lut + prmt(w1[j >> 2], lane_sel, sel));
            }
            if constexpr (FMT == FMT_MXFP4) {
#pragma unroll
                for (int q = 0; q < BPL / 4; ++q) {
                    uint32_t o4[4];
                    decode_word<FMT>(w1[q], L, o4);
                    d1[4 * q] = o4[0]; d1[4 * q + 1] = o4[1]; d1[4 * q + 2] = o4[2]; d1[4 * q + 3] = o4[3];
                }
            }
#pragma unroll
            for (int j = 0; j < NG; ++j) {
                // activations of routed row 8j + g of the pass, from global memory (L1);
                // lanes past the pass's rows feed zeros to output columns never stored
                uint32_t xw[XW];
#pragma unroll
                for (int w = 0; w < XW; ++w) xw[w] = 0u;
                const uint16_t* xr = (j == 0) ? xr0 : xr1;
                if (xr != nullptr) {
                    const uint4* xs = reinterpret_cast<const uint4*>(xr + kc * kChunkK + b * SB + t * (SB / 4));
#pragma unroll
                    for (int w = 0; w < XW / 4; ++w) {
                        const uint4 v = __ldg(xs + w);
                        xw[4 * w] = v.x; xw[4 * w + 1] = v.y; xw[4 * w + 2] = v.z; xw[4 * w + 3] = v.w;
                    }
                }
                // two independent MMA chains per block (first and second half of its steps)
                float c0[4] = {0.f, 0.f, 0.f, 0.f}, c1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int s = 0; s < STEPS; ++s) {
                    if (s < STEPS / 2)
                        mma_bf16_16816(c0, d0[2 * s], d1[2 * s], d0[2 * s + 1], d1[2 * s + 1], xw[2 * s], xw[2 * s + 1]);
                    else
                        mma_bf16_16816(c1, d0[2 * s], d1[2 * s], d0[2 * s + 1], d1[2 * s + 1], xw[2 * s], xw[2 * s + 1]);
                }
                acc[j][0] = fmaf(c0[0] + c1[0], sa, acc[j][0]);
                acc[j][1] = fmaf(c0[1] + c1[1], sa, acc[j][1]);
                acc[j][2] = fmaf(c0[2] + c1[2], sb, acc[j][2]);
                acc[j][3] = fmaf(c0[3] + c1[3], sb, acc[j][3]);
            }
        }
    }
}

}  // namespace db

template <int FMT, int GMAX>
__global__ void __launch_bounds__(db::kRegBound, 1)
decode_band_kernel(const GroupedArgs p, const db::Plan plan, const __grid_constant__ CUtensorMap wmap) {
    using namespace db;
    constexpr int SB = (FMT == FMT_NF4) ? 64 : 32;   // K elements per scale block

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    // [lut (+ partial-sum slots in its holes)][ring: stages x stage_bytes][scale slots][barriers]
    // [abort, count, warp counts, tags][experts][row table]
    uint8_t* lut = smem;                                            // [256][64] words
    uint8_t* ring = smem + kLutBytes;                               // 1024-aligned stages
    uint8_t* sslots = ring + plan.nstages * plan.stage_bytes;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sslots + plan.nslots * plan.scale_bytes);
    // full[ns], empty[ns], scale slot free[nslots], scale slot full[nslots],
    // partials ready[2][kMaxRowTiles], partial slots free[2][kMaxRowTiles]
    int* tailw = reinterpret_cast<int*>(bars + 2 * plan.nstages + 2 * plan.nslots + 4 * kMaxRowTiles);
    volatile int* abort_flag = tailw;
    int* s_wcnt = tailw + 8;                                       // [16] active experts per warp (scan)
    int* tags = tailw + 24;                                        // [ns] chunk counter last issued per slot
    int64_t* s_r0 = reinterpret_cast<int64_t*>(tailw + 24 + ((plan.nstages + 1) & ~1)); // [E] first routed row
    int* s_active = reinterpret_cast<int*>(s_r0 + p.E);            // [E] expert id
    int* s_cnt = s_active + p.E;                                   // [E] routed rows
    int* t_tok = s_cnt + p.E;                                      // [kMaxTableRows] per routed row
    float* t_wt = reinterpret_cast<float*>(t_tok + kMaxTableRows);
    int* t_dst = reinterpret_cast<int*>(t_wt + kMaxTableRows);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ns = plan.nstages, nsl = plan.nslots;
    const int ROWS = plan.rows;
    const int nrt = ROWS / 16, nks = kConsumers / nrt;
    uint64_t* full = bars;
    uint64_t* empty = bars + ns;
    uint64_t* sfree = bars + 2 * ns;
    uint64_t* sfull = bars + 2 * ns + nsl;
    uint64_t* rready = bars + 2 * ns + 2 * nsl;                   // [buffer * kMaxRowTiles + rt]
    uint64_t* rfree = rready + 2 * kMaxRowTiles;

    if (warp == kProducerWarp && lane == 0) {
        for (int i = 0; i < ns; ++i) {
            mbar_init(smem_addr(full + i), 1);       // producer + tx bytes
            mbar_init(smem_addr(empty + i), nrt);    // the warps that own the chunk
        }
        for (int i = 0; i < nsl; ++i) {
            mbar_init(smem_addr(sfree + i), kConsumers);
            mbar_init(smem_addr(sfull + i), 1);
        }
        for (int i = 0; i < 2 * kMaxRowTiles; ++i) {
            mbar_init(smem_addr(rready + i), nks);   // the K-split warps of the row tile
            mbar_init(smem_addr(rfree + i), 1);      // the epilogue warp
        }
        for (int i = 0; i < ns; ++i) tags[i] = -1;
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    // experts of this band, in id order (every CTA derives the same list): one
    // expert per thread, a ballot per warp, a prefix over the warps
    int nact = 0;
    for (int e0 = 0; e0 < p.E; e0 += kThreads) {
        const int e = e0 + (int)threadIdx.x;
        bool act = false;
        int64_t o0 = 0, o1 = 0;
        if (e < p.E) {
            o0 = p.offsets[e];
            o1 = p.offsets[e + 1];
            act = (o1 - o0 >= p.m_lo) && (o1 - o0 <= p.m_hi);
        }
        const unsigned bal = __ballot_sync(0xffffffffu, act);
        if (lane == 0) s_wcnt[warp] = __popc(bal);
        __syncthreads();
        int before = nact, total = 0;
        for (int w = 0; w < kThreads / 32; ++w) {
            const int c = s_wcnt[w];
            if (w < warp) before += c;
            total += c;
        }
        if (act) {
            const int idx = before + __popc(bal & ((1u << lane) - 1u));
            s_active[idx] = e;
            s_r0[idx] = o0;
            s_cnt[idx] = (int)(o1 - o0);
        }
        nact += total;
        __syncthreads();
    }

    const int nit = (p.N + ROWS - 1) / ROWS;           // items per expert
    const int total = nact * nit;
    const int i0 = (int)((int64_t)blockIdx.x * total / gridDim.x);
    const int i1 = (int)((int64_t)(blockIdx.x + 1) * total / gridDim.x);
    const int nbk = p.K / SB;                          // scale blocks per weight row
    const int ssz = FMT == FMT_NF4 ? 4 : 1;

    // routed rows of this CTA's experts: one contiguous range [rlo, rhi)
    int64_t rlo = 0, rhi = 0;
    if (i0 < i1) {
        const int a0 = i0 / nit, a1 = (i1 - 1) / nit;
        rlo = s_r0[a0];
        rhi = s_r0[a1] + s_cnt[a1];
    }
    const bool table = (rhi - rlo) <= kMaxTableRows;

    const int nch = plan.nch;
    if (warp == kProducerWarp) {
        // ================= producer (one thread): starts right away =================
        if (lane == 0) {
            uint32_t ctr = 0, slot = 0, ph = 1;       // ring position; empty-barrier parity to wait on
            uint32_t sslot = 0, sph = 1;              // next scale slot to fill; its free-barrier parity
            int sa_ = (i1 > i0) ? i0 / nit : 0, sit = (i1 > i0) ? i0 % nit : 0;   // next item whose scales go out
            int s_next = i0;
            int a = sa_, it = sit;
            bool ok = true;
            for (int item = i0; item < i1 && ok; ++item) {
                // scales go out one item ahead: those of this item and of the next
                while (s_next < i1 && s_next <= item + 1) {
                    // an item's scales: its rows x all blocks, one contiguous range (a multiple of 16 bytes)
                    if (!mbar_wait_bounded(smem_addr(sfree + sslot), sph, abort_flag, &g_decode_error, 4u)) {
                        ok = false;
                        break;
                    }
                    const int se = s_active[sa_];
                    const int sn0 = sit * ROWS;
                    const uint32_t sbytes = (uint32_t)(min(ROWS, p.N - sn0) * nbk * ssz);
                    const uint8_t* ssrc = reinterpret_cast<const uint8_t*>(p.scales) + ((int64_t)se * p.N + sn0) * nbk * ssz;
                    const uint32_t sb = smem_addr(sfull + sslot);
                    mbar_arrive_tx(sb, sbytes);
                    bulk_1d(smem_addr(sslots + sslot * plan.scale_bytes), ssrc, sbytes, sb);
                    if (++sslot == (uint32_t)nsl) {
                        sslot = 0;
                        sph ^= 1u;
                    }
                    if (++sit == nit) {
                        sit = 0;
                        ++sa_;
                    }
                    ++s_next;
                }
                const int e = s_active[a];
                const int n0 = it * ROWS;
                const int npass = (s_cnt[a] + 8 * GMAX - 1) / (8 * GMAX);
                for (int pass = 0; pass < npass && ok; ++pass) {
                    for (int kc = 0; kc < nch; ++kc) {
                        if (!mbar_wait_bounded(smem_addr(empty + slot), ph, abort_flag, &g_decode_error, 1u)) {
                            ok = false;
                            break;
                        }
                        // the slot's previous chunk is consumed: name the chunk it now receives
                        asm volatile("st.release.cta.shared::cta.u32 [%0], %1;" ::"r"(smem_addr(tags + slot)), "r"(ctr)
                                     : "memory");
                        const uint32_t fb = smem_addr(full + slot);
                        mbar_arrive_tx(fb, (uint32_t)(kBoxBytes * ROWS));
                        tma_2d(smem_addr(ring + slot * plan.stage_bytes), &wmap, kc * (kChunkK / 2), e * p.N + n0, fb);
                        ++ctr;
                        if (++slot == (uint32_t)ns) {
                            slot = 0;
                            ph ^= 1u;
                        }
                    }
                }
                if (++it == nit) {
                    it = 0;
                    ++a;
                }
            }
        }
        __syncwarp();
        return;
    }

    // consumers and the epilogue warp, while the producer's first copies are in flight:
    // the byte -> bf16x2 table (one copy per lane: 8 sixteen-byte pieces per byte value)
    // and the routing metadata of the CTA's rows
    if (threadIdx.x < kConsumers * 32) {
        const LutPlanes Lt = p.lut;
        for (int i = threadIdx.x; i < 256 * 8; i += kConsumers * 32) {
            const int b = i >> 3, q = i & 7;
            const uint32_t v = byte_bf16x2<FMT>((uint32_t)b, Lt);
            *reinterpret_cast<uint4*>(lut + b * 256 + q * 16) = make_uint4(v, v, v, v);
        }
    }
    if (table) {
        for (int64_t r = rlo + threadIdx.x; r < rhi; r += kConsumers * 32)
            if (threadIdx.x < kConsumers * 32) {
                const int k = (int)(r - rlo);
                t_tok[k] = p.row_token ? __ldg(p.row_token + r) : (int)r;
                t_wt[k] = p.row_weight ? __ldg(p.row_weight + r) : 1.f;
                t_dst[k] = p.row_dest ? __ldg(p.row_dest + r) : (int)r;
            }
    }
    asm volatile("bar.sync 1, %0;" ::"r"((kConsumers + 1) * 32) : "memory");

    if (warp == kEpilogueWarp) {
        // ================= epilogue: fixed-order K-split sums, weight, bf16, scatter =================
        bool dead = false;
        uint32_t P = 0;                                 // pass counter of the CTA
        int a = (i1 > i0) ? i0 / nit : 0, it = (i1 > i0) ? i0 % nit : 0;
        for (int item = i0; item < i1; ++item) {
            const int m = s_cnt[a];
            const int n0 = it * ROWS;
            const int64_t r0 = s_r0[a];
            const int npass = (m + 8 * GMAX - 1) / (8 * GMAX);
            const int vrows = min(ROWS, p.N - n0);
            for (int pass = 0; pass < npass; ++pass, ++P) {
                const int mc = pass * 8 * GMAX;
                const int nvalid = min(8 * GMAX, m - mc);
                const int G = (nvalid + 7) >> 3;
                const uint32_t buf = P & 1u, ph = (P >> 1) & 1u;
                for (int rt = 0; rt < nrt; ++rt) {
                    const int bi = (int)buf * kMaxRowTiles + rt;
                    if (!dead && !mbar_wait_bounded(smem_addr(rready + bi), ph, abort_flag, &g_decode_error, 32u))
                        dead = true;
                    if (!dead) {
                        for (int q = lane; q < G * 32; q += 32) {
                            const int j = q >> 5, ln = q & 31;
                            float4 v = *red_slot(lut, (((int)buf * nrt + rt) * nks + 0) * GMAX + j, ln);
                            for (int k2 = 1; k2 < nks; ++k2) {
                                const float4 w = *red_slot(lut, (((int)buf * nrt + rt) * nks + k2) * GMAX + j, ln);
                                v.x += w.x; v.y += w.y; v.z += w.z; v.w += w.w;
                            }
                            const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                const int row = mc + 8 * j + 2 * (ln & 3) + (i & 1);       // C column 2t (+1)
                                const int nr = rt * 16 + (ln >> 2) + ((i & 2) ? 8 : 0);    // C row g (+8)
                                if (row < m && nr < vrows) {
                                    const int64_t r = r0 + row;
                                    float wgt;
                                    int64_t dst;
                                    if (table) {
                                        wgt = t_wt[r - rlo];
                                        dst = t_dst[r - rlo];
                                    } else {
                                        wgt = p.row_weight ? __ldg(p.row_weight + r) : 1.f;
                                        dst = p.row_dest ? (int64_t)__ldg(p.row_dest + r) : r;
                                    }
                                    p.out[dst * p.N + n0 + nr] = f32_to_bf16_rne(vv[i] * wgt);
                                }
                            }
                        }
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(smem_addr(rfree + bi));
                }
            }
            if (++it == nit) {
                it = 0;
                ++a;
            }
        }
        return;
    }

    // ================= consumers =================
    const int rt = warp % nrt, ks = warp / nrt;     // row tile, K split (chunks kc % nks == ks)
    const int g = lane >> 2, t = lane & 3;
    const int ra = rt * 16 + g, rb = ra + 8;        // the two item rows of this lane
    const uint32_t lane_sel = (uint32_t)lane * 4u;  // lut offset of this lane's copy
    const LutPlanes L = p.lut;                      // register tables for the permute decode
    const bool vec_scales = (FMT == FMT_NF4) ? (nbk % 4 == 0) : (nbk % 8 == 0);
    bool dead = false;   // set when a wait gives up: the warp then only keeps the barrier schedule
    float acc[GMAX][4];
#pragma unroll
    for (int j = 0; j < GMAX; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
    uint32_t base = 0;                              // chunk counter at the start of the pass
    uint32_t P = 0;                                 // pass counter of the CTA
    uint32_t sslot = 0, sph = 0;                    // scale slot; its full-barrier parity
    int a = (i1 > i0) ? i0 / nit : 0, it = (i1 > i0) ? i0 % nit : 0;
    for (int item = i0; item < i1; ++item) {
        const int m = s_cnt[a];
        const int64_t r0 = s_r0[a];
        const int npass = (m + 8 * GMAX - 1) / (8 * GMAX);
        // every warp waits for the item's scales (also those that own no chunk of it)
        if (!dead && !mbar_wait_bounded(smem_addr(sfull + sslot), sph, abort_flag, &g_decode_error, 8u))
            dead = true;
        const uint8_t* ss = sslots + sslot * plan.scale_bytes;
        for (int pass = 0; pass < npass; ++pass, ++P) {
            const int mc = pass * 8 * GMAX;
            const int nvalid = min(8 * GMAX, m - mc);   // routed rows of this pass
            // x rows of this lane's routed rows (8j + g of the pass), or null past the pass's end
            const uint16_t* xr0 = nullptr;
            const uint16_t* xr1 = nullptr;
            if (g < nvalid) {
                const int64_t r = r0 + mc + g;
                const int tk = table ? t_tok[r - rlo] : (p.row_token ? __ldg(p.row_token + r) : (int)r);
                xr0 = p.x + (int64_t)tk * p.K;
            }
            if (GMAX == 2 && 8 + g < nvalid) {
                const int64_t r = r0 + mc + 8 + g;
                const int tk = table ? t_tok[r - rlo] : (p.row_token ? __ldg(p.row_token + r) : (int)r);
                xr1 = p.x + (int64_t)tk * p.K;
            }
            int kc = ks;                                // chunks kc = ks, ks + nks, ...
            uint32_t ctr = base + (uint32_t)kc;
            uint32_t slot = ctr % (uint32_t)ns, ph = (ctr / (uint32_t)ns) & 1u;
            for (; kc < nch; kc += nks) {
                // bring this chunk's activations into L1 while the weights are on their way
                // (lane t of row g: the t-th 128-byte line of the row's 512-byte chunk)
                if (kc * kChunkK + t * 64 < p.K) {
                    if (xr0 != nullptr) prefetch_l1(xr0 + kc * kChunkK + t * 64);
                    if (xr1 != nullptr) prefetch_l1(xr1 + kc * kChunkK + t * 64);
                }
                if (!dead && !wait_tag(tags + slot, ctr, abort_flag, &g_decode_error, 16u)) dead = true;
                if (!dead && !mbar_wait_bounded(smem_addr(full + slot), ph, abort_flag, &g_decode_error, 2u))
                    dead = true;
                if (!dead) {
                    const uint8_t* st = ring + slot * plan.stage_bytes;
                    const int kb = kc * kChunkK;
                    if (p.K - kb >= kChunkK) {
                        if (GMAX == 2 && nvalid > 8)
                            chunk_mma<FMT, GMAX, (GMAX == 2 ? 2 : 1), true>(st, ss, lut, lane_sel, L, xr0, xr1, ra, rb, t, nbk, kc,
                                                                            0, vec_scales, acc);
                        else
                            chunk_mma<FMT, GMAX, 1, true>(st, ss, lut, lane_sel, L, xr0, xr1, ra, rb, t, nbk, kc, 0, vec_scales,
                                                          acc);
                    } else {
                        const int nbc = (p.K - kb) / SB;
                        chunk_mma<FMT, GMAX, GMAX, false>(st, ss, lut, lane_sel, L, xr0, xr1, ra, rb, t, nbk, kc, nbc, vec_scales,
                                                          acc);
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_addr(empty + slot));
                ctr += (uint32_t)nks;
                slot += (uint32_t)nks;                      // nks <= ns: at most one wrap
                if (slot >= (uint32_t)ns) {
                    slot -= (uint32_t)ns;
                    ph ^= 1u;
                }
            }
            base += (uint32_t)nch;
            // end of a pass: hand the partial sums to the epilogue warp
            const uint32_t buf = P & 1u, fph = ((P >> 1) & 1u) ^ 1u;
            const int bi = (int)buf * kMaxRowTiles + rt;
            if (!dead && !mbar_wait_bounded(smem_addr(rfree + bi), fph, abort_flag, &g_decode_error, 64u))
                dead = true;
            if (!dead) {
#pragma unroll
                for (int j = 0; j < GMAX; ++j)
                    *red_slot(lut, (((int)buf * nrt + rt) * nks + ks) * GMAX + j, lane) =
                        make_float4(acc[j][0], acc[j][1], acc[j][2], acc[j][3]);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_addr(rready + bi));
#pragma unroll
            for (int j = 0; j < GMAX; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
        }
        // every warp is done with this item's scales
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_addr(sfree + sslot));
        if (++sslot == (uint32_t)nsl) {
            sslot = 0;
            sph ^= 1u;
        }
        if (++it == nit) {
            it = 0;
            ++a;
        }
    }
}

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn_db() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

template <int FMT, int GMAX>
static cudaError_t launch_db(const GroupedArgs& a, cudaStream_t s) {
    using namespace db;
    const int SB = (FMT == FMT_NF4) ? 64 : 32;
    const int ssz = (FMT == FMT_NF4) ? 4 : 1;
    Plan plan;
    plan.nch = (a.K + kChunkK - 1) / kChunkK;
    const int tables = 96 + 16 * a.E + 12 * kMaxTableRows;
    int smem = 0;
    plan.rows = 0;
    for (int rows = 48; rows >= 16 && plan.rows == 0; rows -= 16) {
        const int stage_bytes = rows * kBoxBytes;       // 6, 4 or 2 KB: multiples of 1024
        const int scale_bytes = ((rows * (a.K / SB) * ssz + 127) / 128) * 128;
        const int nks = kConsumers * 16 / rows;          // K-split warps per row tile: the ring holds at least one chunk each
        for (int nst = 12; nst >= nks && plan.rows == 0; --nst) {
            for (int nsl = 3; nsl >= 2; --nsl) {
                const int need = 1024 + kLutBytes + nst * stage_bytes + nsl * scale_bytes +
                                 (2 * nst + 2 * nsl + 4 * kMaxRowTiles) * 8 + 4 * ((nst + 1) & ~1) + tables;
                if (need <= 226 * 1024) {
                    plan.rows = rows;
                    plan.stage_bytes = stage_bytes;
                    plan.scale_bytes = scale_bytes;
                    plan.nstages = nst;
                    plan.nslots = nsl;
                    smem = need;
                    break;
                }
            }
        }
    }
    if (plan.rows == 0) return cudaErrorInvalidValue;
    static int smem_set = 0;                 // largest dynamic shared memory opted in so far
    if (smem > smem_set) {
        cudaError_t e = cudaFuncSetAttribute(decode_band_kernel<FMT, GMAX>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        smem_set = smem;
    }
    auto enc = encode_fn_db();
    if (!enc) return cudaErrorNotSupported;
    // packed weights as bytes [E*N, K/2]: boxes of 128 bytes x rows, 128B swizzle
    CUtensorMap wmap;
    cuuint64_t dims[2] = {(cuuint64_t)(a.K / 2), (cuuint64_t)a.E * (cuuint64_t)a.N};
    cuuint64_t strides[1] = {(cuuint64_t)(a.K / 2)};
    cuuint32_t box[2] = {(cuuint32_t)kBoxBytes, (cuuint32_t)plan.rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(&wmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(a.W), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    const int64_t groups_max = a.R < (int64_t)a.E ? a.R : (int64_t)a.E;
    const int64_t items_max = groups_max * ((a.N + plan.rows - 1) / plan.rows);
    int64_t grid = device_sm_count();
    if (items_max < grid) grid = items_max;
    if (grid < 1) return cudaSuccess;
    decode_band_kernel<FMT, GMAX><<<(unsigned)grid, kThreads, smem, s>>>(a, plan, wmap);
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
