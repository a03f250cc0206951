// Decode band of the grouped 4-bit GEMM: groups with few routed rows, where
// the packed weight bytes are the whole cost (the GEMV path of the solution page
// "How do I run a grouped GEMM directly on NF4 packed MoE expert weights,
// without dequantizing to bf16 first?", "Supported scope": one-token groups
// take the GEMV path).
//
// One persistent CTA per SM takes a contiguous run of work items; an item is
// (active expert, ROWS = 64 weight rows; 32 when K is very large). A producer
// thread streams each item's packed rows, one K chunk of 512 at a time, into a
// ring of 16 KB shared-memory stages with 2-D TMA loads (boxes of 128 bytes x
// ROWS rows, 128B-swizzled), several stages ahead; big requests are what lets
// the copy engine keep HBM busy. The same stage also carries the chunk of each
// routed row's activations (1-D bulk copies, one per row), and the item's block
// scales (ROWS rows x all blocks, one contiguous range) arrive with its first
// chunk, so the consumers never wait on a global load. The CTA's routing
// metadata (token, weight, destination of each of its routed rows) is staged in
// shared memory once at the start.
//
// 16 consumer warps split an item as (ROWS/16 row tiles) x (16/(ROWS/16)) K
// splits of every chunk. Nibble pairs are decoded by a table in shared memory
// that maps each packed byte to its two bf16 values (one bf16x2 word),
// replicated per lane so that 32 lookups never conflict; a byte permute forms
// the lookup address. The products run on warp-level bf16 MMAs with 16 weight
// rows as the M side and up to 8 routed rows per MMA as the N side. Every MMA
// chain covers exactly one scale block (64 K for NF4, 32 K for MXFP4), so the
// block sum leaves the tensor core in fp32 and is scaled and accumulated in
// fp32 outside it. At the end of an item the K splits' partial sums are added
// in a fixed order through shared memory (deterministic), weighted, rounded to
// bf16 and stored at the destination rows.
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

constexpr int kConsumers = 16;                     // consumer warps
constexpr int kThreads = (kConsumers + 1) * 32;    // + one producer warp
constexpr int kChunkK = 512;                       // K per stage: 256 packed bytes per row
constexpr int kBoxBytes = 128;                     // TMA box width (one 128B swizzle row)
constexpr int kLutBytes = 256 * 256;               // byte value b, lane l -> offset b*256 + l*4
constexpr int kXStride = kChunkK * 2 + 16;         // bytes per staged activation row (padded)
constexpr int kMaxTableRows = 1024;                // routed rows whose metadata fits the CTA's table

struct Plan {
    int rows;         // weight rows per item (64 or 32)
    int nch;          // stages per item pass
    int wbytes;       // packed-weight part of a stage: rows x 256 bytes
    int stage_bytes;  // wbytes + activation rows (8*GMAX x kXStride)
    int scale_bytes;  // slot for one item's scales (rows x all blocks), rounded to 128
    int nstages;      // ring stages
    int nslots;       // item scale slots
};

struct Pos {
    int item, pass, kc;
};

__device__ __forceinline__ void tma_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar) : "memory");
}

}  // namespace db

template <int FMT, int GMAX>
__global__ void __launch_bounds__(db::kThreads, 1)
decode_band_kernel(const GroupedArgs p, const db::Plan plan, const __grid_constant__ CUtensorMap wmap) {
    using namespace db;
    constexpr int SB = (FMT == FMT_NF4) ? 64 : 32;   // K elements per scale block
    constexpr int STEPS = SB / 16;                   // k16 MMA steps per block
    constexpr int BPL = SB / 8;                      // packed bytes per lane per row per block (8 or 4)
    constexpr int XW = SB / 8;                       // bf16x2 words of x per lane per block
    constexpr int BPW = 4;                           // most blocks a warp takes from one chunk

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    // [lut][ring: stages x stage_bytes][scale slots][red][barriers][abort, count][experts]
    uint8_t* lut = smem;                                            // [256][64] words
    uint8_t* ring = smem + kLutBytes;                               // 1024-aligned stages
    uint8_t* sslots = ring + plan.nstages * plan.stage_bytes;
    float4* red = reinterpret_cast<float4*>(sslots + plan.nslots * plan.scale_bytes);
    uint64_t* bars = reinterpret_cast<uint64_t*>(red + kConsumers * GMAX * 32);   // full[s], empty[s]
    int* tailw = reinterpret_cast<int*>(bars + 2 * plan.nstages);
    volatile int* abort_flag = tailw;
    int* s_nact = tailw + 4;
    int64_t* s_r0 = reinterpret_cast<int64_t*>(tailw + 8);         // [E] first routed row
    int* s_active = reinterpret_cast<int*>(s_r0 + p.E);            // [E] expert id
    int* s_cnt = s_active + p.E;                                   // [E] routed rows
    int* t_tok = s_cnt + p.E;                                      // [kMaxTableRows] per routed row
    float* t_wt = reinterpret_cast<float*>(t_tok + kMaxTableRows);
    int* t_dst = reinterpret_cast<int*>(t_wt + kMaxTableRows);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ns = plan.nstages;
    const int ROWS = plan.rows;

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
        for (int i = 0; i < ns; ++i) {
            mbar_init(smem_addr(bars + i), 1);                 // full: producer + tx bytes
            mbar_init(smem_addr(bars + ns + i), kConsumers);   // empty: every consumer warp
        }
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    const int nit = (p.N + ROWS - 1) / ROWS;           // items per expert
    const int total = s_nact[0] * nit;
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
    if (table) {
        for (int64_t r = rlo + threadIdx.x; r < rhi; r += kThreads) {
            const int k = (int)(r - rlo);
            t_tok[k] = p.row_token ? __ldg(p.row_token + r) : (int)r;
            t_wt[k] = p.row_weight ? __ldg(p.row_weight + r) : 1.f;
            t_dst[k] = p.row_dest ? __ldg(p.row_dest + r) : (int)r;
        }
    }
    __syncthreads();
    auto tok_of = [&](int64_t r) -> int {
        return table ? t_tok[r - rlo] : (p.row_token ? __ldg(p.row_token + r) : (int)r);
    };

    auto advance = [&](Pos q) -> Pos {
        if (++q.kc == plan.nch) {
            q.kc = 0;
            const int m = s_cnt[q.item / nit];
            if (++q.pass == (m + 8 * GMAX - 1) / (8 * GMAX)) {
                q.pass = 0;
                ++q.item;
            }
        }
        return q;
    };

    if (warp == kConsumers) {
        // ================= producer (one thread) =================
        if (lane == 0) {
            uint32_t ctr = 0, jitem = 0;
            for (Pos ps{i0, 0, 0}; ps.item < i1; ps = advance(ps), ++ctr) {
                const uint32_t slot = ctr % ns, ph = ((ctr / ns) & 1u) ^ 1u;
                if (!mbar_wait_bounded(smem_addr(bars + ns + slot), ph, abort_flag, &g_decode_error, 1u)) break;
                const int a = ps.item / nit;
                const int e = s_active[a];
                const int n0 = (ps.item % nit) * ROWS;
                const int xb = ps.kc * (kChunkK / 2);                 // first packed byte of the chunk
                const int nbox = (p.K / 2 - xb) > kBoxBytes ? 2 : 1;  // the last chunk may be half
                const uint32_t fb = smem_addr(bars + slot);
                const bool first = ps.kc == 0 && ps.pass == 0;
                const int vrows = min(ROWS, p.N - n0);
                const uint32_t sbytes = (uint32_t)(vrows * nbk * ssz);   // a multiple of 16
                // activation rows of this pass: their chunk of K, one bulk copy each
                const int64_t r0 = s_r0[a];
                const int mc = ps.pass * 8 * GMAX;
                const int nx = min(8 * GMAX, s_cnt[a] - mc);
                const int kb = ps.kc * kChunkK;
                const uint32_t xbytes = (uint32_t)(min(kChunkK, p.K - kb) * 2);
                mbar_arrive_tx(fb, (uint32_t)(nbox * kBoxBytes * ROWS) + (uint32_t)nx * xbytes + (first ? sbytes : 0u));
                const uint32_t dst = smem_addr(ring + slot * plan.stage_bytes);
                for (int bx = 0; bx < nbox; ++bx)
                    tma_2d(dst + bx * kBoxBytes * ROWS, &wmap, xb + bx * kBoxBytes, e * p.N + n0, fb);
                for (int j = 0; j < nx; ++j) {
                    const int tk = tok_of(r0 + mc + j);
                    asm volatile(
                        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                        ::"r"(dst + plan.wbytes + j * kXStride), "l"(p.x + (int64_t)tk * p.K + kb), "r"(xbytes),
                          "r"(fb) : "memory");
                }
                if (first) {
                    // the item's scales: its rows x all blocks, one contiguous range
                    const uint8_t* ssrc = reinterpret_cast<const uint8_t*>(p.scales) +
                                          ((int64_t)e * p.N + n0) * nbk * ssz;
                    asm volatile(
                        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                        ::"r"(smem_addr(sslots + (jitem % plan.nslots) * plan.scale_bytes)), "l"(ssrc),
                          "r"(sbytes), "r"(fb) : "memory");
                    ++jitem;
                }
            }
        }
        __syncwarp();
    } else {
        // ================= consumers =================
        const int nrt = ROWS / 16, nks = kConsumers / nrt;
        const int rt = warp % nrt, ks = warp / nrt;     // row tile, K split
        const int g = lane >> 2, t = lane & 3;
        const int ra = rt * 16 + g, rb = ra + 8;        // the two item rows of this lane
        const uint32_t lane_sel = (uint32_t)lane * 4u;  // lut offset of this lane's copy
        uint32_t ctr = 0, jitem = 0;
        bool dead = false;   // set when a wait gives up: the warp then only keeps the barrier schedule
        float acc[GMAX][4];
        Pos cur{i0, 0, 0};
        while (cur.item < i1) {
            const int a = cur.item / nit;
            const int n0 = (cur.item % nit) * ROWS;
            const int64_t r0 = s_r0[a];
            const int m = s_cnt[a];
            const int mc = cur.pass * 8 * GMAX;
            const int G = min(GMAX, (m - mc + 7) >> 3);
            const Pos nxt = advance(cur);
            if (cur.kc == 0) {
#pragma unroll
                for (int j = 0; j < GMAX; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
            }
            const int kb = cur.kc * kChunkK;
            const int nbc = min(kChunkK, p.K - kb) / SB;
            const int b0 = ks * nbc / nks, b1 = (ks + 1) * nbc / nks;
            const uint32_t slot = ctr % ns, ph = (ctr / ns) & 1u;
            ++ctr;
            if (!dead && !mbar_wait_bounded(smem_addr(bars + slot), ph, abort_flag, &g_decode_error, 2u)) dead = true;
            const uint8_t* st = ring + slot * plan.stage_bytes;
            const uint8_t* ss = sslots + (jitem % plan.nslots) * plan.scale_bytes;
            const int bg0 = cur.kc * (kChunkK / SB);      // first scale block of the chunk
#pragma unroll
            for (int c = 0; c < BPW; ++c) {
                if (!dead && b0 + c < b1) {
                    const int b = b0 + c;
                    float s0, s1;
                    if constexpr (FMT == FMT_NF4) {
                        s0 = reinterpret_cast<const float*>(ss)[ra * nbk + bg0 + b];
                        s1 = reinterpret_cast<const float*>(ss)[rb * nbk + bg0 + b];
                    } else {
                        s0 = e8m0_to_f32(ss[ra * nbk + bg0 + b]);
                        s1 = e8m0_to_f32(ss[rb * nbk + bg0 + b]);
                    }
                    // this lane's packed bytes of rows ra and rb: byte o of the row's 256-byte
                    // chunk lives in box o/128, 16-byte piece ((o%128)/16) ^ (row%8)
                    const int o = b * (SB / 2) + t * BPL;
                    const uint8_t* bx = st + (o >> 7) * (kBoxBytes * ROWS);
                    const int pc = (o & 127) >> 4, po = o & 15;
                    const uint8_t* rp0 = bx + ra * kBoxBytes + ((pc ^ (ra & 7)) << 4) + po;
                    const uint8_t* rp1 = bx + rb * kBoxBytes + ((pc ^ (rb & 7)) << 4) + po;
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
                            // staged activations of routed row mc + 8j + g (rows past m hold stale
                            // data and only feed output columns that are never stored)
                            uint32_t xw[XW];
                            const uint8_t* xs = st + plan.wbytes + (8 * j + g) * kXStride + (b * SB + t * (SB / 4)) * 2;
#pragma unroll
                            for (int w = 0; w < XW / 4; ++w) {
                                const uint4 v = *reinterpret_cast<const uint4*>(xs + 16 * w);
                                xw[4 * w] = v.x; xw[4 * w + 1] = v.y; xw[4 * w + 2] = v.z; xw[4 * w + 3] = v.w;
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
            if (lane == 0) mbar_arrive(smem_addr(bars + ns + slot));
            if (cur.kc == plan.nch - 1) {
                // the K splits' partial sums, added in a fixed order, then the epilogue
#pragma unroll
                for (int j = 0; j < GMAX; ++j)
                    if (j < G) red[((ks * nrt + rt) * GMAX + j) * 32 + lane] =
                                   make_float4(acc[j][0], acc[j][1], acc[j][2], acc[j][3]);
                asm volatile("bar.sync 1, %0;" ::"n"(kConsumers * 32) : "memory");
                const int vrows = min(ROWS, p.N - n0);
                for (int qq = threadIdx.x; qq < nrt * G * 128; qq += kConsumers * 32) {
                    const int i = qq & 3, ln = (qq >> 2) & 31, rest = qq >> 7;
                    const int j = rest % G, rtt = rest / G;
                    const int row = mc + 8 * j + 2 * (ln & 3) + (i & 1);     // C column 2t (+1)
                    const int nr = rtt * 16 + (ln >> 2) + ((i & 2) ? 8 : 0);  // C row g (+8)
                    if (row < m && nr < vrows) {
                        float v = 0.f;
                        for (int k2 = 0; k2 < nks; ++k2)
                            v += reinterpret_cast<const float*>(&red[((k2 * nrt + rtt) * GMAX + j) * 32 + ln])[i];
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
                        p.out[dst * p.N + n0 + nr] = f32_to_bf16_rne(v * wgt);
                    }
                }
                asm volatile("bar.sync 1, %0;" ::"n"(kConsumers * 32) : "memory");
                if (nxt.item != cur.item) ++jitem;
            }
            cur = nxt;
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
    const int red_bytes = kConsumers * GMAX * 32 * (int)sizeof(float4);
    const int tables = 32 + 16 * a.E + 12 * kMaxTableRows;
    int smem = 0;
    plan.rows = 0;
    for (int rows = 64; rows >= 32 && plan.rows == 0; rows >>= 1) {
        const int wbytes = rows * (kChunkK / 2);
        const int stage_bytes = wbytes + ((8 * GMAX * kXStride + 1023) / 1024) * 1024;
        const int scale_bytes = ((rows * (a.K / SB) * ssz + 127) / 128) * 128;
        for (int nst = 6; nst >= 3; --nst) {
            const int nsl = (nst - 1 + plan.nch - 1) / plan.nch + 1;   // items in flight at once
            const int need = 1024 + kLutBytes + nst * stage_bytes + nsl * scale_bytes + red_bytes + 2 * nst * 8 + tables;
            if (need <= 226 * 1024) {
                plan.rows = rows;
                plan.wbytes = wbytes;
                plan.stage_bytes = stage_bytes;
                plan.scale_bytes = scale_bytes;
                plan.nstages = nst;
                plan.nslots = nsl;
                smem = need;
                break;
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
