#include <atomic>
// Prefill band of the grouped 4-bit GEMM: groups with many routed rows, where
// the work is a dense contraction and runs on the 5th-generation tensor cores
// (tcgen05, accumulators in tensor memory). The M-tile path of the solution
// page "How do I run a grouped GEMM directly on NF4 packed MoE expert
// weights, without dequantizing to bf16 first?" ("Supported scope": larger
// groups take the M-tile path), redesigned for sm_100a.
//
// Tile = 128 weight rows (the MMA's M side, one tensor-memory lane each) x up
// to 128 routed rows of one expert (the N side), all of K. Persistent CTAs walk
// the tiles of every expert in the band, computed on the device from the
// expert offsets. Roles (23 warps, 80 registers a thread):
//   warp 0      tensor-memory owner and MMA issuer (one thread)
//   warp 1      activation loader: TMA tile loads of contiguous rows, or
//               16-byte cp.async copies (all 32 lanes) of the rows named by
//               row_token, both into the 128B-swizzled K-major layout
//   warp 2      packed-weight loader: TMA loads of the tile's 128 rows x 32
//               bytes per 64 K into a deep ring of its own
//   warps 3-6   decoders: one weight row per thread (its tensor-memory lane);
//               nibbles -> bf16 by byte permutes, stored straight into the MMA's
//               A operand in tensor memory (tcgen05.st), so the decoded tile
//               never touches shared memory
//   warps 7-22  rescale epilogue, four warps per tensor-memory lane quadrant, 32
//               of the tile's columns each: per scale block, read the block's
//               fp32 sums from tensor memory, multiply by the block scale
//               (fetched four blocks ahead)
//               and add into fp32 running sums held in registers; at the end of
//               a tile, weight and round, stage the tile's outputs in shared
//               memory (two buffers), meet once on an mbarrier, and send each
//               routed row's slice to its destination row with one bulk copy, so
//               the warps go on to the next tile while the copies drain
// The MMA (A from tensor memory, B from shared memory) chain of each scale block
// (64 K for NF4, 32 K for MXFP4) goes to one of three tensor-memory accumulators,
// so the scale is applied in fp32 outside the MMA while the tensor core fills
// the next ones. Tensor memory: 3 x 128 accumulator columns + 4 x 32 operand
// columns = 512.
//
// Every wait on a barrier is bounded: after ~2^32 cycles without progress the
// CTA records an error in g_prefill_error, stops its roles and returns.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <climits>
#include <cstdint>

#include "gnf4_common.cuh"
#include "gnf4_kernels.h"

namespace gnf4 {

__device__ unsigned g_prefill_error;

namespace pf {

constexpr int kThreads = 23 * 32;  // see the role list above
constexpr int kBM = 128;             // weight rows per tile
constexpr int kBNMax = 128;          // routed rows per tile (MMA N)
constexpr int kStages = 4;           // pipeline stages: B (activations) in shared memory, A slots in tensor memory
constexpr int kWStages = 12;         // packed-weight stages (128 rows x 32 bytes)
constexpr int kAccBufs = 3;          // tensor-memory block accumulators of kBNMax columns
constexpr int kACol0 = kAccBufs * kBNMax;   // first tensor-memory column of the A operand slots
constexpr int kKStage = 64;          // K per pipeline stage (one 128-byte swizzle row of bf16)
constexpr int kAColsPerStage = kKStage / 2;  // 64 K of bf16 pairs = 32 tensor-memory columns per stage
constexpr int kBStageBytes = kBNMax * 128;
constexpr int kWStageBytes = kBM * 32;
constexpr int kMaxExperts = 2048;
constexpr int kDecWarp0 = 3;         // decoders: warps 3-6
constexpr int kDecWarps = 4;
constexpr int kEpiWarp0 = 7;         // epilogue: warps 7-22
constexpr int kEpiWarps = 16;
constexpr int kScaleAhead = 4;       // block scales held ahead in epilogue registers

// shared memory map (offsets from a 1024-aligned base)
constexpr int kOffB = 0;
constexpr int kOffW = kOffB + kStages * kBStageBytes;
constexpr int kOffBar = kOffW + kWStages * kWStageBytes;
constexpr int kNumBars = 3 * kStages + 2 * kWStages + 2 * kAccBufs + 1;
constexpr int kOffTmem = kOffBar + kNumBars * 8;
constexpr int kOffAbort = kOffTmem + 4;
constexpr int kOffRows = kOffTmem + 16;                       // int[kBNMax] gathered rows of the loader's tile
constexpr int kOffList = kOffRows + kBNMax * 4;               // int[kMaxExperts] experts of the band
constexpr int kOffCum = kOffList + kMaxExperts * 4;           // int[kMaxExperts+1] tile prefix
constexpr int kOffCount = kOffCum + (kMaxExperts + 1) * 4;
// a tile's outputs, staged for the bulk stores: [routed row][weight row] rounded values,
// two tiles deep (the stores of one tile drain while the next is computed)
constexpr int kOutRowBytes = kBM * 2;
constexpr int kOutBufBytes = kBNMax * kOutRowBytes;
constexpr int kOffOut = (kOffCount + 16 + 127) & ~127;
constexpr int kSmemBytes = kOffOut + 2 * kOutBufBytes + 1024;  // + alignment slack

struct Tile {
    int e;          // expert
    int64_t r0;     // first routed row of the tile
    int cnt;        // routed rows in the tile (<= kBNMax)
    int bn;         // MMA N: cnt rounded up to 16
    int n0;         // first weight row
};

__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// UMMA shared-memory descriptor: K-major, 128-byte swizzle, 8-row groups 1024 B apart.
__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr) {
    uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)1 << 16;                 // leading byte offset (unused for swizzled K-major)
    d |= (uint64_t)(1024 >> 4) << 32;       // stride byte offset
    d |= (uint64_t)1 << 46;                 // descriptor version
    d |= (uint64_t)2 << 61;                 // SWIZZLE_128B
    return d;
}

// Instruction descriptor, kind::f16: A and B both bf16 (XH = 0) or both fp16 (XH = 1),
// fp32 D, both K-major, M = 128.
template <int XH>
__device__ __forceinline__ uint32_t idesc_f16kind(int n) {
    const uint32_t ab = (XH == 0) ? ((1u << 7) | (1u << 10)) : 0u;   // operand formats: 1 = bf16, 0 = f16
    return (1u << 4) | ab | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);
}

__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n"
        ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate) : "memory");
}
// D (tensor memory) (+)= A (tensor memory: row i in lane i, K pairs along columns) x B (shared memory)
__device__ __forceinline__ void mma_bf16_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n"
        ::"r"(tmem_d), "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate) : "memory");
}
// 16 consecutive 32-bit columns written for this warp's 32 lanes
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
        ::"r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
          "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tma_tile_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar) : "memory");
}
// 16-byte asynchronous copy global -> shared; bytes past src_bytes (0 or 16) are zero-filled
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
// arrive on the barrier once this thread's earlier cp.async copies have landed
__device__ __forceinline__ void cp_async_arrive(uint32_t bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// shared -> global bulk copy (async proxy), tracked by this thread's bulk groups
__device__ __forceinline__ void bulk_store(void* gdst, uint32_t ssrc, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;"
                 ::"l"(reinterpret_cast<uint64_t>(gdst)), "r"(ssrc), "r"(bytes) : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// every bulk group of this thread has finished reading shared memory
__device__ __forceinline__ void bulk_wait_read_all() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// acc[0..1] += v[0..1] * s, as one packed fp32x2 FMA
__device__ __forceinline__ void ffma2(float& a0, float& a1, uint32_t v0, uint32_t v1, float s) {
    uint64_t acc = ((uint64_t)__float_as_uint(a1) << 32) | __float_as_uint(a0);
    const uint64_t vv = ((uint64_t)v1 << 32) | v0;
    const uint64_t ss = ((uint64_t)__float_as_uint(s) << 32) | __float_as_uint(s);
    asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(vv), "l"(ss));
    a0 = __uint_as_float((uint32_t)acc);
    a1 = __uint_as_float((uint32_t)(acc >> 32));
}

struct Sched {
    const int* list;
    const int* cum;
    int count;
    int total;
};

__device__ __forceinline__ Tile tile_at(const GroupedArgs& p, const Sched& s, int t, int nnt) {
    // expert i of the band with cum[i] <= t < cum[i+1]
    int lo = 0, hi = s.count - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s.cum[mid] <= t) lo = mid; else hi = mid - 1;
    }
    Tile tl;
    tl.e = s.list[lo];
    const int local = t - s.cum[lo];
    const int64_t base = p.offsets[tl.e];
    const int m = (int)(p.offsets[tl.e + 1] - base);
    const int ntt = (m + kBNMax - 1) / kBNMax;
    const int tpt = (m + ntt - 1) / ntt;
    const int tt = local / nnt;
    tl.n0 = (local % nnt) * kBM;
    tl.r0 = base + (int64_t)tt * tpt;
    tl.cnt = min(tpt, m - tt * tpt);
    tl.bn = (tl.cnt + 15) & ~15;
    return tl;
}

}  // namespace pf

template <int FMT, bool SBF16, int XH>
__global__ void __maxnreg__(80)
prefill_band_kernel(const GroupedArgs p, const __grid_constant__ CUtensorMap xmap,
                    const __grid_constant__ CUtensorMap wmap,
                    const int gather) {
    using namespace pf;
    constexpr int SB = (FMT == FMT_NF4) ? 64 : 32;      // scale block
    constexpr int SBPS = kKStage / SB;                  // scale blocks per stage (1 or 2)
    constexpr int K16PSB = SB / 16;                     // k16 MMAs per scale block

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_addr(smem);
    const uint32_t bar_afull = sbase + kOffBar;                  // [kStages] decoders -> MMA
    const uint32_t bar_bfull = bar_afull + 8 * kStages;          // [kStages] activation loaders -> MMA
    const uint32_t bar_empty = bar_bfull + 8 * kStages;          // [kStages] MMA -> decoders, loaders
    const uint32_t bar_wfull = bar_empty + 8 * kStages;          // [kWStages] weight loader -> decoders
    const uint32_t bar_wempty = bar_wfull + 8 * kWStages;        // [kWStages] decoders -> weight loader
    const uint32_t bar_accfull = bar_wempty + 8 * kWStages;      // [kAccBufs] MMA -> epilogue
    const uint32_t bar_accempty = bar_accfull + 8 * kAccBufs;    // [kAccBufs] epilogue -> MMA
    const uint32_t bar_ostaged = bar_accempty + 8 * kAccBufs;    // epilogue warps: a tile's outputs are staged
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffAbort);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffTmem);
    int* s_list = reinterpret_cast<int*>(smem + kOffList);
    int* s_cum = reinterpret_cast<int*>(smem + kOffCum);
    int* s_count = reinterpret_cast<int*>(smem + kOffCount);
    unsigned* err = &g_prefill_error;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nnt = (p.N + kBM - 1) / kBM;
    const int nst = p.K / kKStage + ((p.K % kKStage) ? 1 : 0);   // stages per tile (last may be half, MXFP4)

    // ---- set-up: band experts and tile prefix (warp 1), barriers (warp 2), tensor memory (warp 0)
    if (warp == 1) {
        int count = 0, tiles = 0;
        for (int e0 = 0; e0 < p.E; e0 += 32) {
            const int e = e0 + lane;
            int m = 0;
            bool act = false;
            if (e < p.E) {
                m = (int)(p.offsets[e + 1] - p.offsets[e]);
                act = (m >= p.m_lo) && (m <= p.m_hi);
            }
            const int nt = act ? ((m + kBNMax - 1) / kBNMax) * nnt : 0;
            int inc = nt;                        // inclusive scan of tile counts across the warp
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, inc, o);
                if (lane >= o) inc += v;
            }
            const unsigned bal = __ballot_sync(0xffffffffu, act);
            if (act) {
                const int idx = count + __popc(bal & ((1u << lane) - 1u));
                s_list[idx] = e;
                s_cum[idx] = tiles + inc - nt;
            }
            count += __popc(bal);
            tiles += __shfl_sync(0xffffffffu, inc, 31);
        }
        if (lane == 0) {
            s_cum[count] = tiles;
            s_count[0] = count;
            s_count[1] = tiles;
        }
    } else if (warp == 2 && lane == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(bar_afull + 8 * i, kDecWarps);            // one arrival per decoder warp
            mbar_init(bar_bfull + 8 * i, gather ? 32 : 1);   // gather: one arrival per loader lane
            mbar_init(bar_empty + 8 * i, 1);
        }
        for (int i = 0; i < kWStages; ++i) {
            mbar_init(bar_wfull + 8 * i, 1);
            mbar_init(bar_wempty + 8 * i, kDecWarps);
        }
        for (int i = 0; i < kAccBufs; ++i) {
            mbar_init(bar_accfull + 8 * i, 1);
            mbar_init(bar_accempty + 8 * i, kEpiWarps);
        }
        mbar_init(bar_ostaged, kEpiWarps);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    // a CTA without a tile (no group of the band, or more CTAs than tiles) leaves
    // before it takes tensor memory
    if ((int)blockIdx.x >= s_count[1]) return;
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;"
                     ::"r"(smem_addr(tmem_slot)) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    Sched sch{s_list, s_cum, s_count[0], s_count[1]};

    if (warp == 0) {
        // ================= MMA issuer =================
        if (lane == 0) {
            uint32_t stage_ctr = 0, acc_ctr = 0;
            for (int t = blockIdx.x; t < sch.total; t += gridDim.x) {
                const Tile tl = tile_at(p, sch, t, nnt);
                const uint32_t idesc = idesc_f16kind<XH>(tl.bn);
                for (int s = 0; s < nst; ++s, ++stage_ctr) {
                    const uint32_t slot = stage_ctr % kStages, ph = (stage_ctr / kStages) & 1u;
                    if (!mbar_wait_bounded(bar_afull + 8 * slot, ph, abort_flag, err, 1u)) goto mma_done;
                    if (!mbar_wait_bounded(bar_bfull + 8 * slot, ph, abort_flag, err, 2u)) goto mma_done;
                    // gathered rows were written by cp.async (generic proxy): order them before the MMA reads
                    if (gather) fence_proxy_async();
                    tc_fence_after();
                    const uint32_t a_col = tmem + kACol0 + slot * kAColsPerStage;
                    const uint32_t b_addr = sbase + kOffB + slot * kBStageBytes;
                    const int nsb = min(SBPS, (p.K - s * kKStage) / SB);
                    for (int sb = 0; sb < nsb; ++sb, ++acc_ctr) {
                        const uint32_t buf = acc_ctr % kAccBufs, aph = ((acc_ctr / kAccBufs) & 1u) ^ 1u;
                        if (!mbar_wait_bounded(bar_accempty + 8 * buf, aph, abort_flag, err, 4u)) goto mma_done;
                        tc_fence_after();
#pragma unroll
                        for (int q = 0; q < K16PSB; ++q) {
                            const uint32_t koff = (uint32_t)(sb * K16PSB + q) * 32u;
                            mma_bf16_ts(tmem + buf * kBNMax, a_col + (uint32_t)(sb * K16PSB + q) * 8u, desc_sw128(b_addr + koff),
                                     idesc, q > 0 ? 1u : 0u);
                        }
                        mma_commit(bar_accfull + 8 * buf);
                    }
                    mma_commit(bar_empty + 8 * slot);
                }
            }
        }
    mma_done:
        __syncwarp();
    } else if (warp == 1) {
        // ================= activation loader =================
        // contiguous routed rows: one TMA tile load of 128 rows x 64 K. Rows named by
        // row_token: the warp's 32 lanes copy 16-byte pieces with cp.async (TMA gathers of
        // 128-byte rows are bound by their request rate). Both land 128B-swizzled, as the
        // MMA reads them.
        int* s_rows = reinterpret_cast<int*>(smem + kOffRows);
        uint32_t stage_ctr = 0;
        for (int t = blockIdx.x; t < sch.total; t += gridDim.x) {
            const Tile tl = tile_at(p, sch, t, nnt);
            if (gather) {
                // the tile's rows; padding rows repeat the tile's first row
                __syncwarp();
                for (int row = lane; row < tl.bn; row += 32)
                    s_rows[row] = __ldg(p.row_token + tl.r0 + (row < tl.cnt ? row : 0));
                __syncwarp();
                for (int s = 0; s < nst; ++s, ++stage_ctr) {
                    const uint32_t slot = stage_ctr % kStages, ph = ((stage_ctr / kStages) & 1u) ^ 1u;
                    if (!mbar_wait_bounded(bar_empty + 8 * slot, ph, abort_flag, err, 8u)) goto load_done;
                    const uint32_t dst = sbase + kOffB + slot * kBStageBytes;
                    const int kk = s * kKStage;
                    const int kvalid = min(kKStage, p.K - kk);       // 64, or 32 at an MXFP4 tail
                    for (int q = lane; q < tl.bn * 8; q += 32) {      // piece c of row r: K elements 8c .. 8c+7
                        const int r = q >> 3, c = q & 7;
                        const bool in = c * 8 < kvalid;
                        const uint16_t* src = p.x + (int64_t)s_rows[r] * p.K + kk + (in ? c * 8 : 0);
                        cp_async16(dst + r * 128 + ((c ^ (r & 7)) << 4), src, in ? 16u : 0u);
                    }
                    cp_async_arrive(bar_bfull + 8 * slot);
                }
            } else if (lane == 0) {
                for (int s = 0; s < nst; ++s, ++stage_ctr) {
                    const uint32_t slot = stage_ctr % kStages, ph = ((stage_ctr / kStages) & 1u) ^ 1u;
                    if (!mbar_wait_bounded(bar_empty + 8 * slot, ph, abort_flag, err, 8u)) goto load_done;
                    // one box of 128 rows (rows past the tile are loaded and never used)
                    const uint32_t full = bar_bfull + 8 * slot;
                    mbar_arrive_tx(full, (uint32_t)kBStageBytes);
                    tma_tile_2d(sbase + kOffB + slot * kBStageBytes, &xmap, s * kKStage, (int)tl.r0, full);
                }
            } else {
                stage_ctr += nst;
            }
        }
    load_done:
        __syncwarp();
    } else if (warp == 2) {
        // ================= packed-weight loader (TMA) =================
        if (lane == 0) {
            uint32_t ctr = 0;
            for (int t = blockIdx.x; t < sch.total; t += gridDim.x) {
                const Tile tl = tile_at(p, sch, t, nnt);
                const int row0 = tl.e * p.N + tl.n0;
                for (int s = 0; s < nst; ++s, ++ctr) {
                    const uint32_t slot = ctr % kWStages, ph = ((ctr / kWStages) & 1u) ^ 1u;
                    if (!mbar_wait_bounded(bar_wempty + 8 * slot, ph, abort_flag, err, 16u)) goto wload_done;
                    const uint32_t full = bar_wfull + 8 * slot;
                    mbar_arrive_tx(full, (uint32_t)kWStageBytes);
                    tma_tile_2d(sbase + kOffW + slot * kWStageBytes, &wmap, s * 32, row0, full);
                }
            }
        }
    wload_done:
        __syncwarp();
    } else if (warp >= kDecWarp0 && warp < kDecWarp0 + kDecWarps) {
        // ================= decoders: one weight row per thread (its tensor-memory lane) =================
        const int i = (warp & 3) * 32 + lane;              // tile row = tensor-memory lane (quadrant warp % 4)
        const uint32_t tlane = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        const LutPlanes L = p.lut;                         // decode tables in registers
        uint32_t stage_ctr = 0;
        for (int t = blockIdx.x; t < sch.total; t += gridDim.x) {
            for (int s = 0; s < nst; ++s, ++stage_ctr) {
                // packed bytes of this row for this stage (64 K = 32 bytes), from the weight ring
                const uint32_t wslot = stage_ctr % kWStages, wph = (stage_ctr / kWStages) & 1u;
                // (waits are made warp-uniform: the tensor-memory stores below need the whole warp)
                if (!__all_sync(0xffffffffu, mbar_wait_bounded(bar_wfull + 8 * wslot, wph, abort_flag, err, 32u)))
                    goto dec_done;
                // the row's 32 bytes as two 16-byte halves; lanes 4..7 of every 8 read the second
                // half first, so that the 8 rows of a group of lanes cover all 32 banks and
                // each load is 4 wavefronts (rows are 32 bytes apart)
                const uint8_t* wrow = smem + kOffW + wslot * kWStageBytes + i * 32;
                const int sw = (lane >> 2) & 1;
                const uint4 q0 = *reinterpret_cast<const uint4*>(wrow + 16 * sw);
                const uint4 q1 = *reinterpret_cast<const uint4*>(wrow + 16 * (sw ^ 1));
                const uint4 c0 = sw ? q1 : q0;
                const uint4 c1 = sw ? q0 : q1;
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_wempty + 8 * wslot);
                const uint32_t slot = stage_ctr % kStages, ph = ((stage_ctr / kStages) & 1u) ^ 1u;
                const uint32_t acol = tlane + kACol0 + slot * kAColsPerStage;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {       // the row in two halves of 32 K = 16 columns each
                    const uint4 cw = hh == 0 ? c0 : c1;
                    const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
                    uint32_t o[4][4];
#pragma unroll
                    for (int c = 0; c < 4; ++c) decode_word<FMT>(words[c], L, o[c]);
                    if (hh == 0) {
                        // the operand slot is free once the MMAs that read it have completed
                        if (!__all_sync(0xffffffffu, mbar_wait_bounded(bar_empty + 8 * slot, ph, abort_flag, err, 64u)))
                            goto dec_done;
                        tc_fence_after();
                    }
                    const uint32_t v[16] = {o[0][0], o[0][1], o[0][2], o[0][3], o[1][0], o[1][1], o[1][2], o[1][3],
                                            o[2][0], o[2][1], o[2][2], o[2][3], o[3][0], o[3][1], o[3][2], o[3][3]};
                    tmem_st16(acol + 16 * hh, v);      // columns: K pairs of this half, in order
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_afull + 8 * slot);
            }
        }
    dec_done:;
    } else if (warp >= kEpiWarp0) {
        // ================= rescale epilogue =================
        const int q4 = warp & 3;                      // tensor-memory lane quadrant
        const int cq = (warp - kEpiWarp0) >> 2;       // its 16-column chunks: cq and cq + 4
        const int i = q4 * 32 + lane;                 // tile row = tensor-memory lane
        const int nsbk = p.K / SB;                    // scale blocks per row
        uint32_t acc_ctr = 0, tile_ctr = 0;
        float acc[2][16];
        for (int t = blockIdx.x; t < sch.total; t += gridDim.x) {
            const Tile tl = tile_at(p, sch, t, nnt);
            const int n = tl.n0 + i;
            const bool valid = n < p.N;
            const int64_t srow = ((int64_t)tl.e * p.N + (valid ? n : 0)) * nsbk;
            const int nck = tl.bn >> 4;
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int c = 0; c < 16; ++c) acc[j][c] = 0.f;
            float sring[kScaleAhead];                 // scales of blocks b .. b+kScaleAhead-1
#pragma unroll
            for (int u = 0; u < kScaleAhead; ++u) sring[u] = (u < nsbk) ? load_scale<FMT, SBF16>(p.scales, srow + u) : 0.f;
            for (int b0 = 0; b0 < nsbk; b0 += kScaleAhead) {
#pragma unroll
                for (int u = 0; u < kScaleAhead; ++u) {
                    const int b = b0 + u;
                    if (b < nsbk) {
                        const float sc = sring[u];
                        if (b + kScaleAhead < nsbk) sring[u] = load_scale<FMT, SBF16>(p.scales, srow + b + kScaleAhead);
                        const uint32_t buf = acc_ctr % kAccBufs, ph = (acc_ctr / kAccBufs) & 1u;
                        ++acc_ctr;
                        if (!__all_sync(0xffffffffu, mbar_wait_bounded(bar_accfull + 8 * buf, ph, abort_flag, err, 128u)))
                            goto epi_done;
                        tc_fence_after();
                        const uint32_t taddr = tmem + ((uint32_t)(q4 * 32) << 16) + buf * kBNMax;
#pragma unroll
                        for (int j = 0; j < 2; ++j) {
                            // 16-column chunk cq + 4j (warp-uniform condition)
                            const int cc = cq + 4 * j;
                            if (cc < nck) {
                                uint32_t v[16];
                                tmem_ld16(taddr + cc * 16, v);
                                tmem_wait_ld();
#pragma unroll
                                for (int c = 0; c < 16; c += 2) ffma2(acc[j][c], acc[j][c + 1], v[c], v[c + 1], sc);
                            }
                        }
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(bar_accempty + 8 * buf);
                    }
                }
            }
            // outputs of this tile: weight row n of routed rows r0 .. r0+cnt-1. Each thread
            // stages its rounded values in [routed row][weight row] order (a warp's 32 lanes
            // write 64 contiguous bytes); then routed row c's slice of up to 128 weight rows,
            // contiguous in the output, goes out with one bulk copy (thread c), so the warps
            // return to the next tile's blocks while the copies drain. The epilogue warps meet
            // once a tile, on an mbarrier (bounded, warp-uniform waits: an abort anywhere leaves
            // no warp waiting forever). Before arriving, each thread waits until its copies of
            // the tile before have read their source; so when the meeting completes, the
            // buffer this tile's writes will reuse two tiles on is free.
            const uint32_t obuf = sbase + kOffOut + (uint32_t)(tile_ctr & 1) * kOutBufBytes;
            const uint32_t oph = tile_ctr & 1u;
            if (valid) {
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int c0 = cq + 4 * j;
                    if (c0 < nck) {
#pragma unroll
                        for (int c = 0; c < 16; ++c) {
                            const int slot = c0 * 16 + c;
                            if (slot < tl.cnt) {
                                float v = acc[j][c];
                                if (p.row_weight) v *= __ldg(p.row_weight + tl.r0 + slot);
                                const uint16_t h = f32_to_out16<XH>(v);
                                asm volatile("st.shared.u16 [%0], %1;" ::"r"(obuf + (uint32_t)slot * kOutRowBytes + (uint32_t)i * 2u),
                                             "h"(h) : "memory");
                            }
                        }
                    }
                }
            }
            fence_proxy_async();
            bulk_wait_read_all();                     // this thread's earlier copies have read their source
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_ostaged);
            if (!__all_sync(0xffffffffu, mbar_wait_bounded(bar_ostaged, oph, abort_flag, err, 256u))) goto epi_done;
            {
                const int c = (warp - kEpiWarp0) * 32 + lane;      // one routed row per thread
                if (c < tl.cnt) {
                    const int64_t r = tl.r0 + c;
                    const int64_t dst = p.row_dest ? (int64_t)__ldg(p.row_dest + r) : r;
                    const uint32_t bytes = (uint32_t)min(kBM, p.N - tl.n0) * 2u;
                    bulk_store(p.out + dst * p.N + tl.n0, obuf + (uint32_t)c * kOutRowBytes, bytes);
                }
                bulk_commit();
            }
            ++tile_ctr;
        }
    epi_done:
        bulk_wait_all();                              // every output copy has landed
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
    }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

template <int FMT, bool SBF16, int XH>
static cudaError_t launch_pf(const GroupedArgs& a, int64_t T_in, cudaStream_t s) {
    static std::atomic<bool> configured[64];         // per device: dynamic shared memory opted in
    const int dev = current_device();
    if (!configured[dev].load(std::memory_order_acquire)) {
        cudaError_t e = cudaFuncSetAttribute(prefill_band_kernel<FMT, SBF16, XH>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             pf::kSmemBytes);
        if (e != cudaSuccess) return e;
        configured[dev].store(true, std::memory_order_release);
    }
    auto enc = encode_fn();
    if (!enc) return cudaErrorNotSupported;
    const int gather = a.row_token != nullptr;
    CUtensorMap xmap, wmap;
    {
        // activations: bf16 or fp16 [T_in, K], boxes of 64 K x 128 rows, 128B swizzle
        cuuint64_t dims[2] = {(cuuint64_t)a.K, (cuuint64_t)T_in};
        cuuint64_t strides[1] = {(cuuint64_t)a.K * 2};
        cuuint32_t box[2] = {64, (cuuint32_t)pf::kBNMax};
        cuuint32_t estr[2] = {1, 1};
        CUresult r = enc(&xmap, XH ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                         const_cast<uint16_t*>(a.x), dims, strides, box,
                         estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    }
    {
        // packed weights: bytes [E*N, K/2], boxes of 32 bytes x 128 rows, no swizzle
        cuuint64_t dims[2] = {(cuuint64_t)(a.K / 2), (cuuint64_t)a.E * (cuuint64_t)a.N};
        cuuint64_t strides[1] = {(cuuint64_t)(a.K / 2)};
        cuuint32_t box[2] = {32, pf::kBM};
        cuuint32_t estr[2] = {1, 1};
        CUresult r = enc(&wmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(a.W), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    }
    // no more CTAs than the R routed rows can form tiles: groups of more than m_lo - 1
    // rows number at most R / m_lo, and their token tiles at most R / kBNMax + R / m_lo
    const int64_t mlo = a.m_lo > 1 ? a.m_lo : 1;
    const int64_t max_tiles = (int64_t)((a.N + pf::kBM - 1) / pf::kBM) * (a.R / pf::kBNMax + a.R / mlo + 1);
    int grid = device_sm_count();
    if (max_tiles < grid) grid = (int)max_tiles;
    prefill_band_kernel<FMT, SBF16, XH><<<grid, pf::kThreads, pf::kSmemBytes, s>>>(a, xmap, wmap, gather);
    return cudaGetLastError();
}

cudaError_t launch_prefill_band(int fmt, const GroupedArgs& a, int64_t T_in, cudaStream_t s) {
    if (fmt == FMT_NF4) {
        if (a.scale_bf16) return a.x_f16 ? launch_pf<FMT_NF4, true, 1>(a, T_in, s) : launch_pf<FMT_NF4, true, 0>(a, T_in, s);
        return a.x_f16 ? launch_pf<FMT_NF4, false, 1>(a, T_in, s) : launch_pf<FMT_NF4, false, 0>(a, T_in, s);
    }
    return a.x_f16 ? launch_pf<FMT_MXFP4, false, 1>(a, T_in, s) : launch_pf<FMT_MXFP4, false, 0>(a, T_in, s);
}

unsigned take_prefill_error(cudaError_t* err) {
    unsigned v = 0;
    const unsigned zero = 0;
    *err = cudaMemcpyFromSymbol(&v, g_prefill_error, sizeof(unsigned));
    if (*err == cudaSuccess && v) *err = cudaMemcpyToSymbol(g_prefill_error, &zero, sizeof(unsigned));
    return v;
}

}  // namespace gnf4
