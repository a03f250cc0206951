#include <atomic>
// Input gradient of the grouped 4-bit GEMM: for every routed row r of expert e,
//   dx[r, k] = w(r) * sum_n g[src(r), n] * What[e, n, k]
// in one launch over all experts, decoding the packed weights on chip (the
// grouped-nf4-gemm README, "Training: the backward is a kernel too (0.7.0)").
//
// Work item: (expert e, a tile of up to 16*RT routed rows of e, a 64-column tile
// of K). S warps of one CTA share an item, each taking a contiguous 1/S of the
// contraction over N; the partial sums meet in shared memory and are added in
// split order, so every result has one fixed summation order. A CTA of 8 warps
// holds 8/S items at a time and strides over all items (persistent grid); the
// item list is derived on the device from expert_offsets.
//
// Mapping onto mma.m16n8k16 (A = gradient rows, B = decoded weights, the MMA's
// k = the contraction index n): lane (g, t) decodes word g (columns 8g..8g+7 of
// the 64-column tile) of weight rows n0+2t, n0+2t+1, n0+2t+8, n0+2t+9. One byte
// permute pairs the same column of two rows, which is the B fragment; MMA tile c
// (c = 0..7) therefore covers the strided output columns {8j + c}, and the
// accumulators of lane (g, t) end up as the 16 contiguous columns 16t..16t+15 of
// rows g and g+8.
//
// Block scale: the contraction crosses rows with different scales, so the scale
// is applied before the MMA (bf16x2 multiply, round to nearest), to the decoded
// weight pair; for MXFP4 the e8m0 scale is a power of two and the product is exact,
// for NF4 the fp32 absmax is rounded to bf16 and the product once more. NF4 items of
// two row tiles instead scale the gradient: an item's 64 output columns are one NF4
// scale block, so the absmax of contraction row n multiplies the gradient's column n.
#include <climits>
#include <cstdint>
#include <cuda_runtime.h>

#include "gnf4_common.cuh"
#include "gnf4_kernels.h"

namespace gnf4 {

namespace {

constexpr int kDgWarps = 8;
constexpr int kDgThreads = kDgWarps * 32;
// ring stages (16 contraction rows each) per warp: fewer with two row tiles, whose
// accumulators take the registers
template <int RT>
constexpr int ring_depth() { return RT == 1 ? 6 : 4; }
constexpr int kDgMaxExperts = 2048;

__device__ __forceinline__ uint32_t mul_bf16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t d;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
    return d;
}

// the block scale of one weight row as a bf16 pair
template <int FMT>
__device__ __forceinline__ uint32_t scale_pair(uint32_t raw) {
    if constexpr (FMT == FMT_NF4) {
        const float s = __uint_as_float(raw);
        return pack_bf16x2(s, s);
    } else {
        // 2^(s-127) in bf16: the exponent field for s = 1..254, the subnormal 2^-127 for 0, NaN for 255
        const uint32_t b = raw == 0u ? 0x0040u : raw == 255u ? 0x7FC0u : (raw << 7);
        return b | (b << 16);
    }
}

__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// words of one stage (16 contraction rows) per lane: 4 weight words, 4 A words per row tile
template <int RT>
constexpr int stage_words() { return 4 + 4 * RT; }

template <int RT>
constexpr size_t ring_bytes() { return (size_t)kDgWarps * ring_depth<RT>() * stage_words<RT>() * 32 * 4; }

template <int RT, int S>
constexpr size_t work_bytes() {
    // the ring, and after the main loop the partial sums of the splits (same space)
    return ring_bytes<RT>() > (S > 1 ? (size_t)kDgWarps * 32 * RT * 32 * 4 : 0)
               ? ring_bytes<RT>() : (size_t)kDgWarps * 32 * RT * 32 * 4;
}

__host__ __device__ constexpr size_t prefix_bytes(int E) { return (((size_t)(E + 1) * 12) + 15) & ~(size_t)15; }

// Issue the copies of one stage (16 contraction rows from n0) into ring slot `slot`:
// each lane copies its own four weight words and its A words; rows past the group
// are zero-filled. Returns this lane's raw scale (row lane & 15; MXFP4: block lane >> 4).
template <int FMT, int RT>
__device__ __forceinline__ uint32_t issue_stage(uint32_t ring, int slot, int n0, const uint8_t* wbase,
                                                int64_t half_k, const uint16_t* const (&grow)[RT][2],
                                                const uint16_t* gbase, const void* scales, int64_t sbase,
                                                int64_t sstride, int lane, int t) {
    const uint32_t stage = ring + (uint32_t)(slot * stage_words<RT>() * 32 * 4) + (uint32_t)lane * 4u;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int n = n0 + 2 * t + (j & 1) + 8 * (j >> 1);
        cp_async4(stage + (uint32_t)(j * 128), wbase + (int64_t)n * half_k, 4u);
    }
#pragma unroll
    for (int r = 0; r < RT; ++r)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            // a0 = row g, cols n0+2t..; a1 = row g+8; a2 = row g, cols n0+2t+8..; a3 = row g+8
            const uint16_t* row = grow[r][j & 1];
            const int col = n0 + 2 * t + 8 * (j >> 1);
            cp_async4(stage + (uint32_t)((4 + 4 * r + j) * 128), row ? row + col : gbase, row ? 4u : 0u);
        }
    const int64_t srow = n0 + (lane & 15);
    if constexpr (FMT == FMT_NF4)
        return __float_as_uint(__ldg(reinterpret_cast<const float*>(scales) + sbase + srow * sstride));
    else
        return __ldg(reinterpret_cast<const uint8_t*>(scales) + sbase + (lane >> 4) + srow * sstride);
}

template <int FMT, int RT>
__device__ __forceinline__ void compute_stage(uint32_t ring, int slot, uint32_t sraw, const LutPlanes& lut,
                                              float (&acc)[RT][8][4], int lane, int g, int t) {
    const uint32_t base = ring + (uint32_t)(slot * stage_words<RT>() * 32 * 4) + (uint32_t)lane * 4u;
    uint32_t w[4], a[RT][4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
        asm volatile("ld.shared.u32 %0, [%1];" : "=r"(w[j]) : "r"(base + (uint32_t)(j * 128)));
#pragma unroll
    for (int r = 0; r < RT; ++r)
#pragma unroll
        for (int j = 0; j < 4; ++j)
            asm volatile("ld.shared.u32 %0, [%1];" : "=r"(a[r][j]) : "r"(base + (uint32_t)((4 + 4 * r + j) * 128)));
    uint32_t dec[4][4];
    if constexpr (FMT == FMT_NF4 && RT == 2) {
        // the 64 output columns of an item lie in one NF4 scale block, so the scale of
        // contraction row n can multiply the gradient's column n (the A fragments: 8 bf16
        // pair multiplies for the two row tiles) instead of every decoded weight pair (16).
        // With one row tile the saving is smaller than the latency it puts in front of the
        // first MMA (measured), so that case scales the weights.
        const float s0 = __uint_as_float(__shfl_sync(0xffffffffu, sraw, 2 * t));
        const float s1 = __uint_as_float(__shfl_sync(0xffffffffu, sraw, 2 * t + 1));
        const float s8 = __uint_as_float(__shfl_sync(0xffffffffu, sraw, 2 * t + 8));
        const float s9 = __uint_as_float(__shfl_sync(0xffffffffu, sraw, 2 * t + 9));
        const uint32_t sp_lo = pack_bf16x2(s0, s1), sp_hi = pack_bf16x2(s8, s9);
#pragma unroll
        for (int r = 0; r < RT; ++r) {
            a[r][0] = mul_bf16x2(a[r][0], sp_lo);
            a[r][1] = mul_bf16x2(a[r][1], sp_lo);
            a[r][2] = mul_bf16x2(a[r][2], sp_hi);
            a[r][3] = mul_bf16x2(a[r][3], sp_hi);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) decode_word<FMT>(w[j], lut, dec[j]);
    } else {
        // each decoded weight pair is scaled (MXFP4: an item's 64 columns span two scale
        // blocks; its e8m0 scale is a power of two, so the product is exact)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int row = 2 * t + (j & 1) + 8 * (j >> 1);
            const int src_lane = (FMT == FMT_NF4) ? row : row + 16 * (g >> 2);
            const uint32_t sp = scale_pair<FMT>(__shfl_sync(0xffffffffu, sraw, src_lane));
            decode_word<FMT>(w[j], lut, dec[j]);
#pragma unroll
            for (int i = 0; i < 4; ++i) dec[j][i] = mul_bf16x2(dec[j][i], sp);
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t b0e = prmt(dec[0][i], dec[1][i], 0x5410u);
        const uint32_t b1e = prmt(dec[2][i], dec[3][i], 0x5410u);
        const uint32_t b0o = prmt(dec[0][i], dec[1][i], 0x7632u);
        const uint32_t b1o = prmt(dec[2][i], dec[3][i], 0x7632u);
#pragma unroll
        for (int r = 0; r < RT; ++r) {
            mma_bf16_16816(acc[r][2 * i], a[r][0], a[r][1], a[r][2], a[r][3], b0e, b1e);
            mma_bf16_16816(acc[r][2 * i + 1], a[r][0], a[r][1], a[r][2], a[r][3], b0o, b1o);
        }
    }
}

template <int FMT, int RT, int S>
__global__ void __launch_bounds__(kDgThreads, 2) dgrad_kernel(const DgradArgs p) {
    extern __shared__ __align__(16) uint8_t smem[];
    int64_t* s_off = reinterpret_cast<int64_t*>(smem);                    // [E + 1]
    int* s_tiles = reinterpret_cast<int*>(s_off + (p.E + 1));             // [E + 1] row-tile prefix
    uint8_t* work = smem + prefix_bytes(p.E);                             // ring, then partial sums
    float* s_red = reinterpret_cast<float*>(work);                        // [kDgWarps][32*RT][32]

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;
    constexpr int kRows = 16 * RT;
    constexpr int kDgDepth = ring_depth<RT>();
    const uint32_t ring = (uint32_t)__cvta_generic_to_shared(work) +
                          (uint32_t)(warp * kDgDepth * stage_words<RT>() * 32 * 4);

    // row tiles of each expert, prefix over experts
    for (int e = tid; e <= p.E; e += kDgThreads) s_off[e] = p.offsets[e];
    __syncthreads();
    if (warp == 0) {
        int carry = 0;
        if (lane == 0) s_tiles[0] = 0;
        for (int base = 0; base < p.E; base += 32) {
            const int e = base + lane;
            int v = 0;
            if (e < p.E) {
                const int64_t m = s_off[e + 1] - s_off[e];
                v = m > 0 ? (int)((m + kRows - 1) / kRows) : 0;
            }
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int u = __shfl_up_sync(0xffffffffu, v, o);
                if (lane >= o) v += u;
            }
            if (e < p.E) s_tiles[e + 1] = carry + v;
            carry += __shfl_sync(0xffffffffu, v, 31);
        }
    }
    __syncthreads();

    const int KT = p.K / 64;
    const int64_t items = (int64_t)s_tiles[p.E] * KT;
    constexpr int kItemsPerCta = kDgWarps / S;
    const int64_t groups = (items + kItemsPerCta - 1) / kItemsPerCta;
    const int nsteps = p.N / 16;
    const int per_split = (nsteps + S - 1) / S;
    const int split = warp % S;
    const int st0 = split * per_split;
    const int st1 = min(nsteps, st0 + per_split);
    const int64_t half_k = p.K / 2;

    for (int64_t grp = blockIdx.x; grp < groups; grp += gridDim.x) {
        const int64_t item = grp * kItemsPerCta + warp / S;
        const bool have = item < items;
        float acc[RT][8][4];
#pragma unroll
        for (int r = 0; r < RT; ++r)
#pragma unroll
            for (int c = 0; c < 8; ++c)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[r][c][j] = 0.0f;

        int e = 0, kt = 0;
        int64_t row0 = 0;
        int rows = 0;
        if (have) {
            const int tile = (int)(item / KT);
            kt = (int)(item - (int64_t)tile * KT);
            int lo = 0, hi = p.E - 1;               // last expert whose tile prefix <= tile
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (s_tiles[mid] <= tile) lo = mid; else hi = mid - 1;
            }
            e = lo;
            row0 = s_off[e] + (int64_t)(tile - s_tiles[e]) * kRows;
            rows = (int)min((int64_t)kRows, s_off[e + 1] - row0);
        }

        if (have && st0 < st1) {
            // this lane's gradient rows (g and g+8 of each 16-row tile), or null past the group
            const uint16_t* grow[RT][2];
#pragma unroll
            for (int r = 0; r < RT; ++r)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int local = 16 * r + 8 * h + g;
                    grow[r][h] = nullptr;
                    if (local < rows) {
                        const int64_t rr = row0 + local;
                        const int64_t src = p.row_src ? (int64_t)__ldg(p.row_src + rr) : rr;
                        grow[r][h] = p.g + src * p.N;
                    }
                }
            const uint8_t* wbase = p.W + (int64_t)e * p.N * half_k + (int64_t)kt * 32 + 4 * g;
            const int64_t sstride = (FMT == FMT_NF4) ? p.K / 64 : p.K / 32;
            const int64_t sbase = (int64_t)e * p.N * sstride + (FMT == FMT_NF4 ? kt : 2 * kt);

            // ring of kDgDepth stages: stage q of the split lives in slot q % kDgDepth; one
            // commit group per issued stage (empty past the end) keeps the wait count fixed
            uint32_t sreg[kDgDepth];
#pragma unroll
            for (int d = 0; d < kDgDepth - 1; ++d) {
                sreg[d] = 0u;
                if (st0 + d < st1)
                    sreg[d] = issue_stage<FMT, RT>(ring, d, 16 * (st0 + d), wbase, half_k, grow, p.g, p.scales,
                                                   sbase, sstride, lane, t);
                cp_async_commit();
            }
            sreg[kDgDepth - 1] = 0u;
            for (int base = st0; base < st1; base += kDgDepth) {
#pragma unroll
                for (int d = 0; d < kDgDepth; ++d) {
                    const int step = base + d;
                    if (step < st1) {                 // uniform across the warp
                        const int ahead = step + kDgDepth - 1;
                        constexpr int kAheadSlotOff = kDgDepth - 1;
                        const int aslot = (d + kAheadSlotOff) % kDgDepth;
                        if (ahead < st1)
                            sreg[(d + kAheadSlotOff) % kDgDepth] =
                                issue_stage<FMT, RT>(ring, aslot, 16 * ahead, wbase, half_k, grow, p.g,
                                                     p.scales, sbase, sstride, lane, t);
                        cp_async_commit();
                        cp_async_wait<kDgDepth - 1>();
                        compute_stage<FMT, RT>(ring, d, sreg[d], p.lut, acc, lane, g, t);
                    }
                }
            }
            cp_async_wait<0>();
        }

        // splits 1..S-1 hand their partial sums to split 0 through shared memory (the
        // ring's space: every warp has drained its copies before the first barrier)
        if constexpr (S > 1) {
            __syncthreads();
            float* mine = s_red + (size_t)warp * (32 * RT) * 32 + lane;
            if (split > 0) {
#pragma unroll
                for (int r = 0; r < RT; ++r)
#pragma unroll
                    for (int c = 0; c < 8; ++c)
#pragma unroll
                        for (int j = 0; j < 4; ++j) mine[((r * 8 + c) * 4 + j) * 32] = acc[r][c][j];
            }
            __syncthreads();
            if (split == 0) {
                for (int q = 1; q < S; ++q) {
                    const float* other = s_red + (size_t)(warp + q) * (32 * RT) * 32 + lane;
#pragma unroll
                    for (int r = 0; r < RT; ++r)
#pragma unroll
                        for (int c = 0; c < 8; ++c)
#pragma unroll
                            for (int j = 0; j < 4; ++j) acc[r][c][j] += other[((r * 8 + c) * 4 + j) * 32];
                }
            }
            __syncthreads();
        }

        if (have && split == 0) {
#pragma unroll
            for (int r = 0; r < RT; ++r)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int local = 16 * r + 8 * h + g;
                    if (local >= rows) continue;
                    const int64_t rr = row0 + local;
                    const float wgt = p.row_weight ? __ldg(p.row_weight + rr) : 1.0f;
                    uint32_t o[8];
#pragma unroll
                    for (int c = 0; c < 8; c += 2) {
                        o[c / 2] = pack_bf16x2(wgt * acc[r][c][2 * h], wgt * acc[r][c + 1][2 * h]);
                        o[4 + c / 2] = pack_bf16x2(wgt * acc[r][c][2 * h + 1], wgt * acc[r][c + 1][2 * h + 1]);
                    }
                    uint4* dst = reinterpret_cast<uint4*>(p.out + rr * p.K + (int64_t)kt * 64 + 16 * t);
                    dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
                    dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
                }
        }
    }
}

template <int FMT, int RT, int S>
cudaError_t launch_dg(const DgradArgs& a, cudaStream_t s) {
    const size_t smem = prefix_bytes(a.E) + work_bytes<RT, S>();
    static std::atomic<bool> attr_set[64];           // per device: dynamic shared memory opted in
    const int dev = current_device();
    if (!attr_set[dev].load(std::memory_order_acquire)) {
        cudaError_t e = cudaFuncSetAttribute(dgrad_kernel<FMT, RT, S>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)(prefix_bytes(kDgMaxExperts) + work_bytes<RT, S>()));
        if (e != cudaSuccess) return e;
        attr_set[dev].store(true, std::memory_order_release);
    }
    const int grid = device_sm_count() * 2;
    dgrad_kernel<FMT, RT, S><<<grid, kDgThreads, smem, s>>>(a);
    return cudaGetLastError();
}

template <int FMT, int RT>
cudaError_t launch_dg_s(const DgradArgs& a, int S, cudaStream_t s) {
    switch (S) {
        case 1: return launch_dg<FMT, RT, 1>(a, s);
        case 2: return launch_dg<FMT, RT, 2>(a, s);
        case 4: return launch_dg<FMT, RT, 4>(a, s);
        default: return launch_dg<FMT, RT, 8>(a, s);
    }
}

}  // namespace

int dgrad_splits(int64_t R, int E, int N, int K, int rt) {
    // enough warps to fill every SM about twice over, each split at least 4 steps of 16 rows
    const int64_t rows_per_tile = 16 * rt;
    const int64_t tiles = (R + rows_per_tile - 1) / rows_per_tile + (R < E ? R : E);
    const int64_t items = tiles * (K / 64);
    const int64_t want = (int64_t)device_sm_count() * 2 * kDgWarps;
    int S = 1;
    while (S < 8 && items * S < want && N / 16 / (2 * S) >= 4) S *= 2;
    return S;
}

int dgrad_row_tiles(int64_t R, int E) {
    // two 16-row tiles per item once the average group is large enough to fill them
    const int64_t active = R < E ? R : E;
    return (active > 0 && R / active >= 24) ? 2 : 1;
}

cudaError_t launch_dgrad(int fmt, const DgradArgs& a, cudaStream_t s) {
    if (a.R == 0) return cudaSuccess;
    const int rt = dgrad_row_tiles(a.R, a.E);
    const int S = dgrad_splits(a.R, a.E, a.N, a.K, rt);
    if (fmt == FMT_NF4)
        return rt == 2 ? launch_dg_s<FMT_NF4, 2>(a, S, s) : launch_dg_s<FMT_NF4, 1>(a, S, s);
    return rt == 2 ? launch_dg_s<FMT_MXFP4, 2>(a, S, s) : launch_dg_s<FMT_MXFP4, 1>(a, S, s);
}

}  // namespace gnf4
