#include <atomic>
// Routing metadata of a grouped call on the device: the router's top-k choices
// become expert_offsets, row_token, row_weight and row_dest (rows sorted by
// expert, then token, then slot), so that a whole MoE layer can run without the
// host. The grouped call takes its rows "group-sorted" with sort and scatter
// outside the kernel (solution page "How do I run a grouped GEMM directly on NF4
// packed MoE expert weights, without dequantizing to bf16 first?", "Supported
// scope"); this is that sort.
//
// One CTA of NW warps (about one per 512 pairs, at most 32). The n = T*k pairs are
// cut into NW contiguous segments, one per warp, in pair order.
//   1. Each warp counts its segment per expert: lanes with the same expert find
//      each other with __match_any_sync and the lowest of them adds the group's
//      size to the warp's row of a [NW][E] count table in shared memory.
//   2. A column scan over warps turns the table into each warp's start within
//      each expert; a scan over experts gives expert_offsets.
//   3. Each warp walks its segment again and places every pair at offset[e] +
//      its warp's start + its rank among the earlier pairs of that expert.
// The result is the stable order, the same on every call; no atomics.
#include <cstdint>
#include <cuda_runtime.h>

#include "gnf4_kernels.h"

namespace gnf4 {

namespace {

constexpr int kRouteMaxWarps = 32;
constexpr int kBatch = 8;              // rounds of 32 pairs whose loads are issued together

__device__ __forceinline__ unsigned lanemask_lt() {
    unsigned m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

__global__ void routing_kernel(const int32_t* __restrict__ ids, const float* __restrict__ weights,
                               int64_t n, int k, int E, int64_t* __restrict__ offsets,
                               int32_t* __restrict__ row_token, float* __restrict__ row_weight,
                               int32_t* __restrict__ row_dest) {
    extern __shared__ __align__(16) uint32_t s_cnt[];      // [NW][E], then off [E + 1]
    const int NW = blockDim.x >> 5;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint32_t* mine = s_cnt + (size_t)warp * E;
    uint32_t* s_off = s_cnt + (size_t)NW * E;

    const int64_t seg = (n + NW - 1) / NW;
    const int64_t i0 = min(n, (int64_t)warp * seg), i1 = min(n, i0 + seg);

    // 1. per-warp counts (the ids of kBatch rounds of 32 pairs are loaded before any is used)
    for (int e = lane; e < E; e += 32) mine[e] = 0u;
    __syncwarp();
    for (int64_t base = i0; base < i1; base += 32 * kBatch) {
        int ev[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int64_t i = base + 32 * u + lane;
            ev[u] = (i < i1) ? __ldg(ids + i) : -1;
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            if (base + 32 * u >= i1) break;           // warp-uniform: no pair left in this round
            const int e = ev[u];
            const bool valid = e >= 0 && e < E;
            const unsigned peers = __match_any_sync(0xffffffffu, valid ? e : -1 - lane);
            if (valid && (peers & lanemask_lt()) == 0u) mine[e] += (uint32_t)__popc(peers);
            __syncwarp();
        }
    }
    __syncthreads();

    // 2. column scan over warps (start of each warp within each expert), totals per expert
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        uint32_t run = 0;
        for (int w = 0; w < NW; ++w) {
            const uint32_t c = s_cnt[(size_t)w * E + e];
            s_cnt[(size_t)w * E + e] = run;
            run += c;
        }
        s_off[e + 1] = run;
    }
    __syncthreads();
    if (warp == 0) {
        uint32_t carry = 0;
        for (int b = 0; b < E; b += 32) {
            const int e = b + lane;
            uint32_t v = (e < E) ? s_off[e + 1] : 0u;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t u = __shfl_up_sync(0xffffffffu, v, o);
                if (lane >= o) v += u;
            }
            __syncwarp();
            if (e < E) s_off[e + 1] = carry + v;
            carry += __shfl_sync(0xffffffffu, v, 31);
        }
        if (lane == 0) s_off[0] = 0u;
    }
    __syncthreads();
    for (int e = threadIdx.x; e <= E; e += blockDim.x) offsets[e] = (int64_t)s_off[e];

    // 3. placement in pair order
    for (int64_t base = i0; base < i1; base += 32 * kBatch) {
        int ev[kBatch];
        float wv[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int64_t i = base + 32 * u + lane;
            ev[u] = (i < i1) ? __ldg(ids + i) : -1;
            wv[u] = (i < i1 && row_weight) ? __ldg(weights + i) : 0.0f;
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            if (base + 32 * u >= i1) break;           // warp-uniform: no pair left in this round
            const int64_t i = base + 32 * u + lane;
            const int e = ev[u];
            const bool valid = e >= 0 && e < E;
            const unsigned peers = __match_any_sync(0xffffffffu, valid ? e : -1 - lane);
            const int leader = __ffs(peers) - 1;
            uint32_t start = 0u;
            if (valid && lane == leader) {
                start = s_off[e] + mine[e];
                mine[e] += (uint32_t)__popc(peers);
            }
            start = __shfl_sync(0xffffffffu, start, leader);
            if (valid) {
                const uint32_t r = start + (uint32_t)__popc(peers & lanemask_lt());
                row_token[r] = (int32_t)(i / k);
                if (row_dest) row_dest[r] = (int32_t)i;
                if (row_weight) row_weight[r] = wv[u];
            }
            __syncwarp();
        }
    }
}

}  // namespace

int routing_warps(int E, int64_t n) {
    // about 512 pairs per warp (a small call takes one warp: every warp pays for the
    // count table and the scans); the table is NW x E words, within 200 KB of shared memory
    const int fit = (int)((200 * 1024) / (4 * (int64_t)(E > 0 ? E : 1))) - 1;
    const int64_t by_n = (n + 511) / 512;
    int nw = fit < kRouteMaxWarps ? fit : kRouteMaxWarps;
    if (by_n < nw) nw = (int)by_n;
    return nw < 1 ? 1 : nw;
}

cudaError_t launch_routing(const int32_t* ids, const float* weights, int64_t T, int64_t k, int E,
                           int64_t* offsets, int32_t* row_token, float* row_weight, int32_t* row_dest,
                           cudaStream_t s) {
    const int nw = routing_warps(E, T * k);
    const size_t smem = ((size_t)nw * E + E + 1) * sizeof(uint32_t);
    static std::atomic<bool> attr[64];               // per device: the largest table opted in
    const int dev = current_device();
    if (smem > 48 * 1024 && !attr[dev].load(std::memory_order_acquire)) {
        cudaError_t e = cudaFuncSetAttribute(routing_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)(201 * 1024 + 4 * 2049));
        if (e != cudaSuccess) return e;
        attr[dev].store(true, std::memory_order_release);
    }
    routing_kernel<<<1, nw * 32, smem, s>>>(ids, weights, T * k, (int)k, E, offsets, row_token, row_weight,
                                            row_dest);
    return cudaGetLastError();
}

}  // namespace gnf4
