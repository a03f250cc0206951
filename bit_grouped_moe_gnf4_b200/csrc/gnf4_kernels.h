// Internal launcher declarations (host side); the public C ABI is include/gnf4.h.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "gnf4_common.cuh"

namespace gnf4 {

cudaError_t launch_quantize_nf4(const float* w, int64_t rows, int64_t K, uint8_t* packed,
                                float* absmax, cudaStream_t s);
cudaError_t launch_quantize_mxfp4(const float* w, int64_t rows, int64_t K, uint8_t* blocks,
                                  uint8_t* scales, cudaStream_t s);

// Decode band: TMA-fed warp MMAs over table-decoded nibbles. Takes the groups whose
// row count m satisfies a.m_lo <= m <= a.m_hi. fuse_swiglu: a.N is the fused gate_up
// width 2I and the output [.., I] holds silu(gate) * up.
cudaError_t launch_decode_band(int fmt, const GroupedArgs& a, cudaStream_t s, bool fuse_swiglu = false);

// Prefill band: tcgen05 MMAs into tensor memory with the per-block fp32
// rescale outside the MMA. Takes the groups with a.m_lo <= m <= a.m_hi.
cudaError_t launch_prefill_band(int fmt, const GroupedArgs& a, int64_t T_in, cudaStream_t s);

// Device-side validation of the routing metadata; writes a status word.
cudaError_t launch_check_routing(const GroupedArgs& a, int64_t T_in, int64_t T_out,
                                 unsigned* status_out, cudaStream_t s);

// SwiGLU over [R, 2I] gate_up rows and the fp32 slot-order top-k combine
// (argument checks are the caller's; sizes already validated).
cudaError_t launch_swiglu(const void* h, int64_t R, int64_t I, void* out, cudaStream_t s);
cudaError_t launch_combine_topk(const void* y, int64_t R, int64_t N, const int32_t* row_of_slot,
                                const float* slot_weight, int64_t T, int64_t k, void* out,
                                cudaStream_t s);

// Input gradient of the grouped GEMM (one launch): out[r, k] = w(r) * sum_n
// g[src(r), n] * What[e(r), n, k]; sizes already validated (N % 16, K % 64, E <= 2048).
struct DgradArgs {
    const uint16_t* g;          // bf16 [T_in, N]
    const uint8_t* W;           // [E, N, K/2]
    const void* scales;         // NF4: f32 [E, N, K/64]; MXFP4: u8 [E, N, K/32]
    const int64_t* offsets;     // [E+1]
    const int32_t* row_src;     // [R] or null
    const float* row_weight;    // [R] or null
    uint16_t* out;              // bf16 [R, K]
    int64_t R;
    int E, N, K;
    LutPlanes lut;
};
cudaError_t launch_dgrad(int fmt, const DgradArgs& a, cudaStream_t s);
// the launch shape the host picks (exported for the tests of the host logic)
int dgrad_row_tiles(int64_t R, int E);
int dgrad_splits(int64_t R, int E, int N, int K, int rt);

// Routing metadata from the router's top-k choices (one CTA; sizes validated).
cudaError_t launch_routing(const int32_t* ids, const float* weights, int64_t T, int64_t k, int E,
                           int64_t* offsets, int32_t* row_token, float* row_weight, int32_t* row_dest,
                           cudaStream_t s);

int device_sm_count();

// The current CUDA device, clamped to [0, 64) for the per-device caches (kernel
// attribute opt-ins are per device, so every cache of them is keyed by this).
int current_device();

// Read and clear the error word a band's kernels set when they give up waiting
// on a barrier (synchronous; 0 = no event). Returns a CUDA error through *err.
unsigned take_decode_error(cudaError_t* err);
unsigned take_prefill_error(cudaError_t* err);

}  // namespace gnf4
