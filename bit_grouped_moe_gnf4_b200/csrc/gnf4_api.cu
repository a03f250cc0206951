// The C ABI of include/gnf4.h: argument validation, band selection, launches.
#include <atomic>
#include <climits>
#include <cstdint>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <cuda_runtime.h>

#include "../../include/gnf4.h"
#include "gnf4_common.cuh"
#include "gnf4_kernels.h"

namespace gnf4 {

// Groups with more than this many routed rows go to the prefill (tensor-core)
// band; the rest to the decode band.
#ifndef GNF4_DECODE_MAX_ROWS
#define GNF4_DECODE_MAX_ROWS 64
#endif
constexpr int kDecodeMaxRows = GNF4_DECODE_MAX_ROWS;
// at most this many routed rows in the whole call: every group runs in the decode band
// (at most one group can exceed kDecodeMaxRows, and a second launch costs more than
// the decode band's extra passes over that group)
constexpr int64_t kDecodeOnlyRows = 2 * kDecodeMaxRows;

static thread_local char g_err[512] = "";

static gnf4_status fail(gnf4_status st, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
    return st;
}

static gnf4_status cuda_fail(cudaError_t e, const char* what) {
    return fail(GNF4_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// device (or managed) memory of the current device; managed memory is accepted on
// any device, since the GPU reaches it through page migration
static bool is_device_ptr(const void* p) {
    cudaPointerAttributes attr;
    if (cudaPointerGetAttributes(&attr, p) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    if (attr.type == cudaMemoryTypeManaged) return true;
    if (attr.type != cudaMemoryTypeDevice) return false;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return attr.device == dev;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        dev = 0;
    }
    return (dev < 0 || dev >= 64) ? 0 : dev;
}

int device_sm_count() {
    static std::atomic<int> cached[64];
    const int dev = current_device();
    int n = cached[dev].load(std::memory_order_relaxed);
    if (n == 0) {
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (n <= 0) n = 1;
        cached[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

static uint16_t host_bf16_rne(float f) {
    uint32_t u;
    std::memcpy(&u, &f, 4);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

// fp32 -> IEEE binary16 bits, round to nearest even; the codebook values are all
// zero or normal binary16 numbers, which is all this handles
static uint16_t host_f16_rne(float f) {
    uint32_t u;
    std::memcpy(&u, &f, 4);
    const uint32_t sign = (u >> 16) & 0x8000u;
    if ((u & 0x7FFFFFFFu) == 0) return (uint16_t)sign;
    int exp = (int)((u >> 23) & 0xFFu) - 127 + 15;
    uint32_t m = (u & 0x7FFFFFu) >> 13;
    const uint32_t rem = u & 0x1FFFu;
    if (rem > 0x1000u || (rem == 0x1000u && (m & 1u))) ++m;
    if (m == 0x400u) {
        m = 0;
        ++exp;
    }
    return (uint16_t)(sign | ((uint32_t)exp << 10) | m);
}

LutPlanes make_lut(int fmt, int f16) {
    // NF4 values (QLoRA / bitsandbytes NF4) and the OCP e2m1 magnitudes
    static const float nf4[16] = {
        -1.0f, -0.6961928009986877f, -0.5250730514526367f, -0.39491748809814453f,
        -0.28444138169288635f, -0.18477343022823334f, -0.09105003625154495f, 0.0f,
        0.07958029955625534f, 0.16093020141124725f, 0.24611230194568634f,
        0.33791524171829224f, 0.44070982933044434f, 0.5626170039176941f,
        0.7229568362236023f, 1.0f};
    static const float e2m1[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};
    LutPlanes L;
    std::memset(&L, 0, sizeof(L));
    const int n = (fmt == FMT_NF4) ? 16 : 8;
    for (int i = 0; i < n; ++i) {
        const float v = fmt == FMT_NF4 ? nf4[i] : e2m1[i];
        const uint16_t b = f16 ? host_f16_rne(v) : host_bf16_rne(v);
        L.lo[i >> 2] |= (uint32_t)(b & 0xFFu) << (8 * (i & 3));
        L.hi[i >> 2] |= (uint32_t)(b >> 8) << (8 * (i & 3));
    }
    return L;
}

static gnf4_status check_quantize_args(const float* w, int64_t rows, int64_t K, const void* o1,
                                       const void* o2, int64_t kmul) {
    if (!w || !o1 || !o2) return fail(GNF4_ERR_INVALID_ARG, "null pointer argument");
    if (rows < 0 || K <= 0) return fail(GNF4_ERR_INVALID_ARG, "rows must be >= 0 and K > 0");
    if (K % kmul) return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "K must be a multiple of %lld", (long long)kmul);
    if (!aligned16(w)) return fail(GNF4_ERR_MISALIGNED, "w must be 16-byte aligned");
    if (!is_device_ptr(w) || !is_device_ptr(o1) || !is_device_ptr(o2))
        return fail(GNF4_ERR_INVALID_ARG, "w and the outputs must be device memory");
    return GNF4_OK;
}

// Status words of the routing check: each checked call takes the next of these slots
// (round robin), so calls checked at the same time on different streams (up to the
// slot count) never share a word.
constexpr int kCheckSlots = 256;
__device__ unsigned g_check_status[kCheckSlots];
static std::atomic<unsigned> g_check_next{0};

__global__ void check_routing_kernel(const GroupedArgs p, int64_t T_in, int64_t T_out, int slot) {
    unsigned bad = 0;
    const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t e = tid; e < p.E; e += stride)
        if (p.offsets[e + 1] < p.offsets[e]) bad |= 1u;
    if (tid == 0 && (p.offsets[0] != 0 || p.offsets[p.E] != p.R)) bad |= 2u;
    for (int64_t r = tid; r < p.R; r += stride) {
        if (p.row_token) {
            const int32_t v = p.row_token[r];
            if (v < 0 || v >= T_in) bad |= 4u;
        }
        if (p.row_dest) {
            const int32_t v = p.row_dest[r];
            if (v < 0 || v >= T_out) bad |= 8u;
        }
        if (p.row_weight && !isfinite(p.row_weight[r])) bad |= 16u;
    }
    if (bad) atomicOr(&g_check_status[slot], bad);
}

cudaError_t launch_check_routing(const GroupedArgs& a, int64_t T_in, int64_t T_out,
                                 unsigned* status_out, cudaStream_t s) {
    const int slot = (int)(g_check_next.fetch_add(1u, std::memory_order_relaxed) % kCheckSlots);
    const size_t off = sizeof(unsigned) * (size_t)slot;
    const unsigned zero = 0;
    cudaError_t e = cudaMemcpyToSymbolAsync(g_check_status, &zero, sizeof(zero), off,
                                            cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) return e;
    check_routing_kernel<<<64, 256, 0, s>>>(a, T_in, T_out, slot);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    e = cudaMemcpyFromSymbolAsync(status_out, g_check_status, sizeof(unsigned), off,
                                  cudaMemcpyDeviceToHost, s);
    if (e != cudaSuccess) return e;
    return cudaStreamSynchronize(s);
}

// The lossless fp32 -> bf16 absmax cast: the high half of each value; any value whose
// low half is not zero (bf16 cannot hold it) marks the call's status slot.
__global__ void absmax_to_bf16_kernel(const uint32_t* a, int64_t n, uint16_t* out, int slot) {
    unsigned bad = 0;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const uint32_t v = a[i];
        bad |= (v & 0xFFFFu) ? 1u : 0u;
        out[i] = (uint16_t)(v >> 16);
    }
    if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0) atomicOr(&g_check_status[slot], 1u);
}

cudaError_t launch_absmax_to_bf16(const float* a, int64_t n, uint16_t* out, unsigned* inexact, cudaStream_t s) {
    const int slot = (int)(g_check_next.fetch_add(1u, std::memory_order_relaxed) % kCheckSlots);
    const size_t off = sizeof(unsigned) * (size_t)slot;
    const unsigned zero = 0;
    cudaError_t e = cudaMemcpyToSymbolAsync(g_check_status, &zero, sizeof(zero), off, cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) return e;
    int64_t blocks = (n + 255) / 256;
    if (blocks > 4 * (int64_t)device_sm_count()) blocks = 4 * (int64_t)device_sm_count();
    absmax_to_bf16_kernel<<<(unsigned)blocks, 256, 0, s>>>(reinterpret_cast<const uint32_t*>(a), n, out, slot);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    e = cudaMemcpyFromSymbolAsync(inexact, g_check_status, sizeof(unsigned), off, cudaMemcpyDeviceToHost, s);
    if (e != cudaSuccess) return e;
    return cudaStreamSynchronize(s);
}

static gnf4_status grouped(int fmt, const void* x, int x_dtype, const uint8_t* W, const void* scales,
                           int scale_dtype, const int64_t* offsets, const int32_t* row_token,
                           const float* row_weight, const int32_t* row_dest, int64_t E,
                           int64_t N, int64_t K, int64_t R, int64_t T_in, int64_t T_out,
                           void* out, int flags, void* stream, bool fuse_swiglu = false) {
    const int64_t kmul = (fmt == FMT_NF4) ? 64 : 32;
    if (x_dtype != GNF4_DTYPE_BF16 && x_dtype != GNF4_DTYPE_F16)
        return fail(GNF4_ERR_INVALID_ARG, "x_dtype must be GNF4_DTYPE_BF16 or GNF4_DTYPE_F16");
    if (fmt == FMT_NF4 && scale_dtype != GNF4_DTYPE_F32 && scale_dtype != GNF4_DTYPE_BF16)
        return fail(GNF4_ERR_INVALID_ARG, "NF4 absmax_dtype must be GNF4_DTYPE_F32 or GNF4_DTYPE_BF16");
    if (!x || !W || !scales || !offsets || !out) return fail(GNF4_ERR_INVALID_ARG, "null pointer argument");
    if (E < 1 || N < 1 || K < 1 || R < 0 || T_in < 0 || T_out < 0)
        return fail(GNF4_ERR_INVALID_ARG, "sizes must be E,N,K >= 1 and R,T_in,T_out >= 0");
    if (flags & ~(GNF4_CHECK | GNF4_FORCE_DECODE | GNF4_FORCE_PREFILL | GNF4_TEST_STALL))
        return fail(GNF4_ERR_INVALID_ARG, "unknown flag bits 0x%x", flags);
    if ((flags & GNF4_TEST_STALL) && (flags & GNF4_FORCE_PREFILL))
        return fail(GNF4_ERR_INVALID_ARG, "GNF4_TEST_STALL runs the decode band only");
    if ((flags & GNF4_FORCE_DECODE) && (flags & GNF4_FORCE_PREFILL))
        return fail(GNF4_ERR_INVALID_ARG, "GNF4_FORCE_DECODE and GNF4_FORCE_PREFILL exclude each other");
    if (K % kmul) return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "K must be a multiple of %lld", (long long)kmul);
    if (N % 16) return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "N must be a multiple of 16");
    if (fuse_swiglu && N % 32) return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "the fused gate_up width N = 2I must be a multiple of 32");
    if (fuse_swiglu && (flags & GNF4_FORCE_PREFILL))
        return fail(GNF4_ERR_INVALID_ARG, "the fused SwiGLU runs in the decode band only");
    if (E > 2048) return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "at most 2048 experts");
    if (K > (int64_t)INT_MAX / 2 || E * N > (int64_t)INT_MAX || T_in > INT_MAX || T_out > INT_MAX)
        return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "K, E*N, T_in and T_out must fit in int32");
    if (!row_token && T_in < R) return fail(GNF4_ERR_INVALID_ARG, "row_token is NULL but T_in < R");
    if (!row_dest && T_out < R) return fail(GNF4_ERR_INVALID_ARG, "row_dest is NULL but T_out < R");
    if (R > 0 && (T_in == 0 || T_out == 0)) return fail(GNF4_ERR_INVALID_ARG, "R > 0 needs T_in, T_out >= 1");
    if (!aligned16(x) || !aligned16(W) || !aligned16(out))
        return fail(GNF4_ERR_MISALIGNED, "x, W and out must be 16-byte aligned");
    if (fmt == FMT_NF4 && scale_dtype == GNF4_DTYPE_F32 && (reinterpret_cast<uintptr_t>(scales) & 3u))
        return fail(GNF4_ERR_MISALIGNED, "absmax must be 4-byte aligned (fp32)");
    if (fmt == FMT_NF4 && scale_dtype == GNF4_DTYPE_BF16 && (reinterpret_cast<uintptr_t>(scales) & 1u))
        return fail(GNF4_ERR_MISALIGNED, "absmax must be 2-byte aligned (bf16)");
    if ((reinterpret_cast<uintptr_t>(offsets) & 7u) || (row_token && (reinterpret_cast<uintptr_t>(row_token) & 3u)) ||
        (row_weight && (reinterpret_cast<uintptr_t>(row_weight) & 3u)) ||
        (row_dest && (reinterpret_cast<uintptr_t>(row_dest) & 3u)))
        return fail(GNF4_ERR_MISALIGNED, "expert_offsets must be 8-byte and row arrays 4-byte aligned");
    if (!is_device_ptr(x) || !is_device_ptr(W) || !is_device_ptr(scales) || !is_device_ptr(offsets) ||
        !is_device_ptr(out) || (row_token && !is_device_ptr(row_token)) ||
        (row_weight && !is_device_ptr(row_weight)) || (row_dest && !is_device_ptr(row_dest)))
        return fail(GNF4_ERR_INVALID_ARG, "every buffer must be device memory of the current device");
    if (R == 0) return GNF4_OK;

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    GroupedArgs a;
    a.x = reinterpret_cast<const uint16_t*>(x);
    a.W = W;
    a.scales = scales;
    a.offsets = offsets;
    a.row_token = row_token;
    a.row_weight = row_weight;
    a.row_dest = row_dest;
    a.out = reinterpret_cast<uint16_t*>(out);
    a.R = R;
    a.E = (int)E;
    a.N = (int)N;
    a.K = (int)K;
    static const LutPlanes lut_nf4 = make_lut(FMT_NF4, 0), lut_nf4_h = make_lut(FMT_NF4, 1);
    static const LutPlanes lut_mx = make_lut(FMT_MXFP4, 0), lut_mx_h = make_lut(FMT_MXFP4, 1);
    a.x_f16 = (x_dtype == GNF4_DTYPE_F16) ? 1 : 0;
    a.test_stall = (flags & GNF4_TEST_STALL) ? 1 : 0;
    a.scale_bf16 = (fmt == FMT_NF4 && scale_dtype == GNF4_DTYPE_BF16) ? 1 : 0;
    a.lut = (fmt == FMT_NF4) ? (a.x_f16 ? lut_nf4_h : lut_nf4) : (a.x_f16 ? lut_mx_h : lut_mx);

    if (flags & GNF4_CHECK) {
        unsigned st = 0;
        cudaError_t e = launch_check_routing(a, T_in, T_out, &st, s);
        if (e != cudaSuccess) return cuda_fail(e, "routing check");
        if (st) return fail(GNF4_ERR_DEVICE_STATUS,
                            "bad routing metadata (status 0x%x: 1 offsets decrease, 2 offsets[0] != 0 "
                            "or offsets[E] != R, 4 row_token out of range, 8 row_dest out of range, "
                            "16 non-finite row_weight)", st);
    }

    if (fuse_swiglu) {
        a.m_lo = 1;
        a.m_hi = INT_MAX;
        cudaError_t e = launch_decode_band(fmt, a, s, true);
        return e == cudaSuccess ? GNF4_OK : cuda_fail(e, "fused gate_up + SwiGLU launch");
    }
    // band split by rows per group; decided on the device from the offsets
    int split = kDecodeMaxRows;
    if (R <= kDecodeOnlyRows) split = INT_MAX;
    if (flags & (GNF4_FORCE_DECODE | GNF4_TEST_STALL)) split = INT_MAX;
    if (flags & GNF4_FORCE_PREFILL) split = 0;
#ifndef GNF4_HAVE_PREFILL
    split = INT_MAX;
#endif
    if (split >= 1) {
        a.m_lo = 1;
        a.m_hi = split;
        cudaError_t e = launch_decode_band(fmt, a, s);
        if (e != cudaSuccess) return cuda_fail(e, "decode band launch");
    }
#ifdef GNF4_HAVE_PREFILL
    if (split < INT_MAX && R > split) {
        a.m_lo = split + 1;
        a.m_hi = INT_MAX;
        cudaError_t e = launch_prefill_band(fmt, a, T_in, s);
        if (e != cudaSuccess) return cuda_fail(e, "prefill band launch");
    }
#endif
    return GNF4_OK;
}

static gnf4_status dgrad(int fmt, const void* grad_out, const uint8_t* W, const void* scales,
                         const int64_t* offsets, const int32_t* row_src, const float* row_weight,
                         int64_t E, int64_t N, int64_t K, int64_t R, int64_t T_in, void* out,
                         int flags, void* stream) {
    if (E < 1 || N < 1 || K < 1 || R < 0 || T_in < 0)
        return fail(GNF4_ERR_INVALID_ARG, "sizes must be E,N,K >= 1 and R,T_in >= 0");
    if (flags & ~GNF4_CHECK) return fail(GNF4_ERR_INVALID_ARG, "only GNF4_CHECK is accepted (flags 0x%x)", flags);
    if (K % 64) return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "K must be a multiple of 64");
    if (N % 16) return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "N must be a multiple of 16");
    if (E > 2048) return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "at most 2048 experts");
    if (K > (int64_t)INT_MAX / 2 || E * N > (int64_t)INT_MAX || T_in > INT_MAX || R > INT_MAX)
        return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "K, E*N, T_in and R must fit in int32");
    if (!row_src && T_in < R) return fail(GNF4_ERR_INVALID_ARG, "row_src is NULL but T_in < R");
    if (R == 0) return GNF4_OK;                // no work: empty buffers may be NULL
    if (!grad_out || !W || !scales || !offsets || !out) return fail(GNF4_ERR_INVALID_ARG, "null pointer argument");
    if (!aligned16(grad_out) || !aligned16(W) || !aligned16(out))
        return fail(GNF4_ERR_MISALIGNED, "grad_out, W and out must be 16-byte aligned");
    if (!is_device_ptr(grad_out) || !is_device_ptr(W) || !is_device_ptr(scales) || !is_device_ptr(offsets) ||
        !is_device_ptr(out) || (row_src && !is_device_ptr(row_src)) || (row_weight && !is_device_ptr(row_weight)))
        return fail(GNF4_ERR_INVALID_ARG, "every buffer must be device memory of the current device");

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    static const LutPlanes lut_nf4 = make_lut(FMT_NF4, 0);
    static const LutPlanes lut_mx = make_lut(FMT_MXFP4, 0);
    if (flags & GNF4_CHECK) {
        GroupedArgs c;
        std::memset(&c, 0, sizeof(c));
        c.offsets = offsets;
        c.row_token = row_src;
        c.row_weight = row_weight;
        c.R = R;
        c.E = (int)E;
        unsigned st = 0;
        cudaError_t e = launch_check_routing(c, T_in, R, &st, s);
        if (e != cudaSuccess) return cuda_fail(e, "routing check");
        if (st) return fail(GNF4_ERR_DEVICE_STATUS,
                            "bad routing metadata (status 0x%x: 1 offsets decrease, 2 offsets[0] != 0 "
                            "or offsets[E] != R, 4 row_src out of range, 16 non-finite row_weight)", st);
    }
    DgradArgs a;
    a.g = reinterpret_cast<const uint16_t*>(grad_out);
    a.W = W;
    a.scales = scales;
    a.offsets = offsets;
    a.row_src = row_src;
    a.row_weight = row_weight;
    a.out = reinterpret_cast<uint16_t*>(out);
    a.R = R;
    a.E = (int)E;
    a.N = (int)N;
    a.K = (int)K;
    a.lut = (fmt == FMT_NF4) ? lut_nf4 : lut_mx;
    cudaError_t e = launch_dgrad(fmt, a, s);
    return e == cudaSuccess ? GNF4_OK : cuda_fail(e, "dgrad launch");
}

}  // namespace gnf4

using namespace gnf4;

extern "C" {

const char* gnf4_last_error(void) { return g_err; }

int gnf4_version(void) { return 100; }

gnf4_status gnf4_quantize_nf4(const float* w, int64_t rows, int64_t K, uint8_t* packed,
                              float* absmax, void* stream) {
    gnf4_status st = check_quantize_args(w, rows, K, packed, absmax, 64);
    if (st != GNF4_OK) return st;
    cudaError_t e = launch_quantize_nf4(w, rows, K, packed, absmax, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? GNF4_OK : cuda_fail(e, "quantize_nf4 launch");
}

gnf4_status gnf4_quantize_mxfp4(const float* w, int64_t rows, int64_t K, uint8_t* blocks,
                                uint8_t* scales, void* stream) {
    gnf4_status st = check_quantize_args(w, rows, K, blocks, scales, 32);
    if (st != GNF4_OK) return st;
    cudaError_t e = launch_quantize_mxfp4(w, rows, K, blocks, scales, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? GNF4_OK : cuda_fail(e, "quantize_mxfp4 launch");
}

gnf4_status gnf4_grouped_gemm_nf4(const void* x, const uint8_t* W, const float* absmax,
                                  const int64_t* expert_offsets, const int32_t* row_token,
                                  const float* row_weight, const int32_t* row_dest, int64_t E,
                                  int64_t N, int64_t K, int64_t R, int64_t T_in, int64_t T_out,
                                  void* out, int flags, void* stream) {
    return grouped(FMT_NF4, x, GNF4_DTYPE_BF16, W, absmax, GNF4_DTYPE_F32, expert_offsets, row_token, row_weight,
                   row_dest, E, N, K, R, T_in, T_out, out, flags, stream);
}

gnf4_status gnf4_grouped_gemm_mxfp4(const void* x, const uint8_t* W, const uint8_t* scales,
                                    const int64_t* expert_offsets, const int32_t* row_token,
                                    const float* row_weight, const int32_t* row_dest, int64_t E,
                                    int64_t N, int64_t K, int64_t R, int64_t T_in, int64_t T_out,
                                    void* out, int flags, void* stream) {
    return grouped(FMT_MXFP4, x, GNF4_DTYPE_BF16, W, scales, GNF4_DTYPE_BF16, expert_offsets, row_token,
                   row_weight, row_dest, E, N, K, R, T_in, T_out, out, flags, stream);
}

gnf4_status gnf4_grouped_gemm_nf4_ex(const void* x, int x_dtype, const uint8_t* W, const void* absmax,
                                     int absmax_dtype, const int64_t* expert_offsets, const int32_t* row_token,
                                     const float* row_weight, const int32_t* row_dest, int64_t E, int64_t N,
                                     int64_t K, int64_t R, int64_t T_in, int64_t T_out, void* out, int flags,
                                     void* stream) {
    return grouped(FMT_NF4, x, x_dtype, W, absmax, absmax_dtype, expert_offsets, row_token, row_weight,
                   row_dest, E, N, K, R, T_in, T_out, out, flags, stream);
}

gnf4_status gnf4_grouped_gemm_mxfp4_ex(const void* x, int x_dtype, const uint8_t* W, const uint8_t* scales,
                                       const int64_t* expert_offsets, const int32_t* row_token,
                                       const float* row_weight, const int32_t* row_dest, int64_t E, int64_t N,
                                       int64_t K, int64_t R, int64_t T_in, int64_t T_out, void* out, int flags,
                                       void* stream) {
    return grouped(FMT_MXFP4, x, x_dtype, W, scales, GNF4_DTYPE_BF16, expert_offsets, row_token, row_weight,
                   row_dest, E, N, K, R, T_in, T_out, out, flags, stream);
}

gnf4_status gnf4_grouped_gemm_swiglu_nf4(const void* x, int x_dtype, const uint8_t* W, const void* absmax,
                                         int absmax_dtype, const int64_t* expert_offsets, const int32_t* row_token,
                                         const float* row_weight, const int32_t* row_dest, int64_t E, int64_t N,
                                         int64_t K, int64_t R, int64_t T_in, int64_t T_out, void* out, int flags,
                                         void* stream) {
    return grouped(FMT_NF4, x, x_dtype, W, absmax, absmax_dtype, expert_offsets, row_token, row_weight,
                   row_dest, E, N, K, R, T_in, T_out, out, flags, stream, true);
}

gnf4_status gnf4_grouped_gemm_swiglu_mxfp4(const void* x, int x_dtype, const uint8_t* W, const uint8_t* scales,
                                           const int64_t* expert_offsets, const int32_t* row_token,
                                           const float* row_weight, const int32_t* row_dest, int64_t E,
                                           int64_t N, int64_t K, int64_t R, int64_t T_in, int64_t T_out,
                                           void* out, int flags, void* stream) {
    return grouped(FMT_MXFP4, x, x_dtype, W, scales, GNF4_DTYPE_BF16, expert_offsets, row_token, row_weight,
                   row_dest, E, N, K, R, T_in, T_out, out, flags, stream, true);
}

gnf4_status gnf4_absmax_to_bf16(const float* absmax, int64_t n, uint16_t* absmax_bf16, void* stream) {
    if (n < 0) return fail(GNF4_ERR_INVALID_ARG, "n must be >= 0");
    if (n == 0) return GNF4_OK;
    if (!absmax || !absmax_bf16) return fail(GNF4_ERR_INVALID_ARG, "null pointer argument");
    if ((reinterpret_cast<uintptr_t>(absmax) & 3u) || (reinterpret_cast<uintptr_t>(absmax_bf16) & 1u))
        return fail(GNF4_ERR_MISALIGNED, "absmax must be 4-byte and absmax_bf16 2-byte aligned");
    if (!is_device_ptr(absmax) || !is_device_ptr(absmax_bf16))
        return fail(GNF4_ERR_INVALID_ARG, "absmax and absmax_bf16 must be device memory of the current device");
    unsigned inexact = 0;
    cudaError_t e = launch_absmax_to_bf16(absmax, n, absmax_bf16, &inexact, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "absmax_to_bf16");
    if (inexact)
        return fail(GNF4_ERR_INVALID_ARG,
                    "some absmax values are not exactly representable in bf16 (the source is not bf16); "
                    "refused, absmax_bf16 holds unspecified values");
    return GNF4_OK;
}

gnf4_status gnf4_device_status(void* stream) {
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
    cudaError_t e1 = cudaSuccess, e2 = cudaSuccess;
    const unsigned d = take_decode_error(&e1), pr = take_prefill_error(&e2);
    if (e1 != cudaSuccess) return cuda_fail(e1, "read device status");
    if (e2 != cudaSuccess) return cuda_fail(e2, "read device status");
    if (d | pr)
        return fail(GNF4_ERR_DEVICE_STATUS, "a kernel gave up waiting on a barrier (decode 0x%x, prefill 0x%x)",
                    d, pr);
    return GNF4_OK;
}

gnf4_status gnf4_swiglu(const void* gate_up, int64_t R, int64_t I, void* out, void* stream) {
    if (R < 0 || I < 1) return fail(GNF4_ERR_INVALID_ARG, "sizes must be R >= 0 and I >= 1");
    if (I % 8) return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "I must be a multiple of 8");
    if (R == 0) return GNF4_OK;               // no work: empty buffers may be NULL
    if (!gate_up || !out) return fail(GNF4_ERR_INVALID_ARG, "null pointer argument");
    if (!aligned16(gate_up) || !aligned16(out))
        return fail(GNF4_ERR_MISALIGNED, "gate_up and out must be 16-byte aligned");
    if (!is_device_ptr(gate_up) || !is_device_ptr(out))
        return fail(GNF4_ERR_INVALID_ARG, "gate_up and out must be device memory");
    cudaError_t e = launch_swiglu(gate_up, R, I, out, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? GNF4_OK : cuda_fail(e, "swiglu launch");
}

gnf4_status gnf4_combine_topk(const void* y, int64_t R, int64_t N, const int32_t* row_of_slot,
                              const float* slot_weight, int64_t T, int64_t k, void* out,
                              void* stream) {
    if (R < 0 || N < 1 || T < 0 || k < 1)
        return fail(GNF4_ERR_INVALID_ARG, "sizes must be R, T >= 0 and N, k >= 1");
    if (N % 8) return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "N must be a multiple of 8");
    if (k > INT_MAX || T > INT64_MAX / k)
        return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "k must fit in int32 and T*k in int64");
    if (T == 0) return GNF4_OK;               // no work: empty buffers may be NULL
    if (!out || (R > 0 && !y)) return fail(GNF4_ERR_INVALID_ARG, "null pointer argument");
    if ((y && !aligned16(y)) || !aligned16(out))
        return fail(GNF4_ERR_MISALIGNED, "y and out must be 16-byte aligned");
    if ((y && !is_device_ptr(y)) || !is_device_ptr(out) || (row_of_slot && !is_device_ptr(row_of_slot)) ||
        (slot_weight && !is_device_ptr(slot_weight)))
        return fail(GNF4_ERR_INVALID_ARG, "every buffer must be device memory of the current device");
    cudaError_t e = launch_combine_topk(y, R, N, row_of_slot, slot_weight, T, k, out,
                                        reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? GNF4_OK : cuda_fail(e, "combine_topk launch");
}

gnf4_status gnf4_dgrad_nf4(const void* grad_out, const uint8_t* W, const float* absmax,
                           const int64_t* expert_offsets, const int32_t* row_src,
                           const float* row_weight, int64_t E, int64_t N, int64_t K, int64_t R,
                           int64_t T_in, void* out, int flags, void* stream) {
    return dgrad(FMT_NF4, grad_out, W, absmax, expert_offsets, row_src, row_weight, E, N, K, R, T_in,
                 out, flags, stream);
}

gnf4_status gnf4_dgrad_mxfp4(const void* grad_out, const uint8_t* W, const uint8_t* scales,
                             const int64_t* expert_offsets, const int32_t* row_src,
                             const float* row_weight, int64_t E, int64_t N, int64_t K, int64_t R,
                             int64_t T_in, void* out, int flags, void* stream) {
    return dgrad(FMT_MXFP4, grad_out, W, scales, expert_offsets, row_src, row_weight, E, N, K, R, T_in,
                 out, flags, stream);
}

gnf4_status gnf4_routing_metadata(const int32_t* topk_ids, const float* topk_weights, int64_t T,
                                  int64_t k, int64_t E, int64_t* expert_offsets, int32_t* row_token,
                                  float* row_weight, int32_t* row_dest, void* stream) {
    if (T < 0 || k < 1 || E < 1) return fail(GNF4_ERR_INVALID_ARG, "sizes must be T >= 0, k >= 1, E >= 1");
    if (E > 2048) return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "at most 2048 experts");
    if (k > INT_MAX || T > (int64_t)INT_MAX / k) return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "T*k must fit in int32");
    if (!expert_offsets || (T > 0 && (!row_token || !topk_ids)))   // T == 0: empty row arrays may be NULL
        return fail(GNF4_ERR_INVALID_ARG, "null pointer argument");
    if (T > 0 && (topk_weights == nullptr) != (row_weight == nullptr))
        return fail(GNF4_ERR_INVALID_ARG, "topk_weights and row_weight are given together or not at all");
    const void* ptrs[] = {topk_ids, topk_weights, expert_offsets, row_token, row_weight, row_dest};
    for (const void* q : ptrs) {
        if (!q) continue;
        if (reinterpret_cast<uintptr_t>(q) & 3u) return fail(GNF4_ERR_MISALIGNED, "buffers must be 4-byte aligned");
        if (!is_device_ptr(q)) return fail(GNF4_ERR_INVALID_ARG, "every buffer must be device memory of the current device");
    }
    if (reinterpret_cast<uintptr_t>(expert_offsets) & 7u)
        return fail(GNF4_ERR_MISALIGNED, "expert_offsets must be 8-byte aligned");
    cudaError_t e = launch_routing(topk_ids, topk_weights, T, k, (int)E, expert_offsets, row_token, row_weight,
                                   row_dest, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? GNF4_OK : cuda_fail(e, "routing launch");
}

int gnf4_grouped_gemm_launches(int64_t R, int flags) {
    if (R <= 0) return 0;
    int n = (flags & GNF4_CHECK) ? 1 : 0;
#ifdef GNF4_HAVE_PREFILL
    if (flags & (GNF4_FORCE_DECODE | GNF4_TEST_STALL)) return n + 1;
    if (flags & GNF4_FORCE_PREFILL) return n + 1;
    return n + 1 + (R > kDecodeOnlyRows ? 1 : 0);
#else
    return n + 1;
#endif
}

}  // extern "C"
