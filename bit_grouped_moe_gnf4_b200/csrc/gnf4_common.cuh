// Shared device-side pieces of the gnf4 kernels: argument block, nibble decode
// through byte permutes, scale decode, small PTX wrappers.
#pragma once

#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace gnf4 {

enum Fmt : int { FMT_NF4 = 0, FMT_MXFP4 = 1 };

// Byte planes of a 16-entry bf16 table for the prmt decode: lo[i] holds the low
// bytes of entries 4i..4i+3 (entry 4i in bits 0..7), hi[i] the high bytes.
// For MXFP4 only entries 0..7 (the e2m1 magnitudes) are used; bit 3 of a code
// is its sign.
struct LutPlanes {
    uint32_t lo[4];
    uint32_t hi[4];
};

struct GroupedArgs {
    const uint16_t* x;          // bf16 [T_in, K]
    const uint8_t* W;           // [E, N, K/2]
    const void* scales;         // NF4: f32 [E, N, K/64]; MXFP4: u8 [E, N, K/32]
    const int64_t* offsets;     // [E+1]
    const int32_t* row_token;   // [R] or null
    const float* row_weight;    // [R] or null
    const int32_t* row_dest;    // [R] or null
    uint16_t* out;              // bf16 [T_out, N]
    int64_t R;
    int E, N, K;
    int m_lo, m_hi;             // this band takes groups with m_lo <= rows <= m_hi
    int x_f16;                  // activations and output: 0 bf16, 1 fp16
    int test_stall;             // testing: the decode band issues no copies and waits at most 2^17 cycles
    int scale_bf16;             // NF4 absmax stored as bf16 (1) or fp32 (0)
    LutPlanes lut;              // codebook in the activations' 16-bit type
};

// Host-side: the decode tables of each format: the codebook values rounded to
// nearest even from fp32, to bf16 (f16 = 0) or to IEEE binary16 (f16 = 1).
LutPlanes make_lut(int fmt, int f16 = 0);

// ---------------------------------------------------------------------------
// device helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// Decode the 8 nibbles of one 32-bit word into four bf16x2 words: o[i] holds the
// two elements of byte i, the lower-k element in the low 16 bits.
//   NF4 (bitsandbytes order): element 2j is the HIGH nibble of byte j.
//   MXFP4 (OCP order):        element 2j is the LOW nibble of byte j.
// Codes are looked up by byte permutes (prmt) from tables held in registers:
// the low three bits of each nibble select a table byte, bit 3 picks the upper
// half of the table (NF4) or sets the sign (MXFP4). The result equals a plain
// 16-entry table lookup bit for bit.
template <int FMT>
__device__ __forceinline__ void decode_word(uint32_t w, const LutPlanes& L, uint32_t (&o)[4]) {
    const uint32_t s_lo = w & 0x77777777u;       // 3-bit selectors, nibbles 0..3 in bits 0..15
    const uint32_t s_hi = s_lo >> 16;            // nibbles 4..7
    const uint32_t w4 = w << 4;                  // puts bit 3 of every low nibble at a byte msb
    // byte i of m = 0xFF when nibble i (of the half) has bit 3 set
    const uint32_t m_lo = prmt(w, w4, 0x9D8Cu);
    const uint32_t m_hi = prmt(w, w4, 0xBFAEu);
    if constexpr (FMT == FMT_NF4) {
        uint32_t lo = (prmt(L.lo[0], L.lo[1], s_lo) & ~m_lo) | (prmt(L.lo[2], L.lo[3], s_lo) & m_lo);
        uint32_t hi = (prmt(L.hi[0], L.hi[1], s_lo) & ~m_lo) | (prmt(L.hi[2], L.hi[3], s_lo) & m_lo);
        o[0] = prmt(lo, hi, 0x4051u);            // byte 0: high nibble first
        o[1] = prmt(lo, hi, 0x6273u);
        lo = (prmt(L.lo[0], L.lo[1], s_hi) & ~m_hi) | (prmt(L.lo[2], L.lo[3], s_hi) & m_hi);
        hi = (prmt(L.hi[0], L.hi[1], s_hi) & ~m_hi) | (prmt(L.hi[2], L.hi[3], s_hi) & m_hi);
        o[2] = prmt(lo, hi, 0x4051u);
        o[3] = prmt(lo, hi, 0x6273u);
    } else {
        uint32_t lo = prmt(L.lo[0], L.lo[1], s_lo);
        uint32_t hi = prmt(L.hi[0], L.hi[1], s_lo) | (m_lo & 0x80808080u);
        o[0] = prmt(lo, hi, 0x5140u);            // byte 0: low nibble first
        o[1] = prmt(lo, hi, 0x7362u);
        lo = prmt(L.lo[0], L.lo[1], s_hi);
        hi = prmt(L.hi[0], L.hi[1], s_hi) | (m_hi & 0x80808080u);
        o[2] = prmt(lo, hi, 0x5140u);
        o[3] = prmt(lo, hi, 0x7362u);
    }
}

// e8m0 -> fp32: 2^(s-127); s = 0 is the subnormal 2^-127, s = 255 is NaN.
__device__ __forceinline__ float e8m0_to_f32(uint32_t s) {
    if (s == 0u) return __uint_as_float(0x00400000u);
    if (s == 255u) return __uint_as_float(0x7FC00000u);
    return __uint_as_float(s << 23);
}

// block scale idx as fp32: NF4 absmax stored as fp32 (SBF16 = false) or bf16 (widened
// exactly), MXFP4 e8m0
template <int FMT, bool SBF16 = false>
__device__ __forceinline__ float load_scale(const void* scales, int64_t idx) {
    if constexpr (FMT == FMT_NF4) {
        if constexpr (SBF16)
            return __uint_as_float((uint32_t)__ldg(reinterpret_cast<const uint16_t*>(scales) + idx) << 16);
        else
            return __ldg(reinterpret_cast<const float*>(scales) + idx);
    } else {
        return e8m0_to_f32(__ldg(reinterpret_cast<const uint8_t*>(scales) + idx));
    }
}

// fp32 -> bf16 bits, round to nearest even (NaN stays NaN).
__device__ __forceinline__ uint16_t f32_to_bf16_rne(float v) {
    uint32_t u = __float_as_uint(v);
    if ((u & 0x7FFFFFFFu) > 0x7F800000u) return (uint16_t)((u >> 16) | 0x40u);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

// SwiGLU pieces shared by the glue kernel and the fused gate_up epilogue.
// e^x for x <= 0 as 2^(x log2 e) on the hardware base-2 exponential (ex2.approx.f32:
// about 2^-22 relative error, subnormal results kept). Rounding x log2 e to fp32 adds
// at most 2^-24 |x log2 e| to the exponent, i.e. 2^-17.5 relative for |x| <= 88 (below
// that the result is subnormal and only the absolute error matters).
__device__ __forceinline__ float exp_via_ex2(float x) {
    float y;
    asm("ex2.approx.f32 %0, %1;" : "=f"(y) : "f"(x * 1.4426950408889634f));
    return y;
}

// silu(g) = g * sigmoid(g), with e = exp(-|g|) in (0, 1] so that nothing overflows:
// sigmoid(g) = 1 / (1 + e) for g >= 0 and e / (1 + e) for g < 0. The divisor is in
// [1, 2], where the fast division is within 2 ulp. For g far below zero g * e underflows
// gradually, as the exact value does.
__device__ __forceinline__ float silu_mul(float g, float u) {
    const float e = exp_via_ex2(-fabsf(g));
    const float num = g >= 0.0f ? g : g * e;
    return __fdividef(num, 1.0f + e) * u;
}

// fp32 -> the output's 16-bit type (XH = 0: bf16, 1: IEEE binary16), nearest even
template <int XH>
__device__ __forceinline__ uint16_t f32_to_out16(float v) {
    if constexpr (XH == 0) return f32_to_bf16_rne(v);
    else return __half_as_ushort(__float2half_rn(v));
}

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}


// ---------------------------------------------------------------------------
// mbarrier helpers shared by the kernels that pipeline through shared memory
// ---------------------------------------------------------------------------
constexpr long long kWaitTimeoutCycles = 1LL << 32;   // ~2 s at B200 clocks

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// One bounded attempt: the thread may sleep up to ~hint_ns inside the instruction.
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity, uint32_t hint_ns) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok) : "r"(bar), "r"(parity), "r"(hint_ns) : "memory");
    return ok != 0;
}

// Wait for the phase with parity `parity` to complete. Bounded: after
// kWaitTimeoutCycles without completion (or as soon as another warp of the CTA
// has given up) it records `code` in *err, raises the CTA's abort flag and
// returns false. The clock and the flag are polled only every 8th attempt.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                                  unsigned* err, unsigned code,
                                                  long long limit = kWaitTimeoutCycles) {
    if (mbar_try_wait(bar, parity, 0u)) return true;
    const long long t0 = clock64();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity, 2000u)) return true;
        if ((it & 7u) == 0u) {
            if (*abort_flag) return false;
            if (clock64() - t0 > limit) {
                *abort_flag = 1;
                atomicOr(err, code);
                return false;
            }
        }
    }
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

// bf16 bit pattern of one 4-bit code (NF4: 16-entry table; MXFP4: magnitude
// table of codes 0..7 plus the sign bit 3)
// (the plane word is chosen by selects, not by a runtime array index, so that
// the tables stay in registers)
__device__ __forceinline__ uint32_t plane_word(const uint32_t (&v)[4], uint32_t i) {
    return i == 0u ? v[0] : i == 1u ? v[1] : i == 2u ? v[2] : v[3];
}
template <int FMT>
__device__ __forceinline__ uint32_t code_bf16(uint32_t c, const LutPlanes& L) {
    if constexpr (FMT == FMT_NF4) {
        const uint32_t sh = 8u * (c & 3u);
        return (((plane_word(L.hi, c >> 2) >> sh) & 0xFFu) << 8) | ((plane_word(L.lo, c >> 2) >> sh) & 0xFFu);
    } else {
        const uint32_t m = c & 7u, sh = 8u * (m & 3u);
        return (((plane_word(L.hi, m >> 2) >> sh) & 0xFFu) << 8) | ((plane_word(L.lo, m >> 2) >> sh) & 0xFFu) |
               ((c & 8u) << 12);
    }
}

// bf16x2 word for one packed byte: the lower-k element in the low 16 bits
// (NF4: the high nibble comes first; MXFP4: the low nibble comes first)
template <int FMT>
__device__ __forceinline__ uint32_t byte_bf16x2(uint32_t b, const LutPlanes& L) {
    const uint32_t first = (FMT == FMT_NF4) ? (b >> 4) : (b & 15u);
    const uint32_t second = (FMT == FMT_NF4) ? (b & 15u) : (b >> 4);
    return code_bf16<FMT>(first, L) | (code_bf16<FMT>(second, L) << 16);
}

}  // namespace gnf4
