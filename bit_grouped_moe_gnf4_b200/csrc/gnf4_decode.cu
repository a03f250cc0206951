// Decode band of the grouped 4-bit GEMM: groups with few routed rows, where the
// packed weight bytes are the whole cost (the GEMV path of the solution page "How
// do I run a grouped GEMM directly on NF4 packed MoE expert weights, without
// dequantizing to bf16 first?", "Supported scope": one-token groups take the
// GEMV path; the status page "MoE Software Status & Known Limits", "Decode and
// serving": a bandwidth-targeted expert GEMV).
//
// Work. A unit is (active expert, tile of 64 weight rows, pass), where a pass
// covers up to 8*NG routed rows of the expert (larger groups take several
// passes). Units are numbered expert by expert, tile-major, and every CTA of the
// persistent grid (one per SM) takes an equal contiguous range; it finds the
// expert of its first unit by binary search. A CTA has 4 box rings ("quads") of
// 4/TPW warps each (TPW 16-row tiles a warp: 8 warps for NF4, 16 for MXFP4). The
// K axis of a tile is cut into np = 1 or 2 parts (the host's choice per call);
// the quads form 4/np groups of np quads, group gi takes the CTA's units gi,
// gi + 4/np, ..., and quad p of the group computes part p of each of them.
//
// Loads. The packed weights stream through the tensor memory accelerator: one
// lane of each quad issues, per 256-K chunk, one 2-D box of 64 rows x 128 bytes
// (8 KB, 128B-swizzled) into a 3-stage ring of the quad, so two chunks are in
// flight while the quad reads the third. When a row of block scales is TMA-able
// (16-byte pitch multiple, aligned array) a second box brings the chunk's scales
// of the same 64 rows into the stage; otherwise each warp loads its rows' scales
// a chunk ahead into registers. A full barrier per stage carries the copies' byte
// count; an empty barrier per stage collects the box's warps' release before the
// stage is refilled. The activations (shared by every tile of an expert) come
// through L1. The table below is built before the kernel's first global read, so
// under a programmatic dependent launch it overlaps the previous kernel's tail.
//
// Decode. A lane-replicated table in shared memory maps each packed byte to its
// two 16-bit values (entry b of lane l at b*256 + l*4: 32 lookups hit 32 banks).
// The table sits on a 64 KB boundary of the shared window, so one byte permute
// forms a lookup's whole address. It holds the codebook rounded to the
// activations' 16-bit type: the NF4 values, or the OCP e2m1 values with bit 3 as
// the sign.
//
// Math. Warp-level MMAs (m16n8k16, 16 weight rows x 8 routed rows) run one
// chain per scale block (64 K for NF4, 32 K for MXFP4), so every block sum
// leaves the tensor core in fp32 and is multiplied by its fp32 block scale and
// accumulated outside it. Lane (g, t) supplies the k-slots 2t, 2t+1, 2t+8, 2t+9
// of rows g and g+8; they are mapped to the four consecutive K positions
// 16t + 4s + {0,1,2,3} (NF4) or 8t + 4s + {..} (MXFP4) of step s inside the
// block, the same for both operands, so each lane reads contiguous bytes.
//
// Order of the fp32 sums. A row's K sum is one chain over its blocks in K order
// when K is a single chunk, and otherwise the sum of its two K halves (chunks
// [0, nc/2) and [nc/2, nc), each a chain in K order), half 0 + half 1. With two
// parts each quad of a group computes one half and the halves meet over shared
// memory (double-buffered, one named barrier per unit), each warp reducing a
// share of its rows; with one part a quad keeps half 0 aside and adds it at the
// unit's end. So a row's bits depend on K alone, never on the other rows of the
// call (row-count invariance), the part count, or which warp or CTA computed it.
// The epilogue applies the routing weight, rounds and scatters; nothing but the
// output is written to global memory.
//
// Waits. Every barrier wait is bounded: a wait that gives up records an error
// for gnf4_device_status, raises the CTA's abort flag (every other wait then
// returns at once, the math is skipped, the named-barrier schedule is kept), and
// before the CTA exits each quad's issuing lane waits, bounded again, for the
// copies it issued.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <climits>
#include <cstdint>

#include "gnf4_common.cuh"
#include "gnf4_kernels.h"

namespace gnf4 {

__device__ unsigned g_decode_error;

namespace db {

// A warp computes TPW tiles of 16 rows per chunk (1 or 2, a kernel template
// parameter): the 64-row box of a unit is shared by 4 / TPW warps, and a CTA has
// kQuads boxes in flight side by side (one ring each), so 16 / TPW warps.
#ifndef GNF4_DB_BOXES
#define GNF4_DB_BOXES 4
#endif
constexpr int kQuads = GNF4_DB_BOXES;
constexpr int kMaxWarps = 16;
constexpr int kTileRows = 64;                  // weight rows of a unit: 16 per warp of a quad
constexpr int kChunkK = 256;                   // K per chunk: 128 packed bytes of every row
constexpr int kBoxBytes = 128;
constexpr int kStageBytes = kTileRows * kBoxBytes;   // 8 KB: one TMA box
#ifndef GNF4_DB_STAGES
#define GNF4_DB_STAGES 3
#endif
constexpr int kStages = GNF4_DB_STAGES;       // ring stages per quad
// with the scales in the stage (ST): a second box of the chunk's block scales of the same
// 64 rows, 16 bytes a row, after the 8 KB of packed weights (stages stay 1024-aligned)
constexpr int kScaleBoxBytes = kTileRows * 16;
template <bool ST>
__host__ __device__ constexpr uint32_t stage_stride() { return ST ? kStageBytes + kScaleBoxBytes : kStageBytes; }
template <bool ST>
__host__ __device__ constexpr uint32_t ring_bytes() { return kStages * stage_stride<ST>(); }
constexpr int kLutBytes = 256 * 256;           // byte b, lane l -> b*256 + l*4 (bytes 128..255 of each row hold the part slots)
constexpr int kMaxTableRows = 1024;            // routed rows whose metadata a CTA stages in shared memory (at most)
constexpr int kMaxSmem = 227 * 1024;

// independent MMA chains per scale block (their sums are added in order afterwards)
#ifndef GNF4_DB_CHAINS
#define GNF4_DB_CHAINS 1
#endif

struct Plan {
    int np;          // K parts
    int nc;          // chunks of kChunkK (the last may be short)
    int nblk;        // scale blocks per weight row
    int vec_scales;  // a chunk's scales of one row can be read with one vector load
    int smem_bytes;  // dynamic shared memory of the launch
    int table_rows;  // routed rows whose metadata a CTA may stage (fewer when many experts fill the space)
};

// Scale storage of the band: f32 (NF4 absmax), bf16 (NF4 absmax stored as bf16),
// e8m0 (MXFP4).
enum ScaleKind : int { SC_F32 = 0, SC_BF16 = 1, SC_E8M0 = 2 };

template <int FMT>
struct ChunkGeom {
    static constexpr int SB = (FMT == FMT_NF4) ? 64 : 32;        // K per scale block
    static constexpr int NB = kChunkK / SB;                       // blocks per chunk (4 or 8)
    static constexpr int LB = SB / 8;                             // packed bytes per lane per row per block (8 or 4)
    static constexpr int LW = LB / 4;                             // 32-bit words of them (2 or 1)
};

// raw scale bits of one chunk for the lane's rows g and g + 8
template <int SCL>
struct Scales {
    uint32_t s[2][(SCL == SC_F32) ? 4 : 2];
};

__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}
__device__ __forceinline__ uint2 ld_nc_v2(const void* p) {
    uint2 v;
    asm volatile("ld.global.nc.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
    return v;
}
__device__ __forceinline__ uint32_t ld_nc_u32(const void* p) {
    uint32_t v;
    asm volatile("ld.global.nc.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}
__device__ __forceinline__ uint32_t ld_nc_u16(const void* p) {
    uint16_t v;
    asm volatile("ld.global.nc.u16 %0, [%1];" : "=h"(v) : "l"(p));
    return v;
}
__device__ __forceinline__ uint32_t ld_nc_u8(const void* p) {
    uint16_t v;
    asm volatile("ld.global.nc.u8 %0, [%1];" : "=h"(v) : "l"(p));
    return v;
}

__device__ __forceinline__ void tma_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar) : "memory");
}

// the chunk's block scales of rows g and g + 8 (sp at row g's first; s8 = 8 rows)
template <int SCL>
__device__ __forceinline__ void load_scales(Scales<SCL>& ck, const uint8_t* sp, int64_t s8, int nb, bool vec) {
    const uint8_t* sq = sp + s8;
    if constexpr (SCL == SC_F32) {
        if (vec) {
            const uint4 a = ld_nc_v4(sp);
            const uint4 b = ld_nc_v4(sq);
            ck.s[0][0] = a.x; ck.s[0][1] = a.y; ck.s[0][2] = a.z; ck.s[0][3] = a.w;
            ck.s[1][0] = b.x; ck.s[1][1] = b.y; ck.s[1][2] = b.z; ck.s[1][3] = b.w;
        } else {
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                ck.s[0][b] = b < nb ? ld_nc_u32(sp + 4 * b) : 0u;
                ck.s[1][b] = b < nb ? ld_nc_u32(sq + 4 * b) : 0u;
            }
        }
    } else if constexpr (SCL == SC_BF16) {
        if (vec) {
            const uint2 a = ld_nc_v2(sp);
            const uint2 b = ld_nc_v2(sq);
            ck.s[0][0] = a.x; ck.s[0][1] = a.y;
            ck.s[1][0] = b.x; ck.s[1][1] = b.y;
        } else {
            uint32_t v0[4], v1[4];
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                v0[b] = b < nb ? ld_nc_u16(sp + 2 * b) : 0u;
                v1[b] = b < nb ? ld_nc_u16(sq + 2 * b) : 0u;
            }
            ck.s[0][0] = v0[0] | (v0[1] << 16); ck.s[0][1] = v0[2] | (v0[3] << 16);
            ck.s[1][0] = v1[0] | (v1[1] << 16); ck.s[1][1] = v1[2] | (v1[3] << 16);
        }
    } else {
        if (vec) {
            const uint2 a = ld_nc_v2(sp);
            const uint2 b = ld_nc_v2(sq);
            ck.s[0][0] = a.x; ck.s[0][1] = a.y;
            ck.s[1][0] = b.x; ck.s[1][1] = b.y;
        } else {
            uint32_t v0[8], v1[8];
#pragma unroll
            for (int b = 0; b < 8; ++b) {
                v0[b] = b < nb ? ld_nc_u8(sp + b) : 0u;
                v1[b] = b < nb ? ld_nc_u8(sq + b) : 0u;
            }
            ck.s[0][0] = v0[0] | (v0[1] << 8) | (v0[2] << 16) | (v0[3] << 24);
            ck.s[0][1] = v0[4] | (v0[5] << 8) | (v0[6] << 16) | (v0[7] << 24);
            ck.s[1][0] = v1[0] | (v1[1] << 8) | (v1[2] << 16) | (v1[3] << 24);
            ck.s[1][1] = v1[4] | (v1[5] << 8) | (v1[6] << 16) | (v1[7] << 24);
        }
    }
}

// fp32 value of block b's scale of one row from the chunk's raw scale words
template <int SCL>
__device__ __forceinline__ float scale_of(const uint32_t* s, int b) {
    if constexpr (SCL == SC_F32) {
        return __uint_as_float(s[b]);
    } else if constexpr (SCL == SC_BF16) {
        return __uint_as_float(((s[b >> 1] >> (16 * (b & 1))) & 0xFFFFu) << 16);
    } else {
        return e8m0_to_f32((s[b >> 2] >> (8 * (b & 3))) & 0xFFu);
    }
}

// m16n8k16 with 16-bit operands of the activations' type, fp32 accumulate (no side
// effects: the compiler may interleave the chains of different blocks)
template <int XH>
__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    if constexpr (XH == 0) {
        asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
            "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
            : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
    } else {
        asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
            "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
            : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
    }
}

// one table lookup: a byte permute assembles the address from the lane's selector
// word (lane * 4 in byte 0, the table's 64 KB-aligned base in bytes 2..3) and packed
// byte i of w (byte 1). Not volatile, so the compiler may schedule it freely; it
// cannot rise above the table fill because lane_sel is produced after the barrier
// that follows the fill.
__device__ __forceinline__ uint32_t lut_lookup(uint32_t w, uint32_t lane_sel, int i) {
    const uint32_t a = prmt(w, lane_sel, 0x7604u | ((uint32_t)i << 4));
    uint32_t v;
    asm("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ uint2 lds_v2(uint32_t a) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
    return v;
}
__device__ __forceinline__ uint4 lds_v4(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}
__device__ __forceinline__ uint32_t lds_u32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}

// The MMAs of one chunk for one warp: for each of its TPW tiles of 16 rows, rows
// g / g+8 against NGC groups of 8 routed rows; acc[tt][j] += blocksum * scale per
// block. The packed bytes come from the stage: rowa[tt] is the lane's row ra = g of
// tile tt in the 128B-swizzled box, woff[b] the lane's byte offset of block b inside
// a row. xp[j] points at this lane's first activation of the chunk (or is null:
// zeros); the activations are shared by the tiles. FULL: every block is present.
template <int FMT, int SCL, int XH, int NGC, int NG, int TPW, bool FULL>
__device__ __forceinline__ void chunk_math(const uint32_t (&rowa)[TPW], const uint32_t (&woff)[ChunkGeom<FMT>::NB],
                                           const Scales<SCL> (&sc)[TPW], uint32_t lane_sel,
                                           const uint16_t* const (&xp)[NG], int nb, float (&acc)[TPW][NG][4]) {
    using G = ChunkGeom<FMT>;
    constexpr int XW = G::SB / 8;               // x words of one lane per block (8 or 4)
    constexpr int STEPS = G::SB / 16;           // k16 steps per block (4 or 2)
    // every packed word of the lane for the chunk: tiles x rows ra, ra + 8
    uint32_t w[TPW][2][G::NB * G::LW];
#pragma unroll
    for (int tt = 0; tt < TPW; ++tt) {
        const uint32_t rowb = rowa[tt] + 8 * kBoxBytes;
#pragma unroll
        for (int b = 0; b < G::NB; ++b) {
            if constexpr (G::LW == 2) {
                const uint2 va = lds_v2(rowa[tt] + woff[b]), vb = lds_v2(rowb + woff[b]);
                w[tt][0][2 * b] = va.x; w[tt][0][2 * b + 1] = va.y;
                w[tt][1][2 * b] = vb.x; w[tt][1][2 * b + 1] = vb.y;
            } else {
                w[tt][0][b] = lds_u32(rowa[tt] + woff[b]);
                w[tt][1][b] = lds_u32(rowb + woff[b]);
            }
        }
    }
    // activations of block b for every group (zeros where the lane has no routed row)
    auto load_x = [&](uint32_t (&xw)[NGC][XW], int b) {
#pragma unroll
        for (int j = 0; j < NGC; ++j) {
            if (xp[j] != nullptr) {
                const uint4* src = reinterpret_cast<const uint4*>(xp[j] + b * G::SB);
#pragma unroll
                for (int q = 0; q < XW / 4; ++q) {
                    const uint4 v = __ldg(src + q);
                    xw[j][4 * q] = v.x; xw[j][4 * q + 1] = v.y; xw[j][4 * q + 2] = v.z; xw[j][4 * q + 3] = v.w;
                }
            } else {
#pragma unroll
                for (int q = 0; q < XW; ++q) xw[j][q] = 0u;
            }
        }
    };
    // the next block's activations are loaded while this block computes
    uint32_t xa[NGC][XW], xb[NGC][XW];
    load_x(xa, 0);
#pragma unroll
    for (int b = 0; b < G::NB; ++b) {
        if (FULL || b < nb) {
            uint32_t (&xw)[NGC][XW] = (b & 1) ? xb : xa;
            uint32_t (&xn)[NGC][XW] = (b & 1) ? xa : xb;
            if (b + 1 < G::NB && (FULL || b + 1 < nb)) load_x(xn, b + 1);
            // CH independent MMA chains per block, tile and group (the block's k16 steps dealt
            // round robin), added in chain order: the same for every group count and tile
            // count, so a row's sum never depends on what shares its pass. The A operand of
            // step st is bytes 2st and 2st + 1 of rows ra and rb, decoded in operand order.
            constexpr int CH = GNF4_DB_CHAINS < STEPS ? GNF4_DB_CHAINS : STEPS;
            float c[TPW][NGC][CH][4];
#pragma unroll
            for (int tt = 0; tt < TPW; ++tt)
#pragma unroll
                for (int j = 0; j < NGC; ++j)
#pragma unroll
                    for (int h = 0; h < CH; ++h) c[tt][j][h][0] = c[tt][j][h][1] = c[tt][j][h][2] = c[tt][j][h][3] = 0.f;
#pragma unroll
            for (int st = 0; st < STEPS; ++st) {
#pragma unroll
                for (int tt = 0; tt < TPW; ++tt) {
                    const uint32_t a0 = lut_lookup(w[tt][0][G::LW * b + ((2 * st) >> 2)], lane_sel, (2 * st) & 3);
                    const uint32_t a1 = lut_lookup(w[tt][1][G::LW * b + ((2 * st) >> 2)], lane_sel, (2 * st) & 3);
                    const uint32_t a2 = lut_lookup(w[tt][0][G::LW * b + ((2 * st + 1) >> 2)], lane_sel, (2 * st + 1) & 3);
                    const uint32_t a3 = lut_lookup(w[tt][1][G::LW * b + ((2 * st + 1) >> 2)], lane_sel, (2 * st + 1) & 3);
#pragma unroll
                    for (int j = 0; j < NGC; ++j)
                        mma16816<XH>(c[tt][j][st % CH], a0, a1, a2, a3, xw[j][2 * st], xw[j][2 * st + 1]);
                }
            }
#pragma unroll
            for (int tt = 0; tt < TPW; ++tt)
#pragma unroll
                for (int j = 0; j < NGC; ++j)
#pragma unroll
                    for (int h = 1; h < CH; ++h)
#pragma unroll
                        for (int q = 0; q < 4; ++q) c[tt][j][0][q] += c[tt][j][h][q];
#pragma unroll
            for (int tt = 0; tt < TPW; ++tt) {
                const float sa = scale_of<SCL>(sc[tt].s[0], b);
                const float sb = scale_of<SCL>(sc[tt].s[1], b);
#pragma unroll
                for (int j = 0; j < NGC; ++j) {
                    acc[tt][j][0] = fmaf(c[tt][j][0][0], sa, acc[tt][j][0]);
                    acc[tt][j][1] = fmaf(c[tt][j][0][1], sa, acc[tt][j][1]);
                    acc[tt][j][2] = fmaf(c[tt][j][0][2], sb, acc[tt][j][2]);
                    acc[tt][j][3] = fmaf(c[tt][j][0][3], sb, acc[tt][j][3]);
                }
            }
        }
    }
}


// bytes of the shared memory other than the table and the rings: barriers and abort
// flag, expert tables, scan scratch, row table (16-byte multiple)
__host__ __device__ constexpr uint32_t other_bytes(int E, int table_rows) {
    return (uint32_t)(((2 * kQuads * kStages * 8 + 16 + 8ull * (E + 1) + 8ull * E + 8ull * kMaxWarps + 4ull * E +
                        4ull * E + 4ull * kMaxWarps + 12ull * table_rows) + 15) & ~15ull);
}

// Where the rings and the rest go, given the window address of the dynamic shared
// memory: the table on the first 64 KB boundary; each quad's ring (1024-aligned) and
// then the rest go into the first of the two gaps (before and after the table) that
// still holds them. Returns false if something does not fit (the host sizes the
// launch so that everything does).
struct Layout {
    uint32_t lut, ring[kQuads], other;
};
__host__ __device__ inline bool make_layout(uint32_t base, uint32_t bytes, int E, uint32_t kRingBytes, int table_rows,
                                            Layout& L) {
    const uint32_t end = base + bytes;
    const uint32_t lut = (base + 0xFFFFu) & ~0xFFFFu;
    if (lut + kLutBytes > end) return false;
    uint32_t lo = base, hi = lut + kLutBytes;         // free space: [lo, lut) and [hi, end)
    for (int q = 0; q < kQuads; ++q) {
        const uint32_t a = (lo + 1023u) & ~1023u;
        if (a + kRingBytes <= lut) {
            L.ring[q] = a;
            lo = a + kRingBytes;
            continue;
        }
        const uint32_t b = (hi + 1023u) & ~1023u;
        if (b + kRingBytes > end) return false;
        L.ring[q] = b;
        hi = b + kRingBytes;
    }
    const uint32_t ob = other_bytes(E, table_rows);
    const uint32_t a = (lo + 15u) & ~15u, b = (hi + 15u) & ~15u;
    if (a + ob <= lut) L.other = a;
    else if (b + ob <= end) L.other = b;
    else return false;
    L.lut = lut;
    return true;
}

// the stall test's limit: long enough for nothing, short enough to end the test fast
constexpr long long kStallTestWaitCycles = 1LL << 17;

__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, volatile int* abort_flag, bool stall_test) {
    return mbar_wait_bounded(bar, parity, abort_flag, &g_decode_error, 1u,
                             stall_test ? kStallTestWaitCycles : kWaitTimeoutCycles);
}

}  // namespace db

template <int FMT, int SCL, int XH, int NG, int TPW, int FUSE, bool ST>
__global__ void __launch_bounds__(db::kQuads * 128 / TPW, 1)
decode_band_kernel(const GroupedArgs p, const db::Plan pl, const __grid_constant__ CUtensorMap wmap,
                   const __grid_constant__ CUtensorMap smap) {
    using namespace db;
    static_assert(!FUSE || TPW == 2, "the fused SwiGLU pairs a gate tile with its up tile in one warp");
    static_assert(2 * kQuads * 4 * NG * 32 <= 256 * 8, "the part-sum slots must fit the table's spare halves");
    constexpr int kTPW = TPW;
    // A row's K sum is fixed by K alone: one chain for a single chunk, else the sum of its
    // two halves (chunks [0, nc/2) and [nc/2, nc)), half 0 + half 1 in fp32. With two K
    // parts each ring of a group computes one half and the hand-over adds them; with one
    // part (only in the variants with the registers for it: NF4, 8 routed rows a pass) a
    // ring keeps half 0 aside at the boundary and adds it at the unit's end. Either way the
    // same bits, so the host can pick the part count from the call's load.
    constexpr bool kHalvesInRing = (FMT == FMT_NF4) && (NG == 1);
    // FUSE: a unit is 32 gate rows [n0, n0 + 32) and their up rows [I + n0, I + n0 + 32) of
    // the fused gate_up matrix (two 32-row boxes per stage: gate in stage rows 0..31, up in
    // 32..63); warp wq takes gate rows n0 + 16 wq .. + 15 as tile 0 and the matching up rows
    // as tile 1, and writes silu(gate) * up into the [.., I] output
    constexpr int kUnitRows = FUSE ? 32 : kTileRows;
    constexpr int kBoxWarps = 4 / TPW;              // warps reading one box
    constexpr int kWarps = kQuads * kBoxWarps;
    constexpr int kThreads = kWarps * 32;
    static_assert(kWarps <= kMaxWarps, "the scan scratch holds one word per warp");
    using G = ChunkGeom<FMT>;
    constexpr int SSZ = (SCL == SC_F32) ? 4 : (SCL == SC_BF16) ? 2 : 1;   // bytes per scale

    extern __shared__ uint8_t smem_raw[];
    const uint32_t smem_s = smem_addr(smem_raw);
    Layout lay;
    constexpr uint32_t kStride = stage_stride<ST>();    // bytes of one ring stage
    if (!make_layout(smem_s, (uint32_t)pl.smem_bytes, p.E, ring_bytes<ST>(), pl.table_rows, lay)) {
        if (threadIdx.x == 0) atomicOr(&g_decode_error, 0x100u);
        return;
    }
    uint8_t* lut = smem_raw + (lay.lut - smem_s);
    uint8_t* other = smem_raw + (lay.other - smem_s);
    uint64_t* bars = reinterpret_cast<uint64_t*>(other);            // full[kQuads][kStages], empty[..]
    volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 2 * kQuads * kStages);
    int64_t* s_up = reinterpret_cast<int64_t*>(other + 2 * kQuads * kStages * 8 + 16);
    int64_t* s_r0 = s_up + (p.E + 1);
    int64_t* s_wu = s_r0 + p.E;                     // [kMaxWarps] scan scratch
    int* s_e = reinterpret_cast<int*>(s_wu + kMaxWarps);
    int* s_m = s_e + p.E;
    int* s_wc = s_m + p.E;                          // [kMaxWarps]
    int* t_tok = s_wc + kMaxWarps;
    float* t_wt = reinterpret_cast<float*>(t_tok + pl.table_rows);
    int* t_dst = reinterpret_cast<int*>(t_wt + pl.table_rows);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;
    const int quad = warp / kBoxWarps, wq = warp % kBoxWarps;   // box ring, warp within it
    const int row0 = 16 * kTPW * wq;                 // the warp's first row inside a unit's 64
    const int I = p.N / 2;                           // FUSE: output columns (the gate half)
    const int nrows = FUSE ? I : p.N;                 // rows that units cover
    const int ntile = (nrows + kUnitRows - 1) / kUnitRows;

    if (tid == 0) {
        for (int i = 0; i < kQuads * kStages; ++i) {
            mbar_init(smem_addr(bars + i), 1);                               // full: issuing lane + bytes
            mbar_init(smem_addr(bars + kQuads * kStages + i), kBoxWarps);    // empty: the box's warps
        }
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&wmap)) : "memory");
        if (ST) asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&smap)) : "memory");
    }
    // the lookup table comes from the kernel parameters alone, so it is built before
    // anything is read from global memory: under a programmatic dependent launch this
    // overlaps the tail of the kernel before; the wait below is the first point where
    // that kernel's results (offsets, routing rows, activations, even weights) are read
    {
        const LutPlanes L = p.lut;
        if constexpr (kWarps == 8 || kWarps == 16 || kWarps == 32) {
            // each of the 256 entries computed once (warp w % 8 owns bytes 32 (w % 8) ..
            // + 31, one a lane), then handed by shuffle to the lanes that store it: a store
            // instruction writes four entries' 128-byte rows, eight lanes a row (no conflict)
            constexpr int kShare = kWarps / 8;          // warps sharing one byte range
            const int wb = warp & 7, half = warp >> 3;
            const uint32_t v = byte_bf16x2<FMT>((uint32_t)(32 * wb + lane), L);
#pragma unroll
            for (int k = half * (8 / kShare); k < (half + 1) * (8 / kShare); ++k) {
                const uint32_t u = __shfl_sync(0xffffffffu, v, 4 * k + (lane >> 3));
                const int b = 32 * wb + 4 * k + (lane >> 3), q = lane & 7;
                *reinterpret_cast<uint4*>(lut + b * 256 + q * 16) = make_uint4(u, u, u, u);
            }
        } else {
            for (int i = tid; i < 256 * 8; i += kThreads) {
                const int b = i >> 3, q = i & 7;
                const uint32_t v = byte_bf16x2<FMT>((uint32_t)b, L);
                *reinterpret_cast<uint4*>(lut + b * 256 + q * 16) = make_uint4(v, v, v, v);
            }
        }
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // the next kernel of the stream may start its own prologue as SMs free up
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    // ---- active experts of this band and their unit counts (every CTA derives the same list) ----
    int nact = 0;
    int64_t utot = 0;
    for (int e0 = 0; e0 < p.E; e0 += kThreads) {
        const int e = e0 + tid;
        int act = 0, m = 0;
        int64_t o0 = 0, u = 0;
        if (e < p.E) {
            o0 = p.offsets[e];
            m = (int)(p.offsets[e + 1] - o0);
            act = (m >= p.m_lo && m <= p.m_hi) ? 1 : 0;
            if (act) u = (int64_t)ntile * ((m + 8 * NG - 1) / (8 * NG));
        }
        int ca = act;
        int64_t cu = u;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int ya = __shfl_up_sync(0xffffffffu, ca, d);
            const int64_t yu = __shfl_up_sync(0xffffffffu, cu, d);
            if (lane >= d) {
                ca += ya;
                cu += yu;
            }
        }
        if (lane == 31) {
            s_wc[warp] = ca;
            s_wu[warp] = cu;
        }
        __syncthreads();
        int pa = nact, ta = 0;
        int64_t pu = utot, tu = 0;
        for (int w = 0; w < kWarps; ++w) {
            const int c = s_wc[w];
            const int64_t cw = s_wu[w];
            if (w < warp) {
                pa += c;
                pu += cw;
            }
            ta += c;
            tu += cw;
        }
        if (act) {
            const int idx = pa + ca - 1;
            s_e[idx] = e;
            s_m[idx] = m;
            s_r0[idx] = o0;
            s_up[idx] = pu + cu - u;
        }
        nact += ta;
        utot += tu;
        __syncthreads();
    }
    const int64_t U0 = (int64_t)blockIdx.x * utot / gridDim.x;
    const int64_t U1 = (int64_t)(blockIdx.x + 1) * utot / gridDim.x;
    if (U0 >= U1) return;                            // whole CTA: no unit (no copy was issued)
    if (tid == 0) s_up[nact] = utot;
    __syncthreads();

    // ---- this quad's units and K part ----
    const int np = pl.np, ngroups = kQuads / np;
    const int gi = quad / np, part = quad - gi * np;
    const int c_lo = part * pl.nc / np, c_hi = (part + 1) * pl.nc / np;
    const int nck = c_hi - c_lo;
    const int nunit = (U1 - U0 > gi) ? (int)((U1 - U0 - gi + ngroups - 1) / ngroups) : 0;
    const int nsteps = nunit * nck;
    const int64_t s8 = 8 * (int64_t)pl.nblk * SSZ;
    const bool vec = pl.vec_scales != 0;
    const uint8_t* Sb = reinterpret_cast<const uint8_t*>(p.scales);
    // the stall test (a documented test flag) issues no copy at all: every first wait for
    // a stage gives up after a short limit, and the abort path runs with nothing in flight
    const bool stall_test = p.test_stall != 0;
    const bool issuer = (wq == 0 && lane == 0) && !stall_test;   // issues the box's copies
    uint64_t* full = bars + quad * kStages;
    uint64_t* empty = bars + kQuads * kStages + quad * kStages;
    uint32_t qring = lay.ring[0];
#pragma unroll
    for (int q = 1; q < kQuads; ++q)
        if (quad == q) qring = lay.ring[q];

    // the active expert that holds unit u: the last a with s_up[a] <= u (s_up rises
    // strictly: every active expert has at least one unit); a binary search, so that a
    // CTA late in the band does not walk every expert before it
    auto find_active = [&](int64_t u) -> int {
        int lo = 0, hi = nact - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (s_up[mid] <= u) lo = mid;
            else hi = mid - 1;
        }
        return lo;
    };
    const int a_first = find_active(U0);             // the expert of the CTA's first unit

    // routed rows [rlo, rhi) of the CTA's experts: staged in shared memory when few
    // enough. Each thread's first row is loaded now, so that the loads do not queue
    // behind the first weight copies; they land in the table after the copies went out.
    const int64_t rlo = s_r0[a_first];
    const int64_t rhi = [&] {
        const int a1 = find_active(U1 - 1);
        return s_r0[a1] + s_m[a1];
    }();
    const bool table = (rhi - rlo) <= pl.table_rows;
    const bool m_have = table && rlo + tid < rhi;
    int m_tok = 0, m_dst = 0;
    float m_wt = 0.f;
    if (m_have) {
        const int64_t r = rlo + tid;
        m_tok = p.row_token ? __ldg(p.row_token + r) : (int)r;
        m_wt = p.row_weight ? __ldg(p.row_weight + r) : 1.f;
        m_dst = p.row_dest ? __ldg(p.row_dest + r) : (int)r;
    }

    // unit u -> (active expert a, first weight row n0, first routed row of the pass mc);
    // a only moves forward along a quad's units (from a_first), so it is found by walking
    auto locate = [&](int64_t u, int& a, int& n0, int& mc) {
        while (s_up[a + 1] <= u) ++a;
        const int m = s_m[a];
        const int npass = (m + 8 * NG - 1) / (8 * NG);
        const int local = (int)(u - s_up[a]);
        int tile = local, pass = 0;
        if (npass > 1) {
            tile = local / npass;
            pass = local - tile * npass;
        }
        n0 = tile * kUnitRows;
        mc = pass * 8 * NG;
    };

    // copy cursor (issuing lane only): chunk j of the quad's sequence into stage j % kStages
    int cp_left = nsteps, cp_c = c_lo, cp_a = a_first, cp_y = 0, cp_j = 0, cp_s = 0;
    int64_t cp_u = U0 + gi;
    auto cp_unit = [&]() {
        int n0, mc;
        locate(cp_u, cp_a, n0, mc);
        cp_y = s_e[cp_a] * p.N + n0;
        cp_c = c_lo;
    };
    auto issue_next = [&]() {
        const uint32_t fb = smem_addr(full + cp_s);
        const uint32_t sdst = qring + (uint32_t)cp_s * kStride;
        mbar_arrive_tx(fb, (uint32_t)(kStageBytes + (ST ? kScaleBoxBytes : 0)));
        tma_2d(sdst, &wmap, cp_c * kBoxBytes, cp_y, fb);
        if (FUSE) tma_2d(sdst + kStageBytes / 2, &wmap, cp_c * kBoxBytes, cp_y + I, fb);
        if constexpr (ST) {
            // the 16 bytes holding this chunk's scales (8-byte formats: the pair of chunks
            // 2j, 2j+1, whose half the math picks)
            const int sx = (SSZ == 4) ? cp_c * 16 : (cp_c & ~1) * 8;
            tma_2d(sdst + kStageBytes, &smap, sx, cp_y, fb);
            if (FUSE) tma_2d(sdst + kStageBytes + kScaleBoxBytes / 2, &smap, sx, cp_y + I, fb);
        }
        if (++cp_s == kStages) cp_s = 0;
        ++cp_j;
        --cp_left;
        if (++cp_c == c_hi && cp_left > 0) {
            cp_u += ngroups;
            cp_unit();
        }
    };
    if (issuer && nsteps > 0) {
        cp_unit();
        // stage 0 of every ring now, the other stages once the table is up: the grid's
        // first chunks then land ahead of the rest of the opening burst
        if (cp_left > 0) issue_next();
    }

    // scale cursor (every warp, its own rows): one chunk ahead of the math
    int sc_left = nsteps, sc_c = c_lo, sc_a = a_first;
    int64_t sc_u = U0 + gi;
    const uint8_t* sc_p[kTPW];
    auto sc_unit = [&]() {
        int n0, mc;
        locate(sc_u, sc_a, n0, mc);
#pragma unroll
        for (int tt = 0; tt < kTPW; ++tt) {
            // rows past the end (a short last unit) read row g of the expert instead: in
            // bounds, unused
            const int r16 = FUSE ? n0 + 16 * wq : n0 + row0 + 16 * tt;
            const int rr = (r16 < nrows) ? r16 + g + (FUSE && tt == 1 ? I : 0) : g;
            const int64_t row = (int64_t)s_e[sc_a] * p.N + rr;
            sc_p[tt] = Sb + (row * pl.nblk + (int64_t)c_lo * G::NB) * SSZ;
        }
        sc_c = c_lo;
    };
    auto scales_next = [&](Scales<SCL> (&sc)[kTPW]) {
        if (sc_left <= 0) return;
        const int nb = min(G::NB, pl.nblk - sc_c * G::NB);
#pragma unroll
        for (int tt = 0; tt < kTPW; ++tt) {
            load_scales<SCL>(sc[tt], sc_p[tt], s8, nb, vec);
            sc_p[tt] += G::NB * SSZ;
        }
        --sc_left;
        if (++sc_c == c_hi && sc_left > 0) {
            sc_u += ngroups;
            sc_unit();
        }
    };
    Scales<SCL> scN[kTPW];                           // the next chunk's scales (scales not in the stage)
    if constexpr (!ST) {
        if (nsteps > 0) {
            sc_unit();
            scales_next(scN);
        }
    }

    // ---- the CTA's routing metadata: the first rows' loads went out before the copies ----
    if (table) {
        if (m_have) {
            t_tok[tid] = m_tok;
            t_wt[tid] = m_wt;
            t_dst[tid] = m_dst;
        }
        for (int64_t r = rlo + kThreads + tid; r < rhi; r += kThreads) {
            const int k = (int)(r - rlo);
            t_tok[k] = p.row_token ? __ldg(p.row_token + r) : (int)r;
            t_wt[k] = p.row_weight ? __ldg(p.row_weight + r) : 1.f;
            t_dst[k] = p.row_dest ? __ldg(p.row_dest + r) : (int)r;
        }
    }
    __syncthreads();

    if (issuer)
        while (cp_j < kStages && cp_left > 0) issue_next();
    // selector word of this lane's table lookups, made after the barrier (the volatile
    // move keeps every lookup, which depends on it, below the table fill)
    uint32_t lane_sel;
    asm volatile("mov.b32 %0, %1;" : "=r"(lane_sel) : "r"((lay.lut & 0xFFFF0000u) | ((uint32_t)lane << 2)) : "memory");
    auto tok_of = [&](int64_t r) -> int {
        return table ? t_tok[r - rlo] : (p.row_token ? __ldg(p.row_token + r) : (int)r);
    };
    auto wt_of = [&](int64_t r) -> float {
        return table ? t_wt[r - rlo] : (p.row_weight ? __ldg(p.row_weight + r) : 1.f);
    };
    auto dst_of = [&](int64_t r) -> int64_t {
        return table ? (int64_t)t_dst[r - rlo] : (p.row_dest ? (int64_t)__ldg(p.row_dest + r) : r);
    };
    uint16_t* out = p.out;
    // part sums of one lane: 16-byte slot s in the unused halves of the table's rows
    auto slot_ptr = [&](int s) -> float4* {
        return reinterpret_cast<float4*>(lut + (s >> 3) * 256 + 128 + (s & 7) * 16);
    };

    // ---- math cursor ----
    int mt_ck = 0, mt_a = a_first, mt_n0 = 0, mt_mc = 0, mt_unit = 0, nvalid = 0, ng = 0;
    int64_t mt_u = U0 + gi, mt_r0 = 0;
    int ntl = 0;                                    // this warp's tiles that exist in the unit (rows < N)
    float acc[kTPW][NG][4];
    float half0[kHalvesInRing ? kTPW : 1][NG][4];   // one part: the unit's half-0 sums
    const uint16_t* xp[NG];
    bool dead = false;

    auto unit_begin = [&]() {
        locate(mt_u, mt_a, mt_n0, mt_mc);
        mt_r0 = s_r0[mt_a];
        nvalid = min(8 * NG, s_m[mt_a] - mt_mc);
        ng = (nvalid + 7) >> 3;
        if (FUSE) ntl = (mt_n0 + 16 * wq < I) ? 2 : 0;
        else ntl = min(kTPW, max(0, (p.N - mt_n0 - row0) / 16));
#pragma unroll
        for (int j = 0; j < NG; ++j) {
            xp[j] = nullptr;
            const int jr = 8 * j + g;
            if (jr < nvalid)
                xp[j] = p.x + (int64_t)tok_of(mt_r0 + mt_mc + jr) * p.K + c_lo * kChunkK + t * (G::SB / 4);
#pragma unroll
            for (int tt = 0; tt < kTPW; ++tt) acc[tt][j][0] = acc[tt][j][1] = acc[tt][j][2] = acc[tt][j][3] = 0.f;
        }
    };
    // store one lane's four sums (rows n0 + row0 + 16 tt + lg and + 8; routed columns 2 lt,
    // 2 lt + 1 of group grp)
    auto store4 = [&](const float4& v, int tt, int lg, int lt, int grp) {
        const int n_a = mt_n0 + row0 + 16 * tt + lg, n_b = n_a + 8;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int jc = 8 * grp + 2 * lt + h;
            if (jc < nvalid) {
                const int64_t r = mt_r0 + mt_mc + jc;
                const float w = wt_of(r);
                const int64_t d = dst_of(r) * p.N;
                out[d + n_a] = f32_to_out16<XH>((h ? v.y : v.x) * w);
                out[d + n_b] = f32_to_out16<XH>((h ? v.w : v.z) * w);
            }
        }
    };
    // FUSE: the same four places of the gate tile (vg) and the up tile (vu) become
    // silu(w gate) * (w up) in output columns n0 + 16 wq + lg and + 8
    auto store4_fused = [&](const float4& vg, const float4& vu, int lg, int lt, int grp) {
        const int c_a = mt_n0 + 16 * wq + lg, c_b = c_a + 8;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int jc = 8 * grp + 2 * lt + h;
            if (jc < nvalid) {
                const int64_t r = mt_r0 + mt_mc + jc;
                const float w = wt_of(r);
                const int64_t d = dst_of(r) * I;
                out[d + c_a] = f32_to_out16<XH>(silu_mul((h ? vg.y : vg.x) * w, (h ? vu.y : vu.x) * w));
                out[d + c_b] = f32_to_out16<XH>(silu_mul((h ? vg.w : vg.z) * w, (h ? vu.w : vu.z) * w));
            }
        }
    };
    auto unit_end = [&]() {
        if (np == 1) {
            if constexpr (kHalvesInRing) {
                if (pl.nc >= 2) {
#pragma unroll
                    for (int tt = 0; tt < kTPW; ++tt)
#pragma unroll
                        for (int j = 0; j < NG; ++j)
#pragma unroll
                            for (int q = 0; q < 4; ++q) acc[tt][j][q] = half0[tt][j][q] + acc[tt][j][q];
                }
            }
            if (!dead) {
                if (FUSE) {
#pragma unroll
                    for (int j = 0; j < NG; ++j)
                        if (ntl == 2 && j < ng)
                            store4_fused(make_float4(acc[0][j][0], acc[0][j][1], acc[0][j][2], acc[0][j][3]),
                                         make_float4(acc[kTPW - 1][j][0], acc[kTPW - 1][j][1], acc[kTPW - 1][j][2],
                                                     acc[kTPW - 1][j][3]),
                                         g, t, j);
                } else {
#pragma unroll
                    for (int tt = 0; tt < kTPW; ++tt)
#pragma unroll
                        for (int j = 0; j < NG; ++j)
                            if (tt < ntl && j < ng)
                                store4(make_float4(acc[tt][j][0], acc[tt][j][1], acc[tt][j][2], acc[tt][j][3]), tt, g, t,
                                       j);
                }
            }
            return;
        }
        // hand the part sums to the group (slot of parity, warp, tile, group, lane), then
        // reduce a share of this warp's rows in part order
        const int par = mt_unit & 1;
#pragma unroll
        for (int tt = 0; tt < kTPW; ++tt)
#pragma unroll
            for (int j = 0; j < NG; ++j)
                if (j < ng)
                    *slot_ptr((((par * kWarps + warp) * kTPW + tt) * NG + j) * 32 + lane) =
                        make_float4(acc[tt][j][0], acc[tt][j][1], acc[tt][j][2], acc[tt][j][3]);
        asm volatile("bar.sync %0, %1;" ::"r"(1 + gi), "r"(np * kBoxWarps * 32) : "memory");
        auto part_sum = [&](int tt, int grp, int src) {
            // warp wq of box (gi * np + pp) holds part pp of these rows
            float4 v = *slot_ptr((((par * kWarps + (gi * np) * kBoxWarps + wq) * kTPW + tt) * NG + grp) * 32 + src);
            for (int pp = 1; pp < np; ++pp) {
                const float4 w = *slot_ptr((((par * kWarps + (gi * np + pp) * kBoxWarps + wq) * kTPW + tt) * NG + grp) * 32 + src);
                v.x += w.x; v.y += w.y; v.z += w.z; v.w += w.w;
            }
            return v;
        };
        if (FUSE) {
            const int ipw = (NG * 32) / np;         // items (one lane's gate and up float4s of one group)
            for (int i = lane; i < ipw && !dead; i += 32) {
                const int q = part * ipw + i;
                const int src = q & 31, grp = q >> 5;
                if (grp < ng && ntl == 2)
                    store4_fused(part_sum(0, grp, src), part_sum(kTPW - 1, grp, src), src >> 2, src & 3, grp);
            }
        } else {
            const int ipw = (kTPW * NG * 32) / np;  // items (one lane's float4 of one tile and group) per warp
            for (int i = lane; i < ipw && !dead; i += 32) {
                const int q = part * ipw + i;
                const int src = q & 31, grp = (q >> 5) % NG, tt = (q >> 5) / NG;
                if (grp < ng && tt < ntl) store4(part_sum(tt, grp, src), tt, src >> 2, src & 3, grp);
            }
        }
    };

    // this lane's byte offset of each block inside a 128-byte row of a stage (swizzled by g)
    uint32_t woff[G::NB];
#pragma unroll
    for (int b = 0; b < G::NB; ++b)
        woff[b] = (G::LW == 2) ? (((uint32_t)((2 * b + (t >> 1)) ^ g) << 4) + (uint32_t)(t & 1) * 8u)
                               : (((uint32_t)(b ^ g) << 4) + (uint32_t)t * 4u);
    const uint32_t lane_row = (uint32_t)(row0 + g) * kBoxBytes;
    const int nfull = pl.nblk / G::NB;              // chunks with every block present
    int cs = 0;                                     // stage of the current chunk
    uint32_t cph = 0;                               // its full-barrier parity
    int rs = 0;                                     // stage the issuing lane refills next
    uint32_t rph = 0;                               // parity of that stage's release

    auto step = [&]() {
        Scales<SCL> use[kTPW];                      // this chunk's scales (loaded a step ago, or from the stage)
        if constexpr (!ST) {
#pragma unroll
            for (int tt = 0; tt < kTPW; ++tt) use[tt] = scN[tt];
            scales_next(scN);
        }
        if (mt_ck == 0) unit_begin();
        if (!dead && !wait_bounded(smem_addr(full + cs), cph, abort_flag, stall_test)) dead = true;
        if (!dead && ntl > 0) {
            const int c = c_lo + mt_ck;
            uint32_t rowa[kTPW];
#pragma unroll
            for (int tt = 0; tt < kTPW; ++tt)
                rowa[tt] = qring + (uint32_t)cs * kStride +
                           (FUSE ? (uint32_t)(32 * tt + 16 * wq + g) * kBoxBytes : lane_row + tt * 16 * kBoxBytes);
            if constexpr (ST) {
                // rows g and g + 8 of each tile, 16 bytes a row after the stage's weights
                const uint32_t sb = qring + (uint32_t)cs * kStride + kStageBytes;
#pragma unroll
                for (int tt = 0; tt < kTPW; ++tt) {
                    const uint32_t ra = sb + (uint32_t)(FUSE ? 32 * tt + 16 * wq + g : row0 + 16 * tt + g) * 16u;
                    if constexpr (SCL == SC_F32) {
                        const uint4 va = lds_v4(ra), vb = lds_v4(ra + 128u);
                        use[tt].s[0][0] = va.x; use[tt].s[0][1] = va.y; use[tt].s[0][2] = va.z; use[tt].s[0][3] = va.w;
                        use[tt].s[1][0] = vb.x; use[tt].s[1][1] = vb.y; use[tt].s[1][2] = vb.z; use[tt].s[1][3] = vb.w;
                    } else {
                        const uint32_t h = (uint32_t)(c & 1) * 8u;
                        const uint2 va = lds_v2(ra + h), vb = lds_v2(ra + 128u + h);
                        use[tt].s[0][0] = va.x; use[tt].s[0][1] = va.y;
                        use[tt].s[1][0] = vb.x; use[tt].s[1][1] = vb.y;
                    }
                }
            }
            if (c < nfull) {
                if (NG == 1 || ng == 1)
                    chunk_math<FMT, SCL, XH, 1, NG, TPW, true>(rowa, woff, use, lane_sel, xp, G::NB, acc);
                else
                    chunk_math<FMT, SCL, XH, (NG > 1 ? 2 : 1), NG, TPW, true>(rowa, woff, use, lane_sel, xp, G::NB, acc);
            } else {
                const int nb = pl.nblk - c * G::NB;
                if (NG == 1 || ng == 1)
                    chunk_math<FMT, SCL, XH, 1, NG, TPW, false>(rowa, woff, use, lane_sel, xp, nb, acc);
                else
                    chunk_math<FMT, SCL, XH, (NG > 1 ? 2 : 1), NG, TPW, false>(rowa, woff, use, lane_sel, xp, nb, acc);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_addr(empty + cs));
        if (++cs == kStages) {
            cs = 0;
            cph ^= 1u;
        }
        // the issuing lane refills the oldest stage once every warp of the box released it
        // (the chunk kStages before the one it now receives)
        if (issuer && cp_left > 0 && cp_j >= kStages) {
            if (!dead && !wait_bounded(smem_addr(empty + rs), rph, abort_flag, stall_test)) dead = true;
            if (!dead) issue_next();
            if (++rs == kStages) {
                rs = 0;
                rph ^= 1u;
            }
        }
#pragma unroll
        for (int q = 0; q < NG; ++q)
            if (xp[q] != nullptr) xp[q] += kChunkK;
        if constexpr (kHalvesInRing) {
            // one part: the end of half 0 (chunk nc/2 - 1) puts its sums aside
            if (np == 1 && pl.nc >= 2 && c_lo + mt_ck + 1 == pl.nc / 2) {
#pragma unroll
                for (int tt = 0; tt < kTPW; ++tt)
#pragma unroll
                    for (int j = 0; j < NG; ++j)
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            half0[tt][j][q] = acc[tt][j][q];
                            acc[tt][j][q] = 0.f;
                        }
            }
        }
        if (++mt_ck == nck) {
            unit_end();
            mt_ck = 0;
            ++mt_unit;
            mt_u += ngroups;
        }
    };

    for (int j = 0; j < nsteps; ++j) step();

    // before the CTA exits: every copy this quad issued has landed. On the normal path
    // the math already waited for all of them; after an abort this wait (bounded, and
    // deaf to the abort flag) keeps the CTA's shared memory alive until they land.
    if (issuer) {
        for (int j = (cp_j > kStages ? cp_j - kStages : 0); j < cp_j; ++j) {
            const uint32_t bar = smem_addr(full + j % kStages), par = (uint32_t)((j / kStages) & 1);
            const long long t0 = clock64();
            while (!mbar_try_wait(bar, par, 2000u))
                if (clock64() - t0 > kWaitTimeoutCycles) {
                    atomicOr(&g_decode_error, 2u);
                    break;
                }
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

// the dynamic shared memory starts after the per-block reserved bytes (this kernel has
// no static shared memory): its window address, per device
static uint32_t decode_smem_base() {
    const int dev = current_device();
    static std::atomic<int> reserved[64];            // per device: reserved shared bytes + 1 (0 = unknown)
    int rsv = reserved[dev].load(std::memory_order_relaxed) - 1;
    if (rsv < 0) {
        if (cudaDeviceGetAttribute(&rsv, cudaDevAttrReservedSharedMemoryPerBlock, dev) != cudaSuccess) {
            cudaGetLastError();
            rsv = 1024;
        }
        reserved[dev].store(rsv + 1, std::memory_order_relaxed);
    }
    return (uint32_t)rsv;
}

// the smallest dynamic shared memory that holds the layout, or 0 if none does
static uint32_t decode_smem_bytes(int E, uint32_t ring_bytes, int table_rows) {
    db::Layout lay;
    const uint32_t base = decode_smem_base();
    for (uint32_t b = 64 * 1024; b <= (uint32_t)db::kMaxSmem; b += 1024)
        if (db::make_layout(base, b, E, ring_bytes, table_rows, lay)) return b;
    return 0;
}

template <int FMT, int SCL, int XH, int NG, int TPW, int FUSE, bool ST>
static cudaError_t launch_db_st(const GroupedArgs& a, db::Plan& pl, cudaStream_t s) {
    const int dev = current_device();
    const uint32_t bytes = (uint32_t)pl.smem_bytes;   // sized by the caller for this variant
    static std::atomic<bool> attr_done[64];          // per device: dynamic shared memory opted in
    if (!attr_done[dev].load(std::memory_order_acquire)) {
        cudaError_t e = cudaFuncSetAttribute(decode_band_kernel<FMT, SCL, XH, NG, TPW, FUSE, ST>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, db::kMaxSmem);
        if (e != cudaSuccess) return e;
        attr_done[dev].store(true, std::memory_order_release);
    }
    auto enc = encode_fn_db();
    if (!enc) return cudaErrorNotSupported;
    // packed weights as bytes [E*N, K/2]: boxes of 128 bytes x 64 rows (x 32 rows, two a
    // stage, for the fused SwiGLU), 128B swizzle
    const cuuint32_t box_rows = (cuuint32_t)(FUSE ? db::kTileRows / 2 : db::kTileRows);
    CUtensorMap wmap, smap;
    {
        cuuint64_t dims[2] = {(cuuint64_t)(a.K / 2), (cuuint64_t)a.E * (cuuint64_t)a.N};
        cuuint64_t strides[1] = {(cuuint64_t)(a.K / 2)};
        cuuint32_t box[2] = {(cuuint32_t)db::kBoxBytes, box_rows};
        cuuint32_t estr[2] = {1, 1};
        CUresult r = enc(&wmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(a.W), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    }
    if (ST) {
        // block scales as bytes [E*N, nblk * scale size]: boxes of 16 bytes x the weight box's rows
        constexpr int SSZ = (SCL == db::SC_F32) ? 4 : (SCL == db::SC_BF16) ? 2 : 1;
        cuuint64_t dims[2] = {(cuuint64_t)pl.nblk * SSZ, (cuuint64_t)a.E * (cuuint64_t)a.N};
        cuuint64_t strides[1] = {(cuuint64_t)pl.nblk * SSZ};
        cuuint32_t box[2] = {16, box_rows};
        cuuint32_t estr[2] = {1, 1};
        CUresult r = enc(&smap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(a.scales), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    } else {
        smap = wmap;                                 // not read
    }
    const int grid = device_sm_count();
    // programmatic dependent launch: the kernel builds its table while the previous
    // kernel of the stream drains, and waits for it (griddepcontrol.wait) before its
    // first global read
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3((unsigned)(db::kQuads * 128 / TPW));
    cfg.dynamicSmemBytes = bytes;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, decode_band_kernel<FMT, SCL, XH, NG, TPW, FUSE, ST>, a, pl, wmap, smap);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

// The chunk's block scales ride in the stage with the weights (a second TMA box) when
// every row's scales can be a TMA tensor: a row pitch of a multiple of 16 bytes and a
// 16-byte-aligned array; else each lane loads its rows' scales itself, a chunk ahead.
template <int FMT, int SCL, int XH, int NG, int TPW, int FUSE = 0>
static cudaError_t launch_db(const GroupedArgs& a, db::Plan& pl, cudaStream_t s) {
    constexpr int SSZ = (SCL == db::SC_F32) ? 4 : (SCL == db::SC_BF16) ? 2 : 1;
    const bool st_ok = ((int64_t)pl.nblk * SSZ) % 16 == 0 && (reinterpret_cast<uintptr_t>(a.scales) & 15u) == 0 &&
                       (int64_t)a.E * a.N < ((int64_t)1 << 31);
    // shared memory: the 9 KB stages of the scale boxes when they fit beside the per-expert
    // tables, with the largest routing-row table that fits (a CTA whose rows do not fit reads
    // them from global memory: the same results); else 8 KB stages, the same way
    for (int st = st_ok ? 1 : 0; st >= 0; --st)
        for (int rows = db::kMaxTableRows; rows >= 0; rows = rows > 64 ? rows / 2 : rows - 64) {
            const uint32_t b = decode_smem_bytes(a.E, st ? db::ring_bytes<true>() : db::ring_bytes<false>(), rows);
            if (b == 0) continue;
            pl.table_rows = rows;
            pl.smem_bytes = (int)b;
            return st ? launch_db_st<FMT, SCL, XH, NG, TPW, FUSE, true>(a, pl, s)
                      : launch_db_st<FMT, SCL, XH, NG, TPW, FUSE, false>(a, pl, s);
        }
    return cudaErrorInvalidConfiguration;
}

cudaError_t launch_decode_band(int fmt, const GroupedArgs& a, cudaStream_t s, bool fuse_swiglu) {
    db::Plan pl;
    const int SB = (fmt == FMT_NF4) ? 64 : 32;
    pl.nblk = a.K / SB;
    pl.nc = (a.K + db::kChunkK - 1) / db::kChunkK;
    pl.np = pl.nc >= 2 ? 2 : 1;                        // K parts (one half each; see below)
    pl.smem_bytes = 0;
    pl.table_rows = db::kMaxTableRows;
    const int per_chunk = db::kChunkK / SB;           // blocks of a chunk: one vector of scales per row
    // one vector load per row for a chunk's scales when every chunk's scales start
    // on a vector boundary (16 bytes of f32 x 4, 8 bytes of e8m0 x 8); else scalar loads
    const uintptr_t sbase = reinterpret_cast<uintptr_t>(a.scales);
    if (fmt == FMT_NF4 && !a.scale_bf16) pl.vec_scales = (pl.nblk % 4 == 0) && (sbase % 16 == 0);
    else if (fmt == FMT_NF4) pl.vec_scales = (pl.nblk % 4 == 0) && (sbase % 8 == 0);   // 8-byte bf16 x 4
    else pl.vec_scales = (pl.nblk % per_chunk == 0) && (sbase % 8 == 0);
    // 8 routed rows per pass when no group can exceed 8, or when groups are small on
    // average (fewer than 4 rows an expert: the rare larger group takes extra passes);
    // 16 per pass otherwise. Both give a row the same bits (one MMA chain per block and
    // group either way), so the choice never changes a result.
    const int64_t mmax = a.R < (int64_t)a.m_hi ? a.R : (int64_t)a.m_hi;      // no group exceeds this
    const bool one = mmax <= 8 || a.R < 4 * (int64_t)a.E;
    // A row's bits are fixed by K (the sum of its two K halves), so the part count may
    // follow the load: one part (a ring takes both halves, fewer part-sum hand-overs)
    // when the call has units for every ring of the grid twice over, in the variants
    // that can hold half 0 aside (NF4, 8 routed rows a pass); else two.
    if (pl.np == 2 && fmt == FMT_NF4 && one) {
        const int64_t rows_per_unit = fuse_swiglu ? db::kTileRows / 2 : db::kTileRows;
        const int64_t unit_rows = fuse_swiglu ? a.N / 2 : a.N;
        const int64_t units = (a.R < (int64_t)a.E ? a.R : (int64_t)a.E) * ((unit_rows + rows_per_unit - 1) / rows_per_unit);
        if (units >= 2 * (int64_t)db::kQuads * device_sm_count()) pl.np = 1;
    }
    if (fuse_swiglu) {
        // gate tile and up tile in one warp: two tiles a warp for both formats
        if (fmt == FMT_NF4) {
            if (a.scale_bf16) {
                if (a.x_f16) return one ? launch_db<FMT_NF4, db::SC_BF16, 1, 1, 2, 1>(a, pl, s) : launch_db<FMT_NF4, db::SC_BF16, 1, 2, 2, 1>(a, pl, s);
                return one ? launch_db<FMT_NF4, db::SC_BF16, 0, 1, 2, 1>(a, pl, s) : launch_db<FMT_NF4, db::SC_BF16, 0, 2, 2, 1>(a, pl, s);
            }
            if (a.x_f16) return one ? launch_db<FMT_NF4, db::SC_F32, 1, 1, 2, 1>(a, pl, s) : launch_db<FMT_NF4, db::SC_F32, 1, 2, 2, 1>(a, pl, s);
            return one ? launch_db<FMT_NF4, db::SC_F32, 0, 1, 2, 1>(a, pl, s) : launch_db<FMT_NF4, db::SC_F32, 0, 2, 2, 1>(a, pl, s);
        }
        if (a.x_f16) return one ? launch_db<FMT_MXFP4, db::SC_E8M0, 1, 1, 2, 1>(a, pl, s) : launch_db<FMT_MXFP4, db::SC_E8M0, 1, 2, 2, 1>(a, pl, s);
        return one ? launch_db<FMT_MXFP4, db::SC_E8M0, 0, 1, 2, 1>(a, pl, s) : launch_db<FMT_MXFP4, db::SC_E8M0, 0, 2, 2, 1>(a, pl, s);
    }
    // NF4 (4 blocks a chunk): two tiles a warp, 8 warps; MXFP4 (8 blocks a chunk, twice
    // the code and registers per tile): one tile a warp, 16 warps (measured faster each)
    if (fmt == FMT_NF4) {
        if (a.scale_bf16) {
            if (a.x_f16) return one ? launch_db<FMT_NF4, db::SC_BF16, 1, 1, 2>(a, pl, s) : launch_db<FMT_NF4, db::SC_BF16, 1, 2, 2>(a, pl, s);
            return one ? launch_db<FMT_NF4, db::SC_BF16, 0, 1, 2>(a, pl, s) : launch_db<FMT_NF4, db::SC_BF16, 0, 2, 2>(a, pl, s);
        }
        if (a.x_f16) return one ? launch_db<FMT_NF4, db::SC_F32, 1, 1, 2>(a, pl, s) : launch_db<FMT_NF4, db::SC_F32, 1, 2, 2>(a, pl, s);
        return one ? launch_db<FMT_NF4, db::SC_F32, 0, 1, 2>(a, pl, s) : launch_db<FMT_NF4, db::SC_F32, 0, 2, 2>(a, pl, s);
    }
    if (a.x_f16) return one ? launch_db<FMT_MXFP4, db::SC_E8M0, 1, 1, 1>(a, pl, s) : launch_db<FMT_MXFP4, db::SC_E8M0, 1, 2, 1>(a, pl, s);
    return one ? launch_db<FMT_MXFP4, db::SC_E8M0, 0, 1, 1>(a, pl, s) : launch_db<FMT_MXFP4, db::SC_E8M0, 0, 2, 1>(a, pl, s);
}

unsigned take_decode_error(cudaError_t* err) {
    unsigned v = 0;
    const unsigned zero = 0;
    *err = cudaMemcpyFromSymbol(&v, g_decode_error, sizeof(unsigned));
    if (*err == cudaSuccess && v) *err = cudaMemcpyToSymbol(g_decode_error, &zero, sizeof(unsigned));
    return v;
}

}  // namespace gnf4
