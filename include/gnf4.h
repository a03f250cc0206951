/*
 * gnf4 -- grouped GEMM for routed Mixture-of-Experts layers computed directly on
 * 4-bit-packed expert weights (NF4 or MXFP4), for NVIDIA B200 (sm_100a).
 *
 * C ABI. Every pointer argument marked "device" must be device (or managed)
 * memory of the current CUDA device; the library checks this and refuses host
 * pointers. The caller owns and allocates every buffer; the library allocates
 * nothing and keeps no per-call state beyond a few status words of its own in
 * device memory (see GNF4_CHECK and gnf4_device_status). Every call is asynchronous on `stream`
 * (a cudaStream_t passed as void*, NULL = the legacy default stream) and does
 * no host synchronisation unless GNF4_CHECK is set.
 *
 * Errors: each entry point returns a gnf4_status; on failure nothing was
 * launched (argument errors) or the CUDA error is reported (GNF4_ERR_CUDA),
 * and gnf4_last_error() returns a message for the calling thread.
 *
 * Citations name the grouped-nf4-gemm pages by title and section.
 */
#ifndef GNF4_H
#define GNF4_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum gnf4_status {
    GNF4_OK = 0,
    GNF4_ERR_INVALID_ARG = 1,      /* null pointer, negative size, host pointer, bad flag */
    GNF4_ERR_UNSUPPORTED_SHAPE = 2,/* K or N not a multiple of what the format needs */
    GNF4_ERR_MISALIGNED = 3,       /* a buffer that must be 16-byte aligned is not */
    GNF4_ERR_CUDA = 4,             /* a CUDA runtime call or launch failed */
    GNF4_ERR_DEVICE_STATUS = 5     /* GNF4_CHECK found bad routing metadata on the device */
} gnf4_status;

/* flags for the grouped GEMM entry points */
#define GNF4_CHECK          0x1  /* validate offsets / row_token / row_dest on the device
                                    first (one extra kernel and a stream sync); a bad
                                    value returns GNF4_ERR_DEVICE_STATUS, nothing else runs.
                                    Each checked call reports through its own status word
                                    (one of 256 taken round robin), so checked calls on
                                    different streams at the same time do not mix up their
                                    results as long as fewer than 256 are in flight */
#define GNF4_FORCE_DECODE   0x2  /* run every group through the decode band (testing) */
#define GNF4_FORCE_PREFILL  0x4  /* run every group through the prefill band (testing) */
#define GNF4_TEST_STALL   0x100  /* testing the error path: every group runs in the decode
                                    band, which issues none of its weight copies and waits at
                                    most 2^17 cycles, so its first wait gives up; the kernel
                                    records the event, skips the math and returns. The output
                                    is unspecified and gnf4_device_status then reports
                                    GNF4_ERR_DEVICE_STATUS; the next call runs normally */

/* storage types of the *_ex entry points */
#define GNF4_DTYPE_BF16 0    /* bfloat16 */
#define GNF4_DTYPE_F16  1    /* IEEE binary16 */
#define GNF4_DTYPE_F32  2    /* IEEE binary32 */

/* Message describing the last failure on the calling thread ("" if none). */
const char* gnf4_last_error(void);

/* Library version, major*10000 + minor*100 + patch. */
int gnf4_version(void);

/*
 * NF4 quantizer (input generation).
 * Follows the grouped-nf4-gemm README (0.11.0), "Try it on CPU right now", block 1:
 * a row-major fp32 matrix [rows, K] becomes [rows, K/2] uint8 codes plus one fp32
 * absmax per 64 consecutive K elements ("Supported scope" on the solution page:
 * blocksize 64, K % 64 == 0, bitsandbytes gemm_4bit layout).
 *   absmax[r, b] = max |w[r, 64b .. 64b+63]|
 *   code = nearest NF4 value to fl32(w / absmax) (ties to the lower code; an
 *          all-zero block gets code 7, the value 0)
 *   packed[r, j] = (code[r, 2j] << 4) | code[r, 2j+1]
 * w      device fp32 [rows, K], finite values (NaN/inf give unspecified codes)
 * packed device uint8 [rows, K/2]     (written)
 * absmax device fp32  [rows, K/64]    (written)
 * Output bytes are bit-identical to the CPU oracle's quantizer.
 * Errors: INVALID_ARG (null/host pointer, rows < 0, K <= 0), UNSUPPORTED_SHAPE (K % 64).
 */
gnf4_status gnf4_quantize_nf4(const float* w, int64_t rows, int64_t K,
                              uint8_t* packed, float* absmax, void* stream);

/*
 * MXFP4 quantizer (input generation): OCP e2m1 codes with one e8m0 scale per 32
 * K elements. README (0.11.0), "Try it on CPU right now", block 2 (blocks
 * [.., K/32, 16] u8 + scales [.., K/32] u8, the same bytes as the kernel view
 * [rows, K/2] + [rows, K/32] of "The NVMe tier").
 *   E = floor(log2 amax) - 2 (from the fp32 exponent field, clamped to [-127,127];
 *       E = 0 for an all-zero block), scales[r, b] = E + 127
 *   code = e2m1 nearest to w * 2^-E, ties to the even code, |.| > 6 -> 6,
 *          sign bit set when w < 0
 *   blocks[r, j] = code[r, 2j] | (code[r, 2j+1] << 4)
 * w device fp32 [rows, K]; blocks device uint8 [rows, K/2]; scales device uint8 [rows, K/32].
 * Errors: INVALID_ARG, UNSUPPORTED_SHAPE (K % 32).
 */
gnf4_status gnf4_quantize_mxfp4(const float* w, int64_t rows, int64_t K,
                                uint8_t* blocks, uint8_t* scales, void* stream);

/*
 * Grouped GEMM on NF4-packed expert weights.
 * The op of the solution page "How do I run a grouped GEMM directly on NF4
 * packed MoE expert weights, without dequantizing to bf16 first?" ("Smallest
 * correct example", "Supported scope"): every active expert in one call, nibbles
 * decoded on chip, fp32 block scaling and accumulation, bf16 output, no bf16
 * copy of any expert in memory. Routed rows r = 0..R-1 are sorted by expert:
 * expert e owns rows [expert_offsets[e], expert_offsets[e+1]).
 *
 *   out[dest(r), n] = bf16_rne( w(r) * sum_k x[tok(r), k] * What[e(r), n, k] )
 *   What[e, n, k]   = nf4[code(e, n, k)] * absmax[e, n, k/64]
 *   tok(r)  = row_token ? row_token[r] : r
 *   w(r)    = row_weight ? row_weight[r] : 1
 *   dest(r) = row_dest ? row_dest[r] : r
 *
 * x              device bf16 [T_in, K], 16-byte aligned
 * W              device uint8 [E, N, K/2] (NF4 codes as gnf4_quantize_nf4 writes them), 16-byte aligned
 * absmax         device fp32  [E, N, K/64], 4-byte aligned (any offset into a float
 *                array). With 16-byte alignment and K % 256 == 0 the decode band brings
 *                each chunk's scales in with its weight copies (TMA); otherwise each lane
 *                loads them itself. Both ways give the same bits.
 * expert_offsets device int64 [E+1], 8-byte aligned: offsets[0] = 0, non-decreasing,
 *                offsets[E] = R; empty experts (equal neighbours) are legal and cost nothing
 * row_token      device int32 [R] in [0, T_in), or NULL (then T_in >= R); 4-byte aligned
 * row_weight     device fp32  [R], or NULL; 4-byte aligned
 * row_dest       device int32 [R] in [0, T_out), pairwise distinct, or NULL (then T_out >= R);
 *                4-byte aligned
 * out            device bf16 [T_out, N], 16-byte aligned; rows that no routed row
 *                names are not written
 * E >= 1, N % 16 == 0, K % 64 == 0, R >= 0 (R == 0 launches nothing), T_in, T_out < 2^31.
 * Offsets are 64-bit everywhere inside, so stacks past 2^31 bytes are addressed
 * correctly (the int64-offset rule under "Supported scope" / "Limitations").
 * flags: 0, or GNF4_CHECK / GNF4_FORCE_DECODE / GNF4_FORCE_PREFILL (above).
 * Bands: groups of at most 64 rows run in the decode band, larger groups in the
 * prefill band (tensor cores); a call with R <= 128 runs every group in the
 * decode band (one launch). Results are deterministic: the same inputs give the
 * same bits on every call. Inside the decode band a row's bits do not depend on
 * the other rows of the call (its fp32 summation order is fixed by K alone); a row
 * computed in the prefill band may differ from it in the last bits.
 */
gnf4_status gnf4_grouped_gemm_nf4(const void* x, const uint8_t* W, const float* absmax,
                                  const int64_t* expert_offsets, const int32_t* row_token,
                                  const float* row_weight, const int32_t* row_dest,
                                  int64_t E, int64_t N, int64_t K, int64_t R,
                                  int64_t T_in, int64_t T_out, void* out,
                                  int flags, void* stream);

/*
 * Grouped GEMM on MXFP4-packed expert weights: identical contract, with
 *   What[e, n, k] = e2m1[code(e, n, k)] * 2^(scales[e, n, k/32] - 127)
 * W      device uint8 [E, N, K/2] (element 2j in the low nibble of byte j)
 * scales device uint8 [E, N, K/32] (e8m0; 255 decodes to NaN), any alignment; with
 *        16-byte alignment and K % 512 == 0 the decode band copies them by TMA (same bits)
 * K % 32 == 0. The README's "MXFP4 native-byte lane": the same mainloop by
 * table swap, on the released bytes.
 */
gnf4_status gnf4_grouped_gemm_mxfp4(const void* x, const uint8_t* W, const uint8_t* scales,
                                    const int64_t* expert_offsets, const int32_t* row_token,
                                    const float* row_weight, const int32_t* row_dest,
                                    int64_t E, int64_t N, int64_t K, int64_t R,
                                    int64_t T_in, int64_t T_out, void* out,
                                    int flags, void* stream);

/*
 * Storage variants of the two grouped GEMMs (the same op, contract and errors as
 * gnf4_grouped_gemm_nf4 / _mxfp4 above, plus the checks of the two type arguments):
 *  - x_dtype: the activations and the output are bf16 (GNF4_DTYPE_BF16) or IEEE
 *    binary16 (GNF4_DTYPE_F16): `a_cat [T, K]` bf16/fp16 on the solution page,
 *    "Supported scope". With fp16 the codebook is decoded to fp16 (rounded to
 *    nearest even once; the e2m1 values are exact), the tensor-core operands are
 *    fp16, accumulation stays fp32, and out[...] is rounded once to fp16 (the
 *    output type follows the activations).
 *  - absmax_dtype (NF4): fp32 (GNF4_DTYPE_F32, 4-byte aligned) or bf16
 *    (GNF4_DTYPE_BF16, 2-byte aligned): the grouped-nf4-gemm README (0.11.0), "Which
 *    entry point? Pick by where the weights live", the --absmax-dtype bf16 paragraph:
 *    5.6 % fewer bytes per NF4 row, lossless for a bf16 source (see
 *    gnf4_absmax_to_bf16). The bf16 absmax is widened exactly to fp32 on chip; the
 *    block scaling is still fp32, outside the MMA. (The decode band copies bf16
 *    absmax by TMA when it is 16-byte aligned and K % 512 == 0; same bits otherwise.)
 * gnf4_grouped_gemm_nf4_ex(x, GNF4_DTYPE_BF16, W, absmax, GNF4_DTYPE_F32, ...) is
 * gnf4_grouped_gemm_nf4(x, W, absmax, ...) bit for bit.
 * Errors: as above; INVALID_ARG for an unknown type, MISALIGNED for an absmax off
 * its type's alignment.
 */
gnf4_status gnf4_grouped_gemm_nf4_ex(const void* x, int x_dtype, const uint8_t* W, const void* absmax,
                                     int absmax_dtype, const int64_t* expert_offsets,
                                     const int32_t* row_token, const float* row_weight,
                                     const int32_t* row_dest, int64_t E, int64_t N, int64_t K, int64_t R,
                                     int64_t T_in, int64_t T_out, void* out, int flags, void* stream);
gnf4_status gnf4_grouped_gemm_mxfp4_ex(const void* x, int x_dtype, const uint8_t* W, const uint8_t* scales,
                                       const int64_t* expert_offsets, const int32_t* row_token,
                                       const float* row_weight, const int32_t* row_dest, int64_t E,
                                       int64_t N, int64_t K, int64_t R, int64_t T_in, int64_t T_out,
                                       void* out, int flags, void* stream);

/*
 * gate_up grouped GEMM with the SwiGLU fused into its epilogue: the step between the
 * gate_up and down projections of a SwiGLU MoE layer (the decode glue "swiglu_rows" of
 * the status page "MoE Software Status & Known Limits", "Correctness contracts"; the
 * SwiGLU architectures of the experts4bit-qlora README, "Scope") done where the gate_up
 * sums are still fp32 in registers, so the [R, 2I] gate_up rows never reach memory.
 * For routed row r, with G and U the gate_up call's fp32 results before rounding
 * (row j of W[e] the gate of column j, row I + j its up; routing weight included):
 *   out[dest(r), j] = round16( silu(w(r) G[r, j]) * (w(r) U[r, j]) ),  j < I = N / 2
 * i.e. gnf4_swiglu applied to gnf4_grouped_gemm_*_ex's output without rounding the
 * gate_up rows in between (silu as in gnf4_swiglu). Arguments as in
 * gnf4_grouped_gemm_{nf4,mxfp4}_ex, with N = 2I the fused gate_up width (N % 32 == 0)
 * and out [T_out, I] of the activations' type. Every group runs in the decode band
 * (one launch; groups above 8 or 16 rows take several passes over their weights), so
 * for prefill-sized groups the unfused GEMM + gnf4_swiglu is the faster pair.
 * flags: 0, GNF4_CHECK or GNF4_FORCE_DECODE (a no-op); GNF4_FORCE_PREFILL is refused.
 * Errors: as for the grouped GEMM; UNSUPPORTED_SHAPE if N % 32.
 */
gnf4_status gnf4_grouped_gemm_swiglu_nf4(const void* x, int x_dtype, const uint8_t* W, const void* absmax,
                                         int absmax_dtype, const int64_t* expert_offsets,
                                         const int32_t* row_token, const float* row_weight,
                                         const int32_t* row_dest, int64_t E, int64_t N, int64_t K, int64_t R,
                                         int64_t T_in, int64_t T_out, void* out, int flags, void* stream);
gnf4_status gnf4_grouped_gemm_swiglu_mxfp4(const void* x, int x_dtype, const uint8_t* W, const uint8_t* scales,
                                           const int64_t* expert_offsets, const int32_t* row_token,
                                           const float* row_weight, const int32_t* row_dest, int64_t E,
                                           int64_t N, int64_t K, int64_t R, int64_t T_in, int64_t T_out,
                                           void* out, int flags, void* stream);

/*
 * The lossless absmax cast of the bf16-absmax storage (README 0.11.0, "Which entry
 * point?", the --absmax-dtype bf16 paragraph: the cast refuses rather than rounds).
 * absmax_bf16[i] = the bf16 pattern of absmax[i] (its high 16 bits); an fp32 value
 * whose low 16 bits are not all zero has no bf16 equal, and then the call returns
 * GNF4_ERR_INVALID_ARG and absmax_bf16 holds unspecified values. For the NF4 absmax
 * of a bf16 source every value passes (each is one of its block's magnitudes).
 * absmax device fp32 [n] (4-byte aligned); absmax_bf16 device uint16 [n] (2-byte
 * aligned). Synchronises `stream` (it reads the verdict back). n == 0 does nothing.
 * Errors: INVALID_ARG, MISALIGNED, CUDA.
 */
gnf4_status gnf4_absmax_to_bf16(const float* absmax, int64_t n, uint16_t* absmax_bf16, void* stream);

/*
 * Synchronise `stream` and report whether any grouped GEMM kernel since the last
 * call gave up waiting on one of its internal barriers (every such wait is
 * bounded, so a kernel never hangs; it stops, records the event and returns).
 * Returns GNF4_ERR_DEVICE_STATUS (and clears the record) if one did, GNF4_ERR_CUDA
 * if the stream reports an error, GNF4_OK otherwise.
 */
gnf4_status gnf4_device_status(void* stream);

/*
 * Input gradient of the grouped GEMM on NF4-packed weights, every group in one launch:
 * the grouped-nf4-gemm README (0.11.0), "Training: the backward is a kernel too (0.7.0)"
 * (grad_out @ dequant(B), decoded on chip, nothing materialised), and the solution page,
 * "Supported scope" (dgrad_4bit_grouped). For routed rows r sorted by expert as in the
 * forward call,
 *
 *   out[r, k] = bf16_rne( w(r) * sum_n grad_out[src(r), n] * What[e(r), n, k] )
 *   src(r) = row_src ? row_src[r] : r      (the forward's row_dest, when it scattered)
 *   w(r)   = row_weight ? row_weight[r] : 1 (the forward's routing weight)
 *
 * so out is the gradient of the forward's routed input rows (a_cat order); summing the
 * rows of one token is gnf4_combine_topk with row_of_slot. The contraction runs over N,
 * across rows with different block scales, so the scale multiplies each decoded bf16
 * pair before the MMA: exact for MXFP4 (a power of two), one extra bf16 rounding of the
 * scaled weight for NF4. fp32 accumulation in a fixed order (deterministic).
 * grad_out   device bf16 [T_in, N], 16-byte aligned
 * W, absmax  the forward's packed stack: u8 [E, N, K/2] (16-byte aligned), f32 [E, N, K/64]
 * expert_offsets device int64 [E+1] as in the forward
 * row_src    device int32 [R] in [0, T_in), or NULL (then T_in >= R)
 * row_weight device fp32 [R], or NULL
 * out        device bf16 [R, K], 16-byte aligned
 * E in [1, 2048], N % 16 == 0, K % 64 == 0 (both formats), R >= 0 (R == 0 launches nothing
 * and accepts NULL buffers). flags: 0 or GNF4_CHECK (validates offsets, row_src, row_weight
 * first, as in the forward). One kernel launch (two with GNF4_CHECK).
 * Errors: INVALID_ARG, UNSUPPORTED_SHAPE, MISALIGNED, DEVICE_STATUS (GNF4_CHECK), CUDA.
 */
gnf4_status gnf4_dgrad_nf4(const void* grad_out, const uint8_t* W, const float* absmax,
                           const int64_t* expert_offsets, const int32_t* row_src,
                           const float* row_weight, int64_t E, int64_t N, int64_t K, int64_t R,
                           int64_t T_in, void* out, int flags, void* stream);

/*
 * The same input gradient on MXFP4-packed weights (scales u8 e8m0 [E, N, K/32]).
 */
gnf4_status gnf4_dgrad_mxfp4(const void* grad_out, const uint8_t* W, const uint8_t* scales,
                             const int64_t* expert_offsets, const int32_t* row_src,
                             const float* row_weight, int64_t E, int64_t N, int64_t K, int64_t R,
                             int64_t T_in, void* out, int flags, void* stream);

/*
 * Routing metadata on the device: the router's top-k choices become the arguments of a
 * grouped call, so that a whole MoE layer runs without the host. The grouped call takes
 * its rows "group-sorted", with sort and scatter outside the kernel (solution page,
 * "Supported scope"; "Smallest correct example": sizes per expert, rows of one expert
 * contiguous). Routed rows are the pairs (t, s), t < T, s < k, ordered by expert
 * topk_ids[t*k + s], then t, then s (a stable counting sort):
 *   expert_offsets[e] = number of pairs with expert < e           (int64 [E+1])
 *   row r = pair (t, s):  row_token[r] = t, row_dest[r] = t*k + s, row_weight[r] = topk_weights[t*k + s]
 * An id outside [0, E) is a dropped slot and gets no row; then R = expert_offsets[E] < T*k
 * and only the first R entries of the row arrays are written. With every id valid R = T*k,
 * known on the host, and the grouped calls can be captured in one CUDA graph with this one.
 * topk_ids     device int32 [T, k] (with T == 0 the row arrays and topk_ids may be NULL;
 *              expert_offsets is still written, all zero)
 * topk_weights device fp32 [T, k], or NULL (then row_weight must be NULL)
 * expert_offsets device int64 [E+1] (8-byte aligned); row_token device int32 [T*k];
 * row_weight device fp32 [T*k] or NULL; row_dest device int32 [T*k] or NULL
 * E in [1, 2048], T*k < 2^31. One kernel launch of one CTA; deterministic (the same bits
 * on every call), no atomics on the outputs.
 * Errors: INVALID_ARG, UNSUPPORTED_SHAPE, MISALIGNED, CUDA.
 */
gnf4_status gnf4_routing_metadata(const int32_t* topk_ids, const float* topk_weights, int64_t T,
                                  int64_t k, int64_t E, int64_t* expert_offsets, int32_t* row_token,
                                  float* row_weight, int32_t* row_dest, void* stream);

/*
 * SwiGLU over gate_up rows: the step between the gate_up and down grouped GEMMs
 * of a SwiGLU MoE layer (the decode glue "swiglu_rows" of the status page "MoE
 * Software Status & Known Limits", section "grouped-nf4-gemm", "Correctness
 * contracts"; the SwiGLU architectures of the experts4bit-qlora README, "Scope").
 *   gate = gate_up[r, j], up = gate_up[r, I + j]          (j < I)
 *   out[r, j] = bf16_rne( silu(gate) * up ),  silu(g) = g / (1 + exp(-g))
 * computed in fp32 as (g >= 0 ? g : g e) / (1 + e) * up with e = exp(-|g|) = 2^(-|g| log2 e)
 * from the hardware base-2 exponential and a fast division by 1 + e in [1, 2] (no overflow
 * for any finite g; about 2^-17 relative error before rounding).
 * |out - exact| <= (2^-8 + 2^-16) |exact| + 2^-118: one bf16 rounding plus the fp32 error;
 * the absolute term covers results that fall below the fp32 normal range.
 * gate_up device bf16 [R, 2I] (row-major, contiguous), 16-byte aligned
 * out     device bf16 [R, I], 16-byte aligned; may not overlap gate_up
 * R >= 0, I % 8 == 0. One kernel launch; R == 0 launches nothing and accepts NULL buffers.
 * Errors: INVALID_ARG (null/host pointer, R < 0, I < 1), UNSUPPORTED_SHAPE (I % 8),
 * MISALIGNED.
 */
gnf4_status gnf4_swiglu(const void* gate_up, int64_t R, int64_t I, void* out, void* stream);

/*
 * Top-k combine: the step after the down grouped GEMM, one output row per token
 * ("combine_rows" / "reduce_partials" of the status page, "Correctness contracts":
 * the partial reduction is bitwise the slot-order sum, and a token's row has the
 * same bits whether it is combined alone or inside a larger call).
 *   src(t, s) = row_of_slot ? row_of_slot[t*k + s] : t*k + s
 *   w(t, s)   = slot_weight ? slot_weight[t*k + s] : 1
 *   acc = +0; for s = 0 .. k-1 in order, if 0 <= src(t,s) < R:
 *       acc = fl32( acc + fl32( w(t,s) * y[src(t,s), n] ) )     (no fused multiply-add)
 *   out[t, n] = bf16_rne(acc)
 * With the down GEMM's epilogue applying the routing weight and scattering slot s of
 * token t to row t*k + s, both optional arrays are NULL (the slot-order sum of
 * already weighted rows); with expert-sorted down rows, row_of_slot is the row of
 * each (token, slot) and slot_weight its routing weight. The result is a function
 * of the token's own k slots only: bitwise reproducible and independent of T.
 * y           device bf16 [R, N], 16-byte aligned (may be NULL when R == 0: every slot dropped)
 * row_of_slot device int32 [T*k], or NULL; entries outside [0, R) are dropped slots
 * slot_weight device fp32 [T*k], or NULL
 * out         device bf16 [T, N], 16-byte aligned; may not overlap y
 * R, T >= 0, N % 8 == 0, 1 <= k < 2^31. One kernel launch; T == 0 launches nothing and
 * accepts NULL buffers.
 * Errors: INVALID_ARG, UNSUPPORTED_SHAPE (N % 8), MISALIGNED.
 */
gnf4_status gnf4_combine_topk(const void* y, int64_t R, int64_t N, const int32_t* row_of_slot,
                              const float* slot_weight, int64_t T, int64_t k, void* out,
                              void* stream);

/*
 * How many kernels one grouped GEMM call with R routed rows and these flags
 * launches (0 when R == 0; GNF4_CHECK adds one). Host-only, no CUDA call.
 */
int gnf4_grouped_gemm_launches(int64_t R, int flags);

#ifdef __cplusplus
}
#endif

#endif /* GNF4_H */
