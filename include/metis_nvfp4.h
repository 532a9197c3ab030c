/*
 * metis_nvfp4.h — C ABI of the NVFP4 routed experts under fast-math (B200, sm_100a).
 *
 * What it computes, from the Metis-1.6 model cards:
 *  - "Lernex/Metis-1.6-Praxis-NVFP4", section "What is in NVFP4": the routed
 *    experts hold 4-bit E2M1 values with one FP8 (E4M3) scale per 16 inputs
 *    and one FP32 scale per expert.
 *  - same card, section "What --fast-math does" (and the note under its
 *    benchmark table): on Blackwell the 4-bit experts multiply in FP4, their
 *    inputs rounded to FP4 as well.
 *
 * The card prints no rounding rule. The readings this library implements, for
 * a row x[0..K) (a token, or an output channel of an expert) whose global
 * scale is shared by a set of rows (the token alone, or the whole expert):
 *  - global scale   g = amax / 2688, amax over the set (2688 = 6 * 448), and
 *                   inv_g = 2688 / amax clamped to FLT_MAX, 0 when amax = 0;
 *  - block scale    per 16 elements with block amax b:
 *                   sb = E4M3_rn_satfinite((b * inv_g) / 6)   (a non-negative code)
 *  - codes          q[k] = E2M1_rn_satfinite((x[k] * inv_g) * (1 / D(sb))),
 *                   +-0 when D(sb) = 0;
 *  - value          D2(q[k]) * D(sb) * g.
 *   Every step is one binary32 operation, rounded to nearest-even. E2M1 holds
 *   +-{0, 0.5, 1, 1.5, 2, 3, 4, 6} (sign bit 3, exponent bits 2..1 with bias 1,
 *   mantissa bit 0) and saturates to +-6.
 *  - GEMM           y[m,n] = bf16_rn( g_a[m] * g_b * sum_k V_a[m,k] V_b[n,k] ),
 *                   V = D2(q) * D(sb), FP32 accumulation on the tensor cores
 *                   (block-scaled tcgen05.mma kind::mxf4nvf4, 16-element blocks).
 *  - routed experts as in metis_moe_fp8_grouped_gemm, with every projection in
 *                   NVFP4: x quantized per token, h quantized per routed row.
 *
 * Storage:
 *  - codes          two per byte, row-major [R, K/2]: element 2i in the low
 *                   nibble of byte i, element 2i + 1 in the high nibble.
 *  - block scales   E4M3 bytes, either row-major [R, K/16] (METIS_SF_ROWMAJOR)
 *                   or tiled for the tensor cores (METIS_SF_TILED):
 *                   [ceil(R/128)][K/64][512] where the 512-byte atom of rows
 *                   128 a .. 128 a + 127 and elements 64 c .. 64 c + 63 holds the
 *                   scale of row 128 a + r, block 4 c + j at byte
 *                   16 (r % 32) + 4 (r / 32) + j. Rows past R read as zero.
 *  - global scales  FP32.
 *
 * Conventions are those of metis_fp8.h: device pointers owned by the caller,
 * nothing allocated or synchronised, asynchronous on `stream`, METIS_OK or a
 * negative metis_status with argument errors found before any launch,
 * bounded device waits, bitwise reproducible results.
 */
#ifndef METIS_NVFP4_H
#define METIS_NVFP4_H

#include "metis_fp8.h"

#ifdef __cplusplus
extern "C" {
#endif

#define METIS_A_F32 2          /* x_kind: FP32 input rows */
#define METIS_SF_ROWMAJOR 0    /* block scales [R, K/16] */
#define METIS_SF_TILED 1       /* block scales in the tensor-core atom layout */
#define METIS_OP_MOE_NVFP4 5   /* metis_workspace_size: the NVFP4 routed-expert layer */

/*
 * NVFP4 quantization of R rows of K elements (the reading above).
 *   x              [R, ldx] BF16 bit patterns (x_kind METIS_A_BF16) or FP32
 *                  (METIS_A_F32); 16-byte aligned, ldx * element size a
 *                  multiple of 16.
 *   rows_per_scale 1: one global scale per row (activations, per token); or
 *                  a divisor of R: rows [i*rps, (i+1)*rps) share one (an
 *                  expert's weights: rps = N for [E*N, K] weights).
 *   q              [R, K/2] packed codes (16-byte aligned).
 *   sf             block scales in `sf_layout` (METIS_SF_TILED needs
 *                  ceil(R/128) * 128 * K/16 bytes; pad rows are written as 0).
 *   g              [R / rows_per_scale] FP32 global scales.
 * K: a multiple of 64, 64 <= K <= 65536. R >= 0 (0: nothing launched).
 * With rows_per_scale > 1 three kernels run (amax, codes, scales).
 */
METIS_API int metis_quant_nvfp4(const void* x, int x_kind, int64_t R, int64_t K, int64_t ldx,
                                int64_t rows_per_scale, uint8_t* q, uint8_t* sf, int sf_layout,
                                float* g, metis_stream_t stream);

/*
 * Re-lays row-major block scales [R, K/16] into the tiled layout
 * [ceil(R/128)][K/64][512] (pad rows zero). Pure byte permutation.
 * K a multiple of 64; pointers 4-byte aligned; the buffers must not overlap.
 */
METIS_API int metis_nvfp4_scales_to_tiled(const uint8_t* sf, int64_t R, int64_t K,
                                          uint8_t* sf_tiled, metis_stream_t stream);

/*
 * y [M, N] = NVFP4 GEMM (the reading above) on the tensor cores.
 *   qa     [ceil(M/128) * 128, K/2] packed codes of A: the rows past M are
 *          read (their results are discarded), so the buffer must hold them.
 *   sfa    tiled block scales of A (ceil(M/128) atoms of rows).
 *   ga     [M] FP32 global scales of A's rows.
 *   qb     [N, K/2] packed codes of B (an expert's weights, output channel n
 *          = row n); sfb tiled block scales of B; gb a DEVICE pointer to B's
 *          one FP32 global scale.
 *   y      [M, N] BF16, row-major.
 * K a multiple of 64 (K >= 64); N a multiple of 128; M >= 0. Codes, tiled
 * scales and y 16-byte aligned.
 */
METIS_API int metis_nvfp4_gemm(const uint8_t* qa, const uint8_t* sfa, const float* ga,
                               const uint8_t* qb, const uint8_t* sfb, const float* gb, void* y,
                               int64_t M, int64_t N, int64_t K, metis_stream_t stream);

/*
 * Routed-expert layer with NVFP4 experts under fast-math: the steps of
 * metis_moe_fp8_grouped_gemm (routing, per-token quantization gathered into
 * expert order, grouped up-projection, per-row re-quantization, grouped
 * down-projection, weighted combine), every projection in NVFP4. Each
 * expert's rows start on a 128-row boundary of the workspace.
 *   x       [T, H] BF16; topk_ids [T, topk] int32; topk_w [T, topk] FP32.
 *   w_up    [E, I, H/2] packed codes; sf_up tiled scales of the [E*I, H]
 *           matrix; g_up [E] FP32. w_down [E, H, I/2]; sf_down tiled scales of
 *           [E*H, I]; g_down [E].
 *   act     METIS_ACT_NONE.
 *   y       [T, H] BF16, or NULL: stop after the down-projection, leaving o
 *           and the routing for metis_moe_shared_fused_combine.
 *   workspace  metis_workspace_size(METIS_OP_MOE_NVFP4, T, I, H, topk, E)
 *           bytes, 256-byte aligned; regions by metis_moe_nvfp4_workspace_offset.
 * H and I multiples of 128, 128 <= H <= 16384, 128 <= I <= 65536;
 * 1 <= topk <= E <= 1024.
 */
METIS_API int metis_moe_nvfp4_grouped_gemm(const void* x_bf16, const int32_t* topk_ids,
                                           const float* topk_w, int64_t T, int64_t topk,
                                           int64_t E, int64_t H, int64_t I, const uint8_t* w_up,
                                           const uint8_t* sf_up, const float* g_up,
                                           const uint8_t* w_down, const uint8_t* sf_down,
                                           const float* g_down, int act, void* y_bf16,
                                           void* workspace, size_t ws_bytes,
                                           metis_stream_t stream);

/* Workspace regions of metis_moe_nvfp4_grouped_gemm. Rows are padded: Sp =
 * T*topk + 127*E rounded up to 128 rows; expert e's rows start at
 * OFFSETS[e] (a multiple of 128) and its first COUNTS[e] rows are real. */
#define METIS_MOE4_WS_COUNTS 0      /* int32 [E]        real rows per expert */
#define METIS_MOE4_WS_OFFSETS 1     /* int32 [E + 1]    padded first rows */
#define METIS_MOE4_WS_SLOT_TO_ROW 2 /* int32 [T*topk]   row of slot t*topk + j */
#define METIS_MOE4_WS_ROW_TO_SLOT 3 /* int32 [Sp]       slot of a real row */
#define METIS_MOE4_WS_AQ 4          /* uint8 [Sp, H/2]  codes of x per row */
#define METIS_MOE4_WS_SFA 5         /* uint8 tiled scales of x (Sp rows, K = H) */
#define METIS_MOE4_WS_GA 6          /* float [Sp]       global scales of x */
#define METIS_MOE4_WS_H 7           /* bf16  [Sp, I]    up-projection */
#define METIS_MOE4_WS_HQ 8          /* uint8 [Sp, I/2]  codes of h */
#define METIS_MOE4_WS_SFH 9         /* uint8 tiled scales of h (K = I) */
#define METIS_MOE4_WS_GH 10         /* float [Sp]       global scales of h */
#define METIS_MOE4_WS_O 11          /* bf16  [Sp, H]    down-projection */

/* Byte offset of a region in the workspace, or -1 for a bad argument. */
METIS_API int64_t metis_moe_nvfp4_workspace_offset(int region, int64_t T, int64_t topk, int64_t E,
                                                   int64_t H, int64_t I);

#ifdef __cplusplus
}
#endif

#endif /* METIS_NVFP4_H */
