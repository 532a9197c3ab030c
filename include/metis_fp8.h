/*
 * metis_fp8.h — C ABI of the B200 (sm_100a) FP8 "fast-math" linear layer.
 *
 * What it computes, from the Metis-1.6 model cards:
 *  - "Lernex/Metis-1.6-Logos-FP8", section "What --fast-math does": every
 *    quantized layer's BF16 input is rounded to FP8 per token and multiplied
 *    with the FP8 weights on FP8 tensor cores (fast-math); by default the FP8
 *    weights are instead widened to 16 bits and the maths is done in 16-bit
 *    precision, so only the weights are rounded.
 *  - same card, section "What is in FP8": E4M3 weights with one scale per
 *    output channel, activations quantized per token at run time; the routed
 *    experts are among the FP8 matrices.
 *  - "Lernex/Metis-1.6-Praxis-NVFP4", section "What --fast-math does": the
 *    fast maths only changes steps that handle many tokens at once; one
 *    stream's decode always uses the default maths.
 *
 * The cards print no formula. The readings this library implements:
 *  - per-token scale  s[m] = amax_k |x[m,k]| / 448          (binary32 IEEE)
 *  - codes            q[m,k] = E4M3_rn_satfinite(x[m,k] * (448 / amax))
 *                     with 448/amax in binary32, clamped to FLT_MAX, and 0
 *                     when amax = 0 (then s = 0 and every code is +-0);
 *  - W8A8             y[m,n] = bf16_rn( s_tok[m] * s_w[n] * sum_k D(q)[m,k] D(w)[n,k] ),
 *                     FP32 accumulation on the tensor cores;
 *  - W8A16            y[m,n] = bf16_rn( s_w[n] * sum_k x[m,k] D(w)[n,k] ), FP32 accumulation;
 *  - routed experts   per routed slot (t, j) with expert e: h = W8A8(x[t], w_up[e]),
 *                     no activation, h re-quantized per row, o = W8A8(h, w_down[e]),
 *                     y[t] = bf16_rn( sum_j topk_w[t,j] * o[t,j] ) in FP32, j ascending.
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers, owned by the caller. The library
 *    never allocates, frees or synchronises; it only launches kernels,
 *    asynchronously, on `stream` (a cudaStream_t; NULL = legacy default stream).
 *  - BF16 tensors are 16-bit bit patterns (`const void*`), E4M3 tensors bytes.
 *  - Matrices are row-major. Unless a leading dimension is passed, rows are
 *    dense (leading dimension = number of columns).
 *  - Return value: METIS_OK (0) or a negative metis_status. Argument errors are
 *    detected on the host BEFORE anything is launched and leave all outputs
 *    untouched; metis_last_error() then returns a message for this thread.
 *  - Device-side watchdog: every wait inside a kernel is bounded. A wait that
 *    runs out sets a sticky device error word and the kernel returns early
 *    with incomplete output; metis_check_device_status() reports it.
 *  - Results are bitwise reproducible run to run (no floating-point atomics).
 */
#ifndef METIS_FP8_H
#define METIS_FP8_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define METIS_API __attribute__((visibility("default")))
#else
#define METIS_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    METIS_OK = 0,
    METIS_ERR_INVALID_ARG = -1, /* bad pointer, size, alignment or layout */
    METIS_ERR_UNSUPPORTED = -2, /* valid request the library does not implement */
    METIS_ERR_CUDA = -3,        /* a CUDA runtime/driver call failed */
    METIS_ERR_TIMEOUT = -4      /* a device-side bounded wait ran out */
} metis_status;

/* Opaque CUDA stream (cudaStream_t). */
typedef void* metis_stream_t;

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
METIS_API int metis_version(void);

/* Message describing the last error returned on the calling thread ("" if none).
 * The pointer stays valid until the next library call on this thread. */
METIS_API const char* metis_last_error(void);

/* Self-test of the device watchdog; the pages have no counterpart. One
 * thread waits on an mbarrier that nothing ever completes, bounded by
 * `limit_ns` (1 .. 1e9 ns); when the limit runs out the kernel sets the
 * sticky device error word and returns, exactly as a stalled wait in any
 * other kernel would. metis_check_device_status() then reports
 * METIS_ERR_TIMEOUT and the CUDA context stays usable. The kernel touches no
 * global memory other than the status word, and no tensor memory or TMA. */
METIS_API int metis_watchdog_selftest(uint64_t limit_ns, metis_stream_t stream);

/* Reads (and, if `clear` != 0, clears) the sticky device error word on the
 * current device, synchronising `stream` first. Returns METIS_OK,
 * METIS_ERR_TIMEOUT if a kernel's bounded wait ran out, METIS_ERR_INVALID_ARG
 * if a routed-expert layer met a routing id outside [0, E) (that slot was
 * dropped), or METIS_ERR_CUDA. This is the one entry point that synchronises. */
METIS_API int metis_check_device_status(metis_stream_t stream, int clear);

/* Sets the per-wait limit of the device watchdog in nanoseconds (default
 * 2e9 = 2 s; 0 restores the default). Affects kernels launched afterwards. */
METIS_API int metis_set_watchdog_ns(uint64_t ns);

/* Per-token FP8 quantization of BF16 activations.
 * Source: "Lernex/Metis-1.6-Logos-FP8", "What --fast-math does" (each layer's
 * input rounded to FP8 per token) and "What is in FP8" (activations quantized
 * per token at run time).
 *   x_bf16 [M, ldx] BF16 (K valid columns), xq [M, ldq] E4M3 out, s_tok [M] FP32 out.
 *   Requires M >= 0, K > 0, K % 8 == 0, ldx >= K, ldq >= K, ldx % 8 == 0,
 *   ldq % 8 == 0, x_bf16 16-byte aligned, xq 8-byte aligned, s_tok 4-byte
 *   aligned. (Codes that feed metis_fp8_gemm need K % 16 == 0 and dense rows.)
 *   M == 0 launches nothing. */
METIS_API int metis_quant_fp8_per_token(const void* x_bf16, int64_t M, int64_t K, int64_t ldx,
                              uint8_t* xq, int64_t ldq, float* s_tok, metis_stream_t stream);

/* Per-output-channel FP8 quantization of FP32 weights, the same rule as the
 * per-token quantizer applied to each weight row (one scale per output
 * channel, "Lernex/Metis-1.6-Logos-FP8", "What is in FP8"). Prepares the
 * weight operand of the GEMMs.
 *   w [N, ldw] FP32, wq [N, ldq] E4M3 out, s_w [N] FP32 out.
 *   Requires K % 4 == 0, ldw % 4 == 0, ldq % 4 == 0, ldw >= K, ldq >= K,
 *   w 16-byte aligned, wq 4-byte aligned. */
METIS_API int metis_quant_fp8_per_channel(const float* w, int64_t N, int64_t K, int64_t ldw,
                                uint8_t* wq, int64_t ldq, float* s_w, metis_stream_t stream);

/* Fast-math W8A8 GEMM with the per-token x per-channel scale epilogue on
 * tcgen05 tensor cores ("Lernex/Metis-1.6-Logos-FP8", "What --fast-math does").
 *   a_kind = METIS_A_E4M3: `a` is E4M3 [M, K] (dense rows), s_tok [M] is an input.
 *   a_kind = METIS_A_BF16: `a` is BF16 [M, K] (dense rows); the per-token
 *            quantization is fused into the GEMM (an amax pre-pass writes
 *            s_tok [M] as an OUTPUT, identical to metis_quant_fp8_per_token,
 *            and the E4M3 codes are produced in shared memory, never in HBM;
 *            the output is bit-identical to quantizer + E4M3 GEMM). Each A
 *            tile is converted once per 256-column output tile, so for wide
 *            N this variant is slower than the two separate calls, which is
 *            what metis_linear uses. Needs `workspace` of
 *            metis_workspace_size(METIS_OP_FP8_GEMM_FUSED, M, N, K, 0, 0)
 *            bytes (16-byte aligned).
 *   wq [N, K] E4M3 (one row per output channel), s_w [N] FP32, y [M, N] BF16 out.
 *   Requires K % 16 == 0, N % 8 == 0, K >= 16, N >= 8, M >= 0; a, wq, y
 *   16-byte aligned. */
#define METIS_A_E4M3 0
#define METIS_A_BF16 1
METIS_API int metis_fp8_gemm(const void* a, int a_kind, float* s_tok, const uint8_t* wq,
                   const float* s_w, void* y_bf16, int64_t M, int64_t N, int64_t K,
                   void* workspace, size_t ws_bytes, metis_stream_t stream);

/* Default-maths weight-only GEMM: the E4M3 weights are widened exactly to
 * 16 bits as they are multiplied, products accumulate in FP32 and the
 * per-channel scale is applied to the sum ("Lernex/Metis-1.6-Logos-FP8",
 * "What --fast-math does": the default maths, which single-stream decode
 * always uses and prefill uses without fast-math).
 *   x [M, K] BF16, wq [N, K] E4M3, s_w [N] FP32, y [M, N] BF16 out.
 *   M <= 8 (decode): an HBM-bound weight stream with mma.sync on FP16
 *   operands; requires K % 16 == 0, 16 <= K <= 12288, N >= 1; x, wq
 *   16-byte aligned.
 *   M > 8: tcgen05 BF16 maths with the widened weights in tensor memory;
 *   requires K % 16 == 0, K >= 16, N % 8 == 0, N >= 8; x, wq, y 16-byte
 *   aligned. */
METIS_API int metis_w8a16_gemm(const void* x_bf16, const uint8_t* wq, const float* s_w, void* y_bf16,
                     int64_t M, int64_t N, int64_t K, metis_stream_t stream);

/* The same default maths for many tokens through a workspace: the weights are
 * first widened exactly to BF16 [N, K] in `workspace` by an HBM-bound pass
 * (E4M3 NaN codes widen to NaN), then multiplied by the BF16 CTA-pair
 * tensor-core GEMM with s_w applied to the FP32 sum in its epilogue:
 *   y[m, n] = bf16_rn( fl32( s_w[n] * sum_k x[m, k] * D(wq[n, k]) ) ).
 * Faster than metis_w8a16_gemm's in-kernel widening once the token count
 * amortises the pass (metis_linear uses it for M >= 2048).
 *   workspace: metis_workspace_size(METIS_OP_W8A16_WIDENED, M, N, K, 0, 0)
 *   bytes, 16-byte aligned; overwritten.
 *   Requires K % 16 == 0, K >= 16, N % 8 == 0, N >= 8, M >= 0; x, wq, y
 *   16-byte aligned, s_w 4-byte aligned. */
METIS_API int metis_w8a16_gemm_widened(const void* x_bf16, const uint8_t* wq, const float* s_w,
                                       void* y_bf16, int64_t M, int64_t N, int64_t K, void* workspace,
                                       size_t ws_bytes, metis_stream_t stream);

/* Router top-k feeding the routed-expert layer. The cards keep "the routers
 * and their balance bias" in FP32 and route each token to a few experts
 * ("Lernex/Metis-1.6-Logos-FP8", "What is in FP8"; four per token in
 * "Lernex/Metis-1.6-Praxis-Base"); they print no formula. Reading: choice j
 * of token t is the expert with the j-th largest binary32 score
 * logits[t, e] + bias[e] (ties to the lower expert index); the weights are a
 * softmax over the chosen experts' own logits (the bias decides the choice
 * only), computed in FP32.
 *   logits [T, E] FP32, bias [E] FP32 or NULL; topk_ids [T, topk] int32 out
 *   (descending score), topk_w [T, topk] FP32 out.
 *   Requires 1 <= E <= 1024, 1 <= topk <= min(E, 32); 4-byte aligned
 *   pointers. NaN scores are never preferred to other scores. */
METIS_API int metis_moe_route_topk(const float* logits, const float* bias, int64_t T, int64_t E,
                                   int64_t topk, int32_t* topk_ids, float* topk_w,
                                   metis_stream_t stream);

/* Routed-expert W8A8 layer ("Lernex/Metis-1.6-Logos-FP8", "What is in FP8":
 * the routed experts are FP8 with per-channel scales and per-token
 * activations). Steps, all on the device, no host synchronisation:
 * routing histogram -> exclusive prefix sum -> stable permutation of the
 * slots (t, j) by expert -> per-token quantization of x (once per token,
 * written into the expert-contiguous rows of its slots) -> grouped up-projection (W8A8) ->
 * per-row re-quantization -> grouped down-projection (W8A8) -> weighted
 * un-permute y[t] = sum_j topk_w[t,j] o[t,j] (FP32, j ascending) -> BF16.
 *   x [T, H] BF16, topk_ids [T, topk] int32 in [0, E), topk_w [T, topk] FP32,
 *   w_up [E, I, H] E4M3, s_up [E, I], w_down [E, H, I] E4M3, s_down [E, H],
 *   y [T, H] BF16 out, or NULL: the layer then stops after the down-projection
 *   and leaves o and the routing in the workspace for
 *   metis_moe_shared_fused_combine (no combine kernel runs).
 *   act must be METIS_ACT_NONE (the cards do not state the experts' activation).
 *   Requires H % 16 == 0, I % 16 == 0, 16 <= H <= 16384, I >= 16, 1 <= topk <= E <= 1024.
 *   Ids outside [0, E) are checked on the device (the ids stay on the GPU, so
 *   the host cannot see them): such a slot is dropped from the layer (its
 *   SLOT_TO_ROW entry is -1 and it adds nothing to y[t]; the token's other
 *   slots are unaffected) and the sticky device error word records it, so the
 *   next metis_check_device_status() returns METIS_ERR_INVALID_ARG.
 *   Needs `workspace` of metis_workspace_size(METIS_OP_MOE, T, I, H, topk, E)
 *   bytes (256-byte aligned); its regions are given by metis_moe_workspace_offset. */
#define METIS_ACT_NONE 0
METIS_API int metis_moe_fp8_grouped_gemm(const void* x_bf16, const int32_t* topk_ids, const float* topk_w,
                               int64_t T, int64_t topk, int64_t E, int64_t H, int64_t I,
                               const uint8_t* w_up, const float* s_up,
                               const uint8_t* w_down, const float* s_down, int act,
                               void* y_bf16, void* workspace, size_t ws_bytes,
                               metis_stream_t stream);

/* Allocation-free form of metis_moe_fp8_grouped_gemm (the model cards have
 * no counterpart: this entry point exists for callers, not for the method).
 * Meant for callers that cannot allocate device memory themselves, such as a
 * host program running inside an engine that planned all GPU memory up front,
 * or a plugin given device pointers but no allocator. It takes the same inputs
 * and output but no workspace: its scratch is a 16 MiB array built into the
 * library, which each GPU that loads the library keeps until the process exits.
 *   - Problems whose metis_workspace_size(METIS_OP_MOE, ...) exceeds 16 MiB are
 *     rejected with METIS_ERR_INVALID_ARG before anything is launched (about
 *     200 tokens at top-8 with H = 2048, I = 1024).
 *   - y must not be NULL: the routed outputs would otherwise stay in the
 *     built-in array, which the caller cannot address (METIS_ERR_INVALID_ARG).
 *   - The first call on each device (and the first after a cudaDeviceReset,
 *     which moves the array) looks up the array's device address; make that
 *     first call before any stream capture.
 *   - All calls on a device share the one array and it keeps the previous
 *     call's contents (nothing in it needs to start at zero). Calls that may
 *     overlap on the GPU, e.g. on two streams, race on it: serialise them. */
METIS_API int metis_moe_fp8_grouped_gemm_noalloc(const void* x_bf16, const int32_t* topk_ids,
                                                 const float* topk_w, int64_t T, int64_t topk,
                                                 int64_t E, int64_t H, int64_t I,
                                                 const uint8_t* w_up, const float* s_up,
                                                 const uint8_t* w_down, const float* s_down,
                                                 int act, void* y_bf16, metis_stream_t stream);

/* BF16 GEMM on the tensor cores (tcgen05.mma kind::f16, FP32 accumulation):
 *   y[m, n] = bf16_rn( sum_k x[m, k] w[n, k] ).
 * The shared expert's projections use it ("Lernex/Metis-1.6-Praxis" card,
 * "Architecture": one shared expert in every layer; the FP8 cards keep it
 * in BF16). x [M, K], w [N, K], y [M, N] BF16, 16-byte aligned; N and K
 * multiples of 8. */
METIS_API int metis_bf16_gemm(const void* x_bf16, const void* w_bf16, void* y_bf16, int64_t M,
                              int64_t N, int64_t K, metis_stream_t stream);

/* The shared expert joined to the routed combine: its two BF16 projections
 * run as tensor-core GEMMs, and one combine pass adds its output s to the
 * routed weighted sum (reading o, s and the routing once, writing y once).
 * Reading of the cards (they print no formula): the shared expert runs on
 * every token with weight 1, with the two projections of a routed expert (no
 * activation), and the layer output adds its BF16 output s to the routed
 * weighted sum before the one final rounding:
 *   h_s[t] = bf16( x[t] W_sup^T )                      W_sup [I_s, H] BF16
 *   s[t]   = bf16( h_s[t] W_sdn^T )                    W_sdn [H, I_s] BF16
 *   y[t]   = bf16( s[t] + sum_j topk_w[t, j] o[slot_to_row[t*topk + j]] )
 *            (FP32, j ascending; slots with slot_to_row < 0 skipped).
 *   o_routed, slot_to_row: the routed layer's O and SLOT_TO_ROW workspace
 *   regions after metis_moe_fp8_grouped_gemm or metis_moe_nvfp4_grouped_gemm
 *   ran with y = NULL (o rows of H BF16 values).
 *   Requires H and I_s multiples of 16 (H <= 16384), 1 <= topk <= 8; needs
 *   `workspace` of metis_workspace_size(METIS_OP_SHARED, T, I_s, H, topk, 0)
 *   bytes (256-byte aligned) for h_s [T, I_s] and s [T, H]. */
METIS_API int metis_moe_shared_fused_combine(const void* x_bf16, int64_t T, int64_t H, int64_t I_s,
                                             const void* w_sup_bf16, const void* w_sdn_bf16,
                                             const void* o_routed_bf16, const int32_t* slot_to_row,
                                             const float* topk_w, int64_t topk, void* y_bf16,
                                             void* workspace, size_t ws_bytes,
                                             metis_stream_t stream);

/* Workspace sizes in bytes.
 *   METIS_OP_FP8_GEMM_FUSED: (M, N, K) of metis_fp8_gemm with a_kind = METIS_A_BF16.
 *   METIS_OP_MOE:            (T, I, H, topk, E) of metis_moe_fp8_grouped_gemm.
 *   METIS_OP_LINEAR:         (M, N, K) of metis_linear with fast_math != 0.
 *   METIS_OP_W8A16_WIDENED:  (M, N, K) of metis_w8a16_gemm_widened, and of
 *                            metis_linear's default maths for many tokens.
 *   Other ops need none (0). Returns 0 for invalid arguments. */
#define METIS_OP_FP8_GEMM 0
#define METIS_OP_FP8_GEMM_FUSED 1
#define METIS_OP_W8A16 2
#define METIS_OP_MOE 3
#define METIS_OP_LINEAR 4
#define METIS_OP_SHARED 6       /* metis_moe_shared_fused_combine: (T, I_s, H, topk, 0) */
#define METIS_OP_W8A16_WIDENED 7 /* metis_w8a16_gemm_widened: 2 * N * K bytes */
METIS_API size_t metis_workspace_size(int op, int64_t M_or_T, int64_t N_or_I, int64_t K_or_H,
                            int64_t topk, int64_t E);

/* Byte offset of one region inside the routed-expert workspace, so callers
 * and tests can read the intermediates (S = T * topk slots):
 *   METIS_MOE_WS_COUNTS      int32 [E]      slots per expert
 *   METIS_MOE_WS_OFFSETS     int32 [E + 1]  exclusive prefix sum of COUNTS
 *   METIS_MOE_WS_SLOT_TO_ROW int32 [S]      row of slot s = t*topk + j in expert order
 *   METIS_MOE_WS_ROW_TO_SLOT int32 [S]      inverse permutation
 *   METIS_MOE_WS_AQ          E4M3  [S, H]   per-token codes of x, one row per slot, expert order
 *   METIS_MOE_WS_SA          FP32  [S]      their per-token scales
 *   METIS_MOE_WS_H           BF16  [S, I]   up-projection output, expert order
 *   METIS_MOE_WS_HQ          E4M3  [S, I]   its per-row codes
 *   METIS_MOE_WS_SH          FP32  [S]      their scales
 *   METIS_MOE_WS_O           BF16  [S, H]   down-projection output, expert order
 * Returns -1 for an unknown region or invalid sizes. */
#define METIS_MOE_WS_COUNTS 0
#define METIS_MOE_WS_OFFSETS 1
#define METIS_MOE_WS_SLOT_TO_ROW 2
#define METIS_MOE_WS_ROW_TO_SLOT 3
#define METIS_MOE_WS_AQ 4
#define METIS_MOE_WS_SA 5
#define METIS_MOE_WS_H 6
#define METIS_MOE_WS_HQ 7
#define METIS_MOE_WS_SH 8
#define METIS_MOE_WS_O 9
METIS_API int64_t metis_moe_workspace_offset(int region, int64_t T, int64_t topk, int64_t E,
                                   int64_t H, int64_t I);

/* The dispatch rule of the cards ("Lernex/Metis-1.6-Praxis-NVFP4", "What
 * --fast-math does"): M <= 8 tokens always take the default maths
 * (metis_w8a16_gemm); more tokens take the fast-math W8A8 path when
 * fast_math != 0 (metis_quant_fp8_per_token into the workspace, then
 * metis_fp8_gemm with a_kind = METIS_A_E4M3), and the default maths
 * otherwise.
 * s_tok [M] receives the per-token scales on the fast-math path; `workspace`
 * holds the E4M3 codes: metis_workspace_size(METIS_OP_LINEAR, M, N, K, 0, 0)
 * bytes, 16-byte aligned (0 for M <= 8).
 * Default maths with M >= 2048: when `workspace` (16-byte aligned) holds
 * metis_workspace_size(METIS_OP_W8A16_WIDENED, M, N, K, 0, 0) bytes,
 * metis_w8a16_gemm_widened runs; otherwise metis_w8a16_gemm (in-kernel
 * widening). Both compute the same products with FP32 accumulation. */
METIS_API int metis_linear(const void* x_bf16, const uint8_t* wq, const float* s_w, void* y_bf16,
                 int64_t M, int64_t N, int64_t K, int fast_math, float* s_tok,
                 void* workspace, size_t ws_bytes, metis_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* METIS_FP8_H */
