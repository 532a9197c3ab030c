// Per-row FP8 (E4M3) quantization: one scale per row, s = amax/448, codes
// E4M3_rn_satfinite(x * (448/amax)). Per-token for BF16 activations ("each
// layer's input is rounded to FP8 per token", "Lernex/Metis-1.6-Logos-FP8",
// "What --fast-math does") and per-output-channel for FP32 weights ("one
// scale per output channel", same card, "What is in FP8").
//
// HBM-bound: 2 (or 4) bytes read + 1 byte written per element. A team of
// TEAM threads owns a row; each thread keeps NV 16-byte chunks of the row in
// registers, so the row is read from HBM exactly once: all loads are issued
// before the amax reduction (warp shuffles, then shared memory across the
// team's warps), then the codes are produced from registers.
#include "common.cuh"

namespace metis {
namespace {

constexpr int kQuantThreads = 256;

__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

template <typename T>
struct Elem;

template <>
struct Elem<__nv_bfloat16> {
    static constexpr int kPerChunk = 8;  // 16 bytes
    __device__ static void unpack(const uint4& c, float (&v)[8]) {
        const uint32_t w[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            v[2 * i] = bf16_lo(w[i]);
            v[2 * i + 1] = bf16_hi(w[i]);
        }
    }
};

template <>
struct Elem<float> {
    static constexpr int kPerChunk = 4;
    __device__ static void unpack(const uint4& c, float (&v)[4]) {
        v[0] = __uint_as_float(c.x);
        v[1] = __uint_as_float(c.y);
        v[2] = __uint_as_float(c.z);
        v[3] = __uint_as_float(c.w);
    }
};

// Register-resident path: K <= TEAM * NV * EPC. With SCATTER, row r's codes
// and scale go to rows dst[r * topk + j] (j < topk; negative entries skipped)
// instead of row r: the routed-expert path quantizes each token once and
// writes it straight into the expert-ordered rows it was routed to.
// With q == null only the scales are written: s[r] and inv_out[r] = 448/amax
// (the prologue of the fused-quantization GEMM).
template <typename T, int TEAM, int NV, bool SCATTER>
__global__ void __launch_bounds__(kQuantThreads)
quant_rows_kernel(const T* __restrict__ x, int64_t M, int K, int64_t ldx, uint8_t* __restrict__ q,
                  int64_t ldq, float* __restrict__ s, const int32_t* __restrict__ dst, int topk,
                  float* __restrict__ inv_out) {
    constexpr int EPC = Elem<T>::kPerChunk;
    constexpr int TEAMS = kQuantThreads / TEAM;
    constexpr int WARPS_PER_TEAM = TEAM / 32;
    __shared__ float red[kQuantThreads / 32];

    grid_dependency_wait();  // x may be the previous kernel's output (PDL launch)
    grid_launch_dependents();
    const int team = threadIdx.x / TEAM;
    const int tid = threadIdx.x % TEAM;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * TEAMS + team;
    const bool row_ok = row < M;
    const T* xr = x + row * ldx;

    uint4 buf[NV];
    float amax = 0.0f;
#pragma unroll
    for (int c = 0; c < NV; ++c) {
        const int e0 = (c * TEAM + tid) * EPC;
        if (row_ok && e0 < K) {
            buf[c] = ld_stream_v4(xr + e0);
        } else {
            buf[c] = make_uint4(0, 0, 0, 0);
        }
    }
#pragma unroll
    for (int c = 0; c < NV; ++c) {
        float v[EPC];
        Elem<T>::unpack(buf[c], v);
#pragma unroll
        for (int i = 0; i < EPC; ++i) amax = fmaxf(amax, fabsf(v[i]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if constexpr (WARPS_PER_TEAM > 1) {
        const int warp = threadIdx.x / 32;
        if ((threadIdx.x & 31) == 0) red[warp] = amax;
        __syncthreads();
        const int w0 = team * WARPS_PER_TEAM;
        amax = red[w0];
#pragma unroll
        for (int w = 1; w < WARPS_PER_TEAM; ++w) amax = fmaxf(amax, red[w0 + w]);
    }
    if (!row_ok) return;

    float sc, inv;
    row_scales(amax, &sc, &inv);
    if (q == nullptr) {
        if (tid == 0) {
            s[row] = sc;
            inv_out[row] = inv;
        }
        return;
    }
    // this thread's codes: 8 (BF16 input) or 4 (FP32 input) bytes per chunk
    uint2 out[NV];
#pragma unroll
    for (int c = 0; c < NV; ++c) {
        float v[EPC];
        Elem<T>::unpack(buf[c], v);
        if constexpr (EPC == 8) {
            out[c].x = f32x2_to_e4m3x2(__fmul_rn(v[0], inv), __fmul_rn(v[1], inv)) |
                       (f32x2_to_e4m3x2(__fmul_rn(v[2], inv), __fmul_rn(v[3], inv)) << 16);
            out[c].y = f32x2_to_e4m3x2(__fmul_rn(v[4], inv), __fmul_rn(v[5], inv)) |
                       (f32x2_to_e4m3x2(__fmul_rn(v[6], inv), __fmul_rn(v[7], inv)) << 16);
        } else {
            out[c].x = f32x2_to_e4m3x2(__fmul_rn(v[0], inv), __fmul_rn(v[1], inv)) |
                       (f32x2_to_e4m3x2(__fmul_rn(v[2], inv), __fmul_rn(v[3], inv)) << 16);
            out[c].y = 0;
        }
    }
    const int ndst = SCATTER ? topk : 1;
    for (int j = 0; j < ndst; ++j) {
        const int64_t r = SCATTER ? static_cast<int64_t>(dst[row * topk + j]) : row;
        if (r < 0) continue;
        if (tid == 0) s[r] = sc;
        uint8_t* qr = q + r * ldq;
#pragma unroll
        for (int c = 0; c < NV; ++c) {
            const int e0 = (c * TEAM + tid) * EPC;
            if (e0 >= K) continue;
            if constexpr (EPC == 8) *reinterpret_cast<uint2*>(qr + e0) = out[c];
            else *reinterpret_cast<uint32_t*>(qr + e0) = out[c].x;
        }
    }
}

// Long rows (K beyond the register-resident range): one CTA per row, two
// passes over the row (the second one mostly hits L2).
template <typename T>
__global__ void __launch_bounds__(kQuantThreads)
quant_rows_long_kernel(const T* __restrict__ x, int64_t M, int K, int64_t ldx,
                       uint8_t* __restrict__ q, int64_t ldq, float* __restrict__ s,
                       float* __restrict__ inv_out) {
    constexpr int EPC = Elem<T>::kPerChunk;
    __shared__ float red[kQuantThreads / 32];
    grid_dependency_wait();
    grid_launch_dependents();
    const int64_t row = blockIdx.x;
    if (row >= M) return;
    const T* xr = x + row * ldx;
    float amax = 0.0f;
    for (int e0 = threadIdx.x * EPC; e0 < K; e0 += kQuantThreads * EPC) {
        float v[EPC];
        Elem<T>::unpack(ld_stream_v4(xr + e0), v);
#pragma unroll
        for (int i = 0; i < EPC; ++i) amax = fmaxf(amax, fabsf(v[i]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x / 32] = amax;
    __syncthreads();
    amax = red[0];
#pragma unroll
    for (int w = 1; w < kQuantThreads / 32; ++w) amax = fmaxf(amax, red[w]);
    float sc, inv;
    row_scales(amax, &sc, &inv);
    if (threadIdx.x == 0) {
        s[row] = sc;
        if (q == nullptr) inv_out[row] = inv;
    }
    if (q == nullptr) return;
    uint8_t* qr = q + row * ldq;
    for (int e0 = threadIdx.x * EPC; e0 < K; e0 += kQuantThreads * EPC) {
        float v[EPC];
        const uint4 c = *reinterpret_cast<const uint4*>(xr + e0);
        Elem<T>::unpack(c, v);
        if constexpr (EPC == 8) {
            uint2 out;
            out.x = f32x2_to_e4m3x2(__fmul_rn(v[0], inv), __fmul_rn(v[1], inv)) |
                    (f32x2_to_e4m3x2(__fmul_rn(v[2], inv), __fmul_rn(v[3], inv)) << 16);
            out.y = f32x2_to_e4m3x2(__fmul_rn(v[4], inv), __fmul_rn(v[5], inv)) |
                    (f32x2_to_e4m3x2(__fmul_rn(v[6], inv), __fmul_rn(v[7], inv)) << 16);
            *reinterpret_cast<uint2*>(qr + e0) = out;
        } else {
            uint32_t out = f32x2_to_e4m3x2(__fmul_rn(v[0], inv), __fmul_rn(v[1], inv)) |
                           (f32x2_to_e4m3x2(__fmul_rn(v[2], inv), __fmul_rn(v[3], inv)) << 16);
            *reinterpret_cast<uint32_t*>(qr + e0) = out;
        }
    }
}

struct Dest {
    const int32_t* rows;  // null: row r -> row r; else row r -> rows[r * topk + j]
    int topk;
    float* inv;           // scales only (q null): 448/amax per row
};

template <typename T, int TEAM, int NV>
cudaError_t launch_fixed(const T* x, int64_t M, int K, int64_t ldx, uint8_t* q, int64_t ldq,
                         float* s, Dest d, cudaStream_t st) {
    constexpr int TEAMS = kQuantThreads / TEAM;
    const unsigned grid = static_cast<unsigned>((M + TEAMS - 1) / TEAMS);
    if (d.rows && q)
        return launch_pdl(quant_rows_kernel<T, TEAM, NV, true>, dim3(grid), dim3(kQuantThreads), 0, st, 1,
                          x, M, K, ldx, q, ldq, s, d.rows, d.topk, static_cast<float*>(nullptr));
    return launch_pdl(quant_rows_kernel<T, TEAM, NV, false>, dim3(grid), dim3(kQuantThreads), 0, st, 1,
                      x, M, K, ldx, q, ldq, s, static_cast<const int32_t*>(nullptr), 1, d.inv);
}

template <typename T, int TEAM>
cudaError_t launch_team(int nv, const T* x, int64_t M, int K, int64_t ldx, uint8_t* q,
                        int64_t ldq, float* s, Dest d, cudaStream_t st) {
    switch (nv) {
        case 1: return launch_fixed<T, TEAM, 1>(x, M, K, ldx, q, ldq, s, d, st);
        case 2: return launch_fixed<T, TEAM, 2>(x, M, K, ldx, q, ldq, s, d, st);
        case 3: return launch_fixed<T, TEAM, 3>(x, M, K, ldx, q, ldq, s, d, st);
        case 4: return launch_fixed<T, TEAM, 4>(x, M, K, ldx, q, ldq, s, d, st);
        case 5: return launch_fixed<T, TEAM, 5>(x, M, K, ldx, q, ldq, s, d, st);
        case 6: return launch_fixed<T, TEAM, 6>(x, M, K, ldx, q, ldq, s, d, st);
        case 7: return launch_fixed<T, TEAM, 7>(x, M, K, ldx, q, ldq, s, d, st);
        default: return launch_fixed<T, TEAM, 8>(x, M, K, ldx, q, ldq, s, d, st);
    }
}

}  // namespace

// Launches the per-row quantizer for T = bf16 or float (arguments already
// validated). Exposed to the other translation units of the library. With
// `dst_rows` non-null, row r is written to rows dst_rows[r * topk + j]
// (register-resident row lengths only: K <= 256 * 8 * chunk elements).
// With q == nullptr no codes are written: s receives the scales and inv_out
// 448/amax per row.
template <typename T>
int launch_quant_rows(const T* x, int64_t M, int64_t K, int64_t ldx, uint8_t* q, int64_t ldq,
                      float* s, cudaStream_t st, const int32_t* dst_rows, int topk, float* inv_out) {
    if (M == 0) return METIS_OK;
    if (q == nullptr && (inv_out == nullptr || dst_rows != nullptr))
        return fail(METIS_ERR_INVALID_ARG, "quantizer: scales-only needs inv_out and no row map");
    const Dest d{dst_rows, topk, inv_out};
    constexpr int EPC = Elem<T>::kPerChunk;
    const int64_t chunks = K / EPC;
    cudaError_t e;
    const int teams[4] = {32, 64, 128, 256};
    int pick = -1;
    for (int i = 0; i < 4; ++i)
        if ((chunks + teams[i] - 1) / teams[i] <= 8) { pick = i; break; }
    if (pick < 0 || M > (int64_t)0x7fffffff * (kQuantThreads / teams[pick])) {
        if (M > 0x7fffffff) return fail(METIS_ERR_UNSUPPORTED, "quantizer: M=%lld too large", (long long)M);
        if (d.rows) return fail(METIS_ERR_UNSUPPORTED, "quantizer: scattered rows need K <= %d",
                                256 * 8 * EPC);
        e = launch_pdl(quant_rows_long_kernel<T>, dim3(static_cast<unsigned>(M)), dim3(kQuantThreads), 0, st,
                       1, x, M, static_cast<int>(K), ldx, q, ldq, s, inv_out);
    } else {
        const int team = teams[pick];
        const int nv = static_cast<int>((chunks + team - 1) / team);
        switch (team) {
            case 32: e = launch_team<T, 32>(nv, x, M, (int)K, ldx, q, ldq, s, d, st); break;
            case 64: e = launch_team<T, 64>(nv, x, M, (int)K, ldx, q, ldq, s, d, st); break;
            case 128: e = launch_team<T, 128>(nv, x, M, (int)K, ldx, q, ldq, s, d, st); break;
            default: e = launch_team<T, 256>(nv, x, M, (int)K, ldx, q, ldq, s, d, st); break;
        }
    }
    return cuda_check(e, "quantizer launch");
}

template int launch_quant_rows<__nv_bfloat16>(const __nv_bfloat16*, int64_t, int64_t, int64_t,
                                              uint8_t*, int64_t, float*, cudaStream_t,
                                              const int32_t*, int, float*);
template int launch_quant_rows<float>(const float*, int64_t, int64_t, int64_t, uint8_t*, int64_t,
                                      float*, cudaStream_t, const int32_t*, int, float*);

}  // namespace metis

using namespace metis;

extern "C" int metis_quant_fp8_per_token(const void* x_bf16, int64_t M, int64_t K, int64_t ldx,
                                         uint8_t* xq, int64_t ldq, float* s_tok,
                                         metis_stream_t stream) {
    clear_error();
    if (M < 0 || K <= 0 || K % 8 != 0 || K > 0x7fffffff)
        return fail(METIS_ERR_INVALID_ARG, "quant_fp8_per_token: need M >= 0, K > 0, K %% 8 == 0 (M=%lld K=%lld)",
                    (long long)M, (long long)K);
    if (ldx < K || ldq < K || ldx % 8 != 0 || ldq % 8 != 0)
        return fail(METIS_ERR_INVALID_ARG,
                    "quant_fp8_per_token: need ldx >= K, ldq >= K, ldx %% 8 == 0, ldq %% 8 == 0 "
                    "(ldx=%lld ldq=%lld K=%lld)", (long long)ldx, (long long)ldq, (long long)K);
    if (M == 0) return METIS_OK;
    if (!x_bf16 || !xq || !s_tok)
        return fail(METIS_ERR_INVALID_ARG, "quant_fp8_per_token: null pointer");
    if (!aligned(x_bf16, 16) || !aligned(xq, 8) || !aligned(s_tok, 4))
        return fail(METIS_ERR_INVALID_ARG,
                    "quant_fp8_per_token: x must be 16-byte and xq 8-byte aligned");
    DeviceInfo di;
    int rc = current_device_info(&di);
    if (rc) return rc;
    return launch_quant_rows<__nv_bfloat16>(static_cast<const __nv_bfloat16*>(x_bf16), M, K, ldx,
                                            xq, ldq, s_tok, static_cast<cudaStream_t>(stream), nullptr, 1);
}

extern "C" int metis_quant_fp8_per_channel(const float* w, int64_t N, int64_t K, int64_t ldw,
                                           uint8_t* wq, int64_t ldq, float* s_w,
                                           metis_stream_t stream) {
    clear_error();
    if (N < 0 || K <= 0 || K % 4 != 0 || K > 0x7fffffff)
        return fail(METIS_ERR_INVALID_ARG, "quant_fp8_per_channel: need N >= 0, K > 0, K %% 4 == 0");
    if (ldw < K || ldq < K || ldw % 4 != 0 || ldq % 4 != 0)
        return fail(METIS_ERR_INVALID_ARG,
                    "quant_fp8_per_channel: need ldw >= K, ldq >= K, ldw %% 4 == 0, ldq %% 4 == 0");
    if (N == 0) return METIS_OK;
    if (!w || !wq || !s_w) return fail(METIS_ERR_INVALID_ARG, "quant_fp8_per_channel: null pointer");
    if (!aligned(w, 16) || !aligned(wq, 4) || !aligned(s_w, 4))
        return fail(METIS_ERR_INVALID_ARG,
                    "quant_fp8_per_channel: w must be 16-byte and wq 4-byte aligned");
    DeviceInfo di;
    int rc = current_device_info(&di);
    if (rc) return rc;
    return launch_quant_rows<float>(w, N, K, ldw, wq, ldq, s_w, static_cast<cudaStream_t>(stream),
                                    nullptr, 1);
}
