// Default-maths weight-only GEMM for decode (M <= 8 tokens):
//   y[m, n] = bf16_rn( s_w[n] * sum_k x[m, k] * D(w[n, k]) ),  FP32 accumulation.
// "Lernex/Metis-1.6-Logos-FP8", "What --fast-math does": by default the FP8
// weights are expanded to 16 bits as they are multiplied, so the weights are
// the only thing rounded; one stream's decode always takes this path because
// its speed is set by how fast the weights are read.
//
// HBM-bound: N*K weight bytes dominate. Design:
//  * one persistent CTA (512 threads) per SM owns a contiguous range of
//    16-row weight tiles; inside a tile, 16 warps split K in 64-byte chunks,
//    so each weight byte is read from HBM exactly once, with coalesced 16-byte
//    streaming loads and 8 chunks in flight per thread;
//  * the 16 rows x 16 k of a chunk step are the A operand of an
//    mma.sync.m16n8k16 (FP16 in, FP32 accumulate); the <= 8 tokens are the
//    B operand (n = 8), staged once per CTA in shared memory;
//  * E4M3 -> FP16 is exact (every E4M3 value is an FP16 normal);
//  * x is staged as FP16 after an exact per-token power-of-two shift that
//    puts the token's amax in [2^14, 2^15): every element within 2^29 of the
//    token's amax keeps its BF16 value exactly, so the products are those of
//    the BF16 maths; the shift is undone exactly in the epilogue;
//  * partial sums of the 16 warps meet in shared memory and are added in a
//    fixed order (deterministic), then scaled by s_w[n] and rounded to BF16.
#include "common.cuh"

namespace metis {
namespace w8a16 {

constexpr int THREADS = 512;
constexpr int WARPS = THREADS / 32;
constexpr int DEPTH = 8;          // chunks in flight per thread
constexpr int MAX_K = 12288;
constexpr int XROW_PAD = 8;       // bytes; row pitch = 2K + 8 (bank-conflict free)

// Weight widening variants (selected once, see metis_internal_w8a16_variant).
enum Conv { kCvt = 0, kAluMul = 1, kAluFold = 2 };
int g_variant = kAluFold;

__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t cvt_e4m3x2_f16x2(uint32_t two_bytes) {
    uint32_t r;
    const uint16_t in = static_cast<uint16_t>(two_bytes);
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(in));
    return r;
}

// Places bytes (e0, e2) resp. (e1, e3) of q into FP16 bit positions. Each
// result half equals the E4M3 value times 2^-8 exactly (subnormals included):
// FP16 has bias 15 where E4M3 has bias 7, and both subnormal ranges scale alike.
__device__ __forceinline__ uint32_t place_even(uint32_t q) {
    return ((q << 8) & 0x80008000u) | ((q << 7) & 0x3F803F80u);
}
__device__ __forceinline__ uint32_t place_odd(uint32_t q) {
    return (q & 0x80008000u) | ((q >> 1) & 0x3F803F80u);
}
__device__ __forceinline__ uint32_t hmul2_256(uint32_t h2) {
    uint32_t r;
    const uint32_t k256 = 0x5C005C00u;  // (256.0, 256.0) in FP16
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(h2), "r"(k256));
    return r;
}

__device__ __forceinline__ void mma_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, "
        "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// One 64-byte chunk step of one warp: 4 MMAs over 16 rows x 64 k.
template <int CONV>
__device__ __forceinline__ void chunk_mma(float (&acc)[4], const uint4& ra, const uint4& rb,
                                          const uint8_t* xs_thread) {
    const uint32_t wa[4] = {ra.x, ra.y, ra.z, ra.w};
    const uint32_t wb[4] = {rb.x, rb.y, rb.z, rb.w};
#pragma unroll
    for (int s = 0; s < 4; ++s) {
        uint32_t a0, a1, a2, a3;
        if constexpr (CONV == kCvt) {
            a0 = cvt_e4m3x2_f16x2(wa[s]);
            a2 = cvt_e4m3x2_f16x2(wa[s] >> 16);
            a1 = cvt_e4m3x2_f16x2(wb[s]);
            a3 = cvt_e4m3x2_f16x2(wb[s] >> 16);
        } else if constexpr (CONV == kAluMul) {
            a0 = hmul2_256(place_even(wa[s]));
            a2 = hmul2_256(place_odd(wa[s]));
            a1 = hmul2_256(place_even(wb[s]));
            a3 = hmul2_256(place_odd(wb[s]));
        } else {
            a0 = place_even(wa[s]);
            a2 = place_odd(wa[s]);
            a1 = place_even(wb[s]);
            a3 = place_odd(wb[s]);
        }
        const uint2 b = *reinterpret_cast<const uint2*>(xs_thread + s * 8);
        mma_16816(acc, a0, a1, a2, a3, b.x, b.y);
    }
}

struct Args {
    const __nv_bfloat16* x;
    const uint8_t* w;
    const float* s_w;
    __nv_bfloat16* y;
    int M, N, K;
    int tiles;   // ceil(N / 16)
    int max_tpc; // max tiles per CTA (sizes the partial-sum buffer)
};

template <int CONV>
__global__ void __launch_bounds__(THREADS, 1) w8a16_kernel(const Args a) {
    extern __shared__ __align__(16) uint8_t smem[];
    const int xpitch = 2 * a.K + XROW_PAD;
    uint8_t* xs = smem;                                                    // [8][xpitch]
    float* unshift = reinterpret_cast<float*>(smem + 8 * xpitch);          // [8]
    int* shift = reinterpret_cast<int*>(unshift + 8);                      // [8]
    float* partial = reinterpret_cast<float*>(smem + 8 * xpitch + 64);     // [max_tpc][16][32][4]

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const int g = lane >> 2;
    const int t = lane & 3;

    // -------- tile range of this CTA
    const int t0 = static_cast<int>(static_cast<int64_t>(blockIdx.x) * a.tiles / gridDim.x);
    const int t1 = static_cast<int>(static_cast<int64_t>(blockIdx.x + 1) * a.tiles / gridDim.x);
    const int ntl = t1 - t0;
    const int nchunks = (a.K + 63) / 64;
    const int cpw = (nchunks + WARPS - 1) / WARPS;  // chunks per warp per tile
    const int units = ntl * cpw;

    // -------- stage x: issue this thread's x loads, then the first weight
    // units, so both are in flight together. x is kept raw (BF16) in shared
    // memory while the per-token amax is reduced, then widened in place.
    constexpr int XB = 8;  // x chunks (16 bytes) per thread per batch
    const int xchunks = a.M * (a.K / 8);
    const int kc = a.K / 8;  // chunks per row
    unsigned* row_amax = reinterpret_cast<unsigned*>(shift);  // reused before shift is set
    if (threadIdx.x < 8) row_amax[threadIdx.x] = 0u;
    uint4 xb[XB];
#pragma unroll
    for (int j = 0; j < XB; ++j) {
        const int c = threadIdx.x + THREADS * j;
        xb[j] = c < xchunks ? *reinterpret_cast<const uint4*>(a.x + static_cast<size_t>(c) * 8)
                            : make_uint4(0, 0, 0, 0);
    }
    uint4 ra[DEPTH], rb[DEPTH];
    auto load_unit = [&](int u, uint4& A, uint4& B) {
        A = make_uint4(0, 0, 0, 0);
        B = make_uint4(0, 0, 0, 0);
        if (u < units) {
            const int tl = u / cpw;
            const int chunk = warp + WARPS * (u - tl * cpw);
            const int k = chunk * 64 + 16 * t;
            const int n = (t0 + tl) * 16 + g;
            if (k < a.K) {
                if (n < a.N) A = ld_stream_v4(a.w + static_cast<size_t>(n) * a.K + k);
                if (n + 8 < a.N) B = ld_stream_v4(a.w + static_cast<size_t>(n + 8) * a.K + k);
            }
        }
    };
#pragma unroll
    for (int d = 0; d < DEPTH; ++d) load_unit(d, ra[d], rb[d]);
    __syncthreads();  // row_amax cleared
    for (int j0 = 0; j0 * THREADS < xchunks; j0 += XB) {
#pragma unroll
        for (int j = 0; j < XB; ++j) {
            const int c = threadIdx.x + THREADS * (j0 + j);
            if (j0 > 0)
                xb[j] = c < xchunks ? *reinterpret_cast<const uint4*>(a.x + static_cast<size_t>(c) * 8)
                                    : make_uint4(0, 0, 0, 0);
            const int m = c < xchunks ? c / kc : -1;
            const uint32_t wv[4] = {xb[j].x, xb[j].y, xb[j].z, xb[j].w};
            float ca = 0.0f;
#pragma unroll
            for (int i = 0; i < 4; ++i) ca = fmaxf(ca, fmaxf(fabsf(bf16_lo(wv[i])), fabsf(bf16_hi(wv[i]))));
            const unsigned peers = __match_any_sync(0xffffffffu, m);
            const unsigned mx = __reduce_max_sync(peers, __float_as_uint(ca));
            if (m >= 0) {
                if ((peers & ((1u << lane) - 1u)) == 0) atomicMax(&row_amax[m], mx);
                const int k = (c - m * kc) * 8;
                uint2* dst = reinterpret_cast<uint2*>(xs + m * xpitch + 2 * k);
                dst[0] = make_uint2(xb[j].x, xb[j].y);
                dst[1] = make_uint2(xb[j].z, xb[j].w);
            }
        }
    }
    __syncthreads();
    // per-token power-of-two shift so amax lands in [2^14, 2^15)
    if (threadIdx.x < 8) {
        const float amax = __uint_as_float(row_amax[threadIdx.x]);
        const int sh = amax > 0.0f ? 14 - ilogbf(amax) : 0;
        shift[threadIdx.x] = sh;
        unshift[threadIdx.x] = ldexpf(1.0f, -sh);
    }
    __syncthreads();
    // widen in place to FP16 (rows >= M are zero)
    for (int c = threadIdx.x; c < 8 * kc; c += THREADS) {
        const int m = c / kc;
        const int k = (c - m * kc) * 8;
        uint2* p = reinterpret_cast<uint2*>(xs + m * xpitch + 2 * k);
        uint4 out = make_uint4(0, 0, 0, 0);
        if (m < a.M) {
            const uint2 lo = p[0], hi = p[1];
            const int sh = shift[m];
            const uint32_t wv[4] = {lo.x, lo.y, hi.x, hi.y};
            float f[8];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                f[2 * j] = ldexpf(bf16_lo(wv[j]), sh);
                f[2 * j + 1] = ldexpf(bf16_hi(wv[j]), sh);
            }
            if constexpr (CONV != kCvt) {
                // the ALU widening pairs bytes (0,2) and (1,3) of each word:
                // store k in the order 0,2,1,3 within every group of four
#pragma unroll
                for (int j = 0; j < 8; j += 4) {
                    const float t1v = f[j + 1];
                    f[j + 1] = f[j + 2];
                    f[j + 2] = t1v;
                }
            }
            __half2 h[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) h[j] = __floats2half2_rn(f[2 * j], f[2 * j + 1]);
            out = *reinterpret_cast<uint4*>(h);
        }
        p[0] = make_uint2(out.x, out.y);
        p[1] = make_uint2(out.z, out.w);
    }
    __syncthreads();

    // -------- main loop over (tile, chunk) units, DEPTH units in flight
    const uint8_t* xs_thread_base = xs + g * xpitch + 2 * (16 * t);
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int u0 = 0; u0 < units; u0 += DEPTH) {
#pragma unroll
        for (int d = 0; d < DEPTH; ++d) {
            const int u = u0 + d;
            if (u < units) {
                const int tl = u / cpw;
                const int i = u - tl * cpw;
                const int chunk = warp + WARPS * i;
                if (chunk < nchunks)
                    chunk_mma<CONV>(acc, ra[d], rb[d], xs_thread_base + chunk * 128);
                load_unit(u + DEPTH, ra[d], rb[d]);
                if (i == cpw - 1) {
                    float4* dst = reinterpret_cast<float4*>(partial) + (tl * WARPS + warp) * 32 + lane;
                    *dst = make_float4(acc[0], acc[1], acc[2], acc[3]);
                    acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
                }
            }
        }
    }
    __syncthreads();

    // -------- fixed-order reduction over warps, scale, round, store
    const float fold = (CONV == kAluFold) ? 256.0f : 1.0f;
    const int per_tok = ntl * 16;
    for (int idx = threadIdx.x; idx < per_tok * a.M; idx += THREADS) {
        const int m = idx / per_tok;
        const int nl = idx - m * per_tok;
        const int tl = nl >> 4;
        const int row = nl & 15;
        const int n = (t0 + tl) * 16 + row;
        if (n >= a.N) continue;
        const int ln = (row & 7) * 4 + (m >> 1);
        const int comp = (row >> 3) * 2 + (m & 1);
        const float* src = partial + ((tl * WARPS) * 32 + ln) * 4 + comp;
        float sum = 0.f;
#pragma unroll
        for (int w = 0; w < WARPS; ++w) sum += src[w * 32 * 4];
        const float v = __fmul_rn(__fmul_rn(__fmul_rn(sum, unshift[m]), fold), a.s_w[n]);
        a.y[static_cast<size_t>(m) * a.N + n] = __float2bfloat16_rn(v);
    }
}

template <int CONV>
int launch(const Args& a, int grid, size_t smem, const DeviceInfo& di, cudaStream_t st) {
    static bool done[64];
    if (!done[di.device]) {
        int rc = cuda_check(cudaFuncSetAttribute(w8a16_kernel<CONV>,
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 di.max_smem_optin),
                            "cudaFuncSetAttribute(w8a16)");
        if (rc) return rc;
        done[di.device] = true;
    }
    w8a16_kernel<CONV><<<grid, THREADS, smem, st>>>(a);
    return cuda_check(cudaGetLastError(), "w8a16 launch");
}

}  // namespace w8a16
}  // namespace metis

using namespace metis;

extern "C" int metis_w8a16_gemm(const void* x_bf16, const uint8_t* wq, const float* s_w,
                                void* y_bf16, int64_t M, int64_t N, int64_t K,
                                metis_stream_t stream) {
    using namespace w8a16;
    clear_error();
    if (M < 1 || M > 8)
        return fail(METIS_ERR_INVALID_ARG, "w8a16_gemm: M=%lld, need 1 <= M <= 8", (long long)M);
    if (K < 16 || K % 16 != 0 || K > MAX_K)
        return fail(METIS_ERR_INVALID_ARG, "w8a16_gemm: K=%lld, need 16 <= K <= %d and K %% 16 == 0",
                    (long long)K, MAX_K);
    if (N < 1 || N > (1ll << 30))
        return fail(METIS_ERR_INVALID_ARG, "w8a16_gemm: N=%lld out of range", (long long)N);
    if (!x_bf16 || !wq || !s_w || !y_bf16)
        return fail(METIS_ERR_INVALID_ARG, "w8a16_gemm: null pointer");
    if (!aligned(x_bf16, 16) || !aligned(wq, 16) || !aligned(s_w, 4) || !aligned(y_bf16, 2))
        return fail(METIS_ERR_INVALID_ARG, "w8a16_gemm: x and wq must be 16-byte aligned");
    DeviceInfo di;
    int rc = current_device_info(&di);
    if (rc) return rc;
    Args a;
    a.x = static_cast<const __nv_bfloat16*>(x_bf16);
    a.w = wq;
    a.s_w = s_w;
    a.y = static_cast<__nv_bfloat16*>(y_bf16);
    a.M = static_cast<int>(M);
    a.N = static_cast<int>(N);
    a.K = static_cast<int>(K);
    a.tiles = static_cast<int>((N + 15) / 16);
    const size_t xbytes = 8 * static_cast<size_t>(2 * K + XROW_PAD) + 64;
    const size_t per_tile = WARPS * 32 * 4 * sizeof(float);
    const size_t budget = static_cast<size_t>(di.max_smem_optin);
    if (xbytes + per_tile > budget) return fail(METIS_ERR_UNSUPPORTED, "w8a16_gemm: K too large");
    const int max_tpc_fit = static_cast<int>((budget - xbytes) / per_tile);
    int grid = a.tiles < di.num_sms ? a.tiles : di.num_sms;
    if ((a.tiles + grid - 1) / grid > max_tpc_fit) grid = (a.tiles + max_tpc_fit - 1) / max_tpc_fit;
    a.max_tpc = (a.tiles + grid - 1) / grid;
    const size_t smem = xbytes + per_tile * a.max_tpc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    switch (g_variant) {
        case kAluMul: return launch<kAluMul>(a, grid, smem, di, st);
        case kAluFold: return launch<kAluFold>(a, grid, smem, di, st);
        default: return launch<kCvt>(a, grid, smem, di, st);
    }
}

// Tuning hook: selects how E4M3 weights are widened to FP16 (0: cvt
// instruction, 1: bit placement + exact x256 multiply, 2: bit placement with
// the x256 folded into the epilogue). Returns the previous setting.
extern "C" METIS_API int metis_internal_w8a16_variant(int v) {
    const int old = w8a16::g_variant;
    if (v >= 0 && v <= 2) w8a16::g_variant = v;
    return old;
}
