// NVFP4 routed-expert maths on sm_100a ("Lernex/Metis-1.6-Praxis-NVFP4",
// "What is in NVFP4": E2M1 values with one E4M3 scale per 16 inputs and one
// FP32 scale per expert; "What --fast-math does": on Blackwell the 4-bit
// experts multiply in FP4, their inputs rounded to FP4 too).
//
//   nvfp4_quant_kernel   one warp per row: the row's (or its set's) amax gives
//                        the global scale g = amax/2688; each lane takes one
//                        16-element block per pass (a warp covers 512
//                        contiguous elements), rounds the block scale to E4M3
//                        and the elements to E2M1 (cvt.rn.satfinite), writes
//                        8 bytes of packed codes, and every fourth lane writes
//                        the 4 scales of its 64-element chunk as one word, in
//                        row-major or in the tensor cores' tiled layout.
//   nvfp4_gemm_kernel    persistent, warp-specialised block-scaled GEMM
//                        (tcgen05.mma kind::mxf4nvf4 block16, K = 64 per
//                        instruction), 704 threads per CTA. CTA pairs
//                        (cta_group::2, 256 x 256 tiles) for the grouped GEMM
//                        and for M > 128; one CTA (128 x 256) otherwise.
//                          warp 0       TMA of the A and B code tiles (128-byte
//                                       swizzle) and of the stage's tiled scale
//                                       atoms (pairs: TMA through a 256-byte-row
//                                       view, completing on the even CTA's
//                                       barrier; one CTA: bulk copies) into a
//                                       ring of 5 (pairs, dense), 4 (pairs,
//                                       grouped) or 3 (one CTA) stages;
//                          warp 1       TMEM owner; one lane of the even CTA
//                                       issues the MMAs;
//                          warps 2-17   epilogue: four warps per TMEM lane
//                                       quadrant, 64 columns each, read the
//                                       whole accumulator at once, hand it back
//                                       with a relaxed arrive, then scale
//                                       (g_a[row] * g_b), round to BF16 and
//                                       store through a swizzled staging block;
//                          warps 18-21  one per 64-element chunk: copy the
//                                       chunk's scale atoms of each stage into
//                                       TMEM (tcgen05.cp 32x128b.warpx4), into
//                                       the next of four 48-column buffers.
//                        TMEM: one 256-column FP32 accumulator (the scale
//                        buffers need columns too, so two accumulators do not
//                        fit in 512). Dense tiles run in groups of RASTER_M row
//                        blocks; grouped tiles follow the padded expert offsets.
#include "common.cuh"
#include "../../include/metis_nvfp4.h"

namespace metis {
namespace nvfp4 {

// ----------------------------------------------------------------- helpers

// Eight binary32 values -> eight E2M1 codes, round-to-nearest-even and
// saturating to +-6 (cvt.rn.satfinite.e2m1x2 puts its first source in the
// high nibble); v[0] lands in bits 0..3 of the result.
// Elementwise maximum of two BF16 pairs (a NaN operand yields the other).
__device__ __forceinline__ uint32_t bf16x2_max(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("max.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

__device__ __forceinline__ uint32_t f32x8_to_e2m1x8(const float* v) {
    uint32_t r;
    asm("{\n\t"
        ".reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t"
        "}"
        : "=r"(r)
        : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
    return r;
}

// Exact value of an E4M3 byte (through FP16, which holds every E4M3 value).
__device__ __forceinline__ float e4m3_to_f32(uint32_t code) {
    float f;
    asm("{\n\t"
        ".reg .b16 q, lo, hi;\n\t"
        ".reg .b32 h;\n\t"
        "cvt.u16.u32 q, %1;\n\t"
        "cvt.rn.f16x2.e4m3x2 h, q;\n\t"
        "mov.b32 {lo, hi}, h;\n\t"
        "cvt.f32.f16 %0, lo;\n\t"
        "}"
        : "=f"(f)
        : "r"(code & 0xFFu));
    return f;
}

__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// 16 consecutive elements of a row, widened to binary32 exactly.
__device__ __forceinline__ void load16(const __nv_bfloat16* p, float (&v)[16]) {
    const uint4 a = ld_nc_v4(p), b = ld_nc_v4(p + 8);
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        v[2 * i] = bf16_lo(w[i]);
        v[2 * i + 1] = bf16_hi(w[i]);
    }
}
__device__ __forceinline__ void load16(const float* p, float (&v)[16]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint4 a = ld_nc_v4(p + 4 * i);
        v[4 * i] = __uint_as_float(a.x);
        v[4 * i + 1] = __uint_as_float(a.y);
        v[4 * i + 2] = __uint_as_float(a.z);
        v[4 * i + 3] = __uint_as_float(a.w);
    }
}

// Byte offset of the 4 scales of (row r, 64-element chunk c) in the tiled
// layout [ceil(R/128)][K/64][512]: atom (r/128, c), byte 16 (r%32) + 4 ((r%128)/32).
__host__ __device__ __forceinline__ int64_t tiled_sf_offset(int64_t r, int64_t c, int64_t kc) {
    return ((r >> 7) * kc + c) * 512 + 16 * (r & 31) + 4 * ((r & 127) >> 5);
}

// ----------------------------------------------------------- quantization

constexpr int QWARPS = 8;

struct QuantArgs {
    const void* x;
    int64_t R, K, ldx;        // rows, elements per row, elements between rows
    uint8_t* q;               // packed codes, K/2 bytes per row
    uint8_t* sf;              // block scales
    int tiled;                // sf layout: 0 row-major [R, K/16], 1 tiled
    float* g;                 // global scales (written when gamax is null)
    const float* gamax;       // sets of rows: amax of the row's set, else null
    int64_t rps;              // rows per set (gamax only)
    const int32_t* dst_rows;  // gather: row r goes to rows dst_rows[r * topk + j]
    int topk;
    const int32_t* row_valid; // rows with row_valid[r] < 0 are skipped
    const int32_t* nrows;     // device row count (rows >= *nrows are skipped)
    int64_t pad_rows;         // tiled, no gather: rows [R, pad_rows) get zero scales
};

// One row's quantization by one warp. NBL > 0 (BF16 rows with K <= 512 NBL):
// the row is already in registers, lane l holding blocks l, l + 32, ... in
// raw; NBL = 0 reads it twice (amax pass, then codes).
template <typename T, int NBL>
__device__ __forceinline__ void quant_row(const QuantArgs& a, int64_t r, int lane,
                                          const uint4 (&raw)[NBL > 0 ? NBL : 1][2],
                                          const float* inv_scale) {
    const T* row = static_cast<const T*>(a.x) + r * a.ldx;
    const int nb = static_cast<int>(a.K / 16);
    const int64_t kc = a.K / 64;
    auto unpack = [&](int i, float (&v)[16]) {
        const uint32_t w[8] = {raw[i][0].x, raw[i][0].y, raw[i][0].z, raw[i][0].w,
                               raw[i][1].x, raw[i][1].y, raw[i][1].z, raw[i][1].w};
#pragma unroll
        for (int h = 0; h < 8; ++h) {
            v[2 * h] = bf16_lo(w[h]);
            v[2 * h + 1] = bf16_hi(w[h]);
        }
    };
    // register-resident rows: each block's maximum, taken once for both the
    // row amax and the block scale, on the packed BF16 pairs (sign cleared,
    // then max.bf16x2, which like fmaxf ignores a NaN operand)
    float bmax[NBL > 0 ? NBL : 1];
    if constexpr (NBL > 0) {
#pragma unroll
        for (int i = 0; i < NBL; ++i) {
            const uint32_t w[8] = {raw[i][0].x, raw[i][0].y, raw[i][0].z, raw[i][0].w,
                                   raw[i][1].x, raw[i][1].y, raw[i][1].z, raw[i][1].w};
            uint32_t m2 = w[0] & 0x7FFF7FFFu;
#pragma unroll
            for (int h = 1; h < 8; ++h) m2 = bf16x2_max(m2, w[h] & 0x7FFF7FFFu);
            bmax[i] = fmaxf(bf16_lo(m2), bf16_hi(m2));
        }
    } else {
        bmax[0] = 0.0f;
    }
    float amax;
    if (a.gamax) {
        amax = a.gamax[r / a.rps];
    } else {
        float m = 0.0f;
        if constexpr (NBL > 0) {
#pragma unroll
            for (int i = 0; i < NBL; ++i) m = fmaxf(m, bmax[i]);
        } else {
            for (int b = lane; b < nb; b += 32) {
                float v[16];
                load16(row + 16 * b, v);
#pragma unroll
                for (int h = 0; h < 16; ++h) m = fmaxf(m, fabsf(v[h]));
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        amax = m;
    }
    const float inv_g = amax > 0.0f ? fminf(__fdiv_rn(2688.0f, amax), 3.402823466e38f) : 0.0f;
    const float g_row = __fdiv_rn(amax, 2688.0f);
    const int ndst = a.dst_rows ? a.topk : 1;
    // the destination rows, loaded once per row: lane j holds destination j
    // (up to 32 of them; more are read from memory where they are used)
    const int my_dst = (a.dst_rows && lane < ndst) ? a.dst_rows[r * a.topk + lane] : -1;
    // one pass over 32 blocks (512 elements); v holds this lane's block b0 + lane
    // and bm its maximum magnitude
    auto block_pass = [&](int b0, const float (&v)[16], float bm) {
        const int b = b0 + lane;
        uint32_t lo = 0, hi = 0, sbc = 0;
        if (b < nb) {
            sbc = f32x2_to_e4m3x2(__fdiv_rn(__fmul_rn(bm, inv_g), 6.0f), 0.0f) & 0xFFu;
            const float inv_s = inv_scale[sbc];
            float w[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) w[i] = __fmul_rn(__fmul_rn(v[i], inv_g), inv_s);
            lo = f32x8_to_e2m1x8(w);
            hi = f32x8_to_e2m1x8(w + 8);
        }
        // the scales of the 4 blocks of a 64-element chunk (lanes 4c .. 4c+3)
        uint32_t s4 = sbc;
        s4 |= __shfl_down_sync(0xffffffffu, sbc, 1) << 8;
        s4 |= __shfl_down_sync(0xffffffffu, sbc, 2) << 16;
        s4 |= __shfl_down_sync(0xffffffffu, sbc, 3) << 24;
        for (int j = 0; j < ndst; ++j) {
            int64_t dr = r;
            if (a.dst_rows) {
                const int d = __shfl_sync(0xffffffffu, my_dst, j & 31);
                dr = j < 32 ? d : a.dst_rows[r * a.topk + j];
            }
            if (dr < 0 || b >= nb) continue;
            *reinterpret_cast<uint2*>(a.q + dr * (a.K / 2) + 8 * b) = make_uint2(lo, hi);
            if ((lane & 3) == 0) {
                const int64_t off = a.tiled ? tiled_sf_offset(dr, b / 4, kc) : dr * (a.K / 16) + b;
                *reinterpret_cast<uint32_t*>(a.sf + off) = s4;
            }
            if (b0 == 0 && lane == 0 && !a.gamax) a.g[dr] = g_row;
        }
    };
    if constexpr (NBL > 0) {
        // register-resident rows: every block of the row is encoded first
        // (lane l: blocks l, l + 32, ...), then stored to each destination
        // row with that row's code and scale offsets computed once
        uint32_t lo[NBL], hi[NBL], s4[NBL];
#pragma unroll
        for (int i = 0; i < NBL; ++i) {
            lo[i] = hi[i] = s4[i] = 0;
            if (32 * i >= nb) continue;  // warp-uniform
            const int b = 32 * i + lane;
            uint32_t sbc = 0;
            if (b < nb) {
                float v[16];
                unpack(i, v);
                sbc = f32x2_to_e4m3x2(__fdiv_rn(__fmul_rn(bmax[i], inv_g), 6.0f), 0.0f) & 0xFFu;
                const float inv_s = inv_scale[sbc];
                float w[16];
#pragma unroll
                for (int h = 0; h < 16; ++h) w[h] = __fmul_rn(__fmul_rn(v[h], inv_g), inv_s);
                lo[i] = f32x8_to_e2m1x8(w);
                hi[i] = f32x8_to_e2m1x8(w + 8);
            }
            // the scales of the 4 blocks of a 64-element chunk (lanes 4c .. 4c+3)
            uint32_t s = sbc;
            s |= __shfl_down_sync(0xffffffffu, sbc, 1) << 8;
            s |= __shfl_down_sync(0xffffffffu, sbc, 2) << 16;
            s |= __shfl_down_sync(0xffffffffu, sbc, 3) << 24;
            s4[i] = s;
        }
        for (int j = 0; j < ndst; ++j) {
            int64_t dr = r;
            if (a.dst_rows) {
                const int d = __shfl_sync(0xffffffffu, my_dst, j & 31);
                dr = j < 32 ? d : a.dst_rows[r * a.topk + j];
            }
            if (dr < 0) continue;  // warp-uniform
            uint8_t* qrow = a.q + dr * (a.K / 2);
            uint8_t* srow = a.sf + (a.tiled ? tiled_sf_offset(dr, 0, kc) : dr * (a.K / 16));
#pragma unroll
            for (int i = 0; i < NBL; ++i) {
                const int b = 32 * i + lane;
                if (b >= nb) continue;
                *reinterpret_cast<uint2*>(qrow + 8 * b) = make_uint2(lo[i], hi[i]);
                if ((lane & 3) == 0)
                    *reinterpret_cast<uint32_t*>(srow + (a.tiled ? 512 * (b >> 2) : b)) = s4[i];
            }
            if (lane == 0 && !a.gamax) a.g[dr] = g_row;
        }
    } else {
        for (int b0 = 0; b0 < nb; b0 += 32) {
            float v[16];
#pragma unroll
            for (int h = 0; h < 16; ++h) v[h] = 0.0f;
            if (b0 + lane < nb) load16(row + 16 * (b0 + lane), v);
            float bm = 0.0f;
#pragma unroll
            for (int h = 0; h < 16; ++h) bm = fmaxf(bm, fabsf(v[h]));
            block_pass(b0, v, bm);
        }
    }
}

// RPW rows per warp (rows r0 .. r0 + RPW - 1): with NBL > 0 every row's loads
// are issued before the first row is encoded, so a warp waits on memory once.
template <typename T, int NBL, int RPW>
__global__ void __launch_bounds__(QWARPS * 32, (NBL > 0 && NBL <= 4) ? 4 : 1) nvfp4_quant_kernel(const QuantArgs a) {
    static_assert(QWARPS * 32 == 256, "one thread per E4M3 code builds the reciprocal table");
    static_assert(NBL == 0 || sizeof(T) == 2, "register-resident rows are BF16");
    static_assert(NBL > 0 || RPW == 1, "two-pass rows are one per warp");
    // 1 / D(code) for every E4M3 block-scale code (0 for a zero scale): the
    // same IEEE division, once per code instead of once per block
    __shared__ float inv_scale[256];
    {
        const float d = e4m3_to_f32(threadIdx.x);
        inv_scale[threadIdx.x] = d > 0.0f ? __fdiv_rn(1.0f, d) : 0.0f;
    }
    __syncthreads();
    grid_dependency_wait();  // the rows may be the previous kernel's output
    grid_launch_dependents();
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int64_t r0 = (static_cast<int64_t>(blockIdx.x) * QWARPS + warp) * RPW;
    const int64_t kc = a.K / 64;
    const int nb = static_cast<int>(a.K / 16);
    uint4 raw[RPW][NBL > 0 ? NBL : 1][2];
    bool live[RPW];
    // which rows are real (the routed layer's padded rows are not): lane u
    // reads row u's validity, one round trip for all RPW rows, so that the
    // rows that are skipped are never read
    {
        bool lv = false;
        if (lane < RPW) {
            const int64_t r = r0 + lane;
            lv = r < a.R && !(a.nrows && r >= *a.nrows) && !(a.row_valid && a.row_valid[r] < 0);
        }
        const unsigned m = __ballot_sync(0xffffffffu, lv);
#pragma unroll
        for (int u = 0; u < RPW; ++u) live[u] = (m >> u) & 1u;
    }
#pragma unroll
    for (int u = 0; u < RPW; ++u) {
        const int64_t r = r0 + u;
#pragma unroll
        for (int i = 0; i < (NBL > 0 ? NBL : 1); ++i) {
            const int b = lane + 32 * i;
            if (NBL > 0 && live[u] && b < nb) {
                const T* row = static_cast<const T*>(a.x) + r * a.ldx;
                raw[u][i][0] = ld_nc_v4(row + 16 * b);
                raw[u][i][1] = ld_nc_v4(row + 16 * b + 8);
            } else {
                raw[u][i][0] = raw[u][i][1] = make_uint4(0u, 0u, 0u, 0u);
            }
        }
    }
#pragma unroll
    for (int u = 0; u < RPW; ++u) {
        const int64_t r = r0 + u;
        if (r >= a.R) {
            // zero scales for the pad rows of the last 128-row atom
            if (a.tiled && r < a.pad_rows) {
                for (int64_t c = lane; c < kc; c += 32)
                    *reinterpret_cast<uint32_t*>(a.sf + tiled_sf_offset(r, c, kc)) = 0u;
            }
        } else if (live[u]) {
            quant_row<T, NBL>(a, r, lane, raw[u], inv_scale);
        }
    }
}

// amax of each set of rows, as the largest binary32 bit pattern (|x| >= 0 so
// the integer order is the float order); gamax zeroed beforehand.
template <typename T>
__global__ void __launch_bounds__(QWARPS * 32) nvfp4_set_amax_kernel(const T* __restrict__ x, int64_t R,
                                                                     int64_t K, int64_t ldx,
                                                                     int64_t rps,
                                                                     unsigned int* gamax) {
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int64_t r = static_cast<int64_t>(blockIdx.x) * QWARPS + warp;
    if (r >= R) return;
    const T* row = x + r * ldx;
    float m = 0.0f;
    for (int64_t b = lane; b < K / 16; b += 32) {
        float v[16];
        load16(row + 16 * b, v);
#pragma unroll
        for (int i = 0; i < 16; ++i) m = fmaxf(m, fabsf(v[i]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) atomicMax(gamax + r / rps, __float_as_uint(m));
}

// g[i] = amax[i] / 2688, in place.
__global__ void nvfp4_finish_scales_kernel(float* g, int64_t n) {
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i < n) g[i] = __fdiv_rn(g[i], 2688.0f);
}

// Row-major [R, K/16] -> tiled, one thread per (row, 64-element chunk).
__global__ void nvfp4_tile_scales_kernel(const uint8_t* __restrict__ sf, int64_t R, int64_t Rp,
                                         int64_t K, uint8_t* __restrict__ out) {
    const int64_t kc = K / 64;
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= Rp * kc) return;
    const int64_t r = i / kc, c = i - r * kc;
    const uint32_t v = r < R ? *reinterpret_cast<const uint32_t*>(sf + r * (K / 16) + 4 * c) : 0u;
    *reinterpret_cast<uint32_t*>(out + tiled_sf_offset(r, c, kc)) = v;
}

}  // namespace nvfp4

// Launches the per-row quantizer (the arguments validated by the caller).
template <typename T>
int launch_nvfp4_quant(const T* x, int64_t R, int64_t K, int64_t ldx, int64_t rps, uint8_t* q,
                       uint8_t* sf, int tiled, float* g, const int32_t* dst_rows, int topk,
                       const int32_t* row_valid, const int32_t* nrows, cudaStream_t st) {
    using namespace nvfp4;
    nvfp4::QuantArgs a{};
    a.x = x;
    a.R = R;
    a.K = K;
    a.ldx = ldx;
    a.q = q;
    a.sf = sf;
    a.tiled = tiled;
    a.g = g;
    a.rps = rps;
    a.dst_rows = dst_rows;
    a.topk = topk;
    a.row_valid = row_valid;
    a.nrows = nrows;
    a.pad_rows = (tiled && !dst_rows) ? (R + 127) / 128 * 128 : R;
    int rc;
    if (rps > 1) {
        // the set amax goes through g, which the last kernel turns into g = amax/2688
        const int64_t sets = R / rps;
        if ((rc = cuda_check(cudaMemsetAsync(g, 0, sets * sizeof(float), st), "nvfp4 amax reset"))) return rc;
        nvfp4_set_amax_kernel<T><<<static_cast<unsigned>((R + QWARPS - 1) / QWARPS), QWARPS * 32, 0, st>>>(
            x, R, K, ldx, rps, reinterpret_cast<unsigned int*>(g));
        if ((rc = cuda_check(cudaGetLastError(), "nvfp4 amax launch"))) return rc;
        a.gamax = g;
    }
    const int64_t rows = a.pad_rows;
    auto go = [&](auto kernel, int rpw) {
        const dim3 grid(static_cast<unsigned>((rows + QWARPS * rpw - 1) / (QWARPS * rpw)));
        return cuda_check(launch_pdl(kernel, grid, dim3(QWARPS * 32), 0, st, 1, a), "nvfp4 quant launch");
    };
    // BF16 rows of up to 4096 elements stay in registers (one read of x);
    // rows of up to 1024 go two to a warp
    if constexpr (sizeof(T) == 2) {
        if (rps == 1 && K <= 512) rc = go(nvfp4_quant_kernel<T, 1, 2>, 2);
        else if (rps == 1 && K <= 1024) rc = go(nvfp4_quant_kernel<T, 2, 2>, 2);
        else if (rps == 1 && K <= 2048) rc = go(nvfp4_quant_kernel<T, 4, 1>, 1);
        else if (rps == 1 && K <= 4096) rc = go(nvfp4_quant_kernel<T, 8, 1>, 1);
        else rc = go(nvfp4_quant_kernel<T, 0, 1>, 1);
    } else {
        rc = go(nvfp4_quant_kernel<T, 0, 1>, 1);
    }
    if (rc) return rc;
    if (rps > 1) {
        const int64_t sets = R / rps;
        nvfp4_finish_scales_kernel<<<static_cast<unsigned>((sets + 255) / 256), 256, 0, st>>>(g, sets);
        if ((rc = cuda_check(cudaGetLastError(), "nvfp4 scale launch"))) return rc;
    }
    return METIS_OK;
}

template int launch_nvfp4_quant<__nv_bfloat16>(const __nv_bfloat16*, int64_t, int64_t, int64_t, int64_t,
                                               uint8_t*, uint8_t*, int, float*, const int32_t*, int,
                                               const int32_t*, const int32_t*, cudaStream_t);
template int launch_nvfp4_quant<float>(const float*, int64_t, int64_t, int64_t, int64_t, uint8_t*,
                                       uint8_t*, int, float*, const int32_t*, int, const int32_t*,
                                       const int32_t*, cudaStream_t);

}  // namespace metis

// ------------------------------------------------------------------- GEMM
namespace metis {
namespace nvfp4 {

constexpr int BKB = 128;        // code bytes per row per k-block (256 elements)
constexpr int KCH = 4;          // 64-element MMA chunks per k-block
constexpr int ROWS = 128;       // rows of A per CTA per tile (TMEM lanes)
constexpr int BN = 256;         // output columns per tile
constexpr int EPI_WARPS = 16;   // four per TMEM lane quadrant
constexpr int SCALE_WARP = 2 + EPI_WARPS;   // first of the warps copying scale factors into TMEM
constexpr int SCALE_WARPS = 4;              // each copies one of a k-block's four 64-element chunks
constexpr int THREADS = 64 + EPI_WARPS * 32 + SCALE_WARPS * 32;
constexpr int ATOM = 512;       // one tiled scale atom: 128 rows x 4 scales
constexpr int SFA_STAGE = KCH * ATOM;       // this CTA's 128 rows of A
constexpr int SFB_STAGE = 2 * KCH * ATOM;   // both 128-row halves of B (every CTA)
constexpr int STAGING = EPI_WARPS * 32 * 64;    // a 32 x 32 BF16 block per epilogue warp
constexpr int MAX_GROUPS = 1024;
constexpr int TMEM_COLS = 512;
constexpr int SF_COL = BN;      // one scale buffer of 48 columns per ring stage after the accumulator
constexpr int SF_BUF = 48;      // SFA: 4 chunks x 4 columns; SFB: 4 chunks x 8 columns
constexpr int SF_ROW = 256;     // the scale buffers seen by TMA as rows of 256 bytes

// Instruction descriptor of tcgen05.mma kind::mxf4nvf4: A and B E2M1 (format
// 1), K-major, UE4M3 scales (bit 23 clear), dense K = 64, N >> 3 at bit 17,
// M >> 4 at bit 24; the scale-factor ids (bits 4-5, 29-30) stay 0.
__host__ __device__ constexpr uint32_t idesc_nvf4(int m, int n) {
    return (1u << 7) | (1u << 10) | (static_cast<uint32_t>(n >> 3) << 17) |
           (static_cast<uint32_t>(m >> 4) << 24);
}

// Shared-memory layout of the one-CTA (CTAS = 1, 128 x 256 tiles) and the
// CTA-pair (CTAS = 2, 256 x 256 tiles: each CTA holds 128 rows of A, 128 rows
// of B and the scales of all 256 rows of B) kernels.
template <int CTAS, bool GROUPED>
struct Lay {
    static constexpr int B_ROWS = BN / CTAS;
    static constexpr int A_STAGE = ROWS * BKB;
    static constexpr int B_STAGE = B_ROWS * BKB;
    static constexpr int STAGES = CTAS == 2 ? (GROUPED ? 4 : 5) : 3;
    static constexpr int A_OFF = 0;
    static constexpr int B_OFF = A_OFF + STAGES * A_STAGE;
    static constexpr int SFA_OFF = B_OFF + STAGES * B_STAGE;
    static constexpr int SFB_OFF = SFA_OFF + STAGES * SFA_STAGE;
    static constexpr int TILES = SFB_OFF + STAGES * SFB_STAGE;
    // landed (TMA bytes), full (scales in TMEM), empty, scale buffer free
    // (grouped), tfull, tempty, drain, scale drain
    static constexpr int NUM_BARS = 4 * STAGES + 3 + SCALE_WARPS;
    static_assert(SF_COL + STAGES * SF_BUF <= TMEM_COLS, "TMEM: accumulator and one scale buffer per stage");
    static constexpr int BAR_OFF = TILES + STAGING;
    static constexpr int MISC_OFF = BAR_OFF + NUM_BARS * 8;
    static constexpr int GROUP_OFF = MISC_OFF + 16;
    static constexpr size_t BYTES = 1024 + GROUP_OFF + (GROUPED ? 3 * (MAX_GROUPS + 1) * 4 : 0);
    static constexpr uint32_t IDESC = idesc_nvf4(ROWS * CTAS, BN);
    // CTA pair: both CTAs' loads of a stage counted on the even CTA's barrier
    static constexpr uint32_t PAIR_TX = CTAS * (A_STAGE + B_STAGE + SFA_STAGE + SFB_STAGE);
};

// Shared-memory descriptor of one scale atom as the tcgen05.cp source: 32
// rows of 16 bytes, no swizzle, 8-row core matrices 128 bytes apart.
__device__ __forceinline__ uint64_t sf_atom_desc(uint32_t saddr) {
    uint64_t d = static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>(1) << 16;          // leading byte offset (one core matrix along K)
    d |= static_cast<uint64_t>(128 >> 4) << 32;   // stride byte offset
    d |= static_cast<uint64_t>(1) << 46;          // descriptor version (sm_100)
    return d;
}

// Copies one 512-byte atom into TMEM columns [taddr, taddr + 4) of every lane
// quadrant: lane l of each quadrant gets bytes 16 l .. 16 l + 15. The pair
// form, issued by the even CTA, copies each CTA's atom at this shared-memory
// offset into its own TMEM.
__device__ __forceinline__ void sf_copy(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
                 : "memory");
}
__device__ __forceinline__ void sf_copy_pair(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
                 : "memory");
}

__device__ __forceinline__ void mma_nvf4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
        : "memory");
}
// The CTA pair's block-scaled MMA (M = 256: 128 rows of A per CTA, B rows
// split between the CTAs, each CTA's TMEM holding its own rows of D, its own
// A scales and all of B's scales).
__device__ __forceinline__ void mma_nvf4_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                              uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                              uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
        : "memory");
}

// Non-tensor bulk copy global -> shared, completing on an mbarrier of this CTA.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(dst), "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

struct GemmParams {
    const uint8_t* sfa;       // tiled scales of A
    const float* ga;          // [rows of A]
    const uint8_t* sfb;       // tiled scales of B ([groups * N] rows)
    const float* gb;          // [groups]
    __nv_bfloat16* y;         // [rows of A, N]
    const int32_t* offsets;   // grouped: [E + 1] first rows (multiples of 128); dense: null
    const int32_t* counts;    // grouped: [E] rows per group
    int M, N, K, E;
    uint32_t* status;
    uint64_t timeout_ns;
};

struct Tile {
    int a_row0, row_end, b_row0, b_base, n0, group;
};

// Row blocks per raster group of the dense schedule (16384 x 8192 x 8192:
// 506 -> 473 us against row-block-fastest order over the whole matrix).
constexpr int RASTER_M = 16;

// Tile t -> rows and columns; a tile is 128 * CTAS rows of A (this CTA's
// 128 at rank * 128) by BN columns.
template <int CTAS>
struct Sched {
    int num_n, num_m, total, N, M;
    uint32_t rank;
    const int* g_tile;   // grouped: prefix sums of tiles per group (smem)
    const int* g_row;    // grouped: first rows (smem)
    const int* g_cnt;    // grouped: rows per group (smem)
    int E;
    __device__ __forceinline__ Tile get(int t) const {
        Tile ti;
        if (g_tile == nullptr) {
            // groups of RASTER_M row blocks, row block fastest inside a group:
            // the tiles running together share a few row blocks of A and
            // column blocks of B in L2
            const int per_group = RASTER_M * num_n;
            const int g = t / per_group, r = t - g * per_group;
            const int gm = min(RASTER_M, num_m - g * RASTER_M);
            const int mb = g * RASTER_M + r % gm, nb = r / gm;
            ti.a_row0 = mb * ROWS * CTAS + static_cast<int>(rank) * ROWS;
            ti.row_end = M;
            ti.b_base = nb * BN;
            ti.n0 = nb * BN;
            ti.group = 0;
        } else {
            int lo = 0, hi = E;
            while (hi - lo > 1) {
                const int mid = (lo + hi) >> 1;
                if (g_tile[mid] <= t) lo = mid; else hi = mid;
            }
            const int e = lo;
            const int local = t - g_tile[e];
            const int mt = (g_cnt[e] + ROWS * CTAS - 1) / (ROWS * CTAS);
            const int mb = local % mt, nb = local / mt;
            ti.a_row0 = g_row[e] + mb * ROWS * CTAS + static_cast<int>(rank) * ROWS;
            ti.row_end = g_row[e] + g_cnt[e];
            ti.b_base = e * N + nb * BN;
            ti.n0 = nb * BN;
            ti.group = e;
        }
        ti.b_row0 = ti.b_base + static_cast<int>(rank) * (BN / CTAS);
        return ti;
    }
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// One 32-column chunk: y = bf16(acc * g_a[row] * g_b), staged in the warp's
// swizzled 32 x 64-byte block (the 64-byte TMA swizzle) and written by one TMA
// store when all 32 rows belong to the tile's group (the map clips columns
// past N), else as 8 rows x 64 bytes per instruction by the lanes.
__device__ __forceinline__ void store_chunk(const uint32_t (&v)[32], int c, const Tile& ti, int q,
                                            int lane, float ga, float gb, uint8_t* stg,
                                            __nv_bfloat16* y, int N, const CUtensorMap* tmY) {
    uint32_t pk[16];
#pragma unroll
    for (int j = 0; j < 16; ++j)
        pk[j] = pack_bf16x2(__fmul_rn(__fmul_rn(__uint_as_float(v[2 * j]), ga), gb),
                            __fmul_rn(__fmul_rn(__uint_as_float(v[2 * j + 1]), ga), gb));
    // the previous chunk's store has read the staging block
    if (lane == 0) bulk_wait_read();
    __syncwarp();
#pragma unroll
    for (int pc = 0; pc < 4; ++pc)
        *reinterpret_cast<uint4*>(stg + lane * 64 + ((pc ^ ((lane >> 1) & 3)) * 16)) =
            make_uint4(pk[4 * pc], pk[4 * pc + 1], pk[4 * pc + 2], pk[4 * pc + 3]);
    const int row0 = ti.a_row0 + q * 32;
    if (ti.n0 + c * 32 >= N) return;  // wholly past the last column: nothing to store
    if (row0 + 32 <= ti.row_end) {
        fence_proxy_async_shared();  // the staging writes, to the TMA engine
        __syncwarp();
        if (lane == 0) {
            tma_store_2d(tmY, smem_u32(stg), ti.n0 + c * 32, row0);
            bulk_commit();
        }
        return;
    }
    __syncwarp();
    const int n = ti.n0 + c * 32 + (lane & 3) * 8;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int rr = (lane >> 2) + 8 * i;
        const uint4 val =
            *reinterpret_cast<const uint4*>(stg + rr * 64 + (((lane & 3) ^ ((rr >> 1) & 3)) * 16));
        const int row = ti.a_row0 + q * 32 + rr;
        if (row < ti.row_end && n < N)
            *reinterpret_cast<uint4*>(y + static_cast<size_t>(row) * N + n) = val;
    }
}

template <int CTAS, bool GROUPED>
__global__ void __launch_bounds__(THREADS, 1)
nvfp4_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                  const __grid_constant__ CUtensorMap tmSFA, const __grid_constant__ CUtensorMap tmSFB,
                  const __grid_constant__ CUtensorMap tmY, const GemmParams p) {
    using L = Lay<CTAS, GROUPED>;
    constexpr int STAGES = L::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint8_t* staging = smem + L::TILES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 4);
    int* g_tile = reinterpret_cast<int*>(smem + L::GROUP_OFF);
    int* g_row = g_tile + (MAX_GROUPS + 1);
    int* g_cnt = g_row + (MAX_GROUPS + 1);

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const uint32_t rank = CTAS == 2 ? cluster_ctarank() : 0u;
    const bool leader = rank == 0;
    // A stage's TMA bytes (codes and scale atoms) complete `landed`, which
    // the scale-copy warps wait on; their copies into the stage's TMEM scale
    // buffer complete `full`. Dense: `full` is the one barrier the MMA thread
    // waits on, and its commit to `empty` frees both the shared-memory stage
    // (for the producer) and the scale buffer (a stage cannot land again
    // before its previous MMAs are done, so the scale warps need no wait of
    // their own for it): one wait and one commit per 4 MMAs, since one
    // thread issues them all at about the tensor pipe's rate (16384 x 8192 x
    // 8192: 492 -> 464 us). Grouped (short k-loops per tile): the MMA thread
    // waits on `landed` and `full`, and frees the scale buffer with a second
    // commit, to `sfree`, that the scale warps wait on; the routed layer
    // measured 1.2 us faster that way.
    auto full = [&](int s) { return smem_u32(&bars[s]); };
    auto empty = [&](int s) { return smem_u32(&bars[STAGES + s]); };
    auto landed = [&](int s) { return smem_u32(&bars[2 * STAGES + s]); };
    auto sfree = [&](int s) { return smem_u32(&bars[3 * STAGES + s]); };
    const uint32_t tfull = smem_u32(&bars[4 * STAGES]);
    const uint32_t tempty = smem_u32(&bars[4 * STAGES + 1]);
    const uint32_t drain = smem_u32(&bars[4 * STAGES + 2]);
    const uint32_t sdrain = smem_u32(&bars[4 * STAGES + 3]);

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(landed(s), 1);
            mbar_init(full(s), SCALE_WARPS);
            mbar_init(empty(s), 1);
            mbar_init(sfree(s), 1);
        }
        mbar_init(tfull, 1);
        mbar_init(tempty, CTAS * EPI_WARPS);
        mbar_init(drain, 1);
        for (int w = 0; w < SCALE_WARPS; ++w) mbar_init(sdrain + 8 * w, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        tma_prefetch_desc(&tmY);
        if constexpr (CTAS == 2) {
            tma_prefetch_desc(&tmSFA);
            tma_prefetch_desc(&tmSFB);
        }
    }
    if (warp == 1) {
        if constexpr (CTAS == 2) {
            tmem_alloc_pair(smem_u32(tmem_slot), TMEM_COLS);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
            tmem_relinquish();
        }
    }

    // operands, scales and offsets may come from the previous kernel (PDL)
    grid_launch_dependents();
    grid_dependency_wait();

    Sched<CTAS> sc;
    sc.N = p.N;
    sc.M = p.M;
    sc.E = p.E;
    sc.rank = rank;
    sc.num_n = (p.N + BN - 1) / BN;
    constexpr int TROWS = ROWS * CTAS;   // rows of A per tile
    if constexpr (GROUPED) {
        if (warp == 0) {
            const int per = (p.E + 31) / 32;
            const int g0 = lane * per;
            int local = 0;
            for (int i = 0; i < per; ++i) {
                const int e = g0 + i;
                if (e < p.E) local += ((p.counts[e] + TROWS - 1) / TROWS) * sc.num_n;
            }
            int incl = local;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += v;
            }
            int run = incl - local;
            for (int i = 0; i < per; ++i) {
                const int e = g0 + i;
                if (e < p.E) {
                    g_tile[e] = run;
                    g_row[e] = p.offsets[e];
                    g_cnt[e] = p.counts[e];
                    run += ((p.counts[e] + TROWS - 1) / TROWS) * sc.num_n;
                }
            }
            if (lane == 31) g_tile[p.E] = incl;
        }
        sc.g_tile = g_tile;
        sc.g_row = g_row;
        sc.g_cnt = g_cnt;
        sc.num_m = 0;
    } else {
        sc.g_tile = nullptr;
        sc.g_row = nullptr;
        sc.g_cnt = nullptr;
        sc.num_m = (p.M + TROWS - 1) / TROWS;
        sc.total = sc.num_m * sc.num_n;
    }
    __syncwarp();
    tc_fence_before();
    if constexpr (CTAS == 2) cluster_sync_all(); else __syncthreads();
    tc_fence_after();
    if constexpr (GROUPED) sc.total = g_tile[p.E];
    const uint32_t tmem_base = *tmem_slot;
    const int kch_total = p.K / 64;             // 64-element chunks per row
    const int num_kb = (kch_total + KCH - 1) / KCH;
    const int first = CTAS == 2 ? static_cast<int>(blockIdx.x / 2) : static_cast<int>(blockIdx.x);
    const int stride = CTAS == 2 ? static_cast<int>(gridDim.x / 2) : static_cast<int>(gridDim.x);

    if (warp == 0) {
        if (lane == 0) {
            // ---------------------------------------------------------- producer
            int stage = 0;
            uint32_t phase = 0;
            uint32_t issued = 0, issued_phase = 0;
            for (int t = first; t < sc.total && !*abort_flag; t += stride) {
                const Tile ti = sc.get(t);
                const int64_t rb_a = ti.a_row0 / ROWS;
                const int64_t rb_b0 = ti.b_base / ROWS;
                // the second 128-row half of B exists only when n0 + 128 < N;
                // otherwise its scale atoms repeat the first half's (the
                // columns it feeds are never stored)
                const int64_t rb_b1 = ti.n0 + ROWS < p.N ? rb_b0 + 1 : rb_b0;
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!mbar_wait(empty(stage), phase ^ 1u, p.timeout_ns, p.status)) {
                        *abort_flag = 1;
                        break;
                    }
                    const int64_t c0 = static_cast<int64_t>(kb) * KCH;
                    const uint32_t sa = smem_u32(smem + L::A_OFF + stage * L::A_STAGE);
                    const uint32_t sb = smem_u32(smem + L::B_OFF + stage * L::B_STAGE);
                    const uint32_t ssa = smem_u32(smem + L::SFA_OFF + stage * SFA_STAGE);
                    const uint32_t ssb = smem_u32(smem + L::SFB_OFF + stage * SFB_STAGE);
                    if constexpr (CTAS == 2) {
                        // whole boxes (4 atoms each, past the last chunk too:
                        // later atoms or zero fill) so that the byte count is fixed
                        const uint32_t fl = mapa_shared(landed(stage), 0);
                        constexpr int RPA = ATOM / SF_ROW;  // 256-byte rows per atom
                        if (leader) mbar_arrive_expect_tx(landed(stage), L::PAIR_TX);
                        tma_load_2d_pair(sa, &tmA, kb * BKB, ti.a_row0, fl);
                        tma_load_2d_pair(sb, &tmB, kb * BKB, ti.b_row0, fl);
                        tma_load_2d_pair(ssa, &tmSFA, 0, static_cast<int32_t>((rb_a * kch_total + c0) * RPA), fl);
                        tma_load_2d_pair(ssb, &tmSFB, 0, static_cast<int32_t>((rb_b0 * kch_total + c0) * RPA), fl);
                        tma_load_2d_pair(ssb + KCH * ATOM, &tmSFB, 0,
                                         static_cast<int32_t>((rb_b1 * kch_total + c0) * RPA), fl);
                    } else {
                        const int nk = min(KCH, kch_total - kb * KCH);
                        const uint32_t sfb = static_cast<uint32_t>(nk * ATOM);
                        mbar_arrive_expect_tx(landed(stage), L::A_STAGE + L::B_STAGE + 3 * sfb);
                        tma_load_2d(sa, &tmA, kb * BKB, ti.a_row0, landed(stage));
                        tma_load_2d(sb, &tmB, kb * BKB, ti.b_row0, landed(stage));
                        bulk_load(ssa, p.sfa + (rb_a * kch_total + c0) * ATOM, sfb, landed(stage));
                        bulk_load(ssb, p.sfb + (rb_b0 * kch_total + c0) * ATOM, sfb, landed(stage));
                        bulk_load(ssb + KCH * ATOM, p.sfb + (rb_b1 * kch_total + c0) * ATOM, sfb, landed(stage));
                    }
                    issued |= 1u << stage;
                    issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
            }
            if (*abort_flag) {
                // let the copies in flight land before the CTA exits (the odd
                // CTA's copies complete on the even CTA's barriers: wait a while)
                if (leader) {
                    for (int s = 0; s < STAGES; ++s)
                        if (issued & (1u << s))
                            mbar_wait(landed(s), (issued_phase >> s) & 1u, p.timeout_ns, p.status);
                } else {
                    const uint64_t t0 = globaltimer_ns();
                    while (globaltimer_ns() - t0 < 100000ull) {}
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            // --------------------------------------------------------- MMA issuer
            int stage = 0;
            uint32_t phase = 0;
            uint32_t acc_phase = 0;
            for (int t = first; t < sc.total && !*abort_flag; t += stride) {
                if (!mbar_wait(tempty, acc_phase ^ 1u, p.timeout_ns, p.status)) {
                    *abort_flag = 1;
                    break;
                }
                tc_fence_after();
                bool ok = true;
                for (int kb = 0; kb < num_kb; ++kb) {
                    if ((GROUPED && !mbar_wait(landed(stage), phase, p.timeout_ns, p.status)) ||
                        !mbar_wait(full(stage), phase, p.timeout_ns, p.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int nk = min(KCH, kch_total - kb * KCH);
                    // this stage's scales, copied into its TMEM buffer by the scale warps
                    const uint32_t sfa_t = tmem_base + SF_COL + SF_BUF * stage;
                    const uint32_t sfb_t = sfa_t + 16;
                    const uint64_t adesc = sw128_kmajor_desc(smem_u32(smem + L::A_OFF + stage * L::A_STAGE));
                    const uint64_t bdesc = sw128_kmajor_desc(smem_u32(smem + L::B_OFF + stage * L::B_STAGE));
#pragma unroll
                    for (int c = 0; c < KCH; ++c) {
                        if (c < nk) {
                            const uint32_t acc = (kb > 0 || c > 0) ? 1u : 0u;
                            if constexpr (CTAS == 2)
                                mma_nvf4_pair(tmem_base, adesc + 2 * c, bdesc + 2 * c, L::IDESC, sfa_t + 4 * c,
                                              sfb_t + 8 * c, acc);
                            else
                                mma_nvf4(tmem_base, adesc + 2 * c, bdesc + 2 * c, L::IDESC, sfa_t + 4 * c,
                                         sfb_t + 8 * c, acc);
                        }
                    }
                    if constexpr (CTAS == 2) mma_commit_pair_mc(empty(stage), 0x3);
                    else mma_commit(empty(stage));
                    if constexpr (GROUPED) {
                        if constexpr (CTAS == 2) mma_commit_pair(sfree(stage));
                        else mma_commit(sfree(stage));
                    }
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) {
                    *abort_flag = 1;
                    break;
                }
                if constexpr (CTAS == 2) mma_commit_pair_mc(tfull, 0x3);
                else mma_commit(tfull);
                acc_phase ^= 1u;
            }
            if constexpr (CTAS == 2) mma_commit_pair(drain);
            else mma_commit(drain);
            mbar_wait(drain, 0, p.timeout_ns, p.status);
        }
    } else if (warp >= SCALE_WARP) {
        const int part = warp - SCALE_WARP;   // chunks [part * KCH / SCALE_WARPS, ...)
        if (lane == 0 && leader) {
            // ------------------------------------------------- scale-factor copies
            // Each stage's scale atoms go into the stage's TMEM scale buffer as
            // soon as the stage has landed (its previous MMAs are then done),
            // so that the copies overlap the MMA thread's work.
            int stage = 0;
            uint32_t phase = 0;
            for (int t = first; t < sc.total && !*abort_flag; t += stride) {
                bool ok = true;
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!mbar_wait(landed(stage), phase, p.timeout_ns, p.status) ||
                        (GROUPED && !mbar_wait(sfree(stage), phase ^ 1u, p.timeout_ns, p.status))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int nk = min(KCH, kch_total - kb * KCH);
                    const uint32_t sfa_t = tmem_base + SF_COL + SF_BUF * stage;
                    const uint32_t sfb_t = sfa_t + 16;
                    const uint32_t sa = smem_u32(smem + L::SFA_OFF + stage * SFA_STAGE);
                    const uint32_t sb = smem_u32(smem + L::SFB_OFF + stage * SFB_STAGE);
#pragma unroll
                    for (int c = 0; c < KCH; ++c) {
                        if (c < nk && c / (KCH / SCALE_WARPS) == part) {
                            if constexpr (CTAS == 2) {
                                sf_copy_pair(sfa_t + 4 * c, sf_atom_desc(sa + c * ATOM));
                                sf_copy_pair(sfb_t + 8 * c, sf_atom_desc(sb + c * ATOM));
                                sf_copy_pair(sfb_t + 8 * c + 4, sf_atom_desc(sb + (KCH + c) * ATOM));
                            } else {
                                sf_copy(sfa_t + 4 * c, sf_atom_desc(sa + c * ATOM));
                                sf_copy(sfb_t + 8 * c, sf_atom_desc(sb + c * ATOM));
                                sf_copy(sfb_t + 8 * c + 4, sf_atom_desc(sb + (KCH + c) * ATOM));
                            }
                        }
                    }
                    if constexpr (CTAS == 2) mma_commit_pair(full(stage));
                    else mma_commit(full(stage));
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) {
                    *abort_flag = 1;
                    break;
                }
            }
            // every copy issued by this thread completes before TMEM is released
            if constexpr (CTAS == 2) mma_commit_pair(sdrain + 8 * part);
            else mma_commit(sdrain + 8 * part);
            mbar_wait(sdrain + 8 * part, 0, p.timeout_ns, p.status);
        }
    } else {
        // -------------------------------------------------------------- epilogue
        const int q = warp & 3;              // TMEM lane quadrant this warp may access
        const int part = (warp - 2) >> 2;    // columns 64 part .. 64 part + 63
        uint8_t* stg = staging + (warp - 2) * (32 * 64);
        uint32_t acc_phase = 0;
        for (int t = first; t < sc.total && !*abort_flag; t += stride) {
            const Tile ti = sc.get(t);
            const int row = ti.a_row0 + q * 32 + lane;
            const float ga = row < ti.row_end ? p.ga[row] : 0.0f;
            const float gb = p.gb[ti.group];
            if (!mbar_wait(tfull, acc_phase, p.timeout_ns, p.status)) {
                *abort_flag = 1;
                break;
            }
            tc_fence_after();
            const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                   static_cast<uint32_t>(part * 64);
            uint32_t va[32], vb[32];
            tmem_ld_32x32b_x32(tbase, va);
            tmem_ld_32x32b_x32(tbase + 32, vb);
            tmem_ld_wait();
            // the whole accumulator has been read by this warp: release it
            // (relaxed: a release would first wait for this warp's stores of
            // the previous tile, holding up the next tile's MMAs)
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if constexpr (CTAS == 2) mbar_arrive_cluster_relaxed(mapa_shared(tempty, 0));
                else mbar_arrive_relaxed(tempty);
            }
            store_chunk(va, 2 * part, ti, q, lane, ga, gb, stg, p.y, p.N, &tmY);
            store_chunk(vb, 2 * part + 1, ti, q, lane, ga, gb, stg, p.y, p.N, &tmY);
            acc_phase ^= 1u;
        }
        // this warp's output stores have completed before the CTA exits
        if (lane == 0) bulk_wait_all();
    }

    __syncwarp();
    tc_fence_before();
    if constexpr (CTAS == 2) cluster_sync_all(); else __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        if constexpr (CTAS == 2) tmem_dealloc_pair(tmem_base, TMEM_COLS);
        else tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

template <int CTAS, bool GROUPED>
int prepare_gemm(const DeviceInfo& di) {
    static std::atomic<uint64_t> done[64];
    const size_t smem = Lay<CTAS, GROUPED>::BYTES;
    if (static_cast<size_t>(di.max_smem_optin) < smem)
        return fail(METIS_ERR_UNSUPPORTED, "nvfp4 gemm needs %zu bytes of shared memory", smem);
    return once_per_context(done, di.device, [&] {
        return cuda_check(cudaFuncSetAttribute(nvfp4_gemm_kernel<CTAS, GROUPED>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               static_cast<int>(smem)),
                          "cudaFuncSetAttribute(nvfp4 gemm)");
    });
}

// Co-resident CTA pairs of the 2-CTA kernel (cached per device).
template <bool GROUPED>
int max_pairs(const DeviceInfo& di, int* out) {
    static int cached[64];
    if (!cached[di.device]) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * (di.num_sms / 2), 1, 1);
        cfg.blockDim = dim3(THREADS, 1, 1);
        cfg.dynamicSmemBytes = Lay<2, GROUPED>::BYTES;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        int rc = cuda_check(cudaOccupancyMaxActiveClusters(&n, nvfp4_gemm_kernel<2, GROUPED>, &cfg),
                            "cudaOccupancyMaxActiveClusters(nvfp4)");
        if (rc) return rc;
        if (n < 1) return fail(METIS_ERR_UNSUPPORTED, "no CTA pair of the nvfp4 gemm fits an SM pair");
        cached[di.device] = n;
    }
    *out = cached[di.device];
    return METIS_OK;
}

}  // namespace nvfp4

// y = NVFP4 GEMM. a_rows: rows of A's code buffer (a multiple of 128);
// b_rows: rows of B ([groups * N]). offsets/counts null: dense with M rows.
// CTA pairs (256-row tiles) for the grouped GEMM and for M > 128.
// Arguments validated by the caller.
int launch_nvfp4_gemm(const uint8_t* qa, const uint8_t* sfa, const float* ga, int64_t a_rows,
                      const uint8_t* qb, const uint8_t* sfb, const float* gb, int64_t b_rows,
                      __nv_bfloat16* y, const int32_t* offsets, const int32_t* counts, int E, int M,
                      int N, int K, cudaStream_t st) {
    using namespace nvfp4;
    DeviceInfo di;
    int rc = current_device_info(&di);
    if (rc) return rc;
    GemmParams p{};
    p.sfa = sfa;
    p.ga = ga;
    p.sfb = sfb;
    p.gb = gb;
    p.y = y;
    p.offsets = offsets;
    p.counts = counts;
    p.M = M;
    p.N = N;
    p.K = K;
    p.E = offsets ? E : 1;
    if ((rc = device_status_word(&p.status))) return rc;
    p.timeout_ns = watchdog_ns();
    const bool grouped = offsets != nullptr;
    const bool pair = grouped || M > ROWS;
    const uint32_t b_box = pair ? BN / 2 : BN;
    CUtensorMap ta, tb, tsa, tsb, ty;
    // y: [M, N] (dense) or one row per row of A (grouped), BF16
    if ((rc = make_tmap_2d_sw64(&ty, y, 2, static_cast<uint64_t>(N), static_cast<uint64_t>(grouped ? a_rows : M),
                                static_cast<uint64_t>(N) * 2, 32, 32)))
        return rc;
    if ((rc = make_tmap_2d(&ta, qa, 1, static_cast<uint64_t>(K / 2), static_cast<uint64_t>(a_rows),
                           static_cast<uint64_t>(K / 2), BKB, ROWS, true)))
        return rc;
    if ((rc = make_tmap_2d(&tb, qb, 1, static_cast<uint64_t>(K / 2), static_cast<uint64_t>(b_rows),
                           static_cast<uint64_t>(K / 2), BKB, b_box, true)))
        return rc;
    // the tiled scales as rows of 256 bytes (two per atom), 4 atoms per box
    if ((rc = make_tmap_2d(&tsa, sfa, 1, SF_ROW, static_cast<uint64_t>(a_rows) * (K / 16) / SF_ROW, SF_ROW,
                           SF_ROW, KCH * ATOM / SF_ROW, false)))
        return rc;
    if ((rc = make_tmap_2d(&tsb, sfb, 1, SF_ROW, static_cast<uint64_t>(b_rows) * (K / 16) / SF_ROW, SF_ROW,
                           SF_ROW, KCH * ATOM / SF_ROW, false)))
        return rc;
    if (pair) {
        int pairs = 0;
        int clusters = 0;
        if (grouped) {
            if ((rc = prepare_gemm<2, true>(di))) return rc;
            if ((rc = max_pairs<true>(di, &pairs))) return rc;
            clusters = pairs;
            return cuda_check(launch_pdl(nvfp4_gemm_kernel<2, true>, dim3(2 * clusters), dim3(THREADS),
                                         Lay<2, true>::BYTES, st, 2, ta, tb, tsa, tsb, ty, p),
                              "nvfp4 grouped gemm (CTA pair) launch");
        }
        if ((rc = prepare_gemm<2, false>(di))) return rc;
        if ((rc = max_pairs<false>(di, &pairs))) return rc;
        const int64_t tiles = ((static_cast<int64_t>(M) + 2 * ROWS - 1) / (2 * ROWS)) * ((N + BN - 1) / BN);
        clusters = static_cast<int>(tiles < pairs ? tiles : pairs);
        return cuda_check(launch_pdl(nvfp4_gemm_kernel<2, false>, dim3(2 * clusters), dim3(THREADS),
                                     Lay<2, false>::BYTES, st, 2, ta, tb, tsa, tsb, ty, p),
                          "nvfp4 gemm (CTA pair) launch");
    }
    const int64_t tiles = ((static_cast<int64_t>(M) + ROWS - 1) / ROWS) * ((N + BN - 1) / BN);
    if (tiles == 0) return METIS_OK;
    const int grid = static_cast<int>(tiles < di.num_sms ? tiles : di.num_sms);
    if ((rc = prepare_gemm<1, false>(di))) return rc;
    return cuda_check(launch_pdl(nvfp4_gemm_kernel<1, false>, dim3(grid), dim3(THREADS), Lay<1, false>::BYTES,
                                 st, 1, ta, tb, tsa, tsb, ty, p),
                      "nvfp4 gemm launch");
}

}  // namespace metis

// ----------------------------------------------------------------- C ABI
using namespace metis;

extern "C" int metis_quant_nvfp4(const void* x, int x_kind, int64_t R, int64_t K, int64_t ldx,
                                 int64_t rows_per_scale, uint8_t* q, uint8_t* sf, int sf_layout,
                                 float* g, metis_stream_t stream) {
    clear_error();
    if (x_kind != METIS_A_BF16 && x_kind != METIS_A_F32)
        return fail(METIS_ERR_INVALID_ARG, "quant_nvfp4: x_kind %d (need METIS_A_BF16 or METIS_A_F32)", x_kind);
    if (sf_layout != METIS_SF_ROWMAJOR && sf_layout != METIS_SF_TILED)
        return fail(METIS_ERR_INVALID_ARG, "quant_nvfp4: sf_layout %d", sf_layout);
    if (R < 0 || R > 0x7fffffffll || K < 64 || K % 64 || K > 65536 || ldx < K)
        return fail(METIS_ERR_INVALID_ARG,
                    "quant_nvfp4: need R >= 0, 64 <= K <= 65536 with K %% 64 == 0, ldx >= K "
                    "(R=%lld K=%lld ldx=%lld)", (long long)R, (long long)K, (long long)ldx);
    if (rows_per_scale < 1 || (R > 0 && R % rows_per_scale))
        return fail(METIS_ERR_INVALID_ARG, "quant_nvfp4: rows_per_scale %lld must divide R=%lld",
                    (long long)rows_per_scale, (long long)R);
    if (R == 0) return METIS_OK;
    if (!x || !q || !sf || !g) return fail(METIS_ERR_INVALID_ARG, "quant_nvfp4: null pointer");
    const int64_t esz = x_kind == METIS_A_BF16 ? 2 : 4;
    if (!aligned(x, 16) || (ldx * esz) % 16 || !aligned(q, 16) || !aligned(sf, 4) || !aligned(g, 4))
        return fail(METIS_ERR_INVALID_ARG,
                    "quant_nvfp4: x and q 16-byte aligned, ldx * element size a multiple of 16, "
                    "sf and g 4-byte aligned");
    DeviceInfo di;
    int rc = current_device_info(&di);
    if (rc) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int tiled = sf_layout == METIS_SF_TILED;
    if (x_kind == METIS_A_BF16)
        return launch_nvfp4_quant(static_cast<const __nv_bfloat16*>(x), R, K, ldx, rows_per_scale, q, sf,
                                  tiled, g, nullptr, 1, nullptr, nullptr, st);
    return launch_nvfp4_quant(static_cast<const float*>(x), R, K, ldx, rows_per_scale, q, sf, tiled, g,
                              nullptr, 1, nullptr, nullptr, st);
}

extern "C" int metis_nvfp4_scales_to_tiled(const uint8_t* sf, int64_t R, int64_t K,
                                           uint8_t* sf_tiled, metis_stream_t stream) {
    clear_error();
    if (R < 0 || R > 0x7fffffffll || K < 64 || K % 64 || K > 65536)
        return fail(METIS_ERR_INVALID_ARG, "nvfp4_scales_to_tiled: need R >= 0 and K a multiple of 64 "
                    "in [64, 65536] (R=%lld K=%lld)", (long long)R, (long long)K);
    if (R == 0) return METIS_OK;
    if (!sf || !sf_tiled) return fail(METIS_ERR_INVALID_ARG, "nvfp4_scales_to_tiled: null pointer");
    if (!aligned(sf, 4) || !aligned(sf_tiled, 4))
        return fail(METIS_ERR_INVALID_ARG, "nvfp4_scales_to_tiled: pointers must be 4-byte aligned");
    const int64_t Rp = (R + 127) / 128 * 128;
    const uint8_t* s_end = sf + R * (K / 16);
    const uint8_t* t_end = sf_tiled + Rp * (K / 16);
    if (sf < t_end && sf_tiled < s_end)
        return fail(METIS_ERR_INVALID_ARG, "nvfp4_scales_to_tiled: the buffers overlap");
    DeviceInfo di;
    int rc = current_device_info(&di);
    if (rc) return rc;
    const int64_t work = Rp * (K / 64);
    nvfp4::nvfp4_tile_scales_kernel<<<static_cast<unsigned>((work + 255) / 256), 256, 0,
                                      static_cast<cudaStream_t>(stream)>>>(sf, R, Rp, K, sf_tiled);
    return cuda_check(cudaGetLastError(), "nvfp4_scales_to_tiled launch");
}

extern "C" int metis_nvfp4_gemm(const uint8_t* qa, const uint8_t* sfa, const float* ga,
                                const uint8_t* qb, const uint8_t* sfb, const float* gb, void* y,
                                int64_t M, int64_t N, int64_t K, metis_stream_t stream) {
    clear_error();
    if (M < 0 || M > (1ll << 30) || N < 128 || N % 128 || N > (1 << 20) || K < 64 || K % 64 || K > 65536)
        return fail(METIS_ERR_INVALID_ARG,
                    "nvfp4_gemm: need M >= 0, N a multiple of 128, K a multiple of 64 in [64, 65536] "
                    "(M=%lld N=%lld K=%lld)", (long long)M, (long long)N, (long long)K);
    if (M == 0) return METIS_OK;
    if (!qa || !sfa || !ga || !qb || !sfb || !gb || !y) return fail(METIS_ERR_INVALID_ARG, "nvfp4_gemm: null pointer");
    if (!aligned(qa, 16) || !aligned(sfa, 16) || !aligned(qb, 16) || !aligned(sfb, 16) || !aligned(y, 16) ||
        !aligned(ga, 4) || !aligned(gb, 4))
        return fail(METIS_ERR_INVALID_ARG, "nvfp4_gemm: codes, tiled scales and y 16-byte aligned");
    const int64_t Mp = (M + 127) / 128 * 128;
    return launch_nvfp4_gemm(qa, sfa, ga, Mp, qb, sfb, gb, N, static_cast<__nv_bfloat16*>(y), nullptr,
                             nullptr, 1, static_cast<int>(M), static_cast<int>(N), static_cast<int>(K),
                             static_cast<cudaStream_t>(stream));
}
