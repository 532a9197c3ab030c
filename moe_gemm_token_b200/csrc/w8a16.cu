// Default-maths weight-only GEMM for decode (M <= 8 tokens):
//   y[m, n] = bf16_rn( s_w[n] * sum_k x[m, k] * D(w[n, k]) ),  FP32 accumulation.
// "Lernex/Metis-1.6-Logos-FP8", "What --fast-math does": by default the FP8
// weights are expanded to 16 bits as they are multiplied, so the weights are
// the only thing rounded; one stream's decode always takes this path because
// its speed is set by how fast the weights are read.
//
// HBM-bound: the N*K weight bytes dominate. One persistent CTA per SM owns a
// contiguous range of 16-row weight tiles, so each weight byte is read from
// HBM exactly once.
//
//  * TMA kernel (K % 64 == 0): a producer thread streams each tile through a
//    3-D view of the weights, {64 bytes, rows (stride K), 64-byte k-groups},
//    one 16 x 16 x 64-byte box (16 KB: 16 rows x a 1024-byte k-window) per
//    ring stage, laid out as one 16-row x 64-byte block per consumer warp,
//    8 stages (128 KB per SM in flight). 16 consumer warps read their box
//    (rows g and g+8, 16 bytes per thread, conflict-free), widen E4M3 to
//    FP16 and issue mma.sync.m16n8k16 with the weights as the M = 16 operand
//    and the <= 8 tokens as n = 8 (four independent FP32 accumulators). For
//    K <= 4096 each thread keeps the x fragments it needs for every k-window
//    in registers (32 registers at K = 4096), so x is read once per CTA and
//    never staged; larger K stages x in shared memory. The rows of W are
//    split over the CTAs in 8-row units (at most 8 rows of imbalance); a
//    CTA walks its rows as 16-row tiles. A reducer warp adds each finished
//    tile's partial sums (double-buffered) and stores it while the stream
//    goes on. Launched as a programmatic dependent: barrier set-up and an L2
//    prefetch of the first 4 stages of weights overlap the previous kernel;
//    x is read, y written and shared memory filled only after the grid
//    dependency is resolved.
//  * register kernel (K % 64 != 0, or when x plus a ring do not fit in
//    shared memory): 16 warps stream 128-byte chunks of the rows straight
//    into registers, 4 chunks in flight per thread.
//
// Both widen with cvt.rn.f16x2.e4m3x2 (exact: every E4M3 value is an FP16
// normal), which measured faster here than placing the E4M3 bits into FP16
// positions with integer operations.
// x is staged as FP16 after an exact per-token power-of-two shift that puts
// the token's amax in [2^14, 2^15): every element within a factor 2^29 of the
// amax keeps its BF16 value exactly, so the products are those of the BF16
// maths; the shift is undone exactly in the epilogue. The warps' partial sums
// meet in shared memory and are added in a fixed order (deterministic).
#include "common.cuh"

namespace metis {
namespace w8a16 {

constexpr int WARPS = 16;             // consumer warps
constexpr int CTHREADS = WARPS * 32;  // consumer threads
constexpr int MAX_K = 12288;


// TMA kernel geometry
constexpr int BOX_K = 64;                   // bytes of K per box (one consumer warp)
constexpr int WIN = WARPS * BOX_K;          // k-window per stage: 1024
constexpr int STAGE_BYTES = 16 * WIN;       // 16 rows x 1024 = 16 KB
// Ring depth and L2 warm-up: measured on B200 (K = 4096, N = 14336, cold
// weights, calls back to back), 8 stages with the first 4 prefetched beat
// deeper rings (12 stages: +1 us) and prefetching a CTA's whole range (+3 us).
constexpr int MAX_STAGES = 8;
constexpr int L2_PREFETCH = 4;

constexpr int MISC_BYTES = 128 + WARPS * 8 * 4;
constexpr int MAX_REG_KWIN = 4;             // x held in registers up to K = 4096

// register kernel geometry
constexpr int DEPTH = 4;    // chunks in flight per thread
constexpr int CHUNK = 128;  // bytes of K per row per chunk

__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// Two E4M3 byte pairs of w, (0,1) and (2,3), to two FP16 pairs (exact).
__device__ __forceinline__ void cvt_pairs(uint32_t w, uint32_t& lo, uint32_t& hi) {
    asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, l;\n\tcvt.rn.f16x2.e4m3x2 %1, h;\n\t}"
        : "=r"(lo), "=r"(hi)
        : "r"(w));
}

__device__ __forceinline__ void mma_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, "
        "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// 16 rows x 16 bytes of K (rows g and g + 8 of this thread: words A, B)
// against the thread's x fragment (8 words, 4 k-steps), into acc[4].
__device__ __forceinline__ void piece_mma(float (&acc)[4][4], const uint4& A, const uint4& B,
                                          const uint4& xa, const uint4& xc) {
    const uint32_t wa[4] = {A.x, A.y, A.z, A.w};
    const uint32_t wb[4] = {B.x, B.y, B.z, B.w};
    const uint32_t bx[8] = {xa.x, xa.y, xa.z, xa.w, xc.x, xc.y, xc.z, xc.w};
#pragma unroll
    for (int s = 0; s < 4; ++s) {
        uint32_t a0, a1, a2, a3;
        cvt_pairs(wa[s], a0, a2);
        cvt_pairs(wb[s], a1, a3);
        mma_16816(acc[s], a0, a1, a2, a3, bx[2 * s], bx[2 * s + 1]);
    }
}

struct Args {
    const __nv_bfloat16* x;
    const uint8_t* w;
    const float* s_w;
    __nv_bfloat16* y;
    int M, N, K;
    int KP;       // K rounded up to the k-range the warps visit (zero-padded in x)
    int cpw;      // register kernel: 128-byte chunks per warp per tile
    int tiles;    // ceil(N / 16)
    int units;    // TMA kernel: ceil(N / 8), split evenly over the CTAs
    int max_tpc;  // max tiles per CTA (sizes the partial-sum buffer)
    int stages;   // TMA kernel: ring stages
    int wlayout;  // TMA kernel box layout: 0 = [k-group][row][64 B], 1 = [row][k-group][64 B]
    uint32_t* status;
    uint64_t timeout_ns;
};

// Shared-memory layout common to both kernels (byte offsets).
struct Smem {
    int xpitch;    // bytes per staged x row (2 * KP + 16: 16 mod 128 -> conflict-free)
    int x_off;     // [M][xpitch] FP16
    int misc_off;  // unshift[8] f32, shift/amax[8], pow2[8], per-warp amax [16][8]
    int part_off;  // [part_tiles][16 warps][32 lanes][4] f32
    int ring_off;  // TMA ring
    int bar_off;   // full[stages], empty[stages], tfull[2], tfree[2]
    int total;
};

// x_rows = 0: x is not staged in shared memory (the register-resident path).
__host__ __device__ inline Smem smem_layout(int x_rows, int KP, int part_tiles, int stages) {
    Smem s;
    s.xpitch = 2 * KP + 16;
    s.x_off = 0;
    s.misc_off = x_rows * s.xpitch;  // 16-byte aligned
    s.part_off = s.misc_off + MISC_BYTES;
    s.ring_off = s.part_off + part_tiles * WARPS * 32 * 16;
    s.ring_off = (s.ring_off + 127) & ~127;  // TMA destination alignment
    s.bar_off = s.ring_off + stages * STAGE_BYTES;
    s.total = s.bar_off + (2 * stages + 4) * 8;
    return s;
}

// Stages x [M][K] BF16 into shared memory as FP16 rows of KP elements
// (zero-padded) with the per-token power-of-two shift.
// Executed by the CTHREADS consumer threads, synchronised on named barrier 1
// (no other thread takes part, and nothing here waits on an mbarrier). When
// all of x fits in the threads' registers (M*K <= 32768) each element is
// read once from global memory and written once to shared memory.
__device__ __forceinline__ void widen8(const uint4& raw, int sh, float p2, uint4& out) {
    const uint32_t wv[4] = {raw.x, raw.y, raw.z, raw.w};
    float f[8];
    if (p2 != 0.0f) {  // 2^sh is a binary32: one exact multiply per element
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            f[2 * j] = bf16_lo(wv[j]) * p2;
            f[2 * j + 1] = bf16_hi(wv[j]) * p2;
        }
    } else {  // extreme token magnitudes only
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            f[2 * j] = ldexpf(bf16_lo(wv[j]), sh);
            f[2 * j + 1] = ldexpf(bf16_hi(wv[j]), sh);
        }
    }
    const __half2 h0 = __floats2half2_rn(f[0], f[1]);
    const __half2 h1 = __floats2half2_rn(f[2], f[3]);
    const __half2 h2 = __floats2half2_rn(f[4], f[5]);
    const __half2 h3 = __floats2half2_rn(f[6], f[7]);
    out = make_uint4(*reinterpret_cast<const uint32_t*>(&h0), *reinterpret_cast<const uint32_t*>(&h1),
                     *reinterpret_cast<const uint32_t*>(&h2), *reinterpret_cast<const uint32_t*>(&h3));
}

__device__ __forceinline__ void stage_x(const Args& a, uint8_t* smem, const Smem& L, int tid) {
    uint8_t* xs = smem + L.x_off;
    float* unshift = reinterpret_cast<float*>(smem + L.misc_off);
    unsigned* row_amax = reinterpret_cast<unsigned*>(smem + L.misc_off + 32);
    int* shift = reinterpret_cast<int*>(smem + L.misc_off + 32);  // replaces row_amax
    float* pow2 = reinterpret_cast<float*>(smem + L.misc_off + 64);
    const int lane = tid & 31;
    constexpr int XB = 8;
    const int kc = a.K / 8;
    const int xchunks = a.M * kc;
    const bool in_regs = xchunks <= XB * CTHREADS;
    if (tid < 8) row_amax[tid] = 0u;
    uint4 xb[XB];
#pragma unroll
    for (int j = 0; j < XB; ++j) {
        const int c = tid + CTHREADS * j;
        xb[j] = c < xchunks ? *reinterpret_cast<const uint4*>(a.x + static_cast<size_t>(c) * 8)
                            : make_uint4(0, 0, 0, 0);
    }
    named_barrier(1, CTHREADS);
    for (int j0 = 0; j0 * CTHREADS < xchunks; j0 += XB) {
#pragma unroll
        for (int j = 0; j < XB; ++j) {
            const int c = tid + CTHREADS * (j0 + j);
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
                if (!in_regs) {
                    const int k = (c - m * kc) * 8;
                    *reinterpret_cast<uint4*>(xs + m * L.xpitch + 2 * k) = xb[j];
                }
            }
        }
    }
    named_barrier(1, CTHREADS);
    if (tid < 8) {
        const float amax = __uint_as_float(row_amax[tid]);
        const int sh = amax > 0.0f ? 14 - ilogbf(amax) : 0;
        shift[tid] = sh;
        unshift[tid] = ldexpf(1.0f, -sh);
        // 2^sh as a binary32 when representable (the common case), else 0:
        // the widening then falls back to ldexpf for that token
        pow2[tid] = (sh >= -126 && sh <= 127) ? __uint_as_float(static_cast<uint32_t>(sh + 127) << 23) : 0.0f;
    }
    named_barrier(1, CTHREADS);
    const int kpc = a.KP / 8;
    if (in_regs) {
        // widen the chunks held in registers; then zero the padding [K, KP)
#pragma unroll
        for (int j = 0; j < XB; ++j) {
            const int c = tid + CTHREADS * j;
            if (c < xchunks) {
                const int m = c / kc;
                const int k = (c - m * kc) * 8;
                uint4 out;
                widen8(xb[j], shift[m], pow2[m], out);
                *reinterpret_cast<uint4*>(xs + m * L.xpitch + 2 * k) = out;
            }
        }
        const int pad = kpc - kc;
        for (int c = tid; c < a.M * pad; c += CTHREADS) {
            const int m = c / pad;
            const int k = a.K + (c - m * pad) * 8;
            *reinterpret_cast<uint4*>(xs + m * L.xpitch + 2 * k) = make_uint4(0, 0, 0, 0);
        }
    } else {
        for (int c = tid; c < a.M * kpc; c += CTHREADS) {
            const int m = c / kpc;
            const int k = (c - m * kpc) * 8;
            uint4* p = reinterpret_cast<uint4*>(xs + m * L.xpitch + 2 * k);
            uint4 out = make_uint4(0, 0, 0, 0);
            if (k < a.K) widen8(*p, shift[m], pow2[m], out);
            *p = out;
        }
    }
    named_barrier(1, CTHREADS);
}

// The thread's x fragment for 16 k starting at element k0 (4 k-steps): rows
// g >= M of the token operand are zero.
__device__ __forceinline__ void load_x(const uint8_t* xs_row, bool row_ok, int k0, uint4& xa,
                                       uint4& xc) {
    if (row_ok) {
        xa = *reinterpret_cast<const uint4*>(xs_row + 2 * k0);
        xc = *reinterpret_cast<const uint4*>(xs_row + 2 * k0 + 16);
    } else {
        xa = xc = make_uint4(0, 0, 0, 0);
    }
}

__device__ __forceinline__ void flush(float (&acc)[4][4], float* partial, int ct, int warp,
                                      int lane) {
    float4 v;
    v.x = (acc[0][0] + acc[1][0]) + (acc[2][0] + acc[3][0]);
    v.y = (acc[0][1] + acc[1][1]) + (acc[2][1] + acc[3][1]);
    v.z = (acc[0][2] + acc[1][2]) + (acc[2][2] + acc[3][2]);
    v.w = (acc[0][3] + acc[1][3]) + (acc[2][3] + acc[3][3]);
    reinterpret_cast<float4*>(partial)[(ct * WARPS + warp) * 32 + lane] = v;
#pragma unroll
    for (int s = 0; s < 4; ++s) acc[s][0] = acc[s][1] = acc[s][2] = acc[s][3] = 0.f;
}

// Fixed-order reduction of the warps' partial sums, scale, round, store.
__device__ __forceinline__ void reduce_store(const Args& a, const uint8_t* smem, const Smem& L,
                                             int t0, int ntl, int tid) {
    const float* partial = reinterpret_cast<const float*>(smem + L.part_off);
    const float* unshift = reinterpret_cast<const float*>(smem + L.misc_off);
    const int per_tok = ntl * 16;
    for (int idx = tid; idx < per_tok * a.M; idx += CTHREADS) {
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
        const float v = __fmul_rn(__fmul_rn(sum, unshift[m]), a.s_w[n]);
        a.y[static_cast<size_t>(m) * a.N + n] = __float2bfloat16_rn(v);
    }
}

// ------------------------------------------------------------- TMA kernel

constexpr int TMA_THREADS = CTHREADS + 64;  // + producer warp + reducer warp

// x fragments of this thread held in registers, KWIN k-windows: token g,
// elements kw * 1024 + warp * 64 + 16 t + [0, 16) as FP16 after the
// per-token power-of-two shift (the same shift as stage_x). The per-token
// amax comes from the four lanes that share g and a per-warp table in shared
// memory (one named barrier over the consumer threads).
template <int KWIN>
__device__ __forceinline__ void x_to_regs(const Args& a, uint8_t* smem, const Smem& L, int warp,
                                          int lane, uint32_t (&xr)[KWIN][8]) {
    const int g = lane >> 2, t = lane & 3;
    float* unshift = reinterpret_cast<float*>(smem + L.misc_off);
    unsigned* wmax = reinterpret_cast<unsigned*>(smem + L.misc_off + 128);  // [16 warps][8]
    uint4 raw[KWIN][2];
    float mx = 0.0f;
#pragma unroll
    for (int kw = 0; kw < KWIN; ++kw) {
        const int k0 = kw * WIN + warp * BOX_K + 16 * t;
        if (g < a.M && k0 < a.K) {
            const uint4* p = reinterpret_cast<const uint4*>(a.x + static_cast<size_t>(g) * a.K + k0);
            raw[kw][0] = p[0];
            raw[kw][1] = p[1];
        } else {
            raw[kw][0] = raw[kw][1] = make_uint4(0, 0, 0, 0);
        }
    }
#pragma unroll
    for (int kw = 0; kw < KWIN; ++kw)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint32_t wv[4] = {raw[kw][h].x, raw[kw][h].y, raw[kw][h].z, raw[kw][h].w};
#pragma unroll
            for (int i = 0; i < 4; ++i) mx = fmaxf(mx, fmaxf(fabsf(bf16_lo(wv[i])), fabsf(bf16_hi(wv[i]))));
        }
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    if (t == 0) wmax[warp * 8 + g] = __float_as_uint(mx);
    named_barrier(1, CTHREADS);
    unsigned am = 0;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) am = max(am, wmax[w * 8 + g]);
    const float amax = __uint_as_float(am);
    const int sh = amax > 0.0f ? 14 - ilogbf(amax) : 0;
    const float p2 = (sh >= -126 && sh <= 127) ? __uint_as_float(static_cast<uint32_t>(sh + 127) << 23) : 0.0f;
    if (warp == 0 && t == 0) unshift[g] = ldexpf(1.0f, -sh);
#pragma unroll
    for (int kw = 0; kw < KWIN; ++kw)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            uint4 out;
            widen8(raw[kw][h], sh, p2, out);
            xr[kw][4 * h] = out.x;
            xr[kw][4 * h + 1] = out.y;
            xr[kw][4 * h + 2] = out.z;
            xr[kw][4 * h + 3] = out.w;
        }
}

// KWIN > 0: K <= KWIN * 1024 and x lives in registers; KWIN == 0: any K up
// to MAX_K, x staged in shared memory. Each CTA owns the rows
// [8 u0, 8 u1) of W (8-row units split evenly over the grid), walked as
// 16-row tiles; rows past 8 u1 that the last tile loads are not stored.
template <int KWIN>
__global__ void __launch_bounds__(TMA_THREADS, 1)
w8a16_tma_kernel(const __grid_constant__ CUtensorMap tmW, const Args a) {
    extern __shared__ __align__(128) uint8_t smem[];
    const Smem L = smem_layout(KWIN > 0 ? 0 : a.M, a.KP, 2, a.stages);
    uint8_t* ring = smem + L.ring_off;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bar_off);
    const int S = a.stages;
    auto full = [&](int s) { return smem_u32(&bars[s]); };
    auto empty = [&](int s) { return smem_u32(&bars[S + s]); };
    auto tfull = [&](int b) { return smem_u32(&bars[2 * S + b]); };
    auto tfree = [&](int b) { return smem_u32(&bars[2 * S + 2 + b]); };

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const int u0 = static_cast<int>(static_cast<int64_t>(blockIdx.x) * a.units / gridDim.x);
    const int u1 = static_cast<int>(static_cast<int64_t>(blockIdx.x + 1) * a.units / gridDim.x);
    const int row0 = 8 * u0;                             // first row of this CTA
    const int row_end = 8 * u1 < a.N ? 8 * u1 : a.N;     // rows it stores
    const int ntl = (u1 - u0 + 1) / 2;                   // 16-row tiles
    const int kwin = a.KP / WIN;    // k-windows per tile
    const int nstage = ntl * kwin;  // stages this CTA streams
    auto box_coords = [&](int i, int& x, int& y, int& z) {
        const int tl = i / kwin;
        const int kw = i - tl * kwin;
        x = 0;
        y = a.wlayout == 0 ? row0 + 16 * tl : kw * WARPS;
        z = a.wlayout == 0 ? kw * WARPS : row0 + 16 * tl;
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full(s), 1);
            mbar_init(empty(s), WARPS);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull(b), WARPS);
            mbar_init(tfree(b), 1);
        }
        fence_mbar_init();
        tma_prefetch_desc(&tmW);
    }
    __syncthreads();
    grid_launch_dependents();

    if (warp == WARPS) {
        // ---------------------------------------------------------- producer
        // Warm L2 with the first ring's worth of weights while the previous
        // kernel may still run (a prefetch reads through the coherent L2, so
        // it is safe whatever that kernel writes), then stream into shared
        // memory once the grid dependency is resolved. Consumers wait for
        // every stage issued here before the CTA ends.
        if (lane == 0) {
            for (int i = 0; i < nstage && i < S && i < L2_PREFETCH; ++i) {
                int x, y, z;
                box_coords(i, x, y, z);
                tma_prefetch_l2_3d(&tmW, x, y, z);
            }
            grid_dependency_wait();
            int s = 0;
            uint32_t ph = 0;
            for (int i = 0; i < nstage; ++i) {
                if (!mbar_wait(empty(s), ph ^ 1u, a.timeout_ns, a.status)) break;
                mbar_arrive_expect_tx(full(s), STAGE_BYTES);
                int x, y, z;
                box_coords(i, x, y, z);
                tma_load_3d(smem_u32(ring + s * STAGE_BYTES), &tmW, x, y, z, full(s));
                if (++s == S) { s = 0; ph ^= 1u; }
            }
        }
        return;
    }
    if (warp == WARPS + 1) {
        // ----------------------------------------------------------- reducer
        // Adds the 16 warps' partial sums of each finished tile in a fixed
        // order, scales, rounds and stores it; frees the partial buffer.
        grid_dependency_wait();
        const float* partial = reinterpret_cast<const float*>(smem + L.part_off);
        const float* unshift = reinterpret_cast<const float*>(smem + L.misc_off);
        for (int tl = 0; tl < ntl; ++tl) {
            const int b = tl & 1;
            if (!mbar_wait(tfull(b), (tl >> 1) & 1u, a.timeout_ns, a.status)) break;
            const float* pb = partial + b * WARPS * 32 * 4;
            for (int o = lane; o < 16 * a.M; o += 32) {
                const int m = o >> 4;
                const int row = o & 15;
                const int n = row0 + 16 * tl + row;
                const int ln = (row & 7) * 4 + (m >> 1);
                const int comp = (row >> 3) * 2 + (m & 1);
                const float* src = pb + ln * 4 + comp;
                float sum = 0.f;
#pragma unroll
                for (int w = 0; w < WARPS; ++w) sum += src[w * 32 * 4];
                if (n < row_end) {
                    const float v = __fmul_rn(__fmul_rn(sum, unshift[m]), a.s_w[n]);
                    a.y[static_cast<size_t>(m) * a.N + n] = __float2bfloat16_rn(v);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(tfree(b));
        }
        return;
    }

    // -------------------------------------------------------------- consumers
    const int tid = threadIdx.x;
    grid_dependency_wait();
    const int g = lane >> 2, t = lane & 3;
    float* partial = reinterpret_cast<float*>(smem + L.part_off);
    float acc[4][4];
#pragma unroll
    for (int s = 0; s < 4; ++s) acc[s][0] = acc[s][1] = acc[s][2] = acc[s][3] = 0.f;
    const uint8_t* box0 = ring + 16 * t + (a.wlayout == 0 ? warp * 16 * BOX_K + g * BOX_K : g * WIN + warp * BOX_K);
    const int rstep = a.wlayout == 0 ? 8 * BOX_K : 8 * WIN;  // rows g -> g + 8
    int s = 0;
    uint32_t ph = 0;
    // one ring stage: this warp's 16 x 64-byte block into registers, slot freed
    auto take = [&](uint4& A, uint4& B) -> bool {
        if (!mbar_wait(full(s), ph, a.timeout_ns, a.status)) return false;
        const uint8_t* box = box0 + s * STAGE_BYTES;
        A = *reinterpret_cast<const uint4*>(box);
        B = *reinterpret_cast<const uint4*>(box + rstep);
        __syncwarp();
        if (lane == 0) mbar_arrive(empty(s));
        if (++s == S) { s = 0; ph ^= 1u; }
        return true;
    };
    // a finished tile: partial sums to the reducer (double-buffered)
    auto tile_done = [&](int ct) -> bool {
        const int b = ct & 1;
        if (!mbar_wait(tfree(b), ((ct >> 1) & 1u) ^ 1u, a.timeout_ns, a.status)) return false;
        flush(acc, partial + b * WARPS * 32 * 4, 0, warp, lane);
        __syncwarp();
        if (lane == 0) mbar_arrive(tfull(b));
        return true;
    };
    if constexpr (KWIN > 0) {
        uint32_t xr[KWIN][8];
        x_to_regs<KWIN>(a, smem, L, warp, lane, xr);
        bool ok = true;
        for (int ct = 0; ct < ntl && ok; ++ct) {
#pragma unroll
            for (int kw = 0; kw < KWIN; ++kw) {
                uint4 A, B;
                if (!take(A, B)) { ok = false; break; }
                piece_mma(acc, A, B, make_uint4(xr[kw][0], xr[kw][1], xr[kw][2], xr[kw][3]),
                          make_uint4(xr[kw][4], xr[kw][5], xr[kw][6], xr[kw][7]));
            }
            if (ok) ok = tile_done(ct);
        }
    } else {
        stage_x(a, smem, L, tid);
        const uint8_t* xrow = smem + L.x_off + g * L.xpitch;
        const bool xok = g < a.M;
        bool ok = true;
        for (int ct = 0; ct < ntl && ok; ++ct) {
            for (int kw = 0; kw < kwin; ++kw) {
                uint4 A, B;
                if (!take(A, B)) { ok = false; break; }
                uint4 xa, xc;
                load_x(xrow, xok, kw * WIN + warp * BOX_K + 16 * t, xa, xc);
                piece_mma(acc, A, B, xa, xc);
            }
            if (ok) ok = tile_done(ct);
        }
    }
}

// -------------------------------------------------------- register kernel

__global__ void __launch_bounds__(CTHREADS, 1) w8a16_reg_kernel(const Args a) {
    extern __shared__ __align__(128) uint8_t smem[];
    const Smem L = smem_layout(a.M, a.KP, a.max_tpc, 0);
    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const int g = lane >> 2;
    const int t = lane & 3;
    const int t0 = static_cast<int>(static_cast<int64_t>(blockIdx.x) * a.tiles / gridDim.x);
    const int t1 = static_cast<int>(static_cast<int64_t>(blockIdx.x + 1) * a.tiles / gridDim.x);
    const int ntl = t1 - t0;
    const int cpw = a.cpw;
    const int units = ntl * cpw;

    // load-side cursor over units (tile lt, chunk slot li) of this warp; a
    // thread reads bytes [16t, 16t+16) and [64+16t, 64+16t+16) of its chunk
    // in rows g and g + 8
    const uint32_t K = static_cast<uint32_t>(a.K);
    const uint8_t* wbase = a.w + static_cast<size_t>(t0 * 16 + g) * K;
    uint32_t lo = warp * CHUNK + 16 * t;
    int li = 0, lt = 0;
    const int iv0 = (a.K - warp * CHUNK - 16 * t + 16 * CHUNK - 1) / (16 * CHUNK);
    const int iv1 = (a.K - warp * CHUNK - 64 - 16 * t + 16 * CHUNK - 1) / (16 * CHUNK);
    bool r0ok = t0 * 16 + g < a.N, r1ok = t0 * 16 + g + 8 < a.N;
    auto load_next = [&](uint4 (&A)[2], uint4 (&B)[2]) {
        A[0] = A[1] = B[0] = B[1] = make_uint4(0, 0, 0, 0);
        if (lt < ntl) {
            const uint8_t* p = wbase + lo;
            if (li < iv0) {
                if (r0ok) A[0] = ld_stream_v4(p);
                if (r1ok) B[0] = ld_stream_v4(p + 8 * K);
            }
            if (li < iv1) {
                if (r0ok) A[1] = ld_stream_v4(p + 64);
                if (r1ok) B[1] = ld_stream_v4(p + 64 + 8 * K);
            }
            lo += 16 * CHUNK;
            if (++li == cpw) {
                li = 0;
                ++lt;
                lo += 16 * K - static_cast<uint32_t>(cpw) * 16 * CHUNK;
                r0ok = (t0 + lt) * 16 + g < a.N;
                r1ok = (t0 + lt) * 16 + g + 8 < a.N;
            }
        }
    };
    uint4 ra[DEPTH][2], rb[DEPTH][2];
#pragma unroll
    for (int d = 0; d < DEPTH; ++d) load_next(ra[d], rb[d]);

    stage_x(a, smem, L, threadIdx.x);
    const uint8_t* xrow = smem + L.x_off + g * L.xpitch;
    const bool xok = g < a.M;
    float* partial = reinterpret_cast<float*>(smem + L.part_off);
    float acc[4][4];
#pragma unroll
    for (int s = 0; s < 4; ++s) acc[s][0] = acc[s][1] = acc[s][2] = acc[s][3] = 0.f;
    int k0 = warp * CHUNK + 16 * t;  // element offset of this thread's first piece
    int ci = 0, ct = 0;
    for (int u0 = 0; u0 < units; u0 += DEPTH) {
#pragma unroll
        for (int d = 0; d < DEPTH; ++d) {
            if (u0 + d < units) {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint4 xa, xc;
                    load_x(xrow, xok, k0 + 64 * h, xa, xc);
                    piece_mma(acc, ra[d][h], rb[d][h], xa, xc);
                }
                load_next(ra[d], rb[d]);
                k0 += 16 * CHUNK;
                if (++ci == cpw) {
                    flush(acc, partial, ct, warp, lane);
                    ci = 0;
                    ++ct;
                    k0 -= cpw * 16 * CHUNK;
                }
            }
        }
    }
    __syncthreads();
    reduce_store(a, smem, L, t0, ntl, threadIdx.x);
}

}  // namespace w8a16
}  // namespace metis

using namespace metis;

extern "C" int metis_w8a16_gemm(const void* x_bf16, const uint8_t* wq, const float* s_w,
                                void* y_bf16, int64_t M, int64_t N, int64_t K,
                                metis_stream_t stream) {
    using namespace w8a16;
    clear_error();
    if (M < 1 || M > 0x7fffffff)
        return fail(METIS_ERR_INVALID_ARG, "w8a16_gemm: M=%lld, need M >= 1", (long long)M);
    if (M > 8) {
        // many tokens: the tensor-core path (weights widened into TMEM)
        if (N < 8 || N % 8 != 0 || N > 0x7fffffff || K < 16 || K % 16 != 0 || K > 0x7fffffff)
            return fail(METIS_ERR_INVALID_ARG,
                        "w8a16_gemm (M > 8): need N >= 8 with N %% 8 == 0, K >= 16 with K %% 16 == 0 "
                        "(N=%lld K=%lld)", (long long)N, (long long)K);
        if (!x_bf16 || !wq || !s_w || !y_bf16) return fail(METIS_ERR_INVALID_ARG, "w8a16_gemm: null pointer");
        if (!aligned(x_bf16, 16) || !aligned(wq, 16) || !aligned(s_w, 4) || !aligned(y_bf16, 16))
            return fail(METIS_ERR_INVALID_ARG, "w8a16_gemm (M > 8): x, wq and y must be 16-byte aligned");
        return launch_w8a16_tensor(static_cast<const __nv_bfloat16*>(x_bf16), wq, s_w,
                                   static_cast<__nv_bfloat16*>(y_bf16), static_cast<int>(M), static_cast<int>(N),
                                   static_cast<int>(K), static_cast<cudaStream_t>(stream));
    }
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
    static std::atomic<uint64_t> attr_done[64];
    rc = once_per_context(attr_done, di.device, [&] {
        const int sm = di.max_smem_optin;
        const cudaError_t es[6] = {
            cudaFuncSetAttribute(w8a16_tma_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm),
            cudaFuncSetAttribute(w8a16_tma_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm),
            cudaFuncSetAttribute(w8a16_tma_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm),
            cudaFuncSetAttribute(w8a16_tma_kernel<3>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm),
            cudaFuncSetAttribute(w8a16_tma_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm),
            cudaFuncSetAttribute(w8a16_reg_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, sm)};
        for (cudaError_t e : es)
            if (int r = cuda_check(e, "cudaFuncSetAttribute(w8a16)")) return r;
        return 0;
    });
    if (rc) return rc;
    uint32_t* status = nullptr;
    if ((rc = device_status_word(&status))) return rc;
    Args a;
    a.x = static_cast<const __nv_bfloat16*>(x_bf16);
    a.w = wq;
    a.s_w = s_w;
    a.y = static_cast<__nv_bfloat16*>(y_bf16);
    a.M = static_cast<int>(M);
    a.N = static_cast<int>(N);
    a.K = static_cast<int>(K);
    a.tiles = static_cast<int>((N + 15) / 16);
    a.status = status;
    a.timeout_ns = watchdog_ns();
    const int budget = di.max_smem_optin;
    cudaStream_t st = static_cast<cudaStream_t>(stream);

    // TMA path (K % 64 == 0, so the 3-D view never reaches past a row): x rows
    // cover whole 1024-byte windows; as many ring stages (12 down to 3) as fit
    a.KP = static_cast<int>((K + WIN - 1) / WIN) * WIN;
    a.cpw = 0;
    if (K % BOX_K == 0) {
        // one CTA per SM; the deepest ring (12 down to 3 stages) that fits next
        // to x and the double-buffered partial sums
        // x in registers for K <= 4096 (KWIN k-windows), else staged
        const int kwin_reg = a.KP / WIN <= MAX_REG_KWIN ? a.KP / WIN : 0;
        a.units = static_cast<int>((N + 7) / 8);
        const int grid = a.units < di.num_sms ? a.units : di.num_sms;
        const int x_rows = kwin_reg > 0 ? 0 : a.M;
        int stages = MAX_STAGES;
        Smem L = smem_layout(x_rows, a.KP, 2, stages);
        while (L.total > budget && stages > 3) L = smem_layout(x_rows, a.KP, 2, --stages);
        if (L.total <= budget) {
            a.max_tpc = 0;
            a.stages = stages;
            // preferred view {64 B, rows, k-groups}: the box lands as one 16-row
            // block per consumer warp (conflict-free reads); if the encoder wants
            // monotonic strides, the view {64 B, k-groups, rows} (row-major box)
            CUtensorMap tm;
            a.wlayout = 0;
            if (make_tmap_3d_u8(&tm, wq, BOX_K, static_cast<uint64_t>(N), static_cast<uint64_t>(K / BOX_K),
                                static_cast<uint64_t>(K), BOX_K, BOX_K, 16, WARPS) != METIS_OK) {
                clear_error();
                a.wlayout = 1;
                if ((rc = make_tmap_3d_u8(&tm, wq, BOX_K, static_cast<uint64_t>(K / BOX_K),
                                          static_cast<uint64_t>(N), BOX_K, static_cast<uint64_t>(K),
                                          BOX_K, WARPS, 16)))
                    return rc;
            }
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(grid, 1, 1);
            cfg.blockDim = dim3(TMA_THREADS, 1, 1);
            cfg.dynamicSmemBytes = L.total;
            cfg.stream = st;
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
            attr[0].val.programmaticStreamSerializationAllowed = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            cudaError_t e;
            switch (kwin_reg) {
                case 1: e = cudaLaunchKernelEx(&cfg, w8a16_tma_kernel<1>, tm, a); break;
                case 2: e = cudaLaunchKernelEx(&cfg, w8a16_tma_kernel<2>, tm, a); break;
                case 3: e = cudaLaunchKernelEx(&cfg, w8a16_tma_kernel<3>, tm, a); break;
                case 4: e = cudaLaunchKernelEx(&cfg, w8a16_tma_kernel<4>, tm, a); break;
                default: e = cudaLaunchKernelEx(&cfg, w8a16_tma_kernel<0>, tm, a); break;
            }
            return cuda_check(e, "w8a16 launch");
        }
    }
    // register path
    a.cpw = static_cast<int>(((K + CHUNK - 1) / CHUNK + WARPS - 1) / WARPS);
    a.KP = a.cpw * WARPS * CHUNK;
    a.stages = 0;
    int grid = a.tiles < di.num_sms ? a.tiles : di.num_sms;
    int max_tpc = (a.tiles + grid - 1) / grid;
    Smem L = smem_layout(a.M, a.KP, max_tpc, 0);
    while (L.total > budget && max_tpc > 1) {
        ++grid;
        max_tpc = (a.tiles + grid - 1) / grid;
        L = smem_layout(a.M, a.KP, max_tpc, 0);
    }
    if (L.total > budget) return fail(METIS_ERR_UNSUPPORTED, "w8a16_gemm: K too large");
    a.max_tpc = max_tpc;
    w8a16_reg_kernel<<<grid, CTHREADS, L.total, st>>>(a);
    return cuda_check(cudaGetLastError(), "w8a16 launch");
}
