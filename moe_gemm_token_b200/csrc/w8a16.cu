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
//    ring stage, laid out as one 16-row x 64-byte block per consumer warp;
//    6 stages keep ~100 KB per SM in flight without occupying registers. 16 consumer
//    warps read their box (rows g and g+8, 16 bytes per thread, conflict-free),
//    widen E4M3 to FP16 and issue mma.sync.m16n8k16 with the weights as the
//    M = 16 operand and the <= 8 tokens as n = 8 (four independent FP32
//    accumulators).
//  * register kernel (K % 64 != 0, or when x plus a ring do not fit in
//    shared memory): 16 warps stream 128-byte chunks of the rows straight
//    into registers, 4 chunks in flight per thread.
//
// Both widen exactly (every E4M3 value is an FP16 normal):
//    CONV_CVT   cvt.rn.f16x2.e4m3x2 on byte pairs (0,1) and (2,3);
//    CONV_PLACE the E4M3 bits placed directly in FP16 bit positions, which is
//               exactly the value times 2^-8 (FP16 bias 15, E4M3 bias 7; both
//               subnormal ranges scale alike), the 2^8 folded into the
//               epilogue; bytes (0,2) and (1,3) form the pairs, so x is staged
//               with k permuted 0,2,1,3 inside every group of four.
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
enum Conv { CONV_CVT = 0, CONV_PLACE = 1 };
int g_conv = CONV_CVT;
int g_layout = -1;  // -1: preferred view if the encoder accepts it, else 1; 0/1: forced

// TMA kernel geometry
constexpr int TMA_THREADS = CTHREADS + 32;  // + producer warp
constexpr int BOX_K = 64;                   // bytes of K per box (one consumer warp)
constexpr int WIN = WARPS * BOX_K;          // k-window per stage: 1024
constexpr int STAGE_BYTES = 16 * WIN;       // 16 rows x 1024 = 16 KB

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

// E4M3 bytes (b0, b2) resp. (b1, b3) of q as an FP16 pair equal to value * 2^-8.
__device__ __forceinline__ uint32_t place_even(uint32_t q) {
    return ((q << 8) & 0x80008000u) | ((q << 7) & 0x3F803F80u);
}
__device__ __forceinline__ uint32_t place_odd(uint32_t q) {
    return (q & 0x80008000u) | ((q >> 1) & 0x3F803F80u);
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
template <int CONV>
__device__ __forceinline__ void piece_mma(float (&acc)[4][4], const uint4& A, const uint4& B,
                                          const uint4& xa, const uint4& xc) {
    const uint32_t wa[4] = {A.x, A.y, A.z, A.w};
    const uint32_t wb[4] = {B.x, B.y, B.z, B.w};
    const uint32_t bx[8] = {xa.x, xa.y, xa.z, xa.w, xc.x, xc.y, xc.z, xc.w};
#pragma unroll
    for (int s = 0; s < 4; ++s) {
        uint32_t a0, a1, a2, a3;
        if constexpr (CONV == CONV_PLACE) {
            a0 = place_even(wa[s]);
            a2 = place_odd(wa[s]);
            a1 = place_even(wb[s]);
            a3 = place_odd(wb[s]);
        } else {
            cvt_pairs(wa[s], a0, a2);
            cvt_pairs(wb[s], a1, a3);
        }
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
    int misc_off;  // unshift[8] f32, shift/amax[8], pow2[8]
    int part_off;  // [max_tpc][16 warps][32 lanes][4] f32
    int ring_off;  // TMA ring
    int bar_off;   // full[stages], empty[stages]
    int total;
};

__host__ __device__ inline Smem smem_layout(int M, int KP, int max_tpc, int stages) {
    Smem s;
    s.xpitch = 2 * KP + 16;
    s.x_off = 0;
    s.misc_off = M * s.xpitch;  // 16-byte aligned
    s.part_off = s.misc_off + 128;
    s.ring_off = s.part_off + max_tpc * WARPS * 32 * 16;
    s.ring_off = (s.ring_off + 127) & ~127;  // TMA destination alignment
    s.bar_off = s.ring_off + stages * STAGE_BYTES;
    s.total = s.bar_off + 2 * stages * 8;
    return s;
}

// Stages x [M][K] BF16 into shared memory as FP16 rows of KP elements (k
// permuted per CONV, zero-padded) with the per-token power-of-two shift.
// Executed by the CTHREADS consumer threads, synchronised on named barrier 1
// (no other thread takes part, and nothing here waits on an mbarrier).
template <int CONV>
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
                const int k = (c - m * kc) * 8;
                *reinterpret_cast<uint4*>(xs + m * L.xpitch + 2 * k) = xb[j];
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
    for (int c = tid; c < a.M * kpc; c += CTHREADS) {
        const int m = c / kpc;
        const int k = (c - m * kpc) * 8;
        uint4* p = reinterpret_cast<uint4*>(xs + m * L.xpitch + 2 * k);
        uint4 out = make_uint4(0, 0, 0, 0);
        if (k < a.K) {
            const uint4 raw = *p;
            const int sh = shift[m];
            const float p2 = pow2[m];
            const uint32_t wv[4] = {raw.x, raw.y, raw.z, raw.w};
            float f[8];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                f[2 * j] = p2 != 0.0f ? bf16_lo(wv[j]) * p2 : ldexpf(bf16_lo(wv[j]), sh);
                f[2 * j + 1] = p2 != 0.0f ? bf16_hi(wv[j]) * p2 : ldexpf(bf16_hi(wv[j]), sh);
            }
            constexpr bool perm = CONV == CONV_PLACE;  // pairs (0,2), (1,3)
            const __half2 h0 = __floats2half2_rn(f[0], perm ? f[2] : f[1]);
            const __half2 h1 = __floats2half2_rn(perm ? f[1] : f[2], f[3]);
            const __half2 h2 = __floats2half2_rn(f[4], perm ? f[6] : f[5]);
            const __half2 h3 = __floats2half2_rn(perm ? f[5] : f[6], f[7]);
            out = make_uint4(*reinterpret_cast<const uint32_t*>(&h0), *reinterpret_cast<const uint32_t*>(&h1),
                             *reinterpret_cast<const uint32_t*>(&h2), *reinterpret_cast<const uint32_t*>(&h3));
        }
        *p = out;
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
template <int CONV>
__device__ __forceinline__ void reduce_store(const Args& a, const uint8_t* smem, const Smem& L,
                                             int t0, int ntl, int tid) {
    const float* partial = reinterpret_cast<const float*>(smem + L.part_off);
    const float* unshift = reinterpret_cast<const float*>(smem + L.misc_off);
    const int per_tok = ntl * 16;
    const float fold = CONV == CONV_PLACE ? 256.0f : 1.0f;
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
        const float v = __fmul_rn(__fmul_rn(__fmul_rn(sum, unshift[m]), fold), a.s_w[n]);
        a.y[static_cast<size_t>(m) * a.N + n] = __float2bfloat16_rn(v);
    }
}

// ------------------------------------------------------------- TMA kernel

template <int CONV>
__global__ void __launch_bounds__(TMA_THREADS, 1)
w8a16_tma_kernel(const __grid_constant__ CUtensorMap tmW, const Args a) {
    extern __shared__ __align__(128) uint8_t smem[];
    const Smem L = smem_layout(a.M, a.KP, a.max_tpc, a.stages);
    uint8_t* ring = smem + L.ring_off;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bar_off);
    const int S = a.stages;
    auto full = [&](int s) { return smem_u32(&bars[s]); };
    auto empty = [&](int s) { return smem_u32(&bars[S + s]); };

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const int t0 = static_cast<int>(static_cast<int64_t>(blockIdx.x) * a.tiles / gridDim.x);
    const int t1 = static_cast<int>(static_cast<int64_t>(blockIdx.x + 1) * a.tiles / gridDim.x);
    const int ntl = t1 - t0;
    const int kwin = a.KP / WIN;    // k-windows per tile
    const int nstage = ntl * kwin;  // stages this CTA streams

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full(s), 1);
            mbar_init(empty(s), WARPS);
        }
        fence_mbar_init();
        tma_prefetch_desc(&tmW);
    }
    __syncthreads();

    if (warp == WARPS) {
        // ---------------------------------------------------------- producer
        // Consumers wait for every stage issued here before the CTA ends, so
        // no copy can land after the CTA exits; a timeout stops the stream.
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            for (int i = 0; i < nstage; ++i) {
                const int tl = i / kwin;
                const int kw = i - tl * kwin;
                if (!mbar_wait(empty(s), ph ^ 1u, a.timeout_ns, a.status)) break;
                mbar_arrive_expect_tx(full(s), STAGE_BYTES);
                if (a.wlayout == 0)
                    tma_load_3d(smem_u32(ring + s * STAGE_BYTES), &tmW, 0, (t0 + tl) * 16, kw * WARPS, full(s));
                else
                    tma_load_3d(smem_u32(ring + s * STAGE_BYTES), &tmW, 0, kw * WARPS, (t0 + tl) * 16, full(s));
                if (++s == S) { s = 0; ph ^= 1u; }
            }
        }
        return;
    }

    // -------------------------------------------------------------- consumers
    const int tid = threadIdx.x;
    stage_x<CONV>(a, smem, L, tid);
    const int g = lane >> 2, t = lane & 3;
    const uint8_t* xrow = smem + L.x_off + g * L.xpitch;
    const bool xok = g < a.M;
    float* partial = reinterpret_cast<float*>(smem + L.part_off);
    float acc[4][4];
#pragma unroll
    for (int s = 0; s < 4; ++s) acc[s][0] = acc[s][1] = acc[s][2] = acc[s][3] = 0.f;
    int s = 0;
    uint32_t ph = 0;
    int kw = 0, ct = 0;
    for (int i = 0; i < nstage; ++i) {
        if (!mbar_wait(full(s), ph, a.timeout_ns, a.status)) break;
        const uint8_t* box = ring + s * STAGE_BYTES + 16 * t +
                             (a.wlayout == 0 ? warp * 16 * BOX_K + g * BOX_K : g * WIN + warp * BOX_K);
        const int rstep = a.wlayout == 0 ? 8 * BOX_K : 8 * WIN;  // rows g -> g + 8
        const uint4 A = *reinterpret_cast<const uint4*>(box);
        const uint4 B = *reinterpret_cast<const uint4*>(box + rstep);
        __syncwarp();
        if (lane == 0) mbar_arrive(empty(s));  // the box is in registers: free the slot
        uint4 xa, xc;
        load_x(xrow, xok, kw * WIN + warp * BOX_K + 16 * t, xa, xc);
        piece_mma<CONV>(acc, A, B, xa, xc);
        if (++kw == kwin) {
            flush(acc, partial, ct, warp, lane);
            kw = 0;
            ++ct;
        }
        if (++s == S) { s = 0; ph ^= 1u; }
    }
    named_barrier(1, CTHREADS);
    reduce_store<CONV>(a, smem, L, t0, ntl, tid);
}

// -------------------------------------------------------- register kernel

template <int CONV>
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

    stage_x<CONV>(a, smem, L, threadIdx.x);
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
                    piece_mma<CONV>(acc, ra[d][h], rb[d][h], xa, xc);
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
    reduce_store<CONV>(a, smem, L, t0, ntl, threadIdx.x);
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
    static bool attr_done[64];
    if (!attr_done[di.device]) {
        const cudaError_t es[4] = {
            cudaFuncSetAttribute(w8a16_tma_kernel<CONV_CVT>, cudaFuncAttributeMaxDynamicSharedMemorySize, di.max_smem_optin),
            cudaFuncSetAttribute(w8a16_tma_kernel<CONV_PLACE>, cudaFuncAttributeMaxDynamicSharedMemorySize, di.max_smem_optin),
            cudaFuncSetAttribute(w8a16_reg_kernel<CONV_CVT>, cudaFuncAttributeMaxDynamicSharedMemorySize, di.max_smem_optin),
            cudaFuncSetAttribute(w8a16_reg_kernel<CONV_PLACE>, cudaFuncAttributeMaxDynamicSharedMemorySize, di.max_smem_optin)};
        for (cudaError_t e : es)
            if ((rc = cuda_check(e, "cudaFuncSetAttribute(w8a16)"))) return rc;
        attr_done[di.device] = true;
    }
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
    const bool cvt = g_conv == CONV_CVT;

    // TMA path (K % 64 == 0, so the 3-D view never reaches past a row): x rows
    // cover whole 1024-byte windows; as many ring stages (12 down to 3) as fit
    a.KP = static_cast<int>((K + WIN - 1) / WIN) * WIN;
    a.cpw = 0;
    if (K % BOX_K == 0) {
        // one CTA per SM; the deepest ring (12 down to 3 stages) that fits next
        // to x and the partial sums; more CTAs only if even 3 stages do not fit
        for (int grid = a.tiles < di.num_sms ? a.tiles : di.num_sms; grid <= a.tiles; ++grid) {
            const int max_tpc = (a.tiles + grid - 1) / grid;
            int stages = 12;
            Smem L = smem_layout(a.M, a.KP, max_tpc, stages);
            while (L.total > budget && stages > 3) L = smem_layout(a.M, a.KP, max_tpc, --stages);
            if (L.total > budget) continue;
            a.max_tpc = max_tpc;
            a.stages = stages;
            // preferred view {64 B, rows, k-groups}: the box lands as one 16-row
            // block per consumer warp (conflict-free reads); if the encoder wants
            // monotonic strides, the view {64 B, k-groups, rows} (row-major box)
            CUtensorMap tm;
            a.wlayout = 0;
            if (g_layout == 1 ||
                make_tmap_3d_u8(&tm, wq, BOX_K, static_cast<uint64_t>(N), static_cast<uint64_t>(K / BOX_K),
                                static_cast<uint64_t>(K), BOX_K, BOX_K, 16, WARPS) != METIS_OK) {
                clear_error();
                a.wlayout = 1;
                if ((rc = make_tmap_3d_u8(&tm, wq, BOX_K, static_cast<uint64_t>(K / BOX_K),
                                          static_cast<uint64_t>(N), BOX_K, static_cast<uint64_t>(K),
                                          BOX_K, WARPS, 16)))
                    return rc;
            }
            if (cvt) w8a16_tma_kernel<CONV_CVT><<<grid, TMA_THREADS, L.total, st>>>(tm, a);
            else w8a16_tma_kernel<CONV_PLACE><<<grid, TMA_THREADS, L.total, st>>>(tm, a);
            return cuda_check(cudaGetLastError(), "w8a16 launch");
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
    if (cvt) w8a16_reg_kernel<CONV_CVT><<<grid, CTHREADS, L.total, st>>>(a);
    else w8a16_reg_kernel<CONV_PLACE><<<grid, CTHREADS, L.total, st>>>(a);
    return cuda_check(cudaGetLastError(), "w8a16 launch");
}

// Tuning hook: bit 0 selects the E4M3 -> FP16 widening of metis_w8a16_gemm
// (0: cvt instruction, 1: bit placement); bit 1 forces the row-major weight
// box layout. Returns the previous setting.
extern "C" METIS_API int metis_internal_w8a16_variant(int v) {
    const int old = w8a16::g_conv | (w8a16::g_layout == 1 ? 2 : 0);
    if (v >= 0 && v <= 3) {
        w8a16::g_conv = v & 1;
        w8a16::g_layout = (v & 2) ? 1 : -1;
    }
    return old;
}
