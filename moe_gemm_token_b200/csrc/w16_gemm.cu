// Default-maths weight-only GEMM for many tokens (M > 8) on the fifth-
// generation tensor cores:
//   y[m, n] = bf16_rn( s_w[n] * sum_k x[m, k] * D(w[n, k]) ),  FP32 accumulation,
// with the E4M3 weights widened exactly to BF16 and BF16 x BF16 products
// ("Lernex/Metis-1.6-Logos-FP8", "What --fast-math does": by default the FP8
// weights are expanded to 16 bits as they are multiplied, so the weights are
// the only thing rounded).
//
// Computed as y^T = W x^T so that the widened weights never pass through
// shared memory: a 128-channel x TM-token tile per CTA (TM = 128 or 256),
// the channels on the 128 TMEM lanes.
//   warp 0      TMA producer of the x tiles (BF16, TM tokens x 128 elements
//               as two 64-element boxes, 128-byte swizzle) into a
//               shared-memory ring (4 stages for TM = 128, 3 for 256);
//   warp 1      allocates all 512 TMEM columns (FP32 accumulators: two of
//               128 columns, or one of 256; 64-column weight stages after
//               them); one lane issues tcgen05.mma.kind::f16 with A = the
//               widened weights in TMEM and B = the x tile in shared memory,
//               8 MMAs (K = 16) per stage;
//   warps 2..9  converters, two per TMEM lane quadrant: each thread streams
//               64 bytes of its weight row per stage from global memory
//               (four stages ahead in registers), widens E4M3 to BF16
//               exactly (through FP16 and FP32: every E4M3 value is a BF16
//               value) and writes the 32 packed words into its lane of a TMEM
//               weight stage (tcgen05.st);
//   warps 10..13 epilogue: tcgen05.ld of 32 channels x 32 tokens, x s_w[n],
//               BF16 RNE, transposed through a 32x32 shared-memory block and
//               stored as 64-byte token rows.
// One thread issues every MMA, and a tcgen05.mma of 128 x 128 x 16 takes
// about as long to issue as twice its tensor time: each stage therefore
// carries 8 MMAs, the MMA thread waits on one barrier per stage (the x
// tile's bytes and the converters' arrivals complete the same barrier) and
// commits to one (which both the producer and the converters wait on), and
// when there are tiles enough the 256-token tiles halve the MMAs per FLOP.
// Every mbarrier wait is bounded by the device watchdog.
#include "common.cuh"

namespace metis {
namespace w16 {

constexpr int BKE = 128;         // K elements per stage (two 128-byte rows of BF16 x per token)
constexpr int BOXE = 64;         // K elements per x box (128 bytes: the swizzle span)
constexpr int TILE_N = 128;      // channels per tile (TMEM lanes)
constexpr int A_COLS = BKE / 2;  // TMEM columns per weight stage (two BF16 per column)
constexpr int TMEM_COLS = 512;
constexpr int CONV_WARPS = 8;   // two per TMEM lane quadrant, each on half of a stage
constexpr int PF = 4;           // stages of weight bytes in flight per converter thread
constexpr int THREADS = 64 + CONV_WARPS * 32 + 4 * 32;

// Tiles of TM tokens (accumulator columns). TM = 128: two accumulators (the
// epilogue drains one while the MMAs fill the other) and 4 weight stages.
// TM = 256: N = 256 MMAs, half as many per FLOP for the one issuing thread;
// TMEM then holds one accumulator and 3 weight stages, so the epilogue's
// drain of a tile is not overlapped with the next tile's MMAs.
template <int TM>
struct Cfg {
    static constexpr int ACCS = TM == 128 ? 2 : 1;
    static constexpr int STAGES = TM == 128 ? 4 : 3;  // x ring and TMEM weight stages
    static constexpr int X_BOX = TM * BOXE * 2;       // 16 or 32 KB
    static constexpr int X_STAGE = 2 * X_BOX;
    static constexpr int A_COL0 = ACCS * TM;          // weight stages after the accumulators
    static constexpr uint32_t IDESC = idesc_bf16_f32(TILE_N, TM);
    // shared memory: x ring | epilogue staging (4 warps x 2 KB) | barriers | misc
    static constexpr int STG_OFF = STAGES * X_STAGE;
    static constexpr int BAR_OFF = STG_OFF + 4 * 2048;
    // full[S] (x bytes + converter arrivals), empty[S], tfull[ACCS], tempty[ACCS], drain
    static constexpr int NUM_BARS = 2 * STAGES + 2 * ACCS + 1;
    static constexpr int MISC_OFF = BAR_OFF + NUM_BARS * 8;
    static constexpr size_t SMEM_BYTES = 1024 + MISC_OFF + 16;
    static_assert(TM == 128 || TM == 256, "tile width");
    static_assert(A_COL0 + STAGES * A_COLS <= TMEM_COLS, "TMEM budget");
};

struct Params {
    const uint8_t* w;     // [N, K] E4M3
    const float* s_w;     // [N]
    __nv_bfloat16* y;     // [M, N]
    int M, N, K;
    uint32_t* status;
    uint64_t timeout_ns;
};

__device__ __forceinline__ uint4 ld_w16(const uint8_t* p) {
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// One 32-byte load (a whole sector) at a 32-byte aligned address.
__device__ __forceinline__ void ld_w32(const uint8_t* p, uint4& a, uint4& b) {
    asm volatile("ld.global.nc.v8.u32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(a.x), "=r"(a.y), "=r"(a.z), "=r"(a.w), "=r"(b.x), "=r"(b.y), "=r"(b.z), "=r"(b.w)
                 : "l"(p));
}

// Four E4M3 bytes -> two BF16 pairs (bytes 0,1 and 2,3), exactly: E4M3 ->
// FP16 (cvt.rn.f16x2.e4m3x2, exact) -> FP32 (exact) -> BF16 (exact, every
// E4M3 value being a BF16 value). Eight instructions per four elements.
__device__ __forceinline__ void e4m3x4_to_bf16x2x2(uint32_t w, uint32_t& lo, uint32_t& hi) {
    asm("{\n\t"
        ".reg .b16 q0, q1, a, b, c, d;\n\t"
        ".reg .b32 h0, h1;\n\t"
        ".reg .f32 fa, fb, fc, fd;\n\t"
        "mov.b32 {q0, q1}, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 h0, q0;\n\t"
        "cvt.rn.f16x2.e4m3x2 h1, q1;\n\t"
        "mov.b32 {a, b}, h0;\n\t"
        "mov.b32 {c, d}, h1;\n\t"
        "cvt.f32.f16 fa, a;\n\t"
        "cvt.f32.f16 fb, b;\n\t"
        "cvt.f32.f16 fc, c;\n\t"
        "cvt.f32.f16 fd, d;\n\t"
        "cvt.rn.bf16x2.f32 %0, fb, fa;\n\t"
        "cvt.rn.bf16x2.f32 %1, fd, fc;\n\t"
        "}"
        : "=r"(lo), "=r"(hi)
        : "r"(w));
}

template <int TM>
__global__ void __launch_bounds__(THREADS, 1)
w16_gemm_kernel(const __grid_constant__ CUtensorMap tmX, const Params p) {
    using C = Cfg<TM>;
    constexpr int STAGES = C::STAGES;
    constexpr int X_BOX = C::X_BOX;
    constexpr int X_STAGE = C::X_STAGE;
    constexpr int A_COL0 = C::A_COL0;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    uint8_t* ring = smem;
    uint8_t* staging = smem + C::STG_OFF;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::MISC_OFF + 4);
    auto full = [&](int s) { return smem_u32(&bars[s]); };
    auto empty = [&](int s) { return smem_u32(&bars[STAGES + s]); };
    auto tfull = [&](int b) { return smem_u32(&bars[2 * STAGES + b]); };
    auto tempty = [&](int b) { return smem_u32(&bars[2 * STAGES + C::ACCS + b]); };
    const uint32_t drain = smem_u32(&bars[2 * STAGES + 2 * C::ACCS]);

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            // the producer's arrival (with the x bytes) and one per converter warp
            mbar_init(full(s), 1 + CONV_WARPS);
            mbar_init(empty(s), 1);
        }
        for (int b = 0; b < C::ACCS; ++b) {
            mbar_init(tfull(b), 1);
            mbar_init(tempty(b), 4);  // the four epilogue warps
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmX);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    grid_launch_dependents();
    grid_dependency_wait();  // x may be the previous kernel's output
    const uint32_t tmem_base = *tmem_slot;
    const int num_m = (p.M + TM - 1) / TM;
    const int total = num_m * ((p.N + TILE_N - 1) / TILE_N);
    const int num_kb = (p.K + BKE - 1) / BKE;
    // tiles: token block fastest, so CTAs running together share weight rows

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------------- producer
            int s = 0;
            uint32_t ph = 0;
            for (int t = blockIdx.x; t < total && !*abort_flag; t += gridDim.x) {
                const int m0 = (t % num_m) * TM;
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!mbar_wait(empty(s), ph ^ 1u, p.timeout_ns, p.status)) {
                        *abort_flag = 1;
                        break;
                    }
                    mbar_arrive_expect_tx(full(s), X_STAGE);
                    const uint32_t dst = smem_u32(ring + s * X_STAGE);
                    tma_load_2d(dst, &tmX, kb * BKE, m0, full(s));
                    tma_load_2d(dst + X_BOX, &tmX, kb * BKE + BOXE, m0, full(s));
                    if (++s == STAGES) { s = 0; ph ^= 1u; }
                }
            }
            if (*abort_flag) {
                // let copies in flight land before the CTA exits
                const uint64_t t0 = globaltimer_ns();
                while (globaltimer_ns() - t0 < 100000ull) {}
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------------------------------------------- MMA issuer
            int s = 0;
            uint32_t ph = 0;
            int acc = 0;
            uint32_t acc_ph = 0;
            for (int t = blockIdx.x; t < total && !*abort_flag; t += gridDim.x) {
                if (!mbar_wait(tempty(acc), acc_ph ^ 1u, p.timeout_ns, p.status)) {
                    *abort_flag = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * TM);
                bool ok = true;
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!mbar_wait(full(s), ph, p.timeout_ns, p.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t bdesc0 = sw128_kmajor_desc(smem_u32(ring + s * X_STAGE));
                    const uint64_t bdesc1 = sw128_kmajor_desc(smem_u32(ring + s * X_STAGE + X_BOX));
                    const uint32_t a_tmem = tmem_base + static_cast<uint32_t>(A_COL0 + s * A_COLS);
                    // K = 16 per MMA: 8 TMEM columns of A, 32 bytes along a box row of B
#pragma unroll
                    for (int k = 0; k < BOXE / 16; ++k)
                        mma_f16_tmem_a(d_tmem, a_tmem + 8 * k, bdesc0 + 2 * k, C::IDESC, (kb > 0 || k > 0) ? 1u : 0u);
#pragma unroll
                    for (int k = 0; k < BOXE / 16; ++k)
                        mma_f16_tmem_a(d_tmem, a_tmem + 8 * (k + BOXE / 16), bdesc1 + 2 * k, C::IDESC, 1u);
                    mma_commit(empty(s));
                    if (++s == STAGES) { s = 0; ph ^= 1u; }
                }
                if (!ok) {
                    *abort_flag = 1;
                    break;
                }
                mma_commit(tfull(acc));
                if (++acc == C::ACCS) { acc = 0; acc_ph ^= 1u; }
            }
            mma_commit(drain);
            mbar_wait(drain, 0, p.timeout_ns, p.status);
        }
    } else if (warp < 2 + CONV_WARPS) {
        // -------------------------------------------------------- converters
        const int q = warp & 3;
        const int half = (warp - 2) / 4;   // which 64 elements of the stage
        const int lane_base = q * 32;
        const bool wide = (p.K % 32) == 0 && (reinterpret_cast<uintptr_t>(p.w) & 31u) == 0;
        int s = 0;
        uint32_t ph = 0;
        for (int t = blockIdx.x; t < total && !*abort_flag; t += gridDim.x) {
            const int row = (t / num_m) * TILE_N + lane_base + lane;  // weight row = output channel
            const bool row_ok = row < p.N;
            const uint8_t* wrow = p.w + static_cast<size_t>(row_ok ? row : 0) * p.K + 64 * half;
            // a thread's 64 bytes of a stage are two sectors: 32-byte loads
            // when the rows are 32-byte aligned (K % 32 == 0; two 16-byte
            // loads of the same sector would each move the whole sector
            // through L1), 16-byte loads otherwise and at the end of K
            auto load_kb = [&](int kb, uint4 (&r)[4]) {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int k0 = kb * BKE + 64 * half + 32 * h;
                    if (wide && row_ok && k0 + 32 <= p.K) {
                        ld_w32(wrow + kb * BKE + 32 * h, r[2 * h], r[2 * h + 1]);
                        continue;
                    }
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        const int k = k0 + 16 * j;
                        r[2 * h + j] = (row_ok && k < p.K) ? ld_w16(wrow + kb * BKE + 32 * h + 16 * j)
                                                           : make_uint4(0, 0, 0, 0);
                    }
                }
            };
            // PF stages of weight bytes in flight per thread (L2 latency)
            uint4 buf[PF][4];
#pragma unroll
            for (int d = 0; d < PF; ++d) load_kb(d, buf[d]);
            bool ok = true;
            for (int kb0 = 0; kb0 < num_kb && ok; kb0 += PF) {
#pragma unroll
                for (int d = 0; d < PF; ++d) {
                    const int kb = kb0 + d;
                    if (kb >= num_kb || !ok) break;
                    uint32_t words[32];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint32_t v[4] = {buf[d][j].x, buf[d][j].y, buf[d][j].z, buf[d][j].w};
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            e4m3x4_to_bf16x2x2(v[i], words[8 * j + 2 * i], words[8 * j + 2 * i + 1]);
                    }
                    load_kb(kb + PF, buf[d]);  // zeros past the end of K
                    if (!mbar_wait(empty(s), ph ^ 1u, p.timeout_ns, p.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    tmem_st_32x32b_x32(tmem_base + (static_cast<uint32_t>(lane_base) << 16) +
                                           static_cast<uint32_t>(A_COL0 + s * A_COLS + 32 * half),
                                       words);
                    tmem_st_wait();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(full(s));
                    if (++s == STAGES) { s = 0; ph ^= 1u; }
                }
            }
            if (!ok) {
                *abort_flag = 1;
                break;
            }
        }
    } else {
        // ---------------------------------------------------------- epilogue
        const int q = warp & 3;  // warps 10..13 -> quadrants 2, 3, 0, 1
        uint8_t* stg = staging + (warp - 2 - CONV_WARPS) * 2048;  // [32 tokens][32 channels] BF16
        int acc = 0;
        uint32_t acc_ph = 0;
        for (int t = blockIdx.x; t < total && !*abort_flag; t += gridDim.x) {
            const int m0 = (t % num_m) * TM;
            const int n_lane = (t / num_m) * TILE_N + q * 32 + lane;  // this thread's channel
            const float sw = n_lane < p.N ? p.s_w[n_lane] : 0.0f;
            if (!mbar_wait(tfull(acc), acc_ph, p.timeout_ns, p.status)) {
                *abort_flag = 1;
                break;
            }
            tc_fence_after();
            const uint32_t tbase =
                tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * TM);
            const int nq0 = (t / num_m) * TILE_N + q * 32;  // first channel of this warp
            for (int c = 0; c < TM / 32; ++c) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(tbase + c * 32, v);
                tmem_ld_wait();
                if (c == TM / 32 - 1) {
                    // the accumulator has been read: release it
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(tempty(acc));
                }
                // lane = channel, j = token: transpose into [token][channel]
                __syncwarp();
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const __nv_bfloat16 b = __float2bfloat16_rn(__fmul_rn(__uint_as_float(v[j]), sw));
                    *reinterpret_cast<__nv_bfloat16*>(stg + j * 64 + lane * 2) = b;
                }
                __syncwarp();
                // 8 tokens x 64 bytes per instruction
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int tk = (lane >> 2) + 8 * i;
                    const int m = m0 + c * 32 + tk;
                    const int n = nq0 + (lane & 3) * 8;
                    const uint4 val = *reinterpret_cast<const uint4*>(stg + tk * 64 + (lane & 3) * 16);
                    if (m < p.M && n < p.N)
                        *reinterpret_cast<uint4*>(p.y + static_cast<size_t>(m) * p.N + n) = val;
                }
            }
            if (++acc == C::ACCS) { acc = 0; acc_ph ^= 1u; }
        }
    }

    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

}  // namespace w16

// Weight-only W8A16 GEMM for M > 8 tokens (arguments validated by the
// caller): x BF16 [M, K], wq E4M3 [N, K], N % 8 == 0, K % 16 == 0.
int launch_w8a16_tensor(const __nv_bfloat16* x, const uint8_t* wq, const float* s_w,
                        __nv_bfloat16* y, int M, int N, int K, cudaStream_t st) {
    using namespace w16;
    DeviceInfo di;
    int rc = current_device_info(&di);
    if (rc) return rc;
    static std::atomic<uint64_t> attr_done[64];
    if (static_cast<size_t>(di.max_smem_optin) < Cfg<256>::SMEM_BYTES)
        return fail(METIS_ERR_UNSUPPORTED, "w8a16 tensor-core GEMM needs %zu bytes of shared memory",
                    Cfg<256>::SMEM_BYTES);
    rc = once_per_context(attr_done, di.device, [] {
        if (int r = cuda_check(cudaFuncSetAttribute(w16_gemm_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                    static_cast<int>(Cfg<128>::SMEM_BYTES)),
                               "cudaFuncSetAttribute(w16 gemm)"))
            return r;
        return cuda_check(cudaFuncSetAttribute(w16_gemm_kernel<256>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               static_cast<int>(Cfg<256>::SMEM_BYTES)),
                          "cudaFuncSetAttribute(w16 gemm)");
    });
    if (rc) return rc;
    uint32_t* status = nullptr;
    if ((rc = device_status_word(&status))) return rc;
    Params p{wq, s_w, y, M, N, K, status, watchdog_ns()};
    // a wave of 256-token tiles takes about 1.25 times as long as one of
    // 128-token tiles (17.7 against 14.0 us for 6144 x 2048 weights) for
    // twice the work (the same MMA count, the epilogue not overlapped): take
    // them unless their fewer, longer waves are slower on this grid
    const int64_t nn = (N + TILE_N - 1) / TILE_N;
    const int64_t t128 = (M + 127) / 128 * nn, t256 = (M + 255) / 256 * nn;
    const int64_t w128 = (t128 + di.num_sms - 1) / di.num_sms, w256 = (t256 + di.num_sms - 1) / di.num_sms;
    const bool wide = 125 * w256 < 100 * w128;
    const int tm = wide ? 256 : 128;
    CUtensorMap tx;
    if ((rc = make_tmap_2d(&tx, x, 2, static_cast<uint64_t>(K), static_cast<uint64_t>(M),
                           static_cast<uint64_t>(K) * 2, BOXE, tm, true)))
        return rc;
    const int64_t tiles = wide ? t256 : t128;
    const int grid = static_cast<int>(tiles < di.num_sms ? tiles : di.num_sms);
    if (wide)
        return cuda_check(launch_pdl(w16_gemm_kernel<256>, dim3(grid), dim3(THREADS), Cfg<256>::SMEM_BYTES, st,
                                     1, tx, p),
                          "w8a16 tensor-core GEMM launch");
    return cuda_check(launch_pdl(w16_gemm_kernel<128>, dim3(grid), dim3(THREADS), Cfg<128>::SMEM_BYTES, st, 1,
                                 tx, p),
                      "w8a16 tensor-core GEMM launch");
}

namespace w16 {

// Exact E4M3 -> BF16 widening of a weight matrix into a workspace, HBM-bound:
// 1 byte read and 2 written per element. A thread widens 8 bytes into one
// 16-byte store, so a warp reads 256 and writes 512 contiguous bytes per
// instruction; each thread has WIDEN_BATCH loads in flight (grid-strided)
// before it widens and stores them. The BF16 copy stays in L2 for the GEMM
// that follows.
constexpr int WIDEN_BATCH = 8;

__global__ void __launch_bounds__(256) widen_e4m3_kernel(const uint2* __restrict__ w, uint4* __restrict__ out,
                                                          int64_t n8) {
    // the workspace may still be read by the previous kernel (the previous
    // layer's GEMM): wait for it before writing
    grid_dependency_wait();
    grid_launch_dependents();
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
         i += WIDEN_BATCH * stride) {
        uint2 v[WIDEN_BATCH];
#pragma unroll
        for (int u = 0; u < WIDEN_BATCH; ++u)
            if (i + u * stride < n8) v[u] = __ldg(w + i + u * stride);
#pragma unroll
        for (int u = 0; u < WIDEN_BATCH; ++u) {
            const int64_t c = i + u * stride;
            if (c < n8) {
                uint4 o;
                widen_e4m3x8(v[u], o);
                out[c] = o;
            }
        }
    }
}

}  // namespace w16

int launch_widen_e4m3(const uint8_t* w, __nv_bfloat16* out, int64_t n, cudaStream_t st) {
    DeviceInfo di;
    int rc = current_device_info(&di);
    if (rc) return rc;
    const int64_t n8 = n / 8;
    if (n8 == 0) return METIS_OK;
    // WIDEN_BATCH chunks per thread, at most 8 resident 256-thread blocks per SM
    int64_t blocks = (n8 + w16::WIDEN_BATCH * 256 - 1) / (w16::WIDEN_BATCH * 256);
    const int64_t cap = static_cast<int64_t>(di.num_sms) * 8;
    if (blocks > cap) blocks = cap;
    return cuda_check(launch_pdl(w16::widen_e4m3_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, st, 1,
                                 reinterpret_cast<const uint2*>(w), reinterpret_cast<uint4*>(out), n8),
                      "e4m3 widening launch");
}

}  // namespace metis

using namespace metis;

extern "C" int metis_w8a16_gemm_widened(const void* x_bf16, const uint8_t* wq, const float* s_w,
                                        void* y_bf16, int64_t M, int64_t N, int64_t K, void* workspace,
                                        size_t ws_bytes, metis_stream_t stream) {
    clear_error();
    if (M < 0 || M > 0x7fffffff || N < 8 || N % 8 != 0 || N > 0x7fffffff || K < 16 || K % 16 != 0 ||
        K > 0x7fffffff)
        return fail(METIS_ERR_INVALID_ARG,
                    "w8a16_gemm_widened: need M >= 0, N >= 8 with N %% 8 == 0, K >= 16 with K %% 16 == 0 "
                    "(M=%lld N=%lld K=%lld)", (long long)M, (long long)N, (long long)K);
    if (M == 0) return METIS_OK;
    if (!x_bf16 || !wq || !s_w || !y_bf16) return fail(METIS_ERR_INVALID_ARG, "w8a16_gemm_widened: null pointer");
    if (!aligned(x_bf16, 16) || !aligned(wq, 16) || !aligned(s_w, 4) || !aligned(y_bf16, 16))
        return fail(METIS_ERR_INVALID_ARG, "w8a16_gemm_widened: x, wq and y must be 16-byte aligned");
    const size_t need = metis_workspace_size(METIS_OP_W8A16_WIDENED, M, N, K, 0, 0);
    if (!workspace || ws_bytes < need || !aligned(workspace, 16))
        return fail(METIS_ERR_INVALID_ARG,
                    "w8a16_gemm_widened: needs a 16-byte aligned workspace of %zu bytes (got %zu)", need,
                    ws_bytes);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    __nv_bfloat16* wb = static_cast<__nv_bfloat16*>(workspace);
    int rc = launch_widen_e4m3(wq, wb, N * K, st);
    if (rc) return rc;
    return launch_bf16_gemm(static_cast<const __nv_bfloat16*>(x_bf16), wb, static_cast<__nv_bfloat16*>(y_bf16),
                            static_cast<int>(M), static_cast<int>(N), static_cast<int>(K), s_w, st);
}
