// W8A8 "fast-math" GEMM on the fifth-generation tensor cores of sm_100a:
//   y[r, n] = bf16_rn( s_a[r] * s_b[n] * sum_k D(a[r, k]) * D(b[n, k]) )
// with E4M3 operands, FP32 accumulation in tensor memory (TMEM) and the
// per-token x per-channel scale applied in the epilogue ("Lernex/Metis-1.6-
// Logos-FP8", "What --fast-math does": each layer's input rounded to FP8 per
// token and multiplied with the FP8 weights on FP8 tensor cores; "What is in
// FP8": one scale per output channel).
//
// One persistent CTA per SM, 192 threads, warp-specialised:
//   warp 0      TMA producer: 128x128-byte A tiles and 256x128-byte B tiles,
//               128-byte swizzle, into a 4-stage shared-memory ring;
//   warp 1      allocates 512 TMEM columns; lane 0 issues tcgen05.mma
//               (kind::f8f6f4, M=128, N=256, K=32) and commits to mbarriers;
//   warps 2..5  epilogue: tcgen05.ld of the accumulator (one TMEM lane = one
//               output row per thread), scale, round to BF16, store.
// The accumulator is double-buffered in TMEM (2 x 256 columns), so the
// epilogue of tile i overlaps the main loop of tile i+1.
//
// The same kernel runs the grouped GEMM of the routed experts: rows of A are
// grouped by expert (offsets[e] .. offsets[e+1]), B is [E * N, K] and the
// scale of output channel n of expert e is s_b[e * N + n]. The tile schedule
// is built on the device from the offsets, so no host synchronisation.
//
// Every mbarrier wait is bounded by the device watchdog: on a timeout the
// CTA sets the sticky error word, stops issuing work, drains what it issued,
// frees TMEM and returns.
#include "common.cuh"

namespace metis {
namespace gemm {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 128;  // bytes = E4M3 elements per stage
constexpr int STAGES = 4;
constexpr int A_STAGE = BM * BK;
constexpr int B_STAGE = BN * BK;
constexpr int THREADS = 192;
constexpr int EPI_THREADS = 128;
constexpr int TMEM_COLS = 2 * BN;
constexpr int MAX_GROUPS = 1024;
constexpr uint32_t IDESC = idesc_e4m3_f32(BM, BN);

// barriers: full[STAGES], empty[STAGES], tfull[2], tempty[2], drain
constexpr int NUM_BARS = 2 * STAGES + 5;
constexpr size_t SMEM_TILES = static_cast<size_t>(STAGES) * (A_STAGE + B_STAGE);
constexpr size_t SMEM_BYTES_DENSE = 1024 + SMEM_TILES + NUM_BARS * 8 + 16;
constexpr size_t SMEM_BYTES_GROUPED = SMEM_BYTES_DENSE + 2 * (MAX_GROUPS + 1) * 4;

struct Params {
    const float* s_a;       // [rows of A]
    const float* s_b;       // [groups * N]
    __nv_bfloat16* y;       // [rows of A, N]
    const int32_t* offsets; // grouped: [E + 1] row offsets into A; dense: null
    int M;                  // dense: rows of A
    int N;                  // output columns (per group)
    int K;
    int E;                  // groups (1 for dense)
    uint32_t* status;
    uint64_t timeout_ns;
};

struct Tile {
    int a_row0;   // first row of A (and y) of this tile
    int row_end;  // rows >= row_end belong to another group (or are past M)
    int b_row0;   // first row of B
    int n0;       // first output column
    int group;
};

struct Sched {
    int num_n;
    int num_m;          // dense only
    int total;
    const int* g_tile;  // grouped: prefix sums of tiles per group [E + 1] (smem)
    const int* g_row;   // grouped: row offsets [E + 1] (smem)
    int E;
    int N;
    int M;

    __device__ __forceinline__ Tile get(int t) const {
        Tile ti;
        if (g_tile == nullptr) {
            const int mb = t % num_m;
            const int nb = t / num_m;
            ti.a_row0 = mb * BM;
            ti.row_end = M;
            ti.b_row0 = nb * BN;
            ti.n0 = nb * BN;
            ti.group = 0;
        } else {
            int lo = 0, hi = E;  // find e with g_tile[e] <= t < g_tile[e + 1]
            while (hi - lo > 1) {
                const int mid = (lo + hi) >> 1;
                if (g_tile[mid] <= t) lo = mid; else hi = mid;
            }
            const int e = lo;
            const int local = t - g_tile[e];
            const int rows = g_row[e + 1] - g_row[e];
            const int mt = (rows + BM - 1) / BM;
            const int mb = local % mt;
            const int nb = local / mt;
            ti.a_row0 = g_row[e] + mb * BM;
            ti.row_end = g_row[e + 1];
            ti.b_row0 = e * N + nb * BN;
            ti.n0 = nb * BN;
            ti.group = e;
        }
        return ti;
    }
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

template <bool GROUPED>
__global__ void __launch_bounds__(THREADS, 1)
fp8_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint8_t* sA = smem;
    uint8_t* sB = smem + STAGES * A_STAGE;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SMEM_TILES);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NUM_BARS);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* g_tile = reinterpret_cast<int*>(tmem_slot + 4);
    int* g_row = g_tile + (MAX_GROUPS + 1);

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    auto full = [&](int s) { return smem_u32(&bars[s]); };
    auto empty = [&](int s) { return smem_u32(&bars[STAGES + s]); };
    auto tfull = [&](int b) { return smem_u32(&bars[2 * STAGES + b]); };
    auto tempty = [&](int b) { return smem_u32(&bars[2 * STAGES + 2 + b]); };
    const uint32_t drain = smem_u32(&bars[2 * STAGES + 4]);

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full(s), 1);
            mbar_init(empty(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull(b), 1);
            mbar_init(tempty(b), EPI_THREADS);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
        tmem_relinquish();
    }

    Sched sc;
    sc.N = p.N;
    sc.M = p.M;
    sc.E = p.E;
    sc.num_n = (p.N + BN - 1) / BN;
    if constexpr (GROUPED) {
        // prefix sums of row offsets and of tiles per group, by warp 0
        if (warp == 0) {
            const int per = (p.E + 31) / 32;
            const int g0 = lane * per;
            int local = 0;
            for (int i = 0; i < per; ++i) {
                const int e = g0 + i;
                if (e < p.E) {
                    const int rows = p.offsets[e + 1] - p.offsets[e];
                    local += ((rows + BM - 1) / BM) * sc.num_n;
                }
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
                    const int rows = p.offsets[e + 1] - p.offsets[e];
                    g_tile[e] = run;
                    g_row[e] = p.offsets[e];
                    run += ((rows + BM - 1) / BM) * sc.num_n;
                }
            }
            if (lane == 31) {
                g_tile[p.E] = incl;
                g_row[p.E] = p.offsets[p.E];
            }
        }
        sc.g_tile = g_tile;
        sc.g_row = g_row;
        sc.num_m = 0;
    } else {
        sc.g_tile = nullptr;
        sc.g_row = nullptr;
        sc.num_m = (p.M + BM - 1) / BM;
        sc.total = sc.num_m * sc.num_n;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if constexpr (GROUPED) sc.total = g_tile[p.E];
    const uint32_t tmem_base = *tmem_slot;
    const int num_kb = (p.K + BK - 1) / BK;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------------------------------------------------- producer
            int stage = 0;
            uint32_t phase = 0;
            uint32_t issued = 0;  // bit s: stage s has a load whose completion is unobserved
            uint32_t issued_phase = 0;
            for (int t = blockIdx.x; t < sc.total && !*abort_flag; t += gridDim.x) {
                const Tile ti = sc.get(t);
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!mbar_wait(empty(stage), phase ^ 1u, p.timeout_ns, p.status)) {
                        *abort_flag = 1;
                        break;
                    }
                    mbar_arrive_expect_tx(full(stage), A_STAGE + B_STAGE);
                    tma_load_2d(smem_u32(sA + stage * A_STAGE), &tmA, kb * BK, ti.a_row0, full(stage));
                    tma_load_2d(smem_u32(sB + stage * B_STAGE), &tmB, kb * BK, ti.b_row0, full(stage));
                    issued |= 1u << stage;
                    issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
            }
            if (*abort_flag) {
                // let the copies in flight land before the CTA exits
                for (int s = 0; s < STAGES; ++s)
                    if (issued & (1u << s))
                        mbar_wait(full(s), (issued_phase >> s) & 1u, p.timeout_ns, p.status);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // --------------------------------------------------------- MMA issuer
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            for (int t = blockIdx.x; t < sc.total && !*abort_flag; t += gridDim.x) {
                if (!mbar_wait(tempty(acc), acc_phase ^ 1u, p.timeout_ns, p.status)) {
                    *abort_flag = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
                bool ok = true;
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!mbar_wait(full(stage), phase, p.timeout_ns, p.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t adesc = sw128_kmajor_desc(smem_u32(sA + stage * A_STAGE));
                    const uint64_t bdesc = sw128_kmajor_desc(smem_u32(sB + stage * B_STAGE));
#pragma unroll
                    for (int k = 0; k < BK / 32; ++k) {
                        // advance 32 bytes along K inside the swizzled 128-byte rows
                        mma_f8f6f4(d_tmem, adesc + 2 * k, bdesc + 2 * k, IDESC,
                                   (kb > 0 || k > 0) ? 1u : 0u);
                    }
                    mma_commit(empty(stage));
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) {
                    *abort_flag = 1;
                    break;
                }
                mma_commit(tfull(acc));
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1u;
            }
            // all MMAs issued by this thread complete before TMEM is released
            mma_commit(drain);
            mbar_wait(drain, 0, p.timeout_ns, p.status);
        }
    } else {
        // -------------------------------------------------------------- epilogue
        const int q = warp & 3;  // TMEM lane quadrant this warp may access
        const int r = q * 32 + lane;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int t = blockIdx.x; t < sc.total && !*abort_flag; t += gridDim.x) {
            const Tile ti = sc.get(t);
            if (!mbar_wait(tfull(acc), acc_phase, p.timeout_ns, p.status)) {
                *abort_flag = 1;
                break;
            }
            tc_fence_after();
            const int row = ti.a_row0 + r;
            const bool row_ok = row < ti.row_end;
            const float rs = row_ok ? p.s_a[row] : 0.0f;
            const float* sb = p.s_b + static_cast<size_t>(ti.group) * p.N;
            __nv_bfloat16* yrow = p.y + static_cast<size_t>(row_ok ? row : 0) * p.N;
#pragma unroll 1
            for (int c = 0; c < BN; c += 32) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                       static_cast<uint32_t>(acc * BN + c),
                                   v);
                tmem_ld_wait();
                const int n = ti.n0 + c;
                if (row_ok) {
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        const int ng = n + 8 * g;
                        if (ng < p.N) {
                            const float4 s0 = __ldg(reinterpret_cast<const float4*>(sb + ng));
                            const float4 s1 = __ldg(reinterpret_cast<const float4*>(sb + ng + 4));
                            const float f[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
                            uint32_t o[4];
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                const float lo = __fmul_rn(__fmul_rn(__uint_as_float(v[8 * g + 2 * j]), rs), f[2 * j]);
                                const float hi = __fmul_rn(__fmul_rn(__uint_as_float(v[8 * g + 2 * j + 1]), rs), f[2 * j + 1]);
                                o[j] = pack_bf16x2(lo, hi);
                            }
                            *reinterpret_cast<uint4*>(yrow + ng) = make_uint4(o[0], o[1], o[2], o[3]);
                        }
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(tempty(acc));
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1u;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

// Per-device one-time opt-in to the large dynamic shared memory.
int prepare(const DeviceInfo& di, bool grouped) {
    static bool done[64][2];
    const size_t need = grouped ? SMEM_BYTES_GROUPED : SMEM_BYTES_DENSE;
    if (static_cast<size_t>(di.max_smem_optin) < need)
        return fail(METIS_ERR_UNSUPPORTED, "fp8 gemm needs %zu bytes of shared memory", need);
    if (!done[di.device][grouped]) {
        cudaError_t e = grouped
            ? cudaFuncSetAttribute(fp8_gemm_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)need)
            : cudaFuncSetAttribute(fp8_gemm_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)need);
        int rc = cuda_check(e, "cudaFuncSetAttribute(fp8 gemm)");
        if (rc) return rc;
        done[di.device][grouped] = true;
    }
    return METIS_OK;
}

}  // namespace gemm

// Dense W8A8 GEMM launch (arguments validated by the caller).
int launch_fp8_gemm_dense(const uint8_t* a, const float* s_a, const uint8_t* b, const float* s_b,
                          __nv_bfloat16* y, int M, int N, int K, cudaStream_t st) {
    using namespace gemm;
    DeviceInfo di;
    int rc = current_device_info(&di);
    if (rc) return rc;
    if ((rc = prepare(di, false))) return rc;
    uint32_t* status = nullptr;
    if ((rc = device_status_word(&status))) return rc;
    CUtensorMap ta, tb;
    if ((rc = make_tmap_2d(&ta, a, 1, K, M, K, BK, BM, true))) return rc;
    if ((rc = make_tmap_2d(&tb, b, 1, K, N, K, BK, BN, true))) return rc;
    Params p{s_a, s_b, y, nullptr, M, N, K, 1, status, watchdog_ns()};
    const int tiles = ((M + BM - 1) / BM) * ((N + BN - 1) / BN);
    const int grid = tiles < di.num_sms ? tiles : di.num_sms;
    fp8_gemm_kernel<false><<<grid, THREADS, SMEM_BYTES_DENSE, st>>>(ta, tb, p);
    return cuda_check(cudaGetLastError(), "fp8 gemm launch");
}

// Grouped W8A8 GEMM launch: A rows [offsets[e], offsets[e+1]) use B rows
// [e*N, (e+1)*N). `rows` is the row count of A and y (offsets[E] <= rows).
int launch_fp8_gemm_grouped(const uint8_t* a, const float* s_a, const uint8_t* b, const float* s_b,
                            __nv_bfloat16* y, const int32_t* offsets, int E, int rows, int N,
                            int K, cudaStream_t st) {
    using namespace gemm;
    if (E > MAX_GROUPS) return fail(METIS_ERR_UNSUPPORTED, "grouped gemm: E=%d > %d", E, MAX_GROUPS);
    DeviceInfo di;
    int rc = current_device_info(&di);
    if (rc) return rc;
    if ((rc = prepare(di, true))) return rc;
    uint32_t* status = nullptr;
    if ((rc = device_status_word(&status))) return rc;
    CUtensorMap ta, tb;
    if ((rc = make_tmap_2d(&ta, a, 1, K, rows, K, BK, BM, true))) return rc;
    if ((rc = make_tmap_2d(&tb, b, 1, K, static_cast<uint64_t>(E) * N, K, BK, BN, true))) return rc;
    Params p{s_a, s_b, y, offsets, rows, N, K, E, status, watchdog_ns()};
    fp8_gemm_kernel<true><<<di.num_sms, THREADS, SMEM_BYTES_GROUPED, st>>>(ta, tb, p);
    return cuda_check(cudaGetLastError(), "grouped fp8 gemm launch");
}

}  // namespace metis

using namespace metis;

extern "C" int metis_fp8_gemm(const void* a, int a_kind, float* s_tok, const uint8_t* wq,
                              const float* s_w, void* y_bf16, int64_t M, int64_t N, int64_t K,
                              void* workspace, size_t ws_bytes, metis_stream_t stream) {
    clear_error();
    if (a_kind != METIS_A_E4M3 && a_kind != METIS_A_BF16)
        return fail(METIS_ERR_INVALID_ARG, "fp8_gemm: a_kind=%d", a_kind);
    if (M < 0 || N < 8 || N % 8 != 0 || K < 16 || K % 16 != 0)
        return fail(METIS_ERR_INVALID_ARG,
                    "fp8_gemm: need M >= 0, N >= 8 with N %% 8 == 0, K >= 16 with K %% 16 == 0 "
                    "(M=%lld N=%lld K=%lld)", (long long)M, (long long)N, (long long)K);
    if (M > 0x7fffffff || N > 0x7fffffff || K > 0x7fffffff)
        return fail(METIS_ERR_INVALID_ARG, "fp8_gemm: dimensions must fit in 31 bits");
    if (M == 0) return METIS_OK;
    if (!a || !s_tok || !wq || !s_w || !y_bf16) return fail(METIS_ERR_INVALID_ARG, "fp8_gemm: null pointer");
    if (!aligned(a, 16) || !aligned(wq, 16) || !aligned(y_bf16, 16) || !aligned(s_w, 16) ||
        !aligned(s_tok, 4))
        return fail(METIS_ERR_INVALID_ARG, "fp8_gemm: a, wq, y and s_w must be 16-byte aligned");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (a_kind == METIS_A_E4M3)
        return launch_fp8_gemm_dense(static_cast<const uint8_t*>(a), s_tok, wq, s_w,
                                     static_cast<__nv_bfloat16*>(y_bf16), static_cast<int>(M),
                                     static_cast<int>(N), static_cast<int>(K), st);
    (void)workspace;
    (void)ws_bytes;
    return fail(METIS_ERR_UNSUPPORTED, "fp8_gemm: the fused BF16 prologue is not built yet");
}
