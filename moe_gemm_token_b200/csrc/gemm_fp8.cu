// W8A8 "fast-math" GEMM on the fifth-generation tensor cores of sm_100a:
//   y[r, n] = bf16_rn( s_a[r] * s_b[n] * sum_k D(a[r, k]) * D(b[n, k]) )
// with E4M3 operands, FP32 accumulation in tensor memory (TMEM) and the
// per-token x per-channel scale applied in the epilogue ("Lernex/Metis-1.6-
// Logos-FP8", "What --fast-math does": each layer's input rounded to FP8 per
// token and multiplied with the FP8 weights on FP8 tensor cores; "What is in
// FP8": one scale per output channel).
//
// Persistent, warp-specialised, 320 threads per CTA:
//   warp 0      TMA producer into a shared-memory ring (128-byte swizzle);
//   warp 1      allocates 512 TMEM columns (two 256-column accumulators); one
//               lane issues tcgen05.mma kind::f8f6f4 and commits to mbarriers;
//   warps 2..9  epilogue, two warps per TMEM lane quadrant, each on half of
//               the 256 columns: per-channel scales staged in shared memory
//               once per tile, tcgen05.ld software-pipelined, the accumulator
//               released as soon as it is read, scaled BF16 rows staged per
//               warp in a swizzled 32x32 block and written out as full 64-byte
//               row pieces. (With one warp per quadrant every instruction's
//               latency was exposed: ~3.5 us per 128 x 256 tile.)
// Two variants:
//   CTAS = 2  a CTA pair (cluster of 2) computes a 256 x 256 tile with
//             tcgen05.mma.cta_group::2: each CTA loads its own 128 rows of A
//             and 128 rows of B (16 + 16 KB per 128-deep k-block, 6 stages),
//             so each SM streams half of the B tile it would need alone. Both
//             CTAs' TMA loads complete on the even CTA's mbarrier; its MMA
//             commits are multicast to both CTAs. Dense GEMMs with M > 128,
//             and the grouped GEMM of the routed experts for K >= 2048.
//   CTAS = 1  one CTA computes 128 x 256 (4 stages of 16 + 32 KB). Used for
//             small M and for the grouped GEMM with K < 2048 (the routed
//             down-projection), where it measured faster than pairs.
// Grouped: rows of A grouped by expert, B = [E * N, K], the tile schedule
// built on the device from the expert offsets. Dense: tiles in groups of
// RASTER_M row blocks, row block fastest inside a group.
// Fused quantization (ABF16): A arrives as BF16. An amax pre-pass has written
// each row's 448/amax; the producer TMA-loads BF16 A tiles into a 2-slot
// staging ring, and 8 converter warps turn each into the swizzled E4M3 tile
// the MMA reads (x * (448/amax), cvt.rn.satfinite: the standalone quantizer's
// bytes), so the codes never go through HBM.
// BF16 operands (W16): the same pipeline with BF16 A and B tiles (64 elements
// = 128 bytes per k-block row, tcgen05.mma kind::f16). Without scales it is
// the shared expert's GEMM ("Lernex/Metis-1.6-Praxis" card, "Architecture":
// one shared expert beside the routed ones; kept in BF16 by the FP8 cards);
// with per-column scales (SCALED) it is the default maths on weights widened
// to BF16 beforehand: y = bf16(acc * s_w[n]).
// Dense tiles whose count leaves a final wave that keeps at most a quarter of
// the CTA pairs busy have that wave's tiles cut into four column pieces, one
// per pair (an MMA of N = 64 and a B box of a quarter of the rows).
// Every mbarrier wait is bounded by the device watchdog: on a timeout the CTA
// sets the sticky error word, stops issuing work, drains what it issued,
// frees TMEM and returns.
#include "common.cuh"

namespace metis {
namespace gemm {

constexpr int BK = 128;    // bytes = E4M3 elements per k-block
constexpr int BN_MAX = 256;  // output columns per tile
constexpr int ROWS = 128;  // output rows per CTA per tile (TMEM lanes)
constexpr int THREADS = 64;  // producer warp + MMA warp (epilogue and converters added per variant)
constexpr int TMEM_COLS = 2 * BN_MAX;
constexpr int MAX_GROUPS = 1024;

constexpr int CONV_WARPS = 8;                  // fused-quantization converter warps
constexpr int RASTER_M = 16;  // row blocks per raster group of the dense schedule
constexpr int ASTG_SLOT = ROWS * BK * 2;       // one BF16 A tile (two 64-column boxes)

template <int CTAS, bool ABF16 = false, int BN = BN_MAX, bool W16 = false, bool GROUPED = false>
struct Layout {
    // BF16 k-blocks take twice the MMA time of E4M3 ones: fewer stages suffice
    // Dense CTA-pair tiles take two 128-byte k-blocks per ring stage: one
    // thread issues every MMA of the pair, at about the pipe's own rate, and
    // each barrier wait and commit it does between MMAs costs throughput
    // (8 MMAs per wait instead of 4: 4096 x 6144 x 2048 44.9 -> 42.4 us).
    // The grouped kernel (short k-loops per tile) measured better with the
    // finer 6-stage ring.
    static constexpr int KPS = (CTAS == 2 && !ABF16 && !GROUPED) ? 2 : 1;
    static constexpr int STAGES = KPS == 2 ? 3
                                           : (W16 ? (CTAS == 2 ? 4 : 3)
                                                  : (CTAS == 2 ? (ABF16 ? 4 : 6) : (ABF16 ? 3 : 4)));
    static constexpr int ASTG = ABF16 ? 2 : 0;  // BF16 staging slots
    // epilogue warps: two per TMEM lane quadrant, each on half the columns
    // (one per quadrant in the fused variants, whose shared memory and
    // registers go to the converter warps)
    static constexpr int EPI = ABF16 ? 4 : 8;
    static constexpr int THREADS_ = THREADS + EPI * 32 + (ABF16 ? CONV_WARPS * 32 : 0);
    static constexpr int B_ROWS = BN / CTAS;   // rows of B loaded by one CTA
    static constexpr int A_BOX = ROWS * BK;
    static constexpr int B_BOX = B_ROWS * BK;
    static constexpr int A_STAGE = KPS * A_BOX;
    static constexpr int B_STAGE = KPS * B_BOX;
    static constexpr int TILES = STAGES * (A_STAGE + B_STAGE) + ASTG * ASTG_SLOT;
    static constexpr int STAGING = EPI * 32 * 64;  // a 32 x 32 BF16 block per epilogue warp
    static constexpr int SW = 2 * BN * 4;                // per-channel scales, double-buffered
    // full, empty, tfull[2], tempty[2], drain, epilogue sync[2], staging full/empty
    static constexpr int NUM_BARS = 2 * STAGES + 7 + 2 * ASTG;
    static constexpr int BAR_OFF = TILES + STAGING + SW;
    static constexpr int MISC_OFF = BAR_OFF + NUM_BARS * 8;
    static constexpr int GROUP_OFF = MISC_OFF + 16;
    static constexpr size_t BYTES_DENSE = 1024 + GROUP_OFF;
    static constexpr size_t BYTES_GROUPED = BYTES_DENSE + 2 * (MAX_GROUPS + 1) * 4;
    static constexpr uint32_t IDESC = W16 ? idesc_bf16_f32(ROWS * CTAS, BN) : idesc_e4m3_f32(ROWS * CTAS, BN);
    static constexpr int KE = W16 ? BK / 2 : BK;  // elements per k-block row
};

struct Params {
    const float* s_a;        // [rows of A]
    const float* inv;        // fused quantization: 448/amax per row of A
    const float* s_b;        // [groups * N]
    __nv_bfloat16* y;        // [rows of A, N]
    const int32_t* offsets;  // grouped: [E + 1] row offsets into A; dense: null
    int M;                   // dense: rows of A
    int N;                   // output columns (per group)
    int K;
    int E;                   // groups (1 for dense)
    uint32_t* status;
    uint64_t timeout_ns;
    // dense tail pieces: tiles past `full` are cut into `split` column pieces,
    // whose B rows come through the second tensor map (box of BN/split/CTAS rows)
    int full;
    int split;
};

struct Tile {
    int a_row0;   // first row of A (and y) of this CTA's part of the tile
    int row_end;  // rows >= row_end belong to another group (or are past M)
    int b_row0;   // first row of B loaded by this CTA
    int n0;       // first output column
    int group;
    int bn;       // output columns of this tile: BN, or BN / split for a piece of the tail
};

template <int CTAS, int BN>
struct Sched {
    int num_n, num_m, total, E, N, M;
    int full;   // dense: tiles [0, full) are whole; each later tile is cut into `split` pieces
    int split;  // dense: 1 (no cut), 2 or 4 column pieces per tail tile
    uint32_t rank;
    const int* g_tile;  // grouped: prefix sums of tiles per group [E + 1] (smem)
    const int* g_row;   // grouped: row offsets [E + 1] (smem)

    __device__ __forceinline__ Tile get(int t) const {
        Tile ti;
        if (g_tile == nullptr) {
            // The last tiles of a persistent grid whose tile count is not a
            // multiple of the CTA pairs would leave most pairs idle in the
            // final wave: those tiles are cut into `split` column pieces
            // (BN / split columns each), one piece per pair.
            int q = 0;
            ti.bn = BN;
            if (t >= full) {
                const int u = t - full;
                t = full + u / split;
                q = u - (u / split) * split;
                ti.bn = BN / split;
            }
            // groups of RASTER_M row blocks, row block fastest inside a group:
            // the tiles running together share a few row blocks of A and
            // column blocks of B in L2
            const int per_group = RASTER_M * num_n;
            const int g = t / per_group, r = t - g * per_group;
            const int gm = min(RASTER_M, num_m - g * RASTER_M);
            const int mb = g * RASTER_M + r % gm;
            const int nb = r / gm;
            ti.a_row0 = mb * ROWS * CTAS + static_cast<int>(rank) * ROWS;
            ti.row_end = M;
            ti.n0 = nb * BN + q * ti.bn;
            ti.b_row0 = ti.n0 + static_cast<int>(rank) * (ti.bn / CTAS);
            ti.group = 0;
        } else {
            int lo = 0, hi = E;  // e with g_tile[e] <= t < g_tile[e + 1]
            while (hi - lo > 1) {
                const int mid = (lo + hi) >> 1;
                if (g_tile[mid] <= t) lo = mid; else hi = mid;
            }
            const int e = lo;
            const int local = t - g_tile[e];
            const int rows = g_row[e + 1] - g_row[e];
            const int mt = (rows + ROWS * CTAS - 1) / (ROWS * CTAS);
            const int mb = local % mt;
            const int nb = local / mt;
            ti.a_row0 = g_row[e] + mb * ROWS * CTAS + static_cast<int>(rank) * ROWS;
            ti.row_end = g_row[e + 1];
            ti.b_row0 = e * N + nb * BN + static_cast<int>(rank) * (BN / CTAS);
            ti.n0 = nb * BN;
            ti.group = e;
            ti.bn = BN;
        }
        return ti;
    }
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Writes one 32 x 32 BF16 block of the output (lane = row, pk = its 32
// values as packed pairs): staged in the warp's swizzled block (16-byte pieces
// of each 64-byte row XOR-ed with (row>>1)&3, which is the 64-byte TMA
// swizzle, so the row-wise writes and the piece-wise reads are conflict-free),
// then stored by one TMA store when all 32 rows belong to the tile's group
// (the map clips columns past N), else by the lanes, 8 rows x 64 bytes per
// instruction, rows at or past row_end skipped.
__device__ __forceinline__ void put_block(const uint32_t (&pk)[16], int c, const Tile& ti, int q, int lane,
                                          uint8_t* stg, __nv_bfloat16* y, int N, const CUtensorMap* tmY) {
    // the previous block's store has read the staging block
    if (lane == 0) bulk_wait_read();
    __syncwarp();
#pragma unroll
    for (int pc = 0; pc < 4; ++pc)
        *reinterpret_cast<uint4*>(stg + lane * 64 + ((pc ^ ((lane >> 1) & 3)) * 16)) =
            make_uint4(pk[4 * pc], pk[4 * pc + 1], pk[4 * pc + 2], pk[4 * pc + 3]);
    const int row0 = ti.a_row0 + q * 32;
    if (ti.n0 + c * 32 >= N) return;  // a block wholly past the last column: nothing to store
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
        const int row = row0 + rr;
        if (row < ti.row_end && n < N)
            *reinterpret_cast<uint4*>(y + static_cast<size_t>(row) * N + n) = val;
    }
}

// One 32-column chunk of the epilogue: y = bf16(acc * s_a[row] * s_b[n]).
__device__ __forceinline__ void store_chunk(const uint32_t (&v)[32], int c, const Tile& ti, int q,
                                            int lane, float rs, const float* sw,
                                            uint8_t* stg, __nv_bfloat16* y, int N, const CUtensorMap* tmY) {
    uint32_t pk[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        const float lo = __fmul_rn(__fmul_rn(__uint_as_float(v[2 * j]), rs), sw[c * 32 + 2 * j]);
        const float hi = __fmul_rn(__fmul_rn(__uint_as_float(v[2 * j + 1]), rs), sw[c * 32 + 2 * j + 1]);
        pk[j] = pack_bf16x2(lo, hi);
    }
    put_block(pk, c, ti, q, lane, stg, y, N, tmY);
}

// The W16 epilogue chunk: y = bf16(acc), or bf16(acc * sw[n]) with per-column
// scales (SCALED).
template <bool SCALED>
__device__ __forceinline__ void store_chunk_w16(const uint32_t (&v)[32], int c, const Tile& ti, int q,
                                                int lane, const float* sw, uint8_t* stg, const Params& p,
                                                const CUtensorMap* tmY) {
    uint32_t pk[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        float lo = __uint_as_float(v[2 * j]), hi = __uint_as_float(v[2 * j + 1]);
        if constexpr (SCALED) {
            lo = __fmul_rn(lo, sw[c * 32 + 2 * j]);
            hi = __fmul_rn(hi, sw[c * 32 + 2 * j + 1]);
        }
        pk[j] = pack_bf16x2(lo, hi);
    }
    put_block(pk, c, ti, q, lane, stg, p.y, p.N, tmY);
}

template <int CTAS, bool GROUPED, bool ABF16, int BN, bool W16 = false, bool SCALED = false>
__global__ void __launch_bounds__(Layout<CTAS, ABF16, BN, W16, GROUPED>::THREADS_, 1)
fp8_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmBq, const __grid_constant__ CUtensorMap tmY,
                const Params p) {
    using L = Layout<CTAS, ABF16, BN, W16, GROUPED>;
    constexpr int STAGES = L::STAGES;
    constexpr int EPI = L::EPI;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint8_t* sA = smem;
    uint8_t* sB = smem + STAGES * L::A_STAGE;
    uint8_t* astg = smem + STAGES * (L::A_STAGE + L::B_STAGE);  // BF16 staging slots
    uint8_t* staging = smem + L::TILES;
    float* sw_smem = reinterpret_cast<float*>(smem + L::TILES + L::STAGING);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 4);
    int* g_tile = reinterpret_cast<int*>(smem + L::GROUP_OFF);
    int* g_row = g_tile + (MAX_GROUPS + 1);

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const uint32_t rank = CTAS == 2 ? cluster_ctarank() : 0u;
    const bool leader = rank == 0;
    auto full = [&](int s) { return smem_u32(&bars[s]); };
    auto empty = [&](int s) { return smem_u32(&bars[STAGES + s]); };
    auto tfull = [&](int b) { return smem_u32(&bars[2 * STAGES + b]); };
    auto tempty = [&](int b) { return smem_u32(&bars[2 * STAGES + 2 + b]); };
    const uint32_t drain = smem_u32(&bars[2 * STAGES + 4]);
    auto epi_sync = [&](int b) { return smem_u32(&bars[2 * STAGES + 5 + b]); };
    auto bfull = [&](int j) { return smem_u32(&bars[2 * STAGES + 7 + j]); };
    auto bempty = [&](int j) { return smem_u32(&bars[2 * STAGES + 7 + L::ASTG + j]); };

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            // fused quantization: the stage is full when B has landed and every
            // converter warp of both CTAs has written its part of A
            mbar_init(full(s), ABF16 ? 1 + CTAS * CONV_WARPS : 1);
            mbar_init(empty(s), 1);
        }
        for (int j = 0; j < L::ASTG; ++j) {
            mbar_init(bfull(j), 1);
            mbar_init(bempty(j), CONV_WARPS);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull(b), 1);
            mbar_init(tempty(b), CTAS * EPI);
        }
        mbar_init(drain, 1);
        mbar_init(epi_sync(0), EPI * 32);
        mbar_init(epi_sync(1), EPI * 32);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        tma_prefetch_desc(&tmY);
        if (p.split > 1) tma_prefetch_desc(&tmBq);
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

    // Everything above touches only this CTA's shared and tensor memory. The
    // operands, scales and group offsets may be the previous kernel's
    // outputs (PDL launch): wait for it here.
    grid_launch_dependents();
    grid_dependency_wait();

    Sched<CTAS, BN> sc;
    sc.N = p.N;
    sc.M = p.M;
    sc.E = p.E;
    sc.rank = rank;
    sc.num_n = (p.N + BN - 1) / BN;
    sc.split = p.split > 1 ? p.split : 1;
    sc.full = p.split > 1 ? p.full : 0x7fffffff;
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
                    local += ((rows + ROWS * CTAS - 1) / (ROWS * CTAS)) * sc.num_n;
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
                    run += ((rows + ROWS * CTAS - 1) / (ROWS * CTAS)) * sc.num_n;
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
        sc.num_m = (p.M + ROWS * CTAS - 1) / (ROWS * CTAS);
        sc.total = sc.num_m * sc.num_n;
        if (sc.split > 1) sc.total = sc.full + (sc.total - sc.full) * sc.split;
    }
    __syncwarp();
    tc_fence_before();
    if constexpr (CTAS == 2) cluster_sync_all(); else __syncthreads();
    tc_fence_after();
    if constexpr (GROUPED) sc.total = g_tile[p.E];
    const uint32_t tmem_base = *tmem_slot;
    const int num_kb = (p.K + L::KE - 1) / L::KE;
    const int num_st = (num_kb + L::KPS - 1) / L::KPS;  // ring stages per tile
    const int first = CTAS == 2 ? static_cast<int>(blockIdx.x / 2) : static_cast<int>(blockIdx.x);
    const int stride = CTAS == 2 ? static_cast<int>(gridDim.x / 2) : static_cast<int>(gridDim.x);

    if (warp == 0) {
        if (lane == 0) {
            // ---------------------------------------------------------- producer
            int stage = 0;
            uint32_t phase = 0;
            int slot = 0;
            uint32_t sphase = 0;
            uint32_t issued = 0, issued_phase = 0;
            for (int t = first; t < sc.total && !*abort_flag; t += stride) {
                const Tile ti = sc.get(t);
                for (int ks = 0; ks < num_st; ++ks) {
                    const int kb = ks * L::KPS;  // first k-block of the stage
                    if (!mbar_wait(empty(stage), phase ^ 1u, p.timeout_ns, p.status)) {
                        *abort_flag = 1;
                        break;
                    }
                    if constexpr (ABF16) {
                        // B into the stage (counted on the even CTA's barrier);
                        // BF16 A into a staging slot for the converter warps
                        if constexpr (CTAS == 2) {
                            const uint32_t fl = mapa_shared(full(stage), 0);
                            if (leader) mbar_arrive_expect_tx(full(stage), CTAS * L::B_STAGE);
                            tma_load_2d_pair(smem_u32(sB + stage * L::B_STAGE), &tmB, kb * BK, ti.b_row0, fl);
                        } else {
                            mbar_arrive_expect_tx(full(stage), L::B_STAGE);
                            tma_load_2d(smem_u32(sB + stage * L::B_STAGE), &tmB, kb * BK, ti.b_row0, full(stage));
                        }
                        if (!mbar_wait(bempty(slot), sphase ^ 1u, p.timeout_ns, p.status)) {
                            *abort_flag = 1;
                            break;
                        }
                        mbar_arrive_expect_tx(bfull(slot), ASTG_SLOT);
                        const uint32_t dst = smem_u32(astg + slot * ASTG_SLOT);
                        tma_load_2d(dst, &tmA, kb * BK, ti.a_row0, bfull(slot));
                        tma_load_2d(dst + ASTG_SLOT / 2, &tmA, kb * BK + BK / 2, ti.a_row0, bfull(slot));
                        if (++slot == L::ASTG) { slot = 0; sphase ^= 1u; }
                    } else if constexpr (CTAS == 2) {
                        // a tail piece loads only its BN/split columns' rows of B
                        // (a k-block past the end of K is zero-filled and not multiplied)
                        const bool piece = ti.bn != BN;
                        const uint32_t b_bytes = piece ? static_cast<uint32_t>(ti.bn / CTAS) * BK : L::B_BOX;
                        const uint32_t fl = mapa_shared(full(stage), 0);
                        if (leader) mbar_arrive_expect_tx(full(stage), CTAS * L::KPS * (L::A_BOX + b_bytes));
#pragma unroll
                        for (int h = 0; h < L::KPS; ++h) {
                            tma_load_2d_pair(smem_u32(sA + stage * L::A_STAGE + h * L::A_BOX), &tmA,
                                             (kb + h) * L::KE, ti.a_row0, fl);
                            tma_load_2d_pair(smem_u32(sB + stage * L::B_STAGE + h * L::B_BOX),
                                             piece ? &tmBq : &tmB, (kb + h) * L::KE, ti.b_row0, fl);
                        }
                    } else {
                        const bool piece = ti.bn != BN;
                        const uint32_t b_bytes = piece ? static_cast<uint32_t>(ti.bn) * BK : L::B_STAGE;
                        mbar_arrive_expect_tx(full(stage), L::A_STAGE + b_bytes);
                        tma_load_2d(smem_u32(sA + stage * L::A_STAGE), &tmA, kb * L::KE, ti.a_row0, full(stage));
                        tma_load_2d(smem_u32(sB + stage * L::B_STAGE), piece ? &tmBq : &tmB, kb * L::KE,
                                    ti.b_row0, full(stage));
                    }
                    issued |= 1u << stage;
                    issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
            }
            if (*abort_flag) {
                // let the copies in flight land before the CTA exits
                if (ABF16) {
                    const uint64_t t0 = globaltimer_ns();
                    while (globaltimer_ns() - t0 < 100000ull) {}
                } else if (leader) {
                    for (int s = 0; s < STAGES; ++s)
                        if (issued & (1u << s))
                            mbar_wait(full(s), (issued_phase >> s) & 1u, p.timeout_ns, p.status);
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
            int acc = 0;
            uint32_t acc_phase = 0;
            for (int t = first; t < sc.total && !*abort_flag; t += stride) {
                if (!mbar_wait(tempty(acc), acc_phase ^ 1u, p.timeout_ns, p.status)) {
                    *abort_flag = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
                // tail pieces of the dense schedule are narrower (N = BN / split)
                uint32_t idesc = L::IDESC;
                if constexpr (!GROUPED && !W16 && !ABF16) {
                    const int bn = sc.get(t).bn;
                    if (bn != BN) idesc = idesc_e4m3_f32(ROWS * CTAS, bn);
                }
                bool ok = true;
                for (int ks = 0; ks < num_st; ++ks) {
                    if (!mbar_wait(full(stage), phase, p.timeout_ns, p.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
#pragma unroll
                    for (int h = 0; h < L::KPS; ++h) {
                        const int kb = ks * L::KPS + h;
                        if (L::KPS > 1 && kb >= num_kb) break;  // the zero-filled k-block past K
                        const uint64_t adesc =
                            sw128_kmajor_desc(smem_u32(sA + stage * L::A_STAGE + h * L::A_BOX));
                        const uint64_t bdesc =
                            sw128_kmajor_desc(smem_u32(sB + stage * L::B_STAGE + h * L::B_BOX));
#pragma unroll
                        for (int k = 0; k < BK / 32; ++k) {
                            // advance 32 bytes along K inside the swizzled 128-byte rows
                            // (32 bytes: 32 E4M3 or 16 BF16 elements per instruction)
                            const uint32_t accum = (kb > 0 || k > 0) ? 1u : 0u;
                            if constexpr (W16 && CTAS == 2)
                                mma_f16_ss_pair(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, accum);
                            else if constexpr (W16)
                                mma_f16_ss(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, accum);
                            else if constexpr (CTAS == 2)
                                mma_f8f6f4_pair(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, accum);
                            else
                                mma_f8f6f4(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, accum);
                        }
                    }
                    if constexpr (CTAS == 2) mma_commit_pair_mc(empty(stage), 0x3);
                    else mma_commit(empty(stage));
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) {
                    *abort_flag = 1;
                    break;
                }
                if constexpr (CTAS == 2) mma_commit_pair_mc(tfull(acc), 0x3);
                else mma_commit(tfull(acc));
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1u;
            }
            // all MMAs issued by this thread complete before TMEM is released
            if constexpr (CTAS == 2) mma_commit_pair(drain);
            else mma_commit(drain);
            mbar_wait(drain, 0, p.timeout_ns, p.status);
        }
    } else if (ABF16 && warp >= 2 + EPI) {
        // ------------------------------------------------- converters (fused)
        const int ct = threadIdx.x - 32 * (2 + EPI);  // 0 .. 255
        int stage = 0;
        uint32_t phase = 0;
        int slot = 0;
        uint32_t sphase = 0;
        for (int t = first; t < sc.total && !*abort_flag; t += stride) {
            const Tile ti = sc.get(t);
            float invr[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int row = ti.a_row0 + (ct >> 3) + 32 * i;
                invr[i] = row < ti.row_end ? p.inv[row] : 0.0f;
            }
            bool ok = true;
            for (int kb = 0; kb < num_kb; ++kb) {
                if (!mbar_wait(bfull(slot), sphase, p.timeout_ns, p.status) ||
                    !mbar_wait(empty(stage), phase ^ 1u, p.timeout_ns, p.status)) {
                    ok = false;
                    break;
                }
                const uint8_t* src0 = astg + slot * ASTG_SLOT;
                uint8_t* dst0 = sA + stage * L::A_STAGE;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    // 16 elements: row r, E4M3 chunk c (k = 16c .. 16c+15)
                    const int task = ct + 256 * i;
                    const int r = task >> 3, c = task & 7;
                    const uint8_t* src = src0 + (c >> 2) * (ASTG_SLOT / 2) + r * 128;
                    // the two BF16 pieces; the second box's threads take the odd
                    // piece first so that 8 threads of a row hit 8 bank groups
                    const int hb = c >> 2;
                    const int cc = 2 * (c & 3);
                    const uint4 va = *reinterpret_cast<const uint4*>(src + (((cc + hb) ^ (r & 7)) << 4));
                    const uint4 vb = *reinterpret_cast<const uint4*>(src + (((cc + 1 - hb) ^ (r & 7)) << 4));
                    const uint4 v0 = hb ? vb : va;
                    const uint4 v1 = hb ? va : vb;
                    const float inv = invr[i];
                    const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
                    uint32_t o[4];
#pragma unroll
                    for (int q2 = 0; q2 < 4; ++q2)
                        o[q2] = f32x2_to_e4m3x2(__fmul_rn(bf16_lo(w[2 * q2]), inv), __fmul_rn(bf16_hi(w[2 * q2]), inv)) |
                                (f32x2_to_e4m3x2(__fmul_rn(bf16_lo(w[2 * q2 + 1]), inv),
                                                 __fmul_rn(bf16_hi(w[2 * q2 + 1]), inv)) << 16);
                    *reinterpret_cast<uint4*>(dst0 + r * 128 + ((c ^ (r & 7)) << 4)) =
                        make_uint4(o[0], o[1], o[2], o[3]);
                }
                fence_proxy_async_shared();  // generic-proxy writes -> tensor-core reads
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(bempty(slot));
                    if constexpr (CTAS == 2) mbar_arrive_cluster(mapa_shared(full(stage), 0));
                    else mbar_arrive(full(stage));
                }
                if (++slot == L::ASTG) { slot = 0; sphase ^= 1u; }
                if (++stage == STAGES) { stage = 0; phase ^= 1u; }
            }
            if (!ok) {
                *abort_flag = 1;
                break;
            }
        }
    } else if (warp < 2 + EPI) {
        // -------------------------------------------------------------- epilogue
        const int q = warp & 3;           // TMEM lane quadrant this warp may access
        const int et = threadIdx.x - 64;  // 0 .. 32 EPI - 1
        constexpr int CPW = (BN / 32) / (EPI / 4);   // 32-column chunks per warp
        const int c0 = ((warp - 2) / 4) * CPW;       // this warp's first chunk
        uint8_t* stg = staging + (warp - 2) * (32 * 64);
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int t = first; t < sc.total && !*abort_flag; t += stride) {
            const Tile ti = sc.get(t);
            if constexpr (W16) {
                if constexpr (SCALED) {
                    // per-column scales (the default maths' s_w)
                    if (et < BN / 2) {
                        const int n = ti.n0 + 2 * et;
                        sw_smem[acc * BN + 2 * et] = n < p.N ? p.s_b[n] : 0.0f;
                        sw_smem[acc * BN + 2 * et + 1] = n + 1 < p.N ? p.s_b[n + 1] : 0.0f;
                    }
                }
            } else {
                // per-channel scales of this tile into shared memory
                const float* sb = p.s_b + static_cast<size_t>(ti.group) * p.N;
                const int n = ti.n0 + 2 * et;
                const float2 v = n < p.N ? *reinterpret_cast<const float2*>(sb + n) : make_float2(0.f, 0.f);
                if (et < BN / 2) reinterpret_cast<float2*>(sw_smem + acc * BN)[et] = v;
            }
            const int row = ti.a_row0 + q * 32 + lane;
            const float rs = (!W16 && row < ti.row_end) ? p.s_a[row] : 0.0f;
            // all epilogue threads have written their scales (bounded wait)
            mbar_arrive(epi_sync(acc));
            if (!mbar_wait(epi_sync(acc), acc_phase, p.timeout_ns, p.status) ||
                !mbar_wait(tfull(acc), acc_phase, p.timeout_ns, p.status)) {
                *abort_flag = 1;
                break;
            }
            tc_fence_after();
            const float* sw = sw_smem + acc * BN;
            const uint32_t tbase =
                tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * BN);
            // hand the accumulator back once every read of it has completed,
            // without a release fence (which would also wait for this warp's
            // earlier global stores)
            auto hand_back = [&]() {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    if constexpr (CTAS == 2) mbar_arrive_cluster_relaxed(mapa_shared(tempty(acc), 0));
                    else mbar_arrive_relaxed(tempty(acc));
                }
            };
            uint32_t va[32], vb[32];
            if (!GROUPED && !W16 && !ABF16 && ti.bn != BN) {
                // a narrow tail piece: this warp's chunks that fall inside it,
                // one at a time
                const int nval = min(CPW, max(0, (ti.bn - c0 * 32 + 31) / 32));
                for (int i = 0; i < nval; ++i) {
                    tmem_ld_32x32b_x32(tbase + (c0 + i) * 32, va);
                    tmem_ld_wait();
                    if (i + 1 == nval) hand_back();
                    store_chunk(va, c0 + i, ti, q, lane, rs, sw, stg, p.y, p.N, &tmY);
                }
                if (nval == 0) hand_back();
            } else {
                // chunks c0 .. c0 + CPW - 1, the next one loading while this
                // one is stored
                tmem_ld_32x32b_x32(tbase + c0 * 32, va);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < CPW; ++i) {
                    uint32_t(&cur)[32] = (i & 1) ? vb : va;
                    uint32_t(&nxt)[32] = (i & 1) ? va : vb;
                    if (i + 1 < CPW) tmem_ld_32x32b_x32(tbase + (c0 + i + 1) * 32, nxt);
                    else hand_back();
                    if constexpr (W16) store_chunk_w16<SCALED>(cur, c0 + i, ti, q, lane, sw, stg, p, &tmY);
                    else store_chunk(cur, c0 + i, ti, q, lane, rs, sw, stg, p.y, p.N, &tmY);
                    if (i + 1 < CPW) tmem_ld_wait();
                }
            }
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1u;
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

template <int CTAS, bool GROUPED, bool ABF16 = false, int BN = BN_MAX, bool W16 = false, bool SCALED = false>
int prepare(const DeviceInfo& di, size_t smem) {
    static std::atomic<uint64_t> done[64];
    if (static_cast<size_t>(di.max_smem_optin) < smem)
        return fail(METIS_ERR_UNSUPPORTED, "fp8 gemm needs %zu bytes of shared memory", smem);
    return once_per_context(done, di.device, [&] {
        return cuda_check(cudaFuncSetAttribute(fp8_gemm_kernel<CTAS, GROUPED, ABF16, BN, W16, SCALED>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               static_cast<int>(smem)),
                          "cudaFuncSetAttribute(fp8 gemm)");
    });
}

// Co-resident CTA pairs of the 2-CTA kernel (cached per device).
template <bool ABF16 = false, int BN = BN_MAX, bool GROUPED = false, bool W16 = false, bool SCALED = false>
int max_pairs(const DeviceInfo& di, int* out) {
    static int cached[64];
    if (!cached[di.device]) {
        using L = Layout<2, ABF16, BN, W16, GROUPED>;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * (di.num_sms / 2), 1, 1);
        cfg.blockDim = dim3(L::THREADS_, 1, 1);
        cfg.dynamicSmemBytes = GROUPED ? L::BYTES_GROUPED : L::BYTES_DENSE;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        int rc = cuda_check(cudaOccupancyMaxActiveClusters(&n, fp8_gemm_kernel<2, GROUPED, ABF16, BN, W16, SCALED>, &cfg),
                            "cudaOccupancyMaxActiveClusters");
        if (rc) return rc;
        if (n < 1) return fail(METIS_ERR_UNSUPPORTED, "no CTA pair of the fp8 gemm fits an SM pair");
        cached[di.device] = n;
    }
    *out = cached[di.device];
    return METIS_OK;
}

// The persistent grid runs `tiles` whole tiles on `workers` CTAs (pairs): the
// last tiles % workers of them form a final wave that keeps few workers busy
// (4096 x 6144 on 74 pairs: 384 tiles, 14 in the last wave). When that wave
// would occupy at most a quarter of the workers, each of its tiles is cut into
// 4 column pieces of BN/4 columns, one piece per worker. Measured on B200:
// 4096 x 6144 x 2048 45.4 against 45.9 us; halves for a final wave of up to
// half the workers measured slower (2560 x 8000 x 2048: 43.2 against 39.2 us),
// so only quarters are cut.
inline int tail_split(int tiles, int workers) {
    if (tiles <= workers) return 1;
    const int r = tiles % workers;
    return (r > 0 && 4 * r <= workers) ? 4 : 1;
}

// Dense E4M3 GEMM with BN-column tiles: CTA pairs (256-row tiles) for
// M > 128, single CTAs otherwise; the final partial wave in column pieces.
template <int BN>
int launch_dense(const DeviceInfo& di, const CUtensorMap& ta, const uint8_t* b, Params p,
                 int M, int N, int K, cudaStream_t st) {
    int rc;
    CUtensorMap tb, tbq, ty;
    const int num_n = (N + BN - 1) / BN;
    if ((rc = make_tmap_2d_sw64(&ty, p.y, 2, N, M, static_cast<uint64_t>(N) * 2, 32, 32))) return rc;
    if (M > ROWS) {
        using L = Layout<2, false, BN>;
        if ((rc = prepare<2, false, false, BN>(di, L::BYTES_DENSE))) return rc;
        int pairs = 0;
        if ((rc = max_pairs<false, BN>(di, &pairs))) return rc;
        if ((rc = make_tmap_2d(&tb, b, 1, K, N, K, BK, L::B_ROWS, true))) return rc;
        const int tiles = ((M + 2 * ROWS - 1) / (2 * ROWS)) * num_n;
        const int clusters = tiles < pairs ? tiles : pairs;
        p.split = tail_split(tiles, clusters);
        p.full = tiles - (p.split > 1 ? tiles % clusters : 0);
        tbq = tb;
        if (p.split > 1 &&
            (rc = make_tmap_2d(&tbq, b, 1, K, N, K, BK, static_cast<uint32_t>(L::B_ROWS / p.split), true)))
            return rc;
        return cuda_check(launch_pdl(fp8_gemm_kernel<2, false, false, BN>, dim3(2 * clusters), dim3(L::THREADS_),
                                     L::BYTES_DENSE, st, 2, ta, tb, tbq, ty, p),
                          "fp8 gemm (CTA pair) launch");
    }
    using L = Layout<1, false, BN>;
    if ((rc = prepare<1, false, false, BN>(di, L::BYTES_DENSE))) return rc;
    if ((rc = make_tmap_2d(&tb, b, 1, K, N, K, BK, L::B_ROWS, true))) return rc;
    const int tiles = ((M + ROWS - 1) / ROWS) * num_n;
    const int grid = tiles < di.num_sms ? tiles : di.num_sms;
    p.split = tail_split(tiles, grid);
    p.full = tiles - (p.split > 1 ? tiles % grid : 0);
    tbq = tb;
    if (p.split > 1 &&
        (rc = make_tmap_2d(&tbq, b, 1, K, N, K, BK, static_cast<uint32_t>(L::B_ROWS / p.split), true)))
        return rc;
    return cuda_check(launch_pdl(fp8_gemm_kernel<1, false, false, BN>, dim3(grid), dim3(L::THREADS_),
                                 L::BYTES_DENSE, st, 1, ta, tb, tbq, ty, p),
                      "fp8 gemm launch");
}

}  // namespace gemm

// Dense W8A8 GEMM launch (arguments validated by the caller).
int launch_fp8_gemm_dense(const uint8_t* a, const float* s_a, const uint8_t* b, const float* s_b,
                          __nv_bfloat16* y, int M, int N, int K, cudaStream_t st) {
    using namespace gemm;
    DeviceInfo di;
    int rc = current_device_info(&di);
    if (rc) return rc;
    uint32_t* status = nullptr;
    if ((rc = device_status_word(&status))) return rc;
    Params p{s_a, nullptr, s_b, y, nullptr, M, N, K, 1, status, watchdog_ns()};
    CUtensorMap ta;
    if ((rc = make_tmap_2d(&ta, a, 1, K, M, K, BK, ROWS, true))) return rc;
    // 256-column tiles: 192-column ones fill the waves better for some shapes
    // (M = 4096, N = 6144: 6.9 instead of 5.2 waves on 74 CTA pairs) but
    // measured 7-25% slower on B200 (more operand traffic per FLOP).
    return launch_dense<BN_MAX>(di, ta, b, p, M, N, K, st);
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
    uint32_t* status = nullptr;
    if ((rc = device_status_word(&status))) return rc;
    Params p{s_a, nullptr, s_b, y, offsets, rows, N, K, E, status, watchdog_ns()};
    CUtensorMap ta, tb, ty;
    if ((rc = make_tmap_2d(&ta, a, 1, K, rows, K, BK, ROWS, true))) return rc;
    if ((rc = make_tmap_2d_sw64(&ty, y, 2, N, rows, static_cast<uint64_t>(N) * 2, 32, 32))) return rc;
    if (K < 1024) {
        // short k-loops: 128-row single-CTA tiles
        using L = Layout<1, false, BN_MAX, false, true>;
        if ((rc = prepare<1, true>(di, L::BYTES_GROUPED))) return rc;
        if ((rc = make_tmap_2d(&tb, b, 1, K, static_cast<uint64_t>(E) * N, K, BK, L::B_ROWS, true)))
            return rc;
        return cuda_check(launch_pdl(fp8_gemm_kernel<1, true, false, BN_MAX>, dim3(di.num_sms), dim3(L::THREADS_),
                                     L::BYTES_GROUPED, st, 1, ta, tb, tb, ty, p),
                          "grouped fp8 gemm launch");
    }
    // CTA pairs on 256-row tiles: each SM streams half of B (routed
    // up-projection, K = 2048: 72 -> 66 us)
    using L = Layout<2, false, BN_MAX, false, true>;
    if ((rc = prepare<2, true>(di, L::BYTES_GROUPED))) return rc;
    int pairs = 0;
    if ((rc = max_pairs<false, BN_MAX, true>(di, &pairs))) return rc;
    if ((rc = make_tmap_2d(&tb, b, 1, K, static_cast<uint64_t>(E) * N, K, BK, L::B_ROWS, true)))
        return rc;
    return cuda_check(launch_pdl(fp8_gemm_kernel<2, true, false, BN_MAX>, dim3(2 * pairs), dim3(L::THREADS_),
                                 L::BYTES_GROUPED, st, 2, ta, tb, tb, ty, p),
                      "grouped fp8 gemm (CTA pair) launch");
}

// Fused-quantization W8A8 GEMM launch: a is BF16 [M, K]; inv [M] holds
// 448/amax per row (written by the scales-only quantizer pass).
int launch_fp8_gemm_fused(const __nv_bfloat16* a, const float* s_a, const float* inv,
                          const uint8_t* b, const float* s_b, __nv_bfloat16* y, int M, int N, int K,
                          cudaStream_t st) {
    using namespace gemm;
    DeviceInfo di;
    int rc = current_device_info(&di);
    if (rc) return rc;
    uint32_t* status = nullptr;
    if ((rc = device_status_word(&status))) return rc;
    Params p{s_a, inv, s_b, y, nullptr, M, N, K, 1, status, watchdog_ns()};
    const int num_n = (N + BN_MAX - 1) / BN_MAX;
    CUtensorMap ta, tb, ty;
    if ((rc = make_tmap_2d(&ta, a, 2, K, M, static_cast<uint64_t>(K) * 2, BK / 2, ROWS, true))) return rc;
    if ((rc = make_tmap_2d_sw64(&ty, y, 2, N, M, static_cast<uint64_t>(N) * 2, 32, 32))) return rc;
    if (M > ROWS) {
        using L = Layout<2, true>;
        if ((rc = prepare<2, false, true>(di, L::BYTES_DENSE))) return rc;
        int pairs = 0;
        if ((rc = max_pairs<true>(di, &pairs))) return rc;
        if ((rc = make_tmap_2d(&tb, b, 1, K, N, K, BK, L::B_ROWS, true))) return rc;
        const int tiles = ((M + 2 * ROWS - 1) / (2 * ROWS)) * num_n;
        const int clusters = tiles < pairs ? tiles : pairs;
        return cuda_check(launch_pdl(fp8_gemm_kernel<2, false, true, BN_MAX>, dim3(2 * clusters), dim3(L::THREADS_),
                                     L::BYTES_DENSE, st, 2, ta, tb, tb, ty, p),
                          "fused fp8 gemm (CTA pair) launch");
    }
    using L = Layout<1, true>;
    if ((rc = prepare<1, false, true>(di, L::BYTES_DENSE))) return rc;
    if ((rc = make_tmap_2d(&tb, b, 1, K, N, K, BK, L::B_ROWS, true))) return rc;
    const int tiles = ((M + ROWS - 1) / ROWS) * num_n;
    const int grid = tiles < di.num_sms ? tiles : di.num_sms;
    return cuda_check(launch_pdl(fp8_gemm_kernel<1, false, true, BN_MAX>, dim3(grid), dim3(L::THREADS_),
                                 L::BYTES_DENSE, st, 1, ta, tb, tb, ty, p),
                      "fused fp8 gemm launch");
}

// BF16 x BF16 GEMM y = bf16(a b^T) on the tcgen05 pipeline (CTA pairs for
// M > 128). Arguments validated by the caller.
namespace gemm {

template <bool SCALED>
int launch_w16(const __nv_bfloat16* a, const __nv_bfloat16* b, const Params& p, int M, int N, int K,
               const DeviceInfo& di, cudaStream_t st) {
    int rc;
    const int num_n = (N + BN_MAX - 1) / BN_MAX;
    CUtensorMap ta, tb, ty;
    if ((rc = make_tmap_2d(&ta, a, 2, K, M, static_cast<uint64_t>(K) * 2, BK / 2, ROWS, true))) return rc;
    if ((rc = make_tmap_2d_sw64(&ty, p.y, 2, N, M, static_cast<uint64_t>(N) * 2, 32, 32))) return rc;
    if (M > ROWS) {
        using L = Layout<2, false, BN_MAX, true>;
        if ((rc = prepare<2, false, false, BN_MAX, true, SCALED>(di, L::BYTES_DENSE))) return rc;
        int pairs = 0;
        if ((rc = max_pairs<false, BN_MAX, false, true, SCALED>(di, &pairs))) return rc;
        if ((rc = make_tmap_2d(&tb, b, 2, K, N, static_cast<uint64_t>(K) * 2, BK / 2, L::B_ROWS, true)))
            return rc;
        const int tiles = ((M + 2 * ROWS - 1) / (2 * ROWS)) * num_n;
        const int clusters = tiles < pairs ? tiles : pairs;
        return cuda_check(launch_pdl(fp8_gemm_kernel<2, false, false, BN_MAX, true, SCALED>, dim3(2 * clusters),
                                     dim3(L::THREADS_), L::BYTES_DENSE, st, 2, ta, tb, tb, ty, p),
                          "bf16 gemm (CTA pair) launch");
    }
    using L = Layout<1, false, BN_MAX, true>;
    if ((rc = prepare<1, false, false, BN_MAX, true, SCALED>(di, L::BYTES_DENSE))) return rc;
    if ((rc = make_tmap_2d(&tb, b, 2, K, N, static_cast<uint64_t>(K) * 2, BK / 2, L::B_ROWS, true))) return rc;
    const int tiles = ((M + ROWS - 1) / ROWS) * num_n;
    const int grid = tiles < di.num_sms ? tiles : di.num_sms;
    return cuda_check(launch_pdl(fp8_gemm_kernel<1, false, false, BN_MAX, true, SCALED>, dim3(grid),
                                 dim3(L::THREADS_), L::BYTES_DENSE, st, 1, ta, tb, tb, ty, p),
                      "bf16 gemm launch");
}

}  // namespace gemm

int launch_bf16_gemm(const __nv_bfloat16* a, const __nv_bfloat16* b, __nv_bfloat16* y, int M, int N,
                     int K, const float* s_b, cudaStream_t st) {
    using namespace gemm;
    DeviceInfo di;
    int rc = current_device_info(&di);
    if (rc) return rc;
    uint32_t* status = nullptr;
    if ((rc = device_status_word(&status))) return rc;
    Params p{nullptr, nullptr, s_b, y, nullptr, M, N, K, 1, status, watchdog_ns()};
    return s_b != nullptr ? launch_w16<true>(a, b, p, M, N, K, di, st) : launch_w16<false>(a, b, p, M, N, K, di, st);
}

}  // namespace metis

using namespace metis;

extern "C" int metis_bf16_gemm(const void* x_bf16, const void* w_bf16, void* y_bf16, int64_t M,
                               int64_t N, int64_t K, metis_stream_t stream) {
    clear_error();
    if (M < 0 || N < 8 || N % 8 || K < 8 || K % 8 || M > 0x7fffffff || N > 0x7fffffff || K > 0x7fffffff)
        return fail(METIS_ERR_INVALID_ARG,
                    "bf16_gemm: need M >= 0, N and K multiples of 8 (M=%lld N=%lld K=%lld)", (long long)M,
                    (long long)N, (long long)K);
    if (M == 0) return METIS_OK;
    if (!x_bf16 || !w_bf16 || !y_bf16) return fail(METIS_ERR_INVALID_ARG, "bf16_gemm: null pointer");
    if (!aligned(x_bf16, 16) || !aligned(w_bf16, 16) || !aligned(y_bf16, 16))
        return fail(METIS_ERR_INVALID_ARG, "bf16_gemm: x, w and y must be 16-byte aligned");
    return launch_bf16_gemm(static_cast<const __nv_bfloat16*>(x_bf16), static_cast<const __nv_bfloat16*>(w_bf16),
                            static_cast<__nv_bfloat16*>(y_bf16), static_cast<int>(M), static_cast<int>(N),
                            static_cast<int>(K), nullptr, static_cast<cudaStream_t>(stream));
}

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
    // fused quantization: scales pass (s_tok out, 448/amax into the workspace),
    // then the GEMM that quantizes A tiles in shared memory
    const size_t need = metis_workspace_size(METIS_OP_FP8_GEMM_FUSED, M, N, K, 0, 0);
    if (!workspace || ws_bytes < need || !aligned(workspace, 16))
        return fail(METIS_ERR_INVALID_ARG,
                    "fp8_gemm (BF16 A): needs a 16-byte aligned workspace of %zu bytes (got %zu)",
                    need, ws_bytes);
    float* inv = static_cast<float*>(workspace);
    int rc = launch_quant_rows<__nv_bfloat16>(static_cast<const __nv_bfloat16*>(a), M, K, K, nullptr,
                                              K, s_tok, st, nullptr, 1, inv);
    if (rc) return rc;
    return launch_fp8_gemm_fused(static_cast<const __nv_bfloat16*>(a), s_tok, inv, wq, s_w,
                                 static_cast<__nv_bfloat16*>(y_bf16), static_cast<int>(M),
                                 static_cast<int>(N), static_cast<int>(K), st);
}
