// Routed-expert W8A8 layer: the FP8 linear layer grouped over top-k routed
// experts ("Lernex/Metis-1.6-Logos-FP8", "What is in FP8": the routed experts
// are FP8, E4M3 with one scale per output channel, activations quantized per
// token at run time).
//
// Device pipeline (no host synchronisation; segment sizes stay on the GPU):
//   1. routing histogram per chunk of slots    (shared-memory integer atomics)
//   2. prefix sums: per-expert offsets and per-(chunk, expert) bases
//   3. stable ranks: row of slot s = t*topk + j in expert order, via warp
//      match + per-warp counts (no atomics decide the order)
//   4. per-token quantization of x, each token once, its codes and scale
//      written straight into the expert-ordered rows it was routed to
//   5. grouped up-projection (tcgen05 W8A8 GEMM, tile schedule from offsets)
//   6. per-row re-quantization of h
//   7. grouped down-projection
//   8. weighted un-permute y[t] = sum_j w[t,j] * o[row(t,j)], FP32, j ascending.
#include <algorithm>
#include <atomic>
#include <mutex>

#include "common.cuh"
#include "../../include/metis_nvfp4.h"

namespace metis {

int launch_fp8_gemm_grouped(const uint8_t* a, const float* s_a, const uint8_t* b, const float* s_b,
                            __nv_bfloat16* y, const int32_t* offsets, int E, int rows, int N,
                            int K, cudaStream_t st);
int64_t moe_region_offset(int region, int64_t T, int64_t topk, int64_t E, int64_t H, int64_t I,
                          int64_t* total);
int64_t moe4_padded_rows(int64_t T, int64_t topk, int64_t E);
int64_t moe4_region_offset(int region, int64_t T, int64_t topk, int64_t E, int64_t H, int64_t I,
                           int64_t* total);

namespace moe {

constexpr int CHUNK = 256;   // slots per routing CTA (one per thread)
constexpr int MAX_E = 1024;

// chunk_counts[c][e] = number of slots of chunk c routed to expert e.
// Ids outside [0, E) are dropped and flagged in the device status word.
__global__ void __launch_bounds__(CHUNK) count_kernel(const int32_t* __restrict__ ids, int S, int E,
                                                      int32_t* __restrict__ chunk_counts,
                                                      uint32_t* status) {
    __shared__ int cnt[MAX_E];
    for (int e = threadIdx.x; e < E; e += CHUNK) cnt[e] = 0;
    __syncthreads();
    const int s = blockIdx.x * CHUNK + threadIdx.x;
    if (s < S) {
        const int e = ids[s];
        if (e >= 0 && e < E) atomicAdd(&cnt[e], 1);
        else atomicOr(status, kDevErrBadIndex);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += CHUNK)
        chunk_counts[static_cast<size_t>(blockIdx.x) * E + e] = cnt[e];
}

// counts[e], offsets[e] (exclusive, E + 1 entries) and, in place,
// chunk_counts[c][e] -> base row of chunk c's slots of expert e.
// One CTA of 1024 threads: G = 1024 / Ep threads per expert (Ep = E rounded
// up to a power of two) each own a contiguous run of chunks, so the counts
// are read in one batch of loads per thread rather than C sequential ones.
constexpr int SCAN_THREADS = 1024;
constexpr int SCAN_BATCH = 8;
// pad > 1: each expert's first row is a multiple of pad (its rows padded up
// to one); row_to_slot of the pad rows is set to -1 when r2s_pad is non-null.
__global__ void __launch_bounds__(SCAN_THREADS) scan_kernel(int32_t* __restrict__ chunk_counts, int C,
                                                            int E, int32_t* __restrict__ counts,
                                                            int32_t* __restrict__ offsets, int pad,
                                                            int32_t* __restrict__ r2s_pad) {
    __shared__ int part[SCAN_THREADS];  // [g][e]: sums, then prefix over g
    __shared__ int warp_tot[32];
    __shared__ int excl_e[MAX_E];
    __shared__ int cnt_e[MAX_E];
    int Ep = 1;
    while (Ep < E) Ep <<= 1;
    const int G = SCAN_THREADS / Ep;
    const int e = threadIdx.x % Ep, g = threadIdx.x / Ep;
    const int c0 = static_cast<int>(static_cast<int64_t>(g) * C / G);
    const int c1 = static_cast<int>(static_cast<int64_t>(g + 1) * C / G);
    int local = 0;
    int first[SCAN_BATCH];  // this thread's first batch of counts, kept for the bases pass
    if (e < E) {
        for (int c = c0; c < c1; c += SCAN_BATCH) {
            int v[SCAN_BATCH];
#pragma unroll
            for (int i = 0; i < SCAN_BATCH; ++i)
                v[i] = c + i < c1 ? chunk_counts[static_cast<size_t>(c + i) * E + e] : 0;
#pragma unroll
            for (int i = 0; i < SCAN_BATCH; ++i) local += v[i];
            if (c == c0) {
#pragma unroll
                for (int i = 0; i < SCAN_BATCH; ++i) first[i] = v[i];
            }
        }
    }
    part[g * Ep + e] = local;
    __syncthreads();
    // thread t < Ep: expert t's total, and the exclusive prefix of its parts over g
    int total = 0;
    if (threadIdx.x < Ep) {
        for (int gg = 0; gg < G; ++gg) {
            const int v = part[gg * Ep + threadIdx.x];
            part[gg * Ep + threadIdx.x] = total;
            total += v;
        }
    }
    // block-wide exclusive scan of the padded totals over e (thread t holds expert t)
    const int ptotal = (total + pad - 1) / pad * pad;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = ptotal;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int w = warp_tot[lane];
        int wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += v;
        }
        warp_tot[lane] = wi - w;  // exclusive prefix of warp totals
    }
    __syncthreads();
    if (threadIdx.x < E) {
        const int excl = warp_tot[warp] + incl - ptotal;
        counts[threadIdx.x] = total;
        offsets[threadIdx.x] = excl;
        excl_e[threadIdx.x] = excl;
        cnt_e[threadIdx.x] = total;
        if (threadIdx.x == E - 1) offsets[E] = excl + ptotal;
    }
    __syncthreads();
    // pad rows (fewer than pad per expert) marked -1, by all threads
    if (r2s_pad) {
        for (int i = threadIdx.x; i < E * pad; i += SCAN_THREADS) {
            const int ee = i / pad, k = i - ee * pad;
            const int c = cnt_e[ee];
            if (k < (c + pad - 1) / pad * pad - c) r2s_pad[excl_e[ee] + c + k] = -1;
        }
    }
    // chunk bases: this thread's run of chunks, from its expert's offset plus
    // the counts of the runs before it
    if (e < E) {
        int run = excl_e[e] + part[g * Ep + e];
        for (int c = c0; c < c1; c += SCAN_BATCH) {
            int v[SCAN_BATCH];
            if (c == c0) {
                // the first batch is still in registers (a run of up to
                // SCAN_BATCH chunks, the common case, is read once)
#pragma unroll
                for (int i = 0; i < SCAN_BATCH; ++i) v[i] = first[i];
            } else {
#pragma unroll
                for (int i = 0; i < SCAN_BATCH; ++i)
                    v[i] = c + i < c1 ? chunk_counts[static_cast<size_t>(c + i) * E + e] : 0;
            }
#pragma unroll
            for (int i = 0; i < SCAN_BATCH; ++i) {
                if (c + i < c1) chunk_counts[static_cast<size_t>(c + i) * E + e] = run;
                run += v[i];
            }
        }
    }
}

// Stable rank of each slot within its expert: slots of the chunk are ranked
// by warp (match + popcount) and then by the per-warp counts of earlier warps.
__global__ void __launch_bounds__(CHUNK) rank_kernel(const int32_t* __restrict__ ids, int S, int E,
                                                     const int32_t* __restrict__ chunk_base,
                                                     int32_t* __restrict__ slot_to_row,
                                                     int32_t* __restrict__ row_to_slot) {
    constexpr int WARPS = CHUNK / 32;
    __shared__ int wcnt[WARPS][MAX_E];  // per-warp counts, then exclusive prefix over warps
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    for (int i = threadIdx.x; i < WARPS * E; i += CHUNK) wcnt[i / E][i % E] = 0;
    __syncthreads();
    const int s = blockIdx.x * CHUNK + threadIdx.x;
    int e = s < S ? ids[s] : -1;
    if (e >= E) e = -1;
    const bool ok = e >= 0;
    if (s < S && !ok) slot_to_row[s] = -1;  // dropped: never written or read again
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int rank_w = __popc(peers & ((1u << lane) - 1u));
    if (ok && rank_w == 0) wcnt[warp][e] = __popc(peers);
    __syncthreads();
    for (int x = threadIdx.x; x < E; x += CHUNK) {
        int run = 0;
        for (int w = 0; w < WARPS; ++w) {
            const int v = wcnt[w][x];
            wcnt[w][x] = run;
            run += v;
        }
    }
    __syncthreads();
    if (ok) {
        const int row = chunk_base[static_cast<size_t>(blockIdx.x) * E + e] + wcnt[warp][e] + rank_w;
        slot_to_row[s] = row;
        row_to_slot[row] = s;
    }
}

// The prefix sums and the stable ranks in one kernel, for routing tables that
// fit in shared memory (C * E <= RS_MAX_TAB counts, E <= RS_MAX_E): every
// block reads the whole per-chunk count table (a few tens of KB from L2),
// derives each expert's total, its own chunk's base row and the expert
// offsets (padded to `pad` rows), and ranks its chunk as rank_kernel does.
// Block 0 writes counts and offsets; the pad rows of expert e (row_to_slot
// -1) are marked by block e % gridDim.x. Saves the single-block scan kernel
// and its launch.
constexpr int RS_MAX_TAB = 16384;
constexpr int RS_MAX_E = 256;
__global__ void __launch_bounds__(CHUNK) rank_scan_kernel(const int32_t* __restrict__ ids, int S, int E,
                                                          const int32_t* __restrict__ chunk_counts,
                                                          int32_t* __restrict__ counts,
                                                          int32_t* __restrict__ offsets, int pad,
                                                          int32_t* __restrict__ slot_to_row,
                                                          int32_t* __restrict__ row_to_slot) {
    constexpr int WARPS = CHUNK / 32;
    extern __shared__ int tab[];                 // [C][E] counts of every chunk
    __shared__ int wcnt[WARPS][RS_MAX_E];        // per-warp counts, then exclusive prefix over warps
    __shared__ int part_tot[CHUNK];              // [g][e] partial totals over chunk groups
    __shared__ int part_bef[CHUNK];              // [g][e] partial counts of the chunks before this one
    __shared__ int base_e[RS_MAX_E];             // this chunk's first row of expert e
    __shared__ int warp_tot[WARPS];
    const int C = gridDim.x;
    const int c = blockIdx.x;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    // the count table, and this chunk's warp-level ranks meanwhile
    if ((C * E & 3) == 0) {
        const int4* src = reinterpret_cast<const int4*>(chunk_counts);
        for (int i = threadIdx.x; i < C * E / 4; i += CHUNK) reinterpret_cast<int4*>(tab)[i] = src[i];
    } else {
        for (int i = threadIdx.x; i < C * E; i += CHUNK) tab[i] = chunk_counts[i];
    }
    for (int i = threadIdx.x; i < WARPS * E; i += CHUNK) wcnt[i / E][i % E] = 0;
    const int s = c * CHUNK + threadIdx.x;
    int e = s < S ? ids[s] : -1;
    if (e >= E) e = -1;
    const bool ok = e >= 0;
    if (s < S && !ok) slot_to_row[s] = -1;  // dropped: never written or read again
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int rank_w = __popc(peers & ((1u << lane) - 1u));
    __syncthreads();
    if (ok && rank_w == 0) wcnt[warp][e] = __popc(peers);
    // expert x's total and the count of its slots in chunks before c:
    // G = CHUNK / Ep groups of threads each sum a run of chunks
    int Ep = 1;
    while (Ep < E) Ep <<= 1;
    const int G = CHUNK / Ep;
    {
        const int x = threadIdx.x % Ep, g = threadIdx.x / Ep;
        const int c0 = g * C / G, c1 = (g + 1) * C / G;
        int tot = 0, bef = 0;
        if (x < E)
            for (int cc = c0; cc < c1; ++cc) {
                const int v = tab[cc * E + x];
                tot += v;
                if (cc < c) bef += v;
            }
        part_tot[g * Ep + x] = tot;
        part_bef[g * Ep + x] = bef;
    }
    __syncthreads();
    // thread t < Ep: expert t's total (padded) and its exclusive prefix over experts
    int total = 0, before = 0;
    if (threadIdx.x < Ep) {
        for (int g = 0; g < G; ++g) {
            total += part_tot[g * Ep + threadIdx.x];
            before += part_bef[g * Ep + threadIdx.x];
        }
    }
    const int ptotal = (total + pad - 1) / pad * pad;
    int incl = ptotal;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) warp_tot[warp] = incl;
    // per-warp exclusive prefix over experts (and warp prefix sums for x)
    for (int i = threadIdx.x; i < E; i += CHUNK) {
        int run = 0;
        for (int w = 0; w < WARPS; ++w) {
            const int v = wcnt[w][i];
            wcnt[w][i] = run;
            run += v;
        }
    }
    __syncthreads();
    int wbase = 0;
    for (int w = 0; w < warp; ++w) wbase += warp_tot[w];
    if (threadIdx.x < E) {
        const int excl = wbase + incl - ptotal;  // offset of expert threadIdx.x
        base_e[threadIdx.x] = excl + before;
        if (c == 0) {
            counts[threadIdx.x] = total;
            offsets[threadIdx.x] = excl;
            if (threadIdx.x == E - 1) offsets[E] = excl + ptotal;
        }
        // pad rows (fewer than pad per expert), expert x by block x % C
        if (pad > 1 && threadIdx.x % C == c)
            for (int k = total; k < ptotal; ++k) row_to_slot[excl + k] = -1;
    }
    __syncthreads();
    if (ok) {
        const int row = base_e[e] + wcnt[warp][e] + rank_w;
        slot_to_row[s] = row;
        row_to_slot[row] = s;
    }
}

// y[t, n..n+7] = bf16( s[t, n..n+7] + sum_j w[t, j] * o[slot_to_row[t*topk + j], n..n+7] ),
// s the shared expert's BF16 output (null: 0).
// HBM-bound. A persistent grid walks the (token, 8-column group) items with
// a stride of its thread count. For topk <= COMBINE_MAXK a thread issues
// every row load of its item before the first add (topk 16-byte loads in
// flight) and reads the next item's row indices and weights while they are
// in flight, so the index round trip is off the critical path. Three blocks
// per SM (80 registers a thread): two blocks, unbounded, measured slower.
// The sum starts from s and runs over j in ascending order in FP32 either
// way.
constexpr int COMBINE_MAXK = 8;
__global__ void __launch_bounds__(256, 3) combine_kernel(const __nv_bfloat16* __restrict__ o,
                                                      const float* __restrict__ w,
                                                      const int32_t* __restrict__ slot_to_row,
                                                      int T, int topk, int H,
                                                      __nv_bfloat16* __restrict__ y,
                                                      const __nv_bfloat16* __restrict__ s) {
    const int groups = H / 8;
    const int64_t total = static_cast<int64_t>(T) * groups;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    auto start = [&](int64_t i, float (&acc)[8]) {
        const int t = static_cast<int>(i / groups);
        const int n = static_cast<int>(i - static_cast<int64_t>(t) * groups) * 8;
#pragma unroll
        for (int k = 0; k < 8; ++k) acc[k] = 0.0f;
        if (s != nullptr) {
            const uint4 v = *reinterpret_cast<const uint4*>(s + static_cast<size_t>(t) * H + n);
            const uint32_t sv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                acc[2 * k] = bf16_lo(sv[k]);
                acc[2 * k + 1] = bf16_hi(sv[k]);
            }
        }
    };
    auto add = [&](float (&acc)[8], float wj, const uint4& c) {
        const uint32_t v[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            acc[2 * k] = fmaf(wj, bf16_lo(v[k]), acc[2 * k]);
            acc[2 * k + 1] = fmaf(wj, bf16_hi(v[k]), acc[2 * k + 1]);
        }
    };
    auto finish = [&](int64_t i, const float (&acc)[8]) {
        const int t = static_cast<int>(i / groups);
        const int n = static_cast<int>(i - static_cast<int64_t>(t) * groups) * 8;
        uint4 out;
        out.x = pack_bf16x2(acc[0], acc[1]);
        out.y = pack_bf16x2(acc[2], acc[3]);
        out.z = pack_bf16x2(acc[4], acc[5]);
        out.w = pack_bf16x2(acc[6], acc[7]);
        *reinterpret_cast<uint4*>(y + static_cast<size_t>(t) * H + n) = out;
    };
    if (topk <= COMBINE_MAXK) {
        // row indices (-1: no row) and weights of an item's token
        auto fetch = [&](int64_t i, int (&r)[COMBINE_MAXK], float (&wj)[COMBINE_MAXK]) {
            const int64_t t = i / groups;
#pragma unroll
            for (int j = 0; j < COMBINE_MAXK; ++j) {
                r[j] = -1;
                wj[j] = 0.0f;
                if (j < topk) {
                    r[j] = slot_to_row[t * topk + j];
                    wj[j] = w[t * topk + j];
                }
            }
        };
        int r[COMBINE_MAXK];
        float wj[COMBINE_MAXK];
        if (idx < total) fetch(idx, r, wj);
        while (idx < total) {
            const int n = static_cast<int>(idx % groups) * 8;
            uint4 c[COMBINE_MAXK];
#pragma unroll
            for (int j = 0; j < COMBINE_MAXK; ++j)
                if (r[j] >= 0) c[j] = *reinterpret_cast<const uint4*>(o + static_cast<size_t>(r[j]) * H + n);
            float acc[8];
            start(idx, acc);
            const int64_t next = idx + stride;
            int rn[COMBINE_MAXK];
            float wn[COMBINE_MAXK];
            if (next < total) fetch(next, rn, wn);
#pragma unroll
            for (int j = 0; j < COMBINE_MAXK; ++j)
                if (r[j] >= 0) add(acc, wj[j], c[j]);
            finish(idx, acc);
            idx = next;
#pragma unroll
            for (int j = 0; j < COMBINE_MAXK; ++j) {
                r[j] = rn[j];
                wj[j] = wn[j];
            }
        }
    } else {
        for (; idx < total; idx += stride) {
            const int64_t t = idx / groups;
            const int n = static_cast<int>(idx % groups) * 8;
            float acc[8];
            start(idx, acc);
            for (int j = 0; j < topk; ++j) {
                const int rj = slot_to_row[t * topk + j];
                if (rj < 0) continue;
                add(acc, w[t * topk + j], *reinterpret_cast<const uint4*>(o + static_cast<size_t>(rj) * H + n));
            }
            finish(idx, acc);
        }
    }
}

// Launches the combine on a persistent grid: as many 256-thread blocks as
// fit on the device at once (occupancy cached per device), at most one per
// 256 items.
int launch_combine(const __nv_bfloat16* o, const float* w, const int32_t* slot_to_row, int64_t T,
                   int64_t topk, int64_t H, __nv_bfloat16* y, const __nv_bfloat16* s, cudaStream_t st) {
    DeviceInfo di;
    int rc;
    if ((rc = current_device_info(&di))) return rc;
    static std::atomic<int> per_sm[64];
    int occ = per_sm[di.device & 63].load(std::memory_order_relaxed);
    if (occ == 0) {
        int n = 0;
        if ((rc = cuda_check(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, combine_kernel, 256, 0),
                             "combine occupancy")))
            return rc;
        occ = n > 0 ? n : 1;
        per_sm[di.device & 63].store(occ, std::memory_order_relaxed);
    }
    const int64_t work = T * (H / 8);
    const int64_t blocks = std::min<int64_t>((work + 255) / 256, static_cast<int64_t>(di.num_sms) * occ);
    if (blocks <= 0) return METIS_OK;
    combine_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(o, w, slot_to_row, static_cast<int>(T),
                                                                  static_cast<int>(topk), static_cast<int>(H), y, s);
    return cuda_check(cudaGetLastError(), "moe combine launch");
}

// Router top-k, one warp per token (the reading of the cards' FP32 router
// and balance bias): choice j = the j-th largest binary32 score logit + bias,
// ties to the lower expert index; weight = softmax over the chosen experts'
// own logits. Lane l keeps the scores of experts l, l + 32, ...; each round
// takes the warp's best (score, expert) pair, the owning lane marks it taken.
constexpr int ROUTE_WARPS = 8;
constexpr int ROUTE_PER_LANE = 32;   // E <= 1024
constexpr int ROUTE_MAX_K = 32;      // one chosen expert per lane
__device__ __forceinline__ bool route_better(float v, int e, float bv, int be) {
    return v > bv || (v == bv && e < be);
}
template <int P>  // scores per lane: E <= 32 P
__global__ void __launch_bounds__(ROUTE_WARPS * 32) route_topk_kernel(const float* __restrict__ logits,
                                                                      const float* __restrict__ bias,
                                                                      int T, int E, int k,
                                                                      int32_t* __restrict__ ids,
                                                                      float* __restrict__ w) {
    grid_dependency_wait();  // the logits may be the previous kernel's output
    grid_launch_dependents();
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int64_t t = static_cast<int64_t>(blockIdx.x) * ROUTE_WARPS + warp;
    if (t >= T) return;
    const float* l = logits + t * E;
    float sc[P];
#pragma unroll
    for (int i = 0; i < P; ++i) {
        const int e = lane + 32 * i;
        const float v = e < E ? (bias ? __fadd_rn(l[e], bias[e]) : l[e]) : 0.0f;
        sc[i] = v != v ? -INFINITY : v;  // a NaN score counts as -inf, so every round finds an expert
    }
    uint32_t taken = 0;
    int my_id = -1;
    for (int j = 0; j < k; ++j) {
        float bv = -INFINITY;
        int be = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < P; ++i) {
            const int e = lane + 32 * i;
            if (e < E && !(taken & (1u << i)) && route_better(sc[i], e, bv, be)) {
                bv = sc[i];
                be = e;
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oe = __shfl_xor_sync(0xffffffffu, be, o);
            if (route_better(ov, oe, bv, be)) {
                bv = ov;
                be = oe;
            }
        }
        if ((be & 31) == lane) taken |= 1u << (be >> 5);
        if (lane == j) my_id = be;
    }
    // weights: a softmax over the chosen experts' logits (lanes 0 .. k-1)
    const float lv = lane < k ? l[my_id] : -INFINITY;
    float m = lv;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const float ex = lane < k ? expf(lv - m) : 0.0f;
    float sum = ex;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (lane < k) {
        ids[t * k + lane] = my_id;
        w[t * k + lane] = __fdiv_rn(ex, sum);
    }
}

// Shape and mode checks of the FP8 routed-expert layer, shared by its two
// entry points (run before any size is computed from T * topk).
int check_moe_shape(int act, int64_t T, int64_t topk, int64_t E, int64_t H, int64_t I) {
    if (act != METIS_ACT_NONE)
        return fail(METIS_ERR_UNSUPPORTED, "moe: act=%d; only METIS_ACT_NONE is built", act);
    if (T < 0 || T > (1ll << 30) || topk < 1 || E < topk || E > MAX_E)
        return fail(METIS_ERR_INVALID_ARG, "moe: need 0 <= T <= 2^30 and 1 <= topk <= E <= %d "
                    "(T=%lld topk=%lld E=%lld)", MAX_E, (long long)T, (long long)topk, (long long)E);
    if (H < 16 || I < 16 || H % 16 || I % 16 || H > 16384 || I > (1 << 20))
        return fail(METIS_ERR_INVALID_ARG,
                    "moe: need 16 <= H <= 16384 and I >= 16, both multiples of 16 (H=%lld I=%lld)",
                    (long long)H, (long long)I);
    if (T * topk > (1ll << 30)) return fail(METIS_ERR_INVALID_ARG, "moe: T*topk too large");
    return METIS_OK;
}

// Routing: histogram per chunk, then the prefix sums and stable ranks (one
// fused kernel when the count table fits in shared memory, else a
// single-block scan followed by the rank kernel). pad > 1: every expert's
// rows padded to a multiple of pad, pad rows of row_to_slot set to -1.
int launch_routing(const int32_t* ids, int S, int E, int32_t* chunk_tab, int32_t* counts, int32_t* offsets,
                   int pad, int32_t* s2r, int32_t* r2s, uint32_t* status, cudaStream_t st) {
    const int C = (S + CHUNK - 1) / CHUNK;
    count_kernel<<<C, CHUNK, 0, st>>>(ids, S, E, chunk_tab, status);
    const size_t tab_bytes = static_cast<size_t>(C) * E * 4;
    if (static_cast<int64_t>(C) * E <= RS_MAX_TAB && E <= RS_MAX_E) {
        static std::atomic<uint64_t> attr_done[64];
        int dev = 0;
        int rc = cuda_check(cudaGetDevice(&dev), "cudaGetDevice");
        if (rc) return rc;
        rc = once_per_context(attr_done, dev, [] {
            return cuda_check(cudaFuncSetAttribute(rank_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   RS_MAX_TAB * 4),
                              "cudaFuncSetAttribute(rank_scan)");
        });
        if (rc) return rc;
        rank_scan_kernel<<<C, CHUNK, tab_bytes, st>>>(ids, S, E, chunk_tab, counts, offsets, pad, s2r, r2s);
    } else {
        scan_kernel<<<1, SCAN_THREADS, 0, st>>>(chunk_tab, C, E, counts, offsets, pad, pad > 1 ? r2s : nullptr);
        rank_kernel<<<C, CHUNK, 0, st>>>(ids, S, E, chunk_tab, s2r, r2s);
    }
    return cuda_check(cudaGetLastError(), "moe routing launch");
}

}  // namespace moe
}  // namespace metis

using namespace metis;

extern "C" int metis_moe_fp8_grouped_gemm(const void* x_bf16, const int32_t* topk_ids,
                                          const float* topk_w, int64_t T, int64_t topk, int64_t E,
                                          int64_t H, int64_t I, const uint8_t* w_up,
                                          const float* s_up, const uint8_t* w_down,
                                          const float* s_down, int act, void* y_bf16,
                                          void* workspace, size_t ws_bytes,
                                          metis_stream_t stream) {
    using namespace moe;
    clear_error();
    int rc = check_moe_shape(act, T, topk, E, H, I);
    if (rc) return rc;
    const int64_t S = T * topk;
    const size_t need = metis_workspace_size(METIS_OP_MOE, T, I, H, topk, E);
    if (T == 0) return METIS_OK;
    if (!x_bf16 || !topk_ids || !topk_w || !w_up || !s_up || !w_down || !s_down || !workspace)
        return fail(METIS_ERR_INVALID_ARG, "moe: null pointer");
    if (ws_bytes < need)
        return fail(METIS_ERR_INVALID_ARG, "moe: workspace of %zu bytes, need %zu", ws_bytes, need);
    if (!aligned(workspace, 256) || !aligned(x_bf16, 16) || !aligned(w_up, 16) || !aligned(w_down, 16) ||
        (y_bf16 && !aligned(y_bf16, 16)) || !aligned(s_up, 16) || !aligned(s_down, 16))
        return fail(METIS_ERR_INVALID_ARG,
                    "moe: workspace must be 256-byte aligned; x, weights, scales and y 16-byte aligned");
    DeviceInfo di;
    if ((rc = current_device_info(&di))) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    auto region = [&](int r) { return ws + moe_region_offset(r, T, topk, E, H, I, nullptr); };
    int32_t* counts = reinterpret_cast<int32_t*>(region(METIS_MOE_WS_COUNTS));
    int32_t* offsets = reinterpret_cast<int32_t*>(region(METIS_MOE_WS_OFFSETS));
    int32_t* s2r = reinterpret_cast<int32_t*>(region(METIS_MOE_WS_SLOT_TO_ROW));
    int32_t* r2s = reinterpret_cast<int32_t*>(region(METIS_MOE_WS_ROW_TO_SLOT));
    uint8_t* aq = region(METIS_MOE_WS_AQ);
    float* sa = reinterpret_cast<float*>(region(METIS_MOE_WS_SA));
    __nv_bfloat16* h = reinterpret_cast<__nv_bfloat16*>(region(METIS_MOE_WS_H));
    uint8_t* hq = region(METIS_MOE_WS_HQ);
    float* sh = reinterpret_cast<float*>(region(METIS_MOE_WS_SH));
    __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(region(METIS_MOE_WS_O));
    // the per-(chunk, expert) table reuses the H region, which is written
    // only later by the up-projection
    const int C = static_cast<int>((S + CHUNK - 1) / CHUNK);
    int32_t* chunk_tab = reinterpret_cast<int32_t*>(h);
    if (static_cast<int64_t>(C) * E * 4 > 2 * S * I)
        return fail(METIS_ERR_UNSUPPORTED, "moe: routing table does not fit the workspace (E too large for T*topk*I)");

    uint32_t* status = nullptr;
    if ((rc = device_status_word(&status))) return rc;
    if ((rc = launch_routing(topk_ids, static_cast<int>(S), static_cast<int>(E), chunk_tab, counts, offsets, 1,
                             s2r, r2s, status, st)))
        return rc;
    // x quantized once per token, its codes and scale written straight into
    // every expert-ordered row the token was routed to (gathering the rows
    // inside the GEMM with 4-row TMA gathers instead measured 3x slower for
    // the up-projection: 205 against 66 us)
    if ((rc = launch_quant_rows<__nv_bfloat16>(static_cast<const __nv_bfloat16*>(x_bf16), T, H, H, aq, H,
                                               sa, st, s2r, static_cast<int>(topk))))
        return rc;
    if ((rc = launch_fp8_gemm_grouped(aq, sa, w_up, s_up, h, offsets, static_cast<int>(E),
                                      static_cast<int>(S), static_cast<int>(I), static_cast<int>(H), st)))
        return rc;
    if ((rc = launch_quant_rows<__nv_bfloat16>(h, S, I, I, hq, I, sh, st, nullptr, 1))) return rc;
    if ((rc = launch_fp8_gemm_grouped(hq, sh, w_down, s_down, o, offsets, static_cast<int>(E),
                                      static_cast<int>(S), static_cast<int>(H), static_cast<int>(I), st)))
        return rc;
    if (!y_bf16) return METIS_OK;  // the caller combines (metis_moe_shared_fused_combine)
    return launch_combine(o, topk_w, s2r, T, topk, H, static_cast<__nv_bfloat16*>(y_bf16), nullptr, st);
}

// ---------------------------------------------------------------------------
// Allocation-free variant of the routed-expert entry point.
//
// Some callers cannot allocate device memory on their own: a host program
// that runs inside an engine which planned all of the GPU's memory when it
// loaded, or a plugin handed device pointers but no allocator, and callers
// for whom a cudaMalloc (which can synchronise the whole device) would stall
// other work. metis_moe_fp8_grouped_gemm_noalloc serves them from a fixed
// scratch array that lives in this file, so they pass only inputs and
// outputs. Its capacity is kMoeStaticScratchBytes; every GPU that loads the
// library keeps that much device memory until the process exits.
//
// The array's name is meaningful to device code only: on the host it is a
// stand-in, so its device address is looked up once per device with
// cudaGetSymbolAddress (on the first call on that device, with the device
// current) and that address is what the kernels receive.
namespace metis {
namespace {
constexpr size_t kMoeStaticScratchBytes = static_cast<size_t>(16) << 20;  // 16 MiB
static __device__ __align__(256) uint8_t g_moe_static_scratch[kMoeStaticScratchBytes];

std::mutex g_static_scratch_mu;
void* g_static_scratch_ptr[64];
uint64_t g_static_scratch_ctx[64];  // context id the cached address belongs to

// Device address of the scratch array on the current device. Looked up with
// cudaGetSymbolAddress the first time a device (or a new context of it, after
// cudaDeviceReset) is seen, with that device current; cached per device and
// context id after that.
int static_scratch_address(void** out) {
    int dev = 0;
    int rc = cuda_check(cudaGetDevice(&dev), "cudaGetDevice");
    if (rc) return rc;
    if (dev < 0 || dev >= 64) return fail(METIS_ERR_UNSUPPORTED, "device %d", dev);
    uint64_t ctx = 0;
    if ((rc = current_context_id(&ctx))) return rc;
    std::lock_guard<std::mutex> lk(g_static_scratch_mu);
    if (!g_static_scratch_ptr[dev] || g_static_scratch_ctx[dev] != ctx) {
        void* p = nullptr;
        rc = cuda_check(cudaGetSymbolAddress(&p, g_moe_static_scratch),
                        "cudaGetSymbolAddress(static MoE scratch)");
        if (rc) return rc;
        g_static_scratch_ptr[dev] = p;
        g_static_scratch_ctx[dev] = ctx;
    }
    *out = g_static_scratch_ptr[dev];
    return METIS_OK;
}
}  // namespace
}  // namespace metis

extern "C" int metis_moe_fp8_grouped_gemm_noalloc(const void* x_bf16, const int32_t* topk_ids,
                                                  const float* topk_w, int64_t T, int64_t topk,
                                                  int64_t E, int64_t H, int64_t I,
                                                  const uint8_t* w_up, const float* s_up,
                                                  const uint8_t* w_down, const float* s_down,
                                                  int act, void* y_bf16, metis_stream_t stream) {
    clear_error();
    // the same checks as the workspace entry point, first, so that an
    // unsupported mode or a bad shape is reported as such
    int rc = moe::check_moe_shape(act, T, topk, E, H, I);
    if (rc) return rc;
    if (T == 0) return METIS_OK;
    // o would stay in the built-in array, which the caller cannot address
    if (!y_bf16)
        return fail(METIS_ERR_INVALID_ARG, "moe_noalloc: y is required (the routed outputs cannot be "
                    "left in the built-in scratch array for a later combine)");
    const size_t need = metis_workspace_size(METIS_OP_MOE, T, I, H, topk, E);
    if (need > kMoeStaticScratchBytes)
        return fail(METIS_ERR_INVALID_ARG,
                    "moe_noalloc: this problem needs %zu bytes of scratch but the built-in array "
                    "holds %zu (16 MiB); use metis_moe_fp8_grouped_gemm with a caller workspace",
                    need, kMoeStaticScratchBytes);
    void* scratch = nullptr;
    if ((rc = static_scratch_address(&scratch))) return rc;
    return metis_moe_fp8_grouped_gemm(x_bf16, topk_ids, topk_w, T, topk, E, H, I, w_up, s_up,
                                      w_down, s_down, act, y_bf16, scratch,
                                      kMoeStaticScratchBytes, stream);
}

extern "C" int metis_moe_route_topk(const float* logits, const float* bias, int64_t T, int64_t E,
                                    int64_t topk, int32_t* topk_ids, float* topk_w,
                                    metis_stream_t stream) {
    using namespace moe;
    clear_error();
    if (T < 0 || T > 0x7fffffff || E < 1 || E > 32 * ROUTE_PER_LANE || topk < 1 || topk > E ||
        topk > ROUTE_MAX_K)
        return fail(METIS_ERR_INVALID_ARG,
                    "moe_route_topk: need T >= 0, 1 <= E <= %d, 1 <= topk <= min(E, %d) "
                    "(T=%lld E=%lld topk=%lld)", 32 * ROUTE_PER_LANE, ROUTE_MAX_K, (long long)T,
                    (long long)E, (long long)topk);
    if (T == 0) return METIS_OK;
    if (!logits || !topk_ids || !topk_w) return fail(METIS_ERR_INVALID_ARG, "moe_route_topk: null pointer");
    if (!aligned(logits, 4) || !aligned(topk_ids, 4) || !aligned(topk_w, 4) || (bias && !aligned(bias, 4)))
        return fail(METIS_ERR_INVALID_ARG, "moe_route_topk: pointers must be 4-byte aligned");
    DeviceInfo di;
    int rc = current_device_info(&di);
    if (rc) return rc;
    const unsigned grid = static_cast<unsigned>((T + ROUTE_WARPS - 1) / ROUTE_WARPS);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int iT = static_cast<int>(T), iE = static_cast<int>(E), ik = static_cast<int>(topk);
    auto go = [&](auto kernel) {
        return cuda_check(launch_pdl(kernel, dim3(grid), dim3(ROUTE_WARPS * 32), 0, st, 1, logits, bias, iT, iE,
                                     ik, topk_ids, topk_w),
                          "moe_route_topk launch");
    };
    if (E <= 32) return go(route_topk_kernel<1>);
    if (E <= 64) return go(route_topk_kernel<2>);
    if (E <= 128) return go(route_topk_kernel<4>);
    if (E <= 256) return go(route_topk_kernel<8>);
    if (E <= 512) return go(route_topk_kernel<16>);
    return go(route_topk_kernel<32>);
}

// ---------------------------------------------------------------------------
// Routed-expert layer with NVFP4 experts under fast-math ("Lernex/Metis-1.6-
// Praxis-NVFP4", "What is in NVFP4" and "What --fast-math does"): the steps
// of the W8A8 layer above, with each expert's rows padded to a multiple of
// 128 so that every tile's scale atoms are whole (one bulk copy each), x and
// h quantized to NVFP4 (per-token global scale, E4M3 scale per 16), and the
// block-scaled tcgen05 GEMM for both projections.
extern "C" int metis_moe_nvfp4_grouped_gemm(const void* x_bf16, const int32_t* topk_ids,
                                            const float* topk_w, int64_t T, int64_t topk,
                                            int64_t E, int64_t H, int64_t I, const uint8_t* w_up,
                                            const uint8_t* sf_up, const float* g_up,
                                            const uint8_t* w_down, const uint8_t* sf_down,
                                            const float* g_down, int act, void* y_bf16,
                                            void* workspace, size_t ws_bytes,
                                            metis_stream_t stream) {
    using namespace moe;
    clear_error();
    if (act != METIS_ACT_NONE)
        return fail(METIS_ERR_UNSUPPORTED, "moe_nvfp4: act=%d; only METIS_ACT_NONE is built", act);
    if (T < 0 || topk < 1 || E < topk || E > MAX_E)
        return fail(METIS_ERR_INVALID_ARG,
                    "moe_nvfp4: need T >= 0 and 1 <= topk <= E <= %d (T=%lld topk=%lld E=%lld)", MAX_E,
                    (long long)T, (long long)topk, (long long)E);
    if (H < 128 || I < 128 || H % 128 || I % 128 || H > 16384 || I > 65536)
        return fail(METIS_ERR_INVALID_ARG,
                    "moe_nvfp4: need H and I multiples of 128, H <= 16384, I <= 65536 (H=%lld I=%lld)",
                    (long long)H, (long long)I);
    const int64_t S = T * topk;
    if (S > (1ll << 28)) return fail(METIS_ERR_INVALID_ARG, "moe_nvfp4: T*topk too large");
    const size_t need = metis_workspace_size(METIS_OP_MOE_NVFP4, T, I, H, topk, E);
    if (T == 0) return METIS_OK;
    if (!x_bf16 || !topk_ids || !topk_w || !w_up || !sf_up || !g_up || !w_down || !sf_down || !g_down ||
        !workspace)
        return fail(METIS_ERR_INVALID_ARG, "moe_nvfp4: null pointer");
    if (ws_bytes < need)
        return fail(METIS_ERR_INVALID_ARG, "moe_nvfp4: workspace of %zu bytes, need %zu", ws_bytes, need);
    if (!aligned(workspace, 256) || !aligned(x_bf16, 16) || !aligned(w_up, 16) || !aligned(w_down, 16) ||
        !aligned(sf_up, 16) || !aligned(sf_down, 16) || (y_bf16 && !aligned(y_bf16, 16)) || !aligned(g_up, 4) ||
        !aligned(g_down, 4))
        return fail(METIS_ERR_INVALID_ARG,
                    "moe_nvfp4: workspace 256-byte aligned; x, codes, tiled scales and y 16-byte aligned");
    DeviceInfo di;
    int rc = current_device_info(&di);
    if (rc) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    auto region = [&](int r) { return ws + moe4_region_offset(r, T, topk, E, H, I, nullptr); };
    int32_t* counts = reinterpret_cast<int32_t*>(region(METIS_MOE4_WS_COUNTS));
    int32_t* offsets = reinterpret_cast<int32_t*>(region(METIS_MOE4_WS_OFFSETS));
    int32_t* s2r = reinterpret_cast<int32_t*>(region(METIS_MOE4_WS_SLOT_TO_ROW));
    int32_t* r2s = reinterpret_cast<int32_t*>(region(METIS_MOE4_WS_ROW_TO_SLOT));
    uint8_t* aq = region(METIS_MOE4_WS_AQ);
    uint8_t* sfa = region(METIS_MOE4_WS_SFA);
    float* ga = reinterpret_cast<float*>(region(METIS_MOE4_WS_GA));
    __nv_bfloat16* h = reinterpret_cast<__nv_bfloat16*>(region(METIS_MOE4_WS_H));
    uint8_t* hq = region(METIS_MOE4_WS_HQ);
    uint8_t* sfh = region(METIS_MOE4_WS_SFH);
    float* gh = reinterpret_cast<float*>(region(METIS_MOE4_WS_GH));
    __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(region(METIS_MOE4_WS_O));
    const int64_t Sp = moe4_padded_rows(T, topk, E);
    const int C = static_cast<int>((S + CHUNK - 1) / CHUNK);
    int32_t* chunk_tab = reinterpret_cast<int32_t*>(h);  // H is written only later
    if (static_cast<int64_t>(C) * E * 4 > 2 * Sp * I)
        return fail(METIS_ERR_UNSUPPORTED, "moe_nvfp4: routing table does not fit the workspace");

    uint32_t* status = nullptr;
    if ((rc = device_status_word(&status))) return rc;
    if ((rc = launch_routing(topk_ids, static_cast<int>(S), static_cast<int>(E), chunk_tab, counts, offsets, 128,
                             s2r, r2s, status, st)))
        return rc;
    // x: NVFP4 per token, each token once, into the rows it was routed to
    if ((rc = launch_nvfp4_quant(static_cast<const __nv_bfloat16*>(x_bf16), T, H, H, 1, aq, sfa, 1, ga,
                                 s2r, static_cast<int>(topk), nullptr, nullptr, st)))
        return rc;
    if ((rc = launch_nvfp4_gemm(aq, sfa, ga, Sp, w_up, sf_up, g_up, E * I, h, offsets, counts,
                                static_cast<int>(E), 0, static_cast<int>(I), static_cast<int>(H), st)))
        return rc;
    // h: NVFP4 per real row (pad rows and rows past offsets[E] skipped)
    if ((rc = launch_nvfp4_quant(h, Sp, I, I, 1, hq, sfh, 1, gh, nullptr, 1, r2s, offsets + E, st)))
        return rc;
    if ((rc = launch_nvfp4_gemm(hq, sfh, gh, Sp, w_down, sf_down, g_down, E * H, o, offsets, counts,
                                static_cast<int>(E), 0, static_cast<int>(H), static_cast<int>(I), st)))
        return rc;
    if (!y_bf16) return METIS_OK;  // the caller combines (metis_moe_shared_fused_combine)
    return launch_combine(o, topk_w, s2r, T, topk, H, static_cast<__nv_bfloat16*>(y_bf16), nullptr, st);
}

// ---------------------------------------------------------------------------
// The shared expert joined to the routed combine ("Lernex/Metis-1.6-Praxis"
// card, "Architecture": one shared expert beside the routed ones in every
// layer; the FP8 cards keep it in BF16):
//   h_s = bf16(x W_sup^T)                       (BF16 tcgen05 GEMM)
//   s   = bf16(h_s W_sdn^T)                     (BF16 tcgen05 GEMM, into the workspace)
//   y   = bf16(s + sum_j w_j o_j)               (the combine kernel, FP32, j ascending)
// The combine adds s in the same pass that sums the routed rows, before the
// one final rounding. (Adding the routed rows inside the down-projection's
// epilogue instead measured slower on B200: its per-thread gathers of the
// routed rows made the epilogue issue-bound.)
extern "C" int metis_moe_shared_fused_combine(const void* x_bf16, int64_t T, int64_t H, int64_t I_s,
                                              const void* w_sup_bf16, const void* w_sdn_bf16,
                                              const void* o_routed_bf16,
                                              const int32_t* slot_to_row, const float* topk_w,
                                              int64_t topk, void* y_bf16, void* workspace,
                                              size_t ws_bytes, metis_stream_t stream) {
    using namespace moe;
    clear_error();
    if (T < 0 || T > (1ll << 28) || topk < 1 || topk > 8)
        return fail(METIS_ERR_INVALID_ARG, "shared_fused_combine: need T >= 0 and 1 <= topk <= 8 "
                    "(T=%lld topk=%lld)", (long long)T, (long long)topk);
    if (H < 16 || H % 16 || H > 16384 || I_s < 16 || I_s % 16 || I_s > 65536)
        return fail(METIS_ERR_INVALID_ARG,
                    "shared_fused_combine: need H and I_s multiples of 16, H <= 16384, I_s <= 65536 "
                    "(H=%lld I_s=%lld)", (long long)H, (long long)I_s);
    if (T == 0) return METIS_OK;
    if (!x_bf16 || !w_sup_bf16 || !w_sdn_bf16 || !o_routed_bf16 || !slot_to_row || !topk_w || !y_bf16 ||
        !workspace)
        return fail(METIS_ERR_INVALID_ARG, "shared_fused_combine: null pointer");
    const size_t need = metis_workspace_size(METIS_OP_SHARED, T, I_s, H, topk, 0);
    if (ws_bytes < need)
        return fail(METIS_ERR_INVALID_ARG, "shared_fused_combine: workspace of %zu bytes, need %zu", ws_bytes, need);
    if (!aligned(x_bf16, 16) || !aligned(w_sup_bf16, 16) || !aligned(w_sdn_bf16, 16) ||
        !aligned(o_routed_bf16, 16) || !aligned(y_bf16, 16) || !aligned(workspace, 256) ||
        !aligned(slot_to_row, 4) || !aligned(topk_w, 4))
        return fail(METIS_ERR_INVALID_ARG,
                    "shared_fused_combine: x, weights, o and y 16-byte aligned, the workspace 256-byte aligned");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    __nv_bfloat16* hs = static_cast<__nv_bfloat16*>(workspace);
    __nv_bfloat16* s = reinterpret_cast<__nv_bfloat16*>(static_cast<uint8_t*>(workspace) +
                                                        ((2 * T * I_s + 255) & ~static_cast<int64_t>(255)));
    int rc = launch_bf16_gemm(static_cast<const __nv_bfloat16*>(x_bf16),
                              static_cast<const __nv_bfloat16*>(w_sup_bf16), hs, static_cast<int>(T),
                              static_cast<int>(I_s), static_cast<int>(H), nullptr, st);
    if (rc) return rc;
    if ((rc = launch_bf16_gemm(hs, static_cast<const __nv_bfloat16*>(w_sdn_bf16), s, static_cast<int>(T),
                               static_cast<int>(H), static_cast<int>(I_s), nullptr, st)))
        return rc;
    return launch_combine(static_cast<const __nv_bfloat16*>(o_routed_bf16), topk_w, slot_to_row, T, topk, H,
                          static_cast<__nv_bfloat16*>(y_bf16), s, st);
}
