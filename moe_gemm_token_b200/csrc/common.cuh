// Internals shared by the kernels of libmetis_fp8: error plumbing, device
// properties, TMA tensor maps, and inline-PTX wrappers for mbarriers, TMA,
// and the fifth-generation tensor cores (tcgen05 + TMEM) of sm_100a.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "../../include/metis_fp8.h"

namespace metis {

// ------------------------------------------------------------------ host side

// Records a formatted error for metis_last_error() and returns `code`.
int fail(int code, const char* fmt, ...);
// Clears the thread's error message.
void clear_error();
// Maps a CUDA runtime error to METIS_ERR_CUDA with a message; METIS_OK if none.
int cuda_check(cudaError_t e, const char* what);

struct DeviceInfo {
    int device = -1;
    int num_sms = 0;
    int max_smem_optin = 0;
    int cc_major = 0, cc_minor = 0;
};
// Properties of the current device (cached per device).
int current_device_info(DeviceInfo* out);

// Device address of the sticky error word of the current device.
int device_status_word(uint32_t** out);
// Unique id of the calling thread's current CUDA context (made current first):
// device addresses of __device__ variables looked up in one context are
// cached under this id and looked up again when it changes.
int current_context_id(uint64_t* out);
// Runs `setup` (a kernel attribute to set, say) the first time it is needed
// on a device in a CUDA context: slots[device] keeps 1 + the id of the
// context it last ran in, so a context made after cudaDeviceReset runs it
// again. Returns setup's status.
template <typename F>
int once_per_context(std::atomic<uint64_t>* slots, int device, F&& setup) {
    uint64_t ctx = 0;
    int rc = current_context_id(&ctx);
    if (rc) return rc;
    std::atomic<uint64_t>& s = slots[device & 63];
    if (s.load(std::memory_order_acquire) == ctx + 1) return 0;
    if ((rc = setup())) return rc;
    s.store(ctx + 1, std::memory_order_release);
    return 0;
}
// Per-wait watchdog limit (ns) for kernels launched now.
uint64_t watchdog_ns();

// Encodes a 2-D tiled TMA descriptor for a row-major [rows, cols] tensor of
// `elem_bytes`-byte elements with row pitch `row_bytes`; box = box_cols x box_rows.
int make_tmap_2d(CUtensorMap* map, const void* base, int elem_bytes, uint64_t cols,
                 uint64_t rows, uint64_t row_bytes, uint32_t box_cols, uint32_t box_rows,
                 bool swizzle128);

// The same for 2-byte elements with the 64-byte swizzle (16-byte pieces of
// each 64-byte row XOR-ed with bits 7-8 of the shared-memory address); for
// TMA stores of 32 x 32 BF16 blocks staged in that layout.
int make_tmap_2d_sw64(CUtensorMap* map, const void* base, int elem_bytes, uint64_t cols, uint64_t rows,
                      uint64_t row_bytes, uint32_t box_cols, uint32_t box_rows);

// Encodes a 3-D tiled TMA descriptor of byte elements: dims {d0, d1, d2},
// byte strides of dims 1 and 2 {s1, s2} (multiples of 16), box {b0, b1, b2}.
int make_tmap_3d_u8(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                    uint64_t s1, uint64_t s2, uint32_t b0, uint32_t b1, uint32_t b2);

// Weight-only W8A16 GEMM for M > 8 tokens on the tensor cores (w16_gemm.cu);
// arguments validated by the caller.
int launch_w8a16_tensor(const __nv_bfloat16* x, const uint8_t* wq, const float* s_w,
                        __nv_bfloat16* y, int M, int N, int K, cudaStream_t st);

// Per-row E4M3 quantizer (quant.cu), for T = __nv_bfloat16 or float; the
// arguments are validated by the caller. dst_rows non-null: row r's codes
// and scale go to rows dst_rows[r * topk + j] (negative entries skipped).
// q null: scales only, s[r] and inv_out[r] = 448/amax.
template <typename T>
int launch_quant_rows(const T* x, int64_t M, int64_t K, int64_t ldx, uint8_t* q, int64_t ldq,
                      float* s, cudaStream_t st, const int32_t* dst_rows, int topk,
                      float* inv_out = nullptr);

// NVFP4 quantizer (nvfp4.cu), T = __nv_bfloat16 or float; arguments
// validated by the caller. rps > 1: rows [i*rps, (i+1)*rps) share a global
// scale. tiled: block scales in the tensor-core atom layout. dst_rows
// non-null: row r goes to rows dst_rows[r * topk + j] (negative skipped).
// row_valid / nrows non-null: rows with row_valid[r] < 0, or r >= *nrows, skipped.
template <typename T>
int launch_nvfp4_quant(const T* x, int64_t R, int64_t K, int64_t ldx, int64_t rps, uint8_t* q,
                       uint8_t* sf, int tiled, float* g, const int32_t* dst_rows, int topk,
                       const int32_t* row_valid, const int32_t* nrows, cudaStream_t st);

// NVFP4 block-scaled GEMM (nvfp4.cu). a_rows: rows of A's code buffer (a
// multiple of 128); offsets/counts null: dense with M rows, else grouped
// (expert e's rows start at offsets[e], a multiple of 128, counts[e] real).
int launch_nvfp4_gemm(const uint8_t* qa, const uint8_t* sfa, const float* ga, int64_t a_rows,
                      const uint8_t* qb, const uint8_t* sfb, const float* gb, int64_t b_rows,
                      __nv_bfloat16* y, const int32_t* offsets, const int32_t* counts, int E, int M,
                      int N, int K, cudaStream_t st);

// BF16 GEMM y = bf16(a b^T) (gemm_fp8.cu); s_b non-null scales column n:
// y = bf16(fl32((a b^T)[., n] * s_b[n])).
int launch_bf16_gemm(const __nv_bfloat16* a, const __nv_bfloat16* b, __nv_bfloat16* y, int M, int N,
                     int K, const float* s_b, cudaStream_t st);

// Exact E4M3 -> BF16 widening of n bytes (w16_gemm.cu); n a multiple of 16,
// both buffers 16-byte aligned.
int launch_widen_e4m3(const uint8_t* w, __nv_bfloat16* out, int64_t n, cudaStream_t st);

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Device error word bits.
constexpr uint32_t kDevErrTimeout = 1u;
constexpr uint32_t kDevErrBadIndex = 2u;  // routing id outside [0, E)

// ---------------------------------------------------------------- device side

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ----------------------------------------------------------------- mbarriers

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Waits until the phase with the given parity has completed, for at most
// `limit_ns`. Returns false (and sets the sticky timeout bit) if it ran out.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, uint64_t limit_ns,
                                          uint32_t* status) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    uint32_t n = 0;
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((++n & 255u) == 0 && globaltimer_ns() - t0 > limit_ns) {
            atomicOr(status, kDevErrTimeout);
            return false;
        }
    }
}

// ---------------------------------------------------------------------- TMA

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* m) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}

// 2-D tiled bulk tensor load global -> shared, completion counted in bytes on
// the mbarrier. No multicast.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* m, int32_t x,
                                            int32_t y, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(x), "r"(y)
        : "memory");
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* m, int32_t x,
                                            int32_t y, int32_t z, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(x), "r"(y), "r"(z)
        : "memory");
}

// Prefetches a 3-D tensor box into L2 (no shared-memory destination).
__device__ __forceinline__ void tma_prefetch_l2_3d(const CUtensorMap* m, int32_t x, int32_t y,
                                                   int32_t z) {
    asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" ::"l"(
                     reinterpret_cast<uint64_t>(m)),
                 "r"(x), "r"(y), "r"(z)
                 : "memory");
}

// Bulk tensor store of a shared-memory box to global memory, its completion
// tracked by this thread's bulk groups; and the group waits. A store must not
// start at a negative coordinate; elements past the tensor's extent are not
// written.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* m, uint32_t src, int32_t x, int32_t y) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(m)),
                 "r"(src), "r"(x), "r"(y)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// the shared-memory sources of every committed store have been read
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// every committed store has completed
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Programmatic dependent launch: wait until the grids this launch depends on
// have completed and their memory is visible; allow dependents to launch.
__device__ __forceinline__ void grid_dependency_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void grid_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Host: launch as a programmatic dependent of the previous kernel in the
// stream (PDL). The kernel must call grid_dependency_wait() before it reads
// anything the previous kernel writes; it may set up shared memory, mbarriers
// and tensor memory before that, overlapping the previous kernel's tail.
// cluster_x > 1 also sets the cluster dimension.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, int cluster_x, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    int n = 1;
    if (cluster_x > 1) {
        attr[1].id = cudaLaunchAttributeClusterDimension;
        attr[1].val.clusterDim.x = cluster_x;
        attr[1].val.clusterDim.y = 1;
        attr[1].val.clusterDim.z = 1;
        n = 2;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

__device__ __forceinline__ void fence_proxy_async_shared() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------- tcgen05/TMEM

__device__ __forceinline__ void tmem_alloc(uint32_t slot_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     slot_smem),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, E4M3 x E4M3 -> FP32, issued by
// one thread.
__device__ __forceinline__ void mma_f8f6f4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                           uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc]^T, BF16 x BF16 -> FP32 (kind::f16),
// issued by one thread. A is M rows (one per TMEM lane) by 16 K elements,
// two per 32-bit column, starting at column a_tmem.
__device__ __forceinline__ void mma_f16_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                               uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrives once on the mbarrier when all previously issued tcgen05.mma of this
// thread have completed.
__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
        : "memory");
}

// Shared-memory matrix descriptor of a K-major operand tile stored with the
// 128-byte swizzle: rows of 128 bytes, 8-row (1024-byte) swizzle atoms.
__device__ __forceinline__ uint64_t sw128_kmajor_desc(uint32_t saddr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);  // start address
    d |= static_cast<uint64_t>(1) << 16;                  // leading byte offset (unused)
    d |= static_cast<uint64_t>(1024 >> 4) << 32;          // stride byte offset: 8 rows
    d |= static_cast<uint64_t>(1) << 46;                  // descriptor version (sm_100)
    d |= static_cast<uint64_t>(2) << 61;                  // 128-byte swizzle
    return d;
}

// Instruction descriptor: E4M3 x E4M3 -> F32, both operands K-major, dense.
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int m, int n) {
    return (1u << 4)                                     // D format F32
           | (0u << 7) | (0u << 10)                      // A, B = E4M3
           | (static_cast<uint32_t>(n >> 3) << 17)       // N / 8
           | (static_cast<uint32_t>(m >> 4) << 24);      // M / 16
}

// Instruction descriptor: BF16 x BF16 -> F32 (kind::f16), dense.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int m, int n) {
    return (1u << 4)                                     // D format F32
           | (1u << 7) | (1u << 10)                      // A, B = BF16
           | (static_cast<uint32_t>(n >> 3) << 17)       // N / 8
           | (static_cast<uint32_t>(m >> 4) << 24);      // M / 16
}

// 32 lanes x 32 consecutive 32-bit columns per warp from TMEM.
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
// 32 lanes x 32 columns of 32-bit values from registers into tensor memory.
__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
        "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]),
        "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]),
        "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}
// 32 lanes x 16 columns of 32-bit values from registers into tensor memory.
__device__ __forceinline__ void tmem_st_32x32b_x16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// ------------------------------------------------------ clusters / CTA pairs

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Address, in the cluster's shared window, of the same shared-memory offset
// in the CTA of the given rank.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}

__device__ __forceinline__ void cluster_sync_all() {
    asm volatile(
        "barrier.cluster.arrive.release.aligned;\n\t"
        "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Arrive on an mbarrier given by its cluster-window address (possibly in the
// peer CTA).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
                 : "memory");
}

// Relaxed arrives (no release fence): for handing over tensor-memory state
// whose accesses are already completed (tcgen05.wait::ld / ::st) and ordered
// by tcgen05.fence::before_thread_sync, where a release would also wait for
// the thread's earlier global stores.
__device__ __forceinline__ void mbar_arrive_relaxed(uint32_t bar) {
    asm volatile("mbarrier.arrive.relaxed.cta.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster_relaxed(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
                 : "memory");
}

// TMA load into this CTA's shared memory whose completion is counted on an
// mbarrier that may live in either CTA of the pair (cta_group::2). No multicast.
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* m, int32_t x,
                                                 int32_t y, uint32_t bar_cluster_addr) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(bar_cluster_addr), "r"(x), "r"(y)
        : "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t slot_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     slot_smem),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

// The CTA pair's MMA (issued by one thread of the even CTA): A rows are split
// between the two CTAs (M = 256), B rows (output columns) too; each CTA's TMEM
// receives its own 128 rows of D.
__device__ __forceinline__ void mma_f8f6f4_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                                uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// BF16 x BF16 -> FP32 (kind::f16) with both operands in shared memory: one
// CTA, or the CTA pair (A and B rows split between the two CTAs as above).
__device__ __forceinline__ void mma_f16_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                           uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void mma_f16_ss_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                                uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrives once on the mbarrier at this offset in every CTA of `mask` when the
// pair's previously issued MMAs have completed.
__device__ __forceinline__ void mma_commit_pair_mc(uint32_t bar, uint16_t mask) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
        " [%0], %1;" ::"r"(bar),
        "h"(mask)
        : "memory");
}
__device__ __forceinline__ void mma_commit_pair(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
        : "memory");
}

// Named barrier over a subset of the CTA's warps.
__device__ __forceinline__ void named_barrier(uint32_t id, uint32_t threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// -------------------------------------------------------------- conversions

// Two binary32 values -> two E4M3 bytes, round-to-nearest-even, saturating to
// +-448 (cvt.rn.satfinite). Returns lo in bits 0..7 and hi in bits 8..15.
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// Four E4M3 bytes -> two BF16 pairs (bytes 0,1 and 2,3), exactly. The byte
// s.eeee.mmm is placed in a BF16 as s | eeee.mmm << 4, which for e > 0 is
// 2^(e-127) (1 + m/8) and for e = 0 the BF16 subnormal m/8 * 2^-126; one
// BF16 multiply by 2^120 (exact; subnormal inputs are kept) gives the E4M3
// value, 2^(e-7) (1 + m/8) or m * 2^-9. prmt's sign-replicating selectors
// put each byte's sign in bit 15 of its half. NaN codes (e = 15, m = 7) come
// out as +-480 here; widen_e4m3x8 repairs them.
__device__ __forceinline__ void widen_e4m3x4(uint32_t w, uint32_t& lo, uint32_t& hi) {
    uint32_t p0, p1;
    asm("prmt.b32 %0, %1, 0, 0x9180;" : "=r"(p0) : "r"(w));
    asm("prmt.b32 %0, %1, 0, 0xB3A2;" : "=r"(p1) : "r"(w));
    const uint32_t u0 = (p0 << 4) & 0x87F087F0u;
    const uint32_t u1 = (p1 << 4) & 0x87F087F0u;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(lo) : "r"(u0), "r"(0x7B807B80u));
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(hi) : "r"(u1), "r"(0x7B807B80u));
}

// Eight E4M3 bytes -> four BF16 pairs, element 2i in the low half of word i.
// A byte whose low 7 bits are all set (E4M3 NaN) becomes a BF16 NaN of the
// same sign (a rarely taken branch).
__device__ __forceinline__ void widen_e4m3x8(const uint2& v, uint4& o) {
    widen_e4m3x4(v.x, o.x, o.y);
    widen_e4m3x4(v.y, o.z, o.w);
    const uint32_t nan = ((v.x & 0x7F7F7F7Fu) + 0x01010101u) | ((v.y & 0x7F7F7F7Fu) + 0x01010101u);
    if (nan & 0x80808080u) {
        uint32_t r[4] = {o.x, o.y, o.z, o.w};
        const uint32_t w[2] = {v.x, v.y};
#pragma unroll
        for (int i = 0; i < 2; ++i) {
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const uint32_t byte = (w[i] >> (8 * b)) & 0xFFu;
                if ((byte & 0x7Fu) == 0x7Fu) {
                    uint32_t& word = r[2 * i + (b >> 1)];
                    const int sh = 16 * (b & 1);
                    word = (word & ~(0xFFFFu << sh)) | (((byte << 8) | 0x7FC0u) << sh);
                }
            }
        }
        o = make_uint4(r[0], r[1], r[2], r[3]);
    }
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Two binary32 -> packed BF16x2 (round-to-nearest-even), lo in bits 0..15.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// The per-row scale rule: s = amax/448 and inv = 448/amax (IEEE binary32,
// inv clamped to FLT_MAX; inv = 0 for an all-zero row).
__device__ __forceinline__ void row_scales(float amax, float* s, float* inv) {
    *s = __fdiv_rn(amax, 448.0f);
    *inv = amax > 0.0f ? fminf(__fdiv_rn(448.0f, amax), 3.402823466e38f) : 0.0f;
}

}  // namespace metis
