// Host runtime of libmetis_fp8: per-thread error messages, cached device
// properties, the device watchdog word, TMA descriptor encoding, workspace
// layout, and the dispatch entry point.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "common.cuh"
#include "../../include/metis_nvfp4.h"

namespace metis {

namespace {
thread_local std::string g_last_error;

constexpr int kMaxDevices = 64;
std::mutex g_mu;
DeviceInfo g_info[kMaxDevices];
uint32_t* g_status_ptr[kMaxDevices];
uint64_t g_status_ctx[kMaxDevices];  // context id the cached status address belongs to
uint64_t g_watchdog_ns = 2000000000ull;

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);
CtxGetCurrentFn g_ctx_current = nullptr;
CtxGetIdFn g_ctx_id = nullptr;
std::once_flag g_ctx_once;

// Sticky error word, one per device that loads the library.
__device__ uint32_t g_device_status;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;
std::once_flag g_encode_once;
}  // namespace

int fail(int code, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return code;
}

void clear_error() { g_last_error.clear(); }

int cuda_check(cudaError_t e, const char* what) {
    if (e == cudaSuccess) return METIS_OK;
    return fail(METIS_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

int current_device_info(DeviceInfo* out) {
    int dev = 0;
    int rc = cuda_check(cudaGetDevice(&dev), "cudaGetDevice");
    if (rc) return rc;
    if (dev < 0 || dev >= kMaxDevices) return fail(METIS_ERR_UNSUPPORTED, "device %d", dev);
    std::lock_guard<std::mutex> lk(g_mu);
    DeviceInfo& d = g_info[dev];
    if (d.device < 0) {
        DeviceInfo n;
        n.device = dev;
        if ((rc = cuda_check(cudaDeviceGetAttribute(&n.num_sms, cudaDevAttrMultiProcessorCount, dev),
                             "cudaDeviceGetAttribute(SMs)")))
            return rc;
        if ((rc = cuda_check(cudaDeviceGetAttribute(&n.max_smem_optin,
                                                    cudaDevAttrMaxSharedMemoryPerBlockOptin, dev),
                             "cudaDeviceGetAttribute(smem)")))
            return rc;
        if ((rc = cuda_check(cudaDeviceGetAttribute(&n.cc_major, cudaDevAttrComputeCapabilityMajor, dev),
                             "cudaDeviceGetAttribute(cc)")))
            return rc;
        if ((rc = cuda_check(cudaDeviceGetAttribute(&n.cc_minor, cudaDevAttrComputeCapabilityMinor, dev),
                             "cudaDeviceGetAttribute(cc)")))
            return rc;
        if (n.cc_major != 10 || n.cc_minor != 0)
            return fail(METIS_ERR_UNSUPPORTED,
                        "libmetis_fp8 is built for sm_100a (B200); device %d is sm_%d%d", dev,
                        n.cc_major, n.cc_minor);
        d = n;
    }
    *out = d;
    return METIS_OK;
}

int current_context_id(uint64_t* out) {
    std::call_once(g_ctx_once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_ctx_current = reinterpret_cast<CtxGetCurrentFn>(fn);
        fn = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_ctx_id = reinterpret_cast<CtxGetIdFn>(fn);
    });
    if (!g_ctx_current || !g_ctx_id) return fail(METIS_ERR_CUDA, "cuCtxGetCurrent / cuCtxGetId are unavailable");
    CUcontext ctx = nullptr;
    if (g_ctx_current(&ctx) != CUDA_SUCCESS) return fail(METIS_ERR_CUDA, "cuCtxGetCurrent failed");
    if (ctx == nullptr) {
        // no CUDA call on this thread yet: cudaSetDevice makes the device's
        // primary context current (CUDA 12)
        int dev = 0;
        int rc = cuda_check(cudaGetDevice(&dev), "cudaGetDevice");
        if (rc) return rc;
        if ((rc = cuda_check(cudaSetDevice(dev), "cudaSetDevice"))) return rc;
        if (g_ctx_current(&ctx) != CUDA_SUCCESS || ctx == nullptr)
            return fail(METIS_ERR_CUDA, "no current CUDA context");
    }
    unsigned long long id = 0;
    if (g_ctx_id(ctx, &id) != CUDA_SUCCESS) return fail(METIS_ERR_CUDA, "cuCtxGetId failed");
    *out = static_cast<uint64_t>(id);
    return METIS_OK;
}

int device_status_word(uint32_t** out) {
    int dev = 0;
    int rc = cuda_check(cudaGetDevice(&dev), "cudaGetDevice");
    if (rc) return rc;
    if (dev < 0 || dev >= kMaxDevices) return fail(METIS_ERR_UNSUPPORTED, "device %d", dev);
    uint64_t ctx = 0;
    if ((rc = current_context_id(&ctx))) return rc;
    std::lock_guard<std::mutex> lk(g_mu);
    // a module's __device__ variables move when its context is re-created
    // (cudaDeviceReset): the cached address is valid for one context only
    if (!g_status_ptr[dev] || g_status_ctx[dev] != ctx) {
        void* p = nullptr;
        rc = cuda_check(cudaGetSymbolAddress(&p, g_device_status), "cudaGetSymbolAddress(status)");
        if (rc) return rc;
        g_status_ptr[dev] = static_cast<uint32_t*>(p);
        g_status_ctx[dev] = ctx;
    }
    *out = g_status_ptr[dev];
    return METIS_OK;
}

uint64_t watchdog_ns() {
    std::lock_guard<std::mutex> lk(g_mu);
    return g_watchdog_ns;
}

int make_tmap_2d(CUtensorMap* map, const void* base, int elem_bytes, uint64_t cols, uint64_t rows,
                 uint64_t row_bytes, uint32_t box_cols, uint32_t box_rows, bool swizzle128) {
    std::call_once(g_encode_once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    });
    if (!g_encode) return fail(METIS_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
    CUtensorMapDataType dt;
    switch (elem_bytes) {
        case 1: dt = CU_TENSOR_MAP_DATA_TYPE_UINT8; break;
        case 2: dt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16; break;
        case 4: dt = CU_TENSOR_MAP_DATA_TYPE_FLOAT32; break;
        default: return fail(METIS_ERR_INVALID_ARG, "tensor map element size %d", elem_bytes);
    }
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE,
                          swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return fail(METIS_ERR_INVALID_ARG,
                    "cuTensorMapEncodeTiled failed (%d): cols=%llu rows=%llu pitch=%llu box=%ux%u",
                    static_cast<int>(r), (unsigned long long)cols, (unsigned long long)rows,
                    (unsigned long long)row_bytes, box_cols, box_rows);
    return METIS_OK;
}

int make_tmap_2d_sw64(CUtensorMap* map, const void* base, int elem_bytes, uint64_t cols, uint64_t rows,
                      uint64_t row_bytes, uint32_t box_cols, uint32_t box_rows) {
    CUtensorMap probe;
    int rc = make_tmap_2d(&probe, base, 1, 16, 1, 16, 16, 1, false);  // resolves the encoder
    if (rc) return rc;
    if (elem_bytes != 2) return fail(METIS_ERR_INVALID_ARG, "64-byte swizzled tensor map of %d-byte elements", elem_bytes);
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
                          estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                          CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return fail(METIS_ERR_INVALID_ARG,
                    "cuTensorMapEncodeTiled (64-byte swizzle) failed (%d): cols=%llu rows=%llu pitch=%llu",
                    static_cast<int>(r), (unsigned long long)cols, (unsigned long long)rows,
                    (unsigned long long)row_bytes);
    return METIS_OK;
}

int make_tmap_3d_u8(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                    uint64_t s1, uint64_t s2, uint32_t b0, uint32_t b1, uint32_t b2) {
    CUtensorMap probe;
    int rc = make_tmap_2d(&probe, base, 1, 16, 1, 16, 16, 1, false);  // resolves the encoder
    if (rc) return rc;
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {s1, s2};
    cuuint32_t box[3] = {b0, b1, b2};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return fail(METIS_ERR_INVALID_ARG, "cuTensorMapEncodeTiled (3-D) failed (%d)", static_cast<int>(r));
    return METIS_OK;
}

// Routed-expert workspace layout (regions 256-byte aligned).
static int64_t align256(int64_t v) { return (v + 255) & ~static_cast<int64_t>(255); }

int64_t moe_region_offset(int region, int64_t T, int64_t topk, int64_t E, int64_t H, int64_t I,
                          int64_t* total) {
    const int64_t S = T * topk;
    const int64_t sizes[10] = {
        4 * E,        // COUNTS
        4 * (E + 1),  // OFFSETS
        4 * S,        // SLOT_TO_ROW
        4 * S,        // ROW_TO_SLOT
        S * H,        // AQ
        4 * S,        // SA
        2 * S * I,    // H
        S * I,        // HQ
        4 * S,        // SH
        2 * S * H,    // O
    };
    (void)T;
    int64_t off = 0, at = -1;
    for (int r = 0; r < 10; ++r) {
        if (r == region) at = off;
        off = align256(off + sizes[r]);
    }
    if (total) *total = off;
    return at;
}

// Rows of the NVFP4 routed-expert workspace: every expert's rows padded to a
// multiple of 128, at most 127 pad rows per expert.
int64_t moe4_padded_rows(int64_t T, int64_t topk, int64_t E) {
    return (T * topk + 127 * E + 127) / 128 * 128;
}

int64_t moe4_region_offset(int region, int64_t T, int64_t topk, int64_t E, int64_t H, int64_t I,
                           int64_t* total) {
    const int64_t S = T * topk;
    const int64_t Sp = moe4_padded_rows(T, topk, E);
    const int64_t sizes[12] = {
        4 * E,          // COUNTS
        4 * (E + 1),    // OFFSETS
        4 * S,          // SLOT_TO_ROW
        4 * Sp,         // ROW_TO_SLOT
        Sp * H / 2,     // AQ
        Sp * H / 16,    // SFA (tiled)
        4 * Sp,         // GA
        2 * Sp * I,     // H
        Sp * I / 2,     // HQ
        Sp * I / 16,    // SFH (tiled)
        4 * Sp,         // GH
        2 * Sp * H,     // O
    };
    int64_t off = 0, at = -1;
    for (int r = 0; r < 12; ++r) {
        if (r == region) at = off;
        off = align256(off + sizes[r]);
    }
    if (total) *total = off;
    return at;
}

}  // namespace metis

using namespace metis;

extern "C" int metis_version(void) { return 100; }

extern "C" const char* metis_last_error(void) { return g_last_error.c_str(); }

extern "C" int metis_set_watchdog_ns(uint64_t ns) {
    std::lock_guard<std::mutex> lk(g_mu);
    g_watchdog_ns = ns ? ns : 2000000000ull;
    return METIS_OK;
}

namespace metis {
// A wait that nothing satisfies: the bounded mbarrier wait gives up after
// limit_ns and records the timeout in the status word.
__global__ void __launch_bounds__(32) watchdog_selftest_kernel(uint64_t limit_ns, uint32_t* status) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        fence_mbar_init();
    }
    __syncwarp();
    if (threadIdx.x == 0) mbar_wait(smem_u32(&bar), 0, limit_ns, status);
}
}  // namespace metis

extern "C" int metis_watchdog_selftest(uint64_t limit_ns, metis_stream_t stream) {
    clear_error();
    if (limit_ns < 1 || limit_ns > 1000000000ull)
        return fail(METIS_ERR_INVALID_ARG, "watchdog_selftest: limit_ns=%llu, need 1 .. 1e9",
                    (unsigned long long)limit_ns);
    uint32_t* status = nullptr;
    int rc = device_status_word(&status);
    if (rc) return rc;
    watchdog_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns, status);
    return cuda_check(cudaGetLastError(), "watchdog self-test launch");
}

extern "C" int metis_check_device_status(metis_stream_t stream, int clear) {
    clear_error();
    uint32_t* word = nullptr;
    int rc = device_status_word(&word);
    if (rc) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if ((rc = cuda_check(cudaStreamSynchronize(s), "cudaStreamSynchronize"))) return rc;
    uint32_t v = 0;
    if ((rc = cuda_check(cudaMemcpy(&v, word, sizeof v, cudaMemcpyDeviceToHost), "read status")))
        return rc;
    if (clear && v) {
        uint32_t z = 0;
        if ((rc = cuda_check(cudaMemcpy(word, &z, sizeof z, cudaMemcpyHostToDevice), "clear status")))
            return rc;
    }
    if (v & kDevErrTimeout)
        return fail(METIS_ERR_TIMEOUT, "a device-side bounded wait ran out (status word 0x%x)", v);
    if (v & kDevErrBadIndex)
        return fail(METIS_ERR_INVALID_ARG, "a routing id outside [0, E) was dropped (status word 0x%x)", v);
    return METIS_OK;
}

extern "C" size_t metis_workspace_size(int op, int64_t M_or_T, int64_t N_or_I, int64_t K_or_H,
                                       int64_t topk, int64_t E) {
    if (M_or_T < 0 || N_or_I < 0 || K_or_H < 0) return 0;
    switch (op) {
        case METIS_OP_FP8_GEMM_FUSED:
            // per-token reciprocal scales 448/amax, one FP32 per row
            return static_cast<size_t>(align256(4 * (M_or_T > 0 ? M_or_T : 1)));
        case METIS_OP_LINEAR:
            // E4M3 codes of x for the W8A8 path (nothing for the M <= 8 path)
            return M_or_T <= 8 ? 0 : static_cast<size_t>(align256(M_or_T * K_or_H));
        case METIS_OP_MOE: {
            if (topk < 1 || E < 1) return 0;
            int64_t total = 0;
            moe_region_offset(0, M_or_T, topk, E, K_or_H, N_or_I, &total);
            return static_cast<size_t>(total);
        }
        case METIS_OP_W8A16_WIDENED:
            // the weights widened to BF16 [N, K]
            return M_or_T < 1 ? 0 : static_cast<size_t>(align256(2 * N_or_I * K_or_H));
        case METIS_OP_SHARED:
            // the shared expert's hidden rows h_s [T, I_s] and its output s [T, H], BF16
            return static_cast<size_t>(align256(2 * M_or_T * N_or_I) + align256(2 * M_or_T * K_or_H));
        case METIS_OP_MOE_NVFP4: {
            if (topk < 1 || E < 1) return 0;
            int64_t total = 0;
            moe4_region_offset(0, M_or_T, topk, E, K_or_H, N_or_I, &total);
            return static_cast<size_t>(total);
        }
        default:
            return 0;
    }
}

extern "C" int64_t metis_moe_nvfp4_workspace_offset(int region, int64_t T, int64_t topk, int64_t E,
                                                    int64_t H, int64_t I) {
    if (region < 0 || region > 11 || T < 0 || topk < 1 || E < 1 || H < 0 || I < 0) return -1;
    return moe4_region_offset(region, T, topk, E, H, I, nullptr);
}

extern "C" int64_t metis_moe_workspace_offset(int region, int64_t T, int64_t topk, int64_t E,
                                              int64_t H, int64_t I) {
    if (region < 0 || region > 9 || T < 0 || topk < 1 || E < 1 || H < 0 || I < 0) return -1;
    return moe_region_offset(region, T, topk, E, H, I, nullptr);
}

// Fewest tokens for which metis_linear's default maths widens the weights
// into the workspace. Measured on B200 for N x K = 6144 x 2048, 2048 x 6144
// and 14336 x 4096 (in-kernel widening against widening pass + BF16 GEMM):
// at 1536 tokens the in-kernel kernel was faster for the three together
// (33.3 + 40.9 + 145.7 against 32.2 + 40.8 + 164.2 us), at 2048 they were
// even (48.0 + 41.7 + 192.3 against 42.2 + 41.8 + 195.3 us), and at 4096 the
// widened weights won (6144 x 2048: 78.1 against 91.3 us).
constexpr int64_t kWidenMinTokens = 2048;

extern "C" int metis_linear(const void* x_bf16, const uint8_t* wq, const float* s_w, void* y_bf16,
                            int64_t M, int64_t N, int64_t K, int fast_math, float* s_tok,
                            void* workspace, size_t ws_bytes, metis_stream_t stream) {
    clear_error();
    // M <= 8 tokens always take the default maths; more tokens take it unless fast_math
    if (M >= 1 && M <= 8) return metis_w8a16_gemm(x_bf16, wq, s_w, y_bf16, M, N, K, stream);
    if (M > 8 && !fast_math) {
        // enough tokens and room for the widened weights: the BF16 CTA-pair GEMM
        if (M >= kWidenMinTokens && workspace && aligned(workspace, 16) &&
            ws_bytes >= metis_workspace_size(METIS_OP_W8A16_WIDENED, M, N, K, 0, 0))
            return metis_w8a16_gemm_widened(x_bf16, wq, s_w, y_bf16, M, N, K, workspace, ws_bytes, stream);
        return metis_w8a16_gemm(x_bf16, wq, s_w, y_bf16, M, N, K, stream);
    }
    if (M > 0 && M * K > 0 && K % 16 == 0) {
        const size_t need = metis_workspace_size(METIS_OP_LINEAR, M, N, K, 0, 0);
        if (!workspace || ws_bytes < need || !aligned(workspace, 16))
            return fail(METIS_ERR_INVALID_ARG,
                        "metis_linear: needs a 16-byte aligned workspace of %zu bytes (got %zu)",
                        need, ws_bytes);
    }
    // the separate quantizer: cheaper than converting each A tile once per
    // output tile inside the GEMM (see metis_fp8_gemm with METIS_A_BF16)
    uint8_t* xq = static_cast<uint8_t*>(workspace);
    int rc = metis_quant_fp8_per_token(x_bf16, M, K, K, xq, K, s_tok, stream);
    if (rc) return rc;
    return metis_fp8_gemm(xq, METIS_A_E4M3, s_tok, wq, s_w, y_bf16, M, N, K, nullptr, 0, stream);
}
