// wq_api.cu -- C ABI of libwq: argument validation, dispatch of the matmul entry
// points, workspace sizing, error reporting, device properties and TMA descriptors.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "wq_format.h"
#include "wq_host.h"

namespace wq {

wq_status skinny_gemm(int WB, int AM, const void *A, const float *a_scale, const uint8_t *Wq, const void *scales,
                      const void *zeros, const void *bias, void *C, int32_t *acc_out, int64_t M, int64_t N, int64_t K,
                      const wq_qconfig &c, void *ws, size_t ws_bytes, cudaStream_t st);
size_t skinny_workspace_size(int WB, int AM, int64_t M, int64_t N, int64_t K);
int skinny_read_error();
wq_status gemv_small_m(int WB, int AM, const void *A, const float *a_scale, const uint8_t *Wq, const void *scales,
                       const void *zeros, const void *bias, void *C, int32_t *acc_out, int64_t M, int64_t N,
                       int64_t K, const wq_qconfig &c, cudaStream_t st);
int gemv_read_error();
wq_status tc_gemm(int WB, int AM, const void *A, const float *a_scale, const uint8_t *Wq, const void *scales,
                  const void *zeros, const void *bias, void *C, int32_t *acc_out, int64_t M, int64_t N, int64_t K,
                  const wq_qconfig &c, void *ws, size_t ws_bytes, cudaStream_t st);
size_t tc_workspace_size(int64_t M, int64_t N, int64_t K);
int tc_read_error();

namespace {
thread_local char g_last_error[512] = "";
}

wq_status fail(wq_status s, const char *fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
    va_end(ap);
    return s;
}

wq_status check_launch(const char *what)
{
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(WQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
    return WQ_OK;
}

const DeviceInfo &device_info()
{
    // A fixed table: references handed out stay valid while other threads add devices.
    static std::mutex mu;
    static DeviceInfo cache[kMaxDevices];
    static DeviceInfo fallback;
    int dev = 0;
    cudaGetDevice(&dev);
    std::lock_guard<std::mutex> lock(mu);
    DeviceInfo &d = (dev >= 0 && dev < kMaxDevices) ? cache[dev] : fallback;
    if (d.device != dev) {
        d.device = dev;
        cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev);
        cudaDeviceGetAttribute(&d.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        if (d.sm_count <= 0) d.sm_count = 1;
        if (d.max_smem_optin <= 0) d.max_smem_optin = 48 * 1024;
    }
    return d;
}

namespace {
using EncodeFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                              const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                              CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeFn encode_fn()
{
    static EncodeFn fn = [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            p = nullptr;
        return reinterpret_cast<EncodeFn>(p);
    }();
    return fn;
}
}  // namespace

wq_status encode_tmap_2d(CUtensorMap *map, CUtensorMapDataType dt, const void *base, uint64_t dim0, uint64_t dim1,
                         uint64_t stride1_bytes, uint32_t box0, uint32_t box1)
{
    EncodeFn fn = encode_fn();
    if (!fn) return fail(WQ_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    cuuint64_t dims[2] = {dim0, dim1};
    cuuint64_t strides[1] = {stride1_bytes};
    cuuint32_t box[2] = {box0, box1};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(WQ_ERR_INVALID_ARG, "cuTensorMapEncodeTiled failed (%d)", int(r));
    return WQ_OK;
}

wq_status encode_tmap(CUtensorMap *map, CUtensorMapDataType dt, int rank, const void *base, const uint64_t *dims,
                      const uint64_t *strides_bytes, const uint32_t *box, int swizzle_bytes)
{
    EncodeFn fn = encode_fn();
    if (!fn) return fail(WQ_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    if (rank < 1 || rank > 3) return fail(WQ_ERR_INVALID_ARG, "tensor map rank %d", rank);
    cuuint64_t d[3] = {}, st[2] = {};
    cuuint32_t b[3] = {}, estr[3] = {1, 1, 1};
    for (int i = 0; i < rank; ++i) {
        d[i] = dims[i];
        b[i] = box[i];
    }
    for (int i = 0; i + 1 < rank; ++i) st[i] = strides_bytes[i];
    CUresult r = fn(map, dt, cuuint32_t(rank), const_cast<void *>(base), d, st, b, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swizzle_bytes == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                    : swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                          : CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(WQ_ERR_INVALID_ARG, "cuTensorMapEncodeTiled (rank %d) failed (%d)", rank, int(r));
    return WQ_OK;
}

wq_status launch_prepared(PreparedLaunch &L, cudaStream_t st, const char *what)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = L.grid;
    cfg.blockDim = L.block;
    cfg.dynamicSmemBytes = L.smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelExC(&cfg, L.func, L.argp);
    if (e != cudaSuccess) return fail(WQ_ERR_CUDA, "%s launch: %s", what, cudaGetErrorString(e));
    return check_launch(what);
}

int read_device_errors()
{
    const int a = skinny_read_error(), b = gemv_read_error(), t = tc_read_error();
    return a ? a : (b ? b : t);
}

namespace {
// Few tokens go to the weight-streaming GEMV; more tokens to the tcgen05 GEMM (the INT32
// group sums included), or else (shapes without a plan there: K below four 128-k blocks,
// ternary FP activations at 9..16 tokens) to the tiled mma.sync path, which serves INT4 and
// INT2 only.  WF: the weight format (wq_format.h).
wq_status dispatch(int WF, int AM, const void *A, const float *a_scale, const uint8_t *Wq, const void *scales,
                   const void *zeros, const void *bias, void *C, int32_t *acc_out, int64_t M, int64_t N, int64_t K,
                   const wq_qconfig &c, void *ws, size_t ws_bytes, cudaStream_t st)
{
    if (M <= 16) {
        wq_status rc = gemv_small_m(WF, AM, A, a_scale, Wq, scales, zeros, bias, C, acc_out, M, N, K, c, st);
        if (rc != WQ_ERR_UNSUPPORTED) return rc;
    } else {
        wq_status rc = tc_gemm(WF, AM, A, a_scale, Wq, scales, zeros, bias, C, acc_out, M, N, K, c, ws, ws_bytes, st);
        if (rc != WQ_ERR_UNSUPPORTED) return rc;
    }
    if (WF != WF_I4 && WF != WF_I2)
        return fail(WQ_ERR_UNSUPPORTED, "no launch plan for M=%lld N=%lld K=%lld with these weights (%s)", (long long)M,
                    (long long)N, (long long)K, wq_last_error());
    if (c.layout == WQ_LAYOUT_NATIVE)
        return fail(WQ_ERR_UNSUPPORTED, "native layout: no launch plan for M=%lld K=%lld (use WQ_LAYOUT_NT)",
                    (long long)M, (long long)K);
    return skinny_gemm(WF, AM, A, a_scale, Wq, scales, zeros, bias, C, acc_out, M, N, K, c, ws, ws_bytes, st);
}
}  // namespace

namespace {

wq_status check_weights(const uint8_t *Wq, const void *scales, const void *zeros, int64_t M, int64_t N, int64_t K,
                        const wq_qconfig &c)
{
    if (M <= 0 || N <= 0 || K <= 0) return fail(WQ_ERR_INVALID_ARG, "M, N and K must be positive");
    if (M > 0x7fffffff || N > 0x7fffffff || K > 0x7fffffff) return fail(WQ_ERR_INVALID_ARG, "sizes exceed int32");
    if (!Wq || !scales) return fail(WQ_ERR_INVALID_ARG, "Wq and scales must be non-null");
    if (!aligned16(Wq) || !aligned16(scales) || (zeros && !aligned16(zeros)))
        return fail(WQ_ERR_ALIGNMENT, "Wq, scales and zeros must be 16-byte aligned");
    if (c.layout != WQ_LAYOUT_NT && c.layout != WQ_LAYOUT_NATIVE) return fail(WQ_ERR_INVALID_ARG, "unknown layout");
    if (c.format != WQ_FMT_INT && c.format != WQ_FMT_E2M1 && c.format != WQ_FMT_E4M3)
        return fail(WQ_ERR_INVALID_ARG, "unknown weight format %d", int(c.format));
    if (c.layout == WQ_LAYOUT_NATIVE && (c.bits != 4 || c.format != WQ_FMT_INT))
        return fail(WQ_ERR_UNSUPPORTED, "the native layout is INT4 only");
    if (c.format != WQ_FMT_INT) {
        if (c.bits != (c.format == WQ_FMT_E2M1 ? 4 : 8))
            return fail(WQ_ERR_INVALID_ARG, "FP4 (e2m1) weights have bits 4, FP8 (e4m3) bits 8");
        if (K % 128) return fail(WQ_ERR_INVALID_ARG, "FP4 / FP8 weights need K %% 128 == 0");
        if (c.group_size <= 0 || K % c.group_size) return fail(WQ_ERR_INVALID_ARG, "K %% group_size != 0");
        if (c.group_size % 128) return fail(WQ_ERR_UNSUPPORTED, "group_size must be a multiple of 128");
    } else if (c.bits == 4) {
        if (K % 128) return fail(WQ_ERR_INVALID_ARG, "INT4 needs K %% 128 == 0");
        if (c.group_size <= 0 || K % c.group_size) return fail(WQ_ERR_INVALID_ARG, "K %% group_size != 0");
        if (c.group_size % 128) return fail(WQ_ERR_UNSUPPORTED, "group_size must be a multiple of 128");
        if (!c.symmetric && !zeros) return fail(WQ_ERR_INVALID_ARG, "asymmetric INT4 needs zeros");
    } else if (c.bits == 2) {
        if (!c.ternary) return fail(WQ_ERR_UNSUPPORTED, "INT2 weights must be ternary");
        if (K % 64) return fail(WQ_ERR_INVALID_ARG, "INT2 needs K %% 64 == 0");
    } else if (c.bits == 1) {
        if (K % 128) return fail(WQ_ERR_INVALID_ARG, "INT1 needs K %% 128 == 0");
    } else {
        return fail(WQ_ERR_INVALID_ARG, "bits must be 4, 2 or 1 (integer codes)");
    }
    return WQ_OK;
}

// The activation paths of each weight type: the pairs of the BitBLAS guide's list (FP16 x
// FP8 / FP4 / INT4 / INT2 / INT1, INT8 x INT4 / INT2 / INT1, FP8 x FP8), plus BF16 with
// INT4 / INT2.  am: 0 FP16, 1 BF16, 2 INT8, 3 FP8 (e4m3).
wq_status check_pair(int wf, int am)
{
    if (am == 3 && wf != WF_E4M3) return fail(WQ_ERR_UNSUPPORTED, "FP8 activations take FP8 (e4m3) weights");
    if (am == 1 && wf != WF_I4 && wf != WF_I2)
        return fail(WQ_ERR_UNSUPPORTED, "BF16 activations take INT4 or INT2 weights");
    if (am == 2 && (wf == WF_E2M1 || wf == WF_E4M3))
        return fail(WQ_ERR_UNSUPPORTED, "FP4 / FP8 weights take FP16 activations (no INT8 path)");
    return WQ_OK;
}

}  // namespace
}  // namespace wq

using namespace wq;

extern "C" const char *wq_status_string(wq_status s)
{
    switch (s) {
    case WQ_OK: return "ok";
    case WQ_ERR_INVALID_ARG: return "invalid argument";
    case WQ_ERR_ALIGNMENT: return "misaligned pointer";
    case WQ_ERR_UNSUPPORTED: return "unsupported configuration";
    case WQ_ERR_CUDA: return "CUDA error";
    case WQ_ERR_WORKSPACE: return "workspace too small";
    }
    return "unknown status";
}

extern "C" const char *wq_last_error(void) { return g_last_error; }

// Reads and clears the device-side error word (a bounded wait that gave up).
// Synchronous; for tests and diagnostics.
extern "C" int wq_device_error(void) { return read_device_errors(); }

extern "C" size_t wq_workspace_size(int64_t M, int64_t N, int64_t K, wq_qconfig c)
{
    const bool known = (c.format == WQ_FMT_INT && (c.bits == 4 || c.bits == 2 || c.bits == 1)) ||
                       (c.format == WQ_FMT_E2M1 && c.bits == 4) || (c.format == WQ_FMT_E4M3 && c.bits == 8);
    if (M <= 0 || N <= 0 || K <= 0 || !known) return 0;
    // the INT8 path has the smaller activation blocks; size for the larger of the two
    if (M <= 16) return 0;  // the few-token kernel needs no workspace
    const int wf = wf_of(c);
    if (wf != WF_I4 && wf != WF_I2) return tc_workspace_size(M, N, K);  // no mma.sync fallback
    return std::max({skinny_workspace_size(wf, 0, M, N, K), skinny_workspace_size(wf, 2, M, N, K),
                     tc_workspace_size(M, N, K)});
}

namespace wq {
wq_status check_a16(const void *A, wq_dtype a_dt, const uint8_t *Wq, const void *scales, const void *zeros,
                    const void *bias, const void *C, int64_t M, int64_t N, int64_t K, const wq_qconfig &c)
{
    wq_status rc = check_weights(Wq, scales, zeros, M, N, K, c);
    if (rc != WQ_OK) return rc;
    if (a_dt != WQ_F16 && a_dt != WQ_BF16) return fail(WQ_ERR_INVALID_ARG, "a_dt must be WQ_F16 or WQ_BF16");
    rc = check_pair(wf_of(c), a_dt == WQ_F16 ? 0 : 1);
    if (rc != WQ_OK) return rc;
    if (!A || !C) return fail(WQ_ERR_INVALID_ARG, "A and C must be non-null");
    if (!aligned16(A) || !aligned16(C) || (bias && !aligned16(bias)))
        return fail(WQ_ERR_ALIGNMENT, "A, C and bias must be 16-byte aligned");
    return WQ_OK;
}
}  // namespace wq

extern "C" wq_status w4a16_gemm(const void *A, wq_dtype a_dt, const uint8_t *Wq, const void *scales,
                                const void *zeros, const void *bias, void *C, int64_t M, int64_t N, int64_t K,
                                wq_qconfig c, void *workspace, size_t ws_bytes, cudaStream_t stream)
{
    wq_status rc = check_a16(A, a_dt, Wq, scales, zeros, bias, C, M, N, K, c);
    if (rc != WQ_OK) return rc;
    if (workspace && !aligned16(workspace)) return fail(WQ_ERR_ALIGNMENT, "workspace must be 16-byte aligned");
    const int wf = wf_of(c);
    return dispatch(wf, a_dt == WQ_F16 ? 0 : 1, A, nullptr, Wq, scales, wf == WF_I4 && !c.symmetric ? zeros : nullptr,
                    bias, C, nullptr, M, N, K, c, workspace, ws_bytes, stream);
}

// W4A8 from FP activations: the per-token INT8 quantization inside the few-token matmul
// when the activations are small and its launch plan stages them whole, else
// act_quant_int8 then w4a8_gemm.
constexpr int64_t kFusedMaxElems = 16384;
extern "C" wq_status w4a8_gemm_fused(const void *A, wq_dtype a_dt, const uint8_t *Wq, const void *scales,
                                     const void *zeros, const void *bias, void *C, int8_t *Aq, float *a_scale,
                                     int32_t *acc_out, int64_t M, int64_t N, int64_t K, wq_qconfig c, void *workspace,
                                     size_t ws_bytes, cudaStream_t stream)
{
    wq_status rc = check_weights(Wq, scales, zeros, M, N, K, c);
    if (rc != WQ_OK) return rc;
    if (a_dt != WQ_F16 && a_dt != WQ_BF16) return fail(WQ_ERR_INVALID_ARG, "a_dt must be WQ_F16 or WQ_BF16");
    if (!A || !C || !Aq || !a_scale) return fail(WQ_ERR_INVALID_ARG, "A, C, Aq and a_scale must be non-null");
    if (!aligned16(A) || !aligned16(Aq) || !aligned16(C) || (bias && !aligned16(bias)) ||
        (workspace && !aligned16(workspace)))
        return fail(WQ_ERR_ALIGNMENT, "A, Aq, C, bias and workspace must be 16-byte aligned");
    const int wf = wf_of(c);
    rc = check_pair(wf, 2);
    if (rc != WQ_OK) return rc;
    if (acc_out && wf == WF_I4 && c.group_size != 128)
        return fail(WQ_ERR_UNSUPPORTED, "acc_out needs group_size == 128");
    // Every CTA of the fused kernel reads all of A twice from L2 (maximum, then codes): worth it
    // while A is small; beyond that the separate quantization kernel is faster.
    if (M <= 16 && M * K <= kFusedMaxElems) {
        const FusedActQuant fa{A, a_dt == WQ_BF16, Aq, a_scale};
        PreparedLaunch L;
        rc = gemv_prepare(wf, 2, Aq, a_scale, Wq, scales, wf == WF_I4 && !c.symmetric ? zeros : nullptr, bias, C,
                          acc_out, M, N, K, c, &L, &fa);
        if (rc == WQ_OK) return launch_prepared(L, stream, "gemv_kernel");
        if (rc != WQ_ERR_UNSUPPORTED) return rc;
    }
    rc = act_quant_int8(A, a_dt, M, K, Aq, a_scale, stream);
    if (rc != WQ_OK) return rc;
    return w4a8_gemm(Aq, a_scale, Wq, scales, zeros, bias, C, acc_out, M, N, K, c, workspace, ws_bytes, stream);
}

extern "C" wq_status w4a8_gemm(const int8_t *Aq, const float *a_scale, const uint8_t *Wq, const void *scales,
                               const void *zeros, const void *bias, void *C, int32_t *acc_out, int64_t M, int64_t N,
                               int64_t K, wq_qconfig c, void *workspace, size_t ws_bytes, cudaStream_t stream)
{
    wq_status rc = check_weights(Wq, scales, zeros, M, N, K, c);
    if (rc != WQ_OK) return rc;
    if (!Aq || !a_scale || !C) return fail(WQ_ERR_INVALID_ARG, "Aq, a_scale and C must be non-null");
    if (!aligned16(Aq) || !aligned16(C) || (bias && !aligned16(bias)) || (workspace && !aligned16(workspace)))
        return fail(WQ_ERR_ALIGNMENT, "Aq, C, bias and workspace must be 16-byte aligned");
    const int wf = wf_of(c);
    rc = check_pair(wf, 2);
    if (rc != WQ_OK) return rc;
    if (acc_out && wf == WF_I4 && c.group_size != 128)
        return fail(WQ_ERR_UNSUPPORTED, "acc_out needs group_size == 128");
    return dispatch(wf, 2, Aq, a_scale, Wq, scales, wf == WF_I4 && !c.symmetric ? zeros : nullptr, bias, C, acc_out,
                    M, N, K, c, workspace, ws_bytes, stream);
}

extern "C" wq_status w8a8_fp8_gemm(const uint8_t *Aq, const float *a_scale, const uint8_t *Wq, const void *scales,
                                   const void *bias, void *C, int64_t M, int64_t N, int64_t K, wq_qconfig c,
                                   void *workspace, size_t ws_bytes, cudaStream_t stream)
{
    wq_status rc = check_weights(Wq, scales, nullptr, M, N, K, c);
    if (rc != WQ_OK) return rc;
    rc = check_pair(wf_of(c), 3);
    if (rc != WQ_OK) return rc;
    if (!Aq || !a_scale || !C) return fail(WQ_ERR_INVALID_ARG, "Aq, a_scale and C must be non-null");
    if (!aligned16(Aq) || !aligned16(C) || (bias && !aligned16(bias)) || (workspace && !aligned16(workspace)))
        return fail(WQ_ERR_ALIGNMENT, "Aq, C, bias and workspace must be 16-byte aligned");
    return dispatch(WF_E4M3, 3, Aq, a_scale, Wq, scales, nullptr, bias, C, nullptr, M, N, K, c, workspace, ws_bytes,
                    stream);
}

// FP8 x FP8 from FP activations: the per-token FP8 quantization inside the few-token matmul
// when the activations are small and its launch plan stages them whole (as for W4A8), else
// act_quant_fp8 then w8a8_fp8_gemm.
extern "C" wq_status w8a8_fp8_gemm_fused(const void *A, wq_dtype a_dt, const uint8_t *Wq, const void *scales,
                                         const void *bias, void *C, uint8_t *Aq, float *a_scale, int64_t M, int64_t N,
                                         int64_t K, wq_qconfig c, void *workspace, size_t ws_bytes,
                                         cudaStream_t stream)
{
    wq_status rc = check_weights(Wq, scales, nullptr, M, N, K, c);
    if (rc != WQ_OK) return rc;
    rc = check_pair(wf_of(c), 3);
    if (rc != WQ_OK) return rc;
    if (a_dt != WQ_F16 && a_dt != WQ_BF16) return fail(WQ_ERR_INVALID_ARG, "a_dt must be WQ_F16 or WQ_BF16");
    if (!A || !C || !Aq || !a_scale) return fail(WQ_ERR_INVALID_ARG, "A, C, Aq and a_scale must be non-null");
    if (!aligned16(A) || !aligned16(Aq) || !aligned16(C) || (bias && !aligned16(bias)) ||
        (workspace && !aligned16(workspace)))
        return fail(WQ_ERR_ALIGNMENT, "A, Aq, C, bias and workspace must be 16-byte aligned");
    if (M <= 16 && M * K <= kFusedMaxElems) {
        const FusedActQuant fa{A, a_dt == WQ_BF16, reinterpret_cast<int8_t *>(Aq), a_scale};
        PreparedLaunch L;
        rc = gemv_prepare(WF_E4M3, 3, Aq, a_scale, Wq, scales, nullptr, bias, C, nullptr, M, N, K, c, &L, &fa);
        if (rc == WQ_OK) return launch_prepared(L, stream, "gemv_kernel");
        if (rc != WQ_ERR_UNSUPPORTED) return rc;
    }
    rc = act_quant_fp8(A, a_dt, M, K, Aq, a_scale, stream);
    if (rc != WQ_OK) return rc;
    return w8a8_fp8_gemm(Aq, a_scale, Wq, scales, bias, C, M, N, K, c, workspace, ws_bytes, stream);
}
