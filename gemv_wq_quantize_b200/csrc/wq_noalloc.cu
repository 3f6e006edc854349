// wq_noalloc.cu -- w4a16_gemm_noalloc: the W4A16 / W2A16 matmul of w4a16_gemm with its
// split-K scratch in a static device array instead of a caller-provided workspace.
//
// Who needs it: callers that cannot hand the library a workspace.  A plain C host loop
// that drives a model through this ABI owns no device allocator of its own, and a
// plug-in running inside another runtime gets no scratch memory from its host.  The
// library cannot allocate on their behalf either: cudaFree synchronises the whole
// device (a stall inside a decode loop), and a workspace sized per shape would have to
// be reallocated whenever a larger shape arrives.  So this entry point allocates
// nothing: no cudaMalloc, cudaFree or allocating library call, on the host or the device.
//
// The scratch is one array per device, compiled into this translation unit (its module is
// loaded, and the array created by the driver, on first use).  The first call on a device
// that needs scratch looks up its address with cudaGetSymbolAddress, with that device
// current, and clears it; later calls reuse the address.  Every such call also clears the
// split-K arrival counters at the end of the scratch on its own stream (a memset of a few
// bytes, which allocates nothing): a kernel that gave up a bounded wait may have left a
// counter off zero, and later calls must not inherit it.  Shapes that need no scratch (up
// to 16 tokens) go straight to w4a16_gemm with no set-up at all.  Calls that overlap on
// the GPU (two streams, or two host threads) share the array and race: serialise them.
#include <cuda_runtime.h>

#include <mutex>

#include "wq_host.h"

namespace {

// Capacity.  The largest scratch the tiled path asks for on a 148-SM device is
// 148 CTAs x 2 slots x 128 rows x 64 tokens x 4 B = 9.25 MiB of partial sums, plus 4 B
// of arrival counter per 128 weight rows.
constexpr size_t kScratchBytes = WQ_NOALLOC_SCRATCH_BYTES;

}  // namespace

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

namespace wq {
namespace {

// Address of the scratch on the current device; set up (looked up and cleared) on the
// first call for that device.  The clear waits for the device, so that first call must
// not be made while a stream is being captured.
wq_status scratch_for_current_device(void **out)
{
    static std::mutex mu;
    static void *table[kMaxDevices] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(WQ_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices)
        return fail(WQ_ERR_UNSUPPORTED, "w4a16_gemm_noalloc supports device ordinals below %d", kMaxDevices);
    std::lock_guard<std::mutex> lock(mu);
    if (!table[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess)
            return fail(WQ_ERR_CUDA, "cudaGetSymbolAddress(static scratch): %s", cudaGetErrorString(e));
        // Start from a zeroed array; the arrival counters are cleared again by every call.
        e = cudaMemset(p, 0, kScratchBytes);
        if (e == cudaSuccess) e = cudaDeviceSynchronize();
        if (e != cudaSuccess) return fail(WQ_ERR_CUDA, "clearing the static scratch: %s", cudaGetErrorString(e));
        table[dev] = p;
    }
    *out = table[dev];
    return WQ_OK;
}

}  // namespace
}  // namespace wq

using namespace wq;

extern "C" wq_status w4a16_gemm_noalloc(const void *A, wq_dtype a_dt, const uint8_t *Wq, const void *scales,
                                        const void *zeros, const void *bias, void *C, int64_t M, int64_t N,
                                        int64_t K, wq_qconfig c, cudaStream_t stream)
{
    // Shapes whose split-K scratch would not fit are refused before anything else runs.
    const size_t need = wq_workspace_size(M, N, K, c);
    if (need > kScratchBytes)
        return fail(WQ_ERR_WORKSPACE,
                    "w4a16_gemm_noalloc: M=%lld N=%lld K=%lld needs %zu bytes of scratch but the static scratch "
                    "holds %zu; call w4a16_gemm with a workspace instead",
                    (long long)M, (long long)N, (long long)K, need, kScratchBytes);
    // Few tokens: the launch plan needs no scratch, so nothing is set up or cleared.
    if (need == 0) return w4a16_gemm(A, a_dt, Wq, scales, zeros, bias, C, M, N, K, c, nullptr, 0, stream);
    void *scratch = nullptr;
    const wq_status rc = scratch_for_current_device(&scratch);
    if (rc != WQ_OK) return rc;
    // The counters follow the partial-sum area; clear them on the caller's stream.
    const size_t cnt0 = ws_scratch_bytes();
    if (need > cnt0) {
        const cudaError_t e = cudaMemsetAsync(static_cast<unsigned char *>(scratch) + cnt0, 0, need - cnt0, stream);
        if (e != cudaSuccess) return fail(WQ_ERR_CUDA, "clearing the scratch counters: %s", cudaGetErrorString(e));
    }
    return w4a16_gemm(A, a_dt, Wq, scales, zeros, bias, C, M, N, K, c, scratch, kScratchBytes, stream);
}
