// wq_host.h -- host-side helpers shared by the libwq translation units:
// status reporting, argument checks, device properties and TMA descriptors.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <cstdarg>
#include <cstdio>

#include "wq.h"
#include "wq_format.h"

namespace wq {

// Records a one-line reason for the calling thread and returns the status.
wq_status fail(wq_status s, const char *fmt, ...);
wq_status check_launch(const char *what);

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct DeviceInfo {
    int device = -1;
    int sm_count = 0;
    int max_smem_optin = 0;  // bytes of shared memory a block may opt in to
};
// Properties of the current device (cached per device ordinal below kMaxDevices).
constexpr int kMaxDevices = 64;
const DeviceInfo &device_info();

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda link).
wq_status encode_tmap_2d(CUtensorMap *map, CUtensorMapDataType dt, const void *base, uint64_t dim0,
                         uint64_t dim1, uint64_t stride1_bytes, uint32_t box0, uint32_t box1);

// Tiled tensor map of rank 2 or 3: dims[0] innermost (elements), strides_bytes[r-1] for
// dims 1..r-1, box[] in elements, swizzle_bytes 0 (none), 64 or 128.
wq_status encode_tmap(CUtensorMap *map, CUtensorMapDataType dt, int rank, const void *base, const uint64_t *dims,
                      const uint64_t *strides_bytes, const uint32_t *box, int swizzle_bytes);

// Layout shared by every kernel that uses the caller's workspace, so that one workspace
// can serve calls of any shape and kernel in turn: scratch partial sums in the first
// ws_scratch_bytes() (64 KB per SM: the most any plan uses), then the self-resetting
// arrival counters.  A counter slot is therefore never some other call's scratch.
inline size_t ws_scratch_bytes() { return size_t(device_info().sm_count) * 65536; }

// Reads (and clears) the device error words of all kernels with bounded waits.
int read_device_errors();

// One prepared kernel launch: the kernel, its shape and a copy of its arguments, usable for a
// direct launch (launch_prepared) or as a CUDA graph kernel node (node_params).
struct PreparedLaunch {
    const void *func = nullptr;
    dim3 grid, block;
    size_t smem = 0;
    alignas(64) unsigned char args[512];  // the kernel's arguments, each at its own offset
    void *argp[4] = {};                   // pointers into args, in parameter order
    int nargs = 0;
    cudaKernelNodeParams node_params()
    {
        cudaKernelNodeParams k = {};
        k.func = const_cast<void *>(func);
        k.gridDim = grid;
        k.blockDim = block;
        k.sharedMemBytes = unsigned(smem);
        k.kernelParams = argp;
        return k;
    }
};
// Launches it on `st` with programmatic dependent launch allowed.
wq_status launch_prepared(PreparedLaunch &L, cudaStream_t st, const char *what);

// Argument checks of w4a16_gemm (all but the workspace).
wq_status check_a16(const void *A, wq_dtype a_dt, const uint8_t *Wq, const void *scales, const void *zeros,
                    const void *bias, const void *C, int64_t M, int64_t N, int64_t K, const wq_qconfig &c);

// FP activations that the few-token INT8 matmul quantizes per token itself (written to Aq
// and a_scale exactly as act_quant_int8 writes them).
struct FusedActQuant {
    const void *A;
    bool bf16;
    int8_t *Aq;
    float *a_scale;
};

// The few-token matmul (M <= 16) as a prepared launch (see gemv_small_m for the arguments);
// with `fa`, INT8 mode starting from FP activations (WQ_ERR_UNSUPPORTED when the launch
// plan does not stage the activations whole).
wq_status gemv_prepare(int WB, int AM, const void *A, const float *a_scale, const uint8_t *Wq, const void *scales,
                       const void *zeros, const void *bias, void *C, int32_t *acc_out, int64_t M, int64_t N,
                       int64_t K, const wq_qconfig &c, PreparedLaunch *out, const FusedActQuant *fa = nullptr);

}  // namespace wq
