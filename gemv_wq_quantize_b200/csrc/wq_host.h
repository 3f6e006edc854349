// wq_host.h -- host-side helpers shared by the libwq translation units:
// status reporting, argument checks, device properties and TMA descriptors.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <cstdarg>
#include <cstdio>

#include "wq.h"

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

}  // namespace wq
