// wq_format.h -- the weight formats inside libwq: the template argument WF of the matmul
// kernels.  INT4 and INT2 keep their bit counts as their codes, so code written for them
// reads unchanged.
#pragma once
#include <cuda_runtime.h>

#include "wq.h"

namespace wq {

constexpr int WF_I1 = 1;    // binary weights 2c - 1, one binary32 scale per tensor
constexpr int WF_I2 = 2;    // ternary weights, one binary32 scale per tensor
constexpr int WF_I4 = 4;    // INT4 codes, binary16 group scales (and zero points)
constexpr int WF_E2M1 = 5;  // FP4 e2m1 codes, binary16 group scales
constexpr int WF_E4M3 = 8;  // FP8 e4m3 codes, binary16 group scales

__host__ __device__ constexpr int wf_bits(int wf) { return wf == WF_E2M1 ? 4 : wf; }
// binary16 scales per group of K (else one binary32 scale for the tensor)
__host__ __device__ constexpr bool wf_grouped(int wf) { return wf == WF_I4 || wf == WF_E2M1 || wf == WF_E4M3; }
__host__ __device__ constexpr bool wf_per_tensor(int wf) { return wf == WF_I2 || wf == WF_I1; }

// The format of a configuration that check_weights accepted.
inline int wf_of(const wq_qconfig &c)
{
    return c.format == WQ_FMT_E2M1 ? WF_E2M1 : c.format == WQ_FMT_E4M3 ? WF_E4M3 : int(c.bits);
}

}  // namespace wq
