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

#ifdef __CUDACC__
// Nearest value of the format to x (|x| <= its largest finite value), ties to even, as a
// code (sign | exponent | mantissa), +0 for a zero result.  Below the smallest normal the
// value is a multiple of the subnormal step; above it x is scaled by an exact power of two so
// that rintf rounds to the format's mantissa bits (a result of 2^(m+1) moves to the next
// binade).
template <int FMT>
__device__ __forceinline__ uint32_t minifloat_code(float x)
{
    constexpr int MB = FMT == WQ_FMT_E2M1 ? 1 : 3;       // mantissa bits
    constexpr int BIAS = FMT == WQ_FMT_E2M1 ? 1 : 7;
    constexpr float kMinNormal = FMT == WQ_FMT_E2M1 ? 1.0f : 0x1p-6f;
    constexpr float kSubStep = FMT == WQ_FMT_E2M1 ? 0.5f : 0x1p-9f;
    const float a = fabsf(x);
    uint32_t code;
    if (a < kMinNormal) {
        code = uint32_t(rintf(__fdiv_rn(a, kSubStep)));  // a power of two: exact; 2^MB is the smallest normal
    } else {
        int e = int((__float_as_uint(a) >> 23) & 0xffu) - 127;                   // floor(log2 a)
        const float scaled = __fmul_rn(a, __uint_as_float(uint32_t(127 + MB - e) << 23));  // in [2^MB, 2^(MB+1))
        uint32_t q = uint32_t(rintf(scaled));
        if (q == (2u << MB)) {
            q = 1u << MB;
            ++e;
        }
        code = (uint32_t(e + BIAS) << MB) | (q - (1u << MB));
    }
    if (code != 0u && x < 0.f) code |= FMT == WQ_FMT_E2M1 ? 0x8u : 0x80u;
    return code;
}
#endif

}  // namespace wq
