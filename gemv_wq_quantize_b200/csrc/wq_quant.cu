// wq_quant.cu -- weight quantization / packing, unpacking and per-token INT8
// activation quantization for sm_100a.
//
// Sources: "Accelerating LLM inference with CUDA Graph and INT4 quantization"
// (cnblogs), part 1: step 1 (absmax scale, round, clip, two INT4 per byte) and
// step 2 (q = round(a / a_scale)); "BitBLAS practical guide: mixed-precision
// compute in vLLM" (mlqm): "Advanced features 2" (group_size 128, scales,
// "original" zero points), the BitNet-b1.58 ternary weights of "Real-world case", and the
// FP4 / FP8 / INT1 weights of "Main features" (e2m1 / e4m3 codes with binary16 group scales;
// binary weights with one mean-|w| scale).
//
// Every decision that turns a float into an integer code is taken in binary32
// with IEEE division (__fdiv_rn) and round-half-to-even (rintf), and the scale is
// rounded to binary16 (RNE) before it is used, so the codes are bit-exact with
// any other implementation of the same readings.
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <algorithm>

#include "wq_device.cuh"
#include "wq_host.h"

namespace wq {
namespace {

template <typename T>
__device__ __forceinline__ float to_f(T v);
template <>
__device__ __forceinline__ float to_f<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f<__half>(__half v) { return __half2float(v); }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

// Four consecutive elements (the pointer is aligned to four elements).
template <typename T>
__device__ __forceinline__ void load4(const T *p, float (&v)[4])
{
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = to_f(p[i]);
}
template <>
__device__ __forceinline__ void load4<float>(const float *p, float (&v)[4])
{
    float4 x = __ldg(reinterpret_cast<const float4 *>(p));
    v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
}

__device__ __forceinline__ float clampf(float v, float lo, float hi) { return fminf(fmaxf(v, lo), hi); }

__device__ __forceinline__ float warp_max(float v)
{
#pragma unroll
    for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ float warp_min(float v)
{
#pragma unroll
    for (int o = 16; o; o >>= 1) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// One warp per (row n, group g).  Lane l handles elements c*128 + 4l .. +3 of the
// group for each 128-chunk c, and writes their four nibbles as two bytes.
template <typename T, bool kSym>
__global__ void __launch_bounds__(256) quant_int4_kernel(const T *__restrict__ W, int64_t N, int64_t K, int gs,
                                                         uint8_t *__restrict__ Wq, __half *__restrict__ scales,
                                                         __half *__restrict__ zeros)
{
    const int64_t G = K / gs;
    const int64_t warp = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (warp >= N * G) return;
    const int64_t n = warp / G, g = warp % G;
    const T *w = W + n * K + g * gs;
    const int chunks = gs / 128;

    float amax = 0.f, mn = 0.f, mx = 0.f;
    for (int c = 0; c < chunks; ++c) {
        float v[4];
        load4(w + c * 128 + 4 * lane, v);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            amax = fmaxf(amax, fabsf(v[i]));
            mn = fminf(mn, v[i]);
            mx = fmaxf(mx, v[i]);
        }
    }
    float s, z = 0.f;
    __half sh;
    if (kSym) {
        amax = warp_max(amax);
        sh = __float2half_rn(__fdiv_rn(amax, 7.0f));
        s = __half2float(sh);
    } else {
        mn = warp_min(mn);   // the range always contains 0
        mx = warp_max(mx);
        sh = __float2half_rn(__fdiv_rn(__fsub_rn(mx, mn), 15.0f));
        s = __half2float(sh);
        if (s != 0.f) z = __fadd_rn(clampf(rintf(__fdiv_rn(-mn, s)), 0.f, 15.f), 0.f);  // -0 -> +0
    }
    if (lane == 0) {
        scales[n * G + g] = sh;
        if (!kSym) zeros[n * G + g] = __float2half_rn(z);
    }
    for (int c = 0; c < chunks; ++c) {
        float v[4];
        load4(w + c * 128 + 4 * lane, v);
        uint32_t packed = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float q = 0.f;
            if (s != 0.f) {
                if (kSym) q = clampf(rintf(__fdiv_rn(v[i], s)), -7.f, 7.f);
                else q = clampf(__fadd_rn(rintf(__fdiv_rn(v[i], s)), z), 0.f, 15.f);
            }
            uint32_t field = kSym ? uint32_t(int(q) + 8) : uint32_t(int(q));
            packed |= field << (4 * i);
        }
        uint8_t *dst = Wq + n * (K / 2) + (g * gs + c * 128 + 4 * lane) / 2;
        *reinterpret_cast<uint16_t *>(dst) = uint16_t(packed);
    }
}

// ---- FP4 e2m1 / FP8 e4m3 codes (minifloat_code, wq_format.h) ------------------
// One warp per (row n, group g), lane l on elements c*128 + 4l .. +3 of each 128-chunk c:
// scale = fp16(absmax / 6 or 448), codes of clip(w / scale, -max, max).
template <typename T, int FMT>
__global__ void __launch_bounds__(256) quant_minifloat_kernel(const T *__restrict__ W, int64_t N, int64_t K, int gs,
                                                              uint8_t *__restrict__ Wq, __half *__restrict__ scales)
{
    constexpr float kMax = FMT == WQ_FMT_E2M1 ? 6.0f : 448.0f;
    const int64_t G = K / gs;
    const int64_t warp = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (warp >= N * G) return;
    const int64_t n = warp / G, g = warp % G;
    const T *w = W + n * K + g * gs;
    const int chunks = gs / 128;
    float amax = 0.f;
    for (int c = 0; c < chunks; ++c) {
        float v[4];
        load4(w + c * 128 + 4 * lane, v);
#pragma unroll
        for (int i = 0; i < 4; ++i) amax = fmaxf(amax, fabsf(v[i]));
    }
    amax = warp_max(amax);
    const __half sh = __float2half_rn(__fdiv_rn(amax, kMax));
    const float s = __half2float(sh);
    if (lane == 0) scales[n * G + g] = sh;
    for (int c = 0; c < chunks; ++c) {
        float v[4];
        load4(w + c * 128 + 4 * lane, v);
        uint32_t packed = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t code = s != 0.f ? minifloat_code<FMT>(clampf(__fdiv_rn(v[i], s), -kMax, kMax)) : 0u;
            packed |= code << ((FMT == WQ_FMT_E2M1 ? 4 : 8) * i);
        }
        const int64_t e0 = g * gs + c * 128 + 4 * lane;
        if (FMT == WQ_FMT_E2M1) *reinterpret_cast<uint16_t *>(Wq + n * (K / 2) + e0 / 2) = uint16_t(packed);
        else *reinterpret_cast<uint32_t *>(Wq + n * K + e0) = packed;
    }
}

// ---- ternary: exact mean |w| via per-exponent integer bins ----------------
// |w| = m * 2^(E-149) with integer m < 2^24 and E = max(biased exponent, 1) - 1,
// so sum|w| = (sum_E bins[E] * 2^E) * 2^-149 exactly, where bins[E] sums the m's.
constexpr int kBins = 256;

template <typename T>
__global__ void __launch_bounds__(256) abs_bins_kernel(const T *__restrict__ W, int64_t count,
                                                       unsigned long long *__restrict__ gbins)
{
    __shared__ unsigned long long bins[kBins];
    for (int i = threadIdx.x; i < kBins; i += blockDim.x) bins[i] = 0;
    __syncthreads();
    const int64_t stride = int64_t(gridDim.x) * blockDim.x;
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i - threadIdx.x < count; i += stride) {
        const bool live = i < count;
        uint32_t u = live ? __float_as_uint(to_f(W[i])) : 0u;
        uint32_t be = (u >> 23) & 0xffu, frac = u & 0x7fffffu;
        uint32_t m = be ? (frac | 0x800000u) : frac;
        int E = (be ? int(be) : 1) - 1;
        // lanes that share an exponent add their mantissas once
        const unsigned act = __activemask();
        unsigned same = __match_any_sync(act, E);
        unsigned sum = __reduce_add_sync(same, m);  // at most 32 * 2^24 < 2^32
        if ((threadIdx.x & 31) == __ffs(same) - 1 && sum) atomicAdd(&bins[E], (unsigned long long)sum);
    }
    __syncthreads();
    for (int i = threadIdx.x; i < kBins; i += blockDim.x)
        if (bins[i]) atomicAdd(&gbins[i], bins[i]);
}

// One thread: the exact integer sum, rounded once to binary64 (ties to even),
// divided by the count in binary64, rounded to binary32.  Clears the bins.
__global__ void ternary_scale_kernel(unsigned long long *__restrict__ gbins, int64_t count, float *__restrict__ scale)
{
    if (threadIdx.x != 0 || blockIdx.x != 0) return;
    unsigned long long limb[12] = {0};
    for (int e = 0; e < kBins; ++e) {
        unsigned long long v = gbins[e];
        gbins[e] = 0;
        if (!v) continue;
        unsigned __int128 x = (unsigned __int128)v << (e & 31);
        int j = e >> 5;
        limb[j] += (uint32_t)x;
        limb[j + 1] += (uint32_t)(x >> 32);
        limb[j + 2] += (uint32_t)(x >> 64);
    }
    for (int j = 0; j < 11; ++j) {
        limb[j + 1] += limb[j] >> 32;
        limb[j] &= 0xffffffffull;
    }
    int top = -1;
    for (int j = 11; j >= 0 && top < 0; --j)
        if (limb[j]) top = 32 * j + 63 - __clzll(limb[j]);
    double sum;
    if (top < 0) {
        sum = 0.0;
    } else {
        auto bit = [&](int p) -> unsigned long long { return p < 0 ? 0ull : (limb[p >> 5] >> (p & 31)) & 1ull; };
        int lo = top - 52;
        unsigned long long mant = 0;
        for (int p = top; p >= (lo > 0 ? lo : 0); --p) mant = (mant << 1) | bit(p);
        if (lo <= 0) {
            sum = scalbn((double)mant, -149);
        } else {
            unsigned long long rb = bit(lo - 1), sticky = 0;
            for (int p = lo - 2; p >= 0 && !sticky; --p) sticky |= bit(p);
            if (rb && (sticky || (mant & 1))) ++mant;
            sum = scalbn((double)mant, lo - 149);
        }
    }
    scale[0] = __double2float_rn(__ddiv_rn(sum, (double)count));
}

// 16 consecutive elements per thread -> 4 bytes of 2-bit codes.
template <typename T>
__global__ void __launch_bounds__(256) pack_ternary_kernel(const T *__restrict__ W, int64_t count,
                                                           const float *__restrict__ scale, uint8_t *__restrict__ Wq)
{
    const int64_t t = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    if (t * 16 >= count) return;
    const float s = *scale;
    uint32_t word = 0;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        float v[4];
        load4(W + t * 16 + 4 * c, v);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float q = s != 0.f ? clampf(rintf(__fdiv_rn(v[i], s)), -1.f, 1.f) : 0.f;
            word |= (uint32_t(int(q)) & 3u) << (2 * (4 * c + i));
        }
    }
    reinterpret_cast<uint32_t *>(Wq)[t] = word;
}

// Binary (INT1) weights: 32 consecutive elements per thread -> one word, bit i = (w >= 0).
template <typename T>
__global__ void __launch_bounds__(256) pack_binary_kernel(const T *__restrict__ W, int64_t count,
                                                          uint32_t *__restrict__ Wq)
{
    const int64_t t = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    if (t * 32 >= count) return;
    uint32_t word = 0;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        float v[4];
        load4(W + t * 32 + 4 * c, v);
#pragma unroll
        for (int i = 0; i < 4; ++i) word |= (v[i] >= 0.f ? 1u : 0u) << (4 * c + i);
    }
    Wq[t] = word;
}

// bits 4 / 2 / 1: signed integer codes; raw: FP4 nibbles / FP8 bytes as they are.
__global__ void __launch_bounds__(256) unpack_kernel(const uint8_t *__restrict__ Wq, int64_t nbytes, int bits, int sym,
                                                     int raw, int8_t *__restrict__ q)
{
    const int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= nbytes) return;
    const uint32_t b = Wq[i];
    if (bits == 8) {
        q[i] = int8_t(b);
    } else if (bits == 4 && raw) {
        q[2 * i] = int8_t(b & 15);
        q[2 * i + 1] = int8_t(b >> 4);
    } else if (bits == 1) {
#pragma unroll
        for (int j = 0; j < 8; ++j) q[8 * i + j] = int8_t(((b >> j) & 1u) ? 1 : -1);
    } else if (bits == 4) {
        int lo = b & 15, hi = b >> 4;
        q[2 * i] = int8_t(sym ? lo - 8 : lo);
        q[2 * i + 1] = int8_t(sym ? hi - 8 : hi);
    } else {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            int f = (b >> (2 * j)) & 3;
            q[4 * i + j] = int8_t(f >= 2 ? f - 4 : f);
        }
    }
}

// Kernel-native order: nibble i of every 32-bit word holds element kNativePos[i] of the word's
// 8 elements (the inverse, kNativeSlot[e], is the nibble that holds element e).
__device__ __constant__ int kNativePos[8] = {0, 2, 4, 6, 1, 3, 5, 7};
__device__ __constant__ int kNativeSlot[8] = {0, 4, 1, 5, 2, 6, 3, 7};

__global__ void __launch_bounds__(256) repack_kernel(const uint32_t *__restrict__ in, int64_t nwords,
                                                     uint32_t *__restrict__ out)
{
    const int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= nwords) return;
    const uint32_t w = in[i];
    uint32_t o = 0;
#pragma unroll
    for (int s = 0; s < 8; ++s) o |= ((w >> (4 * kNativePos[s])) & 15u) << (4 * s);
    out[i] = o;
}

__global__ void __launch_bounds__(256) unpack_native_kernel(const uint32_t *__restrict__ in, int64_t nwords, int sym,
                                                            int8_t *__restrict__ q)
{
    const int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= nwords) return;
    const uint32_t w = in[i];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        const int v = int((w >> (4 * kNativeSlot[e])) & 15u);
        q[8 * i + e] = int8_t(sym ? v - 8 : v);
    }
}

// One block per token row: absmax, a_scale = absmax / 127 (INT8 codes) or absmax / 448
// (FP8 e4m3 codes, F8), codes.  8 elements per access.  Rows of up to kActHeld * 8 * 256
// elements are read once and held in registers for both passes; longer rows are read twice.
// INT8 codes come from the reciprocal of the scale with a tie check (quant_i8), which gives
// the codes of the IEEE quotient; FP8 codes divide.
constexpr int kActHeld = 8;  // 16-byte vectors a thread holds

template <typename T, bool F8>
__device__ __forceinline__ uint2 act_codes(const uint4 &raw, float sc, float rc)
{
    const T *e = reinterpret_cast<const T *>(&raw);
    uint32_t w[2] = {0, 0};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        uint32_t code;
        if constexpr (F8)
            code = sc != 0.f ? minifloat_code<WQ_FMT_E4M3>(clampf(__fdiv_rn(to_f(e[i]), sc), -448.f, 448.f)) : 0u;
        else
            code = uint32_t(quant_i8(to_f(e[i]), sc, rc)) & 0xffu;
        w[i / 4] |= code << (8 * (i % 4));
    }
    return make_uint2(w[0], w[1]);
}

template <typename T>
__device__ __forceinline__ float absmax8(const uint4 &raw, float amax)
{
    const T *e = reinterpret_cast<const T *>(&raw);
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(to_f(e[i])));
    return amax;
}

template <typename T, bool F8 = false>
__global__ void __launch_bounds__(256) act_quant_kernel(const T *__restrict__ A, int64_t K, int8_t *__restrict__ Aq,
                                                        float *__restrict__ a_scale)
{
    const int64_t m = blockIdx.x;
    const uint4 *a = reinterpret_cast<const uint4 *>(A + m * K);
    uint2 *q = reinterpret_cast<uint2 *>(Aq + m * K);
    const int64_t K8 = K / 8;
    const bool held = K8 <= int64_t(kActHeld) * blockDim.x;
    // programmatic dependent launch: the matmul that reads Aq may start its prologue (its
    // weights do not depend on this kernel); A may be written by the previous kernel
    grid_dep_launch();
    grid_dep_wait();
    uint4 v[kActHeld];
    float amax = 0.f;
    if (held) {
#pragma unroll
        for (int i = 0; i < kActHeld; ++i) {
            const int64_t j = threadIdx.x + int64_t(i) * blockDim.x;
            v[i] = j < K8 ? __ldg(a + j) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int i = 0; i < kActHeld; ++i) amax = absmax8<T>(v[i], amax);
    } else {
        for (int64_t j = threadIdx.x; j < K8; j += blockDim.x) amax = absmax8<T>(__ldg(a + j), amax);
    }
    __shared__ float red[32];
    amax = warp_max(amax);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
    __syncthreads();
    if (threadIdx.x < 32) {
        float x = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
        x = warp_max(x);
        if (threadIdx.x == 0) red[0] = x;
    }
    __syncthreads();
    const float sc = __fdiv_rn(red[0], F8 ? 448.0f : 127.0f);
    const float rc = sc != 0.f ? __frcp_rn(sc) : 0.f;
    if (threadIdx.x == 0) a_scale[m] = sc;
    if (held) {
#pragma unroll
        for (int i = 0; i < kActHeld; ++i) {
            const int64_t j = threadIdx.x + int64_t(i) * blockDim.x;
            if (j < K8) q[j] = act_codes<T, F8>(v[i], sc, rc);
        }
    } else {
        for (int64_t j = threadIdx.x; j < K8; j += blockDim.x) q[j] = act_codes<T, F8>(__ldg(a + j), sc, rc);
    }
}

int blocks_for(int64_t threads, int per_block = 256) { return int((threads + per_block - 1) / per_block); }

template <typename T>
wq_status quantize_typed(const T *W, int64_t N, int64_t K, wq_qconfig c, uint8_t *Wq, void *scales, void *zeros,
                         void *ws, size_t ws_bytes, cudaStream_t st)
{
    if (c.format != WQ_FMT_INT) {
        const int64_t warps = N * (K / c.group_size);
        const int grid = blocks_for(warps * 32);
        if (c.format == WQ_FMT_E2M1)
            quant_minifloat_kernel<T, WQ_FMT_E2M1><<<grid, 256, 0, st>>>(W, N, K, c.group_size, Wq,
                                                                          static_cast<__half *>(scales));
        else
            quant_minifloat_kernel<T, WQ_FMT_E4M3><<<grid, 256, 0, st>>>(W, N, K, c.group_size, Wq,
                                                                          static_cast<__half *>(scales));
        return check_launch("quant_minifloat_kernel");
    }
    if (c.bits == 4) {
        const int64_t G = K / c.group_size;
        const int64_t warps = N * G;
        const int grid = blocks_for(warps * 32);
        if (c.symmetric)
            quant_int4_kernel<T, true><<<grid, 256, 0, st>>>(W, N, K, c.group_size, Wq,
                                                             static_cast<__half *>(scales), nullptr);
        else
            quant_int4_kernel<T, false><<<grid, 256, 0, st>>>(W, N, K, c.group_size, Wq,
                                                              static_cast<__half *>(scales),
                                                              static_cast<__half *>(zeros));
        return check_launch("quant_int4_kernel");
    }
    // ternary / binary: one mean-|w| scale for the tensor
    auto *bins = static_cast<unsigned long long *>(ws);
    if (!bins || ws_bytes < kBins * sizeof(unsigned long long))
        return fail(WQ_ERR_WORKSPACE, "ternary / binary quantization needs %zu bytes of workspace",
                    size_t(kBins * sizeof(unsigned long long)));
    const int64_t count = N * K;
    if (cudaMemsetAsync(bins, 0, kBins * sizeof(unsigned long long), st) != cudaSuccess)
        return check_launch("cudaMemsetAsync(bins)");
    const int grid = int(std::min<int64_t>(4 * device_info().sm_count, blocks_for(count)));
    abs_bins_kernel<T><<<grid, 256, 0, st>>>(W, count, bins);
    ternary_scale_kernel<<<1, 32, 0, st>>>(bins, count, static_cast<float *>(scales));
    if (c.bits == 1) {
        pack_binary_kernel<T><<<blocks_for(count / 32), 256, 0, st>>>(W, count, reinterpret_cast<uint32_t *>(Wq));
        return check_launch("binary quantization kernels");
    }
    pack_ternary_kernel<T><<<blocks_for(count / 16), 256, 0, st>>>(W, count, static_cast<const float *>(scales), Wq);
    return check_launch("ternary quantization kernels");
}

}  // namespace
}  // namespace wq

using namespace wq;

extern "C" size_t wq_quantize_workspace_size(int64_t, int64_t, wq_qconfig c)
{
    return (c.format == WQ_FMT_INT && (c.bits == 2 || c.bits == 1)) ? kBins * sizeof(unsigned long long) : 0;
}

extern "C" wq_status wq_quantize_pack(const void *W, wq_dtype w_dt, int64_t N, int64_t K, wq_qconfig c, uint8_t *Wq,
                                      void *scales, void *zeros, void *workspace, size_t ws_bytes,
                                      cudaStream_t stream)
{
    if (N <= 0 || K <= 0) return fail(WQ_ERR_INVALID_ARG, "N and K must be positive");
    if (!W || !Wq || !scales) return fail(WQ_ERR_INVALID_ARG, "W, Wq and scales must be non-null");
    if (c.layout != WQ_LAYOUT_NT)
        return fail(WQ_ERR_UNSUPPORTED, "quantize with layout WQ_LAYOUT_NT, then wq_repack");
    if (w_dt != WQ_F32 && w_dt != WQ_F16 && w_dt != WQ_BF16)
        return fail(WQ_ERR_INVALID_ARG, "w_dt must be WQ_F32, WQ_F16 or WQ_BF16");
    if (!aligned16(W) || !aligned16(Wq) || (zeros && !aligned16(zeros)) || !aligned16(scales))
        return fail(WQ_ERR_ALIGNMENT, "device pointers must be 16-byte aligned");
    if (c.format == WQ_FMT_E2M1 || c.format == WQ_FMT_E4M3) {
        if (c.bits != (c.format == WQ_FMT_E2M1 ? 4 : 8))
            return fail(WQ_ERR_INVALID_ARG, "FP4 (e2m1) weights have bits 4, FP8 (e4m3) bits 8");
        if (c.group_size <= 0 || K % c.group_size) return fail(WQ_ERR_INVALID_ARG, "K %% group_size != 0");
        if (c.group_size % 128) return fail(WQ_ERR_UNSUPPORTED, "group_size must be a multiple of 128");
    } else if (c.format != WQ_FMT_INT) {
        return fail(WQ_ERR_INVALID_ARG, "unknown weight format %d", int(c.format));
    } else if (c.bits == 4) {
        if (c.group_size <= 0 || K % c.group_size) return fail(WQ_ERR_INVALID_ARG, "K %% group_size != 0");
        if (c.group_size % 128) return fail(WQ_ERR_UNSUPPORTED, "group_size must be a multiple of 128");
        if (!c.symmetric && !zeros) return fail(WQ_ERR_INVALID_ARG, "asymmetric INT4 needs a zeros buffer");
    } else if (c.bits == 2) {
        if (!c.ternary) return fail(WQ_ERR_UNSUPPORTED, "INT2 weights are produced by the ternary quantizer only");
        if (K % 64) return fail(WQ_ERR_INVALID_ARG, "INT2 needs K %% 64 == 0");
    } else if (c.bits == 1) {
        if (K % 128) return fail(WQ_ERR_INVALID_ARG, "INT1 needs K %% 128 == 0");
    } else {
        return fail(WQ_ERR_INVALID_ARG, "bits must be 4, 2 or 1 (integer codes)");
    }
    switch (w_dt) {
    case WQ_F32: return quantize_typed(static_cast<const float *>(W), N, K, c, Wq, scales, zeros, workspace, ws_bytes, stream);
    case WQ_F16: return quantize_typed(static_cast<const __half *>(W), N, K, c, Wq, scales, zeros, workspace, ws_bytes, stream);
    default: return quantize_typed(static_cast<const __nv_bfloat16 *>(W), N, K, c, Wq, scales, zeros, workspace, ws_bytes, stream);
    }
}

extern "C" wq_status wq_unpack(const uint8_t *Wq, int64_t N, int64_t K, wq_qconfig c, int8_t *q, cudaStream_t stream)
{
    if (N <= 0 || K <= 0 || !Wq || !q) return fail(WQ_ERR_INVALID_ARG, "bad sizes or null pointer");
    const bool ok = (c.format == WQ_FMT_INT && (c.bits == 4 || c.bits == 2 || c.bits == 1)) ||
                    (c.format == WQ_FMT_E2M1 && c.bits == 4) || (c.format == WQ_FMT_E4M3 && c.bits == 8);
    if (!ok) return fail(WQ_ERR_INVALID_ARG, "bits / format: INT 4, 2 or 1; E2M1 4; E4M3 8");
    if (c.bits < 8 && K % (8 / c.bits)) return fail(WQ_ERR_INVALID_ARG, "K must fill whole bytes");
    const int64_t nbytes = N * K * c.bits / 8;
    if (c.layout == WQ_LAYOUT_NATIVE) {
        if (c.bits != 4 || c.format != WQ_FMT_INT) return fail(WQ_ERR_UNSUPPORTED, "the native layout is INT4 only");
        if (K % 8 || !aligned16(Wq)) return fail(WQ_ERR_INVALID_ARG, "native layout: K %% 8 == 0, Wq 16-byte aligned");
        const int64_t nwords = nbytes / 4;
        unpack_native_kernel<<<blocks_for(nwords), 256, 0, stream>>>(reinterpret_cast<const uint32_t *>(Wq), nwords,
                                                                     c.symmetric, q);
        return check_launch("unpack_native_kernel");
    }
    if (c.layout != WQ_LAYOUT_NT) return fail(WQ_ERR_INVALID_ARG, "unknown layout %d", int(c.layout));
    unpack_kernel<<<blocks_for(nbytes), 256, 0, stream>>>(Wq, nbytes, c.bits, c.bits == 4 ? c.symmetric : 1,
                                                          c.format != WQ_FMT_INT ? 1 : 0, q);
    return check_launch("unpack_kernel");
}

extern "C" wq_status wq_repack(const uint8_t *Wq, int64_t N, int64_t K, wq_qconfig c, uint8_t *Wq_native,
                               cudaStream_t stream)
{
    if (N <= 0 || K <= 0 || !Wq || !Wq_native) return fail(WQ_ERR_INVALID_ARG, "bad sizes or null pointer");
    if (c.bits != 4 || c.format != WQ_FMT_INT) return fail(WQ_ERR_UNSUPPORTED, "the native layout is INT4 only");
    if (c.layout != WQ_LAYOUT_NT) return fail(WQ_ERR_INVALID_ARG, "wq_repack reads weights in WQ_LAYOUT_NT");
    if (K % 8) return fail(WQ_ERR_INVALID_ARG, "K %% 8 != 0");
    if (!aligned16(Wq) || !aligned16(Wq_native)) return fail(WQ_ERR_ALIGNMENT, "Wq and Wq_native must be 16-byte aligned");
    const int64_t nwords = N * K / 8;
    repack_kernel<<<blocks_for(nwords), 256, 0, stream>>>(reinterpret_cast<const uint32_t *>(Wq), nwords,
                                                          reinterpret_cast<uint32_t *>(Wq_native));
    return check_launch("repack_kernel");
}

namespace {
wq_status act_quant_launch(bool f8, const void *A, wq_dtype a_dt, int64_t M, int64_t K, int8_t *Aq, float *a_scale,
                           cudaStream_t stream);
}

extern "C" wq_status act_quant_fp8(const void *A, wq_dtype a_dt, int64_t M, int64_t K, uint8_t *Aq, float *a_scale,
                                   cudaStream_t stream)
{
    return act_quant_launch(true, A, a_dt, M, K, reinterpret_cast<int8_t *>(Aq), a_scale, stream);
}

extern "C" wq_status act_quant_int8(const void *A, wq_dtype a_dt, int64_t M, int64_t K, int8_t *Aq, float *a_scale,
                                    cudaStream_t stream)
{
    return act_quant_launch(false, A, a_dt, M, K, Aq, a_scale, stream);
}

namespace {
wq_status act_quant_launch(bool f8, const void *A, wq_dtype a_dt, int64_t M, int64_t K, int8_t *Aq, float *a_scale,
                           cudaStream_t stream)
{
    if (M <= 0 || K <= 0 || !A || !Aq || !a_scale) return fail(WQ_ERR_INVALID_ARG, "bad sizes or null pointer");
    if (a_dt != WQ_F16 && a_dt != WQ_BF16) return fail(WQ_ERR_INVALID_ARG, "a_dt must be WQ_F16 or WQ_BF16");
    if (K % 8) return fail(WQ_ERR_INVALID_ARG, "K %% 8 != 0");
    if (!aligned16(A) || !aligned16(Aq)) return fail(WQ_ERR_ALIGNMENT, "A and Aq must be 16-byte aligned");
    if (M > 0x7fffffff) return fail(WQ_ERR_INVALID_ARG, "M too large");
    // Each block reserves shared memory that it does not use, so that at most two blocks share
    // an SM: programmatic dependent launch places the blocks while the previous kernel still
    // holds most SMs, and without the reservation they pack onto the few free ones (measured:
    // W4A8 at 16 tokens 11.7 -> 9.9 us for the quantization and matmul together).
    constexpr int kSpreadSmem = 100 * 1024;
    static bool spread_set[kMaxDevices][4];
    const int d = device_info().device;
    const int kv = (a_dt == WQ_F16 ? 0 : 2) + (f8 ? 1 : 0);
    if (d >= 0 && d < kMaxDevices && !spread_set[d][kv]) {
        const void *fn = a_dt == WQ_F16 ? (f8 ? reinterpret_cast<const void *>(act_quant_kernel<__half, true>)
                                               : reinterpret_cast<const void *>(act_quant_kernel<__half>))
                                        : (f8 ? reinterpret_cast<const void *>(act_quant_kernel<__nv_bfloat16, true>)
                                              : reinterpret_cast<const void *>(act_quant_kernel<__nv_bfloat16>));
        if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, kSpreadSmem) != cudaSuccess)
            return check_launch("cudaFuncSetAttribute(act_quant_kernel)");
        spread_set[d][kv] = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(M));
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = d >= 0 && d < kMaxDevices ? kSpreadSmem : 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e;
    if (a_dt == WQ_F16 && f8)
        e = cudaLaunchKernelEx(&cfg, act_quant_kernel<__half, true>, static_cast<const __half *>(A), K, Aq, a_scale);
    else if (a_dt == WQ_F16)
        e = cudaLaunchKernelEx(&cfg, act_quant_kernel<__half>, static_cast<const __half *>(A), K, Aq, a_scale);
    else if (f8)
        e = cudaLaunchKernelEx(&cfg, act_quant_kernel<__nv_bfloat16, true>, static_cast<const __nv_bfloat16 *>(A), K,
                               Aq, a_scale);
    else
        e = cudaLaunchKernelEx(&cfg, act_quant_kernel<__nv_bfloat16>, static_cast<const __nv_bfloat16 *>(A), K, Aq,
                               a_scale);
    if (e != cudaSuccess) return fail(WQ_ERR_CUDA, "act_quant_kernel launch: %s", cudaGetErrorString(e));
    return check_launch("act_quant_kernel");
}
}  // namespace
