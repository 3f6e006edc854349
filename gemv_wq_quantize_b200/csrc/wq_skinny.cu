// wq_skinny.cu -- weight-streaming matmul for few tokens (decode GEMV, M <= 64 per launch).
//
// Computes C[M,N] = A[M,K] x dequant(Wq[N,K])^T ("BitBLAS practical guide", "What is
// BitBLAS"; layout "nt") for packed INT4 (group scales, optional zero points) or INT2
// ternary (one scale) weights, with FP16 / BF16 activations (W4A16) or per-token INT8
// activations with exact INT32 group sums and a float dequantization epilogue (W4A8:
// "Accelerating LLM inference with CUDA Graph and INT4 quantization", part 1, steps 3-4).
//
// Design (HBM-bound: every weight byte is read once):
//  * The weight matrix is cut into units of 128 rows x 64 bytes (128 k of INT4, 256 k of
//    INT2).  Units are ordered row-group-major and each CTA (one per SM) takes a contiguous
//    range of them (stream-K), so every SM streams the same number of bytes.
//  * A producer warp issues one 2D TMA load per unit for the weight tile and one for the
//    matching activation block, plus 4-byte cp.async copies of the 128 rows' scale / zero
//    words, into an S-stage shared-memory ring guarded by mbarriers.  All of a CTA's units
//    are in flight at once when they fit in the ring.
//  * A fragment warp turns each activation block into mma.sync B fragments (the k order the
//    nibble unpack produces) and, for INT8 activations, the per-token sums of the unit.
//  * Eight consumer warps (16 rows each) unpack nibbles with LOP3 into exact integers
//    q - z in f16/bf16 (magic-exponent trick) or u8, run mma.sync (f32 or s32
//    accumulators), and fold each group's sum into an fp32 total with the group scale.
//    Integer group sums are exact; FP totals carry only fp32 accumulation error.
//  * Row groups split between CTAs are combined through a workspace: every contributor
//    writes its partial, the last one to arrive (atomicInc, which also resets the counter)
//    adds them in CTA order and runs the epilogue.  No CTA ever waits for another.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include <algorithm>
#include <type_traits>

#include "wq_device.cuh"
#include "wq_host.h"

namespace wq {

static __device__ int g_skinny_error;

namespace {

enum AMode { A_F16 = 0, A_BF16 = 1, A_I8 = 2 };

constexpr int kRows = 128;            // weight rows per unit
constexpr int kUnitBytes = 64;        // packed bytes per row per unit
constexpr int kWTile = kRows * kUnitBytes;
constexpr int kScaleBytes = kRows * 2 * 4;  // scale word + zero word per row
constexpr int kConsumerWarps = 8;
constexpr int kThreads = (kConsumerWarps + 2) * 32;
constexpr int kFragBufs = 2;

struct SkinnyParams {
    int M, N, K;        // M: tokens in this launch (<= 8 * NT)
    int m0;             // first token of this launch in A / C / acc_out
    int G, gs, sym;     // INT4 groups
    int KB, RG;         // units along K, row groups along N
    long long U;        // total units
    int P, split, S;
    int ablk_bytes, frag_bytes;
    const uint16_t *scales16;
    const float *scale32;
    const uint16_t *zeros;
    const void *bias;
    const float *a_scale;
    void *C;
    int32_t *acc_out;
    float *ws_partial;
    unsigned *ws_counter;
};

__device__ __forceinline__ long long range_begin(const SkinnyParams &p, int c)
{
    if (p.split) return (long long)c * p.U / p.P;
    return (long long)((long long)c * p.RG / p.P) * p.KB;
}
// CTA whose range holds unit u (split plans only).
__device__ __forceinline__ int cta_of_unit(const SkinnyParams &p, long long u)
{
    return int(((u + 1) * p.P + p.U - 1) / p.U) - 1;
}

__device__ __forceinline__ uint64_t globaltimer()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// Wait with a wall-clock limit of ~2 s; records an error and returns false on expiry.
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity)
{
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    for (;;) {
        for (int i = 0; i < 4; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (globaltimer() - t0 > 2000000000ull) {
            atomicCAS(&g_skinny_error, kErrNone, kErrWaitTimeout);
            return false;
        }
    }
}

__host__ __device__ constexpr int kunit_of(int WB) { return WB == 4 ? 128 : 256; }
__host__ __device__ constexpr int steps_of(int WB, int AM) { return AM == A_I8 ? (WB == 4 ? 4 : 8) : (WB == 4 ? 8 : 16); }

template <int AM>
__device__ __forceinline__ void store_out(void *C, long long idx, float v)
{
    if constexpr (AM == A_BF16) static_cast<__nv_bfloat16 *>(C)[idx] = __float2bfloat16_rn(v);
    else static_cast<__half *>(C)[idx] = __float2half_rn(v);
}

template <int AM>
__device__ __forceinline__ float bias_at(const void *bias, int n)
{
    if (!bias) return 0.f;
    if constexpr (AM == A_BF16) return __bfloat162float(static_cast<const __nv_bfloat16 *>(bias)[n]);
    return __half2float(static_cast<const __half *>(bias)[n]);
}

// Final value of one output from its (summed) total.
template <int WB, int AM>
__device__ __forceinline__ float finish(const SkinnyParams &p, float total_f, int total_i, int n, int m)
{
    float v;
    if constexpr (AM == A_I8) {
        const float as = p.a_scale[p.m0 + m];
        v = (WB == 2) ? as * (p.scale32[0] * float(total_i)) : as * total_f;
    } else {
        v = (WB == 2) ? p.scale32[0] * total_f : total_f;
    }
    return v + bias_at<AM>(p.bias, n);
}

// ---------------------------------------------------------------- fragment builder
// Writes, for unit data in `ablk` ([MP][kunit] elements), the B fragments of every
// (n8 tile, pair of mma k-steps, lane) as one uint4, and for INT8 activations the
// per-token sums of the unit.
template <int WB, int AM, int NT>
__device__ __forceinline__ void build_frags(const uint8_t *ablk, uint8_t *frag, int lane)
{
    constexpr int QN = steps_of(WB, AM) / 2;
    const int g = lane >> 2, t = lane & 3;
    uint4 *out = reinterpret_cast<uint4 *>(frag);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int m = nt * 8 + g;
        int asum = 0;
#pragma unroll
        for (int q = 0; q < QN; ++q) {
            uint4 r;
            if constexpr (AM != A_I8 && WB == 4) {
                const uint4 v = lds128(ablk + (m * 128 + 32 * t + 8 * q) * 2);
                r.x = prmt(v.x, v.z, 0x5410);
                r.y = prmt(v.x, v.z, 0x7632);
                r.z = prmt(v.y, v.w, 0x5410);
                r.w = prmt(v.y, v.w, 0x7632);
            } else if constexpr (AM != A_I8 && WB == 2) {
                const int j = q >> 1, hh = q & 1;
                const uint8_t *base = ablk + (m * 256 + 64 * t + 16 * j + 4 * hh) * 2;
                const uint2 lo = *reinterpret_cast<const uint2 *>(base);
                const uint2 hi = *reinterpret_cast<const uint2 *>(base + 16);
                r.x = prmt(lo.x, hi.x, 0x5410);
                r.y = prmt(lo.x, hi.x, 0x7632);
                r.z = prmt(lo.y, hi.y, 0x5410);
                r.w = prmt(lo.y, hi.y, 0x7632);
            } else if constexpr (WB == 4) {  // INT8 activations, INT4 weights
                const uint4 v = lds128(ablk + m * 128 + 32 * t + 16 * q);
                r.x = prmt(v.x, v.y, 0x6420);
                r.y = prmt(v.x, v.y, 0x7531);
                r.z = prmt(v.z, v.w, 0x6420);
                r.w = prmt(v.z, v.w, 0x7531);
                asum = __dp4a(int(v.x), 0x01010101, asum);
                asum = __dp4a(int(v.y), 0x01010101, asum);
                asum = __dp4a(int(v.z), 0x01010101, asum);
                asum = __dp4a(int(v.w), 0x01010101, asum);
            } else {  // INT8 activations, INT2 weights
                const uint4 v = lds128(ablk + m * 256 + 64 * t + 16 * q);
                const uint32_t x0 = prmt(v.x, v.y, 0x5140), y0 = prmt(v.z, v.w, 0x5140);
                const uint32_t x1 = prmt(v.x, v.y, 0x7362), y1 = prmt(v.z, v.w, 0x7362);
                r.x = prmt(x0, y0, 0x5410);
                r.y = prmt(x0, y0, 0x7632);
                r.z = prmt(x1, y1, 0x5410);
                r.w = prmt(x1, y1, 0x7632);
                asum = __dp4a(int(v.x), 0x01010101, asum);
                asum = __dp4a(int(v.y), 0x01010101, asum);
                asum = __dp4a(int(v.z), 0x01010101, asum);
                asum = __dp4a(int(v.w), 0x01010101, asum);
            }
            sts128(out + (nt * QN + q) * 32 + lane, r);
        }
        if constexpr (AM == A_I8) {
            asum += __shfl_xor_sync(0xffffffffu, asum, 1);
            asum += __shfl_xor_sync(0xffffffffu, asum, 2);
            if (t == 0) reinterpret_cast<int *>(frag + NT * QN * 512)[m] = asum;
        }
    }
}

// ---------------------------------------------------------------- the kernel
template <int WB, int AM, int NT>
__global__ void __launch_bounds__(kThreads, 1)
    skinny_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_a,
                  const SkinnyParams p)
{
    constexpr int MP = NT * 8;
    constexpr int KU = kunit_of(WB);
    constexpr int STEPS = steps_of(WB, AM);
    constexpr int QN = STEPS / 2;
    using Acc = typename std::conditional<AM == A_I8, int, float>::type;

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int S = p.S;
    const int stage_bytes = kWTile + p.ablk_bytes + kScaleBytes;
    uint8_t *frag_base = smem + size_t(S) * stage_bytes;
    uint64_t *bars = reinterpret_cast<uint64_t *>(frag_base + kFragBufs * p.frag_bytes);
    uint64_t *full = bars, *empty = bars + S, *ffull = bars + 2 * S, *fempty = bars + 2 * S + kFragBufs;
    uint64_t *csync = bars + 2 * S + 2 * kFragBufs;
    int *flag = reinterpret_cast<int *>(csync + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int cta = blockIdx.x;
    const long long begin = range_begin(p, cta), end = range_begin(p, cta + 1);
    const int nunits = int(end - begin);

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1 + 32);  // expect_tx arrival + 32 cp.async arrivals
            mbar_init(&empty[s], kConsumerWarps);
        }
        for (int f = 0; f < kFragBufs; ++f) {
            mbar_init(&ffull[f], 32);
            mbar_init(&fempty[f], kConsumerWarps);
        }
        mbar_init(csync, kConsumerWarps * 32);
        *flag = 0;
        fence_barrier_init();
    }
    __syncthreads();

    if (warp == kConsumerWarps) {
        // ------------------------------------------------------------ producer warp
        if (lane == 0) {
            tma_prefetch_desc(&tmap_w);
            tma_prefetch_desc(&tmap_a);
        }
        const long long total_sc = (long long)p.N * p.G;
        int i = 0;
        for (; i < nunits; ++i) {
            const int s = i % S;
            if (i >= S && !wait_bar(&empty[s], ((i / S) - 1) & 1)) break;
            const long long u = begin + i;
            const int r = int(u / p.KB), kb = int(u % p.KB);
            uint8_t *st = smem + size_t(s) * stage_bytes;
            if (lane == 0) {
                mbar_arrive_expect_tx(&full[s], kWTile + p.ablk_bytes);
                tma_load_2d(st, &tmap_w, kb * kUnitBytes, r * kRows, &full[s]);
                tma_load_2d(st + kWTile, &tmap_a, kb * KU, p.m0, &full[s]);
            }
            if constexpr (WB == 4) {
                uint32_t *sw = reinterpret_cast<uint32_t *>(st + kWTile + p.ablk_bytes);
                const int gi = (kb * KU) / p.gs;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int row = lane * 4 + j;
                    const int n = r * kRows + row;
                    if (n < p.N) {
                        const long long idx = (long long)n * p.G + gi;
                        const long long w0 = idx & ~1ll;
                        if (w0 + 1 < total_sc) {
                            cp_async4(sw + 2 * row, p.scales16 + w0);
                            if (!p.sym) cp_async4(sw + 2 * row + 1, p.zeros + w0);
                        } else {  // last element of the array: no 4-byte word around it
                            sw[2 * row] = p.scales16[idx];
                            sw[2 * row + 1] = p.sym ? 0u : p.zeros[idx];
                        }
                    } else {
                        sw[2 * row] = 0u;
                        sw[2 * row + 1] = 0u;
                    }
                }
            }
            cp_async_mbar_arrive_noinc(&full[s]);
        }
        // drain: every copy this warp issued has landed before the CTA may exit
        for (int k = std::max(0, i - S); k < i; ++k) wait_bar(&full[k % S], (k / S) & 1);
        return;
    }

    if (warp == kConsumerWarps + 1) {
        // ------------------------------------------------------------ fragment warp
        for (int i = 0; i < nunits; ++i) {
            const int s = i % S, f = i % kFragBufs;
            if (!wait_bar(&full[s], (i / S) & 1)) break;
            if (i >= kFragBufs && !wait_bar(&fempty[f], ((i / kFragBufs) - 1) & 1)) break;
            build_frags<WB, AM, NT>(smem + size_t(s) * stage_bytes + kWTile, frag_base + f * p.frag_bytes, lane);
            mbar_arrive(&ffull[f]);
        }
        return;
    }

    // ---------------------------------------------------------------- consumer warps
    const int g = lane >> 2, t = lane & 3;
    const int rl0 = warp * 16 + g;  // this thread's two local rows: rl0 and rl0 + 8
    Acc total[NT][4];
    int tsum[NT][2];  // INT2 x INT8: running per-token activation sums
    uint32_t csync_phase = 0;
    int seg_start = 0;
    bool ok = true;

    for (int i = 0; i < nunits && ok; ++i) {
        const int s = i % S, f = i % kFragBufs;
        const long long u = begin + i;
        const int r = int(u / p.KB), kb = int(u % p.KB);
        if (i == 0 || kb == 0) {
            seg_start = kb;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
                for (int e = 0; e < 4; ++e) total[nt][e] = Acc(0);
                tsum[nt][0] = tsum[nt][1] = 0;
            }
        }
        if (!wait_bar(&full[s], (i / S) & 1) || !wait_bar(&ffull[f], (i / kFragBufs) & 1)) {
            ok = false;
            break;
        }
        const uint8_t *st = smem + size_t(s) * stage_bytes;
        const uint4 wa = lds128(st + rl0 * kUnitBytes + 16 * t);
        const uint4 wb = lds128(st + (rl0 + 8) * kUnitBytes + 16 * t);
        float s_lo = 0.f, s_hi = 0.f;
        uint32_t z_lo = 8, z_hi = 8;
        if constexpr (WB == 4) {
            const uint32_t *sw = reinterpret_cast<const uint32_t *>(st + kWTile + p.ablk_bytes);
            const int gi = (kb * KU) / p.gs;
            const int n_lo = r * kRows + rl0, n_hi = n_lo + 8;
            const int sh_lo = int(((long long)n_lo * p.G + gi) & 1) * 16;
            const int sh_hi = int(((long long)n_hi * p.G + gi) & 1) * 16;
            const uint32_t sw_lo = lds32(sw + 2 * rl0), sw_hi = lds32(sw + 2 * (rl0 + 8));
            s_lo = __half2float(__ushort_as_half(uint16_t(sw_lo >> sh_lo)));
            s_hi = __half2float(__ushort_as_half(uint16_t(sw_hi >> sh_hi)));
            if (!p.sym) {
                const uint32_t zw_lo = lds32(sw + 2 * rl0 + 1), zw_hi = lds32(sw + 2 * (rl0 + 8) + 1);
                z_lo = uint32_t(__half2float(__ushort_as_half(uint16_t(zw_lo >> sh_lo))));
                z_hi = uint32_t(__half2float(__ushort_as_half(uint16_t(zw_hi >> sh_hi))));
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);  // weight tile and scales are in registers

        const uint8_t *fr = frag_base + f * p.frag_bytes;
        const uint4 *frq = reinterpret_cast<const uint4 *>(fr);
        const uint32_t wlo[4] = {wa.x, wa.y, wa.z, wa.w};
        const uint32_t whi[4] = {wb.x, wb.y, wb.z, wb.w};
        Acc acc[NT][4];
        if constexpr (WB == 4) {
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[nt][e] = Acc(0);
        }

        if constexpr (AM == A_F16 && WB == 4) {
            // x = 1024 + nibble (low nibbles) or 1024 + 16 * nibble (high nibbles);
            // subtract exactly to q - z.
            const uint32_t c_lo0 = __half_as_ushort(__float2half_rn(-(1024.f + float(z_lo))));
            const uint32_t c_lo1 = __half_as_ushort(__float2half_rn(-(1024.f + float(z_hi))));
            const uint32_t c_hi0 = __half_as_ushort(__float2half_rn(-(64.f + float(z_lo))));
            const uint32_t c_hi1 = __half_as_ushort(__float2half_rn(-(64.f + float(z_hi))));
            const uint32_t clo0 = c_lo0 | (c_lo0 << 16), clo1 = c_lo1 | (c_lo1 << 16);
            const uint32_t chi0 = c_hi0 | (c_hi0 << 16), chi1 = c_hi1 | (c_hi1 << 16);
            const uint32_t sixteenth = 0x2C002C00u;  // 1/16 in both halves
#pragma unroll
            for (int j = 0; j < 4; ++j) {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint32_t x0 = h ? (wlo[j] >> 8) : wlo[j];
                    const uint32_t x1 = h ? (whi[j] >> 8) : whi[j];
                    uint32_t a[4];
                    a[0] = h2_add(and_or(x0, 0x000f000fu, 0x64006400u), clo0);
                    a[1] = h2_add(and_or(x1, 0x000f000fu, 0x64006400u), clo1);
                    a[2] = h2_fma(and_or(x0, 0x00f000f0u, 0x64006400u), sixteenth, chi0);
                    a[3] = h2_fma(and_or(x1, 0x00f000f0u, 0x64006400u), sixteenth, chi1);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        const uint4 b = lds128(frq + (nt * QN + j) * 32 + lane);
                        mma_f16(reinterpret_cast<float(&)[4]>(acc[nt]), a, h ? b.z : b.x, h ? b.w : b.y);
                    }
                }
            }
        } else if constexpr (AM == A_BF16 && WB == 4) {
            // x = 128 + nibble in bf16 (shifted nibbles), minus 128 + z, exact.
            const uint32_t c0 = __bfloat16_as_ushort(__float2bfloat16_rn(-(128.f + float(z_lo))));
            const uint32_t c1 = __bfloat16_as_ushort(__float2bfloat16_rn(-(128.f + float(z_hi))));
            const uint32_t cc0 = c0 | (c0 << 16), cc1 = c1 | (c1 << 16);
            const uint32_t one = 0x3F803F80u;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint32_t a[4];
                    a[0] = bf2_fma(and_or(wlo[j] >> (8 * h), 0x000f000fu, 0x43004300u), one, cc0);
                    a[1] = bf2_fma(and_or(whi[j] >> (8 * h), 0x000f000fu, 0x43004300u), one, cc1);
                    a[2] = bf2_fma(and_or(wlo[j] >> (8 * h + 4), 0x000f000fu, 0x43004300u), one, cc0);
                    a[3] = bf2_fma(and_or(whi[j] >> (8 * h + 4), 0x000f000fu, 0x43004300u), one, cc1);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        const uint4 b = lds128(frq + (nt * QN + j) * 32 + lane);
                        mma_bf16(reinterpret_cast<float(&)[4]>(acc[nt]), a, h ? b.z : b.x, h ? b.w : b.y);
                    }
                }
            }
        } else if constexpr (AM != A_I8 && WB == 2) {
            // 2-bit fields f; c' = f ^ 2 in [0,3]; value c' - 2.  Accumulate across units.
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t y0 = wlo[j] ^ 0xAAAAAAAAu, y1 = whi[j] ^ 0xAAAAAAAAu;
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    // pairs P_{2h}, P_{2h+1}: field shift 2*(2h) and 2*(2h+1) within y (h>=2 use y>>8)
                    const int i0 = 2 * h, i1 = 2 * h + 1;
                    uint32_t a[4];
                    if constexpr (AM == A_F16) {
                        const uint32_t sh0 = (i0 & 3) * 2, sh1 = (i1 & 3) * 2;
                        const uint32_t s0 = (i0 >= 4) ? 8 : 0;
                        const uint32_t m0 = 0x00030003u << sh0, m1 = 0x00030003u << sh1;
                        // multiply by 4^-sh, subtract 1024 * 4^-sh + 2
                        const uint32_t mul0 = sh0 == 0 ? 0x3C003C00u : (sh0 == 2 ? 0x34003400u : (sh0 == 4 ? 0x2C002C00u : 0x24002400u));
                        const uint32_t mul1 = sh1 == 0 ? 0x3C003C00u : (sh1 == 2 ? 0x34003400u : (sh1 == 4 ? 0x2C002C00u : 0x24002400u));
                        const uint32_t add0 = sh0 == 0 ? 0xE402E402u : (sh0 == 2 ? 0xDC08DC08u : (sh0 == 4 ? 0xD420D420u : 0xCC80CC80u));
                        const uint32_t add1 = sh1 == 0 ? 0xE402E402u : (sh1 == 2 ? 0xDC08DC08u : (sh1 == 4 ? 0xD420D420u : 0xCC80CC80u));
                        a[0] = h2_fma(and_or(y0 >> s0, m0, 0x64006400u), mul0, add0);
                        a[1] = h2_fma(and_or(y1 >> s0, m0, 0x64006400u), mul0, add0);
                        a[2] = h2_fma(and_or(y0 >> s0, m1, 0x64006400u), mul1, add1);
                        a[3] = h2_fma(and_or(y1 >> s0, m1, 0x64006400u), mul1, add1);
                    } else {
                        const uint32_t c = 0xC302C302u;  // -(128 + 2) in bf16
                        const uint32_t one = 0x3F803F80u;
                        const int s_0 = (i0 & 3) * 2 + ((i0 >= 4) ? 8 : 0);
                        const int s_1 = (i1 & 3) * 2 + ((i1 >= 4) ? 8 : 0);
                        a[0] = bf2_fma(and_or(y0 >> s_0, 0x00030003u, 0x43004300u), one, c);
                        a[1] = bf2_fma(and_or(y1 >> s_0, 0x00030003u, 0x43004300u), one, c);
                        a[2] = bf2_fma(and_or(y0 >> s_1, 0x00030003u, 0x43004300u), one, c);
                        a[3] = bf2_fma(and_or(y1 >> s_1, 0x00030003u, 0x43004300u), one, c);
                    }
                    const int q = 2 * j + (h >> 1);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        const uint4 b = lds128(frq + (nt * QN + q) * 32 + lane);
                        const uint32_t b0 = (h & 1) ? b.z : b.x, b1 = (h & 1) ? b.w : b.y;
                        if constexpr (AM == A_F16) mma_f16(reinterpret_cast<float(&)[4]>(total[nt]), a, b0, b1);
                        else mma_bf16(reinterpret_cast<float(&)[4]>(total[nt]), a, b0, b1);
                    }
                }
            }
        } else if constexpr (AM == A_I8 && WB == 4) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                uint32_t a[4];
                a[0] = wlo[j] & 0x0f0f0f0fu;
                a[1] = whi[j] & 0x0f0f0f0fu;
                a[2] = (wlo[j] >> 4) & 0x0f0f0f0fu;
                a[3] = (whi[j] >> 4) & 0x0f0f0f0fu;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const uint4 b = lds128(frq + (nt * QN + (j >> 1)) * 32 + lane);
                    mma_u8s8(reinterpret_cast<int(&)[4]>(acc[nt]), a, (j & 1) ? b.z : b.x, (j & 1) ? b.w : b.y);
                }
            }
        } else {  // INT8 activations, INT2 weights: accumulate across units
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t y0 = wlo[j] ^ 0xAAAAAAAAu, y1 = whi[j] ^ 0xAAAAAAAAu;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint32_t a[4];
                    a[0] = (y0 >> (4 * h)) & 0x03030303u;
                    a[1] = (y1 >> (4 * h)) & 0x03030303u;
                    a[2] = (y0 >> (4 * h + 2)) & 0x03030303u;
                    a[3] = (y1 >> (4 * h + 2)) & 0x03030303u;
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        const uint4 b = lds128(frq + (nt * QN + j) * 32 + lane);
                        mma_u8s8(reinterpret_cast<int(&)[4]>(total[nt]), a, h ? b.z : b.x, h ? b.w : b.y);
                    }
                }
            }
        }

        // per-unit fold
        if constexpr (AM == A_I8) {
            const int *sums = reinterpret_cast<const int *>(fr + NT * QN * 512);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int sA0 = sums[nt * 8 + 2 * t], sA1 = sums[nt * 8 + 2 * t + 1];
                if constexpr (WB == 2) {
                    tsum[nt][0] += sA0;
                    tsum[nt][1] += sA1;
                } else {
                    int corr[4];
                    corr[0] = acc[nt][0] - int(z_lo) * sA0;
                    corr[1] = acc[nt][1] - int(z_lo) * sA1;
                    corr[2] = acc[nt][2] - int(z_hi) * sA0;
                    corr[3] = acc[nt][3] - int(z_hi) * sA1;
                    if (p.acc_out) {
                        const int n_lo = r * kRows + rl0, n_hi = n_lo + 8;
                        const int m = nt * 8 + 2 * t;
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int n = (e < 2) ? n_lo : n_hi, mm = m + (e & 1);
                            if (n < p.N && mm < p.M)
                                p.acc_out[((long long)(p.m0 + mm) * p.N + n) * p.G + kb] = corr[e];
                        }
                    }
                    float *tf = reinterpret_cast<float *>(total[nt]);
                    tf[0] = fmaf(s_lo, float(corr[0]), tf[0]);
                    tf[1] = fmaf(s_lo, float(corr[1]), tf[1]);
                    tf[2] = fmaf(s_hi, float(corr[2]), tf[2]);
                    tf[3] = fmaf(s_hi, float(corr[3]), tf[3]);
                }
            }
        } else if constexpr (WB == 4) {
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                float *tf = reinterpret_cast<float *>(total[nt]);
                const float *af = reinterpret_cast<const float *>(acc[nt]);
                tf[0] = fmaf(s_lo, af[0], tf[0]);
                tf[1] = fmaf(s_lo, af[1], tf[1]);
                tf[2] = fmaf(s_hi, af[2], tf[2]);
                tf[3] = fmaf(s_hi, af[3], tf[3]);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&fempty[f]);

        // ------------------------------------------------ end of a row-group segment
        const bool seg_end = (kb == p.KB - 1) || (i == nunits - 1);
        if (!seg_end) continue;
        if constexpr (AM == A_I8 && WB == 2) {
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                int *ti = reinterpret_cast<int *>(total[nt]);
                ti[0] -= 2 * tsum[nt][0];
                ti[1] -= 2 * tsum[nt][1];
                ti[2] -= 2 * tsum[nt][0];
                ti[3] -= 2 * tsum[nt][1];
            }
        }
        const int n_lo = r * kRows + rl0;
        if (seg_start == 0 && kb == p.KB - 1) {
            // the whole row group is ours: finish and store
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int n = n_lo + ((e & 2) ? 8 : 0), m = nt * 8 + 2 * t + (e & 1);
                    if (n >= p.N || m >= p.M) continue;
                    const float tf = reinterpret_cast<const float *>(total[nt])[e];
                    const int ti = reinterpret_cast<const int *>(total[nt])[e];
                    store_out<AM>(p.C, (long long)(p.m0 + m) * p.N + n, finish<WB, AM>(p, tf, ti, n, m));
                    if (AM == A_I8 && WB == 2 && p.acc_out) p.acc_out[(long long)(p.m0 + m) * p.N + n] = ti;
                }
            continue;
        }
        // partial row group: publish, count, and let the last contributor finish
        const int slot = (r == int(begin / p.KB)) ? 0 : 1;
        float *mine = p.ws_partial + ((size_t)(cta * 2 + slot) * kRows) * MP;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int m = nt * 8 + 2 * t;
            *reinterpret_cast<float2 *>(mine + rl0 * MP + m) = make_float2(reinterpret_cast<float *>(total[nt])[0],
                                                                           reinterpret_cast<float *>(total[nt])[1]);
            *reinterpret_cast<float2 *>(mine + (rl0 + 8) * MP + m) =
                make_float2(reinterpret_cast<float *>(total[nt])[2], reinterpret_cast<float *>(total[nt])[3]);
        }
        __threadfence();
        mbar_arrive(csync);
        if (!wait_bar(csync, csync_phase & 1)) { ok = false; break; }
        ++csync_phase;
        const long long u0 = (long long)r * p.KB;
        const int c_first = cta_of_unit(p, u0), c_last = cta_of_unit(p, u0 + p.KB - 1);
        if (threadIdx.x == 0) {
            const unsigned old = atomicInc(&p.ws_counter[r], unsigned(c_last - c_first));
            *flag = (old == unsigned(c_last - c_first)) ? 1 : 0;
        }
        mbar_arrive(csync);
        if (!wait_bar(csync, csync_phase & 1)) { ok = false; break; }
        ++csync_phase;
        if (*flag) {
            __threadfence();
            for (int e = threadIdx.x; e < kRows * MP; e += kConsumerWarps * 32) {
                const int rl = e / MP, m = e % MP;
                const int n = r * kRows + rl;
                float sf = 0.f;
                int si = 0;
                for (int c = c_first; c <= c_last; ++c) {
                    const int sl = (int(range_begin(p, c) / p.KB) == r) ? 0 : 1;
                    const float v = __ldcg(p.ws_partial + ((size_t)(c * 2 + sl) * kRows + rl) * MP + m);
                    sf += v;
                    si += __float_as_int(v);
                }
                if (n >= p.N || m >= p.M) continue;
                store_out<AM>(p.C, (long long)(p.m0 + m) * p.N + n, finish<WB, AM>(p, sf, si, n, m));
                if (AM == A_I8 && WB == 2 && p.acc_out) p.acc_out[(long long)(p.m0 + m) * p.N + n] = si;
            }
        }
        // the flag word is reused by the next partial segment: make sure everyone read it
        mbar_arrive(csync);
        if (!wait_bar(csync, csync_phase & 1)) { ok = false; break; }
        ++csync_phase;
    }
}

// ---------------------------------------------------------------- host side
struct Plan {
    int NT = 1, MP = 8, KU = 128, KB = 0, RG = 0, P = 0, split = 0, S = 0;
    long long U = 0;
    int ablk = 0, frag = 0;
    size_t smem = 0, ws_need = 0;
};

int choose_nt(int64_t M) { return M <= 8 ? 1 : (M <= 16 ? 2 : (M <= 32 ? 4 : 8)); }

Plan make_plan(int64_t M, int64_t N, int64_t K, int WB, int AM, size_t ws_bytes, const DeviceInfo &dev)
{
    Plan pl;
    pl.NT = choose_nt(M);
    pl.MP = pl.NT * 8;
    pl.KU = kunit_of(WB);
    pl.KB = int((K + pl.KU - 1) / pl.KU);
    pl.RG = int((N + kRows - 1) / kRows);
    pl.U = (long long)pl.KB * pl.RG;
    const int esize = AM == A_I8 ? 1 : 2;
    pl.ablk = pl.MP * pl.KU * esize;
    const int steps = steps_of(WB, AM);
    pl.frag = pl.NT * steps * 256 + (AM == A_I8 ? 256 : 0);
    // partials: sm_count CTAs x 2 x kRows x MP floats (<= 64 KB per SM); counters after the
    // shared scratch area
    pl.ws_need = ws_scratch_bytes() + size_t(pl.RG) * sizeof(unsigned);
    pl.ws_need = (pl.ws_need + 255) & ~size_t(255);
    pl.split = (ws_bytes >= pl.ws_need) ? 1 : 0;
    pl.P = int(std::min<long long>(dev.sm_count, pl.split ? pl.U : pl.RG));
    const long long max_units = pl.split ? (pl.U + pl.P - 1) / pl.P : (long long)((pl.RG + pl.P - 1) / pl.P) * pl.KB;
    const size_t stage = kWTile + pl.ablk + kScaleBytes;
    const size_t fixed = 1024 /*align*/ + kFragBufs * size_t(pl.frag) + 8 * (2 * 16 + 2 * kFragBufs + 1) + 16;
    const long long fit = (long long)((size_t(dev.max_smem_optin) - fixed) / stage);
    pl.S = int(std::max<long long>(2, std::min<long long>({16, fit, std::max<long long>(2, max_units)})));
    pl.smem = fixed + size_t(pl.S) * stage;
    return pl;
}

template <int WB, int AM, int NT>
wq_status launch_one(const Plan &pl, const CUtensorMap &tw, const CUtensorMap &ta, const SkinnyParams &p,
                     cudaStream_t st)
{
    auto kern = skinny_kernel<WB, AM, NT>;
    static size_t configured = 0;
    if (pl.smem > configured) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(pl.smem)) != cudaSuccess)
            return check_launch("cudaFuncSetAttribute(skinny)");
        configured = pl.smem;
    }
    kern<<<pl.P, kThreads, pl.smem, st>>>(tw, ta, p);
    return check_launch("skinny_kernel");
}

template <int WB, int AM>
wq_status launch_nt(int NT, const Plan &pl, const CUtensorMap &tw, const CUtensorMap &ta, const SkinnyParams &p,
                    cudaStream_t st)
{
    switch (NT) {
    case 1: return launch_one<WB, AM, 1>(pl, tw, ta, p, st);
    case 2: return launch_one<WB, AM, 2>(pl, tw, ta, p, st);
    case 4: return launch_one<WB, AM, 4>(pl, tw, ta, p, st);
    default: return launch_one<WB, AM, 8>(pl, tw, ta, p, st);
    }
}

}  // namespace

// Entry used by the C ABI: validated arguments, any M (launched in chunks of <= 64 tokens).
wq_status skinny_gemm(int WB, int AM, const void *A, const float *a_scale, const uint8_t *Wq, const void *scales,
                      const void *zeros, const void *bias, void *C, int32_t *acc_out, int64_t M, int64_t N, int64_t K,
                      const wq_qconfig &c, void *ws, size_t ws_bytes, cudaStream_t st)
{
    const DeviceInfo &dev = device_info();
    const int64_t chunk = std::min<int64_t>(M, 64);
    Plan pl = make_plan(chunk, N, K, WB, AM, ws_bytes, dev);
    if (!ws) pl = make_plan(chunk, N, K, WB, AM, 0, dev);

    CUtensorMap tw, ta;
    const uint64_t row_bytes = uint64_t(K) * WB / 8;
    wq_status rc = encode_tmap_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, Wq, row_bytes, uint64_t(N), row_bytes,
                                  kUnitBytes, kRows);
    if (rc != WQ_OK) return rc;
    const int esize = AM == A_I8 ? 1 : 2;
    rc = encode_tmap_2d(&ta, AM == A_I8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_UINT16, A,
                        uint64_t(K), uint64_t(M), uint64_t(K) * esize, uint32_t(pl.KU), uint32_t(pl.MP));
    if (rc != WQ_OK) return rc;

    SkinnyParams p{};
    p.N = int(N);
    p.K = int(K);
    p.G = WB == 4 ? int(K / c.group_size) : 1;
    p.gs = WB == 4 ? c.group_size : int(K);
    p.sym = WB == 4 ? c.symmetric : 1;
    p.KB = pl.KB;
    p.RG = pl.RG;
    p.U = pl.U;
    p.P = pl.P;
    p.split = pl.split;
    p.S = pl.S;
    p.ablk_bytes = pl.ablk;
    p.frag_bytes = pl.frag;
    p.scales16 = static_cast<const uint16_t *>(scales);
    p.scale32 = static_cast<const float *>(scales);
    p.zeros = static_cast<const uint16_t *>(zeros);
    p.bias = bias;
    p.a_scale = a_scale;
    p.C = C;
    p.acc_out = acc_out;
    p.ws_partial = pl.split ? static_cast<float *>(ws) : nullptr;
    p.ws_counter = pl.split ? reinterpret_cast<unsigned *>(static_cast<uint8_t *>(ws) + ws_scratch_bytes()) : nullptr;
    for (int64_t m0 = 0; m0 < M; m0 += 64) {
        p.m0 = int(m0);
        p.M = int(std::min<int64_t>(64, M - m0));
        const int NT = choose_nt(p.M);
        Plan plc = (NT == pl.NT) ? pl : make_plan(p.M, N, K, WB, AM, p.split ? ws_bytes : 0, dev);
        if (NT != pl.NT) {
            // the activation box height follows the tile width of this chunk
            rc = encode_tmap_2d(&ta, AM == A_I8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_UINT16, A,
                                uint64_t(K), uint64_t(M), uint64_t(K) * esize, uint32_t(plc.KU), uint32_t(plc.MP));
            if (rc != WQ_OK) return rc;
            p.ablk_bytes = plc.ablk;
            p.frag_bytes = plc.frag;
            p.S = plc.S;
            p.P = plc.P;
            p.split = plc.split;
        }
        if (WB == 4 && AM == A_F16) rc = launch_nt<4, A_F16>(NT, plc, tw, ta, p, st);
        else if (WB == 4 && AM == A_BF16) rc = launch_nt<4, A_BF16>(NT, plc, tw, ta, p, st);
        else if (WB == 4) rc = launch_nt<4, A_I8>(NT, plc, tw, ta, p, st);
        else if (AM == A_F16) rc = launch_nt<2, A_F16>(NT, plc, tw, ta, p, st);
        else if (AM == A_BF16) rc = launch_nt<2, A_BF16>(NT, plc, tw, ta, p, st);
        else rc = launch_nt<2, A_I8>(NT, plc, tw, ta, p, st);
        if (rc != WQ_OK) return rc;
    }
    return WQ_OK;
}

size_t skinny_workspace_size(int WB, int AM, int64_t M, int64_t N, int64_t K)
{
    const Plan pl = make_plan(std::min<int64_t>(M, 64), N, K, WB, AM, 0, device_info());
    return pl.ws_need;
}

int skinny_read_error()
{
    int v = 0, zero = 0;
    cudaMemcpyFromSymbol(&v, g_skinny_error, sizeof v);
    cudaMemcpyToSymbol(g_skinny_error, &zero, sizeof zero);
    return v;
}

}  // namespace wq
