// wq_gemv.cu -- decode GEMV / few-token matmul (M <= 16) over packed INT4 / INT2 weights.
//
// C[M,N] = A[M,K] x dequant(Wq[N,K])^T ("BitBLAS practical guide", "What is BitBLAS",
// layout "nt"), FP16 / BF16 activations (W4A16) or per-token INT8 activations with exact
// INT32 group sums and the (a_scale x w_scale) epilogue (W4A8: "Accelerating LLM inference
// with CUDA Graph and INT4 quantization", part 1, steps 3-4).
//
// The kernel is HBM-bound: it must keep every SM's share of the packed weights in flight.
//  * Rows are cut into 16-row tiles; CTA c (one per SM) owns tiles [cT/P, (c+1)T/P) and all
//    of K, so no CTA ever needs another's result (no cross-CTA reduction).
//  * K is walked in chunks of 8 units (a unit = 64 packed bytes of a row: 128 k of INT4,
//    256 k of INT2).  A producer warp issues, per chunk, one 2D TMA box (16 rows x 64 B) per
//    (tile, unit) and one box (M tokens x unit) of activations into an S-stage ring.  The
//    weight boxes of the first S chunks are issued before griddepcontrol.wait, so with
//    programmatic dependent launch they stream while the previous kernel finishes.
//  * The CTA's scale / zero rows (contiguous in the [N, K/g] layout) arrive with one bulk
//    copy each.
//  * Consumer warp w handles unit w of every chunk for all of the CTA's tiles: it builds the
//    mma.sync B fragments of its unit once (in registers) and reuses them for every tile.
//    Weights are unpacked with LOP3 into exact integers q - z and multiplied on the tensor
//    cores; each unit's fp32 (or int32) sum is folded with its group scale.
//  * At the end the 8 warps' partial sums are added in a fixed order through shared memory
//    (deterministic) and the epilogue writes C.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include <algorithm>
#include <type_traits>

#include "wq_device.cuh"
#include "wq_host.h"
#include "wq_unit.cuh"

namespace wq {

static __device__ int g_gemv_error;

namespace {

constexpr int kCW = 8;                   // consumer warps; one unit of each chunk per warp
constexpr int kThreads = (kCW + 1) * 32; // + producer warp
constexpr int kKC = 8;                   // units per chunk
constexpr int kTileRows = 16;
constexpr int kUnitBytes = 64;
constexpr int kBox = kTileRows * kUnitBytes;  // one unit of one tile: 1 KB
// tiles processed together (their sums live in registers)
__host__ __device__ constexpr int tg_max(int WB, int AM, int NT) { return (AM != A_I8 && WB == 4) ? (NT == 1 ? 8 : 6) : 4; }

struct GemvParams {
    int M, N, K, G, gs, sym, m0;
    int KB, T, P, nch, TG, S;
    int a_pitch, ablk_bytes, wpart_bytes, stage_bytes;
    int sc_smem, sc_rows_cap;
    const uint16_t *scales16;
    const float *scale32;
    const uint16_t *zeros;
    const void *bias;
    const float *a_scale;
    void *C;
    int32_t *acc_out;
};

__device__ __forceinline__ uint64_t globaltimer()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// Bounded wait (~2 s of wall clock); records an error and returns false on expiry.
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity)
{
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    for (;;) {
        for (int i = 0; i < 64; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (globaltimer() - t0 > 2000000000ull) {
            atomicCAS(&g_gemv_error, kErrNone, kErrWaitTimeout);
            return false;
        }
    }
}

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

template <int WB, int AM>
__device__ __forceinline__ float finish(const GemvParams &p, float total_f, int total_i, int n, int m)
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

// ACC: also write every INT32 group sum to p.acc_out (a debugging output of W4A8).
template <int WB, int AM, int NT, bool ACC>
__global__ void __launch_bounds__(kThreads, 1)
    gemv_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_a,
                const GemvParams p)
{
    constexpr int MP = NT * 8;
    constexpr int KU = kunit_of(WB);
    constexpr int QN = qn_of(WB, AM);
    constexpr int kTGMax = tg_max(WB, AM, NT);

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int S = p.S;
    uint8_t *ring = smem;
    uint16_t *sc = reinterpret_cast<uint16_t *>(ring + size_t(S) * p.stage_bytes);
    uint16_t *zc = sc + size_t(p.sc_rows_cap) * p.G;
    uint64_t *bars = reinterpret_cast<uint64_t *>(
        (reinterpret_cast<uintptr_t>(zc + size_t(p.sc_rows_cap) * p.G) + 15) & ~uintptr_t(15));
    uint64_t *full = bars, *empty = bars + S, *scbar = bars + 2 * S, *cbar = bars + 2 * S + 1;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = blockIdx.x;
    const int t0 = int((long long)c * p.T / p.P), t1 = int((long long)(c + 1) * p.T / p.P);
    const int ntc = t1 - t0;
    const int ngrp = (ntc + p.TG - 1) / p.TG;
    const int total_it = ngrp * p.nch;
    const int r0 = t0 * kTileRows, r1 = min(t1 * kTileRows, p.N);

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kCW);
        }
        mbar_init(scbar, 2);
        mbar_init(cbar, kCW * 32);
        fence_barrier_init();
    }
    __syncthreads();
    // the next kernel in the stream may start launching on SMs as they free up
    grid_dep_launch();

    if (warp == kCW) {
        // ------------------------------------------------------------ producer warp
        if (lane == 0) {
            tma_prefetch_desc(&tmap_w);
            tma_prefetch_desc(&tmap_a);
        }
        // scale / zero rows of this CTA: contiguous, 16-byte aligned at the start
        const bool want_sc = (WB == 4) && p.sc_smem;
        const uint32_t sc_bytes = want_sc ? uint32_t(r1 - r0) * p.G * 2 : 0u;
        const uint32_t sc16 = sc_bytes & ~15u;
        if (lane == 0) {
            mbar_arrive_expect_tx(scbar, sc16 * (p.sym ? 1 : 2));
            if (sc16) {
                bulk_load(sc, p.scales16 + (size_t)r0 * p.G, sc16, scbar);
                if (!p.sym) bulk_load(zc, p.zeros + (size_t)r0 * p.G, sc16, scbar);
            }
        }
        if constexpr (WB == 4) {
            for (uint32_t e = (sc16 >> 1) + uint32_t(lane); e < (sc_bytes >> 1); e += 32u) {  // ragged tail
                sc[e] = p.scales16[(size_t)r0 * p.G + e];
                if (!p.sym) zc[e] = p.zeros[(size_t)r0 * p.G + e];
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(scbar);

        auto issue = [&](int it, bool weights, bool acts) {
            const int s = it % S;
            const int grp = it / p.nch, ch = it % p.nch;
            const int ntg = min(p.TG, ntc - grp * p.TG);
            const int kb0 = ch * kKC, nkb = min(kKC, p.KB - kb0);
            uint8_t *st = ring + size_t(s) * p.stage_bytes;
            if (weights) {
                if (lane == 0) mbar_arrive_expect_tx(&full[s], uint32_t(ntg * nkb * kBox + nkb * p.ablk_bytes));
                __syncwarp();
                for (int idx = lane; idx < ntg * nkb; idx += 32) {
                    const int i = idx / nkb, kk = idx % nkb;
                    tma_load_2d(st + (i * kKC + kk) * kBox, &tmap_w, (kb0 + kk) * kUnitBytes,
                                (t0 + grp * p.TG + i) * kTileRows, &full[s]);
                }
            }
            if (acts)
                for (int kk = lane; kk < nkb; kk += 32)
                    tma_load_2d(st + p.wpart_bytes + kk * p.ablk_bytes, &tmap_a, (kb0 + kk) * KU, p.m0, &full[s]);
        };
        const int pro = min(S, total_it);
        for (int it = 0; it < pro; ++it) issue(it, true, false);
        grid_dep_wait();  // activations may be produced by the previous kernel
        for (int it = 0; it < pro; ++it) issue(it, false, true);
        int it = pro;
        for (; it < total_it; ++it) {
            if (!wait_bar(&empty[it % S], ((it / S) - 1) & 1)) break;
            issue(it, true, true);
        }
        for (int k = max(0, it - S); k < it; ++k) wait_bar(&full[k % S], (k / S) & 1);
        return;
    }

    // ---------------------------------------------------------------- consumer warps
    const int g = lane >> 2, t = lane & 3;
    if (!wait_bar(scbar, 0)) return;
    grid_dep_wait();
    uint32_t cphase = 0;
    auto csync = [&]() -> bool {
        mbar_arrive(cbar);
        const bool ok = wait_bar(cbar, cphase & 1);
        ++cphase;
        return ok;
    };

    for (int grp = 0; grp < ngrp; ++grp) {
        const int ntg = min(p.TG, ntc - grp * p.TG);
        // running sums: fp32, or exact int32 for INT2 x INT8 (one group spans K)
        using Tot = typename std::conditional<AM == A_I8 && WB == 2, int, float>::type;
        Tot tot[kTGMax][NT][4];
        int tsum[NT][2];
#pragma unroll
        for (int i = 0; i < kTGMax; ++i)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) tot[i][nt][e] = Tot(0);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) tsum[nt][0] = tsum[nt][1] = 0;

        int s = 0;
        for (int ch = 0; ch < p.nch; ++ch) {
            const int it = grp * p.nch + ch;
            s = it % S;
            if (!wait_bar(&full[s], (it / S) & 1)) return;
            const uint8_t *st = ring + size_t(s) * p.stage_bytes;
            const int kb = ch * kKC + warp;
            if (kb < p.KB) {
                uint4 bf[NT][QN];
                int asum[NT];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
                    build_bfrag<WB, AM>(st + p.wpart_bytes + warp * p.ablk_bytes, p.a_pitch, p.M, nt, lane, bf[nt],
                                        asum[nt]);
                int sA[NT][2];  // INT8 activations: unit sums of tokens 2t, 2t+1 of each tile
                if constexpr (AM == A_I8) {
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        int v = asum[nt];
                        v += __shfl_xor_sync(0xffffffffu, v, 1);
                        v += __shfl_xor_sync(0xffffffffu, v, 2);
                        sA[nt][0] = __shfl_sync(0xffffffffu, v, (2 * t) * 4);
                        sA[nt][1] = __shfl_sync(0xffffffffu, v, (2 * t + 1) * 4);
                        tsum[nt][0] += sA[nt][0];
                        tsum[nt][1] += sA[nt][1];
                    }
                }
                const int gi = (WB == 4) ? (kb * KU) / p.gs : 0;
#pragma unroll
                for (int i = 0; i < kTGMax; ++i) {
                    if (i >= ntg) break;
                    const uint8_t *wt = st + (i * kKC + warp) * kBox;
                    const uint4 wa = lds128(wt + g * kUnitBytes + 16 * t);
                    const uint4 wb = lds128(wt + (g + 8) * kUnitBytes + 16 * t);
                    const int rl = (grp * p.TG + i) * kTileRows + g;  // row within the CTA
                    const int n_lo = r0 + rl, n_hi = n_lo + 8;
                    float s_lo = 0.f, s_hi = 0.f;
                    uint32_t z_lo = 8, z_hi = 8;
                    if constexpr (WB == 4) {
                        uint16_t hs_lo = 0, hs_hi = 0, hz_lo = 0, hz_hi = 0;
                        if (p.sc_smem) {
                            if (n_lo < p.N) { hs_lo = sc[rl * p.G + gi]; hz_lo = p.sym ? 0 : zc[rl * p.G + gi]; }
                            if (n_hi < p.N) { hs_hi = sc[(rl + 8) * p.G + gi]; hz_hi = p.sym ? 0 : zc[(rl + 8) * p.G + gi]; }
                        } else {
                            if (n_lo < p.N) { hs_lo = p.scales16[(size_t)n_lo * p.G + gi]; hz_lo = p.sym ? 0 : p.zeros[(size_t)n_lo * p.G + gi]; }
                            if (n_hi < p.N) { hs_hi = p.scales16[(size_t)n_hi * p.G + gi]; hz_hi = p.sym ? 0 : p.zeros[(size_t)n_hi * p.G + gi]; }
                        }
                        s_lo = __half2float(__ushort_as_half(hs_lo));
                        s_hi = __half2float(__ushort_as_half(hs_hi));
                        if (!p.sym) {
                            z_lo = uint32_t(__half2float(__ushort_as_half(hz_lo)));
                            z_hi = uint32_t(__half2float(__ushort_as_half(hz_hi)));
                        }
                    }
                    if constexpr (WB == 2) {
                        // INT2: no per-unit scale; accumulate straight into the totals
                        unit_mma<WB, AM, NT>(wa, wb, bf, z_lo, z_hi, tot[i]);
                    } else {
                        acc_t<AM> ua[NT][4];
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                            for (int e = 0; e < 4; ++e) ua[nt][e] = acc_t<AM>(0);
                        unit_mma<WB, AM, NT>(wa, wb, bf, z_lo, z_hi, ua);
                        if constexpr (AM == A_I8) {
#pragma unroll
                            for (int nt = 0; nt < NT; ++nt) {
                                int corr[4];
                                corr[0] = ua[nt][0] - int(z_lo) * sA[nt][0];
                                corr[1] = ua[nt][1] - int(z_lo) * sA[nt][1];
                                corr[2] = ua[nt][2] - int(z_hi) * sA[nt][0];
                                corr[3] = ua[nt][3] - int(z_hi) * sA[nt][1];
                                if constexpr (ACC) {
                                    const int m = nt * 8 + 2 * t;
#pragma unroll
                                    for (int e = 0; e < 4; ++e) {
                                        const int n = (e < 2) ? n_lo : n_hi, mm = m + (e & 1);
                                        if (n < p.N && mm < p.M)
                                            p.acc_out[((long long)(p.m0 + mm) * p.N + n) * p.G + kb] = corr[e];
                                    }
                                }
                                tot[i][nt][0] = fmaf(s_lo, float(corr[0]), tot[i][nt][0]);
                                tot[i][nt][1] = fmaf(s_lo, float(corr[1]), tot[i][nt][1]);
                                tot[i][nt][2] = fmaf(s_hi, float(corr[2]), tot[i][nt][2]);
                                tot[i][nt][3] = fmaf(s_hi, float(corr[3]), tot[i][nt][3]);
                            }
                        } else {
#pragma unroll
                            for (int nt = 0; nt < NT; ++nt) {
                                tot[i][nt][0] = fmaf(s_lo, ua[nt][0], tot[i][nt][0]);
                                tot[i][nt][1] = fmaf(s_lo, ua[nt][1], tot[i][nt][1]);
                                tot[i][nt][2] = fmaf(s_hi, ua[nt][2], tot[i][nt][2]);
                                tot[i][nt][3] = fmaf(s_hi, ua[nt][3], tot[i][nt][3]);
                            }
                        }
                    }
                }
            }
            if (ch + 1 < p.nch) {
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[s]);
            }
        }

        // ---- add the 8 warps' partial sums (fixed order) and write C ----
        // The last chunk's stage stays held; its weight part becomes the reduction buffer.
        if constexpr (AM == A_I8 && WB == 2) {
#pragma unroll
            for (int i = 0; i < kTGMax; ++i)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    tot[i][nt][0] -= 2 * tsum[nt][0];
                    tot[i][nt][1] -= 2 * tsum[nt][1];
                    tot[i][nt][2] -= 2 * tsum[nt][0];
                    tot[i][nt][3] -= 2 * tsum[nt][1];
                }
        }
        if (!csync()) return;  // every warp is done reading the held stage
        float *red = reinterpret_cast<float *>(ring + size_t(s) * p.stage_bytes);
#pragma unroll
        for (int i = 0; i < kTGMax; ++i) {
            if (i >= ntg) break;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                float v[4];
#pragma unroll
                for (int e = 0; e < 4; ++e)
                {
                    if constexpr (AM == A_I8 && WB == 2) v[e] = __int_as_float(tot[i][nt][e]);
                    else v[e] = tot[i][nt][e];
                }
                const int m = nt * 8 + 2 * t;
                float *base = red + ((size_t)(warp * p.TG + i) * kTileRows) * MP;
                *reinterpret_cast<float2 *>(base + g * MP + m) = make_float2(v[0], v[1]);
                *reinterpret_cast<float2 *>(base + (g + 8) * MP + m) = make_float2(v[2], v[3]);
            }
        }
        if (!csync()) return;
        const int rows = ntg * kTileRows;
        for (int e = threadIdx.x; e < rows * MP; e += kCW * 32) {
            const int m = e / rows, rr = e % rows;
            const int i = rr / kTileRows, r = rr % kTileRows;
            const int n = r0 + (grp * p.TG + i) * kTileRows + r;
            if (n >= p.N || m >= p.M) continue;
            float sf = 0.f;
            int si = 0;
#pragma unroll
            for (int w = 0; w < kCW; ++w) {
                const float v = red[((size_t)(w * p.TG + i) * kTileRows + r) * MP + m];
                sf += v;
                si += __float_as_int(v);
            }
            store_out<AM>(p.C, (long long)(p.m0 + m) * p.N + n, finish<WB, AM>(p, sf, si, n, m));
            if constexpr (AM == A_I8 && WB == 2)
                if (p.acc_out) p.acc_out[(long long)(p.m0 + m) * p.N + n] = si;
        }
        if (!csync()) return;
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
    }
}

// ---------------------------------------------------------------- host side
struct Plan {
    int NT = 1, MP = 8, KU = 128, KB = 0, T = 0, P = 0, nch = 0, TG = 1, S = 2;
    int a_pitch = 0, ablk = 0, wpart = 0, stage = 0, sc_smem = 0, sc_rows_cap = 0;
    size_t smem = 0;
    bool ok = false;
};

Plan make_plan(int64_t M, int64_t N, int64_t K, int WB, int AM, int G, const DeviceInfo &dev)
{
    Plan pl;
    pl.NT = M <= 8 ? 1 : 2;
    pl.MP = pl.NT * 8;
    pl.KU = kunit_of(WB);
    pl.KB = int((K + pl.KU - 1) / pl.KU);
    pl.T = int((N + kTileRows - 1) / kTileRows);
    pl.P = std::min(dev.sm_count, pl.T);
    pl.nch = (pl.KB + kKC - 1) / kKC;
    const int tiles_max = (pl.T + pl.P - 1) / pl.P;
    const int esize = AM == A_I8 ? 1 : 2;
    pl.a_pitch = pl.KU * esize;
    pl.ablk = int(M) * pl.a_pitch;
    pl.sc_rows_cap = tiles_max * kTileRows;
    const size_t sc_bytes = (WB == 4) ? size_t(pl.sc_rows_cap) * G * 2 * 2 : 0;
    pl.sc_smem = (WB == 4 && sc_bytes <= 48 * 1024) ? 1 : 0;
    if (!pl.sc_smem) pl.sc_rows_cap = 0;
    const size_t sc_area = pl.sc_smem ? sc_bytes : 0;
    const size_t budget = size_t(dev.max_smem_optin) - 1024 - 64 - 16 * 8 - 16;
    for (pl.TG = std::min(tg_max(WB, AM, pl.NT), tiles_max); pl.TG >= 1; --pl.TG) {
        pl.wpart = pl.TG * kKC * kBox;
        // the weight part doubles as the cross-warp reduction buffer
        const int red = kCW * pl.TG * kTileRows * pl.MP * 4;
        if (red > pl.wpart) continue;
        pl.stage = pl.wpart + kKC * pl.ablk;
        pl.stage = (pl.stage + 127) & ~127;
        const int ngrp = (tiles_max + pl.TG - 1) / pl.TG;
        const long long fit = (long long)((budget - sc_area) / pl.stage);
        const long long want = std::min<long long>(8, (long long)ngrp * pl.nch);
        if (fit < 2 && want >= 2) continue;
        pl.S = int(std::max<long long>(1, std::min(fit, want)));
        pl.smem = 1024 + size_t(pl.S) * pl.stage + sc_area + 16 + 8 * (2 * pl.S + 2) + 16;
        pl.ok = true;
        break;
    }
    return pl;
}

template <int WB, int AM, int NT, bool ACC = false>
wq_status launch(const Plan &pl, const CUtensorMap &tw, const CUtensorMap &ta, const GemvParams &p, cudaStream_t st)
{
    auto kern = gemv_kernel<WB, AM, NT, ACC>;
    static size_t configured = 0;
    if (pl.smem > configured) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(pl.smem)) != cudaSuccess)
            return check_launch("cudaFuncSetAttribute(gemv)");
        configured = pl.smem;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(pl.P);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = pl.smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, tw, ta, p);
    if (e != cudaSuccess) return fail(WQ_ERR_CUDA, "gemv_kernel launch: %s", cudaGetErrorString(e));
    return check_launch("gemv_kernel");
}

}  // namespace

// Few-token path (1 <= M <= 16).  Returns WQ_ERR_UNSUPPORTED if no launch plan fits.
wq_status gemv_small_m(int WB, int AM, const void *A, const float *a_scale, const uint8_t *Wq, const void *scales,
                       const void *zeros, const void *bias, void *C, int32_t *acc_out, int64_t M, int64_t N,
                       int64_t K, const wq_qconfig &c, cudaStream_t st)
{
    const DeviceInfo &dev = device_info();
    const int G = WB == 4 ? int(K / c.group_size) : 1;
    const Plan pl = make_plan(M, N, K, WB, AM, G, dev);
    if (!pl.ok) return fail(WQ_ERR_UNSUPPORTED, "no shared-memory plan for M=%lld K=%lld", (long long)M, (long long)K);
    CUtensorMap tw, ta;
    const uint64_t row_bytes = uint64_t(K) * WB / 8;
    wq_status rc = encode_tmap_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, Wq, row_bytes, uint64_t(N), row_bytes,
                                  kUnitBytes, kTileRows);
    if (rc != WQ_OK) return rc;
    const int esize = AM == A_I8 ? 1 : 2;
    rc = encode_tmap_2d(&ta, AM == A_I8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_UINT16, A,
                        uint64_t(K), uint64_t(M), uint64_t(K) * esize, uint32_t(pl.KU), uint32_t(M));
    if (rc != WQ_OK) return rc;
    GemvParams p{};
    p.M = int(M);
    p.N = int(N);
    p.K = int(K);
    p.G = G;
    p.gs = WB == 4 ? c.group_size : int(K);
    p.sym = WB == 4 ? c.symmetric : 1;
    p.m0 = 0;
    p.KB = pl.KB;
    p.T = pl.T;
    p.P = pl.P;
    p.nch = pl.nch;
    p.TG = pl.TG;
    p.S = pl.S;
    p.a_pitch = pl.a_pitch;
    p.ablk_bytes = pl.ablk;
    p.wpart_bytes = pl.wpart;
    p.stage_bytes = pl.stage;
    p.sc_smem = pl.sc_smem;
    p.sc_rows_cap = pl.sc_rows_cap;
    p.scales16 = static_cast<const uint16_t *>(scales);
    p.scale32 = static_cast<const float *>(scales);
    p.zeros = static_cast<const uint16_t *>(zeros);
    p.bias = bias;
    p.a_scale = a_scale;
    p.C = C;
    p.acc_out = acc_out;
    const int NT = pl.NT;
#define WQ_LAUNCH(wb, am)                                                         \
    return NT == 1 ? launch<wb, am, 1>(pl, tw, ta, p, st) : launch<wb, am, 2>(pl, tw, ta, p, st)
    if (WB == 4 && AM == A_F16) WQ_LAUNCH(4, A_F16);
    if (WB == 4 && AM == A_BF16) WQ_LAUNCH(4, A_BF16);
    if (WB == 4 && acc_out)
        return NT == 1 ? launch<4, A_I8, 1, true>(pl, tw, ta, p, st) : launch<4, A_I8, 2, true>(pl, tw, ta, p, st);
    if (WB == 4) WQ_LAUNCH(4, A_I8);
    if (AM == A_F16) WQ_LAUNCH(2, A_F16);
    if (AM == A_BF16) WQ_LAUNCH(2, A_BF16);
    WQ_LAUNCH(2, A_I8);
#undef WQ_LAUNCH
}

int gemv_read_error()
{
    int v = 0, zero = 0;
    cudaMemcpyFromSymbol(&v, g_gemv_error, sizeof v);
    cudaMemcpyToSymbol(g_gemv_error, &zero, sizeof zero);
    return v;
}

}  // namespace wq
