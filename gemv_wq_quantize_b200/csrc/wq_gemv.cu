// wq_gemv.cu -- decode GEMV / few-token matmul (M <= 16) over packed INT4 / INT2 weights.
//
// C[M,N] = A[M,K] x dequant(Wq[N,K])^T ("BitBLAS practical guide", "What is BitBLAS",
// layout "nt"), FP16 / BF16 activations (W4A16) or per-token INT8 activations with exact
// INT32 group sums and the (a_scale x w_scale) epilogue (W4A8: "Accelerating LLM inference
// with CUDA Graph and INT4 quantization", part 1, steps 3-4).
//
// The kernel is HBM-bound and short (a few microseconds); it is built to have every SM's
// share of the packed weights in flight early and to keep the tensor pipe fed:
//  * Rows are cut into 16-row tiles; CTA c (one per SM) owns tiles [cT/P, (c+1)T/P) and all
//    of K, so no CTA needs another's result.
//  * K is walked in chunks of 8 units (a unit = 64 packed bytes of a row: 128 k of INT4,
//    256 k of INT2).  A producer warp issues, per chunk, two 2D TMA boxes of 16 rows x 256 B
//    per tile into an S-stage ring (256-byte rows: narrower TMA rows stream markedly slower,
//    and each TMA instruction costs tens of nanoseconds to issue).  The weight boxes of the
//    first S chunks are issued before griddepcontrol.wait, so with programmatic dependent
//    launch they stream while the previous kernel finishes; only the activations wait.
//  * The activations are staged once for all of K (one bulk copy per token row) when they
//    fit, else per chunk by TMA.  The CTA's scale / zero rows (contiguous in the [N, K/g]
//    layout) arrive with one bulk copy each and are turned into an fp32 table.
//  * Sixteen consumer warps: warp w takes unit w % 8 of every chunk and half (w / 8) of its
//    k-steps, for all of the CTA's tiles, two tiles at a time.  It builds its mma.sync B
//    fragments once per chunk and reuses them for every tile; weights are unpacked with LOP3
//    into exact integers q - z and multiplied on the tensor cores (two tiles x two k-step
//    chains in flight); each unit's fp32 / int32 sum is folded with its group scale.
//  * The warps' partial sums are added in a fixed order through shared memory
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

constexpr int kCW = 16;                    // consumer warps
constexpr int kThreads = (kCW + 1) * 32;   // + producer warp
constexpr int kKC = 8;                     // units per chunk
constexpr int kTileRows = 16;
constexpr int kUnitBytes = 64;
constexpr int kWBoxBytes = 256;                      // weight box row: 4 units
constexpr int kUPB = kWBoxBytes / kUnitBytes;        // units per weight box
constexpr int kWBox = kTileRows * kWBoxBytes;        // 4 KB
constexpr int kTileChunk = kKC * kTileRows * kUnitBytes;  // one tile's part of a chunk: 8 KB
constexpr int kABoxElems = 256;                      // activation box row: 256 elements
constexpr int kAPadBytes = 16;                       // activation row padding (bank spread)

// tiles whose sums live in registers at once (even: tiles go through the MMA in pairs)
__host__ __device__ constexpr int tg_max(int NT) { return NT == 1 ? 6 : 2; }

struct GemvParams {
    const void *A;
    int M, N, K, G, gs, sym;
    int KB, T, P, nch, TG, S;
    int a_whole;     // 1: all of K staged once; 0: per chunk by TMA
    int a_pitch_b;   // bytes between token rows of the staged activations
    int abox_bytes;  // chunked activations: bytes of one TMA box (M x 256 elements)
    int wpart_bytes, stage_bytes;
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

__device__ __forceinline__ uint2 lds64(const void *p)
{
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(smem_u32(p)));
    return v;
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
        const float as = p.a_scale[m];
        v = (WB == 2) ? as * (p.scale32[0] * float(total_i)) : as * total_f;
    } else {
        v = (WB == 2) ? p.scale32[0] * total_f : total_f;
    }
    return v + bias_at<AM>(p.bias, n);
}

// ACC: also add every INT32 group sum into p.acc_out (W4A8 debugging output; zeroed by the
// host first, the two halves of a unit arrive from two warps).
template <int WB, int AM, int NT, bool ACC>
__global__ void __launch_bounds__(kThreads, 1)
    gemv_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_a,
                const GemvParams p)
{
    constexpr int MP = NT * 8;
    constexpr int KU = kunit_of(WB);
    constexpr int QH = qh_of(WB, AM);
    constexpr int kTGMax = tg_max(NT);
    constexpr int ES = (AM == A_I8) ? 1 : 2;
    constexpr int UPA = kABoxElems / KU;  // units per activation box
    using Tot = typename std::conditional<AM == A_I8 && WB == 2, int, float>::type;

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int S = p.S;
    uint8_t *ring = smem;
    uint8_t *abuf = ring + size_t(S) * p.stage_bytes;  // whole activations (a_whole)
    const size_t abuf_bytes = p.a_whole ? ((size_t(p.M) * p.a_pitch_b + 127) & ~size_t(127)) : 0;
    float2 *stab = reinterpret_cast<float2 *>(abuf + abuf_bytes);
    uint16_t *sc = reinterpret_cast<uint16_t *>(stab + size_t(p.sc_rows_cap) * p.G);
    uint16_t *zc = sc + size_t(p.sc_rows_cap) * p.G;
    float *red = reinterpret_cast<float *>(
        (reinterpret_cast<uintptr_t>(zc + size_t(p.sc_rows_cap) * p.G) + 15) & ~uintptr_t(15));
    uint64_t *bars = reinterpret_cast<uint64_t *>(red + size_t(kCW) * p.TG * kTileRows * MP);
    uint64_t *full = bars, *empty = bars + S, *scbar = bars + 2 * S, *abar = scbar + 1, *cbar = scbar + 2;

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
        mbar_init(scbar, 1);
        mbar_init(abar, 1);
        mbar_init(cbar, kCW * 32);
        fence_barrier_init();
    }
    __syncthreads();
    grid_dep_launch();  // the next kernel in the stream may start launching as SMs free up

    if (warp == kCW) {
        // ------------------------------------------------------------ producer warp
        if (lane == 0) {
            tma_prefetch_desc(&tmap_w);
            if (!p.a_whole) tma_prefetch_desc(&tmap_a);
        }
        // scale / zero rows of this CTA: contiguous, 16-byte aligned at the start
        const uint32_t sc_bytes = (WB == 4 && p.sc_smem) ? uint32_t(r1 - r0) * p.G * 2 : 0u;
        const uint32_t sc16 = sc_bytes & ~15u;
        if constexpr (WB == 4) {
            for (uint32_t e = (sc16 >> 1) + uint32_t(lane); e < (sc_bytes >> 1); e += 32u) {  // ragged tail
                sc[e] = p.scales16[(size_t)r0 * p.G + e];
                if (!p.sym) zc[e] = p.zeros[(size_t)r0 * p.G + e];
            }
        }
        __syncwarp();
        if (lane == 0) {
            mbar_arrive_expect_tx(scbar, sc16 * (p.sym ? 1 : 2));
            if (sc16) {
                bulk_load(sc, p.scales16 + (size_t)r0 * p.G, sc16, scbar);
                if (!p.sym) bulk_load(zc, p.zeros + (size_t)r0 * p.G, sc16, scbar);
            }
        }

        auto issue = [&](int it, bool weights, bool acts) {
            const int s = it % S;
            const int grp = it / p.nch, ch = it % p.nch;
            const int ntg = min(p.TG, ntc - grp * p.TG);
            const int kb0 = ch * kKC, nkb = min(kKC, p.KB - kb0);
            const int nwb = (nkb + kUPB - 1) / kUPB, nab = p.a_whole ? 0 : (nkb + UPA - 1) / UPA;
            uint8_t *st = ring + size_t(s) * p.stage_bytes;
            if (weights) {
                if (lane == 0) mbar_arrive_expect_tx(&full[s], uint32_t(ntg * nwb * kWBox + nab * p.abox_bytes));
                __syncwarp();
                for (int idx = lane; idx < ntg * nwb; idx += 32) {
                    const int i = idx / nwb, b = idx % nwb;
                    tma_load_2d(st + i * kTileChunk + b * kWBox, &tmap_w, (kb0 + b * kUPB) * kUnitBytes,
                                (t0 + grp * p.TG + i) * kTileRows, &full[s]);
                }
            }
            if (acts)
                for (int b = lane; b < nab; b += 32)
                    tma_load_2d(st + p.wpart_bytes + b * p.abox_bytes, &tmap_a, (kb0 + b * UPA) * KU, 0, &full[s]);
        };
        const int pro = min(S, total_it);
        for (int it = 0; it < pro; ++it) issue(it, true, false);
        grid_dep_wait();  // activations may be produced by the previous kernel
        if (p.a_whole) {
            if (lane == 0) {
                // all of K, one bulk copy per token row; zeros past K up to the last unit
                const int kpad = p.KB * KU;
                for (int m = 0; m < p.M; ++m)
                    for (int k = p.K; k < kpad; ++k) {
                        if constexpr (ES == 1) abuf[(size_t)m * p.a_pitch_b + k] = 0;
                        else reinterpret_cast<uint16_t *>(abuf + (size_t)m * p.a_pitch_b)[k] = 0;
                    }
                const uint32_t bytes = uint32_t(p.K) * ES;
                mbar_arrive_expect_tx(abar, bytes * p.M);
                for (int m = 0; m < p.M; ++m)
                    bulk_load(abuf + (size_t)m * p.a_pitch_b, static_cast<const uint8_t *>(p.A) + (size_t)m * bytes,
                              bytes, abar);
            }
        } else {
            for (int it = 0; it < pro; ++it) issue(it, false, true);
        }
        int it = pro;
        for (; it < total_it; ++it) {
            if (!wait_bar(&empty[it % S], ((it / S) - 1) & 1)) break;
            issue(it, true, true);
        }
        for (int k = max(0, it - S); k < it; ++k) wait_bar(&full[k % S], (k / S) & 1);
        if (p.a_whole) wait_bar(abar, 0);
        return;
    }

    // ---------------------------------------------------------------- consumer warps
    const int g = lane >> 2, t = lane & 3;
    const int us = warp & (kKC - 1), hf = warp >> 3;  // unit slot in the chunk, k-step half
    uint32_t cphase = 0;
    auto csync = [&]() -> bool {  // bounded barrier of the consumer warps
        mbar_arrive(cbar);
        const bool ok = wait_bar(cbar, cphase & 1);
        ++cphase;
        return ok;
    };
    if (!wait_bar(scbar, 0)) return;
    if constexpr (WB == 4) {
        if (p.sc_smem) {
            const int nent = (r1 - r0) * p.G;
            for (int e = threadIdx.x; e < nent; e += kCW * 32)
                stab[e] = make_float2(__half2float(__ushort_as_half(sc[e])),
                                      p.sym ? 8.f : __half2float(__ushort_as_half(zc[e])));
        }
    }
    if (!csync()) return;
    grid_dep_wait();  // a_scale and bias may come from the previous kernel
    if (p.a_whole && !wait_bar(abar, 0)) return;

    // this lane's bytes inside a tile's 8 KB chunk part: box us/4, bytes (us%4)*64 + 16t + 8hf
    const int woff = (us / kUPB) * kWBox + (us % kUPB) * kUnitBytes + 16 * t + 8 * hf;

    for (int grp = 0; grp < ngrp; ++grp) {
        const int ntg = min(p.TG, ntc - grp * p.TG);
        Tot tot[kTGMax][NT][4];
#pragma unroll
        for (int i = 0; i < kTGMax; ++i)
#pragma unroll
            for (int j = 0; j < NT; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e) tot[i][j][e] = Tot(0);

        for (int ch = 0; ch < p.nch; ++ch) {
            const int it = grp * p.nch + ch;
            const int s = it % S;
            if (!wait_bar(&full[s], (it / S) & 1)) return;
            const uint8_t *st = ring + size_t(s) * p.stage_bytes;
            const int kb = ch * kKC + us;
            if (kb < p.KB) {
                const uint8_t *ablk = p.a_whole ? abuf + (size_t)kb * KU * ES
                                                : st + p.wpart_bytes + (us / UPA) * p.abox_bytes + (us % UPA) * KU * ES;
                const int pitch = p.a_whole ? p.a_pitch_b : kABoxElems * ES;
                uint4 bf[NT][QH];
                int asum[NT];
#pragma unroll
                for (int j = 0; j < NT; ++j) build_bfrag_half<WB, AM>(ablk, pitch, p.M, j, lane, hf, bf[j], asum[j]);
                int sA[NT][2];
                if constexpr (AM == A_I8) {
#pragma unroll
                    for (int j = 0; j < NT; ++j) {
                        int v = asum[j];
                        v += __shfl_xor_sync(0xffffffffu, v, 1);
                        v += __shfl_xor_sync(0xffffffffu, v, 2);
                        sA[j][0] = __shfl_sync(0xffffffffu, v, (2 * t) * 4);
                        sA[j][1] = __shfl_sync(0xffffffffu, v, (2 * t + 1) * 4);
                    }
                }
                const int gi = (WB == 4) ? (kb * KU) / p.gs : 0;
#pragma unroll
                for (int ip = 0; ip < kTGMax / 2; ++ip) {
                    if (2 * ip >= ntg) break;
                    uint2 wa[2], wb[2];
                    float s_lo[2], s_hi[2];
                    uint32_t zl[2], zh[2];
#pragma unroll
                    for (int l = 0; l < 2; ++l) {
                        const int i = 2 * ip + l;  // tile i >= ntg: stale data, result discarded
                        const uint8_t *wt = st + i * kTileChunk + woff;
                        wa[l] = lds64(wt + g * kWBoxBytes);
                        wb[l] = lds64(wt + (g + 8) * kWBoxBytes);
                        s_lo[l] = s_hi[l] = 0.f;
                        zl[l] = zh[l] = 8;
                        if constexpr (WB == 4) {
                            const int rl = (grp * p.TG + i) * kTileRows + g;  // row within the CTA
                            if (p.sc_smem) {
                                // rows past the CTA's end read stale table entries: never stored
                                const float2 v_lo = stab[rl * p.G + gi];
                                const float2 v_hi = stab[(rl + 8) * p.G + gi];
                                s_lo[l] = v_lo.x;
                                s_hi[l] = v_hi.x;
                                zl[l] = uint32_t(v_lo.y) & 15u;
                                zh[l] = uint32_t(v_hi.y) & 15u;
                            } else {
                                const int n_lo = r0 + rl, n_hi = n_lo + 8;
                                if (n_lo < p.N) {
                                    s_lo[l] = __half2float(__ushort_as_half(p.scales16[(size_t)n_lo * p.G + gi]));
                                    if (!p.sym) zl[l] = uint32_t(__half2float(__ushort_as_half(p.zeros[(size_t)n_lo * p.G + gi])));
                                }
                                if (n_hi < p.N) {
                                    s_hi[l] = __half2float(__ushort_as_half(p.scales16[(size_t)n_hi * p.G + gi]));
                                    if (!p.sym) zh[l] = uint32_t(__half2float(__ushort_as_half(p.zeros[(size_t)n_hi * p.G + gi])));
                                }
                            }
                        }
                    }
                    acc_t<AM> ua[2][2][NT][4];
#pragma unroll
                    for (int a = 0; a < 2; ++a)
#pragma unroll
                        for (int l = 0; l < 2; ++l)
#pragma unroll
                            for (int j = 0; j < NT; ++j)
#pragma unroll
                                for (int e = 0; e < 4; ++e) ua[a][l][j][e] = acc_t<AM>(0);
                    unit_mma_half<WB, AM, NT, 2>(wa, wb, bf, zl, zh, ua);
#pragma unroll
                    for (int l = 0; l < 2; ++l) {
                        const int i = 2 * ip + l;
#pragma unroll
                        for (int j = 0; j < NT; ++j)
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const acc_t<AM> v = ua[0][l][j][e] + ua[1][l][j][e];
                                const float sc_e = (e < 2) ? s_lo[l] : s_hi[l];
                                if constexpr (AM == A_I8 && WB == 2) {
                                    tot[i][j][e] += v - 2 * sA[j][e & 1];
                                } else if constexpr (AM == A_I8) {
                                    const int corr = v - int((e < 2) ? zl[l] : zh[l]) * sA[j][e & 1];
                                    if constexpr (ACC) {
                                        const int n = r0 + (grp * p.TG + i) * kTileRows + g + ((e & 2) ? 8 : 0);
                                        const int m = j * 8 + 2 * t + (e & 1);
                                        if (i < ntg && n < p.N && m < p.M)
                                            atomicAdd(&p.acc_out[((long long)m * p.N + n) * p.G + kb], corr);
                                    }
                                    tot[i][j][e] = fmaf(sc_e, float(corr), tot[i][j][e]);
                                } else if constexpr (WB == 2) {
                                    tot[i][j][e] += v;
                                } else {
                                    tot[i][j][e] = fmaf(sc_e, v, tot[i][j][e]);
                                }
                            }
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
        }

        // ---- add the 16 warps' partial sums (fixed order) and write C ----
#pragma unroll
        for (int i = 0; i < kTGMax; ++i) {
            if (i >= ntg) break;
#pragma unroll
            for (int j = 0; j < NT; ++j) {
                float v[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    if constexpr (AM == A_I8 && WB == 2) v[e] = __int_as_float(tot[i][j][e]);
                    else v[e] = tot[i][j][e];
                }
                const int m = j * 8 + 2 * t;
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
            store_out<AM>(p.C, (long long)m * p.N + n, finish<WB, AM>(p, sf, si, n, m));
            if constexpr (AM == A_I8 && WB == 2)
                if (p.acc_out) p.acc_out[(long long)m * p.N + n] = si;
        }
        if (grp + 1 < ngrp && !csync()) return;  // red is reused by the next group
    }
}

// ---------------------------------------------------------------- host side
struct Plan {
    int NT = 1, MP = 8, KU = 128, KB = 0, T = 0, P = 0, nch = 0, TG = 1, S = 2;
    int a_whole = 0, a_pitch_b = 0, abox = 0, wpart = 0, stage = 0, sc_smem = 0, sc_rows_cap = 0;
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
    const int es = AM == A_I8 ? 1 : 2;
    pl.sc_rows_cap = tiles_max * kTileRows;
    const size_t sc_bytes = (WB == 4) ? size_t(pl.sc_rows_cap) * G * (8 + 2 + 2) : 0;
    pl.sc_smem = (WB == 4 && sc_bytes <= 48 * 1024) ? 1 : 0;
    if (!pl.sc_smem) pl.sc_rows_cap = 0;
    const size_t sc_area = pl.sc_smem ? sc_bytes : 0;
    pl.TG = std::min(tg_max(pl.NT), tiles_max);
    const int tg_alloc = pl.TG + (pl.TG & 1);  // pairs: the odd tile's partner is read but unused
    pl.wpart = tg_alloc * kTileChunk;
    const size_t red = size_t(kCW) * pl.TG * kTileRows * pl.MP * 4;
    const size_t fixed = 1024 + sc_area + 16 + red + 8 * (2 * 8 + 3) + 16;
    const size_t budget = size_t(dev.max_smem_optin);
    const int ngrp = (tiles_max + pl.TG - 1) / pl.TG;
    const long long total = (long long)ngrp * pl.nch;
    auto stages_for = [&](size_t stage, size_t extra) -> long long {
        if (budget <= fixed + extra) return 0;
        return std::min<long long>({8, total, (long long)((budget - fixed - extra) / stage)});
    };
    // whole activations: one copy for all of K; otherwise per chunk by TMA
    const int a_pitch_whole = pl.KB * pl.KU * es + kAPadBytes;
    const size_t abuf = (size_t(M) * a_pitch_whole + 127) & ~size_t(127);
    const long long s_whole = stages_for(pl.wpart, abuf);
    const int abox = int(M) * kABoxElems * es;
    const int apart = (kKC * pl.KU / kABoxElems) * abox;
    const size_t stage_chunked = (size_t(pl.wpart + apart) + 1023) & ~size_t(1023);
    const long long s_chunked = stages_for(stage_chunked, 0);
    const long long want = std::min<long long>(4, total);
    if (s_whole >= want || (s_whole >= 1 && s_whole >= s_chunked)) {
        pl.a_whole = 1;
        pl.a_pitch_b = a_pitch_whole;
        pl.stage = pl.wpart;
        pl.S = int(s_whole);
        pl.smem = fixed + abuf + size_t(pl.S) * pl.stage;
    } else {
        pl.a_whole = 0;
        pl.a_pitch_b = kABoxElems * es;
        pl.abox = abox;
        pl.stage = int(stage_chunked);
        pl.S = int(s_chunked);
        pl.smem = fixed + size_t(pl.S) * pl.stage;
    }
    pl.ok = pl.S >= 1 && pl.smem <= budget;
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
                                  kWBoxBytes, kTileRows);
    if (rc != WQ_OK) return rc;
    const int esize = AM == A_I8 ? 1 : 2;
    ta = tw;  // unused when the activations are staged whole
    if (!pl.a_whole) {
        rc = encode_tmap_2d(&ta, AM == A_I8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_UINT16, A,
                            uint64_t(K), uint64_t(M), uint64_t(K) * esize, uint32_t(kABoxElems), uint32_t(M));
        if (rc != WQ_OK) return rc;
    }
    GemvParams p{};
    p.A = A;
    p.M = int(M);
    p.N = int(N);
    p.K = int(K);
    p.G = G;
    p.gs = WB == 4 ? c.group_size : int(K);
    p.sym = WB == 4 ? c.symmetric : 1;
    p.KB = pl.KB;
    p.T = pl.T;
    p.P = pl.P;
    p.nch = pl.nch;
    p.TG = pl.TG;
    p.S = pl.S;
    p.a_whole = pl.a_whole;
    p.a_pitch_b = pl.a_pitch_b;
    p.abox_bytes = pl.abox;
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
#define WQ_LAUNCH(wb, am) return NT == 1 ? launch<wb, am, 1>(pl, tw, ta, p, st) : launch<wb, am, 2>(pl, tw, ta, p, st)
    if (WB == 4 && AM == A_F16) WQ_LAUNCH(4, A_F16);
    if (WB == 4 && AM == A_BF16) WQ_LAUNCH(4, A_BF16);
    if (WB == 4 && acc_out) {
        // each group sum arrives in two halves from two warps: start from zero
        if (cudaMemsetAsync(acc_out, 0, size_t(M) * N * G * sizeof(int32_t), st) != cudaSuccess)
            return check_launch("cudaMemsetAsync(acc_out)");
        return NT == 1 ? launch<4, A_I8, 1, true>(pl, tw, ta, p, st) : launch<4, A_I8, 2, true>(pl, tw, ta, p, st);
    }
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
