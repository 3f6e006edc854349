// wq_gemv.cu -- decode GEMV / few-token matmul (M <= 16) over packed INT4 / INT2 / INT1 /
// FP4 / FP8 weights.
//
// C[M,N] = A[M,K] x dequant(Wq[N,K])^T ("BitBLAS practical guide", "What is BitBLAS",
// layout "nt"), FP16 / BF16 activations (W4A16) or per-token INT8 activations with exact
// INT32 group sums and the (a_scale x w_scale) epilogue (W4A8: "Accelerating LLM inference
// with CUDA Graph and INT4 quantization", part 1, steps 3-4).
//
// The kernel is HBM-bound and lasts a few microseconds, so it is built to put each SM's
// whole share of the packed weights in flight at once and to spend few instructions per
// byte once it arrives:
//  * Rows are cut into 16-row tiles; CTA c (one per SM) owns a contiguous run of tiles and all
//    of K, so no CTA needs another's result.  K is walked in chunks of KC units (a unit =
//    64 packed bytes of a row: 128 k of INT4 or FP4, 256 k of INT2, 512 k of INT1, 64 k of
//    FP8).
//  * One TMA box per tile and chunk brings 16 rows x KC units (a 3D box over unit pairs;
//    a 2D box per unit pair when rows are not a whole number of pairs), written with the
//    128-byte swizzle; MMA row g reads tile row (g >> 1) | ((g & 1) << 2), so the two rows of
//    a quarter-warp fall in opposite bank halves and a 16-byte load per lane is conflict-free.
//    Thread 0 sends the first chunk's boxes right after setting up the barriers, the other
//    warps the next S - 1, all before griddepcontrol.wait: with programmatic dependent launch
//    they stream while the previous kernel in the stream finishes.  When all chunks fit in
//    shared memory nothing else is issued; otherwise the last warp to finish a stage
//    refills it.
//  * The activations are staged once for all of K (one bulk copy per token row) when they
//    fit, else per chunk by a swizzled 3D TMA box.  The CTA's scales / zero points become a
//    group-major fp32 table.
//  * 16 warps; warp w takes unit w % KC of every chunk and, for 9..16 tokens with more than
//    two tiles per CTA, every other tile.  It builds the unit's mma.sync B fragments (activations in the k order of the
//    nibble unpack) once and uses them for all its tiles: weights are unpacked with LOP3
//    into the exact integers q - z, multiplied on the tensor cores, and each unit's fp32 /
//    int32 sum is folded with its group scale.
//  * The warps' partial sums are added in a fixed order through shared memory
//    (deterministic) and the epilogue writes C.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include <algorithm>
#include <cstring>
#include <type_traits>

#include "wq_device.cuh"
#include "wq_host.h"
#include "wq_unit.cuh"

namespace wq {

static __device__ int g_gemv_error;

namespace {

constexpr int kCW = 16;  // warps
constexpr int kThreads = kCW * 32;
constexpr int kTileRows = 16;
constexpr int kPairBytes = 128;                   // two units of a row: one swizzle line
constexpr int kPairBox = kTileRows * kPairBytes;  // 2 KB
// Work split by token tiles NT.  `wide` (9..16 tokens, at most two row tiles per CTA): one
// warp per unit takes both tiles, so each unit's B fragments are built once, not per warp half.
__host__ __device__ constexpr int wpu_of(int NT, bool wide = false) { return (NT == 1 || wide) ? 1 : 2; }  // warps sharing a unit
__host__ __device__ constexpr int kc_of(int NT, bool wide = false) { return kCW / wpu_of(NT, wide); }  // units per chunk
__host__ __device__ constexpr int tm_of(int NT, bool wide = false) { return NT == 1 ? 6 : (wide ? 2 : 3); }  // tiles per warp and pass
__host__ __device__ constexpr int ntl_of(int NT, bool wide = false) { return (NT == 1 || wide) ? 2 : 1; }  // tiles per MMA batch

struct GemvParams {
    const void *A;
    int M, N, K, G, gs, sym;
    int upg;                 // units per scale group (INT4: group_size / 128)
    int KB, T, P;
    int nch, TPP, S;         // chunks per pass, tiles per pass, ring stages
    int w3d;                 // 1: one 3D box per tile and chunk; 0: one 2D box per unit pair
    int wtile_bytes;         // one tile's weights of a chunk: KC x 1 KB
    int wpart_bytes;         // TPP tiles
    int stage_bytes;         // weights + chunked activations
    int a_whole, a_pitch_b;  // whole activations: bytes between token rows
    int abox_bytes, MB;      // chunked activations: bytes per stage, token rows of the box
    int rows_cap;            // CTA rows covered by the scale table
    int tab_rs;              // table row stride (float2 entries, odd: spreads the banks)
    int abuf_off, scst_off, stab_off, red_off, bar_off;
    const uint16_t *scales16;
    const float *scale32;
    const uint16_t *zeros;
    const void *bias;
    const float *a_scale;
    void *C;
    int32_t *acc_out;
    // fused per-token INT8 quantization of FP activations (FS != 0): source, outputs and
    // the shared-memory offset of the tokens' scales and their reciprocals
    const void *A_src;
    int8_t *Aq_out;
    float *a_scale_out;
    int fs_off;
    int nat;  // INT4 weights in the kernel-native order
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
    if (mbar_test_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    for (;;) {
        for (int i = 0; i < 4; ++i)
            if (mbar_try_wait_short(bar, parity)) return true;
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

template <int WF, int AM>
__device__ __forceinline__ float finish(const GemvParams &p, float total_f, int total_i, int n, float as)
{
    float v;
    if constexpr (AM == A_I8) {
        v = wf_per_tensor(WF) ? as * (p.scale32[0] * float(total_i)) : as * total_f;
    } else if constexpr (AM == A_F8) {
        v = as * total_f;  // the token's FP8 scale times the group-scaled sums
    } else {
        v = wf_per_tensor(WF) ? p.scale32[0] * total_f : total_f;
    }
    return v + bias_at<AM>(p.bias, n);
}

template <int FS>
__device__ __forceinline__ float src_at(const uint4 &raw, int i)
{
    const uint16_t h = reinterpret_cast<const uint16_t *>(&raw)[i];
    if constexpr (FS == 2) return __bfloat162float(__ushort_as_bfloat16(h));
    return __half2float(__ushort_as_half(h));
}

// ACC: also store every INT32 group sum into p.acc_out (W4A8 with group_size 128).
// FS: 0, or the FP activations to quantize per token first (1: binary16, 2: bfloat16; INT8 or
// FP8 mode and whole-K activation staging only): the "fused kernel" of the same page's section
// on combining the strategies, here the quantization done in the matmul's prologue.
template <int WF, int AM, int NT, bool ACC, bool WIDE, int FS = 0>
__global__ void __launch_bounds__(kThreads, 1)
    gemv_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_a,
                const GemvParams p)
{
    static_assert(FS == 0 || byte_acts(AM), "the fused quantization feeds the INT8 / FP8 paths");
    constexpr int KU = kunit_of(WF);
    constexpr int QN = qn_of(WF, AM);
    constexpr bool GROUPED = wf_grouped(WF);
    constexpr int ES = byte_acts(AM) ? 1 : 2;
    constexpr int AU = KU * ES;  // activation bytes of one unit and token
    constexpr int WPU = wpu_of(NT, WIDE), KC = kc_of(NT, WIDE), TM = tm_of(NT, WIDE), NTL = ntl_of(NT, WIDE);
    using Tot = typename std::conditional<AM == A_I8 && wf_per_tensor(WF), int, float>::type;

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int S = p.S;
    uint8_t *ring = smem;
    uint8_t *abuf = smem + p.abuf_off;
    uint16_t *sc_st = reinterpret_cast<uint16_t *>(smem + p.scst_off);  // [rows][G] fp16 scales
    uint16_t *zc_st = sc_st + size_t(p.rows_cap) * p.G;                 // then zero points
    float2 *stab = reinterpret_cast<float2 *>(smem + p.stab_off);       // [G][tab_rs] {scale, zero}
    float *red = reinterpret_cast<float *>(smem + p.red_off);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + p.bar_off);
    uint64_t *abar = full + S, *cbar = full + S + 1, *scbar = full + S + 2;
    unsigned *cnt = reinterpret_cast<unsigned *>(full + S + 3);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = blockIdx.x;
    // tiles T = base * P + R: the first R CTAs take one more.  CTAs start in index order as the
    // previous kernel's CTAs leave their SMs, so the late ones get the smaller share.
    const int base = p.T / p.P, rem = p.T - base * p.P;
    const int t0 = c * base + min(c, rem), t1 = t0 + base + (c < rem ? 1 : 0);
    const int ntc = t1 - t0;
    const int npass = (ntc + p.TPP - 1) / p.TPP;
    const int total_it = npass * p.nch;
    const int r0 = t0 * kTileRows;

    // ---- stage `it` of the ring: weights of the pass's tiles (and the expected bytes of all)
    auto issue_w = [&](int it) {
        const int s = it % S;
        const int pass = it / p.nch, ch = it % p.nch;
        const int tp0 = t0 + pass * p.TPP;
        const int ntp = min(p.TPP, ntc - pass * p.TPP);
        const int pair0 = ch * KC / 2;
        const int npair = min(KC / 2, (p.KB + 1) / 2 - pair0);
        uint8_t *st = ring + size_t(s) * p.stage_bytes;
        const uint32_t wbytes = p.w3d ? uint32_t(ntp * p.wtile_bytes) : uint32_t(ntp * npair * kPairBox);
        mbar_arrive_expect_tx(&full[s], wbytes + (p.a_whole ? 0u : uint32_t(p.abox_bytes)));
        for (int i = 0; i < ntp; ++i) {
            uint8_t *dst = st + size_t(i) * p.wtile_bytes;
            if (p.w3d) {
                tma_load_3d(dst, &tmap_w, 0, (tp0 + i) * kTileRows, pair0, &full[s]);
            } else {
                for (int q = 0; q < npair; ++q)
                    tma_load_2d(dst + q * kPairBox, &tmap_w, (pair0 + q) * kPairBytes, (tp0 + i) * kTileRows,
                                &full[s]);
            }
        }
    };
    auto issue_a = [&](int it) {  // chunked activations (after the grid dependency)
        const int s = it % S, ch = it % p.nch;
        tma_load_3d(ring + size_t(s) * p.stage_bytes + p.wpart_bytes, &tmap_a, 0, 0, ch * KC * AU / 128, &full[s]);
    };

    // the CTA's scale / zero rows are contiguous in [N, G]: one bulk copy each (a ragged
    // tail of < 16 bytes is read directly below)
    const int nrows = min(ntc * kTileRows, p.N - r0);
    const uint32_t sc_bytes = GROUPED ? uint32_t(nrows) * p.G * 2u : 0u;
    const uint32_t sc16 = sc_bytes & ~15u;
    const int pro = min(S, total_it);
    // Thread 0 sets up the barriers and at once sends the first stage's weights, which are on
    // the critical path, then the scales; the other stages follow after the block barrier.
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            cnt[s] = 0;
        }
        mbar_init(abar, 1);
        mbar_init(cbar, kCW);
        mbar_init(scbar, 1);
        fence_barrier_init();
        tma_prefetch_desc(&tmap_w);
        if (!p.a_whole) tma_prefetch_desc(&tmap_a);
        issue_w(0);
        if constexpr (GROUPED) {
            mbar_arrive_expect_tx(scbar, sc16 * (p.sym ? 1u : 2u));
            if (sc16) {
                bulk_load(sc_st, p.scales16 + (size_t)r0 * p.G, sc16, scbar);
                if (!p.sym) bulk_load(zc_st, p.zeros + (size_t)r0 * p.G, sc16, scbar);
            }
        }
    }
    __syncthreads();
    grid_dep_launch();  // the next kernel in the stream may start launching as SMs free up
    if (lane == 0)
        for (int it = warp; it < pro; it += kCW)
            if (it > 0) issue_w(it);

    // ---- scale / zero table of the CTA's rows, group-major: {scale, zero point as integer bits}
    if constexpr (GROUPED) {
        wait_bar(scbar, 0);  // on expiry the error is recorded; carry on to the next barrier
        const int nsm = int(sc16 >> 1);
        const int nrow_t = ntc * kTileRows;  // a warp per row, its lanes over the groups
        for (int rl = warp; rl < nrow_t; rl += kCW) {
            for (int gi = lane; gi < p.G; gi += 32) {
                const int e = rl * p.G + gi;
                float sv = 0.f;
                uint32_t zv = 8;
                if (rl < nrows) {
                    const uint16_t sb = e < nsm ? sc_st[e] : p.scales16[(size_t)r0 * p.G + e];
                    sv = __half2float(__ushort_as_half(sb));
                    if (!p.sym) {
                        const uint16_t zb = e < nsm ? zc_st[e] : p.zeros[(size_t)r0 * p.G + e];
                        zv = uint32_t(__half2float(__ushort_as_half(zb))) & 15u;
                    }
                }
                stab[(size_t)gi * p.tab_rs + rl] = make_float2(sv, __uint_as_float(zv));
            }
        }
    }

    grid_dep_wait();  // activations, a_scale and bias may be written by the previous kernel
    float *fsc = reinterpret_cast<float *>(smem + p.fs_off);  // FS: [16] token scales, [16] their reciprocals
    if constexpr (FS != 0) {
        // per-token absolute maximum (a warp per token), then the codes of all of A into the
        // activation buffer; each 8-element chunk of Aq is also written out by one CTA
        if (threadIdx.x == 0) {
            const int kpad = p.KB * KU;
            for (int m = 0; m < p.M; ++m)
                for (int k = p.K; k < kpad; ++k) abuf[(size_t)m * p.a_pitch_b + k] = 0;
        }
        const int K8 = p.K / 8;
        const uint4 *src = static_cast<const uint4 *>(p.A_src);
        for (int m = warp; m < p.M; m += kCW) {
            float amax = 0.f;
            for (int j = lane; j < K8; j += 32) {
                const uint4 raw = __ldg(src + (size_t)m * K8 + j);
#pragma unroll
                for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(src_at<FS>(raw, i)));
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
            if (lane == 0) {
                const float sc = __fdiv_rn(amax, AM == A_F8 ? 448.0f : 127.0f);
                fsc[m] = sc;
                fsc[16 + m] = sc != 0.f ? __frcp_rn(sc) : 0.f;
                if (blockIdx.x == 0) p.a_scale_out[m] = sc;
            }
        }
        __syncthreads();
        for (int e = threadIdx.x; e < p.M * K8; e += kThreads) {
            const int m = e / K8, j = e - m * K8;
            const uint4 raw = __ldg(src + (size_t)m * K8 + j);
            const float sc = fsc[m], rc = fsc[16 + m];
            uint32_t w[2] = {0u, 0u};
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                uint32_t code;
                if constexpr (AM == A_F8)  // the e4m3 code of clip(a / scale, -448, 448), as act_quant_fp8
                    code = sc != 0.f ? minifloat_code<WQ_FMT_E4M3>(fminf(fmaxf(__fdiv_rn(src_at<FS>(raw, i), sc), -448.f), 448.f)) : 0u;
                else
                    code = uint32_t(quant_i8(src_at<FS>(raw, i), sc, rc)) & 0xffu;
                w[i >> 2] |= code << (8 * (i & 3));
            }
            *reinterpret_cast<uint2 *>(abuf + (size_t)m * p.a_pitch_b + 8 * j) = make_uint2(w[0], w[1]);
            if (int(e % gridDim.x) == blockIdx.x)
                reinterpret_cast<uint2 *>(p.Aq_out + (size_t)m * p.K)[j] = make_uint2(w[0], w[1]);
        }
    }
    if (lane == 0 && !p.a_whole)
        for (int it = warp; it < pro; it += kCW) issue_a(it);
    if (FS == 0 && p.a_whole && threadIdx.x == 0) {
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
            bulk_load(abuf + (size_t)m * p.a_pitch_b, static_cast<const uint8_t *>(p.A) + (size_t)m * bytes, bytes,
                      abar);
    }
    __syncthreads();  // table (and activation padding) visible; no early exit before this point
    if (FS == 0 && p.a_whole && !wait_bar(abar, 0)) return;

    uint32_t cphase = 0;
    auto csync = [&]() -> bool {  // bounded barrier of all threads (one arrival per warp)
        __syncwarp();
        if (lane == 0) mbar_arrive(cbar);
        const bool ok = wait_bar(cbar, cphase & 1);
        ++cphase;
        return ok;
    };

    const int g = lane >> 2, t = lane & 3;
    // MMA row g holds tile row gr (and g + 8 row gr + 8).  The lanes of a quarter-warp (g = 2q,
    // 2q + 1) then read rows q and q + 4, whose 128-byte swizzle phases put their 64 bytes in
    // opposite halves of the banks: one 128-bit load is 4 shared-memory wavefronts, not 8.
    const int gr = (g >> 1) | ((g & 1) << 2);
    const int us = warp % KC, hf = warp / KC;
    // this lane's 16 bytes of rows gr and gr+8 of a tile, unit slot us ([pair][16 rows][128 B], swizzled)
    const uint32_t lin_lo = uint32_t(((us >> 1) * kTileRows + gr) * kPairBytes + (us & 1) * 64 + 16 * t);
    const uint32_t off_lo = swz128(lin_lo), off_hi = swz128(lin_lo + 8 * kPairBytes);

    int it = 0;
    for (int pass = 0; pass < npass; ++pass) {
        const int ntp = min(p.TPP, ntc - pass * p.TPP);
        const int nmine = max(0, (ntp - hf + WPU - 1) / WPU);  // tiles hf, hf + WPU, ...
        Tot tot[TM][NT][4];
#pragma unroll
        for (int i = 0; i < TM; ++i)
#pragma unroll
            for (int j = 0; j < NT; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e) tot[i][j][e] = Tot(0);

        for (int ch = 0; ch < p.nch; ++ch, ++it) {
            const int s = it % S;
            if (!wait_bar(&full[s], (it / S) & 1)) return;
            const uint8_t *st = ring + size_t(s) * p.stage_bytes;
            const int kb = ch * KC + us;
            if (kb < p.KB && nmine > 0) {
                uint4 bf[NT][QN];
                int asum[NT];
                if constexpr (WF == WF_I1) {
                    // fragments are formed per word inside unit_mma_b1
                } else if (p.a_whole) {
                    const uint8_t *ablk = abuf + (size_t)kb * AU;
                    const int pitch = p.a_pitch_b;
                    auto addr = [=](int m, int o) { return ablk + m * pitch + o; };
#pragma unroll
                    for (int j = 0; j < NT; ++j) build_bfrag<WF, AM>(addr, p.M, j, lane, bf[j], asum[j], p.nat != 0);
                } else {
                    const uint8_t *abase = st + p.wpart_bytes;
                    const int MB = p.MB;
                    auto addr = [=](int m, int o) {
                        const uint32_t x = uint32_t(us * AU + o);
                        return abase + swz128(((x >> 7) * MB + m) * 128u + (x & 127u));
                    };
#pragma unroll
                    for (int j = 0; j < NT; ++j) build_bfrag<WF, AM>(addr, p.M, j, lane, bf[j], asum[j], p.nat != 0);
                }
                int sA[NT][2];
                if constexpr (AM == A_I8 && WF != WF_I1) {
#pragma unroll
                    for (int j = 0; j < NT; ++j) {
                        int v = asum[j];
                        v += __shfl_xor_sync(0xffffffffu, v, 1);
                        v += __shfl_xor_sync(0xffffffffu, v, 2);
                        sA[j][0] = __shfl_sync(0xffffffffu, v, (2 * t) * 4);
                        sA[j][1] = __shfl_sync(0xffffffffu, v, (2 * t + 1) * 4);
                    }
                }
                const int gi = GROUPED ? (p.upg == 1 ? kb : kb / p.upg) : 0;
                const float2 *srow = stab + (size_t)gi * p.tab_rs + pass * p.TPP * kTileRows + gr;
                // a batch of B tiles (jp .. jp + B - 1); an odd last tile runs alone
                auto batch = [&](int jp, auto nb) {
                    constexpr int B = decltype(nb)::value;
                    uint4 wa[B], wb[B];
                    float s_lo[B], s_hi[B];
                    uint32_t zl[B], zh[B];
#pragma unroll
                    for (int l = 0; l < B; ++l) {
                        const int i = hf + WPU * (jp + l);
                        const uint8_t *wt = st + i * p.wtile_bytes;
                        wa[l] = lds128(wt + off_lo);
                        wb[l] = lds128(wt + off_hi);
                        s_lo[l] = s_hi[l] = 0.f;
                        zl[l] = zh[l] = 8;
                        if constexpr (GROUPED) {
                            const uint2 v_lo = lds64(srow + i * kTileRows);
                            const uint2 v_hi = lds64(srow + i * kTileRows + 8);
                            s_lo[l] = __uint_as_float(v_lo.x);
                            s_hi[l] = __uint_as_float(v_hi.x);
                            zl[l] = v_lo.y;
                            zh[l] = v_hi.y;
                        }
                    }
                    acc_t<AM> ua[2][B][NT][4];
#pragma unroll
                    for (int a = 0; a < 2; ++a)
#pragma unroll
                        for (int l = 0; l < B; ++l)
#pragma unroll
                            for (int j = 0; j < NT; ++j)
#pragma unroll
                                for (int e = 0; e < 4; ++e) ua[a][l][j][e] = acc_t<AM>(0);
                    if constexpr (WF == WF_I1) {
                        const bool whole = p.a_whole != 0;
                        const uint8_t *ablk = abuf + (size_t)kb * AU;
                        const uint8_t *abase = st + p.wpart_bytes;
                        const int pitch = p.a_pitch_b, MB = p.MB;
                        auto addr = [=](int m, int o) -> const uint8_t * {
                            if (whole) return ablk + m * pitch + o;
                            const uint32_t x = uint32_t(us * AU + o);
                            return abase + swz128(((x >> 7) * MB + m) * 128u + (x & 127u));
                        };
                        unit_mma_b1<AM, NT, B>(wa, wb, addr, p.M, lane, ua);
                    } else {
                        unit_mma<WF, AM, NT, B>(wa, wb, bf, zl, zh, ua);
                    }
#pragma unroll
                    for (int l = 0; l < B; ++l) {
                        const int i = hf + WPU * (jp + l);
#pragma unroll
                        for (int j = 0; j < NT; ++j)
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const acc_t<AM> v = ua[0][l][j][e] + ua[1][l][j][e];
                                const float sc_e = (e < 2) ? s_lo[l] : s_hi[l];
                                if constexpr (AM == A_I8 && WF == WF_I1) {
                                    tot[jp + l][j][e] += v;  // signed +-1 weights: no correction
                                } else if constexpr (AM == A_I8 && WF == WF_I2) {
                                    tot[jp + l][j][e] += v - 2 * sA[j][e & 1];
                                } else if constexpr (AM == A_I8) {
                                    const int corr = v - int((e < 2) ? zl[l] : zh[l]) * sA[j][e & 1];
                                    if constexpr (ACC) {
                                        const int n = r0 + (pass * p.TPP + i) * kTileRows + gr + ((e & 2) ? 8 : 0);
                                        const int m = j * 8 + 2 * t + (e & 1);
                                        if (n < p.N && m < p.M) p.acc_out[((long long)m * p.N + n) * p.G + kb] = corr;
                                    }
                                    tot[jp + l][j][e] = fmaf(sc_e, float(corr), tot[jp + l][j][e]);
                                } else if constexpr (wf_per_tensor(WF)) {
                                    tot[jp + l][j][e] += v;
                                } else {
                                    tot[jp + l][j][e] = fmaf(sc_e, v, tot[jp + l][j][e]);
                                }
                            }
                    }
                };
#pragma unroll
                for (int jp = 0; jp < TM; jp += NTL) {
                    if (jp >= nmine) break;
                    if (NTL == 1 || jp + NTL <= nmine) batch(jp, std::integral_constant<int, NTL>{});
                    else batch(jp, std::integral_constant<int, 1>{});
                }
            }
            // stage consumed: the last of the 16 warps refills it with chunk it + S
            __syncwarp();
            if (lane == 0) {
                __threadfence_block();
                if ((atomicAdd(&cnt[s], 1u) + 1u) % kCW == 0u) {
                    __threadfence_block();
                    fence_proxy_async();
                    if (it + S < total_it) {
                        issue_w(it + S);
                        if (!p.a_whole) issue_a(it + S);
                    }
                }
            }
        }

        // ---- the pass's partial sums: red[tile][unit slot][row][token], then a fixed-order sum
        if (!csync()) return;  // every warp is past the pass's last chunk
#pragma unroll
        for (int jj = 0; jj < TM; ++jj) {
            if (jj >= nmine) break;
            const int i = hf + WPU * jj;
#pragma unroll
            for (int j = 0; j < NT; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int m = j * 8 + 2 * t + (e & 1);
                    const int r = gr + ((e & 2) ? 8 : 0);
                    if (m < p.M) {
                        float v;
                        if constexpr (AM == A_I8 && wf_per_tensor(WF)) v = __int_as_float(tot[jj][j][e]);
                        else v = tot[jj][j][e];
                        red[((size_t)(m * p.TPP + i) * KC + us) * kTileRows + r] = v;
                    }
                }
        }
        if (!csync()) return;
        const int rows = ntp * kTileRows;
        for (int e = threadIdx.x; e < rows * p.M; e += kThreads) {
            const int m = e / rows, rr = e - m * rows;
            const int i = rr / kTileRows, r = rr % kTileRows;
            const int n = r0 + (pass * p.TPP + i) * kTileRows + r;
            if (n >= p.N) continue;
            float sf = 0.f;
            int si = 0;
#pragma unroll
            for (int u = 0; u < KC; ++u) {
                const float v = red[((size_t)(m * p.TPP + i) * KC + u) * kTileRows + r];
                sf += v;
                si += __float_as_int(v);
            }
            const float as = !byte_acts(AM) ? 1.f : (FS != 0 ? fsc[m] : p.a_scale[m]);
            store_out<AM>(p.C, (long long)m * p.N + n, finish<WF, AM>(p, sf, si, n, as));
            if constexpr (AM == A_I8 && wf_per_tensor(WF))
                if (p.acc_out) p.acc_out[(long long)m * p.N + n] = si;
        }
        if (pass + 1 < npass && !csync()) return;  // red is reused by the next pass
    }
}

// ---------------------------------------------------------------- host side
struct Plan {
    int NT = 1, wide = 0, KC = 16, KU = 128, KB = 0, T = 0, P = 0, nch = 0, TPP = 1, S = 1;
    int w3d = 0, wtile = 0, wpart = 0, stage = 0;
    int a_whole = 0, a_pitch_b = 0, abox = 0, MB = 8, rows_cap = 0, tab_rs = 1;
    int abuf_off = 0, scst_off = 0, stab_off = 0, red_off = 0, fs_off = 0, bar_off = 0;
    size_t smem = 0;
    bool ok = false;
};

size_t up(size_t v, size_t a) { return (v + a - 1) / a * a; }

Plan make_plan(int64_t M, int64_t N, int64_t K, int WF, int AM, int G, const DeviceInfo &dev)
{
    Plan pl;
    pl.NT = M <= 8 ? 1 : 2;
    if (WF == WF_I2 && AM != A_I8 && pl.NT == 2) return pl;  // B fragments would not fit in registers
    pl.KU = kunit_of(WF);
    pl.KB = int((K + pl.KU - 1) / pl.KU);
    pl.T = int((N + kTileRows - 1) / kTileRows);
    pl.P = std::min(dev.sm_count, pl.T);
    const int ntc_max = (pl.T + pl.P - 1) / pl.P;
    pl.wide = (WF == WF_I4 && pl.NT == 2 && !byte_acts(AM) && ntc_max <= 2) ? 1 : 0;
    pl.KC = kc_of(pl.NT, pl.wide);
    pl.TPP = std::min(ntc_max, tm_of(pl.NT, pl.wide) * wpu_of(pl.NT, pl.wide));
    const int npass = (ntc_max + pl.TPP - 1) / pl.TPP;
    pl.nch = (pl.KB + pl.KC - 1) / pl.KC;
    const long long total = (long long)npass * pl.nch;
    const int es = byte_acts(AM) ? 1 : 2;
    const int au = pl.KU * es;
    const int64_t row_bytes = K * wf_bits(WF) / 8;
    pl.w3d = (row_bytes % kPairBytes) == 0 ? 1 : 0;
    pl.wtile = pl.KC * kTileRows * 64;
    pl.wpart = pl.TPP * pl.wtile;
    pl.rows_cap = ntc_max * kTileRows;
    pl.tab_rs = pl.rows_cap | 1;
    const size_t scst = wf_grouped(WF) ? up(size_t(pl.rows_cap) * G * 2 * 2, 16) : 0;
    const size_t table = wf_grouped(WF) ? up(size_t(pl.tab_rs) * G * 8, 16) : 0;
    const size_t red = up(size_t(pl.TPP) * pl.KC * kTileRows * M * 4, 16);
    const size_t tail = scst + table + red + 128 + 8 * 19 + 4 * 16 + 64;  // + fused scales, barriers (S <= 16), counters
    const size_t budget = size_t(dev.max_smem_optin) - 1024;  // 1 KB for the alignment of the base
    auto stages_for = [&](size_t stage, size_t extra) -> long long {
        if (budget <= tail + extra) return 0;
        return std::min<long long>({16, total, (long long)((budget - tail - extra) / stage)});
    };
    const int a_pitch_whole = pl.KB * au + 16;  // padded rows spread the token rows over the banks
    const size_t abuf = up(size_t(M) * a_pitch_whole, 128);
    const long long s_whole = stages_for(pl.wpart, abuf);
    pl.MB = int(up(size_t(M), 8));
    const int abox = pl.MB * pl.KC * au;
    const bool chunk_ok = (K * es) % 128 == 0;
    const long long s_chunked = chunk_ok ? stages_for(size_t(pl.wpart) + abox, 0) : 0;
    const long long want = std::min<long long>(2, total);
    if (s_whole >= want || (s_whole >= 1 && s_whole >= s_chunked)) {
        pl.a_whole = 1;
        pl.a_pitch_b = a_pitch_whole;
        pl.stage = pl.wpart;
        pl.S = int(s_whole);
    } else if (s_chunked >= 1) {
        pl.a_whole = 0;
        pl.abox = abox;
        pl.stage = pl.wpart + abox;
        pl.S = int(s_chunked);
    } else {
        return pl;
    }
    size_t off = size_t(pl.S) * pl.stage;
    pl.abuf_off = int(off);
    off += pl.a_whole ? abuf : 0;
    pl.scst_off = int(off);
    off += scst;
    pl.stab_off = int(off);
    off += table;
    pl.red_off = int(off);
    off += red;
    pl.fs_off = int(up(off, 16));  // fused quantization: 16 token scales and their reciprocals
    off = pl.fs_off + 128;
    pl.bar_off = int(up(off, 8));
    off = pl.bar_off + size_t(8) * (pl.S + 3) + size_t(4) * pl.S;
    pl.smem = up(off, 16) + 1024;
    pl.ok = pl.smem <= size_t(dev.max_smem_optin);
    return pl;
}

// The kernel instance for the plan, with its dynamic shared memory limit raised as needed.
template <int WF, int AM, int NT, bool ACC = false, bool WIDE = false, int FS = 0>
wq_status kernel_for(const Plan &pl, const void **func)
{
    auto kern = gemv_kernel<WF, AM, NT, ACC, WIDE, FS>;
    static size_t configured = 0;
    if (pl.smem > configured) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(pl.smem)) != cudaSuccess)
            return check_launch("cudaFuncSetAttribute(gemv)");
        configured = pl.smem;
    }
    *func = reinterpret_cast<const void *>(kern);
    return WQ_OK;
}

}  // namespace

// Few-token path (1 <= M <= 16) as a prepared launch.  WQ_ERR_UNSUPPORTED if no plan fits.
wq_status gemv_prepare(int WF, int AM, const void *A, const float *a_scale, const uint8_t *Wq, const void *scales,
                       const void *zeros, const void *bias, void *C, int32_t *acc_out, int64_t M, int64_t N,
                       int64_t K, const wq_qconfig &c, PreparedLaunch *out, const FusedActQuant *fa)
{
    const DeviceInfo &dev = device_info();
    const int G = wf_grouped(WF) ? int(K / c.group_size) : 1;
    Plan pl = make_plan(M, N, K, WF, AM, G, dev);
    if (!pl.ok) return fail(WQ_ERR_UNSUPPORTED, "no few-token plan for M=%lld K=%lld", (long long)M, (long long)K);
    if (fa && (!byte_acts(AM) || !pl.a_whole))
        return fail(WQ_ERR_UNSUPPORTED, "the activations of M=%lld K=%lld are not staged whole", (long long)M,
                    (long long)K);
    CUtensorMap tw, ta;
    const uint64_t row_bytes = uint64_t(K) * wf_bits(WF) / 8;
    wq_status rc = WQ_ERR_UNSUPPORTED;
    if (pl.w3d) {
        // (128-byte unit pair, row, pair): one box = 16 rows x KC units
        const uint64_t dims[3] = {uint64_t(kPairBytes), uint64_t(N), row_bytes / kPairBytes};
        const uint64_t strides[2] = {row_bytes, uint64_t(kPairBytes)};
        const uint32_t box[3] = {uint32_t(kPairBytes), uint32_t(kTileRows), uint32_t(pl.KC / 2)};
        rc = encode_tmap(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, Wq, dims, strides, box, 128);
        if (rc != WQ_OK) pl.w3d = 0;  // same shared-memory layout from one 2D box per unit pair
    }
    if (!pl.w3d) {
        const uint64_t dims[2] = {row_bytes, uint64_t(N)};
        const uint64_t strides[1] = {row_bytes};
        const uint32_t box[2] = {uint32_t(kPairBytes), uint32_t(kTileRows)};
        rc = encode_tmap(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, Wq, dims, strides, box, 128);
    }
    if (rc != WQ_OK) return rc;
    const int es = byte_acts(AM) ? 1 : 2;
    ta = tw;  // unused when the activations are staged whole
    if (!pl.a_whole) {
        // (128 bytes, token, 128-byte block of K): one box = MB tokens x KC units
        const uint64_t kbytes = uint64_t(K) * es;
        const uint64_t dims[3] = {uint64_t(128 / es), uint64_t(M), kbytes / 128};
        const uint64_t strides[2] = {kbytes, 128};
        const uint32_t box[3] = {uint32_t(128 / es), uint32_t(pl.MB), uint32_t(pl.KC * pl.KU * es / 128)};
        rc = encode_tmap(&ta, es == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_UINT16, 3, A, dims,
                         strides, box, 128);
        if (rc != WQ_OK) return fail(WQ_ERR_UNSUPPORTED, "few-token plan: activation tensor map (%s)", wq_last_error());
    }
    GemvParams p{};
    p.A = A;
    p.M = int(M);
    p.N = int(N);
    p.K = int(K);
    p.G = G;
    p.gs = wf_grouped(WF) ? c.group_size : int(K);
    p.upg = wf_grouped(WF) ? c.group_size / kunit_of(WF) : 1;
    p.sym = WF == WF_I4 ? c.symmetric : 1;
    p.KB = pl.KB;
    p.T = pl.T;
    p.P = pl.P;
    p.nch = pl.nch;
    p.TPP = pl.TPP;
    p.S = pl.S;
    p.w3d = pl.w3d;
    p.wtile_bytes = pl.wtile;
    p.wpart_bytes = pl.wpart;
    p.stage_bytes = pl.stage;
    p.a_whole = pl.a_whole;
    p.a_pitch_b = pl.a_pitch_b;
    p.abox_bytes = pl.abox;
    p.MB = pl.MB;
    p.rows_cap = pl.rows_cap;
    p.tab_rs = pl.tab_rs;
    p.abuf_off = pl.abuf_off;
    p.scst_off = pl.scst_off;
    p.stab_off = pl.stab_off;
    p.red_off = pl.red_off;
    p.bar_off = pl.bar_off;
    p.scales16 = static_cast<const uint16_t *>(scales);
    p.scale32 = static_cast<const float *>(scales);
    p.zeros = static_cast<const uint16_t *>(zeros);
    p.bias = bias;
    p.a_scale = a_scale;
    p.C = C;
    p.acc_out = acc_out;
    p.fs_off = pl.fs_off;
    p.nat = WF == WF_I4 && c.layout == WQ_LAYOUT_NATIVE;
    const bool one = pl.NT == 1;
    const void *func = nullptr;
    if (fa) {
        p.A_src = fa->A;
        p.Aq_out = fa->Aq;
        p.a_scale_out = fa->a_scale;
        const bool bf = fa->bf16;
        if (WF == WF_E4M3)
            rc = bf ? (one ? kernel_for<WF_E4M3, A_F8, 1, false, false, 2>(pl, &func) : kernel_for<WF_E4M3, A_F8, 2, false, false, 2>(pl, &func))
                    : (one ? kernel_for<WF_E4M3, A_F8, 1, false, false, 1>(pl, &func) : kernel_for<WF_E4M3, A_F8, 2, false, false, 1>(pl, &func));
        else if (WF == WF_I1)
            rc = bf ? (one ? kernel_for<1, A_I8, 1, false, false, 2>(pl, &func) : kernel_for<1, A_I8, 2, false, false, 2>(pl, &func))
                    : (one ? kernel_for<1, A_I8, 1, false, false, 1>(pl, &func) : kernel_for<1, A_I8, 2, false, false, 1>(pl, &func));
        else if (WF == WF_I4 && acc_out)
            rc = bf ? (one ? kernel_for<4, A_I8, 1, true, false, 2>(pl, &func) : kernel_for<4, A_I8, 2, true, false, 2>(pl, &func))
                    : (one ? kernel_for<4, A_I8, 1, true, false, 1>(pl, &func) : kernel_for<4, A_I8, 2, true, false, 1>(pl, &func));
        else if (WF == WF_I4)
            rc = bf ? (one ? kernel_for<4, A_I8, 1, false, false, 2>(pl, &func) : kernel_for<4, A_I8, 2, false, false, 2>(pl, &func))
                    : (one ? kernel_for<4, A_I8, 1, false, false, 1>(pl, &func) : kernel_for<4, A_I8, 2, false, false, 1>(pl, &func));
        else
            rc = bf ? (one ? kernel_for<2, A_I8, 1, false, false, 2>(pl, &func) : kernel_for<2, A_I8, 2, false, false, 2>(pl, &func))
                    : (one ? kernel_for<2, A_I8, 1, false, false, 1>(pl, &func) : kernel_for<2, A_I8, 2, false, false, 1>(pl, &func));
    } else if (WF == WF_E2M1)
        rc = one ? kernel_for<WF_E2M1, A_F16, 1>(pl, &func) : kernel_for<WF_E2M1, A_F16, 2>(pl, &func);
    else if (WF == WF_E4M3 && AM == A_F8)
        rc = one ? kernel_for<WF_E4M3, A_F8, 1>(pl, &func) : kernel_for<WF_E4M3, A_F8, 2>(pl, &func);
    else if (WF == WF_E4M3)
        rc = one ? kernel_for<WF_E4M3, A_F16, 1>(pl, &func) : kernel_for<WF_E4M3, A_F16, 2>(pl, &func);
    else if (WF == WF_I1 && AM == A_F16)
        rc = one ? kernel_for<WF_I1, A_F16, 1>(pl, &func) : kernel_for<WF_I1, A_F16, 2>(pl, &func);
    else if (WF == WF_I1)
        rc = one ? kernel_for<WF_I1, A_I8, 1>(pl, &func) : kernel_for<WF_I1, A_I8, 2>(pl, &func);
    else if (WF == WF_I4 && AM == A_F16)
        rc = one ? kernel_for<4, A_F16, 1>(pl, &func)
                 : pl.wide ? kernel_for<4, A_F16, 2, false, true>(pl, &func) : kernel_for<4, A_F16, 2>(pl, &func);
    else if (WF == WF_I4 && AM == A_BF16)
        rc = one ? kernel_for<4, A_BF16, 1>(pl, &func)
                 : pl.wide ? kernel_for<4, A_BF16, 2, false, true>(pl, &func) : kernel_for<4, A_BF16, 2>(pl, &func);
    else if (WF == WF_I4 && acc_out) rc = one ? kernel_for<4, A_I8, 1, true>(pl, &func) : kernel_for<4, A_I8, 2, true>(pl, &func);
    else if (WF == WF_I4) rc = one ? kernel_for<4, A_I8, 1>(pl, &func) : kernel_for<4, A_I8, 2>(pl, &func);
    else if (AM == A_F16) rc = kernel_for<2, A_F16, 1>(pl, &func);
    else if (AM == A_BF16) rc = kernel_for<2, A_BF16, 1>(pl, &func);
    else rc = one ? kernel_for<2, A_I8, 1>(pl, &func) : kernel_for<2, A_I8, 2>(pl, &func);
    if (rc != WQ_OK) return rc;
    static_assert(sizeof(CUtensorMap) == 128 && sizeof(GemvParams) <= 256, "argument layout");
    out->func = func;
    out->grid = dim3(pl.P);
    out->block = dim3(kThreads);
    out->smem = pl.smem;
    memcpy(out->args, &tw, sizeof tw);
    memcpy(out->args + 128, &ta, sizeof ta);
    memcpy(out->args + 256, &p, sizeof p);
    out->argp[0] = out->args;
    out->argp[1] = out->args + 128;
    out->argp[2] = out->args + 256;
    out->nargs = 3;
    return WQ_OK;
}

// Few-token path (1 <= M <= 16).  Returns WQ_ERR_UNSUPPORTED if no launch plan fits.
wq_status gemv_small_m(int WF, int AM, const void *A, const float *a_scale, const uint8_t *Wq, const void *scales,
                       const void *zeros, const void *bias, void *C, int32_t *acc_out, int64_t M, int64_t N,
                       int64_t K, const wq_qconfig &c, cudaStream_t st)
{
    PreparedLaunch L;
    const wq_status rc = gemv_prepare(WF, AM, A, a_scale, Wq, scales, zeros, bias, C, acc_out, M, N, K, c, &L);
    if (rc != WQ_OK) return rc;
    return launch_prepared(L, st, "gemv_kernel");
}

int gemv_read_error()
{
    int v = 0, zero = 0;
    cudaMemcpyFromSymbol(&v, g_gemv_error, sizeof v);
    cudaMemcpyToSymbol(g_gemv_error, &zero, sizeof zero);
    return v;
}

}  // namespace wq
