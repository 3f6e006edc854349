// wq_gemm_tc.cu -- many-token weight-quantized matmul on the 5th-generation tensor cores
// (tcgen05), for INT4 (group scales, optional zero points), ternary INT2 and binary INT1
// weights (one scale per tensor), and FP4 e2m1 / FP8 e4m3 weights (group scales).
//
// C[M,N] = A[M,K] x dequant(Wq[N,K])^T: "BitBLAS practical guide", "What is BitBLAS",
// "Weight group quantization" and the FP16 x INT4 / INT2 and INT8 x INT4 / INT2 rows of its
// data-type table.  FP16 / BF16 activations use kind::f16 MMAs with fp32 accumulation;
// FP8 (e4m3) activations with FP8 weights use kind::f8f6f4 MMAs on the codes as they are;
// per-token INT8 activations ("Accelerating LLM inference with CUDA Graph and INT4
// quantization", part 1, steps 2-4) use kind::i8 MMAs whose int32 group sums are exact,
// followed by the (a_scale x w_scale) epilogue.
//
// At these sizes the product is tensor-bound.  The weights are the MMA's A operand
// (M = 128 weight rows) and live in Tensor Memory; the activations are the B operand
// (N = 128 tokens), brought into shared memory by TMA with the 128-byte swizzle that the
// MMA's K-major descriptor expects.  Per block of 128 k:
//  * a producer warp TMAs the block's activations and packed weights into a 4-stage ring;
//  * eight unpacking warps turn the packed weights of their own row (thread = weight row,
//    warp pairs split the 128 k) into exact values in natural k order -- q - z (INT4), the
//    ternary value (INT2), +-1 (INT1) or the e2m1 / e4m3 value (hardware conversion), as
//    f16 / bf16 pairs, or as signed bytes for INT8 activations -- and store them to the
//    stage's TMEM A-buffer (tcgen05.st);
//  * one thread issues the block's MMAs (8 of k 16, or 4 of k 32 for INT8) into a TMEM
//    accumulator of that block alone, and one tcgen05.commit frees the stage, its A-buffer
//    and announces the accumulator;
//  * eight folding warps read the accumulator back (tcgen05.ld) and add it, times the
//    row's group scale, into fp32 totals held in registers (each thread: one weight row x
//    64 tokens), then write C.
// Four A-buffers and two accumulators let unpacking run ahead of the MMAs and folding
// trail them.  The products are exact (|q - z| <= 15 times an f16 / bf16 / int8
// activation); the only rounding besides fp32 accumulation (int32 for INT8) is the
// final conversion.  Persistent CTAs walk the (weight tile, token tile) grid token-tile
// fastest so that concurrent CTAs share weight tiles in L2.  With fewer tiles than SMs, K is
// split over the CTAs of a thread-block cluster, one per slice: each keeps its fp32 partials
// in its (by then idle) ring, and after a cluster handshake each adds up its share of the
// tile's tokens from all slices' rings (distributed shared memory) in slice order.
// Long K (many scale groups) builds the scale tables from global memory, and keeps a single
// table if shared memory requires it.  Every wait is bounded; on expiry the CTA records an
// error, stops, waits for what it has in flight and frees its Tensor Memory.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include <algorithm>
#include <type_traits>

#include "wq_device.cuh"
#include "wq_format.h"
#include "wq_host.h"
#include "wq_tc.cuh"

namespace wq {

static __device__ int g_tc_error;

namespace {

constexpr int kBW = 128;  // weight rows per tile: MMA M
constexpr int kBT = 128;  // tokens per tile: MMA N
constexpr int kKB = 128;  // k per block
constexpr int kDeqWarps = 8;   // unpack weights into TMEM (two per TMEM lane quadrant: k halves)
constexpr int kFoldWarps = 8;  // fold block accumulators into the totals, write C
constexpr int kThreads = (2 + kDeqWarps + kFoldWarps) * 32;  // + warp 0 TMA, warp 1 MMA / TMEM
constexpr int kActBox = kBT * 128;  // one box of activations: 128 rows x 128 B (64 k FP, 128 k INT8)
// AM: 0 binary16, 1 bfloat16, 2 int8, 3 e4m3 activations (the last two one byte each)
__host__ __device__ constexpr int act_bytes(int AM) { return AM >= 2 ? kActBox : 2 * kActBox; }
// packed weights of a block: 16 KB FP8, 8 KB INT4 / FP4, 4 KB INT2, 2 KB INT1
__host__ __device__ constexpr int w_bytes(int WF) { return kBW * kKB * wf_bits(WF) / 8; }
__host__ __device__ constexpr int stage_bytes(int WF, int AM) { return act_bytes(AM) + w_bytes(WF); }
constexpr uint32_t kTmemCols = 512;
constexpr int kNA = 4;          // TMEM A-buffers: unpacked weights of a block, 64 columns each
constexpr int kND = 2;          // TMEM accumulators of a block, 128 columns each
constexpr uint32_t kAcol = 0;
constexpr uint32_t kDcol = kNA * 64;

struct TcParams {
    int M, N, K, G, gs, sym;
    int upg;               // blocks of 128 k per scale group (group_size / 128)
    const float *a_scale;  // INT8 activations: per-token scale
    const float *scale32;  // INT2 / INT1 weights: per-tensor scale
    int nkb;     // blocks of 128 k
    int ks;      // K slices per tile (split-K when tiles are fewer than SMs): the CTAs of one
                 // tile form a cluster of ks, cluster rank = slice
    int TT, NT;  // token tiles, tiles
    int S;       // ring stages
    int scst_off, tab_off, bar_off;
    int tab_rs;    // table row stride (entries; odd)
    int stage_sc;  // 1: scales / zeros are bulk-copied to shared memory first; 0: read from global
    int ntab;      // scale tables in shared memory (2: the next tile's is built while one is used)
    const uint16_t *scales16;
    const uint16_t *zeros;
    const void *bias;
    void *C;
    int32_t *acc_out;  // ACC: INT32 group sums [M][N][G] (INT4, group 128) or totals [M][N] (INT2, INT1)
    int nat;           // INT4 weights in the kernel-native order
};

__device__ __forceinline__ uint64_t globaltimer()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// Bounded wait (~2 s); on expiry, or once another warp has given up, returns false.
__device__ __forceinline__ bool tc_wait(uint64_t *bar, uint32_t parity, volatile int *abort)
{
    if (mbar_test_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    for (;;) {
        for (int i = 0; i < 4; ++i)
            if (mbar_try_wait_short(bar, parity)) return true;
        if (*abort) return false;
        if (globaltimer() - t0 > 2000000000ull) {
            atomicCAS(&g_tc_error, kErrNone, kErrWaitTimeout);
            *abort = 1;
            return false;
        }
    }
}

// The same for a barrier that other CTAs of the cluster arrive on (cluster-scope acquire).
__device__ __forceinline__ bool tc_wait_cluster(uint64_t *bar, uint32_t parity, volatile int *abort)
{
    const uint64_t t0 = globaltimer();
    for (;;) {
        for (int i = 0; i < 4; ++i)
            if (mbar_try_wait_cluster(bar, parity)) return true;
        if (*abort) return false;
        if (globaltimer() - t0 > 2000000000ull) {
            atomicCAS(&g_tc_error, kErrNone, kErrWaitTimeout);
            *abort = 1;
            return false;
        }
    }
}

template <bool BF16>
__device__ __forceinline__ void store_out(void *C, long long idx, float v)
{
    if constexpr (BF16) static_cast<__nv_bfloat16 *>(C)[idx] = __float2bfloat16_rn(v);
    else static_cast<__half *>(C)[idx] = __float2half_rn(v);
}

// INT4, INT8 activations: one word (8 nibbles) -> 8 signed bytes q - z in natural k order.
// zc = (0x80 - z) in every byte: q + 128 - z stays in 113 .. 143, no carries; ^0x80 makes it
// the two's complement byte of q - z.
__device__ __forceinline__ void unpack_word_s8(uint32_t w, uint32_t zc, uint32_t *o)
{
    const uint32_t lo = w & 0x0F0F0F0Fu, hi = (w >> 4) & 0x0F0F0F0Fu;
    o[0] = (prmt(lo, hi, 0x5140) + zc) ^ 0x80808080u;  // k0 k1 k2 k3
    o[1] = (prmt(lo, hi, 0x7362) + zc) ^ 0x80808080u;  // k4 .. k7
}

// Ternary INT2 (two's complement code, element 4j+i in bits 2i of byte j): with c = code ^ 2
// in 0..3 the value is c - 2.  FP: one word (16 codes) -> 8 pairs (k0,k1) .. (k14,k15): the
// nibble of a pair is placed in both halves, masked to (c_even, 4 c_odd), offset by the magic
// number (f16 1024, bf16 128) and mapped exactly to (c - 2) by one fma with (1, 1/4).
template <bool BF16>
__device__ __forceinline__ void unpack2_word(uint32_t w, uint32_t *o)
{
    const uint32_t y = w ^ 0xAAAAAAAAu;
    const uint32_t lo = y & 0x0F0F0F0Fu, hi = (y >> 4) & 0x0F0F0F0Fu;  // pairs 0,2,4,6 / 1,3,5,7
    const uint32_t magic = BF16 ? 0x43004300u : 0x64006400u;
    const uint32_t mul = BF16 ? 0x3E803F80u : 0x34003C00u;  // (1, 1/4)
    const uint32_t add = BF16 ? 0xC208C302u : 0xDC08E402u;  // (-(magic + 2), -(magic / 4 + 2))
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const uint32_t b = uint32_t(q >> 1);
        const uint32_t x = prmt((q & 1) ? hi : lo, 0u, b | (4u << 4) | (b << 8) | (4u << 12));
        const uint32_t v = and_or(x, 0x000C0003u, magic);
        o[q] = BF16 ? bf2_fma(v, mul, add) : h2_fma(v, mul, add);
    }
}

// Ternary INT2, INT8 activations: one word -> 16 signed bytes c - 2 in natural k order.
__device__ __forceinline__ void unpack2_word_s8(uint32_t w, uint32_t *o)
{
    const uint32_t y = w ^ 0xAAAAAAAAu;
    const uint32_t t0 = y & 0x03030303u, t1 = (y >> 2) & 0x03030303u;  // k0 k4 k8 k12 / k1 k5 ..
    const uint32_t t2 = (y >> 4) & 0x03030303u, t3 = (y >> 6) & 0x03030303u;
    const uint32_t u0 = prmt(t0, t1, 0x5140), u1 = prmt(t2, t3, 0x5140);  // k0 k1 k4 k5 / k2 k3 k6 k7
    const uint32_t u2 = prmt(t0, t1, 0x7362), u3 = prmt(t2, t3, 0x7362);  // k8 k9 k12 k13 / ..
    o[0] = (prmt(u0, u1, 0x5410) + 0x7E7E7E7Eu) ^ 0x80808080u;
    o[1] = (prmt(u0, u1, 0x7632) + 0x7E7E7E7Eu) ^ 0x80808080u;
    o[2] = (prmt(u2, u3, 0x5410) + 0x7E7E7E7Eu) ^ 0x80808080u;
    o[3] = (prmt(u2, u3, 0x7632) + 0x7E7E7E7Eu) ^ 0x80808080u;
}

// Unpacks one 32-bit word (8 nibbles, k0 in the low nibble) into 4 pairs (k0,k1) .. (k6,k7)
// of magic + nibble (f16: 1024 + q, bf16: 128 + q), then adds zc = -(magic + z): exact q - z.
template <bool BF16>
__device__ __forceinline__ void unpack_word(uint32_t w, uint32_t zc, uint32_t *o)
{
    const uint32_t magic = BF16 ? 0x43434343u : 0x64646464u;
    const uint32_t lo = w & 0x0F0F0F0Fu;         // k0 k2 k4 k6
    const uint32_t hi = (w >> 4) & 0x0F0F0F0Fu;  // k1 k3 k5 k7
    const uint32_t p0 = prmt(lo, hi, 0x5140);    // k0 k1 k2 k3
    const uint32_t p1 = prmt(lo, hi, 0x7362);    // k4 k5 k6 k7
    uint32_t x[4] = {prmt(p0, magic, 0x4140), prmt(p0, magic, 0x4342), prmt(p1, magic, 0x4140),
                     prmt(p1, magic, 0x4342)};
#pragma unroll
    for (int i = 0; i < 4; ++i) o[i] = BF16 ? bf2_fma(x[i], 0x3F803F80u, zc) : h2_add(x[i], zc);
}

// ACC (INT8 activations only): also store the exact INT32 sums in p.acc_out.  For INT4
// with group_size 128 a block of 128 k is one group, so each block accumulator read from
// Tensor Memory is one acc_g (the zero point is already inside the weight bytes); for
// ternary INT2 the fp32 totals are exact integers (|sum| < 2^24) and are stored at the end.
// Kernel-native INT4 order (nibble i of a word = element 0,2,4,6,1,3,5,7): the masks give the
// natural pairs directly.  f16: (x & 0x000F000F) | magic = 1024 + q of (k, k+1);
// (x & 0x00F000F0) | magic = 1024 + 16 q of (k+2, k+3), made q - z by one fma with 1/16;
// the upper byte the same after one shift.  bf16 has 7 mantissa bits, so its odd pairs are
// shifted into place instead of scaled.
template <bool BF16>
__device__ __forceinline__ void unpack_word_nat(uint32_t w, uint32_t z, uint32_t *o)
{
    if constexpr (BF16) {
        const uint32_t c1 = 0xC300u | z, cc = c1 | (c1 << 16);  // -(128 + z)
#pragma unroll
        for (int i = 0; i < 4; ++i) o[i] = bf2_fma(and_or(w >> (4 * i), 0x000F000Fu, 0x43004300u), 0x3F803F80u, cc);
    } else {
        const uint32_t a1 = 0xE400u | z, clo = a1 | (a1 << 16);                // -(1024 + z)
        const uint32_t b1 = 0xD400u | (z << 4), chi = b1 | (b1 << 16);         // -(64 + z)
        const uint32_t w8 = w >> 8;
        o[0] = h2_add(and_or(w, 0x000F000Fu, 0x64006400u), clo);
        o[1] = h2_fma(and_or(w, 0x00F000F0u, 0x64006400u), 0x2C002C00u, chi);
        o[2] = h2_add(and_or(w8, 0x000F000Fu, 0x64006400u), clo);
        o[3] = h2_fma(and_or(w8, 0x00F000F0u, 0x64006400u), 0x2C002C00u, chi);
    }
}

// Kernel-native INT4, INT8 activations: one word -> 8 signed bytes q - z in natural k order.
__device__ __forceinline__ void unpack_word_s8_nat(uint32_t w, uint32_t zc, uint32_t *o)
{
    const uint32_t lo = w & 0x0F0F0F0Fu, hi = (w >> 4) & 0x0F0F0F0Fu;  // k0 k4 k1 k5 / k2 k6 k3 k7
    o[0] = (prmt(lo, hi, 0x6420) + zc) ^ 0x80808080u;  // k0 k1 k2 k3
    o[1] = (prmt(lo, hi, 0x7531) + zc) ^ 0x80808080u;  // k4 .. k7
}

// (a & m) | (b & ~m) in one LOP3.
__device__ __forceinline__ uint32_t bitsel(uint32_t a, uint32_t b, uint32_t m)
{
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xE4;" : "=r"(d) : "r"(a), "r"(b), "r"(m));
    return d;
}

// INT1, FP16 activations: one word (32 bits, k0 in bit 0) -> 16 binary16 pairs (k0,k1) ..
// (k30,k31) of +-1: bit 2p moved to bit 15 and bit 2p+1 to bit 31, then one LOP3.
__device__ __forceinline__ void unpack1_word(uint32_t w, uint32_t *o)
{
#pragma unroll
    for (int p = 0; p < 16; ++p) {
        const uint32_t lo = p <= 7 ? (w << (15 - 2 * p)) : (w >> (2 * p - 15));
        const uint32_t hi = w << (30 - 2 * p);
        o[p] = pm1_f16x2(bitsel(lo, hi, 0x0000FFFFu));
    }
}

// INT1, INT8 activations: one word -> 32 signed bytes +-1 in natural k order.  Nibble i
// times 0x00204081 puts its bits at 0, 8, 16 and 24 (no carries); 2c + 0x7F, ^0x80 -> -1 / +1.
__device__ __forceinline__ void unpack1_word_s8(uint32_t w, uint32_t *o)
{
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const uint32_t x = (((w >> (4 * i)) & 15u) * 0x00204081u) & 0x01010101u;
        o[i] = ((x << 1) + 0x7F7F7F7Fu) ^ 0x80808080u;
    }
}

template <int WF, int AM, bool ACC = false>
__global__ void __launch_bounds__(kThreads, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_w,
                   const TcParams p)
{
    constexpr bool BF16 = AM == 1, I8 = AM == 2, F8 = AM == 3, B8 = I8 || F8;
    constexpr bool GROUPED = wf_grouped(WF);
    constexpr int kActBytes = act_bytes(AM), kStageBytes = stage_bytes(WF, AM);
    static_assert(kBW * kBT * 4 <= kNA * kStageBytes, "split-K totals must fit in the ring");
    // scale table entries: binary16 scale | zero point << 16 (INT4), the scale alone (FP4 / FP8)
    using TabT = typename std::conditional<WF == WF_I4, uint32_t, uint16_t>::type;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *ring = smem;  // kNA x (activations | packed weights)
    uint16_t *scst = reinterpret_cast<uint16_t *>(smem + p.scst_off);  // 2 x (scales, zeros) [128][G]
    TabT *tabs = reinterpret_cast<TabT *>(smem + p.tab_off);           // 2 x [G][tab_rs]
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + p.bar_off);
    // rel[s]: the MMAs of the step in stage s have completed: stage s and A-buffer s are free
    // and accumulator step % kND holds the block's sums
    uint64_t *full = bars, *rel = bars + kNA;
    uint64_t *afull = bars + 2 * kNA, *dfree = afull + kNA;
    uint64_t *scbar = dfree + kND, *tready = scbar + 2, *tdone = tready + 2, *fin = tdone + 2, *mbar = fin + 1;
    // xbar: every slice of the cluster has its partial totals in its ring; dbar: every slice
    // has read its share of them (one arrival per CTA of the cluster on each)
    uint64_t *fbar = mbar + 1, *xbar = fbar + 1, *dbar = xbar + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(dbar + 1);
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const size_t stab_elems = size_t(kBW) * p.G;          // one staging buffer (scales or zeros)
    const size_t tab_elems = size_t(p.G) * p.tab_rs;      // one table

    if (threadIdx.x == 0) {
        for (int b = 0; b < kNA; ++b) {
            mbar_init(&full[b], 1);
            mbar_init(&rel[b], 1);
            mbar_init(&afull[b], kDeqWarps);
        }
        for (int b = 0; b < kND; ++b) mbar_init(&dfree[b], kFoldWarps);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&scbar[b], 1);
            mbar_init(&tready[b], 1);
            mbar_init(&tdone[b], kFoldWarps);
        }
        mbar_init(fin, 1);
        mbar_init(mbar, kDeqWarps);
        mbar_init(fbar, kFoldWarps);
        mbar_init(xbar, p.ks);
        mbar_init(dbar, p.ks);
        *abort = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tc::tmem_alloc(tmem_slot, kTmemCols);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (p.ks > 1) {
        // every thread announces that its CTA's barriers are initialised (published by thread
        // 0's fence_barrier_init); the folding warps wait for all CTAs of the cluster before
        // their first arrival on another's barrier
        cluster_arrive_relaxed();
        if (threadIdx.x == 0 && (cluster_size() != uint32_t(p.ks) || cluster_rank() != blockIdx.x % uint32_t(p.ks))) {
            atomicCAS(&g_tc_error, kErrNone, kErrBadLaunch);
            *abort = 1;
        }
        __syncthreads();
    }
    const uint32_t tbase = *tmem_slot;
    grid_dep_launch();

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&tmap_a);
            tma_prefetch_desc(&tmap_w);
            auto issue_scales = [&](int n0, int tl) {  // the tile's scale / zero rows: contiguous in [N, G]
                if constexpr (GROUPED) {
                    if (!p.stage_sc) return;
                    const int nrows = min(kBW, p.N - n0);
                    const uint32_t bytes16 = (uint32_t(nrows) * p.G * 2u) & ~15u;
                    uint16_t *sc = scst + size_t(tl & 1) * 2 * stab_elems;
                    mbar_arrive_expect_tx(&scbar[tl & 1], bytes16 * (p.sym ? 1u : 2u));
                    if (bytes16) {
                        bulk_load(sc, p.scales16 + (size_t)n0 * p.G, bytes16, &scbar[tl & 1]);
                        if (!p.sym) bulk_load(sc + stab_elems, p.zeros + (size_t)n0 * p.G, bytes16, &scbar[tl & 1]);
                    }
                }
            };
            // Weights and scales do not depend on the previous kernel: the first task's scales and
            // the packed weights of its first kNA blocks go out before griddepcontrol.wait.
            int npre = 0;
            if (blockIdx.x < p.NT * p.ks) {
                const int tile = blockIdx.x / p.ks, sp = blockIdx.x - tile * p.ks;
                const int kb0 = sp * p.nkb / p.ks, kb1 = (sp + 1) * p.nkb / p.ks;
                const int n0 = (tile / p.TT) * kBW;
                issue_scales(n0, 0);
                npre = min(kNA, kb1 - kb0);
                for (int i = 0; i < npre; ++i) {
                    uint8_t *st = ring + size_t(i) * kStageBytes;
                    mbar_arrive_expect_tx(&full[i], kStageBytes);
                    tma_load_2d(st + kActBytes, &tmap_w, (kb0 + i) * (kKB * wf_bits(WF) / 8), n0, &full[i]);
                }
            }
            grid_dep_wait();  // activations may be written by the previous kernel
            uint32_t step = 0;
            int tl = 0;
            for (int t = blockIdx.x; t < p.NT * p.ks && !*abort; t += gridDim.x, ++tl) {
                const int tile = t / p.ks, sp = t - tile * p.ks;
                const int kb0 = sp * p.nkb / p.ks, kb1 = (sp + 1) * p.nkb / p.ks;
                const int n0 = (tile / p.TT) * kBW, m0 = (tile % p.TT) * kBT;
                if (tl > 0) issue_scales(n0, tl);
                for (int kb = kb0; kb < kb1; ++kb, ++step) {
                    const int s = int(step % kNA);
                    uint8_t *st = ring + size_t(s) * kStageBytes;
                    const bool pre = tl == 0 && kb - kb0 < npre;  // weights already on their way
                    if (!pre) {
                        if (!tc_wait(&rel[s], ((step / kNA) & 1) ^ 1, abort)) break;
                        mbar_arrive_expect_tx(&full[s], kStageBytes);
                        tma_load_2d(st + kActBytes, &tmap_w, kb * (kKB * wf_bits(WF) / 8), n0, &full[s]);
                    }
                    tma_load_2d(st, &tmap_a, kb * kKB, m0, &full[s]);
                    if constexpr (!B8) tma_load_2d(st + kActBox, &tmap_a, kb * kKB + 64, m0, &full[s]);
                }
            }
            // nothing may land in shared memory after the CTA exits: wait for the last stages
            for (uint32_t k = step > uint32_t(kNA) ? step - kNA : 0; k < step; ++k)
                tc_wait(&full[k % kNA], (k / kNA) & 1, abort);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc = I8 ? tc::idesc_i8(kBW, kBT) : F8 ? tc::idesc_f8(kBW, kBT) : tc::idesc_f16(BF16, kBW, kBT);
            uint64_t desc0[kNA];  // descriptor of each stage's activations (k step 0)
#pragma unroll
            for (int b = 0; b < kNA; ++b) desc0[b] = tc::sdesc_sw128(smem_u32(ring + size_t(b) * kStageBytes));
            uint32_t step = 0;
            bool issued = false;
            for (int t = blockIdx.x; t < p.NT * p.ks && !*abort; t += gridDim.x) {
                const int tile = t / p.ks, sp = t - tile * p.ks;
                const int nb = (sp + 1) * p.nkb / p.ks - sp * p.nkb / p.ks;
                for (int kb = 0; kb < nb; ++kb, ++step) {
                    const uint32_t s = step % kNA, db = step % kND;
                    // afull: the unpacking warps have seen the stage's data and stored the weights
                    if (!tc_wait(&afull[s], (step / kNA) & 1, abort)) break;
                    if (!tc_wait(&dfree[db], ((step / kND) & 1) ^ 1, abort)) break;
                    tc::fence_after_sync();
                    const uint64_t d0 = s == 0 ? desc0[0] : s == 1 ? desc0[1] : s == 2 ? desc0[2] : desc0[3];
                    const uint32_t dcol = tbase + kDcol + db * kBT, acol = tbase + kAcol + s * 64;
                    if constexpr (I8) {
#pragma unroll
                        for (int kk = 0; kk < kKB / 32; ++kk)  // k 32: 32 bytes per step
                            tc::mma_i8_ts(dcol, acol + kk * 8, d0 + uint64_t((kk * 32) >> 4), idesc, kk > 0 ? 1u : 0u);
                    } else if constexpr (F8) {
#pragma unroll
                        for (int kk = 0; kk < kKB / 32; ++kk)  // k 32: 32 bytes per step
                            tc::mma_f8_ts(dcol, acol + kk * 8, d0 + uint64_t((kk * 32) >> 4), idesc, kk > 0 ? 1u : 0u);
                    } else {
#pragma unroll
                        for (int kk = 0; kk < kKB / 16; ++kk)  // k 16: 32 bytes per step
                            tc::mma_f16_ts(dcol, acol + kk * 8,
                                           d0 + uint64_t(((kk >> 2) * kActBox + (kk & 3) * 32) >> 4), idesc,
                                           kk > 0 ? 1u : 0u);
                    }
                    tc::commit(&rel[s]);
                    issued = true;
                }
            }
            if (issued) {  // all MMAs complete before the Tensor Memory is freed
                tc::commit(fin);
                tc_wait(fin, 0, abort);
            }
        }
    } else if (warp < 2 + kDeqWarps) {
        // ------------------------------------------------------------ unpacking warps
        const int q = warp & 3;          // TMEM lane quadrant of this warp
        const int kh = (warp - 2) >> 2;  // k half of the block
        const int r = q * 32 + lane;     // weight row within the tile
        const uint32_t tlane = tbase + (uint32_t(q * 32) << 16);
        const uint32_t magic_z = BF16 ? 0xC300u : 0xE400u;  // -(magic + z) = magic_z | z
        uint32_t step = 0, mphase = 0;
        auto deq_sync = [&]() -> bool {  // bounded barrier of the unpacking warps (one arrival per warp)
            __syncwarp();
            if (lane == 0) mbar_arrive(mbar);
            const bool ok = tc_wait(mbar, mphase & 1, abort);
            ++mphase;
            return ok;
        };
        int tl = 0;
        for (int t = blockIdx.x; t < p.NT * p.ks && !*abort; t += gridDim.x, ++tl) {
            const int tile = t / p.ks, sp = t - tile * p.ks;
            const int kb0 = sp * p.nkb / p.ks, kb1 = (sp + 1) * p.nkb / p.ks;
            const int n0 = (tile / p.TT) * kBW;
            const int nrows = min(kBW, p.N - n0);
            const int tb = tl % p.ntab;  // this tile's table buffer
            TabT *tab = tabs + size_t(tb) * tab_elems;
            // ---- scale / zero table of the tile: [g][row] = fp16 scale bits (| z << 16 for INT4)
            if constexpr (GROUPED) {
            if (p.stage_sc && !tc_wait(&scbar[tl & 1], (tl >> 1) & 1, abort)) break;
            // the folding warps are done with tile tl - ntab, the buffer's previous user
            if (tl >= p.ntab && !tc_wait(&tdone[tb], ((tl - p.ntab) / p.ntab) & 1, abort)) break;
            if (!deq_sync()) break;
            {
                // entries e = row * G + g of the staged copy, 8 per 16-byte vector and thread;
                // what the copy left out (a ragged tail, rows past N, or all of it when the
                // scales are not staged) is read directly from global memory
                const uint16_t *sc = scst + size_t(tl & 1) * 2 * stab_elems;
                const int cnt = nrows * p.G;
                const int n16 = p.stage_sc ? int(((uint32_t(cnt) * 2u) & ~15u) >> 1) : 0;
                const int tid = threadIdx.x - 64;  // 0 .. 255 over the unpacking warps
                for (int v8 = tid; v8 < n16 / 8; v8 += kDeqWarps * 32) {
                    const uint4 sv = *reinterpret_cast<const uint4 *>(sc + v8 * 8);
                    const uint4 zv = p.sym ? make_uint4(0, 0, 0, 0) : *reinterpret_cast<const uint4 *>(sc + stab_elems + v8 * 8);
                    const uint32_t sw[4] = {sv.x, sv.y, sv.z, sv.w}, zw[4] = {zv.x, zv.y, zv.z, zv.w};
                    int rl = (v8 * 8) / p.G, gi = v8 * 8 - rl * p.G;
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const uint32_t sb = (sw[i >> 1] >> (16 * (i & 1))) & 0xffffu;
                        uint32_t z = 8;
                        if (!p.sym) z = uint32_t(__half2float(__ushort_as_half(uint16_t(zw[i >> 1] >> (16 * (i & 1)))))) & 15u;
                        tab[(size_t)gi * p.tab_rs + rl] = TabT(sb | (z << 16));
                        if (++gi == p.G) {
                            gi = 0;
                            ++rl;
                        }
                    }
                }
                for (int e = n16 + tid; e < kBW * p.G; e += kDeqWarps * 32) {
                    const int rl = e / p.G, gi = e - rl * p.G;
                    uint32_t v = 0;
                    if (e < cnt) {
                        const uint16_t sb = __ldg(p.scales16 + (size_t)n0 * p.G + e);
                        uint32_t z = 8;
                        if (!p.sym) z = uint32_t(__half2float(__ushort_as_half(__ldg(p.zeros + (size_t)n0 * p.G + e)))) & 15u;
                        v = uint32_t(sb) | (z << 16);
                    }
                    tab[(size_t)gi * p.tab_rs + rl] = TabT(v);
                }
            }
            if (!deq_sync()) break;
            if (threadIdx.x == 64) mbar_arrive(&tready[tb]);
            }

            for (int kb = kb0; kb < kb1; ++kb, ++step) {
                const uint32_t s = step % kNA;  // ring stage and TMEM A-buffer
                // full also tells that the MMAs of step - kNA (stage and A-buffer s) have completed
                if (!tc_wait(&full[s], (step / kNA) & 1, abort)) break;
                const uint8_t *wst = ring + size_t(s) * kStageBytes + kActBytes;
                if constexpr (F8) {
                    // FP8 weights for e4m3 activations: this row's 64 code bytes of the k half
                    // (128-byte rows, 128-byte swizzle), stored to Tensor Memory as they are
                    static_assert(WF == WF_E4M3, "FP8 activations take FP8 weights");
                    const uint8_t *wrow = wst + r * 128;
                    const uint32_t sw = uint32_t(r & 7);
                    uint32_t v[16];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const uint4 c = lds128(wrow + ((uint32_t(4 * kh + i) ^ sw) << 4));
                        v[4 * i + 0] = c.x;
                        v[4 * i + 1] = c.y;
                        v[4 * i + 2] = c.z;
                        v[4 * i + 3] = c.w;
                    }
                    tc::fence_after_sync();
                    tc::st_32x32b_x16(tlane + kAcol + s * 64 + kh * 16, v);
                } else if constexpr (WF == WF_E2M1) {
                    // this row's 32 packed bytes of the k half (64-byte rows, 64-byte swizzle)
                    const uint8_t *wrow = wst + r * 64;
                    const uint32_t sw = uint32_t((r >> 1) & 3);
                    const uint4 w0 = lds128(wrow + ((uint32_t(2 * kh) ^ sw) << 4));
                    const uint4 w1 = lds128(wrow + ((uint32_t(2 * kh + 1) ^ sw) << 4));
                    tc::fence_after_sync();
                    uint32_t v[32];
                    const uint32_t wd[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        v[4 * i + 0] = e2m1x2_to_f16x2<0>(wd[i]);
                        v[4 * i + 1] = e2m1x2_to_f16x2<1>(wd[i]);
                        v[4 * i + 2] = e2m1x2_to_f16x2<2>(wd[i]);
                        v[4 * i + 3] = e2m1x2_to_f16x2<3>(wd[i]);
                    }
                    tc::st_32x32b_x32(tlane + kAcol + s * 64 + kh * 32, v);
                } else if constexpr (WF == WF_E4M3) {
                    // this row's 64 bytes of the k half (128-byte rows, 128-byte swizzle)
                    const uint8_t *wrow = wst + r * 128;
                    const uint32_t sw = uint32_t(r & 7);
                    uint4 c4[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) c4[i] = lds128(wrow + ((uint32_t(4 * kh + i) ^ sw) << 4));
                    tc::fence_after_sync();
                    uint32_t v[32];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const uint32_t wd[4] = {c4[i].x, c4[i].y, c4[i].z, c4[i].w};
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            v[8 * i + 2 * j] = e4m3x2_to_f16x2<0>(wd[j]);
                            v[8 * i + 2 * j + 1] = e4m3x2_to_f16x2<1>(wd[j]);
                        }
                    }
                    tc::st_32x32b_x32(tlane + kAcol + s * 64 + kh * 32, v);
                } else if constexpr (WF == WF_I1) {
                    // this row's 8 packed bytes of the k half (16-byte rows, not swizzled)
                    const uint2 w = lds64(wst + r * 16 + kh * 8);
                    tc::fence_after_sync();
                    if constexpr (I8) {
                        uint32_t v[16];
                        unpack1_word_s8(w.x, v);
                        unpack1_word_s8(w.y, v + 8);
                        tc::st_32x32b_x16(tlane + kAcol + s * 64 + kh * 16, v);
                    } else {
                        uint32_t v[32];
                        unpack1_word(w.x, v);
                        unpack1_word(w.y, v + 16);
                        tc::st_32x32b_x32(tlane + kAcol + s * 64 + kh * 32, v);
                    }
                } else if constexpr (WF == WF_I4) {
                    // this row's 32 packed bytes of the k half (64-byte rows, 64-byte swizzle)
                    const uint8_t *wrow = wst + r * 64;
                    const uint32_t sw = uint32_t((r >> 1) & 3);
                    const uint4 w0 = lds128(wrow + ((uint32_t(2 * kh) ^ sw) << 4));
                    const uint4 w1 = lds128(wrow + ((uint32_t(2 * kh + 1) ^ sw) << 4));
                    const uint32_t z = tab[(size_t)(p.upg == 1 ? kb : kb / p.upg) * p.tab_rs + r] >> 16;
                    tc::fence_after_sync();
                    if constexpr (I8) {
                        const uint32_t zc = (0x80u - z) * 0x01010101u;
                        uint32_t v[16];
                        const uint32_t wd[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
                        if (p.nat) {
#pragma unroll
                            for (int i = 0; i < 8; ++i) unpack_word_s8_nat(wd[i], zc, v + 2 * i);
                        } else {
#pragma unroll
                            for (int i = 0; i < 8; ++i) unpack_word_s8(wd[i], zc, v + 2 * i);
                        }
                        tc::st_32x32b_x16(tlane + kAcol + s * 64 + kh * 16, v);
                    } else {
                        const uint32_t zc1 = magic_z | z;
                        const uint32_t zc = zc1 | (zc1 << 16);
                        uint32_t v[32];
                        const uint32_t wd[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
                        if (p.nat) {
#pragma unroll
                            for (int i = 0; i < 8; ++i) unpack_word_nat<BF16>(wd[i], z, v + 4 * i);
                        } else {
#pragma unroll
                            for (int i = 0; i < 8; ++i) unpack_word<BF16>(wd[i], zc, v + 4 * i);
                        }
                        tc::st_32x32b_x32(tlane + kAcol + s * 64 + kh * 32, v);
                    }
                } else {
                    // this row's 16 packed bytes of the k half (32-byte rows, not swizzled)
                    const uint4 w = lds128(wst + r * 32 + kh * 16);
                    tc::fence_after_sync();
                    if constexpr (I8) {
                        uint32_t v[16];
                        unpack2_word_s8(w.x, v + 0);
                        unpack2_word_s8(w.y, v + 4);
                        unpack2_word_s8(w.z, v + 8);
                        unpack2_word_s8(w.w, v + 12);
                        tc::st_32x32b_x16(tlane + kAcol + s * 64 + kh * 16, v);
                    } else {
                        uint32_t v[32];
                        unpack2_word<BF16>(w.x, v + 0);
                        unpack2_word<BF16>(w.y, v + 8);
                        unpack2_word<BF16>(w.z, v + 16);
                        unpack2_word<BF16>(w.w, v + 24);
                        tc::st_32x32b_x32(tlane + kAcol + s * 64 + kh * 32, v);
                    }
                }
                tc::wait_st();
                tc::fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(&afull[s]);
            }
        }
    } else {
        // ------------------------------------------------------------ folding warps
        const int q = warp & 3;                       // TMEM lane quadrant of this warp
        const int th = (warp - 2 - kDeqWarps) >> 2;   // token half of the tile
        const int r = q * 32 + lane;                  // weight row within the tile
        const uint32_t tlane = tbase + (uint32_t(q * 32) << 16);
        grid_dep_wait();  // C and bias belong to this kernel only once the previous one is done
        uint32_t step = 0;
        int tl = 0;
        uint32_t fphase = 0;
        auto fold_sync = [&]() -> bool {  // bounded barrier of the folding warps (one arrival per warp)
            __syncwarp();
            if (lane == 0) mbar_arrive(fbar);
            const bool ok = tc_wait(fbar, fphase & 1, abort);
            ++fphase;
            return ok;
        };
        for (int t = blockIdx.x; t < p.NT * p.ks && !*abort; t += gridDim.x, ++tl) {
            const int tile = t / p.ks, sp = t - tile * p.ks;
            const int kb0 = sp * p.nkb / p.ks, kb1 = (sp + 1) * p.nkb / p.ks;
            const int n0 = (tile / p.TT) * kBW, m0 = (tile % p.TT) * kBT;
            const int tb = tl % p.ntab;
            const TabT *tab = tabs + size_t(tb) * tab_elems;
            if constexpr (GROUPED)
                if (!tc_wait(&tready[tb], (tl / p.ntab) & 1, abort)) break;
            float tot[64];
#pragma unroll
            for (int j = 0; j < 64; ++j) tot[j] = 0.f;
            bool ok = true;
            for (int kb = kb0; kb < kb1; ++kb, ++step) {
                const uint32_t db = step % kND, s = step % kNA;
                float sv = 1.f;  // INT2 / INT1: the per-tensor scale is applied at the end
                if constexpr (GROUPED)
                    sv = __half2float(__ushort_as_half(uint16_t(tab[(size_t)(p.upg == 1 ? kb : kb / p.upg) * p.tab_rs + r])));
                if (!tc_wait(&rel[s], (step / kNA) & 1, abort)) { ok = false; break; }
                tc::fence_after_sync();
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t d[16];
                    tc::ld_32x32b_x16(tlane + kDcol + db * kBT + th * 64 + c * 16, d);
                    tc::wait_ld();
                    if (c == 3) {
                        tc::fence_before_sync();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&dfree[db]);
                    }
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        // INT8: exact int32 block sums (< 2^24 in magnitude, exact in fp32)
                        const float dv = I8 ? float(int(d[j])) : __uint_as_float(d[j]);
                        tot[c * 16 + j] = fmaf(sv, dv, tot[c * 16 + j]);
                    }
                    if constexpr (ACC && WF == WF_I4) {
                        const int n = n0 + r, mb = m0 + th * 64 + c * 16;
                        if (n < p.N)
#pragma unroll
                            for (int j = 0; j < 16; ++j)
                                if (mb + j < p.M) p.acc_out[((size_t)(mb + j) * p.N + n) * p.G + kb] = int(d[j]);
                    }
                }
            }
            if (!ok) break;
            __syncwarp();
            if constexpr (GROUPED)
                if (lane == 0) mbar_arrive(&tdone[tb]);

            // C[m][n] = total (+ bias[n]) for weight row n of this thread
            const int n = n0 + r;
            float b = 0.f;
            if (p.bias && n < p.N) {
                if constexpr (BF16) b = __bfloat162float(__ldg(static_cast<const __nv_bfloat16 *>(p.bias) + n));
                else b = __half2float(__ldg(static_cast<const __half *>(p.bias) + n));
            }
            const float ws = wf_per_tensor(WF) ? __ldg(p.scale32) : 1.f;
            // as: the token's activation scale (INT8 / FP8 activations)
            auto emit = [&](int m, float total, float as) {
                if constexpr (ACC && wf_per_tensor(WF)) p.acc_out[(size_t)m * p.N + n] = int(total);
                float v;
                if constexpr (B8) v = as * (wf_per_tensor(WF) ? ws * total : total);
                else v = ws * total;
                store_out<BF16>(p.C, (long long)m * p.N + n, v + b);
            };

            if (p.ks > 1) {
                // Split K over the tile's cluster: each slice leaves its totals in its own ring
                // (idle now: the tile's copies and MMAs have completed), [token][row] in fp32;
                // once all slices have theirs in place, slice sp adds up its share of the tokens
                // from every slice's ring (distributed shared memory) in slice order, so the sum
                // does not depend on which slice finishes first, and writes those outputs.
                float *part = reinterpret_cast<float *>(ring);
                fence_proxy_async();  // the ring's last users were TMA writes and MMA reads
#pragma unroll
                for (int j = 0; j < 64; ++j) part[(th * 64 + j) * kBW + r] = tot[j];
                if (!fold_sync()) break;
                if (tl == 0) cluster_wait();  // every CTA of the cluster has initialised its barriers
                if (warp == 2 + kDeqWarps && lane < p.ks) mbar_arrive_cluster(dsmem_addr(smem_u32(xbar), uint32_t(lane)));
                if (!tc_wait_cluster(xbar, 0, abort)) break;
                const int mt = min(kBT, p.M - m0);  // tokens of the tile
                const int lo = sp * mt / p.ks, hi = (sp + 1) * mt / p.ks, mid = (lo + hi) / 2;
                const int ma = th ? mid : lo, mb = th ? hi : mid;
                const uint32_t part0 = smem_u32(part) + uint32_t(r) * 4u;
                for (int m = ma; m < mb; m += 4) {
                    float v[4] = {0.f, 0.f, 0.f, 0.f}, as4[4] = {1.f, 1.f, 1.f, 1.f};
                    if constexpr (B8)  // in flight together with the loads below
#pragma unroll
                        for (int u = 0; u < 4; ++u)
                            if (m + u < mb) as4[u] = __ldg(p.a_scale + m0 + m + u);
                    for (int q2 = 0; q2 < p.ks; ++q2) {
                        const uint32_t src = dsmem_addr(part0, uint32_t(q2));
#pragma unroll
                        for (int u = 0; u < 4; ++u)
                            if (m + u < mb) v[u] += ld_dsmem_f32(src + uint32_t((m + u) * kBW) * 4u);
                    }
                    if (n < p.N)
#pragma unroll
                        for (int u = 0; u < 4; ++u)
                            if (m + u < mb) emit(m0 + m + u, v[u], as4[u]);
                }
                // every slice may leave once all have read their shares from its ring (the values
                // read are used above, so the loads have completed)
                if (!fold_sync()) break;
                if (warp == 2 + kDeqWarps && lane < p.ks)
                    mbar_arrive_cluster_relaxed(dsmem_addr(smem_u32(dbar), uint32_t(lane)));
                if (!tc_wait_cluster(dbar, 0, abort)) break;
                continue;
            }

            // ---- one weight row x 64 tokens per thread
            if (n < p.N) {
                const int mb = m0 + th * 64;
#pragma unroll
                for (int j = 0; j < 64; ++j)
                    if (mb + j < p.M) emit(mb + j, tot[j], B8 ? __ldg(p.a_scale + mb + j) : 1.f);
            }
        }
    }

    // every role has stopped, and its copies and MMAs have completed: free the Tensor Memory
    __syncwarp();
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tbase, kTmemCols);
    }
}

struct TcPlan {
    int S = 0, scst_off = 0, tab_off = 0, bar_off = 0, tab_rs = 1, stage_sc = 1, ntab = 2;
    size_t smem = 0;
    bool ok = false;
};

// G: groups of the scale table (0 for INT2 / INT1: one per-tensor scale, no table); tab_es:
// bytes per table entry.  Preferred: scales staged by bulk copy and two tables (the next
// tile's built while one is in use).  Long K (many groups) drops the staging, then the
// second table, to keep the ring.
TcPlan make_plan(int nkb, int G, int stage, int tab_es, const DeviceInfo &dev)
{
    TcPlan pl;
    pl.tab_rs = kBW + 1;
    const size_t bars = 8 * (3 * kNA + 2 * kND + 12) + 16;
    const size_t budget = size_t(dev.max_smem_optin) - 1024;
    if (nkb < kNA) return pl;  // the ring has one stage per TMEM A-buffer
    const int forms[3][2] = {{1, 2}, {0, 2}, {0, 1}};
    for (const auto &f : forms) {
        const size_t scst = f[0] ? (size_t(2) * 2 * kBW * G * 2 + 15) & ~size_t(15) : 0;
        const size_t tab = (size_t(f[1]) * G * pl.tab_rs * tab_es + 15) & ~size_t(15);
        if (budget <= scst + tab + bars || (budget - scst - tab - bars) / size_t(stage) < size_t(kNA)) continue;
        pl.stage_sc = f[0];
        pl.ntab = f[1];
        pl.S = kNA;
        size_t off = size_t(pl.S) * stage;
        pl.scst_off = int(off);
        off += scst;
        pl.tab_off = int(off);
        off += tab;
        pl.bar_off = int((off + 7) & ~size_t(7));
        off = pl.bar_off + bars;
        pl.smem = ((off + 15) & ~size_t(15)) + 1024;
        pl.ok = pl.smem <= size_t(dev.max_smem_optin);
        return pl;
    }
    return pl;
}

constexpr int kMaxSlices = 8;  // the portable thread-block cluster size

// K slices per tile: when the tiles are fewer than the SMs, each tile's K range is cut
// into slices (at least 4 blocks each) so that tiles x slices <= SMs.
int choose_slices(int64_t M, int64_t N, int64_t K, int sm_count)
{
    const int64_t tiles = ((M + kBT - 1) / kBT) * ((N + kBW - 1) / kBW);
    const int64_t nkb = (K + kKB - 1) / kKB;
    if (tiles >= sm_count) return 1;
    return int(std::max<int64_t>(1, std::min<int64_t>({sm_count / tiles, nkb / 4, int64_t(kMaxSlices)})));
}

// Launches the kernel; with p.ks > 1 the slices of a tile are one cluster.  The slice count is
// lowered until all tiles' clusters fit on the GPU at once (clusters of CTAs that each fill an
// SM must find that many free SMs in one GPU processing cluster).
template <int WF, int AM, bool ACC = false>
wq_status launch(const TcPlan &pl, const CUtensorMap &ta, const CUtensorMap &tw, TcParams p, cudaStream_t st)
{
    auto kern = tc_gemm_kernel<WF, AM, ACC>;
    const DeviceInfo &dev = device_info();
    // per device: the configured shared-memory size, and the clusters of each size that fit
    static size_t configured[kMaxDevices];
    static int fits[kMaxDevices][kMaxSlices + 1];
    const int d = dev.device >= 0 && dev.device < kMaxDevices ? dev.device : 0;
    if (pl.smem > configured[d]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(pl.smem)) != cudaSuccess)
            return check_launch("cudaFuncSetAttribute(tc_gemm)");
        configured[d] = pl.smem;
        for (int k = 0; k <= kMaxSlices; ++k) fits[d][k] = 0;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = pl.smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    cfg.attrs = attr;
    for (; p.ks > 1; --p.ks) {
        if (fits[d][p.ks] == 0) {
            cfg.gridDim = dim3(unsigned(p.NT * p.ks));
            attr[1].val.clusterDim.x = unsigned(p.ks);
            attr[1].val.clusterDim.y = 1;
            attr[1].val.clusterDim.z = 1;
            cfg.numAttrs = 2;
            int n = 0;
            if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
                (void)cudaGetLastError();
                n = 0;
            }
            fits[d][p.ks] = n > 0 ? n : -1;
        }
        if (fits[d][p.ks] >= p.NT) break;
    }
    const int grid = p.ks > 1 ? p.NT * p.ks : std::min(dev.sm_count, p.NT);
    cfg.gridDim = dim3(unsigned(grid));
    attr[1].val.clusterDim.x = unsigned(p.ks);
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.numAttrs = p.ks > 1 ? 2 : 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, ta, tw, p);
    if (e != cudaSuccess) return fail(WQ_ERR_CUDA, "tc_gemm_kernel launch: %s", cudaGetErrorString(e));
    return check_launch("tc_gemm_kernel");
}

}  // namespace

// The tcgen05 path needs no workspace: its split-K partial sums stay in shared memory.
size_t tc_workspace_size(int64_t, int64_t, int64_t) { return 0; }

// Many-token path on the tcgen05 tensor cores: INT4, FP4 or FP8 (group size a multiple of 128),
// ternary INT2 or binary INT1 weights, FP16 / BF16 (AM 0 / 1) or INT8 (AM 2, with a_scale)
// activations (the entry points admit the pairs listed in the ABI).
// WQ_ERR_UNSUPPORTED when the configuration has no plan here (the caller then uses the
// tiled mma.sync path).
// The caller's workspace is not used (split K runs in thread-block clusters).
wq_status tc_gemm(int WF, int AM, const void *A, const float *a_scale, const uint8_t *Wq, const void *scales,
                  const void *zeros, const void *bias, void *C, int32_t *acc_out, int64_t M, int64_t N, int64_t K,
                  const wq_qconfig &c, void *, size_t, cudaStream_t st)
{
    if (acc_out && (AM != 2 || (WF == WF_I4 && c.group_size != kKB)))
        return fail(WQ_ERR_UNSUPPORTED, "tc_gemm: INT32 sums need INT8 activations (and group_size 128 for INT4)");
    if (wf_grouped(WF) && (K % kKB || c.group_size % kKB))
        return fail(WQ_ERR_UNSUPPORTED, "tc_gemm: group-scaled weights need K and group_size multiples of 128");
    if (WF == WF_I1 && K % kKB) return fail(WQ_ERR_UNSUPPORTED, "tc_gemm: INT1 needs K %% 128 == 0");
    const int es = AM >= 2 ? 1 : 2;
    if ((K * es) % 16) return fail(WQ_ERR_UNSUPPORTED, "tc_gemm: activation rows must be 16-byte multiples");
    const DeviceInfo &dev = device_info();
    const int G = wf_grouped(WF) ? int(K / c.group_size) : 0;
    const int nkb = int((K + kKB - 1) / kKB);
    const int stage = act_bytes(AM >= 2 ? 2 : 0) + w_bytes(WF);
    const TcPlan pl = make_plan(nkb, G, stage, WF == WF_I4 ? 4 : 2, dev);
    if (!pl.ok) return fail(WQ_ERR_UNSUPPORTED, "tc_gemm: no shared-memory plan for K=%lld", (long long)K);
    CUtensorMap ta, tw;
    {
        // activations [M][K]: one box = 128 tokens x 128 bytes (past K: zeros)
        const uint64_t dims[2] = {uint64_t(K), uint64_t(M)};
        const uint64_t strides[1] = {uint64_t(K) * es};
        const uint32_t box[2] = {uint32_t(128 / es), uint32_t(kBT)};
        wq_status rc = encode_tmap(&ta, es == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_UINT16, 2,
                                   A, dims, strides, box, 128);
        if (rc != WQ_OK) return rc;
    }
    {
        // packed weights [N][K*bits/8]: one box = 128 rows x one block (128 B FP8, 64 B INT4 / FP4,
        // 32 B INT2, 16 B INT1), swizzled as the unpacking warps read it
        const int blk = kKB * wf_bits(WF) / 8;
        const uint64_t row_bytes = uint64_t(K) * wf_bits(WF) / 8;
        const uint64_t dims[2] = {row_bytes, uint64_t(N)};
        const uint64_t strides[1] = {row_bytes};
        const uint32_t box[2] = {uint32_t(blk), uint32_t(kBW)};
        wq_status rc = encode_tmap(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, Wq, dims, strides, box,
                                   blk == 128 ? 128 : blk == 64 ? 64 : 0);
        if (rc != WQ_OK) return rc;
    }
    TcParams p{};
    p.M = int(M);
    p.N = int(N);
    p.K = int(K);
    p.G = G;
    p.gs = wf_grouped(WF) ? c.group_size : int(K);
    p.upg = wf_grouped(WF) ? c.group_size / kKB : 1;
    p.sym = WF == WF_I4 ? c.symmetric : 1;
    p.a_scale = a_scale;
    p.scale32 = static_cast<const float *>(scales);
    p.nkb = nkb;
    p.TT = int((M + kBT - 1) / kBT);
    p.NT = p.TT * int((N + kBW - 1) / kBW);
    p.ks = choose_slices(M, N, K, dev.sm_count);
    p.S = pl.S;
    p.scst_off = pl.scst_off;
    p.tab_off = pl.tab_off;
    p.bar_off = pl.bar_off;
    p.tab_rs = pl.tab_rs;
    p.stage_sc = pl.stage_sc;
    p.ntab = pl.ntab;
    p.scales16 = static_cast<const uint16_t *>(scales);
    p.zeros = static_cast<const uint16_t *>(zeros);
    p.bias = bias;
    p.C = C;
    p.acc_out = acc_out;
    p.nat = WF == WF_I4 && c.layout == WQ_LAYOUT_NATIVE;
    if (WF == WF_E2M1) return AM == 0 ? launch<WF_E2M1, 0>(pl, ta, tw, p, st)
                                      : fail(WQ_ERR_UNSUPPORTED, "tc_gemm: FP4 weights take FP16 activations");
    if (WF == WF_E4M3) return AM == 0   ? launch<WF_E4M3, 0>(pl, ta, tw, p, st)
                              : AM == 3 ? launch<WF_E4M3, 3>(pl, ta, tw, p, st)
                                        : fail(WQ_ERR_UNSUPPORTED, "tc_gemm: FP8 weights take FP16 or FP8 activations");
    if (WF == WF_I1) {
        if (AM == 0) return launch<WF_I1, 0>(pl, ta, tw, p, st);
        if (AM == 1) return fail(WQ_ERR_UNSUPPORTED, "tc_gemm: INT1 weights take FP16 or INT8 activations");
        return acc_out ? launch<WF_I1, 2, true>(pl, ta, tw, p, st) : launch<WF_I1, 2>(pl, ta, tw, p, st);
    }
    if (WF == WF_I4) {
        if (AM == 0) return launch<4, 0>(pl, ta, tw, p, st);
        if (AM == 1) return launch<4, 1>(pl, ta, tw, p, st);
        return acc_out ? launch<4, 2, true>(pl, ta, tw, p, st) : launch<4, 2>(pl, ta, tw, p, st);
    }
    if (AM == 0) return launch<2, 0>(pl, ta, tw, p, st);
    if (AM == 1) return launch<2, 1>(pl, ta, tw, p, st);
    return acc_out ? launch<2, 2, true>(pl, ta, tw, p, st) : launch<2, 2>(pl, ta, tw, p, st);
}

int tc_read_error()
{
    int v = 0, zero = 0;
    cudaMemcpyFromSymbol(&v, g_tc_error, sizeof v);
    cudaMemcpyToSymbol(g_tc_error, &zero, sizeof zero);
    return v;
}

}  // namespace wq
