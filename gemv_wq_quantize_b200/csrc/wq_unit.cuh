// wq_unit.cuh -- the arithmetic of one weight "unit" (16 rows x 64 packed bytes per row:
// 128 k of INT4 or 256 k of INT2) on mma.sync, shared by the few-token kernels.
//
// Exactness: weights enter the tensor cores as the integers q - z (|q - z| <= 15), which
// f16, bf16 and int8 represent exactly, so every product is exact; FP paths accumulate in
// fp32 and apply the group scale once per group, INT8 paths accumulate exactly in int32.
//
// k order: the nibble unpack of a 32-bit word naturally yields pairs (k, k+4) of INT4
// (pairs (k, k+8) of INT2; byte quads (k, k+2, k+4, k+6) for INT8 activations).  Since
// an MMA sums over k, the activations (B operand) are loaded in the same permuted order,
// so the weights are used straight from the packed layout with no reordering.  INT4 weights
// in the kernel-native order (see wq_repack) unpack to pairs (k, k+1), the activations'
// own order, and their B fragments need no permutation.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include <type_traits>

#include "wq_device.cuh"

namespace wq {

enum AMode { A_F16 = 0, A_BF16 = 1, A_I8 = 2 };

__host__ __device__ constexpr int kunit_of(int WB) { return WB == 4 ? 128 : 256; }
// mma k-steps per unit (k16 for f16/bf16, k32 for int8)
__host__ __device__ constexpr int steps_of(int WB, int AM)
{
    return AM == A_I8 ? (WB == 4 ? 4 : 8) : (WB == 4 ? 8 : 16);
}
__host__ __device__ constexpr int qn_of(int WB, int AM) { return steps_of(WB, AM) / 2; }

// B fragments of one unit for the n8 token tile `nt`: bf[q] holds {b0, b1} of k-steps 2q
// and 2q+1.  addr(m, o) gives the shared-memory address of byte o of token m's activations
// of the unit (o < KU * element size, 16-byte chunks contiguous); tokens >= M give zeros.
// For INT8 activations `asum` receives this lane's partial sum of the token's activations
// over the unit (the quad of lanes sharing a token adds up to the token's sum).
// nat: INT4 weights in the kernel-native order (nibble i of a word = element 0,2,4,6,1,3,5,7),
// whose unpack yields the pairs (k, k+1) (FP) or the byte quads (k, k+4, k+1, k+5) (INT8).
template <int WB, int AM, typename Addr>
__device__ __forceinline__ void build_bfrag(Addr addr, int M, int nt, int lane, uint4 (&bf)[qn_of(WB, AM)],
                                            int &asum, bool nat = false)
{
    constexpr int QN = qn_of(WB, AM);
    const int g = lane >> 2, t = lane & 3;
    const int m = nt * 8 + g;
    asum = 0;
    if (m >= M) {
#pragma unroll
        for (int q = 0; q < QN; ++q) bf[q] = make_uint4(0, 0, 0, 0);
        return;
    }
#pragma unroll
    for (int q = 0; q < QN; ++q) {
        uint4 r;
        if constexpr (AM != A_I8 && WB == 4) {
            // k-steps 2q, 2q+1 use halves 32t + 8q + {0..7} as pairs (0,4),(1,5) / (2,6),(3,7)
            // (native order: (0,1),(2,3) / (4,5),(6,7), the halves as they lie)
            const uint4 v = lds128(addr(m, (32 * t + 8 * q) * 2));
            if (nat) {
                r = v;
            } else {
                r.x = prmt(v.x, v.z, 0x5410);
                r.y = prmt(v.x, v.z, 0x7632);
                r.z = prmt(v.y, v.w, 0x5410);
                r.w = prmt(v.y, v.w, 0x7632);
            }
        } else if constexpr (AM != A_I8 && WB == 2) {
            // k-steps 4j + 2hh (+1): pairs (i, i+8) of halves 64t + 16j + 4hh + {0..3, 8..11}
            const int j = q >> 1, hh = q & 1;
            const int o = (64 * t + 16 * j + 4 * hh) * 2;
            const uint2 lo = lds64(addr(m, o));
            const uint2 hi = lds64(addr(m, o + 16));
            r.x = prmt(lo.x, hi.x, 0x5410);
            r.y = prmt(lo.x, hi.x, 0x7632);
            r.z = prmt(lo.y, hi.y, 0x5410);
            r.w = prmt(lo.y, hi.y, 0x7632);
        } else if constexpr (WB == 4) {
            // k-steps 2q, 2q+1 (k32): bytes 32t + 16q + {0..15} as quads (0,2,4,6),(1,3,5,7)
            // (native order: (0,4,1,5),(2,6,3,7))
            const uint4 v = lds128(addr(m, 32 * t + 16 * q));
            const uint32_t s0 = nat ? 0x5140u : 0x6420u, s1 = nat ? 0x7362u : 0x7531u;
            r.x = prmt(v.x, v.y, s0);
            r.y = prmt(v.x, v.y, s1);
            r.z = prmt(v.z, v.w, s0);
            r.w = prmt(v.z, v.w, s1);
            asum = __dp4a(int(v.x), 0x01010101, asum);
            asum = __dp4a(int(v.y), 0x01010101, asum);
            asum = __dp4a(int(v.z), 0x01010101, asum);
            asum = __dp4a(int(v.w), 0x01010101, asum);
        } else {
            // k-steps 2q, 2q+1 (k32): bytes 64t + 16q + {0..15} as quads (i, i+4, i+8, i+12)
            const uint4 v = lds128(addr(m, 64 * t + 16 * q));
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
        bf[q] = r;
    }
}

// Multiply one unit of NTL tiles at once (their MMA chains are independent, which keeps
// the tensor pipe busy): wa[l] / wb[l] are this lane's 16 packed bytes of rows g and g+8
// of tile l (bytes 16t .. 16t+15 of the unit's 64), bf the B fragments of NT token tiles.
// The k-steps alternate between two accumulator sets acc[0] / acc[1] (two independent MMA
// chains per tile); the caller adds them.
// FP activations: acc[.][l][nt] += sum over the unit of A * (q - z) (z_lo / z_hi: integer
// zero points 0..15 of rows g / g+8; 8 for symmetric INT4; ignored for INT2, whose value is
// the 2-bit code).  INT8 activations: acc[.][l][nt] += sum of Aq * field, with the unsigned
// field (nibble for INT4, code ^ 2 for INT2); the caller subtracts z * sum(Aq) (2 * sum(Aq)
// for INT2).
template <int AM>
using acc_t = typename std::conditional<AM == A_I8, int, float>::type;

template <int WB, int AM, int NT, int NTL>
__device__ __forceinline__ void unit_mma(const uint4 (&wa)[NTL], const uint4 (&wb)[NTL],
                                         const uint4 (&bf)[NT][qn_of(WB, AM)], const uint32_t (&z_lo)[NTL],
                                         const uint32_t (&z_hi)[NTL], acc_t<AM> (&acc)[2][NTL][NT][4])
{
    if constexpr (AM == A_F16 && WB == 4) {
        // x = 1024 + nibble (low nibbles) or 1024 + 16 * nibble (high nibbles), made the
        // exact integer q - z by one half2 add / fma
        uint32_t clo0[NTL], clo1[NTL], chi0[NTL], chi1[NTL];
#pragma unroll
        for (int l = 0; l < NTL; ++l) {
            const uint32_t a0 = 0xE400u | z_lo[l], a1 = 0xE400u | z_hi[l];                // -(1024 + z)
            const uint32_t b0 = 0xD400u | (z_lo[l] << 4), b1 = 0xD400u | (z_hi[l] << 4);  // -(64 + z)
            clo0[l] = a0 | (a0 << 16);
            clo1[l] = a1 | (a1 << 16);
            chi0[l] = b0 | (b0 << 16);
            chi1[l] = b1 | (b1 << 16);
        }
        const uint32_t sixteenth = 0x2C002C00u;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
#pragma unroll
                for (int l = 0; l < NTL; ++l) {
                    const uint32_t wl = j == 0 ? wa[l].x : j == 1 ? wa[l].y : j == 2 ? wa[l].z : wa[l].w;
                    const uint32_t wh = j == 0 ? wb[l].x : j == 1 ? wb[l].y : j == 2 ? wb[l].z : wb[l].w;
                    const uint32_t x0 = h ? (wl >> 8) : wl;
                    const uint32_t x1 = h ? (wh >> 8) : wh;
                    uint32_t a[4];
                    a[0] = h2_add(and_or(x0, 0x000f000fu, 0x64006400u), clo0[l]);
                    a[1] = h2_add(and_or(x1, 0x000f000fu, 0x64006400u), clo1[l]);
                    a[2] = h2_fma(and_or(x0, 0x00f000f0u, 0x64006400u), sixteenth, chi0[l]);
                    a[3] = h2_fma(and_or(x1, 0x00f000f0u, 0x64006400u), sixteenth, chi1[l]);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
                        mma_f16(acc[(j & 1)][l][nt], a, h ? bf[nt][j].z : bf[nt][j].x, h ? bf[nt][j].w : bf[nt][j].y);
                }
            }
        }
    } else if constexpr (AM == A_BF16 && WB == 4) {
        // x = 128 + nibble in bf16 (shifted nibbles), minus 128 + z
        uint32_t cc0[NTL], cc1[NTL];
#pragma unroll
        for (int l = 0; l < NTL; ++l) {
            const uint32_t c0 = 0xC300u | z_lo[l], c1 = 0xC300u | z_hi[l];  // -(128 + z) in bf16
            cc0[l] = c0 | (c0 << 16);
            cc1[l] = c1 | (c1 << 16);
        }
        const uint32_t one = 0x3F803F80u;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
#pragma unroll
                for (int l = 0; l < NTL; ++l) {
                    const uint32_t wl = j == 0 ? wa[l].x : j == 1 ? wa[l].y : j == 2 ? wa[l].z : wa[l].w;
                    const uint32_t wh = j == 0 ? wb[l].x : j == 1 ? wb[l].y : j == 2 ? wb[l].z : wb[l].w;
                    uint32_t a[4];
                    a[0] = bf2_fma(and_or(wl >> (8 * h), 0x000f000fu, 0x43004300u), one, cc0[l]);
                    a[1] = bf2_fma(and_or(wh >> (8 * h), 0x000f000fu, 0x43004300u), one, cc1[l]);
                    a[2] = bf2_fma(and_or(wl >> (8 * h + 4), 0x000f000fu, 0x43004300u), one, cc0[l]);
                    a[3] = bf2_fma(and_or(wh >> (8 * h + 4), 0x000f000fu, 0x43004300u), one, cc1[l]);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
                        mma_bf16(acc[(j & 1)][l][nt], a, h ? bf[nt][j].z : bf[nt][j].x, h ? bf[nt][j].w : bf[nt][j].y);
                }
            }
        }
    } else if constexpr (AM != A_I8 && WB == 2) {
        // 2-bit field f, c' = f ^ 2 in [0,3], value c' - 2.  Field pairs (i, i+8) of a word.
#pragma unroll
        for (int j = 0; j < 4; ++j) {
#pragma unroll
            for (int h = 0; h < 4; ++h) {
#pragma unroll
                for (int l = 0; l < NTL; ++l) {
                    const uint32_t wl = j == 0 ? wa[l].x : j == 1 ? wa[l].y : j == 2 ? wa[l].z : wa[l].w;
                    const uint32_t wh = j == 0 ? wb[l].x : j == 1 ? wb[l].y : j == 2 ? wb[l].z : wb[l].w;
                    const uint32_t y0 = wl ^ 0xAAAAAAAAu, y1 = wh ^ 0xAAAAAAAAu;
                    const int i0 = 2 * h, i1 = 2 * h + 1;
                    uint32_t a[4];
                    if constexpr (AM == A_F16) {
                        // (f << 2s) | 0x6400 = 1024 + 4^s c'; times 4^-s, minus 1024 * 4^-s + 2
                        const int sh0 = (i0 & 3) * 2, sh1 = (i1 & 3) * 2;
                        const int s0 = (i0 >= 4) ? 8 : 0;
                        const uint32_t m0 = 0x00030003u << sh0, m1 = 0x00030003u << sh1;
                        constexpr uint32_t kMul[4] = {0x3C003C00u, 0x34003400u, 0x2C002C00u, 0x24002400u};
                        constexpr uint32_t kAdd[4] = {0xE402E402u, 0xDC08DC08u, 0xD420D420u, 0xCC80CC80u};
                        a[0] = h2_fma(and_or(y0 >> s0, m0, 0x64006400u), kMul[sh0 / 2], kAdd[sh0 / 2]);
                        a[1] = h2_fma(and_or(y1 >> s0, m0, 0x64006400u), kMul[sh0 / 2], kAdd[sh0 / 2]);
                        a[2] = h2_fma(and_or(y0 >> s0, m1, 0x64006400u), kMul[sh1 / 2], kAdd[sh1 / 2]);
                        a[3] = h2_fma(and_or(y1 >> s0, m1, 0x64006400u), kMul[sh1 / 2], kAdd[sh1 / 2]);
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
                        const uint32_t b0 = (h & 1) ? bf[nt][q].z : bf[nt][q].x;
                        const uint32_t b1 = (h & 1) ? bf[nt][q].w : bf[nt][q].y;
                        if constexpr (AM == A_F16) mma_f16(acc[(h & 1)][l][nt], a, b0, b1);
                        else mma_bf16(acc[(h & 1)][l][nt], a, b0, b1);
                    }
                }
            }
        }
    } else if constexpr (AM == A_I8 && WB == 4) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
#pragma unroll
            for (int l = 0; l < NTL; ++l) {
                const uint32_t wl = j == 0 ? wa[l].x : j == 1 ? wa[l].y : j == 2 ? wa[l].z : wa[l].w;
                const uint32_t wh = j == 0 ? wb[l].x : j == 1 ? wb[l].y : j == 2 ? wb[l].z : wb[l].w;
                uint32_t a[4];
                a[0] = wl & 0x0f0f0f0fu;
                a[1] = wh & 0x0f0f0f0fu;
                a[2] = (wl >> 4) & 0x0f0f0f0fu;
                a[3] = (wh >> 4) & 0x0f0f0f0fu;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
                    mma_u8s8(acc[(j & 1)][l][nt], a, (j & 1) ? bf[nt][j >> 1].z : bf[nt][j >> 1].x,
                         (j & 1) ? bf[nt][j >> 1].w : bf[nt][j >> 1].y);
            }
        }
    } else {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
#pragma unroll
                for (int l = 0; l < NTL; ++l) {
                    const uint32_t wl = j == 0 ? wa[l].x : j == 1 ? wa[l].y : j == 2 ? wa[l].z : wa[l].w;
                    const uint32_t wh = j == 0 ? wb[l].x : j == 1 ? wb[l].y : j == 2 ? wb[l].z : wb[l].w;
                    const uint32_t y0 = wl ^ 0xAAAAAAAAu, y1 = wh ^ 0xAAAAAAAAu;
                    uint32_t a[4];
                    a[0] = (y0 >> (4 * h)) & 0x03030303u;
                    a[1] = (y1 >> (4 * h)) & 0x03030303u;
                    a[2] = (y0 >> (4 * h + 2)) & 0x03030303u;
                    a[3] = (y1 >> (4 * h + 2)) & 0x03030303u;
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
                        mma_u8s8(acc[h][l][nt], a, h ? bf[nt][j].z : bf[nt][j].x, h ? bf[nt][j].w : bf[nt][j].y);
                }
            }
        }
    }
}

}  // namespace wq
