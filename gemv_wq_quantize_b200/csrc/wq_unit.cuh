// wq_unit.cuh -- the arithmetic of one weight "unit" (16 rows x 64 packed bytes per row:
// 128 k of INT4 or FP4, 256 k of INT2, 512 k of INT1, 64 k of FP8) on mma.sync, shared by
// the few-token kernels.
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
// own order, and their B fragments need no permutation.  FP4 (e2m1) and FP8 (e4m3) codes are
// turned into exact binary16 values by the hardware conversions, pairs (k, k+1) in natural
// order; INT1 bits become +-1 (pairs (k, k+16) of a word, whose activation pairs are formed
// per word).
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include <type_traits>

#include "wq_device.cuh"
#include "wq_format.h"

namespace wq {

// activations: binary16, bfloat16, int8 codes, or e4m3 codes (FP8, with FP8 weights only)
enum AMode { A_F16 = 0, A_BF16 = 1, A_I8 = 2, A_F8 = 3 };
__host__ __device__ constexpr bool byte_acts(int AM) { return AM == A_I8 || AM == A_F8; }

// k of one unit (64 packed bytes of a row) for weight format WF
__host__ __device__ constexpr int kunit_of(int WF) { return 512 / wf_bits(WF); }
// mma k-steps per unit (k16 for f16/bf16, k32 for int8)
__host__ __device__ constexpr int steps_of(int WF, int AM) { return byte_acts(AM) ? kunit_of(WF) / 32 : kunit_of(WF) / 16; }
__host__ __device__ constexpr int qn_of(int WF, int AM) { return steps_of(WF, AM) / 2; }

// B fragments of one unit for the n8 token tile `nt`: bf[q] holds {b0, b1} of k-steps 2q
// and 2q+1.  addr(m, o) gives the shared-memory address of byte o of token m's activations
// of the unit (o < KU * element size, 16-byte chunks contiguous); tokens >= M give zeros.
// For INT8 activations `asum` receives this lane's partial sum of the token's activations
// over the unit (the quad of lanes sharing a token adds up to the token's sum).
// nat: INT4 weights in the kernel-native order (nibble i of a word = element 0,2,4,6,1,3,5,7),
// whose unpack yields the pairs (k, k+1) (FP) or the byte quads (k, k+4, k+1, k+5) (INT8).
// FP4 weights unpack to the pairs (k, k+1) like native INT4; FP8 lanes hold 16 consecutive k.
// (INT1 builds its fragments per word inside unit_mma_b1.)
template <int WF, int AM, typename Addr>
__device__ __forceinline__ void build_bfrag(Addr addr, int M, int nt, int lane, uint4 (&bf)[qn_of(WF, AM)],
                                            int &asum, bool nat = false)
{
    constexpr int QN = qn_of(WF, AM);
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
        if constexpr (AM == A_F8) {
            // e4m3 activations with e4m3 weights: k-steps 0 / 1 (k32) use bytes 16t + {0..7} / {8..15}
            // as they lie (b0 = the first 4 of each 8, b1 = the next 4)
            r = lds128(addr(m, 16 * t));
        } else if constexpr (AM != A_I8 && WF == WF_E4M3) {
            // k-steps 2q, 2q+1 use halves 16t + 8q + {0..7} as the pairs (0,1),(2,3) / (4,5),(6,7)
            r = lds128(addr(m, (16 * t + 8 * q) * 2));
        } else if constexpr (AM != A_I8 && (WF == WF_I4 || WF == WF_E2M1)) {
            // k-steps 2q, 2q+1 use halves 32t + 8q + {0..7} as pairs (0,4),(1,5) / (2,6),(3,7)
            // (native order and FP4: (0,1),(2,3) / (4,5),(6,7), the halves as they lie)
            const uint4 v = lds128(addr(m, (32 * t + 8 * q) * 2));
            if (WF == WF_E2M1 || nat) {
                r = v;
            } else {
                r.x = prmt(v.x, v.z, 0x5410);
                r.y = prmt(v.x, v.z, 0x7632);
                r.z = prmt(v.y, v.w, 0x5410);
                r.w = prmt(v.y, v.w, 0x7632);
            }
        } else if constexpr (AM != A_I8 && WF == WF_I2) {
            // k-steps 4j + 2hh (+1): pairs (i, i+8) of halves 64t + 16j + 4hh + {0..3, 8..11}
            const int j = q >> 1, hh = q & 1;
            const int o = (64 * t + 16 * j + 4 * hh) * 2;
            const uint2 lo = lds64(addr(m, o));
            const uint2 hi = lds64(addr(m, o + 16));
            r.x = prmt(lo.x, hi.x, 0x5410);
            r.y = prmt(lo.x, hi.x, 0x7632);
            r.z = prmt(lo.y, hi.y, 0x5410);
            r.w = prmt(lo.y, hi.y, 0x7632);
        } else if constexpr (WF == WF_I4) {
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

template <int WF, int AM, int NT, int NTL>
__device__ __forceinline__ void unit_mma(const uint4 (&wa)[NTL], const uint4 (&wb)[NTL],
                                         const uint4 (&bf)[NT][qn_of(WF, AM)], const uint32_t (&z_lo)[NTL],
                                         const uint32_t (&z_hi)[NTL], acc_t<AM> (&acc)[2][NTL][NT][4])
{
    if constexpr (AM == A_F8) {
        static_assert(WF == WF_E4M3, "FP8 activations take FP8 weights");
        // the weight bytes are the A fragments as they lie: k-step j uses words 2j, 2j + 1
        // (k = 16t + 8j + 0..3 and 4..7) of rows g and g + 8
#pragma unroll
        for (int j = 0; j < 2; ++j) {
#pragma unroll
            for (int l = 0; l < NTL; ++l) {
                uint32_t a[4];
                a[0] = j ? wa[l].z : wa[l].x;
                a[1] = j ? wb[l].z : wb[l].x;
                a[2] = j ? wa[l].w : wa[l].y;
                a[3] = j ? wb[l].w : wb[l].y;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
                    mma_e4m3(acc[j][l][nt], a, j ? bf[nt][0].z : bf[nt][0].x, j ? bf[nt][0].w : bf[nt][0].y);
            }
        }
    } else if constexpr (AM == A_F16 && WF == WF_E2M1) {
        // byte b of word j -> the exact binary16 pair (8j + 2b, 8j + 2b + 1); no zero point
#pragma unroll
        for (int j = 0; j < 4; ++j) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
#pragma unroll
                for (int l = 0; l < NTL; ++l) {
                    const uint32_t wl = j == 0 ? wa[l].x : j == 1 ? wa[l].y : j == 2 ? wa[l].z : wa[l].w;
                    const uint32_t wh = j == 0 ? wb[l].x : j == 1 ? wb[l].y : j == 2 ? wb[l].z : wb[l].w;
                    uint32_t a[4];
                    if (h == 0) {
                        a[0] = e2m1x2_to_f16x2<0>(wl);
                        a[1] = e2m1x2_to_f16x2<0>(wh);
                        a[2] = e2m1x2_to_f16x2<1>(wl);
                        a[3] = e2m1x2_to_f16x2<1>(wh);
                    } else {
                        a[0] = e2m1x2_to_f16x2<2>(wl);
                        a[1] = e2m1x2_to_f16x2<2>(wh);
                        a[2] = e2m1x2_to_f16x2<3>(wl);
                        a[3] = e2m1x2_to_f16x2<3>(wh);
                    }
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
                        mma_f16(acc[(j & 1)][l][nt], a, h ? bf[nt][j].z : bf[nt][j].x, h ? bf[nt][j].w : bf[nt][j].y);
                }
            }
        }
    } else if constexpr (AM == A_F16 && WF == WF_E4M3) {
        // word j holds k = 16t + 4j .. 4j + 3: halves 0 / 1 -> the exact binary16 pairs (4j, 4j+1) /
        // (4j+2, 4j+3) of k-step j
#pragma unroll
        for (int j = 0; j < 4; ++j) {
#pragma unroll
            for (int l = 0; l < NTL; ++l) {
                const uint32_t wl = j == 0 ? wa[l].x : j == 1 ? wa[l].y : j == 2 ? wa[l].z : wa[l].w;
                const uint32_t wh = j == 0 ? wb[l].x : j == 1 ? wb[l].y : j == 2 ? wb[l].z : wb[l].w;
                uint32_t a[4];
                a[0] = e4m3x2_to_f16x2<0>(wl);
                a[1] = e4m3x2_to_f16x2<0>(wh);
                a[2] = e4m3x2_to_f16x2<1>(wl);
                a[3] = e4m3x2_to_f16x2<1>(wh);
                const int q = j >> 1;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
                    mma_f16(acc[(j & 1)][l][nt], a, (j & 1) ? bf[nt][q].z : bf[nt][q].x,
                            (j & 1) ? bf[nt][q].w : bf[nt][q].y);
            }
        }
    } else if constexpr (AM == A_F16 && WF == WF_I4) {
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
    } else if constexpr (AM == A_BF16 && WF == WF_I4) {
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
    } else if constexpr (AM != A_I8 && WF == WF_I2) {
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
    } else if constexpr (AM == A_I8 && WF == WF_I4) {
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

// INT1 (binary) weights, one unit = 512 k: lane t holds k = 128t .. 128t + 127 of each of its
// two rows as four words, bit i of word j being k = 128t + 32j + i (value 2c - 1).
//  FP16 activations: k-step s of word j pairs (2s, 2s+16) and (2s+1, 2s+17), so one shift and
//  one LOP3 give each +-1 pair, and the activation pairs are formed from the word's 32 halves
//  by one byte permute each.
//  INT8 activations: (w >> i) & 0x01010101 gives the quad (i, i+8, i+16, i+24) of bits, made
//  signed bytes +-1; k-step s of word j uses quads 2s and 2s+1, the activation quads likewise.
// addr(m, o): byte o of token m's activations of the unit; tokens >= M give zeros.
template <int AM, int NT, int NTL, typename Addr>
__device__ __forceinline__ void unit_mma_b1(const uint4 (&wa)[NTL], const uint4 (&wb)[NTL], Addr addr, int M,
                                            int lane, acc_t<AM> (&acc)[2][NTL][NT][4])
{
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        if constexpr (AM == A_F16) {
            uint32_t R[NT][16];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int m = nt * 8 + g;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint4 v = m < M ? lds128(addr(m, (128 * t + 32 * j) * 2 + 16 * i)) : make_uint4(0, 0, 0, 0);
                    R[nt][4 * i + 0] = v.x;
                    R[nt][4 * i + 1] = v.y;
                    R[nt][4 * i + 2] = v.z;
                    R[nt][4 * i + 3] = v.w;
                }
            }
#pragma unroll
            for (int s2 = 0; s2 < 8; ++s2) {
                uint32_t b0[NT], b1[NT];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    b0[nt] = prmt(R[nt][s2], R[nt][s2 + 8], 0x5410);  // halves 2s, 2s + 16
                    b1[nt] = prmt(R[nt][s2], R[nt][s2 + 8], 0x7632);  // halves 2s + 1, 2s + 17
                }
#pragma unroll
                for (int l = 0; l < NTL; ++l) {
                    const uint32_t wl = j == 0 ? wa[l].x : j == 1 ? wa[l].y : j == 2 ? wa[l].z : wa[l].w;
                    const uint32_t wh = j == 0 ? wb[l].x : j == 1 ? wb[l].y : j == 2 ? wb[l].z : wb[l].w;
                    uint32_t a[4];
                    a[0] = pm1_f16x2(wl << (15 - 2 * s2));
                    a[1] = pm1_f16x2(wh << (15 - 2 * s2));
                    a[2] = pm1_f16x2(wl << (14 - 2 * s2));
                    a[3] = pm1_f16x2(wh << (14 - 2 * s2));
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) mma_f16(acc[s2 & 1][l][nt], a, b0[nt], b1[nt]);
                }
            }
        } else {
            static_assert(AM == A_I8, "INT1 weights take FP16 or INT8 activations");
            uint32_t R[NT][8];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int m = nt * 8 + g;
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const uint4 v = m < M ? lds128(addr(m, 128 * t + 32 * j + 16 * i)) : make_uint4(0, 0, 0, 0);
                    R[nt][4 * i + 0] = v.x;
                    R[nt][4 * i + 1] = v.y;
                    R[nt][4 * i + 2] = v.z;
                    R[nt][4 * i + 3] = v.w;
                }
            }
#pragma unroll
            for (int a2 = 0; a2 < 2; ++a2) {
                uint32_t E0[NT], E1[NT], O0[NT], O1[NT];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    E0[nt] = prmt(R[nt][a2], R[nt][a2 + 2], 0x6420);
                    E1[nt] = prmt(R[nt][a2 + 4], R[nt][a2 + 6], 0x6420);
                    O0[nt] = prmt(R[nt][a2], R[nt][a2 + 2], 0x7531);
                    O1[nt] = prmt(R[nt][a2 + 4], R[nt][a2 + 6], 0x7531);
                }
#pragma unroll
                for (int hs = 0; hs < 2; ++hs) {
                    const int s2 = 2 * a2 + hs;  // activation bytes 2s + 8u (b0) and 2s + 1 + 8u (b1)
                    uint32_t b0[NT], b1[NT];
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        b0[nt] = prmt(E0[nt], E1[nt], hs ? 0x7531 : 0x6420);
                        b1[nt] = prmt(O0[nt], O1[nt], hs ? 0x7531 : 0x6420);
                    }
#pragma unroll
                    for (int l = 0; l < NTL; ++l) {
                        const uint32_t wl = j == 0 ? wa[l].x : j == 1 ? wa[l].y : j == 2 ? wa[l].z : wa[l].w;
                        const uint32_t wh = j == 0 ? wb[l].x : j == 1 ? wb[l].y : j == 2 ? wb[l].z : wb[l].w;
                        // bits -> bytes 0 / 1 -> 2c + 0x7F -> ^0x80: signed bytes -1 / +1 (no carries)
                        uint32_t a[4];
                        a[0] = ((((wl >> (2 * s2)) & 0x01010101u) << 1) + 0x7F7F7F7Fu) ^ 0x80808080u;
                        a[1] = ((((wh >> (2 * s2)) & 0x01010101u) << 1) + 0x7F7F7F7Fu) ^ 0x80808080u;
                        a[2] = ((((wl >> (2 * s2 + 1)) & 0x01010101u) << 1) + 0x7F7F7F7Fu) ^ 0x80808080u;
                        a[3] = ((((wh >> (2 * s2 + 1)) & 0x01010101u) << 1) + 0x7F7F7F7Fu) ^ 0x80808080u;
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) mma_s8s8(acc[s2 & 1][l][nt], a, b0[nt], b1[nt]);
                    }
                }
            }
        }
    }
}

}  // namespace wq
