/*
 * wq.h -- C ABI of libwq: INT4 / INT2 / INT1 / FP4 / FP8 weight-quantized matmul on NVIDIA
 * B200 (sm_100a).
 *
 * The operation (statement of the problem in "BitBLAS practical guide: mixed-precision
 * compute in vLLM" (mlqm), section "What is BitBLAS"):
 *
 *     C[M,N] = A[M,K] x dequant(Wq[N,K])^T          (layout "nt": A and W both K-contiguous,
 *                                                    section "Advanced features 1")
 *
 * with packed low-bit weights Wq, per-group scales and optional zero points
 * (section "Advanced features 2, weight group quantization": group_size 128, with_scaling,
 * with_zeros, zeros_mode "original"), in two activation paths:
 *
 *   W4A16  FP16 / BF16 activations; weights dequantized in registers; FP32 accumulation.
 *   W4A8   per-token INT8 activations ("Accelerating LLM inference with CUDA Graph and INT4
 *          quantization" (cnblogs), part 1, step 2); exact INT32 accumulation of integer
 *          dot products (step 3, the DP4A definition c += a0*b0 + ... + a3*b3); then the
 *          float dequantization by weight_scale x activation_scale and an optional bias
 *          (steps 3-4).
 *
 * and the same two paths for ternary / INT2 weights with one scale per tensor
 * (BitBLAS guide, "Core advantages 2" FP16xINT2 and INT8xINT2, "Real-world case"
 * BitNet-b1.58).  The other weight types of the guide's "Main features" list:
 *   FP16 x FP4 (e2m1) and FP16 x FP8 (e4m3) with group scales (W4A16 path only), and
 *   FP16 x INT1 / INT8 x INT1 (binary weights, one scale per tensor; both paths), and the
 *   table's FP8_E4M3 x FP8_E4M3 row (FP8 activations per token, FP8 weights; w8a8_fp8_gemm).
 *
 * Data formats (fixed):
 *   - all matrices row-major; A [M,K], W [N,K], C [M,N];
 *   - INT4: byte j of a row holds element 2j in bits 0..3 and element 2j+1 in bits 4..7;
 *     symmetric weights store q + 8 (q in [-7,7]); asymmetric weights store q in [0,15]
 *     and dequantize as (q - z) * s;
 *   - INT2 (ternary): element 4j+i in bits 2i..2i+1 of byte j, 2-bit two's complement;
 *   - INT1 (binary): element 8j+i in bit i of byte j; bit c stands for the value 2c - 1;
 *   - FP4: e2m1 codes (bit 3 sign, bits 2..1 exponent with bias 1, bit 0 mantissa: values
 *     0, 0.5, 1, 1.5, 2, 3, 4, 6 and negatives), packed two per byte as INT4;
 *   - FP8: e4m3 codes (sign, 4 exponent bits with bias 7, 3 mantissa bits, largest finite
 *     448, no infinities), one per byte;
 *   - scales / zeros: binary16 [N, K/group_size] row-major (INT4, FP4, FP8); one binary32
 *     (INT2, INT1).
 *
 * Quantization readings (the pages print an INT8 range inside the INT4 passage):
 *   symmetric  s = fp16(absmax/7), q = clip(rint(w/s), -7, 7);
 *   asymmetric s = fp16((max(w,0) - min(w,0))/15), z = clip(rint(-min/s), 0, 15),
 *              q = clip(rint(w/s) + z, 0, 15);
 *   ternary    s = mean|w| (exact sum rounded once to binary64, / count, -> binary32),
 *              q = clip(rint(w/s), -1, 1);
 *   binary     s = mean|w| as for ternary, c = (w >= 0) (so -0 and +0 give 1);
 *   FP4 / FP8  s = fp16(absmax/6) / fp16(absmax/448), code = the format's value nearest to
 *              clip(w/s, -max, max), ties to the even last mantissa bit, +0 for a zero result;
 *   activations a_scale[m] = absmax_k|A[m,k]| / 127 (binary32), Aq = clip(rint(A/a_scale), -127, 127).
 * rint is round-half-to-even; divisions are IEEE binary32 divisions; the stored binary16 scale
 * is the one used to quantize.  Scale 0 gives code 0.
 *
 * Conventions for every entry point:
 *   - Pointers named W, A, Aq, a_scale, Wq, scales, zeros, bias, C, acc_out, q, workspace are
 *     DEVICE pointers owned by the caller; the library never allocates, frees or keeps them.
 *   - Every call is asynchronous on `stream` (0 = legacy default stream): it validates its
 *     arguments on the host, enqueues its kernels and returns.  No call synchronizes.
 *   - Argument errors return before anything is enqueued: WQ_ERR_INVALID_ARG (bad sizes,
 *     null required pointer, unsupported combination of flags), WQ_ERR_ALIGNMENT (a device
 *     pointer not 16-byte aligned), WQ_ERR_UNSUPPORTED (a valid request this build does not
 *     implement, e.g. a group size that is not a multiple of 128).  A failed launch returns
 *     WQ_ERR_CUDA.  wq_last_error() gives a one-line reason for the calling thread.
 *   - Nothing traps on the device.
 */
#ifndef WQ_H
#define WQ_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    WQ_OK = 0,
    WQ_ERR_INVALID_ARG = 1,
    WQ_ERR_ALIGNMENT = 2,
    WQ_ERR_UNSUPPORTED = 3,
    WQ_ERR_CUDA = 4,
    WQ_ERR_WORKSPACE = 5
} wq_status;

typedef enum { WQ_F32 = 0, WQ_F16 = 1, WQ_BF16 = 2, WQ_I8 = 3, WQ_I32 = 4 } wq_dtype;

typedef struct {
    int32_t bits;        /* WQ_FMT_INT: 4 (INT4), 2 (INT2 / ternary) or 1 (INT1 / binary);   */
                         /* WQ_FMT_E2M1: 4; WQ_FMT_E4M3: 8.                                  */
    int32_t group_size;  /* INT4, FP4, FP8: elements of K per scale, a multiple of 128        */
                         /*       dividing K; K itself means one scale per output channel.  */
                         /* INT2, INT1: ignored (one scale per tensor).                    */
    int32_t symmetric;   /* INT4: 1 = symmetric (q + 8 stored, no zeros), 0 = zero points.  */
                         /* Ignored for the other types (no zero points).                  */
    int32_t ternary;     /* INT2: must be 1 (codes -1, 0, 1 from the ternary quantizer).    */
    int32_t layout;      /* INT4 only: WQ_LAYOUT_NT (0), the packing described above, or     */
                         /* WQ_LAYOUT_NATIVE (1), the order written by wq_repack.           */
    int32_t format;      /* WQ_FMT_INT (0), WQ_FMT_E2M1 (1) or WQ_FMT_E4M3 (2).             */
} wq_qconfig;

#define WQ_LAYOUT_NT 0
#define WQ_LAYOUT_NATIVE 1
#define WQ_FMT_INT 0
#define WQ_FMT_E2M1 1
#define WQ_FMT_E4M3 2

/* Weight quantization and packing ("Accelerating LLM inference with CUDA Graph and INT4
 * quantization", part 1, step 1; BitBLAS guide, "Advanced features 2").
 *   W       [N,K] device, dtype w_dt in {WQ_F32, WQ_F16, WQ_BF16}.
 *   Wq      [N, K*bits/8] bytes, device, written.
 *   scales  INT4, FP4, FP8: binary16 [N, K/group_size]; INT2, INT1: one binary32. Written.
 *   zeros   INT4 asymmetric: binary16 [N, K/group_size] (integers 0..15), written; else NULL.
 *   workspace / ws_bytes: scratch for the INT2 / INT1 per-tensor mean
 *   (wq_quantize_workspace_size bytes); unused otherwise (may be NULL).
 * Requires K % group_size == 0 (INT4, FP4, FP8), K % 64 == 0 (INT2) or K % 128 == 0 (INT1),
 * N >= 1, K >= 1.  Bit-exact with the CPU reference of the same readings. */
wq_status wq_quantize_pack(const void *W, wq_dtype w_dt, int64_t N, int64_t K, wq_qconfig c,
                           uint8_t *Wq, void *scales, void *zeros,
                           void *workspace, size_t ws_bytes, cudaStream_t stream);
size_t wq_quantize_workspace_size(int64_t N, int64_t K, wq_qconfig c);

/* Kernel-native weight layout ("BitBLAS practical guide", "use the BitBLAS compressed format":
 * weights stored offline in the order the kernels consume them).  Within every 32-bit word
 * (8 codes of k = 8j .. 8j+7), nibble i holds element 8j + p(i) with p = 0, 2, 4, 6, 1, 3, 5, 7,
 * so that masking the word with 0x000F000F / 0x00F000F0 yields the half pairs (k, k+1) in
 * natural order (one LOP3 per pair in the tensor-core unpack, and activation fragments that
 * need no byte permutation).  Scales and zero points are unchanged.
 *   Wq [N, K/2] INT4 in WQ_LAYOUT_NT (c.layout 0); Wq_native [N, K/2] written (may equal Wq).
 *   Matmuls given c.layout = WQ_LAYOUT_NATIVE read it.  Their results are bit-identical to the
 *   "nt" call on the INT8 paths (exact sums) and above 16 tokens (the tensor-core unpack yields
 *   the same values in the same order); up to 16 tokens on the FP path each MMA step sums a
 *   different grouping of k, so results agree within the FP accuracy bar, not bit for bit.
 * INT4 only (WQ_ERR_UNSUPPORTED for INT2); K % 8 == 0. */
wq_status wq_repack(const uint8_t *Wq, int64_t N, int64_t K, wq_qconfig c, uint8_t *Wq_native,
                    cudaStream_t stream);

/* Inverse of the packing: signed codes q [N,K] int8 (symmetric INT4: nibble - 8; asymmetric
 * INT4: nibble; INT2: two's complement; INT1: 2c - 1), or for FP4 / FP8 the raw e2m1 / e4m3
 * code of every element (one per byte).  For tests and debugging ("Accelerating LLM
 * inference...", part 1, step 3: unpack each byte into two INT4 values). */
wq_status wq_unpack(const uint8_t *Wq, int64_t N, int64_t K, wq_qconfig c, int8_t *q,
                    cudaStream_t stream);

/* Per-token dynamic INT8 activation quantization ("Accelerating LLM inference...", part 1,
 * step 2).  A [M,K] binary16 or bfloat16 (a_dt); Aq [M,K] int8 and a_scale [M] binary32
 * written.  K % 8 == 0.  Bit-exact with the CPU reference. */
wq_status act_quant_int8(const void *A, wq_dtype a_dt, int64_t M, int64_t K,
                         int8_t *Aq, float *a_scale, cudaStream_t stream);

/* W4A16 (and W2A16, W1A16, FP4 / FP8 weights):
 *     C[m,n] = sum_k A[m,k] * (q[n,k] - z[n,g]) * s[n,g]  (+ bias[n]),
 * with (q - z) the code's value for FP4 / FP8 and 2c - 1 for INT1, accumulated in binary32
 * and rounded once to a_dt.
 *   A      [M,K] a_dt in {WQ_F16, WQ_BF16} (INT4, INT2); WQ_F16 only for INT1, FP4 and FP8
 *          (the pairs of the BitBLAS guide's list; WQ_ERR_UNSUPPORTED otherwise);
 *          C [M,N] a_dt;  bias [N] a_dt or NULL.
 *   Wq, scales, zeros as written by wq_quantize_pack (zeros NULL unless asymmetric INT4).
 *   workspace: device scratch of at least wq_workspace_size(M,N,K,c) bytes, ZERO-FILLED
 *   once before its first use.  Only the tiled mma.sync path (INT4 / INT2 shapes that the
 *   tensor-core kernel has no plan for) uses it: split-K partial sums (overwritten by every
 *   call) and arrival counters that every call leaves at zero again, so it can be reused
 *   by later calls of any shape without clearing.  The few-token kernel and the tensor-core
 *   kernel (whose split-K partial sums stay in the shared memory of a thread-block cluster)
 *   need none.  A workspace that is NULL or too small is allowed: the call then uses a
 *   launch plan that needs none (possibly slower).  Calls that share one workspace must not
 *   overlap on the GPU.
 * Requires K % 128 == 0 for INT4, FP4, FP8 and INT1 (K % 64 == 0 for INT2), M, N >= 1.
 * Above 16 tokens INT1, FP4 and FP8 need K >= 512 (the tensor-core kernel's shortest K);
 * shorter K gives WQ_ERR_UNSUPPORTED. */
wq_status w4a16_gemm(const void *A, wq_dtype a_dt, const uint8_t *Wq, const void *scales,
                     const void *zeros, const void *bias, void *C,
                     int64_t M, int64_t N, int64_t K, wq_qconfig c,
                     void *workspace, size_t ws_bytes, cudaStream_t stream);

/* W4A8 (and W2A8, W1A8):
 *   acc_g[m,n] = sum_{k in group g} Aq[m,k] * (q[n,k] - z[n,g])        exact INT32
 *   C[m,n]     = fp16( a_scale[m] * sum_g s[n,g] * acc_g[m,n]  (+ bias[n]) )
 * INT2 and INT1 weights have a single group spanning K and a single binary32 scale; FP4 and
 * FP8 weights are not in this path (WQ_ERR_UNSUPPORTED).
 *   Aq [M,K] int8, a_scale [M] binary32 (from act_quant_int8); C [M,N] binary16;
 *   bias [N] binary16 or NULL; zeros (asymmetric INT4) must hold integers.
 *   acc_out: NULL, or int32 [M, N, G] receiving every acc_g (G = K/128 for INT4, which
 *   then requires group_size == 128; G = 1 for INT2 and INT1), bit-exact with the CPU
 *   reference.
 *   workspace: as for w4a16_gemm. */
wq_status w4a8_gemm(const int8_t *Aq, const float *a_scale, const uint8_t *Wq, const void *scales,
                    const void *zeros, const void *bias, void *C, int32_t *acc_out,
                    int64_t M, int64_t N, int64_t K, wq_qconfig c,
                    void *workspace, size_t ws_bytes, cudaStream_t stream);

/* W4A8 from FP16 / BF16 activations, with the per-token INT8 quantization fused into the
 * matmul ("Accelerating LLM inference with CUDA Graph and INT4 quantization", part 1, steps 2-4,
 * and the fused-kernel item of its section on combining the strategies).  Results are
 * bit-identical to act_quant_int8(A, a_dt, M, K, Aq, a_scale) followed by
 * w4a8_gemm(Aq, a_scale, Wq, scales, zeros, bias, C, acc_out, ...).
 *   A [M,K] a_dt (WQ_F16 or WQ_BF16), K % 8 == 0.
 *   Aq [M,K] int8 and a_scale [M] binary32: required outputs, written with the values
 *   act_quant_int8 writes.  C, bias, acc_out, workspace as for w4a8_gemm.
 * When M <= 16, M * K <= 16384 and the few-token kernel stages the activations whole, this is
 * ONE launch: every CTA forms the per-token scales and codes itself in its prologue (no second
 * kernel, no INT8 round trip through memory).  Otherwise it enqueues act_quant_int8 and
 * w4a8_gemm (each CTA would read all of a larger A twice). */
wq_status w4a8_gemm_fused(const void *A, wq_dtype a_dt, const uint8_t *Wq, const void *scales,
                          const void *zeros, const void *bias, void *C, int8_t *Aq, float *a_scale,
                          int32_t *acc_out, int64_t M, int64_t N, int64_t K, wq_qconfig c,
                          void *workspace, size_t ws_bytes, cudaStream_t stream);

/* Per-token FP8 (e4m3) activation quantization, for the FP8_E4M3 x FP8_E4M3 row of the
 * BitBLAS guide's data-type table.  a_scale[m] = absmax_k|A[m,k]| / 448 (binary32 division);
 * Aq[m,k] = the e4m3 code of clip(A[m,k] / a_scale[m], -448, 448) (binary32 quotient), rounded
 * to the nearest e4m3 value, ties to the even last mantissa bit, +0 for a zero result; an
 * all-zero token gives scale 0 and codes 0.
 *   A [M,K] a_dt (WQ_F16 or WQ_BF16); Aq [M,K] e4m3 codes (bytes) and a_scale [M] binary32
 *   written.  K % 8 == 0.  Bit-exact with the CPU reference. */
wq_status act_quant_fp8(const void *A, wq_dtype a_dt, int64_t M, int64_t K, uint8_t *Aq, float *a_scale,
                        cudaStream_t stream);

/* W8A8 FP8 (the guide's FP8_E4M3 x FP8_E4M3 -> FP32 -> FP16 row):
 *   C[m,n] = fp16( a_scale[m] * sum_g s[n,g] * sum_{k in g} v(Aq[m,k]) v(Wq[n,k])  (+ bias[n]) )
 * with v the e4m3 value of a code; the products are exact and the sums are accumulated in
 * binary32 (one per 128 k on the tensor cores, then scaled by s and added).
 *   Aq [M,K] e4m3 codes and a_scale [M] binary32 (from act_quant_fp8); Wq [N,K] e4m3 codes
 *   and scales binary16 [N, K/group_size] from wq_quantize_pack with c.format = WQ_FMT_E4M3,
 *   c.bits = 8 (other weight types: WQ_ERR_UNSUPPORTED); C [M,N] binary16; bias [N] binary16
 *   or NULL; workspace as for w4a16_gemm.  K % 128 == 0; above 16 tokens K >= 512. */
wq_status w8a8_fp8_gemm(const uint8_t *Aq, const float *a_scale, const uint8_t *Wq, const void *scales,
                        const void *bias, void *C, int64_t M, int64_t N, int64_t K, wq_qconfig c,
                        void *workspace, size_t ws_bytes, cudaStream_t stream);

/* W8A8 FP8 from FP16 / BF16 activations, with the per-token FP8 quantization fused into the
 * matmul (as w4a8_gemm_fused for INT8).  Results are bit-identical to act_quant_fp8 followed by
 * w8a8_fp8_gemm; Aq and a_scale are required outputs, written with the values act_quant_fp8
 * writes.  When M <= 16, M * K <= 16384 and the few-token kernel stages the activations whole,
 * this is ONE launch; otherwise it enqueues the two calls. */
wq_status w8a8_fp8_gemm_fused(const void *A, wq_dtype a_dt, const uint8_t *Wq, const void *scales,
                              const void *bias, void *C, uint8_t *Aq, float *a_scale, int64_t M, int64_t N,
                              int64_t K, wq_qconfig c, void *workspace, size_t ws_bytes, cudaStream_t stream);

/* Bytes of workspace that lets w4a16_gemm / w4a8_gemm use their split-K plans on the
 * current device (those of the tiled mma.sync path; 0 where that path is not used). */
size_t wq_workspace_size(int64_t M, int64_t N, int64_t K, wq_qconfig c);

/* Capacity of the static scratch that w4a16_gemm_noalloc uses (one array per device). */
#define WQ_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)

/* w4a16_gemm without a workspace argument, and without allocating anything.
 * (A library convenience: the quantised-matmul method itself has no counterpart of it.)
 * For callers that cannot provide a workspace: a plain C host loop that owns no device
 * allocator, or a plug-in inside a runtime that hands out no scratch.  Allocating for
 * them is no way out, because cudaFree synchronises the device and a per-shape workspace
 * would be reallocated whenever a larger shape arrives.
 *   Arguments, layouts, results and errors as for w4a16_gemm (bit-identical output).
 *   Scratch: a static device array of WQ_NOALLOC_SCRATCH_BYTES per device, inside
 *   libwq.  The FIRST call on a device looks up its address (cudaGetSymbolAddress, with
 *   that device current), clears it and waits for the device: make that first call
 *   before any stream capture.  Later calls allocate, clear and wait for nothing.
 *   A shape with wq_workspace_size(M,N,K,c) > WQ_NOALLOC_SCRATCH_BYTES is refused with
 *   WQ_ERR_WORKSPACE (see wq_last_error) before anything runs.
 *   Calls that overlap on the GPU (several streams or host threads on one device) share
 *   the one array and race: the caller must serialise them. */
wq_status w4a16_gemm_noalloc(const void *A, wq_dtype a_dt, const uint8_t *Wq, const void *scales,
                             const void *zeros, const void *bias, void *C,
                             int64_t M, int64_t N, int64_t K, wq_qconfig c, cudaStream_t stream);

/* ---- A decode step as one CUDA graph ("Accelerating LLM inference with CUDA Graph and INT4
 * quantization", part 2: capture the step's kernels in a graph once, update the arguments that
 * change from step to step, and launch the whole step with one call).
 *
 * A wq_graph holds a chain of up to WQ_GRAPH_MAX_OPS W4A16 / W2A16 matmuls of at most 16
 * tokens each (for example the QKV, output, gate/up and down projections of one transformer
 * layer at decode time), as kernel nodes of one CUDA graph in the given order.  Consecutive
 * nodes are joined by programmatic-dependent-launch edges, so each matmul streams its weights
 * while the previous one finishes; a node may read the output of an earlier one.
 *   ops[i]: the arguments of w4a16_gemm for matmul i (same meaning, layouts and checks;
 *           M <= 16, else WQ_ERR_UNSUPPORTED).  The weights, scales, zeros and bias stay
 *           fixed for the graph's life; A and C can be changed per step with wq_graph_set_io.
 *   Each launch computes exactly what w4a16_gemm computes for the same arguments (the same
 *   kernels and launch plans: bit-identical outputs).
 * Ownership: the graph keeps the device pointers it was given (the caller keeps those buffers
 * alive and unchanged in shape until wq_graph_destroy).  Creating it captures the launches on a
 * private stream (created and destroyed inside the call; nothing runs) and allocates host
 * memory and the driver's graph objects, never device memory.  One wq_graph is used by one
 * host thread at a time.  Errors as for w4a16_gemm; a failed create returns no
 * graph. */
#define WQ_GRAPH_MAX_OPS 64
typedef struct {
    const void *A;
    wq_dtype a_dt;
    const uint8_t *Wq;
    const void *scales;
    const void *zeros;
    const void *bias;
    void *C;
    int64_t M, N, K;
    wq_qconfig c;
} wq_matmul_desc;

typedef struct wq_graph wq_graph;

wq_status wq_graph_create(const wq_matmul_desc *ops, int n_ops, wq_graph **out);
/* New activation and output pointers for matmul `op` (16-byte aligned device pointers of the
 * same shapes), taking effect from the next wq_graph_launch: the node's arguments are
 * rewritten in the instantiated graph (cudaGraphExecKernelNodeSetParams); nothing is
 * re-instantiated.  Launches already enqueued keep the pointers they were launched with. */
wq_status wq_graph_set_io(wq_graph *g, int op, const void *A, void *C);
/* Enqueues one run of the whole chain on `stream` (asynchronous). */
wq_status wq_graph_launch(wq_graph *g, cudaStream_t stream);
void wq_graph_destroy(wq_graph *g);

const char *wq_status_string(wq_status s);

/* Reads and clears the library's device-side error word.  Non-zero means that a kernel's
 * outputs are not valid: 1, it gave up a bounded wait on one of its own barriers (about
 * 2 s) and returned early; 2, it found itself launched in another thread-block cluster
 * shape than planned and did no work.  Synchronous (device-to-host copy of one word); for
 * tests and diagnostics. */
int wq_device_error(void);
/* One-line reason for the last non-OK status returned on the calling thread. */
const char *wq_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* WQ_H */
