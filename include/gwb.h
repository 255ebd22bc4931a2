/*
 * gwb.h -- C ABI of the group-wise low-bit linear-layer library for NVIDIA B200
 * (sm_100a).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All tensor pointers are DEVICE pointers owned by the caller; the library
 *    never allocates, frees or retains them.  Tensors are dense and row-major
 *    with the shapes stated per call; no strides are taken.
 *  - The library owns two kinds of device buffer.  The first is the persistent
 *    tensor-core GEMM's stream-K workspace (partial tiles, up to about 19 MB):
 *    one per (device, stream), allocated by the first call on that stream that
 *    runs that GEMM with split tiles (qmm_affine, gptq_qmm and awq_qmm above 8
 *    tokens, gemm_i8i4, gemm_i8i8 off its decode path), grown once if a later
 *    call needs more (after synchronizing the stream), and kept until the
 *    process exits.  The second is gptq_qmm's act-order scratch (see there).  A call made while its stream is being captured
 *    into a CUDA graph never allocates: it uses the stream's workspace if an
 *    earlier call made one, else it runs without (whole tiles per CTA or pair).
 *    Each launch takes its stream-K epoch from a counter in the workspace, on
 *    the device, so graph replays stay correct.  gwb_qmm_affine_noalloc is the
 *    entry point that allocates nothing.
 *  - bf16 and fp16 values are passed as their raw 16-bit patterns (uint16_t).
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  Every call
 *    validates its arguments synchronously, on the host, before launching
 *    anything; on success the work is enqueued on `stream` and the call returns
 *    without synchronizing.  A call that returns an error has launched nothing.
 *  - Pointers must be 16-byte aligned (GWB_ERR_ALIGN otherwise); optional
 *    pointers that may be NULL say so.
 *  - The return value is a gwb_status; gwb_last_error() gives a readable
 *    message for the calling thread's most recent failure.
 *  - Device-side waits inside the tensor-core kernels are bounded; a wait that
 *    gives up records GWB_ERR_TIMEOUT in a device flag that
 *    gwb_check_device_error() reads and clears.
 *  - Quantized weights follow four layouts (bits b, group size gs):
 *      MLX affine   wq      uint32 [N, K*b/32]  codes packed along K, lowest bits
 *                                              = lowest column
 *                   scales  bf16   [N, K/gs]
 *                   biases  bf16   [N, K/gs]    w[n,k] = code*scale + bias
 *      GPTQ int4    qweight int32  [K/8, N]     packed along IN (K)
 *                   scales  fp16   [K/gs, N]
 *                   qzeros  int32  [K/gs, N/8]  packed along OUT, stores zero-1
 *                   g_idx   int32  [K]          optional group of each in-feature
 *                   (AWQ: the same tensors without g_idx, zero as stored)
 *      sym int4     wq      uint32 [N, K/8]     two's-complement nibbles along K
 *                   sw      fp32   [N]          w[n,k] = code*sw[n]
 *      sym int8     wq      int8   [N, K]       w[n,k] = wq[n,k]*sw[n]
 *                   sw      fp32   [N]
 *    A linear layer computes y[M,N] = x[M,K] . W^T, with W stored [N = out, K = in].
 *
 * Sources (page title, then section): "MLX" = metrale_gpu_runtime/mlx_int8.rs
 * module doc "Layout" and the Hugging Face transformers "Metal" quantization
 * page; "GPTQ" = TinyGPT "Quantization Expansion", section 1 "GPTQReader",
 * "Format" and dequant recipe; "QAT" = the same page, section 4, "Fake-quant +
 * STE"; "W4A8" = executorch PR #24467 "mlx::int8_int4_gemm".
 */
#ifndef GWB_H
#define GWB_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum gwb_status {
    GWB_OK = 0,
    GWB_ERR_INVALID_ARG = 1,  /* NULL where a tensor is required, negative size, ...     */
    GWB_ERR_SHAPE = 2,        /* sizes that the layout cannot hold (K % gs, N % 8, ...)  */
    GWB_ERR_UNSUPPORTED = 3,  /* bits not in {2,4,8}, group size not in {32,64,128}, ... */
    GWB_ERR_ALIGN = 4,        /* a pointer is not 16-byte aligned                        */
    GWB_ERR_CUDA = 5,         /* a CUDA runtime/driver call or kernel launch failed      */
    GWB_ERR_TIMEOUT = 6       /* a bounded device-side wait gave up                      */
} gwb_status;

/* Message for the calling thread's most recent non-GWB_OK return ("" if none).
 * The string is owned by the library and valid until the next call on this thread. */
const char *gwb_last_error(void);

/* Library version string. */
const char *gwb_version(void);

/* Synchronizes `stream`, then reads and clears the current device's error
 * flag, which every bounded wait of the library's kernels sets when it gives
 * up (one flag per device, shared by all kernels).  Returns GWB_OK when no wait
 * gave up since the last check, GWB_ERR_TIMEOUT otherwise, GWB_ERR_CUDA when
 * the synchronization itself failed.  A kernel whose wait gave up stops
 * issuing work, lets the copies it started land, frees its tensor memory and
 * returns, so the context stays usable; its outputs are then undefined.
 * Source: metrale_gpu_runtime/mlx_int8.rs, MlxInt8Weight::load (failures are
 * returned as errors, never as a crash). */
gwb_status gwb_check_device_error(void *stream);

/* Failure-path testing hooks (the pages have no counterpart; they exist so
 * that the bounded-wait path above can be exercised without faulting a GPU).
 *
 * gwb_debug_set_wait_cycles -- sets, on the current device, the number of SM
 * clock cycles after which a device wait gives up (0 restores the default of
 * 4e9 cycles, about 2 s).  Takes effect for kernels launched afterwards;
 * synchronous.  GWB_ERR_CUDA if the device symbol cannot be written. */
gwb_status gwb_debug_set_wait_cycles(unsigned long long cycles);

/* gwb_debug_inject_stream_k_stall -- armed != 0: the next launch in this
 * process of the persistent tensor-core GEMM that splits tiles between CTA
 * pairs (stream-K) waits for partial tiles that no CTA publishes; its head
 * CTAs' bounded waits run out, the kernel returns early with undefined outputs,
 * and the next gwb_check_device_error() reports GWB_ERR_TIMEOUT.  One-shot: that
 * launch disarms it.  armed == 0 disarms it.  Always GWB_OK. */
gwb_status gwb_debug_inject_stream_k_stall(int armed);

/* ------------------------------------------------------------------ MLX affine */

/* qpack_affine -- per-group min/max affine quantization and packing (MLX layout).
 * For each row n and group g of `group_size` consecutive columns, in fp32 with
 * one IEEE rounding per step:
 *   mn = min, mx = max of the group;  s = (mx - mn) / (2^bits - 1);
 *   code = clip(round_half_even((w - mn) / s), 0, 2^bits - 1)   (0 when s == 0)
 * scales[n,g] = bf16_rne(s), biases[n,g] = bf16_rne(mn); codes are packed
 * 32/bits per uint32, lowest bits = lowest column.
 * Source: MLX (affine scheme, packed uint32 layout, bf16 scales/biases).
 *   w       fp32  [N, K]             input weights (finite values)
 *   wq      u32   [N, K*bits/32]     output
 *   scales  bf16  [N, K/group_size]  output
 *   biases  bf16  [N, K/group_size]  output
 * bits in {2,4,8}; group_size in {32,64,128}; K % group_size == 0.
 * Results are bit-exact and independent of the launch configuration. */
gwb_status gwb_qpack_affine(const float *w, int64_t N, int64_t K, int bits, int group_size,
                            uint32_t *wq, uint16_t *scales, uint16_t *biases, void *stream);

/* dequant_affine -- w_out[n,k] = bf16_rne(fp32(code*scale + bias)): the exact
 * value rounded once to fp32, then to bf16.  Source: MLX (the dequant formula
 * w[r,c] = byte*scales[r,c/G] + biases[r,c/G] and its dequantize_to output).
 *   w_out   bf16  [N, K]             output
 * Same layout arguments and limits as gwb_qpack_affine. */
gwb_status gwb_dequant_affine(const uint32_t *wq, const uint16_t *scales, const uint16_t *biases,
                              int64_t N, int64_t K, int bits, int group_size,
                              uint16_t *w_out, void *stream);

/* qmm_affine -- fused dequant + matmul (the affine_qmm_t operation):
 *   y[m,n] = sum_k x[m,k] * (code(n,k)*scale[n,k/gs] + bias[n,k/gs])
 * with fp32 accumulation and a bf16 (round-to-nearest-even) result.
 * Source: MLX (Hugging Face "Metal" quantization: fused dequant + matmul
 * affine_qmm_t; mlx_int8.rs gemv / gemm docs for y = W x and Y = X W^T).
 *   x   bf16  [M, K]   activations;   y   bf16  [M, N]   output
 * M >= 1.  M <= 8 runs the memory-bound split-K GEMV regime; larger M runs the
 * tensor-core (tcgen05) GEMM regime.  For bits == 2 the packed row length
 * K/16 words must be a multiple of 4 (K % 64 == 0).
 * The result is deterministic for a given shape (no atomics), but not bitwise
 * equal to any particular summation order. */
gwb_status gwb_qmm_affine(const uint16_t *x, int64_t M, const uint32_t *wq, const uint16_t *scales,
                          const uint16_t *biases, int64_t N, int64_t K, int bits, int group_size,
                          uint16_t *y, void *stream);

/* qmm_affine_noalloc -- gwb_qmm_affine's prefill GEMM for callers that cannot
 * allocate device memory.  Such callers exist: code running under an allocator
 * that owns all of the GPU's memory (a framework's caching pool, a serving
 * runtime that reserves memory up front), and code that must not call cudaMalloc
 * or cudaFree at all (both may synchronize the whole device).  The pages
 * describe no counterpart of this entry point; it is a property of this library.
 * Same arguments, layouts and result as gwb_qmm_affine, for M > 128 only
 * (GWB_ERR_SHAPE otherwise: smaller M needs no scratch, call gwb_qmm_affine).
 * The GEMM's stream-K scratch (partial tiles and their flags) is a file-scope
 * device array of the library, 8 MiB + 512 bytes, which holds the partials of
 * at most 32 CTA pairs, so the GEMM runs on at most 32 pairs (64 of the 148
 * SMs); every problem size fits, because a pair's share of the work grows with
 * the problem while its partial tile does not.  Every GPU that loads the
 * library holds the array until the process exits.
 *  - The call allocates nothing: no cudaMalloc, cudaFree or allocating library
 *    routine.  The first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress, with that device current) and caches it; make that
 *    first call before any stream capture.
 *  - All calls share the one array, which keeps the last call's contents; each
 *    call clears the flags it needs before its kernel runs.  Calls that overlap
 *    on the GPU (concurrent streams, or several devices' threads racing on one
 *    device) race on the array and give wrong results: serialize them.
 * Also GWB_ERR_UNSUPPORTED when K/group_size is odd, and GWB_ERR_ALIGN when x,
 * y or the weight tensors are not 16-byte aligned. */
gwb_status gwb_qmm_affine_noalloc(const uint16_t *x, int64_t M, const uint32_t *wq, const uint16_t *scales,
                                  const uint16_t *biases, int64_t N, int64_t K, int bits, int group_size,
                                  uint16_t *y, void *stream);

/* ------------------------------------------------------------------ GPTQ */

/* gptq_dequant -- the GPTQ dequant recipe, one weight at a time:
 *   int4 = (qweight[i/8, o] >> ((i%8)*4)) & 0xF
 *   g    = g_idx ? g_idx[i] : i / group_size
 *   zero = ((qzeros[g, o/8] >> ((o%8)*4)) & 0xF) + 1        (the "+1" convention)
 *   w_out[o, i] = fp16_rne(scales[g, o] * (int4 - zero))     (exact product, one rounding)
 * Source: GPTQ (format and dequant recipe).
 *   qweight i32 [K/8, N], scales fp16 [K/gs, N], qzeros i32 [K/gs, N/8],
 *   g_idx   i32 [K] or NULL, w_out fp16 [N, K] (out-features major, as HF stores W)
 * K % 8 == 0, N % 8 == 0, K % group_size == 0, group_size in {32,64,128}.
 * g_idx values must lie in [0, K/group_size); they are not checked (an
 * out-of-range value reads outside `scales`/`qzeros`). */
gwb_status gwb_gptq_dequant(const int32_t *qweight, const uint16_t *scales, const int32_t *qzeros,
                            const int32_t *g_idx, int64_t K, int64_t N, int group_size,
                            uint16_t *w_out, void *stream);

/* gptq_qmm -- y[m,o] = sum_i x[m,i] * W[o,i] with W as gwb_gptq_dequant defines
 * it (each weight rounded to fp16, as the dequantized checkpoint would hold it),
 * fp32 accumulation, fp16 result.
 *   x  fp16 [M, K],  y  fp16 [M, N].   Limits as gwb_gptq_dequant; M >= 1.
 * With g_idx and M > 8 the weights are first dequantized into a scratch buffer
 * owned by the library (2*N*K bytes, one per device and stream, grown to the
 * largest layer seen and kept until exit; a call under stream capture never
 * allocates it and then runs a slower kernel without it). */
gwb_status gwb_gptq_qmm(const uint16_t *x, int64_t M, const int32_t *qweight, const uint16_t *scales,
                        const int32_t *qzeros, const int32_t *g_idx, int64_t K, int64_t N,
                        int group_size, uint16_t *y, void *stream);

/* ------------------------------------------------------- fused decode products
 * Source: metrale_gpu_runtime/mlx_int8.rs, the free function gemv_gate_up and
 * MlxInt8Weight::gemv_silu_gate / gemv_silu_gate_resid (decode-time MLP fusion
 * for MLX affine weights).  Every weight is in the layout of gwb_qmm_affine
 * (wq u32 [N, K*bits/32], scales and biases bf16 [N, K/group_size]); vectors
 * are bf16 rows of 1 <= M <= 8 tokens, 16-byte aligned.  K/group_size must be a
 * multiple of 8 (GWB_ERR_UNSUPPORTED otherwise).  Float results: fp32
 * accumulation, one rounding to bf16, within the tolerance of gwb_qmm_affine.
 * M > 8 is GWB_ERR_SHAPE: these are single-token products.
 *
 * gemv_gate_up -- y_gate = x W_gate^T and y_up = x W_up^T in one launch; the
 * two weights share N, K, bits and group_size.
 *   x bf16 [M, K];  y_gate, y_up bf16 [M, N]. */
gwb_status gwb_gemv_gate_up(const uint16_t *x, int64_t M, const uint32_t *wq_gate,
                            const uint16_t *scales_gate, const uint16_t *biases_gate,
                            const uint32_t *wq_up, const uint16_t *scales_up,
                            const uint16_t *biases_up, int64_t N, int64_t K, int bits, int group_size,
                            uint16_t *y_gate, uint16_t *y_up, void *stream);

/* gemv_silu_gate -- y = (silu(gate) * up) W^T, silu(g) = g / (1 + exp(-g)); the
 * product silu(gate) * up is formed in fp32 and never written to memory.
 *   gate, up bf16 [M, K];  y bf16 [M, N]. */
gwb_status gwb_gemv_silu_gate(const uint16_t *gate, const uint16_t *up, int64_t M, const uint32_t *wq,
                              const uint16_t *scales, const uint16_t *biases, int64_t N, int64_t K,
                              int bits, int group_size, uint16_t *y, void *stream);

/* gemv_silu_gate_resid -- y = x_resid + (silu(gate) * up) W^T, the residual
 * added to the fp32 sum before its rounding.  x_resid bf16 [M, N] (non-NULL;
 * it may be y itself: each element is read before it is written). */
gwb_status gwb_gemv_silu_gate_resid(const uint16_t *gate, const uint16_t *up, int64_t M,
                                    const uint32_t *wq, const uint16_t *scales,
                                    const uint16_t *biases, int64_t N, int64_t K, int bits,
                                    int group_size, const uint16_t *x_resid, uint16_t *y,
                                    void *stream);

/* awq_dequant / awq_qmm -- the same layout and shapes as gwb_gptq_dequant /
 * gwb_gptq_qmm, with the zero taken as stored: zero = (qzeros[g, o/8] >> ((o%8)*4)) & 0xF,
 * no "+1", and no g_idx (g = i / group_size).
 * Source: GPTQ page (section 1, after the dequant recipe): auto-gptq stores
 * zero - 1 and re-adds 1, AWQ does not; the AWQ reader has identical shapes.
 * Only that difference is stated, so only it is implemented. */
gwb_status gwb_awq_dequant(const int32_t *qweight, const uint16_t *scales, const int32_t *qzeros, int64_t K,
                           int64_t N, int group_size, uint16_t *w_out, void *stream);
gwb_status gwb_awq_qmm(const uint16_t *x, int64_t M, const int32_t *qweight, const uint16_t *scales,
                       const int32_t *qzeros, int64_t K, int64_t N, int group_size, uint16_t *y, void *stream);

/* ------------------------------------------------------------------ W4A8 */

/* quant_per_token_i8 -- dynamic symmetric per-token int8 (qMax = 127), fp32:
 *   amax = max_k |x[m,k]|;  sx[m] = amax / 127;
 *   qx[m,k] = clip(round_half_even(x[m,k] / sx[m]), -127, 127)   (0 when amax == 0)
 * Source: W4A8 (dynamic symmetric per-token int8 activations) with the
 * symmetric quantizer of QAT.
 *   x bf16 [M, K] (finite), qx int8 [M, K], sx fp32 [M].   Bit-exact. */
gwb_status gwb_quant_per_token_i8(const uint16_t *x, int64_t M, int64_t K, int8_t *qx, float *sx,
                                  void *stream);

/* qpack_sym_i4 -- symmetric per-output-channel int4 weights (qMax = 7):
 *   sw[n] = max_k |w[n,k]| / 7;  code = clip(round_half_even(w / sw[n]), -8, 7)
 * (0 when sw == 0), stored as two's-complement nibbles, 8 per uint32 along K,
 * lowest nibble = lowest k.  Source: QAT (per-row symmetric scale, qMax) and W4A8.
 *   w fp32 [N, K] (finite), wq u32 [N, K/8], sw fp32 [N].  K % 32 == 0.  Bit-exact. */
gwb_status gwb_qpack_sym_i4(const float *w, int64_t N, int64_t K, uint32_t *wq, float *sw,
                            void *stream);

/* gemm_i8i4 -- int8 activations x int4 weights with int32 accumulation:
 *   acc[m,n] = sum_k qx[m,k] * code(n,k)                 (exact int32)
 *   y[m,n]   = bf16_rne(fp32(acc[m,n]) * (sx[m] * sw[n]))
 * Source: W4A8 (INT8 x INT4 -> INT32, per-token and per-channel scales).
 *   qx int8 [M, K], sx fp32 [M], wq u32 [N, K/8], sw fp32 [N]
 *   y   bf16  [M, N] or NULL;  acc int32 [M, N] or NULL (at least one non-NULL)
 * K % 32 == 0 and K <= 131072 (so that the tensor-core partial sums, which
 * carry each int4 code multiplied by 16, stay inside int32).  The int32 result
 * is exact; y is a single rounding of its fp32 product. */
gwb_status gwb_gemm_i8i4(const int8_t *qx, const float *sx, int64_t M, const uint32_t *wq,
                         const float *sw, int64_t N, int64_t K, uint16_t *y, int32_t *acc,
                         void *stream);

/* gemv_w4a8 -- W4A8 at decode with the activation quantization fused into the
 * product: x is quantized to int8 per token (as gwb_quant_per_token_i8 does)
 * inside the kernel and never written to memory, then
 *   acc[m,n] = sum_k q[m,k] * code(n,k);  y[m,n] = bf16_rne(fp32(acc) * (sx[m] * sw[n]))
 * Source: W4A8 ("staged" lowering of mlx::int8_int4_gemm, which quantizes the
 * activations inside the product kernel).  Bit-identical to
 * gwb_quant_per_token_i8 followed by gwb_gemm_i8i4 on the same x.
 *   x bf16 [M, K] (16-byte aligned), wq u32 [N, K/8] and sw fp32 [N] from
 *   gwb_qpack_sym_i4, y bf16 [M, N].
 * 1 <= M <= 8 (GWB_ERR_SHAPE beyond: quantize once with gwb_quant_per_token_i8
 * and call gwb_gemm_i8i4), K % 512 == 0 and K <= 16384 (GWB_ERR_UNSUPPORTED
 * otherwise: the kernel's fp16 tensor-core sums are exact integers only up to
 * that K).  The quantized rows are kept on chip; where a CTA cannot hold all
 * of K, K is split over a cluster of CTAs that exchange their per-token maxima
 * first (the scale is always the whole row's).  GWB_ERR_UNSUPPORTED only when
 * no split fits. */
gwb_status gwb_gemv_w4a8(const uint16_t *x, int64_t M, const uint32_t *wq, const float *sw, int64_t N,
                         int64_t K, uint16_t *y, void *stream);

/* ------------------------------------------------------------------ W8A8 */

/* qpack_sym_i8 -- symmetric per-output-channel int8 weights (qMax = 127):
 *   sw[n] = max_k |w[n,k]| / 127;  wq[n,k] = clip(round_half_even(w / sw[n]), -127, 127)
 * (0 when sw == 0), fp32 arithmetic.  Source: Parakeet export README of
 * executorch PR #17234 ("Quantization Configs": 8da8w, 8-bit dynamic
 * activations x 8-bit weights) with the per-row symmetric quantizer of QAT at
 * bits = 8.
 *   w fp32 [N, K] (finite), wq int8 [N, K], sw fp32 [N].  K % 16 == 0.  Bit-exact. */
gwb_status gwb_qpack_sym_i8(const float *w, int64_t N, int64_t K, int8_t *wq, float *sw, void *stream);

/* gemm_i8i8 -- int8 activations x int8 weights with int32 accumulation:
 *   acc[m,n] = sum_k qx[m,k] * wq[n,k]                   (exact int32)
 *   y[m,n]   = bf16_rne(fp32(acc[m,n]) * (sx[m] * sw[n]))
 * Source: 8da8w (Parakeet export README, executorch PR #17234); scales as in
 * gwb_gemm_i8i4.  qx, sx from gwb_quant_per_token_i8; wq, sw from
 * gwb_qpack_sym_i8.
 *   qx int8 [M, K], sx fp32 [M], wq int8 [N, K], sw fp32 [N]
 *   y   bf16  [M, N] or NULL;  acc int32 [M, N] or NULL (at least one non-NULL)
 * K % 16 == 0 (16-byte rows) and K <= 131072 (127 * 127 * K fits in int32);
 * qx and wq 16-byte aligned (GWB_ERR_ALIGN otherwise).
 * The int32 result is exact; y is a single rounding of its fp32 product. */
gwb_status gwb_gemm_i8i8(const int8_t *qx, const float *sx, int64_t M, const int8_t *wq,
                         const float *sw, int64_t N, int64_t K, uint16_t *y, int32_t *acc,
                         void *stream);

#ifdef __cplusplus
}
#endif
#endif /* GWB_H */
