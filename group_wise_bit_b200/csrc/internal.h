// Host-side declarations shared by the library's translation units: the
// thread-local error message and the kernel launchers that the C ABI
// (api.cu) dispatches to.  Launchers assume validated arguments.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/gwb.h"

namespace gwb {

// Records a message for gwb_last_error() and returns `st`.
gwb_status fail(gwb_status st, const char *fmt, ...);

// Maps the launch error (if any) of the last kernel to a gwb_status.
gwb_status check_launch(const char *what);

// Synchronizes `st`, then reads and clears the device error flag (bit 0: a
// bounded device wait gave up) of the current device.
gwb_status read_and_clear_device_error(cudaStream_t st, unsigned int *flag);
// Sets the clock cycles after which device waits give up on the current
// device (0: the default, about 2 s).
gwb_status set_wait_cycles(unsigned long long cycles);
// armed: the next stream-K launch of the persistent GEMM waits for a partial
// tile that no CTA publishes (failure-path testing); false disarms it.
void inject_stream_k_stall(bool armed);

// ------------------------------------------------------------ elementwise kernels
void launch_qpack_affine(const float *w, int64_t N, int64_t K, int bits, int gs, uint32_t *wq,
                         uint16_t *scales, uint16_t *biases, cudaStream_t st);
void launch_dequant_affine(const uint32_t *wq, const uint16_t *scales, const uint16_t *biases, int64_t N,
                           int64_t K, int bits, int gs, uint16_t *w_out, cudaStream_t st);
// zadd: added to each stored zero nibble (1: GPTQ's "+1" convention, 0: AWQ's).
void launch_gptq_dequant(const int32_t *qweight, const uint16_t *scales, const int32_t *qzeros,
                         const int32_t *g_idx, int64_t K, int64_t N, int gs, uint16_t *w_out, cudaStream_t st,
                         int zadd = 1);
void launch_quant_per_token_i8(const uint16_t *x, int64_t M, int64_t K, int8_t *qx, float *sx,
                               cudaStream_t st);
void launch_qpack_sym_i8(const float *w, int64_t N, int64_t K, int8_t *wq, float *sw, cudaStream_t st);
void launch_qpack_sym_i4(const float *w, int64_t N, int64_t K, uint32_t *wq, float *sw, cudaStream_t st);

// ------------------------------------------------------------ GEMV regime (M <= 8)
// Returns false when the (bits, gs) combination has no GEMV kernel (the caller
// then uses the tensor-core path).
bool gemv_affine_supported(int bits, int gs);
gwb_status launch_gemv_affine(const uint16_t *x, int M, const uint32_t *wq, const uint16_t *scales,
                              const uint16_t *biases, int64_t N, int64_t K, int bits, int gs, uint16_t *y,
                              cudaStream_t st);
// Streaming (TMA-fed) GEMV for the MLX affine layout; returns GWB_ERR_UNSUPPORTED
// (without a message) for layouts it does not cover, and the register-fed GEMV
// is used instead.
gwb_status launch_gemv_stream(const uint16_t *x, int M, const uint32_t *wq, const uint16_t *scales,
                              const uint16_t *biases, int64_t N, int64_t K, int bits, int gs, uint16_t *y,
                              cudaStream_t st);
// Producer/consumer decode GEMV (the main decode kernel); GWB_ERR_UNSUPPORTED
// (without a message) for layouts it does not cover (K / gs not a multiple of 8).
gwb_status launch_gemv_pipe(const uint16_t *x, int M, const uint32_t *wq, const uint16_t *scales,
                            const uint16_t *biases, int64_t N, int64_t K, int bits, int gs, uint16_t *y,
                            cudaStream_t st);
gwb_status launch_gemv_i8w8(const int8_t *qx, const float *sx, int M, const int8_t *wq, const float *sw, int64_t N,
                            int64_t K, uint16_t *y, int32_t *acc, cudaStream_t st);
gwb_status launch_gemv_w4a8(const uint16_t *x, int M, const uint32_t *wq, const float *sw, int64_t N, int64_t K,
                            uint16_t *y, cudaStream_t st);
gwb_status launch_gemv_gate_up(const uint16_t *x, int M, const uint32_t *wq_gate, const uint16_t *sc_gate,
                               const uint16_t *bi_gate, const uint32_t *wq_up, const uint16_t *sc_up,
                               const uint16_t *bi_up, int64_t N, int64_t K, int bits, int gs, uint16_t *y_gate,
                               uint16_t *y_up, cudaStream_t st);
gwb_status launch_gemv_silu_gate(const uint16_t *gate, const uint16_t *up, int M, const uint32_t *wq,
                                 const uint16_t *scales, const uint16_t *biases, int64_t N, int64_t K, int bits,
                                 int gs, const uint16_t *resid, uint16_t *y, cudaStream_t st);
// GPTQ / AWQ GEMV: the shared-memory streamed kernel where the layout allows
// (launch_gemv_gptq_pipe: N % 32 == 0, K % 256 == 0, 16-byte aligned weight
// tensors, M <= 8; GWB_ERR_UNSUPPORTED without a message otherwise), else the
// register-fed one.
gwb_status launch_gemv_gptq_pipe(const uint16_t *x, int M, const int32_t *qweight, const uint16_t *scales,
                                 const int32_t *qzeros, const int32_t *g_idx, int64_t K, int64_t N, int gs,
                                 uint16_t *y, cudaStream_t st, int zadd);
gwb_status launch_gemv_gptq(const uint16_t *x, int M, const int32_t *qweight, const uint16_t *scales,
                            const int32_t *qzeros, const int32_t *g_idx, int64_t K, int64_t N, int gs,
                            uint16_t *y, cudaStream_t st, int zadd = 1);

// ------------------------------------------------------------ tensor-core GEMM regime
gwb_status launch_tc_affine(const uint16_t *x, int64_t M, const uint32_t *wq, const uint16_t *scales,
                            const uint16_t *biases, int64_t N, int64_t K, int bits, int gs, uint16_t *y,
                            cudaStream_t st);
gwb_status launch_tc_gptq(const uint16_t *x, int64_t M, const int32_t *qweight, const uint16_t *scales,
                          const int32_t *qzeros, const int32_t *g_idx, int64_t K, int64_t N, int gs,
                          uint16_t *y, cudaStream_t st, int zadd = 1);
// Persistent tensor-core GEMM (M > 8); GWB_ERR_UNSUPPORTED (without a
// message) when the layout needs the per-tile kernel (unstaged scales, g_idx).
gwb_status launch_tc2_affine(const uint16_t *x, int64_t M, const uint32_t *wq, const uint16_t *scales,
                             const uint16_t *biases, int64_t N, int64_t K, int bits, int gs, uint16_t *y,
                             cudaStream_t st);
gwb_status launch_tc2_gptq(const uint16_t *x, int64_t M, const int32_t *qweight, const uint16_t *scales,
                           const int32_t *qzeros, const int32_t *g_idx, int64_t K, int64_t N, int gs, uint16_t *y,
                           cudaStream_t st, int zadd = 1);
gwb_status launch_tc2_i8i8(const int8_t *qx, const float *sx, int64_t M, const int8_t *wq, const float *sw,
                           int64_t N, int64_t K, uint16_t *y, int32_t *acc, cudaStream_t st);
gwb_status launch_tc2_i8i4(const int8_t *qx, const float *sx, int64_t M, const uint32_t *wq, const float *sw,
                           int64_t N, int64_t K, uint16_t *y, int32_t *acc, cudaStream_t st);
// Dense fp16 weights [N, K] on the persistent GEMM (fp16 in and out);
// GWB_ERR_UNSUPPORTED (without a message) for K % 8 != 0 or unaligned operands.
gwb_status launch_tc2_f16(const uint16_t *x, int64_t M, const uint16_t *w, int64_t N, int64_t K, uint16_t *y,
                          cudaStream_t st);
// The library's scratch for dequantized weights on this stream, at least
// `bytes` long; false when it cannot be had (allocation under stream capture,
// or out of memory).
bool dequant_scratch(cudaStream_t st, size_t bytes, uint16_t **out);
// The persistent GEMM with its stream-K scratch in a fixed device array (no
// allocation); M must exceed 128.
gwb_status launch_tc2_affine_noalloc(const uint16_t *x, int64_t M, const uint32_t *wq, const uint16_t *scales,
                                     const uint16_t *biases, int64_t N, int64_t K, int bits, int gs, uint16_t *y,
                                     cudaStream_t st);

}  // namespace gwb
