// The C ABI (include/gwb.h): argument validation, the thread-local error
// message and dispatch to the kernel launchers.  Nothing here computes.
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include "internal.h"

namespace gwb {

static thread_local char g_msg[512] = "";

gwb_status fail(gwb_status st, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
  return st;
}

gwb_status check_launch(const char *what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(GWB_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return GWB_OK;
}

}  // namespace gwb

using gwb::fail;

namespace {

constexpr int64_t kMaxDim = (int64_t)1 << 31;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

gwb_status need(const void *p, const char *name) {
  if (!p) return fail(GWB_ERR_INVALID_ARG, "%s must not be NULL", name);
  if (!aligned16(p)) return fail(GWB_ERR_ALIGN, "%s is not 16-byte aligned", name);
  return GWB_OK;
}

gwb_status check_layout(int64_t N, int64_t K, int bits, int gs) {
  if (N < 0 || K < 0) return fail(GWB_ERR_INVALID_ARG, "negative size (N=%lld, K=%lld)", (long long)N, (long long)K);
  if (N >= kMaxDim || K >= kMaxDim) return fail(GWB_ERR_SHAPE, "N and K must be below 2^31");
  if (bits != 2 && bits != 4 && bits != 8) return fail(GWB_ERR_UNSUPPORTED, "bits=%d not in {2,4,8}", bits);
  if (gs != 32 && gs != 64 && gs != 128) return fail(GWB_ERR_UNSUPPORTED, "group_size=%d not in {32,64,128}", gs);
  if (K % gs != 0) return fail(GWB_ERR_SHAPE, "K=%lld is not a multiple of group_size=%d", (long long)K, gs);
  return GWB_OK;
}

gwb_status check_gptq(int64_t K, int64_t N, int gs) {
  if (N < 0 || K < 0) return fail(GWB_ERR_INVALID_ARG, "negative size (K=%lld, N=%lld)", (long long)K, (long long)N);
  if (N >= kMaxDim || K >= kMaxDim) return fail(GWB_ERR_SHAPE, "N and K must be below 2^31");
  if (gs != 32 && gs != 64 && gs != 128) return fail(GWB_ERR_UNSUPPORTED, "group_size=%d not in {32,64,128}", gs);
  if (K % gs != 0) return fail(GWB_ERR_SHAPE, "K=%lld is not a multiple of group_size=%d", (long long)K, gs);
  if (N % 8 != 0) return fail(GWB_ERR_SHAPE, "N=%lld is not a multiple of 8 (qzeros packs 8 per word)", (long long)N);
  return GWB_OK;
}

#define GWB_TRY(expr)                   \
  do {                                  \
    gwb_status _s = (expr);             \
    if (_s != GWB_OK) return _s;        \
  } while (0)

cudaStream_t as_stream(void *s) { return reinterpret_cast<cudaStream_t>(s); }

gwb_status zero_fill(void *p, size_t bytes, void *stream) {
  if (bytes == 0) return GWB_OK;
  cudaError_t e = cudaMemsetAsync(p, 0, bytes, as_stream(stream));
  if (e != cudaSuccess) return fail(GWB_ERR_CUDA, "cudaMemsetAsync: %s", cudaGetErrorString(e));
  return GWB_OK;
}

}  // namespace

extern "C" {

const char *gwb_last_error(void) { return gwb::g_msg; }

const char *gwb_version(void) { return "group_wise_bit_b200 0.1 (sm_100a)"; }

gwb_status gwb_check_device_error(void *stream) {
  unsigned int flag = 0;
  GWB_TRY(gwb::read_and_clear_device_error(as_stream(stream), &flag));
  if (flag) return fail(GWB_ERR_TIMEOUT, "a bounded device-side wait gave up (flag 0x%x)", flag);
  return GWB_OK;
}

gwb_status gwb_debug_set_wait_cycles(unsigned long long cycles) { return gwb::set_wait_cycles(cycles); }

gwb_status gwb_debug_inject_stream_k_stall(int armed) {
  gwb::inject_stream_k_stall(armed != 0);
  return GWB_OK;
}

gwb_status gwb_qpack_affine(const float *w, int64_t N, int64_t K, int bits, int group_size, uint32_t *wq,
                            uint16_t *scales, uint16_t *biases, void *stream) {
  GWB_TRY(check_layout(N, K, bits, group_size));
  if (N == 0 || K == 0) return GWB_OK;
  GWB_TRY(need(w, "w"));
  GWB_TRY(need(wq, "wq"));
  GWB_TRY(need(scales, "scales"));
  GWB_TRY(need(biases, "biases"));
  gwb::launch_qpack_affine(w, N, K, bits, group_size, wq, scales, biases, as_stream(stream));
  return gwb::check_launch("qpack_affine");
}

gwb_status gwb_dequant_affine(const uint32_t *wq, const uint16_t *scales, const uint16_t *biases, int64_t N,
                              int64_t K, int bits, int group_size, uint16_t *w_out, void *stream) {
  GWB_TRY(check_layout(N, K, bits, group_size));
  if (N == 0 || K == 0) return GWB_OK;
  GWB_TRY(need(wq, "wq"));
  GWB_TRY(need(scales, "scales"));
  GWB_TRY(need(biases, "biases"));
  GWB_TRY(need(w_out, "w_out"));
  gwb::launch_dequant_affine(wq, scales, biases, N, K, bits, group_size, w_out, as_stream(stream));
  return gwb::check_launch("dequant_affine");
}

gwb_status gwb_qmm_affine(const uint16_t *x, int64_t M, const uint32_t *wq, const uint16_t *scales,
                          const uint16_t *biases, int64_t N, int64_t K, int bits, int group_size, uint16_t *y,
                          void *stream) {
  GWB_TRY(check_layout(N, K, bits, group_size));
  if (M < 0) return fail(GWB_ERR_INVALID_ARG, "negative M=%lld", (long long)M);
  if (M >= kMaxDim) return fail(GWB_ERR_SHAPE, "M must be below 2^31");
  if (M == 0 || N == 0) return GWB_OK;
  GWB_TRY(need(y, "y"));
  if (K == 0) return zero_fill(y, (size_t)M * N * 2, stream);
  GWB_TRY(need(x, "x"));
  GWB_TRY(need(wq, "wq"));
  GWB_TRY(need(scales, "scales"));
  GWB_TRY(need(biases, "biases"));
  if (M <= 8 && gwb::gemv_affine_supported(bits, group_size)) {
    gwb_status s =
        gwb::launch_gemv_pipe(x, (int)M, wq, scales, biases, N, K, bits, group_size, y, as_stream(stream));
    if (s != GWB_ERR_UNSUPPORTED) return s;
    s = gwb::launch_gemv_stream(x, (int)M, wq, scales, biases, N, K, bits, group_size, y, as_stream(stream));
    if (s != GWB_ERR_UNSUPPORTED) return s;
    return gwb::launch_gemv_affine(x, (int)M, wq, scales, biases, N, K, bits, group_size, y, as_stream(stream));
  }
  if (bits == 2 && K % 64 != 0)
    return fail(GWB_ERR_UNSUPPORTED, "bits=2 needs K %% 64 == 0 on the tensor-core path (K=%lld)", (long long)K);
  {   // the persistent stream-K GEMM; the per-tile kernel takes the layouts it does not stage
    const gwb_status s =
        gwb::launch_tc2_affine(x, M, wq, scales, biases, N, K, bits, group_size, y, as_stream(stream));
    if (s != GWB_ERR_UNSUPPORTED) return s;
  }
  return gwb::launch_tc_affine(x, M, wq, scales, biases, N, K, bits, group_size, y, as_stream(stream));
}

namespace {

// Checks shared by the fused decode products: the affine layout, 1 <= M <= 8
// tokens, and 16-byte aligned activation and output rows.
gwb_status check_fused(int64_t M, int64_t N, int64_t K, int bits, int group_size) {
  GWB_TRY(check_layout(N, K, bits, group_size));
  if (M < 0) return fail(GWB_ERR_INVALID_ARG, "negative M=%lld", (long long)M);
  if (M > 8) return fail(GWB_ERR_SHAPE, "fused decode products take at most 8 tokens (M=%lld)", (long long)M);
  return GWB_OK;
}

gwb_status fused_unsupported(const char *what, int64_t K, int group_size) {
  return fail(GWB_ERR_UNSUPPORTED, "%s needs K/group_size to be a multiple of 8 (K=%lld, group_size=%d)", what,
              (long long)K, group_size);
}

}  // namespace

gwb_status gwb_gemv_gate_up(const uint16_t *x, int64_t M, const uint32_t *wq_gate, const uint16_t *scales_gate,
                            const uint16_t *biases_gate, const uint32_t *wq_up, const uint16_t *scales_up,
                            const uint16_t *biases_up, int64_t N, int64_t K, int bits, int group_size,
                            uint16_t *y_gate, uint16_t *y_up, void *stream) {
  GWB_TRY(check_fused(M, N, K, bits, group_size));
  if (M == 0 || N == 0) return GWB_OK;
  GWB_TRY(need(y_gate, "y_gate"));
  GWB_TRY(need(y_up, "y_up"));
  if (K == 0) {
    GWB_TRY(zero_fill(y_gate, (size_t)M * N * 2, stream));
    return zero_fill(y_up, (size_t)M * N * 2, stream);
  }
  GWB_TRY(need(x, "x"));
  GWB_TRY(need(wq_gate, "wq_gate"));
  GWB_TRY(need(scales_gate, "scales_gate"));
  GWB_TRY(need(biases_gate, "biases_gate"));
  GWB_TRY(need(wq_up, "wq_up"));
  GWB_TRY(need(scales_up, "scales_up"));
  GWB_TRY(need(biases_up, "biases_up"));
  if (!aligned16(x)) return fail(GWB_ERR_ALIGN, "x is not 16-byte aligned");
  const gwb_status s = gwb::launch_gemv_gate_up(x, (int)M, wq_gate, scales_gate, biases_gate, wq_up, scales_up,
                                                biases_up, N, K, bits, group_size, y_gate, y_up, as_stream(stream));
  return s == GWB_ERR_UNSUPPORTED ? fused_unsupported("gemv_gate_up", K, group_size) : s;
}

namespace {

gwb_status silu_gate_impl(const uint16_t *gate, const uint16_t *up, int64_t M, const uint32_t *wq,
                          const uint16_t *scales, const uint16_t *biases, int64_t N, int64_t K, int bits,
                          int group_size, const uint16_t *x_resid, uint16_t *y, void *stream, const char *what) {
  GWB_TRY(check_fused(M, N, K, bits, group_size));
  if (M == 0 || N == 0) return GWB_OK;
  GWB_TRY(need(y, "y"));
  if (K == 0) {
    if (!x_resid) return zero_fill(y, (size_t)M * N * 2, stream);
    const cudaError_t e = cudaMemcpyAsync(y, x_resid, (size_t)M * N * 2, cudaMemcpyDeviceToDevice, as_stream(stream));
    return e == cudaSuccess ? GWB_OK : fail(GWB_ERR_CUDA, "cudaMemcpyAsync: %s", cudaGetErrorString(e));
  }
  GWB_TRY(need(gate, "gate"));
  GWB_TRY(need(up, "up"));
  GWB_TRY(need(wq, "wq"));
  GWB_TRY(need(scales, "scales"));
  GWB_TRY(need(biases, "biases"));
  if (!aligned16(gate) || !aligned16(up)) return fail(GWB_ERR_ALIGN, "gate and up must be 16-byte aligned");
  const gwb_status s = gwb::launch_gemv_silu_gate(gate, up, (int)M, wq, scales, biases, N, K, bits, group_size,
                                                  x_resid, y, as_stream(stream));
  return s == GWB_ERR_UNSUPPORTED ? fused_unsupported(what, K, group_size) : s;
}

}  // namespace

gwb_status gwb_gemv_silu_gate(const uint16_t *gate, const uint16_t *up, int64_t M, const uint32_t *wq,
                              const uint16_t *scales, const uint16_t *biases, int64_t N, int64_t K, int bits,
                              int group_size, uint16_t *y, void *stream) {
  return silu_gate_impl(gate, up, M, wq, scales, biases, N, K, bits, group_size, nullptr, y, stream,
                        "gemv_silu_gate");
}

gwb_status gwb_gemv_silu_gate_resid(const uint16_t *gate, const uint16_t *up, int64_t M, const uint32_t *wq,
                                    const uint16_t *scales, const uint16_t *biases, int64_t N, int64_t K, int bits,
                                    int group_size, const uint16_t *x_resid, uint16_t *y, void *stream) {
  if (M > 0 && N > 0) GWB_TRY(need(x_resid, "x_resid"));
  return silu_gate_impl(gate, up, M, wq, scales, biases, N, K, bits, group_size, x_resid, y, stream,
                        "gemv_silu_gate_resid");
}

gwb_status gwb_qmm_affine_noalloc(const uint16_t *x, int64_t M, const uint32_t *wq, const uint16_t *scales,
                                  const uint16_t *biases, int64_t N, int64_t K, int bits, int group_size,
                                  uint16_t *y, void *stream) {
  GWB_TRY(check_layout(N, K, bits, group_size));
  if (M < 0) return fail(GWB_ERR_INVALID_ARG, "negative M=%lld", (long long)M);
  if (M >= kMaxDim) return fail(GWB_ERR_SHAPE, "M must be below 2^31");
  if (M <= 128)
    return fail(GWB_ERR_SHAPE, "qmm_affine_noalloc runs the prefill GEMM: M must exceed 128 (M=%lld)", (long long)M);
  if (N == 0) return GWB_OK;
  if (K == 0) return fail(GWB_ERR_SHAPE, "qmm_affine_noalloc needs K > 0");
  GWB_TRY(need(y, "y"));
  GWB_TRY(need(x, "x"));
  GWB_TRY(need(wq, "wq"));
  GWB_TRY(need(scales, "scales"));
  GWB_TRY(need(biases, "biases"));
  if (bits == 2 && K % 64 != 0)
    return fail(GWB_ERR_UNSUPPORTED, "bits=2 needs K %% 64 == 0 on the tensor-core path (K=%lld)", (long long)K);
  return gwb::launch_tc2_affine_noalloc(x, M, wq, scales, biases, N, K, bits, group_size, y, as_stream(stream));
}

namespace {

// The GPTQ layout's dequant and qmm; zadd is added to each stored zero nibble
// (1: GPTQ's "+1" convention, 0: AWQ's stored zero as is).
gwb_status gptq_dequant_impl(const int32_t *qweight, const uint16_t *scales, const int32_t *qzeros,
                             const int32_t *g_idx, int64_t K, int64_t N, int group_size, uint16_t *w_out,
                             void *stream, int zadd) {
  GWB_TRY(check_gptq(K, N, group_size));
  if (N == 0 || K == 0) return GWB_OK;
  GWB_TRY(need(qweight, "qweight"));
  GWB_TRY(need(scales, "scales"));
  GWB_TRY(need(qzeros, "qzeros"));
  GWB_TRY(need(w_out, "w_out"));
  if (g_idx && !aligned16(g_idx)) return fail(GWB_ERR_ALIGN, "g_idx is not 16-byte aligned");
  gwb::launch_gptq_dequant(qweight, scales, qzeros, g_idx, K, N, group_size, w_out, as_stream(stream), zadd);
  return gwb::check_launch(zadd ? "gptq_dequant" : "awq_dequant");
}

gwb_status gptq_qmm_impl(const uint16_t *x, int64_t M, const int32_t *qweight, const uint16_t *scales,
                         const int32_t *qzeros, const int32_t *g_idx, int64_t K, int64_t N, int group_size,
                         uint16_t *y, void *stream, int zadd) {
  GWB_TRY(check_gptq(K, N, group_size));
  if (M < 0) return fail(GWB_ERR_INVALID_ARG, "negative M=%lld", (long long)M);
  if (M >= kMaxDim) return fail(GWB_ERR_SHAPE, "M must be below 2^31");
  if (M == 0 || N == 0) return GWB_OK;
  GWB_TRY(need(y, "y"));
  if (K == 0) return zero_fill(y, (size_t)M * N * 2, stream);
  GWB_TRY(need(x, "x"));
  GWB_TRY(need(qweight, "qweight"));
  GWB_TRY(need(scales, "scales"));
  GWB_TRY(need(qzeros, "qzeros"));
  if (g_idx && !aligned16(g_idx)) return fail(GWB_ERR_ALIGN, "g_idx is not 16-byte aligned");
  if (M <= 8)
    return gwb::launch_gemv_gptq(x, (int)M, qweight, scales, qzeros, g_idx, K, N, group_size, y, as_stream(stream),
                                 zadd);
  {   // the persistent stream-K GEMM without g_idx
    const gwb_status s =
        gwb::launch_tc2_gptq(x, M, qweight, scales, qzeros, g_idx, K, N, group_size, y, as_stream(stream), zadd);
    if (s != GWB_ERR_UNSUPPORTED) return s;
  }
  if (g_idx) {
    // act order: every in-feature has its own group, so the weights are dequantized
    // once (exactly as gwb_gptq_dequant writes them) into the library's scratch and
    // multiplied as dense fp16 on the persistent GEMM
    uint16_t *wd = nullptr;
    if (aligned16(x) && gwb::dequant_scratch(as_stream(stream), (size_t)N * (size_t)K * 2, &wd)) {
      gwb::launch_gptq_dequant(qweight, scales, qzeros, g_idx, K, N, group_size, wd, as_stream(stream), zadd);
      GWB_TRY(gwb::check_launch("gptq_dequant"));
      const gwb_status s = gwb::launch_tc2_f16(x, M, wd, N, K, y, as_stream(stream));
      if (s != GWB_ERR_UNSUPPORTED) return s;
    }
  }
  return gwb::launch_tc_gptq(x, M, qweight, scales, qzeros, g_idx, K, N, group_size, y, as_stream(stream), zadd);
}

}  // namespace

gwb_status gwb_gptq_dequant(const int32_t *qweight, const uint16_t *scales, const int32_t *qzeros,
                            const int32_t *g_idx, int64_t K, int64_t N, int group_size, uint16_t *w_out,
                            void *stream) {
  return gptq_dequant_impl(qweight, scales, qzeros, g_idx, K, N, group_size, w_out, stream, 1);
}

gwb_status gwb_gptq_qmm(const uint16_t *x, int64_t M, const int32_t *qweight, const uint16_t *scales,
                        const int32_t *qzeros, const int32_t *g_idx, int64_t K, int64_t N, int group_size,
                        uint16_t *y, void *stream) {
  return gptq_qmm_impl(x, M, qweight, scales, qzeros, g_idx, K, N, group_size, y, stream, 1);
}

gwb_status gwb_awq_dequant(const int32_t *qweight, const uint16_t *scales, const int32_t *qzeros, int64_t K,
                           int64_t N, int group_size, uint16_t *w_out, void *stream) {
  return gptq_dequant_impl(qweight, scales, qzeros, nullptr, K, N, group_size, w_out, stream, 0);
}

gwb_status gwb_awq_qmm(const uint16_t *x, int64_t M, const int32_t *qweight, const uint16_t *scales,
                       const int32_t *qzeros, int64_t K, int64_t N, int group_size, uint16_t *y, void *stream) {
  return gptq_qmm_impl(x, M, qweight, scales, qzeros, nullptr, K, N, group_size, y, stream, 0);
}

gwb_status gwb_quant_per_token_i8(const uint16_t *x, int64_t M, int64_t K, int8_t *qx, float *sx, void *stream) {
  if (M < 0 || K < 0) return fail(GWB_ERR_INVALID_ARG, "negative size (M=%lld, K=%lld)", (long long)M, (long long)K);
  if (M >= kMaxDim || K >= kMaxDim) return fail(GWB_ERR_SHAPE, "M and K must be below 2^31");
  if (M == 0) return GWB_OK;
  GWB_TRY(need(sx, "sx"));
  if (K > 0) {
    GWB_TRY(need(x, "x"));
    GWB_TRY(need(qx, "qx"));
  }
  gwb::launch_quant_per_token_i8(x, M, K, qx, sx, as_stream(stream));
  return gwb::check_launch("quant_per_token_i8");
}

gwb_status gwb_qpack_sym_i4(const float *w, int64_t N, int64_t K, uint32_t *wq, float *sw, void *stream) {
  if (N < 0 || K < 0) return fail(GWB_ERR_INVALID_ARG, "negative size (N=%lld, K=%lld)", (long long)N, (long long)K);
  if (N >= kMaxDim || K >= kMaxDim) return fail(GWB_ERR_SHAPE, "N and K must be below 2^31");
  if (K % 32 != 0) return fail(GWB_ERR_SHAPE, "K=%lld is not a multiple of 32", (long long)K);
  if (N == 0) return GWB_OK;
  GWB_TRY(need(sw, "sw"));
  if (K > 0) {
    GWB_TRY(need(w, "w"));
    GWB_TRY(need(wq, "wq"));
  }
  gwb::launch_qpack_sym_i4(w, N, K, wq, sw, as_stream(stream));
  return gwb::check_launch("qpack_sym_i4");
}

gwb_status gwb_gemm_i8i4(const int8_t *qx, const float *sx, int64_t M, const uint32_t *wq, const float *sw,
                         int64_t N, int64_t K, uint16_t *y, int32_t *acc, void *stream) {
  if (M < 0 || N < 0 || K < 0)
    return fail(GWB_ERR_INVALID_ARG, "negative size (M=%lld, N=%lld, K=%lld)", (long long)M, (long long)N,
                (long long)K);
  if (M >= kMaxDim || N >= kMaxDim) return fail(GWB_ERR_SHAPE, "M and N must be below 2^31");
  if (K % 32 != 0) return fail(GWB_ERR_SHAPE, "K=%lld is not a multiple of 32", (long long)K);
  if (K > 131072) return fail(GWB_ERR_SHAPE, "K=%lld exceeds 131072 (int32 partial-sum bound)", (long long)K);
  if (!y && !acc) return fail(GWB_ERR_INVALID_ARG, "at least one of y and acc must be non-NULL");
  if (y && !aligned16(y)) return fail(GWB_ERR_ALIGN, "y is not 16-byte aligned");
  if (acc && !aligned16(acc)) return fail(GWB_ERR_ALIGN, "acc is not 16-byte aligned");
  if (M == 0 || N == 0) return GWB_OK;
  if (K == 0) {
    if (y) GWB_TRY(zero_fill(y, (size_t)M * N * 2, stream));
    if (acc) GWB_TRY(zero_fill(acc, (size_t)M * N * 4, stream));
    return GWB_OK;
  }
  GWB_TRY(need(qx, "qx"));
  GWB_TRY(need(sx, "sx"));
  GWB_TRY(need(wq, "wq"));
  GWB_TRY(need(sw, "sw"));
  return gwb::launch_tc2_i8i4(qx, sx, M, wq, sw, N, K, y, acc, as_stream(stream));
}

gwb_status gwb_qpack_sym_i8(const float *w, int64_t N, int64_t K, int8_t *wq, float *sw, void *stream) {
  if (N < 0 || K < 0) return fail(GWB_ERR_INVALID_ARG, "negative size (N=%lld, K=%lld)", (long long)N, (long long)K);
  if (N >= kMaxDim || K >= kMaxDim) return fail(GWB_ERR_SHAPE, "N and K must be below 2^31");
  if (K % 16 != 0) return fail(GWB_ERR_SHAPE, "K=%lld is not a multiple of 16", (long long)K);
  if (N == 0) return GWB_OK;
  GWB_TRY(need(sw, "sw"));
  if (K > 0) {
    GWB_TRY(need(w, "w"));
    GWB_TRY(need(wq, "wq"));
  }
  gwb::launch_qpack_sym_i8(w, N, K, wq, sw, as_stream(stream));
  return gwb::check_launch("qpack_sym_i8");
}

gwb_status gwb_gemm_i8i8(const int8_t *qx, const float *sx, int64_t M, const int8_t *wq, const float *sw,
                         int64_t N, int64_t K, uint16_t *y, int32_t *acc, void *stream) {
  if (M < 0 || N < 0 || K < 0)
    return fail(GWB_ERR_INVALID_ARG, "negative size (M=%lld, N=%lld, K=%lld)", (long long)M, (long long)N,
                (long long)K);
  if (M >= kMaxDim || N >= kMaxDim) return fail(GWB_ERR_SHAPE, "M and N must be below 2^31");
  if (K % 16 != 0) return fail(GWB_ERR_SHAPE, "K=%lld is not a multiple of 16", (long long)K);
  if (K > 131072) return fail(GWB_ERR_SHAPE, "K=%lld exceeds 131072 (int32 accumulator bound)", (long long)K);
  if (!y && !acc) return fail(GWB_ERR_INVALID_ARG, "at least one of y and acc must be non-NULL");
  if (M == 0 || N == 0) return GWB_OK;
  if (K == 0) {
    if (y) GWB_TRY(zero_fill(y, (size_t)M * N * 2, stream));
    if (acc) GWB_TRY(zero_fill(acc, (size_t)M * N * 4, stream));
    return GWB_OK;
  }
  GWB_TRY(need(qx, "qx"));
  GWB_TRY(need(sx, "sx"));
  GWB_TRY(need(wq, "wq"));
  GWB_TRY(need(sw, "sw"));
  if (!aligned16(qx) || !aligned16(wq)) return fail(GWB_ERR_ALIGN, "qx and wq must be 16-byte aligned");
  if (M <= 8 && K % 512 == 0) {
    // decode: the weight-streaming kernel (falls through when the rows do not fit on chip)
    const gwb_status s = gwb::launch_gemv_i8w8(qx, sx, (int)M, wq, sw, N, K, y, acc, as_stream(stream));
    if (s != GWB_ERR_UNSUPPORTED) return s;
  }
  return gwb::launch_tc2_i8i8(qx, sx, M, wq, sw, N, K, y, acc, as_stream(stream));
}

gwb_status gwb_gemv_w4a8(const uint16_t *x, int64_t M, const uint32_t *wq, const float *sw, int64_t N, int64_t K,
                         uint16_t *y, void *stream) {
  if (M < 0 || N < 0 || K < 0)
    return fail(GWB_ERR_INVALID_ARG, "negative size (M=%lld, N=%lld, K=%lld)", (long long)M, (long long)N,
                (long long)K);
  if (N >= kMaxDim || K >= kMaxDim) return fail(GWB_ERR_SHAPE, "N and K must be below 2^31");
  if (M > 8) return fail(GWB_ERR_SHAPE, "gemv_w4a8 takes at most 8 tokens (M=%lld)", (long long)M);
  if (K % 512 != 0 || K > 16384)
    return fail(GWB_ERR_UNSUPPORTED, "gemv_w4a8 needs K %% 512 == 0 and K <= 16384 (K=%lld)", (long long)K);
  if (M == 0 || N == 0) return GWB_OK;
  GWB_TRY(need(y, "y"));
  if (K == 0) return zero_fill(y, (size_t)M * N * 2, stream);
  GWB_TRY(need(x, "x"));
  GWB_TRY(need(wq, "wq"));
  GWB_TRY(need(sw, "sw"));
  if (!aligned16(x)) return fail(GWB_ERR_ALIGN, "x is not 16-byte aligned");
  const gwb_status s = gwb::launch_gemv_w4a8(x, (int)M, wq, sw, N, K, y, as_stream(stream));
  return s == GWB_ERR_UNSUPPORTED
             ? fail(GWB_ERR_UNSUPPORTED,
                    "gemv_w4a8: the staged activations of %lld tokens x K=%lld do not fit on chip; quantize with "
                    "quant_per_token_i8 and call gemm_i8i4", (long long)M, (long long)K)
             : s;
}

}  // extern "C"
