// W4A8 at decode with the activation quantization fused: one launch of the
// kernel in gemv_pipe.cuh (kOpW4A8) quantizes x to int8 per token while it is
// staged and multiplies it with the symmetric int4 weights, so the int8
// activations never reach memory (the "staged" lowering of executorch PR
// #24467, mlx::int8_int4_gemm).  The result is bit-identical to
// quant_per_token_i8 followed by gemm_i8i4.
#include "gemv_pipe.cuh"

namespace gwb {

gwb_status launch_gemv_w4a8(const uint16_t *x, int M, const uint32_t *wq, const float *sw, int64_t N, int64_t K,
                            uint16_t *y, cudaStream_t st) {
  const int MP = pad_tokens(M);
  PipeIn in;
  in.x = x; in.M = M; in.wq = wq; in.sw = sw; in.N = N; in.K = K; in.y = y;
  // the 4-bit codes go through the MMAs 64 k at a time (the "group" of the
  // kernel's layout), which keeps every partial sum an exact fp32 integer
  if (MP == 1) return run_pipe<4, 64, 1, kOpW4A8>(in, st);
  if (MP == 2) return run_pipe<4, 64, 2, kOpW4A8>(in, st);
  if (MP == 4) return run_pipe<4, 64, 4, kOpW4A8>(in, st);
  return run_pipe<4, 64, 8, kOpW4A8>(in, st);
}

}  // namespace gwb
