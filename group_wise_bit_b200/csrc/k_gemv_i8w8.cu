// W8A8 at decode: int8 activations (already quantized per token) x int8 weights
// with one scale per row, exact int32 sums, in one launch of the kernel in
// gemv_pipe.cuh (kOpI8W8).  Serves gwb_gemm_i8i8 for M <= 8.
#include "gemv_pipe.cuh"

namespace gwb {

gwb_status launch_gemv_i8w8(const int8_t *qx, const float *sx, int M, const int8_t *wq, const float *sw, int64_t N,
                            int64_t K, uint16_t *y, int32_t *acc, cudaStream_t st) {
  const int MP = pad_tokens(M);
  PipeIn in;
  in.x = reinterpret_cast<const uint16_t *>(qx);   // int8 rows; the kernel reads them as such
  in.M = M;
  in.wq = reinterpret_cast<const uint32_t *>(wq);   // four int8 codes per word, lowest k in the low byte
  in.sw = sw; in.sx = sx; in.acc = acc; in.N = N; in.K = K; in.y = y;
  // the codes go through the MMAs 64 k at a time (the "group" of the kernel's
  // layout): each chain is an exact fp32 integer
  if (MP == 1) return run_pipe<8, 64, 1, kOpI8W8>(in, st);
  if (MP == 2) return run_pipe<8, 64, 2, kOpI8W8>(in, st);
  if (MP == 4) return run_pipe<8, 64, 4, kOpI8W8>(in, st);
  return run_pipe<8, 64, 8, kOpI8W8>(in, st);
}

}  // namespace gwb
