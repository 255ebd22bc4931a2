// Decode GEMV (M <= 8 tokens) for the MLX affine layout: the plain product
// y = x W^T of the kernel in gemv_pipe.cuh.
#include "gemv_pipe.cuh"

namespace gwb {

gwb_status launch_gemv_pipe(const uint16_t *x, int M, const uint32_t *wq, const uint16_t *scales,
                            const uint16_t *biases, int64_t N, int64_t K, int bits, int gs, uint16_t *y,
                            cudaStream_t st) {
  const int MP = pad_tokens(M);
  PipeIn in;
  in.x = x; in.M = M; in.wq = wq; in.scales = scales; in.biases = biases; in.N = N; in.K = K; in.y = y;
#define GWB_GP(B, S, P) \
  if (bits == B && gs == S && MP == P) return run_pipe<B, S, P, kOpPlain>(in, st);
#define GWB_GP_MP(B, S) GWB_GP(B, S, 1) GWB_GP(B, S, 2) GWB_GP(B, S, 4) GWB_GP(B, S, 8)
  GWB_GP_MP(2, 64) GWB_GP_MP(2, 128)
  GWB_GP_MP(4, 32) GWB_GP_MP(4, 64) GWB_GP_MP(4, 128)
  GWB_GP_MP(8, 32) GWB_GP_MP(8, 64) GWB_GP_MP(8, 128)
#undef GWB_GP_MP
#undef GWB_GP
  return GWB_ERR_UNSUPPORTED;
}

}  // namespace gwb
