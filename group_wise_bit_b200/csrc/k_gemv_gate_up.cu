// Fused decode product: gate_y = x W_gate^T and up_y = x W_up^T in one launch of
// the kernel in gemv_pipe.cuh (kOpDual), as gemv_gate_up does for MLX 8-bit
// weights (metrale_gpu_runtime/mlx_int8.rs): both weights share the shape,
// bits and group size, and the activations are staged once per CTA for both.
#include "gemv_pipe.cuh"

namespace gwb {

gwb_status launch_gemv_gate_up(const uint16_t *x, int M, const uint32_t *wq_gate, const uint16_t *sc_gate,
                               const uint16_t *bi_gate, const uint32_t *wq_up, const uint16_t *sc_up,
                               const uint16_t *bi_up, int64_t N, int64_t K, int bits, int gs, uint16_t *y_gate,
                               uint16_t *y_up, cudaStream_t st) {
  const int MP = pad_tokens(M);
  PipeIn in;
  in.x = x; in.M = M; in.N = N; in.K = K;
  in.wq = wq_gate; in.scales = sc_gate; in.biases = bi_gate; in.y = y_gate;
  in.wq2 = wq_up; in.scales2 = sc_up; in.biases2 = bi_up; in.y2 = y_up;
#define GWB_GP(B, S, P) \
  if (bits == B && gs == S && MP == P) return run_pipe<B, S, P, kOpDual>(in, st);
#define GWB_GP_MP(B, S) GWB_GP(B, S, 1) GWB_GP(B, S, 2) GWB_GP(B, S, 4) GWB_GP(B, S, 8)
  GWB_GP_MP(2, 64) GWB_GP_MP(2, 128)
  GWB_GP_MP(4, 32) GWB_GP_MP(4, 64) GWB_GP_MP(4, 128)
  GWB_GP_MP(8, 32) GWB_GP_MP(8, 64) GWB_GP_MP(8, 128)
#undef GWB_GP_MP
#undef GWB_GP
  return GWB_ERR_UNSUPPORTED;
}

}  // namespace gwb
