// Fused decode product: y = (resid +) (silu(gate) * up) W^T in one launch of the
// kernel in gemv_pipe.cuh (kOpSilu), as MlxInt8Weight::gemv_silu_gate and
// gemv_silu_gate_resid do for MLX 8-bit weights (metrale_gpu_runtime/mlx_int8.rs):
// the product silu(gate) * up is formed in fp32 while the activations are
// staged and is never written to memory.
#include "gemv_pipe.cuh"

namespace gwb {

gwb_status launch_gemv_silu_gate(const uint16_t *gate, const uint16_t *up, int M, const uint32_t *wq,
                                 const uint16_t *scales, const uint16_t *biases, int64_t N, int64_t K, int bits,
                                 int gs, const uint16_t *resid, uint16_t *y, cudaStream_t st) {
  const int MP = pad_tokens(M);
  PipeIn in;
  in.x = gate; in.x2 = up; in.resid = resid; in.M = M; in.N = N; in.K = K;
  in.wq = wq; in.scales = scales; in.biases = biases; in.y = y;
#define GWB_GP(B, S, P) \
  if (bits == B && gs == S && MP == P) return run_pipe<B, S, P, kOpSilu>(in, st);
#define GWB_GP_MP(B, S) GWB_GP(B, S, 1) GWB_GP(B, S, 2) GWB_GP(B, S, 4) GWB_GP(B, S, 8)
  GWB_GP_MP(2, 64) GWB_GP_MP(2, 128)
  GWB_GP_MP(4, 32) GWB_GP_MP(4, 64) GWB_GP_MP(4, 128)
  GWB_GP_MP(8, 32) GWB_GP_MP(8, 64) GWB_GP_MP(8, 128)
#undef GWB_GP_MP
#undef GWB_GP
  return GWB_ERR_UNSUPPORTED;
}

}  // namespace gwb
