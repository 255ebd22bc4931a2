// Per-tile tensor-core (tcgen05) GEMM of the fused dequant + matmul, for the
// layouts the persistent kernel (k_gemm_tc2.cu) does not take:
//   * the MLX affine layout (bf16 activations, kind::f16 with bf16 operands)
//     with an odd number of groups per row or scale tensors without a common
//     stride,
//   * the GPTQ layout (fp16 activations, kind::f16 with fp16 operands) with an
//     act-order g_idx when no dequant scratch can be had.
//
// The problem is computed transposed ("swap AB"): the tensor core's M side is
// 128 output features (rows of W), its N side is BT tokens.  One CTA owns a
// 128 x BT output tile and the whole K loop:
//
//   warp 0      TMA producer: per K step, the activation tile (BT x BK, 128-byte
//               swizzled, zero-filled past M/K) and the packed weight tile
//               (raw words) into a ring of STAGES shared-memory stages.
//   warp 1      TMEM allocation and the single MMA-issuing thread: waits for the
//               dequantized A tile and the activation tile of a stage, issues
//               BK/16 tcgen05.mma into the TMEM accumulator and
//               commits the stage back to the producer.
//   warps 2-9   dequantizers: unpack the stage's raw words in registers, apply
//               the group scale / bias (or zero), and store the 128 x BK A tile
//               in the same 128-byte-swizzled K-major layout TMA produces, then
//               signal the MMA thread; after the K loop they drain TMEM with
//               tcgen05.ld and write the output tile.
//
// Every mbarrier wait is bounded (see ptx.cuh); on a timeout the CTA stops
// issuing work, drains what it issued, frees its TMEM and exits.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "dequant.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace gwb {
namespace {
using namespace dq;

constexpr int kTcThreads = 320;
constexpr int kDqThreads = 256;
constexpr int kTileN = 128;  // output features per CTA (tensor-core M)
constexpr int kMaxSmem = 232448;

enum class Fmt { Affine, Gptq };

struct TcArgs {
  int M, N, K, gs;
  const uint16_t *scales;   // affine: bf16 [N, K/gs];   gptq: fp16 [K/gs, N]
  const uint16_t *biases;   // affine: bf16 [N, K/gs]
  const int32_t *qzeros;    // gptq: [K/gs, N/8]
  const int32_t *g_idx;     // gptq: [K] or null
  uint16_t *y;              // bf16 (affine) or fp16 (gptq) [M, N]
  int staged_scales;        // 1: the producer copies each stage's scales (and zeros) into shared memory
  int zadd;                 // gptq: added to the stored zero (1: GPTQ's convention, 0: AWQ's)
};

template <Fmt F, int BITS>
struct Traits;
template <int BITS>
struct Traits<Fmt::Affine, BITS> {
  static constexpr int BK = 64;                       // bf16: 64 elements = 128 bytes per row
  static constexpr int RAW_BYTES = kTileN * BK * BITS / 8;
  static constexpr int NMMA = BK / 16;
  static constexpr int SC_BYTES = 1024;               // (scales, biases) x 128 rows x an aligned pair of groups
};
template <>
struct Traits<Fmt::Gptq, 4> {
  static constexpr int BK = 64;
  static constexpr int RAW_BYTES = (BK / 8) * kTileN * 4;
  static constexpr int NMMA = BK / 16;
  static constexpr int SC_BYTES = 1024;               // 2 groups x (128 fp16 scales + 16 qzeros words)
};

// ---------------------------------------------------------------- the kernel
template <Fmt F, int BITS, int BT, int STAGES>
__global__ void __launch_bounds__(kTcThreads, 1)
    k_tc(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w, const TcArgs args) {
  using T = Traits<F, BITS>;
  constexpr int BK = T::BK;
  constexpr int B_BYTES = BT * 128;
  constexpr int A_BYTES = kTileN * 128;
  constexpr int STAGE = B_BYTES + A_BYTES + T::RAW_BYTES + T::SC_BYTES;
  constexpr uint32_t NCOLS = BT < 32 ? 32 : BT;
  constexpr uint32_t IDESC = (F == Fmt::Gptq) ? make_idesc(1, 0, kTileN, BT) : make_idesc(1, 1, kTileN, BT);

  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char *base = align_smem_1024(smem_raw);
  uint64_t *full = reinterpret_cast<uint64_t *>(base + STAGES * STAGE);
  uint64_t *afull = full + STAGES;
  uint64_t *empty = afull + STAGES;
  uint64_t *accf = empty + STAGES;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(accf + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * kTileN, m0 = blockIdx.y * BT;
  const int nk = (args.K + BK - 1) / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; s++) {
      mbar_init(&full[s], 1 + 32);   // producer arrive.expect_tx + one cp.async arrive per producer lane
      mbar_init(&afull[s], kDqThreads / 32);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accf, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_w);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, NCOLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // Lane 0 issues the TMA loads; every lane copies a share of the stage's
    // scales / biases (GPTQ: scales and qzeros words) with cp.async, so the
    // dequantizers find them in shared memory when the stage completes.
    int issued = 0;
    for (int i = 0; i < nk; i++) {
      const int s = i % STAGES, r = i / STAGES;
      if (!mbar_wait(&empty[s], (r & 1) ^ 1)) { *abort_flag = 1; break; }
      unsigned char *st = base + s * STAGE;
      if (lane == 0) {
        mbar_arrive_expect_tx(&full[s], B_BYTES + T::RAW_BYTES);
        tma_load_2d(st, &tm_x, i * BK, m0, &full[s]);
        if constexpr (F == Fmt::Gptq) tma_load_2d(st + B_BYTES + A_BYTES, &tm_w, n0, i * (BK / 8), &full[s]);
        else tma_load_2d(st + B_BYTES + A_BYTES, &tm_w, i * (BK * BITS / 32), n0, &full[s]);
      }
      unsigned char *sc = st + B_BYTES + A_BYTES + T::RAW_BYTES;
      if constexpr (F == Fmt::Affine) {
        if (args.staged_scales) {
          const int G = args.K / args.gs;
          const int gp = ((i * BK) / args.gs) & ~1;
          for (int e = lane; e < 2 * kTileN; e += 32) {   // (array, row) -> 4 bytes: groups gp, gp+1
            const int arr = e / kTileN, row = e % kTileN, n = n0 + row;
            const bool ok = n < args.N && gp < G;
            const uint16_t *src = (arr ? args.biases : args.scales) + (ok ? (int64_t)n * G + gp : 0);
            cp_async_4(sc + e * 4, src, ok ? 4u : 0u);
          }
        }
      } else if constexpr (F == Fmt::Gptq) {
        if (args.staged_scales) {
          const int G = args.K / args.gs;
          const int gp = (i * BK) / args.gs;
          {   // scales: 2 groups x 128 columns = 32 chunks of 16 bytes, one per lane
            const int gi = lane >> 4, ch = lane & 15, g = gp + gi, n = n0 + ch * 8;
            const bool ok = g < G && n < args.N;
            cp_async_16(sc + lane * 16, args.scales + (ok ? (int64_t)g * args.N + n : 0), ok ? 16u : 0u);
          }
          {   // qzeros: 2 groups x 16 words, one word per lane
            const int gi = lane >> 4, wz = lane & 15, g = gp + gi, n = n0 + wz * 8;
            const bool ok = g < G && n < args.N;
            cp_async_4(sc + 512 + lane * 4, args.qzeros + (ok ? (int64_t)g * (args.N / 8) + n / 8 : 0), ok ? 4u : 0u);
          }
        }
      }
      cp_async_arrive_noinc(&full[s]);
      issued = i + 1;
    }
    // Drain: every issued copy has landed before the CTA can exit.
    for (int i = issued - STAGES < 0 ? 0 : issued - STAGES; i < issued; i++)
      mbar_wait(&full[i % STAGES], (i / STAGES) & 1);
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int done = 0;
      for (int i = 0; i < nk; i++) {
        const int s = i % STAGES, ph = (i / STAGES) & 1;
        if (*abort_flag) break;
        if (!mbar_wait(&afull[s], ph) || !mbar_wait(&full[s], ph)) { *abort_flag = 1; break; }
        tc_fence_after();
        unsigned char *st = base + s * STAGE;
        const uint32_t a0 = smem_u32(st + B_BYTES), b0 = smem_u32(st);
#pragma unroll
        for (int kk = 0; kk < T::NMMA; kk++) {
          const uint64_t ad = smem_desc_sw128(a0 + kk * 32), bd = smem_desc_sw128(b0 + kk * 32);
          umma_f16(tmem, ad, bd, IDESC, (i | kk) != 0);
        }
        umma_commit(&empty[s]);
        done = i + 1;
      }
      umma_commit(accf);
      // Wait for the commits' arrivals so no asynchronous arrive targets this
      // CTA's shared memory after it exits.
      for (int i = done - STAGES < 0 ? 0 : done - STAGES; i < done; i++)
        mbar_wait(&empty[i % STAGES], (i / STAGES) & 1);
    }
  } else {
    // ------------------------------------------------------------ dequantizers
    const int d = threadIdx.x - 64;
    const int r = d & (kTileN - 1), h = d >> 7;   // tile row, half of the K step
    const int n = n0 + r;
    const int nc = n < args.N ? n : args.N - 1;    // clamped row for scale loads
    for (int i = 0; i < nk; i++) {
      const int s = i % STAGES, ph = (i / STAGES) & 1;
      // Scale data for this thread's half step (loaded before the wait so the
      // latency overlaps it).
      const int kh = i * BK + h * (BK / 2);        // first k of this half step
      float sf = 0.f, bfv = 0.f;
      uint32_t z2[4], s2[4];
      if constexpr (F == Fmt::Affine) {
        if (!args.staged_scales) {
          const int G = args.K / args.gs;
          int g = kh / args.gs;
          g = g < G ? g : G - 1;
          sf = bf16_val(__ldg(args.scales + (int64_t)nc * G + g));
          bfv = bf16_val(__ldg(args.biases + (int64_t)nc * G + g));
        }
      } else if constexpr (F == Fmt::Gptq) {
        if (args.g_idx == nullptr && !args.staged_scales) {
          const int G = args.K / args.gs;
          int g = kh / args.gs;
          g = g < G ? g : G - 1;
          const uint32_t sv = __ldg(args.scales + (int64_t)g * args.N + nc);
          const uint32_t zw = (uint32_t)__ldg(args.qzeros + (int64_t)g * (args.N / 8) + nc / 8);
          const uint32_t zv = 0x6400u | (((zw >> ((nc % 8) * 4)) & 0xFu) + (uint32_t)args.zadd);
#pragma unroll
          for (int p = 0; p < 4; p++) { s2[p] = sv | (sv << 16); z2[p] = zv | (zv << 16); }
        }
      }
      if (*abort_flag) break;
      if (!mbar_wait(&full[s], ph)) { *abort_flag = 1; break; }
      unsigned char *st = base + s * STAGE;
      unsigned char *A = st + B_BYTES;
      const unsigned char *R = st + B_BYTES + A_BYTES;
      if constexpr (F == Fmt::Affine) {
        if (args.staged_scales) {   // this half step's group within the staged pair
          int idx = kh / args.gs - (((i * BK) / args.gs) & ~1);
          idx = idx < 1 ? idx : 1;
          const uint16_t *sc = reinterpret_cast<const uint16_t *>(R + T::RAW_BYTES);
          sf = bf16_val(sc[r * 2 + idx]);
          bfv = bf16_val(sc[(kTileN + r) * 2 + idx]);
        }
      } else if constexpr (F == Fmt::Gptq) {
        if (args.g_idx == nullptr && args.staged_scales) {
          int idx = kh / args.gs - (i * BK) / args.gs;
          idx = idx < 1 ? idx : 1;
          const uint16_t *sc = reinterpret_cast<const uint16_t *>(R + T::RAW_BYTES);
          const uint32_t *zc = reinterpret_cast<const uint32_t *>(R + T::RAW_BYTES + 512);
          const uint32_t sv = sc[idx * kTileN + r];
          const uint32_t zv = 0x6400u | (((zc[idx * 16 + r / 8] >> ((r % 8) * 4)) & 0xFu) + (uint32_t)args.zadd);
#pragma unroll
          for (int p = 0; p < 4; p++) { s2[p] = sv | (sv << 16); z2[p] = zv | (zv << 16); }
        }
      }
      if constexpr (F == Fmt::Affine && BITS == 4) {
        const uint4 raw = *reinterpret_cast<const uint4 *>(R + (r * 8 + h * 4) * 4);
        const __nv_bfloat162 s2b = __floats2bfloat162_rn(sf, sf), b2b = __floats2bfloat162_rn(bfv, bfv);
        const uint32_t wv[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int j = 0; j < 4; j++)
          *reinterpret_cast<uint4 *>(A + sw128_off(r, 4 * h + j)) = dq_affine4(wv[j], s2b, b2b);
      } else if constexpr (F == Fmt::Affine && BITS == 2) {
        const uint2 raw = *reinterpret_cast<const uint2 *>(R + (r * 4 + h * 2) * 4);
        const __nv_bfloat162 s2q = __floats2bfloat162_rn(sf, sf * 0.25f), b2b = __floats2bfloat162_rn(bfv, bfv);
        uint4 c0, c1;
        dq_affine2(raw.x, s2q, b2b, c0, c1);
        *reinterpret_cast<uint4 *>(A + sw128_off(r, 4 * h + 0)) = c0;
        *reinterpret_cast<uint4 *>(A + sw128_off(r, 4 * h + 1)) = c1;
        dq_affine2(raw.y, s2q, b2b, c0, c1);
        *reinterpret_cast<uint4 *>(A + sw128_off(r, 4 * h + 2)) = c0;
        *reinterpret_cast<uint4 *>(A + sw128_off(r, 4 * h + 3)) = c1;
      } else if constexpr (F == Fmt::Affine && BITS == 8) {
        const uint4 *rp = reinterpret_cast<const uint4 *>(R + (r * 16 + h * 8) * 4);
        const uint4 ra = rp[0], rb = rp[1];
        *reinterpret_cast<uint4 *>(A + sw128_off(r, 4 * h + 0)) = dq_affine8(ra.x, ra.y, sf, bfv);
        *reinterpret_cast<uint4 *>(A + sw128_off(r, 4 * h + 1)) = dq_affine8(ra.z, ra.w, sf, bfv);
        *reinterpret_cast<uint4 *>(A + sw128_off(r, 4 * h + 2)) = dq_affine8(rb.x, rb.y, sf, bfv);
        *reinterpret_cast<uint4 *>(A + sw128_off(r, 4 * h + 3)) = dq_affine8(rb.z, rb.w, sf, bfv);
      } else if constexpr (F == Fmt::Gptq) {
        const uint32_t *Rw = reinterpret_cast<const uint32_t *>(R);
#pragma unroll
        for (int j = 0; j < 4; j++) {
          const int kq = 4 * h + j;                  // k-octet within the step = chunk index
          const uint32_t w = Rw[kq * kTileN + r];
          if (args.g_idx != nullptr) {
#pragma unroll
            for (int p = 0; p < 4; p++) {
              uint32_t sv[2], zv[2];
#pragma unroll
              for (int e = 0; e < 2; e++) {
                const int k = i * BK + kq * 8 + 2 * p + e;
                const int g = k < args.K ? __ldg(args.g_idx + k) : 0;
                sv[e] = __ldg(args.scales + (int64_t)g * args.N + nc);
                const uint32_t zw = (uint32_t)__ldg(args.qzeros + (int64_t)g * (args.N / 8) + nc / 8);
                zv[e] = 0x6400u | (((zw >> ((nc % 8) * 4)) & 0xFu) + (uint32_t)args.zadd);
              }
              s2[p] = sv[0] | (sv[1] << 16);
              z2[p] = zv[0] | (zv[1] << 16);
            }
          }
          *reinterpret_cast<uint4 *>(A + sw128_off(r, kq)) = dq_gptq(w, z2, s2);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&afull[s]);
    }

    // ------------------------------------------------------------ epilogue
    if (!*abort_flag && mbar_wait(accf, 0)) {
      tc_fence_after();
      const int q = warp & 3, eh = (warp - 2) >> 2;
      const int row = n0 + 32 * q + lane;
      for (int ch = eh; ch < BT / 16; ch += 2) {
        uint32_t v[16];
        tmem_ld16(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(ch * 16), v);
        tmem_ld_wait();
        if (row < args.N) {
#pragma unroll
          for (int j = 0; j < 16; j++) {
            const int m = m0 + ch * 16 + j;
            if (m < args.M) {
              const int64_t o = (int64_t)m * args.N + row;
              if constexpr (F == Fmt::Gptq) {
                args.y[o] = __half_as_ushort(__float2half_rn(__uint_as_float(v[j])));
              } else {
                args.y[o] = __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(v[j])));
              }
            }
          }
        }
      }
    } else {
      *abort_flag = 1;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, NCOLS);
  }
}

// ---------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

gwb_status make_map(CUtensorMap *m, CUtensorMapDataType dt, const void *ptr, uint64_t inner, uint64_t outer,
                    uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw) {
  auto fn = encode_fn();
  if (!fn) return fail(GWB_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t es[2] = {1, 1};
  CUresult r = fn(m, dt, 2, const_cast<void *>(ptr), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(GWB_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return GWB_OK;
}

template <Fmt F, int BITS, int BT>
constexpr int stages_for() {
  constexpr int stage = BT * 128 + kTileN * 128 + Traits<F, BITS>::RAW_BYTES + Traits<F, BITS>::SC_BYTES;
  constexpr int s = (kMaxSmem - 2048) / stage;
  return s > 6 ? 6 : s;
}

template <Fmt F, int BITS, int BT>
gwb_status run_tc(const CUtensorMap &tx, const CUtensorMap &tw, const TcArgs &a, cudaStream_t st) {
  constexpr int STAGES = stages_for<F, BITS, BT>();
  static_assert(STAGES >= 2, "shared memory too small");
  constexpr int stage = BT * 128 + kTileN * 128 + Traits<F, BITS>::RAW_BYTES + Traits<F, BITS>::SC_BYTES;
  const size_t smem = (size_t)STAGES * stage + 1024 + 256;
  auto kern = k_tc<F, BITS, BT, STAGES>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return fail(GWB_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
  dim3 grid((a.N + kTileN - 1) / kTileN, (a.M + BT - 1) / BT);
  kern<<<grid, kTcThreads, smem, st>>>(tx, tw, a);
  return check_launch("tensor-core GEMM");
}

int pick_bt(int64_t M) { return M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : M <= 128 ? 128 : 256; }

// Builds the activation tensor map for the chosen token tile and launches.
template <Fmt F, int BITS>
gwb_status dispatch_bt(int64_t M, const void *xptr, CUtensorMapDataType xdt, int xelem, const CUtensorMap &tw,
                       const TcArgs &a, cudaStream_t st) {
  const int BT = pick_bt(M);
  CUtensorMap tx;
  const int bk_elems = 128 / xelem;
  gwb_status s = make_map(&tx, xdt, xptr, (uint64_t)a.K, (uint64_t)a.M, (uint64_t)a.K * xelem, bk_elems,
                          (uint32_t)BT, CU_TENSOR_MAP_SWIZZLE_128B);
  if (s != GWB_OK) return s;
  switch (BT) {
    case 16: return run_tc<F, BITS, 16>(tx, tw, a, st);
    case 32: return run_tc<F, BITS, 32>(tx, tw, a, st);
    case 64: return run_tc<F, BITS, 64>(tx, tw, a, st);
    case 128: return run_tc<F, BITS, 128>(tx, tw, a, st);
    default: return run_tc<F, BITS, 256>(tx, tw, a, st);
  }
}

}  // namespace

gwb_status launch_tc_affine(const uint16_t *x, int64_t M, const uint32_t *wq, const uint16_t *scales,
                            const uint16_t *biases, int64_t N, int64_t K, int bits, int gs, uint16_t *y,
                            cudaStream_t st) {
  TcArgs a{};
  a.M = (int)M; a.N = (int)N; a.K = (int)K; a.gs = gs;
  a.scales = scales; a.biases = biases; a.y = y;
  // 4-byte copies of aligned group pairs: an even group count and 4-byte aligned arrays.
  a.staged_scales = ((K / gs) % 2 == 0 && (((uintptr_t)scales | (uintptr_t)biases) & 3) == 0) ? 1 : 0;
  CUtensorMap tw;
  const uint64_t words = (uint64_t)K * bits / 32;
  gwb_status s = make_map(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT32, wq, words, (uint64_t)N, words * 4,
                          (uint32_t)(64 * bits / 32), (uint32_t)kTileN, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (s != GWB_OK) return s;
  if (bits == 4) return dispatch_bt<Fmt::Affine, 4>(M, x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, tw, a, st);
  if (bits == 8) return dispatch_bt<Fmt::Affine, 8>(M, x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, tw, a, st);
  return dispatch_bt<Fmt::Affine, 2>(M, x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, tw, a, st);
}

gwb_status launch_tc_gptq(const uint16_t *x, int64_t M, const int32_t *qweight, const uint16_t *scales,
                          const int32_t *qzeros, const int32_t *g_idx, int64_t K, int64_t N, int gs,
                          uint16_t *y, cudaStream_t st, int zadd) {
  TcArgs a{};
  a.M = (int)M; a.N = (int)N; a.K = (int)K; a.gs = gs;
  a.scales = scales; a.qzeros = qzeros; a.g_idx = g_idx; a.y = y;
  a.zadd = zadd;
  // 16-byte scale copies and 4-byte qzeros copies need those alignments.
  a.staged_scales = (g_idx == nullptr && ((uintptr_t)scales & 15) == 0 && ((uintptr_t)qzeros & 3) == 0) ? 1 : 0;
  CUtensorMap tw;
  gwb_status s = make_map(&tw, CU_TENSOR_MAP_DATA_TYPE_INT32, qweight, (uint64_t)N, (uint64_t)(K / 8),
                          (uint64_t)N * 4, (uint32_t)kTileN, 8u, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (s != GWB_OK) return s;
  return dispatch_bt<Fmt::Gptq, 4>(M, x, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, tw, a, st);
}

}  // namespace gwb
