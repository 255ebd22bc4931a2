// GPTQ decode GEMV (M <= 8 tokens), streamed through shared memory.
//
//   y[t, n] = sum_k x[t, k] * s[g(k), n] * (q[k, n] - (z[g(k), n] + zadd))
//
// for the GPTQ layout: qweight int32 [K/8, N] holding eight 4-bit codes of
// consecutive in-features per word (lowest bits = lowest k), scales fp16
// [G, N], qzeros int32 [G, N/8] holding eight stored zeros per word along N
// (GPTQ adds 1 to the stored zero, AWQ adds nothing), g(k) = k / gs or
// g_idx[k] for act-order checkpoints; fp16 activations and output.
//
// Work: a strip is 32 output features, i.e. one 128-byte run of every qweight
// row.  A stage is 256 in-features of a strip: 32 runs of 128 bytes (4 KB of
// codes) plus, without g_idx, the strip's scales and zero words of the stage's
// groups.  One CTA of 8 warps per SM takes a contiguous range of strips and
// cuts its (strip, stage) list into 8 equal contiguous pieces, one per warp.
// A warp streams its stages through a private ring of D shared-memory slots:
// each lane issues one bulk copy (one 128-byte run), and two more lanes per
// group copy the scale and zero runs, all completing on the slot's mbarrier;
// a slot is refilled as soon as the warp has read it.  A warp holds only a few
// stages, so most of a CTA's weights are requested at once, at kernel start.
//
// Per 32 in-features of a stage (4 qweight rows), lane (g = lane / 4,
// c = lane % 4) reads the 16 bytes of row c that hold features 4g .. 4g + 3
// of the strip.  Each code becomes the fp16 value 1024 + code (one LOP3 per
// two codes); subtracting 1024 + zero and multiplying by the scale (one half2
// operation each, one rounding) gives exactly the fp16 weight that
// gptq_dequant writes.  The weights of features (4g, 4g + 1) and of
// (4g + 2, 4g + 3) are the A fragments (rows g, g + 8) of two m16n8k16 MMA
// chains (fp16 in, fp32 accumulate), against activations staged once per CTA
// as ready-made B fragments (tokens are the MMA's N dimension, padded to 8).
// The order of in-features inside the 32 is free, so the staged activations
// follow the order the unpacked registers imply.
//
// A strip whose stages are split between warps is finished through shared
// memory in warp order, i.e. in K order: results are deterministic.
#include <cuda_fp16.h>

#include <atomic>
#include <climits>
#include <cstdint>

#include "internal.h"
#include "ptx.cuh"

namespace gwb {
namespace {

constexpr int kGW = 8;                               // warps per CTA
constexpr int kGThreads = kGW * 32;
constexpr int kStripN = 32;                          // output features per strip
constexpr int kStageK = 256;                         // in-features per stage
constexpr int kCodesB = kStripN * 4 * (kStageK / 8); // 4096 bytes of codes per stage
constexpr int kScaleBoxB = 8 * kStripN * 2;          // up to 8 groups x 32 fp16 scales
constexpr int kZeroBoxB = 8 * 16;                    // up to 8 groups x 4 zero words
constexpr int kMaxDynSmem = 232448;
constexpr int kNumSMs = 148;
constexpr int kMaxSlots = 8;

struct GArgs {
  const uint16_t *x;        // fp16 [M, K]
  const uint32_t *qw;       // [K/8, N]
  const uint16_t *scales;   // fp16 [G, N]
  const uint32_t *qzeros;   // [G, N/8]
  const int32_t *g_idx;     // [K] (act order) or null
  uint16_t *y;              // fp16 [M, N]
  int M, N, K, G;
  int gs_log2, zadd;
  int nks;                  // stages per strip (K / 256)
  int ns_per, ns_rem;       // strips per CTA: ns_per, one more for the first ns_rem CTAs
  int D;                    // ring slots per warp
};

__device__ __forceinline__ void mma_f16_16816(float *d, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                              uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// s * ((1024 + q) - (1024 + z)) for two fp16 lanes at once (exact subtraction,
// one rounding in the product).
__device__ __forceinline__ uint32_t dq2(uint32_t q2, uint32_t z2, uint32_t s2) {
  __half2 q = *reinterpret_cast<__half2 *>(&q2);
  const __half2 z = *reinterpret_cast<const __half2 *>(&z2), s = *reinterpret_cast<const __half2 *>(&s2);
  q = __hmul2(__hsub2(q, z), s);
  return *reinterpret_cast<uint32_t *>(&q);
}

template <int MP, bool GIDX>
__global__ void __launch_bounds__(kGThreads, 1) k_gemv_gptq_pipe(const GArgs a) {
  constexpr int SLOT = GIDX ? kCodesB : kCodesB + kScaleBoxB + kZeroBoxB;
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ int rec[kGW][2];   // strip of each warp's partial slot (first, last segment), or -1

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, c = lane & 3;
  const int D = a.D, nks = a.nks, N = a.N;
  unsigned char *ring = smem + (size_t)warp * D * SLOT;
  uint2 *XB = reinterpret_cast<uint2 *>(smem + (size_t)kGW * D * SLOT);   // [K/32][2][4][MP]
  float *PART = reinterpret_cast<float *>(XB + (size_t)(a.K / 32) * 8 * MP);   // [kGW][2][32][MP]
  uint64_t *full = reinterpret_cast<uint64_t *>(PART + kGW * 2 * 32 * MP) + warp * D;

  // this CTA's strips [sb, se) and this warp's stages [u0, u1) of their list
  const int bx = blockIdx.x;
  const int sb = bx * a.ns_per + (bx < a.ns_rem ? bx : a.ns_rem);
  const int se = sb + a.ns_per + (bx < a.ns_rem ? 1 : 0);
  const int tot = (se - sb) * nks;
  const int u0 = (int)((int64_t)warp * tot / kGW), u1 = (int)((int64_t)(warp + 1) * tot / kGW);
  const int nst = u1 - u0;

  if (lane < D) mbar_init(&full[lane], 1);
  if (lane < 2) rec[warp][lane] = -1;
  fence_mbar_init();
  __syncwarp();

  // stage i of this warp into ring slot `slot` (the whole warp takes part)
  auto issue = [&](int i, int slot) {
    const int su = u0 + i;
    const int sq = su / nks;
    const int strip = sb + sq, ks = su - sq * nks;
    const int n0 = strip * kStripN;
    unsigned char *dst = ring + slot * SLOT;
    uint64_t *bar = &full[slot];
    const int gps = kStageK >> a.gs_log2;             // groups per stage (gs <= 256)
    if (lane == 0) mbar_arrive_expect_tx(bar, kCodesB + (GIDX ? 0 : gps * (kStripN * 2 + 16)));
    __syncwarp();
    bulk_load(dst + lane * 128, a.qw + (size_t)(ks * (kStageK / 8) + lane) * N + n0, 128, bar);
    if constexpr (!GIDX) {
      const int g0 = (ks * kStageK) >> a.gs_log2;
      if (lane < gps)
        bulk_load(dst + kCodesB + lane * (kStripN * 2), a.scales + (size_t)(g0 + lane) * N + n0, kStripN * 2, bar);
      else if (lane >= 16 && lane < 16 + gps)
        bulk_load(dst + kCodesB + kScaleBoxB + (lane - 16) * 16, a.qzeros + (size_t)(g0 + lane - 16) * (N / 8) + n0 / 8,
                  16, bar);
    }
  };

  const int pre = nst < D ? nst : D;
  for (int i = 0; i < pre; i++) issue(i, i);
  int issued = pre;

  // activations as B fragments: XB[u][j][c][t] = pairs (x[k + 2j], x[k + 2j + 4]) and
  // (x[k + 2j + 1], x[k + 2j + 5]) with k = 32u + 8c, matching the unpacked registers
  {
    const int total = (a.K / 32) * 8 * MP;
    for (int e = threadIdx.x; e < total; e += kGThreads) {
      const int t = e % MP, cc = (e / MP) & 3, j = (e / (4 * MP)) & 1, u = e / (8 * MP);
      uint32_t b0 = 0u, b1 = 0u;
      if (t < a.M) {
        const uint16_t *xr = a.x + (size_t)t * a.K + u * 32 + cc * 8 + 2 * j;
        b0 = (uint32_t)__ldg(xr) | ((uint32_t)__ldg(xr + 4) << 16);
        b1 = (uint32_t)__ldg(xr + 1) | ((uint32_t)__ldg(xr + 5) << 16);
      }
      XB[e] = make_uint2(b0, b1);
    }
  }
  __syncthreads();

  float acc[8];   // features 4g, 4g+1 (tokens 2c, 2c+1 each), then 4g+2, 4g+3
  int cur = -1, seg_first = 0, seg_last = 0;
  bool first_seg = true;
  // writes the open segment: whole strips straight to y, a partial strip to
  // this warp's first or last partial slot
  auto flush = [&]() {
    const int n0 = cur * kStripN;
    if (seg_first == 0 && seg_last == nks - 1) {
#pragma unroll
      for (int jn = 0; jn < 4; jn++)
#pragma unroll
        for (int h = 0; h < 2; h++) {
          const int t = 2 * c + h;
          if (t < a.M) a.y[(size_t)t * N + n0 + 4 * g + jn] = __half_as_ushort(__float2half_rn(acc[2 * jn + h]));
        }
    } else {
      const int sl = first_seg ? 0 : 1;
      float *P = PART + (warp * 2 + sl) * 32 * MP;
#pragma unroll
      for (int jn = 0; jn < 4; jn++)
#pragma unroll
        for (int h = 0; h < 2; h++) {
          const int t = 2 * c + h;
          if (t < MP) P[(4 * g + jn) * MP + t] = acc[2 * jn + h];
        }
      if (lane == 0) rec[warp][sl] = cur;
    }
    first_seg = false;
  };

  const bool hasB = g < MP;
  int i = 0;
  bool ok = true;
  for (; i < nst; i++) {
    const int slot = i % D;
    if (!mbar_wait(&full[slot], (uint32_t)((i / D) & 1))) {
      ok = false;
      break;
    }
    const int su = u0 + i;
    const int sq = su / nks;
    const int strip = sb + sq, ks = su - sq * nks;
    if (strip != cur) {
      if (cur >= 0) flush();
#pragma unroll
      for (int q = 0; q < 8; q++) acc[q] = 0.0f;
      cur = strip;
      seg_first = ks;
    }
    seg_last = ks;
    const unsigned char *S = ring + slot * SLOT;
    const uint2 *xb = XB + (size_t)ks * 8 * 8 * MP + c * MP + (hasB ? g : 0);
#pragma unroll
    for (int u = 0; u < 8; u++) {
      const uint4 wv = *reinterpret_cast<const uint4 *>(S + (4 * u + c) * 128 + 16 * g);
      const uint32_t w4[4] = {wv.x, wv.y, wv.z, wv.w};
      uint32_t A[4][4];   // [feature 4g + jn][register i: codes (i, i + 4)]
      if constexpr (!GIDX) {
        const int gl = (32 * u) >> a.gs_log2;       // the stage-local group of these 32 in-features
        const uint2 s4 = *reinterpret_cast<const uint2 *>(S + kCodesB + gl * (kStripN * 2) + 8 * g);
        const uint32_t zw = *reinterpret_cast<const uint32_t *>(S + kCodesB + kScaleBoxB + gl * 16 + 4 * (g >> 1));
        const uint32_t sv[4] = {s4.x & 0xffffu, s4.x >> 16, s4.y & 0xffffu, s4.y >> 16};
#pragma unroll
        for (int jn = 0; jn < 4; jn++) {
          const uint32_t z = 0x6400u | (((zw >> ((g & 1) * 16 + 4 * jn)) & 0xFu) + (uint32_t)a.zadd);
          const uint32_t z2 = z | (z << 16), s2 = sv[jn] | (sv[jn] << 16);
#pragma unroll
          for (int r = 0; r < 4; r++) A[jn][r] = dq2(((w4[jn] >> (4 * r)) & 0x000F000Fu) | 0x64006400u, z2, s2);
        }
      } else {
        // every in-feature has its own group: the lane's eight in-features k0 .. k0 + 7
        const int k0 = ks * kStageK + 32 * u + 8 * c;
        const int4 ga = __ldg(reinterpret_cast<const int4 *>(a.g_idx + k0));
        const int4 gb = __ldg(reinterpret_cast<const int4 *>(a.g_idx + k0 + 4));
        const int gv[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
        const int ncol = cur * kStripN + 4 * g;
        uint32_t sv[8][2], zv[8];
#pragma unroll
        for (int p = 0; p < 8; p++) {
          const unsigned gq = (unsigned)gv[p] < (unsigned)a.G ? (unsigned)gv[p] : 0u;
          const uint2 s = __ldg(reinterpret_cast<const uint2 *>(a.scales + (size_t)gq * N + ncol));
          sv[p][0] = s.x;
          sv[p][1] = s.y;
          zv[p] = __ldg(a.qzeros + (size_t)gq * (N / 8) + ncol / 8) >> ((g & 1) * 16);
        }
#pragma unroll
        for (int jn = 0; jn < 4; jn++)
#pragma unroll
          for (int r = 0; r < 4; r++) {
            // codes r (low half) and r + 4 (high half) of feature 4g + jn
            const uint32_t slo = (sv[r][jn >> 1] >> ((jn & 1) * 16)) & 0xffffu;
            const uint32_t shi = (sv[r + 4][jn >> 1] >> ((jn & 1) * 16)) & 0xffffu;
            const uint32_t zlo = 0x6400u | (((zv[r] >> (4 * jn)) & 0xFu) + (uint32_t)a.zadd);
            const uint32_t zhi = 0x6400u | (((zv[r + 4] >> (4 * jn)) & 0xFu) + (uint32_t)a.zadd);
            A[jn][r] = dq2(((w4[jn] >> (4 * r)) & 0x000F000Fu) | 0x64006400u, zlo | (zhi << 16), slo | (shi << 16));
          }
      }
#pragma unroll
      for (int j = 0; j < 2; j++) {
        uint2 b = make_uint2(0u, 0u);
        if (hasB) b = xb[(u * 2 + j) * 4 * MP];
        mma_f16_16816(acc, A[0][2 * j], A[1][2 * j], A[0][2 * j + 1], A[1][2 * j + 1], b.x, b.y);
        mma_f16_16816(acc + 4, A[2][2 * j], A[3][2 * j], A[2][2 * j + 1], A[3][2 * j + 1], b.x, b.y);
      }
    }
    __syncwarp();   // every lane has read the slot
    if (issued < nst) {
      issue(issued, slot);
      issued++;
    }
  }
  if (ok) {
    if (cur >= 0) flush();
  } else {
    // a wait gave up (the error flag is set): let the copies still in flight land
    for (int j = i; j < issued; j++) mbar_wait(&full[j % D], (uint32_t)((j / D) & 1));
  }
  __syncthreads();

  // strips split between warps: their partials, summed in warp order
  const int entries = (se - sb) * 32 * MP;
  for (int e = threadIdx.x; e < entries; e += kGThreads) {
    const int t = e % MP, rl = (e / MP) % 32, strip = sb + e / (32 * MP);
    if (t >= a.M) continue;
    float s = 0.0f;
    bool any = false;
    for (int w = 0; w < kGW; w++)
#pragma unroll
      for (int sl = 0; sl < 2; sl++)
        if (rec[w][sl] == strip) {
          s += PART[((w * 2 + sl) * 32 + rl) * MP + t];
          any = true;
        }
    if (any) a.y[(size_t)t * N + strip * kStripN + rl] = __half_as_ushort(__float2half_rn(s));
  }
}

int pad_tokens(int M) { return M <= 1 ? 1 : (M <= 2 ? 2 : (M <= 4 ? 4 : 8)); }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

template <int MP, bool GIDX>
gwb_status run_gptq_pipe(const GArgs &a0, int strips, cudaStream_t st) {
  constexpr int SLOT = GIDX ? kCodesB : kCodesB + kScaleBoxB + kZeroBoxB;
  GArgs a = a0;
  const int grid = strips < kNumSMs ? strips : kNumSMs;
  a.ns_per = strips / grid;
  a.ns_rem = strips % grid;
  const size_t xb = (size_t)a.K * 2 * MP, part = (size_t)kGW * 2 * 32 * MP * 4;
  const int64_t max_stages = ((int64_t)(a.ns_per + (a.ns_rem ? 1 : 0)) * a.nks + kGW - 1) / kGW;
  const int64_t room = (int64_t)kMaxDynSmem - 1024 - (int64_t)xb - (int64_t)part;
  int64_t D = room / (kGW * (SLOT + 8));
  if (D > max_stages) D = max_stages;
  if (D > kMaxSlots) D = kMaxSlots;
  if (D < 2 && !(D == 1 && max_stages == 1)) return GWB_ERR_UNSUPPORTED;
  a.D = (int)D;
  const size_t smem = (size_t)kGW * D * SLOT + xb + part + (size_t)kGW * D * 8;
  auto kern = k_gemv_gptq_pipe<MP, GIDX>;
  // the shared-memory allowance is per device: raised once on each to what any
  // plan may take (the block's static shared memory stays within the other 1 KB)
  static std::atomic<uint64_t> allowed{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(GWB_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  const uint64_t bit = 1ull << (dev & 63);
  if (!(allowed.load() & bit)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynSmem - 1024);
    if (e != cudaSuccess) return fail(GWB_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    allowed.fetch_or(bit);
  }
  kern<<<grid, kGThreads, smem, st>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return fail(GWB_ERR_CUDA, "GPTQ GEMV launch: %s", cudaGetErrorString(e));
  return GWB_OK;
}

}  // namespace

gwb_status launch_gemv_gptq_pipe(const uint16_t *x, int M, const int32_t *qweight, const uint16_t *scales,
                                 const int32_t *qzeros, const int32_t *g_idx, int64_t K, int64_t N, int gs,
                                 uint16_t *y, cudaStream_t st, int zadd) {
  // the layout this kernel covers; anything else takes the register-fed GEMV
  if (N % kStripN != 0 || K % kStageK != 0 || (gs != 32 && gs != 64 && gs != 128)) return GWB_ERR_UNSUPPORTED;
  if (!aligned16(qweight) || !aligned16(scales) || !aligned16(qzeros)) return GWB_ERR_UNSUPPORTED;
  if (M < 1 || M > 8 || N > INT_MAX || K > INT_MAX) return GWB_ERR_UNSUPPORTED;
  GArgs a{};
  a.x = x;
  a.qw = reinterpret_cast<const uint32_t *>(qweight);
  a.scales = scales;
  a.qzeros = reinterpret_cast<const uint32_t *>(qzeros);
  a.g_idx = g_idx;
  a.y = y;
  a.M = M;
  a.N = (int)N;
  a.K = (int)K;
  a.G = (int)(K / gs);
  a.gs_log2 = gs == 32 ? 5 : (gs == 64 ? 6 : 7);
  a.zadd = zadd;
  a.nks = (int)(K / kStageK);
  const int strips = (int)(N / kStripN);
  const int MP = pad_tokens(M);
#define GWB_GP(P)                                                     \
  if (MP == P) return g_idx ? run_gptq_pipe<P, true>(a, strips, st) : run_gptq_pipe<P, false>(a, strips, st);
  GWB_GP(1) GWB_GP(2) GWB_GP(4) GWB_GP(8)
#undef GWB_GP
  return GWB_ERR_UNSUPPORTED;
}

}  // namespace gwb
