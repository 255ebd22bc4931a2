// GEMV / skinny regime (M <= 8 tokens) of the fused dequant + matmul, for the
// MLX affine layout and the GPTQ layout.
//
// Design (memory-bound: every packed weight byte is read from HBM once):
//   * A warp owns 16 output features (rows n) and walks K one quantization
//     group at a time.  Lane (g = lane/4, c = lane%4) loads, for rows g and
//     g+8, the c-th quarter of the group's packed words with one vector load,
//     so the four lanes of a quad cover exactly one group.
//   * The codes are unpacked in registers straight into fp16 pairs holding
//     1024 + code (OR-ing the code into the mantissa of 1024.0 is exact), and
//     those registers are used, unchanged, as the A fragments of
//     mma.sync.m16n8k16 (fp16 x fp16 -> fp32).  The tensor core thus does the
//     multiply-adds; the ALU only masks bits.
//   * The K order inside a group is free (a dot product does not depend on
//     it), so the activations are staged once per CTA in shared memory in
//     exactly the order the unpacked registers imply, as ready-made B
//     fragments (tokens are the MMA's N dimension, padded to 8).
//   * Per group, the MMA yields P = sum_k (1024 + q_k) x_k per (row, token);
//     with X = sum_k x_k (also staged once per CTA) the group contributes
//     s * P + (b - 1024 s) * X = sum_k (q_k s + b) x_k, accumulated in fp32.
//   * Activations are converted to fp16 after an exact power-of-two rescale
//     per token (max |x| -> [2^13, 2^14)), so any bf16 range fits fp16; the
//     scale is undone on the fp32 result.
//   * Split-K: the warps of a CTA split the CTA's K range and reduce through
//     shared memory; when the CTA count would otherwise not fill the GPU, a
//     thread-block cluster of up to 8 CTAs splits K further and CTA rank 0
//     reduces the partials through distributed shared memory.  The reduction
//     order is fixed, so results are deterministic.
// GPTQ (qweight packed along K with N contiguous) uses the same machinery; its
// weights are dequantized to fp16 in registers (s * (q - zero), one rounding,
// equal to what gptq_dequant writes) because a permuted g_idx gives every
// in-feature its own group.
#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "internal.h"

namespace cg = cooperative_groups;

namespace gwb {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

__device__ __forceinline__ float bf16_val(uint16_t h) { return __uint_as_float(static_cast<uint32_t>(h) << 16); }

__device__ __forceinline__ void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Unpacks one packed word into RPW fp16 pairs (1024 + code_lo, 1024 + code_hi).
// Pair i holds the codes at in-word positions i (low half) and i + RPW (high half).
template <int BITS>
__device__ __forceinline__ void unpack_word(uint32_t w, uint32_t *r) {
  if constexpr (BITS == 4) {
#pragma unroll
    for (int i = 0; i < 4; i++) r[i] = ((w >> (4 * i)) & 0x000F000Fu) | 0x64006400u;
  } else if constexpr (BITS == 8) {
    r[0] = __byte_perm(w, 0x64646464u, 0x4240);
    r[1] = __byte_perm(w, 0x64646464u, 0x4341);
  } else {
#pragma unroll
    for (int i = 0; i < 8; i++) r[i] = ((w >> (2 * i)) & 0x00030003u) | 0x64006400u;
  }
}

template <int N>
__device__ __forceinline__ void load_words(const uint32_t *p, uint32_t *w) {
  if constexpr (N == 1) {
    w[0] = __ldg(p);
  } else if constexpr (N == 2) {
    const uint2 t = __ldg(reinterpret_cast<const uint2 *>(p));
    w[0] = t.x; w[1] = t.y;
  } else {
#pragma unroll
    for (int i = 0; i < N / 4; i++) {
      const uint4 t = __ldg(reinterpret_cast<const uint4 *>(p) + i);
      w[4 * i] = t.x; w[4 * i + 1] = t.y; w[4 * i + 2] = t.z; w[4 * i + 3] = t.w;
    }
  }
}

// Position, inside a "unit" of K (one quantization group for the affine
// layout, 32 in-features for GPTQ), of the element carried by half `h` of
// unpacked register `rho` of quad lane `c`.  W = words per lane, CPW = codes
// per word, RPW = registers per word.
template <int W, int CPW, int RPW>
__device__ __forceinline__ int unit_pos(int rho, int c, int h) {
  const int v = rho / RPW, i = rho % RPW;
  return (c * W + v) * CPW + i + h * RPW;
}

// Stages the B fragments for the CTA's K range: XB[u][j][c][t] = {b0, b1} of
// MMA j of unit u for quad lane c and token t (t < MP), each a pair of fp16
// x values at the positions unit_pos() gives.  Tokens >= M are zero.
template <int UNIT, int NMMA, int W, int CPW, int RPW, int MP, bool BF16_IN>
__device__ void stage_b_fragments(const uint16_t *__restrict__ x, int M, int K, int k0, int KR, const float *scale,
                                  uint2 *XB) {
  const int units = KR / UNIT;
  const int total = units * NMMA * 4 * MP;
  for (int e = threadIdx.x; e < total; e += blockDim.x) {
    const int t = e % MP, c = (e / MP) % 4, j = (e / (4 * MP)) % NMMA, u = e / (4 * MP * NMMA);
    uint32_t out[2] = {0u, 0u};
    if (t < M) {
      const uint16_t *xr = x + (int64_t)t * K + k0 + u * UNIT;
#pragma unroll
      for (int r = 0; r < 2; r++) {
        const int rho = 2 * j + r;
        const int plo = unit_pos<W, CPW, RPW>(rho, c, 0), phi = unit_pos<W, CPW, RPW>(rho, c, 1);
        uint16_t lo, hi;
        if constexpr (BF16_IN) {
          lo = __half_as_ushort(__float2half_rn(bf16_val(xr[plo]) * scale[t]));
          hi = __half_as_ushort(__float2half_rn(bf16_val(xr[phi]) * scale[t]));
        } else {
          lo = xr[plo];
          hi = xr[phi];
        }
        out[r] = (uint32_t)lo | ((uint32_t)hi << 16);
      }
    }
    XB[e] = make_uint2(out[0], out[1]);
  }
}

// Per-token exact power-of-two rescale for bf16 activations: max|x| over the
// CTA's K range is mapped into [2^13, 2^14).  Writes scale[t] = 2^e and
// inv[t] = 2^-e for t < 8 (1 for absent tokens).
__device__ void token_scales(const uint16_t *__restrict__ x, int M, int K, int k0, int KR, float *red, float *scale,
                             float *inv) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int t = 0; t < M; t++) {
    float a = 0.0f;
    for (int k = threadIdx.x; k < KR; k += blockDim.x) a = fmaxf(a, fabsf(bf16_val(x[(int64_t)t * K + k0 + k])));
    for (int off = 16; off; off >>= 1) a = fmaxf(a, __shfl_xor_sync(kFull, a, off));
    if (lane == 0) red[warp * 8 + t] = a;
  }
  __syncthreads();
  if (threadIdx.x < 8) {
    const int t = threadIdx.x;
    float a = 0.0f;
    if (t < M)
      for (int w = 0; w < kWarps; w++) a = fmaxf(a, red[w * 8 + t]);
    int e = 0;
    if (a > 0.0f) {
      int ex;
      frexpf(a, &ex);  // a = f * 2^ex, f in [0.5, 1)
      e = 14 - ex;
      e = e > 120 ? 120 : (e < -120 ? -120 : e);
    }
    scale[t] = ldexpf(1.0f, e);
    inv[t] = ldexpf(1.0f, -e);
  }
  __syncthreads();
}

// Sums the fp16-rounded, rescaled activations of every group: XS[u][t] (t < 8).
template <int UNIT>
__device__ void stage_group_sums(const uint16_t *__restrict__ x, int M, int K, int k0, int KR, const float *scale,
                                 float *XS) {
  const int units = KR / UNIT;
  for (int e = threadIdx.x; e < units * 8; e += blockDim.x) {
    const int t = e % 8, u = e / 8;
    float s = 0.0f;
    if (t < M) {
      const uint16_t *xr = x + (int64_t)t * K + k0 + u * UNIT;
      for (int i = 0; i < UNIT; i++) s += __half2float(__float2half_rn(bf16_val(xr[i]) * scale[t]));
    }
    XS[e] = s;
  }
}

// Reduces the per-warp accumulators (rows g, g+8 x tokens 2c, 2c+1) over the
// warps sharing a row subtile, then over the CTAs of the cluster (fixed order),
// and writes y.  OUT_BF16 selects bf16 (else fp16) output.
template <int MP, bool OUT_BF16>
__device__ void reduce_and_store(const float (&acc)[4], int RS, float *RED, float *PART, const float *inv, int row0,
                                 int N, int M, uint16_t *__restrict__ y) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, c = lane & 3;
  float *mine = RED + warp * 128;  // [16 rows][8 tokens]
  mine[g * 8 + 2 * c] = acc[0];
  mine[g * 8 + 2 * c + 1] = acc[1];
  mine[(g + 8) * 8 + 2 * c] = acc[2];
  mine[(g + 8) * 8 + 2 * c + 1] = acc[3];
  __syncthreads();
  const int KW = kWarps / RS;
  const int entries = RS * 16 * MP;
  for (int e = threadIdx.x; e < entries; e += blockDim.x) {
    const int t = e % MP, r = (e / MP) % 16, rs = e / (16 * MP);
    float s = 0.0f;
    for (int ks = 0; ks < KW; ks++) s += RED[(ks * RS + rs) * 128 + r * 8 + t];
    PART[e] = s * inv[t];
  }
  const int S = gridDim.y;
  if (S > 1) {
    cg::cluster_group cluster = cg::this_cluster();
    cluster.sync();
    if (cluster.block_rank() == 0) {
      for (int e = threadIdx.x; e < entries; e += blockDim.x) {
        float s = 0.0f;
        for (int q = 0; q < S; q++) s += cluster.map_shared_rank(PART, q)[e];
        PART[e] = s;  // own slot only; peers read theirs before the final sync
      }
    }
    cluster.sync();
    if (cluster.block_rank() != 0) return;
  } else {
    __syncthreads();
  }
  for (int e = threadIdx.x; e < entries; e += blockDim.x) {
    const int t = e % MP, r = (e / MP) % 16, rs = e / (16 * MP);
    const int n = row0 + rs * 16 + r;
    if (t < M && n < N) {
      const float v = PART[e];
      y[(int64_t)t * N + n] = OUT_BF16 ? __bfloat16_as_ushort(__float2bfloat16_rn(v))
                                       : __half_as_ushort(__float2half_rn(v));
    }
  }
}

// ----------------------------------------------------------------------------
// MLX affine GEMV.
template <int BITS, int GS, int MP>
__global__ void __launch_bounds__(kThreads, 2)
    k_gemv_affine(const uint16_t *__restrict__ x, int M, const uint32_t *__restrict__ wq,
                  const uint16_t *__restrict__ scales, const uint16_t *__restrict__ biases, int N, int K,
                  uint16_t *__restrict__ y, int RS, int KR) {
  constexpr int CPW = 32 / BITS;       // codes per word
  constexpr int RPW = CPW / 2;         // fp16 pairs per word
  constexpr int GW = GS / CPW;         // words per group (per row)
  constexpr int W = GW / 4;            // words per lane per group
  constexpr int NMMA = GS / 16;        // MMAs per group
  constexpr int NR = W * RPW;          // registers per row per group (= 2 * NMMA)
  constexpr int U = (8 / W) < 1 ? 1 : ((8 / W) > 4 ? 4 : (8 / W));  // groups per load batch
  static_assert(W >= 1, "group too small for the quad layout");

  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ float red[kWarps * 8], s_scale[8], s_inv[8];
  const int GR = KR / GS;
  uint2 *XB = reinterpret_cast<uint2 *>(smem);
  float *XS = reinterpret_cast<float *>(XB + GR * NMMA * 4 * MP);
  float *RED = XS + GR * 8;
  float *PART = RED + kWarps * 128;

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int k0 = blockIdx.y * KR;
  const int row0 = blockIdx.x * RS * 16;
  const int G = K / GS;
  const int64_t words_per_row = K / CPW;

  token_scales(x, M, K, k0, KR, red, s_scale, s_inv);
  stage_b_fragments<GS, NMMA, W, CPW, RPW, MP, true>(x, M, K, k0, KR, s_scale, XB);
  stage_group_sums<GS>(x, M, K, k0, KR, s_scale, XS);
  __syncthreads();

  const int rs = warp % RS, ks = warp / RS, KW = kWarps / RS;
  const int g8 = lane >> 2, c = lane & 3;
  const int rA = row0 + rs * 16 + g8, rB = rA + 8;
  const bool vA = rA < N, vB = rB < N;
  const int tB = (g8 < MP) ? g8 : 0;  // token index of this lane's B fragment
  const bool hasB = g8 < MP;
  const uint32_t *pA = wq + (int64_t)(vA ? rA : 0) * words_per_row + (k0 / CPW) + c * W;
  const uint32_t *pB = wq + (int64_t)(vB ? rB : 0) * words_per_row + (k0 / CPW) + c * W;
  const int64_t sA0 = (int64_t)(vA ? rA : 0) * G + k0 / GS, sB0 = (int64_t)(vB ? rB : 0) * G + k0 / GS;

  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int gb = ks; gb < GR; gb += KW * U) {
    uint32_t wa[U][W], wb[U][W];
    float sa[U], ba[U], sb[U], bb[U];
#pragma unroll
    for (int u = 0; u < U; u++) {
      const int g = gb + u * KW;
      if (g < GR) {
        if (vA) load_words<W>(pA + g * GW, wa[u]); else for (int i = 0; i < W; i++) wa[u][i] = 0;
        if (vB) load_words<W>(pB + g * GW, wb[u]); else for (int i = 0; i < W; i++) wb[u][i] = 0;
        sa[u] = vA ? bf16_val(__ldg(scales + sA0 + g)) : 0.f;
        ba[u] = vA ? bf16_val(__ldg(biases + sA0 + g)) : 0.f;
        sb[u] = vB ? bf16_val(__ldg(scales + sB0 + g)) : 0.f;
        bb[u] = vB ? bf16_val(__ldg(biases + sB0 + g)) : 0.f;
      }
    }
#pragma unroll
    for (int u = 0; u < U; u++) {
      const int g = gb + u * KW;
      if (g >= GR) break;
      uint32_t ra[NR], rb[NR];
#pragma unroll
      for (int v = 0; v < W; v++) {
        unpack_word<BITS>(wa[u][v], ra + v * RPW);
        unpack_word<BITS>(wb[u][v], rb + v * RPW);
      }
      float p[4] = {0.f, 0.f, 0.f, 0.f};
      const uint2 *xb = XB + ((g * NMMA) * 4 + c) * MP + tB;
#pragma unroll
      for (int j = 0; j < NMMA; j++) {
        uint2 b = make_uint2(0u, 0u);
        if (hasB) b = xb[j * 4 * MP];
        const uint32_t a[4] = {ra[2 * j], rb[2 * j], ra[2 * j + 1], rb[2 * j + 1]};
        mma_f16_16816(p, a, b.x, b.y);
      }
      const float X0 = XS[g * 8 + 2 * c], X1 = XS[g * 8 + 2 * c + 1];
      const float cA = fmaf(-1024.0f, sa[u], ba[u]), cB = fmaf(-1024.0f, sb[u], bb[u]);
      acc[0] = fmaf(sa[u], p[0], fmaf(cA, X0, acc[0]));
      acc[1] = fmaf(sa[u], p[1], fmaf(cA, X1, acc[1]));
      acc[2] = fmaf(sb[u], p[2], fmaf(cB, X0, acc[2]));
      acc[3] = fmaf(sb[u], p[3], fmaf(cB, X1, acc[3]));
    }
  }
  reduce_and_store<MP, true>(acc, RS, RED, PART, s_inv, row0, N, M, y);
}

// ----------------------------------------------------------------------------
// GPTQ GEMV.  A unit is 32 in-features (four k-octets, one per quad lane);
// each lane loads one qweight word per row (rows g and g+8 of the tile) and
// dequantizes its eight codes to fp16 with the group's scale and zero.
template <int MP, bool GIDX>
__global__ void __launch_bounds__(kThreads, 2)
    k_gemv_gptq(const uint16_t *__restrict__ x, int M, const int32_t *__restrict__ qweight,
                const uint16_t *__restrict__ scales, const int32_t *__restrict__ qzeros,
                const int32_t *__restrict__ g_idx, int N, int K, int gs, uint16_t *__restrict__ y, int RS,
                int KR, int zadd) {
  constexpr int UNIT = 32, NMMA = 2, U = 4;
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ float s_inv[8];
  const int units = KR / UNIT;
  uint2 *XB = reinterpret_cast<uint2 *>(smem);
  float *RED = reinterpret_cast<float *>(XB + units * NMMA * 4 * MP);
  float *PART = RED + kWarps * 128;
  int *GT = reinterpret_cast<int *>(PART + RS * 16 * 8);  // [KR] group of each in-feature (GIDX only)

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int k0 = blockIdx.y * KR;
  const int row0 = blockIdx.x * RS * 16;
  if (threadIdx.x < 8) s_inv[threadIdx.x] = 1.0f;
  stage_b_fragments<UNIT, NMMA, 1, 8, 4, MP, false>(x, M, K, k0, KR, nullptr, XB);
  if constexpr (GIDX)
    for (int k = threadIdx.x; k < KR; k += blockDim.x) GT[k] = g_idx[k0 + k];
  __syncthreads();

  const int rs = warp % RS, ks = warp / RS, KW = kWarps / RS;
  const int g8 = lane >> 2, c = lane & 3;
  const int rA = row0 + rs * 16 + g8, rB = rA + 8;
  const bool vA = rA < N, vB = rB < N;
  const int nA = vA ? rA : 0, nB = vB ? rB : 0;
  const int tB = (g8 < MP) ? g8 : 0;
  const bool hasB = g8 < MP;
  const int NZ = N / 8;

  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int ub = ks; ub < units; ub += KW * U) {
    uint32_t wa[U], wb[U];
    // without g_idx the octet's group scale and zero word are loaded with its
    // codes (gs is a multiple of 8: one group per octet), not after them
    [[maybe_unused]] uint16_t sa_[U], sb_[U];
    [[maybe_unused]] uint32_t za_[U], zb_[U];
#pragma unroll
    for (int u = 0; u < U; u++) {
      const int un = ub + u * KW;
      wa[u] = wb[u] = 0u;
      if constexpr (!GIDX) { sa_[u] = sb_[u] = 0; za_[u] = zb_[u] = 0u; }
      if (un < units) {
        const int64_t kq = (k0 + un * UNIT) / 8 + c;
        if (vA) wa[u] = (uint32_t)__ldg(qweight + kq * N + nA);
        if (vB) wb[u] = (uint32_t)__ldg(qweight + kq * N + nB);
        if constexpr (!GIDX) {
          const int64_t gq = (k0 + un * UNIT + c * 8) / gs;
          sa_[u] = __ldg(scales + gq * N + nA);
          sb_[u] = __ldg(scales + gq * N + nB);
          za_[u] = (uint32_t)__ldg(qzeros + gq * NZ + nA / 8);
          zb_[u] = (uint32_t)__ldg(qzeros + gq * NZ + nB / 8);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < U; u++) {
      const int un = ub + u * KW;
      if (un >= units) break;
      const int kbase = un * UNIT + c * 8;  // first in-feature of this lane's octet (CTA-local)
      uint32_t ra[4], rb[4];
      unpack_word<4>(wa[u], ra);
      unpack_word<4>(wb[u], rb);
      if constexpr (!GIDX) {
        const __half sAh = __ushort_as_half(sa_[u]);
        const __half sBh = __ushort_as_half(sb_[u]);
        const uint32_t zwA = za_[u];
        const uint32_t zwB = zb_[u];
        const uint32_t zA = 0x6400u | (((zwA >> ((nA % 8) * 4)) & 0xFu) + (uint32_t)zadd);
        const uint32_t zB = 0x6400u | (((zwB >> ((nB % 8) * 4)) & 0xFu) + (uint32_t)zadd);
        const __half2 zA2 = __halves2half2(__ushort_as_half(zA), __ushort_as_half(zA));
        const __half2 zB2 = __halves2half2(__ushort_as_half(zB), __ushort_as_half(zB));
        const __half2 sA2 = __halves2half2(sAh, sAh), sB2 = __halves2half2(sBh, sBh);
#pragma unroll
        for (int i = 0; i < 4; i++) {
          __half2 qa = *reinterpret_cast<__half2 *>(&ra[i]), qb = *reinterpret_cast<__half2 *>(&rb[i]);
          qa = __hmul2(__hsub2(qa, zA2), sA2);
          qb = __hmul2(__hsub2(qb, zB2), sB2);
          ra[i] = *reinterpret_cast<uint32_t *>(&qa);
          rb[i] = *reinterpret_cast<uint32_t *>(&qb);
        }
      } else {
#pragma unroll
        for (int i = 0; i < 4; i++) {
          const int glo = GT[kbase + i], ghi = GT[kbase + i + 4];
          const uint16_t sAl = __ldg(scales + (int64_t)glo * N + nA), sAh = __ldg(scales + (int64_t)ghi * N + nA);
          const uint16_t sBl = __ldg(scales + (int64_t)glo * N + nB), sBh = __ldg(scales + (int64_t)ghi * N + nB);
          const uint32_t zAl = 0x6400u | ((((uint32_t)__ldg(qzeros + (int64_t)glo * NZ + nA / 8) >> ((nA % 8) * 4)) & 0xFu) + (uint32_t)zadd);
          const uint32_t zAh = 0x6400u | ((((uint32_t)__ldg(qzeros + (int64_t)ghi * NZ + nA / 8) >> ((nA % 8) * 4)) & 0xFu) + (uint32_t)zadd);
          const uint32_t zBl = 0x6400u | ((((uint32_t)__ldg(qzeros + (int64_t)glo * NZ + nB / 8) >> ((nB % 8) * 4)) & 0xFu) + (uint32_t)zadd);
          const uint32_t zBh = 0x6400u | ((((uint32_t)__ldg(qzeros + (int64_t)ghi * NZ + nB / 8) >> ((nB % 8) * 4)) & 0xFu) + (uint32_t)zadd);
          const uint32_t zA2 = zAl | (zAh << 16), zB2 = zBl | (zBh << 16);
          const uint32_t sA2 = (uint32_t)sAl | ((uint32_t)sAh << 16), sB2 = (uint32_t)sBl | ((uint32_t)sBh << 16);
          __half2 qa = *reinterpret_cast<__half2 *>(&ra[i]), qb = *reinterpret_cast<__half2 *>(&rb[i]);
          qa = __hmul2(__hsub2(qa, *reinterpret_cast<const __half2 *>(&zA2)), *reinterpret_cast<const __half2 *>(&sA2));
          qb = __hmul2(__hsub2(qb, *reinterpret_cast<const __half2 *>(&zB2)), *reinterpret_cast<const __half2 *>(&sB2));
          ra[i] = *reinterpret_cast<uint32_t *>(&qa);
          rb[i] = *reinterpret_cast<uint32_t *>(&qb);
        }
      }
      const uint2 *xb = XB + ((un * NMMA) * 4 + c) * MP + tB;
#pragma unroll
      for (int j = 0; j < NMMA; j++) {
        uint2 b = make_uint2(0u, 0u);
        if (hasB) b = xb[j * 4 * MP];
        const uint32_t a[4] = {ra[2 * j], rb[2 * j], ra[2 * j + 1], rb[2 * j + 1]};
        mma_f16_16816(acc, a, b.x, b.y);
      }
    }
  }
  reduce_and_store<MP, false>(acc, RS, RED, PART, s_inv, row0, N, M, y);
}

// ----------------------------------------------------------------------------
// Launch geometry: rows per CTA = 16 * RS (RS in {8,4,2,1}), K per CTA = KR
// (split over S = K / KR CTAs of one cluster, S <= 8).  Shrinks the CTA tile
// until the grid holds about two CTAs per SM, then splits K; KR stays a
// multiple of the unit and keeps the staged activations within `smem_cap`.
struct GemvGeom {
  int RS, S, KR;
  size_t smem;
};

GemvGeom plan(int64_t N, int64_t K, int unit, int MP, size_t per_k_bytes, size_t fixed_bytes) {
  const int sms = 148;
  const int64_t units = K / unit;
  GemvGeom g{8, 1, (int)K, 0};
  auto ctas = [&](int RS, int S) { return ((N + 16 * RS - 1) / (16 * RS)) * S; };
  while (g.RS > 1 && ctas(g.RS, 1) < 2 * sms) g.RS >>= 1;
  const int KW = kWarps / g.RS;
  const size_t smem_cap = 96 * 1024;
  auto fits = [&](int S) { return (units % S == 0) && (size_t)(K / S) * per_k_bytes + fixed_bytes <= smem_cap; };
  auto ok = [&](int S) { return units % S == 0 && units / S >= KW; };
  int S = 1;
  while (!fits(S) && S < 8) S <<= 1;
  while (S < 8 && ctas(g.RS, S) < 2 * sms && ok(S * 2) && fits(S * 2)) S <<= 1;
  g.S = S;
  g.KR = (int)(K / S);
  g.smem = (size_t)g.KR * per_k_bytes + fixed_bytes;
  (void)MP;
  return g;
}

template <typename Kern, typename... Args>
gwb_status launch_cluster(Kern kern, dim3 grid, size_t smem, int S, cudaStream_t st, Args... args) {
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return fail(GWB_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = (unsigned)S;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, args...);
  if (e != cudaSuccess) return fail(GWB_ERR_CUDA, "GEMV launch: %s", cudaGetErrorString(e));
  return GWB_OK;
}

template <int BITS, int GS, int MP>
gwb_status run_affine(const uint16_t *x, int M, const uint32_t *wq, const uint16_t *scales, const uint16_t *biases,
                      int64_t N, int64_t K, uint16_t *y, cudaStream_t st) {
  // per K: B fragments (2*MP bytes) + group sums (32/GS bytes); fixed: reductions
  const size_t per_k = 2 * MP + 32 / GS + 1;
  const size_t fixed = (kWarps * 128 + 8 * 16 * 8) * sizeof(float) + 64;
  GemvGeom g = plan(N, K, GS, MP, per_k, fixed);
  dim3 grid((unsigned)((N + 16 * g.RS - 1) / (16 * g.RS)), (unsigned)g.S);
  return launch_cluster(k_gemv_affine<BITS, GS, MP>, grid, g.smem, g.S, st, x, M, wq, scales, biases, (int)N,
                        (int)K, y, g.RS, g.KR);
}

template <int MP, bool GIDX>
gwb_status run_gptq(const uint16_t *x, int M, const int32_t *qweight, const uint16_t *scales, const int32_t *qzeros,
                    const int32_t *g_idx, int64_t N, int64_t K, int gs, uint16_t *y, cudaStream_t st, int zadd) {
  const size_t per_k = 2 * MP + (GIDX ? 4 : 0);
  const size_t fixed = (kWarps * 128 + 8 * 16 * 8) * sizeof(float) + 64;
  GemvGeom g = plan(N, K, 32, MP, per_k, fixed);
  dim3 grid((unsigned)((N + 16 * g.RS - 1) / (16 * g.RS)), (unsigned)g.S);
  return launch_cluster(k_gemv_gptq<MP, GIDX>, grid, g.smem, g.S, st, x, M, qweight, scales, qzeros, g_idx, (int)N,
                        (int)K, gs, y, g.RS, g.KR, zadd);
}

int pad_tokens(int M) { return M <= 1 ? 1 : (M <= 2 ? 2 : (M <= 4 ? 4 : 8)); }

}  // namespace

bool gemv_affine_supported(int bits, int gs) { return gs * bits / 32 >= 4; }

gwb_status launch_gemv_affine(const uint16_t *x, int M, const uint32_t *wq, const uint16_t *scales,
                              const uint16_t *biases, int64_t N, int64_t K, int bits, int gs, uint16_t *y,
                              cudaStream_t st) {
  const int MP = pad_tokens(M);
#define GWB_GV(B, S, P) \
  if (bits == B && gs == S && MP == P) return run_affine<B, S, P>(x, M, wq, scales, biases, N, K, y, st);
#define GWB_GV_MP(B, S) GWB_GV(B, S, 1) GWB_GV(B, S, 2) GWB_GV(B, S, 4) GWB_GV(B, S, 8)
  GWB_GV_MP(2, 64) GWB_GV_MP(2, 128)
  GWB_GV_MP(4, 32) GWB_GV_MP(4, 64) GWB_GV_MP(4, 128)
  GWB_GV_MP(8, 32) GWB_GV_MP(8, 64) GWB_GV_MP(8, 128)
#undef GWB_GV_MP
#undef GWB_GV
  return fail(GWB_ERR_UNSUPPORTED, "no GEMV kernel for bits=%d group_size=%d", bits, gs);
}

gwb_status launch_gemv_gptq(const uint16_t *x, int M, const int32_t *qweight, const uint16_t *scales,
                            const int32_t *qzeros, const int32_t *g_idx, int64_t K, int64_t N, int gs,
                            uint16_t *y, cudaStream_t st, int zadd) {
  {   // the shared-memory streamed GEMV where the layout allows
    const gwb_status s = launch_gemv_gptq_pipe(x, M, qweight, scales, qzeros, g_idx, K, N, gs, y, st, zadd);
    if (s != GWB_ERR_UNSUPPORTED) return s;
  }
  const int MP = pad_tokens(M);
#define GWB_GG(P)                                                                                   \
  if (MP == P) {                                                                                     \
    if (g_idx) return run_gptq<P, true>(x, M, qweight, scales, qzeros, g_idx, N, K, gs, y, st, zadd); \
    return run_gptq<P, false>(x, M, qweight, scales, qzeros, g_idx, N, K, gs, y, st, zadd);         \
  }
  GWB_GG(1) GWB_GG(2) GWB_GG(4) GWB_GG(8)
#undef GWB_GG
  return fail(GWB_ERR_UNSUPPORTED, "no GPTQ GEMV kernel for M=%d", M);
}

}  // namespace gwb
