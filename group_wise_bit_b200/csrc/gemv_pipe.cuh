#pragma once
// Decode GEMV (M <= 8 tokens) for the MLX affine layout: the main decode
// kernel, and its fused variants.
//
//   y[t, n] = sum_k x[t, k] * (code[n, k] * scale[n, k / gs] + bias[n, k / gs])
//
// (the affine dequantization of the MLX `quantized_matmul` with transposed
// weights, "affine_qmm_t"; codes packed 32 / bits per uint32 word along K,
// lowest bits = lowest column, bf16 scales and biases [N, K / gs]).
//
// Work unit ("stage") = 16 output rows x 256 bytes of packed codes per row
// (2048 / bits values of k), plus the scales and biases of those rows and
// groups.  One CTA of 8 warps per SM (two when every warp gets at least four
// stages), persistent; a warp owns a contiguous range of the CTA's stages and
// streams them through a private ring of D slots:
//   * lane 0 issues, per stage, one TMA load of the packed words as a 3-D box
//     [2 segments][16 rows][128 bytes] (128-byte swizzle) and one of the scales
//     and biases as a 3-D box over both arrays [2][16 rows][8 or 16 groups]
//     (two 2-D loads each where the driver refuses those views), all
//     completing on the slot's mbarrier, and refills a slot as soon as the
//     warp has read it;
//   * per stage the warp fetches the packed words with ldmatrix (lane c of a quad gets word c
//     of each 16-byte chunk of its two rows), turns each code into an fp16
//     value 1024 + code * 2^sigma with one LOP3 (two codes per register), and
//     runs mma.sync m16n8k16 against activations staged once per CTA and
//     divided by the same powers of two.  The accumulator of each group starts
//     at -1024 * sum(x / 2^sigma), which removes the 1024 offsets exactly, so
//     the MMA returns sum(code * x) and the group scale is applied with one FMA
//     per row and token;
//   * the bias term sum_g bias[n, g] * sum_{k in g} x[t, k] is one bf16 MMA
//     (m16n8k8) per 8 groups, on the bias box as it landed in shared memory,
//     against the per-group activation sums split into two bf16 parts.
// Activations are rescaled per token by an exact power of two so that their
// magnitude fits fp16 (undone on output).  A strip whose stages are split
// between two warps is finished through shared memory in warp order.  When the
// strips cannot fill the GPU, a cluster of up to 8 CTAs splits K and CTA rank 0
// adds the partial results through distributed shared memory, in rank order.
// Every reduction has a fixed order, so results are deterministic.
//
// The kernel is launched with programmatic stream serialization: it lets the
// next kernel in the stream launch early, and waits for the previous one
// (griddepcontrol.wait) before it reads any global memory.
//
// Fused decode products (the `OP` template parameter), as the MLX 8-bit
// runtime ships them for an MLP at decode time (metrale_gpu_runtime/mlx_int8.rs,
// gemv_gate_up, MlxInt8Weight::gemv_silu_gate and gemv_silu_gate_resid):
//   * kOpDual: two weights of one shape against the same activations in one
//     grid: the second weight's strips follow the first's, each weight with its
//     own tensor maps and output;
//   * kOpSilu: the activations are silu(gate) * up, formed in fp32 while they
//     are staged (never written to memory), and an optional residual is added
//     to the fp32 result before its single rounding to bf16.
//
// W4A8 with the per-token quantization fused (kOpW4A8; executorch PR #24467,
// mlx::int8_int4_gemm, whose "staged" lowering quantizes the activations inside
// the product kernel): the staging quantizes x to int8 per token (sx = max|x| /
// 127 over all of K, q = rint(x / sx) clipped to +-127, in fp32 as the
// standalone quantizer does), the weights are symmetric int4 codes with one
// scale per row (no groups, no biases).  The fp16 MMAs then compute the exact
// int32 sum: codes and q are exact in fp16, every partial sum is an integer
// below 2^24 for K <= 16384 (the chains run 64 k at a time), and the signed
// codes enter the magic-number unpack as code ^ 8 with the -8 folded into the
// accumulator start.  y = bf16(acc * (sx[t] * sw[n])), bit-identical to the
// two-launch path.  When K is split over a cluster, the CTAs exchange their
// per-token maxima through distributed shared memory before quantizing; the
// partial sums stay exact integers, so their fp32 reduction is exact too.
//
// W8A8 at decode (kOpI8W8; the 8da8w config of executorch PR #17234): int8
// activations (already quantized) and int8 weights with one scale per row.
// The codes enter the 8-bit unpack as code ^ 0x80 = code + 128 (the -128 is
// folded into the accumulator start); each 64-k chain is an exact fp32
// integer, and the chains are summed in int32 (the whole sum may pass 2^24),
// through the partial-strip reduction too.  The int32 sums are exact; K is
// not split.
//
// This header holds the kernel template and its host-side planner; each
// translation unit that includes it instantiates the modes it launches.
#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <functional>
#include <map>
#include <mutex>
#include <type_traits>
#include <unordered_map>

#include "internal.h"
#include "ptx.cuh"

namespace cg = cooperative_groups;

namespace gwb {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kCW = 8;                       // warps per CTA
constexpr int kCWLog = 3;
constexpr int kThreads = kCW * 32;
constexpr int kSmemPerSM = 232448;
constexpr int kSMs = 148;

// What the kernel computes around the quantized product (see the file comment).
constexpr int kOpPlain = 0;   // y = x W^T
constexpr int kOpDual = 1;    // y = x W^T and y2 = x W2^T, one grid over both weights' strips
constexpr int kOpSilu = 2;    // y = (resid +) (silu(x) * x2) W^T, the product formed in the staging
constexpr int kOpW4A8 = 3;    // y = (sum_k q[t,k] c[n,k]) sx[t] sw[n]: x quantized to int8 per token in the staging
constexpr int kOpI8W8 = 4;    // acc = sum_k qx[t,k] wq[n,k] (int8 x int8, exact int32), y = acc sx[t] sw[n]

template <int BITS, int GS>
struct PCfg {
  static constexpr int CPW = 32 / BITS;               // codes per word
  static constexpr int RPW = CPW / 2;                 // fp16 pairs per word
  static constexpr int KST = 2048 / BITS;             // k per stage: 256 bytes of codes per row
  static constexpr int GST = KST / GS;                // groups per stage
  static constexpr int SBG = GST < 8 ? 8 : GST;       // groups per scale / bias box (16-byte rows at least)
  static constexpr int NCH = GS * BITS / 128;         // 16-byte chunks per row per group
  static constexpr int NMMA = GS / 16;                // k16 MMAs per group
  static constexpr int NREG = GS / 8;                 // A registers per row per group (NCH * RPW)
  static constexpr int NBM = SBG / 8;                 // bias MMAs (k8) per stage
  static constexpr int WB = 4096;                     // packed-word bytes per stage
  static constexpr int SBB = 16 * SBG * 2;            // bytes of one scale (or bias) box
  static constexpr int GI = GST < 256 / GS ? GST : 256 / GS;   // groups whose MMA chains interleave
  static_assert(NCH >= 1 && GST >= 2, "layout not covered");
};

__device__ __forceinline__ float bf16_val(uint32_t h) { return __uint_as_float(h << 16); }

__device__ __forceinline__ void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1,
                                              const float4 &c) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%11,%12,%13};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(c.x), "f"(c.y), "f"(c.z), "f"(c.w));
}
__device__ __forceinline__ void mma_f16_16816_acc(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// D += A (16 x 8, bf16) * B (8 x 8, bf16), fp32 accumulate.
__device__ __forceinline__ void mma_bf16_1688(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t b0) {
  asm(
      "mma.sync.aligned.m16n8k8.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5}, {%6}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(b0));
}
// Four 8x8 b16 matrices: lanes 8i..8i+7 give the row addresses of matrix i;
// lane l receives 32 bits of row l / 4 (columns 2 (l % 4), +1) of each matrix.
__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr)
               : "memory");
}

__device__ __forceinline__ void tma_load_2d_l(uint32_t dst, const CUtensorMap *map, int32_t x, int32_t y,
                                              uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void tma_load_3d_l(uint32_t dst, const CUtensorMap *map, int32_t x, int32_t y, int32_t z,
                                              uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" :::); }

// Code positions held by A register i of a word (low / high fp16 half) and the
// power of two (sigma) the codes carry there.
template <int BITS>
__host__ __device__ constexpr int reg_lo(int i) { return i; }
template <int BITS>
__host__ __device__ constexpr int reg_hi(int i) { return i + 16 / BITS; }
template <int BITS>
__host__ __device__ constexpr int reg_sig(int i) { return BITS == 8 ? 0 : BITS * (i % (8 / BITS)); }

// (w & mask) | mag in one LOP3; `mag` lives in a register (see unpack_word).
template <uint32_t MASK>
__device__ __forceinline__ uint32_t and_or(uint32_t w, uint32_t mag) {
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(w), "n"(MASK), "r"(mag));
  return r;
}
__device__ __forceinline__ uint32_t shr8(uint32_t w) {
  uint32_t r;
  asm("shr.b32 %0, %1, 8;" : "=r"(r) : "r"(w));
  return r;
}
// The fp16 exponent bits of 1024.0 in both halves, as an opaque register value:
// written by inline asm so that the compiler keeps one register for it instead
// of rebuilding the constant next to every use (each use is then a single LOP3
// or PRMT with its mask or selector as the immediate operand).
__device__ __forceinline__ uint32_t mag_reg(uint32_t v) {
  uint32_t r;
  asm volatile("mov.b32 %0, %1;" : "=r"(r) : "r"(v));
  return r;
}

// One word -> RPW fp16 pairs (1024 + code * 2^sigma), see reg_lo / reg_hi /
// reg_sig.  mag = 0x64006400 (2-/4-bit) or 0x64646464 (8-bit).
template <int BITS>
__device__ __forceinline__ void unpack_word(uint32_t w, uint32_t *r, uint32_t mag) {
  if constexpr (BITS == 4) {
    const uint32_t t = shr8(w);
    r[0] = and_or<0x000F000Fu>(w, mag);
    r[1] = and_or<0x00F000F0u>(w, mag);
    r[2] = and_or<0x000F000Fu>(t, mag);
    r[3] = and_or<0x00F000F0u>(t, mag);
  } else if constexpr (BITS == 8) {
    asm("prmt.b32 %0, %1, %2, 0x4240;" : "=r"(r[0]) : "r"(w), "r"(mag));
    asm("prmt.b32 %0, %1, %2, 0x4341;" : "=r"(r[1]) : "r"(w), "r"(mag));
  } else {
    const uint32_t t = shr8(w);
    r[0] = and_or<0x00030003u>(w, mag);
    r[1] = and_or<0x000C000Cu>(w, mag);
    r[2] = and_or<0x00300030u>(w, mag);
    r[3] = and_or<0x00C000C0u>(w, mag);
    r[4] = and_or<0x00030003u>(t, mag);
    r[5] = and_or<0x000C000Cu>(t, mag);
    r[6] = and_or<0x00300030u>(t, mag);
    r[7] = and_or<0x00C000C0u>(t, mag);
  }
}

// k offset, within its group, of code position p of word wi (the lane's word
// of chunk wi of the group) held by quad lane c.
template <int BITS>
__host__ __device__ constexpr int k_in_group(int wi, int c, int p) {
  return (wi * 4 + c) * (32 / BITS) + p;
}

struct PipeArgs {
  const uint16_t *x;
  const uint16_t *x2;     // silu: the up vectors [M, K] (x holds the gate vectors)
  const uint16_t *resid;  // silu: optional residual [M, N]
  uint16_t *y;
  uint16_t *y2;           // dual: the second weight's output
  int M, N, K;
  int NS;          // strips of 16 rows (dual: of both weights)
  int NSH;         // dual: strips of one weight (the second weight's strips follow)
  int sb_swap2;    // dual: sb_swap of the second weight
  const float *sw;        // w4a8, i8w8: per-row weight scales [N]
  const float *sx;        // i8w8: per-token activation scales [M]
  int32_t *acc;           // i8w8: optional int32 sums [M, N] (y may then be null)
  int ns_per, ns_rem;   // strips per CTA: ns_per, and one more for the first ns_rem CTAs
  int w3d;         // packed words: one 3-D box per stage (else two 2-D boxes)
  int sb_joint;    // scales and biases: one 3-D box per stage (else one each)
  int sb_swap;     // joint box: biases come first (they sit below the scales in memory)
  int NCS;         // stages per strip in this CTA's K-slice
  int D;           // ring depth per consumer warp
  int out_strips;  // split-K only: strips per CTA that the OUT buffer holds
};

struct PartRec {   // a strip result that one warp holds only part of
  int strip, first;
};

// silu(g) = g * sigmoid(g) with the fast exponential and an IEEE reciprocal
// (relative error far below the fp16 rounding the staged value takes next);
// for g < -88 the exponential overflows to +inf and the reciprocal gives 0.
__device__ __forceinline__ float silu_f(float g) { return g * __frcp_rn(1.0f + __expf(-g)); }

// One staged item of int8 activations: NCH runs of 4 values, one word each.
template <int NCH>
struct XItemI8 {
  uint32_t r[NCH];
  __device__ __forceinline__ float get(int wi, int p) const { return (float)(int8_t)(r[wi] >> (8 * p)); }
  __device__ __forceinline__ float bound(int wi, int p) const { return fabsf(get(wi, p)); }
};
// An upper bound of |silu(g) * u| without the exponential: silu(g) <= g for
// g >= 0, and |silu(g)| < 0.2785 for g < 0 (its minimum, near g = -1.278).
__device__ __forceinline__ float silu_bound(float g, float u) { return fmaxf(g, 0.28f) * fabsf(u); }

// One staged activation item: NCH runs of CPW values as loaded (bf16 pairs);
// for the silu product, the gate and up pairs, combined when a value is read.
template <int NCH, int CPW, bool SILU>
struct XItem {
  uint32_t r[NCH][CPW / 2];
  __device__ __forceinline__ float get(int wi, int p) const {
    return bf16_val((p & 1) ? (r[wi][p >> 1] >> 16) : (r[wi][p >> 1] & 0xffffu));
  }
  __device__ __forceinline__ float bound(int wi, int p) const { return fabsf(get(wi, p)); }
};
template <int NCH, int CPW>
struct XItem<NCH, CPW, true> {
  uint32_t g[NCH][CPW / 2], u[NCH][CPW / 2];
  __device__ __forceinline__ float get(int wi, int p) const {
    const uint32_t gw = g[wi][p >> 1], uw = u[wi][p >> 1];
    return silu_f(bf16_val((p & 1) ? (gw >> 16) : (gw & 0xffffu))) * bf16_val((p & 1) ? (uw >> 16) : (uw & 0xffffu));
  }
  // an upper bound of |get(wi, p)| without the exponential
  __device__ __forceinline__ float bound(int wi, int p) const {
    const uint32_t gw = g[wi][p >> 1], uw = u[wi][p >> 1];
    return silu_bound(bf16_val((p & 1) ? (gw >> 16) : (gw & 0xffffu)), bf16_val((p & 1) ? (uw >> 16) : (uw & 0xffffu)));
  }
};

// The tensor maps of a launch: packed words, scales (or the joint scale and
// bias box), biases; dual: the same three of the second weight follow.  Only
// the maps a mode uses are passed, to keep the parameter block small.
template <int NM>
struct MapSet {
  CUtensorMap m[NM];
};
template <int OP>
using MapsOf = MapSet<OP == kOpDual ? 6 : 3>;

template <int BITS, int GS, int MP, int OP>
__global__ void __launch_bounds__(kThreads, 2)
    k_gemv_pipe(const __grid_constant__ MapsOf<OP> maps, const PipeArgs a) {
  const CUtensorMap &tm_w = maps.m[0], &tm_sb = maps.m[1], &tm_b = maps.m[2];
  const CUtensorMap &tm_w2 = maps.m[OP == kOpDual ? 3 : 0], &tm_sb2 = maps.m[OP == kOpDual ? 4 : 1],
                    &tm_b2 = maps.m[OP == kOpDual ? 5 : 2];
  using C = PCfg<BITS, GS>;
  using Item = std::conditional_t<OP == kOpI8W8, XItemI8<C::NCH>, XItem<C::NCH, C::CPW, OP == kOpSilu>>;
  static_assert(OP != kOpI8W8 || (BITS == 8 && C::CPW == 4), "int8 activations go with 8-bit codes");
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  __shared__ float red[kCW][8];
  __shared__ PartRec rec[kCW][2];
  __shared__ volatile int abort_flag;
  __shared__ float tok_sx[8];   // w4a8: the per-token activation scales
  unsigned char *base = align_smem_1024(smem_raw);

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int D = a.D, NCS = a.NCS, S = gridDim.y;
  const int KR = NCS * C::KST, GR = KR / GS;    // this CTA's K-slice
  const int k0 = blockIdx.y * KR, g0 = k0 / GS;

  unsigned char *ringW = base;                                        // [kCW][D][4096]
  unsigned char *ringSB = ringW + kCW * D * C::WB;                    // [kCW][D][scales box, biases box]
  uint4 *XB = reinterpret_cast<uint4 *>(ringSB + kCW * D * 2 * C::SBB);   // [GR][NMMA/2][4][MP]
  float4 *XNF = reinterpret_cast<float4 *>(XB + GR * (C::NMMA / 2) * 4 * MP);   // [GR][4]
  uint2 *XF = reinterpret_cast<uint2 *>(XNF + GR * 4);                // [NCS][NBM][32]
  float *PART = reinterpret_cast<float *>(XF + NCS * C::NBM * 32);    // [kCW][2][16][MP]
  float *OUT = PART + kCW * 2 * 16 * MP;                              // split-K: [strips][16][MP]
  uint64_t *full = reinterpret_cast<uint64_t *>(OUT + (S > 1 ? a.out_strips * 16 * MP : 0));

  // ---- this CTA's strips [sb, se) (the first ns_rem CTAs take one more), and
  // warp w's stages [ub(w), ub(w + 1)) of them
  const int bx = blockIdx.x;
  const int sb = bx * a.ns_per + (bx < a.ns_rem ? bx : a.ns_rem);
  const int se = sb + a.ns_per + (bx < a.ns_rem ? 1 : 0);
  const int ucta = (se - sb) * NCS;
  auto ub = [&](int w) { return (int)(((int64_t)w * ucta) >> kCWLog); };
  // the output of (virtual) row vrow and token t; dual: rows past NSH * 16 are
  // the second weight's; silu: plus the residual, if any
  auto put_y = [&](int vrow, int t, float v) {
    uint16_t *yp = a.y;
    int row = vrow;
    if constexpr (OP == kOpDual) {
      if (vrow >= a.NSH * 16) {
        yp = a.y2;
        row = vrow - a.NSH * 16;
      }
    }
    if (t < a.M && row < a.N) {
      if constexpr (OP == kOpSilu) {
        if (a.resid) v += bf16_val(a.resid[(int64_t)t * a.N + row]);
      }
      if constexpr (OP == kOpW4A8) v = v * (tok_sx[t] * __ldg(a.sw + row));   // v is the exact int32 sum
      if constexpr (OP == kOpI8W8) {
        // v carries the bits of the int32 sum
        const int vi = __float_as_int(v);
        if (a.acc) a.acc[(int64_t)t * a.N + row] = vi;
        if (yp) yp[(int64_t)t * a.N + row] = __bfloat16_as_ushort(__float2bfloat16_rn((float)vi * (__ldg(a.sx + t) * __ldg(a.sw + row))));
        return;
      }
      yp[(int64_t)t * a.N + row] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
    }
  };

  if (threadIdx.x < kCW * D) mbar_init(&full[threadIdx.x], 1);
  if (threadIdx.x < kCW * 2) rec[threadIdx.x >> 1][threadIdx.x & 1] = PartRec{-1, -1};
  for (int e = threadIdx.x; e < NCS * C::NBM * 32; e += kThreads) XF[e] = make_uint2(0u, 0u);
  if (threadIdx.x == 0) {
    abort_flag = 0;
    tma_prefetch_desc(&tm_w);
    if (OP != kOpW4A8 && OP != kOpI8W8) {
      tma_prefetch_desc(&tm_sb);
      if (!a.sb_joint) tma_prefetch_desc(&tm_b);
    }
    if (OP == kOpDual) {
      tma_prefetch_desc(&tm_w2);
      tma_prefetch_desc(&tm_sb2);
      if (!a.sb_joint) tma_prefetch_desc(&tm_b2);
    }
  }
  fence_mbar_init();
  __syncthreads();
  pdl_launch_dependents();
  pdl_wait();   // the previous kernel's writes (x, and possibly the weights) are visible from here on

  // loads the stage (strip, st) of this warp into its ring slot: packed words
  // as one 3-D box ([2 segments][16 rows][128 bytes], or two 2-D boxes) and the
  // scale and bias boxes as one 3-D box ([2 arrays][16 rows][SBG], or two)
  const int units = ub(warp + 1) - ub(warp);
  auto issue = [&](int strip, int st, int slot) {
    // dual: the strips past NSH belong to the second weight
    const bool hi = OP == kOpDual && strip >= a.NSH;
    const int r0 = (hi ? strip - a.NSH : strip) * 16;
    const CUtensorMap *mw = hi ? &tm_w2 : &tm_w, *msb = hi ? &tm_sb2 : &tm_sb, *mb = hi ? &tm_b2 : &tm_b;
    const int ks = k0 + st * C::KST;
    const uint32_t bar = smem_u32(&full[slot]);
    const uint32_t dw = smem_u32(ringW + slot * C::WB);
    const uint32_t ds = smem_u32(ringSB + slot * 2 * C::SBB);
    const int gsx = ks / GS;
    const int gbox = C::GST < 8 ? (gsx & ~7) : gsx;
    mbar_arrive_expect_tx(&full[slot], C::WB + (OP == kOpW4A8 || OP == kOpI8W8 ? 0 : 2 * C::SBB));
    if (a.w3d) {
      tma_load_3d_l(dw, mw, 0, r0, ks / (32 * C::CPW), bar);
    } else {
      tma_load_2d_l(dw, mw, ks / C::CPW, r0, bar);
      tma_load_2d_l(dw + 2048, mw, ks / C::CPW + 32, r0, bar);
    }
    if (OP == kOpW4A8 || OP == kOpI8W8) {
      // no scale or bias boxes
    } else if (a.sb_joint) {
      tma_load_3d_l(ds, msb, gbox, r0, 0, bar);
    } else {
      tma_load_2d_l(ds, msb, gbox, r0, bar);
      tma_load_2d_l(ds + C::SBB, mb, gbox, r0, bar);
    }
  };
  // issue-side position (strip, stage) of this warp, advanced without divisions
  int is_strip = sb + ub(warp) / NCS, is_st = ub(warp) % NCS;
  // ---- activations of the K-slice, staged per item = (group, token, quad lane c):
  // the item's NCH runs of CPW values at k = group start + (wi * 4 + c) * CPW.
  // A thread loads its first item into registers before the ring fill below
  // (so the load latency hides behind the TMA issue) and keeps it for pass B.
  const int items = GR * MP * 4;
  // the item's element offset t * K + (group start), or -1 when it holds nothing
  auto item_src = [&](int idx, int &t, int &c, int &g) -> int64_t {
    c = idx & 3;
    t = (idx >> 2) % MP;
    g = (idx >> 2) / MP;
    const int kg = k0 + g * GS;
    return (idx < items && t < a.M && kg < a.K) ? (int64_t)t * a.K + kg : -1;
  };
  // CPW consecutive bf16 values at p, as CPW / 2 packed pairs
  auto load_pairs = [&](const uint16_t *p, uint32_t (&w)[C::CPW / 2]) {
    if constexpr (C::CPW == 4) {
      const uint2 v = __ldg(reinterpret_cast<const uint2 *>(p));
      w[0] = v.x; w[1] = v.y;
    } else {
#pragma unroll
      for (int q = 0; q < C::CPW / 8; q++) {
        const uint4 v = __ldg(reinterpret_cast<const uint4 *>(p) + q);
        w[4 * q] = v.x; w[4 * q + 1] = v.y; w[4 * q + 2] = v.z; w[4 * q + 3] = v.w;
      }
    }
  };
  auto load_item = [&](int64_t off, int c, Item &it) {
#pragma unroll
    for (int wi = 0; wi < C::NCH; wi++) {
      const int64_t o = off + k_in_group<BITS>(wi, c, 0);
      const uint16_t *p = off >= 0 ? a.x + o : nullptr;
      if constexpr (OP == kOpI8W8) {
        // 4 int8 values in one aligned word (K and the run start are multiples of 4)
        it.r[wi] = off >= 0 ? __ldg(reinterpret_cast<const uint32_t *>(reinterpret_cast<const int8_t *>(a.x) + o)) : 0u;
      } else if constexpr (OP == kOpSilu) {
        // the up value sits at the same offset of x2
#pragma unroll
        for (int q = 0; q < C::CPW / 2; q++) it.g[wi][q] = it.u[wi][q] = 0u;
        if (p) {
          load_pairs(p, it.g[wi]);
          load_pairs(a.x2 + (p - a.x), it.u[wi]);
        }
      } else {
#pragma unroll
        for (int q = 0; q < C::CPW / 2; q++) it.r[wi][q] = 0u;
        if (p) load_pairs(p, it.r[wi]);
      }
    }
  };
  Item raw0;
  int t0i, c0i, g0i;
  const int64_t src0 = item_src(threadIdx.x, t0i, c0i, g0i);
  load_item(src0, c0i, raw0);

  for (int i = 0; i < (units < D ? units : D); i++) {
    if (lane == 0) issue(is_strip, is_st, warp * D + i);
    if (++is_st == NCS) { is_st = 0; ++is_strip; }
  }

  // max|x| of token t over this CTA's K-slice (every thread derives it from red[]);
  // w4a8 with K split over a cluster: over the whole row, from every CTA's red[]
  // through distributed shared memory (after the cluster barrier that ends pass A)
  auto token_amax = [&](int t) -> float {
    float m = 0.0f;
    if (OP == kOpW4A8 && S > 1) {
      cg::cluster_group cluster = cg::this_cluster();
      for (int q = 0; q < S; q++) {
        const float *rr = cluster.map_shared_rank(&red[0][0], q);
#pragma unroll
        for (int w = 0; w < kCW; w++) m = fmaxf(m, rr[w * 8 + t]);
      }
      return m;
    }
#pragma unroll
    for (int w = 0; w < kCW; w++) m = fmaxf(m, red[w][t]);
    return m;
  };
  // Per-token power of two e: the largest |x| * 2^e lands in [2^13, 2^14), so
  // the rescaled activations fit fp16 (every thread derives it from red[]).
  auto token_exp = [&](int t) -> int {
    if (OP == kOpW4A8 || OP == kOpI8W8) return 0;   // integer values need no rescale
    float m = 0.0f;
#pragma unroll
    for (int w = 0; w < kCW; w++) m = fmaxf(m, red[w][t]);
    if (!(m > 0.0f)) return 0;
    const int be = (int)((__float_as_uint(m) >> 23) & 0xffu);   // m in [2^(be-127), 2^(be-126))
    const int e = 140 - be;                                       // 14 - (be - 126)
    return e > 120 ? 120 : (e < -120 ? -120 : e);
  };
  // Passes A and B take PB items per round and issue all their loads before
  // using any; the first item of round 0 is the one loaded above.  One item
  // per round when one round covers them all (the loop then carries no dead
  // slots), else PB_MAX.
  auto staging = [&](auto pb_tag) {
    constexpr int PB = decltype(pb_tag)::value;
    // Pass A: |x| max per token (per warp), over every item; silu: a bound of
    // |silu(gate) * up| (no exponential) is enough to place the power of two
    {
      float m[MP];
#pragma unroll
      for (int t = 0; t < MP; t++) m[t] = 0.0f;
      for (int b0 = 0; b0 < items; b0 += PB * kThreads) {
        Item itb[PB];
#pragma unroll
        for (int u = 0; u < PB; u++) {
          int t, c, g;
          const int64_t src = item_src(b0 + u * kThreads + threadIdx.x, t, c, g);
          if (b0 == 0 && u == 0) {
            itb[0] = raw0;
          } else {
            load_item(src, c, itb[u]);
          }
        }
#pragma unroll
        for (int u = 0; u < PB; u++) {
          if (b0 + u * kThreads >= items) break;   // the same for the whole block
          const int t = ((b0 + u * kThreads + (int)threadIdx.x) >> 2) % MP;   // the item's token
          float mx = 0.0f;
#pragma unroll
          for (int wi = 0; wi < C::NCH; wi++)
#pragma unroll
            for (int p = 0; p < C::CPW; p++) mx = fmaxf(mx, itb[u].bound(wi, p));
#pragma unroll
          for (int tt = 0; tt < MP; tt++)
            if (tt == t) m[tt] = fmaxf(m[tt], mx);
        }
      }
#pragma unroll
      for (int t = 0; t < MP; t++) {
        float v = m[t];
        for (int off = 16; off; off >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, off));
        if (lane == 0) red[warp][t] = v;
      }
    }
    __syncthreads();
    // w4a8 with a K split: every CTA's maxima are complete before any CTA reads
    // them (and red[] is not written again; no CTA leaves before the final
    // cluster barrier of the split-K reduction)
    if (OP == kOpW4A8 && S > 1) cg::this_cluster().sync();
    // Pass B: one thread per item: the B fragments of the lane's codes, and
    // (combined over c in order) the group's activation sum X and magic sum XN,
    // written straight into the accumulator start quads (XNF) and the
    // split-bf16 B operand of the bias MMAs (XF).
    {
      if (OP == kOpW4A8 && threadIdx.x < MP) tok_sx[threadIdx.x] = __fdiv_rn(token_amax(threadIdx.x), 127.0f);
      if constexpr (OP == kOpW4A8) __syncthreads();   // every item reads its token's scale
      const int total = items;
      for (int b0 = 0; b0 < total; b0 += PB * kThreads) {
      Item itb[PB];
      int tq[PB], cq[PB], gq[PB];
      int64_t sq[PB];
#pragma unroll
      for (int u = 0; u < PB; u++) {
        sq[u] = item_src(b0 + u * kThreads + threadIdx.x, tq[u], cq[u], gq[u]);
        if (b0 == 0 && u == 0) {
          itb[0] = raw0;
        } else {
          load_item(sq[u], cq[u], itb[u]);
        }
      }
#pragma unroll
      for (int u = 0; u < PB; u++) {
        if (b0 + u * kThreads >= total) break;   // the same for the whole block: the shuffles stay converged
        const int idx = b0 + u * kThreads + threadIdx.x;
        const bool valid = idx < total;
        const int t = tq[u], c = cq[u], g = gq[u];
        const bool live = sq[u] >= 0;
        const float sc = pow2f(live ? token_exp(t) : 0);
        // w4a8: the token's int8 scale, max|x| / 127 over the whole row (over every CTA's
        // K-slice when a cluster splits K)
        [[maybe_unused]] const float sq = OP == kOpW4A8 ? tok_sx[t] : 0.0f;
        const Item &rawb = itb[u];
        float sx = 0.0f, sn = 0.0f;
        uint32_t pr[C::NREG];
#pragma unroll
        for (int wi = 0; wi < C::NCH; wi++) {
          uint16_t h[C::CPW];
#pragma unroll
          for (int p = 0; p < C::CPW; p++) {
            if constexpr (OP == kOpW4A8) {
              // q = clip(round_half_even(x / sx), -127, 127), exactly as the standalone quantizer
              const float q = sq == 0.0f ? 0.0f : fminf(fmaxf(rintf(__fdiv_rn(rawb.get(wi, p), sq)), -127.0f), 127.0f);
              h[p] = __half_as_ushort(__float2half_rn(q));
            } else {
              h[p] = __half_as_ushort(__float2half_rn(rawb.get(wi, p) * sc));
            }
            sx += __half2float(__ushort_as_half(h[p]));
          }
#pragma unroll
          for (int i = 0; i < C::RPW; i++) {
            const float inv = pow2f(-reg_sig<BITS>(i));
            const __half lo = __float2half_rn(__half2float(__ushort_as_half(h[reg_lo<BITS>(i)])) * inv);
            const __half hi = __float2half_rn(__half2float(__ushort_as_half(h[reg_hi<BITS>(i)])) * inv);
            sn += __half2float(lo) + __half2float(hi);
            pr[wi * C::RPW + i] = (uint32_t)__half_as_ushort(lo) | ((uint32_t)__half_as_ushort(hi) << 16);
          }
        }
        if (valid) {
#pragma unroll
          for (int mp = 0; mp < C::NMMA / 2; mp++)
            XB[((g * (C::NMMA / 2) + mp) * 4 + c) * MP + t] =
                make_uint4(pr[4 * mp], pr[4 * mp + 1], pr[4 * mp + 2], pr[4 * mp + 3]);
        }
        sx += __shfl_xor_sync(kFull, sx, 1);
        sn += __shfl_xor_sync(kFull, sn, 1);
        sx += __shfl_xor_sync(kFull, sx, 2);
        sn += __shfl_xor_sync(kFull, sn, 2);
        if (valid && c == 0) {
          // w4a8: the codes enter as (code ^ 8) = code + 8, so the start also takes 8 sum(q) off
          const float xn = live ? (OP == kOpW4A8 ? -1024.0f * sn - 8.0f * sx : OP == kOpI8W8 ? -1024.0f * sn - 128.0f * sx : -1024.0f * sn) : 0.0f;
          const float X = live ? sx : 0.0f;
          // accumulator quad of quad lane t / 2: components t % 2 and t % 2 + 2
          float *q = reinterpret_cast<float *>(XNF + g * 4 + (t >> 1));
          q[t & 1] = xn;
          q[(t & 1) + 2] = xn;
          // bias-MMA B operand: stage st, box column jj = 8 bm + 2 c' + h, lane t * 4 + c'
          const int st = g / C::GST;
          const int gbox = C::GST < 8 ? ((g0 + st * C::GST) & ~7) - g0 : st * C::GST;
          const int jj = g - gbox, bm = jj >> 3, cq = (jj & 7) >> 1, hh = jj & 1;
          const __nv_bfloat16 xh = __float2bfloat16_rn(X);
          const __nv_bfloat16 xl = __float2bfloat16_rn(X - __bfloat162float(xh));
          uint16_t *f = reinterpret_cast<uint16_t *>(XF + (st * C::NBM + bm) * 32 + t * 4 + cq);
          f[hh] = __bfloat16_as_ushort(xh);
          f[2 + hh] = __bfloat16_as_ushort(xl);
        }
      }
      }
    }
    __syncthreads();
  };
  constexpr int PB_MAX = OP == kOpSilu ? 2 : 4;
  if (items > kThreads)
    staging(std::integral_constant<int, PB_MAX>{});
  else
    staging(std::integral_constant<int, 1>{});

  {
    // ------------------------------------------------------------ consumers
    const int g8 = lane >> 2, c = lane & 3;
    const int lx = lane & 7, hh = (lane >> 3) & 1, qq = lane >> 4;
    const uint32_t rowoff = (uint32_t)((lx + 8 * hh) * 128);
    uint32_t swz[4];
#pragma unroll
    for (int p4 = 0; p4 < 4; p4++) swz[p4] = (uint32_t)(((2 * p4 + qq) ^ lx) << 4);
    // Lanes whose token is absent (g8 >= MP) borrow token g8 % MP: that only
    // fills MMA columns >= MP, which are never stored.
    const uint4 *xbl = XB + c * MP + (MP == 1 ? 0 : g8 % MP);
    const uint32_t mag = mag_reg(BITS == 8 ? 0x64646464u : 0x64006400u);
    // undoes the per-token rescale of the lane's two tokens
    const float inv0 = pow2f(2 * c < a.M ? -token_exp(2 * c) : 0);
    const float inv1 = pow2f(2 * c + 1 < a.M ? -token_exp(2 * c + 1) : 0);
    constexpr int xbs = 4 * MP;

    constexpr int SW = C::SBG / 2;          // 32-bit words per scale-box row
    constexpr int NSW = C::GST / 2;         // of which this stage uses NSW

    float acc[4] = {0.f, 0.f, 0.f, 0.f}, accb[4] = {0.f, 0.f, 0.f, 0.f};
    const int u_beg = ub(warp);
    const int first_strip = sb + u_beg / NCS;
    int strip = first_strip, st = u_beg % NCS, first_st = st;

    auto flush = [&](int strip_, int fst, int lst) {
      const bool whole = fst == 0 && lst == NCS - 1;
      float v[4];
#pragma unroll
      for (int i = 0; i < 4; i++) v[i] = OP == kOpI8W8 ? acc[i] : (acc[i] + accb[i]) * ((i & 1) ? inv1 : inv0);
      if (whole && S == 1) {
        const int rA = strip_ * 16 + g8;
#pragma unroll
        for (int i = 0; i < 4; i++) put_y(rA + ((i < 2) ? 0 : 8), 2 * c + (i & 1), v[i]);
      } else {
        float *dst;
        if (whole) {
          dst = OUT + (strip_ - sb) * 16 * MP;
        } else {
          const int z = (strip_ == first_strip) ? 0 : 1;   // only a warp's first and last strip can be partial
          dst = PART + (warp * 2 + z) * 16 * MP;
          if (lane == 0) rec[warp][z] = PartRec{strip_, fst};
        }
#pragma unroll
        for (int i = 0; i < 4; i++) {
          const int t = 2 * c + (i & 1), r = g8 + ((i < 2) ? 0 : 8);
          if (t < MP) dst[r * MP + t] = v[i];
        }
      }
#pragma unroll
      for (int i = 0; i < 4; i++) acc[i] = accb[i] = 0.f;
    };

    int slot = 0, consumed = 0;
    uint32_t phase = 0;
    for (int i = 0; i < units; i++) {
      if (abort_flag) break;
      if (!mbar_wait(&full[warp * D + slot], phase)) { abort_flag = 1; break; }
      const uint32_t sw = smem_u32(ringW + (warp * D + slot) * C::WB) + rowoff;
      const uint32_t *sp = reinterpret_cast<const uint32_t *>(ringSB + (warp * D + slot) * 2 * C::SBB);
      const uint32_t *bp = sp + C::SBB / 4;
      if (OP == kOpDual && strip >= a.NSH ? a.sb_swap2 : a.sb_swap) {
        const uint32_t *tmp = sp;
        sp = bp;
        bp = tmp;
      }
      const int jb = C::GST < 8 ? ((g0 + st * C::GST) & 7) : 0;   // box column of the stage's first group
      // ---- everything this stage needs from shared memory, then release the slot
      uint32_t wd[16][2];
#pragma unroll
      for (int p = 0; p < 8; p++)
        ldmatrix_x4(sw + (p >> 2) * 2048 + swz[p & 3], wd[2 * p][0], wd[2 * p][1], wd[2 * p + 1][0], wd[2 * p + 1][1]);
      uint32_t sA[NSW], sB[NSW];
      if constexpr (OP == kOpW4A8 || OP == kOpI8W8) {
#pragma unroll
        for (int q = 0; q < NSW; q++) sA[q] = sB[q] = 0u;   // no group scales
      } else {
        const uint32_t *ra = sp + g8 * SW + (jb >> 1), *rb = sp + (g8 + 8) * SW + (jb >> 1);
        if constexpr (NSW >= 4) {
#pragma unroll
          for (int q = 0; q < NSW / 4; q++) {
            const uint4 va = reinterpret_cast<const uint4 *>(ra)[q], vb = reinterpret_cast<const uint4 *>(rb)[q];
            sA[4 * q] = va.x; sA[4 * q + 1] = va.y; sA[4 * q + 2] = va.z; sA[4 * q + 3] = va.w;
            sB[4 * q] = vb.x; sB[4 * q + 1] = vb.y; sB[4 * q + 2] = vb.z; sB[4 * q + 3] = vb.w;
          }
        } else if constexpr (NSW == 2) {
          const uint2 va = *reinterpret_cast<const uint2 *>(ra), vb = *reinterpret_cast<const uint2 *>(rb);
          sA[0] = va.x; sA[1] = va.y; sB[0] = vb.x; sB[1] = vb.y;
        } else {
          sA[0] = ra[0]; sB[0] = rb[0];
        }
      }
      uint32_t ba0[C::NBM], ba1[C::NBM];
#pragma unroll
      for (int b = 0; b < C::NBM; b++) {
        ba0[b] = OP == kOpW4A8 || OP == kOpI8W8 ? 0u : bp[g8 * SW + b * 4 + c];
        ba1[b] = OP == kOpW4A8 || OP == kOpI8W8 ? 0u : bp[(g8 + 8) * SW + b * 4 + c];
      }
      __syncwarp();
      if (i + D < units) {   // the slot has been read: refill it D stages ahead
        if (lane == 0) {
          fence_proxy_async_smem();
          issue(is_strip, is_st, warp * D + slot);
        }
        if (++is_st == NCS) { is_st = 0; ++is_strip; }
      }

      const uint4 *xst = xbl + st * (C::GST * (C::NMMA / 2) * xbs);   // this stage's B fragments
      const float4 *xnst = XNF + st * (C::GST * 4) + c;                // and accumulator start values
      // ---- bias term: sum over the box's groups of bias * (x sums of this stage)
      if constexpr (OP != kOpW4A8 && OP != kOpI8W8) {   // (the integer modes have no biases)
#pragma unroll
        for (int b = 0; b < C::NBM; b++) {
          const uint2 xf = XF[(st * C::NBM + b) * 32 + lane];
          mma_bf16_1688(accb, ba0[b], ba1[b], xf.x);
          mma_bf16_1688(accb, ba0[b], ba1[b], xf.y);
        }
      }
      // ---- codes: GI groups at a time, their MMA chains interleaved (independent
      // accumulators), then each group's scale
#pragma unroll
      for (int j0 = 0; j0 < C::GST; j0 += C::GI) {
        uint32_t ra[C::GI][C::NREG], rb[C::GI][C::NREG];
        float p[C::GI][4];
        const uint4 *xg[C::GI];
#pragma unroll
        for (int gi = 0; gi < C::GI; gi++) {
          const int j = j0 + gi;
#pragma unroll
          for (int wi = 0; wi < C::NCH; wi++) {
            // w4a8 / i8w8: two's-complement nibbles / bytes flipped to code + 8 / code + 128
            constexpr uint32_t flip = OP == kOpW4A8 ? 0x88888888u : OP == kOpI8W8 ? 0x80808080u : 0u;
            unpack_word<BITS>(wd[j * C::NCH + wi][0] ^ flip, &ra[gi][wi * C::RPW], mag);
            unpack_word<BITS>(wd[j * C::NCH + wi][1] ^ flip, &rb[gi][wi * C::RPW], mag);
          }
          xg[gi] = xst + j * (C::NMMA / 2) * xbs;
        }
#pragma unroll
        for (int m2 = 0; m2 < C::NMMA / 2; m2++) {
#pragma unroll
          for (int gi = 0; gi < C::GI; gi++) {
            const uint4 bq = xg[gi][m2 * xbs];
            const uint32_t A0[4] = {ra[gi][4 * m2], rb[gi][4 * m2], ra[gi][4 * m2 + 1], rb[gi][4 * m2 + 1]};
            if (m2 == 0) {
              const float4 xn4 = xnst[(j0 + gi) * 4];
              mma_f16_16816(p[gi], A0, bq.x, bq.y, xn4);
            } else {
              mma_f16_16816_acc(p[gi], A0, bq.x, bq.y);
            }
          }
#pragma unroll
          for (int gi = 0; gi < C::GI; gi++) {
            const uint4 bq = xg[gi][m2 * xbs];
            const uint32_t A1[4] = {ra[gi][4 * m2 + 2], rb[gi][4 * m2 + 2], ra[gi][4 * m2 + 3], rb[gi][4 * m2 + 3]};
            mma_f16_16816_acc(p[gi], A1, bq.z, bq.w);
          }
        }
#pragma unroll
        for (int gi = 0; gi < C::GI; gi++) {
          if constexpr (OP == kOpI8W8) {
            // int32 sums (the bit pattern lives in the float registers): each
            // chain is an exact integer, the total may pass 2^24
#pragma unroll
            for (int q = 0; q < 4; q++)
              if (MP > 1 || (q & 1) == 0) acc[q] = __int_as_float(__float_as_int(acc[q]) + __float2int_rn(p[gi][q]));
          } else if constexpr (OP == kOpW4A8) {
            // exact integer sums: one scale per row, applied at the output
            acc[0] += p[gi][0];
            acc[2] += p[gi][2];
            if constexpr (MP > 1) {
              acc[1] += p[gi][1];
              acc[3] += p[gi][3];
            }
          } else {
            const int j = j0 + gi;
            const uint32_t su = sA[j >> 1], sv = sB[j >> 1];
            const float fa = (j & 1) ? __uint_as_float(su & 0xffff0000u) : __uint_as_float(su << 16);
            const float fb = (j & 1) ? __uint_as_float(sv & 0xffff0000u) : __uint_as_float(sv << 16);
            acc[0] = fmaf(fa, p[gi][0], acc[0]);
            acc[2] = fmaf(fb, p[gi][2], acc[2]);
            if constexpr (MP > 1) {
              acc[1] = fmaf(fa, p[gi][1], acc[1]);
              acc[3] = fmaf(fb, p[gi][3], acc[3]);
            }
          }
        }
      }
      if (st == NCS - 1 || i == units - 1) {
        flush(strip, first_st, st);
        first_st = 0;
      }
      if (++st == NCS) { st = 0; ++strip; }
      if (++slot == D) { slot = 0; phase ^= 1; }
      consumed = i + 1;
    }
    if (consumed < units && lane == 0) {
      // stopped early: every issued load lands before the CTA may exit (waits are bounded)
      const int issued = units < consumed + D ? units : consumed + D;
      for (int i = consumed; i < issued; i++) mbar_wait(&full[warp * D + i % D], (i / D) & 1);
    }
    __syncwarp();
  }
  __syncthreads();

  // ---- strips split between warps: the record holding stage 0 adds the others in warp order
  for (int e = warp; e < kCW * 2; e += kCW) {
    const int w = e >> 1, z = e & 1;
    const PartRec r = rec[w][z];
    if (r.strip < 0 || r.first != 0) continue;
    for (int idx = lane; idx < 16 * MP; idx += 32) {
      float s = PART[(w * 2 + z) * 16 * MP + idx];
      for (int w2 = w; w2 < kCW; w2++)
        for (int z2 = 0; z2 < 2; z2++)
          if ((w2 > w || z2 > z) && rec[w2][z2].strip == r.strip) {
            const float pv = PART[(w2 * 2 + z2) * 16 * MP + idx];
            s = OP == kOpI8W8 ? __int_as_float(__float_as_int(s) + __float_as_int(pv)) : s + pv;   // i8w8: int32 bits
          }
      const int row = r.strip * 16 + idx / MP, t = idx % MP;
      if (S == 1) {
        put_y(row, t, s);
      } else {
        OUT[(r.strip - sb) * 16 * MP + idx] = s;
      }
    }
  }

  if (S > 1) {
    cg::cluster_group cluster = cg::this_cluster();
    cluster.sync();
    if (cluster.block_rank() == 0) {
      for (int e = threadIdx.x; e < (se - sb) * 16 * MP; e += kThreads) {
        float s = 0.f;
        for (int q = 0; q < S; q++) s += cluster.map_shared_rank(OUT, q)[e];
        put_y(sb * 16 + e / MP, e % MP, s);
      }
    }
    cluster.sync();
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

// Caches of the dynamic shared-memory attribute and of the number of
// co-resident clusters per (kernel, cluster size, shared memory), so that
// steady-state calls and calls under stream capture make no occupancy queries.
struct ClusterKey {
  const void *fn;
  int S;
  size_t smem;
  bool operator<(const ClusterKey &o) const {
    return fn != o.fn ? fn < o.fn : (S != o.S ? S < o.S : smem < o.smem);
  }
};
std::mutex g_mu;
std::map<ClusterKey, int> g_max_clusters;
std::map<const void *, size_t> g_smem_attr;

bool ensure_smem_attr(const void *fn, size_t smem) {
  std::lock_guard<std::mutex> lk(g_mu);
  size_t &cur = g_smem_attr[fn];
  if (cur >= smem) return true;
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess) return false;
  cur = smem;
  return true;
}

template <typename Kern>
int max_clusters(Kern kern, int S, size_t smem) {
  {
    std::lock_guard<std::mutex> lk(g_mu);
    auto it = g_max_clusters.find(ClusterKey{reinterpret_cast<const void *>(kern), S, smem});
    if (it != g_max_clusters.end()) return it->second;
  }
  cudaLaunchConfig_t q = {};
  q.gridDim = dim3(1u, (unsigned)S);
  q.blockDim = dim3(kThreads);
  q.dynamicSmemBytes = smem;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 1;
  at[0].val.clusterDim.y = (unsigned)S;
  at[0].val.clusterDim.z = 1;
  q.attrs = at;
  q.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &q) != cudaSuccess || n < 1) {
    (void)cudaGetLastError();
    return 0;
  }
  std::lock_guard<std::mutex> lk(g_mu);
  g_max_clusters[ClusterKey{reinterpret_cast<const void *>(kern), S, smem}] = n;
  return n;
}

CUresult encode_2d(CUtensorMap *m, CUtensorMapDataType dt, const void *ptr, uint64_t inner, uint64_t outer,
                   uint64_t row_bytes, uint32_t box_in, uint32_t box_out, CUtensorMapSwizzle sw) {
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_in, box_out};
  const cuuint32_t es[2] = {1, 1};
  return encode_fn()(m, dt, 2, const_cast<void *>(ptr), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

// The operands of one launch.  dual: wq2 / scales2 / biases2 and y2 are the
// second weight and its output; silu: x holds the gate vectors, x2 the up
// vectors and resid the optional residual.
struct PipeIn {
  const uint16_t *x = nullptr, *x2 = nullptr, *resid = nullptr;
  const float *sw = nullptr;   // w4a8, i8w8: per-row weight scales
  const float *sx = nullptr;   // i8w8: per-token activation scales
  int32_t *acc = nullptr;      // i8w8: optional int32 sums
  int M = 0;
  const uint32_t *wq = nullptr, *wq2 = nullptr;
  const uint16_t *scales = nullptr, *biases = nullptr, *scales2 = nullptr, *biases2 = nullptr;
  int64_t N = 0, K = 0;
  uint16_t *y = nullptr, *y2 = nullptr;
};

// Tensor maps of one weight: packed words as one 3-D box per stage
// ([2 segments][16 rows][32 words]) when allow_w3d and the driver accepts the
// view, else two 2-D boxes; scales and biases as one 3-D box over both arrays
// (the third dimension steps from the lower array to the higher one) when
// allow_joint, else one 2-D box each.
template <int BITS, int GS>
CUresult weight_maps(const uint32_t *wq, const uint16_t *scales, const uint16_t *biases, int64_t N, int64_t K,
                     bool allow_w3d, bool allow_joint, CUtensorMap &tw, CUtensorMap &tsb, CUtensorMap &tb, int &w3d,
                     int &joint, int &swap, bool with_sb = true) {
  using C = PCfg<BITS, GS>;
  const int64_t G = K / GS;
  const uint64_t words = (uint64_t)K / C::CPW;
  w3d = 0;
  if (allow_w3d && words % 32 == 0) {
    const cuuint64_t dims[3] = {32, (cuuint64_t)N, words / 32};
    const cuuint64_t strides[2] = {words * 4, 128};
    const cuuint32_t box[3] = {32, 16, 2};
    const cuuint32_t es[3] = {1, 1, 1};
    if (encode_fn()(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<uint32_t *>(wq), dims, strides, box, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS)
      w3d = 1;
  }
  CUresult r = CUDA_SUCCESS;
  if (!w3d)
    r = encode_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT32, wq, words, (uint64_t)N, words * 4, 32u, 16u,
                  CU_TENSOR_MAP_SWIZZLE_128B);
  joint = 0;
  swap = 0;
  if (!with_sb) {   // (w4a8: no scale or bias boxes)
    tsb = tw;
    tb = tw;
    return r;
  }
  const uintptr_t ps = reinterpret_cast<uintptr_t>(scales), pb = reinterpret_cast<uintptr_t>(biases);
  const uint64_t diff = ps > pb ? ps - pb : pb - ps;
  swap = pb < ps ? 1 : 0;
  if (r == CUDA_SUCCESS && allow_joint && diff != 0 && diff % 16 == 0 && diff < (1ull << 39)) {
    const cuuint64_t dims[3] = {(cuuint64_t)G, (cuuint64_t)N, 2};
    const cuuint64_t strides[2] = {(cuuint64_t)G * 2, diff};
    const cuuint32_t box[3] = {(cuuint32_t)C::SBG, 16, 2};
    const cuuint32_t es[3] = {1, 1, 1};
    const void *lo = swap ? biases : scales;
    if (encode_fn()(&tsb, CU_TENSOR_MAP_DATA_TYPE_UINT16, 3, const_cast<void *>(lo), dims, strides, box, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS)
      joint = 1;
  }
  if (r == CUDA_SUCCESS && !joint) {
    swap = 0;
    r = encode_2d(&tsb, CU_TENSOR_MAP_DATA_TYPE_UINT16, scales, (uint64_t)G, (uint64_t)N, (uint64_t)G * 2,
                  (uint32_t)C::SBG, 16u, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (r == CUDA_SUCCESS)
      r = encode_2d(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT16, biases, (uint64_t)G, (uint64_t)N, (uint64_t)G * 2,
                    (uint32_t)C::SBG, 16u, CU_TENSOR_MAP_SWIZZLE_NONE);
  } else {
    tb = tsb;   // unused
  }
  return r;
}

// The launch set-up of one weight (or weight pair) at one shape: the plan, the
// weight-dependent kernel arguments and the weights' tensor maps.  It depends
// only on the device, the weight pointers and N, K (a tensor map is a function
// of its address, sizes and strides), so it is computed once and cached.
struct PipeSetup {
  PipeArgs a;
  int P, S;
  size_t smem;
  MapSet<6> maps;
};
struct PipeKey {
  int dev;
  const void *w[6];
  int64_t N, K;
  bool operator==(const PipeKey &o) const {
    return dev == o.dev && N == o.N && K == o.K && std::equal(w, w + 6, o.w);
  }
};
struct PipeKeyHash {
  size_t operator()(const PipeKey &k) const {
    size_t h = std::hash<int64_t>()(k.N * 1315423911ll + k.K) ^ (size_t)k.dev;
    for (const void *p : k.w) h = h * 1099511628211ull ^ std::hash<const void *>()(p);
    return h;
  }
};
struct PipeCache {
  std::mutex mu;
  std::unordered_map<PipeKey, PipeSetup, PipeKeyHash> map;
  bool get(const PipeKey &k, PipeSetup &out) {
    std::lock_guard<std::mutex> lk(mu);
    auto it = map.find(k);
    if (it == map.end()) return false;
    out = it->second;
    return true;
  }
  void put(const PipeKey &k, const PipeSetup &v) {
    std::lock_guard<std::mutex> lk(mu);
    if (map.size() >= 4096) map.clear();   // bounded: a model holds far fewer weights
    map[k] = v;
  }
};

template <int BITS, int GS, int MP, int OP>
gwb_status setup_pipe(const PipeIn &in, PipeSetup &su) {
  using C = PCfg<BITS, GS>;
  const int64_t N = in.N, K = in.K;
  const int64_t G = K / GS;
  if (G % 8 != 0) return GWB_ERR_UNSUPPORTED;                 // scale rows must be 16-byte multiples for TMA
  if ((K * BITS / 8) % 16 != 0) return GWB_ERR_UNSUPPORTED;   // packed rows likewise
  if (!encode_fn()) return fail(GWB_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  const int NSH = (int)((N + 15) / 16);
  const int NS = OP == kOpDual ? 2 * NSH : NSH;
  const int nst = (int)((K + C::KST - 1) / C::KST);
  auto kern = k_gemv_pipe<BITS, GS, MP, OP>;
  // one attribute value for every plan (the cluster occupancy query needs it set)
  if (!ensure_smem_attr(reinterpret_cast<const void *>(kern), (size_t)kSmemPerSM - 4096))
    return fail(GWB_ERR_CUDA, "cudaFuncSetAttribute failed for the decode GEMV");

  // Plan for a K split over S CTAs of a cluster: P CTAs along the strips (at
  // most one wave), ring depth D and shared memory.
  // Launch plan for a K split over S CTAs of a cluster: P CTAs along the
  // strips (one wave), ring depth D and shared memory; per_sm = 2 puts two
  // CTAs on an SM (twice the warps to hide latency, half the ring each).
  struct Plan { int S, P, D, NCS, out_strips; size_t smem; double est; };
  auto plan_for = [&](int S, int per_sm, Plan &pl) -> bool {
    if (nst % S != 0) return false;
    const int NCS = nst / S, KR = NCS * C::KST, GR = KR / GS;
    int P = NS < per_sm * kSMs / S ? NS : per_sm * kSMs / S;
    if (S > 1) {
      const int mc = max_clusters(kern, S, (size_t)kSmemPerSM - 4096);
      if (mc < 1) return false;
      P = P < mc ? P : mc;
    }
    const int out_strips = (NS + P - 1) / P;
    const size_t fixed = (size_t)GR * (C::NMMA / 2) * 4 * MP * 16 + (size_t)GR * 4 * 16 +
                         (size_t)NCS * C::NBM * 32 * 8 + (size_t)kCW * 2 * 16 * MP * 4 +
                         (S > 1 ? (size_t)out_strips * 16 * MP * 4 : 0);
    const size_t per = (size_t)kCW * (C::WB + 2 * C::SBB + 8);
    const size_t avail = (size_t)kSmemPerSM / per_sm - 4096 - 1024;
    if (fixed + 2 * per > avail) return false;
    int D = (int)((avail - fixed) / per);
    D = D > 6 ? 6 : D;
    // estimated critical path, in stage times: stages of the busiest warp,
    // the cost of a cluster barrier pair (about two stages), and the staging
    // of the CTA's K-slice of activations, which every CTA does for itself
    // (measured at about 1.2 stage times per item per thread, three times as
    // much when the silu product is formed there)
    const double items_per_thread = (double)GR * MP * 4 / kThreads;
    const double est = (double)((out_strips * NCS + kCW - 1) / kCW) + (S > 1 ? 2.0 : 0.0) +
                       (OP == kOpSilu ? 3.6 : 1.2) * items_per_thread;
    pl = Plan{S, P, D, NCS, out_strips, 1024 + fixed + (size_t)D * per, est};
    return true;
  };
  Plan best{0, 0, 0, 0, 0, 0, 0.0};
  bool have = false;
  auto consider = [&](int S, int per_sm) {
    Plan pl{0, 0, 0, 0, 0, 0, 0.0};
    if (plan_for(S, per_sm, pl) && (!have || pl.est < best.est)) {
      best = pl;
      have = true;
    }
  };
  if ((int64_t)NS * nst >= 2LL * kSMs * kCW * 4) consider(1, 2);
  consider(1, 1);
  if (OP != kOpI8W8)   // i8w8: the int32 sums are not reduced across a cluster
    for (int S = 2; S <= 8; S *= 2) consider(S, 1);
  if (!have) return GWB_ERR_UNSUPPORTED;
  if (!ensure_smem_attr(reinterpret_cast<const void *>(kern), best.smem))
    return fail(GWB_ERR_CUDA, "cudaFuncSetAttribute failed for %zu bytes of shared memory", best.smem);

  PipeArgs a{};
  a.x = in.x; a.x2 = in.x2; a.resid = in.resid; a.sw = in.sw; a.sx = in.sx; a.acc = in.acc;
  a.y = in.y; a.y2 = in.y2;
  a.M = in.M; a.N = (int)N; a.K = (int)K;
  a.NS = NS; a.NSH = NSH;
  a.NCS = best.NCS; a.D = best.D; a.out_strips = best.S > 1 ? best.out_strips : 0;
  a.ns_per = NS / best.P;
  a.ns_rem = NS % best.P;

  CUtensorMap tw, tsb, tb, tw2, tsb2, tb2;
  int w3d = 0, joint = 0, swap = 0, w3d2 = 0, joint2 = 0, swap2 = 0;
  CUresult r = weight_maps<BITS, GS>(in.wq, in.scales, in.biases, N, K, true, true, tw, tsb, tb, w3d, joint, swap,
                                     OP != kOpW4A8 && OP != kOpI8W8);
  if (OP == kOpDual && r == CUDA_SUCCESS) {
    r = weight_maps<BITS, GS>(in.wq2, in.scales2, in.biases2, N, K, true, true, tw2, tsb2, tb2, w3d2, joint2, swap2);
    // both weights take the same box forms (the kernel has one flag of each)
    if (r == CUDA_SUCCESS && (w3d2 != w3d || joint2 != joint)) {
      const bool w3 = w3d && w3d2, jt = joint && joint2;
      r = weight_maps<BITS, GS>(in.wq, in.scales, in.biases, N, K, w3, jt, tw, tsb, tb, w3d, joint, swap);
      if (r == CUDA_SUCCESS)
        r = weight_maps<BITS, GS>(in.wq2, in.scales2, in.biases2, N, K, w3, jt, tw2, tsb2, tb2, w3d2, joint2, swap2);
    }
  } else {
    tw2 = tw; tsb2 = tsb; tb2 = tb;   // unused
  }
  if (r != CUDA_SUCCESS) return fail(GWB_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  a.w3d = w3d;
  a.sb_joint = joint;
  a.sb_swap = swap;
  a.sb_swap2 = swap2;

  su.a = a;
  su.P = best.P;
  su.S = best.S;
  su.smem = best.smem;
  su.maps.m[0] = tw;
  su.maps.m[1] = tsb;
  su.maps.m[2] = tb;
  su.maps.m[3] = tw2;
  su.maps.m[4] = tsb2;
  su.maps.m[5] = tb2;
  return GWB_OK;
}

template <int BITS, int GS, int MP, int OP>
gwb_status run_pipe(const PipeIn &in, cudaStream_t st) {
  static PipeCache cache;   // one per kernel instance
  if ((in.K / GS) % 8 != 0 || (in.K * BITS / 8) % 16 != 0) return GWB_ERR_UNSUPPORTED;   // (see setup_pipe)
  int dev = 0;
  const cudaError_t de = cudaGetDevice(&dev);
  if (de != cudaSuccess) return fail(GWB_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(de));
  const PipeKey key{dev, {in.wq, in.scales, in.biases, in.wq2, in.scales2, in.biases2}, in.N, in.K};
  PipeSetup su;
  if (!cache.get(key, su)) {
    const gwb_status s = setup_pipe<BITS, GS, MP, OP>(in, su);
    if (s != GWB_OK) return s;
    cache.put(key, su);
  }
  // the arguments of this call
  PipeArgs a = su.a;
  a.x = in.x; a.x2 = in.x2; a.resid = in.resid; a.sw = in.sw; a.sx = in.sx; a.acc = in.acc;
  a.y = in.y; a.y2 = in.y2;
  a.M = in.M;

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)su.P, (unsigned)su.S);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = su.smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int na = 0;
  attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[na].val.programmaticStreamSerializationAllowed = 1;
  na++;
  if (su.S > 1) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = 1;
    attr[na].val.clusterDim.y = (unsigned)su.S;
    attr[na].val.clusterDim.z = 1;
    na++;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  MapsOf<OP> maps;
  for (int i = 0; i < (OP == kOpDual ? 6 : 3); i++) maps.m[i] = su.maps.m[i];
  const cudaError_t e = cudaLaunchKernelEx(&cfg, k_gemv_pipe<BITS, GS, MP, OP>, maps, a);
  if (e != cudaSuccess) return fail(GWB_ERR_CUDA, "decode GEMV launch: %s", cudaGetErrorString(e));
  return GWB_OK;
}

int pad_tokens(int M) { return M <= 1 ? 1 : (M <= 2 ? 2 : (M <= 4 ? 4 : 8)); }

}  // namespace
}  // namespace gwb
