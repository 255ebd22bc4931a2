// Streaming GEMV regime (M <= 8 tokens) for the MLX affine layout: the main
// decode kernel.
//
// Work unit = (strip of 16 output features, K chunk of one 128-byte row
// segment per feature).  Each CTA (16 warps, persistent) owns a contiguous
// range of strips; the CTA's units are cut into 16 equal contiguous ranges,
// one per warp, so the load balance is within one unit.  A warp streams its
// units through a private ring of D shared-memory slots that it refills itself:
//   * lane 0 issues one TMA tile load per slot (16 rows x 128 bytes of packed
//     words, 128-byte swizzled, zero-filled past N and K) and every lane copies
//     one row's bf16 scales or biases with cp.async; all of them complete on
//     the slot's mbarrier;
//   * the warp waits for a slot, unpacks two groups at a time in registers and
//     runs the mma.sync dot products of both groups interleaved on independent
//     accumulators (the same quad layout and K reordering as the register-fed
//     GEMV in k_gemv.cu), then refills the slot D units ahead.
// A strip whose units are split between two warps is finished through shared
// memory in warp order.  The activation staging (B fragments and per-group
// sums) is done once per CTA while the first slots load.  When the strips
// cannot fill the GPU, a cluster of up to 8 CTAs splits K and CTA rank 0 sums
// the partial results through distributed shared memory.  Every reduction has
// a fixed order, so results are deterministic.
#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include <map>
#include <mutex>

#include "internal.h"
#include "ptx.cuh"

namespace cg = cooperative_groups;

namespace gwb {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kSmemPerSM = 232448;
constexpr int kSMs = 148;

__device__ __forceinline__ float bf16_val(uint16_t h) { return __uint_as_float(static_cast<uint32_t>(h) << 16); }

__device__ __forceinline__ void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Unpacks one word into fp16 pairs with 2 + log2 ops per pair at most: pair i
// holds the codes at in-word positions i (low half) and i + RPW (high half),
// each OR-ed into the mantissa of 1024.0 at the bit offset it already has in
// the word, so pair i carries 1024 + code * 2^lsig(i) (exact).  The staged
// activations for pair i are divided by the same power of two, which makes
// every product (1024 + code * 2^lsig) * x / 2^lsig = 1024 * x / 2^lsig + code * x.
template <int BITS>
__host__ __device__ constexpr int lsig(int i) {
  return BITS == 4 ? (i & 1) * 4 : (BITS == 2 ? (i & 3) * 2 : 0);
}

template <int BITS>
__device__ __forceinline__ void unpack_word(uint32_t w, uint32_t *r) {
  constexpr uint32_t MAG = 0x64006400u;
  if constexpr (BITS == 4) {
    const uint32_t t = w >> 8;
    r[0] = (w & 0x000F000Fu) | MAG;
    r[1] = (w & 0x00F000F0u) | MAG;
    r[2] = (t & 0x000F000Fu) | MAG;
    r[3] = (t & 0x00F000F0u) | MAG;
  } else if constexpr (BITS == 8) {
    r[0] = __byte_perm(w, 0x64646464u, 0x4240);
    r[1] = __byte_perm(w, 0x64646464u, 0x4341);
  } else {
    const uint32_t t = w >> 8;
#pragma unroll
    for (int i = 0; i < 4; i++) {
      r[i] = (w & (0x00030003u << (2 * i))) | MAG;
      r[4 + i] = (t & (0x00030003u << (2 * i))) | MAG;
    }
  }
}

template <int BITS, int GS>
struct SCfg {
  static constexpr int CPW = 32 / BITS;               // codes per word
  static constexpr int RPW = CPW / 2;                 // fp16 pairs per word
  static constexpr int GW = GS / CPW;                 // words per group per row
  static constexpr int W = GW / 4;                    // words per lane per group
  static constexpr int NMMA = GS / 16;                // MMAs per group
  static constexpr int NR = W * RPW;                  // registers per row per group
  static constexpr int KS = 32 * CPW;                 // k per slot: one 128-byte row segment
  static constexpr int GPS = KS / GS;                 // groups per slot
  static constexpr int GB = GPS >= 2 ? 2 : 1;         // groups processed together
  static constexpr int WBYTES = 2048;                 // 16 rows x 128 bytes
  // bytes of scales (or biases) per row per slot; a single group (8-bit, gs 128)
  // is copied as the aligned pair of groups that holds it
  static constexpr int SROW = GPS * 2 < 4 ? 4 : GPS * 2;
  static constexpr int SLOT = (WBYTES + 2 * 16 * SROW + 1023) / 1024 * 1024;
  static_assert(W >= 1, "group too small for the quad layout");
};

template <int W, int CPW, int RPW>
__device__ __forceinline__ int unit_pos(int rho, int c, int h) {
  return (c * W + rho / RPW) * CPW + rho % RPW + h * RPW;
}

struct StreamArgs {
  const uint16_t *x;
  const uint16_t *scales, *biases;
  uint16_t *y;
  int M, N, K, G;
  int NS;          // strips of 16 rows
  int NC;          // chunks (slots) per strip in this CTA's K-slice
  int D;           // ring depth per warp
  int scale_align; // widest aligned copy of a row's scales: 16, 8 or 4 bytes
  int out_strips;  // split-K only: strips per CTA that the OUT buffer holds
};

struct PartRec {   // a strip result that one warp holds only part of
  int strip, first_chunk;
};

template <int BITS, int GS, int MP>
__global__ void __launch_bounds__(kThreads, 1)
    k_gemv_stream(const __grid_constant__ CUtensorMap tm_w, const StreamArgs a) {
  using C = SCfg<BITS, GS>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  __shared__ float red[kWarps * 8], s_scale[8], s_inv[8];
  __shared__ PartRec rec[kWarps][2];
  __shared__ uint2 zero_b[C::GPS * C::NMMA * 4 * MP];
  unsigned char *base = align_smem_1024(smem_raw);

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int D = a.D, NC = a.NC, S = gridDim.y;
  const int KR = NC * C::KS;                       // this CTA's K-slice (whole slots)
  const int GR = KR / GS;
  const int k0 = blockIdx.y * KR;
  unsigned char *ring = base + warp * D * C::SLOT;
  uint2 *XB = reinterpret_cast<uint2 *>(base + kWarps * D * C::SLOT);
  float *XS = reinterpret_cast<float *>(XB + GR * C::NMMA * 4 * MP);
  uint16_t *XR = reinterpret_cast<uint16_t *>(XS + GR * 16);   // [M][KR] raw bf16 activations of the slice
  float *PART = reinterpret_cast<float *>(XR + MP * KR);         // [warp][2][16 rows][MP]
  float *OUT = PART + kWarps * 2 * 16 * MP;                      // split-K only: [strip][16 rows][MP]
  uint64_t *bars = reinterpret_cast<uint64_t *>(OUT + (S > 1 ? a.out_strips * 16 * MP : 0));
  uint64_t *mybar = bars + warp * D;

  // ---- this CTA's strips and this warp's contiguous range of units
  const int sb = (int)((int64_t)blockIdx.x * a.NS / gridDim.x);
  const int se = (int)((int64_t)(blockIdx.x + 1) * a.NS / gridDim.x);
  const int ucta = (se - sb) * NC;
  const int u0 = (int)((int64_t)warp * ucta / kWarps), u1 = (int)((int64_t)(warp + 1) * ucta / kWarps);
  const int units = u1 - u0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kWarps * D; i++) mbar_init(&bars[i], 33);   // 1 expect_tx arrive + 32 cp.async arrives
    fence_mbar_init();
  }
  if (lane == 0) rec[warp][0].strip = rec[warp][1].strip = -1;
  for (int e = threadIdx.x; e < C::GPS * C::NMMA * 4 * MP; e += kThreads) zero_b[e] = make_uint2(0u, 0u);
  __syncthreads();

  const int srow = lane & 15;
  const bool is_bias = lane >= 16;
  const uint16_t *sbase = is_bias ? a.biases : a.scales;
  // loads unit (strip, chunk) into ring slot `slot`
  auto issue = [&](int strip, int chunk, int slot) {
    unsigned char *sl = ring + slot * C::SLOT;
    const int kc = k0 + chunk * C::KS;
    if (lane == 0) {
      fence_proxy_async_smem();
      mbar_arrive_expect_tx(&mybar[slot], C::WBYTES);
      tma_load_2d(sl, &tm_w, kc / C::CPW, strip * 16, &mybar[slot]);
    }
    const int row = strip * 16 + srow;
    const int g0 = (kc / GS) & ~1;                 // even: 4-byte aligned pieces
    unsigned char *dst = sl + C::WBYTES + (is_bias ? 16 * C::SROW : 0) + srow * C::SROW;
    const bool rok = row < a.N;
    const uint16_t *src = sbase + (int64_t)(rok ? row : 0) * a.G;
    if (a.scale_align >= 16 && (C::SROW % 16) == 0) {
#pragma unroll
      for (int q = 0; q < C::SROW / 16; q++) {
        const int g = g0 + q * 8;
        const uint32_t nb = (rok && g < a.G) ? 16u : 0u;
        cp_async_16(dst + q * 16, src + (nb ? g : 0), nb);
      }
    } else if (a.scale_align >= 8 && (C::SROW % 8) == 0) {
#pragma unroll
      for (int q = 0; q < C::SROW / 8; q++) {
        const int g = g0 + q * 4;
        const uint32_t nb = (rok && g < a.G) ? 8u : 0u;
        cp_async_8(dst + q * 8, src + (nb ? g : 0), nb);
      }
    } else {
#pragma unroll
      for (int q = 0; q < C::SROW / 4; q++) {
        const int g = g0 + q * 2;
        const uint32_t nb = (rok && g < a.G) ? 4u : 0u;
        cp_async_4(dst + q * 4, src + (nb ? g : 0), nb);
      }
    }
    cp_async_arrive_noinc(&mybar[slot]);
  };
  // issue-side position (strip, chunk), advanced without divisions
  const int first_strip = sb + u0 / NC;
  int is_strip = first_strip, is_chunk = u0 - (first_strip - sb) * NC;
  auto advance = [&](int &st, int &ch) {
    if (++ch == NC) { ch = 0; ++st; }
  };
  const int pre = units < D ? units : D;
  for (int i = 0; i < pre; i++) {
    issue(is_strip, is_chunk, i);
    advance(is_strip, is_chunk);
  }

  // ---- activations: one vectorized pass over x (raw bf16 into shared memory,
  // |x| max per token), then a per-token power-of-two rescale into fp16
  {
    float m[MP];
#pragma unroll
    for (int t = 0; t < MP; t++) m[t] = 0.0f;
    const int vpt = KR / 8;                        // 16-byte vectors per token
    for (int idx = threadIdx.x; idx < a.M * vpt; idx += kThreads) {
      const int t = idx / vpt, i = idx % vpt;
      const int k = k0 + 8 * i;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (k < a.K) v = __ldg(reinterpret_cast<const uint4 *>(a.x + (int64_t)t * a.K + k));
      reinterpret_cast<uint4 *>(XR + t * KR)[i] = v;
      const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
      float mx = 0.0f;
#pragma unroll
      for (int q = 0; q < 4; q++)
        mx = fmaxf(mx, fmaxf(fabsf(__uint_as_float(w4[q] << 16)), fabsf(__uint_as_float(w4[q] & 0xffff0000u))));
#pragma unroll
      for (int tt = 0; tt < MP; tt++)
        if (tt == t) m[tt] = fmaxf(m[tt], mx);
    }
#pragma unroll
    for (int t = 0; t < MP; t++) {
      float v = m[t];
      for (int off = 16; off; off >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, off));
      if (lane == 0) red[warp * 8 + t] = v;
    }
  }
  __syncthreads();
  if (threadIdx.x < 8) {
    const int t = threadIdx.x;
    float m = 0.0f;
    if (t < a.M)
      for (int w = 0; w < kWarps; w++) m = fmaxf(m, red[w * 8 + t]);
    int e = 0;
    if (m > 0.0f) {
      int ex;
      frexpf(m, &ex);
      e = 14 - ex;
      e = e > 120 ? 120 : (e < -120 ? -120 : e);
    }
    s_scale[t] = pow2f(e);
    s_inv[t] = pow2f(-e);
  }
  __syncthreads();
  // fp16 bits of the rescaled x[t, k0 + kk] divided by 2^ls (0 past K or for absent tokens)
  auto x16 = [&](int t, int kk, int ls) -> uint16_t {
    if (t >= a.M) return 0;                        // XR holds zeros past K
    return __half_as_ushort(__float2half_rn(bf16_val(XR[t * KR + kk]) * s_scale[t] * pow2f(-ls)));
  };
  {
    const int total = GR * C::NMMA * 4 * MP;
    for (int e = threadIdx.x; e < total; e += kThreads) {
      const int t = e % MP, c = (e / MP) % 4, j = (e / (4 * MP)) % C::NMMA, g = e / (4 * MP * C::NMMA);
      uint32_t out[2];
#pragma unroll
      for (int r = 0; r < 2; r++) {
        const int rho = 2 * j + r;
        const int ls = lsig<BITS>(rho % C::RPW);
        const int lo = g * GS + unit_pos<C::W, C::CPW, C::RPW>(rho, c, 0);
        const int hi = g * GS + unit_pos<C::W, C::CPW, C::RPW>(rho, c, 1);
        out[r] = (uint32_t)x16(t, lo, ls) | ((uint32_t)x16(t, hi, ls) << 16);
      }
      XB[e] = make_uint2(out[0], out[1]);
    }
    // per (group, token): X = sum of the fp16 activations (bias term) and
    // XN = -1024 * sum of the staged B values (the magic offsets' contribution)
    for (int e = threadIdx.x; e < GR * 16; e += blockDim.x) XS[e] = 0.0f;   // absent tokens stay 0
    __syncthreads();
    for (int e = warp; e < GR * a.M; e += kWarps) {   // one warp per (group, present token)
      const int t = e % a.M, g = e / a.M;
      float sx = 0.0f, sb = 0.0f;
        for (int i = lane; i < GS; i += 32) {
          sx += __half2float(__ushort_as_half(x16(t, g * GS + i, 0)));
          sb += __half2float(__ushort_as_half(x16(t, g * GS + i, lsig<BITS>((i % C::CPW) % C::RPW))));
        }
      for (int off = 16; off; off >>= 1) {
        sx += __shfl_xor_sync(kFull, sx, off);
        sb += __shfl_xor_sync(kFull, sb, off);
      }
      if (lane == 0) {
        XS[g * 16 + t] = sx;
        XS[g * 16 + 8 + t] = -1024.0f * sb;
      }
    }
  }
  __syncthreads();

  // ---- main loop
  const int g8 = lane >> 2, c = lane & 3;
  const int tB = (g8 < MP) ? g8 : 0;
  const bool hasB = g8 < MP;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  bool aborted = false;
  int consumed = 0, strip_first_chunk = -1;

  // Flushes the accumulators of `strip`: straight to y (or the split-K OUT
  // buffer) when this warp computed all of its chunks, else to a partial record.
  auto flush = [&](int strip, int first_chunk, int last_chunk) {
    const bool whole = first_chunk == 0 && last_chunk == NC - 1;
    float v[4];
#pragma unroll
    for (int i = 0; i < 4; i++) v[i] = acc[i] * s_inv[2 * c + (i & 1)];
    if (whole && S == 1) {
      const int rA = strip * 16 + g8, rB = rA + 8;
#pragma unroll
      for (int i = 0; i < 4; i++) {
        const int t = 2 * c + (i & 1), row = (i < 2) ? rA : rB;
        if (t < a.M && row < a.N) a.y[(int64_t)t * a.N + row] = __bfloat16_as_ushort(__float2bfloat16_rn(v[i]));
      }
    } else {
      float *dst;
      if (whole) {
        dst = OUT + (strip - sb) * 16 * MP;
      } else {
        // only a warp's first and last strip can be partial: record 0 / record 1
        const int z = (strip == first_strip) ? 0 : 1;
        dst = PART + (warp * 2 + z) * 16 * MP;
        if (lane == 0) rec[warp][z] = PartRec{strip, first_chunk};
        __syncwarp();
      }
#pragma unroll
      for (int i = 0; i < 4; i++) {
        const int t = 2 * c + (i & 1), r = g8 + ((i < 2) ? 0 : 8);
        if (t < MP) dst[r * MP + t] = v[i];
      }
    }
#pragma unroll
    for (int i = 0; i < 4; i++) acc[i] = 0.f;
  };

  // lane constants: byte offsets (within a slot) of this lane's words of group j
  // in row g8 (row g8 + 8 is 1024 bytes further: same swizzle phase), and
  // per-lane bases of the staged B fragments and group sums
  constexpr int Q = (C::W + 3) / 4;
  constexpr int SH = C::SROW / 2;                  // halves per row in the slot's scale area
  int woff[C::GPS][Q];
#pragma unroll
  for (int j = 0; j < C::GPS; j++)
#pragma unroll
    for (int q = 0; q < Q; q++) {
      const int wo = j * C::GW + c * C::W + q * 4;
      woff[j][q] = g8 * 128 + ((((wo >> 2) ^ g8) & 7) << 4) + ((wo & 3) << 2);
    }
  // lanes whose token is absent (g8 >= MP) read a block of zeros that does not move with the chunk
  constexpr int XB_CHUNK = C::GPS * C::NMMA * 4 * MP;   // uint2 entries per chunk
  const uint2 *xbl = hasB ? XB + c * MP + tB : zero_b;
  const int xb_stride = hasB ? XB_CHUNK : 0;
  const float *xsl = XS + 2 * c;

  int slot = 0;
  uint32_t phase = 0;
  int cur_strip = first_strip, chunk = u0 - (first_strip - sb) * NC;
  for (int i = 0; i < units; i++) {
    if (!mbar_wait(&mybar[slot], phase)) { aborted = true; break; }
    const unsigned char *sl = ring + slot * C::SLOT;
    if (strip_first_chunk < 0) strip_first_chunk = chunk;
    const int goff = (C::GPS == 1) ? (((k0 + chunk * C::KS) / GS) & 1) : 0;
    const uint16_t *sc = reinterpret_cast<const uint16_t *>(sl + C::WBYTES) + goff + g8 * SH;
    const uint16_t *bi = sc + 16 * SH;
    const uint2 *xb = xbl + chunk * xb_stride;
    const float *xs = xsl + chunk * (C::GPS * 16);
#pragma unroll
    for (int j0 = 0; j0 < C::GPS; j0 += C::GB) {
      float sa[C::GB], ba[C::GB], sbv[C::GB], bbv[C::GB];
      if constexpr (C::GB == 2) {   // scales / biases of groups j0, j0+1 as one 32-bit load each
        const uint32_t s2a = *reinterpret_cast<const uint32_t *>(sc + j0);
        const uint32_t b2a = *reinterpret_cast<const uint32_t *>(bi + j0);
        const uint32_t s2b = *reinterpret_cast<const uint32_t *>(sc + 8 * SH + j0);
        const uint32_t b2b = *reinterpret_cast<const uint32_t *>(bi + 8 * SH + j0);
        sa[0] = __uint_as_float(s2a << 16); sa[1] = __uint_as_float(s2a & 0xffff0000u);
        ba[0] = __uint_as_float(b2a << 16); ba[1] = __uint_as_float(b2a & 0xffff0000u);
        sbv[0] = __uint_as_float(s2b << 16); sbv[1] = __uint_as_float(s2b & 0xffff0000u);
        bbv[0] = __uint_as_float(b2b << 16); bbv[1] = __uint_as_float(b2b & 0xffff0000u);
      } else {
        sa[0] = bf16_val(sc[j0]);
        ba[0] = bf16_val(bi[j0]);
        sbv[0] = bf16_val(sc[8 * SH + j0]);
        bbv[0] = bf16_val(bi[8 * SH + j0]);
      }
      uint32_t ra[C::GB][C::NR], rb[C::GB][C::NR];
#pragma unroll
      for (int gi = 0; gi < C::GB; gi++) {
        uint32_t wa[C::W], wb[C::W];
#pragma unroll
        for (int q = 0; q < Q; q++) {
          const unsigned char *pa = sl + woff[j0 + gi][q];
          if constexpr (C::W == 1) {
            wa[0] = *reinterpret_cast<const uint32_t *>(pa);
            wb[0] = *reinterpret_cast<const uint32_t *>(pa + 1024);
          } else if constexpr (C::W == 2) {
            const uint2 va = *reinterpret_cast<const uint2 *>(pa), vb = *reinterpret_cast<const uint2 *>(pa + 1024);
            wa[0] = va.x; wa[1] = va.y; wb[0] = vb.x; wb[1] = vb.y;
          } else {
            const uint4 va = *reinterpret_cast<const uint4 *>(pa), vb = *reinterpret_cast<const uint4 *>(pa + 1024);
            wa[4 * q] = va.x; wa[4 * q + 1] = va.y; wa[4 * q + 2] = va.z; wa[4 * q + 3] = va.w;
            wb[4 * q] = vb.x; wb[4 * q + 1] = vb.y; wb[4 * q + 2] = vb.z; wb[4 * q + 3] = vb.w;
          }
        }
#pragma unroll
        for (int w = 0; w < C::W; w++) {
          unpack_word<BITS>(wa[w], &ra[gi][w * C::RPW]);
          unpack_word<BITS>(wb[w], &rb[gi][w * C::RPW]);
        }
      }
      // the GB groups' MMA chains interleaved (independent accumulators)
      float p[C::GB][4];
#pragma unroll
      for (int gi = 0; gi < C::GB; gi++)
#pragma unroll
        for (int q = 0; q < 4; q++) p[gi][q] = 0.f;
#pragma unroll
      for (int m = 0; m < C::NMMA; m++) {
#pragma unroll
        for (int gi = 0; gi < C::GB; gi++) {
          const uint2 b = xb[((j0 + gi) * C::NMMA + m) * 4 * MP];
          const uint32_t af[4] = {ra[gi][2 * m], rb[gi][2 * m], ra[gi][2 * m + 1], rb[gi][2 * m + 1]};
          mma_f16_16816(p[gi], af, b.x, b.y);
        }
      }
#pragma unroll
      for (int gi = 0; gi < C::GB; gi++) {
        const float2 X = *reinterpret_cast<const float2 *>(xs + (j0 + gi) * 16);
        const float2 XN = *reinterpret_cast<const float2 *>(xs + (j0 + gi) * 16 + 8);
        acc[0] = fmaf(sa[gi], p[gi][0] + XN.x, fmaf(ba[gi], X.x, acc[0]));
        acc[1] = fmaf(sa[gi], p[gi][1] + XN.y, fmaf(ba[gi], X.y, acc[1]));
        acc[2] = fmaf(sbv[gi], p[gi][2] + XN.x, fmaf(bbv[gi], X.x, acc[2]));
        acc[3] = fmaf(sbv[gi], p[gi][3] + XN.y, fmaf(bbv[gi], X.y, acc[3]));
      }
    }
    __syncwarp();
    consumed = i + 1;
    if (chunk == NC - 1 || i == units - 1) {
      flush(cur_strip, strip_first_chunk, chunk);
      strip_first_chunk = -1;
    }
    advance(cur_strip, chunk);
    if (i + D < units) {
      issue(is_strip, is_chunk, slot);
      advance(is_strip, is_chunk);
    }
    if (++slot == D) { slot = 0; phase ^= 1; }
  }
  if (aborted) {
    // drain: every issued slot must land before the CTA may exit
    const int issued = units < consumed + D ? units : consumed + D;
    for (int i = consumed; i < issued; i++) mbar_wait(&mybar[i % D], (i / D) & 1);
  }
  __syncthreads();

  // ---- strips split between warps: the record holding chunk 0 sums the others in warp order
  for (int e = warp; e < kWarps * 2; e += kWarps) {
    const int w = e >> 1, z = e & 1;
    const PartRec r = rec[w][z];
    if (r.strip < 0 || r.first_chunk != 0) continue;
    for (int idx = lane; idx < 16 * MP; idx += 32) {
      float s = PART[(w * 2 + z) * 16 * MP + idx];
      for (int w2 = w + 1; w2 < kWarps; w2++)
        for (int z2 = 0; z2 < 2; z2++)
          if (rec[w2][z2].strip == r.strip) s += PART[(w2 * 2 + z2) * 16 * MP + idx];
      const int row = r.strip * 16 + idx / MP, t = idx % MP;
      if (S == 1) {
        if (t < a.M && row < a.N) a.y[(int64_t)t * a.N + row] = __bfloat16_as_ushort(__float2bfloat16_rn(s));
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
        const int row = sb * 16 + e / MP, t = e % MP;
        if (t < a.M && row < a.N) a.y[(int64_t)t * a.N + row] = __bfloat16_as_ushort(__float2bfloat16_rn(s));
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

// Per-kernel caches of the dynamic shared-memory attribute and of the number
// of co-resident clusters, so that steady-state calls (and calls made while a
// stream is being captured into a CUDA graph) do no occupancy queries.
struct ClusterKey {
  const void *fn;
  int S;
  size_t smem;
  bool operator<(const ClusterKey &o) const {
    return fn != o.fn ? fn < o.fn : (S != o.S ? S < o.S : smem < o.smem);
  }
};
std::mutex g_cache_mu;
std::map<ClusterKey, int> g_max_clusters;
std::map<const void *, size_t> g_smem_attr;

bool cached_max_clusters(const void *fn, int S, size_t smem, int *n) {
  std::lock_guard<std::mutex> lk(g_cache_mu);
  auto it = g_max_clusters.find(ClusterKey{fn, S, smem});
  if (it == g_max_clusters.end()) return false;
  *n = it->second;
  return true;
}
void store_max_clusters(const void *fn, int S, size_t smem, int n) {
  std::lock_guard<std::mutex> lk(g_cache_mu);
  g_max_clusters[ClusterKey{fn, S, smem}] = n;
}
bool ensure_smem_attr(const void *fn, size_t smem) {
  std::lock_guard<std::mutex> lk(g_cache_mu);
  size_t &cur = g_smem_attr[fn];
  if (cur >= smem) return true;
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess) return false;
  cur = smem;
  return true;
}

template <int BITS, int GS, int MP>
gwb_status run_stream(const uint16_t *x, int M, const uint32_t *wq, const uint16_t *scales, const uint16_t *biases,
                      int64_t N, int64_t K, uint16_t *y, cudaStream_t st) {
  using C = SCfg<BITS, GS>;
  const int G = (int)(K / GS);
  if (G % 2 != 0) return GWB_ERR_UNSUPPORTED;                // scales are copied in 4-byte pieces
  if ((K * BITS / 8) % 16 != 0) return GWB_ERR_UNSUPPORTED;   // TMA row stride
  const int NS = (int)((N + 15) / 16);
  const int nc_total = (int)((K + C::KS - 1) / C::KS);
  auto kern = k_gemv_stream<BITS, GS, MP>;

  // Launch plan for a K split over S CTAs of a cluster: P clusters (CTAs along
  // the strips), ring depth D and shared memory.  P is capped by how many such
  // clusters can be co-resident, so the grid runs in a single wave.
  struct Plan { int S, P, D, NC; size_t smem; };
  auto plan_for = [&](int S, Plan &pl) -> bool {
    if (nc_total % S != 0) return false;
    const int NC = nc_total / S, KR = NC * C::KS;
    int P = NS < kSMs / S ? NS : kSMs / S;
    for (int pass = 0; pass < 2; pass++) {
      const int out_strips = S > 1 ? (NS + P - 1) / P : 0;
      const size_t fixed = (size_t)KR * 2 * MP + (size_t)(KR / GS) * 16 * 4 + (size_t)MP * KR * 2 +
                           (size_t)kWarps * 2 * 16 * MP * 4 + (size_t)out_strips * 16 * MP * 4;
      int D = 4;
      size_t smem = 0;
      for (; D >= 2; D--) {
        smem = 1024 + (size_t)kWarps * D * C::SLOT + fixed + (size_t)kWarps * D * 8;
        if (smem <= (size_t)kSmemPerSM - 8192) break;   // leave room for static shared memory
      }
      if (D < 2) return false;
      if (!ensure_smem_attr(reinterpret_cast<const void *>(kern), smem)) return false;
      int maxc = kSMs / S;
      if (S > 1 && !cached_max_clusters(reinterpret_cast<const void *>(kern), S, smem, &maxc)) {
        cudaLaunchConfig_t q = {};
        q.gridDim = dim3((unsigned)P, (unsigned)S);
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
        if (cudaOccupancyMaxActiveClusters(&n, kern, &q) != cudaSuccess || n < 1) return false;
        maxc = n;
        store_max_clusters(reinterpret_cast<const void *>(kern), S, smem, n);
      }
      pl = Plan{S, P, D, NC, smem};
      if (P <= maxc) return true;
      P = maxc;   // second pass: fewer clusters, more strips each
    }
    return pl.P > 0;
  };
  // Persistent CTAs when every warp gets units; otherwise the K split that keeps
  // the most CTAs busy.
  Plan best{0, 0, 0, 0, 0};
  if (!plan_for(1, best)) return GWB_ERR_UNSUPPORTED;
  if ((int64_t)NS * nc_total < 2LL * kSMs * kWarps) {
    for (int S = 2; S <= 8; S *= 2) {
      Plan pl{0, 0, 0, 0, 0};
      if (plan_for(S, pl) && pl.S * pl.P > best.S * best.P) best = pl;
    }
  }
  const int S = best.S, P = best.P, D = best.D, NC = best.NC;
  const size_t smem = best.smem;
  if (!ensure_smem_attr(reinterpret_cast<const void *>(kern), smem))
    return fail(GWB_ERR_CUDA, "cudaFuncSetAttribute failed for %zu bytes of shared memory", smem);

  auto fn = encode_fn();
  if (!fn) return fail(GWB_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  CUtensorMap tm;
  const uint64_t words = (uint64_t)K / C::CPW;
  const cuuint64_t dims[2] = {words, (cuuint64_t)N};
  const cuuint64_t strides[1] = {words * 4};
  const cuuint32_t box[2] = {32, 16};
  const cuuint32_t es[2] = {1, 1};
  CUresult r = fn(&tm, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t *>(wq), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(GWB_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);

  StreamArgs a{};
  a.x = x; a.scales = scales; a.biases = biases; a.y = y;
  a.M = M; a.N = (int)N; a.K = (int)K; a.G = G;
  a.NS = NS; a.NC = NC; a.D = D;
  a.scale_align = (G % 8 == 0) ? 16 : ((G % 4 == 0) ? 8 : 4);
  a.out_strips = S > 1 ? (NS + P - 1) / P : 0;

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)P, (unsigned)S);
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
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, tm, a);
  if (e != cudaSuccess) return fail(GWB_ERR_CUDA, "streaming GEMV launch: %s", cudaGetErrorString(e));
  return GWB_OK;
}

int pad_tokens(int M) { return M <= 1 ? 1 : (M <= 2 ? 2 : (M <= 4 ? 4 : 8)); }

}  // namespace

gwb_status launch_gemv_stream(const uint16_t *x, int M, const uint32_t *wq, const uint16_t *scales,
                              const uint16_t *biases, int64_t N, int64_t K, int bits, int gs, uint16_t *y,
                              cudaStream_t st) {
  const int MP = pad_tokens(M);
#define GWB_GS(B, S, P) \
  if (bits == B && gs == S && MP == P) return run_stream<B, S, P>(x, M, wq, scales, biases, N, K, y, st);
#define GWB_GS_MP(B, S) GWB_GS(B, S, 1) GWB_GS(B, S, 2) GWB_GS(B, S, 4) GWB_GS(B, S, 8)
  GWB_GS_MP(2, 64) GWB_GS_MP(2, 128)
  GWB_GS_MP(4, 32) GWB_GS_MP(4, 64) GWB_GS_MP(4, 128)
  GWB_GS_MP(8, 32) GWB_GS_MP(8, 64) GWB_GS_MP(8, 128)
#undef GWB_GS_MP
#undef GWB_GS
  return GWB_ERR_UNSUPPORTED;
}

}  // namespace gwb
