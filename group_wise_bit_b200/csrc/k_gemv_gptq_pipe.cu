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
// lane 0 issues three tiled TMA loads per stage (the codes as one box of 32
// rows x 128 bytes, the scales and the zero words as boxes of the stage's
// groups), all completing on the slot's mbarrier; a slot is refilled as soon
// as the warp has read it.  (Copies of single 128-byte runs were bound by the
// rate of TMA operations, about one per 25 cycles per SM.)  A warp holds only a few
// stages, so most of a CTA's weights are requested at once, at kernel start.
//
// Per 32 in-features of a stage (4 qweight rows, stored with the 128-byte
// swizzle), lane (g = lane / 4, c = lane % 4) reads the 16 bytes of row c that
// hold the strip's features 4G .. 4G + 3 (G = g / 2 + 4 (g % 2): the two quads
// of a quarter-warp read chunks q and q + 4, conflict-free).  Each code
// becomes the fp16 value 1024 + code (one LOP3 per two codes).  The codes of
// features (4G, 4G + 1) and of (4G + 2, 4G + 3) are the A fragments (rows g,
// g + 8) of two m16n8k16 MMAs (fp16 in, fp32 accumulate) against activations
// staged once per CTA as ready-made B fragments (tokens are the MMA's N
// dimension, padded to 8); the order of in-features inside the 32 is free, so
// the staged activations follow the order the unpacked registers imply.
//   * Without g_idx the MMAs sum (1024 + q) x over each group, and the group
//     adds s * (that - (1024 + zero) * sum_k x) to the output (the x sums are
//     staged with the fragments): the scale and zero cost two FMAs per value
//     and group, not one operation per weight.
//   * With g_idx every in-feature has its own group, so the weights are
//     dequantized before the MMA: (1024 + q) - (1024 + zero), times the scale
//     (one half2 operation each, one rounding: the fp16 weight gptq_dequant
//     writes), with the scales and zeros read through the L1 cache.
// Consecutive units feed four rotating accumulator chains, so that the MMAs of
// a stage do not wait on one another.
//
// A strip whose stages are split between warps is finished through shared
// memory in warp order, i.e. in K order: results are deterministic.
#include <cuda_fp16.h>

#include <cudaTypedefs.h>

#include <atomic>
#include <climits>
#include <cstdint>
#include <functional>
#include <mutex>
#include <unordered_map>

#include "internal.h"
#include "ptx.cuh"

namespace gwb {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kGW = 8;                               // warps per CTA
constexpr int kGThreads = kGW * 32;
constexpr int kStripN = 32;                          // output features per strip
constexpr int kStageK = 256;                         // in-features per stage
constexpr int kCodesB = kStripN * 4 * (kStageK / 8); // 4096 bytes of codes per stage
constexpr int kScaleBoxB = 8 * kStripN * 2;          // up to 8 groups x 32 fp16 scales
constexpr int kZeroBoxB = 8 * 16;                    // up to 8 groups x 4 zero words
constexpr int kSlotB = 5120;                         // codes (1024-aligned for the swizzle), scales, zeros
static_assert(kCodesB + kScaleBoxB + kZeroBoxB <= kSlotB && kSlotB % 1024 == 0, "ring slot layout");
constexpr int kMaxDynSmem = 232448;                  // per CTA
constexpr int kSmemPerSM = 233472;
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

// Feature chunk of quad g: quads 2q and 2q + 1 take the 4-feature chunks q and
// q + 4, so that a quarter-warp's eight 16-byte reads (four qweight rows x two
// chunks) fall in eight different bank groups of the 128-byte-swizzled stage.
__device__ __forceinline__ int quad_chunk(int g) { return (g >> 1) | ((g & 1) << 2); }

template <int MP, bool GIDX, int GS>
__global__ void __launch_bounds__(kGThreads, 2)
    k_gemv_gptq_pipe(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_s,
                     const __grid_constant__ CUtensorMap tm_z, const GArgs a) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char *smem = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ int rec[kGW][2];   // strip of each warp's partial slot (first, last segment), or -1

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, c = lane & 3, G4 = quad_chunk(g);
  const int D = a.D, nks = a.nks, N = a.N;
  unsigned char *ring = smem + (size_t)warp * D * kSlotB;
  uint2 *XB = reinterpret_cast<uint2 *>(smem + (size_t)kGW * D * kSlotB);      // [K/32][2][4][MP]
  float *XS = reinterpret_cast<float *>(XB + (size_t)(a.K / 32) * 8 * MP);      // [G][MP] group sums of x
  float *PART = XS + (GIDX ? 0 : (size_t)a.G * MP);                              // [kGW][2][32][MP]
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
  if (threadIdx.x == 0) {
    tma_prefetch_desc(&tm_w);
    if (!GIDX) {
      tma_prefetch_desc(&tm_s);
      tma_prefetch_desc(&tm_z);
    }
  }
  fence_mbar_init();
  __syncwarp();

  // stage i of this warp into ring slot `slot` (issued by lane 0)
  auto issue = [&](int i, int slot) {
    if (lane != 0) return;
    const int su = u0 + i;
    const int sq = su / nks;
    const int strip = sb + sq, ks = su - sq * nks;
    const int n0 = strip * kStripN;
    unsigned char *dst = ring + slot * kSlotB;
    uint64_t *bar = &full[slot];
    constexpr int gps = kStageK / GS;                 // groups per stage
    mbar_arrive_expect_tx(bar, kCodesB + (GIDX ? 0 : gps * (kStripN * 2 + 16)));
    tma_load_2d(dst, &tm_w, n0, ks * (kStageK / 8), bar);
    if constexpr (!GIDX) {
      const int g0 = ks * gps;
      tma_load_2d(dst + kCodesB, &tm_s, n0, g0, bar);
      tma_load_2d(dst + kCodesB + kScaleBoxB, &tm_z, n0 / 8, g0, bar);
    }
  };

  // the first stage is requested before the activations are staged, the rest of
  // the ring after (the staging's loads are not held up by the copies' issue)
  const int pre = nst < D ? nst : D;
  if (pre > 0) issue(0, 0);
  int issued = pre;

  // Activations.  Item e = (token t, chunk q of 8 in-features) loads x[t, 8q .. 8q + 7]
  // with one 16-byte load and writes the two B fragments of quad lane c = q % 4 of
  // unit u = q / 4: XB[u][j][c][t] = pairs (x[k + 2j], x[k + 2j + 4]) and
  // (x[k + 2j + 1], x[k + 2j + 5]), k = 8q, matching the unpacked registers.
  // Without g_idx the chunk sums (fp32, in order) are added over each group's
  // chunks, which sit in consecutive lanes, by a fixed shuffle tree: XS[group][t].
  // Two items per round, both loaded before either is used.
  {
    const int kq = a.K / 8;                 // chunks per token, a multiple of 32
    const int total = kq * MP;
    constexpr int cpg = GS / 8;             // chunks per group: 4, 8 or 16
    for (int e0 = threadIdx.x; e0 < total; e0 += 2 * kGThreads) {
      uint4 v[2];
#pragma unroll
      for (int h = 0; h < 2; h++) {
        const int e = e0 + h * kGThreads;
        const int t = e / kq, q = e - t * kq;
        v[h] = make_uint4(0u, 0u, 0u, 0u);
        if (e < total && t < a.M) v[h] = __ldg(reinterpret_cast<const uint4 *>(a.x + (size_t)t * a.K + (size_t)q * 8));
      }
#pragma unroll
      for (int h = 0; h < 2; h++) {
        const int e = e0 + h * kGThreads;
        if (e >= total) break;                // the same for the whole warp (total is a multiple of 32)
        const int t = e / kq, q = e - t * kq;
        const int u = q >> 2, cc = q & 3;
        XB[((u * 2 + 0) * 4 + cc) * MP + t] =
            make_uint2(__byte_perm(v[h].x, v[h].z, 0x5410), __byte_perm(v[h].x, v[h].z, 0x7632));
        XB[((u * 2 + 1) * 4 + cc) * MP + t] =
            make_uint2(__byte_perm(v[h].y, v[h].w, 0x5410), __byte_perm(v[h].y, v[h].w, 0x7632));
        if constexpr (!GIDX) {
          const uint32_t w[4] = {v[h].x, v[h].y, v[h].z, v[h].w};
          float s = 0.0f;
#pragma unroll
          for (int p = 0; p < 4; p++) {
            s += __half2float(__ushort_as_half((uint16_t)(w[p] & 0xffffu)));
            s += __half2float(__ushort_as_half((uint16_t)(w[p] >> 16)));
          }
#pragma unroll
          for (int off = 1; off < cpg; off <<= 1) s += __shfl_xor_sync(kFull, s, off);
          if ((q & (cpg - 1)) == 0) XS[(q / cpg) * MP + t] = s;
        }
      }
    }
  }
  for (int i = 1; i < pre; i++) issue(i, i);
  __syncthreads();

  // Output accumulators (features 4G4, 4G4 + 1 at tokens 2c, 2c + 1, then 4G4 + 2,
  // 4G4 + 3) and four rotating MMA chains (unit u feeds chain u % 4), so that no
  // MMA waits for the one before it in the same stage.
  float yacc[8], pc[GIDX ? 4 : GS / 32][8];
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
          if (t < a.M) a.y[(size_t)t * N + n0 + 4 * G4 + jn] = __half_as_ushort(__float2half_rn(yacc[2 * jn + h]));
        }
    } else {
      const int sl = first_seg ? 0 : 1;
      float *P = PART + (warp * 2 + sl) * 32 * MP;
#pragma unroll
      for (int jn = 0; jn < 4; jn++)
#pragma unroll
        for (int h = 0; h < 2; h++) {
          const int t = 2 * c + h;
          if (t < MP) P[(4 * G4 + jn) * MP + t] = yacc[2 * jn + h];
        }
      if (lane == 0) rec[warp][sl] = cur;
    }
    first_seg = false;
  };

  const bool hasB = g < MP;
  constexpr int UPG = GS / 32;                  // units per group (without g_idx): 1, 2 or 4
  constexpr int NCH = GIDX ? 4 : UPG;           // MMA chains: one per unit of a group
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
      for (int q = 0; q < 8; q++) yacc[q] = 0.0f;
      cur = strip;
      seg_first = ks;
    }
    seg_last = ks;
#pragma unroll
    for (int ch = 0; ch < NCH; ch++)
#pragma unroll
      for (int q = 0; q < 8; q++) pc[ch][q] = 0.0f;
    const unsigned char *S = ring + slot * kSlotB;
    const uint2 *xb = XB + (size_t)ks * 8 * 8 * MP + c * MP + (hasB ? g : 0);
    float sf[4], zf[4], X0 = 0.0f, X1 = 0.0f;   // the current group's scales, 1024 + zero, and x sums
#pragma unroll
    for (int hh = 0; hh < 2; hh++) {
      // the half-stage's codes first (four 16-byte reads in flight together)
      uint4 wv[4];
      uint2 bv[4][2];   // and the half-stage's activation fragments
#pragma unroll
      for (int q = 0; q < 4; q++) {
        const int r = 4 * (4 * hh + q) + c;     // qweight row of the stage (128-byte swizzle)
        wv[q] = *reinterpret_cast<const uint4 *>(S + r * 128 + ((G4 ^ (r & 7)) << 4));
#pragma unroll
        for (int j = 0; j < 2; j++) {
          bv[q][j] = make_uint2(0u, 0u);
          if (hasB) bv[q][j] = xb[((4 * hh + q) * 2 + j) * 4 * MP];
        }
      }
#pragma unroll
      for (int q = 0; q < 4; q++) {
        const int u = 4 * hh + q;
        const uint32_t w4[4] = {wv[q].x, wv[q].y, wv[q].z, wv[q].w};
        uint32_t A[4][4];   // [feature 4G4 + jn][register p: codes (p, p + 4)]
        if constexpr (!GIDX) {
          // y = sum_groups s * (sum_k (1024 + q) x - (1024 + zero) * sum_k x): the MMAs take the
          // codes as unpacked, the group's scale and zero are applied once per group
          if (u % UPG == 0) {
            const int gl = u / UPG;
            const uint2 s4 = *reinterpret_cast<const uint2 *>(S + kCodesB + gl * (kStripN * 2) + 8 * G4);
            const uint32_t zw =
                *reinterpret_cast<const uint32_t *>(S + kCodesB + kScaleBoxB + gl * 16 + 4 * (G4 >> 1)) >>
                ((G4 & 1) * 16);
            sf[0] = __half2float(__ushort_as_half((uint16_t)(s4.x & 0xffffu)));
            sf[1] = __half2float(__ushort_as_half((uint16_t)(s4.x >> 16)));
            sf[2] = __half2float(__ushort_as_half((uint16_t)(s4.y & 0xffffu)));
            sf[3] = __half2float(__ushort_as_half((uint16_t)(s4.y >> 16)));
#pragma unroll
            for (int jn = 0; jn < 4; jn++) zf[jn] = (float)(1024 + (int)((zw >> (4 * jn)) & 0xFu) + a.zadd);
            const int gq = ks * (kStageK / GS) + gl;
            X0 = 2 * c < MP ? XS[gq * MP + 2 * c] : 0.0f;
            X1 = 2 * c + 1 < MP ? XS[gq * MP + 2 * c + 1] : 0.0f;
          }
#pragma unroll
          for (int jn = 0; jn < 4; jn++)
#pragma unroll
            for (int p = 0; p < 4; p++) A[jn][p] = ((w4[jn] >> (4 * p)) & 0x000F000Fu) | 0x64006400u;
        } else {
          // every in-feature has its own group: the lane's eight in-features k0 .. k0 + 7
          const int k0 = ks * kStageK + 32 * u + 8 * c;
          const int4 ga = __ldg(reinterpret_cast<const int4 *>(a.g_idx + k0));
          const int4 gb = __ldg(reinterpret_cast<const int4 *>(a.g_idx + k0 + 4));
          const int gv[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
          const int ncol = cur * kStripN + 4 * G4;
          uint32_t sv[8][2], zv[8];
#pragma unroll
          for (int p = 0; p < 8; p++) {
            const unsigned gq = (unsigned)gv[p] < (unsigned)a.G ? (unsigned)gv[p] : 0u;
            const uint2 s = __ldg(reinterpret_cast<const uint2 *>(a.scales + (size_t)gq * N + ncol));
            sv[p][0] = s.x;
            sv[p][1] = s.y;
            zv[p] = __ldg(a.qzeros + (size_t)gq * (N / 8) + ncol / 8) >> ((G4 & 1) * 16);
          }
#pragma unroll
          for (int jn = 0; jn < 4; jn++)
#pragma unroll
            for (int p = 0; p < 4; p++) {
              // codes p (low half) and p + 4 (high half) of feature 4G4 + jn
              const uint32_t slo = (sv[p][jn >> 1] >> ((jn & 1) * 16)) & 0xffffu;
              const uint32_t shi = (sv[p + 4][jn >> 1] >> ((jn & 1) * 16)) & 0xffffu;
              const uint32_t zlo = 0x6400u | (((zv[p] >> (4 * jn)) & 0xFu) + (uint32_t)a.zadd);
              const uint32_t zhi = 0x6400u | (((zv[p + 4] >> (4 * jn)) & 0xFu) + (uint32_t)a.zadd);
              A[jn][p] = dq2(((w4[jn] >> (4 * p)) & 0x000F000Fu) | 0x64006400u, zlo | (zhi << 16), slo | (shi << 16));
            }
        }
        float *chn = pc[u % NCH];
#pragma unroll
        for (int j = 0; j < 2; j++) {
          const uint2 b = bv[q][j];
          mma_f16_16816(chn, A[0][2 * j], A[1][2 * j], A[0][2 * j + 1], A[1][2 * j + 1], b.x, b.y);
          mma_f16_16816(chn + 4, A[2][2 * j], A[3][2 * j], A[2][2 * j + 1], A[3][2 * j + 1], b.x, b.y);
        }
        if constexpr (!GIDX) {
          if (u % UPG == UPG - 1) {
            // the group's last unit: its chains, then the scale and zero
            float P[8];
#pragma unroll
            for (int q2 = 0; q2 < 8; q2++) {
              float v = 0.0f;
#pragma unroll
              for (int ch = 0; ch < NCH; ch++) {
                v += pc[ch][q2];
                pc[ch][q2] = 0.0f;
              }
              P[q2] = v;
            }
#pragma unroll
            for (int jn = 0; jn < 4; jn++) {
              yacc[2 * jn] = fmaf(sf[jn], fmaf(-zf[jn], X0, P[2 * jn]), yacc[2 * jn]);
              yacc[2 * jn + 1] = fmaf(sf[jn], fmaf(-zf[jn], X1, P[2 * jn + 1]), yacc[2 * jn + 1]);
            }
          }
        }
      }
    }
    if constexpr (GIDX) {
#pragma unroll
      for (int q = 0; q < 8; q++) yacc[q] += (pc[0][q] + pc[1][q]) + (pc[2][q] + pc[3][q]);
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

// ---------------------------------------------------------------- tensor maps
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

// A 2-D row-major view [rows][cols] (cols contiguous) read in boxes of
// [box_rows][box_cols]; false when the driver refuses it.
bool map_2d(CUtensorMap *m, CUtensorMapDataType dt, int es, const void *base, uint64_t cols, uint64_t rows,
            uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_NONE) {
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * (uint64_t)es};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return encode_fn()(m, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The three maps of one weight (codes, scales, zero words), cached per
// (device, tensors, shape, group size): encoding costs host time on every call.
struct GMaps {
  CUtensorMap w, s, z;
};
struct GKey {
  int dev, gs;
  const void *p[3];
  int64_t N, K;
  bool operator==(const GKey &o) const {
    return dev == o.dev && gs == o.gs && N == o.N && K == o.K && p[0] == o.p[0] && p[1] == o.p[1] && p[2] == o.p[2];
  }
};
struct GKeyHash {
  size_t operator()(const GKey &k) const {
    size_t h = std::hash<int64_t>()(k.N * 1315423911ll + k.K * 31 + k.gs) ^ (size_t)k.dev;
    for (const void *q : k.p) h = h * 1099511628211ull ^ std::hash<const void *>()(q);
    return h;
  }
};

gwb_status gptq_maps(const GArgs &a, int gs, GMaps &out) {
  static std::mutex mu;
  static std::unordered_map<GKey, GMaps, GKeyHash> cache;
  if (!encode_fn()) return fail(GWB_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  int dev = 0;
  const cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(GWB_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  const GKey key{dev, gs, {a.qw, a.scales, a.qzeros}, a.N, a.K};
  {
    std::lock_guard<std::mutex> lk(mu);
    auto it = cache.find(key);
    if (it != cache.end()) {
      out = it->second;
      return GWB_OK;
    }
  }
  const uint32_t gps = (uint32_t)(kStageK / gs);
  GMaps m;
  if (!map_2d(&m.w, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, a.qw, (uint64_t)a.N, (uint64_t)a.K / 8, kStripN, kStageK / 8,
              CU_TENSOR_MAP_SWIZZLE_128B) ||
      !map_2d(&m.s, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, a.scales, (uint64_t)a.N, (uint64_t)a.G, kStripN, gps) ||
      !map_2d(&m.z, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, a.qzeros, (uint64_t)a.N / 8, (uint64_t)a.G, kStripN / 8, gps))
    return GWB_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(mu);
  if (cache.size() >= 4096) cache.clear();   // bounded: a model holds far fewer weights
  cache.emplace(key, m);
  out = m;
  return GWB_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

template <int MP, bool GIDX, int GS>
gwb_status run_gptq_pipe(const GArgs &a0, const GMaps &m, int strips, cudaStream_t st) {
  constexpr int SLOT = kSlotB;
  GArgs a = a0;
  const size_t xb = (size_t)a.K * 2 * MP + (GIDX ? 0 : (size_t)a.G * MP * 4), part = (size_t)kGW * 2 * 32 * MP * 4;
  // Two CTAs per SM where each still gets a ring of two slots per warp (a warp
  // takes a few thousand cycles per stage, bound by latency: 16 warps per SM
  // hide twice as much of it as 8), else one CTA per SM with a deeper ring.
  int grid = 0;
  int64_t D = 0;
  for (int per_sm = 2; per_sm >= 1 && grid == 0; per_sm--) {
    const int cap = kNumSMs * per_sm;
    const int gr = strips < cap ? strips : cap;
    const int ns_per = strips / gr, ns_rem = strips % gr;
    const int64_t max_stages = ((int64_t)(ns_per + (ns_rem ? 1 : 0)) * a.nks + kGW - 1) / kGW;
    // dynamic shared memory a CTA may take: half an SM less the static part and the
    // per-CTA reservation, or a whole CTA's maximum
    const int64_t budget = per_sm == 2 ? kSmemPerSM / 2 - 3 * 1024 : kMaxDynSmem - 1024;
    int64_t d = (budget - 1024 - (int64_t)xb - (int64_t)part) / (kGW * (SLOT + 8));
    if (d > max_stages) d = max_stages;
    if (d > kMaxSlots) d = kMaxSlots;
    if (d >= 2 || (d == 1 && max_stages == 1)) {
      grid = gr;
      D = d;
      a.ns_per = ns_per;
      a.ns_rem = ns_rem;
    }
  }
  if (grid == 0) return GWB_ERR_UNSUPPORTED;
  a.D = (int)D;
  const size_t smem = 1024 + (size_t)kGW * D * SLOT + xb + part + (size_t)kGW * D * 8;   // + the alignment
  auto kern = k_gemv_gptq_pipe<MP, GIDX, GS>;
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
  kern<<<grid, kGThreads, smem, st>>>(m.w, m.s, m.z, a);
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
  if (!aligned16(x) || !aligned16(qweight) || !aligned16(scales) || !aligned16(qzeros)) return GWB_ERR_UNSUPPORTED;
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
  GMaps m;
  const gwb_status ms = gptq_maps(a, gs, m);
  if (ms != GWB_OK) return ms;
  // act order: one kernel for every group size (its groups are per in-feature)
#define GWB_GP(P)                                                                           \
  if (MP == P) {                                                                             \
    if (g_idx) return run_gptq_pipe<P, true, 128>(a, m, strips, st);                         \
    if (gs == 32) return run_gptq_pipe<P, false, 32>(a, m, strips, st);                      \
    if (gs == 64) return run_gptq_pipe<P, false, 64>(a, m, strips, st);                      \
    return run_gptq_pipe<P, false, 128>(a, m, strips, st);                                   \
  }
  GWB_GP(1) GWB_GP(2) GWB_GP(4) GWB_GP(8)
#undef GWB_GP
  return GWB_ERR_UNSUPPORTED;
}

}  // namespace gwb
