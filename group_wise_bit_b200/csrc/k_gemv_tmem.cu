// Decode GEMV (M <= 8 tokens) for the MLX affine layout on the tcgen05 tensor
// cores with the weights as a TMEM operand: the main decode kernel.
//
// A CTA owns 128-row tiles of W (persistent over tiles).  Its warps:
//   warps 0-7  row threads: warp w serves row 32*(w%4) + lane of the tile, for
//              half b = w/4 of the tile's K chunks (the two halves are summed at
//              the end of the tile).  Per group of GS columns a thread unpacks
//              its row's codes in registers into fp16 pairs holding
//              1024 + code * 2^lsig (exact), writes them to its own TMEM lane
//              with tcgen05.st (that is the MMA's A operand, 128 rows x GS),
//              and, LAG groups later, reads back the MMA result for its row
//              with tcgen05.ld and applies the group's scale and bias:
//                 acc += s * (P + XN) + b * X
//              where P = sum_k (1024 + code*2^lsig) * x / 2^lsig, XN = -1024 *
//              sum_k x / 2^lsig and X = sum_k x (both staged per group).
//   warp 8     producer: TMA tile loads of the packed words (128 rows x 128
//              bytes per K chunk and half, 128-byte swizzled, zero-filled past
//              N and K) into a ring of stages; its 32 lanes copy the rows' bf16
//              scales and biases of the stage with cp.async onto the same
//              mbarrier.
//   warp 9     TMEM allocation and the MMA thread: per group and half, GS/16
//              tcgen05.mma.kind::f16 with A from TMEM and the staged
//              activations (B, 8 token rows, 128-byte swizzled K-major shared
//              memory) into a 16-column TMEM accumulator, then a commit.
// The activations are rescaled per token by an exact power of two into the
// fp16 range and staged once per CTA, in the K order the unpacked pairs imply.
// When the tiles cannot fill the GPU, a cluster of up to 8 CTAs splits K and CTA
// rank 0 adds the partial results through distributed shared memory.  Every
// reduction has a fixed order (deterministic results), and every wait is bounded.
#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "internal.h"
#include "ptx.cuh"

namespace cg = cooperative_groups;

namespace gwb {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kRowThreads = 256;
constexpr int kThreads = 320;
constexpr int kTile = 128;
constexpr int kSMs = 148;
constexpr int kSmemBudget = 232448 - 8192;
constexpr int kStages = 4;
constexpr int kBoxBytes = kTile * 128;   // 128 rows x 128 bytes

__device__ __forceinline__ float bf16_val(uint16_t h) { return __uint_as_float(static_cast<uint32_t>(h) << 16); }

template <int BITS>
__host__ __device__ constexpr int lsig(int i) {
  return BITS == 4 ? (i & 1) * 4 : (BITS == 2 ? (i & 3) * 2 : 0);
}

// One word -> RPW fp16 pairs; pair i holds in-word positions i and i + RPW as
// 1024 + code * 2^lsig(i) (the code is OR-ed into the mantissa at its own bit offset).
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
struct TCfg {
  static constexpr int CPW = 32 / BITS;                 // codes per word
  static constexpr int RPW = CPW / 2;                   // fp16 pairs per word
  static constexpr int KS = 32 * CPW;                   // k per chunk (one 128-byte row segment)
  static constexpr int GPS = KS / GS;                   // groups per chunk
  static constexpr int GW = GS / CPW;                   // words per group
  static constexpr int AC = GS / 2;                     // TMEM columns of A per group
  static constexpr int NSLOT = (2 * 4 * (AC + 16) <= 512) ? 4 : 3;   // A/D slots per half
  static constexpr int LAG = NSLOT - 1;                 // groups between a group's MMA issue and its epilogue
  static constexpr int SROW = GPS * 2 < 4 ? 4 : GPS * 2;   // bytes of scales (or biases) per row per chunk
  static constexpr int SCALE_BYTES = 2 * 2 * kTile * SROW; // two halves x (scales, biases)
  static constexpr int STAGE = (2 * kBoxBytes + SCALE_BYTES + 1023) / 1024 * 1024;
  static constexpr uint32_t IDESC = make_idesc(1, 0, 128, 16);   // f32 <- f16 x f16, M=128, N=16
  static_assert(GW >= 1, "group narrower than a word");
};

struct TArgs {
  const uint16_t *x;
  const uint16_t *scales, *biases;
  uint16_t *y;
  int M, N, K, G;
  int NT;          // 128-row tiles
  int NCH;         // chunks per half per tile (this CTA's K-slice holds 2*NCH chunks)
  int scale16;     // scale rows and chunk offsets are 16-byte aligned
};

template <int BITS, int GS, int MP>
__global__ void __launch_bounds__(kThreads, 1)
    k_gemv_tmem(const __grid_constant__ CUtensorMap tm_w, const TArgs a) {
  using C = TCfg<BITS, GS>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  __shared__ float red[10 * 8], s_scale[8], s_inv[8];
  __shared__ uint32_t tmem_slot;
  __shared__ uint64_t bar_full[kStages], bar_empty[kStages], bar_aready[2][C::NSLOT], bar_dready[2][C::NSLOT];
  __shared__ uint64_t bar_part_full, bar_part_free;   // half 1 -> half 0 hand-over of a tile's partial sums
  __shared__ volatile int abort_flag;
  unsigned char *base = align_smem_1024(smem_raw);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = gridDim.y;
  const int NCH = a.NCH;
  const int KR = 2 * NCH * C::KS;                 // this CTA's K-slice
  const int GR = KR / GS;
  const int k0 = blockIdx.y * KR;
  const int natoms = KR / 64 + 1;                 // B: one 8-row x 128-byte atom per 64 k, plus a pad atom
  unsigned char *stages = base;
  unsigned char *Bsm = base + kStages * C::STAGE;
  float *XS = reinterpret_cast<float *>(Bsm + natoms * 1024);    // [GR][16]: X[8], XN[8]
  float *SB = XS + GR * 16;                                       // [NSLOT][256 threads][2]: s, b ring
  float *PART = SB + C::NSLOT * kRowThreads * 2;                  // [128 rows][MP]: half 1 -> half 0
  float *OUT = PART + kTile * MP;                                 // split-K: [128 rows][MP]

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; s++) {
      mbar_init(&bar_full[s], 1 + 32);   // producer arrive.expect_tx + 32 cp.async arrivals
      mbar_init(&bar_empty[s], 8);       // one arrive per row warp
    }
    for (int b = 0; b < 2; b++)
      for (int s = 0; s < C::NSLOT; s++) {
        mbar_init(&bar_aready[b][s], 4);
        mbar_init(&bar_dready[b][s], 1);
      }
    mbar_init(&bar_part_full, 4);
    mbar_init(&bar_part_free, 4);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(&tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;

  // tiles of this CTA: t = blockIdx.x, + gridDim.x, ...
  int ntiles = 0;
  for (int t = blockIdx.x; t < a.NT; t += gridDim.x) ntiles++;
  const int steps = ntiles * NCH;                 // stages consumed by each half

  // ---------------------------------------------------------------- producer step i (warp 8)
  // Loads stage i % kStages with chunk `ch` of both halves of tile `pt`.
  int pt = blockIdx.x, pch = 0;
  auto produce = [&](int i) -> bool {
    const int st = i % kStages;
    if (i >= kStages && !mbar_wait(&bar_empty[st], ((i / kStages) - 1) & 1)) return false;
    unsigned char *sp = stages + st * C::STAGE;
    if (lane == 0) {
      mbar_arrive_expect_tx(&bar_full[st], 2 * kBoxBytes);
      for (int h = 0; h < 2; h++) {
        const int kc = k0 + (h * NCH + pch) * C::KS;
        tma_load_2d(sp + h * kBoxBytes, &tm_w, kc / C::CPW, pt * kTile, &bar_full[st]);
      }
    }
    // scales / biases: each lane covers 16 (half, array, row) entries
    for (int e = lane; e < 2 * 2 * kTile; e += 32) {
      const int h = e / (2 * kTile), arr = (e / kTile) & 1, r = e % kTile;
      const int row = pt * kTile + r;
      const int g0 = ((k0 + (h * NCH + pch) * C::KS) / GS) & ~1;
      unsigned char *dst = sp + 2 * kBoxBytes + ((h * 2 + arr) * kTile + r) * C::SROW;
      const bool rok = row < a.N;
      const uint16_t *src = (arr ? a.biases : a.scales) + (int64_t)(rok ? row : 0) * a.G;
      if (a.scale16 && (C::SROW % 16) == 0) {
#pragma unroll
        for (int q = 0; q < C::SROW / 16; q++) {
          const int g = g0 + q * 8;
          const uint32_t nb = (rok && g < a.G) ? 16u : 0u;
          cp_async_16(dst + q * 16, src + (nb ? g : 0), nb);
        }
      } else {
#pragma unroll
        for (int q = 0; q < C::SROW / 4; q++) {
          const int g = g0 + q * 2;
          const uint32_t nb = (rok && g < a.G) ? 4u : 0u;
          cp_async_4(dst + q * 4, src + (nb ? g : 0), nb);
        }
      }
    }
    cp_async_arrive_noinc(&bar_full[st]);
    if (++pch == NCH) { pch = 0; pt += gridDim.x; }
    return true;
  };
  const int prefetch = steps < kStages ? steps : kStages;
  if (warp == 8)
    for (int i = 0; i < prefetch; i++) produce(i);   // weights do not depend on x: load them first

  // ---------------------------------------------------------------- activations (all threads)
  for (int t = 0; t < a.M; t++) {
    float m = 0.0f;
    for (int k = threadIdx.x; k < KR; k += kThreads)
      if (k0 + k < a.K) m = fmaxf(m, fabsf(bf16_val(a.x[(int64_t)t * a.K + k0 + k])));
    for (int off = 16; off; off >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, off));
    if (lane == 0) red[warp * 8 + t] = m;
  }
  __syncthreads();
  if (threadIdx.x < 8) {
    const int t = threadIdx.x;
    float m = 0.0f;
    if (t < a.M)
      for (int w = 0; w < kThreads / 32; w++) m = fmaxf(m, red[w * 8 + t]);
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
  auto x16 = [&](int t, int kk, int ls) -> uint16_t {   // fp16 bits of x[t, k0+kk] * 2^e / 2^ls (0 if absent)
    const int k = k0 + kk;
    if (t >= a.M || k >= a.K) return 0;
    return __half_as_ushort(__float2half_rn(bf16_val(a.x[(int64_t)t * a.K + k]) * s_scale[t] * pow2f(-ls)));
  };
  // B: element (token t, slice-k kb) in K-major 128-byte-swizzled atoms of 8 rows x 64 k
  for (int e = threadIdx.x; e < natoms * 8 * 64; e += kThreads) {
    const int kk = e % 64, t = (e / 64) % 8, at = e / 512;
    const int kb = at * 64 + kk;
    uint16_t v = 0;
    if (kb < KR && t < a.M) {
      const int gk = kb / GS, kap = kb % GS;            // group within slice, MMA k within group
      const int col = kap >> 1, h = kap & 1;            // A column and half
      const int wv = col / C::RPW, i = col % C::RPW;    // word, pair
      const int phys = wv * C::CPW + i + h * C::RPW;
      v = x16(t, gk * GS + phys, lsig<BITS>(i));
    }
    *reinterpret_cast<uint16_t *>(Bsm + at * 1024 + t * 128 + ((((kk >> 3) ^ t) & 7) << 4) + (kk & 7) * 2) = v;
  }
  for (int e = threadIdx.x; e < GR * 16; e += blockDim.x) XS[e] = 0.0f;   // absent tokens stay 0
  __syncthreads();
  for (int e = warp; e < GR * a.M; e += kThreads / 32) {   // X and XN per (group, present token)
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
  fence_proxy_async_smem();   // B is read by the tensor core (async proxy)
  __syncthreads();

  const int groups = steps * C::GPS;              // groups per half
  if (warp == 8) {
    // ---------------------------------------------------------------- producer (rest of the steps)
    int i = prefetch;
    for (; i < steps; i++)
      if (abort_flag || !produce(i)) { abort_flag = 1; break; }
    // drain: every issued load must land before the CTA may exit
    for (int d = (i - kStages > 0 ? i - kStages : 0); d < i; d++) mbar_wait(&bar_full[d % kStages], (d / kStages) & 1);
  } else if (warp == 9) {
    // ---------------------------------------------------------------- MMA thread
    if (lane == 0) {
      const uint32_t b_base = smem_u32(Bsm);
      int ch = 0, j = 0, issued = 0;
      for (int g = 0; g < groups; g++) {
        const int slot = g % C::NSLOT;
        const uint32_t ph = (g / C::NSLOT) & 1;
        for (int h = 0; h < 2; h++) {
          if (abort_flag || !mbar_wait(&bar_aready[h][slot], ph)) { abort_flag = 1; break; }
          tc_fence_after();
          const int kb0 = ((h * NCH + ch) * C::KS) + j * GS;     // slice-k of this group
          const uint32_t acol = (uint32_t)((h * C::NSLOT + slot) * C::AC);
          const uint32_t dcol = (uint32_t)(2 * C::NSLOT * C::AC + (h * C::NSLOT + slot) * 16);
#pragma unroll
          for (int m = 0; m < GS / 16; m++) {
            const int kb = kb0 + 16 * m;
            const uint64_t bd = smem_desc_sw128(b_base + (kb >> 6) * 1024 + (kb & 63) * 2);
            umma_f16_ts(tmem + dcol, tmem + acol + 8 * m, bd, C::IDESC, m != 0);
          }
          umma_commit(&bar_dready[h][slot]);
        }
        if (abort_flag) break;
        if (++j == C::GPS) { j = 0; if (++ch == NCH) ch = 0; }
        issued = g + 1;
      }
      // drain: the last commits must have arrived before the CTA may exit
      for (int d = (issued - C::NSLOT > 0 ? issued - C::NSLOT : 0); d < issued; d++)
        for (int hh = 0; hh < 2; hh++) mbar_wait(&bar_dready[hh][d % C::NSLOT], (d / C::NSLOT) & 1);
    }
  } else if (warp < 8) {
    // ---------------------------------------------------------------- row threads
    const int h = warp >> 2, q = warp & 3;
    const int r = 32 * q + lane;                  // row within the tile (TMEM lane)
    const uint32_t lane_addr = (uint32_t)(32 * q) << 16;
    const int tid = threadIdx.x;                  // 0..255
    float acc[MP];
#pragma unroll
    for (int t = 0; t < MP; t++) acc[t] = 0.f;
    int tile = blockIdx.x;
    int eg = 0, e_ch = 0, e_j = 0;                // epilogue position (group counter, chunk, group in chunk)
    int tiles_done = 0;
    // epilogue of group eg: wait for its accumulator, apply scale / bias, and at
    // the end of a tile combine the halves and write the result
    auto epilogue = [&]() -> bool {
      const int slot = eg % C::NSLOT;
      if (!mbar_wait(&bar_dready[h][slot], (eg / C::NSLOT) & 1)) return false;
      tc_fence_after();
      uint32_t v[MP];
      tmem_ld<MP>(tmem + lane_addr + (uint32_t)(2 * C::NSLOT * C::AC + (h * C::NSLOT + slot) * 16), v);
      tmem_ld_wait();
      const float2 sbv = *reinterpret_cast<const float2 *>(SB + (slot * kRowThreads + tid) * 2);
      const int gk = (h * NCH + e_ch) * C::GPS + e_j;           // group within the slice
#pragma unroll
      for (int t = 0; t < MP; t++)
        acc[t] = fmaf(sbv.x, __uint_as_float(v[t]) + XS[gk * 16 + 8 + t], fmaf(sbv.y, XS[gk * 16 + t], acc[t]));
      eg++;
      if (++e_j == C::GPS) {
        e_j = 0;
        if (++e_ch == NCH) {                                     // tile finished for this half
          e_ch = 0;
          // half 1 hands its partial sums to half 0 through PART (bounded waits)
          const uint32_t tp = (uint32_t)(tiles_done & 1);
          if (h == 1) {
            if (tiles_done > 0 && !mbar_wait(&bar_part_free, tp ^ 1)) return false;
#pragma unroll
            for (int t = 0; t < MP; t++) PART[r * MP + t] = acc[t];
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar_part_full);
          } else {
            if (!mbar_wait(&bar_part_full, tp)) return false;
            const int row = tile * kTile + r;
#pragma unroll
            for (int t = 0; t < MP; t++) {
              const float v2 = (acc[t] + PART[r * MP + t]) * s_inv[t];
              if (S == 1) {
                if (t < a.M && row < a.N) a.y[(int64_t)t * a.N + row] = __bfloat16_as_ushort(__float2bfloat16_rn(v2));
              } else {
                OUT[r * MP + t] = v2;
              }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar_part_free);
          }
#pragma unroll
          for (int t = 0; t < MP; t++) acc[t] = 0.f;
          tile += gridDim.x;
          tiles_done++;
        }
      }
      return true;
    };

    int g = 0;
    bool ok = true;
    for (int i = 0; i < steps && ok; i++) {
      const int st = i % kStages;
      if (!mbar_wait(&bar_full[st], (i / kStages) & 1)) { ok = false; break; }
      const unsigned char *sp = stages + st * C::STAGE;
      // this row's 128 bytes of packed words (swizzled 16-byte chunks) and its scales / biases
      uint32_t wds[32];
      const unsigned char *rowp = sp + h * kBoxBytes + r * 128;
#pragma unroll
      for (int c = 0; c < 8; c++) {
        const uint4 v = *reinterpret_cast<const uint4 *>(rowp + ((c ^ (r & 7)) << 4));
        wds[4 * c] = v.x; wds[4 * c + 1] = v.y; wds[4 * c + 2] = v.z; wds[4 * c + 3] = v.w;
      }
      const uint16_t *scp = reinterpret_cast<const uint16_t *>(sp + 2 * kBoxBytes + (h * 2 * kTile + r) * C::SROW);
      const uint16_t *bip = scp + kTile * (C::SROW / 2);
      const int goff = (C::GPS == 1) ? ((((k0 + (h * NCH + (i % NCH)) * C::KS) / GS) & 1)) : 0;
      float sv[C::GPS], bv[C::GPS];
#pragma unroll
      for (int j = 0; j < C::GPS; j++) {
        sv[j] = bf16_val(scp[goff + j]);
        bv[j] = bf16_val(bip[goff + j]);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_empty[st]);
#pragma unroll
      for (int j = 0; j < C::GPS; j++) {
        const int slot = g % C::NSLOT;
        uint32_t ra[C::AC];
#pragma unroll
        for (int v = 0; v < C::GW; v++) unpack_word<BITS>(wds[j * C::GW + v], ra + v * C::RPW);
        tmem_st<C::AC>(tmem + lane_addr + (uint32_t)((h * C::NSLOT + slot) * C::AC), ra);
        *reinterpret_cast<float2 *>(SB + (slot * kRowThreads + tid) * 2) = make_float2(sv[j], bv[j]);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar_aready[h][slot]);
        g++;
        if (g > C::LAG) {
          if (!epilogue()) { ok = false; break; }
        }
      }
    }
    while (ok && eg < g) {
      if (!epilogue()) ok = false;
    }
    if (!ok) abort_flag = 1;
  }

  // ---------------------------------------------------------------- split-K reduction over the cluster
  if (S > 1) {
    cg::cluster_group cluster = cg::this_cluster();
    cluster.sync();
    if (cluster.block_rank() == 0 && threadIdx.x < kTile) {
      const int r = threadIdx.x, row = blockIdx.x * kTile + r;
      for (int t = 0; t < MP; t++) {
        float s = 0.f;
        for (int qq = 0; qq < S; qq++) s += cluster.map_shared_rank(OUT, qq)[r * MP + t];
        if (t < a.M && row < a.N) a.y[(int64_t)t * a.N + row] = __bfloat16_as_ushort(__float2bfloat16_rn(s));
      }
    }
    cluster.sync();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
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

template <int BITS, int GS, int MP>
gwb_status run_tmem(const uint16_t *x, int M, const uint32_t *wq, const uint16_t *scales, const uint16_t *biases,
                    int64_t N, int64_t K, uint16_t *y, cudaStream_t st) {
  using C = TCfg<BITS, GS>;
  const int G = (int)(K / GS);
  if (G % 2 != 0) return GWB_ERR_UNSUPPORTED;                 // scales copied in 4-byte pieces
  if ((K * BITS / 8) % 16 != 0) return GWB_ERR_UNSUPPORTED;    // TMA row stride
  const int nc_total = (int)((K + C::KS - 1) / C::KS);
  if (nc_total % 2 != 0) return GWB_ERR_UNSUPPORTED;          // two halves of equal length
  const int NT = (int)((N + kTile - 1) / kTile);
  // split K over a cluster only when the tiles cannot fill the GPU
  int S = 1;
  while (S < 8 && NT * 2 * S <= kSMs && nc_total % (4 * S) == 0) S *= 2;
  const int NCH = nc_total / (2 * S);
  const int KR = 2 * NCH * C::KS;
  const size_t smem = 1024 + (size_t)kStages * C::STAGE + (size_t)(KR / 64 + 1) * 1024 + (size_t)(KR / GS) * 16 * 4 +
                      (size_t)C::NSLOT * kRowThreads * 2 * 4 + (size_t)2 * kTile * MP * 4;
  if (smem > (size_t)kSmemBudget) return GWB_ERR_UNSUPPORTED;
  const int P = S > 1 ? NT : (NT < kSMs ? NT : kSMs);

  auto fn = encode_fn();
  if (!fn) return fail(GWB_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  CUtensorMap tm;
  const uint64_t words = (uint64_t)K / C::CPW;
  const cuuint64_t dims[2] = {words, (cuuint64_t)N};
  const cuuint64_t strides[1] = {words * 4};
  const cuuint32_t box[2] = {32, (cuuint32_t)kTile};
  const cuuint32_t es[2] = {1, 1};
  CUresult r = fn(&tm, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t *>(wq), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(GWB_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);

  TArgs a{};
  a.x = x; a.scales = scales; a.biases = biases; a.y = y;
  a.M = M; a.N = (int)N; a.K = (int)K; a.G = G;
  a.NT = NT; a.NCH = NCH;
  a.scale16 = (G % 8 == 0) ? 1 : 0;

  auto kern = k_gemv_tmem<BITS, GS, MP>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return fail(GWB_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
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
  e = cudaLaunchKernelEx(&cfg, kern, tm, a);
  if (e != cudaSuccess) return fail(GWB_ERR_CUDA, "TMEM GEMV launch: %s", cudaGetErrorString(e));
  return GWB_OK;
}

int pad_tokens(int M) { return M <= 1 ? 1 : (M <= 2 ? 2 : (M <= 4 ? 4 : 8)); }

}  // namespace

gwb_status launch_gemv_tmem(const uint16_t *x, int M, const uint32_t *wq, const uint16_t *scales,
                            const uint16_t *biases, int64_t N, int64_t K, int bits, int gs, uint16_t *y,
                            cudaStream_t st) {
  const int MP = pad_tokens(M);
#define GWB_GT(B, S, P) \
  if (bits == B && gs == S && MP == P) return run_tmem<B, S, P>(x, M, wq, scales, biases, N, K, y, st);
#define GWB_GT_MP(B, S) GWB_GT(B, S, 1) GWB_GT(B, S, 2) GWB_GT(B, S, 4) GWB_GT(B, S, 8)
  GWB_GT_MP(2, 64) GWB_GT_MP(2, 128)
  GWB_GT_MP(4, 32) GWB_GT_MP(4, 64) GWB_GT_MP(4, 128)
  GWB_GT_MP(8, 32) GWB_GT_MP(8, 64) GWB_GT_MP(8, 128)
#undef GWB_GT_MP
#undef GWB_GT
  return GWB_ERR_UNSUPPORTED;
}

gwb_status read_and_clear_device_error_tmem(cudaStream_t st, unsigned int *flag) {
  unsigned int zero = 0;
  cudaError_t e = cudaStreamSynchronize(st);
  if (e == cudaSuccess) e = cudaMemcpyFromSymbol(flag, g_device_error, sizeof(unsigned int));
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof(unsigned int));
  if (e != cudaSuccess) return fail(GWB_ERR_CUDA, "device error check: %s", cudaGetErrorString(e));
  return GWB_OK;
}

}  // namespace gwb
