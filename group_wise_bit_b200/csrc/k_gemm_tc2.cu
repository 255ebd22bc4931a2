// Persistent tensor-core (tcgen05) GEMM for the prefill regime (M >= 128) of
// the fused dequant + matmul, for the MLX affine layout (bf16, kind::f16), the
// GPTQ layout without g_idx (fp16, kind::f16) and W4A8 (int8, kind::i8).
//
// As in the per-tile kernel the product is computed transposed ("swap AB"):
// the tensor core's M side is 128 output features, its N side BT tokens.  Each
// CTA (one per SM) walks a static list of 128 x BT output tiles (features
// fastest, so the CTAs in flight share one activation tile through L2), and
// its warps form a pipeline of three decoupled shared-memory rings:
//
//   warp 0      TMA producer of the activation ring X (BT x BK, 128-byte
//               swizzle, zero-filled past M and K);
//   warp 2      producer of the packed-weight ring R: lane 0 issues the TMA
//               tile load of the step's packed words, all lanes copy the
//               step's group scales / biases (GPTQ: scales and qzeros) with
//               cp.async onto the same mbarrier;
//   warps 3-10  dequantizers: R stage -> the 128 x BK A operand (bf16, fp16 or
//               int8) in the 128-byte-swizzled K-major layout, into ring A;
//               the R ring is deeper than X and A, so the dequantizers run
//               ahead of the tensor core instead of waiting for each load;
//   warp 1      TMEM allocation and the single MMA-issuing thread: per K step
//               BK/16 (int8: BK/32) tcgen05.mma into one of two TMEM
//               accumulators, then commits the X and A slots back;
//   warps 11-14 epilogue: drain the finished accumulator with tcgen05.ld and
//               write the output tile while the next tile accumulates in the
//               other TMEM buffer.
//
// With PAIR = 2 two CTAs of a cluster share one 256 x BT tile through the
// tensor core's two-SM mode (tcgen05 cta_group::2): each CTA dequantizes its
// own 128 feature rows (its half of A) and loads half of the BT tokens (its
// half of B), so every SM moves half the activation bytes per flop.  The
// leader CTA (rank 0) issues the MMAs; its barriers collect both CTAs' TMA
// bytes and dequantizer arrivals, and its commits release the slots of both.
//
// Every mbarrier wait is bounded (ptx.cuh); on a timeout the CTA stops issuing
// work, drains what it issued, frees its TMEM and exits.
#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <map>
#include <mutex>
#include <utility>

#include "dequant.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace cg = cooperative_groups;

namespace gwb {
namespace {
using namespace dq;

// ---------------------------------------------------------------- two-SM helpers
__device__ __forceinline__ uint32_t cta_rank_in_cluster() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// shared::cluster address of the same shared-memory location in CTA `rank`
__device__ __forceinline__ uint32_t map_rank(const void *p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}
// Arrive on a barrier of either CTA of the pair (release at CTA scope: the data
// it publishes, a dequantized A half, is read by this CTA's own tensor core).
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// TMA tile load into this CTA's shared memory whose bytes complete on a barrier
// of either CTA of the pair (cluster address).
__device__ __forceinline__ void tma_load_2d_pair(void *dst, const CUtensorMap *map, int32_t x, int32_t y,
                                                 uint32_t bar_cluster_addr) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar_cluster_addr)
      : "memory");
}
__device__ __forceinline__ void umma_f16_pair(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
__device__ __forceinline__ void umma_i8_pair(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
// 3-D tile load (x, y, z = 0 .. box) into this CTA's shared memory.
__device__ __forceinline__ void tma_load_3d_sb(void *dst, const CUtensorMap *map, int32_t x, int32_t y, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(0), "r"(smem_u32(bar))
      : "memory");
}
// An epoch no launch takes (launch epochs run from 1 to 0x7ffffffe): a head CTA
// told to wait for it gives up (tests of the bounded-wait failure path).
constexpr uint32_t kNeverEpoch = 0xffffffffu;

// Stream-K handshake on a global word: publish (release) the epoch once this
// CTA's partial is stored; wait (acquire, bounded) until a peer published it.
__device__ __forceinline__ void flag_publish(uint32_t *f, uint32_t epoch) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(f), "r"(epoch) : "memory");
}
__device__ __forceinline__ bool flag_wait(const uint32_t *f, uint32_t epoch) {
  const unsigned long long limit = g_wait_cycles;
  const unsigned long long t0 = clock64();
  while (true) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(f) : "memory");
    if (v == epoch) return true;
    if (clock64() - t0 > limit) {
      atomicOr(&g_device_error, 1u);
      return false;
    }
    __nanosleep(64);
  }
}
// Same, with A read from tensor memory (each CTA's TMEM holds its 128 rows).
__device__ __forceinline__ void umma_f16_ts_pair(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t idesc,
                                                 uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
__device__ __forceinline__ void umma_i8_ts_pair(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t idesc,
                                                uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
// Arrive once on the barrier at this offset in both CTAs of the pair when the
// pair's MMAs issued so far complete.
__device__ __forceinline__ void umma_commit_pair(uint64_t *bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"((uint16_t)3)
      : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t *dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

constexpr int kWarps = 15;
constexpr int kThreads = kWarps * 32;
constexpr int kDqWarps = 8;
constexpr int kDqGroupWarps = kDqWarps / 2;   // dequantizer warps per K step (two groups alternate)
constexpr int kFirstDq = 3, kFirstEpi = 11;
constexpr int kTileN = 128;      // output features per tile (tensor-core M)
constexpr int kMaxSmem = 232448;
constexpr int kSMs = 148;
constexpr bool kAInTmem = true;   // pairs keep the dequantized A operand in tensor memory

// Affine / Gptq: 16-bit activations x dequantized weights; I8: int8
// activations x int4 codes; W8: int8 activations x int8 weights, which need no
// dequantization and go by TMA straight into the A stages.
enum class Fmt { Affine, Gptq, I8, W8, F16 };

struct Args {
  int M, N, K, gs;
  int gs_log2;              // group size = 1 << gs_log2
  int sc_tma;               // affine: scales + biases arrive by TMA as [2 arrays][128 rows][8 groups]
  int sc_swap;              //   ... with the biases first (they sit below the scales in memory)
  int zadd;                 // gptq: added to the stored zero (1: GPTQ's convention, 0: AWQ's)
  int Nt, Mt, T;            // feature tiles, token tiles, tiles (token tiles fastest)
  int dpw;                  // stream-K: whole waves walked round robin before the split tail
  const uint16_t *scales;   // affine: bf16 [N, K/gs];   gptq: fp16 [K/gs, N]
  const uint16_t *biases;   // affine: bf16 [N, K/gs]
  const int32_t *qzeros;    // gptq: [K/gs, N/8]
  const float *sx, *sw;     // i8: per-token / per-channel scales
  uint16_t *y;              // bf16 (affine, i8) or fp16 (gptq) [M, N]
  int32_t *acc;             // i8: optional int32 [M, N]
  // stream-K: partial tiles through a workspace (null: whole tiles per unit)
  uint32_t *ws;             // [CTAs][BT tokens][128 rows] fp32 (i8: s32) partial accumulators
  uint32_t *flags;          // [CTAs] epoch at which the CTA's partial is complete
  uint32_t *ctr;            // [2]: launches so far (the epoch counter), CTAs finished in this launch
  int stall;                // a test made this launch's heads wait for an epoch nobody publishes
};

// A unit's work, walked as segments of one tile each: first whole tiles taken
// round robin (unit, unit + units, ...: the units running at one time work on
// consecutive tiles, which share their feature tile's weights and the token
// tiles' activations through L2), then, with a workspace, an equal contiguous
// share of the flattened (tile, K step) space of the remaining tiles (stream-K:
// a tile may be split between units).  Without a workspace all tiles are whole.
struct SegWalk {
  int64_t L, Le;
  int nk, dp_t, dp_left, step;
  __device__ SegWalk(const Args &a, int nk_, int unit, int units) : nk(nk_), dp_t(unit), step(units) {
    if (a.ws) {
      dp_left = a.dpw;
      const int64_t T0 = (int64_t)a.dpw * units * nk_, W = (int64_t)a.T * nk_ - T0;
      L = T0 + (int64_t)unit * W / units;
      Le = T0 + (int64_t)(unit + 1) * W / units;
    } else {
      dp_left = unit < a.T ? (a.T - 1 - unit) / units + 1 : 0;
      L = Le = 0;
    }
  }
  __device__ bool next(int &t, int &k0, int &k1) {
    if (dp_left > 0) {
      t = dp_t;
      dp_t += step;
      dp_left--;
      k0 = 0;
      k1 = nk;
      return true;
    }
    if (L >= Le) return false;
    t = (int)(L / nk);
    k0 = (int)(L - (int64_t)t * nk);
    k1 = (Le - L) < (int64_t)(nk - k0) ? k0 + (int)(Le - L) : nk;
    L += k1 - k0;
    return true;
  }
};

template <Fmt F, int BITS>
struct Tr;
template <int BITS>
struct Tr<Fmt::Affine, BITS> {
  static constexpr int BK = 64;                       // 64 bf16 = 128 bytes per row
  static constexpr int RAW = kTileN * BK * BITS / 8;  // packed words of a step
  static constexpr int SC = 4096;                     // scales + biases: 2 x 128 rows x 8 groups (or a pair by cp.async)
  static constexpr int NMMA = BK / 16;
  static constexpr int CP = 32;                       // cp.async arrivals per step (when not by TMA)
};
template <>
struct Tr<Fmt::Gptq, 4> {
  static constexpr int BK = 64;
  static constexpr int RAW = (BK / 8) * kTileN * 4;
  static constexpr int SC = 1024;                     // 2 groups x (128 fp16 scales + 16 qzeros words)
  static constexpr int NMMA = BK / 16;
  static constexpr int CP = 32;
};
template <>
struct Tr<Fmt::W8, 8> {
  static constexpr int BK = 128;
  static constexpr int RAW = 0;
  static constexpr int SC = 0;
  static constexpr int NMMA = BK / 32;
  static constexpr int CP = 0;
};
template <>
struct Tr<Fmt::F16, 16> {                             // dense fp16 weights (act-order GPTQ, dequantized first)
  static constexpr int BK = 64;
  static constexpr int RAW = 0;
  static constexpr int SC = 0;
  static constexpr int NMMA = BK / 16;
  static constexpr int CP = 0;
};
template <>
struct Tr<Fmt::I8, 4> {
  static constexpr int BK = 128;                      // 128 int8 = 128 bytes per row
  static constexpr int RAW = kTileN * BK / 2;
  static constexpr int SC = 0;
  static constexpr int NMMA = BK / 32;
  static constexpr int CP = 0;
};

// Ring depths.  A CTA pair holds half the tokens per CTA, which leaves room for
// 6 dequantized slots (the dequantizers then run well ahead of the tensor core)
// next to 4 activation slots; a single CTA keeps 3 A slots and fits as many
// activation slots as it can.  The packed-weight ring takes what is left, up to 8.
// With ATM the dequantized A stages live in tensor memory (8 slots of 32
// columns next to one 256-column accumulator) and take no shared memory.
// W8 and F16 (weights that need no dequantization) have no packed-weight ring:
// activation and weight stages go in lockstep, as many of each as fit (up to 8).
template <Fmt F, int BITS, int BT, int PAIR, bool ATM>
struct Plan2 {
  static constexpr bool W8 = F == Fmt::W8 || F == Fmt::F16;   // the weight tile goes straight to the A stage
  static constexpr int XB = BT / PAIR * 128;
  static constexpr int AB = kTileN * 128;
  static constexpr int RB = (Tr<F, BITS>::RAW + Tr<F, BITS>::SC + 127) / 128 * 128;
  // ATM: a bf16 staging tile [BT tokens][128 rows] for the epilogue, so that it
  // frees the single accumulator before writing the output
  // The epilogue's staging: ATM, a whole bf16 tile (so that it frees the single
  // accumulator before writing); otherwise the chunked staging of 32-token chunks
  // (two 32-bit partial chunks and one 16-bit output chunk, 40 KB)
  static constexpr int EPI = ATM ? BT * kTileN * 2 : 2 * 32 * kTileN * 4 + 32 * kTileN * 2;
  static constexpr int BUDGET = kMaxSmem - 1024 - 1024 - 1024;   // alignment, barriers, static
  static constexpr int SW8 = (BUDGET - EPI) / (XB + AB) > 8 ? 8 : (BUDGET - EPI) / (XB + AB);
  static constexpr int SA = ATM ? 8 : W8 ? SW8 : (PAIR == 2 ? 6 : 3);
  static constexpr int A_SMEM = ATM ? 0 : SA * AB;
  static constexpr int SXF = (BUDGET - A_SMEM - EPI - 4 * RB) / XB > 6 ? 6 : (BUDGET - A_SMEM - EPI - 4 * RB) / XB;
  static constexpr int SX = W8 ? SW8 : PAIR == 2 && !ATM && SXF > 4 ? 4 : SXF;
  static constexpr int SR0 = RB ? (BUDGET - A_SMEM - EPI - SX * XB) / RB : 0;
  static constexpr int SR = W8 ? 0 : SR0 > 8 ? 8 : SR0;
  static constexpr int SMEM = SX * XB + A_SMEM + EPI + SR * RB + 1024 + 1024;
  static_assert(SX >= 2 && (W8 || SR >= 4), "shared memory too small");
  static_assert(!(W8 && ATM), "dense weights are read from shared memory");
};

__device__ __forceinline__ void put4(uint32_t (&o)[16], int j, uint4 v) {
  o[4 * j] = v.x; o[4 * j + 1] = v.y; o[4 * j + 2] = v.z; o[4 * j + 3] = v.w;
}

// Affine with scales by TMA: the 8-group block of scales and biases travels
// only with the first two steps of a segment and of each new block (every 8
// groups: 4 to 16 steps), one for each dequantizer group (they take alternate
// steps); the dequantizers keep their row's block in registers.
__device__ __forceinline__ bool affine_box_step(int k, int k0, int gs_log2) {
  constexpr int BK = Tr<Fmt::Affine, 4>::BK;
  return k - k0 < 2 || ((k * BK) & ((8 << gs_log2) - 1)) < 2 * BK;
}

// Dequantizes K step `k` (row r, half h of the step) from the R stage into the
// 16 words of A the thread owns: o[4j .. 4j+3] = 16-byte chunk 4h + j of row r
// (k = 8 (4h + j) .. +7 for 16-bit operands, 16 (4h + j) .. +15 for int8).
// sbv: affine with scales by TMA, the row's block of 8 scales and 8 biases.
template <Fmt F, int BITS>
__device__ __forceinline__ void dequant_words(const Args &a, int k, int r, int h, const unsigned char *R,
                                              const uint4 (&sbv)[2], uint32_t (&o)[16]) {
  using T = Tr<F, BITS>;
  constexpr int BK = T::BK;
  const int kh = k * BK + h * (BK / 2);    // first k of this thread's half step
  if constexpr (F == Fmt::Affine) {
    float sf, bfv;
    if (a.sc_tma) {
      // the half step's group within the row's block of 8 groups
      const int g8 = (kh >> a.gs_log2) & 7;
      const uint4 vs = sbv[0], vb = sbv[1];
      const int wsel = g8 >> 1;
      const uint32_t ws = wsel == 0 ? vs.x : wsel == 1 ? vs.y : wsel == 2 ? vs.z : vs.w;
      const uint32_t wb = wsel == 0 ? vb.x : wsel == 1 ? vb.y : wsel == 2 ? vb.z : vb.w;
      sf = __uint_as_float((g8 & 1) ? (ws & 0xffff0000u) : (ws << 16));
      bfv = __uint_as_float((g8 & 1) ? (wb & 0xffff0000u) : (wb << 16));
    } else {
      int idx = (kh >> a.gs_log2) - (((k * BK) >> a.gs_log2) & ~1);   // group within the staged pair
      idx = idx < 1 ? idx : 1;
      const uint16_t *sc = reinterpret_cast<const uint16_t *>(R + T::RAW);
      sf = bf16_val(sc[r * 2 + idx]);
      bfv = bf16_val(sc[(kTileN + r) * 2 + idx]);
    }
    if constexpr (BITS == 4) {
      const uint4 raw = *reinterpret_cast<const uint4 *>(R + (r * 8 + h * 4) * 4);
      const __nv_bfloat162 s2b = __floats2bfloat162_rn(sf, sf), b2b = __floats2bfloat162_rn(bfv, bfv);
      const uint32_t wv[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
      for (int j = 0; j < 4; j++) put4(o, j, dq_affine4(wv[j], s2b, b2b));
    } else if constexpr (BITS == 2) {
      const uint2 raw = *reinterpret_cast<const uint2 *>(R + (r * 4 + h * 2) * 4);
      const __nv_bfloat162 s2q = __floats2bfloat162_rn(sf, sf * 0.25f), b2b = __floats2bfloat162_rn(bfv, bfv);
      uint4 c0, c1;
      dq_affine2(raw.x, s2q, b2b, c0, c1);
      put4(o, 0, c0);
      put4(o, 1, c1);
      dq_affine2(raw.y, s2q, b2b, c0, c1);
      put4(o, 2, c0);
      put4(o, 3, c1);
    } else {
      const uint4 *rp = reinterpret_cast<const uint4 *>(R + (r * 16 + h * 8) * 4);
      const uint4 ra = rp[0], rb = rp[1];
      put4(o, 0, dq_affine8(ra.x, ra.y, sf, bfv));
      put4(o, 1, dq_affine8(ra.z, ra.w, sf, bfv));
      put4(o, 2, dq_affine8(rb.x, rb.y, sf, bfv));
      put4(o, 3, dq_affine8(rb.z, rb.w, sf, bfv));
    }
  } else if constexpr (F == Fmt::Gptq) {
    int idx = (kh >> a.gs_log2) - ((k * BK) >> a.gs_log2);
    idx = idx < 1 ? idx : 1;
    const uint16_t *sc = reinterpret_cast<const uint16_t *>(R + T::RAW);
    const uint32_t *zc = reinterpret_cast<const uint32_t *>(R + T::RAW + 512);
    const uint32_t sv = sc[idx * kTileN + r];
    const uint32_t zv = 0x6400u | (((zc[idx * 16 + r / 8] >> ((r % 8) * 4)) & 0xFu) + (uint32_t)a.zadd);
    uint32_t s2[4], z2[4];
#pragma unroll
    for (int p = 0; p < 4; p++) { s2[p] = sv | (sv << 16); z2[p] = zv | (zv << 16); }
    const uint32_t *Rw = reinterpret_cast<const uint32_t *>(R);
#pragma unroll
    for (int j = 0; j < 4; j++) {
      const int kq = 4 * h + j;                  // k-octet within the step = chunk index
      put4(o, j, dq_gptq(Rw[kq * kTileN + r], z2, s2));
    }
  } else {
    const uint4 *rp = reinterpret_cast<const uint4 *>(R + (r * 16 + h * 8) * 4);
    const uint4 ra = rp[0], rb = rp[1];
    const uint32_t wv[8] = {ra.x, ra.y, ra.z, ra.w, rb.x, rb.y, rb.z, rb.w};
#pragma unroll
    for (int j = 0; j < 4; j++) {
      const uint2 lo = dq_i4(wv[2 * j]), hi = dq_i4(wv[2 * j + 1]);
      put4(o, j, make_uint4(lo.x, lo.y, hi.x, hi.y));
    }
  }
}

// The thread's 16 words of A into the 128-byte-swizzled shared-memory A stage.
__device__ __forceinline__ void store_a_smem(unsigned char *A, int r, int h, const uint32_t (&o)[16]) {
#pragma unroll
  for (int j = 0; j < 4; j++)
    *reinterpret_cast<uint4 *>(A + sw128_off(r, 4 * h + j)) = make_uint4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
}

template <Fmt F, int BITS, int BT, int PAIR, bool ATM>
__global__ void __launch_bounds__(kThreads, 1)
    k_tc2(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
          const __grid_constant__ CUtensorMap tm_sb, const Args a) {
  using T = Tr<F, BITS>;
  using P = Plan2<F, BITS, BT, PAIR, ATM>;
  constexpr int BK = T::BK;
  constexpr int SX = P::SX, SA = P::SA, SR = P::SR;
  constexpr int XT = BT / PAIR;                        // tokens of this CTA's activation slot
  // TMEM: two accumulators of BT fp32 / s32 columns, or (ATM) one accumulator
  // and SA A slots of 32 columns (64 bf16 or 128 int8 k per row)
  constexpr uint32_t NCOLS = ATM ? 512u : 2u * BT;
  constexpr int NACC = ATM ? 1 : 2;
  constexpr uint32_t ACOL = BT;                        // first A slot column (ATM)
  static_assert(!ATM || (PAIR == 2 && BT == 256), "A in tensor memory is laid out for 256-token pairs");
  constexpr bool kInt = F == Fmt::I8 || F == Fmt::W8;   // kind::i8, s32 accumulators
  constexpr bool kDense = F == Fmt::W8 || F == Fmt::F16;   // weights by TMA straight into the A stage
  constexpr bool kOutF16 = F == Fmt::Gptq || F == Fmt::F16;
  constexpr uint32_t IDESC = kInt ? make_idesc(2, 1, kTileN * PAIR, BT)
                             : kOutF16 ? make_idesc(1, 0, kTileN * PAIR, BT)
                                                : make_idesc(1, 1, kTileN * PAIR, BT);

  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char *base = align_smem_1024(smem_raw);
  unsigned char *ringX = base;
  unsigned char *ringA = ringX + SX * P::XB;
  unsigned char *ringR = ringA + P::A_SMEM;
  uint16_t *stage = reinterpret_cast<uint16_t *>(ringR + SR * P::RB);   // ATM epilogue staging
  uint64_t *xfull = reinterpret_cast<uint64_t *>(ringR + SR * P::RB + P::EPI);
  uint64_t *xempty = xfull + SX;
  uint64_t *afull = xempty + SX;
  uint64_t *aempty = afull + SA;
  uint64_t *rfull = aempty + SA;
  uint64_t *rempty = rfull + SR;
  uint64_t *accfull = rempty + SR;
  uint64_t *accempty = accfull + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(accempty + 2);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  uint32_t *epoch_slot = tmem_slot + 2;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nk = (a.K + BK - 1) / BK;
  // tile walk: this CTA's pair (or itself) and its rank within the pair
  const int rank = PAIR == 2 ? (int)cta_rank_in_cluster() : 0;
  const int unit = blockIdx.x / PAIR, units = gridDim.x / PAIR;
  const bool leader = rank == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < SX; s++) { mbar_init(&xfull[s], 1); mbar_init(&xempty[s], 1); }
    for (int s = 0; s < SA; s++) { mbar_init(&afull[s], kDense ? 1 : kDqGroupWarps * PAIR); mbar_init(&aempty[s], 1); }
    for (int s = 0; s < SR; s++) {
      mbar_init(&rfull[s], 1 + (F == Fmt::Affine && a.sc_tma ? 0 : T::CP));
      mbar_init(&rempty[s], kDqGroupWarps);
    }
    for (int b = 0; b < 2; b++) { mbar_init(&accfull[b], 1); mbar_init(&accempty[b], 4 * PAIR); }
    *abort_flag = 0;
    // stream-K: this launch's epoch, from the workspace's launch counter (so a CUDA
    // graph that replays the launch gets a fresh epoch every time); never 0, the
    // flags' initial value, nor kNeverEpoch
    *epoch_slot = a.ws ? *reinterpret_cast<volatile uint32_t *>(a.ctr) % 0x7ffffffeu + 1u : 0u;
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_w);
    if (F == Fmt::Affine && a.sc_tma) tma_prefetch_desc(&tm_sb);
    fence_mbar_init();
  }
  if (warp == 1) {
    if constexpr (PAIR == 2) {
      tmem_alloc_pair(tmem_slot, NCOLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, NCOLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR == 2) cg::this_cluster().sync();   // both CTAs' barriers exist before any remote use
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // the leader's copies of the barriers both CTAs report to
  const uint32_t lead_afull = PAIR == 2 ? map_rank(afull, 0) : 0u;
  const uint32_t lead_accempty = PAIR == 2 ? map_rank(accempty, 0) : 0u;
  const uint32_t lead_xfull = PAIR == 2 ? map_rank(xfull, 0) : 0u;

  if (warp == 0) {
    // ------------------------------------------------------------ X producer
    if (lane == 0) {
      int it = 0, t, k0, k1;
      bool ok = true;
      SegWalk sw(a, nk, unit, units);
      while (ok && sw.next(t, k0, k1)) {
        const int mx = (t % a.Mt) * BT + rank * XT;    // first token of this CTA's half
        for (int k = k0; k < k1; k++, it++) {
          const int s = it % SX;
          if (*abort_flag || !mbar_wait(&xempty[s], ((it / SX) & 1) ^ 1)) { *abort_flag = 1; ok = false; break; }
          if constexpr (PAIR == 2) {
            if (leader) mbar_arrive_expect_tx(&xfull[s], 2 * P::XB);
            tma_load_2d_pair(ringX + s * P::XB, &tm_x, k * BK, mx, lead_xfull + s * 8);
          } else {
            mbar_arrive_expect_tx(&xfull[s], P::XB);
            tma_load_2d(ringX + s * P::XB, &tm_x, k * BK, mx, &xfull[s]);
          }
        }
      }
      // every issued load lands before the CTA may exit (the leader sees both halves)
      if (leader)
        for (int i = it - SX < 0 ? 0 : it - SX; i < it; i++) mbar_wait(&xfull[i % SX], (i / SX) & 1);
    }
  } else if (warp == 2) {
    if constexpr (kDense) {
    // ------------------------------------------------------------ A producer (dense weights)
    // The weight tile [128 rows][128 bytes of k] lands in the A stage by one
    // swizzled TMA copy; with a pair, both CTAs' copies complete on the leader's barrier.
    if (lane == 0) {
      int it = 0, t, k0, k1;
      bool ok = true;
      SegWalk sw(a, nk, unit, units);
      while (ok && sw.next(t, k0, k1)) {
        const int n0 = (t / a.Mt) * kTileN * PAIR + rank * kTileN;
        for (int k = k0; k < k1; k++, it++) {
          const int s = it % SA;
          if (*abort_flag || !mbar_wait(&aempty[s], ((it / SA) & 1) ^ 1)) { *abort_flag = 1; ok = false; break; }
          if constexpr (PAIR == 2) {
            if (leader) mbar_arrive_expect_tx(&afull[s], 2 * P::AB);
            tma_load_2d_pair(ringA + s * P::AB, &tm_w, k * BK, n0, lead_afull + s * 8);
          } else {
            mbar_arrive_expect_tx(&afull[s], P::AB);
            tma_load_2d(ringA + s * P::AB, &tm_w, k * BK, n0, &afull[s]);
          }
        }
      }
      if (leader)
        for (int i = it - SA < 0 ? 0 : it - SA; i < it; i++) mbar_wait(&afull[i % SA], (i / SA) & 1);
    }
    } else {
    // ------------------------------------------------------------ R producer
    int it = 0, t, k0, k1;
    bool ok = true;
    SegWalk sw(a, nk, unit, units);
    while (ok && sw.next(t, k0, k1)) {
      const int n0 = (t / a.Mt) * kTileN * PAIR + rank * kTileN;
      for (int k = k0; k < k1; k++, it++) {
        const int s = it % SR;
        if (*abort_flag || !mbar_wait(&rempty[s], ((it / SR) & 1) ^ 1)) { *abort_flag = 1; ok = false; break; }
        unsigned char *st = ringR + s * P::RB;
        if (lane == 0) {
          const bool sct = F == Fmt::Affine && a.sc_tma && affine_box_step(k, k0, a.gs_log2);
          mbar_arrive_expect_tx(&rfull[s], T::RAW + (sct ? 4096 : 0));
          if constexpr (F == Fmt::Gptq) tma_load_2d(st, &tm_w, n0, k * (BK / 8), &rfull[s]);
          else if constexpr (F == Fmt::I8) tma_load_2d(st, &tm_w, k * (BK / 8), n0, &rfull[s]);
          else tma_load_2d(st, &tm_w, k * (BK * BITS / 32), n0, &rfull[s]);
          if (sct) tma_load_3d_sb(st + T::RAW, &tm_sb, ((k * BK) >> a.gs_log2) & ~7, n0, &rfull[s]);
        }
        unsigned char *sc = st + T::RAW;
        if constexpr (F == Fmt::Affine) {
          if (!a.sc_tma) {
          const int G = a.K / a.gs;
          const int gp = ((k * BK) >> a.gs_log2) & ~1;
          for (int e = lane; e < 2 * kTileN; e += 32) {   // (array, row) -> 4 bytes: groups gp, gp+1
            const int arr = e / kTileN, row = e % kTileN, n = n0 + row;
            const bool okc = n < a.N && gp < G;
            const uint16_t *src = (arr ? a.biases : a.scales) + (okc ? (int64_t)n * G + gp : 0);
            cp_async_4(sc + e * 4, src, okc ? 4u : 0u);
          }
          cp_async_arrive_noinc(&rfull[s]);
          }
        } else if constexpr (F == Fmt::Gptq) {
          const int G = a.K / a.gs;
          const int gp = (k * BK) >> a.gs_log2;
          {   // scales: 2 groups x 128 columns = 32 chunks of 16 bytes, one per lane
            const int gi = lane >> 4, ch = lane & 15, g = gp + gi, n = n0 + ch * 8;
            const bool okc = g < G && n < a.N;
            cp_async_16(sc + lane * 16, a.scales + (okc ? (int64_t)g * a.N + n : 0), okc ? 16u : 0u);
          }
          {   // qzeros: 2 groups x 16 words, one word per lane
            const int gi = lane >> 4, wz = lane & 15, g = gp + gi, n = n0 + wz * 8;
            const bool okc = g < G && n < a.N;
            cp_async_4(sc + 512 + lane * 4, a.qzeros + (okc ? (int64_t)g * (a.N / 8) + n / 8 : 0), okc ? 4u : 0u);
          }
          cp_async_arrive_noinc(&rfull[s]);
        }
      }
    }
    if (lane == 0)
      for (int i = it - SR < 0 ? 0 : it - SR; i < it; i++) mbar_wait(&rfull[i % SR], (i / SR) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (the leader's)
    if (lane == 0 && leader) {
      int xi = 0, tc = 0, t, k0, k1;
      // ring positions and phases, advanced without divisions; the operand
      // descriptors of a slot differ from slot 0's only in the start-address field
      // (16-byte units, shared-memory addresses stay below 2^18)
      int sx = 0, sa = 0;
      uint32_t px = 0, pa = 0;
      const uint64_t xdesc0 = smem_desc_sw128(smem_u32(ringX)), adesc0 = smem_desc_sw128(smem_u32(ringA));
      bool ok = true;
      SegWalk sw(a, nk, unit, units);
      for (; ok && sw.next(t, k0, k1); tc++) {
        const int buf = tc % NACC, use = tc / NACC;
        if (*abort_flag || !mbar_wait(&accempty[buf], (use & 1) ^ 1)) { *abort_flag = 1; break; }
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(buf * BT);
        for (int k = k0; k < k1; k++, xi++) {
          // (a role that gave up makes these waits give up too: no flag check per step)
          if (!mbar_wait(&afull[sa], pa) || !mbar_wait(&xfull[sx], px)) {
            *abort_flag = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad0 = adesc0 + (uint64_t)(sa * (P::AB >> 4)), bd0 = xdesc0 + (uint64_t)(sx * (P::XB >> 4));
#pragma unroll
          for (int kk = 0; kk < T::NMMA; kk++) {
            const uint64_t ad = ad0 + (uint64_t)(2 * kk), bd = bd0 + (uint64_t)(2 * kk);
            if constexpr (ATM) {
              const uint32_t at = tmem + ACOL + (uint32_t)(32 * sa + 8 * kk);
              if constexpr (kInt) umma_i8_ts_pair(d, at, bd, IDESC, (k - k0) | kk);
              else umma_f16_ts_pair(d, at, bd, IDESC, (k - k0) | kk);
              (void)ad;
            } else if constexpr (PAIR == 2) {
              if constexpr (kInt) umma_i8_pair(d, ad, bd, IDESC, (k - k0) | kk);
              else umma_f16_pair(d, ad, bd, IDESC, (k - k0) | kk);
            } else {
              if constexpr (kInt) umma_i8(d, ad, bd, IDESC, (k - k0) | kk);
              else umma_f16(d, ad, bd, IDESC, (k - k0) | kk);
            }
          }
          if constexpr (PAIR == 2) {
            umma_commit_pair(&xempty[sx]);
            umma_commit_pair(&aempty[sa]);
          } else {
            umma_commit(&xempty[sx]);
            umma_commit(&aempty[sa]);
          }
          if (++sx == SX) { sx = 0; px ^= 1; }
          if (++sa == SA) { sa = 0; pa ^= 1; }
        }
        if (!ok) break;
        if constexpr (PAIR == 2) umma_commit_pair(&accfull[buf]);
        else umma_commit(&accfull[buf]);
      }
      // the last commits' arrivals land before the CTA may exit
      for (int i = xi - SX < 0 ? 0 : xi - SX; i < xi; i++) mbar_wait(&xempty[i % SX], (i / SX) & 1);
      for (int i = xi - SA < 0 ? 0 : xi - SA; i < xi; i++) mbar_wait(&aempty[i % SA], (i / SA) & 1);
    }
  } else if (warp < kFirstEpi) {
    // ------------------------------------------------------------ dequantizers
    // Two groups of four warps take alternate K steps, so that two steps are
    // dequantized at once; a thread writes a whole row of its group's steps
    // (both halves).  With A in TMEM a warp owns the row quarter its warp index
    // may address (32 * (warp % 4) ..); each group covers all four quarters.
    if constexpr (!kDense) {
    const int d = threadIdx.x - kFirstDq * 32;
    const int grp = (warp - kFirstDq) >> 2;
    const int r = ATM ? 32 * (warp & 3) + lane : (d & (kTileN - 1));
    uint4 sbv[2] = {make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u)};
    int it = 0, t, k0, k1;
    bool ok = true;
    SegWalk sw(a, nk, unit, units);
    while (ok && sw.next(t, k0, k1)) {
      for (int k = k0; k < k1; k++, it++) {
        if ((it & 1) != grp) continue;
        const int sr = it % SR, sa = it % SA;
        if (*abort_flag || !mbar_wait(&rfull[sr], (it / SR) & 1) || !mbar_wait(&aempty[sa], ((it / SA) & 1) ^ 1)) {
          *abort_flag = 1;
          ok = false;
          break;
        }
        const unsigned char *R = ringR + sr * P::RB;
        if constexpr (F == Fmt::Affine) {
          if (a.sc_tma && affine_box_step(k, k0, a.gs_log2)) {
            // a new block: the row's 8 scales and 8 biases (16 bytes each, conflict-free)
            const uint4 *box = reinterpret_cast<const uint4 *>(R + T::RAW);
            sbv[0] = box[a.sc_swap ? kTileN + r : r];
            sbv[1] = box[a.sc_swap ? r : kTileN + r];
          }
        }
        if constexpr (ATM) {
          uint32_t o0[16], o1[16];
          dequant_words<F, BITS>(a, k, r, 0, R, sbv, o0);
          dequant_words<F, BITS>(a, k, r, 1, R, sbv, o1);
          const uint32_t col = tmem + ((uint32_t)(32 * (warp & 3)) << 16) + ACOL + (uint32_t)(32 * sa);
          tmem_st<16>(col, o0);
          tmem_st<16>(col + 16, o1);
          tmem_st_wait();
          tc_fence_before();
        } else {
#pragma unroll
          for (int h = 0; h < 2; h++) {
            uint32_t o[16];
            dequant_words<F, BITS>(a, k, r, h, R, sbv, o);
            store_a_smem(ringA + sa * P::AB, r, h, o);
          }
          fence_proxy_async_smem();
        }
        __syncwarp();
        if (lane == 0) {
          if constexpr (PAIR == 2) mbar_arrive_remote(lead_afull + sa * 8);
          else mbar_arrive(&afull[sa]);
          mbar_arrive(&rempty[sr]);
        }
      }
    }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // Per segment: a whole tile is written out; a segment that starts inside
    // its tile (this unit's first) is stored as a partial for the unit that
    // holds the tile's head; the head segment (this unit's last) adds the
    // later units' partials, in unit order, and writes the tile.
    const int q = warp & 3;                        // TMEM lanes 32q .. 32q + 31 (this warp's quarter)
    const int lrow = 32 * q + lane;                // row within the CTA's 128
    const bool lead_thread = threadIdx.x == kFirstEpi * 32;
    int tc = 0, t, k0, k1;
    SegWalk sw(a, nk, unit, units);
    for (; sw.next(t, k0, k1); tc++) {
      const int buf = tc % NACC, use = tc / NACC;
      const int n0 = (t / a.Mt) * kTileN * PAIR + rank * kTileN, m0 = (t % a.Mt) * BT;
      if (*abort_flag || !mbar_wait(&accfull[buf], use & 1)) { *abort_flag = 1; break; }
      tc_fence_after();
      const bool contrib = k0 > 0;                  // store a partial
      const bool head = k0 == 0 && k1 < nk;         // finish a split tile
      int vfirst = 0, vlast = -1;                   // contributing units of a split tile
      if (head) {
        // the later units whose stream-K shares hold the rest of this tile
        const int64_t T0 = (int64_t)a.dpw * units * nk, W = (int64_t)a.T * nk - T0;
        const int64_t tile_end = (int64_t)(t + 1) * nk;
        vfirst = unit + 1;
        vlast = unit;
        while (vlast + 1 < units && T0 + (int64_t)(vlast + 1) * W / units < tile_end) vlast++;
        if (lead_thread) {
          for (int v = vfirst; v <= vlast; v++) {
            const uint32_t *f = a.flags + v * PAIR + rank;
            if (!flag_wait(f, a.stall ? kNeverEpoch : *epoch_slot)) { *abort_flag = 1; break; }
          }
        }
        named_bar_sync(1, 128);
      }
      const int row = n0 + lrow;
      float swn = 0.f;
      if constexpr (kInt) swn = row < a.N ? a.sw[row] : 0.f;
      if constexpr (ATM) {
        if (!contrib && !head && (!kInt || a.acc == nullptr)) {
          // whole tile: TMEM -> bf16 / fp16 staging, free the accumulator, then
          // write the tile row by row of tokens with 16-byte stores
          for (int ch = 0; ch < BT / 16; ch += 2) {
            uint32_t v0[16], v1[16];
            float sxv[32];
            if constexpr (kInt) {
#pragma unroll
              for (int j = 0; j < 32; j++) {
                const int m = m0 + ch * 16 + j;
                sxv[j] = m < a.M ? __ldg(a.sx + m) : 0.f;
              }
            }
            tmem_ld16(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(ch * 16), v0);
            tmem_ld16(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(ch * 16 + 16), v1);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; j++) {
              const uint32_t u = j < 16 ? v0[j] : v1[j - 16];
              float f;
              if constexpr (kInt) {
                const int acc = F == Fmt::I8 ? static_cast<int>(u) >> 4 : static_cast<int>(u);
                f = (float)acc * (sxv[j] * swn);
              } else {
                f = __uint_as_float(u);
              }
              stage[(ch * 16 + j) * kTileN + lrow] = kOutF16 ? __half_as_ushort(__float2half_rn(f))
                                                                    : __bfloat16_as_ushort(__float2bfloat16_rn(f));
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            if constexpr (PAIR == 2) mbar_arrive_remote(lead_accempty + buf * 8);
            else mbar_arrive(&accempty[buf]);
          }
          named_bar_sync(1, 128);
          const bool vec = (a.N % 8) == 0;
          const int tid = threadIdx.x - kFirstEpi * 32;
          for (int e = tid; e < BT * (kTileN / 8); e += 128) {
            const int tok = e / (kTileN / 8), c8 = (e % (kTileN / 8)) * 8;
            const int m = m0 + tok, n = n0 + c8;
            if (m >= a.M || n >= a.N) continue;
            const uint16_t *src = stage + tok * kTileN + c8;
            if (vec && n + 8 <= a.N) {
              *reinterpret_cast<uint4 *>(a.y + (int64_t)m * a.N + n) = *reinterpret_cast<const uint4 *>(src);
            } else {
              for (int i = 0; i < 8 && n + i < a.N; i++) a.y[(int64_t)m * a.N + n + i] = src[i];
            }
          }
          named_bar_sync(1, 128);   // the staging tile is free for the next segment
          continue;
        }
      }
      // split tiles (and, without tensor-memory A, whole tiles too) through the
      // chunked staging
      if ((contrib || head || !ATM) && (!kInt || a.acc == nullptr)) {
        {
          // Split tile, in chunks of 32 tokens through the staging buffer: two fp32
          // (s32) partial chunks [32 tokens][128 rows] (double-buffered), then the
          // bf16 / fp16 output chunk.  A contributing segment copies each chunk to its
          // workspace slot with coalesced 16-byte stores.  The head pulls the next
          // chunk of the first later unit's partial with cp.async while it finishes
          // the current one (adding any further units' partials, in unit order, and
          // its own accumulator), then writes the output chunk.
          constexpr int CT = 32, NCH = BT / CT, CW = CT * kTileN / 4;        // tokens, chunks, 16-byte words
          uint32_t *pq = reinterpret_cast<uint32_t *>(stage);                  // [2][CT][128] 32-bit
          uint16_t *po = stage + 2 * CT * kTileN * 2;                            // [CT][128] 16-bit
          const int tid = threadIdx.x - kFirstEpi * 32;
          auto part = [&](int v, int c) {   // chunk c of CTA slot v's partial, as 16-byte words
            return reinterpret_cast<const uint4 *>(a.ws + ((size_t)(v * PAIR + rank) * BT + c * CT) * kTileN);
          };
          auto pull = [&](int c) {          // chunk c of the first later unit's partial -> pq[c % 2]
            const uint4 *src = part(vfirst, c);
            uint4 *dst = reinterpret_cast<uint4 *>(pq + (c & 1) * CT * kTileN);
#pragma unroll
            for (int i = 0; i < CW / 128; i++) cp_async_16(dst + tid + 128 * i, src + tid + 128 * i, 16u);
            cp_async_commit();
          };
          if (head && vlast >= vfirst) pull(0);
          for (int c = 0; c < NCH; c++) {
            uint32_t *pc = pq + (c & 1) * CT * kTileN;
            if (head && vlast >= vfirst) {
              if (c + 1 < NCH) {
                pull(c + 1);
                cp_async_wait<1>();
              } else {
                cp_async_wait<0>();
              }
              // further units' partials of this chunk, added to the words this thread pulled
              for (int vv = vfirst + 1; vv <= vlast; vv++) {
                const uint4 *src = part(vv, c);
#pragma unroll
                for (int i = 0; i < CW / 128; i++) {
                  const uint4 w = __ldcg(src + tid + 128 * i);
                  uint4 &d = reinterpret_cast<uint4 *>(pc)[tid + 128 * i];
                  if constexpr (kInt) {
                    d.x = (uint32_t)((int)d.x + (int)w.x); d.y = (uint32_t)((int)d.y + (int)w.y);
                    d.z = (uint32_t)((int)d.z + (int)w.z); d.w = (uint32_t)((int)d.w + (int)w.w);
                  } else {
                    d.x = __float_as_uint(__uint_as_float(d.x) + __uint_as_float(w.x));
                    d.y = __float_as_uint(__uint_as_float(d.y) + __uint_as_float(w.y));
                    d.z = __float_as_uint(__uint_as_float(d.z) + __uint_as_float(w.z));
                    d.w = __float_as_uint(__uint_as_float(d.w) + __uint_as_float(w.w));
                  }
                }
              }
              named_bar_sync(1, 128);
            }
            uint32_t v0[16], v1[16];
            tmem_ld16(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(buf * BT + c * CT), v0);
            tmem_ld16(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(buf * BT + c * CT + 16), v1);
            tmem_ld_wait();
            if (c == NCH - 1) {   // the accumulator is free for the next segment
              tc_fence_before();
              __syncwarp();
              if (lane == 0) {
                if constexpr (PAIR == 2) mbar_arrive_remote(lead_accempty + buf * 8);
                else mbar_arrive(&accempty[buf]);
              }
            }
            if (contrib) {
#pragma unroll
              for (int j = 0; j < CT; j++) pc[j * kTileN + lrow] = j < 16 ? v0[j] : v1[j - 16];
              named_bar_sync(1, 128);
              uint4 *d4 = reinterpret_cast<uint4 *>(a.ws + ((size_t)blockIdx.x * BT + c * CT) * kTileN);
#pragma unroll
              for (int i = 0; i < CW / 128; i++) d4[tid + 128 * i] = reinterpret_cast<const uint4 *>(pc)[tid + 128 * i];
              // (the next chunk fills the other buffer: no barrier needed here)
            } else {
#pragma unroll
              for (int j = 0; j < CT; j++) {
                const uint32_t u = j < 16 ? v0[j] : v1[j - 16];
                const uint32_t p = vlast >= vfirst ? pc[j * kTileN + lrow] : 0u;
                float f;
                if constexpr (kInt) {
                  const int m = m0 + c * CT + j;
                  const int s32 = (int)u + (int)p;
                  const int acc = F == Fmt::I8 ? s32 >> 4 : s32;
                  f = (float)acc * ((m < a.M ? __ldg(a.sx + m) : 0.f) * swn);
                } else {
                  f = __uint_as_float(u) + __uint_as_float(p);
                }
                po[j * kTileN + lrow] = kOutF16 ? __half_as_ushort(__float2half_rn(f))
                                                       : __bfloat16_as_ushort(__float2bfloat16_rn(f));
              }
              named_bar_sync(1, 128);
              const bool vec = (a.N % 8) == 0;
#pragma unroll
              for (int i = 0; i < CT * (kTileN / 8) / 128; i++) {
                const int e = tid + 128 * i;
                const int tok = e / (kTileN / 8), c8 = (e % (kTileN / 8)) * 8;
                const int m = m0 + c * CT + tok, n = n0 + c8;
                if (m >= a.M || n >= a.N) continue;
                const uint16_t *src = po + tok * kTileN + c8;
                if (vec && n + 8 <= a.N) {
                  *reinterpret_cast<uint4 *>(a.y + (int64_t)m * a.N + n) = *reinterpret_cast<const uint4 *>(src);
                } else {
                  for (int k2 = 0; k2 < 8 && n + k2 < a.N; k2++) a.y[(int64_t)m * a.N + n + k2] = src[k2];
                }
              }
              named_bar_sync(1, 128);   // po and this chunk's partial buffer are free
            }
          }
          if (contrib) {   // publish the partial once all four warps stored theirs
            __threadfence();
            named_bar_sync(1, 128);
            if (lead_thread) flag_publish(a.flags + blockIdx.x, *epoch_slot);
          }
          continue;
        }
      }
      // two 16-token chunks at a time: the partial loads of both are in flight
      // together with the TMEM loads
      for (int ch = 0; ch < BT / 16; ch += 2) {
        uint32_t v[32], pv[32];
        if (!contrib) {
#pragma unroll
          for (int j = 0; j < 32; j++) pv[j] = 0u;
          for (int vv = vfirst; vv <= vlast; vv++) {
            const uint32_t *src = a.ws + ((size_t)(vv * PAIR + rank) * BT + ch * 16) * kTileN + lrow;
            uint32_t w[32];
#pragma unroll
            for (int j = 0; j < 32; j++) w[j] = __ldcg(src + j * kTileN);
#pragma unroll
            for (int j = 0; j < 32; j++) {
              if constexpr (kInt) pv[j] = (uint32_t)((int)pv[j] + (int)w[j]);
              else pv[j] = __float_as_uint(__uint_as_float(pv[j]) + __uint_as_float(w[j]));
            }
          }
        }
        {
          uint32_t v0[16], v1[16];
          tmem_ld16(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(buf * BT + ch * 16), v0);
          tmem_ld16(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(buf * BT + ch * 16 + 16), v1);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 16; j++) { v[j] = v0[j]; v[16 + j] = v1[j]; }
        }
        if (contrib) {
          uint32_t *dst = a.ws + ((size_t)blockIdx.x * BT + ch * 16) * kTileN + lrow;
#pragma unroll
          for (int j = 0; j < 32; j++) dst[j * kTileN] = v[j];
          continue;
        }
        if (vlast >= vfirst) {
#pragma unroll
          for (int j = 0; j < 32; j++) {
            if constexpr (kInt) v[j] = (uint32_t)((int)v[j] + (int)pv[j]);
            else v[j] = __float_as_uint(__uint_as_float(v[j]) + __uint_as_float(pv[j]));
          }
        }
        if (row < a.N) {
          // the chunk's token scales, loaded together before any store (the
          // stores below could alias them as far as the compiler knows)
          float sxv[32];
          if constexpr (kInt) {
#pragma unroll
            for (int j = 0; j < 32; j++) {
              const int m = m0 + ch * 16 + j;
              sxv[j] = m < a.M ? __ldg(a.sx + m) : 0.f;
            }
          }
#pragma unroll
          for (int j = 0; j < 32; j++) {
            const int m = m0 + ch * 16 + j;
            if (m < a.M) {
              const int64_t o = (int64_t)m * a.N + row;
              if constexpr (kInt) {
                // I8: the tensor core summed 16 * code; W8: the codes themselves
                const int acc = F == Fmt::I8 ? static_cast<int>(v[j]) >> 4 : static_cast<int>(v[j]);
                if (a.acc) a.acc[o] = acc;
                if (a.y) a.y[o] = __bfloat16_as_ushort(__float2bfloat16_rn((float)acc * (sxv[j] * swn)));
              } else if constexpr (kOutF16) {
                a.y[o] = __half_as_ushort(__float2half_rn(__uint_as_float(v[j])));
              } else {
                a.y[o] = __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(v[j])));
              }
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if constexpr (PAIR == 2) mbar_arrive_remote(lead_accempty + buf * 8);
        else mbar_arrive(&accempty[buf]);
      }
      if (contrib) {   // publish the partial once all four warps stored theirs
        __threadfence();
        named_bar_sync(1, 128);
        if (lead_thread) flag_publish(a.flags + blockIdx.x, *epoch_slot);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR == 2) cg::this_cluster().sync();   // no CTA leaves while its peer may still signal it
  if (warp == 1) {
    tc_fence_after();
    if constexpr (PAIR == 2) tmem_dealloc_pair(tmem, NCOLS);
    else tmem_dealloc(tmem, NCOLS);
  }
  if (a.ws && threadIdx.x == 0) {
    // the last CTA of the launch to finish advances the epoch counter: every CTA has
    // read it by then, and the next launch on the stream starts after this one ends
    __threadfence();
    if (atomicAdd(&a.ctr[1], 1u) == gridDim.x - 1) {
      a.ctr[1] = 0u;
      atomicAdd(&a.ctr[0], 1u);
    }
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

gwb_status map2d(CUtensorMap *m, CUtensorMapDataType dt, const void *ptr, uint64_t inner, uint64_t outer,
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

// Stream-K workspace, owned by the library: one per (device, stream), so that
// GEMMs on different streams never share partial slots; allocated (and its
// flags and counters zeroed) on the first call that needs it, outside stream
// capture, and kept until the process exits.  Each launch takes a fresh epoch
// from the workspace's launch counter on the device (graph replays included),
// so the flags never need clearing again.
struct Workspace {
  uint32_t *base = nullptr;
  size_t partial_bytes = 0;
  int nflags = 0;
};
std::mutex g_ws_mu;
std::map<std::pair<int, cudaStream_t>, Workspace> g_ws;
// Armed by inject_stream_k_stall(): the next stream-K launch's heads wait for
// kNeverEpoch (tests of the bounded-wait failure path).
std::atomic<int> g_stall_next{0};

bool stream_workspace(cudaStream_t st, size_t partial_bytes, int nflags, uint32_t **ws, uint32_t **flags) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  std::lock_guard<std::mutex> lk(g_ws_mu);
  Workspace &w = g_ws[std::make_pair(dev, st)];
  if (w.base == nullptr || w.partial_bytes < partial_bytes || w.nflags < nflags) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone) return false;
    if (w.base) {
      if (cudaStreamSynchronize(st) != cudaSuccess) return false;
      cudaFree(w.base);
      w = Workspace{};
    }
    const size_t fbytes = ((size_t)nflags * 4 + 255) / 256 * 256;
    void *p = nullptr;
    if (cudaMalloc(&p, partial_bytes + fbytes) != cudaSuccess) {
      (void)cudaGetLastError();
      return false;
    }
    if (cudaMemsetAsync(static_cast<unsigned char *>(p) + partial_bytes, 0, fbytes, st) != cudaSuccess) {
      cudaFree(p);
      return false;
    }
    w.base = static_cast<uint32_t *>(p);
    w.partial_bytes = partial_bytes;
    w.nflags = nflags;
  }
  *ws = w.base;
  *flags = w.base + w.partial_bytes / 4;
  return true;
}

// fixed_ws: stream-K scratch supplied by the caller of this function (partials
// then flags, room for max_units units) instead of the stream workspace.
template <Fmt F, int BITS, int BT, int PAIR, bool ATM>
gwb_status run_tc2(const void *xptr, CUtensorMapDataType xdt, int xelem, const CUtensorMap &tw,
                   const CUtensorMap &tsb, Args a, cudaStream_t st, uint32_t *fixed_ws = nullptr,
                   int max_units = 0) {
  using P = Plan2<F, BITS, BT, PAIR, ATM>;
  CUtensorMap tx;
  gwb_status s = map2d(&tx, xdt, xptr, (uint64_t)a.K, (uint64_t)a.M, (uint64_t)a.K * xelem, 128u / xelem,
                       (uint32_t)(BT / PAIR), CU_TENSOR_MAP_SWIZZLE_128B);
  if (s != GWB_OK) return s;
  a.Nt = (a.N + kTileN * PAIR - 1) / (kTileN * PAIR);
  a.Mt = (a.M + BT - 1) / BT;
  a.T = a.Nt * a.Mt;
  a.dpw = 0;
  auto kern = k_tc2<F, BITS, BT, PAIR, ATM>;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [&] {
    attr_err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, P::SMEM);
  });
  if (attr_err != cudaSuccess) return fail(GWB_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(attr_err));
  int units = kSMs / PAIR;
  if (max_units > 0 && max_units < units) units = max_units;
  const int nk = (a.K + Tr<F, BITS>::BK - 1) / Tr<F, BITS>::BK;
  // At most half as many tiles as units: each tile is split into s equal K parts
  // on s units (all parts finish together, so no head waits on a longer tail).
  // More than half: stream-K over all units (a tile then spans two or three
  // units), rather than whole tiles on part of the GPU.  More tiles than units:
  // stream-K over all units when whole tiles would leave part of the last wave
  // idle.  Stream-K only where every unit gets a few K steps.
  int grid_units = a.T < units ? a.T : units;
  int split_units = units;
  bool want_ws;
  if (a.T < units) {
    int s = units / a.T;
    if (s > 8) s = 8;                              // at most 7 partials per finished tile
    while (s > 1 && nk / s < 4) s--;               // and at least 4 K steps per part
    if (s > 1) {
      split_units = a.T * s;
      want_ws = true;
    } else {
      want_ws = (int64_t)a.T * nk >= 4LL * units;
    }
  } else {
    want_ws = a.T % units != 0 && (int64_t)a.T * nk >= 4LL * units;
  }
  a.ws = nullptr;
  a.flags = nullptr;
  a.ctr = nullptr;
  a.stall = 0;
  if (want_ws) {
    uint32_t *ws = nullptr, *fl = nullptr, *ctr = nullptr;
    bool have_ws = false;
    if (fixed_ws) {
      // flags of the units, then the two counters, cleared for this call
      ws = fixed_ws;
      fl = fixed_ws + (size_t)split_units * PAIR * BT * kTileN;
      ctr = fl + split_units * PAIR;
      have_ws = cudaMemsetAsync(fl, 0, ((size_t)split_units * PAIR + 2) * 4, st) == cudaSuccess;
    } else {
      // sized for the widest token tile, so that later calls never grow it
      have_ws = stream_workspace(st, (size_t)kSMs * 256 * kTileN * 4, kSMs + 2, &ws, &fl);
      ctr = fl + kSMs;
    }
    if (have_ws) {
      a.ws = ws;
      a.flags = fl;
      a.ctr = ctr;
      a.stall = g_stall_next.exchange(0);
      grid_units = split_units;
      // all but the last one or two waves of whole tiles go round robin; stream-K
      // balances the rest
      a.dpw = a.T >= 2 * split_units ? a.T / split_units - 1 : 0;
    }
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(PAIR * grid_units));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = P::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)PAIR;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = PAIR == 2 ? 1 : 0;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, tx, tw, tsb, a);
  if (e != cudaSuccess) return fail(GWB_ERR_CUDA, "persistent tensor-core GEMM: %s", cudaGetErrorString(e));
  return GWB_OK;
}

// Tokens above one 128-token tile: 256 x 256 tiles on CTA pairs (two-SM MMA,
// half the activation bytes per SM); else 128 x 128 tiles on single CTAs.
template <Fmt F, int BITS>
gwb_status dispatch2(int64_t M, const void *x, CUtensorMapDataType xdt, int xelem, const CUtensorMap &tw,
                     const CUtensorMap &tsb, const Args &a, cudaStream_t st, uint32_t *fixed_ws = nullptr,
                     int max_units = 0) {
  if (M <= 32) return run_tc2<F, BITS, 32, 1, false>(x, xdt, xelem, tw, tsb, a, st, fixed_ws, max_units);
  if (M <= 64) return run_tc2<F, BITS, 64, 1, false>(x, xdt, xelem, tw, tsb, a, st, fixed_ws, max_units);
  if (M <= 128) return run_tc2<F, BITS, 128, 1, false>(x, xdt, xelem, tw, tsb, a, st, fixed_ws, max_units);
  return run_tc2<F, BITS, 256, 2, kAInTmem>(x, xdt, xelem, tw, tsb, a, st, fixed_ws, max_units);
}

}  // namespace

void inject_stream_k_stall(bool armed) { g_stall_next.store(armed ? 1 : 0); }

namespace {

// ---------------------------------------------------------------- scratch without allocation
// Some callers cannot allocate device memory: code running under an allocator
// that owns all of the GPU's memory (a framework's caching pool, a serving
// runtime that reserves memory up front), or code that must not call
// cudaMalloc / cudaFree at all, since both may synchronize the device.  For
// them the prefill GEMM can run with its stream-K scratch in this fixed array:
// the partial tiles of at most kScratchPairs CTA pairs (8 MiB), their flags and
// the launch counters (512 bytes).
// It lives in every GPU that loads the library until the process exits.
constexpr int kScratchPairs = 32;
constexpr size_t kScratchPartialWords = (size_t)kScratchPairs * 2 * 256 * kTileN;
constexpr size_t kScratchFlagWords = 128;
static __device__ __align__(256) uint32_t g_noalloc_scratch[kScratchPartialWords + kScratchFlagWords];
// one 256-token x 128-row partial per CTA of the pairs, one flag per CTA and the
// two launch counters
static_assert(kScratchPartialWords == (size_t)kScratchPairs * 2 * 256 * kTileN &&
                  kScratchFlagWords >= (size_t)kScratchPairs * 2 + 2,
              "the scratch array must hold every pair's partials and flags");

// Device address of the array on the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up once
// per device (with that device current) and cached.
std::mutex g_scratch_mu;
std::map<int, uint32_t *> g_scratch_addr;

gwb_status noalloc_scratch(uint32_t **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(GWB_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  auto it = g_scratch_addr.find(dev);
  if (it == g_scratch_addr.end()) {
    uint32_t *p = nullptr;
    e = cudaGetSymbolAddress(reinterpret_cast<void **>(&p), g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr)
      return fail(GWB_ERR_CUDA, "cudaGetSymbolAddress of the GEMM scratch: %s", cudaGetErrorString(e));
    it = g_scratch_addr.emplace(dev, p).first;
  }
  *out = it->second;
  return GWB_OK;
}

}  // namespace

gwb_status launch_tc2_affine(const uint16_t *x, int64_t M, const uint32_t *wq, const uint16_t *scales,
                             const uint16_t *biases, int64_t N, int64_t K, int bits, int gs, uint16_t *y,
                             cudaStream_t st) {
  // scales are staged in 4-byte copies of aligned group pairs
  if ((K / gs) % 2 != 0 || (((uintptr_t)scales | (uintptr_t)biases) & 3) != 0) return GWB_ERR_UNSUPPORTED;
  Args a{};
  a.M = (int)M; a.N = (int)N; a.K = (int)K; a.gs = gs;
  a.gs_log2 = gs == 32 ? 5 : (gs == 64 ? 6 : 7);
  a.scales = scales; a.biases = biases; a.y = y;
  CUtensorMap tw, tsb;
  const uint64_t words = (uint64_t)K * bits / 32;
  gwb_status s = map2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT32, wq, words, (uint64_t)N, words * 4,
                       (uint32_t)(64 * bits / 32), (uint32_t)kTileN, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (s != GWB_OK) return s;
  // Scales and biases by TMA: one 3-D box [2 arrays][128 rows][8 groups] per K
  // step over both arrays (the third dimension steps from the lower array to
  // the higher one); needs 16-byte scale rows.  Else 4-byte cp.async copies.
  const int64_t G = K / gs;
  const uintptr_t ps = (uintptr_t)scales, pb = (uintptr_t)biases;
  const uint64_t diff = ps > pb ? ps - pb : pb - ps;
  a.sc_tma = 0;
  a.sc_swap = pb < ps ? 1 : 0;
  tsb = tw;
  if (G % 8 == 0 && diff != 0 && diff % 16 == 0 && diff < (1ull << 39)) {
    const cuuint64_t dims[3] = {(cuuint64_t)G, (cuuint64_t)N, 2};
    const cuuint64_t strides[2] = {(cuuint64_t)G * 2, diff};
    const cuuint32_t box[3] = {8, (cuuint32_t)kTileN, 2};
    const cuuint32_t es[3] = {1, 1, 1};
    if (encode_fn()(&tsb, CU_TENSOR_MAP_DATA_TYPE_UINT16, 3, (void *)(a.sc_swap ? pb : ps), dims, strides, box, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS)
      a.sc_tma = 1;
  }
  if (bits == 4) return dispatch2<Fmt::Affine, 4>(M, x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, tw, tsb, a, st);
  if (bits == 8) return dispatch2<Fmt::Affine, 8>(M, x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, tw, tsb, a, st);
  return dispatch2<Fmt::Affine, 2>(M, x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, tw, tsb, a, st);
}

gwb_status launch_tc2_affine_noalloc(const uint16_t *x, int64_t M, const uint32_t *wq, const uint16_t *scales,
                                     const uint16_t *biases, int64_t N, int64_t K, int bits, int gs, uint16_t *y,
                                     cudaStream_t st) {
  if (M <= 128)
    return fail(GWB_ERR_SHAPE, "qmm_affine_noalloc runs the prefill GEMM: M must exceed 128 (M=%lld)", (long long)M);
  if ((K / gs) % 2 != 0)
    return fail(GWB_ERR_UNSUPPORTED, "qmm_affine_noalloc needs an even number of groups per row (K/gs=%lld)",
                (long long)(K / gs));
  if ((((uintptr_t)scales | (uintptr_t)biases) & 3) != 0)
    return fail(GWB_ERR_ALIGN, "qmm_affine_noalloc needs 4-byte aligned scales and biases");
  uint32_t *scratch = nullptr;
  gwb_status s = noalloc_scratch(&scratch);
  if (s != GWB_OK) return s;
  Args a{};
  a.M = (int)M; a.N = (int)N; a.K = (int)K; a.gs = gs;
  a.gs_log2 = gs == 32 ? 5 : (gs == 64 ? 6 : 7);
  a.scales = scales; a.biases = biases; a.y = y;
  a.sc_tma = 0;
  CUtensorMap tw;
  const uint64_t words = (uint64_t)K * bits / 32;
  s = map2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT32, wq, words, (uint64_t)N, words * 4, (uint32_t)(64 * bits / 32),
            (uint32_t)kTileN, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (s != GWB_OK) return s;
  if (bits == 4)
    return dispatch2<Fmt::Affine, 4>(M, x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, tw, tw, a, st, scratch, kScratchPairs);
  if (bits == 8)
    return dispatch2<Fmt::Affine, 8>(M, x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, tw, tw, a, st, scratch, kScratchPairs);
  return dispatch2<Fmt::Affine, 2>(M, x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, tw, tw, a, st, scratch, kScratchPairs);
}

gwb_status launch_tc2_gptq(const uint16_t *x, int64_t M, const int32_t *qweight, const uint16_t *scales,
                           const int32_t *qzeros, const int32_t *g_idx, int64_t K, int64_t N, int gs, uint16_t *y,
                           cudaStream_t st, int zadd) {
  if (g_idx != nullptr || ((uintptr_t)scales & 15) != 0 || ((uintptr_t)qzeros & 3) != 0) return GWB_ERR_UNSUPPORTED;
  Args a{};
  a.M = (int)M; a.N = (int)N; a.K = (int)K; a.gs = gs;
  a.gs_log2 = gs == 32 ? 5 : (gs == 64 ? 6 : 7);
  a.scales = scales; a.qzeros = qzeros; a.y = y;
  a.zadd = zadd;
  CUtensorMap tw;
  gwb_status s = map2d(&tw, CU_TENSOR_MAP_DATA_TYPE_INT32, qweight, (uint64_t)N, (uint64_t)(K / 8), (uint64_t)N * 4,
                       (uint32_t)kTileN, 8u, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (s != GWB_OK) return s;
  return dispatch2<Fmt::Gptq, 4>(M, x, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, tw, tw, a, st);
}

gwb_status launch_tc2_i8i4(const int8_t *qx, const float *sx, int64_t M, const uint32_t *wq, const float *sw,
                           int64_t N, int64_t K, uint16_t *y, int32_t *acc, cudaStream_t st) {
  Args a{};
  a.M = (int)M; a.N = (int)N; a.K = (int)K; a.gs = 0;
  a.sx = sx; a.sw = sw; a.y = y; a.acc = acc;
  CUtensorMap tw;
  gwb_status s = map2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT32, wq, (uint64_t)(K / 8), (uint64_t)N, (uint64_t)(K / 8) * 4,
                       16u, (uint32_t)kTileN, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (s != GWB_OK) return s;
  return dispatch2<Fmt::I8, 4>(M, qx, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, tw, tw, a, st);
}

gwb_status launch_tc2_i8i8(const int8_t *qx, const float *sx, int64_t M, const int8_t *wq, const float *sw,
                           int64_t N, int64_t K, uint16_t *y, int32_t *acc, cudaStream_t st) {
  Args a{};
  a.M = (int)M; a.N = (int)N; a.K = (int)K; a.gs = 0;
  a.sx = sx; a.sw = sw; a.y = y; a.acc = acc;
  CUtensorMap tw;
  gwb_status s = map2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, wq, (uint64_t)K, (uint64_t)N, (uint64_t)K, 128u,
                       (uint32_t)kTileN, CU_TENSOR_MAP_SWIZZLE_128B);
  if (s != GWB_OK) return s;
  // a token tile no wider than the batch needs: 32 (decode), 128, or 256 on CTA pairs
  if (M <= 32) return run_tc2<Fmt::W8, 8, 32, 1, false>(qx, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, tw, tw, a, st);
  if (M <= 128) return run_tc2<Fmt::W8, 8, 128, 1, false>(qx, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, tw, tw, a, st);
  return run_tc2<Fmt::W8, 8, 256, 2, false>(qx, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, tw, tw, a, st);
}

// Dense fp16 weights [N, K] (act-order GPTQ after its dequantization): the weight
// tile goes by one swizzled TMA copy into the A stage, fp16 operands, fp16 output.
gwb_status launch_tc2_f16(const uint16_t *x, int64_t M, const uint16_t *w, int64_t N, int64_t K, uint16_t *y,
                          cudaStream_t st) {
  if (K % 8 != 0 || (reinterpret_cast<uintptr_t>(x) & 15) || (reinterpret_cast<uintptr_t>(w) & 15))
    return GWB_ERR_UNSUPPORTED;
  Args a{};
  a.M = (int)M; a.N = (int)N; a.K = (int)K; a.gs = 0;
  a.y = y;
  CUtensorMap tw;
  gwb_status s = map2d(&tw, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, w, (uint64_t)K, (uint64_t)N, (uint64_t)K * 2, 64u,
                       (uint32_t)kTileN, CU_TENSOR_MAP_SWIZZLE_128B);
  if (s != GWB_OK) return s;
  if (M <= 32) return run_tc2<Fmt::F16, 16, 32, 1, false>(x, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, tw, tw, a, st);
  if (M <= 64) return run_tc2<Fmt::F16, 16, 64, 1, false>(x, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, tw, tw, a, st);
  if (M <= 128) return run_tc2<Fmt::F16, 16, 128, 1, false>(x, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, tw, tw, a, st);
  return run_tc2<Fmt::F16, 16, 256, 2, false>(x, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, tw, tw, a, st);
}

// Scratch for dequantized weights, owned by the library like the stream-K
// workspace: one per (device, stream), grown on demand outside stream capture
// and kept until exit.  False when it would have to be allocated under capture
// (or the allocation fails); the caller then takes a path without it.
namespace {
std::mutex g_dq_mu;
std::map<std::pair<int, cudaStream_t>, std::pair<void *, size_t>> g_dq;
}  // namespace

bool dequant_scratch(cudaStream_t st, size_t bytes, uint16_t **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  std::lock_guard<std::mutex> lk(g_dq_mu);
  auto &e = g_dq[std::make_pair(dev, st)];
  if (e.first == nullptr || e.second < bytes) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone) return false;
    if (e.first) {
      if (cudaStreamSynchronize(st) != cudaSuccess) return false;
      cudaFree(e.first);
      e = {nullptr, 0};
    }
    void *p = nullptr;
    if (cudaMalloc(&p, bytes) != cudaSuccess) {
      (void)cudaGetLastError();
      return false;
    }
    e = {p, bytes};
  }
  *out = static_cast<uint16_t *>(e.first);
  return true;
}

}  // namespace gwb
