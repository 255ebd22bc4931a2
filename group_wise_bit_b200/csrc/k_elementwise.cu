// Elementwise / per-row kernels: affine quantize+pack, affine dequant, GPTQ
// dequant, per-token int8 quantization and symmetric int4 packing.
//
// All of them are bit-exact by construction: fp32 steps use the explicitly
// rounded intrinsics (__fsub_rn, __fdiv_rn, __fmaf_rn, __fmul_rn) so that the
// compiler cannot contract or reassociate them, rounding to integers uses
// rintf (round half to even), and min/max reductions are exact.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "dequant.cuh"
#include "internal.h"

namespace gwb {
namespace {

constexpr unsigned kFull = 0xffffffffu;

// Monotone map of finite floats to int32 under the total order -0 < +0; the
// per-group min/max of the affine quantizer are taken on these keys so that a
// group holding both zeros reports -0 as its min and +0 as its max.
__device__ __forceinline__ int order_key(float f) {
  int i = __float_as_int(f);
  return i >= 0 ? i : (i ^ 0x7fffffff);
}
__device__ __forceinline__ float key_to_float(int k) { return __int_as_float(k >= 0 ? k : (k ^ 0x7fffffff)); }

__device__ __forceinline__ uint16_t bf16_bits(float f) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}
__device__ __forceinline__ float bf16_val(uint16_t h) { return __uint_as_float(static_cast<uint32_t>(h) << 16); }

// ----------------------------------------------------------------------------
// qpack_affine: one warp per (row, group).  Lane l holds E = gs/32 consecutive
// columns of the group; the lanes sharing a packed word OR their fields
// together with a butterfly of shuffles and the first of them stores it.
template <int BITS, int GS>
__global__ void __launch_bounds__(256) k_qpack_affine(const float *__restrict__ w, int64_t N, int64_t K,
                                                      uint32_t *__restrict__ wq, uint16_t *__restrict__ scales,
                                                      uint16_t *__restrict__ biases) {
  constexpr int E = GS / 32;          // columns per lane
  constexpr int PW = 32 / BITS;       // codes per word
  constexpr int LPW = PW / E;         // lanes per word
  constexpr int QMAX = (1 << BITS) - 1;
  const int lane = threadIdx.x & 31;
  const int64_t G = K / GS;
  const int64_t unit = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (unit >= N * G) return;
  const int64_t n = unit / G, g = unit % G;
  const float *src = w + n * K + g * GS + lane * E;

  float v[E];
  if constexpr (E == 4) {
    float4 t = *reinterpret_cast<const float4 *>(src);
    v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
  } else if constexpr (E == 2) {
    float2 t = *reinterpret_cast<const float2 *>(src);
    v[0] = t.x; v[1] = t.y;
  } else {
    v[0] = src[0];
  }
  int kmin = order_key(v[0]), kmax = kmin;
#pragma unroll
  for (int j = 1; j < E; j++) {
    kmin = min(kmin, order_key(v[j]));
    kmax = max(kmax, order_key(v[j]));
  }
  kmin = __reduce_min_sync(kFull, kmin);
  kmax = __reduce_max_sync(kFull, kmax);
  const float mn = key_to_float(kmin), mx = key_to_float(kmax);
  const float s = __fdiv_rn(__fsub_rn(mx, mn), (float)QMAX);

  uint32_t part = 0;
#pragma unroll
  for (int j = 0; j < E; j++) {
    uint32_t q = 0;
    if (s != 0.0f) {
      float r = rintf(__fdiv_rn(__fsub_rn(v[j], mn), s));
      r = fminf(fmaxf(r, 0.0f), (float)QMAX);
      q = static_cast<uint32_t>(r);
    }
    part |= q << (((lane * E + j) % PW) * BITS);
  }
#pragma unroll
  for (int off = 1; off < LPW; off <<= 1) part |= __shfl_xor_sync(kFull, part, off);
  if (lane % LPW == 0) {
    const int64_t words_per_row = K / PW;
    wq[n * words_per_row + (g * GS + lane * E) / PW] = part;
  }
  if (lane == 0) {
    scales[n * G + g] = bf16_bits(s);
    biases[n * G + g] = bf16_bits(mn);
  }
}

// ----------------------------------------------------------------------------
// dequant_affine: one thread per packed word; the word's 32/bits outputs are
// contiguous in the bf16 [N, K] result and are written with 16-byte stores
// (8-byte stores for 8-bit words).
template <int BITS>
__global__ void __launch_bounds__(256) k_dequant_affine(const uint32_t *__restrict__ wq,
                                                        const uint16_t *__restrict__ scales,
                                                        const uint16_t *__restrict__ biases, int64_t N,
                                                        int64_t K, int gs, uint16_t *__restrict__ out) {
  constexpr int PW = 32 / BITS;
  constexpr uint32_t MASK = (1u << BITS) - 1u;
  const int64_t words_per_row = K / PW;
  const int64_t total = N * words_per_row;
  const int64_t G = K / gs;
  for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int64_t n = idx / words_per_row, wi = idx % words_per_row;
    const int64_t k0 = wi * PW;
    const uint32_t word = wq[idx];
    const float s = bf16_val(scales[n * G + k0 / gs]);
    const float b = bf16_val(biases[n * G + k0 / gs]);
    uint32_t packed[PW / 2];
#pragma unroll
    for (int j = 0; j < PW; j += 2) {
      const float lo = __fmaf_rn((float)((word >> (j * BITS)) & MASK), s, b);
      const float hi = __fmaf_rn((float)((word >> ((j + 1) * BITS)) & MASK), s, b);
      packed[j / 2] = (uint32_t)bf16_bits(lo) | ((uint32_t)bf16_bits(hi) << 16);
    }
    uint16_t *dst = out + n * K + k0;
    if constexpr (PW == 4) {
      *reinterpret_cast<uint2 *>(dst) = make_uint2(packed[0], packed[1]);
    } else {
#pragma unroll
      for (int j = 0; j < PW / 8; j++)
        reinterpret_cast<uint4 *>(dst)[j] =
            make_uint4(packed[4 * j], packed[4 * j + 1], packed[4 * j + 2], packed[4 * j + 3]);
    }
  }
}

// ----------------------------------------------------------------------------
// gptq_dequant: one CTA per tile of 64 out-features x 256 in-features.  The
// qweight words are read coalesced along the out-features (one 256-byte row
// segment per k-octet), each word becomes its eight fp16 weights in shared
// memory, and the tile leaves as 512-byte runs of each out-feature's row (the
// output is [N, K], K contiguous).  scale * (int4 - zero) is exact in fp32 (an
// 11-bit scale times a 5-bit integer), so __float2half_rn is the single rounding.
constexpr int kGdN = 64, kGdK = 256;                  // tile: out-features x in-features
constexpr int kGdRow = kGdK * 2 + 16;                 // bytes per staged row (16 bytes of padding: no bank conflicts)

__global__ void __launch_bounds__(256) k_gptq_dequant(const int32_t *__restrict__ qweight,
                                                      const uint16_t *__restrict__ scales,
                                                      const int32_t *__restrict__ qzeros,
                                                      const int32_t *__restrict__ g_idx, int64_t K, int64_t N,
                                                      int gs, int zadd, uint16_t *__restrict__ out) {
  __shared__ __align__(16) unsigned char tile[kGdN * kGdRow];
  const int64_t n0 = (int64_t)blockIdx.x * kGdN, k0 = (int64_t)blockIdx.y * kGdK;
  const int t = threadIdx.x;
  const int nl = t % kGdN, kb = t / kGdN;             // this thread: out-feature nl, k-octets kb*8 .. kb*8+7
  const int64_t o = n0 + nl;
  if (o < N && g_idx == nullptr) {
    // gs is a multiple of 8: the eight in-features of a word share one group, so
    // each word takes one scale and one zero, and all loads are issued up front
    uint32_t word[8], zw[8];
    uint16_t sh[8];
#pragma unroll
    for (int i = 0; i < 8; i++) {
      const int64_t kq = k0 / 8 + kb * 8 + i;
      const bool in = kq * 8 < K;
      const int64_t g = in ? kq * 8 / gs : 0;
      word[i] = in ? static_cast<uint32_t>(__ldg(qweight + kq * N + o)) : 0u;
      sh[i] = __ldg(scales + g * N + o);
      zw[i] = static_cast<uint32_t>(__ldg(qzeros + g * (N / 8) + o / 8));
    }
#pragma unroll
    for (int i = 0; i < 8; i++) {
      // pairs of fp16 (1024 + q) - (1024 + zero) = q - zero (exact), times the fp16
      // scale: one IEEE rounding of the exact product, as the scalar recipe
      const int kql = kb * 8 + i;
      const uint32_t zv = 0x6400u | (((zw[i] >> ((o % 8) * 4)) & 0xFu) + (uint32_t)zadd);
      const uint32_t sv = sh[i];
      const uint32_t z2[4] = {zv | (zv << 16), zv | (zv << 16), zv | (zv << 16), zv | (zv << 16)};
      const uint32_t s2[4] = {sv | (sv << 16), sv | (sv << 16), sv | (sv << 16), sv | (sv << 16)};
      *reinterpret_cast<uint4 *>(tile + nl * kGdRow + kql * 16) = dq::dq_gptq(word[i], z2, s2);
    }
  } else if (o < N) {
    // g_idx: every in-feature has its own group
#pragma unroll 2
    for (int i = 0; i < 8; i++) {
      const int kql = kb * 8 + i;                     // k-octet within the tile
      const int64_t kq = k0 / 8 + kql;
      if (kq * 8 >= K) break;
      const uint32_t word = static_cast<uint32_t>(__ldg(qweight + kq * N + o));
      uint32_t packed[4];
#pragma unroll
      for (int j = 0; j < 8; j++) {
        const int64_t k = kq * 8 + j;
        const int64_t g = (int64_t)__ldg(g_idx + k);
        const float s = __half2float(__ushort_as_half(__ldg(scales + g * N + o)));
        const uint32_t zw = static_cast<uint32_t>(__ldg(qzeros + g * (N / 8) + o / 8));
        const int zero = (int)((zw >> ((o % 8) * 4)) & 0xFu) + zadd;
        const int q = (int)((word >> (j * 4)) & 0xFu);
        const uint16_t h = __half_as_ushort(__float2half_rn(__fmul_rn(s, (float)(q - zero))));
        if (j & 1) packed[j / 2] |= (uint32_t)h << 16;
        else packed[j / 2] = h;
      }
      *reinterpret_cast<uint4 *>(tile + nl * kGdRow + kql * 16) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    }
  }
  __syncthreads();
  // each warp writes whole row runs: 32 lanes x 16 bytes = the row's 256 in-features
  const int lane = t & 31, warp = t >> 5;
  const int64_t kcols = K - k0 < kGdK ? K - k0 : kGdK;   // a multiple of 8 (K % gs == 0, gs % 8 == 0)
  for (int r = warp; r < kGdN; r += 8) {
    const int64_t orow = n0 + r;
    if (orow >= N) break;
    if ((int64_t)lane * 8 < kcols)
      *reinterpret_cast<uint4 *>(out + orow * K + k0 + lane * 8) = *reinterpret_cast<const uint4 *>(tile + r * kGdRow + lane * 16);
  }
}

// ----------------------------------------------------------------------------
// quant_per_token_i8: one block per token row; pass 1 reduces max|x| (exact),
// pass 2 quantizes (the row is re-read from L1/L2).
__device__ __forceinline__ float block_max(float v, float *red) {
  v = fmaxf(v, __shfl_xor_sync(kFull, v, 16));
  v = fmaxf(v, __shfl_xor_sync(kFull, v, 8));
  v = fmaxf(v, __shfl_xor_sync(kFull, v, 4));
  v = fmaxf(v, __shfl_xor_sync(kFull, v, 2));
  v = fmaxf(v, __shfl_xor_sync(kFull, v, 1));
  const int wid = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[wid] = v;
  __syncthreads();
  if (wid == 0) {
    float t = lane < (int)(blockDim.x >> 5) ? red[lane] : 0.0f;
    t = fmaxf(t, __shfl_xor_sync(kFull, t, 16));
    t = fmaxf(t, __shfl_xor_sync(kFull, t, 8));
    t = fmaxf(t, __shfl_xor_sync(kFull, t, 4));
    t = fmaxf(t, __shfl_xor_sync(kFull, t, 2));
    t = fmaxf(t, __shfl_xor_sync(kFull, t, 1));
    if (lane == 0) red[32] = t;
  }
  __syncthreads();
  return red[32];
}

__device__ __forceinline__ int8_t quant_i8(float x, float s) {
  if (s == 0.0f) return 0;
  float r = rintf(__fdiv_rn(x, s));
  r = fminf(fmaxf(r, -127.0f), 127.0f);
  return static_cast<int8_t>(r);
}

__global__ void __launch_bounds__(256) k_quant_per_token_i8(const uint16_t *__restrict__ x, int64_t K,
                                                            int8_t *__restrict__ qx, float *__restrict__ sx) {
  __shared__ float red[33];
  const int64_t m = blockIdx.x;
  const uint16_t *row = x + m * K;
  int8_t *qrow = qx + m * K;
  const bool vec = (K % 8) == 0;
  float amax = 0.0f;
  if (vec) {
    for (int64_t i = threadIdx.x; i < K / 8; i += blockDim.x) {
      const uint4 u = reinterpret_cast<const uint4 *>(row)[i];
      const uint32_t p[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int j = 0; j < 4; j++) {
        amax = fmaxf(amax, fabsf(__uint_as_float(p[j] << 16)));
        amax = fmaxf(amax, fabsf(__uint_as_float(p[j] & 0xffff0000u)));
      }
    }
  } else {
    for (int64_t i = threadIdx.x; i < K; i += blockDim.x) amax = fmaxf(amax, fabsf(bf16_val(row[i])));
  }
  amax = block_max(amax, red);
  const float s = __fdiv_rn(amax, 127.0f);
  if (threadIdx.x == 0) sx[m] = s;
  if (vec) {
    for (int64_t i = threadIdx.x; i < K / 8; i += blockDim.x) {
      const uint4 u = reinterpret_cast<const uint4 *>(row)[i];
      const uint32_t p[4] = {u.x, u.y, u.z, u.w};
      uint32_t o[2] = {0, 0};
#pragma unroll
      for (int j = 0; j < 4; j++) {
        const uint32_t lo = (uint8_t)quant_i8(__uint_as_float(p[j] << 16), s);
        const uint32_t hi = (uint8_t)quant_i8(__uint_as_float(p[j] & 0xffff0000u), s);
        o[j / 2] |= (lo | (hi << 8)) << ((j % 2) * 16);
      }
      reinterpret_cast<uint2 *>(qrow)[i] = make_uint2(o[0], o[1]);
    }
  } else {
    for (int64_t i = threadIdx.x; i < K; i += blockDim.x) qrow[i] = quant_i8(bf16_val(row[i]), s);
  }
}

// ----------------------------------------------------------------------------
// qpack_sym_i4: one warp per output row; pass 1 reduces max|w|, pass 2 packs
// eight two's-complement nibbles per word (lowest k in the lowest nibble).
__global__ void __launch_bounds__(256) k_qpack_sym_i4(const float *__restrict__ w, int64_t N, int64_t K,
                                                      uint32_t *__restrict__ wq, float *__restrict__ sw) {
  const int lane = threadIdx.x & 31;
  const int64_t n = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (n >= N) return;
  const float *row = w + n * K;
  float amax = 0.0f;
  for (int64_t i = lane; i < K / 4; i += 32) {
    const float4 t = reinterpret_cast<const float4 *>(row)[i];
    amax = fmaxf(amax, fmaxf(fmaxf(fabsf(t.x), fabsf(t.y)), fmaxf(fabsf(t.z), fabsf(t.w))));
  }
  for (int off = 16; off; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, off));
  const float s = __fdiv_rn(amax, 7.0f);
  if (lane == 0) sw[n] = s;
  for (int64_t wi = lane; wi < K / 8; wi += 32) {
    const float4 a = reinterpret_cast<const float4 *>(row + wi * 8)[0];
    const float4 b = reinterpret_cast<const float4 *>(row + wi * 8)[1];
    const float v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint32_t word = 0;
#pragma unroll
    for (int j = 0; j < 8; j++) {
      int q = 0;
      if (s != 0.0f) {
        float r = rintf(__fdiv_rn(v[j], s));
        r = fminf(fmaxf(r, -8.0f), 7.0f);
        q = (int)r;
      }
      word |= ((uint32_t)q & 0xFu) << (4 * j);
    }
    wq[n * (K / 8) + wi] = word;
  }
}

int grid_for(int64_t work, int threads) {
  int64_t b = (work + threads - 1) / threads;
  if (b > (int64_t)148 * 64) b = (int64_t)148 * 64;  // grid-stride beyond this
  return (int)(b < 1 ? 1 : b);
}


// ----------------------------------------------------------------------------
// qpack_sym_i8: one warp per output row; pass 1 reduces max|w|, pass 2 writes
// sixteen int8 codes per 16-byte store (K % 16 == 0).
__global__ void __launch_bounds__(256) k_qpack_sym_i8(const float *__restrict__ w, int64_t N, int64_t K,
                                                      int8_t *__restrict__ wq, float *__restrict__ sw) {
  const int lane = threadIdx.x & 31;
  const int64_t n = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (n >= N) return;
  const float *row = w + n * K;
  float amax = 0.0f;
  for (int64_t i = lane; i < K / 4; i += 32) {
    const float4 t = reinterpret_cast<const float4 *>(row)[i];
    amax = fmaxf(amax, fmaxf(fmaxf(fabsf(t.x), fabsf(t.y)), fmaxf(fabsf(t.z), fabsf(t.w))));
  }
  for (int off = 16; off; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, off));
  const float s = __fdiv_rn(amax, 127.0f);
  if (lane == 0) sw[n] = s;
  for (int64_t ci = lane; ci < K / 16; ci += 32) {
    const float4 *src = reinterpret_cast<const float4 *>(row + ci * 16);
    uint32_t packed[4];
#pragma unroll
    for (int q4 = 0; q4 < 4; q4++) {
      const float4 t = src[q4];
      const float v[4] = {t.x, t.y, t.z, t.w};
      uint32_t word = 0;
#pragma unroll
      for (int j = 0; j < 4; j++) {
        int q = 0;
        if (s != 0.0f) q = (int)fminf(fmaxf(rintf(__fdiv_rn(v[j], s)), -127.0f), 127.0f);
        word |= ((uint32_t)q & 0xFFu) << (8 * j);
      }
      packed[q4] = word;
    }
    reinterpret_cast<uint4 *>(wq + n * K)[ci] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
  }
}

}  // namespace

void launch_qpack_affine(const float *w, int64_t N, int64_t K, int bits, int gs, uint32_t *wq,
                         uint16_t *scales, uint16_t *biases, cudaStream_t st) {
  const int64_t units = N * (K / gs);
  const unsigned blocks = (unsigned)((units + 7) / 8);
#define GWB_QP(B, S)                                                                      \
  if (bits == B && gs == S) {                                                             \
    k_qpack_affine<B, S><<<blocks, 256, 0, st>>>(w, N, K, wq, scales, biases);            \
    return;                                                                               \
  }
  GWB_QP(2, 32) GWB_QP(2, 64) GWB_QP(2, 128)
  GWB_QP(4, 32) GWB_QP(4, 64) GWB_QP(4, 128)
  GWB_QP(8, 32) GWB_QP(8, 64) GWB_QP(8, 128)
#undef GWB_QP
}

void launch_dequant_affine(const uint32_t *wq, const uint16_t *scales, const uint16_t *biases, int64_t N,
                           int64_t K, int bits, int gs, uint16_t *w_out, cudaStream_t st) {
  const int64_t words = N * K * bits / 32;
  const int grid = grid_for(words, 256);
  if (bits == 2) k_dequant_affine<2><<<grid, 256, 0, st>>>(wq, scales, biases, N, K, gs, w_out);
  if (bits == 4) k_dequant_affine<4><<<grid, 256, 0, st>>>(wq, scales, biases, N, K, gs, w_out);
  if (bits == 8) k_dequant_affine<8><<<grid, 256, 0, st>>>(wq, scales, biases, N, K, gs, w_out);
}

void launch_gptq_dequant(const int32_t *qweight, const uint16_t *scales, const int32_t *qzeros,
                         const int32_t *g_idx, int64_t K, int64_t N, int gs, uint16_t *w_out, cudaStream_t st,
                         int zadd) {
  const dim3 grid((unsigned)((N + kGdN - 1) / kGdN), (unsigned)((K + kGdK - 1) / kGdK));
  k_gptq_dequant<<<grid, 256, 0, st>>>(qweight, scales, qzeros, g_idx, K, N, gs, zadd, w_out);
}

void launch_quant_per_token_i8(const uint16_t *x, int64_t M, int64_t K, int8_t *qx, float *sx,
                               cudaStream_t st) {
  k_quant_per_token_i8<<<(unsigned)M, 256, 0, st>>>(x, K, qx, sx);
}

void launch_qpack_sym_i8(const float *w, int64_t N, int64_t K, int8_t *wq, float *sw, cudaStream_t st) {
  k_qpack_sym_i8<<<(unsigned)((N + 7) / 8), 256, 0, st>>>(w, N, K, wq, sw);
}

void launch_qpack_sym_i4(const float *w, int64_t N, int64_t K, uint32_t *wq, float *sw, cudaStream_t st) {
  k_qpack_sym_i4<<<(unsigned)((N + 7) / 8), 256, 0, st>>>(w, N, K, wq, sw);
}

}  // namespace gwb
