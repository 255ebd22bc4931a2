/*
 * Plain, slow CPU oracle for group-wise low-bit linear layers.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the library's product path may call,
 * link or load this file; only the tests, the smoke check and the benchmark's
 * CPU-baseline / reference arm use it.  It shares no code, header, table or
 * constant with the CUDA library: every formula below is written out again
 * from the pages it cites.
 *
 * Rules kept throughout:
 *   - naive loops in the order the pages state them, no blocking or fusion;
 *   - floating-point results that the method defines in fp32 (the quantizers)
 *     are computed in fp32 with one IEEE rounding per operation (the file is
 *     compiled with -ffp-contract=off, so no FMA is formed);
 *   - everything else (dequantized weights, matmuls) is computed in fp64, and
 *     the integer W4A8 accumulator in int64;
 *   - bf16 / fp16 values are carried as their raw 16-bit patterns (uint16_t)
 *     and decoded / rounded by the small helpers at the top of this file.
 *
 * Sources (page title, then section):
 *   [MLX8]  metrale_gpu_runtime/mlx_int8.rs, module doc "Layout": uint32 words
 *           of four bytes, low byte = lowest column; bf16 scales and biases of
 *           shape [out, in/G]; w[r,c] = byte*scales[r,c/G] + biases[r,c/G].
 *   [HFMTL] Hugging Face transformers docs, "Metal" quantization: affine
 *           quantization, codes packed in uint32 tensors with per-group scales
 *           and biases, fused dequant + matmul kernel affine_qmm_t, bits 2/4/8.
 *   [GPTQ]  TinyGPT "Quantization Expansion", section 1 "GPTQReader", "Format"
 *           and the dequant recipe (qweight packed along IN, qzeros packed
 *           along OUT, zero = stored + 1, g = g_idx[i]).
 *   [AWQZ]  TinyGPT "Quantization Expansion", section 1 "GPTQReader", the note
 *           after the dequant recipe: the "+1" on the stored zero belongs to
 *           GPTQ only; AWQ uses the stored zero as is.  The same note names
 *           the AWQ reader as a sibling of identical shapes, and its g_idx
 *           remark says plain AWQ has no g_idx.
 *   [FUSE]  metrale_gpu_runtime/mlx_int8.rs, doc comments of
 *           MlxInt8Weight::gemv_silu_gate (y = W (silu(gate) * up), the product
 *           never written to memory), MlxInt8Weight::gemv_silu_gate_resid
 *           (y[n] = x_resid[n] + sum_k W[n,k] (silu(gate[k]) up[k])) and the
 *           free function gemv_gate_up (gate_y = gate x, up_y = up x, x read
 *           once); silu(g) = g * sigmoid(g) = g / (1 + exp(-g)).
 *   [QAT]   TinyGPT "Quantization Expansion", section 4 "QAT", "Fake-quant +
 *           STE": per-row symmetric scale = max|W|/qMax, clip(round(W/scale)),
 *           qMax = 2^(bits-1) - 1.
 *   [W4A8]  executorch PR #24467 "mlx::int8_int4_gemm": dynamic symmetric
 *           per-token int8 activations x symmetric per-channel int4 weights,
 *           INT32 accumulation.
 *   [W8A8]  executorch PR #17234, Parakeet README "Quantization Configs":
 *           8da8w = 8-bit dynamic activations x 8-bit weights; the weights
 *           take the per-row symmetric quantizer of [QAT] with bits = 8
 *           (qMax = 127, clip to [-qMax, +qMax]).
 *   [LIN]   executorch PR #17234 DecomposeLinearPass and mlx_int8.rs gemm doc:
 *           linear(x, W) = x . W^T with W stored [out, in].
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* 16-bit float helpers (IEEE-754 binary16 and bfloat16), written from the   */
/* format definitions.                                                       */
/* ------------------------------------------------------------------------ */

static float bits_to_f32(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t f32_to_bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

/* bfloat16 is the top half of an fp32; decoding is exact. */
double orc_bf16_to_f64(uint16_t h) { return (double)bits_to_f32((uint32_t)h << 16); }

/* fp32 -> bfloat16, round to nearest, ties to even, on the 16 dropped bits. */
uint16_t orc_f32_to_bf16(float f)
{
    uint32_t u = f32_to_bits(f);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu) != 0)
        return (uint16_t)((u >> 16) | 0x0040u);            /* quiet NaN */
    uint32_t lsb = (u >> 16) & 1u;
    uint32_t rounded = u + 0x7fffu + lsb;                   /* carries into exponent as needed */
    return (uint16_t)(rounded >> 16);
}

/* binary16 -> double, exact: sign, 5-bit exponent (bias 15), 10-bit fraction. */
double orc_f16_to_f64(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int m = h & 0x3ff;
    double v;
    if (e == 0)        v = ldexp((double)m, -24);                 /* subnormal */
    else if (e == 31)  v = m ? NAN : INFINITY;
    else               v = ldexp((double)(m | 0x400), e - 25);    /* 1.m * 2^(e-15) */
    return sign ? -v : v;
}

/* double -> binary16, round to nearest, ties to even, with subnormals and
 * overflow to infinity.  The value is rounded on the binary16 grid at its own
 * binade; the quantum is a power of two, so v/quantum is exact in double. */
uint16_t orc_f64_to_f16(double v)
{
    uint16_t sign = 0;
    if (isnan(v)) return 0x7e00u;
    if (signbit(v)) { sign = 0x8000u; v = -v; }
    if (v == 0.0) return sign;
    int e2;
    frexp(v, &e2);                 /* v = f * 2^e2, f in [0.5, 1) -> binade exponent e2-1 */
    int binade = e2 - 1;
    if (binade < -14) binade = -14;                   /* subnormal range shares the 2^-24 quantum */
    double quantum = ldexp(1.0, binade - 10);
    double r = nearbyint(v / quantum) * quantum;      /* default rounding mode: ties to even */
    if (r > 65504.0) return (uint16_t)(sign | 0x7c00u);              /* past the largest finite */
    if (r < ldexp(1.0, -14)) {                        /* subnormal (or rounded to zero) */
        return (uint16_t)(sign | (uint16_t)(r / ldexp(1.0, -24)));
    }
    int e3;
    double f = frexp(r, &e3);                          /* r = f * 2^e3, f in [0.5,1) */
    int exp_field = (e3 - 1) + 15;
    int mant = (int)((f * 2.0 - 1.0) * 1024.0);        /* exact: r lies on the grid */
    return (uint16_t)(sign | (uint16_t)(exp_field << 10) | (uint16_t)mant);
}

/* ------------------------------------------------------------------------ */
/* MLX affine layout [MLX8] [HFMTL]                                          */
/*   word w of row n holds codes for columns k = w*(32/b) ... +(32/b)-1,     */
/*   column k at bit offset (k % (32/b)) * b: lowest bits = lowest column.   */
/* ------------------------------------------------------------------------ */

static int per_word(int bits) { return 32 / bits; }

/* code(n, k) = (Wq[n, k/(32/b)] >> ((k % (32/b)) * b)) & (2^b - 1) */
void orc_unpack_affine(const uint32_t *wq, int64_t N, int64_t K, int bits, int32_t *codes)
{
    int pw = per_word(bits);
    int64_t words = K / pw;
    uint32_t mask = (1u << bits) - 1u;
    for (int64_t n = 0; n < N; n++)
        for (int64_t k = 0; k < K; k++) {
            uint32_t word = wq[n * words + k / pw];
            codes[n * K + k] = (int32_t)((word >> ((k % pw) * bits)) & mask);
        }
}

/* Inverse of orc_unpack_affine: OR each code into its word at its offset. */
void orc_pack_affine(const int32_t *codes, int64_t N, int64_t K, int bits, uint32_t *wq)
{
    int pw = per_word(bits);
    int64_t words = K / pw;
    uint32_t mask = (1u << bits) - 1u;
    for (int64_t i = 0; i < N * words; i++) wq[i] = 0;
    for (int64_t n = 0; n < N; n++)
        for (int64_t k = 0; k < K; k++)
            wq[n * words + k / pw] |= ((uint32_t)codes[n * K + k] & mask) << ((k % pw) * bits);
}

/* Comparison under the total order of finite floats in which -0 < +0, so that
 * a group's min and max are unique bit patterns (the pages do not say which
 * zero a group holding both would report; this is the reading taken). */
static int less_total(float a, float b)
{
    return a < b || (a == b && signbit(a) && !signbit(b));
}

/* Per-group min/max affine quantizer, in fp32 with one rounding per step:
 *   mn = min, mx = max over the group's gs columns of row n
 *   s  = (mx - mn) / (2^b - 1)
 *   q  = clip(round_half_even((w - mn) / s), 0, 2^b - 1)     (q = 0 when s == 0)
 * Stored scale = bf16(s), stored bias = bf16(mn); the codes are computed from
 * the fp32 s and mn.  [HFMTL] gives the affine scheme (per-group scales and
 * biases); the min/max formula is this library's stated quantizer. */
void orc_qpack_affine(const float *w, int64_t N, int64_t K, int bits, int gs,
                      uint32_t *wq, uint16_t *scales, uint16_t *biases, int32_t *codes_out)
{
    int64_t G = K / gs;
    int qmax = (1 << bits) - 1;
    int pw = per_word(bits);
    int64_t words = K / pw;
    for (int64_t i = 0; i < N * words; i++) wq[i] = 0;
    for (int64_t n = 0; n < N; n++) {
        for (int64_t g = 0; g < G; g++) {
            const float *row = w + n * K + g * gs;
            float mn = row[0], mx = row[0];
            for (int j = 1; j < gs; j++) {
                if (less_total(row[j], mn)) mn = row[j];
                if (less_total(mx, row[j])) mx = row[j];
            }
            float range = mx - mn;
            float s = range / (float)qmax;
            scales[n * G + g] = orc_f32_to_bf16(s);
            biases[n * G + g] = orc_f32_to_bf16(mn);
            for (int j = 0; j < gs; j++) {
                int q = 0;
                if (s != 0.0f) {
                    float t = row[j] - mn;
                    float u = t / s;
                    float r = rintf(u);
                    if (r < 0.0f) r = 0.0f;
                    if (r > (float)qmax) r = (float)qmax;
                    q = (int)r;
                }
                int64_t k = g * gs + j;
                wq[n * words + k / pw] |= (uint32_t)q << ((k % pw) * bits);
                if (codes_out) codes_out[n * K + k] = q;
            }
        }
    }
}

/* w[n,k] = code * scale[n, k/gs] + bias[n, k/gs], exactly, in fp64 [MLX8]. */
void orc_dequant_affine_f64(const uint32_t *wq, const uint16_t *scales, const uint16_t *biases,
                            int64_t N, int64_t K, int bits, int gs, double *w)
{
    int pw = per_word(bits);
    int64_t words = K / pw;
    int64_t G = K / gs;
    uint32_t mask = (1u << bits) - 1u;
    for (int64_t n = 0; n < N; n++)
        for (int64_t k = 0; k < K; k++) {
            uint32_t code = (wq[n * words + k / pw] >> ((k % pw) * bits)) & mask;
            double s = orc_bf16_to_f64(scales[n * G + k / gs]);
            double b = orc_bf16_to_f64(biases[n * G + k / gs]);
            w[n * K + k] = (double)code * s + b;
        }
}

/* The standalone dequant's bf16 value: the exact code*s+b rounded once to fp32
 * and then to bf16.  code*s is exact in fp64 (at most 16 significant bits);
 * the fp64 sum with the bf16 bias is exact unless the two differ by more than
 * ~2^37 in magnitude, and then the smaller one is far below half an fp32 ulp
 * of the larger, which is itself an fp32 value, so the fp32 result is the same. */
void orc_dequant_affine_bf16(const uint32_t *wq, const uint16_t *scales, const uint16_t *biases,
                             int64_t N, int64_t K, int bits, int gs, uint16_t *w_bf16)
{
    int pw = per_word(bits);
    int64_t words = K / pw;
    int64_t G = K / gs;
    uint32_t mask = (1u << bits) - 1u;
    for (int64_t n = 0; n < N; n++)
        for (int64_t k = 0; k < K; k++) {
            uint32_t code = (wq[n * words + k / pw] >> ((k % pw) * bits)) & mask;
            double s = orc_bf16_to_f64(scales[n * G + k / gs]);
            double b = orc_bf16_to_f64(biases[n * G + k / gs]);
            double exact = (double)code * s + b;
            w_bf16[n * K + k] = orc_f32_to_bf16((float)exact);
        }
}

/* y[r, n] = sum_k x[rows[r], k] * w[n, k]  (fp64, k ascending)  [LIN] [HFMTL]
 * x is bf16 [M, K]; only the listed rows of x are evaluated (all rows when
 * rows == NULL, nrows == M).  w is dequantized on the fly from the packed
 * layout, exactly as orc_dequant_affine_f64 defines it. */
void orc_qmm_affine(const uint16_t *x, int64_t M, const int64_t *rows, int64_t nrows,
                    const uint32_t *wq, const uint16_t *scales, const uint16_t *biases,
                    int64_t N, int64_t K, int bits, int gs, double *y)
{
    int pw = per_word(bits);
    int64_t words = K / pw;
    int64_t G = K / gs;
    uint32_t mask = (1u << bits) - 1u;
    (void)M;
    for (int64_t r = 0; r < nrows; r++) {
        int64_t m = rows ? rows[r] : r;
        const uint16_t *xr = x + m * K;
        for (int64_t n = 0; n < N; n++) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; k++) {
                uint32_t code = (wq[n * words + k / pw] >> ((k % pw) * bits)) & mask;
                double s = orc_bf16_to_f64(scales[n * G + k / gs]);
                double b = orc_bf16_to_f64(biases[n * G + k / gs]);
                acc += orc_bf16_to_f64(xr[k]) * ((double)code * s + b);
            }
            y[r * N + n] = acc;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* GPTQ layout [GPTQ]                                                        */
/*   qweight int32 [K/8, N], scales fp16 [K/gs, N], qzeros int32 [K/gs, N/8], */
/*   g_idx int32 [K] (NULL means g = i / gs).                                */
/* ------------------------------------------------------------------------ */

/* The dequant recipe, one weight at a time, in the page's order:
 *   int4 = (qweight[i/8, o] >> ((i%8)*4)) & 0xF
 *   g    = g_idx[i]
 *   zero = ((qzeros[g, o/8] >> ((o%8)*4)) & 0xF) + 1
 *   W[o, i] = scales[g, o] * (int4 - zero)                               */
static double gptq_weight(const int32_t *qweight, const uint16_t *scales, const int32_t *qzeros,
                          const int32_t *g_idx, int64_t K, int64_t N, int gs, int64_t o, int64_t i)
{
    (void)K;
    uint32_t qint32 = (uint32_t)qweight[(i / 8) * N + o];
    int bit = (int)(i % 8) * 4;
    int int4 = (int)((qint32 >> bit) & 0xFu);
    int64_t g = g_idx ? (int64_t)g_idx[i] : i / gs;
    double scale = orc_f16_to_f64(scales[g * N + o]);
    uint32_t zint32 = (uint32_t)qzeros[g * (N / 8) + o / 8];
    int zbit = (int)(o % 8) * 4;
    int zero = (int)((zint32 >> zbit) & 0xFu) + 1;
    return scale * (double)(int4 - zero);
}

void orc_gptq_dequant_f64(const int32_t *qweight, const uint16_t *scales, const int32_t *qzeros,
                          const int32_t *g_idx, int64_t K, int64_t N, int gs, double *w /* [N,K] */)
{
    for (int64_t o = 0; o < N; o++)
        for (int64_t i = 0; i < K; i++)
            w[o * K + i] = gptq_weight(qweight, scales, qzeros, g_idx, K, N, gs, o, i);
}

/* fp16 output: the product scale*(int4-zero) is exact in fp64 (11-bit scale
 * times a 5-bit integer), so this is a single rounding to binary16. */
void orc_gptq_dequant_f16(const int32_t *qweight, const uint16_t *scales, const int32_t *qzeros,
                          const int32_t *g_idx, int64_t K, int64_t N, int gs, uint16_t *w /* [N,K] */)
{
    for (int64_t o = 0; o < N; o++)
        for (int64_t i = 0; i < K; i++)
            w[o * K + i] = orc_f64_to_f16(gptq_weight(qweight, scales, qzeros, g_idx, K, N, gs, o, i));
}

/* y[r, o] = sum_i x[rows[r], i] * W[o, i], x fp16 [M, K], fp64 accumulation. */
void orc_gptq_qmm(const uint16_t *x, int64_t M, const int64_t *rows, int64_t nrows,
                  const int32_t *qweight, const uint16_t *scales, const int32_t *qzeros,
                  const int32_t *g_idx, int64_t K, int64_t N, int gs, double *y)
{
    (void)M;
    for (int64_t r = 0; r < nrows; r++) {
        int64_t m = rows ? rows[r] : r;
        for (int64_t o = 0; o < N; o++) {
            double acc = 0.0;
            for (int64_t i = 0; i < K; i++)
                acc += orc_f16_to_f64(x[m * K + i]) *
                       gptq_weight(qweight, scales, qzeros, g_idx, K, N, gs, o, i);
            y[r * N + o] = acc;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* AWQ zero convention [AWQZ]: the GPTQ tensors and shapes, no g_idx, and    */
/* the stored zero nibble taken as the zero itself.                          */
/* ------------------------------------------------------------------------ */

/* W[o, i] = scales[i/gs, o] * (int4 - zero),
 *   int4 = (qweight[i/8, o] >> ((i%8)*4)) & 0xF,
 *   zero = (qzeros[i/gs, o/8] >> ((o%8)*4)) & 0xF                         */
static double awq_weight(const int32_t *qweight, const uint16_t *scales, const int32_t *qzeros,
                         int64_t N, int gs, int64_t o, int64_t i)
{
    int64_t g = i / gs;
    int int4 = (int)(((uint32_t)qweight[(i / 8) * N + o] >> ((i % 8) * 4)) & 0xFu);
    int zero = (int)(((uint32_t)qzeros[g * (N / 8) + o / 8] >> ((o % 8) * 4)) & 0xFu);
    return orc_f16_to_f64(scales[g * N + o]) * (double)(int4 - zero);
}

void orc_awq_dequant_f64(const int32_t *qweight, const uint16_t *scales, const int32_t *qzeros,
                         int64_t K, int64_t N, int gs, double *w /* [N,K] */)
{
    for (int64_t o = 0; o < N; o++)
        for (int64_t i = 0; i < K; i++)
            w[o * K + i] = awq_weight(qweight, scales, qzeros, N, gs, o, i);
}

/* One rounding to binary16 of the exact fp64 product (11-bit scale times an
 * integer in [-15, 15]). */
void orc_awq_dequant_f16(const int32_t *qweight, const uint16_t *scales, const int32_t *qzeros,
                         int64_t K, int64_t N, int gs, uint16_t *w /* [N,K] */)
{
    for (int64_t o = 0; o < N; o++)
        for (int64_t i = 0; i < K; i++)
            w[o * K + i] = orc_f64_to_f16(awq_weight(qweight, scales, qzeros, N, gs, o, i));
}

/* y[r, o] = sum_i x[rows[r], i] * W[o, i], x fp16 [M, K], fp64 accumulation. */
void orc_awq_qmm(const uint16_t *x, int64_t M, const int64_t *rows, int64_t nrows,
                 const int32_t *qweight, const uint16_t *scales, const int32_t *qzeros,
                 int64_t K, int64_t N, int gs, double *y)
{
    (void)M;
    for (int64_t r = 0; r < nrows; r++) {
        int64_t m = rows ? rows[r] : r;
        for (int64_t o = 0; o < N; o++) {
            double acc = 0.0;
            for (int64_t i = 0; i < K; i++)
                acc += orc_f16_to_f64(x[m * K + i]) * awq_weight(qweight, scales, qzeros, N, gs, o, i);
            y[r * N + o] = acc;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* W4A8 [W4A8] with the symmetric quantizer of [QAT]                         */
/* ------------------------------------------------------------------------ */

/* Dynamic per-token symmetric int8 (qMax = 127), fp32 arithmetic:
 *   amax = max_k |x[m,k]|;  sx = amax / 127;
 *   q = clip(round_half_even(x / sx), -127, 127); amax == 0 gives sx = 0, q = 0. */
void orc_quant_per_token_i8(const uint16_t *x, int64_t M, int64_t K, int8_t *qx, float *sx)
{
    for (int64_t m = 0; m < M; m++) {
        float amax = 0.0f;
        for (int64_t k = 0; k < K; k++) {
            float v = fabsf((float)orc_bf16_to_f64(x[m * K + k]));
            if (v > amax) amax = v;
        }
        float s = amax / 127.0f;
        sx[m] = s;
        for (int64_t k = 0; k < K; k++) {
            int q = 0;
            if (s != 0.0f) {
                float u = (float)orc_bf16_to_f64(x[m * K + k]) / s;
                float r = rintf(u);
                if (r < -127.0f) r = -127.0f;
                if (r > 127.0f) r = 127.0f;
                q = (int)r;
            }
            qx[m * K + k] = (int8_t)q;
        }
    }
}

/* Per-output-channel symmetric int4: sw = max_k |w[n,k]| / 7 (qMax = 7),
 * q = clip(round_half_even(w / sw), -8, 7), stored as the two's-complement
 * nibble q & 0xF, eight per uint32 along K, lowest nibble = lowest k. */
void orc_qpack_sym_i4(const float *w, int64_t N, int64_t K, uint32_t *wq, float *sw, int32_t *codes_out)
{
    int64_t words = K / 8;
    for (int64_t i = 0; i < N * words; i++) wq[i] = 0;
    for (int64_t n = 0; n < N; n++) {
        float amax = 0.0f;
        for (int64_t k = 0; k < K; k++) {
            float v = fabsf(w[n * K + k]);
            if (v > amax) amax = v;
        }
        float s = amax / 7.0f;
        sw[n] = s;
        for (int64_t k = 0; k < K; k++) {
            int q = 0;
            if (s != 0.0f) {
                float r = rintf(w[n * K + k] / s);
                if (r < -8.0f) r = -8.0f;
                if (r > 7.0f) r = 7.0f;
                q = (int)r;
            }
            wq[n * words + k / 8] |= ((uint32_t)q & 0xFu) << ((k % 8) * 4);
            if (codes_out) codes_out[n * K + k] = q;
        }
    }
}

/* Signed nibble k of row n: the 4-bit two's-complement value in [-8, 7]. */
static int sym_i4_code(const uint32_t *wq, int64_t K, int64_t n, int64_t k)
{
    uint32_t nib = (wq[n * (K / 8) + k / 8] >> ((k % 8) * 4)) & 0xFu;
    return nib >= 8 ? (int)nib - 16 : (int)nib;
}

/* acc[r, n] = sum_k qx[rows[r], k] * qw[n, k] in int64;  y = acc * sx[m] * sw[n]
 * in fp64.  Returns 0, or 1 when some accumulator does not fit in int32. */
int orc_gemm_i8i4(const int8_t *qx, const float *sx, int64_t M, const int64_t *rows, int64_t nrows,
                  const uint32_t *wq, const float *sw, int64_t N, int64_t K,
                  int64_t *acc, double *y)
{
    int overflow = 0;
    (void)M;
    for (int64_t r = 0; r < nrows; r++) {
        int64_t m = rows ? rows[r] : r;
        for (int64_t n = 0; n < N; n++) {
            int64_t a = 0;
            for (int64_t k = 0; k < K; k++)
                a += (int64_t)qx[m * K + k] * (int64_t)sym_i4_code(wq, K, n, k);
            if (a > INT32_MAX || a < INT32_MIN) overflow = 1;
            if (acc) acc[r * N + n] = a;
            if (y) y[r * N + n] = (double)a * (double)sx[m] * (double)sw[n];
        }
    }
    return overflow;
}

/* ------------------------------------------------------------------------ */
/* W8A8 [W8A8]: per-token int8 activations (orc_quant_per_token_i8) x       */
/* per-output-channel symmetric int8 weights, INT32 accumulation.           */
/* ------------------------------------------------------------------------ */

/* [QAT] with bits = 8: sw = max_k |w[n,k]| / 127, q = clip(round_half_even(w / sw),
 * -127, 127), fp32 arithmetic; sw == 0 gives q = 0.  wq int8 [N, K]. */
void orc_qpack_sym_i8(const float *w, int64_t N, int64_t K, int8_t *wq, float *sw)
{
    for (int64_t n = 0; n < N; n++) {
        float amax = 0.0f;
        for (int64_t k = 0; k < K; k++) {
            float v = fabsf(w[n * K + k]);
            if (v > amax) amax = v;
        }
        float s = amax / 127.0f;
        sw[n] = s;
        for (int64_t k = 0; k < K; k++) {
            int q = 0;
            if (s != 0.0f) {
                float r = rintf(w[n * K + k] / s);
                if (r < -127.0f) r = -127.0f;
                if (r > 127.0f) r = 127.0f;
                q = (int)r;
            }
            wq[n * K + k] = (int8_t)q;
        }
    }
}

/* acc[r, n] = sum_k qx[rows[r], k] * wq[n, k] in int64;  y = acc * sx[m] * sw[n]
 * in fp64.  Returns 0, or 1 when some accumulator does not fit in int32. */
int orc_gemm_i8i8(const int8_t *qx, const float *sx, int64_t M, const int64_t *rows, int64_t nrows,
                  const int8_t *wq, const float *sw, int64_t N, int64_t K, int64_t *acc, double *y)
{
    int overflow = 0;
    (void)M;
    for (int64_t r = 0; r < nrows; r++) {
        int64_t m = rows ? rows[r] : r;
        for (int64_t n = 0; n < N; n++) {
            int64_t a = 0;
            for (int64_t k = 0; k < K; k++)
                a += (int64_t)qx[m * K + k] * (int64_t)wq[n * K + k];
            if (a > INT32_MAX || a < INT32_MIN) overflow = 1;
            if (acc) acc[r * N + n] = a;
            if (y) y[r * N + n] = (double)a * (double)sx[m] * (double)sw[n];
        }
    }
    return overflow;
}

/* ------------------------------------------------------------------------ */
/* Fused decode products [FUSE] on the MLX affine layout                    */
/* ------------------------------------------------------------------------ */

static double silu(double g) { return g / (1.0 + exp(-g)); }

/* h[i] = silu(gate[i]) * up[i] in fp64, gate and up bf16 [n]. */
void orc_silu_mul(const uint16_t *gate, const uint16_t *up, int64_t n, double *h)
{
    for (int64_t i = 0; i < n; i++)
        h[i] = silu(orc_bf16_to_f64(gate[i])) * orc_bf16_to_f64(up[i]);
}

/* y[r, n] = (resid ? resid[m, n] : 0) + sum_k W[n, k] * silu(gate[m, k]) * up[m, k],
 * m = rows[r]; gate, up bf16 [M, K], resid bf16 [M, N] or NULL; fp64
 * throughout, W dequantized as orc_dequant_affine_f64 defines it. */
void orc_qmv_silu_gate(const uint16_t *gate, const uint16_t *up, int64_t M, const int64_t *rows, int64_t nrows,
                       const uint32_t *wq, const uint16_t *scales, const uint16_t *biases,
                       int64_t N, int64_t K, int bits, int gs, const uint16_t *resid, double *y)
{
    int pw = per_word(bits);
    int64_t words = K / pw;
    int64_t G = K / gs;
    uint32_t mask = (1u << bits) - 1u;
    (void)M;
    for (int64_t r = 0; r < nrows; r++) {
        int64_t m = rows ? rows[r] : r;
        for (int64_t n = 0; n < N; n++) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; k++) {
                double h = silu(orc_bf16_to_f64(gate[m * K + k])) * orc_bf16_to_f64(up[m * K + k]);
                uint32_t code = (wq[n * words + k / pw] >> ((k % pw) * bits)) & mask;
                double sc = orc_bf16_to_f64(scales[n * G + k / gs]);
                double b = orc_bf16_to_f64(biases[n * G + k / gs]);
                acc += ((double)code * sc + b) * h;
            }
            y[r * N + n] = (resid ? orc_bf16_to_f64(resid[m * N + n]) : 0.0) + acc;
        }
    }
}
