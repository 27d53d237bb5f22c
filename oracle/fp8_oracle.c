/*
 * fp8_oracle.c — CPU oracle of the FP8 delayed-scaling Linear step and its fused AdamW.
 *
 * TEST INFRASTRUCTURE. This is the plain, slow, obviously correct statement of what the GPU
 * library computes. Only the test suite, the package smoke check and the benchmark's CPU
 * baseline load it; the product path never does. It shares no code, header, table or constant
 * generator with the CUDA library: every FP8 value is encoded and decoded here from the bit
 * fields, by integer manipulation written out below. Build: gcc -O2 -ffp-contract=off -fopenmp
 * (plain IEEE single/double arithmetic, no fused multiply-add, no fast-math).
 * Threads (OpenMP) only split work whose pieces are independent (output elements, rows, the
 * fixed chunks of the norm sum) or combine integer counts and maxima, so every result is the
 * same bit for bit whatever the thread count (orc_set_threads; 1 gives the plain sequential
 * program).
 *
 * Sources, cited by page title and section:
 *   [P1] "算子与编译器：FP8 训练与优化器 Kernel"
 *   [P2] "FP8 混合精度训练工程实践：从 H100 到大模型训练的范式跃迁"
 *   [P3] "LLM FP8 微调上线生产实战：用 Amax Scaling、层级白名单与 BF16 回退守住收敛"
 *
 * Where the pages are silent or disagree, the reading taken is stated at the function.
 */
#include <float.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_E4M3 0
#define ORC_E5M2 1
#define ORC_AMAX_MAX 0
#define ORC_AMAX_MOST_RECENT 1

/* Threads used by the functions below (0 or less: all the host offers). Returns the count now
 * in effect. */
int orc_set_threads(int n)
{
#ifdef _OPENMP
    omp_set_num_threads(n > 0 ? n : omp_get_num_procs());
    return omp_get_max_threads();
#else
    (void)n;
    return 1;
#endif
}

int orc_get_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

static uint32_t f32_bits(float f) { uint32_t b; memcpy(&b, &f, 4); return b; }
static float bits_f32(uint32_t b) { float f; memcpy(&f, &b, 4); return f; }

/* ---------------------------------------------------------------------------------------
 * BF16 <-> f32. A BF16 value is the top half of an f32, so widening is exact.
 * Narrowing rounds to nearest, ties to even; NaN becomes the quiet NaN 0x7FC0.
 * ------------------------------------------------------------------------------------- */
float orc_bf16_to_f32(uint16_t h) { return bits_f32(((uint32_t)h) << 16); }

uint16_t orc_f32_to_bf16(float f)
{
    uint32_t b = f32_bits(f);
    if ((b & 0x7FFFFFFFu) > 0x7F800000u) return 0x7FC0;
    uint32_t upper = b >> 16, lower = b & 0xFFFFu;
    if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u))) upper += 1; /* may carry into inf */
    return (uint16_t)upper;
}

/* ---------------------------------------------------------------------------------------
 * FP8 formats [P2 §一, FP8 格式设计]: E4M3 = 1 sign, 4 exponent, 3 mantissa bits, bias 7,
 * range +-448; E5M2 = 1-5-2 bits, bias 15, range +-57344.
 *
 * Reading (the pages give only bias and range): the largest finite values 448 = 1.75 * 2^8 and
 * 57344 = 1.75 * 2^15 fix the special encodings. E4M3 reaches 2^8 only if the all-ones exponent
 * (15) holds finite values, so only S.1111.111 is NaN and there is no infinity. E5M2's maximum
 * sits at exponent 30, so exponent 31 is reserved IEEE-style: mantissa 0 = infinity, else NaN.
 * Exponent field 0 holds subnormals (no implicit one, exponent 1 - bias).
 * ------------------------------------------------------------------------------------- */
static int fmt_mbits(int fmt) { return fmt == ORC_E4M3 ? 3 : 2; }
static int fmt_bias(int fmt) { return fmt == ORC_E4M3 ? 7 : 15; }
static uint8_t fmt_maxcode(int fmt) { return fmt == ORC_E4M3 ? 0x7E : 0x7B; }
static float fmt_max(int fmt) { return fmt == ORC_E4M3 ? 448.0f : 57344.0f; }

int orc_fp8_is_finite(uint8_t code, int fmt)
{
    uint8_t mag = code & 0x7F;
    if (fmt == ORC_E4M3) return mag != 0x7F;
    return mag < 0x7C;
}

/* Value of an FP8 code, read from its fields. */
double orc_fp8_decode(uint8_t code, int fmt)
{
    const int mb = fmt_mbits(fmt), bias = fmt_bias(fmt);
    const int ebits = 7 - mb;
    const int sign = code >> 7;
    const int e = (code >> mb) & ((1 << ebits) - 1);
    const int man = code & ((1 << mb) - 1);
    double mag;
    if (fmt == ORC_E4M3 && e == 15 && man == 7) return NAN;
    if (fmt == ORC_E5M2 && e == 31) {
        if (man != 0) return NAN;
        mag = INFINITY;
    } else if (e == 0) {
        mag = ldexp((double)man, 1 - bias - mb);             /* (man / 2^mb) * 2^(1-bias)  */
    } else {
        mag = ldexp((double)((1 << mb) + man), e - bias - mb); /* (1 + man/2^mb) * 2^(e-bias) */
    }
    return sign ? -mag : mag;
}

/* Shift right by s with round-to-nearest, ties to even. */
static uint64_t rne_shift(uint64_t x, int s)
{
    if (s <= 0) return x << (-s);
    if (s >= 64) return 0;
    uint64_t q = x >> s;
    uint64_t rem = x & ((1ull << s) - 1);
    uint64_t half = 1ull << (s - 1);
    if (rem > half || (rem == half && (q & 1))) q += 1;
    return q;
}

/*
 * f32 -> FP8 code, round to nearest even with saturation.
 * Saturation: the FP8Tensor quantize step clamps to +-max before storing [P2 §四]; a finite
 * value above max, and an infinity, give +-max. Reading for NaN (pages silent): the byte 0x7F
 * for both formats, sign dropped.
 */
uint8_t orc_fp8_encode(float v, int fmt)
{
    const uint32_t b = f32_bits(v);
    const uint32_t sign = (b >> 31) & 1u;
    const uint32_t mag = b & 0x7FFFFFFFu;
    const int mb = fmt_mbits(fmt), bias = fmt_bias(fmt);
    const uint8_t maxcode = fmt_maxcode(fmt);
    uint32_t code;

    if (mag > 0x7F800000u) return 0x7F;                                   /* NaN            */
    if (mag > f32_bits(fmt_max(fmt))) return (uint8_t)((sign << 7) | maxcode); /* saturate   */

    /* |v| = sig * 2^(e - 23) with a 24-bit significand sig. */
    int e;
    uint64_t sig;
    if (mag >= 0x00800000u) {
        e = (int)(mag >> 23) - 127;
        sig = (mag & 0x7FFFFFu) | 0x800000u;
    } else {
        e = -126;                     /* f32 subnormal (or zero) */
        sig = mag & 0x7FFFFFu;
    }
    const int emin = 1 - bias;        /* exponent of the smallest FP8 normal */
    if (e < emin) {
        /* FP8 subnormal range: code = round(|v| / 2^(emin - mb)); a result of 2^mb is
         * exactly the smallest normal, whose code is also 2^mb. */
        code = (uint32_t)rne_shift(sig, 23 + emin - mb - e);
    } else {
        uint32_t t = (uint32_t)rne_shift(sig, 23 - mb);  /* in [2^mb, 2^(mb+1)] */
        int ee = e;
        if (t == (1u << (mb + 1))) { t >>= 1; ee += 1; }
        code = ((uint32_t)(ee + bias) << mb) | (t & ((1u << mb) - 1));
    }
    if (code > maxcode) code = maxcode;  /* cannot trigger once |v| <= max; kept as a guard */
    return (uint8_t)((sign << 7) | code);
}

/* Encode an array of f32 values (the encode above, element by element). */
void orc_fp8_encode_array(const float* x, int64_t n, int fmt, uint8_t* out)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = orc_fp8_encode(x[i], fmt);
}

/* ---------------------------------------------------------------------------------------
 * Cast / transpose / amax.
 * q = encode(f32(x) * scale): one f32 multiply rounded to nearest, then the encode above
 * (the FP8Tensor quantize: x * scale, clamp, store as FP8 [P2 §四]).
 * amax = max |x| over the BF16 input [P2 §四, quantize records max(abs(x))] — taken on the
 * unscaled input. Computed as the largest magnitude bit pattern (bits & 0x7FFF), which orders
 * non-negative BF16 values exactly and puts NaN above infinity; a NaN result is 0x7FC0.
 * The amax slot is max-accumulated: it becomes the larger of its previous content and max|x|,
 * both non-negative f32 values or NaN, compared as bit patterns (so NaN dominates).
 * Counters [P3 工程落地, 第四步 量化质量: fraction near the FP8 maximum, fraction of zeros
 * after quantisation; 梯度健康: NaN/Inf counts]:
 *   c[0] += #{ |f32(x*scale)| > FP8 max }   (infinite products included, NaN not)
 *   c[1] += #{ q is 0x00 or 0x80 }
 *   c[2] += #{ x is NaN or infinite }
 * scale_inv = 1 / scale (f32 division), the dequantise factor [P2 §四, dequantize].
 * ------------------------------------------------------------------------------------- */
void orc_cast_transpose_amax(const uint16_t* x, int64_t rows, int64_t cols, int fmt, float scale,
                             uint8_t* q, uint8_t* qT, float* amax_out, float* scale_inv_out,
                             uint64_t* counters)
{
    const float maxv = fmt_max(fmt);
    uint32_t amax_bits = 0;
    uint64_t nsat = 0, nzero = 0, nnonfinite = 0;
#pragma omp parallel for schedule(static) reduction(max : amax_bits) reduction(+ : nsat, nzero, nnonfinite)
    for (int64_t i = 0; i < rows; ++i) {
        for (int64_t j = 0; j < cols; ++j) {
            const uint16_t h = x[i * cols + j];
            const uint32_t m = h & 0x7FFFu;
            if (m > amax_bits) amax_bits = m;
            if (m >= 0x7F80u) nnonfinite++;
            const float prod = orc_bf16_to_f32(h) * scale;
            if (fabsf(prod) > maxv) nsat++;
            const uint8_t c = orc_fp8_encode(prod, fmt);
            if ((c & 0x7F) == 0) nzero++;
            if (q) q[i * cols + j] = c;
            if (qT) qT[j * rows + i] = c;
        }
    }
    if (amax_bits > 0x7F80u) amax_bits = 0x7FC0u;
    if (amax_out) {
        const uint32_t prev = f32_bits(*amax_out), cur = amax_bits << 16;
        *amax_out = bits_f32(prev > cur ? prev : cur);
    }
    if (scale_inv_out) *scale_inv_out = 1.0f / scale;
    if (counters) {
        counters[0] += nsat;
        counters[1] += nzero;
        counters[2] += nnonfinite;
    }
}

/* ---------------------------------------------------------------------------------------
 * Scale update [P3 核心原理: scale = (FP8_MAX / amax) / 2^margin; Delayed Scaling: record the
 * amax into a history window, choose a representative value (max of the window, or the most
 * recent entry), and use the resulting scale in the NEXT iteration].
 * Readings (pages silent): the history is shifted so entry 0 is the newest; the window
 * includes the amax just recorded; rep = 0 gives scale 1.0 (the fallback the ScalingFactor
 * sketch of [P2 §四] uses for an empty history); a NaN or infinite rep keeps the previous
 * scale; a scale that overflows f32 becomes FLT_MAX. History entries are magnitudes, and rep
 * is taken over |h| with NaN propagating. Each consumed amax entry is reset to 0 afterwards
 * (the state a step starts from: casts max-accumulate into zeroed slots).
 * ------------------------------------------------------------------------------------- */
static float mag_max(float a, float b)  /* NaN-propagating max of |a|, |b| */
{
    if (isnan(a) || isnan(b)) return NAN;
    a = fabsf(a); b = fabsf(b);
    return a > b ? a : b;
}

void orc_scale_update(int32_t n, float* amax, float* hist, int32_t H, const float* fp8_max,
                      int algo, int32_t margin, float* scale, float* scale_inv)
{
    const float pow2_neg_margin = (float)ldexp(1.0, -margin); /* exact for 0 <= margin <= 126 */
    for (int32_t t = 0; t < n; ++t) {
        float* h = hist + (int64_t)t * H;
        for (int32_t i = H - 1; i >= 1; --i) h[i] = h[i - 1];
        h[0] = amax[t];
        float rep = fabsf(h[0]);
        if (algo == ORC_AMAX_MAX)
            for (int32_t i = 1; i < H; ++i) rep = mag_max(rep, h[i]);
        float s;
        if (isnan(rep) || isinf(rep)) {
            s = scale[t];
        } else if (rep == 0.0f) {
            s = 1.0f;
        } else {
            s = fp8_max[t] / rep;
            s = s * pow2_neg_margin;
            if (isinf(s)) s = FLT_MAX;
        }
        scale[t] = s;
        scale_inv[t] = 1.0f / s;
        amax[t] = 0.0f;
    }
}

/* ---------------------------------------------------------------------------------------
 * Per-tensor scaled FP8 GEMM, D = A . B^T with A: M x K, B: N x K (both row-major).
 * [P2 §三: FP8 GEMM inputs, higher-precision accumulation, 16-bit output; P2 §五: per-tensor
 *  mode, FP8 x FP8, FP32 accumulate, BF16 output; P2 §四 dequantize = divide by the scale,
 *  applied here as a multiply by the product of the two f32 scale inverses.]
 * Exactness: every finite E4M3 / E5M2 value times 2^16 is an integer of magnitude < 2^32
 * (smallest step 2^-16), so every product times 2^32 is an integer below 2^64 and the sum over
 * k is accumulated EXACTLY in a 128-bit integer. The only roundings are the final ones:
 *   y = double(acc) * 2^-32 * double(sa *f32 sb);   D = bf16_rne(float(y)).
 * Any NaN or infinite operand in a dot product makes that element's sum a plain double sum
 * (IEEE NaN/inf propagation).
 * abs_out (may be NULL) receives sum_k |a_k b_k| * sa * sb, the scale of the tolerance.
 * ------------------------------------------------------------------------------------- */
static int64_t fp8_times_2p16(uint8_t code, int fmt)
{
    const double v = orc_fp8_decode(code, fmt);   /* finite here; v * 2^16 is an integer */
    return (int64_t)ldexp(v, 16);
}

static void gemm_element(const uint8_t* a_row, int afmt, const uint8_t* b_row, int bfmt, int64_t K,
                         float alpha, uint16_t* d_out, double* abs_out)
{
    __int128 acc = 0, absacc = 0;
    int nonfinite = 0;
    for (int64_t k = 0; k < K; ++k) {
        if (!orc_fp8_is_finite(a_row[k], afmt) || !orc_fp8_is_finite(b_row[k], bfmt)) {
            nonfinite = 1;
            break;
        }
        const __int128 p = (__int128)fp8_times_2p16(a_row[k], afmt) * fp8_times_2p16(b_row[k], bfmt);
        acc += p;
        absacc += p < 0 ? -p : p;
    }
    double y, yabs;
    if (nonfinite) {
        double s = 0.0, sa = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            const double p = orc_fp8_decode(a_row[k], afmt) * orc_fp8_decode(b_row[k], bfmt);
            s += p;
            sa += fabs(p);
        }
        y = s * (double)alpha;
        yabs = sa * (double)alpha;
    } else {
        y = ldexp((double)acc, -32) * (double)alpha;
        yabs = ldexp((double)absacc, -32) * (double)alpha;
    }
    *d_out = orc_f32_to_bf16((float)y);
    if (abs_out) *abs_out = yabs;
}

void orc_gemm(const uint8_t* A, int afmt, const uint8_t* B, int bfmt, int64_t M, int64_t N,
              int64_t K, float a_scale_inv, float b_scale_inv, uint16_t* D, double* abs_out)
{
    const float alpha = a_scale_inv * b_scale_inv;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < M; ++i)
        for (int64_t j = 0; j < N; ++j)
            gemm_element(A + i * K, afmt, B + j * K, bfmt, K, alpha, D + i * N + j,
                         abs_out ? abs_out + i * N + j : NULL);
}

/* The same GEMM at chosen output positions (ii[s], jj[s]) only. */
void orc_gemm_at(const uint8_t* A, int afmt, const uint8_t* B, int bfmt, int64_t K,
                 float a_scale_inv, float b_scale_inv, int64_t n, const int64_t* ii,
                 const int64_t* jj, uint16_t* out, double* abs_out)
{
    const float alpha = a_scale_inv * b_scale_inv;
#pragma omp parallel for schedule(static)
    for (int64_t s = 0; s < n; ++s)
        gemm_element(A + ii[s] * K, afmt, B + jj[s] * K, bfmt, K, alpha, out + s,
                     abs_out ? abs_out + s : NULL);
}

/* ---------------------------------------------------------------------------------------
 * Global gradient norm for clipping [P1 FP8 训练主路径图: unscale / clip before the fused
 * optimizer; P2 §四: gradients of the loss-scaled loss are divided by the loss scale].
 * Reading (pages give no formula): G = sum of f32(g)^2 in double over every element; each
 * tensor is cut into fixed chunks of 65,536 elements, each chunk summed in order, and the chunk
 * sums (tensor by tensor, chunk by chunk) combined by pairwise summation; norm =
 * float(sqrt(G) * (1 / loss_scale)), the norm of the unscaled gradient. (Any FP64 order agrees
 * to far below an f32 ulp here; this one is fixed, so it does not depend on the thread count.)
 * ------------------------------------------------------------------------------------- */
#define ORC_NORM_CHUNK 65536

static double pairwise_sum(const double* v, int64_t n)
{
    if (n == 1) return v[0];
    const int64_t h = n / 2;
    return pairwise_sum(v, h) + pairwise_sum(v + h, n - h);
}

float orc_global_norm(int32_t n, const uint16_t* const* grads, const int64_t* numel,
                      float loss_scale)
{
    int64_t nchunks = 0;
    for (int32_t t = 0; t < n; ++t) nchunks += (numel[t] + ORC_NORM_CHUNK - 1) / ORC_NORM_CHUNK;
    if (nchunks == 0) return 0.0f;
    double* part = (double*)malloc((size_t)nchunks * sizeof(double));
    int64_t* tens = (int64_t*)malloc((size_t)nchunks * sizeof(int64_t));
    int64_t* first = (int64_t*)malloc((size_t)nchunks * sizeof(int64_t));
    int64_t c = 0;
    for (int32_t t = 0; t < n; ++t)
        for (int64_t i = 0; i < numel[t]; i += ORC_NORM_CHUNK) {
            tens[c] = t;
            first[c++] = i;
        }
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t k = 0; k < nchunks; ++k) {
        const int64_t t = tens[k], i0 = first[k];
        const int64_t i1 = i0 + ORC_NORM_CHUNK < numel[t] ? i0 + ORC_NORM_CHUNK : numel[t];
        double acc = 0.0;
        for (int64_t i = i0; i < i1; ++i) {
            const double g = (double)orc_bf16_to_f32(grads[t][i]);
            acc += g * g;
        }
        part[k] = acc;
    }
    const double G = pairwise_sum(part, nchunks);
    free(part);
    free(tens);
    free(first);
    return (float)(sqrt(G) * (1.0 / (double)loss_scale));
}

/* ---------------------------------------------------------------------------------------
 * AdamW update given the global norm [P1 Fused Optimizer 的意义: read the gradient, update the
 * first and second moments, bias correction, weight decay, parameter update — in that order;
 * P1 FP8 与优化器之间的精度分层 and P2 §三 recipe table: FP32 optimizer state; P2 §四: FP32
 * optimizer step after gradient un-scaling].
 * Readings (pages give no formula): decoupled weight decay p *= (1 - lr*wd) applied before the
 * Adam step; eps added after the bias-corrected square root; clip coefficient max/norm when the
 * unscaled norm exceeds max (max <= 0: no clip); a non-finite norm skips the whole update.
 * Host scalars are formed in double and rounded once to f32; each per-element operation is one
 * f32 operation rounded to nearest (no fused multiply-add).
 * Returns 1 if the update was skipped, else 0.
 * ------------------------------------------------------------------------------------- */
int orc_adamw_update(int32_t n, float* const* master, float* const* m, float* const* v,
                     const uint16_t* const* g, uint16_t* const* w, const int64_t* numel,
                     float lr, float beta1, float beta2, float eps, float wd, int64_t step,
                     float loss_scale, float max_norm, float norm)
{
    if (!isfinite(norm)) return 1;
    const float coef = (max_norm > 0.0f && norm > max_norm) ? max_norm / norm : 1.0f;
    const float inv_s = (float)(1.0 / (double)loss_scale);
    const float f = coef * inv_s;
    const float omb1 = (float)(1.0 - (double)beta1);
    const float omb2 = (float)(1.0 - (double)beta2);
    const float decay = (float)(1.0 - (double)lr * (double)wd);
    const float step_size = (float)((double)lr / (1.0 - pow((double)beta1, (double)step)));
    const float bc2_sqrt = (float)sqrt(1.0 - pow((double)beta2, (double)step));
    for (int32_t t = 0; t < n; ++t) {
#pragma omp parallel for schedule(static)
        for (int64_t i = 0; i < numel[t]; ++i) {
            const float gg = orc_bf16_to_f32(g[t][i]) * f;
            const float mm = beta1 * m[t][i] + omb1 * gg;
            const float vv = beta2 * v[t][i] + omb2 * (gg * gg);
            float p = master[t][i] * decay;
            const float denom = sqrtf(vv) / bc2_sqrt + eps;
            p = p - step_size * (mm / denom);
            m[t][i] = mm;
            v[t][i] = vv;
            master[t][i] = p;
            if (w) w[t][i] = orc_f32_to_bf16(p);
        }
    }
    return 0;
}

/* Norm, then update: the whole fused AdamW call. Returns 1 if skipped. */
int orc_fused_adamw(int32_t n, float* const* master, float* const* m, float* const* v,
                    const uint16_t* const* g, uint16_t* const* w, const int64_t* numel, float lr,
                    float beta1, float beta2, float eps, float wd, int64_t step, float loss_scale,
                    float max_norm, float* norm_out)
{
    const float norm = orc_global_norm(n, g, numel, loss_scale);
    if (norm_out) *norm_out = norm;
    return orc_adamw_update(n, master, m, v, g, w, numel, lr, beta1, beta2, eps, wd, step,
                            loss_scale, max_norm, norm);
}

/* ---------------------------------------------------------------------------------------
 * MXFP8 block scaling [P2 §九, Blackwell Microscaling: groups of 32 values share one 8-bit
 * E8M0 scale, each value stored as FP8; P2 §三, "为什么权重梯度用 E5M2": micro scaling with
 * E4M3 elements is the Blackwell direction for gradients too].
 *
 * Readings (the pages fix the block size, the scale type and the element type only):
 *   - E8M0 (8 exponent bits, no sign or mantissa) is 2^(code - 127); code 0xFF is NaN. (The
 *     page's "FP32 scale per 32 elements" line contradicts its own E8M0 diagram; the diagram is
 *     taken.)
 *   - A block is 32 consecutive values along the contraction dimension: along a row for the
 *     row-wise copy, down a column for the column-wise copy (the 32 x 32 "sub-block" wording of
 *     §三 is read as this 1 x 32 grouping, which is what the diagram shows).
 *   - The shared exponent follows the published MX rule: X = floor(log2(amax)) - emax, emax the
 *     exponent of the element format's largest value (8 for E4M3, 448 = 1.75 * 2^8; 15 for
 *     E5M2), clamped to [-127, 127]; elements are encode(f32(x) * 2^-X) with the same
 *     round-to-nearest-even and saturation as the per-tensor cast, so the top of a block may
 *     saturate (values in [448, 512) * 2^X become 448 * 2^X).
 *   - amax = 0: X = -127 (all elements are zero). amax = +inf: X = 127. A NaN in the block:
 *     scale code 0xFF and the elements encoded with X = 0.
 * ------------------------------------------------------------------------------------- */
double orc_e8m0_decode(uint8_t code)
{
    if (code == 0xFF) return NAN;
    return ldexp(1.0, (int)code - 127);
}

/* floor(log2(|v|)) of a non-zero finite BF16 magnitude pattern (normal or subnormal). */
static int bf16_floor_log2(uint16_t mag)
{
    const int e = (mag >> 7) & 0xFF;
    if (e) return e - 127;
    int top = 6;                                   /* subnormal: m * 2^-133, m < 128 */
    while (!((mag >> top) & 1)) --top;
    return top - 133;
}

static uint8_t mx_block(const uint16_t* x, int64_t stride, int fmt, uint8_t* q, int64_t qstride)
{
    uint16_t amax = 0;
    for (int i = 0; i < 32; ++i) {
        const uint16_t m = x[i * stride] & 0x7FFF;
        if (m > amax) amax = m;                    /* NaN patterns sort above infinity */
    }
    int X;
    uint8_t code;
    if (amax > 0x7F80) {                           /* NaN in the block */
        X = 0;
        code = 0xFF;
    } else {
        if (amax == 0) X = -127;
        else if (amax == 0x7F80) X = 127;
        else {
            X = bf16_floor_log2(amax) - (fmt == ORC_E4M3 ? 8 : 15);
            if (X < -127) X = -127;
            if (X > 127) X = 127;
        }
        code = (uint8_t)(X + 127);
    }
    const float inv = (float)ldexp(1.0, -X);      /* exact power of two in f32 */
    for (int i = 0; i < 32; ++i)
        q[i * qstride] = orc_fp8_encode(orc_bf16_to_f32(x[i * stride]) * inv, fmt);
    return code;
}

/* MX quantisation of a BF16 matrix x [rows x cols]. axis 0: blocks of 32 consecutive columns
 * of a row, sf [rows x cols/32]; axis 1: blocks of 32 consecutive rows of a column, sf
 * [rows/32 x cols]. q [rows x cols] in the same layout as x either way. */
void orc_mx_quantise(const uint16_t* x, int64_t rows, int64_t cols, int axis, int fmt,
                     uint8_t* q, uint8_t* sf)
{
    if (axis == 0) {
#pragma omp parallel for schedule(static)
        for (int64_t r = 0; r < rows; ++r)
            for (int64_t b = 0; b < cols / 32; ++b)
                sf[r * (cols / 32) + b] = mx_block(x + r * cols + 32 * b, 1, fmt, q + r * cols + 32 * b, 1);
    } else {
#pragma omp parallel for schedule(static)
        for (int64_t b = 0; b < rows / 32; ++b)
            for (int64_t c = 0; c < cols; ++c)
                sf[b * cols + c] = mx_block(x + 32 * b * cols + c, cols, fmt, q + 32 * b * cols + c, cols);
    }
}

/* One output of the MX GEMM: sum over K-blocks of 2^(Xa + Xb) * sum_k a_k b_k. Each block sum
 * is exact in __int128 (FP8 values times 2^16 are integers); blocks are combined in 64-bit-
 * mantissa long double (relative error below 2^-55 of the sum of magnitudes, far inside the
 * GEMM tolerance), then rounded to f32 and BF16. NaN scales or non-finite codes fall back to a
 * plain sum with IEEE propagation. abs_out: sum |a_k b_k| 2^(Xa + Xb). */
static void mx_element(const uint8_t* a, const uint8_t* sa, int afmt, const uint8_t* b,
                       const uint8_t* sb, int bfmt, int64_t K, uint16_t* d_out, double* abs_out)
{
    long double acc = 0.0L, absacc = 0.0L;
    for (int64_t kb = 0; kb < K / 32; ++kb) {
        const double s = orc_e8m0_decode(sa[kb]) * orc_e8m0_decode(sb[kb]);
        __int128 blk = 0, babs = 0;
        int plain = isnan(s);
        for (int k = 0; k < 32 && !plain; ++k)
            if (!orc_fp8_is_finite(a[32 * kb + k], afmt) || !orc_fp8_is_finite(b[32 * kb + k], bfmt))
                plain = 1;
        if (plain) {
            for (int k = 0; k < 32; ++k) {
                const double p = orc_fp8_decode(a[32 * kb + k], afmt) * orc_fp8_decode(b[32 * kb + k], bfmt);
                acc += (long double)p * s;
                absacc += fabsl((long double)p * s);
            }
            continue;
        }
        for (int k = 0; k < 32; ++k) {
            const __int128 p = (__int128)fp8_times_2p16(a[32 * kb + k], afmt) *
                               fp8_times_2p16(b[32 * kb + k], bfmt);
            blk += p;
            babs += p < 0 ? -p : p;
        }
        const int e = ((int)sa[kb] - 127) + ((int)sb[kb] - 127) - 32;
        acc += ldexpl((long double)blk, e);
        absacc += ldexpl((long double)babs, e);
    }
    *d_out = orc_f32_to_bf16((float)(double)acc);
    if (abs_out) *abs_out = (double)absacc;
}

/* D [M x N] = bf16(A . B^T) with block scales: A [M x K] and B [N x K] codes (K contiguous),
 * sfa [M x K/32], sfb [N x K/32]. */
void orc_mx_gemm(const uint8_t* A, const uint8_t* sfa, int afmt, const uint8_t* B,
                 const uint8_t* sfb, int bfmt, int64_t M, int64_t N, int64_t K, uint16_t* D,
                 double* abs_out)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < M; ++i)
        for (int64_t j = 0; j < N; ++j)
            mx_element(A + i * K, sfa + i * (K / 32), afmt, B + j * K, sfb + j * (K / 32), bfmt, K,
                       D + i * N + j, abs_out ? abs_out + i * N + j : NULL);
}

/* The MX GEMM at chosen output positions (ii[s], jj[s]). */
void orc_mx_gemm_at(const uint8_t* A, const uint8_t* sfa, int afmt, const uint8_t* B,
                    const uint8_t* sfb, int bfmt, int64_t K, int64_t n, const int64_t* ii,
                    const int64_t* jj, uint16_t* out, double* abs_out)
{
#pragma omp parallel for schedule(static)
    for (int64_t s = 0; s < n; ++s)
        mx_element(A + ii[s] * K, sfa + ii[s] * (K / 32), afmt, B + jj[s] * K, sfb + jj[s] * (K / 32),
                   bfmt, K, out + s, abs_out ? abs_out + s : NULL);
}
