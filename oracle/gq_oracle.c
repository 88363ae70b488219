/*
 * gq_oracle.c -- plain, slow, single-threaded CPU oracle for per-row and
 * per-tensor int6/int8 weight quantization (STE fake-quant forward, identity
 * backward, percentile clipping, fp16 scales, int6 packing, dequant on load,
 * fp16 passthrough of small tensors).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file: it exists so that tests, the smoke check and the CPU
 * baseline leg of the benchmark can compare the CUDA library against a
 * definition a reader can check by eye.  It shares no code, header, table or
 * helper with the CUDA library.
 *
 * Sources (web pages describing the method; none prints a formula or code):
 *  - "Swiglu gating_ QAT_Residual Attention Scalin _EMA- Sliding window_
 *    Optimizations for 10min/16MB Track" (openai/parameter-golf PR #2159),
 *    list "Key Explored Modifications", items 1 (STE fake quantization),
 *    13 (int8 export), 14 (per-row / per-tensor quantization), 15 (percentile
 *    clipping), 16 (small-tensor FP16 passthrough); "Final Observed Results"
 *    (int8 export validation, i.e. the dequant round trip).
 *  - "SubSixteen v2: Int6 QAT + MLP 3x + SWA + Sliding Window"
 *    (learn-parameter-golf PR #69), "Training Techniques / Quantization"
 *    (STE QAT, bits 6) and "Other" (straight-through estimator fake
 *    quantization in the forward pass, quant_range [-31, 31]).
 *  - "Record: Unified Attention + FA3 + Legal TTT" (PR #1202),
 *    "Quantization" (int8, bits 8, scope embeddings).
 *  - "Add non-record submission: 12L 24min Vocab1792 ... Int6AWQ MixedBits"
 *    (PR #1495), "Mixed-bit quantization details" (int6 default, named
 *    tensors promoted to int8); the summary list and the Community Review
 *    (AWQ column scaling from activation statistics).
 *
 * The pages give bit widths, the int6 range and the list of features, but no
 * rounding rule, percentile definition, scale format or packing layout.  The
 * readings taken here (each one is the plainest reading that the rest of the
 * pages supports):
 *   R1 percentile clip c = k-th smallest |w| of the group, 1-indexed, no
 *      interpolation, k = min(n, max(1, ceil(p*n))) with p*n one IEEE double
 *      multiply; p in (0, 1]; p = 1 gives the absolute maximum.
 *   R2 int6 codes in [-31, 31] (the page's quant_range); int8 codes in
 *      [-127, 127] (symmetric; -128 never produced).
 *   R3 scale s32 = c / qmax, one IEEE binary32 division.  Export mode stores
 *      h = binary16 round-to-nearest-even of s32 and quantizes AND dequantizes
 *      with s = (float)h, so that the loader rebuilds the exact same weights;
 *      training mode uses s = s32.  h = +inf is a range error.
 *   R4 quantize: clip w to [-c, c], t = w / s (binary32 division), round to
 *      the nearest integer with ties to even, clamp to [-qmax, qmax].  s = 0
 *      (an all-zero group, or a scale that underflows binary16) gives q = 0.
 *   R5 dequant: w_hat = (float)q * s, one binary32 multiply; q = 0 gives +0.0.
 *      bf16 output is the round-to-nearest-even of that binary32 value.
 *   R6 int6 packing per row: 4 codes in 3 bytes, 6-bit two's complement,
 *      first code in the least significant bits, little-endian 24-bit group,
 *      a short last group zero-padded; row stride 3*ceil(cols/4) bytes.
 *      int8 packing is the code byte itself.
 *   R7 STE backward: the gradient of the fp weight is the gradient of the
 *      fake-quant weight (bitwise copy), or is added to an accumulator with
 *      one binary32 add (bf16: rounded back to nearest even).
 *   R8 bf16 input is widened exactly to binary32 and computed in binary32.
 *   R9 a group holding NaN or +-inf is outside the method; it is reported.
 *   R10 averaging of quantize-dequantize snapshots ("stochastic quantized
 *      weight averaging"): a binary32 running average a of snapshots x, the
 *      fake-quant outputs as the model holds them (bf16 widened exactly).
 *      Mean (the SWA form): with n snapshots already in a, the next one gives
 *      a' = a + (x - a) * t, t = 1 / (n + 1), each step one binary32
 *      operation; n = 0 sets a' = x.
 *   R11 exponential moving average of the snapshots: a' = d*a + c*x with
 *      c = 1 - d, each product, the difference and the sum one binary32
 *      operation (the pages give d = 0.997).
 *   R12 AWQ column scaling ("... Int6AWQ MixedBits", PR #1495: "mixed-bit
 *      int6 AWQ" export, and its Community Review: activation statistics
 *      collected for "AWQ column scaling" before post-training
 *      quantization).  The pages give no rule from the statistics to the
 *      scales, so the per-column scale vector t[cols] (binary32) is an
 *      input.  The weight is rescaled column by column in its own dtype,
 *      w'[r, c] = RN_dtype(w[r, c] * t[c]) (the product one binary32
 *      multiply; bf16 then rounded to nearest even), and w' goes through the
 *      unchanged per-row clip, scale, quantize, dequant and pack.  The
 *      activations are divided by t at inference, outside the quantizer.
 *
 * Build: plain C11, gcc -O2 -ffp-contract=off, no fast-math, SSE (never x87)
 * binary32 arithmetic, default rounding mode (round to nearest even).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { OR_OK = 0, OR_ERR_ARG = 1, OR_ERR_RANGE = 2, OR_ERR_NONFINITE = 3,
       OR_ERR_NOMEM = 4 };
enum { OR_F32 = 0, OR_BF16 = 1 };
enum { OR_AVG_MEAN = 0, OR_AVG_EMA = 1 };

/* ---------------------------------------------------------------- bits --- */

static uint32_t f32_to_bits(float x) { uint32_t u; memcpy(&u, &x, 4); return u; }
static float bits_to_f32(uint32_t u) { float x; memcpy(&x, &u, 4); return x; }

/* ------------------------------------------------- binary16 conversion --- */

/*
 * binary32 -> binary16, round to nearest, ties to even, written from the
 * IEEE 754 definition: the result is the binary16 value nearest to x; of two
 * equally near, the one with an even significand.  Subnormal results are
 * kept; magnitudes that round past 65504 give infinity.  NaN gives a quiet
 * NaN with the input's sign.
 */
uint16_t or_f32_to_f16(float x)
{
    uint32_t u = f32_to_bits(x);
    uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
    uint32_t e32 = (u >> 23) & 0xFFu;
    uint32_t frac = u & 0x7FFFFFu;

    if (e32 == 0xFFu)                      /* inf or NaN */
        return (uint16_t)(sign | 0x7C00u | (frac ? 0x0200u : 0u));
    if (e32 == 0u)                         /* zero or binary32 subnormal: */
        return sign;                       /* below 2^-126 < 2^-25 -> +-0 */

    /* x = M * 2^(E - 23) with M the 24-bit significand, E the exponent */
    uint32_t M = 0x800000u | frac;
    int E = (int)e32 - 127;

    if (E < -25)                           /* |x| < 2^-25: nearer to 0 */
        return sign;

    if (E < -14) {
        /* binary16 subnormal range: result is n * 2^-24, n in [0, 1024].
         * In units of 2^-24, |x| = M * 2^(E - 23 + 24) = M >> (-E - 1). */
        int shift = -E - 1;                /* 14 .. 24 */
        uint32_t n = M >> shift;
        uint32_t rem = M & ((1u << shift) - 1u);
        uint32_t half = 1u << (shift - 1);
        if (rem > half || (rem == half && (n & 1u)))
            n += 1u;                       /* n == 1024 encodes 2^-14 */
        return (uint16_t)(sign | n);
    }

    /* binary16 normal range: keep 11 significant bits (drop 13) */
    uint32_t n = M >> 13;
    uint32_t rem = M & 0x1FFFu;
    if (rem > 0x1000u || (rem == 0x1000u && (n & 1u)))
        n += 1u;
    if (n == 0x800u) {                     /* significand overflowed */
        n = 0x400u;
        E += 1;
    }
    if (E > 15)
        return (uint16_t)(sign | 0x7C00u);
    return (uint16_t)(sign | ((uint32_t)(E + 15) << 10) | (n & 0x3FFu));
}

/* binary16 -> binary32 (exact) */
float or_f16_to_f32(uint16_t h)
{
    uint32_t sign = (h & 0x8000u) ? 1u : 0u;
    uint32_t e = (h >> 10) & 0x1Fu;
    uint32_t m = h & 0x3FFu;
    float mag;
    if (e == 0u)
        mag = ldexpf((float)m, -24);
    else if (e == 31u)
        mag = m ? NAN : INFINITY;
    else
        mag = ldexpf((float)(0x400u | m), (int)e - 25);
    return sign ? -mag : mag;
}

/* ---------------------------------------------------- bf16 conversion --- */

/* binary32 -> bfloat16 (upper 16 bits), round to nearest, ties to even. */
uint16_t or_f32_to_bf16(float x)
{
    uint32_t u = f32_to_bits(x);
    if ((u & 0x7FFFFFFFu) > 0x7F800000u)   /* NaN -> quiet NaN */
        return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t upper = u >> 16;
    uint32_t lower = u & 0xFFFFu;
    if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u)))
        upper += 1u;                       /* a carry may reach inf: correct */
    return (uint16_t)upper;
}

float or_bf16_to_f32(uint16_t b) { return bits_to_f32((uint32_t)b << 16); }

/* ------------------------------------------------------ k from p (R1) --- */

int64_t or_k_from_p(int64_t n, double p)
{
    double prod = p * (double)n;           /* one IEEE double multiply */
    double up = ceil(prod);
    int64_t k = (int64_t)up;
    if (k < 1) k = 1;
    if (k > n) k = n;
    return k;
}

int64_t or_packed_row_bytes(int64_t cols, int qbits)
{
    if (qbits == 6) return 3 * ((cols + 3) / 4);
    if (qbits == 8) return cols;
    if (qbits == 16) return 2 * cols;
    return -1;
}

/* ------------------------------------------------ clip selection (R1) --- */

static int cmp_float_ascending(const void* a, const void* b)
{
    float x = *(const float*)a, y = *(const float*)b;
    return (x > y) - (x < y);
}

/* c = k-th smallest of |v[0..n)|, by copying the magnitudes and sorting. */
float or_kth_smallest_abs(const float* v, int64_t n, int64_t k, float* scratch)
{
    for (int64_t i = 0; i < n; ++i)
        scratch[i] = fabsf(v[i]);
    qsort(scratch, (size_t)n, sizeof(float), cmp_float_ascending);
    return scratch[k - 1];
}

/* ----------------------------------------------------- quantize (R4) --- */

/* Code of one weight w for clip c, scale s and range qmax. */
int or_quantize_one(float w, float c, float s, int qmax)
{
    if (s == 0.0f)
        return 0;
    float wc = w;                           /* clip to [-c, c] */
    if (wc > c) wc = c;
    if (wc < -c) wc = -c;
    float t = wc / s;                       /* binary32 division */
    float r = nearbyintf(t);                /* ties to even (default mode) */
    if (r > (float)qmax) r = (float)qmax;   /* clamp */
    if (r < (float)-qmax) r = (float)-qmax;
    return (int)r;
}

/* w_hat = (float)q * s (R5) */
float or_dequant_one(int q, float s) { return (float)q * s; }

/* --------------------------------------------------------- pack (R6) --- */

void or_pack6_row(const int8_t* q, int64_t cols, uint8_t* out)
{
    int64_t groups = (cols + 3) / 4;
    for (int64_t g = 0; g < groups; ++g) {
        uint32_t v = 0;
        for (int j = 0; j < 4; ++j) {
            int64_t col = 4 * g + j;
            uint32_t u = 0;
            if (col < cols)
                u = (uint32_t)q[col] & 0x3Fu;   /* 6-bit two's complement */
            v |= u << (6 * j);
        }
        out[3 * g + 0] = (uint8_t)(v & 0xFFu);
        out[3 * g + 1] = (uint8_t)((v >> 8) & 0xFFu);
        out[3 * g + 2] = (uint8_t)((v >> 16) & 0xFFu);
    }
}

void or_unpack6_row(const uint8_t* in, int64_t cols, int8_t* q)
{
    for (int64_t col = 0; col < cols; ++col) {
        int64_t g = col / 4;
        int j = (int)(col % 4);
        uint32_t v = (uint32_t)in[3 * g] | ((uint32_t)in[3 * g + 1] << 8) |
                     ((uint32_t)in[3 * g + 2] << 16);
        int u = (int)((v >> (6 * j)) & 0x3Fu);
        q[col] = (int8_t)(u >= 32 ? u - 64 : u);   /* sign-extend 6 bits */
    }
}

/* ----------------------------------------------------- element access --- */

static float load_elem(const void* base, int dtype, int64_t idx)
{
    if (dtype == OR_F32)
        return ((const float*)base)[idx];
    return or_bf16_to_f32(((const uint16_t*)base)[idx]);
}

static void store_elem(void* base, int dtype, int64_t idx, float v)
{
    if (dtype == OR_F32)
        ((float*)base)[idx] = v;
    else
        ((uint16_t*)base)[idx] = or_f32_to_bf16(v);
}

/* --------------------------------------------- one group, all outputs --- */

/*
 * Quantize one group (a row, or the whole tensor) whose elements have been
 * gathered into vals[0..n).  Writes the group's clip and scales and the codes
 * q_out[0..n).  Returns OR_OK, OR_ERR_RANGE (binary16 scale overflow) or
 * OR_ERR_NONFINITE.
 */
static int quantize_group(const float* vals, int64_t n, double p, int qmax,
                          int export_mode, float* scratch, float* clip_out,
                          float* s_out, uint16_t* h_out, int8_t* q_out)
{
    for (int64_t i = 0; i < n; ++i)
        if (!isfinite(vals[i]))
            return OR_ERR_NONFINITE;

    int64_t k = or_k_from_p(n, p);
    float c = or_kth_smallest_abs(vals, n, k, scratch);
    float s32 = c / (float)qmax;            /* R3 */
    float s = s32;
    uint16_t h = 0;
    if (export_mode) {
        h = or_f32_to_f16(s32);
        if ((h & 0x7FFFu) == 0x7C00u)
            return OR_ERR_RANGE;
        s = or_f16_to_f32(h);
    }
    *clip_out = c;
    *s_out = s;
    *h_out = h;
    for (int64_t i = 0; i < n; ++i)
        q_out[i] = (int8_t)or_quantize_one(vals[i], c, s, qmax);
    return OR_OK;
}

/*
 * Full forward for one tensor W (row-major [rows, ld], first cols used).
 *   qbits 6 or 8; per_tensor 0 (one group per row) or 1 (one group);
 *   export_mode 0 (training: fp32 scale) or 1 (export: fp16 scale).
 * Outputs (each may be NULL): clip[groups], scale_f32[groups],
 * scale_f16[groups] (export mode only), codes [rows, cols] int8,
 * dq [rows, cols] in the input dtype, packed [rows, packed_row_bytes].
 */
int or_quantize(const void* w, int dtype, int64_t rows, int64_t cols,
                int64_t ld, int qbits, int per_tensor, double p,
                int export_mode, float* clip, float* scale_f32,
                uint16_t* scale_f16, int8_t* codes, void* dq, uint8_t* packed)
{
    if (!w || rows < 0 || cols < 0 || ld < cols || !(p > 0.0 && p <= 1.0))
        return OR_ERR_ARG;
    if (qbits != 6 && qbits != 8)
        return OR_ERR_ARG;
    if (dtype != OR_F32 && dtype != OR_BF16)
        return OR_ERR_ARG;
    if (scale_f16 && !export_mode)
        return OR_ERR_ARG;
    if (rows == 0 || cols == 0)
        return OR_OK;

    int qmax = (qbits == 6) ? 31 : 127;
    int64_t gsize = per_tensor ? rows * cols : cols;
    int64_t ngroups = per_tensor ? 1 : rows;
    float* vals = (float*)malloc((size_t)gsize * sizeof(float));
    float* scratch = (float*)malloc((size_t)gsize * sizeof(float));
    int8_t* q = (int8_t*)malloc((size_t)gsize);
    if (!vals || !scratch || !q) {
        free(vals); free(scratch); free(q);
        return OR_ERR_NOMEM;
    }

    int status = OR_OK;
    int64_t prb = or_packed_row_bytes(cols, qbits);
    for (int64_t g = 0; g < ngroups && status == OR_OK; ++g) {
        int64_t r0 = per_tensor ? 0 : g;
        int64_t r1 = per_tensor ? rows : g + 1;
        for (int64_t r = r0; r < r1; ++r)
            for (int64_t col = 0; col < cols; ++col)
                vals[(r - r0) * cols + col] = load_elem(w, dtype, r * ld + col);

        float c, s;
        uint16_t h;
        status = quantize_group(vals, gsize, p, qmax, export_mode, scratch,
                                &c, &s, &h, q);
        if (status != OR_OK)
            break;
        if (clip) clip[g] = c;
        if (scale_f32) scale_f32[g] = s;
        if (scale_f16) scale_f16[g] = h;

        for (int64_t r = r0; r < r1; ++r) {
            const int8_t* qr = q + (r - r0) * cols;
            if (codes)
                memcpy(codes + r * cols, qr, (size_t)cols);
            if (dq)
                for (int64_t col = 0; col < cols; ++col)
                    store_elem(dq, dtype, r * cols + col,
                               or_dequant_one(qr[col], s));
            if (packed) {
                if (qbits == 6)
                    or_pack6_row(qr, cols, packed + r * prb);
                else
                    for (int64_t col = 0; col < cols; ++col)
                        packed[r * prb + col] = (uint8_t)qr[col];
            }
        }
    }
    free(vals);
    free(scratch);
    free(q);
    return status;
}

/*
 * Dequant on load: rebuild w_hat [rows, cols] from packed codes and binary16
 * scales (scale_f16[rows], or scale_f16[0] when per_tensor).
 */
int or_dequant(const uint8_t* packed, const uint16_t* scale_f16, int qbits,
               int per_tensor, int64_t rows, int64_t cols, void* out,
               int out_dtype)
{
    if (!packed || !scale_f16 || !out || rows < 0 || cols < 0)
        return OR_ERR_ARG;
    if (qbits != 6 && qbits != 8)
        return OR_ERR_ARG;
    if (out_dtype != OR_F32 && out_dtype != OR_BF16)
        return OR_ERR_ARG;
    int64_t prb = or_packed_row_bytes(cols, qbits);
    int8_t* q = (int8_t*)malloc((size_t)(cols > 0 ? cols : 1));
    if (!q)
        return OR_ERR_NOMEM;
    for (int64_t r = 0; r < rows; ++r) {
        float s = or_f16_to_f32(scale_f16[per_tensor ? 0 : r]);
        if (qbits == 6)
            or_unpack6_row(packed + r * prb, cols, q);
        else
            for (int64_t col = 0; col < cols; ++col)
                q[col] = (int8_t)packed[r * prb + col];
        for (int64_t col = 0; col < cols; ++col)
            store_elem(out, out_dtype, r * cols + col, or_dequant_one(q[col], s));
    }
    free(q);
    return OR_OK;
}

/* STE backward (R7): g_w = g_out, or g_w = g_w + g_out. */
int or_ste_bwd(const void* g_out, void* g_w, int dtype, int64_t numel,
               int accumulate)
{
    if (!g_out || !g_w || numel < 0)
        return OR_ERR_ARG;
    if (dtype != OR_F32 && dtype != OR_BF16)
        return OR_ERR_ARG;
    for (int64_t i = 0; i < numel; ++i) {
        if (!accumulate) {
            if (dtype == OR_F32)
                ((float*)g_w)[i] = ((const float*)g_out)[i];
            else
                ((uint16_t*)g_w)[i] = ((const uint16_t*)g_out)[i];
        } else {
            float a = load_elem(g_w, dtype, i);
            float b = load_elem(g_out, dtype, i);
            store_elem(g_w, dtype, i, a + b);
        }
    }
    return OR_OK;
}

/* ------------------------------------------------- snapshot averaging --- */

/*
 * Running average of quantize-dequantize snapshots, in place (R10, R11).
 * Sources: "Record: Unified Attention + FA3 + Legal TTT" (PR #1202), Novel
 * Contributions (stochastic quantized weight averaging of
 * quantize-dequantize snapshots); "SubSixteen v2: Int6 QAT + MLP 3x + SWA +
 * Sliding Window" (PR #69), Weight Averaging (EMA decay 0.997; SWA every 50
 * steps after 20 % of training).
 */
int or_average_update(float* a, const void* x, int dtype, int64_t numel, int kind,
                      int64_t count, float decay)
{
    if (!a || !x || numel < 0)
        return OR_ERR_ARG;
    if (dtype != OR_F32 && dtype != OR_BF16)
        return OR_ERR_ARG;
    if (kind == OR_AVG_MEAN) {
        if (count < 0 || count >= (1 << 24))       /* n + 1 exact in binary32 */
            return OR_ERR_ARG;
        float t = 1.0f / (float)(count + 1);
        for (int64_t i = 0; i < numel; ++i) {
            float xi = load_elem(x, dtype, i);
            if (count == 0) {
                a[i] = xi;
            } else {
                float e = xi - a[i];
                float u = e * t;
                a[i] = a[i] + u;
            }
        }
        return OR_OK;
    }
    if (kind == OR_AVG_EMA) {
        if (!(decay >= 0.0f && decay <= 1.0f))
            return OR_ERR_ARG;
        float c = 1.0f - decay;
        for (int64_t i = 0; i < numel; ++i) {
            float xi = load_elem(x, dtype, i);
            float kept = decay * a[i];
            float added = c * xi;
            a[i] = kept + added;
        }
        return OR_OK;
    }
    return OR_ERR_ARG;
}

/*
 * AWQ column scaling (R12): out[r, c] = RN_dtype(w[r, ld-strided] * t[c]),
 * dense [rows, cols] in the input dtype.  The result is the weight that the
 * per-row quantizer (or_quantize) then takes.
 */
int or_col_scale(const void* w, int dtype, int64_t rows, int64_t cols, int64_t ld,
                 const float* t, void* out)
{
    if (!w || !t || !out || rows < 0 || cols < 0 || ld < cols)
        return OR_ERR_ARG;
    if (dtype != OR_F32 && dtype != OR_BF16)
        return OR_ERR_ARG;
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t c = 0; c < cols; ++c) {
            float x = load_elem(w, dtype, r * ld + c);
            float y = x * t[c];                    /* one binary32 multiply */
            store_elem(out, dtype, r * cols + c, y);
        }
    }
    return OR_OK;
}

/* Small-tensor passthrough: binary16 round-to-nearest-even of each value. */
int or_passthrough_f16(const void* x, int dtype, int64_t numel, uint16_t* out)
{
    if (!x || !out || numel < 0)
        return OR_ERR_ARG;
    if (dtype != OR_F32 && dtype != OR_BF16)
        return OR_ERR_ARG;
    for (int64_t i = 0; i < numel; ++i)
        out[i] = or_f32_to_f16(load_elem(x, dtype, i));
    return OR_OK;
}

/* Array forms of the conversions, for exhaustive checks from Python. */
void or_f32_to_f16_array(const float* x, int64_t n, uint16_t* out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = or_f32_to_f16(x[i]);
}

void or_f16_to_f32_array(const uint16_t* h, int64_t n, float* out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = or_f16_to_f32(h[i]);
}

void or_f32_to_bf16_array(const float* x, int64_t n, uint16_t* out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = or_f32_to_bf16(x[i]);
}

void or_quantize_array(const float* w, int64_t n, float c, float s, int qmax,
                       int8_t* q)
{
    for (int64_t i = 0; i < n; ++i)
        q[i] = (int8_t)or_quantize_one(w[i], c, s, qmax);
}
