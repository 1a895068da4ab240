/*
 * Paged GQA decode attention: CPU ORACLE (test infrastructure only).
 *
 * This file is a plain, slow, obviously correct restatement of what the
 * paged decode path computes, in double precision.  Only the test suite,
 * the smoke check and the CPU-baseline leg of the benchmark may load it;
 * the product library never links or calls it, and it shares no code,
 * header or constant with the CUDA sources.
 *
 * Sources (the four web pages on KV caching that define the method):
 *  - "KV Cache 深度解析：显存黑洞、PagedAttention 与三路省内存方案"
 *    (d7kj.com), §一 (the attention formula softmax(Q·Kᵀ/√d)·V evaluated
 *    for the new token against the cached K/V) and §六 (the numpy
 *    KVCacheAttention.step: append k/v, score q against every cached key,
 *    subtract the max, exponentiate, normalise, weight V).
 *  - "KV Cache 深度解析", §四 (fp16 → fp8 E4M3 KV quantisation with a
 *    per-token scale to hold outliers) for the FP8 codec and scales.
 *  - k1-blog 2026-07-13 "AI", "KV Cache 量化" (FP8 and INT8 both halve the
 *    fp16 cache) and "大模型推理为何这么慢", "KV Cache量化" (INT8 among the
 *    lower-precision KV formats) for the INT8 cache.
 *  - "llm-inference-optimization" notes, §四 (the printed 4-bit group
 *    quantiser: range / 15, a zero point rounded from -min / scale, codes
 *    clamped to 0..15) and "大模型推理为何这么慢", "KV Cache量化" (a 4-bit
 *    cache is 4x smaller than fp16) for the INT4 cache.
 *  - "大模型推理为何这么慢？从内存带宽瓶颈到KV Cache优化的技术突围"
 *    (freetools), section on GQA (H query heads share G groups of K/V).
 *
 * Readings where the pages are silent:
 *  - query head h reads KV head floor(h / (Hq/Hkv))  (consecutive groups);
 *  - scale is caller supplied (1/sqrt(head_dim) on the pages);
 *  - the FP8 scale of a (token, kv head) row is absmax/448 computed in
 *    IEEE fp32, the code is E4M3(x / scale) with round-to-nearest-even and
 *    saturation to ±448, and an all-zero row has scale 0 and codes 0x00;
 *  - FP8 attention dequantises exactly: value(code) * scale, in double;
 *  - the INT8 cache follows the FP8 design: symmetric, scale = absmax/127 in
 *    IEEE fp32, code = x / scale (fp32 division) rounded to the nearest
 *    integer, ties to even, clamped to [-127, 127]; an all-zero row has scale
 *    0 and codes 0; dequantisation is code * scale in double;
 *  - the INT4 cache applies the §四 routine to each (token, kv head) row, in
 *    IEEE fp32 in the routine's order: scale = (max - min) / 15, zero =
 *    rint(-min / scale), code = clamp(rint(x / scale) + zero, 0, 15); a
 *    constant row, where the routine would divide by zero, is stored exactly
 *    (scale |min|, zero -1 / +1 / 0, codes 0); value = (code - zero) * scale
 *    in double;
 *  - the KIVI cache ("大模型推理为何这么慢", KV Cache量化: Key quantised per
 *    channel, Value per token, the newest tokens kept at full precision) runs
 *    the same routine on different groups: each channel of a full 16-token
 *    block of K (16 values), each token row of V (head_dim values); the
 *    tokens of a sequence's incomplete last block stay unquantised.
 *
 * Build: gcc -O2 -ffp-contract=off -fopenmp -shared -fPIC (no fast-math).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#include <stdlib.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Stored element types of K/V and q, as the callers of this file pass them. */
enum { ORC_F32 = 0, ORC_BF16 = 1, ORC_FP8_E4M3 = 2, ORC_INT8 = 3, ORC_INT4 = 4, ORC_F64 = 5 };

/* ---- exact widening of stored values ------------------------------------ */

/* bf16 is the upper half of an IEEE binary32: widening is exact. */
static double bf16_bits_to_double(uint16_t b) {
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/*
 * OCP 8-bit floating point, E4M3 variant: 1 sign bit, 4 exponent bits with
 * bias 7, 3 mantissa bits; no infinities; S.1111.111 is NaN; exponent field
 * 0 holds subnormals m * 2^-9.  Every finite code is exact in double.
 */
double oracle_e4m3_decode(uint8_t code) {
    int sign = (code >> 7) & 1;
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    double v;
    if (e == 0xF && m == 0x7) return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);               /* m/8 * 2^(1-7) */
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -v : v;
}

/*
 * fp32 -> E4M3, round to nearest with ties to even, saturating finite
 * overflow to ±448.  Done by comparison against the sorted positive
 * magnitudes and the exact midpoints between neighbours (every midpoint of
 * two E4M3 values has at most 5 significant bits, so it is an exact float).
 */
uint8_t oracle_e4m3_encode(float x) {
    uint8_t sign;
    float a;
    int c;
    if (isnan(x)) return 0x7F;
    sign = signbit(x) ? 0x80 : 0x00;
    a = fabsf(x);
    if (a >= 448.0f) return (uint8_t)(sign | 0x7E);
    /* largest code c (0..0x7D) with value(c) <= a: the positive codes 0..0x7E
       decode to increasing magnitudes, so bisect over them */
    {
        int lo = 0, hi = 0x7E;                   /* value(lo) <= a < value(hi) */
        while (hi - lo > 1) {
            int mid = (lo + hi) / 2;
            if (oracle_e4m3_decode((uint8_t)mid) <= (double)a)
                lo = mid;
            else
                hi = mid;
        }
        c = lo;
    }
    if (c < 0x7E) {
        double lo = oracle_e4m3_decode((uint8_t)c);
        double hi = oracle_e4m3_decode((uint8_t)(c + 1));
        double mid = 0.5 * (lo + hi);
        if ((double)a > mid)
            c = c + 1;
        else if ((double)a == mid && (c & 1))
            c = c + 1;                           /* tie: even mantissa */
    }
    return (uint8_t)(sign | c);
}

/*
 * Per-(token, kv head) quantisation of `rows` rows of length d (fp32 values,
 * already rounded to the source dtype by the caller):
 *   a = max |x|;  s = a / 448 (fp32 division);  code = E4M3(x / s) (fp32
 *   division), or s = 0 and every code 0x00 when a == 0.
 */
void oracle_quantize_rows(const float* x, int64_t rows, int32_t d,
                          uint8_t* codes, float* scales) {
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        const float* xr = x + r * d;
        float a = 0.0f, s;
        int32_t i;
        for (i = 0; i < d; ++i) {
            float v = fabsf(xr[i]);
            if (v > a) a = v;
        }
        s = a / 448.0f;
        scales[r] = (a == 0.0f) ? 0.0f : s;
        for (i = 0; i < d; ++i) {
            if (a == 0.0f) {
                codes[r * d + i] = 0x00;
            } else {
                float y = xr[i] / s;
                codes[r * d + i] = oracle_e4m3_encode(y);
            }
        }
    }
}

/*
 * INT8 quantisation of `rows` rows of length d (fp32 values, already rounded
 * to the source dtype by the caller), symmetric per (token, kv head):
 *   a = max |x|;  s = a / 127 (fp32 division);  y = x / s (fp32 division);
 *   code = the integer nearest y (ties to the even one), clamped to
 *   [-127, 127]; or s = 0 and every code 0 when a == 0.
 */
static int8_t round_half_even_clamped(float y) {
    double f = floor((double)y);
    double r = (double)y - f;                  /* exact: y and f are close */
    double n = (r > 0.5) ? f + 1.0 : (r < 0.5) ? f : (fmod(f, 2.0) == 0.0 ? f : f + 1.0);
    if (n > 127.0) n = 127.0;
    if (n < -127.0) n = -127.0;
    return (int8_t)n;
}

void oracle_quantize_rows_int8(const float* x, int64_t rows, int32_t d,
                               int8_t* codes, float* scales) {
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        const float* xr = x + r * d;
        float a = 0.0f, s;
        int32_t i;
        for (i = 0; i < d; ++i) {
            float v = fabsf(xr[i]);
            if (v > a) a = v;
        }
        s = a / 127.0f;
        scales[r] = (a == 0.0f) ? 0.0f : s;
        for (i = 0; i < d; ++i)
            codes[r * d + i] = (a == 0.0f) ? 0 : round_half_even_clamped(xr[i] / s);
    }
}

/*
 * INT4 quantisation of `rows` rows of length d ("llm-inference-optimization"
 * notes §四's routine per row).  codes: one code (0..15) per element, unpacked;
 * params: per row (scale, zero point).
 */
void oracle_quantize_rows_int4(const float* x, int64_t rows, int32_t d,
                               uint8_t* codes, float* params) {
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        const float* xr = x + r * d;
        float hi = xr[0], lo = xr[0], s, z;
        int32_t i;
        for (i = 1; i < d; ++i) {
            if (xr[i] > hi) hi = xr[i];
            if (xr[i] < lo) lo = xr[i];
        }
        if (hi == lo) {
            /* the routine's scale would be 0: store the constant exactly */
            s = fabsf(lo);
            z = lo > 0.0f ? -1.0f : (lo < 0.0f ? 1.0f : 0.0f);
            for (i = 0; i < d; ++i) codes[r * d + i] = 0;
        } else {
            float range = hi - lo;
            s = range / 15.0f;
            z = rintf(-lo / s);
            for (i = 0; i < d; ++i) {
                float q = rintf(xr[i] / s);
                float c = q + z;
                if (c < 0.0f) c = 0.0f;
                if (c > 15.0f) c = 15.0f;
                codes[r * d + i] = (uint8_t)c;
            }
        }
        params[2 * r] = s;
        params[2 * r + 1] = z;
    }
}

/*
 * The 4-bit routine on one group of n values read with a stride (the same
 * arithmetic as oracle_quantize_rows_int4, which runs it on contiguous rows).
 */
static void quantize_group_int4(const float* x, int32_t n, int64_t stride, uint8_t* codes,
                                int64_t code_stride, float* scale, float* zero) {
    float hi = x[0], lo = x[0], s, z;
    int32_t i;
    for (i = 1; i < n; ++i) {
        float v = x[i * stride];
        if (v > hi) hi = v;
        if (v < lo) lo = v;
    }
    if (hi == lo) {
        s = fabsf(lo);
        z = lo > 0.0f ? -1.0f : (lo < 0.0f ? 1.0f : 0.0f);
        for (i = 0; i < n; ++i) codes[i * code_stride] = 0;
    } else {
        float range = hi - lo;
        s = range / 15.0f;
        z = rintf(-lo / s);
        for (i = 0; i < n; ++i) {
            float q = rintf(x[i * stride] / s);
            float c = q + z;
            if (c < 0.0f) c = 0.0f;
            if (c > 15.0f) c = 15.0f;
            codes[i * code_stride] = (uint8_t)c;
        }
    }
    *scale = s;
    *zero = z;
}

/*
 * KIVI quantisation of `blocks` full blocks of one kv head each.
 *   k, v   : [blocks][16][d] fp32 (already rounded to the source dtype)
 *   k_codes, v_codes : [blocks][16][d], one code (0..15) per element
 *   k_params : [blocks][d][2]  (scale, zero) per channel over the block's 16 tokens
 *   v_params : [blocks][16][2] (scale, zero) per token row
 */
void oracle_quantize_blocks_kivi(const float* k, const float* v, int64_t blocks, int32_t d,
                                 uint8_t* k_codes, float* k_params, uint8_t* v_codes,
                                 float* v_params) {
#pragma omp parallel for schedule(static)
    for (int64_t b = 0; b < blocks; ++b) {
        const int64_t base = b * 16 * d;
        int32_t c, t;
        for (c = 0; c < d; ++c)
            quantize_group_int4(k + base + c, 16, d, k_codes + base + c, d,
                                &k_params[(b * d + c) * 2], &k_params[(b * d + c) * 2 + 1]);
        for (t = 0; t < 16; ++t)
            quantize_group_int4(v + base + (int64_t)t * d, d, 1, v_codes + base + (int64_t)t * d, 1,
                                &v_params[(b * 16 + t) * 2], &v_params[(b * 16 + t) * 2 + 1]);
    }
}

/* Value of element i of a stored row, widened to double (codes dequantised).
 * For INT4 `scales` holds (scale, zero) pairs per row. */
static double load_elem(const void* base, int dtype, int64_t idx, const float* scales,
                        int64_t scale_idx) {
    switch (dtype) {
    case ORC_F32:
        return (double)((const float*)base)[idx];
    case ORC_BF16:
        return bf16_bits_to_double(((const uint16_t*)base)[idx]);
    case ORC_INT8:
        return (double)((const int8_t*)base)[idx] * (double)scales[scale_idx];
    case ORC_F64:
        return ((const double*)base)[idx];
    case ORC_INT4:
        return ((double)((const uint8_t*)base)[idx] - (double)scales[2 * scale_idx + 1]) *
               (double)scales[2 * scale_idx];
    default:
        return oracle_e4m3_decode(((const uint8_t*)base)[idx]) * (double)scales[scale_idx];
    }
}

/*
 * Single-token GQA decode over CONTIGUOUS (unpaged) per-sequence K/V.
 *
 *   q    : [B][Hq][D] in q_dtype (F32 or BF16)
 *   k, v : [total_tokens][Hkv][D] in kv_dtype, sequence b occupying tokens
 *          [seq_offsets[b], seq_offsets[b] + lens[b])
 *   k_scale, v_scale : [total_tokens][Hkv] fp32, FP8 / INT8 only; for INT4
 *          [total_tokens][Hkv][2] (scale, zero); else NULL
 *   out  : [B][Hq][D] double
 *   weights (nullable): [B][Hq][max_len] double, the softmax weights
 *
 * For query head h of sequence b, with g = floor(h / (Hq/Hkv)):
 *   s_t = scale * sum_d q[b,h,d] * K[b,t,g,d]        t in [0, L_b)
 *   m = max_t s_t,  w_t = exp(s_t - m),  Z = sum_t w_t
 *   out[b,h,:] = sum_t (w_t / Z) * V[b,t,g,:]
 * Two passes in double, parallel over (b, h).  Returns 0, or -1 on an
 * argument it cannot evaluate (L_b < 1, Hq not a multiple of Hkv).
 */
int oracle_decode_attention(int32_t kv_dtype, int32_t q_dtype,
                            const void* q, const void* k, const void* v,
                            const float* k_scale, const float* v_scale,
                            const int64_t* seq_offsets, const int32_t* lens,
                            int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
                            int32_t head_dim, double scale,
                            double* out, double* weights, int32_t max_len) {
    int32_t group, b;
    int bad = 0;
    if (num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0) return -1;
    group = num_q_heads / num_kv_heads;
    for (b = 0; b < batch; ++b)
        if (lens[b] < 1 || (weights && lens[b] > max_len)) bad = 1;
    if (bad) return -1;

#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t bh = 0; bh < (int64_t)batch * num_q_heads; ++bh) {
        int32_t bb = (int32_t)(bh / num_q_heads);
        int32_t h = (int32_t)(bh % num_q_heads);
        int32_t g = h / group;
        int32_t L = lens[bb];
        int64_t t0 = seq_offsets[bb];
        double* s = (double*)malloc(sizeof(double) * (size_t)L);
        double* qd = (double*)malloc(sizeof(double) * (size_t)head_dim);
        double m = -INFINITY, Z = 0.0;
        int32_t t, d;
        for (d = 0; d < head_dim; ++d) {
            int64_t qi = ((int64_t)bb * num_q_heads + h) * head_dim + d;
            qd[d] = (q_dtype == ORC_F32) ? (double)((const float*)q)[qi]
                                         : bf16_bits_to_double(((const uint16_t*)q)[qi]);
        }
        /* pass 1: scores and their maximum */
        for (t = 0; t < L; ++t) {
            int64_t row = (t0 + t) * num_kv_heads + g;
            double acc = 0.0;
            for (d = 0; d < head_dim; ++d)
                acc += qd[d] * load_elem(k, kv_dtype, row * head_dim + d, k_scale, row);
            s[t] = scale * acc;
            if (s[t] > m) m = s[t];
        }
        /* pass 2: weights, normaliser, weighted sum of V */
        for (t = 0; t < L; ++t) {
            s[t] = exp(s[t] - m);
            Z += s[t];
        }
        for (d = 0; d < head_dim; ++d) out[bh * head_dim + d] = 0.0;
        for (t = 0; t < L; ++t) {
            int64_t row = (t0 + t) * num_kv_heads + g;
            double w = s[t] / Z;
            for (d = 0; d < head_dim; ++d)
                out[bh * head_dim + d] += w * load_elem(v, kv_dtype, row * head_dim + d, v_scale, row);
            if (weights) weights[bh * max_len + t] = w;
        }
        if (weights)
            for (t = L; t < max_len; ++t) weights[bh * max_len + t] = 0.0;
        free(s);
        free(qd);
    }
    return 0;
}

/* Threads the OpenMP runtime will use for the parallel loop above. */
int oracle_num_threads(void) {
    int n = 1;
#ifdef _OPENMP
#pragma omp parallel
    {
#pragma omp single
        n = omp_get_num_threads();
    }
#endif
    return n;
}

/*
 * Causal multi-query attention over CONTIGUOUS per-sequence K/V: Q query
 * tokens per sequence are the last Q tokens of its context ("KV Cache 深度解析"
 * §五 chunked prefill; speculative verification).  Query token i of sequence b
 * sits at position L_b - Q + i and attends to positions 0 .. L_b - Q + i:
 *   s_t = scale * q[b,i,h,:] . K[b,t,g,:],  t <= L_b - Q + i
 *   out[b,i,h,:] = sum_t softmax(s)_t V[b,t,g,:]
 *   q, out : [B][Q][Hq][D] (q in q_dtype, out double); K/V as oracle_decode_attention.
 * Each (b, i, h) row is evaluated exactly like oracle_decode_attention with a
 * context of L_b - Q + i + 1 tokens.  Returns -1 when some L_b < Q.
 */
int oracle_multi_query_attention(int32_t kv_dtype, int32_t q_dtype, int32_t num_query_tokens,
                                 const void* q, const void* k, const void* v,
                                 const float* k_scale, const float* v_scale,
                                 const int64_t* seq_offsets, const int32_t* lens,
                                 int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
                                 int32_t head_dim, double scale, double* out) {
    int32_t group, b;
    const int32_t Q = num_query_tokens;
    if (num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0 || Q < 1) return -1;
    group = num_q_heads / num_kv_heads;
    for (b = 0; b < batch; ++b)
        if (lens[b] < Q) return -1;

#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t row = 0; row < (int64_t)batch * Q * num_q_heads; ++row) {
        int32_t bb = (int32_t)(row / ((int64_t)Q * num_q_heads));
        int32_t i = (int32_t)((row / num_q_heads) % Q);
        int32_t h = (int32_t)(row % num_q_heads);
        int32_t g = h / group;
        int32_t L = lens[bb] - Q + i + 1;          /* keys this query token sees */
        int64_t t0 = seq_offsets[bb];
        double* s = (double*)malloc(sizeof(double) * (size_t)L);
        double* qd = (double*)malloc(sizeof(double) * (size_t)head_dim);
        double m = -INFINITY, Z = 0.0;
        int32_t t, d;
        for (d = 0; d < head_dim; ++d) {
            int64_t qi = row * head_dim + d;
            qd[d] = (q_dtype == ORC_F32) ? (double)((const float*)q)[qi]
                                         : bf16_bits_to_double(((const uint16_t*)q)[qi]);
        }
        for (t = 0; t < L; ++t) {
            int64_t r = (t0 + t) * num_kv_heads + g;
            double acc = 0.0;
            for (d = 0; d < head_dim; ++d)
                acc += qd[d] * load_elem(k, kv_dtype, r * head_dim + d, k_scale, r);
            s[t] = scale * acc;
            if (s[t] > m) m = s[t];
        }
        for (t = 0; t < L; ++t) {
            s[t] = exp(s[t] - m);
            Z += s[t];
        }
        for (d = 0; d < head_dim; ++d) out[row * head_dim + d] = 0.0;
        for (t = 0; t < L; ++t) {
            int64_t r = (t0 + t) * num_kv_heads + g;
            double w = s[t] / Z;
            for (d = 0; d < head_dim; ++d)
                out[row * head_dim + d] += w * load_elem(v, kv_dtype, r * head_dim + d, v_scale, r);
        }
        free(s);
        free(qd);
    }
    return 0;
}
