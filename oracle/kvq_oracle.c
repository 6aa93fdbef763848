/*
 * kvq_oracle.c -- plain, slow CPU oracle for blockwise NVFP4 KV-cache quantization.
 *
 * TEST INFRASTRUCTURE ONLY. This file is the yardstick the CUDA library is checked
 * against. Only the tests, the package smoke check and the benchmark's timed CPU
 * baseline load it. It shares no code, header, table or constant with the CUDA path,
 * and the CUDA path never loads it.
 *
 * Sources (web pages, cited by title and section):
 *   [NVFP4]  "How NVFP4 Quantization Works in LongLive 2.0 for Transformer Inference"
 *            sections "Understanding the NVFP4 Format and Architecture",
 *            "Stage 1: Weight Quantization (FP32 to NVFP4)",
 *            "Stage 3: KV-Cache De-quantization at Inference", FAQ.
 *   [CFG]    "How to Use KV Cache Quantization with LongLive's LongLiveQuantizationConfig"
 *            sections "FP4 Quantization in the Causal Model", "CUDA De-quantization
 *            Pipeline", "Configuration Parameters Reference".
 *   [STUDY]  "KV Cache Quantization for Self-Forcing Video Generation: A 33-Method
 *            Empirical Study", appendix Table 3 (block size 16, quantize-on-write,
 *            dequantize the active cache before attention).
 *
 * Everything is IEEE binary32 with round-to-nearest-even, one operation at a time, in
 * the order written here. Build with -ffp-contract=off and without fast-math: the
 * only fused operations are the explicit fmaf() calls of the mse error (rule 5).
 *
 * Readings taken where the pages are silent or garbled (each one is listed in the
 * design notes):
 *   - values are FP4 e2m1 (max 6); block scales are FP8 e4m3 (max 448); [NVFP4] calls
 *     the value format "e4m3" but also gives amax/6 and two values per byte, which
 *     only e2m1 satisfies.
 *   - a block is 16 consecutive elements of a row (along head_dim).
 *   - the global scale is gs = amax_t / (6 * 448), amax_t over the quantized tensor
 *     (or over one appended chunk of a cache).
 *   - block scale code c = e4m3((amax_b / R) / gs), saturating at 448;
 *     S = e4m3_value(c) * gs; values are x * (1/S) rounded to e2m1 (nearest, ties to
 *     the even code, saturating at 6, sign kept, so negative values that round to
 *     zero give code 0x8). When 1/S is infinite (S == 0) every product is x * 0.
 *   - rule mse keeps R = 4 only when its squared error is strictly smaller than R = 6's.
 *     The pages fix no evaluation order for that error; the order used (block_sq_error)
 *     is pinned by hand-worked near-tie blocks and an exact-rational restatement of
 *     the quantizer in the tests.
 *   - the even-indexed element of a pair goes in the low nibble.
 *   - dequant: y = bf16_rne(e2m1_value(q) * S), the product rounded to fp32 first.
 *
 * The RTN integer codecs of [STUDY] appendix Table 3 (RTN_INT4, RTN_INT2, and K2_V4 =
 * INT2 keys with INT4 values) are restated at the end of the file, with their readings.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_BLOCK 16

enum { ORC_RULE_STATIC_6 = 0, ORC_RULE_STATIC_4 = 1, ORC_RULE_MSE = 2 };
enum { ORC_OK = 0, ORC_ERR_ARG = 1, ORC_ERR_CAPACITY = 4 };

/* ---------------------------------------------------------------- formats */

/* FP4 e2m1 magnitude of a 3-bit field: 2 exponent bits, 1 mantissa bit, bias 1,
 * exponent field 0 is subnormal. [NVFP4] "Understanding the NVFP4 Format": the
 * largest magnitude is 6 (scale = amax / 6.0). */
static double e2m1_magnitude(int field3)
{
    int e = (field3 >> 1) & 3, m = field3 & 1;
    if (e == 0)
        return m * 0.5;
    return (1.0 + 0.5 * m) * ldexp(1.0, e - 1);
}

double orc_e2m1_decode(uint8_t nibble)
{
    double mag = e2m1_magnitude(nibble & 7);
    return (nibble & 8) ? -mag : mag;
}

/* Nearest e2m1 magnitude, ties to the even field (mantissa bit 0), saturating at 6.
 * The sign bit is the sign of v, also when the magnitude rounds to 0. */
uint8_t orc_e2m1_encode(float v)
{
    double a = fabs((double)v);
    int best = 7; /* anything above 6 (and +inf) saturates to the largest magnitude */
    if (a <= 6.0) {
        double best_d = INFINITY;
        for (int f = 0; f < 8; ++f) {
            double d = fabs(a - e2m1_magnitude(f));
            if (d < best_d || (d == best_d && (f & 1) == 0 && (best & 1) == 1)) {
                best_d = d;
                best = f;
            }
        }
    }
    return (uint8_t)((signbit(v) ? 8 : 0) | best);
}

/* FP8 e4m3 (the "fn" variant: no infinities; 0x7F/0xFF are NaN): 4 exponent bits,
 * bias 7, 3 mantissa bits, exponent field 0 subnormal (step 2^-9), max 448.
 * [NVFP4] "Understanding the NVFP4 Format": block scales quantized to FP8 e4m3. */
static double e4m3_magnitude(int field7)
{
    int e = (field7 >> 3) & 15, m = field7 & 7;
    if (e == 0)
        return m * ldexp(1.0, -9);
    return (1.0 + m / 8.0) * ldexp(1.0, e - 7);
}

double orc_e4m3_decode(uint8_t code)
{
    if ((code & 0x7F) == 0x7F)
        return NAN;
    double mag = e4m3_magnitude(code & 0x7F);
    return (code & 0x80) ? -mag : mag;
}

/* Nearest finite e4m3 value, ties to the even code, saturating at 448. Inputs of the
 * method are >= 0; a negative input gets the sign bit. */
uint8_t orc_e4m3_encode(float r)
{
    double a = fabs((double)r);
    int f;
    if (!(a < 448.0)) {
        f = 126; /* 448 and above, +inf included: saturate */
    } else {
        /* largest field lo with magnitude(lo) <= a (magnitudes increase with the field) */
        int lo = 0, hi = 126;
        while (lo < hi) {
            int mid = (lo + hi + 1) / 2;
            if (e4m3_magnitude(mid) <= a)
                lo = mid;
            else
                hi = mid - 1;
        }
        f = lo;
        if (lo < 126) {
            double dlo = a - e4m3_magnitude(lo), dhi = e4m3_magnitude(lo + 1) - a;
            if (dhi < dlo || (dhi == dlo && ((lo + 1) & 1) == 0))
                f = lo + 1;
        }
    }
    return (uint8_t)((signbit(r) ? 0x80 : 0) | f);
}

/* bf16 <-> fp32. bf16 is the upper half of an fp32; widening is exact. */
static float bf16_to_f32(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* Round an fp32 to bf16, nearest with ties to even (inputs are finite). */
uint16_t orc_bf16_rne(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    uint32_t keep = u >> 16, rest = u & 0xFFFFu;
    if (rest > 0x8000u || (rest == 0x8000u && (keep & 1u)))
        keep += 1;
    return (uint16_t)keep;
}

/* ---------------------------------------------------------------- one block */

/* Global scale from the tensor amax: [NVFP4] "Stage 3", global_scale = amax / (e2m1_max * e4m3_max). */
static float global_scale(float amax_t) { return amax_t / (6.0f * 448.0f); }

typedef struct {
    uint8_t c;      /* e4m3 scale code */
    uint8_t q[ORC_BLOCK];
    float S;        /* decoded block scale e4m3_value(c) * gs */
} cand_t;

/* Encode one block of 16 values under denominator R ([NVFP4] "Stage 1" steps 1-3;
 * [CFG] "Configuration Parameters Reference": the rule picks the FP4 denominator). */
static void encode_block(const float x[ORC_BLOCK], float amax_b, float gs, float R, cand_t* out)
{
    uint8_t c = 0;
    if (gs != 0.0f) {
        float s = amax_b / R; /* per-block scale, amax / R */
        float r = s / gs;     /* the block scale relative to the global scale */
        c = orc_e4m3_encode(r);
    }
    float S = (float)orc_e4m3_decode(c) * gs;
    float inv = 1.0f / S;
    if (isinf(inv))
        inv = 0.0f;
    for (int i = 0; i < ORC_BLOCK; ++i)
        out->q[i] = orc_e2m1_encode(x[i] * inv);
    out->c = c;
    out->S = S;
}

/* Squared reconstruction error of a candidate, in the fixed order of rule 5: the
 * residual x - value*S with one rounding (fmaf), squares accumulated with fmaf in two
 * interleaved partial sums (even and odd positions, in index order), then added. */
static float block_sq_error(const float x[ORC_BLOCK], const cand_t* cd)
{
    float s_even = 0.0f, s_odd = 0.0f;
    for (int i = 0; i < ORC_BLOCK; ++i) {
        float val = (float)orc_e2m1_decode(cd->q[i]);
        float d = fmaf(-val, cd->S, x[i]);
        if (i & 1)
            s_odd = fmaf(d, d, s_odd);
        else
            s_even = fmaf(d, d, s_even);
    }
    return s_even + s_odd;
}

/* Quantize one block. Writes the scale code and 8 packed bytes; optionally reports
 * both candidates' errors (used by the tests' brute-force check of the mse rule). */
static void quantize_block(const uint16_t* xb, float gs, int rule, uint8_t* scale_out, uint8_t* packed_out,
                           float* err6_out, float* err4_out)
{
    float x[ORC_BLOCK], amax_b = 0.0f;
    for (int i = 0; i < ORC_BLOCK; ++i) {
        x[i] = bf16_to_f32(xb[i]);
        float a = fabsf(x[i]);
        if (a > amax_b)
            amax_b = a;
    }
    cand_t c6, c4;
    const cand_t* pick;
    if (rule == ORC_RULE_STATIC_6) {
        encode_block(x, amax_b, gs, 6.0f, &c6);
        pick = &c6;
    } else if (rule == ORC_RULE_STATIC_4) {
        encode_block(x, amax_b, gs, 4.0f, &c4);
        pick = &c4;
    } else {
        /* [CFG] "Configuration Parameters Reference": "mse" minimises the reconstruction
         * error per block; the two candidates are the denominators 6 and 4. */
        encode_block(x, amax_b, gs, 6.0f, &c6);
        encode_block(x, amax_b, gs, 4.0f, &c4);
        float e6 = block_sq_error(x, &c6), e4 = block_sq_error(x, &c4);
        if (err6_out)
            *err6_out = e6;
        if (err4_out)
            *err4_out = e4;
        pick = (e4 < e6) ? &c4 : &c6;
    }
    *scale_out = pick->c;
    /* [NVFP4] "Stage 1" step 3: two FP4 values per uint8, even element low nibble. */
    for (int j = 0; j < ORC_BLOCK / 2; ++j)
        packed_out[j] = (uint8_t)(pick->q[2 * j] | (pick->q[2 * j + 1] << 4));
}

static void dequantize_block(const uint8_t* packed, uint8_t scale, float gs, uint16_t* y)
{
    float S = (float)orc_e4m3_decode(scale) * gs;
    for (int j = 0; j < ORC_BLOCK / 2; ++j) {
        uint8_t b = packed[j];
        y[2 * j] = orc_bf16_rne((float)orc_e2m1_decode(b & 15) * S);
        y[2 * j + 1] = orc_bf16_rne((float)orc_e2m1_decode(b >> 4) * S);
    }
}

/* ---------------------------------------------------------------- threading */

typedef struct {
    int kind; /* 0 amax, 1 quantize, 2 dequantize */
    const uint16_t* x;
    const uint8_t* packed_in;
    const uint8_t* scales_in;
    uint8_t* packed;
    uint8_t* scales;
    uint16_t* y;
    int64_t b0, b1; /* block range */
    float gs;
    int rule;
    float amax; /* result of kind 0 */
} job_t;

static void* run_job(void* arg)
{
    job_t* j = (job_t*)arg;
    if (j->kind == 0) {
        float m = 0.0f;
        for (int64_t i = j->b0 * ORC_BLOCK; i < j->b1 * ORC_BLOCK; ++i) {
            float a = fabsf(bf16_to_f32(j->x[i]));
            if (a > m)
                m = a;
        }
        j->amax = m;
    } else if (j->kind == 1) {
        for (int64_t b = j->b0; b < j->b1; ++b)
            quantize_block(j->x + b * ORC_BLOCK, j->gs, j->rule, j->scales + b, j->packed + b * (ORC_BLOCK / 2),
                           NULL, NULL);
    } else {
        for (int64_t b = j->b0; b < j->b1; ++b)
            dequantize_block(j->packed_in + b * (ORC_BLOCK / 2), j->scales_in[b], j->gs, j->y + b * ORC_BLOCK);
    }
    return NULL;
}

/* Split blocks [0, nb) into nthreads contiguous ranges. Blocks are independent and the
 * max is order-free, so the result does not depend on the thread count. */
static void run_parallel(job_t proto, int64_t nb, int nthreads, float* amax_result)
{
    if (nthreads < 1)
        nthreads = 1;
    if ((int64_t)nthreads > nb)
        nthreads = nb > 0 ? (int)nb : 1;
    job_t* jobs = (job_t*)calloc((size_t)nthreads, sizeof(job_t));
    pthread_t* th = (pthread_t*)calloc((size_t)nthreads, sizeof(pthread_t));
    for (int t = 0; t < nthreads; ++t) {
        jobs[t] = proto;
        jobs[t].b0 = nb * t / nthreads;
        jobs[t].b1 = nb * (t + 1) / nthreads;
    }
    for (int t = 1; t < nthreads; ++t)
        pthread_create(&th[t], NULL, run_job, &jobs[t]);
    run_job(&jobs[0]);
    for (int t = 1; t < nthreads; ++t)
        pthread_join(th[t], NULL);
    if (amax_result) {
        float m = 0.0f;
        for (int t = 0; t < nthreads; ++t)
            if (jobs[t].amax > m)
                m = jobs[t].amax;
        *amax_result = m;
    }
    free(jobs);
    free(th);
}

/* ---------------------------------------------------------------- tensor API */

/* Global amax of a bf16 tensor, max |x| in fp32 ([NVFP4] "Stage 1" step 4). */
float orc_amax(const uint16_t* x, int64_t n, int nthreads)
{
    if (n <= 0)
        return 0.0f;
    job_t p = {0};
    p.kind = 0;
    p.x = x;
    float m = 0.0f;
    run_parallel(p, n / ORC_BLOCK, nthreads, &m);
    return m;
}

static int check_shape(int64_t n, int32_t head_dim)
{
    if (n < 0 || head_dim <= 0 || head_dim % ORC_BLOCK != 0 || n % head_dim != 0)
        return ORC_ERR_ARG;
    return ORC_OK;
}

/* Quantize a bf16 tensor of n elements (rows of head_dim). amax_in may be NULL, in
 * which case the amax of the tensor is computed. amax_out receives the amax used. */
int orc_quantize(const uint16_t* x, int64_t n, int32_t head_dim, int32_t rule, const float* amax_in,
                 float* amax_out, uint8_t* packed, uint8_t* scales, int32_t nthreads)
{
    if (check_shape(n, head_dim) != ORC_OK || rule < 0 || rule > 2)
        return ORC_ERR_ARG;
    float amax_t = amax_in ? *amax_in : orc_amax(x, n, nthreads);
    if (amax_out)
        *amax_out = amax_t;
    job_t p = {0};
    p.kind = 1;
    p.x = x;
    p.packed = packed;
    p.scales = scales;
    p.gs = global_scale(amax_t);
    p.rule = rule;
    run_parallel(p, n / ORC_BLOCK, nthreads, NULL);
    return ORC_OK;
}

/* One block in detail, for the tests: the chosen scale code and packed bytes under
 * the given amax_t, and (rule mse) both candidates' squared errors. */
int orc_quantize_block_detail(const uint16_t* x16, float amax_t, int32_t rule, uint8_t* scale, uint8_t* packed8,
                              float* err6, float* err4)
{
    if (rule < 0 || rule > 2)
        return ORC_ERR_ARG;
    quantize_block(x16, global_scale(amax_t), rule, scale, packed8, err6, err4);
    return ORC_OK;
}

int orc_dequantize(const uint8_t* packed, const uint8_t* scales, float amax_t, int64_t n, int32_t head_dim,
                   uint16_t* y, int32_t nthreads)
{
    if (check_shape(n, head_dim) != ORC_OK)
        return ORC_ERR_ARG;
    job_t p = {0};
    p.kind = 2;
    p.packed_in = packed;
    p.scales_in = scales;
    p.y = y;
    p.gs = global_scale(amax_t);
    run_parallel(p, n / ORC_BLOCK, nthreads, NULL);
    return ORC_OK;
}

/* ---------------------------------------------------------------- KV cache */

/* A cache for one (layer, K or V) tensor: rows of head_dim elements, token-major
 * (row = token * heads + head). Rows are grouped in chunks of rows_per_chunk; each
 * chunk holds the amax of the append that wrote it. [CFG] "FP4 Quantization in the
 * Causal Model": every new K/V block is quantized on its own; [STUDY] Table 3:
 * quantize-on-write every step. */
int orc_append(uint8_t* cache_packed, uint8_t* cache_scales, float* cache_amax, int64_t capacity_rows,
               int64_t rows_per_chunk, int32_t head_dim, int64_t row_offset, const uint16_t* x, int64_t n_rows,
               int32_t rule, int32_t nthreads)
{
    if (head_dim <= 0 || head_dim % ORC_BLOCK != 0 || rows_per_chunk <= 0 || n_rows < 0 || row_offset < 0)
        return ORC_ERR_ARG;
    if (row_offset % rows_per_chunk != 0 || n_rows > rows_per_chunk)
        return ORC_ERR_ARG;
    if (row_offset + n_rows > capacity_rows)
        return ORC_ERR_CAPACITY;
    if (n_rows == 0)
        return ORC_OK;
    int64_t e0 = row_offset * head_dim;
    return orc_quantize(x, n_rows * head_dim, head_dim, rule, NULL, &cache_amax[row_offset / rows_per_chunk],
                        cache_packed + e0 / 2, cache_scales + e0 / ORC_BLOCK, nthreads);
}

/* Dequantize cache rows [row_begin, row_end) into y (row-major, same order). */
int orc_dequantize_cache(const uint8_t* cache_packed, const uint8_t* cache_scales, const float* cache_amax,
                         int64_t capacity_rows, int64_t rows_per_chunk, int32_t head_dim, int64_t row_begin,
                         int64_t row_end, uint16_t* y, int32_t nthreads)
{
    if (head_dim <= 0 || head_dim % ORC_BLOCK != 0 || rows_per_chunk <= 0 || row_begin < 0 ||
        row_end < row_begin)
        return ORC_ERR_ARG;
    if (row_end > capacity_rows)
        return ORC_ERR_CAPACITY;
    int64_t r = row_begin;
    while (r < row_end) {
        int64_t chunk = r / rows_per_chunk;
        int64_t stop = (chunk + 1) * rows_per_chunk;
        if (stop > row_end)
            stop = row_end;
        int64_t e0 = r * head_dim;
        int rc = orc_dequantize(cache_packed + e0 / 2, cache_scales + e0 / ORC_BLOCK, cache_amax[chunk],
                                (stop - r) * head_dim, head_dim, y + (r - row_begin) * head_dim, nthreads);
        if (rc != ORC_OK)
            return rc;
        r = stop;
    }
    return ORC_OK;
}

/* Bytes of a cache for `layers` layers x {K, V}: 4 bits per element, one e4m3 byte per
 * 16 elements, one fp32 amax per chunk of tokens_per_chunk tokens. [NVFP4] FAQ: packed
 * 4-bit values plus per-block scales plus a global amax; [STUDY] Figure 6: compressed
 * versus BF16-equivalent footprint. */
int orc_cache_bytes(int32_t layers, int32_t heads, int64_t capacity_tokens, int32_t head_dim,
                    int64_t tokens_per_chunk, uint64_t out[3])
{
    if (layers <= 0 || heads <= 0 || capacity_tokens < 0 || head_dim <= 0 || head_dim % ORC_BLOCK != 0 ||
        tokens_per_chunk <= 0)
        return ORC_ERR_ARG;
    uint64_t tensors = (uint64_t)layers * 2u;
    uint64_t elems = (uint64_t)capacity_tokens * (uint64_t)heads * (uint64_t)head_dim;
    uint64_t chunks = ((uint64_t)capacity_tokens + (uint64_t)tokens_per_chunk - 1) / (uint64_t)tokens_per_chunk;
    out[0] = tensors * (elems / 2);
    out[1] = tensors * (elems / ORC_BLOCK);
    out[2] = tensors * chunks * 4u;
    return ORC_OK;
}

/* ---------------------------------------------------------------- RTN integer codecs */

/* [STUDY] appendix Table 3: "symmetric blockwise quantization ... block_size=16, 2-bit
 * (4-bit) packed storage plus per-block scales". Readings (listed in the design notes):
 *   - symmetric levels q in [-qmax, qmax], qmax = 2^(bits-1) - 1 (7 for INT4, 1 for INT2);
 *   - one 16-bit scale per block, stored as bf16: the study's compression column gives
 *     5.33x for RTN INT2 = 16 / (2 + 16/16), i.e. 16 scale bits per 16 values;
 *     S = bf16_rne(amax_b / qmax), the quotient in fp32;
 *   - q = clamp(round_half_even(x / S), -qmax, qmax), the quotient an IEEE fp32
 *     division by the stored scale; q = 0 when S == 0;
 *   - codes are two's complement: INT4 two per byte (even element low nibble), INT2 four
 *     per byte (element 4j + k in bits 2k..2k+1);
 *   - dequant: y = bf16_rne(q * S) (the product is exact in fp32). */
static int rtn_qmax(int bits) { return (1 << (bits - 1)) - 1; }

static void rtn_quantize_block(const uint16_t* xb, int bits, uint8_t* packed_out, uint16_t* scale_out)
{
    const int qmax = rtn_qmax(bits);
    float x[ORC_BLOCK], amax_b = 0.0f;
    for (int i = 0; i < ORC_BLOCK; ++i) {
        x[i] = bf16_to_f32(xb[i]);
        float a = fabsf(x[i]);
        if (a > amax_b)
            amax_b = a;
    }
    const uint16_t sb = orc_bf16_rne(amax_b / (float)qmax);
    const float S = bf16_to_f32(sb);
    int q[ORC_BLOCK];
    for (int i = 0; i < ORC_BLOCK; ++i) {
        if (S == 0.0f) {
            q[i] = 0;
            continue;
        }
        float t = nearbyintf(x[i] / S); /* round half to even (default rounding mode) */
        if (t > (float)qmax)
            t = (float)qmax;
        if (t < -(float)qmax)
            t = -(float)qmax;
        q[i] = (int)t;
    }
    *scale_out = sb;
    const int per_byte = 8 / bits, mask = (1 << bits) - 1;
    for (int j = 0; j < ORC_BLOCK / per_byte; ++j) {
        int byte = 0;
        for (int k = 0; k < per_byte; ++k)
            byte |= (q[per_byte * j + k] & mask) << (bits * k);
        packed_out[j] = (uint8_t)byte;
    }
}

static void rtn_dequantize_block(const uint8_t* packed, uint16_t scale, int bits, uint16_t* y)
{
    const float S = bf16_to_f32(scale);
    const int per_byte = 8 / bits, mask = (1 << bits) - 1;
    for (int i = 0; i < ORC_BLOCK; ++i) {
        int v = (packed[i / per_byte] >> (bits * (i % per_byte))) & mask;
        if (v >= (1 << (bits - 1)))
            v -= (1 << bits); /* two's complement */
        y[i] = orc_bf16_rne((float)v * S);
    }
}

int orc_rtn_quantize(const uint16_t* x, int64_t n, int32_t head_dim, int32_t bits, uint8_t* packed,
                     uint16_t* scales)
{
    if (check_shape(n, head_dim) != ORC_OK || (bits != 2 && bits != 4))
        return ORC_ERR_ARG;
    const int64_t bytes_per_block = ORC_BLOCK * bits / 8;
    for (int64_t b = 0; b < n / ORC_BLOCK; ++b)
        rtn_quantize_block(x + b * ORC_BLOCK, bits, packed + b * bytes_per_block, scales + b);
    return ORC_OK;
}

int orc_rtn_dequantize(const uint8_t* packed, const uint16_t* scales, int64_t n, int32_t head_dim, int32_t bits,
                       uint16_t* y)
{
    if (check_shape(n, head_dim) != ORC_OK || (bits != 2 && bits != 4))
        return ORC_ERR_ARG;
    const int64_t bytes_per_block = ORC_BLOCK * bits / 8;
    for (int64_t b = 0; b < n / ORC_BLOCK; ++b)
        rtn_dequantize_block(packed + b * bytes_per_block, scales[b], bits, y + b * ORC_BLOCK);
    return ORC_OK;
}

/* ---------------------------------------------------------------- blocked scale layout */

/* The "blocked" layout of a [rows, cols] scale matrix that block-scaled MMA operands use
 * and that [NVFP4] "Stage 3" step 1 undoes ("from_blocked"): rows padded to a multiple
 * of 128, cols to a multiple of 4, zero filled; 128 x 4 tiles of 512 bytes in row-tile
 * major order; inside a tile, scale (r, c) at byte (r % 32) * 16 + ((r % 128) / 32) * 4
 * + c % 4. */
static int64_t blocked_offset(int64_t r, int64_t c, int64_t col_tiles)
{
    return ((r / 128) * col_tiles + c / 4) * 512 + (r % 32) * 16 + ((r % 128) / 32) * 4 + (c % 4);
}

int orc_scales_to_blocked(const uint8_t* scales, int64_t rows, int32_t cols, uint8_t* blocked)
{
    if (rows < 0 || cols <= 0)
        return ORC_ERR_ARG;
    const int64_t row_tiles = (rows + 127) / 128, col_tiles = (cols + 3) / 4;
    memset(blocked, 0, (size_t)(row_tiles * col_tiles * 512));
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c)
            blocked[blocked_offset(r, c, col_tiles)] = scales[r * cols + c];
    return ORC_OK;
}

int orc_scales_from_blocked(const uint8_t* blocked, int64_t rows, int32_t cols, uint8_t* scales)
{
    if (rows < 0 || cols <= 0)
        return ORC_ERR_ARG;
    const int64_t col_tiles = (cols + 3) / 4;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c)
            scales[r * cols + c] = blocked[blocked_offset(r, c, col_tiles)];
    return ORC_OK;
}
