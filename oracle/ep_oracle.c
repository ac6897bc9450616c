/*
 * ep_oracle.c -- plain, slow CPU oracle for the single-GPU MoE
 * expert-parallel permutation path: dispatch layout, dispatch (BF16 copy or
 * FP8 e4m3 1x128 quantisation) and weighted combine.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the package smoke check and
 * the CPU-baseline leg of the benchmark may load this library.  The product
 * path (the CUDA library) shares no code, header, table or helper with it.
 *
 * What is computed, and where it is defined:
 *   - The stage table of "DeepEP是什麼？MoE Dispatch、Combine、All-to-all與V2架構"
 *     (yololab.net, section "MoE為什麼需要All-to-all") fixes the contract:
 *     dispatch takes tokens, top-k indices and weights and yields hidden
 *     states arranged by expert; combine takes expert outputs and routing
 *     weights and yields results in the original token order.
 *   - "DeepEP 编址服务深度对抗分析" (backyes.github.io, section 五.2) fixes the
 *     volume: each stage moves batch x top_k x hidden x sizeof(dtype), i.e.
 *     one row per (token, top-k slot).
 *   - The pages leave the exact layout open ("Dispatch Layout" in the
 *     ElasticBuffer section of the yololab page; "GEMM layout" in the V2
 *     notes).  This oracle takes the plainest reading: one flat expert-major
 *     receive buffer, experts in index order, each expert's block padded up
 *     to a multiple of block_m rows, rows inside a block in (token, slot)
 *     order; expert e lives on rank floor(e / (E/R)).
 *   - FP8: the yololab page's FP8 section asks to confirm scale granularity
 *     and format but does not state them.  Reading taken: one fp32 scale per
 *     token per 128 channels, s = amax / 448, q = e4m3(x / s) with
 *     round-to-nearest-even and saturation to +-448; amax == 0 gives s = 0
 *     and q = +0.
 *   - Combine: fp32 accumulation in slot order j = 0..k-1 with one fused
 *     multiply-add per term, then round-to-nearest-even to bf16.
 *   - FP16 rows: the yololab page lists BF16, FP16 and FP8 as the precisions
 *     to test (section Benchmark矩陣); binary16 values are widened exactly and
 *     results rounded to nearest even binary16 (formats written below from
 *     IEEE 754).
 *   - Backward (training use: the pomoai page, section 核心使用场景): the
 *     gradients of the dispatch and combine definitions above.
 *   - GEMM-ready receive layout (the V2 notes' "GEMM layout"): per-row
 *     weights, zeroed pad rows, MN-major FP8 scales.
 *
 * Parity pins (tests, not this file): every function here is checked against
 * brute-force invariants, closed forms, the OCP FP8 grid and a library cast;
 * see the test files named test_oracle_*.py.
 *
 * Build: gcc -O2 -std=c11 -fPIC -shared -ffp-contract=off (no fast-math).
 * The same source also builds with -fopenmp, only to time the oracle on all
 * host cores: the token loops of dispatch, combine and the backward then run
 * in parallel over tokens.  Every token's arithmetic is the same sequence of
 * operations either way (a token is computed by one thread), so both builds
 * give identical bytes; the layout stays serial.  Without -fopenmp the
 * pragmas are ignored.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define OR_OK 0
#define OR_ERR_ARG 1
#define OR_ERR_BAD_INDEX 5
#define OR_ERR_CAPACITY 4

/* ------------------------------------------------------------------ */
/* Number formats, written from their definitions.                     */
/* ------------------------------------------------------------------ */

/* bfloat16: the upper 16 bits of an IEEE-754 binary32 (1 sign bit,
 * 8 exponent bits, 7 fraction bits).  Widening is exact. */
float oracle_bf16_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* binary32 -> bfloat16, round to nearest, ties to even.  The 16 dropped
 * bits are compared with one half of the kept unit in the last place.  A
 * carry out of the fraction correctly bumps the exponent (and reaches
 * infinity from the largest finite values).  NaN stays NaN (made quiet). */
uint16_t oracle_f32_to_bf16_rn(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu) != 0u)
        return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t kept = u >> 16;
    uint32_t dropped = u & 0xffffu;
    if (dropped > 0x8000u || (dropped == 0x8000u && (kept & 1u)))
        kept += 1u;
    return (uint16_t)kept;
}

/* IEEE-754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction
 * bits; exponent field 0 holds zero and the subnormals m * 2^-24; field 31
 * holds the infinities (fraction 0) and NaNs.  Widening is exact. */
float oracle_fp16_to_f32(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int ex = (h >> 10) & 0x1f;
    int man = h & 0x3ff;
    double v;
    if (ex == 0x1f)
        v = man ? NAN : INFINITY;
    else if (ex == 0)
        v = ldexp((double)man, -24);
    else
        v = ldexp(1.0 + man / 1024.0, ex - 15);
    return (float)(sign ? -v : v);
}

/* binary32 -> binary16, round to nearest, ties to even.  Magnitudes are
 * rounded on the binary16 grid: spacing 2^-24 below 2^-14 (subnormals) and
 * 2^(floor(log2 a) - 10) above; a result of 2^16 or more (any a >= 65520,
 * the midpoint between 65504 and 2^16) overflows to infinity.  NaN stays NaN
 * (quiet, sign kept). */
uint16_t oracle_f32_to_fp16_rn(float f)
{
    uint16_t sign = signbit(f) ? 0x8000 : 0x0000;
    if (isnan(f))
        return (uint16_t)(sign | 0x7e00);
    double a = fabs((double)f);
    if (isinf(f))
        return (uint16_t)(sign | 0x7c00);
    double step;
    int e2 = 0;
    if (a < ldexp(1.0, -14)) {
        step = ldexp(1.0, -24);
    } else {
        (void)frexp(a, &e2);                /* a = f * 2^e2, f in [0.5, 1) */
        step = ldexp(1.0, (e2 - 1) - 10);   /* binade [2^(e2-1), 2^e2) */
    }
    double q = a / step;                    /* exact */
    double n = floor(q);
    double rem = q - n;
    if (rem > 0.5 || (rem == 0.5 && fmod(n, 2.0) != 0.0))
        n += 1.0;
    double r = n * step;
    if (r >= 65536.0)
        return (uint16_t)(sign | 0x7c00);
    if (r < ldexp(1.0, -14))                /* zero or subnormal */
        return (uint16_t)(sign | (uint16_t)(r / ldexp(1.0, -24)));
    int er = 0;
    double fr = frexp(r, &er);              /* r = fr * 2^er, fr in [0.5, 1) */
    int ex = (er - 1) + 15;
    int man = (int)((fr * 2.0 - 1.0) * 1024.0);
    return (uint16_t)(sign | (ex << 10) | man);
}

void oracle_fp16_to_f32_array(const uint16_t* h, float* v, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        v[i] = oracle_fp16_to_f32(h[i]);
}

void oracle_f32_to_fp16_array(const float* v, uint16_t* h, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        h[i] = oracle_f32_to_fp16_rn(v[i]);
}

/* A 16-bit input value of the given type (0 = bfloat16, 1 = binary16) as
 * binary32, and binary32 rounded to it. */
static float in16_to_f32(uint16_t v, int dtype)
{
    return dtype == 1 ? oracle_fp16_to_f32(v) : oracle_bf16_to_f32(v);
}

static uint16_t f32_to_out16(float f, int dtype)
{
    return dtype == 1 ? oracle_f32_to_fp16_rn(f) : oracle_f32_to_bf16_rn(f);
}

/* OCP 8-bit floating point, E4M3 ("fn" variant): 1 sign bit, 4 exponent
 * bits with bias 7, 3 mantissa bits; no infinities; S.1111.111 is NaN, so
 * the largest finite magnitude is 1.75 * 2^8 = 448.  Exponent field 0
 * encodes subnormals m * 2^-9, m = 1..7. */
float oracle_e4m3_to_f32(uint8_t q)
{
    int sign = (q >> 7) & 1;
    int ex = (q >> 3) & 0xf;
    int man = q & 7;
    double v;
    if (ex == 0xf && man == 7)
        return NAN;
    if (ex == 0)
        v = ldexp((double)man, -9);
    else
        v = ldexp(1.0 + man / 8.0, ex - 7);
    return (float)(sign ? -v : v);
}

/* binary32 -> E4M3, round to nearest with ties to even, saturating finite
 * overflow (and infinities) to +-448.  The grid spacing of E4M3 at
 * magnitude a is 2^-9 below 2^-6 (subnormals) and 2^(floor(log2 a) - 3)
 * above.  Scaling by a power of two and flooring are exact in double. */
uint8_t oracle_f32_to_e4m3_rn_sat(float v)
{
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    if (isnan(v))
        return (uint8_t)(sign | 0x7f);
    double a = fabs((double)v);
    if (a >= 448.0)
        return (uint8_t)(sign | 0x7e);
    int e2 = 0;
    double step;
    if (a < ldexp(1.0, -6)) {
        step = ldexp(1.0, -9);
    } else {
        (void)frexp(a, &e2);           /* a = f * 2^e2, f in [0.5, 1) */
        step = ldexp(1.0, (e2 - 1) - 3); /* binade [2^(e2-1), 2^e2) */
    }
    double q = a / step;               /* exact */
    double n = floor(q);
    double rem = q - n;
    if (rem > 0.5 || (rem == 0.5 && fmod(n, 2.0) != 0.0))
        n += 1.0;
    double r = n * step;               /* rounded magnitude, exact */
    if (r >= 448.0)                    /* cannot exceed 448 here, kept for clarity */
        return (uint8_t)(sign | 0x7e);
    if (r == 0.0)
        return sign;
    if (r < ldexp(1.0, -6)) {
        int m = (int)(r / ldexp(1.0, -9));
        return (uint8_t)(sign | m);
    }
    int er = 0;
    double fr = frexp(r, &er);         /* r = fr * 2^er, fr in [0.5,1) */
    int ex = (er - 1) + 7;             /* biased exponent */
    int man = (int)((fr * 2.0 - 1.0) * 8.0);
    return (uint8_t)(sign | (ex << 3) | man);
}

/* Array forms used by the tests (pins against a library cast). */
void oracle_f32_to_e4m3_array(const float* v, uint8_t* q, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        q[i] = oracle_f32_to_e4m3_rn_sat(v[i]);
}

void oracle_e4m3_to_f32_array(const uint8_t* q, float* v, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        v[i] = oracle_e4m3_to_f32(q[i]);
}

void oracle_f32_to_bf16_array(const float* v, uint16_t* b, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        b[i] = oracle_f32_to_bf16_rn(v[i]);
}

/* ------------------------------------------------------------------ */
/* Dispatch layout.                                                     */
/* ------------------------------------------------------------------ */

static int64_t pad_up(int64_t c, int64_t block_m)
{
    return ((c + block_m - 1) / block_m) * block_m;
}

/* Upper bound on the padded receive rows for T tokens: every non-empty
 * expert adds at most block_m - 1 pad rows, and at most min(E, T*k)
 * experts are non-empty.  (Capacity headroom for uneven routing, which
 * "DeepEP是什麼？…", section ElasticBuffer, asks a buffer to keep.) */
int64_t oracle_recv_rows_bound(int64_t T, int k, int E, int block_m)
{
    int64_t n = T * (int64_t)k;
    int64_t m = n < E ? n : E;
    int64_t b = n + m * (int64_t)(block_m - 1);
    return (b / block_m) * block_m;
}

/*
 * get_dispatch_layout, as a plain definition.
 *
 * Inputs: topk_idx [T][k] (int64), value in [0, E) or -1 for an unused slot.
 * Outputs (caller-allocated):
 *   num_tokens_per_expert[E]   cnt[e] = #{(t,j) : topk_idx[t][j] == e}
 *   num_tokens_per_rank[R]     #{t : token t has a slot on rank r}
 *   num_rows_per_rank[R]       sum of cnt[e] over the experts of rank r
 *   expert_off[E+1]            exclusive prefix of pad(cnt[e])
 *   rank_off[R+1]              expert_off[r * (E/R)]
 *   is_token_in_rank[T][R]     1 if some slot of token t is on rank r
 *   dst_row[T][k]              receive row of slot (t, j), -1 if unused
 *   recv_src[recv_cap]         source token of each receive row, -1 on pad
 *   total_rows[1]              P = expert_off[E]
 * Returns OR_ERR_BAD_INDEX for an index outside [-1, E) (outputs then
 * undefined), OR_ERR_CAPACITY if recv_cap < P.
 * Source: the "dispatch layout" the pages' ElasticBuffer manages
 * ("DeepEP是什麼？…", section ElasticBuffer), the per-expert token counts and
 * per-rank traffic of its Load Imbalance section, and hidden states arranged
 * by expert as dispatch's output (stage table, section MoE為什麼需要All-to-all).
 * Expert-major order, block_m padding and (token, slot) order inside a block
 * are the reading taken where the pages leave the "GEMM layout" undefined.
 */
int oracle_layout(const int64_t* topk_idx, int64_t T, int k, int E, int R, int block_m,
                  int32_t* num_tokens_per_expert, int32_t* num_tokens_per_rank,
                  int32_t* num_rows_per_rank, int32_t* expert_off, int32_t* rank_off,
                  uint8_t* is_token_in_rank, int32_t* dst_row, int32_t* recv_src,
                  int64_t recv_cap, int32_t* total_rows)
{
    if (T < 0 || k < 1 || E < 1 || R < 1 || E % R != 0 || block_m < 1)
        return OR_ERR_ARG;
    const int epr = E / R;

    for (int64_t i = 0; i < T * (int64_t)k; ++i)
        if (topk_idx[i] < -1 || topk_idx[i] >= E)
            return OR_ERR_BAD_INDEX;

    /* Each expert's list of (t, j), appended in lexicographic order: the
     * position of a slot in its expert's list is its rank inside the block. */
    int64_t* pos_in_list = (int64_t*)malloc(sizeof(int64_t) * (size_t)(T * k + 1));
    int64_t* list_len = (int64_t*)calloc((size_t)E, sizeof(int64_t));
    if (!pos_in_list || !list_len) {
        free(pos_in_list);
        free(list_len);
        return OR_ERR_ARG;
    }
    for (int64_t t = 0; t < T; ++t)
        for (int j = 0; j < k; ++j) {
            int64_t e = topk_idx[t * k + j];
            if (e < 0) {
                pos_in_list[t * k + j] = -1;
                continue;
            }
            pos_in_list[t * k + j] = list_len[e];
            list_len[e] += 1;
        }

    for (int e = 0; e < E; ++e)
        num_tokens_per_expert[e] = (int32_t)list_len[e];

    expert_off[0] = 0;
    for (int e = 0; e < E; ++e)
        expert_off[e + 1] = (int32_t)(expert_off[e] + pad_up(list_len[e], block_m));
    for (int r = 0; r <= R; ++r)
        rank_off[r] = expert_off[r * epr];
    *total_rows = expert_off[E];

    for (int r = 0; r < R; ++r) {
        int64_t rows = 0;
        for (int e = r * epr; e < (r + 1) * epr; ++e)
            rows += list_len[e];
        num_rows_per_rank[r] = (int32_t)rows;
    }

    for (int64_t t = 0; t < T; ++t)
        for (int j = 0; j < k; ++j) {
            int64_t e = topk_idx[t * k + j];
            dst_row[t * k + j] = e < 0 ? -1 : (int32_t)(expert_off[e] + pos_in_list[t * k + j]);
        }

    for (int64_t t = 0; t < T; ++t)
        for (int r = 0; r < R; ++r) {
            uint8_t hit = 0;
            for (int j = 0; j < k; ++j) {
                int64_t e = topk_idx[t * k + j];
                if (e >= 0 && e / epr == r)
                    hit = 1;
            }
            is_token_in_rank[t * R + r] = hit;
        }
    for (int r = 0; r < R; ++r) {
        int64_t n = 0;
        for (int64_t t = 0; t < T; ++t)
            n += is_token_in_rank[t * R + r];
        num_tokens_per_rank[r] = (int32_t)n;
    }

    free(pos_in_list);
    free(list_len);

    if (recv_cap < *total_rows)
        return OR_ERR_CAPACITY;
    for (int64_t i = 0; i < *total_rows; ++i)
        recv_src[i] = -1;
    for (int64_t t = 0; t < T; ++t)
        for (int j = 0; j < k; ++j) {
            int32_t d = dst_row[t * k + j];
            if (d >= 0)
                recv_src[d] = (int32_t)t;
        }
    return OR_OK;
}

/* Threads of the parallel build (a no-op returning 1 in the serial one). */
int oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0)
        omp_set_num_threads(n);
    return omp_get_max_threads();
#else
    (void)n;
    return 1;
#endif
}

/* 1 if every row named in dst_row[0..n) is below cap (checked before the
 * token loops, which then have no early exit). */
static int rows_below(const int32_t* dst_row, int64_t n, int64_t cap)
{
    for (int64_t i = 0; i < n; ++i)
        if (dst_row[i] >= cap)
            return 0;
    return 1;
}

/* ------------------------------------------------------------------ */
/* Dispatch.                                                            */
/* ------------------------------------------------------------------ */

/* BF16 dispatch: every used slot (t, j) receives a byte copy of x[t]
 * (dispatch as the stage table of "DeepEP是什麼？…", section
 * MoE為什麼需要All-to-all, defines it: tokens in, rows arranged by expert out). */
int oracle_dispatch_bf16(const uint16_t* x, int64_t T, int k, int64_t H,
                         const int32_t* dst_row, uint16_t* recv_x, int64_t recv_cap)
{
    if (!rows_below(dst_row, T * k, recv_cap))
        return OR_ERR_CAPACITY;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t)
        for (int j = 0; j < k; ++j) {
            int64_t d = dst_row[t * k + j];
            if (d >= 0)
                memcpy(recv_x + d * H, x + t * H, sizeof(uint16_t) * (size_t)H);
        }
    return OR_OK;
}

/* FP8 quantisation of one token: H/128 blocks of 128 channels; per block
 * amax = max |x|, s = amax / 448 (fp32 division), q = e4m3(x / s) (fp32
 * division, then round-to-nearest-even with saturation); amax == 0 gives
 * s = 0 and q = +0 for the whole block.  x holds bfloat16 (dtype 0) or
 * binary16 (dtype 1) values, widened exactly to binary32.  "DeepEP是什麼？…",
 * section FP8與低精度通訊, asks to confirm the scale granularity and format
 * without fixing them; this is the reading taken. */
void oracle_quantize_token_fp8(const uint16_t* x, int64_t H, int dtype, uint8_t* q,
                               float* scales)
{
    for (int64_t b = 0; b < H / 128; ++b) {
        float amax = 0.0f;
        for (int i = 0; i < 128; ++i) {
            float v = fabsf(in16_to_f32(x[b * 128 + i], dtype));
            if (v > amax)
                amax = v;
        }
        if (amax == 0.0f) {
            scales[b] = 0.0f;
            for (int i = 0; i < 128; ++i)
                q[b * 128 + i] = 0x00;
            continue;
        }
        float s = amax / 448.0f;
        scales[b] = s;
        for (int i = 0; i < 128; ++i) {
            float v = in16_to_f32(x[b * 128 + i], dtype) / s;
            q[b * 128 + i] = oracle_f32_to_e4m3_rn_sat(v);
        }
    }
}

/* FP8 dispatch: every used slot (t, j) receives the e4m3 row of x[t] and
 * its H/128 fp32 scales (row-major [rows][H/128]).  FP8 dispatch with BF16
 * combine is the pages' configuration (DeepEP v2 release notes, section Số
 * liệu kỹ thuật). */
int oracle_dispatch_fp8(const uint16_t* x, int64_t T, int k, int64_t H, int dtype,
                        const int32_t* dst_row, uint8_t* recv_q, float* recv_scales,
                        int64_t recv_cap)
{
    if (H % 128 != 0)
        return OR_ERR_ARG;
    if (!rows_below(dst_row, T * k, recv_cap))
        return OR_ERR_CAPACITY;
    const int64_t nb = H / 128;
    int rc = OR_OK;
#pragma omp parallel
    {
        uint8_t* q = (uint8_t*)malloc((size_t)(H > 0 ? H : 1));
        float* s = (float*)malloc(sizeof(float) * (size_t)(nb > 0 ? nb : 1));
        if (!q || !s) {
#pragma omp atomic write
            rc = OR_ERR_ARG;
        }
#pragma omp for schedule(static)
        for (int64_t t = 0; t < T; ++t) {
            if (!q || !s)
                continue;
            oracle_quantize_token_fp8(x + t * H, H, dtype, q, s);
            for (int j = 0; j < k; ++j) {
                int64_t d = dst_row[t * k + j];
                if (d < 0)
                    continue;
                memcpy(recv_q + d * H, q, (size_t)H);
                memcpy(recv_scales + d * nb, s, sizeof(float) * (size_t)nb);
            }
        }
        free(q);
        free(s);
    }
    return rc;
}

/* ------------------------------------------------------------------ */
/* Stand-in expert op (harness, not on the path): y = bf16(c[e] * x~).  */
/* ------------------------------------------------------------------ */

/* BF16 receive rows: y = bf16_rn(c[e] * float(x)). */
void oracle_expert_scale_bf16(const uint16_t* recv_x, const int32_t* recv_src,
                              const int32_t* expert_off, int E, int64_t H,
                              const float* c, uint16_t* y)
{
    for (int e = 0; e < E; ++e)
        for (int64_t r = expert_off[e]; r < expert_off[e + 1]; ++r) {
            if (recv_src[r] < 0)
                continue;
            for (int64_t h = 0; h < H; ++h) {
                float v = c[e] * oracle_bf16_to_f32(recv_x[r * H + h]);
                y[r * H + h] = oracle_f32_to_bf16_rn(v);
            }
        }
}

/* FP8 receive rows: y = bf16_rn(c[e] * (float(q) * s)), two fp32 products
 * in that order. */
void oracle_expert_scale_fp8(const uint8_t* recv_q, const float* recv_scales,
                             const int32_t* recv_src, const int32_t* expert_off, int E,
                             int64_t H, const float* c, uint16_t* y)
{
    const int64_t nb = H / 128;
    for (int e = 0; e < E; ++e)
        for (int64_t r = expert_off[e]; r < expert_off[e + 1]; ++r) {
            if (recv_src[r] < 0)
                continue;
            for (int64_t h = 0; h < H; ++h) {
                float deq = oracle_e4m3_to_f32(recv_q[r * H + h]) * recv_scales[r * nb + h / 128];
                y[r * H + h] = oracle_f32_to_bf16_rn(c[e] * deq);
            }
        }
}

/* ------------------------------------------------------------------ */
/* Combine.                                                             */
/* ------------------------------------------------------------------ */

/* out[t][h] = rn16(acc), acc = 0; for j = 0..k-1 over used slots:
 * acc = fmaf(w[t][j], float(y[dst_row[t][j]][h]), acc); y and out are
 * bfloat16 (dtype 0) or binary16 (dtype 1), rn16 the round-to-nearest-even
 * into that type.  The slot loop is
 * the outer loop over a row of accumulators; each element still sees its
 * terms in slot order.  Source: the Combine row of the stage table in
 * "DeepEP是什麼？…", section MoE為什麼需要All-to-all (expert outputs and routing
 * weights in, the original token order out, by a reduction); the fp32 fma
 * chain in slot order is the reading taken of the reduction's arithmetic. */
int oracle_combine(const uint16_t* y, int64_t y_rows, const float* w, const int32_t* dst_row,
                   int64_t T, int k, int64_t H, int dtype, uint16_t* out)
{
    if (!rows_below(dst_row, T * k, y_rows))
        return OR_ERR_CAPACITY;
    int rc = OR_OK;
#pragma omp parallel
    {
        float* acc = (float*)malloc(sizeof(float) * (size_t)(H > 0 ? H : 1));
        if (!acc) {
#pragma omp atomic write
            rc = OR_ERR_ARG;
        }
#pragma omp for schedule(static)
        for (int64_t t = 0; t < T; ++t) {
            if (!acc)
                continue;
            for (int64_t h = 0; h < H; ++h)
                acc[h] = 0.0f;
            for (int j = 0; j < k; ++j) {
                int64_t d = dst_row[t * k + j];
                if (d < 0)
                    continue;
                const float wj = w[t * k + j];
                for (int64_t h = 0; h < H; ++h)
                    acc[h] = fmaf(wj, in16_to_f32(y[d * H + h], dtype), acc[h]);
            }
            for (int64_t h = 0; h < H; ++h)
                out[t * H + h] = f32_to_out16(acc[h], dtype);
        }
        free(acc);
    }
    return rc;
}

/* ------------------------------------------------------------------ */
/* Backward.  The pages name training as a use (the pomoai page, section */
/* 核心使用场景; the yololab page, high-throughput mode for training) but */
/* do not define gradients; these are the gradients of the forward       */
/* definitions above.                                                    */
/* ------------------------------------------------------------------ */

/* Backward of dispatch: every used slot (t, j) copied x[t] to row
 * dst_row[t][j], so grad_x[t] = sum over used slots of grad_recv[row],
 * accumulated in fp32 in slot order j = 0..k-1 (plain additions), rounded to
 * the 16-bit type (bfloat16, dtype 0, or binary16, dtype 1) at the end. */
int oracle_dispatch_backward(const uint16_t* grad_recv, int64_t rows, const int32_t* dst_row,
                             int64_t T, int k, int64_t H, int dtype, uint16_t* grad_x)
{
    if (!rows_below(dst_row, T * k, rows))
        return OR_ERR_CAPACITY;
    int rc = OR_OK;
#pragma omp parallel
    {
        float* acc = (float*)malloc(sizeof(float) * (size_t)(H > 0 ? H : 1));
        if (!acc) {
#pragma omp atomic write
            rc = OR_ERR_ARG;
        }
#pragma omp for schedule(static)
        for (int64_t t = 0; t < T; ++t) {
            if (!acc)
                continue;
            for (int64_t h = 0; h < H; ++h)
                acc[h] = 0.0f;
            for (int j = 0; j < k; ++j) {
                int64_t d = dst_row[t * k + j];
                if (d < 0)
                    continue;
                for (int64_t h = 0; h < H; ++h)
                    acc[h] = acc[h] + in16_to_f32(grad_recv[d * H + h], dtype);
            }
            for (int64_t h = 0; h < H; ++h)
                grad_x[t * H + h] = f32_to_out16(acc[h], dtype);
        }
        free(acc);
    }
    return rc;
}

/* Backward of combine, out[t] = sum_j w[t][j] y[dst_row[t][j]]:
 *   grad_y[dst_row[t][j]][h] = rn16(w[t][j] * grad_out[t][h])  (one fp32 product)
 *   grad_w[t][j] = sum_h grad_out[t][h] * y[dst_row[t][j]][h]   (fp64, rounded to fp32)
 * Unused slots get grad_w = 0 and write no row.  The 16-bit rows are
 * bfloat16 (dtype 0) or binary16 (dtype 1); rn16 rounds to that type. */
int oracle_combine_backward(const uint16_t* grad_out, const uint16_t* y, int64_t y_rows,
                            const float* w, const int32_t* dst_row, int64_t T, int k, int64_t H,
                            int dtype, uint16_t* grad_y, float* grad_w)
{
    if (!rows_below(dst_row, T * k, y_rows))
        return OR_ERR_CAPACITY;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t)
        for (int j = 0; j < k; ++j) {
            int64_t d = dst_row[t * k + j];
            if (d < 0) {
                grad_w[t * k + j] = 0.0f;
                continue;
            }
            double dot = 0.0;
            for (int64_t h = 0; h < H; ++h) {
                const float g = in16_to_f32(grad_out[t * H + h], dtype);
                dot += (double)g * (double)in16_to_f32(y[d * H + h], dtype);
                grad_y[d * H + h] = f32_to_out16(w[t * k + j] * g, dtype);
            }
            grad_w[t * k + j] = (float)dot;
        }
    return OR_OK;
}

/* ------------------------------------------------------------------ */
/* GEMM-ready receive layout.  The pages say high-throughput and low-    */
/* latency kernels share one "GEMM layout" (DeepEP v2 release notes,     */
/* "Có gì mới trong v2"; the pomoai page, ElasticBuffer paragraph)       */
/* without defining it; these are the readings taken for an expert GEMM  */
/* that consumes the receive buffer directly.                            */
/* ------------------------------------------------------------------ */

/* Per-row routing weight: recv_w[dst_row[t][j]] = w[t][j] for every used
 * slot; pad rows are not written. */
int oracle_dispatch_weights(const float* w, const int32_t* dst_row, int64_t T, int k,
                            float* recv_w, int64_t recv_cap)
{
    for (int64_t t = 0; t < T; ++t)
        for (int j = 0; j < k; ++j) {
            int64_t d = dst_row[t * k + j];
            if (d < 0)
                continue;
            if (d >= recv_cap)
                return OR_ERR_CAPACITY;
            recv_w[d] = w[t * k + j];
        }
    return OR_OK;
}

/* Zero the pad rows of a row buffer in the receive layout: every row r < P
 * with recv_src[r] == -1 gets row_bytes zero bytes. */
void oracle_zero_pad_rows(const int32_t* recv_src, int64_t P, uint8_t* rows, int64_t row_bytes)
{
    for (int64_t r = 0; r < P; ++r)
        if (recv_src[r] < 0)
            memset(rows + r * row_bytes, 0, (size_t)row_bytes);
}

/* MN-major FP8 scales: the same scales as oracle_dispatch_fp8, stored as
 * scales_mn[b][row] with leading dimension ld (b = 128-channel block). */
int oracle_dispatch_fp8_mn(const uint16_t* x, int64_t T, int k, int64_t H, int dtype,
                           const int32_t* dst_row, uint8_t* recv_q, float* scales_mn,
                           int64_t ld, int64_t recv_cap)
{
    if (H % 128 != 0 || ld < recv_cap)
        return OR_ERR_ARG;
    const int64_t nb = H / 128;
    uint8_t* q = (uint8_t*)malloc((size_t)H);
    float* s = (float*)malloc(sizeof(float) * (size_t)(nb > 0 ? nb : 1));
    if (!q || !s) {
        free(q);
        free(s);
        return OR_ERR_ARG;
    }
    int rc = OR_OK;
    for (int64_t t = 0; t < T && rc == OR_OK; ++t) {
        oracle_quantize_token_fp8(x + t * H, H, dtype, q, s);
        for (int j = 0; j < k; ++j) {
            int64_t d = dst_row[t * k + j];
            if (d < 0)
                continue;
            if (d >= recv_cap) {
                rc = OR_ERR_CAPACITY;
                break;
            }
            memcpy(recv_q + d * H, q, (size_t)H);
            for (int64_t b = 0; b < nb; ++b)
                scales_mn[b * ld + d] = s[b];
        }
    }
    free(q);
    free(s);
    return rc;
}
