/*
 * echo_oracle.c -- plain, slow, single-threaded CPU definition of one call of
 * Echo, the error-compensated 4-bit tensor-parallel all-reduce
 * ("Echo: Error-Compensated 4-Bit Tensor-Parallel Communication for LLM
 * Training and Inference", arXiv 2610.14277).
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the oracle that the CUDA path is
 * checked against.  Only the tests, the smoke check of the build entry point
 * and the CPU-baseline leg of the benchmark may load it.  It shares no code,
 * header, table or helper with the CUDA library, and the CUDA library never
 * loads it.
 *
 * Build: gcc -O2 -ffp-contract=off -fPIC -shared (no -ffast-math, so fp32
 * arithmetic is IEEE-754 single precision with round-to-nearest-even, no
 * fused multiply-add, no flush-to-zero).
 *
 * Sources for each step (page title + section):
 *  - ai4snews news summary, "Interpretation" paragraph 1: the all-reduce is
 *    replaced by 4-bit integer transport plus a high-precision sum.
 *  - ai4snews news summary, "Interpretation" paragraph 2: the compensator is
 *    a pair of exponential moving averages, one fast and one slow; a weighted
 *    mix of the two is added to each input before it is quantized; both are
 *    then updated from the residual of the output, which the sum exposes.
 *  - arXiv abstract (fugumt mirror, "Abstract"): codes travel at 4 bits and
 *    are added at high precision, and no value is rounded more than twice in
 *    a call whatever the number of GPUs (reduce-scatter, requantize,
 *    all-gather).
 *  - heraldofai explainer, "How Echo keeps errors from snowballing": the
 *    same bound of two roundings per value.
 * The pages fix no constants, no scale format and no rounding rule; the
 * readings taken here (symmetric absmax int4 with levels -7..7, fp32 scale
 * per group of G contiguous elements, round half to even, requantization
 * error revealed to the owner rank of the chunk only, EMA m <- b*m + (1-b)*e
 * split into a partial update at entry and an owner fix-up after the sum)
 * are the plainest ones consistent with those passages.
 *
 * Notation: P ranks, N elements per rank, G group size, owner of element i
 * is floor(i / (N/P)).  A "group column" c is the G elements
 * [c*G, (c+1)*G) of every rank; everything at element i depends only on the
 * group column of i, across the P ranks, and on earlier calls at the same
 * column, so the call can be evaluated on any list of group columns.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define EO_OK 0
#define EO_ERR_ARG 1

/* fp32 arithmetic, one rounding per operation (the file is built with
 * -ffp-contract=off, so nothing here is fused). */
static float fadd(float a, float b) { return a + b; }
static float fsub(float a, float b) { return a - b; }
static float fmul(float a, float b) { return a * b; }
static float fdiv(float a, float b) { return a / b; }

/* bf16 -> fp32 is exact: the bf16 bits are the top half of the fp32 bits. */
float eo_bf16_to_f32(uint16_t b)
{
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* fp32 -> bf16, round to nearest, ties to even (IEEE default rounding). */
uint16_t eo_f32_to_bf16_rne(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7fffffffu) > 0x7f800000u) /* NaN: keep it a quiet NaN */
        return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

/*
 * Quantize one group of G fp32 values to symmetric codes with L levels on
 * each side (L = 7 for 4-bit codes, 127 for 8-bit codes).
 *   a = max |v|;  scale = a / L;  k = clamp(rint(v / scale), -L, L).
 * A group with a == 0 (or whose scale underflows to 0) gets scale 0 and all
 * codes 0.  rintf rounds half to even in the default rounding mode.
 * If count is not NULL, count[j] is incremented for every element j that is
 * quantized (the instrumented oracle counts quantizer applications).
 */
void eo_quantize_group_levels(const float *v, int G, int L, int8_t *k,
                              float *scale_out, int32_t *count)
{
    const float levels = (float)L;
    float a = 0.0f;
    for (int j = 0; j < G; ++j)
        a = fmaxf(a, fabsf(v[j]));
    float scale = 0.0f;
    if (a != 0.0f)
        scale = fdiv(a, levels);
    for (int j = 0; j < G; ++j) {
        int code = 0;
        if (scale != 0.0f) {
            float r = rintf(fdiv(v[j], scale));
            if (r > levels) r = levels;
            if (r < -levels) r = -levels;
            code = (int)r;
        }
        k[j] = (int8_t)code;
        if (count) count[j] += 1;
    }
    *scale_out = scale;
}

/* The 4-bit quantizer: L = 7. */
void eo_quantize_group(const float *v, int G, int8_t *k, float *scale_out,
                       int32_t *count)
{
    eo_quantize_group_levels(v, G, 7, k, scale_out, count);
}

/* Dequantize one code: k * scale in fp32. */
float eo_dequant(int8_t k, float scale) { return fmul((float)k, scale); }

/* Pack n codes (n even), two per byte: element 2j in bits 0..3, element
 * 2j+1 in bits 4..7, each nibble two's complement. */
void eo_pack(const int8_t *k, int64_t n, uint8_t *bytes)
{
    for (int64_t j = 0; j < n / 2; ++j) {
        uint8_t lo = (uint8_t)(k[2 * j] & 0x0f);
        uint8_t hi = (uint8_t)(k[2 * j + 1] & 0x0f);
        bytes[j] = (uint8_t)(lo | (hi << 4));
    }
}

/* 8-bit codes: one per byte, two's complement. */
void eo_pack8(const int8_t *k, int64_t n, uint8_t *bytes)
{
    for (int64_t j = 0; j < n; ++j)
        bytes[j] = (uint8_t)k[j];
}

/* Inverse of eo_pack: sign-extend each nibble. */
void eo_unpack(const uint8_t *bytes, int64_t n, int8_t *k)
{
    for (int64_t j = 0; j < n / 2; ++j) {
        int lo = bytes[j] & 0x0f;
        int hi = (bytes[j] >> 4) & 0x0f;
        k[2 * j] = (int8_t)(lo >= 8 ? lo - 16 : lo);
        k[2 * j + 1] = (int8_t)(hi >= 8 ? hi - 16 : hi);
    }
}

typedef struct {
    int32_t P;          /* ranks */
    int32_t G;          /* group size (even) */
    int64_t N;          /* elements per rank; N % (P*G) == 0 */
    int32_t compensate; /* 1: dual-EMA compensator on; 0: off */
    float alpha;        /* weight of the fast EMA in the correction */
    float beta_fast;    /* decay of the fast EMA */
    float beta_slow;    /* decay of the slow EMA */
    int32_t bits;       /* 4: int4 codes, two per byte; 8: int8 codes */
} eo_params;

/*
 * One call, evaluated on ncols group columns (requantize = 1: the
 * all-reduce; 0: the reduce-scatter).
 *
 * cols: ncols group-column ids in [0, N/G), or NULL for every column in
 * order (then ncols must be N/G).  Every per-rank array below is dense over
 * the listed columns: rank r's element j of listed column t is at index
 * r*(ncols*G) + t*G + j.
 *
 *   x       [P][ncols*G]   bf16 bits, input of each rank (read)
 *   m_fast  [P][ncols*G]   fast EMA state (read, updated in place)
 *   m_slow  [P][ncols*G]   slow EMA state (read, updated in place)
 *   codes   [P][ncols*G*bits/8] entry codes, packed (written)
 *   scales  [P][ncols]     entry scales (written)
 *   xt      [P][ncols*G]   corrected input x + c (written, may be NULL)
 *   e_in    [P][ncols*G]   entry quantization error (written, may be NULL)
 *   s       [ncols*G]      fp32 sum of the dequantized entries (may be NULL)
 *   rcodes  [ncols*G*bits/8] requantized sum, packed (written)
 *   rscales [ncols]        requantization scales (written)
 *   e_req   [ncols*G]      requantization error s - float(y) (written)
 *   y       [ncols*G]      bf16 bits of the result every rank receives
 *   qcount  [ncols*G]      if not NULL: quantizer applications on the path
 *                          of each result element (max over the entry
 *                          quantizations of its P contributions, plus the
 *                          requantizations of its sum); zeroed first
 *
 * With compensate == 0 the states are neither read nor written (they may
 * be NULL) and the correction is zero.
 * Returns 0, or 1 for an invalid argument.
 */
static int call_columns(const eo_params *prm, int64_t ncols, const int64_t *cols,
                        const uint16_t *x, float *m_fast, float *m_slow,
                        uint8_t *codes, float *scales, float *xt_out, float *e_in,
                        float *s, uint8_t *rcodes, float *rscales, float *e_req,
                        uint16_t *y, int32_t *qcount, int requantize)
{
    const int P = prm->P, G = prm->G;
    const int64_t N = prm->N;
    if (P < 1 || G < 2 || (G & 1) || N <= 0 || N % ((int64_t)P * G) != 0)
        return EO_ERR_ARG;
    if (prm->bits != 4 && prm->bits != 8)
        return EO_ERR_ARG;
    const int L = prm->bits == 8 ? 127 : 7;   /* levels on each side */
    if (cols == NULL && ncols != N / G)
        return EO_ERR_ARG;
    if (prm->compensate && (m_fast == NULL || m_slow == NULL))
        return EO_ERR_ARG;
    if (!x || !codes || !scales || !e_req || !y)
        return EO_ERR_ARG;
    if (requantize && (!rcodes || !rscales))
        return EO_ERR_ARG;
    for (int64_t t = 0; cols && t < ncols; ++t)
        if (cols[t] < 0 || cols[t] >= N / G)
            return EO_ERR_ARG;

    const int64_t n = ncols * G;          /* elements per rank, listed */
    const int64_t chunk = N / P;          /* owner chunk length */
    const float alpha = prm->alpha;
    const float one_m_alpha = fsub(1.0f, alpha);
    const float bf = prm->beta_fast, bs = prm->beta_slow;
    const float one_m_bf = fsub(1.0f, bf), one_m_bs = fsub(1.0f, bs);

    float *xt = (float *)malloc(sizeof(float) * (size_t)G);
    float *sum = (float *)malloc(sizeof(float) * (size_t)G);
    int8_t *k = (int8_t *)malloc((size_t)G);
    int32_t *cnt_entry = (int32_t *)calloc((size_t)G, sizeof(int32_t));
    int32_t *cnt_req = (int32_t *)calloc((size_t)G, sizeof(int32_t));
    int32_t *max_entry_count = (int32_t *)calloc((size_t)G, sizeof(int32_t));
    float *ein_local = (float *)malloc(sizeof(float) * (size_t)P * G);
    if (!xt || !sum || !k || !cnt_entry || !cnt_req || !max_entry_count ||
        !ein_local) {
        free(xt); free(sum); free(k); free(cnt_entry); free(cnt_req);
        free(max_entry_count); free(ein_local);
        return EO_ERR_ARG;
    }

    for (int64_t t = 0; t < ncols; ++t) {
        const int64_t col = cols ? cols[t] : t;
        const int owner = (int)((col * G) / chunk);
        const int64_t base = t * G; /* offset of this column in a rank row */

        for (int j = 0; j < G; ++j)
            sum[j] = 0.0f;
        if (qcount)
            memset(cnt_req, 0, sizeof(int32_t) * (size_t)G);
        if (qcount)
            memset(max_entry_count, 0, sizeof(int32_t) * (size_t)G);

        /* Entry, for every rank in ascending order, followed by its term in
         * the reduce-scatter sum (the sum runs in ascending rank order from
         * +0.0f). */
        for (int r = 0; r < P; ++r) {
            const int64_t row = (int64_t)r * n + base;
            /* 1-2. correction c = a*m_f + (1-a)*m_s, added to the input */
            for (int j = 0; j < G; ++j) {
                float v = eo_bf16_to_f32(x[row + j]);
                if (prm->compensate) {
                    float c = fadd(fmul(alpha, m_fast[row + j]),
                                   fmul(one_m_alpha, m_slow[row + j]));
                    v = fadd(v, c);
                }
                xt[j] = v;
                if (xt_out)
                    xt_out[row + j] = v;
            }
            /* 3-4. quantize the group and pack it */
            float scale;
            if (qcount)
                memset(cnt_entry, 0, sizeof(int32_t) * (size_t)G);
            eo_quantize_group_levels(xt, G, L, k, &scale, qcount ? cnt_entry : NULL);
            if (prm->bits == 8)
                eo_pack8(k, G, codes + (int64_t)r * n + base);
            else
                eo_pack(k, G, codes + ((int64_t)r * n + base) / 2);
            scales[(int64_t)r * ncols + t] = scale;
            for (int j = 0; j < G; ++j) {
                float d = eo_dequant(k[j], scale);
                /* 5. local entry error, relative to the corrected input */
                float e = fsub(xt[j], d);
                ein_local[r * G + j] = e;
                if (e_in)
                    e_in[row + j] = e;
                /* 7. reduce-scatter term of this rank */
                sum[j] = fadd(sum[j], d);
                if (qcount && cnt_entry[j] > max_entry_count[j])
                    max_entry_count[j] = cnt_entry[j];
            }
            /* 6. partial EMA update from the entry error */
            if (prm->compensate) {
                for (int j = 0; j < G; ++j) {
                    float e = ein_local[r * G + j];
                    m_fast[row + j] = fadd(fmul(bf, m_fast[row + j]),
                                           fmul(one_m_bf, e));
                    m_slow[row + j] = fadd(fmul(bs, m_slow[row + j]),
                                           fmul(one_m_bs, e));
                }
            }
        }

        /* 8. all-reduce: requantize the owner's sum for the all-gather and
         * deliver it as bf16; reduce-scatter: the owner keeps its sum and
         * receives it as bf16 directly.  er is the owner's output residual. */
        float scale2 = 0.0f;
        if (requantize) {
            eo_quantize_group_levels(sum, G, L, k, &scale2, qcount ? cnt_req : NULL);
            if (prm->bits == 8)
                eo_pack8(k, G, rcodes + base);
            else
                eo_pack(k, G, rcodes + base / 2);
            rscales[t] = scale2;
        }
        for (int j = 0; j < G; ++j) {
            uint16_t yb = requantize ? eo_f32_to_bf16_rne(eo_dequant(k[j], scale2))
                                     : eo_f32_to_bf16_rne(sum[j]);
            float er = fsub(sum[j], eo_bf16_to_f32(yb));
            y[base + j] = yb;
            e_req[base + j] = er;
            if (s)
                s[base + j] = sum[j];
            if (qcount)
                qcount[base + j] = max_entry_count[j] + cnt_req[j];
            /* 9. the owner alone also folds the requantization error in */
            if (prm->compensate) {
                const int64_t orow = (int64_t)owner * n + base;
                m_fast[orow + j] = fadd(m_fast[orow + j], fmul(one_m_bf, er));
                m_slow[orow + j] = fadd(m_slow[orow + j], fmul(one_m_bs, er));
            }
        }
    }

    free(xt); free(sum); free(k); free(cnt_entry); free(cnt_req);
    free(max_entry_count); free(ein_local);
    return EO_OK;
}

/*
 * One all-reduce call (see call_columns above for the arguments): every
 * rank receives y, the requantized sum as bf16, and e_req = s - float(y)
 * goes to the owner of each chunk.
 */
int eo_allreduce(const eo_params *prm, int64_t ncols, const int64_t *cols,
                 const uint16_t *x, float *m_fast, float *m_slow,
                 uint8_t *codes, float *scales, float *xt_out, float *e_in,
                 float *s, uint8_t *rcodes, float *rscales, float *e_req,
                 uint16_t *y, int32_t *qcount)
{
    return call_columns(prm, ncols, cols, x, m_fast, m_slow, codes, scales,
                        xt_out, e_in, s, rcodes, rscales, e_req, y, qcount, 1);
}

/*
 * One reduce-scatter call: steps 1-7 as for the all-reduce, then the owner
 * of each chunk receives y = bf16(s) for its own chunk (each value is
 * quantized once, at entry) and folds its output residual s - float(y)
 * into its EMAs (returned in e_req).  rcodes and rscales are not used and
 * may be NULL.  The reduce-scatter of sequence parallelism is named as a
 * next target on the ai4snews news summary, "Perspective".
 */
int eo_reduce_scatter(const eo_params *prm, int64_t ncols, const int64_t *cols,
                      const uint16_t *x, float *m_fast, float *m_slow,
                      uint8_t *codes, float *scales, float *xt_out, float *e_in,
                      float *s, float *e_req, uint16_t *y, int32_t *qcount)
{
    return call_columns(prm, ncols, cols, x, m_fast, m_slow, codes, scales,
                        xt_out, e_in, s, NULL, NULL, e_req, y, qcount, 0);
}
