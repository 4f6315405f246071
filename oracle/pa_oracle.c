/*
 * pa_oracle.c -- plain CPU oracle for paged decode attention and the two
 * cache-maintenance operations that go with it.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the tests, the smoke check and the benchmark's CPU
 * baseline leg use it.  It shares no code, header, table or constant with the
 * CUDA library; the only thing both sides share is the seeded input generator.
 *
 * What it computes, and where that comes from:
 *
 *  - Paged KV layout: one pool tensor per K and V of shape
 *    [num_blocks][block_size][num_kv_heads][head_dim] (zingnex.cn,
 *    "vLLM与PagedAttention深度剖析", section 3.2, the global block tensor),
 *    addressed through a per-sequence block table that maps logical block
 *    j / block_size to a physical block (same page, section 3.2 item 2;
 *    5688vip.com notes, section 2.2, "logical block 0 -> physical block 7").
 *
 *  - Decode attention: the pages state no formula.  The plain reading is that
 *    paging changes only where K/V live, so the result is ordinary single-query
 *    attention over the sequence's tokens: for query head h of sequence s,
 *    with kv head h / (Hq / Hkv),
 *        x_j = scale * sum_d q[d] * K_j[d]           j = 0 .. ctx_s - 1
 *        m   = max_j x_j,  p_j = exp(x_j - m)
 *        out = sum_j p_j V_j / sum_j p_j
 *    all in fp64 after an exact widening of the fp16/bf16 inputs.  A context
 *    of length 0 gives out = 0.  The result is returned unrounded (fp64).
 *
 *  - Partitioned form: the same quantity assembled from independent
 *    partitions of partition_tokens tokens, each reduced to (m_p, l_p, acc_p)
 *    and merged with M = max_p m_p, out = sum_p e^(m_p-M) acc_p /
 *    sum_p e^(m_p-M) l_p.  This is the split-K merge of the decode kernel.
 *
 *  - Append: each new token's K and V row is copied into slot
 *    slot_mapping[t] = physical_block * block_size + offset (the "update KV
 *    cache" step of the decode loop, 5688vip.com section 2.1; on-demand
 *    block use, zingnex.cn section 3.2 item 1).  Negative slots are skipped.
 *
 *  - Copy-on-write: for each (src, dst) pair the whole block of K and of V is
 *    copied (zingnex.cn section 3.2 item 3).
 *
 *  - Swap: whole blocks copied between two pools, for instance a device
 *    pool and a pool in host memory (zingnex.cn section 5, tuning advice:
 *    CPU offload through swap space): block src of the source pools
 *    becomes block dst of the destination pools.
 *
 *  - Several query tokens per sequence (the scope table's multi-token
 *    queries: speculative verification and chunked prefill under continuous
 *    batching, 5688vip.com section 2.2): context_lens[s] counts the
 *    sequence's Tq new tokens,
 *    already appended, and query token t (0 <= t < Tq) attends causally to
 *    tokens 0 .. ctx_s - Tq + t, i.e. to every cached token before the new
 *    ones plus the new ones up to itself.  A query whose range is empty
 *    (ctx_s - Tq + t < 0) gives a zero row.
 *
 *  - FP8 cache (the pages name FP8 only as a quantisation format that saves
 *    memory: zingnex.cn sections 4.1 and 6, 5688vip.com section 2.3; the
 *    encoding below is the plain reading): K and V stored as OCP 8-bit E4M3
 *    codes with one fp32 scale per kv head and tensor.  E4M3 is 1 sign bit,
 *    4 exponent bits (bias 7) and 3 mantissa bits; exponent field 0 is
 *    subnormal (mantissa * 2^-9); S.1111.111 is NaN; there is no infinity;
 *    the largest finite value is 1.75 * 2^8 = 448.  A stored value is code * scale.  Append divides the
 *    input (widened exactly to fp32) by the scale in fp32 and rounds the
 *    quotient to the nearest code, ties to the even code, with magnitudes of
 *    448 and above (infinity included) saturated to 448.  Decode widens each
 *    code exactly and multiplies by the scale in fp64, then proceeds as
 *    above.
 *
 * Every function returns 0 on success and a negative value on an input it
 * refuses (bad shape, a table entry or slot outside the pool); on refusal the
 * outputs are unspecified.  Loops only: no BLAS, no SIMD intrinsics, no
 * blocking or reordering of any sum beyond the definition above.  OpenMP
 * parallelises over independent (sequence, head) outputs only.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORACLE_F16 = 0, ORACLE_BF16 = 1 };

/* IEEE binary16 -> double, exact: sign, 5-bit exponent (bias 15), 10-bit
 * fraction; exponent 0 is subnormal (fraction * 2^-24), 31 is Inf/NaN. */
double oracle_f16_to_f64(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int f = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)f, -24);
    else if (e == 31)
        v = f ? NAN : INFINITY;
    else
        v = ldexp((double)(f | 0x400), e - 25);
    return sign ? -v : v;
}

/* bfloat16 is the upper half of an IEEE binary32: widen by placing the 16
 * bits on top of a zero low half. */
double oracle_bf16_to_f64(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* OCP E4M3 code -> double, exact. */
double oracle_e4m3_to_f64(uint8_t c)
{
    int sign = (c >> 7) & 1;
    int e = (c >> 3) & 0xf;
    int m = c & 7;
    double v;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);
    else
        v = ldexp((double)(8 + m), e - 10);
    return sign ? -v : v;
}

/* fp32 -> nearest E4M3 code, ties to the even code, saturating at 448;
 * NaN -> 0x7F. */
uint8_t oracle_e4m3_from_f32(float y)
{
    if (isnan(y)) return 0x7f;
    uint8_t sign = signbit(y) ? 0x80 : 0x00;
    double a = fabs((double)y);
    if (a >= 448.0) return sign | 0x7e;
    if (a < ldexp(1.0, -6)) {
        /* subnormal step 2^-9; a count of 8 is the smallest normal, code 0x08 */
        double n = rint(ldexp(a, 9));
        return sign | (uint8_t)n;
    }
    int e;
    frexp(a, &e);            /* a = f * 2^e with f in [0.5, 1) */
    e -= 1;                  /* a in [2^e, 2^(e+1)) */
    double n = rint(ldexp(a, 3 - e));  /* in [8, 16] */
    if (n == 16.0) {
        n = 8.0;
        e += 1;
    }
    return sign | (uint8_t)(((e + 7) << 3) | ((int)n - 8));
}

static double widen(int dtype, uint16_t x)
{
    return dtype == ORACLE_F16 ? oracle_f16_to_f64(x) : oracle_bf16_to_f64(x);
}

static int shape_ok(int dtype, int S, int Hq, int Hkv, int D, int bs, int NB, int MBS)
{
    if (dtype != ORACLE_F16 && dtype != ORACLE_BF16) return 0;
    if (S < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || bs <= 0 || NB < 0 || MBS < 0) return 0;
    if (Hq % Hkv) return 0;
    return 1;
}

/* Element offset of token j's row for kv head kvh, or -1 when the table
 * entry that covers j lies outside the pool. */
static long long token_row(const int32_t *tables, int MBS, int s, int j, int bs, int NB,
                           int Hkv, int D, int kvh)
{
    int logical = j / bs;
    int phys = tables[(long long)s * MBS + logical];
    if (phys < 0 || phys >= NB) return -1;
    long long slot = (long long)phys * bs + (j % bs);
    return (slot * Hkv + kvh) * (long long)D;
}

/* Attention of one query head over tokens [t0, t1) of sequence s.
 * Writes m, l = sum p and acc[d] = sum p V[d] (p relative to m). */
static int attend_range(int dtype, int Hkv, int D, int bs, int NB, int MBS,
                        const uint16_t *qrow, const uint16_t *kc, const uint16_t *vc,
                        const int32_t *tables, int s, int kvh, int t0, int t1, double scale,
                        double *x, double *m_out, double *l_out, double *acc)
{
    int n = t1 - t0;
    double m = -INFINITY;
    for (int j = 0; j < n; ++j) {
        long long r = token_row(tables, MBS, s, t0 + j, bs, NB, Hkv, D, kvh);
        if (r < 0) return -2;
        double dot = 0.0;
        for (int d = 0; d < D; ++d)
            dot += widen(dtype, qrow[d]) * widen(dtype, kc[r + d]);
        x[j] = scale * dot;
        if (x[j] > m) m = x[j];
    }
    double l = 0.0;
    for (int d = 0; d < D; ++d) acc[d] = 0.0;
    for (int j = 0; j < n; ++j) {
        double p = exp(x[j] - m);
        l += p;
        long long r = token_row(tables, MBS, s, t0 + j, bs, NB, Hkv, D, kvh);
        for (int d = 0; d < D; ++d)
            acc[d] += p * widen(dtype, vc[r + d]);
    }
    *m_out = m;
    *l_out = l;
    return 0;
}

static int resolve_threads(int num_threads)
{
#ifdef _OPENMP
    return num_threads > 0 ? num_threads : omp_get_max_threads();
#else
    (void)num_threads;
    return 1;
#endif
}

int oracle_num_threads(int requested) { return resolve_threads(requested); }

/* Direct definition.  out: double [S][Hq][D]. */
int oracle_decode(int dtype, int S, int Hq, int Hkv, int D, int bs, int NB, int MBS,
                  const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                  const int32_t *block_tables, const int32_t *context_lens, double scale,
                  double *out, int num_threads)
{
    if (!shape_ok(dtype, S, Hq, Hkv, D, bs, NB, MBS)) return -1;
    for (int s = 0; s < S; ++s)
        if (context_lens[s] < 0 || (long long)context_lens[s] > (long long)MBS * bs) return -1;
    int g = Hq / Hkv;
    int err = 0;
    int nt = resolve_threads(num_threads);
    long long total = (long long)S * Hq;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nt) reduction(| : err)
    for (long long sh = 0; sh < total; ++sh) {
        int s = (int)(sh / Hq), h = (int)(sh % Hq);
        int L = context_lens[s];
        double *o = out + sh * D;
        if (L == 0) {
            for (int d = 0; d < D; ++d) o[d] = 0.0;
            continue;
        }
        double *x = (double *)malloc(sizeof(double) * (size_t)L);
        double *acc = (double *)malloc(sizeof(double) * (size_t)D);
        double m, l;
        int rc = attend_range(dtype, Hkv, D, bs, NB, MBS, q + sh * D, k_cache, v_cache,
                              block_tables, s, h / g, 0, L, scale, x, &m, &l, acc);
        if (rc) err |= 1;
        else
            for (int d = 0; d < D; ++d) o[d] = acc[d] / l;
        free(x);
        free(acc);
    }
    return err ? -2 : 0;
}

/* Split form: partitions of partition_tokens tokens merged by the
 * log-sum-exp rule.  Same output as oracle_decode up to rounding. */
int oracle_decode_partitioned(int dtype, int S, int Hq, int Hkv, int D, int bs, int NB, int MBS,
                              const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                              const int32_t *block_tables, const int32_t *context_lens,
                              double scale, int partition_tokens, double *out, int num_threads)
{
    if (!shape_ok(dtype, S, Hq, Hkv, D, bs, NB, MBS) || partition_tokens <= 0) return -1;
    for (int s = 0; s < S; ++s)
        if (context_lens[s] < 0 || (long long)context_lens[s] > (long long)MBS * bs) return -1;
    int g = Hq / Hkv;
    int err = 0;
    int nt = resolve_threads(num_threads);
    long long total = (long long)S * Hq;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nt) reduction(| : err)
    for (long long sh = 0; sh < total; ++sh) {
        int s = (int)(sh / Hq), h = (int)(sh % Hq);
        int L = context_lens[s];
        double *o = out + sh * D;
        for (int d = 0; d < D; ++d) o[d] = 0.0;
        if (L == 0) continue;
        int P = (L + partition_tokens - 1) / partition_tokens;
        double *x = (double *)malloc(sizeof(double) * (size_t)partition_tokens);
        double *pm = (double *)malloc(sizeof(double) * (size_t)P);
        double *pl = (double *)malloc(sizeof(double) * (size_t)P);
        double *pacc = (double *)malloc(sizeof(double) * (size_t)P * D);
        int bad = 0;
        for (int p = 0; p < P && !bad; ++p) {
            int t0 = p * partition_tokens;
            int t1 = t0 + partition_tokens < L ? t0 + partition_tokens : L;
            if (attend_range(dtype, Hkv, D, bs, NB, MBS, q + sh * D, k_cache, v_cache,
                             block_tables, s, h / g, t0, t1, scale, x, &pm[p], &pl[p],
                             pacc + (long long)p * D))
                bad = 1;
        }
        if (bad) err |= 1;
        else {
            double M = -INFINITY;
            for (int p = 0; p < P; ++p)
                if (pm[p] > M) M = pm[p];
            double den = 0.0;
            for (int p = 0; p < P; ++p) den += exp(pm[p] - M) * pl[p];
            for (int d = 0; d < D; ++d) {
                double num = 0.0;
                for (int p = 0; p < P; ++p) num += exp(pm[p] - M) * pacc[(long long)p * D + d];
                o[d] = num / den;
            }
        }
        free(x);
        free(pm);
        free(pl);
        free(pacc);
    }
    return err ? -2 : 0;
}

/* Append: row_bytes = num_kv_heads * head_dim * element bytes.  The pool is
 * num_slots = num_blocks * block_size rows of row_bytes; k and v hold
 * num_tokens rows each. */
int oracle_cache_append(long long num_slots, long long row_bytes, int num_tokens,
                        const uint8_t *k, const uint8_t *v, const int32_t *slot_mapping,
                        uint8_t *k_cache, uint8_t *v_cache)
{
    if (num_slots < 0 || row_bytes <= 0 || num_tokens < 0) return -1;
    for (int t = 0; t < num_tokens; ++t) {
        long long slot = slot_mapping[t];
        if (slot < 0) continue;
        if (slot >= num_slots) return -2;
        memcpy(k_cache + slot * row_bytes, k + (long long)t * row_bytes, (size_t)row_bytes);
        memcpy(v_cache + slot * row_bytes, v + (long long)t * row_bytes, (size_t)row_bytes);
    }
    return 0;
}

/* Copy-on-write: block_bytes = block_size * num_kv_heads * head_dim * element
 * bytes.  Pairs are applied in order. */
int oracle_copy_blocks(int num_blocks, long long block_bytes, int num_pairs, const int32_t *pairs,
                       uint8_t *k_cache, uint8_t *v_cache)
{
    if (num_blocks < 0 || block_bytes <= 0 || num_pairs < 0) return -1;
    for (int i = 0; i < num_pairs; ++i) {
        int src = pairs[2 * i], dst = pairs[2 * i + 1];
        if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) return -2;
        memmove(k_cache + (long long)dst * block_bytes, k_cache + (long long)src * block_bytes,
                (size_t)block_bytes);
        memmove(v_cache + (long long)dst * block_bytes, v_cache + (long long)src * block_bytes,
                (size_t)block_bytes);
    }
    return 0;
}

/* ---------------------------------------------------------------------
 * FP8 (E4M3) cache.  k_cache, v_cache: uint8 codes [NB][bs][Hkv][D];
 * k_scale, v_scale: fp32 [Hkv].  Same definition as oracle_decode with
 * K_j[d] = e4m3(k code) * k_scale[kv head] (and V likewise), in fp64. */
static int attend_range_fp8(int dtype, int Hkv, int D, int bs, int NB, int MBS,
                            const uint16_t *qrow, const uint8_t *kc, const uint8_t *vc,
                            double ks, double vs, const int32_t *tables, int s, int kvh,
                            int L, double scale, double *x, double *acc, double *l_out)
{
    double m = -INFINITY;
    for (int j = 0; j < L; ++j) {
        long long r = token_row(tables, MBS, s, j, bs, NB, Hkv, D, kvh);
        if (r < 0) return -2;
        double dot = 0.0;
        for (int d = 0; d < D; ++d)
            dot += widen(dtype, qrow[d]) * (oracle_e4m3_to_f64(kc[r + d]) * ks);
        x[j] = dot * scale;
        m = x[j] > m ? x[j] : m;
    }
    double l = 0.0;
    for (int d = 0; d < D; ++d) acc[d] = 0.0;
    for (int j = 0; j < L; ++j) {
        double w = exp(x[j] - m);
        l += w;
        long long r = token_row(tables, MBS, s, j, bs, NB, Hkv, D, kvh);
        for (int d = 0; d < D; ++d)
            acc[d] += w * (oracle_e4m3_to_f64(vc[r + d]) * vs);
    }
    *l_out = l;
    return 0;
}

/* out: double [S][Hq][D]; dtype is that of q (fp16 or bf16). */
int oracle_decode_fp8(int dtype, int S, int Hq, int Hkv, int D, int bs, int NB, int MBS,
                      const uint16_t *q, const uint8_t *k_cache, const uint8_t *v_cache,
                      const float *k_scale, const float *v_scale, const int32_t *block_tables,
                      const int32_t *context_lens, double scale, double *out, int num_threads)
{
    if (!shape_ok(dtype, S, Hq, Hkv, D, bs, NB, MBS)) return -1;
    for (int s = 0; s < S; ++s)
        if (context_lens[s] < 0 || (long long)context_lens[s] > (long long)MBS * bs) return -1;
    int g = Hq / Hkv;
    int err = 0;
    int nt = resolve_threads(num_threads);
    long long total = (long long)S * Hq;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nt) reduction(| : err)
    for (long long sh = 0; sh < total; ++sh) {
        int s = (int)(sh / Hq), h = (int)(sh % Hq);
        int L = context_lens[s];
        double *o = out + sh * D;
        if (L == 0) {
            for (int d = 0; d < D; ++d) o[d] = 0.0;
            continue;
        }
        double *x = (double *)malloc(sizeof(double) * (size_t)L);
        double *acc = (double *)malloc(sizeof(double) * (size_t)D);
        double lsum;
        int kvh = h / g;
        int rc = attend_range_fp8(dtype, Hkv, D, bs, NB, MBS, q + sh * D, k_cache, v_cache,
                                  (double)k_scale[kvh], (double)v_scale[kvh], block_tables, s,
                                  kvh, L, scale, x, acc, &lsum);
        if (rc) err |= 1;
        else
            for (int d = 0; d < D; ++d) o[d] = acc[d] / lsum;
        free(x);
        free(acc);
    }
    return err ? -2 : 0;
}

/* Append into an FP8 cache: k, v are [num_tokens][Hkv][D] in dtype (fp16 or
 * bf16); the codes of token t go to slot slot_mapping[t] (negative: skipped). */
int oracle_cache_append_fp8(int dtype, long long num_slots, int Hkv, int D, int num_tokens,
                            const uint16_t *k, const uint16_t *v, const int32_t *slot_mapping,
                            const float *k_scale, const float *v_scale, uint8_t *k_cache,
                            uint8_t *v_cache)
{
    if ((dtype != ORACLE_F16 && dtype != ORACLE_BF16) || num_slots < 0 || Hkv <= 0 || D <= 0 ||
        num_tokens < 0)
        return -1;
    long long row = (long long)Hkv * D;
    for (int t = 0; t < num_tokens; ++t) {
        long long slot = slot_mapping[t];
        if (slot < 0) continue;
        if (slot >= num_slots) return -2;
        for (long long i = 0; i < row; ++i) {
            int h = (int)(i / D);
            float xk = (float)widen(dtype, k[(long long)t * row + i]);
            float xv = (float)widen(dtype, v[(long long)t * row + i]);
            k_cache[slot * row + i] = oracle_e4m3_from_f32(xk / k_scale[h]);
            v_cache[slot * row + i] = oracle_e4m3_from_f32(xv / v_scale[h]);
        }
    }
    return 0;
}

/* ---------------------------------------------------------------------
 * Tq query tokens per sequence, causal over the new tokens.
 * q: [S][Tq][Hq][D]; out: double [S][Tq][Hq][D]. */
int oracle_decode_multi(int dtype, int S, int Tq, int Hq, int Hkv, int D, int bs, int NB,
                        int MBS, const uint16_t *q, const uint16_t *k_cache,
                        const uint16_t *v_cache, const int32_t *block_tables,
                        const int32_t *context_lens, double scale, double *out, int num_threads)
{
    if (!shape_ok(dtype, S, Hq, Hkv, D, bs, NB, MBS) || Tq <= 0) return -1;
    for (int s = 0; s < S; ++s)
        if (context_lens[s] < 0 || (long long)context_lens[s] > (long long)MBS * bs) return -1;
    int g = Hq / Hkv;
    int err = 0;
    int nt = resolve_threads(num_threads);
    long long total = (long long)S * Tq * Hq;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nt) reduction(| : err)
    for (long long row = 0; row < total; ++row) {
        int h = (int)(row % Hq);
        long long st = row / Hq;
        int t = (int)(st % Tq), s = (int)(st / Tq);
        int last = context_lens[s] - Tq + t;   /* last token this query sees */
        double *o = out + row * D;
        if (last < 0) {
            for (int d = 0; d < D; ++d) o[d] = 0.0;
            continue;
        }
        int L = last + 1;
        double *x = (double *)malloc(sizeof(double) * (size_t)L);
        double *acc = (double *)malloc(sizeof(double) * (size_t)D);
        double m, l;
        int kv_head = h / g;
        int rc = attend_range(dtype, Hkv, D, bs, NB, MBS, q + row * D, k_cache, v_cache,
                              block_tables, s, kv_head, 0, L, scale, x, &m, &l, acc);
        if (rc) err |= 1;
        else {
            double inv = 1.0 / l;
            for (int d = 0; d < D; ++d) o[d] = acc[d] * inv;
        }
        free(x);
        free(acc);
    }
    return err ? -2 : 0;
}

/* Swap: for each pair, dst block pairs[2i+1] of (dst_k, dst_v) becomes a copy
 * of src block pairs[2i] of (src_k, src_v).  The pools are distinct; blocks
 * hold block_bytes bytes. */
int oracle_swap_blocks(int src_blocks, int dst_blocks, long long block_bytes, int num_pairs,
                       const int32_t *pairs, const uint8_t *src_k, const uint8_t *src_v,
                       uint8_t *dst_k, uint8_t *dst_v)
{
    if (src_blocks < 0 || dst_blocks < 0 || block_bytes <= 0 || num_pairs < 0) return -1;
    for (int i = 0; i < num_pairs; ++i) {
        int from = pairs[2 * i], to = pairs[2 * i + 1];
        if (from < 0 || from >= src_blocks || to < 0 || to >= dst_blocks) return -2;
        memcpy(dst_k + (long long)to * block_bytes, src_k + (long long)from * block_bytes,
               (size_t)block_bytes);
        memcpy(dst_v + (long long)to * block_bytes, src_v + (long long)from * block_bytes,
               (size_t)block_bytes);
    }
    return 0;
}
