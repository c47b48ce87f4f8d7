/*
 * Paged decode attention, computed the slow and obvious way in fp64.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the oracle that the CUDA path is
 * checked against.  Only the tests, the package's smoke check and the bench's
 * CPU-baseline leg may load it; the product path never calls it and shares no
 * code, header, table or constant with it.
 *
 * What it computes (the plain definition, no partitions, no online softmax):
 * for every sequence s and query head h,
 *     g     = h / (num_heads / num_kv_heads)         (consecutive q heads share a kv head)
 *     T     = seq_lens[s]
 *     for t in [0, T): pb = block_tables[s][t / block_size], o = t % block_size
 *         K_t[d] = key_cache  [pb][g][d / x][o][d % x]
 *         V_t[d] = value_cache[pb][g][d][o]
 *     l_t   = scale * sum_d q[s][h][d] * K_t[d]
 *     p_t   = exp(l_t - max_t l_t)
 *     out   = sum_t p_t V_t / sum_t p_t              (out = 0 when T = 0)
 *
 * Sources on the pages:
 *  - block table as a page table, and the address of a logical block:
 *    "Why PagedAttention was retired", section 1 (block_table row pointer and
 *    physical_block_number loaded as a 64-bit integer); the PagedAttention
 *    idea in "vLLM 0.25.0 release notes", section 1 (sequence = process,
 *    block = page, block table = page table).
 *  - cache layouts: "Why PagedAttention was retired", section 2 (the k_cache
 *    5-D and v_cache 4-D comments).
 *  - the computation itself: the same page, section 3 (logits and softmax,
 *    then the softmax-weighted V), with the formula softmax(q K^T scale) V.
 *  - FP8 storage: section 4 of the same page (e4m3 codes, converted on load
 *    and multiplied by the per-tensor k_scale / v_scale).
 *
 * Readings where the pages are silent (each one is listed in the design notes):
 *  - x = 16 bytes / element size is passed in by the caller;
 *  - e4m3 is the OCP "fn" variant: bias 7, no infinities, S.1111.111 = NaN;
 *  - dequantised values are code * scale, formed exactly in fp64;
 *  - seq_len = 0 gives a zero output row; no causal mask (decode reads all T).
 *
 * Optional ALiBi bias: the call on "PR #47361 report: Delete PagedAttention"
 * (benchmark snippet) carries an alibi_slopes argument but the pages do not
 * print the bias.  Reading: the usual linear bias, per query head,
 *     l_t += slope[h] * (t - (T - 1))
 * i.e. the key position minus the decoding query's position T - 1.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_KV_BF16 0
#define ORACLE_KV_E4M3 1

/* bf16 is the top half of an IEEE binary32; widening is exact. */
double oracle_bf16_to_double(uint16_t bits) {
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* OCP E4M3 (fn): 1 sign, 4 exponent (bias 7), 3 mantissa bits.
 * exponent 0 -> subnormal m * 2^-9; S.1111.111 -> NaN; no infinities. */
double oracle_e4m3_to_double(uint8_t code) {
    int sign = code >> 7;
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    double v;
    if (e == 0xF && m == 0x7) return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);
    else
        v = ldexp((double)(8 + m), e - 10); /* (1 + m/8) * 2^(e-7) */
    return sign ? -v : v;
}

/* The 256 e4m3 values, each from oracle_e4m3_to_double (a cache of that
 * function's results, so a long e4m3 sequence does not redo the ldexp per
 * element).  Filled before any worker thread reads it. */
static double e4m3_value[256];
static int e4m3_value_ready = 0;

static void fill_e4m3_values(void) {
    int c;
    if (e4m3_value_ready) return;
    for (c = 0; c < 256; ++c) e4m3_value[c] = oracle_e4m3_to_double((uint8_t)c);
    e4m3_value_ready = 1;
}

static double load_elem(const void* base, int64_t idx, int kv_dtype, double scl) {
    if (kv_dtype == ORACLE_KV_BF16)
        return oracle_bf16_to_double(((const uint16_t*)base)[idx]);
    return e4m3_value[((const uint8_t*)base)[idx]] * scl;
}

/* One (s, h) output row.  logit: scratch of at least T doubles. */
static void one_row(double* out_row, const uint16_t* q_row, const void* key_cache,
                    const void* value_cache, int kv_dtype, int Hk, int D, int B, int x,
                    double scale, const int32_t* bt_row, int T, int g, double k_scale,
                    double v_scale, double slope, double* logit) {
    int d, t;
    double qd[512];
    for (d = 0; d < D; ++d) qd[d] = oracle_bf16_to_double(q_row[d]);
    for (d = 0; d < D; ++d) out_row[d] = 0.0;
    if (T <= 0) return;

    /* logits */
    double mx = -INFINITY;
    for (t = 0; t < T; ++t) {
        int64_t pb = (int64_t)bt_row[t / B];
        int o = t % B;
        double acc = 0.0;
        for (d = 0; d < D; ++d) {
            int64_t ki = ((((pb * Hk + g) * (D / x) + d / x) * B + o) * x) + d % x;
            acc += qd[d] * load_elem(key_cache, ki, kv_dtype, k_scale);
        }
        logit[t] = scale * acc + slope * (double)(t - (T - 1));
        if (logit[t] > mx) mx = logit[t];
    }
    /* softmax weights and the weighted sum of V */
    double denom = 0.0;
    for (t = 0; t < T; ++t) {
        int64_t pb = (int64_t)bt_row[t / B];
        int o = t % B;
        double p = exp(logit[t] - mx);
        denom += p;
        for (d = 0; d < D; ++d) {
            int64_t vi = ((pb * Hk + g) * D + d) * B + o;
            out_row[d] += p * load_elem(value_cache, vi, kv_dtype, v_scale);
        }
    }
    for (d = 0; d < D; ++d) out_row[d] /= denom;
}

/*
 * alibi_slopes: fp32 [Hq] or NULL (no bias).
 * out:        fp64 [n_rows][D]; rows are (s, h) in row-major order when
 *             pairs == NULL (n_rows = S * Hq), else pairs[2i], pairs[2i+1].
 * query:      bf16 bits [S][Hq][D]
 * key_cache:  bf16 bits or e4m3 codes, [num_blocks][Hk][D/x][B][x]
 * value_cache:bf16 bits or e4m3 codes, [num_blocks][Hk][D][B]
 * Returns 0, or -1 on an argument the definition cannot take.
 */
int oracle_pa_decode(double* out, const uint16_t* query, const void* key_cache,
                     const void* value_cache, int kv_dtype, int S, int Hq, int Hk, int D, int B,
                     int x, double scale, const int32_t* block_tables, int max_blocks_per_seq,
                     const int32_t* seq_lens, double k_scale, double v_scale, int n_pairs,
                     const int32_t* pairs, int n_threads, const float* alibi_slopes) {
    if (S < 0 || Hq <= 0 || Hk <= 0 || Hq % Hk || D <= 0 || D > 512 || B <= 0 || x <= 0 ||
        D % x)
        return -1;
    int G = Hq / Hk;
    int n_rows = pairs ? n_pairs : S * Hq;
    fill_e4m3_values();
    int max_T = 0, i;
    for (i = 0; i < S; ++i)
        if (seq_lens[i] > max_T) max_T = seq_lens[i];
    for (i = 0; i < S; ++i)
        if (seq_lens[i] > max_blocks_per_seq * B) return -1;
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#else
    (void)n_threads;
#endif
    int bad = 0;
#pragma omp parallel reduction(| : bad)
    {
        double* logit = (double*)malloc(sizeof(double) * (size_t)(max_T > 0 ? max_T : 1));
        if (!logit) bad = 1;
#pragma omp for schedule(dynamic, 1)
        for (i = 0; i < n_rows; ++i) {
            if (!logit) continue;
            int s = pairs ? pairs[2 * i] : i / Hq;
            int h = pairs ? pairs[2 * i + 1] : i % Hq;
            if (s < 0 || s >= S || h < 0 || h >= Hq) {
                bad = 1;
                continue;
            }
            one_row(out + (int64_t)i * D, query + ((int64_t)s * Hq + h) * D, key_cache,
                    value_cache, kv_dtype, Hk, D, B, x, scale,
                    block_tables + (int64_t)s * max_blocks_per_seq, seq_lens[s], h / G, k_scale,
                    v_scale, alibi_slopes ? (double)alibi_slopes[h] : 0.0, logit);
        }
        free(logit);
    }
    return bad ? -1 : 0;
}

/* Threads the OpenMP runtime would use for a parallel region. */
int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
