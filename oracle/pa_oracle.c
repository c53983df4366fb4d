/*
 * pa_oracle.c -- plain fp64 CPU oracle for paged-KV attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no code, header, table or helper with
 * the CUDA library; it reads the same documented cache layout independently.
 *
 * What it computes (sources, by page title and section):
 *   - "Production Serving: Continuous Batching and PagedAttention",
 *     The Build, Step 4 "Implement the paged KV cache": a token's K and V go
 *     to slot (length mod 16) of the page named by the page table.
 *   - same page, Step 6 "Implement attention over paged storage": for every
 *     logical block, look up the physical page, score each stored token
 *     against the query divided by sqrt(head_dim), softmax over the sequence,
 *     sum the softmax-weighted values.  Read per query head (the printed
 *     step sums the dot product over all heads at once, which cannot be what
 *     attention means for a multi-head query).
 *   - "Continuous batching and PagedAttention" (How the scheduler works):
 *     chunked prefill -- a prompt chunk attends causally to everything stored
 *     before it plus itself.
 *   - same page (PagedAttention: KV cache memory): blocks shared by
 *     copy-on-write are copied when a sharer diverges.
 *
 * Readings taken where the pages are silent:
 *   - cache layout: separate K and V caches, each [num_blocks][Hkv][16][D];
 *   - grouped-query attention: query head h reads kv head floor(h*Hkv/Hq);
 *   - slot mapping: slot = physical_block*16 + offset, slot < 0 is padding;
 *   - fp8 cache: OCP 8-bit floating point E4M3 ("fn" variant: no infinities,
 *     S.1111.111 is NaN, largest finite 448).  Encoding multiplies the
 *     value by the fp32 reciprocal of the per-head scale (one IEEE fp32
 *     multiply, round to nearest even), then rounds to E4M3 with round to
 *     nearest even, saturating finite overflow and infinities to +-448;
 *     decoding multiplies the E4M3 value by the per-head scale;
 *   - seq_len == 0 yields an all-zero output row.
 *
 * Precision: every arithmetic step is IEEE double.  bf16 -> double and
 * E4M3 -> double are exact.
 *
 * Return value of every entry point: 0 on success, a negative number if an
 * index read from the metadata points outside the cache or the arguments are
 * inconsistent.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_BLOCK 16

enum { ORACLE_BF16 = 0, ORACLE_FP8_E4M3 = 1 };

/* ---------------------------------------------------------------- numbers */

/* bf16 is the top half of an IEEE binary32; widening is exact. */
double oracle_bf16_to_double(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* OCP FP8 E4M3: sign bit, 4 exponent bits (bias 7), 3 mantissa bits.
 * exponent field 0 -> subnormal m * 2^-9; S.1111.111 -> NaN. */
double oracle_e4m3_to_double(uint8_t code) {
    int sign = code >> 7;
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    double mag;
    if (e == 0xF && m == 0x7) return NAN;
    if (e == 0)
        mag = ldexp((double)m, -9);
    else
        mag = ldexp(1.0 + m / 8.0, e - 7);
    return sign ? -mag : mag;
}

/* Round a binary32 value to E4M3: nearest, ties to even; finite overflow and
 * infinities saturate to +-448; NaN -> 0x7F.  -0 keeps its sign. */
uint8_t oracle_e4m3_from_float(float xf) {
    double x = (double)xf;
    uint8_t sign = signbit(xf) ? 0x80 : 0x00;
    if (isnan(xf)) return 0x7F;
    double a = fabs(x);
    if (a >= 448.0) return (uint8_t)(sign | 0x7E); /* includes +-inf */
    if (a < ldexp(1.0, -6)) {
        /* subnormal range: quantum 2^-9; 8 quanta is the smallest normal,
         * whose code (exponent field 1, mantissa 0) is also 8. */
        double n = nearbyint(a * 512.0); /* exact scaling, RNE */
        return (uint8_t)(sign | (uint8_t)n);
    }
    int k;
    frexp(a, &k);      /* a = f * 2^k, f in [0.5, 1) */
    int e = k - 1;     /* a in [2^e, 2^(e+1)), e in [-6, 8] */
    double q = ldexp(a, 3 - e); /* in [8, 16): mantissa with hidden bit */
    double n = nearbyint(q);
    if (n == 16.0) {
        n = 8.0;
        e += 1;
    }
    /* a < 448 guarantees the rounded value is at most 448 (e=8, n=14). */
    return (uint8_t)(sign | (uint8_t)(((e + 7) << 3) | ((int)n - 8)));
}

static double load_elem(const void *cache, int dtype, size_t idx, double scale) {
    if (dtype == ORACLE_BF16) return oracle_bf16_to_double(((const uint16_t *)cache)[idx]);
    return oracle_e4m3_to_double(((const uint8_t *)cache)[idx]) * scale;
}

/* index of element d of token slot `slot` of kv head `kvh` in physical block `blk` */
static size_t cache_index(int64_t blk, int kvh, int slot, int d, int Hkv, int D) {
    return (((size_t)blk * (size_t)Hkv + (size_t)kvh) * ORACLE_BLOCK + (size_t)slot) * (size_t)D + (size_t)d;
}

/* ----------------------------------------------------------------- writes */

/* Slot-mapped write of T new tokens.  k, v: bf16 [T][Hkv][D].
 * For token t with slot s >= 0, block s/16, offset s%16 receives k[t], v[t];
 * for an fp8 cache each element is encoded as described in the header. */
int oracle_write_kv(const uint16_t *k, const uint16_t *v, const int64_t *slot_mapping, int64_t T,
                    void *k_cache, void *v_cache, int dtype, int64_t num_blocks, int Hkv, int D,
                    const float *k_scale, const float *v_scale) {
    for (int64_t t = 0; t < T; ++t) {
        int64_t s = slot_mapping[t];
        if (s < 0) continue;
        int64_t blk = s / ORACLE_BLOCK;
        int off = (int)(s % ORACLE_BLOCK);
        if (blk >= num_blocks) return -1;
        for (int h = 0; h < Hkv; ++h) {
            for (int d = 0; d < D; ++d) {
                size_t src = ((size_t)t * Hkv + h) * D + d;
                size_t dst = cache_index(blk, h, off, d, Hkv, D);
                if (dtype == ORACLE_BF16) {
                    ((uint16_t *)k_cache)[dst] = k[src];
                    ((uint16_t *)v_cache)[dst] = v[src];
                } else {
                    float kinv = 1.0f / k_scale[h];
                    float vinv = 1.0f / v_scale[h];
                    uint32_t ku = ((uint32_t)k[src]) << 16, vu = ((uint32_t)v[src]) << 16;
                    float kf, vf;
                    memcpy(&kf, &ku, 4);
                    memcpy(&vf, &vu, 4);
                    float kx = kf * kinv; /* one binary32 multiply */
                    float vx = vf * vinv;
                    ((uint8_t *)k_cache)[dst] = oracle_e4m3_from_float(kx);
                    ((uint8_t *)v_cache)[dst] = oracle_e4m3_from_float(vx);
                }
            }
        }
    }
    return 0;
}

/* Copy-on-write block copy: for each pair (src, dst) every element of
 * physical block src (all kv heads, all 16 slots) is copied to block dst,
 * in both caches.  Pairs are applied in order. */
int oracle_copy_blocks(void *k_cache, void *v_cache, const int32_t *pairs, int n_pairs, int dtype,
                       int64_t num_blocks, int Hkv, int D) {
    size_t esz = dtype == ORACLE_BF16 ? 2 : 1;
    size_t block_bytes = (size_t)Hkv * ORACLE_BLOCK * (size_t)D * esz;
    for (int i = 0; i < n_pairs; ++i) {
        int64_t s = pairs[2 * i], d = pairs[2 * i + 1];
        if (s < 0 || d < 0 || s >= num_blocks || d >= num_blocks) return -1;
        memmove((char *)k_cache + (size_t)d * block_bytes, (char *)k_cache + (size_t)s * block_bytes, block_bytes);
        memmove((char *)v_cache + (size_t)d * block_bytes, (char *)v_cache + (size_t)s * block_bytes, block_bytes);
    }
    return 0;
}

/* -------------------------------------------------------------- attention */

/* Dense softmax attention of one query row (D doubles, already decoded)
 * against logical tokens 0..n-1 of one sequence reached through `table`.
 * out[d] = sum_t softmax_t(scale * q.k_t) * v_t[d]. */
static int attend_one(double *out, const double *q, const int32_t *table, int n, const void *k_cache,
                      const void *v_cache, int dtype, int64_t num_blocks, int Hkv, int kvh, int D, double scale,
                      double ks, double vs, double *s) {
    for (int d = 0; d < D; ++d) out[d] = 0.0;
    if (n <= 0) return 0;
    for (int t = 0; t < n; ++t) {
        int64_t blk = table[t / ORACLE_BLOCK];
        if (blk < 0 || blk >= num_blocks) return -1;
        double acc = 0.0;
        for (int d = 0; d < D; ++d)
            acc += q[d] * load_elem(k_cache, dtype, cache_index(blk, kvh, t % ORACLE_BLOCK, d, Hkv, D), ks);
        s[t] = scale * acc;
    }
    double m = s[0];
    for (int t = 1; t < n; ++t)
        if (s[t] > m) m = s[t];
    double z = 0.0;
    for (int t = 0; t < n; ++t) {
        s[t] = exp(s[t] - m);
        z += s[t];
    }
    for (int t = 0; t < n; ++t) {
        int64_t blk = table[t / ORACLE_BLOCK];
        for (int d = 0; d < D; ++d)
            out[d] += s[t] * load_elem(v_cache, dtype, cache_index(blk, kvh, t % ORACLE_BLOCK, d, Hkv, D), vs);
    }
    for (int d = 0; d < D; ++d) out[d] /= z;
    return 0;
}

static void set_threads(int nthreads) {
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
}

/* Paged decode: q bf16 [B][Hq][D]; out double [B][Hq][D].
 * Sequence b attends its tokens 0..seq_lens[b]-1 through row b of
 * block_tables [B][max_blocks]. */
int oracle_decode(double *out, const uint16_t *q, const void *k_cache, const void *v_cache, int dtype,
                  const int32_t *block_tables, const int32_t *seq_lens, int B, int max_blocks, int Hq, int Hkv,
                  int D, int64_t num_blocks, double scale, const float *k_scale, const float *v_scale,
                  int nthreads) {
    if (Hkv <= 0 || Hq % Hkv != 0) return -2;
    int status = 0;
    set_threads(nthreads);
#pragma omp parallel
    {
        double *qd = (double *)malloc(sizeof(double) * D);
        int cap = max_blocks * ORACLE_BLOCK;
        double *s = (double *)malloc(sizeof(double) * (cap > 0 ? cap : 1));
#pragma omp for schedule(dynamic, 1)
        for (long bh = 0; bh < (long)B * Hq; ++bh) {
            int b = (int)(bh / Hq), h = (int)(bh % Hq);
            int kvh = (int)((long)h * Hkv / Hq);
            int n = seq_lens[b];
            if (n > cap) {
#pragma omp atomic write
                status = -1;
                continue;
            }
            for (int d = 0; d < D; ++d) qd[d] = oracle_bf16_to_double(q[((size_t)b * Hq + h) * D + d]);
            double ks = dtype == ORACLE_BF16 ? 1.0 : (double)k_scale[kvh];
            double vs = dtype == ORACLE_BF16 ? 1.0 : (double)v_scale[kvh];
            int r = attend_one(out + ((size_t)b * Hq + h) * D, qd, block_tables + (size_t)b * max_blocks, n,
                               k_cache, v_cache, dtype, num_blocks, Hkv, kvh, D, scale, ks, vs, s);
            if (r) {
#pragma omp atomic write
                status = r;
            }
        }
        free(qd);
        free(s);
    }
    return status;
}

/* Split-K decode with a log-sum-exp merge.  Partition p of a sequence covers
 * tokens [p*P, min((p+1)*P, len)).  Each partition yields its running max m_p,
 * its normaliser l_p = sum exp(s - m_p) and its normalised output
 * o_p = sum exp(s - m_p) v / l_p; the merge takes M = max_p m_p,
 * w_p = l_p * exp(m_p - M) and out = sum_p w_p o_p / sum_p w_p. */
int oracle_decode_split(double *out, const uint16_t *q, const void *k_cache, const void *v_cache, int dtype,
                        const int32_t *block_tables, const int32_t *seq_lens, int B, int max_blocks, int Hq,
                        int Hkv, int D, int64_t num_blocks, double scale, const float *k_scale,
                        const float *v_scale, int partition_tokens, int nthreads) {
    if (Hkv <= 0 || Hq % Hkv != 0 || partition_tokens <= 0) return -2;
    int status = 0;
    set_threads(nthreads);
#pragma omp parallel
    {
        int cap = max_blocks * ORACLE_BLOCK;
        int maxp = cap / partition_tokens + 2;
        double *qd = (double *)malloc(sizeof(double) * D);
        double *s = (double *)malloc(sizeof(double) * (cap > 0 ? cap : 1));
        double *op = (double *)malloc(sizeof(double) * (size_t)maxp * D);
        double *mp = (double *)malloc(sizeof(double) * maxp);
        double *lp = (double *)malloc(sizeof(double) * maxp);
#pragma omp for schedule(dynamic, 1)
        for (long bh = 0; bh < (long)B * Hq; ++bh) {
            int b = (int)(bh / Hq), h = (int)(bh % Hq);
            int kvh = (int)((long)h * Hkv / Hq);
            int n = seq_lens[b];
            double *o = out + ((size_t)b * Hq + h) * D;
            const int32_t *table = block_tables + (size_t)b * max_blocks;
            for (int d = 0; d < D; ++d) o[d] = 0.0;
            if (n > cap) {
#pragma omp atomic write
                status = -1;
                continue;
            }
            if (n <= 0) continue;
            for (int d = 0; d < D; ++d) qd[d] = oracle_bf16_to_double(q[((size_t)b * Hq + h) * D + d]);
            double ks = dtype == ORACLE_BF16 ? 1.0 : (double)k_scale[kvh];
            double vs = dtype == ORACLE_BF16 ? 1.0 : (double)v_scale[kvh];
            int np = (n + partition_tokens - 1) / partition_tokens;
            int bad = 0;
            for (int p = 0; p < np; ++p) {
                int t0 = p * partition_tokens;
                int t1 = t0 + partition_tokens < n ? t0 + partition_tokens : n;
                for (int t = t0; t < t1; ++t) {
                    int64_t blk = table[t / ORACLE_BLOCK];
                    if (blk < 0 || blk >= num_blocks) {
                        bad = 1;
                        break;
                    }
                    double acc = 0.0;
                    for (int d = 0; d < D; ++d)
                        acc += qd[d] *
                               load_elem(k_cache, dtype, cache_index(blk, kvh, t % ORACLE_BLOCK, d, Hkv, D), ks);
                    s[t] = scale * acc;
                }
                if (bad) break;
                double m = s[t0];
                for (int t = t0 + 1; t < t1; ++t)
                    if (s[t] > m) m = s[t];
                double l = 0.0;
                double *opp = op + (size_t)p * D;
                for (int d = 0; d < D; ++d) opp[d] = 0.0;
                for (int t = t0; t < t1; ++t) {
                    double w = exp(s[t] - m);
                    int64_t blk = table[t / ORACLE_BLOCK];
                    l += w;
                    for (int d = 0; d < D; ++d)
                        opp[d] +=
                            w * load_elem(v_cache, dtype, cache_index(blk, kvh, t % ORACLE_BLOCK, d, Hkv, D), vs);
                }
                for (int d = 0; d < D; ++d) opp[d] /= l;
                mp[p] = m;
                lp[p] = l;
            }
            if (bad) {
#pragma omp atomic write
                status = -1;
                continue;
            }
            double M = mp[0];
            for (int p = 1; p < np; ++p)
                if (mp[p] > M) M = mp[p];
            double W = 0.0;
            for (int p = 0; p < np; ++p) {
                double w = lp[p] * exp(mp[p] - M);
                W += w;
                for (int d = 0; d < D; ++d) o[d] += w * op[(size_t)p * D + d];
            }
            for (int d = 0; d < D; ++d) o[d] /= W;
        }
        free(qd);
        free(s);
        free(op);
        free(mp);
        free(lp);
    }
    return status;
}

/* Causal chunked prefill.  Chunk c owns query rows cu_q[c]..cu_q[c+1]-1 of
 * q bf16 [sum C][Hq][D].  Its i-th query sits at absolute position
 * prefix_lens[c] + i and attends keys 0..prefix_lens[c]+i (inclusive) of the
 * sequence reached through row c of block_tables; the chunk's own keys are
 * already in the cache.  out double [sum C][Hq][D]. */
int oracle_prefill(double *out, const uint16_t *q, const int32_t *cu_q, const int32_t *prefix_lens,
                   const int32_t *block_tables, int n_chunks, int max_blocks, int Hq, int Hkv, int D,
                   const void *k_cache, const void *v_cache, int dtype, int64_t num_blocks, double scale,
                   const float *k_scale, const float *v_scale, int nthreads) {
    if (Hkv <= 0 || Hq % Hkv != 0) return -2;
    int status = 0;
    int total = cu_q[n_chunks];
    set_threads(nthreads);
#pragma omp parallel
    {
        int cap = max_blocks * ORACLE_BLOCK;
        double *qd = (double *)malloc(sizeof(double) * D);
        double *s = (double *)malloc(sizeof(double) * (cap > 0 ? cap : 1));
#pragma omp for schedule(dynamic, 4)
        for (long rh = 0; rh < (long)total * Hq; ++rh) {
            int row = (int)(rh / Hq), h = (int)(rh % Hq);
            int c = 0;
            while (c + 1 < n_chunks && cu_q[c + 1] <= row) ++c;
            int i = row - cu_q[c];
            int n = prefix_lens[c] + i + 1;
            int kvh = (int)((long)h * Hkv / Hq);
            if (n > cap) {
#pragma omp atomic write
                status = -1;
                continue;
            }
            for (int d = 0; d < D; ++d) qd[d] = oracle_bf16_to_double(q[((size_t)row * Hq + h) * D + d]);
            double ks = dtype == ORACLE_BF16 ? 1.0 : (double)k_scale[kvh];
            double vs = dtype == ORACLE_BF16 ? 1.0 : (double)v_scale[kvh];
            int r = attend_one(out + ((size_t)row * Hq + h) * D, qd, block_tables + (size_t)c * max_blocks, n,
                               k_cache, v_cache, dtype, num_blocks, Hkv, kvh, D, scale, ks, vs, s);
            if (r) {
#pragma omp atomic write
                status = r;
            }
        }
        free(qd);
        free(s);
    }
    return status;
}

/* Number of threads an OpenMP region of this library would use. */
int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
