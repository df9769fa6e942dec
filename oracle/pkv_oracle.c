/*
 * pkv_oracle.c -- CPU oracle for the paged KV-cache hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may include, link or
 * call this file.  Only the tests, the smoke check and the bench's CPU-baseline
 * leg use it.  It shares no code, header, table or helper with the CUDA library.
 *
 * It is deliberately plain and slow: every value is carried in fp64, the cache
 * is gathered into a contiguous per-request K/V first, and attention is then
 * the textbook formula.  There is no blocking, fusion or reordering beyond what
 * the definition states.  OpenMP spreads independent (request, query head)
 * pairs over host threads; each pair is computed by one thread in plain order.
 *
 * Sources (web pages on the subject; cited by title and section):
 *   [KVOPT]  "KV Cache Optimization and PagedAttention" -- intro prose (cache
 *            size formula, blocks + per-request block table, shared prefix
 *            blocks) and its byte/waste code example.
 *   [PAMEM]  "PagedAttention: Optimizing KV Cache Utilization in Large Language
 *            Models" -- sections "The Mechanics of PagedAttention" (logical vs
 *            physical blocks, page table, scattered writes) and "The Math: Block
 *            Attention Calculation" (Softmax(q K^T / sqrt(d_k)) after a page-table
 *            lookup of each K_j).
 *   [KVMGMT] "KV Cache Management" -- sections "The Solution: PagedAttention
 *            (vLLM)" (fixed-size blocks, block table) and "The Bonus: Zero-Copy
 *            Sharing" (block tables of many users point at one physical block).
 *
 * Readings where the pages are silent or garbled (each one is a convention the
 * CUDA library follows too; they are interfaces, not shared code):
 *   R1  [PAMEM] "The Math" prints a softmax per block b.  Normalising each block
 *       alone is not attention; the formula is read as the block's slice of ONE
 *       softmax over all L_b tokens of the request.
 *   R2  The scale is an explicit argument (1/sqrt(d_k) in every workload).
 *   R3  seq_lens count tokens AFTER the new token was appended; the new token
 *       sits at position L_b-1 and is attended to.
 *   R4  GQA: query head h reads KV head h / (Hq/Hkv) (consecutive grouping).
 *   R5  Cache layout [num_blocks, Hkv, block_size, head_dim]; slot encoding
 *       slot = physical_block * block_size + offset; slot < 0 = padding, skipped.
 *   R6  Block-table entries past ceil(L_b / block_size) are never read.
 *   R7  L_b == 0 gives an all-zero output row (softmax of an empty set).
 *
 * Element types: 0 = fp32, 1 = bf16 (upper 16 bits of an fp32, so the upcast is
 * exact), 2 = fp8 e4m3 (1 sign, 4 exponent bits with bias 7, 3 mantissa bits;
 * exponent field 0 is subnormal; S.1111.111 is NaN; there is no infinity) whose
 * stored value is multiplied by a per-kv-head fp32 scale.
 *
 * Build: gcc -O2 -fopenmp -shared -fPIC (see oracle/__init__.py).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Mutation hooks for the oracle's own self-test: the test suite rebuilds this
 * file with ORACLE_MUTANT=n to plant one plausible mistake and checks that the
 * pins catch it.  The normal build has ORACLE_MUTANT == 0, which compiles none
 * of them. */
#ifndef ORACLE_MUTANT
#define ORACLE_MUTANT 0
#endif

enum { OR_F32 = 0, OR_BF16 = 1, OR_FP8E4M3 = 2 };

/* ---- element decoding (exact) ------------------------------------------- */

static double bf16_bits_to_double(uint16_t b) {
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* fp8 e4m3 decoded from its definition (OCP 8-bit floating point, E4M3). */
static double e4m3_bits_to_double(uint8_t b) {
    int sign = (b >> 7) & 1;
    int e = (b >> 3) & 0xF;
    int m = b & 0x7;
    double v;
    if (e == 0xF && m == 0x7) return NAN;
    int bias = 7, sub_exp = -6;
#if ORACLE_MUTANT == 11
    bias = 8; /* planted: exponent bias of e5m2-like formats */
#endif
#if ORACLE_MUTANT == 12
    sub_exp = -7; /* planted: subnormals one binade too low */
#endif
    if (e == 0)
        v = ldexp((double)m / 8.0, sub_exp);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - bias);
    return sign ? -v : v;
}

static double load_elem(const void* base, size_t i, int dtype) {
    if (dtype == OR_F32) return (double)((const float*)base)[i];
    if (dtype == OR_BF16) return bf16_bits_to_double(((const uint16_t*)base)[i]);
    return e4m3_bits_to_double(((const uint8_t*)base)[i]);
}

/* Index of element (block p, kv head g, offset o, dim k) under layout R5. */
static size_t cache_index(long p, int g, int o, int k, int Hkv, int bs, int d) {
    return (((size_t)p * Hkv + g) * bs + o) * d + k;
}

/* ---- gather (block-table walk) ------------------------------------------- */

/*
 * For request b and kv head g, copy the L tokens' K and V into contiguous fp64
 * rows: logical token t lives in logical block t / bs at offset t % bs, and the
 * block table maps the logical block to a physical one ([KVOPT] intro; [PAMEM]
 * "The Mechanics of PagedAttention"; [KVMGMT] "The Solution").  kscale/vscale
 * (one fp32 per kv head) are applied for the fp8 type, else ignored.
 * Returns -1 if a needed table entry lies outside [0, num_blocks).
 */
static int gather_request(const void* k_cache, const void* v_cache, int kv_dtype,
                          const float* kscale, const float* vscale,
                          const int32_t* table_row, int L, int g, int Hkv, int bs,
                          int d, int num_blocks, double* Kc, double* Vc) {
    for (int t = 0; t < L; ++t) {
        int j = t / bs;
        int o = t % bs;
#if ORACLE_MUTANT == 3
        o = t % d; /* planted: wrong in-block offset */
        if (o >= bs) o = bs - 1;
#endif
        long p = table_row[j];
        if (p < 0 || p >= num_blocks) return -1;
        double ks = 1.0, vs = 1.0;
        if (kv_dtype == OR_FP8E4M3) {
            ks = (double)kscale[g];
            vs = (double)vscale[g];
        }
        for (int k = 0; k < d; ++k) {
            size_t idx = cache_index(p, g, o, k, Hkv, bs, d);
            Kc[(size_t)t * d + k] = load_elem(k_cache, idx, kv_dtype) * ks;
            Vc[(size_t)t * d + k] = load_elem(v_cache, idx, kv_dtype) * vs;
        }
    }
    return 0;
}

/* ---- attention over a contiguous K/V ------------------------------------- */

/*
 * Textbook softmax attention for one query row over L contiguous keys/values
 * ([PAMEM] "The Math", read per R1/R2):
 *   s_t = scale * sum_k q_k K[t][k]
 *   w_t = exp(s_t - max_u s_u) / sum_u exp(s_u - max_u s_u)
 *   out = sum_t w_t V[t]
 * If w is non-NULL the L weights are stored there.
 */
static void attend_contiguous(const double* q, const double* Kc, const double* Vc,
                              int L, int d, double scale, double* s, double* w,
                              double* out) {
    for (int k = 0; k < d; ++k) out[k] = 0.0;
    if (L <= 0) return; /* R7 */
    for (int t = 0; t < L; ++t) {
        double acc = 0.0;
        for (int k = 0; k < d; ++k) acc += q[k] * Kc[(size_t)t * d + k];
#if ORACLE_MUTANT == 4
        s[t] = acc; /* planted: scale dropped */
#else
        s[t] = scale * acc;
#endif
    }
    double M = s[0];
    for (int t = 1; t < L; ++t)
        if (s[t] > M) M = s[t];
    double Z = 0.0;
    for (int t = 0; t < L; ++t) Z += exp(s[t] - M);
    for (int t = 0; t < L; ++t) {
#if ORACLE_MUTANT == 5
        double wt = exp(s[t] - M) / (Z + 1.0); /* planted: bad normaliser */
#else
        double wt = exp(s[t] - M) / Z;
#endif
        if (w) w[t] = wt;
        for (int k = 0; k < d; ++k) {
#if ORACLE_MUTANT == 6
            out[k] += wt * Kc[(size_t)t * d + k]; /* planted: K used for V */
#else
            out[k] += wt * Vc[(size_t)t * d + k];
#endif
        }
    }
}

static int kv_head_of(int h, int Hq, int Hkv) {
#if ORACLE_MUTANT == 1
    return h % Hkv; /* planted: interleaved instead of consecutive grouping */
#else
    return h / (Hq / Hkv); /* R4 */
#endif
}

static int effective_len(const int32_t* seq_lens, int b) {
#if ORACLE_MUTANT == 2
    int L = seq_lens[b] - 1; /* planted: new token not attended (R3 violated) */
    return L < 0 ? 0 : L;
#else
    return seq_lens[b];
#endif
}

/*
 * Paged decode attention, plain definition.
 *   q            [B, Hq, d]          element type q_dtype (fp32 or bf16)
 *   k/v_cache    [NB, Hkv, bs, d]    element type kv_dtype
 *   k/v_scale    [Hkv] fp32          used only for fp8 (may be NULL otherwise)
 *   block_tables [B, max_blocks] int32, seq_lens [B] int32
 *   out          [B, Hq, d] fp64 (written)
 * Returns 0, or -1 if a table entry needed by some request is out of range, or
 * -2 for inconsistent sizes.
 */
int oracle_decode(const void* q, int q_dtype, const void* k_cache,
                  const void* v_cache, int kv_dtype, const float* k_scale,
                  const float* v_scale, const int32_t* block_tables,
                  const int32_t* seq_lens, int B, int Hq, int Hkv, int d, int bs,
                  int max_blocks, int num_blocks, double scale, double* out,
                  int nthreads) {
    if (B < 0 || Hq <= 0 || Hkv <= 0 || d <= 0 || bs <= 0 || Hq % Hkv) return -2;
    for (int b = 0; b < B; ++b) {
        int L = effective_len(seq_lens, b);
        if (L < 0 || (long)L > (long)max_blocks * bs) return -2;
    }
    int status = 0;
    int n_pairs = B * Hq;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel
#endif
    {
        int maxL = 1;
        for (int b = 0; b < B; ++b)
            if (effective_len(seq_lens, b) > maxL) maxL = effective_len(seq_lens, b);
        double* Kc = (double*)malloc(sizeof(double) * (size_t)maxL * d);
        double* Vc = (double*)malloc(sizeof(double) * (size_t)maxL * d);
        double* s = (double*)malloc(sizeof(double) * (size_t)maxL);
        double* qv = (double*)malloc(sizeof(double) * (size_t)d);
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
        for (int pair = 0; pair < n_pairs; ++pair) {
            int b = pair / Hq, h = pair % Hq;
            int g = kv_head_of(h, Hq, Hkv);
            int L = effective_len(seq_lens, b);
            double* o = out + ((size_t)b * Hq + h) * d;
            for (int k = 0; k < d; ++k)
                qv[k] = load_elem(q, ((size_t)b * Hq + h) * d + k, q_dtype);
            if (gather_request(k_cache, v_cache, kv_dtype, k_scale, v_scale,
                               block_tables + (size_t)b * max_blocks, L, g, Hkv, bs,
                               d, num_blocks, Kc, Vc) != 0) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
                status = -1;
                for (int k = 0; k < d; ++k) o[k] = NAN;
                continue;
            }
            attend_contiguous(qv, Kc, Vc, L, d, scale, s, NULL, o);
        }
        free(Kc);
        free(Vc);
        free(s);
        free(qv);
    }
    return status;
}

/*
 * The softmax weights w_t of one (request b, query head h) pair, in token
 * order (L_b values written to w).  Used by the weights-sum-to-one pin.
 */
int oracle_decode_weights(const void* q, int q_dtype, const void* k_cache,
                          const void* v_cache, int kv_dtype, const float* k_scale,
                          const float* v_scale, const int32_t* block_tables,
                          const int32_t* seq_lens, int Hq, int Hkv, int d, int bs,
                          int max_blocks, int num_blocks, double scale, int b, int h,
                          double* w) {
    int L = effective_len(seq_lens, b);
    int g = kv_head_of(h, Hq, Hkv);
    int n = L > 0 ? L : 1;
    double* Kc = (double*)malloc(sizeof(double) * (size_t)n * d);
    double* Vc = (double*)malloc(sizeof(double) * (size_t)n * d);
    double* s = (double*)malloc(sizeof(double) * (size_t)n);
    double* qv = (double*)malloc(sizeof(double) * (size_t)d);
    double* o = (double*)malloc(sizeof(double) * (size_t)d);
    int st = 0;
    for (int k = 0; k < d; ++k)
        qv[k] = load_elem(q, ((size_t)b * Hq + h) * d + k, q_dtype);
    if (gather_request(k_cache, v_cache, kv_dtype, k_scale, v_scale,
                       block_tables + (size_t)b * max_blocks, L, g, Hkv, bs, d,
                       num_blocks, Kc, Vc) != 0)
        st = -1;
    else
        attend_contiguous(qv, Kc, Vc, L, d, scale, s, w, o);
    free(Kc);
    free(Vc);
    free(s);
    free(qv);
    free(o);
    return st;
}

/*
 * Split-and-merge restatement of the same attention, used only to pin the
 * algebra of a split-sequence decode against the plain definition above.
 * The L_b tokens are cut into partitions of P tokens.  Inside a partition the
 * tokens are visited one physical block at a time with a running maximum m,
 * running normaliser l and running weighted sum acc (rescaled by exp(m_old -
 * m_new) whenever m grows).  Partition p ends with (m_p, l_p, acc_p); the
 * merge is M = max_p m_p, out = sum_p exp(m_p - M) acc_p / sum_p exp(m_p - M) l_p.
 */
int oracle_decode_partitioned(const void* q, int q_dtype, const void* k_cache,
                              const void* v_cache, int kv_dtype,
                              const float* k_scale, const float* v_scale,
                              const int32_t* block_tables, const int32_t* seq_lens,
                              int B, int Hq, int Hkv, int d, int bs, int max_blocks,
                              int num_blocks, double scale, int P, double* out) {
    if (P <= 0) return -2;
    int status = 0;
    double* qv = (double*)malloc(sizeof(double) * (size_t)d);
    double* acc = (double*)malloc(sizeof(double) * (size_t)d);
    double* tot = (double*)malloc(sizeof(double) * (size_t)d);
    for (int b = 0; b < B && status == 0; ++b) {
        int L = effective_len(seq_lens, b);
        int n = L > 0 ? L : 1;
        double* Kc = (double*)malloc(sizeof(double) * (size_t)n * d);
        double* Vc = (double*)malloc(sizeof(double) * (size_t)n * d);
        int nparts = (L + P - 1) / P;
        double* pm = (double*)malloc(sizeof(double) * (size_t)(nparts > 0 ? nparts : 1));
        double* pl = (double*)malloc(sizeof(double) * (size_t)(nparts > 0 ? nparts : 1));
        double* pacc = (double*)malloc(sizeof(double) * (size_t)(nparts > 0 ? nparts : 1) * d);
        for (int h = 0; h < Hq; ++h) {
            int g = kv_head_of(h, Hq, Hkv);
            double* o = out + ((size_t)b * Hq + h) * d;
            for (int k = 0; k < d; ++k)
                qv[k] = load_elem(q, ((size_t)b * Hq + h) * d + k, q_dtype);
            if (gather_request(k_cache, v_cache, kv_dtype, k_scale, v_scale,
                               block_tables + (size_t)b * max_blocks, L, g, Hkv, bs,
                               d, num_blocks, Kc, Vc) != 0) {
                status = -1;
                break;
            }
            for (int p = 0; p < nparts; ++p) {
                int t0 = p * P, t1 = (p + 1) * P < L ? (p + 1) * P : L;
                double m = -INFINITY, l = 0.0;
                for (int k = 0; k < d; ++k) acc[k] = 0.0;
                /* one physical block (or the part of it inside [t0,t1)) at a time */
                for (int tb = t0; tb < t1;) {
                    int te = (tb / bs + 1) * bs;
                    if (te > t1) te = t1;
                    double bm = -INFINITY;
                    for (int t = tb; t < te; ++t) {
                        double sc = 0.0;
                        for (int k = 0; k < d; ++k) sc += qv[k] * Kc[(size_t)t * d + k];
                        sc *= scale;
                        if (sc > bm) bm = sc;
                    }
                    double mn = m > bm ? m : bm;
                    double alpha = (m == -INFINITY) ? 0.0 : exp(m - mn);
                    l *= alpha;
#if ORACLE_MUTANT != 14 /* planted (14): the running sum is not rescaled */
                    for (int k = 0; k < d; ++k) acc[k] *= alpha;
#endif
                    for (int t = tb; t < te; ++t) {
                        double sc = 0.0;
                        for (int k = 0; k < d; ++k) sc += qv[k] * Kc[(size_t)t * d + k];
                        double e = exp(sc * scale - mn);
                        l += e;
                        for (int k = 0; k < d; ++k) acc[k] += e * Vc[(size_t)t * d + k];
                    }
                    m = mn;
                    tb = te;
                }
                pm[p] = m;
                pl[p] = l;
                for (int k = 0; k < d; ++k) pacc[(size_t)p * d + k] = acc[k];
            }
            for (int k = 0; k < d; ++k) o[k] = 0.0;
            if (nparts == 0) continue;
            double M = pm[0];
            for (int p = 1; p < nparts; ++p)
                if (pm[p] > M) M = pm[p];
            double Z = 0.0;
            for (int k = 0; k < d; ++k) tot[k] = 0.0;
            for (int p = 0; p < nparts; ++p) {
                double f = exp(pm[p] - M);
#if ORACLE_MUTANT == 15
                Z += pl[p]; /* planted: the normaliser merged without its weight */
#else
                Z += f * pl[p];
#endif
                for (int k = 0; k < d; ++k) tot[k] += f * pacc[(size_t)p * d + k];
            }
            for (int k = 0; k < d; ++k) o[k] = tot[k] / Z;
        }
        free(Kc);
        free(Vc);
        free(pm);
        free(pl);
        free(pacc);
    }
    free(qv);
    free(acc);
    free(tot);
    return status;
}

/* ---- cache write (scatter) ------------------------------------------------ */

/*
 * For every new token t with slot s = slot_mapping[t] >= 0, copy the bytes of
 * k[t, h, :] into k_cache[s / bs, h, s % bs, :] (same for v) for all kv heads h
 * ([PAMEM] "The Mechanics of PagedAttention": new K/V vectors are written into
 * their allocated, possibly scattered, blocks; slot encoding R5).
 *   k, v     [T, Hkv, d]            elements of elem_size bytes
 *   k/v_cache [NB, Hkv, bs, d]
 * Returns the number of tokens whose slot was outside [0, NB*bs) (skipped).
 */
int oracle_kv_cache_write(const void* k, const void* v, const int64_t* slot_mapping,
                          void* k_cache, void* v_cache, int T, int num_blocks,
                          int Hkv, int d, int bs, int elem_size) {
    int bad = 0;
    size_t row = (size_t)d * elem_size;
    for (int t = 0; t < T; ++t) {
        int64_t s = slot_mapping[t];
        if (s < 0) continue;
        if (s >= (int64_t)num_blocks * bs) {
            ++bad;
            continue;
        }
        long p = (long)(s / bs);
        int o = (int)(s % bs);
#if ORACLE_MUTANT == 7
        o = (int)(s / num_blocks) % bs; /* planted: slot decoded the wrong way */
#endif
        for (int h = 0; h < Hkv; ++h) {
            size_t src = ((size_t)t * Hkv + h) * row;
            size_t dst = cache_index(p, h, o, 0, Hkv, bs, d) * elem_size;
            memcpy((char*)k_cache + dst, (const char*)k + src, row);
            memcpy((char*)v_cache + dst, (const char*)v + src, row);
        }
    }
    return bad;
}

/* ---- copy-on-write block copy -------------------------------------------- */

/*
 * For each pair (src, dst) of block_mapping [n, 2] (int64), copy the whole
 * physical block (all kv heads, all slots) of both caches: cache[dst] =
 * cache[src].  This is the private copy a request takes of a block it shares
 * with others before appending into it ([KVOPT] intro on shared prefix blocks
 * and copy-on-write; [KVMGMT] "The Bonus: Zero-Copy Sharing").  Pairs are
 * applied in order.  Returns the number of pairs skipped for out-of-range ids.
 */
int oracle_copy_blocks(void* k_cache, void* v_cache, const int64_t* block_mapping,
                       int n, int num_blocks, int Hkv, int d, int bs,
                       int elem_size) {
    int bad = 0;
    size_t blk = (size_t)Hkv * bs * d * elem_size;
    for (int i = 0; i < n; ++i) {
        int64_t src = block_mapping[2 * i], dst = block_mapping[2 * i + 1];
#if ORACLE_MUTANT == 8
        int64_t tmp = src; src = dst; dst = tmp; /* planted: pair read backwards */
#endif
        if (src < 0 || dst < 0 || src >= num_blocks || dst >= num_blocks) {
            ++bad;
            continue;
        }
        memmove((char*)k_cache + (size_t)dst * blk, (const char*)k_cache + (size_t)src * blk, blk);
        memmove((char*)v_cache + (size_t)dst * blk, (const char*)v_cache + (size_t)src * blk, blk);
    }
    return bad;
}

/* ---- swap between two pools (preemption) ---------------------------------- */

/*
 * For each pair (src, dst) of block_mapping [n, 2], copy block src of the
 * source pools into block dst of the destination pools (both K and V).  This is
 * the swap-out / swap-in a serving engine performs when it preempts a request
 * instead of recomputing it ([PAMEM] "Conclusion": requests are preempted and
 * their KV cache recomputed or swapped when blocks run out).  Returns the
 * number of pairs skipped for out-of-range ids.
 */
int oracle_swap_blocks(const void* src_k, const void* src_v, void* dst_k, void* dst_v,
                       const int64_t* block_mapping, int n, int src_blocks,
                       int dst_blocks, int Hkv, int d, int bs, int elem_size) {
    int bad = 0;
    size_t blk = (size_t)Hkv * bs * d * elem_size;
    for (int i = 0; i < n; ++i) {
        int64_t s = block_mapping[2 * i], t = block_mapping[2 * i + 1];
#if ORACLE_MUTANT == 13
        int64_t tmp = s; s = t; t = tmp; /* planted: pair read backwards */
#endif
        if (s < 0 || t < 0 || s >= src_blocks || t >= dst_blocks) {
            ++bad;
            continue;
        }
        memcpy((char*)dst_k + (size_t)t * blk, (const char*)src_k + (size_t)s * blk, blk);
        memcpy((char*)dst_v + (size_t)t * blk, (const char*)src_v + (size_t)s * blk, blk);
    }
    return bad;
}

/* ---- fp8 e4m3 quantisation (KV-cache compression) ------------------------ */

/*
 * e4m3 code of y = x / scale, where the quotient is the correctly rounded fp32
 * division.  The code is the representable value nearest to y, ties going to
 * the code with an even last mantissa bit; magnitudes at or above 448 (the
 * largest finite e4m3 value) saturate to 448; NaN maps to the NaN code.  The
 * search runs over all 127 non-negative finite codes, straight from the
 * format's definition.  ("KV Cache Management", "Watch Out For" / "What to Read
 * Next": compress the KV cache to 8-bit floats to fit long contexts.)
 */
void oracle_quantize_e4m3(const float* x, int n, float scale, uint8_t* out) {
    for (int i = 0; i < n; ++i) {
        float yf = x[i] / scale;
        double y = (double)yf;
        uint8_t sign = signbit(yf) ? 0x80 : 0x00;
        if (isnan(y)) {
            out[i] = (uint8_t)(sign | 0x7F);
            continue;
        }
        double a = fabs(y);
        if (a >= 448.0) {
            out[i] = (uint8_t)(sign | 0x7E);
#if ORACLE_MUTANT == 10
            out[i] = (uint8_t)(sign | 0x7F); /* planted: saturates to the NaN code */
#endif
            continue;
        }
        int best = 0;
        double bestd = INFINITY;
        for (int c = 0; c <= 0x7E; ++c) {
            double dv = fabs(a - e4m3_bits_to_double((uint8_t)c));
            int tie_to = 0;
#if ORACLE_MUTANT == 9
            tie_to = 1; /* planted: ties go to the odd code */
#endif
            if (dv < bestd || (dv == bestd && (c & 1) == tie_to)) {
                bestd = dv;
                best = c;
            }
        }
        out[i] = (uint8_t)(sign | best);
    }
}

/* Threads OpenMP would use (reported by the CPU baseline). */
int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
