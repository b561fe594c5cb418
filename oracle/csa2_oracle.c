/*
 * csa2_oracle.c -- plain CPU oracle for the CSA2 step over an FP4 main KV cache.
 *
 * TEST INFRASTRUCTURE: only the tests, the smoke check and the CPU-baseline leg
 * of the benchmark use it. It is independent of the CUDA library (no shared
 * code, tables or constants) and follows the definitions one step at a time in
 * double precision. The page references and the readings taken where the pages
 * are silent are listed in csa2_oracle.h.
 */
#include "csa2_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* Number formats.                                                           */
/* ------------------------------------------------------------------------ */

/* OCP 8-bit floating point, E4M3 variant: 1 sign bit, 4 exponent bits with
 * bias 7, 3 mantissa bits; exponent field 0 is subnormal (2^-6 * m/8); the
 * all-ones pattern S.1111.111 is NaN; there are no infinities. */
double or_e4m3_value(uint8_t code) {
    int sign = code >> 7;
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, -6);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -v : v;
}

/* Round to the nearest E4M3 value, ties to the code with an even mantissa,
 * saturating to +-448 (the largest finite magnitude). */
uint8_t or_e4m3_from_double(double x) {
    if (isnan(x)) return 0x7F;
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    double a = fabs(x);
    if (a >= 448.0) return sign | 0x7E;
    for (int c = 0; c < 126; ++c) {
        double lo = or_e4m3_value((uint8_t)c);
        double hi = or_e4m3_value((uint8_t)(c + 1));
        if (a <= hi) {
            double dlo = a - lo, dhi = hi - a;
            int pick;
            if (dlo < dhi) pick = c;
            else if (dhi < dlo) pick = c + 1;
            else pick = (c % 2 == 0) ? c : c + 1;
            return sign | (uint8_t)pick;
        }
    }
    return sign | 0x7E;
}

/* MX FP4 (E2M1): 1 sign bit, 2 exponent bits with bias 1, 1 mantissa bit;
 * exponent field 0 is subnormal (0.5 * m). Grid: 0 0.5 1 1.5 2 3 4 6. */
double or_e2m1_value(uint8_t code) {
    int sign = (code >> 3) & 1;
    int e = (code >> 1) & 3;
    int m = code & 1;
    double v = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return sign ? -v : v;
}

double or_bf16_value(uint16_t bits) {
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

uint8_t or_e2m1_code(double x, double s) {
    if (s == 0.0) return 0;
    uint8_t sign = signbit(x) ? 0x8 : 0x0;
    double a = fabs(x);
    for (int c = 0; c < 7; ++c) {
        double lo = or_e2m1_value((uint8_t)c) * s;
        double hi = or_e2m1_value((uint8_t)(c + 1)) * s;
        if (a <= hi) {
            double dlo = a - lo, dhi = hi - a;
            int pick;
            if (dlo < dhi) pick = c;
            else if (dhi < dlo) pick = c + 1;
            else pick = (c % 2 == 0) ? c : c + 1;
            return sign | (uint8_t)pick;
        }
    }
    return sign | 0x7;
}

static double g_e4m3_table[256];
static int g_e4m3_ready = 0;

static void e4m3_table_init(void) {
    if (g_e4m3_ready) return;
    for (int i = 0; i < 256; ++i) g_e4m3_table[i] = or_e4m3_value((uint8_t)i);
    g_e4m3_ready = 1;
}

/* ------------------------------------------------------------------------ */
/* FP4 main KV: one E4M3 scale per channel per 64-entry block.               */
/* ------------------------------------------------------------------------ */

#define OR_BLOCK 64

int or_fp4_kv_pack(const float* kv, int B, int N, int D,
                   uint8_t* kv_packed, uint8_t* kv_scale) {
    if (!kv || !kv_packed || !kv_scale || B < 0 || N < 0 || D <= 0) return OR_BAD_ARG;
    if (N % OR_BLOCK != 0 || D % 2 != 0) return OR_BAD_ARG;
    int nblk = N / OR_BLOCK;
    for (int b = 0; b < B; ++b) {
        for (int blk = 0; blk < nblk; ++blk) {
            for (int c = 0; c < D; ++c) {
                double amax = 0.0;
                for (int r = 0; r < OR_BLOCK; ++r) {
                    int n = blk * OR_BLOCK + r;
                    float x = kv[((size_t)b * N + n) * D + c];
                    if (!isfinite(x)) return OR_NONFINITE;
                    if (fabs((double)x) > amax) amax = fabs((double)x);
                }
                uint8_t sc = or_e4m3_from_double(amax / 6.0);
                kv_scale[((size_t)b * nblk + blk) * D + c] = sc;
                double s = or_e4m3_value(sc);
                for (int r = 0; r < OR_BLOCK; ++r) {
                    int n = blk * OR_BLOCK + r;
                    float x = kv[((size_t)b * N + n) * D + c];
                    uint8_t code = or_e2m1_code((double)x, s);
                    uint8_t* byte = &kv_packed[((size_t)b * N + n) * (D / 2) + c / 2];
                    if (c % 2 == 0)
                        *byte = (uint8_t)((*byte & 0xF0) | code);
                    else
                        *byte = (uint8_t)((*byte & 0x0F) | (code << 4));
                }
            }
        }
    }
    return OR_OK;
}

static double kv_value(const uint8_t* kv_packed, const uint8_t* kv_scale,
                       int N, int D, int b, int n, int c) {
    uint8_t byte = kv_packed[((size_t)b * N + n) * (D / 2) + c / 2];
    uint8_t code = (c % 2 == 0) ? (byte & 0xF) : (byte >> 4);
    uint8_t sc = kv_scale[((size_t)b * (N / OR_BLOCK) + n / OR_BLOCK) * D + c];
    return or_e2m1_value(code) * or_e4m3_value(sc);
}

int or_fp4_kv_unpack(const uint8_t* kv_packed, const uint8_t* kv_scale,
                     int B, int N, int D, double* out) {
    if (!kv_packed || !kv_scale || !out || B < 0 || N < 0 || D <= 0) return OR_BAD_ARG;
    if (N % OR_BLOCK != 0 || D % 2 != 0) return OR_BAD_ARG;
    for (int b = 0; b < B; ++b)
        for (int n = 0; n < N; ++n)
            for (int c = 0; c < D; ++c)
                out[((size_t)b * N + n) * D + c] = kv_value(kv_packed, kv_scale, N, D, b, n, c);
    return OR_OK;
}

/* ------------------------------------------------------------------------ */
/* FP4 main KV in the pages' own layout: one E4M3 scale per 16 channels of    */
/* an entry, no second-level scale ("Detailed Notes On DeepSeek V4 Point 1    */
/* Flash In Simple Words", "FP4 Main KV Cache To Halve Storage Again"; the    */
/* mengman.github.io interpretation, 3.5). An entry row holds its D/2 code     */
/* bytes followed by its D/16 scale bytes. The scale of a group follows the   */
/* same reading as the block layout: E4M3 (nearest, ties even) of max|x|/6.   */
/* ------------------------------------------------------------------------ */

#define OR_GROUP 16

static size_t g16_row_bytes(int D) { return (size_t)D / 2 + (size_t)D / OR_GROUP; }

/* Quantise one entry of D values into its row. */
static int g16_quantise_row(const float* x, int D, uint8_t* row) {
    for (int g = 0; g < D / OR_GROUP; ++g) {
        double amax = 0.0;
        for (int i = 0; i < OR_GROUP; ++i) {
            float v = x[g * OR_GROUP + i];
            if (!isfinite(v)) return OR_NONFINITE;
            if (fabs((double)v) > amax) amax = fabs((double)v);
        }
        uint8_t sc = or_e4m3_from_double(amax / 6.0);
        row[D / 2 + g] = sc;
        double s = or_e4m3_value(sc);
        for (int i = 0; i < OR_GROUP; ++i) {
            int c = g * OR_GROUP + i;
            uint8_t code = or_e2m1_code((double)x[c], s);
            uint8_t* byte = &row[c / 2];
            if (c % 2 == 0)
                *byte = (uint8_t)((*byte & 0xF0) | code);
            else
                *byte = (uint8_t)((*byte & 0x0F) | (code << 4));
        }
    }
    return OR_OK;
}

static int g16_shape_ok(int B, int N, int D) {
    return B >= 0 && N >= 0 && D > 0 && D % OR_GROUP == 0;
}

int or_fp4_kv_pack_g16(const float* kv, int B, int N, int D, uint8_t* kv_rows) {
    if (!kv || !kv_rows || !g16_shape_ok(B, N, D)) return OR_BAD_ARG;
    const size_t rb = g16_row_bytes(D);
    for (int b = 0; b < B; ++b)
        for (int n = 0; n < N; ++n) {
            int rc = g16_quantise_row(kv + ((size_t)b * N + n) * D, D,
                                      kv_rows + ((size_t)b * N + n) * rb);
            if (rc != OR_OK) return rc;
        }
    return OR_OK;
}

/* Appending new entries: entry t of row b is quantised into position
 * pos[b][t] of the cache; no other row changes (each row carries its own
 * scales). */
int or_fp4_kv_append_g16(const float* kv_new, const int32_t* pos, int B, int T, int N, int D,
                         uint8_t* kv_rows) {
    if (!kv_new || !pos || !kv_rows || !g16_shape_ok(B, N, D) || T < 0) return OR_BAD_ARG;
    const size_t rb = g16_row_bytes(D);
    for (int b = 0; b < B; ++b)
        for (int t = 0; t < T; ++t) {
            int32_t n = pos[(size_t)b * T + t];
            if (n < 0 || n >= N) return OR_BAD_INDEX;
            int rc = g16_quantise_row(kv_new + ((size_t)b * T + t) * D, D,
                                      kv_rows + ((size_t)b * N + n) * rb);
            if (rc != OR_OK) return rc;
        }
    return OR_OK;
}

static double g16_value(const uint8_t* kv_rows, int N, int D, int b, int n, int c) {
    const uint8_t* row = kv_rows + ((size_t)b * N + n) * g16_row_bytes(D);
    uint8_t byte = row[c / 2];
    uint8_t code = (c % 2 == 0) ? (byte & 0xF) : (byte >> 4);
    return or_e2m1_value(code) * or_e4m3_value(row[D / 2 + c / OR_GROUP]);
}

int or_fp4_kv_unpack_g16(const uint8_t* kv_rows, int B, int N, int D, double* out) {
    if (!kv_rows || !out || !g16_shape_ok(B, N, D)) return OR_BAD_ARG;
    for (int b = 0; b < B; ++b)
        for (int n = 0; n < N; ++n)
            for (int c = 0; c < D; ++c)
                out[((size_t)b * N + n) * D + c] = g16_value(kv_rows, N, D, b, n, c);
    return OR_OK;
}

/* ------------------------------------------------------------------------ */
/* Indexer score: s_j = sum_h w_h * ReLU(q_h . k_j).                          */
/* ------------------------------------------------------------------------ */

static double score_one(const uint8_t* q, const float* w, const uint8_t* k, int Hi, int Di) {
    double s = 0.0;
    for (int h = 0; h < Hi; ++h) {
        double dot = 0.0;
        for (int c = 0; c < Di; ++c)
            dot += g_e4m3_table[q[(size_t)h * Di + c]] * g_e4m3_table[k[c]];
        double relu = dot > 0.0 ? dot : 0.0;
        s += (double)w[h] * relu;
    }
    return s;
}

int or_index_score(const uint8_t* idx_q, const float* idx_w, const uint8_t* idx_k,
                   int B, int Tq, int N, int Hi, int Di,
                   const int32_t* nvalid, const int32_t* cand, int C,
                   double* scores) {
    if (!idx_q || !idx_w || !idx_k || !scores || B < 0 || Tq < 0 || N < 0 || Hi <= 0 || Di <= 0)
        return OR_BAD_ARG;
    if (!cand && !nvalid) return OR_BAD_ARG;
    if (cand && C <= 0) return OR_BAD_ARG;
    e4m3_table_init();
    for (int b = 0; b < B; ++b) {
        for (int t = 0; t < Tq; ++t) {
            size_t row = (size_t)b * Tq + t;
            const uint8_t* q = idx_q + row * Hi * Di;
            const float* w = idx_w + row * Hi;
            if (!cand) {
                int nv = nvalid[row];
                if (nv < 0 || nv > N) return OR_BAD_ARG;
                for (int j = 0; j < N; ++j) {
                    double* dst = &scores[row * N + j];
                    if (j < nv)
                        *dst = score_one(q, w, idx_k + ((size_t)b * N + j) * Di, Hi, Di);
                    else
                        *dst = -INFINITY;
                }
            } else {
                for (int i = 0; i < C; ++i) {
                    int j = cand[row * C + i];
                    double* dst = &scores[row * C + i];
                    if (j < 0) { *dst = -INFINITY; continue; }
                    if (j >= N) return OR_BAD_INDEX;
                    *dst = score_one(q, w, idx_k + ((size_t)b * N + j) * Di, Hi, Di);
                }
            }
        }
    }
    return OR_OK;
}

/* ------------------------------------------------------------------------ */
/* Top-K by (score descending, id ascending); output ascending by id.        */
/* ------------------------------------------------------------------------ */

typedef struct { double score; int32_t id; } scored_id;

static int cmp_rank(const void* pa, const void* pb) {
    const scored_id* a = (const scored_id*)pa;
    const scored_id* b = (const scored_id*)pb;
    if (a->score > b->score) return -1;
    if (a->score < b->score) return 1;
    return (a->id < b->id) ? -1 : (a->id > b->id);
}

static int cmp_i32(const void* pa, const void* pb) {
    int32_t a = *(const int32_t*)pa, b = *(const int32_t*)pb;
    return (a < b) ? -1 : (a > b);
}

int or_topk(const double* scores, int rows, int ld,
            const int32_t* nvalid, const int32_t* cand,
            int K, int32_t* topk) {
    if (!scores || !topk || rows < 0 || ld < 0 || K <= 0) return OR_BAD_ARG;
    if (!cand && !nvalid) return OR_BAD_ARG;
    scored_id* list = (scored_id*)malloc(sizeof(scored_id) * (size_t)(ld > 0 ? ld : 1));
    int32_t* chosen = (int32_t*)malloc(sizeof(int32_t) * (size_t)K);
    if (!list || !chosen) { free(list); free(chosen); return OR_BAD_ARG; }
    int rc = OR_OK;
    for (int r = 0; r < rows && rc == OR_OK; ++r) {
        int n = 0;
        if (!cand) {
            int nv = nvalid[r];
            if (nv < 0 || nv > ld) { rc = OR_BAD_ARG; break; }
            for (int j = 0; j < nv; ++j) {
                list[n].score = scores[(size_t)r * ld + j];
                list[n].id = j;
                ++n;
            }
        } else {
            for (int i = 0; i < ld; ++i) {
                int32_t id = cand[(size_t)r * ld + i];
                if (id < 0) continue;
                list[n].score = scores[(size_t)r * ld + i];
                list[n].id = id;
                ++n;
            }
        }
        for (int i = 0; i < n; ++i)
            if (isnan(list[i].score)) { rc = OR_NONFINITE; break; }
        if (rc != OR_OK) break;
        qsort(list, (size_t)n, sizeof(scored_id), cmp_rank);
        int m = n < K ? n : K;
        for (int i = 0; i < m; ++i) chosen[i] = list[i].id;
        qsort(chosen, (size_t)m, sizeof(int32_t), cmp_i32);
        for (int i = 0; i < K; ++i) topk[(size_t)r * K + i] = (i < m) ? chosen[i] : -1;
    }
    free(list);
    free(chosen);
    return rc;
}

/* Blockwise candidate pool of the hierarchical indexer ("Detailed Notes On
 * DeepSeek V4 Point 1 Flash In Simple Words", "Hierarchical Sparse Indexer In
 * Simple Terms"; mengman.github.io 3.4): the first FULL layer groups positions
 * into blocks of `block`, scores each block by the maximum score of its valid
 * positions, keeps the best `nblocks` blocks (ranked like entries: block score
 * descending, block index ascending) and hands their positions to the later
 * REINDEX layers. Output per row: the kept blocks' valid positions ascending,
 * padded with -1 to nblocks * block. */
int or_block_pool(const double* scores, int rows, int ld, const int32_t* nvalid,
                  int block, int nblocks, int32_t* cand) {
    if (!scores || !nvalid || !cand || rows < 0 || ld < 0 || block <= 0 || nblocks <= 0)
        return OR_BAD_ARG;
    const int nbmax = (ld + block - 1) / block;
    const size_t C = (size_t)nblocks * block;
    double* bscore = (double*)malloc(sizeof(double) * (size_t)(nbmax > 0 ? nbmax : 1));
    int32_t* kept = (int32_t*)malloc(sizeof(int32_t) * (size_t)nblocks);
    if (!bscore || !kept) { free(bscore); free(kept); return OR_BAD_ARG; }
    int rc = OR_OK;
    for (int r = 0; r < rows && rc == OR_OK; ++r) {
        const int nv = nvalid[r];
        if (nv < 0 || nv > ld) { rc = OR_BAD_ARG; break; }
        const int nb = (nv + block - 1) / block;          /* blocks with a valid position */
        for (int bk = 0; bk < nb; ++bk) {
            double m = -INFINITY;
            for (int j = bk * block; j < (bk + 1) * block && j < nv; ++j) {
                double x = scores[(size_t)r * ld + j];
                if (isnan(x)) { rc = OR_NONFINITE; break; }
                if (x > m) m = x;
            }
            bscore[bk] = m;
        }
        if (rc != OR_OK) break;
        /* the best blocks, by the entries' own ranking rule */
        rc = or_topk(bscore, 1, nb > 0 ? nb : 0, &nb, NULL, nblocks, kept);
        if (rc != OR_OK) break;
        size_t n = 0;
        for (int i = 0; i < nblocks; ++i) {
            if (kept[i] < 0) continue;
            for (int t = 0; t < block; ++t) {
                int j = kept[i] * block + t;
                if (j < nv) cand[(size_t)r * C + n++] = j;
            }
        }
        while (n < C) cand[(size_t)r * C + n++] = -1;
    }
    free(bscore);
    free(kept);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* Sparse softmax attention over the selected rows; K doubles as V.          */
/* ------------------------------------------------------------------------ */

/* Dequantised value of channel c of entry n of row b, for either layout. */
typedef struct {
    const uint8_t* kv_packed;   /* block layout: codes; 16-channel layout: rows */
    const uint8_t* kv_scale;    /* block layout: scales; NULL for the 16-channel layout */
    int N, D;
} kv_source;

static double kv_source_value(const kv_source* src, int b, int n, int c) {
    if (src->kv_scale)
        return kv_value(src->kv_packed, src->kv_scale, src->N, src->D, b, n, c);
    return g16_value(src->kv_packed, src->N, src->D, b, n, c);
}

/* Softmax attention of every head of query row `row` over the n value rows
 * v[0..n) (each serving as key and value): out = sum_k softmax(l)_k v_k with
 * l_k = softmax_scale * q . v_k; lse = log sum_k exp(l_k). No row: out = 0,
 * lse = -inf. `logit` has room for n values. */
static void attend_rows(const uint16_t* q, size_t row, int Hq, int D, const double* v, int n,
                        double softmax_scale, double* logit, double* out, double* lse) {
    for (int h = 0; h < Hq; ++h) {
        const uint16_t* qh = q + (row * Hq + h) * D;
        double* oh = out + (row * Hq + h) * D;
        if (n == 0) {
            for (int c = 0; c < D; ++c) oh[c] = 0.0;
            if (lse) lse[row * Hq + h] = -INFINITY;
            continue;
        }
        double m = -INFINITY;
        for (int k = 0; k < n; ++k) {
            double dot = 0.0;
            for (int c = 0; c < D; ++c) dot += or_bf16_value(qh[c]) * v[(size_t)k * D + c];
            logit[k] = softmax_scale * dot;
            if (logit[k] > m) m = logit[k];
        }
        double z = 0.0;
        for (int k = 0; k < n; ++k) {
            logit[k] = exp(logit[k] - m); /* now the unnormalised weight */
            z += logit[k];
        }
        for (int c = 0; c < D; ++c) {
            double acc = 0.0;
            for (int k = 0; k < n; ++k) acc += logit[k] * v[(size_t)k * D + c];
            oh[c] = acc / z;
        }
        if (lse) lse[row * Hq + h] = m + log(z);
    }
}

/* The selected main-KV rows of query row (b, row), dequantised into v; returns
 * their number, or -1 for an index outside [-1, N). */
static int gather_selected(const kv_source* src, const int32_t* topk, int b, size_t row, int D,
                           int N, int K, double* v) {
    int n = 0;
    for (int k = 0; k < K; ++k) {
        int32_t id = topk[row * K + k];
        if (id < 0) continue;
        if (id >= N) return -1;
        for (int c = 0; c < D; ++c)
            v[(size_t)n * D + c] = kv_source_value(src, b, id, c);
        ++n;
    }
    return n;
}

static int sparse_attn_rows(const uint16_t* q, const kv_source* src, const int32_t* topk,
                            int B, int Tq, int Hq, int D, int N, int K,
                            double softmax_scale, double* out, double* lse) {
    double* v = (double*)malloc(sizeof(double) * (size_t)K * D);
    double* logit = (double*)malloc(sizeof(double) * (size_t)K);
    if (!v || !logit) { free(v); free(logit); return OR_BAD_ARG; }
    int rc = OR_OK;
    for (int b = 0; b < B && rc == OR_OK; ++b) {
        for (int t = 0; t < Tq && rc == OR_OK; ++t) {
            size_t row = (size_t)b * Tq + t;
            int n = gather_selected(src, topk, b, row, D, N, K, v);
            if (n < 0) { rc = OR_BAD_INDEX; break; }
            attend_rows(q, row, Hq, D, v, n, softmax_scale, logit, out, lse);
        }
    }
    free(v);
    free(logit);
    return rc;
}

/* The sliding-window branch beside the sparse set ("Detailed Notes On
 * DeepSeek V4 Point 1 Flash In Simple Words": every layer also looks at the
 * recent tokens through sliding-window attention, window 128, its memory kept
 * at 8 bits; mengman.github.io 3.3, 3.5). How the two branches combine is not
 * stated; here one softmax runs over the union of the selected main rows and
 * the window's tokens. The window memory of row b is swa_kv[b][0..Tw) (one
 * E4M3 row of D values per token, no scale, serving as key and value); query
 * (b, t) sees its tokens [max(0, swa_n - W), swa_n), swa_n = swa_n[b][t]. */
int or_swa_sparse_attn(const uint16_t* q, const uint8_t* kv_packed, const uint8_t* kv_scale,
                       const int32_t* topk, const uint8_t* swa_kv, const int32_t* swa_n,
                       int B, int Tq, int Hq, int D, int N, int K, int Tw, int W,
                       double softmax_scale, double* out, double* lse) {
    if (!q || !kv_packed || !kv_scale || !topk || !swa_kv || !swa_n || !out || B < 0 ||
        Tq < 0 || Hq <= 0 || D <= 0 || N < 0 || K <= 0 || Tw < 0 || W < 0)
        return OR_BAD_ARG;
    if (N % OR_BLOCK != 0 || D % 2 != 0) return OR_BAD_ARG;
    e4m3_table_init();
    kv_source src = {kv_packed, kv_scale, N, D};
    double* v = (double*)malloc(sizeof(double) * ((size_t)K + (size_t)W) * D);
    double* logit = (double*)malloc(sizeof(double) * ((size_t)K + (size_t)W > 0 ? (size_t)K + W : 1));
    if (!v || !logit) { free(v); free(logit); return OR_BAD_ARG; }
    int rc = OR_OK;
    for (int b = 0; b < B && rc == OR_OK; ++b) {
        for (int t = 0; t < Tq && rc == OR_OK; ++t) {
            size_t row = (size_t)b * Tq + t;
            int n = gather_selected(&src, topk, b, row, D, N, K, v);
            if (n < 0) { rc = OR_BAD_INDEX; break; }
            int hi = swa_n[row];
            if (hi < 0 || hi > Tw) { rc = OR_BAD_ARG; break; }
            int lo = hi - W > 0 ? hi - W : 0;
            for (int j = lo; j < hi; ++j) {
                for (int c = 0; c < D; ++c)
                    v[(size_t)n * D + c] = g_e4m3_table[swa_kv[((size_t)b * Tw + j) * D + c]];
                ++n;
            }
            attend_rows(q, row, Hq, D, v, n, softmax_scale, logit, out, lse);
        }
    }
    free(v);
    free(logit);
    return rc;
}

int or_sparse_attn(const uint16_t* q, const uint8_t* kv_packed, const uint8_t* kv_scale,
                   const int32_t* topk, int B, int Tq, int Hq, int D, int N, int K,
                   double softmax_scale, double* out, double* lse) {
    if (!q || !kv_packed || !kv_scale || !topk || !out || B < 0 || Tq < 0 || Hq <= 0 ||
        D <= 0 || N < 0 || K <= 0)
        return OR_BAD_ARG;
    if (N % OR_BLOCK != 0 || D % 2 != 0) return OR_BAD_ARG;
    kv_source src = {kv_packed, kv_scale, N, D};
    return sparse_attn_rows(q, &src, topk, B, Tq, Hq, D, N, K, softmax_scale, out, lse);
}

int or_sparse_attn_g16(const uint16_t* q, const uint8_t* kv_rows, const int32_t* topk,
                       int B, int Tq, int Hq, int D, int N, int K,
                       double softmax_scale, double* out, double* lse) {
    if (!q || !kv_rows || !topk || !out || Tq < 0 || Hq <= 0 || K <= 0 ||
        !g16_shape_ok(B, N, D))
        return OR_BAD_ARG;
    kv_source src = {kv_rows, NULL, N, D};
    return sparse_attn_rows(q, &src, topk, B, Tq, Hq, D, N, K, softmax_scale, out, lse);
}

int or_dense_attn(const uint16_t* q, const uint8_t* kv_packed, const uint8_t* kv_scale,
                  const int32_t* nvalid, int B, int Tq, int Hq, int D, int N,
                  double softmax_scale, double* out, double* lse) {
    if (!q || !kv_packed || !kv_scale || !nvalid || !out || B < 0 || Tq < 0 || Hq <= 0 ||
        D <= 0 || N < 0)
        return OR_BAD_ARG;
    if (N % OR_BLOCK != 0 || D % 2 != 0) return OR_BAD_ARG;
    double* p = (double*)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
    if (!p) return OR_BAD_ARG;
    for (int b = 0; b < B; ++b) {
        for (int t = 0; t < Tq; ++t) {
            size_t row = (size_t)b * Tq + t;
            int nv = nvalid[row];
            if (nv < 0 || nv > N) { free(p); return OR_BAD_ARG; }
            for (int h = 0; h < Hq; ++h) {
                const uint16_t* qh = q + (row * Hq + h) * D;
                double* oh = out + (row * Hq + h) * D;
                /* pass 1: logits and their maximum */
                double m = -INFINITY;
                for (int j = 0; j < nv; ++j) {
                    double dot = 0.0;
                    for (int c = 0; c < D; ++c)
                        dot += or_bf16_value(qh[c]) * kv_value(kv_packed, kv_scale, N, D, b, j, c);
                    p[j] = softmax_scale * dot;
                    if (p[j] > m) m = p[j];
                }
                /* pass 2: normalised probabilities and the weighted sum */
                double z = 0.0;
                for (int j = 0; j < nv; ++j) z += exp(p[j] - m);
                for (int c = 0; c < D; ++c) oh[c] = 0.0;
                for (int j = 0; j < nv; ++j) {
                    double pj = exp(p[j] - m) / z;
                    for (int c = 0; c < D; ++c)
                        oh[c] += pj * kv_value(kv_packed, kv_scale, N, D, b, j, c);
                }
                if (lse) lse[row * Hq + h] = (nv > 0) ? m + log(z) : -INFINITY;
            }
        }
    }
    free(p);
    return OR_OK;
}

/* ------------------------------------------------------------------------ */
/* One layer in FULL / REINDEX / REUSE mode.                                 */
/* ------------------------------------------------------------------------ */

int or_layer_step(int mode, const uint16_t* q, const uint8_t* idx_q, const float* idx_w,
                  const uint8_t* idx_k, const uint8_t* kv_packed, const uint8_t* kv_scale,
                  const int32_t* nvalid, int B, int Tq, int N, int D, int Hq,
                  int Hi, int Di, int K, int C, int use_pool, double softmax_scale,
                  int32_t* topk_io, int32_t* cand_io, double* out, double* lse) {
    int rows = B * Tq;
    int rc;
    if (!topk_io) return OR_BAD_ARG;
    if (mode == OR_MODE_FULL || mode == OR_MODE_REINDEX) {
        int pooled = (mode == OR_MODE_REINDEX) && use_pool;
        if (pooled && (!cand_io || C <= 0)) return OR_BAD_ARG;
        int ld = pooled ? C : N;
        double* scores = (double*)malloc(sizeof(double) * (size_t)rows * (ld > 0 ? ld : 1));
        if (!scores) return OR_BAD_ARG;
        rc = or_index_score(idx_q, idx_w, idx_k, B, Tq, N, Hi, Di, nvalid,
                            pooled ? cand_io : NULL, C, scores);
        if (rc == OR_OK)
            rc = or_topk(scores, rows, ld, pooled ? NULL : nvalid, pooled ? cand_io : NULL,
                         K, topk_io);
        if (rc == OR_OK && mode == OR_MODE_FULL && C > 0 && cand_io)
            rc = or_topk(scores, rows, ld, nvalid, NULL, C, cand_io);
        free(scores);
        if (rc != OR_OK) return rc;
    } else if (mode != OR_MODE_REUSE) {
        return OR_BAD_ARG;
    }
    return or_sparse_attn(q, kv_packed, kv_scale, topk_io, B, Tq, Hq, D, N, K,
                          softmax_scale, out, lse);
}
