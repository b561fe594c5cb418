/*
 * csa2_oracle.h -- plain CPU oracle for the CSA2 step over an FP4 main KV cache.
 *
 * TEST INFRASTRUCTURE. Only the tests, the smoke check and the CPU-baseline leg
 * of the benchmark may load this library. It shares no code, header, table or
 * constant with the CUDA library; it is written from the definitions on the
 * pages, in double precision, with no blocking, fusion or reordering:
 *
 *  - "Detailed Notes On DeepSeek V4 Point 1 Flash In Simple Words",
 *    sections "Compressed Sparse Attention 2 Or CSA2 In Simple Terms",
 *    "The Three Modes Full Reindex And Reuse", "Hierarchical Sparse Indexer In
 *    Simple Terms" and "FP4 Main KV Cache To Halve Storage Again";
 *  - "DeepSeek-V4.1-Flash tech-report interpretation" (mengman.github.io),
 *    section 3.3 (CSA2 modes table), 3.4 (hierarchical sparse indexer) and
 *    3.5 (FP4 main KV cache: E2M1 values, E4M3 scales, no global scale).
 *
 * The pages fix no score formula, scale granularity, tie-break or rounding
 * mode; the readings taken here are: score = sum_h w_h * ReLU(q_h . k) with one
 * shared key per entry; one E4M3 scale per channel per 64-entry block equal to
 * round_e4m3(blockmax / 6); E2M1 codes by round-to-nearest-even on the E2M1
 * grid, saturating at 6; top-K ranked by (score descending, index ascending),
 * emitted ascending by index and padded with -1. For the pages' own layout
 * (one E4M3 scale per 16 channels of an entry) the same scale rule is applied
 * per group, and an entry's scale bytes follow its code bytes in one row.
 *
 * All functions return 0 on success and a nonzero code on a bad argument or a
 * non-finite value, never abort. Every pointer is host memory owned by the
 * caller. Layouts are row-major and contiguous:
 *   kv           float [B][N][D]
 *   kv_packed    u8    [B][N][D/2]     low nibble = even channel
 *   kv_scale     u8    [B][N/64][D]    E4M3 bytes
 *   kv_rows      u8    [B][N][D/2 + D/16]  16-channel layout: codes, then scales
 *   q            u16   [B][Tq][Hq][D]  bf16 bit patterns
 *   idx_q        u8    [B][Tq][Hi][Di] E4M3 bytes
 *   idx_w        float [B][Tq][Hi]
 *   idx_k        u8    [B][N][Di]      E4M3 bytes
 *   nvalid       i32   [B][Tq]         entries [0, nvalid) are visible
 *   cand         i32   [B][Tq][C]      candidate entry ids, -1 = none
 *   topk         i32   [B][Tq][K]      ascending, -1 padded
 *   out          double[B][Tq][Hq][D]
 *   lse          double[B][Tq][Hq]
 */
#ifndef CSA2_ORACLE_H
#define CSA2_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { OR_OK = 0, OR_BAD_ARG = 1, OR_NONFINITE = 2, OR_BAD_INDEX = 3 };
enum { OR_MODE_FULL = 0, OR_MODE_REINDEX = 1, OR_MODE_REUSE = 2 };

/* number formats (OCP 8-bit floating point and MX FP4 definitions) */
double or_e4m3_value(uint8_t code);
uint8_t or_e4m3_from_double(double x);      /* round to nearest even, saturate to +-448 */
double or_e2m1_value(uint8_t code);          /* low 4 bits used */
double or_bf16_value(uint16_t bits);

/* E2M1 code of x at scale s: nearest grid point of |x|/s, ties to the even
 * code, saturating at 6; sign from x. s == 0 gives code 0. */
uint8_t or_e2m1_code(double x, double s);

int or_fp4_kv_pack(const float* kv, int B, int N, int D,
                   uint8_t* kv_packed, uint8_t* kv_scale);
int or_fp4_kv_unpack(const uint8_t* kv_packed, const uint8_t* kv_scale,
                     int B, int N, int D, double* out);

/* The pages' own FP4 layout: one E4M3 scale per 16 channels of an entry.
 * kv_rows[b][n] = D/2 code bytes (channel c in byte c/2, low nibble = even c)
 * followed by D/16 scale bytes; scale = E4M3(max |x| of the group / 6). */
int or_fp4_kv_pack_g16(const float* kv, int B, int N, int D, uint8_t* kv_rows);
int or_fp4_kv_unpack_g16(const uint8_t* kv_rows, int B, int N, int D, double* out);
/* Quantise kv_new[b][t] into row pos[b][t] of kv_rows; other rows unchanged. */
int or_fp4_kv_append_g16(const float* kv_new, const int32_t* pos, int B, int T, int N, int D,
                         uint8_t* kv_rows);

/* scores[b][t][j] for j < nvalid[b][t] (cand == NULL), or scores[b][t][i] for
 * candidate i (cand != NULL); positions with no valid entry get -infinity.
 * The output row length is N without a pool and C with one. */
int or_index_score(const uint8_t* idx_q, const float* idx_w, const uint8_t* idx_k,
                   int B, int Tq, int N, int Hi, int Di,
                   const int32_t* nvalid, const int32_t* cand, int C,
                   double* scores);

/* Top-K per (b, t). Row r of `scores` has `ld` values. Without a pool the
 * valid entries are j < nvalid[r] with id j; with a pool (cand != NULL) the
 * entries are i < ld with cand[r][i] >= 0 and id cand[r][i]. Ranking is
 * (score descending, id ascending); the selected ids are written ascending,
 * padded with -1. */
int or_topk(const double* scores, int rows, int ld,
            const int32_t* nvalid, const int32_t* cand,
            int K, int32_t* topk);

/* Blockwise candidate pool: blocks of `block` positions scored by the maximum
 * over their valid positions (j < nvalid[r]); the top `nblocks` blocks by
 * (block score descending, block index ascending) are kept and their valid
 * positions written ascending to cand[r][0 .. nblocks*block), -1 padded. */
int or_block_pool(const double* scores, int rows, int ld, const int32_t* nvalid,
                  int block, int nblocks, int32_t* cand);

int or_sparse_attn(const uint16_t* q, const uint8_t* kv_packed, const uint8_t* kv_scale,
                   const int32_t* topk, int B, int Tq, int Hq, int D, int N, int K,
                   double softmax_scale, double* out, double* lse);

/* Sparse attention over a cache in the 16-channel-scale layout. */
int or_sparse_attn_g16(const uint16_t* q, const uint8_t* kv_rows, const int32_t* topk,
                       int B, int Tq, int Hq, int D, int N, int K,
                       double softmax_scale, double* out, double* lse);

/* Sparse attention with the sliding-window branch: one softmax over the
 * selected main rows and the window tokens [max(0, swa_n[b][t] - W),
 * swa_n[b][t]) of swa_kv[b] (u8 E4M3 [B][Tw][D], no scale, key = value). */
int or_swa_sparse_attn(const uint16_t* q, const uint8_t* kv_packed, const uint8_t* kv_scale,
                       const int32_t* topk, const uint8_t* swa_kv, const int32_t* swa_n,
                       int B, int Tq, int Hq, int D, int N, int K, int Tw, int W,
                       double softmax_scale, double* out, double* lse);

/* Softmax attention of every head over all entries j < nvalid[b][t] (dense). */
int or_dense_attn(const uint16_t* q, const uint8_t* kv_packed, const uint8_t* kv_scale,
                  const int32_t* nvalid, int B, int Tq, int Hq, int D, int N,
                  double softmax_scale, double* out, double* lse);

/* One CSA2 layer in `mode`. FULL: score [0, nvalid) -> top-K (and, when
 * C > 0 and cand_io != NULL, the top-C pool into cand_io) -> attention.
 * REINDEX: score [0, nvalid), or only the pool cand_io when use_pool != 0,
 * -> top-K -> attention. REUSE: attention over topk_io as given.
 * topk_io is written by FULL and REINDEX and read by every mode. */
int or_layer_step(int mode, const uint16_t* q, const uint8_t* idx_q, const float* idx_w,
                  const uint8_t* idx_k, const uint8_t* kv_packed, const uint8_t* kv_scale,
                  const int32_t* nvalid, int B, int Tq, int N, int D, int Hq,
                  int Hi, int Di, int K, int C, int use_pool, double softmax_scale,
                  int32_t* topk_io, int32_t* cand_io, double* out, double* lse);

#ifdef __cplusplus
}
#endif
#endif
