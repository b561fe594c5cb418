/*
 * csa2.h -- C ABI of libcsa2_fp4: the CSA2 attention step over an FP4 main KV
 * cache on NVIDIA B200 (sm_100a).
 *
 * What the step computes follows two of the pages that describe
 * DeepSeek-V4.1-Flash:
 *   [N] "Detailed Notes On DeepSeek V4 Point 1 Flash In Simple Words"
 *       (personal-website-enc.pages.dev), sections "Compressed Sparse
 *       Attention 2 Or CSA2 In Simple Terms", "The Three Modes Full Reindex And
 *       Reuse", "Hierarchical Sparse Indexer In Simple Terms", "FP4 Main KV
 *       Cache To Halve Storage Again";
 *   [M] "DeepSeek-V4.1-Flash tech-report interpretation" (mengman.github.io),
 *       section 3.3 (CSA2, its three static modes), 3.4 (hierarchical sparse
 *       indexer) and 3.5 (FP4 main KV cache).
 * A layer's indexer scores past main-KV entries against the current query and
 * keeps the top-K; attention then runs over only those entries, which are
 * stored as E2M1 values with E4M3 scales and dequantised before attention.
 *
 * Conventions for every call:
 *  - Pointers are DEVICE pointers unless stated; the caller owns every buffer.
 *    The library allocates no device memory; scratch comes from the caller's
 *    workspace (size from the matching *_workspace_bytes query).
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL is the legacy
 *    default stream) and runs on the device that stream belongs to: the call
 *    makes that device current while it works and restores the caller's
 *    current device before it returns (the legacy and per-thread default
 *    streams belong to the current device). Device pointers must be on that
 *    device. Host-side argument errors are reported before anything is
 *    launched; nothing is thrown across the ABI.
 *  - Device-side data errors (an index outside [-1, N), a non-finite value, an
 *    unsorted candidate list) do not trap: the kernel skips the bad element and
 *    records the first error code in a per-device word that
 *    csa2_check_device_errors() returns and clears.
 *  - Layouts are row-major and contiguous. bf16 values are passed as their
 *    16-bit patterns (uint16_t), E4M3 values as bytes.
 *  - Packed FP4: byte c/2 of an entry holds channel c, low nibble = even c.
 *    Scales: one E4M3 byte per channel per 64-entry block,
 *    kv_scale[b][n/64][c] (the block-scale layout of the benchmark
 *    workloads). The pages' own layout, one E4M3 scale per 16
 *    channels of an entry, has its own calls (*_g16): an entry is one row of
 *    D/2 code bytes followed by D/16 scale bytes, kv_rows[b][n][D/2 + D/16].
 *  - Pointers must be 16-byte aligned; D must be 512 for attention; N must be a
 *    multiple of 64.
 */
#ifndef CSA2_H
#define CSA2_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define CSA2_API __attribute__((visibility("default")))
#else
#define CSA2_API
#endif

/* Same type as cudaStream_t, declared here so the header needs no CUDA headers. */
typedef struct CUstream_st* csa2_stream_t;

typedef enum {
  CSA2_OK = 0,
  CSA2_ERR_INVALID_ARG = 1,   /* bad pointer, size, alignment or mode */
  CSA2_ERR_UNSUPPORTED = 2,   /* valid but not built (e.g. D != 512) */
  CSA2_ERR_CUDA = 3,          /* a CUDA runtime call or launch failed */
  CSA2_ERR_DEVICE_INDEX = 4,  /* device saw an index outside its range or an unsorted pool */
  CSA2_ERR_NONFINITE = 5,     /* device saw a NaN or infinity where a finite value is needed */
  CSA2_ERR_TIMEOUT = 6,       /* a bounded device wait ran out */
  CSA2_ERR_WORKSPACE = 7      /* workspace pointer NULL or smaller than required */
} csa2_status;

/* The three static per-layer modes ([N] "The Three Modes Full Reindex And
 * Reuse"; [M] 3.3): FULL scores its own indexer query against the shared
 * indexer keys and picks fresh top-K; REINDEX reuses the main KV and indexer
 * keys of an earlier FULL layer but scores with its own indexer query
 * (optionally only inside the candidate pool, [M] 3.4); REUSE attends over the
 * latest top-K indices with no indexing at all. */
typedef enum {
  CSA2_MODE_FULL = 0,
  CSA2_MODE_REINDEX = 1,
  CSA2_MODE_REUSE = 2
} csa2_mode;

/* ------------------------------------------------------------------------
 * fp4_kv_pack -- quantise the main KV cache to E2M1 with E4M3 block scales
 * ([N] "FP4 Main KV Cache To Halve Storage Again"; [M] 3.5: E2M1 values,
 * E4M3 scales, no second-level global scale).
 *
 * For each (b, 64-entry block, channel c): amax = max |kv| over the block;
 * scale = round-to-nearest-even E4M3 of amax / 6 (saturating at 448); each
 * value gets the E2M1 code nearest to x / scale, ties to the even code,
 * saturating at +-6, sign from x (scale 0 gives code 0).
 *   kv         float   [B][N][D]      input, finite
 *   kv_packed  uint8   [B][N][D/2]    output
 *   kv_scale   uint8   [B][N/64][D]   output, E4M3
 * Requires N % 64 == 0, D % 32 == 0. A NaN or infinity in kv records
 * CSA2_ERR_NONFINITE on the device (its block is still written).
 * ------------------------------------------------------------------------ */
CSA2_API csa2_status fp4_kv_pack(const float* kv, int B, int N, int D,
                        uint8_t* kv_packed, uint8_t* kv_scale, csa2_stream_t stream);

/* fp4_kv_unpack -- exact dequantisation: out[b][n][c] = e2m1(code) * e4m3(scale).
 *   out        float   [B][N][D]      output (every value is exact in fp32) */
CSA2_API csa2_status fp4_kv_unpack(const uint8_t* kv_packed, const uint8_t* kv_scale,
                          int B, int N, int D, float* out, csa2_stream_t stream);

/* ------------------------------------------------------------------------
 * fp4_kv_pack_g16 -- quantise the main KV cache in the pages' own layout:
 * E2M1 values with one E4M3 scale per 16 channels of an entry and no
 * second-level global scale ([N] "FP4 Main KV Cache To Halve Storage Again";
 * [M] 3.5). Where the scale bytes sit and how a scale is chosen is not stated;
 * this library stores each entry as one row, its D/2 code bytes then its D/16
 * scale bytes (288 bytes at D = 512), and takes the block layout's rule per
 * group: scale = nearest-even E4M3 of max|x| / 6 (saturating at 448), codes as
 * in fp4_kv_pack.
 *   kv       float [B][N][D]              input, finite
 *   kv_rows  uint8 [B][N][D/2 + D/16]     output; group g's scale is byte
 *                                         D/2 + g of the row (channels
 *                                         16g .. 16g + 15)
 * Requires D % 128 == 0 (every row 8-byte aligned); N is free. A NaN or
 * infinity records CSA2_ERR_NONFINITE on the device (the row is still written).
 * ------------------------------------------------------------------------ */
CSA2_API csa2_status fp4_kv_pack_g16(const float* kv, int B, int N, int D, uint8_t* kv_rows,
                                     csa2_stream_t stream);

/* fp4_kv_unpack_g16 -- exact dequantisation of the 16-channel layout:
 * out[b][n][c] = e2m1(code) * e4m3(scale of group c / 16).
 *   out      float [B][N][D]              output (every value exact in fp32)
 * Requires D % 128 == 0, as fp4_kv_pack_g16. */
CSA2_API csa2_status fp4_kv_unpack_g16(const uint8_t* kv_rows, int B, int N, int D, float* out,
                                       csa2_stream_t stream);

/* fp4_kv_append_g16 -- quantise new entries into an existing cache of the
 * 16-channel layout (entries are quantised after the rotary embedding,
 * [N] "FP4 Main KV Cache To Halve Storage Again"; [M] 3.5, so the caller
 * passes post-RoPE values). Entry t of row b goes to cache row pos[b][t];
 * every other row is left as it is, since each row carries its own scales.
 *   kv_new   float [B][T][D]              input, finite
 *   pos      int32 [B][T]                 destination rows in [0, N); a
 *                                         position outside it is skipped and
 *                                         CSA2_ERR_DEVICE_INDEX recorded; the
 *                                         positions of one b must differ
 *   kv_rows  uint8 [B][N][D/2 + D/16]     updated in place
 * Requires D % 128 == 0, T >= 0. A NaN or infinity records CSA2_ERR_NONFINITE
 * (the row is still written).
 * ------------------------------------------------------------------------ */
CSA2_API csa2_status fp4_kv_append_g16(const float* kv_new, const int32_t* pos, int B, int T,
                                       int N, int D, uint8_t* kv_rows, csa2_stream_t stream);

/* ------------------------------------------------------------------------
 * csa2_index_score -- indexer scores ([N] "Compressed Sparse Attention 2 Or
 * CSA2 In Simple Terms": each layer's small indexer scores which past entries
 * are most relevant to the current query; the indexer keys are one shared key
 * per entry).  Score of entry j for query (b, t):
 *     s = sum_h idx_w[b][t][h] * max(0, sum_c idx_q[b][t][h][c] * idx_k[b][j][c])
 * with E4M3 inputs and fp32 accumulation (exact for integer-valued inputs
 * whose score magnitude stays below 2^24).
 *   idx_q   uint8 [B][Tq][Hi][Di]  E4M3
 *   idx_w   float [B][Tq][Hi]
 *   idx_k   uint8 [B][N][Di]       E4M3, shared by all indexing layers
 *   nvalid  int32 [B][Tq]          entries [0, nvalid) are visible (causal mask)
 *   cand    int32 [B][Tq][C]       NULL for a full scan; otherwise the candidate
 *                                  pool ([M] 3.4): ascending entry ids then -1
 *   scores  float [B][Tq][N]       full scan: written for j < nvalid, the rest
 *                                  of the row is not written;
 *           float [B][Tq][C]       pool: score of cand[i], -inf where cand[i] < 0
 * Requires Di % 16 == 0, Di <= 256, Hi <= 128.
 * ------------------------------------------------------------------------ */
CSA2_API csa2_status csa2_index_score(const uint8_t* idx_q, const float* idx_w, const uint8_t* idx_k,
                             int B, int Tq, int N, int Hi, int Di,
                             const int32_t* nvalid, const int32_t* cand, int C,
                             float* scores, csa2_stream_t stream);

/* ------------------------------------------------------------------------
 * csa2_topk -- top-K selection ([N] CSA2 section: the indexer picks the top
 * entries to attend to; [M] 3.3). Entries are ranked by (score descending,
 * entry id ascending) -- the lower index wins a tie, and -0 equals +0 -- and
 * the selected ids are written ascending, padded with -1 when fewer than K
 * entries are valid.
 *   scores   float [B][Tq][ld]
 *   nvalid   int32 [B][Tq]     full scan: entries j < nvalid, id = j (cand NULL)
 *   cand     int32 [B][Tq][ld] pool: entry i has id cand[i], skipped when < 0;
 *                              ids must be ascending (checked on the device)
 *   topk_idx int32 [B][Tq][K]  output
 *   cand_out int32 [B][Tq][Cout] optional second selection with the same
 *                              ranking (the hierarchical pool, [M] 3.4); the
 *                              top-K is a subset of it. NULL to skip.
 * Requires 1 <= K, Cout <= 65536 and ld <= 2^30. A NaN score records
 * CSA2_ERR_NONFINITE.
 * ------------------------------------------------------------------------ */
CSA2_API csa2_status csa2_topk(const float* scores, int ld, const int32_t* nvalid, const int32_t* cand,
                      int B, int Tq, int K, int32_t* topk_idx,
                      int Cout, int32_t* cand_out, csa2_stream_t stream);

/* ------------------------------------------------------------------------
 * csa2_block_pool -- the blockwise candidate pool of the hierarchical indexer
 * ([N] "Hierarchical Sparse Indexer In Simple Terms"; [M] 3.4): the first FULL
 * layer groups positions into blocks of `block` (8 in the model), scores each
 * block by the largest score among its valid positions (j < nvalid), keeps the
 * best `nblocks` blocks (2048 in the model: about 16384 candidates) ranked like
 * entries (block score descending, lower block index first) and gives their
 * valid positions to later REINDEX layers as the pool (csa2_index_score and
 * csa2_topk with `cand`).
 *   scores   float [B][Tq][ld]               from csa2_index_score (full scan)
 *   nvalid   int32 [B][Tq]                   clamped to [0, ld]
 *   cand_out int32 [B][Tq][nblocks * block]  ascending positions, -1 padded
 *   workspace device scratch of csa2_block_pool_workspace_bytes() bytes
 * Requires 1 <= nblocks <= 65536, block >= 1, block * nblocks <= 2^30. A NaN
 * score records CSA2_ERR_NONFINITE.
 * ------------------------------------------------------------------------ */
CSA2_API size_t csa2_block_pool_workspace_bytes(int B, int Tq, int ld, int block, int nblocks);

CSA2_API csa2_status csa2_block_pool(const float* scores, int ld, const int32_t* nvalid, int B,
                                     int Tq, int block, int nblocks, int32_t* cand_out,
                                     void* workspace, size_t workspace_bytes,
                                     csa2_stream_t stream);

/* ------------------------------------------------------------------------
 * csa2_sparse_attn -- gather + FP4 dequantisation + softmax attention over
 * the selected entries only ([N] CSA2 section and "FP4 Main KV Cache To Halve
 * Storage Again": values are dequantised back before attention). One shared
 * main-KV head of dimension D serves as both key and value:
 *     l_k = softmax_scale * q[b][t][h] . v_k,   v_k = dequant(kv row idx_k)
 *     out[b][t][h] = sum_k softmax(l)_k v_k,     lse[b][t][h] = log sum_k e^{l_k}
 * over the entries topk_idx[b][t][*] >= 0 (-1 is skipped; no valid entry gives
 * out = 0 and lse = -inf). Accumulation is fp32; the output is rounded to bf16.
 *   q         uint16 [B][Tq][Hq][D]  bf16
 *   kv_packed uint8  [B][N][D/2],  kv_scale uint8 [B][N/64][D]
 *   topk_idx  int32  [B][Tq][K]      ids in [-1, N); out-of-range ids are
 *                                    skipped and recorded
 *   out       uint16 [B][Tq][Hq][D]  bf16
 *   lse       float  [B][Tq][Hq]     optional (NULL to skip), natural log
 *   workspace device scratch of csa2_sparse_attn_workspace_bytes() bytes
 * Requires D == 512, 1 <= Hq <= 65535, K >= 1.
 * ------------------------------------------------------------------------ */
CSA2_API size_t csa2_sparse_attn_workspace_bytes(int B, int Tq, int Hq, int D, int K);

CSA2_API csa2_status csa2_sparse_attn(const uint16_t* q, const uint8_t* kv_packed, const uint8_t* kv_scale,
                             const int32_t* topk_idx, int B, int Tq, int Hq, int D, int N, int K,
                             float softmax_scale, uint16_t* out, float* lse,
                             void* workspace, size_t workspace_bytes, csa2_stream_t stream);

/* csa2_sparse_attn_g16 -- csa2_sparse_attn over a cache in the 16-channel
 * layout (fp4_kv_pack_g16): the same computation, with v_k dequantised from
 * row idx_k's codes and its own group scales. Same arguments otherwise, the
 * same workspace (csa2_sparse_attn_workspace_bytes), D == 512 (288-byte rows),
 * any N >= 0.
 *   kv_rows  uint8 [B][N][D/2 + D/16] */
CSA2_API csa2_status csa2_sparse_attn_g16(const uint16_t* q, const uint8_t* kv_rows,
                                          const int32_t* topk_idx, int B, int Tq, int Hq, int D,
                                          int N, int K, float softmax_scale, uint16_t* out,
                                          float* lse, void* workspace, size_t workspace_bytes,
                                          csa2_stream_t stream);

/* ------------------------------------------------------------------------
 * csa2_sparse_attn_swa -- csa2_sparse_attn plus the sliding-window branch
 * that every CSA2 layer has beside its selected entries ([N] "The Three Modes
 * Full Reindex And Reuse" and "Model Setup Numbers Without Jargon": a window
 * of the last 128 tokens; [N] "FP4 Main KV Cache To Halve Storage Again" and
 * [M] 3.5: the window's cache stays at 8 bits). The pages do not say how the
 * two branches combine; here one softmax runs over the union of the selected
 * main-KV rows and the window's tokens, each window row (D E4M3 values, no
 * scale) serving as key and value:
 *     entries of row (b, t) = {v_k : topk_idx[b][t][k] >= 0}
 *                           + {e4m3(swa_kv[b][j]) : max(0, n - W) <= j < n},
 *     n = swa_n[b][t]; then out and lse as in csa2_sparse_attn.
 * Same arguments as csa2_sparse_attn (with kv_scale NULL, kv_packed holds the
 * 16-channel layout as in csa2_sparse_attn_g16), plus:
 *   swa_kv   uint8 [B][Tw][D]  E4M3 window memory; 16-byte aligned
 *   swa_n    int32 [B][Tq]     end of each query row's window, in [0, Tw];
 *                              an end outside it is recorded
 *                              (CSA2_ERR_DEVICE_INDEX) and empties that window
 *   Tw       tokens in each row's window memory (>= 0)
 *   W        window length (128 in the pages; 0 <= W <= 65536)
 * An E4M3 NaN byte (0x7f, 0xff) in a window row that is read records
 * CSA2_ERR_NONFINITE (the outputs of that query row are then unspecified).
 * The workspace is csa2_sparse_attn_workspace_bytes(B, Tq, Hq, D, K + W):
 * the window's W slots follow the K selected entries in each row's list.
 * ------------------------------------------------------------------------ */
CSA2_API csa2_status csa2_sparse_attn_swa(const uint16_t* q, const uint8_t* kv_packed,
                                          const uint8_t* kv_scale, const int32_t* topk_idx,
                                          const uint8_t* swa_kv, const int32_t* swa_n, int B,
                                          int Tq, int Hq, int D, int N, int K, int Tw, int W,
                                          float softmax_scale, uint16_t* out, float* lse,
                                          void* workspace, size_t workspace_bytes,
                                          csa2_stream_t stream);

/* ------------------------------------------------------------------------
 * csa2_sparse_attn_noalloc -- csa2_sparse_attn without a caller workspace.
 * (An interface addition of this library; the pages describe no such call.)
 *
 * For callers that cannot allocate device memory at all: code inside an engine
 * that owns and pre-partitions all device memory, a custom-op hook that offers
 * no allocator, or a latency-critical path that must avoid an allocation and
 * its implicit synchronisation. Same arguments, semantics and results as
 * csa2_sparse_attn minus the workspace: the split scratch comes from a fixed
 * device array of CSA2_NOALLOC_SCRATCH_BYTES built into the library. Under
 * CUDA's lazy module loading (the default since CUDA 12) the array is reserved
 * on a device when this function is first used there and stays until the
 * process exits; with CUDA_MODULE_LOADING=EAGER every context that loads the
 * library reserves it, whether or not this function is ever called.
 *  - Returns CSA2_ERR_WORKSPACE, launching nothing, when the shape needs more
 *    split scratch than the array holds (compare with
 *    csa2_sparse_attn_workspace_bytes()). The split plan gives each SM at most
 *    one (row, head block, split) slot of 131,584 bytes, so on a GPU with up to
 *    255 SMs (a B200 has 148) no shape needs more than the array.
 *  - All calls on a device share the array: calls that overlap on the GPU
 *    (e.g. two streams at once) race. The array keeps the last call's contents;
 *    nothing in it needs to start at zero.
 *  - The first call on each device looks up the array's address on the host
 *    (with the stream's device current); make that first call before any
 *    stream capture.
 *  - Calls no cudaMalloc, cudaFree or allocating library routine.
 * ------------------------------------------------------------------------ */
#define CSA2_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)

CSA2_API csa2_status csa2_sparse_attn_noalloc(const uint16_t* q, const uint8_t* kv_packed,
                                              const uint8_t* kv_scale, const int32_t* topk_idx,
                                              int B, int Tq, int Hq, int D, int N, int K,
                                              float softmax_scale, uint16_t* out, float* lse,
                                              csa2_stream_t stream);

/* ------------------------------------------------------------------------
 * csa2_layer_step -- one CSA2 layer in its static mode ([N] "The Three Modes
 * Full Reindex And Reuse"; [M] 3.3, 3.4). The shared state holds non-owning
 * device pointers that several layers pass to each other without copies: the
 * main KV and indexer keys built by a FULL layer, and the latest top-K indices
 * (and candidate pool) that REINDEX/REUSE layers consume.
 *   FULL    : score [0, nvalid) -> top-K into st->topk_idx (and, when
 *             args->emit_pool and st->C > 0, a pool into st->cand_idx: the
 *             top-C entries for emit_pool == 1, or the blockwise pool of
 *             csa2_block_pool with blocks of 8 and C / 8 blocks for
 *             emit_pool == 2) -> attention
 *   REINDEX : score [0, nvalid), or only st->cand_idx when args->use_pool,
 *             with this layer's own indexer query -> top-K into st->topk_idx
 *             -> attention
 *   REUSE   : attention over st->topk_idx as it stands
 * ------------------------------------------------------------------------ */
typedef struct {
  const uint8_t* kv_packed;   /* [B][N][D/2]; with kv_scale NULL, the rows
                                 [B][N][D/2 + D/16] of the 16-channel layout
                                 (fp4_kv_pack_g16) */
  const uint8_t* kv_scale;    /* [B][N/64][D]; NULL selects the 16-channel layout */
  const uint8_t* idx_k;       /* [B][N][Di] E4M3; may be NULL when only REUSE runs */
  int32_t* topk_idx;          /* [B][Tq][K]: written by FULL/REINDEX, read by all */
  int32_t* cand_idx;          /* [B][Tq][C]: written by FULL (emit_pool), read by REINDEX (use_pool) */
  int C;                      /* candidate pool size (0 = no pool) */
} csa2_shared_state;

typedef struct {
  int B, Tq, N, D, Hq, Hi, Di, K;
  const int32_t* nvalid;      /* [B][Tq] */
  const uint16_t* q;          /* [B][Tq][Hq][D] bf16 attention query of this layer */
  const uint8_t* idx_q;       /* [B][Tq][Hi][Di] E4M3 indexer query (FULL/REINDEX) */
  const float* idx_w;         /* [B][Tq][Hi] indexer head weights (FULL/REINDEX) */
  float softmax_scale;
  uint16_t* out;              /* [B][Tq][Hq][D] bf16 */
  float* lse;                 /* [B][Tq][Hq] or NULL */
  int emit_pool;              /* FULL: 0 no pool; 1 the top-C entries; 2 the blockwise
                                 pool (blocks of 8, C/8 blocks, C % 8 == 0) into st->cand_idx */
  int use_pool;               /* REINDEX: score only st->cand_idx */
  /* The sliding-window branch (csa2_sparse_attn_swa), in every mode; swa_kv
     NULL leaves it out. The workspace then grows by the window's W slots. */
  const uint8_t* swa_kv;      /* [B][Tw][D] E4M3 window memory, or NULL */
  const int32_t* swa_n;       /* [B][Tq] end of each query row's window */
  int Tw, W;
} csa2_layer_args;

CSA2_API size_t csa2_layer_step_workspace_bytes(const csa2_layer_args* args, csa2_mode mode,
                                       const csa2_shared_state* st);

CSA2_API csa2_status csa2_layer_step(const csa2_layer_args* args, csa2_mode mode, csa2_shared_state* st,
                            void* workspace, size_t workspace_bytes, csa2_stream_t stream);

/* ------------------------------------------------------------------------
 * Errors.
 * csa2_check_device_errors: synchronises `stream`, returns the first device
 * data error recorded on the stream's device since the last check (CSA2_OK if
 * none) and clears it.
 * csa2_last_error: thread-local text for the last non-OK status returned on
 * this thread (empty string if none). The pointer stays valid until the next
 * call on the same thread.
 * ------------------------------------------------------------------------ */
CSA2_API csa2_status csa2_check_device_errors(csa2_stream_t stream);
CSA2_API const char* csa2_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* CSA2_H */
