// attn_tc.cu -- fused gather + FP4 dequantisation + sparse softmax attention
// on the 5th-generation tensor cores.
//
// "Detailed Notes On DeepSeek V4 Point 1 Flash In Simple Words", sections
// "Compressed Sparse Attention 2 Or CSA2 In Simple Terms" (attend only to the
// top-K entries the indexer picked), "FP4 Main KV Cache To Halve Storage Again"
// (E2M1 values are dequantised back before attention) and "Model Setup Numbers
// Without Jargon" (64 query heads of dimension 512 share one main-KV head,
// which serves as both key and value).
//
// One CTA = (query row, block of 64 heads, split of the selected-entry list),
// processed in tiles of 64 entries through three-deep rings: while the softmax
// works on tile t, the tensor core runs P(t-1) V(t-1) and S(t+1), and the
// producers fill tile t+2. Every selected row is gathered and dequantised ONCE,
// into a shared-memory tile that serves both products:
//   S(t) = Q V(t)^T   M = 64 heads, N = 64 entries, K = 512: 32 MMAs with the
//                     query block as the A operand held in tensor memory (so
//                     only the V tile is read from shared memory) and the V
//                     tile read K-major;
//   O   += P(t) V(t)  M = 64 heads, N = 256 dims per half, K = 64 entries:
//                     8 MMAs, P and the V tile (read MN-major) from shared memory.
// Tensor memory (an M = 64 operand or accumulator occupies 16 lanes of each
// 32-lane quadrant): lanes 0-15 hold S(t) (three buffers of 64 columns) and the
// query block (256 columns of fp16 pairs, columns 192-447); lanes 16-31 hold O
// (all 512 columns).
// A softmax thread owns half of one head's 64 logits of a tile (the other half
// is the thread 16 lanes away): its logits, the head's reference maximum and
// its part of the row sum live in registers. The maximum is lazy: P = 2^(s - m)
// with m raised (and O and the row sum rescaled) only when a tile holds a logit
// more than 8 above it, so P stays below 2^8 in fp16 and rescaling is rare.
// Values are dequantised exactly into fp16 by the hardware E2M1 and E4M3
// conversions and one fp16 product per value. A producer dequantises a tile into
// registers BEFORE waiting for its ring slot, so after the slot frees only the
// shared-memory stores stand between P(t-3) V(t-3) and S(t).
// Roles: warps 0-7 gather and dequantise, and stage Q into tensor memory while
// the first tile's rows are in flight; warp 8 owns tensor memory and issues the MMAs; warps 9-12 run
// the softmax. At the
// end every warp that can reach a quadrant's O lanes (its softmax warp and two
// producer warps) writes that quadrant's output, partial or final. Every
// mbarrier wait is bounded.
#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace csa2 {
namespace {

namespace cg = cooperative_groups;

using namespace sm100;

constexpr int kD = kHeadDim;             // 512
constexpr int kHB = 64;                  // heads per CTA
constexpr int kT = 64;                   // entries per tile
constexpr int kAtom = 8192;              // 64 rows x 128 B: a K atom of P, or of a V tile
constexpr int kVTile = 8 * kAtom;        // 64 entries x 512 dims of fp16
constexpr int kRing = 3;                 // V tiles, S buffers and P buffers in flight
constexpr int kProducerWarps = 8;
constexpr int kMmaWarp = 8;
constexpr int kThreads = 13 * 32;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemQ = 192;         // first column of the query block (lanes 0-15)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleSlack = 8.0f;    // log2 units: P <= 2^8 before a rescale
constexpr int kMaxClusterSplits = 8;

struct __align__(8) Bars {
  uint64_t q_ld, q_conv, q_full, q_free, o_full;
  uint64_t v_full[kRing], v_free[kRing], s_full[kRing], p_full[kRing];
};

struct Smem {
  Bars bar;
  uint32_t tmem_slot;
  int abort_flag;
  uint32_t valid[kRing][kT / 32];   // bit i of word w: entry 32 w + i of the tile is selected
                                    // (byte w' of the pair written by producer warp w')
  float2 mlf[kHB];                  // this split's (reference maximum, row sum) per head
  float qdown[kHB];                 // the power of two each head's query was scaled up by, inverted
};

constexpr size_t kSmemBytes = 1024 + kRing * kVTile /*V*/ + kRing * kAtom /*P*/ + sizeof(Smem);
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");

// In-cluster merge, inside the (idle) V region of every split: each split
// stages its partial output of every head, normalised by its own row sum and
// rounded to fp16, grouped by the split that merges the head ([owner r][head hh
// of r's share][512], 1 KB rows whose 16-byte chunks are swizzled by hh), with
// its (max, sum) pairs; every thread then copies 16-byte pieces of each group
// into its owner's receive area ([source split r][hh][512]) through
// distributed shared memory; the owner merges its heads.
constexpr uint32_t kMergeSendOff = 0;               // bytes into the V region
constexpr uint32_t kMergeSendMlOff = 72 * 1024;
constexpr uint32_t kMergeRecvOff = 76 * 1024;
constexpr uint32_t kMergeRecvMlOff = 148 * 1024;
static_assert(kMergeRecvMlOff + 4 * 1024 <= (size_t)kRing * kVTile,
              "merge staging fits in the V region");
// heads each split of a cluster of ns merges, and the 16-byte-padded bytes of
// their (max, sum) pairs
__host__ __device__ constexpr int merge_share(int ns) { return (kHB + ns - 1) / ns; }
__host__ __device__ constexpr uint32_t merge_ml_bytes(int ns) {
  return (uint32_t)((merge_share(ns) * 8 + 15) / 16 * 16);
}
static_assert(3 * merge_share(3) * 1024 <= 72 * 1024 && 8 * merge_share(8) * 1024 <= 72 * 1024 &&
                  5 * merge_share(5) * 1024 <= 72 * 1024 && 7 * merge_share(7) * 1024 <= 72 * 1024,
              "a send or receive area holds every split's share");
static_assert(kMaxClusterSplits * 176 <= 4 * 1024, "(max, sum) areas");

// byte offset of 16-byte chunk c (0..7) of row r in a [rows][128 B] swizzled block
__device__ __forceinline__ int swz(int r, int c) { return r * 128 + ((c ^ (r & 7)) << 4); }

__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// kind::f16, F16 x F16 -> F32; A K-major; B K-major (0) or N-major (1).
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N, int b_mn) {
  return (1u << 4) | ((uint32_t)b_mn << 16) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

// One MMA, both operands in shared memory, each descriptor given as its low
// word (start address and leading offset: advancing it by (bytes >> 4) cannot
// carry out, shared-memory addresses being below 2^18) and a common high word.
__device__ __forceinline__ void mma_ss(uint32_t d, uint32_t a_lo, uint32_t b_lo, uint32_t hi_a,
                                       uint32_t hi_b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 da, db;\n\t"
      "setp.ne.b32 p, %6, 0;\n\t"
      "mov.b64 da, {%1, %3};\n\t"
      "mov.b64 db, {%2, %4};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %5, p;\n\t}" ::"r"(d),
      "r"(a_lo), "r"(b_lo), "r"(hi_a), "r"(hi_b), "r"(idesc), "r"(acc)
      : "memory");
}

// One MMA with A in tensor memory (the same lanes as the accumulator) and B in
// shared memory.
__device__ __forceinline__ void mma_ts(uint32_t d, uint32_t a_tmem, uint32_t b_lo, uint32_t hi_b,
                                       uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 db;\n\t"
      "setp.ne.b32 p, %5, 0;\n\t"
      "mov.b64 db, {%2, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], db, %4, p;\n\t}" ::"r"(d),
      "r"(a_tmem), "r"(b_lo), "r"(hi_b), "r"(idesc), "r"(acc)
      : "memory");
}

// 16-byte shared-memory accesses by 32-bit shared address
__device__ __forceinline__ void sts128(uint32_t a, const uint4& v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}
__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(a)
               : "memory");
  return v;
}

__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 2^x with the hardware approximation (relative error about 2^-22; results
// below 2^-126 flush to zero, far below the fp16 the probabilities are stored in)
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ uint32_t pack_bf162(float lo, float hi) {
  __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&b);
}

// Read-only global loads that the compiler keeps in program order among the
// other volatile asm (shared-memory stores, barrier waits), so that a gather
// issued a tile ahead is not sunk to its use.
__device__ __forceinline__ uint2 ldg_v2(const void* ptr) {
  uint2 r;
  asm volatile("ld.global.nc.v2.u32 {%0, %1}, [%2];" : "=r"(r.x), "=r"(r.y) : "l"(ptr));
  return r;
}
__device__ __forceinline__ uint4 ldg_v4(const void* ptr) {
  uint4 r;
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(ptr));
  return r;
}
__device__ __forceinline__ uint32_t ldg_u8(const void* ptr) {
  uint32_t r;
  asm volatile("ld.global.nc.u8 %0, [%1];" : "=r"(r) : "l"(ptr));
  return r;
}

// Hardware conversions of packed FP4/FP8 pairs to f16x2 (the first, lower
// nibble or byte into the lower half).
__device__ __forceinline__ void e2m1x8_to_f16(uint32_t codes, uint32_t (&h)[4]) {
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
      : "r"(codes));
}
__device__ __forceinline__ void e4m3x4_to_f16(uint32_t bytes, uint32_t& lo, uint32_t& hi) {
  asm("{\n\t.reg .b16 h0, h1;\n\t"
      "mov.b32 {h0, h1}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, h0;\n\t"
      "cvt.rn.f16x2.e4m3x2 %1, h1;\n\t}"
      : "=r"(lo), "=r"(hi)
      : "r"(bytes));
}

// 8 E2M1 codes (one 32-bit word, low nibble first) times their 8 E4M3 scales
// (two words) -> one 16-byte chunk of fp16 values. The product is exact in
// fp16: at most 6 significant bits, between 0.5 * 2^-9 and 6 * 448 = 2688.
__device__ __forceinline__ uint4 dq8(uint32_t codes, uint32_t s_lo, uint32_t s_hi) {
  uint32_t v[4], sc[4];
  e2m1x8_to_f16(codes, v);
  e4m3x4_to_f16(s_lo, sc[0], sc[1]);
  e4m3x4_to_f16(s_hi, sc[2], sc[3]);
  uint32_t h[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const __half2 r = __hmul2(*reinterpret_cast<const __half2*>(&v[j]),
                              *reinterpret_cast<const __half2*>(&sc[j]));
    h[j] = *reinterpret_cast<const uint32_t*>(&r);
  }
  return make_uint4(h[0], h[1], h[2], h[3]);
}

// 8 E4M3 bytes (two words, the first byte lowest) -> one 16-byte chunk of
// fp16 values (exact: E4M3 is a subset of fp16). *nan gets a nonzero bit for
// each E4M3 NaN byte (0x7f, 0xff).
__device__ __forceinline__ uint4 e4m3x8(uint32_t a, uint32_t b, uint32_t* nan) {
  uint4 r;
  e4m3x4_to_f16(a, r.x, r.y);
  e4m3x4_to_f16(b, r.z, r.w);
  *nan |= __vcmpeq4(a & 0x7f7f7f7fu, 0x7f7f7f7fu) | __vcmpeq4(b & 0x7f7f7f7fu, 0x7f7f7f7fu);
  return r;
}

struct AttnParams {
  const uint16_t* q;
  const uint8_t* kv_packed;     // codes [B][N][D/2]; or rows [B][N][D/2 + D/16] (16-channel scales)
  const uint8_t* kv_scale;      // block scales [B][N/64][D]; unused for the 16-channel layout
  const int32_t* topk;
  const uint8_t* swa_kv;        // window memory [B][Tw][D] E4M3 (entries K .. Ktot-1), or null
  const int32_t* swa_n;         // [B][Tq]: the window of row (b, t) ends before token swa_n
  int Tw, W;
  int Ktot;                     // K selected entries, then W window slots
  int Tq, Hq, N, K, split_len, nsplit, nhb;
  float softmax_scale;
  uint16_t* out;
  float* lse;
  float* ws_o;
  float2* ws_ml;
  int* err;
  int cluster_merge;   // the splits of a (row, head block) form a cluster and merge in DSMEM
  int q_before_wait;   // the query may be read before the wait for the preceding kernel
};

// Raw bytes a producer lane holds for one entry: the codes (8 B) and scales
// (16 B) of dims 16u .. 16u+15 and of dims 256+16u .. 256+16u+15; for a window
// token (win), its E4M3 bytes of those dims in s[0] and s[1].
struct Raw {
  uint2 c[2];
  uint4 s[2];
  bool win;
};

// The columns of the O accumulator a warp writes out at the end: its quadrant's
// softmax warp takes chunks 0-2 of 32 columns, producer warp q (q < 4) chunks
// 3-5 and producer warp q + 4 chunks 6-7 (a 16x32bx2 load covers chunk c and
// chunk c + 8, 256 columns apart).
__device__ __forceinline__ void out_chunks(int warp, int& c_begin, int& c_end) {
  if (warp > kMmaWarp) {
    c_begin = 0;
    c_end = 3;
  } else if (warp < 4) {
    c_begin = 3;
    c_end = 6;
  } else {
    c_begin = 6;
    c_end = 8;
  }
}

// kG16: the cache is in the pages' own layout, one E4M3 scale per 16 channels
// stored after the entry's codes (288 bytes per entry), instead of one scale
// per channel per 64-entry block in a separate array.
template <bool kG16>
__global__ void __launch_bounds__(kThreads, 1) sparse_attn_tc_kernel(const AttnParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* vs = base;                              // [3 buffers][8 atoms][64 entries][128 B]
  uint8_t* ps = vs + kRing * kVTile;               // [3 buffers][64 heads][128 B]
  Smem& sm = *reinterpret_cast<Smem*>(ps + kRing * kAtom);
  volatile int* abort_flag = &sm.abort_flag;

  const size_t row = blockIdx.x;
  const int hb = blockIdx.y, split = blockIdx.z;
  const int b = (int)(row / p.Tq);
  const int h0 = hb * kHB;
  const int nh = min(kHB, p.Hq - h0);
  const int k_begin = split * p.split_len;
  const int k_end = min(p.Ktot, k_begin + p.split_len);
  const int nt = (k_end - k_begin + kT - 1) / kT;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(&sm.bar.q_ld, 1);
    mbar_init(&sm.bar.q_conv, kProducerWarps);
    mbar_init(&sm.bar.q_full, kProducerWarps);
    mbar_init(&sm.bar.q_free, kProducerWarps);
    mbar_init(&sm.bar.o_full, 1);
    for (int i = 0; i < kRing; ++i) {
      mbar_init(&sm.bar.v_full[i], kProducerWarps);
      mbar_init(&sm.bar.v_free[i], 1);
      mbar_init(&sm.bar.s_full[i], 1);
      mbar_init(&sm.bar.p_full[i], 4);
    }
    sm.abort_flag = 0;
    fence_mbar_init();
    // the block's query rows (1 KB each, contiguous) into V slot 2 in one bulk
    // copy: before the wait for the preceding kernel when the caller vouches
    // that the query was complete before it (the layer step: it comes from
    // before the scorer, two kernels back)
    if (p.q_before_wait) {
      const uint32_t qbytes = (uint32_t)nh * kD * 2;
      mbar_arrive_expect_tx(&sm.bar.q_ld, qbytes);
      bulk_load(vs + 2 * kVTile, p.q + ((row * p.Hq) + h0) * kD, qbytes, &sm.bar.q_ld);
    }
  }
  if (warp == kMmaWarp) tmem_alloc(&sm.tmem_slot, kTmemCols);
  pdl_wait_and_release();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0 && !p.q_before_wait) {
    const uint32_t qbytes = (uint32_t)nh * kD * 2;
    mbar_arrive_expect_tx(&sm.bar.q_ld, qbytes);
    bulk_load(vs + 2 * kVTile, p.q + ((row * p.Hq) + h0) * kD, qbytes, &sm.bar.q_ld);
  }
  const uint32_t tmem = sm.tmem_slot;
  const uint32_t vs_s = smem_u32(vs), ps_s = smem_u32(ps);
  const int quad = warp & 3;
  const uint32_t lanes_s = (uint32_t)(quad * 32) << 16;        // S and Q rows: lanes 0-15
  const uint32_t lanes_o = (uint32_t)(quad * 32 + 16) << 16;   // O rows: lanes 16-31
  float m_ref = -INFINITY, l = 0.0f;    // softmax threads: the head's maximum, partial row sum

  if (warp < kProducerWarps) {
    // ------------------------------------------------------------ gather + dequantise
    // Warp w gathers entries 8w .. 8w+7 of every tile, two per round: lane
    // 16 j + u takes dims 16u .. 16u+15 and 256+16u .. 256+16u+15 of entry
    // 8w + 2r + j, so each load of a warp covers whole 128-byte lines of two
    // rows (one line of codes or two of scales per row) instead of 32 rows.
    const int u = lane & 15, half = lane >> 4;
    constexpr size_t kRowBytes = kG16 ? kD / 2 + kD / 16 : kD / 2;   // bytes of an entry's row
    const uint8_t* pk_b = p.kv_packed + (size_t)b * p.N * kRowBytes;
    const uint8_t* sc_b = kG16 ? nullptr : p.kv_scale + (size_t)b * (p.N / kBlockEntries) * kD;
    const int32_t* topk_row = p.topk + row * p.K;
    // the row's window: tokens [w_lo, w_hi) of its window memory (an end
    // outside [0, Tw] is recorded and leaves the window empty)
    const uint8_t* swa_b = p.swa_kv ? p.swa_kv + (size_t)b * p.Tw * kD : nullptr;
    int w_hi = 0, w_lo = 0;
    if (p.swa_kv && p.Ktot > p.K) {
      w_hi = __ldg(p.swa_n + row);
      if (w_hi < 0 || w_hi > p.Tw) {
        if (lane == 0 && warp == 0 && hb == 0 && split == 0) record_error(p.err, CSA2_ERR_DEVICE_INDEX);
        w_hi = 0;
      }
      w_lo = max(0, w_hi - p.W);
    }

    // lanes 0-7: index of entry 8w + lane of tile t, as loaded (checked later:
    // the check waits for the load, so it runs a tile after the load was
    // issued). Window slot s (entry K + s) is token w_lo + s, given as
    // -2 - token, or -1 past the window's end.
    auto fetch_index = [&](int t) -> int {
      const int kk = k_begin + t * kT + warp * 8 + lane;
      if (lane >= 8 || t >= nt || kk >= k_end) return -1;
      if (kk < p.K) return __ldg(topk_row + kk);
      const int tok = w_lo + (kk - p.K);
      return tok < w_hi ? -2 - tok : -1;
    };
    auto check_index = [&](int id, int t) -> int {
      if (k_begin + t * kT + warp * 8 + lane >= p.K) return id;   // a window slot, not loaded
      if (id >= p.N || id < -1) {
        record_error(p.err, CSA2_ERR_DEVICE_INDEX);
        id = -1;
      }
      return id;
    };
    // L2 prefetch of the warp's 8 rows: lane 4 j + q, q = 0, 1, half of the
    // packed row of entry j; q = 2, 3, half of its scale row. A 288-byte row
    // of the 16-channel layout starts 32-byte aligned, so lines q = 0, 1, 2
    // cover it.
    auto prefetch_rows = [&](int ids) {
      const int id = __shfl_sync(0xffffffffu, ids, lane >> 2);
      if (id <= -2) {
        // a window token: its 512-byte E4M3 row, one line per lane
        const uint8_t* wr = swa_b + (size_t)(-2 - id) * kD + (lane & 3) * 128;
        asm volatile("prefetch.global.L2::evict_last [%0];" ::"l"(wr));
      } else if (id >= 0) {
        const int q = lane & 3;
        if (kG16) {
          if (q < 3) {
            const uint8_t* pr = pk_b + (size_t)id * kRowBytes + q * 128;
            asm volatile("prefetch.global.L2::evict_last [%0];" ::"l"(pr));
          }
        } else if (q < 2) {
          const uint8_t* pr = pk_b + (size_t)id * kRowBytes + q * 128;
          asm volatile("prefetch.global.L2::evict_last [%0];" ::"l"(pr));
        } else {
          const uint8_t* sr = sc_b + (size_t)(id / kBlockEntries) * kD + (q - 2) * 256;
          asm volatile("prefetch.global.L2::evict_last [%0];" ::"l"(sr));
          asm volatile("prefetch.global.L2::evict_last [%0];" ::"l"(sr + 128));
        }
      }
    };
    // half hf of a warp's share of a tile: rounds 2 hf and 2 hf + 1 (four entries)
    auto load_half = [&](int ids, Raw (&r)[2], int hf) {
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int id = __shfl_sync(0xffffffffu, ids, 2 * (2 * hf + k) + half);
        r[k].win = id <= -2;
        if (id <= -2) {
          const uint8_t* wr = swa_b + (size_t)(-2 - id) * kD + 16 * u;
          r[k].s[0] = ldg_v4(wr);
          r[k].s[1] = ldg_v4(wr + 256);
        } else if (id >= 0) {
          const uint8_t* pr = pk_b + (size_t)id * kRowBytes + 8 * u;
          r[k].c[0] = ldg_v2(pr);
          r[k].c[1] = ldg_v2(pr + 128);
          if (kG16) {
            // dims 16u .. 16u+15 are group u, dims 256+16u .. group 16+u: one
            // scale byte each, repeated for the eight dims of a dequantised chunk
            const uint8_t* sr = pk_b + (size_t)id * kRowBytes + kD / 2 + u;
            const uint32_t s0 = 0x01010101u * ldg_u8(sr), s1 = 0x01010101u * ldg_u8(sr + 16);
            r[k].s[0] = make_uint4(s0, s0, s0, s0);
            r[k].s[1] = make_uint4(s1, s1, s1, s1);
          } else {
            const uint8_t* sr = sc_b + (size_t)(id / kBlockEntries) * kD + 16 * u;
            r[k].s[0] = ldg_v4(sr);
            r[k].s[1] = ldg_v4(sr + 256);
          }
        } else {
          r[k].c[0] = r[k].c[1] = make_uint2(0, 0);
          r[k].s[0] = r[k].s[1] = make_uint4(0, 0, 0, 0);
        }
      }
    };
    auto dequant_half = [&](const Raw (&r)[2], uint4 (&d)[2][4]) {
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        if (r[k].win) {
          uint32_t nan = 0;
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            d[k][2 * hh] = e4m3x8(r[k].s[hh].x, r[k].s[hh].y, &nan);
            d[k][2 * hh + 1] = e4m3x8(r[k].s[hh].z, r[k].s[hh].w, &nan);
          }
          if (nan) record_error(p.err, CSA2_ERR_NONFINITE);
        } else {
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            d[k][2 * hh] = dq8(r[k].c[hh].x, r[k].s[hh].x, r[k].s[hh].y);
            d[k][2 * hh + 1] = dq8(r[k].c[hh].y, r[k].s[hh].z, r[k].s[hh].w);
          }
        }
      }
    };
    auto store_half = [&](uint32_t tile, const uint4 (&d)[2][4], int hf) {
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int e = warp * 8 + 2 * (2 * hf + k) + half;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          // dims 256 hh + 16 u .. + 15: atom 4 hh + u / 4, chunks 2 (u % 4) and 2 (u % 4) + 1;
          // the two rows of a store differ in parity, so its 32 lanes cover
          // all eight 16-byte bank groups four times
          const uint32_t dst = tile + (uint32_t)((4 * hh + (u >> 2)) * kAtom);
          const int c = (u & 3) * 2;
          sts128(dst + swz(e, c), d[k][2 * hh]);
          sts128(dst + swz(e, c + 1), d[k][2 * hh + 1]);
        }
      }
    };
    // ---- Q into tensor memory (lanes 0-15, columns 192 + d/2). The block's
    // query rows arrive by one bulk copy into V slot 2. Producer warps w and
    // w + 4 convert quadrant w % 4's 16 rows in place, 8 rows each, two rows
    // at a time with all 32 lanes: bf16 -> fp16 scaled per head by a power of
    // two (so every bf16 bit survives), 16-byte chunk c of row hh stored at chunk
    // c ^ (hh & 7). A row's largest magnitude is taken on the bf16 bit patterns
    // (non-negative floats order like their bits) with one warp reduction. Then
    // thread (h, ch) of warp w moves dims 256 ch + 128 (w / 4) .. + 127 of row h
    // into tensor memory. This overlaps the first tile's row loads.
    auto stage_q = [&]() {
      const uint32_t qsm = vs_s + 2 * kVTile;
      bool ok = mbar_wait_warp(&sm.bar.q_ld, 0, abort_flag);
      if (ok) {
        constexpr int kQRows = 2;
#pragma unroll 1
        for (int i0 = 0; i0 < 8; i0 += kQRows) {
          uint4 a[kQRows], c[kQRows];
          uint32_t amax[kQRows];
#pragma unroll
          for (int r = 0; r < kQRows; ++r) {
            const int hh = quad * 16 + (warp >> 2) * 8 + i0 + r;
            a[r] = c[r] = make_uint4(0, 0, 0, 0);
            if (hh < nh) {                                   // warp-uniform
              a[r] = lds128(qsm + hh * 1024 + 16 * lane);
              c[r] = lds128(qsm + hh * 1024 + 512 + 16 * lane);
            }
            // |x| of 16 bf16 values as 16-bit integers, maximum by pairs
            const uint32_t m = __vmaxu2(
                __vmaxu2(__vmaxu2(a[r].x & 0x7fff7fffu, a[r].y & 0x7fff7fffu),
                         __vmaxu2(a[r].z & 0x7fff7fffu, a[r].w & 0x7fff7fffu)),
                __vmaxu2(__vmaxu2(c[r].x & 0x7fff7fffu, c[r].y & 0x7fff7fffu),
                         __vmaxu2(c[r].z & 0x7fff7fffu, c[r].w & 0x7fff7fffu)));
            amax[r] = __reduce_max_sync(0xffffffffu, max(m & 0xffffu, m >> 16));
          }
          __syncwarp();                                      // the rows are read before they are rewritten
#pragma unroll
          for (int r = 0; r < kQRows; ++r) {
            const int hh = quad * 16 + (warp >> 2) * 8 + i0 + r;
            if (hh >= nh) continue;                          // warp-uniform
            // amax < 2^ex with ex from the exponent field; scaling by 2^e, e = 15 - ex,
            // keeps every magnitude below 2^15 and is exact (clamped to |e| <= 100)
            int ex2 = 0;
            const uint32_t eb = (amax[r] >> 7) & 0xffu;      // bf16 exponent field
            if (amax[r] != 0u && eb != 0xffu) {
              // subnormal maxima (eb == 0) are below 2^-126: the clamp decides
              const int ex = (int)eb - 126;
              ex2 = min(100, max(-100, 15 - ex));
            }
            const float up = __uint_as_float((uint32_t)(127 + ex2) << 23);
            const uint32_t w[8] = {a[r].x, a[r].y, a[r].z, a[r].w, c[r].x, c[r].y, c[r].z, c[r].w};
            uint32_t f[8];
#pragma unroll
            for (int k = 0; k < 8; ++k)
              f[k] = pack_half2(__uint_as_float(w[k] << 16) * up,
                                __uint_as_float(w[k] & 0xffff0000u) * up);
            const uint32_t qr = qsm + hh * 1024;
            sts128(qr + ((lane ^ (hh & 7)) << 4), make_uint4(f[0], f[1], f[2], f[3]));
            sts128(qr + (((32 + lane) ^ (hh & 7)) << 4), make_uint4(f[4], f[5], f[6], f[7]));
            if (lane == 0) sm.qdown[hh] = __uint_as_float((uint32_t)(127 - ex2) << 23);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.bar.q_conv);
      ok = mbar_wait_warp(&sm.bar.q_conv, 0, abort_flag) && ok;
      const int h = quad * 16 + (lane & 15), ch = lane >> 4;
#pragma unroll 1
      for (int i = 2 * (warp >> 2); i < 2 * (warp >> 2) + 2; ++i) {
        uint32_t pk[32];
        if (ok && h < nh) {
          const uint32_t qr = qsm + h * 1024;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int cl = 32 * ch + 8 * i + j;                // logical 16-byte chunk of the row
            const uint4 v = lds128(qr + ((cl ^ (h & 7)) << 4));
            pk[4 * j] = v.x;
            pk[4 * j + 1] = v.y;
            pk[4 * j + 2] = v.z;
            pk[4 * j + 3] = v.w;
          }
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) pk[j] = 0u;
        }
        // threads 0-15: columns 192 + 32 i + j (dims 64 i + 2 j, + 1); threads
        // 16-31: 128 columns further (dims 256 + ...)
        tmem_st16x2_32<128>(tmem + lanes_s + kTmemQ + 32u * i, pk);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&sm.bar.q_full);
        mbar_arrive(&sm.bar.q_free);
      }
    };

    // Indices loaded three tiles ahead (and checked a tile later, when the load
    // has landed), rows prefetched into L2 two tiles ahead, and the next tile's
    // raw bytes loaded while this tile is dequantised (half by half), so a
    // producer never waits for a load it has just issued.
    int id_cur = check_index(fetch_index(0), 0);
    int id_next = check_index(fetch_index(1), 1);
    int id_after = check_index(fetch_index(2), 2);
    int id_far = fetch_index(3);
    prefetch_rows(id_cur);
    prefetch_rows(id_next);
    prefetch_rows(id_after);
    Raw ra[2], rb[2];
    load_half(id_cur, ra, 0);
    load_half(id_cur, rb, 1);
    // the query block is staged while the first tile's rows are in flight
    stage_q();
    for (int t = 0; t < nt; ++t) {
      const int buf = t % kRing;
      uint4 dq[2][4];
      dequant_half(ra, dq);
      load_half(id_next, ra, 0);
      const uint32_t vb = __ballot_sync(0xffffffffu, id_cur != -1);   // lanes 8-31 hold -1
      // the slot (and its valid bits) is free once P(t-3) V(t-3) has completed;
      // slot 2 first holds the query block until the softmax warps have read it
      if (!mbar_wait_warp(&sm.bar.v_free[buf], ((t / kRing) & 1) ^ 1, abort_flag)) break;
      if (t == 2 && !mbar_wait_warp(&sm.bar.q_free, 0, abort_flag)) break;
      if (lane == 0) reinterpret_cast<uint8_t*>(sm.valid[buf])[warp] = (uint8_t)vb;
      const uint32_t tile = vs_s + (uint32_t)(buf * kVTile);
      store_half(tile, dq, 0);
      dequant_half(rb, dq);
      load_half(id_next, rb, 1);
      store_half(tile, dq, 1);
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.bar.v_full[buf]);
      const int id_far_checked = check_index(id_far, t + 3);
      prefetch_rows(id_far_checked);
      id_far = fetch_index(t + 4);
      id_cur = id_next;
      id_next = id_after;
      id_after = id_far_checked;
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t id_s = idesc_f16(64, kT, 0);
      const uint32_t id_o = idesc_f16(64, 256, 1);
      const uint64_t vk = desc_sw128(smem_u32(vs), 16, 1024);       // V tile as K-major B
      const uint64_t vn = desc_sw128(smem_u32(vs), kAtom, 1024);    // V tile as N-major B
      const uint64_t pd = desc_sw128(smem_u32(ps), 16, 1024);       // P as K-major A
      bool ok = mbar_wait(&sm.bar.q_full, 0, abort_flag);
      tc_fence_after();
      // S(t) into buffer t % 3: lanes 0-15, columns 64 (t % 3) .. + 63
      auto issue_s = [&](int t) -> bool {
        const int buf = t % kRing;
        if (!mbar_wait(&sm.bar.v_full[buf], (t / kRing) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint32_t d = tmem + 64u * buf;
        const uint32_t v_lo = (uint32_t)vk + (uint32_t)((buf * kVTile) >> 4);
        const uint32_t v_hi = (uint32_t)(vk >> 32);
#pragma unroll
        for (int a = 0; a < 8; ++a)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ts(d, tmem + kTmemQ + 8u * (4 * a + kk),
                   v_lo + (uint32_t)((a * kAtom + kk * 32) >> 4), v_hi, id_s,
                   (a > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&sm.bar.s_full[buf]);
        return true;
      };
      auto issue_pv = [&](int t) {
        const int buf = t % kRing;
        tc_fence_after();
        const uint32_t p_lo = (uint32_t)pd + (uint32_t)((buf * kAtom) >> 4);
        const uint32_t p_hi = (uint32_t)(pd >> 32);
        const uint32_t n_lo = (uint32_t)vn + (uint32_t)((buf * kVTile) >> 4);
        const uint32_t n_hi = (uint32_t)(vn >> 32);
        const uint32_t acc0 = t > 0 ? 1u : 0u;
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int ks = 0; ks < kT / 16; ++ks)
            mma_ss(tmem + (16u << 16) + 256u * h, p_lo + (uint32_t)((ks * 32) >> 4),
                   n_lo + (uint32_t)((h * 4 * kAtom + ks * 2048) >> 4), p_hi, n_hi, id_o,
                   ks > 0 ? 1u : acc0);
        // the V slot, and (through the in-order completion of later MMAs) the P
        // buffer, are free once this has completed
        mma_commit(&sm.bar.v_free[buf]);
      };
      if (ok && nt > 0) ok = issue_s(0);
      // Then whichever is ready first: P(t) V(t) once the softmax published P(t),
      // or S(t') (t' <= t + 2: its S and P buffers were released by the issue of
      // P(t'-3) V(t'-3), which completes before S(t')) once the producers
      // published its tile. Polling is bounded like mbar_wait.
      int next_pv = 0, next_s = min(nt, 1);
      const uint64_t t0 = global_ns();
      uint32_t spins = 0;
      while (ok && next_pv < nt) {
        bool did = false;
        if (mbar_test_wait(&sm.bar.p_full[next_pv % kRing], (next_pv / kRing) & 1)) {
          issue_pv(next_pv++);
          did = true;
        }
        if (next_s < nt && next_s <= next_pv + kRing - 1 &&
            mbar_test_wait(&sm.bar.v_full[next_s % kRing], (next_s / kRing) & 1)) {
          ok = issue_s(next_s++);
          did = true;
        }
        if (!did) {
          // test_wait does not suspend: sleep between polls, so that this
          // warp leaves its sub-partition's issue slots to the producer and
          // softmax warps that share it
          __nanosleep(40);
          if ((++spins & 63u) == 0u && (*abort_flag || global_ns() - t0 > kWaitLimitNs)) {
            *abort_flag = 1;
            ok = false;
          }
        }
      }
      mma_commit(&sm.bar.o_full);
      // nothing may be in flight when tensor memory is released
      mbar_wait(&sm.bar.o_full, 0, abort_flag);
    }
  } else {
    // ------------------------------------------------------------ Q, softmax
    const int hl = lane & 15, ch = lane >> 4;        // head in the quadrant, half of the tile
    const int h = quad * 16 + hl;                    // head of this thread within the block
    // the producers stage Q (and the per-head scales) first
    bool ok = mbar_wait_warp(&sm.bar.q_full, 0, abort_flag);
    const float hs = (ok && h < nh) ? p.softmax_scale * kLog2e * sm.qdown[h] : 0.0f;
    for (int t = 0; ok && t < nt; ++t) {
      const int buf = t % kRing;
      const uint32_t ph = (t / kRing) & 1;
      // S(t) complete also means P(t-3) V(t-3) is: P buffer t % 3 is free; the
      // valid bits of tile t were written before its V tile was published
      ok = mbar_wait_warp(&sm.bar.v_full[buf], ph, abort_flag) &&
           mbar_wait_warp(&sm.bar.s_full[buf], ph, abort_flag);
      if (!ok) break;
      tc_fence_after();
      const uint32_t vw0 = sm.valid[buf][0], vw1 = sm.valid[buf][1];
      const bool all_valid = (vw0 & vw1) == 0xffffffffu;     // the same for every lane
      const uint32_t vw = ch ? vw1 : vw0;                      // entries 32 ch .. 32 ch + 31
      float y[32];
      tmem_ld16x2_32<32>(tmem + lanes_s + 64u * buf, y);
      // logits in the log2 domain and their maximum over the selected entries
      float xmax = -INFINITY;
      if (all_valid) {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          y[j] *= hs;
          xmax = fmaxf(xmax, y[j]);
        }
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          y[j] *= hs;
          xmax = fmaxf(xmax, ((vw >> j) & 1u) ? y[j] : -INFINITY);
        }
      }
      xmax = fmaxf(xmax, __shfl_xor_sync(0xffffffffu, xmax, 16));
      // lazy reference maximum: raise it only when P would exceed 2^8 (always on
      // the first tile with a selected entry, where the reference is -inf)
      const bool raise = xmax > m_ref + kRescaleSlack;
      if (__any_sync(0xffffffffu, raise)) {
        float alpha = 1.0f;
        const bool had = m_ref != -INFINITY;
        if (raise) {
          alpha = had ? fast_exp2(m_ref - xmax) : 0.0f;
          m_ref = xmax;
          l *= alpha;
        }
        // O (lanes 16-31) holds P(0..t-1) V: rescale it by the head's factor once
        // P(t-1) V(t-1) has completed (P(t) V(t) waits for this tile's P)
        const bool need = raise && had;
        if (t > 0 && __any_sync(0xffffffffu, need)) {
          ok = mbar_wait_warp(&sm.bar.v_free[(t - 1) % kRing], ((t - 1) / kRing) & 1,
                              abort_flag);
          if (!ok) break;
          tc_fence_after();
          const float f = need ? alpha : 1.0f;
#pragma unroll 1
          for (int c0 = 0; c0 < kD / 2; c0 += 32) {
            float o[32];
            tmem_ld16x2_32<256>(tmem + lanes_o + c0, o);
            uint32_t ow[32];
#pragma unroll
            for (int c = 0; c < 32; ++c) ow[c] = __float_as_uint(o[c] * f);
            tmem_st16x2_32<256>(tmem + lanes_o + c0, ow);
          }
        }
      }
      // P = 2^(y - m) in fp16 (<= 2^8) as the A operand of P V, and the row sum
      const bool live = m_ref != -INFINITY;
      uint32_t pk[16];
#pragma unroll
      for (int j = 0; j < 32; j += 2) {
        const bool v0 = live && (all_valid || ((vw >> j) & 1u));
        const bool v1 = live && (all_valid || ((vw >> (j + 1)) & 1u));
        const float p0 = v0 ? fast_exp2(y[j] - m_ref) : 0.0f;
        const float p1 = v1 ? fast_exp2(y[j + 1] - m_ref) : 0.0f;
        l += p0 + p1;
        pk[j / 2] = pack_half2(p0, p1);
      }
      const uint32_t prow = ps_s + (uint32_t)(buf * kAtom);
#pragma unroll
      for (int c = 0; c < 4; ++c)
        sts128(prow + swz(h, 4 * ch + c),
               make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]));
      fence_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.bar.p_full[buf]);
    }
    const float l_tot = l + __shfl_xor_sync(0xffffffffu, l, 16);
    if (ch == 0) sm.mlf[h] = make_float2(l_tot > 0.0f ? m_ref : -INFINITY, l_tot);
  }

  // ---------------------------------------------------------------- output
  // Every warp that reaches a quadrant's O lanes waits for the last P V, then
  // handles its chunks of the quadrant's 16 heads: the final output (one
  // split), the partial staged for the in-cluster merge, or the partial in the
  // workspace.
  const bool writer = warp != kMmaWarp;
  bool have_o = false;
  if (writer) have_o = mbar_wait_warp(&sm.bar.o_full, 0, abort_flag);
  tc_fence_before();
  __syncthreads();                 // O is final, the (max, sum) pairs are in shared memory
  tc_fence_after();
  const int ns = p.nsplit;
  const int share = merge_share(ns);                   // heads each split of a cluster merges
  const uint32_t mlb = merge_ml_bytes(ns);
  if (writer && have_o) {
    const int hl = lane & 15, ch = lane >> 4;
    const int h = quad * 16 + hl;
    const float2 mlh = sm.mlf[h];
    const float l_tot = mlh.y;
    int cb, ce;
    out_chunks(warp, cb, ce);
    const size_t slot = (row * p.nhb + hb) * p.nsplit + split;
    const int owner = h / share, hh = h - owner * share;
    const uint32_t send_row = vs_s + kMergeSendOff + (uint32_t)(owner * share + hh) * 1024u;
#pragma unroll 1
    for (int c = cb; c < ce; ++c) {
      float o[32];
      tmem_ld16x2_32<256>(tmem + lanes_o + 32u * c, o);
      if (h >= nh) continue;
      const int d0 = 256 * ch + 32 * c;           // this thread's dims d0 .. d0 + 31
      if (ns == 1) {
        const float f = l_tot > 0.0f ? 1.0f / l_tot : 0.0f;
        uint4* dst = reinterpret_cast<uint4*>(p.out + ((row * p.Hq) + h0 + h) * kD + d0);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          dst[k] = make_uint4(pack_bf162(o[8 * k] * f, o[8 * k + 1] * f),
                              pack_bf162(o[8 * k + 2] * f, o[8 * k + 3] * f),
                              pack_bf162(o[8 * k + 4] * f, o[8 * k + 5] * f),
                              pack_bf162(o[8 * k + 6] * f, o[8 * k + 7] * f));
      } else if (p.cluster_merge) {
        // normalised by this split's row sum (a convex combination of values,
        // |o| <= 2688, so fp16 holds it); nothing selected gives zeros
        const float f = l_tot > 0.0f ? 1.0f / l_tot : 0.0f;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int cl = d0 / 8 + k;                  // logical 16-byte chunk of the row
          sts128(send_row + ((cl ^ (hh & 7)) << 4),
                 make_uint4(pack_half2(o[8 * k] * f, o[8 * k + 1] * f),
                            pack_half2(o[8 * k + 2] * f, o[8 * k + 3] * f),
                            pack_half2(o[8 * k + 4] * f, o[8 * k + 5] * f),
                            pack_half2(o[8 * k + 6] * f, o[8 * k + 7] * f)));
        }
      } else {
        // unnormalised, with the split's (max, sum), for the combine kernel;
        // a split with nothing selected contributes zeros
        const float f = l_tot > 0.0f ? 1.0f : 0.0f;
        float4* dst = reinterpret_cast<float4*>(p.ws_o + (slot * kHB + h) * kD + d0);
#pragma unroll
        for (int k = 0; k < 8; ++k)
          dst[k] = make_float4(f * o[4 * k], f * o[4 * k + 1], f * o[4 * k + 2],
                               f * o[4 * k + 3]);
      }
    }
    if (warp > kMmaWarp && ch == 0 && h < nh) {
      if (ns == 1) {
        if (p.lse)
          p.lse[row * p.Hq + h0 + h] =
              l_tot > 0.0f ? (mlh.x + log2f(l_tot)) * kLn2 : -INFINITY;
      } else if (p.cluster_merge) {
        reinterpret_cast<float2*>(vs + kMergeSendMlOff + owner * mlb)[hh] = mlh;
      } else {
        p.ws_ml[slot * kHB + h] = mlh;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }

  if (p.cluster_merge) {
    // Every split has staged its partials and, after the first cluster
    // barrier, every V region is idle. Split s copies its group for owner r into
    // r's receive area, slot s (all threads, 16 bytes at a time through
    // distributed shared memory); after the second barrier each split merges
    // the heads [s share, (s + 1) share) from its own group and the ones it
    // received: out = sum_r w_r o_r with o_r the partial normalised by its row
    // sum l_r, w_r = 2^(m_r - M) l_r / L, L = sum_r 2^(m_r - M) l_r,
    // M = max_r m_r. No shared memory of another CTA is touched after the
    // second barrier, so a split may leave as soon as its merge is written.
    cg::cluster_group cl = cg::this_cluster();
    cl.sync();
    {
      const uint32_t blk = (uint32_t)share * 1024u;
      for (int r = 0; r < ns; ++r) {
        if (r == split) continue;
        const uint32_t src = vs_s + kMergeSendOff + (uint32_t)r * blk;
        const uint32_t dst = cluster_addr(vs_s + kMergeRecvOff + (uint32_t)split * blk, (uint32_t)r);
        for (uint32_t o = 16u * threadIdx.x; o < blk; o += 16u * kThreads)
          st_cluster128(dst + o, lds128(src + o));
        const uint32_t msrc = vs_s + kMergeSendMlOff + (uint32_t)r * mlb;
        const uint32_t mdst = cluster_addr(vs_s + kMergeRecvMlOff + (uint32_t)split * mlb, (uint32_t)r);
        for (uint32_t o = 16u * threadIdx.x; o < mlb; o += 16u * kThreads)
          st_cluster128(mdst + o, lds128(msrc + o));
      }
    }
    cl.sync();
    const bool got = !*abort_flag;
    const int hA = split * share, hB = min(nh, hA + share);
    const int nhm = max(0, hB - hA);
    auto part_row = [&](int r, int i) -> uint32_t {
      return r == split ? vs_s + kMergeSendOff + (uint32_t)(split * share + i) * 1024u
                        : vs_s + kMergeRecvOff + (uint32_t)(r * share + i) * 1024u;
    };
    auto part_ml = [&](int r, int i) -> float2 {
      return r == split ? reinterpret_cast<const float2*>(vs + kMergeSendMlOff + split * mlb)[i]
                        : reinterpret_cast<const float2*>(vs + kMergeRecvMlOff + r * mlb)[i];
    };
    // one 16-byte chunk (8 dims) of one head per unit, in a compact loop over
    // the splits (this code runs once per CTA: its size, not its issue rate,
    // decides its time)
    const int units = got ? nhm * (kD / 8) : 0;
#pragma unroll 1
    for (int uo = threadIdx.x; uo < units; uo += kThreads) {
      const int i = uo / (kD / 8), cl16 = uo % (kD / 8);
      const int off = (cl16 ^ (i & 7)) << 4;
      float M = -INFINITY;
#pragma unroll 1
      for (int r = 0; r < ns; ++r) M = fmaxf(M, part_ml(r, i).x);
      float L = 0.0f;
      float acc[8] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll 1
      for (int r = 0; r < ns; ++r) {
        const float2 ml = part_ml(r, i);
        const float wr = (ml.x != -INFINITY && ml.y > 0.0f) ? fast_exp2(ml.x - M) * ml.y : 0.0f;
        L += wr;
        const uint4 v = lds128(part_row(r, i) + off);
        const uint32_t vw[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float2 f2 = __half22float2(*reinterpret_cast<const __half2*>(&vw[k]));
          acc[2 * k] = fmaf(wr, f2.x, acc[2 * k]);
          acc[2 * k + 1] = fmaf(wr, f2.y, acc[2 * k + 1]);
        }
      }
      const float inv = L > 0.0f ? 1.0f / L : 0.0f;
#pragma unroll
      for (int k = 0; k < 8; ++k) acc[k] *= inv;
      *reinterpret_cast<uint4*>(p.out + ((row * p.Hq) + h0 + hA + i) * kD + 8 * cl16) =
          make_uint4(pack_bf162(acc[0], acc[1]), pack_bf162(acc[2], acc[3]),
                     pack_bf162(acc[4], acc[5]), pack_bf162(acc[6], acc[7]));
      if (cl16 == 0 && p.lse)
        p.lse[row * p.Hq + h0 + hA + i] = L > 0.0f ? (M + log2f(L)) * kLn2 : -INFINITY;
    }
  }
  if (threadIdx.x == 0 && *abort_flag) record_error(p.err, CSA2_ERR_TIMEOUT);
}

template <bool kG16>
struct KernelSetup {
  // cudaFuncSetAttribute and the cluster occupancy queries (how many clusters
  // of each size 2 .. kMaxClusterSplits can be resident at once), once per
  // device
  static cudaError_t prepare(bool* clusters_ok, int* capacity = nullptr) {
    static int done[64] = {};
    static int cap[64][kMaxClusterSplits + 1] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!done[dev]) {
      e = cudaFuncSetAttribute(sparse_attn_tc_kernel<kG16>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
      if (e != cudaSuccess) return e;
      for (int cs = 2; cs <= kMaxClusterSplits; ++cs) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(kMaxClusterSplits, 1, (unsigned)cs);
        cfg.blockDim = dim3(kThreads, 1, 1);
        cfg.dynamicSmemBytes = kSmemBytes;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 1;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = (unsigned)cs;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        cap[dev][cs] = cudaOccupancyMaxActiveClusters(&n, sparse_attn_tc_kernel<kG16>, &cfg) ==
                               cudaSuccess ? n : 0;
        (void)cudaGetLastError();
      }
      done[dev] = 1;
    }
    *clusters_ok = cap[dev][kMaxClusterSplits] > 0;
    if (capacity)
      for (int cs = 0; cs <= kMaxClusterSplits; ++cs) capacity[cs] = cs < 2 ? 0 : cap[dev][cs];
    return cudaSuccess;
  }
};

}  // namespace

int sparse_attn_tc_tile() { return kT; }
int sparse_attn_tc_max_cluster() { return kMaxClusterSplits; }

int sparse_attn_tc_cluster_capacity(int cs) {
  if (cs < 2 || cs > kMaxClusterSplits) return 0;
  bool ok = false;
  int cap[kMaxClusterSplits + 1];
  // with no device to ask, assume one wave of clusters fits (host-side sizing)
  if (KernelSetup<false>::prepare(&ok, cap) != cudaSuccess) return 1 << 20;
  return cap[cs];
}

cudaError_t launch_sparse_attn_tc(const uint16_t* q, const uint8_t* kv_packed,
                                  const uint8_t* kv_scale, const int32_t* topk_idx, int rows,
                                  int Tq, int Hq, int N, int K, float softmax_scale, int nhb,
                                  int nsplit, int split_len, uint16_t* out, float* lse,
                                  float* ws_o, float2* ws_ml, int* err, cudaStream_t stream,
                                  bool* merged, const SwaWindow* swa, bool q_ready) {
  AttnParams p;
  p.q = q;
  p.kv_packed = kv_packed;
  p.kv_scale = kv_scale;
  p.topk = topk_idx;
  p.swa_kv = swa ? swa->kv : nullptr;
  p.swa_n = swa ? swa->n : nullptr;
  p.Tw = swa ? swa->Tw : 0;
  p.W = swa ? swa->W : 0;
  p.Ktot = K + p.W;
  p.Tq = Tq;
  p.Hq = Hq;
  p.N = N;
  p.K = K;
  p.split_len = split_len;
  p.nsplit = nsplit;
  p.nhb = nhb;
  p.softmax_scale = softmax_scale;
  p.out = out;
  p.lse = lse;
  p.ws_o = ws_o;
  p.ws_ml = ws_ml;
  p.err = err;
  p.cluster_merge = 0;
  p.q_before_wait = q_ready ? 1 : 0;
  // no block-scale array: rows of the 16-channel layout
  const bool g16 = kv_scale == nullptr;
  void (*kernel)(AttnParams) = g16 ? sparse_attn_tc_kernel<true> : sparse_attn_tc_kernel<false>;
  bool clusters_ok = false;
  cudaError_t e = g16 ? KernelSetup<true>::prepare(&clusters_ok)
                      : KernelSetup<false>::prepare(&clusters_ok);
  if (e != cudaSuccess) return e;
  dim3 grid(rows, nhb, nsplit);
  if (merged != nullptr) *merged = false;
  if (nsplit > 1 && nsplit <= kMaxClusterSplits && merged != nullptr && clusters_ok) {
    // the splits of each (row, head block) as one cluster: merged in DSMEM
    p.cluster_merge = 1;
    e = launch_pdl(kernel, grid, dim3(kThreads), kSmemBytes, stream,
                   dim3(1, 1, (unsigned)nsplit), p);
    if (e == cudaSuccess) {
      *merged = true;
      return cudaSuccess;
    }
    (void)cudaGetLastError();   // fall back to partials in the workspace
    p.cluster_merge = 0;
  }
  if (nsplit > 1 && ws_o == nullptr) return cudaErrorInvalidValue;
  return launch_pdl(kernel, grid, dim3(kThreads), kSmemBytes, stream, dim3(1), p);
}

}  // namespace csa2
