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
// processed in tiles of 64 entries through a two-deep pipeline: while the
// softmax works on tile t, the tensor core runs P(t-1) V(t-1) and S(t+1), and
// the producers dequantise tile t+2. Every selected row is gathered and
// dequantised ONCE, into a shared-memory tile that serves both products:
//   S(t) = Q V(t)^T   M = 64 heads, N = 64 entries, K = 512 (32 MMAs, V tile
//                     read K-major), accumulator in TMEM lanes 16-31 (two
//                     buffers of 64 columns);
//   O   += P(t) V(t)  M = 64 heads, N = 256 dims per half, K = 64 entries
//                     (8 MMAs, V tile read MN-major), accumulator in TMEM
//                     lanes 0-15, all 512 columns.
// A softmax thread owns one head: its 64 logits of a tile, its reference
// maximum and its row sum live in registers, so the softmax needs no barrier.
// The maximum is lazy: P = 2^(s - m) with m raised (and O, l rescaled) only
// when a tile holds a logit more than 8 above it, so P stays below 2^8 in fp16
// and rescaling is rare.
// Values are dequantised with integer ops only (E2M1 magnitudes from a byte
// table, E4M3 scales shifted into fp16 fields); they carry an exact factor 2^-8
// that the softmax scale and the epilogue undo.
// Roles: warps 0-7 gather and dequantise; warp 8 owns TMEM and issues the MMAs;
// warps 9-12 stage Q, run the softmax (S rows in lanes 16-31 of their
// quadrant), the O rescales and the epilogue (O rows in lanes 0-15). Every
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
constexpr int kAtom = 8192;              // 64 rows x 128 B: a K atom of Q or P, or of a V tile
constexpr int kVTile = 8 * kAtom;        // 64 entries x 512 dims of fp16
constexpr int kProducerWarps = 8;
constexpr int kMmaWarp = 8;
constexpr int kThreads = 13 * 32;
constexpr uint32_t kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleSlack = 8.0f;    // log2 units: P <= 2^8 before a rescale

struct __align__(8) Bars {
  uint64_t q_full, o_full;
  uint64_t v_full[2], v_free[2], s_full[2], p_full[2], p_free[2];
};

struct Smem {
  Bars bar;
  uint32_t tmem_slot;
  int abort_flag;
  uint32_t valid[2][kT / 32];   // bit i of word w: entry 32 w + i of the tile is selected
                                // (byte w of a buffer written by producer warp w)
  float head_scale[kHB];
  float2 ml[kHB];               // this split's (reference maximum, row sum) per head
};

constexpr size_t kSmemBytes = 1024 + 8 * kAtom /*Q*/ + 2 * kVTile /*V*/ + 2 * kAtom /*P*/ +
                              sizeof(Smem);

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

// One MMA with each descriptor given as its low word (start address and
// leading offset: advancing it by (bytes >> 4) cannot carry out, shared-memory
// addresses being below 2^18) and a common high word.
__device__ __forceinline__ void mma_f16_lo(uint32_t d, uint32_t a_lo, uint32_t b_lo, uint32_t hi_a,
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

// 8 E2M1 codes (one 32-bit word, low nibble first) times their 8 E4M3 scales
// (two words) -> one 16-byte chunk of fp16 values, times 2^-8. Integer ops only:
//  - E2M1 magnitude m -> high byte of fp16(m) from an 8-entry byte table
//    (0, 0.5, 1, 1.5, 2, 3, 4, 6 -> 00 38 3C 3E 40 42 44 46), sign spliced in;
//  - a non-negative E4M3 byte shifted left by 7 is the fp16 of its value * 2^-8
//    (exponent bias 7 -> 15, mantissa 3 -> 10 bits; subnormals line up too);
//  - the fp16 product is exact (<= 6 significant bits, >= 2^-18).
__device__ __forceinline__ uint4 dq8(uint32_t codes, uint32_t s_lo, uint32_t s_hi) {
  const uint32_t mag = codes & 0x77777777u;
  const uint32_t m_lo = __byte_perm(0x3E3C3800u, 0x46444240u, mag);         // codes 0-3
  const uint32_t m_hi = __byte_perm(0x3E3C3800u, 0x46444240u, mag >> 16);   // codes 4-7
  const uint32_t t = codes << 4;    // sign of each even code -> bit 7 of its byte
  uint32_t h[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t mg = __byte_perm(j < 2 ? m_lo : m_hi, 0u, (j & 1) ? 0x3424u : 0x1404u);
    const uint32_t sg = __byte_perm(t, codes, (uint32_t)((4 + j) * 0x1100 + j * 0x0011));
    const uint32_t v = (mg & 0x7fff7fffu) | (sg & 0x80008000u);
    const uint32_t sc = __byte_perm(j < 2 ? s_lo : s_hi, 0u, (j & 1) ? 0x4342u : 0x4140u) << 7;
    const __half2 r = __hmul2(*reinterpret_cast<const __half2*>(&v),
                              *reinterpret_cast<const __half2*>(&sc));
    h[j] = *reinterpret_cast<const uint32_t*>(&r);
  }
  return make_uint4(h[0], h[1], h[2], h[3]);
}

struct AttnParams {
  const uint16_t* q;
  const uint8_t* kv_packed;     // codes [B][N][D/2]; or rows [B][N][D/2 + D/16] (16-channel scales)
  const uint8_t* kv_scale;      // block scales [B][N/64][D]; unused for the 16-channel layout
  const int32_t* topk;
  int Tq, Hq, N, K, split_len, nsplit, nhb;
  float softmax_scale;
  uint16_t* out;
  float* lse;
  float* ws_o;
  float2* ws_ml;
  int* err;
  int cluster_merge;   // the splits of a (row, head block) form a cluster and merge in DSMEM
};

// float4 chunk c (0..127) of head row h of the fp32 partial staged in the
// V region; the chunk index is swizzled with the row so that the 16 rows
// written at once by a warp fall on different banks
__device__ __forceinline__ int stage_off(int h, int c) { return h * kD + ((c ^ (h & 7)) << 2); }

// 64 columns c0 .. c0 + 63 of head row h of a split's partial O, times f, into
// the fp32 staging area (the idle V region) that the cluster merge reads
__device__ __forceinline__ void stage_partial64(float* stage, int h, int c0, const float (&o)[64],
                                                float f) {
#pragma unroll
  for (int c = 0; c < 16; ++c)
    *reinterpret_cast<float4*>(stage + stage_off(h, c0 / 4 + c)) =
        make_float4(f * o[4 * c], f * o[4 * c + 1], f * o[4 * c + 2], f * o[4 * c + 3]);
}

// Raw bytes a producer lane holds for one entry: the codes (8 B) and scales
// (16 B) of dims 16u .. 16u+15 and of dims 256+16u .. 256+16u+15.
struct Raw {
  uint2 c[2];
  uint4 s[2];
};

// kG16: the cache is in the pages' own layout, one E4M3 scale per 16 channels
// stored after the entry's codes (288 bytes per entry), instead of one scale
// per channel per 64-entry block in a separate array.
template <bool kG16>
__global__ void __launch_bounds__(kThreads, 1) sparse_attn_tc_kernel(const AttnParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* qs = base;                              // [8 atoms][64 heads][128 B]
  uint8_t* vs = qs + 8 * kAtom;                    // [2 buffers][8 atoms][64 entries][128 B]
  uint8_t* ps = vs + 2 * kVTile;                   // [2 buffers][64 heads][128 B]
  Smem& sm = *reinterpret_cast<Smem*>(ps + 2 * kAtom);
  volatile int* abort_flag = &sm.abort_flag;

  const size_t row = blockIdx.x;
  const int hb = blockIdx.y, split = blockIdx.z;
  const int b = (int)(row / p.Tq);
  const int h0 = hb * kHB;
  const int nh = min(kHB, p.Hq - h0);
  const int k_begin = split * p.split_len;
  const int k_end = min(p.K, k_begin + p.split_len);
  const int nt = (k_end - k_begin + kT - 1) / kT;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(&sm.bar.q_full, 4);
    mbar_init(&sm.bar.o_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.bar.v_full[i], kProducerWarps);
      mbar_init(&sm.bar.v_free[i], 1);
      mbar_init(&sm.bar.s_full[i], 1);
      mbar_init(&sm.bar.p_full[i], 4);
      mbar_init(&sm.bar.p_free[i], 1);
    }
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) tmem_alloc(&sm.tmem_slot, kTmemCols);
  // the block's 64 query rows (64 KB) into L2 now: the softmax warps read them
  // in two dependent batches while the producers wait for their first rows
  for (int i = threadIdx.x; i < nh * (kD * 2 / 128); i += kThreads) {
    const uint16_t* qr = p.q + ((row * p.Hq) + h0 + i / 8) * kD + (i % 8) * 64;
    asm volatile("prefetch.global.L2 [%0];" ::"l"(qr));
  }
  pdl_wait_and_release();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_slot;

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

    // lanes 0-7: index of entry 8w + lane of tile t, as loaded (checked later:
    // the check waits for the load, so it runs a tile after the load was issued)
    auto fetch_index = [&](int t) -> int {
      const int kk = k_begin + t * kT + warp * 8 + lane;
      return (lane < 8 && t < nt && kk < k_end) ? __ldg(topk_row + kk) : -1;
    };
    auto check_index = [&](int id) -> int {
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
      if (id >= 0) {
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
    auto load_raw = [&](int ids, Raw (&r)[4]) {
#pragma unroll
      for (int rr = 0; rr < 4; ++rr) {
        const int id = __shfl_sync(0xffffffffu, ids, 2 * rr + half);
        if (id >= 0) {
          const uint8_t* pr = pk_b + (size_t)id * kRowBytes + 8 * u;
          r[rr].c[0] = __ldg(reinterpret_cast<const uint2*>(pr));
          r[rr].c[1] = __ldg(reinterpret_cast<const uint2*>(pr + 128));
          if (kG16) {
            // dims 16u .. 16u+15 are group u, dims 256+16u .. group 16+u: one
            // scale byte each, repeated for the eight dims of a dequantised chunk
            const uint8_t* sr = pk_b + (size_t)id * kRowBytes + kD / 2 + u;
            const uint32_t s0 = 0x01010101u * __ldg(sr), s1 = 0x01010101u * __ldg(sr + 16);
            r[rr].s[0] = make_uint4(s0, s0, s0, s0);
            r[rr].s[1] = make_uint4(s1, s1, s1, s1);
          } else {
            const uint8_t* sr = sc_b + (size_t)(id / kBlockEntries) * kD + 16 * u;
            r[rr].s[0] = __ldg(reinterpret_cast<const uint4*>(sr));
            r[rr].s[1] = __ldg(reinterpret_cast<const uint4*>(sr + 256));
          }
        } else {
          r[rr].c[0] = r[rr].c[1] = make_uint2(0, 0);
          r[rr].s[0] = r[rr].s[1] = make_uint4(0, 0, 0, 0);
        }
      }
    };

    // Indices loaded three tiles ahead (and checked a tile later, when the load
    // has landed), rows prefetched into L2 two tiles ahead, raw bytes loaded one
    // tile ahead: nothing on a producer's path waits for a load it just issued.
    int id_cur = check_index(fetch_index(0));
    int id_next = check_index(fetch_index(1));
    int id_after = check_index(fetch_index(2));
    int id_far = fetch_index(3);
    prefetch_rows(id_cur);
    prefetch_rows(id_next);
    prefetch_rows(id_after);
    Raw raw[4];
    load_raw(id_cur, raw);
    bool go = true;
    for (int t = 0; go && t < nt; ++t) {
      const int buf = t & 1;
      // the buffer (and its valid bits) is free once P(t-2) V(t-2) has completed
      if (!mbar_wait_warp(&sm.bar.v_free[buf], ((t >> 1) & 1) ^ 1, abort_flag)) {
        go = false;
        break;
      }
      const uint32_t vb = __ballot_sync(0xffffffffu, id_cur >= 0);   // lanes 8-31 hold -1
      if (lane == 0) reinterpret_cast<uint8_t*>(sm.valid[buf])[warp] = (uint8_t)vb;
      uint8_t* tile = vs + buf * kVTile;
#pragma unroll
      for (int rr = 0; rr < 4; ++rr) {
        const int e = warp * 8 + 2 * rr + half;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          // dims 256 hh + 16 u .. + 15: atom 4 hh + u / 4, chunks 2 (u % 4) and 2 (u % 4) + 1;
          // the two rows of a store differ in parity, so its 32 lanes cover
          // all eight 16-byte bank groups four times
          uint8_t* dst = tile + (4 * hh + (u >> 2)) * kAtom;
          const int c = (u & 3) * 2;
          const uint2 cw = raw[rr].c[hh];
          const uint4 sw = raw[rr].s[hh];
          *reinterpret_cast<uint4*>(dst + swz(e, c)) = dq8(cw.x, sw.x, sw.y);
          *reinterpret_cast<uint4*>(dst + swz(e, c + 1)) = dq8(cw.y, sw.z, sw.w);
        }
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.bar.v_full[buf]);
      const int id_far_checked = check_index(id_far);
      prefetch_rows(id_far_checked);
      id_far = fetch_index(t + 4);
      id_cur = id_next;
      id_next = id_after;
      id_after = id_far_checked;
      load_raw(id_cur, raw);
    }
    if (p.cluster_merge && go) {
      // Staging of the split's partial for the merge, shared with the softmax
      // warps: producer warps q and q + 4 take columns 192 (w >> 2) .. + 191 of
      // the 16 O rows of TMEM quadrant q (heads 16 q ..), the softmax warp of
      // the quadrant the last 128. x 2^8 undoes the factor the dequantised
      // values carry; an empty split is skipped by the merge, whatever it stages.
      if (mbar_wait_warp(&sm.bar.o_full, 0, abort_flag)) {
        tc_fence_after();
        const int quad = warp & 3;
        const int hq = quad * 16 + (lane & 15);
        const uint32_t la = (uint32_t)(quad * 32) << 16;
#pragma unroll 1
        for (int k = 0; k < 3; ++k) {
          const int c0 = (warp >> 2) * 192 + k * 64;
          float o[64];
          tmem_ld_64(tmem + la + c0, o);
          if (lane < 16 && hq < nh) stage_partial64(reinterpret_cast<float*>(vs), hq, c0, o, 256.0f);
        }
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t id_s = idesc_f16(64, kT, 0);
      const uint32_t id_o = idesc_f16(64, 256, 1);
      const uint64_t qd = desc_sw128(smem_u32(qs), 16, 1024);
      const uint64_t vk = desc_sw128(smem_u32(vs), 16, 1024);       // V tile as K-major B
      const uint64_t vn = desc_sw128(smem_u32(vs), kAtom, 1024);    // V tile as N-major B
      const uint64_t pd = desc_sw128(smem_u32(ps), 16, 1024);       // P as K-major A
      bool ok = mbar_wait(&sm.bar.q_full, 0, abort_flag);
      // S(t) into buffer t & 1: lanes 16-31, columns 64 (t & 1) .. + 63
      auto issue_s = [&](int t) -> bool {
        const int buf = t & 1;
        if (!mbar_wait(&sm.bar.v_full[buf], (t >> 1) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint32_t d = tmem + (16u << 16) + 64u * buf;
        const uint32_t q_lo = (uint32_t)qd, q_hi = (uint32_t)(qd >> 32);
        const uint32_t v_lo = (uint32_t)vk + (uint32_t)((buf * kVTile) >> 4);
        const uint32_t v_hi = (uint32_t)(vk >> 32);
#pragma unroll
        for (int a = 0; a < 8; ++a)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_f16_lo(d, q_lo + (uint32_t)((a * kAtom + kk * 32) >> 4),
                       v_lo + (uint32_t)((a * kAtom + kk * 32) >> 4), q_hi, v_hi, id_s,
                       (a > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&sm.bar.s_full[buf]);
        return true;
      };
      auto issue_pv = [&](int t) {
        const int buf = t & 1;
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
            mma_f16_lo(tmem + 256u * h, p_lo + (uint32_t)((ks * 32) >> 4),
                       n_lo + (uint32_t)((h * 4 * kAtom + ks * 2048) >> 4), p_hi, n_hi, id_o,
                       ks > 0 ? 1u : acc0);
        mma_commit(&sm.bar.v_free[buf]);
        mma_commit(&sm.bar.p_free[buf]);
      };
      if (ok && nt > 0) ok = issue_s(0);
      if (ok && nt > 1) ok = issue_s(1);
      // Then whichever is ready first: P(t) V(t) once the softmax published P(t),
      // or S(t') (t' <= t + 1: its S and P buffers were released by P(t'-2) V(t'-2))
      // once the producers published its tile. Polling is bounded like mbar_wait.
      int next_pv = 0, next_s = 2;
      const uint64_t t0 = global_ns();
      uint32_t spins = 0;
      while (ok && next_pv < nt) {
        bool did = false;
        if (mbar_test_wait(&sm.bar.p_full[next_pv & 1], (next_pv >> 1) & 1)) {
          issue_pv(next_pv++);
          did = true;
        }
        if (next_s < nt && next_s <= next_pv + 1 &&
            mbar_test_wait(&sm.bar.v_full[next_s & 1], (next_s >> 1) & 1)) {
          ok = issue_s(next_s++);
          did = true;
        }
        if (!did && (++spins & 63u) == 0u) {
          __nanosleep(32);
          if (*abort_flag || global_ns() - t0 > kWaitLimitNs) {
            *abort_flag = 1;
            ok = false;
          }
        }
      }
      mma_commit(&sm.bar.o_full);
      // nothing may be in flight when TMEM is released
      mbar_wait(&sm.bar.o_full, 0, abort_flag);
    }
  } else {
    // ------------------------------------------------------------ Q, softmax, epilogue
    const int quad = warp & 3;
    const int sw = warp - (kMmaWarp + 1);            // 0..3: Q heads 16 sw .. 16 sw + 15
    const bool s_owner = lane >= 16;                 // S rows live in lanes 16-31
    const int h = quad * 16 + (lane & 15);           // head of this lane's S (or O) row
    const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
    // ---- Q, scaled per head by a power of two so that its bf16 values keep
    // every bit in fp16; two batches of eight heads per warp
#pragma unroll 1
    for (int bt = 0; bt < 2; ++bt) {
      uint4 qraw[16];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int hh = sw * 16 + bt * 8 + j;
        if (hh < nh) {
          const uint4* src =
              reinterpret_cast<const uint4*>(p.q + ((row * p.Hq) + h0 + hh) * kD + lane * 16);
          qraw[2 * j] = __ldg(src);
          qraw[2 * j + 1] = __ldg(src + 1);
        } else {
          qraw[2 * j] = make_uint4(0, 0, 0, 0);
          qraw[2 * j + 1] = make_uint4(0, 0, 0, 0);
        }
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int hh = sw * 16 + bt * 8 + j;
        const uint32_t w[8] = {qraw[2 * j].x, qraw[2 * j].y, qraw[2 * j].z, qraw[2 * j].w,
                               qraw[2 * j + 1].x, qraw[2 * j + 1].y, qraw[2 * j + 1].z,
                               qraw[2 * j + 1].w};
        float vals[16];
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          vals[2 * i] = __uint_as_float(w[i] << 16);
          vals[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
          amax = fmaxf(amax, fmaxf(fabsf(vals[2 * i]), fabsf(vals[2 * i + 1])));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        // amax < 2^ex with ex from the exponent field; scaling by 2^e, e = 15 - ex,
        // keeps every magnitude below 2^15 and is exact (clamped to |e| <= 100)
        int ex2 = 0;
        if (amax > 0.0f && isfinite(amax)) {
          const int ex = (int)((__float_as_uint(amax) >> 23) & 0xffu) - 126;
          ex2 = min(100, max(-100, 15 - ex));
        }
        const float up = __uint_as_float((uint32_t)(127 + ex2) << 23);
        uint32_t pk[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) pk[i] = pack_half2(vals[2 * i] * up, vals[2 * i + 1] * up);
        const int atom = lane >> 2, c0 = (lane & 3) * 2;
        uint8_t* dst = qs + atom * kAtom;
        *reinterpret_cast<uint4*>(dst + swz(hh, c0)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        *reinterpret_cast<uint4*>(dst + swz(hh, c0 + 1)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        const float down = __uint_as_float((uint32_t)(127 - ex2) << 23);
        // x 2^8: the dequantised keys/values carry a factor 2^-8
        if (lane == 0) sm.head_scale[hh] = hh < nh ? p.softmax_scale * kLog2e * down * 256.0f : 0.0f;
      }
    }
    fence_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.bar.q_full);
    // every softmax warp reads the scales of its own heads after all four staged Q
    bool ok = mbar_wait_warp(&sm.bar.q_full, 0, abort_flag);
    const float hs = sm.head_scale[h];
    float m_ref = -INFINITY, l = 0.0f;    // meaningful in the S lanes
    for (int t = 0; ok && t < nt; ++t) {
      const int buf = t & 1;
      const uint32_t ph = (t >> 1) & 1;
      // S(t) complete also means P(t-2) V(t-2) is: P buffer t & 1 is free; the
      // valid bits of tile t were written before its V tile was published
      ok = mbar_wait_warp(&sm.bar.v_full[buf], ph, abort_flag) &&
           mbar_wait_warp(&sm.bar.s_full[buf], ph, abort_flag);
      if (!ok) break;
      tc_fence_after();
      const uint32_t vw0 = sm.valid[buf][0], vw1 = sm.valid[buf][1];
      const bool all_valid = (vw0 & vw1) == 0xffffffffu;     // the same for every lane
      float y[64];
      tmem_ld_64(tmem + lane_addr + 64u * buf, y);
      // logits in the log2 domain relative to the current reference maximum,
      // and their maximum over the selected entries
      float xmax = -INFINITY;
      if (all_valid) {
#pragma unroll
        for (int j = 0; j < 64; ++j) {
          y[j] = fmaf(y[j], hs, -m_ref);
          xmax = fmaxf(xmax, y[j]);
        }
      } else {
#pragma unroll
        for (int j = 0; j < 64; ++j) {
          y[j] = fmaf(y[j], hs, -m_ref);
          const bool v = (((j < 32 ? vw0 : vw1) >> (j & 31)) & 1u) != 0u;
          xmax = fmaxf(xmax, v ? y[j] : -INFINITY);
        }
      }
      // lazy reference maximum: raise it only when P would exceed 2^8 (always on
      // the first tile with a selected entry, where the reference is -inf)
      const bool raise = s_owner && xmax > kRescaleSlack;
      float alpha = 1.0f;
      const float m_old = m_ref;
      if (__any_sync(0xffffffffu, raise)) {
        tmem_ld_64(tmem + lane_addr + 64u * buf, y);
        float ymax = -INFINITY;
#pragma unroll
        for (int j = 0; j < 64; ++j) {
          y[j] *= hs;
          const bool v = (((j < 32 ? vw0 : vw1) >> (j & 31)) & 1u) != 0u;
          ymax = fmaxf(ymax, v ? y[j] : -INFINITY);
        }
        if (raise) {
          alpha = m_ref == -INFINITY ? 0.0f : exp2f(m_ref - ymax);
          m_ref = ymax;
          l *= alpha;
        }
#pragma unroll
        for (int j = 0; j < 64; ++j) y[j] -= m_ref;
      }
      // O (lanes 0-15) is rescaled by its S lane's factor once P(t-1) V(t-1) is done
      const bool need = s_owner && alpha != 1.0f && m_old != -INFINITY;
      if (t > 0 && __any_sync(0xffffffffu, need)) {
        // the TMEM loads and stores below cover all 32 lanes of the quadrant:
        // wait until nothing writes them, i.e. P(t-1) V(t-1) (O, lanes 0-15) and
        // S(t+1) (the other S buffer, lanes 16-31, stored back unchanged) are done
        ok = mbar_wait_warp(&sm.bar.p_free[(t - 1) & 1], ((t - 1) >> 1) & 1, abort_flag);
        if (ok && t + 1 < nt)
          ok = mbar_wait_warp(&sm.bar.s_full[(t + 1) & 1], ((t + 1) >> 1) & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
        const float a_o = __shfl_down_sync(0xffffffffu, need ? alpha : 1.0f, 16);
        const float f = s_owner ? 1.0f : a_o;
#pragma unroll 1
        for (int c0 = 0; c0 < kD; c0 += 32) {
          float o[32];
          tmem_ld_32(tmem + lane_addr + c0, o);
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] *= f;
          tmem_st_32(tmem + lane_addr + c0, o);
        }
      }
      // P = 2^y in fp16 (y <= 8) as the A operand of P V, and the row sum
      const bool live = s_owner && m_ref != -INFINITY;
      uint8_t* prow = ps + buf * kAtom;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        uint32_t pk[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int j = 8 * c + 2 * u;
          const uint32_t vw = j < 32 ? vw0 : vw1;
          const bool v0 = live && (all_valid || ((vw >> (j & 31)) & 1u));
          const bool v1 = live && (all_valid || ((vw >> ((j + 1) & 31)) & 1u));
          const float p0 = v0 ? fast_exp2(y[j]) : 0.0f;
          const float p1 = v1 ? fast_exp2(y[j + 1]) : 0.0f;
          l += p0 + p1;
          pk[u] = pack_half2(p0, p1);
        }
        if (s_owner)
          *reinterpret_cast<uint4*>(prow + swz(h, c)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
      fence_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.bar.p_full[buf]);
    }
    // epilogue: O rows live in lanes 0-15; fetch m and l from the S lane (+16)
    const float m_o = __shfl_down_sync(0xffffffffu, m_ref, 16);
    const float l_o = __shfl_down_sync(0xffffffffu, l, 16);
    ok = mbar_wait_warp(&sm.bar.o_full, 0, abort_flag) && ok;
    if (ok) {
      tc_fence_after();
      const bool o_owner = lane < 16 && h < nh;
      const size_t slot = (row * p.nhb + hb) * p.nsplit + split;
      // x 2^8 undoes the 2^-8 carried by the dequantised values; a split with
      // nothing selected writes zeros whatever the accumulator holds
      const float f = l_o > 0.0f ? (p.nsplit == 1 ? 256.0f / l_o : 256.0f) : 0.0f;
#pragma unroll 1
      for (int c0 = p.cluster_merge ? 384 : 0; c0 < kD; c0 += 64) {
        float o[64];
        tmem_ld_64(tmem + lane_addr + c0, o);
        if (!o_owner) continue;
        if (p.nsplit == 1) {
          uint4* dst = reinterpret_cast<uint4*>(p.out + ((row * p.Hq) + h0 + h) * kD + c0);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            uint32_t w[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              __nv_bfloat162 bb = __floats2bfloat162_rn(l_o > 0.0f ? o[8 * c + 2 * u] * f : 0.0f,
                                                        l_o > 0.0f ? o[8 * c + 2 * u + 1] * f : 0.0f);
              w[u] = *reinterpret_cast<uint32_t*>(&bb);
            }
            dst[c] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        } else if (p.cluster_merge) {
          // partial into the idle V region; merged over DSMEM below
          stage_partial64(reinterpret_cast<float*>(vs), h, c0, o, 256.0f);
        } else {
          float4* dst = reinterpret_cast<float4*>(p.ws_o + (slot * kHB + h) * kD + c0);
#pragma unroll
          for (int c = 0; c < 16; ++c)
            dst[c] = l_o > 0.0f ? make_float4(f * o[4 * c], f * o[4 * c + 1], f * o[4 * c + 2],
                                              f * o[4 * c + 3])
                                : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        }
      }
      if (lane < 16 && h < nh) {
        const float2 ml = make_float2(l_o > 0.0f ? m_o : -INFINITY, l_o);
        if (p.nsplit == 1) {
          if (p.lse) p.lse[row * p.Hq + h0 + h] = l_o > 0.0f ? (m_o + log2f(l_o)) * kLn2 : -INFINITY;
        } else if (p.cluster_merge) {
          sm.ml[h] = ml;
        } else {
          p.ws_ml[slot * kHB + h] = ml;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (threadIdx.x == 0 && *abort_flag) record_error(p.err, CSA2_ERR_TIMEOUT);

  if (p.cluster_merge) {
    // Split s of the cluster merges heads [s share, (s + 1) share) of all splits'
    // partials, read over DSMEM: out = sum_r w_r O_r with w_r = 2^(m_r - M) / L,
    // L = sum_r 2^(m_r - M) l_r, M = max_r m_r. The weights of a head are
    // computed once (into the idle Q region); then every thread loads its
    // outputs' partials from all splits before combining them.
    cg::cluster_group cl = cg::this_cluster();
    cl.sync();                                   // every split's partial is staged
    const int ns = p.nsplit;
    const int share = (kHB + ns - 1) / ns;
    const int hA = split * share, hB = min(nh, hA + share);
    const int nhm = max(0, hB - hA);
    float* wts = reinterpret_cast<float*>(qs);   // [head - hA][8 splits]
    for (int i = threadIdx.x; i < nhm; i += kThreads) {
      const int hh = hA + i;
      float mv[8], lv[8];
      float M = -INFINITY;
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        mv[r] = -INFINITY;
        lv[r] = 0.0f;
        if (r < ns) {
          const float2 ml = cl.map_shared_rank(&sm.ml[hh], r)[0];
          mv[r] = ml.x;
          lv[r] = ml.y;
          M = fmaxf(M, ml.x);
        }
      }
      float w[8];
      float L = 0.0f;
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        w[r] = mv[r] != -INFINITY ? exp2f(mv[r] - M) : 0.0f;
        L += w[r] * lv[r];
      }
      const float inv = L > 0.0f ? 1.0f / L : 0.0f;
#pragma unroll
      for (int r = 0; r < 8; ++r) wts[i * 8 + r] = w[r] * inv;
      if (p.lse) p.lse[row * p.Hq + h0 + hh] = L > 0.0f ? (M + log2f(L)) * kLn2 : -INFINITY;
    }
    __syncthreads();
    const int units = nhm * (kD / 4);
    constexpr int kBatch = 2;                    // outputs per thread whose loads are in flight together
#pragma unroll 1
    for (int base = threadIdx.x; base < units; base += kBatch * kThreads) {
      float4 v[kBatch][8];
      float wv[kBatch][8];
#pragma unroll
      for (int j = 0; j < kBatch; ++j) {
        const int u = base + j * kThreads;
        const int i = u / (kD / 4), c = u % (kD / 4);
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          wv[j][r] = (u < units && r < ns) ? wts[i * 8 + r] : 0.0f;
          v[j][r] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
          if (wv[j][r] != 0.0f) {
            const float* st = cl.map_shared_rank(reinterpret_cast<float*>(vs), r);
            v[j][r] = *reinterpret_cast<const float4*>(st + stage_off(hA + i, c));
          }
        }
      }
#pragma unroll
      for (int j = 0; j < kBatch; ++j) {
        const int u = base + j * kThreads;
        if (u >= units) break;
        const int i = u / (kD / 4), c = u % (kD / 4);
        float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          acc.x = fmaf(wv[j][r], v[j][r].x, acc.x);
          acc.y = fmaf(wv[j][r], v[j][r].y, acc.y);
          acc.z = fmaf(wv[j][r], v[j][r].z, acc.z);
          acc.w = fmaf(wv[j][r], v[j][r].w, acc.w);
        }
        __nv_bfloat162 lo2 = __floats2bfloat162_rn(acc.x, acc.y);
        __nv_bfloat162 hi2 = __floats2bfloat162_rn(acc.z, acc.w);
        uint2 pk;
        pk.x = *reinterpret_cast<uint32_t*>(&lo2);
        pk.y = *reinterpret_cast<uint32_t*>(&hi2);
        *reinterpret_cast<uint2*>(p.out + ((row * p.Hq) + h0 + hA + i) * kD + 4 * c) = pk;
      }
    }
    cl.sync();                                   // no split leaves while others read it
  }
}

}  // namespace

int sparse_attn_tc_tile() { return kT; }

cudaError_t launch_sparse_attn_tc(const uint16_t* q, const uint8_t* kv_packed,
                                  const uint8_t* kv_scale, const int32_t* topk_idx, int rows,
                                  int Tq, int Hq, int N, int K, float softmax_scale, int nhb,
                                  int nsplit, int split_len, uint16_t* out, float* lse,
                                  float* ws_o, float2* ws_ml, int* err, cudaStream_t stream,
                                  bool* merged) {
  AttnParams p;
  p.q = q;
  p.kv_packed = kv_packed;
  p.kv_scale = kv_scale;
  p.topk = topk_idx;
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
  // no block-scale array: rows of the 16-channel layout
  void (*kernel)(AttnParams) =
      kv_scale == nullptr ? sparse_attn_tc_kernel<true> : sparse_attn_tc_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid(rows, nhb, nsplit);
  if (merged != nullptr) *merged = false;
  if (nsplit > 1 && nsplit <= 8 && merged != nullptr) {
    // the splits of each (row, head block) as one cluster: merged in DSMEM
    p.cluster_merge = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = (unsigned)nsplit;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int nclusters = 0;
    if (cudaOccupancyMaxActiveClusters(&nclusters, kernel, &cfg) == cudaSuccess &&
        nclusters > 0) {
      e = launch_pdl(kernel, grid, dim3(kThreads), kSmemBytes, stream,
                     dim3(1, 1, (unsigned)nsplit), p);
      if (e == cudaSuccess) {
        *merged = true;
        return cudaSuccess;
      }
    }
    (void)cudaGetLastError();   // fall back to partials in the workspace
    p.cluster_merge = 0;
  }
  return launch_pdl(kernel, grid, dim3(kThreads), kSmemBytes, stream, dim3(1), p);
}

}  // namespace csa2
