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
// processed in tiles of 128 entries. Every selected row is gathered and
// dequantised ONCE, into a shared-memory tile that serves both products, which
// are computed transposed so that the 128 entries (or dims) fill the M = 128
// rows of the tensor core and the TMEM lanes:
//   S^T(t) = V(t) Q^T    M = 128 entries, N = 64 heads, K = 512 (32 MMAs, V tile
//                        read K-major): thread e of the softmax warps owns entry
//                        e and its 64 head logits;
//   O^T   += V(t)^T P^T  M = 128 dims (4 blocks), N = 64 heads, K = 128 entries
//                        (32 MMAs, V tile read MN-major, P^T written row by row);
//   l     += 1^T P^T     one more block whose A operand is a constant tile with
//                        ones in row 0: the softmax row sums come out of the MMA.
// The V tile is stored as two halves of 256 dims, so the producers can refill
// the first half for tile t + 1 while the second half of the products runs.
// The softmax is online with a lazy reference maximum per head: P = 2^(s - m)
// with m raised (and O, l rescaled) only when a tile holds a logit more than 8
// above it, so P stays below 2^8 in fp16 and the exact per-head maximum (a
// warp max-reduction over order-preserving integer keys) is needed only then.
// Values are dequantised with integer ops only (E2M1 magnitudes from a byte
// table, E4M3 scales shifted into fp16 fields); they carry an exact factor 2^-8
// that the softmax scale and the epilogue undo.
// Roles: warps 0-7 gather and dequantise; warp 8 owns TMEM and issues the MMAs;
// warps 9-12 stage Q, run the softmax and the epilogue. Every mbarrier wait is
// bounded.
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace csa2 {
namespace {

using namespace sm100;

constexpr int kD = kHeadDim;             // 512
constexpr int kHB = 64;                  // heads per CTA
constexpr int kT = 128;                  // entries per tile
constexpr int kAtom = 8192;              // 64 rows x 128 B (one K atom of Q)
constexpr int kVAtom = kT * 128;         // 128 entries x 64 dims of fp16
constexpr int kVHalf = 4 * kVAtom;       // 128 entries x 256 dims
constexpr int kPBytes = kT * 128;        // P^T: 128 entries x 64 heads of fp16
constexpr int kOnesBytes = 2 * 16 * 128; // constant A tile of the row-sum block
constexpr int kProducerWarps = 8;
constexpr int kMmaWarp = 8;
constexpr int kSoftmaxWarp0 = 9;
constexpr int kThreads = 13 * 32;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;            // S^T: 64 columns
constexpr uint32_t kColO = 128;          // O^T: 4 blocks of 64 columns
constexpr uint32_t kColL = 384;          // row sums: row 0 of one more block
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleSlack = 8.0f;    // log2 units: P <= 2^8 before a rescale

struct __align__(8) Bars {
  uint64_t q_full, s_full, p_full, p_free, o_full;
  uint64_t v_full[2], v_free[2];
};

struct alignas(16) Smem {
  Bars bar;
  uint32_t tmem_slot;
  int abort_flag;
  int rescale;                  // the current tile raises some head's reference maximum
  uint32_t valid[2][kT / 32];   // bit i of word w: entry 32 w + i of the tile is selected
  // read as float4: 16-byte aligned
  alignas(16) float hs[kHB];    // per-head logit scale (log2 domain, undoes the Q and V factors)
  alignas(16) float m_ref[kHB]; // per-head reference maximum (log2 domain)
  alignas(16) float alpha[kHB]; // per-head rescale factor of the current tile
  alignas(16) float wmax[4][kHB];  // per-warp tile maxima (slow path)
  alignas(16) float l[kHB];     // row sums for the epilogue
};

constexpr size_t kSmemBytes = 1024 + 8 * kAtom /*Q*/ + 2 * kVHalf /*V*/ + kPBytes /*P^T*/ +
                              kOnesBytes + sizeof(Smem);

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

// kind::f16, F16 x F16 -> F32; A and B K-major (0) or M/N-major (1).
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N, int a_mn, int b_mn) {
  return (1u << 4) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void mma_f16(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                        uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}

__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// barrier among the four softmax warps
__device__ __forceinline__ void softmax_bar() {
  asm volatile("bar.sync 2, 128;" ::: "memory");
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// order-preserving unsigned key of a float (0 is below every number)
__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float order_key_inv(uint32_t k) {
  if (k == 0u) return -INFINITY;
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
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
  const uint8_t* kv_packed;
  const uint8_t* kv_scale;
  const int32_t* topk;
  int Tq, Hq, N, K, split_len, nsplit, nhb;
  float softmax_scale;
  uint16_t* out;
  float* lse;
  float* ws_o;
  float2* ws_ml;
  int* err;
};

// Raw bytes of one producer item: the codes (32 B) and scales (64 B) of 64
// dims of one entry.
struct Raw {
  uint4 c[2];
  uint4 s[4];
};

__global__ void __launch_bounds__(kThreads, 1) sparse_attn_tc_kernel(const AttnParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* qs = base;                              // [8 atoms][64 heads][128 B]
  uint8_t* vs = qs + 8 * kAtom;                    // [2 halves][4 atoms][128 entries][128 B]
  uint8_t* ps = vs + 2 * kVHalf;                   // P^T: [128 entries][64 heads] fp16
  uint8_t* ones = ps + kPBytes;                    // [2 atoms][16 rows][128 B]
  Smem& sm = *reinterpret_cast<Smem*>(ones + kOnesBytes);
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
    mbar_init(&sm.bar.s_full, 1);
    mbar_init(&sm.bar.p_full, 4);
    mbar_init(&sm.bar.p_free, 1);
    mbar_init(&sm.bar.o_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.bar.v_full[i], kProducerWarps);
      mbar_init(&sm.bar.v_free[i], 1);
    }
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) tmem_alloc(&sm.tmem_slot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_slot;

  if (warp < kProducerWarps) {
    const int tid = threadIdx.x;          // 0..255
    const int e = tid & (kT - 1);         // entry of the tile this thread gathers
    const int apair = tid >> 7;           // atoms 2 apair, 2 apair + 1 of each half
    const uint8_t* pk_b = p.kv_packed + (size_t)b * p.N * (kD / 2);
    const uint8_t* sc_b = p.kv_scale + (size_t)b * (p.N / kBlockEntries) * kD;
    const int32_t* topk_row = p.topk + row * p.K;

    auto load_index = [&](int t) -> int {
      const int kk = k_begin + t * kT + e;
      int id = (t < nt && kk < k_end) ? __ldg(topk_row + kk) : -1;
      if (id >= p.N || id < -1) {
        record_error(p.err, CSA2_ERR_DEVICE_INDEX);
        id = -1;
      }
      return id;
    };
    auto prefetch_rows = [&](int id) {
      if (id >= 0) {
        const uint8_t* pr = pk_b + (size_t)id * (kD / 2);
        const uint8_t* sr = sc_b + (size_t)(id / kBlockEntries) * kD;
        // threads 0-127 fetch the packed row, threads 128-255 the scale row
        if (apair == 0) {
          asm volatile("prefetch.global.L2::evict_last [%0];" ::"l"(pr));
          asm volatile("prefetch.global.L2::evict_last [%0];" ::"l"(pr + 128));
        } else {
#pragma unroll
          for (int j = 0; j < 4; ++j)
            asm volatile("prefetch.global.L2::evict_last [%0];" ::"l"(sr + 128 * j));
        }
      }
    };
    // item i (0, 1) of half h: atom 4 h + 2 apair + i of entry e
    auto load_raw = [&](int id, int h, Raw (&r)[2]) {
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int a = 4 * h + 2 * apair + i;
        if (id >= 0) {
          const uint4* pc = reinterpret_cast<const uint4*>(pk_b + (size_t)id * (kD / 2) + a * 32);
          const uint4* psc =
              reinterpret_cast<const uint4*>(sc_b + (size_t)(id / kBlockEntries) * kD + a * 64);
          r[i].c[0] = __ldg(pc);
          r[i].c[1] = __ldg(pc + 1);
#pragma unroll
          for (int j = 0; j < 4; ++j) r[i].s[j] = __ldg(psc + j);
        } else {
          r[i].c[0] = r[i].c[1] = make_uint4(0, 0, 0, 0);
#pragma unroll
          for (int j = 0; j < 4; ++j) r[i].s[j] = make_uint4(0, 0, 0, 0);
        }
      }
    };

    // the constant A tile of the row-sum block: ones in row 0 (element 0 of
    // every 16-entry row of atom 0), zeros elsewhere
    for (int i = tid; i < kOnesBytes / 16; i += 256) {
      const int r = i >> 3, c = i & 7;                    // atom-major rows of 8 chunks
      uint4 v = make_uint4(0, 0, 0, 0);
      if (r < 16 && c == (r & 7)) v.x = 0x3C00u;          // fp16 1.0 at element 0 of row r
      *reinterpret_cast<uint4*>(ones + i * 16) = v;
    }

    int id_cur = load_index(0);
    int id_next = load_index(1);
    prefetch_rows(id_cur);
    prefetch_rows(id_next);
    Raw raw[2];
    load_raw(id_cur, 0, raw);
    int id_after = -1;   // index of tile t + 2
    bool go = true;
    for (int t = 0; go && t < nt; ++t) {
      for (int h = 0; h < 2; ++h) {
        if (h == 0 && apair == 0) {
          const uint32_t vb = __ballot_sync(0xffffffffu, id_cur >= 0);
          if (lane == 0) sm.valid[t & 1][warp] = vb;
        }
        if (!mbar_wait_warp(&sm.bar.v_free[h], (t & 1) ^ 1, abort_flag)) { go = false; break; }
        uint8_t* half = vs + h * kVHalf;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int j = 2 * apair + i;              // atom within the half
          uint8_t* dst = half + j * kVAtom;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint4 cw = raw[i].c[c >> 2];
            const uint32_t codes = (c & 3) == 0 ? cw.x : (c & 3) == 1 ? cw.y : (c & 3) == 2 ? cw.z : cw.w;
            const uint4 sw = raw[i].s[c >> 1];
            const uint32_t s_lo = (c & 1) ? sw.z : sw.x;
            const uint32_t s_hi = (c & 1) ? sw.w : sw.y;
            *reinterpret_cast<uint4*>(dst + swz(e, c)) = dq8(codes, s_lo, s_hi);
          }
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.bar.v_full[h]);
        // gather ahead: the other half of this tile, or the first half of the next
        if (h == 0) {
          load_raw(id_cur, 1, raw);
          id_after = load_index(t + 2);
        } else {
          prefetch_rows(id_after);
          id_cur = id_next;
          id_next = id_after;
          load_raw(id_cur, 0, raw);
        }
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t id_s = idesc_f16(128, kHB, 0, 0);   // S^T: A = V (K-major), B = Q (K-major)
      const uint32_t id_o = idesc_f16(128, kHB, 1, 1);   // O^T: A = V^T, B = P^T (both MN-major)
      const uint64_t qd = desc_sw128(smem_u32(qs), 16, 1024);
      const uint64_t vk = desc_sw128(smem_u32(vs), 16, 1024);          // V as K-major A
      const uint64_t vm = desc_sw128(smem_u32(vs), kVAtom, 1024);      // V^T as MN-major A
      const uint64_t pd = desc_sw128(smem_u32(ps), kPBytes, 1024);     // P^T as MN-major B
      const uint64_t od = desc_sw128(smem_u32(ones), 2048, 1024);      // ones as MN-major A
      bool ok = mbar_wait(&sm.bar.q_full, 0, abort_flag);
      for (int t = 0; ok && t < nt; ++t) {
        const uint32_t ph = t & 1;
        for (int h = 0; h < 2; ++h) {
          if (!mbar_wait(&sm.bar.v_full[h], ph, abort_flag)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_f16(tmem + kColS, vk + (uint64_t)((h * kVHalf + j * kVAtom + kk * 32) >> 4),
                      qd + (uint64_t)(((4 * h + j) * kAtom + kk * 32) >> 4), id_s,
                      (h > 0 || j > 0 || kk > 0) ? 1u : 0u);
        }
        if (!ok) break;
        mma_commit(&sm.bar.s_full);
        if (!mbar_wait(&sm.bar.p_full, ph, abort_flag)) { ok = false; break; }
        tc_fence_after();
        for (int mb = 0; mb < 4; ++mb) {
          const int vo = (mb >> 1) * kVHalf + (mb & 1) * 2 * kVAtom;
#pragma unroll
          for (int ks = 0; ks < kT / 16; ++ks)
            mma_f16(tmem + kColO + 64u * mb, vm + (uint64_t)((vo + ks * 2048) >> 4),
                    pd + (uint64_t)((ks * 2048) >> 4), id_o, (t > 0 || ks > 0) ? 1u : 0u);
          if (mb == 1) mma_commit(&sm.bar.v_free[0]);
        }
#pragma unroll
        for (int ks = 0; ks < kT / 16; ++ks)
          mma_f16(tmem + kColL, od, pd + (uint64_t)((ks * 2048) >> 4), id_o,
                  (t > 0 || ks > 0) ? 1u : 0u);
        mma_commit(&sm.bar.v_free[1]);
        mma_commit(&sm.bar.p_free);
      }
      mma_commit(&sm.bar.o_full);
      // nothing may be in flight when TMEM is released
      mbar_wait(&sm.bar.o_full, 0, abort_flag);
    }
  } else {
    // ------------------------------------------------------------ Q, softmax, epilogue
    const int sw = warp - kSoftmaxWarp0;             // 0..3
    const int quad = warp & 3;                       // TMEM lanes 32 quad .. 32 quad + 31
    const int e = quad * 32 + lane;                  // entry (S^T row) / dim (O^T row) of this thread
    const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
    // ---- Q: warp sw stages heads 16 sw .. 16 sw + 15, scaled per head by a power
    // of two so that its bf16 values keep every bit in fp16
    for (int j = 0; j < 16; ++j) {
      const int hh = sw * 16 + j;
      uint4 q0 = make_uint4(0, 0, 0, 0), q1 = make_uint4(0, 0, 0, 0);
      if (hh < nh) {
        const uint4* src =
            reinterpret_cast<const uint4*>(p.q + ((row * p.Hq) + h0 + hh) * kD + lane * 16);
        q0 = __ldg(src);
        q1 = __ldg(src + 1);
      }
      const uint32_t w[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
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
      if (lane == 0) {
        sm.hs[hh] = hh < nh ? p.softmax_scale * kLog2e * down * 256.0f : 0.0f;
        sm.m_ref[hh] = -INFINITY;
      }
    }
    fence_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.bar.q_full);
    softmax_bar();   // hs and m_ref visible to all four warps

    // Every softmax warp passes every named barrier the same number of times,
    // also after a wait gave up (then it skips the work, not the barriers).
    bool ok = true;
    for (int t = 0; t < nt; ++t) {
      const uint32_t ph = t & 1;
      // the valid bits of tile t were written before its first half was published
      if (ok)
        ok = mbar_wait_warp(&sm.bar.v_full[0], ph, abort_flag) &&
             mbar_wait_warp(&sm.bar.s_full, ph, abort_flag);
      tc_fence_after();
      const bool valid = (sm.valid[t & 1][e >> 5] >> (e & 31)) & 1u;
      float x[64];
      tmem_ld_64(tmem + lane_addr + kColS, x);
      // logits relative to the reference maxima; does any exceed the slack?
      bool over = false;
#pragma unroll
      for (int h = 0; h < kHB; h += 4) {
        const float4 hs4 = *reinterpret_cast<const float4*>(&sm.hs[h]);
        const float4 m4 = *reinterpret_cast<const float4*>(&sm.m_ref[h]);
        x[h] = x[h] * hs4.x - m4.x;
        x[h + 1] = x[h + 1] * hs4.y - m4.y;
        x[h + 2] = x[h + 2] * hs4.z - m4.z;
        x[h + 3] = x[h + 3] * hs4.w - m4.w;
        over |= fmaxf(fmaxf(x[h], x[h + 1]), fmaxf(x[h + 2], x[h + 3])) > kRescaleSlack;
      }
      over = over && valid;
      if (lane == 0 && sw == 0) sm.rescale = 0;
      softmax_bar();
      if (__any_sync(0xffffffffu, over) && lane == 0) sm.rescale = 1;
      // P(t-1) V(t-1) must be complete before O is rescaled or P^T is rewritten
      if (t > 0 && ok) {
        ok = mbar_wait_warp(&sm.bar.p_free, (t - 1) & 1, abort_flag);
        tc_fence_after();
      }
      softmax_bar();
      if (sm.rescale) {
        // exact maximum of this tile's logits per head (warp max over
        // order-preserving keys, then over the four warps)
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
          float sv[32];
          tmem_ld_32(tmem + lane_addr + kColS + 32u * c, sv);
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int h = 32 * c + j;
            const float lg = sv[j] * sm.hs[h];         // logit in the log2 domain
            const uint32_t wk = __reduce_max_sync(0xffffffffu, valid ? order_key(lg) : 0u);
            if (lane == 0) sm.wmax[sw][h] = order_key_inv(wk);
          }
        }
        softmax_bar();
        if (threadIdx.x - kSoftmaxWarp0 * 32 < kHB) {
          const int h = threadIdx.x - kSoftmaxWarp0 * 32;
          const float m_old = sm.m_ref[h];
          const float tmax = fmaxf(fmaxf(sm.wmax[0][h], sm.wmax[1][h]),
                                   fmaxf(sm.wmax[2][h], sm.wmax[3][h]));
          float a = 1.0f;
          if (tmax > m_old + kRescaleSlack) {
            a = m_old == -INFINITY ? 0.0f : exp2f(m_old - tmax);
            sm.m_ref[h] = tmax;
          }
          sm.alpha[h] = a;
        }
        softmax_bar();
        // rescale O^T and the row sums (columns = heads) when a maximum moved
        if (t > 0) {
#pragma unroll 1
          for (int c = 0; c < 10; ++c) {               // 5 blocks x 2 halves of the heads
            float o[32];
            tmem_ld_32(tmem + lane_addr + kColO + 32u * c, o);
            const float* a = &sm.alpha[(c & 1) * 32];
#pragma unroll
            for (int h = 0; h < 32; ++h) o[h] *= a[h];
            tmem_st_32(tmem + lane_addr + kColO + 32u * c, o);
          }
        }
        // logits relative to the new reference maxima (reloaded: x was not kept
        // live across the rescale)
        tmem_ld_64(tmem + lane_addr + kColS, x);
#pragma unroll
        for (int h = 0; h < kHB; ++h) x[h] = x[h] * sm.hs[h] - sm.m_ref[h];
      }
      // P^T row of this entry: 2^x in fp16 (x <= 8), zero for an unselected entry
      uint8_t* prow = ps;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        uint32_t pk[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int h = 8 * c + 2 * u;
          const float p0 = valid ? exp2f(x[h]) : 0.0f;
          const float p1 = valid ? exp2f(x[h + 1]) : 0.0f;
          pk[u] = pack_half2(p0, p1);
        }
        *reinterpret_cast<uint4*>(prow + swz(e, c)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
      fence_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0 && ok) mbar_arrive(&sm.bar.p_full);
    }
    // ---- epilogue: l from row 0 of the row-sum block, O^T rows are dims
    ok = mbar_wait_warp(&sm.bar.o_full, 0, abort_flag) && ok;
    {
      tc_fence_after();
      if (quad == 0) {
        float lv[64];
        tmem_ld_64(tmem + lane_addr + kColL, lv);
        if (lane == 0) {
#pragma unroll
          for (int h = 0; h < kHB; ++h) sm.l[h] = lv[h];
        }
      }
      softmax_bar();
      // x 2^8 undoes the 2^-8 carried by the dequantised values
      if (threadIdx.x - kSoftmaxWarp0 * 32 < kHB) {
        const int h = threadIdx.x - kSoftmaxWarp0 * 32;
        const float lh = sm.l[h];
        sm.alpha[h] = lh > 0.0f ? (p.nsplit == 1 ? 256.0f / lh : 256.0f) : 0.0f;
      }
      softmax_bar();
      // stage the [64 heads][512 dims] result in the (now idle) V tile, then copy
      // it out with 16-byte stores
      const size_t slot = (row * p.nhb + hb) * p.nsplit + split;
      if (p.nsplit == 1) {
        uint16_t* stage = reinterpret_cast<uint16_t*>(vs);      // [64][512] bf16
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {                 // 4 dim blocks x 2 halves of the heads
          float o[32];
          tmem_ld_32(tmem + lane_addr + kColO + 32u * c, o);
          const int d = (c >> 1) * 128 + e, hbase = (c & 1) * 32;
#pragma unroll
          for (int h = 0; h < 32; ++h)
            stage[(hbase + h) * kD + d] =
                __bfloat16_as_ushort(__float2bfloat16_rn(o[h] * sm.alpha[hbase + h]));
        }
        softmax_bar();
        const int tid = threadIdx.x - kSoftmaxWarp0 * 32;   // 0..127
        for (int i = tid; ok && i < nh * kD / 8; i += 128) {
          const int h = i / (kD / 8), c = i % (kD / 8);
          *reinterpret_cast<uint4*>(p.out + ((row * p.Hq) + h0 + h) * kD + c * 8) =
              *reinterpret_cast<const uint4*>(stage + h * kD + c * 8);
        }
        if (ok && tid < nh && p.lse) {
          const float lh = sm.l[tid];
          p.lse[row * p.Hq + h0 + tid] = lh > 0.0f ? (sm.m_ref[tid] + log2f(lh)) * kLn2 : -INFINITY;
        }
      } else {
        float* stage = reinterpret_cast<float*>(vs);            // [64][512] fp32
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
          float o[32];
          tmem_ld_32(tmem + lane_addr + kColO + 32u * c, o);
          const int d = (c >> 1) * 128 + e, hbase = (c & 1) * 32;
#pragma unroll
          for (int h = 0; h < 32; ++h) stage[(hbase + h) * kD + d] = o[h] * sm.alpha[hbase + h];
        }
        softmax_bar();
        const int tid = threadIdx.x - kSoftmaxWarp0 * 32;
        for (int i = tid; ok && i < nh * kD / 4; i += 128) {
          const int h = i / (kD / 4), c = i % (kD / 4);
          *reinterpret_cast<float4*>(p.ws_o + (slot * kHB + h) * kD + c * 4) =
              *reinterpret_cast<const float4*>(stage + h * kD + c * 4);
        }
        if (ok && tid < nh) {
          const float lh = sm.l[tid];
          p.ws_ml[slot * kHB + tid] = make_float2(lh > 0.0f ? sm.m_ref[tid] : -INFINITY, lh);
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
}

}  // namespace

int sparse_attn_tc_tile() { return kT; }

cudaError_t launch_sparse_attn_tc(const uint16_t* q, const uint8_t* kv_packed,
                                  const uint8_t* kv_scale, const int32_t* topk_idx, int rows,
                                  int Tq, int Hq, int N, int K, float softmax_scale, int nhb,
                                  int nsplit, int split_len, uint16_t* out, float* lse,
                                  float* ws_o, float2* ws_ml, int* err, cudaStream_t stream) {
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
  cudaError_t e = cudaFuncSetAttribute(sparse_attn_tc_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid(rows, nhb, nsplit);
  sparse_attn_tc_kernel<<<grid, kThreads, kSmemBytes, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace csa2
