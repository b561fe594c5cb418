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
// One CTA = (query row, block of 64 heads, split of at most 512 selected
// entries = two tiles of 256). A tcgen05.mma costs about the same issue time
// for any N up to 256, so both products use N = 256:
//   S(t) = Q V(t)^T   M=64 heads, N=256 entries, K=512: 32 MMAs per tile,
//                     accumulators in TMEM lanes 16-31 of each quadrant
//                     (columns 256 t .. 256 t + 255);
//   O   += P(t) V(t)  M=64 heads, N=256 dims (two halves), K=256 entries:
//                     32 MMAs per tile, accumulator in TMEM lanes 0-15, all 512
//                     columns.
// V is dequantised (with integer ops; values carry an exact factor 2^-8 that the
// softmax scale and the epilogue undo) twice into a ring of 32 KB stages: first as
// 64-dim K atoms of all 256 entries (K-major B operand of S), then as 32-entry
// slices of all 512 dims (MN-major B operand of P V). The softmax is exact in
// two passes over the CTA's (at most 512) scores, so O is never rescaled.
// Roles: warps 0-7 gather/dequantise (and stage Q, each head scaled by a power
// of two so its bf16 values keep their bits in fp16), warp 8 owns TMEM and
// issues the MMAs, warps 9-12 run the softmax (S rows live in lanes 16-31) and
// the epilogue (O rows in lanes 0-15). Every mbarrier wait is bounded.
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace csa2 {
namespace {

using namespace sm100;

constexpr int kD = kHeadDim;             // 512
constexpr int kHB = 64;                  // heads per CTA
constexpr int kT = 256;                  // entries per tile
constexpr int kMaxTiles = 2;             // tiles per CTA
constexpr int kStages = 2;               // fp16 ring depth
constexpr int kRawBytes = 6 * 4096;      // raw (packed + scale) bytes of one stage: 6 x 16 B per thread
constexpr int kStageBytes = 32768;
constexpr int kAtom = 8192;              // 64 rows x 128 B (one K atom of Q or P)
constexpr int kProducerWarps = 8;
constexpr int kMmaWarp = 8;
constexpr int kThreads = 13 * 32;
constexpr uint32_t kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

struct __align__(8) Bars {
  uint64_t q_full, s_full, p_full, p_empty, o_full;
  uint64_t full[kStages], empty[kStages];
};

struct Smem {
  Bars bar;
  uint32_t tmem_slot;
  int abort_flag;
  int idx[kMaxTiles][kT];
  uint32_t valid[kMaxTiles][kT / 32];   // bit i of word w: entry 32 w + i is selected
  float head_scale[kHB];
};

constexpr size_t kSmemBytes = 1024 + 8 * kAtom /*Q*/ + kStages * kStageBytes + 4 * kAtom /*P*/ +
                              2 * kRawBytes /*raw ring*/ + sizeof(Smem);

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

__device__ __forceinline__ void producer_bar() {
  asm volatile("bar.sync 1, 256;" ::: "memory");
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
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

__global__ void __launch_bounds__(kThreads, 1) sparse_attn_tc_kernel(const AttnParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* qs = base;                              // [8 atoms][64 heads][128 B]
  uint8_t* ring = qs + 8 * kAtom;                  // kStages x 32 KB
  uint8_t* ps = ring + kStages * kStageBytes;      // [4 atoms][64 heads][128 B]
  uint8_t* rawbuf = ps + 4 * kAtom;                // 2 x [6 fields][256 threads][16 B]
  Smem& sm = *reinterpret_cast<Smem*>(rawbuf + 2 * kRawBytes);
  volatile int* abort_flag = &sm.abort_flag;

  const size_t row = blockIdx.x;
  const int hb = blockIdx.y, split = blockIdx.z;
  const int b = (int)(row / p.Tq);
  const int h0 = hb * kHB;
  const int nh = min(kHB, p.Hq - h0);
  const int k_begin = split * p.split_len;
  const int k_end = min(p.K, k_begin + p.split_len);
  const int nt = (k_end - k_begin + kT - 1) / kT;   // 1 or 2
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(&sm.bar.q_full, kProducerWarps);
    mbar_init(&sm.bar.s_full, 1);
    mbar_init(&sm.bar.p_full, 4);
    mbar_init(&sm.bar.p_empty, 1);
    mbar_init(&sm.bar.o_full, 1);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&sm.bar.full[i], kProducerWarps);
      mbar_init(&sm.bar.empty[i], 1);
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
    // ------------------------------------------------------------ Q and indices
    {
      uint4 qraw[16];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int hh = warp * 8 + j;
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
      const int tid = threadIdx.x;   // 0..255: one entry of each tile
      const uint8_t* pk_row0 = p.kv_packed + (size_t)b * p.N * (kD / 2);
      const uint8_t* sc_row0 = p.kv_scale + (size_t)b * (p.N / kBlockEntries) * kD;
#pragma unroll
      for (int t = 0; t < kMaxTiles; ++t) {
        const int kk = k_begin + t * kT + tid;
        int id = (t < nt && kk < k_end) ? __ldg(p.topk + row * p.K + kk) : -1;
        if (id >= p.N || id < -1) {
          record_error(p.err, CSA2_ERR_DEVICE_INDEX);
          id = -1;
        }
        sm.idx[t][tid] = id;
        const uint32_t vb = __ballot_sync(0xffffffffu, id >= 0);
        if (lane == 0) sm.valid[t][tid >> 5] = vb;
        if (id >= 0) {
          // the stages read every row in 32- to 64-byte pieces: bring the whole
          // packed row (256 B) and scale row (512 B) into L2 once, now
          const uint8_t* pr = pk_row0 + (size_t)id * (kD / 2);
          const uint8_t* sr = sc_row0 + (size_t)(id / kBlockEntries) * kD;
          asm volatile("prefetch.global.L2::evict_last [%0];" ::"l"(pr));
          asm volatile("prefetch.global.L2::evict_last [%0];" ::"l"(pr + 128));
#pragma unroll
          for (int j = 0; j < 4; ++j) asm volatile("prefetch.global.L2::evict_last [%0];" ::"l"(sr + 128 * j));
        }
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int hh = warp * 8 + j;
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
        int e = 0;
        if (amax > 0.0f && isfinite(amax)) {
          const int ex = (int)((__float_as_uint(amax) >> 23) & 0xffu) - 126;
          e = min(100, max(-100, 15 - ex));
        }
        const float up = __uint_as_float((uint32_t)(127 + e) << 23);
        uint32_t pk[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) pk[i] = pack_half2(vals[2 * i] * up, vals[2 * i + 1] * up);
        const int atom = lane >> 2, c0 = (lane & 3) * 2;
        uint8_t* dst = qs + atom * kAtom;
        *reinterpret_cast<uint4*>(dst + swz(hh, c0)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        *reinterpret_cast<uint4*>(dst + swz(hh, c0 + 1)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        const float down = __uint_as_float((uint32_t)(127 - e) << 23);
        // x 2^8: the dequantised keys/values carry a factor 2^-8
        if (lane == 0) sm.head_scale[hh] = hh < nh ? p.softmax_scale * kLog2e * down * 256.0f : 0.0f;
      }
      fence_async_smem();
      producer_bar();                         // indices visible to every producer warp
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.bar.q_full);
    }

    // ------------------------------------------------------------ V stages
    // Stage k < 8 nt: K atom a = k % 8 of tile k / 8; four lanes per entry, each
    //   16 channels, four passes of 64 entries (a warp instruction touches 8 rows).
    // Stage k >= 8 nt: 32-entry slice of a tile; eight lanes per entry, one
    //   64-channel atom each (a warp instruction reads 4 whole rows).
    // Each thread keeps the loads of the next two stages in flight (6 x 16 B).
    const uint8_t* pk_b = p.kv_packed + (size_t)b * p.N * (kD / 2);
    const uint8_t* sc_b = p.kv_scale + (size_t)b * (p.N / kBlockEntries) * kD;
    const int nstages = 16 * nt;
    const int tid = threadIdx.x;
    // Raw bytes of stage k go to raw slot k & 1 with cp.async (completion tracked
    // per thread by commit groups, so the gather of stage k + 2 stays in flight
    // while stage k is dequantised). Field f of thread tid is at f * 4096 + tid * 16.
    auto cp16 = [](uint8_t* dst, const uint8_t* src) {
      asm volatile("cp.async.cg.shared.global.L2::256B [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src)
                   : "memory");
    };
    auto cp8 = [](uint8_t* dst, const uint8_t* src) {
      asm volatile("cp.async.ca.shared.global.L2::256B [%0], [%1], 8;" ::"r"(smem_u32(dst)), "l"(src)
                   : "memory");
    };
    auto issue = [&](int k) {
      if (k < nstages) {
        uint8_t* raw = rawbuf + (k & 1) * kRawBytes + tid * 16;
        if (k < 8 * nt) {
          const int t = k >> 3, atom = k & 7, sub = tid & 3;
#pragma unroll
          for (int ps = 0; ps < 4; ++ps) {
            const int id = sm.idx[t][ps * 64 + (tid >> 2)];
            if (id >= 0) {
              cp16(raw + ps * 4096, sc_b + (size_t)(id / kBlockEntries) * kD + atom * 64 + sub * 16);
              cp8(raw + (4 + (ps >> 1)) * 4096 + (ps & 1) * 8,
                  pk_b + (size_t)id * (kD / 2) + atom * 32 + sub * 8);
            }
          }
        } else {
          const int kk = k - 8 * nt;
          const int id = sm.idx[kk >> 3][(kk & 7) * 32 + (tid >> 3)];
          const int atom = tid & 7;
          if (id >= 0) {
            const uint8_t* pr = pk_b + (size_t)id * (kD / 2) + atom * 32;
            const uint8_t* sr = sc_b + (size_t)(id / kBlockEntries) * kD + atom * 64;
            cp16(raw, pr);
            cp16(raw + 4096, pr + 16);
#pragma unroll
            for (int j = 0; j < 4; ++j) cp16(raw + (2 + j) * 4096, sr + 16 * j);
          }
        }
      }
      asm volatile("cp.async.commit_group;" ::: "memory");
    };
    auto fetch = [&](int k, uint4 (&cur)[6]) {
      asm volatile("cp.async.wait_group 1;" ::: "memory");   // stage k landed (k + 1 may not have)
      const uint8_t* raw = rawbuf + (k & 1) * kRawBytes + tid * 16;
#pragma unroll
      for (int f = 0; f < 6; ++f) cur[f] = *reinterpret_cast<const uint4*>(raw + f * 4096);
    };
    // 8 E2M1 codes (one 32-bit word) times their 8 E4M3 scales (two words) -> one
    // 16-byte chunk of fp16 values, times 2^-8. Integer ops only (byte permutes,
    // shifts, one logic op): the conversion pipe stays free for the softmax.
    //  - E2M1 magnitude m -> high byte of fp16(m) from an 8-entry byte table
    //    (0, 0.5, 1, 1.5, 2, 3, 4, 6 -> 00 38 3C 3E 40 42 44 46), sign spliced in;
    //  - a non-negative E4M3 byte shifted left by 7 is the fp16 of its value * 2^-8
    //    (exponent bias 7 -> 15, mantissa 3 -> 10 bits; subnormals line up too);
    //  - the fp16 product is exact (<= 6 significant bits, >= 2^-18).
    auto dq8 = [](uint32_t codes, uint32_t s_lo, uint32_t s_hi) -> uint4 {
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
    };
    auto publish = [&](int st) {
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.bar.full[st]);
    };
    // Each stage: wait for its raw bytes and its fp16 slot, dequantise, start
    // the gather of stage k + 2 into the raw slot just consumed, store, publish.
    auto stage_s = [&](int k) -> bool {
      const int st = k % kStages;
      uint4 cur[6];
      fetch(k, cur);
      if (!mbar_wait_warp(&sm.bar.empty[st], ((k / kStages) & 1) ^ 1, abort_flag)) return false;
      const int t = k >> 3, sub = tid & 3;
      uint4 v[8];
#pragma unroll
      for (int ps = 0; ps < 4; ++ps) {
        const uint32_t keep = sm.idx[t][ps * 64 + (tid >> 2)] >= 0 ? 0xffffffffu : 0u;
        const uint4 s = cur[ps];
        const uint32_t c0 = (ps & 1) ? cur[4 + (ps >> 1)].z : cur[4 + (ps >> 1)].x;
        const uint32_t c1 = (ps & 1) ? cur[4 + (ps >> 1)].w : cur[4 + (ps >> 1)].y;
        const uint4 d0 = dq8(c0, s.x, s.y), d1 = dq8(c1, s.z, s.w);   // branch-free
        v[2 * ps] = make_uint4(d0.x & keep, d0.y & keep, d0.z & keep, d0.w & keep);
        v[2 * ps + 1] = make_uint4(d1.x & keep, d1.y & keep, d1.z & keep, d1.w & keep);
      }
      issue(k + 2);   // after the raw slot's values were consumed
      uint8_t* dst = ring + st * kStageBytes;
#pragma unroll
      for (int ps = 0; ps < 4; ++ps) {
        const int e = ps * 64 + (tid >> 2);
        *reinterpret_cast<uint4*>(dst + swz(e, 2 * sub)) = v[2 * ps];
        *reinterpret_cast<uint4*>(dst + swz(e, 2 * sub + 1)) = v[2 * ps + 1];
      }
      publish(st);
      return true;
    };
    auto stage_pv = [&](int k) -> bool {
      const int st = k % kStages;
      uint4 cur[6];
      fetch(k, cur);
      if (!mbar_wait_warp(&sm.bar.empty[st], ((k / kStages) & 1) ^ 1, abort_flag)) return false;
      const int kk = k - 8 * nt;
      const int e = tid >> 3, atom = tid & 7;
      const uint32_t keep = sm.idx[kk >> 3][(kk & 7) * 32 + e] >= 0 ? 0xffffffffu : 0u;
      uint4 v[8];
      const uint32_t cw[8] = {cur[0].x, cur[0].y, cur[0].z, cur[0].w,
                              cur[1].x, cur[1].y, cur[1].z, cur[1].w};
      const uint32_t sw[16] = {cur[2].x, cur[2].y, cur[2].z, cur[2].w, cur[3].x, cur[3].y,
                               cur[3].z, cur[3].w, cur[4].x, cur[4].y, cur[4].z, cur[4].w,
                               cur[5].x, cur[5].y, cur[5].z, cur[5].w};
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint4 d = dq8(cw[j], sw[2 * j], sw[2 * j + 1]);   // branch-free
        v[j] = make_uint4(d.x & keep, d.y & keep, d.z & keep, d.w & keep);
      }
      issue(k + 2);   // after the raw slot's values were consumed
      uint8_t* dst = ring + st * kStageBytes + atom * 4096;
#pragma unroll
      for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4*>(dst + swz(e, c)) = v[c];
      publish(st);
      return true;
    };
    issue(0);
    issue(1);
    bool go = true;
    for (int k = 0; go && k < 8 * nt; ++k) go = stage_s(k);
    for (int k = 8 * nt; go && k < nstages; ++k) go = stage_pv(k);
    asm volatile("cp.async.wait_group 0;" ::: "memory");   // nothing in flight at exit
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t id_s = idesc_f16(64, 256, 0);
      const uint32_t id_o = idesc_f16(64, 256, 1);
      const uint32_t qa = smem_u32(qs), pa = smem_u32(ps), ra = smem_u32(ring);
      bool ok = mbar_wait(&sm.bar.q_full, 0, abort_flag);
      int k = 0;
      for (int t = 0; ok && t < nt; ++t) {
        const uint32_t d = tmem + (16u << 16) + 256u * t;   // S(t): lanes 16-31
        for (int a = 0; ok && a < 8; ++a, ++k) {
          const int st = k % kStages;
          if (!mbar_wait(&sm.bar.full[st], (k / kStages) & 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = ra + st * kStageBytes;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_f16(d, desc_sw128(qa + a * kAtom + kk * 32, 16, 1024),
                    desc_sw128(sa + kk * 32, 16, 1024), id_s, (a > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&sm.bar.empty[st]);
        }
      }
      mma_commit(&sm.bar.s_full);
      for (int t = 0; ok && t < nt; ++t) {
        if (!mbar_wait(&sm.bar.p_full, t & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        for (int j = 0; ok && j < kT / 32; ++j, ++k) {
          const int st = k % kStages;
          if (!mbar_wait(&sm.bar.full[st], (k / kStages) & 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = ra + st * kStageBytes;
#pragma unroll
          for (int ks = 0; ks < 2; ++ks) {
            const uint64_t ad = desc_sw128(pa + (j >> 1) * kAtom + (j & 1) * 64 + ks * 32, 16, 1024);
#pragma unroll
            for (int n = 0; n < 2; ++n)
              mma_f16(tmem + 256u * n, ad, desc_sw128(sa + ks * 2048 + n * 4 * 4096, 4096, 1024),
                      id_o, (t > 0 || j > 0 || ks > 0) ? 1u : 0u);
          }
          mma_commit(&sm.bar.empty[st]);
        }
        mma_commit(&sm.bar.p_empty);
      }
      mma_commit(&sm.bar.o_full);
      // nothing may be in flight when TMEM is released
      mbar_wait(&sm.bar.o_full, 0, abort_flag);
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int quad = warp & 3;
    const bool s_owner = lane >= 16;                 // S rows live in lanes 16-31
    const int h = quad * 16 + (lane & 15);           // head of this lane's S (or O) row
    const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
    bool ok = mbar_wait_warp(&sm.bar.q_full, 0, abort_flag);
    const float hs = sm.head_scale[h];
    ok = mbar_wait_warp(&sm.bar.s_full, 0, abort_flag) && ok;
    if (ok) tc_fence_after();
    // pass 1: exact row maximum over the CTA's entries
    float m = -INFINITY;
    if (ok) {
      for (int t = 0; t < nt; ++t) {
#pragma unroll 1
        for (int c0 = 0; c0 < kT; c0 += 64) {
          float s[64];
          tmem_ld_64(tmem + lane_addr + 256u * t + c0, s);
          const uint32_t v0 = sm.valid[t][c0 / 32], v1 = sm.valid[t][c0 / 32 + 1];
#pragma unroll
          for (int c = 0; c < 64; ++c)
            m = fmaxf(m, (((c < 32 ? v0 : v1) >> (c & 31)) & 1u) ? s[c] * hs : -INFINITY);
        }
      }
    }
    // pass 2: P = 2^(s - m) in fp16 as the A operand of P V, and the row sum
    float l = 0.0f;
    for (int t = 0; ok && t < nt; ++t) {
      if (t > 0 && !mbar_wait_warp(&sm.bar.p_empty, (t - 1) & 1, abort_flag)) { ok = false; break; }
#pragma unroll 1
      for (int c0 = 0; c0 < kT; c0 += 64) {
        float s[64];
        tmem_ld_64(tmem + lane_addr + 256u * t + c0, s);
        const uint32_t vw0 = sm.valid[t][c0 / 32], vw1 = sm.valid[t][c0 / 32 + 1];
        uint8_t* dst = ps + (c0 / 64) * kAtom;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint32_t pk[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int i0 = 8 * c + 2 * u;
            const uint32_t vw = i0 < 32 ? vw0 : vw1;
            const bool v0 = (vw >> (i0 & 31)) & 1u, v1 = (vw >> ((i0 + 1) & 31)) & 1u;
            const float p0 = (v0 && m != -INFINITY) ? exp2f(s[i0] * hs - m) : 0.0f;
            const float p1 = (v1 && m != -INFINITY) ? exp2f(s[i0 + 1] * hs - m) : 0.0f;
            l += p0 + p1;
            pk[u] = pack_half2(p0, p1);
          }
          if (s_owner)
            *reinterpret_cast<uint4*>(dst + swz(h, c)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
      }
      fence_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.bar.p_full);
    }
    // epilogue: O rows live in lanes 0-15; fetch m and l from the S lane (+16)
    const float m_o = __shfl_down_sync(0xffffffffu, m, 16);
    const float l_o = __shfl_down_sync(0xffffffffu, l, 16);
    ok = mbar_wait_warp(&sm.bar.o_full, 0, abort_flag) && ok;
    if (ok) {
      tc_fence_after();
      const bool o_owner = lane < 16 && h < nh;
      const size_t slot = (row * p.nhb + hb) * p.nsplit + split;
      // x 2^8 undoes the 2^-8 carried by the dequantised values
      const float inv = l_o > 0.0f ? 256.0f / l_o : 0.0f;
#pragma unroll 1
      for (int c0 = 0; c0 < kD; c0 += 64) {
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
              __nv_bfloat162 bb = __floats2bfloat162_rn(o[8 * c + 2 * u] * inv, o[8 * c + 2 * u + 1] * inv);
              w[u] = *reinterpret_cast<uint32_t*>(&bb);
            }
            dst[c] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        } else {
          float4* dst = reinterpret_cast<float4*>(p.ws_o + (slot * kHB + h) * kD + c0);
#pragma unroll
          for (int c = 0; c < 16; ++c)
            dst[c] = make_float4(256.0f * o[4 * c], 256.0f * o[4 * c + 1], 256.0f * o[4 * c + 2],
                                 256.0f * o[4 * c + 3]);
        }
      }
      if (lane < 16 && h < nh) {
        if (p.nsplit == 1) {
          if (p.lse) p.lse[row * p.Hq + h0 + h] = l_o > 0.0f ? (m_o + log2f(l_o)) * kLn2 : -INFINITY;
        } else {
          p.ws_ml[slot * kHB + h] = make_float2(l_o > 0.0f ? m_o : -INFINITY, l_o);
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

int sparse_attn_tc_max_split_len() { return kMaxTiles * kT; }

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
  if (split_len > kMaxTiles * kT) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(sparse_attn_tc_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid(rows, nhb, nsplit);
  sparse_attn_tc_kernel<<<grid, kThreads, kSmemBytes, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace csa2
