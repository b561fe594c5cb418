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
// V is dequantised twice into a ring of 32 KB shared-memory stages: first as
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
constexpr int kStages = 3;               // shared-memory ring depth
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
  float head_scale[kHB];
};

constexpr size_t kSmemBytes = 1024 + 8 * kAtom /*Q*/ + kStages * kStageBytes + 4 * kAtom /*P*/ +
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

__device__ __forceinline__ void ldg_nc_v4(const void* p, uint4& v) {
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
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
  Smem& sm = *reinterpret_cast<Smem*>(ps + 4 * kAtom);
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
#pragma unroll
      for (int t = 0; t < kMaxTiles; ++t) {
        const int kk = k_begin + t * kT + tid;
        int id = (t < nt && kk < k_end) ? __ldg(p.topk + row * p.K + kk) : -1;
        if (id >= p.N || id < -1) {
          record_error(p.err, CSA2_ERR_DEVICE_INDEX);
          id = -1;
        }
        sm.idx[t][tid] = id;
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
        if (lane == 0) sm.head_scale[hh] = hh < nh ? p.softmax_scale * kLog2e * down : 0.0f;
      }
      fence_async_smem();
      producer_bar();                         // indices visible to every producer warp
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.bar.q_full);
    }

    // ------------------------------------------------------------ V stages
    // Stage k < 8 nt: K atom (k % 8) of tile k / 8, thread = entry.
    // Stage k >= 8 nt: 32-entry slice of a tile, warp = 64-dim atom, lane = entry.
    // Each warp keeps the loads of the next two stages in flight.
    const uint8_t* pk_b = p.kv_packed + (size_t)b * p.N * (kD / 2);
    const uint8_t* sc_b = p.kv_scale + (size_t)b * (p.N / kBlockEntries) * kD;
    const int nstages = 16 * nt;
    auto stage_src = [&](int k, int& id, int& atom) {
      if (k < 8 * nt) {
        id = sm.idx[k >> 3][threadIdx.x];
        atom = k & 7;
      } else {
        const int kk = k - 8 * nt;
        id = sm.idx[kk >> 3][(kk & 7) * 32 + lane];
        atom = warp;
      }
    };
    auto issue = [&](int k, uint4 (&raw)[6]) {
      if (k >= nstages) return;
      int id, atom;
      stage_src(k, id, atom);
      if (id >= 0) {
        const uint8_t* pr = pk_b + (size_t)id * (kD / 2) + atom * 32;
        const uint8_t* sr = sc_b + (size_t)(id / kBlockEntries) * kD + atom * 64;
        // volatile: issued here, two stages before their use, not sunk to it
        ldg_nc_v4(pr, raw[0]);
        ldg_nc_v4(pr + 16, raw[1]);
        ldg_nc_v4(sr, raw[2]);
        ldg_nc_v4(sr + 16, raw[3]);
        ldg_nc_v4(sr + 32, raw[4]);
        ldg_nc_v4(sr + 48, raw[5]);
      }
    };
    // one stage: wait for its slot, dequantise the registers loaded two stages
    // ago, refill them with stage k + 2, store, publish
    auto run_stage = [&](int k, uint4 (&cur)[6]) -> bool {
      const int st = k % kStages;
      if (!mbar_wait_warp(&sm.bar.empty[st], ((k / kStages) & 1) ^ 1, abort_flag)) return false;
      int id, atom;
      stage_src(k, id, atom);
      uint4 v[8];
      if (id >= 0) {
        const uint32_t cw[8] = {cur[0].x, cur[0].y, cur[0].z, cur[0].w,
                                cur[1].x, cur[1].y, cur[1].z, cur[1].w};
        const uint32_t sw[16] = {cur[2].x, cur[2].y, cur[2].z, cur[2].w, cur[3].x, cur[3].y,
                                 cur[3].z, cur[3].w, cur[4].x, cur[4].y, cur[4].z, cur[4].w,
                                 cur[5].x, cur[5].y, cur[5].z, cur[5].w};
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          uint32_t h[4];
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const __half2 vv = e2m1x2_to_half2((uint8_t)(cw[j] >> (8 * t)));
            const __half2 ss = e4m3x2_to_half2((uint16_t)(sw[2 * j + (t >> 1)] >> (16 * (t & 1))));
            const __half2 r = __hmul2(vv, ss);
            h[t] = *reinterpret_cast<const uint32_t*>(&r);
          }
          v[j] = make_uint4(h[0], h[1], h[2], h[3]);
        }
      } else {
#pragma unroll
        for (int c = 0; c < 8; ++c) v[c] = make_uint4(0, 0, 0, 0);
      }
      issue(k + 2, cur);
      uint8_t* dst = ring + st * kStageBytes;
      if (k < 8 * nt) {
#pragma unroll
        for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4*>(dst + swz(threadIdx.x, c)) = v[c];
      } else {
#pragma unroll
        for (int c = 0; c < 8; ++c)
          *reinterpret_cast<uint4*>(dst + warp * 4096 + swz(lane, c)) = v[c];
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.bar.full[st]);
      return true;
    };
    // two statically addressed register sets (the stage count is even)
    uint4 ra[6], rb[6];
    issue(0, ra);
    issue(1, rb);
    for (int k = 0; k < nstages; k += 2) {
      if (!run_stage(k, ra)) break;
      if (!run_stage(k + 1, rb)) break;
    }
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
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (sm.idx[t][c0 + c] >= 0) m = fmaxf(m, s[c] * hs);
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
        uint8_t* dst = ps + (c0 / 64) * kAtom;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint32_t pk[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int i0 = 8 * c + 2 * u;
            const bool v0 = sm.idx[t][c0 + i0] >= 0, v1 = sm.idx[t][c0 + i0 + 1] >= 0;
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
      const float inv = l_o > 0.0f ? 1.0f / l_o : 0.0f;
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
          for (int c = 0; c < 16; ++c) dst[c] = make_float4(o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]);
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
