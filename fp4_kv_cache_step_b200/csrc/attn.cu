// attn.cu -- fused gather + FP4 dequantisation + sparse softmax attention.
//
// "Detailed Notes On DeepSeek V4 Point 1 Flash In Simple Words", sections
// "Compressed Sparse Attention 2 Or CSA2 In Simple Terms" (attend only to the
// top-K entries the indexer picked) and "FP4 Main KV Cache To Halve Storage
// Again" (E2M1 values are dequantised back before attention); "Model Setup
// Numbers Without Jargon": 64 query heads of dimension 512 share one main-KV
// head, which serves as both key and value.
//
// One CTA = (query row, 64-head block, split of the index list). Per tile of
// 64 selected entries the CTA gathers the packed rows and their scale rows with
// plain vector loads, dequantises them exactly to fp16 in shared memory, then
// runs S = Q V^T (tensor cores, fp32 accumulate), an online softmax in fp32, and
// O += P V with P in fp16. Queries are scaled per head by a power of two before
// the fp16 conversion so that every bf16 query value keeps its bits (values more
// than 2^31 below the head's largest magnitude excepted); the factor is undone
// in the softmax scale. Splits are merged by log-sum-exp weights.
#include "common.cuh"
#include "kernels.h"

namespace csa2 {
namespace {

constexpr int kThreads = 512;           // 16 warps
constexpr int kHB = 64;                 // heads per CTA
constexpr int kTile = 64;               // selected entries per tile
constexpr int kD = kHeadDim;            // 512
constexpr int kQS = kD + 8;             // padded row strides (halves) -> conflict-free ldmatrix
constexpr int kVS = kD + 8;
constexpr int kPS = kTile + 8;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

struct __align__(16) AttnSmem {
  __half q[kHB][kQS];
  __half v[kTile][kVS];
  __half p[kHB][kPS];
  float red_max[4][kHB];
  float red_sum[4][kHB];
  float head_scale[kHB];
  int idx[kTile];
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void mma_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                        uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__global__ void __launch_bounds__(kThreads, 1)
sparse_attn_kernel(const uint16_t* __restrict__ q, const uint8_t* __restrict__ kv_packed,
                   const uint8_t* __restrict__ kv_scale, const int32_t* __restrict__ topk,
                   int Tq, int Hq, int N, int K, float softmax_scale, int split_len, int nsplit,
                   uint16_t* __restrict__ out, float* __restrict__ lse,
                   float* __restrict__ ws_o, float2* __restrict__ ws_ml, int* err) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  AttnSmem& sm = *reinterpret_cast<AttnSmem*>(smem_raw);
  const size_t row = blockIdx.x;
  const int hb = blockIdx.y, split = blockIdx.z;
  const int b = (int)(row / Tq);
  const int h0 = hb * kHB;
  const int nh = min(kHB, Hq - h0);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, qd = lane & 3;
  const int k_begin = split * split_len;
  const int k_end = min(K, k_begin + split_len);

  // ---- queries -> fp16 with a power-of-two scale per head
  for (int hh = warp * 4; hh < warp * 4 + 4; ++hh) {
    float vals[16];
    float amax = 0.0f;
    if (hh < nh) {
      const uint4* src = reinterpret_cast<const uint4*>(q + ((row * Hq) + h0 + hh) * kD + lane * 16);
      uint4 u[2] = {src[0], src[1]};
      const uint32_t* w = reinterpret_cast<const uint32_t*>(u);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        vals[2 * i] = __uint_as_float(w[i] << 16);
        vals[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        amax = fmaxf(amax, fmaxf(fabsf(vals[2 * i]), fabsf(vals[2 * i + 1])));
      }
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i) vals[i] = 0.0f;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    int e = 0;
    if (amax > 0.0f && isfinite(amax)) {
      int ex;
      frexpf(amax, &ex);          // amax < 2^ex
      e = 15 - ex;                // scaled magnitudes < 2^15
    }
    uint32_t packed[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
      packed[i] = pack_half2(ldexpf(vals[2 * i], e), ldexpf(vals[2 * i + 1], e));
    uint4* dst = reinterpret_cast<uint4*>(&sm.q[hh][lane * 16]);
    dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
    if (lane == 0) sm.head_scale[hh] = (hh < nh) ? softmax_scale * ldexpf(kLog2e, -e) : 0.0f;
  }

  // ---- per-thread running softmax state for rows (hg*16 + g) and (+8)
  const int hg = warp & 3;             // head group (16 rows) for both matmuls
  const int eg = warp >> 2;            // entry group (16 entries) for S
  const int ds = warp >> 2;            // dim slice (128 dims) for O
  const int r_lo = hg * 16 + g, r_hi = r_lo + 8;
  float m_lo = -INFINITY, m_hi = -INFINITY, l_lo = 0.0f, l_hi = 0.0f;
  float o[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.0f;

  const uint8_t* pk_b = kv_packed + (size_t)b * N * (kD / 2);
  const uint8_t* sc_b = kv_scale + (size_t)b * (N / kBlockEntries) * kD;
  const int32_t* idx_row = topk + row * K;

  for (int t0 = k_begin; t0 < k_end; t0 += kTile) {
    __syncthreads();   // previous tile's P V (and the query staging) done
    // ---- gather + dequantise: thread = (entry, 8-channel lane of each 64)
    {
      const int e = threadIdx.x >> 3, part = threadIdx.x & 7;
      const int kk = t0 + e;
      int id = kk < k_end ? idx_row[kk] : -1;
      if (id >= N) { record_error(err, CSA2_ERR_DEVICE_INDEX); id = -1; }
      if (id < -1) { record_error(err, CSA2_ERR_DEVICE_INDEX); id = -1; }
      if (part == 0) sm.idx[e] = id;
      const uint8_t* prow = pk_b + (size_t)max(id, 0) * (kD / 2);
      const uint8_t* srow = sc_b + (size_t)(max(id, 0) / kBlockEntries) * kD;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int c = j * 64 + part * 8;
        uint4 res = make_uint4(0, 0, 0, 0);
        if (id >= 0) {
          uint32_t codes = *reinterpret_cast<const uint32_t*>(prow + c / 2);
          uint2 sv = *reinterpret_cast<const uint2*>(srow + c);
          uint32_t h[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            __half2 vv = e2m1x2_to_half2((uint8_t)(codes >> (8 * i)));
            uint32_t sw = i < 2 ? sv.x : sv.y;
            __half2 ss = e4m3x2_to_half2((uint16_t)(sw >> (16 * (i & 1))));
            __half2 pr = __hmul2(vv, ss);
            h[i] = *reinterpret_cast<uint32_t*>(&pr);
          }
          res = make_uint4(h[0], h[1], h[2], h[3]);
        }
        *reinterpret_cast<uint4*>(&sm.v[e][c]) = res;
      }
    }
    __syncthreads();

    // ---- S = Q V^T for rows hg*16.., entries eg*16..
    float s[2][4] = {{0, 0, 0, 0}, {0, 0, 0, 0}};
    {
      const uint32_t a_base = smem_u32(&sm.q[hg * 16 + (lane & 15)][(lane >> 4) * 8]);
      const int mi = lane >> 3, r = lane & 7;
      const uint32_t b_base = smem_u32(&sm.v[eg * 16 + (mi >> 1) * 8 + r][(mi & 1) * 8]);
#pragma unroll 8
      for (int ks = 0; ks < kD / 16; ++ks) {
        uint32_t a0, a1, a2, a3, b0, b1, b2, b3;
        ldsm_x4(a_base + ks * 32, a0, a1, a2, a3);
        ldsm_x4(b_base + ks * 32, b0, b1, b2, b3);
        mma_f16(s[0], a0, a1, a2, a3, b0, b1);
        mma_f16(s[1], a0, a1, a2, a3, b2, b3);
      }
    }
    const float sc_lo = sm.head_scale[r_lo], sc_hi = sm.head_scale[r_hi];
    float mx_lo = -INFINITY, mx_hi = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const int c = eg * 16 + nt * 8 + 2 * qd;
      const bool v0 = sm.idx[c] >= 0, v1 = sm.idx[c + 1] >= 0;
      s[nt][0] = v0 ? s[nt][0] * sc_lo : -INFINITY;
      s[nt][1] = v1 ? s[nt][1] * sc_lo : -INFINITY;
      s[nt][2] = v0 ? s[nt][2] * sc_hi : -INFINITY;
      s[nt][3] = v1 ? s[nt][3] * sc_hi : -INFINITY;
      mx_lo = fmaxf(mx_lo, fmaxf(s[nt][0], s[nt][1]));
      mx_hi = fmaxf(mx_hi, fmaxf(s[nt][2], s[nt][3]));
    }
#pragma unroll
    for (int o2 = 1; o2 < 4; o2 <<= 1) {
      mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, o2));
      mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, o2));
    }
    if (qd == 0) {
      sm.red_max[eg][r_lo] = mx_lo;
      sm.red_max[eg][r_hi] = mx_hi;
    }
    __syncthreads();
    float mn_lo = m_lo, mn_hi = m_hi;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      mn_lo = fmaxf(mn_lo, sm.red_max[i][r_lo]);
      mn_hi = fmaxf(mn_hi, sm.red_max[i][r_hi]);
    }
    float sum_lo = 0.0f, sum_hi = 0.0f;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      float p0 = mn_lo == -INFINITY ? 0.0f : exp2f(s[nt][0] - mn_lo);
      float p1 = mn_lo == -INFINITY ? 0.0f : exp2f(s[nt][1] - mn_lo);
      float p2 = mn_hi == -INFINITY ? 0.0f : exp2f(s[nt][2] - mn_hi);
      float p3 = mn_hi == -INFINITY ? 0.0f : exp2f(s[nt][3] - mn_hi);
      sum_lo += p0 + p1;
      sum_hi += p2 + p3;
      const int c = eg * 16 + nt * 8 + 2 * qd;
      *reinterpret_cast<uint32_t*>(&sm.p[r_lo][c]) = pack_half2(p0, p1);
      *reinterpret_cast<uint32_t*>(&sm.p[r_hi][c]) = pack_half2(p2, p3);
    }
#pragma unroll
    for (int o2 = 1; o2 < 4; o2 <<= 1) {
      sum_lo += __shfl_xor_sync(0xffffffffu, sum_lo, o2);
      sum_hi += __shfl_xor_sync(0xffffffffu, sum_hi, o2);
    }
    if (qd == 0) {
      sm.red_sum[eg][r_lo] = sum_lo;
      sm.red_sum[eg][r_hi] = sum_hi;
    }
    __syncthreads();
    const float al_lo = (m_lo == -INFINITY) ? 0.0f : exp2f(m_lo - mn_lo);
    const float al_hi = (m_hi == -INFINITY) ? 0.0f : exp2f(m_hi - mn_hi);
    l_lo = al_lo * l_lo + sm.red_sum[0][r_lo] + sm.red_sum[1][r_lo] + sm.red_sum[2][r_lo] +
           sm.red_sum[3][r_lo];
    l_hi = al_hi * l_hi + sm.red_sum[0][r_hi] + sm.red_sum[1][r_hi] + sm.red_sum[2][r_hi] +
           sm.red_sum[3][r_hi];
    m_lo = mn_lo;
    m_hi = mn_hi;

    // ---- O = alpha O + P V for rows hg*16.., dims ds*128..
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      o[i][0] *= al_lo;
      o[i][1] *= al_lo;
      o[i][2] *= al_hi;
      o[i][3] *= al_hi;
    }
    {
      const uint32_t a_base = smem_u32(&sm.p[hg * 16 + (lane & 15)][(lane >> 4) * 8]);
      const int mi = lane >> 3, r = lane & 7;
      const uint32_t b_base = smem_u32(&sm.v[(mi & 1) * 8 + r][ds * 128 + (mi >> 1) * 8]);
#pragma unroll
      for (int ks = 0; ks < kTile / 16; ++ks) {
        uint32_t a0, a1, a2, a3;
        ldsm_x4(a_base + ks * 32, a0, a1, a2, a3);
#pragma unroll
        for (int np = 0; np < 8; ++np) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(b_base + ks * 16 * kVS * 2 + np * 32, b0, b1, b2, b3);
          mma_f16(o[2 * np], a0, a1, a2, a3, b0, b1);
          mma_f16(o[2 * np + 1], a0, a1, a2, a3, b2, b3);
        }
      }
    }
  }

  // ---- write results
  const int d0 = ds * 128 + 2 * qd;
  if (nsplit == 1) {
    const float inv_lo = l_lo > 0.0f ? 1.0f / l_lo : 0.0f;
    const float inv_hi = l_hi > 0.0f ? 1.0f / l_hi : 0.0f;
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) {
      const int d = d0 + nt * 8;
      if (r_lo < nh) {
        __nv_bfloat162 v = __floats2bfloat162_rn(o[nt][0] * inv_lo, o[nt][1] * inv_lo);
        *reinterpret_cast<__nv_bfloat162*>(out + ((row * Hq) + h0 + r_lo) * kD + d) = v;
      }
      if (r_hi < nh) {
        __nv_bfloat162 v = __floats2bfloat162_rn(o[nt][2] * inv_hi, o[nt][3] * inv_hi);
        *reinterpret_cast<__nv_bfloat162*>(out + ((row * Hq) + h0 + r_hi) * kD + d) = v;
      }
    }
    if (lse != nullptr && ds == 0 && qd == 0) {
      if (r_lo < nh) lse[row * Hq + h0 + r_lo] = l_lo > 0.0f ? (m_lo + log2f(l_lo)) * kLn2 : -INFINITY;
      if (r_hi < nh) lse[row * Hq + h0 + r_hi] = l_hi > 0.0f ? (m_hi + log2f(l_hi)) * kLn2 : -INFINITY;
    }
  } else {
    const size_t slot = (row * gridDim.y + hb) * nsplit + split;
    float* wo = ws_o + slot * kHB * kD;
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) {
      const int d = d0 + nt * 8;
      *reinterpret_cast<float2*>(wo + r_lo * kD + d) = make_float2(o[nt][0], o[nt][1]);
      *reinterpret_cast<float2*>(wo + r_hi * kD + d) = make_float2(o[nt][2], o[nt][3]);
    }
    if (ds == 0 && qd == 0) {
      ws_ml[slot * kHB + r_lo] = make_float2(m_lo, l_lo);
      ws_ml[slot * kHB + r_hi] = make_float2(m_hi, l_hi);
    }
  }
}

// Merge the splits of one (row, head): weights 2^(m_s - M) l_s.
__global__ void __launch_bounds__(128)
attn_combine_kernel(const float* __restrict__ ws_o, const float2* __restrict__ ws_ml, int Hq,
                    int nhb, int nsplit, uint16_t* __restrict__ out, float* __restrict__ lse) {
  const size_t row = blockIdx.x;
  const int h = blockIdx.y;
  const int hb = h / kHB, r = h % kHB;
  const size_t slot0 = (row * nhb + hb) * nsplit;
  float M = -INFINITY;
  for (int s = 0; s < nsplit; ++s) M = fmaxf(M, ws_ml[(slot0 + s) * kHB + r].x);
  float L = 0.0f;
  float4 acc = make_float4(0, 0, 0, 0);
  const int d = threadIdx.x * 4;
  if (M != -INFINITY) {
    for (int s = 0; s < nsplit; ++s) {
      float2 ml = ws_ml[(slot0 + s) * kHB + r];
      if (ml.x == -INFINITY) continue;
      float w = exp2f(ml.x - M);
      L += w * ml.y;
      float4 v = *reinterpret_cast<const float4*>(ws_o + ((slot0 + s) * kHB + r) * kD + d);
      acc.x += w * v.x;
      acc.y += w * v.y;
      acc.z += w * v.z;
      acc.w += w * v.w;
    }
  }
  const float inv = L > 0.0f ? 1.0f / L : 0.0f;
  __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
  __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
  uint2 pk;
  pk.x = *reinterpret_cast<uint32_t*>(&lo);
  pk.y = *reinterpret_cast<uint32_t*>(&hi);
  *reinterpret_cast<uint2*>(out + (row * Hq + h) * kD + d) = pk;
  if (lse != nullptr && threadIdx.x == 0)
    lse[row * Hq + h] = L > 0.0f ? (M + log2f(L)) * kLn2 : -INFINITY;
}

struct SplitPlan {
  int nhb, nsplit, split_len;
};

SplitPlan plan_splits(int rows, int Hq, int K) {
  SplitPlan p;
  p.nhb = ceil_div(Hq, kHB);
  const int ctas = rows * p.nhb;
  const int target = 2 * 148;
  int nsplit = ctas >= target ? 1 : ceil_div(target, ctas);
  const int max_split = ceil_div(K, kTile);
  if (nsplit > max_split) nsplit = max_split;
  p.split_len = ceil_div(ceil_div(K, nsplit), kTile) * kTile;
  p.nsplit = ceil_div(K, p.split_len);
  return p;
}

}  // namespace

size_t sparse_attn_workspace_bytes(int B, int Tq, int Hq, int K) {
  const int rows = B * Tq;
  SplitPlan p = plan_splits(rows, Hq, K);
  if (p.nsplit == 1) return 0;
  size_t slots = (size_t)rows * p.nhb * p.nsplit;
  return slots * kHB * (kD * sizeof(float) + sizeof(float2));
}

cudaError_t launch_sparse_attn(const uint16_t* q, const uint8_t* kv_packed,
                               const uint8_t* kv_scale, const int32_t* topk_idx, int B, int Tq,
                               int Hq, int N, int K, float softmax_scale, uint16_t* out,
                               float* lse, void* workspace, int* err, cudaStream_t stream) {
  const int rows = B * Tq;
  if (rows == 0) return cudaSuccess;
  SplitPlan p = plan_splits(rows, Hq, K);
  const size_t smem = sizeof(AttnSmem);
  cudaError_t e = cudaFuncSetAttribute(sparse_attn_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  float* ws_o = nullptr;
  float2* ws_ml = nullptr;
  if (p.nsplit > 1) {
    size_t slots = (size_t)rows * p.nhb * p.nsplit;
    ws_o = static_cast<float*>(workspace);
    ws_ml = reinterpret_cast<float2*>(ws_o + slots * kHB * kD);
  }
  dim3 grid(rows, p.nhb, p.nsplit);
  sparse_attn_kernel<<<grid, kThreads, smem, stream>>>(q, kv_packed, kv_scale, topk_idx, Tq, Hq, N,
                                                       K, softmax_scale, p.split_len, p.nsplit,
                                                       out, lse, ws_o, ws_ml, err);
  e = cudaGetLastError();
  if (e != cudaSuccess || p.nsplit == 1) return e;
  attn_combine_kernel<<<dim3(rows, Hq), 128, 0, stream>>>(ws_o, ws_ml, Hq, p.nhb, p.nsplit, out,
                                                          lse);
  return cudaGetLastError();
}

}  // namespace csa2
