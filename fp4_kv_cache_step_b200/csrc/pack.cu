// pack.cu -- FP4 (E2M1) main-KV quantisation with one E4M3 scale per channel
// per 64-entry block, and its exact inverse.
//
// Format: "Detailed Notes On DeepSeek V4 Point 1 Flash In Simple Words",
// section "FP4 Main KV Cache To Halve Storage Again" (E2M1 values with E4M3
// scales, no global scale) and the mengman.github.io interpretation, section
// 3.5. The scale of a block channel is round-to-nearest-even E4M3 of
// blockmax / 6; codes are the nearest E2M1 grid point with ties to the even
// code. Both kernels are HBM-bound streaming kernels: 8 B read + 0.5 B
// (+ 1/64 B of scale) written per value for the pack, the reverse for unpack.
//
// The same section and the interpretation's 3.5 give the production layout:
// one E4M3 scale per 16 channels of an entry, with no second-level scale. The
// *_g16 kernels store it as one row per entry, its D/2 code bytes followed by
// its D/16 scale bytes (288 bytes at D = 512); a group's scale follows the same
// rule (nearest E4M3 of max|x| / 6). Each row depends on its own entry alone,
// so appending an entry writes its row and nothing else.
#include "common.cuh"
#include "kernels.h"

namespace csa2 {
namespace {

constexpr int kPackThreads = 256;    // 64 channel groups x 4 entry groups
constexpr int kChanPerThread = 8;
constexpr int kSlab = 64 * kChanPerThread;   // 512 channels per CTA

// E2M1 magnitude code of |x| at scale s by exact comparison with the
// midpoints between grid points (t * s is exact in fp32: t has <= 3 and s
// <= 4 significant bits). At a midpoint the even code wins.
__device__ __forceinline__ uint32_t e2m1_code(float x, float s) {
  if (s == 0.0f) return 0u;
  float a = fabsf(x);
  uint32_t c = (a > 0.25f * s) + (a >= 0.75f * s) + (a > 1.25f * s) + (a >= 1.75f * s) +
               (a > 2.5f * s) + (a >= 3.5f * s) + (a > 5.0f * s);
  return c | (signbit(x) ? 8u : 0u);
}

__global__ void __launch_bounds__(kPackThreads)
fp4_pack_kernel(const float* __restrict__ kv, int N, int D, uint8_t* __restrict__ packed,
                uint8_t* __restrict__ scale, int* err) {
  __shared__ float amax_part[4][kSlab];
  const int blk = blockIdx.x, b = blockIdx.y, slab = blockIdx.z;
  const int cg = threadIdx.x & 63, eg = threadIdx.x >> 6;
  const int c0 = slab * kSlab + cg * kChanPerThread;
  const bool active = c0 < D;
  const size_t row0 = (size_t)b * N + (size_t)blk * kBlockEntries + eg * 16;

  float amax[kChanPerThread];
#pragma unroll
  for (int i = 0; i < kChanPerThread; ++i) amax[i] = 0.0f;
  bool bad = false;
  if (active) {
#pragma unroll 4
    for (int r = 0; r < 16; ++r) {
      const float4* p = reinterpret_cast<const float4*>(kv + (row0 + r) * D + c0);
      float4 v0 = __ldg(p), v1 = __ldg(p + 1);
      float v[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        bad |= !isfinite(v[i]);
        amax[i] = fmaxf(amax[i], fabsf(v[i]));
      }
    }
  }
  if (bad) record_error(err, CSA2_ERR_NONFINITE);
#pragma unroll
  for (int i = 0; i < kChanPerThread; ++i) amax_part[eg][cg * kChanPerThread + i] = amax[i];
  __syncthreads();
  if (!active) return;

  float s[kChanPerThread];
  uint8_t sbytes[kChanPerThread];
#pragma unroll
  for (int i = 0; i < kChanPerThread; i += 2) {
    float m0 = amax_part[0][cg * 8 + i], m1 = amax_part[0][cg * 8 + i + 1];
#pragma unroll
    for (int g = 1; g < 4; ++g) {
      m0 = fmaxf(m0, amax_part[g][cg * 8 + i]);
      m1 = fmaxf(m1, amax_part[g][cg * 8 + i + 1]);
    }
    // IEEE division then RNE to E4M3: equal to rounding the exact quotient,
    // since an fp32 quotient never lands on an E4M3 tie unless it is exact.
    __nv_fp8x2_storage_t sc =
        __nv_cvt_float2_to_fp8x2(make_float2(m0 / 6.0f, m1 / 6.0f), __NV_SATFINITE, __NV_E4M3);
    sbytes[i] = (uint8_t)(sc & 0xff);
    sbytes[i + 1] = (uint8_t)(sc >> 8);
    float2 sf = __half22float2(e4m3x2_to_half2(sc));
    s[i] = sf.x;
    s[i + 1] = sf.y;
  }
  if (eg == 0) {
    uint2 w;
    w.x = sbytes[0] | (sbytes[1] << 8) | (sbytes[2] << 16) | ((uint32_t)sbytes[3] << 24);
    w.y = sbytes[4] | (sbytes[5] << 8) | (sbytes[6] << 16) | ((uint32_t)sbytes[7] << 24);
    *reinterpret_cast<uint2*>(scale + ((size_t)b * (N / kBlockEntries) + blk) * D + c0) = w;
  }
#pragma unroll 4
  for (int r = 0; r < 16; ++r) {
    const float4* p = reinterpret_cast<const float4*>(kv + (row0 + r) * D + c0);
    float4 v0 = __ldg(p), v1 = __ldg(p + 1);
    float v[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
    uint32_t word = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) word |= e2m1_code(v[i], s[i]) << (4 * i);
    *reinterpret_cast<uint32_t*>(packed + (row0 + r) * (D / 2) + c0 / 2) = word;
  }
}

// One thread per 8 channels of one entry.
__global__ void fp4_unpack_kernel(const uint8_t* __restrict__ packed,
                                  const uint8_t* __restrict__ scale, int B, int N, int D,
                                  float* __restrict__ out) {
  const int groups = D / 8;
  const size_t total = (size_t)B * N * groups;
  for (size_t g = blockIdx.x * (size_t)blockDim.x + threadIdx.x; g < total;
       g += (size_t)gridDim.x * blockDim.x) {
    const size_t row = g / groups;
    const int c0 = (int)(g % groups) * 8;
    const int b = (int)(row / N), n = (int)(row % N);
    uint32_t codes = *reinterpret_cast<const uint32_t*>(packed + row * (D / 2) + c0 / 2);
    uint2 sw = *reinterpret_cast<const uint2*>(
        scale + ((size_t)b * (N / kBlockEntries) + n / kBlockEntries) * D + c0);
    uint32_t sv[2] = {sw.x, sw.y};
    float res[8];
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
      __half2 v = e2m1x2_to_half2((uint8_t)(codes >> (4 * i)));
      __half2 sc = e4m3x2_to_half2((uint16_t)(sv[i / 4] >> (8 * (i % 4))));
      float2 f = __half22float2(__hmul2(v, sc));   // exact: <= 6 significant bits
      res[i] = f.x;
      res[i + 1] = f.y;
    }
    float4* o = reinterpret_cast<float4*>(out + row * D + c0);
    o[0] = make_float4(res[0], res[1], res[2], res[3]);
    o[1] = make_float4(res[4], res[5], res[6], res[7]);
  }
}

// One thread per 16-channel group of one source entry; the entry is written to
// cache row pos[b][t] (pos NULL: row t).
__global__ void fp4_pack_g16_kernel(const float* __restrict__ kv, const int32_t* __restrict__ pos,
                                    int B, int T, int N, int D, uint8_t* __restrict__ rows,
                                    int* err) {
  const int groups = D / 16;
  const size_t rb = (size_t)D / 2 + groups;
  const size_t total = (size_t)B * T * groups;
  for (size_t g = blockIdx.x * (size_t)blockDim.x + threadIdx.x; g < total;
       g += (size_t)gridDim.x * blockDim.x) {
    const size_t src = g / groups;            // b * T + t
    const int grp = (int)(g % groups);
    const int b = (int)(src / T);
    int n = (int)(src % T);
    if (pos != nullptr) {
      n = __ldg(pos + src);
      if (n < 0 || n >= N) {
        record_error(err, CSA2_ERR_DEVICE_INDEX);
        continue;
      }
    }
    const float4* x4 = reinterpret_cast<const float4*>(kv + src * D + grp * 16);
    float v[16];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 f = __ldg(x4 + i);
      v[4 * i] = f.x;
      v[4 * i + 1] = f.y;
      v[4 * i + 2] = f.z;
      v[4 * i + 3] = f.w;
    }
    float amax = 0.0f;
    bool bad = false;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      bad |= !isfinite(v[i]);
      amax = fmaxf(amax, fabsf(v[i]));
    }
    if (bad) record_error(err, CSA2_ERR_NONFINITE);
    // IEEE division then RNE to E4M3 (saturating), as in the block layout
    const __nv_fp8_storage_t sc = __nv_cvt_float_to_fp8(amax / 6.0f, __NV_SATFINITE, __NV_E4M3);
    const float s = __low2float(e4m3x2_to_half2((uint16_t)sc));
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int i = 0; i < 16; ++i) w[i >> 3] |= e2m1_code(v[i], s) << (4 * (i & 7));
    uint8_t* dst = rows + ((size_t)b * N + n) * rb;
    *reinterpret_cast<uint2*>(dst + grp * 8) = make_uint2(w[0], w[1]);
    dst[D / 2 + grp] = (uint8_t)sc;
  }
}

// One thread per 16-channel group of one entry: exact values.
__global__ void fp4_unpack_g16_kernel(const uint8_t* __restrict__ rows, int B, int N, int D,
                                      float* __restrict__ out) {
  const int groups = D / 16;
  const size_t rb = (size_t)D / 2 + groups;
  const size_t total = (size_t)B * N * groups;
  for (size_t g = blockIdx.x * (size_t)blockDim.x + threadIdx.x; g < total;
       g += (size_t)gridDim.x * blockDim.x) {
    const size_t row = g / groups;
    const int grp = (int)(g % groups);
    const uint8_t* src = rows + row * rb;
    const uint2 c = *reinterpret_cast<const uint2*>(src + grp * 8);
    const uint8_t sc = src[D / 2 + grp];
    const __half2 s2 = e4m3x2_to_half2((uint16_t)(sc | (sc << 8)));
    const uint32_t cw[2] = {c.x, c.y};
    float res[16];
#pragma unroll
    for (int i = 0; i < 16; i += 2) {
      const float2 f = __half22float2(
          __hmul2(e2m1x2_to_half2((uint8_t)(cw[i >> 3] >> (4 * (i & 7)))), s2));   // exact
      res[i] = f.x;
      res[i + 1] = f.y;
    }
    float4* o = reinterpret_cast<float4*>(out + row * D + grp * 16);
#pragma unroll
    for (int i = 0; i < 4; ++i)
      o[i] = make_float4(res[4 * i], res[4 * i + 1], res[4 * i + 2], res[4 * i + 3]);
  }
}

int grid_for(size_t total, int threads) {
  size_t blocks = (total + threads - 1) / threads;
  if (blocks > 148 * 64) blocks = 148 * 64;
  return (int)blocks;
}

}  // namespace

cudaError_t launch_fp4_pack_g16(const float* kv, const int32_t* pos, int B, int T, int N, int D,
                                uint8_t* rows, int* err, cudaStream_t stream) {
  const size_t total = (size_t)B * T * (D / 16);
  if (total == 0) return cudaSuccess;
  fp4_pack_g16_kernel<<<grid_for(total, 256), 256, 0, stream>>>(kv, pos, B, T, N, D, rows, err);
  return cudaGetLastError();
}

cudaError_t launch_fp4_unpack_g16(const uint8_t* rows, int B, int N, int D, float* out,
                                  cudaStream_t stream) {
  const size_t total = (size_t)B * N * (D / 16);
  if (total == 0) return cudaSuccess;
  fp4_unpack_g16_kernel<<<grid_for(total, 256), 256, 0, stream>>>(rows, B, N, D, out);
  return cudaGetLastError();
}

cudaError_t launch_fp4_pack(const float* kv, int B, int N, int D, uint8_t* packed,
                            uint8_t* scale, int* err, cudaStream_t stream) {
  if (B == 0 || N == 0) return cudaSuccess;
  dim3 grid(N / kBlockEntries, B, ceil_div(D, kSlab));
  fp4_pack_kernel<<<grid, kPackThreads, 0, stream>>>(kv, N, D, packed, scale, err);
  return cudaGetLastError();
}

cudaError_t launch_fp4_unpack(const uint8_t* packed, const uint8_t* scale, int B, int N, int D,
                              float* out, cudaStream_t stream) {
  size_t total = (size_t)B * N * (D / 8);
  if (total == 0) return cudaSuccess;
  int threads = 256;
  size_t blocks = (total + threads - 1) / threads;
  if (blocks > 148 * 64) blocks = 148 * 64;
  fp4_unpack_kernel<<<(unsigned)blocks, threads, 0, stream>>>(packed, scale, B, N, D, out);
  return cudaGetLastError();
}

}  // namespace csa2
