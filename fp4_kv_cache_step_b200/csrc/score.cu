// score.cu -- CSA2 indexer scoring.
//
// "Detailed Notes On DeepSeek V4 Point 1 Flash In Simple Words", section
// "Compressed Sparse Attention 2 Or CSA2 In Simple Terms": a small per-layer
// indexer scores past main-KV entries against the current query; the indexer
// keys are one shared key per entry. Score of entry j for query (b, t):
//     s_j = sum_h w_h * max(0, q_h . k_j)
// with E4M3 queries and keys and fp32 accumulation. The mengman.github.io
// interpretation, section 3.4: a REINDEX layer can score only inside the
// candidate pool of the first FULL layer.
//
// This file holds the dispatcher and the CUDA-core scorer: one CTA per (query
// row, 128 entries), the query decoded once into shared memory (broadcast
// reads), each thread one entry, heads in groups of 32 register accumulators.
// The CUDA-core scorer serves the candidate-pool gather and shapes the
// tensor-core scorer (score_tc.cu) does not take.
#include "common.cuh"
#include "kernels.h"

namespace csa2 {
namespace {

constexpr int kTileEntries = 128;

__global__ void __launch_bounds__(kTileEntries)
index_score_simt_kernel(const uint8_t* __restrict__ idx_q, const float* __restrict__ idx_w,
                        const uint8_t* __restrict__ idx_k, int Tq, int N, int Hi, int Di,
                        const int32_t* __restrict__ nvalid, const int32_t* __restrict__ cand,
                        int C, float* __restrict__ scores, int* err) {
  extern __shared__ __align__(16) float qs[];   // [Hi][Di] then w[Hi]
  float* ws = qs + Hi * Di;
  pdl_wait_and_release();
  const int tile = blockIdx.x;
  const size_t row = (size_t)blockIdx.z * Tq + blockIdx.y;
  const int b = blockIdx.z;
  const int len = cand ? C : max(0, min(N, nvalid[row]));
  const int i0 = tile * kTileEntries;
  if (i0 >= len) return;

  const uint16_t* q2 = reinterpret_cast<const uint16_t*>(idx_q + row * Hi * Di);
  for (int e = threadIdx.x; e < Hi * Di / 2; e += blockDim.x) {
    float2 f = __half22float2(e4m3x2_to_half2(q2[e]));
    qs[2 * e] = f.x;
    qs[2 * e + 1] = f.y;
  }
  for (int h = threadIdx.x; h < Hi; h += blockDim.x) ws[h] = idx_w[row * Hi + h];
  __syncthreads();

  const int i = i0 + threadIdx.x;
  if (i >= len) return;
  const size_t ld = cand ? (size_t)C : (size_t)N;
  int j = i;
  if (cand) {
    j = cand[row * C + i];
    if (j < 0 || j >= N) {
      if (j >= N || j < -1) record_error(err, CSA2_ERR_DEVICE_INDEX);
      scores[row * ld + i] = -INFINITY;
      return;
    }
  }
  const uint8_t* k = idx_k + ((size_t)b * N + j) * Di;
  float total = 0.0f;
  bool nan = false;
  for (int h0 = 0; h0 < Hi; h0 += 32) {
    float acc[32];
#pragma unroll
    for (int hh = 0; hh < 32; ++hh) acc[hh] = 0.0f;
    for (int c0 = 0; c0 < Di; c0 += 16) {
      uint4 kb = *reinterpret_cast<const uint4*>(k + c0);
      const uint32_t w4[4] = {kb.x, kb.y, kb.z, kb.w};
      float kf[16];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        float2 f = __half22float2(e4m3x2_to_half2((uint16_t)(w4[u / 2] >> (16 * (u & 1)))));
        kf[2 * u] = f.x;
        kf[2 * u + 1] = f.y;
      }
#pragma unroll
      for (int hh = 0; hh < 32; ++hh) {
        if (h0 + hh < Hi) {
          const float4* qp = reinterpret_cast<const float4*>(qs + (h0 + hh) * Di + c0);
          float a = acc[hh];
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            float4 qq = qp[v];
            a = fmaf(qq.x, kf[4 * v], a);
            a = fmaf(qq.y, kf[4 * v + 1], a);
            a = fmaf(qq.z, kf[4 * v + 2], a);
            a = fmaf(qq.w, kf[4 * v + 3], a);
          }
          acc[hh] = a;
        }
      }
    }
#pragma unroll
    for (int hh = 0; hh < 32; ++hh) {
      if (h0 + hh < Hi) {
        nan |= isnan(acc[hh]);
        total = fmaf(ws[h0 + hh], fmaxf(acc[hh], 0.0f), total);
      }
    }
  }
  if (nan) record_error(err, CSA2_ERR_NONFINITE);
  scores[row * ld + i] = total;
}

}  // namespace

cudaError_t launch_index_score(const uint8_t* idx_q, const float* idx_w, const uint8_t* idx_k,
                               int B, int Tq, int N, int Hi, int Di, const int32_t* nvalid,
                               const int32_t* cand, int C, float* scores, int* err,
                               cudaStream_t stream) {
  if (B == 0 || Tq == 0) return cudaSuccess;
  if (index_score_tc_supported(B, Tq, Hi, Di, cand))
    return launch_index_score_tc(idx_q, idx_w, idx_k, B, Tq, N, Hi, Di, nvalid, scores, err,
                                 stream);
  const int len = cand ? C : N;
  if (len == 0) return cudaSuccess;
  const size_t smem = ((size_t)Hi * Di + Hi) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(index_score_simt_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(ceil_div(len, kTileEntries), Tq, B);
  return launch_pdl(index_score_simt_kernel, grid, dim3(kTileEntries), smem, stream, dim3(1),
                    idx_q, idx_w, idx_k, Tq, N, Hi, Di, nvalid, cand, C, scores, err);
}

}  // namespace csa2
