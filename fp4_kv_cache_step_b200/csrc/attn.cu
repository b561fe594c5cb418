// attn.cu -- sparse attention launcher: split planning and the log-sum-exp
// merge of split partials. The fused gather + dequant + attention kernel itself
// is in attn_tc.cu.
//
// A CTA handles one (query row, 64-head block, split of the index list). When
// the batch has too few rows to fill the GPU the index list is split so that
// rows x splits is about one CTA per SM; each split writes its unnormalised
// output with its running max m (log2 domain) and sum l, and
// attn_combine_kernel merges them with weights 2^(m_s - M) l_s.
#include "common.cuh"
#include "kernels.h"

namespace csa2 {
namespace {

constexpr int kHB = 64;                 // heads per CTA
constexpr int kD = kHeadDim;            // 512
constexpr float kLn2 = 0.6931471805599453f;

// Merge the splits of one (row, head): weights 2^(m_s - M) l_s.
__global__ void __launch_bounds__(128)
attn_combine_kernel(const float* __restrict__ ws_o, const float2* __restrict__ ws_ml, int Hq,
                    int nhb, int nsplit, uint16_t* __restrict__ out, float* __restrict__ lse) {
  pdl_wait_and_release();
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
  bool cluster;   // up to the largest cluster, the splits may merge inside a cluster
};

int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

// A CTA walks its split of the index list in tiles of sparse_attn_tc_tile()
// entries, so any split length works; the list is split only when the batch
// has too few (row, head block) pairs to give every SM a CTA.
SplitPlan plan_splits(int rows, int Hq, int K) {
  SplitPlan p;
  p.nhb = ceil_div(Hq, kHB);
  const int tile = sparse_attn_tc_tile();
  const int ctas = rows * p.nhb;
  const int sms = sm_count();
  int nsplit = ctas >= sms ? 1 : sms / ctas;
  // up to twice the largest cluster, the splits stay one cluster that merges on
  // chip (a few idle SMs cost less than the workspace round trip and the
  // combine launch)
  const int cmax = sparse_attn_tc_max_cluster();
  if (nsplit > cmax && nsplit < 2 * cmax) nsplit = cmax;
  nsplit = min(nsplit, ceil_div(K, tile));
  nsplit = max(nsplit, 1);
  // ... as long as all of the clusters are resident at once: where they would
  // need a second wave, the splits go through the workspace and the combine
  // kernel instead, one wave of as many splits as the SMs allow
  p.cluster = true;
  if (nsplit > 1 && nsplit <= cmax && sparse_attn_tc_cluster_capacity(nsplit) < ctas) {
    nsplit = ctas >= sms ? 1 : sms / ctas;
    nsplit = max(1, min(nsplit, ceil_div(K, tile)));
    p.cluster = false;
  }
  p.split_len = ceil_div(ceil_div(K, nsplit), tile) * tile;
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
                               float* lse, void* workspace, int* err, cudaStream_t stream,
                               const SwaWindow* swa, bool q_ready) {
  const int rows = B * Tq;
  if (rows == 0) return cudaSuccess;
  // the window's entries follow the selected ones in each row's entry list
  SplitPlan p = plan_splits(rows, Hq, K + (swa ? swa->W : 0));
  float* ws_o = nullptr;
  float2* ws_ml = nullptr;
  if (p.nsplit > 1) {
    size_t slots = (size_t)rows * p.nhb * p.nsplit;
    ws_o = static_cast<float*>(workspace);
    ws_ml = reinterpret_cast<float2*>(ws_o + slots * kHB * kD);
  }
  bool merged = false;
  cudaError_t e = launch_sparse_attn_tc(q, kv_packed, kv_scale, topk_idx, rows, Tq, Hq, N, K,
                                        softmax_scale, p.nhb, p.nsplit, p.split_len, out, lse,
                                        ws_o, ws_ml, err, stream, p.cluster ? &merged : nullptr,
                                        swa, q_ready);
  if (e != cudaSuccess || p.nsplit == 1 || merged) return e;
  return launch_pdl(attn_combine_kernel, dim3(rows, Hq), dim3(128), 0, stream, dim3(1), ws_o,
                    ws_ml, Hq, p.nhb, p.nsplit, out, lse);
}

}  // namespace csa2
