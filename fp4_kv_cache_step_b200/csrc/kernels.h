// kernels.h -- internal launchers behind the C ABI (not exported).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <utility>

#include "csa2.h"

namespace csa2 {

// Launches `kernel` with programmatic dependent launch (see
// pdl_wait_and_release) and, when cluster.x * y * z > 1, a cluster shape.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, dim3 cluster, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  int n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cluster.x * cluster.y * cluster.z > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster.x;
    attr[n].val.clusterDim.y = cluster.y;
    attr[n].val.clusterDim.z = cluster.z;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Makes the device a stream belongs to current for the rest of an entry point
// (restoring the caller's current device on exit), so that the error word, any
// built-in scratch and every launch belong to the stream's device. The legacy
// and per-thread default streams belong to the current device. Entering again
// for the same stream changes nothing (the caller's device stays the one
// restored).
class DeviceScope {
 public:
  DeviceScope() = default;
  DeviceScope(const DeviceScope&) = delete;
  DeviceScope& operator=(const DeviceScope&) = delete;
  ~DeviceScope() {
    if (prev_ >= 0) cudaSetDevice(prev_);
  }
  cudaError_t enter(cudaStream_t s) {
    int cur = 0;
    cudaError_t e = cudaGetDevice(&cur);
    if (e != cudaSuccess) return e;
    int dev = cur;
    if (s != nullptr && s != cudaStreamLegacy && s != cudaStreamPerThread) {
      e = cudaStreamGetDevice(s, &dev);
      if (e != cudaSuccess) return e;
    }
    if (dev != cur) {
      e = cudaSetDevice(dev);
      if (e != cudaSuccess) return e;
      prev_ = cur;
    }
    dev_ = dev;
    return cudaSuccess;
  }
  int device() const { return dev_; }

 private:
  int prev_ = -1;
  int dev_ = 0;
};

// Argument checks, error word and last-error text of api.cu, for entry points
// that live in other files.
csa2_status api_check_attn_args(const uint16_t* q, const uint8_t* kv_packed,
                                const uint8_t* kv_scale, const int32_t* topk_idx, int B, int Tq,
                                int Hq, int D, int N, int K, const uint16_t* out, const float* lse);
// Enters the stream's device (see DeviceScope) and returns that device's error
// word, or nullptr with *e set.
int* api_error_word(cudaStream_t stream, DeviceScope& scope, cudaError_t* e);
csa2_status api_fail(csa2_status s, const char* msg);
csa2_status api_cuda_fail(cudaError_t e, const char* where);
csa2_status api_ok();

cudaError_t launch_fp4_pack(const float* kv, int B, int N, int D, uint8_t* packed,
                            uint8_t* scale, int* err, cudaStream_t stream);
cudaError_t launch_fp4_unpack(const uint8_t* packed, const uint8_t* scale, int B, int N, int D,
                              float* out, cudaStream_t stream);
// The 16-channel layout: rows [B][N][D/2 + D/16]. Entry t of row b of kv
// ([B][T][D]) is quantised into cache row pos[b][t] (pos NULL: row t, T = N).
cudaError_t launch_fp4_pack_g16(const float* kv, const int32_t* pos, int B, int T, int N, int D,
                                uint8_t* rows, int* err, cudaStream_t stream);
cudaError_t launch_fp4_unpack_g16(const uint8_t* rows, int B, int N, int D, float* out,
                                  cudaStream_t stream);

// Indexer scores; see csa2_index_score for the contract.
cudaError_t launch_index_score(const uint8_t* idx_q, const float* idx_w, const uint8_t* idx_k,
                               int B, int Tq, int N, int Hi, int Di, const int32_t* nvalid,
                               const int32_t* cand, int C, float* scores, int* err,
                               cudaStream_t stream);

// Tensor-core scorer (score_tc.cu): full scans with Hi in {64, 128}, Di in {64, 128}.
bool index_score_tc_supported(int B, int Tq, int Hi, int Di, const int32_t* cand);
cudaError_t launch_index_score_tc(const uint8_t* idx_q, const float* idx_w, const uint8_t* idx_k,
                                  int B, int Tq, int N, int Hi, int Di, const int32_t* nvalid,
                                  float* scores, int* err, cudaStream_t stream);

// Top-K (and optional second, larger selection) per row; see csa2_topk.
cudaError_t launch_topk(const float* scores, int ld, const int32_t* nvalid, const int32_t* cand,
                        int rows, int K, int32_t* topk_idx, int Cout, int32_t* cand_out,
                        int* err, cudaStream_t stream);

// Blockwise candidate pool (pool.cu); see csa2_block_pool.
size_t block_pool_workspace_bytes(int rows, int ld, int block, int nblocks);
cudaError_t launch_block_pool(const float* scores, int ld, const int32_t* nvalid, int rows,
                              int block, int nblocks, int32_t* cand, void* workspace, int* err,
                              cudaStream_t stream);

// The sliding-window branch (csa2_sparse_attn_swa): window memory kv
// [B][Tw][D] E4M3, one row per token, serving as key and value; query row
// (b, t) also attends tokens [max(0, n[b][t] - W), n[b][t]). The kernels treat
// the window as W more entries after the K selected ones.
struct SwaWindow {
  const uint8_t* kv;
  const int32_t* n;
  int Tw, W;
};

// The blockwise pool of blocks of 8 in one launch of the register top-K (true
// when it applied; *e holds the launch status).
bool launch_block_pool_reg(const float* scores, int ld, const int32_t* nvalid, int rows,
                           int block, int nblocks, int32_t* cand, int* err, cudaStream_t stream,
                           cudaError_t* e);

// Sparse attention; see csa2_sparse_attn. With kv_scale NULL, kv_packed holds
// the 16-channel layout (csa2_sparse_attn_g16): per entry D/2 code bytes then
// D/16 E4M3 scale bytes. With swa non-null the window branch joins the same
// softmax; the workspace is then sized for K + swa->W entries. q_ready: the
// query was complete before the kernel that precedes this one on the stream
// started, so it may be read before the wait for that kernel.
size_t sparse_attn_workspace_bytes(int B, int Tq, int Hq, int K);
cudaError_t launch_sparse_attn(const uint16_t* q, const uint8_t* kv_packed,
                               const uint8_t* kv_scale, const int32_t* topk_idx, int B, int Tq,
                               int Hq, int N, int K, float softmax_scale, uint16_t* out,
                               float* lse, void* workspace, int* err, cudaStream_t stream,
                               const SwaWindow* swa = nullptr, bool q_ready = false);

// Tensor-core attention kernel (attn_tc.cu). With nsplit > 1 the splits are
// merged inside the kernel (thread-block clusters, *merged set to true) when
// `merged` is non-null and the cluster fits; otherwise partials go to
// ws_o/ws_ml for attn_combine_kernel.
int sparse_attn_tc_tile();
int sparse_attn_tc_max_cluster();   // splits of a row that merge inside one cluster
// how many clusters of `cs` splits can be resident at once on the current
// device (a large number when no device can be asked)
int sparse_attn_tc_cluster_capacity(int cs);
cudaError_t launch_sparse_attn_tc(const uint16_t* q, const uint8_t* kv_packed,
                                  const uint8_t* kv_scale, const int32_t* topk_idx, int rows,
                                  int Tq, int Hq, int N, int K, float softmax_scale, int nhb,
                                  int nsplit, int split_len, uint16_t* out, float* lse,
                                  float* ws_o, float2* ws_ml, int* err, cudaStream_t stream,
                                  bool* merged, const SwaWindow* swa = nullptr,
                                  bool q_ready = false);

}  // namespace csa2
