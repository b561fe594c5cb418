// noalloc.cu -- csa2_sparse_attn_noalloc: sparse attention for callers that
// cannot allocate device memory.
//
// csa2_sparse_attn needs caller-provided scratch whenever the index list is
// split across CTAs (few query rows). Some callers have no way to provide it:
// code that runs where cudaMalloc is not allowed or not wanted (inside an engine
// that owns and pre-partitions all device memory, in a custom-op hook that
// exposes no allocator, or on a latency-critical path that must not pay for an
// allocation or its implicit synchronisation). This variant takes the same
// inputs and outputs but keeps the split scratch in a fixed device array that
// lives in this file's module (loaded only when this entry point is first used)
// and stays resident on every device that used it until the process exits.
//
// Rules that follow from the shared array:
//  - the array holds kNoAllocScratchBytes; calls whose split scratch would be
//    larger are rejected with CSA2_ERR_WORKSPACE before anything is launched;
//  - every call on a device uses the same array, so calls that overlap on the
//    GPU (for example on two streams at once) race and must not be issued;
//  - the array keeps the previous call's contents; nothing in it has to start
//    at zero because every split writes its partial result before the merge
//    reads it;
//  - the first call on each device looks up the array's device address (a
//    host-side symbol query that may load this module), so make that first
//    call outside any stream capture;
//  - the call runs on the device its stream belongs to, which it makes current
//    for the lookup and the launch (the caller's current device is restored);
//  - under CUDA's lazy module loading (the default since CUDA 12) the array is
//    reserved on a device when this module is first used there; with
//    CUDA_MODULE_LOADING=EAGER every context that loads the library reserves
//    it, whether or not this entry point is ever called.
// No cudaMalloc, cudaFree or allocating library routine is called.
#include <mutex>
#include <string>

#include "common.cuh"
#include "kernels.h"

namespace {

constexpr size_t kNoAllocScratchBytes = CSA2_NOALLOC_SCRATCH_BYTES;

// The scratch itself. In host code this name is only a stand-in for the
// symbol: its device address must be fetched with cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch on device `dev`, which must be current
// (looked up once per device).
void* scratch_address(int dev, cudaError_t* e_out) {
  static std::mutex mu;
  static void* addr[128] = {};
  if (dev < 0 || dev >= 128) {
    *e_out = cudaErrorInvalidDevice;
    return nullptr;
  }
  cudaError_t e;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) {
      *e_out = e;
      return nullptr;
    }
    addr[dev] = p;
  }
  *e_out = cudaSuccess;
  return addr[dev];
}

}  // namespace

extern "C" {

csa2_status csa2_sparse_attn_noalloc(const uint16_t* q, const uint8_t* kv_packed,
                                     const uint8_t* kv_scale, const int32_t* topk_idx, int B,
                                     int Tq, int Hq, int D, int N, int K, float softmax_scale,
                                     uint16_t* out, float* lse, csa2_stream_t stream) {
  csa2_status s = csa2::api_check_attn_args(q, kv_packed, kv_scale, topk_idx, B, Tq, Hq, D, N, K,
                                            out, lse);
  if (s != CSA2_OK) return s;
  // the stream's device is current from here on: the split plan, and with it
  // the scratch size, follows its SM count
  csa2::DeviceScope scope;
  const cudaError_t se = scope.enter((cudaStream_t)stream);
  const size_t need = csa2_sparse_attn_workspace_bytes(B, Tq, Hq, D, K);
  if (need > kNoAllocScratchBytes) {
    std::string msg = "csa2_sparse_attn_noalloc: this shape needs " + std::to_string(need) +
                      " bytes of split scratch but the built-in array holds " +
                      std::to_string(kNoAllocScratchBytes) +
                      "; use csa2_sparse_attn with a caller workspace";
    return csa2::api_fail(CSA2_ERR_WORKSPACE, msg.c_str());
  }
  if (se != cudaSuccess) return csa2::api_cuda_fail(se, "csa2_sparse_attn_noalloc device");
  cudaError_t e;
  int* err = csa2::api_error_word((cudaStream_t)stream, scope, &e);
  if (!err) return csa2::api_cuda_fail(e, "csa2_sparse_attn_noalloc");
  void* scratch = nullptr;
  if (need > 0) {
    scratch = scratch_address(scope.device(), &e);
    if (!scratch) return csa2::api_cuda_fail(e, "csa2_sparse_attn_noalloc scratch address");
  }
  e = csa2::launch_sparse_attn(q, kv_packed, kv_scale, topk_idx, B, Tq, Hq, N, K, softmax_scale,
                               out, lse, scratch, err, (cudaStream_t)stream);
  if (e != cudaSuccess) return csa2::api_cuda_fail(e, "csa2_sparse_attn_noalloc launch");
  return csa2::api_ok();
}

}  // extern "C"
