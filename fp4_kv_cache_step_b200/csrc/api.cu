// api.cu -- the exported C ABI of libcsa2_fp4 (declared in include/csa2.h):
// argument checks, the per-device error word, workspace planning and the
// FULL / REINDEX / REUSE layer-step dispatcher.
//
// Modes: "Detailed Notes On DeepSeek V4 Point 1 Flash In Simple Words",
// section "The Three Modes Full Reindex And Reuse", and the mengman.github.io
// interpretation, section 3.3 (mode table) and 3.4 (hierarchical indexer):
// FULL indexes for itself; REINDEX reuses the main KV and indexer keys but
// scores with its own indexer query, optionally only inside the candidate pool
// the first FULL layer kept; REUSE takes the latest top-K unchanged. The modes
// only choose which kernels run; the shared buffers are passed by pointer.
#include <cstdarg>
#include <cstdio>
#include <mutex>
#include <string>

#include "common.cuh"
#include "kernels.h"

namespace {

thread_local std::string g_last_error;

// First device-side data error per device (0 = none).
__device__ int g_device_error;

csa2_status fail(csa2_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

csa2_status cuda_fail(cudaError_t e, const char* where) {
  return fail(CSA2_ERR_CUDA, "%s: CUDA error %d (%s)", where, (int)e, cudaGetErrorString(e));
}

csa2_status ok() {
  g_last_error.clear();
  return CSA2_OK;
}

// Enters the stream's device and returns its error word (looked up once per
// device, with that device current).
int* device_error_word(cudaStream_t stream, csa2::DeviceScope& scope, cudaError_t* e_out) {
  static std::mutex mu;
  static int* words[128] = {};
  cudaError_t e = scope.enter(stream);
  const int dev = scope.device();
  if (e != cudaSuccess || dev < 0 || dev >= 128) {
    *e_out = e != cudaSuccess ? e : cudaErrorInvalidDevice;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (!words[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_device_error);
    if (e != cudaSuccess) {
      *e_out = e;
      return nullptr;
    }
    words[dev] = static_cast<int*>(p);
  }
  *e_out = cudaSuccess;
  return words[dev];
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr size_t kAlign = 256;
size_t round_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

#define CHECK_ARG(cond, ...) \
  do {                        \
    if (!(cond)) return fail(CSA2_ERR_INVALID_ARG, __VA_ARGS__); \
  } while (0)

#define CHECK_PTR(p) CHECK_ARG((p) != nullptr && aligned16(p), "%s must be a non-null 16-byte aligned device pointer", #p)

csa2_status check_kv(const void* kv_packed, const void* kv_scale, int B, int N, int D) {
  CHECK_PTR(kv_packed);
  CHECK_PTR(kv_scale);
  CHECK_ARG(B >= 0 && N >= 0, "B=%d and N=%d must be >= 0", B, N);
  CHECK_ARG(N % csa2::kBlockEntries == 0, "N=%d must be a multiple of 64", N);
  CHECK_ARG(D > 0 && D % 32 == 0, "D=%d must be a positive multiple of 32", D);
  return CSA2_OK;
}

// The 16-channel layout: rows of D/2 + D/16 bytes; D % 128 == 0 keeps every
// row 8-byte aligned (the kernels store a group's codes as one 8-byte word).
csa2_status check_kv_g16(const void* kv_rows, int B, int N, int D) {
  CHECK_PTR(kv_rows);
  CHECK_ARG(B >= 0 && N >= 0, "B=%d and N=%d must be >= 0", B, N);
  CHECK_ARG(D > 0 && D % 128 == 0, "D=%d must be a positive multiple of 128", D);
  return CSA2_OK;
}

csa2_status check_score_args(const uint8_t* idx_q, const float* idx_w, const uint8_t* idx_k,
                             int B, int Tq, int N, int Hi, int Di, const int32_t* nvalid,
                             const int32_t* cand, int C) {
  CHECK_PTR(idx_q);
  CHECK_PTR(idx_w);
  CHECK_PTR(idx_k);
  CHECK_ARG(B >= 0 && Tq >= 0 && N >= 0, "B, Tq, N must be >= 0");
  CHECK_ARG(B <= 65535 && Tq <= 65535, "B=%d and Tq=%d must be <= 65535", B, Tq);
  CHECK_ARG(Hi >= 1 && Hi <= 128, "Hi=%d must be in [1, 128]", Hi);
  CHECK_ARG(Di >= 16 && Di <= 256 && Di % 16 == 0, "Di=%d must be a multiple of 16 in [16, 256]", Di);
  if (cand) {
    CHECK_PTR(cand);
    CHECK_ARG(C >= 1, "C=%d must be >= 1 with a candidate pool", C);
  } else {
    CHECK_PTR(nvalid);
  }
  return CSA2_OK;
}

csa2_status check_attn_args(const uint16_t* q, const uint8_t* kv_packed, const uint8_t* kv_scale,
                            const int32_t* topk_idx, int B, int Tq, int Hq, int D, int N, int K,
                            const uint16_t* out, const float* lse) {
  csa2_status s = check_kv(kv_packed, kv_scale, B, N, D);
  if (s != CSA2_OK) return s;
  CHECK_PTR(q);
  CHECK_PTR(topk_idx);
  CHECK_PTR(out);
  if (lse) CHECK_ARG(((uintptr_t)lse & 3u) == 0, "lse must be 4-byte aligned");
  CHECK_ARG(Tq >= 0, "Tq=%d must be >= 0", Tq);
  CHECK_ARG(Hq >= 1 && Hq <= 65535, "Hq=%d must be in [1, 65535]", Hq);
  CHECK_ARG(K >= 1, "K=%d must be >= 1", K);
  if (D != csa2::kHeadDim)
    return fail(CSA2_ERR_UNSUPPORTED, "attention is built for D=512 only (got D=%d)", D);
  return CSA2_OK;
}

// Attention over the 16-channel layout (kv_rows) or the block layout.
csa2_status check_attn_any(const uint16_t* q, const uint8_t* kv_packed, const uint8_t* kv_scale,
                           const int32_t* topk_idx, int B, int Tq, int Hq, int D, int N, int K,
                           const uint16_t* out, const float* lse) {
  if (kv_scale != nullptr)
    return check_attn_args(q, kv_packed, kv_scale, topk_idx, B, Tq, Hq, D, N, K, out, lse);
  csa2_status s = check_kv_g16(kv_packed, B, N, D);
  if (s != CSA2_OK) return s;
  CHECK_PTR(q);
  CHECK_PTR(topk_idx);
  CHECK_PTR(out);
  if (lse) CHECK_ARG(((uintptr_t)lse & 3u) == 0, "lse must be 4-byte aligned");
  CHECK_ARG(Tq >= 0, "Tq=%d must be >= 0", Tq);
  CHECK_ARG(Hq >= 1 && Hq <= 65535, "Hq=%d must be in [1, 65535]", Hq);
  CHECK_ARG(K >= 1, "K=%d must be >= 1", K);
  if (D != csa2::kHeadDim)
    return fail(CSA2_ERR_UNSUPPORTED, "attention is built for D=512 only (got D=%d)", D);
  return CSA2_OK;
}

size_t layer_scores_bytes(const csa2_layer_args* a, csa2_mode mode, const csa2_shared_state* st) {
  if (mode == CSA2_MODE_REUSE) return 0;
  const bool pooled = mode == CSA2_MODE_REINDEX && a->use_pool;
  const size_t ld = pooled ? (size_t)st->C : (size_t)a->N;
  return round_up((size_t)a->B * a->Tq * ld * sizeof(float));
}

}  // namespace

// Internal helpers shared with the other exported entry points' files.
namespace csa2 {
csa2_status api_check_attn_args(const uint16_t* q, const uint8_t* kv_packed,
                                const uint8_t* kv_scale, const int32_t* topk_idx, int B, int Tq,
                                int Hq, int D, int N, int K, const uint16_t* out, const float* lse) {
  return check_attn_args(q, kv_packed, kv_scale, topk_idx, B, Tq, Hq, D, N, K, out, lse);
}
int* api_error_word(cudaStream_t stream, DeviceScope& scope, cudaError_t* e) {
  return device_error_word(stream, scope, e);
}
csa2_status api_fail(csa2_status s, const char* msg) { return fail(s, "%s", msg); }
csa2_status api_cuda_fail(cudaError_t e, const char* where) { return cuda_fail(e, where); }
csa2_status api_ok() { return ok(); }
}  // namespace csa2

extern "C" {

csa2_status fp4_kv_pack(const float* kv, int B, int N, int D, uint8_t* kv_packed,
                        uint8_t* kv_scale, csa2_stream_t stream) {
  CHECK_PTR(kv);
  csa2_status s = check_kv(kv_packed, kv_scale, B, N, D);
  if (s != CSA2_OK) return s;
  cudaError_t e;
  csa2::DeviceScope scope;
  int* err = device_error_word((cudaStream_t)stream, scope, &e);
  if (!err) return cuda_fail(e, "fp4_kv_pack");
  e = csa2::launch_fp4_pack(kv, B, N, D, kv_packed, kv_scale, err, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "fp4_kv_pack launch");
  return ok();
}

csa2_status fp4_kv_unpack(const uint8_t* kv_packed, const uint8_t* kv_scale, int B, int N, int D,
                          float* out, csa2_stream_t stream) {
  CHECK_PTR(out);
  csa2_status s = check_kv(kv_packed, kv_scale, B, N, D);
  if (s != CSA2_OK) return s;
  csa2::DeviceScope scope;
  cudaError_t e = scope.enter((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "fp4_kv_unpack device");
  e = csa2::launch_fp4_unpack(kv_packed, kv_scale, B, N, D, out, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "fp4_kv_unpack launch");
  return ok();
}

csa2_status fp4_kv_pack_g16(const float* kv, int B, int N, int D, uint8_t* kv_rows,
                            csa2_stream_t stream) {
  CHECK_PTR(kv);
  csa2_status s = check_kv_g16(kv_rows, B, N, D);
  if (s != CSA2_OK) return s;
  cudaError_t e;
  csa2::DeviceScope scope;
  int* err = device_error_word((cudaStream_t)stream, scope, &e);
  if (!err) return cuda_fail(e, "fp4_kv_pack_g16");
  e = csa2::launch_fp4_pack_g16(kv, nullptr, B, N, N, D, kv_rows, err, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "fp4_kv_pack_g16 launch");
  return ok();
}

csa2_status fp4_kv_unpack_g16(const uint8_t* kv_rows, int B, int N, int D, float* out,
                              csa2_stream_t stream) {
  CHECK_PTR(out);
  csa2_status s = check_kv_g16(kv_rows, B, N, D);
  if (s != CSA2_OK) return s;
  csa2::DeviceScope scope;
  cudaError_t e = scope.enter((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "fp4_kv_unpack_g16 device");
  e = csa2::launch_fp4_unpack_g16(kv_rows, B, N, D, out, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "fp4_kv_unpack_g16 launch");
  return ok();
}

csa2_status fp4_kv_append_g16(const float* kv_new, const int32_t* pos, int B, int T, int N, int D,
                              uint8_t* kv_rows, csa2_stream_t stream) {
  CHECK_PTR(kv_new);
  CHECK_PTR(pos);
  CHECK_ARG(T >= 0, "T=%d must be >= 0", T);
  csa2_status s = check_kv_g16(kv_rows, B, N, D);
  if (s != CSA2_OK) return s;
  cudaError_t e;
  csa2::DeviceScope scope;
  int* err = device_error_word((cudaStream_t)stream, scope, &e);
  if (!err) return cuda_fail(e, "fp4_kv_append_g16");
  e = csa2::launch_fp4_pack_g16(kv_new, pos, B, T, N, D, kv_rows, err, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "fp4_kv_append_g16 launch");
  return ok();
}

csa2_status csa2_index_score(const uint8_t* idx_q, const float* idx_w, const uint8_t* idx_k,
                             int B, int Tq, int N, int Hi, int Di, const int32_t* nvalid,
                             const int32_t* cand, int C, float* scores, csa2_stream_t stream) {
  CHECK_PTR(scores);
  csa2_status s = check_score_args(idx_q, idx_w, idx_k, B, Tq, N, Hi, Di, nvalid, cand, C);
  if (s != CSA2_OK) return s;
  cudaError_t e;
  csa2::DeviceScope scope;
  int* err = device_error_word((cudaStream_t)stream, scope, &e);
  if (!err) return cuda_fail(e, "csa2_index_score");
  e = csa2::launch_index_score(idx_q, idx_w, idx_k, B, Tq, N, Hi, Di, nvalid, cand, cand ? C : 0,
                               scores, err, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "csa2_index_score launch");
  return ok();
}

csa2_status csa2_topk(const float* scores, int ld, const int32_t* nvalid, const int32_t* cand,
                      int B, int Tq, int K, int32_t* topk_idx, int Cout, int32_t* cand_out,
                      csa2_stream_t stream) {
  CHECK_PTR(scores);
  CHECK_PTR(topk_idx);
  CHECK_ARG(B >= 0 && Tq >= 0, "B=%d and Tq=%d must be >= 0", B, Tq);
  CHECK_ARG(ld >= 0 && ld <= (1 << 30), "ld=%d must be in [0, 2^30]", ld);
  CHECK_ARG(K >= 1 && K <= 65536, "K=%d must be in [1, 65536]", K);
  if (cand) CHECK_PTR(cand); else CHECK_PTR(nvalid);
  if (cand_out) {
    CHECK_PTR(cand_out);
    CHECK_ARG(Cout >= 1 && Cout <= 65536, "Cout=%d must be in [1, 65536]", Cout);
  }
  cudaError_t e;
  csa2::DeviceScope scope;
  int* err = device_error_word((cudaStream_t)stream, scope, &e);
  if (!err) return cuda_fail(e, "csa2_topk");
  e = csa2::launch_topk(scores, ld, cand ? nullptr : nvalid, cand, B * Tq, K, topk_idx,
                        cand_out ? Cout : 0, cand_out, err, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "csa2_topk launch");
  return ok();
}

size_t csa2_sparse_attn_workspace_bytes(int B, int Tq, int Hq, int D, int K) {
  (void)D;
  if (B <= 0 || Tq <= 0 || Hq <= 0 || K <= 0) return 0;
  return round_up(csa2::sparse_attn_workspace_bytes(B, Tq, Hq, K));
}

csa2_status csa2_sparse_attn(const uint16_t* q, const uint8_t* kv_packed, const uint8_t* kv_scale,
                             const int32_t* topk_idx, int B, int Tq, int Hq, int D, int N, int K,
                             float softmax_scale, uint16_t* out, float* lse, void* workspace,
                             size_t workspace_bytes, csa2_stream_t stream) {
  csa2_status s = check_attn_args(q, kv_packed, kv_scale, topk_idx, B, Tq, Hq, D, N, K, out, lse);
  if (s != CSA2_OK) return s;
  // the workspace is sized on the stream's device, as the launch plans it
  // (with no device at all, for 148 SMs, so that the check still runs)
  csa2::DeviceScope scope;
  const cudaError_t se = scope.enter((cudaStream_t)stream);
  const size_t need = csa2_sparse_attn_workspace_bytes(B, Tq, Hq, D, K);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need || !aligned16(workspace)))
    return fail(CSA2_ERR_WORKSPACE, "csa2_sparse_attn needs %zu workspace bytes (got %zu)", need,
                workspace_bytes);
  if (se != cudaSuccess) return cuda_fail(se, "csa2_sparse_attn device");
  cudaError_t e;
  int* err = device_error_word((cudaStream_t)stream, scope, &e);
  if (!err) return cuda_fail(e, "csa2_sparse_attn");
  e = csa2::launch_sparse_attn(q, kv_packed, kv_scale, topk_idx, B, Tq, Hq, N, K, softmax_scale,
                               out, lse, workspace, err, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "csa2_sparse_attn launch");
  return ok();
}

csa2_status csa2_sparse_attn_g16(const uint16_t* q, const uint8_t* kv_rows,
                                 const int32_t* topk_idx, int B, int Tq, int Hq, int D, int N,
                                 int K, float softmax_scale, uint16_t* out, float* lse,
                                 void* workspace, size_t workspace_bytes, csa2_stream_t stream) {
  csa2_status s = check_attn_any(q, kv_rows, nullptr, topk_idx, B, Tq, Hq, D, N, K, out, lse);
  if (s != CSA2_OK) return s;
  csa2::DeviceScope scope;
  const cudaError_t se = scope.enter((cudaStream_t)stream);
  const size_t need = csa2_sparse_attn_workspace_bytes(B, Tq, Hq, D, K);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need || !aligned16(workspace)))
    return fail(CSA2_ERR_WORKSPACE, "csa2_sparse_attn_g16 needs %zu workspace bytes (got %zu)",
                need, workspace_bytes);
  if (se != cudaSuccess) return cuda_fail(se, "csa2_sparse_attn_g16 device");
  cudaError_t e;
  int* err = device_error_word((cudaStream_t)stream, scope, &e);
  if (!err) return cuda_fail(e, "csa2_sparse_attn_g16");
  // a NULL block-scale array selects the 16-channel layout
  e = csa2::launch_sparse_attn(q, kv_rows, nullptr, topk_idx, B, Tq, Hq, N, K, softmax_scale, out,
                               lse, workspace, err, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "csa2_sparse_attn_g16 launch");
  return ok();
}

namespace {
csa2_status check_swa_args(const uint8_t* swa_kv, const int32_t* swa_n, int B, int Tw, int W,
                           int K) {
  CHECK_PTR(swa_kv);
  CHECK_ARG(swa_n != nullptr && ((uintptr_t)swa_n & 3u) == 0,
            "swa_n must be a non-null 4-byte aligned device pointer");
  CHECK_ARG(Tw >= 0 && (size_t)B * Tw <= ((size_t)1 << 40), "Tw=%d must be >= 0", Tw);
  CHECK_ARG(W >= 0 && W <= 65536, "W=%d must be in [0, 65536]", W);
  CHECK_ARG((long long)K + W <= ((long long)1 << 30), "K + W must be <= 2^30");
  return CSA2_OK;
}
}  // namespace

csa2_status csa2_sparse_attn_swa(const uint16_t* q, const uint8_t* kv_packed,
                                 const uint8_t* kv_scale, const int32_t* topk_idx,
                                 const uint8_t* swa_kv, const int32_t* swa_n, int B, int Tq, int Hq,
                                 int D, int N, int K, int Tw, int W, float softmax_scale,
                                 uint16_t* out, float* lse, void* workspace,
                                 size_t workspace_bytes, csa2_stream_t stream) {
  csa2_status s = check_attn_any(q, kv_packed, kv_scale, topk_idx, B, Tq, Hq, D, N, K, out, lse);
  if (s != CSA2_OK) return s;
  s = check_swa_args(swa_kv, swa_n, B, Tw, W, K);
  if (s != CSA2_OK) return s;
  csa2::DeviceScope scope;
  const cudaError_t se = scope.enter((cudaStream_t)stream);
  const size_t need = csa2_sparse_attn_workspace_bytes(B, Tq, Hq, D, K + W);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need || !aligned16(workspace)))
    return fail(CSA2_ERR_WORKSPACE, "csa2_sparse_attn_swa needs %zu workspace bytes (got %zu)",
                need, workspace_bytes);
  if (se != cudaSuccess) return cuda_fail(se, "csa2_sparse_attn_swa device");
  cudaError_t e;
  int* err = device_error_word((cudaStream_t)stream, scope, &e);
  if (!err) return cuda_fail(e, "csa2_sparse_attn_swa");
  const csa2::SwaWindow win{swa_kv, swa_n, Tw, W};
  e = csa2::launch_sparse_attn(q, kv_packed, kv_scale, topk_idx, B, Tq, Hq, N, K, softmax_scale,
                               out, lse, workspace, err, (cudaStream_t)stream, &win);
  if (e != cudaSuccess) return cuda_fail(e, "csa2_sparse_attn_swa launch");
  return ok();
}

size_t csa2_block_pool_workspace_bytes(int B, int Tq, int ld, int block, int nblocks) {
  if (B <= 0 || Tq <= 0) return 0;
  return round_up(csa2::block_pool_workspace_bytes(B * Tq, ld, block, nblocks));
}

csa2_status csa2_block_pool(const float* scores, int ld, const int32_t* nvalid, int B, int Tq,
                            int block, int nblocks, int32_t* cand_out, void* workspace,
                            size_t workspace_bytes, csa2_stream_t stream) {
  CHECK_PTR(scores);
  CHECK_PTR(nvalid);
  CHECK_PTR(cand_out);
  CHECK_ARG(B >= 0 && Tq >= 0, "B=%d and Tq=%d must be >= 0", B, Tq);
  CHECK_ARG(ld >= 0 && ld <= (1 << 30), "ld=%d must be in [0, 2^30]", ld);
  CHECK_ARG(block >= 1 && nblocks >= 1 && nblocks <= 65536,
            "block=%d must be >= 1 and nblocks=%d in [1, 65536]", block, nblocks);
  CHECK_ARG((long long)block * nblocks <= (1 << 30), "block x nblocks must be <= 2^30");
  const size_t need = csa2_block_pool_workspace_bytes(B, Tq, ld, block, nblocks);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need || !aligned16(workspace)))
    return fail(CSA2_ERR_WORKSPACE, "csa2_block_pool needs %zu workspace bytes (got %zu)", need,
                workspace_bytes);
  cudaError_t e;
  csa2::DeviceScope scope;
  int* err = device_error_word((cudaStream_t)stream, scope, &e);
  if (!err) return cuda_fail(e, "csa2_block_pool");
  e = csa2::launch_block_pool(scores, ld, nvalid, B * Tq, block, nblocks, cand_out, workspace, err,
                              (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "csa2_block_pool launch");
  return ok();
}

// FULL with emit_pool == 2: the blockwise pool, blocks of 8, C / 8 of them
constexpr int kPoolBlock = 8;

static size_t layer_pool_bytes(const csa2_layer_args* a, csa2_mode mode,
                               const csa2_shared_state* st) {
  if (mode != CSA2_MODE_FULL || a->emit_pool != 2 || st->C < kPoolBlock) return 0;
  return csa2_block_pool_workspace_bytes(a->B, a->Tq, a->N, kPoolBlock, st->C / kPoolBlock);
}

size_t csa2_layer_step_workspace_bytes(const csa2_layer_args* a, csa2_mode mode,
                                       const csa2_shared_state* st) {
  if (!a || !st) return 0;
  // with a window, its W slots follow the K selected entries
  const int W = a->swa_kv ? a->W : 0;
  return layer_scores_bytes(a, mode, st) + layer_pool_bytes(a, mode, st) +
         csa2_sparse_attn_workspace_bytes(a->B, a->Tq, a->Hq, a->D, a->K + W);
}

csa2_status csa2_layer_step(const csa2_layer_args* a, csa2_mode mode, csa2_shared_state* st,
                            void* workspace, size_t workspace_bytes, csa2_stream_t stream) {
  CHECK_ARG(a != nullptr && st != nullptr, "args and shared state must be non-null");
  CHECK_ARG(mode == CSA2_MODE_FULL || mode == CSA2_MODE_REINDEX || mode == CSA2_MODE_REUSE,
            "unknown mode %d", (int)mode);
  // st->kv_scale NULL: st->kv_packed holds the 16-channel layout
  csa2_status s = check_attn_any(a->q, st->kv_packed, st->kv_scale, st->topk_idx, a->B, a->Tq,
                                 a->Hq, a->D, a->N, a->K, a->out, a->lse);
  if (s != CSA2_OK) return s;
  const bool pooled = mode == CSA2_MODE_REINDEX && a->use_pool;
  const bool emit = mode == CSA2_MODE_FULL && a->emit_pool;
  const bool emit_blocks = emit && a->emit_pool == 2;
  CHECK_ARG(a->emit_pool >= 0 && a->emit_pool <= 2, "emit_pool=%d must be 0, 1 or 2",
            a->emit_pool);
  if (mode != CSA2_MODE_REUSE) {
    s = check_score_args(a->idx_q, a->idx_w, st->idx_k, a->B, a->Tq, a->N, a->Hi, a->Di, a->nvalid,
                         pooled ? st->cand_idx : nullptr, st->C);
    if (s != CSA2_OK) return s;
    CHECK_PTR(a->nvalid);
    if (pooled || emit) {
      CHECK_PTR(st->cand_idx);
      CHECK_ARG(st->C >= 1 && st->C <= 65536, "pool size C=%d must be in [1, 65536]", st->C);
    }
    if (emit && !emit_blocks)
      CHECK_ARG(st->C >= a->K, "pool size C=%d must be >= K=%d", st->C, a->K);
    if (emit_blocks)
      CHECK_ARG(st->C % kPoolBlock == 0 && st->C / kPoolBlock >= a->K,
                "a blockwise pool needs C=%d a multiple of 8 with C/8 >= K=%d", st->C, a->K);
  }
  if (a->swa_kv) {
    s = check_swa_args(a->swa_kv, a->swa_n, a->B, a->Tw, a->W, a->K);
    if (s != CSA2_OK) return s;
  }
  csa2::DeviceScope scope;
  const cudaError_t se = scope.enter((cudaStream_t)stream);
  const size_t need = csa2_layer_step_workspace_bytes(a, mode, st);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need || !aligned16(workspace)))
    return fail(CSA2_ERR_WORKSPACE, "csa2_layer_step needs %zu workspace bytes (got %zu)", need,
                workspace_bytes);
  if (se != cudaSuccess) return cuda_fail(se, "csa2_layer_step device");
  cudaError_t e;
  int* err = device_error_word((cudaStream_t)stream, scope, &e);
  if (!err) return cuda_fail(e, "csa2_layer_step");
  cudaStream_t cs = (cudaStream_t)stream;
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  const size_t scores_bytes = layer_scores_bytes(a, mode, st);
  const size_t pool_bytes = layer_pool_bytes(a, mode, st);
  if (mode != CSA2_MODE_REUSE) {
    float* scores = reinterpret_cast<float*>(ws);
    const int ld = pooled ? st->C : a->N;
    e = csa2::launch_index_score(a->idx_q, a->idx_w, st->idx_k, a->B, a->Tq, a->N, a->Hi, a->Di,
                                 a->nvalid, pooled ? st->cand_idx : nullptr, pooled ? st->C : 0,
                                 scores, err, cs);
    if (e != cudaSuccess) return cuda_fail(e, "csa2_layer_step score");
    const bool emit_entries = emit && !emit_blocks;
    e = csa2::launch_topk(scores, ld, pooled ? nullptr : a->nvalid, pooled ? st->cand_idx : nullptr,
                          a->B * a->Tq, a->K, st->topk_idx, emit_entries ? st->C : 0,
                          emit_entries ? st->cand_idx : nullptr, err, cs);
    if (e != cudaSuccess) return cuda_fail(e, "csa2_layer_step top-k");
    if (emit_blocks) {
      e = csa2::launch_block_pool(scores, a->N, a->nvalid, a->B * a->Tq, kPoolBlock,
                                  st->C / kPoolBlock, st->cand_idx, ws + scores_bytes, err, cs);
      if (e != cudaSuccess) return cuda_fail(e, "csa2_layer_step block pool");
    }
  }
  const csa2::SwaWindow win{a->swa_kv, a->swa_n, a->Tw, a->W};
  e = csa2::launch_sparse_attn(a->q, st->kv_packed, st->kv_scale, st->topk_idx, a->B, a->Tq, a->Hq,
                               a->N, a->K, a->softmax_scale, a->out, a->lse,
                               ws ? ws + scores_bytes + pool_bytes : nullptr, err, cs,
                               a->swa_kv ? &win : nullptr,
                               // FULL / REINDEX: two kernels of this call precede
                               // the attention, so the caller's query is complete
                               mode != CSA2_MODE_REUSE);
  if (e != cudaSuccess) return cuda_fail(e, "csa2_layer_step attention");
  return ok();
}

csa2_status csa2_check_device_errors(csa2_stream_t stream) {
  csa2::DeviceScope scope;   // the error word of the stream's device
  cudaError_t e = scope.enter((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "csa2_check_device_errors device");
  e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "csa2_check_device_errors sync");
  int code = 0, zero = 0;
  e = cudaMemcpyFromSymbol(&code, g_device_error, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "csa2_check_device_errors read");
  if (code != 0) {
    e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e, "csa2_check_device_errors clear");
    return fail((csa2_status)code, "device reported error code %d", code);
  }
  return ok();
}

const char* csa2_last_error(void) { return g_last_error.c_str(); }

}  // extern "C"
