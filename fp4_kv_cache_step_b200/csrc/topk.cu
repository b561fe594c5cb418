// topk.cu -- top-K selection for the CSA2 indexer.
//
// "Detailed Notes On DeepSeek V4 Point 1 Flash In Simple Words", section
// "Compressed Sparse Attention 2 Or CSA2 In Simple Terms": the indexer keeps
// the top entries for attention; the mengman.github.io interpretation, section
// 3.4: the first FULL layer also keeps a larger candidate pool that later
// REINDEX layers score inside. The pages fix no tie rule; the ranking here is
// (score descending, entry id ascending), and the selected ids are emitted in
// ascending order, padded with -1.
//
// One CTA per (b, t) row. Scores become order-preserving 32-bit keys (key 0 is
// reserved for "not a candidate"), an MSB-first 8-bit radix select finds the
// K-th key T and how many entries equal to T are still needed, and an ordered
// compaction writes every entry above T plus the first needed entries equal to
// T, in id order. Rows that fit are staged once in shared memory.
#include "common.cuh"
#include "kernels.h"

namespace csa2 {
namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kSmemKeyCap = 48 * 1024;   // 192 KB of staged keys

struct Scratch {
  uint32_t hist[256];
  int warp_sum[kWarps];
  int bcast[4];
};

// Exclusive prefix sum over the block; returns this thread's prefix and the
// block total through `total`.
__device__ __forceinline__ int block_exclusive_scan(int v, int& total, Scratch& sc) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int u = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += u;
  }
  if (lane == 31) sc.warp_sum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = sc.warp_sum[lane];
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int u = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += u;
    }
    sc.warp_sum[lane] = wi - w;   // exclusive
    if (lane == 31) sc.bcast[3] = wi;
  }
  __syncthreads();
  int res = sc.warp_sum[warp] + incl - v;
  total = sc.bcast[3];
  __syncthreads();
  return res;
}

struct Row {
  const float* s;       // scores of this row
  const int32_t* cand;  // candidate ids (pool mode) or null
  const uint32_t* keys; // staged keys in shared memory or null
  int n;                // entries in the row
};

__device__ __forceinline__ uint32_t key_at(const Row& r, int i, int* err) {
  if (r.keys) return r.keys[i];
  if (r.cand && r.cand[i] < 0) return 0u;
  bool nan = false;
  uint32_t k = rank_key(r.s[i], nan);
  if (nan) record_error(err, CSA2_ERR_NONFINITE);
  return k;
}

// Finds the key T of the k-th largest non-zero key (1 <= k <= number of
// non-zero keys) and how many entries equal to T belong to the selection.
__device__ void radix_select(const Row& r, int k, uint32_t& T, int& need_eq, Scratch& sc,
                             int* err) {
  uint32_t prefix = 0, mask = 0;
  int krem = k;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = threadIdx.x; i < 256; i += kThreads) sc.hist[i] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < r.n; i += kThreads) {
      uint32_t key = key_at(r, i, err);
      bool match = key != 0u && (key & mask) == prefix;
      uint32_t digit = (key >> shift) & 0xffu;
      // aggregate equal digits within the warp before touching shared memory
      uint32_t peers = __match_any_sync(__activemask(), match ? digit : 0x100u);
      if (match && (__ffs(peers) - 1) == (threadIdx.x & 31))
        atomicAdd(&sc.hist[digit], (uint32_t)__popc(peers));
    }
    __syncthreads();
    int v = threadIdx.x < 256 ? (int)sc.hist[255 - threadIdx.x] : 0;
    int total;
    int excl = block_exclusive_scan(v, total, sc);
    if (threadIdx.x < 256 && excl < krem && krem <= excl + v) {
      sc.bcast[0] = 255 - threadIdx.x;
      sc.bcast[1] = krem - excl;
    }
    __syncthreads();
    prefix |= (uint32_t)sc.bcast[0] << shift;
    mask |= 0xffu << shift;
    krem = sc.bcast[1];
    __syncthreads();
  }
  T = prefix;
  need_eq = krem;
}

// Writes, in ascending id order, every entry with key > T plus the first
// `need_eq` entries with key == T, then pads with -1 up to `k`.
__device__ void ordered_emit(const Row& r, uint32_t T, int need_eq, int k, int32_t* out,
                             Scratch& sc, int* err) {
  const int per = ceil_div(r.n, kThreads);
  const int i0 = min(r.n, threadIdx.x * per), i1 = min(r.n, i0 + per);
  int n_eq = 0;
  for (int i = i0; i < i1; ++i) n_eq += key_at(r, i, err) == T ? 1 : 0;
  int tot;
  const int eq_before = block_exclusive_scan(n_eq, tot, sc);
  int n_sel = 0, eq_seen = eq_before;
  for (int i = i0; i < i1; ++i) {
    uint32_t key = key_at(r, i, err);
    if (key > T) ++n_sel;
    else if (key == T && key != 0u && eq_seen++ < need_eq) ++n_sel;
  }
  int written;
  int pos = block_exclusive_scan(n_sel, written, sc);
  eq_seen = eq_before;
  for (int i = i0; i < i1; ++i) {
    uint32_t key = key_at(r, i, err);
    bool take = key > T || (key == T && key != 0u && eq_seen++ < need_eq);
    if (take) out[pos++] = r.cand ? r.cand[i] : i;
  }
  for (int i = written + threadIdx.x; i < k; i += kThreads) out[i] = -1;
}

__device__ void select_into(const Row& r, int n_valid, int k, int32_t* out, Scratch& sc,
                            int* err) {
  uint32_t T = 0;
  int need_eq = 0;
  if (n_valid > k) radix_select(r, k, T, need_eq, sc, err);
  ordered_emit(r, T, need_eq, k, out, sc, err);
}

template <bool kStage>
__global__ void __launch_bounds__(kThreads, 1)
topk_kernel(const float* __restrict__ scores, int ld, const int32_t* __restrict__ nvalid,
            const int32_t* __restrict__ cand, int K, int32_t* __restrict__ topk_out, int Cout,
            int32_t* __restrict__ cand_out, int* err) {
  extern __shared__ uint32_t staged[];
  __shared__ Scratch sc;
  const size_t row = blockIdx.x;
  Row r;
  r.s = scores + row * ld;
  r.cand = cand ? cand + row * ld : nullptr;
  r.keys = nullptr;
  r.n = cand ? ld : max(0, min(ld, nvalid[row]));

  // count the real candidates (and stage their keys); check the pool's order
  int mine = 0;
  bool nan = false, unsorted = false;
  for (int i = threadIdx.x; i < r.n; i += kThreads) {
    uint32_t key;
    if (r.cand) {
      int32_t id = r.cand[i];
      if (i > 0 && id >= 0 && (r.cand[i - 1] < 0 || r.cand[i - 1] >= id)) unsorted = true;
      key = id < 0 ? 0u : rank_key(r.s[i], nan);
    } else {
      key = rank_key(r.s[i], nan);
    }
    if (kStage) staged[i] = key;
    mine += key != 0u;
  }
  if (nan) record_error(err, CSA2_ERR_NONFINITE);
  if (unsorted) record_error(err, CSA2_ERR_DEVICE_INDEX);
  int n_valid;
  block_exclusive_scan(mine, n_valid, sc);   // also a barrier for the staged keys
  if (kStage) r.keys = staged;

  select_into(r, n_valid, K, topk_out + row * K, sc, err);
  if (cand_out) select_into(r, n_valid, Cout, cand_out + row * Cout, sc, err);
}

}  // namespace

cudaError_t launch_topk(const float* scores, int ld, const int32_t* nvalid, const int32_t* cand,
                        int rows, int K, int32_t* topk_idx, int Cout, int32_t* cand_out,
                        int* err, cudaStream_t stream) {
  if (rows == 0) return cudaSuccess;
  if (ld <= kSmemKeyCap) {
    size_t smem = (size_t)ld * sizeof(uint32_t);
    cudaError_t e = cudaFuncSetAttribute(topk_kernel<true>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    topk_kernel<true><<<rows, kThreads, smem, stream>>>(scores, ld, nvalid, cand, K, topk_idx,
                                                        Cout, cand_out, err);
  } else {
    topk_kernel<false><<<rows, kThreads, 0, stream>>>(scores, ld, nvalid, cand, K, topk_idx, Cout,
                                                      cand_out, err);
  }
  return cudaGetLastError();
}

}  // namespace csa2
