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
// reserved for "not a candidate"). The row's key range [kmin, kmax] is cut into
// 4096 equal power-of-two bins (so the histogram adapts to where the scores
// actually lie), a suffix scan finds the bin holding the K-th key, and the few
// keys of that bin are ranked exactly against each other. A crowded threshold
// bin (many equal scores) falls back to an MSB-first 8-bit radix select. The
// selection is written in id order by a two-pass, ballot-based compaction.
// Rows that fit are staged once in shared memory. Rows of up to 32768 keys take
// the register variant at the end of this file.
#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels.h"

namespace csa2 {
namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kBins = 4096;
constexpr int kBinsPerThread = kBins / kThreads;
constexpr int kCandCap = 512;            // exact in-bin ranking up to this many keys
constexpr int kSmemKeyCap = 40 * 1024;   // 160 KB of staged keys

struct Scratch {
  uint32_t hist[256];
  int warp_sum[kWarps];
  int bcast[4];
  int bins[kBins];
  uint32_t cand_key[kCandCap];
  int cand_pos[kCandCap];
  int wgt[kWarps], weq[kWarps];
  uint32_t red_min[kWarps], red_max[kWarps];
  int ncand;
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

constexpr int kBatch = 8;   // independent loads in flight per thread

// Keys at positions base + stride * j (j < kBatch); 0 past `end`.
__device__ __forceinline__ void keys_batch(const Row& r, int base, int stride, int end,
                                           uint32_t (&k)[kBatch], int* err) {
  if (r.keys) {
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const int i = base + stride * j;
      k[j] = i < end ? r.keys[i] : 0u;
    }
    return;
  }
  float f[kBatch];
  int32_t c[kBatch];
#pragma unroll
  for (int j = 0; j < kBatch; ++j) {
    const int i = base + stride * j;
    f[j] = i < end ? __ldg(r.s + i) : 0.0f;
    c[j] = (r.cand && i < end) ? __ldg(r.cand + i) : 0;
  }
  bool nan = false;
#pragma unroll
  for (int j = 0; j < kBatch; ++j) {
    const int i = base + stride * j;
    k[j] = (i < end && c[j] >= 0) ? rank_key(f[j], nan) : 0u;
  }
  if (nan) record_error(err, CSA2_ERR_NONFINITE);
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
    // the loop bound is warp-uniform so every lane reaches __match_any_sync
    const int lane = threadIdx.x & 31;
    for (int w0 = threadIdx.x - lane; w0 < r.n; w0 += kThreads * kBatch) {
      uint32_t kb[kBatch];
      keys_batch(r, w0 + lane, kThreads, r.n, kb, err);
#pragma unroll
      for (int j = 0; j < kBatch; ++j) {
        const uint32_t key = kb[j];
        const bool match = key != 0u && (key & mask) == prefix;
        const uint32_t digit = (key >> shift) & 0xffu;
        // aggregate equal digits within the warp before touching shared memory
        const uint32_t peers = __match_any_sync(0xffffffffu, match ? digit : 0x100u);
        if (match && (__ffs(peers) - 1) == (threadIdx.x & 31))
          atomicAdd(&sc.hist[digit], (uint32_t)__popc(peers));
      }
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
// `need_eq` entries with key == T (T = 0 selects every real entry), then pads
// with -1 up to `k`. Warp w owns a contiguous segment of the row; pass 1 counts,
// pass 2 writes with ballot prefix counts.
__device__ void ordered_emit(const Row& r, uint32_t T, int need_eq, int k, int32_t* out,
                             Scratch& sc, int* err) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int seg = ceil_div(ceil_div(r.n, kWarps), 32) * 32;
  const int w0 = min(r.n, warp * seg), w1 = min(r.n, w0 + seg);
  const uint32_t lt_mask = (1u << lane) - 1u;
  int cnt_gt = 0, cnt_eq = 0;
  for (int base = w0; base < w1; base += 32 * kBatch) {
    uint32_t kb[kBatch];
    keys_batch(r, base + lane, 32, w1, kb, err);
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      cnt_gt += __popc(__ballot_sync(0xffffffffu, kb[j] > T));
      cnt_eq += __popc(__ballot_sync(0xffffffffu, kb[j] == T && kb[j] != 0u));
    }
  }
  if (lane == 0) {
    sc.wgt[warp] = cnt_gt;
    sc.weq[warp] = cnt_eq;
  }
  __syncthreads();
  int eq_before = 0, pos = 0, total = 0;
  {
    int eqb = 0;
    for (int w = 0; w < kWarps; ++w) {
      const int sel = sc.wgt[w] + min(sc.weq[w], max(0, need_eq - eqb));
      if (w < warp) {
        pos += sel;
        eq_before += sc.weq[w];
      }
      total += sel;
      eqb += sc.weq[w];
    }
  }
  int eq_seen = eq_before;
  for (int base = w0; base < w1; base += 32 * kBatch) {
    uint32_t kb[kBatch];
    keys_batch(r, base + lane, 32, w1, kb, err);
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const int i = base + lane + 32 * j;
      const uint32_t key = kb[j];
      const bool eq = key == T && key != 0u;
      const uint32_t eqmask = __ballot_sync(0xffffffffu, eq);
      const bool take = key > T || (eq && eq_seen + __popc(eqmask & lt_mask) < need_eq);
      const uint32_t tmask = __ballot_sync(0xffffffffu, take);
      if (take) out[pos + __popc(tmask & lt_mask)] = r.cand ? r.cand[i] : i;
      pos += __popc(tmask);
      eq_seen += __popc(eqmask);
    }
  }
  for (int i = total + threadIdx.x; i < k; i += kThreads) out[i] = -1;
  __syncthreads();
}

struct Range {
  uint32_t kmin;
  int shift;
};

__device__ __forceinline__ int bin_of(uint32_t key, Range rg) {
  return (int)((key - rg.kmin) >> rg.shift);
}

// Histogram of the real keys over kBins bins of the row's key range.
__device__ void build_hist(const Row& r, Range rg, Scratch& sc, int* err) {
  for (int i = threadIdx.x; i < kBins; i += kThreads) sc.bins[i] = 0;
  __syncthreads();
  for (int i0 = threadIdx.x; i0 < r.n; i0 += kThreads * kBatch) {
    uint32_t kb[kBatch];
    keys_batch(r, i0, kThreads, r.n, kb, err);
#pragma unroll
    for (int j = 0; j < kBatch; ++j)
      if (kb[j] != 0u) atomicAdd(&sc.bins[bin_of(kb[j], rg)], 1);
  }
  __syncthreads();
}

// Finds (T, need_eq) for the k-th largest real key, 1 <= k <= n_valid.
__device__ void find_threshold(const Row& r, Range rg, int k, uint32_t& T, int& need_eq,
                               Scratch& sc, int* err) {
  // bins in descending order: thread t owns bins kBins-1-4t .. kBins-4-4t
  int local[kBinsPerThread];
  int mine = 0;
#pragma unroll
  for (int j = 0; j < kBinsPerThread; ++j) {
    local[j] = sc.bins[kBins - 1 - kBinsPerThread * threadIdx.x - j];
    mine += local[j];
  }
  int tot;
  int above = block_exclusive_scan(mine, tot, sc);
  if (above < k && k <= above + mine) {
#pragma unroll
    for (int j = 0; j < kBinsPerThread; ++j) {
      if (above < k && k <= above + local[j]) {
        sc.bcast[0] = kBins - 1 - kBinsPerThread * (int)threadIdx.x - j;
        sc.bcast[1] = k - above;   // how many to take from the bin
        sc.bcast[2] = local[j];
      }
      above += local[j];
    }
  }
  if (threadIdx.x == 0) sc.ncand = 0;
  __syncthreads();
  const int bT = sc.bcast[0], rT = sc.bcast[1], cT = sc.bcast[2];
  if (cT > kCandCap) {
    // crowded bin: exact radix select over the whole row
    radix_select(r, k, T, need_eq, sc, err);
    return;
  }
  for (int i0 = threadIdx.x; i0 < r.n; i0 += kThreads * kBatch) {
    uint32_t kb[kBatch];
    keys_batch(r, i0, kThreads, r.n, kb, err);
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      if (kb[j] != 0u && bin_of(kb[j], rg) == bT) {
        const int slot = atomicAdd(&sc.ncand, 1);
        if (slot < kCandCap) {
          sc.cand_key[slot] = kb[j];
          sc.cand_pos[slot] = i0 + kThreads * j;
        }
      }
    }
  }
  __syncthreads();
  const int c = min(sc.ncand, kCandCap);
  for (int s = threadIdx.x; s < c; s += kThreads) {
    const uint32_t ks = sc.cand_key[s];
    const int ps = sc.cand_pos[s];
    int gt = 0, eqb = 0;
    for (int u = 0; u < c; ++u) {
      const uint32_t ku = sc.cand_key[u];
      gt += ku > ks;
      eqb += (ku == ks) && (sc.cand_pos[u] < ps);
    }
    if (gt + eqb == rT - 1) {
      sc.bcast[0] = (int)ks;
      sc.bcast[1] = eqb + 1;
    }
  }
  __syncthreads();
  T = (uint32_t)sc.bcast[0];
  need_eq = sc.bcast[1];
  __syncthreads();
}

__device__ void select_into(const Row& r, int n_valid, Range rg, bool& hist_ready, int k,
                            int32_t* out, Scratch& sc, int* err) {
  uint32_t T = 0;
  int need_eq = 0;
  if (n_valid > k) {
    if (!hist_ready) {
      build_hist(r, rg, sc, err);
      hist_ready = true;
    }
    find_threshold(r, rg, k, T, need_eq, sc, err);
  }
  ordered_emit(r, T, need_eq, k, out, sc, err);
}

template <bool kStage>
__global__ void __launch_bounds__(kThreads, 1)
topk_kernel(const float* __restrict__ scores, int ld, const int32_t* __restrict__ nvalid,
            const int32_t* __restrict__ cand, int K, int32_t* __restrict__ topk_out, int Cout,
            int32_t* __restrict__ cand_out, int* err) {
  extern __shared__ uint32_t staged[];
  __shared__ Scratch sc;
  pdl_wait_and_release();
  const size_t row = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  Row r;
  r.s = scores + row * ld;
  r.cand = cand ? cand + row * ld : nullptr;
  r.keys = nullptr;
  r.n = cand ? ld : max(0, min(ld, nvalid[row]));

  // stage the keys; count the real ones and find their range; check the pool's order
  int mine = 0;
  uint32_t kmin = 0xffffffffu, kmax = 0u;
  bool unsorted = false;
  for (int i0 = threadIdx.x; i0 < r.n; i0 += kThreads * kBatch) {
    uint32_t kb[kBatch];
    keys_batch(r, i0, kThreads, r.n, kb, err);
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const int i = i0 + kThreads * j;
      if (i >= r.n) break;
      if (r.cand && i > 0) {
        const int32_t id = __ldg(r.cand + i), prev = __ldg(r.cand + i - 1);
        if (id >= 0 && (prev < 0 || prev >= id)) unsorted = true;
      }
      if (kStage) staged[i] = kb[j];
      if (kb[j] != 0u) {
        ++mine;
        kmin = min(kmin, kb[j]);
        kmax = max(kmax, kb[j]);
      }
    }
  }
  if (unsorted) record_error(err, CSA2_ERR_DEVICE_INDEX);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
    kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
  }
  if (lane == 0) {
    sc.red_min[warp] = kmin;
    sc.red_max[warp] = kmax;
  }
  int n_valid;
  block_exclusive_scan(mine, n_valid, sc);   // also a barrier for the staged keys
  if (kStage) r.keys = staged;
  Range rg;
  kmin = sc.red_min[0];
  kmax = sc.red_max[0];
  for (int w = 1; w < kWarps; ++w) {
    kmin = min(kmin, sc.red_min[w]);
    kmax = max(kmax, sc.red_max[w]);
  }
  rg.kmin = kmin;
  const uint32_t span = kmax >= kmin ? kmax - kmin : 0u;   // largest offset
  const int bits = span == 0u ? 0 : 32 - __clz(span);      // offsets fit in `bits` bits
  rg.shift = bits > 12 ? bits - 12 : 0;                    // -> at most 4096 bins
  bool hist_ready = false;

  select_into(r, n_valid, rg, hist_ready, K, topk_out + row * K, sc, err);
  if (cand_out) select_into(r, n_valid, rg, hist_ready, Cout, cand_out + row * Cout, sc, err);
}


// ---------------------------------------------------------------------------
// Cluster variant: when there are too few rows to give every SM a CTA, each
// row is cut into `cs` contiguous slices, one per CTA of a thread-block
// cluster. Every CTA stages its slice's keys in shared memory; the CTAs agree
// on the threshold through histograms summed over distributed shared memory
// (12-bit digits refined from the row's key range down to the exact key T),
// then each writes its part of the ascending output at an offset given by the
// counts of the CTAs before it. Same ranking and output as topk_kernel.
namespace cg = cooperative_groups;

constexpr int kCThreads = 1024;
constexpr int kCWarps = kCThreads / 32;
constexpr int kCBins = 4096;                    // one 12-bit digit per pass
constexpr int kCBinsPerThread = kCBins / kCThreads;
static_assert(kCBinsPerThread == 4, "the cluster histogram is read as one uint4 per thread");

constexpr int kCCandCap = 512;                  // exact ranking of a threshold bin up to this size

struct __align__(16) ClusterShared {
  uint32_t hist[kCBins];      // this CTA's histogram of the current pass (read by the cluster)
  uint32_t cand_key[kCCandCap];   // this CTA's keys in the threshold bin (read by the cluster)
  int cand_pos[kCCandCap];        // and their positions in the row
  uint32_t all_key[kCCandCap];    // the threshold bin of the whole row
  int all_pos[kCCandCap];
  int ncand;
  uint32_t kmin, kmax;        // this CTA's key range
  int nvalid;                 // real keys in this CTA's slice
  int gt, eq;                 // keys > T and == T in this slice (emit)
  int warp_sum[kCWarps];
  int bcast[4];
};

__device__ __forceinline__ int cblock_exclusive_scan(int v, int& total, ClusterShared& sc) {
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
    sc.warp_sum[lane] = wi - w;
    if (lane == 31) sc.bcast[3] = wi;
  }
  __syncthreads();
  const int res = sc.warp_sum[warp] + incl - v;
  total = sc.bcast[3];
  __syncthreads();
  return res;
}

// (T, need_eq) of the k-th largest real key of the row (1 <= k <= n_valid):
// T is the key, need_eq how many keys equal to T the selection takes.
__device__ void cluster_threshold(cg::cluster_group& cl, const uint32_t* keys, int nloc, int i0,
                                  uint32_t kmin, uint32_t kmax, int k, uint32_t& T, int& need_eq,
                                  ClusterShared& sc) {
  const int cs = (int)cl.num_blocks();
  uint32_t lo = kmin;
  const uint32_t span = kmax - kmin;
  int bits = span == 0u ? 0 : 32 - __clz(span);   // offsets from lo fit in `bits` bits
  int shift = bits > 12 ? bits - 12 : 0;
  uint32_t width_m1 = span;                        // current range is [lo, lo + width_m1]
  int krem = k;
  const int lane = threadIdx.x & 31;
  for (;;) {
    for (int i = threadIdx.x; i < kCBins; i += kCThreads) sc.hist[i] = 0;
    __syncthreads();
    for (int w0 = threadIdx.x - lane; w0 < nloc; w0 += kCThreads) {
      const int i = w0 + lane;
      const uint32_t key = i < nloc ? keys[i] : 0u;
      const bool in = key != 0u && key - lo <= width_m1 && key >= lo;
      if (in) atomicAdd(&sc.hist[(key - lo) >> shift], 1u);
    }
    cl.sync();
    // bins in descending order: thread t owns bins kCBins-1-4t .. kCBins-4-4t,
    // read as one 16-byte vector from every CTA of the cluster (loads first)
    const int vb = kCBins - kCBinsPerThread * (threadIdx.x + 1);   // lowest of the four
    uint4 part[8];
#pragma unroll
    for (int r = 0; r < 8; ++r)
      if (r < cs) part[r] = *reinterpret_cast<const uint4*>(cl.map_shared_rank(&sc.hist[vb], r));
    int local[kCBinsPerThread] = {0, 0, 0, 0};
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      if (r < cs) {
        local[0] += (int)part[r].w;   // bin vb + 3 first: descending order
        local[1] += (int)part[r].z;
        local[2] += (int)part[r].y;
        local[3] += (int)part[r].x;
      }
    }
    const int mine = local[0] + local[1] + local[2] + local[3];
    int total;
    int above = cblock_exclusive_scan(mine, total, sc);
    if (above < krem && krem <= above + mine) {
#pragma unroll
      for (int j = 0; j < kCBinsPerThread; ++j) {
        if (above < krem && krem <= above + local[j]) {
          sc.bcast[0] = kCBins - 1 - kCBinsPerThread * (int)threadIdx.x - j;
          sc.bcast[1] = krem - above;
          sc.bcast[2] = local[j];
        }
        above += local[j];
      }
    }
    if (threadIdx.x == 0) sc.ncand = 0;
    __syncthreads();
    const uint32_t bstar = (uint32_t)sc.bcast[0];
    krem = sc.bcast[1];
    const int cbin = sc.bcast[2];
    lo += bstar << shift;
    if (shift == 0) {
      // every CTA has read the others' histograms before any clears its own
      cl.sync();
      T = lo;
      need_eq = krem;
      return;
    }
    if (cbin <= kCCandCap) {
      // few keys in the threshold bin: gather them from the whole cluster and
      // rank them exactly against each other (score desc, position asc)
      const uint32_t bw_m1 = (1u << shift) - 1u;
      for (int i = threadIdx.x; i < nloc; i += kCThreads) {
        const uint32_t key = keys[i];
        if (key != 0u && key >= lo && key - lo <= bw_m1) {
          const int slot = atomicAdd(&sc.ncand, 1);
          if (slot < kCCandCap) {
            sc.cand_key[slot] = key;
            sc.cand_pos[slot] = i0 + i;
          }
        }
      }
      cl.sync();   // candidate lists complete (and the histograms read)
      int off = 0, c = 0;
      for (int r = 0; r < cs; ++r) {
        ClusterShared* o = cl.map_shared_rank(&sc, r);
        const int nr = min(o->ncand, kCCandCap);
        for (int u = threadIdx.x; u < nr; u += kCThreads) {
          if (off + u < kCCandCap) {
            sc.all_key[off + u] = o->cand_key[u];
            sc.all_pos[off + u] = o->cand_pos[u];
          }
        }
        off += nr;
      }
      c = min(off, kCCandCap);
      __syncthreads();
      for (int u = threadIdx.x; u < c; u += kCThreads) {
        const uint32_t ku = sc.all_key[u];
        const int pu = sc.all_pos[u];
        int gt = 0, eqb = 0;
        for (int v = 0; v < c; ++v) {
          const uint32_t kv = sc.all_key[v];
          gt += kv > ku;
          eqb += (kv == ku) && (sc.all_pos[v] < pu);
        }
        if (gt + eqb == krem - 1) {
          sc.bcast[0] = (int)ku;
          sc.bcast[1] = eqb + 1;
        }
      }
      __syncthreads();
      T = (uint32_t)sc.bcast[0];
      need_eq = sc.bcast[1];
      // the candidate lists are read remotely: no CTA may rewrite its own
      // before all have gathered (the caller's next cluster barrier)
      return;
    }
    // every CTA has read the others' histograms before any clears its own
    cl.sync();
    width_m1 = (1u << shift) - 1u;
    shift = shift > 12 ? shift - 12 : 0;
  }
}

__global__ void __launch_bounds__(kCThreads, 1)
topk_cluster_kernel(const float* __restrict__ scores, int ld, const int32_t* __restrict__ nvalid,
                    const int32_t* __restrict__ cand, int K, int32_t* __restrict__ topk_out,
                    int Cout, int32_t* __restrict__ cand_out, int slice, int* err) {
  extern __shared__ uint32_t keys[];
  __shared__ ClusterShared sc;
  pdl_wait_and_release();
  cg::cluster_group cl = cg::this_cluster();
  const int cs = (int)cl.num_blocks();
  const int rank = (int)cl.block_rank();
  const size_t row = blockIdx.x / cs;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const float* srow = scores + row * ld;
  const int32_t* crow = cand ? cand + row * ld : nullptr;
  const int n = cand ? ld : max(0, min(ld, nvalid[row]));
  const int i0 = min(n, rank * slice), i1 = min(n, i0 + slice);
  const int nloc = i1 - i0;

  // stage this slice's keys (kBatch loads in flight per thread); count the real
  // ones and find their range
  int mine = 0;
  uint32_t kmin = 0xffffffffu, kmax = 0u;
  bool nan = false, unsorted = false;
  for (int b0 = threadIdx.x; b0 < nloc; b0 += kCThreads * kBatch) {
    float f[kBatch];
    int32_t id[kBatch], prev[kBatch];
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const int i = b0 + kCThreads * j;
      const int gi = i0 + i;
      f[j] = i < nloc ? __ldg(srow + gi) : 0.0f;
      id[j] = (crow && i < nloc) ? __ldg(crow + gi) : 0;
      prev[j] = (crow && i < nloc && gi > 0) ? __ldg(crow + gi - 1) : -1;
    }
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const int i = b0 + kCThreads * j;
      if (i >= nloc) break;
      if (crow && id[j] >= 0 && i0 + i > 0 && (prev[j] < 0 || prev[j] >= id[j])) unsorted = true;
      const uint32_t key = id[j] >= 0 ? rank_key(f[j], nan) : 0u;
      keys[i] = key;
      if (key != 0u) {
        ++mine;
        kmin = min(kmin, key);
        kmax = max(kmax, key);
      }
    }
  }
  if (nan) record_error(err, CSA2_ERR_NONFINITE);
  if (unsorted) record_error(err, CSA2_ERR_DEVICE_INDEX);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
    kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
    mine += __shfl_xor_sync(0xffffffffu, mine, o);
  }
  if (lane == 0) sc.warp_sum[warp] = mine;
  if (threadIdx.x == 0) {
    sc.kmin = 0xffffffffu;
    sc.kmax = 0u;
  }
  __syncthreads();
  if (lane == 0) {
    atomicMin(&sc.kmin, kmin);
    atomicMax(&sc.kmax, kmax);
  }
  if (threadIdx.x == 0) {
    int tot = 0;
    for (int w = 0; w < kCWarps; ++w) tot += sc.warp_sum[w];
    sc.nvalid = tot;
  }
  cl.sync();
  uint32_t gmin = 0xffffffffu, gmax = 0u;
  int n_valid = 0;
  for (int r = 0; r < cs; ++r) {
    ClusterShared* o = cl.map_shared_rank(&sc, r);
    gmin = min(gmin, o->kmin);
    gmax = max(gmax, o->kmax);
    n_valid += o->nvalid;
  }

  for (int pass = 0; pass < 2; ++pass) {
    const int k = pass == 0 ? K : Cout;
    int32_t* out = pass == 0 ? topk_out + row * (size_t)K : cand_out + row * (size_t)Cout;
    if (pass == 1 && cand_out == nullptr) break;
    uint32_t T = 0u;
    int need_eq = 0;
    if (n_valid > k) cluster_threshold(cl, keys, nloc, i0, gmin, gmax, k, T, need_eq, sc);
    // warp w takes a contiguous segment of the slice, its lanes interleaved
    const int seg = ceil_div(ceil_div(nloc, kCWarps), 32) * 32;
    const int w0 = min(nloc, warp * seg), w1 = min(nloc, w0 + seg);
    const uint32_t lt_mask = (1u << lane) - 1u;
    int cnt_gt = 0, cnt_eq = 0;
    for (int base = w0; base < w1; base += 32) {
      const int i = base + lane;
      const uint32_t key = i < w1 ? keys[i] : 0u;
      cnt_gt += __popc(__ballot_sync(0xffffffffu, key > T));
      cnt_eq += __popc(__ballot_sync(0xffffffffu, key == T && key != 0u));
    }
    int tot_gt, tot_eq;
    int gt_before_w = cblock_exclusive_scan(lane == 0 ? cnt_gt : 0, tot_gt, sc);
    int eq_before_w = cblock_exclusive_scan(lane == 0 ? cnt_eq : 0, tot_eq, sc);
    gt_before_w = __shfl_sync(0xffffffffu, gt_before_w, 0);
    eq_before_w = __shfl_sync(0xffffffffu, eq_before_w, 0);
    if (threadIdx.x == 0) {
      sc.gt = tot_gt;
      sc.eq = tot_eq;
    }
    cl.sync();
    int gt_before = 0, eq_before = 0;
    for (int r = 0; r < rank; ++r) {
      ClusterShared* o = cl.map_shared_rank(&sc, r);
      gt_before += o->gt;
      eq_before += o->eq;
    }
    // entries selected before this warp: all > T keys of earlier CTAs and
    // warps, and the first need_eq of the == T keys in order
    int eq_seen = eq_before + eq_before_w;
    int pos = gt_before + gt_before_w + min(eq_seen, need_eq);
    for (int base = w0; base < w1; base += 32) {
      const int i = base + lane;
      const uint32_t key = i < w1 ? keys[i] : 0u;
      const bool eq = key == T && key != 0u;
      const uint32_t eqmask = __ballot_sync(0xffffffffu, eq);
      const bool take = key > T || (eq && eq_seen + __popc(eqmask & lt_mask) < need_eq);
      const uint32_t tmask = __ballot_sync(0xffffffffu, take);
      if (take) {
        const int gi = i0 + i;
        out[pos + __popc(tmask & lt_mask)] = crow ? crow[gi] : gi;
      }
      pos += __popc(tmask);
      eq_seen += __popc(eqmask);
    }
    // padding: the last CTA of the cluster writes the -1 tail
    if (rank == cs - 1) {
      const int total = min(k, n_valid);
      for (int i = total + threadIdx.x; i < k; i += kCThreads) out[i] = -1;
    }
    // the counts are read remotely before the next pass overwrites them
    cl.sync();
  }
}

// ---------------------------------------------------------------------------
// Register variant. A row is split over a cluster of CS CTAs (CS = 1, 2, 4 or
// 8) of 512 threads; CTA r of the cluster covers positions r S .. r S + S - 1,
// S = 512 KPT (KPT a multiple of 4, at most 64). Warp w of a CTA covers 32 KPT
// consecutive positions of its slice; its lane l holds the 4-key chunks at
// w 32 KPT + 128 j + 4 l (j < KPT / 4), so every warp load is one coalesced
// 512-byte line set, and after that single pass over the scores every step
// works on registers and a few kilobytes of shared memory:
//   1. keys, their count and range [kmin, kmax] (block reductions, then the
//      cluster's ranges combined over distributed shared memory);
//   2. a 4096-bin histogram over that range per CTA (shared-memory atomics),
//      summed over the cluster, and a suffix scan to the bin holding the k-th
//      key; a crowded bin is refined with the next 12 bits of the key, down to
//      the key itself;
//   3. the few keys of the threshold bin, gathered from the cluster, ranked
//      exactly (score desc, index asc);
//   4. the ordered write: each CTA's (greater, equal) counts give the offset
//      of its slice, a block scan the offset of each warp, and per chunk row a
//      warp scan the slot of each lane's keys.
// Same ranking and output as the kernels above.

constexpr int kRThreads = 512;
constexpr int kRWarps = kRThreads / 32;
constexpr int kRBins = 4096;
constexpr int kRBinsPerThread = kRBins / kRThreads;
constexpr int kRCandCap = 1024;
constexpr int kRGroups = 64;                      // groups of 64 bins

struct __align__(16) RegShared {
  int bins[kRBins];                 // this CTA's histogram (fine bins read by the cluster)
  uint32_t all_key[kRCandCap];      // the whole row's threshold bin (written by every CTA)
  int all_pos[kRCandCap];
  // written by every CTA of the cluster into every CTA (slot = the writer's
  // rank), so that after a cluster barrier each CTA reads them locally
  int coarse[8][kRGroups];          // per rank: its counts of 64 groups of 64 bins (descending)
  uint32_t rng_min[8], rng_max[8];  // per rank: its key range and count of real keys
  int rng_cnt[8];
  uint32_t emit_from[2][8];         // per pass and rank: its (greater << 16 | equal) counts
  int rank_cnt[8];                  // per rank: its keys in the threshold bin
  int warp_a[kRWarps], warp_b[kRWarps];
  uint32_t red_min[kRWarps], red_max[kRWarps];
  int bcast[8];
  int ncand;
};

template <int CS>
__device__ __forceinline__ void csync(cg::cluster_group& cl) {
  if (CS > 1) cl.sync(); else __syncthreads();
}

template <int CS, typename T>
__device__ __forceinline__ T* at_rank(cg::cluster_group& cl, T* p, int r) {
  return CS > 1 ? cl.map_shared_rank(p, r) : p;
}

// position in the row of key (chunk j, element q) of this thread
template <int KPT>
__device__ __forceinline__ int reg_pos(int base, int j, int q) {
  return base + (int)(threadIdx.x >> 5) * 32 * KPT + 128 * j + 4 * (int)(threadIdx.x & 31) + q;
}

// Inclusive prefix sum over the 32 lanes of a warp.
__device__ __forceinline__ int warp_incl_scan(int v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += u;
  }
  return v;
}

// (T, need_eq) of the k-th largest real key of the row (1 <= k <= its real
// keys): T is the key, need_eq how many keys equal to T the selection takes.
// `reads_pending`: the cluster may still read this CTA's histogram or
// candidates from an earlier call.
// Per digit: each CTA counts its keys into 4096 bins over the current range
// and writes its 64 group counts (64 bins each, descending) into every CTA;
// after one cluster barrier warp 0 of each CTA finds, locally, the group that
// holds the k-th key, then reads that group's 64 bins from every CTA and finds
// the bin.
template <int KPT, int CS>
__device__ void reg_threshold(cg::cluster_group& cl, const uint32_t (&key)[KPT], int base,
                              uint32_t kmin, uint32_t kmax, int k, bool reads_pending,
                              uint32_t& T, int& need_eq, RegShared& sc) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rank = CS > 1 ? (int)cl.block_rank() : 0;
  uint32_t lo = kmin;
  uint32_t width_m1 = kmax - kmin;                 // range [lo, lo + width_m1]
  const int bits = width_m1 == 0u ? 0 : 32 - __clz(width_m1);
  int shift = bits > 12 ? bits - 12 : 0;
  int krem = k;
  bool first = true;
  for (;;) {
    // nobody still reads our histogram or our group counts
    if (CS > 1 && (reads_pending || !first)) cl.sync();
    for (int i = threadIdx.x; i < kRBins; i += kRThreads) sc.bins[i] = 0;
    if (threadIdx.x == 0) sc.ncand = 0;
    __syncthreads();
    if (first) {
      // every real key lies in the range
#pragma unroll
      for (int j = 0; j < KPT; ++j)
        if (key[j] != 0u) atomicAdd(&sc.bins[(key[j] - lo) >> shift], 1);
    } else {
#pragma unroll
      for (int j = 0; j < KPT; ++j) {
        const uint32_t kk = key[j];
        if (kk != 0u && kk >= lo && kk - lo <= width_m1) atomicAdd(&sc.bins[(kk - lo) >> shift], 1);
      }
    }
    first = false;
    __syncthreads();
    {
      // thread t sums bins 4095 - 8t .. 4088 - 8t; 8 threads make group t / 8
      const int b0 = kRBins - kRBinsPerThread * ((int)threadIdx.x + 1);
      const int4 x = *reinterpret_cast<const int4*>(sc.bins + b0);
      const int4 y = *reinterpret_cast<const int4*>(sc.bins + b0 + 4);
      int s8 = x.x + x.y + x.z + x.w + y.x + y.y + y.z + y.w;
      s8 += __shfl_xor_sync(0xffffffffu, s8, 1);
      s8 += __shfl_xor_sync(0xffffffffu, s8, 2);
      s8 += __shfl_xor_sync(0xffffffffu, s8, 4);
      if ((lane & 7) == 0) {
        const int g = (int)threadIdx.x >> 3;
#pragma unroll
        for (int r = 0; r < CS; ++r) at_rank<CS>(cl, &sc.coarse[rank][g], r)[0] = s8;
      }
    }
    csync<CS>(cl);                                 // every CTA's group counts are everywhere
    if (warp == 0) {
      // groups 2 lane and 2 lane + 1, summed over the cluster
      int c0 = 0, c1 = 0;
#pragma unroll
      for (int r = 0; r < CS; ++r) {
        c0 += sc.coarse[r][2 * lane];
        c1 += sc.coarse[r][2 * lane + 1];
      }
      const int incl = warp_incl_scan(c0 + c1);
      const int before = incl - c0 - c1;
      int g = -1, kg = 0;
      if (before < krem && krem <= before + c0) {
        g = 2 * lane;
        kg = krem - before;
      } else if (before + c0 < krem && krem <= incl) {
        g = 2 * lane + 1;
        kg = krem - before - c0;
      }
      const uint32_t hit = __ballot_sync(0xffffffffu, g >= 0);
      const int src = hit ? __ffs(hit) - 1 : 0;      // exactly one lane holds the k-th key
      g = max(0, __shfl_sync(0xffffffffu, g, src));
      kg = __shfl_sync(0xffffffffu, kg, src);
      // its 64 bins, descending: bin top - 2 lane and top - 2 lane - 1
      const int top = kRBins - 1 - 64 * g;
      int f0 = 0, f1 = 0;
#pragma unroll
      for (int r = 0; r < CS; ++r) {
        const int* br = at_rank<CS>(cl, sc.bins, r);
        f0 += br[top - 2 * lane];
        f1 += br[top - 2 * lane - 1];
      }
      const int fi = warp_incl_scan(f0 + f1);
      const int fb = fi - f0 - f1;
      int win = -1;                                  // 0: bin top - 2 lane; 1: the next
      if (fb < kg && kg <= fb + f0) {
        sc.bcast[0] = top - 2 * lane;
        sc.bcast[1] = kg - fb;
        sc.bcast[2] = f0;
        win = 0;
      } else if (fb + f0 < kg && kg <= fi) {
        sc.bcast[0] = top - 2 * lane - 1;
        sc.bcast[1] = kg - fb - f0;
        sc.bcast[2] = f1;
        win = 1;
      }
      if (win >= 0) {
        // every CTA's count of the threshold bin: the offsets of their candidates
#pragma unroll
        for (int r = 0; r < CS; ++r) sc.rank_cnt[r] = at_rank<CS>(cl, sc.bins, r)[top - 2 * lane - win];
      }
    }
    __syncthreads();
    const uint32_t bstar = (uint32_t)sc.bcast[0];
    krem = sc.bcast[1];
    const int cbin = sc.bcast[2];
    lo += bstar << shift;
    if (shift == 0) {
      // the bin is a single key value
      T = lo;
      need_eq = krem;
      __syncthreads();
      return;
    }
    const uint32_t bw_m1 = (1u << shift) - 1u;
    if (cbin <= kRCandCap) {
      // the keys of the threshold bin, from the whole cluster, ranked exactly:
      // each CTA writes its own into every CTA's list, at the offset given by
      // the counts of the CTAs before it
      int off = 0;
#pragma unroll
      for (int r = 0; r < CS; ++r) off += r < rank ? sc.rank_cnt[r] : 0;
#pragma unroll
      for (int j = 0; j < KPT; ++j) {
        const uint32_t kk = key[j];
        if (kk != 0u && kk >= lo && kk - lo <= bw_m1) {
          const int slot = off + atomicAdd(&sc.ncand, 1);
          if (slot < kRCandCap) {
            const int pos = reg_pos<KPT>(base, j / 4, j % 4);
#pragma unroll
            for (int r = 0; r < CS; ++r) {
              RegShared* o = at_rank<CS>(cl, &sc, r);
              o->all_key[slot] = kk;
              o->all_pos[slot] = pos;
            }
          }
        }
      }
      csync<CS>(cl);                               // every CTA's candidates are everywhere
      const int c = min(cbin, kRCandCap);
      const uint32_t* ck = sc.all_key;
      const int* cp = sc.all_pos;
      for (int u = threadIdx.x; u < c; u += kRThreads) {
        const uint32_t ku = ck[u];
        const int pu = cp[u];
        int gt = 0, eqb = 0;
        for (int v = 0; v < c; ++v) {
          const uint32_t kv = ck[v];
          gt += kv > ku;
          eqb += (kv == ku) && (cp[v] < pu);
        }
        if (gt + eqb == krem - 1) {
          sc.bcast[0] = (int)ku;
          sc.bcast[1] = eqb + 1;
        }
      }
      __syncthreads();
      T = (uint32_t)sc.bcast[0];
      need_eq = sc.bcast[1];
      __syncthreads();
      return;
    }
    // crowded bin: the next 12 bits within it
    width_m1 = bw_m1;
    shift = shift > 12 ? shift - 12 : 0;
    __syncthreads();
  }
}

// Writes, in position order, every key above T and the first need_eq keys equal
// to T (T = 0 selects every real key), then pads with -1 up to k.
// kBlk > 0: a kept block b is written as positions kBlk b .. kBlk b + kBlk - 1
// (-1 from nv_pos on), and the padding covers kBlk slots per missing block.
template <int KPT, int CS, int kBlk>
__device__ void reg_emit(cg::cluster_group& cl, int rank, int pass, const uint32_t (&key)[KPT],
                         int base, uint32_t T, int need_eq, int k, int n_valid, int nv_pos,
                         const int32_t* crow, int32_t* out, RegShared& sc) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // (greater << 16 | equal) counts: a CTA's totals (at most 512 x 64) fit 16 bits each
  uint32_t c = 0;
#pragma unroll
  for (int j = 0; j < KPT; ++j) c += ((uint32_t)(key[j] > T) << 16) | (uint32_t)(key[j] == T && key[j] != 0u);
  const uint32_t wc = __reduce_add_sync(0xffffffffu, c);
  if (lane == 0) sc.warp_a[warp] = (int)wc;
  __syncthreads();
  if (warp == 0) {
    const uint32_t v = lane < kRWarps ? (uint32_t)sc.warp_a[lane] : 0u;
    uint32_t incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t u = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += u;
    }
    if (lane < kRWarps) sc.warp_b[lane] = (int)(incl - v);
    // this CTA's totals (lane 31's inclusive sum) into every later CTA
    const uint32_t total = __shfl_sync(0xffffffffu, incl, 31);
    if (lane < CS && lane > rank) at_rank<CS>(cl, &sc.emit_from[pass][rank], lane)[0] = total;
  }
  csync<CS>(cl);                                   // every CTA's counts are published
  // selected before this warp's first chunk row: the earlier CTAs' and warps'
  int gt_run = 0, eq_run = 0;
  for (int r = 0; r < rank; ++r) {
    const uint32_t e = sc.emit_from[pass][r];
    gt_run += (int)(e >> 16);
    eq_run += (int)(e & 0xffffu);
  }
  gt_run += (int)((uint32_t)sc.warp_b[warp] >> 16);
  eq_run += (int)((uint32_t)sc.warp_b[warp] & 0xffffu);
#pragma unroll
  for (int j = 0; j < KPT / 4; ++j) {
    uint32_t cj = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q)
      cj += ((uint32_t)(key[4 * j + q] > T) << 16) |
            (uint32_t)(key[4 * j + q] == T && key[4 * j + q] != 0u);
    uint32_t incl = cj;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t u = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += u;
    }
    const uint32_t tot = __shfl_sync(0xffffffffu, incl, 31);
    const uint32_t ex = incl - cj;
    int eq_seen = eq_run + (int)(ex & 0xffffu);
    int pos = gt_run + (int)(ex >> 16) + min(eq_seen, need_eq);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t kk = key[4 * j + q];
      bool take = kk > T;
      if (kk == T && kk != 0u) take = eq_seen++ < need_eq;
      if (take) {
        const int i = reg_pos<KPT>(base, j, q);
        if (kBlk == 8) {
          // the block's 8 positions as two 16-byte stores (rows and slots are
          // 32-byte aligned)
          const int j0 = i * 8;
          int4 lo4, hi4;
          lo4.x = j0 < nv_pos ? j0 : -1;
          lo4.y = j0 + 1 < nv_pos ? j0 + 1 : -1;
          lo4.z = j0 + 2 < nv_pos ? j0 + 2 : -1;
          lo4.w = j0 + 3 < nv_pos ? j0 + 3 : -1;
          hi4.x = j0 + 4 < nv_pos ? j0 + 4 : -1;
          hi4.y = j0 + 5 < nv_pos ? j0 + 5 : -1;
          hi4.z = j0 + 6 < nv_pos ? j0 + 6 : -1;
          hi4.w = j0 + 7 < nv_pos ? j0 + 7 : -1;
          int4* o4 = reinterpret_cast<int4*>(out + (size_t)pos * 8);
          o4[0] = lo4;
          o4[1] = hi4;
          ++pos;
        } else if (kBlk) {
#pragma unroll
          for (int e = 0; e < kBlk; ++e) {
            const int jj = i * kBlk + e;
            out[(size_t)pos * kBlk + e] = jj < nv_pos ? jj : -1;
          }
          ++pos;
        } else {
          out[pos++] = crow ? __ldg(crow + i) : i;
        }
      }
    }
    gt_run += (int)(tot >> 16);
    eq_run += (int)(tot & 0xffffu);
  }
  if (rank == CS - 1) {
    const int total = min(k, n_valid);
    const int per = kBlk ? kBlk : 1;
    for (int i = total * per + threadIdx.x; i < k * per; i += kRThreads) out[i] = -1;
  }
  __syncthreads();
}

// kBlk > 0 (blockwise pool): key slot b is block b, positions kBlk b ..
// kBlk b + kBlk - 1 of the row, keyed by the largest score among its valid
// positions (j < nvalid); a block with no valid position is not a candidate;
// each kept block is written as its kBlk positions (-1 past nvalid), blocks
// ascending, the pool -1 padded to K blocks.
template <int KPT, int CS, bool kPool, int kBlk>
__global__ void __launch_bounds__(kRThreads, 1)
topk_reg_kernel(const float* __restrict__ scores, int ld, const int32_t* __restrict__ nvalid,
                const int32_t* __restrict__ cand, int K, int32_t* __restrict__ topk_out,
                int Cout, int32_t* __restrict__ cand_out, int* err) {
  static_assert(KPT % 4 == 0 && KPT <= 64, "chunks of four keys, at most 64 per thread");
  __shared__ RegShared sc;
  // every CTA of the cluster must be running before any writes into another's
  // shared memory: arrive now, wait just before the first such write
  if (CS > 1) asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
  pdl_wait_and_release();
  cg::cluster_group cl = cg::this_cluster();
  const int rank = CS > 1 ? (int)cl.block_rank() : 0;
  const size_t row = blockIdx.x / CS;
  const int base = rank * kRThreads * KPT;          // first position of this CTA's slice
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float* srow = scores + row * ld;
  const int32_t* crow = kPool ? cand + row * ld : nullptr;
  // candidates: valid positions, or blocks holding one
  const int nv_pos = kPool ? ld : max(0, min(ld, nvalid[row]));
  const int n = kBlk ? (nv_pos + kBlk - 1) / kBlk : nv_pos;
  // Whole rows of 16-byte aligned, 4-key-divisible length take branch-free
  // 16-byte loads (chunks past the row end read its first chunk, masked below),
  // so all of a thread's loads are in flight together; other rows load keys one
  // by one.
  const bool vec = ld % 4 == 0 && ld >= 4 &&
                   ((reinterpret_cast<uintptr_t>(srow) | reinterpret_cast<uintptr_t>(crow)) & 15u) == 0;
  uint32_t key[KPT];
  int ids[kPool ? KPT : 1];
  if (kBlk) {
    // each block's maximum over its valid positions (a NaN is kept, to be flagged)
    const bool vec8 = kBlk % 4 == 0 && ld % 4 == 0 && (reinterpret_cast<uintptr_t>(srow) & 15u) == 0;
#pragma unroll
    for (int j = 0; j < KPT; ++j) {
      const int b = reg_pos<KPT>(base, j / 4, j % 4);
      float m = -INFINITY;
      bool isnan_b = false;
      if (b < n) {
        const int j0 = b * kBlk;
#pragma unroll
        for (int e = 0; e < kBlk; e += 4) {
          float v[4];
          if (vec8 && j0 + e + 4 <= ld) {
            const float4 x = __ldg(reinterpret_cast<const float4*>(srow + j0 + e));
            v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
          } else {
#pragma unroll
            for (int q = 0; q < 4; ++q) v[q] = (e + q < kBlk && j0 + e + q < ld) ? __ldg(srow + j0 + e + q) : 0.0f;
          }
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            if (e + q < kBlk && j0 + e + q < nv_pos) {
              isnan_b |= v[q] != v[q];
              m = fmaxf(m, v[q]);
            }
          }
        }
      }
      key[j] = isnan_b ? 0x7fc00000u : __float_as_uint(m);
    }
  } else if (vec) {
#pragma unroll
    for (int j = 0; j < KPT / 4; ++j) {
      const int p0 = reg_pos<KPT>(base, j, 0);
      const int pl = p0 < ld ? p0 : 0;
      const float4 v = __ldg(reinterpret_cast<const float4*>(srow + pl));
      key[4 * j] = __float_as_uint(v.x);
      key[4 * j + 1] = __float_as_uint(v.y);
      key[4 * j + 2] = __float_as_uint(v.z);
      key[4 * j + 3] = __float_as_uint(v.w);
      if (kPool) {
        const int4 cv = __ldg(reinterpret_cast<const int4*>(crow + pl));
        ids[4 * j] = cv.x;
        ids[4 * j + 1] = cv.y;
        ids[4 * j + 2] = cv.z;
        ids[4 * j + 3] = cv.w;
      }
    }
  } else {
#pragma unroll
    for (int j = 0; j < KPT; ++j) {
      const int p = reg_pos<KPT>(base, j / 4, j % 4);
      key[j] = p < n ? __float_as_uint(__ldg(srow + p)) : 0u;
      if (kPool) ids[j] = p < n ? __ldg(crow + p) : -1;
    }
  }
  uint64_t real = 0u;                  // bit 4 j + q: key (j, q) is a candidate
  bool unsorted = false;
  int prev_last = -1;                  // a pool's id at the position before the current chunk row
#pragma unroll
  for (int j = 0; j < KPT / 4; ++j) {
    const int p0 = reg_pos<KPT>(base, j, 0);
#pragma unroll
    for (int q = 0; q < 4; ++q)
      real |= (uint64_t)((p0 + q < n && (!kPool || ids[4 * j + q] >= 0)) ? 1u : 0u) << (4 * j + q);
    if (kPool) {
      // ids ascending: each real id exceeds the id before it, which is real; the
      // id before a chunk is the previous lane's last (lane 0: the last of lane
      // 31 in the previous chunk row, or before the warp's first, from memory)
      int prev = __shfl_up_sync(0xffffffffu, ids[4 * j + 3], 1);
      if (lane == 0) prev = j > 0 ? prev_last : ((p0 > 0 && p0 - 1 < n) ? __ldg(crow + p0 - 1) : -1);
      prev_last = __shfl_sync(0xffffffffu, ids[4 * j + 3], 31);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int id = ids[4 * j + q];
        if (p0 + q < n && id >= 0 && p0 + q > 0 && (prev < 0 || prev >= id)) unsorted = true;
        prev = id;
      }
    }
  }
  // order-preserving keys, branch-free: x ^ (sign ? ~0 : 0x80000000), -0 as +0,
  // NaN and non-candidates 0 (a NaN is reported)
  bool nan = false;
  int mine = 0;
  uint32_t kmin = 0xffffffffu, kmax = 0u;
#pragma unroll
  for (int j = 0; j < KPT; ++j) {
    const uint32_t u = key[j], a = u & 0x7fffffffu;
    const bool is_real = (real >> j) & 1u;
    const bool isnan = a > 0x7f800000u;
    nan |= isnan && is_real;
    uint32_t kk = a == 0u ? 0x80000000u : u ^ ((uint32_t)((int32_t)u >> 31) | 0x80000000u);
    kk = (isnan || !is_real) ? 0u : kk;
    key[j] = kk;
    mine += kk != 0u;
    kmin = min(kmin, kk == 0u ? 0xffffffffu : kk);
    kmax = max(kmax, kk);
  }
  if (nan) record_error(err, CSA2_ERR_NONFINITE);
  if (unsorted) record_error(err, CSA2_ERR_DEVICE_INDEX);
  kmin = __reduce_min_sync(0xffffffffu, kmin);
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  mine = __reduce_add_sync(0xffffffffu, mine);
  if (lane == 0) {
    sc.red_min[warp] = kmin;
    sc.red_max[warp] = kmax;
    sc.warp_a[warp] = mine;
  }
  __syncthreads();
  if (CS > 1) asm volatile("barrier.cluster.wait.aligned;" ::: "memory");   // all threads
  if (warp == 0) {
    const uint32_t a = __reduce_min_sync(0xffffffffu, lane < kRWarps ? sc.red_min[lane] : 0xffffffffu);
    const uint32_t b = __reduce_max_sync(0xffffffffu, lane < kRWarps ? sc.red_max[lane] : 0u);
    const int c = __reduce_add_sync(0xffffffffu, lane < kRWarps ? sc.warp_a[lane] : 0);
    // this CTA's range and count into every CTA of the cluster
    if (lane < CS) {
      at_rank<CS>(cl, &sc.rng_min[rank], lane)[0] = a;
      at_rank<CS>(cl, &sc.rng_max[rank], lane)[0] = b;
      at_rank<CS>(cl, &sc.rng_cnt[rank], lane)[0] = c;
    }
  }
  csync<CS>(cl);                                   // every CTA's range is everywhere
  kmin = 0xffffffffu;
  kmax = 0u;
  int n_valid = 0;
#pragma unroll
  for (int r = 0; r < CS; ++r) {
    kmin = min(kmin, sc.rng_min[r]);
    kmax = max(kmax, sc.rng_max[r]);
    n_valid += sc.rng_cnt[r];
  }
  for (int pass = 0; pass < 2; ++pass) {
    const int k = pass == 0 ? K : Cout;
    if (pass == 1 && cand_out == nullptr) break;
    int32_t* out = pass == 0 ? topk_out + row * (size_t)K * (kBlk ? kBlk : 1)
                             : cand_out + row * (size_t)Cout;
    uint32_t T = 0u;
    int need_eq = 0;
    if (n_valid > k)
      reg_threshold<KPT, CS>(cl, key, base, kmin, kmax, k, pass > 0, T, need_eq, sc);
    reg_emit<KPT, CS, kBlk>(cl, rank, pass, key, base, T, need_eq, k, n_valid, nv_pos, crow, out,
                            sc);
  }
  // Every access to another CTA's shared memory (the fine bins, the candidate
  // lists, and the values written into every CTA) precedes the last cluster
  // barrier in reg_emit, so a CTA may leave without waiting for the others.
}

template <int KPT, int CS, int kBlk>
cudaError_t launch_topk_reg(const float* scores, int ld, const int32_t* nvalid,
                            const int32_t* cand, int rows, int K, int32_t* topk_idx, int Cout,
                            int32_t* cand_out, int* err, cudaStream_t stream) {
  const dim3 grid((unsigned)(rows * CS)), cluster((unsigned)CS, 1, 1);
  if (cand != nullptr && kBlk == 0)
    return launch_pdl(topk_reg_kernel<KPT, CS, true, 0>, grid, dim3(kRThreads), 0, stream,
                      cluster, scores, ld, nvalid, cand, K, topk_idx, Cout, cand_out, err);
  return launch_pdl(topk_reg_kernel<KPT, CS, false, kBlk>, grid, dim3(kRThreads), 0, stream,
                    cluster, scores, ld, nvalid, cand, K, topk_idx, Cout, cand_out, err);
}

// `slots`: key slots per row (positions, or blocks in the block mode)
template <int CS, int kBlk>
cudaError_t launch_topk_reg_cs(const float* scores, int ld, int slots, const int32_t* nvalid,
                               const int32_t* cand, int rows, int K, int32_t* topk_idx, int Cout,
                               int32_t* cand_out, int* err, cudaStream_t stream) {
  const int per = ceil_div(ceil_div(max(slots, 1), CS), kRThreads);
  if (per <= 4)
    return launch_topk_reg<4, CS, kBlk>(scores, ld, nvalid, cand, rows, K, topk_idx, Cout,
                                        cand_out, err, stream);
  if (per <= 16)
    return launch_topk_reg<16, CS, kBlk>(scores, ld, nvalid, cand, rows, K, topk_idx, Cout,
                                         cand_out, err, stream);
  if constexpr (kBlk == 0)
    return launch_topk_reg<64, CS, 0>(scores, ld, nvalid, cand, rows, K, topk_idx, Cout,
                                      cand_out, err, stream);
  else
    return cudaErrorInvalidValue;   // the block mode keeps at most 16 blocks per thread
}

// Cluster size for the register kernel: the largest of 1, 2, 4, 8 that keeps
// rows x CS within the SMs.
int reg_cluster_size(int rows, int sms) {
  int rcs = 1;
  while (rcs < 8 && rows * rcs * 2 <= sms) rcs *= 2;
  return rcs;
}

template <int kBlk>
cudaError_t launch_topk_reg_any(const float* scores, int ld, int slots, const int32_t* nvalid,
                                const int32_t* cand, int rows, int K, int32_t* topk_idx,
                                int Cout, int32_t* cand_out, int* err, cudaStream_t stream,
                                int rcs) {
  if (rcs == 8)
    return launch_topk_reg_cs<8, kBlk>(scores, ld, slots, nvalid, cand, rows, K, topk_idx, Cout,
                                       cand_out, err, stream);
  if (rcs == 4)
    return launch_topk_reg_cs<4, kBlk>(scores, ld, slots, nvalid, cand, rows, K, topk_idx, Cout,
                                       cand_out, err, stream);
  if (rcs == 2)
    return launch_topk_reg_cs<2, kBlk>(scores, ld, slots, nvalid, cand, rows, K, topk_idx, Cout,
                                       cand_out, err, stream);
  return launch_topk_reg_cs<1, kBlk>(scores, ld, slots, nvalid, cand, rows, K, topk_idx, Cout,
                                     cand_out, err, stream);
}

}  // namespace

int topk_sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

cudaError_t launch_topk(const float* scores, int ld, const int32_t* nvalid, const int32_t* cand,
                        int rows, int K, int32_t* topk_idx, int Cout, int32_t* cand_out,
                        int* err, cudaStream_t stream) {
  if (rows == 0) return cudaSuccess;
  // Register variant: a cluster of CS CTAs per row (as many as keep rows x CS
  // within the SMs), each holding at most 64 keys per thread in registers
  {
    int rcs = reg_cluster_size(rows, topk_sm_count());
    // rows too long for that many CTAs: the smallest cluster that holds them,
    // in more than one wave (still far ahead of the shared-memory kernels)
    while (rcs < 8 && ld > rcs * kRThreads * 64) rcs *= 2;
    if (ld <= rcs * kRThreads * 64)
      return launch_topk_reg_any<0>(scores, ld, ld, nvalid, cand, rows, K, topk_idx, Cout,
                                    cand_out, err, stream, rcs);
  }
  // Few rows: a cluster of cs CTAs per row (cs = 2, 4 or 8, as many as keep
  // rows x cs within one wave), each staging a slice of the row.
  const int sms = topk_sm_count();
  int cs = 1;
  while (cs < 8 && rows * cs * 2 <= sms) cs *= 2;
  const size_t kSmemCap = 200 * 1024;
  while (cs > 1 && cs < 8 && (size_t)ceil_div(ld, cs) * sizeof(uint32_t) > kSmemCap) cs *= 2;
  const int slice = ceil_div(ld, cs);
  if (cs > 1 && (size_t)slice * sizeof(uint32_t) <= kSmemCap) {
    const size_t smem = (size_t)slice * sizeof(uint32_t);
    cudaError_t e = cudaFuncSetAttribute(topk_cluster_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(topk_cluster_kernel, dim3((unsigned)(rows * cs)), dim3(kCThreads), smem,
                      stream, dim3((unsigned)cs, 1, 1), scores, ld, nvalid, cand, K, topk_idx,
                      Cout, cand_out, slice, err);
  }
  if (ld <= kSmemKeyCap) {
    size_t smem = (size_t)ld * sizeof(uint32_t);
    cudaError_t e = cudaFuncSetAttribute(topk_kernel<true>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(topk_kernel<true>, dim3(rows), dim3(kThreads), smem, stream, dim3(1), scores,
                      ld, nvalid, cand, K, topk_idx, Cout, cand_out, err);
  }
  return launch_pdl(topk_kernel<false>, dim3(rows), dim3(kThreads), 0, stream, dim3(1), scores, ld,
                    nvalid, cand, K, topk_idx, Cout, cand_out, err);
}

// The blockwise pool in one launch of the register kernel (blocks of 8
// positions); false when the shape is outside its range.
bool launch_block_pool_reg(const float* scores, int ld, const int32_t* nvalid, int rows,
                           int block, int nblocks, int32_t* cand, int* err, cudaStream_t stream,
                           cudaError_t* e) {
  if (block != 8 || rows == 0) return false;
  const int nbmax = (ld + 7) / 8;
  const int rcs = reg_cluster_size(rows, topk_sm_count());
  if (nbmax > rcs * kRThreads * 16) return false;
  *e = launch_topk_reg_any<8>(scores, ld, nbmax, nvalid, nullptr, rows, nblocks, cand, 0, nullptr,
                              err, stream, rcs);
  return true;
}

}  // namespace csa2
