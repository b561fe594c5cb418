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
// Rows that fit are staged once in shared memory.
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

}  // namespace csa2
