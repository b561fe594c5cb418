// score_tc.cu -- CSA2 indexer scoring on the 5th-generation tensor cores.
//
// "Detailed Notes On DeepSeek V4 Point 1 Flash In Simple Words", section
// "Compressed Sparse Attention 2 Or CSA2 In Simple Terms": every indexing layer
// scores all visible entries against its query; the keys are one shared
// indexer key per entry. Score of entry j for query (b, t):
//     s_j = sum_h w_h * max(0, q_h . k_j)
//
// Per (b, group of nq consecutive queries) the dot products form a dense
// contraction D[j][(t, h)] = sum_c K[j][c] Q[(t, h)][c] with E4M3 operands and
// fp32 accumulation: M = 128 entries (TMEM lanes), N = nq * Hi (TMEM columns),
// K = Di. The kernel is persistent (one CTA per SM, a contiguous share of all
// (group, 128-entry) tiles) and warp-specialised:
//   warp 0     TMA producer: indexer-key tiles (128 x Di bytes, 128/64-byte
//              swizzle) into a ring of shared-memory stages, and the group's
//              query block (N x Di) into one of two query buffers;
//   warp 1     allocates TMEM and issues tcgen05.mma kind::f8f6f4 (one thread),
//              committing each tile to "stage free" and "accumulator full";
//   warps 2-9  two epilogue warpgroups taking alternate tiles: TMEM -> registers,
//              ReLU, head-weighted sum, masked store of the score.
// Decode (nq = 1) streams the keys once at HBM rate; the tensor core is ~1/5
// busy. Prefill chunks (nq = 256 / Hi) make it a real dense FP8 contraction.
// Every mbarrier wait is bounded; a timeout is reported as CSA2_ERR_TIMEOUT.
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace csa2 {
namespace {

using namespace sm100;

constexpr int kTileM = 128;
constexpr int kThreads = 320;
constexpr int kEpiWarps = 8;                // warps 2-9
constexpr int kMaxGroups = 8192;
constexpr size_t kSmemLimit = 227 * 1024;   // opt-in dynamic shared memory per CTA

struct TcParams {
  int Tq, N, Hi, Di, nq, G, groups_per_b, stages, nacc;
  int sub;            // 128-entry MMA blocks per pipeline tile (2 for decode, 1 for prefill)
  uint32_t ncols;
  const int32_t* nvalid;
  const float* idx_w;
  float* scores;
  int* err;
};

__device__ __forceinline__ int group_tiles(const TcParams& p, int g) {
  const int b = g / p.groups_per_b;
  const int t0 = (g % p.groups_per_b) * p.nq;
  int nmax = 0;
  for (int t = t0; t < min(t0 + p.nq, p.Tq); ++t)
    nmax = max(nmax, min(p.N, max(0, p.nvalid[(size_t)b * p.Tq + t])));
  const int rows = kTileM * p.sub;
  return (nmax + rows - 1) / rows;
}

// Two fp32 fused multiply-adds as one packed instruction (each rounded once,
// like fmaf).
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  uint64_t ua, ub, uc, d;
  asm("mov.b64 %0, {%1, %2};" : "=l"(ua) : "f"(a.x), "f"(a.y));
  asm("mov.b64 %0, {%1, %2};" : "=l"(ub) : "f"(b.x), "f"(b.y));
  asm("mov.b64 %0, {%1, %2};" : "=l"(uc) : "f"(c.x), "f"(c.y));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(ua), "l"(ub), "l"(uc));
  float2 r;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(d));
  return r;
}

// The MMAs of one pipeline tile: SUB blocks of 128 entries x KSTEPS steps of
// 32 key bytes. Descriptor start addresses advance by adding (bytes >> 4) to
// the low field (shared-memory addresses stay below 2^18, so no carry).
template <int SUB, int KSTEPS>
__device__ __forceinline__ void issue_tile(uint32_t d0, uint64_t ad, uint64_t bd, uint32_t idesc,
                                           uint32_t n_mma) {
#pragma unroll
  for (int sb = 0; sb < SUB; ++sb)
#pragma unroll
    for (int kk = 0; kk < KSTEPS; ++kk)
      mma_e4m3(d0 + (uint32_t)sb * n_mma,
               ad + (uint64_t)((sb * kTileM * KSTEPS * 32 + kk * 32) >> 4),
               bd + (uint64_t)((kk * 32) >> 4), idesc, kk > 0 ? 1u : 0u);
}

// kHi indexer heads, kNq queries per group: (64, 1) is the decode path (the
// weights stay in registers); otherwise the multi-query epilogue, with every
// index constant, so that each shape gets the registers and instructions it
// needs.
template <int kHi, int kNq>
__global__ void __launch_bounds__(kThreads, 1)
index_score_tc_kernel(const __grid_constant__ CUtensorMap kmap,
                      const __grid_constant__ CUtensorMap qmap, const TcParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int tile_rows = kTileM * p.sub;
  const int tile_bytes = tile_rows * p.Di;
  const int n_mma = p.Hi * p.nq;
  const int q_bytes = n_mma * p.Di;
  uint8_t* kbuf = base;
  uint8_t* qbuf = kbuf + p.stages * tile_bytes;
  // the current group's head weights, one copy per epilogue warp ([qi][h])
  float* wbuf = reinterpret_cast<float*>(qbuf + 2 * q_bytes);
  uint64_t* full = reinterpret_cast<uint64_t*>(wbuf + kEpiWarps * n_mma);
  uint64_t* empty = full + p.stages;
  uint64_t* acc_full = empty + p.stages;
  uint64_t* acc_empty = acc_full + 4;
  uint64_t* q_full = acc_empty + 4;
  uint64_t* q_empty = q_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(q_empty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* tile_pre = const_cast<int*>(reinterpret_cast<volatile int*>(tmem_slot + 2));   // [G + 1]
  int* scan_tmp = tile_pre + p.G + 1;                                               // [kThreads/32]

  constexpr bool kDecode = kHi == 64 && kNq == 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_wait_and_release();

  // ---- prefix of tile counts over groups (contiguous chunk per thread)
  {
    const int per = (p.G + kThreads - 1) / kThreads;
    const int g0 = min(p.G, (int)threadIdx.x * per), g1 = min(p.G, g0 + per);
    int local = 0;
    for (int g = g0; g < g1; ++g) {
      const int c = group_tiles(p, g);
      tile_pre[g + 1] = c;
      local += c;
    }
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int u = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += u;
    }
    if (lane == 31) scan_tmp[warp] = incl;
    __syncthreads();
    int before = 0;
    for (int w2 = 0; w2 < warp; ++w2) before += scan_tmp[w2];
    int run = before + incl - local;
    if (threadIdx.x == 0) tile_pre[0] = 0;
    for (int g = g0; g < g1; ++g) {
      run += tile_pre[g + 1];
      tile_pre[g + 1] = run;
    }
  }

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 4);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&kmap);
    tma_prefetch_desc(&qmap);
  }
  if (warp == 1) tmem_alloc(tmem_slot, p.ncols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const long long T = tile_pre[p.G];
  const int lo = (int)(T * blockIdx.x / gridDim.x);
  const int hi = (int)(T * (blockIdx.x + 1) / gridDim.x);
  // first group whose tile range contains `lo`
  int g_first = 0;
  {
    int a = 0, bnd = p.G;   // find largest g with tile_pre[g] <= lo
    while (a < bnd) {
      int m = (a + bnd + 1) >> 1;
      if (tile_pre[m] <= lo) a = m; else bnd = m - 1;
    }
    g_first = min(a, max(p.G - 1, 0));
  }

  if (warp == 0) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t ph = 0;
      int qseq = -1, cur_g = -1, g = g_first;
      for (int tile = lo; tile < hi; ++tile) {
        while (tile >= tile_pre[g + 1]) ++g;
        const int b = g / p.groups_per_b;
        if (g != cur_g) {
          ++qseq;
          const int qb = qseq & 1;
          if (!mbar_wait(&q_empty[qb], ((qseq >> 1) & 1) ^ 1, abort_flag)) break;
          mbar_arrive_expect_tx(&q_full[qb], q_bytes);
          const int qrow = (b * p.Tq + (g % p.groups_per_b) * p.nq) * p.Hi;
          tma_load_2d(&qmap, &q_full[qb], qbuf + qb * q_bytes, 0, qrow);
          cur_g = g;
        }
        const int e = tile - tile_pre[g];
        if (!mbar_wait(&empty[stage], ph ^ 1, abort_flag)) break;
        mbar_arrive_expect_tx(&full[stage], tile_bytes);
        tma_load_2d(&kmap, &full[stage], kbuf + stage * tile_bytes, 0, b * p.N + e * tile_rows);
        if (++stage == p.stages) { stage = 0; ph ^= 1; }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_e4m3_f32(kTileM, n_mma);
      const int ksteps = p.Di / 32;
      const uint32_t acc_cols = (uint32_t)(n_mma * p.sub);
      int stage = 0, acc = 0;
      uint32_t ph = 0, acc_ph = 1;
      int qseq = -1, cur_g = -1, g = g_first;
      int next_g_tile = tile_pre[g + 1];
      uint32_t b0 = 0;
      for (int tile = lo; tile < hi; ++tile) {
        if (tile >= next_g_tile) {
          while (tile >= tile_pre[g + 1]) ++g;
          next_g_tile = tile_pre[g + 1];
        }
        if (g != cur_g) {
          if (cur_g >= 0) mma_commit(&q_empty[qseq & 1]);
          ++qseq;
          if (!mbar_wait(&q_full[qseq & 1], (qseq >> 1) & 1, abort_flag)) break;
          cur_g = g;
          b0 = smem_u32(qbuf + (qseq & 1) * q_bytes);
        }
        if (!mbar_wait(&acc_empty[acc], acc_ph, abort_flag)) break;
        if (!mbar_wait(&full[stage], ph, abort_flag)) break;
        tc_fence_after();
        const uint64_t ad = smem_desc_kmajor(smem_u32(kbuf + stage * tile_bytes), p.Di);
        const uint64_t bd = smem_desc_kmajor(b0, p.Di);
        const uint32_t d0 = tmem_base + (uint32_t)acc * acc_cols;
        if (p.sub == 2 && ksteps == 4)
          issue_tile<2, 4>(d0, ad, bd, idesc, (uint32_t)n_mma);
        else if (ksteps == 4)
          issue_tile<1, 4>(d0, ad, bd, idesc, (uint32_t)n_mma);
        else
          issue_tile<1, 2>(d0, ad, bd, idesc, (uint32_t)n_mma);
        mma_commit(&empty[stage]);
        mma_commit(&acc_full[acc]);
        if (++stage == p.stages) { stage = 0; ph ^= 1; }
        if (++acc == p.nacc) { acc = 0; acc_ph ^= 1; }
      }
    }
  } else {
    // ------------------------------------------------ epilogue warpgroups
    const int wg = (warp - 2) >> 2;
    const int quad = warp & 3;                 // TMEM lane quadrant this warp may access
    const int m = quad * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
    int g = g_first, k = 0, wg_group = -1;
    float wreg[64];                            // head weights of the current query (nq == 1)
    int nvq[kNq];                              // the group's query lengths (multi-query)
    int nv_cur = 0;
    for (int tile = lo; tile < hi; ++tile, ++k) {
      while (tile >= tile_pre[g + 1]) ++g;
      if ((k & 1) != wg) continue;
      const int acc = k % p.nacc;
      const int b = g / p.groups_per_b;
      const int t0 = (g % p.groups_per_b) * p.nq;
      if (kDecode && g != wg_group) {
        // load this query's weights and length once per group, before the wait
        const size_t row = (size_t)b * p.Tq + t0;
        const float4* w4 = reinterpret_cast<const float4*>(p.idx_w + row * 64);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float4 wv = __ldg(w4 + i);
          wreg[4 * i] = wv.x;
          wreg[4 * i + 1] = wv.y;
          wreg[4 * i + 2] = wv.z;
          wreg[4 * i + 3] = wv.w;
        }
        nv_cur = min(__ldg(p.nvalid + row), p.N);
        wg_group = g;
      }
      if (!mbar_wait_warp(&acc_full[acc], (k / p.nacc) & 1, abort_flag)) break;
      tc_fence_after();
      const int j = (tile - tile_pre[g]) * (kTileM * p.sub) + m;
      const uint32_t acc_addr = tmem_base + lane_addr + (uint32_t)(acc * n_mma * p.sub);
      if (kDecode) {
        float* dst = p.scores + ((size_t)b * p.Tq + t0) * p.N;
        for (int sb = 0; sb < p.sub; ++sb) {
          float v[64];
          tmem_ld_64(acc_addr + (uint32_t)(sb * 64), v);
          if (sb == p.sub - 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[acc]);
          }
          float s0 = 0.0f, s1 = 0.0f;
#pragma unroll
          for (int i = 0; i < 64; i += 2) {
            s0 = fmaf(wreg[i], fmaxf(v[i], 0.0f), s0);
            s1 = fmaf(wreg[i + 1], fmaxf(v[i + 1], 0.0f), s1);
          }
          if (j + sb * kTileM < nv_cur) dst[j + sb * kTileM] = s0 + s1;
        }
        continue;
      }
      // this warp's copy of the group's weights ([qi][h]), read by broadcast
      // below, and the group's query lengths
      float* wwarp = wbuf + (warp - 2) * (kNq * kHi);
      if (g != wg_group) {
        __syncwarp();
#pragma unroll
        for (int i = lane; i < kNq * kHi; i += 32) {
          const int qi = i / kHi, t = t0 + qi;
          wwarp[i] = t < p.Tq ? __ldg(p.idx_w + ((size_t)b * p.Tq + t) * kHi + (i - qi * kHi))
                              : 0.0f;
        }
#pragma unroll
        for (int qi = 0; qi < kNq; ++qi)
          nvq[qi] = t0 + qi < p.Tq ? min(__ldg(p.nvalid + (size_t)b * p.Tq + t0 + qi), p.N) : 0;
        __syncwarp();
        wg_group = g;
      }
      // one 64-column chunk (64 heads of one query) at a time: ReLU, then the
      // head weights by packed fp32 pairs into 4 partial sums per chunk
      // (integer-valued terms add exactly in any order)
#pragma unroll
      for (int qi = 0; qi < kNq; ++qi) {
        float2 acc2[4] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f),
                          make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f)};
#pragma unroll
        for (int h0 = 0; h0 < kHi; h0 += 64) {
          float v[64];
          tmem_ld_64(acc_addr + (uint32_t)(qi * kHi + h0), v);
          const float4* w4 = reinterpret_cast<const float4*>(wwarp + qi * kHi + h0);
#pragma unroll
          for (int i = 0; i < 64; i += 8) {
            const float4 wa = w4[i / 4], wb = w4[i / 4 + 1];
            acc2[0] = ffma2(make_float2(wa.x, wa.y),
                            make_float2(fmaxf(v[i], 0.0f), fmaxf(v[i + 1], 0.0f)), acc2[0]);
            acc2[1] = ffma2(make_float2(wa.z, wa.w),
                            make_float2(fmaxf(v[i + 2], 0.0f), fmaxf(v[i + 3], 0.0f)), acc2[1]);
            acc2[2] = ffma2(make_float2(wb.x, wb.y),
                            make_float2(fmaxf(v[i + 4], 0.0f), fmaxf(v[i + 5], 0.0f)), acc2[2]);
            acc2[3] = ffma2(make_float2(wb.z, wb.w),
                            make_float2(fmaxf(v[i + 6], 0.0f), fmaxf(v[i + 7], 0.0f)), acc2[3]);
          }
        }
        const float sc = ((acc2[0].x + acc2[0].y) + (acc2[1].x + acc2[1].y)) +
                         ((acc2[2].x + acc2[2].y) + (acc2[3].x + acc2[3].y));
        if (j < nvq[qi]) p.scores[((size_t)b * p.Tq + t0 + qi) * p.N + j] = sc;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[acc]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, p.ncols);
  }
  if (threadIdx.x == 0 && *abort_flag) record_error(p.err, CSA2_ERR_TIMEOUT);
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static std::once_flag once;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

bool make_map(CUtensorMap* map, const void* ptr, uint64_t rows, int row_bytes, int box_rows) {
  auto encode = get_encode();
  if (!encode) return false;
  cuuint64_t dims[2] = {(cuuint64_t)row_bytes, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
  cuuint32_t box[2] = {(cuuint32_t)row_bytes, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides,
                      box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                      row_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

}  // namespace

bool index_score_tc_supported(int B, int Tq, int Hi, int Di, const int32_t* cand) {
  if (cand != nullptr) return false;
  if (!(Di == 64 || Di == 128)) return false;
  if (!(Hi == 64 || Hi == 128)) return false;
  const int nq = Tq == 1 ? 1 : min(Tq, 256 / Hi);
  const long long G = (long long)B * ((Tq + nq - 1) / nq);
  return G >= 1 && G <= kMaxGroups;
}

cudaError_t launch_index_score_tc(const uint8_t* idx_q, const float* idx_w, const uint8_t* idx_k,
                                  int B, int Tq, int N, int Hi, int Di, const int32_t* nvalid,
                                  float* scores, int* err, cudaStream_t stream) {
  TcParams p;
  p.Tq = Tq;
  p.N = N;
  p.Hi = Hi;
  p.Di = Di;
  p.nq = Tq == 1 ? 1 : min(Tq, 256 / Hi);
  p.groups_per_b = (Tq + p.nq - 1) / p.nq;
  p.G = B * p.groups_per_b;
  const int n_mma = Hi * p.nq;
  // Decode (64 query columns): 256-entry pipeline tiles (32 KB of keys, two
  // M = 128 blocks), so the per-tile barrier round trips are spread over
  // twice the bytes; prefill keeps 128-entry tiles for its wider accumulators.
  p.sub = (n_mma <= 64 && Di == 128) ? 2 : 1;
  p.nacc = n_mma <= 128 ? 4 : 2;          // accumulator ring depth
  p.ncols = 32;
  while (p.ncols < (uint32_t)(p.nacc * n_mma * p.sub)) p.ncols <<= 1;
  // key-tile ring: as deep as the shared memory left after the query
  // buffers, barriers and the group prefix allows (at most 6 or 8 stages)
  const size_t fixed = 1024 + 2 * (size_t)n_mma * Di + (size_t)kEpiWarps * n_mma * sizeof(float) +
                       (2 * 16 + 12) * sizeof(uint64_t) + 16 + (size_t)(p.G + 1 + 32) * sizeof(int);
  const size_t tile_bytes = (size_t)kTileM * p.sub * Di;
  const int max_stages = p.sub == 2 ? 6 : (n_mma <= 64 ? 8 : 5);
  p.stages = (int)std::min<size_t>(max_stages, (kSmemLimit - fixed) / tile_bytes);
  if (p.stages < 2) return cudaErrorInvalidValue;
  p.nvalid = nvalid;
  p.idx_w = idx_w;
  p.scores = scores;
  p.err = err;

  CUtensorMap kmap, qmap;
  if (!make_map(&kmap, idx_k, (uint64_t)B * N, Di, kTileM * p.sub) ||
      !make_map(&qmap, idx_q, (uint64_t)B * Tq * Hi, Di, n_mma))
    return cudaErrorInvalidValue;

  const size_t smem = fixed + (size_t)p.stages * tile_bytes;
  void (*kernel)(CUtensorMap, CUtensorMap, TcParams) = nullptr;
  if (Hi == 64) {
    kernel = p.nq == 1   ? index_score_tc_kernel<64, 1>
             : p.nq == 2 ? index_score_tc_kernel<64, 2>
             : p.nq == 3 ? index_score_tc_kernel<64, 3>
                         : index_score_tc_kernel<64, 4>;
  } else {
    kernel = p.nq == 1 ? index_score_tc_kernel<128, 1> : index_score_tc_kernel<128, 2>;
  }
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  // upper bound on the tile count; CTAs beyond the real count get empty ranges
  const long long max_tiles = (long long)p.G * ((N + kTileM * p.sub - 1) / (kTileM * p.sub));
  const int grid = (int)std::min<long long>(sm_count(), std::max<long long>(1, max_tiles));
  return launch_pdl(kernel, dim3(grid), dim3(kThreads), smem, stream, dim3(1), kmap, qmap, p);
}

}  // namespace csa2
