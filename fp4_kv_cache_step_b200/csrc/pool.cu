// pool.cu -- blockwise candidate pool of the hierarchical indexer.
//
// "Detailed Notes On DeepSeek V4 Point 1 Flash In Simple Words", section
// "Hierarchical Sparse Indexer In Simple Terms", and the mengman.github.io
// interpretation, section 3.4: the first FULL layer of the decoder groups
// positions into blocks of 8, scores each block by the best score inside it
// and keeps the best 2048 blocks; the later REINDEX layers score only those
// (about 16384) positions. Blocks are ranked by the entries' own rule (score
// descending, lower index first), by the top-K kernel itself:
//   block_max_kernel   scores [rows][ld] -> block scores [rows][nbmax] and the
//                      number of blocks holding a valid position per row
//   launch_topk        the best nblocks blocks, ascending block ids
//   block_expand_kernel block ids -> their valid positions, ascending, -1 padded
// All three are small next to the scan that produced the scores (4 bytes read
// per valid position, from L2 right after the scorer wrote them). For blocks
// of 8 the register top-K does all three in one launch (block mode: keys are
// block maxima, the kept blocks written as their positions).
#include "common.cuh"
#include "kernels.h"

namespace csa2 {
namespace {

// One thread per (row, block), then one per row for the number of blocks
// holding a valid position. A NaN score is kept, so that the selection flags
// it as it would for an entry.
__global__ void block_max_kernel(const float* __restrict__ scores, int ld,
                                 const int32_t* __restrict__ nvalid, int rows, int block,
                                 int nbmax, float* __restrict__ bscores,
                                 int32_t* __restrict__ nvb) {
  const size_t total = (size_t)rows * nbmax;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total;
       i += (size_t)gridDim.x * blockDim.x) {
    const int r = (int)(i / nbmax), bk = (int)(i % nbmax);
    const int nv = max(0, min(ld, __ldg(nvalid + r)));
    const int j0 = bk * block, j1 = min(j0 + block, nv);
    float m = -INFINITY;
    bool nan = false;
    for (int j = j0; j < j1; ++j) {
      const float x = scores[(size_t)r * ld + j];
      nan |= x != x;
      m = fmaxf(m, x);
    }
    bscores[i] = nan ? __int_as_float(0x7fc00000) : m;
  }
  for (size_t r = blockIdx.x * (size_t)blockDim.x + threadIdx.x; r < (size_t)rows;
       r += (size_t)gridDim.x * blockDim.x) {
    const int nv = max(0, min(ld, __ldg(nvalid + r)));
    nvb[r] = (nv + block - 1) / block;
  }
}

// One thread per (row, pool slot): slot s belongs to kept block s / block.
// Kept blocks come ascending and -1 padded, and only the last block holding a
// valid position can be partial, so the positions come out ascending with all
// the -1 slots at the end.
__global__ void block_expand_kernel(const int32_t* __restrict__ bids, int nblocks,
                                    const int32_t* __restrict__ nvalid, int ld, int rows,
                                    int block, int32_t* __restrict__ cand) {
  const size_t C = (size_t)nblocks * block;
  const size_t total = (size_t)rows * C;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total;
       i += (size_t)gridDim.x * blockDim.x) {
    const int r = (int)(i / C);
    const size_t s = i % C;
    const int b = __ldg(bids + (size_t)r * nblocks + s / block);
    const int nv = max(0, min(ld, __ldg(nvalid + r)));
    const long long j = (long long)b * block + (long long)(s % block);
    cand[i] = (b >= 0 && j < nv) ? (int32_t)j : -1;
  }
}

constexpr size_t kAlign = 256;
size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

int grid_for(size_t total) {
  size_t blocks = (total + 255) / 256;
  if (blocks > 148 * 32) blocks = 148 * 32;
  return (int)(blocks > 0 ? blocks : 1);
}

}  // namespace

size_t block_pool_workspace_bytes(int rows, int ld, int block, int nblocks) {
  if (rows <= 0 || ld < 0 || block <= 0 || nblocks <= 0) return 0;
  const size_t nbmax = ((size_t)ld + block - 1) / block;
  return align_up((size_t)rows * nbmax * sizeof(float)) + align_up((size_t)rows * sizeof(int32_t)) +
         align_up((size_t)rows * nblocks * sizeof(int32_t));
}

cudaError_t launch_block_pool(const float* scores, int ld, const int32_t* nvalid, int rows,
                              int block, int nblocks, int32_t* cand, void* workspace, int* err,
                              cudaStream_t stream) {
  if (rows == 0) return cudaSuccess;
  const int nbmax = (int)(((size_t)ld + block - 1) / block);
  if (nbmax == 0)   // no position at all: an empty pool (all bytes 0xff = -1)
    return cudaMemsetAsync(cand, 0xff, (size_t)rows * nblocks * block * sizeof(int32_t), stream);
  // blocks of 8 (the pages' size) in one launch: the register top-K keys each
  // block by its maximum and writes the kept blocks' positions itself
  cudaError_t er = cudaSuccess;
  if (launch_block_pool_reg(scores, ld, nvalid, rows, block, nblocks, cand, err, stream, &er))
    return er;
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  float* bscores = reinterpret_cast<float*>(ws);
  int32_t* nvb = reinterpret_cast<int32_t*>(ws + align_up((size_t)rows * nbmax * sizeof(float)));
  int32_t* bids = reinterpret_cast<int32_t*>(reinterpret_cast<unsigned char*>(nvb) +
                                             align_up((size_t)rows * sizeof(int32_t)));
  block_max_kernel<<<grid_for((size_t)rows * (nbmax > 0 ? nbmax : 1)), 256, 0, stream>>>(
      scores, ld, nvalid, rows, block, nbmax, bscores, nvb);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = launch_topk(bscores, nbmax, nvb, nullptr, rows, nblocks, bids, 0, nullptr, err, stream);
  if (e != cudaSuccess) return e;
  block_expand_kernel<<<grid_for((size_t)rows * nblocks * block), 256, 0, stream>>>(
      bids, nblocks, nvalid, ld, rows, block, cand);
  return cudaGetLastError();
}

}  // namespace csa2
