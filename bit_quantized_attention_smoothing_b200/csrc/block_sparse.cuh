// block_sparse.cuh -- key-tile selection for block-sparse attention on B200.
//
// The page "ThriftAttention: Selective Mixed Precision for Long-Context FP4 Attention" (technical
// summary, method, heuristic block selection) rates each (query block, key block) pair by the dot
// product of the two blocks' mean vectors and singles out the top-k pairs; its results compare
// against sparse top-k attention, which computes only those pairs.  Here a query block is the
// 256 rows one attention CTA owns (two 128-row Q tiles), a key block is one 128-key tile:
//  * block_means_kernel: per-block channel means of the fp16 input, exact (int64 fixed point of
//    the fp16 values, one binary64 division);
//  * block_scores_kernel: score[i][j] = qmean_i . kmean_j in binary64, one fma per channel in
//    channel order (so every score is one fixed function of the means);
//  * block_select_kernel: per query block, the diagonal key tiles (causal), then the topk
//    highest-scoring other tiles it may see (ties to the lower index), as an ascending list --
//    the attention kernel's CTA for that block streams exactly these tiles.
#pragma once

#include <cuda_fp16.h>
#include <cstdint>

namespace qattn {

constexpr int kSelQRows = 256;  // query rows per selection block (one attention CTA)
constexpr int kSelKRows = 128;  // keys per key tile

// means[o][blk][c] = mean over the rows of block blk (rows_per_block rows; the last block holds
// the rest) of x[o][n][c].  grid (outer, nblocks), 256 threads.
template <int D>
__global__ void __launch_bounds__(256) block_means_kernel(const uint16_t* __restrict__ x, int N,
                                                          int rows_per_block,
                                                          double* __restrict__ means) {
  constexpr int PH = 256 / D;  // row phases per channel
  __shared__ long long part[PH][D];
  const long long o = blockIdx.x;
  const int blk = blockIdx.y;
  const int nb = gridDim.y;
  const int c = threadIdx.x % D, ph = threadIdx.x / D;
  const int n0 = blk * rows_per_block;
  const int n1 = min(N, n0 + rows_per_block);
  const uint16_t* src = x + static_cast<size_t>(o) * N * D;
  long long s = 0;
  for (int n = n0 + ph; n < n1; n += PH)
    s += __float2ll_rn(__half2float(__ushort_as_half(src[static_cast<size_t>(n) * D + c])) * 16777216.0f);
  part[ph][c] = s;
  __syncthreads();
  if (threadIdx.x < D) {
    long long t = 0;
#pragma unroll
    for (int p = 0; p < PH; ++p) t += part[p][threadIdx.x];
    means[(static_cast<size_t>(o) * nb + blk) * D + threadIdx.x] =
        __ddiv_rn(__ll2double_rn(t), static_cast<double>(n1 - n0) * 16777216.0);
  }
}

// scores[bh][i][j] for a 32 x 32 tile of (query block i, key tile j) per CTA; grid
// (ceil(nkt/32), ceil(nsb/32), B*H), 256 threads, each 4 scores.
constexpr int kScoreTile = 32;
template <int D>
__global__ void __launch_bounds__(256) block_scores_kernel(const double* __restrict__ qmeans,
                                                           const double* __restrict__ kmeans,
                                                           int H, int Hkv, int nsb, int nkt,
                                                           double* __restrict__ scores) {
  extern __shared__ double sm[];
  double* qs = sm;                        // [32][D]
  double* ks = sm + kScoreTile * D;       // [32][D]
  const long long bh = blockIdx.z;
  const long long bg = (bh / H) * Hkv + (bh % H) / (H / Hkv);
  const int i0 = blockIdx.y * kScoreTile, j0 = blockIdx.x * kScoreTile;
  for (int e = threadIdx.x; e < kScoreTile * D; e += 256) {
    const int r = e / D, c = e % D;
    qs[e] = i0 + r < nsb ? qmeans[(static_cast<size_t>(bh) * nsb + i0 + r) * D + c] : 0.0;
    ks[e] = j0 + r < nkt ? kmeans[(static_cast<size_t>(bg) * nkt + j0 + r) * D + c] : 0.0;
  }
  __syncthreads();
  const int jj = threadIdx.x % kScoreTile;
  for (int ii = threadIdx.x / kScoreTile; ii < kScoreTile; ii += 256 / kScoreTile) {
    if (i0 + ii >= nsb || j0 + jj >= nkt) continue;
    double acc = 0.0;
    for (int c = 0; c < D; ++c) acc = __fma_rn(qs[ii * D + c], ks[jj * D + c], acc);
    scores[(static_cast<size_t>(bh) * nsb + i0 + ii) * nkt + j0 + jj] = acc;
  }
}

// Selection for query block i of head bh: grid (nsb, B*H), 256 threads.  list[bh][i][0..count)
// ascending; entries past count are left alone.
__global__ void __launch_bounds__(256) block_select_kernel(const double* __restrict__ scores,
                                                           int nsb, int nkt, int causal, int topk,
                                                           int* __restrict__ list,
                                                           int* __restrict__ count) {
  extern __shared__ unsigned char sel_smem[];
  unsigned char* pick = sel_smem;  // [nkt]
  __shared__ double best_s[8];
  __shared__ int best_j[8];
  const long long bh = blockIdx.y;
  const int i = blockIdx.x;
  const double* sc = scores + (static_cast<size_t>(bh) * nsb + i) * nkt;
  int last = causal ? 2 * i + 1 : nkt - 1;  // highest key tile the block may see
  if (last > nkt - 1) last = nkt - 1;
  for (int j = threadIdx.x; j < nkt; j += 256) pick[j] = (causal && j >= 2 * i && j <= last) ? 1 : 0;
  __syncthreads();
  for (int r = 0; r < topk; ++r) {
    // the best unpicked candidate: highest score, lowest index among equal scores
    double bs = 0.0;
    int bj = -1;
    for (int j = threadIdx.x; j <= last; j += 256)
      if (!pick[j] && (bj < 0 || sc[j] > bs)) {
        bs = sc[j];
        bj = j;
      }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const double os = __shfl_xor_sync(0xFFFFFFFFu, bs, off);
      const int oj = __shfl_xor_sync(0xFFFFFFFFu, bj, off);
      if (oj >= 0 && (bj < 0 || os > bs || (os == bs && oj < bj))) {
        bs = os;
        bj = oj;
      }
    }
    if ((threadIdx.x & 31) == 0) {
      best_s[threadIdx.x >> 5] = bs;
      best_j[threadIdx.x >> 5] = bj;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      double s = 0.0;
      int jb = -1;
      for (int w = 0; w < 8; ++w)
        if (best_j[w] >= 0 && (jb < 0 || best_s[w] > s || (best_s[w] == s && best_j[w] < jb))) {
          s = best_s[w];
          jb = best_j[w];
        }
      best_j[0] = jb;
      if (jb >= 0) pick[jb] = 1;
    }
    __syncthreads();
    const bool done = best_j[0] < 0;
    __syncthreads();
    if (done) break;
  }
  if (threadIdx.x == 0) {
    int* out = list + (static_cast<size_t>(bh) * nsb + i) * nkt;
    int n = 0;
    for (int j = 0; j < nkt; ++j)
      if (pick[j]) out[n++] = j;
    count[static_cast<size_t>(bh) * nsb + i] = n;
  }
}

}  // namespace qattn
