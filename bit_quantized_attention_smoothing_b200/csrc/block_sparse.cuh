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
// the rest) of x[o][n][c].  grid (outer, nblocks), 256 threads: each thread sums 8 channels
// (one 16-byte load per row) of every (256 / (D / 8))-th row.
template <int D>
__global__ void __launch_bounds__(256) block_means_kernel(const uint16_t* __restrict__ x, int N,
                                                          int rows_per_block,
                                                          double* __restrict__ means) {
  constexpr int VPR = D / 8;        // 16-byte vectors per row
  constexpr int RPI = 256 / VPR;    // rows per iteration of the CTA
  __shared__ long long part[RPI][D];
  const long long o = blockIdx.x;
  const int blk = blockIdx.y;
  const int nb = gridDim.y;
  const int cg = threadIdx.x % VPR, r_in = threadIdx.x / VPR;
  const int n0 = blk * rows_per_block;
  const int n1 = min(N, n0 + rows_per_block);
  const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<size_t>(o) * N * D);
  long long acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0;
  for (int n = n0 + r_in; n < n1; n += RPI) {
    const uint4 v = __ldg(src + static_cast<size_t>(n) * VPR + cg);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      acc[2 * e] += __float2ll_rn(__half2float(__ushort_as_half(static_cast<unsigned short>(w[e] & 0xFFFFu))) * 16777216.0f);
      acc[2 * e + 1] += __float2ll_rn(__half2float(__ushort_as_half(static_cast<unsigned short>(w[e] >> 16))) * 16777216.0f);
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) part[r_in][cg * 8 + e] = acc[e];
  __syncthreads();
  for (int c = threadIdx.x; c < D; c += 256) {
    long long t = 0;
    for (int r = 0; r < RPI; ++r) t += part[r][c];
    means[(static_cast<size_t>(o) * nb + blk) * D + c] =
        __ddiv_rn(__ll2double_rn(t), static_cast<double>(n1 - n0) * 16777216.0);
  }
}

// scores[bh][i][j] for a 64 x 64 tile of (query block i, key tile j) per CTA; grid
// (ceil(nkt/64), ceil(nsb/64), B*H), 256 threads, each 4 x 4 scores (rows ty + 16 r, columns
// tx + 16 s) from 8 shared-memory loads per channel.  The means pass through shared memory 32
// channels at a time, channel-major (a warp's loads are broadcasts or 16 consecutive doubles);
// every score is still one fma per channel in channel order.  Causal: tiles no query block of
// the CTA may see are skipped (their scores are never read).
constexpr int kScoreTile = 64;
constexpr int kScoreChunk = 32;
template <int D>
__global__ void __launch_bounds__(256) block_scores_kernel(const double* __restrict__ qmeans,
                                                           const double* __restrict__ kmeans,
                                                           int H, int Hkv, int nsb, int nkt,
                                                           int causal,
                                                           double* __restrict__ scores) {
  __shared__ double qs[kScoreChunk][kScoreTile + 1];
  __shared__ double ks[kScoreChunk][kScoreTile + 1];
  const long long bh = blockIdx.z;
  const long long bg = (bh / H) * Hkv + (bh % H) / (H / Hkv);
  const int i0 = blockIdx.y * kScoreTile, j0 = blockIdx.x * kScoreTile;
  if (causal && j0 > 2 * (i0 + kScoreTile - 1) + 1) return;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  double acc[4][4];
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[r][c] = 0.0;
  for (int c0 = 0; c0 < D; c0 += kScoreChunk) {
    __syncthreads();
    for (int e = threadIdx.x; e < kScoreTile * kScoreChunk; e += 256) {
      const int r = e / kScoreChunk, c = e % kScoreChunk;
      qs[c][r] = i0 + r < nsb ? qmeans[(static_cast<size_t>(bh) * nsb + i0 + r) * D + c0 + c] : 0.0;
      ks[c][r] = j0 + r < nkt ? kmeans[(static_cast<size_t>(bg) * nkt + j0 + r) * D + c0 + c] : 0.0;
    }
    __syncthreads();
#pragma unroll 4
    for (int c = 0; c < kScoreChunk; ++c) {
      double qv[4], kv[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) qv[r] = qs[c][ty + 16 * r];
#pragma unroll
      for (int u = 0; u < 4; ++u) kv[u] = ks[c][tx + 16 * u];
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int u = 0; u < 4; ++u) acc[r][u] = __fma_rn(qv[r], kv[u], acc[r][u]);
    }
  }
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int ii = ty + 16 * r;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int jj = tx + 16 * u;
      if (i0 + ii < nsb && j0 + jj < nkt)
        scores[(static_cast<size_t>(bh) * nsb + i0 + ii) * nkt + j0 + jj] = acc[r][u];
    }
  }
}

// Selection, one warp per query block (block i = blockIdx.x * 8 + warp of head blockIdx.y):
// lane l holds the scores of tiles l, l + 32, ... (up to kSelMaxTiles / 32 of them) in
// registers, and each of the topk rounds takes the warp-wide best unpicked candidate (highest
// score, lowest index among equal scores) by shuffles.  list[bh][i][0..count) ascending; entries
// past count are left alone.
constexpr int kSelMaxTiles = 1024;  // N <= 2^17 keys
__global__ void __launch_bounds__(256) block_select_kernel(const double* __restrict__ scores,
                                                           int nsb, int nkt, int causal, int topk,
                                                           int* __restrict__ list,
                                                           int* __restrict__ count) {
  constexpr int PER = kSelMaxTiles / 32;
  const int lane = threadIdx.x & 31;
  const int i = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (i >= nsb) return;
  const long long bh = blockIdx.y;
  const double* sc = scores + (static_cast<size_t>(bh) * nsb + i) * nkt;
  int last = causal ? 2 * i + 1 : nkt - 1;  // highest key tile the block may see
  if (last > nkt - 1) last = nkt - 1;
  const int lo_forced = causal ? 2 * i : nkt;  // tiles lo_forced .. last are always kept
  double v[PER];
  uint32_t picked = 0;                         // bit t: tile lane + 32 t taken
#pragma unroll
  for (int t = 0; t < PER; ++t) {
    const int j = lane + 32 * t;
    v[t] = j <= last ? sc[j] : 0.0;
    if (j >= lo_forced && j <= last) picked |= 1u << t;
  }
  for (int r = 0; r < topk; ++r) {
    // the lane's best unpicked candidate, as four independent scans over t = p (mod 4) (each
    // keeps the lowest tile among equal scores), merged with the same rule; stripes past the
    // last visible tile are skipped (warp-uniform)
    double ps[4] = {0.0, 0.0, 0.0, 0.0};
    int pj[4] = {-1, -1, -1, -1};
#pragma unroll
    for (int tg = 0; tg < PER / 4; ++tg) {
      if (128 * tg > last) break;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int t = 4 * tg + q;
        const int j = lane + 32 * t;
        if (j <= last && !((picked >> t) & 1u) && (pj[q] < 0 || v[t] > ps[q])) {
          ps[q] = v[t];
          pj[q] = j;
        }
      }
    }
    double bs = ps[0];
    int bj = pj[0];
#pragma unroll
    for (int q = 1; q < 4; ++q) {
      if (pj[q] >= 0 && (bj < 0 || ps[q] > bs || (ps[q] == bs && pj[q] < bj))) {
        bs = ps[q];
        bj = pj[q];
      }
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
    if (bj < 0) break;  // warp-uniform: every candidate taken
    if ((bj & 31) == lane) picked |= 1u << (bj >> 5);
  }
  // ascending list: tiles in order t-major within each lane are lane + 32 t; a warp-wide prefix
  // count per 32-tile stripe gives each picked tile its position
  int* out = list + (static_cast<size_t>(bh) * nsb + i) * nkt;
  int base = 0;
#pragma unroll
  for (int t = 0; t < PER; ++t) {
    if (32 * t > last) break;
    const bool p = (picked >> t) & 1u;
    const unsigned m = __ballot_sync(0xFFFFFFFFu, p);
    if (p) out[base + __popc(m & ((1u << lane) - 1u))] = lane + 32 * t;
    base += __popc(m);
  }
  if (lane == 0) count[static_cast<size_t>(bh) * nsb + i] = base;
}

}  // namespace qattn
