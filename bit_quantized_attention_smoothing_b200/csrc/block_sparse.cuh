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
// registers as order-preserving 64-bit keys (binary64 bits with the sign flipped, negative values
// complemented; -0 taken as +0, so equal scores give equal keys).  The topk candidates with the
// highest scores, lowest index among equal scores, are found without ranking them: a bisection
// over the key bits (from the highest bit on which the candidates differ) finds the topk-th
// largest key T, with one warp-wide count per bit; every candidate above T is taken, and of those
// equal to T the lowest-indexed ones.  list[bh][i][0..count) ascending; entries past count are
// left alone.
constexpr int kSelMaxTiles = 1024;  // N <= 2^17 keys
__device__ __forceinline__ uint64_t score_key(double v) {
  const uint64_t u = static_cast<uint64_t>(__double_as_longlong(v + 0.0));
  return (u >> 63) ? ~u : (u | (1ull << 63));
}
__global__ void __launch_bounds__(256) block_select_kernel(const double* __restrict__ scores,
                                                           int nsb, int nkt, int causal, int topk,
                                                           int* __restrict__ list,
                                                           int* __restrict__ count) {
  constexpr int PER = kSelMaxTiles / 32;
  constexpr uint32_t kFull = 0xFFFFFFFFu;
  const int lane = threadIdx.x & 31;
  const int i = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (i >= nsb) return;
  const long long bh = blockIdx.y;
  const double* sc = scores + (static_cast<size_t>(bh) * nsb + i) * nkt;
  int last = causal ? 2 * i + 1 : nkt - 1;  // highest key tile the block may see
  if (last > nkt - 1) last = nkt - 1;
  const int lo_forced = causal ? 2 * i : nkt;  // tiles lo_forced .. last are always kept
  const int cand_end = min(last + 1, lo_forced);  // candidates: tiles 0 .. cand_end - 1
  const int kk = min(topk, cand_end);
  uint64_t key[PER];
  uint32_t picked = 0;  // bit t: tile lane + 32 t taken
  uint32_t cand = 0;    // bit t: tile lane + 32 t is a candidate
#pragma unroll
  for (int t = 0; t < PER; ++t) {
    const int j = lane + 32 * t;
    key[t] = j < cand_end ? score_key(sc[j]) : 0ull;
    if (j < cand_end) cand |= 1u << t;
    if (j >= lo_forced && j <= last) picked |= 1u << t;
  }
  if (kk == cand_end) {
    picked |= cand;
  } else if (kk > 0) {
    // bits common to every candidate key fix the top of T
    uint64_t k_and = ~0ull, k_or = 0ull;
#pragma unroll
    for (int t = 0; t < PER; ++t) {
      if (32 * t >= cand_end) break;
      if ((cand >> t) & 1u) {
        k_and &= key[t];
        k_or |= key[t];
      }
    }
    const uint32_t and_hi = __reduce_and_sync(kFull, static_cast<uint32_t>(k_and >> 32));
    const uint32_t and_lo = __reduce_and_sync(kFull, static_cast<uint32_t>(k_and));
    const uint32_t or_hi = __reduce_or_sync(kFull, static_cast<uint32_t>(k_or >> 32));
    const uint32_t or_lo = __reduce_or_sync(kFull, static_cast<uint32_t>(k_or));
    const uint64_t kand = (static_cast<uint64_t>(and_hi) << 32) | and_lo;
    const uint64_t diff = kand ^ ((static_cast<uint64_t>(or_hi) << 32) | or_lo);
    const int top = diff ? 63 - __clzll(static_cast<long long>(diff)) : -1;
    // T = the largest key with at least kk candidate keys >= T
    uint64_t T = top >= 63 ? 0ull : (kand >> (top + 1)) << (top + 1);
    for (int bit = top; bit >= 0; --bit) {
      const uint64_t thr = T | (1ull << bit);
      uint32_t n = 0;
#pragma unroll
      for (int t = 0; t < PER; ++t) {
        if (32 * t >= cand_end) break;
        n += ((cand >> t) & 1u) && key[t] >= thr ? 1u : 0u;
      }
      if (__reduce_add_sync(kFull, n) >= static_cast<uint32_t>(kk)) T = thr;
    }
    // every candidate above T, then the lowest-indexed ones equal to T
    uint32_t n_gt = 0;
#pragma unroll
    for (int t = 0; t < PER; ++t) {
      if (32 * t >= cand_end) break;
      if (((cand >> t) & 1u) && key[t] > T) {
        picked |= 1u << t;
        ++n_gt;
      }
    }
    int need = kk - static_cast<int>(__reduce_add_sync(kFull, n_gt));
#pragma unroll
    for (int t = 0; t < PER; ++t) {
      if (need <= 0 || 32 * t >= cand_end) break;
      const uint32_t eq = __ballot_sync(kFull, ((cand >> t) & 1u) && key[t] == T);
      const int ne = __popc(eq);
      const uint32_t take = ne <= need ? eq : [&] {
        // the need lowest set bits of eq
        uint32_t m = eq, r = 0;
        for (int x = 0; x < need; ++x) {
          const uint32_t lowbit = m & (~m + 1u);
          r |= lowbit;
          m ^= lowbit;
        }
        return r;
      }();
      if ((take >> lane) & 1u) picked |= 1u << t;
      need -= __popc(take);
    }
  }
  // ascending list: tiles in order t-major within each lane are lane + 32 t; a warp-wide prefix
  // count per 32-tile stripe gives each picked tile its position
  int* out = list + (static_cast<size_t>(bh) * nsb + i) * nkt;
  int base = 0;
#pragma unroll
  for (int t = 0; t < PER; ++t) {
    if (32 * t > last) break;
    const bool p = (picked >> t) & 1u;
    const unsigned m = __ballot_sync(kFull, p);
    if (p) out[base + __popc(m & ((1u << lane) - 1u))] = lane + 32 * t;
    base += __popc(m);
  }
  if (lane == 0) count[static_cast<size_t>(bh) * nsb + i] = base;
}

}  // namespace qattn
