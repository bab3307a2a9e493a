// quant.cuh -- smoothing of K and per-block INT8 quantization of Q and K' (SageAttention summary
// page, aibr.jp/archives/102657, sec. 3: smooth K, quantize to INT8).  The forward's two launches
// (Q's quantization with the K channel sums, then K's smoothing and quantization) are bound by
// HBM bandwidth: 16-byte coalesced loads, warp-shuffle reductions; Q is read once, K twice (the
// second time mostly from L2).
//
// Bit-exactness.  The codes and scales are exact functions of the inputs:
//  * the channel sums are exact int64 sums of K * 2^24 (every fp16 value is an integer multiple of
//    2^-24), so the order of the atomic additions does not matter;
//  * mean = (float)((double)sum / (N * 2^24)) with correctly rounded operations;
//  * K' = (float)K - mean, amax, scale = amax / 127 are single correctly rounded binary32 ops;
//  * code = rint(x / scale): computed as rint(x * (1/scale)), which equals rint(x / scale) unless
//    x / scale lies within 2^-13 of a half-integer: for |x / scale| <= 127 the product carries two
//    roundings of relative size <= 2^-24 each (< 2^-16 absolute) and the correctly rounded
//    quotient one more (< 2^-17), so the two differ by less than 2^-15; those rare elements take
//    the correctly rounded division.
// Build without fast-math so that division, reciprocal and conversions round to nearest-even
// and subnormals are kept.
#pragma once

#include <cuda_fp16.h>
#include <cstdint>

namespace qattn {

constexpr int kQBlock = 128;  // Q quantization block: 128 consecutive rows of one head
constexpr int kKBlock = 64;   // K quantization block: 64 consecutive rows of one kv head
constexpr int kSumRowsPerCta = 512;
constexpr float kRoundBias = 12582912.0f;  // 1.5 * 2^23

__device__ __forceinline__ float half_bits_to_float(uint32_t bits16) {
  return __half2float(__ushort_as_half(static_cast<unsigned short>(bits16)));
}

// ---------------------------------------------------------------------------------------------
// K channel sums: sums[bg * D + c] += sum over rows kSumRowsPerCta * chunk .. of K[bg, n, c] * 2^24
// (exact), one 256-thread CTA.  sums must be zeroed beforehand.
// ---------------------------------------------------------------------------------------------
template <int D>
__device__ __forceinline__ void k_channel_sums_cta(const uint16_t* __restrict__ k, int N, int bg,
                                                   int chunk, long long* __restrict__ sums) {
  constexpr int VPR = D / 8;            // 16-byte vectors per row
  constexpr int RPI = 256 / VPR;        // rows per iteration of the CTA
  __shared__ long long red[RPI][D];
  const int tid = threadIdx.x;
  const int cg = tid % VPR;
  const int r_in = tid / VPR;
  const int n0 = chunk * kSumRowsPerCta;
  const int n1 = min(N, n0 + kSumRowsPerCta);
  const uint4* base = reinterpret_cast<const uint4*>(k + static_cast<size_t>(bg) * N * D);
  long long acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0;
  for (int n = n0 + r_in; n < n1; n += RPI) {
    const uint4 v = __ldg(base + static_cast<size_t>(n) * VPR + cg);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      acc[2 * e] += __float2ll_rn(half_bits_to_float(w[e] & 0xFFFFu) * 16777216.0f);
      acc[2 * e + 1] += __float2ll_rn(half_bits_to_float(w[e] >> 16) * 16777216.0f);
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) red[r_in][cg * 8 + e] = acc[e];
  __syncthreads();
  for (int c = tid; c < D; c += 256) {
    long long s = 0;
#pragma unroll 4
    for (int r = 0; r < RPI; ++r) s += red[r][c];
    atomicAdd(reinterpret_cast<unsigned long long*>(sums + static_cast<size_t>(bg) * D + c),
              static_cast<unsigned long long>(s));
  }
}

// grid (B*Hkv, ceil(N / kSumRowsPerCta)), 256 threads.
template <int D>
__global__ void __launch_bounds__(256) k_channel_sums_kernel(const uint16_t* __restrict__ k, int N,
                                                             long long* __restrict__ sums) {
  k_channel_sums_cta<D>(k, N, blockIdx.x, blockIdx.y, sums);
}

// rint(x / s) for x, s > 0 as described in the file header.
__device__ __forceinline__ float quant_code(float x, float s, float rcp) {
  const float y = x * rcp;
  const float f = y - floorf(y);
  float t = y;
  if (fabsf(f - 0.5f) < 1.220703125e-4f) t = __fdiv_rn(x, s);  // within 2^-13 of a tie
  float r = rintf(t);
  r = fminf(fmaxf(r, -127.0f), 127.0f);
  return r;
}

__device__ __forceinline__ uint32_t pack4_i8(float a, float b, float c, float d) {
  const uint32_t ua = static_cast<uint32_t>(static_cast<int>(a)) & 0xFFu;
  const uint32_t ub = static_cast<uint32_t>(static_cast<int>(b)) & 0xFFu;
  const uint32_t uc = static_cast<uint32_t>(static_cast<int>(c)) & 0xFFu;
  const uint32_t ud = static_cast<uint32_t>(static_cast<int>(d)) & 0xFFu;
  return ua | (ub << 8) | (uc << 16) | (ud << 24);
}

// One quantization block of R rows x D channels, 256 threads.  src: fp16 rows of the block
// (head base + r0 * D); mean: per-channel smoothing offsets in shared memory (K) or nullptr (Q).
// One quantization block of R rows x D values per 256-thread CTA: x = fp16 value (minus the
// channel mean for K), amax over the block, scale = amax / 127, codes rint(x * (1 / scale)); a
// group of 8 values holding one within 2^-13 of a half-integer is recomputed with quant_code
// (the correctly rounded quotient decides there), so every code is rint(x / scale).  Values stay
// as fp16 pairs in registers between the two passes (the mean is subtracted again when needed),
// keeping the CTA small enough for several to share an SM.
template <int D, int R>
__device__ __forceinline__ void quantize_block_cta(const uint16_t* __restrict__ src, int rows,
                                                   const float* mean_s, int8_t* __restrict__ dst,
                                                   float* __restrict__ scale_out, float* red) {
  constexpr int VPR = D / 8;
  constexpr int VPT = R * VPR / 256;  // vectors per thread
  static_assert(256 % VPR == 0, "a thread keeps one column group");
  const int tid = threadIdx.x;
  const int cg = tid % VPR;
  float m[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) m[e] = mean_s ? mean_s[cg * 8 + e] : 0.0f;
  // every load issued before any is used: rows past the block's end read its first row and are
  // dropped afterwards
  uint4 v[VPT];
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int vi = tid + i * 256;
    v[i] = __ldg(reinterpret_cast<const uint4*>(src) + (vi / VPR < rows ? vi : cg));
  }
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    if ((tid + i * 256) / VPR >= rows) continue;
    const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      amax = fmaxf(amax, fabsf(half_bits_to_float(w[e] & 0xFFFFu) - m[2 * e]));
      amax = fmaxf(amax, fabsf(half_bits_to_float(w[e] >> 16) - m[2 * e + 1]));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
  if ((tid & 31) == 0) red[tid >> 5] = amax;
  __syncthreads();
  amax = red[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) amax = fmaxf(amax, red[w]);
  const float s = __fdiv_rn(amax, 127.0f);
  const float rcp = amax > 0.0f ? __frcp_rn(s) : 0.0f;
  if (tid == 0) *scale_out = amax > 0.0f ? s : 0.0f;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int vi = tid + i * 256;
    const bool in = vi / VPR < rows;
    const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
    float x[8];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      x[2 * e] = half_bits_to_float(w[e] & 0xFFFFu) - m[2 * e];
      x[2 * e + 1] = half_bits_to_float(w[e] >> 16) - m[2 * e + 1];
    }
    // rint(y) by adding 1.5 * 2^23 (the sum rounds to nearest-even, leaving rint(y) in two's
    // complement in the low mantissa bits for |y| < 2^22; |y| <= 127 here), on the FMA pipe
    // instead of a rounding and a float-to-int conversion per value
    uint32_t t[8];
    bool near_tie = false;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float y = __fmul_rn(x[e], rcp);
      const float tb = __fadd_rn(y, kRoundBias);
      const float ry = __fadd_rn(tb, -kRoundBias);
      near_tie |= fabsf(y - ry) > 0.4998779296875f;  // within 2^-13 of a half-integer
      t[e] = __float_as_uint(tb);
    }
    // the low byte of each biased sum is the int8 code
    uint2 out;
    out.x = __byte_perm(__byte_perm(t[0], t[1], 0x0040), __byte_perm(t[2], t[3], 0x0040), 0x5410);
    out.y = __byte_perm(__byte_perm(t[4], t[5], 0x0040), __byte_perm(t[6], t[7], 0x0040), 0x5410);
    if (__any_sync(0xFFFFFFFFu, near_tie) && near_tie) {
      float q[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) q[e] = quant_code(x[e], s, rcp);
      out.x = pack4_i8(q[0], q[1], q[2], q[3]);
      out.y = pack4_i8(q[4], q[5], q[6], q[7]);
    }
    if (in) reinterpret_cast<uint2*>(dst)[vi] = out;
  }
}

// The second pre-pass launch: K' = K - mean and its per-64-row INT8 quantization, one CTA per K
// block (mean from the exact channel sums, written to k_mean by each kv group's first block when
// k_mean is not null).
template <int D>
__global__ void __launch_bounds__(256) k_quantize_kernel(
    const uint16_t* __restrict__ k, int N, int nkb, const long long* __restrict__ sums,
    int8_t* __restrict__ k_i8, float* __restrict__ k_scale, float* __restrict__ k_mean) {
  __shared__ float mean_s[D];
  __shared__ float red[8];
  const long long kblk = blockIdx.x;
  const long long bg = kblk / nkb;
  const int kb = static_cast<int>(kblk % nkb);
  if (threadIdx.x < D) {
    const long long s = sums[bg * D + threadIdx.x];
    const double den = static_cast<double>(N) * 16777216.0;
    const float mu = __double2float_rn(__ddiv_rn(__ll2double_rn(s), den));
    mean_s[threadIdx.x] = mu;
    if (kb == 0 && k_mean != nullptr) k_mean[bg * D + threadIdx.x] = mu;
  }
  __syncthreads();
  const int r0 = kb * kKBlock;
  const int rows = min(kKBlock, N - r0);
  const size_t off = (static_cast<size_t>(bg) * N + r0) * D;
  quantize_block_cta<D, kKBlock>(k + off, rows, mean_s, k_i8 + off, k_scale + kblk, red);
}

// The first of the forward's two pre-pass launches: Q's quantization (which needs no K mean) and
// the K channel sums in one grid of nq + nsum CTAs.  CTAs 0 .. nq-1 quantize Q's 128-row blocks;
// the last nsum sum K rows (chunk index % nchunk of kv group index / nchunk), so that K has just
// passed through L2 when the second launch (k_quantize_kernel) reads it again.
template <int D>
__global__ void __launch_bounds__(256) q_quant_k_sums_kernel(
    const uint16_t* __restrict__ q, const uint16_t* __restrict__ k, int N, int nqb, long long nq,
    int nchunk, int8_t* __restrict__ q_i8, float* __restrict__ q_scale,
    long long* __restrict__ sums) {
  __shared__ float red[8];
  const long long blk = blockIdx.x;
  if (blk < nq) {
    const long long bh = blk / nqb;
    const int qb = static_cast<int>(blk % nqb);
    const int r0 = qb * kQBlock;
    const int rows = min(kQBlock, N - r0);
    const size_t off = (static_cast<size_t>(bh) * N + r0) * D;
    quantize_block_cta<D, kQBlock>(q + off, rows, nullptr, q_i8 + off, q_scale + blk, red);
  } else {
    const long long i = blk - nq;
    k_channel_sums_cta<D>(k, N, static_cast<int>(i / nchunk), static_cast<int>(i % nchunk), sums);
  }
}

}  // namespace qattn
