// nvfp4.cuh -- NVFP4 quantization, the operand format of the FP4 path of the ThriftAttention page
// ("ThriftAttention: Selective Mixed Precision for Long-Context FP4 Attention",
// gist.science/ja/paper/2605.23081, method section, "FP4 path": the blocks that are not promoted
// to FP16 are computed in FP4 with the NVFP4 micro-scaling format of Blackwell GPUs).
//
// The page names the format without defining it; this follows NVIDIA's published definition:
// FP4 E2M1 elements in blocks of 16, one unsigned FP8 E4M3 scale per block, one binary32 scale per
// tensor, here per (batch, head) slice.  With every binary32 operation rounded once to nearest-even:
//   x'   = (float)x - mean[c]                    (mean optional: the smoothing of K)
//   amax = max |x'| over the slice,  g = amax / 2688             (2688 = 448 * 6)
//   per block: s = E4M3(bmax / (6 * g)),  sc = E4M3value(s) * g,  code_i = E2M1(x'_i / sc)
// Both conversions are the hardware's cvt.rn.satfinite (nearest-even, saturating to 448 and 6).
// A block whose scale rounds to 0, and every block of a slice with amax == 0, gets scale byte 0
// and codes 0; a code whose value is zero is written as +0.  Two codes per byte, the element with
// the lower index in bits 0-3.
//
// Three launches, all bound by HBM bandwidth: the slice maxima (atomicMax on the bit patterns of
// non-negative floats, which order like unsigned integers, into the zeroed gscale buffer), the
// quantization (which derives g from the maximum itself), and g = amax / 2688 in place.
#pragma once

#include <cuda_fp16.h>
#include <cstdint>

namespace qattn {

constexpr float kNvfp4Div = 2688.0f;  // largest E4M3 value (448) times largest E2M1 value (6)
constexpr int kNvfp4Tile = 64;        // transposed quantizer: rows and channels per CTA

// Eight binary32 values to eight E2M1 codes, v[0] in bits 0-3 ... v[7] in bits 28-31.  The cvt
// places its first source in the upper nibble of the byte, so each pair is passed high first.
__device__ __forceinline__ uint32_t e2m1x8(const float* v) {
  uint32_t r;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(r)
      : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
  // a zero magnitude is written as +0: nibble magnitude m in 0..7, m + 7 sets bit 3 iff m >= 1
  const uint32_t mag = r & 0x77777777u;
  const uint32_t nonzero = (mag + 0x77777777u) & 0x88888888u;
  return mag | (r & nonzero);
}

// E4M3 byte of t >= 0 (nearest-even, saturating to 448).
__device__ __forceinline__ uint32_t ue4m3_byte(float t) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(t));
  return r & 0xFFu;
}

// Exact binary32 value of an E4M3 byte with sign 0 (exponent bias 7, subnormals m * 2^-9).
__device__ __forceinline__ float ue4m3_value(uint32_t s) {
  const uint32_t e = s >> 3, m = s & 7u;
  return e ? __uint_as_float(((e + 120u) << 23) | (m << 20)) : static_cast<float>(m) * 0.001953125f;
}

// One block of 16 smoothed values with the slice's global scale g.
__device__ __forceinline__ void nvfp4_block16(const float (&x)[16], float g, uint2& codes,
                                              uint32_t& scale) {
  float bmax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) bmax = fmaxf(bmax, fabsf(x[i]));
  uint32_t s = 0;
  if (g > 0.0f) s = ue4m3_byte(__fdiv_rn(bmax, __fmul_rn(6.0f, g)));
  scale = s;
  if (s == 0) {
    codes = make_uint2(0u, 0u);
    return;
  }
  const float sc = __fmul_rn(ue4m3_value(s), g);
  float q[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) q[i] = __fdiv_rn(x[i], sc);
  codes = make_uint2(e2m1x8(q), e2m1x8(q + 8));
}

__device__ __forceinline__ void unpack8_minus(const uint4& v, const float* m, float* out) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    out[2 * e] = __fsub_rn(__half2float(__ushort_as_half(static_cast<unsigned short>(w[e] & 0xFFFFu))), m[2 * e]);
    out[2 * e + 1] = __fsub_rn(__half2float(__ushort_as_half(static_cast<unsigned short>(w[e] >> 16))), m[2 * e + 1]);
  }
}

// The slice's 8 means starting at channel c (zeros without smoothing; x - 0 is x exactly).
__device__ __forceinline__ void load_mean8(const float* __restrict__ mean, int c, float* m) {
  if (mean) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(mean + c));
    const float4 b = __ldg(reinterpret_cast<const float4*>(mean + c + 4));
    m[0] = a.x; m[1] = a.y; m[2] = a.z; m[3] = a.w; m[4] = b.x; m[5] = b.y; m[6] = b.z; m[7] = b.w;
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e) m[e] = 0.0f;
  }
}

// amax_bits[s] = max(amax_bits[s], bits of max |x'| over this CTA's share of slice s).
// grid (gx, S), 256 threads; C % 16 == 0.
__global__ void __launch_bounds__(256) nvfp4_amax_kernel(const uint16_t* __restrict__ x,
                                                         const float* __restrict__ mean, int R,
                                                         int C, unsigned* __restrict__ amax_bits) {
  __shared__ float red[8];
  const int s = blockIdx.y;
  const size_t nvec = static_cast<size_t>(R) * C / 8;
  const uint4* base = reinterpret_cast<const uint4*>(x + static_cast<size_t>(s) * R * C);
  const float* ms = mean ? mean + static_cast<size_t>(s) * C : nullptr;
  float amax = 0.0f;
  for (size_t i = static_cast<size_t>(blockIdx.x) * 256 + threadIdx.x; i < nvec;
       i += static_cast<size_t>(gridDim.x) * 256) {
    const uint4 v = __ldg(base + i);
    float m[8], f[8];
    load_mean8(ms, static_cast<int>((i * 8) % C), m);
    unpack8_minus(v, m, f);
#pragma unroll
    for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(f[e]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  if (threadIdx.x == 0) {
#pragma unroll
    for (int w = 1; w < 8; ++w) amax = fmaxf(amax, red[w]);
    atomicMax(amax_bits + s, __float_as_uint(amax));
  }
}

// Blocks along the channels: one thread per 16 consecutive values of a row (block b covers
// elements 16 b .. 16 b + 15 of the contiguous [S][R][C] tensor).  codes: 8 bytes per block,
// scales: 1 byte per block, both in block order.
__global__ void __launch_bounds__(256) nvfp4_quant_rows_kernel(
    const uint16_t* __restrict__ x, const float* __restrict__ mean, int R, int C, long long total,
    const unsigned* __restrict__ amax_bits, uint8_t* __restrict__ codes,
    uint8_t* __restrict__ scales) {
  const long long per_slice = static_cast<long long>(R) * (C / 16);
  for (long long b = static_cast<long long>(blockIdx.x) * 256 + threadIdx.x; b < total;
       b += static_cast<long long>(gridDim.x) * 256) {
    const int s = static_cast<int>(b / per_slice);
    const int c0 = static_cast<int>(b % (C / 16)) * 16;
    const float g = __fdiv_rn(__uint_as_float(__ldg(amax_bits + s)), kNvfp4Div);
    const uint4* src = reinterpret_cast<const uint4*>(x) + 2 * b;
    const uint4 v0 = __ldg(src), v1 = __ldg(src + 1);
    const float* ms = mean ? mean + static_cast<size_t>(s) * C : nullptr;
    float m[8], xv[16];
    load_mean8(ms, c0, m);
    unpack8_minus(v0, m, xv);
    load_mean8(ms, c0 + 8, m);
    unpack8_minus(v1, m, xv + 8);
    uint2 cw;
    uint32_t sb;
    nvfp4_block16(xv, g, cw, sb);
    reinterpret_cast<uint2*>(codes)[b] = cw;
    scales[b] = static_cast<uint8_t>(sb);
  }
}

// Blocks along the rows, written transposed: CTA (bx, by, s) quantizes rows 64 bx .. 64 bx + 63
// of channels 64 by .. 64 by + 63 of slice s.  Rows R .. Rp - 1 are zero padding (Rp = R rounded
// up to 128).  codes [S][C][Rp/2], scales [S][C][Rp/16].  256 threads; C % 16 == 0.
__global__ void __launch_bounds__(256) nvfp4_quant_cols_kernel(
    const uint16_t* __restrict__ x, const float* __restrict__ mean, int R, int C, int Rp,
    const unsigned* __restrict__ amax_bits, uint8_t* __restrict__ codes,
    uint8_t* __restrict__ scales) {
  constexpr int T = kNvfp4Tile;
  __shared__ float tile[T][T + 1];
  __shared__ uint2 cstage[T][4];
  __shared__ uint8_t sstage[T][4];
  const int s = blockIdx.z;
  const int r0 = blockIdx.x * T, c0 = blockIdx.y * T;
  const float* ms = mean ? mean + static_cast<size_t>(s) * C : nullptr;
  for (int i = threadIdx.x; i < T * T / 8; i += 256) {
    const int rr = i / (T / 8), cv = (i % (T / 8)) * 8;
    const int r = r0 + rr, c = c0 + cv;
    float f[8];
    if (r < R && c < C) {  // C % 16 == 0: the whole 8-vector is inside the row
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(
          x + (static_cast<size_t>(s) * R + r) * C + c));
      float m[8];
      load_mean8(ms, c, m);
      unpack8_minus(v, m, f);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) f[e] = 0.0f;
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) tile[rr][cv + e] = f[e];
  }
  __syncthreads();
  {
    const int c = threadIdx.x % T, grp = threadIdx.x / T;
    const float g = __fdiv_rn(__uint_as_float(__ldg(amax_bits + s)), kNvfp4Div);
    float xv[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) xv[i] = tile[grp * 16 + i][c];
    uint2 cw;
    uint32_t sb;
    nvfp4_block16(xv, g, cw, sb);
    cstage[c][grp] = cw;
    sstage[c][grp] = static_cast<uint8_t>(sb);
  }
  __syncthreads();
  {
    const int cc = threadIdx.x / 4, gg = threadIdx.x % 4;
    const int r = r0 + gg * 16;
    if (c0 + cc < C && r < Rp) {
      const size_t row = static_cast<size_t>(s) * C + c0 + cc;
      *reinterpret_cast<uint2*>(codes + row * (Rp / 2) + r / 2) = cstage[cc][gg];
      scales[row * (Rp / 16) + r / 16] = sstage[cc][gg];
    }
  }
}

// mean[i] = (float)((double)sums[i] / (N * 2^24)): the smoothing mean from the exact channel sums
// of K * 2^24, one binary64 division and one rounding to binary32 (as the INT8 path's quantizer).
__global__ void k_mean_from_sums_kernel(const long long* __restrict__ sums, int N, int n,
                                        float* __restrict__ mean) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n)
    mean[i] = __double2float_rn(__ddiv_rn(__ll2double_rn(sums[i]), static_cast<double>(N) * 16777216.0));
}

// gscale[s] = amax / 2688 in place (gscale holds the maxima as floats on entry).
__global__ void nvfp4_finalize_kernel(float* __restrict__ gscale, int S) {
  const int s = blockIdx.x * blockDim.x + threadIdx.x;
  if (s < S) gscale[s] = __fdiv_rn(gscale[s], kNvfp4Div);
}

}  // namespace qattn
