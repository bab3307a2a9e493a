// adaptive.cuh -- the parts of the adaptive quantization (SageAttention summary page,
// aibr.jp/archives/102657: dialogue and sec. 2-4, the quantization strength chosen per layer or
// head so that important parts keep precision while the rest runs faster) outside the attention
// kernel: V in FP8 E4M3 for the coarser P V variant, and the per-group cosine similarity that
// chooses between the variants.
//
// V in E4M3, per (batch, kv head) slice: sV = amax / 448 (binary32 division; 448 is the largest
// E4M3 value), code = E4M3(v / sV) (binary32 division, the hardware's cvt.rn.satfinite:
// nearest-even, saturating at 448), a zero code written as +0; stored transposed, [slice][channel]
// rows of Np bytes (Np = N rounded up to 128, zero padding), the K-major B operand of the FP8
// P V product.  Bound by HBM bandwidth: a slice-maximum pass (nvfp4_amax_kernel) and one
// transposing pass through a shared-memory tile.
#pragma once

#include <cuda_fp16.h>
#include <cstdint>

#include "nvfp4.cuh"  // nvfp4_amax_kernel, unpack8_minus, load_mean8

namespace qattn {

constexpr float kE4m3Max = 448.0f;
constexpr int kV8Tile = 64;  // rows and channels of one CTA's transposing tile

// scale[s] = amax / 448 in place (scale holds the slice maxima as floats on entry).
__global__ void v_fp8_scale_kernel(float* __restrict__ scale, int S) {
  const int s = blockIdx.x * blockDim.x + threadIdx.x;
  if (s < S) scale[s] = __fdiv_rn(scale[s], kE4m3Max);
}

// E4M3 byte pair of (hi, lo) with the zero magnitudes written as +0.
__device__ __forceinline__ uint32_t e4m3x2_plus0(float hi, float lo) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  uint32_t w = r;
  if ((w & 0x7Fu) == 0u) w &= 0xFF00u;
  if ((w & 0x7F00u) == 0u) w &= 0x00FFu;
  return w;
}

// CTA (bx, by, s) quantizes rows 64 bx .. 64 bx + 63 of channels 64 by .. 64 by + 63 of slice s and
// writes them transposed: vt8[s][c][r], rows R .. Rp - 1 zero.  256 threads; C % 8 == 0.
__global__ void __launch_bounds__(256) v_fp8_quant_kernel(const uint16_t* __restrict__ v, int R,
                                                          int C, int Rp,
                                                          const float* __restrict__ scale,
                                                          uint8_t* __restrict__ vt8) {
  constexpr int T = kV8Tile;
  __shared__ float tile[T][T + 1];
  const int s = blockIdx.z;
  const int r0 = blockIdx.x * T, c0 = blockIdx.y * T;
  for (int i = threadIdx.x; i < T * T / 8; i += 256) {
    const int rr = i / (T / 8), cv = (i % (T / 8)) * 8;
    const int r = r0 + rr, c = c0 + cv;
    float f[8];
    if (r < R && c < C) {  // C % 8 == 0: the whole 8-vector is inside the row
      const uint4 x = __ldg(reinterpret_cast<const uint4*>(v + (static_cast<size_t>(s) * R + r) * C + c));
      float m[8];
      load_mean8(nullptr, c, m);
      unpack8_minus(x, m, f);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) f[e] = 0.0f;
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) tile[rr][cv + e] = f[e];
  }
  __syncthreads();
  // thread: channel c0 + (t % 64), rows r0 + 16 (t / 64) .. + 15 -> 16 bytes of its row of vt8
  const int cc = threadIdx.x % T, grp = threadIdx.x / T;
  const int c = c0 + cc, r = r0 + grp * 16;
  if (c < C && r < Rp) {
    const float sv = __ldg(scale + s);
    uint32_t w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float q[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float x = tile[grp * 16 + 4 * k + e][cc];
        q[e] = sv > 0.0f ? __fdiv_rn(x, sv) : 0.0f;
      }
      w[k] = e4m3x2_plus0(q[1], q[0]) | (e4m3x2_plus0(q[3], q[2]) << 16);
    }
    *reinterpret_cast<uint4*>(vt8 + (static_cast<size_t>(s) * C + c) * Rp + r) =
        make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// Per (batch, kv head) group g: the dot product of two fp16 outputs a and b over the group's rows
// (its H / Hkv query heads, all N rows, d channels) and both squared norms, in binary64:
// acc[3 g + 0] += sum a b, acc[3 g + 1] += sum a a, acc[3 g + 2] += sum b b.  grid (gx, groups),
// 256 threads; a group is a contiguous run of `per` halves.
__global__ void __launch_bounds__(256) group_cosine_parts_kernel(const __half* __restrict__ a,
                                                                 const __half* __restrict__ b,
                                                                 long long per,
                                                                 double* __restrict__ acc) {
  __shared__ double red[3][8];
  const long long base = static_cast<long long>(blockIdx.y) * per;
  double ab = 0.0, aa = 0.0, bb = 0.0;
  for (long long i = static_cast<long long>(blockIdx.x) * 256 + threadIdx.x; i < per;
       i += static_cast<long long>(gridDim.x) * 256) {
    const double x = __half2float(a[base + i]), y = __half2float(b[base + i]);
    ab = fma(x, y, ab);
    aa = fma(x, x, aa);
    bb = fma(y, y, bb);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    ab += __shfl_xor_sync(0xFFFFFFFFu, ab, o);
    aa += __shfl_xor_sync(0xFFFFFFFFu, aa, o);
    bb += __shfl_xor_sync(0xFFFFFFFFu, bb, o);
  }
  const int w = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) {
    red[0][w] = ab;
    red[1][w] = aa;
    red[2][w] = bb;
  }
  __syncthreads();
  if (threadIdx.x < 3) {
    double t = 0.0;
#pragma unroll
    for (int k = 0; k < 8; ++k) t += red[threadIdx.x][k];
    atomicAdd(acc + 3 * static_cast<size_t>(blockIdx.y) + threadIdx.x, t);
  }
}

// variant[g] = 1 (FP8 P V) when cos_g = ab / sqrt(aa bb) >= tau, else 0 (FP16 P V); groups whose
// outputs are both zero count as cosine 1.  cosine[g] (nullable) receives cos_g.
__global__ void choose_variant_kernel(const double* __restrict__ acc, int G, float tau,
                                      uint8_t* __restrict__ variant, float* __restrict__ cosine) {
  const int g = blockIdx.x * blockDim.x + threadIdx.x;
  if (g >= G) return;
  const double ab = acc[3 * g], aa = acc[3 * g + 1], bb = acc[3 * g + 2];
  const double c = (aa > 0.0 && bb > 0.0) ? ab / sqrt(aa * bb) : (aa == bb ? 1.0 : 0.0);
  variant[g] = c >= static_cast<double>(tau) ? 1 : 0;
  if (cosine) cosine[g] = static_cast<float>(c);
}

}  // namespace qattn
