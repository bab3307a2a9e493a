// attn_sm100.cuh -- smoothed-K INT8 attention forward for B200 (sm_100a).
//
// Method (SageAttention summary page, aibr.jp/archives/102657): INT8 Q K^T with exact 32-bit
// accumulation (sec. 3, mma(u8.u8.s32)), FP16 operands for P V (sec. 2-3, mma(f16.f16.f16)),
// FlashAttention-style blockwise online softmax (sec. 4).  The page's kernel is written for
// warp-level mma on an RTX4090; this one is built for Blackwell instead:
//
//  * one CTA owns two 128-row Q tiles of one (batch, head) and streams 128-key K/V tiles;
//  * warp 8 (TMA): loads both Q tiles once, then K (int8) and V (fp16) tiles into a STAGES-deep
//    shared-memory ring (128-byte / 64-byte swizzled tiles, mbarrier transaction counts);
//  * warp 9 (MMA; the whole warp runs the loop on warp-uniform descriptors and one elected lane
//    issues each instruction): S_w = Q_w K^T as tcgen05.mma kind::i8 (M=128, N=128, K=32 per
//    instruction) into tensor memory, then O_w += P_w V as tcgen05.mma kind::f16 with P read
//    from tensor memory (M=128, N=d, K=16), fp32 accumulator in tensor memory; issue order
//    PV_0(j), QK_0(j+1), PV_1(j), QK_1(j+1) so that one Q tile's softmax overlaps the other's MMAs;
//  * warps 0-3 and 4-7 (softmax, one warpgroup per Q tile, thread = score row, setmaxnreg 224):
//    one tcgen05.ld of the row's 128 int32 scores, exact int->float, row maximum per 64-key K
//    scale block (3-input max), dequantization and exp2 argument with packed fp32x2 FMAs, MUFU
//    ex2, P packed to fp16 and written back over the scores' tensor-memory columns, row sum of the
//    fp16-rounded P; lazy rescaling of O only when the running max grows by more than 2^8; P
//    scaled into the top of the fp16 range; the two warpgroups' steps are kept half a step apart
//    (a warp starts a step when the other tile's warp on its SM sub-partition is half through its
//    exponentials), so the MUFU-bound passes of the two tiles alternate instead of contending;
//  * causal: key tiles above the diagonal are never loaded or multiplied; the diagonal tile is
//    masked in registers (a compile-time-specialised path); CTAs are launched heaviest-first;
//  * grouped-query attention: query head h reads kv head h / (H / Hkv); CTAs of the heads that
//    share a kv head are adjacent in launch order so their K/V tiles are reused from L2
//    (non-causal: the pairs of one head run together, since each reads the head's whole K/V).
//
// Tensor memory (512 columns): S_0 [0,128), S_1 [128,256), O_0 [256,256+d), O_1 [256+d,256+2d).
#pragma once

#include <cuda_fp16.h>
#include <climits>
#include <cstdint>

#include "sm100_ptx.cuh"
#include "quant.cuh"

namespace qattn {

constexpr int kBM = 128;     // rows per Q tile
constexpr int kBN = 128;     // keys per K/V tile
constexpr int kAttnThreads = 384;     // 3 warpgroups: softmax Q tile 0, softmax Q tile 1, TMA + MMA
constexpr int kAttnLaunchRegs = 168;   // 384 x 168 = 256 x 224 (softmax) + 128 x 56 (setmaxnreg)
constexpr int kSoftmaxThreads = 256;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: O is rescaled only when the max grows more
// P = 2^(x - m + kPOffset): with the lazy max above, P <= 2^15 < 65504 (fp16 max), and keys down to
// about 2^-(24 + kPOffset) of the row maximum still reach the fp16 P instead of underflowing.  At
// 131072 keys per row, P normalised to 1 loses enough weight in fp16 subnormals to cost ~4e-3 of
// output accuracy; the offset cancels in O / l.
constexpr float kPOffset = 7.0f;
// The FP8 P V variant (adaptive quantization): the running maximum moves only when it grows by
// more than kRescaleThreshold8, and P = 2^(x - m + kPOffset8) <= 2^(4 + 4) = 256, inside E4M3's
// 448 (keys down to ~2^-10 of the running maximum stay normal E4M3 numbers).
constexpr float kRescaleThreshold8 = 4.0f;
constexpr float kPOffset8 = 4.0f;

// P V variants of the attention kernel: FP16 P and V (the product), FP8 E4M3 P and V, or the
// variant chosen per (batch, kv head) group by a table (adaptive quantization).
constexpr int kPvF16 = 0;
constexpr int kPvF8 = 1;
constexpr int kPvTable = 2;

template <int D>
struct AttnCfg {
  static constexpr int kStages = D == 128 ? 3 : 6;
  static constexpr int kQTile = kBM * D;        // bytes, int8
  static constexpr int kKTile = kBN * D;        // bytes, int8
  static constexpr int kVTile = kBN * D * 2;    // bytes, fp16
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = 2 * kQTile;
  static constexpr int kOffV = kOffK + kStages * kKTile;
  static constexpr int kOffBar = kOffV + kStages * kVTile;
  static constexpr int kBarBytes = 256;
  static constexpr int kOffRed = kOffBar + kBarBytes;  // [Q tile][warp] row maxima (fused Q)
  static constexpr int kSmemBytes = kOffRed + 64 + 1024;  // + alignment slack
  // K-major int8 operands: rows of D bytes, 8-row swizzle atoms.
  static constexpr uint32_t kSwQK = D == 128 ? kSwizzle128B : kSwizzle64B;
  static constexpr uint32_t kSboQK = 8 * D;
  // V: MN-major fp16 operand, 64-column (128-byte) swizzled boxes of 128 rows.
  static constexpr uint32_t kVBox = kBN * 128;  // bytes of one 64-column box
  // FP8 variant: V^T tile of D channel rows x 128 keys (E4M3 bytes, 128-byte swizzle), the K-major
  // B operand of P V; it uses the first half of a V stage.
  static constexpr int kV8Tile = D * kBN;
};

struct __align__(16) AttnBars {
  uint64_t q_full;
  uint64_t kv_full[6];
  uint64_t kv_empty[6];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t pv_done[2];
  uint64_t mx_done[2][4];  // warp (w, quadrant) half through a step's exponentials (1 arrive)
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(AttnBars) <= 256, "barrier block");

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// acc + lo + hi, where lo and hi are the two fp16 halves of h2, with the sm_100 mixed-precision
// add (f16 operand widened exactly, one fp32 rounding per add).
__device__ __forceinline__ float add_half2_f32(float acc, uint32_t h2) {
  asm("{\n\t.reg .f16 lo, hi;\n\t"
      "mov.b32 {lo, hi}, %1;\n\t"
      "add.rn.f32.f16 %0, lo, %0;\n\t"
      "add.rn.f32.f16 %0, hi, %0;\n\t}"
      : "+f"(acc)
      : "r"(h2));
  return acc;
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// (d0, d1) = (a0 * b + c, a1 * b + c) as one packed sm_100 fp32x2 FMA (each lane rounds once).
__device__ __forceinline__ void ffma2(float& d0, float& d1, float a0, float a1, float b, float c) {
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %4};\n\tmov.b64 rc, {%5, %5};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b), "f"(c));
}

// (d0, d1) = (a0 + b0, a1 + b1) as one packed sm_100 fp32x2 add.
__device__ __forceinline__ void fadd2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

constexpr float kRoundMagic = 12582912.0f;  // 1.5 * 2^23: x + M rounds x to an integer

__device__ __forceinline__ float scaled_max(float m, float c) {
  return m == -INFINITY ? -INFINITY : m * c;
}

// The int32 score s as the float 1.5 * 2^23 + s, by one integer add on the bit pattern (exact and
// order-preserving for |s| < 2^22; an int8 dot product of length <= 128 stays below 2^21).  The
// float s itself is that value minus kRoundMagic, also exact.
__device__ __forceinline__ float score_biased(uint32_t s) { return __uint_as_float(s + 0x4B400000u); }
static_assert(127 * 127 * 128 < (1 << 22), "biased score conversion range");

// One 128-key step of the softmax for the thread's score row: int32 -> float (exact, see
// score_biased), masked keys (MASK; key offset above lim) -> -inf, row maximum per 64-key K scale block, lazy
// update of the running max m (alpha = rescale factor, need = O must be rescaled), then
// P = 2^(x * c - m + offset) packed as fp16 pairs (even key in the low half) and stored over the
// row's first 64 TMEM columns, and the row sum of the fp16-rounded P.  Once the first 64 keys'
// P are stored, the warp arrives on mx_bar (the other Q tile's softmax waits for it).  MASK is a
// compile-time switch so the unmasked steps carry no per-element tests.
// PV8 (the FP8 P V variant): the running max moves when it grows by more than 4, P =
// 2^(x * c - m + 4) is rounded to E4M3, four keys per tensor-memory column (the lowest key in the
// lowest byte) over the row's first 32 columns, and the row sum takes the E4M3 values.
template <int D, bool MASK, bool PV8>
__device__ __forceinline__ void softmax_row(uint32_t (&sr)[4][32], int lim, float c0, float c1,
                                            bool first, float& m, float& l, float& alpha,
                                            bool& need, uint32_t s_tm, uint64_t* mx_bar) {
  float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      float x = score_biased(sr[c][e]);
      if (MASK && c * 32 + e > lim) x = -INFINITY;
      sr[c][e] = __float_as_uint(x);
    }
#pragma unroll
    for (int e = 0; e < 32; e += 4) {
      float& a = (c < 2) ? ((e & 4) ? mx1 : mx0) : ((e & 4) ? mx3 : mx2);
      a = fmax3(a, __uint_as_float(sr[c][e]), __uint_as_float(sr[c][e + 1]));
      a = fmax3(a, __uint_as_float(sr[c][e + 2]), __uint_as_float(sr[c][e + 3]));
    }
  }
  const float t = fmaxf(scaled_max(fmaxf(mx0, mx1) - kRoundMagic, c0),
                       scaled_max(fmaxf(mx2, mx3) - kRoundMagic, c1));
  const float mn = fmaxf(m, t);
  need = mn > m + (PV8 ? kRescaleThreshold8 : kRescaleThreshold);
  alpha = 1.0f;
  if (need) {
    alpha = first ? 0.0f : ex2_approx(m - mn);
    m = mn;
    l *= alpha;
  }
  const float g = (PV8 ? kPOffset8 : kPOffset) - m;
  float acc0 = 0.0f, acc1 = 0.0f;
#pragma unroll
  for (int hf = 0; hf < 2; ++hf) {
    const float c = hf == 0 ? c0 : c1;
    if constexpr (PV8) {
      uint32_t pk8[16];
#pragma unroll
      for (int q = 0; q < 2; ++q) {
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          uint32_t* w = &sr[2 * hf + q][e];
          float x0, x1, x2, x3, y0, y1, y2, y3;
          fadd2(x0, x1, __uint_as_float(w[0]), __uint_as_float(w[1]), -kRoundMagic, -kRoundMagic);
          fadd2(x2, x3, __uint_as_float(w[2]), __uint_as_float(w[3]), -kRoundMagic, -kRoundMagic);
          ffma2(y0, y1, x0, x1, c, g);
          ffma2(y2, y3, x2, x3, c, g);
          float p0 = ex2_approx(y0), p1 = ex2_approx(y1), p2 = ex2_approx(y2), p3 = ex2_approx(y3);
          if (MASK) {
            if (x0 == -INFINITY) p0 = 0.0f;
            if (x1 == -INFINITY) p1 = 0.0f;
            if (x2 == -INFINITY) p2 = 0.0f;
            if (x3 == -INFINITY) p3 = 0.0f;
          }
          uint16_t lo, hi;
          asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(p1), "f"(p0));
          asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(p3), "f"(p2));
          pk8[q * 8 + (e >> 2)] = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
          // the row sum takes the E4M3 values the P V product uses (exact in fp16)
          uint32_t h01, h23;
          asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h01) : "h"(lo));
          asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h23) : "h"(hi));
          acc0 = add_half2_f32(acc0, h01);
          acc1 = add_half2_f32(acc1, h23);
        }
      }
      // keys 64 * hf .. 64 * hf + 63 -> P columns 16 * hf .. 16 * hf + 15
      tmem_st32x16(s_tm + hf * 16, pk8);
    } else {
      uint32_t pk[32];
#pragma unroll
      for (int q = 0; q < 2; ++q) {
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          float x0, x1, y0, y1, p0, p1;
          fadd2(x0, x1, __uint_as_float(sr[2 * hf + q][e]), __uint_as_float(sr[2 * hf + q][e + 1]),
                -kRoundMagic, -kRoundMagic);
          ffma2(y0, y1, x0, x1, c, g);
          p0 = ex2_approx(y0);
          p1 = ex2_approx(y1);
          if (MASK) {
            // -inf * 0 would be NaN for a zero-scale block: select instead
            if (x0 == -INFINITY) p0 = 0.0f;
            if (x1 == -INFINITY) p1 = 0.0f;
          }
          const uint32_t h2 = pack_half2(p0, p1);
          pk[q * 16 + (e >> 1)] = h2;
          // the row sum takes the fp16-rounded P that the P V product uses, so that O / l is a
          // weighted mean of V with exactly those weights
          if (e & 2) acc1 = add_half2_f32(acc1, h2);
          else acc0 = add_half2_f32(acc0, h2);
        }
      }
      // keys 64 * hf .. 64 * hf + 63 -> P columns 32 * hf .. 32 * hf + 31; all scores are in
      // registers by now, so these columns are free
      tmem_st32(s_tm + hf * 32, pk);
    }
    if (hf == 0) {
      // half of the row's exponentials done: the other Q tile's softmax may start its step
      __syncwarp();
      if ((threadIdx.x & 31) == 0) mbar_arrive(mx_bar);
    }
  }
  l += acc0 + acc1;
}

// Fused Q quantization for one 128-row Q tile by its softmax warpgroup (128 threads, tid 0-127,
// Q tile wt, first row r0): the tile's fp16 values (coalesced 16-byte loads of 8 values; zeros
// past N), the tile's amax (|x| and max on packed fp16 pairs, exact) through a warp shuffle and
// a warpgroup barrier, scale = amax / 127 and codes rint(x * (1 / scale)) -- with the correctly
// rounded quotient x / scale instead where a value lies within 2^-13 of a half-integer, which is
// the pre-pass's rule (quantize_block_cta), so codes and scales are bit-identical to it (an
// 8-value chunk holding such a value is recomputed on its own) -- written into the K-major
// swizzled layout the TMA would produce (128-byte rows with 128-byte swizzle at d = 128, 64-byte
// rows with 64-byte swizzle at d = 64).  |x| <= amax keeps every code within [-127, 127].
// Returns the scale (0 for an all-zero tile).
template <int D>
__device__ __forceinline__ float quantize_q_tile(const uint16_t* __restrict__ q_head, int r0,
                                                 int N, int tid, int wt, uint8_t* tile,
                                                 float* red) {
  constexpr int CPR = D / 8;              // 16-byte input chunks (8 values) per row
  constexpr int NCH = kBM * CPR / 128;    // chunks per thread
  const uint4* src = reinterpret_cast<const uint4*>(q_head + static_cast<size_t>(r0) * D);
  // all NCH loads are issued before any is used: no branch around them (rows past N read row
  // r0, which exists, and are zeroed afterwards)
  uint4 v[NCH];
#pragma unroll
  for (int i = 0; i < NCH; ++i) {
    const int c = i * 128 + tid;          // chunk index within the tile
    v[i] = __ldg(src + (r0 + c / CPR < N ? c : 0));
  }
#pragma unroll
  for (int i = 0; i < NCH; ++i) {
    if (r0 + (i * 128 + tid) / CPR >= N) v[i] = make_uint4(0, 0, 0, 0);
  }
  __half2 m2 = __floats2half2_rn(0.0f, 0.0f);
#pragma unroll
  for (int i = 0; i < NCH; ++i) {
    m2 = __hmax2(m2, __habs2(*reinterpret_cast<const __half2*>(&v[i].x)));
    m2 = __hmax2(m2, __habs2(*reinterpret_cast<const __half2*>(&v[i].y)));
    m2 = __hmax2(m2, __habs2(*reinterpret_cast<const __half2*>(&v[i].z)));
    m2 = __hmax2(m2, __habs2(*reinterpret_cast<const __half2*>(&v[i].w)));
  }
  float amax = fmaxf(__low2float(m2), __high2float(m2));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
  if ((tid & 31) == 0) red[wt * 4 + (tid >> 5)] = amax;
  named_bar_sync(1 + wt, 128);
  amax = fmaxf(fmaxf(red[wt * 4], red[wt * 4 + 1]), fmaxf(red[wt * 4 + 2], red[wt * 4 + 3]));
  const float s = __fdiv_rn(amax, 127.0f);
  const float rcp = amax > 0.0f ? __frcp_rn(s) : 0.0f;
  // 8 codes of input chunk col land in 16-byte output chunk col / 2 of the row, half col % 2;
  // that 16-byte chunk sits at position (col / 2) ^ (the row's 128-byte line index bits)
  auto dst = [&](int c) -> uint32_t {
    const int row = c / CPR, col = c % CPR;
    const uint32_t swz = D == 128 ? static_cast<uint32_t>(row & 7) : static_cast<uint32_t>((row >> 1) & 3);
    return smem_u32(tile + row * D + (((static_cast<uint32_t>(col) >> 1) ^ swz) << 4) + ((col & 1) << 3));
  };
#pragma unroll
  for (int i = 0; i < NCH; ++i) {
    const uint32_t hw[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
    uint32_t w[2];
    bool near_tie = false;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      int r[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t word = hw[2 * k + (e >> 1)];
        const float y = half_bits_to_float((e & 1) ? (word >> 16) : (word & 0xFFFFu)) * rcp;
        const float ry = rintf(y);
        near_tie |= fabsf(y - ry) > 0.4998779296875f;  // within 2^-13 of a half-integer
        r[e] = static_cast<int>(ry);
      }
      w[k] = __byte_perm(__byte_perm(r[0], r[1], 0x0040), __byte_perm(r[2], r[3], 0x0040), 0x5410);
    }
    if (__any_sync(0xFFFFFFFFu, near_tie) && near_tie) {
      // rare: this chunk again with the exact quotient where it decides the rounding
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        float x[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t word = hw[2 * k + (e >> 1)];
          x[e] = quant_code(half_bits_to_float((e & 1) ? (word >> 16) : (word & 0xFFFFu)), s, rcp);
        }
        w[k] = pack4_i8(x[0], x[1], x[2], x[3]);
      }
    }
    asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(dst(i * 128 + tid)), "r"(w[0]), "r"(w[1])
                 : "memory");
  }
  return amax > 0.0f ? s : 0.0f;
}

__device__ __forceinline__ void setmaxnreg_inc224() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 224;" ::: "memory");
}
__device__ __forceinline__ void setmaxnreg_dec56() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 56;" ::: "memory");
}

// Instantiations of the attention kernel.  kOutF16 is the product (fp16 output); kDumpS is the
// same kernel, which also writes the int32 score tiles it reads (the exactness check of Q K^T);
// kOutF32 writes O / l as fp32 instead of rounding it to fp16 (the fp16 output is exactly its
// round-to-nearest).
constexpr int kOutF16 = 0;
constexpr int kDumpS = 1;
constexpr int kOutF32 = 2;

// Score-tile dump of the kDumpS instantiation: the CTAs of query head bh, pairs pair0 .. (one per
// block), store the raw int32 scores each softmax thread loads from tensor memory for query tiles
// qt0 .. qt0+nqt-1 and key tiles kt0 .. kt0+nkt-1 into s_out [nqt*128][ld] (row-major).
struct ScoreDump {
  int32_t* s_out;
  int ld, bh, pair0, qt0, nqt, kt0, nkt;
};

// QF16: Q arrives as fp16 (q16) and the softmax warps quantize their own Q tile into shared
// memory before the first QK^T (per-tile amax, scale = amax / 127, the same rounding as
// the pre-pass); otherwise int8 Q and its scales come from the smoothing + quantization pass
// (tm_q, q_scale).  MODE: kOutF16, kDumpS (only its block-to-work mapping differs, see
// ScoreDump) or kOutF32 (out points to fp32).  PVK: kPvF16 (P and V in fp16), kPvF8 (P and V in
// E4M3: tm_v8 maps V^T in E4M3, v_scale its per-(batch, kv head) scale) or kPvTable (pv_variant[bg]
// chooses per group, 1 = E4M3).
template <int D, bool CAUSAL, bool QF16, int MODE = kOutF16, int PVK = kPvF16>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_v8,
                    const float* __restrict__ q_scale,
                    const uint16_t* __restrict__ q16, const int* __restrict__ kv_list,
                    const int* __restrict__ kv_count,
                    const float* __restrict__ k_scale, const float* __restrict__ v_scale,
                    const uint8_t* __restrict__ pv_variant, void* __restrict__ out_any, int B, int H,
                    int Hkv, int N, float scale_log2, ScoreDump dump) {
  constexpr bool DUMP = MODE == kDumpS;
  __half* out = static_cast<__half*>(out_any);
  using Cfg = AttnCfg<D>;
  constexpr int ST = Cfg::kStages;
  constexpr int kTmaWarp = kSoftmaxThreads / 32;  // warp 8
  constexpr int kMmaWarp = kTmaWarp + 1;          // warp 9: MMA issue
  constexpr int kAllocWarp = kTmaWarp + 2;        // warp 10: tensor-memory allocation
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  AttnBars* bars = reinterpret_cast<AttnBars*>(smem + Cfg::kOffBar);
  volatile int* abort = &bars->abort;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const int nqt = (N + kBM - 1) / kBM;
  const int npairs = (nqt + 1) / 2;
  const int nkt = (N + kBN - 1) / kBN;
  const int nkb = (N + 63) / 64;
  const int BH = B * H;
  // Launch order.  Causal: pairs heaviest first, all heads of a pair together (the K/V prefix
  // they read is shared by the heads of a kv head and stays in L2).  Non-causal: every CTA reads
  // its head's whole K/V, so the pairs of one head run together and reuse it from L2 (all heads at
  // once would need every head's K/V resident).
  const int pair = DUMP ? dump.pair0 + static_cast<int>(blockIdx.x)
                 : CAUSAL ? npairs - 1 - static_cast<int>(blockIdx.x / BH)
                          : static_cast<int>(blockIdx.x % npairs);
  const int bh = DUMP ? dump.bh
                 : CAUSAL ? static_cast<int>(blockIdx.x % BH) : static_cast<int>(blockIdx.x / npairs);
  const int b = bh / H;
  const int h = bh % H;
  const int g = h / (H / Hkv);
  const int bg = b * Hkv + g;
  // the P V variant of this CTA's (batch, kv head) group
  const bool pv8 = PVK == kPvF8 || (PVK == kPvTable && __ldg(pv_variant + bg) != 0);
  const int tq0 = 2 * pair, tq1 = 2 * pair + 1;
  const bool has1 = tq1 < nqt;
  // Block-sparse: the CTA streams only the key tiles listed for its 256 query rows (ascending;
  // kv_list null = all of them).  Causal lists end with the diagonal tiles tq0, tq1 (when they
  // exist); tile 0 stops before tq1.
  const int* klist = kv_list ? kv_list + (static_cast<size_t>(bh) * npairs + pair) * nkt : nullptr;
  int nw0, nw1;
  if (klist) {
    const int cnt = kv_count[static_cast<size_t>(bh) * npairs + pair];
    nw1 = has1 ? cnt : 0;
    nw0 = (CAUSAL && cnt > 0 && __ldg(klist + cnt - 1) > tq0) ? cnt - 1 : cnt;
  } else {
    nw0 = CAUSAL ? tq0 + 1 : nkt;
    nw1 = has1 ? (CAUSAL ? tq1 + 1 : nkt) : 0;
  }
  const int n_kv = max(nw0, nw1);
  auto ktile = [&](int j) -> int { return klist ? __ldg(klist + j) : j; };

  if (threadIdx.x == 0) {
    // QF16: one arrive per softmax warp once its rows of the Q tiles are in shared memory
    mbar_init(&bars->q_full, QF16 ? kSoftmaxThreads / 32 : 1);
    for (int s = 0; s < ST; ++s) {
      mbar_init(&bars->kv_full[s], 1);
      mbar_init(&bars->kv_empty[s], 1);
    }
    for (int w = 0; w < 2; ++w) {
      mbar_init(&bars->s_full[w], 1);
      mbar_init(&bars->p_full[w], 4);  // one arrive per softmax warp of the Q tile
      mbar_init(&bars->pv_done[w], 1);
      for (int qd = 0; qd < 4; ++qd) mbar_init(&bars->mx_done[w][qd], 1);
    }
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == kAllocWarp) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp >= kTmaWarp) {
    // warpgroup 2 (TMA, MMA and allocator warps, one idle) hands registers to the softmax groups
    setmaxnreg_dec56();
    if (warp == kTmaWarp && lane == 0) {
      // ---------------------------------------------------------------- TMA producer
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      if (!QF16) {
        tma_prefetch_desc(&tm_q);
        mbar_arrive_expect_tx(&bars->q_full, Cfg::kQTile * (has1 ? 2 : 1));
        tma_load_3d(smem + Cfg::kOffQ, &tm_q, &bars->q_full, 0, tq0 * kBM, bh);
        if (has1) tma_load_3d(smem + Cfg::kOffQ + Cfg::kQTile, &tm_q, &bars->q_full, 0, tq1 * kBM, bh);
      }
      for (int j = 0; j < n_kv; ++j) {
        const int s = j % ST;
        const uint32_t u = static_cast<uint32_t>(j / ST);
        if (!mbar_wait(&bars->kv_empty[s], (u & 1u) ^ 1u, abort)) break;
        mbar_arrive_expect_tx(&bars->kv_full[s], Cfg::kKTile + (pv8 ? Cfg::kV8Tile : Cfg::kVTile));
        const int kt = ktile(j);
        tma_load_3d(smem + Cfg::kOffK + s * Cfg::kKTile, &tm_k, &bars->kv_full[s], 0, kt * kBN, bg);
        uint8_t* vdst = smem + Cfg::kOffV + s * Cfg::kVTile;
        if (pv8) {
          tma_load_3d(vdst, &tm_v8, &bars->kv_full[s], kt * kBN, 0, bg);
        } else {
#pragma unroll
          for (int x = 0; x < D / 64; ++x)
            tma_load_3d(vdst + x * Cfg::kVBox, &tm_v, &bars->kv_full[s], x * 64, kt * kBN, bg);
        }
      }
    } else if (warp == kMmaWarp) {
      // ---------------------------------------------------------------- MMA issuer
      // The whole warp runs this loop, so the descriptors and addresses are warp-uniform values;
      // one elected lane issues each tcgen05 instruction.
      // Order per key tile j: PV_0(j), QK_0(j+1), PV_1(j), QK_1(j+1).  tcgen05.mma operations
      // from one thread execute in issue order, so QK_w(j+1) may be issued right behind PV_w(j)
      // although it overwrites the tensor-memory columns PV_w(j) reads P_w from; the softmax of
      // one Q tile then overlaps the other tile's PV + QK^T on the tensor pipe.  Descriptors are
      // computed once and advanced by constants (start-address field, 16-byte units), keeping
      // the instructions per MMA few.
      constexpr uint32_t idq = idesc_i8_s32(kBM, kBN);
      constexpr uint32_t idv = idesc_f16_f32_bmn(kBM, D);
      const uint64_t dq0 = smem_desc(smem_u32(smem + Cfg::kOffQ), 16, Cfg::kSboQK, Cfg::kSwQK);
      const uint64_t dk0 = smem_desc(smem_u32(smem + Cfg::kOffK), 16, Cfg::kSboQK, Cfg::kSwQK);
      const uint64_t dv0 = smem_desc(smem_u32(smem + Cfg::kOffV), Cfg::kVBox, 1024, kSwizzle128B);
      // FP8 variant: V^T rows of 128 keys (128 bytes), 8-row swizzle atoms, K = 32 keys per MMA
      constexpr uint32_t idv8 = idesc_f8_f32(kBM, D);
      const uint64_t dv80 = smem_desc(smem_u32(smem + Cfg::kOffV), 16, 1024, kSwizzle128B);
      // a CTA whose lists hold no key tile (n_kv == 0: block-sparse lists with zero entries) has
      // nothing to multiply; its softmax warps write zero rows
      bool ok = n_kv > 0 &&
                __all_sync(0xFFFFFFFFu, mbar_wait(&bars->q_full, 0, abort) && mbar_wait(&bars->kv_full[0], 0, abort));
      tc_fence_after();
      if (ok) {
#pragma unroll
        for (int w = 0; w < 2; ++w) {
          if ((w == 0 ? nw0 : nw1) == 0) continue;  // a tile without key tiles waits on no score
          const uint64_t da = dq0 + static_cast<uint64_t>((w * Cfg::kQTile) >> 4);
          mma_i8_ss_warp(tmem + w * 128, da, dk0, idq, 0u);
#pragma unroll
          for (int kk = 1; kk < D / 32; ++kk) mma_i8_ss_warp(tmem + w * 128, da + 2 * kk, dk0 + 2 * kk, idq, 1u);
          mma_commit_warp(&bars->s_full[w]);
        }
      }
      int s = 0;
      for (int j = 0; ok && j < n_kv; ++j) {
        const int s1 = s + 1 == ST ? 0 : s + 1;
        const uint64_t dk1 = dk0 + static_cast<uint64_t>((s1 * Cfg::kKTile) >> 4);
        const uint64_t dv = dv0 + static_cast<uint64_t>((s * Cfg::kVTile) >> 4);
        bool next_ready = false;
#pragma unroll
        for (int w = 0; w < 2; ++w) {
          const int nw = w == 0 ? nw0 : nw1;
          if (!ok || j >= nw) continue;
          ok = __all_sync(0xFFFFFFFFu, mbar_wait(&bars->p_full[w], static_cast<uint32_t>(j) & 1u, abort));
          if (!ok) continue;
          tc_fence_after();
          const uint32_t ts = tmem + w * 128, to = tmem + 256 + w * D;
          if (pv8) {
            const uint64_t dv8 = dv80 + static_cast<uint64_t>((s * Cfg::kVTile) >> 4);
            mma_f8_ts_warp(to, ts, dv8, idv8, j == 0 ? 0u : 1u);
#pragma unroll
            for (int kk = 1; kk < kBN / 32; ++kk) mma_f8_ts_warp(to, ts + kk * 8, dv8 + 2 * kk, idv8, 1u);
          } else {
            if (j == 0) mma_f16_ts_warp(to, ts, dv, idv, 0u);
            else mma_f16_ts_warp(to, ts, dv, idv, 1u);
#pragma unroll
            for (int kk = 1; kk < kBN / 16; ++kk) mma_f16_ts_warp(to, ts + kk * 8, dv + kk * 128, idv, 1u);
          }
          mma_commit_warp(&bars->pv_done[w]);
          if (j + 1 < nw) {
            if (!next_ready) {
              ok = __all_sync(0xFFFFFFFFu, mbar_wait(&bars->kv_full[s1], static_cast<uint32_t>((j + 1) / ST) & 1u, abort));
              if (!ok) continue;
              tc_fence_after();
              next_ready = true;
            }
            const uint64_t da = dq0 + static_cast<uint64_t>((w * Cfg::kQTile) >> 4);
            mma_i8_ss_warp(ts, da, dk1, idq, 0u);
#pragma unroll
            for (int kk = 1; kk < D / 32; ++kk) mma_i8_ss_warp(ts, da + 2 * kk, dk1 + 2 * kk, idq, 1u);
            mma_commit_warp(&bars->s_full[w]);
          }
        }
        if (!ok) break;
        mma_commit_warp(&bars->kv_empty[s]);
        s = s1;
      }
    }
  } else {
    // ------------------------------------------------------------------ softmax warpgroups
    // Warps 0-3: Q tile 0, warps 4-7: Q tile 1; thread = score row (TMEM lane 32 * (warp % 4)
    // + lane), read with the 32x32b shape.
    setmaxnreg_inc224();
    const int wt = warp >> 2;
    const int row = (warp & 3) * 32 + lane;
    const int nt = wt == 0 ? nw0 : nw1;
    float sq_fused = 0.0f;
    if (QF16) {
      // quantize this warpgroup's Q tile (thread = row) into the MMA's swizzled int8 layout
      float* red = reinterpret_cast<float*>(smem + Cfg::kOffRed);
      if (nt > 0)
        sq_fused = quantize_q_tile<D>(q16 + (static_cast<size_t>(bh) * N) * D,
                                      (wt == 0 ? tq0 : tq1) * kBM, N, row, wt,
                                      smem + Cfg::kOffQ + wt * Cfg::kQTile, red);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->q_full);
    }
    if (nt > 0) {
      const int t = wt == 0 ? tq0 : tq1;
      const int qrow = t * kBM + row;
      const float sq = QF16 ? sq_fused : __ldg(q_scale + static_cast<size_t>(bh) * nqt + t);
      const float* ksc = k_scale + static_cast<size_t>(bg) * nkb;
      const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
      const uint32_t s_tm = tmem + lane_off + wt * 128;
      const uint32_t o_tm = tmem + lane_off + 256 + wt * D;
      float m = -INFINITY, l = 0.0f;
      bool ok = true;
      // key tiles of steps j and j + 1 in registers; the list entry of step j + 2 is loaded one
      // step ahead, so the K scales of step j + 1 never wait on a dependent list load
      int kt = ktile(0);
      int kt1 = nt > 1 ? ktile(1) : 0;
      float ks0 = __ldg(ksc + 2 * kt);
      float ks1 = 2 * kt + 1 < nkb ? __ldg(ksc + 2 * kt + 1) : 0.0f;
      for (int j = 0; j < nt; ++j) {
        const int nkt_next = kt1;
        kt1 = j + 2 < nt ? ktile(j + 2) : 0;
        const float nks0 = (2 * nkt_next < nkb) ? __ldg(ksc + 2 * nkt_next) : 0.0f;
        const float nks1 = (2 * nkt_next + 1 < nkb) ? __ldg(ksc + 2 * nkt_next + 1) : 0.0f;
        // The two Q tiles' softmax steps are kept half a step apart, so that their MUFU-bound
        // exponential passes do not run at the same time: tile 1's warp of a TMEM lane quadrant
        // (and SM sub-partition) starts step j once tile 0's warp of that quadrant is half through
        // its exponentials of step j, tile 0's warp starts step j once tile 1's is half through
        // step j - 1 (mx_done[w][quadrant], one arrive per step).  Without this the two tiles
        // settle nearly in phase and each step's softmax runs ~40 % longer.  Tile 0 has no step
        // nw0 (causal, one key tile fewer than tile 1), so tile 1's last step is not gated;
        // neither barrier gets two phases ahead of its waiter, since each warp's next arrive needs
        // its partner's.
        if (wt == 1 && j < nw0)
          ok = __all_sync(0xFFFFFFFFu, mbar_wait(&bars->mx_done[0][warp & 3], static_cast<uint32_t>(j) & 1u, abort));
        else if (wt == 0 && j > 0 && j - 1 < nw1)
          ok = __all_sync(0xFFFFFFFFu, mbar_wait(&bars->mx_done[1][warp & 3], static_cast<uint32_t>(j - 1) & 1u, abort));
        if (!ok) break;
        ok = __all_sync(0xFFFFFFFFu, mbar_wait(&bars->s_full[wt], static_cast<uint32_t>(j) & 1u, abort));
        if (!ok) break;
        tc_fence_after();
        uint32_t sr[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(s_tm + c * 32, sr[c]);
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld_wait(sr[c]);
        if constexpr (DUMP) {
          if (t >= dump.qt0 && t < dump.qt0 + dump.nqt && kt >= dump.kt0 && kt < dump.kt0 + dump.nkt) {
            int4* dst = reinterpret_cast<int4*>(dump.s_out + static_cast<size_t>((t - dump.qt0) * kBM + row) * dump.ld +
                                                (kt - dump.kt0) * kBN);
#pragma unroll
            for (int c = 0; c < 4; ++c)
#pragma unroll
              for (int e = 0; e < 32; e += 4)
                dst[c * 8 + e / 4] = make_int4(static_cast<int>(sr[c][e]), static_cast<int>(sr[c][e + 1]),
                                               static_cast<int>(sr[c][e + 2]), static_cast<int>(sr[c][e + 3]));
          }
        }
        int lim = N - 1 - kt * kBN;
        if (CAUSAL && kt == t) lim = min(lim, row);
        const float c0 = sq * ks0 * scale_log2;
        const float c1 = sq * ks1 * scale_log2;
        ks0 = nks0;
        ks1 = nks1;
        kt = nkt_next;
        // warp-uniform, so that every lane runs the same tensor-memory access sequence
        const bool masked = __any_sync(0xFFFFFFFFu, lim < kBN - 1);
        float alpha;
        bool need;
        uint64_t* gate = &bars->mx_done[wt][warp & 3];
        if (pv8) {
          if (masked) softmax_row<D, true, true>(sr, lim, c0, c1, j == 0, m, l, alpha, need, s_tm, gate);
          else softmax_row<D, false, true>(sr, lim, c0, c1, j == 0, m, l, alpha, need, s_tm, gate);
        } else {
          if (masked) softmax_row<D, true, false>(sr, lim, c0, c1, j == 0, m, l, alpha, need, s_tm, gate);
          else softmax_row<D, false, false>(sr, lim, c0, c1, j == 0, m, l, alpha, need, s_tm, gate);
        }
        if (j > 0 && __any_sync(0xFFFFFFFFu, need)) {
          // O holds PV up to tile j-1 (complete: QK(j) was issued after PV(j-1)), and PV(j)
          // waits for this warp's arrive below.
#pragma unroll
          for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t o[32];
            tmem_ld32(o_tm + cc * 32, o);
            tmem_ld_wait(o);
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tmem_st32(o_tm + cc * 32, o);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->p_full[wt]);
      }
      if (ok) ok = mbar_wait(&bars->pv_done[wt], static_cast<uint32_t>(nt - 1) & 1u, abort);
      ok = __all_sync(0xFFFFFFFFu, ok);
      tc_fence_after();
      if (ok) {
        // the FP8 variant's O is in units of V's E4M3 codes: times its scale
        const float inv_l = (pv8 ? __ldg(v_scale + bg) : 1.0f) / l;
        __half* orow = out + (static_cast<size_t>(bh) * N + qrow) * D;
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t o[32];
          tmem_ld32(o_tm + cc * 32, o);
          tmem_ld_wait(o);
          if (MODE == kOutF32 && qrow < N) {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(out_any) +
                                                    (static_cast<size_t>(bh) * N + qrow) * D + cc * 32);
#pragma unroll
            for (int v = 0; v < 8; ++v)
              dst[v] = make_float4(__uint_as_float(o[4 * v + 0]) * inv_l, __uint_as_float(o[4 * v + 1]) * inv_l,
                                   __uint_as_float(o[4 * v + 2]) * inv_l, __uint_as_float(o[4 * v + 3]) * inv_l);
          } else if (qrow < N) {
            uint4* dst = reinterpret_cast<uint4*>(orow + cc * 32);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              uint4 pkt;
              pkt.x = pack_half2(__uint_as_float(o[8 * v + 0]) * inv_l, __uint_as_float(o[8 * v + 1]) * inv_l);
              pkt.y = pack_half2(__uint_as_float(o[8 * v + 2]) * inv_l, __uint_as_float(o[8 * v + 3]) * inv_l);
              pkt.z = pack_half2(__uint_as_float(o[8 * v + 4]) * inv_l, __uint_as_float(o[8 * v + 5]) * inv_l);
              pkt.w = pack_half2(__uint_as_float(o[8 * v + 6]) * inv_l, __uint_as_float(o[8 * v + 7]) * inv_l);
              dst[v] = pkt;
            }
          }
        }
      }
    } else {
      // no key tile for this Q tile (an empty block-sparse list): the softmax over no keys is
      // empty, and its rows are written as zeros
      const int qrow = (wt == 0 ? tq0 : tq1) * kBM + row;
      if ((wt == 0 || has1) && qrow < N) {
        constexpr int kBytes = MODE == kOutF32 ? 4 : 2;
        uint4* dst = reinterpret_cast<uint4*>(static_cast<uint8_t*>(out_any) +
                                              (static_cast<size_t>(bh) * N + qrow) * D * kBytes);
#pragma unroll
        for (int v = 0; v < D * kBytes / 16; ++v) dst[v] = make_uint4(0, 0, 0, 0);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kAllocWarp) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace qattn
