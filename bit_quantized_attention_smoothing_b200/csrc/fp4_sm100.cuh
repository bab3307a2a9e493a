// fp4_sm100.cuh -- the FP4 path of the ThriftAttention page ("ThriftAttention: Selective Mixed
// Precision for Long-Context FP4 Attention", gist.science/ja/paper/2605.23081, method section,
// "FP4 path": blocks computed in FP4 with the NVFP4 micro-scaling format on Blackwell's native FP4
// tensor cores) on the block-scaled tensor cores: FP4 score tiles (qk_nvfp4_kernel) and the
// attention with FP16 promotion of selected key tiles (attn_nvfp4_kernel, further down).
//
// Operands are NVFP4 as qattn_quant_nvfp4 writes them along the channels: E2M1 codes packed two
// per byte (rows of d/2 bytes) and one E4M3 scale byte per 16 channels (rows of d/16 bytes).
// tcgen05.mma kind::mxf4nvf4 with block16 scaling multiplies 128 x 64 by 64 x N E2M1 tiles, each
// 16-element product sum weighted by the two E4M3 block scales, into an fp32 accumulator in
// tensor memory; the slice scales gQ gK are applied when the accumulator is read back.
//
// Scale factors live in tensor memory.  For M = 128 (and for N = 128 of the B operand) the
// instruction reads them in this arrangement: row r = r0 + 32 r1 (r0 < 32, r1 < 4) of the operand
// has its four scale bytes of one 64-element K step (blocks 4 kc .. 4 kc + 3, the lowest block in
// the lowest byte) in the 32-bit column (base + r1) of lane r0, and the same 32 lanes are repeated
// in each of the four 32-lane sub-partitions.  Q's, K's and V's scales are written by each warp
// into its own sub-partition with tcgen05.st; P's, whose rows belong to all sub-partitions, are
// staged in shared memory in that order ([K step][r0][r1] words) and copied into all four
// sub-partitions at once by the issuing warp (tcgen05.cp .32x128b.warpx4).
#pragma once

#include <cstdint>

#include "attn_sm100.cuh"  // pack_half2, add_half2_f32
#include "nvfp4.cuh"       // E2M1 / E4M3 conversions
#include "quant.cuh"       // half_bits_to_float
#include "sm100_ptx.cuh"

namespace qattn {

constexpr uint32_t kSwizzle32B = 6;

// Instruction descriptor of kind::mxf4nvf4 (block-scaled): B scale-factor id [4,6) = 0, A format
// [7,10) = 1 (E2M1), B format [10,13) = 1 (E2M1), A and B K-major (bits 15, 16 = 0), N >> 3 in
// [17,23), scale format bit 23 = 0 (UE4M3), M >> 4 in [24,29), A scale-factor id [29,31) = 0,
// bit 31 = 0 (K = 64 per instruction).  The accumulator is always f32.
__host__ __device__ constexpr uint32_t idesc_nvf4(int M, int N) {
  return (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// D[tmem] (+)= (A[smem] x SFA) * (B[smem] x SFB)^T, E2M1 inputs with UE4M3 scales per 16.
__device__ __forceinline__ void mma_nvf4_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                            uint32_t idesc, uint32_t sfa_tmem, uint32_t sfb_tmem,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;"
      "\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// Warp-collective store of 4 consecutive 32-bit columns of the warp's 32 lanes.
__device__ __forceinline__ void tmem_st32x4(uint32_t taddr, uint32_t a, uint32_t b, uint32_t c,
                                            uint32_t d) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};" ::"r"(taddr),
               "r"(a), "r"(b), "r"(c), "r"(d)
               : "memory");
}

// The four scale words of rows r0 + lane + 32 r1 (r1 = 0..3) for K step kc, 0 past the end.
__device__ __forceinline__ void load_sf_words(const uint8_t* __restrict__ scales, int D, int N,
                                              int row0, int kc, uint32_t (&w)[4]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int r1 = 0; r1 < 4; ++r1) {
    const int row = row0 + lane + 32 * r1;
    w[r1] = row < N ? __ldg(reinterpret_cast<const uint32_t*>(
                          scales + static_cast<size_t>(row) * (D / 16) + 4 * kc))
                    : 0u;
  }
}

template <int D>
struct Fp4Cfg {
  static constexpr int kRowBytes = D / 2;                // E2M1 codes of one row
  static constexpr int kTile = 128 * kRowBytes;          // one 128-row operand tile
  static constexpr uint32_t kSw = D == 128 ? kSwizzle64B : kSwizzle32B;
  static constexpr uint32_t kSbo = 8 * kRowBytes;        // 8-row swizzle atoms
  static constexpr int kSteps = D / 64;                  // K = 64 per instruction
  static constexpr uint32_t kColSfa = 128;               // TMEM columns: accumulator 0..127,
  static constexpr uint32_t kColSfb = 144;               // scales of A, then of B
  static constexpr int kSmem = 2 * kTile + 64 + 1024;
};

// FP4 score tiles S = (gQ gK) * sum_c Q[r][c] K[n][c] for query tiles qt0 + blockIdx.x and key
// tiles kt0 + blockIdx.y (128 rows each) of query slice bh and kv slice bg.  s_out: fp32 rows of
// ldo elements.  128 threads.
template <int D>
__global__ void __launch_bounds__(128, 1)
    qk_nvfp4_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const uint8_t* __restrict__ q_scales, const uint8_t* __restrict__ k_scales,
                    const float* __restrict__ q_g, const float* __restrict__ k_g,
                    float* __restrict__ s_out, int N, int bh, int bg, int qt0, int kt0, int ldo) {
  using Cfg = Fp4Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sq = smem;
  uint8_t* sk = smem + Cfg::kTile;
  uint64_t* bar_ld = reinterpret_cast<uint64_t*>(smem + 2 * Cfg::kTile);
  uint64_t* bar_mma = bar_ld + 1;
  uint32_t* tbase = reinterpret_cast<uint32_t*>(bar_ld + 2);
  volatile int* abort = reinterpret_cast<volatile int*>(bar_ld + 3);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int qt = qt0 + blockIdx.x;
  const int kt = kt0 + blockIdx.y;
  if (threadIdx.x == 0) {
    mbar_init(bar_ld, 1);
    mbar_init(bar_mma, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tbase, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tbase;
  // scale factors: every warp writes the same 32 lanes into its own sub-partition
  {
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const uint8_t* qs = q_scales + static_cast<size_t>(bh) * N * (D / 16);
    const uint8_t* ks = k_scales + static_cast<size_t>(bg) * N * (D / 16);
#pragma unroll
    for (int kc = 0; kc < Cfg::kSteps; ++kc) {
      uint32_t w[4];
      load_sf_words(qs, D, N, qt * 128, kc, w);
      tmem_st32x4(lane_base + Cfg::kColSfa + 4 * kc, w[0], w[1], w[2], w[3]);
      load_sf_words(ks, D, N, kt * 128, kc, w);
      tmem_st32x4(lane_base + Cfg::kColSfb + 4 * kc, w[0], w[1], w[2], w[3]);
    }
    tmem_st_wait();
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) {
    tc_fence_after();
    mbar_arrive_expect_tx(bar_ld, 2 * Cfg::kTile);
    tma_load_3d(sq, &tm_q, bar_ld, 0, qt * 128, bh);
    tma_load_3d(sk, &tm_k, bar_ld, 0, kt * 128, bg);
    if (mbar_wait(bar_ld, 0, abort)) {
      tc_fence_after();
      constexpr uint32_t id = idesc_nvf4(128, 128);
#pragma unroll
      for (int kc = 0; kc < Cfg::kSteps; ++kc) {
        const uint64_t ad = smem_desc(smem_u32(sq) + kc * 32, 16, Cfg::kSbo, Cfg::kSw);
        const uint64_t bd = smem_desc(smem_u32(sk) + kc * 32, 16, Cfg::kSbo, Cfg::kSw);
        mma_nvf4_ss(tmem, ad, bd, id, tmem + Cfg::kColSfa + 4 * kc, tmem + Cfg::kColSfb + 4 * kc,
                    kc > 0 ? 1u : 0u);
      }
      mma_commit(bar_mma);
    }
  }
  __syncwarp();
  const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait(bar_mma, 0, abort));
  tc_fence_after();
  if (ok) {
    const float gg = __ldg(q_g + bh) * __ldg(k_g + bg);
    const int r = warp * 32 + lane;
    float* orow = s_out + static_cast<size_t>(blockIdx.x * 128 + r) * ldo + blockIdx.y * 128;
#pragma unroll 1
    for (int cc = 0; cc < 4; ++cc) {
      uint32_t v[32];
      tmem_ld32(tmem + (static_cast<uint32_t>(warp * 32) << 16) + 32 * cc, v);
      tmem_ld_wait(v);
#pragma unroll
      for (int j = 0; j < 32; j += 4)
        *reinterpret_cast<float4*>(orow + 32 * cc + j) =
            make_float4(__uint_as_float(v[j]) * gg, __uint_as_float(v[j + 1]) * gg,
                        __uint_as_float(v[j + 2]) * gg, __uint_as_float(v[j + 3]) * gg);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

}  // namespace qattn

namespace qattn {

// ------------------------------------------------------------------------------------------------
// Attention on the FP4 path with FP16 promotion (ThriftAttention page, method section: the top-k
// query-key block pairs computed in FP16, the rest in FP4, both merged by one online softmax; the
// FP4 probability blocks quantized in two levels).  FP4 tiles: Q and smoothed K NVFP4 along the
// channels, V NVFP4 along the tokens (transposed, rows of Np = ceil(N / 128) * 128 tokens), P
// quantized per row in two levels (binary32 row scale gP = max p / 2688, then NVFP4 blocks of 16
// keys with UE4M3 scales).  Promoted tiles (the key tiles listed for the CTA's 256-row query
// block): fp16 Q K^T on the f16 tensor cores with q . mean subtracted (the FP16 scores see the
// same smoothed keys as the FP4 ones), P rounded to fp16 into tensor memory, fp16 V.
//
// One CTA of 16 softmax warps and one issuing warp per 128-row query tile.  Query row r of the
// tile is tensor-memory lane r; the four softmax warps of a lane quadrant (warps q, q + 4, q + 8,
// q + 12) share its rows: part pt takes keys 32 pt .. 32 pt + 31 of every key tile and output
// channels pt D/4 .. pt D/4 + D/4 - 1, so a thread holds a quarter row; the four parts exchange the
// row maximum (and at the end the row sum) through shared memory.  S is double-buffered in tensor
// memory, so Q K^T(j + 1) runs while the softmax works on S(j).
//   Issuing warp (16): TMA loads of Q, K, V (K and V double-buffered in shared memory, FP4 and
//   fp16 buffers apart) and the MMAs: Q K^T(j + 1) once the softmax warps have read S(j - 1)'s
//   buffer and written tile j + 1's K scales (s_free), P V(j) once P(j) and its scales are written
//   (p_full); K(j + 2) is loaded once Q K^T(j) is known done, V(j + 1) once P V(j - 1) is.
//   Softmax warps, per key tile j: wait S(j), load the quarter row's 32 scores, write tile j + 1's
//   K scales, arrive on s_free; exchange the row maximum; wait P V(j - 1) and fold it into the
//   outputs (O = O corr + acc f); compute P (FP4: two-level codes and scales, codes into the
//   swizzled shared-memory operand; FP16: pairs into tensor memory over the consumed scores),
//   write tile j's V scales and stage P's block scales in shared memory, arrive on p_full; the
//   issuing warp copies P's scales into tensor memory ahead of P V(j).
// Exponentials and reciprocals are MUFU ex2 / rcp, code and scale quotients products with those
// reciprocals; they differ from the correctly rounded operations only within a relative 2^-20 of a
// rounding tie.  Every wait is bounded; the softmax warps agree on each step's outcome at their
// first barrier (a reducing named barrier), so a wait that runs out ends their loops together, and
// the issuing warp leaves its loop on the abort flag; it then drains its tensor-core operations
// and loads (bounded) before tensor memory is freed.
// ------------------------------------------------------------------------------------------------

constexpr int kFp4Parts = 4;                      // threads per query row
constexpr int kFp4Softmax = 128 * kFp4Parts;      // 16 softmax warps
constexpr int kFp4Threads = kFp4Softmax + 32;     // + the issuing warp

template <int D>
struct Fp4AttnCfg {
  static constexpr int kQK = 128 * (D / 2);  // E2M1 Q or K tile: 128 rows of D/2 bytes
  static constexpr int kVt = D * 64;         // E2M1 V^T tile: D channel rows of 128 keys
  static constexpr int kP = 128 * 64;        // E2M1 P tile: 128 rows of 128 keys
  static constexpr int kT16 = 128 * D * 2;   // fp16 tile of 128 rows (D/64 boxes of 64 columns)
  static constexpr int kBox16 = 128 * 128;   // one 64-column fp16 box: 128 rows of 128 bytes
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kQK;                   // two K tiles
  static constexpr int kOffV = kOffK + 2 * kQK;       // two V^T tiles
  static constexpr int kOffP = kOffV + 2 * kVt;
  static constexpr int kOffQ16 = kOffP + kP;
  static constexpr int kOffK16 = kOffQ16 + kT16;      // two fp16 K tiles
  static constexpr int kOffV16 = kOffK16 + 2 * kT16;  // two fp16 V tiles
  static constexpr int kOffSfp = kOffV16 + 2 * kT16;  // uint32 [2][32][4]: P scale words, K step,
                                                      // row % 32, row / 32 (tcgen05.cp source)
  static constexpr int kOffRed = kOffSfp + 1024;      // float [2][4][128]: row parts' maxima by
                                                      // step parity; sums
  static constexpr int kOffMask = kOffRed + 4096;     // uint32 [32]: promoted key tiles, bit t
  static constexpr int kOffBar = kOffMask + 128;
  static constexpr int kSmemUsed = kOffBar + 128 + 1024;  // + alignment slack
  static constexpr uint32_t kSwQK = D == 128 ? kSwizzle64B : kSwizzle32B;
  static constexpr uint32_t kSboQK = 8 * (D / 2);
  static constexpr int kStepsQK = D / 64;         // K = 64 per FP4 instruction
  static constexpr int kSfvCols = D / 32;         // V scale columns per K step (N = D)
  // tensor-memory columns: two S buffers (fp16 P of a promoted tile over the first 64 of its
  // buffer), the P V tile, the four scale-factor areas
  static constexpr uint32_t kColS = 0, kColO = 256, kColSfq = 384, kColSfk = 392, kColSfp = 400,
                            kColSfv = 408;
  static constexpr int kMaxTiles = 1024;          // promoted-tile mask: 32 words
};

__device__ __forceinline__ void tmem_st32x2(uint32_t taddr, uint32_t a, uint32_t b) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x2.b32 [%0], {%1, %2};" ::"r"(taddr), "r"(a),
               "r"(b)
               : "memory");
}
__device__ __forceinline__ void tmem_st32x1(uint32_t taddr, uint32_t a) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};" ::"r"(taddr), "r"(a) : "memory");
}
__device__ __forceinline__ void tmem_ld32x16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

// Waits for outstanding tcgen05.ld and ties the wait to the 16 destination registers.
__device__ __forceinline__ void tmem_ld_wait(uint32_t (&r)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                 "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                 "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15])
               :
               : "memory");
}

// The C = D/4 output channels' accumulator words of one quarter row (32 or 16 columns), loaded
// and waited for.
template <int C>
__device__ __forceinline__ void tmem_ld_part(uint32_t taddr, uint32_t (&r)[C]) {
  if constexpr (C == 32) tmem_ld32(taddr, r);
  else tmem_ld32x16(taddr, r);
  tmem_ld_wait(r);
}

__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Eight non-negative binary32 values to eight E2M1 codes, v[0] in bits 0-3 ... v[7] in bits 28-31
// (the cvt places its first source in the upper nibble; a non-negative input never sets a sign).
__device__ __forceinline__ uint32_t e2m1x8_nonneg(float v0, float v1, float v2, float v3, float v4,
                                                  float v5, float v6, float v7) {
  uint32_t r;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(r)
      : "f"(v0), "f"(v1), "f"(v2), "f"(v3), "f"(v4), "f"(v5), "f"(v6), "f"(v7));
  return r;
}

// Twice the sum of the values of the eight non-negative E2M1 codes in w, exact: a byte permute
// looks up each code's doubled magnitude (0, 1, 2, 3, 4, 6, 8, 12 for codes 0..7) four codes at a
// time, and a four-byte dot product with ones adds them.
__device__ __forceinline__ int e2m1x8_twice_sum(uint32_t w, int acc) {
  const uint32_t lo = __byte_perm(0x03020100u, 0x0C080604u, w & 0xFFFFu);
  const uint32_t hi = __byte_perm(0x03020100u, 0x0C080604u, w >> 16);
  return __dp4a(static_cast<int>(hi), 0x01010101, __dp4a(static_cast<int>(lo), 0x01010101, acc));
}

// Exact binary32 value of an E4M3 byte with sign 0, by the hardware conversion to fp16.
__device__ __forceinline__ float ue4m3_value_cvt(uint32_t s) {
  uint32_t h;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(static_cast<unsigned short>(s)));
  return __half2float(__ushort_as_half(static_cast<unsigned short>(h & 0xFFFFu)));
}

// Instruction descriptor of kind::f16 with fp16 A and B, both K-major, f32 accumulator.
__host__ __device__ constexpr uint32_t idesc_f16_f32_kk(int M, int N) {
  return (1u << 4) | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// Single-thread forms of the f16 MMAs (A from shared memory, or from tensor memory).
__device__ __forceinline__ void mma_f16_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                           uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem), "l"(adesc),
      "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void mma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                           uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Warp-collective forms for the issuing warp: the whole warp runs them with the same operands and
// one lane, picked by elect.sync, issues the instruction.
__device__ __forceinline__ void mma_nvf4_ss_warp(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                                 uint32_t idesc, uint32_t sfa_tmem, uint32_t sfb_tmem,
                                                 uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;"
      "\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// tcgen05.cp of 32 rows x 128 bits from shared memory (descriptor sdesc: no swizzle, rows 16 bytes
// apart, 8-row groups 128 bytes apart) into the four columns at taddr of lanes 0-31 of every
// 32-lane sub-partition; one lane, picked by elect.sync, issues it.  It executes in order with the
// tensor-core operations the same lane issues after it.
__device__ __forceinline__ void tmem_cp32x128_warpx4_warp(uint32_t taddr, uint64_t sdesc) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;\n\t}" ::"r"(taddr),
      "l"(sdesc)
      : "memory");
}

__device__ __forceinline__ void mma_f16_ss_warp(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                                uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem), "l"(adesc),
      "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Barrier `id` among `n` threads that also returns whether `v` holds for all of them.
__device__ __forceinline__ bool named_bar_and(int id, int n, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v)), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}

// (o0, o1) = (o0 * c + a0 * f, o1 * c + a1 * f) with packed sm_100 fp32x2 operations.
__device__ __forceinline__ void fold2(float& o0, float& o1, float a0, float a1, float c, float f) {
  asm("{\n\t.reg .b64 ro, ra, rc, rf, rt;\n\t"
      "mov.b64 ro, {%0, %1};\n\tmov.b64 ra, {%2, %3};\n\t"
      "mov.b64 rc, {%4, %4};\n\tmov.b64 rf, {%5, %5};\n\t"
      "mul.rn.f32x2 rt, ra, rf;\n\t"
      "fma.rn.f32x2 ro, ro, rc, rt;\n\t"
      "mov.b64 {%0, %1}, ro;\n\t}"
      : "+f"(o0), "+f"(o1)
      : "f"(a0), "f"(a1), "f"(c), "f"(f));
}

// (d0, d1) = (a0 * b0, a1 * b1) as one packed sm_100 fp32x2 multiply.
__device__ __forceinline__ void fmul2(float& d0, float& d1, float a0, float a1, float b) {
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %4};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b));
}

// A bounded wait that ignores the CTA's abort flag (the final drain of thread 0's operations).
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  int zero = 0;
  (void)mbar_wait(bar, parity, &zero, kWaitLimitCycles / 8);
}

// One quarter row's P for an FP4 key tile: 32 scores s[] (fp32 bits) of keys kb .. kb + 31, row
// `row`; MASK: keys past N or after the row (causal) get p = 0.  Writes the four code words and the
// two scale bytes (low 16 bits of sw) of its two 16-key blocks and returns the sum of the
// dequantized p.
template <bool MASK, bool CAUSAL>
__device__ __forceinline__ float fp4_quarter_row(const uint32_t (&s)[32], int kb, int row, int N,
                                                 float gqk, float m_new, float gp,
                                                 uint32_t (&cw)[4], uint32_t& sw) {
  const float r6g = gp > 0.0f ? rcp_approx(__fmul_rn(6.0f, gp)) : 0.0f;
  float lsum = 0.0f;
  sw = 0;
#pragma unroll
  for (int blk = 0; blk < 2; ++blk) {
    float p[16];
#pragma unroll
    for (int i = 0; i < 16; i += 2) {
      float y0, y1;
      ffma2(y0, y1, __uint_as_float(s[16 * blk + i]), __uint_as_float(s[16 * blk + i + 1]), gqk, -m_new);
      p[i] = ex2_approx(y0);
      p[i + 1] = ex2_approx(y1);
      if (MASK) {
        const int k = kb + 16 * blk + i;
        if (k >= N || (CAUSAL && k > row)) p[i] = 0.0f;
        if (k + 1 >= N || (CAUSAL && k + 1 > row)) p[i + 1] = 0.0f;
      }
    }
    float bmax = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; i += 2) bmax = fmax3(bmax, p[i], p[i + 1]);
    const uint32_t sc_byte = gp > 0.0f ? ue4m3_byte(bmax * r6g) : 0u;
    cw[2 * blk] = 0u;
    cw[2 * blk + 1] = 0u;
    if (sc_byte != 0u) {
      const float sc = __fmul_rn(ue4m3_value_cvt(sc_byte), gp);
      const float rs = rcp_approx(sc);
#pragma unroll
      for (int i = 0; i < 16; i += 2) fmul2(p[i], p[i + 1], p[i], p[i + 1], rs);
      cw[2 * blk] = e2m1x8_nonneg(p[0], p[1], p[2], p[3], p[4], p[5], p[6], p[7]);
      cw[2 * blk + 1] = e2m1x8_nonneg(p[8], p[9], p[10], p[11], p[12], p[13], p[14], p[15]);
      const int twice = e2m1x8_twice_sum(cw[2 * blk + 1], e2m1x8_twice_sum(cw[2 * blk], 0));
      lsum = fmaf(0.5f * sc, static_cast<float>(twice), lsum);
    }
    sw |= sc_byte << (8 * blk);
  }
  return lsum;
}

// One quarter row's P for a promoted (FP16) key tile: p = 2^((s - cq) sl2 - m_new) rounded to fp16
// pairs in pk (keys 2c, 2c + 1 in word c); returns the sum of the rounded p.
template <bool MASK, bool CAUSAL>
__device__ __forceinline__ float fp16_quarter_row(const uint32_t (&s)[32], int kb, int row, int N,
                                                  float cq, float sl2, float m_new,
                                                  uint32_t (&pk)[16]) {
  float acc0 = 0.0f, acc1 = 0.0f;
#pragma unroll
  for (int c = 0; c < 16; ++c) {
    const int k = 2 * c;
    float y0, y1;
    ffma2(y0, y1, __uint_as_float(s[k]) - cq, __uint_as_float(s[k + 1]) - cq, sl2, -m_new);
    float p0 = ex2_approx(y0);
    float p1 = ex2_approx(y1);
    if (MASK) {
      if (kb + k >= N || (CAUSAL && kb + k > row)) p0 = 0.0f;
      if (kb + k + 1 >= N || (CAUSAL && kb + k + 1 > row)) p1 = 0.0f;
    }
    pk[c] = pack_half2(p0, p1);
    if (c & 1) acc1 = add_half2_f32(acc1, pk[c]);
    else acc0 = add_half2_f32(acc0, pk[c]);
  }
  return acc0 + acc1;
}

template <int D, bool CAUSAL>
__global__ void __launch_bounds__(kFp4Threads, 1)
    attn_nvfp4_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_vt,
                      const __grid_constant__ CUtensorMap tm_q16,
                      const __grid_constant__ CUtensorMap tm_k16,
                      const __grid_constant__ CUtensorMap tm_v16, const uint8_t* __restrict__ q_sf,
                      const uint8_t* __restrict__ k_sf, const uint8_t* __restrict__ vt_sf,
                      const float* __restrict__ q_g, const float* __restrict__ k_g,
                      const float* __restrict__ v_g, const uint16_t* __restrict__ q16,
                      const float* __restrict__ k_mean, const int* __restrict__ kv_list,
                      const int* __restrict__ kv_count, __half* __restrict__ out, int H, int Hkv,
                      int N, int Np, float sl2) {
  using Cfg = Fp4AttnCfg<D>;
  constexpr int DP = D / kFp4Parts;  // output channels per softmax thread
  constexpr int kIssueWarp = kFp4Softmax / 32;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sq = smem + Cfg::kOffQ;
  uint8_t* sk = smem + Cfg::kOffK;
  uint8_t* sv = smem + Cfg::kOffV;
  uint8_t* sp = smem + Cfg::kOffP;
  uint8_t* sq16 = smem + Cfg::kOffQ16;
  uint8_t* sk16 = smem + Cfg::kOffK16;
  uint8_t* sv16 = smem + Cfg::kOffV16;
  uint32_t* sfp = reinterpret_cast<uint32_t*>(smem + Cfg::kOffSfp);
  float* red = reinterpret_cast<float*>(smem + Cfg::kOffRed);
  uint32_t* pmask = reinterpret_cast<uint32_t*>(smem + Cfg::kOffMask);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kOffBar);
  uint64_t* q_full = bars;
  uint64_t* q16_full = bars + 1;
  uint64_t* k_full = bars + 2;  // [2] K tile loaded into buffer b
  uint64_t* v_full = bars + 4;  // [2] V tile loaded into buffer b
  uint64_t* s_full = bars + 6;  // [2] Q K^T into S buffer b done
  uint64_t* o_full = bars + 8;  // P V done
  uint64_t* s_free = bars + 9;  // softmax warps: S read, next K scales written (16 arrivals)
  uint64_t* p_full = bars + 10; // softmax warps: P and its scales written (16 arrivals)
  uint64_t* drain = bars + 11;
  uint32_t* tbase = reinterpret_cast<uint32_t*>(bars + 12);
  volatile int* abort = reinterpret_cast<volatile int*>(bars + 13);
  static_assert(14 * 8 <= 128, "barrier block");

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int quad = warp & 3, pt = warp >> 2;  // softmax warps: lane quadrant, part of the row
  const int rl = quad * 32 + lane;            // row within the tile = tensor-memory lane
  const int qt = CAUSAL ? static_cast<int>(gridDim.x) - 1 - static_cast<int>(blockIdx.x)
                        : static_cast<int>(blockIdx.x);
  const int bh = blockIdx.y;
  const int b = bh / H, h = bh % H;
  const int bg = b * Hkv + h / (H / Hkv);
  const int row = qt * 128 + rl;
  const int ntk = (N + 127) / 128;
  const int nkt = CAUSAL ? qt + 1 : ntk;
  // this CTA's promoted key tiles: the list of its 256-row query block
  const int* plist = nullptr;
  int pcount = 0;
  if (kv_list != nullptr) {
    const long long qb = static_cast<long long>(bh) * ((N + 255) / 256) + qt / 2;
    plist = kv_list + qb * ntk;
    pcount = min(max(__ldg(kv_count + qb), 0), ntk);  // a list row holds at most ntk tiles
  }

  if (tid == 0) {
    for (int i = 0; i < 9; ++i) mbar_init(bars + i, 1);
    mbar_init(s_free, kFp4Softmax / 32);
    mbar_init(p_full, kFp4Softmax / 32);
    mbar_init(drain, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (tid < 32) pmask[tid] = 0u;
  if (warp == 0) {
    tmem_alloc(tbase, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  for (int i = tid; i < pcount; i += kFp4Threads) {
    const int t = __ldg(plist + i);
    if (t >= 0 && t < ntk && t < Cfg::kMaxTiles) atomicOr(&pmask[t >> 5], 1u << (t & 31));
  }
  __syncthreads();
  auto promoted = [&](int t) -> bool {
    return pcount > 0 && t < Cfg::kMaxTiles && ((pmask[t >> 5] >> (t & 31)) & 1u) != 0u;
  };
  const uint32_t tmem = *tbase;

  if (warp == kIssueWarp) {
    // -------------------------------------------------------------------------- issuing warp
    // The whole warp runs this loop on warp-uniform values; lane 0 issues the TMA loads and one
    // elected lane each tensor-core instruction.
    // loads issued and waited per K / V buffer (two scalars each: an array indexed by the buffer
    // number would live in local memory)
    struct Count2 {
      int v0, v1;
      __device__ int operator[](int b) const { return b ? v1 : v0; }
      __device__ void inc(int b) {
        if (b) ++v1;
        else ++v0;
      }
    };
    Count2 n_kl{0, 0}, n_kw{0, 0}, n_vl{0, 0}, n_vw{0, 0};
    bool q_waited = false, q16_waited = false;
    auto load_k = [&](int t) {
      const int bb = t & 1;
      if (lane == 0) {
        if (promoted(t)) {
          mbar_arrive_expect_tx(k_full + bb, Cfg::kT16);
#pragma unroll
          for (int x = 0; x < D / 64; ++x)
            tma_load_3d(sk16 + bb * Cfg::kT16 + x * Cfg::kBox16, &tm_k16, k_full + bb, 64 * x, t * 128, bg);
        } else {
          mbar_arrive_expect_tx(k_full + bb, Cfg::kQK);
          tma_load_3d(sk + bb * Cfg::kQK, &tm_k, k_full + bb, 0, t * 128, bg);
        }
      }
      __syncwarp();
      n_kl.inc(bb);
    };
    auto load_v = [&](int t) {
      const int bb = t & 1;
      if (lane == 0) {
        if (promoted(t)) {
          mbar_arrive_expect_tx(v_full + bb, Cfg::kT16);
#pragma unroll
          for (int x = 0; x < D / 64; ++x)
            tma_load_3d(sv16 + bb * Cfg::kT16 + x * Cfg::kBox16, &tm_v16, v_full + bb, 64 * x, t * 128, bg);
        } else {
          mbar_arrive_expect_tx(v_full + bb, Cfg::kVt);
          tma_load_3d(sv + bb * Cfg::kVt, &tm_vt, v_full + bb, t * 64, 0, bg);
        }
      }
      __syncwarp();
      n_vl.inc(bb);
    };
    auto wait_all = [&](uint64_t* bar, uint32_t parity) {
      return __all_sync(0xFFFFFFFFu, mbar_wait(bar, parity, abort));
    };
    // Q K^T of tile t into S buffer t & 1 (its K tile, and for FP4 its scales, ready)
    auto issue_qk = [&](int t) -> bool {
      const int bb = t & 1;
      const bool pr = promoted(t);
      if (pr && !q16_waited) q16_waited = wait_all(q16_full, 0);
      if (!pr && !q_waited) q_waited = wait_all(q_full, 0);
      if (!(pr ? q16_waited : q_waited)) return false;
      if (!wait_all(k_full + bb, static_cast<uint32_t>(n_kw[bb]) & 1u)) return false;
      n_kw.inc(bb);
      tc_fence_after();
      const uint32_t ds = tmem + Cfg::kColS + 128 * bb;
      if (pr) {
        constexpr uint32_t id = idesc_f16_f32_kk(128, 128);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk / 4) * Cfg::kBox16 + (kk % 4) * 32;
          const uint64_t ad = smem_desc(smem_u32(sq16) + off, 16, 1024, kSwizzle128B);
          const uint64_t bd = smem_desc(smem_u32(sk16 + bb * Cfg::kT16) + off, 16, 1024, kSwizzle128B);
          mma_f16_ss_warp(ds, ad, bd, id, kk > 0 ? 1u : 0u);
        }
      } else {
        constexpr uint32_t id = idesc_nvf4(128, 128);
#pragma unroll
        for (int kc = 0; kc < Cfg::kStepsQK; ++kc) {
          const uint64_t ad = smem_desc(smem_u32(sq) + kc * 32, 16, Cfg::kSboQK, Cfg::kSwQK);
          const uint64_t bd = smem_desc(smem_u32(sk + bb * Cfg::kQK) + kc * 32, 16, Cfg::kSboQK, Cfg::kSwQK);
          mma_nvf4_ss_warp(ds, ad, bd, id, tmem + Cfg::kColSfq + 4 * kc,
                           tmem + Cfg::kColSfk + 4 * kc, kc > 0 ? 1u : 0u);
        }
      }
      mma_commit_warp(s_full + bb);
      return true;
    };
    // P V of tile t into the P V tile (P and, for FP4, its scales ready)
    auto issue_pv = [&](int t) -> bool {
      const int bb = t & 1;
      if (!wait_all(v_full + bb, static_cast<uint32_t>(n_vw[bb]) & 1u)) return false;
      n_vw.inc(bb);
      tc_fence_after();
      if (promoted(t)) {
        constexpr uint32_t id = idesc_f16_f32_bmn(128, D);
        const uint64_t dv = smem_desc(smem_u32(sv16 + bb * Cfg::kT16), Cfg::kBox16, 1024, kSwizzle128B);
        const uint32_t ap = tmem + Cfg::kColS + 128 * bb;  // fp16 P over S buffer bb
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_f16_ts_warp(tmem + Cfg::kColO, ap + 8 * kk, dv + 128 * kk, id, kk > 0 ? 1u : 0u);
      } else {
        // P's block scales, staged by the softmax warps, into every sub-partition
#pragma unroll
        for (int kc = 0; kc < 2; ++kc)
          tmem_cp32x128_warpx4_warp(tmem + Cfg::kColSfp + 4 * kc, smem_desc(smem_u32(sfp) + kc * 512, 128, 128, 0));
        constexpr uint32_t id = idesc_nvf4(128, D);
#pragma unroll
        for (int kc = 0; kc < 2; ++kc) {
          const uint64_t ad = smem_desc(smem_u32(sp) + kc * 32, 16, 512, kSwizzle64B);
          const uint64_t bd = smem_desc(smem_u32(sv + bb * Cfg::kVt) + kc * 32, 16, 512, kSwizzle64B);
          mma_nvf4_ss_warp(tmem + Cfg::kColO, ad, bd, id, tmem + Cfg::kColSfp + 4 * kc,
                           tmem + Cfg::kColSfv + Cfg::kSfvCols * kc, kc > 0 ? 1u : 0u);
        }
      }
      mma_commit_warp(o_full);
      return true;
    };

    if (lane == 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_vt);
      mbar_arrive_expect_tx(q_full, Cfg::kQK);
      tma_load_3d(sq, &tm_q, q_full, 0, qt * 128, bh);
      if (pcount > 0) {
        mbar_arrive_expect_tx(q16_full, Cfg::kT16);
#pragma unroll
        for (int x = 0; x < D / 64; ++x)
          tma_load_3d(sq16 + x * Cfg::kBox16, &tm_q16, q16_full, 64 * x, qt * 128, bh);
      }
    }
    __syncwarp();
    load_k(0);
    if (nkt > 1) load_k(1);
    load_v(0);
    // Q K^T(0) once the softmax warps have put Q's and tile 0's K scales into tensor memory
    bool ok = wait_all(s_free, 0) && issue_qk(0);
    for (int t = 0; ok && t < nkt; ++t) {
      if (t + 1 < nkt) {
        // the softmax warps have read S(t) (so Q K^T(t) is done) and written tile t + 1's K scales
        ok = wait_all(s_free, static_cast<uint32_t>(t + 1) & 1u);
        if (!ok) break;
        if (t + 2 < nkt) load_k(t + 2);
        ok = issue_qk(t + 1);
        if (!ok) break;
      }
      // P(t) and its scales are written (so the softmax warps have folded P V(t - 1): done)
      ok = wait_all(p_full, static_cast<uint32_t>(t) & 1u);
      if (!ok) break;
      if (t + 1 < nkt) load_v(t + 1);
      ok = issue_pv(t);
    }
    // every tensor-core operation and load of this warp has finished before the tensor memory and
    // shared memory go away (immediate on the normal path; bounded after a timeout)
    mma_commit_warp(drain);
    drain_wait(drain, 0);
    if (!q_waited) drain_wait(q_full, 0);
    if (pcount > 0 && !q16_waited) drain_wait(q16_full, 0);
#pragma unroll
    for (int bb = 0; bb < 2; ++bb) {
      for (int n = n_kw[bb]; n < n_kl[bb]; ++n) drain_wait(k_full + bb, static_cast<uint32_t>(n) & 1u);
      for (int n = n_vw[bb]; n < n_vl[bb]; ++n) drain_wait(v_full + bb, static_cast<uint32_t>(n) & 1u);
    }
  } else {
    // -------------------------------------------------------------------------- softmax warps
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const uint8_t* ksf = k_sf + static_cast<size_t>(bg) * N * (D / 16);
    const uint8_t* vsf = vt_sf + static_cast<size_t>(bg) * D * (Np / 16);
    // K scale words of tile t for this thread: d = 128, K step pt >> 1, keys lane + 32 r1 with
    // r1 = 2 (pt & 1), 2 (pt & 1) + 1; d = 64 (one step), r1 = pt.
    auto load_k_words = [&](int t, uint32_t (&w)[2]) {
      if constexpr (D == 128) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int key = t * 128 + lane + 32 * (2 * (pt & 1) + e);
          w[e] = key < N ? __ldg(reinterpret_cast<const uint32_t*>(ksf + static_cast<size_t>(key) * (D / 16) + 4 * (pt >> 1)))
                         : 0u;
        }
      } else {
        const int key = t * 128 + lane + 32 * pt;
        w[0] = key < N ? __ldg(reinterpret_cast<const uint32_t*>(ksf + static_cast<size_t>(key) * (D / 16))) : 0u;
        w[1] = 0u;
      }
    };
    auto store_k_words = [&](const uint32_t (&w)[2]) {
      if constexpr (D == 128) tmem_st32x2(lane_base + Cfg::kColSfk + 4 * (pt >> 1) + 2 * (pt & 1), w[0], w[1]);
      else tmem_st32x1(lane_base + Cfg::kColSfk + pt, w[0]);
    };
    // V scale words of tile t: K step pt >> 1, channel rows lane + 32 r1 with r1 = 2 (pt & 1) + e
    // (d = 128) or r1 = pt & 1 (d = 64).
    auto load_v_words = [&](int t, uint32_t (&w)[2]) {
      constexpr int kPer = D == 128 ? 2 : 1;
#pragma unroll
      for (int e = 0; e < kPer; ++e) {
        const int ch = lane + 32 * (kPer * (pt & 1) + e);
        w[e] = __ldg(reinterpret_cast<const uint32_t*>(vsf + static_cast<size_t>(ch) * (Np / 16) + t * 8 + 4 * (pt >> 1)));
      }
      if constexpr (kPer == 1) w[1] = 0u;
    };
    auto store_v_words = [&](const uint32_t (&w)[2]) {
      if constexpr (D == 128) tmem_st32x2(lane_base + Cfg::kColSfv + 4 * (pt >> 1) + 2 * (pt & 1), w[0], w[1]);
      else tmem_st32x1(lane_base + Cfg::kColSfv + 2 * (pt >> 1) + (pt & 1), w[0]);
    };
    auto arrive = [&](uint64_t* bar) {
      __syncwarp();
      if (lane == 0) mbar_arrive(bar);
    };
    // Q's scales (all K steps, part 0's warps) and tile 0's K scales into this warp's
    // sub-partition, then s_free phase 0
    if (pt == 0) {
      const uint8_t* qsf = q_sf + static_cast<size_t>(bh) * N * (D / 16);
#pragma unroll
      for (int kc = 0; kc < Cfg::kStepsQK; ++kc) {
        uint32_t w[4];
        load_sf_words(qsf, D, N, qt * 128, kc, w);
        tmem_st32x4(lane_base + Cfg::kColSfq + 4 * kc, w[0], w[1], w[2], w[3]);
      }
    }
    if (!promoted(0)) {
      uint32_t w[2];
      load_k_words(0, w);
      store_k_words(w);
    }
    tmem_st_wait();
    tc_fence_before();
    arrive(s_free);
    // c = q . mean for this row (FP16 scores minus c see the smoothed keys)
    float cq = 0.0f;
    if (pcount > 0 && row < N) {
      const uint4* qr = reinterpret_cast<const uint4*>(q16 + (static_cast<size_t>(bh) * N + row) * D);
      const float* mr = k_mean + static_cast<size_t>(bg) * D;
#pragma unroll 4
      for (int c8 = 0; c8 < D / 8; ++c8) {
        const uint4 v = __ldg(qr + c8);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          cq = fmaf(half_bits_to_float(w[e] & 0xFFFFu), __ldg(mr + 8 * c8 + 2 * e), cq);
          cq = fmaf(half_bits_to_float(w[e] >> 16), __ldg(mr + 8 * c8 + 2 * e + 1), cq);
        }
      }
    }
    const float gqk = __ldg(q_g + bh) * __ldg(k_g + bg) * sl2;  // FP4 S to log2 units
    const float gv = __ldg(v_g + bg);
    float m = -INFINITY, l = 0.0f, corr_prev = 0.0f, f_prev = 0.0f;
    float o[DP];
#pragma unroll
    for (int c = 0; c < DP; ++c) o[c] = 0.0f;
    bool ok = true;
    const uint32_t swz = static_cast<uint32_t>((rl >> 1) & 3);
    const uint32_t prow = smem_u32(sp) + rl * 64;

    for (int j = 0; j < nkt; ++j) {
      const int sb = j & 1;  // S buffer of tile j
      const bool prom = promoted(j);
      const bool next_fp4 = j + 1 < nkt && !promoted(j + 1);
      // scale words for this step's tensor-memory writes, loaded before the S wait
      uint32_t kw[2] = {0u, 0u}, vw[2] = {0u, 0u};
      if (next_fp4) load_k_words(j + 1, kw);
      if (!prom) load_v_words(j, vw);
      // (1) S(j), this quarter row's 32 scores
      const bool wok = mbar_wait(s_full + sb, static_cast<uint32_t>(j >> 1) & 1u, abort);
      tc_fence_after();
      uint32_t s[32];
      tmem_ld32(lane_base + Cfg::kColS + 128 * sb + 32 * pt, s);
      tmem_ld_wait(s);
      // (2) tile j + 1's K scales (Q K^T(j) is done; Q K^T(j + 1) waits for s_free)
      if (next_fp4) store_k_words(kw);
      tmem_st_wait();
      tc_fence_before();
      if (j + 1 < nkt) arrive(s_free);
      // (3) row maximum of the raw scores (the scaling below is monotone), exchanged among the
      // parts; the softmax warps agree here on whether every wait so far succeeded
      const int kb = j * 128 + 32 * pt;
      const bool masked = j * 128 + 127 >= N || (CAUSAL && j == qt);
      float smax = -INFINITY;
      if (masked) {
#pragma unroll
        for (int k = 0; k < 32; ++k)
          if (kb + k < N && (!CAUSAL || kb + k <= row)) smax = fmaxf(smax, __uint_as_float(s[k]));
      } else {
#pragma unroll
        for (int k = 0; k < 32; k += 2) smax = fmax3(smax, __uint_as_float(s[k]), __uint_as_float(s[k + 1]));
      }
      // by step parity: a part writes this buffer again two steps on, after the next step's
      // barrier, which every part reaches only after its reads below.  The barrier joins the four
      // parts of this lane quadrant (the only readers of its rows' entries; named barrier 5 +
      // quadrant, 128 threads); a quadrant whose wait gave up leaves here, and the others leave at
      // their next wait once the issuing warp raises the abort flag.
      float* rm = red + 512 * (j & 1);
      rm[pt * 128 + rl] = smax;
      ok = named_bar_and(5 + quad, 128, ok && wok);
      if (!ok) break;
      tc_fence_after();
      const float row_smax = fmaxf(fmaxf(rm[rl], rm[128 + rl]), fmaxf(rm[256 + rl], rm[384 + rl]));
      // (4) running maximum
      const float t = prom ? (row_smax - cq) * sl2 : row_smax * gqk;
      const float m_new = fmaxf(m, t);
      const float corr = ex2_approx(m - m_new);
      // (5) P of this quarter row, in registers (the scores die here)
      float lsum, f, gp = 0.0f;
      uint32_t cw[4] = {0u, 0u, 0u, 0u}, sw = 0u;
      if (prom) {
        uint32_t pk[16];
        lsum = masked ? fp16_quarter_row<true, CAUSAL>(s, kb, row, N, cq, sl2, m_new, pk)
                      : fp16_quarter_row<false, CAUSAL>(s, kb, row, N, cq, sl2, m_new, pk);
        // keys 32 pt .. 32 pt + 31 -> P columns 16 pt .. 16 pt + 15 of S buffer sb (every score
        // of S(j) is in registers by now: the barrier above follows all loads; P V(j - 1) reads
        // the other buffer)
        tmem_st32x16(lane_base + Cfg::kColS + 128 * sb + 16 * pt, pk);
        f = 1.0f;
      } else {
        gp = __fdiv_rn(ex2_approx(fmaf(row_smax, gqk, -m_new)), kNvfp4Div);
        lsum = masked ? fp4_quarter_row<true, CAUSAL>(s, kb, row, N, gqk, m_new, gp, cw, sw)
                      : fp4_quarter_row<false, CAUSAL>(s, kb, row, N, gqk, m_new, gp, cw, sw);
        f = gp * gv;
      }
      // (6) P V(j - 1) into the outputs; its completion also frees the P operand and the P and V
      // scales for this tile
      bool pok = true;
      if (j > 0) {
        pok = mbar_wait(o_full, static_cast<uint32_t>(j - 1) & 1u, abort);
        tc_fence_after();
        uint32_t acc[DP];
        tmem_ld_part<DP>(lane_base + Cfg::kColO + DP * pt, acc);
#pragma unroll
        for (int c = 0; c < DP; c += 2)
          fold2(o[c], o[c + 1], __uint_as_float(acc[c]), __uint_as_float(acc[c + 1]), corr_prev, f_prev);
      }
      if (!prom) {
        // 16 bytes (keys 32 pt .. 32 pt + 31) into the 64-byte-swizzled row of the P operand
        st_shared_v4(prow + ((static_cast<uint32_t>(pt) ^ swz) << 4), cw[0], cw[1], cw[2], cw[3]);
        // the two scale bytes: half (pt & 1) of row rl's word for K step pt >> 1, at word
        // (pt >> 1, rl % 32, rl / 32) of the staging area the issuing warp copies from
        reinterpret_cast<uint16_t*>(sfp)[((pt >> 1) * 128 + (rl & 31) * 4 + (rl >> 5)) * 2 + (pt & 1)] =
            static_cast<uint16_t>(sw);
        fence_proxy_async_smem();
        store_v_words(vw);
      }
      l = l * corr + lsum;
      tmem_st_wait();
      tc_fence_before();
      arrive(p_full);
      ok = ok && pok;
      corr_prev = corr;
      f_prev = f;
      m = m_new;
    }
    // the last P V, folded; then the row sum over the parts and the output
    bool fin = ok && mbar_wait(o_full, static_cast<uint32_t>(nkt - 1) & 1u, abort);
    fin = named_bar_and(3, kFp4Softmax, fin);
    tc_fence_after();
    if (fin) {
      uint32_t acc[DP];
      tmem_ld_part<DP>(lane_base + Cfg::kColO + DP * pt, acc);
#pragma unroll
      for (int c = 0; c < DP; c += 2)
        fold2(o[c], o[c + 1], __uint_as_float(acc[c]), __uint_as_float(acc[c + 1]), corr_prev, f_prev);
      red[pt * 128 + rl] = l;
    }
    named_bar_sync(4, kFp4Softmax);
    if (fin && row < N) {
      const float inv = 1.0f / ((red[rl] + red[128 + rl]) + (red[256 + rl] + red[384 + rl]));
      uint4* dst = reinterpret_cast<uint4*>(out + (static_cast<size_t>(bh) * N + row) * D + DP * pt);
#pragma unroll
      for (int c = 0; c < DP; c += 8) {
        uint4 w;
        w.x = pack_half2(o[c] * inv, o[c + 1] * inv);
        w.y = pack_half2(o[c + 2] * inv, o[c + 3] * inv);
        w.z = pack_half2(o[c + 4] * inv, o[c + 5] * inv);
        w.w = pack_half2(o[c + 6] * inv, o[c + 7] * inv);
        dst[c / 8] = w;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace qattn
