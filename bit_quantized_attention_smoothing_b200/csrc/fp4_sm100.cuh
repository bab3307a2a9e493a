// fp4_sm100.cuh -- FP4 scores on the block-scaled tensor cores: the Q K^T product of the FP4 path
// of the ThriftAttention page ("ThriftAttention: Selective Mixed Precision for Long-Context FP4
// Attention", gist.science/ja/paper/2605.23081, method section, "FP4 path": blocks computed in
// FP4 with the NVFP4 micro-scaling format on Blackwell's native FP4 tensor cores).
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
// in each of the four 32-lane sub-partitions.  Each warp writes its own sub-partition's copy with
// tcgen05.st, so no shared-memory staging is needed for the scales.
#pragma once

#include <cstdint>

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
