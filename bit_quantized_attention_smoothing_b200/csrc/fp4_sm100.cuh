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
// in each of the four 32-lane sub-partitions.  Each warp writes its own sub-partition's copy with
// tcgen05.st, so no shared-memory staging is needed for the scales.
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
// One CTA of 4 warps per 128-row query tile; thread t owns query row 128 qt + t, which is TMEM lane
// t.  Per key tile: (a) FP4 tiles: the warps put K's and V's block scales into tensor memory;
// (b) one thread loads the tile's operands by TMA and issues Q K^T; (c) every thread reads its row
// of S, takes the online maximum and writes its P row (FP4: codes into the swizzled shared-memory
// operand, scales through shared memory into every sub-partition; FP16: pairs into tensor memory);
// (d) one thread issues P V into a tensor-memory tile; (e) the threads fold it into their fp32
// output rows.  The FP16 query tile is loaded only by CTAs with promoted tiles.  The steps run one
// after another (no pipelining across tiles).  Every wait is bounded and each outcome is agreed by
// the whole CTA (__syncthreads_and), so a wait that runs out ends every thread's loop together.
// ------------------------------------------------------------------------------------------------

template <int D>
struct Fp4AttnCfg {
  static constexpr int kQK = 128 * (D / 2);  // E2M1 Q or K tile: 128 rows of D/2 bytes
  static constexpr int kVt = D * 64;         // E2M1 V^T tile: D channel rows of 128 keys
  static constexpr int kP = 128 * 64;        // E2M1 P tile: 128 rows of 128 keys
  static constexpr int kT16 = 128 * D * 2;   // fp16 tile of 128 rows (D/64 boxes of 64 columns)
  static constexpr int kBox16 = 128 * 128;   // one 64-column fp16 box: 128 rows of 128 bytes
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kQK;
  static constexpr int kOffV = 2 * kQK;
  static constexpr int kOffP = 2 * kQK + kVt;
  static constexpr int kOffSfp = kOffP + kP;      // uint32 [2][128]: P scale words by K step
  static constexpr int kOffQ16 = kOffSfp + 1024;
  static constexpr int kOffK16 = kOffQ16 + kT16;
  static constexpr int kOffV16 = kOffK16 + kT16;
  static constexpr int kOffBar = kOffV16 + kT16;
  static constexpr int kSmemUsed = kOffBar + 64 + 1024;
  static constexpr uint32_t kSwQK = D == 128 ? kSwizzle64B : kSwizzle32B;
  static constexpr uint32_t kSboQK = 8 * (D / 2);
  static constexpr int kStepsQK = D / 64;         // K = 64 per FP4 instruction
  static constexpr int kSfvCols = D / 32;         // V scale columns per K step (N = D)
  // tensor-memory columns: S, the P V tile, the four scale-factor areas, fp16 P (64 columns)
  static constexpr uint32_t kColS = 0, kColO = 128, kColSfq = 256, kColSfk = 264, kColSfp = 272,
                            kColSfv = 280, kColP16 = 288;
};

// Sum of twice the E2M1 magnitudes of the eight codes in w (values 0, .5, 1, 1.5, 2, 3, 4, 6 are
// 0, 1, 2, 3, 4, 6, 8, 12 when doubled: one nibble each in the table 0xC8643210).
__device__ __forceinline__ uint32_t e2m1x8_twice_sum(uint32_t w) {
  uint32_t s = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) s += (0xC8643210u >> (4 * ((w >> (4 * i)) & 7u))) & 15u;
  return s;
}

__device__ __forceinline__ void tmem_st32x2(uint32_t taddr, uint32_t a, uint32_t b) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x2.b32 [%0], {%1, %2};" ::"r"(taddr), "r"(a),
               "r"(b)
               : "memory");
}

__device__ __forceinline__ void tmem_st32x16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
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

template <int D, bool CAUSAL>
__global__ void __launch_bounds__(128, 1)
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
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kOffBar);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;
  uint64_t* s_done = bars + 2;
  uint64_t* o_done = bars + 3;
  uint64_t* q16_full = bars + 4;
  uint32_t* tbase = reinterpret_cast<uint32_t*>(bars + 5);
  volatile int* abort = reinterpret_cast<volatile int*>(bars + 6);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int qt = CAUSAL ? static_cast<int>(gridDim.x) - 1 - static_cast<int>(blockIdx.x)
                        : static_cast<int>(blockIdx.x);
  const int bh = blockIdx.y;
  const int b = bh / H, h = bh % H;
  const int bg = b * Hkv + h / (H / Hkv);
  const int row = qt * 128 + tid;
  const int ntk = (N + 127) / 128;
  const int nkt = CAUSAL ? qt + 1 : ntk;
  // this CTA's promoted key tiles: the list of its 256-row query block (ascending)
  const int* plist = nullptr;
  int pcount = 0;
  if (kv_list != nullptr) {
    const long long qb = static_cast<long long>(bh) * ((N + 255) / 256) + qt / 2;
    plist = kv_list + qb * ntk;
    pcount = __ldg(kv_count + qb);
  }

  if (tid == 0) {
    for (int i = 0; i < 5; ++i) mbar_init(bars + i, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tbase, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tbase;
  const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
  const uint8_t* ksf = k_sf + static_cast<size_t>(bg) * N * (D / 16);
  const uint8_t* vsf = vt_sf + static_cast<size_t>(bg) * D * (Np / 16);
  {
    const uint8_t* qsf = q_sf + static_cast<size_t>(bh) * N * (D / 16);
#pragma unroll
    for (int kc = 0; kc < Cfg::kStepsQK; ++kc) {
      uint32_t w[4];
      load_sf_words(qsf, D, N, qt * 128, kc, w);
      tmem_st32x4(lane_base + Cfg::kColSfq + 4 * kc, w[0], w[1], w[2], w[3]);
    }
  }
  if (tid == 0) {
    mbar_arrive_expect_tx(q_full, Cfg::kQK);
    tma_load_3d(sq, &tm_q, q_full, 0, qt * 128, bh);
    if (pcount > 0) {
      mbar_arrive_expect_tx(q16_full, Cfg::kT16);
#pragma unroll
      for (int x = 0; x < D / 64; ++x)
        tma_load_3d(sq16 + x * Cfg::kBox16, &tm_q16, q16_full, 64 * x, qt * 128, bh);
    }
  }
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
  float m = -INFINITY, l = 0.0f;
  float o[D];
#pragma unroll
  for (int c = 0; c < D; ++c) o[c] = 0.0f;
  bool ok = true;
  bool q16_ready = false;
  int pi = 0;

  for (int kt = 0; kt < nkt; ++kt) {
    const uint32_t ph = static_cast<uint32_t>(kt & 1);
    while (pi < pcount && __ldg(plist + pi) < kt) ++pi;
    const bool promoted = pi < pcount && __ldg(plist + pi) == kt;
    // (a) FP4 tiles: K's and V's block scales into this warp's sub-partition
    if (!promoted) {
#pragma unroll
      for (int kc = 0; kc < Cfg::kStepsQK; ++kc) {
        uint32_t w[4];
        load_sf_words(ksf, D, N, kt * 128, kc, w);
        tmem_st32x4(lane_base + Cfg::kColSfk + 4 * kc, w[0], w[1], w[2], w[3]);
      }
#pragma unroll
      for (int kc = 0; kc < 2; ++kc) {
        uint32_t w[4];
#pragma unroll
        for (int r1 = 0; r1 < Cfg::kSfvCols; ++r1)
          w[r1] = __ldg(reinterpret_cast<const uint32_t*>(
              vsf + static_cast<size_t>(lane + 32 * r1) * (Np / 16) + kt * 8 + 4 * kc));
        if constexpr (D == 128)
          tmem_st32x4(lane_base + Cfg::kColSfv + 4 * kc, w[0], w[1], w[2], w[3]);
        else
          tmem_st32x2(lane_base + Cfg::kColSfv + 2 * kc, w[0], w[1]);
      }
    }
    tmem_st_wait();
    tc_fence_before();
    __syncthreads();
    // (b) the tile's operands, then S = Q K^T
    if (tid == 0) {
      tc_fence_after();
      bool loaded;
      if (promoted) {
        mbar_arrive_expect_tx(kv_full, 2 * Cfg::kT16);
#pragma unroll
        for (int x = 0; x < D / 64; ++x) {
          tma_load_3d(sk16 + x * Cfg::kBox16, &tm_k16, kv_full, 64 * x, kt * 128, bg);
          tma_load_3d(sv16 + x * Cfg::kBox16, &tm_v16, kv_full, 64 * x, kt * 128, bg);
        }
        loaded = (q16_ready || mbar_wait(q16_full, 0, abort)) && mbar_wait(kv_full, ph, abort);
        q16_ready = true;
      } else {
        mbar_arrive_expect_tx(kv_full, Cfg::kQK + Cfg::kVt);
        tma_load_3d(sk, &tm_k, kv_full, 0, kt * 128, bg);
        tma_load_3d(sv, &tm_vt, kv_full, kt * 64, 0, bg);
        loaded = (kt > 0 || mbar_wait(q_full, 0, abort)) && mbar_wait(kv_full, ph, abort);
      }
      if (kt == 0 && promoted && loaded) loaded = mbar_wait(q_full, 0, abort);
      if (loaded) {
        tc_fence_after();
        if (promoted) {
          constexpr uint32_t id = idesc_f16_f32_kk(128, 128);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk / 4) * Cfg::kBox16 + (kk % 4) * 32;
            const uint64_t ad = smem_desc(smem_u32(sq16) + off, 16, 1024, kSwizzle128B);
            const uint64_t bd = smem_desc(smem_u32(sk16) + off, 16, 1024, kSwizzle128B);
            mma_f16_ss(tmem + Cfg::kColS, ad, bd, id, kk > 0 ? 1u : 0u);
          }
        } else {
          constexpr uint32_t id = idesc_nvf4(128, 128);
#pragma unroll
          for (int kc = 0; kc < Cfg::kStepsQK; ++kc) {
            const uint64_t ad = smem_desc(smem_u32(sq) + kc * 32, 16, Cfg::kSboQK, Cfg::kSwQK);
            const uint64_t bd = smem_desc(smem_u32(sk) + kc * 32, 16, Cfg::kSboQK, Cfg::kSwQK);
            mma_nvf4_ss(tmem + Cfg::kColS, ad, bd, id, tmem + Cfg::kColSfq + 4 * kc,
                        tmem + Cfg::kColSfk + 4 * kc, kc > 0 ? 1u : 0u);
          }
        }
        mma_commit(s_done);
      }
    }
    ok = __syncthreads_and(mbar_wait(s_done, ph, abort));
    if (!ok) break;
    tc_fence_after();
    // (c) this row's online softmax step
    const int kbase = kt * 128;
    const float xs = promoted ? sl2 : gqk;   // x = (S - xo) * xs, log2 units
    const float xo = promoted ? cq : 0.0f;
    float tmax = -INFINITY;
#pragma unroll 1
    for (int cc = 0; cc < 4; ++cc) {
      uint32_t v[32];
      tmem_ld32(lane_base + Cfg::kColS + 32 * cc, v);
      tmem_ld_wait(v);
#pragma unroll
      for (int t = 0; t < 32; ++t) {
        const int key = kbase + 32 * cc + t;
        const bool valid = key < N && (!CAUSAL || key <= row);
        if (valid) tmax = fmaxf(tmax, (__uint_as_float(v[t]) - xo) * xs);
      }
    }
    const float m_new = fmaxf(m, tmax);
    const float corr = exp2f(m - m_new);
    float f;      // factor of the tile's P V accumulator
    float lsum = 0.0f;
    if (promoted) {
      // fp16 P pairs (keys 2c, 2c + 1 in column c) into tensor memory; l takes the rounded P
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t v[32];
        tmem_ld32(lane_base + Cfg::kColS + 32 * cc, v);
        tmem_ld_wait(v);
        uint32_t pk[16];
#pragma unroll
        for (int t = 0; t < 32; t += 2) {
          const int key = kbase + 32 * cc + t;
          const bool v0 = key < N && (!CAUSAL || key <= row);
          const bool v1 = key + 1 < N && (!CAUSAL || key + 1 <= row);
          const float p0 = v0 ? exp2f((__uint_as_float(v[t]) - xo) * xs - m_new) : 0.0f;
          const float p1 = v1 ? exp2f((__uint_as_float(v[t + 1]) - xo) * xs - m_new) : 0.0f;
          pk[t / 2] = pack_half2(p0, p1);
          lsum = add_half2_f32(lsum, pk[t / 2]);
        }
        tmem_st32x16(lane_base + Cfg::kColP16 + 16 * cc, pk);
      }
      l = l * corr + lsum;
      f = 1.0f;
      tmem_st_wait();
      tc_fence_before();
      __syncthreads();
      if (tid == 0) {
        tc_fence_after();
        constexpr uint32_t id = idesc_f16_f32_bmn(128, D);
        const uint64_t dv = smem_desc(smem_u32(sv16), Cfg::kBox16, 1024, kSwizzle128B);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_f16_ts(tmem + Cfg::kColO, tmem + Cfg::kColP16 + 8 * kk, dv + 128 * kk, id,
                     kk > 0 ? 1u : 0u);
        mma_commit(o_done);
      }
    } else {
      // two-level FP4 quantization of the P row
      const float gp = __fdiv_rn(exp2f(tmax - m_new), kNvfp4Div);
      const float sixg = __fmul_rn(6.0f, gp);
      uint32_t sfw0 = 0, sfw1 = 0;
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t v[32];
        tmem_ld32(lane_base + Cfg::kColS + 32 * cc, v);
        tmem_ld_wait(v);
        float p[32];
#pragma unroll
        for (int t = 0; t < 32; ++t) {
          const int key = kbase + 32 * cc + t;
          const bool valid = key < N && (!CAUSAL || key <= row);
          p[t] = valid ? exp2f(__uint_as_float(v[t]) * gqk - m_new) : 0.0f;
        }
        uint32_t cw[4];
#pragma unroll
        for (int hb = 0; hb < 2; ++hb) {
          float* pb = p + 16 * hb;
          float bmax = 0.0f;
#pragma unroll
          for (int i = 0; i < 16; ++i) bmax = fmaxf(bmax, pb[i]);
          const uint32_t s = gp > 0.0f ? ue4m3_byte(__fdiv_rn(bmax, sixg)) : 0u;
          cw[2 * hb] = 0u;
          cw[2 * hb + 1] = 0u;
          if (s != 0u) {
            const float sc = __fmul_rn(ue4m3_value(s), gp);
#pragma unroll
            for (int i = 0; i < 16; ++i) pb[i] = __fdiv_rn(pb[i], sc);
            cw[2 * hb] = e2m1x8(pb);
            cw[2 * hb + 1] = e2m1x8(pb + 8);
            lsum += 0.5f * sc *
                    static_cast<float>(e2m1x8_twice_sum(cw[2 * hb]) + e2m1x8_twice_sum(cw[2 * hb + 1]));
          }
          const int blk = 2 * cc + hb;  // 16-key block 0..7 of the tile
          if (blk < 4) sfw0 |= s << (8 * blk);
          else sfw1 |= s << (8 * (blk - 4));
        }
        // 16 bytes (keys 32 cc .. 32 cc + 31) into the 64-byte-swizzled row of the P operand
        st_shared_v4(smem_u32(sp) + tid * 64 + ((cc ^ ((tid >> 1) & 3)) << 4), cw[0], cw[1], cw[2],
                     cw[3]);
      }
      l = l * corr + lsum;
      f = gp * gv;
      sfp[tid] = sfw0;
      sfp[128 + tid] = sfw1;
      fence_proxy_async_smem();
      __syncthreads();
      // (d) P's scales: row r0 + 32 r1 in column r1 of lane r0, in every sub-partition
#pragma unroll
      for (int kc = 0; kc < 2; ++kc)
        tmem_st32x4(lane_base + Cfg::kColSfp + 4 * kc, sfp[128 * kc + lane],
                    sfp[128 * kc + lane + 32], sfp[128 * kc + lane + 64], sfp[128 * kc + lane + 96]);
      tmem_st_wait();
      tc_fence_before();
      __syncthreads();
      if (tid == 0) {
        tc_fence_after();
        constexpr uint32_t id = idesc_nvf4(128, D);
#pragma unroll
        for (int kc = 0; kc < 2; ++kc) {
          const uint64_t ad = smem_desc(smem_u32(sp) + kc * 32, 16, 512, kSwizzle64B);
          const uint64_t bd = smem_desc(smem_u32(sv) + kc * 32, 16, 512, kSwizzle64B);
          mma_nvf4_ss(tmem + Cfg::kColO, ad, bd, id, tmem + Cfg::kColSfp + 4 * kc,
                      tmem + Cfg::kColSfv + Cfg::kSfvCols * kc, kc > 0 ? 1u : 0u);
        }
        mma_commit(o_done);
      }
    }
    ok = __syncthreads_and(mbar_wait(o_done, ph, abort));
    if (!ok) break;
    tc_fence_after();
    // (e) fold the tile's P V into the output row: O = O * corr + acc * f
#pragma unroll
    for (int cc = 0; cc < D / 32; ++cc) {
      uint32_t v[32];
      tmem_ld32(lane_base + Cfg::kColO + 32 * cc, v);
      tmem_ld_wait(v);
#pragma unroll
      for (int t = 0; t < 32; ++t) o[32 * cc + t] = o[32 * cc + t] * corr + __uint_as_float(v[t]) * f;
    }
    m = m_new;
  }
  // a promoted list with no tile up to the causal diagonal leaves the fp16 Q load unconsumed
  if (tid == 0 && pcount > 0 && !q16_ready) (void)mbar_wait(q16_full, 0, abort);
  if (ok && row < N) {
    const float inv = 1.0f / l;
    uint4* dst = reinterpret_cast<uint4*>(out + (static_cast<size_t>(bh) * N + row) * D);
#pragma unroll
    for (int c = 0; c < D; c += 8) {
      uint4 w;
      w.x = pack_half2(o[c] * inv, o[c + 1] * inv);
      w.y = pack_half2(o[c + 2] * inv, o[c + 3] * inv);
      w.z = pack_half2(o[c + 4] * inv, o[c + 5] * inv);
      w.w = pack_half2(o[c + 6] * inv, o[c + 7] * inv);
      dst[c / 8] = w;
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
