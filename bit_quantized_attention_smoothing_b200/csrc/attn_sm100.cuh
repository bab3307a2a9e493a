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
//  * warp 9 (MMA, one thread): S_w = Q_w K^T as tcgen05.mma kind::i8 (M=128, N=128, K=32 per
//    instruction) into tensor memory, then O_w += P_w V as tcgen05.mma kind::f16 with P read
//    from tensor memory (M=128, N=d, K=16), fp32 accumulator in tensor memory;
//  * warps 0-3 and 4-7 (softmax warpgroups, one per Q tile, thread = row): tcgen05.ld of the int32
//    scores, dequantization with the two block scales, running max / sum in registers, exp2,
//    P written back as fp16 into the same tensor-memory columns (aliasing S), lazy rescaling of
//    O only when the running max grows by more than 2^8;
//  * while one warpgroup runs its softmax the tensor cores work on the other Q tile;
//  * causal: key tiles above the diagonal are never loaded or multiplied; the diagonal tile is
//    masked in registers; CTAs are launched heaviest-first;
//  * grouped-query attention: query head h reads kv head h / (H / Hkv); CTAs of the heads that
//    share a kv head are adjacent in launch order so their K/V tiles are reused from L2.
//
// Tensor memory (512 columns): S_0 [0,128), S_1 [128,256), O_0 [256,256+d), O_1 [256+d,256+2d).
#pragma once

#include <cuda_fp16.h>
#include <climits>
#include <cstdint>

#include "sm100_ptx.cuh"

namespace qattn {

constexpr int kBM = 128;     // rows per Q tile
constexpr int kBN = 128;     // keys per K/V tile
constexpr int kAttnThreads = 384;     // 3 warpgroups: softmax 0, softmax 1, TMA + MMA
constexpr int kAttnLaunchRegs = 168;   // 384 threads x 168 = 128 x 56 + 256 x 224 (setmaxnreg)
constexpr float kRescaleThreshold = 8.0f;  // log2 units: P stays <= 2^8 between rescales

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
  static constexpr int kSmemBytes = kOffBar + kBarBytes + 1024;  // + alignment slack
  // K-major int8 operands: rows of D bytes, 8-row swizzle atoms.
  static constexpr uint32_t kSwQK = D == 128 ? kSwizzle128B : kSwizzle64B;
  static constexpr uint32_t kSboQK = 8 * D;
  // V: MN-major fp16 operand, 64-column (128-byte) swizzled boxes of 128 rows.
  static constexpr uint32_t kVBox = kBN * 128;  // bytes of one 64-column box
};

struct __align__(8) AttnBars {
  uint64_t q_full;
  uint64_t kv_full[6];
  uint64_t kv_empty[6];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t pv_done[2];
  uint32_t tmem_base;
  int abort;
};

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

// One 128-key score row of one thread, held in registers as floats (exact: |S_int| < 2^24).
// Masked keys (offset > kmax) are set to -inf.  Returns the row maximum of each 64-key half,
// each half being one K scale block.
template <bool MASK>
__device__ __forceinline__ void row_to_float_max(uint32_t (&s)[4][32], int kmax, float& mx0,
                                                 float& mx1) {
  float m[2][2];
#pragma unroll
  for (int hf = 0; hf < 2; ++hf) m[hf][0] = m[hf][1] = -INFINITY;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      float x = static_cast<float>(static_cast<int>(s[c][e]));
      if (MASK && c * 32 + e > kmax) x = -INFINITY;
      s[c][e] = __float_as_uint(x);
    }
#pragma unroll
    for (int e = 0; e < 32; e += 4) {
      float& acc = m[c >> 1][(e >> 2) & 1];
      acc = fmax3(acc, __uint_as_float(s[c][e]), __uint_as_float(s[c][e + 1]));
      acc = fmax3(acc, __uint_as_float(s[c][e + 2]), __uint_as_float(s[c][e + 3]));
    }
  }
  mx0 = fmaxf(m[0][0], m[0][1]);
  mx1 = fmaxf(m[1][0], m[1][1]);
}

// p = 2^(x * c - m) for the 128 keys of the row (c = c0 for keys 0-63, c1 for keys 64-127; x
// the float scores from row_to_float_max), masked keys give 0.  P is packed as fp16 pairs (even
// key in the low half) and stored into the row's first 64 tensor-memory columns, aliasing the
// scores, which are all in registers by now.  Returns the fp32 sum of the fp16-rounded p.
template <bool MASK>
__device__ __forceinline__ float row_exp_store(const uint32_t (&s)[4][32], float c0, float c1,
                                               float neg_m, uint32_t s_tm) {
  float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
  for (int hf = 0; hf < 2; ++hf) {
    const float cc = hf == 0 ? c0 : c1;
    uint32_t pk[32];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int c = 2 * hf + q;
#pragma unroll
      for (int e = 0; e < 32; e += 2) {
        const float x0 = __uint_as_float(s[c][e]);
        const float x1 = __uint_as_float(s[c][e + 1]);
        float p0 = ex2_approx(fmaf(x0, cc, neg_m));
        float p1 = ex2_approx(fmaf(x1, cc, neg_m));
        if (MASK) {
          // -inf * 0 would be NaN for a zero-scale block: select instead
          p0 = x0 == -INFINITY ? 0.0f : p0;
          p1 = x1 == -INFINITY ? 0.0f : p1;
        }
        const uint32_t h2 = pack_half2(p0, p1);
        pk[q * 16 + (e >> 1)] = h2;
        // the row sum takes the fp16-rounded P that the P V product uses, so that O / l is a
        // weighted mean of V with exactly those weights
        acc[(e >> 1) & 3] = add_half2_f32(acc[(e >> 1) & 3], h2);
      }
    }
    tmem_st32(s_tm + hf * 32, pk);
  }
  return (acc[0] + acc[1]) + (acc[2] + acc[3]);
}

__device__ __forceinline__ void setmaxnreg_inc224() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 224;" ::: "memory");
}
__device__ __forceinline__ void setmaxnreg_dec56() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 56;" ::: "memory");
}

template <int D, bool CAUSAL>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const float* __restrict__ q_scale,
                    const float* __restrict__ k_scale, __half* __restrict__ out, int B, int H,
                    int Hkv, int N, float scale_log2) {
  using Cfg = AttnCfg<D>;
  constexpr int ST = Cfg::kStages;
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
  int pair = blockIdx.x / BH;
  const int bh = blockIdx.x % BH;
  if (CAUSAL) pair = npairs - 1 - pair;
  const int b = bh / H;
  const int h = bh % H;
  const int g = h / (H / Hkv);
  const int bg = b * Hkv + g;
  const int tq0 = 2 * pair, tq1 = 2 * pair + 1;
  const bool has1 = tq1 < nqt;
  const int nw0 = CAUSAL ? tq0 + 1 : nkt;
  const int nw1 = has1 ? (CAUSAL ? tq1 + 1 : nkt) : 0;
  const int n_kv = max(nw0, nw1);

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int s = 0; s < ST; ++s) {
      mbar_init(&bars->kv_full[s], 1);
      mbar_init(&bars->kv_empty[s], 1);
    }
    for (int w = 0; w < 2; ++w) {
      mbar_init(&bars->s_full[w], 1);
      mbar_init(&bars->p_full[w], 128);
      mbar_init(&bars->pv_done[w], 1);
    }
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp >= 8) {
    // warpgroup 2 (TMA warp, MMA warp, two idle warps) hands registers to the softmax groups
    setmaxnreg_dec56();
    if (warp == 8 && lane == 0) {
      // ---------------------------------------------------------------- TMA producer
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      mbar_arrive_expect_tx(&bars->q_full, Cfg::kQTile * (has1 ? 2 : 1));
      tma_load_3d(smem + Cfg::kOffQ, &tm_q, &bars->q_full, 0, tq0 * kBM, bh);
      if (has1) tma_load_3d(smem + Cfg::kOffQ + Cfg::kQTile, &tm_q, &bars->q_full, 0, tq1 * kBM, bh);
      for (int j = 0; j < n_kv; ++j) {
        const int s = j % ST;
        const uint32_t u = static_cast<uint32_t>(j / ST);
        if (!mbar_wait(&bars->kv_empty[s], (u & 1u) ^ 1u, abort)) break;
        mbar_arrive_expect_tx(&bars->kv_full[s], Cfg::kKTile + Cfg::kVTile);
        tma_load_3d(smem + Cfg::kOffK + s * Cfg::kKTile, &tm_k, &bars->kv_full[s], 0, j * kBN, bg);
        uint8_t* vdst = smem + Cfg::kOffV + s * Cfg::kVTile;
#pragma unroll
        for (int x = 0; x < D / 64; ++x)
          tma_load_3d(vdst + x * Cfg::kVBox, &tm_v, &bars->kv_full[s], x * 64, j * kBN, bg);
      }
    } else if (warp == 9 && lane == 0) {
      // ---------------------------------------------------------------- MMA issuer
      // Order per key tile j: PV_0(j), QK_0(j+1), PV_1(j), QK_1(j+1).  tcgen05.mma operations
      // from one thread execute in issue order, so QK_w(j+1) may be issued right behind PV_w(j)
      // although it overwrites the tensor-memory columns PV_w(j) reads P_w from; each softmax
      // group then overlaps the other group's PV + QK^T on the tensor pipe.
      constexpr uint32_t idq = idesc_i8_s32(kBM, kBN);
      constexpr uint32_t idv = idesc_f16_f32_bmn(kBM, D);
      const uint32_t q_addr = smem_u32(smem + Cfg::kOffQ);
      const uint32_t k_addr = smem_u32(smem + Cfg::kOffK);
      const uint32_t v_addr = smem_u32(smem + Cfg::kOffV);
      auto issue_qk = [&](int w, int s) {
        const uint32_t qa = q_addr + w * Cfg::kQTile;
        const uint32_t ka = k_addr + s * Cfg::kKTile;
#pragma unroll
        for (int kk = 0; kk < D / 32; ++kk) {
          const uint64_t ad = smem_desc(qa + kk * 32, 16, Cfg::kSboQK, Cfg::kSwQK);
          const uint64_t bd = smem_desc(ka + kk * 32, 16, Cfg::kSboQK, Cfg::kSwQK);
          mma_i8_ss(tmem + w * 128, ad, bd, idq, kk > 0 ? 1u : 0u);
        }
        mma_commit(&bars->s_full[w]);
      };
      bool ok = mbar_wait(&bars->q_full, 0, abort) && mbar_wait(&bars->kv_full[0], 0, abort);
      tc_fence_after();
      if (ok) {
        issue_qk(0, 0);
        if (nw1 > 0) issue_qk(1, 0);
      }
      for (int j = 0; ok && j < n_kv; ++j) {
        const int s = j % ST;
        const int s1 = (j + 1) % ST;
        bool next_ready = false;
#pragma unroll
        for (int w = 0; w < 2; ++w) {
          const int nw = w == 0 ? nw0 : nw1;
          if (!ok || j >= nw) continue;
          ok = mbar_wait(&bars->p_full[w], static_cast<uint32_t>(j) & 1u, abort);
          if (!ok) continue;
          tc_fence_after();
          const uint32_t va = v_addr + s * Cfg::kVTile;
#pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk) {
            const uint64_t bd = smem_desc(va + kk * 2048, Cfg::kVBox, 1024, kSwizzle128B);
            mma_f16_ts(tmem + 256 + w * D, tmem + w * 128 + kk * 8, bd, idv,
                       (j > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&bars->pv_done[w]);
          if (j + 1 < nw) {
            if (!next_ready) {
              ok = mbar_wait(&bars->kv_full[s1], static_cast<uint32_t>((j + 1) / ST) & 1u, abort);
              if (!ok) continue;
              tc_fence_after();
              next_ready = true;
            }
            issue_qk(w, s1);
          }
        }
        if (!ok) break;
        mma_commit(&bars->kv_empty[s]);
      }
    }
  } else {
    // ------------------------------------------------------------------ softmax warpgroups
    setmaxnreg_inc224();
    const int wg = warp >> 2;
    const int wq = warp & 3;
    const int row = wq * 32 + lane;
    const int nt = wg == 0 ? nw0 : nw1;
    if (nt > 0) {
      const int t = wg == 0 ? tq0 : tq1;
      const int qrow = t * kBM + row;
      const float sq = __ldg(q_scale + static_cast<size_t>(bh) * nqt + t);
      const float* ksc = k_scale + static_cast<size_t>(bg) * nkb;
      const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
      const uint32_t s_tm = tmem + lane_off + wg * 128;
      const uint32_t o_tm = tmem + lane_off + 256 + wg * D;
      float m_used = -INFINITY;
      float l = 0.0f;
      bool ok = true;
      float ks0 = __ldg(ksc);
      float ks1 = nkb > 1 ? __ldg(ksc + 1) : 0.0f;
      for (int j = 0; j < nt; ++j) {
        // K scales of the next tile, fetched ahead of the wait
        const float nks0 = (2 * j + 2 < nkb) ? __ldg(ksc + 2 * j + 2) : 0.0f;
        const float nks1 = (2 * j + 3 < nkb) ? __ldg(ksc + 2 * j + 3) : 0.0f;
        ok = __all_sync(0xFFFFFFFFu, mbar_wait(&bars->s_full[wg], static_cast<uint32_t>(j) & 1u, abort));
        if (!ok) break;
        tc_fence_after();
        uint32_t sr[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(s_tm + c * 32, sr[c]);
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld_wait(sr[c]);
        int kmax = N - 1 - j * kBN;
        if (CAUSAL && j == t) kmax = min(kmax, row);
        const float c0 = sq * ks0 * scale_log2;
        const float c1 = sq * ks1 * scale_log2;
        ks0 = nks0;
        ks1 = nks1;
        // warp-uniform, so that every lane runs the same tensor-memory access sequence
        const bool masked = __any_sync(0xFFFFFFFFu, kmax < kBN - 1);
        float mx0, mx1;
        if (masked) row_to_float_max<true>(sr, kmax, mx0, mx1);
        else row_to_float_max<false>(sr, kmax, mx0, mx1);
        float mt = -INFINITY;
        if (mx0 != -INFINITY) mt = mx0 * c0;
        if (mx1 != -INFINITY) mt = fmaxf(mt, mx1 * c1);
        const float m_new = fmaxf(m_used, mt);
        const bool need = m_new > m_used + kRescaleThreshold;
        if (j == 0) {
          m_used = m_new;
        } else if (__any_sync(0xFFFFFFFFu, need)) {
          // O holds PV up to tile j-1 (complete: QK(j) was issued after PV(j-1)).
          float alpha = 1.0f;
          if (need) {
            alpha = ex2_approx(m_used - m_new);
            m_used = m_new;
            l *= alpha;
          }
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(o_tm + c * 32, o);
            tmem_ld_wait(o);
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tmem_st32(o_tm + c * 32, o);
          }
        }
        float psum;
        if (masked) psum = row_exp_store<true>(sr, c0, c1, -m_used, s_tm);
        else psum = row_exp_store<false>(sr, c0, c1, -m_used, s_tm);
        l += psum;
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&bars->p_full[wg]);
      }
      if (ok) ok = mbar_wait(&bars->pv_done[wg], static_cast<uint32_t>(nt - 1) & 1u, abort);
      ok = __all_sync(0xFFFFFFFFu, ok);
      tc_fence_after();
      if (ok) {
        const float inv_l = 1.0f / l;
        __half* orow = out + (static_cast<size_t>(bh) * N + qrow) * D;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(o_tm + c * 32, o);
          tmem_ld_wait(o);
          if (qrow < N) {
            uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
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
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------------------------------------
// int32 score tiles through the same TMA -> tcgen05.mma kind::i8 -> TMEM -> tcgen05.ld path.
// grid (nqt, nkt), 128 threads; each CTA computes one 128x128 tile of S_int = Q_i8 K_i8^T.
// ------------------------------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(128, 1)
    qk_int32_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    int32_t* __restrict__ s_out, int bh, int bg, int qt0, int kt0, int ldo) {
  using Cfg = AttnCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sq = smem;
  uint8_t* sk = smem + Cfg::kQTile;
  uint64_t* bar_ld = reinterpret_cast<uint64_t*>(smem + Cfg::kQTile + Cfg::kKTile);
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
    tmem_alloc(tbase, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tbase;
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(bar_ld, Cfg::kQTile + Cfg::kKTile);
    tma_load_3d(sq, &tm_q, bar_ld, 0, qt * kBM, bh);
    tma_load_3d(sk, &tm_k, bar_ld, 0, kt * kBN, bg);
    if (mbar_wait(bar_ld, 0, abort)) {
      tc_fence_after();
      constexpr uint32_t idq = idesc_i8_s32(kBM, kBN);
#pragma unroll
      for (int kk = 0; kk < D / 32; ++kk) {
        const uint64_t ad = smem_desc(smem_u32(sq) + kk * 32, 16, Cfg::kSboQK, Cfg::kSwQK);
        const uint64_t bd = smem_desc(smem_u32(sk) + kk * 32, 16, Cfg::kSboQK, Cfg::kSwQK);
        mma_i8_ss(tmem, ad, bd, idq, kk > 0 ? 1u : 0u);
      }
      mma_commit(bar_mma);
    }
  }
  __syncwarp();
  const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait(bar_mma, 0, abort));
  tc_fence_after();
  if (ok) {
    const int row = warp * 32 + lane;
    int32_t* orow = s_out + static_cast<size_t>(blockIdx.x * kBM + row) * ldo + blockIdx.y * kBN;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint32_t r[32];
      tmem_ld32(tmem + (static_cast<uint32_t>(warp * 32) << 16) + c * 32, r);
      tmem_ld_wait(r);
#pragma unroll
      for (int v = 0; v < 8; ++v)
        reinterpret_cast<uint4*>(orow + c * 32)[v] = make_uint4(r[4 * v], r[4 * v + 1], r[4 * v + 2], r[4 * v + 3]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

}  // namespace qattn
