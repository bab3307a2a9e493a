// attn_sm100.cuh -- smoothed-K INT8 attention forward for B200 (sm_100a).
//
// Method (SageAttention summary page, aibr.jp/archives/102657): INT8 Q K^T with exact 32-bit
// accumulation (sec. 3, mma(u8.u8.s32)), FP16 operands for P V (sec. 2-3, mma(f16.f16.f16)),
// FlashAttention-style blockwise online softmax (sec. 4).  The page's kernel is written for
// warp-level mma on an RTX4090; this one is built for Blackwell instead:
//
//  * one CTA owns two 128-row Q tiles of one (batch, head) and streams 128-key K/V tiles;
//  * warp 16 (TMA): loads both Q tiles once, then K (int8) and V (fp16) tiles into a STAGES-deep
//    shared-memory ring (128-byte / 64-byte swizzled tiles, mbarrier transaction counts);
//  * warp 17 (MMA, one thread): S_w = Q_w K^T as tcgen05.mma kind::i8 (M=128, N=128, K=32 per
//    instruction) into tensor memory, then O_w += P_w V as tcgen05.mma kind::f16 with P read
//    from tensor memory (M=128, N=d, K=16), fp32 accumulator in tensor memory;
//  * warps 0-15 (softmax, four warpgroups, two per Q tile): each score row is shared by two
//    threads, one per 64-key half (= one K scale block); tcgen05.ld of the int32 scores,
//    dequantization with the block scales, half-row maxima swapped through shared memory,
//    running max / sum in registers, exp2, P written back as fp16 into the same tensor-memory
//    columns (aliasing S), lazy rescaling of O only when the running max grows by more than 2^8,
//    P scaled into the top of the fp16 range;
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
constexpr int kAttnThreads = 640;     // 5 warpgroups: 4 softmax (2 per Q tile), TMA + MMA
constexpr int kAttnLaunchRegs = 96;    // 640 x 96 = 512 x 104 (softmax) + 128 x 64 (setmaxnreg)
constexpr int kSoftmaxThreads = 512;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: O is rescaled only when the max grows more
// P = 2^(x - m + kPOffset): with the lazy max above, P <= 2^15 < 65504 (fp16 max), and keys down to
// about 2^-(24 + kPOffset) of the row maximum still reach the fp16 P instead of underflowing.  At
// 131072 keys per row, P normalised to 1 loses enough weight in fp16 subnormals to cost ~4e-3 of
// output accuracy; the offset cancels in O / l.
constexpr float kPOffset = 7.0f;

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
  static constexpr int kBarBytes = 256 + 4096;  // barriers + half-row max / sum exchange
  static constexpr int kSmemBytes = kOffBar + kBarBytes + 1024;  // + alignment slack
  // K-major int8 operands: rows of D bytes, 8-row swizzle atoms.
  static constexpr uint32_t kSwQK = D == 128 ? kSwizzle128B : kSwizzle64B;
  static constexpr uint32_t kSboQK = 8 * D;
  // V: MN-major fp16 operand, 64-column (128-byte) swizzled boxes of 128 rows.
  static constexpr uint32_t kVBox = kBN * 128;  // bytes of one 64-column box
};

struct __align__(16) AttnBars {
  uint64_t q_full;
  uint64_t kv_full[6];
  uint64_t kv_empty[6];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t pv_done[2];
  uint32_t tmem_base;
  int abort;
  uint8_t pad[256 - 8 * 19 - 8];
  // [step parity][Q tile][key half][row]: the two threads of a score row swap half-row maxima
  // (and, at the end, half-row sums) here
  float xch[2][2][2][128];
};
static_assert(sizeof(AttnBars) <= 256 + 4096, "barrier block");

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

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// One thread's 64 scores of a row (one K scale block), in registers as floats (exact:
// |S_int| < 2^24); keys with offset above lim are set to -inf.  Returns their maximum.
template <bool MASK>
__device__ __forceinline__ float half_row_to_float_max(uint32_t (&s)[2][32], int lim) {
  float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
  for (int c = 0; c < 2; ++c) {
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      float x = static_cast<float>(static_cast<int>(s[c][e]));
      if (MASK && c * 32 + e > lim) x = -INFINITY;
      s[c][e] = __float_as_uint(x);
    }
#pragma unroll
    for (int e = 0; e < 32; e += 4) {
      m0 = fmax3(m0, __uint_as_float(s[c][e]), __uint_as_float(s[c][e + 1]));
      m1 = fmax3(m1, __uint_as_float(s[c][e + 2]), __uint_as_float(s[c][e + 3]));
    }
  }
  return fmaxf(m0, m1);
}

// p = 2^(x * c - m) for the thread's 64 keys, masked keys (x = -inf) give 0.  P is packed as
// fp16 pairs (even key in the low half) and stored into 32 tensor-memory columns at p_tm.
// Returns the fp32 sum of the fp16-rounded p.
template <bool MASK>
__device__ __forceinline__ float half_row_exp_store(const uint32_t (&s)[2][32], float c,
                                                    float neg_m, uint32_t p_tm) {
  float acc0 = 0.0f, acc1 = 0.0f;
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    uint32_t pk[16];
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
      const float x0 = __uint_as_float(s[k][e]);
      const float x1 = __uint_as_float(s[k][e + 1]);
      float y0, y1;
      ffma2(y0, y1, x0, x1, c, neg_m);
      float p0 = ex2_approx(y0);
      float p1 = ex2_approx(y1);
      if (MASK) {
        // -inf * 0 would be NaN for a zero-scale block: select instead
        p0 = x0 == -INFINITY ? 0.0f : p0;
        p1 = x1 == -INFINITY ? 0.0f : p1;
      }
      const uint32_t h2 = pack_half2(p0, p1);
      pk[e >> 1] = h2;
      // the row sum takes the fp16-rounded P that the P V product uses, so that O / l is a
      // weighted mean of V with exactly those weights
      if ((e >> 1) & 1) acc1 = add_half2_f32(acc1, h2);
      else acc0 = add_half2_f32(acc0, h2);
    }
    tmem_st16(p_tm + k * 16, pk);
  }
  return acc0 + acc1;
}

__device__ __forceinline__ void setmaxnreg_inc104() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 104;" ::: "memory");
}
__device__ __forceinline__ void setmaxnreg_dec64() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 64;" ::: "memory");
}

template <int D, bool CAUSAL>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const float* __restrict__ q_scale,
                    const float* __restrict__ k_scale, __half* __restrict__ out, int B, int H,
                    int Hkv, int N, float scale_log2) {
  using Cfg = AttnCfg<D>;
  constexpr int ST = Cfg::kStages;
  constexpr int kTmaWarp = kSoftmaxThreads / 32;  // warp 16
  constexpr int kMmaWarp = kTmaWarp + 1;          // warp 17
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
      mbar_init(&bars->p_full[w], 256);
      mbar_init(&bars->pv_done[w], 1);
    }
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp >= kTmaWarp) {
    // warpgroup 4 (TMA warp, MMA warp, two idle warps) hands registers to the softmax groups
    setmaxnreg_dec64();
    if (warp == kTmaWarp && lane == 0) {
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
    } else if (warp == kMmaWarp && lane == 0) {
      // ---------------------------------------------------------------- MMA issuer
      // Order per key tile j: PV_0(j), QK_0(j+1), PV_1(j), QK_1(j+1).  tcgen05.mma operations
      // from one thread execute in issue order, so QK_w(j+1) may be issued right behind PV_w(j)
      // although it overwrites the tensor-memory columns PV_w(j) reads P_w from; the softmax of
      // one Q tile then overlaps the other tile's PV + QK^T on the tensor pipe.
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
    // warp = 8 * tile + 4 * half + lane group: two threads share each score row, one per
    // 64-key half (= one K scale block); they swap half-row maxima through shared memory.
    setmaxnreg_inc104();
    const int wt = warp >> 3;
    const int half = (warp >> 2) & 1;
    const int lg = warp & 3;
    const int row = lg * 32 + lane;
    const int pair_bar = 1 + wt * 4 + lg;  // named barrier of the two warps sharing these rows
    const int nt = wt == 0 ? nw0 : nw1;
    if (nt > 0) {
      const int t = wt == 0 ? tq0 : tq1;
      const int qrow = t * kBM + row;
      const float sq = __ldg(q_scale + static_cast<size_t>(bh) * nqt + t);
      const float* ksc = k_scale + static_cast<size_t>(bg) * nkb;
      const uint32_t lane_off = static_cast<uint32_t>(lg * 32) << 16;
      const uint32_t s_tm = tmem + lane_off + wt * 128 + half * 64;
      const uint32_t p_tm = tmem + lane_off + wt * 128 + half * 32;
      const uint32_t o_tm = tmem + lane_off + 256 + wt * D + half * (D / 2);
      float m_used = -INFINITY;
      float l = 0.0f;
      bool ok = true;
      float ks = (half < nkb) ? __ldg(ksc + half) : 0.0f;
      for (int j = 0; j < nt; ++j) {
        const int kb_next = 2 * j + 2 + half;
        const float ks_next = kb_next < nkb ? __ldg(ksc + kb_next) : 0.0f;
        ok = __all_sync(0xFFFFFFFFu, mbar_wait(&bars->s_full[wt], static_cast<uint32_t>(j) & 1u, abort));
        if (!ok) break;
        tc_fence_after();
        uint32_t sr[2][32];
        tmem_ld32(s_tm, sr[0]);
        tmem_ld32(s_tm + 32, sr[1]);
        tmem_ld_wait(sr[0]);
        tmem_ld_wait(sr[1]);
        int lim = N - 1 - j * kBN - half * 64;
        if (CAUSAL && j == t) lim = min(lim, row - half * 64);
        const float c = sq * ks * scale_log2;
        ks = ks_next;
        // warp-uniform, so that every lane runs the same tensor-memory access sequence
        const bool masked = __any_sync(0xFFFFFFFFu, lim < 63);
        float hm = masked ? half_row_to_float_max<true>(sr, lim) : half_row_to_float_max<false>(sr, lim);
        hm = hm == -INFINITY ? -INFINITY : hm * c;
        // swap half-row maxima; the barrier also orders this thread's score reads before the
        // partner's P writes, which land on columns 32-63 of the row
        bars->xch[j & 1][wt][half][row] = hm;
        tc_fence_before();
        named_bar_sync(pair_bar, 64);
        tc_fence_after();
        const float mt = fmaxf(hm, bars->xch[j & 1][wt][half ^ 1][row]);
        const float m_new = fmaxf(m_used, mt);
        const bool need = m_new > m_used + kRescaleThreshold;
        float alpha = 1.0f;
        if (need) {
          alpha = j == 0 ? 0.0f : ex2_approx(m_used - m_new);
          m_used = m_new;
          l *= alpha;
        }
        const float neg_m = kPOffset - m_used;
        const float psum = masked ? half_row_exp_store<true>(sr, c, neg_m, p_tm)
                                  : half_row_exp_store<false>(sr, c, neg_m, p_tm);
        l += psum;
        if (j > 0 && __any_sync(0xFFFFFFFFu, need)) {
          // O holds PV up to tile j-1 (complete: QK(j) was issued after PV(j-1)), and PV(j)
          // waits for this group's arrive below.  Both threads of a row take the same decision;
          // each rescales its half of the O row.
#pragma unroll
          for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t o[16];
            tmem_ld16(o_tm + cc * 16, o);
            tmem_ld_wait(o);
#pragma unroll
            for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tmem_st16(o_tm + cc * 16, o);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&bars->p_full[wt]);
      }
      if (ok) ok = mbar_wait(&bars->pv_done[wt], static_cast<uint32_t>(nt - 1) & 1u, abort);
      ok = __all_sync(0xFFFFFFFFu, ok);
      // total row sum from the two halves (parity slot nt&1 is free: last used at step nt-2)
      bars->xch[nt & 1][wt][half][row] = l;
      named_bar_sync(pair_bar, 64);
      l += bars->xch[nt & 1][wt][half ^ 1][row];
      tc_fence_after();
      if (ok) {
        const float inv_l = 1.0f / l;
        __half* orow = out + (static_cast<size_t>(bh) * N + qrow) * D + half * (D / 2);
#pragma unroll
        for (int cc = 0; cc < D / 64; ++cc) {
          uint32_t o[32];
          tmem_ld32(o_tm + cc * 32, o);
          tmem_ld_wait(o);
          if (qrow < N) {
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
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
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
