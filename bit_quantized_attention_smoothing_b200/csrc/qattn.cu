// qattn.cu -- the C ABI declared in include/qattn.h: argument checks, TMA tensor maps, workspace
// management and kernel launches for the smoothed-K INT8 attention forward on B200 (sm_100a).
// One translation unit: the kernels live in the included .cuh files.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <map>
#include <mutex>

#include "qattn.h"
#include "attn_sm100.cuh"
#include "quant.cuh"
#include "block_sparse.cuh"
#include "nvfp4.cuh"
#include "fp4_sm100.cuh"
#include "adaptive.cuh"

namespace {

using namespace qattn;

constexpr int kMaxN = 1 << 20;
constexpr size_t kAlign = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

qattn_status check_shape(int B, int H, int Hkv, int N, int d) {
  if (B < 1 || H < 1 || Hkv < 1 || N < 1) return QATTN_ERR_INVALID_ARG;
  if (H % Hkv != 0) return QATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return QATTN_ERR_UNSUPPORTED;
  if (N > kMaxN) return QATTN_ERR_UNSUPPORTED;
  // grid-size and 32-bit index limits of the kernels
  if (static_cast<long long>(B) * H > (1 << 20)) return QATTN_ERR_UNSUPPORTED;
  return QATTN_OK;
}

template <typename... P>
qattn_status check_ptrs(P... ptrs) {
  const void* arr[] = {static_cast<const void*>(ptrs)...};
  for (const void* p : arr)
    if (p == nullptr) return QATTN_ERR_INVALID_ARG;
  for (const void* p : arr)
    if (!aligned16(p)) return QATTN_ERR_MISALIGNED;
  return QATTN_OK;
}

qattn_status device_ok() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return QATTN_ERR_CUDA;
  int major = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return QATTN_ERR_CUDA;
  if (major != 10) return QATTN_ERR_UNSUPPORTED;
  return QATTN_OK;
}

qattn_status launch_status() {
  return cudaGetLastError() == cudaSuccess ? QATTN_OK : QATTN_ERR_CUDA;
}

// ---------------------------------------------------------------------------------------------
// Tensor maps (driver entry point fetched through the runtime, so no link against libcuda)
// ---------------------------------------------------------------------------------------------

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 3-D map over a contiguous [dim2][dim1][dim0] tensor with a (box0 x box1 x 1) box.
bool make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int elem_bytes,
              uint64_t dim0, uint64_t dim1, uint64_t dim2, uint32_t box0, uint32_t box1,
              CUtensorMapSwizzle sw) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {dim0, dim1, dim2};
  cuuint64_t strides[2] = {dim0 * elem_bytes, dim0 * dim1 * elem_bytes};
  cuuint32_t box[3] = {box0, box1, 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = fn(m, dt, 3, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// int8 [rows_outer][N][d] tiles of 128 rows x d bytes, swizzled to match the MMA descriptors.
bool make_i8_map(CUtensorMap* m, const void* base, int d, int N, long long outer) {
  return make_map(m, base, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, d, N, outer, d, 128,
                  d == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B);
}

// NVFP4 codes [outer][N][d/2] bytes: tiles of 128 rows x d/2 bytes, swizzled to match the
// FP4 MMA descriptors (64-byte rows for d = 128, 32-byte rows for d = 64).
bool make_fp4_map(CUtensorMap* m, const void* base, int d, int N, long long outer) {
  return make_map(m, base, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, d / 2, N, outer, d / 2, 128,
                  d == 128 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
}

// NVFP4 V^T codes [outer][d][Np/2] bytes: tiles of d channel rows x 64 bytes (128 keys).
bool make_fp4_vt_map(CUtensorMap* m, const void* base, int d, int Np, long long outer) {
  return make_map(m, base, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, Np / 2, d, outer, 64, d,
                  CU_TENSOR_MAP_SWIZZLE_64B);
}

template <int D, bool CAUSAL>
qattn_status launch_attn_nvfp4(const CUtensorMap* maps, const uint8_t* q_sf, const uint8_t* k_sf,
                               const uint8_t* vt_sf, const float* q_g, const float* k_g,
                               const float* v_g, const void* q16, const float* k_mean,
                               const int* kv_list, const int* kv_count, void* out, int B, int H,
                               int Hkv, int N, int Np, cudaStream_t st) {
  // One CTA per SM (its 512 tensor-memory columns); at d = 128 the double-buffered FP4 and fp16
  // K/V tiles take ~211 KB of shared memory.
  const int smem = Fp4AttnCfg<D>::kSmemUsed;
  static_assert(Fp4AttnCfg<D>::kSmemUsed <= 227 * 1024, "shared memory");
  auto kern = attn_nvfp4_kernel<D, CAUSAL>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return QATTN_ERR_CUDA;
  const dim3 grid((N + 127) / 128, B * H);
  const float sl2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(D)));
  kern<<<grid, kFp4Threads, smem, st>>>(maps[0], maps[1], maps[2], maps[3], maps[4], maps[5], q_sf, k_sf,
                                vt_sf, q_g, k_g, v_g, static_cast<const uint16_t*>(q16), k_mean,
                                kv_list, kv_count, static_cast<__half*>(out), H, Hkv, N, Np, sl2);
  return launch_status();
}

// fp16 V [outer][N][d]: boxes of 64 columns (128 bytes) x 128 rows, 128-byte swizzle.
bool make_v_map(CUtensorMap* m, const void* base, int d, int N, long long outer) {
  return make_map(m, base, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, d, N, outer, 64, 128,
                  CU_TENSOR_MAP_SWIZZLE_128B);
}

// E4M3 V^T [outer][d][Np] bytes: tiles of d channel rows x 128 keys, 128-byte swizzle.
bool make_v8_map(CUtensorMap* m, const void* base, int d, int Np, long long outer) {
  return make_map(m, base, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, Np, d, outer, 128, d,
                  CU_TENSOR_MAP_SWIZZLE_128B);
}

// ---------------------------------------------------------------------------------------------
// Launchers
// ---------------------------------------------------------------------------------------------

struct QuantLayout {
  int nqb, nkb;
  size_t q_i8, k_i8, q_scale, k_scale, sums, total;
};

QuantLayout forward_layout(int B, int H, int Hkv, int N, int d) {
  QuantLayout L;
  L.nqb = (N + kQBlock - 1) / kQBlock;
  L.nkb = (N + kKBlock - 1) / kKBlock;
  size_t off = 0;
  L.q_i8 = off;
  off = align_up(off + static_cast<size_t>(B) * H * N * d);
  L.k_i8 = off;
  off = align_up(off + static_cast<size_t>(B) * Hkv * N * d);
  L.q_scale = off;
  off = align_up(off + sizeof(float) * B * H * L.nqb);
  L.k_scale = off;
  off = align_up(off + sizeof(float) * B * Hkv * L.nkb);
  L.sums = off;
  off = align_up(off + sizeof(long long) * B * Hkv * d);
  L.total = off;
  return L;
}

// Two launches.  With q: Q's quantization together with the K channel sums (the K-sum CTAs last,
// so that K is still in L2), then the K quantization.  Without q (the fused forward quantizes Q
// inside the attention kernel): the channel sums, then the K quantization.
template <int D>
qattn_status run_smooth_quant(const void* q, const void* k, int B, int H, int Hkv, int N,
                              int8_t* q_i8, float* q_scale, int8_t* k_i8, float* k_scale,
                              float* k_mean, long long* sums, cudaStream_t st) {
  const int nqb = (N + kQBlock - 1) / kQBlock;
  const int nkb = (N + kKBlock - 1) / kKBlock;
  const int nchunk = (N + kSumRowsPerCta - 1) / kSumRowsPerCta;
  const long long nq = q ? static_cast<long long>(B) * H * nqb : 0;
  const long long nsum = static_cast<long long>(B) * Hkv * nchunk;
  const long long nk = static_cast<long long>(B) * Hkv * nkb;
  if (nq + nsum > 0x7FFFFFFFLL || nk > 0x7FFFFFFFLL) return QATTN_ERR_UNSUPPORTED;
  if (cudaMemsetAsync(sums, 0, sizeof(long long) * B * Hkv * D, st) != cudaSuccess)
    return QATTN_ERR_CUDA;
  if (q) {
    q_quant_k_sums_kernel<D><<<static_cast<unsigned>(nq + nsum), 256, 0, st>>>(
        static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(k), N, nqb, nq, nchunk, q_i8,
        q_scale, sums);
  } else {
    dim3 g1(B * Hkv, nchunk);
    k_channel_sums_kernel<D><<<g1, 256, 0, st>>>(static_cast<const uint16_t*>(k), N, sums);
  }
  if (launch_status() != QATTN_OK) return QATTN_ERR_CUDA;
  k_quantize_kernel<D><<<static_cast<unsigned>(nk), 256, 0, st>>>(
      static_cast<const uint16_t*>(k), N, nkb, sums, k_i8, k_scale, k_mean);
  return launch_status();
}

// q is int8 (with q_scale) or, for QF16, the fp16 Q that the kernel quantizes itself.  MODE
// kDumpS: the score-dumping instantiation, one CTA per Q-tile pair dump->pair0 .. of head
// dump->bh; kOutF32: out is fp32.
// The E4M3 operands of the FP8 P V variant (PVK kPvF8 or kPvTable): V^T codes, per-group scales and,
// for kPvTable, the per-group variant table.
struct Pv8Args {
  const uint8_t* vt8 = nullptr;
  const float* v_scale = nullptr;
  const uint8_t* variant = nullptr;
};

template <int D, bool CAUSAL, bool QF16, int MODE = kOutF16, int PVK = kPvF16>
qattn_status run_attn(const void* q, const float* q_scale, const int8_t* k_i8,
                      const float* k_scale, const void* v, void* out, int B, int H, int Hkv,
                      int N, cudaStream_t st, const int* kv_list = nullptr,
                      const int* kv_count = nullptr, const ScoreDump* dump = nullptr,
                      int dump_pairs = 0, Pv8Args pv = Pv8Args()) {
  CUtensorMap tq, tk, tv, tv8;
  std::memset(&tq, 0, sizeof(tq));  // unused by the QF16 kernel
  if ((!QF16 && !make_i8_map(&tq, q, D, N, static_cast<long long>(B) * H)) ||
      !make_i8_map(&tk, k_i8, D, N, static_cast<long long>(B) * Hkv) ||
      (v != nullptr && !make_v_map(&tv, v, D, N, static_cast<long long>(B) * Hkv)))
    return QATTN_ERR_CUDA;
  if (PVK != kPvF16) {
    if (!make_v8_map(&tv8, pv.vt8, D, (N + 127) / 128 * 128, static_cast<long long>(B) * Hkv))
      return QATTN_ERR_CUDA;
    if (v == nullptr) tv = tv8;  // every group on the FP8 path: the fp16 map is never read
  } else {
    tv8 = tv;  // never read
  }
  using Cfg = AttnCfg<D>;
  constexpr bool DUMP = MODE == kDumpS;
  auto kern = attn_fwd_kernel<D, CAUSAL, QF16, MODE, PVK>;
  // The kernel moves registers between its warpgroups with setmaxnreg; the split adds up only if
  // the launch allocates exactly kAttnLaunchRegs per thread, so never launch it otherwise.
  static int regs_checked = 0;
  if (regs_checked == 0) {
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return QATTN_ERR_CUDA;
    regs_checked = fa.numRegs == kAttnLaunchRegs ? 1 : -1;
  }
  if (regs_checked != 1) return QATTN_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmemBytes) !=
      cudaSuccess)
    return QATTN_ERR_CUDA;
  const int nqt = (N + kBM - 1) / kBM;
  const long long grid = DUMP ? dump_pairs : static_cast<long long>(B) * H * ((nqt + 1) / 2);
  if (grid > 0x7FFFFFFFLL) return QATTN_ERR_UNSUPPORTED;
  const float scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(D)));
  kern<<<static_cast<unsigned>(grid), kAttnThreads, Cfg::kSmemBytes, st>>>(
      tq, tk, tv, tv8, q_scale, QF16 ? static_cast<const uint16_t*>(q) : nullptr, kv_list, kv_count,
      k_scale, pv.v_scale, pv.variant, out, B, H, Hkv, N, scale_log2, dump ? *dump : ScoreDump{});
  return launch_status();
}

template <bool QF16, int MODE = kOutF16>
qattn_status dispatch_attn(const void* q, const float* q_scale, const int8_t* k_i8,
                           const float* k_scale, const void* v, void* out, int B, int H, int Hkv,
                           int N, int d, int causal, cudaStream_t st, const int* kv_list = nullptr,
                           const int* kv_count = nullptr) {
  if (d == 128)
    return causal ? run_attn<128, true, QF16, MODE>(q, q_scale, k_i8, k_scale, v, out, B, H, Hkv, N, st, kv_list, kv_count)
                  : run_attn<128, false, QF16, MODE>(q, q_scale, k_i8, k_scale, v, out, B, H, Hkv, N, st, kv_list, kv_count);
  return causal ? run_attn<64, true, QF16, MODE>(q, q_scale, k_i8, k_scale, v, out, B, H, Hkv, N, st, kv_list, kv_count)
                : run_attn<64, false, QF16, MODE>(q, q_scale, k_i8, k_scale, v, out, B, H, Hkv, N, st, kv_list, kv_count);
}

// The attention on int8 Q and K with the FP8 P V variant for every group (PVK kPvF8) or per group
// (kPvTable; v is the fp16 V for the groups on the FP16 path).
template <int PVK>
qattn_status dispatch_attn_pv8(const int8_t* q_i8, const float* q_scale, const int8_t* k_i8,
                               const float* k_scale, const void* v, Pv8Args pv, void* out, int B,
                               int H, int Hkv, int N, int d, int causal, cudaStream_t st) {
#define QATTN_PV_ARGS q_i8, q_scale, k_i8, k_scale, v, out, B, H, Hkv, N, st, nullptr, nullptr, nullptr, 0, pv
  if (d == 128)
    return causal ? run_attn<128, true, false, kOutF16, PVK>(QATTN_PV_ARGS)
                  : run_attn<128, false, false, kOutF16, PVK>(QATTN_PV_ARGS);
  return causal ? run_attn<64, true, false, kOutF16, PVK>(QATTN_PV_ARGS)
                : run_attn<64, false, false, kOutF16, PVK>(QATTN_PV_ARGS);
#undef QATTN_PV_ARGS
}

// E4M3 V: slice maxima, scales, transposed codes (arguments already checked).
qattn_status dispatch_quant_v_fp8(const void* v, int S, int R, int C, uint8_t* vt8, float* scale,
                                  cudaStream_t st) {
  const uint16_t* vh = static_cast<const uint16_t*>(v);
  if (cudaMemsetAsync(scale, 0, sizeof(float) * static_cast<size_t>(S), st) != cudaSuccess)
    return QATTN_ERR_CUDA;
  const long long nvec = static_cast<long long>(R) * C / 8;
  long long gx = (nvec + 1023) / 1024;
  const long long cap = (148LL * 16 + S - 1) / S;
  if (gx > cap) gx = cap;
  if (gx < 1) gx = 1;
  nvfp4_amax_kernel<<<dim3(static_cast<unsigned>(gx), S), 256, 0, st>>>(
      vh, nullptr, R, C, reinterpret_cast<unsigned*>(scale));
  if (launch_status() != QATTN_OK) return QATTN_ERR_CUDA;
  v_fp8_scale_kernel<<<(S + 255) / 256, 256, 0, st>>>(scale, S);
  if (launch_status() != QATTN_OK) return QATTN_ERR_CUDA;
  const int Rp = (R + 127) / 128 * 128;
  const dim3 grid(Rp / kV8Tile, (C + kV8Tile - 1) / kV8Tile, S);
  v_fp8_quant_kernel<<<grid, 256, 0, st>>>(vh, R, C, Rp, scale, vt8);
  return launch_status();
}

// Block selection workspace: query-block means, key-tile means, scores (binary64).
struct SelLayout {
  int nsb, nkt;
  size_t qmeans, kmeans, scores, total;
};

SelLayout sel_layout(int B, int H, int Hkv, int N, int d) {
  SelLayout L;
  L.nsb = (N + kSelQRows - 1) / kSelQRows;
  L.nkt = (N + kSelKRows - 1) / kSelKRows;
  size_t off = 0;
  L.qmeans = off;
  off = align_up(off + sizeof(double) * B * H * L.nsb * d);
  L.kmeans = off;
  off = align_up(off + sizeof(double) * B * Hkv * L.nkt * d);
  L.scores = off;
  off = align_up(off + sizeof(double) * B * H * static_cast<size_t>(L.nsb) * L.nkt);
  L.total = off;
  return L;
}

template <int D>
qattn_status run_block_select(const void* q, const void* k, int B, int H, int Hkv, int N,
                              int causal, int topk, int* list, int* count, uint8_t* ws,
                              cudaStream_t st) {
  const SelLayout L = sel_layout(B, H, Hkv, N, D);
  double* qm = reinterpret_cast<double*>(ws + L.qmeans);
  double* km = reinterpret_cast<double*>(ws + L.kmeans);
  double* sc = reinterpret_cast<double*>(ws + L.scores);
  if (static_cast<long long>(B) * H > 65535 * 1024LL) return QATTN_ERR_UNSUPPORTED;
  block_means_kernel<D><<<dim3(B * H, L.nsb), 256, 0, st>>>(static_cast<const uint16_t*>(q), N,
                                                           kSelQRows, qm);
  block_means_kernel<D><<<dim3(B * Hkv, L.nkt), 256, 0, st>>>(static_cast<const uint16_t*>(k), N,
                                                             kSelKRows, km);
  if (launch_status() != QATTN_OK) return QATTN_ERR_CUDA;
  if (B * H > 65535) return QATTN_ERR_UNSUPPORTED;
  dim3 gs((L.nkt + kScoreTile - 1) / kScoreTile, (L.nsb + kScoreTile - 1) / kScoreTile, B * H);
  block_scores_kernel<D><<<gs, 256, 0, st>>>(qm, km, H, Hkv, L.nsb, L.nkt, causal, sc);
  if (launch_status() != QATTN_OK) return QATTN_ERR_CUDA;
  block_select_kernel<<<dim3((L.nsb + 7) / 8, B * H), 256, 0, st>>>(sc, L.nsb, L.nkt, causal,
                                                                    topk, list, count);
  return launch_status();
}

qattn_status dispatch_smooth_quant(const void* q, const void* k, int B, int H, int Hkv, int N,
                                   int d, int8_t* q_i8, float* q_scale, int8_t* k_i8,
                                   float* k_scale, float* k_mean, long long* sums,
                                   cudaStream_t st) {
  if (d == 128)
    return run_smooth_quant<128>(q, k, B, H, Hkv, N, q_i8, q_scale, k_i8, k_scale, k_mean, sums,
                                 st);
  return run_smooth_quant<64>(q, k, B, H, Hkv, N, q_i8, q_scale, k_i8, k_scale, k_mean, sums, st);
}

// NVFP4 quantization launches (arguments already checked): zeroed slice maxima, maxima,
// quantization along the channels or transposed along the rows, slice scales.
qattn_status dispatch_quant_nvfp4(const void* x, const float* mean, int S, int R, int C,
                                  int along_rows, uint8_t* codes, uint8_t* scales, float* gscale,
                                  cudaStream_t st) {
  const uint16_t* xh = static_cast<const uint16_t*>(x);
  unsigned* amax_bits = reinterpret_cast<unsigned*>(gscale);
  if (cudaMemsetAsync(gscale, 0, sizeof(float) * static_cast<size_t>(S), st) != cudaSuccess)
    return QATTN_ERR_CUDA;
  // slice maxima: about 16 resident CTAs per SM over all slices, at least 4 vectors a thread
  const long long nvec = static_cast<long long>(R) * C / 8;
  long long gx = (nvec + 1023) / 1024;
  const long long cap = (148LL * 16 + S - 1) / S;
  if (gx > cap) gx = cap;
  if (gx < 1) gx = 1;
  nvfp4_amax_kernel<<<dim3(static_cast<unsigned>(gx), S), 256, 0, st>>>(xh, mean, R, C, amax_bits);
  if (launch_status() != QATTN_OK) return QATTN_ERR_CUDA;
  if (along_rows) {
    const int Rp = (R + 127) / 128 * 128;
    const dim3 grid((Rp + kNvfp4Tile - 1) / kNvfp4Tile, (C + kNvfp4Tile - 1) / kNvfp4Tile, S);
    nvfp4_quant_cols_kernel<<<grid, 256, 0, st>>>(xh, mean, R, C, Rp, amax_bits, codes, scales);
  } else {
    const long long total = static_cast<long long>(S) * R * (C / 16);
    long long blocks = (total + 255) / 256;
    if (blocks > 148LL * 32) blocks = 148LL * 32;
    nvfp4_quant_rows_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(xh, mean, R, C, total,
                                                                          amax_bits, codes, scales);
  }
  if (launch_status() != QATTN_OK) return QATTN_ERR_CUDA;
  nvfp4_finalize_kernel<<<(S + 255) / 256, 256, 0, st>>>(gscale, S);
  return launch_status();
}

// FP4-path attention launch (arguments already checked).
qattn_status dispatch_attn_nvfp4(const uint8_t* q_codes, const uint8_t* q_scales, const float* q_g,
                                 const uint8_t* k_codes, const uint8_t* k_scales, const float* k_g,
                                 const uint8_t* vt_codes, const uint8_t* vt_scales,
                                 const float* v_g, const void* q, const void* k, const void* v,
                                 const float* k_mean, const int* kv_list, const int* kv_count,
                                 void* out, int B, int H, int Hkv, int N, int d, int causal,
                                 cudaStream_t st) {
  const int Np = (N + 127) / 128 * 128;
  CUtensorMap maps[6];
  if (!make_fp4_map(&maps[0], q_codes, d, N, static_cast<long long>(B) * H) ||
      !make_fp4_map(&maps[1], k_codes, d, N, static_cast<long long>(B) * Hkv) ||
      !make_fp4_vt_map(&maps[2], vt_codes, d, Np, static_cast<long long>(B) * Hkv))
    return QATTN_ERR_CUDA;
  if (kv_list != nullptr) {
    // fp16 Q, K, V tiles: boxes of 64 columns x 128 rows, 128-byte swizzle
    if (!make_v_map(&maps[3], q, d, N, static_cast<long long>(B) * H) ||
        !make_v_map(&maps[4], k, d, N, static_cast<long long>(B) * Hkv) ||
        !make_v_map(&maps[5], v, d, N, static_cast<long long>(B) * Hkv))
      return QATTN_ERR_CUDA;
  } else {
    maps[3] = maps[4] = maps[5] = maps[0];  // never read without promotion
  }
  const uint16_t* q16 = static_cast<const uint16_t*>(q);
#define QATTN_FP4_ARGS maps, q_scales, k_scales, vt_scales, q_g, k_g, v_g, q16, k_mean, kv_list, \
                       kv_count, out, B, H, Hkv, N, Np, st
  if (d == 128)
    return causal ? launch_attn_nvfp4<128, true>(QATTN_FP4_ARGS)
                  : launch_attn_nvfp4<128, false>(QATTN_FP4_ARGS);
  return causal ? launch_attn_nvfp4<64, true>(QATTN_FP4_ARGS)
                : launch_attn_nvfp4<64, false>(QATTN_FP4_ARGS);
#undef QATTN_FP4_ARGS
}

// ---------------------------------------------------------------------------------------------
// Per-device memory pools for the allocating entry points
// ---------------------------------------------------------------------------------------------

std::mutex g_pool_mu;
std::map<int, cudaMemPool_t> g_pools;

qattn_status get_pool(cudaMemPool_t* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return QATTN_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_pool_mu);
  auto it = g_pools.find(dev);
  if (it != g_pools.end()) {
    *out = it->second;
    return QATTN_OK;
  }
  cudaMemPoolProps props;
  std::memset(&props, 0, sizeof(props));
  props.allocType = cudaMemAllocationTypePinned;
  props.handleTypes = cudaMemHandleTypeNone;
  props.location.type = cudaMemLocationTypeDevice;
  props.location.id = dev;
  cudaMemPool_t pool;
  if (cudaMemPoolCreate(&pool, &props) != cudaSuccess) return QATTN_ERR_CUDA;
  uint64_t keep = UINT64_MAX;  // keep freed blocks cached for reuse
  cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
  g_pools[dev] = pool;
  *out = pool;
  return QATTN_OK;
}

qattn_status pool_alloc(void** p, size_t bytes, cudaStream_t st) {
  cudaMemPool_t pool;
  qattn_status s = get_pool(&pool);
  if (s != QATTN_OK) return s;
  return cudaMallocFromPoolAsync(p, bytes, pool, st) == cudaSuccess ? QATTN_OK : QATTN_ERR_CUDA;
}

// ---------------------------------------------------------------------------------------------
// Fixed scratch for the allocation-free smoothing + quantization entry point
// ---------------------------------------------------------------------------------------------

// Exact int64 channel sums of K for qattn_smooth_quant_noalloc: room for B * Hkv * d <= 65536
// (512 KiB), held by every GPU that loads the library until the process exits.
constexpr size_t kNoAllocMaxSums = 65536;
static __device__ __align__(256) long long g_noalloc_sums[kNoAllocMaxSums];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
long long* g_noalloc_ptr[kMaxDevices] = {};

// Device address of g_noalloc_sums on the current device.  Host code cannot pass the symbol itself
// (on the host it names a stand-in, not device memory), so the address is looked up once per
// device with that device current and cached.
qattn_status noalloc_scratch(long long** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return QATTN_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return QATTN_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_sums) != cudaSuccess || p == nullptr)
      return QATTN_ERR_CUDA;
    g_noalloc_ptr[dev] = static_cast<long long*>(p);
  }
  *out = g_noalloc_ptr[dev];
  return QATTN_OK;
}

}  // namespace

// =============================================================================================
// C ABI
// =============================================================================================

extern "C" {

const char* qattn_status_string(int status) {
  switch (status) {
    case QATTN_OK: return "ok";
    case QATTN_ERR_INVALID_ARG: return "invalid argument";
    case QATTN_ERR_UNSUPPORTED: return "unsupported shape or device";
    case QATTN_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case QATTN_ERR_CUDA: return "CUDA error";
    case QATTN_ERR_TIMEOUT: return "bounded wait inside a kernel timed out";
    case QATTN_ERR_WORKSPACE: return "workspace missing or too small";
    default: return "unknown status";
  }
}

int qattn_version(void) { return 100; }

size_t qattn_smooth_quant_workspace(int B, int Hkv, int d) {
  if (B < 1 || Hkv < 1 || d < 1) return 0;
  return align_up(sizeof(long long) * static_cast<size_t>(B) * Hkv * d);
}

qattn_status qattn_smooth_quant(const void* q, const void* k, int B, int H, int Hkv, int N, int d,
                                int8_t* q_i8, float* q_scale, int8_t* k_i8, float* k_scale,
                                float* k_mean, void* ws, size_t ws_bytes, qattn_stream_t stream) {
  qattn_status s = check_shape(B, H, Hkv, N, d);
  if (s != QATTN_OK) return s;
  s = check_ptrs(q, k, q_i8, q_scale, k_i8, k_scale);
  if (s != QATTN_OK) return s;
  if (k_mean && !aligned16(k_mean)) return QATTN_ERR_MISALIGNED;
  if (ws == nullptr || ws_bytes < qattn_smooth_quant_workspace(B, Hkv, d))
    return QATTN_ERR_WORKSPACE;
  if (!aligned16(ws)) return QATTN_ERR_MISALIGNED;
  if ((s = device_ok()) != QATTN_OK) return s;
  return dispatch_smooth_quant(q, k, B, H, Hkv, N, d, q_i8, q_scale, k_i8, k_scale, k_mean,
                               static_cast<long long*>(ws), reinterpret_cast<cudaStream_t>(stream));
}

// qattn_smooth_quant for callers that cannot allocate device memory: the channel-sum scratch is
// the library's static g_noalloc_sums instead of a caller workspace.  Same kernels and results.
qattn_status qattn_smooth_quant_noalloc(const void* q, const void* k, int B, int H, int Hkv, int N,
                                        int d, int8_t* q_i8, float* q_scale, int8_t* k_i8,
                                        float* k_scale, float* k_mean, qattn_stream_t stream) {
  qattn_status s = check_shape(B, H, Hkv, N, d);
  if (s != QATTN_OK) return s;
  s = check_ptrs(q, k, q_i8, q_scale, k_i8, k_scale);
  if (s != QATTN_OK) return s;
  if (k_mean && !aligned16(k_mean)) return QATTN_ERR_MISALIGNED;
  if (static_cast<size_t>(B) * Hkv * d > kNoAllocMaxSums) return QATTN_ERR_WORKSPACE;
  if ((s = device_ok()) != QATTN_OK) return s;
  long long* sums = nullptr;
  if ((s = noalloc_scratch(&sums)) != QATTN_OK) return s;
  // the shared scratch keeps the previous call's sums: the dispatch zeroes it on `stream` first
  return dispatch_smooth_quant(q, k, B, H, Hkv, N, d, q_i8, q_scale, k_i8, k_scale, k_mean, sums,
                               reinterpret_cast<cudaStream_t>(stream));
}

qattn_status qattn_attn_quantized(const int8_t* q_i8, const float* q_scale, const int8_t* k_i8,
                                  const float* k_scale, const void* v, void* out, int B, int H,
                                  int Hkv, int N, int d, int causal, qattn_stream_t stream) {
  qattn_status s = check_shape(B, H, Hkv, N, d);
  if (s != QATTN_OK) return s;
  s = check_ptrs(q_i8, q_scale, k_i8, k_scale, v, out);
  if (s != QATTN_OK) return s;
  if ((s = device_ok()) != QATTN_OK) return s;
  return dispatch_attn<false>(q_i8, q_scale, k_i8, k_scale, v, out, B, H, Hkv, N, d, causal,
                              reinterpret_cast<cudaStream_t>(stream));
}

qattn_status qattn_attn_quantized_f32(const int8_t* q_i8, const float* q_scale, const int8_t* k_i8,
                                      const float* k_scale, const void* v, float* out, int B,
                                      int H, int Hkv, int N, int d, int causal,
                                      qattn_stream_t stream) {
  qattn_status s = check_shape(B, H, Hkv, N, d);
  if (s != QATTN_OK) return s;
  s = check_ptrs(q_i8, q_scale, k_i8, k_scale, v, out);
  if (s != QATTN_OK) return s;
  if ((s = device_ok()) != QATTN_OK) return s;
  return dispatch_attn<false, kOutF32>(q_i8, q_scale, k_i8, k_scale, v, out, B, H, Hkv, N, d,
                                       causal, reinterpret_cast<cudaStream_t>(stream));
}

qattn_status qattn_smooth_k(const void* k, int B, int Hkv, int N, int d, int8_t* k_i8,
                            float* k_scale, float* k_mean, void* ws, size_t ws_bytes,
                            qattn_stream_t stream) {
  qattn_status s = check_shape(B, Hkv, Hkv, N, d);
  if (s != QATTN_OK) return s;
  s = check_ptrs(k, k_i8, k_scale);
  if (s != QATTN_OK) return s;
  if (k_mean && !aligned16(k_mean)) return QATTN_ERR_MISALIGNED;
  if (ws == nullptr || ws_bytes < qattn_smooth_quant_workspace(B, Hkv, d))
    return QATTN_ERR_WORKSPACE;
  if (!aligned16(ws)) return QATTN_ERR_MISALIGNED;
  if ((s = device_ok()) != QATTN_OK) return s;
  return dispatch_smooth_quant(nullptr, k, B, Hkv, Hkv, N, d, nullptr, nullptr, k_i8, k_scale,
                               k_mean, static_cast<long long*>(ws),
                               reinterpret_cast<cudaStream_t>(stream));
}

size_t qattn_block_select_workspace(int B, int H, int Hkv, int N, int d) {
  if (check_shape(B, H, Hkv, N, d) != QATTN_OK) return 0;
  return sel_layout(B, H, Hkv, N, d).total;
}

qattn_status qattn_block_select(const void* q, const void* k, int B, int H, int Hkv, int N, int d,
                                int causal, int topk, int* kv_list, int* kv_count, void* ws,
                                size_t ws_bytes, qattn_stream_t stream) {
  qattn_status s = check_shape(B, H, Hkv, N, d);
  if (s != QATTN_OK) return s;
  s = check_ptrs(q, k, kv_list, kv_count);
  if (s != QATTN_OK) return s;
  // non-causal with topk 0 would list no key tile for any query block
  if (topk < 0 || (!causal && topk == 0)) return QATTN_ERR_INVALID_ARG;
  if ((N + kSelKRows - 1) / kSelKRows > kSelMaxTiles) return QATTN_ERR_UNSUPPORTED;
  if (ws == nullptr || ws_bytes < sel_layout(B, H, Hkv, N, d).total) return QATTN_ERR_WORKSPACE;
  if (!aligned16(ws)) return QATTN_ERR_MISALIGNED;
  if ((s = device_ok()) != QATTN_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* w = static_cast<uint8_t*>(ws);
  return d == 128 ? run_block_select<128>(q, k, B, H, Hkv, N, causal, topk, kv_list, kv_count, w, st)
                  : run_block_select<64>(q, k, B, H, Hkv, N, causal, topk, kv_list, kv_count, w, st);
}

qattn_status qattn_attn_quantized_sparse(const int8_t* q_i8, const float* q_scale,
                                         const int8_t* k_i8, const float* k_scale, const void* v,
                                         void* out, int B, int H, int Hkv, int N, int d,
                                         int causal, const int* kv_list, const int* kv_count,
                                         qattn_stream_t stream) {
  qattn_status s = check_shape(B, H, Hkv, N, d);
  if (s != QATTN_OK) return s;
  s = check_ptrs(q_i8, q_scale, k_i8, k_scale, v, out, kv_list, kv_count);
  if (s != QATTN_OK) return s;
  if ((s = device_ok()) != QATTN_OK) return s;
  return dispatch_attn<false>(q_i8, q_scale, k_i8, k_scale, v, out, B, H, Hkv, N, d, causal,
                              reinterpret_cast<cudaStream_t>(stream), kv_list, kv_count);
}

qattn_status qattn_attn_fused_q(const void* q, const int8_t* k_i8, const float* k_scale,
                                const void* v, void* out, int B, int H, int Hkv, int N, int d,
                                int causal, qattn_stream_t stream) {
  qattn_status s = check_shape(B, H, Hkv, N, d);
  if (s != QATTN_OK) return s;
  s = check_ptrs(q, k_i8, k_scale, v, out);
  if (s != QATTN_OK) return s;
  if ((s = device_ok()) != QATTN_OK) return s;
  return dispatch_attn<true>(q, nullptr, k_i8, k_scale, v, out, B, H, Hkv, N, d, causal,
                             reinterpret_cast<cudaStream_t>(stream));
}

size_t qattn_forward_workspace(int B, int H, int Hkv, int N, int d) {
  if (check_shape(B, H, Hkv, N, d) != QATTN_OK) return 0;
  return forward_layout(B, H, Hkv, N, d).total;
}

qattn_status qattn_forward_ws(const void* q, const void* k, const void* v, void* out, int B,
                              int H, int Hkv, int N, int d, int causal, void* ws, size_t ws_bytes,
                              qattn_stream_t stream) {
  qattn_status s = check_shape(B, H, Hkv, N, d);
  if (s != QATTN_OK) return s;
  s = check_ptrs(q, k, v, out);
  if (s != QATTN_OK) return s;
  const QuantLayout L = forward_layout(B, H, Hkv, N, d);
  if (ws == nullptr || ws_bytes < L.total) return QATTN_ERR_WORKSPACE;
  if (!aligned16(ws)) return QATTN_ERR_MISALIGNED;
  if ((s = device_ok()) != QATTN_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* w = static_cast<uint8_t*>(ws);
  int8_t* q_i8 = reinterpret_cast<int8_t*>(w + L.q_i8);
  int8_t* k_i8 = reinterpret_cast<int8_t*>(w + L.k_i8);
  float* q_scale = reinterpret_cast<float*>(w + L.q_scale);
  float* k_scale = reinterpret_cast<float*>(w + L.k_scale);
  long long* sums = reinterpret_cast<long long*>(w + L.sums);
  // Smoothing + quantization of Q and K in one pass, then attention on the int8 operands.  (The
  // variant with Q quantized inside the attention kernel, qattn_smooth_k + qattn_attn_fused_q,
  // gives identical results but measured slower: its per-CTA quantization prologue lies on
  // every CTA's critical path.)
  s = dispatch_smooth_quant(q, k, B, H, Hkv, N, d, q_i8, q_scale, k_i8, k_scale, nullptr, sums, st);
  if (s != QATTN_OK) return s;
  return dispatch_attn<false>(q_i8, q_scale, k_i8, k_scale, v, out, B, H, Hkv, N, d, causal, st);
}

qattn_status qattn_forward(const void* q, const void* k, const void* v, void* out, int B, int H,
                           int Hkv, int N, int d, int causal, qattn_stream_t stream) {
  qattn_status s = check_shape(B, H, Hkv, N, d);
  if (s != QATTN_OK) return s;
  s = check_ptrs(q, k, v, out);
  if (s != QATTN_OK) return s;
  if ((s = device_ok()) != QATTN_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const size_t bytes = forward_layout(B, H, Hkv, N, d).total;
  void* ws = nullptr;
  if ((s = pool_alloc(&ws, bytes, st)) != QATTN_OK) return s;
  s = qattn_forward_ws(q, k, v, out, B, H, Hkv, N, d, causal, ws, bytes, stream);
  if (cudaFreeAsync(ws, st) != cudaSuccess && s == QATTN_OK) s = QATTN_ERR_CUDA;
  return s;
}

qattn_status qattn_forward_sparse(const void* q, const void* k, const void* v, void* out, int B,
                                  int H, int Hkv, int N, int d, int causal, int topk,
                                  qattn_stream_t stream) {
  qattn_status s = check_shape(B, H, Hkv, N, d);
  if (s != QATTN_OK) return s;
  s = check_ptrs(q, k, v, out);
  if (s != QATTN_OK) return s;
  // non-causal with topk 0 would leave every row without a key
  if (topk < 0 || (!causal && topk == 0)) return QATTN_ERR_INVALID_ARG;
  if ((N + kSelKRows - 1) / kSelKRows > kSelMaxTiles) return QATTN_ERR_UNSUPPORTED;
  if ((s = device_ok()) != QATTN_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // one stream-ordered workspace: the quantized operands, the selection's scratch and the
  // tile lists (kv_list [B*H][ceil(N/256)][ceil(N/128)], kv_count [B*H][ceil(N/256)])
  const QuantLayout L = forward_layout(B, H, Hkv, N, d);
  const SelLayout S = sel_layout(B, H, Hkv, N, d);
  const size_t off_sel = L.total;
  const size_t off_list = align_up(off_sel + S.total);
  const size_t n_list = static_cast<size_t>(B) * H * S.nsb * S.nkt;
  const size_t off_count = align_up(off_list + sizeof(int) * n_list);
  const size_t total = align_up(off_count + sizeof(int) * static_cast<size_t>(B) * H * S.nsb);
  void* ws = nullptr;
  if ((s = pool_alloc(&ws, total, st)) != QATTN_OK) return s;
  uint8_t* w = static_cast<uint8_t*>(ws);
  int8_t* q_i8 = reinterpret_cast<int8_t*>(w + L.q_i8);
  int8_t* k_i8 = reinterpret_cast<int8_t*>(w + L.k_i8);
  float* q_scale = reinterpret_cast<float*>(w + L.q_scale);
  float* k_scale = reinterpret_cast<float*>(w + L.k_scale);
  long long* sums = reinterpret_cast<long long*>(w + L.sums);
  int* kv_list = reinterpret_cast<int*>(w + off_list);
  int* kv_count = reinterpret_cast<int*>(w + off_count);
  s = dispatch_smooth_quant(q, k, B, H, Hkv, N, d, q_i8, q_scale, k_i8, k_scale, nullptr, sums, st);
  if (s == QATTN_OK)
    s = d == 128 ? run_block_select<128>(q, k, B, H, Hkv, N, causal, topk, kv_list, kv_count, w + off_sel, st)
                 : run_block_select<64>(q, k, B, H, Hkv, N, causal, topk, kv_list, kv_count, w + off_sel, st);
  if (s == QATTN_OK)
    s = dispatch_attn<false>(q_i8, q_scale, k_i8, k_scale, v, out, B, H, Hkv, N, d, causal, st,
                             kv_list, kv_count);
  if (cudaFreeAsync(ws, st) != cudaSuccess && s == QATTN_OK) s = QATTN_ERR_CUDA;
  return s;
}

namespace {

// Copy streams of the host-buffer forward, created once per device (non-blocking, so they do
// not serialise with the legacy default stream).
std::mutex g_copy_mu;
std::map<int, std::pair<cudaStream_t, cudaStream_t>> g_copy_streams;

qattn_status copy_streams(cudaStream_t* in, cudaStream_t* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return QATTN_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_copy_mu);
  auto it = g_copy_streams.find(dev);
  if (it == g_copy_streams.end()) {
    cudaStream_t a = nullptr, b = nullptr;
    if (cudaStreamCreateWithFlags(&a, cudaStreamNonBlocking) != cudaSuccess) return QATTN_ERR_CUDA;
    if (cudaStreamCreateWithFlags(&b, cudaStreamNonBlocking) != cudaSuccess) {
      cudaStreamDestroy(a);
      return QATTN_ERR_CUDA;
    }
    it = g_copy_streams.emplace(dev, std::make_pair(a, b)).first;
  }
  *in = it->second.first;
  *out = it->second.second;
  return QATTN_OK;
}

constexpr int kHostChunks = 8;  // pipeline depth of the host-buffer forward

}  // namespace

qattn_status qattn_forward_host(const void* q_host, const void* k_host, const void* v_host,
                                void* out_host, int B, int H, int Hkv, int N, int d, int causal,
                                qattn_stream_t stream) {
  qattn_status s = check_shape(B, H, Hkv, N, d);
  if (s != QATTN_OK) return s;
  if (!q_host || !k_host || !v_host || !out_host) return QATTN_ERR_INVALID_ARG;
  if ((s = device_ok()) != QATTN_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaStream_t s_in = nullptr, s_out = nullptr;
  if ((s = copy_streams(&s_in, &s_out)) != QATTN_OK) return s;
  const size_t qb = sizeof(uint16_t) * static_cast<size_t>(B) * H * N * d;
  const size_t kb = sizeof(uint16_t) * static_cast<size_t>(B) * Hkv * N * d;
  const size_t off_k = align_up(qb), off_v = off_k + align_up(kb), off_o = off_v + align_up(kb);
  const size_t total = off_o + align_up(qb);
  void* buf = nullptr;
  if ((s = pool_alloc(&buf, total, st)) != QATTN_OK) return s;
  uint8_t* b8 = static_cast<uint8_t*>(buf);
  // Every (batch, kv head) group -- its kv head and the H / Hkv query heads reading it -- is an
  // independent forward (the smoothing mean is per group), and group f = b * Hkv + g owns
  // contiguous bytes of q, k, v and out (its query heads too).  The groups are cut into up to
  // kHostChunks chunks; chunk c's upload (s_in), forward (the caller's stream) and download (s_out)
  // are ordered by events, so one chunk's copies overlap another chunk's kernels.  When the chunks
  // are single groups of two or more query heads, the first and the last group run as two pieces
  // of half their query heads each (the first piece uploads the group's K and V): the first
  // forward starts after a smaller upload and the last download is smaller, at the price of one
  // more smoothing pass of those groups' K.
  const int G = B * Hkv, r = H / Hkv;
  const int nch = G < kHostChunks ? G : kHostChunks;
  const int per = (G + nch - 1) / nch;
  const size_t q_head = sizeof(uint16_t) * static_cast<size_t>(N) * d;
  const size_t q_grp = q_head * r;
  const size_t k_grp = q_head;
  struct Piece {
    int f0, nf, h0, nh;  // groups f0 .. f0 + nf - 1, query heads h0 .. h0 + nh - 1 of each
    bool kv;             // this piece uploads the groups' K and V
  };
  Piece pcs[kHostChunks + 2];
  int np = 0;
  const bool split = per == 1 && r >= 2;
  for (int c = 0; c < nch; ++c) {
    const int f0 = c * per, nf = (f0 + per <= G ? per : G - f0);
    if (nf <= 0) break;
    if (split && (c == 0 || c == nch - 1)) {
      pcs[np++] = Piece{f0, 1, 0, r / 2, true};
      pcs[np++] = Piece{f0, 1, r / 2, r - r / 2, false};
    } else {
      pcs[np++] = Piece{f0, nf, 0, r, true};
    }
  }
  cudaEvent_t ev[2 * (kHostChunks + 2) + 2] = {};
  int nev = 0;
  for (int i = 0; i < 2 * np + 2 && s == QATTN_OK; ++i, ++nev)
    if (cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming) != cudaSuccess) s = QATTN_ERR_CUDA;
  const char* qh = static_cast<const char*>(q_host);
  const char* kh = static_cast<const char*>(k_host);
  const char* vh = static_cast<const char*>(v_host);
  char* oh = static_cast<char*>(out_host);
  // s_in and s_out start after the work already queued on the caller's stream (the pool
  // allocation above and anything before this call)
  if (s == QATTN_OK && (cudaEventRecord(ev[2 * np], st) != cudaSuccess ||
                        cudaStreamWaitEvent(s_in, ev[2 * np], 0) != cudaSuccess ||
                        cudaStreamWaitEvent(s_out, ev[2 * np], 0) != cudaSuccess))
    s = QATTN_ERR_CUDA;
  // q and out bytes of a piece: its query heads are contiguous within each of its groups, and a
  // piece of several groups takes all their heads, so the piece's bytes are one contiguous run
  auto q_off = [&](const Piece& p) { return p.f0 * q_grp + p.h0 * q_head; };
  auto q_len = [&](const Piece& p) { return p.nf * static_cast<size_t>(p.nh) * q_head; };
  for (int c = 0; c < np && s == QATTN_OK; ++c) {
    const Piece& p = pcs[c];
    if (cudaMemcpyAsync(b8 + q_off(p), qh + q_off(p), q_len(p), cudaMemcpyHostToDevice, s_in) != cudaSuccess ||
        (p.kv && (cudaMemcpyAsync(b8 + off_k + p.f0 * k_grp, kh + p.f0 * k_grp, p.nf * k_grp,
                                  cudaMemcpyHostToDevice, s_in) != cudaSuccess ||
                  cudaMemcpyAsync(b8 + off_v + p.f0 * k_grp, vh + p.f0 * k_grp, p.nf * k_grp,
                                  cudaMemcpyHostToDevice, s_in) != cudaSuccess)) ||
        cudaEventRecord(ev[c], s_in) != cudaSuccess)
      s = QATTN_ERR_CUDA;
  }
  for (int c = 0; c < np && s == QATTN_OK; ++c) {
    const Piece& p = pcs[c];
    // a piece's K and V arrived with it or with an earlier piece (s_in runs in order)
    if (cudaStreamWaitEvent(st, ev[c], 0) != cudaSuccess) {
      s = QATTN_ERR_CUDA;
      break;
    }
    // the piece as a forward of nf "batches" of one kv head and nh query heads each
    s = qattn_forward(b8 + q_off(p), b8 + off_k + p.f0 * k_grp, b8 + off_v + p.f0 * k_grp,
                      b8 + off_o + q_off(p), p.nf, p.nh, 1, N, d, causal, stream);
    if (s == QATTN_OK && (cudaEventRecord(ev[np + c], st) != cudaSuccess ||
                          cudaStreamWaitEvent(s_out, ev[np + c], 0) != cudaSuccess ||
                          cudaMemcpyAsync(oh + q_off(p), b8 + off_o + q_off(p), q_len(p),
                                          cudaMemcpyDeviceToHost, s_out) != cudaSuccess))
      s = QATTN_ERR_CUDA;
  }
  // the caller's stream takes up both copy streams again before the buffer goes back to the pool
  if (nev < 2 * np + 2) {
    // not every event exists, so nothing was queued on the copy streams
  } else if (cudaEventRecord(ev[2 * np + 1], s_out) != cudaSuccess ||
      cudaStreamWaitEvent(st, ev[2 * np + 1], 0) != cudaSuccess ||
      cudaEventRecord(ev[2 * np], s_in) != cudaSuccess ||
      cudaStreamWaitEvent(st, ev[2 * np], 0) != cudaSuccess) {
    if (s == QATTN_OK) s = QATTN_ERR_CUDA;
  }
  if (cudaFreeAsync(buf, st) != cudaSuccess && s == QATTN_OK) s = QATTN_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess && s == QATTN_OK) s = QATTN_ERR_CUDA;
  for (int i = 0; i < nev; ++i) cudaEventDestroy(ev[i]);
  return s;
}

qattn_status qattn_debug_qk_int32(const int8_t* q_i8, const int8_t* k_i8, int32_t* s_out, int B,
                                  int H, int Hkv, int N, int d, int causal, int b, int h, int qt0,
                                  int nqt, int kt0, int nkt, qattn_stream_t stream) {
  qattn_status s = check_shape(B, H, Hkv, N, d);
  if (s != QATTN_OK) return s;
  s = check_ptrs(q_i8, k_i8, s_out);
  if (s != QATTN_OK) return s;
  const int ntiles = (N + 127) / 128;
  if (b < 0 || b >= B || h < 0 || h >= H || qt0 < 0 || nqt < 1 || kt0 < 0 || nkt < 1 ||
      qt0 + nqt > ntiles || kt0 + nkt > ntiles)
    return QATTN_ERR_INVALID_ARG;
  if ((s = device_ok()) != QATTN_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // The attention kernel itself runs, so it needs V, an output and scales: zero V and zero scales
  // (every score then dequantizes to 0; the int32 tiles do not depend on them), from the pool.
  const size_t nqb = (N + 127) / 128, nkb = (N + 63) / 64;
  const size_t vb = align_up(sizeof(uint16_t) * static_cast<size_t>(B) * Hkv * N * d);
  const size_t ob = align_up(sizeof(uint16_t) * static_cast<size_t>(B) * H * N * d);
  const size_t qsb = align_up(sizeof(float) * static_cast<size_t>(B) * H * nqb);
  const size_t ksb = align_up(sizeof(float) * static_cast<size_t>(B) * Hkv * nkb);
  void* ws = nullptr;
  if ((s = pool_alloc(&ws, vb + ob + qsb + ksb, st)) != QATTN_OK) return s;
  uint8_t* w = static_cast<uint8_t*>(ws);
  const size_t s_bytes = sizeof(int32_t) * static_cast<size_t>(nqt) * 128 * nkt * 128;
  // tiles the causal kernel never computes (key tile above the query tile) read as 0
  if (cudaMemsetAsync(w, 0, vb, st) != cudaSuccess ||
      cudaMemsetAsync(w + vb + ob, 0, qsb + ksb, st) != cudaSuccess ||
      cudaMemsetAsync(s_out, 0, s_bytes, st) != cudaSuccess)
    s = QATTN_ERR_CUDA;
  ScoreDump dump;
  dump.s_out = s_out;
  dump.ld = nkt * 128;
  dump.bh = b * H + h;
  dump.pair0 = qt0 / 2;
  dump.qt0 = qt0;
  dump.nqt = nqt;
  dump.kt0 = kt0;
  dump.nkt = nkt;
  const int pairs = (qt0 + nqt - 1) / 2 - qt0 / 2 + 1;
  const float* qs = reinterpret_cast<const float*>(w + vb + ob);
  const float* ks = reinterpret_cast<const float*>(w + vb + ob + qsb);
  if (s == QATTN_OK) {
#define QATTN_DUMP_ARGS q_i8, qs, k_i8, ks, w, w + vb, B, H, Hkv, N, st, nullptr, nullptr, &dump, pairs
    if (d == 128)
      s = causal ? run_attn<128, true, false, kDumpS>(QATTN_DUMP_ARGS)
                 : run_attn<128, false, false, kDumpS>(QATTN_DUMP_ARGS);
    else
      s = causal ? run_attn<64, true, false, kDumpS>(QATTN_DUMP_ARGS)
                 : run_attn<64, false, false, kDumpS>(QATTN_DUMP_ARGS);
#undef QATTN_DUMP_ARGS
  }
  if (cudaFreeAsync(ws, st) != cudaSuccess && s == QATTN_OK) s = QATTN_ERR_CUDA;
  return s;
}

qattn_status qattn_attn_nvfp4(const uint8_t* q_codes, const uint8_t* q_scales, const float* q_g,
                              const uint8_t* k_codes, const uint8_t* k_scales, const float* k_g,
                              const uint8_t* vt_codes, const uint8_t* vt_scales, const float* v_g,
                              const void* q, const void* k, const void* v, const float* k_mean,
                              const int* kv_list, const int* kv_count, void* out, int B, int H,
                              int Hkv, int N, int d, int causal, qattn_stream_t stream) {
  qattn_status s = check_shape(B, H, Hkv, N, d);
  if (s != QATTN_OK) return s;
  s = check_ptrs(q_codes, q_scales, q_g, k_codes, k_scales, k_g, vt_codes, vt_scales, v_g, out);
  if (s != QATTN_OK) return s;
  if (kv_list != nullptr && (s = check_ptrs(q, k, v, k_mean, kv_list, kv_count)) != QATTN_OK)
    return s;
  if (static_cast<long long>(B) * H > 65535) return QATTN_ERR_UNSUPPORTED;
  // promotion lists index at most 1024 key tiles (N <= 131072, the selection's limit)
  if (kv_list != nullptr && (N + 127) / 128 > Fp4AttnCfg<128>::kMaxTiles) return QATTN_ERR_UNSUPPORTED;
  if ((s = device_ok()) != QATTN_OK) return s;
  return dispatch_attn_nvfp4(q_codes, q_scales, q_g, k_codes, k_scales, k_g, vt_codes, vt_scales,
                             v_g, q, k, v, k_mean, kv_list, kv_count, out, B, H, Hkv, N, d, causal,
                             reinterpret_cast<cudaStream_t>(stream));
}

qattn_status qattn_forward_nvfp4(const void* q, const void* k, const void* v, void* out, int B,
                                 int H, int Hkv, int N, int d, int causal, int topk,
                                 qattn_stream_t stream) {
  qattn_status s = check_shape(B, H, Hkv, N, d);
  if (s != QATTN_OK) return s;
  s = check_ptrs(q, k, v, out);
  if (s != QATTN_OK) return s;
  // topk -1: every tile in FP4; topk >= 0: the selected tiles in FP16 (non-causal topk 0 would
  // promote nothing and is the same as -1, so it is accepted)
  if (topk < -1) return QATTN_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * H > 65535) return QATTN_ERR_UNSUPPORTED;
  if (topk >= 0 && (N + kSelKRows - 1) / kSelKRows > kSelMaxTiles) return QATTN_ERR_UNSUPPORTED;
  if ((s = device_ok()) != QATTN_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // one stream-ordered workspace: channel sums and mean, the three NVFP4 operands, and (with
  // promotion) the selection's scratch and tile lists
  const size_t BH = static_cast<size_t>(B) * H, BG = static_cast<size_t>(B) * Hkv;
  const size_t Np = (static_cast<size_t>(N) + 127) / 128 * 128;
  size_t off = 0;
  auto take = [&](size_t bytes) { const size_t o = off; off = align_up(off + bytes); return o; };
  const size_t o_sums = take(sizeof(long long) * BG * d), o_mean = take(sizeof(float) * BG * d);
  const size_t o_qc = take(BH * N * d / 2), o_qs = take(BH * N * d / 16), o_qg = take(4 * BH);
  const size_t o_kc = take(BG * N * d / 2), o_ks = take(BG * N * d / 16), o_kg = take(4 * BG);
  const size_t o_vc = take(BG * d * Np / 2), o_vs = take(BG * d * Np / 16), o_vg = take(4 * BG);
  const SelLayout S = sel_layout(B, H, Hkv, N, d);
  const size_t o_sel = topk >= 0 ? take(S.total) : 0;
  const size_t o_list = topk >= 0 ? take(sizeof(int) * BH * S.nsb * S.nkt) : 0;
  const size_t o_count = topk >= 0 ? take(sizeof(int) * BH * S.nsb) : 0;
  void* ws = nullptr;
  if ((s = pool_alloc(&ws, off, st)) != QATTN_OK) return s;
  uint8_t* w = static_cast<uint8_t*>(ws);
  long long* sums = reinterpret_cast<long long*>(w + o_sums);
  float* mean = reinterpret_cast<float*>(w + o_mean);
  int* kv_list = topk >= 0 ? reinterpret_cast<int*>(w + o_list) : nullptr;
  int* kv_count = topk >= 0 ? reinterpret_cast<int*>(w + o_count) : nullptr;
  if (cudaMemsetAsync(sums, 0, sizeof(long long) * BG * d, st) != cudaSuccess) s = QATTN_ERR_CUDA;
  if (s == QATTN_OK) {
    const dim3 g1(static_cast<unsigned>(BG), (N + kSumRowsPerCta - 1) / kSumRowsPerCta);
    if (d == 128) k_channel_sums_kernel<128><<<g1, 256, 0, st>>>(static_cast<const uint16_t*>(k), N, sums);
    else k_channel_sums_kernel<64><<<g1, 256, 0, st>>>(static_cast<const uint16_t*>(k), N, sums);
    const int n = static_cast<int>(BG) * d;
    k_mean_from_sums_kernel<<<(n + 255) / 256, 256, 0, st>>>(sums, N, n, mean);
    s = launch_status();
  }
  if (s == QATTN_OK)
    s = dispatch_quant_nvfp4(q, nullptr, static_cast<int>(BH), N, d, 0, w + o_qc, w + o_qs,
                             reinterpret_cast<float*>(w + o_qg), st);
  if (s == QATTN_OK)
    s = dispatch_quant_nvfp4(k, mean, static_cast<int>(BG), N, d, 0, w + o_kc, w + o_ks,
                             reinterpret_cast<float*>(w + o_kg), st);
  if (s == QATTN_OK)
    s = dispatch_quant_nvfp4(v, nullptr, static_cast<int>(BG), N, d, 1, w + o_vc, w + o_vs,
                             reinterpret_cast<float*>(w + o_vg), st);
  if (s == QATTN_OK && topk >= 0)
    s = d == 128 ? run_block_select<128>(q, k, B, H, Hkv, N, causal, topk, kv_list, kv_count, w + o_sel, st)
                 : run_block_select<64>(q, k, B, H, Hkv, N, causal, topk, kv_list, kv_count, w + o_sel, st);
  if (s == QATTN_OK)
    s = dispatch_attn_nvfp4(w + o_qc, w + o_qs, reinterpret_cast<float*>(w + o_qg), w + o_kc,
                            w + o_ks, reinterpret_cast<float*>(w + o_kg), w + o_vc, w + o_vs,
                            reinterpret_cast<float*>(w + o_vg), q, k, v, mean, kv_list, kv_count,
                            out, B, H, Hkv, N, d, causal, st);
  if (cudaFreeAsync(ws, st) != cudaSuccess && s == QATTN_OK) s = QATTN_ERR_CUDA;
  return s;
}

qattn_status qattn_debug_qk_nvfp4(const uint8_t* q_codes, const uint8_t* q_scales,
                                  const float* q_g, const uint8_t* k_codes,
                                  const uint8_t* k_scales, const float* k_g, float* s_out, int B,
                                  int H, int Hkv, int N, int d, int b, int h, int qt0, int nqt,
                                  int kt0, int nkt, qattn_stream_t stream) {
  qattn_status s = check_shape(B, H, Hkv, N, d);
  if (s != QATTN_OK) return s;
  s = check_ptrs(q_codes, q_scales, q_g, k_codes, k_scales, k_g, s_out);
  if (s != QATTN_OK) return s;
  const int ntiles = (N + 127) / 128;
  if (b < 0 || b >= B || h < 0 || h >= H || qt0 < 0 || nqt < 1 || kt0 < 0 || nkt < 1 ||
      qt0 + nqt > ntiles || kt0 + nkt > ntiles || nqt > 65535 || nkt > 65535)
    return QATTN_ERR_INVALID_ARG;
  if ((s = device_ok()) != QATTN_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  CUtensorMap tq, tk;
  if (!make_fp4_map(&tq, q_codes, d, N, static_cast<long long>(B) * H) ||
      !make_fp4_map(&tk, k_codes, d, N, static_cast<long long>(B) * Hkv))
    return QATTN_ERR_CUDA;
  // 100 KB of shared memory per CTA caps residency at 2 CTAs (512 TMEM columns) per SM.
  const int smem = 100 * 1024;
  const int bh = b * H + h;
  const int bg = b * Hkv + h / (H / Hkv);
  dim3 grid(nqt, nkt);
  if (d == 128) {
    if (cudaFuncSetAttribute(qk_nvfp4_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem) != cudaSuccess)
      return QATTN_ERR_CUDA;
    qk_nvfp4_kernel<128><<<grid, 128, smem, st>>>(tq, tk, q_scales, k_scales, q_g, k_g, s_out, N,
                                                  bh, bg, qt0, kt0, nkt * 128);
  } else {
    if (cudaFuncSetAttribute(qk_nvfp4_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem) != cudaSuccess)
      return QATTN_ERR_CUDA;
    qk_nvfp4_kernel<64><<<grid, 128, smem, st>>>(tq, tk, q_scales, k_scales, q_g, k_g, s_out, N,
                                                 bh, bg, qt0, kt0, nkt * 128);
  }
  return launch_status();
}

qattn_status qattn_debug_wait_timeout(long long limit_cycles, int* gave_up,
                                      qattn_stream_t stream) {
  if (gave_up == nullptr || limit_cycles < 0 || limit_cycles > kWaitLimitCycles)
    return QATTN_ERR_INVALID_ARG;
  qattn_status s = device_ok();
  if (s != QATTN_OK) return s;
  wait_timeout_probe_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(limit_cycles,
                                                                                  gave_up);
  return launch_status();
}

qattn_status qattn_quant_nvfp4(const void* x, const float* mean, int S, int R, int C,
                               int along_rows, uint8_t* codes, uint8_t* scales, float* gscale,
                               qattn_stream_t stream) {
  if (S < 1 || R < 1 || C < 1) return QATTN_ERR_INVALID_ARG;
  if (C % 16 != 0 || S > 65535 || static_cast<long long>(R) * C > (1LL << 31))
    return QATTN_ERR_UNSUPPORTED;
  qattn_status s = check_ptrs(x, codes, scales, gscale);
  if (s != QATTN_OK) return s;
  if (mean && !aligned16(mean)) return QATTN_ERR_MISALIGNED;
  if ((s = device_ok()) != QATTN_OK) return s;
  return dispatch_quant_nvfp4(x, mean, S, R, C, along_rows, codes, scales, gscale,
                              reinterpret_cast<cudaStream_t>(stream));
}

qattn_status qattn_quant_v_fp8(const void* v, int B, int Hkv, int N, int d, uint8_t* vt8,
                              float* v_scale, qattn_stream_t stream) {
  qattn_status s = check_shape(B, Hkv, Hkv, N, d);
  if (s != QATTN_OK) return s;
  s = check_ptrs(v, vt8, v_scale);
  if (s != QATTN_OK) return s;
  if (static_cast<long long>(B) * Hkv > 65535) return QATTN_ERR_UNSUPPORTED;
  if ((s = device_ok()) != QATTN_OK) return s;
  return dispatch_quant_v_fp8(v, B * Hkv, N, d, vt8, v_scale, reinterpret_cast<cudaStream_t>(stream));
}

qattn_status qattn_attn_quantized_pv8(const int8_t* q_i8, const float* q_scale, const int8_t* k_i8,
                                      const float* k_scale, const uint8_t* vt8,
                                      const float* v_scale, void* out, int B, int H, int Hkv,
                                      int N, int d, int causal, qattn_stream_t stream) {
  qattn_status s = check_shape(B, H, Hkv, N, d);
  if (s != QATTN_OK) return s;
  s = check_ptrs(q_i8, q_scale, k_i8, k_scale, vt8, v_scale, out);
  if (s != QATTN_OK) return s;
  if ((s = device_ok()) != QATTN_OK) return s;
  Pv8Args pv;
  pv.vt8 = vt8;
  pv.v_scale = v_scale;
  return dispatch_attn_pv8<kPvF8>(q_i8, q_scale, k_i8, k_scale, nullptr, pv, out, B, H, Hkv, N, d,
                                  causal, reinterpret_cast<cudaStream_t>(stream));
}

namespace {

// Workspace of the adaptive entry points: the INT8 path's operands, E4M3 V^T and its scales.
struct AdaptiveLayout {
  QuantLayout q;
  size_t vt8, vscale, total;
};

AdaptiveLayout adaptive_layout(int B, int H, int Hkv, int N, int d) {
  AdaptiveLayout L;
  L.q = forward_layout(B, H, Hkv, N, d);
  const size_t Np = (static_cast<size_t>(N) + 127) / 128 * 128;
  L.vt8 = L.q.total;
  L.vscale = align_up(L.vt8 + static_cast<size_t>(B) * Hkv * d * Np);
  L.total = align_up(L.vscale + sizeof(float) * B * Hkv);
  return L;
}

// Smoothing + INT8 quantization of Q and K and E4M3 V into workspace w.
qattn_status adaptive_operands(const void* q, const void* k, const void* v, int B, int H, int Hkv,
                               int N, int d, const AdaptiveLayout& L, uint8_t* w, cudaStream_t st) {
  qattn_status s = dispatch_smooth_quant(
      q, k, B, H, Hkv, N, d, reinterpret_cast<int8_t*>(w + L.q.q_i8),
      reinterpret_cast<float*>(w + L.q.q_scale), reinterpret_cast<int8_t*>(w + L.q.k_i8),
      reinterpret_cast<float*>(w + L.q.k_scale), nullptr, reinterpret_cast<long long*>(w + L.q.sums),
      st);
  if (s != QATTN_OK) return s;
  return dispatch_quant_v_fp8(v, B * Hkv, N, d, w + L.vt8, reinterpret_cast<float*>(w + L.vscale), st);
}

}  // namespace

qattn_status qattn_forward_adaptive(const void* q, const void* k, const void* v, void* out, int B,
                                    int H, int Hkv, int N, int d, int causal,
                                    const uint8_t* variant, qattn_stream_t stream) {
  qattn_status s = check_shape(B, H, Hkv, N, d);
  if (s != QATTN_OK) return s;
  s = check_ptrs(q, k, v, out);
  if (s != QATTN_OK) return s;
  if (variant == nullptr) return QATTN_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * Hkv > 65535) return QATTN_ERR_UNSUPPORTED;
  if ((s = device_ok()) != QATTN_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const AdaptiveLayout L = adaptive_layout(B, H, Hkv, N, d);
  void* ws = nullptr;
  if ((s = pool_alloc(&ws, L.total, st)) != QATTN_OK) return s;
  uint8_t* w = static_cast<uint8_t*>(ws);
  s = adaptive_operands(q, k, v, B, H, Hkv, N, d, L, w, st);
  if (s == QATTN_OK) {
    Pv8Args pv;
    pv.vt8 = w + L.vt8;
    pv.v_scale = reinterpret_cast<const float*>(w + L.vscale);
    pv.variant = variant;
    s = dispatch_attn_pv8<kPvTable>(reinterpret_cast<const int8_t*>(w + L.q.q_i8),
                                    reinterpret_cast<const float*>(w + L.q.q_scale),
                                    reinterpret_cast<const int8_t*>(w + L.q.k_i8),
                                    reinterpret_cast<const float*>(w + L.q.k_scale), v, pv, out, B,
                                    H, Hkv, N, d, causal, st);
  }
  if (cudaFreeAsync(ws, st) != cudaSuccess && s == QATTN_OK) s = QATTN_ERR_CUDA;
  return s;
}

qattn_status qattn_adaptive_calibrate(const void* q, const void* k, const void* v, int B, int H,
                                      int Hkv, int N, int d, int causal, float tau,
                                      uint8_t* variant, float* cosine, qattn_stream_t stream) {
  qattn_status s = check_shape(B, H, Hkv, N, d);
  if (s != QATTN_OK) return s;
  s = check_ptrs(q, k, v, variant);
  if (s != QATTN_OK) return s;
  if (!(tau >= -1.0f && tau <= 2.0f)) return QATTN_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * Hkv > 65535) return QATTN_ERR_UNSUPPORTED;
  if ((s = device_ok()) != QATTN_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const AdaptiveLayout L = adaptive_layout(B, H, Hkv, N, d);
  const size_t ob = align_up(sizeof(uint16_t) * static_cast<size_t>(B) * H * N * d);
  const size_t G = static_cast<size_t>(B) * Hkv;
  const size_t off_a = L.total, off_b = off_a + ob, off_acc = off_b + ob;
  const size_t total = align_up(off_acc + sizeof(double) * 3 * G);
  void* ws = nullptr;
  if ((s = pool_alloc(&ws, total, st)) != QATTN_OK) return s;
  uint8_t* w = static_cast<uint8_t*>(ws);
  double* acc = reinterpret_cast<double*>(w + off_acc);
  s = adaptive_operands(q, k, v, B, H, Hkv, N, d, L, w, st);
  const int8_t* q_i8 = reinterpret_cast<const int8_t*>(w + L.q.q_i8);
  const int8_t* k_i8 = reinterpret_cast<const int8_t*>(w + L.q.k_i8);
  const float* q_s = reinterpret_cast<const float*>(w + L.q.q_scale);
  const float* k_s = reinterpret_cast<const float*>(w + L.q.k_scale);
  // both variants on the calibration input, then the cosine of their outputs per group
  if (s == QATTN_OK)
    s = dispatch_attn<false>(q_i8, q_s, k_i8, k_s, v, w + off_a, B, H, Hkv, N, d, causal, st);
  if (s == QATTN_OK) {
    Pv8Args pv;
    pv.vt8 = w + L.vt8;
    pv.v_scale = reinterpret_cast<const float*>(w + L.vscale);
    s = dispatch_attn_pv8<kPvF8>(q_i8, q_s, k_i8, k_s, nullptr, pv, w + off_b, B, H, Hkv, N, d,
                                 causal, st);
  }
  if (s == QATTN_OK && cudaMemsetAsync(acc, 0, sizeof(double) * 3 * G, st) != cudaSuccess)
    s = QATTN_ERR_CUDA;
  if (s == QATTN_OK) {
    const long long per = static_cast<long long>(H / Hkv) * N * d;
    long long gx = per / (256 * 64);
    const long long cap = (148LL * 8 + static_cast<long long>(G) - 1) / static_cast<long long>(G);
    if (gx > cap) gx = cap;
    if (gx < 1) gx = 1;
    group_cosine_parts_kernel<<<dim3(static_cast<unsigned>(gx), static_cast<unsigned>(G)), 256, 0, st>>>(
        reinterpret_cast<const __half*>(w + off_a), reinterpret_cast<const __half*>(w + off_b), per, acc);
    s = launch_status();
  }
  if (s == QATTN_OK) {
    choose_variant_kernel<<<static_cast<unsigned>((G + 255) / 256), 256, 0, st>>>(
        acc, static_cast<int>(G), tau, variant, cosine);
    s = launch_status();
  }
  if (cudaFreeAsync(ws, st) != cudaSuccess && s == QATTN_OK) s = QATTN_ERR_CUDA;
  return s;
}

qattn_status qattn_check_device_status(qattn_stream_t stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return QATTN_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, qattn::g_device_status, sizeof(v)) != cudaSuccess)
    return QATTN_ERR_CUDA;
  if (v != 0) {
    const unsigned int zero = 0;
    cudaMemcpyToSymbol(qattn::g_device_status, &zero, sizeof(zero));
    return static_cast<qattn_status>(v);
  }
  return QATTN_OK;
}

}  // extern "C"
