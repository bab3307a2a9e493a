/*
 * qattn.h -- C ABI of the B200 (sm_100a) smoothed-K INT8 attention forward (prefill).
 *
 * The method is the 8-bit attention summarised on the SageAttention page
 * ("SAGEATTENTION: accurate 8-bit attention for plug-and-play inference acceleration",
 * aibr.jp/archives/102657):
 *   - sec. 3: K is smoothed before quantization, Q and K are quantized to INT8, Q K^T runs on the
 *     tensor cores with 32-bit integer accumulation (mma(u8.u8.s32) on the page's GPU; signed
 *     s8 x s8 -> s32 here), P V runs with FP16 operands (mma(f16.f16.f16) on the page's GPU);
 *   - sec. 4: the kernel keeps FlashAttention's blockwise online softmax;
 *   - dialogue and sec. 2: it is a plug-and-play replacement of the attention call.
 * Where the page is silent this library takes these readings:
 *   - smoothing subtracts the per-channel mean of K over all N tokens of each (batch, kv head);
 *     the channel sum is exact (int64 of K * 2^24), mean = (float)((double)sum / (N * 2^24)),
 *     K' = (float)K - mean in binary32;
 *   - Q is quantized in blocks of 128 consecutive rows, K' in blocks of 64 rows (all d channels
 *     of one head); scale = amax / 127 (binary32 division), code = clamp(rint(x / scale), -127,
 *     127), ties to even; amax == 0 gives scale 0 and codes 0;
 *   - scores are S = S_int * sQ * sK / sqrt(d); causal attention keeps key j <= query i;
 *   - grouped-query attention maps query head h to kv head h / (H / Hkv).
 *
 * Conventions for every entry point:
 *   - All tensors are contiguous row-major device buffers owned by the caller:
 *       q, out      fp16 [B, H,   N, d]
 *       k, v        fp16 [B, Hkv, N, d]
 *       q_i8        int8 [B, H,   N, d]      q_scale float [B, H,   ceil(N/128)]
 *       k_i8        int8 [B, Hkv, N, d]      k_scale float [B, Hkv, ceil(N/64)]
 *       k_mean      float [B, Hkv, d]
 *     The library never frees or retains a caller pointer.
 *   - Supported: d in {64, 128}; 1 <= N <= 1048576; H % Hkv == 0; every pointer 16-byte aligned.
 *     Inputs must be finite (NaN/Inf give undefined results).
 *   - Arguments are checked on the host before anything is launched; a failed check returns an
 *     error status and launches nothing.  All work is asynchronous on `stream` (0 = legacy default
 *     stream) unless an entry point says otherwise.  Launch failures return QATTN_ERR_CUDA.
 *   - Every wait inside a kernel is bounded; a wait that runs out records QATTN_ERR_TIMEOUT in a
 *     device status word that qattn_check_device_status() reads.
 */
#ifndef QATTN_H
#define QATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t, declared here so that the header needs no CUDA header. */
typedef struct CUstream_st* qattn_stream_t;

typedef enum {
    QATTN_OK = 0,
    QATTN_ERR_INVALID_ARG = 1,   /* null pointer, non-positive size, H % Hkv != 0 */
    QATTN_ERR_UNSUPPORTED = 2,   /* d not in {64, 128}, N out of range, no sm_100 device */
    QATTN_ERR_MISALIGNED = 3,    /* a pointer is not 16-byte aligned */
    QATTN_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed */
    QATTN_ERR_TIMEOUT = 5,       /* a bounded wait inside a kernel ran out (device status) */
    QATTN_ERR_WORKSPACE = 6      /* workspace missing or smaller than required */
} qattn_status;

/* Static text for a status code (never NULL). */
const char* qattn_status_string(int status);

/* Library version, major * 10000 + minor * 100 + patch. */
int qattn_version(void);

/* ------------------------------------------------------------------------------------------
 * Pre-processing: smoothing of K and per-block INT8 quantization of Q and K' (page sec. 3).
 * ------------------------------------------------------------------------------------------ */

/* Bytes of device workspace qattn_smooth_quant needs (the exact int64 channel sums). */
size_t qattn_smooth_quant_workspace(int B, int Hkv, int d);

/* Smooths K and quantizes Q and K'.  Writes q_i8, q_scale, k_i8, k_scale and, when k_mean is
 * not NULL, the per-channel means.  ws: caller-owned device buffer of at least
 * qattn_smooth_quant_workspace() bytes (256-byte alignment recommended), clobbered.  The codes
 * and scales are bit-exact functions of the inputs (no dependence on launch order). */
qattn_status qattn_smooth_quant(const void* q, const void* k, int B, int H, int Hkv, int N, int d,
                                int8_t* q_i8, float* q_scale, int8_t* k_i8, float* k_scale,
                                float* k_mean, void* ws, size_t ws_bytes, qattn_stream_t stream);

/* Same as qattn_smooth_quant, but it allocates nothing and takes no workspace: for callers that
 * cannot allocate device memory at call time, e.g. runtimes whose device memory is entirely
 * reserved and sub-allocated by their own allocator, or code that must not add an allocation (and
 * the synchronization it may bring) to the stream.  The pages have no counterpart: this is an
 * interface convenience of this library.
 *  - Scratch: the exact int64 channel sums live in a fixed device array inside the library,
 *    65536 entries (512 KiB) on every GPU that loads it, held until the process exits.  Calls
 *    with B * Hkv * d > 65536 return QATTN_ERR_WORKSPACE and launch nothing.
 *  - The first call on a device looks up that array's device address (cudaGetSymbolAddress, with
 *    that device current) and caches it; make that first call before any stream capture.
 *  - All calls on a device share the array, which keeps the last call's contents; each call
 *    clears it on `stream` before use.  Calls that overlap on the GPU (different streams, no
 *    ordering between them) race on it and give wrong results: serialize them.
 *  - No cudaMalloc, cudaFree or other allocating call is made.  Results are bit-identical to
 *    qattn_smooth_quant's. */
qattn_status qattn_smooth_quant_noalloc(const void* q, const void* k, int B, int H, int Hkv, int N,
                                        int d, int8_t* q_i8, float* q_scale, int8_t* k_i8,
                                        float* k_scale, float* k_mean, qattn_stream_t stream);

/* ------------------------------------------------------------------------------------------
 * Attention on already-quantized Q and K (page sec. 3 and 4): S_int = Q_i8 K_i8^T exactly in
 * int32 on the tensor cores (tcgen05 kind::i8, accumulator in tensor memory), dequantized with
 * the block scales, blockwise online softmax in fp32, P rounded to fp16, O += P V on the tensor
 * cores (tcgen05 kind::f16, fp32 accumulator), O / l rounded to fp16.
 * causal != 0 keeps key j <= query i and skips tiles above the diagonal.
 * ------------------------------------------------------------------------------------------ */
qattn_status qattn_attn_quantized(const int8_t* q_i8, const float* q_scale, const int8_t* k_i8,
                                  const float* k_scale, const void* v, void* out, int B, int H,
                                  int Hkv, int N, int d, int causal, qattn_stream_t stream);

/* qattn_attn_quantized with the output O = sum_j P_j V_j / l in fp32 (out: device float
 * [B][H][N][d]) instead of fp16: the same kernel and arithmetic up to its last step, so
 * qattn_attn_quantized's fp16 output is exactly this output rounded to the nearest fp16.  For
 * callers that keep the attention in fp32, and for checking the attention's value apart from the
 * rounding of the fp16 output type.  Errors as qattn_attn_quantized. */
qattn_status qattn_attn_quantized_f32(const int8_t* q_i8, const float* q_scale, const int8_t* k_i8,
                                      const float* k_scale, const void* v, float* out, int B,
                                      int H, int Hkv, int N, int d, int causal,
                                      qattn_stream_t stream);

/* ------------------------------------------------------------------------------------------
 * Block-sparse attention.  The page "ThriftAttention: Selective Mixed Precision for
 * Long-Context FP4 Attention" (technical summary, method, heuristic block selection) rates each
 * (query block, key block) pair by the dot product of the blocks' mean vectors and singles out
 * the top-k pairs; its results compare against sparse top-k attention, which computes only those
 * pairs.  That sparse variant, on this library's quantized attention: query blocks of 256 rows
 * (one attention CTA), key blocks of 128 keys (one key tile).
 * ------------------------------------------------------------------------------------------ */

/* Bytes of device workspace qattn_block_select needs (binary64 block means and scores). */
size_t qattn_block_select_workspace(int B, int H, int Hkv, int N, int d);

/* Selects the key tiles each query block computes.  q [B][H][N][d], k [B][Hkv][N][d] fp16.
 * Query block i of head bh (rows 256 i .. 256 i + 255) and key tile j (keys 128 j .. 128 j + 127)
 * score qmean_i . kmean_j, where the means are exact over the block's rows that exist (< N) and
 * the dot product is a binary64 fma chain in channel order.  The list of block i holds, when
 * causal, its diagonal tiles 2i and 2i + 1 (those < ceil(N/128)), and then the topk
 * highest-scoring other tiles it may see (ties to the lower index), in ascending order.
 * Writes kv_list [B*H][ceil(N/256)][ceil(N/128)] (entries past the count are not written) and
 * kv_count [B*H][ceil(N/256)], both int32.  ws: at least qattn_block_select_workspace() bytes,
 * clobbered.  Lists are bit-exact functions of the inputs.  N <= 131072 (else
 * QATTN_ERR_UNSUPPORTED); topk < 0, or topk == 0 without causal (no tile for any block):
 * QATTN_ERR_INVALID_ARG. */
qattn_status qattn_block_select(const void* q, const void* k, int B, int H, int Hkv, int N, int d,
                                int causal, int topk, int* kv_list, int* kv_count, void* ws,
                                size_t ws_bytes, qattn_stream_t stream);

/* qattn_attn_quantized over the selected key tiles only: query rows of block i see the keys of
 * the tiles in kv_list[bh][i][0 .. kv_count[bh][i]) (and, when causal, only keys <= their own
 * index); the other tiles are neither loaded nor multiplied.  With every tile listed the result
 * equals qattn_attn_quantized's bit for bit.  Lists as written by qattn_block_select; a causal
 * list must hold its block's diagonal tiles (every row needs a key).  A query tile whose list
 * holds no tile it may see (kv_count 0) has no key to attend to: its rows are written as zeros. */
qattn_status qattn_attn_quantized_sparse(const int8_t* q_i8, const float* q_scale,
                                         const int8_t* k_i8, const float* k_scale, const void* v,
                                         void* out, int B, int H, int Hkv, int N, int d,
                                         int causal, const int* kv_list, const int* kv_count,
                                         qattn_stream_t stream);

/* The whole block-sparse forward in one call: smoothing + quantization, key-tile selection with
 * topk (qattn_block_select's rule) and the sparse attention, fp16 in, fp16 out; results equal
 * those of the three calls.  The workspace (quantized operands, selection scratch, tile lists)
 * is taken stream-ordered from the library's per-device pool and returned.  Errors as
 * qattn_block_select (topk < 0, or topk == 0 without causal, which would leave rows with no
 * key: QATTN_ERR_INVALID_ARG; N > 131072: QATTN_ERR_UNSUPPORTED) and qattn_forward. */
qattn_status qattn_forward_sparse(const void* q, const void* k, const void* v, void* out, int B,
                                  int H, int Hkv, int N, int d, int causal, int topk,
                                  qattn_stream_t stream);

/* ------------------------------------------------------------------------------------------
 * Q quantization fused into the attention kernel: an alternative split of the forward into
 * two calls.  Results are identical to qattn_smooth_quant + qattn_attn_quantized; on B200 it
 * measured slower at 32K tokens (each CTA's quantization prologue lies on its critical path), so
 * qattn_forward does not use it.
 * ------------------------------------------------------------------------------------------ */

/* K half of the pre-processing (page sec. 3): smooths K (subtracts the per-channel mean over
 * the tokens of each batch and kv head) and quantizes K' per 64-row block.  k [B][Hkv][N][d]
 * fp16; writes k_i8 [B][Hkv][N][d], k_scale [B][Hkv][ceil(N/64)] and, when not NULL, k_mean
 * [B][Hkv][d].  ws: at least qattn_smooth_quant_workspace(B, Hkv, d) bytes, clobbered.  Codes
 * and scales are bit-identical to qattn_smooth_quant's. */
qattn_status qattn_smooth_k(const void* k, int B, int Hkv, int N, int d, int8_t* k_i8,
                            float* k_scale, float* k_mean, void* ws, size_t ws_bytes,
                            qattn_stream_t stream);

/* Attention as qattn_attn_quantized, but on fp16 Q [B][H][N][d]: each CTA quantizes its own
 * 128-row Q tiles (the page's per-block INT8 quantization of Q, sec. 3: scale = amax / 127,
 * round-half-even codes, bit-identical to qattn_smooth_quant's q_i8 and q_scale) in shared
 * memory before the first Q K^T, so Q makes one trip through HBM instead of three.  k_i8 and
 * k_scale as written by qattn_smooth_k. */
qattn_status qattn_attn_fused_q(const void* q, const int8_t* k_i8, const float* k_scale,
                                const void* v, void* out, int B, int H, int Hkv, int N, int d,
                                int causal, qattn_stream_t stream);

/* ------------------------------------------------------------------------------------------
 * The whole forward: fp16 q, k, v in, fp16 out (the plug-and-play call of the page's dialogue
 * and sec. 2).  Smoothing + quantization (qattn_smooth_quant), then attention
 * (qattn_attn_quantized).
 * ------------------------------------------------------------------------------------------ */

/* Bytes of device workspace qattn_forward_ws needs (int8 Q and K, scales, channel sums). */
size_t qattn_forward_workspace(int B, int H, int Hkv, int N, int d);

/* Forward with a caller-owned workspace of at least qattn_forward_workspace() bytes. */
qattn_status qattn_forward_ws(const void* q, const void* k, const void* v, void* out, int B,
                              int H, int Hkv, int N, int d, int causal, void* ws, size_t ws_bytes,
                              qattn_stream_t stream);

/* Forward that takes its workspace, stream-ordered, from a memory pool the library keeps per
 * device (allocated on first use, reused afterwards, released at process exit). */
qattn_status qattn_forward(const void* q, const void* k, const void* v, void* out, int B, int H,
                           int Hkv, int N, int d, int causal, qattn_stream_t stream);

/* Forward on HOST buffers: copies q, k, v to the device, runs the forward, copies the result
 * back to out_host, and returns after the copy has finished (the stream is synchronized).  The
 * (batch, kv head) groups are processed in up to 8 chunks (the first and last single-group
 * chunks as two pieces of half their query heads) whose uploads, kernels (on `stream`) and
 * downloads overlap through two copy streams the library keeps per device; results are
 * identical to qattn_forward.  Device buffers come from the library's pool.  Page-locked host
 * memory gives asynchronous, overlapped copies; pageable memory works but is slower. */
qattn_status qattn_forward_host(const void* q_host, const void* k_host, const void* v_host,
                                void* out_host, int B, int H, int Hkv, int N, int d, int causal,
                                qattn_stream_t stream);

/* ------------------------------------------------------------------------------------------
 * NVFP4 quantization: the operand format of the FP4 path on the ThriftAttention page
 * ("ThriftAttention: Selective Mixed Precision for Long-Context FP4 Attention",
 * gist.science/ja/paper/2605.23081, method section, "FP4 path": the blocks not promoted to FP16
 * are computed in FP4 with Blackwell's NVFP4 micro-scaling format).  The page does not define
 * the format; this follows NVIDIA's published definition.
 * ------------------------------------------------------------------------------------------ */

/* Quantizes fp16 x [S][R][C] (S independent slices, e.g. the (batch, head) slices of Q, K or V)
 * to NVFP4: E2M1 codes, one unsigned E4M3 scale byte per 16 values, one binary32 scale per slice.
 * With binary32 operations rounded once to nearest-even:
 *   x' = (float)x - mean[s][c] (mean: binary32 [S][C], or NULL for none; the smoothing of K),
 *   g = max|x'| over the slice / 2688,
 *   per block of 16: s = E4M3(max|x'| / (6 * g)), code = E2M1(x' / (E4M3value(s) * g)),
 * both conversions nearest-even and saturating (448, 6); decoded x' ~ E2M1value * E4M3value * g.
 * A block whose scale rounds to 0 (and every block of an all-zero slice) has scale 0, codes 0;
 * a zero code is always +0.  Two codes per byte, the lower-indexed element in bits 0-3.
 *   along_rows == 0: blocks of 16 consecutive channels of a row (Q and K along d);
 *     codes uint8 [S][R][C/2], scales uint8 [S][R][C/16].
 *   along_rows != 0: blocks of 16 consecutive rows of a channel, written transposed (V along the
 *     tokens, the contraction dimension of P V); rows R .. Rp-1, Rp = R rounded up to 128 (one
 *     key tile, so that every row of codes and of scales starts 16-byte aligned), are zero
 *     padding; codes uint8 [S][C][Rp/2], scales uint8 [S][C][Rp/16].
 *   gscale: float [S], the g of each slice (also used as scratch during the call).
 * Requirements: C % 16 == 0, S <= 65535, R * C <= 2^31; all pointers device, 16-byte aligned.
 * Errors: INVALID_ARG for non-positive sizes or a NULL buffer (mean may be NULL), UNSUPPORTED
 * for the limits above, MISALIGNED, CUDA.  Three kernels and one memset on `stream`; results
 * are a deterministic function of the inputs (bit-exact against a plain CPU implementation). */
qattn_status qattn_quant_nvfp4(const void* x, const float* mean, int S, int R, int C,
                               int along_rows, uint8_t* codes, uint8_t* scales, float* gscale,
                               qattn_stream_t stream);

/* Attention on the FP4 path with FP16 promotion (ThriftAttention page, method section: the top-k
 * query-key block pairs in FP16, the rest in FP4 with NVFP4, merged by one online softmax; the
 * FP4 probability blocks quantized in two levels).
 * FP4 tiles: S = FP4 Q K^T on the block-scaled tensor cores; each tile's P row quantized as a
 * binary32 row scale gP = max p / 2688, then NVFP4 blocks of 16 keys with E4M3 scales (the same
 * binary32 steps as qattn_quant_nvfp4); O += P^ V^ on the block-scaled tensor cores, V NVFP4
 * along the tokens.  Promoted tiles (kv_list non-NULL): the key tiles listed for the query tile's
 * 256-row block (qattn_block_select's lists) run as fp16 q . (k - k_mean) on the f16 tensor cores
 * (the same smoothed keys as the FP4 tiles), fp16-rounded P, fp16 V.  l sums the P values the
 * P V product uses; out = O / l in fp16 [B][H][N][d].
 * Inputs as qattn_quant_nvfp4 writes them: q_* along the channels over B*H slices, k_* (K minus
 * k_mean) over B*Hkv slices, vt_* along the rows (transposed, Np = N rounded up to 128) over B*Hkv
 * slices.  With kv_list == NULL every tile runs in FP4 and q, k, v, k_mean, kv_count are not read;
 * otherwise q [B][H][N][d], k and v [B][Hkv][N][d] are the fp16 inputs, k_mean float [B*Hkv][d],
 * kv_list / kv_count as qattn_block_select writes them (a count above the row's ceil(N/128)
 * entries is read as that many).  Same checks and errors as qattn_attn_quantized; B * H <= 65535;
 * with kv_list, N <= 131072 (else QATTN_ERR_UNSUPPORTED). */
qattn_status qattn_attn_nvfp4(const uint8_t* q_codes, const uint8_t* q_scales, const float* q_g,
                              const uint8_t* k_codes, const uint8_t* k_scales, const float* k_g,
                              const uint8_t* vt_codes, const uint8_t* vt_scales, const float* v_g,
                              const void* q, const void* k, const void* v, const float* k_mean,
                              const int* kv_list, const int* kv_count, void* out, int B, int H,
                              int Hkv, int N, int d, int causal, qattn_stream_t stream);

/* The FP4-path forward in one call, fp16 in, fp16 out: K's channel mean (exact sums, as
 * qattn_smooth_quant), NVFP4 quantization of Q, of K minus the mean and of V along the tokens
 * (qattn_quant_nvfp4), with topk >= 0 the key-tile selection (qattn_block_select's rule) whose
 * tiles run in FP16, then qattn_attn_nvfp4.  topk == -1: every tile in FP4.  Results equal those
 * of the separate calls.  The workspace comes stream-ordered from the library's per-device pool.
 * Errors: topk < -1 QATTN_ERR_INVALID_ARG; with topk >= 0, N > 131072 QATTN_ERR_UNSUPPORTED;
 * otherwise as qattn_attn_nvfp4. */
qattn_status qattn_forward_nvfp4(const void* q, const void* k, const void* v, void* out, int B,
                                 int H, int Hkv, int N, int d, int causal, int topk,
                                 qattn_stream_t stream);

/* ------------------------------------------------------------------------------------------
 * Adaptive quantization (SageAttention summary page, aibr.jp/archives/102657: dialogue and
 * sec. 2-4 -- the quantization strength is chosen per layer or head, keeping precision where it
 * matters and speed elsewhere; +11.7 % speed without metric loss on the page).  The page names no
 * variants.  Here the choice is per (batch, kv head) group between the INT8 path above (FP16
 * P V) and a coarser variant that keeps INT8 Q K^T and runs P V in FP8 E4M3 on the tensor cores
 * (twice the FP16 rate).  FP8 variant: V is E4M3 per group (sV = max |v| / 448, code =
 * E4M3(v / sV), nearest-even, saturating, transposed); P = 2^(x - m + 4) against the running
 * maximum m, which moves (rescaling O and l) when the tile maximum exceeds it by more than 4, so
 * P <= 256; P rounded to E4M3; l sums those values; out = O sV / l in fp16.
 * ------------------------------------------------------------------------------------------ */

/* E4M3 V for the FP8 variant: v fp16 [B][Hkv][N][d] -> vt8 [B*Hkv][d][Np] bytes (Np = N rounded
 * up to 128; rows N .. Np-1 zero; a zero code is +0) and v_scale float [B*Hkv] (sV of each
 * group).  Every binary32 step rounds once; codes and scales are a deterministic function of v.
 * Errors as qattn_smooth_k; B * Hkv <= 65535. */
qattn_status qattn_quant_v_fp8(const void* v, int B, int Hkv, int N, int d, uint8_t* vt8,
                               float* v_scale, qattn_stream_t stream);

/* qattn_attn_quantized with P V in FP8 (every group): q_i8 / q_scale / k_i8 / k_scale as
 * qattn_smooth_quant writes them, vt8 / v_scale as qattn_quant_v_fp8 writes them; fp16 out
 * [B][H][N][d].  P V runs as tcgen05.mma kind::f8f6f4 (E4M3 P from tensor memory, E4M3 V^T from
 * shared memory, f32 accumulator).  Errors as qattn_attn_quantized. */
qattn_status qattn_attn_quantized_pv8(const int8_t* q_i8, const float* q_scale, const int8_t* k_i8,
                                      const float* k_scale, const uint8_t* vt8,
                                      const float* v_scale, void* out, int B, int H, int Hkv,
                                      int N, int d, int causal, qattn_stream_t stream);

/* Calibration of the adaptive choice on the given (calibration) input: both variants' outputs
 * (FP16 P V and FP8 P V, on the same INT8 Q and K), then per (batch, kv head) group the cosine
 * similarity of the two over the group's rows (its H / Hkv query heads, all N rows, d channels;
 * binary64 sums); variant[g] = 1 (FP8 P V) when that cosine >= tau, else 0 (FP16 P V).
 * variant: device uint8 [B*Hkv]; cosine: device float [B*Hkv] or NULL.  Workspace (operands and
 * both outputs) from the library's per-device pool.  Errors: tau outside [-1, 2] or a NULL
 * variant QATTN_ERR_INVALID_ARG; otherwise as qattn_forward; B * Hkv <= 65535. */
qattn_status qattn_adaptive_calibrate(const void* q, const void* k, const void* v, int B, int H,
                                      int Hkv, int N, int d, int causal, float tau,
                                      uint8_t* variant, float* cosine, qattn_stream_t stream);

/* The forward with the per-group choice: smoothing + INT8 quantization of Q and K, E4M3 V, then
 * one attention launch in which each group runs the variant variant[b * Hkv + g] names (0: FP16
 * P V, the result qattn_forward gives; 1: FP8 P V, the result qattn_attn_quantized_pv8 gives), bit
 * for bit.  variant: device uint8 [B*Hkv] (e.g. from qattn_adaptive_calibrate).  Workspace from
 * the library's pool.  Errors as qattn_forward; a NULL variant QATTN_ERR_INVALID_ARG;
 * B * Hkv <= 65535. */
qattn_status qattn_forward_adaptive(const void* q, const void* k, const void* v, void* out, int B,
                                    int H, int Hkv, int N, int d, int causal,
                                    const uint8_t* variant, qattn_stream_t stream);

/* ------------------------------------------------------------------------------------------
 * Checks.
 * ------------------------------------------------------------------------------------------ */

/* int32 score tiles S_int = Q_i8 K_i8^T as the attention kernel itself computes and reads them
 * (SageAttention page, sec. 3: the integer Q K^T with 32-bit accumulation): the kernel of
 * qattn_attn_quantized (causal or not) runs for the Q-tile pairs that hold query tiles
 * qt0 .. qt0+nqt-1 of batch b, query head h, and its softmax threads store the int32 scores they
 * load from tensor memory for key tiles kt0 .. kt0+nkt-1 (128 rows each) before any masking.  V
 * and the scales are zeros from the library's pool (the int32 tiles do not depend on them).
 * s_out: device int32 [nqt*128][nkt*128], row-major; rows or columns beyond N hold the product
 * with zero-filled rows (0); with causal != 0, tiles whose key tile lies above the query tile are
 * never computed by the causal kernel and read as 0.  Errors: window outside the tiles of N, or
 * b, h out of range: QATTN_ERR_INVALID_ARG; otherwise as qattn_attn_quantized. */
qattn_status qattn_debug_qk_int32(const int8_t* q_i8, const int8_t* k_i8, int32_t* s_out, int B,
                                  int H, int Hkv, int N, int d, int causal, int b, int h, int qt0,
                                  int nqt, int kt0, int nkt, qattn_stream_t stream);

/* FP4 score tiles through the block-scaled tensor cores: S = gQ gK * sum over the d channels of
 * E2M1(q) E4M3(sq) * E2M1(k) E4M3(sk), i.e. the dot products of the decoded NVFP4 rows, computed
 * by TMA -> tcgen05.mma kind::mxf4nvf4 (block16 UE4M3 scales in tensor memory, f32 accumulator)
 * -> tcgen05.ld: the Q K^T of the FP4 path (ThriftAttention page, method section, "FP4 path").
 * Inputs as qattn_quant_nvfp4 writes them along the channels with S = B*H slices for Q and
 * B*Hkv for K: q_codes [B*H][N][d/2], q_scales [B*H][N][d/16], q_g [B*H]; k_* likewise with Hkv.
 * Tiles as in qattn_debug_qk_int32 (query tiles qt0 .. qt0+nqt-1, key tiles kt0 .. kt0+nkt-1 of
 * batch b, query head h, its kv head h / (H / Hkv)); s_out: device float [nqt*128][nkt*128],
 * rows or keys past N read as zero. */
qattn_status qattn_debug_qk_nvfp4(const uint8_t* q_codes, const uint8_t* q_scales,
                                  const float* q_g, const uint8_t* k_codes,
                                  const uint8_t* k_scales, const float* k_g, float* s_out, int B,
                                  int H, int Hkv, int N, int d, int b, int h, int qt0, int nqt,
                                  int kt0, int nkt, qattn_stream_t stream);

/* Failure-detection check: launches one block that waits on an mbarrier nothing arrives on,
 * with a wait limit of limit_cycles SM clock cycles (0 .. the kernels' own limit of 2e9), so the
 * bounded-wait path runs out on purpose.  The kernel then records QATTN_ERR_TIMEOUT in the device
 * status word (read by qattn_check_device_status) and exits normally, leaving the context usable;
 * *gave_up (device int) is set to 1.  No page counterpart: this tests the library's own waits. */
qattn_status qattn_debug_wait_timeout(long long limit_cycles, int* gave_up,
                                      qattn_stream_t stream);

/* Synchronizes `stream`, then reports and clears the device status word: QATTN_OK, or
 * QATTN_ERR_TIMEOUT when a bounded wait inside a kernel ran out since the last check. */
qattn_status qattn_check_device_status(qattn_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* QATTN_H */
