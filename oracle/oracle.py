"""Python wrapper of the CPU oracle (``qattn_oracle.c``) for the smoothed-K INT8 attention forward.

TEST INFRASTRUCTURE ONLY: the test suite, the package smoke check and the benchmark's CPU-baseline
leg are the only callers.  The product (the CUDA library and its Python binding) never imports
this module.

The C source states the method and the readings it follows (SageAttention summary page,
aibr.jp/archives/102657, sec. 2-4).  This wrapper marshals numpy arrays; every step of the INT8
path's arithmetic is in the C file.  The NVFP4 quantizer is in the C file too; decoding NVFP4 data
and the FP4 score product (decode, then a float64 matmul) are the numpy functions at the end.
fp16 arrays travel as their uint16 bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "qattn_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

QBLOCK = 128  # Q quantization block (rows)
KBLOCK = 64   # K quantization block (rows)

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2 -ffp-contract=off, no fast-math) if it is stale."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        cmd = ["gcc", "-std=c11", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
               "-pthread", "-Wall", "-o", tmp, _SRC, "-lm"]
        subprocess.check_call(cmd)
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i = ctypes.c_int
        L.oracle_f16_to_f64.argtypes = [ctypes.c_uint16]
        L.oracle_f16_to_f64.restype = ctypes.c_double
        L.oracle_f64_to_f16.argtypes = [ctypes.c_double]
        L.oracle_f64_to_f16.restype = ctypes.c_uint16
        L.oracle_k_channel_sums.argtypes = [P, i, i, i, i, P]
        L.oracle_k_channel_sums.restype = None
        L.oracle_mean_from_sum.argtypes = [ctypes.c_int64, i]
        L.oracle_mean_from_sum.restype = ctypes.c_float
        L.oracle_quantize_block.argtypes = [P, i, i, P]
        L.oracle_quantize_block.restype = ctypes.c_float
        L.oracle_smooth_quant.argtypes = [P, P, i, i, i, i, i, i, P, P, P, P, P]
        L.oracle_smooth_quant.restype = None
        L.oracle_qk_int32.argtypes = [P, P, i, i, i, i, i, i, i, i, i, i, i, P]
        L.oracle_qk_int32.restype = None
        L.oracle_attention_quantized.argtypes = [P, P, P, P, P, i, i, i, i, i, i, P, P,
                                                 ctypes.c_long, P, i]
        L.oracle_attention_quantized.restype = i
        L.oracle_attention_fp64.argtypes = [P, P, P, i, i, i, i, i, i, i, P, P, ctypes.c_long, P, i]
        L.oracle_attention_fp64.restype = i
        L.oracle_attention_quantized_sparse.argtypes = [P, P, P, P, P, i, i, i, i, i, i, P, P, P,
                                                        ctypes.c_long, P, i]
        L.oracle_attention_quantized_sparse.restype = i
        L.oracle_block_means.argtypes = [P, ctypes.c_long, i, i, i, P]
        L.oracle_block_means.restype = None
        L.oracle_block_scores.argtypes = [P, P, i, i, i, i, i, i, P]
        L.oracle_block_scores.restype = None
        L.oracle_select_blocks.argtypes = [P, i, i, i, i, i, P, P]
        L.oracle_select_blocks.restype = None
        L.oracle_e2m1_decode.argtypes = [ctypes.c_uint8]
        L.oracle_e2m1_decode.restype = ctypes.c_double
        L.oracle_e2m1_encode.argtypes = [ctypes.c_float]
        L.oracle_e2m1_encode.restype = ctypes.c_uint8
        L.oracle_ue4m3_decode.argtypes = [ctypes.c_uint8]
        L.oracle_ue4m3_decode.restype = ctypes.c_double
        L.oracle_ue4m3_encode.argtypes = [ctypes.c_float]
        L.oracle_ue4m3_encode.restype = ctypes.c_uint8
        L.oracle_quant_nvfp4.argtypes = [P, P, i, i, i, i, P, P, P]
        L.oracle_quant_nvfp4.restype = i
        L.oracle_attention_nvfp4.argtypes = [P, P, P, P, P, P, P, P, P, P, P, P, P, P,
                                             i, i, i, i, i, i, i, P, P, ctypes.c_long, P, P]
        L.oracle_attention_nvfp4.restype = i
        L.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        L.oracle_e4m3_encode.restype = ctypes.c_uint8
        L.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_decode.restype = ctypes.c_double
        L.oracle_quant_v_fp8.argtypes = [P, i, i, i, P, P]
        L.oracle_quant_v_fp8.restype = i
        L.oracle_attention_pv8.argtypes = [P, P, P, P, P, P, i, i, i, i, i, i, i, P, P,
                                           ctypes.c_long, P, P]
        L.oracle_attention_pv8.restype = i
        _lib = L
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def _bits16(x) -> np.ndarray:
    """fp16 input (numpy float16 or uint16 bit patterns) as a contiguous uint16 array."""
    x = np.ascontiguousarray(x)
    if x.dtype == np.float16:
        return x.view(np.uint16)
    assert x.dtype == np.uint16, x.dtype
    return x


def f16_to_f64(bits: int) -> float:
    return lib().oracle_f16_to_f64(int(bits))


def f64_to_f16(x: float) -> int:
    return int(lib().oracle_f64_to_f16(float(x)))


def f64_to_f16_array(x: np.ndarray) -> np.ndarray:
    f = lib().oracle_f64_to_f16
    flat = np.asarray(x, dtype=np.float64).ravel()
    return np.array([f(float(v)) for v in flat], dtype=np.uint16).reshape(np.shape(x))


def k_channel_sums(k, B, Hkv, N, d) -> np.ndarray:
    k = _bits16(k)
    out = np.zeros((B, Hkv, d), dtype=np.int64)
    lib().oracle_k_channel_sums(_ptr(k), B, Hkv, N, d, _ptr(out))
    return out


def mean_from_sum(s: int, N: int) -> np.float32:
    return np.float32(lib().oracle_mean_from_sum(int(s), int(N)))


def quantize_block(x: np.ndarray):
    """x: float32 [rows, d] -> (int8 codes [rows, d], float32 scale)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    rows, d = x.shape
    codes = np.zeros((rows, d), dtype=np.int8)
    s = lib().oracle_quantize_block(_ptr(x), rows, d, _ptr(codes))
    return codes, np.float32(s)


def smooth_quant(q, k, B, H, Hkv, N, d, smooth=True):
    """Returns dict with q_i8 [B,H,N,d], q_scale [B,H,ceil(N/128)], k_i8 [B,Hkv,N,d],
    k_scale [B,Hkv,ceil(N/64)], k_mean [B,Hkv,d] (float32)."""
    q = _bits16(q)
    k = _bits16(k)
    nqb = (N + QBLOCK - 1) // QBLOCK
    nkb = (N + KBLOCK - 1) // KBLOCK
    r = dict(
        q_i8=np.zeros((B, H, N, d), dtype=np.int8),
        q_scale=np.zeros((B, H, nqb), dtype=np.float32),
        k_i8=np.zeros((B, Hkv, N, d), dtype=np.int8),
        k_scale=np.zeros((B, Hkv, nkb), dtype=np.float32),
        k_mean=np.zeros((B, Hkv, d), dtype=np.float32),
    )
    lib().oracle_smooth_quant(_ptr(q), _ptr(k), B, H, Hkv, N, d, 1 if smooth else 0,
                              _ptr(r["q_i8"]), _ptr(r["q_scale"]), _ptr(r["k_i8"]),
                              _ptr(r["k_scale"]), _ptr(r["k_mean"]))
    return r


def qk_int32(q_i8, k_i8, B, H, Hkv, N, d, b, h, i0, ni, j0, nj) -> np.ndarray:
    q_i8 = np.ascontiguousarray(q_i8, dtype=np.int8)
    k_i8 = np.ascontiguousarray(k_i8, dtype=np.int8)
    out = np.zeros((ni, nj), dtype=np.int32)
    lib().oracle_qk_int32(_ptr(q_i8), _ptr(k_i8), B, H, Hkv, N, d, b, h, i0, ni, j0, nj, _ptr(out))
    return out


def all_rows(B, H, N):
    bh = np.repeat(np.arange(B * H, dtype=np.int64), N)
    i = np.tile(np.arange(N, dtype=np.int64), B * H)
    return bh, i


def attention_quantized(q_i8, q_scale, k_i8, k_scale, v, B, H, Hkv, N, d, causal,
                        rows=None, nthreads=0):
    """Rows of the quantized attention output (float64 [nrows, d]).  rows = (row_bh, row_i) or
    None for all rows in (b, h, i) order."""
    row_bh, row_i = all_rows(B, H, N) if rows is None else rows
    row_bh = np.ascontiguousarray(row_bh, dtype=np.int64)
    row_i = np.ascontiguousarray(row_i, dtype=np.int64)
    out = np.zeros((row_bh.size, d), dtype=np.float64)
    v = _bits16(v)
    q_i8 = np.ascontiguousarray(q_i8, dtype=np.int8)
    k_i8 = np.ascontiguousarray(k_i8, dtype=np.int8)
    q_scale = np.ascontiguousarray(q_scale, dtype=np.float32)
    k_scale = np.ascontiguousarray(k_scale, dtype=np.float32)
    lib().oracle_attention_quantized(_ptr(q_i8), _ptr(q_scale), _ptr(k_i8), _ptr(k_scale), _ptr(v),
                                     B, H, Hkv, N, d, 1 if causal else 0, _ptr(row_bh),
                                     _ptr(row_i), row_bh.size, _ptr(out), int(nthreads))
    return out


def attention_quantized_all(q_i8, q_scale, k_i8, k_scale, v, B, H, Hkv, N, d, causal,
                            chunk=2048):
    """Every row of the quantized attention output (float64 [B*H*N, d], rows in (b, h, i) order):
    the definition attention_quantized evaluates row by row in C, written here with float64
    library matmuls on the CPU (torch), one query head and up to `chunk` of its rows at a time, so
    that whole workloads finish in minutes.  Per row i of head (b, h), kv head g = h / (H / Hkv):
      S_int[i, j] = sum_c q_i8[i, c] k_i8[j, c]  (a float64 matmul of integers: every partial sum
                    is an integer below 2^53, so it is exact),
      S[i, j]     = ((S_int[i, j] * sQ[i / 128]) * sK[j / 64]) * (1 / sqrt(d)),
      keys j > i dropped when causal, P = exp(S - max_j S), O[i] = sum_j P[i, j] V[j] / sum_j P[i, j]
    (SageAttention page, sec. 3-4: the int32 product, dequantized with the two block scales, then
    the softmax and P V; the blockwise online softmax equals this plain row softmax up to rounding).
    Only the summation order of the float64 sums differs from the C loops."""
    import torch
    q_i8 = np.ascontiguousarray(q_i8, dtype=np.int8).reshape(B, H, N, d)
    k_i8 = np.ascontiguousarray(k_i8, dtype=np.int8).reshape(B, Hkv, N, d)
    q_scale = np.asarray(q_scale, dtype=np.float32).reshape(B, H, -1)
    k_scale = np.asarray(k_scale, dtype=np.float32).reshape(B, Hkv, -1)
    vv = _bits16(v).reshape(B, Hkv, N, d)
    inv_sqrt_d = 1.0 / np.sqrt(float(d))
    G = H // Hkv
    out = np.empty((B * H * N, d), dtype=np.float64)
    for b in range(B):
        for g in range(Hkv):
            K = torch.from_numpy(k_i8[b, g].astype(np.float64))
            V = torch.from_numpy(vv[b, g].view(np.float16).astype(np.float64))
            sk = torch.from_numpy(np.repeat(k_scale[b, g].astype(np.float64), KBLOCK)[:N])
            for h in range(g * G, (g + 1) * G):
                Q = q_i8[b, h]
                sq = np.repeat(q_scale[b, h].astype(np.float64), QBLOCK)[:N]
                for r0 in range(0, N, chunk):
                    r1 = min(N, r0 + chunk)
                    nk = r1 if causal else N
                    S = torch.from_numpy(Q[r0:r1].astype(np.float64)) @ K[:nk].T
                    S = S * torch.from_numpy(sq[r0:r1])[:, None]
                    S = S * sk[None, :nk]
                    S = S * inv_sqrt_d
                    if causal:
                        later = torch.arange(nk)[None, :] > torch.arange(r0, r1)[:, None]
                        S.masked_fill_(later, -np.inf)
                    P = torch.exp(S - S.max(dim=1, keepdim=True).values)
                    O = (P @ V[:nk]) / P.sum(dim=1, keepdim=True)
                    row0 = (b * H + h) * N
                    out[row0 + r0: row0 + r1] = O.numpy()
    return out


SBLOCK = 256  # block-sparse selection: query rows per selection block
KTILE = 128   # block-sparse selection: keys per key tile


def block_means(x, outer, N, d, rows_per_block):
    """Exact per-block channel means (float64 [outer, nblocks, d]) of fp16 x [outer, N, d]."""
    nb = -(-N // rows_per_block)
    out = np.zeros((outer, nb, d), dtype=np.float64)
    lib().oracle_block_means(_ptr(_bits16(x)), outer, N, d, rows_per_block, _ptr(out))
    return out


def block_scores(qmeans, kmeans, B, H, Hkv, d):
    """Importance of each (query block, key tile) pair: float64 [B*H, nsb, nkt]."""
    qmeans = np.ascontiguousarray(qmeans, dtype=np.float64)
    kmeans = np.ascontiguousarray(kmeans, dtype=np.float64)
    nsb, nkt = qmeans.shape[1], kmeans.shape[1]
    out = np.zeros((B * H, nsb, nkt), dtype=np.float64)
    lib().oracle_block_scores(_ptr(qmeans), _ptr(kmeans), B, H, Hkv, nsb, nkt, d, _ptr(out))
    return out


def select_blocks(scores, B, H, N, causal, topk):
    """(list int32 [B*H, nsb, nkt], count int32 [B*H, nsb]): the selected key tiles of each query
    block, ascending (entries past count are unused)."""
    scores = np.ascontiguousarray(scores, dtype=np.float64)
    nsb, nkt = scores.shape[1], scores.shape[2]
    lst = np.full((B * H, nsb, nkt), -1, dtype=np.int32)
    cnt = np.zeros((B * H, nsb), dtype=np.int32)
    lib().oracle_select_blocks(_ptr(scores), B, H, N, 1 if causal else 0, int(topk), _ptr(lst),
                               _ptr(cnt))
    return lst, cnt


def block_select(q, k, B, H, Hkv, N, d, causal, topk):
    """The whole selection from fp16 q, k: means, scores, top-k lists."""
    qm = block_means(q, B * H, N, d, SBLOCK)
    km = block_means(k, B * Hkv, N, d, KTILE)
    return select_blocks(block_scores(qm, km, B, H, Hkv, d), B, H, N, causal, topk)


def tile_mask(lst, cnt, N):
    """uint8 [B*H, nsb, nkt] mask of the selected key tiles."""
    nkt = -(-N // KTILE)
    mask = np.zeros(lst.shape[:2] + (nkt,), dtype=np.uint8)
    for bh in range(lst.shape[0]):
        for i in range(lst.shape[1]):
            mask[bh, i, lst[bh, i, :cnt[bh, i]]] = 1
    return mask


def attention_quantized_sparse(q_i8, q_scale, k_i8, k_scale, v, B, H, Hkv, N, d, causal, mask,
                               rows=None, nthreads=0):
    """attention_quantized with query row i of head bh seeing only the key tiles with
    mask[bh, i // 256, tile] != 0."""
    row_bh, row_i = all_rows(B, H, N) if rows is None else rows
    row_bh = np.ascontiguousarray(row_bh, dtype=np.int64)
    row_i = np.ascontiguousarray(row_i, dtype=np.int64)
    out = np.zeros((row_bh.size, d), dtype=np.float64)
    mask = np.ascontiguousarray(mask, dtype=np.uint8)
    lib().oracle_attention_quantized_sparse(
        _ptr(np.ascontiguousarray(q_i8, dtype=np.int8)), _ptr(np.ascontiguousarray(q_scale, dtype=np.float32)),
        _ptr(np.ascontiguousarray(k_i8, dtype=np.int8)), _ptr(np.ascontiguousarray(k_scale, dtype=np.float32)),
        _ptr(_bits16(v)), B, H, Hkv, N, d, 1 if causal else 0, _ptr(mask), _ptr(row_bh), _ptr(row_i),
        row_bh.size, _ptr(out), int(nthreads))
    return out


def attention_fp64(q, k, v, B, H, Hkv, N, d, causal, smooth=False, rows=None, nthreads=0):
    """Rows of the full-precision attention softmax(Q K'^T/sqrt(d)) V (float64 [nrows, d])."""
    row_bh, row_i = all_rows(B, H, N) if rows is None else rows
    row_bh = np.ascontiguousarray(row_bh, dtype=np.int64)
    row_i = np.ascontiguousarray(row_i, dtype=np.int64)
    out = np.zeros((row_bh.size, d), dtype=np.float64)
    lib().oracle_attention_fp64(_ptr(_bits16(q)), _ptr(_bits16(k)), _ptr(_bits16(v)), B, H, Hkv,
                                N, d, 1 if causal else 0, 1 if smooth else 0, _ptr(row_bh),
                                _ptr(row_i), row_bh.size, _ptr(out), int(nthreads))
    return out


def forward(q, k, v, B, H, Hkv, N, d, causal, rows=None, nthreads=0, smooth=True):
    """The whole path: smoothing + quantization, then quantized attention rows (float64)."""
    sq = smooth_quant(q, k, B, H, Hkv, N, d, smooth=smooth)
    out = attention_quantized(sq["q_i8"], sq["q_scale"], sq["k_i8"], sq["k_scale"], v,
                              B, H, Hkv, N, d, causal, rows=rows, nthreads=nthreads)
    return out, sq


# ---- NVFP4 quantization (the FP4 path's operand format; the C file states the readings) ----

def e2m1_encode(x: float) -> int:
    return int(lib().oracle_e2m1_encode(float(x)))


def e2m1_decode(code: int) -> float:
    return lib().oracle_e2m1_decode(int(code))


def ue4m3_encode(x: float) -> int:
    return int(lib().oracle_ue4m3_encode(float(x)))


def ue4m3_decode(code: int) -> float:
    return lib().oracle_ue4m3_decode(int(code))


def quant_nvfp4(x, mean=None, along_rows=False):
    """NVFP4 codes of fp16 x [S, R, C] (optionally minus mean [S, C]).

    Returns (codes uint8, scales uint8, gscale float32 [S]); codes hold two E2M1 codes per byte
    (lower index in the low nibble).  along_rows=False: 16-blocks along C, codes [S, R, C/2],
    scales [S, R, C/16].  along_rows=True: 16-blocks along R, transposed, R padded with zeros to
    Rp = 128 * ceil(R / 128): codes [S, C, Rp/2], scales [S, C, Rp/16]."""
    x = _bits16(x)
    S, R, C = x.shape
    Rp = -(-R // 128) * 128
    if along_rows:
        codes = np.zeros((S, C, Rp // 2), dtype=np.uint8)
        scales = np.zeros((S, C, Rp // 16), dtype=np.uint8)
    else:
        codes = np.zeros((S, R, C // 2), dtype=np.uint8)
        scales = np.zeros((S, R, C // 16), dtype=np.uint8)
    g = np.zeros(S, dtype=np.float32)
    mp = None if mean is None else _ptr(np.ascontiguousarray(mean, dtype=np.float32))
    rc = lib().oracle_quant_nvfp4(_ptr(x), mp, S, R, C, 1 if along_rows else 0, _ptr(codes),
                                  _ptr(scales), _ptr(g))
    if rc != 0:
        raise ValueError("oracle_quant_nvfp4: bad argument")
    return codes, scales, g


def nvfp4_dequant(codes, scales, gscale):
    """float64 values of NVFP4 data laid out as quant_nvfp4 returns it: [S, rows, 2 * bytes]."""
    e2m1 = np.array([e2m1_decode(c) for c in range(16)])
    e4m3 = np.array([ue4m3_decode(c) if c != 0x7F else np.nan for c in range(256)])
    lo = e2m1[codes & 15]
    hi = e2m1[codes >> 4]
    vals = np.stack([lo, hi], axis=-1).reshape(codes.shape[:-1] + (2 * codes.shape[-1],))
    sc = np.repeat(e4m3[scales], 16, axis=-1) * np.asarray(gscale, dtype=np.float64)[:, None, None]
    return vals * sc


def qk_nvfp4(q_codes, q_scales, q_g, k_codes, k_scales, k_g, H, Hkv, b, h, r0, nr, c0, nc):
    """FP4 scores of batch b, query head h: rows r0 .. r0+nr-1 of Q against keys c0 .. c0+nc-1
    of the kv head h // (H // Hkv), from NVFP4 data laid out as quant_nvfp4 writes it along the
    channels (slices = batch * heads).  S = sum over channels of decoded q * decoded k, i.e. per
    16-channel block the exact integer-valued product sum of the E2M1 codes times the two E4M3
    block scales, times gQ * gK; float64.  Rows or keys past the end read as zero.  Returns
    (S, M) with M = |Q| |K|^T, the magnitude sum that bounds accumulation error."""
    bh = b * H + h
    bg = b * Hkv + h // (H // Hkv)

    def rows(codes, scales, g, s, r, n):
        sl = slice(r, min(r + n, codes.shape[1]))
        x = nvfp4_dequant(codes[s:s + 1, sl], scales[s:s + 1, sl], np.asarray(g)[s:s + 1])[0]
        out = np.zeros((n, x.shape[1]))
        out[: x.shape[0]] = x
        return out

    Q = rows(q_codes, q_scales, q_g, bh, r0, nr)
    K = rows(k_codes, k_scales, k_g, bg, c0, nc)
    return Q @ K.T, np.abs(Q) @ np.abs(K).T


def attention_nvfp4(qn, kn, vn, B, H, Hkv, N, d, causal, rows=None, promote=None, q16=None,
                    k16=None, v16=None, k_mean=None):
    """Rows of the FP4-path attention (the C file states the readings).

    qn, kn: (codes, scales, gscale) along the channels over B*H and B*Hkv slices; vn: the same for
    V along the tokens (transposed).  promote: uint8 [B*H, ceil(N/256), ceil(N/128)] marking the
    key tiles computed in FP16 from q16, k16, v16 (fp16) with the smoothed keys (k_mean float32
    [B*Hkv, d]); None = every tile in FP4.  Returns (out float64 [nrows, d], slack [nrows])."""
    row_bh, row_i = all_rows(B, H, N) if rows is None else rows
    row_bh = np.ascontiguousarray(row_bh, dtype=np.int64)
    row_i = np.ascontiguousarray(row_i, dtype=np.int64)
    out = np.zeros((row_bh.size, d), dtype=np.float64)
    slack = np.zeros(row_bh.size, dtype=np.float64)
    c = lambda a, t: _ptr(np.ascontiguousarray(a, dtype=t))
    Np = vn[0].shape[2] * 2
    rc = lib().oracle_attention_nvfp4(
        c(qn[0], np.uint8), c(qn[1], np.uint8), c(qn[2], np.float32),
        c(kn[0], np.uint8), c(kn[1], np.uint8), c(kn[2], np.float32),
        c(vn[0], np.uint8), c(vn[1], np.uint8), c(vn[2], np.float32),
        None if promote is None else _ptr(_bits16(q16)),
        None if promote is None else _ptr(_bits16(k16)),
        None if promote is None else _ptr(_bits16(v16)),
        None if promote is None else c(k_mean, np.float32),
        None if promote is None else c(promote, np.uint8),
        B, H, Hkv, N, Np, d, 1 if causal else 0, _ptr(row_bh), _ptr(row_i), row_bh.size,
        _ptr(out), _ptr(slack))
    if rc != 0:
        raise ValueError("oracle_attention_nvfp4: bad argument")
    return out, slack


# ---- adaptive quantization: the FP8 (E4M3) P V variant (the C file states the readings) ----

def e4m3_encode(x: float) -> int:
    return int(lib().oracle_e4m3_encode(float(x)))


def e4m3_decode(code: int) -> float:
    return lib().oracle_e4m3_decode(int(code))


def e4m3_decode_array(codes) -> np.ndarray:
    """Values of an array of E4M3 bytes (float64), by the oracle's decoder."""
    table = np.array([e4m3_decode(c) for c in range(256)], dtype=np.float64)
    return table[np.asarray(codes, dtype=np.uint8)]


def quant_v_fp8(v):
    """E4M3 quantization of fp16 v [S, R, C] per slice, transposed: (codes uint8 [S, C, Rp],
    scale float32 [S]), Rp = R rounded up to 128."""
    v = _bits16(v)
    S, R, C = v.shape
    Rp = -(-R // 128) * 128
    codes = np.zeros((S, C, Rp), dtype=np.uint8)
    scale = np.zeros(S, dtype=np.float32)
    assert lib().oracle_quant_v_fp8(_ptr(v), S, R, C, _ptr(codes), _ptr(scale)) == 0
    return codes, scale


def attention_pv8(q_i8, q_scale, k_i8, k_scale, vt8, v_scale, B, H, Hkv, N, d, causal,
                  rows=None):
    """Rows of the attention with INT8 Q K^T and E4M3 P V (float64 [nrows, d]) and the per-row
    slack for E4M3 decisions near a tie.  vt8, v_scale as quant_v_fp8 returns them over the
    B*Hkv slices."""
    row_bh, row_i = all_rows(B, H, N) if rows is None else rows
    row_bh = np.ascontiguousarray(row_bh, dtype=np.int64)
    row_i = np.ascontiguousarray(row_i, dtype=np.int64)
    vt8 = np.ascontiguousarray(vt8, dtype=np.uint8)
    Np = vt8.shape[-1]
    out = np.zeros((row_bh.size, d), dtype=np.float64)
    slack = np.zeros(row_bh.size, dtype=np.float64)
    assert lib().oracle_attention_pv8(
        _ptr(np.ascontiguousarray(q_i8, dtype=np.int8)), _ptr(np.ascontiguousarray(q_scale, dtype=np.float32)),
        _ptr(np.ascontiguousarray(k_i8, dtype=np.int8)), _ptr(np.ascontiguousarray(k_scale, dtype=np.float32)),
        _ptr(vt8), _ptr(np.ascontiguousarray(v_scale, dtype=np.float32)), B, H, Hkv, N, Np, d,
        1 if causal else 0, _ptr(row_bh), _ptr(row_i), row_bh.size, _ptr(out), _ptr(slack)) == 0
    return out, slack


def forward_pv8(q, k, v, B, H, Hkv, N, d, causal, rows=None):
    """The FP8 P V variant's whole path: smoothing + INT8 quantization of Q and K, E4M3 V, then
    the attention rows; returns (out, slack)."""
    sq = smooth_quant(q, k, B, H, Hkv, N, d)
    vt8, vs = quant_v_fp8(_bits16(v).reshape(B * Hkv, N, d))
    return attention_pv8(sq["q_i8"], sq["q_scale"], sq["k_i8"], sq["k_scale"], vt8, vs, B, H,
                         Hkv, N, d, causal, rows=rows)
