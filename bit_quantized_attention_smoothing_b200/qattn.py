"""ctypes binding of the C ABI in include/qattn.h (argument marshalling only).

Every computation runs in the CUDA library ``libqattn.so``; there is no CPU or PyTorch fallback.
If the library is missing (or cannot be built) every call raises.  PyTorch supplies device
memory and streams.  Function names match the C entry points.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

from . import build as _build

QATTN_OK = 0
STATUS = {
    0: "QATTN_OK", 1: "QATTN_ERR_INVALID_ARG", 2: "QATTN_ERR_UNSUPPORTED",
    3: "QATTN_ERR_MISALIGNED", 4: "QATTN_ERR_CUDA", 5: "QATTN_ERR_TIMEOUT",
    6: "QATTN_ERR_WORKSPACE",
}
QBLOCK = 128
KBLOCK = 64

# Every symbol include/qattn.h declares.
EXPORTS = [
    "qattn_status_string", "qattn_version", "qattn_smooth_quant_workspace", "qattn_smooth_quant",
    "qattn_smooth_quant_noalloc",
    "qattn_attn_quantized", "qattn_attn_quantized_f32", "qattn_smooth_k", "qattn_attn_fused_q",
    "qattn_block_select_workspace", "qattn_block_select", "qattn_attn_quantized_sparse",
    "qattn_forward_sparse",
    "qattn_forward_workspace", "qattn_forward_ws", "qattn_forward",
    "qattn_forward_host", "qattn_debug_qk_int32", "qattn_debug_wait_timeout",
    "qattn_quant_nvfp4", "qattn_attn_nvfp4", "qattn_forward_nvfp4", "qattn_debug_qk_nvfp4",
    "qattn_quant_v_fp8", "qattn_attn_quantized_pv8", "qattn_adaptive_calibrate",
    "qattn_forward_adaptive", "qattn_check_device_status",
]


class QattnError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {STATUS.get(status, status)} "
                         f"({_lib().qattn_status_string(status).decode()})")


_L = None


def library_path() -> str:
    return _build.LIB


def _lib():
    global _L
    if _L is None:
        if _build.stale():
            if not os.path.exists(_build.NVCC):
                raise RuntimeError("libqattn.so is missing or stale and nvcc is not available")
            _build.build()
        L = ctypes.CDLL(_build.LIB)
        P, i, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        L.qattn_status_string.argtypes = [i]
        L.qattn_status_string.restype = ctypes.c_char_p
        L.qattn_version.argtypes = []
        L.qattn_version.restype = i
        L.qattn_smooth_quant_workspace.argtypes = [i, i, i]
        L.qattn_smooth_quant_workspace.restype = sz
        L.qattn_smooth_quant.argtypes = [P, P, i, i, i, i, i, P, P, P, P, P, P, sz, P]
        L.qattn_smooth_quant.restype = i
        L.qattn_smooth_quant_noalloc.argtypes = [P, P, i, i, i, i, i, P, P, P, P, P, P]
        L.qattn_smooth_quant_noalloc.restype = i
        L.qattn_attn_quantized.argtypes = [P, P, P, P, P, P, i, i, i, i, i, i, P]
        L.qattn_attn_quantized.restype = i
        L.qattn_attn_quantized_f32.argtypes = [P, P, P, P, P, P, i, i, i, i, i, i, P]
        L.qattn_attn_quantized_f32.restype = i
        L.qattn_smooth_k.argtypes = [P, i, i, i, i, P, P, P, P, sz, P]
        L.qattn_smooth_k.restype = i
        L.qattn_attn_fused_q.argtypes = [P, P, P, P, P, i, i, i, i, i, i, P]
        L.qattn_attn_fused_q.restype = i
        L.qattn_block_select_workspace.argtypes = [i, i, i, i, i]
        L.qattn_block_select_workspace.restype = sz
        L.qattn_block_select.argtypes = [P, P, i, i, i, i, i, i, i, P, P, P, sz, P]
        L.qattn_block_select.restype = i
        L.qattn_attn_quantized_sparse.argtypes = [P, P, P, P, P, P, i, i, i, i, i, i, P, P, P]
        L.qattn_attn_quantized_sparse.restype = i
        L.qattn_forward_sparse.argtypes = [P, P, P, P, i, i, i, i, i, i, i, P]
        L.qattn_forward_sparse.restype = i
        L.qattn_forward_workspace.argtypes = [i, i, i, i, i]
        L.qattn_forward_workspace.restype = sz
        L.qattn_forward_ws.argtypes = [P, P, P, P, i, i, i, i, i, i, P, sz, P]
        L.qattn_forward_ws.restype = i
        L.qattn_forward.argtypes = [P, P, P, P, i, i, i, i, i, i, P]
        L.qattn_forward.restype = i
        L.qattn_forward_host.argtypes = [P, P, P, P, i, i, i, i, i, i, P]
        L.qattn_forward_host.restype = i
        L.qattn_debug_qk_int32.argtypes = [P, P, P, i, i, i, i, i, i, i, i, i, i, i, i, P]
        L.qattn_debug_qk_int32.restype = i
        L.qattn_debug_wait_timeout.argtypes = [ctypes.c_longlong, P, P]
        L.qattn_debug_wait_timeout.restype = i
        L.qattn_quant_nvfp4.argtypes = [P, P, i, i, i, i, P, P, P, P]
        L.qattn_quant_nvfp4.restype = i
        L.qattn_attn_nvfp4.argtypes = [P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P,
                                       i, i, i, i, i, i, P]
        L.qattn_attn_nvfp4.restype = i
        L.qattn_forward_nvfp4.argtypes = [P, P, P, P, i, i, i, i, i, i, i, P]
        L.qattn_forward_nvfp4.restype = i
        L.qattn_debug_qk_nvfp4.argtypes = [P, P, P, P, P, P, P, i, i, i, i, i, i, i, i, i, i, i, P]
        L.qattn_debug_qk_nvfp4.restype = i
        L.qattn_quant_v_fp8.argtypes = [P, i, i, i, i, P, P, P]
        L.qattn_quant_v_fp8.restype = i
        L.qattn_attn_quantized_pv8.argtypes = [P, P, P, P, P, P, P, i, i, i, i, i, i, P]
        L.qattn_attn_quantized_pv8.restype = i
        L.qattn_adaptive_calibrate.argtypes = [P, P, P, i, i, i, i, i, i, ctypes.c_float, P, P, P]
        L.qattn_adaptive_calibrate.restype = i
        L.qattn_forward_adaptive.argtypes = [P, P, P, P, i, i, i, i, i, i, P, P]
        L.qattn_forward_adaptive.restype = i
        L.qattn_check_device_status.argtypes = [P]
        L.qattn_check_device_status.restype = i
        _L = L
    return _L


def load():
    """Loads (building if needed) the CUDA library; returns the ctypes handle."""
    return _lib()


def _p(t: Optional[torch.Tensor]):
    if t is None:
        return None
    assert t.is_contiguous(), "tensors must be contiguous"
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _check(fn: str, st: int):
    if st != QATTN_OK:
        raise QattnError(fn, st)


def _dims(q: torch.Tensor, k: torch.Tensor):
    B, H, N, d = q.shape
    Hkv = k.shape[1]
    return B, H, Hkv, N, d


# ------------------------------------------------------------------------------------------------

def qattn_smooth_quant_workspace(B: int, Hkv: int, d: int) -> int:
    return int(_lib().qattn_smooth_quant_workspace(B, Hkv, d))


def qattn_smooth_quant(q, k, q_i8=None, q_scale=None, k_i8=None, k_scale=None, k_mean=None,
                       ws=None, stream=None, want_mean=True):
    """Smooths K and quantizes Q, K' on the GPU.  Allocates missing outputs with torch; returns
    (q_i8, q_scale, k_i8, k_scale, k_mean)."""
    B, H, Hkv, N, d = _dims(q, k)
    dev = q.device
    nqb, nkb = -(-N // QBLOCK), -(-N // KBLOCK)
    q_i8 = torch.empty(B, H, N, d, dtype=torch.int8, device=dev) if q_i8 is None else q_i8
    k_i8 = torch.empty(B, Hkv, N, d, dtype=torch.int8, device=dev) if k_i8 is None else k_i8
    q_scale = torch.empty(B, H, nqb, dtype=torch.float32, device=dev) if q_scale is None else q_scale
    k_scale = torch.empty(B, Hkv, nkb, dtype=torch.float32, device=dev) if k_scale is None else k_scale
    if k_mean is None and want_mean:
        k_mean = torch.empty(B, Hkv, d, dtype=torch.float32, device=dev)
    wsb = qattn_smooth_quant_workspace(B, Hkv, d)
    if ws is None:
        ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device=dev)
    st = _lib().qattn_smooth_quant(_p(q), _p(k), B, H, Hkv, N, d, _p(q_i8), _p(q_scale), _p(k_i8),
                                   _p(k_scale), _p(k_mean), _p(ws), ws.numel(), _stream(stream))
    _check("qattn_smooth_quant", st)
    return q_i8, q_scale, k_i8, k_scale, k_mean


def qattn_smooth_quant_noalloc(q, k, q_i8, q_scale, k_i8, k_scale, k_mean=None, stream=None):
    """qattn_smooth_quant without a workspace or any allocation: the caller passes every output
    buffer, and the library's fixed device scratch (B*Hkv*d <= 65536) holds the channel sums.
    For callers that cannot allocate device memory at call time.  Every buffer is checked for
    dtype, device and size first: the library writes them without knowing their sizes."""
    B, H, Hkv, N, d = _dims(q, k)
    nqb, nkb = -(-N // QBLOCK), -(-N // KBLOCK)
    want = [("q_i8", q_i8, torch.int8, B * H * N * d), ("q_scale", q_scale, torch.float32, B * H * nqb),
            ("k_i8", k_i8, torch.int8, B * Hkv * N * d), ("k_scale", k_scale, torch.float32, B * Hkv * nkb)]
    if k_mean is not None:
        want.append(("k_mean", k_mean, torch.float32, B * Hkv * d))
    for name, t, dt, n in want:
        if t.dtype != dt or t.device != q.device or t.numel() != n:
            raise ValueError(f"{name}: need {dt} with {n} elements on {q.device}, got {t.dtype} "
                             f"with {t.numel()} on {t.device}")
    st = _lib().qattn_smooth_quant_noalloc(_p(q), _p(k), B, H, Hkv, N, d, _p(q_i8), _p(q_scale),
                                           _p(k_i8), _p(k_scale), _p(k_mean), _stream(stream))
    _check("qattn_smooth_quant_noalloc", st)
    return q_i8, q_scale, k_i8, k_scale, k_mean


def qattn_attn_quantized(q_i8, q_scale, k_i8, k_scale, v, out=None, causal=False, stream=None):
    B, H, Hkv, N, d = _dims(q_i8, k_i8)
    out = torch.empty(B, H, N, d, dtype=torch.float16, device=v.device) if out is None else out
    st = _lib().qattn_attn_quantized(_p(q_i8), _p(q_scale), _p(k_i8), _p(k_scale), _p(v), _p(out),
                                     B, H, Hkv, N, d, int(bool(causal)), _stream(stream))
    _check("qattn_attn_quantized", st)
    return out


def qattn_attn_quantized_f32(q_i8, q_scale, k_i8, k_scale, v, out=None, causal=False, stream=None):
    """qattn_attn_quantized with an fp32 output (the fp16 output is exactly its nearest fp16)."""
    B, H, Hkv, N, d = _dims(q_i8, k_i8)
    out = torch.empty(B, H, N, d, dtype=torch.float32, device=v.device) if out is None else out
    st = _lib().qattn_attn_quantized_f32(_p(q_i8), _p(q_scale), _p(k_i8), _p(k_scale), _p(v),
                                         _p(out), B, H, Hkv, N, d, int(bool(causal)),
                                         _stream(stream))
    _check("qattn_attn_quantized_f32", st)
    return out


def qattn_smooth_k(k, k_i8=None, k_scale=None, k_mean=None, ws=None, stream=None):
    """K half of the pre-processing: smoothing and per-64-row-block INT8 quantization of K.
    Returns (k_i8, k_scale, k_mean); k_mean is only written when passed."""
    B, Hkv, N, d = k.shape
    dev = k.device
    nkb = -(-N // KBLOCK)
    k_i8 = torch.empty(B, Hkv, N, d, dtype=torch.int8, device=dev) if k_i8 is None else k_i8
    k_scale = torch.empty(B, Hkv, nkb, dtype=torch.float32, device=dev) if k_scale is None else k_scale
    wsb = qattn_smooth_quant_workspace(B, Hkv, d)
    if ws is None:
        ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device=dev)
    st = _lib().qattn_smooth_k(_p(k), B, Hkv, N, d, _p(k_i8), _p(k_scale), _p(k_mean), _p(ws),
                               ws.numel(), _stream(stream))
    _check("qattn_smooth_k", st)
    return k_i8, k_scale, k_mean


def qattn_attn_fused_q(q, k_i8, k_scale, v, out=None, causal=False, stream=None):
    """Attention on fp16 Q (quantized inside the kernel) and qattn_smooth_k's int8 K."""
    B, H, Hkv, N, d = _dims(q, k_i8)
    out = torch.empty(B, H, N, d, dtype=torch.float16, device=v.device) if out is None else out
    st = _lib().qattn_attn_fused_q(_p(q), _p(k_i8), _p(k_scale), _p(v), _p(out), B, H, Hkv, N, d,
                                   int(bool(causal)), _stream(stream))
    _check("qattn_attn_fused_q", st)
    return out


def qattn_block_select_workspace(B: int, H: int, Hkv: int, N: int, d: int) -> int:
    return int(_lib().qattn_block_select_workspace(B, H, Hkv, N, d))


def qattn_block_select(q, k, topk, causal=False, kv_list=None, kv_count=None, ws=None,
                       stream=None):
    """Key tiles per 256-row query block by the block-mean score, top-k (plus the causal
    diagonals).  Returns (kv_list int32 [B*H, nsb, nkt], kv_count int32 [B*H, nsb])."""
    B, H, Hkv, N, d = _dims(q, k)
    nsb, nkt = -(-N // 256), -(-N // 128)
    dev = q.device
    kv_list = torch.full((B * H, nsb, nkt), -1, dtype=torch.int32, device=dev) if kv_list is None else kv_list
    kv_count = torch.empty(B * H, nsb, dtype=torch.int32, device=dev) if kv_count is None else kv_count
    wsb = int(_lib().qattn_block_select_workspace(B, H, Hkv, N, d))
    if ws is None:
        ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device=dev)
    st = _lib().qattn_block_select(_p(q), _p(k), B, H, Hkv, N, d, int(bool(causal)), int(topk),
                                   _p(kv_list), _p(kv_count), _p(ws), ws.numel(), _stream(stream))
    _check("qattn_block_select", st)
    return kv_list, kv_count


def qattn_forward_sparse(q, k, v, topk, out=None, causal=False, stream=None):
    """The whole block-sparse forward (smoothing + quantization, top-k key-tile selection,
    sparse attention) in one call; fp16 in, fp16 out."""
    B, H, Hkv, N, d = _dims(q, k)
    out = torch.empty(B, H, N, d, dtype=torch.float16, device=q.device) if out is None else out
    st = _lib().qattn_forward_sparse(_p(q), _p(k), _p(v), _p(out), B, H, Hkv, N, d,
                                     int(bool(causal)), int(topk), _stream(stream))
    _check("qattn_forward_sparse", st)
    return out


def qattn_attn_quantized_sparse(q_i8, q_scale, k_i8, k_scale, v, kv_list, kv_count, out=None,
                                causal=False, stream=None):
    """qattn_attn_quantized over the listed key tiles only."""
    B, H, Hkv, N, d = _dims(q_i8, k_i8)
    out = torch.empty(B, H, N, d, dtype=torch.float16, device=v.device) if out is None else out
    st = _lib().qattn_attn_quantized_sparse(_p(q_i8), _p(q_scale), _p(k_i8), _p(k_scale), _p(v),
                                            _p(out), B, H, Hkv, N, d, int(bool(causal)),
                                            _p(kv_list), _p(kv_count), _stream(stream))
    _check("qattn_attn_quantized_sparse", st)
    return out


def qattn_quant_nvfp4(x, mean=None, along_rows=False, stream=None):
    """NVFP4 quantization of fp16 x [S, R, C] (optionally minus mean, float32 [S, C]).

    Returns (codes, scales, gscale): uint8 codes with two E2M1 codes per byte, uint8 E4M3 block
    scales, float32 [S] slice scales.  along_rows=False: 16-blocks along C, codes [S, R, C/2],
    scales [S, R, C/16]; along_rows=True: 16-blocks along R, transposed and zero-padded to
    Rp = 128 * ceil(R / 128): codes [S, C, Rp/2], scales [S, C, Rp/16]."""
    assert x.dim() == 3 and x.dtype == torch.float16, "x: fp16 [S, R, C]"
    S, R, C = x.shape
    if mean is not None:
        assert mean.dtype == torch.float32 and tuple(mean.shape) == (S, C), "mean: float32 [S, C]"
    dev = x.device
    if along_rows:
        Rp = -(-R // 128) * 128
        codes = torch.empty(S, C, Rp // 2, dtype=torch.uint8, device=dev)
        scales = torch.empty(S, C, Rp // 16, dtype=torch.uint8, device=dev)
    else:
        codes = torch.empty(S, R, C // 2, dtype=torch.uint8, device=dev)
        scales = torch.empty(S, R, max(C // 16, 1), dtype=torch.uint8, device=dev)
    gscale = torch.empty(S, dtype=torch.float32, device=dev)
    st = _lib().qattn_quant_nvfp4(_p(x), _p(mean), S, R, C, int(bool(along_rows)), _p(codes),
                                  _p(scales), _p(gscale), _stream(stream))
    _check("qattn_quant_nvfp4", st)
    return codes, scales, gscale


def qattn_forward_workspace(B: int, H: int, Hkv: int, N: int, d: int) -> int:
    return int(_lib().qattn_forward_workspace(B, H, Hkv, N, d))


def qattn_forward_ws(q, k, v, out=None, causal=False, ws=None, stream=None):
    B, H, Hkv, N, d = _dims(q, k)
    out = torch.empty_like(q) if out is None else out
    if ws is None:
        ws = torch.empty(qattn_forward_workspace(B, H, Hkv, N, d), dtype=torch.uint8,
                         device=q.device)
    st = _lib().qattn_forward_ws(_p(q), _p(k), _p(v), _p(out), B, H, Hkv, N, d,
                                 int(bool(causal)), _p(ws), ws.numel(), _stream(stream))
    _check("qattn_forward_ws", st)
    return out


def qattn_forward(q, k, v, out=None, causal=False, stream=None):
    """The plug-and-play forward: fp16 q [B,H,N,d], k/v [B,Hkv,N,d] on the GPU -> fp16 out."""
    B, H, Hkv, N, d = _dims(q, k)
    out = torch.empty_like(q) if out is None else out
    st = _lib().qattn_forward(_p(q), _p(k), _p(v), _p(out), B, H, Hkv, N, d, int(bool(causal)),
                              _stream(stream))
    _check("qattn_forward", st)
    return out


def qattn_forward_host(q, k, v, out=None, causal=False, stream=None):
    """Forward on host (CPU, preferably pinned) fp16 tensors; returns after out_host is filled."""
    B, H, Hkv, N, d = _dims(q, k)
    out = torch.empty_like(q) if out is None else out
    st = _lib().qattn_forward_host(_p(q), _p(k), _p(v), _p(out), B, H, Hkv, N, d,
                                   int(bool(causal)), _stream(stream))
    _check("qattn_forward_host", st)
    return out


def qattn_debug_qk_int32(q_i8, k_i8, b, h, qt0, nqt, kt0, nkt, causal=False, s_out=None,
                         stream=None):
    """int32 score tiles as the attention kernel (causal or not) loads them from tensor memory:
    int32 [nqt*128, nkt*128] for query tiles qt0.. and key tiles kt0.. of batch b, head h."""
    B, H, Hkv, N, d = _dims(q_i8, k_i8)
    if s_out is None:
        s_out = torch.empty(nqt * 128, nkt * 128, dtype=torch.int32, device=q_i8.device)
    st = _lib().qattn_debug_qk_int32(_p(q_i8), _p(k_i8), _p(s_out), B, H, Hkv, N, d,
                                     int(bool(causal)), b, h, qt0, nqt, kt0, nkt, _stream(stream))
    _check("qattn_debug_qk_int32", st)
    return s_out


def qattn_attn_nvfp4(q_nvfp4, k_nvfp4, vt_nvfp4, B, H, Hkv, N, d, causal=False, out=None,
                     promote=None, stream=None):
    """FP4-path attention from NVFP4 operands (each the (codes, scales, gscale) triple of
    qattn_quant_nvfp4: Q and smoothed K along the channels, V along the tokens); fp16 out
    [B, H, N, d].  promote = (q, k, v, k_mean, kv_list, kv_count): fp16 inputs, the mean K was
    smoothed with, and qattn_block_select's lists of the key tiles to compute in FP16."""
    qc, qs, qg = q_nvfp4
    kc, ks, kg = k_nvfp4
    vc, vs, vg = vt_nvfp4
    if out is None:
        out = torch.empty(B, H, N, d, dtype=torch.float16, device=qc.device)
    pq = pk = pv = pm = pl = pc = None
    if promote is not None:
        pq, pk, pv, pm, pl, pc = promote
    st = _lib().qattn_attn_nvfp4(_p(qc), _p(qs), _p(qg), _p(kc), _p(ks), _p(kg), _p(vc), _p(vs),
                                 _p(vg), _p(pq), _p(pk), _p(pv), _p(pm), _p(pl), _p(pc), _p(out),
                                 B, H, Hkv, N, d, int(bool(causal)), _stream(stream))
    _check("qattn_attn_nvfp4", st)
    return out


def qattn_forward_nvfp4(q, k, v, topk=-1, out=None, causal=False, stream=None):
    """The FP4-path forward in one call (smoothing, NVFP4 operands, optional top-k FP16
    promotion, attention); fp16 in, fp16 out."""
    B, H, Hkv, N, d = _dims(q, k)
    out = torch.empty(B, H, N, d, dtype=torch.float16, device=q.device) if out is None else out
    st = _lib().qattn_forward_nvfp4(_p(q), _p(k), _p(v), _p(out), B, H, Hkv, N, d,
                                    int(bool(causal)), int(topk), _stream(stream))
    _check("qattn_forward_nvfp4", st)
    return out


def qattn_debug_qk_nvfp4(q_nvfp4, k_nvfp4, B, H, Hkv, N, d, b, h, qt0, nqt, kt0, nkt,
                         s_out=None, stream=None):
    """FP4 score tiles from NVFP4 Q and K, each the (codes, scales, gscale) triple that
    qattn_quant_nvfp4 returns along the channels (slices B*H for Q, B*Hkv for K)."""
    qc, qs, qg = q_nvfp4
    kc, ks, kg = k_nvfp4
    if s_out is None:
        s_out = torch.empty(nqt * 128, nkt * 128, dtype=torch.float32, device=qc.device)
    st = _lib().qattn_debug_qk_nvfp4(_p(qc), _p(qs), _p(qg), _p(kc), _p(ks), _p(kg), _p(s_out),
                                     B, H, Hkv, N, d, b, h, qt0, nqt, kt0, nkt, _stream(stream))
    _check("qattn_debug_qk_nvfp4", st)
    return s_out


def qattn_quant_v_fp8(v, stream=None):
    """E4M3 V of the FP8 P V variant: v fp16 [B, Hkv, N, d] -> (vt8 uint8 [B*Hkv, d, Np],
    v_scale float32 [B*Hkv]), Np = N rounded up to 128."""
    B, Hkv, N, d = v.shape
    Np = -(-N // 128) * 128
    vt8 = torch.empty(B * Hkv, d, Np, dtype=torch.uint8, device=v.device)
    vs = torch.empty(B * Hkv, dtype=torch.float32, device=v.device)
    _check("qattn_quant_v_fp8", _lib().qattn_quant_v_fp8(_p(v), B, Hkv, N, d, _p(vt8), _p(vs),
                                                          _stream(stream)))
    return vt8, vs


def qattn_attn_quantized_pv8(q_i8, q_scale, k_i8, k_scale, vt8, v_scale, out=None, causal=False,
                             stream=None):
    """Attention on int8 Q, K with P V in FP8 E4M3 (vt8, v_scale from qattn_quant_v_fp8)."""
    B, H, Hkv, N, d = _dims(q_i8, k_i8)
    out = torch.empty(B, H, N, d, dtype=torch.float16, device=q_i8.device) if out is None else out
    st = _lib().qattn_attn_quantized_pv8(_p(q_i8), _p(q_scale), _p(k_i8), _p(k_scale), _p(vt8),
                                         _p(v_scale), _p(out), B, H, Hkv, N, d,
                                         int(bool(causal)), _stream(stream))
    _check("qattn_attn_quantized_pv8", st)
    return out


def qattn_adaptive_calibrate(q, k, v, tau, causal=False, variant=None, cosine=None, stream=None):
    """Per (batch, kv head) group: cosine of the FP8-P V output against the FP16-P V output on
    this input, and variant = cosine >= tau.  Returns (variant uint8 [B*Hkv], cosine float32
    [B*Hkv])."""
    B, H, Hkv, N, d = _dims(q, k)
    dev = q.device
    variant = torch.empty(B * Hkv, dtype=torch.uint8, device=dev) if variant is None else variant
    cosine = torch.empty(B * Hkv, dtype=torch.float32, device=dev) if cosine is None else cosine
    st = _lib().qattn_adaptive_calibrate(_p(q), _p(k), _p(v), B, H, Hkv, N, d, int(bool(causal)),
                                         float(tau), _p(variant), _p(cosine), _stream(stream))
    _check("qattn_adaptive_calibrate", st)
    return variant, cosine


def qattn_forward_adaptive(q, k, v, variant, out=None, causal=False, stream=None):
    """The forward with each (batch, kv head) group on the variant variant[b * Hkv + g] names
    (0: FP16 P V, 1: FP8 P V); fp16 in, fp16 out."""
    B, H, Hkv, N, d = _dims(q, k)
    out = torch.empty_like(q) if out is None else out
    st = _lib().qattn_forward_adaptive(_p(q), _p(k), _p(v), _p(out), B, H, Hkv, N, d,
                                       int(bool(causal)), _p(variant), _stream(stream))
    _check("qattn_forward_adaptive", st)
    return out


def qattn_debug_wait_timeout(limit_cycles: int, stream=None) -> int:
    """Runs the deliberately unsatisfied bounded wait; returns 1 if the kernel gave up."""
    flag = torch.full((4,), -1, dtype=torch.int32, device="cuda")
    _check("qattn_debug_wait_timeout",
           _lib().qattn_debug_wait_timeout(int(limit_cycles), _p(flag), _stream(stream)))
    return int(flag[0].item())


def qattn_check_device_status(stream=None) -> int:
    return int(_lib().qattn_check_device_status(_stream(stream)))
