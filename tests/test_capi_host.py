"""Host-side checks of the C ABI (no GPU needed): the library builds and loads, exports every
symbol include/qattn.h declares, and rejects bad arguments before touching the device."""
import ctypes
import os
import re

import pytest

from bit_quantized_attention_smoothing_b200 import build as B
from bit_quantized_attention_smoothing_b200 import qattn as Q

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                      "qattn.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(qattn_[a-z0-9_]+)\s*\(", text)))


def test_library_builds_and_loads():
    path = B.build()
    assert os.path.exists(path)
    Q.load()


def test_exports_every_declared_symbol():
    L = ctypes.CDLL(B.build())
    names = declared_functions()
    assert set(names) == set(Q.EXPORTS)
    for n in names:
        assert hasattr(L, n), n


def test_status_strings_and_version():
    L = Q.load()
    for code in range(7):
        assert L.qattn_status_string(code)
    assert L.qattn_status_string(99) == b"unknown status"
    assert L.qattn_version() >= 100


def test_workspace_sizes():
    L = Q.load()
    assert L.qattn_smooth_quant_workspace(1, 8, 128) == 8 * 128 * 8
    assert L.qattn_smooth_quant_workspace(0, 8, 128) == 0
    ws = L.qattn_forward_workspace(1, 32, 8, 32768, 128)
    need = 32 * 32768 * 128 + 8 * 32768 * 128 + 4 * 32 * 256 + 4 * 8 * 512 + 8 * 8 * 128
    assert need <= ws <= need + 5 * 256
    assert L.qattn_forward_workspace(1, 32, 8, 32768, 96) == 0
    assert L.qattn_forward_workspace(1, 30, 8, 32768, 128) == 0


P = ctypes.c_void_p


@pytest.mark.parametrize("args,expect", [
    ((P(16), P(32), P(48), P(64), 1, 4, 2, 256, 128, 0, None), Q.QATTN_OK - 0 + 4),  # device call
    ((None, P(32), P(48), P(64), 1, 4, 2, 256, 128, 0, None), 1),
    ((P(16), P(32), P(48), P(64), 1, 4, 3, 256, 128, 0, None), 1),
    ((P(16), P(32), P(48), P(64), 0, 4, 2, 256, 128, 0, None), 1),
    ((P(16), P(32), P(48), P(64), 1, 4, 2, 0, 128, 0, None), 1),
    ((P(16), P(32), P(48), P(64), 1, 4, 2, 256, 96, 0, None), 2),
    ((P(16), P(32), P(48), P(64), 1, 4, 2, (1 << 20) + 1, 128, 0, None), 2),
    ((P(16), P(33), P(48), P(64), 1, 4, 2, 256, 128, 0, None), 3),
])
def test_forward_argument_checks(args, expect):
    L = Q.load()
    st = L.qattn_forward(*args)
    if expect == 4:
        # valid arguments reach the device query; without a GPU that fails as a CUDA error
        import torch
        if torch.cuda.is_available():
            pytest.skip("argument check only; this box has a GPU")
        assert st == 4
    else:
        assert st == expect


def test_workspace_and_alignment_checks():
    L = Q.load()
    need = L.qattn_forward_workspace(1, 4, 2, 256, 128)
    st = L.qattn_forward_ws(P(16), P(32), P(48), P(64), 1, 4, 2, 256, 128, 1, P(4096), need - 1, None)
    assert st == 6
    st = L.qattn_forward_ws(P(16), P(32), P(48), P(64), 1, 4, 2, 256, 128, 1, None, need, None)
    assert st == 6
    st = L.qattn_forward_ws(P(16), P(32), P(48), P(64), 1, 4, 2, 256, 128, 1, P(4100), need, None)
    assert st == 3
    st = L.qattn_smooth_quant(P(16), P(32), 1, 4, 2, 256, 128, P(48), P(64), P(80), P(96), None,
                              P(112), 8, None)
    assert st == 6
    st = L.qattn_smooth_quant(P(16), P(32), 1, 4, 2, 256, 128, P(48), P(64), P(80), P(96), P(20),
                              P(112), 1 << 20, None)
    assert st == 3
    st = L.qattn_debug_qk_int32(P(16), P(32), P(48), 1, 4, 2, 256, 128, 0, 0, 0, 1, 2, 0, 1, None)
    assert st == 1
    st = L.qattn_debug_qk_int32(P(16), P(32), P(48), 1, 4, 2, 256, 128, 1, 0, 4, 0, 1, 0, 1, None)
    assert st == 1
    assert L.qattn_debug_wait_timeout(1000, None, None) == 1
    assert L.qattn_debug_wait_timeout(-1, P(16), None) == 1
    assert L.qattn_debug_wait_timeout(3_000_000_000, P(16), None) == 1


@pytest.mark.parametrize("args,expect", [
    ((None, P(32), P(48), P(64), 1, 4, 2, 256, 128, 1, 4, None), 1),     # null pointer
    ((P(16), P(32), P(48), P(64), 1, 4, 3, 256, 128, 1, 4, None), 1),    # H % Hkv != 0
    ((P(16), P(32), P(48), P(64), 1, 4, 2, 256, 128, 1, -1, None), 1),   # topk < 0
    ((P(16), P(32), P(48), P(64), 1, 4, 2, 256, 128, 0, 0, None), 1),    # no key for any row
    ((P(16), P(32), P(48), P(64), 1, 4, 2, 256, 96, 1, 4, None), 2),     # d
    ((P(16), P(32), P(48), P(64), 1, 4, 2, 131073, 128, 1, 4, None), 2), # past the selection limit
    ((P(16), P(33), P(48), P(64), 1, 4, 2, 256, 128, 1, 4, None), 3),    # misaligned
])
def test_forward_sparse_argument_checks(args, expect):
    L = Q.load()
    assert L.qattn_forward_sparse(*args) == expect


@pytest.mark.parametrize("causal,topk,expect", [(0, 0, 1), (0, -1, 1), (1, -1, 1)])
def test_block_select_rejects_empty_selections(causal, topk, expect):
    # non-causal topk 0 would list no key tile for any query block
    L = Q.load()
    st = L.qattn_block_select(P(16), P(32), 1, 4, 2, 256, 128, causal, topk, P(48), P(64),
                              P(4096), 1 << 20, None)
    assert st == expect


@pytest.mark.parametrize("bad", ["q_i8", "q_scale", "k_i8", "k_scale", "k_mean"])
def test_noalloc_binding_checks_output_buffers(bad):
    # the allocation-free entry writes caller buffers whose sizes it cannot see: the binding
    # checks dtype and size before calling it (CPU tensors here, so nothing reaches a device)
    import torch
    B, H, Hkv, N, d = 1, 4, 2, 300, 64
    q = torch.zeros(B, H, N, d, dtype=torch.float16)
    k = torch.zeros(B, Hkv, N, d, dtype=torch.float16)
    bufs = {"q_i8": torch.empty(B, H, N, d, dtype=torch.int8),
            "q_scale": torch.empty(B, H, 3, dtype=torch.float32),
            "k_i8": torch.empty(B, Hkv, N, d, dtype=torch.int8),
            "k_scale": torch.empty(B, Hkv, 5, dtype=torch.float32),
            "k_mean": torch.empty(B, Hkv, d, dtype=torch.float32)}
    t = bufs[bad]
    bufs[bad] = torch.empty(t.numel() - 1, dtype=t.dtype) if bad != "k_i8" else t.to(torch.uint8)
    with pytest.raises(ValueError, match=bad):
        Q.qattn_smooth_quant_noalloc(q, k, **bufs)


@pytest.mark.parametrize("args,expect", [
    ((None, None, 2, 64, 128, 0, P(16), P(32), P(48), None), 1),        # null x
    ((P(16), None, 2, 64, 128, 0, P(16), None, P(48), None), 1),        # null scales
    ((P(16), None, 0, 64, 128, 0, P(16), P(32), P(48), None), 1),       # S < 1
    ((P(16), None, 2, 0, 128, 1, P(16), P(32), P(48), None), 1),        # R < 1
    ((P(16), None, 2, 64, 120, 0, P(16), P(32), P(48), None), 2),       # C % 16 != 0
    ((P(16), None, 65536, 64, 128, 0, P(16), P(32), P(48), None), 2),   # S past the grid limit
    ((P(16), None, 1, 1 << 24, 256, 1, P(16), P(32), P(48), None), 2),  # R * C > 2^31
    ((P(16), P(20), 2, 64, 128, 0, P(16), P(32), P(48), None), 3),      # misaligned mean
    ((P(16), None, 2, 64, 128, 0, P(16), P(32), P(52), None), 3),       # misaligned gscale
])
def test_quant_nvfp4_argument_checks(args, expect):
    L = Q.load()
    assert L.qattn_quant_nvfp4(*args) == expect


def test_debug_qk_nvfp4_argument_checks():
    L = Q.load()
    a = (P(16), P(32), P(48), P(64), P(80), P(96), P(112))
    assert L.qattn_debug_qk_nvfp4(None, *a[1:], 1, 4, 2, 256, 128, 0, 0, 0, 1, 0, 1, None) == 1
    assert L.qattn_debug_qk_nvfp4(*a, 1, 4, 3, 256, 128, 0, 0, 0, 1, 0, 1, None) == 1    # H % Hkv
    assert L.qattn_debug_qk_nvfp4(*a, 1, 4, 2, 256, 128, 0, 0, 1, 2, 0, 1, None) == 1    # tiles
    assert L.qattn_debug_qk_nvfp4(*a, 1, 4, 2, 256, 128, 0, 4, 0, 1, 0, 1, None) == 1    # head
    assert L.qattn_debug_qk_nvfp4(*a, 1, 4, 2, 256, 96, 0, 0, 0, 1, 0, 1, None) == 2     # d
    assert L.qattn_debug_qk_nvfp4(P(17), *a[1:], 1, 4, 2, 256, 128, 0, 0, 0, 1, 0, 1, None) == 3


def test_attn_nvfp4_argument_checks():
    L = Q.load()
    a = tuple(P(16 * (i + 1)) for i in range(9))
    none6 = (None,) * 6
    prom = tuple(P(256 + 16 * i) for i in range(6))
    o = P(1024)
    assert L.qattn_attn_nvfp4(None, *a[1:], *none6, o, 1, 4, 2, 256, 128, 1, None) == 1
    assert L.qattn_attn_nvfp4(*a, *none6, o, 1, 4, 3, 256, 128, 1, None) == 1         # H % Hkv
    assert L.qattn_attn_nvfp4(*a, *none6, o, 1, 4, 2, 0, 128, 1, None) == 1           # N
    assert L.qattn_attn_nvfp4(*a, *none6, o, 1, 4, 2, 256, 96, 1, None) == 2          # d
    assert L.qattn_attn_nvfp4(*a, *none6, o, 300, 256, 2, 256, 128, 1, None) == 2    # B * H
    assert L.qattn_attn_nvfp4(*a, *none6, P(24), 1, 4, 2, 256, 128, 1, None) == 3     # out
    # promotion: lists given, an fp16 operand or the mean missing / misaligned
    assert L.qattn_attn_nvfp4(*a, None, *prom[1:], o, 1, 4, 2, 256, 128, 1, None) == 1
    assert L.qattn_attn_nvfp4(*a, *prom[:3], P(20), *prom[4:], o, 1, 4, 2, 256, 128, 1, None) == 3


@pytest.mark.parametrize("args,expect", [
    ((None, P(32), P(48), P(64), 1, 4, 2, 256, 128, 1, 4, None), 1),     # null pointer
    ((P(16), P(32), P(48), P(64), 1, 4, 3, 256, 128, 1, 4, None), 1),    # H % Hkv != 0
    ((P(16), P(32), P(48), P(64), 1, 4, 2, 256, 128, 1, -2, None), 1),   # topk < -1
    ((P(16), P(32), P(48), P(64), 1, 4, 2, 256, 96, 1, 4, None), 2),     # d
    ((P(16), P(32), P(48), P(64), 1, 4, 2, 131073, 128, 1, 4, None), 2), # selection limit
    ((P(16), P(33), P(48), P(64), 1, 4, 2, 256, 128, 1, -1, None), 3),   # misaligned
])
def test_forward_nvfp4_argument_checks(args, expect):
    L = Q.load()
    assert L.qattn_forward_nvfp4(*args) == expect


def test_binding_argument_counts_match_the_header():
    """Every declaration in include/qattn.h has as many parameters as the binding passes."""
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    L = Q.load()
    decls = re.findall(r"\b(qattn_[a-z0-9_]+)\s*\(([^)]*)\)\s*;", text)
    assert len(decls) >= len(Q.EXPORTS) - 1
    for name, params in decls:
        params = params.strip()
        n = 0 if params in ("", "void") else params.count(",") + 1
        assert len(getattr(L, name).argtypes) == n, name


def test_adaptive_argument_checks():
    L = Q.load()
    # null pointers, a bad threshold, a missing variant table, d
    assert L.qattn_quant_v_fp8(None, 1, 2, 256, 128, P(16), P(32), None) == 1
    assert L.qattn_quant_v_fp8(P(16), 1, 2, 256, 96, P(16), P(32), None) == 2
    assert L.qattn_quant_v_fp8(P(16), 1, 2, 256, 128, P(20), P(32), None) == 3
    assert L.qattn_attn_quantized_pv8(P(16), P(32), P(48), P(64), None, P(80), P(96), 1, 4, 2,
                                      256, 128, 1, None) == 1
    assert L.qattn_adaptive_calibrate(P(16), P(32), P(48), 1, 4, 2, 256, 128, 1, 3.0, P(64),
                                      None, None) == 1
    assert L.qattn_adaptive_calibrate(P(16), P(32), P(48), 1, 4, 2, 256, 128, 1, 0.99, None,
                                      None, None) == 1
    assert L.qattn_forward_adaptive(P(16), P(32), P(48), P(64), 1, 4, 2, 256, 128, 1, None,
                                    None) == 1
    assert L.qattn_forward_adaptive(P(16), P(32), P(48), P(64), 1, 4, 3, 256, 128, 1, P(80),
                                    None) == 1
