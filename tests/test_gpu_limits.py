"""GPU parity at the largest shapes the C ABI accepts (N <= 2^20, B * H <= 2^20).

* N = 2^20 (one kv head, two query heads, d = 128, causal): int8 codes, block scales and channel
  means bit-exact against the oracle; int32 score tiles of the attention kernel at the far end of
  the sequence (the largest row and column offsets) bit-exact; the attention's value (the
  fp32-output instantiation) within max-abs 2e-3 / mean-abs 2e-4 of the oracle on sampled rows,
  and the fp16 output its nearest-fp16 rounding bit for bit.
* B * H = 2^20 with N = 1 (GQA, 4 query heads per kv head): one key per row, so the softmax puts
  all of its weight on it and the output is that key's V row, exactly (the only P is 2^7, exact in
  fp16, and O / l = 2^7 v / 2^7).
"""
import numpy as np
import pytest
import torch

from bit_quantized_attention_smoothing_b200.workloads import WORKLOADS
from conftest import check_output, np16

pytestmark = pytest.mark.gpu


def test_longest_sequence(lib, oracle):
    w = WORKLOADS["llama8b_32k"].with_(H=2, Hkv=1, N=1 << 20, seed=2024)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(w.seed)
    shape_q, shape_kv = (w.B, w.H, w.N, w.d), (w.B, w.Hkv, w.N, w.d)
    q = torch.randn(shape_q, generator=gen, device="cuda").half()
    offset = torch.randn(w.d, generator=gen, device="cuda") * 2.0
    k = (torch.randn(shape_kv, generator=gen, device="cuda") + offset).half()
    v = torch.randn(shape_kv, generator=gen, device="cuda").half()

    q_i8, q_s, k_i8, k_s, k_mean = lib.qattn_smooth_quant(q, k)
    torch.cuda.synchronize()
    ref = oracle.smooth_quant(np16(q), np16(k), w.B, w.H, w.Hkv, w.N, w.d)
    assert np.array_equal(k_mean.cpu().numpy().view(np.uint32), ref["k_mean"].view(np.uint32))
    assert np.array_equal(k_s.cpu().numpy().view(np.uint32), ref["k_scale"].view(np.uint32))
    assert np.array_equal(q_s.cpu().numpy().view(np.uint32), ref["q_scale"].view(np.uint32))
    assert np.array_equal(k_i8.cpu().numpy(), ref["k_i8"])
    assert np.array_equal(q_i8.cpu().numpy(), ref["q_i8"])

    nt = w.N // 128
    b, h = 0, w.H - 1
    for qt, kt, nk in [(nt - 1, nt - 1, 1), (nt - 1, 0, 2), (nt - 1, nt - 3, 2), (nt // 2, nt // 2 - 1, 2)]:
        s = lib.qattn_debug_qk_int32(q_i8, k_i8, b, h, qt, 1, kt, nk, causal=True).cpu().numpy()
        r = oracle.qk_int32(ref["q_i8"], ref["k_i8"], w.B, w.H, w.Hkv, w.N, w.d,
                            b, h, qt * 128, 128, kt * 128, nk * 128)
        assert np.array_equal(s, r)

    out32 = lib.qattn_attn_quantized_f32(q_i8, q_s, k_i8, k_s, v, causal=True)
    out = lib.qattn_forward(q, k, v, causal=True)
    assert lib.qattn_check_device_status() == 0
    assert torch.equal(out, out32.half())

    rng = np.random.default_rng(11)
    i = np.concatenate([np.arange(4), np.arange(w.N - 4, w.N),
                        rng.integers(0, w.N, 8), np.arange(nt // 2 * 128, nt // 2 * 128 + 2)])
    rows = (np.repeat(np.arange(w.H), i.size).astype(np.int64), np.tile(i, w.H).astype(np.int64))
    flat32 = out32.reshape(-1, w.d)
    idx = torch.as_tensor(rows[0] * w.N + rows[1], device="cuda")
    got = flat32[idx].cpu().numpy()
    want = oracle.attention_quantized(ref["q_i8"], ref["q_scale"], ref["k_i8"], ref["k_scale"],
                                      np16(v), w.B, w.H, w.Hkv, w.N, w.d, True, rows=rows)
    ok, msg = check_output(got, want)
    print("N = 2^20:", msg)
    assert ok, msg


def test_most_heads_one_key(lib):
    B, H, Hkv, N, d = 1, 1 << 20, 1 << 18, 1, 128
    gen = torch.Generator(device="cuda")
    gen.manual_seed(77)
    q = torch.randn(B, H, N, d, generator=gen, device="cuda").half()
    k = torch.randn(B, Hkv, N, d, generator=gen, device="cuda").half()
    v = torch.randn(B, Hkv, N, d, generator=gen, device="cuda").half()
    for causal in (True, False):
        out = lib.qattn_forward(q, k, v, causal=causal)
        assert lib.qattn_check_device_status() == 0
        assert torch.equal(out, v.repeat_interleave(H // Hkv, dim=1))
