"""The allocation-free smoothing + quantization entry point (qattn_smooth_quant_noalloc).

Some callers cannot allocate device memory when they call the library: their device memory is
all reserved up front and handed out by their own allocator, or they must not put an allocation
(and the synchronization it can bring) on the stream.  For them the library keeps the one piece of
scratch this step needs, the exact int64 channel sums of K, in a fixed device array of 65536
entries.  This test calls that entry point through the C ABI twice in a row, with different
shapes so the second call runs on scratch the first call left behind, and checks that every
output is bit-identical to the workspace-taking qattn_smooth_quant (the same tolerance the other
quantization tests use: exact).
"""
import numpy as np
import pytest
import torch

from bit_quantized_attention_smoothing_b200.workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from bit_quantized_attention_smoothing_b200 import qattn as Q
    Q.load()
    return Q


def _outputs_like(q, k):
    B, H, N, d = q.shape
    Hkv = k.shape[1]
    dev = q.device
    return (torch.empty(B, H, N, d, dtype=torch.int8, device=dev),
            torch.empty(B, H, -(-N // 128), dtype=torch.float32, device=dev),
            torch.empty(B, Hkv, N, d, dtype=torch.int8, device=dev),
            torch.empty(B, Hkv, -(-N // 64), dtype=torch.float32, device=dev),
            torch.empty(B, Hkv, d, dtype=torch.float32, device=dev))


def _same_bits(a, b):
    return np.array_equal(a.cpu().numpy().view(np.uint8), b.cpu().numpy().view(np.uint8))


def test_noalloc_matches_workspace_entry_on_two_calls(lib):
    cases = [WORKLOADS["prefill4k"].with_(B=2, H=4, Hkv=2, N=1000),
             WORKLOADS["wide64"].with_(B=1, H=3, Hkv=3, N=700)]
    for w in cases:
        q, k, _ = (t.cuda() for t in make_inputs(w))
        ref = lib.qattn_smooth_quant(q, k)
        got = lib.qattn_smooth_quant_noalloc(q, k, *_outputs_like(q, k))
        torch.cuda.synchronize()
        assert lib.qattn_check_device_status() == 0
        for name, a, b in zip(["q_i8", "q_scale", "k_i8", "k_scale", "k_mean"], got, ref):
            assert _same_bits(a, b), (w.name, name)


def test_noalloc_rejects_sizes_beyond_its_scratch(lib):
    # B * Hkv * d = 2 * 257 * 128 > 65536 channel sums
    q = torch.zeros(2, 257, 128, 128, dtype=torch.float16, device="cuda")
    with pytest.raises(lib.QattnError) as e:
        lib.qattn_smooth_quant_noalloc(q, q, *_outputs_like(q, q))
    assert e.value.status == 6
