"""GPU parity: the CUDA path through the C ABI against the CPU oracle on the same seeded inputs.

* smoothing + quantization (int8 codes, block scales, channel means): bit-exact;
* int32 score tiles, as the attention kernel itself loads them from tensor memory (its DUMP
  instantiation, causal and non-causal): bit-exact;
* forward output: max-abs <= 2e-3 and mean-abs <= 2e-4 against the oracle's unrounded float64
  output, flat (tests/conftest.py, check_output; the oracle rounds nothing after the int32
  product, the GPU rounds P to fp16, accumulates in fp32, uses a hardware exp2 and rounds O to
  fp16).

Small cases compare every output element and cover ragged N (partial Q tile, partial K block,
odd tile counts), N=1, GQA, causal and non-causal, d=64 and d=128.  The five named workloads run at
full size with the bench's launch configuration, comparing every int8 code and scale, every
output row of tiny, prefill4k and wide64 and a seeded sample of rows of llama8b_32k and long128k
(first and last rows of every head plus random rows).
"""
import numpy as np
import pytest
import torch

from bit_quantized_attention_smoothing_b200.workloads import ORDER, WORKLOADS, make_inputs, sample_rows
from conftest import check_output, np16

pytestmark = pytest.mark.gpu

SMALL = [
    ("tiny", {}),
    ("tiny", {"N": 200}),
    ("tiny", {"N": 1}),
    ("tiny", {"N": 129, "causal": True}),
    ("tiny", {"N": 64, "d": 128}),
    ("prefill4k", {"B": 1, "H": 4, "Hkv": 2, "N": 1000}),
    ("prefill4k", {"B": 2, "H": 2, "Hkv": 2, "N": 640, "causal": False}),
    ("wide64", {"B": 1, "H": 2, "Hkv": 1, "N": 1500}),
    ("long128k", {"H": 4, "Hkv": 1, "N": 2048}),
    ("llama8b_32k", {"H": 8, "Hkv": 2, "N": 768}),
    ("llama8b_32k", {"H": 2, "Hkv": 1, "N": 384}),
    ("wide64", {"B": 1, "H": 3, "Hkv": 3, "N": 300, "causal": True}),
    # causal pairs whose second Q tile has an odd number of 64-key tiles, or one more than the
    # first: the two tiles' pipelines end out of step
    ("tiny", {"N": 192, "causal": True}),
    ("tiny", {"N": 320, "causal": True, "d": 128}),
    ("wide64", {"B": 1, "H": 2, "Hkv": 1, "N": 700, "causal": True}),
]
SMALL_IDS = [f"{n}-" + "-".join(f"{k}{v}" for k, v in o.items()) for n, o in SMALL]

# rows sampled per head at full size (plus the first 128 and last 128 rows of every head); None:
# every row (the oracle's matmul form for the larger ones)
FULL_SAMPLES = {"tiny": None, "prefill4k": None, "llama8b_32k": 32, "long128k": 4, "wide64": None}


def _inputs(w, device="cuda"):
    q, k, v = make_inputs(w, device=device)
    return q.cuda(), k.cuda(), v.cuda()


def _check_quant(lib, oracle, w, q, k):
    q_i8, q_scale, k_i8, k_scale, k_mean = lib.qattn_smooth_quant(q, k)
    torch.cuda.synchronize()
    ref = oracle.smooth_quant(np16(q), np16(k), w.B, w.H, w.Hkv, w.N, w.d)
    assert np.array_equal(k_mean.cpu().numpy().view(np.uint32), ref["k_mean"].view(np.uint32))
    assert np.array_equal(k_scale.cpu().numpy().view(np.uint32), ref["k_scale"].view(np.uint32))
    assert np.array_equal(q_scale.cpu().numpy().view(np.uint32), ref["q_scale"].view(np.uint32))
    assert np.array_equal(k_i8.cpu().numpy(), ref["k_i8"])
    assert np.array_equal(q_i8.cpu().numpy(), ref["q_i8"])
    return (q_i8, q_scale, k_i8, k_scale), ref


def _rows_of(out, w, rows):
    bh, i = rows
    flat = out.reshape(w.B * w.H * w.N, w.d)
    idx = torch.as_tensor(np.asarray(bh) * w.N + np.asarray(i), device=out.device)
    return flat[idx].float().cpu().numpy()


@pytest.mark.parametrize("name,over", SMALL, ids=SMALL_IDS)
def test_smooth_quant_bit_exact_small(lib, oracle, name, over):
    w = WORKLOADS[name].with_(**over)
    q, k, _ = _inputs(w, "cpu")
    _check_quant(lib, oracle, w, q, k)


@pytest.mark.parametrize("name,over", SMALL, ids=SMALL_IDS)
def test_qk_int32_tiles_bit_exact_small(lib, oracle, name, over):
    """The int32 scores the attention kernel's softmax threads load from tensor memory (non-causal
    kernel: every tile; causal kernel: the tiles it computes, the others untouched)."""
    w = WORKLOADS[name].with_(**over)
    q, k, _ = _inputs(w, "cpu")
    (q_i8, _, k_i8, _), ref = _check_quant(lib, oracle, w, q, k)
    nt = -(-w.N // 128)
    lower = np.kron(np.tril(np.ones((nt, nt), dtype=bool)), np.ones((128, 128), dtype=bool))
    for b, h in {(0, 0), (w.B - 1, w.H - 1)}:
        # rows/columns beyond N are products with zero-filled rows
        full = np.zeros((nt * 128, nt * 128), dtype=np.int32)
        full[: w.N, : w.N] = oracle.qk_int32(ref["q_i8"], ref["k_i8"], w.B, w.H, w.Hkv, w.N, w.d,
                                             b, h, 0, w.N, 0, w.N)
        s = lib.qattn_debug_qk_int32(q_i8, k_i8, b, h, 0, nt, 0, nt, causal=False).cpu().numpy()
        assert np.array_equal(s, full)
        s = lib.qattn_debug_qk_int32(q_i8, k_i8, b, h, 0, nt, 0, nt, causal=True).cpu().numpy()
        assert np.array_equal(s, np.where(lower, full, 0))
    assert lib.qattn_check_device_status() == 0


@pytest.mark.parametrize("name,over", SMALL, ids=SMALL_IDS)
def test_forward_small_all_rows(lib, oracle, name, over):
    w = WORKLOADS[name].with_(**over)
    q, k, v = _inputs(w, "cpu")
    out = lib.qattn_forward(q, k, v, causal=w.causal)
    assert lib.qattn_check_device_status() == 0
    ref, _ = oracle.forward(np16(q), np16(k), np16(v), w.B, w.H, w.Hkv, w.N, w.d, w.causal)
    ok, msg = check_output(out.float().cpu().numpy().reshape(-1, w.d), ref)
    assert ok, msg


@pytest.mark.parametrize("name,over", SMALL, ids=SMALL_IDS)
def test_fp32_output_is_the_fp16_outputs_value(lib, oracle, name, over):
    """qattn_attn_quantized_f32 within the bar of the oracle, and qattn_attn_quantized's fp16
    output equal to its nearest-fp16 rounding, bit for bit (rows past N are not written)."""
    w = WORKLOADS[name].with_(**over)
    q, k, v = _inputs(w)
    q_i8, q_s, k_i8, k_s, _ = lib.qattn_smooth_quant(q, k)
    o16 = lib.qattn_attn_quantized(q_i8, q_s, k_i8, k_s, v, causal=w.causal)
    o32 = lib.qattn_attn_quantized_f32(q_i8, q_s, k_i8, k_s, v, causal=w.causal)
    torch.cuda.synchronize()
    assert lib.qattn_check_device_status() == 0
    assert torch.equal(o16, o32.half())
    ref, _ = oracle.forward(np16(q), np16(k), np16(v), w.B, w.H, w.Hkv, w.N, w.d, w.causal)
    ok, msg = check_output(o32.cpu().numpy().reshape(-1, w.d), ref)
    assert ok, msg


@pytest.mark.parametrize("name,over", SMALL[:6], ids=SMALL_IDS[:6])
def test_attention_on_oracle_codes(lib, oracle, name, over):
    """The attention kernel alone, fed the oracle's int8 codes and scales."""
    w = WORKLOADS[name].with_(**over)
    q, k, v = _inputs(w, "cpu")
    ref_sq = oracle.smooth_quant(np16(q), np16(k), w.B, w.H, w.Hkv, w.N, w.d)
    t = {key: torch.from_numpy(val).cuda() for key, val in ref_sq.items()}
    out = lib.qattn_attn_quantized(t["q_i8"], t["q_scale"], t["k_i8"], t["k_scale"], v,
                                   causal=w.causal)
    ref = oracle.attention_quantized(ref_sq["q_i8"], ref_sq["q_scale"], ref_sq["k_i8"],
                                     ref_sq["k_scale"], np16(v), w.B, w.H, w.Hkv, w.N, w.d, w.causal)
    ok, msg = check_output(out.float().cpu().numpy().reshape(-1, w.d), ref)
    assert ok, msg


@pytest.mark.parametrize("name,over", SMALL, ids=SMALL_IDS)
def test_fused_q_forward_against_oracle(lib, oracle, name, over):
    """qattn_smooth_k + qattn_attn_fused_q (Q quantized inside the attention kernel) against the
    oracle's whole path, every output element."""
    w = WORKLOADS[name].with_(**over)
    q, k, v = _inputs(w)
    k_i8, k_s, _ = lib.qattn_smooth_k(k)
    out = lib.qattn_attn_fused_q(q, k_i8, k_s, v, causal=w.causal)
    assert lib.qattn_check_device_status() == 0
    ref, _ = oracle.forward(np16(q), np16(k), np16(v), w.B, w.H, w.Hkv, w.N, w.d, w.causal)
    ok, msg = check_output(out.float().cpu().numpy().reshape(-1, w.d), ref)
    assert ok, msg


@pytest.mark.parametrize("name,over", SMALL, ids=SMALL_IDS)
def test_fused_q_halves_match_separate_quantization(lib, name, over):
    """The fused forward's halves: qattn_smooth_k writes the same K codes, scales and means as
    qattn_smooth_quant, and the attention kernel that quantizes Q in its prologue gives the same
    output, bit for bit, as the one fed qattn_smooth_quant's int8 Q (its Q codes and scales are
    pinned to the oracle by test_smooth_quant_bit_exact_small)."""
    w = WORKLOADS[name].with_(**over)
    q, k, v = _inputs(w)
    q_i8, q_s, k_i8, k_s, k_mean = lib.qattn_smooth_quant(q, k)
    k_mean2 = torch.empty_like(k_mean)
    k_i8b, k_sb, _ = lib.qattn_smooth_k(k, k_mean=k_mean2)
    ref = lib.qattn_attn_quantized(q_i8, q_s, k_i8, k_s, v, causal=w.causal)
    got = lib.qattn_attn_fused_q(q, k_i8b, k_sb, v, causal=w.causal)
    fwd = lib.qattn_forward(q, k, v, causal=w.causal)
    torch.cuda.synchronize()
    assert lib.qattn_check_device_status() == 0
    assert torch.equal(k_i8, k_i8b) and torch.equal(k_s, k_sb) and torch.equal(k_mean, k_mean2)
    assert torch.equal(ref, got)
    assert torch.equal(ref, fwd)


def _planted_jumps(w):
    """Seeded inputs whose row maxima jump by far more than the lazy-rescale threshold after the
    first key tile: one direction u is added to every query, and three keys are replaced by
    large multiples of u (token 300 inside the diagonal tile of rows 256-383, tokens 700 and 901
    further on), so that rows reaching them see their running max grow by ~20-60 log2 units.
    The softmax must then void its optimistic P for that step, move the max and rescale O."""
    q, k, v = make_inputs(w)
    gen = torch.Generator().manual_seed(77)
    u = torch.randn(w.d, generator=gen)
    u = u / u.norm()
    q = (q.float() + 3.0 * u).half()
    k = k.float()
    for t, a in ((300, 40.0), (700, 80.0), (901, 120.0)):
        k[:, :, t] = a * u
    return q, k.half(), v


@pytest.mark.parametrize("d,causal", [(64, True), (128, True), (128, False)])
def test_forward_planted_max_jumps(lib, oracle, d, causal):
    w = WORKLOADS["tiny"].with_(B=1, H=2, Hkv=1, N=1000, d=d, causal=causal)
    q, k, v = _planted_jumps(w)
    out = lib.qattn_forward(q.cuda(), k.cuda(), v.cuda(), causal=causal)
    assert lib.qattn_check_device_status() == 0
    ref, _ = oracle.forward(np16(q), np16(k), np16(v), w.B, w.H, w.Hkv, w.N, w.d, causal)
    ok, msg = check_output(out.float().cpu().numpy().reshape(-1, w.d), ref)
    assert ok, msg


def test_forward_variants_agree(lib):
    w = WORKLOADS["prefill4k"].with_(B=1, H=4, Hkv=2, N=777)
    q, k, v = _inputs(w, "cpu")
    a = lib.qattn_forward(q, k, v, causal=True)
    b = lib.qattn_forward_ws(q, k, v, causal=True)
    c = lib.qattn_forward_host(q.cpu().pin_memory(), k.cpu().pin_memory(), v.cpu().pin_memory(),
                               causal=True)
    d = lib.qattn_forward_host(q.cpu(), k.cpu(), v.cpu(), causal=True)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    assert torch.equal(a.cpu(), c) and torch.equal(a.cpu(), d)


HOST_SHAPES = [
    # 9 groups: uneven chunks of 2, 2, 2, 2, 1 groups
    {"B": 3, "H": 6, "Hkv": 3, "N": 300},
    # 8 single-group chunks of 4 query heads: the first and last run as two pieces of 2 heads
    {"B": 1, "H": 32, "Hkv": 8, "N": 300},
    # one group of 3 query heads: pieces of 1 and 2 heads; two groups of 2: both split
    {"B": 1, "H": 3, "Hkv": 1, "N": 520},
    {"B": 1, "H": 4, "Hkv": 2, "N": 129},
    # one group of one query head: no split
    {"B": 1, "H": 1, "Hkv": 1, "N": 700},
]


@pytest.mark.parametrize("shape", HOST_SHAPES, ids=lambda o: "-".join(f"{k}{v}" for k, v in o.items()))
@pytest.mark.parametrize("pinned", [True, False])
def test_host_forward_pipeline_chunks(lib, pinned, shape):
    """qattn_forward_host cuts the (batch, kv head) groups into chunks whose copies and kernels
    overlap, and the first and last single-group chunks into two pieces of half their query heads.
    Results must equal the device-buffer forward bit for bit."""
    w = WORKLOADS["wide64"].with_(causal=True, **shape)
    q, k, v = _inputs(w, "cpu")
    a = lib.qattn_forward(q.cuda(), k.cuda(), v.cuda(), causal=True)
    hq, hk, hv = (t.cpu() for t in (q, k, v))
    if pinned:
        hq, hk, hv = hq.pin_memory(), hk.pin_memory(), hv.pin_memory()
    c = lib.qattn_forward_host(hq, hk, hv, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(a.cpu(), c)


def test_repeated_calls_are_deterministic(lib):
    w = WORKLOADS["wide64"].with_(B=1, H=2, Hkv=2, N=1024)
    q, k, v = _inputs(w, "cpu")
    a = lib.qattn_forward(q, k, v, causal=False)
    for _ in range(3):
        assert torch.equal(a, lib.qattn_forward(q, k, v, causal=False))


def test_gpu_rejects_bad_arguments(lib):
    q = torch.zeros(1, 2, 64, 96, dtype=torch.float16, device="cuda")
    with pytest.raises(lib.QattnError) as e:
        lib.qattn_forward(q, q, q)
    assert e.value.status == 2
    q = torch.zeros(1, 3, 64, 64, dtype=torch.float16, device="cuda")
    k = torch.zeros(1, 2, 64, 64, dtype=torch.float16, device="cuda")
    with pytest.raises(lib.QattnError) as e:
        lib.qattn_forward(q, k, k)
    assert e.value.status == 1
    assert lib.qattn_check_device_status() == 0


@pytest.mark.parametrize("name", ORDER)
def test_full_size_workload(lib, oracle, name):
    """Full-size workload, same launch as the benchmark: every code and scale bit-exact, int32
    score tiles of the product kernel (causal as the workload) on the first, last, a middle and the
    whole last row of key tiles; the attention's value (the fp32-output instantiation) within
    max-abs 2e-3 / mean-abs 2e-4 of the oracle on every row (tiny, prefill4k, wide64) or a seeded
    sample of rows, and the product's fp16 output equal to that value rounded to the nearest fp16,
    bit for bit, everywhere.  The fp16 output's own error against the oracle is printed: where
    |O| >= 4 the fp16 grid's half-spacing (1.95e-3) alone nearly fills the 2e-3 budget."""
    w = WORKLOADS[name]
    q, k, v = make_inputs(w, device="cuda")
    (q_i8, q_s, k_i8, k_s), ref_sq = _check_quant(lib, oracle, w, q, k)
    nt = -(-w.N // 128)
    b, h = w.B - 1, w.H - 1
    for qt, kt, nk in {(0, 0, 1), (nt - 1, nt - 1, 1), (nt // 2, nt // 3, 1), (nt - 1, 0, nt)}:
        s = lib.qattn_debug_qk_int32(q_i8, k_i8, b, h, qt, 1, kt, nk, causal=w.causal).cpu().numpy()
        r = oracle.qk_int32(ref_sq["q_i8"], ref_sq["k_i8"], w.B, w.H, w.Hkv, w.N, w.d,
                            b, h, qt * 128, min(128, w.N - qt * 128), kt * 128, min(nk * 128, w.N - kt * 128))
        assert np.array_equal(s[: r.shape[0], : r.shape[1]], r)
    # the fp32-output instantiation on the same (bit-exact) int8 operands
    out32 = lib.qattn_attn_quantized_f32(q_i8, q_s, k_i8, k_s, v, causal=w.causal)
    del q_i8, k_i8
    out = lib.qattn_forward(q, k, v, causal=w.causal)
    assert lib.qattn_check_device_status() == 0
    # the product's fp16 output is the fp32 result rounded to nearest, bit for bit
    assert torch.equal(out, out32.half())
    per = FULL_SAMPLES[name]
    if per is None:
        got = out32.cpu().numpy().reshape(-1, w.d)
        got16 = out.float().cpu().numpy().reshape(-1, w.d)
        del out, out32
        if w.B * w.H * w.N <= 4096:
            ref = oracle.attention_quantized(ref_sq["q_i8"], ref_sq["q_scale"], ref_sq["k_i8"],
                                             ref_sq["k_scale"], np16(v), w.B, w.H, w.Hkv, w.N,
                                             w.d, w.causal)
        else:
            ref = oracle.attention_quantized_all(ref_sq["q_i8"], ref_sq["q_scale"], ref_sq["k_i8"],
                                                 ref_sq["k_scale"], np16(v), w.B, w.H, w.Hkv, w.N,
                                                 w.d, w.causal)
    else:
        rows = tuple(t.numpy() for t in sample_rows(w, per, edge_first=128, edge_last=128 if per > 4 else 8))
        got = _rows_of(out32, w, rows)
        got16 = _rows_of(out, w, rows)
        ref = oracle.attention_quantized(ref_sq["q_i8"], ref_sq["q_scale"], ref_sq["k_i8"],
                                         ref_sq["k_scale"], np16(v), w.B, w.H, w.Hkv, w.N, w.d,
                                         w.causal, rows=rows)
    ok, msg = check_output(got, ref)
    _, msg16 = check_output(got16, ref)
    print(name, "fp32 output:", msg)
    print(name, "fp16 output (its nearest-fp16 rounding):", msg16)
    assert ok, msg


def test_bounded_wait_times_out_and_context_survives(lib):
    """An mbarrier wait that nothing satisfies gives up after its limit (about 1 ms here), records
    QATTN_ERR_TIMEOUT in the device status word and returns; the context stays usable."""
    assert lib.qattn_check_device_status() == 0
    assert lib.qattn_debug_wait_timeout(2_000_000) == 1
    assert lib.qattn_check_device_status() == 5
    assert lib.qattn_check_device_status() == 0      # reading clears it
    w = WORKLOADS["tiny"]
    q, k, v = _inputs(w, "cpu")
    a = lib.qattn_forward(q, k, v)
    torch.cuda.synchronize()
    assert torch.isfinite(a.float()).all() and lib.qattn_check_device_status() == 0
