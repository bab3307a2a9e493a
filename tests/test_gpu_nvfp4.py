"""The FP4 path of the ThriftAttention page (method section) on the GPU against the oracle.

- NVFP4 quantization (E2M1 codes, E4M3 scale per 16 values, binary32 scale per slice; the format
  per NVIDIA's definition): codes, block scales and slice scales are results of the same binary32
  operations on both sides, so every byte and float is compared exactly.  Covered: small ragged
  cases of both block directions with and without a channel mean, the degenerate cases (all-zero
  slice, blocks whose scale rounds to 0, fp16 subnormals, a single row), the workload generator's
  Q, smoothed K and V, and sampled slices at 32K tokens.
- FP4 score tiles on the block-scaled tensor cores: within 2^-20 of the magnitude sum.
- The FP4-path attention (two-level FP4 P, online merge), with and without FP16 promotion of the
  block-mean top-k key tiles: within the INT8 path's output bar of the oracle (plus the oracle's
  per-row slack for FP4 decisions within 2^-16 of a tie), a one-hot closed form, sampled rows at
  32K tokens; the one-call forward equals the separate calls bit for bit.
"""
import numpy as np
import pytest
import torch

from bit_quantized_attention_smoothing_b200.workloads import WORKLOADS, make_inputs
from conftest import np16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from bit_quantized_attention_smoothing_b200 import qattn as Q
    Q.load()
    return Q


def _draw(kind, S, R, C, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((S, R, C))
    if kind == "rowscale":
        x *= np.exp(1.5 * rng.standard_normal((S, R, 1)))
    elif kind == "channel":
        x = x * np.exp(rng.standard_normal((S, 1, C))) + 3 * rng.standard_normal((S, 1, C))
    elif kind == "outlier":
        idx = rng.integers(0, x.size, size=max(1, x.size // 500))
        x.flat[idx] *= 200.0
    elif kind == "zero_slice":
        x[0] = 0.0
        x[1, :3] *= 1e-5                      # blocks whose E4M3 scale rounds to 0 or is subnormal
        x[1, 5, :16] = -0.0
    elif kind == "tiny":
        x *= 3e-6                             # fp16 subnormals
    return np.clip(x, -60000, 60000).astype(np.float16)


def _compare(lib, oracle, x16, mean, along_rows):
    xg = torch.from_numpy(x16).cuda()
    mg = None if mean is None else torch.from_numpy(mean).cuda()
    codes, scales, g = lib.qattn_quant_nvfp4(xg, mg, along_rows=along_rows)
    torch.cuda.synchronize()
    rc, rs, rg = oracle.quant_nvfp4(x16, mean=mean, along_rows=along_rows)
    c, s, gg = codes.cpu().numpy(), scales.cpu().numpy(), g.cpu().numpy()
    assert c.shape == rc.shape and s.shape == rs.shape
    assert np.array_equal(gg.view(np.uint32), rg.view(np.uint32)), (gg, rg)
    bad = np.argwhere(s != rs)
    assert bad.size == 0, f"{bad.shape[0]} scale bytes differ, first at {bad[0]}: {s[tuple(bad[0])]} vs {rs[tuple(bad[0])]}"
    bad = np.argwhere(c != rc)
    assert bad.size == 0, f"{bad.shape[0]} code bytes differ, first at {bad[0]}: {c[tuple(bad[0])]:#04x} vs {rc[tuple(bad[0])]:#04x}"
    return c, s, gg


CASES = [
    (3, 200, 128, False, False, "rowscale"),
    (3, 200, 128, True, False, "rowscale"),
    (2, 37, 48, True, True, "channel"),
    (2, 37, 48, False, True, "channel"),
    (4, 1000, 64, True, True, "outlier"),
    (4, 1000, 64, False, True, "outlier"),
    (1, 1, 16, False, False, "normal"),
    (1, 1, 16, True, False, "normal"),
    (2, 130, 128, False, False, "zero_slice"),
    (2, 130, 128, True, False, "zero_slice"),
    (5, 64, 80, True, False, "tiny"),
    (5, 64, 80, False, True, "tiny"),
]


@pytest.mark.parametrize("S,R,C,along_rows,with_mean,kind", CASES,
                         ids=[f"S{c[0]}-R{c[1]}-C{c[2]}-{'rows' if c[3] else 'cols'}-"
                              f"{'mean' if c[4] else 'nomean'}-{c[5]}" for c in CASES])
def test_quant_nvfp4_bit_exact(lib, oracle, S, R, C, along_rows, with_mean, kind):
    x = _draw(kind, S, R, C, seed=S * 1000 + R + C + 7 * along_rows)
    mean = None
    if with_mean:
        mean = np.random.default_rng(R).standard_normal((S, C)).astype(np.float32)
    _compare(lib, oracle, x, mean, along_rows)


def test_quant_nvfp4_workload_q_k_v(lib, oracle):
    """The attention operands of a small workload: Q and smoothed K along d (K's mean is the
    oracle's exact channel mean), V along the tokens."""
    w = WORKLOADS["llama8b_32k"].with_(H=4, Hkv=2, N=1500)
    q, k, v = make_inputs(w, device="cpu")
    sums = oracle.k_channel_sums(np16(k), w.B, w.Hkv, w.N, w.d)
    mean = np.array([oracle.lib().oracle_mean_from_sum(int(s), w.N) for s in sums.ravel()],
                    dtype=np.float32).reshape(w.B * w.Hkv, w.d)
    qs = q.reshape(w.B * w.H, w.N, w.d).numpy()
    ks = k.reshape(w.B * w.Hkv, w.N, w.d).numpy()
    vs = v.reshape(w.B * w.Hkv, w.N, w.d).numpy()
    _compare(lib, oracle, qs, None, False)
    _compare(lib, oracle, ks, mean, False)
    _compare(lib, oracle, vs, None, True)


def test_quant_nvfp4_full_size_sampled_slices(lib, oracle):
    """Q [32 x 32768 x 128], K [8 x 32768 x 128] and V (along the tokens) of the 32K-token
    workload quantized whole on the GPU; the oracle recomputes sampled slices (each slice's
    result depends only on that slice)."""
    w = WORKLOADS["llama8b_32k"]
    q, k, v = make_inputs(w, device="cuda")
    for x, along_rows, picks in ((q, False, (0, w.H - 1)), (k, False, (3,)), (v, True, (5,))):
        S = x.shape[0] * x.shape[1]
        xs = x.reshape(S, w.N, w.d)
        codes, scales, g = lib.qattn_quant_nvfp4(xs, None, along_rows=along_rows)
        torch.cuda.synchronize()
        for s in picks:
            x16 = np16(xs[s:s + 1])
            rc, rs, rg = oracle.quant_nvfp4(x16.view(np.float16), along_rows=along_rows)
            assert np.array_equal(g[s:s + 1].cpu().numpy().view(np.uint32), rg.view(np.uint32))
            assert np.array_equal(scales[s:s + 1].cpu().numpy(), rs)
            assert np.array_equal(codes[s:s + 1].cpu().numpy(), rc)
        del codes, scales, g
    assert lib.qattn_check_device_status() == 0


def test_quant_nvfp4_dequantized_error(lib, oracle):
    """The decoded GPU result stays within one block-scale step of the input below saturation
    (the format's own bound: half the largest E2M1 spacing, 2, times the block scale)."""
    x16 = _draw("rowscale", 2, 256, 128, seed=3)
    c, s, g = _compare(lib, oracle, x16, None, False)
    deq = oracle.nvfp4_dequant(c, s, g)
    e4 = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    sc = np.repeat(e4[s], 16, axis=-1) * g.astype(np.float64)[:, None, None]
    err = np.abs(deq - x16.astype(np.float64))
    sat = np.abs(x16.astype(np.float64)) > 6 * sc
    assert np.all(err[~sat] <= 1.0001 * sc[~sat])


# ---- FP4 scores through tcgen05.mma kind::mxf4nvf4 (block16 UE4M3 scales) ----
#
# The tensor core sums 16-element E2M1 products (exact) weighted by the two block scales into an
# f32 accumulator; against the exact float64 score the only error is the f32 accumulation over
# the d / 16 blocks and the final product with gQ gK, a few units of 2^-24 of the magnitude sum
# M = |Q| |K|^T.  The bound used: |S_gpu - S| <= 2^-20 * M.
FP4_REL = 2.0 ** -20


def _check_scores(got, S, M, what):
    err = np.abs(got.astype(np.float64) - S)
    ratio = float((err / np.maximum(M, 1e-300)).max())
    print(what, "max |err| / M =", ratio)
    assert np.all(err <= FP4_REL * M + 1e-30), (what, ratio)


def _upload(t):
    return tuple(torch.from_numpy(np.ascontiguousarray(a)).cuda() for a in t)


@pytest.mark.parametrize("d", [128, 64])
def test_qk_nvfp4_random_codes_and_scales(lib, oracle, d):
    """Arbitrary code bytes and per-block scale bytes (no quantizer structure), so that every
    block's scale is independent: checks where each scale byte lands in tensor memory."""
    rng = np.random.default_rng(40 + d)
    B, H, Hkv, N = 1, 2, 1, 300
    qc = rng.integers(0, 256, size=(B * H, N, d // 2), dtype=np.uint8)
    kc = rng.integers(0, 256, size=(B * Hkv, N, d // 2), dtype=np.uint8)
    qs = rng.integers(0x20, 0x50, size=(B * H, N, d // 16), dtype=np.uint8)
    ks = rng.integers(0x20, 0x50, size=(B * Hkv, N, d // 16), dtype=np.uint8)
    qg = np.array([1.0, 0.5], dtype=np.float32)
    kg = np.array([2.0], dtype=np.float32)
    gq, gk = _upload((qc, qs, qg)), _upload((kc, ks, kg))
    nt = 3
    for h in range(H):
        got = lib.qattn_debug_qk_nvfp4(gq, gk, B, H, Hkv, N, d, 0, h, 0, nt, 0, nt).cpu().numpy()
        S, M = oracle.qk_nvfp4(qc, qs, qg, kc, ks, kg, H, Hkv, 0, h, 0, nt * 128, 0, nt * 128)
        _check_scores(got, S, M, f"random d{d} h{h}")
    assert lib.qattn_check_device_status() == 0


@pytest.mark.parametrize("name,over", [("llama8b_32k", {"H": 4, "Hkv": 2, "N": 700}),
                                       ("wide64", {"B": 2, "H": 2, "Hkv": 1, "N": 333})])
def test_qk_nvfp4_on_oracle_quantized_workload(lib, oracle, name, over):
    """The workload's Q and smoothed K, quantized by the oracle, scored on the tensor cores."""
    w = WORKLOADS[name].with_(**over)
    q, k, _ = make_inputs(w, device="cpu")
    sums = oracle.k_channel_sums(np16(k), w.B, w.Hkv, w.N, w.d)
    mean = np.array([oracle.lib().oracle_mean_from_sum(int(s), w.N) for s in sums.ravel()],
                    dtype=np.float32).reshape(w.B * w.Hkv, w.d)
    qn = oracle.quant_nvfp4(q.reshape(w.B * w.H, w.N, w.d).numpy())
    kn = oracle.quant_nvfp4(k.reshape(w.B * w.Hkv, w.N, w.d).numpy(), mean=mean)
    gq, gk = _upload(qn), _upload(kn)
    nt = -(-w.N // 128)
    for b, h in {(0, 0), (w.B - 1, w.H - 1)}:
        got = lib.qattn_debug_qk_nvfp4(gq, gk, w.B, w.H, w.Hkv, w.N, w.d, b, h, 0, nt, 0, nt)
        S, M = oracle.qk_nvfp4(*qn, *kn, w.H, w.Hkv, b, h, 0, nt * 128, 0, nt * 128)
        _check_scores(got.cpu().numpy(), S, M, f"{name} b{b} h{h}")


def test_qk_nvfp4_full_size_tiles(lib, oracle):
    """32K-token Q and smoothed K quantized on the GPU (the codes checked equal to the oracle's
    for the slices used), FP4 score tiles at the corners and the middle of the score matrix."""
    w = WORKLOADS["llama8b_32k"]
    q, k, _ = make_inputs(w, device="cuda")
    h, g = w.H - 1, (w.H - 1) // (w.H // w.Hkv)
    sums = oracle.k_channel_sums(np16(k[:, g:g + 1]), 1, 1, w.N, w.d)
    mean1 = np.array([oracle.lib().oracle_mean_from_sum(int(s), w.N) for s in sums.ravel()],
                     dtype=np.float32)
    mean = torch.zeros(w.B * w.Hkv, w.d, dtype=torch.float32, device="cuda")
    mean[g] = torch.from_numpy(mean1).cuda()
    gq = lib.qattn_quant_nvfp4(q.reshape(w.H, w.N, w.d))
    gk = lib.qattn_quant_nvfp4(k.reshape(w.Hkv, w.N, w.d), mean)
    qn = oracle.quant_nvfp4(np16(q[0, h:h + 1]).view(np.float16))
    kn = oracle.quant_nvfp4(np16(k[0, g:g + 1]).view(np.float16), mean=mean1[None])
    for mine, ref, s in ((gq, qn, h), (gk, kn, g)):
        for a, r in zip(mine, ref):
            assert np.array_equal(a[s:s + 1].cpu().numpy(), r)
    nt = w.N // 128
    for qt, kt in {(0, 0), (nt - 1, nt - 1), (nt - 1, 0), (nt // 2, nt // 3)}:
        got = lib.qattn_debug_qk_nvfp4(gq, gk, w.B, w.H, w.Hkv, w.N, w.d, 0, h, qt, 1, kt, 1)
        S, M = oracle.qk_nvfp4(qn[0], qn[1], qn[2], kn[0], kn[1], kn[2], 1, 1, 0, 0,
                               qt * 128, 128, kt * 128, 128)
        _check_scores(got.cpu().numpy(), S, M, f"full qt{qt} kt{kt}")


# ---- FP4-path attention (every key tile in FP4, two-level P, online merge) ----
#
# Against the oracle's FP4-path attention on the same NVFP4 operands.  The GPU's scores carry f32
# accumulation and its exponentials binary32 rounding; elsewhere the arithmetic is the oracle's
# (binary32 quantization steps), so outside FP4 decisions taken within 2^-16 of a tie the output
# agrees to the fp16 output rounding: max-abs 2e-3 and mean-abs 2e-4, as the INT8 path.  A row
# holding such near-tie decisions may differ by the oracle's per-row slack on top.

def _nvfp4_operands(oracle, w, q, k, v):
    sums = oracle.k_channel_sums(np16(k), w.B, w.Hkv, w.N, w.d)
    mean = np.array([oracle.lib().oracle_mean_from_sum(int(s), w.N) for s in sums.ravel()],
                    dtype=np.float32).reshape(w.B * w.Hkv, w.d)
    qn = oracle.quant_nvfp4(np16(q).reshape(w.B * w.H, w.N, w.d))
    kn = oracle.quant_nvfp4(np16(k).reshape(w.B * w.Hkv, w.N, w.d), mean=mean)
    vn = oracle.quant_nvfp4(np16(v).reshape(w.B * w.Hkv, w.N, w.d), along_rows=True)
    return qn, kn, vn


def _check_fp4_out(got_rows, ref, slack, what):
    g = got_rows.astype(np.float64)
    err = np.abs(g - ref)
    allow = 2e-3 + slack[:, None]
    n_slack = int((slack > 0).sum())
    print(what, f"max-abs {err.max():.3e} mean-abs {err.mean():.3e} rows with slack {n_slack}"
          f" worst excess {(err - allow).max():.3e}")
    assert np.all(err <= allow), what
    assert err.mean() <= 2e-4, what


FP4_CASES = [
    ("tiny", {"N": 300}),
    ("tiny", {"N": 129, "causal": True}),
    ("llama8b_32k", {"H": 4, "Hkv": 2, "N": 700}),
    ("llama8b_32k", {"B": 2, "H": 2, "Hkv": 1, "N": 200, "causal": False}),
    ("wide64", {"B": 1, "H": 3, "Hkv": 1, "N": 513, "causal": True}),
    ("long128k", {"H": 2, "Hkv": 1, "N": 1, "causal": True}),
]


@pytest.mark.parametrize("name,over", FP4_CASES,
                         ids=[f"{n}-" + "-".join(f"{k}{v}" for k, v in o.items()) for n, o in FP4_CASES])
def test_attn_nvfp4_against_oracle(lib, oracle, name, over):
    w = WORKLOADS[name].with_(**over)
    q, k, v = make_inputs(w, device="cpu")
    qn, kn, vn = _nvfp4_operands(oracle, w, q, k, v)
    out = lib.qattn_attn_nvfp4(_upload(qn), _upload(kn), _upload(vn), w.B, w.H, w.Hkv, w.N, w.d,
                               causal=w.causal)
    assert lib.qattn_check_device_status() == 0
    ref, slack = oracle.attention_nvfp4(qn, kn, vn, w.B, w.H, w.Hkv, w.N, w.d, w.causal)
    _check_fp4_out(out.float().cpu().numpy().reshape(-1, w.d), ref, slack, name)


@pytest.mark.parametrize("d,causal", [(64, False), (128, True)])
def test_attn_nvfp4_one_hot_scores(lib, oracle, d, causal):
    """Scores built from codes so that each row's softmax is the plain mean of V over its
    visible keys j == i (mod d) (closed form, several key tiles)."""
    rng = np.random.default_rng(50 + d)
    B, H, Hkv, N = 1, 2, 1, 400

    def onehot(S):
        codes = np.zeros((S, N, d // 2), dtype=np.uint8)
        scales = np.zeros((S, N, d // 16), dtype=np.uint8)
        for n in range(N):
            c = n % d
            codes[:, n, c // 2] = 7 << (4 * (c % 2))
            scales[:, n, c // 16] = 0x7E
        return codes, scales, np.ones(S, dtype=np.float32)

    Np = 512
    vc = rng.integers(0, 256, size=(B * Hkv, d, Np // 2), dtype=np.uint8)
    vs = rng.integers(0x30, 0x40, size=(B * Hkv, d, Np // 16), dtype=np.uint8)
    vn = (vc, vs, np.array([0.75], dtype=np.float32))
    qn, kn = onehot(B * H), onehot(B * Hkv)
    out = lib.qattn_attn_nvfp4(_upload(qn), _upload(kn), _upload(vn), B, H, Hkv, N, d,
                               causal=causal).float().cpu().numpy()
    vdec = oracle.nvfp4_dequant(*vn)[0]
    for h in range(H):
        for i in range(N):
            keys = [j for j in range(N) if j % d == i % d and (not causal or j <= i)]
            want = vdec[:, keys].mean(axis=1)
            assert np.abs(out[0, h, i] - want).max() <= 1e-3 + np.abs(want).max() * 2 ** -11


def test_attn_nvfp4_full_size_sampled_rows(lib, oracle):
    """32K-token workload, operands quantized on the GPU (slices used here checked equal to the
    oracle's), FP4-path attention of all 32 heads; sampled rows of one head against the oracle."""
    w = WORKLOADS["llama8b_32k"]
    q, k, v = make_inputs(w, device="cuda")
    h = 5
    g = h // (w.H // w.Hkv)
    sums = oracle.k_channel_sums(np16(k[:, g:g + 1]), 1, 1, w.N, w.d)
    mean1 = np.array([oracle.lib().oracle_mean_from_sum(int(s), w.N) for s in sums.ravel()],
                     dtype=np.float32)
    mean = torch.zeros(w.Hkv, w.d, dtype=torch.float32, device="cuda")
    mean[g] = torch.from_numpy(mean1).cuda()
    gq = lib.qattn_quant_nvfp4(q.reshape(w.H, w.N, w.d))
    gk = lib.qattn_quant_nvfp4(k.reshape(w.Hkv, w.N, w.d), mean)
    gv = lib.qattn_quant_nvfp4(v.reshape(w.Hkv, w.N, w.d), along_rows=True)
    out = lib.qattn_attn_nvfp4(gq, gk, gv, w.B, w.H, w.Hkv, w.N, w.d, causal=True)
    assert lib.qattn_check_device_status() == 0
    qn = oracle.quant_nvfp4(np16(q[0, h:h + 1]).view(np.float16))
    kn = oracle.quant_nvfp4(np16(k[0, g:g + 1]).view(np.float16), mean=mean1[None])
    vn = oracle.quant_nvfp4(np16(v[0, g:g + 1]).view(np.float16), along_rows=True)
    for mine, ref, s in ((gq, qn, h), (gk, kn, g), (gv, vn, g)):
        for a, r in zip(mine, ref):
            assert np.array_equal(a[s:s + 1].cpu().numpy(), r)
    rows_i = np.array([0, 1, 127, 128, 4095, 20000, w.N - 129, w.N - 1], dtype=np.int64)
    ref, slack = oracle.attention_nvfp4(qn, kn, vn, 1, 1, 1, w.N, w.d, True,
                                        rows=(np.zeros_like(rows_i), rows_i))
    got = out[0, h, torch.from_numpy(rows_i).cuda()].float().cpu().numpy()
    _check_fp4_out(got, ref, slack, "llama8b_32k full")


# ---- FP16 promotion of the selected key tiles (the ThriftAttention page's method) ----

def _lists_equal(gl, gc, ol, oc):
    gl, gc = gl.cpu().numpy(), gc.cpu().numpy()
    assert np.array_equal(gc, oc)
    for bh in range(oc.shape[0]):
        for i in range(oc.shape[1]):
            assert np.array_equal(gl[bh, i, :oc[bh, i]], ol[bh, i, :oc[bh, i]])


PROMO_CASES = [
    ("tiny", {"N": 300}, 1),
    ("llama8b_32k", {"H": 4, "Hkv": 2, "N": 700}, 1),
    ("llama8b_32k", {"B": 2, "H": 2, "Hkv": 1, "N": 600, "causal": False}, 2),
    ("wide64", {"B": 1, "H": 3, "Hkv": 1, "N": 513, "causal": True}, 0),
    ("prefill4k", {"B": 1, "H": 2, "Hkv": 2, "N": 640}, 100),          # every tile promoted
]


@pytest.mark.parametrize("name,over,topk", PROMO_CASES,
                         ids=[f"{n}-" + "-".join(f"{k}{v}" for k, v in o.items()) + f"-top{t}"
                              for n, o, t in PROMO_CASES])
def test_attn_nvfp4_promoted_against_oracle(lib, oracle, name, over, topk):
    """Key tiles chosen by the block-mean top-k (lists bit-exact against the oracle's) run in
    FP16, the others in FP4, merged by one online softmax."""
    w = WORKLOADS[name].with_(**over)
    q, k, v = make_inputs(w, device="cpu")
    qn, kn, vn = _nvfp4_operands(oracle, w, q, k, v)
    sums = oracle.k_channel_sums(np16(k), w.B, w.Hkv, w.N, w.d)
    mean = np.array([oracle.lib().oracle_mean_from_sum(int(s), w.N) for s in sums.ravel()],
                    dtype=np.float32).reshape(w.B * w.Hkv, w.d)
    qg, kg, vg = q.cuda(), k.cuda(), v.cuda()
    gl, gc = lib.qattn_block_select(qg, kg, topk, causal=w.causal)
    ol, oc = oracle.block_select(np16(q), np16(k), w.B, w.H, w.Hkv, w.N, w.d, w.causal, topk)
    _lists_equal(gl, gc, ol, oc)
    out = lib.qattn_attn_nvfp4(_upload(qn), _upload(kn), _upload(vn), w.B, w.H, w.Hkv, w.N, w.d,
                               causal=w.causal,
                               promote=(qg, kg, vg, torch.from_numpy(mean).cuda(), gl, gc))
    assert lib.qattn_check_device_status() == 0
    mask = oracle.tile_mask(ol, oc, w.N)
    ref, slack = oracle.attention_nvfp4(qn, kn, vn, w.B, w.H, w.Hkv, w.N, w.d, w.causal,
                                        promote=mask, q16=np16(q), k16=np16(k), v16=np16(v),
                                        k_mean=mean)
    _check_fp4_out(out.float().cpu().numpy().reshape(-1, w.d), ref, slack, f"{name} top{topk}")


def test_attn_nvfp4_promoted_full_size_sampled_rows(lib, oracle):
    """32K tokens, top-16 key tiles per 256-row block in FP16 (plus the diagonals), the rest in
    FP4; lists, quantization and the mean from the GPU path (lists and the used slices checked
    against the oracle), sampled rows of one head against the oracle."""
    w = WORKLOADS["llama8b_32k"]
    topk = 16
    q, k, v = make_inputs(w, device="cuda")
    h = 9
    g = h // (w.H // w.Hkv)
    sums = oracle.k_channel_sums(np16(k), 1, w.Hkv, w.N, w.d)
    mean = np.array([oracle.lib().oracle_mean_from_sum(int(s), w.N) for s in sums.ravel()],
                    dtype=np.float32).reshape(w.Hkv, w.d)
    meang = torch.from_numpy(mean).cuda()
    gq = lib.qattn_quant_nvfp4(q.reshape(w.H, w.N, w.d))
    gk = lib.qattn_quant_nvfp4(k.reshape(w.Hkv, w.N, w.d), meang)
    gv = lib.qattn_quant_nvfp4(v.reshape(w.Hkv, w.N, w.d), along_rows=True)
    gl, gc = lib.qattn_block_select(q, k, topk, causal=True)
    out = lib.qattn_attn_nvfp4(gq, gk, gv, w.B, w.H, w.Hkv, w.N, w.d, causal=True,
                               promote=(q, k, v, meang, gl, gc))
    assert lib.qattn_check_device_status() == 0
    ol, oc = oracle.block_select(np16(q), np16(k), w.B, w.H, w.Hkv, w.N, w.d, True, topk)
    _lists_equal(gl, gc, ol, oc)
    qh, kh, vh = np16(q[0, h:h + 1]), np16(k[0, g:g + 1]), np16(v[0, g:g + 1])
    qn = oracle.quant_nvfp4(qh.view(np.float16))
    kn = oracle.quant_nvfp4(kh.view(np.float16), mean=mean[g:g + 1])
    vn = oracle.quant_nvfp4(vh.view(np.float16), along_rows=True)
    for mine, ref, s in ((gq, qn, h), (gk, kn, g), (gv, vn, g)):
        for a, r in zip(mine, ref):
            assert np.array_equal(a[s:s + 1].cpu().numpy(), r)
    mask = oracle.tile_mask(ol[h:h + 1], oc[h:h + 1], w.N)
    rows_i = np.array([0, 1, 255, 256, 5000, 20000, w.N - 129, w.N - 1], dtype=np.int64)
    ref, slack = oracle.attention_nvfp4(qn, kn, vn, 1, 1, 1, w.N, w.d, True,
                                        rows=(np.zeros_like(rows_i), rows_i), promote=mask,
                                        q16=qh, k16=kh, v16=vh, k_mean=mean[g:g + 1])
    got = out[0, h, torch.from_numpy(rows_i).cuda()].float().cpu().numpy()
    _check_fp4_out(got, ref, slack, "llama8b_32k promoted full")


def test_attn_nvfp4_promoted_longest_lists(lib, oracle):
    """131072 tokens = 1024 key tiles, the most the promotion lists may index (the kernel's tile
    mask holds 1024 bits): one head, causal, top-8; the last query block's diagonal tiles 1022
    and 1023 are promoted.  Lists, quantized operands and mean from the GPU path (checked against
    the oracle), sampled rows at both ends of the sequence against the oracle."""
    w = WORKLOADS["long128k"].with_(H=1, Hkv=1)
    assert (w.N + 127) // 128 == 1024
    topk = 8
    q, k, v = make_inputs(w, device="cuda")
    sums = oracle.k_channel_sums(np16(k), 1, 1, w.N, w.d)
    mean = np.array([oracle.lib().oracle_mean_from_sum(int(s), w.N) for s in sums.ravel()],
                    dtype=np.float32).reshape(1, w.d)
    meang = torch.from_numpy(mean).cuda()
    gq = lib.qattn_quant_nvfp4(q.reshape(1, w.N, w.d))
    gk = lib.qattn_quant_nvfp4(k.reshape(1, w.N, w.d), meang)
    gv = lib.qattn_quant_nvfp4(v.reshape(1, w.N, w.d), along_rows=True)
    gl, gc = lib.qattn_block_select(q, k, topk, causal=True)
    out = lib.qattn_attn_nvfp4(gq, gk, gv, 1, 1, 1, w.N, w.d, causal=True,
                               promote=(q, k, v, meang, gl, gc))
    assert lib.qattn_check_device_status() == 0
    ol, oc = oracle.block_select(np16(q), np16(k), 1, 1, 1, w.N, w.d, True, topk)
    _lists_equal(gl, gc, ol, oc)
    qh, kh, vh = np16(q[0]), np16(k[0]), np16(v[0])
    qn = oracle.quant_nvfp4(qh.view(np.float16))
    kn = oracle.quant_nvfp4(kh.view(np.float16), mean=mean)
    vn = oracle.quant_nvfp4(vh.view(np.float16), along_rows=True)
    for mine, ref in ((gq, qn), (gk, kn), (gv, vn)):
        for a, r in zip(mine, ref):
            assert np.array_equal(a.cpu().numpy(), r)
    mask = oracle.tile_mask(ol, oc, w.N)
    assert mask[0, -1, -1] and mask[0, -1, -2]
    rows_i = np.array([0, 255, 256, 65535, w.N - 257, w.N - 129, w.N - 128, w.N - 1], dtype=np.int64)
    ref, slack = oracle.attention_nvfp4(qn, kn, vn, 1, 1, 1, w.N, w.d, True,
                                        rows=(np.zeros_like(rows_i), rows_i), promote=mask,
                                        q16=qh, k16=kh, v16=vh, k_mean=mean)
    got = out[0, 0, torch.from_numpy(rows_i).cuda()].float().cpu().numpy()
    _check_fp4_out(got, ref, slack, "long128k promoted, 1024 tiles")


@pytest.mark.parametrize("name,over,topk", [("llama8b_32k", {"H": 4, "Hkv": 2, "N": 700}, 2),
                                            ("tiny", {"N": 300}, -1),
                                            ("wide64", {"B": 2, "H": 2, "Hkv": 1, "N": 400,
                                                        "causal": True}, 0)])
def test_forward_nvfp4_one_call_equals_the_separate_calls(lib, oracle, name, over, topk):
    """qattn_forward_nvfp4 = channel mean + three quantizations + selection + attention, bit for
    bit; its mean is the oracle's exact channel mean."""
    w = WORKLOADS[name].with_(**over)
    q, k, v = (t.cuda() for t in make_inputs(w, device="cpu"))
    one = lib.qattn_forward_nvfp4(q, k, v, topk, causal=w.causal)
    sums = oracle.k_channel_sums(np16(k), w.B, w.Hkv, w.N, w.d)
    mean = torch.from_numpy(np.array([oracle.lib().oracle_mean_from_sum(int(s), w.N)
                                      for s in sums.ravel()], dtype=np.float32)
                            .reshape(w.B * w.Hkv, w.d)).cuda()
    qn = lib.qattn_quant_nvfp4(q.reshape(w.B * w.H, w.N, w.d))
    kn = lib.qattn_quant_nvfp4(k.reshape(w.B * w.Hkv, w.N, w.d), mean)
    vn = lib.qattn_quant_nvfp4(v.reshape(w.B * w.Hkv, w.N, w.d), along_rows=True)
    prom = None
    if topk >= 0:
        gl, gc = lib.qattn_block_select(q, k, topk, causal=w.causal)
        prom = (q, k, v, mean, gl, gc)
    sep = lib.qattn_attn_nvfp4(qn, kn, vn, w.B, w.H, w.Hkv, w.N, w.d, causal=w.causal, promote=prom)
    assert lib.qattn_check_device_status() == 0
    assert torch.equal(one.view(torch.int16), sep.view(torch.int16))
