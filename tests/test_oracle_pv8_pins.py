"""Pins of the oracle's FP8 (E4M3) P V variant, the coarser variant of the adaptive quantization
(SageAttention summary page, aibr.jp/archives/102657: dialogue and sec. 2-4, per-layer/head choice
of the quantization strength), against what fixes it independently of the oracle:

* E4M3 encoding and decoding against torch's float8_e4m3fn conversion (every code, every
  midpoint and its neighbours, random values), saturation at 448, zeros as +0;
* the V quantizer on slices built from E4M3 values times a power of two (exact codes, transposed
  with zero padding, scale 2^e) and on random data (every code torch's E4M3 of v / sV);
* the attention on hand-built int8 codes whose scores are one-hot per residue class of the key
  index (the output is then the plain mean of the selected E4M3 V values, causal or not, across
  tiles), with a later tile scoring far higher (the rescale by 2^(m - m') must drop the earlier
  tiles), identical keys (uniform weights), V scaled by 2 (the output doubles exactly), and
  closeness to float64 attention of the dequantized operands on random data.
Planted mistakes (no rescale, V read untransposed, the scale left out) fail these pins.
"""
import numpy as np
import pytest
import torch

from bit_quantized_attention_smoothing_b200.workloads import WORKLOADS, make_inputs


def _torch_e4m3(x):
    return torch.tensor(np.asarray(x, dtype=np.float32)).to(torch.float8_e4m3fn).to(torch.float64).numpy()


def _all_magnitudes():
    return np.array(sorted({abs(float(v)) for v in torch.arange(256, dtype=torch.uint8)
                            .view(torch.float8_e4m3fn).to(torch.float64).numpy() if np.isfinite(v)}))


def test_e4m3_decode_every_code(oracle):
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.tensor(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([oracle.e4m3_decode(int(c)) for c in codes])
    finite = np.isfinite(ref)
    assert finite.sum() == 254
    assert np.array_equal(got[finite], ref[finite])


def test_e4m3_encode_against_torch(oracle):
    mags = _all_magnitudes()
    mids = (mags[1:] + mags[:-1]) / 2
    grid = np.concatenate([mags, mids, np.nextafter(mids.astype(np.float32), np.float32(0)),
                           np.nextafter(mids.astype(np.float32), np.float32(1e9))])
    rng = np.random.default_rng(3)
    grid = np.concatenate([grid, rng.uniform(0, 448, 4000), np.exp(rng.uniform(-14, 6, 4000))])
    grid = grid[grid <= 448].astype(np.float32)
    x = np.concatenate([grid, -grid])
    got = np.array([oracle.e4m3_decode(oracle.e4m3_encode(float(v))) for v in x])
    ref = _torch_e4m3(x)
    assert np.array_equal(got, ref)      # -0.0 == 0.0 compares equal: zeros checked below
    zeros = [oracle.e4m3_encode(float(v)) for v in x if _torch_e4m3([v])[0] == 0]
    assert zeros and all(c == 0 for c in zeros)


def test_e4m3_saturates(oracle):
    for v in (448.0, 449.0, 464.0, 1e6):
        assert oracle.e4m3_decode(oracle.e4m3_encode(v)) == 448.0
        assert oracle.e4m3_decode(oracle.e4m3_encode(-v)) == -448.0


def test_quant_v_fp8_exact_codes_transposed(oracle):
    rng = np.random.default_rng(4)
    mags = _all_magnitudes()
    S, R, C = 2, 150, 16
    codes_val = rng.choice(mags, size=(S, R, C)) * rng.choice([-1.0, 1.0], size=(S, R, C))
    codes_val[:, 7, 3] = 448.0                      # each slice's maximum: 448 * 2^e
    scale = np.array([2.0 ** -3, 2.0 ** -7])
    v = (codes_val * scale[:, None, None]).astype(np.float16)
    assert np.array_equal(v.astype(np.float64), codes_val * scale[:, None, None])
    vt8, sv = oracle.quant_v_fp8(v)
    assert vt8.shape == (S, C, 256) and sv.tolist() == scale.tolist()
    assert not vt8[:, :, R:].any()
    got = oracle.e4m3_decode_array(vt8[:, :, :R]).transpose(0, 2, 1)
    assert np.array_equal(got, codes_val)


def test_quant_v_fp8_random_against_torch(oracle):
    w = WORKLOADS["wide64"].with_(B=1, H=3, Hkv=3, N=300)
    _, _, v = make_inputs(w)
    v = v.numpy().reshape(3, 300, 64)
    vt8, sv = oracle.quant_v_fp8(v)
    amax = np.abs(v.astype(np.float32)).max(axis=(1, 2))
    assert np.array_equal(sv, (amax / np.float32(448)).astype(np.float32))
    q = (v.astype(np.float32) / sv[:, None, None]).astype(np.float32)
    ref = _torch_e4m3(q).transpose(0, 2, 1)
    assert np.array_equal(oracle.e4m3_decode_array(vt8[:, :, :300]), ref)
    z = oracle.quant_v_fp8(np.zeros((1, 5, 16), dtype=np.float16))
    assert not z[0].any() and z[1][0] == 0.0


def _one_hot_case(N, d, causal, jump):
    """int8 Q row i and K row j are 127 e_(i mod d) and 127 e_(j mod d): S_int = 127^2 when
    j = i (mod d), else 0.  K scales 1 (or, with jump, 2^5 for the keys of the second tile), Q
    scales 1."""
    H = Hkv = B = 1
    idx = np.arange(N) % d
    q_i8 = np.zeros((B, H, N, d), dtype=np.int8)
    q_i8[0, 0, np.arange(N), idx] = 127
    k_i8 = q_i8.reshape(B, Hkv, N, d).copy()
    q_scale = np.ones((B, H, -(-N // 128)), dtype=np.float32)
    k_scale = np.ones((B, Hkv, -(-N // 64)), dtype=np.float32)
    if jump:
        k_scale[0, 0, 2:4] = 32.0
    return q_i8, q_scale, k_i8, k_scale


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("jump", [False, True])
def test_attention_pv8_one_hot_scores(oracle, causal, jump):
    N, d = 300, 16
    q_i8, q_scale, k_i8, k_scale = _one_hot_case(N, d, causal, jump)
    rng = np.random.default_rng(5)
    v = rng.standard_normal((1, N, d)).astype(np.float16)
    vt8, sv = oracle.quant_v_fp8(v)
    vv = oracle.e4m3_decode_array(vt8[0, :, :N]).T * float(sv[0])
    out, slack = oracle.attention_pv8(q_i8, q_scale, k_i8, k_scale, vt8, sv, 1, 1, 1, N, d, causal)
    ref = np.zeros((N, d))
    for i in range(N):
        last = i if causal else N - 1
        sel = [j for j in range(last + 1) if j % d == i % d]
        if jump:
            # keys 128 .. 255 score 32x higher: once one is visible, the earlier ones vanish
            hi = [j for j in sel if 128 <= j < 256]
            sel = hi if hi else sel
        ref[i] = vv[sel].mean(axis=0)
    assert np.abs(out - ref).max() <= 1e-12
    assert not slack.any()


@pytest.mark.parametrize("causal", [False, True])
def test_attention_pv8_identical_keys_and_v_scaling(oracle, causal):
    N, d = 260, 64
    rng = np.random.default_rng(6)
    q_i8 = rng.integers(-127, 128, (1, 2, N, d)).astype(np.int8)
    k_i8 = np.tile(rng.integers(-127, 128, d).astype(np.int8), (1, 1, N, 1))
    q_scale = rng.uniform(0.01, 0.02, (1, 2, 3)).astype(np.float32)
    k_scale = np.full((1, 1, 5), 0.015, dtype=np.float32)
    v = rng.standard_normal((1, N, d)).astype(np.float16)
    vt8, sv = oracle.quant_v_fp8(v)
    out, _ = oracle.attention_pv8(q_i8, q_scale, k_i8, k_scale, vt8, sv, 1, 2, 1, N, d, causal)
    vv = oracle.e4m3_decode_array(vt8[0, :, :N]).T * float(sv[0])
    ref = np.cumsum(vv, 0) / np.arange(1, N + 1)[:, None] if causal else np.tile(vv.mean(0), (N, 1))
    np.testing.assert_allclose(out, np.concatenate([ref, ref]), rtol=0, atol=1e-12)
    vt8b, sv2 = oracle.quant_v_fp8((v.astype(np.float32) * 2).astype(np.float16))
    assert np.array_equal(vt8b, vt8) and sv2[0] == 2 * sv[0]
    out2, _ = oracle.attention_pv8(q_i8, q_scale, k_i8, k_scale, vt8b, sv2, 1, 2, 1, N, d, causal)
    assert np.array_equal(out2, 2 * out)


@pytest.mark.parametrize("name,over", [("tiny", {}), ("llama8b_32k", {"H": 4, "Hkv": 2, "N": 600}),
                                       ("wide64", {"B": 1, "H": 2, "Hkv": 1, "N": 700})])
def test_attention_pv8_close_to_float64_of_its_operands(oracle, name, over):
    """Against float64 softmax(S_int sQ sK / sqrt(d)) (v^ sV) on the same int8 and E4M3 operands:
    only P's E4M3 rounding (relative 2^-4) separates them."""
    w = WORKLOADS[name].with_(**over)
    q, k, v = (t.numpy().view(np.uint16) for t in make_inputs(w))
    sq = oracle.smooth_quant(q, k, w.B, w.H, w.Hkv, w.N, w.d)
    vt8, sv = oracle.quant_v_fp8(v.reshape(w.B * w.Hkv, w.N, w.d))
    out, _ = oracle.attention_pv8(sq["q_i8"], sq["q_scale"], sq["k_i8"], sq["k_scale"], vt8, sv,
                                  w.B, w.H, w.Hkv, w.N, w.d, w.causal)
    vdq = (oracle.e4m3_decode_array(vt8[:, :, :w.N]).transpose(0, 2, 1) * sv[:, None, None].astype(np.float64))
    vdq16 = vdq.reshape(w.B, w.Hkv, w.N, w.d)
    ref = oracle.attention_quantized(sq["q_i8"], sq["q_scale"], sq["k_i8"], sq["k_scale"],
                                     np.zeros_like(v), w.B, w.H, w.Hkv, w.N, w.d, w.causal)
    # the float64 attention with V = v^ sV: the quantized oracle's weights applied to vdq
    G = w.H // w.Hkv
    qi = sq["q_i8"].astype(np.float64)
    ki = sq["k_i8"].astype(np.float64)
    refs = []
    for b in range(w.B):
        for h in range(w.H):
            g = h // G
            s = qi[b, h] @ ki[b, g].T
            s *= np.repeat(sq["q_scale"][b, h].astype(np.float64), 128)[: w.N, None]
            s *= np.repeat(sq["k_scale"][b, g].astype(np.float64), 64)[None, : w.N]
            s /= np.sqrt(w.d)
            if w.causal:
                s[np.triu_indices(w.N, 1)] = -np.inf
            p = np.exp(s - s.max(1, keepdims=True))
            refs.append(p @ vdq16[b, g] / p.sum(1, keepdims=True))
    ref = np.concatenate(refs)
    cos = (out * ref).sum() / np.sqrt((out * out).sum() * (ref * ref).sum())
    assert cos > 0.999, cos
    assert np.abs(out - ref).max() < 0.1
