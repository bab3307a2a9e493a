"""Block-sparse attention on the GPU against the oracle.

Key tiles are selected per 256-row query block by the block-mean importance score (the
heuristic block selection of the page "ThriftAttention: Selective Mixed Precision for
Long-Context FP4 Attention", method section), top-k plus the causal diagonals, and only those
tiles are computed (the sparse top-k variant its results section compares against).
 * the selection lists and counts are index work: bit-exact against the oracle;
 * the attention over the selected tiles: within the same tolerance as the dense path, against
   the oracle's attention restricted to the same tile mask on the oracle's own int8 codes;
 * with every tile listed, the sparse kernel reproduces the dense kernel bit for bit;
 * a query block whose list is empty has no key: its rows come out as zeros;
 * at full size (llama8b_32k top-16, long128k top-64, the bench's sparse modes) the lists are
   compared in full and a seeded sample of output rows against the oracle.
"""
import numpy as np
import pytest
import torch

from bit_quantized_attention_smoothing_b200.workloads import WORKLOADS, make_inputs, sample_rows
from conftest import check_output, np16

pytestmark = pytest.mark.gpu

CASES = [
    ("tiny", {"N": 1000, "causal": True}, 2),
    ("tiny", {"N": 1000, "causal": False}, 3),
    ("prefill4k", {"B": 1, "H": 4, "Hkv": 2, "N": 1500}, 1),
    ("llama8b_32k", {"H": 4, "Hkv": 1, "N": 2048}, 4),
    ("wide64", {"B": 2, "H": 2, "Hkv": 1, "N": 700, "causal": True}, 0),
    ("long128k", {"H": 2, "Hkv": 1, "N": 3000}, 5),
]
IDS = [f"{n}-" + "-".join(f"{k}{v}" for k, v in o.items()) + f"-top{t}" for n, o, t in CASES]


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from bit_quantized_attention_smoothing_b200 import qattn as Q
    Q.load()
    return Q


def _lists_equal(got_l, got_c, ref_l, ref_c):
    got_l, got_c = got_l.cpu().numpy(), got_c.cpu().numpy()
    assert np.array_equal(got_c, ref_c)
    for bh in range(ref_c.shape[0]):
        for i in range(ref_c.shape[1]):
            n = ref_c[bh, i]
            assert np.array_equal(got_l[bh, i, :n], ref_l[bh, i, :n]), (bh, i)


@pytest.mark.parametrize("name,over,topk", CASES, ids=IDS)
def test_block_select_bit_exact(lib, oracle, name, over, topk):
    w = WORKLOADS[name].with_(**over)
    q, k, _ = make_inputs(w)
    gl, gc = lib.qattn_block_select(q.cuda(), k.cuda(), topk, causal=w.causal)
    torch.cuda.synchronize()
    rl, rc = oracle.block_select(np16(q), np16(k), w.B, w.H, w.Hkv, w.N, w.d, w.causal, topk)
    _lists_equal(gl, gc, rl, rc)


@pytest.mark.parametrize("name,over,topk", CASES, ids=IDS)
def test_sparse_attention_vs_oracle(lib, oracle, name, over, topk):
    w = WORKLOADS[name].with_(**over)
    q, k, v = make_inputs(w)
    sq = oracle.smooth_quant(np16(q), np16(k), w.B, w.H, w.Hkv, w.N, w.d)
    rl, rc = oracle.block_select(np16(q), np16(k), w.B, w.H, w.Hkv, w.N, w.d, w.causal, topk)
    mask = oracle.tile_mask(rl, rc, w.N)
    t = {key: torch.from_numpy(val).cuda() for key, val in sq.items()}
    out = lib.qattn_attn_quantized_sparse(t["q_i8"], t["q_scale"], t["k_i8"], t["k_scale"],
                                          v.cuda(), torch.from_numpy(rl).cuda(),
                                          torch.from_numpy(rc).cuda(), causal=w.causal)
    assert lib.qattn_check_device_status() == 0
    ref = oracle.attention_quantized_sparse(sq["q_i8"], sq["q_scale"], sq["k_i8"], sq["k_scale"],
                                            np16(v), w.B, w.H, w.Hkv, w.N, w.d, w.causal, mask)
    ok, msg = check_output(out.float().cpu().numpy().reshape(-1, w.d), ref)
    assert ok, msg


@pytest.mark.parametrize("causal", [False, True])
def test_all_tiles_listed_equals_dense(lib, causal):
    w = WORKLOADS["prefill4k"].with_(B=1, H=2, Hkv=1, N=1200, causal=causal)
    q, k, v = (t.cuda() for t in make_inputs(w))
    q_i8, q_s, k_i8, k_s, _ = lib.qattn_smooth_quant(q, k)
    kl, kc = lib.qattn_block_select(q, k, 10 ** 6, causal=causal)
    dense = lib.qattn_attn_quantized(q_i8, q_s, k_i8, k_s, v, causal=causal)
    sparse = lib.qattn_attn_quantized_sparse(q_i8, q_s, k_i8, k_s, v, kl, kc, causal=causal)
    torch.cuda.synchronize()
    assert torch.equal(dense, sparse)


@pytest.mark.parametrize("causal,topk", [(True, 2), (False, 3), (True, 0)])
def test_forward_sparse_one_call_equals_the_three_calls(lib, causal, topk):
    """qattn_forward_sparse (one call, its own workspace) gives the same output, bit for bit, as
    smoothing + quantization, selection and the sparse attention called one by one."""
    w = WORKLOADS["llama8b_32k"].with_(H=4, Hkv=2, N=1300, causal=causal)
    q, k, v = (t.cuda() for t in make_inputs(w))
    q_i8, q_s, k_i8, k_s, _ = lib.qattn_smooth_quant(q, k)
    kl, kc = lib.qattn_block_select(q, k, topk, causal=causal)
    ref = lib.qattn_attn_quantized_sparse(q_i8, q_s, k_i8, k_s, v, kl, kc, causal=causal)
    got = lib.qattn_forward_sparse(q, k, v, topk, causal=causal)
    torch.cuda.synchronize()
    assert torch.equal(got, ref)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("pattern", ["all_equal", "two_kinds"])
def test_block_select_ties_bit_exact(lib, oracle, causal, pattern):
    """Equal scores: K built from repeated 128-row tiles, so key tiles share their block means and
    their scores tie exactly; the selection must take the lowest-indexed among equal scores, as
    the oracle does."""
    w = WORKLOADS["tiny"].with_(B=1, H=2, Hkv=1, N=128 * 24, d=128, causal=causal)
    q, k, _ = make_inputs(w)
    tile = k[:, :, :128, :]
    if pattern == "all_equal":
        k = tile.repeat(1, 1, 24, 1).contiguous()
    else:
        other = k[:, :, 128:256, :]
        k = torch.cat([tile if (t % 3) else other for t in range(24)], dim=2).contiguous()
    for topk in (1, 3, 7):
        gl, gc = lib.qattn_block_select(q.cuda(), k.cuda(), topk, causal=causal)
        torch.cuda.synchronize()
        rl, rc = oracle.block_select(np16(q), np16(k), w.B, w.H, w.Hkv, w.N, w.d, causal, topk)
        _lists_equal(gl, gc, rl, rc)


@pytest.mark.parametrize("causal", [False, True])
def test_empty_lists_give_zero_rows(lib, causal):
    """Query blocks whose kv_count is 0 (lists a caller built; the selection never writes one)
    have no key to attend to: the kernel writes their rows as zeros and reports no error; the
    other blocks are unaffected (equal to the dense kernel, since they list every tile)."""
    w = WORKLOADS["prefill4k"].with_(B=1, H=2, Hkv=1, N=1000, causal=causal)
    q, k, v = (t.cuda() for t in make_inputs(w))
    q_i8, q_s, k_i8, k_s, _ = lib.qattn_smooth_quant(q, k)
    kl, kc = lib.qattn_block_select(q, k, 10 ** 6, causal=causal)
    kc[:, 1] = 0        # rows 256 .. 511 of both heads
    dense = lib.qattn_attn_quantized(q_i8, q_s, k_i8, k_s, v, causal=causal)
    sparse = lib.qattn_attn_quantized_sparse(q_i8, q_s, k_i8, k_s, v, kl, kc, causal=causal)
    torch.cuda.synchronize()
    assert lib.qattn_check_device_status() == 0
    assert torch.count_nonzero(sparse[:, :, 256:512]) == 0
    assert torch.equal(sparse[:, :, :256], dense[:, :, :256])
    assert torch.equal(sparse[:, :, 512:], dense[:, :, 512:])


@pytest.mark.parametrize("name,topk", [("llama8b_32k", 16), ("long128k", 64)])
def test_full_size_sparse(lib, oracle, name, topk):
    """The bench's block-sparse modes at full size: every list and count bit-exact against the
    oracle's selection, then the one-call sparse forward on a seeded sample of rows per head (the
    first and last rows of the sequence and random ones) against the oracle's attention restricted
    to the same tiles."""
    w = WORKLOADS[name]
    q, k, v = make_inputs(w, device="cuda")
    gl, gc = lib.qattn_block_select(q, k, topk, causal=w.causal)
    torch.cuda.synchronize()
    qh, kh, vh = np16(q), np16(k), np16(v)
    rl, rc = oracle.block_select(qh, kh, w.B, w.H, w.Hkv, w.N, w.d, w.causal, topk)
    _lists_equal(gl, gc, rl, rc)
    del gl, gc
    out = lib.qattn_forward_sparse(q, k, v, topk, causal=w.causal)
    assert lib.qattn_check_device_status() == 0
    rows = tuple(t.numpy() for t in sample_rows(w, 8, edge_first=8, edge_last=8))
    flat = out.reshape(-1, w.d)
    got = flat[torch.as_tensor(rows[0] * w.N + rows[1], device=out.device)].float().cpu().numpy()
    del out, flat, q, k, v
    sq = oracle.smooth_quant(qh, kh, w.B, w.H, w.Hkv, w.N, w.d)
    ref = oracle.attention_quantized_sparse(sq["q_i8"], sq["q_scale"], sq["k_i8"], sq["k_scale"],
                                            vh, w.B, w.H, w.Hkv, w.N, w.d, w.causal,
                                            oracle.tile_mask(rl, rc, w.N), rows=rows)
    ok, msg = check_output(got, ref)
    print(name, f"top{topk}", msg)
    assert ok, msg
