"""Seeded synthetic inputs for the smoothed-K INT8 attention forward.

This module only draws random numbers: it holds none of the method's arithmetic (no smoothing, no
quantization, no attention), so both the CUDA path and the CPU oracle can be fed from it.

The pages measure on real models and long-context benchmarks that are not available here; these
synthetic workloads stand in for them, shaped like the long-context prefill they describe:

* ``tiny``      B=1, H=1, N=256, d=64, non-causal; Q, K, V ~ N(0,1); K plus a per-channel offset
                drawn once from N(0, 4) (variance 4).
* ``prefill4k`` B=4, H=32, N=4096, d=128, causal; Q, V ~ N(0,1); K ~ N(0,1) + offset N(0,4), then
                4 seeded outlier channels (whole channel, offset included) scaled x20.
* ``llama8b_32k`` B=1, H=32, Hkv=8 (GQA), N=32768, d=128, causal; K as ``prefill4k``.
* ``long128k``  B=1, H=32, Hkv=8, N=131072, d=128, causal; Q, K ~ Student-t(3)/sqrt(3) (unit
                variance); V ~ N(0,1); K offset N(0,4).
* ``wide64``    B=2, H=24, N=16384, d=64, non-causal; Q, K, V ~ N(0,1); K offset N(0,1); every
                512th token of K (n % 512 == 0) scaled x10 after the offset.

The offset vector (length d) and the outlier channel set are drawn once and shared by every
(batch, kv head).  Values are drawn in float32 and rounded to fp16.  Seeds default to
1000 + workload index (1..5).
"""
from __future__ import annotations

import dataclasses
import hashlib
from typing import Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    Hkv: int
    N: int
    d: int
    causal: bool
    qk_dist: str = "normal"          # "normal" or "student_t3"
    k_offset_var: float = 4.0        # variance of the per-channel K offset
    k_outlier_channels: int = 0      # number of K channels scaled by k_outlier_scale
    k_outlier_scale: float = 20.0
    k_token_stride: int = 0          # every k_token_stride-th K token is scaled by k_token_scale
    k_token_scale: float = 10.0
    seed: int = 1000

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    @property
    def ops(self) -> float:
        """Operation count of the metric: 4*B*H*N^2*d, halved for causal."""
        o = 4.0 * self.B * self.H * float(self.N) ** 2 * self.d
        return o / 2 if self.causal else o


WORKLOADS = {
    "tiny": Workload("tiny", 1, 1, 1, 256, 64, False, seed=1001),
    "prefill4k": Workload("prefill4k", 4, 32, 32, 4096, 128, True, k_outlier_channels=4,
                          seed=1002),
    "llama8b_32k": Workload("llama8b_32k", 1, 32, 8, 32768, 128, True, k_outlier_channels=4,
                            seed=1003),
    "long128k": Workload("long128k", 1, 32, 8, 131072, 128, True, qk_dist="student_t3",
                         seed=1004),
    "wide64": Workload("wide64", 2, 24, 24, 16384, 64, False, k_offset_var=1.0,
                       k_token_stride=512, seed=1005),
}
ORDER = ["tiny", "prefill4k", "llama8b_32k", "long128k", "wide64"]


def _draw(shape, dist: str, gen: torch.Generator, device) -> torch.Tensor:
    if dist == "normal":
        return torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    if dist == "student_t3":
        # t_3 = Z / sqrt(chi2_3 / 3); divided by sqrt(3) for unit variance: Z / sqrt(chi2_3).
        z = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
        chi = torch.zeros(shape, device=device, dtype=torch.float32)
        for _ in range(3):
            w = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
            chi.addcmul_(w, w)
        return z / chi.sqrt()
    raise ValueError(dist)


def make_inputs(w: Workload, device="cpu", seed: Optional[int] = None):
    """Returns (q, k, v) fp16 tensors on `device`: q [B,H,N,d], k and v [B,Hkv,N,d]."""
    seed = w.seed if seed is None else seed
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    d = w.d
    offset = torch.randn(d, generator=gen, device=device) * float(w.k_offset_var) ** 0.5
    scale_c = torch.ones(d, device=device)
    if w.k_outlier_channels:
        ch = torch.randperm(d, generator=gen, device=device)[: w.k_outlier_channels]
        scale_c[ch] = w.k_outlier_scale
    q = torch.empty(w.B, w.H, w.N, d, dtype=torch.float16, device=device)
    k = torch.empty(w.B, w.Hkv, w.N, d, dtype=torch.float16, device=device)
    v = torch.empty(w.B, w.Hkv, w.N, d, dtype=torch.float16, device=device)
    for b in range(w.B):
        for h in range(w.H):
            q[b, h] = _draw((w.N, d), w.qk_dist, gen, device).half()
        for g in range(w.Hkv):
            kk = _draw((w.N, d), w.qk_dist, gen, device)
            kk = (kk + offset) * scale_c
            if w.k_token_stride:
                kk[:: w.k_token_stride] *= w.k_token_scale
            k[b, g] = kk.half()
            v[b, g] = torch.randn((w.N, d), generator=gen, device=device).half()
    return q, k, v


def digest(*tensors: torch.Tensor) -> str:
    """SHA-256 of the tensors' bytes (for result records)."""
    h = hashlib.sha256()
    for t in tensors:
        h.update(t.detach().contiguous().cpu().view(torch.uint8).numpy().tobytes())
    return h.hexdigest()[:16]


def sample_rows(w: Workload, per_head: int, seed: int = 7, edge_first: int = 128,
                edge_last: int = 128):
    """Seeded query rows to compare on large workloads: per (b, h), the first `edge_first` and last
    `edge_last` rows of the sequence (clipped to N) plus `per_head` uniformly drawn rows.  Returns
    (row_bh, row_i) as int64 CPU tensors, sorted within each head."""
    gen = torch.Generator().manual_seed(seed)
    bh_all, i_all = [], []
    edge = torch.cat([torch.arange(0, min(edge_first, w.N)),
                      torch.arange(max(0, w.N - edge_last), w.N)])
    for bh in range(w.B * w.H):
        rnd = torch.randint(0, w.N, (per_head,), generator=gen)
        rows = torch.unique(torch.cat([edge, rnd]))
        bh_all.append(torch.full_like(rows, bh))
        i_all.append(rows)
    return torch.cat(bh_all).long(), torch.cat(i_all).long()
