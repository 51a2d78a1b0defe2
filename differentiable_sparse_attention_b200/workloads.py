"""Seeded synthetic inputs for alpha-entmax attention.

This module draws random numbers and nothing else: it holds none of the
method's arithmetic, so both the CUDA path and the float64 oracle can be fed
from it.  Every tensor is drawn on the CPU with ``torch.Generator`` in the fixed
order q, k, v, dO as N(0, 1) fp32 of shape [B, H, N, D]; a temperature scales q
before the cast to the compute dtype, and the planted workload mixes a shared
direction into q and into a few key blocks.

The AdaSplash-2 summaries benchmark on synthetic data over 4K-128K contexts
(zh §4.1, ja §4, es §4) without giving the generator; the workloads below
stand in for it.
"""

from __future__ import annotations

from dataclasses import dataclass, field, replace

import torch

_DTYPES = {"bf16": torch.bfloat16, "fp32": torch.float32}


@dataclass(frozen=True)
class Workload:
    """One synthetic attention problem: shapes, alpha, data recipe."""

    name: str
    B: int
    H: int
    N: int
    D: int
    dtype: str = "bf16"
    alpha: float = 1.5
    causal: bool = True
    block: int = 128
    temperature: float = 1.0
    planted_blocks: int = 0          # key blocks per head aligned with q
    planted_cos: float = 0.8         # cosine of q and planted keys with u
    seed: int = 0
    extra: dict = field(default_factory=dict, compare=False)

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)

    @property
    def torch_dtype(self):
        return _DTYPES[self.dtype]


# The five problem families.  Names describe the problem, not where it came from.
TINY_FP32 = Workload("tiny_fp32_n256_d64", B=1, H=2, N=256, D=64, dtype="fp32",
                     alpha=1.5, block=64)
ALPHA15_4K = Workload("alpha1.5_n4096_d64", B=2, H=16, N=4096, D=64, alpha=1.5)
SPARSEMAX_16K = Workload("alpha2_n16384_d128_t3", B=1, H=16, N=16384, D=128,
                         alpha=2.0, temperature=3.0)
PLANTED_32K = Workload("alpha1.5_n32768_d128_planted32", B=1, H=8, N=32768, D=128,
                       alpha=1.5, planted_blocks=32)
LONG_SWEEP = Workload("long_n{N}_alpha{alpha}_t4", B=1, H=8, N=65536, D=128,
                      alpha=1.5, temperature=4.0)

ALPHA15_4K_TEMPERATURES = (1.0, 2.0, 4.0)
LONG_SWEEP_POINTS = tuple((n, a) for a in (1.5, 2.0) for n in (65536, 131072))


def long_sweep_point(n: int, alpha: float) -> Workload:
    return LONG_SWEEP.with_(name=f"long_n{n}_alpha{alpha}_t4", N=n, alpha=alpha)


def make_inputs(w: Workload, device="cpu", need_grad_inputs: bool = True):
    """Draw (q, k, v, dout) for workload ``w`` and cast to its dtype.

    Returns a dict of CPU tensors (moved to ``device`` if given) with shapes
    [B, H, N, D], contiguous.  ``dout`` is omitted when need_grad_inputs is
    False (it is still drawn, so the other tensors do not change).
    """
    g = torch.Generator().manual_seed(w.seed)
    shape = (w.B, w.H, w.N, w.D)
    q = torch.randn(shape, generator=g, dtype=torch.float32)
    k = torch.randn(shape, generator=g, dtype=torch.float32)
    v = torch.randn(shape, generator=g, dtype=torch.float32)
    do = torch.randn(shape, generator=g, dtype=torch.float32)
    if w.planted_blocks:
        # One seeded unit direction u per head; every query and every key of
        # the planted blocks becomes cos*sqrt(D)*u + sin*noise, so that both
        # have cosine ~cos with u (noise vectors have norm ~sqrt(D)).
        u = torch.randn((w.B, w.H, 1, w.D), generator=g, dtype=torch.float32)
        u = u / u.norm(dim=-1, keepdim=True)
        c = w.planted_cos
        sn = (1.0 - c * c) ** 0.5
        scale = c * (w.D ** 0.5)
        q = scale * u + sn * q
        tc = (w.N + w.block - 1) // w.block
        nb = min(w.planted_blocks, tc)
        for b in range(w.B):
            for h in range(w.H):
                blocks = torch.randperm(tc, generator=g)[:nb]
                for j in blocks.tolist():
                    sl = slice(j * w.block, min(w.N, (j + 1) * w.block))
                    k[b, h, sl] = scale * u[b, h, 0] + sn * k[b, h, sl]
    if w.temperature != 1.0:
        q = q * w.temperature
    dt = w.torch_dtype
    out = {"q": q.to(dt).contiguous(), "k": k.to(dt).contiguous(),
           "v": v.to(dt).contiguous()}
    if need_grad_inputs:
        out["dout"] = do.to(dt).contiguous()
    if device != "cpu":
        out = {n: t.to(device) for n, t in out.items()}
    return out


def head_slice(t, b: int, h: int):
    """The [N, D] slice of one (batch, head) pair as float64 numpy."""
    return t[b, h].to(torch.float64).cpu().numpy()
