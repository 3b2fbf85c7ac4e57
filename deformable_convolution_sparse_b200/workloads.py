"""Seeded synthetic inputs for the DCNv4 aggregation (forward and backward).

This module only draws random numbers in the shapes the operator takes. It
holds none of the operator's arithmetic: the output extent of every named
workload is written here as a literal and the tests check it against both the
library's and the oracle's own output-size functions; the generic generator
takes Hout/Wout from its caller.

Workloads (shapes and value distributions of the pages' use cases; no dataset
or trained weights are involved, the random values stand in for activations
and for the predictor's offsets and masks):
  tiny_f32     N=1  H=W=8   C=16  G=2  K=3 pad 1; offsets U[-2,2], masks N(0,1), seed 0
  stage1       N=64 H=W=56  C=64  G=4  K=3 pad 1; offsets N(0,1.5^2), masks N(0,0.5^2), seed 1
               (FlashInternImage-T stage 1 shape: GROUPS[0] = 4)
  stage3       N=64 H=W=14  C=256 G=16 K=3 pad 1; offsets N(0,1), masks N(0,0.5^2), seed 2
               (FlashInternImage-T stage 3 shape: GROUPS[2] = 16)
  sd_latent    N=8  H=W=64  C=320 G=8  K=3 pad 1; offsets U[-4,4], masks N(0,1/8), seed 3
               (Stable Diffusion 1.5 latent U-Net block)
  highres      N=2  H=W=256 C=128 G=8  K=3 pad 1 dilation 2; offsets U[-8,8], masks N(0,1), seed 4
x ~ N(0,1) everywhere. Draw order on one CPU torch.Generator: x [N,H,W,C],
then offsets [N,Hout,Wout,G,2*K*K], then masks [N,Hout,Wout,G,K*K], all
fp32; offsets and masks are concatenated on the last axis and the tensors are
then rounded to the storage dtype. The backward's upstream gradient
dL/dout ~ N(0,1) [N,Hout,Wout,C] comes from a second generator seeded with
1000 + seed.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import torch

DTYPES = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


@dataclass(frozen=True)
class Workload:
    name: str
    dtype: str
    N: int
    H: int
    W: int
    C: int
    G: int
    K: int
    stride: int
    pad: int
    dilation: int
    offset_scale: float
    Hout: int
    Wout: int
    offsets: tuple  # ("normal", mean, std) or ("uniform", lo, hi)
    masks: tuple
    seed: int

    @property
    def Cg(self) -> int:
        return self.C // self.G

    @property
    def points(self) -> int:
        """Sampling points: one per (n, ho, wo, g, k)."""
        return self.N * self.Hout * self.Wout * self.G * self.K * self.K

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    def algorithmic_bytes(self) -> int:
        """x read once + offset_mask read once + out written once."""
        e = self.elem_bytes
        x = self.N * self.H * self.W * self.C
        om = self.N * self.Hout * self.Wout * self.G * 3 * self.K * self.K
        out = self.N * self.Hout * self.Wout * self.C
        return (x + om + out) * e

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)

    def kwargs(self) -> dict:
        return dict(G=self.G, K=self.K, stride=self.stride, pad=self.pad,
                    dilation=self.dilation, offset_scale=self.offset_scale)


WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", "f32", 1, 8, 8, 16, 2, 3, 1, 1, 1, 1.0, 8, 8,
                         ("uniform", -2.0, 2.0), ("normal", 0.0, 1.0), 0),
    "stage1_f32": Workload("stage1_f32", "f32", 64, 56, 56, 64, 4, 3, 1, 1, 1, 1.0, 56, 56,
                           ("normal", 0.0, 1.5), ("normal", 0.0, 0.5), 1),
    "stage1_f16": Workload("stage1_f16", "f16", 64, 56, 56, 64, 4, 3, 1, 1, 1, 1.0, 56, 56,
                           ("normal", 0.0, 1.5), ("normal", 0.0, 0.5), 1),
    "stage3_f16": Workload("stage3_f16", "f16", 64, 14, 14, 256, 16, 3, 1, 1, 1, 1.0, 14, 14,
                           ("normal", 0.0, 1.0), ("normal", 0.0, 0.5), 2),
    "sd_latent_f16": Workload("sd_latent_f16", "f16", 8, 64, 64, 320, 8, 3, 1, 1, 1, 1.0, 64, 64,
                              ("uniform", -4.0, 4.0), ("normal", 0.0, (1.0 / 8.0) ** 0.5), 3),
    "highres_bf16": Workload("highres_bf16", "bf16", 2, 256, 256, 128, 8, 3, 1, 1, 2, 1.0, 254, 254,
                             ("uniform", -8.0, 8.0), ("normal", 0.0, 1.0), 4),
}

# the workload the throughput benchmark times
BENCH_WORKLOAD = "stage1_f16"


def _draw(gen: torch.Generator, shape, dist) -> torch.Tensor:
    kind, a, b = dist
    if kind == "normal":
        return torch.randn(shape, generator=gen, dtype=torch.float32) * float(b) + float(a)
    if kind == "uniform":
        return torch.rand(shape, generator=gen, dtype=torch.float32) * float(b - a) + float(a)
    if kind == "zeros":
        return torch.zeros(shape, dtype=torch.float32)
    raise ValueError(f"unknown distribution {kind!r}")


def make_inputs(N: int, H: int, W: int, C: int, G: int, K: int, Hout: int, Wout: int,
                dtype: str = "f32", offsets=("normal", 0.0, 1.0), masks=("normal", 0.0, 1.0),
                x_dist=("normal", 0.0, 1.0), seed: int = 0, points: int | None = None):
    """Return (x [N,H,W,C], offset_mask [N,Hout,Wout,G,3*P]) as CPU tensors in ``dtype``.

    P = ``points`` (default K*K; K*K - 1 for the variant without the centre point).
    """
    P = K * K if points is None else int(points)
    gen = torch.Generator(device="cpu")
    gen.manual_seed(int(seed))
    x = _draw(gen, (N, H, W, C), x_dist)
    off = _draw(gen, (N, Hout, Wout, G, 2 * P), offsets)
    msk = _draw(gen, (N, Hout, Wout, G, P), masks)
    om = torch.cat([off, msk], dim=-1)
    t = DTYPES[dtype]
    return x.to(t).contiguous(), om.to(t).contiguous()


def workload_inputs(w: Workload):
    """Seeded inputs of a named workload (CPU tensors in its storage dtype)."""
    return make_inputs(w.N, w.H, w.W, w.C, w.G, w.K, w.Hout, w.Wout, w.dtype,
                       w.offsets, w.masks, seed=w.seed)


def make_grad_out(N: int, Hout: int, Wout: int, C: int, dtype: str = "f32", seed: int = 0,
                  dist=("normal", 0.0, 1.0)) -> torch.Tensor:
    """Seeded upstream gradient dL/dout [N,Hout,Wout,C] (CPU tensor in ``dtype``) for the backward.

    Drawn on its own generator, seeded with 1000 + seed, so that it does not
    shift the draws of ``make_inputs``.
    """
    gen = torch.Generator(device="cpu")
    gen.manual_seed(1000 + int(seed))
    return _draw(gen, (N, Hout, Wout, C), dist).to(DTYPES[dtype]).contiguous()


def workload_grad_out(w: Workload) -> torch.Tensor:
    """Seeded dL/dout of a named workload (CPU tensor in its storage dtype)."""
    return make_grad_out(w.N, w.Hout, w.Wout, w.C, w.dtype, seed=w.seed)


def make_center_logit(N: int, Hout: int, Wout: int, G: int, dtype: str = "f32", seed: int = 0,
                      dist=("normal", 0.0, 1.5)) -> torch.Tensor:
    """Seeded gate logits [N,Hout,Wout,G] for centre feature scaling (own generator, seed 2000 + seed)."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(2000 + int(seed))
    return _draw(gen, (N, Hout, Wout, G), dist).to(DTYPES[dtype]).contiguous()


def make_inputs_on(device, N: int, H: int, W: int, C: int, G: int, K: int, Hout: int, Wout: int,
                   dtype: str = "f16", offsets=("normal", 0.0, 1.0), masks=("normal", 0.0, 1.0), seed: int = 0):
    """``make_inputs`` drawn directly on ``device`` (a seeded generator of that device) for batches too large
    to draw on the host; the same draw order (x, offsets, masks), a different random stream."""
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))

    def draw(shape, dist):
        kind, a, b = dist
        if kind == "normal":
            return torch.randn(shape, generator=gen, device=device) * float(b) + float(a)
        return torch.rand(shape, generator=gen, device=device) * float(b - a) + float(a)

    t = DTYPES[dtype]
    x = draw((N, H, W, C), ("normal", 0.0, 1.0)).to(t)
    om = torch.empty((N, Hout, Wout, G, 3 * K * K), dtype=t, device=device)
    om[..., :2 * K * K] = draw((N, Hout, Wout, G, 2 * K * K), offsets).to(t)
    om[..., 2 * K * K:] = draw((N, Hout, Wout, G, K * K), masks).to(t)
    return x, om
