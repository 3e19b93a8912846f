"""Seeded synthetic inputs for linear attention -- shared by tests, bench and smoke.

This module holds none of the method's arithmetic: it draws normal samples,
scales them, adds the optional smooth 2-D offset of the vision-style workload,
rounds them to the storage dtype (round-to-nearest-even, via torch's cast) and
computes the per-head decay constants that the retention workloads are defined
with.  Both the CUDA path and the oracle receive exactly these tensors.

Every tensor gets its own stream: seed * 16 + id, with ids q=0, k=1, v=2, dO=3.
Samples are float32 standard normals from torch's CPU generator.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

STREAM_IDS = {"q": 0, "k": 1, "v": 2, "do": 3}

DTYPES = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


@dataclass(frozen=True)
class Workload:
    """One named synthetic workload (shapes, dtype and the input recipe)."""
    name: str
    op: str                      # "bidir" | "simple" | "retention" | "causal_norm" | "gated"
    B: int
    H: int
    T: int
    D: int
    dtype: str                   # "f32" | "f16" | "bf16"
    eps: float = 1e-6
    q_scale: float = 1.0
    k_scale: float = 1.0
    v_scale: float = 1.0
    vision_offset: bool = False  # smooth 2-D sinusoid on a sqrt(T) x sqrt(T) grid
    bwd: bool = True
    extra: dict = field(default_factory=dict)

    def with_T(self, T: int) -> "Workload":
        return Workload(self.name, self.op, self.B, self.H, T, self.D, self.dtype, self.eps,
                        self.q_scale, self.k_scale, self.v_scale, self.vision_offset, self.bwd, dict(self.extra))

    def with_shape(self, B=None, H=None, T=None, D=None) -> "Workload":
        return Workload(self.name, self.op, B or self.B, H or self.H, T if T is not None else self.T,
                        D or self.D, self.dtype, self.eps, self.q_scale, self.k_scale, self.v_scale,
                        self.vision_offset, self.bwd, dict(self.extra))


# The five workloads the library is specified against.
WORKLOADS = {
    # bidirectional, fp32, tiny: phi = elu+1, eps = 1e-6, inputs N(0,1)
    "bidir_f32_small": Workload("bidir_f32_small", "bidir", 1, 2, 256, 64, "f32"),
    # bidirectional, fp16 storage / fp32 accumulation, inputs 0.5*N(0,1), dO N(0,1)
    "bidir_f16": Workload("bidir_f16", "bidir", 8, 16, 4096, 64, "f16",
                          q_scale=0.5, k_scale=0.5, v_scale=0.5),
    # simple_la, bf16, q and k scaled by D^-1/2 (T swept 128 .. 16384)
    "simple_bf16": Workload("simple_bf16", "simple", 8, 16, 4096, 64, "bf16",
                            q_scale=64 ** -0.5, k_scale=64 ** -0.5),
    # retention, bf16, q scaled by D^-1/2 (T swept 128 .. 8192)
    "retention_bf16": Workload("retention_bf16", "retention", 8, 32, 2048, 128, "bf16",
                               q_scale=128 ** -0.5),
    # plain causal linear attention (the decay op with gamma = 1 on every head, no feature map,
    # no norm term), bf16, q scaled by D^-1/2, at the shape of the other causal workloads
    "causal_bf16": Workload("causal_bf16", "retention", 8, 16, 4096, 64, "bf16", q_scale=64 ** -0.5,
                            extra={"gamma": 1.0}),
    # causal linear attention with the norm term (phi = elu+1, no decay), the bidir recipe and shape
    "causal_norm_f16": Workload("causal_norm_f16", "causal_norm", 8, 16, 4096, 64, "f16",
                                q_scale=0.5, k_scale=0.5, v_scale=0.5),
    # gated linear attention, bf16: q scaled by D^-1/2, log gates log(sigmoid(N(0,1))) / 16 per token
    # and key dimension (about -0.04: decays near 0.96)
    "gated_bf16": Workload("gated_bf16", "gated", 8, 16, 4096, 64, "bf16", q_scale=64 ** -0.5),
    # the bidirectional and simple_la recipes at D = 128 (the head size the CUDA-core kernels cover)
    "bidir_f16_d128": Workload("bidir_f16_d128", "bidir", 8, 16, 4096, 128, "f16",
                               q_scale=0.5, k_scale=0.5, v_scale=0.5),
    "simple_bf16_d128": Workload("simple_bf16_d128", "simple", 8, 16, 4096, 128, "bf16",
                                 q_scale=128 ** -0.5, k_scale=128 ** -0.5),
    # vision-style long sequence, forward only, 256x256 token grid
    "vision_f16": Workload("vision_f16", "bidir", 2, 10, 65536, 64, "f16",
                           q_scale=0.5, k_scale=0.5, v_scale=0.5, vision_offset=True, bwd=False),
}

SIMPLE_T_SWEEP = (128, 256, 512, 1024, 2048, 4096, 8192, 16384)
RETENTION_T_SWEEP = (128, 256, 512, 1024, 2048, 4096, 8192)


def normal(shape, seed: int, stream: int) -> torch.Tensor:
    """float32 N(0,1) samples from torch's CPU generator, stream seed*16+stream."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed) * 16 + int(stream))
    return torch.randn(tuple(shape), generator=g, dtype=torch.float32)


def vision_offset(T: int, D: int, amplitude: float = 0.1) -> torch.Tensor:
    """[T, D] smooth 2-D offset for a flattened side x side token grid (T = side^2):
    token t = side*y + x gets amplitude * sin(2 pi y/side + pi d/D) * cos(2 pi x/side + pi d/(2D))."""
    side = int(round(math.sqrt(T)))
    if side * side != T:
        raise ValueError("vision offset needs a square token grid, T=%d" % T)
    t = torch.arange(T, dtype=torch.float64)
    y = torch.div(t, side, rounding_mode="floor")
    x = t - side * y
    d = torch.arange(D, dtype=torch.float64)
    a = torch.sin(2 * math.pi * y[:, None] / side + math.pi * d[None, :] / D)
    b = torch.cos(2 * math.pi * x[:, None] / side + math.pi * d[None, :] / (2 * D))
    return (amplitude * a * b).to(torch.float32)


def retention_gammas(H: int) -> torch.Tensor:
    """Per-head decay gamma_h = 1 - 2^(-5 - 7h/(H-1)), h = 0..H-1, computed in fp64 and
    stored as float32 (the value both sides use)."""
    if H == 1:
        return torch.tensor([1.0 - 2.0 ** -5], dtype=torch.float32)
    h = torch.arange(H, dtype=torch.float64)
    return (1.0 - torch.pow(2.0, -5.0 - 7.0 * h / (H - 1))).to(torch.float32)


def make_inputs(w: Workload, seed: int = 0, with_grad: bool | None = None) -> dict:
    """CPU tensors q, k, v (and do, gamma when relevant) in the workload's dtype."""
    dt = DTYPES[w.dtype]
    shape = (w.B, w.H, w.T, w.D)
    scales = {"q": w.q_scale, "k": w.k_scale, "v": w.v_scale, "do": 1.0}
    names = ["q", "k", "v"]
    if with_grad if with_grad is not None else w.bwd:
        names.append("do")
    off = vision_offset(w.T, w.D) if w.vision_offset else None
    out = {}
    for n in names:
        x = normal(shape, seed, STREAM_IDS[n])
        if scales[n] != 1.0:
            x = x * scales[n]
        if off is not None and n != "do":
            x = x + off
        out[n] = x.to(dt).contiguous()
    if w.op == "retention":
        g = w.extra.get("gamma")
        out["gamma"] = retention_gammas(w.H) if g is None else torch.full((w.H,), float(g), dtype=torch.float32)
    if w.op == "gated":
        out["g"] = (torch.nn.functional.logsigmoid(normal(shape, seed, 4)) / 16.0).to(dt).contiguous()
    return out
