"""Seeded synthetic inputs and the layer shapes they are drawn for.

This module holds random-number generation and shapes only -- none of the
layer's arithmetic -- so both the CUDA path and the fp64 oracle can consume
exactly the same values.  Tensors are produced on the host with a seeded
``torch.Generator`` and rounded once to the I/O dtype (round-to-nearest-even
for bf16); callers upload them or widen them to float64 as they need.

Shapes come from the Mamba-2 settings on the pages:
  * Nemotron feasibility report, section 1.4 (Nemotron 3 Nano: 64 heads x
    head_dim 64, d_state 128, conv 4, n_groups 8, chunk 128) and section 1.5
    (Nemotron-H 8B: d_model 4096, expand 2, d_state 128, head_dim 64);
  * the same report, section 2.2 (FRANKENSTALLM-H 3B proposal: 40 Mamba heads
    of 64 at d_model 2560, d_state 128, expand 2, conv 4).
Distributions (not given on the pages; a plain choice that keeps every stage
at unit scale): x ~ N(0,1); B, C ~ N(0,1)/sqrt(d_state); dt_raw ~ U(-4,-1)
with dt_bias 0; A = -exp(U(log 1, log 16)) per head, the default A range that
the hybrid-architecture summary's appendix E mentions ([0.01, 2] there is
offered as the long-memory variant); D ~ N(0,1); conv taps ~ N(0, 1/4).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class LayerShape:
    name: str
    b: int          # batch
    L: int          # sequence length (1 for decode)
    H: int          # heads
    P: int          # head dim
    N: int          # state size (d_state)
    G: int          # B/C groups
    Q: int          # chunk length of the SSD scan
    k: int          # conv width
    dtype: str      # I/O dtype: "f32" or "bf16"

    @property
    def d_inner(self) -> int:
        return self.H * self.P

    @property
    def conv_dim(self) -> int:
        return self.H * self.P + 2 * self.G * self.N

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    def with_(self, **kw) -> "LayerShape":
        return replace(self, **kw)


# The five workloads, in order.  Index 0 is the tiny fp32 correctness case,
# 1-3 are prefill layers, 4 is one decode token per sequence.
CONFIGS = [
    LayerShape("tiny_fp32_b1_L256_h4_n16", 1, 256, 4, 64, 16, 1, 64, 4, "f32"),
    LayerShape("frankenstallm_h_3b_b8_L2048_h40", 8, 2048, 40, 64, 128, 8, 128, 4, "bf16"),
    LayerShape("nemotron_h_8b_b4_L4096_h128", 4, 4096, 128, 64, 128, 8, 128, 4, "bf16"),
    LayerShape("nemotron3_nano_b1_L262144_h64", 1, 262144, 64, 64, 128, 8, 128, 4, "bf16"),
    LayerShape("decode_b256_h128", 256, 1, 128, 64, 128, 8, 128, 4, "bf16"),
]

SEED_BASE = 20260000


def config_seed(index: int) -> int:
    return SEED_BASE + index


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def _xbc(shape: LayerShape, lead: tuple, g: torch.Generator) -> torch.Tensor:
    """Pre-conv channels [x | B | C] with B, C scaled by 1/sqrt(N), in fp32."""
    t = torch.randn(*lead, shape.conv_dim, generator=g, dtype=torch.float32)
    t[..., shape.d_inner:] *= 1.0 / math.sqrt(shape.N)
    return t


def _a_log_uniform(H: int, lo: float, hi: float, g: torch.Generator) -> torch.Tensor:
    u = torch.rand(H, generator=g, dtype=torch.float64)
    return (-torch.exp(math.log(lo) + u * (math.log(hi) - math.log(lo)))).to(torch.float32)


def layer_inputs(shape: LayerShape, seed: int, *, conv_bias: bool = False,
                 conv_state: bool = False, init_state: bool = False,
                 a_range: tuple = (1.0, 16.0), dt_range: tuple = (-4.0, -1.0)) -> dict:
    """Inputs of one prefill layer call (conv1d+SiLU then the scan).

    Returns host tensors: xBC [b,L,conv_dim] (I/O dtype), w [conv_dim,k] f32,
    bias [conv_dim] f32 or None, conv_state [b,conv_dim,k] (I/O dtype) or None,
    dt_raw [b,L,H] (I/O dtype), dt_bias/A/D [H] f32, init_state [b,H,P,N] f32
    or None.
    """
    g = _gen(seed)
    s = shape
    io = s.torch_dtype
    out = {}
    out["xBC"] = _xbc(s, (s.b, s.L), g).to(io)
    out["w"] = torch.randn(s.conv_dim, s.k, generator=g) * 0.5
    out["dt_raw"] = (torch.rand(s.b, s.L, s.H, generator=g) * (dt_range[1] - dt_range[0]) + dt_range[0]).to(io)
    out["dt_bias"] = torch.zeros(s.H, dtype=torch.float32)
    out["A"] = _a_log_uniform(s.H, a_range[0], a_range[1], g)
    out["D"] = torch.randn(s.H, generator=g)
    out["bias"] = (torch.randn(s.conv_dim, generator=g) * math.sqrt(0.1)) if conv_bias else None
    out["conv_state"] = (_xbc(s, (s.b, s.k), g).transpose(1, 2).contiguous().to(io)) if conv_state else None
    out["init_state"] = (torch.randn(s.b, s.H, s.P, s.N, generator=g) * math.sqrt(0.1)) if init_state else None
    return out


def scan_inputs(shape: LayerShape, seed: int, *, init_state: bool = False,
                a_range: tuple = (1.0, 16.0), dt_range: tuple = (-4.0, -1.0),
                dt_bias: bool = False) -> dict:
    """Inputs of the scan alone, drawn directly (no conv): u [b,L,conv_dim]
    holding x | B | C channels (I/O dtype), dt_raw [b,L,H] (I/O dtype),
    dt_bias/A/D [H] f32, init_state [b,H,P,N] f32 or None."""
    g = _gen(seed)
    s = shape
    io = s.torch_dtype
    out = {}
    out["u"] = _xbc(s, (s.b, s.L), g).to(io)
    out["dt_raw"] = (torch.rand(s.b, s.L, s.H, generator=g) * (dt_range[1] - dt_range[0]) + dt_range[0]).to(io)
    out["dt_bias"] = (torch.randn(s.H, generator=g) * 0.5) if dt_bias else torch.zeros(s.H)
    out["A"] = _a_log_uniform(s.H, a_range[0], a_range[1], g)
    out["D"] = torch.randn(s.H, generator=g)
    out["init_state"] = (torch.randn(s.b, s.H, s.P, s.N, generator=g) * math.sqrt(0.1)) if init_state else None
    return out


def decode_inputs(shape: LayerShape, seed: int) -> dict:
    """Inputs of one decode token per sequence: ssm state [b,H,P,N] f32 ~ N(0,0.1),
    conv_state [b,conv_dim,k] and xBC [b,conv_dim] (I/O dtype) from the xBC
    distributions, dt_raw [b,H] (I/O dtype), w, dt_bias, A, D as for prefill."""
    g = _gen(seed)
    s = shape
    io = s.torch_dtype
    out = {}
    out["state"] = torch.randn(s.b, s.H, s.P, s.N, generator=g) * math.sqrt(0.1)
    out["conv_state"] = _xbc(s, (s.b, s.k), g).transpose(1, 2).contiguous().to(io)
    out["xBC"] = _xbc(s, (s.b,), g).to(io)
    out["w"] = torch.randn(s.conv_dim, s.k, generator=g) * 0.5
    out["dt_raw"] = (torch.rand(s.b, s.H, generator=g) * 3.0 - 4.0).to(io)
    out["dt_bias"] = torch.zeros(s.H, dtype=torch.float32)
    out["A"] = _a_log_uniform(s.H, 1.0, 16.0, g)
    out["D"] = torch.randn(s.H, generator=g)
    return out


def split_channels(u: torch.Tensor, shape: LayerShape):
    """Views of the x, B, C channel ranges of a [.., conv_dim] tensor."""
    s = shape
    x = u[..., : s.d_inner]
    B = u[..., s.d_inner: s.d_inner + s.G * s.N]
    C = u[..., s.d_inner + s.G * s.N:]
    return x, B, C


def mixer_inputs(shape: LayerShape, d_model: int, seed: int, *, conv_bias: bool = False,
                 conv_state: bool = False, init_state: bool = False) -> dict:
    """Inputs of the whole mixer (in_proj, the path, gated RMSNorm, out_proj),
    host tensors: hidden [b, L, d_model] ~ N(0, 1) (the block's pre-norm makes
    its input unit-scale), W_in [2HP + 2GN + H, d_model] bf16 whose rows give
    z and x ~ N(0, 1), B and C ~ N(0, 1)/sqrt(N) and dt_raw ~ N(0, 1/4)
    (the scan inputs' scales), dt_bias = -2.5 (dt around softplus(-2.5) =
    0.08, inside the scan workloads' dt range), W_out [d_model, HP] bf16 with
    N(0, 1/HP) entries, norm_w ~ 1 + N(0, 0.01), and the conv, A and D of the
    scan workloads."""
    g = _gen(seed)
    s = shape
    d_inner = s.H * s.P
    out = {}
    out["hidden"] = torch.randn(s.b, s.L, d_model, generator=g).to(torch.bfloat16)
    scale = torch.cat([torch.ones(d_inner + d_inner), torch.full((2 * s.G * s.N,), 1.0 / math.sqrt(s.N)),
                       torch.full((s.H,), 0.5)])
    W_in = torch.randn(2 * d_inner + 2 * s.G * s.N + s.H, d_model, generator=g) / math.sqrt(d_model)
    out["W_in"] = (W_in * scale[:, None]).to(torch.bfloat16)
    out["conv_w"] = torch.randn(s.conv_dim, s.k, generator=g) * 0.5
    out["conv_bias"] = (torch.randn(s.conv_dim, generator=g) * math.sqrt(0.1)) if conv_bias else None
    out["dt_bias"] = torch.full((s.H,), -2.5)
    out["A"] = _a_log_uniform(s.H, 1.0, 16.0, g)
    out["D"] = torch.randn(s.H, generator=g)
    out["norm_w"] = 1.0 + torch.randn(d_inner, generator=g) * 0.1
    out["W_out"] = (torch.randn(d_model, d_inner, generator=g) / math.sqrt(d_inner)).to(torch.bfloat16)
    out["conv_state"] = (_xbc(s, (s.b, s.k), g).transpose(1, 2).contiguous().to(torch.bfloat16)) if conv_state else None
    out["init_state"] = (torch.randn(s.b, s.H, s.P, s.N, generator=g) * math.sqrt(0.1)) if init_state else None
    return out


def ragged_lengths(total: int, seed: int, lo: int = 64, hi: int = 4096) -> list:
    """A serving-like prefill batch of `total` packed tokens: prompt lengths
    drawn log-uniformly from [lo, hi] until the next one would overflow the
    total, the last prompt taking what is left (the pages give no length
    mix; this one spans a chunk's 128 tokens on both sides)."""
    g = _gen(seed)
    lens, left = [], total
    while left > 0:
        u = float(torch.rand(1, generator=g))
        n = int(round(math.exp(math.log(lo) + u * (math.log(hi) - math.log(lo)))))
        n = min(n, left) if left - n >= lo else left
        lens.append(n)
        left -= n
    return lens
