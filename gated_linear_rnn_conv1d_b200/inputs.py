"""Seeded synthetic inputs for the RG-LRU temporal core.

This module only draws random numbers: it holds none of the layer's arithmetic.
The same draws feed the CUDA path and the CPU oracle, so both see identical
values (bf16 tensors are rounded here, once, and the oracle reads the rounded
values upcast exactly to float64).

Initialisation follows "Griffin：将门控线性循环与局部注意力混合以实现高效的语言模型",
§实门线性循环单元 (RG-LRU), parameterisation paragraph after Eq. (4):
  * W_a, W_x: LeCun normal, std = 1/sqrt(fan_in) (fan_in = D_RNN);
  * Λ such that a^c is uniform on [0.9, 0.999] with a = σ(Λ), c = 8:
    draw s ~ U[0.9, 0.999], a = s^(1/8), Λ = logit(a);
and the same page's §循环块 (recurrent block) for the width-4 Conv1D and the two
D → D_RNN linears plus the D_RNN → D output linear (LeCun normal, no biases).
Conv weights and bias are N(0, 1/4) (std 0.5); gate biases b_a = b_x = 0; x ~ N(0, 1).

Draw order (one torch CPU generator per workload, seeded):
    x, conv_w, conv_b, W_a, W_x, s(→Λ), [W_1, W_2, W_o, [γ₁, γ₂, W_gate, W_up, W_down]]
(the bracketed draws for the recurrent block and the Hawk residual layer). Each draw is float32 and is then cast to the IO dtype where the tensor is IO.
Decode inputs x_t for step k come from their own generator seeded 1_000_003 + k.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional

import torch

DECODE_SEED_BASE = 1_000_003


@dataclass
class RGLRUParams:
    """Per-layer parameters. conv_w is [4][R] (tap k multiplies x_{t-3+k});
    W_a, W_x are [R][R] row-major [out][in]; vectors are [R] float32."""
    conv_w: torch.Tensor
    conv_b: torch.Tensor
    W_a: torch.Tensor
    b_a: torch.Tensor
    W_x: torch.Tensor
    b_x: torch.Tensor
    Lambda: torch.Tensor


@dataclass
class Workload:
    name: str
    B: int
    T: int
    R: int
    io_dtype: torch.dtype
    x: torch.Tensor                      # [B][T][R] (or [B][T][D] for the block)
    params: RGLRUParams
    h0: torch.Tensor                     # [B][R] float32
    D: Optional[int] = None              # block model width
    W_1: Optional[torch.Tensor] = None   # [R][D]
    W_2: Optional[torch.Tensor] = None   # [R][D]
    W_o: Optional[torch.Tensor] = None   # [D][R]
    extra: dict = field(default_factory=dict)


def _normal(g: torch.Generator, shape, std: float) -> torch.Tensor:
    return torch.randn(*shape, generator=g, dtype=torch.float32) * std


def lambda_from_uniform(s: torch.Tensor) -> torch.Tensor:
    """Λ = logit(s^(1/8)) so that σ(Λ)^8 = s; computed in float64, stored fp32."""
    a = s.double() ** (1.0 / 8.0)
    return (torch.log(a) - torch.log1p(-a)).float()


def make_params(g: torch.Generator, R: int, io_dtype: torch.dtype,
                fan_in: Optional[int] = None) -> RGLRUParams:
    """Draws conv_w, conv_b, W_a, W_x, s(→Λ) in that order (the caller draws x first)."""
    fan_in = R if fan_in is None else fan_in
    conv_w = _normal(g, (4, R), 0.5)
    conv_b = _normal(g, (R,), 0.5)
    W_a = _normal(g, (R, R), 1.0 / math.sqrt(fan_in)).to(io_dtype)
    W_x = _normal(g, (R, R), 1.0 / math.sqrt(fan_in)).to(io_dtype)
    s = torch.empty(R, dtype=torch.float32).uniform_(0.9, 0.999, generator=g)
    Lam = lambda_from_uniform(s)
    zeros = torch.zeros(R, dtype=torch.float32)
    return RGLRUParams(conv_w, conv_b, W_a, zeros.clone(), W_x, zeros.clone(), Lam)


def make_forward(B: int, T: int, R: int, io_dtype: torch.dtype = torch.bfloat16,
                 seed: int = 0, name: str = "") -> Workload:
    g = torch.Generator("cpu").manual_seed(seed)
    x = _normal(g, (B, T, R), 1.0).to(io_dtype)
    p = make_params(g, R, io_dtype)
    h0 = torch.zeros(B, R, dtype=torch.float32)
    return Workload(name or f"rglru_fwd_B{B}_T{T}_R{R}", B, T, R, io_dtype, x, p, h0)


def make_block(B: int, T: int, D: int, R: int, io_dtype: torch.dtype = torch.bfloat16,
               seed: int = 0, name: str = "", g: Optional[torch.Generator] = None) -> Workload:
    g = torch.Generator("cpu").manual_seed(seed) if g is None else g
    x = _normal(g, (B, T, D), 1.0).to(io_dtype)
    p = make_params(g, R, io_dtype)
    W_1 = _normal(g, (R, D), 1.0 / math.sqrt(D)).to(io_dtype)
    W_2 = _normal(g, (R, D), 1.0 / math.sqrt(D)).to(io_dtype)
    W_o = _normal(g, (D, R), 1.0 / math.sqrt(R)).to(io_dtype)
    h0 = torch.zeros(B, R, dtype=torch.float32)
    return Workload(name or f"block_B{B}_T{T}_D{D}_R{R}", B, T, R, io_dtype, x, p, h0,
                    D=D, W_1=W_1, W_2=W_2, W_o=W_o)


def make_layer(B: int, T: int, D: int, R: int, M: int = 3, io_dtype: torch.dtype = torch.bfloat16,
               seed: int = 0, name: str = "") -> Workload:
    """One Hawk residual layer: the block's draws (same order as make_block), then the two
    RMSNorm gains ~ U[0.5, 1.5] (float32; a gain other than 1 keeps it visible in the
    output) and the gated MLP's linears, LeCun normal: W_gate, W_up [M·D][D] (std 1/√D),
    W_down [D][M·D] (std 1/√(M·D)). All of it goes to `extra`."""
    g = torch.Generator("cpu").manual_seed(seed)
    w = make_block(B, T, D, R, io_dtype, seed, name or f"layer_B{B}_T{T}_D{D}_R{R}_M{M}", g=g)
    H = M * D
    w.extra["norm1_scale"] = 0.5 + torch.rand(D, generator=g, dtype=torch.float32)
    w.extra["norm2_scale"] = 0.5 + torch.rand(D, generator=g, dtype=torch.float32)
    w.extra["W_gate"] = _normal(g, (H, D), 1.0 / math.sqrt(D)).to(io_dtype)
    w.extra["W_up"] = _normal(g, (H, D), 1.0 / math.sqrt(D)).to(io_dtype)
    w.extra["W_down"] = _normal(g, (D, H), 1.0 / math.sqrt(H)).to(io_dtype)
    return w


def make_decode(B: int, R: int, io_dtype: torch.dtype = torch.bfloat16, seed: int = 0,
                name: str = "") -> Workload:
    """Parameters for a decode run; the per-step tokens come from decode_token()."""
    g = torch.Generator("cpu").manual_seed(seed)
    p = make_params(g, R, io_dtype)
    h0 = torch.zeros(B, R, dtype=torch.float32)
    x = torch.zeros(B, 0, R, dtype=io_dtype)
    return Workload(name or f"rglru_decode_B{B}_R{R}", B, 0, R, io_dtype, x, p, h0)


def make_attention(D: int, M: int = 3, io_dtype: torch.dtype = torch.bfloat16, seed: int = 0,
                   layer: bool = True) -> dict:
    """Weights of Griffin's local-attention residual layer (D_head = 128, H = D/128 query
    heads, one key/value head), LeCun normal (std 1/√fan_in), drawn in the order W_q [D][D],
    W_k [128][D], W_v [128][D], W_o [D][D], then the two RMSNorm gains ~ U[0.5, 1.5] and
    the gated MLP as make_layer draws it (W_gate, W_up [M·D][D], W_down [D][M·D]). With
    layer=False only the attention block's four matrices are drawn (the same values). The
    decode tokens come from decode_token."""
    g = torch.Generator("cpu").manual_seed(seed)
    w = {"W_q": _normal(g, (D, D), 1.0 / math.sqrt(D)).to(io_dtype),
         "W_k": _normal(g, (128, D), 1.0 / math.sqrt(D)).to(io_dtype),
         "W_v": _normal(g, (128, D), 1.0 / math.sqrt(D)).to(io_dtype),
         "W_o": _normal(g, (D, D), 1.0 / math.sqrt(D)).to(io_dtype)}
    if not layer:
        return w
    w["norm1_scale"] = 0.5 + torch.rand(D, generator=g, dtype=torch.float32)
    w["norm2_scale"] = 0.5 + torch.rand(D, generator=g, dtype=torch.float32)
    H = M * D
    w["W_gate"] = _normal(g, (H, D), 1.0 / math.sqrt(D)).to(io_dtype)
    w["W_up"] = _normal(g, (H, D), 1.0 / math.sqrt(D)).to(io_dtype)
    w["W_down"] = _normal(g, (D, H), 1.0 / math.sqrt(H)).to(io_dtype)
    return w


def decode_token(step: int, B: int, R: int, io_dtype: torch.dtype = torch.bfloat16) -> torch.Tensor:
    g = torch.Generator("cpu").manual_seed(DECODE_SEED_BASE + step)
    return _normal(g, (B, R), 1.0).to(io_dtype)


# The five workloads the layer is measured and checked on.
CONFIGS = {
    "fwd_small_f32": dict(kind="forward", B=1, T=256, R=256, io="f32"),
    "fwd_hawk_bf16": dict(kind="forward", B=8, T=2048, R=2048, io="bf16"),
    "fwd_long_bf16": dict(kind="forward", B=1, T=32768, R=4096, io="bf16"),
    "decode_bf16": dict(kind="decode", B=256, R=4096, steps=1024, io="bf16"),
    "block_bf16": dict(kind="block", B=4, T=4096, D=4096, R=5632, io="bf16"),
}


def io_dtype_of(tag: str) -> torch.dtype:
    return {"f32": torch.float32, "bf16": torch.bfloat16}[tag]
