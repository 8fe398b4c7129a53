"""Seeded synthetic inputs for the quantized linear layer.

This module only draws numbers: it holds none of the method's arithmetic
(no scales, no codes, no outlier tests). Both the CPU oracle tests and the
CUDA path take their inputs from here, so the two sides see identical
tensors.

Shapes and value distributions follow the workloads of the model-card pages:
Qwen-Image-2.1 DiT projections at 1024^2 (4096 image + 256 text tokens,
hidden 3072, fused QKV 9216, MLP 12288) and Qwen3-VL text-encoder MLPs
(hidden 4096, MLP 12288). Massive activations (about 9000 and 13000 in
channel 2276 of two text-encoder tokens, about 9000 on DiT text tokens) come
from the "What 4-bit breaks here" section of the Image21-Turbo-OrbitQuant-W4A4
page. The weights, prompts and images of the real model are not available,
so every tensor is a seeded random draw of that shape.

Draw order inside one workload is fixed: X, then outlier positions and
values, then W, then any calibration draw. All draws use a CPU
``torch.Generator`` seeded per workload and are cast to the workload dtype
at the end (fp32 draw -> fp16/bf16, round to nearest even).
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict, List, Optional

import torch

__all__ = [
    "Linear", "Workload", "WORKLOADS", "make_x", "make_w", "make_linear",
    "make_calibration", "get_workload",
]


@dataclass(frozen=True)
class Linear:
    """One quantized linear: Y[M,N] = X[M,K] @ W[N,K]^T."""
    name: str
    M: int
    K: int
    N: int


@dataclass(frozen=True)
class Workload:
    """A named synthetic workload: its linears, dtype, mode and outlier recipe."""
    name: str
    mode: str                 # "int8_outlier" | "fp8_static" | "fp8_dynamic" | "w4a8" | "fp8_weight_only" | "fp_linear" | "nvfp4_weight_only"
    dtype: torch.dtype
    linears: List[Linear]
    seed: int
    # outlier recipe, applied on top of X ~ N(0, 1):
    fixed_channels: Optional[List[int]] = None     # channels set to +-U(lo, hi)
    fixed_tokens: int = 0                          # ... on this many random tokens
    fixed_range: tuple = (8.0, 12.0)
    random_channels: int = 0                       # random channels with |x| ~ U(lo, hi)
    random_token_frac: float = 0.0                 # ... on this fraction of tokens
    random_range: tuple = (8.0, 40.0)
    massive_text_tokens: int = 0                   # rows < text_prefix get one channel at +-massive
    text_prefix: int = 256
    massive_value: float = 9000.0
    massive_pairs: Optional[List[tuple]] = None    # explicit (token, channel, value) triples
    w_std: float = 0.02
    extra: Dict[str, object] = field(default_factory=dict)


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def _signs(g: torch.Generator, n: int) -> torch.Tensor:
    return torch.randint(0, 2, (n,), generator=g).to(torch.float32) * 2.0 - 1.0


def _uniform(g: torch.Generator, n: int, lo: float, hi: float) -> torch.Tensor:
    return torch.rand((n,), generator=g, dtype=torch.float32) * (hi - lo) + lo


def make_x(wl: Workload, M: int, K: int, g: torch.Generator) -> torch.Tensor:
    """X ~ N(0,1) [M,K] with the workload's outlier recipe, cast to wl.dtype."""
    x = torch.randn((M, K), generator=g, dtype=torch.float32)
    if wl.fixed_channels and wl.fixed_tokens > 0:
        ntok = min(wl.fixed_tokens, M)
        toks = torch.randperm(M, generator=g)[:ntok]
        for ch in wl.fixed_channels:
            if ch >= K:
                continue
            vals = _signs(g, ntok) * _uniform(g, ntok, *wl.fixed_range)
            x[toks, ch] = vals
    if wl.random_channels > 0 and wl.random_token_frac > 0:
        chans = torch.randperm(K, generator=g)[: wl.random_channels]
        ntok = max(1, int(round(wl.random_token_frac * M)))
        for ch in chans.tolist():
            toks = torch.randperm(M, generator=g)[:ntok]
            x[toks, ch] = _signs(g, ntok) * _uniform(g, ntok, *wl.random_range)
    if wl.massive_text_tokens > 0:
        prefix = min(wl.text_prefix, M)
        toks = torch.randperm(prefix, generator=g)[: wl.massive_text_tokens]
        chans = torch.randint(0, K, (toks.numel(),), generator=g)
        x[toks, chans] = _signs(g, toks.numel()) * wl.massive_value
    if wl.massive_pairs:
        for tok, ch, val in wl.massive_pairs:
            if tok < M and ch < K:
                x[tok, ch] = float(val)
    return x.to(wl.dtype)


def make_w(wl: Workload, N: int, K: int, g: torch.Generator) -> torch.Tensor:
    """W ~ N(0, w_std) [N,K], cast to wl.dtype."""
    return (torch.randn((N, K), generator=g, dtype=torch.float32) * wl.w_std).to(wl.dtype)


def make_linear(wl: Workload, lin: Linear, index: int = 0, M: Optional[int] = None):
    """Draw (X, W, bias) for one linear of a workload.

    ``index`` offsets the seed so every linear of a workload has its own draw;
    ``M`` overrides the token count (used for bounded samples). The bias is
    all-zero, as the workloads state.
    """
    g = _gen(wl.seed * 1000 + index)
    m = lin.M if M is None else M
    x = make_x(wl, m, lin.K, g)
    w = make_w(wl, lin.N, lin.K, g)
    bias = torch.zeros((lin.N,), dtype=wl.dtype)
    return x, w, bias


def make_calibration(wl: Workload, lin: Linear, index: int = 0, M: Optional[int] = None) -> torch.Tensor:
    """A separate seeded draw of X with the workload's distribution (for max calibration)."""
    g = _gen(wl.seed * 1000 + 500 + index)
    m = lin.M if M is None else M
    return make_x(wl, m, lin.K, g)


_TOK_1024 = 4096 + 256       # 1024^2 image: 64x64 latent patches + 256 text tokens
_TOK_2048 = 16384 + 256      # 2048^2 image: 128x128 latent patches + 256 text tokens
_H = 3072

WORKLOADS: Dict[str, Workload] = {
    # Tiny LLM.int8 linear that the CPU oracle finishes in well under a second.
    "tiny_int8": Workload(
        name="tiny_int8", mode="int8_outlier", dtype=torch.float16, seed=0,
        linears=[Linear("tiny", 64, 256, 512)],
        fixed_channels=[17, 200], fixed_tokens=10, fixed_range=(8.0, 12.0)),
    # LLM.int8 DiT MLP up- and down-projection at 1024^2.
    "dit1024_int8_mlp": Workload(
        name="dit1024_int8_mlp", mode="int8_outlier", dtype=torch.bfloat16, seed=1,
        linears=[Linear("mlp_up", _TOK_1024, _H, 4 * _H),
                 Linear("mlp_down", _TOK_1024, 4 * _H, _H)],
        random_channels=4, random_token_frac=0.05, random_range=(8.0, 40.0),
        massive_text_tokens=4, massive_value=9000.0),
    # FP8 E4M3 static per-tensor scales, DiT fused QKV at 1024^2.
    "dit1024_fp8_static_qkv": Workload(
        name="dit1024_fp8_static_qkv", mode="fp8_static", dtype=torch.bfloat16, seed=2,
        linears=[Linear("qkv", _TOK_1024, _H, 3 * _H)],
        fixed_channels=[17, 200], fixed_tokens=10, fixed_range=(8.0, 12.0)),
    # FP8 E4M3 per-channel weight scale + dynamic per-token activations,
    # Qwen3-VL text-encoder MLP with massive activations in channel 2276.
    "te_fp8_dynamic_mlp": Workload(
        name="te_fp8_dynamic_mlp", mode="fp8_dynamic", dtype=torch.bfloat16, seed=3,
        linears=[Linear("gate", 512, 4096, 12288), Linear("up", 512, 4096, 12288),
                 Linear("down", 512, 12288, 4096)],
        massive_pairs=[(5, 2276, 9000.0), (0, 2276, 13000.0)]),
    # One DiT block's four linears at 2048^2 (the sweep repeats it 32 times).
    "dit2048_block_int8": Workload(
        name="dit2048_block_int8", mode="int8_outlier", dtype=torch.bfloat16, seed=4,
        linears=[Linear("qkv", _TOK_2048, _H, 3 * _H), Linear("out", _TOK_2048, _H, _H),
                 Linear("mlp_up", _TOK_2048, _H, 4 * _H), Linear("mlp_down", _TOK_2048, 4 * _H, _H)],
        fixed_channels=[17, 200], fixed_tokens=10, fixed_range=(8.0, 12.0),
        extra={"blocks": 32}),
    "dit2048_block_w4a8": Workload(
        name="dit2048_block_w4a8", mode="w4a8", dtype=torch.bfloat16, seed=5,
        linears=[Linear("qkv", _TOK_2048, _H, 3 * _H), Linear("out", _TOK_2048, _H, _H),
                 Linear("mlp_up", _TOK_2048, _H, 4 * _H), Linear("mlp_down", _TOK_2048, 4 * _H, _H)],
        fixed_channels=[17, 200], fixed_tokens=10, fixed_range=(8.0, 12.0),
        extra={"blocks": 32, "group": 128}),
    # Weight-only FP8 (E4M3 weights, bf16 per-channel scales, bf16 activations)
    # at the text-encoder MLP shapes.
    "te_fp8_weight_only_mlp": Workload(
        name="te_fp8_weight_only_mlp", mode="fp8_weight_only", dtype=torch.bfloat16, seed=6,
        linears=[Linear("gate", 512, 4096, 12288), Linear("up", 512, 4096, 12288),
                 Linear("down", 512, 12288, 4096)],
        massive_pairs=[(5, 2276, 9000.0), (0, 2276, 13000.0)]),
    # NVFP4 weights (E2M1 codes, E4M3 per-16 and fp32 per-tensor scales) with
    # bf16 activations at the same text-encoder MLP shapes and inputs.
    "te_nvfp4_weight_only_mlp": Workload(
        name="te_nvfp4_weight_only_mlp", mode="nvfp4_weight_only", dtype=torch.bfloat16, seed=6,
        linears=[Linear("gate", 512, 4096, 12288), Linear("up", 512, 4096, 12288),
                 Linear("down", 512, 12288, 4096)],
        massive_pairs=[(5, 2276, 9000.0), (0, 2276, 13000.0)]),
    # The unquantised 16-bit linear (a layer kept in floating point) at the
    # DiT MLP shapes of 1024^2, bf16.
    "dit1024_bf16_mlp": Workload(
        name="dit1024_bf16_mlp", mode="fp_linear", dtype=torch.bfloat16, seed=7,
        linears=[Linear("mlp_up", _TOK_1024, _H, 4 * _H),
                 Linear("mlp_down", _TOK_1024, 4 * _H, _H)],
        random_channels=4, random_token_frac=0.05, random_range=(8.0, 40.0),
        massive_text_tokens=4, massive_value=9000.0),
}


def get_workload(name: str) -> Workload:
    return WORKLOADS[name]
