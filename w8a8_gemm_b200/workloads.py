"""Seeded synthetic inputs shaped like the DiT layers SegQuant quantizes.

This module holds none of the quantization method's arithmetic: it only draws
activations, calibration slices, weights, biases and SmoothQuant divisors, and
builds the segment tables.  Both the CUDA path and the CPU oracle receive the
same tensors from here.  Every tensor comes from its own
``torch.Generator('cpu').manual_seed(seed * 1000 + tensor_id)`` so that any one
of them can be re-drawn on its own.

Shapes and statistics follow the SegQuant pages:
  * activation polarity table ("SegQuant" papernotes.org, section DualScale):
    AdaNorm (DiT, SiLU) 0.955 negative-dominated channels, FFN (DiT, GELU) 0.744;
  * SiLU/GELU outputs reach about +3.5 but stay within about [-0.3, 0]
    (same page, research background);
  * SD3.5-medium: hidden 1536, FFN 6144, 24 heads x 64, 4096 image + 333 text
    tokens per sample, batch 2; FLUX: hidden 3072, FFN 12288, 24 heads x 128,
    4096 + 512 tokens.

The SmoothQuant divisor is part of the input recipe, not of the method: the
pages name SmoothQuant as a pluggable optimizer but print no formula, so the
usual migration rule d_c = sqrt(amax|X_c| / amax|W_c|) (alpha = 0.5) over the
calibration slice stands in for it, clamped to [1e-5, 1e5].
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import List, Optional

import torch
import torch.nn.functional as F

MODE_NONE, MODE_OUTPUT, MODE_INPUT = 0, 1, 2
CAL_ROWS = 64


def _gen(seed: int, tensor_id: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed * 1000 + tensor_id)
    return g


@dataclass
class Layer:
    """One quantized linear layer's inputs (all CPU tensors).

    x      bf16 [M][K]   activations
    x_cal  bf16 [64][K]  calibration slice, a separate draw of the same law
    w      bf16 [N][K]   nn.Linear weight
    bias   bf16 [N] or None
    d      fp32 [G][K] or None (SmoothQuant divisor per activation group)
    mode   0 none, 1 output-segmented, 2 input-segmented
    offsets segment boundaries over N (mode 1) or K (mode 2)
    G      activation groups (1, or the number of output segments)
    """
    name: str
    x: torch.Tensor
    x_cal: torch.Tensor
    w: torch.Tensor
    bias: Optional[torch.Tensor]
    d: Optional[torch.Tensor]
    mode: int
    offsets: List[int]
    G: int
    meta: dict = field(default_factory=dict)

    @property
    def M(self):
        return self.x.shape[0]

    @property
    def K(self):
        return self.x.shape[1]

    @property
    def N(self):
        return self.w.shape[0]

    @property
    def S(self):
        return len(self.offsets) - 1 if self.mode == MODE_INPUT else 1


def bits(t: torch.Tensor):
    """bf16 tensor -> numpy uint16 bit patterns (for the C oracle)."""
    import numpy as np
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def negative_dominated_fraction(x: torch.Tensor) -> float:
    """Share of channels in which more than half of the values are < 0."""
    return float(((x.float() < 0).float().mean(0) > 0.5).float().mean())


def _loguniform(n, lo, hi, g):
    u = torch.rand(n, generator=g, dtype=torch.float64)
    return torch.exp(math.log(lo) + u * (math.log(hi) - math.log(lo)))


def _smooth_divisor(x_cal: torch.Tensor, w_rows: torch.Tensor) -> torch.Tensor:
    ax = x_cal.float().abs().amax(0).clamp_min(1e-5)
    aw = w_rows.float().abs().amax(0).clamp_min(1e-5)
    return (ax.sqrt() / aw.sqrt()).clamp(1e-5, 1e5).float()


def _even_offsets(total: int, parts: int) -> List[int]:
    assert total % parts == 0
    step = total // parts
    return [i * step for i in range(parts + 1)]


# ----------------------------------------------------------------- activations
def gelu_gaussian_act(rows, K, sigma, g):
    z = torch.randn(rows, K, generator=g, dtype=torch.float32) * sigma
    return F.gelu(z, approximate="tanh").to(torch.bfloat16)


def gaussian_act(rows, K, sigma, g):
    return (torch.randn(rows, K, generator=g, dtype=torch.float32) * sigma).to(torch.bfloat16)


def silu_temb_act(rows, K, sign, g, unique_rows=None):
    """SiLU(t_emb) with t_emb[r, c] = sign_c * |z_rc|, z ~ N(0, 1).

    A plain N(0, 1) t_emb would give about 50% negative channels; the pages'
    AdaNorm (DiT) row has 95.5%, so each channel carries a sign drawn once."""
    r = unique_rows or rows
    z = torch.randn(r, K, generator=g, dtype=torch.float32).abs() * sign
    a = F.silu(z)
    if unique_rows and unique_rows < rows:
        reps = (rows + unique_rows - 1) // unique_rows
        a = a.repeat(reps, 1)[:rows]
    return a.to(torch.bfloat16)


# ------------------------------------------------------------------ layer kinds
def gelu_layer(name, M, K, N, seed, bias=False):
    """GELU(z), z ~ N(0, sigma_c), sigma_c log-uniform in [0.5, 3]; W ~ N(0, 0.02)."""
    sigma = _loguniform(K, 0.5, 3.0, _gen(seed, 1)).float()
    x = gelu_gaussian_act(M, K, sigma, _gen(seed, 2))
    x_cal = gelu_gaussian_act(CAL_ROWS, K, sigma, _gen(seed, 3))
    w = (torch.randn(N, K, generator=_gen(seed, 4)) * 0.02).to(torch.bfloat16)
    b = (torch.randn(N, generator=_gen(seed, 5)) * 0.02).to(torch.bfloat16) if bias else None
    return Layer(name, x, x_cal, w, b, None, MODE_NONE, [0, K], 1)


def adanorm_layer(name, M, K, N, n_seg, seed, G=None, unique_rows=2):
    """SiLU(t_emb) rows replicated to M; W split into n_seg output segments with
    per-segment weight std from {0.005, 0.02, 0.08}; per-group SmoothQuant d."""
    G = n_seg if G is None else G
    sign = torch.where(torch.rand(K, generator=_gen(seed, 1)) < 0.955, -1.0, 1.0)
    x = silu_temb_act(M, K, sign, _gen(seed, 2), unique_rows=unique_rows)
    x_cal = silu_temb_act(CAL_ROWS, K, sign, _gen(seed, 3))
    offs = _even_offsets(N, n_seg)
    choice = torch.randint(0, 3, (n_seg,), generator=_gen(seed, 4))
    stds = torch.tensor([0.005, 0.02, 0.08])[choice]
    w = torch.randn(N, K, generator=_gen(seed, 5))
    for j in range(n_seg):
        w[offs[j]:offs[j + 1]] *= stds[j]
    w = w.to(torch.bfloat16)
    b = (torch.randn(N, generator=_gen(seed, 6)) * 0.02).to(torch.bfloat16)
    if G == 1:
        d = _smooth_divisor(x_cal, w)[None]
    else:
        d = torch.stack([_smooth_divisor(x_cal, w[offs[j]:offs[j + 1]]) for j in range(n_seg)])
    return Layer(name, x, x_cal, w, b, d, MODE_OUTPUT, offs, G,
                 meta=dict(segment_weight_std=stds.tolist()))


def qkv_layer(name, M, K, N, n_seg, seed, G=None):
    """N(0, sigma_c) activations (sigma_c log-uniform [0.5, 3]); n_seg output
    segments (q, k, v) with per-group SmoothQuant d."""
    G = n_seg if G is None else G
    sigma = _loguniform(K, 0.5, 3.0, _gen(seed, 1)).float()
    x = gaussian_act(M, K, sigma, _gen(seed, 2))
    x_cal = gaussian_act(CAL_ROWS, K, sigma, _gen(seed, 3))
    offs = _even_offsets(N, n_seg)
    w = (torch.randn(N, K, generator=_gen(seed, 5)) * 0.02).to(torch.bfloat16)
    b = (torch.randn(N, generator=_gen(seed, 6)) * 0.02).to(torch.bfloat16)
    if G == 1:
        d = _smooth_divisor(x_cal, w)[None]
    else:
        d = torch.stack([_smooth_divisor(x_cal, w[offs[j]:offs[j + 1]]) for j in range(n_seg)])
    return Layer(name, x, x_cal, w, b, d, MODE_OUTPUT, offs, G)


def outproj_layer(name, M, K, N, head_dim, seed):
    """Concatenated attention heads: head h ~ N(0, sigma_h), sigma_h log-uniform
    in [0.2, 5]; 1% of channels scaled x20; K split into one input segment per
    head, each with its own SmoothQuant divisor and s+/s-."""
    assert K % head_dim == 0
    heads = K // head_dim
    sig_h = _loguniform(heads, 0.2, 5.0, _gen(seed, 1)).float()
    sigma = sig_h.repeat_interleave(head_dim)
    n_out = max(1, round(0.01 * K))
    out_idx = torch.randperm(K, generator=_gen(seed, 7))[:n_out]
    sigma[out_idx] *= 20.0
    x = gaussian_act(M, K, sigma, _gen(seed, 2))
    x_cal = gaussian_act(CAL_ROWS, K, sigma, _gen(seed, 3))
    w = (torch.randn(N, K, generator=_gen(seed, 5)) * 0.02).to(torch.bfloat16)
    b = (torch.randn(N, generator=_gen(seed, 6)) * 0.02).to(torch.bfloat16)
    d = _smooth_divisor(x_cal, w)[None]
    return Layer(name, x, x_cal, w, b, d, MODE_INPUT, _even_offsets(K, heads), 1,
                 meta=dict(outlier_channels=out_idx.tolist()))


def ffn_pair(prefix, M, hidden, ffn, seed):
    """FFN fc1 (hidden -> ffn) and fc2 (ffn -> hidden).

    fc1: X ~ N(0, sigma_c), sigma_c log-uniform [0.5, 3]; W1 ~ N(0, 0.02);
    b1 has sign -1 on 74.4% of channels (FFN (DiT) row of the polarity table)
    and magnitude |N(0, std(X W1))|.
    fc2: X = GELU(fc1 output).  The fc1 output is drawn per channel as
    b1_c + N(0, std(X W1)) rather than computed, so that no GEMM is needed to
    make inputs; its law matches the product's (a sum of K independent terms).
    """
    sigma = _loguniform(hidden, 0.5, 3.0, _gen(seed, 1)).float()
    x1 = gaussian_act(M, hidden, sigma, _gen(seed, 2))
    x1_cal = gaussian_act(CAL_ROWS, hidden, sigma, _gen(seed, 3))
    w1 = (torch.randn(ffn, hidden, generator=_gen(seed, 4)) * 0.02).to(torch.bfloat16)
    std_h = float(0.02 * sigma.double().pow(2).sum().sqrt())
    sgn = torch.where(torch.rand(ffn, generator=_gen(seed, 5)) < 0.744, -1.0, 1.0)
    b1 = (sgn * (torch.randn(ffn, generator=_gen(seed, 6)) * std_h).abs()).to(torch.bfloat16)
    fc1 = Layer(prefix + "fc1", x1, x1_cal, w1, b1, None, MODE_NONE, [0, hidden], 1)

    def fc2_act(rows, tid):
        z = b1.float()[None] + torch.randn(rows, ffn, generator=_gen(seed, tid)) * std_h
        return F.gelu(z, approximate="tanh").to(torch.bfloat16)

    x2 = fc2_act(M, 7)
    x2_cal = fc2_act(CAL_ROWS, 8)
    w2 = (torch.randn(hidden, ffn, generator=_gen(seed, 9)) * 0.02).to(torch.bfloat16)
    b2 = (torch.randn(hidden, generator=_gen(seed, 10)) * 0.02).to(torch.bfloat16)
    fc2 = Layer(prefix + "fc2", x2, x2_cal, w2, b2, None, MODE_NONE, [0, ffn], 1)
    return [fc1, fc2]


# ---------------------------------------------------------------- configurations
SD35_TOKENS = 2 * (4096 + 333)   # 8858
FLUX_TOKENS = 2 * (4096 + 512)   # 9216

CONFIGS = {
    "c1_tiny_dualscale": "GELU activations [256x1536] x W [1536x1536], one segment",
    "c2_sd35_adanorm": "SD3.5-medium AdaNorm, SiLU(t_emb) [2048x1536] x W [1536x9216], 6 output segments",
    "c3_sd35_attn_out": "SD3.5-medium attention out-projection [8858x1536] x W [1536x1536], 24 input segments",
    "c4_sd35_ffn": "SD3.5-medium FFN pair [8858x1536]->[6144]->[1536], one segment each",
    "c5_flux_block": "FLUX DiT block linears at M=9216: AdaNorm, QKV, out-proj, fc1, fc2",
    "c5_flux_adanorm_m2": "FLUX AdaNorm at its real batch M=2: SiLU(t_emb) [2x3072] x W "
                          "[3072x18432], 6 output segments (a latency point)",
}


def config_layers(name: str, seed: int = 0, G_output: Optional[int] = None) -> List[Layer]:
    """Layers of one named configuration.  G_output=1 forces one shared
    activation group on output-segmented layers (the pages' formula)."""
    if name == "c1_tiny_dualscale":
        return [gelu_layer("c1", 256, 1536, 1536, seed)]
    if name == "c2_sd35_adanorm":
        return [adanorm_layer("c2_adanorm", 2048, 1536, 9216, 6, seed, G=G_output)]
    if name == "c3_sd35_attn_out":
        return [outproj_layer("c3_attn_out", SD35_TOKENS, 1536, 1536, 64, seed)]
    if name == "c4_sd35_ffn":
        return ffn_pair("c4_", SD35_TOKENS, 1536, 6144, seed)
    if name == "c5_flux_block":
        M = FLUX_TOKENS
        return [adanorm_layer("c5_adanorm", M, 3072, 18432, 6, seed, G=G_output, unique_rows=M),
                qkv_layer("c5_qkv", M, 3072, 9216, 3, seed + 1, G=G_output),
                outproj_layer("c5_attn_out", M, 3072, 3072, 128, seed + 2),
                *ffn_pair("c5_", M, 3072, 12288, seed + 3)]
    if name == "c5_flux_adanorm_m2":
        return [adanorm_layer("c5_adanorm_m2", 2, 3072, 18432, 6, seed, G=G_output)]
    raise KeyError(f"unknown configuration {name!r}; known: {sorted(CONFIGS)}")
