"""Seeded synthetic workloads shaped like the DiT projections the OrbitQuant pages evaluate.

This module holds ONLY input generation: it contains none of the quantizer's arithmetic, so
both the CUDA path and the fp64 oracle can be fed the same bytes from it.  Everything is
drawn on the CPU with ``torch.Generator`` in fp32 and, for bf16 workloads, cast to bf16 with
round-to-nearest-even.

Workload shapes stand in for the FLUX.1 / Wan 2.1 projections named by the rcap.io summary
"OrbitQuant: Data-Agnostic Quantization for Image and Video" (image DiT at W4A4 and W2A4,
video DiT) and the W4A8 FLUX-3-Klein card; no dataset or checkpoint is used.

Seeds: the seed of stream k (1 activations, 2 weights, 3 outlier-channel set, 4 per-token
scale, 5 second per-token scale) of projection p of workload c is 1000*c + 100*p + k.  Rows
are drawn in chunks of ``CHUNK`` rows, chunk j seeded with (seed * 1_000_003 + j), so any
subset of rows can be regenerated without drawing the whole matrix.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence

import numpy as np
import torch

CHUNK = 4096


@dataclasses.dataclass(frozen=True)
class Projection:
    """One linear layer of a workload: T tokens of dimension d into `out` features."""
    name: str
    T: int
    d: int
    out: int
    h: int
    bits_w: int
    bits_a: int
    dtype: torch.dtype
    outlier_count: int          # channels scaled by outlier_scale, shared by all tokens
    outlier_scale: float
    token_scale: str            # "none" | "lognormal" | "lognormal_cfg" (two halves)
    gelu: bool = False          # x = GELU_erf(z) before the per-token scale
    w_outlier_rows: int = 0     # weight rows scaled by w_outlier_scale
    w_outlier_scale: float = 1.0
    cfg: int = 0
    proj: int = 0
    # variants of the path (how the projection is quantized, not how its data are drawn)
    rotation: str = "rpbh"      # "rpbh" | "block_rht" (identity permutation)
    marginal: str = "gauss"     # codebook target: "gauss" (N(0, 1/d)) | "exact" (f_d)
    fused_gelu: bool = False    # rows are pre-activations; the quantizer applies GELU itself


def _outliers(d: int, frac: float) -> int:
    return int(round(frac * d))


def _bf16():
    return torch.bfloat16


# Workloads.  C1 toy, C2 FLUX attention projection, C3 FLUX MLP (up, down), C4 video FFN
# (up, down; W3A4 and W4A8 variants), C5 is the activation-only sweep (see sweep_points()).
WORKLOADS = {
    "toy_w4a4": [Projection("toy_w4a4", 64, 256, 256, 64, 4, 4, torch.float32, 4, 30.0,
                            "none", w_outlier_rows=2, w_outlier_scale=10.0, cfg=1, proj=0)],
    "flux_attn_w4a4": [Projection("flux_attn_w4a4", 4608, 3072, 3072, 128, 4, 4, _bf16(),
                                  _outliers(3072, 0.01), 50.0, "lognormal", cfg=2, proj=0)],
    "flux_mlp_w2a4": [
        Projection("flux_mlp_up_w2a4", 4608, 3072, 12288, 128, 2, 4, _bf16(),
                   _outliers(3072, 0.01), 50.0, "lognormal", cfg=3, proj=0),
        Projection("flux_mlp_down_w2a4", 4608, 12288, 3072, 128, 2, 4, _bf16(),
                   _outliers(12288, 0.01), 50.0, "lognormal", gelu=True, cfg=3, proj=1),
    ],
    "video_ffn_w3a4": [
        Projection("video_ffn_up_w3a4", 65520, 5120, 13824, 128, 3, 4, _bf16(),
                   _outliers(5120, 0.005), 100.0, "lognormal_cfg", cfg=4, proj=0),
        Projection("video_ffn_down_w3a4", 65520, 13824, 5120, 128, 3, 4, _bf16(),
                   _outliers(13824, 0.005), 100.0, "lognormal_cfg", cfg=4, proj=1),
    ],
    # The MLP down projection quantized from the up projection's pre-activation u = z * scale
    # (GELU applied by the quantizer: oq_quantize_act_gelu).
    "flux_mlp_down_gelu_w2a4": [
        Projection("flux_mlp_down_gelu_w2a4", 4608, 12288, 3072, 128, 2, 4, _bf16(),
                   _outliers(12288, 0.01), 50.0, "lognormal", cfg=6, proj=0,
                   fused_gelu=True)],
    # W6A6, the setting the FLUX-3-Klein card gives its Qwen3-VL-4B text encoder: the
    # language model's MLP (hidden 2560, intermediate 9728) on a 4096-token batch.
    "text_encoder_w6a6": [
        Projection("text_encoder_up_w6a6", 4096, 2560, 9728, 128, 6, 6, _bf16(),
                   _outliers(2560, 0.01), 50.0, "lognormal", cfg=7, proj=0),
        Projection("text_encoder_down_w6a6", 4096, 9728, 2560, 128, 6, 6, _bf16(),
                   _outliers(9728, 0.01), 50.0, "lognormal", cfg=7, proj=1),
    ],
    # W2A3, the floor setting of the pages' Z-Image-Turbo remark, on the attention shape.
    "flux_attn_w2a3": [Projection("flux_attn_w2a3", 4608, 3072, 3072, 128, 2, 3, _bf16(),
                                  _outliers(3072, 0.01), 50.0, "lognormal", cfg=2, proj=0)],
    # The attention projection under the Block-RHT ablation and under the exact-marginal
    # codebook (same data as flux_attn_w4a4).
    "flux_attn_w4a4_block_rht": [
        Projection("flux_attn_w4a4_block_rht", 4608, 3072, 3072, 128, 4, 4, _bf16(),
                   _outliers(3072, 0.01), 50.0, "lognormal", cfg=2, proj=0,
                   rotation="block_rht")],
    "flux_attn_w4a4_exact": [
        Projection("flux_attn_w4a4_exact", 4608, 3072, 3072, 128, 4, 4, _bf16(),
                   _outliers(3072, 0.01), 50.0, "lognormal", cfg=2, proj=0,
                   marginal="exact")],
    "video_ffn_w4a8": [
        Projection("video_ffn_up_w4a8", 65520, 5120, 13824, 128, 4, 8, _bf16(),
                   _outliers(5120, 0.005), 100.0, "lognormal_cfg", cfg=4, proj=0),
        Projection("video_ffn_down_w4a8", 65520, 13824, 5120, 128, 4, 8, _bf16(),
                   _outliers(13824, 0.005), 100.0, "lognormal_cfg", cfg=4, proj=1),
    ],
}

SWEEP_D = (1024, 2048, 3072, 5120, 12288, 16384)
SWEEP_H = (64, 128, 256)
SWEEP_BITS = (4, 8)
SWEEP_T = (1, 16, 256, 4096, 65536)


def sweep_projection(d: int, h: int, bits_a: int, T: int) -> Projection:
    """One point of the activation-only sweep: bf16 N(0,1), 1% channels x50, no token scale.
    The data depend on d only (projection index = position of d in SWEEP_D)."""
    p = SWEEP_D.index(d) if d in SWEEP_D else 50 + (d // 128) % 40
    return Projection(f"sweep_d{d}_h{h}_a{bits_a}_T{T}", T, d, 0, h, 0, bits_a, _bf16(),
                      _outliers(d, 0.01), 50.0, "none", cfg=5, proj=p)


def sweep_points():
    return [sweep_projection(d, h, b, T) for d in SWEEP_D for h in SWEEP_H
            for b in SWEEP_BITS for T in SWEEP_T]


def seed_of(p: Projection, stream: int) -> int:
    return 1000 * p.cfg + 100 * p.proj + stream


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def _rows_normal(seed: int, rows: np.ndarray, ncols: int) -> torch.Tensor:
    """N(0,1) fp32 rows `rows` of an (inf x ncols) matrix drawn in seeded chunks."""
    out = torch.empty((len(rows), ncols), dtype=torch.float32)
    rows = np.asarray(rows, dtype=np.int64)
    if len(rows) == 0:
        return out
    chunks = rows // CHUNK
    for j in np.unique(chunks):
        sel = np.nonzero(chunks == j)[0]
        block = torch.randn((CHUNK, ncols), generator=_gen(seed * 1_000_003 + int(j)),
                            dtype=torch.float32)
        out[torch.from_numpy(sel)] = block[torch.from_numpy(rows[sel] - int(j) * CHUNK)]
    return out


def _rows_scalar_normal(seed: int, rows: np.ndarray) -> torch.Tensor:
    return _rows_normal(seed, rows, 1)[:, 0]


def outlier_channels(p: Projection) -> torch.Tensor:
    """Fixed channel subset scaled for every token: randperm(d)[:count]."""
    if p.outlier_count == 0:
        return torch.empty(0, dtype=torch.int64)
    return torch.randperm(p.d, generator=_gen(seed_of(p, 3)))[: p.outlier_count]


def activations(p: Projection, rows: Optional[Sequence[int]] = None) -> torch.Tensor:
    """Activation rows of projection p (all T rows by default), CPU tensor of p.dtype."""
    rows = np.arange(p.T) if rows is None else np.asarray(rows, dtype=np.int64)
    x = _rows_normal(seed_of(p, 1), rows, p.d)
    ch = outlier_channels(p)
    if len(ch):
        x[:, ch] *= p.outlier_scale
    if p.gelu:
        x = torch.nn.functional.gelu(x, approximate="none")
    # (fused_gelu rows are left as pre-activations z * scale; the quantizer applies GELU)
    if p.token_scale == "lognormal":
        x *= torch.exp(_rows_scalar_normal(seed_of(p, 4), rows))[:, None]
    elif p.token_scale == "lognormal_cfg":
        # two guidance halves (conditional rows first), each with its own scale stream
        half = p.T // 2
        cond = rows < half
        sc = torch.empty(len(rows), dtype=torch.float32)
        if cond.any():
            sc[torch.from_numpy(cond)] = torch.exp(
                _rows_scalar_normal(seed_of(p, 4), rows[cond]))
        if (~cond).any():
            sc[torch.from_numpy(~cond)] = torch.exp(
                _rows_scalar_normal(seed_of(p, 5), rows[~cond] - half))
        x *= sc[:, None]
    return x.to(p.dtype)


def weight(p: Projection, rows: Optional[Sequence[int]] = None) -> torch.Tensor:
    """Weight rows W[out, d] ~ N(0, 1/d) (C1 adds outlier rows), CPU tensor of p.dtype."""
    rows = np.arange(p.out) if rows is None else np.asarray(rows, dtype=np.int64)
    W = _rows_normal(seed_of(p, 2), rows, p.d) * (1.0 / math.sqrt(p.d))
    if p.w_outlier_rows:
        hot = torch.randperm(p.out, generator=_gen(seed_of(p, 6)))[: p.w_outlier_rows]
        mask = torch.isin(torch.from_numpy(rows), hot)
        W[mask] *= p.w_outlier_scale
    return W.to(p.dtype)


def get(name: str):
    return WORKLOADS[name]
