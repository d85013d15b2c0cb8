"""Seeded synthetic inputs for the BinaryAttention forward (no method arithmetic).

This module is the only code that both the CUDA path's tests/benchmark and the
CPU oracle's tests use.  It draws random numbers and nothing else: no sign,
scale, score, softmax or quantisation step lives here.

The five workloads mirror the model shapes the BinaryAttention paper-notes page
evaluates (Table 1: DeiT-T/S/B on ImageNet-1K, DeiT-B at 384^2; Table 3:
DiT-XL/2 at 256^2) plus a 128x128-patch high-resolution ViT, the regime the
page's motivation section names.  A sixth, deit_b384_rpc, is the DeiT-B at
384^2 shape with a 2-D relative-position bias over its 24x24 patch grid plus
the class token, the bias variant Key design 2 names, on a token set with a
class token.  No dataset or trained weight is involved:
activations are Gaussian with a per-channel offset, which gives each channel a
non-zero mean the way trained Q/K/V projections do.

Recipe (all draws from ``numpy.random.default_rng(seed)`` in this order):
  for each tensor in (q, k, v):
    offset[h, c] ~ N(0, offset_std)      (std, not variance; 0 for DiT)
    x[b, h, n, c] = offset[h, c] + N(0, 1)
    if outlier_frac > 0: round(outlier_frac * H * d) of the H*d channels,
       drawn without replacement, are multiplied by 8 (after the offset)
  bias: dense [H, N, N], a 2-D relative-position table
        [H, (2 gh - 1) * (2 gw - 1)], or that table followed by three class-token
        entries per head [H, (2 gh - 1) * (2 gw - 1) + 3]; entries ~ N(0, bias_std)
Values are then rounded to the workload's input dtype (bf16: round to nearest
even through torch) and returned as float32 numpy arrays holding exactly the
rounded values.  The dense bias is returned with a padded row stride
``ld = round_up(N, 4)`` (padding columns are zero) so every row starts on a
16-byte boundary.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass

import numpy as np


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    dtype: str = "bf16"          # input dtype: "bf16" or "f32"
    bias: str = "dense"          # "none", "dense", "relpos2d" or "relpos2d_cls"
    grid: tuple = (0, 0)         # (gh, gw) patch grid for the rel-pos biases
    offset_std: float = 0.5
    outlier_frac: float = 0.0
    bias_std: float = 0.02
    seed: int = 0
    note: str = ""

    def scaled(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    @property
    def ld(self) -> int:
        return round_up(self.N, 4)

    @property
    def ops(self) -> float:
        """Effective operations of one attention call, 4*B*H*N^2*d."""
        return 4.0 * self.B * self.H * self.N * self.N * self.d


def round_up(x: int, m: int) -> int:
    return (x + m - 1) // m * m


WORKLOADS = {
    "deit_t": Workload("deit_t", 1, 3, 197, 64, dtype="f32",
                       note="DeiT-T shape, 14x14 patches + CLS, fp32 inputs"),
    "deit_s": Workload("deit_s", 64, 6, 197, 64, outlier_frac=0.02,
                       note="DeiT-S shape, 2% outlier channels x8"),
    "deit_b384": Workload("deit_b384", 32, 12, 577, 64,
                          note="DeiT-B at 384^2, 24x24 patches + CLS"),
    "dit_xl2": Workload("dit_xl2", 32, 16, 256, 72, offset_std=0.0,
                        note="DiT-XL/2 at 256^2 latent, 16x16 patches, d=72"),
    "hires16k": Workload("hires16k", 4, 12, 16384, 64, bias="relpos2d", grid=(128, 128),
                         note="high-resolution ViT, 128x128 patch grid, 2-D rel-pos table"),
    "deit_b384_rpc": Workload("deit_b384_rpc", 32, 12, 577, 64, bias="relpos2d_cls", grid=(24, 24),
                              note="DeiT-B at 384^2 with a 2-D rel-pos table over 24x24 patches + CLS"),
}


def _round_dtype(x: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "f32":
        return x.astype(np.float32)
    if dtype == "bf16":
        import torch
        t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
        return t.to(torch.bfloat16).to(torch.float32).numpy()
    raise ValueError(dtype)


def make_inputs(w: Workload, seed: int | None = None) -> dict:
    """Draw q, k, v [B, H, N, d] and the bias for workload ``w``."""
    rng = np.random.default_rng(w.seed if seed is None else seed)
    out = {}
    for name in ("q", "k", "v"):
        offset = (rng.standard_normal((w.H, w.d), dtype=np.float32) * np.float32(w.offset_std)
                  if w.offset_std > 0 else np.zeros((w.H, w.d), np.float32))
        x = rng.standard_normal((w.B, w.H, w.N, w.d), dtype=np.float32)
        x += offset[None, :, None, :]
        if w.outlier_frac > 0:
            n_out = int(round(w.outlier_frac * w.H * w.d))
            chosen = rng.choice(w.H * w.d, size=n_out, replace=False)
            for flat in chosen:
                h, c = divmod(int(flat), w.d)
                x[:, h, :, c] *= np.float32(8.0)
        out[name] = _round_dtype(x, w.dtype)
    if w.bias == "dense":
        b = rng.standard_normal((w.H, w.N, w.N), dtype=np.float32) * np.float32(w.bias_std)
        padded = np.zeros((w.H, w.N, w.ld), np.float32)
        padded[:, :, : w.N] = b
        out["bias"] = padded
        out["ld"] = w.ld
    elif w.bias in ("relpos2d", "relpos2d_cls"):
        gh, gw = w.grid
        cls = w.bias == "relpos2d_cls"
        assert gh * gw + cls == w.N, "rel-pos bias needs N == gh * gw (+ 1 with a class token)"
        out["bias"] = (rng.standard_normal((w.H, (2 * gh - 1) * (2 * gw - 1) + 3 * cls), dtype=np.float32)
                       * np.float32(w.bias_std))
        out["ld"] = 0
    else:
        out["bias"] = None
        out["ld"] = 0
    return out


BIAS_KIND = {"none": 0, "dense": 1, "relpos2d": 2, "relpos2d_cls": 3}


@dataclass(frozen=True)
class DecodeWorkload:
    """Nq new query tokens per (batch, head) against an Nk-token cache."""
    name: str
    B: int
    H: int
    Nq: int
    Nk: int
    d: int
    dtype: str = "bf16"
    offset_std: float = 0.5
    seed: int = 0
    note: str = ""

    @property
    def ops(self) -> float:
        """Effective operations of one decode call, 4*B*H*Nq*Nk*d."""
        return 4.0 * self.B * self.H * self.Nq * self.Nk * self.d


DECODE_WORKLOADS = {
    "decode_16k": DecodeWorkload("decode_16k", 32, 12, 1, 16384, 64,
                                 note="one new query per head against a 16384-token cache, DeiT-B-sized heads"),
}


def make_decode_inputs(w: DecodeWorkload, seed: int | None = None) -> dict:
    """Draw the new queries q [B, H, Nq, d] and the cache's raw keys and
    values k, v [B, H, Nk, d] (per-channel offsets as in make_inputs)."""
    rng = np.random.default_rng(w.seed if seed is None else seed)
    out = {}
    for name, n in (("q", w.Nq), ("k", w.Nk), ("v", w.Nk)):
        offset = rng.standard_normal((w.H, w.d), dtype=np.float32) * np.float32(w.offset_std)
        x = rng.standard_normal((w.B, w.H, n, w.d), dtype=np.float32)
        x += offset[None, :, None, :]
        out[name] = _round_dtype(x, w.dtype)
    return out
