"""Seeded synthetic inputs for the attention library and its checks.

This module holds no attention arithmetic: it only draws random bf16 tensors.
It is the one piece of code that both the CUDA path (tests, bench) and the CPU
oracle's callers use, so that both see the same bits.

Recipe (the FlashAttention-2 kernel benchmark isolates attention on random
inputs; no dataset is involved):
  * "normal":     Q, K, V (and dO) i.i.d. N(0, 1) in fp32, rounded to bf16
                  (round-to-nearest-even, torch's cast).
  * "row_scaled": each (b, h, n) row of Q, K and V is N(0, 0.5^2) times a
                  factor r ~ U(0.5, 2) drawn per row and per tensor; dO stays
                  N(0, 1).  This varies score magnitudes as in GPT-style layers.
All draws come from one ``torch.Generator('cpu')`` seeded with ``seed``, in the
order q, k, v, dO, so a given (shape, seed, dist) always yields the same bits.
"""
from __future__ import annotations

import math
import numpy as np
import torch


def _normal(gen: torch.Generator, shape, std: float = 1.0) -> torch.Tensor:
    x = torch.randn(shape, generator=gen, dtype=torch.float32)
    if std != 1.0:
        x = x * std
    return x


def _row_scaled(gen: torch.Generator, shape) -> torch.Tensor:
    x = _normal(gen, shape, 0.5)
    r = torch.rand(shape[:-1] + (1,), generator=gen, dtype=torch.float32)
    return x * (0.5 + 1.5 * r)


def attention_inputs(B: int, H: int, N: int, d: int, seed: int,
                     dist: str = "normal", with_dout: bool = False):
    """Return a dict of CPU bf16 tensors q, k, v (and dO) of shape [B,H,N,d]."""
    gen = torch.Generator("cpu").manual_seed(int(seed))
    shape = (B, H, N, d)
    out = {}
    for name in ("q", "k", "v"):
        if dist == "normal":
            x = _normal(gen, shape)
        elif dist == "row_scaled":
            x = _row_scaled(gen, shape)
        else:
            raise ValueError(f"unknown input distribution {dist!r}")
        out[name] = x.to(torch.bfloat16)
    if with_dout:
        out["dO"] = _normal(gen, shape).to(torch.bfloat16)
    return out


def attention_inputs_device(B: int, H: int, N: int, d: int, seed: int,
                            device="cuda", dist: str = "normal"):
    """q, k, v, dO of shape [B,H,N,d], drawn directly on the device by a
    seeded ``torch.Generator`` of that device (in the order q, k, v, dO; the
    same recipes as above) -- for shapes whose host-side generation and
    transfer would take minutes.  The bits differ from ``attention_inputs``
    with the same seed; a caller that checks a slice against the oracle copies
    that slice back."""
    gen = torch.Generator(device).manual_seed(int(seed))
    shape = (B, H, N, d)
    out = {}
    for name in ("q", "k", "v", "dO"):
        x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
        if dist == "row_scaled" and name != "dO":
            r = torch.rand(shape[:-1] + (1,), generator=gen, device=device,
                           dtype=torch.float32)
            x = (x * 0.5) * (0.5 + 1.5 * r)
        elif dist not in ("normal", "row_scaled"):
            raise ValueError(f"unknown input distribution {dist!r}")
        out[name] = x.to(torch.bfloat16)
    return out


def decode_inputs(B: int, H: int, Nq: int, Nk: int, d: int, seed: int,
                  dist: str = "normal"):
    """CPU bf16 q [B,H,Nq,d] and k, v [B,H,Nk,d] for decoding (Nq query rows
    against Nk cached keys); same recipe and draw order (q, k, v) as above."""
    gen = torch.Generator("cpu").manual_seed(int(seed))
    out = {}
    for name, n in (("q", Nq), ("k", Nk), ("v", Nk)):
        shape = (B, H, n, d)
        if dist == "normal":
            x = _normal(gen, shape)
        elif dist == "row_scaled":
            x = _row_scaled(gen, shape)
        else:
            raise ValueError(f"unknown input distribution {dist!r}")
        out[name] = x.to(torch.bfloat16)
    return out


def to_e4m3(x: torch.Tensor):
    """Per-tensor e4m3 (float8_e4m3fn) quantisation of a CPU tensor, as a
    caller of the 8-bit score path would do it: descale = max|x| / 448 (the
    largest finite e4m3 value), x8 = round-to-nearest(x / descale).  Returns
    (x8, descale); the dequantised tensor is x8 * descale."""
    amax = float(x.abs().max())
    descale = float(np.float32(amax / 448.0)) if amax > 0 else 1.0
    x8 = (x.to(torch.float32) / descale).to(torch.float8_e4m3fn)
    return x8, descale


def default_scale(d: int) -> float:
    """1/sqrt(d) rounded to fp32, the value both sides receive."""
    return float(np.float32(1.0 / math.sqrt(d)))


def to_f64(t: torch.Tensor) -> np.ndarray:
    """Widen a bf16/fp32 CPU tensor exactly to a float64 numpy array."""
    return t.detach().to("cpu", torch.float64).numpy()
