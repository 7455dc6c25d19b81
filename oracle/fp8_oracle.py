"""Row-wise FP8 (e4m3) linear layers for the CPU oracle.

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: only ``tests/`` and ``bench.py``'s CPU
legs import it; the product path never does.

Source: "FLUX.3 Image Klein in Diffusers: Architektur, Layout-Steuerung und
Systemanforderungen im Überblick" (mindverse), section "Hardwareanforderungen, Quantisierung und
Inferenzlatenz": the transformer ships as fp8r, row-wise FP8, with fast kernels from compute
capability 8.9 on (Blackwell included); the we0.ai FLUX 3 Image Klein article lists 11.2 GB of
generator weights in BF16 and 5.6 GB in FP8 (one byte per weight).

Readings where the pages are silent:
* the format is e4m3 ("fn": no infinities, largest finite 448), round to nearest even,
  saturating at +-448;
* row-wise means one fp32 scale per row of every operand: per output row of a weight matrix and
  per token row of the activation, computed from the row's absolute maximum:
      amax = max_j |x_j|,  scale = amax / 448,  inv = 448 / amax  (0 for an all-zero row),
      code_j = e4m3(x_j * inv),  value_j = code_j * scale,
  with the scale, the reciprocal and the product x_j * inv each rounded to float32 (the
  precision the quantised codes are decided in); y = (codes_x codes_w^T) * scale_x * scale_w + b;
* it applies to the linears inside the transformer blocks (qkv, projection, MLP in / out;
  linear1 / linear2), which carry all but 0.1 % of the FLOPs; the input and output projections
  and the modulation layers stay in the bf16 weights' precision.
"""
from __future__ import annotations

import torch

__all__ = ["E4M3_MAX", "round_e4m3", "quantize_rows", "dequantize_rows", "linear_fp8"]

E4M3_MAX = 448.0


def round_e4m3(x: torch.Tensor) -> torch.Tensor:
    """Nearest e4m3 value (ties to even), saturating at +-448, as float64.

    e4m3: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits.  Normal values 2^e (1 + m/8),
    e = -6 .. 8 (the top code of e = 8 is NaN, so the largest finite value is 1.75 * 2^8 = 448);
    subnormals m/8 * 2^-6.  In every binade [2^e, 2^(e+1)) the spacing is 2^(e-3); below 2^-6 it
    is 2^-9.
    """
    x = torch.as_tensor(x, dtype=torch.float64)
    a = x.abs().clamp(max=E4M3_MAX)
    _, ex = torch.frexp(a)                       # a = f 2^ex with f in [0.5, 1): floor(log2 a) = ex - 1
    e = torch.clamp(ex.to(torch.float64) - 1.0, min=-6.0)
    quantum = torch.pow(2.0, e - 3.0)
    r = torch.round(a / quantum) * quantum      # torch.round: half to even
    return torch.copysign(r, x)


def quantize_rows(x: torch.Tensor):
    """(codes as float64 values, scale [rows] float32) of the row-wise e4m3 quantisation of x [rows, k]."""
    x32 = torch.as_tensor(x).to(torch.float32)
    amax = x32.abs().amax(dim=1)
    scale = amax / torch.tensor(E4M3_MAX, dtype=torch.float32)
    inv = torch.where(amax > 0, torch.tensor(E4M3_MAX, dtype=torch.float32) / amax,
                      torch.zeros_like(amax))
    codes = round_e4m3((x32 * inv[:, None]).to(torch.float64))
    return codes, scale


def dequantize_rows(codes: torch.Tensor, scale: torch.Tensor) -> torch.Tensor:
    return codes * scale.to(torch.float64)[:, None]


def linear_fp8(x: torch.Tensor, w: torch.Tensor, b: torch.Tensor | None) -> torch.Tensor:
    """x W^T + b with x (per token row) and W (per output row) quantised to e4m3; the products of
    codes are summed exactly (float64) and scaled by both rows' scales."""
    dtype = torch.as_tensor(x).dtype
    qx, sx = quantize_rows(x)
    qw, sw = quantize_rows(w)
    y = torch.matmul(qx, qw.t()) * sx.to(torch.float64)[:, None] * sw.to(torch.float64)[None, :]
    y = y.to(dtype)
    return y if b is None else y + b
