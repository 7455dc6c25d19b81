"""Pins of the row-wise FP8 oracle (oracle/fp8_oracle.py) against torch's own float8_e4m3fn
conversion, the format's complete value set and closed forms.  CPU only."""
import numpy as np
import torch

from oracle import flux_oracle as O
from oracle import fp8_oracle as Q
from synthetic import WORKLOADS, make_weights, make_inputs


def torch_e4m3(x):
    return torch.as_tensor(x, dtype=torch.float64).to(torch.float8_e4m3fn).to(torch.float64)


def all_finite_e4m3():
    v = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64)
    return v[v.isfinite()]


def test_round_e4m3_matches_torch_conversion_inside_the_range():
    g = torch.Generator().manual_seed(0)
    mag = torch.pow(2.0, torch.empty(200000, dtype=torch.float64).uniform_(-14, 8.85, generator=g))
    x = mag * torch.where(torch.rand(200000, generator=g) < 0.5, -1.0, 1.0).double()
    vals = all_finite_e4m3().unique()
    mids = (vals[1:] + vals[:-1]) / 2                           # every exact tie
    x = torch.cat([x, vals, mids, torch.tensor([0.0, -0.0, 2.0 ** -10, 448.0, 464.0, -464.0])])
    x = x[x.abs() <= 464]
    assert torch.equal(Q.round_e4m3(x), torch_e4m3(x))


def test_e4m3_value_set_closed_form():
    vals = all_finite_e4m3()
    assert vals.numel() == 254                                  # 256 codes minus the two NaNs
    pos = vals[vals > 0].unique()
    assert pos.numel() == 126 and pos.max() == 448.0 and pos.min() == 2.0 ** -9
    assert torch.equal(Q.round_e4m3(vals), vals)                # every value is a fixed point
    normals = pos[pos >= 2.0 ** -6]
    assert normals.numel() == 15 * 8 - 1                        # exponents -6..8, minus the NaN slot
    assert Q.round_e4m3(torch.tensor([1000.0, -1e9]))[0] == 448.0   # saturation (a reading)
    assert Q.round_e4m3(torch.tensor([-1e9]))[0] == -448.0


def test_quantize_rows_scale_rule_and_error_bound():
    g = torch.Generator().manual_seed(1)
    x = torch.randn(64, 3072, generator=g) * torch.logspace(-3, 3, 64)[:, None]
    x[5] = 0.0
    codes, scale = Q.quantize_rows(x)
    assert scale.dtype == torch.float32
    assert torch.all(codes.abs() <= 448.0)
    amax_idx = x.abs().argmax(dim=1)
    top = codes[torch.arange(64), amax_idx].abs()
    assert torch.all(top[torch.arange(64) != 5] == 448.0)       # the row maximum maps to the top code
    assert torch.all(codes[5] == 0) and scale[5] == 0
    deq = Q.dequantize_rows(codes, scale)
    err = (deq - x.double()).abs()
    # round to nearest: half a spacing, i.e. 2^-4 of the value in the normal range, 2^-10 of the
    # scale below it (plus float32 rounding of x * inv)
    bound = torch.maximum(x.double().abs() * 2.0 ** -4, scale.double()[:, None] * 2.0 ** -10) * (1 + 1e-6)
    assert torch.all(err <= bound + 1e-30)


def test_linear_fp8_is_exact_on_representable_operands():
    """Operands that are e4m3 values times a power of two with the row maximum at 448 * 2^k
    quantise exactly, so the FP8 linear equals the plain one; a transposed or swapped scale
    would not."""
    g = torch.Generator().manual_seed(2)
    vals = all_finite_e4m3()

    def rows(n, k):
        idx = torch.randint(0, vals.numel(), (n, k), generator=g)
        r = vals[idx]
        r[:, 0] = 448.0
        return r * torch.pow(2.0, torch.randint(-6, 6, (n, 1), generator=g).double())

    x, w = rows(9, 256), rows(17, 256)
    b = torch.randn(17, generator=g, dtype=torch.float64)
    assert torch.equal(Q.linear_fp8(x, w, b), O.linear(x, w, b))
    wc = w.clone()
    wc[3] *= 4.0                                                # row-wise: one row's scale changes only its column
    d = Q.linear_fp8(x, wc, b) - Q.linear_fp8(x, w, b)
    assert torch.all(d[:, [i for i in range(17) if i != 3]] == 0) and torch.any(d[:, 3] != 0)


def test_linear_fp8_error_against_the_plain_linear():
    """Random operands: the relative error is that of e4m3 rounding on both operands (about
    2^-4 / sqrt(3) each in RMS), neither zero nor beyond the worst case 2 * 2^-4."""
    g = torch.Generator().manual_seed(3)
    x = torch.randn(128, 3072, generator=g, dtype=torch.float64)
    w = torch.randn(256, 3072, generator=g, dtype=torch.float64) / 3072 ** 0.5
    ref = O.linear(x, w, None)
    rel = ((Q.linear_fp8(x, w, None) - ref).norm() / ref.norm()).item()
    assert 0.01 < rel < 0.125


def test_fp8_forward_stays_near_the_exact_forward():
    """The tiny workload through the FP8 block linears: a few percent from the exact forward
    (e4m3 rounding through four block linears and the residual stream), and only the block
    linears change (with zero blocks the two forwards are identical)."""
    w = WORKLOADS["tiny64"]
    _, p = make_weights(w.dims, w.seed, threads=4)
    lat, txt, _ = make_inputs(w)
    tok = O.pack_latents(torch.from_numpy(lat))
    hp, hq = O.hyper(w.dims), dict(O.hyper(w.dims), fp8=True)
    a = O.forward(p, hp, tok, torch.from_numpy(txt), 0.7, (w.grid, w.grid))
    b = O.forward(p, hq, tok, torch.from_numpy(txt), 0.7, (w.grid, w.grid))
    rel = ((a - b).norm() / a.norm()).item()
    assert 0.002 < rel < 0.1, rel
    none = {k: v for k, v in p.items() if not k.startswith(("double.", "single."))}
    a0 = O.forward(none, hp, tok, torch.from_numpy(txt), 0.7, (w.grid, w.grid))
    b0 = O.forward(none, hq, tok, torch.from_numpy(txt), 0.7, (w.grid, w.grid))
    assert torch.equal(a0, b0)
