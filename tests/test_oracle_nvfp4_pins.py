"""Pins of the NVFP4 oracle (oracle/nvfp4_oracle.py): the e2m1 value set from its bit-level
definition, nearest-value rounding by brute force, exact recovery of values already on the
block-scaled grid, the worst-case rounding error, and the linear layer on grid values.  CPU only."""
import itertools

import torch

from oracle import fp8_oracle as Q8
from oracle import nvfp4_oracle as Q4


def e2m1_from_bits(code):
    """Value of a 4-bit e2m1 code from the bit fields: sign, exponent (bias 1), mantissa."""
    s, e, m = (code >> 3) & 1, (code >> 1) & 3, code & 1
    mag = (m * 0.5) if e == 0 else (2.0 ** (e - 1)) * (1.0 + m / 2.0)
    return -mag if s else mag


def test_e2m1_value_set_from_the_bit_fields():
    vals = [e2m1_from_bits(c) for c in range(16)]
    assert sorted(set(abs(v) for v in vals)) == list(Q4.E2M1_VALUES)
    assert max(vals) == Q4.E2M1_MAX and min(vals) == -Q4.E2M1_MAX
    t = torch.tensor(vals, dtype=torch.float64)
    assert torch.equal(Q4.round_e2m1(t), t)                   # every value is a fixed point


def test_round_e2m1_is_the_nearest_value_with_ties_to_the_even_code():
    """Brute force over the 16 codes: nearest value; on a tie the code with mantissa bit 0."""
    g = torch.Generator().manual_seed(1)
    x = torch.cat([torch.empty(20000, dtype=torch.float64).uniform_(-7.5, 7.5, generator=g),
                   torch.tensor([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, -1.75, -5.0, 6.5, -100.0])])
    codes = [c for c in range(16) if c != 8]                  # -0 duplicates +0
    vals = torch.tensor([e2m1_from_bits(c) for c in codes], dtype=torch.float64)
    even = torch.tensor([(c & 1) == 0 for c in codes])
    xc = x.clamp(-6.0, 6.0)
    dist = (xc[:, None] - vals[None, :]).abs()
    best = dist.min(dim=1, keepdim=True).values
    cand = dist == best
    pick = torch.where(cand & even[None, :], 1, 0) + cand.long()       # prefer even codes among ties
    want = vals[pick.argmax(dim=1)]
    assert torch.equal(Q4.round_e2m1(x), want)
    # the ties by name: 0.25 -> 0, 0.75 -> 1, 1.25 -> 1, 1.75 -> 2, 2.5 -> 2, 3.5 -> 4, 5 -> 4
    assert Q4.round_e2m1(torch.tensor([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])).tolist() == [0, 1, 1, 2, 2, 4, 4]


def test_values_on_the_block_scaled_grid_are_recovered_exactly():
    """x = code * s_b * S with e4m3 block scales and a block holding +-6 at the row's largest
    scale: quantisation returns the same codes, block scales and x."""
    g = torch.Generator().manual_seed(2)
    rows, k = 6, 128
    vals = torch.tensor(Q4.E2M1_VALUES, dtype=torch.float64)
    codes = vals[torch.randint(0, 8, (rows, k), generator=g)] * torch.where(
        torch.rand(rows, k, generator=g) < 0.5, -1.0, 1.0).double()
    codes.view(rows, k // 16, 16)[:, :, 0] = 6.0             # every block reaches the e2m1 maximum
    sb = Q8.round_e4m3(torch.empty(rows, k // 16, dtype=torch.float64).uniform_(0.5, 300.0, generator=g))
    sb[:, 0] = 448.0                                          # the row maximum sits in block 0
    S = torch.pow(2.0, torch.randint(-12, -2, (rows,), generator=g).double())
    x = (codes.view(rows, k // 16, 16) * sb[:, :, None]).view(rows, k) * S[:, None]
    q, qsb, qS = Q4.quantize_rows_nvfp4(x.float())
    assert torch.equal(qS.double(), S)
    assert torch.equal(qsb, sb)
    assert torch.equal(q, codes)
    assert torch.equal(Q4.dequantize_nvfp4(q, qsb, qS), x)


def test_rounding_error_is_within_half_a_step_of_the_block_grid():
    """Each element is within half an e2m1 step (at most 1, between 4 and 6) of its value after
    scaling, allowing for the block scale's own e4m3 rounding (at most 1/16 above 6)."""
    g = torch.Generator().manual_seed(3)
    x = torch.randn(64, 3072, generator=g) * torch.exp(torch.randn(64, 1, generator=g))
    q, sb, S = Q4.quantize_rows_nvfp4(x)
    d = (sb * S.double()[:, None]).repeat_interleave(16, dim=1)
    err = (x.double() - Q4.dequantize_nvfp4(q, sb, S)).abs()
    assert (err <= d * (1.0 + 6.0 / 16.0) + 1e-30).all()
    assert (q.abs() <= 6.0).all()
    rel = (err.norm() / x.double().norm()).item()
    assert 0.02 < rel < 0.15                                  # a 4-bit format: visible but bounded error


def test_zero_rows_and_blocks_have_zero_codes():
    x = torch.randn(3, 64)
    x[1] = 0.0
    x[2, 16:32] = 0.0
    q, sb, S = Q4.quantize_rows_nvfp4(x)
    assert S[1] == 0 and (q[1] == 0).all() and (sb[1] == 0).all()
    assert sb[2, 1] == 0 and (q[2, 16:32] == 0).all()
    assert torch.isfinite(Q4.dequantize_nvfp4(q, sb, S)).all()


def test_linear_on_grid_values_is_the_exact_product():
    """Operands already on their NVFP4 grids: linear_nvfp4 is x W^T + b in float64."""
    g = torch.Generator().manual_seed(4)

    def grid(rows, k):
        x = torch.randn(rows, k, generator=g, dtype=torch.float64)
        q, sb, S = Q4.quantize_rows_nvfp4(x.float())
        return Q4.dequantize_nvfp4(q, sb, S)

    x, w = grid(5, 256), grid(7, 256)
    b = torch.randn(7, generator=g, dtype=torch.float64)
    y = Q4.linear_nvfp4(x, w, b)
    assert torch.allclose(y, x @ w.t() + b, rtol=1e-12, atol=1e-12)
    # and it differs from the unquantised product for general inputs
    xr, wr = torch.randn(5, 256, generator=g, dtype=torch.float64), torch.randn(7, 256, generator=g, dtype=torch.float64)
    assert (Q4.linear_nvfp4(xr, wr, None) - xr @ wr.t()).abs().max() > 1e-2


def test_block_scale_is_the_e4m3_of_the_scaled_block_maximum():
    """s_b = e4m3(amax_b * 448 / amax): the row's largest block gets 448, smaller blocks their ratio."""
    x = torch.zeros(1, 48)
    x[0, 0], x[0, 16], x[0, 32] = 8.0, 2.0, -0.5
    q, sb, S = Q4.quantize_rows_nvfp4(x)
    assert S.item() == 8.0 / 2688.0 or abs(S.item() - 8.0 / 2688.0) < 1e-9
    assert sb[0].tolist() == [448.0, 112.0, 28.0]
    assert q[0, 0] == 6.0 and q[0, 16] == 6.0 and q[0, 32] == -6.0
    assert [e for e in itertools.islice(q[0].tolist(), 1, 16)] == [0.0] * 15


def test_nvfp4_forward_error_and_its_sensitivity_to_bf16_sized_perturbations(monkeypatch):
    """Two properties of the NVFP4 forward itself (oracle only, tiny 1 + 1 block workload), which
    fix the tolerance of the GPU's NVFP4 forward:

    * eps: the NVFP4 forward is 3.5-6 % (rel-L2) from the exact forward (the format's own error);
    * sigma: perturbing every quantiser input by at most one bf16 rounding (relative 2^-9, seeded
      uniform) moves the NVFP4 forward by 2-3 %, more than the bf16 path's 2e-2 bar.  A code
      sits on one side of a rounding boundary; an input that crosses it moves the value by a whole
      e2m1 step (1/4 to 1/2 of the value), so the forward is not continuous in its quantiser inputs,
      and any path whose attention runs on bf16 operands carries at least this perturbation.
    Also sigma < 0.7 eps: a forward that did not quantise at all would sit eps away, well outside a
    bar set from sigma."""
    from oracle import flux_oracle as O
    from synthetic import WORKLOADS, make_weights
    torch.set_grad_enabled(False)
    w = WORKLOADS["tiny64"]
    _, p = make_weights(w.dims, w.seed)
    g = torch.Generator().manual_seed(196)
    tok = torch.randn(16, 128, generator=g).to(torch.bfloat16).float()
    txt = torch.randn(16, 3072, generator=g).to(torch.bfloat16).float()
    exact = O.forward(p, O.hyper(w.dims), tok, txt, 0.6, (4, 4))
    hq = dict(O.hyper(w.dims), nvfp4=True)
    pure = O.forward(p, hq, tok, txt, 0.6, (4, 4))
    plain = Q4.linear_nvfp4
    gp = torch.Generator().manual_seed(0)

    def perturbed(x, wt, b):
        x = torch.as_tensor(x)
        u = torch.rand(x.shape, generator=gp, dtype=torch.float64) * 2 - 1
        return plain(x * (1 + u * 2.0 ** -9).to(x.dtype), wt, b)
    monkeypatch.setattr(Q4, "linear_nvfp4", perturbed)
    pert = O.forward(p, hq, tok, txt, 0.6, (4, 4))

    def rel(a, b):
        return ((a - b).norm() / b.norm()).item()
    eps, sigma = rel(pure, exact), rel(pert, pure)
    assert 0.035 <= eps <= 0.06, eps
    assert 0.02 <= sigma <= 0.03, sigma
    assert sigma < 0.7 * eps, (sigma, eps)
