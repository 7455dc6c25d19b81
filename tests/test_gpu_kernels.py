"""Per-kernel parity of the CUDA path (through the C ABI) against the CPU oracle.

Bars: pack/unpack bit-exact; Euler within 1 ulp of the exactly rounded value;
every other kernel normalised max error max|gpu - ref| / max|ref| <= 1e-2, with
the oracle evaluated in float64 on the same bf16-rounded inputs.
"""
import math

import numpy as np
import pytest
import torch

import latent_flow_matching_b200 as F
from oracle import flux_oracle as O

pytestmark = pytest.mark.gpu
torch.set_grad_enabled(False)
TOL = 1e-2
DEV = "cuda"


def nmax(gpu, ref):
    gpu = gpu.double().cpu()
    ref = ref.double().cpu()
    return ((gpu - ref).abs().max() / ref.abs().max()).item()


def rand(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(*shape, generator=g) * scale)


def bf(x):
    return x.to(torch.bfloat16)


@pytest.fixture(autouse=True)
def _device_clean():
    yield
    assert F.flux_device_error() == 0


# ---------------------------------------------------------------------------- pack / unpack / Euler
@pytest.mark.parametrize("h8,w8", [(8, 8), (128, 128), (6, 10), (2, 2), (64, 32), (4, 66), (2, 130)])
def test_pack_unpack_bit_exact(h8, w8):
    """Pack tiles hold 32 tokens of one token row: 33 and 65 tokens per row leave a ragged tile."""
    lat = rand((32, h8, w8), h8 * 100 + w8)
    tok = torch.empty((h8 // 2) * (w8 // 2), 128, device=DEV)
    F.flux_pack_latents(lat.to(DEV), tok)
    assert torch.equal(tok.cpu(), O.pack_latents(lat))
    back = torch.empty(32, h8, w8, device=DEV)
    F.flux_unpack_latents(tok, back)
    assert torch.equal(back.cpu(), lat)


@pytest.mark.parametrize("n", [4096 * 128, 1, 7, 1000003])
def test_euler_within_one_ulp(n):
    x = rand((n,), 1)
    v = rand((n,), 2)
    dt = -0.25
    xd = x.to(DEV)
    F.flux_euler_step(xd, v.to(DEV), dt)
    exact = O.euler_update(x.double(), v.double(), dt)
    gpu = xd.cpu()
    ulp = torch.abs(torch.nextafter(exact.float(), torch.tensor(math.inf)) - exact.float())
    assert ((gpu.double() - exact).abs() <= ulp.double()).all()


# ---------------------------------------------------------------------------- LayerNorm + modulation
@pytest.mark.parametrize("rows,dim", [(4608 + 5, 3072), (33, 3072), (17, 256)])
def test_layernorm_modulate(rows, dim):
    x = rand((rows, dim), 3, 2.0) + 0.5
    sh, sc = rand((dim,), 4), rand((dim,), 5)
    y = torch.empty(rows, dim, device=DEV, dtype=torch.bfloat16)
    F.flux_layernorm_modulate(x.to(DEV), y, sh.to(DEV), sc.to(DEV), 1e-6)
    ref = O.modulate(O.layer_norm(x.double(), 1e-6), sh.double(), sc.double())
    assert nmax(y, ref) <= TOL
    # bf16 output: each element within one bf16 rounding (plus fp32 statistics)
    assert ((y.double().cpu() - ref).abs() <= ref.abs() * 2 ** -8 + 1e-3).all()


# ---------------------------------------------------------------------------- QK-RMSNorm + RoPE
def test_rope_table_matches_oracle_angles():
    nt, gh, gw, rh, rw = 7, 5, 6, 4, 4
    n = nt + gh * gw + rh * rw
    table = torch.empty(n, 64, 2, device=DEV)
    F.flux_rope_table(table, nt, (gh, gw), (rh, rw), 1e4)
    ang = O.rope_angles(O.token_positions(nt, gh, gw, rh, rw), 128, 1e4)
    t = table.cpu().double()
    assert (t[..., 0] - torch.cos(ang)).abs().max() < 1e-6
    assert (t[..., 1] - torch.sin(ang)).abs().max() < 1e-6


@pytest.mark.parametrize("nt,gh,gw,rh,rw,heads", [(7, 5, 6, 4, 4, 24), (512, 16, 16, 0, 0, 24), (7, 5, 6, 0, 0, 5),
                                                  (3, 4, 4, 0, 0, 1)])
def test_qk_rmsnorm_rope(nt, gh, gw, rh, rw, heads):
    """Odd head counts leave the second half-warp without a head on the last pair."""
    D = heads * 128
    n = nt + gh * gw + rh * rw
    qkv = bf(rand((n, 3 * D), 6, 1.5))
    gq, gk = bf(rand((128,), 7)), bf(rand((128,), 8))
    table = torch.empty(n, 64, 2, device=DEV)
    F.flux_rope_table(table, nt, (gh, gw), (rh, rw), 1e4)
    dq = qkv.to(DEV)
    F.flux_qk_rmsnorm_rope(dq, D, heads, gq.to(DEV), gk.to(DEV), table, 1e-6)
    out = dq.cpu()
    ang = O.rope_angles(O.token_positions(nt, gh, gw, rh, rw), 128, 1e4)
    x = qkv.double()
    for col, g in ((0, gq), (D, gk)):
        h = x[:, col:col + D].reshape(n, heads, 128)
        ref = O.apply_rope(O.rms_norm(h, g.double(), 1e-6), ang).reshape(n, D)
        assert nmax(out[:, col:col + D], ref) <= TOL
    assert torch.equal(out[:, 2 * D:], qkv[:, 2 * D:])           # v untouched


@pytest.mark.parametrize("m,row0", [(300, 7), (4608, 0)])
def test_qkv_projection_fused_norm_rope(m, row0):
    """GEMM with the fused QK-RMSNorm + RoPE epilogue vs linear -> rms_norm -> rope in float64."""
    heads, k = 24, 3072
    D = heads * 128
    nt, gh, gw = 512, 64, 64                       # table for the 1024^2 joint sequence (4608 rows)
    a = bf(rand((m, k), 60))
    w = bf(rand((3 * D, k), 61, k ** -0.5))
    b = bf(rand((3 * D,), 62, 0.5))
    gq, gk = bf(rand((128,), 63)), bf(rand((128,), 64))
    table = torch.empty(nt + gh * gw, 64, 2, device=DEV)
    F.flux_rope_table(table, nt, (gh, gw), (0, 0), 1e4)
    out = torch.empty(m, 3 * D, device=DEV, dtype=torch.bfloat16)
    F.flux_qkv_projection(a.to(DEV), w.to(DEV), b.to(DEV), heads, gq.to(DEV), gk.to(DEV), table, out, row0, 1e-6)
    rows = torch.arange(0, m, max(1, m // 64))
    y = O.linear(a[rows].double(), w.double(), b.double())
    ang = O.rope_angles(O.token_positions(nt, gh, gw), 128, 1e4)[row0 + rows]
    got = out.cpu()[rows]
    for col, g in ((0, gq), (D, gk)):
        h = y[:, col:col + D].reshape(len(rows), heads, 128)
        ref = O.apply_rope(O.rms_norm(h, g.double(), 1e-6), ang).reshape(len(rows), D)
        assert nmax(got[:, col:col + D], ref) <= TOL
    assert nmax(got[:, 2 * D:], y[:, 2 * D:]) <= TOL


# ---------------------------------------------------------------------------- tcgen05 GEMM
def interleave_swiglu(w):
    """[a; b] rows -> per 128 output columns: 128 a-rows then 128 b-rows (GEMM order)."""
    f = w.shape[0] // 2
    a, b = w[:f], w[f:]
    parts = []
    for g in range(f // 128):
        parts += [a[128 * g:128 * g + 128], b[128 * g:128 * g + 128]]
    return torch.cat(parts)


@pytest.mark.parametrize("m,k,n,mode", [
    (300, 3072, 512, F.EPI_BF16_BIAS),
    (129, 128, 3072, F.EPI_F32_BIAS),
    (4096, 3072, 128, F.EPI_F32_BIAS),
    (257, 3072, 1024, F.EPI_SWIGLU),
    (200, 9216, 384, F.EPI_RESID_GATE),
    (1, 64, 32, F.EPI_BF16_BIAS),
    (128 * 3 + 1, 12288, 256 + 32, F.EPI_RESID_GATE),
])
def test_linear_modes(m, k, n, mode):
    a = bf(rand((m, k), 10))
    w = bf(rand((n, k), 11, k ** -0.5))
    b = bf(rand((n,), 12, 0.5))
    A = a.double()
    if mode == F.EPI_SWIGLU:
        ref_h = O.linear(A, w.double(), b.double())
        aa, bb = ref_h.chunk(2, dim=1)
        ref = O.silu(aa) * bb
        out = torch.empty(m, n // 2, device=DEV, dtype=torch.bfloat16)
        F.flux_linear(a.to(DEV), interleave_swiglu(w).to(DEV).contiguous(),
                      interleave_swiglu(b[:, None])[:, 0].to(DEV).contiguous(), mode, out)
    elif mode == F.EPI_RESID_GATE:
        x0 = rand((m, n), 13)
        gate = rand((n,), 14)
        ref = x0.double() + gate.double() * O.linear(A, w.double(), b.double())
        out = x0.to(DEV)
        F.flux_linear(a.to(DEV), w.to(DEV), b.to(DEV), mode, out, gate=gate.to(DEV))
    else:
        ref = O.linear(A, w.double(), b.double())
        dt = torch.bfloat16 if mode == F.EPI_BF16_BIAS else torch.float32
        out = torch.empty(m, n, device=DEV, dtype=dt)
        F.flux_linear(a.to(DEV), w.to(DEV), b.to(DEV), mode, out)
    err = nmax(out, ref)
    assert err <= TOL, err
    if mode == F.EPI_F32_BIAS:
        assert err < 1e-5, err                  # fp32 output: only accumulation order differs


def test_linear_full_size_sampled_rows():
    """Single-block fused linear1 size (4608 x 3072 -> 27648 rows of W, bf16 out), sampled rows."""
    m, k, n = 4608, 3072, 27648
    a = bf(rand((m, k), 20)).to(DEV)
    w = bf(rand((n, k), 21, k ** -0.5)).to(DEV)
    b = bf(rand((n,), 22, 0.5)).to(DEV)
    out = torch.empty(m, n, device=DEV, dtype=torch.bfloat16)
    F.flux_linear(a, w, b, F.EPI_BF16_BIAS, out)
    rows = torch.arange(0, m, 97)
    ref = O.linear(a[rows].cpu().double(), w.cpu().double(), b.cpu().double())
    assert nmax(out[rows], ref) <= TOL


# ---------------------------------------------------------------------------- attention
@pytest.mark.parametrize("n,heads,qscale", [(1, 2, 1.0), (77, 3, 1.0), (128, 1, 1.0), (200, 2, 1.0), (300, 2, 1.0),
                                            (1030, 2, 1.0), (700, 2, 6.0), (2500, 1, 4.0)])
def test_attention(n, heads, qscale):
    q = bf(rand((n, heads, 128), 30, qscale))
    k = bf(rand((n, heads, 128), 31))
    v = bf(rand((n, heads, 128), 32))
    o = torch.empty(n, heads, 128, device=DEV, dtype=torch.bfloat16)
    F.flux_joint_attention(q.to(DEV), k.to(DEV), v.to(DEV), o)
    ref = O.attention(q.double(), k.double(), v.double())
    assert nmax(o.reshape(n, -1), ref) <= TOL


def test_attention_full_size_sampled_rows():
    """Joint sequence of the 1024^2 workload (4608 tokens, 24 heads); rows sampled for the oracle."""
    n, heads = 4608, 24
    q = bf(rand((n, heads, 128), 40))
    k = bf(rand((n, heads, 128), 41))
    v = bf(rand((n, heads, 128), 42))
    o = torch.empty(n, heads, 128, device=DEV, dtype=torch.bfloat16)
    F.flux_joint_attention(q.to(DEV), k.to(DEV), v.to(DEV), o)
    rows = torch.arange(3, n, 131)
    ref = O.attention(q[rows].double(), k.double(), v.double())   # queries are independent
    assert nmax(o.cpu()[rows].reshape(len(rows), -1), ref) <= TOL


def test_attention_zero_query_is_mean_of_values():
    n, heads = 257, 2
    q = torch.zeros(n, heads, 128, dtype=torch.bfloat16)
    k = bf(rand((n, heads, 128), 50))
    v = bf(rand((n, heads, 128), 51))
    o = torch.empty(n, heads, 128, device=DEV, dtype=torch.bfloat16)
    F.flux_joint_attention(q.to(DEV), k.to(DEV), v.to(DEV), o)
    ref = v.double().mean(0, keepdim=True).expand(n, heads, 128)
    assert nmax(o, ref) <= TOL


@pytest.mark.parametrize("t", [0.0, 0.25, 0.75, 1.0])
def test_blend_latents(t):
    x = rand((32, 64, 64), 70)
    noise = rand((32, 64, 64), 71)
    out = torch.empty(32, 64, 64, device=DEV)
    F.flux_blend_latents(x.to(DEV), noise.to(DEV), t, out)
    ref = O.blend_latents(x.double(), noise.double(), t)
    assert (out.cpu().double() - ref).abs().max() <= 1e-6
    if t in (0.0, 1.0):
        assert torch.equal(out.cpu(), x if t == 0.0 else noise)


# ---------------------------------------------------------------------------- guidance, batched attention
@pytest.mark.parametrize("n", [1, 7, 4096 * 128 + 3])
def test_cfg_euler_step(n):
    g = torch.Generator().manual_seed(n % 1000)
    x = torch.randn(n, generator=g)
    vc = torch.randn(n, generator=g)
    vu = torch.randn(n, generator=g)
    xd = x.to(DEV)
    F.flux_cfg_euler_step(xd, vc.to(DEV), vu.to(DEV), 3.5, -0.25)
    v_ref = O.guided_velocity(vc.double(), vu.double(), 3.5)
    ref = O.euler_update(x.double(), v_ref, -0.25)
    assert (xd.cpu().double() - ref).abs().max().item() <= 1e-5
    # the same update with the guided velocity written out: the same x, and v within fp32 rounding
    xo, vg = x.to(DEV), torch.full((n,), float("nan"), device=DEV)
    F.flux_cfg_euler_step(xo, vc.to(DEV), vu.to(DEV), 3.5, -0.25, v_guided=vg)
    assert torch.equal(xo, xd)
    assert (vg.cpu().double() - v_ref).abs().max().item() <= 1e-5 * v_ref.abs().max().item()


@pytest.mark.parametrize("batch,n", [(2, 77), (2, 300), (3, 129), (2, 4608)])
def test_attention_batch_sequences_are_independent(batch, n):
    """Each sequence of the batch attends only to itself; rows equal the one-sequence call bit for bit."""
    heads = 2
    q = bf(rand((batch * n, heads, 128), 60))
    k = bf(rand((batch * n, heads, 128), 61))
    v = bf(rand((batch * n, heads, 128), 62))
    o = torch.empty(batch * n, heads, 128, device=DEV, dtype=torch.bfloat16)
    F.flux_joint_attention_batch(q.to(DEV), k.to(DEV), v.to(DEV), o, batch)
    for b in range(batch):
        sl = slice(b * n, (b + 1) * n)
        one = torch.empty(n, heads, 128, device=DEV, dtype=torch.bfloat16)
        F.flux_joint_attention(q[sl].to(DEV), k[sl].to(DEV), v[sl].to(DEV), one)
        assert torch.equal(o[sl], one)
        rows = torch.arange(0, n, max(1, n // 40))
        ref = O.attention(q[sl][rows].double(), k[sl].double(), v[sl].double())
        assert nmax(o[sl].cpu()[rows].reshape(len(rows), -1), ref) <= TOL


# ---------------------------------------------------------------------------- bounded waits
def test_bounded_wait_gives_up_records_the_code_and_leaves_the_context_usable():
    """A wait on an mbarrier that nothing arrives on returns after its limit; the kernel records its
    code, flux_device_error reports it once (and clears it), and the next launches run normally."""
    assert F.flux_device_error() == 0
    F.flux_selftest_bounded_wait(20_000_000, arrive=True)          # the phase completes: no error
    assert F.flux_device_error() == 0
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record()
    F.flux_selftest_bounded_wait(20_000_000, arrive=False)         # nothing arrives: gives up after 20 ms
    ev1.record()
    torch.cuda.synchronize()
    assert ev0.elapsed_time(ev1) >= 19.0
    assert F.flux_device_error() == F.DEVERR_TIMEOUT_SELFTEST
    assert F.flux_device_error() == 0                               # read and cleared
    x = torch.zeros(1000, device=DEV)
    F.flux_euler_step(x, torch.ones(1000, device=DEV), -0.5)        # the context still works
    assert torch.equal(x.cpu(), torch.full((1000,), -0.5))
    with pytest.raises(F.FluxError):
        F.flux_selftest_bounded_wait(2_000_000_000, arrive=False)   # above the pipelines' 1 s limit
