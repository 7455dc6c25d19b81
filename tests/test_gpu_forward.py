"""Forward and sampler parity of the CUDA path (through the C ABI) against the CPU oracle.

Bars: velocity relative L2 <= 2e-2 at every step, final latent relative L2 <=
3e-2 after all steps, modulation vector normalised max error <= 1e-2.
* tiny 64^2 workload (1 double + 1 single block): the oracle runs live in float64.
* 256^2 .. 1024^2(+reference) workloads: the oracle's sampled rows, written by
  tests/golden/make_goldens.py (oracle only), are compared row by row.
"""
import json
import os

import numpy as np
import pytest
import torch

import latent_flow_matching_b200 as F
from oracle import flux_oracle as O
from synthetic import WORKLOADS, FluxDims, Workload, make_weights, make_inputs, make_uncond_text

pytestmark = pytest.mark.gpu
torch.set_grad_enabled(False)
DEV = "cuda"
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
V_TOL, X_TOL, K_TOL = 2e-2, 3e-2, 1e-2


def rel_l2(a, b):
    a = torch.as_tensor(a).double().cpu()
    b = torch.as_tensor(b).double().cpu()
    return ((a - b).norm() / b.norm()).item()


def gpu_sample(model, w, lat, txt, ref):
    vs = []
    if isinstance(ref, list):
        ref = [torch.from_numpy(r).to(DEV) for r in ref]
    elif ref is not None:
        ref = torch.from_numpy(ref).to(DEV)
    guided = {}
    if w.guidance is not None:
        guided = {"txt_uncond": torch.from_numpy(make_uncond_text(w)).to(DEV), "guidance": w.guidance}
    final = F.flux_sample(model, torch.from_numpy(lat).to(DEV), torch.from_numpy(txt).to(DEV), w.n_steps, ref,
                          on_step=lambda i, v: vs.append(v.cpu().clone()), **guided)
    return final.cpu(), vs


@pytest.fixture(scope="module")
def tiny():
    w = WORKLOADS["tiny64"]
    blob, p = make_weights(w.dims, w.seed)
    model = F.FluxDiT(blob, w.dims)
    yield w, p, model
    model.close()


def test_tiny_modulation_vector(tiny):
    w, p, model = tiny
    for t in (1.0, 0.25):
        out = torch.empty(model.modulation_size(), device=DEV)
        model.modulation(t, out)
        temb = O.timestep_embedding(t)
        h = O.silu(O.linear(temb, O.weight(p, "time_in.w1", torch.float64), O.weight(p, "time_in.b1", torch.float64)))
        s = O.silu(O.linear(h, O.weight(p, "time_in.w2", torch.float64), O.weight(p, "time_in.b2", torch.float64)))
        names = [k for k in p if k.endswith("mod.w")]
        ref = torch.cat([O.linear(s, O.weight(p, n, torch.float64), O.weight(p, n[:-1] + "b", torch.float64))
                         for n in names])
        err = ((out.cpu().double() - ref).abs().max() / ref.abs().max()).item()
        assert err <= K_TOL, err


@pytest.mark.parametrize("n", [1, 3, 5])
def test_prepared_timesteps_match_per_forward_modulation(tiny, n):
    """Vectors computed together (up to four per weight read) equal, bit for bit, the ones a
    forward computes alone; a forward at a prepared t gives the same velocity."""
    w, p, model = tiny
    ts = [float(np.float32(1.0 - i / 7)) for i in range(n)]
    size = model.modulation_size()
    alone = []
    model.prepare_timesteps([])
    for t in ts:
        out = torch.empty(size, device=DEV)
        model.modulation(t, out)
        alone.append(out)
    lat, txt, _ = make_inputs(w)
    tok = O.pack_latents(torch.from_numpy(lat)).float().to(DEV)
    v0 = torch.empty(w.n_img, 128, device=DEV)
    model.forward(tok, (w.grid, w.grid), torch.from_numpy(txt).to(DEV), ts[-1], v0)
    model.prepare_timesteps(ts)
    try:
        for t, ref in zip(ts, alone):
            out = torch.empty(size, device=DEV)
            model.modulation(t, out)
            assert torch.equal(out, ref)
        v1 = torch.empty_like(v0)
        model.forward(tok, (w.grid, w.grid), torch.from_numpy(txt).to(DEV), ts[-1], v1)
        assert torch.equal(v0, v1)
    finally:
        model.prepare_timesteps([])
    assert F.flux_device_error() == 0


@pytest.mark.parametrize("n_double,n_single", [(0, 0), (1, 0), (1, 1)])
def test_tiny_forward_block_by_block(tiny, n_double, n_single):
    w, p, model = tiny
    lat, txt, _ = make_inputs(w)
    keep = {k: v for k, v in p.items()
            if not ((k.startswith("double.") and int(k.split(".")[1]) >= n_double) or
                    (k.startswith("single.") and int(k.split(".")[1]) >= n_single))}
    tok = O.pack_latents(torch.from_numpy(lat))
    ref = O.forward(keep, O.hyper(w.dims), tok, torch.from_numpy(txt), 0.75, (w.grid, w.grid))
    model.set_active_blocks(n_double, n_single)
    try:
        v = torch.empty(w.n_img, 128, device=DEV)
        model.forward(tok.float().to(DEV), (w.grid, w.grid), torch.from_numpy(txt).to(DEV), 0.75, v)
    finally:
        model.set_active_blocks(-1, -1)
    assert rel_l2(v, ref) <= V_TOL
    assert F.flux_device_error() == 0


def test_tiny_sampler_matches_oracle(tiny):
    w, p, model = tiny
    lat, txt, _ = make_inputs(w)
    ref_final, ref_vs = O.sample(p, O.hyper(w.dims), torch.from_numpy(lat), torch.from_numpy(txt), w.n_steps)
    final, vs = gpu_sample(model, w, lat, txt, None)
    for i in range(w.n_steps):
        assert rel_l2(vs[i], ref_vs[i]) <= V_TOL
    assert rel_l2(final, ref_final) <= X_TOL
    assert F.flux_device_error() == 0


def test_forward_is_deterministic(tiny):
    w, p, model = tiny
    lat, txt, _ = make_inputs(w)
    a, _ = gpu_sample(model, w, lat, txt, None)
    b, _ = gpu_sample(model, w, lat, txt, None)
    assert torch.equal(a, b)


@pytest.mark.parametrize("precision", ["bf16", "fp8", "nvfp4"])
def test_programmatic_launches_change_nothing(tiny, precision, monkeypatch):
    """With programmatic dependent launches (the default) every kernel waits for its predecessor
    before touching memory, so the sampler's output is bit-identical to plain stream order."""
    w, p, model = tiny
    lat, txt, _ = make_inputs(w)
    prec = {"bf16": F.PRECISION_BF16, "fp8": F.PRECISION_FP8, "nvfp4": F.PRECISION_NVFP4}[precision]
    model.set_precision(prec)
    try:
        monkeypatch.setenv("FLUX_PDL", "0")
        plain, vs_plain = gpu_sample(model, w, lat, txt, None)
        monkeypatch.setenv("FLUX_PDL", "1")
        pdl, vs_pdl = gpu_sample(model, w, lat, txt, None)
    finally:
        model.set_precision(F.PRECISION_BF16)
    assert torch.equal(plain, pdl)
    assert all(torch.equal(a, b) for a, b in zip(vs_plain, vs_pdl))
    assert F.flux_device_error() == 0


def test_sampling_step_replayed_from_a_cuda_graph_equals_plain_launches(tiny):
    """One sampling step as the benchmark times it (a device copy of the noise, the run's modulation
    vectors, pack, forward, Euler, unpack), captured in a CUDA graph with programmatic launches and
    replayed, against the same launches run directly: bit-identical latents."""
    w, p, model = tiny
    lat_h, txt_h, _ = make_inputs(w)
    lat0 = torch.from_numpy(lat_h).to(DEV)
    txt = torch.from_numpy(txt_h).to(DEV)
    ts = F.euler_schedule(w.n_steps)
    tok = torch.empty(w.n_img, 128, device=DEV)
    v = torch.empty_like(tok)
    lat = torch.empty_like(lat0)

    def step():
        lat.copy_(lat0)
        model.prepare_timesteps(ts[:-1])
        F.flux_pack_latents(lat, tok)
        model.forward(tok, (w.grid, w.grid), txt, ts[0], v)
        F.flux_euler_step(tok, v, ts[1] - ts[0])
        F.flux_unpack_latents(tok, lat)

    step()
    torch.cuda.synchronize()
    plain = lat.clone()
    lat.fill_(float("nan"))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    lat.fill_(float("nan"))
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(lat, plain)
    del g
    assert F.flux_device_error() == 0


@pytest.mark.parametrize("precision", [F.PRECISION_BF16, F.PRECISION_FP8, F.PRECISION_NVFP4])
def test_profile_counts_the_algorithmic_work(tiny, precision):
    """The profiling hook's FLOPs and bytes (from which the benchmark's rooflines are computed) equal
    the closed forms for the tiny model: per block N 2D(4D + 3F) of linears and 4 N^2 D of attention,
    the input and output projections; GEMM bytes read A and W once in the format that runs (bf16 2
    bytes, e4m3 1, NVFP4 1/2 + 1/16 per element, the quantised formats plus a 4-byte scale per row)
    and write each output once (bf16 2 bytes, SwiGLU half the columns in bf16, fp32 4, the gated
    residual's fp32 rows read and written)."""
    w, p, model = tiny
    d = w.dims
    D, Fh, C, T = d.hidden, d.mlp_hidden, d.in_ch, d.txt_dim
    ni, nt = w.n_img, w.n_txt
    n = ni + nt
    blocks = d.n_double + d.n_single
    lat, txt, _ = make_inputs(w)
    tok = O.pack_latents(torch.from_numpy(lat)).float().to(DEV)
    v = torch.empty(ni, 128, device=DEV)
    elt, row = {F.PRECISION_BF16: (2.0, 0.0), F.PRECISION_FP8: (1.0, 4.0),
                F.PRECISION_NVFP4: (0.5 + 1.0 / 16.0, 4.0)}[precision]

    def linear_bytes(m, k, nn, out_per_elt, e=elt, r=row):
        return e * (m * k + nn * k) + r * (m + nn) + out_per_elt * m * nn

    blk = 0.0
    for rows in (nt, ni):                       # double block, per stream
        blk += linear_bytes(rows, D, 3 * D, 2) + linear_bytes(rows, D, D, 8)
        blk += linear_bytes(rows, D, 2 * Fh, 1) + linear_bytes(rows, Fh, D, 8)
    sgl = linear_bytes(n, D, 3 * D, 2) + linear_bytes(n, D, 2 * Fh, 1) + linear_bytes(n, D + Fh, D, 8)
    io = (linear_bytes(nt, T, D, 4, 2.0, 0.0) + linear_bytes(ni, C, D, 4, 2.0, 0.0) +
          linear_bytes(ni, D, C, 4, 2.0, 0.0))
    want_bytes = d.n_double * blk + d.n_single * sgl + io
    want_flops = blocks * n * 2.0 * D * (4 * D + 3 * Fh) + 2.0 * ni * C * D + 2.0 * nt * T * D + 2.0 * ni * D * C
    model.set_precision(precision)
    try:
        model.forward(tok, (w.grid, w.grid), torch.from_numpy(txt).to(DEV), 0.5, v)
        model.profile(True)
        model.forward(tok, (w.grid, w.grid), torch.from_numpy(txt).to(DEV), 0.5, v)
        prof = model.profile_read()
    finally:
        model.profile(False)
        model.set_precision(F.PRECISION_BF16)
    _, g_fl, g_by, g_n = prof["gemm"]
    _, a_fl, _, a_n = prof["attention"]
    assert g_n == 4 * d.n_double + 2 * d.n_single + 2
    assert a_n == blocks
    assert g_fl == pytest.approx(want_flops, rel=1e-12)
    assert a_fl == pytest.approx(blocks * 4.0 * n * n * D, rel=1e-12)
    assert g_by == pytest.approx(want_bytes, rel=1e-12)


@pytest.mark.parametrize("n_txt,grid,ref_grid", [(0, (4, 6), (0, 0)), (5, (6, 4), (4, 4)), (131, (8, 8), (4, 8))])
def test_tiny_forward_ragged_and_degenerate_shapes(tiny, n_txt, grid, ref_grid):
    """No text, non-square grids, a reference of another size, sequence lengths off the 128-row tiles."""
    w, p, model = tiny
    g = torch.Generator().manual_seed(n_txt)
    tok = torch.randn(grid[0] * grid[1], 128, generator=g).to(torch.bfloat16).float()
    txt = torch.randn(n_txt, 3072, generator=g).to(torch.bfloat16).float()
    ref = None
    if ref_grid[0]:
        ref = torch.randn(ref_grid[0] * ref_grid[1], 128, generator=g).to(torch.bfloat16).float()
    want = O.forward(p, O.hyper(w.dims), tok, txt, 0.5, grid, ref, ref_grid)
    v = torch.empty(grid[0] * grid[1], 128, device=DEV)
    model.forward(tok.to(DEV), grid, txt.to(DEV) if n_txt else None, 0.5, v,
                  None if ref is None else ref.to(DEV), ref_grid)
    assert rel_l2(v, want) <= V_TOL


def test_forward_rejects_bad_shapes(tiny):
    w, p, model = tiny
    v = torch.empty(16, 128, device=DEV)
    tok = torch.zeros(16, 128, device=DEV)
    txt = torch.zeros(4, 3072, device=DEV)
    for grid in ((2, 8), (65, 4)):
        with pytest.raises(F.FluxError):
            model.forward(tok, grid, txt, 1.0, v)
    with pytest.raises(F.FluxError):
        model.forward(tok, (4, 4), txt, 1.0, v, None, (4, 4))       # reference grid without tokens
    with pytest.raises(F.FluxError):
        model.forward(tok, (4, 4), txt, float("nan"), v)


# ---------------------------------------------------------------------------- full-size workloads vs goldens
def _golden(name):
    path = os.path.join(GOLDEN, f"{name}.npz")
    if not os.path.exists(path):
        pytest.skip(f"golden {path} not generated")
    return np.load(path)


@pytest.mark.parametrize("name", ["t2i256", "t2i512", "t2i1024", "i2i1024", "mref1024", "cfg256"])
def test_full_workload_against_oracle_goldens(name):
    gd = _golden(name)
    w = WORKLOADS[name]
    meta = json.loads(str(gd["meta"]))
    assert meta["workload"] == name and meta["seed"] == w.seed
    blob, _ = make_weights(w.dims, w.seed)
    lat, txt, ref = make_inputs(w)
    model = F.FluxDiT(blob, w.dims)
    del blob
    try:
        final, vs = gpu_sample(model, w, lat, txt, ref)
    finally:
        model.close()
    rows = torch.from_numpy(gd["rows"]).long()
    for i in range(w.n_steps):
        err = rel_l2(vs[i][rows], gd["v"][i])
        assert err <= V_TOL, (i, err)
    tok = O.pack_latents(final)
    err = rel_l2(tok[rows], gd["final"])
    assert err <= X_TOL, err
    assert F.flux_device_error() == 0


# ---------------------------------------------------------------------------- several references, img2img
def test_tiny_forward_with_several_references(tiny):
    """Two references of different sizes (RoPE l = -1, -2) against the oracle."""
    w, p, model = tiny
    g = torch.Generator().manual_seed(21)
    tok = torch.randn(16, 128, generator=g).to(torch.bfloat16).float()
    txt = torch.randn(7, 3072, generator=g).to(torch.bfloat16).float()
    grids = [(4, 4), (6, 4)]
    refs = [torch.randn(h * w_, 128, generator=g).to(torch.bfloat16).float() for h, w_ in grids]
    want = O.forward(p, O.hyper(w.dims), tok, txt, 0.5, (4, 4), refs, grids)
    v = torch.empty(16, 128, device=DEV)
    model.forward(tok.to(DEV), (4, 4), txt.to(DEV), 0.5, v, torch.cat(refs).to(DEV), grids)
    assert rel_l2(v, want) <= V_TOL
    # swapping the references changes the result (their RoPE offsets differ)
    v2 = torch.empty(16, 128, device=DEV)
    model.forward(tok.to(DEV), (4, 4), txt.to(DEV), 0.5, v2, torch.cat(refs[::-1]).to(DEV), grids[::-1])
    assert rel_l2(v2, v) > 1e-3
    assert F.flux_device_error() == 0


def test_tiny_img2img_sampler_matches_oracle(tiny):
    """strength 0.75 with 4 steps: the last 3 steps from the blended start state."""
    w, p, model = tiny
    lat, txt, _ = make_inputs(w)
    init = torch.randn(32, 8, 8, generator=torch.Generator().manual_seed(5)).to(torch.bfloat16).float()
    ref_final, ref_vs = O.sample(p, O.hyper(w.dims), torch.from_numpy(lat), torch.from_numpy(txt), 4,
                                 init_latent=init, strength=0.75)
    vs = []
    final = F.flux_sample(model, torch.from_numpy(lat).to(DEV), torch.from_numpy(txt).to(DEV), 4,
                          init_latent=init.to(DEV), strength=0.75, on_step=lambda i, v: vs.append(v.cpu().clone()))
    assert len(vs) == len(ref_vs) == 3
    for a, b in zip(vs, ref_vs):
        assert rel_l2(a, b) <= V_TOL
    assert rel_l2(final.cpu(), ref_final) <= X_TOL
    kept = F.flux_sample(model, torch.from_numpy(lat).to(DEV), torch.from_numpy(txt).to(DEV), 4,
                         init_latent=init.to(DEV), strength=0.0)
    assert torch.equal(kept.cpu(), init)                      # strength 0 keeps the image


def test_forward_rejects_too_many_references(tiny):
    w, p, model = tiny
    v = torch.empty(16, 128, device=DEV)
    tok = torch.zeros(16, 128, device=DEV)
    refs = torch.zeros(11 * 16, 128, device=DEV)
    with pytest.raises(F.FluxError):
        model.forward(tok, (4, 4), None, 1.0, v, refs, [(4, 4)] * 11)


# ---------------------------------------------------------------------------- classifier-free guidance
@pytest.mark.parametrize("n_txt,grid,refs", [(7, (4, 4), []), (5, (6, 4), [(4, 4), (4, 6)]), (0, (4, 5), []),
                                             (131, (8, 8), [(4, 8)])])
def test_tiny_cfg_batch_equals_two_single_forwards(tiny, n_txt, grid, refs):
    """The batch-2 forward returns, bit for bit, the two single-text forwards (no row depends on
    another sequence); sequence lengths off the 128-row tiles put the batch boundary inside a tile."""
    w, p, model = tiny
    g = torch.Generator().manual_seed(40 + n_txt)
    tok = torch.randn(grid[0] * grid[1], 128, generator=g).to(torch.bfloat16).float().to(DEV)
    tc = torch.randn(n_txt, 3072, generator=g).to(torch.bfloat16).float().to(DEV)
    tu = torch.randn(n_txt, 3072, generator=g).to(torch.bfloat16).float().to(DEV)
    ref = None
    if refs:
        ref = torch.randn(sum(h * w_ for h, w_ in refs), 128, generator=g).to(torch.bfloat16).float().to(DEV)
    ni = grid[0] * grid[1]
    vc, vu, a, b = (torch.empty(ni, 128, device=DEV) for _ in range(4))
    model.forward_cfg(tok, grid, tc if n_txt else None, tu if n_txt else None, 0.6, vc, vu, ref, refs)
    hw = refs if refs else (0, 0)
    model.forward(tok, grid, tc if n_txt else None, 0.6, a, ref, hw)
    model.forward(tok, grid, tu if n_txt else None, 0.6, b, ref, hw)
    assert torch.equal(vc, a) and torch.equal(vu, b)
    if n_txt:
        assert not torch.equal(vc, vu)
    assert F.flux_device_error() == 0


def test_tiny_cfg_sampler_matches_oracle(tiny):
    """Guidance 3.5 with an unconditional text: every guided velocity and the final latent
    against the live float64 oracle."""
    w, p, model = tiny
    lat, txt, _ = make_inputs(w)
    txt_u = np.random.default_rng(77).standard_normal(txt.shape).astype(np.float32)
    txt_u = torch.from_numpy(txt_u).to(torch.bfloat16).float()
    ref_final, ref_vs = O.sample(p, O.hyper(w.dims), torch.from_numpy(lat), torch.from_numpy(txt), 3,
                                 txt_uncond=txt_u, guidance=3.5)
    vs = []
    final = F.flux_sample(model, torch.from_numpy(lat).to(DEV), torch.from_numpy(txt).to(DEV), 3,
                          txt_uncond=txt_u.to(DEV), guidance=3.5, on_step=lambda i, v: vs.append(v.cpu().clone()))
    assert len(vs) == len(ref_vs) == 3
    for a, b in zip(vs, ref_vs):
        assert rel_l2(a, b) <= V_TOL
    assert rel_l2(final.cpu(), ref_final) <= X_TOL
    # guidance 1 is the prompt-only sampler, bit for bit
    one = F.flux_sample(model, torch.from_numpy(lat).to(DEV), torch.from_numpy(txt).to(DEV), 3,
                        txt_uncond=txt_u.to(DEV), guidance=1.0)
    plain = F.flux_sample(model, torch.from_numpy(lat).to(DEV), torch.from_numpy(txt).to(DEV), 3)
    assert rel_l2(one.cpu(), plain.cpu()) <= 1e-6
    assert F.flux_device_error() == 0


def test_cfg_rejects_bad_arguments(tiny):
    w, p, model = tiny
    tok = torch.zeros(16, 128, device=DEV)
    v = torch.empty(16, 128, device=DEV)
    tc, tu = torch.zeros(4, 3072, device=DEV), torch.zeros(5, 3072, device=DEV)
    with pytest.raises(ValueError):
        model.forward_cfg(tok, (4, 4), tc, tu, 1.0, v, torch.empty_like(v))
    with pytest.raises(F.FluxError):                         # one buffer for both velocities
        model.forward_cfg(tok, (4, 4), tc, tc, 1.0, v, v)
    with pytest.raises(F.FluxError):
        F.flux_cfg_euler_step(v, v, v, float("nan"), 0.1)


def test_cfg_batch_bit_exact_at_full_size():
    """1024^2 workload (4608 tokens per sequence, full model): the batch-2 forward equals the two
    single-text forwards bit for bit, so the single-text goldens pin both velocities."""
    w = WORKLOADS["t2i1024"]
    blob, _ = make_weights(w.dims, w.seed)
    lat, txt, _ = make_inputs(w)
    model = F.FluxDiT(blob, w.dims)
    del blob
    try:
        tok = O.pack_latents(torch.from_numpy(lat)).float().to(DEV)
        tc = torch.from_numpy(txt).to(DEV)
        tu = torch.from_numpy(make_uncond_text(WORKLOADS["cfg1024"])).to(DEV)
        vc, vu, a, b = (torch.empty(w.n_img, 128, device=DEV) for _ in range(4))
        model.forward_cfg(tok, (w.grid, w.grid), tc, tu, 0.75, vc, vu)
        model.forward(tok, (w.grid, w.grid), tc, 0.75, a)
        model.forward(tok, (w.grid, w.grid), tu, 0.75, b)
        torch.cuda.synchronize()
        assert torch.equal(vc, a) and torch.equal(vu, b)
        assert rel_l2(vc, vu) > 1e-3
    finally:
        model.close()
    assert F.flux_device_error() == 0
