"""The allocation-free timestep conditioning entry point against flux_dit_modulation.

flux_timestep_modulation_noalloc serves callers that may not allocate device
memory once running (a runtime that owns all device memory in a pool sized at
start-up, or a latency-critical loop that cannot stall on cudaMalloc/cudaFree).
It must give what the model's own flux_dit_modulation gives, call after call,
while its intermediates sit in the library's fixed device array.  This file is
collected last so that a run stopping at the first failure has run every other
test first; it also passes on its own in a fresh process.
"""
import ctypes

import pytest
import torch

import latent_flow_matching_b200 as F
from synthetic import WORKLOADS, make_weights

pytestmark = pytest.mark.gpu
torch.set_grad_enabled(False)
TOL = 1e-2          # normalised max error, as for every other kernel-level test


def _bf16_dev(arr):
    return torch.from_numpy(arr.copy()).view(torch.bfloat16).cuda()


@pytest.fixture(scope="module")
def tiny_weights():
    w = WORKLOADS["tiny64"]
    blob, p = make_weights(w.dims, w.seed)
    model = F.FluxDiT(blob, w.dims)
    mod_names = [k for k in p if k.endswith("mod.w")]          # blob order
    dev = {
        "w1": _bf16_dev(p["time_in.w1"]), "b1": _bf16_dev(p["time_in.b1"]),
        "w2": _bf16_dev(p["time_in.w2"]), "b2": _bf16_dev(p["time_in.b2"]),
        "wmod": torch.cat([_bf16_dev(p[n]) for n in mod_names]).contiguous(),
        "bmod": torch.cat([_bf16_dev(p[n[:-1] + "b"]) for n in mod_names]).contiguous(),
    }
    yield model, dev
    model.close()


def test_matches_model_modulation_on_consecutive_calls(tiny_weights):
    """Both paths run the same timestep-embedding and GEMV kernels in the same order, so two calls in
    a row (sharing the scratch array) equal flux_dit_modulation bit for bit."""
    model, d = tiny_weights
    rows = model.modulation_size()
    assert d["wmod"].shape[0] == rows
    for t in (1.0, 0.25):                       # two calls in a row share the scratch array
        want = torch.empty(rows, device="cuda")
        model.modulation(t, want)
        got = torch.full((rows,), float("nan"), device="cuda")
        F.flux_timestep_modulation_noalloc(d["w1"], d["b1"], d["w2"], d["b2"], d["wmod"], d["bmod"], t, got)
        torch.cuda.synchronize()
        assert torch.equal(got, want), t
    assert F.flux_device_error() == 0


def test_matches_the_oracle_modulation(tiny_weights):
    """Against the oracle's time MLP and modulation linears (float64) at the kernel-level bar."""
    from oracle import flux_oracle as O
    model, d = tiny_weights
    w = WORKLOADS["tiny64"]
    _, p = make_weights(w.dims, w.seed)
    t = 0.6
    got = torch.empty(model.modulation_size(), device="cuda")
    F.flux_timestep_modulation_noalloc(d["w1"], d["b1"], d["w2"], d["b2"], d["wmod"], d["bmod"], t, got)
    f64 = torch.float64
    h = O.silu(O.linear(O.timestep_embedding(t), O.weight(p, "time_in.w1", f64), O.weight(p, "time_in.b1", f64)))
    s = O.silu(O.linear(h, O.weight(p, "time_in.w2", f64), O.weight(p, "time_in.b2", f64)))
    names = [k for k in p if k.endswith("mod.w")]
    ref = torch.cat([O.linear(s, O.weight(p, n, f64), O.weight(p, n[:-1] + "b", f64)) for n in names])
    err = ((got.cpu().double() - ref).abs().max() / ref.abs().max()).item()
    assert err <= TOL, err


def test_largest_accepted_sizes_against_the_oracle():
    """hidden 8192 and t_freq_dim 1024, the limits the scratch array is sized for, on small random
    weights: the same arithmetic as the oracle's time MLP and modulation linear."""
    from oracle import flux_oracle as O
    hidden, tf, rows, t = 8192, 1024, 40, 0.3
    g = torch.Generator().manual_seed(7)

    def bf(*shape, scale):
        return (torch.randn(*shape, generator=g) * scale).to(torch.bfloat16)
    w1, b1 = bf(hidden, tf, scale=tf ** -0.5), bf(hidden, scale=1.0)
    w2, b2 = bf(hidden, hidden, scale=hidden ** -0.5), bf(hidden, scale=1.0)
    wm, bm = bf(rows, hidden, scale=hidden ** -0.5), bf(rows, scale=1.0)
    got = torch.full((rows,), float("nan"), device="cuda")
    F.flux_timestep_modulation_noalloc(*(x.cuda() for x in (w1, b1, w2, b2, wm, bm)), t, got)
    f64 = torch.float64
    h = O.silu(O.linear(O.timestep_embedding(t, tf), w1.to(f64), b1.to(f64)))
    s = O.silu(O.linear(h, w2.to(f64), b2.to(f64)))
    ref = O.linear(s, wm.to(f64), bm.to(f64))
    err = ((got.cpu().double() - ref).abs().max() / ref.abs().max()).item()
    assert err <= TOL, err


def test_repeated_calls_allocate_no_device_memory(tiny_weights):
    """After the first call, ten more leave the device's free memory unchanged (nothing is
    allocated, by this library or the caching allocator: the output buffer already exists)."""
    model, d = tiny_weights
    out = torch.empty(model.modulation_size(), device="cuda")
    F.flux_timestep_modulation_noalloc(d["w1"], d["b1"], d["w2"], d["b2"], d["wmod"], d["bmod"], 1.0, out)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    reserved0 = torch.cuda.memory_reserved()
    for i in range(10):
        F.flux_timestep_modulation_noalloc(d["w1"], d["b1"], d["w2"], d["b2"], d["wmod"], d["bmod"], i / 10, out)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
    assert torch.cuda.memory_reserved() == reserved0


def test_rejects_sizes_beyond_the_scratch_limit(tiny_weights):
    _, d = tiny_weights
    L = F.lib()
    out = torch.empty(16, device="cuda")
    p = ctypes.c_void_p
    args = [p(d[k].data_ptr()) for k in ("w1", "b1", "w2", "b2", "wmod", "bmod")]
    rc = L.flux_timestep_modulation_noalloc(*args, 8192 + 8, 256, 16, 1.0, p(out.data_ptr()), None)
    assert rc == F.FLUX_EINVAL
    assert "8192" in F.get_error()
    rc = L.flux_timestep_modulation_noalloc(*args, 3072, 2048, 16, 1.0, p(out.data_ptr()), None)
    assert rc == F.FLUX_EINVAL
    assert "1024" in F.get_error()
