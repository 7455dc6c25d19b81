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
    model, d = tiny_weights
    rows = model.modulation_size()
    assert d["wmod"].shape[0] == rows
    for t in (1.0, 0.25):                       # two calls in a row share the scratch array
        want = torch.empty(rows, device="cuda")
        model.modulation(t, want)
        got = torch.full((rows,), float("nan"), device="cuda")
        F.flux_timestep_modulation_noalloc(d["w1"], d["b1"], d["w2"], d["b2"], d["wmod"], d["bmod"], t, got)
        torch.cuda.synchronize()
        err = ((got - want).abs().max() / want.abs().max()).item()
        assert err <= TOL, (t, err)
    assert F.flux_device_error() == 0


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
