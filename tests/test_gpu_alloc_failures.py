"""Out-of-memory handling, driven by the library's allocation test hook (flux_test_fail_alloc_after):
every entry point that allocates device memory returns FLUX_ENOMEM with a message when an
allocation fails, releases what it allocated in that call, and leaves the model as it was, so the
next call succeeds and computes exactly what a model that never failed computes.  The pages'
convention is an int status (or NULL) plus a message (hakusoku.com story 4662, "エラーハンドリング").
No GPU is faulted: the hook makes the library see a failed allocation without asking the driver.
"""
import numpy as np
import pytest
import torch

import latent_flow_matching_b200 as F
from oracle import flux_oracle as O
from synthetic import WORKLOADS, make_weights, make_inputs

pytestmark = pytest.mark.gpu
torch.set_grad_enabled(False)
DEV = "cuda"
LEAK_BYTES = 64 << 20          # driver bookkeeping may move free memory a little; a leaked weight buffer is GBs


@pytest.fixture(autouse=True)
def _disarm():
    yield
    F.flux_test_fail_alloc_after(-1)
    torch.cuda.synchronize()
    assert F.flux_device_error() == 0


@pytest.fixture(scope="module")
def tiny_blob():
    w = WORKLOADS["tiny64"]
    blob, _ = make_weights(w.dims, w.seed)
    return w, blob


def free_bytes():
    torch.cuda.synchronize()
    return torch.cuda.mem_get_info()[0]


def expect_enomem(fn):
    with pytest.raises(F.FluxError) as e:
        fn()
    assert e.value.code == F.FLUX_ENOMEM, e.value
    assert "allocation" in str(e.value)


def inputs(w, grid, nt, seed):
    g = torch.Generator().manual_seed(seed)
    tok = torch.randn(grid[0] * grid[1], 128, generator=g).to(torch.bfloat16).float().to(DEV)
    txt = torch.randn(nt, w.dims.txt_dim, generator=g).to(torch.bfloat16).float().to(DEV)
    return tok, txt


def forward(model, tok, grid, txt, t=0.625):
    v = torch.empty(tok.shape[0], 128, device=DEV)
    model.forward(tok, grid, txt, t, v)
    torch.cuda.synchronize()
    return v


def test_create_fails_cleanly_at_each_allocation(tiny_blob):
    """Model creation with its k-th device allocation failing, for every k until creation succeeds:
    NULL with FLUX_ENOMEM, and no device memory kept."""
    w, blob = tiny_blob
    before = free_bytes()
    k = 0
    while True:
        F.flux_test_fail_alloc_after(k)
        try:
            model = F.FluxDiT(blob, w.dims)
        except F.FluxError as e:
            assert e.code == F.FLUX_ENOMEM and "allocation" in str(e), e
            assert before - free_bytes() < LEAK_BYTES, k
            k += 1
            assert k < 64
            continue
        break
    F.flux_test_fail_alloc_after(-1)
    assert k >= 2                                 # the weights and the modulation buffers at least
    model.close()
    assert before - free_bytes() < LEAK_BYTES


def test_forward_workspace_failures_leave_the_model_usable(tiny_blob):
    """The first forward allocates the activation workspace; failing each of its allocations in
    turn returns FLUX_ENOMEM, and the forward that finally runs equals a fresh model's, bit for bit.
    Then a shape that needs only a larger token buffer fails on it, and a forward at the earlier
    shape (whose tensor maps must be rebuilt over the new buffer) and one at the new shape both
    equal the fresh model's."""
    w, blob = tiny_blob
    ref = F.FluxDiT(blob, w.dims)
    model = F.FluxDiT(blob, w.dims)
    try:
        tok, txt = inputs(w, (4, 4), 64, 1)
        want = forward(ref, tok, (4, 4), txt)
        k = 0
        while True:
            F.flux_test_fail_alloc_after(k)
            try:
                got = forward(model, tok, (4, 4), txt)
            except F.FluxError as e:
                assert e.code == F.FLUX_ENOMEM and "allocation" in str(e), e
                k += 1
                assert k < 64
                continue
            break
        F.flux_test_fail_alloc_after(-1)
        assert k >= 5
        assert torch.equal(got, want)
        # 16 text + 36 image rows (fewer rows than 64 + 16, more image tokens): only the token
        # staging buffer grows, and that allocation fails
        tok2, txt2 = inputs(w, (6, 6), 16, 2)
        F.flux_test_fail_alloc_after(0)
        expect_enomem(lambda: forward(model, tok2, (6, 6), txt2))
        F.flux_test_fail_alloc_after(-1)
        assert torch.equal(forward(model, tok, (4, 4), txt), want)
        assert torch.equal(forward(model, tok2, (6, 6), txt2), forward(ref, tok2, (6, 6), txt2))
    finally:
        model.close()
        ref.close()


@pytest.mark.parametrize("precision", [F.PRECISION_FP8, F.PRECISION_NVFP4])
def test_precision_and_its_workspace_failures_leave_the_model_usable(tiny_blob, precision):
    """Switching precision allocates the quantised weights, and the first forward in it the
    quantised activations: a failure in either returns FLUX_ENOMEM and changes nothing (the model
    stays in bf16 after a failed switch); the calls that follow match a fresh model's."""
    w, blob = tiny_blob
    ref = F.FluxDiT(blob, w.dims)
    model = F.FluxDiT(blob, w.dims)
    try:
        tok, txt = inputs(w, (4, 4), 16, 3)
        want_bf16 = forward(ref, tok, (4, 4), txt)
        F.flux_test_fail_alloc_after(0)
        expect_enomem(lambda: model.set_precision(precision))
        F.flux_test_fail_alloc_after(-1)
        assert torch.equal(forward(model, tok, (4, 4), txt), want_bf16)
        model.set_precision(precision)
        ref.set_precision(precision)
        want = forward(ref, tok, (4, 4), txt)
        F.flux_test_fail_alloc_after(0)
        expect_enomem(lambda: forward(model, tok, (4, 4), txt))
        F.flux_test_fail_alloc_after(-1)
        assert torch.equal(forward(model, tok, (4, 4), txt), want)
    finally:
        model.close()
        ref.close()


def test_timestep_preparation_failure_leaves_per_forward_modulation(tiny_blob):
    """A failed flux_dit_prepare_timesteps keeps no vectors: forwards compute their own modulation
    and equal a fresh model's; a later preparation succeeds."""
    w, blob = tiny_blob
    ref = F.FluxDiT(blob, w.dims)
    model = F.FluxDiT(blob, w.dims)
    try:
        tok, txt = inputs(w, (4, 4), 16, 4)
        want = forward(ref, tok, (4, 4), txt, t=0.5)
        F.flux_test_fail_alloc_after(0)
        expect_enomem(lambda: model.prepare_timesteps([1.0, 0.5]))
        F.flux_test_fail_alloc_after(-1)
        assert torch.equal(forward(model, tok, (4, 4), txt, t=0.5), want)
        model.prepare_timesteps([1.0, 0.5])
        assert torch.equal(forward(model, tok, (4, 4), txt, t=0.5), want)
    finally:
        model.close()
        ref.close()


def test_flux3_create_and_forward_fail_cleanly(tiny_blob):
    """The FLUX.3 runner: creation and the first forward, each with one allocation failing, then
    both succeeding and matching a fresh model's forward."""
    w3 = WORKLOADS["f3tiny64"]
    blob3, _ = make_weights(w3.dims, w3.seed)
    before = free_bytes()
    for k in (0, 1):
        F.flux_test_fail_alloc_after(k)
        with pytest.raises(F.FluxError) as e:
            F.Flux3DiT(blob3, w3.dims)
        assert e.value.code == F.FLUX_ENOMEM
        assert before - free_bytes() < LEAK_BYTES
    F.flux_test_fail_alloc_after(-1)
    ref = F.Flux3DiT(blob3, w3.dims)
    model = F.Flux3DiT(blob3, w3.dims)
    try:
        g = torch.Generator().manual_seed(5)
        tok = torch.randn(16, 128, generator=g).to(torch.bfloat16).float().to(DEV)
        txt = torch.randn(16, w3.dims.txt_dim, generator=g).to(torch.bfloat16).float().to(DEV)

        def fwd(m):
            v = torch.empty(16, 128, device=DEV)
            m.forward(tok, (4, 4), txt, 0.75, v, t_target=0.5)
            torch.cuda.synchronize()
            return v
        want = fwd(ref)
        F.flux_test_fail_alloc_after(2)
        with pytest.raises(F.FluxError) as e:
            fwd(model)
        assert e.value.code == F.FLUX_ENOMEM
        F.flux_test_fail_alloc_after(-1)
        assert torch.equal(fwd(model), want)
    finally:
        model.close()
        ref.close()
