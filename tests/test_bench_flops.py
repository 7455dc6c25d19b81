"""The bench's algorithmic FLOP count, recounted from the model's own weight list.

Every 2-D weight that multiplies token rows costs 2 x rows x out x in; the rows of a weight follow
from the stream it belongs to (text, image + references, all tokens, image only for the output
layer).  Modulation and time-embedding linears act on one vector per forward and are not counted.
Attention costs 4 N^2 D per block over the sequence it attends (FLUX.3 per-mode blocks: each
stream on its own).  The bench's closed form must equal this recount, and the FLUX.2 figures the
value quoted for the five configurations (4.90 / 10.16 / 34.80 / 76.68 TFLOP at 256^2, 512^2,
1024^2 and 1024^2 + a 1024^2 reference).
"""
import pytest

import bench
from synthetic import WORKLOADS, tensor_specs

F2 = ["tiny64", "t2i256", "t2i512", "t2i1024", "i2i1024", "mref1024"]
F3 = ["f3tiny64", "f3t2i256", "f3i2i256", "f3t2i1024", "f3i2i1024"]


def rows_of(name, w):
    img, txt = w.n_img + w.n_ref, w.n_txt
    if name.startswith("img_in") or ".img." in name:
        return img
    if name.startswith("txt_in") or ".txt." in name:
        return txt
    if ".ref." in name:
        return w.n_ref
    if name.startswith("final.out"):
        return w.n_img
    if name.startswith(("single.", "joint.")):
        return w.n_tokens
    raise AssertionError(name)


def recount(w, only=None):
    """FLOPs of the forward; with `only`, of the weights it accepts (and no attention)."""
    d = w.dims
    total = 0.0
    for name, shape, _ in tensor_specs(d):
        modulation = name.endswith(".mod.w") or name.startswith(("mode_mod.", "joint_mod."))
        if len(shape) != 2 or modulation or name.startswith(("time_in", "target_in")):
            continue
        if only is not None and not only(name):
            continue
        if ".img." in name and name.startswith("mode."):
            rows = w.n_img                      # FLUX.3 per-mode: the image stream without references
        else:
            rows = rows_of(name, w)
        total += 2.0 * rows * shape[0] * shape[1]
    D = d.hidden
    if only is not None:
        return total
    if hasattr(d, "n_mode"):
        total += d.n_joint * 4.0 * w.n_tokens ** 2 * D
        total += d.n_mode * 4.0 * D * (w.n_txt ** 2 + w.n_img ** 2 + w.n_ref ** 2)
    else:
        total += (d.n_double + d.n_single) * 4.0 * w.n_tokens ** 2 * D
    return total


@pytest.mark.parametrize("name", F2 + F3)
def test_forward_flops_equal_the_recount_from_the_weight_list(name):
    w = WORKLOADS[name]
    assert bench.forward_flops(w) == pytest.approx(recount(w), rel=1e-12)


@pytest.mark.parametrize("name,tflop", [("t2i256", 4.90), ("t2i512", 10.16), ("t2i1024", 34.80),
                                        ("i2i1024", 76.68)])
def test_flux2_forward_flops_match_the_quoted_figures(name, tflop):
    assert bench.forward_flops(WORKLOADS[name]) / 1e12 == pytest.approx(tflop, abs=0.006)


def test_guided_step_counts_two_sequences():
    for name in ("cfg256", "cfg1024"):
        w = WORKLOADS[name]
        assert bench.step_flops(w) == pytest.approx(2 * bench.forward_flops(w), rel=1e-12)


def test_flux3_guided_step_shares_the_text_free_streams():
    """A FLUX.3 guided step is two forwards, less what the two sequences share: the image input
    projection and the per-mode image and reference streams (linears and their own attention)."""
    w = WORKLOADS["f3cfg256"]
    d = w.dims
    shared = recount(w, lambda n: n.startswith("img_in") or (n.startswith("mode.") and (".img." in n or ".ref." in n)))
    shared += d.n_mode * 4.0 * d.hidden * (w.n_img ** 2 + w.n_ref ** 2)
    assert bench.step_flops(w) == pytest.approx(2 * recount(w) - shared, rel=1e-12)
