"""Write the oracle's sampled outputs for the full-size workloads to tests/golden/.

Calls only ``synthetic`` (seeded inputs) and ``oracle`` (CPU definition).  For
each workload it runs the whole Euler sampler in float32 (the precision of the
pages' own C implementation) and stores, for a fixed set of token rows, every
step's velocity and the final packed latent:

    <workload>.npz: rows int32 [R], v float32 [S, R, 128], final float32 [R, 128]

Row sets: all rows at 256^2, every 2nd at 512^2, every 8th at 1024^2.  For a guided workload
the stored velocities are the guided ones.

Quantised goldens (``<workload>_fp8``, ``<workload>_nvfp4``) run the same sampler with the block
linears in row-wise FP8 or NVFP4 (the oracle's ``hp["fp8"]`` / ``hp["nvfp4"]``), on the same seeded
weights and inputs as the bf16 workload they name; ``meta.precision`` says which.  They also hold
``v_pert``: the step-0 velocity of the same quantised oracle with every quantiser input multiplied
by (1 + u 2^-9), u uniform in [-1, 1] from a seeded generator (one bf16 rounding's worth).  Over 25
blocks a quantised forward is not continuous in its quantiser inputs (an input crossing a rounding
boundary moves a whole code step), so rel-L2(v_pert[0], v[0]) measures how far any evaluation
carrying bf16-sized perturbations must land from the oracle; the GPU test sets its bar from it.
At 1024^2 the quantised goldens run the first STEPS_RUN steps (``meta.steps_run``).

FLUX.3 workloads (``f3*``) use the FLUX.3 oracle with the flow-map target time t_{i+1}; the
8272-token image-to-image case runs the first STEPS_RUN steps of its 16-step schedule (``v`` then
holds those steps and ``final`` the packed state after them, ``meta.steps_run`` says how many).
The base-checkpoint workload (``f3cfg256``, no target time) is guided: each step evaluates the
prompt and the unconditional text and stores the guided velocity.

Usage: python tests/golden/make_goldens.py [workload ...]   (about an hour on 8 cores)
"""
import json
import os
import sys
import time

import numpy as np
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from synthetic import WORKLOADS, make_weights, make_inputs, make_uncond_text  # noqa: E402
from oracle import flux_oracle as O  # noqa: E402
from oracle import flux3_oracle as O3  # noqa: E402

ROW_STRIDE = {"t2i256": 1, "t2i512": 2, "t2i1024": 8, "i2i1024": 8, "mref1024": 8, "cfg256": 1,
              "f3t2i256": 1, "f3i2i256": 1, "f3t2i1024": 8, "f3i2i1024": 8, "f3cfg256": 1,
              "t2i256_fp8": 1, "t2i256_nvfp4": 1, "t2i1024_fp8": 8, "t2i1024_nvfp4": 8,
              "f3t2i256_fp8": 1, "f3t2i256_nvfp4": 1, "f3t2i1024_fp8": 8, "f3t2i1024_nvfp4": 8}
STEPS_RUN = {"f3i2i1024": 4, "t2i1024_fp8": 2, "t2i1024_nvfp4": 2, "f3t2i1024_fp8": 2, "f3t2i1024_nvfp4": 2}
PRECISIONS = ("fp8", "nvfp4")


def split_name(name):
    """(workload, precision): 't2i256_nvfp4' -> ('t2i256', 'nvfp4'); plain names are bf16."""
    base, _, prec = name.rpartition("_")
    return (base, prec) if prec in PRECISIONS else (name, "bf16")


def rows_for(name):
    w = WORKLOADS[split_name(name)[0]]
    return np.arange(0, w.n_img, ROW_STRIDE[name], dtype=np.int32)


def make3(name):
    """FLUX.3 sampler: forward3 with target time t_{i+1}, Euler update, for the first k steps."""
    base, precision = split_name(name)
    w = WORKLOADS[base]
    t0 = time.time()
    _, p = make_weights(w.dims, w.seed)
    lat, txt, ref = make_inputs(w)
    rows = rows_for(name)
    k = STEPS_RUN.get(name, w.n_steps)
    hp = O.hyper(w.dims)
    if precision != "bf16":
        hp[precision] = True
    ts = O.schedule(w.n_steps)
    tok = O.pack_latents(torch.from_numpy(lat)).float()
    refs = [] if ref is None else (ref if isinstance(ref, list) else [ref])
    ref_toks = [O.pack_latents(torch.from_numpy(r)).float() for r in refs]
    ref_grids = [(r.shape[1] // 2, r.shape[2] // 2) for r in refs]
    txt_u = torch.from_numpy(make_uncond_text(w)) if w.guidance is not None else None
    extra = {}
    if precision != "bf16":
        tt = ts[1] if w.dims.flow_map else None
        extra["v_pert"] = perturbed(precision, lambda: O3.forward3(
            p, hp, tok, torch.from_numpy(txt), ts[0], (w.grid, w.grid), ref_toks, ref_grids, t_target=tt,
            dtype=torch.float32))[rows].float().numpy()[None]
        print(f"  {name} perturbed step 0 done at {time.time() - t0:.0f}s", flush=True)
    vs = []
    for i in range(k):
        tt = ts[i + 1] if w.dims.flow_map else None
        v = O3.forward3(p, hp, tok, torch.from_numpy(txt), ts[i], (w.grid, w.grid), ref_toks, ref_grids,
                        t_target=tt, dtype=torch.float32)
        if txt_u is not None:
            v_u = O3.forward3(p, hp, tok, txt_u, ts[i], (w.grid, w.grid), ref_toks, ref_grids, t_target=tt,
                              dtype=torch.float32)
            v = O.guided_velocity(v, v_u, w.guidance)
        vs.append(v[rows].float().numpy())
        tok = O.euler_update(tok, v, ts[i + 1] - ts[i])
        print(f"  {name} step {i} done at {time.time() - t0:.0f}s", flush=True)
    meta = {"workload": base, "precision": precision, "seed": w.seed, "oracle_dtype": "float32",
            "n_steps": w.n_steps, "steps_run": k, "flow_map": bool(w.dims.flow_map), "guidance": w.guidance,
            "row_stride": ROW_STRIDE[name], "seconds": round(time.time() - t0, 1)}
    np.savez(os.path.join(HERE, f"{name}.npz"), rows=rows, v=np.stack(vs), final=tok[rows].float().numpy(),
             meta=np.array(json.dumps(meta)), **extra)
    print(f"{name}: wrote {len(rows)} rows x {k} steps in {time.time() - t0:.0f}s", flush=True)


def perturbed(precision, run):
    """run() with every quantiser input of the oracle's FP8 / NVFP4 linears multiplied by
    (1 + u 2^-9), u uniform in [-1, 1] from a generator seeded with 0 (one bf16 rounding's worth)."""
    from oracle import fp8_oracle as Q8
    from oracle import nvfp4_oracle as Q4
    mod, attr = (Q8, "linear_fp8") if precision == "fp8" else (Q4, "linear_nvfp4")
    plain = getattr(mod, attr)
    g = torch.Generator().manual_seed(0)

    def perturbed_linear(x, wt, b):
        x = torch.as_tensor(x)
        u = torch.rand(x.shape, generator=g, dtype=torch.float64) * 2 - 1
        return plain(x * (1 + u * 2.0 ** -9).to(x.dtype), wt, b)
    setattr(mod, attr, perturbed_linear)
    try:
        return run()
    finally:
        setattr(mod, attr, plain)


def perturbed_step0(p, hp, precision, lat, txt, ref, w):
    """Step-0 velocity of the quantised FLUX.2 oracle with its quantiser inputs perturbed."""
    tok = O.pack_latents(torch.from_numpy(lat)).float()
    refs, grids = [], []
    for r in ([] if ref is None else (ref if isinstance(ref, list) else [ref])):
        refs.append(O.pack_latents(torch.from_numpy(r)).float())
        grids.append((r.shape[1] // 2, r.shape[2] // 2))
    return perturbed(precision, lambda: O.forward(p, hp, tok, torch.from_numpy(txt), O.schedule(w.n_steps)[0],
                                                  (w.grid, w.grid), refs, grids, dtype=torch.float32))


def make(name):
    if name.startswith("f3"):
        return make3(name)
    base, precision = split_name(name)
    w = WORKLOADS[base]
    t0 = time.time()
    _, p = make_weights(w.dims, w.seed)
    lat, txt, ref = make_inputs(w)
    rows = rows_for(name)
    k = STEPS_RUN.get(name, w.n_steps)
    hp = O.hyper(w.dims)
    if precision != "bf16":
        hp[precision] = True
    extra = {}
    if precision != "bf16":
        extra["v_pert"] = perturbed_step0(p, hp, precision, lat, txt, ref, w)[rows].float().numpy()[None]
        print(f"  {name} perturbed step 0 done at {time.time() - t0:.0f}s", flush=True)
    if k < w.n_steps:                              # the first k steps of the schedule, by hand
        ts = O.schedule(w.n_steps)
        tok = O.pack_latents(torch.from_numpy(lat)).float()
        vs = []
        for i in range(k):
            v = O.forward(p, hp, tok, torch.from_numpy(txt), ts[i], (w.grid, w.grid), dtype=torch.float32)
            vs.append(v[rows].float().numpy())
            tok = O.euler_update(tok, v, ts[i + 1] - ts[i])
            print(f"  {name} step {i} done at {time.time() - t0:.0f}s", flush=True)
        final_tok = tok[rows].float().numpy()
    else:
        vs = []

        def on_step(i, v):
            vs.append(v[rows].float().numpy())
            print(f"  {name} step {i} done at {time.time() - t0:.0f}s", flush=True)

        with torch.no_grad():
            if isinstance(ref, list):
                ref = [torch.from_numpy(r) for r in ref]
            elif ref is not None:
                ref = torch.from_numpy(ref)
            guided = {}
            if w.guidance is not None:
                guided = {"txt_uncond": torch.from_numpy(make_uncond_text(w)), "guidance": w.guidance}
            final, _ = O.sample(p, hp, torch.from_numpy(lat), torch.from_numpy(txt),
                                w.n_steps, ref, dtype=torch.float32, on_step=on_step, **guided)
        final_tok = O.pack_latents(final)[rows].float().numpy()
    meta = {"workload": base, "precision": precision, "seed": w.seed, "oracle_dtype": "float32",
            "n_steps": w.n_steps, "steps_run": k, "guidance": w.guidance, "row_stride": ROW_STRIDE[name],
            "seconds": round(time.time() - t0, 1)}
    np.savez(os.path.join(HERE, f"{name}.npz"), rows=rows, v=np.stack(vs), final=final_tok,
             meta=np.array(json.dumps(meta)), **extra)
    print(f"{name}: wrote {len(rows)} rows x {k} steps in {time.time() - t0:.0f}s", flush=True)


if __name__ == "__main__":
    torch.set_grad_enabled(False)
    for n in (sys.argv[1:] or list(ROW_STRIDE)):
        make(n)
