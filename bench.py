#!/usr/bin/env python
"""Benchmark of the FLUX.2-klein denoising-transformer step on B200.

One step = one sampling step of the 1024x1024 text-to-image workload (4096
image + 512 text tokens, 5 double + 20 single blocks, width 3072, 24 heads):
pack the latent -> transformer forward -> Euler update -> unpack, all through
the library's C ABI on one CUDA stream.  Prints one JSON line (rank 0):

  value     ms per DiT forward (whole job: max-over-ranks time / forwards of all ranks)
  e2e       the same through host buffers (H2D of latent + text, D2H of the latent, per step)
  roofline  the tcgen05 GEMM (most of the FLOPs) from CUDA events around its launches
  cpu_baseline   the CPU oracle on a bounded sample (rank 0, one GPU only)

``--impl reference`` times the CPU oracle instead (rank 0 only).

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
Multi-GPU: torchrun --nproc-per-node N bench.py --gpus N  (independent replicas, no data-path collective)
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from synthetic import WORKLOADS, Flux3Dims, make_weights, make_inputs, make_uncond_text  # noqa: E402

METRIC = "ms per DiT forward & TFLOP/s at 1024^2 (4096+512 tok), % of BF16 peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
SPEC_BF16_TFLOPS = 2250.0


def is_flux3(w):
    return isinstance(w.dims, Flux3Dims)


def n_blocks(w):
    d = w.dims
    return d.n_mode + d.n_joint if is_flux3(w) else d.n_double + d.n_single


def blocks_text(w):
    d = w.dims
    if is_flux3(w):
        return f"FLUX.3 Image Klein: {d.n_mode} per-mode + {d.n_joint} joint blocks"
    return f"{d.n_double} double + {d.n_single} single blocks"


def forward_flops(w):
    """Algorithmic FLOPs of one forward: dense linears + non-causal attention (QK^T and PV).

    Every block's linears cost N 2D(4D + 3F) over its rows.  FLUX.2 blocks and FLUX.3 joint blocks
    attend over the whole sequence (4 N^2 D); FLUX.3 per-mode blocks attend within each stream
    (4 D (Nt^2 + Ni^2 + Nr^2))."""
    d = w.dims
    D, F_, C = d.hidden, d.mlp_hidden, d.in_ch
    n = w.n_tokens
    lin = n * 2.0 * D * (4 * D + 3 * F_)
    if is_flux3(w):
        total = (d.n_mode + d.n_joint) * lin + d.n_joint * 4.0 * n * n * D
        total += d.n_mode * 4.0 * D * (w.n_txt ** 2 + w.n_img ** 2 + w.n_ref ** 2)
    else:
        total = (d.n_double + d.n_single) * (lin + 4.0 * n * n * D)
    total += 2.0 * (w.n_img + w.n_ref) * C * D + 2.0 * w.n_txt * d.txt_dim * D + 2.0 * w.n_img * D * C
    return total


def n_sequences(w):
    """Sequences per forward: 2 for a guided workload (prompt and unconditional text in one batch)."""
    return 1 if w.guidance is None else 2


def step_flops(w):
    """FLOPs of one sampling step's forward work.  A guided step evaluates two sequences; in a
    FLUX.3 guided batch the per-mode image and reference streams (which never see the text) and
    the image input projection are computed once for both."""
    total = n_sequences(w) * forward_flops(w)
    if is_flux3(w) and n_sequences(w) == 2:
        d = w.dims
        D, F_, C = d.hidden, d.mlp_hidden, d.in_ch
        rows = w.n_img + w.n_ref
        shared = d.n_mode * (rows * 2.0 * D * (4 * D + 3 * F_) + 4.0 * D * (w.n_img ** 2 + w.n_ref ** 2))
        total -= shared + 2.0 * rows * C * D
    return total


def step_unit(w):
    return "ms/forward" if w.guidance is None else "ms/guided step (batch-2 forward)"


def single_block_flops(w):
    d, n = w.dims, w.n_tokens
    return n * 2.0 * d.hidden * (4 * d.hidden + 3 * d.mlp_hidden) + 4.0 * n * n * d.hidden


def weight_gb(w):
    from synthetic import blob_layout
    return blob_layout(w.dims)[1] / 1e9


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        j = json.load(open(p))
        return {k: float(j[k]) for k in FALLBACK_PEAKS}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"fluxdit_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for nm, val in zip(names, f[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------- helpers
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(x, world):
    """Max of a host scalar over all ranks (NCCL on the GPU machine; gloo in the CPU tests)."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_ms_per_forward(ms_total_max, steps, world):
    """Whole-job time per forward: every rank runs `steps` independent forwards (replicas)."""
    return ms_total_max / (steps * world)


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


CPU_SAMPLE_BLOCKS = 4      # double and single blocks the CPU sample runs (FLUX.2): about 12 s on 16 cores


def cpu_oracle_sample(w, params, lat, txt, ref):
    """The fp32 oracle on host cores, on this workload's own latent and text: a forward of the model
    cut to its first CPU_SAMPLE_BLOCKS double and single blocks (time MLP, input projections, those
    blocks in order on the real activations, output layer), scaled to the full forward by algorithmic
    FLOPs (FLUX.3: one joint block, scaled the same way)."""
    import dataclasses
    from oracle import flux_oracle as O
    torch.set_grad_enabled(False)
    if is_flux3(w):
        ms_block, secs = oracle_joint_block_ms(w, params)
        return ms_block * forward_flops(w) / single_block_flops(w), secs
    k = CPU_SAMPLE_BLOCKS
    keep = {name: v for name, v in params.items()
            if not ((name.startswith("double.") and int(name.split(".")[1]) >= k) or
                    (name.startswith("single.") and int(name.split(".")[1]) >= k))}
    cut = dataclasses.replace(w, dims=dataclasses.replace(w.dims, n_double=k, n_single=k))
    tok = O.pack_latents(torch.from_numpy(lat)).float()
    refs, ref_grids = [], []
    if ref is not None:
        for r in (ref if isinstance(ref, list) else [ref]):
            refs.append(O.pack_latents(torch.from_numpy(r)).float())
            ref_grids.append((r.shape[1] // 2, r.shape[2] // 2))
    t0 = time.perf_counter()
    O.forward(keep, O.hyper(w.dims), tok, torch.from_numpy(txt), 1.0, (w.grid, w.grid), refs, ref_grids,
              dtype=torch.float32)
    secs = time.perf_counter() - t0
    return 1e3 * secs * forward_flops(w) / forward_flops(cut), secs


def oracle_joint_block_ms(w, params, repeats=1):
    """fp32 oracle time of one FLUX.3 joint block at the workload's full size (host cores)."""
    from oracle import flux_oracle as O
    from oracle import flux3_oracle as O3
    torch.set_grad_enabled(False)
    hp = O.hyper(w.dims)
    D = w.dims.hidden
    g = torch.Generator().manual_seed(0)
    x = torch.randn(w.n_tokens, D, generator=g)
    sh, sc, gt = (torch.randn(D, generator=g) for _ in range(3))
    ang = O.rope_angles(O.token_positions(w.n_txt, w.grid, w.grid, ref_grids=w.ref_grids), 128, 1e4).float()
    t0 = time.perf_counter()
    for _ in range(repeats):
        O3.parallel_block(params, "joint.0.", x, sh, sc, gt, ang, hp, torch.float32)
    secs = time.perf_counter() - t0
    return 1e3 * secs / repeats, secs


# ---------------------------------------------------------------------------- reference arm (CPU oracle)
def run_reference(args, w):
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    from oracle import flux_oracle as O
    torch.set_grad_enabled(False)
    _, params = make_weights(w.dims, w.seed)
    if is_flux3(w):
        return run_reference3(args, w, params)
    hp = O.hyper(w.dims)
    D = w.dims.hidden
    g = torch.Generator().manual_seed(0)
    x = torch.randn(w.n_tokens, D, generator=g)
    s = torch.randn(D, generator=g)
    ang = O.rope_angles(O.token_positions(w.n_txt, w.grid, w.grid, ref_grids=w.ref_grids), 128, 1e4).float()
    scale = n_sequences(w) * forward_flops(w) / single_block_flops(w)
    for _ in range(args.warmup):
        O.single_block(params, 0, x, s, ang, hp, torch.float32)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        O.single_block(params, 0, x, s, ang, hp, torch.float32)
        times.append(time.perf_counter() - t0)
    ms_block = 1e3 * sum(times) / len(times)
    value = ms_block * scale
    sample = (f"one single-stream block at the full {w.name} size ({w.n_tokens} tokens) per step, fp32 oracle; "
              f"value scaled by (sequences x forward FLOPs) / block FLOPs = {scale:.2f}")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": step_unit(w),
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_block, 3),
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded N(0,1) bf16-rounded weights and inputs)",
        "config": {"workload": f"{w.name}: {w.image}x{w.image}, {w.n_img} image + {w.n_txt} text + {w.n_ref} "
                               f"reference tokens, {blocks_text(w)}, width 3072", "seq_len": w.n_tokens,
                   "global_batch": 1, "parallelism": "CPU oracle on rank 0"},
        "tflops": round(n_sequences(w) * forward_flops(w) / (value / 1e3) / 1e12, 4),
        "cpu_baseline": {"value": round(value, 3), "unit": step_unit(w), "cores": torch.get_num_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 3), "unit": step_unit(w), "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_reference3(args, w, params):
    """Reference arm for a FLUX.3 workload: the fp32 oracle's joint block, scaled to a forward."""
    for _ in range(args.warmup):
        oracle_joint_block_ms(w, params)
    times = [oracle_joint_block_ms(w, params)[0] for _ in range(args.steps)]
    ms_block = sum(times) / len(times)
    scale = n_sequences(w) * forward_flops(w) / single_block_flops(w)
    value = ms_block * scale
    sample = (f"one joint block at the full {w.name} size ({w.n_tokens} tokens) per step, fp32 oracle; "
              f"value scaled by (sequences x forward FLOPs) / block FLOPs = {scale:.2f}")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": step_unit(w),
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_block, 3),
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded N(0,1) bf16-rounded weights and inputs)",
        "config": {"workload": f"{w.name}: {w.image}x{w.image}, {w.n_img} image + {w.n_txt} text + {w.n_ref} "
                               f"reference tokens, {blocks_text(w)}, width 3072", "seq_len": w.n_tokens,
                   "global_batch": 1, "parallelism": "CPU oracle on rank 0"},
        "tflops": round(n_sequences(w) * forward_flops(w) / (value / 1e3) / 1e12, 4),
        "cpu_baseline": {"value": round(value, 3), "unit": step_unit(w), "cores": torch.get_num_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 3), "unit": step_unit(w), "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def fractions(tflops, peaks, fp4=False, fp8=False):
    """A tensor-bound rate against every bf16 ceiling: the measured sustained and burst cuBLAS figures
    and the 2250 TFLOP/s dense datasheet figure (FP8 / NVFP4 rates against 2x / 4x each)."""
    mult = 4.0 if fp4 else 2.0 if fp8 else 1.0
    return {"measured_sustained": round(tflops / (mult * peaks["bf16_tflops_sustained"]), 4),
            "measured_burst": round(tflops / (mult * peaks["bf16_tflops"]), 4),
            "spec_2250": round(tflops / (mult * SPEC_BF16_TFLOPS), 4)}


def gemm_roofline(g_ms, g_fl, g_by, peaks, peak_src, fp4=False, fp8=False):
    """The linears' roofline entries from their summed device time, FLOPs and algorithmic bytes.

    The GEMM peak is the measured sustained bf16 rate (2x for FP8, 4x for NVFP4: the nominal dense
    ratios).  When the FLOPs per algorithmic byte fall below the ridge point (peak / measured copy
    bandwidth), as on the tiny model's 16-row problems where the weights' read bounds each launch,
    the entries are the HBM roofline in GB/s; otherwise the tensor roofline in TFLOP/s."""
    gemm_peak = peaks["bf16_tflops_sustained"] * (4.0 if fp4 else 2.0 if fp8 else 1.0)
    peak_kind = ("nvfp4 = 4 x bf16 sustained (nominal dense ratio), " if fp4 else
                 "fp8 = 2 x bf16 sustained (nominal dense ratio), " if fp8 else "bf16 sustained, ") + peak_src
    tflops = g_fl / (g_ms / 1e3) / 1e12
    gbs = g_by / (g_ms / 1e3) / 1e9
    intensity = g_fl / g_by if g_by else float("inf")
    ridge = gemm_peak * 1e12 / (peaks["hbm_gbs"] * 1e9)
    if intensity < ridge:
        out = {"bound": "hbm", "achieved": round(gbs, 1), "peak": round(peaks["hbm_gbs"], 1), "unit": "GB/s",
               "frac": round(gbs / peaks["hbm_gbs"], 4), "peak_kind": f"HBM copy, {peak_src}",
               "tflops": round(tflops, 2)}
    else:
        out = {"bound": "tensor", "achieved": round(tflops, 1), "peak": round(gemm_peak, 1), "unit": "TFLOP/s",
               "frac": round(tflops / gemm_peak, 4), "peak_kind": peak_kind,
               "frac_of": fractions(tflops, peaks, fp4=fp4, fp8=fp8)}
    out.update(flop_per_byte=round(intensity, 1), ridge_flop_per_byte=round(ridge, 1))
    return out


TENSOR_KINDS = ("gemm", "attention")


def kernel_kind_line(kind, v_, steps, peaks):
    """One kernel kind's per-forward time and rate: TFLOP/s for the tensor-core kinds, GB/s of
    algorithmic bytes (against the measured copy bandwidth) for the memory-bound ones."""
    ms, fl, by, n = v_
    line = {"ms_per_forward": round(ms / steps, 4), "launches_per_forward": round(n / steps, 3)}
    if kind in TENSOR_KINDS:
        line.update(achieved=round(fl / (ms / 1e3) / 1e12, 1), unit="TFLOP/s")
    else:
        gbs = by / (ms / 1e3) / 1e9
        line.update(achieved=round(gbs, 1), unit="GB/s", frac_of_hbm_copy=round(gbs / peaks["hbm_gbs"], 4))
    return line


# ---------------------------------------------------------------------------- our arm
def run_ours(args, w):
    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=torch.device("cuda", local))
    import latent_flow_matching_b200 as F
    if not os.path.exists(F.LIB_PATH):             # a fresh checkout: compile the sm_100a library first
        from latent_flow_matching_b200 import build as B
        B.build()
    F.lib()                                         # fails loudly if the library is missing
    torch.set_grad_enabled(False)

    blob, params = make_weights(w.dims, w.seed)
    lat_h, txt_h, ref_h = make_inputs(w)
    flux3 = is_flux3(w)
    model = (F.Flux3DiT if flux3 else F.FluxDiT)(blob, w.dims)
    del blob
    fp8 = args.precision == "fp8"
    fp4 = args.precision == "nvfp4"
    if fp8:
        model.set_precision(F.PRECISION_FP8)
    if fp4:
        model.set_precision(F.PRECISION_NVFP4)
    stream = torch.cuda.current_stream()
    dev = torch.device("cuda", local)
    lat0 = torch.from_numpy(lat_h).to(dev)
    lat = lat0.clone()
    txt = torch.from_numpy(txt_h).to(dev)
    gh = w.grid
    tok = torch.empty(w.n_img, 128, device=dev)
    v = torch.empty_like(tok)
    ref_tok, ref_hw = None, (0, 0)
    if ref_h is not None:
        ref_tok = torch.empty(w.n_ref, 128, device=dev)
        row = 0
        for r, (h, w_) in zip(ref_h if isinstance(ref_h, list) else [ref_h], w.ref_grids):
            F.flux_pack_latents(torch.from_numpy(r).to(dev), ref_tok[row:row + h * w_])
            row += h * w_
        ref_hw = w.ref_grids if isinstance(ref_h, list) else w.ref_grids[0]
    ts = F.euler_schedule(w.n_steps)
    guided = w.guidance is not None
    txt_u_h = make_uncond_text(w) if guided else None
    txt_u = torch.from_numpy(txt_u_h).to(dev) if guided else None
    v_u = torch.empty_like(tok)
    hw_list = list(w.ref_grids)

    def forward_update(k):
        """The forward(s) of one sampling step and its Euler update."""
        if guided:
            if flux3:
                model.forward_cfg(tok, (gh, gh), txt, txt_u, ts[k], v, v_u, ref_tok, hw_list, t_target=ts[k + 1])
            else:
                model.forward_cfg(tok, (gh, gh), txt, txt_u, ts[k], v, v_u, ref_tok, hw_list)
            F.flux_cfg_euler_step(tok, v, v_u, w.guidance, ts[k + 1] - ts[k])
        elif flux3:                                 # flow-map checkpoint: target time t_{k+1}
            model.forward(tok, (gh, gh), txt, ts[k], v, ref_tok, hw_list, t_target=ts[k + 1])
            F.flux_euler_step(tok, v, ts[k + 1] - ts[k])
        else:
            model.forward(tok, (gh, gh), txt, ts[k], v, ref_tok, ref_hw)
            F.flux_euler_step(tok, v, ts[k + 1] - ts[k])

    def step(i, lat_buf):
        k = i % w.n_steps
        if k == 0:
            lat_buf.copy_(lat0)                     # every sampling run starts from the same noise
            if not flux3:                           # the run's modulation vectors, one weight pass per 4 steps
                model.prepare_timesteps(ts[:-1])
        F.flux_pack_latents(lat_buf, tok)
        forward_update(k)
        F.flux_unpack_latents(tok, lat_buf)

    for i in range(args.warmup):
        step(i, lat)
    torch.cuda.synchronize()
    assert F.flux_device_error() == 0

    # ---- every step of one sampling run captured as a CUDA graph (the same launches, replayed
    # without per-launch host work, so host jitter does not enter the device-timed region)
    graphs, launch_mode = [], "plain launches"
    if not args.no_graph:
        try:
            for k in range(w.n_steps):
                g = torch.cuda.CUDAGraph()
                c0 = F.flux_kernel_launches()
                with torch.cuda.graph(g):
                    step(k, lat)
                graphs.append((g, F.flux_kernel_launches() - c0))
            for g, _ in graphs:                     # one full sampling run from the graphs
                g.replay()
            torch.cuda.synchronize()
            assert F.flux_device_error() == 0
            launch_mode = "one CUDA graph per sampling step, replayed"
        except Exception as ex:                    # capture refused: time plain launches
            torch.cuda.synchronize()
            graphs, launch_mode = [], f"plain launches (graph capture failed: {type(ex).__name__})"

    def timed_step(i):
        if graphs:
            graphs[i % w.n_steps][0].replay()
            return graphs[i % w.n_steps][1]
        c0 = F.flux_kernel_launches()
        step(i, lat)
        return F.flux_kernel_launches() - c0

    # ---- timed region: K steps, device time, max over ranks
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    launches = 0
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    ev0.record(stream)
    for i in range(args.steps):
        launches += timed_step(i)
    ev1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    ms_total = ev0.elapsed_time(ev1)
    graphs = []                                     # released before the model
    clk = clocks.stop()
    ms_total = max_over_ranks(ms_total, world)
    ms_step = ms_total / args.steps
    value = aggregate_ms_per_forward(ms_total, args.steps, world)

    # ---- per-kernel device time (CUDA events around every launch of the forward)
    model.profile(True)
    for i in range(args.steps):
        step(i, lat)
    prof = model.profile_read()
    model.profile(False)
    assert F.flux_device_error() == 0

    # ---- end to end through host buffers (pinned), H2D inputs and D2H latent every step
    lat_pin = torch.from_numpy(lat_h).pin_memory()
    txt_pin = torch.from_numpy(txt_h).pin_memory()
    txt_u_pin = torch.from_numpy(txt_u_h).pin_memory() if guided else None
    out_pin = torch.empty_like(lat_pin).pin_memory()
    lat_d = torch.empty_like(lat0)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    e0.record(stream)
    for i in range(args.steps):
        k = i % w.n_steps
        if k == 0 and not flux3:
            model.prepare_timesteps(ts[:-1])
        lat_d.copy_(lat_pin if k == 0 else out_pin, non_blocking=True)
        txt.copy_(txt_pin, non_blocking=True)
        if guided:
            txt_u.copy_(txt_u_pin, non_blocking=True)
        F.flux_pack_latents(lat_d, tok)
        forward_update(k)
        F.flux_unpack_latents(tok, lat_d)
        out_pin.copy_(lat_d, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = aggregate_ms_per_forward(max_over_ranks(e0.elapsed_time(e1), world), args.steps, world)
    assert torch.isfinite(out_pin).all()
    h2d = lat_pin.numel() * 4 + txt_pin.numel() * 4 * n_sequences(w)
    d2h = out_pin.numel() * 4

    peaks, peak_src = load_peaks()
    flops = step_flops(w)
    tflops = flops / (ms_step / 1e3) / 1e12
    g_ms, g_fl, g_by, g_n = prof["gemm"]
    a_ms, a_fl, a_by, a_n = prof["attention"]
    attn_tflops = a_fl / (a_ms / 1e3) / 1e12
    kinds = {k: kernel_kind_line(k, v_, args.steps, peaks) for k, v_ in prof.items() if v_[3]}

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 4), "unit": step_unit(w), "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
            "higher_is_better": False, "scaling": "weak", "vs_baseline": None,
            "dtype": ("nvfp4 (e2m1, e4m3 per 16, fp32 per row) block linears, bf16 attention" if fp4 else
                      "fp8-e4m3 row-wise block linears, bf16 attention" if fp8 else "bf16"),
            "data": "synthetic (seeded N(0,1) weights scaled 1/sqrt(fan_in), bf16; N(0,1) latent and text)",
            "config": {"workload": f"{w.name}: {w.image}x{w.image}, {w.n_img} image + {w.n_txt} text + {w.n_ref} "
                                   f"reference tokens ({len(w.ref_grids)} reference images), {blocks_text(w)}, "
                                   f"width 3072, 24x128 heads, one Euler step (pack, forward, Euler, unpack)"
                                   + ("" if not guided else f"; guidance {w.guidance}: prompt and unconditional "
                                      f"text as one batch-2 forward, fused guided Euler update"),
                       "global_batch": world, "seq_len": w.n_tokens,
                       "parallelism": f"replicas x{world}, no data-path collective",
                       "l2": f"inputs larger than L2: {weight_gb(w):.1f} GB of bf16 weights streamed every forward"},
            "tflops": round(tflops, 1),
            "frac_bf16_peak": {"measured_burst": round(tflops / peaks["bf16_tflops"], 4),
                               "measured_sustained": round(tflops / peaks["bf16_tflops_sustained"], 4),
                               "spec_2250": round(tflops / SPEC_BF16_TFLOPS, 4), "peaks": peak_src},
            "forwards_per_s": round(1e3 / value, 3),
            "roofline": {"kernel": ("gemm_fp4_tc2 (CTA-pair tcgen05 kind::mxf4nvf4 with block scales) for the block "
                                    "linears, bf16 for the input / output projections" if fp4 else
                                    "gemm_bf16_tc2<fp8> (CTA-pair tcgen05 kind::f8f6f4) for the block linears, "
                                    "bf16 for the input / output projections" if fp8 else
                                    "gemm_bf16_tc2 (CTA-pair tcgen05 GEMM) + the 128-wide output GEMM, all linear layers"),
                         **gemm_roofline(g_ms, g_fl, g_by, peaks, peak_src, fp4=fp4, fp8=fp8),
                         "traffic": None,
                         "traffic_note": ("DRAM bytes need a profiler's counters, which this timed run does "
                                          "not take; the ncu capture of the same kernel is kept beside the "
                                          "sources as a cross-check"),
                         "launches_per_forward": round(g_n / args.steps, 3),
                         "share_of_step": round(g_ms / args.steps / ms_step, 3)},
            "attention": {"achieved": round(attn_tflops, 1), "unit": "TFLOP/s",
                          "peak": round(peaks["bf16_tflops_sustained"], 1),
                          "frac": round(attn_tflops / peaks["bf16_tflops_sustained"], 4),
                          "frac_of": fractions(attn_tflops, peaks),
                          "launches_per_forward": round(a_n / args.steps, 3),
                          "share_of_step": round(a_ms / args.steps / ms_step, 3)},
            "kernels": kinds,
            "e2e": {"value": round(e2e_ms, 4), "unit": step_unit(w), "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": launches,
            "launch": launch_mode,
            "clocks": clk,
        }
        if world == 1 and not args.no_cpu_baseline:
            ms_cpu, secs = cpu_oracle_sample(w, params, lat_h, txt_h, ref_h)
            line["cpu_baseline"] = {"value": round(ms_cpu * n_sequences(w), 1), "unit": step_unit(w),
                                    "cores": torch.get_num_threads(), "kind": "oracle",
                                    "sample": (f"one joint block at full {w.name} size, fp32 oracle ({secs:.1f} s), "
                                               f"scaled by forward FLOPs / block FLOPs" if flux3 else
                                               f"the {w.name} forward on its own latent and text, cut to its first "
                                               f"{CPU_SAMPLE_BLOCKS} double + {CPU_SAMPLE_BLOCKS} single blocks, fp32 "
                                               f"oracle ({secs:.1f} s), scaled by algorithmic FLOPs to the "
                                               f"{n_blocks(w)}-block forward")
                                              + ("" if not guided else ", x2 for the two guided sequences")}
        print(json.dumps(line), flush=True)
    model.close()
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=4)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default="t2i1024", choices=sorted(WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true",
                    help="time plain per-step launches instead of replaying each step's captured CUDA graph")
    ap.add_argument("--precision", choices=("bf16", "fp8", "nvfp4"), default="bf16",
                    help="block linears in bf16, row-wise FP8 (e4m3 codes with per-row scales) or NVFP4 "
                         "(e2m1 codes, e4m3 scales per 16 elements, fp32 per row)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    w = WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)
    return run_ours(args, w)


if __name__ == "__main__":
    sys.exit(main())
