#!/usr/bin/env python
"""Benchmark of the selective-scan (S6) forward pass on B200.

One step = one forward scan (ssm_scan_fwd through the C ABI) over one batch of the workload
the metric is quoted on: the Mamba-370m-shaped layer, batch 8 x dim 2048 x L 2048, N 16, bf16
io, f32 state.  Inputs are seeded synthetic tensors resident in HBM when timing starts
(270 MB of compulsory traffic per step, more than the 126 MB L2, so no flush is needed
between steps).  Prints ONE JSON line on rank 0.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

--impl reference times the fp64 CPU oracle on a bounded sample of the same workload on this
machine's host cores (the reference arm; there is no upstream implementation to install).
Multi-GPU (torchrun, one process per GPU): every rank scans its own batch (weak scaling; the
path has no exchange step, so no collective touches the data); time is the max over ranks.
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from selective_state_space_23_b200.inputs import make_inputs, workload  # noqa: E402

METRIC = "selective-scan fwd tokens/s and achieved HBM GB/s (% of B200 peak) at 1 GPU"
UNIT = "tokens/s"
WORKLOAD = "mamba370m_fwd"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "sm_max_mhz": 1965.0, "source": "fallback"}

# Unit counts of a B200 SM used for the ALU roofline (per clock): 128 FP32 FMA lanes, 16 MUFU
# (ex2) lanes.  One (channel, step, state) element needs 4 FP32 ops (Δ*A, Δ*x*B, state FMA,
# C readout) plus one 2^x, which costs 1 MUFU op or 7 FP32 ops on the FMA pipe (range
# reduction 3 + polynomial 4).  With a fraction f of the exponentials on MUFU the two pipes
# balance at (4 + 7(1-f))/128 = f/16, i.e. f = 11/15, giving 16*15/11 = 21.8 elements/clk/SM.
FP32_PER_CLK, MUFU_PER_CLK, BASE_FP32, EXP_FP32 = 128, 16, 4, 7


def alu_peak_elems_per_s(sms: int, mhz: float) -> float:
    f = (BASE_FP32 + EXP_FP32) / (EXP_FP32 + FP32_PER_CLK / MUFU_PER_CLK)
    per_clk = MUFU_PER_CLK / f
    return sms * mhz * 1e6 * per_clk


def compulsory_bytes(w) -> int:
    es = 2 if w.io_dtype == torch.bfloat16 else 4
    x = w.batch * w.dim * w.seqlen * es
    bc = w.batch * w.dstate * w.seqlen * es
    return 4 * x + 2 * bc + w.dim * w.dstate * 4 + 2 * w.dim * 4


def compulsory_bytes_shape(b, d, L, N, es=2) -> int:
    """u, delta, z, out + B, C + per-channel parameters (A taken as [dim])."""
    return 4 * b * d * L * es + 2 * b * N * L * es + 3 * d * 4


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            d = json.load(fh)
        return {"hbm_gbs": float(d["hbm_gbs"]), "sm_max_mhz": float(d.get("sm_max_mhz", 1965.0)),
                "source": "measured"}
    return dict(FALLBACK_PEAKS)


# Sources of the kernel that runs the benchmark step (the general two-lanes forward kernel)
KERNEL_SOURCES = ("ssm_fwd_impl.cuh", "ssm_fwd_bf16.cu", "ssm_device.cuh", "ssm_kernels.h", "ssm_rows.cuh")


def kernel_source_hash() -> str:
    """Hash of the forward kernel's code: its sources, and of the shared header only the argument
    struct the kernel reads (comments dropped), so that unrelated declarations do not count."""
    import re
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "selective_state_space_23_b200", "csrc", f), "r") as fh:
            text = fh.read()
        if f == "ssm_kernels.h":
            m = re.search(r"struct FwdArgs \{.*?\n\};", text, re.S)
            text = re.sub(r"//[^\n]*", "", m.group(0)) if m else text
        h.update(text.encode())
    return h.hexdigest()[:16]


def recorded_traffic():
    """DRAM bytes per launch of the forward kernel from the committed ncu summary, or None when
    the kernel source changed since that capture."""
    p = os.path.join(ROOT, "profiles", "fwd_kernel_mamba370m_traffic.txt")
    if not os.path.exists(p):
        return None
    kv = {}
    with open(p) as fh:
        for line in fh:
            if "=" in line and not line.startswith("#"):
                k, v = line.split("=", 1)
                kv[k.strip()] = v.strip()
    if kv.get("kernel_source_hash") != kernel_source_hash():
        return None
    try:
        return int(kv["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled while the timed region runs."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]
        return False

    def summary(self):
        sm, mx, reasons, power = [], None, set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in self.lines:
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
                power.append(float(f[3]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        busy = [s for s in sm if mx and s > 0.5 * mx] or sm
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "power_w_max": max(power) if power else None}


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def max_over_ranks(value: float, world: int, device) -> float:
    from selective_state_space_23_b200.dist import max_over_ranks as _max
    return _max(value, device) if world > 1 else value


def barrier(world: int):
    from selective_state_space_23_b200.dist import barrier as _barrier
    if world > 1:
        _barrier()


# ------------------------------------------------------------------ CPU oracle baseline
# Both arms time the same thing: the fp64 oracle, as it stands, on the first REF_CHANNELS
# channels of every batch row of the workload (full L and N), with the oracle's default thread
# count; the full-width throughput is that sample's measured time scaled by dim / REF_CHANNELS.
REF_CHANNELS = int(os.environ.get("SSM_REF_CHANNELS", "512"))


def oracle_sample(w, seed: int = 0, nd: int = REF_CHANNELS, nthreads: int = 0):
    """A callable running the oracle forward on nd channels (all batch rows) of the workload."""
    import oracle
    x = make_inputs(w, seed=seed)
    f = {k: v.to(torch.float64).numpy() for k, v in x.items()}
    sel = np.arange(min(nd, w.dim))
    sub = dict(u=np.ascontiguousarray(f["u"][:, sel]), delta=np.ascontiguousarray(f["delta"][:, sel]),
               A=f["A"][sel], B=f["B"], C=f["C"], D=f["D"][sel],
               z=np.ascontiguousarray(f["z"][:, sel]), dt_bias=f["dt_bias"][sel])
    run = lambda: oracle.scan_fwd(sub["u"], sub["delta"], sub["A"], sub["B"], sub["C"], D=sub["D"],
                                  z=sub["z"], dt_bias=sub["dt_bias"], nthreads=nthreads)
    return run, len(sel)


def oracle_timing(w, warmup: int, steps: int, nthreads: int = 0):
    """Measured seconds per sample run (mean over `steps` after `warmup`), the sample's channel
    count, the threads used and the full-width tokens/s extrapolated by channel count."""
    import oracle
    run, nd = oracle_sample(w, nthreads=nthreads)
    for _ in range(warmup):
        run()
    t0 = time.perf_counter()
    for _ in range(steps):
        run()
    per_run = (time.perf_counter() - t0) / steps
    cores = nthreads if nthreads > 0 else oracle.max_threads()
    return per_run, nd, cores, w.tokens / (per_run * w.dim / nd)


def sample_desc(w, nd, per_run, steps):
    return (f"oracle fp64 on {w.batch}x{nd} of {w.batch}x{w.dim} channels (L {w.seqlen}, N "
            f"{w.dstate}): measured {per_run * 1e3:.1f} ms per run (mean of {steps}); tokens/s "
            f"= {w.batch}x{w.seqlen} tokens / (that time x {w.dim}/{nd})")


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as fh:
            for ln in fh:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def run_reference(args, rank, world):
    if rank != 0:
        return 0
    w = workload(WORKLOAD)
    # W untimed warm-up runs, then K timed runs of the bounded channel sample
    per_run, nd, cores, value = oracle_timing(w, args.warmup, args.steps)
    sample = sample_desc(w, nd, per_run, args.steps)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_run * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded)",
        "config": {"workload": f"{WORKLOAD}: batch 8 x dim 2048 x L 2048, N 16, bf16 io rounded then f64",
                   "global_batch": w.batch, "seq_len": w.seqlen, "parallelism": "host cores",
                   "step": f"one oracle run over {w.batch}x{nd} of the {w.batch}x{w.dim} channels "
                           "(ms_per_step is its measured time; value is extrapolated to the full "
                           "width by channel count)"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ our arm
EXTRAS = ("train", "scalar_decay", "variants", "long_seq", "decode", "ssd")


def bench_extras(dev, which=EXTRAS):
    """Timing of the other hot-path calls on their workloads (inputs drawn on the GPU); `which`
    selects the measurements."""
    import selective_state_space_23_b200 as ssm
    g = torch.Generator(device=dev).manual_seed(1)
    out = {}

    def rnd(shape, std=1.0):
        return (torch.randn(shape, device=dev, generator=g) * std).to(torch.bfloat16)

    def prm(dim, N, lo, hi):
        dt = torch.exp(torch.rand(dim, device=dev, generator=g) * (np.log(hi) - np.log(lo)) + np.log(lo))
        bias = dt + torch.log(-torch.expm1(-dt))
        A = -torch.arange(1, N + 1, device=dev, dtype=torch.float32).repeat(dim, 1)
        return A.contiguous(), torch.randn(dim, device=dev, generator=g), bias.float()

    def timeit(fn, reps):
        for _ in range(2):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps

    N = 16
    # training step (forward with checkpoints + backward) on the Mamba-2.8B-shaped layer
    if "train" in which:
        out.update(_train_step(dev, rnd, prm, timeit))
    if "scalar_decay" in which or "variants" in which:
        out.update(_variants(dev, rnd, prm, timeit, g, which))
    if "long_seq" in which:
        out.update(_long_seq(dev, rnd, prm, timeit))
    if "decode" in which:
        out.update(_decode(dev, rnd, prm, timeit))
    if "ssd" in which:
        out.update(_ssd(dev, rnd, prm, timeit, g))
    return out


def _ssd(dev, rnd, prm, timeit, g):
    """Scalar decay with 16, 64 and 128 states on the Mamba-370m-shaped layer (the chunked matrix
    form on the tensor cores): forward at 64 and 128 states, backward at all three."""
    import selective_state_space_23_b200 as ssm
    out = {}
    b, d, L = 8, 2048, 2048
    u, de, z = rnd((b, d, L)), rnd((b, d, L), 0.5), rnd((b, d, L))
    _, D, bias = prm(d, 16, 1e-3, 1e-1)
    A1 = -(torch.rand(d, device=dev, generator=g) * 15.0 + 1.0)
    o = torch.empty_like(u)
    res = {"shape": "8x2048x2048 bf16, A [dim]"}
    for N in (64, 128):
        B, C = rnd((b, N, L)), rnd((b, N, L))
        ms = timeit(lambda: ssm.ssm_scan_fwd_scalar_a(u, de, A1, B, C, D=D, z=z, dt_bias=bias, out=o), 10)
        # the chunk products per 16 steps and 64 channels: C B^T, mask(G) X', C H, B^T X''
        flops = 2.0 * b * (L // 16) * (d // 64) * (16 * 16 * N + 16 * 16 * 64 + 16 * N * 64 + N * 16 * 64)
        res[f"N{N}"] = {"fwd_ms": ms, "tokens_per_s": b * L / (ms * 1e-3),
                        "hbm_gbs": (4 * b * d * L * 2 + 2 * b * N * L * 2) / (ms * 1e-3) / 1e9,
                        "mma_tflops": flops / (ms * 1e-3) / 1e12}
    # f32 io with 64 states: the sum of four 16-state f32 forwards over the state slices
    N = 64
    uf, df, zf = u.float(), de.float(), z.float()
    Bf, Cf = rnd((b, N, L)).float(), rnd((b, N, L)).float()
    of = torch.empty_like(uf)
    wsf = torch.empty(max(1, ssm._abi.lib().ssm_scan_fwd_ex_workspace_size(b, d, L, N, 1, 0, 1)),
                      dtype=torch.uint8, device=dev)
    ms = timeit(lambda: ssm.ssm_scan_fwd_scalar_a(uf, df, A1, Bf, Cf, D=D, z=zf, dt_bias=bias,
                                                  out=of, workspace=wsf), 5)
    res["N64_f32_slices"] = {"fwd_ms": ms, "tokens_per_s": b * L / (ms * 1e-3)}
    del uf, df, zf, Bf, Cf, of, wsf
    # the backward (chunked form: checkpoint pass, reverse walk, dB/dC finish) with 16, 64 and
    # 128 states; compulsory bytes: u, delta, z, dout in, du, ddelta, dz out, B, C in, dB, dC out
    dout = rnd((b, d, L))
    res["bwd"] = {}
    for N in (16, 64, 128):
        B, C = rnd((b, N, L)), rnd((b, N, L))
        wsb = torch.empty(ssm._abi.lib().ssm_scan_bwd_ex_workspace_size(b, d, L, N, 1, 1, 0, 1),
                          dtype=torch.uint8, device=dev)
        ms = timeit(lambda: ssm.ssm_scan_bwd_scalar_a(u, de, A1, B, C, dout, D=D, z=z,
                                                      dt_bias=bias, workspace=wsb), 5)
        byt = 7 * b * d * L * 2 + 4 * b * N * L * 2
        # a training step: the forward writing checkpoints, the backward taking them
        wsc = torch.empty(ssm._abi.lib().ssm_scan_bwd_ex_workspace_size(b, d, L, N, 1, 1, 1, 1),
                          dtype=torch.uint8, device=dev)

        def train():
            _, ck = ssm.ssm_scan_fwd_scalar_a(u, de, A1, B, C, D=D, z=z, dt_bias=bias, out=o,
                                              return_ckpt=True)
            ssm.ssm_scan_bwd_scalar_a(u, de, A1, B, C, dout, D=D, z=z, dt_bias=bias, ckpt=ck,
                                      workspace=wsc)
        mt = timeit(train, 5)
        res["bwd"][f"N{N}"] = {"bwd_ms": ms, "tokens_per_s": b * L / (ms * 1e-3),
                               "compulsory_gbs": byt / (ms * 1e-3) / 1e9,
                               "train_step_ms": mt}
        del B, C, wsb, wsc
    del u, de, z, o, dout
    # the long sequence (1 x 256 x 2^20) with 64 states: 16 warps of channels, so the time axis
    # is split into segments (summary, chain, output launches)
    b, d, L, N = 1, 256, 1 << 20, 64
    u, de, z = rnd((b, d, L)), rnd((b, d, L), 0.5), rnd((b, d, L))
    _, D, bias = prm(d, 16, 1e-4, 1e-2)
    A1 = -(torch.rand(d, device=dev, generator=g) * 15.0 + 1.0)
    B, C = rnd((b, N, L)), rnd((b, N, L))
    ws = torch.empty(max(1, ssm._abi.lib().ssm_scan_fwd_ex_workspace_size(b, d, L, N, 1, 1, 1)),
                     dtype=torch.uint8, device=dev)
    ms = timeit(lambda: ssm.ssm_scan_fwd_scalar_a(u, de, A1, B, C, D=D, z=z, dt_bias=bias,
                                                  workspace=ws), 5)
    del ws
    # its backward: the reverse walk split into segments (summary, adjoint chain, segments)
    dout = rnd((b, d, L))
    wsb = torch.empty(ssm._abi.lib().ssm_scan_bwd_ex_workspace_size(b, d, L, N, 1, 1, 0, 1),
                      dtype=torch.uint8, device=dev)
    msb = timeit(lambda: ssm.ssm_scan_bwd_scalar_a(u, de, A1, B, C, dout, D=D, z=z, dt_bias=bias,
                                                   workspace=wsb), 3)
    res["long_seq_N64"] = {"shape": "1x256x1048576 bf16, A [dim]", "fwd_ms": ms,
                           "tokens_per_s": b * L / (ms * 1e-3), "bwd_ms": msb}
    del u, de, z, B, C, dout, wsb
    torch.cuda.empty_cache()
    out["scalar_decay_large_n"] = res
    return out


def _train_step(dev, rnd, prm, timeit):
    import selective_state_space_23_b200 as ssm
    out = {}
    b, d, L, N = 4, 5120, 2048, 16
    u, de, z, dout = rnd((b, d, L)), rnd((b, d, L), 0.5), rnd((b, d, L)), rnd((b, d, L))
    B, C = rnd((b, N, L)), rnd((b, N, L))
    A, D, bias = prm(d, N, 1e-3, 1e-1)
    ws = torch.empty(ssm.bwd_workspace_bytes(b, d, L, N, torch.bfloat16, True), dtype=torch.uint8, device=dev)

    def train():
        _, ck = ssm.ssm_scan_fwd(u, de, A, B, C, D=D, z=z, dt_bias=bias, return_ckpt=True)
        ssm.ssm_scan_bwd(u, de, A, B, C, dout, D=D, z=z, dt_bias=bias, ckpt=ck, workspace=ws)

    def fwd_only():
        ssm.ssm_scan_fwd(u, de, A, B, C, D=D, z=z, dt_bias=bias)

    ms_tr = timeit(train, 5)
    ms_f = timeit(fwd_only, 10)
    out["mamba2p8b_train"] = {"shape": "4x5120x2048 N16 bf16", "fwd_ms": ms_f,
                              "fwd_bwd_ms": ms_tr, "tokens_per_s": b * L / (ms_tr * 1e-3)}
    del u, de, z, dout, ws
    torch.cuda.empty_cache()
    return out


def _variants(dev, rnd, prm, timeit, g, which):
    import selective_state_space_23_b200 as ssm
    out = {}
    N = 16
    # scalar decay (one rate per channel) on the Mamba-370m-shaped layer
    b, d, L = 8, 2048, 2048
    u, de, z = rnd((b, d, L)), rnd((b, d, L), 0.5), rnd((b, d, L))
    B, C = rnd((b, N, L)), rnd((b, N, L))
    _, D, bias = prm(d, N, 1e-3, 1e-1)
    A1 = -(torch.rand(d, device=dev, generator=g) * 15.0 + 1.0)
    o = torch.empty_like(u)
    if "scalar_decay" in which:
        ms = timeit(lambda: ssm.ssm_scan_fwd_scalar_a(u, de, A1, B, C, D=D, z=z, dt_bias=bias, out=o), 20)
        out["scalar_decay_fwd"] = {"shape": "8x2048x2048 N16 bf16, A [dim]", "fwd_ms": ms,
                                   "tokens_per_s": b * L / (ms * 1e-3),
                                   "hbm_gbs": compulsory_bytes_shape(b, d, L, N) / (ms * 1e-3) / 1e9}
        if "variants" not in which:
            return out

    # the other variants of the forward scan on the same layer
    A, D, bias = prm(d, N, 1e-3, 1e-1)
    Bg, Cg = rnd((b, 4, N, L)), rnd((b, 4, N, L))
    uc, dec, zc = (t.transpose(1, 2).contiguous() for t in (u, de, z))
    Bc, Cc = B.transpose(1, 2).contiguous(), C.transpose(1, 2).contiguous()
    oc = torch.empty_like(uc)
    def lane_kernel():  # the default variant in the one-lane-per-channel kernel
        os.environ["SSM_FWD_KERNEL"] = "lane"
        try:
            ssm.ssm_scan_fwd(u, de, A, B, C, D=D, z=z, dt_bias=bias, out=o)
        finally:
            del os.environ["SSM_FWD_KERNEL"]

    var = {
        "default": lambda: ssm.ssm_scan_fwd(u, de, A, B, C, D=D, z=z, dt_bias=bias, out=o),
        "default_lane_kernel": lane_kernel,
        "zoh": lambda: ssm.ssm_scan_fwd(u, de, A, B, C, D=D, z=z, dt_bias=bias, out=o, zoh=True),
        "reverse": lambda: ssm.ssm_scan_fwd(u, de, A, B, C, D=D, z=z, dt_bias=bias, out=o,
                                            reverse=True),
        "groups4": lambda: ssm.ssm_scan_fwd(u, de, A, Bg, Cg, D=D, z=z, dt_bias=bias, out=o),
        "channels_last": lambda: ssm.ssm_scan_fwd(uc, dec, A, Bc, Cc, D=D, z=zc, dt_bias=bias,
                                                  out=oc, channels_last=True),
    }
    out["variants_fwd_ms"] = {"shape": "8x2048x2048 N16 bf16",
                              **{k: timeit(f, 20) for k, f in var.items()}}
    del u, de, z, B, C, o, Bg, Cg, uc, dec, zc, Bc, Cc, oc
    torch.cuda.empty_cache()
    return out


def _long_seq(dev, rnd, prm, timeit):
    import selective_state_space_23_b200 as ssm
    out = {}
    N = 16
    # long sequence
    b, d, L = 1, 256, 1 << 20
    u, de, z = rnd((b, d, L)), rnd((b, d, L), 0.5), rnd((b, d, L))
    B, C = rnd((b, N, L)), rnd((b, N, L))
    A, D, bias = prm(d, N, 1e-4, 1e-2)
    ws = torch.empty(max(1, ssm.fwd_workspace_bytes(b, d, L, N, torch.bfloat16)), dtype=torch.uint8, device=dev)
    ms = timeit(lambda: ssm.ssm_scan_fwd(u, de, A, B, C, D=D, z=z, dt_bias=bias, workspace=ws), 5)
    byt = 4 * b * d * L * 2 + 2 * b * N * L * 2
    out["long_seq_1m"] = {"shape": "1x256x1048576 N16 bf16", "fwd_ms": ms,
                          "tokens_per_s": b * L / (ms * 1e-3), "hbm_gbs": byt / (ms * 1e-3) / 1e9}
    # backward of the same sequence (time-split history backward) from the forward's checkpoints
    _, ck = ssm.ssm_scan_fwd(u, de, A, B, C, D=D, z=z, dt_bias=bias, return_ckpt=True, workspace=ws)
    dout = rnd((b, d, L))
    wsb = torch.empty(ssm.bwd_workspace_bytes(b, d, L, N, torch.bfloat16, True), dtype=torch.uint8,
                      device=dev)
    ms_b = timeit(lambda: ssm.ssm_scan_bwd(u, de, A, B, C, dout, D=D, z=z, dt_bias=bias, ckpt=ck,
                                           workspace=wsb), 5)
    out["long_seq_1m"]["bwd_ms"] = ms_b
    del u, de, z, B, C, ws, ck, dout, wsb
    torch.cuda.empty_cache()
    return out


def _decode(dev, rnd, prm, timeit):
    import selective_state_space_23_b200 as ssm
    out = {}
    N = 16
    # decode: 256 x 5120 x 16 state.  The 84 MB state fits in L2 (126 MB).  Side figures: L2
    # flushed before every step by READING 256 MB (the flush is timed separately and
    # subtracted; the previous step's dirty state is written back during the flush and so
    # counted), and the state left in L2.  Main figure: below, one state per layer
    b, d = 256, 5120
    state = torch.zeros((b, d, N), device=dev)
    x, dtr, zz = rnd((b, d)), rnd((b, d), 0.5), rnd((b, d))
    Bd, Cd = rnd((b, N)), rnd((b, N))
    A, D, bias = prm(d, N, 1e-3, 1e-1)
    flush = torch.ones(64 << 20, dtype=torch.float32, device=dev)
    sink = torch.empty((), device=dev)
    read_flush = lambda: torch.sum(flush, dim=0, out=sink)
    t_flush = timeit(read_flush, 20)
    t_all = timeit(lambda: (read_flush(), ssm.ssm_state_update(state, x, dtr, A, Bd, Cd, D=D, z=zz,
                                                                dt_bias=bias)), 50)
    us = (t_all - t_flush) * 1e3
    t_hot = timeit(lambda: ssm.ssm_state_update(state, x, dtr, A, Bd, Cd, D=D, z=zz,
                                                dt_bias=bias), 50) * 1e3
    byt = 2 * b * d * N * 4 + 4 * b * d * 2 + 2 * b * N * 2
    del flush
    # the steps of a model with several layers: each step updates another layer's state (4 of
    # them, 336 MB, more than twice L2), so no step finds its state in L2 and every step's
    # written state leaves L2 during later steps, as in a decode over many layers
    states = [state] + [torch.zeros((b, d, N), device=dev) for _ in range(3)]
    cyc = [0]

    def layer_step():
        st = states[cyc[0] % len(states)]
        cyc[0] += 1
        ssm.ssm_state_update(st, x, dtr, A, Bd, Cd, D=D, z=zz, dt_bias=bias)
    t_rot = timeit(layer_step, 48) * 1e3
    out["decode_b256"] = {"shape": "256x5120x16 f32 state, bf16 io",
                          "us_per_step": t_rot, "hbm_gbs": byt / (t_rot * 1e-6) / 1e9,
                          "l2": "each step updates another of 4 layer states (336 MB)",
                          "us_per_step_after_read_flush": us,
                          "us_per_step_state_in_l2": t_hot}
    del state, states
    # one rate per channel with 64 and 128 states (a Mamba-2 layer's decode): the state (335 and
    # 671 MB) is larger than L2, so no flush is needed
    A1 = -(torch.rand(d, device=dev) * 15.0 + 1.0)
    for N2 in (64, 128):
        st2 = torch.zeros((b, d, N2), device=dev)
        B2, C2 = rnd((b, N2)), rnd((b, N2))
        t2 = timeit(lambda: ssm.ssm_state_update(st2, x, dtr, A1, B2, C2, D=D, z=zz, dt_bias=bias,
                                                 scalar_a=True), 50) * 1e3
        byt2 = 2 * b * d * N2 * 4 + 4 * b * d * 2 + 2 * b * N2 * 2
        out[f"decode_b256_scalar_n{N2}"] = {"shape": f"256x5120x{N2} f32 state, bf16 io, A [dim]",
                                            "us_per_step": t2, "hbm_gbs": byt2 / (t2 * 1e-6) / 1e9}
        del st2
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-extras", action="store_true")
    ap.add_argument("--extras", default=",".join(EXTRAS),
                    help="comma-separated side measurements to run: " + ",".join(EXTRAS))
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--no-baseline", action="store_true", help="skip the CPU oracle timing")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    rank, world, local = dist_env()

    if args.impl == "reference":
        return run_reference(args, rank, world)

    import selective_state_space_23_b200 as ssm
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA GPU (the library has no CPU path)")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    ssm.library_path()

    w = workload(WORKLOAD)
    x = make_inputs(w, seed=rank)  # each rank scans its own batch
    xd = {k: v.to(dev) for k, v in x.items()}
    out = torch.empty_like(xd["u"])
    nws = ssm.fwd_workspace_bytes(w.batch, w.dim, w.seqlen, w.dstate, w.io_dtype)
    ws = torch.empty(nws, dtype=torch.uint8, device=dev) if nws else None
    launches_per_step = 3 if nws else 1  # time split: summary, carry, output passes

    def step():
        ssm.ssm_scan_fwd(xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"], D=xd["D"], z=xd["z"],
                         dt_bias=xd["dt_bias"], out=out, workspace=ws)

    K, W = args.steps, args.warmup
    for _ in range(W):
        step()
    torch.cuda.synchronize()
    barrier(world)
    ev_s = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ev_e = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        torch.cuda.synchronize()
        barrier(world)
        e0.record()
        for i in range(K):
            ev_s[i].record()
            step()
            ev_e[i].record()
        e1.record()
        torch.cuda.synchronize()
        barrier(world)
    total_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    kern_ms = statistics.fmean(ev_s[i].elapsed_time(ev_e[i]) for i in range(K))
    kern_ms = max_over_ranks(kern_ms, world, dev)
    ms_step = total_ms / K
    value = world * w.tokens / (ms_step * 1e-3)

    # end to end through the public host-memory call (ssm_scan_fwd_host): every step copies the
    # inputs from pinned host memory, scans and copies the output back, pipelined over batch rows
    hx = {k: v.pin_memory() for k, v in x.items()}
    hout = torch.empty_like(x["u"]).pin_memory()
    names_in = ("u", "delta", "z", "B", "C")
    h2d = sum(hx[k].numel() * hx[k].element_size() for k in names_in)
    d2h = hout.numel() * hout.element_size()
    hws = torch.empty(max(1, ssm.fwd_host_workspace_bytes(w.batch, w.dim, w.seqlen, w.dstate,
                                                          w.io_dtype)), dtype=torch.uint8,
                      device=dev)

    def e2e_step():
        ssm.ssm_scan_fwd_host(hx["u"], hx["delta"], xd["A"], hx["B"], hx["C"], D=xd["D"],
                              z=hx["z"], dt_bias=xd["dt_bias"], out=hout, workspace=hws)

    e2e_ms = e2e_value = None
    if args.e2e_steps > 0:
        for _ in range(3):
            e2e_step()
        torch.cuda.synchronize()
        barrier(world)
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record()
        for _ in range(args.e2e_steps):
            e2e_step()
        f1.record()
        torch.cuda.synchronize()
        barrier(world)
        e2e_ms = max_over_ranks(f0.elapsed_time(f1), world, dev) / args.e2e_steps
        e2e_value = world * w.tokens / (e2e_ms * 1e-3)

    if rank != 0:
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
            dist.destroy_process_group()
        return 0

    peaks = load_peaks()
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    byts = compulsory_bytes(w)
    elems = w.batch * w.dim * w.seqlen * w.dstate
    hbm_gbs = byts / (kern_ms * 1e-3) / 1e9
    alu_peak = alu_peak_elems_per_s(sms, peaks["sm_max_mhz"])
    alu_ach = elems / (kern_ms * 1e-3)
    traffic = recorded_traffic()
    if args.no_baseline or world > 1:
        cb_value = cb_cores = None
        cb_desc = "skipped (--no-baseline)" if args.no_baseline else "timed at N=1 only"
        sc_value, sc_desc = None, cb_desc
    else:
        reps = 5
        per_run, nd, cb_cores, cb_value = oracle_timing(w, 1, reps)
        cb_desc = sample_desc(w, nd, per_run, reps)
        per1, nd1, _, sc_value = oracle_timing(w, 0, 1, nthreads=1)
        sc_desc = sample_desc(w, nd1, per1, 1) + " (1 thread)"
    extras = {} if world == 1 else {"skipped": "the side measurements run at N=1 only"}
    if not args.no_extras and world == 1:
        try:  # side measurements: a failure here is reported, it does not cost the main line
            extras = bench_extras(dev, tuple(x for x in args.extras.split(",") if x))
        except Exception as e:  # noqa: BLE001
            extras = {"error": f"{type(e).__name__}: {e}"[:300]}
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16 io / f32 state", "data": "synthetic (seeded)",
        "config": {"workload": "mamba370m_fwd: batch 8 x dim 2048 x L 2048, N 16 (Mamba-370m layer shape)",
                   "global_batch": w.batch * world, "seq_len": w.seqlen, "dstate": w.dstate,
                   "parallelism": f"dp{world} (independent batches, no collective)",
                   "l2": "inputs (270 MB/step) larger than L2 (126 MB); no flush",
                   "hbm_gbs": hbm_gbs, "hbm_frac_of_measured": hbm_gbs / peaks["hbm_gbs"]},
        "roofline": {"bound": "alu", "achieved": alu_ach / 1e9, "peak": alu_peak / 1e9,
                     "unit": "Gelem/s", "frac": alu_ach / alu_peak, "traffic": traffic,
                     "element": "one (channel, step, state) update: 4 fp32 ops + one 2^x",
                     "peak_basis": f"{sms} SMs x {peaks['sm_max_mhz']:.0f} MHz x 21.8 elem/clk/SM "
                                   "(128 FMA + 16 MUFU lanes, best exp split)",
                     "hbm": {"achieved": hbm_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                             "frac": hbm_gbs / peaks["hbm_gbs"], "peak_source": peaks["source"],
                             "bytes_per_launch": byts},
                     "kernel_ms": kern_ms},
        "cpu_baseline": {"value": cb_value, "unit": UNIT, "cores": cb_cores, "kind": "oracle",
                         "sample": cb_desc, "cpu_model": cpu_model(),
                         "same_as": "the --impl reference arm (same sample, threads and oracle)",
                         "single_core": {"value": sc_value, "unit": UNIT, "sample": sc_desc}},
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e2e_ms},
        "gpu_launches": K * launches_per_step,
        "clocks": clk.summary(),
        "extras": extras,
    }
    print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
