"""Edge cases of the step size Δ, CUDA library against the fp64 oracle: forward, backward and
decode with the softplus argument v = delta + dt_bias spread over [-30, 30].

That range drives every branch of the kernels' softplus -- the series for e^v < 1/32, the
log2(1 + e^v) form, and v itself above 15 -- and the backward's softplus' = sigmoid(v) near 0 and
near 1.  It also drives the two limits the "Sorular" section of the Mamba summary page describes:
a large Δ (Δ|A| >> 1, so exp(ΔA) -> 0) resets the state to the current input term Δ B_t x_t,
and Δ -> 0 keeps the state and ignores the input.  Without softplus, Δ = delta + dt_bias may be
negative ("Seçim Mekanizması (S6)" defines Δ through softplus; the flag-off form is the plain
sum), which the last cases cover.
"""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_23_b200 as ssm
from selective_state_space_23_b200.inputs import make_inputs, workload

from _parity import assert_bf16_elementwise, assert_close, bf16_ulp, f64

DEV = "cuda"
GRADS = ("du", "ddelta", "dz", "dB", "dC", "dA", "dD", "ddt_bias", "dh0")


def on_dev(x):
    return {k: v.to(DEV) for k, v in x.items()}


def spread_delta(x, io, lo=-30.0, hi=30.0, seed=0, key="delta"):
    """Raw steps uniform on [lo, hi] with a zero bias, so v = delta covers the whole range."""
    shape = x[key].shape
    v = np.random.default_rng(seed).uniform(lo, hi, size=shape).astype(np.float32)
    x[key] = torch.from_numpy(v).to(io)
    x["dt_bias"] = torch.zeros_like(x["dt_bias"])
    return x


def fwd_gpu(x, softplus=True, **kw):
    return ssm.ssm_scan_fwd(x["u"], x["delta"], x["A"], x["B"], x["C"], D=x.get("D"),
                            z=x.get("z"), dt_bias=x.get("dt_bias"), delta_softplus=softplus,
                            h0=x.get("h0"), **kw)


def fwd_oracle(x, softplus=True):
    c = lambda k: None if x.get(k) is None else f64(x[k])
    return oracle.scan_fwd(c("u"), c("delta"), c("A"), c("B"), c("C"), D=c("D"), z=c("z"),
                           dt_bias=c("dt_bias"), delta_softplus=softplus, h0=c("h0"))


def bwd_gpu(x, softplus=True, use_ckpt=False):
    ck = None
    if use_ckpt:
        _, ck = fwd_gpu(x, softplus, return_ckpt=True)
    return ssm.ssm_scan_bwd(x["u"], x["delta"], x["A"], x["B"], x["C"], x["dout"], D=x.get("D"),
                            z=x.get("z"), dt_bias=x.get("dt_bias"), delta_softplus=softplus,
                            h0=x.get("h0"), ckpt=ck)


def bwd_oracle(x, softplus=True):
    c = lambda k: None if x.get(k) is None else f64(x[k])
    return oracle.scan_bwd(c("u"), c("delta"), c("A"), c("B"), c("C"), c("dout"), D=c("D"),
                           z=c("z"), dt_bias=c("dt_bias"), delta_softplus=softplus, h0=c("h0"))


def check_fwd(x, io, softplus=True, elementwise=True):
    out, hL = fwd_gpu(on_dev(x), softplus, return_final_state=True)
    ref = fwd_oracle(x, softplus)
    assert_close(out, ref["out"], io, "out")
    assert_close(hL, ref["hL"], io, "hL")
    if io == torch.bfloat16 and elementwise:
        assert_bf16_elementwise(out, ref["out"], "out")
    return out, hL, ref


# Summed gradients (dA, dD, ddt_bias) add hundreds of per-step terms in f32.  With steps up to
# Δ = 30 the terms span many decades and partly cancel, and f32 summation error grows with the
# sum's condition number (sum of |terms| over |sum|), not with the f32 unit roundoff alone; for
# these adversarial ranges the f32 bound on them is 5e-5 instead of 1e-5.  Per-element outputs
# keep the 1e-5 bound.
SUMMED = ("dA", "dD", "ddt_bias")


def check_bwd(x, io, softplus=True, use_ckpt=False, summed_scale=1.0):
    g = bwd_gpu(on_dev(x), softplus, use_ckpt)
    r = bwd_oracle(x, softplus)
    for k in GRADS:
        if r.get(k) is not None and g.get(k) is not None:
            scale = summed_scale if (k in SUMMED and io == torch.float32) else 1.0
            assert_close(g[k], r[k], io, k, scale=scale)


# ------------------------------------------------------------------ helper (CPU)
def test_bf16_ulp_helper():
    assert bf16_ulp(1.0) == 2.0 ** -7 and bf16_ulp(1.99) == 2.0 ** -7
    assert bf16_ulp(0.75) == 2.0 ** -8 and bf16_ulp(-3.0) == 2.0 ** -6
    x = np.random.default_rng(0).standard_normal(10000) * 50
    r = torch.from_numpy(x).to(torch.bfloat16).double().numpy()
    assert np.all(np.abs(r - x) <= 0.5 * bf16_ulp(x) * (1 + 1e-12))


# ------------------------------------------------------------------ forward
@pytest.mark.gpu
@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("shape", [(2, 96, 333, 16), (1, 40, 100, 5), (3, 64, 2048, 16)])
def test_fwd_softplus_over_the_whole_range(io, shape):
    batch, dim, L, N = shape
    w = workload("tiny_f32", batch=batch, dim=dim, seqlen=L, dstate=N, io_dtype=io)
    x = spread_delta(make_inputs(w, seed=41, with_h0=True), io, seed=1)
    check_fwd(x, io)


@pytest.mark.gpu
@pytest.mark.parametrize("kmufu", [8, 14, 16])
def test_fwd_softplus_range_with_polynomial_exponentials(monkeypatch, kmufu):
    """v up to 3 keeps |Δ A log2 e| below the FMA-pipe exponential's range limit in every
    block, so the polynomial runs on v's whole lower range (down to Δ ~ 1e-13)."""
    monkeypatch.setenv("SSM_FWD_KMUFU", str(kmufu))
    w = workload("mamba370m_fwd", batch=2, dim=192, seqlen=1000)
    x = spread_delta(make_inputs(w, seed=42, with_h0=True), torch.bfloat16, -30.0, 3.0, seed=2)
    check_fwd(x, torch.bfloat16)


@pytest.mark.gpu
@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
def test_fwd_large_step_resets_the_state(io):
    """v = 30 (Δ = 30, exp(ΔA) <= e^-30 with A <= -1) at every 7th step: the state restarts from
    Δ B_t x_t there.  After a reset at the last step, hL is that input term alone."""
    batch, dim, L, N = 2, 64, 301, 16
    w = workload("tiny_f32", batch=batch, dim=dim, seqlen=L, dstate=N, io_dtype=io)
    x = make_inputs(w, seed=43, with_h0=True)
    d = x["delta"].float()
    d[..., 3::7] = 30.0
    d[..., L - 1] = 30.0
    x["delta"] = d.to(io)
    x["dt_bias"] = torch.zeros_like(x["dt_bias"])
    _, hL, ref = check_fwd(x, io)
    # the closed form of the reset: h_{L-1} = Δ B_{L-1} x_{L-1}, Δ = softplus(30)
    dl = np.logaddexp(0.0, 30.0)
    want = dl * f64(x["B"])[:, None, :, L - 1] * f64(x["u"])[:, :, L - 1:L]
    np.testing.assert_allclose(ref["hL"], want, rtol=1e-9, atol=1e-9)  # Ā <= e^-30 is not 0
    np.testing.assert_allclose(f64(hL), want, rtol=2e-6 if io == torch.float32 else 1e-2,
                               atol=1e-5 if io == torch.float32 else 5e-2)


@pytest.mark.gpu
@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
def test_fwd_vanishing_step_keeps_the_state(io):
    """v = -30 everywhere (Δ = 9.4e-14): the state stays h0 and y_t = C_t h0 + D x_t."""
    batch, dim, L, N = 2, 48, 130, 16
    w = workload("tiny_f32", batch=batch, dim=dim, seqlen=L, dstate=N, io_dtype=io)
    x = make_inputs(w, seed=44, with_h0=True, gate=False)
    x["delta"] = torch.full_like(x["delta"], -30.0)
    x["dt_bias"] = torch.zeros_like(x["dt_bias"])
    out, hL, ref = check_fwd(x, io)
    want = np.einsum("bnt,bdn->bdt", f64(x["C"]), f64(x["h0"])) + \
        f64(x["D"])[None, :, None] * f64(x["u"])
    np.testing.assert_allclose(ref["out"], want, rtol=1e-9, atol=1e-9)
    np.testing.assert_allclose(f64(hL), f64(x["h0"]), rtol=1e-6, atol=1e-6)


@pytest.mark.gpu
@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
def test_fwd_signed_steps_without_softplus(io):
    """Without softplus Δ = delta + dt_bias may be negative (growth for A < 0) as well as
    positive; steps of both signs, a positive mean so the state stays bounded."""
    w = workload("tiny_f32", batch=2, dim=80, seqlen=400, dstate=16, io_dtype=io)
    x = spread_delta(make_inputs(w, seed=45, with_h0=True), io, -0.01, 0.12, seed=3)
    check_fwd(x, io, softplus=False)


# ------------------------------------------------------------------ backward
@pytest.mark.gpu
@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("use_ckpt", [False, True])
def test_bwd_softplus_over_the_whole_range(io, use_ckpt):
    """Every gradient with v over [-30, 30]: softplus' = sigmoid(v) from 1e-13 to 1, resets
    and vanishing steps in the same sequences."""
    w = workload("tiny_f32", batch=2, dim=96, seqlen=333, dstate=16, io_dtype=io)
    x = spread_delta(make_inputs(w, seed=46, with_h0=True, with_dout=True), io, seed=4)
    check_bwd(x, io, use_ckpt=use_ckpt, summed_scale=5.0)


@pytest.mark.gpu
@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
def test_bwd_resets_and_vanishing_steps(io):
    """Runs of large steps (v = 25) and of vanishing ones (v = -25) between ordinary ones."""
    w = workload("tiny_f32", batch=2, dim=64, seqlen=256, dstate=16, io_dtype=io)
    x = make_inputs(w, seed=47, with_h0=True, with_dout=True)
    d = x["delta"].float() + x["dt_bias"].float()[None, :, None]
    d[..., 20:40] = 25.0
    d[..., 100:180] = -25.0
    d[..., 200::9] = 25.0
    x["delta"] = d.to(io)
    x["dt_bias"] = torch.zeros_like(x["dt_bias"])
    check_bwd(x, io, summed_scale=5.0)


@pytest.mark.gpu
@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
def test_bwd_signed_steps_without_softplus(io):
    w = workload("tiny_f32", batch=2, dim=64, seqlen=300, dstate=16, io_dtype=io)
    x = spread_delta(make_inputs(w, seed=48, with_h0=True, with_dout=True), io, -0.01, 0.12,
                     seed=5)
    check_bwd(x, io, softplus=False)


# ------------------------------------------------------------------ decode
@pytest.mark.gpu
@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
def test_decode_softplus_over_the_whole_range(io):
    """Step by step against the oracle's recurrence with the raw step dt over [-30, 30]."""
    w = workload("decode_b256", batch=3, dim=96, dstate=16, io_dtype=io)
    r = np.random.default_rng(6)
    state0 = (0.5 * r.standard_normal((3, 96, 16))).astype(np.float32)
    state = torch.from_numpy(state0).to(DEV)
    ref_state = state0.astype(np.float64).copy()
    for t in range(24):
        x = spread_delta(make_inputs(w, seed=49, step=t), io, seed=100 + t, key="dt")
        xd = on_dev(x)
        out = ssm.ssm_state_update(state, xd["x"], xd["dt"], xd["A"], xd["B"], xd["C"],
                                   D=xd["D"], z=xd["z"], dt_bias=xd["dt_bias"])
        ro = oracle.state_update(ref_state, f64(x["x"]), f64(x["dt"]), f64(x["A"]), f64(x["B"]),
                                 f64(x["C"]), D=f64(x["D"]), z=f64(x["z"]),
                                 dt_bias=f64(x["dt_bias"]))
        assert_close(out, ro, io, f"out step {t}")
        assert_close(state, ref_state, io, f"state step {t}")
        if io == torch.bfloat16:
            assert_bf16_elementwise(out, ro, f"out step {t}")


@pytest.mark.gpu
@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
def test_decode_signed_steps_without_softplus(io):
    w = workload("decode_b256", batch=2, dim=64, dstate=16, io_dtype=io)
    state = torch.zeros((2, 64, 16), device=DEV)
    ref_state = np.zeros((2, 64, 16))
    for t in range(16):
        x = spread_delta(make_inputs(w, seed=50, step=t), io, -0.01, 0.12, seed=200 + t, key="dt")
        xd = on_dev(x)
        out = ssm.ssm_state_update(state, xd["x"], xd["dt"], xd["A"], xd["B"], xd["C"],
                                   D=xd["D"], z=xd["z"], dt_bias=xd["dt_bias"],
                                   delta_softplus=False)
        ro = oracle.state_update(ref_state, f64(x["x"]), f64(x["dt"]), f64(x["A"]), f64(x["B"]),
                                 f64(x["C"]), D=f64(x["D"]), z=f64(x["z"]),
                                 dt_bias=f64(x["dt_bias"]), delta_softplus=False)
        assert_close(out, ro, io, f"out step {t}")
        assert_close(state, ref_state, io, f"state step {t}")
