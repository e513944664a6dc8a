"""Scalar decay (one rate A_d per channel shared by its N states; the Mamba-2 restriction noted
on the "2024 Reading List: Neural Network" page): CUDA forward and backward through the C ABI
against the fp64 oracle run with A[d, n] = A_d for every n.  The oracle's scalar-decay results
are pinned in test_oracle_pins.py (masked Gram-matrix form; rate gradient by central
differences)."""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_23_b200 as ssm
from selective_state_space_23_b200.inputs import make_inputs, workload

from _parity import assert_close, f64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def on_dev(x):
    return {k: v.to(DEV) for k, v in x.items()}


def full_a(x):
    """[dim] rates -> [dim, N] for the oracle."""
    return np.repeat(f64(x["A"])[:, None], x["B"].shape[1], 1)


def oracle_fwd(x, softplus=True, sel=None):
    c = lambda k: None if x.get(k) is None else f64(x[k])
    A = full_a(x)
    u, delta, z, D, bias, h0 = c("u"), c("delta"), c("z"), c("D"), c("dt_bias"), c("h0")
    if sel is not None:
        u, delta = u[:, sel], delta[:, sel]
        z = None if z is None else z[:, sel]
        A, D = A[sel], None if D is None else D[sel]
        bias = None if bias is None else bias[sel]
        h0 = None if h0 is None else h0[:, sel]
    return oracle.scan_fwd(u, delta, A, c("B"), c("C"), D=D, z=z, dt_bias=bias,
                           delta_softplus=softplus, h0=h0)


def gpu_fwd(x, softplus=True, **kw):
    return ssm.ssm_scan_fwd_scalar_a(x["u"], x["delta"], x["A"], x["B"], x["C"], D=x.get("D"),
                                     z=x.get("z"), dt_bias=x.get("dt_bias"),
                                     delta_softplus=softplus, h0=x.get("h0"), **kw)


@pytest.fixture(autouse=True)
def _clean_env(monkeypatch):
    monkeypatch.delenv("SSM_FWD_SPLIT", raising=False)
    yield


@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("shape", [(2, 70, 250, 5), (1, 33, 37, 16), (3, 100, 1000, 16),
                                   (1, 1, 1, 1), (2, 64, 17, 3)])
def test_forward_ragged(io, shape):
    batch, dim, L, N = shape
    w = workload("tiny_f32", batch=batch, dim=dim, seqlen=L, dstate=N, io_dtype=io)
    x = make_inputs(w, seed=21, with_h0=True, scalar_a=True)
    out, hL, ck = gpu_fwd(on_dev(x), return_final_state=True, return_ckpt=True)
    ref = oracle_fwd(x)
    tol = torch.float32 if io == torch.float32 else io
    assert_close(out, ref["out"], io, "out")
    assert_close(hL, ref["hL"], tol, "hL")
    # checkpoints: state entering every 16-step block, from the oracle's prefix runs
    for k in range(0, (L + 15) // 16, max(1, (L + 15) // 16 // 3)):
        if k == 0:
            want = f64(x["h0"])
        else:
            xs = dict(x, u=x["u"][..., :16 * k], delta=x["delta"][..., :16 * k],
                      z=x["z"][..., :16 * k], B=x["B"][..., :16 * k], C=x["C"][..., :16 * k])
            want = oracle_fwd(xs)["hL"]
        assert_close(ck[:, :, k], want, tol, f"ckpt block {k}")


@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
def test_forward_without_gate_skip_bias_softplus(io):
    w = workload("tiny_f32", batch=2, dim=96, seqlen=320, dstate=16, io_dtype=io)
    x = make_inputs(w, seed=22, gate=False, scalar_a=True)
    x["delta"] = (x["delta"].float().abs() * 0.05 + 1e-3).to(io)
    del x["D"], x["dt_bias"]
    out = gpu_fwd(on_dev(x), softplus=False)
    assert_close(out, oracle_fwd(x, softplus=False)["out"], io, "out")


@pytest.mark.parametrize("split", [2, 7])
def test_forward_time_split(monkeypatch, split):
    monkeypatch.setenv("SSM_FWD_SPLIT", str(split))
    w = workload("tiny_f32", batch=2, dim=48, seqlen=900, io_dtype=torch.bfloat16)
    x = make_inputs(w, seed=23, with_h0=True, scalar_a=True)
    assert ssm.fwd_workspace_bytes(2, 48, 900, 16, torch.bfloat16) > 0
    out, hL = gpu_fwd(on_dev(x), return_final_state=True)
    ref = oracle_fwd(x)
    assert_close(out, ref["out"], torch.bfloat16, "out")
    assert_close(hL, ref["hL"], torch.bfloat16, "hL")


def test_forward_rejects_wrong_a_shape():
    w = workload("tiny_f32", batch=1, dim=32, seqlen=64)
    x = on_dev(make_inputs(w, seed=24))          # A is [dim, N]
    with pytest.raises(ValueError):
        gpu_fwd(x)


def test_forward_deterministic_and_matches_full_rate_matrix():
    """Same result as ssm_scan_fwd with A broadcast to [dim, N] (within rounding: the scalar
    path uses one exponential per step for all states)."""
    w = workload("mamba370m_fwd", batch=2, dim=256, seqlen=1024)
    x = on_dev(make_inputs(w, seed=25, scalar_a=True))
    a = gpu_fwd(x)
    b = gpu_fwd(x)
    assert torch.equal(a, b)
    full = ssm.ssm_scan_fwd(x["u"], x["delta"], x["A"][:, None].repeat(1, 16).contiguous(),
                            x["B"], x["C"], D=x["D"], z=x["z"], dt_bias=x["dt_bias"])
    assert_close(a, f64(full), torch.bfloat16, "scalar vs broadcast")


@pytest.mark.slow
def test_mamba370m_shape_full():
    w = workload("mamba370m_fwd")
    x = make_inputs(w, seed=26, scalar_a=True)
    out = gpu_fwd(on_dev(x))
    assert_close(out, oracle_fwd(x)["out"], torch.bfloat16, "out")


# ------------------------------------------------------------------ backward
GRADS = ("du", "ddelta", "dz", "dB", "dC", "dA", "dD", "ddt_bias", "dh0")


def oracle_bwd(x, softplus=True, dhL=None):
    c = lambda k: None if x.get(k) is None else f64(x[k])
    g = oracle.scan_bwd(c("u"), c("delta"), full_a(x), c("B"), c("C"), c("dout"), D=c("D"),
                        z=c("z"), dt_bias=c("dt_bias"), delta_softplus=softplus, h0=c("h0"),
                        dhL=None if dhL is None else f64(dhL))
    g["dA"] = g["dA"].sum(1)     # chain rule through A[d, n] = A_d
    return g


@pytest.mark.parametrize("use_ckpt", [False, True])
@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
def test_backward(io, use_ckpt):
    w = workload("tiny_f32", batch=2, dim=80, seqlen=333, io_dtype=io)
    x = make_inputs(w, seed=27, with_dout=True, with_h0=True, scalar_a=True)
    dhL = torch.randn((2, 80, 16), generator=torch.Generator().manual_seed(3))
    xd = on_dev(x)
    ck = None
    if use_ckpt:
        _, ck = gpu_fwd(xd, return_ckpt=True)
    g = ssm.ssm_scan_bwd_scalar_a(xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"], xd["dout"],
                                  D=xd["D"], z=xd["z"], dt_bias=xd["dt_bias"], h0=xd["h0"],
                                  dhL=dhL.to(DEV), ckpt=ck)
    assert g["dA"].shape == (80,)
    r = oracle_bwd(x, dhL=dhL)
    for k in GRADS:
        assert_close(g[k], r[k], io, k)
