"""Zero-order-hold input term (SSM_ZOH; "Mamba: ..." summary page, "Yöntem": B̄ = (ΔA)^{-1}
(exp(ΔA) - I) ΔB, i.e. the coefficient c = (e^{ΔA} - 1)/A of B_t x_t per state): CUDA forward
and backward through the C ABI against the fp64 oracle run with zoh=True (its forward is pinned
by the exact gating case, its gradients by finite differences in test_oracle_pins.py).  Covers
the A -> 0 limit, tiny and positive rates, rates outside the checked exponent range, the time
split, checkpoints, and the combinations with the scalar decay and the reverse scan."""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_23_b200 as ssm
from selective_state_space_23_b200.inputs import make_inputs, workload

from _parity import assert_close, f64

pytestmark = pytest.mark.gpu
DEV = "cuda"
GRADS = ("du", "ddelta", "dz", "dB", "dC", "dA", "dD", "ddt_bias", "dh0")


def on_dev(x):
    return {k: v.to(DEV) for k, v in x.items()}


def c64(x, k):
    return None if x.get(k) is None else f64(x[k])


def full_a(x, scalar_a):
    A = c64(x, "A")
    return np.repeat(A[:, None], x["B"].shape[1], 1) if scalar_a else A


def oracle_fwd(x, scalar_a=False, reverse=False, softplus=True):
    return oracle.scan_fwd(c64(x, "u"), c64(x, "delta"), full_a(x, scalar_a), c64(x, "B"),
                           c64(x, "C"), D=c64(x, "D"), z=c64(x, "z"), dt_bias=c64(x, "dt_bias"),
                           delta_softplus=softplus, h0=c64(x, "h0"), zoh=True, reverse=reverse)


def gpu_fwd(x, scalar_a=False, reverse=False, softplus=True, **kw):
    f = ssm.ssm_scan_fwd_scalar_a if scalar_a else ssm.ssm_scan_fwd
    return f(x["u"], x["delta"], x["A"], x["B"], x["C"], D=x.get("D"), z=x.get("z"),
             dt_bias=x.get("dt_bias"), delta_softplus=softplus, h0=x.get("h0"), zoh=True,
             reverse=reverse, **kw)


def special_rates(A):
    """Zero, tiny, positive and very negative rates (the last outside the exponent range the
    unclamped FMA-pipe form is used for, so its warp takes the clamped form)."""
    A = A.clone()
    A[0, :] = 0.0
    A[1, 0] = -1e-7
    A[2, 3] = 2e-4
    A[3, 5] = 0.05
    A[-1, 2] = -3e4
    return A


@pytest.fixture(autouse=True)
def _clean_env(monkeypatch):
    monkeypatch.delenv("SSM_FWD_SPLIT", raising=False)
    yield


@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("shape", [(2, 70, 256, 16), (1, 33, 37, 16), (3, 100, 1000, 16),
                                   (2, 40, 250, 5), (1, 1, 1, 1)])
def test_forward(io, shape):
    batch, dim, L, N = shape
    w = workload("tiny_f32", batch=batch, dim=dim, seqlen=L, dstate=N, io_dtype=io)
    x = make_inputs(w, seed=41, with_h0=True)
    out, hL = gpu_fwd(on_dev(x), return_final_state=True)
    ref = oracle_fwd(x)
    assert_close(out, ref["out"], io, "out")
    assert_close(hL, ref["hL"], torch.float32 if io == torch.float32 else io, "hL")


@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
def test_forward_special_rates(io):
    w = workload("tiny_f32", batch=2, dim=48, seqlen=300, io_dtype=io)
    x = make_inputs(w, seed=42, with_h0=True)
    x["A"] = special_rates(x["A"])
    out, hL = gpu_fwd(on_dev(x), return_final_state=True)
    ref = oracle_fwd(x)
    assert_close(out, ref["out"], io, "out")
    assert_close(hL, ref["hL"], torch.float32 if io == torch.float32 else io, "hL")


def test_forward_differs_from_first_order_term():
    w = workload("tiny_f32", batch=1, dim=16, seqlen=64)
    x = on_dev(make_inputs(w, seed=43))
    a = gpu_fwd(x)
    b = ssm.ssm_scan_fwd(x["u"], x["delta"], x["A"], x["B"], x["C"], D=x["D"], z=x["z"],
                         dt_bias=x["dt_bias"])
    assert (a - b).abs().max() > 1e-3


@pytest.mark.parametrize("split", [2, 6])
def test_forward_time_split(monkeypatch, split):
    monkeypatch.setenv("SSM_FWD_SPLIT", str(split))
    w = workload("tiny_f32", batch=2, dim=48, seqlen=1000, io_dtype=torch.bfloat16)
    x = make_inputs(w, seed=44, with_h0=True)
    out, hL = gpu_fwd(on_dev(x), return_final_state=True)
    ref = oracle_fwd(x)
    assert_close(out, ref["out"], torch.bfloat16, "out")
    assert_close(hL, ref["hL"], torch.bfloat16, "hL")


@pytest.mark.parametrize("scalar_a,reverse", [(True, False), (False, True), (True, True)])
@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
def test_forward_combined(io, scalar_a, reverse):
    w = workload("tiny_f32", batch=2, dim=80, seqlen=333, io_dtype=io)
    x = make_inputs(w, seed=45, with_h0=True, scalar_a=scalar_a)
    out, hL = gpu_fwd(on_dev(x), scalar_a=scalar_a, reverse=reverse, return_final_state=True)
    ref = oracle_fwd(x, scalar_a=scalar_a, reverse=reverse)
    assert_close(out, ref["out"], io, "out")
    assert_close(hL, ref["hL"], torch.float32 if io == torch.float32 else io, "hL")


@pytest.mark.slow
def test_mamba370m_shape_full():
    w = workload("mamba370m_fwd")
    x = make_inputs(w, seed=46)
    out = gpu_fwd(on_dev(x))
    assert_close(out, oracle_fwd(x)["out"], torch.bfloat16, "out")


# ------------------------------------------------------------------ backward
def oracle_bwd(x, dhL, scalar_a=False, reverse=False):
    g = oracle.scan_bwd(c64(x, "u"), c64(x, "delta"), full_a(x, scalar_a), c64(x, "B"),
                        c64(x, "C"), c64(x, "dout"), D=c64(x, "D"), z=c64(x, "z"),
                        dt_bias=c64(x, "dt_bias"), h0=c64(x, "h0"), dhL=f64(dhL), zoh=True,
                        reverse=reverse)
    if scalar_a:
        g["dA"] = g["dA"].sum(1)
    return g


def run_bwd(x, dhL, scalar_a=False, reverse=False, use_ckpt=False):
    xd = on_dev(x)
    ck = None
    if use_ckpt:
        _, ck = gpu_fwd(xd, scalar_a=scalar_a, reverse=reverse, return_ckpt=True)
    f = ssm.ssm_scan_bwd_scalar_a if scalar_a else ssm.ssm_scan_bwd
    return f(xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"], xd["dout"], D=xd["D"], z=xd["z"],
             dt_bias=xd["dt_bias"], h0=xd["h0"], dhL=dhL.to(DEV), ckpt=ck, zoh=True,
             reverse=reverse)


@pytest.mark.parametrize("use_ckpt", [False, True])
@pytest.mark.parametrize("io,L", [(torch.float32, 333), (torch.bfloat16, 256), (torch.bfloat16, 101)])
def test_backward(io, L, use_ckpt):
    w = workload("tiny_f32", batch=2, dim=80, seqlen=L, io_dtype=io)
    x = make_inputs(w, seed=47, with_dout=True, with_h0=True)
    dhL = torch.randn((2, 80, 16), generator=torch.Generator().manual_seed(7))
    g = run_bwd(x, dhL, use_ckpt=use_ckpt)
    r = oracle_bwd(x, dhL)
    for k in GRADS:
        assert_close(g[k], r[k], io, k)


@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
def test_backward_special_rates(io):
    w = workload("tiny_f32", batch=2, dim=48, seqlen=200, io_dtype=io)
    x = make_inputs(w, seed=48, with_dout=True, with_h0=True)
    x["A"] = special_rates(x["A"])
    dhL = torch.randn((2, 48, 16), generator=torch.Generator().manual_seed(8))
    g = run_bwd(x, dhL)
    r = oracle_bwd(x, dhL)
    for k in GRADS:
        assert_close(g[k], r[k], io, k)


@pytest.mark.parametrize("scalar_a,reverse", [(True, False), (False, True)])
def test_backward_combined(scalar_a, reverse):
    w = workload("tiny_f32", batch=2, dim=64, seqlen=256, io_dtype=torch.bfloat16)
    x = make_inputs(w, seed=49, with_dout=True, with_h0=True, scalar_a=scalar_a)
    dhL = torch.randn((2, 64, 16), generator=torch.Generator().manual_seed(9))
    g = run_bwd(x, dhL, scalar_a=scalar_a, reverse=reverse, use_ckpt=True)
    r = oracle_bwd(x, dhL, scalar_a=scalar_a, reverse=reverse)
    for k in GRADS:
        assert_close(g[k], r[k], torch.bfloat16, k)
