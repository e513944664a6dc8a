"""Reverse scan (t = L-1 down to 0; the anti-causal half of a bidirectional layer, Hydra notes
on the "2024 Reading List: Neural Network" page): CUDA forward and backward through the C ABI
against the fp64 oracle's reverse scan (pinned in test_oracle_pins.py by the anti-causal
quadratic form and finite differences).  The kernels read and write every time row mirrored,
so both the 128-bit path (L a multiple of 8) and the element path (other L) are covered."""
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


def oracle_fwd(x, softplus=True, scalar_a=False):
    A = c64(x, "A")
    if scalar_a:
        A = np.repeat(A[:, None], x["B"].shape[1], 1)
    return oracle.scan_fwd(c64(x, "u"), c64(x, "delta"), A, c64(x, "B"), c64(x, "C"),
                           D=c64(x, "D"), z=c64(x, "z"), dt_bias=c64(x, "dt_bias"),
                           delta_softplus=softplus, h0=c64(x, "h0"), reverse=True)


def gpu_fwd(x, softplus=True, scalar_a=False, **kw):
    f = ssm.ssm_scan_fwd_scalar_a if scalar_a else ssm.ssm_scan_fwd
    return f(x["u"], x["delta"], x["A"], x["B"], x["C"], D=x.get("D"), z=x.get("z"),
             dt_bias=x.get("dt_bias"), delta_softplus=softplus, h0=x.get("h0"), reverse=True, **kw)


@pytest.fixture(autouse=True)
def _clean_env(monkeypatch):
    monkeypatch.delenv("SSM_FWD_SPLIT", raising=False)
    yield


@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("shape", [(2, 70, 256, 16), (1, 33, 37, 16), (3, 100, 1000, 16),
                                   (2, 40, 250, 5), (1, 1, 1, 1), (2, 64, 17, 3)])
def test_forward(io, shape):
    batch, dim, L, N = shape
    w = workload("tiny_f32", batch=batch, dim=dim, seqlen=L, dstate=N, io_dtype=io)
    x = make_inputs(w, seed=31, with_h0=True)
    out, hL = gpu_fwd(on_dev(x), return_final_state=True)
    ref = oracle_fwd(x)
    assert_close(out, ref["out"], io, "out")
    assert_close(hL, ref["hL"], torch.float32 if io == torch.float32 else io, "hL")


@pytest.mark.parametrize("L", [96, 101])
def test_checkpoints_in_scan_order(L):
    """Block k of the checkpoints holds the state before scan steps 16k.., i.e. after the time
    suffix [L-16k, L) has been scanned."""
    w = workload("tiny_f32", batch=2, dim=24, seqlen=L)
    x = make_inputs(w, seed=32, with_h0=True)
    _, ck = gpu_fwd(on_dev(x), return_ckpt=True)
    for k in range((L + 15) // 16):
        if k == 0:
            want = f64(x["h0"])
        else:
            tail = {key: (v[..., L - 16 * k:] if key in ("u", "delta", "z", "B", "C") else v)
                    for key, v in x.items()}
            want = oracle_fwd(tail)["hL"]
        assert_close(ck[:, :, k], want, torch.float32, f"ckpt block {k}")


@pytest.mark.parametrize("split", [2, 5])
def test_forward_time_split(monkeypatch, split):
    monkeypatch.setenv("SSM_FWD_SPLIT", str(split))
    w = workload("tiny_f32", batch=2, dim=48, seqlen=1000, io_dtype=torch.bfloat16)
    x = make_inputs(w, seed=33, with_h0=True)
    out, hL = gpu_fwd(on_dev(x), return_final_state=True)
    ref = oracle_fwd(x)
    assert_close(out, ref["out"], torch.bfloat16, "out")
    assert_close(hL, ref["hL"], torch.bfloat16, "hL")


def test_forward_scalar_decay():
    w = workload("tiny_f32", batch=2, dim=80, seqlen=333, io_dtype=torch.bfloat16)
    x = make_inputs(w, seed=34, with_h0=True, scalar_a=True)
    out = gpu_fwd(on_dev(x), scalar_a=True)
    assert_close(out, oracle_fwd(x, scalar_a=True)["out"], torch.bfloat16, "out")


def test_reverse_equals_forward_on_reversed_rows(monkeypatch):
    """Bitwise: the reverse scan of the rows equals the forward scan of the flipped rows,
    flipped back (same kernel arithmetic in the same order: the general kernel, which runs the
    reverse scan)."""
    monkeypatch.setenv("SSM_FWD_KERNEL", "pair")
    w = workload("mamba370m_fwd", batch=2, dim=128, seqlen=512)
    x = on_dev(make_inputs(w, seed=35))
    fl = {k: (v.flip(-1).contiguous() if k in ("u", "delta", "z", "B", "C") else v)
          for k, v in x.items()}
    a = gpu_fwd(x)
    b = ssm.ssm_scan_fwd(fl["u"], fl["delta"], fl["A"], fl["B"], fl["C"], D=fl["D"], z=fl["z"],
                         dt_bias=fl["dt_bias"]).flip(-1)
    assert torch.equal(a, b)


@pytest.mark.slow
def test_mamba370m_shape_full():
    w = workload("mamba370m_fwd")
    x = make_inputs(w, seed=36)
    out = gpu_fwd(on_dev(x))
    assert_close(out, oracle_fwd(x)["out"], torch.bfloat16, "out")


# ------------------------------------------------------------------ backward
def oracle_bwd(x, dhL, scalar_a=False):
    A = c64(x, "A")
    if scalar_a:
        A = np.repeat(A[:, None], x["B"].shape[1], 1)
    g = oracle.scan_bwd(c64(x, "u"), c64(x, "delta"), A, c64(x, "B"), c64(x, "C"),
                        c64(x, "dout"), D=c64(x, "D"), z=c64(x, "z"), dt_bias=c64(x, "dt_bias"),
                        h0=c64(x, "h0"), dhL=f64(dhL), reverse=True)
    if scalar_a:
        g["dA"] = g["dA"].sum(1)
    return g


@pytest.mark.parametrize("scalar_a", [False, True])
@pytest.mark.parametrize("use_ckpt", [False, True])
@pytest.mark.parametrize("io,L", [(torch.float32, 333), (torch.bfloat16, 256),
                                  (torch.bfloat16, 101)])
def test_backward(io, L, use_ckpt, scalar_a):
    w = workload("tiny_f32", batch=2, dim=80, seqlen=L, io_dtype=io)
    x = make_inputs(w, seed=37, with_dout=True, with_h0=True, scalar_a=scalar_a)
    dhL = torch.randn((2, 80, 16), generator=torch.Generator().manual_seed(5))
    xd = on_dev(x)
    ck = None
    if use_ckpt:
        _, ck = gpu_fwd(xd, scalar_a=scalar_a, return_ckpt=True)
    f = ssm.ssm_scan_bwd_scalar_a if scalar_a else ssm.ssm_scan_bwd
    g = f(xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"], xd["dout"], D=xd["D"], z=xd["z"],
          dt_bias=xd["dt_bias"], h0=xd["h0"], dhL=dhL.to(DEV), ckpt=ck, reverse=True)
    r = oracle_bwd(x, dhL, scalar_a)
    for k in GRADS:
        assert_close(g[k], r[k], io, k)
