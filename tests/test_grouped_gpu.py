"""Grouped B/C (B, C, dB, dC of shape [batch, G, N, L]; channel d uses group d // (dim // G), the
per-token B_t, C_t of the selection mechanism computed once per group of channels): CUDA
forward and backward through the C ABI against the fp64 oracle, which runs each group as its
own scan (pinned in test_oracle_pins.py by the per-group quadratic form and finite
differences).  Also: one group equals the shared layout bitwise, unsupported splits are
refused on the host, and the combinations with the reverse scan, the scalar decay and ZOH."""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_23_b200 as ssm
from selective_state_space_23_b200 import _abi
from selective_state_space_23_b200.inputs import make_inputs, workload

from _parity import assert_close, f64

pytestmark = pytest.mark.gpu
DEV = "cuda"
GRADS = ("du", "ddelta", "dz", "dB", "dC", "dA", "dD", "ddt_bias", "dh0")


def grouped_inputs(batch, dim, L, G, io=torch.bfloat16, seed=0, **kw):
    """The workload's inputs with B, C drawn per group ([batch, G, N, L])."""
    w = workload("tiny_f32", batch=batch, dim=dim, seqlen=L, io_dtype=io)
    x = make_inputs(w, seed=seed, **kw)
    wg = workload("tiny_f32", batch=batch * G, dim=dim, seqlen=L, io_dtype=io)
    xg = make_inputs(wg, seed=seed + 1000)
    x["B"] = xg["B"].reshape(batch, G, 16, L).contiguous()
    x["C"] = xg["C"].reshape(batch, G, 16, L).contiguous()
    return x


def on_dev(x):
    return {k: v.to(DEV) for k, v in x.items()}


def c64(x, k):
    return None if x.get(k) is None else f64(x[k])


def full_a(x, scalar_a):
    A = c64(x, "A")
    return np.repeat(A[:, None], x["B"].shape[2], 1) if scalar_a else A


def oracle_fwd(x, scalar_a=False, reverse=False, zoh=False):
    return oracle.scan_fwd(c64(x, "u"), c64(x, "delta"), full_a(x, scalar_a), c64(x, "B"),
                           c64(x, "C"), D=c64(x, "D"), z=c64(x, "z"), dt_bias=c64(x, "dt_bias"),
                           h0=c64(x, "h0"), reverse=reverse, zoh=zoh)


def gpu_fwd(x, scalar_a=False, **kw):
    f = ssm.ssm_scan_fwd_scalar_a if scalar_a else ssm.ssm_scan_fwd
    return f(x["u"], x["delta"], x["A"], x["B"], x["C"], D=x.get("D"), z=x.get("z"),
             dt_bias=x.get("dt_bias"), h0=x.get("h0"), **kw)


@pytest.fixture(autouse=True)
def _clean_env(monkeypatch):
    monkeypatch.delenv("SSM_FWD_SPLIT", raising=False)
    yield


@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("batch,dim,L,G", [(2, 64, 250, 4), (1, 128, 1000, 2), (3, 96, 37, 6),
                                           (2, 32, 256, 2)])
def test_forward(io, batch, dim, L, G):
    x = grouped_inputs(batch, dim, L, G, io, seed=51, with_h0=True)
    out, hL = gpu_fwd(on_dev(x), return_final_state=True)
    ref = oracle_fwd(x)
    assert_close(out, ref["out"], io, "out")
    assert_close(hL, ref["hL"], torch.float32 if io == torch.float32 else io, "hL")


def test_one_group_equals_shared_layout():
    w = workload("mamba370m_fwd", batch=2, dim=128, seqlen=512)
    x = on_dev(make_inputs(w, seed=52))
    a = gpu_fwd(x)
    b = gpu_fwd(dict(x, B=x["B"][:, None], C=x["C"][:, None]))
    assert torch.equal(a, b)


def test_unsupported_splits_are_refused():
    x = on_dev(grouped_inputs(1, 48, 64, 3, seed=53))      # 16 channels per group: fine
    gpu_fwd(x)
    y = on_dev(grouped_inputs(1, 48, 64, 6, seed=54))      # 8 channels per group
    with pytest.raises(RuntimeError, match="multiple of 16"):
        gpu_fwd(y)
    z = on_dev(grouped_inputs(1, 50, 64, 4, seed=55))      # 50 channels do not split in 4
    with pytest.raises(RuntimeError):
        gpu_fwd(z)


@pytest.mark.parametrize("split", [3])
def test_forward_time_split(monkeypatch, split):
    monkeypatch.setenv("SSM_FWD_SPLIT", str(split))
    x = grouped_inputs(2, 64, 1000, 4, seed=56, with_h0=True)
    out, hL = gpu_fwd(on_dev(x), return_final_state=True)
    ref = oracle_fwd(x)
    assert_close(out, ref["out"], torch.bfloat16, "out")
    assert_close(hL, ref["hL"], torch.bfloat16, "hL")


@pytest.mark.parametrize("scalar_a,reverse,zoh", [(False, True, False), (True, False, False),
                                                  (False, False, True), (True, True, True)])
def test_forward_combined(scalar_a, reverse, zoh):
    x = grouped_inputs(2, 64, 333, 2, seed=57, with_h0=True, scalar_a=scalar_a)
    out = gpu_fwd(on_dev(x), scalar_a=scalar_a, reverse=reverse, zoh=zoh)
    ref = oracle_fwd(x, scalar_a=scalar_a, reverse=reverse, zoh=zoh)
    assert_close(out, ref["out"], torch.bfloat16, "out")


@pytest.mark.slow
def test_mamba2p8b_shape_eight_groups_sampled():
    """4 x 5120 x 2048 with 8 groups: every channel of 4 sampled groups' first 16 channels and
    of the last channel block, against the oracle on those channels' groups."""
    x = grouped_inputs(4, 5120, 2048, 8, seed=58)
    out = f64(gpu_fwd(on_dev(x)))
    per = 640
    for g in (0, 3, 7):
        sl = slice(g * per, g * per + 16)
        xs = {k: (v[:, sl] if k in ("u", "delta", "z") else v[sl] if k in ("A", "D", "dt_bias")
                  else v[:, g:g + 1] if k in ("B", "C") else v) for k, v in x.items()}
        ref = oracle_fwd(xs)["out"]
        assert_close(out[:, sl], ref, torch.bfloat16, f"group {g}")


# ------------------------------------------------------------------ backward
def oracle_bwd(x, dhL, scalar_a=False, reverse=False, zoh=False):
    g = oracle.scan_bwd(c64(x, "u"), c64(x, "delta"), full_a(x, scalar_a), c64(x, "B"),
                        c64(x, "C"), c64(x, "dout"), D=c64(x, "D"), z=c64(x, "z"),
                        dt_bias=c64(x, "dt_bias"), h0=c64(x, "h0"), dhL=f64(dhL),
                        reverse=reverse, zoh=zoh)
    if scalar_a:
        g["dA"] = g["dA"].sum(1)
    return g


@pytest.mark.parametrize("use_ckpt", [False, True])
@pytest.mark.parametrize("io,L,G", [(torch.float32, 333, 4), (torch.bfloat16, 256, 2),
                                    (torch.bfloat16, 101, 4)])
def test_backward(io, L, G, use_ckpt):
    x = grouped_inputs(2, 64, L, G, io, seed=59, with_dout=True, with_h0=True)
    dhL = torch.randn((2, 64, 16), generator=torch.Generator().manual_seed(11))
    xd = on_dev(x)
    ck = None
    if use_ckpt:
        _, ck = gpu_fwd(xd, return_ckpt=True)
    g = ssm.ssm_scan_bwd(xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"], xd["dout"], D=xd["D"],
                         z=xd["z"], dt_bias=xd["dt_bias"], h0=xd["h0"], dhL=dhL.to(DEV), ckpt=ck)
    assert g["dB"].shape == (2, G, 16, L)
    r = oracle_bwd(x, dhL)
    for k in GRADS:
        assert_close(g[k], r[k], io, k)


@pytest.mark.parametrize("scalar_a,reverse,zoh", [(False, True, False), (True, False, True)])
def test_backward_combined(scalar_a, reverse, zoh):
    x = grouped_inputs(2, 64, 200, 2, seed=60, with_dout=True, with_h0=True, scalar_a=scalar_a)
    dhL = torch.randn((2, 64, 16), generator=torch.Generator().manual_seed(12))
    xd = on_dev(x)
    f = ssm.ssm_scan_bwd_scalar_a if scalar_a else ssm.ssm_scan_bwd
    g = f(xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"], xd["dout"], D=xd["D"], z=xd["z"],
          dt_bias=xd["dt_bias"], h0=xd["h0"], dhL=dhL.to(DEV), reverse=reverse, zoh=zoh)
    r = oracle_bwd(x, dhL, scalar_a=scalar_a, reverse=reverse, zoh=zoh)
    for k in GRADS:
        assert_close(g[k], r[k], torch.bfloat16, k)
