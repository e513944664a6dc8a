"""The (B, L, D) layout (SSM_CHANNELS_LAST; the projections' own output layout): u, delta, z,
out, dout, du, ddelta, dz as [batch, L, dim] and B, C, dB, dC as [batch, L, N] or
[batch, L, G, N].  The same scan in another memory order: results equal the default layout's
bitwise, and match the fp64 oracle (run on the transposed tensors) for the forward, the
backward, the time split and the other variants."""
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
TIME_ROWS = ("u", "delta", "z", "dout")


def to_cl(x):
    """[batch, dim, L] -> [batch, L, dim]; B, C [batch, (G,) N, L] -> [batch, L, (G,) N]."""
    y = {}
    for k, v in x.items():
        if k in TIME_ROWS:
            y[k] = v.transpose(1, 2).contiguous()
        elif k in ("B", "C"):
            y[k] = v.movedim(-1, 1).contiguous()
        else:
            y[k] = v
    return y


def from_cl_bc(t):
    return t.movedim(1, -1)


def on_dev(x):
    return {k: v.to(DEV) for k, v in x.items()}


def run_fwd(x, cl, **kw):
    return ssm.ssm_scan_fwd(x["u"], x["delta"], x["A"], x["B"], x["C"], D=x.get("D"),
                            z=x.get("z"), dt_bias=x.get("dt_bias"), h0=x.get("h0"),
                            channels_last=cl, **kw)


@pytest.fixture(autouse=True)
def _clean_env(monkeypatch):
    # the channels-last layout runs in the general (two-lanes-per-channel) kernels; the default
    # layout is compared with it bitwise, so it runs there too
    monkeypatch.delenv("SSM_FWD_SPLIT", raising=False)
    monkeypatch.setenv("SSM_FWD_KERNEL", "pair")
    monkeypatch.setenv("SSM_BWD_KERNEL", "pair")
    yield


@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("shape", [(2, 70, 250, 16), (1, 33, 37, 16), (2, 64, 512, 5)])
def test_forward_matches_oracle_and_default_layout(io, shape):
    batch, dim, L, N = shape
    w = workload("tiny_f32", batch=batch, dim=dim, seqlen=L, dstate=N, io_dtype=io)
    x = make_inputs(w, seed=71, with_h0=True)
    out_cl, hL_cl = run_fwd(on_dev(to_cl(x)), True, return_final_state=True)
    out, hL = run_fwd(on_dev(x), False, return_final_state=True)
    assert out_cl.shape == (batch, L, dim)
    assert torch.equal(out_cl.transpose(1, 2), out) and torch.equal(hL_cl, hL)
    c = lambda k: None if x.get(k) is None else f64(x[k])
    ref = oracle.scan_fwd(c("u"), c("delta"), c("A"), c("B"), c("C"), D=c("D"), z=c("z"),
                          dt_bias=c("dt_bias"), h0=c("h0"))
    assert_close(out_cl.transpose(1, 2), ref["out"], io, "out")


@pytest.mark.parametrize("reverse,zoh,groups,split", [(True, False, 1, 0), (False, True, 2, 0),
                                                      (False, False, 4, 3), (True, True, 1, 2)])
def test_forward_variants_equal_default_layout(monkeypatch, reverse, zoh, groups, split):
    if split:
        monkeypatch.setenv("SSM_FWD_SPLIT", str(split))
    w = workload("tiny_f32", batch=2, dim=64, seqlen=700, io_dtype=torch.bfloat16)
    x = make_inputs(w, seed=72, with_h0=True)
    if groups > 1:
        wg = workload("tiny_f32", batch=2 * groups, dim=64, seqlen=700, io_dtype=torch.bfloat16)
        xg = make_inputs(wg, seed=73)
        x["B"] = xg["B"].reshape(2, groups, 16, 700).contiguous()
        x["C"] = xg["C"].reshape(2, groups, 16, 700).contiguous()
    a = run_fwd(on_dev(to_cl(x)), True, reverse=reverse, zoh=zoh)
    b = run_fwd(on_dev(x), False, reverse=reverse, zoh=zoh)
    assert torch.equal(a.transpose(1, 2), b)


# dim a multiple of 16 with N = 16 takes the 16-byte tile loads and stores; dim = 72 or N = 5
# takes the element-stride path
@pytest.mark.parametrize("io,dim,N,L,use_ckpt", [(torch.float32, 80, 16, 333, False),
                                                 (torch.bfloat16, 80, 16, 256, True),
                                                 (torch.bfloat16, 80, 16, 101, False),
                                                 (torch.bfloat16, 72, 16, 101, False),
                                                 (torch.float32, 80, 5, 64, False)])
def test_backward(io, dim, N, L, use_ckpt):
    w = workload("tiny_f32", batch=2, dim=dim, seqlen=L, dstate=N, io_dtype=io)
    x = make_inputs(w, seed=74, with_dout=True, with_h0=True)
    dhL = torch.randn((2, dim, N), generator=torch.Generator().manual_seed(13))
    xc = on_dev(to_cl(x))
    ck = None
    if use_ckpt:
        _, ck = run_fwd(xc, True, return_ckpt=True)
    g = ssm.ssm_scan_bwd(xc["u"], xc["delta"], xc["A"], xc["B"], xc["C"], xc["dout"], D=xc["D"],
                         z=xc["z"], dt_bias=xc["dt_bias"], h0=xc["h0"], dhL=dhL.to(DEV), ckpt=ck,
                         channels_last=True)
    c = lambda k: None if x.get(k) is None else f64(x[k])
    r = oracle.scan_bwd(c("u"), c("delta"), c("A"), c("B"), c("C"), c("dout"), D=c("D"),
                        z=c("z"), dt_bias=c("dt_bias"), h0=c("h0"), dhL=f64(dhL))
    for k in GRADS:
        got = g[k]
        if k in ("du", "ddelta", "dz"):
            got = got.transpose(1, 2)
        elif k in ("dB", "dC"):
            got = from_cl_bc(got)
        assert_close(got, r[k], io, k)


def test_backward_grouped_reverse_zoh_equals_default_layout():
    w = workload("tiny_f32", batch=2, dim=64, seqlen=200, io_dtype=torch.bfloat16)
    x = make_inputs(w, seed=75, with_dout=True, with_h0=True)
    wg = workload("tiny_f32", batch=4, dim=64, seqlen=200, io_dtype=torch.bfloat16)
    xg = make_inputs(wg, seed=76)
    x["B"] = xg["B"].reshape(2, 2, 16, 200).contiguous()
    x["C"] = xg["C"].reshape(2, 2, 16, 200).contiguous()
    kw = dict(reverse=True, zoh=True)
    xd, xc = on_dev(x), on_dev(to_cl(x))
    gd = ssm.ssm_scan_bwd(xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"], xd["dout"], D=xd["D"],
                          z=xd["z"], dt_bias=xd["dt_bias"], h0=xd["h0"], **kw)
    gc = ssm.ssm_scan_bwd(xc["u"], xc["delta"], xc["A"], xc["B"], xc["C"], xc["dout"], D=xc["D"],
                          z=xc["z"], dt_bias=xc["dt_bias"], h0=xc["h0"], channels_last=True, **kw)
    for k in GRADS:
        a = gc[k]
        if k in ("du", "ddelta", "dz"):
            a = a.transpose(1, 2)
        elif k in ("dB", "dC"):
            a = from_cl_bc(a)
        assert torch.equal(a, gd[k]), k


@pytest.mark.parametrize("io,dim,L", [(torch.bfloat16, 48, 77), (torch.float32, 48, 16),
                                      (torch.bfloat16, 32, 1)])
def test_backward_tiles_equal_default_layout(io, dim, L):
    w = workload("tiny_f32", batch=3, dim=dim, seqlen=L, io_dtype=io)
    x = make_inputs(w, seed=77, with_dout=True, with_h0=True)
    xd, xc = on_dev(x), on_dev(to_cl(x))
    gd = ssm.ssm_scan_bwd(xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"], xd["dout"], D=xd["D"],
                          z=xd["z"], dt_bias=xd["dt_bias"], h0=xd["h0"])
    gc = ssm.ssm_scan_bwd(xc["u"], xc["delta"], xc["A"], xc["B"], xc["C"], xc["dout"], D=xc["D"],
                          z=xc["z"], dt_bias=xc["dt_bias"], h0=xc["h0"], channels_last=True)
    for k in GRADS:
        a = gc[k]
        if k in ("du", "ddelta", "dz"):
            a = a.transpose(1, 2)
        elif k in ("dB", "dC"):
            a = from_cl_bc(a)
        assert torch.equal(a, gd[k]), k
