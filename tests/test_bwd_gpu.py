"""Backward pass: CUDA library gradients against the fp64 oracle's chain-rule gradients (which
are themselves pinned by finite differences in test_oracle_pins.py)."""
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


def gpu_grads(x, softplus=True, use_ckpt=False, dhL=None):
    ck = None
    if use_ckpt:
        _, ck = ssm.ssm_scan_fwd(x["u"], x["delta"], x["A"], x["B"], x["C"], D=x.get("D"),
                                 z=x.get("z"), dt_bias=x.get("dt_bias"), delta_softplus=softplus,
                                 h0=x.get("h0"), return_ckpt=True)
    return ssm.ssm_scan_bwd(x["u"], x["delta"], x["A"], x["B"], x["C"], x["dout"], D=x.get("D"),
                            z=x.get("z"), dt_bias=x.get("dt_bias"), delta_softplus=softplus,
                            h0=x.get("h0"), dhL=dhL, ckpt=ck)


def oracle_grads(x, softplus=True, dhL=None, channels=None):
    c = lambda k: None if x.get(k) is None else f64(x[k])
    return oracle.scan_bwd(c("u"), c("delta"), c("A"), c("B"), c("C"), c("dout"), D=c("D"),
                           z=c("z"), dt_bias=c("dt_bias"), delta_softplus=softplus, h0=c("h0"),
                           dhL=None if dhL is None else f64(dhL), channels=channels)


def compare(g, r, io, names=GRADS):
    for k in names:
        if r.get(k) is None or g.get(k) is None:
            continue
        tol_io = io if k in ("du", "ddelta", "dz", "dB", "dC") or io == torch.float32 else io
        assert_close(g[k], r[k], tol_io, k)


@pytest.mark.parametrize("use_ckpt", [False, True])
def test_tiny_f32_all_gradients(use_ckpt):
    w = workload("tiny_f32", batch=2, dim=64, seqlen=256)
    x = make_inputs(w, seed=0, with_dout=True, with_h0=True)
    dhL = torch.randn((2, 64, 16), generator=torch.Generator().manual_seed(1))
    g = gpu_grads(on_dev(x), use_ckpt=use_ckpt, dhL=dhL.to(DEV))
    r = oracle_grads(x, dhL=dhL)
    compare(g, r, torch.float32)


@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("shape", [(1, 40, 37, 5), (2, 100, 250, 16), (1, 1, 1, 1)])
def test_ragged_shapes(io, shape):
    batch, dim, L, N = shape
    w = workload("tiny_f32", batch=batch, dim=dim, seqlen=L, dstate=N, io_dtype=io)
    x = make_inputs(w, seed=2, with_dout=True, with_h0=True)
    g = gpu_grads(on_dev(x))
    r = oracle_grads(x)
    compare(g, r, io)


@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
def test_no_gate_no_softplus(io):
    w = workload("tiny_f32", batch=2, dim=64, seqlen=128, io_dtype=io)
    x = make_inputs(w, seed=3, with_dout=True, gate=False)
    x["delta"] = (x["delta"].float().abs() * 0.05 + 1e-3).to(io)   # positive steps, no bias
    del x["dt_bias"]
    g = gpu_grads(on_dev(x), softplus=False)
    assert g["dz"] is None
    r = oracle_grads(x, softplus=False)
    compare(g, r, io)


def test_bf16_medium_all_gradients():
    w = workload("mamba2p8b_train", batch=2, dim=256, seqlen=512)
    x = make_inputs(w, seed=4, with_dout=True)
    g = gpu_grads(on_dev(x), use_ckpt=True)
    r = oracle_grads(x)
    compare(g, r, torch.bfloat16)


def test_deterministic_bitwise():
    w = workload("mamba2p8b_train", batch=2, dim=128, seqlen=256)
    x = on_dev(make_inputs(w, seed=5, with_dout=True))
    a = gpu_grads(x)
    b = gpu_grads(x)
    for k in GRADS:
        if a[k] is not None:
            assert torch.equal(a[k], b[k]), k


def test_workspace_too_small_is_an_error():
    w = workload("mamba2p8b_train", batch=1, dim=64, seqlen=64)
    x = on_dev(make_inputs(w, seed=6, with_dout=True))
    ws = torch.empty(64, dtype=torch.uint8, device=DEV)
    with pytest.raises(ValueError):
        ssm.ssm_scan_bwd(x["u"], x["delta"], x["A"], x["B"], x["C"], x["dout"], workspace=ws)


@pytest.mark.slow
def test_mamba2p8b_train_step_full_size():
    """4 x 5120 x 2048 (the training-step workload): per-channel gradients on 64 sampled d of
    every batch row (dA, dD, ddt_bias of those d are then complete sums); dB, dC of batch row 0
    against a full fp64 sum over all 5120 channels."""
    w = workload("mamba2p8b_train")
    x = make_inputs(w, seed=0, with_dout=True)
    g = gpu_grads(on_dev(x), use_ckpt=True)
    torch.cuda.synchronize()
    sel = list(range(0, 5120, 80))
    chans = [b * 5120 + d for b in range(4) for d in sel]
    r = oracle_grads(x, channels=chans)
    idx = torch.as_tensor(sel)
    for k in ("du", "ddelta", "dz", "dh0"):
        assert_close(g[k].index_select(1, idx.to(DEV)), r[k][:, sel], torch.bfloat16, k)
    for k in ("dA", "dD", "ddt_bias"):
        assert_close(g[k].index_select(0, idx.to(DEV)), r[k][sel], torch.bfloat16, k)
    r0 = oracle_grads(x, channels=list(range(5120)))  # batch row 0, every channel
    for k in ("dB", "dC"):
        assert_close(g[k][0], r0[k][0], torch.bfloat16, k)


@pytest.mark.parametrize("fwd_kernel", ["pair", "lane"])
@pytest.mark.parametrize("bwd_kernel", ["pair", "hist"])
def test_kernel_families(monkeypatch, fwd_kernel, bwd_kernel):
    """Every pairing of the forward kernel that writes the checkpoints (or replays the states
    when none are given) with the backward kernel that consumes them: the one-lane-per-channel
    or two-lanes-per-channel forward, and the register-history or general backward."""
    monkeypatch.setenv("SSM_FWD_KERNEL", fwd_kernel)
    if bwd_kernel == "pair":
        monkeypatch.setenv("SSM_BWD_KERNEL", "pair")
    else:
        monkeypatch.delenv("SSM_BWD_KERNEL", raising=False)
    w = workload("mamba2p8b_train", batch=2, dim=96, seqlen=312)
    x = make_inputs(w, seed=14, with_dout=True, with_h0=True)
    r = oracle_grads(x)
    for use_ckpt in (False, True):
        compare(gpu_grads(on_dev(x), use_ckpt=use_ckpt), r, torch.bfloat16)
