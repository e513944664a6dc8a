"""ssm_scan_fwd_host (inputs and outputs in host memory, copies and scan pipelined over batch
rows on three streams) against ssm_scan_fwd on device copies of the inputs, for chunked and
ragged batches, with and without a gate and initial/final states, in pinned and pageable host
memory, and ordered after earlier work on the caller's stream.  A chunk of few rows may take the
time split where the whole batch does not (or with another chunk count), which changes the
rounding: results are compared element by element within a few bf16 steps (a stale, missing or
misplaced chunk is far outside that), and bitwise on a shape that neither path splits."""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_23_b200 as ssm
from selective_state_space_23_b200.inputs import make_inputs, workload

from _parity import assert_close, f64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def device_result(x, **kw):
    xd = {k: v.to(DEV) for k, v in x.items()}
    return ssm.ssm_scan_fwd(xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"], D=xd.get("D"),
                            z=xd.get("z"), dt_bias=xd.get("dt_bias"), h0=xd.get("h0"), **kw)


def host_result(x, pin, **kw):
    h = {k: (v.pin_memory() if pin else v.contiguous()) for k, v in x.items()
         if k in ("u", "delta", "z", "B", "C", "h0")}
    r = ssm.ssm_scan_fwd_host(h["u"], h["delta"], x["A"].to(DEV), h["B"], h["C"],
                              D=x["D"].to(DEV) if "D" in x else None, z=h.get("z"),
                              dt_bias=x["dt_bias"].to(DEV) if "dt_bias" in x else None,
                              h0=h.get("h0"), **kw)
    torch.cuda.synchronize()
    return r


def near(a, b, io):
    """Element-wise agreement within a few steps of the io type's rounding."""
    a, b = a.double(), b.double().cpu()
    step = 2.0 ** -7 if io == torch.bfloat16 else 2.0 ** -18
    assert torch.all((a - b).abs() <= step * b.abs() + step * 1e-2), float((a - b).abs().max())


@pytest.mark.parametrize("pin", [True, False])
@pytest.mark.parametrize("batch,dim,L,io", [(20, 64, 300, torch.bfloat16), (5, 48, 64, torch.float32),
                                            (1, 16, 17, torch.bfloat16), (9, 128, 1024, torch.bfloat16)])
def test_matches_device_call(pin, batch, dim, L, io):
    w = workload("tiny_f32", batch=batch, dim=dim, seqlen=L, io_dtype=io)
    x = make_inputs(w, seed=91, with_h0=True)
    out_d, hL_d = device_result(x, return_final_state=True)
    out_h, hL_h = host_result(x, pin, return_final_state=True)
    assert out_h.device.type == "cpu"
    near(out_h, out_d, io)
    near(hL_h, hL_d, torch.float32 if io == torch.float32 else io)
    c = lambda k: f64(x[k])
    ref = oracle.scan_fwd(c("u"), c("delta"), c("A"), c("B"), c("C"), D=c("D"), z=c("z"),
                          dt_bias=c("dt_bias"), h0=c("h0"))
    assert_close(out_h, ref["out"], io, "out")


def test_bitwise_when_no_time_split(monkeypatch):
    """Two rows of 5120 channels (the host call's chunk for a batch of 16) fill the GPU: no chunk
    and no full call splits time, so the host call and the device call run the same kernel
    launches on the same rows (the exponential split is pinned too)."""
    monkeypatch.setenv("SSM_FWD_KMUFU", "16")
    w = workload("mamba2p8b_train", batch=16, seqlen=256)
    x = make_inputs(w, seed=95)
    assert torch.equal(host_result(x, True), device_result(x).cpu())


def test_without_gate_and_states():
    w = workload("tiny_f32", batch=12, dim=32, seqlen=200, io_dtype=torch.bfloat16)
    x = make_inputs(w, seed=92, gate=False)
    near(host_result(x, True), device_result(x), torch.bfloat16)


def test_runs_after_earlier_work_on_the_stream():
    """Parameters written on the caller's stream just before the call are the ones used."""
    w = workload("tiny_f32", batch=8, dim=64, seqlen=256, io_dtype=torch.bfloat16)
    x = make_inputs(w, seed=93)
    h = {k: x[k].pin_memory() for k in ("u", "delta", "z", "B", "C")}
    A = torch.zeros_like(x["A"], device=DEV)
    A.copy_(x["A"].to(DEV))               # queued on the current stream
    D = torch.empty(64, device=DEV)
    D.fill_(0.0).add_(x["D"].to(DEV))     # queued on the current stream
    out = ssm.ssm_scan_fwd_host(h["u"], h["delta"], A, h["B"], h["C"], D=D, z=h["z"],
                                dt_bias=x["dt_bias"].to(DEV))
    torch.cuda.current_stream().synchronize()
    near(out, device_result(x), torch.bfloat16)


def test_workspace_too_small_is_refused():
    w = workload("tiny_f32", batch=4, dim=32, seqlen=64, io_dtype=torch.bfloat16)
    x = make_inputs(w, seed=94)
    h = {k: x[k].pin_memory() for k in ("u", "delta", "z", "B", "C")}
    small = torch.empty(256, dtype=torch.uint8, device=DEV)
    with pytest.raises(ValueError):
        ssm.ssm_scan_fwd_host(h["u"], h["delta"], x["A"].to(DEV), h["B"], h["C"], workspace=small)
