"""ssm_scan_fwd_noalloc: the forward scan for callers that cannot allocate device memory (their
memory is fully planned in advance, or cudaMalloc on their hot path would stall the device).
It takes its time-split scratch from a static device array inside the library instead of a
workspace.  Checked through the C ABI against the workspace-taking ssm_scan_fwd on the same
inputs, on two calls in a row (the second call reuses whatever the first left in the array).

This file is named so that pytest collects it last."""
import ctypes

import pytest
import torch

import selective_state_space_23_b200 as ssm
from selective_state_space_23_b200 import _abi
from selective_state_space_23_b200.inputs import make_inputs, workload

from _parity import assert_close, f64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _noalloc(x, out, hL, batch, dim, L, N, io_code):
    return _abi.lib().ssm_scan_fwd_noalloc(
        _p(x["u"]), _p(x["delta"]), _p(x["A"]), _p(x["B"]), _p(x["C"]), _p(x["D"]), _p(x["z"]),
        _p(x["dt_bias"]), 1, _p(x.get("h0")), _p(hL), _p(out), None, batch, dim, L, N, io_code,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("io", [torch.bfloat16, torch.float32])
def test_noalloc_matches_workspace_entry_point_twice(monkeypatch, io):
    """Two calls in a row with different time splits and lengths: the second call's chunk
    boundaries move, so words the first call left in the array lie under the second call's
    reads; the second call must write every word it reads first."""
    batch, dim, N = 1, 64, 16                    # few channels: the plan splits time
    code = _abi.SSM_BF16 if io == torch.bfloat16 else _abi.SSM_F32
    for call, (seed, L, split) in enumerate(((11, 16384, "16"), (12, 12000, "3"))):
        monkeypatch.setenv("SSM_FWD_SPLIT", split)
        need = ssm.fwd_workspace_bytes(batch, dim, L, N, io)
        assert 0 < need <= _abi.NOALLOC_SCRATCH_BYTES
        w = workload("long_seq_1m", batch=batch, dim=dim, seqlen=L, dstate=N, io_dtype=io)
        x = {k: v.to(DEV) for k, v in make_inputs(w, seed=seed, with_h0=True).items()}
        ref, ref_hL = ssm.ssm_scan_fwd(x["u"], x["delta"], x["A"], x["B"], x["C"], D=x["D"], z=x["z"],
                                       dt_bias=x["dt_bias"], h0=x["h0"], return_final_state=True)
        out = torch.empty_like(x["u"])
        hL = torch.empty_like(x["h0"])
        rc = _noalloc(x, out, hL, batch, dim, L, N, code)
        assert rc == _abi.SSM_OK, _abi.last_error()
        torch.cuda.synchronize()
        assert_close(out, f64(ref), io, f"out, call {call}")
        assert_close(hL, f64(ref_hL), torch.float32 if io == torch.float32 else io, f"hL, call {call}")


def test_noalloc_rejects_plans_larger_than_the_static_array(monkeypatch):
    # forcing 8 chunks on 16384 channels asks for ~17 MB of scratch: refused before any launch
    monkeypatch.setenv("SSM_FWD_SPLIT", "8")
    batch, dim, L, N = 8, 2048, 2048, 16
    assert ssm.fwd_workspace_bytes(batch, dim, L, N, torch.bfloat16) > _abi.NOALLOC_SCRATCH_BYTES
    u = torch.empty((batch, dim, L), dtype=torch.bfloat16, device=DEV)
    rc = _abi.lib().ssm_scan_fwd_noalloc(_p(u), *([None] * 7), 1, *([None] * 4), batch, dim, L, N,
                                         _abi.SSM_BF16, None)
    assert rc == _abi.SSM_EUNSUPPORTED
    assert b"scratch" in _abi.lib().ssm_last_error()
