"""Decode step (ssm_state_update): CUDA library against the fp64 oracle recurrence step by step,
and against the library's own forward scan over the same tokens."""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_23_b200 as ssm
from selective_state_space_23_b200.inputs import make_inputs, workload

from _parity import assert_close, f64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def step_inputs(w, seed, t, gate=True):
    return make_inputs(w, seed=seed, step=t, gate=gate)


@pytest.mark.parametrize("io,N", [(torch.float32, 16), (torch.bfloat16, 16), (torch.bfloat16, 5),
                                  (torch.float32, 3)])
def test_steps_match_oracle(io, N):
    w = workload("decode_b256", batch=3, dim=70, dstate=N, io_dtype=io)
    r = np.random.default_rng(0)
    state0 = (0.5 * r.standard_normal((3, 70, N))).astype(np.float32)
    state = torch.from_numpy(state0).to(DEV)
    ref_state = state0.astype(np.float64).copy()
    for t in range(24):
        x = step_inputs(w, 1, t)
        xd = {k: v.to(DEV) for k, v in x.items()}
        out = ssm.ssm_state_update(state, xd["x"], xd["dt"], xd["A"], xd["B"], xd["C"], D=xd["D"],
                                   z=xd["z"], dt_bias=xd["dt_bias"])
        ro = oracle.state_update(ref_state, f64(x["x"]), f64(x["dt"]), f64(x["A"]), f64(x["B"]),
                                 f64(x["C"]), D=f64(x["D"]), z=f64(x["z"]), dt_bias=f64(x["dt_bias"]))
        assert_close(out, ro, io, f"out step {t}")
        assert_close(state, ref_state, torch.float32 if io == torch.float32 else io, f"state {t}")


def test_decode_equals_scan():
    """L decode steps reproduce the forward scan over the same L tokens (P-decode)."""
    w = workload("mamba370m_fwd", batch=2, dim=96, seqlen=48)
    x = {k: v.to(DEV) for k, v in make_inputs(w, seed=2, with_h0=True).items()}
    out_scan, hL = ssm.ssm_scan_fwd(x["u"], x["delta"], x["A"], x["B"], x["C"], D=x["D"], z=x["z"],
                                    dt_bias=x["dt_bias"], h0=x["h0"], return_final_state=True)
    state = x["h0"].clone()
    outs = []
    for t in range(48):
        outs.append(ssm.ssm_state_update(
            state, x["u"][..., t].contiguous(), x["delta"][..., t].contiguous(), x["A"],
            x["B"][..., t].contiguous(), x["C"][..., t].contiguous(), D=x["D"],
            z=x["z"][..., t].contiguous(), dt_bias=x["dt_bias"]))
    dec = torch.stack(outs, -1)
    assert_close(dec, f64(out_scan), torch.bfloat16, "decode vs scan")
    assert_close(state, f64(hL), torch.bfloat16, "state vs hL")


def test_no_gate_no_softplus():
    w = workload("decode_b256", batch=4, dim=64, io_dtype=torch.float32)
    x = step_inputs(w, 3, 0, gate=False)
    x["dt"] = x["dt"].abs() * 0.1 + 1e-3
    state0 = np.zeros((4, 64, 16))
    st = torch.zeros((4, 64, 16), device=DEV)
    xd = {k: v.to(DEV) for k, v in x.items()}
    out = ssm.ssm_state_update(st, xd["x"], xd["dt"], xd["A"], xd["B"], xd["C"], delta_softplus=False)
    ro = oracle.state_update(state0, f64(x["x"]), f64(x["dt"]), f64(x["A"]), f64(x["B"]), f64(x["C"]),
                             delta_softplus=False)
    assert_close(out, ro, torch.float32, "out")
    assert_close(st, state0, torch.float32, "state")


@pytest.mark.slow
def test_decode_b256_workload_sampled_channels():
    """256 x 5120 x 16 state, 1024 consecutive steps; 64 channels followed step by step."""
    w = workload("decode_b256")
    steps = w.steps
    sel_b = torch.tensor([0, 37, 128, 255])
    sel_d = torch.tensor(list(range(0, 5120, 320)))      # 16 d per batch row -> 64 channels
    state = torch.zeros((256, 5120, 16), device=DEV)
    ref_state = np.zeros((4, 16, 16))
    prm = make_inputs(w, seed=0, step=0)
    A = prm["A"].to(DEV); D = prm["D"].to(DEV); bias = prm["dt_bias"].to(DEV)
    A_s = f64(prm["A"][sel_d]); D_s = f64(prm["D"][sel_d]); b_s = f64(prm["dt_bias"][sel_d])
    for t in range(steps):
        x = make_inputs(w, seed=0, step=t)
        xd = {k: v.to(DEV, non_blocking=True) for k, v in x.items() if k in ("x", "dt", "z", "B", "C")}
        out = ssm.ssm_state_update(state, xd["x"], xd["dt"], A, xd["B"], xd["C"], D=D, z=xd["z"],
                                   dt_bias=bias)
        sub = lambda k: f64(x[k][sel_b][:, sel_d])
        ro = oracle.state_update(ref_state, sub("x"), sub("dt"), A_s, f64(x["B"][sel_b]),
                                 f64(x["C"][sel_b]), D=D_s, z=sub("z"), dt_bias=b_s)
        if t % 64 == 0 or t == steps - 1:
            assert_close(out[sel_b][:, sel_d.to(DEV)], ro, torch.bfloat16, f"out {t}")
            assert_close(state[sel_b][:, sel_d.to(DEV)], ref_state, torch.bfloat16, f"state {t}")


@pytest.mark.parametrize("io", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("variant", ["plain", "no_gate", "groups", "scalar_a", "zoh"])
def test_streamed_decode_matches_oracle_and_per_thread_form(monkeypatch, io, variant):
    """dim a multiple of 128 with N = 16 takes the streamed form (bulk copies of 128-channel
    tiles through a shared-memory ring): step by step against the oracle, bitwise against the
    per-thread form (the same arithmetic), and no bounded wait ran out."""
    from selective_state_space_23_b200 import _abi
    batch, dim, N = 7, 384, 16
    groups = 3 if variant == "groups" else 1
    w = workload("decode_b256", batch=batch * groups, dim=dim, dstate=N, io_dtype=io)
    r = np.random.default_rng(5)
    state0 = (0.5 * r.standard_normal((batch, dim, N))).astype(np.float32)
    st_a = torch.from_numpy(state0).to(DEV)
    st_b = st_a.clone()
    ref = state0.astype(np.float64).copy()
    kw = dict(scalar_a=variant == "scalar_a", zoh=variant == "zoh")
    for t in range(12):
        x = make_inputs(w, seed=7, step=t, gate=variant != "no_gate", scalar_a=kw["scalar_a"])
        x = {k: (v[:batch] if k in ("x", "dt", "z") else v) for k, v in x.items()}
        if groups > 1:  # [batch, G, N]: draw G rows of B, C per batch row
            x["B"] = x["B"].reshape(batch, groups, N)
            x["C"] = x["C"].reshape(batch, groups, N)
        else:
            x["B"], x["C"] = x["B"][:batch], x["C"][:batch]
        xd = {k: v.to(DEV) for k, v in x.items()}
        monkeypatch.delenv("SSM_DECODE_STREAM", raising=False)
        out_a = ssm.ssm_state_update(st_a, xd["x"], xd["dt"], xd["A"], xd["B"], xd["C"], D=xd["D"],
                                     z=xd.get("z"), dt_bias=xd["dt_bias"], **kw)
        monkeypatch.setenv("SSM_DECODE_STREAM", "0")
        out_b = ssm.ssm_state_update(st_b, xd["x"], xd["dt"], xd["A"], xd["B"], xd["C"], D=xd["D"],
                                     z=xd.get("z"), dt_bias=xd["dt_bias"], **kw)
        A_ref = f64(x["A"])
        if kw["scalar_a"]:
            A_ref = np.repeat(A_ref[:, None], N, axis=1)
        ro = oracle.state_update(ref, f64(x["x"]), f64(x["dt"]), A_ref, f64(x["B"]), f64(x["C"]),
                                 D=f64(x["D"]), z=None if "z" not in x else f64(x["z"]),
                                 dt_bias=f64(x["dt_bias"]), zoh=kw["zoh"])
        assert torch.equal(out_a, out_b) and torch.equal(st_a, st_b), f"step {t}"
        assert_close(out_a, ro, io, f"out step {t}")
        assert_close(st_a, ref, torch.float32 if io == torch.float32 else io, f"state step {t}")
    assert _abi.wait_timeouts() == 0
