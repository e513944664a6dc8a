"""Decode step variants (ssm_state_update_ex): one decay rate per channel, the zero-order-hold
input coefficient, grouped B/C, and their combination, step by step against the fp64 oracle's
decode step (itself pinned to the oracle scan for each variant in test_oracle_pins.py), and L
decode steps against the CUDA scan with the same variant.  A reverse decode is refused."""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_23_b200 as ssm
from selective_state_space_23_b200.inputs import make_inputs, workload

from _parity import assert_close, f64

pytestmark = pytest.mark.gpu
DEV = "cuda"
CASES = [(True, False, 1), (False, True, 1), (False, False, 4), (True, True, 2)]


def step_inputs(batch, dim, steps, io, seed, scalar_a, groups):
    w = workload("decode_b256", batch=batch, dim=dim, io_dtype=io, steps=steps)
    xs = []
    for t in range(steps):
        x = make_inputs(w, seed=seed, step=t, scalar_a=scalar_a)
        if groups > 1:
            wg = workload("decode_b256", batch=batch * groups, dim=dim, io_dtype=io)
            xg = make_inputs(wg, seed=seed + 500, step=t)
            x["B"] = xg["B"].reshape(batch, groups, 16)
            x["C"] = xg["C"].reshape(batch, groups, 16)
        xs.append(x)
    return xs


def full_a(A, scalar_a, N=16):
    A = f64(A)
    return np.repeat(A[:, None], N, 1) if scalar_a else A


@pytest.mark.parametrize("scalar_a,zoh,groups", CASES)
@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
def test_steps_against_oracle(io, scalar_a, zoh, groups):
    batch, dim, steps = 3, 64, 12
    xs = step_inputs(batch, dim, steps, io, 61, scalar_a, groups)
    state = torch.randn((batch, dim, 16), generator=torch.Generator().manual_seed(3)) * 0.5
    ref_state = np.ascontiguousarray(f64(state))
    st = state.to(DEV)
    for t, x in enumerate(xs):
        xd = {k: v.to(DEV) for k, v in x.items()}
        out = ssm.ssm_state_update(st, xd["x"], xd["dt"], xd["A"], xd["B"], xd["C"], D=xd["D"],
                                   z=xd["z"], dt_bias=xd["dt_bias"], scalar_a=scalar_a, zoh=zoh)
        ref = oracle.state_update(ref_state, f64(x["x"]), f64(x["dt"]), full_a(x["A"], scalar_a),
                                  f64(x["B"]), f64(x["C"]), D=f64(x["D"]), z=f64(x["z"]),
                                  dt_bias=f64(x["dt_bias"]), zoh=zoh)
        assert_close(out, ref, io, f"out step {t}")
    assert_close(st, ref_state, torch.float32 if io == torch.float32 else io, "state")


@pytest.mark.parametrize("scalar_a,zoh,groups", CASES)
def test_decode_equals_scan(scalar_a, zoh, groups):
    batch, dim, L = 2, 64, 40
    xs = step_inputs(batch, dim, L, torch.float32, 62, scalar_a, groups)
    st = (torch.randn((batch, dim, 16), generator=torch.Generator().manual_seed(4)) * 0.5).to(DEV)
    h0 = st.clone()
    outs = []
    for x in xs:
        xd = {k: v.to(DEV) for k, v in x.items()}
        outs.append(ssm.ssm_state_update(st, xd["x"], xd["dt"], xd["A"], xd["B"], xd["C"],
                                         D=xd["D"], z=xd["z"], dt_bias=xd["dt_bias"],
                                         scalar_a=scalar_a, zoh=zoh))
    seq = lambda k: torch.stack([x[k] for x in xs], -1).contiguous().to(DEV)
    x0 = {k: v.to(DEV) for k, v in xs[0].items()}
    f = ssm.ssm_scan_fwd_scalar_a if scalar_a else ssm.ssm_scan_fwd
    out, hL = f(seq("x"), seq("dt"), x0["A"], seq("B"), seq("C"), D=x0["D"], z=seq("z"),
                dt_bias=x0["dt_bias"], h0=h0, zoh=zoh, return_final_state=True)
    assert_close(torch.stack(outs, -1), f64(out), torch.float32, "out")
    assert_close(st, f64(hL), torch.float32, "state")


def test_reverse_decode_is_refused():
    from selective_state_space_23_b200 import _abi
    st = torch.zeros((1, 16, 16), device=DEV)
    x = torch.zeros((1, 16), device=DEV)
    A = -torch.ones((16, 16), device=DEV)
    B = torch.zeros((1, 16), device=DEV)
    out = torch.empty((1, 16), device=DEV)
    p = lambda t: t.data_ptr()
    rc = _abi.lib().ssm_state_update_ex(p(st), p(x), p(x), p(A), p(B), p(B), None, None, None, 1,
                                        p(out), 1, 16, 16, 1, _abi.SSM_F32, _abi.SSM_REVERSE, None)
    assert rc == _abi.SSM_EINVAL


# ------------------------------------------------------------------ one rate, N = 32 .. 128
def step_inputs_n(batch, dim, steps, N, io, seed, groups=1):
    w = workload("decode_b256", batch=batch, dim=dim, io_dtype=io, steps=steps, dstate=N)
    xs = []
    for t in range(steps):
        x = make_inputs(w, seed=seed, step=t, scalar_a=True)
        if groups > 1:
            wg = workload("decode_b256", batch=batch * groups, dim=dim, io_dtype=io, dstate=N)
            xg = make_inputs(wg, seed=seed + 500, step=t)
            x["B"] = xg["B"].reshape(batch, groups, N)
            x["C"] = xg["C"].reshape(batch, groups, N)
        xs.append(x)
    return xs


@pytest.mark.parametrize("N", [32, 64, 128])
@pytest.mark.parametrize("zoh,groups", [(False, 1), (True, 1), (False, 2)])
@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
def test_large_n_steps_against_oracle(io, N, zoh, groups):
    """The decode step of a scan with one rate per channel and 32 to 128 states (Mamba-2's state
    sizes): step by step against the oracle's decode step."""
    batch, dim, steps = 3, 64, 8
    xs = step_inputs_n(batch, dim, steps, N, io, 63, groups)
    state = torch.randn((batch, dim, N), generator=torch.Generator().manual_seed(5)) * 0.5
    ref_state = np.ascontiguousarray(f64(state))
    st = state.to(DEV)
    for t, x in enumerate(xs):
        xd = {k: v.to(DEV) for k, v in x.items()}
        out = ssm.ssm_state_update(st, xd["x"], xd["dt"], xd["A"], xd["B"], xd["C"], D=xd["D"],
                                   z=xd["z"], dt_bias=xd["dt_bias"], scalar_a=True, zoh=zoh)
        ref = oracle.state_update(ref_state, f64(x["x"]), f64(x["dt"]), full_a(x["A"], True, N),
                                  f64(x["B"]), f64(x["C"]), D=f64(x["D"]), z=f64(x["z"]),
                                  dt_bias=f64(x["dt_bias"]), zoh=zoh)
        assert_close(out, ref, io, f"out step {t}")
    assert_close(st, ref_state, torch.float32 if io == torch.float32 else io, "state")


@pytest.mark.parametrize("N", [32, 64, 128])
@pytest.mark.parametrize("zoh", [False, True])
def test_large_n_decode_equals_chunked_scan(N, zoh):
    """L decode steps against the chunked-form scan of the same L steps (bf16 io): outputs and
    final state."""
    batch, dim, L = 2, 64, 48
    xs = step_inputs_n(batch, dim, L, N, torch.bfloat16, 64)
    st = (torch.randn((batch, dim, N), generator=torch.Generator().manual_seed(6)) * 0.5).to(DEV)
    h0 = st.clone()
    outs = []
    for x in xs:
        xd = {k: v.to(DEV) for k, v in x.items()}
        outs.append(ssm.ssm_state_update(st, xd["x"], xd["dt"], xd["A"], xd["B"], xd["C"],
                                         D=xd["D"], z=xd["z"], dt_bias=xd["dt_bias"],
                                         scalar_a=True, zoh=zoh))
    seq = lambda k: torch.stack([x[k] for x in xs], -1).contiguous().to(DEV)
    x0 = {k: v.to(DEV) for k, v in xs[0].items()}
    out, hL = ssm.ssm_scan_fwd_scalar_a(seq("x"), seq("dt"), x0["A"], seq("B"), seq("C"),
                                        D=x0["D"], z=seq("z"), dt_bias=x0["dt_bias"], h0=h0,
                                        zoh=zoh, return_final_state=True)
    assert_close(torch.stack(outs, -1), f64(out), torch.bfloat16, "out")
    assert_close(st, f64(hL), torch.bfloat16, "state")
