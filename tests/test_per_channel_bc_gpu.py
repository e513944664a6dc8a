"""B and C per channel (bc_groups == dim: B, C of shape [batch, dim, N, L]), CUDA library against
the fp64 oracle run with one B/C group per channel ("Seçim Mekanizması (S6)" on the Mamba summary
page: B_t and C_t are functions of the input; computed per channel they are per-channel rows):
forward, backward and the decode step, with ragged lengths, N < 16 and the options."""
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


def per_channel_inputs(batch, dim, L, N, io, seed, with_dout=False, gate=True):
    """Shared-layout inputs with B, C redrawn per channel: [batch, dim, N, L]."""
    w = workload("tiny_f32", batch=batch, dim=dim, seqlen=L, dstate=N, io_dtype=io)
    x = make_inputs(w, seed=seed, with_h0=True, with_dout=with_dout, gate=gate)
    wb = workload("tiny_f32", batch=batch * dim, dim=1, seqlen=L, dstate=N, io_dtype=io)
    xb = make_inputs(wb, seed=seed + 1000)
    x["B"] = xb["B"].reshape(batch, dim, N, L).contiguous()
    x["C"] = xb["C"].reshape(batch, dim, N, L).contiguous()
    return x


def c64(x, k):
    return None if x.get(k) is None else f64(x[k])


@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("shape", [(2, 40, 333, 16), (1, 3, 17, 5), (2, 16, 256, 16), (1, 7, 1, 3)])
def test_forward_matches_oracle(io, shape):
    batch, dim, L, N = shape
    x = per_channel_inputs(batch, dim, L, N, io, seed=81)
    xd = {k: v.to(DEV) for k, v in x.items()}
    out, hL, ck = ssm.ssm_scan_fwd(xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"], D=xd["D"],
                                   z=xd["z"], dt_bias=xd["dt_bias"], h0=xd["h0"],
                                   return_final_state=True, return_ckpt=True)
    ref = oracle.scan_fwd(c64(x, "u"), c64(x, "delta"), c64(x, "A"), c64(x, "B"), c64(x, "C"),
                          D=c64(x, "D"), z=c64(x, "z"), dt_bias=c64(x, "dt_bias"), h0=c64(x, "h0"))
    assert_close(out, ref["out"], io, "out")
    assert_close(hL, ref["hL"], io, "hL")
    # checkpoints are the states entering every 16-step block
    np.testing.assert_array_equal(f64(ck)[:, :, 0], f64(x["h0"]))
    for k in range(1, (L + 15) // 16):
        pre = {kk: (v[..., :16 * k] if kk in ("u", "delta", "z", "B", "C") else v) for kk, v in x.items()}
        r = oracle.scan_fwd(c64(pre, "u"), c64(pre, "delta"), c64(pre, "A"), c64(pre, "B"),
                            c64(pre, "C"), D=c64(pre, "D"), z=c64(pre, "z"),
                            dt_bias=c64(pre, "dt_bias"), h0=c64(pre, "h0"))
        assert_close(f64(ck)[:, :, k], r["hL"], io, f"ckpt {k}")


@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
def test_forward_without_gate_bias_softplus(io):
    x = per_channel_inputs(2, 24, 200, 16, io, seed=82, gate=False)
    x["delta"] = (x["delta"].float().abs() * 0.05 + 1e-3).to(io)
    del x["dt_bias"], x["D"]
    xd = {k: v.to(DEV) for k, v in x.items()}
    out = ssm.ssm_scan_fwd(xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"], h0=xd["h0"],
                           delta_softplus=False)
    ref = oracle.scan_fwd(c64(x, "u"), c64(x, "delta"), c64(x, "A"), c64(x, "B"), c64(x, "C"),
                          h0=c64(x, "h0"), delta_softplus=False)
    assert_close(out, ref["out"], io, "out")


@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("shape,use_ckpt", [((2, 40, 333, 16), False), ((2, 40, 333, 16), True),
                                            ((1, 5, 37, 5), False), ((1, 16, 64, 16), True)])
def test_backward_matches_oracle(io, shape, use_ckpt):
    batch, dim, L, N = shape
    x = per_channel_inputs(batch, dim, L, N, io, seed=83, with_dout=True)
    xd = {k: v.to(DEV) for k, v in x.items()}
    dhL = torch.randn((batch, dim, N), generator=torch.Generator().manual_seed(3))
    ck = None
    if use_ckpt:
        _, ck = ssm.ssm_scan_fwd(xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"], D=xd["D"],
                                 z=xd["z"], dt_bias=xd["dt_bias"], h0=xd["h0"], return_ckpt=True)
    g = ssm.ssm_scan_bwd(xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"], xd["dout"], D=xd["D"],
                         z=xd["z"], dt_bias=xd["dt_bias"], h0=xd["h0"], dhL=dhL.to(DEV), ckpt=ck)
    r = oracle.scan_bwd(c64(x, "u"), c64(x, "delta"), c64(x, "A"), c64(x, "B"), c64(x, "C"),
                        c64(x, "dout"), D=c64(x, "D"), z=c64(x, "z"), dt_bias=c64(x, "dt_bias"),
                        h0=c64(x, "h0"), dhL=f64(dhL))
    assert g["dB"].shape == (batch, dim, N, L)
    for k in GRADS:
        assert_close(g[k], r[k], io, k)


@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
def test_decode_steps_match_oracle(io):
    batch, dim, N = 3, 40, 16
    w = workload("decode_b256", batch=batch * dim, dim=dim, dstate=N, io_dtype=io)
    r = np.random.default_rng(4)
    state0 = (0.5 * r.standard_normal((batch, dim, N))).astype(np.float32)
    state = torch.from_numpy(state0).to(DEV)
    ref = state0.astype(np.float64).copy()
    for t in range(10):
        x = make_inputs(w, seed=84, step=t)
        x = {k: (v[:batch] if k in ("x", "dt", "z") else v) for k, v in x.items()}
        x["B"] = x["B"].reshape(batch, dim, N)
        x["C"] = x["C"].reshape(batch, dim, N)
        xd = {k: v.to(DEV) for k, v in x.items()}
        out = ssm.ssm_state_update(state, xd["x"], xd["dt"], xd["A"], xd["B"], xd["C"], D=xd["D"],
                                   z=xd["z"], dt_bias=xd["dt_bias"])
        ro = oracle.state_update(ref, f64(x["x"]), f64(x["dt"]), f64(x["A"]), f64(x["B"]),
                                 f64(x["C"]), D=f64(x["D"]), z=f64(x["z"]),
                                 dt_bias=f64(x["dt_bias"]))
        assert_close(out, ro, io, f"out step {t}")
        assert_close(state, ref, io, f"state step {t}")


def test_other_variant_flags_are_refused():
    x = per_channel_inputs(1, 16, 32, 16, torch.bfloat16, seed=85)
    xd = {k: v.to(DEV) for k, v in x.items()}
    with pytest.raises(RuntimeError):
        ssm.ssm_scan_fwd(xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"], reverse=True)
