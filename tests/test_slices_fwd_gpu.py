"""The f32 forward of the scalar-decay scan with N = 32 to 128 in steps of 16 (64 and 128 are the
Mamba-2 state sizes of the "2024 Reading List: Neural Network" page), run as the sum of 16-state
forwards over slices of the state: with one decay rate per channel the states of the recurrence
(Mamba paper, Section 3.2, eq. 2a-2b) do not interact, and the gate multiplies the whole
readout, so the output is the sum of the slices' gated outputs.  Compared with the fp64 oracle at the f32 tolerance, in every
variant; final states and checkpoints are checked slice by slice against the 16-state call on
the same slice, bitwise."""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_23_b200 as ssm
from selective_state_space_23_b200.inputs import make_inputs, workload

from _parity import assert_close, f64

pytestmark = pytest.mark.gpu
DEV = "cuda"
F32 = torch.float32


def inputs(batch, dim, L, N, seed, groups=1, gate=True):
    w = workload("mamba370m_fwd", batch=batch, dim=dim, seqlen=L, dstate=N, io_dtype=F32)
    x = make_inputs(w, seed=seed, with_dout=True, with_h0=True, scalar_a=True, gate=gate)
    if groups > 1:
        wg = workload("mamba370m_fwd", batch=batch * groups, dim=1, seqlen=L, dstate=N, io_dtype=F32)
        xg = make_inputs(wg, seed=seed + 1)
        x["B"] = xg["B"].reshape(batch, groups, N, L).contiguous()
        x["C"] = xg["C"].reshape(batch, groups, N, L).contiguous()
    return x


def gpu(x, B=None, C=None, h0=None, **kw):
    xd = {k: v.to(DEV) for k, v in x.items()}
    return ssm.ssm_scan_fwd_scalar_a(xd["u"], xd["delta"], xd["A"],
                                     xd["B"] if B is None else B, xd["C"] if C is None else C,
                                     D=xd.get("D"), z=xd.get("z"), dt_bias=xd.get("dt_bias"),
                                     h0=xd.get("h0") if h0 is None else h0, **kw)


def ref(x, **kw):
    c = lambda k: None if x.get(k) is None else f64(x[k])
    N = x["B"].shape[-2]
    A = np.repeat(c("A")[:, None], N, axis=1)
    return oracle.scan_fwd(c("u"), c("delta"), A, c("B"), c("C"), D=c("D"), z=c("z"),
                           dt_bias=c("dt_bias"), h0=c("h0"), **kw)


@pytest.mark.parametrize("N", [32, 48, 64, 96, 128])
@pytest.mark.parametrize("shape", [(2, 64, 160), (1, 40, 45), (2, 24, 17)])
def test_matches_oracle(N, shape):
    """Ragged time tails (45, 17 steps) and channel counts that fill no whole tile; any multiple
    of 16 states up to 128."""
    batch, dim, L = shape
    x = inputs(batch, dim, L, N, seed=211)
    out, hL = gpu(x, return_final_state=True)
    r = ref(x)
    assert_close(out, r["out"], F32, "out")
    assert_close(hL, r["hL"], F32, "hL")


@pytest.mark.parametrize("variant", ["reverse", "zoh", "reverse_zoh", "groups", "no_gate"])
def test_variants_match_oracle(variant):
    kw = dict(reverse=variant.startswith("reverse"), zoh=variant.endswith("zoh"))
    x = inputs(2, 64, 96, 64, seed=212, groups=2 if variant == "groups" else 1,
               gate=variant != "no_gate")
    if variant == "no_gate":
        del x["D"]
    out, hL = gpu(x, return_final_state=True, **kw)
    r = ref(x, **kw)
    assert_close(out, r["out"], F32, "out")
    assert_close(hL, r["hL"], F32, "hL")


@pytest.mark.parametrize("reverse", [False, True])
def test_slices_equal_the_16_state_calls(reverse):
    """Each 16-state slice of hL and of the checkpoints is, bit for bit, what the 16-state call
    on that slice of B, C, h0 returns; the output is the f32 sum of the slices' outputs (D in
    the first slice only)."""
    N, L = 64, 70
    x = inputs(2, 48, L, N, seed=213)
    xd = {k: v.to(DEV) for k, v in x.items()}
    out, hL, ck = gpu(x, return_final_state=True, return_ckpt=True, reverse=reverse)
    assert ck.shape == (2, 48, (L + 15) // 16, N)
    acc = torch.zeros_like(out)
    for j in range(N // 16):
        sl = slice(16 * j, 16 * j + 16)
        o, h, c = ssm.ssm_scan_fwd_scalar_a(
            xd["u"], xd["delta"], xd["A"], xd["B"][:, sl].contiguous(),
            xd["C"][:, sl].contiguous(), D=xd["D"] if j == 0 else None, z=xd["z"],
            dt_bias=xd["dt_bias"], h0=xd["h0"][..., sl].contiguous(), return_final_state=True,
            return_ckpt=True, reverse=reverse)
        assert torch.equal(hL[..., sl], h), f"hL slice {j}"
        assert torch.equal(ck[..., sl], c), f"checkpoint slice {j}"
        acc += o
    torch.testing.assert_close(out, acc, rtol=1e-6, atol=1e-6)


def test_checkpoints_are_block_entry_states():
    """Checkpoint k is the state entering step 16 k: h0, then the oracle's final state of each
    prefix."""
    N, L = 32, 50
    x = inputs(1, 24, L, N, seed=214)
    _, ck = gpu(x, return_ckpt=True)
    c = lambda k: f64(x[k])
    A = np.repeat(c("A")[:, None], N, axis=1)
    for k in range(ck.shape[2]):
        t = 16 * k
        if t == 0:
            h = c("h0")
        else:
            h = oracle.scan_fwd(c("u")[..., :t], c("delta")[..., :t], A, c("B")[..., :t],
                                c("C")[..., :t], D=c("D"), z=c("z")[..., :t],
                                dt_bias=c("dt_bias"), h0=c("h0"))["hL"]
        assert_close(ck[:, :, k, :], h, F32, f"checkpoint {k}")


def test_forward_and_backward_pair_in_f32():
    """A training step in f32 with N = 64: the forward above and the slice backward, both against
    the oracle."""
    N = 64
    x = inputs(1, 32, 80, N, seed=215)
    xd = {k: v.to(DEV) for k, v in x.items()}
    out = gpu(x)
    g = ssm.ssm_scan_bwd_scalar_a(xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"], xd["dout"],
                                  D=xd["D"], z=xd["z"], dt_bias=xd["dt_bias"], h0=xd["h0"])
    c = lambda k: f64(x[k])
    A = np.repeat(c("A")[:, None], N, axis=1)
    assert_close(out, ref(x)["out"], F32, "out")
    r = oracle.scan_bwd(c("u"), c("delta"), A, c("B"), c("C"), c("dout"), D=c("D"), z=c("z"),
                        dt_bias=c("dt_bias"), h0=c("h0"))
    r["dA"] = r["dA"].sum(1)
    for k in ("du", "ddelta", "dz", "dB", "dC", "dA", "dD", "ddt_bias", "dh0"):
        assert_close(g[k], r[k], F32, k)


def test_refusals():
    """The channels-last layout and a state size above 16 that is no multiple of 16 are refused
    on the host."""
    x = inputs(1, 32, 32, 64, seed=216)
    xd = {k: v.to(DEV) for k, v in x.items()}
    ucl = xd["u"].transpose(1, 2).contiguous()
    with pytest.raises(RuntimeError):
        ssm.ssm_scan_fwd_scalar_a(ucl, xd["delta"].transpose(1, 2).contiguous(), xd["A"],
                                  xd["B"].transpose(1, 2).contiguous(),
                                  xd["C"].transpose(1, 2).contiguous(), channels_last=True)
    y = inputs(1, 32, 32, 40, seed=217)
    with pytest.raises(RuntimeError):
        gpu(y)


@pytest.mark.parametrize("shape", [(1, 1, 1), (1, 3, 2), (1, 16, 4000)])
def test_edge_shapes(shape):
    """One step, one channel, and few channels over a long sequence (the 16-state forward then
    splits time inside each slice's call)."""
    batch, dim, L = shape
    x = inputs(batch, dim, L, 64, seed=218)
    out, hL = gpu(x, return_final_state=True)
    r = ref(x)
    assert_close(out, r["out"], F32, "out")
    assert_close(hL, r["hL"], F32, "hL")
