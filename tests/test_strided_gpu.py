"""General element strides: io tensors given as views (slices of a wider projection output,
transposed (B, L, D) views, B/C expanded over the batch with stride 0, strided outputs) through
the *_strided entry points.  Each result must equal the dense call on contiguous copies bitwise,
and the forward also matches the fp64 oracle ("Seçim Mekanizması (S6)": the selective
parameters are projections of the input, held in whatever layout the projection writes)."""
import pytest
import torch

import oracle
import selective_state_space_23_b200 as ssm
from selective_state_space_23_b200.inputs import make_inputs, workload

from _parity import assert_close, f64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def strided_copies(x, seed=0):
    """The same values as x, held in non-dense views."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    batch, dim, L = x["u"].shape
    io = x["u"].dtype
    out = {}
    # u and delta: the two halves of one [batch, 2 dim, L] projection output
    proj = torch.empty((batch, 2 * dim, L), dtype=io, device=DEV)
    proj[:, :dim] = x["u"].to(DEV)
    proj[:, dim:] = x["delta"].to(DEV)
    out["u"], out["delta"] = proj[:, :dim], proj[:, dim:]
    # z: a (B, L, D) buffer seen as [batch, dim, L]
    zt = x["z"].to(DEV).transpose(1, 2).contiguous()
    out["z"] = zt.transpose(1, 2)
    # B, C: every other time step of a buffer twice as long
    for k in ("B", "C"):
        wide = torch.randn(x[k].shape[:-1] + (2 * L,), generator=g).to(io).to(DEV)
        wide[..., ::2] = x[k].to(DEV)
        out[k] = wide[..., ::2]
    for k in ("A", "D", "dt_bias", "h0"):
        if x.get(k) is not None:
            out[k] = x[k].to(DEV)
    if "dout" in x:
        dt_ = torch.empty((batch, dim, L + 3), dtype=io, device=DEV)
        dt_[..., :L] = x["dout"].to(DEV)
        out["dout"] = dt_[..., :L]
    return out


@pytest.mark.parametrize("io", [torch.bfloat16, torch.float32])
def test_forward_strided_equals_dense_and_oracle(io):
    w = workload("mamba2p8b_train", batch=2, dim=80, seqlen=200, io_dtype=io)
    x = make_inputs(w, seed=81, with_h0=True)
    s = strided_copies(x, seed=1)
    assert not s["u"].is_contiguous() and not s["z"].is_contiguous() and not s["B"].is_contiguous()
    obuf = torch.zeros((2, 80, 256), dtype=io, device=DEV)
    out_view = obuf[..., 7:207]
    got, hL = ssm.ssm_scan_fwd_strided(s["u"], s["delta"], s["A"], s["B"], s["C"], D=s["D"],
                                       z=s["z"], dt_bias=s["dt_bias"], h0=s["h0"],
                                       return_final_state=True, out=out_view)
    xd = {k: v.to(DEV) for k, v in x.items()}
    ref, hL_ref = ssm.ssm_scan_fwd(xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"], D=xd["D"],
                                   z=xd["z"], dt_bias=xd["dt_bias"], h0=xd["h0"],
                                   return_final_state=True)
    assert torch.equal(got, ref) and torch.equal(hL, hL_ref)
    assert torch.count_nonzero(obuf[..., :7]) == 0 and torch.count_nonzero(obuf[..., 207:]) == 0
    c = lambda k: f64(x[k])
    r = oracle.scan_fwd(c("u"), c("delta"), c("A"), c("B"), c("C"), D=c("D"), z=c("z"),
                        dt_bias=c("dt_bias"), h0=c("h0"))
    assert_close(got, r["out"], io, "out")


def test_forward_bc_broadcast_over_batch():
    """B, C shared by every batch row: a [1, N, L] tensor expanded with batch stride 0."""
    w = workload("mamba2p8b_train", batch=3, dim=64, seqlen=160)
    x = make_inputs(w, seed=82)
    B1, C1 = x["B"][:1].to(DEV), x["C"][:1].to(DEV)
    xd = {k: v.to(DEV) for k, v in x.items()}
    got = ssm.ssm_scan_fwd_strided(xd["u"], xd["delta"], xd["A"], B1.expand(3, -1, -1),
                                   C1.expand(3, -1, -1), D=xd["D"], z=xd["z"],
                                   dt_bias=xd["dt_bias"])
    ref = ssm.ssm_scan_fwd(xd["u"], xd["delta"], xd["A"], B1.expand(3, -1, -1).contiguous(),
                           C1.expand(3, -1, -1).contiguous(), D=xd["D"], z=xd["z"],
                           dt_bias=xd["dt_bias"])
    assert torch.equal(got, ref)


@pytest.mark.parametrize("flags", ["plain", "reverse_zoh", "scalar_a"])
def test_backward_strided_equals_dense(flags):
    kw = dict(reverse=flags == "reverse_zoh", zoh=flags == "reverse_zoh",
              scalar_a=flags == "scalar_a")
    w = workload("mamba2p8b_train", batch=2, dim=64, seqlen=160)
    x = make_inputs(w, seed=83, with_dout=True, with_h0=True, scalar_a=kw["scalar_a"])
    s = strided_copies(x, seed=2)
    gbuf = torch.zeros((2, 16, 2, 160), dtype=torch.bfloat16, device=DEV)
    grads = {"dB": gbuf[:, :, 0], "dC": gbuf[:, :, 1]}   # interleaved outputs
    dubuf = torch.zeros((2, 160, 64), dtype=torch.bfloat16, device=DEV)
    grads["du"] = dubuf.transpose(1, 2)
    g = ssm.ssm_scan_bwd_strided(s["u"], s["delta"], s["A"], s["B"], s["C"], s["dout"], D=s["D"],
                                 z=s["z"], dt_bias=s["dt_bias"], h0=s["h0"], grads=grads, **kw)
    xd = {k: v.to(DEV) for k, v in x.items()}
    bwd = ssm.ssm_scan_bwd_scalar_a if kw["scalar_a"] else ssm.ssm_scan_bwd
    r = bwd(xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"], xd["dout"], D=xd["D"], z=xd["z"],
            dt_bias=xd["dt_bias"], h0=xd["h0"], reverse=kw["reverse"], zoh=kw["zoh"])
    for k in ("du", "ddelta", "dz", "dB", "dC", "dA", "dD", "ddt_bias", "dh0"):
        assert torch.equal(g[k], r[k]), k
    assert g["dB"].data_ptr() == gbuf.data_ptr()


@pytest.mark.parametrize("io", [torch.bfloat16, torch.float32])
def test_decode_strided_equals_dense(io):
    batch, dim, N = 5, 256, 16
    gen = torch.Generator().manual_seed(11)
    rnd = lambda *sh: torch.randn(*sh, generator=gen)
    sbuf = torch.zeros((batch, dim, 2 * N), device=DEV)
    state = sbuf[..., :N]
    state.copy_(0.5 * rnd(batch, dim, N).to(DEV))
    dense_state = state.contiguous()
    xz = rnd(batch, 2, dim).to(io).to(DEV)        # x and z interleaved by rows
    dt = (0.3 * rnd(dim, batch)).to(io).to(DEV).t()  # [batch, dim] seen through a transpose
    B = rnd(1, N).to(io).to(DEV).expand(batch, N)  # shared by every row
    C = rnd(batch, N).to(io).to(DEV)
    A = -torch.rand(dim, N, generator=gen).to(DEV) * 4 - 0.1
    D, bias = rnd(dim).to(DEV), (0.1 * rnd(dim)).to(DEV)
    obuf = torch.zeros((batch, dim, 2), dtype=io, device=DEV)
    out = ssm.ssm_state_update_strided(state, xz[:, 0], dt, A, B, C, D=D, z=xz[:, 1],
                                       dt_bias=bias, out=obuf[..., 1])
    ref = ssm.ssm_state_update(dense_state, xz[:, 0].contiguous(), dt.contiguous(), A,
                               B.contiguous(), C, D=D, z=xz[:, 1].contiguous(), dt_bias=bias)
    assert torch.equal(out, ref) and torch.equal(state, dense_state)
    assert torch.count_nonzero(sbuf[..., N:]) == 0 and torch.count_nonzero(obuf[..., 0]) == 0


def test_overlapping_output_is_refused():
    w = workload("mamba2p8b_train", batch=2, dim=64, seqlen=64)
    x = make_inputs(w, seed=84)
    xd = {k: v.to(DEV) for k, v in x.items()}
    one = torch.empty((1, 64, 64), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(RuntimeError, match="one address"):
        ssm.ssm_scan_fwd_strided(xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"],
                                 out=one.expand(2, -1, -1))



@pytest.mark.parametrize("io", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("N", [64, 128])
@pytest.mark.parametrize("reverse", [False, True])
def test_large_n_chunked_form_takes_strided_views(io, N, reverse):
    """Scalar decay with 64 or 128 states (the chunked matrix form in bf16, the 16-state slices
    in f32) from the views a Mamba-2 block holds: the projection halves, a (B, L, D) gate,
    strided B, C.  Forward and backward equal the dense calls bitwise."""
    w = workload("mamba2p8b_train", batch=2, dim=128, seqlen=160, dstate=N, io_dtype=io)
    x = make_inputs(w, seed=84, with_dout=True, with_h0=True, scalar_a=True)
    s = strided_copies(x, seed=3)
    xd = {k: v.to(DEV) for k, v in x.items()}
    kw = dict(scalar_a=True, reverse=reverse)
    out, hL = ssm.ssm_scan_fwd_strided(s["u"], s["delta"], s["A"], s["B"], s["C"], D=s["D"],
                                       z=s["z"], dt_bias=s["dt_bias"], h0=s["h0"],
                                       return_final_state=True, **kw)
    ref, hL_ref = ssm.ssm_scan_fwd_scalar_a(xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"],
                                            D=xd["D"], z=xd["z"], dt_bias=xd["dt_bias"],
                                            h0=xd["h0"], return_final_state=True, reverse=reverse)
    assert torch.equal(out, ref) and torch.equal(hL, hL_ref)
    g = ssm.ssm_scan_bwd_strided(s["u"], s["delta"], s["A"], s["B"], s["C"], s["dout"], D=s["D"],
                                 z=s["z"], dt_bias=s["dt_bias"], h0=s["h0"], **kw)
    r = ssm.ssm_scan_bwd_scalar_a(xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"], xd["dout"],
                                  D=xd["D"], z=xd["z"], dt_bias=xd["dt_bias"], h0=xd["h0"],
                                  reverse=reverse)
    for k in ("du", "ddelta", "dz", "dB", "dC", "dA", "dD", "ddt_bias", "dh0"):
        assert torch.equal(g[k], r[k]), k
