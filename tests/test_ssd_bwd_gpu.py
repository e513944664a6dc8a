"""Backward of the scalar-decay scan with N = 32, 64, 128 (the Mamba-2 state sizes of the "2024
Reading List: Neural Network" page).  bf16 calls in the default direction run the chunked
matrix form on the tensor cores; f32, reverse and ZOH calls (and SSM_SCALAR_BWD=slices) run the
sum over 16-state slices (the states of a scalar-decay scan do not interact).  Every gradient is
compared with the fp64 oracle's chain-rule gradients (A broadcast over the states, dA summed
over them), with dhL, h0, the ZOH input term, the reverse scan and grouped B/C."""
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


def inputs(batch, dim, L, N, io, seed, groups=1, gate=True):
    w = workload("mamba370m_fwd", batch=batch, dim=dim, seqlen=L, dstate=N, io_dtype=io)
    x = make_inputs(w, seed=seed, with_dout=True, with_h0=True, scalar_a=True, gate=gate)
    if groups > 1:
        wg = workload("mamba370m_fwd", batch=batch * groups, dim=1, seqlen=L, dstate=N, io_dtype=io)
        xg = make_inputs(wg, seed=seed + 1)
        x["B"] = xg["B"].reshape(batch, groups, N, L).contiguous()
        x["C"] = xg["C"].reshape(batch, groups, N, L).contiguous()
    return x


def run(x, dhL, **kw):
    xd = {k: v.to(DEV) for k, v in x.items()}
    return ssm.ssm_scan_bwd_scalar_a(xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"], xd["dout"],
                                     D=xd.get("D"), z=xd.get("z"), dt_bias=xd.get("dt_bias"),
                                     h0=xd["h0"], dhL=None if dhL is None else dhL.to(DEV), **kw)


def ref(x, dhL, **kw):
    c = lambda k: None if x.get(k) is None else f64(x[k])
    N = x["B"].shape[-2]
    A = np.repeat(c("A")[:, None], N, axis=1)
    g = oracle.scan_bwd(c("u"), c("delta"), A, c("B"), c("C"), c("dout"), D=c("D"), z=c("z"),
                        dt_bias=c("dt_bias"), h0=c("h0"), dhL=None if dhL is None else f64(dhL),
                        **kw)
    g["dA"] = g["dA"].sum(1)  # chain rule through A[d, n] = A_d
    return g


@pytest.mark.parametrize("io", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("N", [32, 64, 128])
def test_gradients_match_oracle(io, N):
    x = inputs(2, 64, 160, N, io, seed=101)
    dhL = torch.randn((2, 64, N), generator=torch.Generator().manual_seed(7))
    g = run(x, dhL)
    assert g["dA"].shape == (64,) and g["dB"].shape == (2, N, 160)
    r = ref(x, dhL)
    for k in GRADS:
        assert_close(g[k], r[k], io, k)


@pytest.mark.parametrize("variant", ["reverse_zoh", "reverse", "groups", "no_gate"])
def test_variants(variant):
    kw = dict(reverse=variant.startswith("reverse"), zoh=variant == "reverse_zoh")
    x = inputs(2, 128, 96, 64, torch.bfloat16, seed=102, groups=2 if variant == "groups" else 1,
               gate=variant != "no_gate")
    if variant == "no_gate":
        del x["D"]
    g = run(x, None, **kw)
    r = ref(x, None, **kw)
    for k in GRADS:
        if r.get(k) is None or g.get(k) is None:
            continue
        assert_close(g[k], r[k], torch.bfloat16, k)


def test_slice_backward_refuses_checkpoints(monkeypatch):
    """The slice path (here forced) recomputes its states and refuses checkpoints."""
    monkeypatch.setenv("SSM_SCALAR_BWD", "slices")
    x = inputs(1, 64, 64, 64, torch.bfloat16, seed=103)
    xd = {k: v.to(DEV) for k, v in x.items()}
    fake_ck = torch.zeros((1, 64, 4, 64), device=DEV)
    with pytest.raises(RuntimeError):
        ssm.ssm_scan_bwd_scalar_a(xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"], xd["dout"],
                                  D=xd["D"], z=xd["z"], dt_bias=xd["dt_bias"], h0=xd["h0"],
                                  ckpt=fake_ck)


def fwd(x, **kw):
    xd = {k: v.to(DEV) for k, v in x.items()}
    return ssm.ssm_scan_fwd_scalar_a(xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"], D=xd["D"],
                                     z=xd["z"], dt_bias=xd["dt_bias"], h0=xd["h0"], **kw)


@pytest.mark.parametrize("N", [16, 64, 128])
@pytest.mark.parametrize("shape", [(2, 128, 333), (1, 80, 96)])
def test_chunked_forward_checkpoints_are_block_entry_states(N, shape):
    """The chunked forward's checkpoints: the state entering every 16-step block (slot 0 = h0),
    against the oracle's final states of the prefixes; the outputs are unchanged by asking for
    them."""
    batch, dim, L = shape
    x = inputs(batch, dim, L, N, torch.bfloat16, seed=119)
    out, ck = fwd(x, return_ckpt=True)
    assert ck.shape == (batch, dim, (L + 15) // 16, N)
    assert torch.equal(out, fwd(x))
    c = lambda k: f64(x[k])
    A = np.repeat(c("A")[:, None], N, axis=1)
    for k in range(ck.shape[2]):
        t = 16 * k
        if t == 0:
            ref_h = c("h0")
        else:
            r = oracle.scan_fwd(c("u")[..., :t], c("delta")[..., :t], A, c("B")[..., :t],
                                c("C")[..., :t], D=c("D"), z=c("z")[..., :t],
                                dt_bias=c("dt_bias"), h0=c("h0"))
            ref_h = r["hL"]
        assert_close(ck[:, :, k, :], ref_h, torch.bfloat16, f"checkpoint {k}")


@pytest.mark.parametrize("N", [16, 64, 128])
def test_chunked_backward_from_forward_checkpoints(N):
    """The backward given the chunked forward's checkpoints (no checkpoint pass) against the
    oracle, and against the same backward recomputing them."""
    x = inputs(2, 128, 333, N, torch.bfloat16, seed=120)
    _, ck = fwd(x, return_ckpt=True)
    dhL = torch.randn((2, 128, N), generator=torch.Generator().manual_seed(12))
    g = run(x, dhL, ckpt=ck)
    g0 = run(x, dhL)
    r = ref(x, dhL)
    for k in GRADS:
        assert_close(g[k], r[k], torch.bfloat16, k)
        assert_close(g[k], f64(g0[k]), torch.bfloat16, k)


def test_chunked_backward_from_per_state_checkpoints(monkeypatch):
    """N = 16: checkpoints written by the per-state forward kernel serve the chunked backward
    (same layout, same states)."""
    x = inputs(2, 64, 200, 16, torch.bfloat16, seed=121)
    monkeypatch.setenv("SSM_SCALAR_FORM", "state")
    _, ck = fwd(x, return_ckpt=True)
    monkeypatch.delenv("SSM_SCALAR_FORM")
    g = run(x, None, ckpt=ck)
    r = ref(x, None)
    for k in GRADS:
        assert_close(g[k], r[k], torch.bfloat16, k)


# ------------------------------------------------------------------ the chunked-form backward
@pytest.mark.parametrize("N", [16, 32, 64, 128])
@pytest.mark.parametrize("shape", [(2, 128, 160), (1, 80, 333), (2, 64, 17)])
def test_chunked_backward_matches_oracle(monkeypatch, N, shape):
    """bf16 scalar decay with N > 16 runs the chunked-form backward (tensor cores): partial
    64-channel tiles, ragged time tails, dhL and h0."""
    monkeypatch.delenv("SSM_SCALAR_BWD", raising=False)
    batch, dim, L = shape
    x = inputs(batch, dim, L, N, torch.bfloat16, seed=111)
    dhL = torch.randn((batch, dim, N), generator=torch.Generator().manual_seed(9))
    g = run(x, dhL)
    r = ref(x, dhL)
    for k in GRADS:
        assert_close(g[k], r[k], torch.bfloat16, k)


@pytest.mark.parametrize("N", [16, 64])
def test_chunked_and_per_state_backwards_agree(monkeypatch, N):
    """The chunked form against the per-state kernels (16-state slices above N = 16)."""
    x = inputs(2, 128, 200, N, torch.bfloat16, seed=112)
    monkeypatch.delenv("SSM_SCALAR_BWD", raising=False)
    a = run(x, None)
    monkeypatch.setenv("SSM_SCALAR_BWD", "state" if N == 16 else "slices")
    b = run(x, None)
    for k in GRADS:
        assert_close(a[k], f64(b[k]), torch.bfloat16, k)


@pytest.mark.parametrize("N", [16, 32, 64, 128])
def test_chunked_backward_range_fallback(N):
    """Steps over v = delta + dt_bias in [-30, 30]: most chunks leave the factorisation's range,
    and their intra-chunk products take the exact per-pair decay.  Gradients of size ~1 are
    differences of terms in the hundreds here, so this also checks that every product feeding
    them keeps ~16 significant bits."""
    x = inputs(1, 64, 96, N, torch.bfloat16, seed=113)
    v = np.random.default_rng(4).uniform(-30, 30, size=x["delta"].shape).astype(np.float32)
    x["delta"] = torch.from_numpy(v).to(torch.bfloat16)
    x["dt_bias"] = torch.zeros_like(x["dt_bias"])
    dhL = torch.randn((1, 64, N), generator=torch.Generator().manual_seed(5))
    g = run(x, dhL)
    r = ref(x, dhL)
    for k in GRADS:
        assert_close(g[k], r[k], torch.bfloat16, k)


def test_chunked_backward_mixed_range():
    """Channels in and out of the factorisation's range side by side in the same warps and
    chunks (every other channel takes large steps), over a ragged tail."""
    x = inputs(2, 64, 150, 64, torch.bfloat16, seed=115)
    v = x["delta"].float().numpy()
    big = np.random.default_rng(6).uniform(-30, 30, size=v.shape).astype(np.float32)
    v[:, 1::2, :] = big[:, 1::2, :]
    x["delta"] = torch.from_numpy(v).to(torch.bfloat16)
    g = run(x, None)
    r = ref(x, None)
    for k in GRADS:
        assert_close(g[k], r[k], torch.bfloat16, k)


def test_chunked_backward_with_time_split_checkpoints():
    """64 channels over 2048 steps: the checkpoint pass splits time by itself."""
    x = inputs(1, 64, 2048, 64, torch.bfloat16, seed=114)
    g = run(x, None)
    r = ref(x, None)
    for k in GRADS:
        assert_close(g[k], r[k], torch.bfloat16, k)


@pytest.mark.parametrize("N", [16, 64, 128])
@pytest.mark.parametrize("split", ["3", "7"])
def test_chunked_backward_forced_time_split(monkeypatch, N, split):
    """Forced segments of the reverse walk (summary launch, adjoint chain, segment launch) over a
    ragged tail, with dhL and h0: the same gradients as the oracle."""
    monkeypatch.setenv("SSM_SSD_BWD_SPLIT", split)
    x = inputs(2, 128, 333, N, torch.bfloat16, seed=116)
    dhL = torch.randn((2, 128, N), generator=torch.Generator().manual_seed(10))
    g = run(x, dhL)
    r = ref(x, dhL)
    for k in GRADS:
        assert_close(g[k], r[k], torch.bfloat16, k)


def test_chunked_backward_long_sequence_splits_by_itself(monkeypatch):
    """64 channels over 16384 steps: one CTA of channels, so the planner cuts the reverse walk
    into segments (and the checkpoint pass into its own)."""
    monkeypatch.delenv("SSM_SSD_BWD_SPLIT", raising=False)
    x = inputs(1, 64, 16384, 64, torch.bfloat16, seed=117)
    dhL = torch.randn((1, 64, 64), generator=torch.Generator().manual_seed(11))
    g = run(x, dhL)
    r = ref(x, dhL)
    for k in GRADS:
        assert_close(g[k], r[k], torch.bfloat16, k)


def test_chunked_backward_split_agrees_with_unsplit(monkeypatch):
    """The split walk against the unsplit one on the same inputs (both in f32 accumulation)."""
    x = inputs(1, 128, 1024, 64, torch.bfloat16, seed=118)
    monkeypatch.setenv("SSM_SSD_BWD_SPLIT", "1")
    a = run(x, None)
    monkeypatch.setenv("SSM_SSD_BWD_SPLIT", "8")
    b = run(x, None)
    for k in GRADS:
        assert_close(a[k], f64(b[k]), torch.bfloat16, k)


# ------------------------------------------------------------------ the reverse scan
@pytest.mark.parametrize("N", [32, 64, 128])
def test_chunked_reverse_forward_matches_oracle(N):
    """The reverse scan (the anti-causal half of a bidirectional layer) in the chunked form:
    outputs, final state and checkpoints (the state entering every block in scan order)."""
    x = inputs(2, 128, 333, N, torch.bfloat16, seed=122)
    out, hL, ck = fwd(x, reverse=True, return_final_state=True, return_ckpt=True)
    c = lambda k: f64(x[k])
    A = np.repeat(c("A")[:, None], N, axis=1)
    r = oracle.scan_fwd(c("u"), c("delta"), A, c("B"), c("C"), D=c("D"), z=c("z"),
                        dt_bias=c("dt_bias"), h0=c("h0"), reverse=True)
    assert_close(out, r["out"], torch.bfloat16, "out")
    assert_close(hL, r["hL"], torch.bfloat16, "hL")
    # checkpoint k: the state after the scan's first 16 k steps, i.e. rows L - 16 k .. L - 1
    L = x["u"].shape[-1]
    for k in (1, 7, ck.shape[2] - 1):
        t = L - 16 * k
        rk = oracle.scan_fwd(c("u")[..., t:], c("delta")[..., t:], A, c("B")[..., t:],
                             c("C")[..., t:], D=c("D"), z=c("z")[..., t:], dt_bias=c("dt_bias"),
                             h0=c("h0"), reverse=True)
        assert_close(ck[:, :, k, :], rk["hL"], torch.bfloat16, f"checkpoint {k}")


@pytest.mark.parametrize("N", [16, 64, 128])
@pytest.mark.parametrize("shape", [(2, 128, 333), (1, 64, 512), (1, 64, 520)])
def test_chunked_reverse_backward_matches_oracle(N, shape):
    """The reverse scan's backward in the chunked form, recomputing its states and from the
    reverse forward's checkpoints, with dhL and h0.  Lengths: ragged (element-wise mirror
    copies), a multiple of 16, and 65 pieces of 8 (the in-place mirror's middle piece)."""
    batch, dim, L = shape
    x = inputs(batch, dim, L, N, torch.bfloat16, seed=123)
    dhL = torch.randn((batch, dim, N), generator=torch.Generator().manual_seed(13))
    r = ref(x, dhL, reverse=True)
    g = run(x, dhL, reverse=True)
    for k in GRADS:
        assert_close(g[k], r[k], torch.bfloat16, k)
    _, ck = fwd(x, reverse=True, return_ckpt=True)
    g2 = run(x, dhL, reverse=True, ckpt=ck)
    for k in GRADS:
        assert_close(g2[k], r[k], torch.bfloat16, k)


# ------------------------------------------------------------------ the zero-order hold
@pytest.mark.parametrize("N", [32, 64, 128])
@pytest.mark.parametrize("reverse", [False, True])
def test_chunked_zoh_forward_matches_oracle(N, reverse):
    """The zero-order-hold input coefficient (e^{ΔA} - 1)/A in the chunked forward, either
    direction: outputs and final state against the oracle."""
    x = inputs(2, 128, 333, N, torch.bfloat16, seed=124)
    out, hL = fwd(x, zoh=True, reverse=reverse, return_final_state=True)
    c = lambda k: f64(x[k])
    A = np.repeat(c("A")[:, None], N, axis=1)
    r = oracle.scan_fwd(c("u"), c("delta"), A, c("B"), c("C"), D=c("D"), z=c("z"),
                        dt_bias=c("dt_bias"), h0=c("h0"), zoh=True, reverse=reverse)
    assert_close(out, r["out"], torch.bfloat16, "out")
    assert_close(hL, r["hL"], torch.bfloat16, "hL")


@pytest.mark.parametrize("N", [16, 64, 128])
@pytest.mark.parametrize("reverse", [False, True])
def test_chunked_zoh_backward_matches_oracle(N, reverse):
    """The zero-order hold's gradients in the chunked backward (through c's step and rate),
    either direction, with dhL and h0, recomputed and from the forward's checkpoints."""
    x = inputs(2, 128, 333, N, torch.bfloat16, seed=125)
    dhL = torch.randn((2, 128, N), generator=torch.Generator().manual_seed(14))
    r = ref(x, dhL, zoh=True, reverse=reverse)
    g = run(x, dhL, zoh=True, reverse=reverse)
    for k in GRADS:
        assert_close(g[k], r[k], torch.bfloat16, k)
    if N > 16:
        _, ck = fwd(x, zoh=True, reverse=reverse, return_ckpt=True)
        g2 = run(x, dhL, zoh=True, reverse=reverse, ckpt=ck)
        for k in GRADS:
            assert_close(g2[k], r[k], torch.bfloat16, k)


def test_chunked_zoh_large_and_small_rates():
    """Rates from 1e-6 to 30 (the dc/dA series near ΔA = 0 and the direct form far from it),
    with steps up to 30 (chunks out of the factorisation's range): gradients against the
    oracle."""
    x = inputs(1, 64, 160, 64, torch.bfloat16, seed=126)
    a = np.geomspace(1e-6, 30, 64).astype(np.float32)
    x["A"] = -torch.from_numpy(a)
    v = np.random.default_rng(7).uniform(-12, 6, size=x["delta"].shape).astype(np.float32)
    x["delta"] = torch.from_numpy(v).to(torch.bfloat16)
    x["dt_bias"] = torch.zeros_like(x["dt_bias"])
    r = ref(x, None, zoh=True)
    g = run(x, None, zoh=True)
    for k in GRADS:
        assert_close(g[k], r[k], torch.bfloat16, k)



@pytest.mark.parametrize("need", [("du", "ddelta", "dA"), ("dB",), ("dC", "dh0"), ("dz", "ddt_bias", "dD")])
def test_chunked_backward_gradient_subsets(need):
    """Any subset of the gradients (the rest NULL at the C ABI; without dB and dC the chunk's
    channel contractions and their reduction are skipped): the requested ones equal the full
    call's bitwise."""
    x = inputs(2, 128, 200, 64, torch.bfloat16, seed=127)
    full = run(x, None)
    part = run(x, None, need=need)
    for k in GRADS:
        if k in need:
            assert torch.equal(part[k], full[k]), k
        else:
            assert part.get(k) is None, k


@pytest.mark.parametrize("N", [64, 128])
def test_chunked_backward_large_entering_state(N):
    """An entering state h0 ~ N(0, 3^2), larger than the inputs' own state: every product that
    reads the state (or its adjoint) takes it as a bf16 pair plus remainder, so the gradients,
    dh0 and dC included, keep the bf16 bound."""
    x = inputs(2, 64, 96, N, torch.bfloat16, seed=131)
    x["h0"] = torch.from_numpy(
        np.random.default_rng(10).normal(0.0, 3.0, size=(2, 64, N)).astype(np.float32))
    dhL = torch.randn((2, 64, N), generator=torch.Generator().manual_seed(11))
    g = run(x, dhL)
    r = ref(x, dhL)
    for k in GRADS:
        assert_close(g[k], r[k], torch.bfloat16, k)
