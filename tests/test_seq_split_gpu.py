"""Sequence split through the library: the segment summaries (end state from zero and ΣΔ), the
chain of segment maps, and each segment's forward from its entering state, run here for every
segment on one GPU (the multi-rank exchange itself is covered on CPU ranks in test_dist.py).
The concatenated outputs are compared with the fp64 oracle's full-sequence run ("Temel
Fikirler" on the Mamba summary page: the recurrence is an associative scan of affine maps)."""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_23_b200 as ssm
from selective_state_space_23_b200.dist import seq_split_scan_fwd, shard_rows
from selective_state_space_23_b200.inputs import make_inputs, workload

from _parity import assert_close, f64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def seg(x, k, t0, t1):
    return x[k][..., t0:t1].contiguous().to(DEV)


def split_run(x, nseg, scalar_a=False, zoh=False, softplus=True):
    """Every segment's summary, the chain, and every segment's forward, as S ranks would."""
    L = x["u"].shape[-1]
    spans = [shard_rows(L, nseg, r) for r in range(nseg)]
    A = x["A"].to(DEV)
    bias = x["dt_bias"].to(DEV) if x.get("dt_bias") is not None else None
    hs, ds = [], []
    for t0, t1 in spans:
        h, d = ssm.ssm_scan_fwd_summary(seg(x, "u", t0, t1), seg(x, "delta", t0, t1), A,
                                        seg(x, "B", t0, t1), seg(x, "C", t0, t1), dt_bias=bias,
                                        delta_softplus=softplus, scalar_a=scalar_a, zoh=zoh)
        hs.append(h)
        ds.append(d)
    h0 = x["h0"].to(DEV) if x.get("h0") is not None else None
    hin = ssm.ssm_scan_chain(torch.stack(hs), torch.stack(ds), A, h0=h0, scalar_a=scalar_a)
    outs, hL = [], None
    f = ssm.ssm_scan_fwd_scalar_a if scalar_a else ssm.ssm_scan_fwd
    for r, (t0, t1) in enumerate(spans):
        o, hL = f(seg(x, "u", t0, t1), seg(x, "delta", t0, t1), A, seg(x, "B", t0, t1),
                  seg(x, "C", t0, t1), D=x["D"].to(DEV), z=seg(x, "z", t0, t1), dt_bias=bias,
                  delta_softplus=softplus, h0=hin[r], return_final_state=True, zoh=zoh)
        outs.append(o)
    return spans, hs, ds, torch.cat(outs, dim=-1), hL


def ref(x, scalar_a=False, zoh=False, softplus=True):
    c = lambda k: None if x.get(k) is None else f64(x[k])
    A = c("A")
    if scalar_a:
        A = np.repeat(A[:, None], x["B"].shape[-2], axis=1)
    return oracle.scan_fwd(c("u"), c("delta"), A, c("B"), c("C"), D=c("D"), z=c("z"),
                           dt_bias=c("dt_bias"), delta_softplus=softplus, h0=c("h0"), zoh=zoh)


@pytest.mark.parametrize("io", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("nseg", [2, 3, 5])
def test_segments_reproduce_the_full_sequence(io, nseg):
    w = workload("long_seq_1m", batch=2, dim=48, seqlen=333, io_dtype=io)
    x = make_inputs(w, seed=91, with_h0=True)
    _, hs, ds, out, hL = split_run(x, nseg)
    r = ref(x)
    assert_close(out, r["out"], io, "out")
    assert_close(hL, r["hL"], io, "hL")


def test_summary_pins():
    """hend is the segment's end state from zero, dsum its summed steps."""
    w = workload("long_seq_1m", batch=2, dim=48, seqlen=200, io_dtype=torch.float32)
    x = make_inputs(w, seed=92)
    xd = {k: v.to(DEV) for k, v in x.items()}
    h, d = ssm.ssm_scan_fwd_summary(xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"],
                                    dt_bias=xd["dt_bias"])
    r = oracle.scan_fwd(f64(x["u"]), f64(x["delta"]), f64(x["A"]), f64(x["B"]), f64(x["C"]),
                        dt_bias=f64(x["dt_bias"]))
    assert_close(h, r["hL"], torch.float32, "hend")
    v = f64(x["delta"]) + f64(x["dt_bias"])[None, :, None]
    np.testing.assert_allclose(d.cpu().numpy(), np.logaddexp(0.0, v).sum(axis=2), rtol=1e-5)


def test_long_segment_summary_uses_the_time_split():
    """64 channels over 8192 steps: the summary runs the forward's chunked summary and carry
    passes inside the call."""
    w = workload("long_seq_1m", batch=1, dim=64, seqlen=8192)
    x = make_inputs(w, seed=93)
    xd = {k: v.to(DEV) for k, v in x.items()}
    h, d = ssm.ssm_scan_fwd_summary(xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"],
                                    dt_bias=xd["dt_bias"])
    _, hL = ssm.ssm_scan_fwd(xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"],
                             dt_bias=xd["dt_bias"], return_final_state=True)
    r = oracle.scan_fwd(f64(x["u"]), f64(x["delta"]), f64(x["A"]), f64(x["B"]), f64(x["C"]),
                        dt_bias=f64(x["dt_bias"]))
    assert_close(h, r["hL"], torch.bfloat16, "hend")
    assert_close(h, hL.cpu().numpy().astype(np.float64), torch.bfloat16, "hend vs forward")


@pytest.mark.parametrize("variant", ["scalar_a", "zoh", "groups", "no_softplus"])
def test_variants(variant):
    kw = dict(scalar_a=variant == "scalar_a", zoh=variant == "zoh",
              softplus=variant != "no_softplus")
    w = workload("long_seq_1m", batch=2, dim=64, seqlen=240)
    x = make_inputs(w, seed=94, with_h0=True, scalar_a=kw["scalar_a"])
    if variant == "groups":
        wg = workload("long_seq_1m", batch=4, dim=1, seqlen=240)
        xg = make_inputs(wg, seed=95)
        x["B"] = xg["B"].reshape(2, 2, 16, 240).contiguous()
        x["C"] = xg["C"].reshape(2, 2, 16, 240).contiguous()
    if variant == "no_softplus":
        x["delta"] = (x["delta"].float().abs() * 0.05 + 1e-3).to(torch.bfloat16)
        x["dt_bias"] = None
    _, _, _, out, hL = split_run(x, 3, **kw)
    r = ref(x, **kw)
    assert_close(out, r["out"], torch.bfloat16, "out")
    assert_close(hL, r["hL"], torch.bfloat16, "hL")


def test_helper_without_process_group():
    """seq_split_scan_fwd with no process group is one segment: the plain forward."""
    w = workload("long_seq_1m", batch=1, dim=32, seqlen=96)
    x = make_inputs(w, seed=96, with_h0=True)
    xd = {k: v.to(DEV) for k, v in x.items()}
    out, hL = seq_split_scan_fwd(xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"], D=xd["D"],
                                 z=xd["z"], dt_bias=xd["dt_bias"], h0=xd["h0"],
                                 return_final_state=True)
    o2, h2 = ssm.ssm_scan_fwd(xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"], D=xd["D"],
                              z=xd["z"], dt_bias=xd["dt_bias"], h0=xd["h0"],
                              return_final_state=True)
    r = ref(x)
    assert_close(out, r["out"], torch.bfloat16, "out")
    assert_close(hL, h2.cpu().numpy().astype(np.float64), torch.bfloat16, "hL")


@pytest.mark.parametrize("io,N", [(torch.bfloat16, 64), (torch.bfloat16, 128), (torch.float32, 32),
                                  (torch.float32, 64)])
@pytest.mark.parametrize("nseg", [1, 3])
def test_large_state_scalar_decay_segments(io, N, nseg):
    """Scalar decay with N = 32 to 128 (the Mamba-2 state sizes): bf16 summaries run the chunked
    matrix form's summary pass, f32 ones sum 16-state slices; the split reproduces the whole
    sequence, and each summary is the segment's end state from zero with its summed steps."""
    w = workload("long_seq_1m", batch=2, dim=64, seqlen=400, dstate=N, io_dtype=io)
    x = make_inputs(w, seed=93, with_h0=True, scalar_a=True)
    spans, hs, ds, out, hL = split_run(x, nseg, scalar_a=True)
    r = ref(x, scalar_a=True)
    assert_close(out, r["out"], io, "out")
    assert_close(hL, r["hL"], io, "hL")
    c = lambda k: f64(x[k])
    A = np.repeat(c("A")[:, None], N, axis=1)
    for (t0, t1), h, d in zip(spans, hs, ds):
        rs = oracle.scan_fwd(c("u")[..., t0:t1], c("delta")[..., t0:t1], A, c("B")[..., t0:t1],
                             c("C")[..., t0:t1], dt_bias=c("dt_bias"))
        assert_close(h, rs["hL"], io, f"hend {t0}")
        v = c("delta")[..., t0:t1] + c("dt_bias")[None, :, None]
        dref = np.logaddexp(0.0, v).sum(-1)
        assert_close(d, dref, torch.float32, f"dsum {t0}")


@pytest.mark.parametrize("N", [64, 128])
def test_large_state_summary_splits_itself(monkeypatch, N):
    """Few channels: the chunked form's planner cuts the segment into several pieces, chained
    from zero inside the call; forced counts agree with the unsplit summary."""
    w = workload("long_seq_1m", batch=1, dim=64, seqlen=1000, dstate=N)
    x = make_inputs(w, seed=94, scalar_a=True)
    xd = {k: v.to(DEV) for k, v in x.items()}
    run = lambda: ssm.ssm_scan_fwd_summary(xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"],
                                           dt_bias=xd["dt_bias"], scalar_a=True)
    monkeypatch.setenv("SSM_SSD_SPLIT", "1")
    h1, d1 = run()
    c = lambda k: f64(x[k])
    A = np.repeat(c("A")[:, None], N, axis=1)
    rs = oracle.scan_fwd(c("u"), c("delta"), A, c("B"), c("C"), dt_bias=c("dt_bias"))
    assert_close(h1, rs["hL"], torch.bfloat16, "hend unsplit")
    for split in ("4", "9"):
        monkeypatch.setenv("SSM_SSD_SPLIT", split)
        h, d = run()
        assert_close(h, rs["hL"], torch.bfloat16, f"hend split {split}")
        torch.testing.assert_close(d, d1, rtol=1e-5, atol=1e-5)


@pytest.mark.parametrize("io", [torch.bfloat16, torch.float32])
def test_large_state_zoh_segments(io):
    """The zero-order-hold input term with 64 states: summaries (chunked summary pass in bf16,
    16-state slices in f32), chain and segment forwards reproduce the whole sequence."""
    w = workload("long_seq_1m", batch=1, dim=64, seqlen=300, dstate=64, io_dtype=io)
    x = make_inputs(w, seed=95, with_h0=True, scalar_a=True)
    _, _, _, out, hL = split_run(x, 3, scalar_a=True, zoh=True)
    r = ref(x, scalar_a=True, zoh=True)
    assert_close(out, r["out"], io, "out")
    assert_close(hL, r["hL"], io, "hL")
