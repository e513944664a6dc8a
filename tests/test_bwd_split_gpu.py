"""Backward with the time split (few channels or long sequences): chunks of whole 16-step blocks
run side by side, each starting from the adjoint that enters it from later time.  Those entering
adjoints come from per-chunk adjoint summaries chained by an associative carry pass (the parallel
scan of "Temel Fikirler" and the recomputation of "Donanım Duyarlı Durum Genişletme" on the Mamba
summary page).  Every gradient is compared with the fp64 oracle; forced splits cover chunk counts
that do not divide the blocks, ragged tails, dhL, h0, checkpoints given or replayed, grouped B/C
and both io types; the natural split runs on a 1 x 256 x 2^18 sequence."""
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


@pytest.fixture(autouse=True)
def _env(monkeypatch):
    for k in ("SSM_BWD_SPLIT", "SSM_BWD_KERNEL", "SSM_BWD_WPB", "SSM_FWD_KERNEL", "SSM_FWD_SPLIT"):
        monkeypatch.delenv(k, raising=False)


def run_gpu(x, dhL=None, use_ckpt=False):
    xd = {k: v.to(DEV) for k, v in x.items()}
    ck = None
    if use_ckpt:
        _, ck = ssm.ssm_scan_fwd(xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"], D=xd["D"],
                                 z=xd["z"], dt_bias=xd["dt_bias"], h0=xd.get("h0"),
                                 return_ckpt=True)
    return ssm.ssm_scan_bwd(xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"], xd["dout"], D=xd["D"],
                            z=xd["z"], dt_bias=xd["dt_bias"], h0=xd.get("h0"),
                            dhL=None if dhL is None else dhL.to(DEV), ckpt=ck)


def run_oracle(x, dhL=None, channels=None):
    c = lambda k: None if x.get(k) is None else f64(x[k])
    return oracle.scan_bwd(c("u"), c("delta"), c("A"), c("B"), c("C"), c("dout"), D=c("D"),
                           z=c("z"), dt_bias=c("dt_bias"), h0=c("h0"),
                           dhL=None if dhL is None else f64(dhL), channels=channels)


@pytest.mark.parametrize("io", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("split", [2, 3, 7])
@pytest.mark.parametrize("use_ckpt", [False, True])
def test_forced_split_matches_oracle(monkeypatch, io, split, use_ckpt):
    """312 steps = 20 blocks (the last one half full) cut into 2, 3 (7 blocks each, the last 6)
    or 7 chunks, with h0 and dhL."""
    monkeypatch.setenv("SSM_BWD_SPLIT", str(split))
    w = workload("mamba2p8b_train", batch=2, dim=64, seqlen=312, io_dtype=io)
    x = make_inputs(w, seed=41, with_dout=True, with_h0=True)
    dhL = torch.randn((2, 64, 16), generator=torch.Generator().manual_seed(4))
    g = run_gpu(x, dhL=dhL, use_ckpt=use_ckpt)
    r = run_oracle(x, dhL=dhL)
    for k in GRADS:
        assert_close(g[k], r[k], io, k)


def test_forced_split_with_grouped_bc(monkeypatch):
    monkeypatch.setenv("SSM_BWD_SPLIT", "4")
    w = workload("mamba2p8b_train", batch=1, dim=128, seqlen=256)
    x = make_inputs(w, seed=42, with_dout=True)
    wg = workload("mamba2p8b_train", batch=2, dim=1, seqlen=256)
    xg = make_inputs(wg, seed=43)
    x["B"] = xg["B"].reshape(1, 2, 16, 256).contiguous()
    x["C"] = xg["C"].reshape(1, 2, 16, 256).contiguous()
    g = run_gpu(x)
    r = run_oracle(x)
    for k in GRADS:
        assert_close(g[k], r[k], torch.bfloat16, k)


def test_natural_split_and_split_replay():
    """64 channels over 4096 steps: the backward splits time by itself, and without checkpoints
    so does the forward replay that recomputes them."""
    w = workload("long_seq_1m", batch=1, dim=64, seqlen=4096)
    x = make_inputs(w, seed=44, with_dout=True, with_h0=True)
    g = run_gpu(x)
    r = run_oracle(x)
    for k in GRADS:
        assert_close(g[k], r[k], torch.bfloat16, k)


@pytest.mark.slow
def test_long_sequence_backward_2_18():
    """1 x 256 x 2^18 (the long-sequence shape at a quarter of its length): du, ddelta, dz and
    dh0 of 32 sampled channels, dA, dD, ddt_bias of those channels, and dB, dC of the row summed
    over all 256 channels (the oracle run in four partitions of 64 channels, whose dB, dC add)."""
    w = workload("long_seq_1m", batch=1, dim=256, seqlen=1 << 18)
    x = make_inputs(w, seed=45, with_dout=True)
    g = run_gpu(x, use_ckpt=True)
    torch.cuda.synchronize()
    sel = list(range(3, 256, 8))
    dB = np.zeros((1, 16, 1 << 18))
    dC = np.zeros((1, 16, 1 << 18))
    for part in range(4):
        lo = 64 * part
        xp = {k: v for k, v in x.items()}
        for k in ("u", "delta", "z", "dout"):
            xp[k] = x[k][:, lo:lo + 64].contiguous()
        for k in ("A",):
            xp[k] = x[k][lo:lo + 64].contiguous()
        for k in ("D", "dt_bias"):
            xp[k] = x[k][lo:lo + 64].contiguous()
        r = run_oracle(xp)
        dB += r["dB"]
        dC += r["dC"]
        mine = [d - lo for d in sel if lo <= d < lo + 64]
        idx = torch.as_tensor([lo + m for m in mine], device=DEV)
        for k in ("du", "ddelta", "dz", "dh0"):
            assert_close(g[k].index_select(1, idx), r[k][:, mine], torch.bfloat16, k)
        for k in ("dA", "dD", "ddt_bias"):
            assert_close(g[k].index_select(0, idx), r[k][mine], torch.bfloat16, k)
        del r
    assert_close(g["dB"], dB, torch.bfloat16, "dB")
    assert_close(g["dC"], dC, torch.bfloat16, "dC")
