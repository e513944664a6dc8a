"""Forward scan: CUDA library (through the C ABI) against the fp64 oracle on the same seeded
inputs -- every tile, ragged tails, the time-split path, the degenerate cases, and the full
workload sizes in the benchmark's launch configuration."""
import os

import numpy as np
import pytest
import torch

import oracle
import selective_state_space_23_b200 as ssm
from selective_state_space_23_b200.inputs import make_inputs, workload

from _parity import assert_close, f64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def on_dev(x):
    return {k: v.to(DEV) for k, v in x.items()}


def run_gpu(x, softplus=True, **kw):
    return ssm.ssm_scan_fwd(x["u"], x["delta"], x["A"], x["B"], x["C"], D=x.get("D"),
                            z=x.get("z"), dt_bias=x.get("dt_bias"), delta_softplus=softplus,
                            h0=x.get("h0"), **kw)


def run_oracle(x, softplus=True, sel=None):
    """Oracle on channels ``sel`` (indices into dim, all batches), slicing before conversion."""
    g = lambda k: None if x.get(k) is None else x[k]
    if sel is not None:
        sel_t = torch.as_tensor(sel)
        sl = lambda k, ax: None if g(k) is None else g(k).index_select(ax, sel_t)
        x = dict(x, u=sl("u", 1), delta=sl("delta", 1), z=sl("z", 1), A=sl("A", 0), D=sl("D", 0),
                 dt_bias=sl("dt_bias", 0), h0=sl("h0", 1))
    c = lambda k: None if x.get(k) is None else f64(x[k])
    return oracle.scan_fwd(c("u"), c("delta"), c("A"), c("B"), c("C"), D=c("D"), z=c("z"),
                           dt_bias=c("dt_bias"), delta_softplus=softplus, h0=c("h0"))


@pytest.fixture(autouse=True)
def _clean_env(monkeypatch):
    for k in ("SSM_FWD_SPLIT", "SSM_FWD_KERNEL", "SSM_FWD_KMUFU"):
        monkeypatch.delenv(k, raising=False)
    yield


def test_tiny_f32_full():
    w = workload("tiny_f32")
    x = make_inputs(w, seed=0)
    out, hL = run_gpu(on_dev(x), return_final_state=True)
    ref = run_oracle(x)
    assert_close(out, ref["out"], torch.float32, "out")
    assert_close(hL, ref["hL"], torch.float32, "hL")


@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("shape", [(2, 70, 250, 5), (1, 33, 37, 16), (3, 100, 1000, 16),
                                   (1, 1, 1, 1), (2, 64, 17, 3)])
def test_ragged_shapes_and_options(io, shape):
    batch, dim, L, N = shape
    w = workload("tiny_f32", batch=batch, dim=dim, seqlen=L, dstate=N, io_dtype=io)
    x = make_inputs(w, seed=1, with_h0=True)
    out, hL = run_gpu(on_dev(x), return_final_state=True)
    ref = run_oracle(x)
    assert_close(out, ref["out"], io, "out")
    assert_close(hL, ref["hL"], torch.float32 if io == torch.float32 else io, "hL")


@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
def test_without_gate_skip_bias_and_softplus(io):
    w = workload("tiny_f32", batch=2, dim=96, seqlen=320, dstate=16, io_dtype=io)
    x = make_inputs(w, seed=2, gate=False)
    x["delta"] = (x["delta"].float().abs() * 0.05 + 1e-3).to(io)   # positive steps
    del x["D"], x["dt_bias"]
    out = run_gpu(on_dev(x), softplus=False)
    ref = run_oracle(x, softplus=False)
    assert_close(out, ref["out"], io, "out")


def test_bf16_medium_full():
    w = workload("mamba370m_fwd", batch=2, dim=256, seqlen=1024)
    x = make_inputs(w, seed=3)
    out = run_gpu(on_dev(x))
    assert_close(out, run_oracle(x)["out"], torch.bfloat16, "out")


@pytest.mark.parametrize("kernel,kmufu", [("lane", k) for k in (10, 11, 12, 13, 14, 15, 16)] +
                         [("pair", k) for k in (14, 16)])
def test_every_exponential_split(monkeypatch, kernel, kmufu):
    """Each split of the exponentials between MUFU and the FMA-pipe polynomial, in both kernel
    families (one lane per channel; two lanes per channel), on a length that is not a multiple
    of the 16-step block so full and partial blocks both run."""
    monkeypatch.setenv("SSM_FWD_KERNEL", kernel)
    monkeypatch.setenv("SSM_FWD_KMUFU", str(kmufu))
    w = workload("mamba370m_fwd", batch=2, dim=200, seqlen=1000)
    x = make_inputs(w, seed=11, with_h0=True)
    out, hL = run_gpu(on_dev(x), return_final_state=True)
    ref = run_oracle(x)
    assert_close(out, ref["out"], torch.bfloat16, "out")
    assert_close(hL, ref["hL"], torch.bfloat16, "hL")


@pytest.mark.parametrize("wide", [0, 1])
@pytest.mark.parametrize("kmufu", [14, 16])
def test_both_register_budgets(monkeypatch, wide, kmufu):
    """The output kernel's default and 255-register forms (chosen by warps per SM) agree with the
    oracle, on a ragged length, and with each other bitwise (two-lanes-per-channel kernel)."""
    monkeypatch.setenv("SSM_FWD_KERNEL", "pair")
    monkeypatch.setenv("SSM_FWD_KMUFU", str(kmufu))
    w = workload("mamba370m_fwd", batch=2, dim=160, seqlen=777)
    x = make_inputs(w, seed=13, with_h0=True)
    monkeypatch.setenv("SSM_FWD_WIDE", str(wide))
    out = run_gpu(on_dev(x))
    assert_close(out, run_oracle(x)["out"], torch.bfloat16, "out")
    monkeypatch.setenv("SSM_FWD_WIDE", str(1 - wide))
    assert torch.equal(out, run_gpu(on_dev(x)))


@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
def test_general_kernel_with_and_without_time_split(monkeypatch, io):
    """The general (two-lanes-per-channel) kernel on the default variant, with the time split
    too (it serves rows that do not allow 16-byte copies, and every other variant)."""
    monkeypatch.setenv("SSM_FWD_KERNEL", "pair")
    w = workload("tiny_f32", batch=2, dim=40, seqlen=301, dstate=16, io_dtype=io)
    x = make_inputs(w, seed=12, with_h0=True)
    out, hL = run_gpu(on_dev(x), return_final_state=True)
    ref = run_oracle(x)
    assert_close(out, ref["out"], io, "out")
    assert_close(hL, ref["hL"], torch.float32 if io == torch.float32 else io, "hL")
    monkeypatch.setenv("SSM_FWD_SPLIT", "3")
    nws = ssm.fwd_workspace_bytes(2, 40, 301, 16, io)
    ws = torch.empty(nws, dtype=torch.uint8, device=DEV)
    out2 = run_gpu(on_dev(x), workspace=ws)
    assert_close(out2, ref["out"], io, "out (time split)")


def test_positive_A_entries_use_the_exact_exponential():
    w = workload("mamba370m_fwd", batch=1, dim=64, seqlen=256)
    x = make_inputs(w, seed=4)
    A = x["A"].clone()
    A[5, 3] = 0.05
    A[40, 0] = 0.01
    x["A"] = A
    out = run_gpu(on_dev(x))
    assert_close(out, run_oracle(x)["out"], torch.bfloat16, "out")


@pytest.mark.parametrize("split", [2, 5, 16])
@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
def test_forced_time_split(monkeypatch, split, io):
    monkeypatch.setenv("SSM_FWD_SPLIT", str(split))
    w = workload("tiny_f32", batch=2, dim=64, seqlen=1000, io_dtype=io)
    x = make_inputs(w, seed=5, with_h0=True)
    ws = ssm.fwd_workspace_bytes(2, 64, 1000, 16, io)
    assert ws > 0
    out, hL = run_gpu(on_dev(x), return_final_state=True)
    ref = run_oracle(x)
    assert_close(out, ref["out"], io, "out")
    assert_close(hL, ref["hL"], torch.float32 if io == torch.float32 else io, "hL")


def test_split_needs_workspace_else_same_result(monkeypatch):
    monkeypatch.setenv("SSM_FWD_SPLIT", "4")
    w = workload("mamba370m_fwd", batch=1, dim=64, seqlen=512)
    x = on_dev(make_inputs(w, seed=6))
    a = run_gpu(x)
    ws = torch.empty(ssm.fwd_workspace_bytes(1, 64, 512, 16, torch.bfloat16), dtype=torch.uint8,
                     device=DEV)
    b = run_gpu(x, workspace=ws)
    assert_close(a, f64(b), torch.bfloat16, "split vs unsplit")


def test_natural_split_few_channels():
    # 64 channels cannot fill the GPU: the planner splits time; result must not change
    w = workload("long_seq_1m", batch=1, dim=64, seqlen=16384)
    assert ssm.fwd_workspace_bytes(1, 64, 16384, 16, torch.bfloat16) > 0
    x = make_inputs(w, seed=7)
    out, hL = run_gpu(on_dev(x), return_final_state=True)
    ref = run_oracle(x)
    assert_close(out, ref["out"], torch.bfloat16, "out")
    assert_close(hL, ref["hL"], torch.bfloat16, "hL")


@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
def test_checkpoints_are_block_entry_states(io):
    L = 200
    w = workload("tiny_f32", batch=2, dim=40, seqlen=L, dstate=7, io_dtype=io)
    x = make_inputs(w, seed=8, with_h0=True)
    out, hL, ck = run_gpu(on_dev(x), return_final_state=True, return_ckpt=True)
    nblk = (L + 15) // 16
    assert ck.shape == (2, 40, nblk, 7)
    ckr = f64(ck)
    np.testing.assert_array_equal(ckr[:, :, 0], f64(x["h0"]))
    for k in range(1, nblk):
        pre = {kk: (v[..., :16 * k] if kk in ("u", "delta", "z", "B", "C") else v) for kk, v in x.items()}
        ref = run_oracle(pre)["hL"]
        assert_close(ckr[:, :, k], ref, torch.float32 if io == torch.float32 else io, f"ckpt {k}")


def test_deterministic_bitwise():
    w = workload("mamba370m_fwd", batch=2, dim=128, seqlen=512)
    x = on_dev(make_inputs(w, seed=9))
    a = run_gpu(x)
    b = run_gpu(x)
    assert torch.equal(a, b)


def test_too_small_device_buffer_rejected():
    """A device buffer smaller than the tensor it must hold is refused on the host.  `out` is
    NULL as well, so even if the size check were missing nothing could be launched."""
    from selective_state_space_23_b200 import _abi
    import ctypes
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    small = torch.empty(16 << 20, dtype=torch.uint8, device=DEV)   # its own 16 MiB segment
    rc = _abi.lib().ssm_scan_fwd(ctypes.c_void_p(small.data_ptr()), *([None] * 7), 1,
                                 *([None] * 5), 0, 1, 512, 32768, 16, 1, None)  # u needs 32 MiB
    assert rc == _abi.SSM_EINVAL
    assert b"allocation" in _abi.lib().ssm_last_error()


# ------------------------------------------------------------------ full workload sizes
def test_mamba370m_layer_full_size():
    """8 x 2048 x 2048, N=16, bf16 -- the benchmark's workload and launch configuration."""
    w = workload("mamba370m_fwd")
    x = make_inputs(w, seed=0)
    out = run_gpu(on_dev(x))
    torch.cuda.synchronize()
    assert_close(out, run_oracle(x)["out"], torch.bfloat16, "out")


@pytest.mark.slow
def test_mamba2p8b_fwd_sampled_channels():
    w = workload("mamba2p8b_train")
    x = make_inputs(w, seed=0)
    out, hL = run_gpu(on_dev(x), return_final_state=True)
    sel = list(range(0, 5120, 80))  # 64 channels of every batch row
    ref = run_oracle(x, sel=sel)
    idx = torch.as_tensor(sel, device=DEV)
    assert_close(out.index_select(1, idx), ref["out"], torch.bfloat16, "out")
    assert_close(hL.index_select(1, idx), ref["hL"], torch.bfloat16, "hL")


@pytest.mark.slow
def test_long_sequence_all_channels_and_final_state():
    """1 x 256 x 2^20 (dt in [1e-4, 1e-2]): output and final state of all 256 channels."""
    w = workload("long_seq_1m")
    x = make_inputs(w, seed=0)
    xd = on_dev(x)
    out, hL = run_gpu(xd, return_final_state=True)
    torch.cuda.synchronize()
    del xd
    for c0 in range(0, 256, 32):
        sel = list(range(c0, c0 + 32))
        ref = run_oracle(x, sel=sel)
        idx = torch.as_tensor(sel, device=DEV)
        assert_close(out.index_select(1, idx), ref["out"], torch.bfloat16, f"out[{c0}]")
        assert_close(hL.index_select(1, idx), ref["hL"], torch.bfloat16, f"hL[{c0}]")
