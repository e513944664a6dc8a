"""The C-ABI library loads and exports every entry point include/ssm_scan.h declares; host-only
behaviour (status strings, workspace sizes, argument validation) works without a GPU."""
import ctypes
import os
import re
import subprocess

import pytest

from selective_state_space_23_b200 import _abi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ssm_scan.h")


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"SSM_API\s+[\w\s\*]+?\b(ssm_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(_abi.LIB_PATH):
        from selective_state_space_23_b200 import build
        build.build()
    return _abi.lib()


def test_header_declares_the_entry_points():
    syms = declared_symbols()
    for s in ("ssm_scan_fwd", "ssm_scan_bwd", "ssm_state_update", "ssm_scan_fwd_workspace_size",
              "ssm_scan_bwd_workspace_size", "ssm_status_string", "ssm_last_error", "ssm_version"):
        assert s in syms


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", _abi.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (ssm_\w+)", out))
    assert set(declared_symbols()) <= exported
    for s in declared_symbols():
        assert getattr(lib, s) is not None
    assert set(_abi.SIGNATURES) == set(declared_symbols())


def test_build_targets_sm100a_only():
    from selective_state_space_23_b200 import build
    assert build.ARCH == ["-gencode", "arch=compute_100a,code=sm_100a"]


def test_status_strings(lib):
    assert lib.ssm_status_string(0) == b"ok"
    assert lib.ssm_status_string(1) == b"invalid argument"
    assert lib.ssm_status_string(4).startswith(b"workspace")
    assert lib.ssm_status_string(99) == b"unknown status"
    assert b"sm_100a" in lib.ssm_version()


def test_workspace_sizes(lib):
    # 370m-shaped layer: enough channels, no time split, no scratch
    assert lib.ssm_scan_fwd_workspace_size(8, 2048, 2048, 16, 1) == 0
    # a long sequence over few channels needs chunk summaries
    assert lib.ssm_scan_fwd_workspace_size(1, 256, 1 << 20, 16, 1) > 0
    assert lib.ssm_scan_fwd_workspace_size(0, 256, 1024, 16, 1) == 0     # invalid -> 0
    with_ck = lib.ssm_scan_bwd_workspace_size(4, 5120, 2048, 16, 1, 1)
    without = lib.ssm_scan_bwd_workspace_size(4, 5120, 2048, 16, 1, 0)
    assert 0 < with_ck < without
    assert without - with_ck >= 4 * 5120 * 128 * 16 * 4


def _fwd(lib, **kw):
    args = dict(u=None, delta=None, A=None, B=None, C=None, D=None, z=None, dt_bias=None, sp=1,
                h0=None, hL=None, out=None, ckpt=None, ws=None, wsb=0, batch=1, dim=64, L=256,
                N=16, io=1, stream=None)
    args.update(kw)
    return lib.ssm_scan_fwd(*args.values())


def test_invalid_arguments_are_rejected_on_the_host(lib):
    # nothing here reaches a kernel: every call fails validation before any launch
    assert _fwd(lib) == _abi.SSM_EINVAL                       # NULL inputs
    assert b"NULL" in lib.ssm_last_error()
    assert _fwd(lib, batch=0) == _abi.SSM_EINVAL
    assert _fwd(lib, io=7) == _abi.SSM_EINVAL
    assert _fwd(lib, N=17) == _abi.SSM_EUNSUPPORTED
    fake = ctypes.c_void_p(0x1001)                             # misaligned for bf16
    assert _fwd(lib, u=fake) == _abi.SSM_EINVAL
    assert b"aligned" in lib.ssm_last_error()
    assert lib.ssm_state_update(*([None] * 9), 1, None, 1, 1, 16, 1, None) == _abi.SSM_EINVAL
    rc = lib.ssm_scan_bwd(*([None] * 8), 1, *([None] * 14), 0, 1, 64, 256, 16, 1, None)
    assert rc == _abi.SSM_EINVAL


def test_host_pageable_pointer_is_rejected(lib):
    """A pageable host buffer must be refused before any kernel could dereference it (on a
    machine without a GPU the pointer query itself fails, which is refused the same way)."""
    buf = (ctypes.c_uint16 * (64 * 256))()
    p = ctypes.cast(buf, ctypes.c_void_p)
    assert _fwd(lib, u=p, delta=p, A=p, B=p, C=p, out=p) == _abi.SSM_EINVAL


def _fwd_ex(lib, flags=0, groups=1, **kw):
    args = dict(u=None, delta=None, A=None, B=None, C=None, D=None, z=None, dt_bias=None, sp=1,
                h0=None, hL=None, out=None, ckpt=None, ws=None, wsb=0, batch=1, dim=64, L=256,
                N=16, groups=groups, io=1, flags=flags, stream=None)
    args.update(kw)
    return lib.ssm_scan_fwd_ex(*args.values())


def _bwd_ex(lib, flags=0, groups=1, dim=64):
    return lib.ssm_scan_bwd_ex(*([None] * 8), 1, *([None] * 14), 0, 1, dim, 256, 16, groups, 1,
                               flags, None)


def test_variant_flags_and_groups_are_checked_on_the_host(lib, monkeypatch):
    """The _ex entry points refuse unknown flag bits and unusable B/C groupings before touching
    any pointer (nothing here needs a GPU)."""
    known = _abi.SSM_SCALAR_A | _abi.SSM_REVERSE | _abi.SSM_ZOH | _abi.SSM_CHANNELS_LAST
    assert _fwd_ex(lib, flags=16) == _abi.SSM_EINVAL
    assert b"flags" in lib.ssm_last_error()
    assert _bwd_ex(lib, flags=32) == _abi.SSM_EINVAL
    assert _fwd_ex(lib, groups=0) == _abi.SSM_EINVAL
    assert _fwd_ex(lib, groups=3) == _abi.SSM_EINVAL               # 64 channels, 3 groups
    assert _fwd_ex(lib, groups=8) == _abi.SSM_EUNSUPPORTED         # 8 channels per group
    assert b"multiple of 16" in lib.ssm_last_error()
    assert _bwd_ex(lib, groups=8) == _abi.SSM_EUNSUPPORTED
    # known flags with valid groups get past these checks (and stop at the NULL inputs)
    assert _fwd_ex(lib, flags=known, groups=4) == _abi.SSM_EINVAL
    assert b"NULL" in lib.ssm_last_error()
    assert lib.ssm_scan_fwd_ex_workspace_size(1, 256, 1 << 20, 16, 1, 1, known) > 0
    assert lib.ssm_scan_bwd_ex_workspace_size(4, 5120, 2048, 16, 8, 1, 1, 0) > 0
    assert lib.ssm_scan_bwd_ex_workspace_size(4, 64, 2048, 16, 8, 1, 1, 0) == 0   # bad groups
    # on the per-state kernel the scalar decay adds the broadcast rate and per-state dA to the
    # backward's workspace
    monkeypatch.setenv("SSM_SCALAR_BWD", "state")
    base = lib.ssm_scan_bwd_ex_workspace_size(4, 5120, 2048, 16, 1, 1, 1, 0)
    sa = lib.ssm_scan_bwd_ex_workspace_size(4, 5120, 2048, 16, 1, 1, 1, _abi.SSM_SCALAR_A)
    assert sa - base == 2 * 5120 * 16 * 4
    # the chunked form (bf16): given checkpoints, it needs no room for them (4 x 5120 x 128
    # chunks x 16 states of f32)
    monkeypatch.delenv("SSM_SCALAR_BWD")
    given = lib.ssm_scan_bwd_ex_workspace_size(4, 5120, 2048, 16, 1, 1, 1, _abi.SSM_SCALAR_A)
    own = lib.ssm_scan_bwd_ex_workspace_size(4, 5120, 2048, 16, 1, 1, 0, _abi.SSM_SCALAR_A)
    assert 0 < given and own - given >= 4 * 5120 * 128 * 16 * 4


def test_decode_variants_refuse_the_reverse_flag(lib):
    rc = lib.ssm_state_update_ex(*([None] * 9), 1, None, 1, 64, 16, 1, 1, _abi.SSM_REVERSE, None)
    assert rc == _abi.SSM_EINVAL
    rc = lib.ssm_state_update_ex(*([None] * 9), 1, None, 1, 64, 16, 8, 1, 0, None)
    assert rc == _abi.SSM_EUNSUPPORTED                              # 8 channels per group


def test_host_memory_call_checks_shape_and_workspace(lib):
    assert lib.ssm_scan_fwd_host_workspace_size(0, 64, 256, 16, 1) == 0
    need = lib.ssm_scan_fwd_host_workspace_size(8, 2048, 2048, 16, 1)
    assert need >= 2 * 4 * 2048 * 2048 * 2                          # two slots of u, delta, z, out
    buf = (ctypes.c_uint16 * 16)()
    p = ctypes.cast(buf, ctypes.c_void_p)
    rc = lib.ssm_scan_fwd_host(p, p, None, p, p, None, None, None, 1, None, None, p, None, 0,
                               8, 2048, 2048, 16, 1, None)
    assert rc == _abi.SSM_EWORKSPACE
    rc = lib.ssm_scan_fwd_host(None, p, None, p, p, None, None, None, 1, None, None, p, None, 0,
                               8, 2048, 2048, 16, 1, None)
    assert rc == _abi.SSM_EINVAL


def test_binding_rejects_host_tensors_before_any_cuda_call():
    """The Python entry points refuse CPU tensors with a ValueError of their own (they never
    reach the CUDA runtime or the library with a host pointer)."""
    import torch
    import selective_state_space_23_b200 as ssm
    from selective_state_space_23_b200.inputs import make_inputs, workload
    x = make_inputs(workload("tiny_f32"), seed=0, with_dout=True)
    calls = {
        "fwd": lambda: ssm.ssm_scan_fwd(x["u"], x["delta"], x["A"], x["B"], x["C"]),
        "fwd_cl": lambda: ssm.ssm_scan_fwd(x["u"], x["delta"], x["A"], x["B"], x["C"],
                                           channels_last=True),
        "bwd": lambda: ssm.ssm_scan_bwd(x["u"], x["delta"], x["A"], x["B"], x["C"], x["dout"]),
        "decode": lambda: ssm.ssm_state_update(torch.zeros(1, 64, 16), x["u"][:, :, 0],
                                               x["delta"][:, :, 0], x["A"], x["B"][:, :, 0],
                                               x["C"][:, :, 0]),
        "host": lambda: ssm.ssm_scan_fwd_host(x["u"], x["delta"], x["A"], x["B"], x["C"]),
    }
    for name, f in calls.items():
        with pytest.raises(ValueError, match="must be a CUDA tensor"):
            f()


def test_wait_timeout_query_rejects_null(lib):
    assert lib.ssm_wait_timeouts(None) == _abi.SSM_EINVAL
    assert b"NULL" in lib.ssm_last_error()


def test_strided_entry_points_check_on_the_host(lib):
    """The strided forms refuse a missing stride table, the channels-last flag (a layout the
    strides already express) and a missing workspace before any pointer is touched."""
    st = _abi.Strides()
    assert lib.ssm_scan_fwd_strided_workspace_size(2, 64, 256, 16, 1, 1, 0) > 0
    assert lib.ssm_scan_fwd_strided_workspace_size(2, 64, 256, 16, 1, 1,
                                                   _abi.SSM_CHANNELS_LAST) == 0
    assert lib.ssm_scan_bwd_strided_workspace_size(2, 64, 256, 16, 1, 1, 0, 0) > 0
    assert lib.ssm_state_update_strided_workspace_size(2, 64, 16, 1, 1) > 0
    args = [None] * 8 + [1] + [None] * 5 + [0, 2, 64, 256, 16, 1, 1]
    assert lib.ssm_scan_fwd_strided(*args, 0, None, None) == _abi.SSM_EINVAL   # strides NULL
    assert lib.ssm_scan_fwd_strided(*args, _abi.SSM_CHANNELS_LAST, ctypes.byref(st),
                                    None) == _abi.SSM_EINVAL
    assert lib.ssm_scan_fwd_strided(*args, 0, ctypes.byref(st), None) == _abi.SSM_EWORKSPACE
    bargs = [None] * 8 + [1] + [None] * 14 + [0, 2, 64, 256, 16, 1, 1, 0]
    assert lib.ssm_scan_bwd_strided(*bargs, None, None) == _abi.SSM_EINVAL
    dst = _abi.DecodeStrides()
    dargs = [None] * 9 + [1, None, None, 0, 2, 64, 16, 1, 1]
    assert lib.ssm_state_update_strided(*dargs, _abi.SSM_REVERSE, ctypes.byref(dst),
                                        None) == _abi.SSM_EINVAL
    assert lib.ssm_state_update_strided(*dargs, 0, ctypes.byref(dst), None) == _abi.SSM_EWORKSPACE


def test_large_n_decode_is_checked_on_the_host(lib):
    """Decode steps: per-state rates stop at 16 states; one rate per channel takes 32, 64 or 128
    (refused before any launch)."""
    assert lib.ssm_state_update_ex(*([None] * 9), 1, None, 2, 64, 64, 1, 1, 0, None) == \
        _abi.SSM_EUNSUPPORTED
    assert lib.ssm_state_update_ex(*([None] * 9), 1, None, 2, 64, 48, 1, 1, _abi.SSM_SCALAR_A,
                                   None) == _abi.SSM_EUNSUPPORTED
    assert b"32, 64 or 128" in lib.ssm_last_error()


def test_large_n_workspace_queries(lib):
    """Scalar decay with N > 16: the forward and summary queries cover the path each call takes
    (bf16: the chunked matrix form, N = 32, 64, 128; f32: 16-state slices, any multiple of 16 up
    to 128); other sizes ask for nothing because the call refuses them."""
    sa = _abi.SSM_SCALAR_A
    for io in (_abi.SSM_BF16, _abi.SSM_F32):
        for N in (32, 64, 128):
            assert lib.ssm_scan_fwd_summary_workspace_size(1, 64, 400, N, 1, io, sa) > 0
            assert lib.ssm_scan_fwd_scalar_a_workspace_size(1, 64, 4096, N, io) > 0
    assert lib.ssm_scan_fwd_summary_workspace_size(1, 64, 400, 48, 1, _abi.SSM_F32, sa) > 0
    assert lib.ssm_scan_fwd_summary_workspace_size(1, 64, 400, 48, 1, _abi.SSM_BF16, sa) == 0
    assert lib.ssm_scan_fwd_summary_workspace_size(1, 64, 400, 40, 1, _abi.SSM_F32, sa) == 0
    assert lib.ssm_scan_fwd_summary_workspace_size(1, 64, 400, 64, 1, _abi.SSM_BF16, 0) == 0
    # the f32 slice forward holds slice copies of B, C and one slice's output at least
    f32 = lib.ssm_scan_fwd_ex_workspace_size(2, 64, 256, 64, 1, _abi.SSM_F32, sa)
    assert f32 >= 2 * 2 * 16 * 256 * 4 + 2 * 64 * 256 * 4
