"""B200-native selective state-space (S6) scan: Python binding of libssm_b200.so.

The three entry points mirror the C ABI (include/ssm_scan.h) and do argument marshalling only:
every step of the computation runs in the library's sm_100a kernels.  Tensors are torch CUDA
tensors (PyTorch provides device memory and streams); outputs not supplied by the caller are
allocated here with torch.  Work is enqueued on the current torch CUDA stream.

  ssm_scan_fwd      forward selective scan (gated output, optional final state / checkpoints)
  ssm_scan_bwd      gradients of ssm_scan_fwd, recomputing the states
  ssm_state_update  one-token recurrent step, state updated in place

with variants (``*_scalar_a``, flags), the host-memory forward ``ssm_scan_fwd_host`` and the
``*_strided`` forms that take io tensors with arbitrary element strides.
"""
import ctypes

import torch

from . import _abi
from ._abi import CKPT_STEPS, MAX_DSTATE

__all__ = ["ssm_scan_fwd", "ssm_scan_bwd", "ssm_scan_fwd_scalar_a", "ssm_scan_bwd_scalar_a",
           "ssm_scan_fwd_host", "fwd_host_workspace_bytes",
           "ssm_state_update", "fwd_workspace_bytes", "ssm_scan_fwd_strided",
           "ssm_scan_bwd_strided", "ssm_state_update_strided", "ssm_scan_fwd_summary",
           "ssm_scan_chain",
           "bwd_workspace_bytes", "CKPT_STEPS", "MAX_DSTATE", "library_path"]

_IO = {torch.float32: _abi.SSM_F32, torch.bfloat16: _abi.SSM_BF16}


def library_path() -> str:
    _abi.lib()
    return _abi.LIB_PATH


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _need(t, name, shape, dtype, device):
    if t is None:
        raise ValueError(f"{name} is required")
    _opt(t, name, shape, dtype, device)


def _opt(t, name, shape, dtype, device):
    if t is None:
        return
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _on_gpu(t, name):
    """The tensor's device, which must be a CUDA device (the library has no host path)."""
    if not isinstance(t, torch.Tensor) or t.device.type != "cuda":
        where = t.device if isinstance(t, torch.Tensor) else type(t).__name__
        raise ValueError(f"{name} must be a CUDA tensor, got {where} (host tensors: "
                         "ssm_scan_fwd_host)")
    return t.device


def _io_code(dtype):
    if dtype not in _IO:
        raise TypeError(f"io dtype must be float32 or bfloat16, got {dtype}")
    return _IO[dtype]


def fwd_workspace_bytes(batch, dim, seqlen, dstate, dtype) -> int:
    return int(_abi.lib().ssm_scan_fwd_workspace_size(batch, dim, seqlen, dstate, _io_code(dtype)))


def bwd_workspace_bytes(batch, dim, seqlen, dstate, dtype, have_ckpt) -> int:
    return int(_abi.lib().ssm_scan_bwd_workspace_size(batch, dim, seqlen, dstate, _io_code(dtype),
                                                       int(bool(have_ckpt))))


def _workspace(nbytes, device, given):
    if nbytes == 0:
        return None
    if given is not None:
        if given.device != device or given.numel() * given.element_size() < nbytes:
            raise ValueError(f"workspace must hold {nbytes} bytes on {device}")
        return given
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def _bc_layout(B, batch, L, channels_last=False):
    """(groups, N, shape) of the B/C layout: [batch, N, L] (one group) or [batch, G, N, L];
    channels last: [batch, L, N] or [batch, L, G, N]."""
    if not isinstance(B, torch.Tensor):
        raise TypeError("B must be a torch.Tensor")
    if channels_last:
        if B.dim() == 3:
            return 1, B.shape[2], (batch, L, B.shape[2])
        if B.dim() == 4:
            return B.shape[2], B.shape[3], (batch, L, B.shape[2], B.shape[3])
        raise ValueError(f"B must be [batch, L, N] or [batch, L, groups, N], got {tuple(B.shape)}")
    if B.dim() == 3:
        return 1, B.shape[1], (batch, B.shape[1], L)
    if B.dim() == 4:
        return B.shape[1], B.shape[2], (batch, B.shape[1], B.shape[2], L)
    raise ValueError(f"B must be [batch, N, L] or [batch, groups, N, L], got {tuple(B.shape)}")


def _flags(scalar_a, reverse, zoh, channels_last=False):
    return ((_abi.SSM_SCALAR_A if scalar_a else 0) | (_abi.SSM_REVERSE if reverse else 0)
            | (_abi.SSM_ZOH if zoh else 0) | (_abi.SSM_CHANNELS_LAST if channels_last else 0))


def _scan_fwd(u, delta, A, B, C, D, z, dt_bias, delta_softplus, h0, return_final_state,
              return_ckpt, out, workspace, scalar_a, reverse, zoh, channels_last=False):
    dev = _on_gpu(u, "u")
    if channels_last:
        batch, L, dim = u.shape
    else:
        batch, dim, L = u.shape
    xs = (batch, L, dim) if channels_last else (batch, dim, L)
    G, N, bc_shape = _bc_layout(B, batch, L, channels_last)
    io = u.dtype
    code = _io_code(io)
    _need(u, "u", xs, io, dev)
    _need(delta, "delta", xs, io, dev)
    _need(A, "A", (dim,) if scalar_a else (dim, N), torch.float32, dev)
    _need(B, "B", bc_shape, io, dev)
    _need(C, "C", bc_shape, io, dev)
    _opt(D, "D", (dim,), torch.float32, dev)
    _opt(z, "z", xs, io, dev)
    _opt(dt_bias, "dt_bias", (dim,), torch.float32, dev)
    _opt(h0, "h0", (batch, dim, N), torch.float32, dev)
    if out is None:
        out = torch.empty(xs, dtype=io, device=dev)
    _need(out, "out", xs, io, dev)
    hL = torch.empty((batch, dim, N), dtype=torch.float32, device=dev) if return_final_state else None
    nblk = (L + CKPT_STEPS - 1) // CKPT_STEPS
    ckpt = torch.empty((batch, dim, nblk, N), dtype=torch.float32, device=dev) if return_ckpt else None
    flags = _flags(scalar_a, reverse, zoh, channels_last)
    nws = int(_abi.lib().ssm_scan_fwd_ex_workspace_size(batch, dim, L, N, G, code, flags))
    ws = _workspace(nws, dev, workspace)
    rc = _abi.lib().ssm_scan_fwd_ex(
        _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(dt_bias),
        int(bool(delta_softplus)), _ptr(h0), _ptr(hL), _ptr(out), _ptr(ckpt), _ptr(ws),
        0 if ws is None else ws.numel(), batch, dim, L, N, G, code, flags, _stream(dev))
    _abi.check(rc, "ssm_scan_fwd_ex")
    if not return_final_state and not return_ckpt:
        return out
    res = (out,)
    if return_final_state:
        res += (hL,)
    if return_ckpt:
        res += (ckpt,)
    return res


def ssm_scan_fwd(u, delta, A, B, C, D=None, z=None, dt_bias=None, delta_softplus=True, h0=None,
                 return_final_state=False, return_ckpt=False, out=None, workspace=None,
                 reverse=False, zoh=False, channels_last=False):
    """Forward scan.  u, delta, z: [batch, dim, L]; B, C: [batch, N, L] or, grouped, [batch, G,
    N, L] (channel d uses group d // (dim // G)) (io dtype f32 or bf16); A: [dim, N] f32; D, dt_bias: [dim] f32; h0: [batch, dim, N] f32.  reverse: scan from
    t = L-1 down to 0.  zoh: zero-order-hold input term (e^{ΔA} - 1)/A B x instead of Δ B x.
    channels_last: the (B, L, D) layout (u, delta, z, out [batch, L, dim]; B, C [batch, L, N]
    or [batch, L, G, N]).  Returns out, or a tuple (out, hL?, ckpt?) when those are requested."""
    return _scan_fwd(u, delta, A, B, C, D, z, dt_bias, delta_softplus, h0, return_final_state,
                     return_ckpt, out, workspace, False, reverse, zoh, channels_last)


def ssm_scan_fwd_scalar_a(u, delta, A, B, C, D=None, z=None, dt_bias=None, delta_softplus=True,
                          h0=None, return_final_state=False, return_ckpt=False, out=None,
                          workspace=None, reverse=False, zoh=False, channels_last=False):
    """Forward scan with one decay rate per channel: as :func:`ssm_scan_fwd` with A [dim] f32."""
    return _scan_fwd(u, delta, A, B, C, D, z, dt_bias, delta_softplus, h0, return_final_state,
                     return_ckpt, out, workspace, True, reverse, zoh, channels_last)


def _scan_bwd(u, delta, A, B, C, dout, D, z, dt_bias, delta_softplus, h0, dhL, ckpt,
              workspace, need, scalar_a, reverse, zoh, channels_last=False):
    dev = _on_gpu(u, "u")
    if channels_last:
        batch, L, dim = u.shape
    else:
        batch, dim, L = u.shape
    xs = (batch, L, dim) if channels_last else (batch, dim, L)
    G, N, bc_shape = _bc_layout(B, batch, L, channels_last)
    io = u.dtype
    code = _io_code(io)
    _need(u, "u", xs, io, dev)
    _need(delta, "delta", xs, io, dev)
    a_shape = (dim,) if scalar_a else (dim, N)
    _need(A, "A", a_shape, torch.float32, dev)
    _need(B, "B", bc_shape, io, dev)
    _need(C, "C", bc_shape, io, dev)
    _need(dout, "dout", xs, io, dev)
    _opt(D, "D", (dim,), torch.float32, dev)
    _opt(z, "z", xs, io, dev)
    _opt(dt_bias, "dt_bias", (dim,), torch.float32, dev)
    _opt(h0, "h0", (batch, dim, N), torch.float32, dev)
    _opt(dhL, "dhL", (batch, dim, N), torch.float32, dev)
    nblk = (L + CKPT_STEPS - 1) // CKPT_STEPS
    _opt(ckpt, "ckpt", (batch, dim, nblk, N), torch.float32, dev)
    want = set(need) if need is not None else {"du", "ddelta", "dA", "dB", "dC", "dD", "dz",
                                                "ddt_bias", "dh0"}
    e = lambda shape, dt: torch.empty(shape, dtype=dt, device=dev)
    g = {
        "du": e(xs, io) if "du" in want else None,
        "ddelta": e(xs, io) if "ddelta" in want else None,
        "dz": e(xs, io) if ("dz" in want and z is not None) else None,
        "dB": e(bc_shape, io) if "dB" in want else None,
        "dC": e(bc_shape, io) if "dC" in want else None,
        "dA": e(a_shape, torch.float32) if "dA" in want else None,
        "dD": e((dim,), torch.float32) if "dD" in want else None,
        "ddt_bias": e((dim,), torch.float32) if "ddt_bias" in want else None,
        "dh0": e((batch, dim, N), torch.float32) if "dh0" in want else None,
    }
    flags = _flags(scalar_a, reverse, zoh, channels_last)
    nws = int(_abi.lib().ssm_scan_bwd_ex_workspace_size(batch, dim, L, N, G, code,
                                                         int(ckpt is not None), flags))
    ws = _workspace(nws, dev, workspace)
    rc = _abi.lib().ssm_scan_bwd_ex(
        _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(dt_bias),
        int(bool(delta_softplus)), _ptr(h0), _ptr(dout), _ptr(dhL), _ptr(ckpt),
        _ptr(g["du"]), _ptr(g["ddelta"]), _ptr(g["dA"]), _ptr(g["dB"]), _ptr(g["dC"]),
        _ptr(g["dD"]), _ptr(g["dz"]), _ptr(g["ddt_bias"]), _ptr(g["dh0"]),
        _ptr(ws), 0 if ws is None else ws.numel(), batch, dim, L, N, G, code, flags,
        _stream(dev))
    _abi.check(rc, "ssm_scan_bwd_ex")
    return g


def ssm_scan_bwd(u, delta, A, B, C, dout, D=None, z=None, dt_bias=None, delta_softplus=True,
                 h0=None, dhL=None, ckpt=None, workspace=None, need=None, reverse=False,
                 zoh=False, channels_last=False):
    """Gradients of :func:`ssm_scan_fwd`.  Returns a dict with du, ddelta, dA, dB, dC, dD, dz,
    ddt_bias, dh0 (entries are None when the matching input is absent or not in ``need``)."""
    return _scan_bwd(u, delta, A, B, C, dout, D, z, dt_bias, delta_softplus, h0, dhL, ckpt,
                     workspace, need, False, reverse, zoh, channels_last)


def ssm_scan_bwd_scalar_a(u, delta, A, B, C, dout, D=None, z=None, dt_bias=None,
                          delta_softplus=True, h0=None, dhL=None, ckpt=None, workspace=None,
                          need=None, reverse=False, zoh=False, channels_last=False):
    """Gradients of :func:`ssm_scan_fwd_scalar_a` (dA is [dim])."""
    return _scan_bwd(u, delta, A, B, C, dout, D, z, dt_bias, delta_softplus, h0, dhL, ckpt,
                     workspace, need, True, reverse, zoh, channels_last)


def _host(t, name, shape, dtype):
    if t is None:
        return
    if not isinstance(t, torch.Tensor) or t.device.type != "cpu":
        raise ValueError(f"{name} must be a CPU tensor")
    if tuple(t.shape) != tuple(shape) or t.dtype != dtype or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous {dtype} tensor of shape {tuple(shape)}")


def ssm_scan_fwd_host(u, delta, A, B, C, D=None, z=None, dt_bias=None, delta_softplus=True,
                      h0=None, return_final_state=False, out=None, workspace=None):
    """Forward scan from and to host memory: u, delta, z, B, C (and h0) are CPU tensors (pinned
    memory lets the copies overlap the scan), A, D, dt_bias live on the GPU.  The batch flows
    through copy-in, scan and copy-out streams in chunks of rows.  Returns out (CPU), or
    (out, hL) with ``return_final_state``; both are complete once the current stream of A's
    device has reached this call."""
    dev = _on_gpu(A, "A")
    batch, dim, L = u.shape
    N = A.shape[-1]
    io = u.dtype
    code = _io_code(io)
    for t, n, shp in ((u, "u", (batch, dim, L)), (delta, "delta", (batch, dim, L)),
                      (z, "z", (batch, dim, L)), (B, "B", (batch, N, L)), (C, "C", (batch, N, L))):
        _host(t, n, shp, io)
    _host(h0, "h0", (batch, dim, N), torch.float32)
    _need(A, "A", (dim, N), torch.float32, dev)
    _opt(D, "D", (dim,), torch.float32, dev)
    _opt(dt_bias, "dt_bias", (dim,), torch.float32, dev)
    pin = u.is_pinned()
    if out is None:
        out = torch.empty((batch, dim, L), dtype=io, pin_memory=pin)
    _host(out, "out", (batch, dim, L), io)
    hL = torch.empty((batch, dim, N), dtype=torch.float32, pin_memory=pin) if return_final_state else None
    nws = int(_abi.lib().ssm_scan_fwd_host_workspace_size(batch, dim, L, N, code))
    ws = _workspace(nws, dev, workspace)
    rc = _abi.lib().ssm_scan_fwd_host(
        _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(dt_bias),
        int(bool(delta_softplus)), _ptr(h0), _ptr(hL), _ptr(out), _ptr(ws),
        0 if ws is None else ws.numel(), batch, dim, L, N, code, _stream(dev))
    _abi.check(rc, "ssm_scan_fwd_host")
    return (out, hL) if return_final_state else out


def fwd_host_workspace_bytes(batch, dim, seqlen, dstate, dtype) -> int:
    return int(_abi.lib().ssm_scan_fwd_host_workspace_size(batch, dim, seqlen, dstate,
                                                            _io_code(dtype)))


def ssm_state_update(state, x, dt, A, B, C, D=None, z=None, dt_bias=None, delta_softplus=True,
                     out=None, scalar_a=False, zoh=False):
    """One decode step; ``state`` [batch, dim, N] f32 is updated in place.  x, dt, z:
    [batch, dim]; B, C: [batch, N] or, grouped, [batch, G, N] (io dtype); A: [dim, N] f32, or
    [dim] with ``scalar_a``; ``zoh``: zero-order-hold input coefficient.  Returns out [batch, dim]."""
    dev = _on_gpu(state, "state")
    batch, dim, N = state.shape
    io = x.dtype
    code = _io_code(io)
    if not isinstance(B, torch.Tensor):
        raise TypeError("B must be a torch.Tensor")
    G = B.shape[1] if B.dim() == 3 else 1
    bc_shape = (batch, G, N) if B.dim() == 3 else (batch, N)
    _need(state, "state", (batch, dim, N), torch.float32, dev)
    _need(x, "x", (batch, dim), io, dev)
    _need(dt, "dt", (batch, dim), io, dev)
    _need(A, "A", (dim,) if scalar_a else (dim, N), torch.float32, dev)
    _need(B, "B", bc_shape, io, dev)
    _need(C, "C", bc_shape, io, dev)
    _opt(D, "D", (dim,), torch.float32, dev)
    _opt(z, "z", (batch, dim), io, dev)
    _opt(dt_bias, "dt_bias", (dim,), torch.float32, dev)
    if out is None:
        out = torch.empty((batch, dim), dtype=io, device=dev)
    _need(out, "out", (batch, dim), io, dev)
    flags = _flags(scalar_a, False, zoh)
    rc = _abi.lib().ssm_state_update_ex(
        _ptr(state), _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z),
        _ptr(dt_bias), int(bool(delta_softplus)), _ptr(out), batch, dim, N, G, code, flags,
        _stream(dev))
    _abi.check(rc, "ssm_state_update_ex")
    return out


# ------------------------------------------------------------------ general element strides
def _view(t, name, shape, dtype, device):
    """A tensor of the given logical shape with any non-negative element strides."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def _bc_view(B, batch, L):
    """(groups, N, strides (batch, group, state, t)) of B/C given as [batch, N, L] or
    [batch, G, N, L] with any strides."""
    if B.dim() == 3:
        return 1, B.shape[1], (B.stride(0), 0, B.stride(1), B.stride(2))
    if B.dim() == 4:
        return B.shape[1], B.shape[2], tuple(B.stride())
    raise ValueError(f"B must be [batch, N, L] or [batch, groups, N, L], got {tuple(B.shape)}")


def _set(arr, vals):
    for i, v in enumerate(vals):
        arr[i] = v


def ssm_scan_fwd_strided(u, delta, A, B, C, D=None, z=None, dt_bias=None, delta_softplus=True,
                         h0=None, return_final_state=False, out=None, workspace=None,
                         scalar_a=False, reverse=False, zoh=False):
    """:func:`ssm_scan_fwd` for io tensors with arbitrary (non-negative) element strides: u,
    delta, z (and ``out``, if given) [batch, dim, L]; B, C [batch, N, L] or [batch, G, N, L]
    (e.g. expanded over the batch with stride 0).  Results equal the dense call's bitwise."""
    dev = _on_gpu(u, "u")
    batch, dim, L = u.shape
    io = u.dtype
    code = _io_code(io)
    G, N, sbc = _bc_view(B, batch, L)
    xs = (batch, dim, L)
    bshape = tuple(B.shape)
    for t, n in ((u, "u"), (delta, "delta")):
        _view(t, n, xs, io, dev)
    if z is not None:
        _view(z, "z", xs, io, dev)
    _view(B, "B", bshape, io, dev)
    _view(C, "C", bshape, io, dev)
    _need(A, "A", (dim,) if scalar_a else (dim, N), torch.float32, dev)
    _opt(D, "D", (dim,), torch.float32, dev)
    _opt(dt_bias, "dt_bias", (dim,), torch.float32, dev)
    _opt(h0, "h0", (batch, dim, N), torch.float32, dev)
    if out is None:
        out = torch.empty(xs, dtype=io, device=dev)
    _view(out, "out", xs, io, dev)
    hL = torch.empty((batch, dim, N), dtype=torch.float32, device=dev) if return_final_state else None
    st = _abi.Strides()
    _set(st.u, u.stride())
    _set(st.delta, delta.stride())
    if z is not None:
        _set(st.z, z.stride())
    _set(st.out, out.stride())
    _set(st.B, sbc)
    _set(st.C, _bc_view(C, batch, L)[2])
    flags = _flags(scalar_a, reverse, zoh)
    nws = int(_abi.lib().ssm_scan_fwd_strided_workspace_size(batch, dim, L, N, G, code, flags))
    ws = _workspace(nws, dev, workspace)
    rc = _abi.lib().ssm_scan_fwd_strided(
        _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(dt_bias),
        int(bool(delta_softplus)), _ptr(h0), _ptr(hL), _ptr(out), None, _ptr(ws),
        0 if ws is None else ws.numel(), batch, dim, L, N, G, code, flags, ctypes.byref(st),
        _stream(dev))
    _abi.check(rc, "ssm_scan_fwd_strided")
    return (out, hL) if return_final_state else out


def ssm_scan_bwd_strided(u, delta, A, B, C, dout, D=None, z=None, dt_bias=None,
                         delta_softplus=True, h0=None, dhL=None, grads=None, workspace=None,
                         scalar_a=False, reverse=False, zoh=False):
    """:func:`ssm_scan_bwd` for io tensors with arbitrary element strides (u, delta, z, dout,
    B, C as in :func:`ssm_scan_fwd_strided`).  ``grads`` may supply any of du, ddelta, dz, dB,
    dC as strided output tensors (the others are allocated dense).  Returns the gradient dict."""
    dev = _on_gpu(u, "u")
    batch, dim, L = u.shape
    io = u.dtype
    code = _io_code(io)
    G, N, sbc = _bc_view(B, batch, L)
    xs = (batch, dim, L)
    bshape = tuple(B.shape)
    for t, n in ((u, "u"), (delta, "delta"), (dout, "dout")):
        _view(t, n, xs, io, dev)
    if z is not None:
        _view(z, "z", xs, io, dev)
    _view(B, "B", bshape, io, dev)
    _view(C, "C", bshape, io, dev)
    a_shape = (dim,) if scalar_a else (dim, N)
    _need(A, "A", a_shape, torch.float32, dev)
    _opt(D, "D", (dim,), torch.float32, dev)
    _opt(dt_bias, "dt_bias", (dim,), torch.float32, dev)
    _opt(h0, "h0", (batch, dim, N), torch.float32, dev)
    _opt(dhL, "dhL", (batch, dim, N), torch.float32, dev)
    given = dict(grads or {})
    e = lambda shape, dt: torch.empty(shape, dtype=dt, device=dev)
    g = {"du": given.get("du", e(xs, io)), "ddelta": given.get("ddelta", e(xs, io)),
         "dz": given.get("dz", e(xs, io)) if z is not None else None,
         "dB": given.get("dB", e(bshape, io)), "dC": given.get("dC", e(bshape, io)),
         "dA": e(a_shape, torch.float32), "dD": e((dim,), torch.float32),
         "ddt_bias": e((dim,), torch.float32), "dh0": e((batch, dim, N), torch.float32)}
    for k in ("du", "ddelta", "dz"):
        if g[k] is not None:
            _view(g[k], k, xs, io, dev)
    for k in ("dB", "dC"):
        _view(g[k], k, bshape, io, dev)
    st = _abi.Strides()
    for k, t in (("u", u), ("delta", delta), ("z", z), ("dout", dout), ("du", g["du"]),
                 ("ddelta", g["ddelta"]), ("dz", g["dz"])):
        if t is not None:
            _set(getattr(st, k), t.stride())
    for k, t in (("B", B), ("C", C), ("dB", g["dB"]), ("dC", g["dC"])):
        _set(getattr(st, k), _bc_view(t, batch, L)[2])
    flags = _flags(scalar_a, reverse, zoh)
    nws = int(_abi.lib().ssm_scan_bwd_strided_workspace_size(batch, dim, L, N, G, code, 0, flags))
    ws = _workspace(nws, dev, workspace)
    rc = _abi.lib().ssm_scan_bwd_strided(
        _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(dt_bias),
        int(bool(delta_softplus)), _ptr(h0), _ptr(dout), _ptr(dhL), None,
        _ptr(g["du"]), _ptr(g["ddelta"]), _ptr(g["dA"]), _ptr(g["dB"]), _ptr(g["dC"]),
        _ptr(g["dD"]), _ptr(g["dz"]), _ptr(g["ddt_bias"]), _ptr(g["dh0"]),
        _ptr(ws), 0 if ws is None else ws.numel(), batch, dim, L, N, G, code, flags,
        ctypes.byref(st), _stream(dev))
    _abi.check(rc, "ssm_scan_bwd_strided")
    return g


def ssm_state_update_strided(state, x, dt, A, B, C, D=None, z=None, dt_bias=None,
                             delta_softplus=True, out=None, scalar_a=False, zoh=False,
                             workspace=None):
    """:func:`ssm_state_update` for tensors with arbitrary element strides: state [batch, dim,
    N] f32 (updated in place), x, dt, z, out [batch, dim], B, C [batch, N] or [batch, G, N]."""
    dev = _on_gpu(state, "state")
    batch, dim, N = state.shape
    io = x.dtype
    code = _io_code(io)
    if not isinstance(B, torch.Tensor):
        raise TypeError("B must be a torch.Tensor")
    G = B.shape[1] if B.dim() == 3 else 1
    bshape = tuple(B.shape)
    sbc = lambda t: tuple(t.stride()) if t.dim() == 3 else (t.stride(0), 0, t.stride(1))
    _view(state, "state", (batch, dim, N), torch.float32, dev)
    for t, n in ((x, "x"), (dt, "dt")):
        _view(t, n, (batch, dim), io, dev)
    if z is not None:
        _view(z, "z", (batch, dim), io, dev)
    _view(B, "B", bshape, io, dev)
    _view(C, "C", bshape, io, dev)
    _need(A, "A", (dim,) if scalar_a else (dim, N), torch.float32, dev)
    _opt(D, "D", (dim,), torch.float32, dev)
    _opt(dt_bias, "dt_bias", (dim,), torch.float32, dev)
    if out is None:
        out = torch.empty((batch, dim), dtype=io, device=dev)
    _view(out, "out", (batch, dim), io, dev)
    st = _abi.DecodeStrides()
    _set(st.state, state.stride())
    _set(st.x, x.stride())
    _set(st.dt, dt.stride())
    if z is not None:
        _set(st.z, z.stride())
    _set(st.out, out.stride())
    _set(st.B, sbc(B))
    _set(st.C, sbc(C))
    nws = int(_abi.lib().ssm_state_update_strided_workspace_size(batch, dim, N, G, code))
    ws = _workspace(nws, dev, workspace)
    rc = _abi.lib().ssm_state_update_strided(
        _ptr(state), _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z),
        _ptr(dt_bias), int(bool(delta_softplus)), _ptr(out), _ptr(ws),
        0 if ws is None else ws.numel(), batch, dim, N, G, code, _flags(scalar_a, False, zoh),
        ctypes.byref(st), _stream(dev))
    _abi.check(rc, "ssm_state_update_strided")
    return out


# ------------------------------------------------------------------ sequence split
def ssm_scan_fwd_summary(u, delta, A, B, C, dt_bias=None, delta_softplus=True, scalar_a=False,
                         zoh=False, workspace=None):
    """The affine map of one sequence segment: returns (hend [batch, dim, N], dsum [batch, dim]),
    the state after the segment from a zero state and ΣΔ over it, so that the segment maps an
    entering state h to exp(A dsum) h + hend.  With scalar_a, N may be 32 to 128 as in the
    scalar-decay scan (bf16: 32, 64 or 128; f32: any multiple of 16)."""
    dev = _on_gpu(u, "u")
    batch, dim, L = u.shape
    io = u.dtype
    code = _io_code(io)
    G, N, bc_shape = _bc_layout(B, batch, L)
    _need(u, "u", (batch, dim, L), io, dev)
    _need(delta, "delta", (batch, dim, L), io, dev)
    _need(A, "A", (dim,) if scalar_a else (dim, N), torch.float32, dev)
    _need(B, "B", bc_shape, io, dev)
    _need(C, "C", bc_shape, io, dev)
    _opt(dt_bias, "dt_bias", (dim,), torch.float32, dev)
    hend = torch.empty((batch, dim, N), dtype=torch.float32, device=dev)
    dsum = torch.empty((batch, dim), dtype=torch.float32, device=dev)
    flags = _flags(scalar_a, False, zoh)
    nws = int(_abi.lib().ssm_scan_fwd_summary_workspace_size(batch, dim, L, N, G, code, flags))
    ws = _workspace(nws, dev, workspace)
    rc = _abi.lib().ssm_scan_fwd_summary(
        _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(dt_bias), int(bool(delta_softplus)),
        _ptr(hend), _ptr(dsum), _ptr(ws), 0 if ws is None else ws.numel(), batch, dim, L, N, G,
        code, flags, _stream(dev))
    _abi.check(rc, "ssm_scan_fwd_summary")
    return hend, dsum


def ssm_scan_chain(hend, dsum, A, h0=None, scalar_a=False):
    """The state entering each of S consecutive segments given their maps (hend [S, batch, dim,
    N], dsum [S, batch, dim], as from :func:`ssm_scan_fwd_summary`) and the state h0 entering the
    first: returns hin [S, batch, dim, N]."""
    dev = _on_gpu(hend, "hend")
    S, batch, dim, N = hend.shape
    _need(hend, "hend", (S, batch, dim, N), torch.float32, dev)
    _need(dsum, "dsum", (S, batch, dim), torch.float32, dev)
    _need(A, "A", (dim,) if scalar_a else (dim, N), torch.float32, dev)
    _opt(h0, "h0", (batch, dim, N), torch.float32, dev)
    hin = torch.empty_like(hend)
    rc = _abi.lib().ssm_scan_chain(_ptr(hend), _ptr(dsum), _ptr(A), _ptr(h0), _ptr(hin), S, batch,
                                   dim, N, _flags(scalar_a, False, False), _stream(dev))
    _abi.check(rc, "ssm_scan_chain")
    return hin
