"""fp64 CPU oracle for the selective state-space (S6) scan -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may import
this package.  It shares no code with the CUDA library (``selective_state_space_23_b200``)
and neither imports the other; both sides receive the same seeded inputs.

The arithmetic lives in ``ssm_oracle.c`` (plain double-precision loops, cited there):
  * ``scan_fwd``      -- h_t = exp(Δ_t A) h_{t-1} + Δ_t B_t x_t,  y_t = C_t.h_t + D x_t,
                         out_t = y_t * silu(z_t); Δ_t = softplus(delta_t + dt_bias).
                         ("Mamba: Linear-Time Sequence Modeling with Selective State Spaces",
                         summary page, sections "Yöntem" and "Seçim Mekanizması (S6)").
  * ``scan_bwd``      -- gradients of ``scan_fwd`` by the chain rule (reverse-time adjoint),
                         for the Euler input term and for the ZOH one (``zoh=True``).
                         The pages give no gradient formula: this function is pinned only by
                         finite differences of ``scan_fwd`` (parity of the gradient formulas
                         themselves is otherwise unpinned by the pages).
  * ``state_update``  -- one recurrent (decode) step of the same recurrence, in place.
  * grouped B/C      -- B, C of shape [batch, G, N, L]: each group of dim/G channels is an
                         independent scan with its own B, C, run as exactly that.
  * ``reverse=True``  -- the scan backwards in time (t = L-1 .. 0), the anti-causal half of a
                         bidirectional layer ("2024 Reading List: Neural Network", Hydra notes):
                         by definition the forward scan of the time-reversed sequences, so it is
                         written as exactly that (reverse the time axis, scan, reverse back).

All arrays are numpy float64, C-contiguous; layouts as in ``ssm_oracle.c``.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_LIB = None

_f64p = ctypes.POINTER(ctypes.c_double)
_i64p = ctypes.POINTER(ctypes.c_int64)


def _lib():
    global _LIB
    if _LIB is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        lib.oracle_scan_fwd.restype = ctypes.c_int
        lib.oracle_scan_bwd.restype = ctypes.c_int
        lib.oracle_state_update.restype = ctypes.c_int
        lib.oracle_max_threads.restype = ctypes.c_int
        _LIB = lib
    return _LIB


def max_threads() -> int:
    """Threads the oracle uses when ``nthreads`` is not given (OpenMP default)."""
    return int(_lib().oracle_max_threads())


def _arr(x, shape=None):
    if x is None:
        return None
    a = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    if shape is not None and a.shape != tuple(shape):
        raise ValueError(f"expected shape {tuple(shape)}, got {a.shape}")
    return a


def _p(a):
    return None if a is None else a.ctypes.data_as(_f64p)


def _chans(channels):
    if channels is None:
        return None, None, 0
    c = np.ascontiguousarray(np.asarray(channels, dtype=np.int64).reshape(-1))
    return c, c.ctypes.data_as(_i64p), int(c.size)


def _flip(x):
    """Time axis (the last one) reversed, or None."""
    return None if x is None else np.ascontiguousarray(np.asarray(x, dtype=np.float64)[..., ::-1])


_PER_CHANNEL = {"u", "delta", "z", "dout"}  # [batch, dim, L]
_PER_D = {"A", "D", "dt_bias"}             # [dim, ...]
_PER_BD = {"h0", "dhL"}                    # [batch, dim, N]


def _grouped(fn, u, delta, A, B, C, *rest, **kw):
    """Grouped B/C ([batch, G, N, L]): channel d uses group d // (dim // G).  By definition each
    group is an independent scan over its channels with its own B, C; run it per group and
    assemble the results (dB, dC per group; every other output per channel)."""
    u = np.asarray(u, dtype=np.float64)
    batch, dim, L = u.shape
    G = np.shape(B)[1]
    if dim % G:
        raise ValueError(f"dim {dim} is not a multiple of {G} groups")
    per = dim // G
    args = {"u": u, "delta": delta, "A": A}
    if rest:
        args["dout"] = rest[0]
    parts = []
    for g in range(G):
        sl = slice(g * per, (g + 1) * per)
        pick = lambda k, v: (None if v is None else
                             np.asarray(v)[:, sl] if k in _PER_CHANNEL or k in _PER_BD else
                             np.asarray(v)[sl] if k in _PER_D else v)
        pos = [pick(k, args[k]) for k in ("u", "delta", "A")]
        pos += [np.asarray(B)[:, g], np.asarray(C)[:, g]]
        if "dout" in args:
            pos.append(pick("dout", args["dout"]))
        parts.append(fn(*pos, **{k: pick(k, v) for k, v in kw.items()}))
    res = {}
    for k in parts[0]:
        if parts[0][k] is None:
            res[k] = None
        elif k in ("dB", "dC"):
            res[k] = np.stack([p[k] for p in parts], 1)
        elif k in ("dA", "dD", "ddt_bias"):
            res[k] = np.concatenate([p[k] for p in parts], 0)
        else:
            res[k] = np.concatenate([p[k] for p in parts], 1)
    return res


def scan_fwd(u, delta, A, B, C, D=None, z=None, dt_bias=None, delta_softplus=True,
             h0=None, zoh=False, channels=None, nthreads=0, out=None, ypre=False, reverse=False):
    """Forward selective scan in fp64.

    u, delta, z: [batch, dim, L]; B, C: [batch, N, L]; A: [dim, N]; D, dt_bias: [dim];
    h0: [batch, dim, N].  ``channels``: optional flat indices b*dim+d to compute (others
    left as in ``out``, default zeros).  ``reverse``: scan from t = L-1 down to 0 (h0 enters
    at t = L-1, hL is the state after t = 0).  Returns dict(out, hL[, ypre]).
    """
    if np.ndim(B) == 4:
        return _grouped(scan_fwd, u, delta, A, B, C, D=D, z=z, dt_bias=dt_bias,
                        delta_softplus=delta_softplus, h0=h0, zoh=zoh, nthreads=nthreads,
                        ypre=ypre, reverse=reverse)
    if reverse:
        res = scan_fwd(_flip(u), _flip(delta), A, _flip(B), _flip(C), D=D, z=_flip(z),
                       dt_bias=dt_bias, delta_softplus=delta_softplus, h0=h0, zoh=zoh,
                       channels=channels, nthreads=nthreads,
                       out=None if out is None else _flip(out), ypre=ypre)
        res["out"] = _flip(res["out"])
        if out is not None:
            out[...] = res["out"]
            res["out"] = out
        if ypre:
            res["ypre"] = _flip(res["ypre"])
        return res
    u = _arr(u)
    batch, dim, L = u.shape
    A = _arr(A)
    N = A.shape[1]
    delta = _arr(delta, (batch, dim, L))
    A = _arr(A, (dim, N))
    B = _arr(B, (batch, N, L))
    C = _arr(C, (batch, N, L))
    D = _arr(D, (dim,))
    z = _arr(z, (batch, dim, L))
    dt_bias = _arr(dt_bias, (dim,))
    h0 = _arr(h0, (batch, dim, N))
    o = np.zeros((batch, dim, L)) if out is None else out
    yp = np.zeros((batch, dim, L)) if ypre else None
    hL = np.zeros((batch, dim, N))
    keep, cp, nc = _chans(channels)
    rc = _lib().oracle_scan_fwd(
        batch, dim, L, N, _p(u), _p(delta), _p(A), _p(B), _p(C), _p(D), _p(z), _p(dt_bias),
        int(bool(delta_softplus)), int(bool(zoh)), _p(h0), _p(o), _p(yp), _p(hL), cp,
        ctypes.c_int64(nc), int(nthreads))
    if rc != 0:
        raise RuntimeError(f"oracle_scan_fwd failed ({rc})")
    del keep
    res = {"out": o, "hL": hL}
    if ypre:
        res["ypre"] = yp
    return res


def scan_bwd(u, delta, A, B, C, dout, D=None, z=None, dt_bias=None, delta_softplus=True,
             h0=None, dhL=None, channels=None, nthreads=0, reverse=False, zoh=False):
    """Gradients of :func:`scan_fwd` (Euler input term, or ZOH with ``zoh``) w.r.t. every
    input, in fp64.

    Returns dict(du, ddelta, dA, dB, dC, dD, dz, ddt_bias, dh0).  With ``channels`` the
    summed gradients (dA, dB, dC, dD, ddt_bias) hold only those channels' contributions.
    ``reverse``: gradients of the reverse scan (time-indexed gradients reversed back).
    """
    if np.ndim(B) == 4:
        return _grouped(scan_bwd, u, delta, A, B, C, dout, D=D, z=z, dt_bias=dt_bias,
                        delta_softplus=delta_softplus, h0=h0, dhL=dhL, nthreads=nthreads,
                        reverse=reverse, zoh=zoh)
    if reverse:
        g = scan_bwd(_flip(u), _flip(delta), A, _flip(B), _flip(C), _flip(dout), D=D, z=_flip(z),
                     dt_bias=dt_bias, delta_softplus=delta_softplus, h0=h0, dhL=dhL,
                     channels=channels, nthreads=nthreads, zoh=zoh)
        for k in ("du", "ddelta", "dz", "dB", "dC"):
            g[k] = _flip(g[k])
        return g
    u = _arr(u)
    batch, dim, L = u.shape
    A = _arr(A)
    N = A.shape[1]
    delta = _arr(delta, (batch, dim, L))
    B = _arr(B, (batch, N, L))
    C = _arr(C, (batch, N, L))
    dout = _arr(dout, (batch, dim, L))
    D = _arr(D, (dim,))
    z = _arr(z, (batch, dim, L))
    dt_bias = _arr(dt_bias, (dim,))
    h0 = _arr(h0, (batch, dim, N))
    dhL = _arr(dhL, (batch, dim, N))
    g = {
        "du": np.zeros((batch, dim, L)), "ddelta": np.zeros((batch, dim, L)),
        "dz": np.zeros((batch, dim, L)), "dA": np.zeros((dim, N)),
        "dB": np.zeros((batch, N, L)), "dC": np.zeros((batch, N, L)),
        "dD": np.zeros((dim,)), "ddt_bias": np.zeros((dim,)),
        "dh0": np.zeros((batch, dim, N)),
    }
    keep, cp, nc = _chans(channels)
    rc = _lib().oracle_scan_bwd(
        batch, dim, L, N, _p(u), _p(delta), _p(A), _p(B), _p(C), _p(D), _p(z), _p(dt_bias),
        int(bool(delta_softplus)), int(bool(zoh)), _p(h0), _p(dout), _p(dhL),
        _p(g["du"]), _p(g["ddelta"]), _p(g["dA"]), _p(g["dB"]), _p(g["dC"]), _p(g["dD"]),
        _p(g["dz"]), _p(g["ddt_bias"]), _p(g["dh0"]), cp, ctypes.c_int64(nc), int(nthreads))
    if rc != 0:
        raise RuntimeError(f"oracle_scan_bwd failed ({rc})")
    del keep
    if z is None:
        g["dz"] = None
    return g


def state_update(state, x, dt, A, B, C, D=None, z=None, dt_bias=None, delta_softplus=True,
                 nthreads=0, zoh=False):
    """One decode step.  ``state`` [batch, dim, N] float64 is updated IN PLACE (it must be a
    C-contiguous float64 array).  x, dt, z: [batch, dim]; B, C: [batch, N], or [batch, G, N]
    (grouped: each group of dim/G channels is an independent step with its own B, C).
    ``zoh``: zero-order-hold input coefficient.  Returns out."""
    if not (isinstance(state, np.ndarray) and state.dtype == np.float64
            and state.flags["C_CONTIGUOUS"]):
        raise TypeError("state must be a C-contiguous float64 numpy array (updated in place)")
    batch, dim, N = state.shape
    if np.ndim(B) == 3:
        G = np.shape(B)[1]
        per = dim // G
        out = np.zeros((batch, dim))
        for g in range(G):
            sl = slice(g * per, (g + 1) * per)
            st = np.ascontiguousarray(state[:, sl])
            cut = lambda v, ax: None if v is None else (np.asarray(v)[:, sl] if ax else np.asarray(v)[sl])
            out[:, sl] = state_update(st, cut(x, 1), cut(dt, 1), np.asarray(A)[sl],
                                      np.asarray(B)[:, g], np.asarray(C)[:, g], D=cut(D, 0),
                                      z=cut(z, 1), dt_bias=cut(dt_bias, 0),
                                      delta_softplus=delta_softplus, nthreads=nthreads, zoh=zoh)
            state[:, sl] = st
        return out
    x = _arr(x, (batch, dim))
    dt = _arr(dt, (batch, dim))
    A = _arr(A, (dim, N))
    B = _arr(B, (batch, N))
    C = _arr(C, (batch, N))
    D = _arr(D, (dim,))
    z = _arr(z, (batch, dim))
    dt_bias = _arr(dt_bias, (dim,))
    out = np.zeros((batch, dim))
    rc = _lib().oracle_state_update(
        batch, dim, N, _p(state), _p(x), _p(dt), _p(A), _p(B), _p(C), _p(D), _p(z),
        _p(dt_bias), int(bool(delta_softplus)), int(bool(zoh)), _p(out), int(nthreads))
    if rc != 0:
        raise RuntimeError(f"oracle_state_update failed ({rc})")
    return out


__all__ = ["scan_fwd", "scan_bwd", "state_update", "max_threads"]
