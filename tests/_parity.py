"""Parity helpers: tolerances and comparison of CUDA results with the fp64 oracle.

Tolerances (stated for the scan on the pages' workloads):
  * f32 io:  relative L2 error <= 1e-5.
  * bf16 io (f32 state): relative L2 error <= 1e-2 and max |err| <= 5e-2 * max(1, |ref|).
    The absolute bound is applied relative to the value once |ref| > 1: a bf16 result carries
    a rounding error of up to 2^-9 |ref| from the final store alone, so a fixed 5e-2 absolute
    bound cannot hold for outputs above ~12 even when every bit before the store is exact.
Gradients are compared the same way.
"""
import numpy as np
import torch

TOL = {
    torch.float32: dict(rel_l2=1e-5, max_abs=None),
    torch.bfloat16: dict(rel_l2=1e-2, max_abs=5e-2),
}


def f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def rel_l2(got, ref):
    num = np.linalg.norm((got - ref).ravel())
    den = np.linalg.norm(ref.ravel())
    return num / den if den > 0 else num


def assert_close(got, ref, io_dtype, name="", scale=1.0):
    """got: CUDA tensor or ndarray; ref: float64 ndarray.  scale loosens the bound for sums of
    many rounded terms (used for nothing by default)."""
    g = f64(got) if isinstance(got, torch.Tensor) else np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert g.shape == ref.shape, (name, g.shape, ref.shape)
    assert np.all(np.isfinite(g)), f"{name}: non-finite values"
    tol = TOL[io_dtype]
    e = rel_l2(g, ref)
    assert e <= tol["rel_l2"] * scale, f"{name}: rel-L2 {e:.3e} > {tol['rel_l2'] * scale:.1e}"
    if tol["max_abs"] is not None:
        m = np.max(np.abs(g - ref) / np.maximum(1.0, np.abs(ref)))
        assert m <= tol["max_abs"] * scale, f"{name}: max normalised error {m:.3e}"
    return e


def bf16_ulp(x):
    """Spacing of bfloat16 numbers at |x| (8 significant bits; normal range)."""
    a = np.maximum(np.abs(np.asarray(x, dtype=np.float64)), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(a)) - 7)


def assert_bf16_elementwise(got, ref, name="", ulps=2.0, floor_rel=1e-3):
    """Element-wise check of a bf16 output against the unrounded fp64 oracle value:
    |got - ref| <= ulps * ulp_bf16(ref) + floor_rel * rms(ref).

    A correct kernel computes in f32 and rounds once at the store, so it lands within one bf16
    ulp of the exact value unless f32 error flips the rounding; two ulps leave room for that.
    The floor (a thousandth of the output's rms, a quarter of a bf16 ulp at that scale) covers
    outputs that are small only because their terms cancel, where f32 error is absolute."""
    g = f64(got) if isinstance(got, torch.Tensor) else np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert g.shape == ref.shape, (name, g.shape, ref.shape)
    rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    bound = ulps * bf16_ulp(ref) + floor_rel * rms
    err = np.abs(g - ref)
    bad = err > bound
    if bad.any():
        i = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(f"{name}: {int(bad.sum())} elements beyond {ulps} bf16 ulp "
                             f"(worst at {i}: got {g[i]!r}, ref {ref[i]!r})")
