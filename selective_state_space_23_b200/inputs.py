"""Seeded synthetic inputs for the selective scan (shared by the CUDA path's tests/benchmark and
the CPU oracle's tests).  This module holds no arithmetic of the scan itself: it only draws
random tensors with the workloads' shapes and distributions.

Recipe (every workload):
  u, z, B, C, dout ~ N(0, 1);  delta (raw step input) ~ N(0, 0.5^2);
  dt ~ log-uniform on [dt_min, dt_max] per channel d, dt_bias = inv_softplus(dt) so that a zero
  raw delta gives a step of exactly dt (inv_softplus(y) = y + log(-expm1(-y)));
  A[d, n] = -(n + 1) (S4D-real initialisation);  D ~ N(0, 1);
  scalar decay (one rate per channel): A[d] = -U(1, 16), the range of Mamba-2's initial rates.
io tensors are drawn in float32 and rounded once to the io dtype (bf16: round-to-nearest-even);
the oracle reads the rounded values.  numpy's PCG64 generator, seeded per tensor name, so each
tensor is reproducible on its own and on any machine.
"""
from dataclasses import dataclass, field, replace
import zlib

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    dim: int
    seqlen: int
    dstate: int = 16
    io_dtype: torch.dtype = torch.bfloat16
    dt_min: float = 1e-3
    dt_max: float = 1e-1
    steps: int = 1            # decode: consecutive one-token steps
    extra: dict = field(default_factory=dict)

    @property
    def tokens(self) -> int:
        return self.batch * self.seqlen


# The five workloads (shapes of Mamba-370m / Mamba-2.8B layers, a 2^20-token sequence, and a
# batch-256 decode step).
WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", 1, 64, 256, 16, torch.float32),
    "mamba370m_fwd": Workload("mamba370m_fwd", 8, 2048, 2048, 16, torch.bfloat16),
    "mamba2p8b_train": Workload("mamba2p8b_train", 4, 5120, 2048, 16, torch.bfloat16),
    "long_seq_1m": Workload("long_seq_1m", 1, 256, 1 << 20, 16, torch.bfloat16, 1e-4, 1e-2),
    "decode_b256": Workload("decode_b256", 256, 5120, 1, 16, torch.bfloat16, steps=1024),
}


def workload(name: str, **overrides) -> Workload:
    return replace(WORKLOADS[name], **overrides)


def _rng(seed: int, tag: str) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64([seed, zlib.crc32(tag.encode())]))


def _normal(seed, tag, shape, std=1.0):
    x = _rng(seed, tag).standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return x


def inv_softplus(y: np.ndarray) -> np.ndarray:
    """Input-recipe helper: the value whose softplus is y (y > 0)."""
    y = np.asarray(y, dtype=np.float64)
    return y + np.log(-np.expm1(-y))


def _io(x: np.ndarray, dtype: torch.dtype) -> torch.Tensor:
    return torch.from_numpy(x).to(dtype)


def make_inputs(w: Workload, seed: int = 0, with_dout: bool = False, with_h0: bool = False,
                gate: bool = True, step: int = None, scalar_a: bool = False) -> dict:
    """CPU tensors for one call.  Scan layout: u, delta, z, dout [batch, dim, L];
    B, C [batch, N, L].  Decode (step is not None): x, dt, z [batch, dim]; B, C [batch, N],
    drawn independently for each step index.  scalar_a: A is [dim] (one decay rate per channel)."""
    b, d, L, N = w.batch, w.dim, w.seqlen, w.dstate
    tag = "" if step is None else f"/step{step}"
    shape_x = (b, d, L) if step is None else (b, d)
    shape_bc = (b, N, L) if step is None else (b, N)
    out = {}
    out["u" if step is None else "x"] = _io(_normal(seed, "u" + tag, shape_x), w.io_dtype)
    out["delta" if step is None else "dt"] = _io(_normal(seed, "delta" + tag, shape_x, 0.5), w.io_dtype)
    if gate:
        out["z"] = _io(_normal(seed, "z" + tag, shape_x), w.io_dtype)
    out["B"] = _io(_normal(seed, "B" + tag, shape_bc), w.io_dtype)
    out["C"] = _io(_normal(seed, "C" + tag, shape_bc), w.io_dtype)
    # per-channel parameters (shared by all steps)
    lo, hi = np.log(w.dt_min), np.log(w.dt_max)
    dt = np.exp(_rng(seed, "dt").uniform(lo, hi, size=(d,)))
    out["dt_bias"] = torch.from_numpy(inv_softplus(dt).astype(np.float32))
    if scalar_a:
        out["A"] = torch.from_numpy(-_rng(seed, "A").uniform(1.0, 16.0, size=(d,)).astype(np.float32))
    else:
        out["A"] = torch.from_numpy(-np.tile(np.arange(1, N + 1, dtype=np.float32), (d, 1)))
    out["D"] = torch.from_numpy(_normal(seed, "D", (d,)))
    if with_h0:
        out["h0"] = torch.from_numpy(_normal(seed, "h0", (b, d, N), 0.5))
    if with_dout and step is None:
        out["dout"] = _io(_normal(seed, "dout", shape_x), w.io_dtype)
    return out


def to_f64(t: torch.Tensor) -> np.ndarray:
    """Exact float64 copy of a (CPU or GPU) tensor for the oracle."""
    return t.detach().to("cpu", torch.float64).numpy()
