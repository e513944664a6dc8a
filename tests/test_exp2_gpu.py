"""The exponentials inside the forward kernel against their error bounds.

With one nonzero step, B = 0, h0 = 1, no softplus and no bias, the final state is exactly the
kernel's discretised decay: hL[b, d, n] = exp(Δ_d A_dn) as computed on the GPU, returned in f32.
The exponential split routes some states to the MUFU unit (ex2.approx) and the others to the
FMA-pipe polynomial (Cody-Waite reduction + Remez cubic); each test names its split.

Bounds checked (relative to the exact exp in float64 of the same Δ and A):
  * polynomial: |err| <= 1.6e-5 |1 - a| + 2e-7 |x| a + 2e-7 a      (x = Δ A log2 e)
    i.e. the decay rate 1 - a keeps ~1.5e-5 relative accuracy even as a -> 1, plus the f32
    rounding of x and of the result;
  * MUFU: |err| <= 1e-6 a + 2e-7 |x| a.
A warp whose |x| exceeds 126 must take the all-MUFU path and still be correct.
"""
import numpy as np
import pytest
import torch

import selective_state_space_23_b200 as ssm

pytestmark = pytest.mark.gpu
DEV = "cuda"
LOG2E = 1.4426950408889634


def run(delta, A, L=1, step=0):
    """One step (index `step`) of size delta[d] from h0 = 1; the other steps have Δ = 0 (a = 1
    exactly in both exponentials).  L = 1 or 2: rows are not 16-byte pieces and the
    two-lanes-per-channel kernel runs; L = 8: the one-lane-per-channel kernel runs."""
    dim, N = A.shape
    u = torch.zeros((1, dim, L), dtype=torch.bfloat16, device=DEV)
    d = torch.zeros((1, dim, L), dtype=torch.bfloat16, device=DEV)
    d[0, :, step] = delta.to(torch.bfloat16).to(DEV)
    Bz = torch.zeros((1, N, L), dtype=torch.bfloat16, device=DEV)
    h0 = torch.ones((1, dim, N), dtype=torch.float32, device=DEV)
    _, hL = ssm.ssm_scan_fwd(u, d, A.to(DEV), Bz, Bz, delta_softplus=False, h0=h0,
                             return_final_state=True)
    torch.cuda.synchronize()
    dl = d[0, :, step].double().cpu().reshape(dim, 1).numpy()
    return hL[0].double().cpu().numpy(), dl * A.double().numpy()


def test_fma_polynomial_and_mufu_within_bounds(monkeypatch):
    """The two-lanes-per-channel kernel with its default split: at an odd step, state pair 3 of
    each lane (states 6, 7, 14, 15) takes the polynomial, the others MUFU."""
    monkeypatch.setenv("SSM_FWD_KERNEL", "pair")
    monkeypatch.setenv("SSM_FWD_KMUFU", "14")
    r = np.random.default_rng(0)
    dim, N = 4096, 16
    delta = torch.from_numpy(np.exp(r.uniform(np.log(1e-4), np.log(2.0), dim)).astype(np.float32))
    # A spans 6 decades; |Δ A log2 e| stays below 126 in every warp except the last one
    A = -np.exp(r.uniform(np.log(1e-3), np.log(40.0), (dim, N))).astype(np.float32)
    A[-16:] *= 200.0  # last warp (16 channels): exponents far beyond the polynomial's range
    a_gpu, x = run(delta, torch.from_numpy(A), L=2, step=1)
    exact = np.exp(x)
    err = np.abs(a_gpu - exact)
    xl = np.abs(x * LOG2E)
    poly = np.zeros(N, bool)
    poly[[6, 7, 14, 15]] = True
    body = slice(0, dim - 16)
    bound_poly = 1.6e-5 * np.abs(1 - exact) + 2e-7 * xl * exact + 2e-7 * exact
    bound_mufu = 1e-6 * exact + 2e-7 * xl * exact + 1e-38
    assert np.all(err[body][:, poly] <= bound_poly[body][:, poly]), float(
        np.max(err[body][:, poly] / bound_poly[body][:, poly]))
    assert np.all(err[body][:, ~poly] <= bound_mufu[body][:, ~poly]), float(
        np.max(err[body][:, ~poly] / bound_mufu[body][:, ~poly]))
    # the out-of-range warp ran every exponential on the MUFU unit
    tail = slice(dim - 16, dim)
    assert np.all(err[tail] <= bound_mufu[tail] + 1e-30)
    # long memories: the decay rate 1 - a is accurate even when a is within 1e-4 of 1
    small = ((xl > 1e-4) & (xl < 1e-3))[body] & poly[None, :]
    assert small.sum() > 100
    rate_err = np.abs((1 - a_gpu[body]) - (1 - exact[body]))[small] / np.abs(1 - exact[body])[small]
    assert rate_err.max() < 2e-3  # limited by the f32 spacing of a near 1, not by the polynomial


@pytest.mark.parametrize("L,kernel", [(1, "pair"), (8, "pair"), (8, "lane")])
def test_exact_one_when_step_is_zero(monkeypatch, L, kernel):
    monkeypatch.setenv("SSM_FWD_KERNEL", kernel)
    dim, N = 64, 16
    A = -torch.rand((dim, N)) * 10
    a_gpu, _ = run(torch.zeros(dim), A, L=L)
    assert np.all(a_gpu == 1.0)


def test_lane_kernel_exponentials_within_bounds(monkeypatch):
    """The one-lane-per-channel kernel with SSM_FWD_KMUFU=8: at an even step, state pairs 0..3
    (states 0..7) take MUFU and states 8..15 the polynomial.  A warp (32 channels) any of whose
    lanes has a step beyond the polynomial's range runs the block with every exponential on
    MUFU."""
    monkeypatch.setenv("SSM_FWD_KERNEL", "lane")
    monkeypatch.setenv("SSM_FWD_KMUFU", "8")
    r = np.random.default_rng(1)
    dim, N = 4096, 16
    delta = torch.from_numpy(np.exp(r.uniform(np.log(1e-4), np.log(2.0), dim)).astype(np.float32))
    A = -np.exp(r.uniform(np.log(1e-3), np.log(40.0), (dim, N))).astype(np.float32)
    A[-32:] *= 200.0  # the last warp: exponents far beyond the polynomial's range
    a_gpu, x = run(delta, torch.from_numpy(A), L=8)
    exact = np.exp(x)
    err = np.abs(a_gpu - exact)
    xl = np.abs(x * LOG2E)
    poly = np.zeros(N, bool)
    poly[8:] = True
    body = slice(0, dim - 32)
    bound_poly = 1.6e-5 * np.abs(1 - exact) + 2e-7 * xl * exact + 2e-7 * exact
    bound_mufu = 1e-6 * exact + 2e-7 * xl * exact + 1e-38
    assert np.all(err[body][:, poly] <= bound_poly[body][:, poly]), float(
        np.max(err[body][:, poly] / bound_poly[body][:, poly]))
    assert np.all(err[body][:, ~poly] <= bound_mufu[body][:, ~poly]), float(
        np.max(err[body][:, ~poly] / bound_mufu[body][:, ~poly]))
    tail = slice(dim - 32, dim)
    assert np.all(err[tail] <= bound_mufu[tail] + 1e-30)
    small = ((xl > 1e-4) & (xl < 1e-3))[body] & poly[None, :]
    assert small.sum() > 100
    rate_err = np.abs((1 - a_gpu[body]) - (1 - exact[body]))[small] / np.abs(1 - exact[body])[small]
    assert rate_err.max() < 2e-3
