"""Pins of the fp64 CPU oracle against facts that do not come from the oracle itself.

Every test builds its expected value independently (a different formula or library routine):
  * brute-force quadratic ("semiseparable matrix") form of the scan -- the zenn.dev reading-list
    page, Hydra notes: sequence mixing of an SSM is a structured, data-dependent matrix;
  * closed forms: L = 1, the geometric series for constant inputs, the LTI causal convolution
    (mamba-minimal news page: a time-invariant SSM can run as one global convolution);
  * the gating special case of the "Seçim Mekanizması (S6)" section (N=1, A=-1, B=1), and the
    ZOH input term against the hold integral of the "Yöntem" discretisation (Gauss-Legendre);
  * the Δ limits of the "Sorular" section (small Δ keeps the state, large Δ resets it);
  * chunked-vs-sequential state passing, superposition, decode-vs-scan;
  * the scalar decay (one A per channel, the Mamba-2 restriction in the reading-list notes) as
    a masked Gram-matrix product, and its rate gradient by central differences;
  * grouped B/C (one B_t, C_t per group of channels) against the quadratic form of each group,
    and its gradients by central differences;
  * the reverse scan (Hydra notes: the anti-causal half of a bidirectional layer) against the
    anti-causal quadratic form, a two-step closed form of its final state, and central
    differences of its gradients;
  * central finite differences of the forward pass for every gradient.
"""
import numpy as np
import pytest
from scipy.special import expit

import oracle

RNG = np.random.default_rng(1234)


def rand_case(batch=2, dim=3, L=7, N=3, gate=True, h0=True, seed=0):
    r = np.random.default_rng(seed)
    c = dict(
        u=r.standard_normal((batch, dim, L)),
        delta=0.5 * r.standard_normal((batch, dim, L)),
        A=-np.exp(r.standard_normal((dim, N))),
        B=r.standard_normal((batch, N, L)),
        C=r.standard_normal((batch, N, L)),
        D=r.standard_normal(dim),
        z=r.standard_normal((batch, dim, L)) if gate else None,
        dt_bias=r.uniform(-3.0, -1.0, dim),
        h0=r.standard_normal((batch, dim, N)) if h0 else None,
    )
    return c


def softplus_ref(v):
    return np.logaddexp(0.0, v)


def quadratic_form(c, softplus=True):
    """y_t = sum_{s<=t} C_t . (prod_{r=s+1..t} exp(Δ_r A)) Δ_s B_s u_s
             + C_t . (prod_{r=0..t} exp(Δ_r A)) h0 + D u_t,  then * silu(z_t).
    Products of exponentials are evaluated as exp(A * sum of Δ) (not as a running product)."""
    u, A, B, C = c["u"], c["A"], c["B"], c["C"]
    batch, dim, L = u.shape
    N = A.shape[1]
    v = c["delta"] + c["dt_bias"][None, :, None]
    dt = softplus_ref(v) if softplus else v
    out = np.zeros_like(u)
    for b in range(batch):
        for d in range(dim):
            cs = np.concatenate([[0.0], np.cumsum(dt[b, d])])  # cs[k] = sum_{r<k} Δ_r
            for t in range(L):
                y = 0.0
                for s in range(t + 1):
                    decay = np.exp(A[d] * (cs[t + 1] - cs[s + 1]))  # prod over r = s+1..t
                    y += np.sum(C[b, :, t] * decay * dt[b, d, s] * B[b, :, s]) * u[b, d, s]
                if c["h0"] is not None:
                    y += np.sum(C[b, :, t] * np.exp(A[d] * cs[t + 1]) * c["h0"][b, d])
                y += c["D"][d] * u[b, d, t]
                if c["z"] is not None:
                    zz = c["z"][b, d, t]
                    y *= zz * expit(zz)
                out[b, d, t] = y
    return out


def run(c, **kw):
    return oracle.scan_fwd(c["u"], c["delta"], c["A"], c["B"], c["C"], D=c["D"], z=c["z"],
                           dt_bias=c["dt_bias"], h0=c["h0"], **kw)


@pytest.mark.parametrize("gate,h0,softplus", [(True, True, True), (False, False, True),
                                               (True, False, False)])
def test_quadratic_form(gate, h0, softplus):
    c = rand_case(batch=2, dim=3, L=8, N=3, gate=gate, h0=h0, seed=7)
    if not softplus:
        c["delta"] = np.abs(c["delta"]) + 0.05
        c["dt_bias"] = np.zeros(3)
    got = run(c, delta_softplus=softplus)["out"]
    np.testing.assert_allclose(got, quadratic_form(c, softplus), rtol=1e-11, atol=1e-12)


def test_single_step_closed_form():
    c = rand_case(batch=2, dim=4, L=1, N=5, seed=3)
    dt = softplus_ref(c["delta"][..., 0] + c["dt_bias"])            # [b, d]
    a = np.exp(dt[..., None] * c["A"][None])                         # [b, d, n]
    h = a * c["h0"] + dt[..., None] * c["B"][:, None, :, 0] * c["u"][..., 0:1]
    y = np.sum(c["C"][:, None, :, 0] * h, -1) + c["D"] * c["u"][..., 0]
    z = c["z"][..., 0]
    res = run(c)
    np.testing.assert_allclose(res["out"][..., 0], y * z * expit(z), rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(res["hL"], h, rtol=1e-13, atol=1e-14)


def test_geometric_series():
    batch, dim, L, N = 1, 2, 40, 2
    c = rand_case(batch, dim, L, N, gate=False, seed=5)
    c["delta"][:] = c["delta"][..., :1]          # constant Δ per channel
    c["u"][:] = c["u"][..., :1]                  # constant input
    c["B"][:] = c["B"][..., :1]
    c["C"][:] = c["C"][..., :1]
    res = run(c)
    dt = softplus_ref(c["delta"][..., 0] + c["dt_bias"])           # [b, d]
    a = np.exp(dt[..., None] * c["A"][None])                        # [b, d, n]
    bterm = dt[..., None] * c["B"][:, None, :, 0] * c["u"][..., 0:1]
    t = np.arange(L)
    p = a[..., None] ** (t + 1)                                     # [b, d, n, L]
    h = p * c["h0"][..., None] + bterm[..., None] * (1 - p) / (1 - a[..., None])
    y = np.einsum("bn,bdnt->bdt", c["C"][..., 0], h) + c["D"][None, :, None] * c["u"]
    np.testing.assert_allclose(res["out"], y, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(res["hL"], h[..., -1], rtol=1e-11, atol=1e-12)


def test_lti_is_causal_convolution():
    batch, dim, L, N = 1, 2, 64, 4
    c = rand_case(batch, dim, L, N, gate=False, h0=False, seed=11)
    c["delta"][:] = c["delta"][..., :1]
    c["B"][:] = c["B"][..., :1]
    c["C"][:] = c["C"][..., :1]
    res = run(c)
    dt = softplus_ref(c["delta"][0, :, 0] + c["dt_bias"])            # [d]
    for d in range(dim):
        a = np.exp(dt[d] * c["A"][d])                                 # [n]
        k = np.arange(L)
        K = np.sum(c["C"][0, :, 0, None] * a[:, None] ** k[None] * dt[d] * c["B"][0, :, 0, None], 0)
        y = np.convolve(c["u"][0, d], K)[:L] + c["D"][d] * c["u"][0, d]
        np.testing.assert_allclose(res["out"][0, d], y, rtol=1e-10, atol=1e-12)


def test_gating_reduction():
    """N=1, A=-1, B=1, Δ = softplus(w): exp(ΔA) = 1 - sigmoid(w).  With the ZOH input term the
    scan is exactly the gated update h_t = (1-g_t) h_{t-1} + g_t x_t; with the first-order term
    it is h_t = (1-g_t) h_{t-1} + Δ_t x_t."""
    L = 50
    r = np.random.default_rng(2)
    w = r.standard_normal((1, 1, L)) * 2
    x = r.standard_normal((1, 1, L))
    ones = np.ones((1, 1, L))
    g = expit(w[0, 0])
    for zoh in (True, False):
        res = oracle.scan_fwd(x, w, -np.ones((1, 1)), ones, ones, delta_softplus=True, zoh=zoh)
        h, ref = 0.0, []
        for t in range(L):
            inp = g[t] * x[0, 0, t] if zoh else softplus_ref(w[0, 0, t]) * x[0, 0, t]
            h = (1 - g[t]) * h + inp
            ref.append(h)
        np.testing.assert_allclose(res["out"][0, 0], ref, rtol=1e-12, atol=1e-14)


def hold_integral(dt, a, nodes=24):
    """Zero-order hold of a diagonal entry: the integral of exp(a tau) over tau in [0, dt],
    by Gauss-Legendre quadrature (not the closed form (exp(a dt) - 1)/a)."""
    x, w = np.polynomial.legendre.leggauss(nodes)
    tau = 0.5 * dt * (x + 1.0)
    return 0.5 * dt * np.sum(w * np.exp(a * tau))


def test_zoh_quadratic_form_from_the_hold_integral():
    """With the ZOH input term ("Yöntem": B̄ = (ΔA)^{-1}(exp(ΔA) - I) ΔB, i.e. the input held
    constant over the step and integrated through exp(A tau)), every output is
    y_t = sum_{s<=t} C_t . (prod_{r=s+1..t} exp(Δ_r A)) (int_0^{Δ_s} exp(A tau) dtau) B_s u_s
          + C_t . (prod_{r<=t} exp(Δ_r A)) h0 + D u_t, gated.  A holds an exact zero and a
    tiny rate, where the hold integral is Δ."""
    c = rand_case(batch=2, dim=3, L=8, N=3, seed=21)
    c["A"][0, 0] = 0.0
    c["A"][1, 1] = -1e-9
    u, A, B, C = c["u"], c["A"], c["B"], c["C"]
    batch, dim, L = u.shape
    N = A.shape[1]
    dt = softplus_ref(c["delta"] + c["dt_bias"][None, :, None])
    want = np.zeros_like(u)
    for b in range(batch):
        for d in range(dim):
            cs = np.concatenate([[0.0], np.cumsum(dt[b, d])])
            hold = np.array([[hold_integral(dt[b, d, s], A[d, n]) for n in range(N)]
                             for s in range(L)])                      # [s, n]
            for t in range(L):
                y = 0.0
                for s in range(t + 1):
                    decay = np.exp(A[d] * (cs[t + 1] - cs[s + 1]))
                    y += np.sum(C[b, :, t] * decay * hold[s] * B[b, :, s]) * u[b, d, s]
                y += np.sum(C[b, :, t] * np.exp(A[d] * cs[t + 1]) * c["h0"][b, d])
                y += c["D"][d] * u[b, d, t]
                zz = c["z"][b, d, t]
                want[b, d, t] = y * zz * expit(zz)
    got = run(c, zoh=True)["out"]
    np.testing.assert_allclose(got, want, rtol=1e-11, atol=1e-12)
    # and the Euler input term differs from it (the two forms are not confused)
    assert not np.allclose(run(c)["out"], want, rtol=1e-6, atol=1e-8)


def test_delta_limits():
    c = rand_case(batch=1, dim=2, L=6, N=3, gate=False, seed=9)
    # Δ -> 0: the state is kept and the input ignored
    c0 = dict(c, delta=np.full_like(c["delta"], -60.0), dt_bias=np.zeros(2))
    res = run(c0)
    y = np.einsum("bnt,bdn->bdt", c["C"], c["h0"]) + c["D"][None, :, None] * c["u"]
    np.testing.assert_allclose(res["out"], y, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(res["hL"], c["h0"], rtol=1e-12)
    # Δ large with A <= -1: the state resets to the current input term Δ B_t x_t
    c1 = dict(c, delta=np.full_like(c["delta"], 100.0), dt_bias=np.zeros(2), A=c["A"] - 1.0)
    res = run(c1)
    dt = 100.0
    y = dt * np.einsum("bnt,bnt->bt", c["C"], c["B"])[:, None, :] * c["u"] + c["D"][None, :, None] * c["u"]
    np.testing.assert_allclose(res["out"], y, rtol=1e-10, atol=1e-10)


@pytest.mark.parametrize("splits", [[1], [3, 5], [2, 3, 4, 9]])
def test_chunked_equals_sequential(splits):
    c = rand_case(batch=2, dim=3, L=12, N=4, seed=13)
    full = run(c)
    h, outs, start = c["h0"], [], 0
    for end in splits + [12]:
        part = {k: (v[..., start:end] if (k in ("u", "delta", "z", "B", "C") and v is not None) else v)
                for k, v in c.items()}
        part["h0"] = h
        r = run(part)
        outs.append(r["out"])
        h = r["hL"]
        start = end
    np.testing.assert_allclose(np.concatenate(outs, -1), full["out"], rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(h, full["hL"], rtol=1e-13, atol=1e-14)


def test_superposition_in_u():
    c = rand_case(batch=1, dim=3, L=20, N=4, gate=False, h0=False, seed=17)
    u2 = np.random.default_rng(3).standard_normal(c["u"].shape)
    y1 = run(c)["out"]
    y2 = run(dict(c, u=u2))["out"]
    y12 = run(dict(c, u=c["u"] + u2))["out"]
    np.testing.assert_allclose(y12, y1 + y2, rtol=1e-11, atol=1e-12)


def test_decode_steps_equal_scan():
    c = rand_case(batch=2, dim=3, L=9, N=4, seed=21)
    full = run(c)
    state = np.ascontiguousarray(c["h0"].copy())
    for t in range(9):
        o = oracle.state_update(state, c["u"][..., t], c["delta"][..., t], c["A"], c["B"][..., t],
                                c["C"][..., t], D=c["D"], z=c["z"][..., t], dt_bias=c["dt_bias"])
        np.testing.assert_allclose(o, full["out"][..., t], rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(state, full["hL"], rtol=1e-13, atol=1e-14)


@pytest.mark.parametrize("zoh,groups", [(True, 1), (False, 2), (True, 2)])
def test_decode_steps_equal_scan_variants(zoh, groups):
    """The decode step with the ZOH coefficient and with grouped B/C reproduces the scan (whose
    ZOH form is pinned by the gating case and finite differences, and grouped form by the
    per-group quadratic form)."""
    c = rand_case(batch=2, dim=4, L=9, N=3, seed=25)
    c["A"][1, 2] = 0.0  # the A -> 0 limit of the ZOH coefficient
    if groups > 1:
        r = np.random.default_rng(26)
        c["B"] = r.standard_normal((2, groups, 3, 9))
        c["C"] = r.standard_normal((2, groups, 3, 9))
    full = run(c, zoh=zoh)
    state = np.ascontiguousarray(c["h0"].copy())
    for t in range(9):
        o = oracle.state_update(state, c["u"][..., t], c["delta"][..., t], c["A"], c["B"][..., t],
                                c["C"][..., t], D=c["D"], z=c["z"][..., t], dt_bias=c["dt_bias"],
                                zoh=zoh)
        np.testing.assert_allclose(o, full["out"][..., t], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(state, full["hL"], rtol=1e-12, atol=1e-13)


def test_channel_subset_matches_full():
    c = rand_case(batch=2, dim=5, L=10, N=3, seed=23)
    full = run(c)
    sub = run(c, channels=[1, 7, 9])
    flat_full = full["out"].reshape(10, -1)
    flat_sub = sub["out"].reshape(10, -1)
    for ch in (1, 7, 9):
        np.testing.assert_array_equal(flat_sub[ch], flat_full[ch])
    assert not flat_sub[0].any()


def _bwd(c, dout, dhL, channels=None):
    return oracle.scan_bwd(c["u"], c["delta"], c["A"], c["B"], c["C"], dout, D=c["D"], z=c["z"],
                           dt_bias=c["dt_bias"], h0=c["h0"], dhL=dhL, channels=channels)


def _one_channel(c, dout, dhL, b, d):
    """The problem restricted to the single channel (b, d): a 1 x 1 scan with that channel's
    rows, parameters and batch row of B, C."""
    one = dict(u=c["u"][b:b + 1, d:d + 1], delta=c["delta"][b:b + 1, d:d + 1],
               A=c["A"][d:d + 1], B=c["B"][b:b + 1], C=c["C"][b:b + 1], D=c["D"][d:d + 1],
               z=c["z"][b:b + 1, d:d + 1], dt_bias=c["dt_bias"][d:d + 1],
               h0=c["h0"][b:b + 1, d:d + 1])
    return one, dout[b:b + 1, d:d + 1], dhL[b:b + 1, d:d + 1]


def test_backward_channel_subset():
    """The channel-subset mode of the backward (used to check large workloads on sampled
    channels): per-channel gradients equal the full run's; the summed gradients of one listed
    channel equal those of the 1 x 1 problem cut out of the inputs (the unsubsetted code path on
    a different problem); and the summed gradients of a partition of the channels add up to the
    full run's (every channel contributes exactly its own share, once)."""
    batch, dim, L, N = 2, 5, 9, 3
    c = rand_case(batch=batch, dim=dim, L=L, N=N, seed=29)
    r = np.random.default_rng(30)
    dout = r.standard_normal((batch, dim, L))
    dhL = r.standard_normal((batch, dim, N))
    full = _bwd(c, dout, dhL)
    sub_idx = [1, 7, 9]                                  # flat b * dim + d
    sub = _bwd(c, dout, dhL, channels=sub_idx)
    for k in ("du", "ddelta", "dz", "dh0"):
        fs, ss = full[k].reshape(batch * dim, -1), sub[k].reshape(batch * dim, -1)
        for ch in sub_idx:
            np.testing.assert_array_equal(ss[ch], fs[ch], err_msg=k)
    # one listed channel: its share equals the whole gradient of the cut-out 1 x 1 problem
    for ch in (7, 3):
        b, d = divmod(ch, dim)
        g1 = _bwd(*_one_channel(c, dout, dhL, b, d))
        gs = _bwd(c, dout, dhL, channels=[ch])
        np.testing.assert_allclose(gs["dA"][d], g1["dA"][0], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(gs["dD"][d], g1["dD"][0], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(gs["ddt_bias"][d], g1["ddt_bias"][0], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(gs["dB"][b], g1["dB"][0], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(gs["dC"][b], g1["dC"][0], rtol=1e-12, atol=1e-14)
        # nothing outside the listed channel's d (for dA, dD, ddt_bias) or row b (for dB, dC)
        others = [i for i in range(dim) if i != d]
        assert not gs["dA"][others].any() and not gs["dD"][others].any()
        assert not gs["ddt_bias"][others].any()
        assert not gs["dB"][1 - b].any() and not gs["dC"][1 - b].any()
    # a partition of the channels: the shares add up to the full sums
    rest = [i for i in range(batch * dim) if i not in sub_idx]
    other = _bwd(c, dout, dhL, channels=rest)
    for k in ("dA", "dB", "dC", "dD", "ddt_bias"):
        np.testing.assert_allclose(sub[k] + other[k], full[k], rtol=1e-12, atol=1e-13, err_msg=k)


# ------------------------------------------------------------------ gradients
def loss_and_grads(c, dout, dhL, softplus=True, zoh=False):
    res = run(c, delta_softplus=softplus, zoh=zoh)
    loss = np.sum(res["out"] * dout) + np.sum(res["hL"] * dhL)
    return loss


@pytest.mark.parametrize("gate,softplus,zoh", [(True, True, False), (False, True, False),
                                               (True, False, False), (True, True, True),
                                               (False, False, True)])
def test_gradients_by_finite_differences(gate, softplus, zoh):
    c = rand_case(batch=2, dim=2, L=5, N=3, gate=gate, seed=31)
    if not softplus:
        c["delta"] = np.abs(c["delta"]) + 0.1
        c["dt_bias"] = np.full(2, 0.05)
    if zoh:
        c["A"][0, 1] = 0.0        # the A -> 0 limit of the ZOH coefficient
        c["A"][1, 2] = -3e-4      # |ΔA| small: the series branch of dc/dA
    r = np.random.default_rng(5)
    dout = r.standard_normal(c["u"].shape)
    dhL = r.standard_normal(c["h0"].shape)
    g = oracle.scan_bwd(c["u"], c["delta"], c["A"], c["B"], c["C"], dout, D=c["D"], z=c["z"],
                        dt_bias=c["dt_bias"], delta_softplus=softplus, h0=c["h0"], dhL=dhL,
                        zoh=zoh)
    names = {"u": "du", "delta": "ddelta", "A": "dA", "B": "dB", "C": "dC", "D": "dD",
             "dt_bias": "ddt_bias", "h0": "dh0"}
    if gate:
        names["z"] = "dz"
    eps = 1e-6
    for key, gname in names.items():
        x = c[key]
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            i = it.multi_index
            xp = x.copy(); xp[i] += eps
            xm = x.copy(); xm[i] -= eps
            num[i] = (loss_and_grads(dict(c, **{key: xp}), dout, dhL, softplus, zoh)
                      - loss_and_grads(dict(c, **{key: xm}), dout, dhL, softplus, zoh)) / (2 * eps)
        np.testing.assert_allclose(g[gname], num, rtol=2e-6, atol=2e-7, err_msg=gname)


# ------------------------------------------------------------------ scalar decay (one A per channel)
def scalar_decay_matrix_form(c, a_d, softplus=True):
    """Scalar decay as one masked matrix product per channel: y = (M o (C^T B)) (Δ u) with
    M[t, s] = exp(a_d (cs[t+1] - cs[s+1])) for s <= t, plus the decayed h0 and D u.  The N-state
    dot products C_t . B_s form a Gram matrix, so no recurrence is run."""
    u, B, C = c["u"], c["B"], c["C"]
    batch, dim, L = u.shape
    v = c["delta"] + c["dt_bias"][None, :, None]
    dt = softplus_ref(v) if softplus else v
    out = np.zeros_like(u)
    tri = np.tril(np.ones((L, L), bool))
    for b in range(batch):
        G = C[b].T @ B[b]                                  # G[t, s] = C_t . B_s
        for d in range(dim):
            cs = np.cumsum(dt[b, d])                       # cs[t] = sum_{r<=t} Δ_r
            M = np.where(tri, np.exp(a_d[d] * (cs[:, None] - cs[None, :])), 0.0)
            y = (M * G) @ (dt[b, d] * u[b, d])
            if c["h0"] is not None:
                y += np.exp(a_d[d] * cs) * (C[b].T @ c["h0"][b, d])
            y += c["D"][d] * u[b, d]
            if c["z"] is not None:
                zz = c["z"][b, d]
                y = y * zz * expit(zz)
            out[b, d] = y
    return out


def test_scalar_decay_matrix_form():
    """The oracle with A[d, n] = a_d for every n against the masked-matrix (dual) form."""
    c = rand_case(batch=2, dim=3, L=48, N=16, seed=61)
    a_d = -np.exp(np.random.default_rng(62).standard_normal(3))
    c["A"] = np.repeat(a_d[:, None], 16, 1)
    np.testing.assert_allclose(run(c)["out"], scalar_decay_matrix_form(c, a_d),
                               rtol=1e-10, atol=1e-11)


def test_scalar_decay_gradient_is_the_state_sum():
    """dL/da_d of a shared rate equals the sum over n of the oracle's per-state dA[d, n]
    (chain rule through A[d, n] = a_d), checked against central differences in a_d."""
    c = rand_case(batch=2, dim=2, L=6, N=4, seed=63)
    a_d = np.array([-0.7, -2.1])
    c["A"] = np.repeat(a_d[:, None], 4, 1)
    r = np.random.default_rng(64)
    dout = r.standard_normal(c["u"].shape)
    dhL = r.standard_normal(c["h0"].shape)
    g = oracle.scan_bwd(c["u"], c["delta"], c["A"], c["B"], c["C"], dout, D=c["D"], z=c["z"],
                        dt_bias=c["dt_bias"], h0=c["h0"], dhL=dhL)
    eps = 1e-6
    for d in range(2):
        ap, am = a_d.copy(), a_d.copy()
        ap[d] += eps
        am[d] -= eps
        lp = loss_and_grads(dict(c, A=np.repeat(ap[:, None], 4, 1)), dout, dhL)
        lm = loss_and_grads(dict(c, A=np.repeat(am[:, None], 4, 1)), dout, dhL)
        np.testing.assert_allclose(g["dA"][d].sum(), (lp - lm) / (2 * eps), rtol=2e-6, atol=2e-7)


# ------------------------------------------------------------------ reverse scan
def quadratic_form_reverse(c, softplus=True):
    """Anti-causal form: y_t = sum_{s>=t} C_t . exp(A sum_{r=t}^{s-1} Δ_r) Δ_s B_s u_s
    + C_t . exp(A sum_{r=t}^{L-1} Δ_r) h0 + D u_t, then * silu(z_t) (h0 enters at t = L-1)."""
    u, A, B, C = c["u"], c["A"], c["B"], c["C"]
    batch, dim, L = u.shape
    v = c["delta"] + c["dt_bias"][None, :, None]
    dt = softplus_ref(v) if softplus else v
    out = np.zeros_like(u)
    for b in range(batch):
        for d in range(dim):
            cs = np.concatenate([[0.0], np.cumsum(dt[b, d])])  # cs[k] = sum_{r<k} Δ_r
            for t in range(L):
                y = 0.0
                for s_ in range(t, L):
                    decay = np.exp(A[d] * (cs[s_] - cs[t]))
                    y += np.sum(C[b, :, t] * decay * dt[b, d, s_] * B[b, :, s_]) * u[b, d, s_]
                if c["h0"] is not None:
                    y += np.sum(C[b, :, t] * np.exp(A[d] * (cs[L] - cs[t])) * c["h0"][b, d])
                y += c["D"][d] * u[b, d, t]
                if c["z"] is not None:
                    zz = c["z"][b, d, t]
                    y *= zz * expit(zz)
                out[b, d, t] = y
    return out


@pytest.mark.parametrize("gate,h0", [(True, True), (False, False)])
def test_reverse_quadratic_form(gate, h0):
    c = rand_case(batch=2, dim=3, L=9, N=3, gate=gate, h0=h0, seed=71)
    got = run(c, reverse=True)["out"]
    np.testing.assert_allclose(got, quadratic_form_reverse(c), rtol=1e-11, atol=1e-12)
    # a reverse scan is not the forward scan: the pin tells them apart
    assert not np.allclose(run(c)["out"], got, rtol=1e-3)


def test_reverse_final_state_single_step_chain():
    """hL of the reverse scan is the state after t = 0: for L = 2 it is
    a_0 (a_1 h0 + b_1) + b_0 with a_t = exp(Δ_t A), b_t = Δ_t B_t u_t."""
    c = rand_case(batch=1, dim=2, L=2, N=4, seed=72)
    dt = softplus_ref(c["delta"] + c["dt_bias"][None, :, None])[0]          # [d, t]
    a = np.exp(dt[:, :, None] * c["A"][:, None, :])                         # [d, t, n]
    bt = dt[:, :, None] * c["B"][0].T[None] * c["u"][0][:, :, None]          # [d, t, n]
    h = a[:, 0] * (a[:, 1] * c["h0"][0] + bt[:, 1]) + bt[:, 0]
    np.testing.assert_allclose(run(c, reverse=True)["hL"][0], h, rtol=1e-13, atol=1e-14)


def test_reverse_gradients_by_finite_differences():
    c = rand_case(batch=1, dim=2, L=5, N=3, seed=73)
    r = np.random.default_rng(74)
    dout = r.standard_normal(c["u"].shape)
    dhL = r.standard_normal(c["h0"].shape)
    g = oracle.scan_bwd(c["u"], c["delta"], c["A"], c["B"], c["C"], dout, D=c["D"], z=c["z"],
                        dt_bias=c["dt_bias"], h0=c["h0"], dhL=dhL, reverse=True)

    def loss(cc):
        res = run(cc, reverse=True)
        return np.sum(res["out"] * dout) + np.sum(res["hL"] * dhL)

    eps = 1e-6
    for key, gname in (("u", "du"), ("delta", "ddelta"), ("B", "dB"), ("C", "dC"), ("z", "dz"),
                       ("A", "dA"), ("h0", "dh0")):
        x = c[key]
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            i = it.multi_index
            xp = x.copy(); xp[i] += eps
            xm = x.copy(); xm[i] -= eps
            num[i] = (loss(dict(c, **{key: xp})) - loss(dict(c, **{key: xm}))) / (2 * eps)
        np.testing.assert_allclose(g[gname], num, rtol=2e-6, atol=2e-7, err_msg=gname)


# ------------------------------------------------------------------ grouped B/C
def test_grouped_bc_quadratic_form():
    """B, C of shape [batch, G, N, L]: channel d reads group d // (dim // G); each group against
    the brute-force quadratic form of its own channels."""
    c = rand_case(batch=2, dim=6, L=7, N=3, seed=81)
    r = np.random.default_rng(82)
    Bg = r.standard_normal((2, 3, 3, 7))
    Cg = r.standard_normal((2, 3, 3, 7))
    got = oracle.scan_fwd(c["u"], c["delta"], c["A"], Bg, Cg, D=c["D"], z=c["z"],
                          dt_bias=c["dt_bias"], h0=c["h0"])["out"]
    for g in range(3):
        sl = slice(2 * g, 2 * g + 2)
        cg = dict(c, u=c["u"][:, sl], delta=c["delta"][:, sl], A=c["A"][sl], D=c["D"][sl],
                  z=c["z"][:, sl], dt_bias=c["dt_bias"][sl], h0=c["h0"][:, sl],
                  B=Bg[:, g], C=Cg[:, g])
        np.testing.assert_allclose(got[:, sl], quadratic_form(cg), rtol=1e-11, atol=1e-12)


def test_grouped_bc_gradients_by_finite_differences():
    c = rand_case(batch=1, dim=4, L=5, N=2, seed=83)
    r = np.random.default_rng(84)
    c["B"] = r.standard_normal((1, 2, 2, 5))
    c["C"] = r.standard_normal((1, 2, 2, 5))
    dout = r.standard_normal(c["u"].shape)
    dhL = r.standard_normal(c["h0"].shape)
    g = oracle.scan_bwd(c["u"], c["delta"], c["A"], c["B"], c["C"], dout, D=c["D"], z=c["z"],
                        dt_bias=c["dt_bias"], h0=c["h0"], dhL=dhL)
    assert g["dB"].shape == (1, 2, 2, 5)
    eps = 1e-6
    for key, gname in (("B", "dB"), ("C", "dC"), ("u", "du"), ("A", "dA"), ("h0", "dh0")):
        x = c[key]
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            i = it.multi_index
            xp = x.copy(); xp[i] += eps
            xm = x.copy(); xm[i] -= eps
            num[i] = (loss_and_grads(dict(c, **{key: xp}), dout, dhL)
                      - loss_and_grads(dict(c, **{key: xm}), dout, dhL)) / (2 * eps)
        np.testing.assert_allclose(g[gname], num, rtol=2e-6, atol=2e-7, err_msg=gname)


def test_combined_variants_forward_quadratic_form():
    """Reverse scan + ZOH input term + grouped B/C at once, against the anti-causal quadratic
    form with the hold integral as input coefficient and each channel's group of B/C:
    h_t = sum_{s>=t} (prod_{r=t..s-1} exp(Δ_r A)) hold(Δ_s) B_s u_s + (prod_{r>=t} exp(Δ_r A)) h0."""
    c = rand_case(batch=2, dim=4, L=7, N=3, seed=93)
    r = np.random.default_rng(94)
    G = 2
    Bg = r.standard_normal((2, G, 3, 7))
    Cg = r.standard_normal((2, G, 3, 7))
    c["A"][1, 2] = 0.0
    u, A = c["u"], c["A"]
    batch, dim, L = u.shape
    N = A.shape[1]
    dt = softplus_ref(c["delta"] + c["dt_bias"][None, :, None])
    want = np.zeros_like(u)
    for b in range(batch):
        for d in range(dim):
            g = d // (dim // G)
            B, C = Bg[b, g], Cg[b, g]                                   # [n, t]
            cs = np.concatenate([[0.0], np.cumsum(dt[b, d])])          # cs[k] = sum_{r<k} Δ_r
            for t in range(L):
                h = np.exp(A[d] * (cs[L] - cs[t])) * c["h0"][b, d]
                for s_ in range(t, L):
                    hold = np.array([hold_integral(dt[b, d, s_], A[d, n]) for n in range(N)])
                    h = h + np.exp(A[d] * (cs[s_] - cs[t])) * hold * B[:, s_] * u[b, d, s_]
                y = np.sum(C[:, t] * h) + c["D"][d] * u[b, d, t]
                zz = c["z"][b, d, t]
                want[b, d, t] = y * zz * expit(zz)
    got = oracle.scan_fwd(u, c["delta"], A, Bg, Cg, D=c["D"], z=c["z"], dt_bias=c["dt_bias"],
                          h0=c["h0"], reverse=True, zoh=True)["out"]
    np.testing.assert_allclose(got, want, rtol=1e-11, atol=1e-12)


def test_combined_variants_gradients_by_finite_differences():
    """Reverse scan, ZOH input term and grouped B/C at once (the variants compose in the
    oracle's wrappers): every gradient against central differences of the same forward."""
    c = rand_case(batch=1, dim=4, L=5, N=2, seed=91)
    r = np.random.default_rng(92)
    c["B"] = r.standard_normal((1, 2, 2, 5))
    c["C"] = r.standard_normal((1, 2, 2, 5))
    c["A"][2, 0] = 0.0                     # the A -> 0 limit of the ZOH coefficient
    dout = r.standard_normal(c["u"].shape)
    dhL = r.standard_normal(c["h0"].shape)
    kw = dict(reverse=True, zoh=True)
    g = oracle.scan_bwd(c["u"], c["delta"], c["A"], c["B"], c["C"], dout, D=c["D"], z=c["z"],
                        dt_bias=c["dt_bias"], h0=c["h0"], dhL=dhL, **kw)

    def loss(cc):
        res = run(cc, **kw)
        return np.sum(res["out"] * dout) + np.sum(res["hL"] * dhL)

    eps = 1e-6
    for key, gname in (("u", "du"), ("delta", "ddelta"), ("A", "dA"), ("B", "dB"), ("C", "dC"),
                       ("D", "dD"), ("z", "dz"), ("dt_bias", "ddt_bias"), ("h0", "dh0")):
        x = c[key]
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            i = it.multi_index
            xp = x.copy(); xp[i] += eps
            xm = x.copy(); xm[i] -= eps
            num[i] = (loss(dict(c, **{key: xp})) - loss(dict(c, **{key: xm}))) / (2 * eps)
        np.testing.assert_allclose(g[gname], num, rtol=2e-6, atol=2e-7, err_msg=gname)


def test_planted_mistake_is_caught():
    """A plausible oracle mistake (reading out h_{t-1} instead of h_t) must fail the pins:
    emulate it by shifting the readout and check the quadratic form tells the two apart."""
    c = rand_case(batch=1, dim=2, L=6, N=2, gate=False, seed=41)
    good = run(c)["out"]
    ref = quadratic_form(c)
    assert np.allclose(good, ref, rtol=1e-11, atol=1e-12)
    # readout of the previous state, computed from the oracle's own pieces
    full_prev = []
    h = c["h0"]
    for t in range(6):
        part = {k: (v[..., t:t + 1] if (k in ("u", "delta", "z", "B", "C") and v is not None) else v)
                for k, v in c.items()}
        part["h0"] = h
        y_prev = np.einsum("bn,bdn->bd", c["C"][..., t], h) + c["D"] * c["u"][..., t]
        full_prev.append(y_prev)
        h = run(part)["hL"]
    wrong = np.stack(full_prev, -1)
    assert not np.allclose(wrong, ref, rtol=1e-3, atol=1e-3)


def test_golden_regression_fixture():
    """The oracle still reproduces its frozen output (tests/golden/oracle_tiny_seed99.json)."""
    import json
    import os
    from selective_state_space_23_b200.inputs import make_inputs, to_f64, workload
    path = os.path.join(os.path.dirname(__file__), "golden", "oracle_tiny_seed99.json")
    with open(path) as fh:
        gold = json.load(fh)
    w = workload("tiny_f32", dim=4, seqlen=24, dstate=5)
    f = {k: to_f64(v) for k, v in make_inputs(w, seed=99, with_dout=True, with_h0=True).items()}
    fwd = oracle.scan_fwd(f["u"], f["delta"], f["A"], f["B"], f["C"], D=f["D"], z=f["z"],
                          dt_bias=f["dt_bias"], h0=f["h0"])
    np.testing.assert_allclose(fwd["out"].ravel(), gold["out"], rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(fwd["hL"].ravel(), gold["hL"], rtol=1e-13, atol=1e-15)
    bwd = oracle.scan_bwd(f["u"], f["delta"], f["A"], f["B"], f["C"], f["dout"], D=f["D"], z=f["z"],
                          dt_bias=f["dt_bias"], h0=f["h0"])
    for k, v in gold["grads"].items():
        np.testing.assert_allclose(bwd[k].ravel(), v, rtol=1e-12, atol=1e-14, err_msg=k)
