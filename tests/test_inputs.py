"""The shared seeded input generator: determinism, shapes, dtypes and the stated distributions."""
import numpy as np
import torch

from selective_state_space_23_b200.inputs import WORKLOADS, inv_softplus, make_inputs, workload


def test_deterministic_and_independent_per_tensor():
    w = workload("tiny_f32")
    a = make_inputs(w, seed=3)
    b = make_inputs(w, seed=3)
    c = make_inputs(w, seed=4)
    for k in a:
        assert torch.equal(a[k], b[k])
    assert not torch.equal(a["u"], c["u"])
    # adding an optional tensor does not change the others
    d = make_inputs(w, seed=3, with_dout=True, with_h0=True)
    for k in a:
        assert torch.equal(a[k], d[k])


def test_shapes_dtypes_and_recipe():
    w = workload("mamba370m_fwd", dim=256, seqlen=512)
    x = make_inputs(w, seed=0, with_dout=True)
    assert x["u"].shape == (8, 256, 512) and x["u"].dtype == torch.bfloat16
    assert x["B"].shape == (8, 16, 512) and x["C"].dtype == torch.bfloat16
    assert x["A"].dtype == torch.float32 and torch.equal(x["A"][3], -torch.arange(1, 17, dtype=torch.float32))
    assert abs(float(x["u"].float().std()) - 1.0) < 0.01
    assert abs(float(x["delta"].float().std()) - 0.5) < 0.01
    dt = np.log1p(np.exp(x["dt_bias"].double().numpy()))  # softplus(dt_bias) recovers dt
    assert dt.min() >= 1e-3 * 0.999 and dt.max() <= 1e-1 * 1.001


def test_inv_softplus_round_trip():
    y = np.array([1e-4, 1e-3, 0.05, 1.0, 7.0])
    np.testing.assert_allclose(np.logaddexp(0, inv_softplus(y)), y, rtol=1e-12)


def test_decode_steps_differ():
    w = WORKLOADS["decode_b256"]
    s0 = make_inputs(workload("decode_b256", batch=2, dim=8), seed=0, step=0)
    s1 = make_inputs(workload("decode_b256", batch=2, dim=8), seed=0, step=1)
    assert s0["x"].shape == (2, 8) and s0["B"].shape == (2, 16)
    assert not torch.equal(s0["x"], s1["x"])
    assert torch.equal(s0["A"], s1["A"]) and torch.equal(s0["dt_bias"], s1["dt_bias"])
    assert w.steps == 1024
