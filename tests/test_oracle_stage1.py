"""Pins for the oracle's stage-1 training step (attention approximation: the
mean squared error between the layer's output and a teacher's attention
output, English summary section 2.B, Chinese summary section 2.2).  CPU only."""

import numpy as np
import pytest

from oracle import lizard_ref as ref


def _inputs(B=1, H=2, L=7, d=4, M=2, seed=21, gate=ref.GATE_PER_DIM):
    r = np.random.default_rng(seed)
    gshape = (B, H, L, d) if gate == ref.GATE_PER_DIM else (B, H, L)
    x = {"q": r.standard_normal((B, H, L, d)) * 0.7, "k": r.standard_normal((B, H, L, d)) * 0.7,
         "v": r.standard_normal((B, H, L, d)), "g": r.standard_normal(gshape) * 1.5}
    kw = {"fmap_wq": r.standard_normal((H, d, d // 2)), "fmap_wk": r.standard_normal((H, d, d // 2)),
          "meta_k": r.standard_normal((H, M, d)), "meta_v": r.standard_normal((H, M, d)),
          "alpha": r.uniform(0.2, 1.8, H), "state_in": r.standard_normal((B, H, d, d)) * 0.3}
    target = r.standard_normal((B, H, L, d))
    return x, kw, target


def test_target_equal_to_the_output_gives_zero_loss_and_gradients():
    x, kw, _ = _inputs()
    o = ref.lizard_forward(**x, window=3, **kw)["o"]
    res = ref.lizard_stage1_step(**x, target=o, window=3, **kw)
    assert res["loss"] == 0.0
    for name in ("dq", "dk", "dv", "dg", "dmeta_k", "dmeta_v", "dfmap_wq", "dfmap_wk", "dalpha",
                 "dstate_in"):
        assert np.all(res[name] == 0.0), name


def test_constant_offset_target():
    """y = o - c: every squared error is c^2, so the loss is c^2 and dL/do is
    the constant 2c/n."""
    x, kw, _ = _inputs()
    o = ref.lizard_forward(**x, window=3, **kw)["o"]
    c = 0.375
    loss, dout = ref.attention_mse(o, o - c)
    assert abs(loss - c * c) < 1e-15
    np.testing.assert_allclose(dout, np.full(o.shape, 2 * c / o.size), rtol=1e-13)


@pytest.mark.parametrize("gate", [ref.GATE_PER_DIM, ref.GATE_SCALAR])
def test_stage1_gradients_match_central_differences(gate):
    """Every gradient of the loss against central differences of the loss
    itself (forward + MSE, fp64)."""
    window = 3
    x, kw, target = _inputs(gate=gate)
    res = ref.lizard_stage1_step(**x, target=target, window=window, gate=gate, **kw)

    def loss():
        o = ref.lizard_forward(**x, window=window, gate=gate, **kw)["o"]
        return float(np.mean((o - target) ** 2))

    assert abs(res["loss"] - loss()) < 1e-14
    eps = 1e-6
    for name, gname in [("q", "dq"), ("k", "dk"), ("v", "dv"), ("g", "dg"),
                        ("fmap_wq", "dfmap_wq"), ("meta_v", "dmeta_v"), ("alpha", "dalpha"),
                        ("state_in", "dstate_in")]:
        base = x[name] if name in x else kw[name]
        num = np.zeros_like(base)
        it = np.nditer(base, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            orig = base[idx]
            base[idx] = orig + eps
            lp = loss()
            base[idx] = orig - eps
            lm = loss()
            base[idx] = orig
            num[idx] = (lp - lm) / (2 * eps)
        scale = max(np.max(np.abs(num)), 1e-12)
        err = np.max(np.abs(res[gname] - num)) / scale
        assert err < 1e-6, f"{gname}: rel err {err:.2e}"
