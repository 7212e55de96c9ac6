"""GPU parity of the stage-1 training step (lizard_stage1_step: forward, mean
squared error against a teacher attention output, every gradient of the loss)
against the oracle, through the C ABI."""

import numpy as np
import pytest
import torch

from gated_linear_sliding_chunkwise_b200.synth import WORKLOADS, Workload, make_inputs, random_alpha
from lizard_testutil import check, gate_of, head_inputs, to64, to_device
from oracle import lizard_ref as ref

pytestmark = pytest.mark.gpu

GRADS = ["dq", "dk", "dv", "dg", "dmeta_k", "dmeta_v", "dfmap_wq", "dfmap_wk", "dalpha",
         "dstate_in"]


@pytest.fixture(scope="module")
def lz():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from gated_linear_sliding_chunkwise_b200 import lizard
    return lizard


def _impl(lz, name):
    return {"simt": lz.IMPL_SIMT, "tc": lz.IMPL_TC, "auto": lz.IMPL_AUTO}[name]


def _target(shape, dtype, seed):
    """Teacher attention output: seeded synthetic values of the output's scale."""
    gen = torch.Generator().manual_seed(seed)
    return (torch.randn(*shape, generator=gen) / 8).to(dtype)


def _kw(x, w):
    return dict(window=w.window, chunk=w.chunk, gate_temp=w.gate_temp, fmap_wq=x.get("fmap_wq"),
                fmap_wk=x.get("fmap_wk"), meta_k=x.get("meta_k"), meta_v=x.get("meta_v"),
                alpha=x.get("alpha"), state_in=x.get("state_in"))


def _oracle(inp, target, w):
    x = {k_: to64(v_) for k_, v_ in inp.items() if v_ is not None}
    return ref.lizard_stage1_step(x["q"], x["k"], x["v"], x["g"], to64(target), window=w.window,
                                  tau=w.gate_temp, fmap_wq=x.get("fmap_wq"), fmap_wk=x.get("fmap_wk"),
                                  meta_k=x.get("meta_k"), meta_v=x.get("meta_v"), alpha=x.get("alpha"),
                                  state_in=x.get("state_in"), gate=gate_of(x))


CASES = [
    # impl, dtype, d, L, window, M, gate, want_o
    ("simt", "fp32", 64, 97, 16, 4, "dim", True),
    ("simt", "fp32", 64, 70, 5, 0, "scalar", False),
    ("tc", "bf16", 128, 300, 128, 4, "dim", True),
    ("tc", "bf16", 128, 300, 64, 4, "scalar", False),
    ("tc", "bf16", 128, 1100, 128, 4, "dim", False),    # few sequences: segmented forward
]


@pytest.mark.parametrize("impl,dtype,d,L,window,M,gate,want_o", CASES)
def test_stage1_step_matches_oracle(lz, impl, dtype, d, L, window, M, gate, want_o):
    B, H = (2, 2) if L < 1000 else (1, 2)
    w = Workload("stage1", B=B, H=H, L=L, d=d, window=window, M=M, dtype=dtype, seed=400 + L,
                 gate=gate)
    inp = make_inputs(w)
    if M == 0:
        inp["meta_k"] = inp["meta_v"] = None
    inp["state_in"] = torch.randn(B, H, d, d, generator=torch.Generator().manual_seed(4)) * 0.1
    inp["alpha"] = random_alpha(H, seed=L)
    target = _target((B, H, L, d), inp["q"].dtype, seed=L)
    x = to_device(inp)
    got = lz.stage1_step(x["q"], x["k"], x["v"], x["g"], target.cuda(), impl=_impl(lz, impl),
                         want_o=want_o, **_kw(x, w))
    assert lz.workspace_status(got["workspace"]) == lz.OK
    want = _oracle(inp, target, w)
    loss = float(got["loss"].item())
    assert abs(loss - want["loss"]) <= (1e-5 if dtype == "fp32" else 1e-2) * want["loss"], \
        (loss, want["loss"])
    if want_o:
        check("o", got["o"], want["o"], dtype)
    else:
        assert got["o"] is None
    for name in GRADS:
        if want[name] is None:
            assert got[name] is None
            continue
        check(name, got[name], want[name], dtype)


def test_stage1_plans(lz):
    w = Workload("plan", B=1, H=2, L=256, d=128, window=128, M=4, dtype="bf16", seed=1)
    x = to_device(make_inputs(w))
    t = torch.zeros_like(x["q"])
    fused = lz.stage1_step(x["q"], x["k"], x["v"], x["g"], t, plan_only=True, **_kw(x, w))
    assert "mse_kernel" not in fused and "tc_fwd_kernel" in fused
    portable = lz.stage1_step(x["q"], x["k"], x["v"], x["g"], t, impl=lz.IMPL_SIMT, plan_only=True,
                              **_kw(x, w))
    assert "mse_kernel" in portable


def test_stage1_train_step_full_size(lz):
    """The training-step shape (B=8, H=32, L=2048) as the default path runs it:
    the loss against the mean squared error of the step's own output (fp64 on
    the host), and sampled sequences' output and gradients against the
    oracle, whose dL/do uses the full element count."""
    w = WORKLOADS["train_step"]
    inp = make_inputs(w, with_dout=False)
    target = _target(inp["q"].shape, inp["q"].dtype, seed=77)
    x = to_device(inp)
    got = lz.stage1_step(x["q"], x["k"], x["v"], x["g"], target.cuda(), want_o=True, **_kw(x, w))
    torch.cuda.synchronize()
    assert lz.workspace_status(got["workspace"]) == lz.OK
    o64, t64 = to64(got["o"]), to64(target)
    host_loss = float(np.mean((o64 - t64) ** 2))
    # the kernel uses o before its bf16 rounding: agreement to the rounding's size
    assert abs(float(got["loss"].item()) - host_loss) <= 1e-2 * host_loss
    n = o64.size
    for (b, h) in [(0, 0), (6, 17)]:
        xh = head_inputs(inp, b, h, keys=("q", "k", "v", "g"))
        kw = dict(window=w.window, tau=w.gate_temp, fmap_wq=xh["fmap_wq"], fmap_wk=xh["fmap_wk"],
                  meta_k=xh["meta_k"], meta_v=xh["meta_v"], alpha=xh["alpha"])
        o = ref.lizard_forward(xh["q"], xh["k"], xh["v"], xh["g"], **kw)["o"]
        check(f"o[{b},{h}]", got["o"][b:b + 1, h:h + 1], o, "bf16")
        dout = 2.0 * (o - t64[b:b + 1, h:h + 1]) / n
        want = ref.lizard_backward(xh["q"], xh["k"], xh["v"], xh["g"], dout, **kw)
        for name in ("dq", "dk", "dv", "dg", "dstate_in"):
            check(f"{name}[{b},{h}]", got[name][b:b + 1, h:h + 1], want[name], "bf16")
