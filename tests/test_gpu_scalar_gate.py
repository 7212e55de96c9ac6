"""GPU parity of the scalar (per-head) gate -- one gate logit per token and
head, shared by every key dimension -- against the oracle, through the C ABI:
forward, backward and decode, on the portable and the tensor-core kernels."""

import numpy as np
import pytest
import torch

from gated_linear_sliding_chunkwise_b200.synth import WORKLOADS, Workload, make_inputs, random_alpha
from lizard_testutil import check, oracle_backward, oracle_forward, report, to64, to_device
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


def _kw(x, w):
    return dict(window=w.window, chunk=w.chunk, gate_temp=w.gate_temp, fmap_wq=x.get("fmap_wq"),
                fmap_wk=x.get("fmap_wk"), meta_k=x.get("meta_k"), meta_v=x.get("meta_v"),
                alpha=x.get("alpha"), state_in=x.get("state_in"))


CASES = [
    # impl, dtype, d, B, H, L, window, M, state_in
    ("simt", "fp32", 64, 2, 2, 97, 16, 4, True),
    ("simt", "fp32", 128, 1, 2, 130, 100, 0, False),
    ("tc", "bf16", 128, 2, 2, 300, 128, 4, True),      # three tiles, ragged tail
    ("tc", "bf16", 128, 1, 2, 1100, 64, 4, True),      # few sequences: segmented forward
]


def _inputs(dtype, d, B, H, L, window, M, state, seed, train):
    w = Workload("scalar_gate", B=B, H=H, L=L, d=d, window=window, M=M, dtype=dtype, seed=seed,
                 kind="train" if train else "fwd", gate="scalar")
    inp = make_inputs(w)
    assert inp["g"].shape == (B, H, L)
    if M == 0:
        inp["meta_k"] = inp["meta_v"] = None
    if state:
        inp["state_in"] = torch.randn(B, H, d, d, generator=torch.Generator().manual_seed(3)) * 0.1
    inp["alpha"] = random_alpha(H, seed=L)
    return w, inp


@pytest.mark.parametrize("impl,dtype,d,B,H,L,window,M,state", CASES)
def test_scalar_gate_forward(lz, impl, dtype, d, B, H, L, window, M, state):
    w, inp = _inputs(dtype, d, B, H, L, window, M, state, seed=200 + L, train=False)
    x = to_device(inp)
    got = lz.attn_fwd(x["q"], x["k"], x["v"], x["g"], impl=_impl(lz, impl), want_state=True,
                      want_lse=True, **_kw(x, w))
    assert lz.workspace_status(got["workspace"]) == lz.OK
    want = oracle_forward(inp, window=window, tau=w.gate_temp)
    for name in ("o", "state_out", "lse"):
        check(name, got[name], want[name], dtype)


@pytest.mark.parametrize("impl,dtype,d,B,H,L,window,M,state", CASES)
def test_scalar_gate_backward(lz, impl, dtype, d, B, H, L, window, M, state):
    w, inp = _inputs(dtype, d, B, H, L, window, M, state, seed=300 + L, train=True)
    x = to_device(inp)
    got = lz.attn_bwd(x["q"], x["k"], x["v"], x["g"], x["dout"], impl=_impl(lz, impl), **_kw(x, w))
    assert lz.workspace_status(got["workspace"]) == lz.OK
    assert got["dg"].shape == (B, H, L)
    want = oracle_backward(inp, window=window, tau=w.gate_temp)
    for name in GRADS:
        if want[name] is None:
            assert got[name] is None
            continue
        check(name, got[name], want[name], dtype)


def test_scalar_gate_train_step_full_size_sampled_heads(lz):
    """The training-step shape (B=8, H=32, L=2048) with a scalar gate, as the
    default (tensor-core) path runs it; sampled sequences against the oracle."""
    base = WORKLOADS["train_step"]
    inp = make_inputs(base, gate="scalar")
    x = to_device(inp)
    fwd = lz.attn_fwd(x["q"], x["k"], x["v"], x["g"], **_kw(x, base))
    bwd = lz.attn_bwd(x["q"], x["k"], x["v"], x["g"], x["dout"], **_kw(x, base))
    torch.cuda.synchronize()
    pairs = [(0, 0), (5, 19)]
    wf = oracle_forward(inp, window=base.window, tau=base.gate_temp, pairs=pairs)
    wb = oracle_backward(inp, window=base.window, tau=base.gate_temp, pairs=pairs)
    for (b, h) in pairs:
        check(f"o[{b},{h}]", fwd["o"][b:b + 1, h:h + 1], wf[(b, h)]["o"], "bf16")
        for name in ("dq", "dk", "dv", "dg", "dstate_in"):
            check(f"{name}[{b},{h}]", bwd[name][b:b + 1, h:h + 1], wb[(b, h)][name], "bf16")


@pytest.mark.parametrize("dtype,d,window,M,pos0", [
    ("bf16", 128, 128, 4, 300),     # streaming kernel
    ("bf16", 128, 64, 0, 10),       # streaming kernel, partly filled window
    ("fp32", 64, 16, 4, 40),        # general kernel
])
def test_scalar_gate_decode_step(lz, dtype, d, window, M, pos0):
    w = Workload("dec_scalar", B=3, H=4, L=1, d=d, window=window, M=M, dtype=dtype, seed=9,
                 kind="decode", decode_pos=pos0, gate="scalar")
    inp = make_inputs(w)
    assert inp["g"].shape == (3, 4)
    if M == 0:
        inp["meta_k"] = inp["meta_v"] = None
    inp["alpha"] = random_alpha(4, seed=2)
    x = to_device(inp)
    o = lz.decode_step(x["q"], x["k"], x["v"], x["g"], x["state"], x["k_cache"], x["v_cache"],
                       x["pos"], gate_temp=w.gate_temp, fmap_wq=x.get("fmap_wq"),
                       fmap_wk=x.get("fmap_wk"), meta_k=x.get("meta_k"), meta_v=x.get("meta_v"),
                       alpha=x.get("alpha"))
    torch.cuda.synchronize()
    assert lz.decode_status() == lz.OK
    y = {k_: (to64(v_) if k_ != "pos" else v_.numpy()) for k_, v_ in inp.items() if v_ is not None}
    want_o, want_S, want_kc, _, want_pos = ref.lizard_decode_step(
        y["q"], y["k"], y["v"], y["g"], y["state"], y["k_cache"], y["v_cache"], y["pos"],
        window=window, tau=w.gate_temp, fmap_wq=y.get("fmap_wq"), fmap_wk=y.get("fmap_wk"),
        meta_k=y.get("meta_k"), meta_v=y.get("meta_v"), alpha=y.get("alpha"), gate=ref.GATE_SCALAR)
    check("o", o, want_o, dtype)
    check("state", x["state"], want_S, "fp32")
    assert torch.equal(x["k_cache"].cpu(), torch.from_numpy(want_kc).to(x["k_cache"].dtype))
    assert np.array_equal(x["pos"].cpu().numpy(), want_pos)


@pytest.mark.parametrize("gate", ["dim", "scalar"])
def test_feature_map_weight_gradients_keep_their_cancellation(lz, gate):
    """At the workloads' small feature-map weights the weight gradients are a
    small remainder of large per-feature terms; the tensor-core backward keeps
    them well inside the bf16 bar (hi + lo operands, row-0-centred state
    copies).  A regression guard at 0.4 of the bar."""
    w = Workload("wprec", B=2, H=2, L=512, d=128, dtype="bf16", seed=13, kind="train", gate=gate)
    inp = make_inputs(w)
    x = to_device(inp)
    got = lz.attn_bwd(x["q"], x["k"], x["v"], x["g"], x["dout"], impl=lz.IMPL_TC, **_kw(x, w))
    want = oracle_backward(inp, window=w.window, tau=w.gate_temp)
    for name in ("dfmap_wq", "dfmap_wk", "dg", "dstate_in"):
        g_, r_ = to64(got[name]), want[name]
        rel = float(np.max(np.abs(g_ - r_)) / np.max(np.abs(r_)))
        report(f"PARITY guard {name} ({gate} gate) normwise={rel:.3e}")
        assert rel <= 8e-3, f"{name}: {rel:.2e}"
