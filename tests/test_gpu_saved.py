"""Training forward + backward through the saved-for-backward buffer: the
forward writes the tiles' fp32 decay factors, their decayed start states S',
the final state and the anchor softmax normalisers, and the backward reads
them instead of recomputing.
Every gradient is held to the same oracle bar as the recomputing backward,
and the forward's own outputs do not change."""

import pytest
import torch

from gated_linear_sliding_chunkwise_b200.synth import WORKLOADS, Workload, make_inputs, random_alpha
from lizard_testutil import check, oracle_backward, oracle_forward, to64, to_device
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


def _kw(x, w, impl):
    return dict(window=w.window, chunk=w.chunk, gate_temp=w.gate_temp, fmap_wq=x.get("fmap_wq"),
                fmap_wk=x.get("fmap_wk"), meta_k=x.get("meta_k"), meta_v=x.get("meta_v"),
                alpha=x.get("alpha"), state_in=x.get("state_in"), impl=impl)


def _train(lz, x, w, impl, dstate_out=None, **extra):
    """Forward with a saved buffer, then the backward that reads it."""
    kw = {**_kw(x, w, impl), **extra}
    f = lz.attn_fwd(x["q"], x["k"], x["v"], x["g"], saved=True, want_state=True, want_lse=True, **kw)
    assert f["saved"] is not None
    assert lz.workspace_status(f["workspace"]) == lz.OK
    b = lz.attn_bwd(x["q"], x["k"], x["v"], x["g"], x["dout"], saved=f["saved"], dstate_out=dstate_out, **kw)
    return f, b


def _oracle(inp, w, G=None, gate=ref.GATE_PER_DIM):
    y = {k_: to64(v_) for k_, v_ in inp.items() if v_ is not None}
    return ref.lizard_backward(y["q"], y["k"], y["v"], y["g"], y["dout"], window=w.window, tau=w.gate_temp,
                               fmap_wq=y["fmap_wq"], fmap_wk=y["fmap_wk"], meta_k=y.get("meta_k"),
                               meta_v=y.get("meta_v"), alpha=y.get("alpha"), state_in=y.get("state_in"),
                               dstate_out=None if G is None else to64(G), gate=gate)


CASES = [
    # B, H, L, window, M, gate, state_in, incoming final-state gradient
    (2, 2, 260, 128, 4, "dim", True, False),     # ragged last tile
    (2, 2, 129, 33, 16, "dim", False, True),     # a one-token last tile
    (2, 2, 300, 128, 4, "scalar", True, True),
    (1, 2, 1300, 128, 4, "dim", True, False),    # few sequences: the forward splits them into segments
]


@pytest.mark.parametrize("B,H,L,window,M,gate,with_state,with_g", CASES)
def test_saved_backward_matches_the_oracle(lz, B, H, L, window, M, gate, with_state, with_g):
    w = Workload("saved", B=B, H=H, L=L, d=128, window=window, M=M, dtype="bf16", seed=40 + L,
                 kind="train", gate=gate)
    inp = make_inputs(w)
    inp["alpha"] = random_alpha(H, seed=L)
    if with_state:
        inp["state_in"] = torch.randn(B, H, 128, 128, generator=torch.Generator().manual_seed(3)) * 0.1
    G = torch.randn(B, H, 128, 128, generator=torch.Generator().manual_seed(6)) if with_g else None
    x = to_device(inp)
    f, got = _train(lz, x, w, lz.IMPL_AUTO, None if G is None else G.cuda())
    assert lz.workspace_status(got["workspace"]) == lz.OK
    fw = oracle_forward(inp, window=w.window, tau=w.gate_temp)
    for name in ("o", "state_out", "lse"):
        check(f"{name} (training forward)", f[name], fw[name], "bf16")
    want = _oracle(inp, w, G, ref.GATE_SCALAR if gate == "scalar" else ref.GATE_PER_DIM)
    for name in GRADS:
        check(f"{name} (saved)", got[name], want[name], "bf16")


def test_saved_backward_gla_branch_alone(lz):
    """The GLA branch alone keeps no softmax normalisers; its saved backward
    still matches the oracle."""
    w = Workload("saved_gla", B=1, H=2, L=200, d=128, window=10, M=4, dtype="bf16", seed=5, kind="train")
    inp = make_inputs(w)
    inp["alpha"] = random_alpha(2, seed=1)
    _, got = _train(lz, to_device(inp), w, lz.IMPL_TC, branch=lz.BRANCH_GLA_ONLY)
    want = oracle_backward(inp, window=w.window, tau=w.gate_temp, branch=ref.BRANCH_GLA_ONLY)
    for name in GRADS:
        check(f"{name} (saved, GLA branch)", got[name], want[name], "bf16")


def test_saved_forward_outputs_and_backward_as_close_as_plain(lz):
    """The training forward writes the same lse and final state as the plain
    forward, bit for bit; its o differs by rounding only (its inter-tile
    product reads S' as the bf16 copy of S' - 1 S'[0] plus the fp32 rank-one
    part, the plain forward the bf16 copy of S'), so both o are compared with
    the oracle, as are the two backwards (the saved one's S' comes from bf16
    decay factors, the recomputing state pass's from fp32 ones): each saved
    error stays within twice the plain one's (and within the bar)."""
    w = Workload("saved_eq", B=2, H=3, L=700, d=128, window=128, M=4, dtype="bf16", seed=77, kind="train")
    inp = make_inputs(w)
    x = to_device(inp)
    kw = _kw(x, w, lz.IMPL_TC)
    plain = lz.attn_fwd(x["q"], x["k"], x["v"], x["g"], want_state=True, want_lse=True, **kw)
    f, b_saved = _train(lz, x, w, lz.IMPL_TC)
    assert torch.equal(plain["lse"], f["lse"])
    assert torch.equal(plain["state_out"], f["state_out"])
    ref_o = oracle_forward(inp, window=w.window, tau=w.gate_temp)["o"]
    e_saved = check("o (saved)", f["o"], ref_o, "bf16")
    e_plain = check("o (plain)", plain["o"], ref_o, "bf16")
    assert e_saved <= 2.0 * e_plain + 1e-7, f"o: saved {e_saved:.3e} vs plain {e_plain:.3e}"
    b_plain = lz.attn_bwd(x["q"], x["k"], x["v"], x["g"], x["dout"], **kw)
    want = oracle_backward(inp, window=w.window, tau=w.gate_temp)
    for name in GRADS:
        e_saved = check(f"{name} (saved)", b_saved[name], want[name], "bf16")
        e_plain = check(f"{name} (recomputed)", b_plain[name], want[name], "bf16")
        assert e_saved <= 2.0 * e_plain + 1e-7, f"{name}: saved {e_saved:.3e} vs recomputed {e_plain:.3e}"


@pytest.mark.parametrize("gate", ["dim", "scalar"])
def test_saved_backward_computes_wide_decay_exactly(lz, gate):
    """Wide in-tile decay: the forward's gate prep marks the sequences in the
    saved buffer, the backward's exact fallback takes them from there."""
    w = Workload("saved_range", B=2, H=2, L=300, d=128, window=128, M=4, dtype="bf16", seed=9,
                 kind="train", gate=gate)
    inp = make_inputs(w)
    g = inp["g"].clone()
    if gate == "dim":
        g[0, 1, 130:200, :3] = -300.0
        g[1, 0, 20:21, :] = -2000.0
    else:
        g[0, 1, 130:200] = -300.0
        g[1, 0, 20:21] = -2000.0
    inp["g"] = g
    inp["state_in"] = torch.randn(2, 2, 128, 128, generator=torch.Generator().manual_seed(4)) * 0.1
    G = torch.randn(2, 2, 128, 128, generator=torch.Generator().manual_seed(5))
    _, got = _train(lz, to_device(inp), w, lz.IMPL_AUTO, G.cuda())
    assert lz.workspace_status(got["workspace"]) == lz.OK
    want = _oracle(inp, w, G, ref.GATE_SCALAR if gate == "scalar" else ref.GATE_PER_DIM)
    for name in GRADS:
        check(f"{name} (saved, {gate} gate)", got[name], want[name], "bf16")


def test_saved_train_step_full_size_sampled_heads(lz):
    """The training-step workload (B=8, H=32, L=2048) as the benchmark runs it
    with the saved buffer; sampled per-sequence gradients vs the oracle."""
    w = WORKLOADS["train_step"]
    inp = make_inputs(w)
    f, got = _train(lz, to_device(inp), w, lz.IMPL_AUTO)
    torch.cuda.synchronize()
    assert lz.workspace_status(got["workspace"]) == lz.OK
    for name in ("dq", "dk", "dv", "dg", "dalpha", "dfmap_wq", "dmeta_k"):
        assert torch.isfinite(got[name]).all(), name
    pairs = [(0, 0), (5, 30)]
    fw = oracle_forward(inp, window=w.window, tau=w.gate_temp, pairs=pairs)
    for (b, h), r in fw.items():
        check(f"o[{b},{h}] (training forward)", f["o"][b:b + 1, h:h + 1], r["o"], "bf16")
    want = oracle_backward(inp, window=w.window, tau=w.gate_temp, pairs=pairs)
    for (b, h), r in want.items():
        for name in ("dq", "dk", "dv", "dg", "dstate_in"):
            check(f"{name}[{b},{h}] (saved)", got[name][b:b + 1, h:h + 1], r[name], "bf16")


def test_saved_parameter_grads_full_length_every_sequence(lz):
    """Per-head parameter gradients at full length and batch (B=8, L=2048,
    two heads) through the saved buffer, over every (b, h)."""
    w = Workload("saved_params", B=8, H=2, L=2048, d=128, dtype="bf16", seed=18, kind="train")
    inp = make_inputs(w)
    _, got = _train(lz, to_device(inp), w, lz.IMPL_TC)
    want = oracle_backward(inp, window=w.window, tau=w.gate_temp)
    for name in ("dmeta_k", "dmeta_v", "dfmap_wq", "dfmap_wk", "dalpha", "dg", "dq", "dk", "dv",
                 "dstate_in"):
        check(f"{name} (saved)", got[name], want[name], "bf16")


def test_saved_plan_and_sizes(lz):
    """With the saved buffer the backward launches neither the gate pass nor
    the state-copy pass; a buffer one byte short is refused by both calls."""
    w = Workload("saved_plan", B=1, H=2, L=256, d=128, dtype="bf16", seed=1, kind="train")
    x = to_device(make_inputs(w))
    kw = _kw(x, w, lz.IMPL_AUTO)
    f = lz.attn_fwd(x["q"], x["k"], x["v"], x["g"], saved=True, **kw)
    names = lz.attn_bwd(x["q"], x["k"], x["v"], x["g"], x["dout"], saved=f["saved"], plan_only=True, **kw)
    assert "gate_prep_kernel" not in names and "tc_fwd_kernel(state copies)" not in names
    full = lz.attn_bwd(x["q"], x["k"], x["v"], x["g"], x["dout"], plan_only=True, **kw)
    assert "gate_prep_kernel" in full and "tc_fwd_kernel(state copies)" in full
    short = f["saved"][:-1]
    with pytest.raises(lz.LizardError):
        lz.attn_fwd(x["q"], x["k"], x["v"], x["g"], saved=short, **kw)
    with pytest.raises(lz.LizardError):
        lz.attn_bwd(x["q"], x["k"], x["v"], x["g"], x["dout"], saved=short, **kw)
