"""GPU parity of lizard_attn_fwd against the fp64 oracle (through the C ABI)."""

import numpy as np
import pytest
import torch

from gated_linear_sliding_chunkwise_b200.synth import WORKLOADS, Workload, make_inputs, random_alpha
from lizard_testutil import check, oracle_forward, to_device, to64
from oracle import lizard_ref as ref

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lz():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from gated_linear_sliding_chunkwise_b200 import lizard
    return lizard


def _run(lz, x, w, impl, **kw):
    return lz.attn_fwd(x["q"], x["k"], x["v"], x["g"], window=w.window, chunk=w.chunk,
                       gate_temp=w.gate_temp, fmap_wq=x.get("fmap_wq"), fmap_wk=x.get("fmap_wk"),
                       meta_k=x.get("meta_k"), meta_v=x.get("meta_v"), alpha=x.get("alpha"),
                       state_in=x.get("state_in"), impl=impl, **kw)


IMPLS = ["simt", "tc"]


def test_a_wait_that_runs_out_is_reported_and_the_context_stays_usable(lz):
    """Failure detection without a fault: the test hook makes the forward's
    first wait run out; the call reports LIZARD_ERR_TIMEOUT through the
    workspace status, and the next call on the same context computes."""
    w = Workload("inject", B=1, H=2, L=256, d=128, window=128, M=4, dtype="bf16", seed=5)
    inp = make_inputs(w)
    x = to_device(inp)
    lz.debug_inject_wait_timeout(1)
    try:
        got = _run(lz, x, w, lz.IMPL_TC)
        assert lz.workspace_status(got["workspace"]) == lz.ERR_TIMEOUT
    finally:
        lz.debug_inject_wait_timeout(0)
    got = _run(lz, x, w, lz.IMPL_TC)
    assert lz.workspace_status(got["workspace"]) == lz.OK
    check("o", got["o"], oracle_forward(inp, window=w.window, tau=w.gate_temp)["o"], "bf16")


def _impl(lz, name):
    return {"simt": lz.IMPL_SIMT, "tc": lz.IMPL_TC, "auto": lz.IMPL_AUTO}[name]


def _skip_unsupported(impl, dtype, d, window, M):
    """The tensor-core forward covers bf16, d = 128, window <= 128, M <= 16."""
    if impl == "tc" and not (dtype == "bf16" and d == 128 and window <= 128 and M <= 16):
        pytest.skip("shape outside the tensor-core forward")


@pytest.mark.parametrize("impl", IMPLS)
def test_tiny_fp32_full(lz, impl):
    """The tiny fp32 workload, every output, max abs error <= 1e-4."""
    w = WORKLOADS["tiny_fp32"]
    _skip_unsupported(impl, w.dtype, w.d, w.window, w.M)
    inp = make_inputs(w)
    x = to_device(inp)
    got = _run(lz, x, w, _impl(lz, impl), want_state=True, want_lse=True)
    want = oracle_forward(inp, window=w.window, tau=w.gate_temp)
    check("o", got["o"], want["o"], "fp32")
    check("state_out", got["state_out"], want["state_out"], "fp32")
    check("lse", got["lse"], want["lse"], "fp32")


SWEEP = [
    # dtype, d, L, window, M, meta_v, state_in, random alpha
    ("fp32", 64, 1, 16, 4, True, False, False),
    ("fp32", 64, 63, 16, 4, True, True, True),
    ("fp32", 128, 130, 100, 0, False, True, True),
    ("fp32", 64, 200, 300, 4, False, False, True),
    ("fp32", 128, 129, 1, 2, True, False, False),
    ("bf16", 128, 200, 128, 4, True, True, True),
    ("bf16", 64, 333, 37, 16, True, False, True),
    ("bf16", 128, 65, 64, 0, False, False, False),
]


@pytest.mark.parametrize("impl", IMPLS)
@pytest.mark.parametrize("dtype,d,L,window,M,with_mv,with_state,rand_alpha", SWEEP)
def test_forward_sweep(lz, impl, dtype, d, L, window, M, with_mv, with_state, rand_alpha):
    """Ragged lengths, windows shorter/longer than a chunk, with and without
    meta tokens, sink-only meta tokens, an initial state and random alpha."""
    _skip_unsupported(impl, dtype, d, window, M)
    w = Workload("sweep", B=2, H=3, L=L, d=d, window=window, M=M, dtype=dtype, seed=11 + L)
    inp = make_inputs(w)
    if not with_mv:
        inp["meta_v"] = None
    if M == 0:
        inp["meta_k"] = inp["meta_v"] = None
    if with_state:
        inp["state_in"] = torch.randn(2, 3, d, d, generator=torch.Generator().manual_seed(5)) * 0.1
    if rand_alpha:
        inp["alpha"] = random_alpha(3, seed=L)
    got = _run(lz, to_device(inp), w, _impl(lz, impl), want_state=True, want_lse=True)
    assert lz.workspace_status(got["workspace"]) == lz.OK
    want = oracle_forward(inp, window=window, tau=w.gate_temp)
    check("o", got["o"], want["o"], dtype)
    check("state_out", got["state_out"], want["state_out"], "fp32" if dtype == "fp32" else dtype)
    check("lse", got["lse"], want["lse"], "fp32" if dtype == "fp32" else dtype)


@pytest.mark.parametrize("impl", IMPLS)
@pytest.mark.parametrize("L", [150, 1100])          # 1100: few sequences, segmented forward
@pytest.mark.parametrize("branch", [ref.BRANCH_GLA_ONLY, ref.BRANCH_SWA_ONLY])
def test_branch_hooks(lz, impl, branch, L):
    dtype, d = ("fp32", 64) if impl == "simt" else ("bf16", 128)
    w = Workload("branch", B=1, H=2, L=L, d=d, window=20, M=4, dtype=dtype, seed=3)
    inp = make_inputs(w)
    inp["alpha"] = random_alpha(2, seed=9)
    got = _run(lz, to_device(inp), w, _impl(lz, impl), branch=branch)
    want = oracle_forward(inp, window=w.window, tau=w.gate_temp, branch=branch)
    check("o", got["o"], want["o"], dtype)


@pytest.mark.parametrize("impl", IMPLS)
def test_alpha_zero_drops_anchor_branch(lz, impl):
    dtype, d = ("fp32", 64) if impl == "simt" else ("bf16", 128)
    w = Workload("alpha0", B=1, H=2, L=200, d=d, window=64, M=4, dtype=dtype, seed=31)
    inp = make_inputs(w)
    inp["alpha"] = torch.tensor([0.0, 0.7])
    got = _run(lz, to_device(inp), w, _impl(lz, impl))
    want = oracle_forward(inp, window=w.window, tau=w.gate_temp)
    check("o", got["o"], want["o"], dtype)


def _wide_decay(inp, heads):
    """Gate logits of -300 over part of a tile (log-decay -18.75 per token on
    a few key dimensions) and one token of -2000 (it wipes the state): the
    in-tile spread leaves the tensor-core absorption's range."""
    g = inp["g"].clone()
    scalar = g.dim() == inp["q"].dim() - 1
    for b, h in heads:
        if scalar:
            g[b, h, 130:200] = -300.0
            g[b, h, 20:21] = -2000.0
        else:
            g[b, h, 130:200, :3] = -300.0
            g[b, h, 20:21, :] = -2000.0
    inp["g"] = g
    return inp


@pytest.mark.parametrize("impl", ["tc", "auto"])
@pytest.mark.parametrize("gate", ["dim", "scalar"])
def test_tc_path_computes_wide_decay_exactly(lz, impl, gate):
    """Sequences whose in-tile decay spread leaves the tensor-core range get
    their GLA branch from the exact token-by-token recurrence inside the
    forward kernel: the output, final state and normaliser match the oracle,
    the status is OK, and the other sequences of the call stay on the tensor
    cores."""
    w = Workload("range", B=2, H=3, L=300, d=128, window=128, M=4, dtype="bf16", seed=2, gate=gate)
    inp = _wide_decay(make_inputs(w), [(0, 1), (1, 2)])
    inp["state_in"] = torch.randn(2, 3, 128, 128, generator=torch.Generator().manual_seed(3)) * 0.1
    got = _run(lz, to_device(inp), w, _impl(lz, impl), want_state=True, want_lse=True)
    assert lz.workspace_status(got["workspace"]) == lz.OK
    want = oracle_forward(inp, window=w.window, tau=w.gate_temp)
    for name in ("o", "state_out", "lse"):
        check(name, got[name], want[name], "bf16")


def test_tc_wide_decay_in_a_segmented_forward(lz):
    """Few sequences and a long one (the forward splits sequences into
    segments with a state pass): a marked sequence's GLA branch still comes
    whole from the exact fallback."""
    w = Workload("range_seg", B=1, H=2, L=1100, d=128, window=128, M=4, dtype="bf16", seed=5)
    inp = _wide_decay(make_inputs(w), [(0, 0)])
    got = _run(lz, to_device(inp), w, lz.IMPL_TC, want_state=True)
    assert lz.workspace_status(got["workspace"]) == lz.OK
    want = oracle_forward(inp, window=w.window, tau=w.gate_temp)
    check("o", got["o"], want["o"], "bf16")
    check("state_out", got["state_out"], want["state_out"], "bf16")


@pytest.mark.parametrize("branch", [ref.BRANCH_BOTH, ref.BRANCH_GLA_ONLY])
def test_tc_forward_computes_every_marked_sequence_exactly(lz, branch):
    """Every sequence of a call marked for wide decay (the forward has no
    limit on how many): all of them match the oracle, also with the anchor
    branch off (the exact recurrence then writes o rather than adds to it)."""
    w = Workload("range_many", B=3, H=2, L=256, d=128, window=128, M=4, dtype="bf16", seed=2)
    inp = _wide_decay(make_inputs(w), [(b, h) for b in range(3) for h in range(2)])
    got = _run(lz, to_device(inp), w, lz.IMPL_TC, want_state=True, branch=branch)
    assert lz.workspace_status(got["workspace"]) == lz.OK
    want = oracle_forward(inp, window=w.window, tau=w.gate_temp, branch=branch)
    check("o", got["o"], want["o"], "bf16")
    check("state_out", got["state_out"], want["state_out"], "bf16")


@pytest.mark.parametrize("impl", ["simt"])
def test_extreme_decay_takes_exact_path(lz, impl):
    """Gate logits near -300 make the in-chunk decay spread exceed the
    log-space absorption's range; the result must still match."""
    w = Workload("extreme", B=1, H=2, L=160, d=64, window=8, M=0, dtype="fp32", seed=21)
    inp = make_inputs(w)
    inp["meta_k"] = inp["meta_v"] = None
    g = inp["g"].clone()
    g[:, :, 10:40, :7] = -300.0    # log-decay -18.75 per token on a few dims
    g[:, 1, 90:91, :] = -2000.0    # one token wipes the state of head 1
    inp["g"] = g
    got = _run(lz, to_device(inp), w, _impl(lz, impl), want_state=True)
    want = oracle_forward(inp, window=w.window, tau=w.gate_temp)
    check("o", got["o"], want["o"], "fp32")
    check("state_out", got["state_out"], want["state_out"], "fp32")


@pytest.mark.parametrize("impl", IMPLS)
def test_segmented_equals_one_shot(lz, impl):
    """state_out of one segment fed as state_in of the next reproduces the
    one-shot forward (prefill handed over in pieces)."""
    dtype = "fp32" if impl == "simt" else "bf16"
    w = Workload("seg", B=2, H=2, L=300, d=128, window=50, M=4, dtype=dtype, seed=4)
    inp = to_device(make_inputs(w))
    full = _run(lz, inp, w, _impl(lz, impl), want_state=True)
    cut = 137
    a = {k_: (v_[:, :, :cut].contiguous() if k_ in ("q", "k", "v", "g") else v_) for k_, v_ in inp.items()}
    b = {k_: (v_[:, :, cut:].contiguous() if k_ in ("q", "k", "v", "g") else v_) for k_, v_ in inp.items()}
    wa = Workload("seg", B=2, H=2, L=cut, d=128, window=50, M=4, dtype=dtype)
    r1 = _run(lz, a, wa, _impl(lz, impl), branch=ref.BRANCH_GLA_ONLY, want_state=True)
    b["state_in"] = r1["state_out"]
    r2 = _run(lz, b, wa, _impl(lz, impl), branch=ref.BRANCH_GLA_ONLY, want_state=True)
    gla = _run(lz, inp, w, _impl(lz, impl), branch=ref.BRANCH_GLA_ONLY, want_state=True)
    check("o", torch.cat([r1["o"], r2["o"]], 2), to64(gla["o"]), dtype)
    check("S", r2["state_out"], to64(full["state_out"]), dtype)


@pytest.mark.parametrize("L", [1000, 3000])
def test_tc_segmented_long_sequence(lz, L):
    """Few (batch, head) pairs and a long sequence: the tensor-core forward
    splits the sequence into segments (gate factors, state pass, combine,
    full pass)."""
    w = Workload("tcseg", B=1, H=2, L=L, d=128, window=128, M=4, dtype="bf16", seed=L)
    inp = make_inputs(w)
    inp["state_in"] = torch.randn(1, 2, 128, 128, generator=torch.Generator().manual_seed(3)) * 0.1
    inp["alpha"] = random_alpha(2, seed=L)
    x = to_device(inp)
    plan = lz.attn_fwd(x["q"], x["k"], x["v"], x["g"], window=w.window, gate_temp=w.gate_temp,
                       fmap_wq=x["fmap_wq"], fmap_wk=x["fmap_wk"], meta_k=x["meta_k"],
                       meta_v=x["meta_v"], alpha=x["alpha"], state_in=x["state_in"],
                       impl=lz.IMPL_TC, plan_only=True)
    assert plan == ["gate_prep_kernel", "tc_fwd_kernel(state pass)", "seg_combine_kernel",
                    "tc_fwd_kernel"], plan
    got = _run(lz, x, w, lz.IMPL_TC, want_state=True, want_lse=True)
    assert lz.workspace_status(got["workspace"]) == lz.OK
    want = oracle_forward(inp, window=w.window, tau=w.gate_temp)
    check("o", got["o"], want["o"], "bf16")
    check("state_out", got["state_out"], want["state_out"], "bf16")
    check("lse", got["lse"], want["lse"], "bf16")


def test_empty_sequence_passes_state_through(lz):
    w = Workload("empty", B=1, H=2, L=0, d=64, window=4, M=0, dtype="bf16")
    inp = make_inputs(w)
    inp["meta_k"] = inp["meta_v"] = None
    inp["state_in"] = torch.randn(1, 2, 64, 64)
    got = _run(lz, to_device(inp), w, lz.IMPL_AUTO, want_state=True)
    assert got["o"].numel() == 0
    assert torch.equal(got["state_out"].cpu(), inp["state_in"])


@pytest.mark.parametrize("impl", IMPLS)
@pytest.mark.parametrize("name,pairs", [
    ("llama8b_layer_fwd", [(0, 0), (1, 17), (3, 31)]),
    ("long_fwd_16k", [(0, 5), (0, 30)]),
])
def test_full_size_sampled_heads(lz, impl, name, pairs):
    """The full-size bf16 workloads in the benchmark's launch configuration;
    the oracle checks every output of a few sampled (batch, head) pairs."""
    w = WORKLOADS[name]
    inp = make_inputs(w)
    got = _run(lz, to_device(inp), w, _impl(lz, impl), want_state=True, want_lse=True)
    torch.cuda.synchronize()
    want = oracle_forward(inp, window=w.window, tau=w.gate_temp, pairs=pairs)
    assert torch.isfinite(got["o"]).all()
    for (b, h), r in want.items():
        check(f"o[{b},{h}]", got["o"][b:b + 1, h:h + 1], r["o"], "bf16")
        check(f"S[{b},{h}]", got["state_out"][b:b + 1, h:h + 1], r["state_out"], "bf16")
        check(f"lse[{b},{h}]", got["lse"][b:b + 1, h:h + 1], r["lse"], "bf16")


def test_identity_feature_map_at_tensor_core_shape(lz):
    """No feature-map weights (the identity map) at bf16, d = 128: the
    forward takes the portable GLA kernels and matches the oracle; forcing
    the tensor-core kernels is refused."""
    w = Workload("ident", B=1, H=2, L=300, d=128, window=64, M=4, dtype="bf16", seed=71)
    inp = make_inputs(w)
    inp["fmap_wq"] = inp["fmap_wk"] = None
    x = to_device(inp)
    got = _run(lz, x, w, lz.IMPL_AUTO, want_state=True)
    want = oracle_forward(inp, window=w.window, tau=w.gate_temp)
    check("o", got["o"], want["o"], "bf16")
    with pytest.raises(RuntimeError):
        _run(lz, x, w, lz.IMPL_TC)
