"""GPU parity of lizard_attn_bwd against the oracle's hand-derived backward
(itself pinned by central differences and autograd on the CPU)."""

import pytest
import torch

from gated_linear_sliding_chunkwise_b200.synth import WORKLOADS, Workload, make_inputs, random_alpha
from lizard_testutil import check, oracle_backward, to64, to_device
from oracle import lizard_ref as ref

pytestmark = pytest.mark.gpu

GRADS = ["dq", "dk", "dv", "dg", "dmeta_k", "dmeta_v", "dfmap_wq", "dfmap_wk", "dalpha",
         "dstate_in"]
IMPLS = ["simt", "tc"]


def _skip_unsupported(impl, dtype, d, window, M):
    """The tensor-core backward kernels cover bf16, d = 128, window <= 128, M <= 16."""
    if impl == "tc" and not (dtype == "bf16" and d == 128 and window <= 128 and M <= 16):
        pytest.skip("shape outside the tensor-core backward")


@pytest.fixture(scope="module")
def lz():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from gated_linear_sliding_chunkwise_b200 import lizard
    return lizard


def _impl(lz, name):
    return {"simt": lz.IMPL_SIMT, "tc": lz.IMPL_TC, "auto": lz.IMPL_AUTO}[name]


def _run(lz, x, w, impl, **kw):
    return lz.attn_bwd(x["q"], x["k"], x["v"], x["g"], x["dout"], window=w.window,
                       chunk=w.chunk, gate_temp=w.gate_temp, fmap_wq=x.get("fmap_wq"),
                       fmap_wk=x.get("fmap_wk"), meta_k=x.get("meta_k"),
                       meta_v=x.get("meta_v"), alpha=x.get("alpha"),
                       state_in=x.get("state_in"), impl=impl, **kw)


def _grad_dtype(name, act_dtype):
    # dq, dk, dv are stored in the activation dtype; the rest in fp32 but
    # computed from bf16-rounded inputs, so they take the same bar.
    return act_dtype


SWEEP = [
    # dtype, d, L, window, M, meta_v, state_in, random alpha
    ("fp32", 64, 1, 4, 2, True, True, False),
    ("fp32", 64, 97, 16, 4, True, True, True),
    ("fp32", 128, 70, 100, 4, False, False, True),
    ("fp32", 64, 150, 1, 0, False, True, False),
    ("bf16", 128, 260, 128, 4, True, True, True),
    ("bf16", 64, 129, 33, 16, True, False, True),
    # the tensor-core dq pass's meta-token gradients past eight meta tokens
    # (a second fragment of meta columns), with and without meta values
    ("bf16", 128, 300, 100, 16, True, False, True),
    ("bf16", 128, 200, 128, 9, False, True, False),
    ("bf16", 128, 150, 64, 2, True, True, False),
]


@pytest.mark.parametrize("impl", IMPLS)
@pytest.mark.parametrize("dtype,d,L,window,M,with_mv,with_state,rand_alpha", SWEEP)
def test_backward_sweep(lz, impl, dtype, d, L, window, M, with_mv, with_state, rand_alpha):
    _skip_unsupported(impl, dtype, d, window, M)
    w = Workload("bsweep", B=2, H=2, L=L, d=d, window=window, M=M, dtype=dtype,
                 seed=100 + L, kind="train")
    inp = make_inputs(w)
    if not with_mv:
        inp["meta_v"] = None
    if M == 0:
        inp["meta_k"] = inp["meta_v"] = None
    if with_state:
        inp["state_in"] = torch.randn(2, 2, d, d, generator=torch.Generator().manual_seed(8)) * 0.1
    if rand_alpha:
        inp["alpha"] = random_alpha(2, seed=L)
    got = _run(lz, to_device(inp), w, _impl(lz, impl))
    want = oracle_backward(inp, window=window, tau=w.gate_temp)
    for name in GRADS:
        if want[name] is None:
            assert got[name] is None
            continue
        check(name, got[name], want[name], _grad_dtype(name, dtype))


@pytest.mark.parametrize("impl", IMPLS)
@pytest.mark.parametrize("branch", [ref.BRANCH_GLA_ONLY, ref.BRANCH_SWA_ONLY])
def test_backward_branch_hooks(lz, impl, branch):
    dtype, d = ("fp32", 64) if impl == "simt" else ("bf16", 128)
    w = Workload("bbranch", B=1, H=2, L=90, d=d, window=10, M=4, dtype=dtype, seed=5,
                 kind="train")
    inp = make_inputs(w)
    inp["alpha"] = random_alpha(2, seed=1)
    got = _run(lz, to_device(inp), w, _impl(lz, impl), branch=branch)
    want = oracle_backward(inp, window=w.window, tau=w.gate_temp, branch=branch)
    for name in GRADS:
        check(name, got[name], want[name], dtype)


@pytest.mark.parametrize("impl", IMPLS)
def test_backward_alpha_zero_and_sink_only(lz, impl):
    """alpha = 0 on one head (the anchor branch still has a gradient for
    alpha) and sink-only meta tokens (no meta values)."""
    dtype, d = ("fp32", 64) if impl == "simt" else ("bf16", 128)
    w = Workload("balpha", B=2, H=2, L=200, d=d, window=64, M=4, dtype=dtype, seed=41,
                 kind="train")
    inp = make_inputs(w)
    inp["alpha"] = torch.tensor([0.0, 1.3])
    inp["meta_v"] = None
    got = _run(lz, to_device(inp), w, _impl(lz, impl))
    want = oracle_backward(inp, window=w.window, tau=w.gate_temp)
    for name in GRADS:
        if want[name] is None:
            assert got[name] is None
            continue
        check(name, got[name], want[name], dtype)


@pytest.mark.parametrize("impl", ["simt"])
def test_backward_extreme_decay(lz, impl):
    w = Workload("bextreme", B=1, H=2, L=100, d=64, window=6, M=2, dtype="fp32", seed=6,
                 kind="train")
    inp = make_inputs(w)
    g = inp["g"].clone()
    g[:, :, 5:40, :9] = -300.0
    inp["g"] = g
    got = _run(lz, to_device(inp), w, _impl(lz, impl))
    want = oracle_backward(inp, window=w.window, tau=w.gate_temp)
    for name in GRADS:
        check(name, got[name], want[name], "fp32")


@pytest.mark.parametrize("impl", ["tc", "auto"])
@pytest.mark.parametrize("gate", ["dim", "scalar"])
@pytest.mark.parametrize("with_g", [False, True])
def test_tc_backward_computes_wide_decay_exactly(lz, impl, gate, with_g):
    """The backward's exact fallback: sequences whose in-tile decay spread
    leaves the tensor-core range get their GLA gradients from the portable
    kernels (dphi, dv, dstate_in, da and dg), the rest of the call from the
    tensor-core kernels; every gradient matches the oracle, with and without
    an incoming final-state gradient."""
    w = Workload("brange", B=2, H=2, L=300, d=128, window=128, M=4, dtype="bf16", seed=9, kind="train",
                 gate=gate)
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
    G = torch.randn(2, 2, 128, 128, generator=torch.Generator().manual_seed(5)) if with_g else None
    got = _run(lz, to_device(inp), w, _impl(lz, impl), dstate_out=None if G is None else G.cuda())
    assert lz.workspace_status(got["workspace"]) == lz.OK
    y = {k_: to64(v_) for k_, v_ in inp.items() if v_ is not None}
    want = ref.lizard_backward(y["q"], y["k"], y["v"], y["g"], y["dout"], window=w.window, tau=w.gate_temp,
                               fmap_wq=y["fmap_wq"], fmap_wk=y["fmap_wk"], meta_k=y["meta_k"],
                               meta_v=y["meta_v"], alpha=y["alpha"], state_in=y["state_in"],
                               dstate_out=None if G is None else to64(G),
                               gate=ref.GATE_SCALAR if gate == "scalar" else ref.GATE_PER_DIM)
    for name in GRADS:
        check(f"{name} ({gate} gate)", got[name], want[name], "bf16")


def test_tc_backward_flags_wide_decay_beyond_its_fallback_slots(lz):
    """More sequences with wide decay in one backward call than its exact
    fallback has slots (four): the status word says RANGE; a call without
    such gates reads OK again."""
    w = Workload("brange_many", B=3, H=2, L=256, d=128, window=128, M=4, dtype="bf16", seed=2, kind="train")
    inp = make_inputs(w)
    g = inp["g"].clone()
    g[:, :, 130:200, :3] = -300.0
    inp["g"] = g
    got = _run(lz, to_device(inp), w, lz.IMPL_TC)
    assert lz.workspace_status(got["workspace"]) == lz.ERR_RANGE
    ok = _run(lz, to_device(make_inputs(w)), w, lz.IMPL_TC)
    assert lz.workspace_status(ok["workspace"]) == lz.OK


@pytest.mark.parametrize("impl", IMPLS)
def test_parameter_grads_bf16_full_reduction(lz, impl):
    """Gradients of the per-head parameters reduce over batch and tokens:
    check them against the oracle over every (b, h) of a mid-size case."""
    w = Workload("params", B=2, H=2, L=512, d=128, dtype="bf16", seed=13, kind="train")
    inp = make_inputs(w)
    got = _run(lz, to_device(inp), w, _impl(lz, impl))
    want = oracle_backward(inp, window=w.window, tau=w.gate_temp)
    for name in GRADS:
        check(name, got[name], want[name], "bf16")


@pytest.mark.parametrize("impl", IMPLS)
def test_train_step_full_size_sampled_heads(lz, impl):
    """The full training-step workload (B=8, H=32, L=2048) as the benchmark
    launches it; per-sequence gradients of sampled (b, h) pairs vs the oracle."""
    w = WORKLOADS["train_step"]
    inp = make_inputs(w)
    got = _run(lz, to_device(inp), w, _impl(lz, impl))
    torch.cuda.synchronize()
    for name in ("dq", "dk", "dv", "dg", "dalpha", "dfmap_wq", "dmeta_k"):
        assert torch.isfinite(got[name]).all(), name
    pairs = [(0, 0), (7, 21)]
    want = oracle_backward(inp, window=w.window, tau=w.gate_temp, pairs=pairs)
    for (b, h), r in want.items():
        for name in ("dq", "dk", "dv", "dg", "dstate_in"):
            check(f"{name}[{b},{h}]", got[name][b:b + 1, h:h + 1], r[name], "bf16")


@pytest.mark.parametrize("gate", ["dim", "scalar"])
def test_parameter_grads_full_length_every_sequence(lz, gate):
    """The per-head parameter gradients at the training step's full length and
    batch (B=8, L=2048, d=128; two heads keep the oracle to seconds): they sum
    fp32 atomics over 8 x 2048 tokens, so they are compared with the oracle
    over every (b, h), with the per-token gradients, on the tensor-core path."""
    w = Workload("params_full", B=8, H=2, L=2048, d=128, dtype="bf16", seed=17, kind="train",
                 gate=gate)
    inp = make_inputs(w)
    got = _run(lz, to_device(inp), w, lz.IMPL_TC)
    assert lz.workspace_status(got["workspace"]) == lz.OK
    want = oracle_backward(inp, window=w.window, tau=w.gate_temp)
    for name in ("dmeta_k", "dmeta_v", "dfmap_wq", "dfmap_wk", "dalpha", "dg", "dq", "dk", "dv",
                 "dstate_in"):
        check(f"{name} ({gate} gate)", got[name], want[name], "bf16")


def test_persistent_kernels_walk_ragged_tiles_across_sequences(lz):
    """256 sequences of a ragged length (three 128-token tiles, the last one
    44 tokens): the persistent backward kernels give every CTA a run of
    tiles or key blocks that crosses sequence boundaries; sampled sequences
    at the start, middle and end of the runs against the oracle."""
    w = Workload("ragged_many", B=8, H=32, L=300, d=128, window=128, M=4, dtype="bf16", seed=31,
                 kind="train")
    inp = make_inputs(w)
    got = _run(lz, to_device(inp), w, lz.IMPL_TC)
    torch.cuda.synchronize()
    pairs = [(0, 0), (3, 17), (7, 31)]
    want = oracle_backward(inp, window=w.window, tau=w.gate_temp, pairs=pairs)
    for (b, h), r in want.items():
        for name in ("dq", "dk", "dv", "dg", "dstate_in"):
            check(f"{name}[{b},{h}]", got[name][b:b + 1, h:h + 1], r[name], "bf16")


DSTATE_CASES = [
    # impl, dtype, d, L, window, M
    ("simt", "fp32", 64, 97, 16, 4),
    ("tc", "bf16", 128, 300, 128, 4),
]


@pytest.mark.parametrize("impl,dtype,d,L,window,M", DSTATE_CASES)
def test_backward_with_incoming_state_gradient(lz, impl, dtype, d, L, window, M):
    """dstate_out: the gradients of sum(dout * o) + sum(G * state_out)."""
    w = Workload("dstate", B=2, H=2, L=L, d=d, window=window, M=M, dtype=dtype, seed=700 + L,
                 kind="train")
    inp = make_inputs(w)
    inp["state_in"] = torch.randn(2, 2, d, d, generator=torch.Generator().manual_seed(9)) * 0.1
    G = torch.randn(2, 2, d, d, generator=torch.Generator().manual_seed(10))
    x = to_device(inp)
    got = _run(lz, x, w, _impl(lz, impl), dstate_out=G.cuda())
    assert lz.workspace_status(got["workspace"]) == lz.OK
    y = {k_: to64(v_) for k_, v_ in inp.items() if v_ is not None}
    want = ref.lizard_backward(y["q"], y["k"], y["v"], y["g"], y["dout"], window=window, tau=w.gate_temp,
                               fmap_wq=y["fmap_wq"], fmap_wk=y["fmap_wk"], meta_k=y["meta_k"],
                               meta_v=y["meta_v"], alpha=y["alpha"], state_in=y["state_in"],
                               dstate_out=to64(G))
    for name in GRADS:
        check(name, got[name], want[name], dtype)


@pytest.mark.parametrize("impl", IMPLS)
def test_chunks_chained_through_states_give_the_whole_backward(lz, impl):
    """A sequence trained in two chunks (the GLA branch, which carries all of
    the history in its state): forward of chunk 1 gives chunk 2 its
    state_in; backward of chunk 2 gives chunk 1 its dstate_out."""
    dtype, d = ("fp32", 64) if impl == "simt" else ("bf16", 128)
    L, cut = 400, 256
    w = Workload("chunks", B=2, H=2, L=L, d=d, window=64, M=0, dtype=dtype, seed=77, kind="train")
    inp = make_inputs(w)
    inp["meta_k"] = inp["meta_v"] = None
    x = to_device(inp)
    kw = dict(window=w.window, gate_temp=w.gate_temp, fmap_wq=x["fmap_wq"], fmap_wk=x["fmap_wk"],
              branch=lz.BRANCH_GLA_ONLY, impl=_impl(lz, impl))
    part = lambda a, b: {k_: x[k_][:, :, a:b].contiguous() for k_ in ("q", "k", "v", "g", "dout")}
    c1, c2 = part(0, cut), part(cut, L)
    S_cut = lz.attn_fwd(c1["q"], c1["k"], c1["v"], c1["g"], want_state=True, **kw)["state_out"]
    b2 = lz.attn_bwd(c2["q"], c2["k"], c2["v"], c2["g"], c2["dout"], state_in=S_cut, **kw)
    b1 = lz.attn_bwd(c1["q"], c1["k"], c1["v"], c1["g"], c1["dout"], dstate_out=b2["dstate_in"], **kw)
    torch.cuda.synchronize()
    want = oracle_backward(inp, window=w.window, tau=w.gate_temp, branch=ref.BRANCH_GLA_ONLY)
    for name in ("dq", "dk", "dv", "dg"):
        check(name, torch.cat([b1[name], b2[name]], dim=2), want[name], dtype)
    check("dstate_in", b1["dstate_in"], want["dstate_in"], dtype)
    for name in ("dfmap_wq", "dfmap_wk"):
        check(name, b1[name] + b2[name], want[name], dtype)


@pytest.mark.parametrize("case", ["swa_portable", "no_fmap_weights"])
def test_backward_mixed_paths(lz, case):
    """bf16, d = 128 combinations outside the fused tensor-core configuration:
    a window above 128 (tensor-core GLA backward, portable anchor backward,
    the tensor-core finish summing fp32 parts) and no feature-map weights
    (identity map: tensor-core GLA backward, portable finish)."""
    window = 200 if case == "swa_portable" else 64
    w = Workload("bmixed", B=1, H=2, L=300, d=128, window=window, M=4, dtype="bf16", seed=61,
                 kind="train")
    inp = make_inputs(w)
    inp["alpha"] = random_alpha(2, seed=5)
    if case == "no_fmap_weights":
        inp["fmap_wq"] = inp["fmap_wk"] = None
    got = _run(lz, to_device(inp), w, lz.IMPL_AUTO)
    want = oracle_backward(inp, window=w.window, tau=w.gate_temp)
    for name in GRADS:
        if want[name] is None:
            assert got[name] is None
            continue
        check(name, got[name], want[name], "bf16")


def test_side_by_side_backward_matches_in_order_run(lz):
    """The backward lets independent kernels run side by side on a second
    stream; with per-kernel timing events everything runs in order.  Both give
    the same gradients (bit for bit where no atomics are involved), and a
    CUDA-graph capture of the call replays to the same result."""
    w = Workload("lanes", B=2, H=4, L=640, d=128, dtype="bf16", seed=29, kind="train")
    inp = make_inputs(w)
    x = to_device(inp)
    a = _run(lz, x, w, lz.IMPL_AUTO)
    names = _run(lz, x, w, lz.IMPL_AUTO, plan_only=True)
    b = _run(lz, x, w, lz.IMPL_AUTO, events=lz.make_events(len(names) + 1))
    torch.cuda.synchronize()
    for name in ("dq", "dk", "dv", "dg", "dstate_in"):
        assert torch.equal(a[name], b[name]), name
    for name in ("dmeta_k", "dmeta_v", "dfmap_wq", "dfmap_wk", "dalpha"):
        # sums of fp32 atomics: their order varies from run to run
        err = float((a[name] - b[name]).abs().max())
        assert err <= 1e-4 * float(b[name].abs().max()), (name, err)
    # graph capture (the side stream exists by now)
    ws = a["workspace"]
    outs = {}
    g = torch.cuda.CUDAGraph()
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        with torch.cuda.graph(g, stream=stream):
            outs = _run(lz, x, w, lz.IMPL_AUTO, workspace=ws, stream=stream)
    g.replay()
    torch.cuda.synchronize()
    for name in ("dq", "dk", "dv", "dg"):
        assert torch.equal(outs[name], a[name]), name
