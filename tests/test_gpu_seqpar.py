"""GPU parity of the sequence-parallel pieces against the oracle, through
the C ABI: the forward and the backward with a key/value prefix, the segment
summary (U, R), the chain of summaries, and a sequence split into segments
run one after another on one GPU (each segment the work of one rank)
against the whole-sequence forward and backward."""

import os

import numpy as np
import pytest
import torch

from gated_linear_sliding_chunkwise_b200.synth import Workload, make_inputs, random_alpha
from lizard_testutil import check, gate_of, to64, to_device
from oracle import lizard_ref as ref

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lz():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from gated_linear_sliding_chunkwise_b200 import lizard
    return lizard


def _impl(lz, name):
    return {"simt": lz.IMPL_SIMT, "tc": lz.IMPL_TC, "auto": lz.IMPL_AUTO}[name]


def _params(x):
    return {k_: x.get(k_) for k_ in ("fmap_wq", "fmap_wk", "meta_k", "meta_v", "alpha")}


def _span(x, a, b):
    return {k_: x[k_][:, :, a:b].contiguous() for k_ in ("q", "k", "v", "g")}


def _whole(dtype, d, B, H, L, window, M, gate, seed):
    w = Workload("seqpar", B=B, H=H, L=L, d=d, window=window, M=M, dtype=dtype, seed=seed, gate=gate)
    inp = make_inputs(w)
    if M == 0:
        inp["meta_k"] = inp["meta_v"] = None
    inp["alpha"] = random_alpha(H, seed=L)
    return w, inp


PREFIX_CASES = [
    # impl, dtype, d, B, H, L, window, M, P, gate
    ("tc", "bf16", 128, 2, 2, 300, 128, 4, 128, "dim"),
    ("tc", "bf16", 128, 2, 2, 200, 64, 4, 37, "dim"),      # prefix shorter than the window
    ("tc", "bf16", 128, 1, 2, 1100, 128, 4, 128, "scalar"),  # few sequences: segmented forward
    ("tc", "bf16", 128, 2, 2, 60, 100, 0, 100, "dim"),     # shorter than one tile
    ("simt", "fp32", 64, 2, 2, 97, 16, 4, 16, "dim"),
    ("simt", "fp32", 64, 2, 3, 70, 30, 2, 7, "scalar"),
    ("simt", "bf16", 128, 1, 2, 130, 100, 4, 100, "dim"),
]


@pytest.mark.parametrize("impl,dtype,d,B,H,L,window,M,P,gate", PREFIX_CASES)
def test_forward_with_prefix_matches_oracle(lz, impl, dtype, d, B, H, L, window, M, P, gate):
    w, inp = _whole(dtype, d, B, H, P + L, window, M, gate, seed=600 + L)
    S_in = torch.randn(B, H, d, d, generator=torch.Generator().manual_seed(6)) * 0.1
    x = to_device(inp)
    t = _span(x, P, P + L)
    kp, vp = x["k"][:, :, :P].contiguous(), x["v"][:, :, :P].contiguous()
    got = lz.attn_fwd(t["q"], t["k"], t["v"], t["g"], window=window, gate_temp=w.gate_temp,
                      state_in=S_in.cuda(), want_state=True, want_lse=True, impl=_impl(lz, impl),
                      k_prefix=kp, v_prefix=vp, **_params(x))
    assert lz.workspace_status(got["workspace"]) == lz.OK
    y = {k_: to64(v_) for k_, v_ in inp.items() if v_ is not None}
    want = ref.lizard_forward(*(y[k_][:, :, P:] for k_ in ("q", "k", "v", "g")), window=window,
                              tau=w.gate_temp, state_in=to64(S_in), k_prefix=y["k"][:, :, :P],
                              v_prefix=y["v"][:, :, :P], gate=gate_of(y), **_params(y))
    for name in ("o", "state_out", "lse"):
        check(name, got[name], want[name], dtype)


BWD_GRADS = ("dq", "dk", "dv", "dg", "dmeta_k", "dmeta_v", "dfmap_wq", "dfmap_wk", "dalpha",
             "dstate_in", "dk_prefix", "dv_prefix")


@pytest.mark.parametrize("impl,dtype,d,B,H,L,window,M,P,gate", PREFIX_CASES)
def test_backward_with_prefix_matches_oracle(lz, impl, dtype, d, B, H, L, window, M, P, gate):
    """lizard_attn_bwd of a segment with a key/value prefix: every gradient,
    the prefix's own key and value gradients included, against the oracle."""
    w, inp = _whole(dtype, d, B, H, P + L, window, M, gate, seed=650 + L)
    S_in = torch.randn(B, H, d, d, generator=torch.Generator().manual_seed(7)) * 0.1
    dout = torch.randn(B, H, L, d, generator=torch.Generator().manual_seed(11)).to(inp["q"].dtype)
    x = to_device(inp)
    t = _span(x, P, P + L)
    kp, vp = x["k"][:, :, :P].contiguous(), x["v"][:, :, :P].contiguous()
    got = lz.attn_bwd(t["q"], t["k"], t["v"], t["g"], dout.cuda(), window=window, gate_temp=w.gate_temp,
                      state_in=S_in.cuda(), impl=_impl(lz, impl), k_prefix=kp, v_prefix=vp, **_params(x))
    assert lz.workspace_status(got["workspace"]) == lz.OK
    y = {k_: to64(v_) for k_, v_ in inp.items() if v_ is not None}
    want = ref.lizard_backward(*(y[k_][:, :, P:] for k_ in ("q", "k", "v", "g")), to64(dout), window=window,
                               tau=w.gate_temp, state_in=to64(S_in), k_prefix=y["k"][:, :, :P],
                               v_prefix=y["v"][:, :, :P], gate=gate_of(y), **_params(y))
    for name in BWD_GRADS:
        if want[name] is None:
            assert got[name] is None, name
            continue
        check(name, got[name], want[name], dtype)


SEG_CASES = [
    # impl, dtype, d, B, H, L, gate
    ("tc", "bf16", 128, 2, 2, 300, "dim"),
    ("tc", "bf16", 128, 1, 3, 1100, "scalar"),
    ("simt", "fp32", 64, 2, 2, 97, "dim"),
    ("simt", "bf16", 128, 1, 2, 130, "scalar"),
]


@pytest.mark.parametrize("impl,dtype,d,B,H,L,gate", SEG_CASES)
def test_segment_state_matches_oracle(lz, impl, dtype, d, B, H, L, gate):
    w, inp = _whole(dtype, d, B, H, L, 64, 0, gate, seed=700 + L)
    x = to_device(inp)
    U, R, ws = lz.segment_state(x["k"], x["v"], x["g"], window=64, gate_temp=w.gate_temp,
                                fmap_wk=x["fmap_wk"], impl=_impl(lz, impl))
    assert lz.workspace_status(ws) == lz.OK
    y = {k_: to64(v_) for k_, v_ in inp.items() if v_ is not None}
    U_want, R_want = ref.gla_segment_state(y["k"], y["v"], y["g"], tau=w.gate_temp, fmap_wk=y["fmap_wk"],
                                           gate=gate_of(y))
    check("U", U, U_want, dtype)
    check("R", R, R_want, "fp32")


@pytest.mark.parametrize("d,rank", [(64, 0), (64, 2), (128, 3)])
def test_chain_states_matches_oracle(lz, d, rank):
    gen = torch.Generator().manual_seed(d + rank)
    nseg, B, H = 3, 2, 3
    U = torch.randn(nseg, B, H, d, d, generator=gen)
    R = -torch.rand(nseg, B, H, d, generator=gen) * 4
    S_in = torch.randn(B, H, d, d, generator=gen)
    got = lz.chain_states(U.cuda(), R.cuda(), rank, state_in=S_in.cuda())
    want = ref.chain_states(list(to64(U)), list(to64(R)), rank, to64(S_in))
    check("S", got, want, "fp32")


SPLIT_CASES = [
    # impl, dtype, d, B, H, cuts, window, M, gate
    ("tc", "bf16", 128, 2, 2, [0, 256, 400, 650], 128, 4, "dim"),
    ("tc", "bf16", 128, 1, 2, [0, 1000, 2200], 128, 4, "scalar"),   # the first segment splits itself
    ("simt", "fp32", 64, 2, 2, [0, 40, 97, 150], 16, 4, "dim"),
]


@pytest.mark.parametrize("impl,dtype,d,B,H,cuts,window,M,gate", SPLIT_CASES)
def test_segments_one_after_another_reproduce_the_whole_forward(lz, impl, dtype, d, B, H, cuts, window,
                                                                 M, gate):
    """Each segment as a rank runs it (summary, chain of the earlier
    summaries, forward with start state and prefix); the gather of the
    summaries is a stack here, the collectives are tested on the CPU."""
    w, inp = _whole(dtype, d, B, H, cuts[-1], window, M, gate, seed=800 + cuts[-1])
    S_in = torch.randn(B, H, d, d, generator=torch.Generator().manual_seed(8)) * 0.1
    x = to_device(inp)
    im = _impl(lz, impl)
    n = len(cuts) - 1
    Us, Rs = [], []
    for r in range(n - 1):
        s = _span(x, cuts[r], cuts[r + 1])
        U, R, _ = lz.segment_state(s["k"], s["v"], s["g"], window=window, gate_temp=w.gate_temp,
                                   fmap_wk=x["fmap_wk"], impl=im)
        Us.append(U)
        Rs.append(R)
    Us.append(torch.zeros_like(Us[0]))
    Rs.append(torch.zeros_like(Rs[0]))
    U_all, R_all = torch.stack(Us), torch.stack(Rs)
    outs, last = [], None
    for r in range(n):
        a, b = cuts[r], cuts[r + 1]
        s = _span(x, a, b)
        S0 = lz.chain_states(U_all, R_all, r, state_in=S_in.cuda())
        pre = {} if r == 0 else {"k_prefix": x["k"][:, :, a - window:a].contiguous(),
                                 "v_prefix": x["v"][:, :, a - window:a].contiguous()}
        res = lz.attn_fwd(s["q"], s["k"], s["v"], s["g"], window=window, gate_temp=w.gate_temp,
                          state_in=S0, want_state=r == n - 1, impl=im, **pre, **_params(x))
        assert lz.workspace_status(res["workspace"]) == lz.OK
        outs.append(res["o"])
        last = res["state_out"]
    y = {k_: to64(v_) for k_, v_ in inp.items() if v_ is not None}
    want = ref.lizard_forward(y["q"], y["k"], y["v"], y["g"], window=window, tau=w.gate_temp,
                              state_in=to64(S_in), gate=gate_of(y), **_params(y))
    check("o", torch.cat(outs, dim=2), want["o"], dtype)
    check("state_out", last, want["state_out"], dtype)


BWD_SPLIT_CASES = [
    # impl, dtype, d, B, H, cuts, window, M, gate
    ("tc", "bf16", 128, 2, 2, [0, 256, 400, 650], 128, 4, "dim"),
    ("tc", "bf16", 128, 2, 2, [0, 300, 517], 100, 4, "scalar"),
    ("simt", "fp32", 64, 2, 2, [0, 40, 97, 150], 16, 4, "dim"),
]


@pytest.mark.parametrize("impl,dtype,d,B,H,cuts,window,M,gate", BWD_SPLIT_CASES)
def test_segments_one_after_another_reproduce_the_whole_backward(lz, impl, dtype, d, B, H, cuts, window,
                                                                  M, gate):
    """The split backward as the ranks run it, one segment after another on
    one GPU (the gathers are stacks here; the collectives are tested on the
    CPU): each segment's backward from its start state and prefix, the
    end-state gradients chained from the last segment down, the GLA-only
    correction with that gradient, the prefix gradients added to the
    previous segment's last keys and values, parameter gradients summed."""
    w, inp = _whole(dtype, d, B, H, cuts[-1], window, M, gate, seed=850 + cuts[-1])
    S_in = torch.randn(B, H, d, d, generator=torch.Generator().manual_seed(9)) * 0.1
    G = torch.randn(B, H, d, d, generator=torch.Generator().manual_seed(10)) * 0.1
    dout = torch.randn(B, H, cuts[-1], d, generator=torch.Generator().manual_seed(12)).to(inp["q"].dtype)
    x = to_device(inp)
    x["dout"] = dout.cuda()
    im = _impl(lz, impl)
    n = len(cuts) - 1
    kw = dict(window=window, gate_temp=w.gate_temp, impl=im, **_params(x))
    seg = [dict(_span(x, cuts[r], cuts[r + 1]), dout=x["dout"][:, :, cuts[r]:cuts[r + 1]].contiguous())
           for r in range(n)]
    sums = [lz.segment_state(s["k"], s["v"], s["g"], window=window, gate_temp=w.gate_temp,
                             fmap_wk=x["fmap_wk"], impl=im) for s in seg]
    U_all = torch.stack([u for u, _, _ in sums])
    R_all = torch.stack([r_ for _, r_, _ in sums])
    S0 = [lz.chain_states(U_all, R_all, r, state_in=S_in.cuda()) for r in range(n)]
    pre = [{}] + [{"k_prefix": x["k"][:, :, cuts[r] - window:cuts[r]].contiguous(),
                   "v_prefix": x["v"][:, :, cuts[r] - window:cuts[r]].contiguous()} for r in range(1, n)]
    gr = [lz.attn_bwd(s["q"], s["k"], s["v"], s["g"], s["dout"], state_in=S0[r],
                      dstate_out=G.cuda() if r == n - 1 else None, **pre[r], **kw)
          for r, s in enumerate(seg)]
    D_all = torch.stack([gr[r]["dstate_in"] for r in range(n)])
    for r in range(n - 1):
        X = lz.chain_states(torch.flip(D_all, dims=[0]).contiguous(), torch.flip(R_all, dims=[0]).contiguous(),
                            n - 1 - r)
        s = seg[r]
        c = lz.attn_bwd(s["q"], s["k"], s["v"], s["g"], torch.zeros_like(s["dout"]), state_in=S0[r],
                        dstate_out=X, branch=lz.BRANCH_GLA_ONLY, **kw)
        for name in ("dq", "dk", "dv", "dg", "dfmap_wq", "dfmap_wk", "dstate_in"):
            gr[r][name] = gr[r][name] + c[name]
    for r in range(1, n):
        gr[r - 1]["dk"][:, :, -window:] += gr[r]["dk_prefix"]
        gr[r - 1]["dv"][:, :, -window:] += gr[r]["dv_prefix"]
    for r in range(n):
        assert lz.workspace_status(gr[r]["workspace"]) == lz.OK
    y = {k_: to64(v_) for k_, v_ in inp.items() if v_ is not None}
    want = ref.lizard_backward(y["q"], y["k"], y["v"], y["g"], to64(dout), window=window, tau=w.gate_temp,
                               state_in=to64(S_in), dstate_out=to64(G), gate=gate_of(y), **_params(y))
    for name in ("dq", "dk", "dv", "dg"):
        check(name, torch.cat([g_[name] for g_ in gr], dim=2), want[name], dtype)
    for name in ("dmeta_k", "dmeta_v", "dfmap_wq", "dfmap_wk", "dalpha"):
        check(name, sum(g_[name] for g_ in gr), want[name], dtype)
    check("dstate_in", gr[0]["dstate_in"], want["dstate_in"], dtype)


@pytest.mark.timeout(300)
def test_driver_on_a_one_rank_nccl_group(lz):
    """The product driver with its default (library) ops over NCCL, one rank:
    no halo, the all-gathers of one, the chain of nothing, the forward."""
    import torch.distributed as dist
    from gated_linear_sliding_chunkwise_b200 import seqpar
    from lizard_testutil import oracle_forward

    w, inp = _whole("bf16", 128, 2, 2, 300, 128, 4, "dim", seed=901)
    x = to_device(inp)
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    os.environ.setdefault("MASTER_PORT", "29517")
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    try:
        res = seqpar.sequence_parallel_forward(x["q"], x["k"], x["v"], x["g"], window=128,
                                               gate_temp=w.gate_temp, **_params(x))
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    want = oracle_forward(inp, window=128, tau=w.gate_temp)
    check("o", res["o"], want["o"], "bf16")
    check("state_out", res["state_out"], want["state_out"], "bf16")
