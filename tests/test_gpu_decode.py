"""GPU parity of lizard_decode_step against the oracle, and decode replay
against the GPU forward."""

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


def _oracle_step(inp, w):
    x = {k_: (to64(v_) if k_ != "pos" else v_.numpy()) for k_, v_ in inp.items() if v_ is not None}
    return ref.lizard_decode_step(x["q"], x["k"], x["v"], x["g"], x["state"], x["k_cache"],
                                  x["v_cache"], x["pos"], window=w.window, tau=w.gate_temp,
                                  fmap_wq=x.get("fmap_wq"), fmap_wk=x.get("fmap_wk"),
                                  meta_k=x.get("meta_k"), meta_v=x.get("meta_v"),
                                  alpha=x.get("alpha"))


def _gpu_step(lz, x, w):
    return lz.decode_step(x["q"], x["k"], x["v"], x["g"], x["state"], x["k_cache"],
                          x["v_cache"], x["pos"], gate_temp=w.gate_temp,
                          fmap_wq=x.get("fmap_wq"), fmap_wk=x.get("fmap_wk"),
                          meta_k=x.get("meta_k"), meta_v=x.get("meta_v"), alpha=x.get("alpha"))


def test_decode_full_batch_one_step(lz):
    """The full decode workload (B=64, H=32, d=128, window 128, 65536 tokens
    seen): every output of one step against the oracle."""
    w = WORKLOADS["decode_b64"]
    inp = make_inputs(w)
    x = to_device(inp)
    o = _gpu_step(lz, x, w)
    torch.cuda.synchronize()
    want_o, want_S, want_kc, want_vc, want_pos = _oracle_step(inp, w)
    check("o", o, want_o, "bf16")
    check("state", x["state"], want_S, "fp32")
    # the ring slot write is a copy: bit-exact
    assert torch.equal(x["k_cache"].cpu(), torch.from_numpy(want_kc).to(x["k_cache"].dtype))
    assert torch.equal(x["v_cache"].cpu(), torch.from_numpy(want_vc).to(x["v_cache"].dtype))
    assert torch.equal(x["pos"].cpu(), torch.from_numpy(want_pos))


# bf16 with d = 128, window <= 128 and M <= 16 runs the streaming kernel;
# the other rows run the general one.
@pytest.mark.parametrize("dtype,d,window,M,pos0", [
    ("fp32", 64, 16, 4, 0), ("fp32", 128, 128, 0, 3), ("fp32", 64, 5, 16, 1000),
    ("bf16", 128, 128, 4, 127), ("bf16", 64, 33, 2, 32),
    ("bf16", 128, 100, 0, 3), ("bf16", 128, 5, 16, 1000), ("bf16", 128, 1, 4, 7),
    ("bf16", 128, 129, 4, 500),
])
def test_decode_small_cases(lz, dtype, d, window, M, pos0):
    w = Workload("dec", B=3, H=2, L=1, d=d, window=window, M=M, dtype=dtype, seed=pos0 + d,
                 kind="decode", decode_pos=pos0)
    inp = make_inputs(w)
    if M == 0:
        inp["meta_k"] = inp["meta_v"] = None
    inp["alpha"] = random_alpha(2, seed=window)
    inp["pos"] = torch.tensor([pos0, pos0 + 1, max(0, pos0 - 1)], dtype=torch.int64)
    x = to_device(inp)
    for step in range(3):
        want = _oracle_step({k_: (v_.cpu() if v_ is not None else None) for k_, v_ in x.items()}, w)
        o = _gpu_step(lz, x, w)
        torch.cuda.synchronize()
        check(f"o@{step}", o, want[0], dtype)
        check(f"S@{step}", x["state"], want[1], "fp32")
        assert torch.equal(x["pos"].cpu(), torch.from_numpy(want[4]))


@pytest.mark.parametrize("dtype,d", [("fp32", 64), ("bf16", 64), ("bf16", 128)])
def test_decode_replay_equals_forward(lz, dtype, d):
    """Prefill nothing, decode L tokens one by one: every output equals the
    parallel forward at the same position (GPU vs GPU and vs the oracle)."""
    B, H, L, window, M = 2, 2, 40, 12, 4
    w = Workload("replay", B=B, H=H, L=L, d=d, window=window, M=M, dtype=dtype, seed=77)
    inp = make_inputs(w)
    x = to_device(inp)
    fwd = lz.attn_fwd(x["q"], x["k"], x["v"], x["g"], window=window, gate_temp=w.gate_temp,
                      fmap_wq=x["fmap_wq"], fmap_wk=x["fmap_wk"], meta_k=x["meta_k"],
                      meta_v=x["meta_v"], alpha=x["alpha"], want_state=True)
    dt = x["q"].dtype
    st = {"state": torch.zeros(B, H, d, d, device="cuda"),
          "k_cache": torch.zeros(B, H, window, d, dtype=dt, device="cuda"),
          "v_cache": torch.zeros(B, H, window, d, dtype=dt, device="cuda"),
          "pos": torch.zeros(B, dtype=torch.int64, device="cuda")}
    outs = []
    for t in range(L):
        step = {"q": x["q"][:, :, t].contiguous(), "k": x["k"][:, :, t].contiguous(),
                "v": x["v"][:, :, t].contiguous(), "g": x["g"][:, :, t].contiguous(),
                "fmap_wq": x["fmap_wq"], "fmap_wk": x["fmap_wk"], "meta_k": x["meta_k"],
                "meta_v": x["meta_v"], "alpha": x["alpha"], **st}
        outs.append(_gpu_step(lz, step, w))
    dec = torch.stack(outs, 2)
    torch.cuda.synchronize()
    want = oracle_forward(inp, window=window, tau=w.gate_temp)
    check("decode vs oracle", dec, want["o"], dtype)
    check("forward vs oracle", fwd["o"], want["o"], dtype)
    check("decode state", st["state"], want["state_out"], "fp32" if dtype == "fp32" else dtype)
    assert torch.equal(st["pos"].cpu(), torch.full((B,), L, dtype=torch.int64))


def test_decode_streaming_without_meta_values_and_status(lz):
    """Sink-only meta tokens (no meta values) on the streaming kernel, more
    (batch, head) pairs than SMs, and the timeout flag stays clear."""
    w = Workload("dec_sink", B=40, H=8, L=1, d=128, window=64, M=4, dtype="bf16", seed=9,
                 kind="decode", decode_pos=200)
    inp = make_inputs(w)
    inp["meta_v"] = None
    x = to_device(inp)
    want = _oracle_step({k_: (v_.cpu() if v_ is not None else None) for k_, v_ in x.items()}, w)
    o = _gpu_step(lz, x, w)
    torch.cuda.synchronize()
    check("o", o, want[0], "bf16")
    check("state", x["state"], want[1], "fp32")
    assert torch.equal(x["k_cache"].cpu(), torch.from_numpy(want[2]).to(x["k_cache"].dtype))
    assert torch.equal(x["v_cache"].cpu(), torch.from_numpy(want[3]).to(x["v_cache"].dtype))
    assert lz.decode_status() == lz.OK


@pytest.mark.parametrize("dtype,d,window,L0", [("bf16", 128, 128, 300), ("bf16", 128, 64, 37),
                                                ("fp32", 64, 12, 50), ("bf16", 128, 32, 0)])
def test_prefill_handoff_then_decode(lz, dtype, d, window, L0):
    """Forward over a prefix of L0 tokens (its end state) and lizard_prefill_cache
    (its window), then decode steps: every decoded output equals the whole
    sequence's forward at that position (oracle), and pos advances from L0."""
    B, H, Ld = 2, 2, 6
    L = L0 + Ld
    w = Workload("handoff", B=B, H=H, L=L, d=d, window=window, M=4, dtype=dtype, seed=L0 + d)
    inp = make_inputs(w)
    x = to_device(inp)
    par = dict(fmap_wq=x["fmap_wq"], fmap_wk=x["fmap_wk"], meta_k=x["meta_k"], meta_v=x["meta_v"],
               alpha=x["alpha"])
    pre = {n: x[n][:, :, :L0].contiguous() for n in ("q", "k", "v", "g")}
    dt = x["q"].dtype
    if L0 > 0:
        fwd = lz.attn_fwd(pre["q"], pre["k"], pre["v"], pre["g"], window=window, gate_temp=w.gate_temp,
                          want_state=True, **par)
        state = fwd["state_out"]
    else:
        state = torch.zeros(B, H, d, d, device="cuda")
    kc = torch.full((B, H, window, d), 7.0, dtype=dt, device="cuda")   # stale contents
    vc = torch.full((B, H, window, d), 7.0, dtype=dt, device="cuda")
    pos = torch.full((B,), 99, dtype=torch.int64, device="cuda")
    lz.prefill_cache(pre["k"], pre["v"], kc, vc, pos)
    torch.cuda.synchronize()
    assert torch.equal(pos.cpu(), torch.full((B,), L0, dtype=torch.int64))
    st = {"state": state, "k_cache": kc, "v_cache": vc, "pos": pos}
    outs = []
    for t in range(L0, L):
        step = {n: x[n][:, :, t].contiguous() for n in ("q", "k", "v", "g")}
        outs.append(_gpu_step(lz, {**step, **par, **st}, w))
    dec = torch.stack(outs, 2)
    torch.cuda.synchronize()
    want = oracle_forward(inp, window=window, tau=w.gate_temp)
    check("decode after prefill", dec, want["o"][:, :, L0:], dtype)
    assert torch.equal(pos.cpu(), torch.full((B,), L, dtype=torch.int64))
