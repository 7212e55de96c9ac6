"""The sequence-parallel exchange logic on the CPU: one process per rank over
gloo, world sizes 2, 3 and 4.  The compute steps are the oracle's (a test
stand-in passed as `ops`; the product's default ops are the CUDA library);
what is tested is the driver: halo send/receive, the all-gather of segment
summaries, each rank's chain, the backward's end-state gradient chain and
prefix-gradient return, and that the segments' outputs and gradients put
together equal the whole sequence's.  A device error reported by one
rank's ops is raised on every rank."""

import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from gated_linear_sliding_chunkwise_b200 import seqpar  # noqa: E402
from oracle import lizard_ref as ref  # noqa: E402

WINDOW, L, D = 4, 29, 4


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _np(t):
    return None if t is None else t.detach().numpy()


def _gate(g, k):
    return ref.GATE_PER_DIM if g.dim() == k.dim() else ref.GATE_SCALAR


class OracleOps:
    """The three compute steps done by the oracle; states come back fp32 as
    the library's do."""

    def segment_state(self, k, v, g, *, window, chunk, gate_temp, fmap_wk, impl):
        U, R = ref.gla_segment_state(_np(k), _np(v), _np(g), tau=gate_temp, fmap_wk=_np(fmap_wk),
                                     gate=_gate(g, k))
        return torch.from_numpy(U).float(), torch.from_numpy(R).float()

    def chain_states(self, seg_state, seg_log_decay, rank, state_in):
        S = ref.chain_states(list(_np(seg_state)), list(_np(seg_log_decay)), rank, _np(state_in))
        return torch.from_numpy(S).float()

    def forward(self, q, k, v, g, *, state_in, k_prefix, v_prefix, want_state, window, gate_temp,
                fmap_wq, fmap_wk, meta_k, meta_v, alpha, **_):
        out = ref.lizard_forward(_np(q), _np(k), _np(v), _np(g), window=window, tau=gate_temp,
                                 fmap_wq=_np(fmap_wq), fmap_wk=_np(fmap_wk), meta_k=_np(meta_k),
                                 meta_v=_np(meta_v), alpha=_np(alpha), state_in=_np(state_in),
                                 k_prefix=_np(k_prefix), v_prefix=_np(v_prefix), gate=_gate(g, k))
        return {"o": torch.from_numpy(out["o"]), "state_out": torch.from_numpy(out["state_out"])}

    def backward(self, q, k, v, g, dout, *, state_in, k_prefix, v_prefix, dstate_out, branch, window,
                 gate_temp, fmap_wq, fmap_wk, meta_k, meta_v, alpha, **_):
        out = ref.lizard_backward(_np(q), _np(k), _np(v), _np(g), _np(dout), window=window, tau=gate_temp,
                                  fmap_wq=_np(fmap_wq), fmap_wk=_np(fmap_wk), meta_k=_np(meta_k),
                                  meta_v=_np(meta_v), alpha=_np(alpha), state_in=_np(state_in),
                                  k_prefix=_np(k_prefix), v_prefix=_np(v_prefix),
                                  dstate_out=_np(dstate_out), branch=branch, gate=_gate(g, k))
        return {n: None if t is None else torch.from_numpy(t) for n, t in out.items()}


class FailingOps(OracleOps):
    """Oracle ops whose device status reads as a timeout on one rank."""

    def __init__(self, bad):
        self.bad = bad

    def status(self):
        return 4 if dist.get_rank() == self.bad else 0


def _inputs(gate):
    r = np.random.default_rng(17)
    B, H = 2, 2
    x = {
        "q": r.standard_normal((B, H, L, D)) * 0.7,
        "k": r.standard_normal((B, H, L, D)) * 0.7,
        "v": r.standard_normal((B, H, L, D)),
        "g": r.standard_normal((B, H, L, D) if gate == "dim" else (B, H, L)) * 2.0,
    }
    p = {
        "fmap_wq": r.standard_normal((H, D, D // 2)),
        "fmap_wk": r.standard_normal((H, D, D // 2)),
        "meta_k": r.standard_normal((H, 2, D)),
        "meta_v": r.standard_normal((H, 2, D)),
        "alpha": r.uniform(0.2, 1.8, H),
        "state_in": r.standard_normal((B, H, D, D)) * 0.3,
    }
    return x, p


def _worker(rank, world, port, cuts, gate, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        x, p = _inputs(gate)
        a, b = cuts[rank], cuts[rank + 1]
        seg = {k_: torch.from_numpy(v_[:, :, a:b].copy()) for k_, v_ in x.items()}
        prm = {k_: torch.from_numpy(v_) for k_, v_ in p.items()}
        try:
            res = seqpar.sequence_parallel_forward(
                seg["q"], seg["k"], seg["v"], seg["g"], window=WINDOW, gate_temp=16.0, ops=OracleOps(),
                **prm)
            out.put((rank, _np(res["o"]), _np(res["state_out"]), None))
        except ValueError as e:
            out.put((rank, None, None, str(e)))
    finally:
        dist.destroy_process_group()


def _run(world, cuts, gate, worker=None, extra=()):
    port = _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.SimpleQueue()
    mp.start_processes(worker or _worker, args=(world, port, cuts, gate, out, *extra), nprocs=world,
                       join=True, start_method="spawn")
    return sorted((out.get() for _ in range(world)), key=lambda r: r[0])


def _dout(gate):
    return np.random.default_rng(23).standard_normal((2, 2, L, D))


def _G():
    return np.random.default_rng(29).standard_normal((2, 2, D, D))


def _bwd_worker(rank, world, port, cuts, gate, out, with_g, bad):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        x, p = _inputs(gate)
        a, b = cuts[rank], cuts[rank + 1]
        seg = {k_: torch.from_numpy(v_[:, :, a:b].copy()) for k_, v_ in x.items()}
        dout = torch.from_numpy(_dout(gate)[:, :, a:b].copy())
        prm = {k_: torch.from_numpy(v_) for k_, v_ in p.items()}
        G = torch.from_numpy(_G()) if with_g else None
        ops = OracleOps() if bad is None else FailingOps(bad)
        try:
            res = seqpar.sequence_parallel_backward(
                seg["q"], seg["k"], seg["v"], seg["g"], dout, window=WINDOW, gate_temp=16.0, ops=ops,
                dstate_out=G, **prm)
            out.put((rank, {n: _np(t) for n, t in res.items()}, None))
        except RuntimeError as e:
            out.put((rank, None, str(e)))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(300)
@pytest.mark.parametrize("world,cuts,gate,with_g", [
    (2, [0, 13, L], "dim", False),
    (3, [0, 9, 18, L], "scalar", True),
    (3, [0, 4, 20, L], "dim", True),      # a segment exactly one window long
    (4, [0, 5, 12, 22, L], "dim", False),
])
def test_split_backward_equals_the_whole_backward(world, cuts, gate, with_g):
    """Every rank's gradients (its tokens' dq, dk, dv, dg; the parameters'
    summed over ranks; dstate_in on rank 0) equal the whole sequence's."""
    got = _run(world, cuts, gate, _bwd_worker, (with_g, None))
    assert all(err is None for _, _, err in got), got
    x, p = _inputs(gate)
    whole = ref.lizard_backward(**x, dout=_dout(gate), window=WINDOW, gate=gate,
                                dstate_out=_G() if with_g else None, **p)
    for name in ("dq", "dk", "dv", "dg"):
        np.testing.assert_allclose(np.concatenate([r[1][name] for r in got], axis=2), whole[name],
                                   rtol=1e-5, atol=1e-6, err_msg=name)
    for name in ("dmeta_k", "dmeta_v", "dfmap_wq", "dfmap_wk", "dalpha"):
        for _, res, _ in got:
            np.testing.assert_allclose(res[name], whole[name], rtol=1e-5, atol=1e-6, err_msg=name)
    np.testing.assert_allclose(got[0][1]["dstate_in"], whole["dstate_in"], rtol=1e-5, atol=1e-6)
    assert all(r[1]["dstate_in"] is None for r in got[1:])


@pytest.mark.timeout(300)
def test_a_device_error_on_one_rank_is_raised_on_every_rank():
    got = _run(3, [0, 9, 18, L], "dim", _bwd_worker, (False, 1))
    assert all(err is not None and "status 4" in err for _, _, err in got), got


@pytest.mark.timeout(300)
@pytest.mark.parametrize("world,cuts,gate", [
    (2, [0, 13, L], "dim"),
    (3, [0, 9, 18, L], "dim"),
    (3, [0, 4, 20, L], "scalar"),     # a segment exactly one window long
    (4, [0, 5, 12, 22, L], "dim"),    # four uneven segments
])
def test_split_forward_equals_the_whole_forward(world, cuts, gate):
    got = _run(world, cuts, gate)
    x, p = _inputs(gate)
    whole = ref.lizard_forward(**x, window=WINDOW, gate=gate, **p)
    assert all(err is None for _, _, _, err in got), got
    o = np.concatenate([r[1] for r in got], axis=2)
    np.testing.assert_allclose(o, whole["o"], rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(got[-1][2], whole["state_out"], rtol=1e-5, atol=1e-6)
    assert all(r[2] is None for r in got[:-1])   # the final state lives on the last rank


@pytest.mark.timeout(300)
def test_a_segment_shorter_than_the_window_is_refused_on_every_rank():
    got = _run(3, [0, 10, 12, L], "dim")
    assert all(err is not None and "ranks [1]" in err for _, _, _, err in got), got
