"""The sequence-parallel forward's exchange logic on the CPU: one process per
rank over gloo, world sizes 2, 3 and 4.  The compute steps are the oracle's
(a test stand-in passed as `ops`; the product's default ops are the CUDA
library); what is tested is the driver: halo send/receive, the all-gather
of segment summaries, each rank's chain, and that the segments' outputs put
together equal the whole-sequence forward."""

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


def _run(world, cuts, gate):
    port = _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.SimpleQueue()
    mp.start_processes(_worker, args=(world, port, cuts, gate, out), nprocs=world, join=True,
                       start_method="spawn")
    return sorted((out.get() for _ in range(world)), key=lambda r: r[0])


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
