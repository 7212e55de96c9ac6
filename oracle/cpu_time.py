"""Time the CPU oracle on the host cores (test infrastructure).

Run as ``python -m oracle.cpu_time --workload NAME ...`` by the CPU-baseline
and reference legs of ``bench.py``; prints one JSON line.  The process draws
the workload's seeded inputs itself, never touches a GPU, and forks one worker
per host core (numpy limited to one thread in each), so every core runs the
fp64 oracle (forward + backward) over whole (batch, head) sequences of the
workload, or over their first ``--tokens`` tokens.

Two modes:
  --budget S        as many sequences as fit in about S seconds of wall time,
                    in rounds of one sequence per core;
  --steps K         K timed steps after --warmup W, each step one sequence per
                    core (the reference arm's steps).
"""

from __future__ import annotations

import os

for _v in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS", "NUMEXPR_NUM_THREADS"):
    os.environ[_v] = "1"

import argparse  # noqa: E402
import json  # noqa: E402
import multiprocessing as mp  # noqa: E402
import sys  # noqa: E402
import time  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

_INP = None     # the workload's inputs, fp64 numpy, set before the fork
_KW = None


def _one(job):
    """Oracle forward + backward of one (b, h) sequence (first n tokens)."""
    from oracle import lizard_ref as ref
    b, h, n = job
    f = {k: _INP[k][b:b + 1, h:h + 1, :n] for k in ("q", "k", "v", "g", "dout")}
    p = {k: _INP[k][h:h + 1] for k in ("fmap_wq", "fmap_wk", "meta_k", "meta_v", "alpha")}
    ref.lizard_forward(f["q"], f["k"], f["v"], f["g"], **_KW, **p)
    ref.lizard_backward(f["q"], f["k"], f["v"], f["g"], f["dout"], **_KW, **p)
    return n


def main(argv=None):
    global _INP, _KW
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="train_step")
    ap.add_argument("--seed", type=int, default=None)
    ap.add_argument("--tokens", type=int, default=None, help="first n tokens of each sequence")
    ap.add_argument("--budget", type=float, default=None)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=0)
    ap.add_argument("--cores", type=int, default=None)
    a = ap.parse_args(argv)

    from gated_linear_sliding_chunkwise_b200.synth import WORKLOADS, make_inputs
    w = WORKLOADS[a.workload]
    inp = make_inputs(w, seed=a.seed, with_dout=True)
    _INP = {k: v.double().numpy() for k, v in inp.items() if v is not None}
    _KW = dict(window=w.window, tau=w.gate_temp)
    n = min(a.tokens or w.L, w.L)
    cores = a.cores or len(os.sched_getaffinity(0))
    pairs = [(b, h) for h in range(w.H) for b in range(w.B)]

    def jobs(k0, count):
        return [(*pairs[(k0 + i) % len(pairs)], n) for i in range(count)]

    with mp.get_context("fork").Pool(cores) as pool:
        pool.map(_one, [(0, 0, min(n, 16))] * cores)      # start every worker
        if a.steps is not None:
            for i in range(a.warmup):
                pool.map(_one, jobs(i * cores, cores))
            t0 = time.perf_counter()
            for i in range(a.steps):
                pool.map(_one, jobs((a.warmup + i) * cores, cores))
            dt = time.perf_counter() - t0
            done = a.steps * cores
            out = {"token_heads_per_s": done * n / dt, "sec_per_step": dt / a.steps,
                   "sequences_per_step": cores}
        else:
            budget = a.budget if a.budget is not None else 15.0
            done, k0 = 0, 0
            t0 = time.perf_counter()
            while True:
                pool.map(_one, jobs(k0, cores))
                done += cores
                k0 += cores
                if time.perf_counter() - t0 > budget or k0 >= len(pairs):
                    break
            dt = time.perf_counter() - t0
            out = {"token_heads_per_s": done * n / dt, "seconds": dt}
    out.update({"sequences": done, "tokens_per_sequence": n, "cores": cores, "H": w.H,
                "host_cores_available": len(os.sched_getaffinity(0))})
    print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
