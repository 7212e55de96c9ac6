"""Helpers shared by the GPU parity tests: run the oracle on the same seeded
inputs (optionally on a sample of (batch, head) pairs) and compare."""

from __future__ import annotations

import os

import numpy as np
import torch

from oracle import lizard_ref as ref

# Tolerances (GPU vs fp64 oracle).
FP32_ATOL = 1e-4          # fp32 activations: max abs error, every output and gradient
BF16_REL = 2e-2           # bf16 activations: max|x - ref| / max|ref|

_LOG = os.environ.get("LIZARD_PARITY_LOG")


def to64(t):
    if t is None:
        return None
    return t.detach().to("cpu", torch.float64).numpy()


def report(line):
    """One parity line on stdout (shown with pytest -s / -rA) and, when
    LIZARD_PARITY_LOG names a file, appended there."""
    print(line)
    if _LOG:
        with open(_LOG, "a") as f:
            f.write(line + "\n")


def check(name, got, want, dtype):
    """Compare one output: fp32 by max abs error <= FP32_ATOL, bf16 by the
    normwise relative error max|x - ref| / max|ref| <= BF16_REL.  Every
    comparison reports both errors."""
    got = to64(got) if isinstance(got, torch.Tensor) else np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert got.shape == want.shape, f"{name}: shape {got.shape} vs {want.shape}"
    assert np.all(np.isfinite(got)), f"{name}: non-finite values"
    err = float(np.max(np.abs(got - want))) if got.size else 0.0
    mx = float(np.max(np.abs(want))) if want.size else 0.0
    rel = err / max(mx, 1e-30)
    report(f"PARITY {name} [{dtype}] max_abs={err:.3e} max_ref={mx:.3e} normwise={rel:.3e}")
    if dtype == "fp32":
        assert err <= FP32_ATOL, f"{name}: max abs err {err:.3e} > {FP32_ATOL} (max|ref| {mx:.3e})"
    else:
        assert rel <= BF16_REL, f"{name}: normwise rel err {rel:.3e} > {BF16_REL} (max|ref| {mx:.3e})"
    return err


def head_inputs(inp, b, h, keys=("q", "k", "v", "g", "dout")):
    """Slice one (batch, head) pair out of a workload's CPU inputs (fp64)."""
    out = {}
    for k_ in keys:
        if k_ in inp and inp[k_] is not None:
            out[k_] = to64(inp[k_][b:b + 1, h:h + 1])
    for k_ in ("fmap_wq", "fmap_wk", "meta_k", "meta_v", "alpha"):
        if k_ in inp and inp[k_] is not None:
            out[k_] = to64(inp[k_][h:h + 1])
    if inp.get("state_in") is not None:
        out["state_in"] = to64(inp["state_in"][b:b + 1, h:h + 1])
    return out


def gate_of(x):
    """Scalar gate when the logits lack q's last axis (one per token and head)."""
    g, q = x.get("g"), x["q"]
    return ref.GATE_SCALAR if g is not None and g.ndim == q.ndim - 1 else ref.GATE_PER_DIM


def oracle_forward(inp, *, window, tau, branch=ref.BRANCH_BOTH, pairs=None):
    """Oracle forward on all pairs (pairs None) or on listed (b, h) pairs.
    Returns {(b, h) or 'all': result dict}."""
    if pairs is None:
        x = {k_: to64(v_) for k_, v_ in inp.items() if v_ is not None and k_ != "dout"}
        return ref.lizard_forward(x["q"], x["k"], x["v"], x["g"], window=window, tau=tau,
                                  fmap_wq=x.get("fmap_wq"), fmap_wk=x.get("fmap_wk"),
                                  meta_k=x.get("meta_k"), meta_v=x.get("meta_v"),
                                  alpha=x.get("alpha"), state_in=x.get("state_in"),
                                  branch=branch, gate=gate_of(x))
    res = {}
    for (b, h) in pairs:
        x = head_inputs(inp, b, h)
        res[(b, h)] = ref.lizard_forward(x["q"], x["k"], x["v"], x["g"], window=window,
                                         tau=tau, fmap_wq=x.get("fmap_wq"),
                                         fmap_wk=x.get("fmap_wk"), meta_k=x.get("meta_k"),
                                         meta_v=x.get("meta_v"), alpha=x.get("alpha"),
                                         state_in=x.get("state_in"), branch=branch,
                                         gate=gate_of(x))
    return res


def oracle_backward(inp, *, window, tau, branch=ref.BRANCH_BOTH, pairs=None):
    if pairs is None:
        x = {k_: to64(v_) for k_, v_ in inp.items() if v_ is not None}
        return ref.lizard_backward(x["q"], x["k"], x["v"], x["g"], x["dout"], window=window,
                                   tau=tau, fmap_wq=x.get("fmap_wq"), fmap_wk=x.get("fmap_wk"),
                                   meta_k=x.get("meta_k"), meta_v=x.get("meta_v"),
                                   alpha=x.get("alpha"), state_in=x.get("state_in"),
                                   branch=branch, gate=gate_of(x))
    res = {}
    for (b, h) in pairs:
        x = head_inputs(inp, b, h)
        res[(b, h)] = ref.lizard_backward(x["q"], x["k"], x["v"], x["g"], x["dout"],
                                          window=window, tau=tau, fmap_wq=x.get("fmap_wq"),
                                          fmap_wk=x.get("fmap_wk"), meta_k=x.get("meta_k"),
                                          meta_v=x.get("meta_v"), alpha=x.get("alpha"),
                                          state_in=x.get("state_in"), branch=branch,
                                         gate=gate_of(x))
    return res


def to_device(inp, device="cuda"):
    return {k_: (None if v_ is None else v_.to(device).contiguous()) for k_, v_ in inp.items()}
