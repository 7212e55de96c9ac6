"""Seeded synthetic inputs for the Lizard attention workloads.

This module only draws random numbers and rounds them to the storage dtype;
it holds none of the layer's arithmetic.  Both the CUDA-path tests and the
CPU oracle consume exactly these tensors, so both sides see identical
(already rounded) values.

Recipe (one torch.Generator on the CPU, seeded per workload, drawn in this
fixed order, fp32 then rounded once to the activation dtype with RNE):

  q, k, v      ~ N(0, 1) / 8          [B, H, L, d]
  g            ~ N(gate_mean, 1)      [B, H, L, d]   gate logits ([B, H, L] for
                                                     the scalar gate)
  fmap_wq, wk  ~ N(0, 1) * 0.02       [H, d, d/2]    fp32 (parameters)
  meta_k, v    ~ N(0, 1) / 8          [H, M, d]      fp32 (parameters)
  alpha        = 1                    [H]            fp32
  dout         ~ N(0, 1)              [B, H, L, d]   (training workloads)

Decode workloads additionally draw state ~ N(0, 1) * 0.1 (fp32) and full
window caches ~ N(0, 1) / 8 in the activation dtype, with pos = 65536 tokens
already seen, after q, k, v, g and before the parameters.
"""

from __future__ import annotations

from dataclasses import dataclass, asdict

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    L: int
    d: int
    chunk: int = 64
    window: int = 128
    M: int = 4
    dtype: str = "bf16"          # activation storage dtype: "bf16" | "fp32"
    gate_mean: float = 0.0
    gate_temp: float = 16.0
    seed: int = 0
    kind: str = "fwd"            # "fwd" | "train" | "decode"
    decode_pos: int = 65536
    gate: str = "dim"            # "dim": a logit per key dimension | "scalar": one per token-head

    def as_dict(self):
        return asdict(self)


# The five workloads: a tiny fp32 correctness case, one Llama-3-8B-shaped
# attention layer, a 16K-token forward with slow decay, a training step and a
# batched decode step.
WORKLOADS = {
    "tiny_fp32": Workload("tiny_fp32", B=1, H=2, L=256, d=64, window=16,
                          dtype="fp32", seed=0),
    "llama8b_layer_fwd": Workload("llama8b_layer_fwd", B=4, H=32, L=2048,
                                  d=128, seed=1),
    "long_fwd_16k": Workload("long_fwd_16k", B=1, H=32, L=16384, d=128,
                             gate_mean=2.0, seed=2),
    "train_step": Workload("train_step", B=8, H=32, L=2048, d=128, seed=3,
                           kind="train"),
    "decode_b64": Workload("decode_b64", B=64, H=32, L=1, d=128, seed=4,
                           kind="decode"),
}
WORKLOAD_ORDER = ["tiny_fp32", "llama8b_layer_fwd", "long_fwd_16k",
                  "train_step", "decode_b64"]


def torch_dtype(name: str) -> torch.dtype:
    return {"bf16": torch.bfloat16, "fp32": torch.float32}[name]


def make_inputs(w: Workload, *, B=None, H=None, L=None, d=None, seed=None,
                M=None, with_dout=None, gate=None):
    """Draw one workload's inputs on the CPU (optionally with new sizes).

    Returns a dict of CPU tensors: activations in the workload's dtype,
    parameters in fp32.
    """
    B = w.B if B is None else B
    H = w.H if H is None else H
    L = w.L if L is None else L
    d = w.d if d is None else d
    M = w.M if M is None else M
    seed = w.seed if seed is None else seed
    gd = () if (w.gate if gate is None else gate) == "scalar" else (d,)
    dt = torch_dtype(w.dtype)
    gen = torch.Generator().manual_seed(seed)

    def rn(*shape):
        return torch.randn(*shape, generator=gen, dtype=torch.float32)

    out = {}
    if w.kind == "decode":
        out["q"] = (rn(B, H, d) / 8).to(dt)
        out["k"] = (rn(B, H, d) / 8).to(dt)
        out["v"] = (rn(B, H, d) / 8).to(dt)
        out["g"] = (rn(B, H, *gd) + w.gate_mean).to(dt)
        out["state"] = rn(B, H, d, d) * 0.1
        out["k_cache"] = (rn(B, H, w.window, d) / 8).to(dt)
        out["v_cache"] = (rn(B, H, w.window, d) / 8).to(dt)
        out["pos"] = torch.full((B,), w.decode_pos, dtype=torch.int64)
    else:
        out["q"] = (rn(B, H, L, d) / 8).to(dt)
        out["k"] = (rn(B, H, L, d) / 8).to(dt)
        out["v"] = (rn(B, H, L, d) / 8).to(dt)
        out["g"] = (rn(B, H, L, *gd) + w.gate_mean).to(dt)
    out["fmap_wq"] = rn(H, d, d // 2) * 0.02
    out["fmap_wk"] = rn(H, d, d // 2) * 0.02
    out["meta_k"] = rn(H, M, d) / 8
    out["meta_v"] = rn(H, M, d) / 8
    out["alpha"] = torch.ones(H, dtype=torch.float32)
    want_dout = (w.kind == "train") if with_dout is None else with_dout
    if want_dout and w.kind != "decode":
        out["dout"] = rn(B, H, L, d).to(dt)
    return out


def random_alpha(H, seed):
    """Per-head mixing weights in (0, 2), for tests that vary alpha."""
    gen = torch.Generator().manual_seed(seed)
    return torch.rand(H, generator=gen, dtype=torch.float32) * 2.0
