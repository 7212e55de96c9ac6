#!/usr/bin/env python
"""Benchmark of the Lizard hybrid attention layer on B200.

One step = one training pass of the layer (forward + backward through
lizard_attn_fwd / lizard_attn_bwd) over the B=8, H=32, L=2048, d=128 bf16
batch (window 128, 4 meta tokens, chunk 64).  The same run times 1000
consecutive single-token decode steps (B=64, H=32, d=128) and reports their
HBM bandwidth in the same JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU: one process per GPU (torchrun); every rank processes its own batch
(independent replicas, no collective on the data path: weak scaling); the
step time is the max over ranks.
"""

from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

METRIC = "hybrid attn fwd+bwd tokens/s & TFLOP/s (% bf16 peak); decode GB/s (% HBM)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "sm_max_mhz": 1965.0}
SM_COUNT = 148
FP32_LANES_PER_SM = 128


# ------------------------------------------------------------ counting ----
def flops_per_token_head(d, C, w, M):
    """Algorithmic FLOPs per (token, head), causal half of the intra tiles,
    feature map excluded: GLA fwd (C+1)(dk+dv) + 4 dk dv, anchor fwd
    2 (dk+dv)(w+M); a training step counts 3x GLA and 3.5x anchor."""
    gla = (C + 1) * (2 * d) + 4 * d * d
    swa = 2 * (2 * d) * (w + M)
    return {"fwd": gla + swa, "train": 3 * gla + 3.5 * swa, "gla_fwd": gla, "swa_fwd": swa}


def bytes_per_token_head(d, esz=2):
    """Minimal HBM bytes per (token, head): forward reads q, k, v, g and
    writes o; the training step adds dout in, dq, dk, dv out (activation
    dtype) and dg out (fp32), and reads q, k, v, g again."""
    fwd = 4 * d * esz + d * esz
    bwd = 5 * d * esz + 3 * d * esz + d * 4
    return {"fwd": fwd, "bwd": bwd, "train": fwd + bwd}


def tc_segments(BH, L, T=128):
    """Segments per sequence of the tensor-core forward (mirrors the library:
    enough (batch, head, segment) CTAs to cover the SMs once, each segment at
    least two tiles long)."""
    nt = math.ceil(L / T)
    n = 1 if BH >= 120 else SM_COUNT // max(BH, 1)
    n = max(1, min(n, nt // 2))
    tps = math.ceil(nt / n)
    return math.ceil(nt / tps)


def kernel_model(name, w, N, BH, train=False):
    """(algorithmic bytes, algorithmic flops) of one launch of a kernel of the
    library over N token-heads (BH sequences): every input and output of the
    kernel counted once (workspace arrays at their stored width), and the
    dense contractions it exists to perform.  train: the forward of a
    training step, which also writes the backward's saved tensors."""
    d, esz = w.d, 2 if w.dtype == "bf16" else 4
    Nd = N * d
    fl = flops_per_token_head(d, w.chunk, w.window, w.M)
    phi = 2 * d * d   # two feature maps: x W for q and k, d x d/2 each
    nch32 = math.ceil(w.L / 32)
    nt = math.ceil(w.L / 128)
    snaps = BH * nt * d * d * 2          # one bf16 d x d state per 128-token tile
    nseg = tc_segments(BH, w.L)
    seg_states = BH * nseg * d * d * 4
    table = {
        # portable kernels
        "prep_kernel": (3 * Nd * esz + 3 * Nd * 4, N * phi),
        "gla_fwd_simt": (3 * Nd * 4 + Nd * esz + Nd * 4, N * fl["gla_fwd"]),
        "swa_mix_simt": (3 * Nd * esz + Nd * 4 + Nd * esz, N * fl["swa_fwd"]),
        "gla_states_simt": (2 * Nd * 4 + Nd * esz + BH * nch32 * d * d * 4, N * 2 * d * d),
        "gla_bwd_simt": (3 * Nd * 4 + 2 * Nd * esz + BH * nch32 * d * d * 4 + 4 * Nd * 4,
                         N * 2 * fl["gla_fwd"]),
        "swa_bwd_q": (4 * Nd * esz + Nd * 4 + 2 * N * 4, N * 1.5 * fl["swa_fwd"]),
        "swa_bwd_kv": (4 * Nd * esz + 2 * N * 4 + 2 * Nd * 4, N * 1.0 * fl["swa_fwd"]),
        "finish_bwd": (3 * Nd * esz + 7 * Nd * 4 + 3 * Nd * esz + Nd * 4, N * 2 * phi),
        # tensor-core kernels (the configuration the bench runs: both branches
        # on the tensor cores, so the branch sums are fused into the anchor
        # kernels and the GLA feature-map parts travel in bf16)
        "gate_prep_kernel": (Nd * esz * 2 + BH * nt * d * 4 + (Nd * 4 if train else 0), 0),
        "tc_fwd_kernel": (5 * Nd * esz + N * 4 + BH * nt * d * 4 + (seg_states if nseg > 1 else 0)
                          + (snaps + BH * nt * d * 4 + BH * d * d * 4 if train else 0),
                          N * (fl["fwd"] + phi)),
        "tc_fwd_kernel(state pass)": ((2 * Nd * esz + Nd * 4) * (nseg - 1) / nseg + seg_states,
                                      N * (nseg - 1) / nseg * (2 * d * d + phi / 2)),
        "seg_combine_kernel": (3 * seg_states, 0),
        "tc_fwd_kernel(state copies)": (2 * Nd * esz + Nd * 4 + snaps, N * (2 * d * d + phi / 2)),
        "tc_gla_dstates_kernel": (2 * Nd * esz + Nd * 4 + snaps + BH * d * d * 4, N * (2 * d * d + phi / 2)),
        "tc_gla_bwd_tile_kernel": (4 * Nd * esz + 2 * snaps + Nd * 4 + 2 * Nd * 4 + 2 * Nd * 2,
                                   N * (2 * fl["gla_fwd"] + phi)),
        "tc_finish_kernel": (4 * Nd * esz + 2 * Nd * 2, N * 3 * phi),
        "tc_swa_bwd_q_kernel": (6 * Nd * esz + 2 * N * 4, N * (1.5 * fl["swa_fwd"] + 4 * d * w.M)),
        "tc_swa_bwd_kv_kernel": (7 * Nd * esz + Nd * 4 + 2 * N * 4, N * 2.0 * fl["swa_fwd"]),
        "gate_grad_kernel": (Nd * 4 + Nd * esz + Nd * 4, 0),
    }
    return table.get(name, (0, 0))


def kernel_io(dom, per, w, N, BH, peaks, args):
    """The dominant kernel's own input/output rate: every array it reads or
    writes (workspace intermediates included, each counted once) over its
    launch time.  These are the bytes of this decomposition into kernels,
    not the step's algorithmic bytes, so they are reported apart from the
    step-level roofline."""
    iob, iofl = kernel_model(dom, w, N, BH, train=True)
    dt = per[dom] / 1e3
    out = {"kernel": dom, "ms_per_launch": per[dom], "io_bytes": iob,
           "io_gbs": iob / dt / 1e9, "io_frac_of_hbm": iob / dt / 1e9 / peaks["hbm_gbs"],
           "tflops": iofl / dt / 1e12, "tflops_frac_of_bf16": iofl / dt / 1e12 / peaks["bf16_tflops"],
           "traffic": MEASURED_TRAFFIC.get(dom) if args.kernels in ("auto", "tc") else None,
           "modeled_step_io_bytes": sum(kernel_model(n, w, N, BH, train=True)[0] for n in per)}
    return out


# ------------------------------------------------------------- clocks -----
class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region."""

    FIELDS = ("index,uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        self.path = None
        try:
            self.uuid = str(torch.cuda.get_device_properties(device_index).uuid)
        except Exception:
            self.uuid = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 10:
                continue
            if self.uuid and self.uuid not in parts[1] and parts[1] not in self.uuid:
                continue
            rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        mx = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[6 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


# -------------------------------------------------------------- helpers ----
# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per launch from
# ncu captures of the current kernels on the train_step workload (B=8, H=32,
# L=2048; profiles/train_step_tc_launches.md,
# profiles/tc_gla_bwd_tile_kernel_train_step.md); "step" sums one training
# step's 14 launches (forward with the saved buffer, backward reading it).
# Kernels changed since their capture are left out.
MEASURED_TRAFFIC = {
    "step": 7_241_256_576,
    "tc_gla_bwd_tile_kernel": 1_852_190_208,
}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        d["source"] = "measured"
        return d
    d = dict(FALLBACK_PEAKS)
    d["source"] = "fallback"
    return d


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def max_over_ranks(x, world, device):
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


DATA = "synthetic (seeded N(0,1)/8 q,k,v; N(0,1) gate logits and dout)"


def train_config(w, world, kernels):
    """The headline workload's config, shared by both arms."""
    return {"workload": "train_step: lizard_attn_fwd + lizard_attn_bwd",
            "B": w.B, "H": w.H, "L": w.L, "d": w.d, "chunk": w.chunk,
            "window": w.window, "M": w.M, "global_batch": w.B * world,
            "seq_len": w.L, "parallelism": f"dp{world} (independent replicas)",
            "kernels": kernels,
            "l2": "inputs larger than L2 (q,k,v,g,dout = 5 x 134 MB per step)"}


# ------------------------------------------------------------ our arm -----
def run_ours(args, rank, world, local):
    from gated_linear_sliding_chunkwise_b200 import lizard as lz
    from gated_linear_sliding_chunkwise_b200.synth import WORKLOADS, make_inputs

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    impl = {"auto": lz.IMPL_AUTO, "simt": lz.IMPL_SIMT, "tc": lz.IMPL_TC}[args.kernels]
    w = WORKLOADS["train_step"]
    inp = make_inputs(w, seed=w.seed + rank)
    x = {k: v.to(dev).contiguous() for k, v in inp.items()}
    kw = dict(window=w.window, chunk=w.chunk, gate_temp=w.gate_temp, fmap_wq=x["fmap_wq"],
              fmap_wk=x["fmap_wk"], meta_k=x["meta_k"], meta_v=x["meta_v"], alpha=x["alpha"],
              impl=impl)
    # persistent outputs/workspaces so the timed loop allocates nothing; the
    # forward keeps its saved-for-backward tensors in `sv` (None on paths
    # that keep nothing), which the backward reads
    o = torch.empty_like(x["q"])
    r0 = lz.attn_fwd(x["q"], x["k"], x["v"], x["g"], out=o, saved=True, **kw)
    fws, sv = r0["workspace"], r0["saved"]
    g0 = lz.attn_bwd(x["q"], x["k"], x["v"], x["g"], x["dout"], saved=sv, **kw)
    bws = g0["workspace"]
    del g0
    fwd_names = lz.attn_fwd(x["q"], x["k"], x["v"], x["g"], plan_only=True, saved=sv, **kw)
    bwd_names = lz.attn_bwd(x["q"], x["k"], x["v"], x["g"], x["dout"], plan_only=True, saved=sv, **kw)
    torch.cuda.synchronize()

    def step(evf=None, evb=None):
        lz.attn_fwd(x["q"], x["k"], x["v"], x["g"], out=o, workspace=fws, events=evf, saved=sv, **kw)
        return lz.attn_bwd(x["q"], x["k"], x["v"], x["g"], x["dout"], workspace=bws,
                           events=evb, saved=sv, **kw)

    for _ in range(args.warmup):
        step()
    K = args.steps
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    start.record()
    for i in range(K):
        step()
    end.record()
    torch.cuda.synchronize()
    clk = clocks.stop()
    barrier(world)
    ms = start.elapsed_time(end) / K
    ms_max = max_over_ranks(ms, world, dev)
    # the device status of every call so far (range, timeout): a step whose
    # kernels gave up or left their range is not a measurement
    for ws_ in (fws, bws):
        st = lz.workspace_status(ws_)
        if st != lz.OK:
            raise RuntimeError(f"training step: device status {st} ({lz.status_string(st)})")
    # Per-kernel device times: the same steps with the library's launch events,
    # which run every kernel in order on the call's stream (the timed steps
    # above let independent backward kernels share the GPU).
    Ka = max(min(K, 20), 3)
    evf = [lz.make_events(len(fwd_names) + 1) for _ in range(Ka)]
    evb = [lz.make_events(len(bwd_names) + 1) for _ in range(Ka)]
    torch.cuda.synchronize()
    for i in range(Ka):
        step(evf[i], evb[i])
    torch.cuda.synchronize()

    N = w.B * w.H * w.L
    BH = w.B * w.H
    tokens = w.B * w.L
    fl = flops_per_token_head(w.d, w.chunk, w.window, w.M)
    by = bytes_per_token_head(w.d)
    value = world * tokens / (ms_max / 1e3)
    tflops = world * N * fl["train"] / (ms_max / 1e3) / 1e12
    peaks = load_peaks()

    # per-kernel device times from the library's launch events
    per = {}
    for names, evs in ((fwd_names, evf), (bwd_names, evb)):
        for j, n in enumerate(names):
            t = statistics.mean(e[j].elapsed_time(e[j + 1]) for e in evs)
            per[n] = per.get(n, 0.0) + t
    dom = max(per, key=per.get)
    kio = kernel_io(dom, per, w, N, BH, peaks, args)
    # Step-level roofline: the training step's algorithmic bytes (q, k, v, g
    # and dout in, o, dq, dk, dv and dg out, q, k, v, g read again: 3840 B per
    # token-head at d = 128) over the measured step time, against the HBM
    # peak (the step's arithmetic intensity, 126 FLOP/B, is below the bf16
    # ridge of about 249 FLOP/B).
    step_bytes = N * by["train"]
    roof = {"bound": "hbm", "achieved": step_bytes / (ms_max / 1e3) / 1e9, "peak": peaks["hbm_gbs"],
            "unit": "GB/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = MEASURED_TRAFFIC.get("step") if args.kernels in ("auto", "tc") else None
    roof["scope"] = ("one training step (every kernel of lizard_attn_fwd + lizard_attn_bwd); "
                     "achieved = 3840 B per token-head x B*H*L / ms_per_step")
    roof["algorithmic_bytes"] = step_bytes
    roof["floor_ms"] = step_bytes / (peaks["hbm_gbs"] * 1e9) * 1e3
    roof["peak_source"] = peaks["source"]
    kernels = {n: round(t, 4) for n, t in per.items()}


    # end to end: pinned host inputs in, gradients out, every step.  Three
    # streams: the inputs of step i + 1 go up and the gradients of step i come
    # down while step i + 1 computes (device inputs and host outputs are
    # double-buffered), so the copies of every step stay inside the timed
    # region but overlap each other and the kernels.
    e2e = None
    if not args.no_e2e:
        ins = ("q", "k", "v", "g", "dout")
        outs_n = ("dq", "dk", "dv", "dg")
        hin = {n: x[n].cpu().pin_memory() for n in ins}
        hout = [{n: torch.empty(x["q"].shape,
                                dtype=torch.float32 if n == "dg" else x["q"].dtype).pin_memory()
                 for n in outs_n} for _ in range(2)]
        h2d = sum(t.numel() * t.element_size() for t in hin.values())
        d2h = sum(t.numel() * t.element_size() for t in hout[0].values())
        dbuf = [{n: torch.empty_like(x[n]) for n in ins} for _ in range(2)]
        s_up, s_comp, s_down = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_used = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]
        ev_down = [torch.cuda.Event() for _ in range(2)]
        grads = [None, None]
        Ke = max(5, min(K, 10))

        def up(i):
            j = i % 2
            with torch.cuda.stream(s_up):
                if i >= 2:
                    s_up.wait_event(ev_used[j])       # step i - 2 has read this input set
                for n in ins:
                    dbuf[j][n].copy_(hin[n], non_blocking=True)
                ev_in[j].record(s_up)

        def compute(i):
            j = i % 2
            d = dbuf[j]
            with torch.cuda.stream(s_comp):
                s_comp.wait_event(ev_in[j])
                lz.attn_fwd(d["q"], d["k"], d["v"], d["g"], out=o, workspace=fws, saved=sv, **kw)
                gr = lz.attn_bwd(d["q"], d["k"], d["v"], d["g"], d["dout"], workspace=bws, saved=sv, **kw)
                ev_used[j].record(s_comp)
                ev_out[j].record(s_comp)
            grads[j] = gr

        def down(i):
            j = i % 2
            with torch.cuda.stream(s_down):
                s_down.wait_event(ev_out[j])
                for n in outs_n:
                    hout[j][n].copy_(grads[j][n], non_blocking=True)
                    grads[j][n].record_stream(s_down)
                ev_down[j].record(s_down)

        def run(nsteps):
            up(0)
            for i in range(nsteps):
                if i + 1 < nsteps:
                    up(i + 1)
                compute(i)
                down(i)

        cur = torch.cuda.current_stream()
        run(2)
        torch.cuda.synchronize()
        barrier(world)
        s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s2.record(cur)
        for st in (s_up, s_comp, s_down):
            st.wait_stream(cur)
        run(Ke)
        for st in (s_up, s_comp, s_down):
            cur.wait_stream(st)
        e2.record(cur)
        torch.cuda.synchronize()
        ems = max_over_ranks(s2.elapsed_time(e2) / Ke, world, dev)
        e2e = {"value": world * tokens / (ems / 1e3), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ems,
               "steps": Ke, "copies": "pinned host, own streams, overlapped across steps"}

    decode = None if args.no_decode else run_decode(args, lz, dev, rank, world, peaks)
    fwd_long = None if args.no_fwd_long else run_forward(args, lz, dev, rank, world, peaks,
                                                         "long_fwd_16k", max(K, 5))
    fwd_layer = None if args.no_fwd_layer else run_forward(args, lz, dev, rank, world, peaks,
                                                           "llama8b_layer_fwd", max(K, 5))
    variants = None if args.no_variants else run_variants(args, lz, dev, rank, world, peaks,
                                                          max(min(K, 30), 5))

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": DATA,
        "config": train_config(w, world, args.kernels),
        "tflops": tflops, "tflops_frac_of_bf16_peak": tflops / peaks["bf16_tflops"],
        "hbm_floor_ms": (N * by["train"]) / (peaks["hbm_gbs"] * 1e9) * 1e3,
        "roofline": roof, "kernel_io": kio, "kernel_ms": kernels,
        "kernel_timing": "per-kernel CUDA events on the launching stream, in a second pass of the same steps "
                         "with every kernel in order (the timed steps run independent backward kernels "
                         "side by side)",
        "gpu_launches": K * (len(fwd_names) + len(bwd_names)),
        "clocks": clk, "e2e": e2e, "decode": decode, "fwd_long_16k": fwd_long,
        "fwd_llama8b_layer": fwd_layer,
        "variants": variants,
    }
    if rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, budget_s=args.cpu_budget, seed=w.seed + rank)
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_forward(args, lz, dev, rank, world, peaks, name, steps):
    """Time lizard_attn_fwd alone on one workload (inputs resident)."""
    from gated_linear_sliding_chunkwise_b200.synth import WORKLOADS, make_inputs

    w = WORKLOADS[name]
    impl = {"auto": lz.IMPL_AUTO, "simt": lz.IMPL_SIMT, "tc": lz.IMPL_TC}[args.kernels]
    inp = make_inputs(w, seed=w.seed + rank)
    x = {k: v.to(dev).contiguous() for k, v in inp.items()}
    kw = dict(window=w.window, chunk=w.chunk, gate_temp=w.gate_temp, fmap_wq=x["fmap_wq"],
              fmap_wk=x["fmap_wk"], meta_k=x["meta_k"], meta_v=x["meta_v"], alpha=x["alpha"],
              impl=impl)
    names = lz.attn_fwd(x["q"], x["k"], x["v"], x["g"], plan_only=True, **kw)
    o = torch.empty_like(x["q"])
    ws = lz.attn_fwd(x["q"], x["k"], x["v"], x["g"], out=o, **kw)["workspace"]
    for _ in range(max(args.warmup, 1)):
        lz.attn_fwd(x["q"], x["k"], x["v"], x["g"], out=o, workspace=ws, **kw)
    evs = [lz.make_events(len(names) + 1) for _ in range(steps)]
    barrier(world)
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for i in range(steps):
        lz.attn_fwd(x["q"], x["k"], x["v"], x["g"], out=o, workspace=ws, events=evs[i], **kw)
    e.record()
    torch.cuda.synchronize()
    ms = max_over_ranks(s.elapsed_time(e) / steps, world, dev)
    per = {n: statistics.mean(ev[j].elapsed_time(ev[j + 1]) for ev in evs) for j, n in enumerate(names)}
    N = w.B * w.H * w.L
    fl = flops_per_token_head(w.d, w.chunk, w.window, w.M)["fwd"] * N
    by = bytes_per_token_head(w.d)["fwd"] * N
    tfl = world * fl / (ms / 1e3) / 1e12
    gbs = world * by / (ms / 1e3) / 1e9
    out = {"workload": f"{name}: B={w.B} H={w.H} L={w.L} d={w.d}", "ms": ms,
           "tokens_per_s": world * w.B * w.L / (ms / 1e3), "tflops": tfl,
           "tflops_frac_of_bf16_peak": tfl / peaks["bf16_tflops"],
           "hbm_gbs": gbs, "hbm_frac": gbs / (world * peaks["hbm_gbs"]),
           "kernel_ms": {n: round(t, 4) for n, t in per.items()}, "launches": len(names)}
    # the forward's algorithmic bytes (q, k, v, g in, o out: 1280 B per
    # token-head) over the whole call's time; arithmetic intensity 117 FLOP/B,
    # below the bf16 ridge, so HBM bounds it
    out["roofline"] = {"bound": "hbm", "achieved": gbs / world, "peak": peaks["hbm_gbs"],
                       "unit": "GB/s", "frac": gbs / (world * peaks["hbm_gbs"]),
                       "floor_ms": by / (peaks["hbm_gbs"] * 1e9) * 1e3,
                       "scope": "one lizard_attn_fwd call (all its kernels)"}
    return out


def run_backward(args, lz, dev, rank, world, peaks, name, steps):
    """Time lizard_attn_bwd alone on one workload (inputs resident)."""
    from gated_linear_sliding_chunkwise_b200.synth import WORKLOADS, make_inputs

    w = WORKLOADS[name]
    impl = {"auto": lz.IMPL_AUTO, "simt": lz.IMPL_SIMT, "tc": lz.IMPL_TC}[args.kernels]
    inp = make_inputs(w, seed=w.seed + rank, with_dout=True)
    x = {k: v.to(dev).contiguous() for k, v in inp.items()}
    kw = dict(window=w.window, chunk=w.chunk, gate_temp=w.gate_temp, fmap_wq=x["fmap_wq"],
              fmap_wk=x["fmap_wk"], meta_k=x["meta_k"], meta_v=x["meta_v"], alpha=x["alpha"],
              impl=impl)
    names = lz.attn_bwd(x["q"], x["k"], x["v"], x["g"], x["dout"], plan_only=True, **kw)
    ws = lz.attn_bwd(x["q"], x["k"], x["v"], x["g"], x["dout"], **kw)["workspace"]
    for _ in range(max(args.warmup, 1)):
        lz.attn_bwd(x["q"], x["k"], x["v"], x["g"], x["dout"], workspace=ws, **kw)
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for i in range(steps):
        lz.attn_bwd(x["q"], x["k"], x["v"], x["g"], x["dout"], workspace=ws, **kw)
    e.record()
    torch.cuda.synchronize()
    ms = s.elapsed_time(e) / steps
    evs = [lz.make_events(len(names) + 1) for _ in range(steps)]   # per kernel, in order
    torch.cuda.synchronize()
    for i in range(steps):
        lz.attn_bwd(x["q"], x["k"], x["v"], x["g"], x["dout"], workspace=ws, events=evs[i], **kw)
    torch.cuda.synchronize()
    per = {n: statistics.mean(ev[j].elapsed_time(ev[j + 1]) for ev in evs) for j, n in enumerate(names)}
    return {"workload": f"{name} backward: B={w.B} H={w.H} L={w.L} d={w.d}", "ms": ms,
            "kernel_ms": {n: round(t, 4) for n, t in per.items()}, "launches": len(names)}


def _time_steps(step, names, lz, world, dev, warmup, steps):
    """Device time per call of step(events) and per kernel (launch events, a
    second pass: with them every kernel runs in order on one stream)."""
    for _ in range(max(warmup, 1)):
        step(None)
    barrier(world)
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for i in range(steps):
        step(None)
    e.record()
    torch.cuda.synchronize()
    ms = max_over_ranks(s.elapsed_time(e) / steps, world, dev)
    evs = [lz.make_events(len(names) + 1) for _ in range(steps)]
    torch.cuda.synchronize()
    for i in range(steps):
        step(evs[i])
    torch.cuda.synchronize()
    per = {}
    for j, n in enumerate(names):
        per[n] = per.get(n, 0.0) + statistics.mean(ev[j].elapsed_time(ev[j + 1]) for ev in evs)
    return ms, {n: round(t, 4) for n, t in per.items()}


def run_variants(args, lz, dev, rank, world, peaks, steps):
    """The training-step shape in the two variants beside the headline step:
    the stage-1 step (forward, mean squared error against a teacher output,
    backward: lizard_stage1_step) and the forward + backward with the scalar
    per-head gate (g [B, H, L])."""
    from gated_linear_sliding_chunkwise_b200.synth import WORKLOADS, make_inputs

    w = WORKLOADS["train_step"]
    impl = {"auto": lz.IMPL_AUTO, "simt": lz.IMPL_SIMT, "tc": lz.IMPL_TC}[args.kernels]
    out = {}
    tokens = w.B * w.L
    fl = flops_per_token_head(w.d, w.chunk, w.window, w.M)["train"] * w.B * w.H * w.L

    inp = make_inputs(w, seed=w.seed + rank)
    x = {k: v.to(dev).contiguous() for k, v in inp.items()}
    gen = torch.Generator().manual_seed(1000 + rank)
    target = (torch.randn(*x["q"].shape, generator=gen) / 8).to(x["q"].dtype).to(dev)
    kw = dict(window=w.window, chunk=w.chunk, gate_temp=w.gate_temp, fmap_wq=x["fmap_wq"],
              fmap_wk=x["fmap_wk"], meta_k=x["meta_k"], meta_v=x["meta_v"], alpha=x["alpha"],
              impl=impl)
    names = lz.stage1_step(x["q"], x["k"], x["v"], x["g"], target, plan_only=True, **kw)
    ws = lz.stage1_step(x["q"], x["k"], x["v"], x["g"], target, **kw)["workspace"]
    ms, per = _time_steps(lambda ev: lz.stage1_step(x["q"], x["k"], x["v"], x["g"], target, workspace=ws,
                                                    events=ev, **kw),
                          names, lz, world, dev, args.warmup, steps)
    out["stage1_step"] = {
        "workload": f"train_step shape, stage-1 step (loss fused in the forward): B={w.B} H={w.H} L={w.L}",
        "ms": ms, "tokens_per_s": world * tokens / (ms / 1e3),
        "tflops": world * fl / (ms / 1e3) / 1e12, "kernel_ms": per, "launches": len(names)}
    del x, ws

    inp = make_inputs(w, seed=w.seed + rank, gate="scalar")
    x = {k: v.to(dev).contiguous() for k, v in inp.items()}
    kw = dict(window=w.window, chunk=w.chunk, gate_temp=w.gate_temp, fmap_wq=x["fmap_wq"],
              fmap_wk=x["fmap_wk"], meta_k=x["meta_k"], meta_v=x["meta_v"], alpha=x["alpha"],
              impl=impl)
    o = torch.empty_like(x["q"])
    r0 = lz.attn_fwd(x["q"], x["k"], x["v"], x["g"], out=o, saved=True, **kw)
    fws, sv = r0["workspace"], r0["saved"]
    bws = lz.attn_bwd(x["q"], x["k"], x["v"], x["g"], x["dout"], saved=sv, **kw)["workspace"]
    fn = lz.attn_fwd(x["q"], x["k"], x["v"], x["g"], plan_only=True, saved=sv, **kw)
    bn = lz.attn_bwd(x["q"], x["k"], x["v"], x["g"], x["dout"], plan_only=True, saved=sv, **kw)
    msf, perf = _time_steps(lambda ev: lz.attn_fwd(x["q"], x["k"], x["v"], x["g"], out=o, workspace=fws,
                                                   events=ev, saved=sv, **kw), fn, lz, world, dev, args.warmup,
                            steps)
    msb, perb = _time_steps(lambda ev: lz.attn_bwd(x["q"], x["k"], x["v"], x["g"], x["dout"], workspace=bws,
                                                   events=ev, saved=sv, **kw), bn, lz, world, dev, args.warmup,
                            steps)
    out["scalar_gate_train_step"] = {
        "workload": f"train_step shape, scalar per-head gate g [B,H,L]: B={w.B} H={w.H} L={w.L}",
        "ms": msf + msb, "fwd_ms": msf, "bwd_ms": msb,
        "tokens_per_s": world * tokens / ((msf + msb) / 1e3),
        "kernel_ms": {**perf, **{("bwd:" + n): t for n, t in perb.items()}},
        "launches": len(fn) + len(bn)}
    return out


def run_decode(args, lz, dev, rank, world, peaks):
    from gated_linear_sliding_chunkwise_b200.synth import WORKLOADS, make_inputs

    w = WORKLOADS["decode_b64"]
    if getattr(args, "decode_batch", None):   # a smaller batch for kernel profiles
        import dataclasses
        w = dataclasses.replace(w, B=args.decode_batch)
    inp = make_inputs(w, seed=w.seed + rank)
    x = {k: v.to(dev).contiguous() for k, v in inp.items()}
    o = torch.empty(w.B, w.H, w.d, dtype=x["q"].dtype, device=dev)

    def st():
        lz.decode_step(x["q"], x["k"], x["v"], x["g"], x["state"], x["k_cache"], x["v_cache"],
                       x["pos"], gate_temp=w.gate_temp, fmap_wq=x["fmap_wq"],
                       fmap_wk=x["fmap_wk"], meta_k=x["meta_k"], meta_v=x["meta_v"],
                       alpha=x["alpha"], out=o)

    for _ in range(10):
        st()
    n = args.decode_steps
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    s.record()
    for _ in range(n):
        st()
    e.record()
    torch.cuda.synchronize()
    us = max_over_ranks(s.elapsed_time(e) * 1e3 / n, world, dev)
    d, W, esz = w.d, w.window, 2
    per_bh = 2 * d * d * 4 + 2 * W * d * esz + 4 * d * esz + 2 * d * esz + d * esz
    step_bytes = w.B * w.H * per_bh + w.H * 2 * d * (d // 2) * 4
    gbs = world * step_bytes / (us * 1e-6) / 1e9
    return {"value": gbs, "unit": "GB/s", "frac_of_hbm": gbs / (world * peaks["hbm_gbs"]),
            "us_per_step": us, "steps": n, "bytes_per_step": step_bytes,
            "workload": f"decode: B={w.B} H={w.H} d={w.d} window {w.window} M={w.M}, pos {w.decode_pos}",
            "launches_per_step": 1}


# ---------------------------------------------------------- CPU oracle ----
def _oracle_timer(*opts):
    """Run the oracle timing harness (oracle/cpu_time.py) in a fresh process
    that never touches a GPU and forks one worker per host core; returns its
    JSON result."""
    cmd = [sys.executable, "-m", "oracle.cpu_time", *map(str, opts)]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=900)
    if r.returncode != 0:
        raise RuntimeError("oracle timing failed: " + r.stderr[-2000:])
    return json.loads(r.stdout.strip().splitlines()[-1])


def cpu_baseline(w, budget_s=15.0, seed=None):
    """Time the fp64 oracle's forward + backward on whole sequences of the
    same workload, on every host core; report layer tokens/s."""
    r = _oracle_timer("--workload", w.name, "--budget", budget_s,
                      *(("--seed", seed) if seed is not None else ()))
    return {"value": r["token_heads_per_s"] / w.H, "unit": "tokens/s", "cores": r["cores"],
            "host_cores_available": r["host_cores_available"], "kind": "oracle",
            "sample": f"{r['sequences']} whole (batch, head) sequences of L={w.L} (fp64 NumPy "
                      f"forward + backward, one process per core), {r['seconds']:.1f} s; tokens/s "
                      f"counts a token of all H={w.H} heads, i.e. token-heads / {w.H}"}


# ------------------------------------------------------ reference arm -----
def run_reference(args, rank, world):
    """The oracle as it stands, timed on the host cores over bounded samples
    of the same workload (rank 0 only): every step runs one (batch, head)
    sequence's first 256 tokens on each core."""
    if rank != 0:
        return
    from gated_linear_sliding_chunkwise_b200.synth import WORKLOADS

    w = WORKLOADS["train_step"]
    L = 256
    r = _oracle_timer("--workload", w.name, "--tokens", L, "--steps", args.steps,
                      "--warmup", args.warmup)
    value = r["token_heads_per_s"] / w.H
    sample = (f"each step: {r['cores']} (batch, head) sequences of the train_step workload, one per "
              f"host core, first {L} tokens each, fp64 NumPy forward + backward; tokens/s counts a "
              f"token of all H={w.H} heads")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": r["sec_per_step"] * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": DATA,
            "config": train_config(w, world, args.kernels),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": r["cores"],
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--kernels", choices=["auto", "simt", "tc"], default="auto",
                    help="kernel family inside the library")
    ap.add_argument("--decode-steps", type=int, default=1000)
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--no-fwd-long", action="store_true")
    ap.add_argument("--no-fwd-layer", action="store_true",
                    help="skip the Llama-3-8B-shaped layer forward (B=4 H=32 L=2048)")
    ap.add_argument("--no-variants", action="store_true",
                    help="skip the stage-1 step and scalar-gate timings")
    ap.add_argument("--only", choices=["train", "fwd", "bwd", "decode"], default="train",
                    help="fwd / bwd / decode: time one entry point alone (profiling aid)")
    ap.add_argument("--decode-batch", type=int, default=None,
                    help="with --only decode: batch size in place of the workload's 64")
    ap.add_argument("--workload", default="llama8b_layer_fwd")
    args = ap.parse_args(argv)
    if args.warmup < 3 and args.impl == "ours":
        print("note: --warmup below 3 is not a valid measurement", file=sys.stderr)
    rank, world, local = dist_env()
    if args.only == "decode":
        from gated_linear_sliding_chunkwise_b200 import lizard as lz
        dev = torch.device("cuda", local)
        torch.cuda.set_device(dev)
        print(json.dumps(run_decode(args, lz, dev, rank, 1, load_peaks())))
        return
    if args.only in ("fwd", "bwd"):
        # one entry point alone on one workload (used for kernel profiles)
        from gated_linear_sliding_chunkwise_b200 import lizard as lz
        dev = torch.device("cuda", local)
        torch.cuda.set_device(dev)
        fn = run_forward if args.only == "fwd" else run_backward
        print(json.dumps(fn(args, lz, dev, rank, 1, load_peaks(), args.workload, args.steps)))
        return
    if world > 1:
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    try:
        if args.impl == "reference":
            run_reference(args, rank, world)
        else:
            run_ours(args, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
