"""lizard_attn_fwd_noalloc: the forward for callers that cannot allocate.

Some callers cannot hand the library a device workspace (a plug-in whose
host application owns all device memory, a client with a fixed device budget
that must not grow).  For them the library keeps the forward's scratch in a
static device array.  These tests call that entry point through the C ABI and
compare it with the regular lizard_attn_fwd, which takes a caller workspace.

This file is collected last on purpose, so that a run that stops at the first
failure has run every other test before it.
"""

import ctypes

import pytest
import torch

from gated_linear_sliding_chunkwise_b200.synth import Workload, make_inputs, random_alpha
from lizard_testutil import check, oracle_forward, to64


@pytest.fixture(scope="module")
def lz():
    from gated_linear_sliding_chunkwise_b200 import build
    build.build()
    from gated_linear_sliding_chunkwise_b200 import lizard
    return lizard


def _args(lz, x, w, o):
    a = lz.FwdArgs()
    B, H, L, d = x["q"].shape
    a.B, a.H, a.L, a.dk, a.dv = B, H, L, d, d
    a.chunk, a.window, a.M = w.chunk, w.window, x["meta_k"].shape[1]
    a.dtype = lz.BF16 if x["q"].dtype == torch.bfloat16 else lz.FP32
    a.branch, a.impl = lz.BRANCH_BOTH, lz.IMPL_AUTO
    a.gate_temp, a.softmax_scale = w.gate_temp, 0.0
    for n in ("q", "k", "v", "g", "fmap_wq", "fmap_wk", "meta_k", "meta_v", "alpha"):
        setattr(a, n, x[n].data_ptr())
    a.o = o.data_ptr()
    return a


def test_noalloc_rejects_sizes_beyond_its_scratch(lz):
    """A forward that needs more than the built-in scratch is refused before
    anything runs (host-side check, no GPU needed)."""
    a = lz.FwdArgs()
    a.B, a.H, a.L, a.dk, a.dv, a.chunk, a.window, a.M = 8, 32, 2048, 128, 128, 64, 128, 0
    a.dtype, a.gate_temp = lz.BF16, 16.0
    a.impl = lz.IMPL_SIMT     # the portable kernels keep fp32 scratch per token
    fake = 0x10000
    a.q = a.k = a.v = a.g = a.o = fake
    assert lz.fwd_workspace_bytes(a) > 32 << 20
    assert lz.lib().lizard_attn_fwd_noalloc(ctypes.byref(a), None) == lz.ERR_UNSUPPORTED
    a.dk = a.dv = 96   # invalid sizes still get the regular error
    assert lz.lib().lizard_attn_fwd_noalloc(ctypes.byref(a), None) == lz.ERR_UNSUPPORTED
    assert lz.lib().lizard_attn_fwd_noalloc(None, None) == lz.ERR_INVALID_ARG


def _case(lz, L, seed):
    w = Workload("noalloc", B=2, H=4, L=L, d=128, dtype="bf16", seed=seed)
    inp = make_inputs(w)
    inp["alpha"] = random_alpha(4, seed=seed)
    x = {k: v.cuda().contiguous() for k, v in inp.items()}
    return w, inp, x


def _regular(lz, x, w):
    return lz.attn_fwd(x["q"], x["k"], x["v"], x["g"], window=w.window, chunk=w.chunk,
                       gate_temp=w.gate_temp, fmap_wq=x["fmap_wq"], fmap_wk=x["fmap_wk"],
                       meta_k=x["meta_k"], meta_v=x["meta_v"], alpha=x["alpha"])["o"]


@pytest.mark.gpu
def test_noalloc_matches_regular_forward_twice(lz):
    """Two calls in a row with different inputs and lengths: each output
    equals the regular forward's within the bf16 parity tolerance, and the
    oracle's too; the status word of the built-in scratch reads OK."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    stream = torch.cuda.current_stream().cuda_stream
    for call, (L, seed) in enumerate([(300, 5), (173, 6)]):
        w, inp, x = _case(lz, L, seed)
        want = _regular(lz, x, w)
        o = torch.full_like(want, float("nan"))
        a = _args(lz, x, w, o)
        assert lz.fwd_workspace_bytes(a) <= 32 << 20
        assert lz.lib().lizard_attn_fwd_noalloc(ctypes.byref(a), stream) == lz.OK
        torch.cuda.synchronize()
        check(f"noalloc call {call} vs regular", o, to64(want), "bf16")
        ref = oracle_forward(inp, window=w.window, tau=w.gate_temp)
        check(f"noalloc call {call} vs oracle", o, ref["o"], "bf16")
        assert lz.noalloc_status(stream) == lz.OK


@pytest.mark.gpu
def test_noalloc_reports_a_device_error_then_computes(lz):
    """A bounded wait made to run out (host-side test hook) is reported by
    lizard_noalloc_status, which reads the status word in the built-in
    scratch; the next call on the same scratch clears it and computes."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    stream = torch.cuda.current_stream().cuda_stream
    w, inp, x = _case(lz, 260, 8)
    want = _regular(lz, x, w)
    o = torch.zeros_like(want)
    a = _args(lz, x, w, o)
    lz.debug_inject_wait_timeout(1)
    try:
        assert lz.lib().lizard_attn_fwd_noalloc(ctypes.byref(a), stream) == lz.OK
        assert lz.noalloc_status(stream) == lz.ERR_TIMEOUT
    finally:
        lz.debug_inject_wait_timeout(0)
    assert lz.noalloc_status(stream) == lz.OK        # reading cleared it
    assert lz.lib().lizard_attn_fwd_noalloc(ctypes.byref(a), stream) == lz.OK
    assert lz.noalloc_status(stream) == lz.OK
    check("noalloc after a timeout", o, to64(want), "bf16")
