"""Thin ctypes binding of liblizard.so (see include/lizard.h).

Argument marshalling only: every step of the layer runs in the library's
CUDA kernels.  PyTorch supplies device memory (outputs and workspaces are
allocated here with torch) and the current CUDA stream.  Importing this
module loads the library and raises ``ImportError`` if it is missing; there
is no fallback.
"""

from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblizard.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with "
        "`python -m gated_linear_sliding_chunkwise_b200.build` (nvcc, sm_100a)")
_lib = ctypes.CDLL(LIB_PATH)

# ---------------------------------------------------------------- codes ---
OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT, ERR_WORKSPACE, ERR_RANGE = range(7)
BF16, FP32 = 0, 1
BRANCH_BOTH, BRANCH_GLA_ONLY, BRANCH_SWA_ONLY = 0, 1, 2
IMPL_AUTO, IMPL_SIMT, IMPL_TC = 0, 1, 2
GATE_PER_DIM, GATE_SCALAR = 0, 1

_vp = ctypes.c_void_p
_i32 = ctypes.c_int32
_f32 = ctypes.c_float


class FwdArgs(ctypes.Structure):
    _fields_ = [("B", _i32), ("H", _i32), ("L", _i32), ("dk", _i32), ("dv", _i32),
                ("chunk", _i32), ("window", _i32), ("M", _i32), ("dtype", _i32),
                ("branch", _i32), ("impl", _i32), ("gate", _i32), ("gate_temp", _f32),
                ("softmax_scale", _f32),
                ("q", _vp), ("k", _vp), ("v", _vp), ("g", _vp),
                ("fmap_wq", _vp), ("fmap_wk", _vp), ("meta_k", _vp), ("meta_v", _vp),
                ("alpha", _vp), ("state_in", _vp), ("o", _vp), ("state_out", _vp),
                ("lse", _vp), ("workspace", _vp), ("workspace_bytes", ctypes.c_size_t),
                ("launch_events", ctypes.POINTER(_vp)), ("n_launch_events", _i32),
                ("k_prefix", _vp), ("v_prefix", _vp), ("prefix_len", _i32),
                ("saved", _vp), ("saved_bytes", ctypes.c_size_t)]


class BwdArgs(ctypes.Structure):
    _fields_ = [("fwd", FwdArgs), ("dout", _vp), ("dq", _vp), ("dk", _vp), ("dv", _vp),
                ("dg", _vp), ("dmeta_k", _vp), ("dmeta_v", _vp), ("dfmap_wq", _vp),
                ("dfmap_wk", _vp), ("dalpha", _vp), ("dstate_in", _vp), ("impl", _i32),
                ("workspace", _vp), ("workspace_bytes", ctypes.c_size_t),
                ("launch_events", ctypes.POINTER(_vp)), ("n_launch_events", _i32),
                ("dstate_out", _vp), ("dk_prefix", _vp), ("dv_prefix", _vp)]


class DecodeArgs(ctypes.Structure):
    _fields_ = [("B", _i32), ("H", _i32), ("dk", _i32), ("dv", _i32), ("window", _i32),
                ("M", _i32), ("dtype", _i32), ("gate", _i32), ("gate_temp", _f32),
                ("softmax_scale", _f32),
                ("q", _vp), ("k", _vp), ("v", _vp), ("g", _vp), ("state", _vp),
                ("k_cache", _vp), ("v_cache", _vp), ("pos", _vp),
                ("fmap_wq", _vp), ("fmap_wk", _vp), ("meta_k", _vp), ("meta_v", _vp),
                ("alpha", _vp), ("o", _vp)]


class Stage1Args(ctypes.Structure):
    _fields_ = [("bwd", BwdArgs), ("target", _vp), ("loss", _vp)]


_lib.lizard_fwd_workspace_size.argtypes = [ctypes.POINTER(FwdArgs)]
_lib.lizard_fwd_workspace_size.restype = ctypes.c_size_t
_lib.lizard_attn_fwd.argtypes = [ctypes.POINTER(FwdArgs), _vp]
_lib.lizard_attn_fwd.restype = ctypes.c_int
_lib.lizard_fwd_saved_size.argtypes = [ctypes.POINTER(FwdArgs)]
_lib.lizard_fwd_saved_size.restype = ctypes.c_size_t
_lib.lizard_bwd_workspace_size.argtypes = [ctypes.POINTER(BwdArgs)]
_lib.lizard_bwd_workspace_size.restype = ctypes.c_size_t
_lib.lizard_attn_bwd.argtypes = [ctypes.POINTER(BwdArgs), _vp]
_lib.lizard_attn_bwd.restype = ctypes.c_int
_lib.lizard_fwd_launch_plan.argtypes = [ctypes.POINTER(FwdArgs), ctypes.POINTER(ctypes.c_char_p), _i32]
_lib.lizard_fwd_launch_plan.restype = _i32
_lib.lizard_bwd_launch_plan.argtypes = [ctypes.POINTER(BwdArgs), ctypes.POINTER(ctypes.c_char_p), _i32]
_lib.lizard_bwd_launch_plan.restype = _i32
_lib.lizard_stage1_workspace_size.argtypes = [ctypes.POINTER(Stage1Args)]
_lib.lizard_stage1_workspace_size.restype = ctypes.c_size_t
_lib.lizard_stage1_step.argtypes = [ctypes.POINTER(Stage1Args), _vp]
_lib.lizard_stage1_step.restype = ctypes.c_int
_lib.lizard_stage1_launch_plan.argtypes = [ctypes.POINTER(Stage1Args), ctypes.POINTER(ctypes.c_char_p), _i32]
_lib.lizard_stage1_launch_plan.restype = _i32
_lib.lizard_decode_step.argtypes = [ctypes.POINTER(DecodeArgs), _vp]
_lib.lizard_decode_step.restype = ctypes.c_int
class CacheArgs(ctypes.Structure):
    _fields_ = [("B", _i32), ("H", _i32), ("L", _i32), ("dk", _i32), ("dv", _i32), ("window", _i32),
                ("dtype", _i32), ("k", _vp), ("v", _vp), ("k_cache", _vp), ("v_cache", _vp),
                ("pos", _vp)]


class ChainArgs(ctypes.Structure):
    _fields_ = [("B", _i32), ("H", _i32), ("dk", _i32), ("dv", _i32), ("nseg", _i32), ("rank", _i32),
                ("seg_state", _vp), ("seg_log_decay", _vp), ("state_in", _vp), ("state_out", _vp)]


_lib.lizard_segment_state_workspace_size.argtypes = [ctypes.POINTER(FwdArgs)]
_lib.lizard_segment_state_workspace_size.restype = ctypes.c_size_t
_lib.lizard_segment_state.argtypes = [ctypes.POINTER(FwdArgs), _vp, _vp]
_lib.lizard_segment_state.restype = ctypes.c_int
_lib.lizard_chain_states.argtypes = [ctypes.POINTER(ChainArgs), _vp]
_lib.lizard_chain_states.restype = ctypes.c_int
_lib.lizard_prefill_cache.argtypes = [ctypes.POINTER(CacheArgs), _vp]
_lib.lizard_prefill_cache.restype = ctypes.c_int
_lib.lizard_decode_status.argtypes = []
_lib.lizard_decode_status.restype = ctypes.c_int
_lib.lizard_workspace_status.argtypes = [_vp, _vp]
_lib.lizard_workspace_status.restype = ctypes.c_int
_lib.lizard_attn_fwd_noalloc.argtypes = [ctypes.POINTER(FwdArgs), _vp]
_lib.lizard_attn_fwd_noalloc.restype = ctypes.c_int
_lib.lizard_noalloc_status.argtypes = [_vp]
_lib.lizard_noalloc_status.restype = ctypes.c_int
_lib.lizard_status_string.argtypes = [ctypes.c_int]
_lib.lizard_status_string.restype = ctypes.c_char_p
_lib.lizard_debug_inject_wait_timeout.argtypes = [_i32]
_lib.lizard_debug_inject_wait_timeout.restype = None
_lib.lizard_version.argtypes = []
_lib.lizard_version.restype = ctypes.c_char_p


class LizardError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {status_string(code)} (status {code})")


def status_string(code: int) -> str:
    return _lib.lizard_status_string(code).decode()


def version() -> str:
    return _lib.lizard_version().decode()


def debug_inject_wait_timeout(count: int) -> None:
    """Test hook: the next `count` tensor-core forward full passes wait on a
    barrier that nothing completes and report LIZARD_ERR_TIMEOUT."""
    _lib.lizard_debug_inject_wait_timeout(int(count))


def lib() -> ctypes.CDLL:
    return _lib


# ------------------------------------------------------------- helpers ----
def _ptr(t):
    return None if t is None else t.data_ptr()


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return FP32
    raise TypeError(f"activations must be bf16 or fp32, got {t.dtype}")


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _check(code: int, where: str):
    if code != OK:
        raise LizardError(code, where)


def _gate_code(q, g):
    """The gate granularity from g's shape: the shape of q (one logit per key
    dimension) or q's without the last axis (one scalar logit per token and
    head)."""
    if g is None or tuple(g.shape) == tuple(q.shape):
        return GATE_PER_DIM
    if tuple(g.shape) == tuple(q.shape[:-1]):
        return GATE_SCALAR
    raise ValueError(f"gate logits of shape {tuple(g.shape)} fit neither {tuple(q.shape)} "
                     f"nor {tuple(q.shape[:-1])}")


def _fwd_struct(q, k, v, g, *, window, chunk, gate_temp, softmax_scale, fmap_wq,
                fmap_wk, meta_k, meta_v, alpha, state_in, branch, impl):
    B, H, L, dk = q.shape
    a = FwdArgs()
    a.gate = _gate_code(q, g)
    a.B, a.H, a.L, a.dk, a.dv = B, H, L, dk, v.shape[-1]
    a.chunk, a.window = chunk, window
    a.M = 0 if meta_k is None else meta_k.shape[1]
    a.dtype = _dtype_code(q)
    a.branch, a.impl = branch, impl
    a.gate_temp, a.softmax_scale = gate_temp, softmax_scale
    a.q, a.k, a.v, a.g = _ptr(q), _ptr(k), _ptr(v), _ptr(g)
    a.fmap_wq, a.fmap_wk = _ptr(fmap_wq), _ptr(fmap_wk)
    a.meta_k, a.meta_v = _ptr(meta_k), _ptr(meta_v)
    a.alpha, a.state_in = _ptr(alpha), _ptr(state_in)
    return a


def fwd_workspace_bytes(args: FwdArgs) -> int:
    return int(_lib.lizard_fwd_workspace_size(ctypes.byref(args)))


def fwd_saved_bytes(args: FwdArgs) -> int:
    """Bytes of the training forward's saved-for-backward buffer (0: none)."""
    return int(_lib.lizard_fwd_saved_size(ctypes.byref(args)))


def _attach_saved(args: FwdArgs, saved):
    """Point the struct at a saved-for-backward buffer (a uint8 tensor)."""
    if saved is None:
        args.saved, args.saved_bytes = None, 0
    else:
        args.saved, args.saved_bytes = saved.data_ptr(), saved.numel() * saved.element_size()


def bwd_workspace_bytes(args: BwdArgs) -> int:
    return int(_lib.lizard_bwd_workspace_size(ctypes.byref(args)))


def _workspace(nbytes, device, workspace):
    if workspace is not None:
        assert workspace.numel() * workspace.element_size() >= nbytes, "workspace too small"
        return workspace
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


def _plan(fn, args):
    names = (ctypes.c_char_p * 16)()
    n = fn(ctypes.byref(args), names, 16)
    if n < 0:
        raise LizardError(ERR_INVALID_ARG, "launch plan")
    return [names[i].decode() for i in range(min(n, 16))]


def _attach_events(args, events):
    """Point the struct at raw cudaEvent_t handles of torch events."""
    if not events:
        args.launch_events, args.n_launch_events = None, 0
        return None
    arr = (_vp * len(events))()
    for i, ev in enumerate(events):
        arr[i] = ev.cuda_event
    args.launch_events = ctypes.cast(arr, ctypes.POINTER(_vp))
    args.n_launch_events = len(events)
    return arr


def make_events(n):
    """n timing events whose CUDA handles exist (torch creates them lazily)."""
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
    for ev in evs:
        ev.record()
    torch.cuda.synchronize()
    return evs


# ----------------------------------------------------------------- API ----
def attn_fwd(q, k, v, g, *, window, chunk=64, gate_temp=16.0, softmax_scale=0.0,
             fmap_wq=None, fmap_wk=None, meta_k=None, meta_v=None, alpha=None,
             state_in=None, want_state=False, want_lse=False,
             branch=BRANCH_BOTH, impl=IMPL_AUTO, out=None, workspace=None, stream=None,
             events=None, plan_only=False, k_prefix=None, v_prefix=None, saved=None):
    """Forward of the hybrid layer (lizard_attn_fwd).  Tensors on one CUDA
    device, contiguous; returns a dict with o, state_out, lse.  `events`
    (torch.cuda.Event list) are recorded around each kernel; plan_only returns
    the kernel names without launching.  k_prefix, v_prefix [B, H, P, d]: the
    P <= window tokens before token 0, seen by the anchor window.  saved: a
    uint8 device tensor of at least fwd_saved_bytes() bytes, or True to
    allocate one, into which a training forward writes what attn_bwd(...,
    saved=) reads instead of recomputing (returned as "saved"; None when the
    forward keeps nothing for these arguments)."""
    a = _fwd_struct(q, k, v, g, window=window, chunk=chunk, gate_temp=gate_temp,
                    softmax_scale=softmax_scale, fmap_wq=fmap_wq, fmap_wk=fmap_wk,
                    meta_k=meta_k, meta_v=meta_v, alpha=alpha, state_in=state_in,
                    branch=branch, impl=impl)
    if (k_prefix is None) != (v_prefix is None):
        raise ValueError("k_prefix and v_prefix go together")
    if k_prefix is not None:
        a.k_prefix, a.v_prefix, a.prefix_len = _ptr(k_prefix), _ptr(v_prefix), k_prefix.shape[2]
    B, H, L, dk = q.shape
    dv = v.shape[-1]
    o = torch.empty(B, H, L, dv, dtype=q.dtype, device=q.device) if out is None else out
    S = torch.empty(B, H, dk, dv, dtype=torch.float32, device=q.device) if want_state else None
    lse = torch.empty(B, H, L, dtype=torch.float32, device=q.device) if want_lse else None
    a.o, a.state_out, a.lse = _ptr(o), _ptr(S), _ptr(lse)
    nbytes = fwd_workspace_bytes(a)
    ws = _workspace(nbytes, q.device, workspace)
    a.workspace, a.workspace_bytes = ws.data_ptr(), ws.numel() * ws.element_size()
    if saved is True:
        n = fwd_saved_bytes(a)
        saved = torch.empty(n, dtype=torch.uint8, device=q.device) if n > 0 else None
    _attach_saved(a, saved)
    if plan_only:
        return _plan(_lib.lizard_fwd_launch_plan, a)
    keep = _attach_events(a, events)
    _check(_lib.lizard_attn_fwd(ctypes.byref(a), _stream(stream)), "lizard_attn_fwd")
    del keep
    return {"o": o, "state_out": S, "lse": lse, "workspace": ws, "saved": saved}


def _bwd_struct(f, q, k, v, g, dout, *, meta_k, meta_v, fmap_wq, fmap_wk, impl, want_dstate):
    """Gradient buffers and the lizard_bwd_args that point at them."""
    B, H, L, dk = q.shape
    dv_ = v.shape[-1]
    dev = q.device
    f32 = torch.float32
    res = {
        "dq": torch.empty_like(q), "dk": torch.empty_like(k), "dv": torch.empty_like(v),
        "dg": torch.empty(g.shape if g is not None else (B, H, L, dk), dtype=f32, device=dev),
        "dmeta_k": None if meta_k is None else torch.empty_like(meta_k),
        "dmeta_v": None if meta_v is None else torch.empty_like(meta_v),
        "dfmap_wq": None if fmap_wq is None else torch.empty_like(fmap_wq),
        "dfmap_wk": None if fmap_wk is None else torch.empty_like(fmap_wk),
        "dalpha": torch.empty(H, dtype=f32, device=dev),
        "dstate_in": torch.empty(B, H, dk, dv_, dtype=f32, device=dev) if want_dstate else None,
    }
    b = BwdArgs()
    b.fwd = f
    b.dout = _ptr(dout)
    for name in ("dq", "dk", "dv", "dg", "dmeta_k", "dmeta_v", "dfmap_wq", "dfmap_wk",
                 "dalpha", "dstate_in"):
        setattr(b, name, _ptr(res[name]))
    b.impl = impl
    return b, res


def attn_bwd(q, k, v, g, dout, *, window, chunk=64, gate_temp=16.0, softmax_scale=0.0,
             fmap_wq=None, fmap_wk=None, meta_k=None, meta_v=None, alpha=None,
             state_in=None, branch=BRANCH_BOTH, impl=IMPL_AUTO, want_dstate=True,
             workspace=None, stream=None, events=None, plan_only=False, dstate_out=None,
             k_prefix=None, v_prefix=None, saved=None):
    """Backward of the hybrid layer (lizard_attn_bwd); returns every gradient.
    dstate_out [B, H, dk, dv] fp32: gradient flowing into the final state
    (None: the final state is unused).  k_prefix, v_prefix [B, H, P, d]: the
    anchor window's prefix, as in attn_fwd; their gradients come back as
    dk_prefix, dv_prefix.  saved: the buffer attn_fwd(..., saved=) filled for
    the same inputs (None: recompute)."""
    f = _fwd_struct(q, k, v, g, window=window, chunk=chunk, gate_temp=gate_temp,
                    softmax_scale=softmax_scale, fmap_wq=fmap_wq, fmap_wk=fmap_wk,
                    meta_k=meta_k, meta_v=meta_v, alpha=alpha, state_in=state_in,
                    branch=branch, impl=impl)
    if (k_prefix is None) != (v_prefix is None):
        raise ValueError("k_prefix and v_prefix go together")
    b, res = _bwd_struct(f, q, k, v, g, dout, meta_k=meta_k, meta_v=meta_v, fmap_wq=fmap_wq,
                         fmap_wk=fmap_wk, impl=impl, want_dstate=want_dstate)
    b.dstate_out = _ptr(dstate_out)
    _attach_saved(b.fwd, saved)
    res["dk_prefix"] = res["dv_prefix"] = None
    if k_prefix is not None:
        b.fwd.k_prefix, b.fwd.v_prefix = _ptr(k_prefix), _ptr(v_prefix)
        b.fwd.prefix_len = k_prefix.shape[2]
        res["dk_prefix"] = torch.empty_like(k_prefix)
        res["dv_prefix"] = torch.empty_like(v_prefix)
        b.dk_prefix, b.dv_prefix = _ptr(res["dk_prefix"]), _ptr(res["dv_prefix"])
    dev = q.device
    nbytes = bwd_workspace_bytes(b)
    ws = _workspace(nbytes, dev, workspace)
    b.workspace, b.workspace_bytes = ws.data_ptr(), ws.numel() * ws.element_size()
    if plan_only:
        return _plan(_lib.lizard_bwd_launch_plan, b)
    keep = _attach_events(b, events)
    _check(_lib.lizard_attn_bwd(ctypes.byref(b), _stream(stream)), "lizard_attn_bwd")
    del keep
    res["workspace"] = ws
    return res


def stage1_step(q, k, v, g, target, *, window, chunk=64, gate_temp=16.0, softmax_scale=0.0,
                fmap_wq=None, fmap_wk=None, meta_k=None, meta_v=None, alpha=None,
                state_in=None, branch=BRANCH_BOTH, impl=IMPL_AUTO, want_o=False,
                want_dstate=True, workspace=None, stream=None, events=None, plan_only=False):
    """One stage-1 training step (lizard_stage1_step): forward, the mean squared
    error against the teacher output `target`, and every gradient of it.
    Returns the gradients plus "loss" (a one-element fp32 tensor) and "o"
    (when want_o)."""
    f = _fwd_struct(q, k, v, g, window=window, chunk=chunk, gate_temp=gate_temp,
                    softmax_scale=softmax_scale, fmap_wq=fmap_wq, fmap_wk=fmap_wk,
                    meta_k=meta_k, meta_v=meta_v, alpha=alpha, state_in=state_in,
                    branch=branch, impl=impl)
    o = torch.empty(*q.shape[:-1], v.shape[-1], dtype=q.dtype, device=q.device) if want_o else None
    f.o = _ptr(o)
    b, res = _bwd_struct(f, q, k, v, g, None, meta_k=meta_k, meta_v=meta_v, fmap_wq=fmap_wq,
                         fmap_wk=fmap_wk, impl=impl, want_dstate=want_dstate)
    loss = torch.zeros(1, dtype=torch.float32, device=q.device)
    a = Stage1Args()
    a.bwd = b
    a.target, a.loss = _ptr(target), _ptr(loss)
    nbytes = int(_lib.lizard_stage1_workspace_size(ctypes.byref(a)))
    ws = _workspace(nbytes, q.device, workspace)
    a.bwd.workspace, a.bwd.workspace_bytes = ws.data_ptr(), ws.numel() * ws.element_size()
    if plan_only:
        return _plan(_lib.lizard_stage1_launch_plan, a)
    keep = _attach_events(a.bwd, events)
    _check(_lib.lizard_stage1_step(ctypes.byref(a), _stream(stream)), "lizard_stage1_step")
    del keep
    res.update(loss=loss, o=o, workspace=ws)
    return res


def decode_step(q, k, v, g, state, k_cache, v_cache, pos, *, gate_temp=16.0,
                softmax_scale=0.0, fmap_wq=None, fmap_wk=None, meta_k=None,
                meta_v=None, alpha=None, out=None, stream=None):
    """One decode step (lizard_decode_step).  state, k_cache, v_cache and pos
    are updated in place; returns o [B, H, dv]."""
    B, H, dk = q.shape
    a = DecodeArgs()
    a.B, a.H, a.dk, a.dv = B, H, dk, v.shape[-1]
    a.window = k_cache.shape[2]
    a.M = 0 if meta_k is None else meta_k.shape[1]
    a.dtype = _dtype_code(q)
    a.gate = _gate_code(q, g)
    a.gate_temp, a.softmax_scale = gate_temp, softmax_scale
    a.q, a.k, a.v, a.g = _ptr(q), _ptr(k), _ptr(v), _ptr(g)
    a.state, a.k_cache, a.v_cache, a.pos = _ptr(state), _ptr(k_cache), _ptr(v_cache), _ptr(pos)
    a.fmap_wq, a.fmap_wk = _ptr(fmap_wq), _ptr(fmap_wk)
    a.meta_k, a.meta_v, a.alpha = _ptr(meta_k), _ptr(meta_v), _ptr(alpha)
    o = torch.empty(B, H, a.dv, dtype=q.dtype, device=q.device) if out is None else out
    a.o = _ptr(o)
    _check(_lib.lizard_decode_step(ctypes.byref(a), _stream(stream)), "lizard_decode_step")
    return o


def workspace_status(workspace, stream=None) -> int:
    """Status word left in a workspace by kernels with bounded waits."""
    return int(_lib.lizard_workspace_status(workspace.data_ptr(), _stream(stream)))


def noalloc_status(stream=None) -> int:
    """Status word of the last lizard_attn_fwd_noalloc call on the current
    device (it lives in the library's built-in scratch); reading clears it."""
    return int(_lib.lizard_noalloc_status(_stream(stream)))


def decode_status() -> int:
    """Timeout flag of the decode steps run on the current device since the
    last call (OK or ERR_TIMEOUT); reading clears it and synchronises."""
    return int(_lib.lizard_decode_status())


def prefill_cache(k, v, k_cache, v_cache, pos, stream=None):
    """Prefill -> decode handoff (lizard_prefill_cache): fill the window
    caches from the prefix keys and values k, v [B, H, L, d] and set
    pos = L, in place."""
    B, H, L, dk = k.shape
    a = CacheArgs()
    a.B, a.H, a.L, a.dk, a.dv, a.window = B, H, L, dk, v.shape[-1], k_cache.shape[2]
    a.dtype = _dtype_code(k)
    a.k, a.v = _ptr(k), _ptr(v)
    a.k_cache, a.v_cache, a.pos = _ptr(k_cache), _ptr(v_cache), _ptr(pos)
    _check(_lib.lizard_prefill_cache(ctypes.byref(a), _stream(stream)), "lizard_prefill_cache")


# ------------------------------------------------- sequence parallelism ---
def segment_state(k, v, g, *, window, chunk=64, gate_temp=16.0, fmap_wk=None, impl=IMPL_AUTO,
                  workspace=None, stream=None):
    """(U, R) of one segment (lizard_segment_state): U [B, H, dk, dv] fp32 the
    GLA state after the segment's tokens from a zero start, R [B, H, dk] fp32
    the summed log-decay; a start state S ends the segment as
    diag(exp R) S + U."""
    a = _fwd_struct(k, k, v, g, window=window, chunk=chunk, gate_temp=gate_temp,
                    softmax_scale=0.0, fmap_wq=None, fmap_wk=fmap_wk, meta_k=None, meta_v=None,
                    alpha=None, state_in=None, branch=BRANCH_GLA_ONLY, impl=impl)
    a.q = None
    B, H, _, dk = k.shape
    U = torch.empty(B, H, dk, v.shape[-1], dtype=torch.float32, device=k.device)
    R = torch.empty(B, H, dk, dtype=torch.float32, device=k.device)
    a.state_out = _ptr(U)
    ws = _workspace(int(_lib.lizard_segment_state_workspace_size(ctypes.byref(a))), k.device, workspace)
    a.workspace, a.workspace_bytes = ws.data_ptr(), ws.numel() * ws.element_size()
    _check(_lib.lizard_segment_state(ctypes.byref(a), _ptr(R), _stream(stream)), "lizard_segment_state")
    return U, R, ws


def chain_states(seg_state, seg_log_decay, rank, *, state_in=None, out=None, stream=None):
    """Start state of segment `rank` (lizard_chain_states) from the gathered
    summaries seg_state [nseg, B, H, dk, dv] and seg_log_decay [nseg, B, H, dk]."""
    nseg, B, H, dk, dv = seg_state.shape
    S = torch.empty(B, H, dk, dv, dtype=torch.float32, device=seg_state.device) if out is None else out
    a = ChainArgs(B, H, dk, dv, nseg, rank, _ptr(seg_state), _ptr(seg_log_decay), _ptr(state_in), _ptr(S))
    _check(_lib.lizard_chain_states(ctypes.byref(a), _stream(stream)), "lizard_chain_states")
    return S
