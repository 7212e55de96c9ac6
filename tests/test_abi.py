"""C-ABI checks that need no GPU: the library loads, exports every function
include/lizard.h declares, the ctypes structs match the C layout, and the
host-side argument checks reject bad calls before anything is launched."""

import ctypes
import os
import re
import subprocess

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lizard.h")


@pytest.fixture(scope="module")
def lz():
    from gated_linear_sliding_chunkwise_b200 import build
    build.build()
    from gated_linear_sliding_chunkwise_b200 import lizard
    return lizard


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(lizard_[a-z_]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = _declared_functions()
    for required in ("lizard_attn_fwd", "lizard_attn_bwd", "lizard_decode_step"):
        assert required in names


def test_library_exports_every_declared_function(lz):
    out = subprocess.run(["nm", "-D", "--defined-only", lz.LIB_PATH],
                         capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\bT (lizard_\w+)", out))
    missing = [n for n in _declared_functions() if n not in exported]
    assert not missing, f"not exported: {missing}"
    for n in _declared_functions():
        assert hasattr(lz.lib(), n)


def test_struct_layouts_match_c(lz, tmp_path):
    """Compile a C program against the header and compare sizeof/offsetof."""
    fields = {
        "lizard_fwd_args": lz.FwdArgs, "lizard_bwd_args": lz.BwdArgs,
        "lizard_decode_args": lz.DecodeArgs, "lizard_cache_args": lz.CacheArgs,
        "lizard_stage1_args": lz.Stage1Args, "lizard_chain_args": lz.ChainArgs,
    }
    lines = ["#include <stdio.h>", "#include <stddef.h>", '#include "lizard.h"',
             "int main(void) {"]
    for cname, py in fields.items():
        lines.append(f'printf("{cname} size %zu\\n", sizeof({cname}));')
        for fname, _ in py._fields_:
            lines.append(f'printf("{cname} {fname} %zu\\n", offsetof({cname}, {fname}));')
    lines.append("return 0; }")
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines))
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-std=c11", "-I", os.path.join(ROOT, "include"), str(src),
                    "-o", str(exe)], check=True)
    got = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout
    for line in got.strip().splitlines():
        cname, what, val = line.split()
        py = fields[cname]
        want = ctypes.sizeof(py) if what == "size" else getattr(py, what).offset
        assert int(val) == want, f"{cname}.{what}: C {val} vs ctypes {want}"


def test_status_strings_and_version(lz):
    for code in range(7):
        assert lz.status_string(code)
    assert lz.status_string(99) == "unknown status"
    assert re.match(r"\d+\.\d+\.\d+$", lz.version())


def _fwd(lz, **over):
    a = lz.FwdArgs()
    a.B, a.H, a.L, a.dk, a.dv, a.chunk, a.window, a.M = 1, 2, 128, 64, 64, 64, 16, 4
    a.dtype, a.branch, a.impl = lz.BF16, 0, 0
    a.gate_temp, a.softmax_scale = 16.0, 0.0
    fake = 0x10000   # never dereferenced: every case fails on the host first
    a.q = a.k = a.v = a.g = a.o = fake
    a.meta_k = fake
    for k_, v_ in over.items():
        setattr(a, k_, v_)
    return a


@pytest.mark.parametrize("over,code", [
    ({"dk": 96, "dv": 96}, 2),
    ({"dk": 64, "dv": 128}, 2),
    ({"chunk": 32}, 2),
    ({"M": 17}, 2),
    ({"window": 0}, 1),
    ({"L": -1}, 1),
    ({"B": 0}, 1),
    ({"dtype": 7}, 1),
    ({"branch": 3}, 1),
    ({"gate": 2}, 1),
    ({"gate": -1}, 1),
    ({"gate_temp": 0.0}, 1),
    ({"gate_temp": float("nan")}, 1),
    ({"softmax_scale": -1.0}, 1),
    ({"q": None}, 1),
    ({"g": None}, 1),
    ({"meta_k": None}, 1),            # M > 0 needs meta keys
    ({"M": 0}, 1),                    # meta keys given but M == 0
    ({"q": 0x10004}, 1),              # not 16-byte aligned
    ({"prefix_len": 17, "k_prefix": 0x10000, "v_prefix": 0x10000}, 1),   # prefix longer than the window
    ({"prefix_len": -1}, 1),
    ({"prefix_len": 4}, 1),           # prefix pointers missing
    ({"k_prefix": 0x10000}, 1),       # prefix pointers without a length
    ({"prefix_len": 4, "k_prefix": 0x10000, "v_prefix": 0x10008}, 1),   # misaligned prefix
])
def test_forward_rejects_bad_arguments_on_host(lz, over, code):
    a = _fwd(lz, **over)
    assert lz.lib().lizard_attn_fwd(ctypes.byref(a), None) == code


def test_forward_checks_workspace_before_launch(lz):
    a = _fwd(lz)
    need = lz.fwd_workspace_bytes(a)
    assert need > 0
    a.workspace, a.workspace_bytes = 0x20000, need - 1
    assert lz.lib().lizard_attn_fwd(ctypes.byref(a), None) == lz.ERR_WORKSPACE
    a.workspace, a.workspace_bytes = None, 0
    assert lz.lib().lizard_attn_fwd(ctypes.byref(a), None) == lz.ERR_WORKSPACE
    # the anchor-only test hook needs no GLA scratch
    b = _fwd(lz, branch=lz.BRANCH_SWA_ONLY)
    assert lz.fwd_workspace_bytes(b) < need


def test_workspace_size_rejects_bad_sizes(lz):
    assert lz.fwd_workspace_bytes(_fwd(lz, dk=96, dv=96)) == 0
    assert lz.lib().lizard_fwd_workspace_size(None) == 0


def test_saved_size_and_refusals_on_host(lz):
    """The training forward's saved buffer: its size follows the tensor-core
    GLA path (0 without it), it shrinks the backward's workspace, a buffer
    one byte short is refused by both calls before anything is enqueued, and
    a misaligned one is an invalid argument."""
    w = dict(dk=128, dv=128, window=128, fmap_wq=0x10000, fmap_wk=0x10000)
    a = _fwd(lz, **w)
    need = lz.fwd_saved_bytes(a)
    BH, L, nt = 2, 128, 1
    # marks, tile decays, fp32 factors, bf16 copies + their fp32 row 0, final state, softmax
    # normalisers (256-byte aligned each); the GLA branch alone keeps no normalisers
    up = lambda x: (x + 255) // 256 * 256
    gla = (up(BH * 4) + up(BH * nt * 128 * 4) + up(BH * L * 128 * 4)
           + up(BH * nt * 128 * 128 * 2 + BH * nt * 128 * 4) + up(BH * 128 * 128 * 4))
    assert need == gla + up(BH * L * 4)
    assert lz.fwd_saved_bytes(_fwd(lz, **w, branch=lz.BRANCH_GLA_ONLY)) == gla
    for over in ({"branch": lz.BRANCH_SWA_ONLY}, {"fmap_wq": None, "fmap_wk": None},
                 {"impl": lz.IMPL_SIMT}, {"dk": 64, "dv": 64}, {"L": 0}):
        assert lz.fwd_saved_bytes(_fwd(lz, **{**w, **over})) == 0, over
    assert lz.lib().lizard_fwd_saved_size(None) == 0
    a.workspace, a.workspace_bytes = 0x20000, lz.fwd_workspace_bytes(a)
    a.saved, a.saved_bytes = 0x30000, need - 1
    assert lz.lib().lizard_attn_fwd(ctypes.byref(a), None) == lz.ERR_WORKSPACE
    a.saved = 0x30008
    assert lz.lib().lizard_attn_fwd(ctypes.byref(a), None) == lz.ERR_INVALID_ARG
    b = lz.BwdArgs()
    b.fwd = _fwd(lz, **w)
    fake = 0x10000
    b.dout = b.dq = b.dk = b.dv = b.dg = fake
    plain = lz.bwd_workspace_bytes(b)
    b.fwd.saved, b.fwd.saved_bytes = 0x30000, need - 1
    lean = lz.bwd_workspace_bytes(b)
    assert 0 < lean < plain
    b.workspace, b.workspace_bytes = 0x20000, lean
    assert lz.lib().lizard_attn_bwd(ctypes.byref(b), None) == lz.ERR_WORKSPACE


def test_backward_rejects_bad_arguments_on_host(lz):
    b = lz.BwdArgs()
    b.fwd = _fwd(lz)
    fake = 0x10000
    b.dout = b.dq = b.dk = b.dv = b.dg = fake
    need = lz.bwd_workspace_bytes(b)
    assert need > lz.fwd_workspace_bytes(b.fwd)
    b.workspace, b.workspace_bytes = 0x20000, need - 1
    assert lz.lib().lizard_attn_bwd(ctypes.byref(b), None) == lz.ERR_WORKSPACE
    b.dg = None
    assert lz.lib().lizard_attn_bwd(ctypes.byref(b), None) == lz.ERR_INVALID_ARG
    b.dg = fake
    b.dfmap_wq = fake          # gradient asked for an absent input
    assert lz.lib().lizard_attn_bwd(ctypes.byref(b), None) == lz.ERR_INVALID_ARG
    assert lz.lib().lizard_attn_bwd(None, None) == lz.ERR_INVALID_ARG


def test_decode_rejects_bad_arguments_on_host(lz):
    d = lz.DecodeArgs()
    d.B, d.H, d.dk, d.dv, d.window, d.M, d.dtype = 2, 2, 128, 128, 128, 0, lz.BF16
    d.gate_temp = 16.0
    fake = 0x10000
    for n in ("q", "k", "v", "g", "state", "k_cache", "v_cache", "pos", "o"):
        setattr(d, n, fake)
    d.dk = d.dv = 80
    assert lz.lib().lizard_decode_step(ctypes.byref(d), None) == lz.ERR_UNSUPPORTED
    d.dk = d.dv = 128
    d.window = 20000
    assert lz.lib().lizard_decode_step(ctypes.byref(d), None) == lz.ERR_UNSUPPORTED
    d.window = 128
    d.pos = None
    assert lz.lib().lizard_decode_step(ctypes.byref(d), None) == lz.ERR_INVALID_ARG
    d.pos = fake
    d.gate = 5                 # neither per-dimension nor scalar
    assert lz.lib().lizard_decode_step(ctypes.byref(d), None) == lz.ERR_INVALID_ARG
    d.gate = lz.GATE_SCALAR
    d.M = 2                    # meta tokens without meta keys
    assert lz.lib().lizard_decode_step(ctypes.byref(d), None) == lz.ERR_INVALID_ARG


def test_gate_granularity_follows_the_logits_shape(lz):
    """The binding marks the gate scalar when g lacks q's last axis."""
    q = torch.zeros(2, 3, 5, 8)
    assert lz._gate_code(q, torch.zeros(2, 3, 5, 8)) == lz.GATE_PER_DIM
    assert lz._gate_code(q, torch.zeros(2, 3, 5)) == lz.GATE_SCALAR
    assert lz._gate_code(q, None) == lz.GATE_PER_DIM
    with pytest.raises(ValueError):
        lz._gate_code(q, torch.zeros(2, 3, 8))


def test_prefill_cache_rejects_bad_arguments_on_host(lz):
    a = lz.CacheArgs()
    a.B, a.H, a.L, a.dk, a.dv, a.window, a.dtype = 1, 1, 4, 128, 128, 8, lz.BF16
    assert lz.lib().lizard_prefill_cache(ctypes.byref(a), None) == lz.ERR_INVALID_ARG   # no buffers
    a.dk = a.dv = 96
    assert lz.lib().lizard_prefill_cache(ctypes.byref(a), None) == lz.ERR_UNSUPPORTED


def _stage1(lz, **over):
    a = lz.Stage1Args()
    a.bwd.fwd = _fwd(lz, dk=128, dv=128)
    fake = 0x10000
    a.bwd.dq = a.bwd.dk = a.bwd.dv = a.bwd.dg = fake
    a.target, a.loss = fake, 0x30000
    for k_, v_ in over.items():
        setattr(a, k_, v_)
    return a


def test_stage1_rejects_bad_arguments_on_host(lz):
    a = _stage1(lz)
    need = lz.lib().lizard_stage1_workspace_size(ctypes.byref(a))
    # dL/do lives in the workspace: it outgrows the backward's own
    assert need > lz.bwd_workspace_bytes(a.bwd)
    a.bwd.workspace, a.bwd.workspace_bytes = 0x20000, need - 1
    assert lz.lib().lizard_stage1_step(ctypes.byref(a), None) == lz.ERR_WORKSPACE
    for over in ({"target": None}, {"loss": None}, {"target": 0x10008}):
        b = _stage1(lz, **over)
        assert lz.lib().lizard_stage1_step(ctypes.byref(b), None) == lz.ERR_INVALID_ARG, over
    assert lz.lib().lizard_stage1_step(None, None) == lz.ERR_INVALID_ARG


def test_stage1_launch_plan_fuses_the_loss_on_tensor_cores(lz):
    """The tensor-core forward forms the loss in its epilogue and keeps the
    backward's tensors; the portable forward adds one elementwise kernel
    before the backward."""
    import ctypes as ct
    for impl, fused in ((lz.IMPL_TC, True), (lz.IMPL_SIMT, False)):
        a = _stage1(lz)
        a.bwd.fwd.impl = a.bwd.impl = impl
        a.bwd.fwd.fmap_wq = a.bwd.fwd.fmap_wk = 0x10000
        names = (ct.c_char_p * 24)()
        n = lz.lib().lizard_stage1_launch_plan(ct.byref(a), names, 24)
        got = [names[i].decode() for i in range(n)]
        assert ("mse_kernel" in got) != fused, got
        assert "gate_grad_kernel" in got or "finish_bwd" in got, got
        if fused:   # the backward reads the forward's saved tensors: no second gate or state pass
            assert got.count("gate_prep_kernel") == 1, got
            assert "tc_fwd_kernel(state copies)" not in got, got


# ------------------------------------------------- sequence parallelism ---
def test_prefix_does_not_change_the_workspaces_and_its_gradients_are_outputs(lz):
    """A prefix needs no extra workspace in either direction; the backward
    requires the prefix's gradient outputs with a prefix and refuses them
    without one; the stage-1 step (whole sequences) refuses a prefix."""
    a = _fwd(lz)
    b = _fwd(lz, prefix_len=16, k_prefix=0x10000, v_prefix=0x10000)
    assert lz.fwd_workspace_bytes(b) == lz.fwd_workspace_bytes(a) > 0
    bw = lz.BwdArgs()
    bw.fwd = b
    fake = 0x10000
    bw.dout = bw.dq = bw.dk = bw.dv = bw.dg = fake
    need = lz.bwd_workspace_bytes(bw)
    assert need > 0
    bw0 = lz.BwdArgs()
    bw0.fwd = a
    bw0.dout = bw0.dq = bw0.dk = bw0.dv = bw0.dg = fake
    assert lz.bwd_workspace_bytes(bw0) == need
    bw.workspace, bw.workspace_bytes = 0x20000, need
    # no prefix gradient outputs: refused before anything runs
    assert lz.lib().lizard_attn_bwd(ctypes.byref(bw), None) == lz.ERR_INVALID_ARG
    bw.dk_prefix = fake
    assert lz.lib().lizard_attn_bwd(ctypes.byref(bw), None) == lz.ERR_INVALID_ARG
    bw.dv_prefix = 0x10008          # misaligned
    assert lz.lib().lizard_attn_bwd(ctypes.byref(bw), None) == lz.ERR_INVALID_ARG
    bw0.workspace, bw0.workspace_bytes = 0x20000, need
    bw0.dk_prefix = bw0.dv_prefix = fake   # gradients of a prefix that is not there
    assert lz.lib().lizard_attn_bwd(ctypes.byref(bw0), None) == lz.ERR_INVALID_ARG
    bw.dk_prefix = bw.dv_prefix = None
    s1 = lz.Stage1Args()
    s1.bwd = bw
    s1.target, s1.loss = fake, fake
    s1.bwd.workspace_bytes = 1 << 40
    assert lz.lib().lizard_stage1_step(ctypes.byref(s1), None) == lz.ERR_UNSUPPORTED


def _seg(lz, **over):
    a = _fwd(lz, M=0, meta_k=None)
    a.q = a.o = None            # not read by the summary
    a.state_out = 0x30000
    for k_, v_ in over.items():
        setattr(a, k_, v_)
    return a


@pytest.mark.parametrize("over,code", [
    ({"state_out": None}, 1),
    ({"branch": 2}, 1),                   # the summary is of the GLA branch
    ({"state_in": 0x30000}, 1),           # summaries start from zero
    ({"prefix_len": 4, "k_prefix": 0x10000, "v_prefix": 0x10000}, 1),
    ({"k": None}, 1),
    ({"dk": 96, "dv": 96}, 2),
    ({"impl": 2}, 2),                     # tensor cores need bf16, d = 128 and W_k
])
def test_segment_state_rejects_bad_arguments_on_host(lz, over, code):
    a = _seg(lz, **over)
    a.workspace, a.workspace_bytes = 0x20000, 1 << 40
    assert lz.lib().lizard_segment_state(ctypes.byref(a), 0x40000, None) == code


def test_segment_state_needs_its_outputs_and_workspace(lz):
    a = _seg(lz)
    assert lz.lib().lizard_segment_state(ctypes.byref(a), None, None) == lz.ERR_INVALID_ARG
    assert lz.lib().lizard_segment_state(ctypes.byref(a), 0x40004, None) == lz.ERR_INVALID_ARG
    need = lz.lib().lizard_segment_state_workspace_size(ctypes.byref(a))
    assert need > 0
    a.workspace, a.workspace_bytes = 0x20000, need - 1
    assert lz.lib().lizard_segment_state(ctypes.byref(a), 0x40000, None) == lz.ERR_WORKSPACE
    # the tensor-core summary (bf16, d = 128, W_k) needs only the gate factors
    tc = _seg(lz, dk=128, dv=128, fmap_wk=0x50000)
    simt = _seg(lz, dk=128, dv=128)
    assert 0 < lz.lib().lizard_segment_state_workspace_size(ctypes.byref(tc)) < \
        lz.lib().lizard_segment_state_workspace_size(ctypes.byref(simt))


@pytest.mark.parametrize("over,code", [
    ({"rank": 3}, 1),                     # rank > nseg
    ({"rank": -1}, 1),
    ({"B": 0}, 1),
    ({"seg_state": None}, 1),             # needed for rank > 0
    ({"state_out": None}, 1),
    ({"dk": 96, "dv": 96}, 2),
    ({"seg_log_decay": 0x10004}, 1),
])
def test_chain_rejects_bad_arguments_on_host(lz, over, code):
    a = lz.ChainArgs(1, 2, 64, 64, 2, 1, 0x10000, 0x20000, None, 0x30000)
    for k_, v_ in over.items():
        setattr(a, k_, v_)
    assert lz.lib().lizard_chain_states(ctypes.byref(a), None) == code


def test_backward_checks_the_incoming_state_gradient(lz):
    fake = 0x10000
    for branch, ds, code in [(lz.BRANCH_SWA_ONLY, 0x30000, lz.ERR_INVALID_ARG),   # no final state
                             (lz.BRANCH_BOTH, 0x30004, lz.ERR_INVALID_ARG)]:     # misaligned
        b = lz.BwdArgs()
        b.fwd = _fwd(lz, branch=branch)
        b.dout = b.dq = b.dk = b.dv = b.dg = fake
        b.dstate_out = ds
        b.workspace, b.workspace_bytes = 0x20000, 1 << 40
        assert lz.lib().lizard_attn_bwd(ctypes.byref(b), None) == code


def test_a_plain_c_program_links_and_calls_the_host_entry_points(lz, tmp_path):
    """The boundary is plain C: a C11 program built with gcc against
    include/lizard.h and linked with liblizard.so calls the size queries,
    the launch plan and the argument checks (none of which needs a GPU)."""
    src = tmp_path / "client.c"
    src.write_text(r"""
#include <stdio.h>
#include <string.h>
#include "lizard.h"
int main(void) {
  lizard_fwd_args a;
  memset(&a, 0, sizeof a);
  a.B = 1; a.H = 2; a.L = 300; a.dk = 128; a.dv = 128; a.chunk = 64; a.window = 128; a.M = 0;
  a.dtype = LIZARD_BF16; a.branch = LIZARD_BRANCH_BOTH; a.impl = LIZARD_IMPL_AUTO;
  a.gate = LIZARD_GATE_PER_DIM; a.gate_temp = 16.f;
  size_t ws = lizard_fwd_workspace_size(&a);
  const char *names[16];
  a.q = a.k = a.v = a.g = (const void *)0x10000; a.o = (void *)0x10000;
  a.fmap_wq = a.fmap_wk = (const float *)0x10000;
  int n = lizard_fwd_launch_plan(&a, names, 16);
  lizard_fwd_args bad = a;
  bad.dk = bad.dv = 96;
  lizard_status st = lizard_attn_fwd(&bad, NULL);
  int tc = 0;
  for (int i = 0; i < n && i < 16; ++i) tc |= strcmp(names[i], "tc_fwd_kernel") == 0;
  printf("%zu %d %s %d %s %s\n", ws, n, tc ? "tc_fwd_kernel" : "-", (int)st,
         lizard_status_string(st), lizard_version());
  return 0;
}
""")
    exe = tmp_path / "client"
    libdir = os.path.dirname(lz.LIB_PATH)
    subprocess.run(["gcc", "-std=c11", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
                    "-L", libdir, "-llizard", "-Wl,-rpath," + libdir], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()
    assert int(out[0]) > 0                       # workspace bytes
    assert int(out[1]) >= 1 and out[2] == "tc_fwd_kernel"   # the tensor-core plan has the full pass
    assert int(out[3]) == lz.ERR_UNSUPPORTED     # d = 96 is refused on the host
    assert out[-1] == lz.version()
