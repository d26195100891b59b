"""The C-ABI library: it loads, exports every entry point include/kda.h
declares, and its host-side validation rejects bad arguments before anything
reaches the GPU.  No test here needs a GPU.

The validation tests pass made-up pointer values; they are skipped when a CUDA
device is present so that a validation bug can never send such a pointer to a
kernel (the GPU tests cover the same checks with real buffers).
"""
import ctypes
import os
import re

import pytest
import torch

import gated_delta_rule_157_b200 as kda
from gated_delta_rule_157_b200 import _lib

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                      "include", "kda.h")
OK, INVALID, UNSUPPORTED, ALIGN, ALIAS = 0, 1, 2, 3, 4

no_gpu_only = pytest.mark.skipif(torch.cuda.is_available(),
                                 reason="made-up pointers are only used without a GPU")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kda_\w+)\s*\(", text)))


def test_header_declares_the_three_entry_points():
    names = declared_functions()
    for n in ("kda_chunk_fwd", "kda_step", "kda_compose"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = kda.load()
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(declared_functions()) == set(_lib.EXPORTS)


def test_library_is_in_tree_and_links_no_oracle():
    path = kda.library_path()
    assert os.path.dirname(path) == os.path.dirname(os.path.abspath(kda.__file__))
    blob = open(path, "rb").read()
    assert b"oracle_kda" not in blob


def test_status_strings_and_version():
    assert kda.kda_status_string(0) == "KDA_OK"
    assert kda.kda_status_string(6) == "KDA_ERR_TIMEOUT"
    assert kda.kda_status_string(7) == "KDA_ERR_RANGE"
    assert kda.kda_status_string(99) == "KDA_ERR_UNKNOWN"
    assert kda.kda_version() >= 100


def _chunk_args(**kw):
    a = _lib.ChunkArgs()
    a.B, a.T, a.H, a.HV, a.Dk, a.Dv, a.chunk = 1, 64, 2, 4, 16, 16, 16
    a.dtype, a.algo = 0, 0
    a.g_min, a.scale, a.l2_eps = -5.0, 1.0, 1e-6
    a.qk_l2norm_in_kernel = a.beta_sigmoid_in_kernel = a.gate_in_kernel = 1
    base = 0x7f0000000000
    sizes = {"q": 1 << 20, "k": 2 << 20, "v": 3 << 20, "g": 4 << 20, "beta": 5 << 20,
             "A_log": 6 << 20, "dt_bias": 7 << 20, "S0": 8 << 20, "o": 9 << 20,
             "S_T": 10 << 20, "M_T": 11 << 20}
    for name, off in sizes.items():
        setattr(a, name, base + off)
    a.dt_bias = None
    a.M_T = None
    for key, val in kw.items():
        setattr(a, key, val)
    return a


def _fwd(a):
    return kda.load().kda_chunk_fwd(ctypes.byref(a), None)


def test_null_args_rejected():
    assert kda.load().kda_chunk_fwd(None, None) == INVALID
    assert kda.load().kda_step(None, None) == INVALID


def test_empty_batch_is_a_no_op():
    # B == 0: nothing to do, nothing launched (works without a GPU).
    assert _fwd(_chunk_args(B=0)) == OK


@no_gpu_only
@pytest.mark.parametrize("field,value,expected", [
    ("H", 3, INVALID),            # HV % H != 0
    ("H", 0, INVALID),
    ("Dk", 0, INVALID),
    ("Dk", 129, UNSUPPORTED),
    ("Dv", 256, UNSUPPORTED),
    ("chunk", 0, INVALID),
    ("chunk", 128, UNSUPPORTED),
    ("dtype", 7, INVALID),
    ("algo", 9, INVALID),
    ("T", -1, INVALID),
    ("g_min", 0.5, INVALID),
    ("q", None, INVALID),
    ("A_log", None, INVALID),     # gate_in_kernel needs A_log
    ("q", 0x7f0000100002, ALIGN),  # fp32 needs 4-byte alignment
    ("S0", 0x7f0000800001, ALIGN),
])
def test_chunk_validation(field, value, expected):
    assert _fwd(_chunk_args(**{field: value})) == expected


@no_gpu_only
def test_chunk_aliasing_rejected():
    a = _chunk_args()
    assert _fwd(_chunk_args(o=a.q)) == ALIAS                  # o over an input
    assert _fwd(_chunk_args(o=a.v + 64)) == ALIAS             # partial overlap
    assert _fwd(_chunk_args(S_T=a.o)) == ALIAS
    assert _fwd(_chunk_args(S_T=a.S0 + 4)) == ALIAS           # partial S_T/S0 overlap
    assert _fwd(_chunk_args(M_T=a.S_T)) == ALIAS


@no_gpu_only
def test_chunk_tc_request_on_unsupported_shape():
    # The tensor-core kernel needs bf16, Dk = Dv = 128, chunk = 64.
    assert _fwd(_chunk_args(algo=2)) == UNSUPPORTED


@no_gpu_only
def test_valid_request_without_gpu_reports_cuda_error():
    # Passes validation, so the launch is attempted and fails: no CPU fallback.
    a = _chunk_args(S_T=_chunk_args().S_T)
    assert _fwd(a) == 5
    # o may be NULL (only the states are wanted): still a valid request
    assert _fwd(_chunk_args(o=None)) == 5


def _step_args(**kw):
    a = _lib.StepArgs()
    a.B, a.H, a.HV, a.Dk, a.Dv, a.dtype = 2, 2, 4, 16, 16, 1
    a.g_min, a.scale, a.l2_eps = -5.0, 1.0, 1e-6
    a.qk_l2norm_in_kernel = a.beta_sigmoid_in_kernel = a.gate_in_kernel = 1
    base = 0x7f1000000000
    for i, name in enumerate(["q", "k", "v", "g", "beta", "A_log", "S", "o"]):
        setattr(a, name, base + (i + 1) * (1 << 20))
    a.dt_bias = None
    for key, val in kw.items():
        setattr(a, key, val)
    return a


@no_gpu_only
@pytest.mark.parametrize("field,value,expected", [
    ("Dv", 6, UNSUPPORTED),       # Dv % 4 != 0
    ("Dk", 200, UNSUPPORTED),
    ("HV", 3, INVALID),
    ("S", None, INVALID),
    ("S", 0x7f1000700008, ALIGN),  # state needs 16-byte alignment
    ("q", 0x7f1000100001, ALIGN),  # bf16 needs 2-byte alignment
])
def test_step_validation(field, value, expected):
    assert kda.load().kda_step(ctypes.byref(_step_args(**{field: value})), None) == expected


@no_gpu_only
def test_step_aliasing_rejected():
    a = _step_args()
    assert kda.load().kda_step(ctypes.byref(_step_args(o=a.S + 32)), None) == ALIAS
    assert kda.load().kda_step(ctypes.byref(_step_args(S=a.v)), None) == ALIAS


@no_gpu_only
def test_compose_validation():
    lib = kda.load()
    p = 0x7f2000000000
    assert lib.kda_compose(-1, 1, 8, 8, p, p + (1 << 20), None, p + (2 << 20), None) == INVALID
    assert lib.kda_compose(2, 1, 8, 200, p, p + (1 << 20), None, p + (2 << 20), None) == UNSUPPORTED
    assert lib.kda_compose(2, 1, 8, 8, p, p + (1 << 20), None, None, None) == INVALID
    assert lib.kda_compose(2, 1, 8, 8, p, p + (1 << 20), None, p + 64, None) == ALIAS
    assert lib.kda_compose(0, 0, 8, 8, None, None, None, None, None) == OK


def test_binding_rejects_cpu_tensors():
    x = torch.zeros(1, 4, 1, 16)
    with pytest.raises(ValueError):
        kda.kda_chunk_fwd(x, x, x, x, torch.zeros(1, 4, 1))


# --- layer prologue / epilogue entry points ---------------------------------
def _conv_args(**kw):
    a = _lib.ConvArgs()
    a.B, a.T, a.C, a.K, a.head_dim, a.silu, a.l2_eps = 2, 64, 256, 4, 128, 1, 1e-6
    base = 0x7f0000000000
    a.x, a.w, a.bias = base + (1 << 20), base + (2 << 20), base + (3 << 20)
    a.state_in, a.y, a.state_out = base + (4 << 20), base + (5 << 20), base + (6 << 20)
    for key, val in kw.items():
        setattr(a, key, val)
    return a


def _gate_args(**kw):
    a = _lib.GateArgs()
    a.N, a.HV, a.D, a.eps = 64, 4, 128, 1e-6
    base = 0x7f0000000000
    a.o, a.gate, a.weight, a.y = base + (1 << 20), base + (2 << 20), base + (3 << 20), base + (4 << 20)
    for key, val in kw.items():
        setattr(a, key, val)
    return a


def test_layer_null_and_empty():
    lib = kda.load()
    assert lib.kda_short_conv(None, None) == INVALID
    assert lib.kda_output_gate(None, None) == INVALID
    assert lib.kda_short_conv(ctypes.byref(_conv_args(B=0)), None) == OK
    assert lib.kda_output_gate(ctypes.byref(_gate_args(N=0)), None) == OK


@no_gpu_only
@pytest.mark.parametrize("field,value,expected", [
    ("K", 0, INVALID),
    ("K", 5, INVALID),
    ("T", -1, INVALID),
    ("C", 192, UNSUPPORTED),          # not a multiple of 128
    ("head_dim", 64, UNSUPPORTED),
    ("w", None, INVALID),
    ("x", None, INVALID),
    ("x", 0x7f0000100004, ALIGN),     # 16-byte rows
    ("x", 0x7f0000100008, ALIGN),     # 8-byte aligned is not enough
    ("state_in", 0x7f0000700008, ALIGN),
    ("state_out", 0x7f0000600002, ALIGN),
    ("y", 0x7f0000100000, ALIAS),     # y == x
    ("state_out", 0x7f0000500000, ALIAS),   # state_out == y
])
def test_short_conv_validation(field, value, expected):
    assert kda.load().kda_short_conv(ctypes.byref(_conv_args(**{field: value})), None) == expected


@no_gpu_only
@pytest.mark.parametrize("field,value,expected", [
    ("D", 64, UNSUPPORTED),
    ("HV", 0, INVALID),
    ("N", -1, INVALID),
    ("gate", None, INVALID),
    ("o", 0x7f0000100004, ALIGN),
    ("y", 0x7f0000200000, ALIAS),     # y == gate
])
def test_output_gate_validation(field, value, expected):
    assert kda.load().kda_output_gate(ctypes.byref(_gate_args(**{field: value})), None) == expected


@no_gpu_only
def test_layer_valid_calls_reach_the_launch_without_a_gpu():
    """Valid arguments pass validation and the launch itself fails without a GPU."""
    assert kda.load().kda_short_conv(ctypes.byref(_conv_args()), None) == 5      # KDA_ERR_CUDA
    assert kda.load().kda_output_gate(ctypes.byref(_gate_args()), None) == 5


# --- struct layouts: ctypes mirrors against the C header ---------------------
_STRUCTS = {"kda_chunk_args": _lib.ChunkArgs, "kda_chunk_bwd_args": _lib.ChunkBwdArgs,
            "kda_step_args": _lib.StepArgs, "kda_conv_args": _lib.ConvArgs,
            "kda_gate_args": _lib.GateArgs}


def test_ctypes_structs_match_the_header(tmp_path):
    """Every field of every argument struct sits at the offset the C compiler
    gives it, and the sizes agree (a mismatch would make the library read a
    pointer from the wrong place)."""
    lines = ['#include <stddef.h>', '#include <stdio.h>', '#include "kda.h"', "int main(void) {"]
    for cname, py in _STRUCTS.items():
        lines.append('printf("%s sizeof %%zu\\n", sizeof(%s));' % (cname, cname))
        for fname, _ in py._fields_:
            lines.append('printf("%s %s %%zu\\n", offsetof(%s, %s));' % (cname, fname, cname, fname))
    lines.append("return 0; }")
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines))
    exe = tmp_path / "layout"
    import subprocess
    subprocess.run(["gcc", "-std=c99", "-I", os.path.dirname(HEADER), str(src), "-o", str(exe)], check=True)
    got = {}
    for line in subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.splitlines():
        s, f, v = line.split()
        got[(s, f)] = int(v)
    for cname, py in _STRUCTS.items():
        assert got[(cname, "sizeof")] == ctypes.sizeof(py), cname
        for fname, _ in py._fields_:
            assert got[(cname, fname)] == getattr(py, fname).offset, (cname, fname)


# --- chunk states (forward output) and the backward entry point --------------
@no_gpu_only
def test_chunk_states_validation():
    a = _chunk_args()
    sc = 0x7f0000000000 + (12 << 20)
    assert _fwd(_chunk_args(S_chunks=sc + 2)) == ALIGN
    assert _fwd(_chunk_args(S_chunks=a.q)) == ALIAS
    assert _fwd(_chunk_args(S_chunks=a.o + 4)) == ALIAS
    assert _fwd(_chunk_args(S_chunks=a.S0)) == ALIAS
    # only the SIMT kernel writes them
    assert _fwd(_chunk_args(S_chunks=sc, algo=2)) == UNSUPPORTED


def _bwd_args(**kw):
    a = _lib.ChunkBwdArgs()
    a.B, a.T, a.H, a.HV, a.Dk, a.Dv, a.chunk = 1, 64, 2, 4, 16, 16, 16
    a.dtype, a.algo = 0, 0
    a.g_min, a.scale, a.l2_eps = -5.0, 1.0, 1e-6
    a.qk_l2norm_in_kernel = a.beta_sigmoid_in_kernel = a.gate_in_kernel = 1
    base = 0x7f3000000000
    names = ["q", "k", "v", "g", "beta", "A_log", "dt_bias", "S_chunks", "dout", "dS_T",
             "dq", "dk", "dv", "dg", "dbeta", "dS0", "dA_log", "ddt_bias"]
    for i, name in enumerate(names):
        setattr(a, name, base + (i + 1) * (1 << 20))
    for key, val in kw.items():
        setattr(a, key, val)
    return a


def _bwd(a):
    return kda.load().kda_chunk_bwd(ctypes.byref(a), None)


def test_bwd_null_and_empty():
    assert kda.load().kda_chunk_bwd(None, None) == INVALID
    assert _bwd(_bwd_args(B=0)) == OK


@no_gpu_only
@pytest.mark.parametrize("field,value,expected", [
    ("H", 3, INVALID),
    ("Dk", 129, UNSUPPORTED),
    ("chunk", 65, UNSUPPORTED),
    ("chunk", 0, INVALID),
    ("algo", 2, UNSUPPORTED),        # no tensor-core backward
    ("algo", 7, INVALID),
    ("dtype", 3, INVALID),
    ("g_min", 1.0, INVALID),
    ("S_chunks", None, INVALID),
    ("dout", None, INVALID),
    ("dq", None, INVALID),
    ("A_log", None, INVALID),        # gate_in_kernel needs A_log
    ("q", 0x7f3000100002, ALIGN),
    ("dS0", 0x7f3001000001, ALIGN),
    ("dq", 0x7f3000100000, ALIAS),   # dq over q
    ("dv", 0x7f3000c00000, ALIAS),   # dv over dk
    ("dS0", 0x7f3000a00000, ALIAS),  # dS0 over dS_T
])
def test_bwd_validation(field, value, expected):
    assert _bwd(_bwd_args(**{field: value})) == expected


@no_gpu_only
def test_bwd_valid_request_without_gpu_reports_cuda_error():
    assert _bwd(_bwd_args()) == 5
    # the parameter gradients are not outputs without the in-kernel gate
    assert _bwd(_bwd_args(gate_in_kernel=0, A_log=None, dA_log=0x7f3000100000)) == 5


def test_header_and_library_link_from_plain_c(tmp_path):
    """A C99 program includes include/kda.h, links libkda_b200.so and calls the
    entry points that need no device (version, status names, argument checks)."""
    import subprocess
    src = tmp_path / "use.c"
    src.write_text(r"""
#include <stdio.h>
#include <string.h>
#include "kda.h"
int main(void) {
    kda_chunk_args a;
    kda_chunk_bwd_args g;
    memset(&a, 0, sizeof a);
    memset(&g, 0, sizeof g);
    if (kda_version() < 100) return 1;
    if (strcmp(kda_status_string(KDA_ERR_ALIAS), "KDA_ERR_ALIAS") != 0) return 2;
    if (kda_chunk_fwd(NULL, NULL) != KDA_ERR_INVALID_ARG) return 3;
    a.H = 1; a.HV = 3;             /* HV % H fine, but sizes zero: invalid */
    if (kda_chunk_fwd(&a, NULL) != KDA_ERR_INVALID_ARG) return 4;
    if (kda_chunk_bwd(&g, NULL) != KDA_ERR_INVALID_ARG) return 5;
    if (kda_compose(-1, 1, 8, 8, NULL, NULL, NULL, NULL, NULL) != KDA_ERR_INVALID_ARG) return 6;
    puts("c abi ok");
    return 0;
}
""")
    lib = kda.library_path()
    exe = tmp_path / "use"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-I", os.path.dirname(HEADER), str(src), "-o", str(exe),
                    "-L", os.path.dirname(lib), "-lkda_b200", "-Wl,-rpath," + os.path.dirname(lib)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0 and "c abi ok" in r.stdout, (r.returncode, r.stdout, r.stderr)


@no_gpu_only
def test_gate_mode_and_per_head_validation():
    """gate_in_kernel must be 0, 1 or 2; with g_per_head the gate tensor is
    [B, T, HV] and dt_bias [HV], and the aliasing checks use those sizes."""
    assert _fwd(_chunk_args(gate_in_kernel=3)) == INVALID
    assert _fwd(_chunk_args(gate_in_kernel=-1)) == INVALID
    assert _bwd(_bwd_args(gate_in_kernel=3)) == INVALID
    st = _step_args()
    st.gate_in_kernel = 5
    assert kda.load().kda_step(ctypes.byref(st), None) == INVALID
    # the softplus gate on the tensor-core kernel is refused (it needs g >= g_min)
    a = _chunk_args(gate_in_kernel=2, algo=2)
    assert _fwd(a) == UNSUPPORTED
    # per head: an output right after the [B*T*HV] gate tensor does not overlap it,
    # one inside the per-channel extent of the same tensor would (checked with per head off)
    base = _chunk_args()
    g_end_per_head = base.g + 1 * 64 * 4 * 4          # B*T*HV floats
    assert _fwd(_chunk_args(g_per_head=1, o=g_end_per_head)) == 5      # valid: reaches the launch
    assert _fwd(_chunk_args(g_per_head=0, o=g_end_per_head)) == ALIAS
