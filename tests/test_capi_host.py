"""Host-side checks of the C ABI (CPU only: no kernel is launched).

* librsm.so loads and exports every function include/rsm.h declares;
* the ctypes structs have the C layout (checked against a C program compiled with gcc);
* argument validation rejects bad calls before any CUDA call;
* the product path has no fallback: without the library, importing the binding fails.
"""
import ctypes
import os
import re
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "rsm.h")


@pytest.fixture(scope="module")
def lib():
    import __graft_entry__
    __graft_entry__.build()
    from sparse_routed_slot_b200 import _lib
    return _lib


def declared_functions():
    src = open(HEADER).read()
    return re.findall(r"RSM_API\s+[\w\s\*]+?\b(rsm_\w+)\s*\(", src)


def test_header_declares_the_three_calls():
    names = declared_functions()
    for n in ("rsm_route", "rsm_forward", "rsm_decode_step"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.check_output(["nm", "-D", "--defined-only", lib.LIB_PATH]).decode()
    exported = set(re.findall(r" T (rsm_\w+)$", out, flags=re.M))
    declared = set(declared_functions())
    assert declared <= exported, declared - exported
    assert set(lib.EXPORTED) == declared
    L = lib.load()
    for n in declared:
        assert hasattr(L, n)


def test_struct_layouts_match_c(lib, tmp_path):
    prog = tmp_path / "sizes.c"
    prog.write_text(
        '#include <stdio.h>\n#include <stddef.h>\n#include "rsm.h"\n'
        "int main(void){printf(\"%zu %zu %zu %zu %zu %zu %zu %zu %zu %zu\\n\", sizeof(rsm_forward_args),"
        " offsetof(rsm_forward_args, workspace_bytes), offsetof(rsm_forward_args, flags),"
        " offsetof(rsm_forward_args, router), offsetof(rsm_forward_args, slot_counts),"
        " sizeof(rsm_decode_args), offsetof(rsm_decode_args, state), offsetof(rsm_decode_args, flags),"
        " offsetof(rsm_decode_args, router), offsetof(rsm_decode_args, slot_counts));"
        "return 0;}\n")
    exe = tmp_path / "sizes"
    subprocess.check_call(["gcc", "-I", os.path.join(ROOT, "include"), "-o", str(exe), str(prog)])
    c = list(map(int, subprocess.check_output([str(exe)]).split()))
    F, D = lib.ForwardArgs, lib.DecodeArgs
    py = [ctypes.sizeof(F), F.workspace_bytes.offset, F.flags.offset, F.router.offset, F.slot_counts.offset,
          ctypes.sizeof(D), D.state.offset, D.flags.offset, D.router.offset, D.slot_counts.offset]
    assert c == py


def test_status_strings(lib):
    assert lib.status_string(lib.RSM_OK) == "RSM_OK"
    assert lib.status_string(lib.RSM_ERR_UNSUPPORTED) == "RSM_ERR_UNSUPPORTED"
    assert lib.load().rsm_version() >= 100


def _fwd(lib, **kw):
    a = lib.ForwardArgs()
    a.B, a.T, a.H, a.M, a.K, a.Dv = 1, 8, 1, 64, 4, 64
    a.qkv_dtype, a.decay = lib.RSM_BF16, lib.RSM_DECAY_HEAD
    fake = 1 << 20  # never dereferenced: every case below fails validation first
    for n in ("q", "k", "v", "logits", "f", "o"):
        setattr(a, n, fake)
    for k, v in kw.items():
        setattr(a, k, v)
    return lib.load().rsm_forward(ctypes.byref(a), None), lib.last_error()


@pytest.mark.parametrize("kw,code", [
    (dict(K=65), 1), (dict(K=0), 1), (dict(M=48, K=4), 2), (dict(M=512, K=4), 2),
    (dict(Dv=66), 2), (dict(Dv=260), 2), (dict(B=-1), 1), (dict(q=None), 1),
    (dict(o=None), 1), (dict(logits=(1 << 20) + 4), 1), (dict(qkv_dtype=7), 1),
    (dict(decay=3), 1), (dict(path=9), 1), (dict(HT=(1 << 20) + 8), 1),
    (dict(qkv_dtype=0, path=2), 2),
])
def test_forward_rejects_bad_arguments(lib, kw, code):
    st, msg = _fwd(lib, **kw)
    assert st == code and msg


def test_forward_empty_batch_is_a_no_op(lib):
    st, _ = _fwd(lib, B=0, q=None, k=None, v=None, logits=None, f=None, o=None)
    assert st == 0


def test_route_rejects_bad_arguments(lib):
    L = lib.load()
    assert L.rsm_route(None, 0, 64, 8, None, None, None) == 0          # nothing to do
    assert L.rsm_route(None, 5, 64, 8, None, None, None) == 1          # NULL logits
    assert L.rsm_route(1 << 20, 5, 64, 65, 1 << 21, None, None) == 1   # K > M
    assert L.rsm_route(1 << 20, 5, 100, 8, 1 << 21, None, None) == 2   # M not supported
    assert L.rsm_route(1 << 20, -1, 64, 8, 1 << 21, None, None) == 1


def test_decode_rejects_bad_arguments(lib):
    L = lib.load()
    a = lib.DecodeArgs()
    a.B, a.H, a.M, a.K, a.Dv = 2, 2, 128, 16, 128
    a.qkv_dtype, a.decay = lib.RSM_BF16, lib.RSM_DECAY_HEAD
    assert L.rsm_decode_step(ctypes.byref(a), None) == 1               # NULL pointers
    assert L.rsm_decode_step(None, None) == 1
    a.K = 129
    assert L.rsm_decode_step(ctypes.byref(a), None) == 1


def test_workspace_size_query_is_host_only(lib):
    a = lib.ForwardArgs()
    a.B, a.T, a.H, a.M, a.K, a.Dv = 1, 64, 2, 128, 16, 128
    a.qkv_dtype, a.decay = lib.RSM_BF16, lib.RSM_DECAY_HEAD
    for n in ("q", "k", "v", "logits", "f", "o"):
        setattr(a, n, 1 << 20)
    n = lib.load().rsm_forward_workspace_size(ctypes.byref(a))
    assert n != ctypes.c_size_t(-1).value
    a.K = 500
    assert lib.load().rsm_forward_workspace_size(ctypes.byref(a)) == ctypes.c_size_t(-1).value


def test_binding_fails_loudly_without_the_library(tmp_path):
    code = ("import sys, os; sys.path.insert(0, %r);"
            "import sparse_routed_slot_b200._lib as L; L.LIB_PATH = %r;"
            "\ntry:\n  L.load()\nexcept ImportError as e:\n  print('raised')\n") % (
                ROOT, str(tmp_path / "missing.so"))
    out = subprocess.check_output([sys.executable, "-c", code]).decode()
    assert "raised" in out


def test_profile_events_arguments(lib):
    L = lib.load()
    fake = (ctypes.c_void_p * 2)(1 << 20, 1 << 21)
    assert L.rsm_forward_set_profile_events(fake, 0) == 1                  # events without a count
    assert L.rsm_forward_set_profile_events(None, 0) == 0                  # recording off
    # too few events for a tensor-path call: rejected on the host, before any launch
    a = lib.ForwardArgs()
    a.B, a.T, a.H, a.M, a.K, a.Dv = 1, 64, 2, 128, 16, 128
    a.qkv_dtype, a.decay = lib.RSM_BF16, lib.RSM_DECAY_HEAD
    for n in ("q", "k", "v", "logits", "f", "o"):
        setattr(a, n, 1 << 20)
    a.workspace = 1 << 24
    a.workspace_bytes = L.rsm_forward_workspace_size(ctypes.byref(a))
    assert L.rsm_forward_set_profile_events(fake, 2) == 0
    try:
        assert L.rsm_forward(ctypes.byref(a), None) == 1
        assert "profiling events" in lib.last_error()
    finally:
        assert L.rsm_forward_set_profile_events(None, 0) == 0
