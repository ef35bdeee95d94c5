"""CPU tests of the C ABI boundary: the library loads, exports every symbol the
header declares, the ctypes structs match the C layouts, and argument errors
are reported before any CUDA call."""

import ctypes as C
import os
import re
import subprocess
import tempfile

import pytest

from persistent_task_runtime_b200 import build, mk

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mk.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return mk.load_library()


def header_functions():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"\b(mk_[a-z_0-9]+)\s*\(", src)))


def test_header_functions_are_the_binding_exports():
    assert header_functions() == sorted(mk.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in header_functions():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", build.LIB], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (mk_\w+)", out))
    assert set(header_functions()) <= exported
    # nothing else with the mk_ prefix leaks out of the library
    assert exported == set(header_functions())


STRUCTS = {
    "mk_model_config": mk.mk_model_config,
    "mk_layer_weights": mk.mk_layer_weights,
    "mk_weights": mk.mk_weights,
    "mk_kv_cache": mk.mk_kv_cache,
    "mk_plan_options": mk.mk_plan_options,
    "mk_step_args": mk.mk_step_args,
    "mk_plan_info_t": mk.mk_plan_info_t,
    "mk_prefill_args": mk.mk_prefill_args,
}


def test_ctypes_layouts_match_the_header():
    lines = ['#include <stdio.h>', '#include <stddef.h>', f'#include "{HEADER}"',
             "int main(void) {"]
    for name, cls in STRUCTS.items():
        lines.append(f'printf("{name} %zu\\n", sizeof({name}));')
        for f, _ in cls._fields_:
            lines.append(f'printf("{name}.{f} %zu\\n", offsetof({name}, {f}));')
    lines.append("return 0; }")
    with tempfile.TemporaryDirectory() as td:
        src = os.path.join(td, "layout.c")
        exe = os.path.join(td, "layout")
        open(src, "w").write("\n".join(lines))
        subprocess.run(["gcc", "-std=c11", src, "-o", exe], check=True)
        out = subprocess.run([exe], capture_output=True, text=True, check=True).stdout
    want = dict(line.rsplit(" ", 1) for line in out.strip().splitlines())
    for name, cls in STRUCTS.items():
        assert int(want[name]) == C.sizeof(cls), name
        for f, _ in cls._fields_:
            assert int(want[f"{name}.{f}"]) == getattr(cls, f).offset, f"{name}.{f}"


def test_argument_errors_before_any_launch(lib):
    out = C.c_void_p()
    assert lib.mk_plan_create(None, None, 1, 16, C.byref(out)) == mk.MK_ERR_INVALID_ARG
    assert b"cfg" in lib.mk_last_error()
    cfg = mk.mk_model_config(2, 256, 4, 2, 48, 688, 4096, 1e-6, 1e6, 1, 64)   # head_dim 48
    w = mk.mk_weights()
    lw = (mk.mk_layer_weights * 2)()
    w.layers = lw
    assert lib.mk_plan_create(C.byref(cfg), C.byref(w), 1, 16, C.byref(out)) == mk.MK_ERR_UNSUPPORTED
    cfg.head_dim = 64
    # NULL weight pointers
    assert lib.mk_plan_create(C.byref(cfg), C.byref(w), 1, 16, C.byref(out)) == mk.MK_ERR_INVALID_ARG
    assert lib.mk_decode_step_ex(None, None, None) == mk.MK_ERR_INVALID_ARG
    assert lib.mk_plan_status(None) == mk.MK_ERR_INVALID_ARG
    assert lib.mk_plan_reset(None) == mk.MK_ERR_INVALID_ARG
    lib.mk_plan_destroy(None)   # no-op


def test_noalloc_argument_errors_before_any_device_call(lib):
    """mk_decode_step_noalloc checks its arguments on the host first."""
    cfg = mk.mk_model_config(2, 256, 4, 2, 64, 688, 4096, 1e-6, 1e6, 1, 64)
    w = mk.mk_weights()
    lw = (mk.mk_layer_weights * 2)()
    w.layers = lw
    kv = mk.mk_kv_cache()
    a = mk.mk_step_args()
    a.kv = C.pointer(kv)
    a.batch = 1
    E = mk.MK_ERR_INVALID_ARG
    assert lib.mk_decode_step_noalloc(None, C.byref(w), 16, C.byref(a), None) == E
    assert lib.mk_decode_step_noalloc(C.byref(cfg), C.byref(w), 16, None, None) == E
    assert lib.mk_decode_step_noalloc(C.byref(cfg), C.byref(w), 8, C.byref(a), None) == E
    assert b"kv_page_size" in lib.mk_last_error()
    a.batch = 0
    assert lib.mk_decode_step_noalloc(C.byref(cfg), C.byref(w), 16, C.byref(a), None) == E
    a.batch = 1
    a.mode = mk.MODE_PER_OP
    assert lib.mk_decode_step_noalloc(C.byref(cfg), C.byref(w), 16, C.byref(a), None) == E
    assert b"MK_MODE_MEGAKERNEL" in lib.mk_last_error()
    a.mode = mk.MODE_MEGAKERNEL
    a.d_trace = 0x1000   # a trace buffer is sized by a plan's task count
    assert lib.mk_decode_step_noalloc(C.byref(cfg), C.byref(w), 16, C.byref(a), None) == E
    assert b"d_trace" in lib.mk_last_error()
    a.d_trace = None
    # NULL ids / positions / outputs / KV pointers
    assert lib.mk_decode_step_noalloc(C.byref(cfg), C.byref(w), 16, C.byref(a), None) == E
    bad = mk.mk_model_config(2, 256, 4, 2, 48, 688, 4096, 1e-6, 1e6, 1, 64)   # head_dim 48
    assert lib.mk_decode_step_noalloc(C.byref(bad), C.byref(w), 16, C.byref(a), None) == \
        mk.MK_ERR_UNSUPPORTED
