"""The C-ABI library loads and exports every entry point include/mk.h declares."""
import ctypes
import os
import re

import pytest

import persistent_runtime_b200 as prb

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "mk.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mk_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_binding_exports():
    assert declared_symbols() == sorted(prb.EXPORTS)


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(prb.LIB_PATH)
    for name in declared_symbols():
        assert hasattr(lib, name), name


def test_bad_arguments_are_rejected_without_a_device():
    lib = prb.lib()
    h = ctypes.c_void_p()
    assert lib.mk_plan_graph(None, None, 4, ctypes.byref(h)) == prb.MK_ERR_ARG
    cfg = prb.ModelConfig(2, 256, 4, 3, 64, 768, 4096, 0, 1e-6, 1e6, 1, 33)  # 4 % 3 != 0
    assert lib.mk_plan_graph(ctypes.byref(cfg), None, 4, ctypes.byref(h)) == prb.MK_ERR_ARG
    assert b"multiple" in lib.mk_last_error(None)
    cfg.n_kv_heads = 2
    assert lib.mk_plan_graph(ctypes.byref(cfg), None, 0, ctypes.byref(h)) == prb.MK_ERR_ARG
    assert lib.mk_plan_graph(ctypes.byref(cfg), None, 4, ctypes.byref(h)) == prb.MK_OK
    # a host-only handle cannot run a step
    assert lib.mk_decode_step(h, None, None, None, None, None, None, None) == prb.MK_ERR_ARG
    lib.mk_destroy(h)
    lib.mk_destroy(None)
    with pytest.raises(prb.MkError):
        prb.graph_from_edges([0, 1], [0, 0], [(1, 0)])


STRUCTS = {"mk_model_config": prb.ModelConfig, "mk_tuning": prb.Tuning, "mk_weights": prb.Weights,
           "mk_graph_view": prb.GraphView, "mk_info": prb.Info}


def test_binding_structures_match_the_header_layouts(tmp_path):
    # a C program compiled against include/mk.h prints every struct's size and
    # the offset of each field the ctypes binding declares
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    lines = ['#include <stddef.h>', '#include <stdio.h>', '#include "mk.h"', "int main(void) {"]
    for cname, py in STRUCTS.items():
        lines.append(f'  printf("{cname} size %zu\\n", sizeof({cname}));')
        for field, _ in py._fields_:
            lines.append(f'  printf("{cname} {field} %zu\\n", offsetof({cname}, {field}));')
    lines += ["  return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines))
    exe = tmp_path / "layout"
    subprocess.check_call([cc, "-std=c99", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)])
    out = subprocess.check_output([str(exe)]).decode().split("\n")
    got = {tuple(l.split()[:2]): int(l.split()[2]) for l in out if l}
    for cname, py in STRUCTS.items():
        assert got[(cname, "size")] == ctypes.sizeof(py), cname
        for field, _ in py._fields_:
            assert got[(cname, field)] == getattr(py, field).offset, (cname, field)
