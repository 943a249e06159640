"""The C-ABI library builds, loads and exports every entry point include/sg.h
declares; host-side argument checks (no GPU compute)."""
import ctypes as C
import os
import re
import subprocess

import pytest

from conftest import ROOT


@pytest.fixture(scope="module")
def lib():
    from learned_sparse_feature_b200 import build, binding
    build.build()
    return binding.load()


def _declared():
    text = open(os.path.join(ROOT, "include", "sg.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sg_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = _declared()
    for n in ("sg_create", "sg_match", "sg_destroy", "sg_status"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    from learned_sparse_feature_b200 import binding
    out = subprocess.run(["nm", "-D", "--defined-only", binding.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (sg_\w+)", out))
    for n in _declared():
        assert n in exported, n
        assert hasattr(lib, n)
    assert set(binding.EXPORTED) == set(_declared())


def test_strerror_and_null_handle(lib):
    assert lib.sg_strerror(0) == b"ok"
    assert lib.sg_strerror(5).startswith(b"a bounded")
    # null handle -> INVALID_ARG, synchronously, no device work
    assert lib.sg_match(None, 1, 1, 1, *([None] * 12)) == 1
    assert lib.sg_status(None, None) == 1
    assert lib.sg_launches_per_match(None, 1, 1, 1) == 0


def test_create_rejects_bad_arguments(lib):
    from learned_sparse_feature_b200 import binding
    h = C.c_void_p()
    assert lib.sg_create(None, None, C.byref(h)) == 1
    w = binding.SgWeights()
    cfg = binding.SgConfig(128, 4, 18, 100, 0.2, 1e-5, 1, 640.0, 480.0, 0, 1, 64, 64)
    assert lib.sg_create(C.byref(w), C.byref(cfg), C.byref(h)) == 7     # D != 256
    cfg = binding.SgConfig(256, 4, 0, 100, 0.2, 1e-5, 1, 640.0, 480.0, 0, 1, 64, 64)
    assert lib.sg_create(C.byref(w), C.byref(cfg), C.byref(h)) == 1     # n_stages = 0
    cfg = binding.SgConfig(256, 4, 18, 100, 0.2, 1e-5, 5, 640.0, 480.0, 0, 1, 64, 64)
    assert lib.sg_create(C.byref(w), C.byref(cfg), C.byref(h)) == 1     # bad precision
    assert not h.value


def test_header_is_plain_c_and_links_against_the_library(lib, tmp_path):
    # a C99 translation unit that includes the header and takes the address of
    # every declared entry point, linked against the built library: the boundary
    # needs no C++ and no torch
    from learned_sparse_feature_b200 import binding
    names = _declared()
    src = tmp_path / "abi_check.c"
    body = "\n".join(f"    (void (*)(void)){n}," for n in names)
    src.write_text(f'#include "sg.h"\n#include <stdio.h>\n'
                   f"void (*entry_points[])(void) = {{\n{body}\n}};\n"
                   "int main(void) {\n"
                   "    sg_weights w = {0};\n    sg_config c = {0};\n    sg_handle *h = 0;\n"
                   "    (void)w; (void)c; (void)h;\n"
                   '    printf("%d\\n", (int)(sizeof entry_points / sizeof entry_points[0]));\n'
                   "    return 0;\n}\n")
    exe = tmp_path / "abi_check"
    libdir = os.path.dirname(binding.LIB_PATH)
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                        "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
                        "-L", libdir, "-lsg", f"-Wl,-rpath,{libdir}", "-Wl,--unresolved-symbols=ignore-in-shared-libs"],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_binding_structs_match_the_header_layout(tmp_path):
    # the ctypes mirrors of sg_weights / sg_config must have the C layout: a C
    # program prints sizeof and offsetof of every field, compared field by field
    from learned_sparse_feature_b200 import binding
    lines = []
    for cname, cls in (("sg_weights", binding.SgWeights), ("sg_config", binding.SgConfig)):
        lines.append(f'    printf("{cname} %zu\\n", sizeof({cname}));')
        for f, _ in cls._fields_:
            lines.append(f'    printf("{cname}.{f} %zu\\n", offsetof({cname}, {f}));')
    src = tmp_path / "layout.c"
    src.write_text('#include <stddef.h>\n#include <stdio.h>\n#include "sg.h"\nint main(void) {\n'
                   + "\n".join(lines) + "\n    return 0;\n}\n")
    exe = tmp_path / "layout"
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                        str(src), "-o", str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    got = dict(l.split() for l in subprocess.run([str(exe)], capture_output=True, text=True).stdout.split("\n") if l)
    for cname, cls in (("sg_weights", binding.SgWeights), ("sg_config", binding.SgConfig)):
        assert int(got[cname]) == C.sizeof(cls), cname
        for f, _ in cls._fields_:
            assert int(got[f"{cname}.{f}"]) == getattr(cls, f).offset, f"{cname}.{f}"
