"""C ABI checks that need no GPU: the library loads, exports every function
include/spa.h declares, and the ctypes mirror of spa_attention_args_t has the
C struct's size and field offsets.  No compute call is made here."""
import ctypes
import os
import re
import subprocess

import pytest

from selected_token_sparse_b200 import build, spa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "spa.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return spa.load_library()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(spa_\w+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in spa.EXPORTED:
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", spa.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT\s+(spa_\w+)$", out, flags=re.M))
    for n in declared_functions():
        assert n in exported, n
        assert getattr(lib, n) is not None


def test_error_strings(lib):
    for code in (0, -1, -2, -3, -4, 99):
        assert isinstance(lib.spa_error_string(code), bytes)


def test_struct_layout_matches_header(tmp_path):
    fields = [f[0] for f in spa.AttentionArgs._fields_]
    prog = ["#include <stdio.h>", "#include <stddef.h>", '#include "spa.h"', "int main(void) {",
            'printf("size %zu\\n", sizeof(spa_attention_args_t));']
    for f in fields:
        prog.append(f'printf("{f} %zu\\n", offsetof(spa_attention_args_t, {f}));')
    prog.append("return 0; }")
    c = tmp_path / "layout.c"
    c.write_text("\n".join(prog))
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-std=c99", "-I", os.path.join(ROOT, "include"), str(c), "-o", str(exe)],
                   check=True)
    got = dict(line.split() for line in subprocess.run([str(exe)], capture_output=True, text=True,
                                                       check=True).stdout.splitlines())
    assert int(got["size"]) == ctypes.sizeof(spa.AttentionArgs)
    for f in fields:
        assert int(got[f]) == getattr(spa.AttentionArgs, f).offset, f


def test_workspace_size_for_invalid_args_is_zero(lib):
    a = spa.AttentionArgs()
    a.struct_size = ctypes.sizeof(spa.AttentionArgs)
    a.is_causal = 0
    assert lib.spa_attention_workspace_size(ctypes.byref(a)) == 0
    assert lib.spa_attention(ctypes.byref(a), None, 0, None) == spa.SPA_ERR_UNSUPPORTED


def test_qkv_struct_layout_matches_header(tmp_path):
    fields = [f[0] for f in spa.QkvArgs._fields_]
    prog = ["#include <stdio.h>", "#include <stddef.h>", '#include "spa.h"', "int main(void) {",
            'printf("size %zu\\n", sizeof(spa_qkv_args_t));']
    for f in fields:
        prog.append(f'printf("{f} %zu\\n", offsetof(spa_qkv_args_t, {f}));')
    prog.append("return 0; }")
    c = tmp_path / "layout_qkv.c"
    c.write_text("\n".join(prog))
    exe = tmp_path / "layout_qkv"
    subprocess.run(["gcc", "-std=c99", "-I", os.path.join(ROOT, "include"), str(c), "-o", str(exe)],
                   check=True)
    got = dict(line.split() for line in subprocess.run([str(exe)], capture_output=True, text=True,
                                                        check=True).stdout.splitlines())
    assert int(got["size"]) == ctypes.sizeof(spa.QkvArgs)
    for f in fields:
        assert int(got[f]) == getattr(spa.QkvArgs, f).offset, f
