"""The C-ABI library loads without a GPU and exports every symbol its header declares."""
import ctypes as C
import os
import re
import subprocess

import pytest

from verified_sparse_attention_b200 import _abi
from verified_sparse_attention_b200.csrc import build as csrc_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    text = open(os.path.join(ROOT, "include", "vattn.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(vattn_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    if csrc_build.needs_build():
        csrc_build.build()
    return C.CDLL(_abi.LIB_PATH)


def test_header_declares_the_binding_surface():
    assert _declared() == sorted(_abi.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in _declared():
        assert hasattr(lib, name), name


def test_binding_struct_layouts_match_header():
    # field order and widths of the two structs, read from the header text
    text = open(os.path.join(ROOT, "include", "vattn.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    for struct, cls in (("vattn_config", _abi.vattn_config), ("vattn_params", _abi.vattn_params)):
        body = re.search(r"typedef struct \{([^{}]*)\}\s*" + struct + ";", text).group(1)
        names = []
        for decl in body.split(";"):
            decl = decl.strip()
            if not decl:
                continue
            for part in decl.split(","):
                names.append(re.findall(r"\w+", part)[-1])
        assert names == [f[0] for f in cls._fields_], struct


def test_binding_struct_offsets_match_the_compiled_header(tmp_path):
    # byte offsets and sizes as a C compiler lays the header's structs out
    fields = {"vattn_config": _abi.vattn_config, "vattn_params": _abi.vattn_params}
    lines = ["#include <stdio.h>", "#include <stddef.h>", '#include "vattn.h"', "int main(void) {"]
    for struct, cls in fields.items():
        lines.append(f'  printf("{struct} size %zu\\n", sizeof({struct}));')
        for name, _ in cls._fields_:
            lines.append(f'  printf("{struct} {name} %zu\\n", offsetof({struct}, {name}));')
    lines += ["  return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-std=c11", "-I", os.path.join(ROOT, "include"), "-o", str(exe), str(src)],
                   check=True)
    got = {}
    for line in subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.splitlines():
        struct, name, val = line.split()
        got[(struct, name)] = int(val)
    for struct, cls in fields.items():
        assert got[(struct, "size")] == C.sizeof(cls), struct
        for name, _ in cls._fields_:
            assert got[(struct, name)] == getattr(cls, name).offset, (struct, name)


def test_strerror_without_device(lib):
    _abi.lib()
    assert _abi.vattn_strerror(_abi.VATTN_EINVAL) == "invalid argument"
