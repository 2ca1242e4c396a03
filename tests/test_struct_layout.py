"""The ctypes mirrors in the binding match the C-ABI structs of include/mk.h
field by field: gcc compiles a probe that prints every field's offset and the
struct sizes, and the test compares them with the ctypes layout (a mismatch
would let mk_default_options write past the Python-side buffer)."""
import ctypes
import os
import subprocess

import pytest

from decode_persistent_block_b200 import mk

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
STRUCTS = {"mk_config": mk.MkConfig, "mk_weights": mk.MkWeights, "mk_options": mk.MkOptions,
           "mk_status": mk.MkStatus}


@pytest.fixture(scope="module")
def c_layout(tmp_path_factory):
    d = tmp_path_factory.mktemp("layout")
    lines = ["#include <stddef.h>", "#include <stdio.h>", '#include "mk.h"', "int main(void) {"]
    for name, cls in STRUCTS.items():
        lines.append(f'    printf("{name} size %zu\\n", sizeof({name}));')
        for field, _ in cls._fields_:
            lines.append(f'    printf("{name} {field} %zu\\n", offsetof({name}, {field}));')
    lines += ["    return 0;", "}"]
    src = d / "probe.c"
    src.write_text("\n".join(lines) + "\n")
    exe = d / "probe"
    subprocess.run(["gcc", "-std=c11", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)],
                   check=True, capture_output=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout
    return {tuple(l.split()[:2]): int(l.split()[2]) for l in out.splitlines()}


@pytest.mark.parametrize("name", list(STRUCTS))
def test_ctypes_mirror_matches_the_header(c_layout, name):
    cls = STRUCTS[name]
    assert c_layout[(name, "size")] == ctypes.sizeof(cls)
    for field, _ in cls._fields_:
        assert c_layout[(name, field)] == getattr(cls, field).offset, field
