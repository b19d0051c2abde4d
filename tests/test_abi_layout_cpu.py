"""The ctypes declarations of the binding against the C header's own layout:
a small C program compiled with the header prints every struct's size and
field offsets, which must equal what ctypes computes.  A field added to one
side only (an ABI drift) fails here, on CPU."""
import ctypes
import os
import shutil
import subprocess

import pytest

from mixed_precision_zero_b200 import _abi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
STRUCTS = ["neox_segment", "neox_hparams", "neox_shard_desc", "neox_step_result", "neox_ipc_handle",
           "neox_scaler_state", "neox_tensor", "neox_tensor_set", "neox_profile"]


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs a C compiler")
def test_ctypes_structs_match_the_header(tmp_path):
    lines = ["#include <stddef.h>", "#include <stdio.h>", '#include "neox_shard.h"', "int main(void) {"]
    for name in STRUCTS:
        cls = getattr(_abi, name)
        lines.append(f'    printf("{name} size %zu\\n", sizeof({name}));')
        for field, _ in cls._fields_:
            lines.append(f'    printf("{name} {field} %zu\\n", offsetof({name}, {field}));')
    lines += ["    return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-std=c99", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split("\n")
    got = {}
    for ln in out:
        if ln:
            parts = ln.split()
            got[tuple(parts[:-1])] = int(parts[-1])
    for name in STRUCTS:
        cls = getattr(_abi, name)
        assert got[(name, "size")] == ctypes.sizeof(cls), name
        for field, _ in cls._fields_:
            assert got[(name, field)] == getattr(cls, field).offset, (name, field)
