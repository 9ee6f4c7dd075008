"""The ctypes binding mirrors include/mk.h exactly (no GPU).

- every status code, flag, buffer id and op kind the header defines has the
  same value in the binding;
- every public struct the binding mirrors has the same size, and every
  field the same offset, as a C compiler lays it out from the header
  (gcc compiles a small program that prints offsetof / sizeof).
"""
import ctypes
import os
import re
import shutil
import subprocess

import pytest

mk = pytest.importorskip("persistent_decode_megakernel_02_b200.mk")

HEADER = mk.HEADER_PATH

# binding class -> header struct
STRUCTS = {
    "Config": "mk_config",
    "Weights": "mk_weights",
    "KV": "mk_kv",
    "PackedWeights": "mk_packed_weights",
    "Info": "mk_info",
    "TraceRec": "mk_trace_rec",
}


def _header_text() -> str:
    text = open(HEADER).read()
    return re.sub(r"/\*.*?\*/", "", text, flags=re.S)


def test_enum_values_match_the_header():
    text = _header_text()
    pairs = dict((n, int(v)) for n, v in re.findall(r"\b(MK_[A-Z0-9_]+)\s*=\s*(\d+)", text))
    assert pairs, "no enumerators found"
    checked = 0
    for name, value in pairs.items():
        if name.startswith("MK_OP_"):
            continue            # op kinds: checked below through OP_NAMES
        assert hasattr(mk, name), f"{name} missing from the binding"
        assert getattr(mk, name) == value, name
        checked += 1
    assert checked >= 13
    ops = sorted((v, n) for n, v in pairs.items() if n.startswith("MK_OP_"))
    assert [v for v, _ in ops] == list(range(len(mk.OP_NAMES)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_struct_layouts_match_the_c_compiler(tmp_path):
    lines = ["#include <stdio.h>", "#include <stddef.h>", f'#include "{HEADER}"', "int main(void) {"]
    for cls, cname in STRUCTS.items():
        st = getattr(mk, cls)
        lines.append(f'printf("{cls} sizeof %zu\\n", sizeof({cname}));')
        for fname, _ in st._fields_:
            lines.append(f'printf("{cls} {fname} %zu\\n", offsetof({cname}, {fname}));')
    lines += ["return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    subprocess.check_call(["gcc", "-std=c11", "-o", str(exe), str(src)])
    out = subprocess.check_output([str(exe)], text=True)
    got = {}
    for line in out.splitlines():
        cls, field, val = line.split()
        got[(cls, field)] = int(val)
    for cls in STRUCTS:
        st = getattr(mk, cls)
        assert got[(cls, "sizeof")] == ctypes.sizeof(st), cls
        for fname, _ in st._fields_:
            assert got[(cls, fname)] == getattr(st, fname).offset, (cls, fname)
