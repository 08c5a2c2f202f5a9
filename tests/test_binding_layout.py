"""The Python binding's argument structs against include/csa.h: the same fields in the same
order, at the offsets and with the sizes a C compiler gives them, and the same struct sizes.
A field the tests never set (an optional weight, a debug output) would otherwise reach
the library in the wrong slot without any test noticing. No GPU and no library needed."""

import ctypes
import os
import re
import shutil
import subprocess

import pytest

import long_context_compressed_layer_b200 as csa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "csa.h")

BINDING = {
    "csa_compress_args": csa.CompressArgs,
    "csa_ikey_args": csa.IkeyArgs,
    "csa_iquery_args": csa.IqueryArgs,
    "csa_oproj_args": csa.OprojArgs,
    "csa_append_args": csa.AppendArgs,
    "csa_topk_args": csa.TopkArgs,
    "csa_attn_args": csa.AttnArgs,
    "csa_prefill_args": csa.PrefillArgs,
    "csa_pages": csa.Pages,
}


def header_structs():
    """{struct name: [field names in order]} from the header's typedef'd structs."""
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    out = {}
    for body, name in re.findall(r"typedef struct\s*\{(.*?)\}\s*(\w+)\s*;", text, flags=re.S):
        fields = []
        for decl in body.split(";"):
            decl = decl.strip()
            if decl:
                m = re.fullmatch(r"(?:const\s+)?\w+\s*\*?\s*(\w+)", decl)
                assert m, f"{name}: cannot read the declaration {decl!r}"
                fields.append(m.group(1))
        out[name] = fields
    return out


def test_every_header_struct_has_a_binding_with_the_same_fields():
    structs = header_structs()
    assert set(structs) == set(BINDING)
    for name, fields in structs.items():
        assert [f for f, _ in BINDING[name]._fields_] == fields, name


def test_offsets_and_sizes_match_the_c_compiler(tmp_path):
    if not shutil.which("gcc"):
        pytest.skip("no C compiler")
    lines = ["#include <stddef.h>", "#include <stdio.h>", '#include "csa.h"', "int main(void) {"]
    for name, cls in BINDING.items():
        lines.append(f'  printf("{name} . %zu %zu\\n", (size_t)0, sizeof({name}));')
        for f, _ in cls._fields_:
            lines.append(f'  printf("{name} {f} %zu %zu\\n", offsetof({name}, {f}), '
                         f'sizeof((({name}*)0)->{f}));')
    lines += ["  return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = str(tmp_path / "layout")
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Werror", "-I",
                           os.path.join(ROOT, "include"), str(src), "-o", exe])
    got = subprocess.run([exe], capture_output=True, text=True, check=True).stdout.split("\n")
    seen = 0
    for line in filter(None, got):
        name, field, off, size = line.split()
        cls = BINDING[name]
        if field == ".":
            assert int(size) == ctypes.sizeof(cls), f"sizeof({name})"
        else:
            d = getattr(cls, field)
            assert (d.offset, d.size) == (int(off), int(size)), f"{name}.{field}"
        seen += 1
    assert seen == sum(len(c._fields_) + 1 for c in BINDING.values())


def test_every_entry_point_has_a_signature_of_the_declared_arity():
    # ctypes passes whatever it is given when argtypes is unset and assumes an int result;
    # every entry point the header declares gets its declared result type and as many
    # argtypes as the declaration has parameters
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    decls = re.findall(r"^\s*((?:const\s+)?[A-Za-z_][\w\s\*]*?)\b(\w+)\s*\(([^;{]*)\)\s*;",
                       text, flags=re.M)
    if not os.path.exists(csa.LIB_PATH):
        pytest.skip("library not built")
    L = csa.lib()
    results = {"int": ctypes.c_int, "size_t": ctypes.c_size_t, "const char*": ctypes.c_char_p,
               "double": ctypes.c_double}
    assert decls
    for ret, name, params in decls:
        ret = re.sub(r"\s*\*", "*", " ".join(ret.split()))
        params = params.strip()
        arity = 0 if params in ("", "void") else params.count(",") + 1
        fn = getattr(L, name)
        assert fn.argtypes is not None and len(fn.argtypes) == arity, name
        assert fn.restype is results[ret], (name, ret)


def test_every_header_field_is_documented():
    # the boundary states each argument's meaning and layout next to it
    text = open(HEADER).read()
    for body, name in re.findall(r"typedef struct\s*\{(.*?)\}\s*(\w+)\s*;", text, flags=re.S):
        bare = [ln.strip() for ln in body.splitlines() if ln.strip() and "/*" not in ln]
        assert not bare, f"{name}: fields without a comment: {bare}"
