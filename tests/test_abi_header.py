"""The Python binding against the C header it marshals for (CPU only, no GPU calls).

The binding declares every entry point's argument and return types and the public
structs by hand (ctypes).  A slip there (a field out of order, an int where the
header has int64_t) passes values in the wrong registers or at the wrong offsets
without any error.  These tests read the truth from include/gptq2d.h itself:
  * struct sizes, field offsets and enum/#define values, from a small C program
    compiled against the header with the host C compiler;
  * every prototype's parameter and return types, parsed from the header, against
    the ctypes declarations of the loaded library.
"""
import ctypes
import json
import os
import re
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gptq2d.h")

STRUCTS = {
    "gptq2d_stats": ["proxy_loss", "n_clamped", "n_near_tie", "n_nonfinite", "status",
                     "n_out_of_range"],
    "gptq2d_grid": ["bits", "clamp", "group_size", "scales", "ld_scales", "zeros", "packed"],
    "gptq2d_layer": ["W", "w_dtype", "m", "n", "ldw", "H_L", "ldhl", "H_R", "ldhr", "h_dtype",
                     "grid", "Q", "ldq", "stats"],
}
CONSTANTS = ["GPTQ2D_OK", "GPTQ2D_ERR_INVALID_ARG", "GPTQ2D_ERR_NOT_SPD", "GPTQ2D_ERR_NONFINITE",
             "GPTQ2D_ERR_WORKSPACE", "GPTQ2D_ERR_TIMEOUT", "GPTQ2D_ERR_CUDA", "GPTQ2D_ERR_RANGE",
             "GPTQ2D_F32",
             "GPTQ2D_BF16", "GPTQ2D_F64", "GPTQ2D_MAX_KRON_FACTORS"]


@pytest.fixture(scope="module")
def header_facts(tmp_path_factory):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no host C compiler")
    d = tmp_path_factory.mktemp("abi")
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "gptq2d.h"', "int main(void) {",
             '  printf("{");']
    for s, fields in STRUCTS.items():
        lines.append(f'  printf("\\"sizeof {s}\\": %zu, ", sizeof({s}));')
        for f in fields:
            lines.append(f'  printf("\\"{s}.{f}\\": %zu, ", offsetof({s}, {f}));')
            lines.append(f'  printf("\\"sizeof {s}.{f}\\": %zu, ", sizeof((({s}*)0)->{f}));')
    for c in CONSTANTS:
        lines.append(f'  printf("\\"{c}\\": %lld, ", (long long)({c}));')
    lines += ['  printf("\\"end\\": 0}\\n");', "  return 0;", "}"]
    src = d / "probe.c"
    src.write_text("\n".join(lines) + "\n")
    exe = d / "probe"
    subprocess.run([cc, "-std=c99", "-Wall", "-Werror", "-I", os.path.dirname(HEADER), str(src),
                    "-o", str(exe)], check=True, capture_output=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout
    return json.loads(out)


@pytest.fixture(scope="module")
def g():
    import two_sided_adaptive_b200 as g
    if not os.path.exists(g.library_path):
        pytest.skip("libgptq2d.so is not built")
    return g


def test_struct_layouts_match_the_header(header_facts, g):
    for cls, name in ((g._Grid, "gptq2d_grid"), (g._Layer, "gptq2d_layer")):
        assert ctypes.sizeof(cls) == header_facts[f"sizeof {name}"], name
        assert [f for f, _ in cls._fields_] == STRUCTS[name], name
        for f in STRUCTS[name]:
            # offsets alone can hide a 4-byte field where the header has 8 (padding)
            assert getattr(cls, f).offset == header_facts[f"{name}.{f}"], (name, f)
            assert getattr(cls, f).size == header_facts[f"sizeof {name}.{f}"], (name, f)
    # gptq2d_stats is read back as STATS_WORDS 8-byte words in field order
    assert g.STATS_WORDS * 8 == header_facts["sizeof gptq2d_stats"]
    for k, f in enumerate(STRUCTS["gptq2d_stats"]):
        assert header_facts[f"gptq2d_stats.{f}"] == 8 * k, f
    words = [0] * g.STATS_WORDS
    words[1:] = [11, 22, 33, 44, 55]
    assert list(g.stats_dict(words).keys())[1:] == ["n_clamped", "n_near_tie", "n_nonfinite",
                                                    "status", "n_out_of_range"]
    assert [g.stats_dict(words)[k] for k in STRUCTS["gptq2d_stats"][1:]] == [11, 22, 33, 44, 55]


def test_constants_match_the_header(header_facts, g):
    for name in ("OK", "INVALID_ARG", "NOT_SPD", "NONFINITE", "WORKSPACE", "TIMEOUT", "CUDA",
                 "RANGE"):
        key = "GPTQ2D_OK" if name == "OK" else f"GPTQ2D_ERR_{name}"
        assert getattr(g.Status, name) == header_facts[key], name
    assert (g.DTYPE_F32, g.DTYPE_BF16, g.DTYPE_F64) == (
        header_facts["GPTQ2D_F32"], header_facts["GPTQ2D_BF16"], header_facts["GPTQ2D_F64"])
    assert g.MAX_KRON_FACTORS == header_facts["GPTQ2D_MAX_KRON_FACTORS"]


def _prototypes():
    """name -> (return class, [parameter classes]) for every gptq2d_* prototype."""
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    text = re.sub(r"\s+", " ", text)
    protos = {}
    for ret, name, params in re.findall(
            r"((?:const )?[A-Za-z_][A-Za-z0-9_]*\s*\**)\s*\b(gptq2d_[a-z0-9_]+)\s*\(([^()]*)\)\s*;",
            text):
        ps = [p.strip() for p in params.split(",")] if params.strip() not in ("", "void") else []
        protos[name] = (_cclass(ret), [_cclass(p) for p in ps])
    return protos


def _cclass(decl):
    """Type class of a C declaration: a parameter with its name, or a return type."""
    decl = decl.strip()
    if "*" in decl:
        return "char*" if re.fullmatch(r"(const )?char\s*\*", decl) else "ptr"
    base = decl.replace("const ", "").split()[0]
    return {"int": "int", "int64_t": "i64", "size_t": "size", "double": "double",
            "void": "void"}.get(base, base)


def _ctclass(t):
    if t is None:
        return "void"
    if t is ctypes.c_char_p:
        return "char*"
    if t is ctypes.c_void_p or (isinstance(t, type) and issubclass(t, ctypes._Pointer)):
        return "ptr"
    if t is ctypes.c_int:
        return "int"
    if t is ctypes.c_size_t:
        return "size"
    if t is ctypes.c_double:
        return "double"
    if ctypes.sizeof(t) == 8 and t in (ctypes.c_int64, ctypes.c_longlong, ctypes.c_long):
        return "i64"
    return repr(t)


def test_every_prototype_matches_its_ctypes_declaration(g):
    protos = _prototypes()
    assert len(protos) >= 20, sorted(protos)
    L = g.lib()
    for name, (ret, params) in sorted(protos.items()):
        fn = getattr(L, name)
        assert _ctclass(fn.restype) == ret, (name, fn.restype, ret)
        declared = getattr(fn, "argtypes", None) or []
        assert [_ctclass(t) for t in declared] == params, (name, declared, params)
