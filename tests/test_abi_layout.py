"""The Python binding's ctypes structures against the C header (CPU): a small
C program compiled with the system compiler against include/dory.h prints
sizeof and offsetof of every struct the ABI passes by pointer, the enum
values the binding copies, and the option numbers; the binding must agree."""
import ctypes
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
dory = pytest.importorskip("looped_ngpt_lm_b200")

STRUCTS = {
    "dory_config": (dory.Config, [f[0] for f in dory.Config._fields_]),
    "dory_weights": (dory.Weights, [f[0] for f in dory.Weights._fields_]),
    "dory_spec_stats": (dory.SpecStats, [f[0] for f in dory.SpecStats._fields_]),
    "dory_mx_weights": (dory.MxWeightsC, [f[0] for f in dory.MxWeightsC._fields_]),
    "dory_nvfp4_weights": (dory.NvWeightsC, [f[0] for f in dory.NvWeightsC._fields_]),
}
CONSTANTS = {
    "DORY_LAST_LOOP": dory.LAST_LOOP, "DORY_PER_LOOP": dory.PER_LOOP, "DORY_F32": dory.F32,
    "DORY_BF16": dory.BF16, "DORY_OPT_CUDA_GRAPHS": dory.OPT_CUDA_GRAPHS, "DORY_OPT_PROFILE": dory.OPT_PROFILE,
    "DORY_OPT_GEMM_IMPL": dory.OPT_GEMM_IMPL, "DORY_OPT_PDL": dory.OPT_PDL, "DORY_OPT_PREFILL_TC": dory.OPT_PREFILL_TC,
    "DORY_OPT_ATTN_CLUSTER": dory.OPT_ATTN_CLUSTER, "DORY_OPT_L2_LOOKAHEAD": dory.OPT_L2_LOOKAHEAD,
    "DORY_OPT_MX_GEMV": dory.OPT_MX_GEMV, "DORY_OPT_FUSED_OPERANDS": dory.OPT_FUSED_OPERANDS,
    "DORY_OPT_ATTN_LOOKAHEAD": dory.OPT_ATTN_LOOKAHEAD,
    "DORY_OPT_L2_OWN": dory.OPT_L2_OWN,
}


@pytest.fixture(scope="module")
def c_layout(tmp_path_factory):
    cc = shutil.which("gcc") or shutil.which("cc")
    if not cc:
        pytest.skip("no C compiler")
    d = tmp_path_factory.mktemp("abi")
    lines = ["#include <stdio.h>", "#include <stddef.h>", '#include "dory.h"', "int main(void) {"]
    for name, (_, fields) in STRUCTS.items():
        lines.append(f'  printf("{name} size %zu\\n", sizeof({name}));')
        for f in fields:
            lines.append(f'  printf("{name}.{f} %zu\\n", offsetof({name}, {f}));')
    for k in CONSTANTS:
        lines.append(f'  printf("{k} %d\\n", (int){k});')
    for code, name in dory.STATUS.items():
        lines.append(f'  printf("{name} %d\\n", (int){name});')
    lines += ["  return 0;", "}"]
    src = d / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = d / "layout"
    subprocess.run([cc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src), "-o",
                    str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout
    return dict(line.rsplit(" ", 1) for line in out.strip().splitlines())


@pytest.mark.parametrize("name", list(STRUCTS))
def test_struct_layouts_match_the_header(c_layout, name):
    cls, fields = STRUCTS[name]
    assert int(c_layout[f"{name} size"]) == ctypes.sizeof(cls)
    for f in fields:
        assert int(c_layout[f"{name}.{f}"]) == getattr(cls, f).offset, f


def test_constants_match_the_header(c_layout):
    for k, v in CONSTANTS.items():
        assert int(c_layout[k]) == v, k
    for code, name in dory.STATUS.items():
        assert int(c_layout[name]) == code, name


def header_prototypes():
    """name -> list of parameter declarations, from include/dory.h (comments removed;
    balanced parentheses, so function-pointer-like parameters such as char (*names)[48] parse)."""
    import re
    text = open(os.path.join(ROOT, "include", "dory.h")).read()
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    out = {}
    for m in re.finditer(r"\b(?:dory_status|const char\*)\s+(dory_\w+)\s*\(", text):
        i, depth = m.end(), 1
        j = i
        while depth:
            depth += {"(": 1, ")": -1}.get(text[j], 0)
            j += 1
        body = text[i:j - 1]
        params, depth, cur = [], 0, ""
        for ch in body:
            if ch == "," and depth == 0:
                params.append(cur.strip())
                cur = ""
                continue
            depth += {"(": 1, ")": -1, "[": 1, "]": -1}.get(ch, 0)
            cur += ch
        if cur.strip() and cur.strip() != "void":
            params.append(cur.strip())
        out[m.group(1)] = params
    return out


def c_class(decl: str) -> str:
    d = " ".join(decl.split())
    if "*" in d or d.startswith("dory_stream") or "[" in d:
        return "ptr"
    for t, c in (("int64_t", "i64"), ("uint64_t", "u64"), ("int32_t", "i32"), ("size_t", "u64"),
                 ("float", "f32"), ("dory_cache_mode", "i32"), ("dory_dtype", "i32")):
        if d.startswith(t + " ") or d.startswith("const " + t + " "):
            return c
    raise AssertionError(f"unclassified parameter {decl!r}")


def py_class(t) -> str:
    if t in (ctypes.c_void_p,) or isinstance(t, type) and issubclass(t, ctypes._Pointer):
        return "ptr"
    # size_t and uint64_t are both 64-bit unsigned here (ctypes makes them one type)
    return {ctypes.c_int32: "i32", ctypes.c_int64: "i64", ctypes.c_uint64: "u64", ctypes.c_size_t: "u64",
            ctypes.c_float: "f32"}[t]


def test_argtypes_match_the_prototypes():
    protos = header_prototypes()
    assert sorted(protos) == sorted(dory.SYMBOLS)
    for name, params in protos.items():
        f = getattr(dory.lib, name)
        want = [c_class(p) for p in params]
        got = [py_class(t) for t in (f.argtypes or [])]
        assert got == want, (name, got, want)


def test_readme_c_example_compiles_against_the_header(tmp_path):
    """The C usage example in the README uses the header's names and
    signatures as they are (compiled, not run)."""
    import re

    cc = shutil.which("gcc") or shutil.which("cc")
    cuda_inc = "/usr/local/cuda/include"
    if not cc or not os.path.exists(os.path.join(cuda_inc, "cuda_runtime.h")):
        pytest.skip("no C compiler or CUDA headers")
    text = open(os.path.join(ROOT, "README.md")).read()
    blocks = re.findall(r"```c\n(.*?)```", text, re.S)
    assert blocks, "README has no C example"
    src = tmp_path / "example.c"
    src.write_text(blocks[0])
    subprocess.run([cc, "-std=c99", "-Wall", "-Werror", "-c", "-I", os.path.join(ROOT, "include"), "-I", cuda_inc,
                    str(src), "-o", str(tmp_path / "example.o")], check=True)
