"""Static check (CPU only) of the Python files whose code paths run only on a
GPU (the benchmark runners, the GPU tests, smoke()): every name a function
reads is defined locally, in an enclosing scope, at module level or as a
builtin, so a misspelt name cannot first show up on the GPU machine."""
import builtins
import os
import symtable

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FILES = ["bench.py", "__graft_entry__.py", "bit_quantized_linear_nvfp4_b200/nvfp4.py",
         "bit_quantized_linear_nvfp4_b200/workloads.py", "bit_quantized_linear_nvfp4_b200/build.py",
         "oracle/nvfp4_oracle.py", "tests/gpu_helpers.py"] + sorted(
    os.path.join("tests", f) for f in os.listdir(os.path.join(ROOT, "tests")) if f.startswith("test_gpu_"))


def _undefined(path):
    src = open(os.path.join(ROOT, path)).read()
    top = symtable.symtable(src, path, "exec")
    module_names = set(top.get_identifiers())
    bad = []

    def walk(tab, enclosing):
        here = set(tab.get_identifiers())
        for sym in tab.get_symbols():
            if sym.is_referenced() and (sym.is_global() or sym.is_free()):
                n = sym.get_name()
                if n not in module_names and not hasattr(builtins, n) and n not in enclosing:
                    bad.append(f"{tab.get_name()} (line {tab.get_lineno()}): {n}")
        for child in tab.get_children():
            walk(child, enclosing | here)

    for child in top.get_children():
        walk(child, set())
    return bad


@pytest.mark.parametrize("path", FILES)
def test_no_undefined_names(path):
    assert _undefined(path) == []


def test_the_check_catches_a_misspelt_name(tmp_path):
    f = tmp_path / "m.py"
    f.write_text("import os\n\ndef run(dist):\n    return dst.barrier() or os.sep\n")
    rel = os.path.relpath(f, ROOT)
    assert _undefined(rel) == ["run (line 3): dst"]
