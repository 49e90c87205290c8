"""The oracle and the CUDA path share nothing, and the product path has no
CPU fallback: checked on the sources and on a copy of the package without
its built library."""
import ast
import os
import shutil
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "bit_weight_quantized_nvq_b200")


def _imported_modules(path):
    tree = ast.parse(open(path).read(), filename=path)
    names = set()
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            names.update(a.name for a in node.names)
        elif isinstance(node, ast.ImportFrom) and node.module:
            names.add(node.module)
    return names


def test_library_never_imports_the_oracle():
    for dirpath, _, files in os.walk(PKG):
        for f in files:
            p = os.path.join(dirpath, f)
            if f.endswith(".py"):
                assert not any("oracle" in m for m in _imported_modules(p)), p
            elif f.endswith((".cu", ".cuh", ".cpp", ".h")):
                text = open(p).read()
                assert "nvq_oracle" not in text and '#include "oracle' not in text, p


def test_oracle_imports_nothing_from_the_library():
    for f in os.listdir(os.path.join(ROOT, "oracle")):
        if f.endswith(".py"):
            mods = _imported_modules(os.path.join(ROOT, "oracle", f))
            assert not any(m.startswith("bit_weight_quantized_nvq_b200") for m in mods), f


def test_input_module_holds_no_method_arithmetic():
    """workloads.py serves both sides, so it must not quantise, pack or dot."""
    mods = _imported_modules(os.path.join(PKG, "workloads.py"))
    assert not any("oracle" in m or m.endswith("capi") for m in mods)
    # identifiers of the code (not its prose): no format decoder, quantiser,
    # packer or dot product among them
    tree = ast.parse(open(os.path.join(PKG, "workloads.py")).read())
    idents = set()
    for node in ast.walk(tree):
        if isinstance(node, ast.Name):
            idents.add(node.id.lower())
        elif isinstance(node, ast.Attribute):
            idents.add(node.attr.lower())
        elif isinstance(node, ast.FunctionDef):
            idents.add(node.name.lower())
    for word in ("e2m1", "ue4m3", "quantize", "pack", "dp4a", "dot", "matmul", "einsum"):
        assert not any(word in i for i in idents), word


def test_binding_fails_loudly_without_the_built_library(tmp_path):
    """A copy of the package without libnvq.so: importing the binding raises
    instead of falling back to anything on the CPU."""
    dst = tmp_path / "bit_weight_quantized_nvq_b200"
    shutil.copytree(PKG, dst, ignore=shutil.ignore_patterns("*.so", "csrc", "__pycache__"))
    code = ("import sys; sys.path.insert(0, %r)\n"
            "try:\n"
            "    import bit_weight_quantized_nvq_b200.capi\n"
            "except ImportError as e:\n"
            "    print('raised', e)\n"
            "else:\n"
            "    print('imported')\n") % str(tmp_path)
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.startswith("raised"), r.stdout
