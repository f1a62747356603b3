"""The product never touches the oracle: no file of the package (Python or
CUDA) imports, includes or names the oracle module, and the oracle shares no
file with the package. Only the tests, the smoke check and the benchmark's
CPU-baseline and reference legs use the oracle."""
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "w8a8_quantized_matmul_b200")


def _sources(top, exts):
    for d, _, files in os.walk(top):
        if "__pycache__" in d:
            continue
        for f in files:
            if f.endswith(exts):
                yield os.path.join(d, f)


def test_package_does_not_use_the_oracle():
    pat = re.compile(r"^\s*(import\s+oracle|from\s+oracle\b|from\s+\.\.oracle|#\s*include\s*[<\"].*oracle)",
                     re.M)
    for path in _sources(PKG, (".py", ".cu", ".cuh", ".h", ".c")):
        src = open(path, encoding="utf-8").read()
        assert not pat.search(src), f"{path} imports the oracle"


def test_oracle_does_not_use_the_package():
    pat = re.compile(r"^\s*(import\s+w8a8_quantized_matmul_b200|from\s+w8a8_quantized_matmul_b200)",
                     re.M)
    for path in _sources(os.path.join(ROOT, "oracle"), (".py", ".cpp", ".h")):
        src = open(path, encoding="utf-8").read()
        assert not pat.search(src), f"{path} imports the CUDA package"
        assert "libint8mm" not in src and "int8mm.h" not in src and "csrc" not in src, path
        assert "w8a8_quantized_matmul_b200" not in src, path


def test_cpp_oracle_includes_only_the_standard_library():
    """The C++ oracle is self-contained: standard headers only, no CUDA, no
    header or source of the package."""
    src = open(os.path.join(ROOT, "oracle", "llm_int8.cpp"), encoding="utf-8").read()
    incs = re.findall(r"^\s*#\s*include\s*([<\"][^>\"]+[>\"])", src, re.M)
    assert incs and all(i.startswith("<") for i in incs), incs
    assert not any("cuda" in i for i in incs), incs
    # the ctypes shim loads one library: the oracle's own build (oracle/build.py)
    shim = open(os.path.join(ROOT, "oracle", "llm_int8.py"), encoding="utf-8").read()
    assert shim.count("ctypes.CDLL(") == 1 and "_build.build()" in shim


def test_synth_holds_no_method_arithmetic():
    """The shared input generators draw numbers only: no quantiser, threshold
    test or scale computation of the method lives there."""
    src = open(os.path.join(ROOT, "synth", "__init__.py"), encoding="utf-8").read()
    for word in ("127", "absmax", "rint", "quantiz"):
        assert word not in src, word
