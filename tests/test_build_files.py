"""The two build descriptions (build.py for Python users, the Makefile for a
native build) compile the same sources with the same flags."""
import importlib.util
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "block_sparse_attention_page_b200")


def _build_py():
    spec = importlib.util.spec_from_file_location("lserve_build_check", os.path.join(PKG, "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_build_py_compiles_every_cuda_source():
    srcs = sorted(f for f in os.listdir(os.path.join(PKG, "csrc")) if f.endswith(".cu"))
    assert sorted(_build_py().SOURCES) == srcs


def test_makefile_uses_the_same_compile_flags():
    with open(os.path.join(PKG, "Makefile")) as f:
        mk = f.read()
    flags = _build_py().FLAGS
    for want in ["arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17", "-fPIC",
                 "--expt-relaxed-constexpr"]:
        assert want in flags and want in mk, want
    assert re.search(r"wildcard csrc/\*\.cu", mk)
