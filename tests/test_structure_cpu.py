"""Structural rules of the repository, checked statically on the CPU:

* the product (the CUDA library's package and its binding) and the oracle share no code: neither
  imports the other, and the seeded input generators import neither;
* only the tests, the smoke check and the bench's CPU-baseline leg reach the oracle;
* without the built library the binding raises instead of falling back to anything;
* the binding's ctypes signature of every entry point matches include/mmf.h parameter by
  parameter (count, pointer or value, width, floating or integer)."""
import ast
import ctypes
import glob
import os
import re

import pytest

import ternary_weight_matmul_b200 as mmf
from ternary_weight_matmul_b200 import build as mbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _imports(path):
    """(module names imported anywhere in the file, {function name: modules imported inside it})."""
    tree = ast.parse(open(path).read(), filename=path)
    mods, by_fn = set(), {}
    for node in ast.walk(tree):
        names = []
        if isinstance(node, ast.Import):
            names = [a.name for a in node.names]
        elif isinstance(node, ast.ImportFrom) and node.module and node.level == 0:
            names = [node.module]
        mods.update(n.split(".")[0] for n in names)
    for fn in ast.walk(tree):
        if isinstance(fn, (ast.FunctionDef, ast.AsyncFunctionDef)):
            inner = set()
            for node in ast.walk(fn):
                if isinstance(node, ast.Import):
                    inner.update(a.name.split(".")[0] for a in node.names)
                elif isinstance(node, ast.ImportFrom) and node.module and node.level == 0:
                    inner.add(node.module.split(".")[0])
            by_fn[fn.name] = inner
    return mods, by_fn


def _py(folder):
    return sorted(glob.glob(os.path.join(ROOT, folder, "**", "*.py"), recursive=True))


def test_product_oracle_and_generators_share_no_imports():
    for path in _py("ternary_weight_matmul_b200"):
        mods, _ = _imports(path)
        assert not mods & {"oracle", "synth", "tests", "bench"}, (path, mods)
    for path in _py("oracle"):
        mods, _ = _imports(path)
        assert not mods & {"ternary_weight_matmul_b200", "synth", "bench", "torch"}, (path, mods)
    for path in _py("synth"):
        mods, _ = _imports(path)
        assert not mods & {"oracle", "ternary_weight_matmul_b200", "bench"}, (path, mods)
    # no C or CUDA source reaches into the oracle either
    for path in glob.glob(os.path.join(ROOT, "ternary_weight_matmul_b200", "csrc", "*")):
        assert "oracle" not in open(path, errors="replace").read().lower(), path


def test_oracle_reached_only_from_tests_smoke_and_the_cpu_baseline():
    mods, by_fn = _imports(os.path.join(ROOT, "bench.py"))
    users = sorted(fn for fn, inner in by_fn.items() if "oracle" in inner)
    assert users == ["oracle_sample_tokens_per_s"], users
    mods, by_fn = _imports(os.path.join(ROOT, "__graft_entry__.py"))
    assert sorted(fn for fn, inner in by_fn.items() if "oracle" in inner) == ["smoke"]
    # nothing else at the top level of the repository imports it
    for path in glob.glob(os.path.join(ROOT, "*.py")):
        if os.path.basename(path) in ("bench.py", "__graft_entry__.py"):
            continue
        assert "oracle" not in _imports(path)[0], path


def test_missing_library_raises(monkeypatch):
    monkeypatch.setattr(mmf, "_lib", None)
    monkeypatch.setattr(mmf, "LIB_PATH", os.path.join(ROOT, "no_such_dir", "libmmf.so"))
    with pytest.raises(ImportError, match="no fallback"):
        mmf.lib()


# C parameter type -> (is pointer, byte width, is floating point)
_C_TYPES = {
    "int32_t": (False, 4, False), "uint32_t": (False, 4, False), "int64_t": (False, 8, False),
    "size_t": (False, 8, False), "float": (False, 4, True), "int": (False, 4, False),
    "mmf_dtype": (False, 4, False), "mmf_op": (False, 4, False), "mmf_status": (False, 4, False),
    "mmf_gemm_path": (False, 4, False), "mmf_decode_path": (False, 4, False),
    "mmf_kernel_class": (False, 4, False), "mmf_stream_t": (True, 8, False),
}


def _header_signatures():
    text = open(os.path.join(ROOT, "include", "mmf.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    sigs = {}
    for m in re.finditer(r"\b(mmf_[a-z_0-9]+)\s*\(([^()]*)\)\s*;", text):
        params = [p.strip() for p in m.group(2).split(",") if p.strip()]
        if params == ["void"]:
            params = []
        kinds = []
        for p in params:
            if "*" in p:
                kinds.append((True, 8, False))
                continue
            base = re.sub(r"\bconst\b", "", p).split()[0]
            kinds.append(_C_TYPES[base])
        sigs[m.group(1)] = kinds
    return sigs


def _ctypes_kind(t):
    if t in (ctypes.c_void_p, ctypes.c_char_p) or (isinstance(t, type) and issubclass(t, ctypes._Pointer)):
        return (True, 8, False)
    return (False, ctypes.sizeof(t), t in (ctypes.c_float, ctypes.c_double))


def test_binding_signatures_match_the_header():
    mbuild.build()
    L = mmf.lib()
    sigs = _header_signatures()
    assert set(sigs) == set(mmf.EXPORTED)
    for name, kinds in sigs.items():
        argtypes = getattr(L, name).argtypes or []
        got = [_ctypes_kind(t) for t in argtypes]
        assert got == kinds, f"{name}: binding {got} vs header {kinds}"
