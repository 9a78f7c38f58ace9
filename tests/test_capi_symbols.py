"""The C-ABI library builds, loads without a GPU, and exports every entry
point that include/ai_index.h declares."""
import ctypes
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "ai_index.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(ai_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_core_calls():
    names = declared_symbols()
    for core in ["ai_index_create", "ai_append_keys", "ai_seal", "ai_refit", "ai_route_refine",
                 "ai_select_exhaustive"]:
        assert core in names


def test_library_exports_every_declared_symbol():
    import __graft_entry__
    lib_path = __graft_entry__._build_module().build()
    lib = ctypes.CDLL(lib_path)
    missing = [n for n in declared_symbols() if not hasattr(lib, n)]
    assert not missing, missing


def test_binding_wraps_every_declared_symbol():
    from ivf_top_key_b200 import _capi
    assert sorted(_capi.EXPORTED) == declared_symbols()


def declared_arities():
    """Parameter count of every entry point's prototype in the header."""
    src = open(os.path.join(ROOT, "include", "ai_index.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    out = {}
    for name, params in re.findall(r"\b(ai_[a-z0-9_]+)\s*\(([^;{]*?)\)\s*;", src, flags=re.S):
        p = " ".join(params.split())
        out[name] = 0 if p in ("", "void") else p.count(",") + 1
    return out


def test_binding_argument_counts_match_the_header():
    """Every ctypes prototype in the binding takes as many arguments as the
    C declaration (a dropped or added parameter would shift every later
    argument silently)."""
    from ivf_top_key_b200 import _capi
    ar = declared_arities()
    assert sorted(ar) == declared_symbols()
    for name, n in ar.items():
        f = getattr(_capi._lib, name)
        assert f.argtypes is not None, name
        assert len(f.argtypes) == n, (name, len(f.argtypes), n)
