"""The C-ABI library loads without a GPU and exports every function include/mk.h declares."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "mk.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*(mk_[a-z_]+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("mk_create", "mk_decode_step", "mk_get_status", "mk_destroy", "mk_status_string",
                     "mk_read_state", "mk_decode_step_noalloc", "mk_decode_greedy", "mk_plan_create"):
        assert required in names


def test_library_exports_every_declared_symbol():
    from auto_regressive_decode_b200 import build
    lib = ctypes.CDLL(build.build())
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_status_strings_and_null_handles():
    import auto_regressive_decode_b200.mk as mk
    for code in (mk.MK_OK, mk.MK_ERR_INVALID_ARG, mk.MK_ERR_UNSUPPORTED, mk.MK_ERR_CUDA, mk.MK_ERR_DEVICE_TIMEOUT,
                 mk.MK_ERR_RANGE):
        assert mk.mk_status_string(code) and mk.mk_status_string(code) != "unknown status"
    assert mk.mk_destroy(None) == mk.MK_OK
    assert mk.mk_get_status(None, None) == mk.MK_ERR_INVALID_ARG
    assert mk.mk_decode_step(None, None, None, None, None, None) == mk.MK_ERR_INVALID_ARG
    assert mk.mk_create(None, None, None, None) == mk.MK_ERR_INVALID_ARG
    assert mk.mk_decode_greedy(None, 1, None, None, None, None, None) == mk.MK_ERR_INVALID_ARG


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    import importlib.util
    src = os.path.join(ROOT, "auto_regressive_decode_b200", "mk.py")
    spec = importlib.util.spec_from_file_location("mk_copy", str(tmp_path / "mk.py"))
    (tmp_path / "mk.py").write_text(open(src).read())
    mod = importlib.util.module_from_spec(spec)
    with pytest.raises(ImportError):
        spec.loader.exec_module(mod)
