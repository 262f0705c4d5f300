"""The C-ABI library builds, loads and exports every declared entry point (no GPU needed)."""
import ctypes
import os
import re

import pytest

import step_flow_map_b200 as fmb
from step_flow_map_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "flashmap.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(fm_[a-z_]+)\s*\(", src)))


def test_header_declares_the_binding_names():
    assert set(_declared()) == set(fmb.EXPORTS)


def test_library_exports_every_declared_symbol():
    path = build.build()
    lib = ctypes.CDLL(path)
    for name in _declared():
        assert hasattr(lib, name), name
    assert fmb.load_library() is not None
    assert isinstance(fmb.fm_last_error(), str)


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(FileNotFoundError):
        fmb._lib_backup = fmb._lib
        fmb._lib = None
        try:
            fmb.load_library(str(tmp_path / "nope.so"))
        finally:
            fmb._lib = fmb._lib_backup
