"""The C ABI library loads and exports every entry point include/sap.h declares
(CPU only: no compute call is made)."""
import ctypes
import os
import re

import packed_sequence_causal_b200 as sap

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if not fn.endswith(".h"):
            continue
        text = open(os.path.join(ROOT, "include", fn)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names |= set(re.findall(r"\b(sap_[a-z0-9_]+)\s*\(", text))
    return names


def test_every_declared_symbol_is_exported():
    lib = ctypes.CDLL(sap.library_path())
    declared = _declared()
    assert "sap_attn_fwd" in declared and "sap_plan" in declared
    for name in sorted(declared):
        assert hasattr(lib, name), name


def test_error_strings():
    for st in range(0, -9, -1):
        assert sap.sap_error_string(st) != "unknown status"
    assert sap.sap_error_string(-100) == "unknown status"


def test_null_arguments_rejected_without_gpu():
    lib = sap.load_library()
    assert lib.sap_plan(None, 0, 0, 1, 128, 128, None) == -1
    assert lib.sap_plan_items(None, None, None) == -1
    assert lib.sap_workspace_size(None, 1, 1, 64, 0, None) == -1
