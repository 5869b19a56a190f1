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


def test_misaligned_workspace_rejected_without_gpu():
    """A workspace that is not 16-byte aligned is refused (SAP_ERR_WORKSPACE) by the forward and the
    merge before any device work: the kernels store and load the partials as 16-byte vectors.  The
    pointers are never dereferenced; the checks run on the host before the first CUDA call."""
    lib = sap.load_library()
    plan = sap.sap_plan([0, 512], 512, 2)  # q tiles 2 and 3 see both chunks: partial slots exist
    assert sap.sap_plan_stats(plan)["n_partial_slots"] > 0
    need = sap.sap_workspace_size(plan, 2, 1, 64, sap.SAP_WS_FWD)
    fake = ctypes.c_void_p(1 << 20)  # 16-byte aligned, never dereferenced
    bad_ws = ctypes.c_void_p((1 << 21) + 8)
    st = lib.sap_attn_fwd(plan.handle, fake, fake, fake, 2, 1, 64, 0.125, fake, fake, bad_ws, need + 64, None)
    assert st == -4
    st = lib.sap_merge(plan.handle, bad_ws, need + 64, 2, 64, fake, fake, None)
    assert st == -4


def test_wait_limit_arguments_checked_without_gpu():
    lib = sap.load_library()
    assert lib.sap_set_wait_limit_ns(10) == -1          # below 1 ms
    assert lib.sap_set_wait_limit_ns(0) == 0            # default restored
    assert lib.sap_test_arm_wait_timeout(0) == -1       # below 100 us
    assert lib.sap_test_arm_wait_timeout(11_000_000_000) == -1


def test_forward_variant_argument_checked_without_gpu():
    lib = sap.load_library()
    assert lib.sap_set_forward_variant(2) == -1
    assert lib.sap_set_forward_variant(-1) == -1
    assert lib.sap_set_forward_variant(0) == 0


def test_kv_add_refuses_a_full_plan_without_gpu():
    """sap_attn_bwd_kv_add takes rank plans only: a full plan's backward stores the dK/dV of kv
    tiles with a single unit directly and never writes their accumulator rows.  The refusal comes
    before any device work (the pointers are never dereferenced)."""
    lib = sap.load_library()
    plan = sap.sap_plan([0, 300, 512], 512, 2)
    assert sap.sap_plan_bwd_direct(plan).tolist() == [1, 1, 1, 1]
    rank = sap.sap_plan_rank(plan, 1)
    assert sap.sap_plan_bwd_direct(rank).tolist() == [0, 0, 0, 0]  # window: kv tiles 0..3 (token 256 is in doc 0)
    fake = ctypes.c_void_p(1 << 20)
    st = lib.sap_attn_bwd_kv_add(plan.handle, fake, 1 << 30, 2, 1, 64, fake, fake, 0, 128, fake, fake, None)
    assert st == -1
