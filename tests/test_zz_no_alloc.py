"""The allocation-free forward entry point (sap_attn_fwd_static_scratch).

Some callers cannot call cudaMalloc -- a framework that owns all device memory
through its own pool, or a plugin handed only input and output pointers.  For
them the library offers one forward + merge call whose scratch (the partial
outputs and LSEs) is a 16 MiB array compiled into the library.  These tests
call it through the C ABI.

The array keeps whatever the previous call left in it, so before the checked
calls it is filled by a call on other data (other seeded inputs and the other
head dimension, whose partial slots overlap the checked ones).  Each checked
call must then give exactly the bytes of the regular entry points on the same
inputs (the same deterministic kernels and schedule; the forward has no
atomics), and must match the oracle within the parity bounds of the other GPU
tests.  This file is collected last on purpose.
"""
import ctypes

import pytest
import torch

import oracle
import packed_sequence_causal_b200 as sap
import workloads
from gpu_helpers import Run, assert_close, assert_lse

pytestmark = pytest.mark.gpu


def _static_call(lib, r, d):
    o = torch.full_like(r.o, float("nan"))
    lse = torch.full_like(r.lse, float("nan"))
    st = lib.sap_attn_fwd_static_scratch(r.plan.handle, ctypes.c_void_p(r.q.data_ptr()),
                                         ctypes.c_void_p(r.k.data_ptr()), ctypes.c_void_p(r.v.data_ptr()), r.hq,
                                         r.hkv, d, r.scale, ctypes.c_void_p(o.data_ptr()),
                                         ctypes.c_void_p(lse.data_ptr()),
                                         ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, sap.sap_error_string(st)
    assert sap.sap_device_status() == 0
    return o, lse


@pytest.mark.parametrize("d", [64, 128])
def test_static_scratch_forward_matches_workspace_forward(d):
    lib = sap.load_library()
    # 2048 tokens, P = 4: most q tiles see several kv chunks, so the partials and the merge are used
    lens = [1500, 300, 248]
    # fill the shared array first: other inputs, other head dimension, same slot layout
    other = Run(workloads.custom_batch(lens, 4, 2, 192 - d, seed=77, with_do=False), 4)
    other.fwd()  # uploads the plan
    _static_call(lib, other, 192 - d)

    b = workloads.custom_batch(lens, 4, 2, d, seed=31, with_do=False)
    r = Run(b, 4)
    ref_o, ref_lse = r.fwd()  # regular entry points (caller-owned workspace); also uploads the plan
    ref_o, ref_lse = ref_o.clone(), ref_lse.clone()
    need = sap.sap_workspace_size(r.plan, 4, 2, d, sap.SAP_WS_FWD)
    assert 0 < need <= 16 << 20
    oo, ol = oracle.attn_fwd(b.q, b.k, b.v, b.cu_seqlens, r.scale)
    for _ in range(2):  # two calls in a row on the same array
        o, lse = _static_call(lib, r, d)
        assert torch.equal(o, ref_o), "O differs from the workspace path"
        assert torch.equal(lse[:, : r.n], ref_lse), "LSE differs from the workspace path"
        assert_close(o, oo, "O (static scratch)")
        assert_lse(lse[:, : r.n], ol, "LSE (static scratch)")


def test_static_scratch_rejects_oversize_and_unuploaded_plans():
    lib = sap.load_library()
    # forward workspace of a 32K-token, 32-head plan is far above 16 MiB
    w = workloads.WORKLOADS["llama32_1b_32k"]
    cu = workloads.cu_seqlens_from_lengths(workloads.doc_lengths(w, 0))
    big = sap.sap_plan(cu, w.n, w.p)
    assert sap.sap_workspace_size(big, 32, 8, 64, sap.SAP_WS_FWD) > 16 << 20
    sap.sap_plan_upload(big)
    dummy = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    args = [ctypes.c_void_p(dummy.data_ptr())] * 3 + [32, 8, 64, 0.125, ctypes.c_void_p(dummy.data_ptr()),
                                                      ctypes.c_void_p(dummy.data_ptr()), None]
    assert lib.sap_attn_fwd_static_scratch(big.handle, *args) == -4  # SAP_ERR_WORKSPACE
    # a plan that was never uploaded is refused rather than uploaded (that would allocate)
    small = sap.sap_plan([0, 256], 256, 1)
    args = [ctypes.c_void_p(dummy.data_ptr())] * 3 + [2, 2, 64, 0.125, ctypes.c_void_p(dummy.data_ptr()),
                                                      ctypes.c_void_p(dummy.data_ptr()), None]
    assert lib.sap_attn_fwd_static_scratch(small.handle, *args) == -1  # SAP_ERR_INVALID_ARG
    assert sap.sap_device_status() == 0
