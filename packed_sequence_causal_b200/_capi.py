"""ctypes marshalling for libsap.so.  Names follow the C entry points."""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libsap.so")

SAP_OK = 0
SAP_TAG_FULL, SAP_TAG_CAUSAL, SAP_TAG_MASKED = 0, 1, 2
SAP_WS_FWD, SAP_WS_BWD = 0, 1

_lib = None


class SapError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        msg = sap_error_string(status) if _lib is not None else str(status)
        extra = ""
        if status == -5 and _lib is not None:
            extra = f" (cudaError {_lib.sap_last_cuda_error()})"
        super().__init__(f"{what}: {msg} [{status}]{extra}")


def library_path() -> str:
    return _LIB_PATH


def load_library():
    """Load libsap.so (built by ``python -m packed_sequence_causal_b200.build``); raises if absent."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise RuntimeError(f"libsap.so is not built ({_LIB_PATH}); run: python -m packed_sequence_causal_b200.build")
    L = ctypes.CDLL(_LIB_PATH)
    P, i32, i64, f32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
    PP = ctypes.POINTER(ctypes.c_void_p)
    L.sap_plan.restype = ctypes.c_int
    L.sap_plan.argtypes = [P, i32, i64, i32, i32, i32, PP]
    L.sap_plan_chunks.restype = ctypes.c_int
    L.sap_plan_chunks.argtypes = [P, i32, i64, P, i32, i32, i32, PP]
    L.sap_balanced_chunks.restype = ctypes.c_int
    L.sap_balanced_chunks.argtypes = [P, i32, i64, i32, i32, P]
    L.sap_plan_chunk_bounds.restype = ctypes.c_int
    L.sap_plan_chunk_bounds.argtypes = [P, PP, ctypes.POINTER(i32)]
    L.sap_plan_chunk_stats.restype = ctypes.c_int
    L.sap_plan_chunk_stats.argtypes = [P, P, P]
    L.sap_plan_rank.restype = ctypes.c_int
    L.sap_plan_rank.argtypes = [P, i32, PP]
    L.sap_plan_window.restype = ctypes.c_int
    L.sap_plan_window.argtypes = [P] + [ctypes.POINTER(i64)] * 4
    L.sap_plan_rank_spans.restype = ctypes.c_int
    L.sap_plan_rank_spans.argtypes = [P, i32, P, ctypes.POINTER(i32)]
    L.sap_workspace_kv_offsets.restype = ctypes.c_int
    L.sap_workspace_kv_offsets.argtypes = [P, i32, i32, i32, ctypes.POINTER(sz), ctypes.POINTER(sz)]
    L.sap_attn_bwd_kv_add.restype = ctypes.c_int
    L.sap_attn_bwd_kv_add.argtypes = [P, P, sz, i32, i32, i32, P, P, i64, i64, P, P, P]
    L.sap_plan_items.restype = ctypes.c_int
    L.sap_plan_items.argtypes = [P, PP, ctypes.POINTER(i64)]
    L.sap_plan_stats.restype = ctypes.c_int
    L.sap_plan_stats.argtypes = [P, ctypes.POINTER(i64), ctypes.POINTER(i64), ctypes.POINTER(i32)]
    L.sap_plan_fwd_schedule.restype = ctypes.c_int
    L.sap_plan_fwd_schedule.argtypes = [P, PP, ctypes.POINTER(i64), PP, PP, ctypes.POINTER(i64)]
    L.sap_plan_bwd_schedule.restype = ctypes.c_int
    L.sap_plan_bwd_schedule.argtypes = [P, PP, ctypes.POINTER(i64), PP]
    L.sap_plan_bwd_direct.restype = ctypes.c_int
    L.sap_plan_bwd_direct.argtypes = [P, PP, ctypes.POINTER(i64)]
    L.sap_plan_set_fused_merge.restype = ctypes.c_int
    L.sap_plan_set_fused_merge.argtypes = [P, ctypes.c_int]
    L.sap_plan_upload.restype = ctypes.c_int
    L.sap_plan_upload.argtypes = [P, P]
    L.sap_plan_destroy.restype = None
    L.sap_plan_destroy.argtypes = [P]
    L.sap_workspace_size.restype = ctypes.c_int
    L.sap_workspace_size.argtypes = [P, i32, i32, i32, i32, ctypes.POINTER(sz)]
    L.sap_attn_fwd.restype = ctypes.c_int
    L.sap_attn_fwd.argtypes = [P, P, P, P, i32, i32, i32, f32, P, P, P, sz, P]
    L.sap_attn_fwd_part.restype = ctypes.c_int
    L.sap_attn_fwd_part.argtypes = [P, i32, i32, P, P, P, i32, i32, i32, f32, P, P, P, sz, P]
    L.sap_plan_fwd_local_units.restype = ctypes.c_int
    L.sap_plan_fwd_local_units.argtypes = [P, ctypes.POINTER(i64), ctypes.POINTER(i64)]
    L.sap_merge.restype = ctypes.c_int
    L.sap_merge.argtypes = [P, P, sz, i32, i32, P, P, P]
    L.sap_attn_bwd.restype = ctypes.c_int
    L.sap_attn_bwd.argtypes = [P, P, P, P, P, P, P, i32, i32, i32, f32, P, P, P, P, sz, P]
    L.sap_attn_fwd_static_scratch.restype = ctypes.c_int
    L.sap_attn_fwd_static_scratch.argtypes = [P, P, P, P, i32, i32, i32, f32, P, P, P]
    L.sap_device_status.restype = ctypes.c_int
    L.sap_device_status.argtypes = [ctypes.POINTER(i32)]
    L.sap_error_string.restype = ctypes.c_char_p
    L.sap_error_string.argtypes = [ctypes.c_int]
    L.sap_last_cuda_error.restype = ctypes.c_int
    L.sap_last_cuda_error.argtypes = []
    L.sap_set_wait_limit_ns.restype = ctypes.c_int
    L.sap_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
    L.sap_set_forward_variant.restype = ctypes.c_int
    L.sap_set_forward_variant.argtypes = [i32]
    L.sap_test_arm_wait_timeout.restype = ctypes.c_int
    L.sap_test_arm_wait_timeout.argtypes = [ctypes.c_uint64]
    _lib = L
    return L


def _check(status: int, what: str):
    if status != SAP_OK:
        raise SapError(status, what)


def sap_error_string(status: int) -> str:
    return load_library().sap_error_string(status).decode()


class Plan:
    """Owner of a sap_plan_t handle (destroyed with the object)."""

    def __init__(self, handle: int, n: int, num_chunks: int, block_m: int, block_n: int):
        self.handle = ctypes.c_void_p(handle)
        self.n, self.num_chunks, self.block_m, self.block_n = n, num_chunks, block_m, block_n

    def __del__(self):
        if _lib is not None and self.handle:
            _lib.sap_plan_destroy(self.handle)
            self.handle = ctypes.c_void_p()

    def destroy(self):
        self.__del__()


def sap_plan(cu_seqlens, total_tokens: int, num_chunks: int, block_m: int = 128, block_n: int = 128) -> Plan:
    L = load_library()
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
    h = ctypes.c_void_p()
    _check(L.sap_plan(cu.ctypes.data_as(ctypes.c_void_p), len(cu) - 1, int(total_tokens), int(num_chunks),
                      int(block_m), int(block_n), ctypes.byref(h)), "sap_plan")
    return Plan(h.value, int(total_tokens), int(num_chunks), int(block_m), int(block_n))


def sap_plan_chunks(cu_seqlens, total_tokens: int, chunk_bounds, block_m: int = 128, block_n: int = 128) -> Plan:
    """Plan over explicit contiguous chunks [bounds[c], bounds[c+1])."""
    L = load_library()
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
    b = np.ascontiguousarray(np.asarray(chunk_bounds, dtype=np.int64))
    h = ctypes.c_void_p()
    _check(L.sap_plan_chunks(cu.ctypes.data_as(ctypes.c_void_p), len(cu) - 1, int(total_tokens),
                             b.ctypes.data_as(ctypes.c_void_p), len(b) - 1, int(block_m), int(block_n),
                             ctypes.byref(h)), "sap_plan_chunks")
    return Plan(h.value, int(total_tokens), len(b) - 1, int(block_m), int(block_n))


def sap_balanced_chunks(cu_seqlens, total_tokens: int, num_chunks: int, block: int = 128) -> np.ndarray:
    """Balanced contiguous chunk bounds (int64, num_chunks + 1 entries)."""
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
    out = np.zeros(int(num_chunks) + 1, dtype=np.int64)
    _check(load_library().sap_balanced_chunks(cu.ctypes.data_as(ctypes.c_void_p), len(cu) - 1, int(total_tokens),
                                              int(num_chunks), int(block), out.ctypes.data_as(ctypes.c_void_p)),
           "sap_balanced_chunks")
    return out


def sap_plan_chunk_bounds(plan: Plan) -> np.ndarray:
    p, n = ctypes.c_void_p(), ctypes.c_int32()
    _check(load_library().sap_plan_chunk_bounds(plan.handle, ctypes.byref(p), ctypes.byref(n)),
           "sap_plan_chunk_bounds")
    return np.ctypeslib.as_array(ctypes.cast(p, ctypes.POINTER(ctypes.c_int64)), shape=(n.value + 1,)).copy()


def sap_plan_chunk_stats(plan: Plan) -> dict:
    """Per q chunk: items and unmasked pairs (int64 arrays of num_chunks entries)."""
    nc = len(sap_plan_chunk_bounds(plan)) - 1
    items = np.zeros(nc, dtype=np.int64)
    pairs = np.zeros(nc, dtype=np.int64)
    _check(load_library().sap_plan_chunk_stats(plan.handle, items.ctypes.data_as(ctypes.c_void_p),
                                               pairs.ctypes.data_as(ctypes.c_void_p)), "sap_plan_chunk_stats")
    return {"items": items, "pairs": pairs}


def sap_plan_rank(plan: Plan, chunk: int) -> Plan:
    """Rank plan of q chunk `chunk` (windowed buffers, see sap_plan_window)."""
    h = ctypes.c_void_p()
    _check(load_library().sap_plan_rank(plan.handle, int(chunk), ctypes.byref(h)), "sap_plan_rank")
    return Plan(h.value, plan.n, plan.num_chunks, plan.block_m, plan.block_n)


def sap_plan_window(plan: Plan) -> dict:
    """q_begin, q_end, kv_begin, span_begin of the plan's buffer window (global token indices)."""
    v = [ctypes.c_int64() for _ in range(4)]
    _check(load_library().sap_plan_window(plan.handle, *[ctypes.byref(x) for x in v]), "sap_plan_window")
    return dict(zip(("q_begin", "q_end", "kv_begin", "span_begin"), (x.value for x in v)))


def sap_plan_rank_spans(plan: Plan, chunk: int) -> np.ndarray:
    """Token ranges the owner of `chunk` receives: int64 [n, 3] = (source chunk, lo, hi)."""
    nc = plan.num_chunks
    out = np.zeros((max(nc, 1), 3), dtype=np.int64)
    n = ctypes.c_int32()
    _check(load_library().sap_plan_rank_spans(plan.handle, int(chunk), out.ctypes.data_as(ctypes.c_void_p),
                                              ctypes.byref(n)), "sap_plan_rank_spans")
    return out[: n.value].copy()


def sap_plan_destroy(plan: Plan):
    plan.destroy()


def _copy_i32(ptr, count: int, width: int) -> np.ndarray:
    if count == 0:
        return np.zeros((0, width) if width > 1 else (0,), dtype=np.int32)
    arr = np.ctypeslib.as_array(ctypes.cast(ptr, ctypes.POINTER(ctypes.c_int32)), shape=(count * width,)).copy()
    return arr.reshape(count, width) if width > 1 else arr


def sap_plan_items(plan: Plan) -> np.ndarray:
    """Canonical items, int32 [n, 5] = (q_tile, kv_tile, q_chunk, kv_chunk, tag)."""
    p, n = ctypes.c_void_p(), ctypes.c_int64()
    _check(load_library().sap_plan_items(plan.handle, ctypes.byref(p), ctypes.byref(n)), "sap_plan_items")
    return _copy_i32(p, n.value, 5)


def sap_plan_stats(plan: Plan) -> dict:
    a, b, c = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int32()
    _check(load_library().sap_plan_stats(plan.handle, ctypes.byref(a), ctypes.byref(b), ctypes.byref(c)),
           "sap_plan_stats")
    return {"unmasked_pairs": a.value, "n_partial_slots": b.value, "n_chunk_pairs": c.value}


def sap_plan_fwd_schedule(plan: Plan):
    """(units [U,4], order [U], merges [M,3]) as int32 arrays."""
    u, nu, o, m, nm = ctypes.c_void_p(), ctypes.c_int64(), ctypes.c_void_p(), ctypes.c_void_p(), ctypes.c_int64()
    _check(load_library().sap_plan_fwd_schedule(plan.handle, ctypes.byref(u), ctypes.byref(nu), ctypes.byref(o),
                                                 ctypes.byref(m), ctypes.byref(nm)), "sap_plan_fwd_schedule")
    return _copy_i32(u, nu.value, 4), _copy_i32(o, nu.value, 1), _copy_i32(m, nm.value, 3)


def sap_plan_bwd_schedule(plan: Plan):
    """(kv_units [V,3], entries [items,2]) as int32 arrays."""
    k, nk, e = ctypes.c_void_p(), ctypes.c_int64(), ctypes.c_void_p()
    _check(load_library().sap_plan_bwd_schedule(plan.handle, ctypes.byref(k), ctypes.byref(nk), ctypes.byref(e)),
           "sap_plan_bwd_schedule")
    n_items = len(sap_plan_items(plan))
    return _copy_i32(k, nk.value, 3), _copy_i32(e, n_items, 2)


def sap_plan_bwd_direct(plan: Plan) -> np.ndarray:
    """int32 [kv tiles of the window]: 1 where sap_attn_bwd stores the tile's dK/dV directly."""
    f, nt = ctypes.c_void_p(), ctypes.c_int64()
    _check(load_library().sap_plan_bwd_direct(plan.handle, ctypes.byref(f), ctypes.byref(nt)), "sap_plan_bwd_direct")
    return _copy_i32(f, nt.value, 1)


def _stream_ptr(stream) -> Optional[int]:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def sap_plan_set_fused_merge(plan: Plan, enable: bool = True):
    _check(load_library().sap_plan_set_fused_merge(plan.handle, int(bool(enable))), "sap_plan_set_fused_merge")


def sap_plan_upload(plan: Plan, stream=None):
    _check(load_library().sap_plan_upload(plan.handle, ctypes.c_void_p(_stream_ptr(stream))), "sap_plan_upload")


def sap_workspace_size(plan: Plan, hq: int, hkv: int, head_dim: int, which: int) -> int:
    b = ctypes.c_size_t()
    _check(load_library().sap_workspace_size(plan.handle, hq, hkv, head_dim, which, ctypes.byref(b)),
           "sap_workspace_size")
    return b.value


def alloc_workspace(plan: Plan, hq: int, hkv: int, head_dim: int, which: int, device="cuda"):
    """Caller-owned workspace as a uint8 torch tensor of sap_workspace_size bytes."""
    import torch
    nbytes = sap_workspace_size(plan, hq, hkv, head_dim, which)
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p()


def _nbytes(t):
    return 0 if t is None else t.numel() * t.element_size()


def _bf16_3d(t, name):
    import torch
    if t.dtype != torch.bfloat16 or t.dim() != 3 or not t.is_contiguous() or not t.is_cuda:
        raise ValueError(f"{name} must be a contiguous CUDA bf16 tensor [N, heads, head_dim]")


def sap_attn_fwd(plan: Plan, q, k, v, softmax_scale: float, o, lse, workspace, stream=None):
    for t, nme in ((q, "q"), (k, "k"), (v, "v"), (o, "o")):
        _bf16_3d(t, nme)
    _, hq, d = q.shape
    hkv = k.shape[1]
    _check(load_library().sap_attn_fwd(plan.handle, _ptr(q), _ptr(k), _ptr(v), hq, hkv, d, float(softmax_scale),
                                       _ptr(o), _ptr(lse), _ptr(workspace), _nbytes(workspace),
                                       ctypes.c_void_p(_stream_ptr(stream))), "sap_attn_fwd")


def sap_attn_fwd_part(plan: Plan, part: int, q, k, v, softmax_scale: float, o, lse, workspace, stream=None,
                      max_ctas: int = 0):
    """One part of the forward (1: own-chunk units of a rank plan, 2: the others, 0: all)."""
    for t, nme in ((q, "q"), (k, "k"), (v, "v"), (o, "o")):
        _bf16_3d(t, nme)
    _, hq, d = q.shape
    hkv = k.shape[1]
    _check(load_library().sap_attn_fwd_part(plan.handle, int(part), int(max_ctas), _ptr(q), _ptr(k), _ptr(v), hq,
                                            hkv, d, float(softmax_scale), _ptr(o), _ptr(lse), _ptr(workspace),
                                            _nbytes(workspace), ctypes.c_void_p(_stream_ptr(stream))),
           "sap_attn_fwd_part")


def sap_plan_fwd_local_units(plan: Plan):
    """(n_local, n_units): forward units, and those of a rank plan's own chunk (listed first)."""
    a, b = ctypes.c_int64(), ctypes.c_int64()
    _check(load_library().sap_plan_fwd_local_units(plan.handle, ctypes.byref(a), ctypes.byref(b)),
           "sap_plan_fwd_local_units")
    return a.value, b.value


def sap_merge(plan: Plan, workspace, hq: int, head_dim: int, o, lse, stream=None):
    _check(load_library().sap_merge(plan.handle, _ptr(workspace), _nbytes(workspace), hq, head_dim, _ptr(o),
                                    _ptr(lse), ctypes.c_void_p(_stream_ptr(stream))), "sap_merge")


def sap_attn_bwd(plan: Plan, q, k, v, o, lse, dout, softmax_scale: float, dq, dk, dv, workspace, stream=None):
    for t, nme in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (dout, "dout"), (dq, "dq"), (dk, "dk"), (dv, "dv")):
        _bf16_3d(t, nme)
    _, hq, d = q.shape
    hkv = k.shape[1]
    _check(load_library().sap_attn_bwd(plan.handle, _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout), hq,
                                       hkv, d, float(softmax_scale), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace),
                                       _nbytes(workspace), ctypes.c_void_p(_stream_ptr(stream))), "sap_attn_bwd")


def sap_workspace_kv_offsets(plan: Plan, hq: int, hkv: int, head_dim: int):
    """(dk_offset, dv_offset): byte offsets of the fp32 dK / dV accumulators in the backward workspace."""
    a, b = ctypes.c_size_t(), ctypes.c_size_t()
    _check(load_library().sap_workspace_kv_offsets(plan.handle, hq, hkv, head_dim, ctypes.byref(a), ctypes.byref(b)),
           "sap_workspace_kv_offsets")
    return a.value, b.value


def sap_attn_bwd_kv_add(plan: Plan, workspace, hq: int, dk_part, dv_part, row_begin: int, dk, dv, stream=None):
    """Add fp32 dK/dV partials for tokens [row_begin, row_begin + rows) into the backward's accumulators
    and rewrite those rows of the bf16 dk, dv."""
    import torch
    for t, nme in ((dk_part, "dk_part"), (dv_part, "dv_part")):
        if t.dtype != torch.float32 or t.dim() != 3 or not t.is_contiguous() or not t.is_cuda:
            raise ValueError(f"{nme} must be a contiguous CUDA fp32 tensor [rows, hkv, head_dim]")
    rows, hkv, d = dk_part.shape
    _check(load_library().sap_attn_bwd_kv_add(plan.handle, _ptr(workspace), _nbytes(workspace), hq, hkv, d,
                                              _ptr(dk_part), _ptr(dv_part), int(row_begin), int(rows), _ptr(dk),
                                              _ptr(dv), ctypes.c_void_p(_stream_ptr(stream))), "sap_attn_bwd_kv_add")


def sap_attn_fwd_static_scratch(plan: Plan, q, k, v, softmax_scale: float, o, lse, stream=None):
    """Forward + merge with the partials in the library's own 16 MiB device array (no allocation).

    For callers that cannot allocate device memory; the plan must already be
    uploaded to the current device, and calls must not overlap on one GPU."""
    for t, nme in ((q, "q"), (k, "k"), (v, "v"), (o, "o")):
        _bf16_3d(t, nme)
    _, hq, d = q.shape
    hkv = k.shape[1]
    _check(load_library().sap_attn_fwd_static_scratch(plan.handle, _ptr(q), _ptr(k), _ptr(v), hq, hkv, d,
                                                      float(softmax_scale), _ptr(o), _ptr(lse),
                                                      ctypes.c_void_p(_stream_ptr(stream))),
           "sap_attn_fwd_static_scratch")


def sap_device_status() -> int:
    """Synchronises; returns the device error word (0 = clean) and clears it."""
    c = ctypes.c_int32()
    st = load_library().sap_device_status(ctypes.byref(c))
    if st not in (SAP_OK, -6):
        raise SapError(st, "sap_device_status")
    return c.value


def sap_set_wait_limit_ns(limit_ns: int):
    """Pipeline wait limit of later kernel launches (0: the default 4 s)."""
    _check(load_library().sap_set_wait_limit_ns(int(limit_ns)), "sap_set_wait_limit_ns")


def sap_set_forward_variant(variant: int):
    """Forward kernel variant of later calls: 0 one CTA per work item, 1 two-CTA clusters (cta_group::2)."""
    _check(load_library().sap_set_forward_variant(int(variant)), "sap_set_forward_variant")
