"""Sequence-aware parallelism across ranks on CPU (gloo, world sizes 2 and 4): the SAP exchange,
the Ulysses head split and their hierarchy (HSAP), with the oracle as every rank's local
computation.

Each rank runs the product's exchange code (packed_sequence_causal_b200.sap_dist: the planner's
exchange lists, point-to-point transfers of key/value spans, the return of dK/dV partials, the
Ulysses all-to-alls); the test replaces only the three local compute steps -- on a GPU they are
the library's kernels -- by the fp64 oracle over the rank's window.  Every rank's O, LSE, dQ, dK
and dV must equal the unsplit oracle on the same batch to 1e-12, and the key/value bytes that
crossed ranks must equal the planner's spans (less than a ring that passes every chunk).
"""
import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
import packed_sequence_causal_b200 as sap
import workloads
from packed_sequence_causal_b200 import sap_dist

LENS = [700, 60, 1500, 300, 37, 900, 599]  # 4096 tokens: documents across several chunk bounds
HQ, HKV, D = 4, 2, 16


def _window_batch(self):
    kv0, q0, q1 = self.window["kv_begin"], self.window["q_begin"], self.window["q_end"]
    cu = np.clip(self.cu.astype(np.int64), kv0, q1) - kv0
    return kv0, q0, q1, cu.astype(np.int32)


class OracleSap(sap_dist.SapAttention):
    """SapAttention whose local steps are the fp64 oracle over the rank's window (test only)."""

    def attend(self, q, k_win, v_win, part=0):
        if part == 1:  # the own-chunk part runs while the exchange is in flight; the oracle does it all below
            return None
        kv0, q0, q1, cu = _window_batch(self)
        qw = torch.zeros(k_win.shape[:1] + q.shape[1:], dtype=torch.float64)
        qw[q0 - kv0:] = q  # window rows before the chunk are not this rank's queries
        o, lse = oracle.attn_fwd(qw, k_win, v_win, cu, self.scale)
        self._qw, self._k, self._v, self._cu = qw, k_win, v_win, cu
        return torch.from_numpy(o[q0 - kv0:]), torch.from_numpy(lse[:, q0 - kv0:].copy())

    def local_backward(self, do):
        kv0, q0, q1, _ = _window_batch(self)
        dow = torch.zeros_like(self._qw)
        dow[q0 - kv0:] = do  # zero dO: the window's other rows add nothing
        dq, dk, dv = oracle.attn_bwd(self._qw, self._k, self._v, dow, self._cu, self.scale)
        self._dk_acc, self._dv_acc = torch.from_numpy(dk), torch.from_numpy(dv)
        return torch.from_numpy(dq[q0 - kv0:])

    def add_partials(self, received):
        kv0, q0, _, _ = _window_batch(self)
        dk = self._dk_acc[q0 - kv0:].clone()
        dv = self._dv_acc[q0 - kv0:].clone()
        for lo, hi, dk_p, dv_p in received:
            dk[lo - q0:hi - q0] += dk_p
            dv[lo - q0:hi - q0] += dv_p
        return dk, dv


class OracleHsap(sap_dist.HsapAttention):
    sap_class = OracleSap


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, sap_degree, ulysses_degree, balanced, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        b = workloads.custom_batch(LENS, HQ, HKV, D, seed=5, with_do=True)
        n = b.q.shape[0]
        f64 = [t.double() for t in (b.q, b.k, b.v, b.do)]
        ug = sap_dist.make_hsap_groups(sap_degree, ulysses_degree)
        h = OracleHsap(b.cu_seqlens, n, HQ, HKV, D, sap_degree, ulysses_degree, ulysses_group=ug,
                       balanced=balanced)
        lo, hi = h.block
        q, k, v, do = (t[lo:hi].contiguous() for t in f64)
        o, lse = h.forward(q, k, v)
        dq, dk, dv = h.backward(do)
        out[rank] = {"block": (lo, hi), "o": o.numpy(), "lse": lse.numpy(), "dq": dq.numpy(), "dk": dk.numpy(),
                     "dv": dv.numpy(), "bytes": dict(h.sap.bytes), "bounds": h.sap.bounds.tolist()}
    finally:
        dist.barrier()
        dist.destroy_process_group()


def _run(world, sap_degree, ulysses_degree, balanced=True):
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), sap_degree, ulysses_degree, balanced, out), nprocs=world,
             join=True)
    return dict(out)


@pytest.fixture(scope="module")
def reference():
    b = workloads.custom_batch(LENS, HQ, HKV, D, seed=5, with_do=True)
    scale = 1.0 / math.sqrt(D)
    o, lse = oracle.attn_fwd(b.q, b.k, b.v, b.cu_seqlens, scale)
    dq, dk, dv = oracle.attn_bwd(b.q, b.k, b.v, b.do, b.cu_seqlens, scale)
    return b, {"o": o, "lse": lse, "dq": dq, "dk": dk, "dv": dv}


@pytest.mark.parametrize("world,sap_degree,ulysses_degree,balanced", [
    (2, 2, 1, True),    # SAP, balanced cut
    (4, 4, 1, True),    # SAP, balanced cut
    (4, 4, 1, False),   # SAP, equal chunks
    (2, 1, 2, True),    # head split only (Ulysses)
    (4, 2, 2, True),    # HSAP: Ulysses inside pairs, SAP across them
])
def test_split_equals_unsplit_oracle(reference, world, sap_degree, ulysses_degree, balanced):
    b, ref = reference
    res = _run(world, sap_degree, ulysses_degree, balanced)
    covered = np.zeros(b.q.shape[0], dtype=np.int64)
    hb = HQ // ulysses_degree
    for rank, r in res.items():
        lo, hi = r["block"]
        covered[lo:hi] += 1
        for key in ("o", "dq", "dk", "dv"):
            np.testing.assert_allclose(r[key], ref[key][lo:hi], atol=1e-12, rtol=0, err_msg=f"rank {rank} {key}")
        np.testing.assert_allclose(r["lse"], ref["lse"][:, lo:hi], atol=1e-12, rtol=0)
    assert np.all(covered == 1)
    # key/value bytes that crossed ranks: exactly the planner's spans, per SAP group
    bounds = res[0]["bounds"]
    row = 2 * (HKV // ulysses_degree) * D * 8  # K and V rows, float64 in this test
    plan = sap.sap_plan_chunks(b.cu_seqlens, b.q.shape[0], bounds)
    span_rows = sum(int(h - l) for c in range(sap_degree) for _, l, h in sap.sap_plan_rank_spans(plan, c))
    got = sum(r["bytes"]["kv_received"] for r in res.values())
    sent = sum(r["bytes"]["kv_sent"] for r in res.values())
    assert got == sent == ulysses_degree * span_rows * row
    assert sum(r["bytes"]["dkv_sent"] for r in res.values()) == got
    if sap_degree > 1:
        assert span_rows * row // 2 < sap_dist.ring_bytes(bounds, row // 2)
    del hb
