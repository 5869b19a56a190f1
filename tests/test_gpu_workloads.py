"""CUDA path at the workloads' full sizes, in the launch configuration the
benchmark uses, against the oracle on sampled rows (forward and dQ rows at
document and chunk boundaries plus random rows, dK/dV rows the sampled oracle
can afford) and against per-document sum identities that hold at any size."""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_helpers import Run, assert_close, assert_lse, cheap_kv_rows, doc_sum_identities, sample_rows

pytestmark = pytest.mark.gpu


def _check_workload(name, seed=0, kv_heads=(0,), q_heads_fwd=None, budget=3e10):
    w = workloads.WORKLOADS[name]
    b = workloads.make_batch(name, seed, device="cuda")
    r = Run(b, w.p)
    o, lse = r.fwd()
    cu = b.cu_seqlens
    rows = sample_rows(cu, w.n, w.p, seed=seed)
    ridx = torch.as_tensor(rows, device="cuda")
    G = w.hq // w.hkv
    for g in kv_heads:
        heads = list(range(g * G, (g + 1) * G))
        # slice the group's heads: identical computation with hq' = G, hkv' = 1
        qg = b.q[:, heads].cpu()
        kg = b.k[:, g:g + 1].cpu()
        vg = b.v[:, g:g + 1].cpu()
        ro, rl = oracle.attn_fwd_rows(qg, kg, vg, cu, r.scale, rows, list(range(G)))
        assert_close(o[ridx][:, heads], ro, f"{name} O rows (kv head {g})")
        assert_lse(lse[heads][:, ridx].T, rl, f"{name} LSE rows (kv head {g})")
    if not w.backward:
        return
    dq, dk, dv = r.bwd()
    doc_sum_identities(dk, dv, r.do, r.q, r.scale, cu, w.hq, w.hkv, name)
    for g in kv_heads:
        heads = list(range(g * G, (g + 1) * G))
        arrays = oracle.widen(b.q[:, heads].cpu(), b.k[:, g:g + 1].cpu(), b.v[:, g:g + 1].cpu(),
                              b.do[:, heads].cpu())
        kv_rows = cheap_kv_rows(cu, rows, w.d, G, budget)
        assert len(kv_rows) >= 8
        sq, sk, sv = oracle.attn_bwd_sampled(None, None, None, None, cu, r.scale, 0, rows, kv_rows, arrays=arrays)
        assert_close(dq[ridx][:, heads], sq, f"{name} dQ rows (kv head {g})")
        kidx = torch.as_tensor(kv_rows, device="cuda")
        assert_close(dk[kidx, g], sk, f"{name} dK rows (kv head {g})")
        assert_close(dv[kidx, g], sv, f"{name} dV rows (kv head {g})")


def test_llama32_1b_32k():
    _check_workload("llama32_1b_32k", kv_heads=(0, 7))


def test_llama31_8b_128k():
    _check_workload("llama31_8b_128k", kv_heads=(3,))


def test_llama2_13b_64k_short_docs():
    _check_workload("llama2_13b_64k_short", kv_heads=(0, 39))


def test_hybrid_512k():
    _check_workload("hybrid_512k", kv_heads=(5,), budget=2e10)
