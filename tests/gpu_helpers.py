"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
and compare with the oracle.

Tolerance: for O, dQ, dK, dV the bound max-abs 2e-2 / mean-abs 2e-3 applies on
top of the half-ulp of the bf16 output format (the kernels round their fp32
results to bf16 once, so an exact result still differs from the fp64 reference
by up to 2^-9 |ref|; 2^-8 leaves room for the fp32 sums), i.e. every element
satisfies
    |out - ref| <= 2e-2 + 2^-8 |ref|
and mean |out - ref| <= 2e-3; for LSE, max-abs 1e-3.

Every comparison also records the plain max-abs and mean-abs error (and the
largest |ref|), so that the distance from the literal max-abs 2e-2 bound is
visible: tests/conftest.py writes the records to the JSON file named by the
SAP_PARITY_REPORT environment variable at the end of the session.
"""
from __future__ import annotations

import math
import os

import numpy as np
import torch

import oracle
import packed_sequence_causal_b200 as sap

ATOL = 2e-2
MEAN_ATOL = 2e-3
LSE_ATOL = 1e-3
BF16_HALF_ULP = 2.0 ** -8

# one record per comparison: test id, tensor, plain max-abs / mean-abs error, max |ref|, elements
PARITY_RECORDS: list = []


def _record(what: str, err: np.ndarray, ref: np.ndarray, **extra):
    rec = {"test": os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0], "what": what,
           "max_abs": float(err.max()) if err.size else 0.0, "mean_abs": float(err.mean()) if err.size else 0.0,
           "max_ref": float(np.abs(ref).max()) if ref.size else 0.0, "elements": int(err.size)}
    rec.update(extra)
    PARITY_RECORDS.append(rec)


def _as_f64(out):
    return out.detach().double().cpu().numpy() if hasattr(out, "detach") else np.asarray(out, dtype=np.float64)


def assert_close(out, ref, what: str, extra_bound=None, mean_extra: float = 0.0):
    """Element bound |out - ref| <= 2e-2 + 2^-8 |ref| (+ extra_bound, an array of the same shape, where a
    test states a larger, derived rounding term) and mean |out - ref| <= 2e-3 (+ mean_extra)."""
    out = _as_f64(out)
    ref = np.asarray(ref, dtype=np.float64)
    assert out.shape == ref.shape, (what, out.shape, ref.shape)
    assert np.all(np.isfinite(out)), f"{what}: non-finite output"
    err = np.abs(out - ref)
    bound = ATOL + BF16_HALF_ULP * np.abs(ref)
    if extra_bound is not None:
        bound = bound + extra_bound
    _record(what, err, ref, **({"max_extra_bound": float(np.max(extra_bound))} if extra_bound is not None else {}))
    excess = err - bound
    worst = int(np.argmax(excess)) if excess.size else 0
    assert excess.size == 0 or excess.max() <= 0, (
        f"{what}: |err| {err.flat[worst]:.4g} at {np.unravel_index(worst, err.shape)} "
        f"(ref {ref.flat[worst]:.4g}, out {out.flat[worst]:.4g}, bound {bound.flat[worst]:.4g})")
    assert err.size == 0 or err.mean() <= MEAN_ATOL + mean_extra, f"{what}: mean |err| {err.mean():.4g}"


def assert_lse(out, ref, what="lse"):
    out = _as_f64(out)
    ref = np.asarray(ref, dtype=np.float64)
    assert np.all(np.isfinite(out)), f"{what}: non-finite"
    err = np.abs(out - ref)
    _record(what, err, ref)
    assert err.size == 0 or err.max() <= LSE_ATOL, f"{what}: max |err| {err.max():.4g}"


def bwd_rounding_bound(q, k, v, do, cu, scale: float, o_ref, lse_ref, k_sigma: float = 6.0):
    """Bound of the backward's rounding error that grows with the logit spread, per element of dQ and
    dK, from the inputs and the oracle's fp64 O and LSE only: k_sigma standard deviations of the
    first-order error model below.

    Each rounding to bf16 (8 significant bits, round to nearest) leaves an error uniform in
    +-2^-9 |x|, standard deviation u|x| with u = 2^-9 / sqrt(3); different roundings are independent.
      * The forward rounds P to bf16 before the PV product and O to bf16 on output, so
        sd(dO_ic) = u sqrt(O_ic^2 + sum_j P_ij^2 V_jc^2).
      * The backward takes D_i = <dO_i, O_i> from that bf16 O (the FlashAttention convention):
        sd(dD_i) = sqrt(sum_c dO_ic^2 sd(dO_ic)^2).  This one error is shared by every key of row i:
        dS_ij = P_ij (dP_ij - D_i) moves by -P_ij dD_i, so dQ_ic moves by -scale dD_i sum_j P_ij K_jc
        and dK_jc by -scale sum_i P_ij dD_i Q_ic (independent over i and over the group's heads).
      * dS is rounded to bf16 before the dQ and dK products: independent errors of sd u |dS_ij|.
    At the default scale (logit standard deviation 1) these terms stay near 1e-3; with a peaky
    softmax (logit spread ~4x) P_ij and |dS_ij| concentrate on few keys and they reach ~1e-2.
    Returns (dq_extra [N,hq,d], dk_extra [N,hkv,d]) as float64 arrays."""
    qd, kd, vd, dod = (torch.as_tensor(oracle.widen(t)[0]) for t in (q, k, v, do))
    o = torch.as_tensor(np.asarray(o_ref, dtype=np.float64))
    lse = torch.as_tensor(np.asarray(lse_ref, dtype=np.float64))
    n, hq, d = qd.shape
    hkv = kd.shape[1]
    G = hq // hkv
    u = 2.0 ** -9 / math.sqrt(3.0)
    var_q = torch.zeros_like(qd)
    var_k = torch.zeros_like(kd)
    for s0, e0 in zip(np.asarray(cu)[:-1].tolist(), np.asarray(cu)[1:].tolist()):
        if e0 <= s0:
            continue
        L = e0 - s0
        causal = torch.tril(torch.ones(L, L, dtype=torch.bool))
        for h in range(hq):
            g = h // G
            Q, K, V, dO, O = qd[s0:e0, h], kd[s0:e0, g], vd[s0:e0, g], dod[s0:e0, h], o[s0:e0, h]
            P = torch.where(causal, torch.exp(scale * (Q @ K.T) - lse[h, s0:e0, None]),
                            torch.zeros((), dtype=torch.float64))
            dS = P * (dO @ V.T - (dO * O).sum(1)[:, None])
            var_o = u * u * (O * O + (P * P) @ (V * V))              # [L, d]
            var_d = (dO * dO * var_o).sum(1)                          # [L]
            var_q[s0:e0, h] += scale ** 2 * (var_d[:, None] * (P @ K) ** 2 + u * u * ((dS * dS) @ (K * K)))
            var_k[s0:e0, g] += scale ** 2 * (((P * P) * var_d[:, None]).T @ (Q * Q) + u * u * ((dS * dS).T @ (Q * Q)))
    return (k_sigma * var_q.sqrt()).numpy(), (k_sigma * var_k.sqrt()).numpy()


class Run:
    """One fwd (+merge) and optionally bwd pass of a batch through the C ABI."""

    def __init__(self, batch, nchunks: int, scale: float | None = None, device="cuda"):
        b = batch
        self.batch = b
        n, hq, d = b.q.shape
        hkv = b.k.shape[1]
        self.n, self.hq, self.hkv, self.d = n, hq, hkv, d
        self.scale = scale if scale is not None else 1.0 / math.sqrt(d)
        self.plan = sap.sap_plan(b.cu_seqlens, n, nchunks)
        self.q, self.k, self.v = (t.to(device).contiguous() for t in (b.q, b.k, b.v))
        self.do = b.do.to(device).contiguous() if b.do is not None else None
        self.o = torch.full((n, hq, d), float("nan"), dtype=torch.bfloat16, device=device)
        self.lse = torch.full((hq, max(n, 1)), float("nan"), dtype=torch.float32, device=device)
        self.ws_fwd = sap.alloc_workspace(self.plan, hq, hkv, d, sap.SAP_WS_FWD, device)

    def fwd(self):
        sap.sap_attn_fwd(self.plan, self.q, self.k, self.v, self.scale, self.o, self.lse, self.ws_fwd)
        sap.sap_merge(self.plan, self.ws_fwd, self.hq, self.d, self.o, self.lse)
        assert sap.sap_device_status() == 0
        return self.o, self.lse[:, : self.n]

    def bwd(self):
        n, hq, hkv, d = self.n, self.hq, self.hkv, self.d
        dev = self.q.device
        self.dq = torch.full((n, hq, d), float("nan"), dtype=torch.bfloat16, device=dev)
        self.dk = torch.full((n, hkv, d), float("nan"), dtype=torch.bfloat16, device=dev)
        self.dv = torch.full((n, hkv, d), float("nan"), dtype=torch.bfloat16, device=dev)
        ws = sap.alloc_workspace(self.plan, hq, hkv, d, sap.SAP_WS_BWD, dev)
        sap.sap_attn_bwd(self.plan, self.q, self.k, self.v, self.o, self.lse, self.do, self.scale, self.dq, self.dk,
                         self.dv, ws)
        assert sap.sap_device_status() == 0
        return self.dq, self.dk, self.dv


def sample_rows(cu, n: int, nchunks: int, k_random: int = 24, seed: int = 0) -> np.ndarray:
    """Rows at document starts/ends, chunk and tile boundaries, plus random rows."""
    rows = set()
    for s, e in zip(cu[:-1], cu[1:]):
        if e > s:
            rows |= {s, min(s + 1, e - 1), e - 1, max(s, e - 2)}
    c = n // nchunks if nchunks > 1 else n
    for b in range(nchunks):
        rows |= {b * c, b * c + 127, b * c + 128}
    rows |= {0, n - 1, 127, 128, 129}
    rng = np.random.default_rng(seed)
    rows |= set(rng.integers(0, n, size=k_random).tolist())
    return np.array(sorted(r for r in rows if 0 <= r < n), dtype=np.int64)


def cheap_kv_rows(cu, rows, d: int, G: int, budget: float = 3e10) -> np.ndarray:
    """The subset of candidate kv rows whose dK/dV the sampled oracle computes within a flop budget."""
    doc_of = np.searchsorted(np.asarray(cu), rows, side="right") - 1
    chosen, need = [], {}
    spent = 0.0
    for j, dk in zip(rows, doc_of):
        s, e = int(cu[dk]), int(cu[dk + 1])
        lo = need.get(dk, e)
        new_lo = min(lo, int(j))
        # stats for rows [new_lo, lo) cost ~ sum (i - s + 1) d G each, plus the row's own sum
        cost = sum_range(new_lo - s + 1, lo - s + 1) * 4.0 * d * G + (e - j) * 4.0 * d * G
        if spent + cost > budget:
            continue
        spent += cost
        need[dk] = new_lo
        chosen.append(int(j))
    return np.array(chosen, dtype=np.int64)


def sum_range(a: int, b: int) -> float:
    """sum of x for x in [a, b)."""
    if b <= a:
        return 0.0
    return (a + b - 1) * (b - a) / 2.0


def doc_sum_identities(dk, dv, do, q, scale: float, cu, hq: int, hkv: int, what: str):
    """Properties that hold at any size: per document and kv head,
    sum_j dK[j] = 0 and sum_j dV[j] = sum over the group's heads and the document's rows of dO.

    Each sum collects one rounding residual per query row (sum_j dS_ij is 0 only
    in exact arithmetic; sum_j P_ij is 1 only in exact arithmetic), so its
    natural scale is that of a random walk over the document's rows and heads:
    sqrt(sum dO^2) for dV and softmax_scale * sqrt(sum Q^2) for dK (per
    element).  Tolerance: 0.1 + 2e-3 * that scale.  Measured deviations of the
    kernel's per-document sums: at most 3e-4 of the dV scale against the full
    oracle on a 16K-token batch with an 8K-token document, and 1.4e-3 of it
    for the 256K-token document of the 512K batch; a dropped near-diagonal
    tile moves a sum by O(1).  The largest fraction of the bound used, per
    tensor, is recorded with the parity records.
    """
    G = hq // hkv
    cu_t = torch.as_tensor(np.asarray(cu, dtype=np.int64), device=dk.device)
    lens = (cu_t[1:] - cu_t[:-1])
    doc_id = torch.repeat_interleave(torch.arange(len(lens), device=dk.device), lens)
    ndoc = len(lens)

    def seg_sum(x):  # x [N, hkv, d] -> [ndoc, hkv, d] in fp64
        out = torch.zeros((ndoc,) + tuple(x.shape[1:]), dtype=torch.float64, device=x.device)
        out.index_add_(0, doc_id, x.double())
        return out

    sk = seg_sum(dk)
    sv = seg_sum(dv)
    dog = do.double().reshape(do.shape[0], hkv, G, do.shape[2])
    ref_v = seg_sum(dog.sum(2))
    scale_v = torch.sqrt(seg_sum((dog ** 2).sum(2)))
    qg = q.double().reshape(q.shape[0], hkv, G, q.shape[2])
    scale_k = scale * torch.sqrt(seg_sum((qg ** 2).sum(2)))
    tol_k = 0.1 + 2e-3 * scale_k
    tol_v = 0.1 + 2e-3 * scale_v
    PARITY_RECORDS.append({"test": os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0], "what": what,
                           "sum_dK_bound_used": float((sk.abs() / tol_k).max().item()),
                           "sum_dV_bound_used": float(((sv - ref_v).abs() / tol_v).max().item()),
                           "sum_dK_max": float(sk.abs().max().item()),
                           "sum_dV_dev_max": float((sv - ref_v).abs().max().item())})
    assert torch.all(sk.abs() <= tol_k), f"{what}: sum dK per doc {sk.abs().max().item():.4g}"
    assert torch.all((sv - ref_v).abs() <= tol_v), f"{what}: sum dV per doc {(sv - ref_v).abs().max().item():.4g}"
