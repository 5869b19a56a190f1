"""Sequence-aware parallelism across devices (SAP) and its hierarchy with a Ulysses head split
(HSAP), one process per GPU over torch.distributed.

HSAP / Sequence-Aware Parallelism page, abstract and method details: a packed batch is cut into
parts, one per device; each device computes the partial attention of its own part, and only the
key/value data of the documents that reach into a part crosses devices, scheduled ahead of time
from the document layout, rather than every chunk passing around a ring.  The hierarchy runs a
Ulysses all-to-all inside a group of devices (afterwards each device holds every token of the
group's part for a subset of the heads: the head split of the explainer page's split-strategy
table) and the sequence-aware exchange across groups.

Data path of one device (rank plan of its chunk, see ``sap_plan_rank`` in include/sap.h):

    forward   [Ulysses all-to-all of Q, K, V]  ->  receive the key/value spans of earlier chunks
              (NCCL point-to-point, exactly the planner's exchange list)  ->  sap_attn_fwd and
              sap_merge  ->  [all-to-all of O and LSE back]
    backward  [all-to-all of dO]  ->  sap_attn_bwd  ->  send the fp32 dK/dV partials of other
              devices' tokens to their owners, add the received ones (sap_attn_bwd_kv_add)  ->
              [all-to-all of dQ, dK, dV back]

Every step of the arithmetic runs in libsap.so's kernels; this module moves tensors and marshals
arguments.  Each transfer lands in this device's own memory before a kernel reads it: no kernel
reads another GPU's memory.  The forward's key/value exchange overlaps the units of the device's
own chunk (they read no received keys); the backward's exchange of partials is not overlapped.
"""
from __future__ import annotations

import math
from typing import List, Optional, Sequence, Tuple

import numpy as np

from . import _capi as sap

Span = Tuple[int, int, int]  # (peer chunk, first token, one past the last token)


# ------------------------------------------------------------------------------ host layout


def chunk_bounds(cu_seqlens, n: int, num_chunks: int, balanced: bool = True, block: int = 128) -> np.ndarray:
    """Chunk bounds of the split: the planner's balanced cut, or equal chunks."""
    if balanced:
        return sap.sap_balanced_chunks(cu_seqlens, n, num_chunks, block)
    if n % num_chunks:
        raise ValueError("equal chunks need N % num_chunks == 0")
    return np.arange(num_chunks + 1, dtype=np.int64) * (n // num_chunks)


def exchange_lists(full_plan, chunk: int) -> Tuple[List[Span], List[Span]]:
    """(recv, send) of the device owning ``chunk``: recv = (source chunk, lo, hi) token ranges of
    earlier chunks it needs; send = (destination chunk, lo, hi) ranges of its own chunk that later
    devices need.  Both come from the planner's per-chunk exchange lists."""
    nc = full_plan.num_chunks
    recv = [tuple(int(x) for x in s) for s in sap.sap_plan_rank_spans(full_plan, chunk)]
    send = []
    for dst in range(chunk + 1, nc):
        for src, lo, hi in sap.sap_plan_rank_spans(full_plan, dst):
            if int(src) == chunk:
                send.append((dst, int(lo), int(hi)))
    return recv, send


def ring_bytes(bounds, row_bytes: int) -> int:
    """Key/value bytes a ring that passes every earlier chunk to every device would move."""
    b = np.asarray(bounds, dtype=np.int64)
    return int(sum(int(b[c]) for c in range(len(b) - 1))) * row_bytes


# ------------------------------------------------------------------------------ exchanges


def exchange_kv(recv: Sequence[Span], send: Sequence[Span], window: dict, k_own, v_own, peers: Sequence[int],
                group=None):
    """Assemble this device's key/value window [kv_begin, q_end) from its own K/V (rows [q_begin,
    q_end)) and the spans received from earlier devices; rows [kv_begin, span_begin) are zeros.
    Returns (k_win, v_win, bytes_sent, bytes_received) once the transfers have completed."""
    k_win, v_win, works, sent, got = start_exchange_kv(recv, send, window, k_own, v_own, peers, group)
    for r in works:
        r.wait()
    return k_win, v_win, sent, got


def start_exchange_kv(recv: Sequence[Span], send: Sequence[Span], window: dict, k_own, v_own,
                      peers: Sequence[int], group=None):
    """exchange_kv without waiting: returns (k_win, v_win, works, bytes_sent, bytes_received); the
    received rows of the window are valid once every work has been waited for (on a CUDA device,
    work.wait() orders the current stream after the transfer)."""
    import torch.distributed as dist
    kv0, q0, q1 = window["kv_begin"], window["q_begin"], window["q_end"]
    shape = (q1 - kv0,) + tuple(k_own.shape[1:])
    k_win = k_own.new_zeros(shape)
    v_win = v_own.new_zeros(shape)
    k_win[q0 - kv0:] = k_own
    v_win[q0 - kv0:] = v_own
    row_bytes = int(k_own[0].numel()) * k_own.element_size() if k_own.shape[0] else 0
    ops, sent, got = [], 0, 0
    for src, lo, hi in recv:  # one span per source; K then V on both sides keeps each pair in order
        ops.append(dist.P2POp(dist.irecv, k_win[lo - kv0:hi - kv0], peers[src], group))
        ops.append(dist.P2POp(dist.irecv, v_win[lo - kv0:hi - kv0], peers[src], group))
        got += 2 * (hi - lo) * row_bytes
    for dst, lo, hi in send:
        ops.append(dist.P2POp(dist.isend, k_own[lo - q0:hi - q0].contiguous(), peers[dst], group))
        ops.append(dist.P2POp(dist.isend, v_own[lo - q0:hi - q0].contiguous(), peers[dst], group))
        sent += 2 * (hi - lo) * row_bytes
    works = dist.batch_isend_irecv(ops) if ops else []
    return k_win, v_win, works, sent, got


def exchange_kv_partials(recv: Sequence[Span], send: Sequence[Span], window: dict, dk_acc, dv_acc,
                         peers: Sequence[int], group=None):
    """Return the partial dK/dV of other devices' tokens to their owners and collect the partials of
    this device's tokens.  dk_acc, dv_acc: [window rows, hkv, d] accumulators (row 0 = kv_begin).
    The partials travel the reverse way of the key/value spans.  Returns (received, bytes_sent)
    with received = [(lo, hi, dk_part, dv_part)] for token ranges of this device's chunk."""
    import torch.distributed as dist
    kv0 = window["kv_begin"]
    row_bytes = int(dk_acc[0].numel()) * dk_acc.element_size() if dk_acc.shape[0] else 0
    ops, received, sent = [], [], 0
    for src, lo, hi in recv:
        ops.append(dist.P2POp(dist.isend, dk_acc[lo - kv0:hi - kv0].contiguous(), peers[src], group))
        ops.append(dist.P2POp(dist.isend, dv_acc[lo - kv0:hi - kv0].contiguous(), peers[src], group))
        sent += 2 * (hi - lo) * row_bytes
    for dst, lo, hi in send:
        dk_p = dk_acc.new_empty((hi - lo,) + tuple(dk_acc.shape[1:]))
        dv_p = dv_acc.new_empty((hi - lo,) + tuple(dv_acc.shape[1:]))
        ops.append(dist.P2POp(dist.irecv, dk_p, peers[dst], group))
        ops.append(dist.P2POp(dist.irecv, dv_p, peers[dst], group))
        received.append((lo, hi, dk_p, dv_p))
    if ops:
        for r in dist.batch_isend_irecv(ops):
            r.wait()
    return received, sent


def heads_from_tokens(x, group, degree: int):
    """Ulysses all-to-all: [L/U, H, ...] token block of this rank -> [L, H/U, ...] (every token of
    the group's part, this rank's head block).  Identity for U = 1."""
    if degree == 1:
        return x
    import torch
    import torch.distributed as dist
    lb, h = x.shape[0], x.shape[1]
    rest = tuple(x.shape[2:])
    xin = x.reshape((lb, degree, h // degree) + rest).transpose(0, 1).contiguous()
    out = torch.empty_like(xin)
    dist.all_to_all_single(out, xin, group=group)
    return out.reshape((degree * lb, h // degree) + rest)


def tokens_from_heads(x, group, degree: int):
    """Inverse of heads_from_tokens: [L, H/U, ...] -> [L/U, H, ...]."""
    if degree == 1:
        return x
    import torch
    import torch.distributed as dist
    L, hu = x.shape[0], x.shape[1]
    rest = tuple(x.shape[2:])
    xin = x.reshape((degree, L // degree, hu) + rest).contiguous()
    out = torch.empty_like(xin)
    dist.all_to_all_single(out, xin, group=group)
    return out.transpose(0, 1).reshape((L // degree, degree * hu) + rest)


def lse_tokens_from_heads(lse, group, degree: int):
    """LSE [H/U, L] (this rank's heads, every token of the part) -> [H, L/U] (its token block)."""
    if degree == 1:
        return lse
    import torch
    import torch.distributed as dist
    hu, L = lse.shape
    xin = lse.reshape(hu, degree, L // degree).transpose(0, 1).contiguous()  # block t' -> rank t'
    out = torch.empty_like(xin)
    dist.all_to_all_single(out, xin, group=group)
    return out.reshape(degree * hu, L // degree)


# ------------------------------------------------------------------------------ one device


class SapAttention:
    """One device's share of sequence-parallel packed causal attention.

    The device owns q chunk ``chunk`` of ``num_chunks`` (balanced or equal cut of the packed batch)
    and holds Q, K, V, dO of that chunk's tokens ([chunk rows, heads, head_dim], bf16, CUDA).
    ``peers[c]`` is the global rank that owns chunk c (default: rank c).  ``forward`` returns
    O [chunk rows, hq, d] and LSE [hq, chunk rows]; ``backward`` returns dQ, dK, dV of the chunk's
    tokens, with the contributions of later devices' queries included."""

    def __init__(self, cu_seqlens, n: int, hq: int, hkv: int, head_dim: int, chunk: int, num_chunks: int, *,
                 peers: Optional[Sequence[int]] = None, group=None, balanced: bool = True,
                 softmax_scale: Optional[float] = None, bounds=None, overlap_sms: int = 8):
        self.cu = np.asarray(cu_seqlens, dtype=np.int32)
        self.n, self.hq, self.hkv, self.d = int(n), int(hq), int(hkv), int(head_dim)
        self.chunk, self.num_chunks = int(chunk), int(num_chunks)
        self.scale = softmax_scale if softmax_scale is not None else 1.0 / math.sqrt(head_dim)
        self.bounds = (np.asarray(bounds, dtype=np.int64) if bounds is not None
                       else chunk_bounds(self.cu, self.n, self.num_chunks, balanced))
        self.full = sap.sap_plan_chunks(self.cu, self.n, self.bounds)
        self.plan = sap.sap_plan_rank(self.full, self.chunk)
        self.window = sap.sap_plan_window(self.plan)
        self.recv, self.send = exchange_lists(self.full, self.chunk)
        self.peers = list(peers) if peers is not None else list(range(self.num_chunks))
        self.group = group
        self.bytes = {"kv_sent": 0, "kv_received": 0, "dkv_sent": 0}
        self._ws_f = self._ws_b = None
        # SMs left free for the transfer kernels while the own-chunk part of the forward runs
        self.overlap_sms = int(overlap_sms)
        import torch.distributed as dist
        if dist.is_available() and dist.is_initialized():
            # point-to-point must not be the first collective of the group with NCCL
            dist.barrier(group=group)

    @property
    def q_rows(self) -> int:
        return self.window["q_end"] - self.window["q_begin"]

    # -- forward
    def forward(self, q, k, v):
        """Post the key/value exchange, run the units of the own chunk while it is in flight (on all
        but overlap_sms SMs), then the units that read received keys, and the merge."""
        k_win, v_win, works, sent, got = start_exchange_kv(self.recv, self.send, self.window, k, v, self.peers,
                                                           self.group)
        self.bytes["kv_sent"], self.bytes["kv_received"] = sent, got
        self.attend(q, k_win, v_win, part=1)
        for r in works:
            r.wait()
        return self.attend(q, k_win, v_win, part=2)

    def attend(self, q, k_win, v_win, part: int = 0):
        """Local partial attention over an assembled key/value window: part 0 all units and the
        merge; part 1 the own-chunk units only (returns None); part 2 the other units and the merge."""
        import torch
        self._q, self._k, self._v = q, k_win, v_win
        if self._ws_f is None:
            sap.sap_plan_upload(self.plan)
            self._ws_f = sap.alloc_workspace(self.plan, self.hq, self.hkv, self.d, sap.SAP_WS_FWD, q.device)
        if part in (0, 1):
            self._o = torch.empty_like(q)
            self._lse = torch.empty((self.hq, max(self.q_rows, 1)), dtype=torch.float32, device=q.device)
        max_ctas = 0
        if part == 1 and self.recv and self.overlap_sms > 0:
            sms = torch.cuda.get_device_properties(q.device).multi_processor_count
            max_ctas = max(1, sms - self.overlap_sms)
        sap.sap_attn_fwd_part(self.plan, part, q, k_win, v_win, self.scale, self._o, self._lse, self._ws_f,
                              max_ctas=max_ctas)
        if part == 1:
            return None
        sap.sap_merge(self.plan, self._ws_f, self.hq, self.d, self._o, self._lse)
        return self._o, self._lse[:, : self.q_rows]

    # -- backward
    def backward(self, do):
        dq = self.local_backward(do)
        received, sent = exchange_kv_partials(self.recv, self.send, self.window, self._dk_acc, self._dv_acc,
                                              self.peers, self.group)
        self.bytes["dkv_sent"] = sent
        dk, dv = self.add_partials(received)
        return dq, dk, dv

    def local_backward(self, do):
        """sap_attn_bwd over the window; leaves the fp32 dK/dV accumulators for the exchange."""
        import torch
        if self._ws_b is None:
            self._ws_b = sap.alloc_workspace(self.plan, self.hq, self.hkv, self.d, sap.SAP_WS_BWD, do.device)
        dq = torch.empty_like(self._q)
        self._dk, self._dv = torch.empty_like(self._k), torch.empty_like(self._v)
        sap.sap_attn_bwd(self.plan, self._q, self._k, self._v, self._o, self._lse, do, self.scale, dq, self._dk,
                         self._dv, self._ws_b)
        rows = self._k.shape[0]
        off_k, off_v = sap.sap_workspace_kv_offsets(self.plan, self.hq, self.hkv, self.d)
        nb = rows * self.hkv * self.d * 4
        self._dk_acc = self._ws_b[off_k:off_k + nb].view(torch.float32).view(rows, self.hkv, self.d)
        self._dv_acc = self._ws_b[off_v:off_v + nb].view(torch.float32).view(rows, self.hkv, self.d)
        return dq

    def add_partials(self, received):
        """Add received fp32 partials of this chunk's tokens; returns the chunk's dK, dV (bf16)."""
        for lo, hi, dk_p, dv_p in received:
            sap.sap_attn_bwd_kv_add(self.plan, self._ws_b, self.hq, dk_p, dv_p, lo, self._dk, self._dv)
        off = self.window["q_begin"] - self.window["kv_begin"]
        return self._dk[off:], self._dv[off:]


# ------------------------------------------------------------------------------ HSAP


def hsap_coords(rank: int, ulysses_degree: int) -> Tuple[int, int]:
    """(sap index s, ulysses index t) of a global rank: Ulysses groups are runs of consecutive ranks
    (the devices of one node share a group), SAP groups take one rank of every Ulysses group."""
    return divmod(rank, ulysses_degree)


def make_hsap_groups(sap_degree: int, ulysses_degree: int):
    """Create every Ulysses group (collectively, same order on all ranks) and return this rank's,
    or None when ulysses_degree == 1."""
    import torch.distributed as dist
    if ulysses_degree == 1:
        return None
    mine = None
    rank = dist.get_rank()
    for s in range(sap_degree):
        ranks = [s * ulysses_degree + t for t in range(ulysses_degree)]
        g = dist.new_group(ranks)
        if rank in ranks:
            mine = g
    return mine


class HsapAttention:
    """Hierarchical sequence-aware parallelism on sap_degree x ulysses_degree devices.

    Rank (s, t) (see hsap_coords) holds token block t of chunk s: tokens
    [bounds[s] + t L_s / U, bounds[s] + (t + 1) L_s / U) with all heads, L_s the chunk's length.
    Inside Ulysses group s an all-to-all gives each rank all L_s tokens for heads block t (hq/U
    query heads, hkv/U key/value heads: GQA groups stay whole); across the SAP group of index t
    the sequence-aware exchange of SapAttention runs on those heads.  sap_degree = 1 is a pure
    head split, ulysses_degree = 1 pure SAP."""

    sap_class = SapAttention

    def __init__(self, cu_seqlens, n: int, hq: int, hkv: int, head_dim: int, sap_degree: int, ulysses_degree: int,
                 *, rank: Optional[int] = None, ulysses_group=None, balanced: bool = True,
                 softmax_scale: Optional[float] = None):
        import torch.distributed as dist
        U, S = int(ulysses_degree), int(sap_degree)
        if hq % U or hkv % U:
            raise ValueError("the Ulysses degree must divide the query and key/value head counts")
        if rank is None:
            rank = dist.get_rank() if dist.is_available() and dist.is_initialized() else 0
        self.rank = int(rank)
        self.s, self.t = hsap_coords(self.rank, U)
        self.U, self.S = U, S
        self.group = ulysses_group
        self.sap = self.sap_class(cu_seqlens, n, hq // U, hkv // U, head_dim, self.s, S,
                                peers=[s * U + self.t for s in range(S)], balanced=balanced,
                                softmax_scale=softmax_scale)
        b = self.sap.bounds
        L = int(b[self.s + 1] - b[self.s])
        if L % U:
            raise ValueError("every chunk length must be a multiple of the Ulysses degree")
        self.block = (int(b[self.s]) + self.t * (L // U), int(b[self.s]) + (self.t + 1) * (L // U))

    def forward(self, q, k, v):
        qh = heads_from_tokens(q, self.group, self.U)
        kh = heads_from_tokens(k, self.group, self.U)
        vh = heads_from_tokens(v, self.group, self.U)
        o, lse = self.sap.forward(qh, kh, vh)
        return tokens_from_heads(o, self.group, self.U), lse_tokens_from_heads(lse.contiguous(), self.group,
                                                                                self.U)

    def backward(self, do):
        dq, dk, dv = self.sap.backward(heads_from_tokens(do, self.group, self.U))
        return (tokens_from_heads(dq, self.group, self.U), tokens_from_heads(dk.contiguous(), self.group, self.U),
                tokens_from_heads(dv.contiguous(), self.group, self.U))
