"""Sharded deployments of the layer over torch.distributed (NCCL between GPUs).

The Chord blog serves the layer as expert-parallel shards (EP8/EP16/EP32: each GPU owns a
slice of the experts) and as tensor-parallel shards (TP8: each GPU owns a slice of every
expert's intermediate dimension), and keeps the communication out of its kernel timings
("TL;DR", "Messungen"). This module is the orchestration around the library's exchange
kernels (include/chord.h, "Exchange steps of sharded deployments"):

* ``ChordEPMoE``: dispatch (``chord_ep_plan`` + ``chord_ep_pack``), an all-to-all of the
  send rows to the ranks that own their experts, the layer on every rank, an all-to-all
  back, and ``chord_ep_combine``.
* ``ChordTPMoE``: the layer on this rank's slice with FP32 partial output, an all-reduce,
  and ``chord_round_bf16``.

It holds no arithmetic of the layer: every value the layer computes comes from the
library's kernels; the collectives only move bytes (and sum the FP32 TP partials).
"""
from __future__ import annotations

import numpy as np
import torch
import torch.distributed as dist

from . import chord


def _rows_as_words(t):
    # collectives move rows as 32-bit words (bf16 pairs): every backend supports int32
    return t.contiguous().view(torch.int32)


def ep_exchange(send_x, send_ids, send_w, send_counts, local_forward, group=None):
    """The two all-to-all legs of expert parallelism.

    send_x bf16 [n_send, H] (H even), send_ids int32 [n_send, topk], send_w fp32
    [n_send, topk]: the rows this rank sends, grouped by destination rank; send_counts: W
    ints, the rows for each rank in rank order. Every rank receives the rows addressed to
    it (in source-rank order), computes ``local_forward(x, ids, w)`` -> bf16 [rows, H] on
    them, and sends each output row back to its source. Returns the returned rows bf16
    [n_send, H] in send order.
    """
    W = dist.get_world_size(group)
    assert len(send_counts) == W
    dev = send_x.device
    counts = torch.tensor(send_counts, dtype=torch.int64, device=dev)
    recv_counts = torch.empty_like(counts)
    dist.all_to_all_single(recv_counts, counts, group=group)
    rc = [int(v) for v in recv_counts.tolist()]
    sc = [int(v) for v in send_counts]
    H, k = send_x.shape[1], send_ids.shape[1]
    n_recv = sum(rc)
    recv_x = torch.empty((n_recv, H), dtype=send_x.dtype, device=dev)
    recv_ids = torch.empty((n_recv, k), dtype=torch.int32, device=dev)
    recv_w = torch.empty((n_recv, k), dtype=torch.float32, device=dev)
    dist.all_to_all_single(_rows_as_words(recv_x), _rows_as_words(send_x), rc, sc, group=group)
    dist.all_to_all_single(recv_ids, send_ids.contiguous(), rc, sc, group=group)
    dist.all_to_all_single(recv_w, send_w.contiguous(), rc, sc, group=group)
    out_recv = local_forward(recv_x, recv_ids, recv_w)
    back = torch.empty((sum(sc), H), dtype=send_x.dtype, device=dev)
    dist.all_to_all_single(_rows_as_words(back), _rows_as_words(out_recv), sc, rc, group=group)
    return back


def tp_reduce(partial_f32, group=None):
    """Sum of the ranks' FP32 partial outputs (in place)."""
    dist.all_reduce(partial_f32, op=dist.ReduceOp.SUM, group=group)
    return partial_f32


def tp_shard_weights(qw13, s13, qw2, s2, rank, world):
    """Rank ``rank``'s slice of the intermediate dimension I of every expert: gate rows
    [r*I_r, (r+1)*I_r) and the matching up rows of W13 (kept in gate-then-up order), and
    the same K columns of W2 (packed words K/8, scale groups K/32). I_r = I / world must
    be a multiple of 128 (the layer's shape rule). Host arrays in, host arrays out."""
    E, N13, _ = qw13.shape
    I = N13 // 2
    if I % world or (I // world) % 128:
        raise ValueError(f"intermediate size {I} does not split into {world} slices of a multiple of 128")
    Ir = I // world
    g, u = slice(rank * Ir, (rank + 1) * Ir), slice(I + rank * Ir, I + (rank + 1) * Ir)
    qw13_r = np.ascontiguousarray(np.concatenate([qw13[:, g], qw13[:, u]], axis=1))
    s13_r = np.ascontiguousarray(np.concatenate([s13[:, g], s13[:, u]], axis=1))
    qw2_r = np.ascontiguousarray(qw2[:, :, rank * Ir // 8:(rank + 1) * Ir // 8])
    s2_r = np.ascontiguousarray(s2[:, :, rank * Ir // 32:(rank + 1) * Ir // 32])
    return qw13_r, s13_r, qw2_r, s2_r


class ChordEPMoE:
    """One expert-parallel rank: experts [rank*E_rank, (rank+1)*E_rank) of E_global.

    qw13/s13/qw2/s2 hold this rank's E_rank experts. forward takes this rank's tokens with
    their GLOBAL top-k ids and weights and returns their full layer output. The send
    counts are read back to the host to size the all-to-all, so a forward is not
    capturable in a CUDA graph.
    """

    def __init__(self, qw13, s13, qw2, s2, topk, E_global, group=None, max_tokens=1, device="cuda"):
        self.group = group
        self.W = dist.get_world_size(group)
        self.E_rank = qw13.shape[0]
        if self.E_rank * self.W != E_global:
            raise ValueError(f"{self.W} ranks x {self.E_rank} experts != {E_global}")
        self.topk = topk
        self.layer = chord.ChordMoE(qw13, s13, qw2, s2, topk=topk, E_global=E_global,
                                    max_tokens=max(max_tokens, 1), device=device)
        self.H = self.layer.H
        self.device = self.layer.device

    def _local(self, x, ids, w):
        if x.shape[0] == 0:
            return torch.empty((0, self.H), dtype=torch.bfloat16, device=self.device)
        return self.layer.forward(x, ids, w)

    def forward(self, hidden, topk_ids, topk_weights):
        T, W, k = hidden.shape[0], self.W, self.topk
        d = self.device
        send_rows = torch.empty(max(T * W, 1), dtype=torch.int32, device=d)
        offsets = torch.empty(W + 1, dtype=torch.int32, device=d)
        row_of = torch.empty(max(T * W, 1), dtype=torch.int32, device=d)
        ws = torch.empty(max(chord.chord_ep_plan_workspace_bytes(T, W), 256), dtype=torch.uint8, device=d)
        chord.chord_ep_plan(topk_ids, self.E_rank, W, send_rows, offsets, row_of, ws)
        send_x = torch.empty((max(T * W, 1), self.H), dtype=torch.bfloat16, device=d)
        send_ids = torch.empty((max(T * W, 1), k), dtype=torch.int32, device=d)
        send_w = torch.empty((max(T * W, 1), k), dtype=torch.float32, device=d)
        chord.chord_ep_pack(hidden, topk_ids, topk_weights, self.E_rank, W, send_rows, offsets, row_of,
                            send_x, send_ids, send_w)
        off = offsets.tolist()  # host readback: the all-to-all needs the split sizes
        n = off[W]
        counts = [off[r + 1] - off[r] for r in range(W)]
        back = ep_exchange(send_x[:n], send_ids[:n], send_w[:n], counts, self._local, self.group)
        out = torch.empty((T, self.H), dtype=torch.bfloat16, device=d)
        chord.chord_ep_combine(back, row_of, W, out)
        return out

    __call__ = forward


class ChordTPMoE:
    """One tensor-parallel rank: a slice of every expert's intermediate dimension
    (``tp_shard_weights``). forward runs the layer on the slice with FP32 output, sums the
    ranks' partials (all-reduce) and rounds once to bf16."""

    def __init__(self, qw13_shard, s13_shard, qw2_shard, s2_shard, topk, E_global=None, group=None, max_tokens=1,
                 device="cuda"):
        self.group = group
        self.layer = chord.ChordMoE(qw13_shard, s13_shard, qw2_shard, s2_shard, topk=topk, E_global=E_global,
                                    max_tokens=max(max_tokens, 1), device=device)
        self.H = self.layer.H
        self.device = self.layer.device

    def forward(self, hidden, topk_ids, topk_weights):
        T = hidden.shape[0]
        L = self.layer
        if T > L.max_tokens:
            L.reserve(T)
        partial = torch.empty((T, self.H), dtype=torch.float32, device=self.device)
        L.align(topk_ids)
        chord.chord_moe_forward(hidden, topk_ids, topk_weights, L.sorted_ids, L.expert_ids, L.ntp, L.block_m, L.w13,
                                L.w2, L.I, L.E, partial, L.workspace, chord.CHORD_FLAG_OUTPUT_FP32)
        tp_reduce(partial, self.group)
        out = torch.empty((T, self.H), dtype=torch.bfloat16, device=self.device)
        chord.chord_round_bf16(partial, out)
        return out

    __call__ = forward
